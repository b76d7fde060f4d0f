"""Pins for the oracle's NVFP4 functions (CPU only).

The format is not spelled out on the pages (the "convrot-mlx" README, "Why
this repository exists", only says the official ConvRot targets NVFP4 on
Blackwell), so each oracle function is tied to an independent statement of
the same definition:
  - E2M1 and E4M3 rounding against brute-force nearest-value searches over
    values decoded from the bit fields here (not from the oracle's tables),
    and E4M3 against torch's float8_e4m3fn conversion (a library rounding);
  - the quantiser against a numpy restatement of its steps, closed forms
    (all-ones rows, zero rows, the block maximum's code) and its error bound;
  - the block-scale storage layout against its index formula;
  - the GEMM against a numpy fp64 product of the decoded values;
  - the whole layer against a from-scratch brute force on tiny inputs;
  - and the expected ordering of errors: 16-value blocks beat one INT4 scale
    per row on the outlier layer.
"""
import numpy as np
import pytest
import torch

import oracle as O
from rotated_w4a4_quantized_b200 import workloads as wl


def _e2m1_decode(c):
    """Value of an E2M1 code from its bit fields: sign bit 3, exponent bits
    2..1 (bias 1, 0 = subnormal), mantissa bit 0."""
    c = int(c)
    e, m = (c >> 1) & 3, c & 1
    mag = m * 0.5 if e == 0 else (1 + m / 2) * 2.0 ** (e - 1)
    return -mag if c & 8 else mag


def _e4m3_decode(c):
    """Unsigned E4M3: exponent bits 6..3 (bias 7, 0 = subnormal), mantissa 2..0."""
    e, m = (int(c) >> 3) & 15, int(c) & 7
    return m * 2.0 ** -9 if e == 0 else (1 + m / 8) * 2.0 ** (e - 7)


E2M1_ALL = np.array([_e2m1_decode(c) for c in range(8)])
E4M3_ALL = np.array([_e4m3_decode(c) for c in range(127)])


def _nearest_even(a, grid):
    """Index of the grid value nearest to a >= 0; on a tie the even index."""
    d = np.abs(grid - a)
    best = np.flatnonzero(d == d.min())
    even = [i for i in best if i % 2 == 0]
    return int(even[0] if even else best[0])


def test_e2m1_grid_and_rounding_by_search():
    assert list(E2M1_ALL) == [0, 0.5, 1, 1.5, 2, 3, 4, 6]
    assert np.array_equal(O.e2m1_value(np.arange(16, dtype=np.uint8)),
                          [_e2m1_decode(c) for c in range(16)])
    rng = np.random.default_rng(3)
    mids = (E2M1_ALL[1:] + E2M1_ALL[:-1]) / 2
    v = np.concatenate([mids, -mids, np.nextafter(mids.astype(np.float32), 0),
                        np.nextafter(mids.astype(np.float32), 10), rng.uniform(-9, 9, 3000),
                        [0.0, 6.0, 7.0, 100.0, -100.0, 6.99, 7.01, 1e-30, -1e-30]]).astype(np.float32)
    got = O.e2m1_round(v)
    for x, g in zip(v, got):
        want = _nearest_even(min(abs(float(x)), 6.0), E2M1_ALL) | (8 if np.signbit(x) else 0)
        assert g == want, (x, g, want)
    # ties: 0.25 -> 0, 0.75 -> 1, 1.25 -> 1, 2.5 -> 2, 5 -> 4 (even codes); 7 -> 6 (saturation)
    assert O.e2m1_round(np.array([0.25, 0.75, 1.25, 2.5, 5.0, 7.0], np.float32)).tolist() == \
        [0, 2, 2, 4, 6, 7]


def test_e4m3_rounding_by_search_and_against_torch():
    assert E4M3_ALL[126] == 448 and E4M3_ALL[1] == 2.0 ** -9
    assert np.array_equal(O.e4m3_value(np.arange(127, dtype=np.uint8)), E4M3_ALL)
    rng = np.random.default_rng(4)
    mids = (E4M3_ALL[1:] + E4M3_ALL[:-1]) / 2
    v = np.concatenate([mids, np.nextafter(mids.astype(np.float32), 0),
                        np.nextafter(mids.astype(np.float32), 500),
                        np.exp(rng.uniform(-12, 6.1, 3000)), [0.0, 448.0, 440.0]]).astype(np.float32)
    got = O.e4m3_round(v)
    for x, g in zip(v, got):
        assert g == _nearest_even(min(float(x), 448.0), E4M3_ALL), (x, g)
    # torch's float -> float8_e4m3fn conversion rounds to nearest even as well
    lib = torch.from_numpy(v).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(got, lib)
    # past 448 the oracle saturates (satfinite)
    assert O.e4m3_round(np.array([460.0, 1e6], np.float32)).tolist() == [126, 126]


def _quantize_np(y):
    """The quantiser's steps restated in numpy float32 (independent code)."""
    rows, K = y.shape
    codes = np.zeros((rows, K), np.uint8)
    sf = np.zeros((rows, K // 16), np.uint8)
    sc = np.zeros(rows, np.float32)
    for r in range(rows):
        y32 = y[r].astype(np.float32)
        a = np.float32(np.abs(y[r]).max())
        s = a / np.float32(2688) if a > 0 else np.float32(0)
        rr = np.float32(448) / a if a > 0 else np.float32(0)
        sc[r] = s
        for b in range(K // 16):
            blk = y[r, 16 * b:16 * b + 16]
            t = np.float32(np.float32(np.abs(blk).max()) * rr)
            c = _nearest_even(min(float(t), 448.0), E4M3_ALL)
            sf[r, b] = c
            d = np.float32(np.float32(E4M3_ALL[c]) * s)
            inv = np.float32(1) / d if d > 0 else np.float32(0)
            for k in range(16):
                v = np.float32(y32[16 * b + k] * inv)
                codes[r, 16 * b + k] = _nearest_even(min(abs(float(v)), 6.0), E2M1_ALL) | \
                    (8 if np.signbit(v) else 0)
    return codes, sf, sc


def test_quantizer_matches_numpy_restatement():
    rng = np.random.default_rng(5)
    y = np.concatenate([rng.standard_normal((3, 128)) * 2.0 ** rng.integers(-10, 10),
                        rng.standard_cauchy((3, 128)).clip(-1e3, 1e3)])
    y[1, 32:48] = 0.0                                  # a zero block
    y[2, :16] *= 1e-6                                  # a block whose scale is subnormal or 0
    codes, sf, sc = O.nvfp4_quantize_rows(y)
    c2, sf2, sc2 = _quantize_np(y)
    assert np.array_equal(sc, sc2) and np.array_equal(sf, sf2)
    # zero has two encodings (0 and 8); both sides keep the sign of the product
    assert np.array_equal(codes, c2)


def test_quantizer_closed_forms_and_error_bound():
    ones = np.ones((1, 256))
    codes, sf, sc = O.nvfp4_quantize_rows(ones)
    assert np.all(codes == 7) and np.all(sf == 126) and sc[0] == np.float32(1 / 2688)
    # dequantised: 6 x 448 x fp32(1 / 2688) = 1 up to the rounding of the scale
    assert abs(E2M1_ALL[7] * 448.0 * np.float64(sc[0]) - 1.0) <= 2.0 ** -24
    z, zsf, zsc = O.nvfp4_quantize_rows(np.zeros((2, 64)))
    assert np.all(z == 0) and np.all(zsf == 0) and np.all(zsc == 0)
    rng = np.random.default_rng(6)
    y = rng.standard_normal((8, 512)) * np.exp(rng.uniform(-3, 3, (8, 1)))
    codes, sf, sc = O.nvfp4_quantize_rows(y)
    d = O.e4m3_value(sf).repeat(16, axis=1) * sc[:, None].astype(np.float64)
    deq = O.e2m1_value(codes) * d
    # every value within half of the widest E2M1 gap (2 -> 1 unit of d) of y,
    # with a margin for the fp32 steps
    assert np.all(np.abs(deq - y) <= d * (1.0 + 1e-5) + 1e-30)
    # the largest element of a block with a normal scale takes the largest code
    for r in range(8):
        for b in range(512 // 16):
            if E4M3_ALL[sf[r, b]] >= 2.0 ** -6:
                k = 16 * b + int(np.argmax(np.abs(y[r, 16 * b:16 * b + 16])))
                assert codes[r, k] & 7 == 7


def test_sf_layout_by_index_formula():
    rows, K = 200, 192
    sf = np.random.default_rng(7).integers(0, 127, (rows, K // 16)).astype(np.uint8)
    out = O.nvfp4_sf_layout(sf, K)
    assert out.size == 256 * (K // 16)
    for r in range(rows):
        for b in range(K // 16):
            off = ((r // 128) * (K // 64) + b // 4) * 512 + 16 * (r % 32) + 4 * ((r % 128) // 32) + b % 4
            assert out[off] == sf[r, b]
    assert np.count_nonzero(out) == np.count_nonzero(sf)   # padding rows are zero


def test_gemm_equals_numpy_product_of_decoded_values():
    rng = np.random.default_rng(8)
    M, N, K = 5, 7, 192
    cx = rng.integers(0, 16, (M, K)).astype(np.uint8)
    cw = rng.integers(0, 16, (N, K)).astype(np.uint8)
    sfx = rng.integers(0, 127, (M, K // 16)).astype(np.uint8)
    sfw = rng.integers(0, 127, (N, K // 16)).astype(np.uint8)
    acc, l1, _ = O.nvfp4_gemm(O.nvfp4_pack(cx), sfx, O.nvfp4_pack(cw), sfw, K)
    dec = np.vectorize(_e2m1_decode)
    xs = dec(cx) * np.array([[_e4m3_decode(c) for c in row] for row in sfx]).repeat(16, axis=1)
    ws = dec(cw) * np.array([[_e4m3_decode(c) for c in row] for row in sfw]).repeat(16, axis=1)
    assert np.array_equal(acc, xs @ ws.T)               # every partial sum is exact in fp64
    assert np.array_equal(l1, np.abs(xs) @ np.abs(ws).T)


@pytest.mark.parametrize("n", [4, 16])
def test_layer_brute_force_tiny(n):
    """Everything again from scratch: numpy.kron for H, the numpy quantiser,
    decoded fp64 product, epilogue rounded by torch."""
    g = torch.Generator().manual_seed(40 + n)
    x = wl.bf16_bits(torch.randn(4, 64, generator=g).to(torch.bfloat16))
    w = wl.bf16_bits((torch.randn(6, 64, generator=g) * 0.02).to(torch.bfloat16))
    b = wl.bf16_bits((torch.randn(6, generator=g) * 0.02).to(torch.bfloat16))
    T = (np.ones((4, 4)) - 2 * np.eye(4)) / 2
    H = np.ones((1, 1))
    while H.shape[0] < n:
        H = np.kron(H, T)
    R = np.kron(np.eye(64 // n), H)
    f64 = lambda bits: (bits.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    cx, sfx, sx = _quantize_np(f64(x) @ R)
    cw, sfw, sw = _quantize_np(f64(w) @ R)
    dec = np.vectorize(_e2m1_decode)
    dx = dec(cx) * np.vectorize(_e4m3_decode)(sfx).repeat(16, axis=1)
    dw = dec(cw) * np.vectorize(_e4m3_decode)(sfw).repeat(16, axis=1)
    t = (dx @ dw.T) * sx.astype(np.float64)[:, None] * sw.astype(np.float64)[None, :] + f64(b)
    want = wl.bf16_bits(torch.from_numpy(t).to(torch.bfloat16))
    px, osfx, osx = O.nvfp4_prepare_rows(x, n)
    pw, osfw, osw = O.nvfp4_prepare_rows(w, n)
    assert np.array_equal(osfx, sfx) and np.array_equal(osx, sx)
    acc, _, _ = O.nvfp4_gemm(px, osfx, pw, osfw, 64)
    t2, y = O.nvfp4_epilogue(acc, osx, osw, b)
    assert np.allclose(t2, t, rtol=1e-15, atol=0)
    assert np.array_equal(y, want)


def test_nvfp4_error_below_int4_rowwise_on_outlier_layer():
    """Sixteen-value blocks with their own scale follow the spread of the
    rotated values more closely than one INT4 scale per row: the NVFP4 layer
    error is below the W4A4 one on a scaled-down outlier layer."""
    lt = wl.make_random_layer(32, 512, 48, 64, seed=9, bias=False)
    x = lt.x.float()
    ch = torch.randperm(512, generator=torch.Generator().manual_seed(1))[:5]
    x[:, ch] *= 50
    xb, wb = wl.bf16_bits(x.to(torch.bfloat16)), wl.bf16_bits(lt.w)
    f64 = lambda bits: (bits.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    dense = f64(xb) @ f64(wb).T
    px, sfx, sx = O.nvfp4_prepare_rows(xb, 64)
    pw, sfw, sw = O.nvfp4_prepare_rows(wb, 64)
    acc, _, _ = O.nvfp4_gemm(px, sfx, pw, sfw, 512)
    y4 = acc * sx.astype(np.float64)[:, None] * sw.astype(np.float64)[None, :]
    e_fp4 = np.linalg.norm(y4 - dense) / np.linalg.norm(dense)
    qw, sww = O.prepare_rows(wb, 64)
    y_int4 = f64(O.linear_prepared_w(xb, qw, sww, None, 64))
    e_int4 = np.linalg.norm(y_int4 - dense) / np.linalg.norm(dense)
    assert e_fp4 < e_int4


def _emulate_nvfp4_kernel(px, sfx, sx, pw, sfw, sw, bias_bits, K, drop_block=None):
    """The GPU product's arithmetic on the CPU: products of two E2M1 codes
    and two E4M3 scales (exact in fp32), summed in fp32 sixteen at a time,
    each 64-deep step added to an fp32 running sum; then the fp32 epilogue
    ((acc sx) sw + b) and one rounding to bf16 (torch).  drop_block leaves
    out the 16-value block starting at that k."""
    cx = O.e2m1_value(np.stack([px & 0xF, px >> 4], -1).reshape(px.shape[0], -1))
    cw = O.e2m1_value(np.stack([pw & 0xF, pw >> 4], -1).reshape(pw.shape[0], -1))
    xs = (cx * O.e4m3_value(sfx).repeat(16, axis=1)).astype(np.float32)
    ws = (cw * O.e4m3_value(sfw).repeat(16, axis=1)).astype(np.float32)
    M, N = xs.shape[0], ws.shape[0]
    run = np.zeros((M, N), np.float32)
    for k0 in range(0, K, 64):
        step = np.zeros((M, N), np.float32)
        for k in range(k0, k0 + 64):
            if drop_block is not None and drop_block <= k < drop_block + 16:
                continue
            step = step + np.outer(xs[:, k], ws[:, k]).astype(np.float32)
        run = run + step
    y = (run * sx[:, None]).astype(np.float32) * sw[None, :]
    if bias_bits is not None:
        y = y + ((bias_bits.astype(np.uint32) << 16).view(np.float32))[None, :]
    return wl.bf16_bits(torch.from_numpy(y.astype(np.float32)).to(torch.bfloat16))


def test_nvfp4_gate_accepts_the_kernel_arithmetic_and_rejects_a_dropped_block():
    from tests import gpu_compare as gc
    M, N, K = 12, 20, 1024
    lt = wl.make_random_layer(M, K, N, 64, seed=21)
    xb, wb, bb = wl.bf16_bits(lt.x), wl.bf16_bits(lt.w), wl.bf16_bits(lt.b)
    px, sfx, sx = O.nvfp4_prepare_rows(xb, 64)
    pw, sfw, sw = O.nvfp4_prepare_rows(wb, 64)
    acc, l1, p64 = O.nvfp4_gemm(px, sfx, pw, sfw, K)
    t, _ = O.nvfp4_epilogue(acc, sx, sw, bb)
    gc.check_nvfp4_outputs(_emulate_nvfp4_kernel(px, sfx, sx, pw, sfw, sw, bb, K), t, acc, l1,
                           p64, sx, sw)
    for drop in (0, 512, K - 16):
        with pytest.raises(AssertionError):
            gc.check_nvfp4_outputs(_emulate_nvfp4_kernel(px, sfx, sx, pw, sfw, sw, bb, K, drop),
                                   t, acc, l1, p64, sx, sw)


def test_scale_atom_index_maps_agree():
    from tests import gpu_compare as gc
    rows, K = 300, 320
    sf = np.random.default_rng(9).integers(0, 127, (rows, K // 16)).astype(np.uint8)
    assert np.array_equal(gc.nvfp4_sf_rowmajor(O.nvfp4_sf_layout(sf, K), rows, K), sf)
