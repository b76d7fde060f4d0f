"""Pins for the oracle's W4A16 functions (CPU only).

Each check ties the oracle to something other than itself: a brute-force
nearest-value search for the bf16 rounding, closed forms (the all-ones fixed
point of the rotation, one-hot rows giving rows of H), the already pinned
integer GEMM of the W4A4 path, hand-computed epilogue values, and the
expected ordering of quantisation errors.
"""
import numpy as np
import pytest

import oracle as O
from rotated_w4a4_quantized_b200 import workloads as wl
from tests.gpu_compare import decode_codes


def _bits_to_f64(b):
    return (np.asarray(b, dtype=np.uint32) << 16).view(np.float32).astype(np.float64)


def _nearest_bf16_by_search(v: float) -> int:
    """Brute force: look at the bf16 patterns around v's truncated fp32
    pattern and take the nearest, ties to the even pattern."""
    f32 = np.float32(v)
    h0 = int(f32.view(np.uint32)) >> 16
    sign = h0 & 0x8000
    mag0 = h0 & 0x7FFF
    best = None
    for mag in range(max(0, mag0 - 2), min(0x7F7F, mag0 + 2) + 1):
        c = _bits_to_f64(np.array([sign | mag]))[0]
        d = abs(c - v)
        key = (d, mag & 1)
        if best is None or key < best[0]:
            best = (key, sign | mag)
    return best[1]


def test_round_bf16_is_nearest_even_by_search():
    rng = np.random.default_rng(7)
    vals = []
    for e in list(range(-132, -120)) + list(range(-30, 30)) + list(range(120, 127)):
        vals += list(rng.uniform(1, 2, 40) * 2.0 ** e * rng.choice([-1, 1], 40))
    # exact midpoints between neighbouring bf16 values, and values next to them
    for e in (-130, -20, 0, 7, 100):
        for m in range(128, 256, 7):
            mid = (m + 0.5) * 2.0 ** (e - 7)
            vals += [mid, -mid, np.nextafter(mid, 0.0), np.nextafter(mid, np.inf)]
    vals = np.array(vals, dtype=np.float64)
    got = O.round_bf16(vals)
    want = np.array([_nearest_bf16_by_search(v) for v in vals], dtype=np.uint16)
    assert np.array_equal(got, want)


def test_round_bf16_rounds_once():
    # 1 + 2^-8 + 2^-30 lies just above the midpoint of 1 and 1 + 2^-7; a
    # detour through fp32 would land exactly on the midpoint and round to 1.
    v = np.array([1 + 2 ** -8, 1 + 2 ** -8 + 2 ** -30, -(1 + 2 ** -8 + 2 ** -30), 255.5, 0.0])
    assert [int(b) for b in O.round_bf16(v)] == [0x3F80, 0x3F81, 0xBF81, 0x4380, 0x0000]


@pytest.mark.parametrize("group", [64, 256])
def test_rotate_act_fixed_points(group):
    K = 2 * group
    ones = np.full((1, K), 0x3F80, dtype=np.uint16)          # bf16 1.0
    assert np.array_equal(O.w4a16_rotate_act(ones, group), ones)
    H = O.hadamard(group)
    for j in (0, 5, group - 1):
        for p in (-3, 0, 4):
            x = np.zeros((1, K), dtype=np.float64)
            x[0, group + j] = 2.0 ** p
            xb = O.round_bf16(x)
            xr = _bits_to_f64(O.w4a16_rotate_act(xb, group))
            want = np.zeros(K)
            want[group:] = 2.0 ** p * H[j]                      # +-2^p / sqrt(n), exact
            assert np.array_equal(xr[0], want)


def _random_codes(rng, rows, K):
    return rng.integers(-7, 8, size=(rows, K)).astype(np.int8)


def test_gemm_all_ones_is_code_sum():
    rng = np.random.default_rng(3)
    K, N = 192, 11
    q = _random_codes(rng, N, K)
    qw = O.pack(q)
    ones = np.full((3, K), 0x3F80, dtype=np.uint16)
    acc, l1, _ = O.w4a16_gemm(ones, qw, K)
    codes = decode_codes(qw).astype(np.int64)
    assert np.array_equal(acc, np.broadcast_to(codes.sum(axis=1), (3, N)).astype(np.float64))
    assert np.array_equal(l1, np.broadcast_to(np.abs(codes).sum(axis=1), (3, N)).astype(np.float64))


def test_gemm_on_integer_activations_equals_the_integer_gemm():
    rng = np.random.default_rng(4)
    M, N, K = 5, 9, 256
    qx = _random_codes(rng, M, K)
    qw = O.pack(_random_codes(rng, N, K))
    xr = O.round_bf16(qx.astype(np.float64))                  # small integers are exact
    acc, l1, _ = O.w4a16_gemm(xr, qw, K)
    assert np.array_equal(acc, O.gemm(O.pack(qx), qw, K).astype(np.float64))
    assert np.all(np.abs(acc) <= l1)


def test_gemm_l1_equals_acc_for_nonnegative_products():
    rng = np.random.default_rng(5)
    K = 128
    x = np.abs(rng.standard_normal((2, K)))
    qw = O.pack(rng.integers(0, 8, size=(4, K)).astype(np.int8))
    acc, l1, _ = O.w4a16_gemm(O.round_bf16(x), qw, K)
    assert np.array_equal(acc, l1)


@pytest.mark.parametrize("K", [16, 64, 200, 4096])
def test_gemm_prefix_magnitudes_closed_form(K):
    """All products +1: the partial sum after 16 j terms is 16 j (the last
    one K), so p16 = 16 (1 + ... + (n - 1)) + K with n = ceil(K / 16)."""
    ones = np.full((1, K), 0x3F80, dtype=np.uint16)
    qw = O.pack(np.ones((2, K), dtype=np.int8))
    acc, l1, p16 = O.w4a16_gemm(ones, qw, K)
    n = -(-K // 16)
    assert acc[0, 0] == K and l1[0, 0] == K
    assert p16[0, 0] == 16 * (n - 1) * n // 2 + K


def test_epilogue_hand_values():
    acc = np.array([[3.0, -5.0, 0.0, 1000.0]])
    sw = np.array([0.5, 0.25, 2.0, 0.125], dtype=np.float32)
    b = O.round_bf16(np.array([0.25, 1.0, -0.5, 3.0]))
    t, y = O.w4a16_epilogue(acc, sw, b)
    assert np.array_equal(t, [[1.75, -0.25, -0.5, 128.0]])
    assert [int(v) for v in y[0]] == [0x3FE0, 0xBE80, 0xBF00, 0x4300]
    t0, y0 = O.w4a16_epilogue(acc, sw, None)
    assert np.array_equal(t0, [[1.5, -1.25, 0.0, 125.0]])


@pytest.mark.parametrize("group", [64, 256])
def test_linear_on_all_ones_rows(group):
    K, N = 512, 7
    lt = wl.make_random_layer(2, K, N, group, seed=11)
    wb, bb = wl.bf16_bits(lt.w), wl.bf16_bits(lt.b)
    qw, sw = O.prepare_rows(wb, group)
    ones = np.full((2, K), 0x3F80, dtype=np.uint16)
    y = O.w4a16_linear(ones, qw, sw, bb, group)
    codes = decode_codes(qw).astype(np.float64)
    t = codes.sum(axis=1) * sw.astype(np.float64) + _bits_to_f64(bb)
    assert np.array_equal(y, np.broadcast_to(O.round_bf16(t), (2, N)))


def test_w4a16_error_is_below_w4a4_error():
    """Keeping the activations in bf16 removes the activation quantisation
    error, so the W4A16 layer is closer to X W^T than the W4A4 one."""
    lt = wl.make_random_layer(32, 1024, 64, 64, seed=2)
    xb, wb = wl.bf16_bits(lt.x), wl.bf16_bits(lt.w)
    qw, sw = O.prepare_rows(wb, 64)
    ref = _bits_to_f64(xb) @ _bits_to_f64(wb).T
    y16 = _bits_to_f64(O.w4a16_linear(xb, qw, sw, None, 64))
    y4 = _bits_to_f64(O.linear_prepared_w(xb, qw, sw, None, 64))
    e16 = np.linalg.norm(y16 - ref) / np.linalg.norm(ref)
    e4 = np.linalg.norm(y4 - ref) / np.linalg.norm(ref)
    assert e16 < e4


def test_bf16_tie_band_marks_midpoints_only():
    y = np.array([[1 + 2 ** -8, 1 + 2 ** -9, 3.0, 1.5 + 2 ** -8]])
    band = O.bf16_tie_band(y, band=1e-5)
    assert band.tolist() == [[True, False, False, True]]


def test_bf16_tie_band_is_exactly_where_rounding_can_flip():
    """Outside the band, moving a value by up to the band width never changes
    its bf16 rounding; every flip found that way lies inside the band."""
    rng = np.random.default_rng(12)
    y = rng.standard_normal((64, 256)) * np.exp2(rng.integers(-8, 8, size=(64, 1)))
    # plant values right at and next to midpoints
    sp = O.bf16_spacing(y[:, :32])
    y[:, :32] = (np.floor(np.abs(y[:, :32]) / sp) + 0.5) * sp * np.sign(y[:, :32])
    band = 1e-5
    mask = O.bf16_tie_band(y, band)
    eps = band * np.abs(y).max(axis=1, keepdims=True)
    lo, mid, hi = O.round_bf16(y - eps), O.round_bf16(y), O.round_bf16(y + eps)
    flips = (lo != mid) | (hi != mid)
    assert not (flips & ~mask).any()
    assert flips[:, :32].all() and mask[:, :32].all()


def _emulate_w4a16_kernel(xr_bits, packed_w, sw, bias_bits, K, drop_block=None, block=64):
    """The GPU GEMM's arithmetic written out on the CPU: products of bf16
    activations and integer codes (exact in fp32), summed in fp32 sixteen at
    a time (one tensor-core K step), each partial added to an fp32 running
    sum; then the fp32 epilogue acc * sw + b and one rounding to bf16 (by
    torch).  drop_block leaves out the K-block starting at that index."""
    import torch
    xf = _bits_to_f64(xr_bits).astype(np.float32)
    q = decode_codes(packed_w).astype(np.float32)
    M, N = xf.shape[0], q.shape[0]
    run = np.zeros((M, N), dtype=np.float32)
    for k0 in range(0, K, 16):
        if drop_block is not None and drop_block <= k0 < drop_block + block:
            continue
        part = np.zeros((M, N), dtype=np.float32)
        for k in range(k0, k0 + 16):
            part = part + np.outer(xf[:, k], q[:, k]).astype(np.float32)
        run = run + part
    y = run * np.asarray(sw, np.float32)[None, :]
    if bias_bits is not None:
        y = y + _bits_to_f64(bias_bits).astype(np.float32)[None, :]
    return wl.bf16_bits(torch.from_numpy(y.astype(np.float32)).to(torch.bfloat16))


@pytest.mark.parametrize("K,group", [(1024, 64), (4096, 256)])
def test_w4a16_gate_accepts_the_kernel_arithmetic_and_rejects_a_dropped_block(K, group):
    """The W4A16 output gate (check_w4a16_outputs) is a tolerance, not an
    equality, so it is pinned from both sides: an emulation of the kernel's
    fp32 tensor-core accumulation passes it, and the same emulation with one
    64-deep K-block left out fails it."""
    from tests import gpu_compare as gc
    lt = wl.make_random_layer(20, K, 36, group, seed=K + group)
    xb, wb, bb = wl.bf16_bits(lt.x), wl.bf16_bits(lt.w), wl.bf16_bits(lt.b)
    xr = O.w4a16_rotate_act(xb, group)
    pw, sw = O.prepare_rows(wb, group)
    acc, l1, p16 = O.w4a16_gemm(xr, pw, K)
    t, _ = O.w4a16_epilogue(acc, sw, bb)
    gc.check_w4a16_outputs(_emulate_w4a16_kernel(xr, pw, sw, bb, K), t, acc, l1, p16, sw)
    for drop in (0, K // 2, K - 64):
        with pytest.raises(AssertionError):
            gc.check_w4a16_outputs(_emulate_w4a16_kernel(xr, pw, sw, bb, K, drop_block=drop),
                                   t, acc, l1, p16, sw)
