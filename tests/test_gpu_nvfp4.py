"""GPU parity of the NVFP4 variant (include/convrot_nvfp4.h) against the
oracle (oracle_nvfp4_*, pinned in tests/test_oracle_nvfp4.py), through the
C ABI.

Quantisation: on the GPU's own rotated values (the W4A4 library's rotation
hook runs the same fp32 butterflies, so they are the values the NVFP4
kernel quantises) the oracle's decisions must come out bit-exact: codes,
block scales (in the atom layout) and row scales.  Against the oracle's own
fp64 rotation the codes may differ only where a decision lies within 1e-5
of a rounding midpoint.  The product is checked against the exact fp64
GEMM of the same codes and scales within the fp32-accumulation gate of
gpu_compare.check_nvfp4_outputs."""
import numpy as np
import pytest
import torch

import oracle as O
import rotated_w4a4_quantized_b200 as cr
from rotated_w4a4_quantized_b200 import workloads as wl
from tests import gpu_compare as gc

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _built():
    if not torch.cuda.is_available():
        pytest.skip("no GPU")
    from rotated_w4a4_quantized_b200 import build
    build.build()
    O.build()


def _gpu_quant(x, group):
    q, sf, s = cr.convrot_nvfp4_quantize(x, group)
    torch.cuda.synchronize()
    assert cr.convrot_nvfp4_check_device_error() == 0
    return q.cpu().numpy(), sf.cpu().numpy(), s.cpu().numpy()


@pytest.mark.parametrize("group", [64, 256])
@pytest.mark.parametrize("M,K", [(1, 256), (7, 1024), (130, 3072), (3, 16384), (1100, 512)])
def test_quantize_bit_exact_on_the_gpu_rotation(group, M, K):
    lt = wl.make_random_layer(M, K, 1, group, seed=M + K + group)
    x = lt.x.clone()
    if M > 2:
        x[1] = 0                                          # a zero row
        x[2, :64] = 0                                     # zero blocks
    xd = x.cuda()
    q, sf, s = _gpu_quant(xd, group)
    y32 = cr.convrot_debug_rotate_f32(xd, group).cpu().numpy().astype(np.float64)
    codes, sf_ref, s_ref = O.nvfp4_quantize_rows(y32)
    assert np.array_equal(s, s_ref)
    assert np.array_equal(gc.nvfp4_sf_rowmajor(sf, M, K), sf_ref)
    assert np.array_equal(sf, O.nvfp4_sf_layout(sf_ref, K))      # padding rows included
    assert gc.nvfp4_codes_equal(q, O.nvfp4_pack(codes)).all()
    if M > 2:
        assert s[1] == 0 and not (q[1] & 0x77).any()


@pytest.mark.parametrize("group", [64, 256])
def test_quantize_against_the_oracle_rotation(group):
    M, K = 64, 4096
    lt = wl.make_random_layer(M, K, 1, group, seed=11 + group)
    xb = wl.bf16_bits(lt.x)
    q, sf, s = _gpu_quant(lt.x.cuda(), group)
    y64 = O.rotate(xb, group)
    p_ref, sf_ref, s_ref = O.nvfp4_prepare_rows(xb, group)
    assert np.allclose(s, s_ref, rtol=1e-5, atol=0)
    # decisions within 1e-5 of a midpoint may go either way
    a = np.abs(y64).max(axis=1).astype(np.float32)
    rr = np.where(a > 0, np.float32(448) / a, 0).astype(np.float64)
    t = np.abs(y64).reshape(M, K // 16, 16).max(axis=2) * rr[:, None]
    e4 = O.e4m3_value(np.arange(127, dtype=np.uint8))
    mids4 = (e4[1:] + e4[:-1]) / 2
    near4 = np.min(np.abs(t[..., None] - mids4), axis=-1) <= 1e-5 * np.maximum(t, 1e-30)
    sf_gpu = gc.nvfp4_sf_rowmajor(sf, M, K)
    assert np.array_equal(sf_gpu[~near4], sf_ref[~near4])
    d = O.e4m3_value(sf_ref) * s_ref.astype(np.float64)[:, None]
    v = np.abs(y64) / np.repeat(np.where(d > 0, d, np.inf), 16, axis=1)
    e2 = np.array([0, 0.5, 1, 1.5, 2, 3, 4, 6])
    mids2 = (e2[1:] + e2[:-1]) / 2
    near2 = np.min(np.abs(v[..., None] - mids2), axis=-1) <= 1e-5 * np.maximum(v, 1.0)
    ok = gc.nvfp4_codes_equal(q, p_ref) | near2 | np.repeat(near4, 16, axis=1)
    assert ok.all(), np.argwhere(~ok)[:5]


def _prepared_case(M, N, K, group, seed, bias=True):
    """Operands quantised by the oracle (from seeded bf16 rows), uploaded in
    the boundary's layout; the exact product from the oracle."""
    lt = wl.make_random_layer(M, K, N, group, seed=seed, bias=bias)
    xb, wb = wl.bf16_bits(lt.x), wl.bf16_bits(lt.w)
    bb = None if lt.b is None else wl.bf16_bits(lt.b)
    px, sfx, sx = O.nvfp4_prepare_rows(xb, group)
    pw, sfw, sw = O.nvfp4_prepare_rows(wb, group)
    acc, l1, p64 = O.nvfp4_gemm(px, sfx, pw, sfw, K)
    t, _ = O.nvfp4_epilogue(acc, sx, sw, bb)
    dev = lambda a: torch.from_numpy(np.ascontiguousarray(a)).cuda()
    ops = (dev(px), dev(O.nvfp4_sf_layout(sfx, K)), dev(sx), dev(pw), dev(O.nvfp4_sf_layout(sfw, K)),
           dev(sw), None if lt.b is None else lt.b.cuda())
    return ops, (t, acc, l1, p64, sx, sw), lt


GEMM_CASES = [(128, 256, 256), (1, 16, 64), (130, 200, 192), (300, 520, 1024), (64, 1000, 3072),
              (257, 256, 4096), (40, 136, 12288), (600, 1300, 320)]


# Every tile width, forced (128 tokens x 256 or 128 weight rows; K tails
# inside a 256-code stage at K = 64, 192, 320; a last weight tile holding
# one 128-row group of scales or less), and the automatic choice.
@pytest.mark.parametrize("form", [cr.NVFP4_AUTO, cr.NVFP4_TILES_256, cr.NVFP4_TILES_128],
                         ids=["auto", "w256", "w128"])
@pytest.mark.parametrize("M,N,K", GEMM_CASES)
def test_gemm_matches_oracle(form, M, N, K):
    ops, (t, acc, l1, p64, sx, sw), _ = _prepared_case(M, N, K, 64, seed=M * N + K)
    y = cr.convrot_nvfp4_debug_gemm_form(*ops, K, form)
    torch.cuda.synchronize()
    assert cr.convrot_nvfp4_check_device_error() == 0
    share = gc.check_nvfp4_outputs(gc.to_np_u16(y), t, acc, l1, p64, sx, sw)
    assert share > 0.9
    if form == cr.NVFP4_AUTO:     # the public call runs the same kernel
        y2 = cr.convrot_nvfp4_linear_prepared(*ops, K)
        torch.cuda.synchronize()
        assert torch.equal(y.view(torch.int16), y2.view(torch.int16))


def test_gemm_form_hook_refuses_other_forms():
    ops, _, _ = _prepared_case(4, 16, 64, 64, seed=1)
    for form in (3, -1):
        with pytest.raises(cr.ConvRotError) as e:
            cr.convrot_nvfp4_debug_gemm_form(*ops, 64, form)
        assert e.value.status == 3


def test_zero_rows_give_exactly_the_bias():
    M, N, K = 130, 264, 512
    lt = wl.make_random_layer(M, K, N, 64, seed=5)
    x = lt.x.clone()
    x[[0, 77, 129]] = 0
    q, sf, s = cr.convrot_nvfp4_quantize(lt.w.cuda(), 64)
    y = cr.convrot_nvfp4_linear(x.cuda(), q, sf, s, lt.b.cuda(), 64)
    torch.cuda.synchronize()
    for r in (0, 77, 129):
        assert torch.equal(y[r].cpu(), lt.b)


@pytest.mark.parametrize("M,K,N,group", [(1, 1024, 300, 64), (16, 4096, 1000, 256),
                                         (200, 3072, 520, 64), (1100, 1024, 264, 256)])
def test_whole_layer_equals_its_steps_and_the_oracle_gemm(M, K, N, group):
    """convrot_nvfp4_linear == quantize then linear_prepared (bit for bit),
    and the product of the GPU's own operands matches the oracle's exact
    GEMM of those operands within the gate."""
    lt = wl.make_random_layer(M, K, N, group, seed=3 * M + N)
    x, w, b = lt.x.cuda(), lt.w.cuda(), lt.b.cuda()
    qw, sfw, sw = cr.convrot_nvfp4_quantize(w, group)
    y = cr.convrot_nvfp4_linear(x, qw, sfw, sw, b, group)
    qx, sfx, sx = cr.convrot_nvfp4_quantize(x, group)
    y2 = cr.convrot_nvfp4_linear_prepared(qx, sfx, sx, qw, sfw, sw, b, K)
    torch.cuda.synchronize()
    assert cr.convrot_nvfp4_check_device_error() == 0
    assert torch.equal(y.view(torch.int16), y2.view(torch.int16))
    rm = lambda sf_, rows: gc.nvfp4_sf_rowmajor(sf_.cpu().numpy(), rows, K)
    acc, l1, p64 = O.nvfp4_gemm(qx.cpu().numpy(), rm(sfx, M), qw.cpu().numpy(), rm(sfw, N), K)
    t, _ = O.nvfp4_epilogue(acc, sx.cpu().numpy(), sw.cpu().numpy(), wl.bf16_bits(lt.b))
    gc.check_nvfp4_outputs(gc.to_np_u16(y), t, acc, l1, p64, sx.cpu().numpy(), sw.cpu().numpy())


def test_nvfp4_error_below_w4a4_on_the_outlier_layer():
    """Full outlier layer (1024 x 3072 -> 3072, 1% of activation channels x50):
    relative Frobenius error against the dense product of the same bf16
    inputs; the 16-value blocks of NVFP4 beat the one INT4 scale per row."""
    lt = wl.make_workload("outlier_g64")[0]
    x, w = lt.x.cuda(), lt.w.cuda()
    dense = x.double() @ w.double().T
    nd = torch.linalg.norm(dense).item()
    qw, sfw, sw = cr.convrot_nvfp4_quantize(w, 64)
    y4 = cr.convrot_nvfp4_linear(x, qw, sfw, sw, None, 64)
    qi, si = cr.convrot_quantize_weight(w, 64)
    yi = cr.convrot_linear(x, qi, si, None, 64)
    torch.cuda.synchronize()
    e4 = torch.linalg.norm(y4.double() - dense).item() / nd
    ei = torch.linalg.norm(yi.double() - dense).item() / nd
    assert e4 < ei


def test_bad_arguments_raise_before_any_launch():
    M, N, K = 8, 32, 256
    lt = wl.make_random_layer(M, K, N, 64, seed=2)
    x, w = lt.x.cuda(), lt.w.cuda()
    qw, sfw, sw = cr.convrot_nvfp4_quantize(w, 64)
    out = torch.full((M, N), 3.0, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(ValueError):
        cr.convrot_nvfp4_linear(x, qw, sfw[:16], sw, None, 64, out=out)
    with pytest.raises(ValueError):
        cr.convrot_nvfp4_linear(x, qw.cpu(), sfw, sw, None, 64, out=out)
    with pytest.raises(cr.ConvRotError) as e:
        cr.convrot_nvfp4_quantize(torch.zeros(4, 1000, dtype=torch.bfloat16, device="cuda"), 64)
    assert e.value.status == 3
    torch.cuda.synchronize()
    assert torch.all(out == 3.0)
