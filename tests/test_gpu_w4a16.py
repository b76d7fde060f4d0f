"""GPU parity of the W4A16 variant (include/convrot_w4a16.h) against the CPU
oracle, element by element, through the C ABI.

Gates:
  - rotated activations xr (bf16): equal to the oracle's bf16_rne of the
    fp64 rotation, except inside the bf16 tie band (the fp64 value within
    1e-5 x the row's max |y| of a bf16 rounding midpoint), where the GPU's
    fp32 butterflies may round to the neighbouring bf16 value;
  - outputs: within the allowance of gpu_compare.check_w4a16_outputs, derived
    from the arithmetic (tensor-core fp32 accumulation 16 terms at a time,
    the fp32 epilogue, the final bf16 rounding, and the exact effect of
    tie-band inputs).  A misplaced K-block or a wrong code moves outputs by
    tens of bf16 spacings, far outside it.
"""
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


def check_xr(xr_gpu_bits: np.ndarray, y64: np.ndarray) -> np.ndarray:
    """xr against the oracle; returns the tie-band mask."""
    ref = O.round_bf16(y64)
    band = O.bf16_tie_band(y64, gc.ROT_TOL)
    g, r = gc.bf16_f64(xr_gpu_bits), gc.bf16_f64(ref)
    diff = g != r
    outside = diff & ~band
    assert not outside.any(), f"{outside.sum()} rotated values differ outside the tie band, e.g. {np.argwhere(outside)[:5]}"
    sp = gc.bf16_spacing(y64)
    assert np.all(np.abs(g - r)[diff] <= sp[diff] * 1.0001), "a rotated value moved by more than one bf16 step"
    return band


# ---------------------------------------------------------------------------
# step 2: rotation to bf16
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("group", [64, 256])
@pytest.mark.parametrize("M,K", [(1, 256), (7, 1024), (33, 3072), (5, 12288), (3, 32768),
                                 (300, 512), (1030, 768)])
def test_w4a16_rotation_matches_oracle(group, M, K):
    x = wl.make_random_layer(M, K, 1, group, seed=M + 2 * K).x
    if M > 2:
        x = x.clone()
        x[1] = 0
    xr = cr.convrot_w4a16_prepare_act(x.cuda(), group)
    torch.cuda.synchronize()
    assert cr.convrot_w4a16_check_device_error() == 0
    xb = wl.bf16_bits(x)
    check_xr(gc.to_np_u16(xr), O.rotate(xb, group))
    if M > 2:
        assert int(xr[1].view(torch.int16).abs().sum()) == 0


# ---------------------------------------------------------------------------
# step 3: the bf16 x INT4 GEMM with scale and bias
# ---------------------------------------------------------------------------

# token-by-weight tiles (M > 64) and the few-token forms with the weights on
# the MMA's M side (16, 32, 64 token columns), with ragged tails everywhere
GEMM_CASES = [(100, 200, 320, True), (130, 264, 1088, False), (257, 385, 2048, True),
              (300, 1000, 4096, True), (128, 128, 32768, False), (1000, 40, 256, True),
              (256, 256, 128, False), (129, 136, 960, True), (65, 72, 192, False),
              (1, 16, 64, True), (5, 13, 192, False), (16, 14336, 4096, False),
              (17, 130, 1088, True), (32, 300, 2048, False), (33, 257, 320, True),
              (64, 1000, 4096, False), (48, 128, 32768, True)]


@pytest.mark.parametrize("M,N,K,bias", GEMM_CASES)
def test_w4a16_gemm_matches_oracle(M, N, K, bias):
    lt = wl.make_random_layer(M, K, N, 64, seed=5 * M + N + K, bias=bias)
    xb, wb = wl.bf16_bits(lt.x), wl.bf16_bits(lt.w)
    bb = None if lt.b is None else wl.bf16_bits(lt.b)
    pw, sw = O.prepare_rows(wb, 64)            # oracle-prepared weights as the GPU's input
    y = cr.convrot_w4a16_linear_prepared(
        lt.x.cuda(), torch.from_numpy(pw).cuda(), torch.from_numpy(sw).cuda(),
        None if lt.b is None else lt.b.cuda())
    torch.cuda.synchronize()
    assert cr.convrot_w4a16_check_device_error() == 0
    acc, l1, p16 = O.w4a16_gemm(xb, pw, K)
    t, _ = O.w4a16_epilogue(acc, sw, bb)
    gc.check_w4a16_outputs(gc.to_np_u16(y), t, acc, l1, p16, sw)


# The two few-token forms, each forced: weights widened to bf16 in shared
# memory (form 2) or straight into TMEM (form 3), with token counts at and
# around the 16 / 32 / 64 tile widths, slices of weight rows with a ragged
# last slice, K tails inside a 256-code stage (K = 64, 192, 1088) and
# stages whose xr K-blocks lie past K.
FEW_CASES = [(1, 16, 64, True), (1, 14336, 4096, False), (3, 1000, 192, True),
             (16, 777, 1088, False), (17, 300, 2048, True), (32, 4000, 3072, False),
             (33, 130, 320, True), (64, 1024, 4096, True), (50, 9, 12288, False)]


@pytest.mark.parametrize("form", [cr.W4A16_FEW_SMEM, cr.W4A16_FEW_TMEM], ids=["smem", "tmem"])
@pytest.mark.parametrize("M,N,K,bias", FEW_CASES)
def test_w4a16_few_token_forms_match_oracle(form, M, N, K, bias):
    lt = wl.make_random_layer(M, K, N, 64, seed=7 * M + N + K, bias=bias)
    xb, wb = wl.bf16_bits(lt.x), wl.bf16_bits(lt.w)
    bb = None if lt.b is None else wl.bf16_bits(lt.b)
    pw, sw = O.prepare_rows(wb, 64)
    y = cr.convrot_w4a16_debug_gemm_form(
        lt.x.cuda(), torch.from_numpy(pw).cuda(), torch.from_numpy(sw).cuda(),
        None if lt.b is None else lt.b.cuda(), form)
    torch.cuda.synchronize()
    assert cr.convrot_w4a16_check_device_error() == 0
    acc, l1, p16 = O.w4a16_gemm(xb, pw, K)
    t, _ = O.w4a16_epilogue(acc, sw, bb)
    gc.check_w4a16_outputs(gc.to_np_u16(y), t, acc, l1, p16, sw)


def test_w4a16_forms_refuse_what_they_cannot_run():
    lt = wl.make_random_layer(65, 256, 32, 64, seed=3)
    qw, sw = cr.convrot_quantize_weight(lt.w.cuda(), 64)
    for form in (cr.W4A16_FEW_SMEM, cr.W4A16_FEW_TMEM, 4):
        with pytest.raises(cr.ConvRotError) as e:
            cr.convrot_w4a16_debug_gemm_form(lt.x.cuda(), qw, sw, None, form)
        assert e.value.status == 3


def test_w4a16_zero_rows_give_exactly_the_bias():
    M, N, K = 140, 96, 512
    lt = wl.make_random_layer(M, K, N, 64, seed=9)
    x = lt.x.clone()
    x[[0, 77, 139]] = 0
    pw, sw = O.prepare_rows(wl.bf16_bits(lt.w), 64)
    qw_d, sw_d = torch.from_numpy(pw).cuda(), torch.from_numpy(sw).cuda()
    y = cr.convrot_w4a16_linear_prepared(x.cuda(), qw_d, sw_d, lt.b.cuda()).cpu()
    y0 = cr.convrot_w4a16_linear_prepared(x.cuda(), qw_d, sw_d, None).cpu()
    for r in (0, 77, 139):
        assert torch.equal(y[r].view(torch.int16), lt.b.view(torch.int16))
        assert int(y0[r].view(torch.int16).abs().sum()) == 0


# ---------------------------------------------------------------------------
# the whole layer
# ---------------------------------------------------------------------------

def _full_case(lt, group, rows=None, cols=None):
    x, w = lt.x.cuda(), lt.w.cuda()
    b = None if lt.b is None else lt.b.cuda()
    qw, sw = cr.convrot_quantize_weight(w, group)
    y = cr.convrot_w4a16_linear(x, qw, sw, b, group)
    torch.cuda.synchronize()
    assert cr.convrot_w4a16_check_device_error() == 0
    assert cr.convrot_check_device_error() == 0
    M, K = lt.x.shape
    N = lt.w.shape[0]
    rows = np.arange(M) if rows is None else np.asarray(rows)
    cols = np.arange(N) if cols is None else np.asarray(cols)
    xb = wl.bf16_bits(lt.x)[rows]
    wb = wl.bf16_bits(lt.w)[cols]
    bb = None if lt.b is None else wl.bf16_bits(lt.b)[cols]
    y64 = O.rotate(xb, group)
    xr = O.round_bf16(y64)
    band_x = O.bf16_tie_band(y64, gc.ROT_TOL)
    pw, swr = O.prepare_rows(wb, group)
    tie_w = O.tie_band(O.rotate(wb, group), swr, gc.TIE_BAND)
    gc.check_prepared(qw.cpu().numpy()[cols], sw.cpu().numpy()[cols], pw, swr, tie_w)
    acc, l1, p16 = O.w4a16_gemm(xr, pw, K)
    t, _ = O.w4a16_epilogue(acc, swr, bb)
    d_acc = gc.w4a16_input_effect(y64, xr, gc.decode_codes(pw), tie_w, band_x)
    gc.check_w4a16_outputs(gc.to_np_u16(y)[np.ix_(rows, cols)], t, acc, l1, p16, swr,
                           d_acc=d_acc, scale_rtol=gc.SCALE_RTOL)
    return y


@pytest.mark.parametrize("group", [64, 256])
@pytest.mark.parametrize("M,K,N", [(1, 256, 16), (2, 512, 200), (63, 1024, 130), (65, 1536, 72),
                                   (129, 512, 600), (300, 1536, 600), (1000, 256, 40)])
def test_w4a16_linear_matches_oracle(group, M, K, N):
    lt = wl.make_random_layer(M, K, N, group, seed=M * 13 + N + group)
    _full_case(lt, group)


def _sample(n, k, seed):
    rng = np.random.default_rng(seed)
    if n <= k:
        return np.arange(n)
    picks = set(rng.choice(n, size=k - 2, replace=False).tolist()) | {0, n - 1}
    return np.array(sorted(picks))


@pytest.mark.parametrize("name", ["outlier_g64", "qkv_g256", "skinny_m1_g64", "skinny_m16_g64",
                                  "skinny_m128_g64", "square_g256"])
def test_w4a16_workload_full_size_sampled(name):
    """The benchmark's workloads at full size, through the same call the
    benchmark's W4A16 line times, compared on sampled rows and columns."""
    lt = wl.make_workload(name)[0]
    M, K = lt.x.shape
    N = lt.w.shape[0]
    _full_case(lt, lt.spec.group, rows=_sample(M, 12, 1), cols=_sample(N, 160, 2))


def test_w4a16_deterministic():
    lt = wl.make_random_layer(700, 2048, 1100, 64, seed=8)
    x, w, b = lt.x.cuda(), lt.w.cuda(), lt.b.cuda()
    qw, sw = cr.convrot_quantize_weight(w, 64)
    y1 = cr.convrot_w4a16_linear(x, qw, sw, b, 64)
    y2 = cr.convrot_w4a16_linear(x, qw, sw, b, 64)
    torch.cuda.synchronize()
    assert torch.equal(y1.view(torch.int16), y2.view(torch.int16))


def test_w4a16_bad_arguments_raise():
    x = torch.zeros(4, 1024, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(cr.ConvRotError) as e:
        cr.convrot_w4a16_prepare_act(x, 128)
    assert e.value.status == 2
    qw = torch.zeros(8, 48, dtype=torch.uint8, device="cuda")
    sw = torch.ones(8, dtype=torch.float32, device="cuda")
    with pytest.raises(cr.ConvRotError) as e:
        cr.convrot_w4a16_linear_prepared(torch.zeros(4, 96, dtype=torch.bfloat16, device="cuda"),
                                         qw, sw, None)
    assert e.value.status == 3
