"""GPU parity: the CUDA path against the CPU oracle, element by element, on
the same seeded inputs (gates in tests/gpu_compare.py).

Small cases span several tiles and a ragged tail in every dimension; the
full-size workloads run in the same launch configuration as the benchmark
and are compared on sampled rows and columns the oracle computes one by one
(rows of a linear layer are independent, so the oracle prepares only the
sampled activation rows and weight rows)."""
import os

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


def _dev(t):
    return t.cuda()


def _layer(M, K, N, group, seed, bias=True, zero_rows=()):
    lt = wl.make_random_layer(M, K, N, group, seed, bias=bias)
    if zero_rows:
        x = lt.x.clone()
        x[list(zero_rows)] = 0
        lt.x = x
    return lt


# ---------------------------------------------------------------------------
# step by step
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("group", [64, 256])
@pytest.mark.parametrize("M,K", [(1, 256), (7, 1024), (33, 3072), (5, 12288), (3, 32768),
                                 (1030, 512)])
def test_rotation_matches_oracle(group, M, K):
    x = wl.make_random_layer(M, K, 1, group, seed=M + K).x
    y = cr.convrot_debug_rotate_f32(_dev(x), group)
    torch.cuda.synchronize()
    gc.check_rotation(y.cpu().numpy(), O.rotate(wl.bf16_bits(x), group))


@pytest.mark.parametrize("group", [64, 256])
@pytest.mark.parametrize("M,K", [(1, 256), (9, 1024), (130, 3072), (4, 12288), (2, 32768),
                                 (1100, 768)])
def test_prepare_matches_oracle(group, M, K):
    x = _layer(M, K, 1, group, seed=3 * M + K, zero_rows=(0,) if M > 2 else ()).x
    xb = wl.bf16_bits(x)
    qx, sx = cr.convrot_prepare_act(_dev(x), group)
    torch.cuda.synchronize()
    y = O.rotate(xb, group)
    q_ref, s_ref = O.prepare_rows(xb, group)
    tie = O.tie_band(y, s_ref, gc.TIE_BAND)
    gc.check_prepared(qx.cpu().numpy(), sx.cpu().numpy(), q_ref, s_ref, tie)
    if M > 2:
        assert sx[0].item() == 0.0 and int(qx[0].abs().sum()) == 0


# The three prep kernels give the same codes and scales bit for bit: up to
# 1024 rows (K <= 16384) the 16-channel kernel runs, beyond that the
# 32-channel one (group 256, K <= 3072) or the 64-channel one.  The first
# rows of a long launch must equal the same rows prepared alone.
@pytest.mark.parametrize("K,group", [(1024, 256), (3072, 256), (4096, 256), (8192, 256),
                                     (3072, 64)])
def test_prep_kernels_agree_bit_for_bit(K, group):
    M, head = 2100, 1000
    x = _dev(_layer(M, K, 1, group, seed=K + group).x)
    qx, sx = cr.convrot_prepare_act(x, group)
    qh, sh = cr.convrot_prepare_act(x[:head].contiguous(), group)
    yr = cr.convrot_debug_rotate_f32(x, group)
    yh = cr.convrot_debug_rotate_f32(x[:head].contiguous(), group)
    torch.cuda.synchronize()
    assert torch.equal(qx[:head], qh)
    assert torch.equal(sx[:head].view(torch.int32), sh.view(torch.int32))
    assert torch.equal(yr[:head].view(torch.int32), yh.view(torch.int32))


def test_prepare_edge_rows():
    # exact ties and saturation: absmax 7 after rotation makes inv = 1
    K, group = 256, 256
    rows = []
    # all ones -> rotated all ones -> all codes 7
    rows.append(np.full(K, 0x3F80, dtype=np.uint16))
    # one-hot -> one row of H (entries +-1/16) -> all codes +-7
    e = np.zeros(K, dtype=np.uint16)
    e[3] = 0x4000  # 2.0
    rows.append(e)
    # zeros
    rows.append(np.zeros(K, dtype=np.uint16))
    xb = np.stack(rows)
    x = torch.from_numpy(xb.view(np.int16)).view(torch.bfloat16)
    qx, sx = cr.convrot_prepare_act(_dev(x), group)
    q_ref, s_ref = O.prepare_rows(xb, group)
    assert np.array_equal(qx.cpu().numpy(), q_ref)
    assert np.array_equal(sx.cpu().numpy(), s_ref)
    assert np.all(qx.cpu().numpy()[0] == 0x77)


# Exact ties, no band: rows whose rotation is a known sparse y of exact
# half-integer multiples of a power-of-two scale (tests/tie_rows.py), so the
# fp32 butterflies reproduce y bit for bit and every nonzero code below 7 is
# decided by the round-half-away rule alone.  Up to 1024 rows of K <= 16384
# run the 16-channel prep kernel, longer launches or rows the 64-channel one.
TIE_PREP_CASES = [(40, 1024, 64), (40, 4096, 256), (5, 16384, 256), (1100, 1024, 64),
                  (1100, 2048, 256), (3, 32768, 256), (2, 20480, 64)]


@pytest.mark.parametrize("M,K,group", TIE_PREP_CASES)
def test_exact_ties_bit_exact_without_band(M, K, group):
    from tests.tie_rows import exact_tie_rows
    xb, y, s0, codes = exact_tie_rows(M, K, group, seed=M + K + group)
    x = _dev(torch.from_numpy(xb.view(np.int16)).view(torch.bfloat16))
    q_ref, s_ref = O.prepare_rows(xb, group)
    assert np.array_equal(O.unpack(q_ref, K), codes) and np.array_equal(s_ref, s0)
    yr = cr.convrot_debug_rotate_f32(x, group)
    qx, sx = cr.convrot_prepare_act(x, group)
    qw, sw = cr.convrot_quantize_weight(x, group)
    torch.cuda.synchronize()
    assert np.array_equal(yr.cpu().numpy().astype(np.float64), y)
    for q, s in ((qx, sx), (qw, sw)):
        assert np.array_equal(q.cpu().numpy(), q_ref)
        assert np.array_equal(s.cpu().numpy(), s_ref)


# The whole layer on exact-tie activations and weights: every code is fixed,
# so the outputs must equal the oracle's bit for bit on every path (the
# one-kernel decode form for 1-4 tokens, the few-token GEMM, the tiled GEMM).
@pytest.mark.parametrize("M,K,N,group", [(1, 2048, 300, 64), (2, 4096, 520, 256),
                                         (4, 8192, 136, 64), (16, 1024, 400, 256),
                                         (100, 2048, 264, 64), (300, 1024, 392, 256),
                                         (1100, 1024, 200, 64)])
def test_exact_ties_whole_layer_bit_exact(M, K, N, group):
    from tests.tie_rows import exact_tie_rows
    xb, _, _, _ = exact_tie_rows(M, K, group, seed=3 * M + K)
    wb, _, _, _ = exact_tie_rows(N, K, group, seed=5 * N + K + 1)
    bb = wl.bf16_bits(wl.make_random_layer(1, 64, N, 64, seed=N).b)
    dev = lambda a: _dev(torch.from_numpy(a.view(np.int16)).view(torch.bfloat16))
    qw, sw = cr.convrot_quantize_weight(dev(wb), group)
    y = cr.convrot_linear(dev(xb), qw, sw, dev(bb), group)
    torch.cuda.synchronize()
    assert cr.convrot_check_device_error() == 0
    px, sx = O.prepare_rows(xb, group)
    pw, swr = O.prepare_rows(wb, group)
    y_ref = O.epilogue(O.gemm(px, pw, K), sx, swr, bb)
    assert np.array_equal(gc.to_np_u16(y), y_ref)


@pytest.mark.parametrize("M,N,K", [(1, 16, 64), (5, 72, 192), (16, 128, 1024), (17, 300, 512),
                                   (64, 1000, 768), (100, 256, 256), (128, 384, 1024),
                                   (129, 257, 320), (300, 600, 1536), (513, 96, 128),
                                   (1024, 4096, 128)])
def test_gemm_s32_bit_exact(M, N, K):
    rng = np.random.default_rng(M * 7 + N)
    a = rng.integers(-7, 8, size=(M, K)).astype(np.int8)
    b = rng.integers(-7, 8, size=(N, K)).astype(np.int8)
    if M > 3:
        a[2] = 7
        b[min(3, N - 1)] = -7
    pa, pb = O.pack(a), O.pack(b)
    acc = cr.convrot_debug_gemm_s32(_dev(torch.from_numpy(pa)), _dev(torch.from_numpy(pb)), K)
    torch.cuda.synchronize()
    assert np.array_equal(acc.cpu().numpy().astype(np.int64), O.gemm(pa, pb, K))


# Every token-major tile shape on its own, whatever the automatic choice:
# ragged M, N and K tails, several tiles per CTA (the persistent loop and the
# double-buffered accumulator), and an odd tile count for the CTA pairs.
TILE_SHAPES = [cr.TILES_128x256, cr.TILES_128x192, cr.TILES_256x192_PAIR, cr.TILES_256x128_PAIR]
TILE_IDS = ["128x256", "128x192tmem", "256x192pair", "256x128pair"]
TILE_CASES = [(1, 16, 64), (100, 200, 192), (257, 385, 1088), (384, 576, 2048),
              (1000, 2000, 512), (2304, 3072, 256), (2304, 3072, 3072)]


@pytest.mark.parametrize("tiles", TILE_SHAPES, ids=TILE_IDS)
@pytest.mark.parametrize("M,N,K", TILE_CASES)
def test_gemm_tiles_s32_bit_exact(tiles, M, N, K):
    rng = np.random.default_rng(M * 13 + N + tiles)
    a = rng.integers(-7, 8, size=(M, K)).astype(np.int8)
    b = rng.integers(-7, 8, size=(N, K)).astype(np.int8)
    if M > 3:
        a[2] = 7
        b[min(3, N - 1)] = -7
    pa, pb = O.pack(a), O.pack(b)
    acc = cr.convrot_debug_gemm_tiles(_dev(torch.from_numpy(pa)), None, _dev(torch.from_numpy(pb)),
                                      None, None, K, tiles, out_s32=True)
    torch.cuda.synchronize()
    assert np.array_equal(acc.cpu().numpy().astype(np.int64), O.gemm(pa, pb, K))


# The three few-token forms (M <= 128): token tiles of 16 .. 128 with ragged
# token counts, weight-row slices with a ragged last slice (and, on CTA
# pairs, a last pair with one slice past N), K tails.
SKINNY_FORMS = [cr.SKINNY_TMEM, cr.SKINNY_SMEM, cr.SKINNY_PAIR]
SKINNY_IDS = ["tmem", "smem", "pair"]
SKINNY_CASES = [(1, 16, 64), (1, 14336, 4096), (5, 300, 1088), (16, 1000, 512), (17, 257, 192),
                (33, 4000, 3072), (64, 1024, 1024), (100, 777, 2048), (128, 14336, 256)]


@pytest.mark.parametrize("form", SKINNY_FORMS, ids=SKINNY_IDS)
@pytest.mark.parametrize("M,N,K", SKINNY_CASES)
def test_gemm_skinny_s32_bit_exact(form, M, N, K):
    rng = np.random.default_rng(M * 17 + N + form)
    a = rng.integers(-7, 8, size=(M, K)).astype(np.int8)
    b = rng.integers(-7, 8, size=(N, K)).astype(np.int8)
    a[0] = 7
    b[N - 1] = -7
    pa, pb = O.pack(a), O.pack(b)
    acc = cr.convrot_debug_gemm_tiles(_dev(torch.from_numpy(pa)), None, _dev(torch.from_numpy(pb)),
                                      None, None, K, form, out_s32=True)
    torch.cuda.synchronize()
    assert np.array_equal(acc.cpu().numpy().astype(np.int64), O.gemm(pa, pb, K))


@pytest.mark.parametrize("form", SKINNY_FORMS, ids=SKINNY_IDS)
@pytest.mark.parametrize("M,N,K,bias", [(1, 4096, 1024, True), (16, 1000, 768, False),
                                        (77, 520, 3072, True), (128, 2048, 512, True)])
def test_gemm_skinny_epilogue_one_ulp(form, M, N, K, bias):
    lt = _layer(M, K, N, 64, seed=M + N + form, bias=bias)
    xb, wb = wl.bf16_bits(lt.x), wl.bf16_bits(lt.w)
    bb = None if lt.b is None else wl.bf16_bits(lt.b)
    px, sx = O.prepare_rows(xb, 64)
    pw, sw = O.prepare_rows(wb, 64)
    y_ref = O.epilogue(O.gemm(px, pw, K), sx, sw, bb)
    t = lambda a: _dev(torch.from_numpy(a))
    y = cr.convrot_debug_gemm_tiles(t(px), t(sx), t(pw), t(sw),
                                    None if lt.b is None else _dev(lt.b), K, form)
    torch.cuda.synchronize()
    gc.check_outputs(gc.to_np_u16(y), y_ref)


def test_gemm_skinny_forms_reject_many_tokens():
    q = torch.zeros(129, 64, dtype=torch.uint8, device="cuda")
    for form in SKINNY_FORMS:
        with pytest.raises(cr.ConvRotError):
            cr.convrot_debug_gemm_tiles(q, None, q, None, None, 128, form, out_s32=True)


@pytest.mark.parametrize("tiles", TILE_SHAPES, ids=TILE_IDS)
@pytest.mark.parametrize("M,N,K,bias", [(130, 520, 768, True), (600, 1000, 1024, False),
                                        (1100, 392, 3072, True)])
def test_gemm_tiles_epilogue_one_ulp(tiles, M, N, K, bias):
    lt = _layer(M, K, N, 64, seed=M + N + tiles, bias=bias)
    xb, wb = wl.bf16_bits(lt.x), wl.bf16_bits(lt.w)
    bb = None if lt.b is None else wl.bf16_bits(lt.b)
    px, sx = O.prepare_rows(xb, 64)
    pw, sw = O.prepare_rows(wb, 64)
    y_ref = O.epilogue(O.gemm(px, pw, K), sx, sw, bb)
    t = lambda a: _dev(torch.from_numpy(a))
    y = cr.convrot_debug_gemm_tiles(t(px), t(sx), t(pw), t(sw),
                                    None if lt.b is None else _dev(lt.b), K, tiles)
    torch.cuda.synchronize()
    gc.check_outputs(gc.to_np_u16(y), y_ref)


# acc * s_x * s_w nearly cancels the bias here: rounding the product to fp32
# before adding the bias (the definition) gives bf16 0x33f0, a fused
# multiply-add gives 0x33f3.  Every GEMM form and both store paths (TMA boxes
# for N % 8 == 0, direct stores otherwise) must round twice.
@pytest.mark.parametrize("M,N", [(1, 16), (1, 7), (5, 40), (200, 16), (200, 9), (130, 520)])
def test_epilogue_rounds_product_before_bias(M, N):
    K = 64
    a = np.zeros((M, K), np.int8)
    b = np.zeros((N, K), np.int8)
    a[:, 0], b[:, 0] = 2, 4                                  # acc = 8 everywhere
    pa, pb = O.pack(a), O.pack(b)
    sx = np.full(M, 0.47859192, np.float32)
    sw = np.full(N, 0.008799647, np.float32)
    bias = np.full(N, 0xBD0A, np.uint16)                      # -0.033691406
    y_ref = O.epilogue(O.gemm(pa, pb, K), sx, sw, bias)
    assert np.all(y_ref == 0x33F0)
    t = lambda v: _dev(torch.from_numpy(v))
    bt = t(bias.view(np.int16)).view(torch.bfloat16)
    forms = [cr.TILES_AUTO] + (TILE_SHAPES + [cr.SKINNY_SMEM] if M <= 128 else TILE_SHAPES)
    for form in forms + ([cr.SKINNY_TMEM, cr.SKINNY_PAIR] if M <= 128 else []):
        y = cr.convrot_debug_gemm_tiles(t(pa), t(sx), t(pb), t(sw), bt, K, form)
        torch.cuda.synchronize()
        assert np.array_equal(gc.to_np_u16(y), y_ref), form
    y = cr.convrot_linear_prepared(t(pa), t(sx), t(pb), t(sw), bt, K)
    torch.cuda.synchronize()
    assert np.array_equal(gc.to_np_u16(y), y_ref)


@pytest.mark.parametrize("M,N,K,bias", [(3, 48, 256, True), (40, 200, 1024, False),
                                        (130, 520, 768, True), (300, 13, 256, True)])
def test_linear_prepared_one_ulp(M, N, K, bias):
    lt = _layer(M, K, N, 64, seed=M + N, bias=bias)
    xb, wb = wl.bf16_bits(lt.x), wl.bf16_bits(lt.w)
    bb = None if lt.b is None else wl.bf16_bits(lt.b)
    px, sx = O.prepare_rows(xb, 64)
    pw, sw = O.prepare_rows(wb, 64)
    y_ref = O.epilogue(O.gemm(px, pw, K), sx, sw, bb)
    t = lambda a: _dev(torch.from_numpy(a))
    y = cr.convrot_linear_prepared(t(px), t(sx), t(pw), t(sw), None if lt.b is None else _dev(lt.b), K)
    torch.cuda.synchronize()
    gc.check_outputs(gc.to_np_u16(y), y_ref)


# ---------------------------------------------------------------------------
# the whole layer
# ---------------------------------------------------------------------------

def _full_path_case(lt, group, rows=None, cols=None):
    """Run the GPU path on the whole layer; compare rows x cols with the
    oracle computed from the same seeded bf16 inputs."""
    x, w = _dev(lt.x), _dev(lt.w)
    b = None if lt.b is None else _dev(lt.b)
    qw, sw = cr.convrot_quantize_weight(w, group)
    y = cr.convrot_linear(x, qw, sw, b, group)
    torch.cuda.synchronize()
    assert cr.convrot_check_device_error() == 0
    M, K = lt.x.shape
    N = lt.w.shape[0]
    rows = np.arange(M) if rows is None else np.asarray(rows)
    cols = np.arange(N) if cols is None else np.asarray(cols)
    xb = wl.bf16_bits(lt.x)[rows]
    wb = wl.bf16_bits(lt.w)[cols]
    bb = None if lt.b is None else wl.bf16_bits(lt.b)[cols]
    px, sx = O.prepare_rows(xb, group)
    pw, swr = O.prepare_rows(wb, group)
    tie_x = O.tie_band(O.rotate(xb, group), sx, gc.TIE_BAND)
    tie_w = O.tie_band(O.rotate(wb, group), swr, gc.TIE_BAND)
    gc.check_prepared(qw.cpu().numpy()[cols], sw.cpu().numpy()[cols], pw, swr, tie_w)
    y_ref = O.epilogue(O.gemm(px, pw, K), sx, swr, bb)
    tol = gc.output_tolerance(y_ref, px, pw, sx, swr, tie_x, tie_w)
    gc.check_outputs(gc.to_np_u16(y)[np.ix_(rows, cols)], y_ref, tol)
    return y


@pytest.mark.parametrize("group", [64, 256])
@pytest.mark.parametrize("M,K,N", [(1, 256, 16), (2, 512, 200), (63, 1024, 130), (64, 768, 1024),
                                   (65, 1536, 72), (128, 1024, 256), (129, 512, 600),
                                   (300, 1536, 600), (1000, 256, 40)])
def test_linear_matches_oracle(group, M, K, N):
    lt = _layer(M, K, N, group, seed=M * 31 + N + group, zero_rows=(M // 2,) if M > 4 else ())
    _full_path_case(lt, group)


# The one-kernel path for 1..4 tokens (K a multiple of 2048, M * K <= 16384
# for 4 tokens' worth of preparation threads): against the oracle, and
# bit-identical to the two-kernel path (prep kernel + GEMM) on the same inputs.
DECODE_CASES = [(1, 2048, 1000, 64, True), (1, 4096, 14336, 64, False), (2, 4096, 777, 256, True),
                (3, 4096, 1024, 256, True), (4, 4096, 3000, 64, True), (1, 16384, 520, 256, False),
                (2, 8192, 384, 64, True), (4, 2048, 130, 256, False),
                # token rows prepared in two rounds
                (2, 12288, 600, 64, True), (3, 6144, 1040, 64, False), (2, 14336, 272, 64, True),
                # slices of 33..64 rows (four consumer threads per weight row)
                (2, 4096, 6144, 256, True), (4, 2048, 8000, 64, False)]


@pytest.mark.parametrize("M,K,N,group,bias", DECODE_CASES)
def test_decode_path_matches_oracle(M, K, N, group, bias):
    assert cr.convrot_linear_single_kernel(M, K, group)      # the one-kernel path runs
    lt = _layer(M, K, N, group, seed=M * 7 + K + N, bias=bias, zero_rows=(1,) if M > 2 else ())
    cols = None if N <= 4096 else np.r_[0:300, N - 300:N]
    _full_path_case(lt, group, cols=cols)


@pytest.mark.parametrize("M,K,N,group,bias", DECODE_CASES)
def test_decode_path_equals_two_kernel_path(M, K, N, group, bias):
    lt = _layer(M, K, N, group, seed=M * 11 + K + N, bias=bias)
    x, w = _dev(lt.x), _dev(lt.w)
    b = None if lt.b is None else _dev(lt.b)
    qw, sw = cr.convrot_quantize_weight(w, group)
    y1 = cr.convrot_linear(x, qw, sw, b, group)
    qx, sx = cr.convrot_prepare_act(x, group)
    y2 = cr.convrot_linear_prepared(qx, sx, qw, sw, b, K)
    torch.cuda.synchronize()
    assert cr.convrot_check_device_error() == 0
    assert torch.equal(y1.view(torch.int16), y2.view(torch.int16))


def test_zero_rows_give_exactly_the_bias():
    lt = _layer(140, 512, 96, 256, seed=5, zero_rows=(0, 77, 139))
    y = _full_path_case(lt, 256)
    yb = y.cpu()
    for r in (0, 77, 139):
        assert torch.equal(yb[r], lt.b)


def test_linear_deterministic():
    lt = _layer(700, 2048, 1100, 64, seed=8)
    x, w, b = _dev(lt.x), _dev(lt.w), _dev(lt.b)
    qw, sw = cr.convrot_quantize_weight(w, 64)
    y1 = cr.convrot_linear(x, qw, sw, b, 64)
    y2 = cr.convrot_linear(x, qw, sw, b, 64)
    torch.cuda.synchronize()
    assert torch.equal(y1, y2)


# ---------------------------------------------------------------------------
# full-size workloads, sampled outputs
# ---------------------------------------------------------------------------

def _sample(n, k, seed, block=None):
    """k random indices of n, the first and last, the edges of the first
    128- and 256-blocks, and (block given) one random index in every block of
    that many, so that every output tile of the launch is checked."""
    rng = np.random.default_rng(seed)
    pick = set(rng.choice(n, size=min(n, k), replace=False).tolist())
    pick |= {0, n - 1, min(n - 1, 127), min(n - 1, 128), min(n - 1, 255), min(n - 1, 256)}
    if block:
        for b0 in range(0, n, block):
            pick.add(int(rng.integers(b0, min(n, b0 + block))))
    return np.array(sorted(pick))


@pytest.mark.parametrize("name", ["small_g256", "outlier_g64", "qkv_g256", "square_g256",
                                  "skinny_m1_g64", "skinny_m16_g64", "skinny_m128_g64",
                                  "skinny_m512_g64"])
def test_workload_full_size_sampled(name):
    lt = wl.make_workload(name)[0]
    M, N = lt.x.shape[0], lt.w.shape[0]
    # one row in every 128-token block (the M side of every tile form) and
    # one column in every 64 columns (tiles are 128, 192 or 256 wide, and
    # the few-token form's weight slices are >= 64 rows)
    _full_path_case(lt, lt.spec.group, rows=_sample(M, 48, 1, block=128),
                    cols=_sample(N, 48, 2, block=64))


def test_dit_mlp_pair_full_size_sampled():
    up, down = wl.make_workload("dit_mlp_g256")
    group = 256
    rows = _sample(up.x.shape[0], 32, 3, block=128)
    # up-projection, sampled (every output tile)
    _full_path_case(up, group, rows=rows, cols=_sample(up.w.shape[0], 48, 4, block=64))
    # down-projection: its input rows at the sampled positions are the
    # oracle's own up-projection output; other rows are seeded noise of the
    # same spread.  The GPU runs the full 1536 x 12288 -> 3072 layer.
    xb = wl.bf16_bits(up.x)[rows]
    px, sx = O.prepare_rows(xb, group)
    pw, sw = O.prepare_rows(wl.bf16_bits(up.w), group)
    h_rows = O.epilogue(O.gemm(px, pw, up.spec.K), sx, sw, wl.bf16_bits(up.b))
    g = torch.Generator().manual_seed(11)
    h = (torch.randn(up.x.shape[0], up.w.shape[0], generator=g) * 1.1).to(torch.bfloat16)
    h_np = wl.bf16_bits(h).copy()
    h_np[rows] = h_rows
    down.x = torch.from_numpy(h_np.view(np.int16)).view(torch.bfloat16)
    _full_path_case(down, group, rows=rows, cols=_sample(down.w.shape[0], 48, 5, block=64))


# ---------------------------------------------------------------------------
# failure detection without faulting the GPU
# ---------------------------------------------------------------------------

def test_bounded_wait_reports_timeout_and_context_survives():
    assert cr.convrot_check_device_error() == 0
    cr.convrot_debug_timeout_probe(2_000_000)      # 2 ms, nothing ever arrives
    assert cr.convrot_check_device_error() == 7    # CONVROT_ERR_DEVICE_TIMEOUT
    assert cr.convrot_check_device_error() == 0    # cleared
    lt = _layer(8, 256, 32, 64, seed=1)
    _full_path_case(lt, 64)


def test_bad_arguments_raise():
    x = torch.zeros(4, 1000, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(cr.ConvRotError) as e:
        cr.convrot_prepare_act(x, 64)
    assert e.value.status == 3
    x = torch.zeros(4, 1024, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(cr.ConvRotError) as e:
        cr.convrot_prepare_act(x, 32)
    assert e.value.status == 2
    misaligned = x.view(-1)[1:1025].view(1, 1024)      # starts 2 bytes past a boundary
    with pytest.raises(cr.ConvRotError) as e:
        cr.convrot_debug_rotate_f32(misaligned, 64)
    assert e.value.status == 4


def test_binding_rejects_bad_tensors_before_any_launch():
    """Every entry point checks every tensor (device, dtype, contiguity,
    shape) before a pointer reaches the library; the output buffer stays
    untouched."""
    K, N, M, group = 256, 32, 8, 64
    lt = _layer(M, K, N, group, seed=2)
    x, w, b = _dev(lt.x), _dev(lt.w), _dev(lt.b)
    qw, sw = cr.convrot_quantize_weight(w, group)
    qx, sx = cr.convrot_prepare_act(x, group)
    xr = cr.convrot_w4a16_prepare_act(x, group)
    torch.cuda.synchronize()
    out = torch.full((M, N), 3.0, dtype=torch.bfloat16, device="cuda")
    sentinel = out.clone()
    bad_weights = [dict(qw=qw.cpu()), dict(bias=b[:16]), dict(sw=sw.double()),
                   dict(qw=qw[:, :64].contiguous()), dict(sw=sw[:16]), dict(out=out[:, :16]),
                   dict(out=out.float()), dict(qw=qw.t())]
    calls = {
        "linear": lambda a: cr.convrot_linear(x, a["qw"], a["sw"], a["bias"], group, out=a["out"]),
        "noalloc": lambda a: cr.convrot_linear_noalloc(x, a["qw"], a["sw"], a["bias"], group,
                                                       out=a["out"]),
        "prepared": lambda a: cr.convrot_linear_prepared(qx, sx, a["qw"], a["sw"], a["bias"], K,
                                                         out=a["out"]),
        "tiles": lambda a: cr.convrot_debug_gemm_tiles(qx, sx, a["qw"], a["sw"], a["bias"], K,
                                                       cr.TILES_AUTO, out=a["out"]),
        "w4a16": lambda a: cr.convrot_w4a16_linear(x, a["qw"], a["sw"], a["bias"], group,
                                                   out=a["out"]),
        "w4a16_prepared": lambda a: cr.convrot_w4a16_linear_prepared(xr, a["qw"], a["sw"],
                                                                     a["bias"], out=a["out"]),
    }
    for name, call in calls.items():
        for change in bad_weights:
            a = dict(qw=qw, sw=sw, bias=b, out=out)
            a.update(change)
            with pytest.raises((ValueError, TypeError)):
                call(a)
    with pytest.raises(ValueError):
        cr.convrot_linear(x.cpu(), qw, sw, b, group, out=out)
    with pytest.raises(ValueError):
        cr.convrot_linear_prepared(qx, sx[:4], qw, sw, b, K, out=out)
    with pytest.raises(ValueError):
        cr.convrot_prepare_act(x, group, qx=qx[:4])
    with pytest.raises(ValueError):
        cr.convrot_linear(x, qw, sw, b, group, workspace=torch.empty(16, dtype=torch.uint8,
                                                                    device="cuda"), out=out)
    torch.cuda.synchronize()
    assert torch.equal(out, sentinel)
    assert cr.convrot_check_device_error() == 0


def test_c_abi_rejects_host_pointers_before_any_launch():
    """Below the binding, each entry point looks its pointers up before any
    launch: pinned and pageable host memory give CONVROT_ERR_NOT_DEVICE (10)
    and the output stays untouched."""
    import ctypes
    K, N, M, group = 256, 32, 8, 64
    lt = _layer(M, K, N, group, seed=4)
    x, w, b = _dev(lt.x), _dev(lt.w), _dev(lt.b)
    qw, sw = cr.convrot_quantize_weight(w, group)
    qx, sx = cr.convrot_prepare_act(x, group)
    ws = torch.empty(cr.convrot_linear_workspace_size(M, K), dtype=torch.uint8, device="cuda")
    ws16 = torch.empty(cr.convrot_w4a16_workspace_size(M, K), dtype=torch.uint8, device="cuda")
    out = torch.full((M, N), 3.0, dtype=torch.bfloat16, device="cuda")
    sentinel = out.clone()
    torch.cuda.synchronize()
    pinned = lt.x.pin_memory()
    pageable = np.zeros(M * K, dtype=np.uint16)
    hosts = [ctypes.c_void_p(pinned.data_ptr()), pageable.ctypes.data_as(ctypes.c_void_p)]
    P = lambda t: ctypes.c_void_p(t.data_ptr())
    s = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    L, L16 = cr.lib(), cr.lib_w4a16()
    for h in hosts:
        assert L.convrot_linear(h, P(qw), P(sw), P(b), M, N, K, group, P(ws), ws.numel(), P(out),
                                s) == 10
        assert L.convrot_linear(P(x), P(qw), P(sw), h, M, N, K, group, P(ws), ws.numel(),
                                P(out), s) == 10
        assert L.convrot_linear_noalloc(P(x), h, P(sw), P(b), M, N, K, group, P(out), s) == 10
        assert L.convrot_linear_prepared(P(qx), P(sx), P(qw), h, P(b), M, N, K, P(out), s) == 10
        assert L.convrot_prepare_act(h, M, K, group, P(qx), P(sx), s) == 10
        assert L.convrot_quantize_weight(P(w), N, K, group, h, P(sw), s) == 10
        assert L.convrot_debug_gemm_tiles(P(qx), P(sx), P(qw), P(sw), P(b), M, N, K, 0, 0, h,
                                          s) == 10
        assert L16.convrot_w4a16_linear(h, P(qw), P(sw), P(b), M, N, K, group, P(ws16),
                                        ws16.numel(), P(out), s) == 10
        assert L16.convrot_w4a16_linear_prepared(P(x), P(qw), h, P(b), M, N, K, P(out), s) == 10
    torch.cuda.synchronize()
    assert torch.equal(out, sentinel)
    assert cr.convrot_check_device_error() == 0
    assert L.convrot_status_string(10).startswith(b"CONVROT_ERR_NOT_DEVICE")


# ---------------------------------------------------------------------------
# host-buffer pipeline
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("M,chunks", [(1000, 8), (37, 4), (256, 1)])
def test_host_pipeline_matches_device_call(M, chunks):
    up = _layer(M, 512, 320, 64, seed=M)
    # chain of two layers: 512 -> 320 -> 96
    w1 = _layer(M, 512, 320, 64, seed=M + 2)
    w2 = _layer(M, 320, 96, 64, seed=M + 3)
    qw1, sw1 = cr.convrot_quantize_weight(_dev(w1.w), 64)
    qw2, sw2 = cr.convrot_quantize_weight(_dev(w2.w), 64)
    b1, b2 = _dev(w1.b), _dev(w2.b)
    x = up.x
    ref = cr.convrot_linear(cr.convrot_linear(_dev(x), qw1, sw1, b1, 64), qw2, sw2, b2, 64)
    pipe = cr.HostPipeline(M, 512, [(qw1, sw1, b1, 64), (qw2, sw2, b2, 64)], chunks=chunks)
    y_host = torch.empty(M, 96, dtype=torch.bfloat16).pin_memory()
    pipe(x.pin_memory(), y_host)
    torch.cuda.synchronize()
    assert torch.equal(y_host, ref.cpu())


def test_outlier_layer_quality_rotation_helps():
    """The outlier layer at full size (1024 x 3072 -> 3072, 1% of activation
    channels x50, 0.1% of weights x10): relative Frobenius error of the GPU
    path's bf16 output against the dense product X W^T of the same bf16
    inputs in fp64, for group 64 (the layer's) and group 256, against the
    same rowwise quantiser with no rotation (the oracle's quantiser on the
    unrotated rows).  Rotation spreads the outlier channels before the
    absmax scale is taken, so both rotated errors must be the smaller."""
    lt = wl.make_workload("outlier_g64")[0]
    x, w = _dev(lt.x), _dev(lt.w)
    dense = x.double() @ w.double().T
    nd = torch.linalg.norm(dense).item()
    errs = {}
    for group in (64, 256):
        qw, sw = cr.convrot_quantize_weight(w, group)
        y = cr.convrot_linear(x, qw, sw, None, group)
        torch.cuda.synchronize()
        errs[f"rotated_g{group}"] = torch.linalg.norm(y.double() - dense).item() / nd
    # the same quantiser without rotation, computed by the oracle on the CPU
    qx, sx = O.quantize_rows(O.bf16_to_f64(wl.bf16_bits(lt.x)))
    qwr, swr = O.quantize_rows(O.bf16_to_f64(wl.bf16_bits(lt.w)))
    acc = qx.astype(np.float64) @ qwr.astype(np.float64).T      # exact: |acc| < 2^53
    plain = acc * sx.astype(np.float64)[:, None] * swr.astype(np.float64)[None, :]
    errs["unrotated"] = float(np.linalg.norm(plain - dense.cpu().numpy()) / nd)
    out = os.environ.get("CONVROT_QUALITY_OUT")
    if out:
        with open(out, "w") as f:
            f.write(" ".join(f"{k}={v:.6f}" for k, v in errs.items()) + "\n")
    assert errs["rotated_g64"] < errs["unrotated"]
    assert errs["rotated_g256"] < errs["unrotated"]
