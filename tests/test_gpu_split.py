"""Split K on the GPU: the token-major GEMM with tiles cut into ranges of K.

The split changes only how the integer product is scheduled (no counterpart
on the pages; the product itself is "convrot-mlx" README, "Install and
test").  Integer addition is exact, so every split plan must give the
oracle's accumulators bit for bit, and the bf16 outputs of a split run must
equal the unsplit run's bit for bit:
- forced plans on every token-major tile shape, with ragged M, N and K
  (parts of one K-stage, uneven parts, one split tile among whole ones,
  every tile split);
- the planner's own choice;
- the whole layer with and without the split area in its workspace, on
  layers the planner splits on a B200 and on layers it leaves whole;
- the split counters are zero again after every call, so one area serves
  call after call."""
import numpy as np
import pytest
import torch

import oracle as O
import rotated_w4a4_quantized_b200 as cr
from rotated_w4a4_quantized_b200 import workloads as wl

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _built():
    if not torch.cuda.is_available():
        pytest.skip("no GPU")
    from rotated_w4a4_quantized_b200 import build
    build.build()
    O.build()


# tile shape: (form, rows of A per tile, BN, packed bytes per K-stage, CTAs per tile)
FORMS = {
    "128x256": (cr.TILES_128x256, 128, 256, 64, 1),
    "128x192tmem": (cr.TILES_128x192, 128, 192, 128, 1),
    "256x192pair": (cr.TILES_256x192_PAIR, 256, 192, 128, 2),
    "256x128pair": (cr.TILES_256x128_PAIR, 256, 128, 128, 2),
}
CASES = [(257, 385, 1088), (300, 600, 3136), (1000, 2000, 512), (129, 130, 64)]
COUNTER_WORDS = cr.SPLIT_COUNTER_BYTES // 4


def _plans(M, N, K, tm, bn, pkb, cg):
    """(name, split_tiles, splits) that fit the area for this shape."""
    tiles = -(-M // tm) * -(-N // bn)
    stages = -(-(K // 2) // pkb)
    slots = (cr.SPLIT_AREA_BYTES - cr.SPLIT_COUNTER_BYTES) // (128 * bn * 4)
    fits = lambda t, s: 2 <= s <= stages and t * s * cg <= slots and t * cg * 8 <= COUNTER_WORDS
    plans = [("none", 0, 1), ("planner", -1, 1)]
    if fits(tiles, 2):
        plans.append(("all2", tiles, 2))
    smax = min(stages, slots // (tiles * cg))
    if smax > 2 and fits(tiles, smax):
        plans.append((f"all{smax}", tiles, smax))     # parts of one or two K-stages
    if fits(1, min(3, stages)):
        plans.append(("one", 1, min(3, stages)))      # one split tile among whole ones
    return plans


def _operands(M, N, K, seed):
    rng = np.random.default_rng(seed)
    a = rng.integers(-7, 8, size=(M, K)).astype(np.int8)
    b = rng.integers(-7, 8, size=(N, K)).astype(np.int8)
    a[0] = 7
    b[N - 1] = -7
    return O.pack(a), O.pack(b)


@pytest.mark.parametrize("form", list(FORMS), ids=list(FORMS))
@pytest.mark.parametrize("M,N,K", CASES)
def test_split_s32_bit_exact(form, M, N, K):
    tiles, tm, bn, pkb, cg = FORMS[form]
    pa, pb = _operands(M, N, K, M * 31 + N + tiles)
    qx, qw = torch.from_numpy(pa).cuda(), torch.from_numpy(pb).cuda()
    ref = O.gemm(pa, pb, K)
    area = cr.new_split_area(qx.device)
    for name, st, sp in _plans(M, N, K, tm, bn, pkb, cg):
        acc = cr.convrot_debug_gemm_split(qx, None, qw, None, None, K, tiles, st, sp, area,
                                          out_s32=True)
        torch.cuda.synchronize()
        assert cr.convrot_check_device_error() == 0
        assert np.array_equal(acc.cpu().numpy().astype(np.int64), ref), name
        assert not area[:cr.SPLIT_COUNTER_BYTES].any(), f"{name}: counters left non-zero"


@pytest.mark.parametrize("form", list(FORMS), ids=list(FORMS))
def test_split_bf16_equals_unsplit(form):
    tiles, tm, bn, pkb, cg = FORMS[form]
    M, N, K = 700, 1000, 2048
    lt = wl.make_random_layer(M, K, N, 64, seed=11 + tiles)
    x, w, b = lt.x.cuda(), lt.w.cuda(), lt.b.cuda()
    qw, sw = cr.convrot_quantize_weight(w, 64)
    qx, sx = cr.convrot_prepare_act(x, 64)
    whole = cr.convrot_debug_gemm_tiles(qx, sx, qw, sw, b, K, tiles)
    area = cr.new_split_area(x.device)
    for name, st, sp in _plans(M, N, K, tm, bn, pkb, cg):
        y = cr.convrot_debug_gemm_split(qx, sx, qw, sw, b, K, tiles, st, sp, area)
        torch.cuda.synchronize()
        assert torch.equal(y.view(torch.int16), whole.view(torch.int16)), name


def test_plans_that_do_not_fit_are_refused():
    M, N, K = 300, 600, 64                            # one K-stage per tile
    pa, pb = _operands(M, N, K, 5)
    qx, qw = torch.from_numpy(pa).cuda(), torch.from_numpy(pb).cuda()
    area = cr.new_split_area(qx.device)
    for st, sp in [(1, 2), (100, 2)]:                 # more parts than stages; more tiles than exist
        with pytest.raises(cr.ConvRotError) as e:
            cr.convrot_debug_gemm_split(qx, None, qw, None, None, K, cr.TILES_256x192_PAIR, st, sp,
                                        area, out_s32=True)
        assert e.value.status == 3
    M, N, K = 2048, 8192, 4096                        # 16 x 32 tiles of 128 x 256
    pa, pb = _operands(M, N, K, 6)
    qx, qw = torch.from_numpy(pa).cuda(), torch.from_numpy(pb).cuda()
    with pytest.raises(cr.ConvRotError) as e:        # 256 tiles x 2 parts > the area's 160 slots
        cr.convrot_debug_gemm_split(qx, None, qw, None, None, K, cr.TILES_128x256, 256, 2, area,
                                    out_s32=True)
    assert e.value.status == 3


# (M, K, N, group, split on a B200 with 74 CTA pairs): the DiT MLP down
# projection (96 tiles of 256 x 192, 48 K-stages each: the last wave's 22
# tiles in 3 parts), the 512-token layer (150 tiles: 2 in 4 parts), a
# 1024-token layer (108 tiles of 32 stages: 34 in 2 parts); left whole: the
# up projection (12-stage tiles, where the split costs what it saves) and a
# layer of 16 tiles, less than one wave.
LAYER_CASES = [(1536, 12288, 3072, 256, True), (512, 4096, 14336, 64, True),
               (1024, 8192, 5120, 64, True), (1536, 3072, 12288, 256, False),
               (300, 1024, 1000, 64, False)]


@pytest.mark.parametrize("M,K,N,group,splits", LAYER_CASES)
def test_whole_layer_split_equals_unsplit(M, K, N, group, splits):
    lt = wl.make_random_layer(M, K, N, group, seed=M + N)
    x, w, b = lt.x.cuda(), lt.w.cuda(), lt.b.cuda()
    qw, sw = cr.convrot_quantize_weight(w, group)
    need = cr.convrot_linear_workspace_size(M, K)
    base = need - cr.SPLIT_AREA_BYTES
    full = torch.full((need,), 0xAB, dtype=torch.uint8, device=x.device)   # counters not zeroed
    short = torch.empty(base, dtype=torch.uint8, device=x.device)
    y_split = cr.convrot_linear(x, qw, sw, b, group, full)
    y_whole = cr.convrot_linear(x, qw, sw, b, group, short)
    torch.cuda.synchronize()
    assert cr.convrot_check_device_error() == 0
    assert torch.equal(y_split.view(torch.int16), y_whole.view(torch.int16))
    # the prep kernel cleared the counters and the GEMM left them clear;
    # partial sums were written exactly where the planner splits
    assert not full[base:base + cr.SPLIT_COUNTER_BYTES].any()
    slots = full[base + cr.SPLIT_COUNTER_BYTES:base + cr.SPLIT_COUNTER_BYTES + 4096]
    if torch.cuda.get_device_properties(x.device).multi_processor_count == 148:
        assert bool((slots != 0xAB).any()) == splits
    # a second call on the same workspace
    y2 = cr.convrot_linear(x, qw, sw, b, group, full)
    torch.cuda.synchronize()
    assert torch.equal(y2.view(torch.int16), y_whole.view(torch.int16))


def test_prepared_split_area_serves_calls_in_a_row():
    area = cr.new_split_area(torch.device("cuda"))
    for (M, K, N, group, seed) in [(1536, 12288, 3072, 256, 1), (512, 4096, 2048, 64, 2),
                                   (1024, 3072, 3072, 64, 3)]:
        lt = wl.make_random_layer(M, K, N, group, seed=seed)
        x, w, b = lt.x.cuda(), lt.w.cuda(), lt.b.cuda()
        qw, sw = cr.convrot_quantize_weight(w, group)
        qx, sx = cr.convrot_prepare_act(x, group)
        y = cr.convrot_linear_prepared_split(qx, sx, qw, sw, b, K, area)
        y_ref = cr.convrot_linear_prepared(qx, sx, qw, sw, b, K)
        torch.cuda.synchronize()
        assert torch.equal(y.view(torch.int16), y_ref.view(torch.int16)), (M, K, N)
        assert not area[:cr.SPLIT_COUNTER_BYTES].any()


def test_split_on_repacked_weights():
    """Forced plans and the whole layer on repacked weights (the block-major
    layout of include/convrot.h) against the canonical unsplit product."""
    M, N, K = 1000, 2000, 3136
    lt = wl.make_random_layer(M, K, N, 64, seed=31)
    x, w, b = lt.x.cuda(), lt.w.cuda(), lt.b.cuda()
    qw, sw = cr.convrot_quantize_weight(w, 64)
    rep = cr.convrot_repack_weight(qw)
    qx, sx = cr.convrot_prepare_act(x, 64)
    area = cr.new_split_area(x.device)
    for tiles in (cr.TILES_256x192_PAIR, cr.TILES_128x192):
        whole = cr.convrot_debug_gemm_tiles(qx, sx, qw, sw, b, K, tiles)
        acc = cr.convrot_debug_gemm_tiles(qx, None, qw, None, None, K, tiles, out_s32=True)
        for st, sp in [(-1, 1), (3, 2), (5, 4)]:
            y = cr.convrot_debug_gemm_split(qx, sx, rep, sw, b, K, tiles | cr.TILES_REPACKED, st, sp,
                                            area, N=N)
            a = cr.convrot_debug_gemm_split(qx, None, rep, None, None, K, tiles | cr.TILES_REPACKED,
                                            st, sp, area, out_s32=True, N=N)
            torch.cuda.synchronize()
            assert torch.equal(y.view(torch.int16), whole.view(torch.int16)), (tiles, st, sp)
            assert torch.equal(a, acc), (tiles, st, sp)
            assert not area[:cr.SPLIT_COUNTER_BYTES].any()
    # the whole layer on repacked weights, where the planner splits
    M, K, N = 1536, 12288, 3072
    lt = wl.make_random_layer(M, K, N, 256, seed=32)
    x, w, b = lt.x.cuda(), lt.w.cuda(), lt.b.cuda()
    qw, sw = cr.convrot_quantize_weight(w, 256)
    rep = cr.convrot_repack_weight(qw)
    y_can = cr.convrot_linear(x, qw, sw, b, 256)
    y_rep = cr.convrot_linear_repacked(x, rep, sw, b, 256)
    torch.cuda.synchronize()
    assert cr.convrot_check_device_error() == 0
    assert torch.equal(y_can.view(torch.int16), y_rep.view(torch.int16))
