"""The split-K planner of the token-major GEMM, on the host (no GPU): the
form and plan convrot_linear takes for a shape (convrot_debug_gemm_plan).

Split K changes only the schedule of the integer product (the product itself:
"convrot-mlx" README, "Install and test"); its results are bit-identical
(tests/test_gpu_split.py).  What is pinned here:
- the decisions measured on a B200 (74 CTA pairs, 148 SMs): split where it
  paid (the DiT down projection in 3 parts, the 512-token layer in 4), whole
  where it did not (12-stage tiles, layers of less than one wave, full last
  waves);
- invariants for any shape: parts within one wave and the split area, 2-4
  parts of at least two K-stages each, never a split without an area, the
  few-token form up to 128 tokens, and a busiest pair that is never busier
  than without the split (by simulating the unit schedule)."""
import itertools

import pytest

import rotated_w4a4_quantized_b200 as cr

PAIRS, SMS = 74, 148
T256x192, T256x128, SKINNY = cr.TILES_256x192_PAIR, cr.TILES_256x128_PAIR, cr.SKINNY_TMEM


@pytest.fixture(scope="module", autouse=True)
def _built():
    from rotated_w4a4_quantized_b200 import build
    build.build()


@pytest.mark.parametrize("M,K,N,expect", [
    (8192, 8192, 8192, (T256x192, 0, 1)),     # square: a full-enough last wave
    (4608, 3072, 9216, (T256x192, 0, 1)),     # QKV
    (1536, 12288, 3072, (T256x192, 22, 3)),   # DiT down: 59.7 -> 44.1 us measured
    (1536, 3072, 12288, (T256x192, 0, 1)),    # DiT up: 12-stage tiles, no gain measured
    (512, 4096, 14336, (T256x192, 2, 4)),     # 34.7 -> 31.1 us measured
    (1024, 3072, 3072, (T256x192, 0, 1)),     # outlier layer: 64 tiles, less than a wave
    (512, 4096, 2048, (T256x128, 0, 1)),      # 22 tiles: 14.8 unsplit vs 15.7 us split
    (16, 4096, 14336, (SKINNY, 0, 1)),        # few tokens
])
def test_measured_decisions_on_a_b200(M, K, N, expect):
    assert cr.convrot_debug_gemm_plan(M, N, K, PAIRS, SMS) == expect


def test_no_area_no_split():
    for M, K, N in [(1536, 12288, 3072), (512, 4096, 14336), (1024, 8192, 5120)]:
        t, st, sp = cr.convrot_debug_gemm_plan(M, N, K, PAIRS, SMS, split_bytes=0)
        assert (st, sp) == (0, 1)
    # without the area the DiT down projection falls back to the narrower pair
    # tile (144 tiles of 256 x 128 take 0.9 of the 256 x 192 time per wave)
    assert cr.convrot_debug_gemm_plan(1536, 3072, 12288, PAIRS, SMS, split_bytes=0) == (T256x128, 0, 1)


def _busiest(tiles, slots, num_kp, split_tiles, splits):
    """Busiest slot's K-stages under the kernel's unit schedule (unit u on
    slot u mod slots; the first split_tiles tiles cut into `splits` parts
    first)."""
    nsu = split_tiles * splits
    load = [0] * slots
    for u in range(tiles + split_tiles * (splits - 1)):
        if u < nsu:
            p = u % splits
            k0, k1 = p * num_kp // splits, (p + 1) * num_kp // splits
            assert k1 > k0
        else:
            k0, k1 = 0, num_kp
        load[u % slots] += k1 - k0
    return max(load)


SHAPE = {T256x192: (256, 192, 128, 2), T256x128: (256, 128, 128, 2),
         cr.TILES_128x192: (128, 192, 128, 1), cr.TILES_128x256: (128, 256, 64, 1)}


@pytest.mark.parametrize("pairs,sms", [(74, 148), (0, 148), (66, 132)])
def test_plan_invariants_over_shapes(pairs, sms):
    Ms = [129, 300, 512, 1024, 1536, 2048, 4096]
    Ns = [64, 1000, 2048, 3072, 5120, 12288]
    Ks = [64, 1024, 3072, 8192, 12288]
    for M, N, K in itertools.product(Ms, Ns, Ks):
        t, st, sp = cr.convrot_debug_gemm_plan(M, N, K, pairs, sms)
        assert t in SHAPE, (M, N, K, t)
        if pairs == 0:
            assert t in (cr.TILES_128x192, cr.TILES_128x256)
        tm, bn, pkb, cg = SHAPE[t]
        tiles = -(-M // tm) * -(-N // bn)
        num_kp = -(-(K // 2) // pkb)
        slots = pairs if cg == 2 else sms
        if st == 0:
            assert sp == 1
            continue
        assert 2 <= sp <= 4 and 2 * sp <= num_kp                      # parts of >= 2 stages
        assert st == tiles % slots and st * sp <= slots                # the last wave only
        assert st * sp * cg <= (cr.SPLIT_AREA_BYTES - cr.SPLIT_COUNTER_BYTES) // (128 * bn * 4)
        assert st * cg * 8 <= cr.SPLIT_COUNTER_BYTES // 4
        assert _busiest(tiles, slots, num_kp, st, sp) < _busiest(tiles, slots, num_kp, 0, 1)


def test_plan_argument_errors():
    with pytest.raises(cr.ConvRotError) as e:
        cr.convrot_debug_gemm_plan(1024, 1024, 1000)
    assert e.value.status == 3
    with pytest.raises(cr.ConvRotError) as e:
        cr.convrot_debug_gemm_plan(1024, 1024, 1024, pairs=-1)
    assert e.value.status == 3
    with pytest.raises(cr.ConvRotError) as e:
        cr.convrot_debug_gemm_plan(1024, 1024, 1024, sms=0)
    assert e.value.status == 3
