"""Guard bytes around every buffer the libraries write.

Out-of-bounds writes are looked for directly: each output, workspace and
split area given to a call is a view into a larger buffer whose bytes before
and after it hold a seeded random pattern (at least one output row's worth on
each side, so that a row written one row too far is caught too).  After each
call:
- the pattern is intact;
- the call's inputs are unchanged;
- its outputs equal, bit for bit, the same call on plain allocations (so the
  kernels do not depend on where in memory the buffers start: outputs here
  begin 16 bytes past a 256-byte boundary, the least alignment the headers
  allow).

The shapes cover every kernel the libraries choose between or can be forced
to run:
- the three activation-prep kernels;
- the one-kernel decode path;
- the few-token and token-major GEMM forms, with both store paths (TMA boxes
  when N % 8 == 0, direct stores otherwise);
- split K, with the planner's and forced plans;
- the repacked-weight forms and the no-alloc entry point;
- the W4A16 and NVFP4 variants, with each NVFP4 tile width.

Empty inputs (M = 0) must write nothing."""
import numpy as np
import pytest
import torch

import rotated_w4a4_quantized_b200 as cr
from rotated_w4a4_quantized_b200 import workloads as wl

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _built():
    if not torch.cuda.is_available():
        pytest.skip("no GPU")
    from rotated_w4a4_quantized_b200 import build
    build.build()


_seed = [0]


class Guarded:
    """A `shape` `dtype` tensor (`.t`) inside a buffer with guard bytes on
    both sides.  `ws=True` starts it on a 256-byte boundary (workspaces and
    split areas need that), otherwise 16 bytes past one."""

    def __init__(self, shape, dtype, ws=False):
        esize = torch.empty((), dtype=dtype).element_size()
        n = int(np.prod(shape)) * esize
        row = (int(shape[-1]) * esize) if len(shape) > 1 else 0
        self.pre = -(-(row + 256) // 256) * 256 + (0 if ws else 16)
        self.n = n
        post = max(4096, row + 256)
        _seed[0] += 1
        g = torch.Generator().manual_seed(1000 + _seed[0])
        self.buf = torch.randint(0, 256, (self.pre + n + post,), dtype=torch.uint8,
                                 generator=g).cuda()
        self.guard = self._guard_bytes().clone()
        self.t = self.buf[self.pre:self.pre + n].view(dtype).view(shape)

    def _guard_bytes(self):
        return torch.cat([self.buf[:self.pre], self.buf[self.pre + self.n:]])

    def intact(self) -> bool:
        return torch.equal(self._guard_bytes(), self.guard)


def _area():
    a = Guarded((cr.SPLIT_AREA_BYTES,), torch.uint8, ws=True)
    a.t[:cr.SPLIT_COUNTER_BYTES].zero_()
    return a


def _bits(t):
    return t.view(torch.int16) if t.dtype == torch.bfloat16 else t


class Inputs:
    """Copies of a call's inputs, to check that the call left them alone."""

    def __init__(self, *ts):
        self.ts = [t for t in ts if t is not None]
        self.copies = [t.clone() for t in self.ts]

    def unchanged(self) -> bool:
        return all(torch.equal(_bits(a), _bits(b)) for a, b in zip(self.ts, self.copies))


def _verify(what, guards, inputs, pairs, check_error=cr.convrot_check_device_error):
    torch.cuda.synchronize()
    assert check_error() == 0, what
    for i, g in enumerate(guards):
        assert g.intact(), f"{what}: guard bytes of buffer {i} overwritten"
    assert inputs.unchanged(), f"{what}: an input changed"
    for i, (got, want) in enumerate(pairs):
        assert torch.equal(_bits(got), _bits(want)), f"{what}: output {i} differs"


def _layer(M, K, N, group, seed, bias=True):
    lt = wl.make_random_layer(M, K, N, group, seed, bias=bias)
    return lt.x.cuda(), lt.w.cuda(), None if lt.b is None else lt.b.cuda()


# ---------------------------------------------------------------------------
# activation prep: 16 channels per thread (<= 1024 rows), 32 (group 256,
# K <= 3072, more rows), 64 (the rest, and K > 16384)
# ---------------------------------------------------------------------------

PREP_CASES = [(37, 1088, 64), (1100, 2048, 256), (1100, 1024, 64), (3, 32768, 256),
              (0, 1024, 64)]


@pytest.mark.parametrize("M,K,group", PREP_CASES)
def test_prep_writes_only_its_outputs(M, K, group):
    x, _, _ = _layer(M, K, 1, group, seed=M + K)
    inp = Inputs(x)
    qx_ref, sx_ref = cr.convrot_prepare_act(x, group)
    rot_ref = cr.convrot_debug_rotate_f32(x, group)
    qx, sx = Guarded((M, K // 2), torch.uint8), Guarded((M,), torch.float32)
    cr.convrot_prepare_act(x, group, qx.t, sx.t)
    rot = Guarded((M, K), torch.float32)
    cr.convrot_debug_rotate_f32(x, group, rot.t)
    qw, sw = Guarded((M, K // 2), torch.uint8), Guarded((M,), torch.float32)
    cr.convrot_quantize_weight(x, group, qw.t, sw.t)
    _verify("prep", [qx, sx, rot, qw, sw], inp,
            [(qx.t, qx_ref), (sx.t, sx_ref), (rot.t, rot_ref), (qw.t, qx_ref), (sw.t, sx_ref)])


# ---------------------------------------------------------------------------
# the whole layer
# ---------------------------------------------------------------------------

# (M, K, N, group): the one-kernel decode path (N % 8 == 0 and not), the
# few-token GEMM (up to 128 tokens), token-major tiles with both store paths,
# prep32 before the tiles, layers the planner splits on 148 SMs, no tokens
LAYER_CASES = [(1, 2048, 1000, 64), (3, 4096, 777, 256), (4, 2048, 130, 256),
               (17, 1088, 385, 64), (128, 2048, 600, 64), (129, 1024, 264, 256),
               (257, 1088, 385, 64), (1000, 3136, 2000, 64), (1100, 2048, 520, 256),
               (512, 4096, 14336, 64), (1536, 12288, 3072, 256), (0, 1024, 264, 64)]


@pytest.mark.parametrize("M,K,N,group", LAYER_CASES)
def test_linear_writes_only_its_workspace_and_output(M, K, N, group):
    x, w, b = _layer(M, K, N, group, seed=3 * M + N)
    qw, sw = cr.convrot_quantize_weight(w, group)
    inp = Inputs(x, qw, sw, b)
    y_ref = cr.convrot_linear(x, qw, sw, b, group)
    need = cr.convrot_linear_workspace_size(M, K)
    base = need - cr.SPLIT_AREA_BYTES if M > 128 and need else need
    for size in sorted({need, base}):                 # with and without the split area
        ws, y = Guarded((size,), torch.uint8, ws=True), Guarded((M, N), torch.bfloat16)
        cr.convrot_linear(x, qw, sw, b, group, ws.t, y.t)
        _verify(f"linear, workspace {size} of {need}", [ws, y], inp, [(y.t, y_ref)])


NOALLOC_CASES = [(1500, 4096, 640, 64), (37, 1024, 264, 256), (2, 4096, 777, 256),
                 (300, 1088, 385, 64)]


@pytest.mark.parametrize("M,K,N,group", NOALLOC_CASES)
def test_noalloc_writes_only_its_output(M, K, N, group):
    x, w, b = _layer(M, K, N, group, seed=5 * M + N)
    qw, sw = cr.convrot_quantize_weight(w, group)
    inp = Inputs(x, qw, sw, b)
    y_ref = cr.convrot_linear(x, qw, sw, b, group)
    y = Guarded((M, N), torch.bfloat16)
    cr.convrot_linear_noalloc(x, qw, sw, b, group, y.t)
    _verify("noalloc", [y], inp, [(y.t, y_ref)])


PREPARED_CASES = [(17, 1088, 385), (257, 1088, 385), (512, 4096, 14336), (1536, 12288, 3072)]


@pytest.mark.parametrize("M,K,N", PREPARED_CASES)
def test_prepared_and_split_write_only_their_outputs(M, K, N):
    x, w, b = _layer(M, K, N, 64, seed=7 * M + N)
    qw, sw = cr.convrot_quantize_weight(w, 64)
    qx, sx = cr.convrot_prepare_act(x, 64)
    inp = Inputs(qx, sx, qw, sw, b)
    y_ref = cr.convrot_linear_prepared(qx, sx, qw, sw, b, K)
    y1, y2, area = Guarded((M, N), torch.bfloat16), Guarded((M, N), torch.bfloat16), _area()
    cr.convrot_linear_prepared(qx, sx, qw, sw, b, K, y1.t)
    cr.convrot_linear_prepared_split(qx, sx, qw, sw, b, K, area.t, y2.t)
    _verify("prepared / prepared_split", [y1, y2, area], inp, [(y1.t, y_ref), (y2.t, y_ref)])
    assert not area.t[:cr.SPLIT_COUNTER_BYTES].any()


# ---------------------------------------------------------------------------
# every GEMM form, forced
# ---------------------------------------------------------------------------

TILE_FORMS = [cr.TILES_128x256, cr.TILES_128x192, cr.TILES_256x192_PAIR, cr.TILES_256x128_PAIR]
FEW_FORMS = [cr.SKINNY_TMEM, cr.SKINNY_SMEM, cr.SKINNY_PAIR]
FORM_CASES = [(17, 257, 1088), (100, 200, 192), (128, 520, 2048), (257, 385, 1088),
              (1000, 2000, 512)]


@pytest.mark.parametrize("M,N,K", FORM_CASES)
def test_gemm_forms_write_only_their_outputs(M, N, K):
    x, w, b = _layer(M, K, N, 64, seed=11 * M + N)
    qw, sw = cr.convrot_quantize_weight(w, 64)
    qx, sx = cr.convrot_prepare_act(x, 64)
    inp = Inputs(qx, sx, qw, sw, b)
    forms = [cr.TILES_AUTO] + TILE_FORMS + (FEW_FORMS if M <= 128 else [])
    for form in forms:
        y_ref = cr.convrot_debug_gemm_tiles(qx, sx, qw, sw, b, K, form)
        a_ref = cr.convrot_debug_gemm_tiles(qx, None, qw, None, None, K, form, out_s32=True)
        y, a = Guarded((M, N), torch.bfloat16), Guarded((M, N), torch.int32)
        cr.convrot_debug_gemm_tiles(qx, sx, qw, sw, b, K, form, out=y.t)
        cr.convrot_debug_gemm_tiles(qx, None, qw, None, None, K, form, out_s32=True, out=a.t)
        _verify(f"form {form}", [y, a], inp, [(y.t, y_ref), (a.t, a_ref)])
    s_ref = cr.convrot_debug_gemm_s32(qx, qw, K)
    s = Guarded((M, N), torch.int32)
    cr.convrot_debug_gemm_s32(qx, qw, K, s.t)
    _verify("debug_gemm_s32", [s], inp, [(s.t, s_ref)])


# (form, rows of A per tile, BN, CTAs per tile)
SPLIT_FORMS = [(cr.TILES_128x256, 128, 256, 1), (cr.TILES_128x192, 128, 192, 1),
               (cr.TILES_256x192_PAIR, 256, 192, 2), (cr.TILES_256x128_PAIR, 256, 128, 2)]


@pytest.mark.parametrize("form,tm,bn,cg", SPLIT_FORMS, ids=["128x256", "128x192tmem",
                                                            "256x192pair", "256x128pair"])
def test_split_plans_write_only_their_outputs_and_area(form, tm, bn, cg):
    M, N, K = 300, 600, 3136                      # 13 or 25 K-stages per tile
    x, w, b = _layer(M, K, N, 64, seed=13 + form)
    qw, sw = cr.convrot_quantize_weight(w, 64)
    qx, sx = cr.convrot_prepare_act(x, 64)
    inp = Inputs(qx, sx, qw, sw, b)
    tiles = -(-M // tm) * -(-N // bn)
    y_ref = cr.convrot_debug_gemm_tiles(qx, sx, qw, sw, b, K, form)
    a_ref = cr.convrot_debug_gemm_tiles(qx, None, qw, None, None, K, form, out_s32=True)
    for st, sp in [(-1, 1), (1, 3), (tiles, 2)]:
        assert tiles * 2 * cg * 128 * bn * 4 <= cr.SPLIT_AREA_BYTES - cr.SPLIT_COUNTER_BYTES
        y, a, area = Guarded((M, N), torch.bfloat16), Guarded((M, N), torch.int32), _area()
        cr.convrot_debug_gemm_split(qx, sx, qw, sw, b, K, form, st, sp, area.t, out=y.t)
        cr.convrot_debug_gemm_split(qx, None, qw, None, None, K, form, st, sp, area.t,
                                    out_s32=True, out=a.t)
        _verify(f"split {st} x {sp}", [y, a, area], inp, [(y.t, y_ref), (a.t, a_ref)])
        assert not area.t[:cr.SPLIT_COUNTER_BYTES].any()


# ---------------------------------------------------------------------------
# repacked weights
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("M,K,N", [(17, 1088, 385), (1000, 3136, 2000)])
def test_repacked_forms_write_only_their_outputs(M, K, N):
    x, w, b = _layer(M, K, N, 64, seed=17 * M + N)
    qw, sw = cr.convrot_quantize_weight(w, 64)
    qx, sx = cr.convrot_prepare_act(x, 64)
    size = cr.convrot_repacked_weight_size(N, K)
    inp = Inputs(x, qw, sw, b, qx, sx)
    rep_ref = cr.convrot_repack_weight(qw)
    rep = Guarded((size,), torch.uint8)
    cr.convrot_repack_weight(qw, rep.t)
    unp = Guarded((N, K // 2), torch.uint8)
    cr.convrot_unpack_weight(rep_ref, N, K, unp.t)
    _verify("repack / unpack", [rep, unp], inp, [(rep.t, rep_ref), (unp.t, qw)])

    inp = Inputs(x, rep_ref, sw, b, qx, sx)
    y_ref = cr.convrot_linear(x, qw, sw, b, 64)
    need = cr.convrot_linear_workspace_size(M, K)
    ws, y1, y2 = (Guarded((need,), torch.uint8, ws=True), Guarded((M, N), torch.bfloat16),
                  Guarded((M, N), torch.bfloat16))
    cr.convrot_linear_repacked(x, rep_ref, sw, b, 64, ws.t, y1.t)
    cr.convrot_linear_prepared_repacked(qx, sx, rep_ref, sw, b, K, y2.t)
    _verify("linear_repacked / prepared_repacked", [ws, y1, y2], inp,
            [(y1.t, y_ref), (y2.t, y_ref)])
    forms = [cr.TILES_256x192_PAIR, cr.TILES_128x192] + (FEW_FORMS if M <= 128 else [])
    for form in forms:
        want = cr.convrot_debug_gemm_tiles(qx, sx, qw, sw, b, K, form)
        y = Guarded((M, N), torch.bfloat16)
        cr.convrot_debug_gemm_tiles(qx, sx, rep_ref, sw, b, K, form | cr.TILES_REPACKED, out=y.t,
                                    N=N)
        _verify(f"repacked form {form}", [y], inp, [(y.t, want)])


# ---------------------------------------------------------------------------
# the W4A16 variant
# ---------------------------------------------------------------------------

W4A16_CASES = [(1, 1000, 192), (17, 300, 2048), (50, 9, 12288), (64, 1024, 4096),
               (130, 264, 1088), (257, 385, 2048), (0, 264, 256)]


@pytest.mark.parametrize("M,N,K", W4A16_CASES)
def test_w4a16_writes_only_its_outputs(M, N, K):
    x, w, b = _layer(M, K, N, 64, seed=19 * M + N)
    qw, sw = cr.convrot_quantize_weight(w, 64)
    rep = cr.convrot_repack_weight(qw)
    inp = Inputs(x, qw, sw, b, rep)
    chk = cr.convrot_w4a16_check_device_error
    xr_ref = cr.convrot_w4a16_prepare_act(x, 64)
    xr = Guarded((M, K), torch.bfloat16)
    cr.convrot_w4a16_prepare_act(x, 64, xr.t)
    _verify("w4a16 prepare", [xr], inp, [(xr.t, xr_ref)], chk)

    y_ref = cr.convrot_w4a16_linear(x, qw, sw, b, 64)
    need = cr.convrot_w4a16_workspace_size(M, K)
    ws, y1, y2 = (Guarded((need,), torch.uint8, ws=True), Guarded((M, N), torch.bfloat16),
                  Guarded((M, N), torch.bfloat16))
    cr.convrot_w4a16_linear(x, qw, sw, b, 64, ws.t, y1.t)
    ws2 = Guarded((need,), torch.uint8, ws=True)
    cr.convrot_w4a16_linear_repacked(x, rep, sw, b, 64, ws2.t, y2.t)
    _verify("w4a16 linear", [ws, y1, ws2, y2], inp, [(y1.t, y_ref), (y2.t, y_ref)], chk)

    inp = Inputs(xr_ref, qw, sw, b, rep)
    y3 = Guarded((M, N), torch.bfloat16)
    cr.convrot_w4a16_linear_prepared_repacked(xr_ref, rep, sw, b, y3.t)
    _verify("w4a16 prepared_repacked", [y3], inp, [(y3.t, y_ref)], chk)
    forms = [cr.W4A16_AUTO, cr.W4A16_TILES] + (
        [cr.W4A16_FEW_SMEM, cr.W4A16_FEW_TMEM] if 0 < M <= 64 else [])
    for form in forms:
        want = cr.convrot_w4a16_debug_gemm_form(xr_ref, qw, sw, b, form)
        y, yr = Guarded((M, N), torch.bfloat16), Guarded((M, N), torch.bfloat16)
        cr.convrot_w4a16_debug_gemm_form(xr_ref, qw, sw, b, form, y.t)
        cr.convrot_w4a16_debug_gemm_form(xr_ref, rep, sw, b, form | cr.TILES_REPACKED, yr.t, N=N)
        _verify(f"w4a16 form {form}", [y, yr], inp, [(y.t, want), (yr.t, want)], chk)


# ---------------------------------------------------------------------------
# the NVFP4 variant
# ---------------------------------------------------------------------------

NVFP4_CASES = [(1, 1024, 300, 64), (130, 192, 200, 64), (300, 1024, 520, 64),
               (257, 4096, 256, 256), (1100, 1024, 264, 256), (0, 1024, 264, 64)]


@pytest.mark.parametrize("M,K,N,group", NVFP4_CASES)
def test_nvfp4_writes_only_its_outputs(M, K, N, group):
    x, w, b = _layer(M, K, N, group, seed=23 * M + N)
    chk = cr.convrot_nvfp4_check_device_error
    qw, sfw, sw = cr.convrot_nvfp4_quantize(w, group)
    qx_ref, sfx_ref, sx_ref = cr.convrot_nvfp4_quantize(x, group)
    inp = Inputs(x, qw, sfw, sw, b)
    nsf = cr.convrot_nvfp4_scale_bytes(M, K)
    q, sf, s = (Guarded((M, K // 2), torch.uint8), Guarded((max(1, nsf),), torch.uint8),
                Guarded((M,), torch.float32))
    cr.convrot_nvfp4_quantize(x, group, q.t, sf.t, s.t)
    pairs = [(q.t, qx_ref), (s.t, sx_ref)] + ([(sf.t, sfx_ref)] if nsf else [])
    _verify("nvfp4 quantize", [q, sf, s], inp, pairs, chk)

    y_ref = cr.convrot_nvfp4_linear(x, qw, sfw, sw, b, group)
    need = cr.convrot_nvfp4_workspace_size(M, K)
    ws, y1, y2 = (Guarded((need,), torch.uint8, ws=True), Guarded((M, N), torch.bfloat16),
                  Guarded((M, N), torch.bfloat16))
    cr.convrot_nvfp4_linear(x, qw, sfw, sw, b, group, ws.t, y1.t)
    inp2 = Inputs(qx_ref, sfx_ref, sx_ref, qw, sfw, sw, b)
    if M:
        cr.convrot_nvfp4_linear_prepared(qx_ref, sfx_ref, sx_ref, qw, sfw, sw, b, K, y2.t)
    _verify("nvfp4 linear", [ws, y1, y2], inp, [(y1.t, y_ref)] + ([(y2.t, y_ref)] if M else []),
            chk)
    assert inp2.unchanged()
    if M:                           # each tile width, forced
        for form in (cr.NVFP4_TILES_256, cr.NVFP4_TILES_128):
            want = cr.convrot_nvfp4_debug_gemm_form(qx_ref, sfx_ref, sx_ref, qw, sfw, sw, b, K, form)
            y3 = Guarded((M, N), torch.bfloat16)
            cr.convrot_nvfp4_debug_gemm_form(qx_ref, sfx_ref, sx_ref, qw, sfw, sw, b, K, form, y3.t)
            _verify(f"nvfp4 form {form}", [y3], inp2, [(y3.t, want)], chk)
