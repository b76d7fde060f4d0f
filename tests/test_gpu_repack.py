"""The reversible weight repack on the GPU ("convrot-mlx" README, "What is
included": lossless repacking of the packed weights; here the block-major
layout of include/convrot.h).

The repack kernel's bytes equal the oracle's (tests/test_oracle.py pins the
oracle's layout and round trip), the unpack kernel inverts both exactly, and
every kernel that reads weights gives bit-identical results on repacked
weights and on the canonical ones: each GEMM form of the token-major and
few-token kernels, the one-kernel decode path, the whole layer, and both
forms of the W4A16 GEMM."""
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


def _eq16(a, b):
    return torch.equal(a.view(torch.int16), b.view(torch.int16))


@pytest.mark.parametrize("N,K", [(1, 64), (7, 192), (300, 320), (1000, 4096), (129, 12288),
                                 (64, 32768)])
def test_repack_matches_oracle_and_unpack_inverts(N, K):
    g = torch.Generator().manual_seed(N + K)
    qw = torch.randint(0, 256, (N, K // 2), dtype=torch.uint8, generator=g)
    rep_ref = O.repack_weight(qw.numpy(), K)
    rep = cr.convrot_repack_weight(qw.cuda())
    back = cr.convrot_unpack_weight(rep, N, K)
    back_ref = cr.convrot_unpack_weight(torch.from_numpy(rep_ref).cuda(), N, K)
    torch.cuda.synchronize()
    assert cr.convrot_check_device_error() == 0
    assert np.array_equal(rep.cpu().numpy(), rep_ref)
    assert torch.equal(back.cpu(), qw) and torch.equal(back_ref.cpu(), qw)


FORMS = [cr.TILES_AUTO, cr.TILES_128x256, cr.TILES_128x192, cr.TILES_256x192_PAIR,
         cr.TILES_256x128_PAIR]
FEW = [cr.SKINNY_TMEM, cr.SKINNY_PAIR, cr.SKINNY_SMEM]


@pytest.mark.parametrize("M,N,K", [(200, 520, 768), (1100, 392, 3072), (300, 264, 320),
                                   (8, 300, 1024), (100, 600, 2048), (40, 136, 192)])
def test_every_gemm_form_is_bit_identical_on_repacked_weights(M, N, K):
    g = torch.Generator().manual_seed(M * N + K)
    qx = torch.randint(0, 256, (M, K // 2), dtype=torch.uint8, generator=g).cuda()
    qw = torch.randint(0, 256, (N, K // 2), dtype=torch.uint8, generator=g).cuda()
    sx = (torch.rand(M, generator=g) * 0.01).cuda()
    sw = (torch.rand(N, generator=g) * 0.01).cuda()
    b = (torch.randn(N, generator=g) * 0.02).to(torch.bfloat16).cuda()
    rep = cr.convrot_repack_weight(qw)
    forms = FORMS + (FEW if M <= 128 else [])
    for form in forms:
        if form == cr.SKINNY_SMEM and M <= 16:
            with pytest.raises(cr.ConvRotError) as e:      # 256-byte boxes: not on this layout
                cr.convrot_debug_gemm_tiles(qx, sx, rep, sw, b, K, form | cr.TILES_REPACKED, N=N)
            assert e.value.status == 8
            continue
        y = cr.convrot_debug_gemm_tiles(qx, sx, qw, sw, b, K, form)
        yr = cr.convrot_debug_gemm_tiles(qx, sx, rep, sw, b, K, form | cr.TILES_REPACKED, N=N)
        acc = cr.convrot_debug_gemm_tiles(qx, None, qw, None, None, K, form, out_s32=True)
        accr = cr.convrot_debug_gemm_tiles(qx, None, rep, None, None, K, form | cr.TILES_REPACKED,
                                           out_s32=True, N=N)
        torch.cuda.synchronize()
        assert cr.convrot_check_device_error() == 0
        assert _eq16(y, yr), form
        assert torch.equal(acc, accr), form
    yp = cr.convrot_linear_prepared(qx, sx, qw, sw, b, K)
    ypr = cr.convrot_linear_prepared_repacked(qx, sx, rep, sw, b, K)
    torch.cuda.synchronize()
    assert _eq16(yp, ypr)


@pytest.mark.parametrize("M,K,N,group", [(1, 4096, 14336, 64), (3, 2048, 300, 256),
                                         (16, 4096, 1000, 64), (100, 1024, 264, 256),
                                         (600, 3072, 520, 64), (37, 320, 72, 64)])
def test_whole_layer_on_repacked_weights(M, K, N, group):
    lt = wl.make_random_layer(M, K, N, group, seed=M + K + N)
    x, w, b = lt.x.cuda(), lt.w.cuda(), lt.b.cuda()
    qw, sw = cr.convrot_quantize_weight(w, group)
    rep = cr.convrot_repack_weight(qw)
    y = cr.convrot_linear(x, qw, sw, b, group)
    yr = cr.convrot_linear_repacked(x, rep, sw, b, group)
    torch.cuda.synchronize()
    assert cr.convrot_check_device_error() == 0
    assert _eq16(y, yr)
    if M <= 40:
        # and the oracle on the same inputs, through the unpacked weights
        pw, swr = O.prepare_rows(wl.bf16_bits(lt.w), group)
        assert np.array_equal(cr.convrot_unpack_weight(rep, N, K).cpu().numpy(), qw.cpu().numpy())
        y_ref = O.linear_prepared_w(wl.bf16_bits(lt.x), qw.cpu().numpy(), sw.cpu().numpy(),
                                    wl.bf16_bits(lt.b), group)
        from tests import gpu_compare as gc
        px, sx = O.prepare_rows(wl.bf16_bits(lt.x), group)
        tie_x = O.tie_band(O.rotate(wl.bf16_bits(lt.x), group), sx)
        tol = gc.output_tolerance(y_ref, px, qw.cpu().numpy(), sx, sw.cpu().numpy(), tie_x,
                                  np.zeros((N, K), dtype=bool))
        gc.check_outputs(gc.to_np_u16(yr), y_ref, tol)


@pytest.mark.parametrize("M,K,N", [(1, 4096, 2000), (16, 1024, 520), (64, 2048, 300),
                                   (200, 3072, 600), (33, 320, 136)])
def test_w4a16_on_repacked_weights(M, K, N):
    lt = wl.make_random_layer(M, K, N, 64, seed=7 * M + N)
    x, w, b = lt.x.cuda(), lt.w.cuda(), lt.b.cuda()
    qw, sw = cr.convrot_quantize_weight(w, 64)
    rep = cr.convrot_repack_weight(qw)
    y = cr.convrot_w4a16_linear(x, qw, sw, b, 64)
    yr = cr.convrot_w4a16_linear_repacked(x, rep, sw, b, 64)
    xr = cr.convrot_w4a16_prepare_act(x, 64)
    yp = cr.convrot_w4a16_linear_prepared_repacked(xr, rep, sw, b)
    torch.cuda.synchronize()
    assert cr.convrot_w4a16_check_device_error() == 0
    assert _eq16(y, yr) and _eq16(y, yp)
    # every form that runs this shape, forced, on both layouts
    forms = [cr.W4A16_TILES] + ([cr.W4A16_FEW_SMEM, cr.W4A16_FEW_TMEM] if M <= 64 else [])
    for form in forms:
        yc = cr.convrot_w4a16_debug_gemm_form(xr, qw, sw, b, form)
        yf = cr.convrot_w4a16_debug_gemm_form(xr, rep, sw, b, form | cr.TILES_REPACKED, N=N)
        torch.cuda.synchronize()
        assert _eq16(yc, yf), form
