"""Comparison helpers for the GPU parity tests (test infrastructure).

Gates (fixed here, used by every GPU test):
  - rotated values: |y_gpu - y_oracle| <= 1e-5 * max|y_oracle| per row
    (fp32 butterflies against the fp64 dense product);
  - scales: relative difference <= 1e-5;
  - codes and packed bytes: identical, except at positions whose oracle
    y/s lies within 1e-5 of a .5 rounding boundary (the "tie band"), where
    the two fp32 evaluations of the rotation may round apart by one code;
  - integer accumulators: identical when both sides start from the same
    codes;
  - bf16 outputs: within 1 bf16 ulp of the oracle's fp32 epilogue when both
    sides start from the same codes and scales; with independently prepared
    codes, within 1 ulp plus the exact effect of the tie-band code
    differences the oracle itself identifies (each moves acc by at most the
    other operand's code magnitude + 1).

GPU bytes are decoded here with numpy, never by the oracle.
"""
from __future__ import annotations

import numpy as np
import torch

TIE_BAND = 1e-5
ROT_TOL = 1e-5
SCALE_RTOL = 1e-5


def to_np_u16(t: torch.Tensor) -> np.ndarray:
    return t.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)


def decode_codes(packed: np.ndarray) -> np.ndarray:
    """uint8 [rows][K/2] -> int8 [rows][K], low nibble first, two's complement."""
    p = packed.astype(np.int16)
    lo = p & 0xF
    hi = (p >> 4) & 0xF
    lo = np.where(lo >= 8, lo - 16, lo)
    hi = np.where(hi >= 8, hi - 16, hi)
    out = np.empty((packed.shape[0], packed.shape[1] * 2), dtype=np.int8)
    out[:, 0::2] = lo
    out[:, 1::2] = hi
    return out


def bf16_f64(bits: np.ndarray) -> np.ndarray:
    return (bits.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def bf16_ulp(v: np.ndarray) -> np.ndarray:
    a = np.abs(v)
    e = np.floor(np.log2(np.where(a > 0, a, 1e-38)))
    return np.where(a > 0, 2.0 ** (e - 7), 2.0 ** -133)


def check_rotation(y_gpu: np.ndarray, y_ref: np.ndarray):
    amax = np.abs(y_ref).max(axis=1, keepdims=True)
    err = np.abs(y_gpu.astype(np.float64) - y_ref)
    bad = err > ROT_TOL * np.maximum(amax, 1e-30)
    assert not bad.any(), f"rotation off at {np.argwhere(bad)[:5]}, max rel {(err / np.maximum(amax, 1e-30)).max()}"


def check_prepared(q_gpu_packed, s_gpu, q_ref_packed, s_ref, tie):
    """Codes/bytes equal outside the tie band; scales within SCALE_RTOL."""
    s_gpu = np.asarray(s_gpu, dtype=np.float64)
    s_ref = np.asarray(s_ref, dtype=np.float64)
    rel = np.abs(s_gpu - s_ref) / np.maximum(np.abs(s_ref), 1e-30)
    assert np.all((s_ref == 0) == (s_gpu == 0)), "zero-scale rows differ"
    assert rel.max() <= SCALE_RTOL, f"scale rel err {rel.max()}"
    cg = decode_codes(q_gpu_packed)
    cr = decode_codes(q_ref_packed)
    diff = cg != cr
    outside = diff & ~tie
    assert not outside.any(), f"{outside.sum()} codes differ outside the tie band, e.g. {np.argwhere(outside)[:5]}"
    assert np.all(np.abs(cg.astype(int) - cr.astype(int)) <= 1), "a code moved by more than one step"
    # bytes whose two codes agree must be identical
    same_pair = ~(diff[:, 0::2] | diff[:, 1::2])
    assert np.array_equal(q_gpu_packed[same_pair], q_ref_packed[same_pair])
    return int(diff.sum())


def output_tolerance(y_ref_bits, qx_ref, qw_ref, sx, sw, tie_x, tie_w):
    """Per-element allowance: 1 bf16 ulp, plus the largest acc change the
    oracle's tie-band positions allow, times the scales, plus one more ulp
    for the re-rounding when that term is nonzero."""
    y = bf16_f64(y_ref_bits)
    cx = np.abs(decode_codes(qx_ref).astype(np.int64)) + 1
    cw = np.abs(decode_codes(qw_ref).astype(np.int64)) + 1
    dacc = (tie_x.astype(np.int64) @ cw.T) + (cx @ tie_w.astype(np.int64).T)
    extra = dacc * np.asarray(sx, np.float64)[:, None] * np.asarray(sw, np.float64)[None, :] * 1.001
    tol = bf16_ulp(y) + extra + np.where(dacc > 0, bf16_ulp(np.abs(y) + extra), 0.0)
    return tol


def check_outputs(y_gpu_bits, y_ref_bits, tol=None):
    g = bf16_f64(y_gpu_bits)
    r = bf16_f64(y_ref_bits)
    if tol is None:
        tol = bf16_ulp(r)
    err = np.abs(g - r)
    bad = err > tol
    assert not bad.any(), (f"{bad.sum()} outputs outside tolerance, e.g. at {np.argwhere(bad)[:5]}: "
                           f"gpu {g[bad][:5]} ref {r[bad][:5]}")
    return int((err > 0).sum())


def bf16_spacing(y: np.ndarray) -> np.ndarray:
    """Distance between the two bf16 values around |y| (2^-133 below the
    normal range)."""
    a = np.abs(np.asarray(y, dtype=np.float64))
    _, e = np.frexp(a)
    return np.ldexp(1.0, np.where(e - 1 < -126, -133, e - 8))


def check_w4a16_outputs(y_gpu_bits, t, acc, l1, p16, sw, d_acc=0.0, scale_rtol=0.0):
    """W4A16 outputs against the exact t = sum xr q * sw + b (oracle, fp64):
    |y - t| <= half the bf16 spacing at max(|t|, |y|) + E, with
      E = |sw| (2^-18 (p16 + l1) + d_acc) + 2^-23 (|acc sw| + |t|)
          + scale_rtol |acc sw|.
    2^-18 (p16 + l1) allows each K = 16 accumulation step of the tensor
    cores 32 fp32 ulps of (|running sum| + its 16 |products|); d_acc is the
    exact effect of tie-band inputs; 2^-23 (...) the two fp32 roundings of
    the epilogue; scale_rtol the weight-scale tolerance when the GPU
    prepared its own weights.  Returns the share of outputs equal to
    bf16_rne(t)."""
    y = bf16_f64(y_gpu_bits)
    swa = np.abs(np.asarray(sw, np.float64))[None, :]
    A = 2.0 ** -18 * (p16 + l1)
    E = swa * (A + d_acc) + 2.0 ** -23 * (np.abs(acc) * swa + np.abs(t)) + scale_rtol * np.abs(acc) * swa
    tol = 0.5 * np.maximum(bf16_spacing(np.abs(t) + E), bf16_spacing(y)) + E
    err = np.abs(y - t)
    bad = err > tol
    assert not bad.any(), (f"{bad.sum()} outputs outside tolerance, e.g. at {np.argwhere(bad)[:5]}: "
                           f"gpu {y[bad][:5]} exact {t[bad][:5]} tol {tol[bad][:5]}")
    sp = bf16_spacing(t)
    return float(np.mean(np.abs(y - t) <= 0.5 * sp))


def w4a16_input_effect(y64_rot, xr_bits, qw_codes, tie_w, rot_band):
    """d_acc: the largest change of sum_k xr q that the tie-band inputs
    allow: one bf16 spacing of xr at each activation position of the band
    (times |q| + 1), one code step at each weight position of the band
    (times |xr| + one spacing)."""
    sp = bf16_spacing(y64_rot)
    qabs = np.abs(qw_codes.astype(np.float64)) + 1.0
    xabs = np.abs(bf16_f64(xr_bits)) + sp
    return (rot_band * sp) @ qabs.T + xabs @ tie_w.astype(np.float64).T


def check_nvfp4_outputs(y_gpu_bits, t, acc, l1, p64, sx, sw):
    """NVFP4 outputs against the exact t = acc sx sw + b (oracle, fp64):
    |y - t| <= half the bf16 spacing at max(|t|, |y|) + E, with
      E = |sx sw| 2^-20 (p64 + l1) + 2^-23 (|acc sx sw| + |t|).
    Every product of two E2M1 codes and two E4M3 scales is exact in fp32;
    2^-20 (p64 + l1) lets each 64-deep tensor-core step err by 8 fp32 ulps
    of its |running sum| and of the |products| it adds; 2^-23 (...) covers the
    three fp32 roundings of the epilogue ((acc sx) sw + b).  Returns the
    share of outputs equal to bf16_rne(t)."""
    y = bf16_f64(y_gpu_bits)
    sxw = np.abs(np.asarray(sx, np.float64))[:, None] * np.abs(np.asarray(sw, np.float64))[None, :]
    E = sxw * 2.0 ** -20 * (p64 + l1) + 2.0 ** -23 * (np.abs(acc) * sxw + np.abs(t)) * 1.5
    tol = 0.5 * np.maximum(bf16_spacing(np.abs(t) + E), bf16_spacing(y)) + E
    err = np.abs(y - t)
    bad = err > tol
    assert not bad.any(), (f"{bad.sum()} outputs outside tolerance, e.g. at {np.argwhere(bad)[:5]}: "
                           f"gpu {y[bad][:5]} exact {t[bad][:5]} tol {tol[bad][:5]}")
    return float(np.mean(np.abs(y - t) <= 0.5 * bf16_spacing(t)))


def nvfp4_sf_rowmajor(sf_atoms: np.ndarray, rows: int, K: int) -> np.ndarray:
    """The boundary's scale atoms -> row-major [rows][K/16] (the index map of
    include/convrot_nvfp4.h, restated here)."""
    r = np.arange(rows)[:, None]
    j = np.arange(K // 16)[None, :]
    off = ((r // 128) * (K // 64) + j // 4) * 512 + 16 * (r % 32) + 4 * ((r // 32) % 4) + j % 4
    return sf_atoms[off]


def nvfp4_codes_equal(a_packed: np.ndarray, b_packed: np.ndarray) -> np.ndarray:
    """Per code (unpacked, [rows][K]): equal, counting the two encodings of
    zero (0 and 8) as the same value."""
    def unpack(p):
        out = np.empty((p.shape[0], 2 * p.shape[1]), np.uint8)
        out[:, 0::2] = p & 0xF
        out[:, 1::2] = p >> 4
        out[out == 8] = 0
        return out
    return unpack(a_packed) == unpack(b_packed)
