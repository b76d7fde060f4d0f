"""CPU oracle for the rotated W4A4 linear layer (test infrastructure only).

Only the test suite, ``__graft_entry__.smoke()`` and the benchmark's CPU
baseline import this package.  The product library never does, and nothing
here touches the CUDA path: this is a ctypes wrapper around the plain C file
``convrot_oracle.c`` (see its header for what each step computes and which
page section it follows).

Arrays are numpy; bf16 values travel as ``uint16`` bit patterns.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "convrot_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")

# Plain IEEE semantics: no fast-math, no contraction of a*b+c into an FMA.
_CFLAGS = ["-O2", "-std=c99", "-fPIC", "-shared", "-fopenmp", "-fno-fast-math",
           "-ffp-contract=off"]


def build(force: bool = False) -> str:
    """Compile the oracle with gcc if the shared object is missing or stale."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.run(["gcc", *_CFLAGS, _SRC, "-o", tmp, "-lm"], check=True)
        os.replace(tmp, _LIB)
    return _LIB


_lib = None


def lib():
    global _lib
    if _lib is None:
        L = ctypes.CDLL(build())
        P = ctypes.c_void_p
        I64 = ctypes.c_int64
        I = ctypes.c_int
        sig = {
            "oracle_bf16_to_double": [P, I64, P],
            "oracle_float_to_bf16": [P, I64, P],
            "oracle_hadamard": [I, P],
            "oracle_hadamard_kron": [I, P],
            "oracle_rotate": [P, I64, I64, I, P],
            "oracle_quantize_rows": [P, I64, I64, P, P],
            "oracle_pack": [P, I64, I64, P],
            "oracle_unpack": [P, I64, I64, P],
            "oracle_gemm": [P, P, I64, I64, I64, P],
            "oracle_epilogue": [P, P, P, P, I64, I64, P],
            "oracle_prepare_rows": [P, I64, I64, I, P, P],
            "oracle_linear_prepared_w": [P, P, P, P, I64, I64, I64, I, P],
            "oracle_round_bf16": [P, I64, P],
            "oracle_w4a16_rotate_act": [P, I64, I64, I, P],
            "oracle_w4a16_gemm": [P, P, I64, I64, I64, P, P, P],
            "oracle_w4a16_epilogue": [P, P, P, I64, I64, P, P],
            "oracle_w4a16_linear": [P, P, P, P, I64, I64, I64, I, P],
            "oracle_repack_weight": [P, I64, I64, P],
            "oracle_e2m1_round": [P, I64, P],
            "oracle_e4m3_round": [P, I64, P],
            "oracle_e2m1_value": [P, I64, P],
            "oracle_e4m3_value": [P, I64, P],
            "oracle_nvfp4_quantize_rows": [P, I64, I64, P, P, P],
            "oracle_nvfp4_pack": [P, I64, I64, P],
            "oracle_nvfp4_sf_layout": [P, I64, I64, P],
            "oracle_nvfp4_gemm": [P, P, P, P, I64, I64, I64, P, P, P],
            "oracle_nvfp4_epilogue": [P, P, P, P, I64, I64, P, P],
            "oracle_unpack_weight": [P, I64, I64, P],
            "oracle_num_threads": [],
        }
        for name, args in sig.items():
            f = getattr(L, name)
            f.argtypes = args
            f.restype = ctypes.c_int
        L.oracle_set_num_threads.argtypes = [I]
        L.oracle_set_num_threads.restype = None
        _lib = L
    return _lib


def _ptr(a: np.ndarray | None):
    if a is None:
        return None
    assert a.flags["C_CONTIGUOUS"], "oracle buffers must be contiguous"
    return a.ctypes.data_as(ctypes.c_void_p)


def _check(rc: int, what: str):
    if rc != 0:
        raise ValueError(f"{what}: oracle rejected the arguments (rc={rc})")


def set_num_threads(t: int) -> None:
    lib().oracle_set_num_threads(int(t))


def num_threads() -> int:
    return int(lib().oracle_num_threads())


# --------------------------------------------------------------------------
# bf16 helpers
# --------------------------------------------------------------------------

def bf16_to_f64(bits: np.ndarray) -> np.ndarray:
    bits = np.ascontiguousarray(bits, dtype=np.uint16)
    out = np.empty(bits.shape, dtype=np.float64)
    _check(lib().oracle_bf16_to_double(_ptr(bits), bits.size, _ptr(out)), "bf16_to_f64")
    return out


def f32_to_bf16(x: np.ndarray) -> np.ndarray:
    x = np.ascontiguousarray(x, dtype=np.float32)
    out = np.empty(x.shape, dtype=np.uint16)
    _check(lib().oracle_float_to_bf16(_ptr(x), x.size, _ptr(out)), "f32_to_bf16")
    return out


# --------------------------------------------------------------------------
# The method's steps
# --------------------------------------------------------------------------

def hadamard(n: int) -> np.ndarray:
    H = np.empty((n, n), dtype=np.float64)
    _check(lib().oracle_hadamard(n, _ptr(H)), "hadamard")
    return H


def hadamard_kron(n: int) -> np.ndarray:
    H = np.empty((n, n), dtype=np.float64)
    _check(lib().oracle_hadamard_kron(n, _ptr(H)), "hadamard_kron")
    return H


def rotate(x_bf16: np.ndarray, group: int) -> np.ndarray:
    """fp64 rows of x (I_G (x) H_group)."""
    x = np.ascontiguousarray(x_bf16, dtype=np.uint16)
    rows, K = x.shape
    y = np.empty((rows, K), dtype=np.float64)
    _check(lib().oracle_rotate(_ptr(x), rows, K, group, _ptr(y)), "rotate")
    return y


def quantize_rows(y: np.ndarray):
    """(codes int8 [rows][K], scales fp32 [rows]) from fp64 rotated rows."""
    y = np.ascontiguousarray(y, dtype=np.float64)
    rows, K = y.shape
    q = np.empty((rows, K), dtype=np.int8)
    s = np.empty((rows,), dtype=np.float32)
    _check(lib().oracle_quantize_rows(_ptr(y), rows, K, _ptr(q), _ptr(s)), "quantize_rows")
    return q, s


def pack(q: np.ndarray) -> np.ndarray:
    q = np.ascontiguousarray(q, dtype=np.int8)
    rows, K = q.shape
    p = np.empty((rows, K // 2), dtype=np.uint8)
    _check(lib().oracle_pack(_ptr(q), rows, K, _ptr(p)), "pack")
    return p


def unpack(p: np.ndarray, K: int) -> np.ndarray:
    p = np.ascontiguousarray(p, dtype=np.uint8)
    rows = p.shape[0]
    q = np.empty((rows, K), dtype=np.int8)
    _check(lib().oracle_unpack(_ptr(p), rows, K, _ptr(q)), "unpack")
    return q


def gemm(qx: np.ndarray, qw: np.ndarray, K: int) -> np.ndarray:
    """int64 acc[m][n] = sum_k qx[m][k] qw[n][k] from packed operands."""
    qx = np.ascontiguousarray(qx, dtype=np.uint8)
    qw = np.ascontiguousarray(qw, dtype=np.uint8)
    M, N = qx.shape[0], qw.shape[0]
    acc = np.empty((M, N), dtype=np.int64)
    _check(lib().oracle_gemm(_ptr(qx), _ptr(qw), M, N, K, _ptr(acc)), "gemm")
    return acc


def epilogue(acc: np.ndarray, sx: np.ndarray, sw: np.ndarray, bias_bf16: np.ndarray | None):
    acc = np.ascontiguousarray(acc, dtype=np.int64)
    sx = np.ascontiguousarray(sx, dtype=np.float32)
    sw = np.ascontiguousarray(sw, dtype=np.float32)
    b = None if bias_bf16 is None else np.ascontiguousarray(bias_bf16, dtype=np.uint16)
    M, N = acc.shape
    y = np.empty((M, N), dtype=np.uint16)
    _check(lib().oracle_epilogue(_ptr(acc), _ptr(sx), _ptr(sw), _ptr(b), M, N, _ptr(y)),
           "epilogue")
    return y


def prepare_rows(x_bf16: np.ndarray, group: int):
    """(packed uint8 [rows][K/2], scales fp32 [rows]): rotate, quantise, pack."""
    x = np.ascontiguousarray(x_bf16, dtype=np.uint16)
    rows, K = x.shape
    p = np.empty((rows, K // 2), dtype=np.uint8)
    s = np.empty((rows,), dtype=np.float32)
    _check(lib().oracle_prepare_rows(_ptr(x), rows, K, group, _ptr(p), _ptr(s)), "prepare_rows")
    return p, s


def linear_prepared_w(x_bf16, qw, sw, bias_bf16, group: int) -> np.ndarray:
    """bf16 bits y [M][N] of the whole layer given prepared weights."""
    x = np.ascontiguousarray(x_bf16, dtype=np.uint16)
    qw = np.ascontiguousarray(qw, dtype=np.uint8)
    sw = np.ascontiguousarray(sw, dtype=np.float32)
    b = None if bias_bf16 is None else np.ascontiguousarray(bias_bf16, dtype=np.uint16)
    M, K = x.shape
    N = qw.shape[0]
    y = np.empty((M, N), dtype=np.uint16)
    _check(lib().oracle_linear_prepared_w(_ptr(x), _ptr(qw), _ptr(sw), _ptr(b), M, N, K, group,
                                          _ptr(y)), "linear_prepared_w")
    return y


def tie_band(y: np.ndarray, s: np.ndarray, band: float = 1e-5) -> np.ndarray:
    """Mask of positions whose fp64 y/s lies within ``band`` of a .5 rounding
    boundary: the only positions where a code may legitimately differ between
    two fp32 evaluations of the rotation (different summation order)."""
    s64 = s.astype(np.float64)[:, None]
    with np.errstate(divide="ignore", invalid="ignore"):
        v = np.where(s64 > 0, y / np.where(s64 > 0, s64, 1.0), 0.0)
    a = np.abs(v)
    return np.abs(a - (np.floor(a) + 0.5)) < band


def repacked_size(N: int, K: int) -> int:
    """Bytes of the repacked weights: N rows x ceil(K/256) blocks x 128."""
    return N * ((K // 2 + 127) // 128) * 128


def repack_weight(qw: np.ndarray, K: int) -> np.ndarray:
    """Canonical packed weights [N][K/2] -> the block-major layout (flat
    uint8 of repacked_size bytes): 128-byte column block b of every row,
    rows in order, before block b + 1; a short last block is zero-padded."""
    qw = np.ascontiguousarray(qw, dtype=np.uint8)
    N = qw.shape[0]
    rep = np.empty(repacked_size(N, K), dtype=np.uint8)
    _check(lib().oracle_repack_weight(_ptr(qw), N, K, _ptr(rep)), "repack_weight")
    return rep


def unpack_weight(rep: np.ndarray, N: int, K: int) -> np.ndarray:
    """The inverse of repack_weight: [N][K/2] canonical packed weights."""
    rep = np.ascontiguousarray(rep, dtype=np.uint8).reshape(-1)
    qw = np.empty((N, K // 2), dtype=np.uint8)
    _check(lib().oracle_unpack_weight(_ptr(rep), N, K, _ptr(qw)), "unpack_weight")
    return qw


# --------------------------------------------------------------------------
# The W4A16 variant
# --------------------------------------------------------------------------

def round_bf16(y: np.ndarray) -> np.ndarray:
    """bf16 bits of fp64 values, rounded once to nearest, ties to even."""
    y = np.ascontiguousarray(y, dtype=np.float64)
    out = np.empty(y.shape, dtype=np.uint16)
    _check(lib().oracle_round_bf16(_ptr(y), y.size, _ptr(out)), "round_bf16")
    return out


def w4a16_rotate_act(x_bf16: np.ndarray, group: int) -> np.ndarray:
    """bf16 bits of the rotated rows, each value rounded once."""
    x = np.ascontiguousarray(x_bf16, dtype=np.uint16)
    rows, K = x.shape
    xr = np.empty((rows, K), dtype=np.uint16)
    _check(lib().oracle_w4a16_rotate_act(_ptr(x), rows, K, group, _ptr(xr)), "w4a16_rotate_act")
    return xr


def w4a16_gemm(xr_bf16: np.ndarray, qw: np.ndarray, K: int):
    """(acc, l1, p16) fp64 [M][N]: sum_k xr q, sum_k |xr q|, and the sum of
    |partial sums| at every 16th K position (packed weights)."""
    xr = np.ascontiguousarray(xr_bf16, dtype=np.uint16)
    qw = np.ascontiguousarray(qw, dtype=np.uint8)
    M, N = xr.shape[0], qw.shape[0]
    acc = np.empty((M, N), dtype=np.float64)
    l1 = np.empty((M, N), dtype=np.float64)
    p16 = np.empty((M, N), dtype=np.float64)
    _check(lib().oracle_w4a16_gemm(_ptr(xr), _ptr(qw), M, N, K, _ptr(acc), _ptr(l1), _ptr(p16)),
           "w4a16_gemm")
    return acc, l1, p16


def w4a16_epilogue(acc: np.ndarray, sw: np.ndarray, bias_bf16: np.ndarray | None):
    """(t fp64, y bf16 bits): t = acc sw + b exactly, y = bf16_rne(t)."""
    acc = np.ascontiguousarray(acc, dtype=np.float64)
    sw = np.ascontiguousarray(sw, dtype=np.float32)
    b = None if bias_bf16 is None else np.ascontiguousarray(bias_bf16, dtype=np.uint16)
    M, N = acc.shape
    t = np.empty((M, N), dtype=np.float64)
    y = np.empty((M, N), dtype=np.uint16)
    _check(lib().oracle_w4a16_epilogue(_ptr(acc), _ptr(sw), _ptr(b), M, N, _ptr(t), _ptr(y)),
           "w4a16_epilogue")
    return t, y


def w4a16_linear(x_bf16, qw, sw, bias_bf16, group: int) -> np.ndarray:
    """bf16 bits y [M][N] of the whole W4A16 layer given prepared weights."""
    x = np.ascontiguousarray(x_bf16, dtype=np.uint16)
    qw = np.ascontiguousarray(qw, dtype=np.uint8)
    sw = np.ascontiguousarray(sw, dtype=np.float32)
    b = None if bias_bf16 is None else np.ascontiguousarray(bias_bf16, dtype=np.uint16)
    M, K = x.shape
    N = qw.shape[0]
    y = np.empty((M, N), dtype=np.uint16)
    _check(lib().oracle_w4a16_linear(_ptr(x), _ptr(qw), _ptr(sw), _ptr(b), M, N, K, group,
                                     _ptr(y)), "w4a16_linear")
    return y


def bf16_spacing(y: np.ndarray) -> np.ndarray:
    """Distance between the two bf16 values around |y| (2^-133 below the
    normal range)."""
    a = np.abs(np.asarray(y, dtype=np.float64))
    _, e = np.frexp(a)
    q = np.where(e - 1 < -126, -133, e - 8)
    return np.ldexp(1.0, q)


def bf16_tie_band(y: np.ndarray, band: float = 1e-5) -> np.ndarray:
    """Mask of fp64 values lying within ``band`` x (the row's max |y|) of a
    bf16 rounding midpoint: where two fp32 evaluations of the rotation may
    round to neighbouring bf16 values."""
    y = np.asarray(y, dtype=np.float64)
    a = np.abs(y)
    sp = bf16_spacing(a)
    mid = (np.floor(a / sp) + 0.5) * sp
    amax = a.max(axis=-1, keepdims=True) if a.ndim > 1 else a.max()
    return np.abs(a - mid) <= band * amax


# --------------------------------------------------------------------------
# The NVFP4 variant
# --------------------------------------------------------------------------

def e2m1_round(v: np.ndarray) -> np.ndarray:
    """E2M1 codes (sign bit 3) of fp32 values: nearest, ties to even, saturating."""
    v = np.ascontiguousarray(v, dtype=np.float32)
    out = np.empty(v.shape, dtype=np.uint8)
    _check(lib().oracle_e2m1_round(_ptr(v), v.size, _ptr(out)), "e2m1_round")
    return out


def e4m3_round(v: np.ndarray) -> np.ndarray:
    """Unsigned E4M3 codes of non-negative fp32 values (nearest, ties to even, saturating)."""
    v = np.ascontiguousarray(v, dtype=np.float32)
    out = np.empty(v.shape, dtype=np.uint8)
    _check(lib().oracle_e4m3_round(_ptr(v), v.size, _ptr(out)), "e4m3_round")
    return out


def e2m1_value(c: np.ndarray) -> np.ndarray:
    c = np.ascontiguousarray(c, dtype=np.uint8)
    out = np.empty(c.shape, dtype=np.float64)
    _check(lib().oracle_e2m1_value(_ptr(c), c.size, _ptr(out)), "e2m1_value")
    return out


def e4m3_value(c: np.ndarray) -> np.ndarray:
    c = np.ascontiguousarray(c, dtype=np.uint8)
    out = np.empty(c.shape, dtype=np.float64)
    _check(lib().oracle_e4m3_value(_ptr(c), c.size, _ptr(out)), "e4m3_value")
    return out


def nvfp4_quantize_rows(y: np.ndarray):
    """(codes uint8 [rows][K] one per byte, block scales uint8 [rows][K/16],
    row scales fp32 [rows]) of fp64 rotated rows."""
    y = np.ascontiguousarray(y, dtype=np.float64)
    rows, K = y.shape
    codes = np.empty((rows, K), dtype=np.uint8)
    sf = np.empty((rows, K // 16), dtype=np.uint8)
    sc = np.empty((rows,), dtype=np.float32)
    _check(lib().oracle_nvfp4_quantize_rows(_ptr(y), rows, K, _ptr(codes), _ptr(sf), _ptr(sc)),
           "nvfp4_quantize_rows")
    return codes, sf, sc


def nvfp4_pack(codes: np.ndarray) -> np.ndarray:
    codes = np.ascontiguousarray(codes, dtype=np.uint8)
    rows, K = codes.shape
    p = np.empty((rows, K // 2), dtype=np.uint8)
    _check(lib().oracle_nvfp4_pack(_ptr(codes), rows, K, _ptr(p)), "nvfp4_pack")
    return p


def nvfp4_prepare_rows(x_bf16: np.ndarray, group: int):
    """Rotate, quantise to NVFP4 and pack: (packed codes [rows][K/2], block
    scales row-major [rows][K/16], row scales fp32 [rows])."""
    codes, sf, sc = nvfp4_quantize_rows(rotate(x_bf16, group))
    return nvfp4_pack(codes), sf, sc


def nvfp4_sf_layout(sf: np.ndarray, K: int) -> np.ndarray:
    """Row-major block scales [rows][K/16] -> the boundary's atom layout
    (flat, rows padded to a multiple of 128)."""
    sf = np.ascontiguousarray(sf, dtype=np.uint8)
    rows = sf.shape[0]
    out = np.empty(((rows + 127) // 128) * 128 * (K // 16), dtype=np.uint8)
    _check(lib().oracle_nvfp4_sf_layout(_ptr(sf), rows, K, _ptr(out)), "nvfp4_sf_layout")
    return out


def nvfp4_gemm(qx, sfx, qw, sfw, K: int):
    """(acc, l1, p64) fp64 [M][N] from packed codes and row-major block scales."""
    qx = np.ascontiguousarray(qx, dtype=np.uint8)
    qw = np.ascontiguousarray(qw, dtype=np.uint8)
    sfx = np.ascontiguousarray(sfx, dtype=np.uint8)
    sfw = np.ascontiguousarray(sfw, dtype=np.uint8)
    M, N = qx.shape[0], qw.shape[0]
    acc = np.empty((M, N), dtype=np.float64)
    l1 = np.empty((M, N), dtype=np.float64)
    p64 = np.empty((M, N), dtype=np.float64)
    _check(lib().oracle_nvfp4_gemm(_ptr(qx), _ptr(sfx), _ptr(qw), _ptr(sfw), M, N, K, _ptr(acc),
                                   _ptr(l1), _ptr(p64)), "nvfp4_gemm")
    return acc, l1, p64


def nvfp4_epilogue(acc, sx, sw, bias_bf16):
    """(t fp64, y bf16 bits): t = acc sx sw + b exactly, y = bf16_rne(t)."""
    acc = np.ascontiguousarray(acc, dtype=np.float64)
    sx = np.ascontiguousarray(sx, dtype=np.float32)
    sw = np.ascontiguousarray(sw, dtype=np.float32)
    b = None if bias_bf16 is None else np.ascontiguousarray(bias_bf16, dtype=np.uint16)
    M, N = acc.shape
    t = np.empty((M, N), dtype=np.float64)
    y = np.empty((M, N), dtype=np.uint16)
    _check(lib().oracle_nvfp4_epilogue(_ptr(acc), _ptr(sx), _ptr(sw), _ptr(b), M, N, _ptr(t),
                                       _ptr(y)), "nvfp4_epilogue")
    return t, y
