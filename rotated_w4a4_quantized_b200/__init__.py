"""B200-native rotated W4A4 (ConvRot-style) linear layer.

A thin ctypes binding over the C ABI in ``include/convrot.h`` (the library
``libconvrot.so`` built in this directory by ``build.py``).  Every step of the
layer runs in that library's CUDA kernels; this module only marshals torch
tensors (device memory and the current stream) into pointers and sizes and
turns status codes into exceptions.  There is no CPU fallback: if the
library is missing, importing the ops raises.

Names follow the C ABI: ``convrot_quantize_weight``, ``convrot_prepare_act``,
``convrot_linear``, ``convrot_linear_prepared`` (plus the test hooks), and for
the W4A16 variant (``include/convrot_w4a16.h``, library
``libconvrot_w4a16.so``) ``convrot_w4a16_prepare_act``,
``convrot_w4a16_linear`` and ``convrot_w4a16_linear_prepared``, and for the
NVFP4 variant (``include/convrot_nvfp4.h``, library ``libconvrot_nvfp4.so``)
``convrot_nvfp4_quantize``, ``convrot_nvfp4_linear`` and
``convrot_nvfp4_linear_prepared``.
"""
from __future__ import annotations

import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libconvrot.so")
LIB_W4A16_PATH = os.path.join(_HERE, "libconvrot_w4a16.so")
LIB_NVFP4_PATH = os.path.join(_HERE, "libconvrot_nvfp4.so")

STATUS = {
    0: "CONVROT_OK", 1: "CONVROT_ERR_NULL", 2: "CONVROT_ERR_GROUP", 3: "CONVROT_ERR_SHAPE",
    4: "CONVROT_ERR_ALIGN", 5: "CONVROT_ERR_WORKSPACE", 6: "CONVROT_ERR_CUDA",
    7: "CONVROT_ERR_DEVICE_TIMEOUT", 8: "CONVROT_ERR_UNSUPPORTED", 9: "CONVROT_ERR_SCRATCH_LIMIT",
    10: "CONVROT_ERR_NOT_DEVICE", 11: "CONVROT_ERR_OVERLAP",
}
MAX_K = 32768


class ConvRotError(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        super().__init__(f"{what}: {STATUS.get(status, status)}")


_lib = None


def lib() -> ctypes.CDLL:
    """The loaded CUDA library; raises if it has not been built."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(
                f"{LIB_PATH} is missing: build it with `python -m rotated_w4a4_quantized_b200.build` "
                "(there is no fallback path)")
        L = ctypes.CDLL(LIB_PATH)
        P, I64, I, SZ = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int, ctypes.c_size_t
        sigs = {
            "convrot_quantize_weight": [P, I64, I64, I, P, P, P],
            "convrot_prepare_act": [P, I64, I64, I, P, P, P],
            "convrot_linear": [P, P, P, P, I64, I64, I64, I, P, SZ, P, P],
            "convrot_linear_prepared": [P, P, P, P, P, I64, I64, I64, P, P],
            "convrot_debug_rotate_f32": [P, I64, I64, I, P, P],
            "convrot_debug_gemm_s32": [P, P, I64, I64, I64, P, P],
            "convrot_check_device_error": [P],
            "convrot_debug_timeout_probe": [I64, P],
            "convrot_linear_noalloc": [P, P, P, P, I64, I64, I64, I, P, P],
            "convrot_debug_gemm_tiles": [P, P, P, P, P, I64, I64, I64, I, I, P, P],
            "convrot_repack_weight": [P, I64, I64, P, P],
            "convrot_unpack_weight": [P, I64, I64, P, P],
            "convrot_linear_repacked": [P, P, P, P, I64, I64, I64, I, P, SZ, P, P],
            "convrot_linear_prepared_repacked": [P, P, P, P, P, I64, I64, I64, P, P],
            "convrot_linear_prepared_split": [P, P, P, P, P, I64, I64, I64, P, SZ, P, P],
            "convrot_debug_gemm_split": [P, P, P, P, P, I64, I64, I64, I, I, I, P, SZ, I, P, P],
            "convrot_debug_gemm_plan": [I64, I64, I64, I, I, SZ, P, P, P],
        }
        for name, args in sigs.items():
            f = getattr(L, name)
            f.argtypes = args
            f.restype = ctypes.c_int
        L.convrot_linear_single_kernel.argtypes = [I64, I64, I]
        L.convrot_linear_single_kernel.restype = I
        L.convrot_linear_workspace_size.argtypes = [I64, I64]
        L.convrot_linear_workspace_size.restype = SZ
        L.convrot_repacked_weight_size.argtypes = [I64, I64]
        L.convrot_repacked_weight_size.restype = SZ
        L.convrot_status_string.argtypes = [I]
        L.convrot_status_string.restype = ctypes.c_char_p
        _lib = L
    return _lib


def _p(t: torch.Tensor | None):
    if t is None:
        return None
    return ctypes.c_void_p(t.data_ptr())


def _stream(stream=None):
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def _check(rc: int, what: str):
    if rc != 0:
        raise ConvRotError(rc, what)


def _need(t, dtype, name: str, shape=None, like=None):
    """Argument checks before any pointer reaches the library: a contiguous
    CUDA tensor of `dtype`, on `like`'s device when given, of `shape` when
    given (None entries match any size)."""
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor, not {type(t).__name__}")
    if not t.is_cuda or t.dtype != dtype or not t.is_contiguous():
        raise ValueError(f"{name} must be a contiguous CUDA {dtype} tensor "
                         f"(got {t.dtype} on {t.device}, contiguous={t.is_contiguous()})")
    if like is not None and t.device != like.device:
        raise ValueError(f"{name} is on {t.device}, the other operands on {like.device}")
    if shape is not None:
        if t.dim() != len(shape) or any(w is not None and int(d) != int(w)
                                        for d, w in zip(t.shape, shape)):
            want = tuple("*" if w is None else int(w) for w in shape)
            raise ValueError(f"{name} has shape {tuple(t.shape)}, expected {want}")
    return t


def _need_opt(t, dtype, name: str, shape=None, like=None):
    return None if t is None else _need(t, dtype, name, shape, like)


def _weights(qw, sw, bias, K: int, like):
    """Packed weights [N, K/2] uint8, scales [N] fp32, bias [N] bf16 or None."""
    _need(qw, torch.uint8, "qw", (None, K // 2), like)
    N = qw.shape[0]
    _need(sw, torch.float32, "sw", (N,), like)
    _need_opt(bias, torch.bfloat16, "bias", (N,), like)
    return N


def _rows(x, dtype, name):
    _need(x, dtype, name, (None, None))
    return x.shape


# ---------------------------------------------------------------------------
# the C ABI, one wrapper each; each call runs on its operands' device
# ---------------------------------------------------------------------------

def convrot_quantize_weight(w: torch.Tensor, group: int, qw=None, sw=None, stream=None):
    """bf16 [N, K] -> (packed codes uint8 [N, K/2], fp32 scales [N])."""
    N, K = _rows(w, torch.bfloat16, "w")
    with torch.cuda.device(w.device):
        qw = torch.empty(N, K // 2, dtype=torch.uint8, device=w.device) if qw is None else qw
        sw = torch.empty(N, dtype=torch.float32, device=w.device) if sw is None else sw
        _need(qw, torch.uint8, "qw", (N, K // 2), w)
        _need(sw, torch.float32, "sw", (N,), w)
        _check(lib().convrot_quantize_weight(_p(w), N, K, group, _p(qw), _p(sw), _stream(stream)),
               "convrot_quantize_weight")
    return qw, sw


def convrot_prepare_act(x: torch.Tensor, group: int, qx=None, sx=None, stream=None):
    """bf16 [M, K] -> (packed codes uint8 [M, K/2], fp32 scales [M])."""
    M, K = _rows(x, torch.bfloat16, "x")
    with torch.cuda.device(x.device):
        qx = torch.empty(M, K // 2, dtype=torch.uint8, device=x.device) if qx is None else qx
        sx = torch.empty(M, dtype=torch.float32, device=x.device) if sx is None else sx
        _need(qx, torch.uint8, "qx", (M, K // 2), x)
        _need(sx, torch.float32, "sx", (M,), x)
        _check(lib().convrot_prepare_act(_p(x), M, K, group, _p(qx), _p(sx), _stream(stream)),
               "convrot_prepare_act")
    return qx, sx


def convrot_linear_single_kernel(M: int, K: int, group: int) -> bool:
    """True when convrot_linear runs this shape as one kernel (1..4 tokens)."""
    return bool(lib().convrot_linear_single_kernel(M, K, group))


def convrot_linear_workspace_size(M: int, K: int) -> int:
    return int(lib().convrot_linear_workspace_size(M, K))


def _base_workspace(M: int, need: int) -> int:
    # the codes and scales alone: a workspace without the split area runs
    # the layer unsplit, with the same results
    return need - SPLIT_AREA_BYTES if M > 128 and need else need


def convrot_linear(x, qw, sw, bias, group: int, workspace=None, out=None, stream=None):
    """The whole layer: bf16 x [M, K] -> bf16 y [M, N]."""
    M, K = _rows(x, torch.bfloat16, "x")
    N = _weights(qw, sw, bias, K, x)
    with torch.cuda.device(x.device):
        need = convrot_linear_workspace_size(M, K)
        if workspace is None:
            workspace = torch.empty(max(1, need), dtype=torch.uint8, device=x.device)
        _need(workspace, torch.uint8, "workspace", None, x)
        if workspace.numel() < _base_workspace(M, need):
            raise ValueError(f"workspace holds {workspace.numel()} bytes, {need} needed "
                             f"({_base_workspace(M, need)} without split K)")
        out = torch.empty(M, N, dtype=torch.bfloat16, device=x.device) if out is None else out
        _need(out, torch.bfloat16, "out", (M, N), x)
        _check(lib().convrot_linear(_p(x), _p(qw), _p(sw), _p(bias), M, N, K, group,
                                    _p(workspace), workspace.numel(), _p(out), _stream(stream)),
               "convrot_linear")
    return out


# ---------------------------------------------------------------------------
# the reversible weight repack (block-major layout, include/convrot.h)
# ---------------------------------------------------------------------------

def convrot_repacked_weight_size(N: int, K: int) -> int:
    return int(lib().convrot_repacked_weight_size(N, K))


def convrot_repack_weight(qw, out=None, stream=None):
    """Packed weights uint8 [N, K/2] -> the block-major repacked layout (a
    flat uint8 tensor of convrot_repacked_weight_size(N, K) bytes)."""
    N, half = _rows(qw, torch.uint8, "qw")
    K = 2 * half
    with torch.cuda.device(qw.device):
        size = convrot_repacked_weight_size(N, K)
        out = torch.empty(size, dtype=torch.uint8, device=qw.device) if out is None else out
        _need(out, torch.uint8, "out", (size,), qw)
        _check(lib().convrot_repack_weight(_p(qw), N, K, _p(out), _stream(stream)),
               "convrot_repack_weight")
    return out


def convrot_unpack_weight(qw_rep, N: int, K: int, out=None, stream=None):
    """The exact inverse of convrot_repack_weight -> uint8 [N, K/2]."""
    _need(qw_rep, torch.uint8, "qw_rep", (convrot_repacked_weight_size(N, K),))
    with torch.cuda.device(qw_rep.device):
        out = torch.empty(N, K // 2, dtype=torch.uint8, device=qw_rep.device) if out is None else out
        _need(out, torch.uint8, "out", (N, K // 2), qw_rep)
        _check(lib().convrot_unpack_weight(_p(qw_rep), N, K, _p(out), _stream(stream)),
               "convrot_unpack_weight")
    return out


def _weights_rep(qw_rep, sw, bias, K: int, like):
    """Repacked weights (flat, sized for N = len(sw) rows), scales, bias."""
    _need(sw, torch.float32, "sw", (None,), like)
    N = sw.shape[0]
    _need(qw_rep, torch.uint8, "qw_rep", (convrot_repacked_weight_size(N, K),), like)
    _need_opt(bias, torch.bfloat16, "bias", (N,), like)
    return N


def convrot_linear_repacked(x, qw_rep, sw, bias, group: int, workspace=None, out=None,
                            stream=None):
    """convrot_linear with the weights in the repacked layout."""
    M, K = _rows(x, torch.bfloat16, "x")
    N = _weights_rep(qw_rep, sw, bias, K, x)
    with torch.cuda.device(x.device):
        need = convrot_linear_workspace_size(M, K)
        if workspace is None:
            workspace = torch.empty(max(1, need), dtype=torch.uint8, device=x.device)
        _need(workspace, torch.uint8, "workspace", None, x)
        if workspace.numel() < _base_workspace(M, need):
            raise ValueError(f"workspace holds {workspace.numel()} bytes, {need} needed "
                             f"({_base_workspace(M, need)} without split K)")
        out = torch.empty(M, N, dtype=torch.bfloat16, device=x.device) if out is None else out
        _need(out, torch.bfloat16, "out", (M, N), x)
        _check(lib().convrot_linear_repacked(_p(x), _p(qw_rep), _p(sw), _p(bias), M, N, K, group,
                                             _p(workspace), workspace.numel(), _p(out),
                                             _stream(stream)), "convrot_linear_repacked")
    return out


def convrot_linear_prepared_repacked(qx, sx, qw_rep, sw, bias, K: int, out=None, stream=None):
    """convrot_linear_prepared with the weights in the repacked layout."""
    M = _prepared(qx, sx, K)
    _need(sx, torch.float32, "sx", (M,), qx)
    N = _weights_rep(qw_rep, sw, bias, K, qx)
    with torch.cuda.device(qx.device):
        out = torch.empty(M, N, dtype=torch.bfloat16, device=qx.device) if out is None else out
        _need(out, torch.bfloat16, "out", (M, N), qx)
        _check(lib().convrot_linear_prepared_repacked(_p(qx), _p(sx), _p(qw_rep), _p(sw), _p(bias),
                                                      M, N, K, _p(out), _stream(stream)),
               "convrot_linear_prepared_repacked")
    return out


def convrot_linear_noalloc(x, qw, sw, bias, group: int, out=None, stream=None):
    """The whole layer without a caller workspace: the library's fixed
    16 MiB scratch array holds the packed activations instead.  Meant for
    callers that cannot allocate device memory (a plugin whose host runtime
    owns every allocation, or a path that must not call cudaMalloc).  Calls
    that overlap on the GPU share that array and race; order them."""
    M, K = _rows(x, torch.bfloat16, "x")
    N = _weights(qw, sw, bias, K, x)
    with torch.cuda.device(x.device):
        out = torch.empty(M, N, dtype=torch.bfloat16, device=x.device) if out is None else out
        _need(out, torch.bfloat16, "out", (M, N), x)
        _check(lib().convrot_linear_noalloc(_p(x), _p(qw), _p(sw), _p(bias), M, N, K, group,
                                            _p(out), _stream(stream)), "convrot_linear_noalloc")
    return out


def _prepared(qx, sx, K: int):
    _need(qx, torch.uint8, "qx", (None, K // 2))
    M = qx.shape[0]
    _need_opt(sx, torch.float32, "sx", (M,), qx)
    return M


def convrot_linear_prepared(qx, sx, qw, sw, bias, K: int, out=None, stream=None):
    """Steps 3-4 on prepared operands -> bf16 y [M, N]."""
    M = _prepared(qx, sx, K)
    _need(sx, torch.float32, "sx", (M,), qx)
    N = _weights(qw, sw, bias, K, qx)
    with torch.cuda.device(qx.device):
        out = torch.empty(M, N, dtype=torch.bfloat16, device=qx.device) if out is None else out
        _need(out, torch.bfloat16, "out", (M, N), qx)
        _check(lib().convrot_linear_prepared(_p(qx), _p(sx), _p(qw), _p(sw), _p(bias), M, N, K,
                                             _p(out), _stream(stream)), "convrot_linear_prepared")
    return out


# Split-K area (include/convrot.h): counters, then one wave of partial slots.
SPLIT_COUNTER_BYTES = 8192
SPLIT_AREA_BYTES = SPLIT_COUNTER_BYTES + 160 * 128 * 256 * 4


def new_split_area(device) -> torch.Tensor:
    """A split area for convrot_linear_prepared_split: its counters start at
    zero (every call that completes leaves them zero)."""
    a = torch.empty(SPLIT_AREA_BYTES, dtype=torch.uint8, device=device)
    a[:SPLIT_COUNTER_BYTES].zero_()
    return a


def _split_area(area, like):
    if area is None:
        return None, 0
    _need(area, torch.uint8, "split area", None, like)
    if area.numel() < SPLIT_AREA_BYTES or area.data_ptr() % 256:
        raise ValueError("the split area needs SPLIT_AREA_BYTES bytes, 256-byte aligned")
    return _p(area), area.numel()


def convrot_linear_prepared_split(qx, sx, qw, sw, bias, K: int, split_area, out=None,
                                  stream=None):
    """convrot_linear_prepared with a split area (new_split_area), so that
    the GEMM may split K where its last wave is part-filled."""
    M = _prepared(qx, sx, K)
    _need(sx, torch.float32, "sx", (M,), qx)
    N = _weights(qw, sw, bias, K, qx)
    with torch.cuda.device(qx.device):
        pa, na = _split_area(split_area, qx)
        out = torch.empty(M, N, dtype=torch.bfloat16, device=qx.device) if out is None else out
        _need(out, torch.bfloat16, "out", (M, N), qx)
        _check(lib().convrot_linear_prepared_split(_p(qx), _p(sx), _p(qw), _p(sw), _p(bias), M, N,
                                                   K, pa, na, _p(out), _stream(stream)),
               "convrot_linear_prepared_split")
    return out


def convrot_debug_rotate_f32(x, group: int, out=None, stream=None):
    M, K = _rows(x, torch.bfloat16, "x")
    with torch.cuda.device(x.device):
        out = torch.empty(M, K, dtype=torch.float32, device=x.device) if out is None else out
        _need(out, torch.float32, "out", (M, K), x)
        _check(lib().convrot_debug_rotate_f32(_p(x), M, K, group, _p(out), _stream(stream)),
               "convrot_debug_rotate_f32")
    return out


def convrot_debug_gemm_s32(qx, qw, K: int, out=None, stream=None):
    M = _prepared(qx, None, K)
    _need(qw, torch.uint8, "qw", (None, K // 2), qx)
    N = qw.shape[0]
    with torch.cuda.device(qx.device):
        out = torch.empty(M, N, dtype=torch.int32, device=qx.device) if out is None else out
        _need(out, torch.int32, "out", (M, N), qx)
        _check(lib().convrot_debug_gemm_s32(_p(qx), _p(qw), M, N, K, _p(out), _stream(stream)),
               "convrot_debug_gemm_s32")
    return out


# GEMM forms of convrot_debug_gemm_tiles: the token-major tile shapes and the
# three few-token forms (M <= 128)
TILES_AUTO, TILES_128x256, TILES_128x192, TILES_256x192_PAIR = 0, 1, 2, 3
SKINNY_TMEM, SKINNY_SMEM = 4, 5
TILES_256x128_PAIR = 6
SKINNY_PAIR = 7


TILES_REPACKED = 0x100


def convrot_debug_gemm_tiles(qx, sx, qw, sw, bias, K: int, tiles: int, out_s32: bool = False,
                             out=None, stream=None, N: int | None = None):
    """Steps 3-4 (bf16 y) or step 3 alone (int32 acc, out_s32=True) with the
    GEMM forced to one tile shape (TILES_*); tiles | TILES_REPACKED takes
    qw in the repacked layout (a flat tensor; give N then)."""
    M = _prepared(qx, sx, K)
    if tiles & TILES_REPACKED:
        if N is None:
            raise ValueError("N is needed with repacked weights")
        _need(qw, torch.uint8, "qw_rep", (convrot_repacked_weight_size(N, K),), qx)
        if not out_s32:
            _need(sx, torch.float32, "sx", (M,), qx)
            _need(sw, torch.float32, "sw", (N,), qx)
            _need_opt(bias, torch.bfloat16, "bias", (N,), qx)
    elif out_s32:
        _need(qw, torch.uint8, "qw", (None, K // 2), qx)
        N = qw.shape[0]
    else:
        _need(sx, torch.float32, "sx", (M,), qx)
        N = _weights(qw, sw, bias, K, qx)
    dt = torch.int32 if out_s32 else torch.bfloat16
    with torch.cuda.device(qx.device):
        out = torch.empty(M, N, dtype=dt, device=qx.device) if out is None else out
        _need(out, dt, "out", (M, N), qx)
        _check(lib().convrot_debug_gemm_tiles(_p(qx), _p(sx), _p(qw), _p(sw), _p(bias), M, N, K,
                                              int(tiles), int(bool(out_s32)), _p(out),
                                              _stream(stream)), "convrot_debug_gemm_tiles")
    return out


def convrot_check_device_error(stream=None) -> int:
    """Synchronise the stream; return (and clear) the device error status."""
    return int(lib().convrot_check_device_error(_stream(stream)))


def convrot_debug_timeout_probe(timeout_ns: int, stream=None):
    _check(lib().convrot_debug_timeout_probe(int(timeout_ns), _stream(stream)),
           "convrot_debug_timeout_probe")


# ---------------------------------------------------------------------------
# the W4A16 variant (include/convrot_w4a16.h)
# ---------------------------------------------------------------------------

_lib_w4a16 = None


def lib_w4a16() -> ctypes.CDLL:
    """The loaded W4A16 library; raises if it has not been built."""
    global _lib_w4a16
    if _lib_w4a16 is None:
        if not os.path.exists(LIB_W4A16_PATH):
            raise RuntimeError(
                f"{LIB_W4A16_PATH} is missing: build it with "
                "`python -m rotated_w4a4_quantized_b200.build` (there is no fallback path)")
        L = ctypes.CDLL(LIB_W4A16_PATH)
        P, I64, I, SZ = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int, ctypes.c_size_t
        sigs = {
            "convrot_w4a16_prepare_act": [P, I64, I64, I, P, P],
            "convrot_w4a16_linear_prepared": [P, P, P, P, I64, I64, I64, P, P],
            "convrot_w4a16_linear": [P, P, P, P, I64, I64, I64, I, P, SZ, P, P],
            "convrot_w4a16_check_device_error": [P],
            "convrot_w4a16_linear_prepared_repacked": [P, P, P, P, I64, I64, I64, P, P],
            "convrot_w4a16_linear_repacked": [P, P, P, P, I64, I64, I64, I, P, SZ, P, P],
            "convrot_w4a16_debug_gemm_form": [P, P, P, P, I64, I64, I64, I, P, P],
        }
        for name, args in sigs.items():
            f = getattr(L, name)
            f.argtypes = args
            f.restype = ctypes.c_int
        L.convrot_w4a16_workspace_size.argtypes = [I64, I64]
        L.convrot_w4a16_workspace_size.restype = SZ
        _lib_w4a16 = L
    return _lib_w4a16


def convrot_w4a16_prepare_act(x: torch.Tensor, group: int, out=None, stream=None):
    """bf16 x [M, K] -> bf16 xr [M, K]: the rotated rows, each value rounded
    once to bf16 (no quantisation)."""
    M, K = _rows(x, torch.bfloat16, "x")
    with torch.cuda.device(x.device):
        out = torch.empty(M, K, dtype=torch.bfloat16, device=x.device) if out is None else out
        _need(out, torch.bfloat16, "out", (M, K), x)
        _check(lib_w4a16().convrot_w4a16_prepare_act(_p(x), M, K, group, _p(out),
                                                     _stream(stream)),
               "convrot_w4a16_prepare_act")
    return out


def convrot_w4a16_workspace_size(M: int, K: int) -> int:
    return int(lib_w4a16().convrot_w4a16_workspace_size(M, K))


def convrot_w4a16_linear_prepared(xr, qw, sw, bias, out=None, stream=None):
    """bf16 xr [M, K] (rotated) x packed INT4 weights -> bf16 y [M, N]."""
    M, K = _rows(xr, torch.bfloat16, "xr")
    N = _weights(qw, sw, bias, K, xr)
    with torch.cuda.device(xr.device):
        out = torch.empty(M, N, dtype=torch.bfloat16, device=xr.device) if out is None else out
        _need(out, torch.bfloat16, "out", (M, N), xr)
        _check(lib_w4a16().convrot_w4a16_linear_prepared(_p(xr), _p(qw), _p(sw), _p(bias), M, N,
                                                         K, _p(out), _stream(stream)),
               "convrot_w4a16_linear_prepared")
    return out


# GEMM forms of convrot_w4a16_debug_gemm_form: automatic, 128 x 256 tiles,
# few tokens (M <= 64) with the weights widened in shared memory or in TMEM
W4A16_AUTO, W4A16_TILES, W4A16_FEW_SMEM, W4A16_FEW_TMEM = 0, 1, 2, 3


def convrot_w4a16_debug_gemm_form(xr, qw, sw, bias, form: int, out=None, stream=None,
                                  N: int | None = None):
    """convrot_w4a16_linear_prepared with the GEMM forced to one form
    (W4A16_*); form | TILES_REPACKED takes qw in the repacked layout (a flat
    tensor; give N then)."""
    M, K = _rows(xr, torch.bfloat16, "xr")
    if form & TILES_REPACKED:
        if N is None:
            raise ValueError("N is needed with repacked weights")
        _need(qw, torch.uint8, "qw_rep", (convrot_repacked_weight_size(N, K),), xr)
        _need(sw, torch.float32, "sw", (N,), xr)
        _need_opt(bias, torch.bfloat16, "bias", (N,), xr)
    else:
        N = _weights(qw, sw, bias, K, xr)
    with torch.cuda.device(xr.device):
        out = torch.empty(M, N, dtype=torch.bfloat16, device=xr.device) if out is None else out
        _need(out, torch.bfloat16, "out", (M, N), xr)
        _check(lib_w4a16().convrot_w4a16_debug_gemm_form(_p(xr), _p(qw), _p(sw), _p(bias), M, N, K,
                                                         int(form), _p(out), _stream(stream)),
               "convrot_w4a16_debug_gemm_form")
    return out


def convrot_w4a16_linear(x, qw, sw, bias, group: int, workspace=None, out=None, stream=None):
    """The whole W4A16 layer: bf16 x [M, K] -> bf16 y [M, N] (rotation, then
    the bf16 x INT4 tensor-core GEMM with scale and bias)."""
    M, K = _rows(x, torch.bfloat16, "x")
    N = _weights(qw, sw, bias, K, x)
    with torch.cuda.device(x.device):
        need = convrot_w4a16_workspace_size(M, K)
        if workspace is None:
            workspace = torch.empty(max(1, need), dtype=torch.uint8, device=x.device)
        _need(workspace, torch.uint8, "workspace", None, x)
        if workspace.numel() < need:
            raise ValueError(f"workspace holds {workspace.numel()} bytes, {need} needed")
        out = torch.empty(M, N, dtype=torch.bfloat16, device=x.device) if out is None else out
        _need(out, torch.bfloat16, "out", (M, N), x)
        _check(lib_w4a16().convrot_w4a16_linear(_p(x), _p(qw), _p(sw), _p(bias), M, N, K, group,
                                                _p(workspace), workspace.numel(), _p(out),
                                                _stream(stream)), "convrot_w4a16_linear")
    return out


def convrot_w4a16_linear_repacked(x, qw_rep, sw, bias, group: int, workspace=None, out=None,
                                  stream=None):
    """convrot_w4a16_linear with the weights in the repacked layout."""
    M, K = _rows(x, torch.bfloat16, "x")
    N = _weights_rep(qw_rep, sw, bias, K, x)
    with torch.cuda.device(x.device):
        need = convrot_w4a16_workspace_size(M, K)
        if workspace is None:
            workspace = torch.empty(max(1, need), dtype=torch.uint8, device=x.device)
        _need(workspace, torch.uint8, "workspace", None, x)
        if workspace.numel() < need:
            raise ValueError(f"workspace holds {workspace.numel()} bytes, {need} needed")
        out = torch.empty(M, N, dtype=torch.bfloat16, device=x.device) if out is None else out
        _need(out, torch.bfloat16, "out", (M, N), x)
        _check(lib_w4a16().convrot_w4a16_linear_repacked(
            _p(x), _p(qw_rep), _p(sw), _p(bias), M, N, K, group, _p(workspace), workspace.numel(),
            _p(out), _stream(stream)), "convrot_w4a16_linear_repacked")
    return out


def convrot_w4a16_linear_prepared_repacked(xr, qw_rep, sw, bias, out=None, stream=None):
    """convrot_w4a16_linear_prepared with the weights in the repacked layout."""
    M, K = _rows(xr, torch.bfloat16, "xr")
    N = _weights_rep(qw_rep, sw, bias, K, xr)
    with torch.cuda.device(xr.device):
        out = torch.empty(M, N, dtype=torch.bfloat16, device=xr.device) if out is None else out
        _need(out, torch.bfloat16, "out", (M, N), xr)
        _check(lib_w4a16().convrot_w4a16_linear_prepared_repacked(
            _p(xr), _p(qw_rep), _p(sw), _p(bias), M, N, K, _p(out), _stream(stream)),
            "convrot_w4a16_linear_prepared_repacked")
    return out


def convrot_w4a16_check_device_error(stream=None) -> int:
    """Synchronise the stream; return (and clear) the W4A16 library's device
    error status."""
    return int(lib_w4a16().convrot_w4a16_check_device_error(_stream(stream)))


# ---------------------------------------------------------------------------
# the NVFP4 variant (include/convrot_nvfp4.h)
# ---------------------------------------------------------------------------

_lib_nvfp4 = None


def lib_nvfp4() -> ctypes.CDLL:
    """The loaded NVFP4 library; raises if it has not been built."""
    global _lib_nvfp4
    if _lib_nvfp4 is None:
        if not os.path.exists(LIB_NVFP4_PATH):
            raise RuntimeError(
                f"{LIB_NVFP4_PATH} is missing: build it with "
                "`python -m rotated_w4a4_quantized_b200.build` (there is no fallback path)")
        L = ctypes.CDLL(LIB_NVFP4_PATH)
        P, I64, I, SZ = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int, ctypes.c_size_t
        sigs = {
            "convrot_nvfp4_quantize": [P, I64, I64, I, P, P, P, P],
            "convrot_nvfp4_linear_prepared": [P, P, P, P, P, P, P, I64, I64, I64, P, P],
            "convrot_nvfp4_linear": [P, P, P, P, P, I64, I64, I64, I, P, SZ, P, P],
            "convrot_nvfp4_check_device_error": [P],
            "convrot_nvfp4_debug_gemm_form": [P, P, P, P, P, P, P, I64, I64, I64, I, P, P],
        }
        for name, args in sigs.items():
            f = getattr(L, name)
            f.argtypes = args
            f.restype = ctypes.c_int
        for name in ("convrot_nvfp4_scale_bytes", "convrot_nvfp4_workspace_size"):
            getattr(L, name).argtypes = [I64, I64]
            getattr(L, name).restype = SZ
        _lib_nvfp4 = L
    return _lib_nvfp4


def convrot_nvfp4_scale_bytes(rows: int, K: int) -> int:
    return int(lib_nvfp4().convrot_nvfp4_scale_bytes(rows, K))


def convrot_nvfp4_workspace_size(M: int, K: int) -> int:
    return int(lib_nvfp4().convrot_nvfp4_workspace_size(M, K))


def convrot_nvfp4_quantize(x: torch.Tensor, group: int, q=None, sf=None, s=None, stream=None):
    """bf16 [rows, K] -> (E2M1 codes uint8 [rows, K/2], E4M3 block scales
    uint8 [scale_bytes] in the tensor cores' atom layout, fp32 row scales [rows])."""
    rows, K = _rows(x, torch.bfloat16, "x")
    with torch.cuda.device(x.device):
        nsf = convrot_nvfp4_scale_bytes(rows, K)
        q = torch.empty(rows, K // 2, dtype=torch.uint8, device=x.device) if q is None else q
        sf = torch.empty(max(1, nsf), dtype=torch.uint8, device=x.device) if sf is None else sf
        s = torch.empty(rows, dtype=torch.float32, device=x.device) if s is None else s
        _need(q, torch.uint8, "q", (rows, K // 2), x)
        _need(sf, torch.uint8, "sf", (max(1, nsf),), x)
        _need(s, torch.float32, "s", (rows,), x)
        _check(lib_nvfp4().convrot_nvfp4_quantize(_p(x), rows, K, group, _p(q), _p(sf), _p(s),
                                                  _stream(stream)), "convrot_nvfp4_quantize")
    return q, sf, s


def _nvfp4_operand(q, sf, s, K: int, name: str, like=None):
    _need(q, torch.uint8, name, (None, K // 2), like)
    rows = q.shape[0]
    _need(sf, torch.uint8, name + " scales", (convrot_nvfp4_scale_bytes(rows, K),), like)
    _need(s, torch.float32, name + " row scales", (rows,), like)
    return rows


def convrot_nvfp4_linear_prepared(qx, sfx, sx, qw, sfw, sw, bias, K: int, out=None, stream=None):
    """The block-scaled FP4 product on prepared operands -> bf16 y [M, N]."""
    M = _nvfp4_operand(qx, sfx, sx, K, "qx")
    N = _nvfp4_operand(qw, sfw, sw, K, "qw", qx)
    _need_opt(bias, torch.bfloat16, "bias", (N,), qx)
    with torch.cuda.device(qx.device):
        out = torch.empty(M, N, dtype=torch.bfloat16, device=qx.device) if out is None else out
        _need(out, torch.bfloat16, "out", (M, N), qx)
        _check(lib_nvfp4().convrot_nvfp4_linear_prepared(
            _p(qx), _p(sfx), _p(sx), _p(qw), _p(sfw), _p(sw), _p(bias), M, N, K, _p(out),
            _stream(stream)), "convrot_nvfp4_linear_prepared")
    return out


# GEMM forms of convrot_nvfp4_debug_gemm_form: automatic, 256- or 128-wide
# weight tiles
NVFP4_AUTO, NVFP4_TILES_256, NVFP4_TILES_128 = 0, 1, 2


def convrot_nvfp4_debug_gemm_form(qx, sfx, sx, qw, sfw, sw, bias, K: int, form: int, out=None,
                                  stream=None):
    """convrot_nvfp4_linear_prepared with the GEMM's tile width forced
    (NVFP4_*)."""
    M = _nvfp4_operand(qx, sfx, sx, K, "qx")
    N = _nvfp4_operand(qw, sfw, sw, K, "qw", qx)
    _need_opt(bias, torch.bfloat16, "bias", (N,), qx)
    with torch.cuda.device(qx.device):
        out = torch.empty(M, N, dtype=torch.bfloat16, device=qx.device) if out is None else out
        _need(out, torch.bfloat16, "out", (M, N), qx)
        _check(lib_nvfp4().convrot_nvfp4_debug_gemm_form(
            _p(qx), _p(sfx), _p(sx), _p(qw), _p(sfw), _p(sw), _p(bias), M, N, K, int(form),
            _p(out), _stream(stream)), "convrot_nvfp4_debug_gemm_form")
    return out


def convrot_nvfp4_linear(x, qw, sfw, sw, bias, group: int, workspace=None, out=None, stream=None):
    """The whole NVFP4 layer: bf16 x [M, K] -> bf16 y [M, N] (rotation and
    NVFP4 quantisation of x, then the block-scaled FP4 product)."""
    M, K = _rows(x, torch.bfloat16, "x")
    N = _nvfp4_operand(qw, sfw, sw, K, "qw", x)
    _need_opt(bias, torch.bfloat16, "bias", (N,), x)
    with torch.cuda.device(x.device):
        need = convrot_nvfp4_workspace_size(M, K)
        if workspace is None:
            workspace = torch.empty(max(1, need), dtype=torch.uint8, device=x.device)
        _need(workspace, torch.uint8, "workspace", None, x)
        if workspace.numel() < need:
            raise ValueError(f"workspace holds {workspace.numel()} bytes, {need} needed")
        out = torch.empty(M, N, dtype=torch.bfloat16, device=x.device) if out is None else out
        _need(out, torch.bfloat16, "out", (M, N), x)
        _check(lib_nvfp4().convrot_nvfp4_linear(
            _p(x), _p(qw), _p(sfw), _p(sw), _p(bias), M, N, K, group, _p(workspace),
            workspace.numel(), _p(out), _stream(stream)), "convrot_nvfp4_linear")
    return out


def convrot_nvfp4_check_device_error(stream=None) -> int:
    """Synchronise the stream; return (and clear) the NVFP4 library's device
    error status."""
    return int(lib_nvfp4().convrot_nvfp4_check_device_error(_stream(stream)))


class HostPipeline:
    """The layer (or a chain of layers) on pinned host buffers, with the
    copies overlapped with the compute.

    Rows are independent, so the batch is cut into row chunks: chunk i is
    copied host -> device on one stream, run through ``convrot_linear`` for
    each layer on the caller's stream, and copied back on a third stream,
    while chunk i+1 is already being copied in.  The results are identical
    to one whole-batch call.  Device buffers are allocated once here.

    ``layers`` is a list of (qweight, scales, bias or None, group) with each
    layer's in_features equal to the previous layer's out_features.

    With ``graph=True`` the first call runs eagerly and the second call for
    the same host buffers captures the whole multi-stream sequence into one
    CUDA graph, which later calls replay (one launch per call instead of a
    dozen stream operations per chunk).
    """

    def __init__(self, M: int, K: int, layers, chunks: int = 8, device=None, graph: bool = True):
        self.M, self.K, self.layers = M, K, layers
        self.use_graph, self._graph, self._key, self._calls = graph, None, None, 0
        dev = torch.device("cuda") if device is None else torch.device(device)
        widths = [K] + [qw.shape[0] for qw, *_ in layers]
        # chunk rows keep every row slice 16-byte aligned (N % 8 == 0 for all outputs)
        if any(w % 8 for w in widths[1:]):
            chunks = 1
        step = max(1, -(-M // max(1, chunks)))
        self.ranges = [(r, min(M, r + step)) for r in range(0, M, step)]
        self.acts = [torch.empty(M, w, dtype=torch.bfloat16, device=dev) for w in widths]
        self.ws = [torch.empty(max(1, convrot_linear_workspace_size(step, widths[i])),
                               dtype=torch.uint8, device=dev) for i in range(len(layers))]
        self.s_in = torch.cuda.Stream(device=dev)
        self.s_out = torch.cuda.Stream(device=dev)
        n = len(self.ranges)
        self.e_start = torch.cuda.Event()
        self.e_in = [torch.cuda.Event() for _ in range(n)]
        self.e_done = [torch.cuda.Event() for _ in range(n)]
        self.e_out = torch.cuda.Event()

    def __call__(self, x_host: torch.Tensor, y_host: torch.Tensor, stream=None):
        main = torch.cuda.current_stream() if stream is None else stream
        key = (x_host.data_ptr(), y_host.data_ptr())
        if self.use_graph and self._calls >= 1:
            if self._graph is None or self._key != key:
                g = torch.cuda.CUDAGraph()
                with torch.cuda.graph(g):
                    self._enqueue(x_host, y_host, torch.cuda.current_stream())
                self._graph, self._key = g, key
            with torch.cuda.stream(main):
                self._graph.replay()
            return y_host
        self._calls += 1
        return self._enqueue(x_host, y_host, main)

    def _enqueue(self, x_host, y_host, main):
        self.e_start.record(main)
        self.s_in.wait_event(self.e_start)
        self.s_out.wait_event(self.e_start)
        for i, (r0, r1) in enumerate(self.ranges):
            with torch.cuda.stream(self.s_in):
                self.acts[0][r0:r1].copy_(x_host[r0:r1], non_blocking=True)
                self.e_in[i].record(self.s_in)
            main.wait_event(self.e_in[i])
            for l, (qw, sw, b, group) in enumerate(self.layers):
                convrot_linear(self.acts[l][r0:r1], qw, sw, b, group, self.ws[l],
                               out=self.acts[l + 1][r0:r1], stream=main)
            self.e_done[i].record(main)
            self.s_out.wait_event(self.e_done[i])
            with torch.cuda.stream(self.s_out):
                y_host[r0:r1].copy_(self.acts[-1][r0:r1], non_blocking=True)
        self.e_out.record(self.s_out)
        main.wait_event(self.e_out)
        return y_host


class ConvRotLinear:
    """A linear layer held as rotated, row-quantised, packed INT4 weights.

    ``ConvRotLinear.from_dense(weight, bias, group)`` prepares the weights once
    (offline step); calling the layer runs the whole fused path on the current
    stream.  It mirrors the page's ``ConvRotLinear`` / ``quantize_convrot_weight``
    pair ("convrot-mlx" README, "Install and test").
    """

    def __init__(self, qweight, scales, bias, group: int, in_features: int):
        self.qweight, self.scales, self.bias = qweight, scales, bias
        self.group, self.in_features = group, in_features
        self.out_features = qweight.shape[0]
        self._ws = None

    @classmethod
    def from_dense(cls, weight: torch.Tensor, bias: torch.Tensor | None, group: int = 256):
        qw, sw = convrot_quantize_weight(weight.contiguous(), group)
        b = None if bias is None else bias.to(torch.bfloat16).contiguous()
        return cls(qw, sw, b, group, weight.shape[1])

    def __call__(self, x: torch.Tensor) -> torch.Tensor:
        lead = x.shape[:-1]
        x2 = x.reshape(-1, self.in_features).contiguous()
        need = convrot_linear_workspace_size(x2.shape[0], self.in_features)
        if self._ws is None or self._ws.numel() < need or self._ws.device != x2.device:
            self._ws = torch.empty(max(1, need), dtype=torch.uint8, device=x2.device)
        y = convrot_linear(x2, self.qweight, self.scales, self.bias, self.group, self._ws)
        return y.reshape(*lead, self.out_features)


def convrot_debug_gemm_split(qx, sx, qw, sw, bias, K: int, tiles: int, split_tiles: int,
                             splits: int, split_area, out_s32: bool = False, out=None,
                             stream=None, N: int | None = None):
    """convrot_debug_gemm_tiles for a token-major form with a given split-K
    plan: the first split_tiles output tiles cut into `splits` ranges of K
    (split_tiles = 0: none; -1: the planner's choice).  split_area as for
    convrot_linear_prepared_split; tiles | TILES_REPACKED takes qw in the
    repacked layout (a flat tensor; give N then)."""
    M = _prepared(qx, sx, K)
    if tiles & TILES_REPACKED:
        if N is None:
            raise ValueError("N is needed with repacked weights")
        _need(qw, torch.uint8, "qw_rep", (convrot_repacked_weight_size(N, K),), qx)
        if not out_s32:
            _need(sx, torch.float32, "sx", (M,), qx)
            _need(sw, torch.float32, "sw", (N,), qx)
            _need_opt(bias, torch.bfloat16, "bias", (N,), qx)
    elif out_s32:
        _need(qw, torch.uint8, "qw", (None, K // 2), qx)
        N = qw.shape[0]
    else:
        _need(sx, torch.float32, "sx", (M,), qx)
        N = _weights(qw, sw, bias, K, qx)
    dt = torch.int32 if out_s32 else torch.bfloat16
    with torch.cuda.device(qx.device):
        _need(split_area, torch.uint8, "split area", None, qx)
        out = torch.empty(M, N, dtype=dt, device=qx.device) if out is None else out
        _need(out, dt, "out", (M, N), qx)
        _check(lib().convrot_debug_gemm_split(_p(qx), _p(sx), _p(qw), _p(sw), _p(bias), M, N, K,
                                              int(tiles), int(split_tiles), int(splits),
                                              _p(split_area), split_area.numel(),
                                              int(bool(out_s32)), _p(out), _stream(stream)),
               "convrot_debug_gemm_split")
    return out


def convrot_debug_gemm_plan(M: int, N: int, K: int, pairs: int = 74, sms: int = 148,
                            split_bytes: int | None = None):
    """Host-only: the GEMM form (numbered as for convrot_debug_gemm_tiles) and
    split-K plan (split_tiles, splits) convrot_linear takes for (M, N, K) on a
    device with `pairs` CTA pairs and `sms` SMs (a B200: 74 and 148)."""
    t, st, sp = ctypes.c_int(), ctypes.c_int(), ctypes.c_int()
    nb = SPLIT_AREA_BYTES if split_bytes is None else split_bytes
    _check(lib().convrot_debug_gemm_plan(M, N, K, pairs, sms, nb, ctypes.byref(t),
                                         ctypes.byref(st), ctypes.byref(sp)),
           "convrot_debug_gemm_plan")
    return t.value, st.value, sp.value
