"""The C ABI library without a GPU: it loads, exports every symbol the header
declares, and rejects bad arguments on the host before touching the device."""
import ctypes
import os
import re

import pytest

import rotated_w4a4_quantized_b200 as cr

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "convrot.h")


@pytest.fixture(scope="module")
def L():
    from rotated_w4a4_quantized_b200 import build
    build.build()
    return cr.lib()


def _declared():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(convrot_[a-z0-9_]+)\s*\(", text)))


def test_header_declares_the_boundary():
    names = _declared()
    for required in ("convrot_quantize_weight", "convrot_prepare_act", "convrot_linear",
                     "convrot_linear_prepared", "convrot_linear_workspace_size",
                     "convrot_debug_rotate_f32", "convrot_debug_gemm_s32",
                     "convrot_status_string", "convrot_check_device_error",
                     "convrot_debug_timeout_probe"):
        assert required in names


def test_library_exports_every_declared_symbol(L):
    for name in _declared():
        assert hasattr(L, name), name


def test_status_strings(L):
    for code in range(9):
        s = L.convrot_status_string(code).decode()
        assert s.startswith("CONVROT_")
    assert L.convrot_status_string(123).decode() == "CONVROT_ERR_UNKNOWN"


def test_workspace_size(L):
    assert cr.convrot_linear_workspace_size(0, 1024) == 0
    assert cr.convrot_linear_workspace_size(3, 1024) == 1536 + 256
    assert cr.convrot_linear_workspace_size(1, 64) == 256 + 256
    # the few-token GEMM (M <= 128) never splits K: codes and scales only
    assert cr.convrot_linear_workspace_size(128, 1024) == 128 * 512 + 512
    # beyond it the split area follows the codes and scales
    assert cr.convrot_linear_workspace_size(129, 1024) == 129 * 512 + 768 + cr.SPLIT_AREA_BYTES
    assert (cr.convrot_linear_workspace_size(1024, 3072)
            == 1024 * 1536 + 4096 + cr.SPLIT_AREA_BYTES)


def test_split_area_constants_match_the_header():
    text = open(HEADER).read()
    counters = int(re.search(r"#define CONVROT_SPLIT_COUNTER_BYTES \(\(size_t\)(\d+)\)", text).group(1))
    m = re.search(r"#define CONVROT_SPLIT_AREA_BYTES \(CONVROT_SPLIT_COUNTER_BYTES \+ "
                  r"\(size_t\)(\d+) \* (\d+) \* (\d+) \* (\d+)\)", text)
    slots, rows, cols, word = map(int, m.groups())
    assert counters == cr.SPLIT_COUNTER_BYTES
    assert counters + slots * rows * cols * word == cr.SPLIT_AREA_BYTES
    # one counter per split tile, CTA and epilogue warp (8): a wave of 148
    # CTAs fits, and so does one wave of 128 x 256 int32 partial slots
    assert counters // 4 >= 148 * 8
    assert slots >= 148 and rows * cols * word == 128 * 256 * 4


A = ctypes.c_void_p(0x10000)    # fake, aligned, never dereferenced: checks fail first
B = ctypes.c_void_p(0x20000)
U = ctypes.c_void_p(0x20008)    # 8-byte aligned only


def test_host_validation_without_device(L):
    s = None
    # group / shape
    assert L.convrot_quantize_weight(A, 4, 1024, 128, B, B, s) == 2
    assert L.convrot_quantize_weight(A, 4, 1000, 64, B, B, s) == 3
    assert L.convrot_quantize_weight(A, 4, 32768 + 256, 256, B, B, s) == 3
    assert L.convrot_quantize_weight(A, -1, 1024, 64, B, B, s) == 3
    assert L.convrot_prepare_act(A, 4, 64, 256, B, B, s) == 3      # K % group
    # empty work is a no-op, even with NULL pointers
    assert L.convrot_prepare_act(None, 0, 1024, 64, None, None, s) == 0
    assert L.convrot_linear(None, None, None, None, 0, 8, 1024, 64, None, 0, None, s) == 0
    # NULL and alignment
    assert L.convrot_prepare_act(None, 4, 1024, 64, B, B, s) == 1
    assert L.convrot_prepare_act(U, 4, 1024, 64, B, B, s) == 4
    ws = cr.convrot_linear_workspace_size(4, 1024)
    assert L.convrot_linear(A, B, B, None, 4, 8, 1024, 64, A, ws - 1, B, s) == 5
    assert L.convrot_linear(A, B, B, None, 4, 8, 1024, 64, U, ws, B, s) == 5
    assert L.convrot_linear(A, B, U, None, 4, 8, 1024, 64, A, ws, B, s) == 4
    assert L.convrot_linear(A, B, B, U, 4, 8, 1024, 64, A, ws, B, s) == 4
    assert L.convrot_linear_prepared(A, B, A, B, None, 4, 8, 1000, B, s) == 3
    assert L.convrot_linear_prepared(None, B, A, B, None, 4, 8, 1024, B, s) == 1
    assert L.convrot_debug_gemm_s32(A, B, 4, 8, 96, B, s) == 3
    assert L.convrot_debug_gemm_s32(A, B, 4, 8, 128, U, s) == 4
    assert L.convrot_debug_rotate_f32(A, 4, 512, 256, None, s) == 1
    # forced tile shapes: only 0..7, and the same argument checks
    assert L.convrot_debug_gemm_tiles(A, B, A, B, None, 4, 8, 128, 8, 0, B, s) == 3
    assert L.convrot_debug_gemm_tiles(A, B, A, B, None, 4, 8, 128, -1, 1, B, s) == 3
    assert L.convrot_debug_gemm_tiles(A, B, A, B, None, 4, 8, 96, 2, 1, B, s) == 3
    assert L.convrot_debug_gemm_tiles(A, None, A, B, None, 4, 8, 128, 2, 0, B, s) == 1
    assert L.convrot_debug_gemm_tiles(A, None, A, None, None, 4, 8, 128, 3, 1, U, s) == 4
    assert L.convrot_debug_gemm_tiles(A, B, A, B, U, 4, 8, 128, 1, 0, B, s) == 4
    assert L.convrot_debug_gemm_tiles(None, None, None, None, None, 0, 8, 128, 3, 1, None, s) == 0
    # split K: the area is checked before anything else of the call
    area = cr.SPLIT_AREA_BYTES
    assert L.convrot_linear_prepared_split(A, B, A, B, None, 400, 8, 1024, B, area - 1, B, s) == 5
    assert L.convrot_linear_prepared_split(A, B, A, B, None, 400, 8, 1024, U, area, B, s) == 5
    assert L.convrot_linear_prepared_split(A, B, A, B, None, 400, 8, 1000, B, area, B, s) == 3
    # forced plans: token-major forms and M > 128 only, a split count of 2 or
    # more, the area present and holding its counters
    g = L.convrot_debug_gemm_split
    assert g(A, B, A, B, None, 400, 8, 1024, 4, 1, 2, B, area, 0, B, s) == 3      # few-token form
    assert g(A, B, A, B, None, 400, 8, 1024, 7, 1, 2, B, area, 0, B, s) == 3
    assert g(A, B, A, B, None, 128, 8, 1024, 3, 1, 2, B, area, 0, B, s) == 3      # M <= 128
    assert g(A, B, A, B, None, 400, 8, 1024, 3, 1, 1, B, area, 0, B, s) == 3      # splits < 2
    assert g(A, B, A, B, None, 400, 8, 1024, 3, -2, 2, B, area, 0, B, s) == 3
    assert g(A, B, A, B, None, 400, 8, 1024, 3, 1, 2, None, area, 0, B, s) == 1
    assert g(A, B, A, B, None, 400, 8, 1024, 3, 1, 2, B, 8191, 0, B, s) == 5
    assert g(A, B, A, B, None, 400, 8, 1024, 3, 1, 2, U, area, 0, B, s) == 5
    assert g(A, B, A, B, None, 400, 8, 1024, 3, 1, 2, B, area, 0, U, s) == 4
    assert g(A, B, A, B, None, 400, 0, 1024, 3, 1, 2, None, 0, 0, None, s) == 0  # empty


def test_single_kernel_rule(L):
    # one kernel for 1..4 tokens when K is a multiple of 2048 up to 16384 and
    # the token rows' buffers (1 + 2 bytes per element for group 64, 1 + 4 for
    # group 256, for 1, 2 or 4 rows) fit beside two 64 KB ring slots
    assert L.convrot_linear_single_kernel(1, 4096, 64) == 1
    assert L.convrot_linear_single_kernel(4, 4096, 256) == 1
    assert L.convrot_linear_single_kernel(2, 8192, 64) == 1
    assert L.convrot_linear_single_kernel(1, 16384, 256) == 1
    assert L.convrot_linear_single_kernel(2, 12288, 64) == 1     # two rounds of 192 threads
    assert L.convrot_linear_single_kernel(2, 14336, 64) == 1
    assert L.convrot_linear_single_kernel(4, 6144, 64) == 1      # two rounds of 2 x 96 threads
    assert L.convrot_linear_single_kernel(3, 8192, 64) == 0      # 4 x 24 KB of rows
    assert L.convrot_linear_single_kernel(2, 16384, 64) == 0
    assert L.convrot_linear_single_kernel(4, 8192, 256) == 0
    assert L.convrot_linear_single_kernel(1, 18432, 64) == 0     # > 256 threads per row
    assert L.convrot_linear_single_kernel(5, 4096, 64) == 0
    assert L.convrot_linear_single_kernel(0, 4096, 64) == 0
    assert L.convrot_linear_single_kernel(1, 3072, 64) == 0      # K % 2048
    assert L.convrot_linear_single_kernel(1, 4096, 128) == 0     # bad group


def test_valid_call_without_gpu_reports_cuda_error(L):
    import torch
    if torch.cuda.is_available():
        pytest.skip("a GPU is present")
    # Arguments pass validation; the device set-up then fails cleanly.
    assert L.convrot_prepare_act(A, 4, 1024, 64, B, B, None) == 6
    # a workspace without the split area is accepted (the call runs unsplit);
    # one byte less than the codes and scales is not
    base = cr.convrot_linear_workspace_size(200, 1024) - cr.SPLIT_AREA_BYTES
    assert L.convrot_linear(A, B, B, None, 200, 8, 1024, 64, A, base, B, None) == 6
    assert L.convrot_linear(A, B, B, None, 200, 8, 1024, 64, A, base - 1, B, None) == 5


# ---------------------------------------------------------------- W4A16 library

HEADER_W4A16 = os.path.join(ROOT, "include", "convrot_w4a16.h")


@pytest.fixture(scope="module")
def L16():
    from rotated_w4a4_quantized_b200 import build
    build.build()
    return cr.lib_w4a16()


def _declared_w4a16():
    text = open(HEADER_W4A16).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(convrot_w4a16_[a-z0-9_]+)\s*\(", text)))


def test_w4a16_header_declares_the_boundary():
    assert _declared_w4a16() == sorted([
        "convrot_w4a16_prepare_act", "convrot_w4a16_workspace_size",
        "convrot_w4a16_linear_prepared", "convrot_w4a16_linear",
        "convrot_w4a16_check_device_error", "convrot_w4a16_linear_repacked",
        "convrot_w4a16_linear_prepared_repacked", "convrot_w4a16_debug_gemm_form"])


def test_w4a16_library_exports_every_declared_symbol(L16):
    for name in _declared_w4a16():
        assert hasattr(L16, name), name


def test_w4a16_workspace_size(L16):
    assert cr.convrot_w4a16_workspace_size(0, 1024) == 0
    assert cr.convrot_w4a16_workspace_size(3, 1024) == 6144
    assert cr.convrot_w4a16_workspace_size(1, 64) == 256
    assert cr.convrot_w4a16_workspace_size(5, 192) == 2048


def test_w4a16_host_validation_without_device(L16):
    s = None
    assert L16.convrot_w4a16_prepare_act(A, 4, 1024, 128, B, s) == 2     # group
    assert L16.convrot_w4a16_prepare_act(A, 4, 1000, 64, B, s) == 3      # K % group
    assert L16.convrot_w4a16_prepare_act(A, 4, 64, 256, B, s) == 3
    assert L16.convrot_w4a16_prepare_act(None, 0, 1024, 64, None, s) == 0
    assert L16.convrot_w4a16_prepare_act(None, 4, 1024, 64, B, s) == 1
    assert L16.convrot_w4a16_prepare_act(U, 4, 1024, 64, B, s) == 4
    # prepared GEMM: K % 64, K range, sizes, NULL, alignment
    assert L16.convrot_w4a16_linear_prepared(A, B, B, None, 4, 8, 96, B, s) == 3
    assert L16.convrot_w4a16_linear_prepared(A, B, B, None, 4, 8, 32768 + 64, B, s) == 3
    assert L16.convrot_w4a16_linear_prepared(A, B, B, None, -1, 8, 1024, B, s) == 3
    assert L16.convrot_w4a16_linear_prepared(None, None, None, None, 0, 8, 1024, None, s) == 0
    assert L16.convrot_w4a16_linear_prepared(A, None, B, None, 4, 8, 1024, B, s) == 1
    assert L16.convrot_w4a16_linear_prepared(A, B, B, U, 4, 8, 1024, B, s) == 4
    assert L16.convrot_w4a16_linear_prepared(A, B, U, None, 4, 8, 1024, B, s) == 4
    # whole layer: workspace size and alignment
    ws = cr.convrot_w4a16_workspace_size(4, 1024)
    assert L16.convrot_w4a16_linear(A, B, B, None, 4, 8, 1024, 64, A, ws - 1, B, s) == 5
    assert L16.convrot_w4a16_linear(A, B, B, None, 4, 8, 1024, 64, U, ws, B, s) == 5
    assert L16.convrot_w4a16_linear(A, B, B, None, 4, 8, 1024, 32, A, ws, B, s) == 2
    assert L16.convrot_w4a16_linear(None, None, None, None, 4, 0, 1024, 64, None, 0, None, s) == 0
    # forced GEMM forms: 0..3 (| repacked), the few-token forms up to 64 tokens
    f = L16.convrot_w4a16_debug_gemm_form
    assert f(A, B, B, None, 4, 8, 1024, 4, B, s) == 3
    assert f(A, B, B, None, 4, 8, 1024, -1, B, s) == 3
    assert f(A, B, B, None, 65, 8, 1024, 2, B, s) == 3
    assert f(A, B, B, None, 65, 8, 1024, 3 | 0x100, B, s) == 3
    assert f(A, B, B, None, 4, 8, 96, 3, B, s) == 3                    # K % 64
    assert f(A, None, B, None, 4, 8, 1024, 3, B, s) == 1
    assert f(A, B, B, U, 4, 8, 1024, 3, B, s) == 4


def test_w4a16_valid_call_without_gpu_reports_cuda_error(L16):
    import torch
    if torch.cuda.is_available():
        pytest.skip("a GPU is present")
    assert L16.convrot_w4a16_prepare_act(A, 4, 1024, 64, B, None) == 6


@pytest.mark.parametrize("attr,loader", [("LIB_PATH", "lib"), ("LIB_W4A16_PATH", "lib_w4a16")])
def test_missing_library_raises_instead_of_falling_back(monkeypatch, tmp_path, attr, loader):
    """Without the built CUDA library every op fails loudly: there is no CPU
    path to fall back to."""
    monkeypatch.setattr(cr, attr, str(tmp_path / "absent.so"))
    monkeypatch.setattr(cr, "_lib" if loader == "lib" else "_lib_w4a16", None)
    with pytest.raises(RuntimeError, match="no fallback"):
        getattr(cr, loader)()


def test_status_strings_cover_every_code(L):
    for code in range(12):
        assert L.convrot_status_string(code).decode().startswith("CONVROT_")
    assert L.convrot_status_string(11).decode().startswith("CONVROT_ERR_OVERLAP")


def test_repacked_size_and_host_checks(L):
    assert cr.convrot_repacked_weight_size(3, 512) == 3 * 2 * 128
    assert cr.convrot_repacked_weight_size(5, 320) == 5 * 2 * 128     # short last block padded
    assert cr.convrot_repacked_weight_size(0, 512) == 0
    f = L.convrot_repack_weight
    assert f(A, 4, 100, B, None) == 3          # K not a multiple of 64
    assert f(A, -1, 512, B, None) == 3
    assert f(None, 4, 512, B, None) == 1
    assert f(A, 4, 512, U, None) == 4          # misaligned output
    assert f(A, 4, 512, A, None) == 11         # the same buffer
    assert f(A, 4, 512, ctypes.c_void_p(0x10000 + 512), None) == 11   # overlapping tails
    assert L.convrot_unpack_weight(A, 4, 512, A, None) == 11
    assert f(A, 0, 512, B, None) == 0          # nothing to do


HEADER_NVFP4 = os.path.join(ROOT, "include", "convrot_nvfp4.h")


def test_nvfp4_library_exports_every_declared_symbol():
    from rotated_w4a4_quantized_b200 import build
    build.build()
    text = re.sub(r"/\*.*?\*/", "", open(HEADER_NVFP4).read(), flags=re.S)
    names = sorted(set(re.findall(r"\b(convrot_nvfp4_[a-z0-9_]+)\s*\(", text)))
    assert names == sorted(["convrot_nvfp4_scale_bytes", "convrot_nvfp4_quantize",
                            "convrot_nvfp4_workspace_size", "convrot_nvfp4_linear_prepared",
                            "convrot_nvfp4_linear", "convrot_nvfp4_check_device_error",
                            "convrot_nvfp4_debug_gemm_form"])
    L = cr.lib_nvfp4()
    for name in names:
        assert hasattr(L, name), name
    assert cr.convrot_nvfp4_scale_bytes(200, 192) == 256 * 12
    assert cr.convrot_nvfp4_scale_bytes(0, 192) == 0
    assert cr.convrot_nvfp4_workspace_size(3, 1024) == 1536 + 128 * 64 + 256
    # host-side validation before any device work
    A, B = ctypes.c_void_p(0x10000), ctypes.c_void_p(0x20000)
    assert L.convrot_nvfp4_quantize(A, 4, 100, 64, B, B, B, None) == 3     # K % 64
    assert L.convrot_nvfp4_quantize(A, 4, 1024, 32, B, B, B, None) == 2    # group
    assert L.convrot_nvfp4_quantize(None, 4, 1024, 64, B, B, B, None) == 1
    assert L.convrot_nvfp4_linear_prepared(A, A, A, A, A, A, None, 4, 4, 100, B, None) == 3
    assert L.convrot_nvfp4_linear(A, A, A, A, None, 4, 4, 1024, 64, B, 16, B, None) == 5
    # forced tile widths: forms 0..2 only; the shape checks as for the product
    f = L.convrot_nvfp4_debug_gemm_form
    assert f(A, A, A, A, A, A, None, 4, 4, 1024, 3, B, None) == 3
    assert f(A, A, A, A, A, A, None, 4, 4, 1024, -1, B, None) == 3
    assert f(A, A, A, A, A, A, None, 4, 4, 100, 1, B, None) == 3      # K % 64
    assert f(None, A, A, A, A, A, None, 4, 4, 1024, 2, B, None) == 1
    assert f(A, A, A, A, A, A, None, 0, 4, 1024, 2, B, None) == 0     # no tokens: nothing to do
