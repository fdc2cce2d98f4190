"""C-ABI checks that need no GPU: the library loads, exports every function
declared in include/nvfp4.h, and rejects bad arguments on the host before
anything is enqueued (fake pointers are never dereferenced)."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "nvfp4.h")

OK, INVALID, SHAPE, MISALIGNED, NONFINITE, CUDA, NOTIMPL, TOOLARGE = range(8)


@pytest.fixture(scope="module")
def L():
    from scale_calibration_nvfp4_b200 import build, nvfp4
    build.build()
    return nvfp4.lib()


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(nvfp4_[a-z_0-9]+)\s*\(", text)))


def test_header_declares_the_api():
    names = declared_functions()
    for n in ["nvfp4_global_scale", "nvfp4_hessian_accumulate", "nvfp4_hessian_accumulate_grouped",
              "nvfp4_scale_search_max", "nvfp4_scale_search_mse",
              "nvfp4_scale_search_local_hessian", "nvfp4_quantize_pack", "nvfp4_dequantize",
              "nvfp4_fake_quant", "nvfp4_status_string", "nvfp4_get_device_status",
              "nvfp4_shutdown"]:
        assert n in names


def test_library_exports_every_declared_symbol(L):
    from scale_calibration_nvfp4_b200 import nvfp4
    for name in declared_functions():
        assert hasattr(L, name), name
    # the binding wraps every declared compute entry point under the same name
    for name in declared_functions():
        if name not in ("nvfp4_status_string", "nvfp4_shutdown"):
            assert name in nvfp4.SIGNATURES, name


def test_status_strings(L):
    for code in range(11):
        s = L.nvfp4_status_string(code).decode()
        assert s.startswith("NVFP4_")
    assert L.nvfp4_status_string(0).decode() == "NVFP4_OK"
    assert L.nvfp4_status_string(99).decode() == "NVFP4_ERR_UNKNOWN"


P = 0x10000   # aligned fake device pointer (never dereferenced: validation fails first)
BAD = 0x10001  # misaligned


def test_validation_rejects_before_launch(L):
    # shape: C not a multiple of 16
    assert L.nvfp4_scale_search_max(P, 1, 4, 17, P, P, None) == SHAPE
    assert L.nvfp4_scale_search_four_over_six(P, 1, 4, 17, P, P, None) == SHAPE
    assert L.nvfp4_scale_search_four_over_six(BAD, 1, 4, 16, P, P, None) == MISALIGNED
    assert L.nvfp4_scale_search_four_over_six(None, 1, 4, 16, P, P, None) == INVALID
    assert L.nvfp4_scale_search_mse(P, 1, 4, 24, P, P, None, None) == SHAPE
    assert L.nvfp4_scale_search_local_hessian(P, 1, 4, 40, P, P, P, None, None) == SHAPE
    assert L.nvfp4_quantize_pack(P, 1, 4, 8, P, P, P, None) == SHAPE
    assert L.nvfp4_dequantize(P, P, P, 1, 4, 20, P, None) == SHAPE
    assert L.nvfp4_fake_quant(P, 4, 33, P, None, None, P, None) == SHAPE
    assert L.nvfp4_hessian_accumulate(P, 10, 50, P, None) == SHAPE
    assert L.nvfp4_hessian_accumulate_grouped(P, P, 2, 10, 50, P, None) == SHAPE
    assert L.nvfp4_global_scale(P, 1, 12, P, None) == SHAPE
    # null pointers and bad counts
    assert L.nvfp4_scale_search_max(None, 1, 4, 16, P, P, None) == INVALID
    assert L.nvfp4_scale_search_max(P, 0, 4, 16, P, P, None) == INVALID
    assert L.nvfp4_scale_search_max(P, 1, -1, 16, P, P, None) == INVALID
    assert L.nvfp4_scale_search_local_hessian(P, 1, 4, 16, P, None, P, None, None) == INVALID
    assert L.nvfp4_quantize_pack(P, 1, 4, 16, P, P, None, None) == INVALID
    assert L.nvfp4_hessian_accumulate(None, 10, 16, P, None) == INVALID
    assert L.nvfp4_hessian_accumulate_grouped(P, None, 2, 10, 16, P, None) == INVALID
    assert L.nvfp4_hessian_accumulate_grouped(P, P, 0, 10, 16, P, None) == INVALID
    assert L.nvfp4_global_scale(P, 1, 16, None, None) == INVALID
    assert L.nvfp4_get_device_status(None, None) == INVALID
    # alignment
    assert L.nvfp4_scale_search_max(BAD, 1, 4, 16, P, P, None) == MISALIGNED
    assert L.nvfp4_quantize_pack(P, 1, 4, 16, P, P, BAD, None) == MISALIGNED
    assert L.nvfp4_dequantize(P, P, P, 1, 4, 16, BAD, None) == MISALIGNED
    assert L.nvfp4_fake_quant(BAD, 4, 16, P, None, None, P, None) == MISALIGNED
    assert L.nvfp4_hessian_accumulate(BAD, 10, 16, P, None) == MISALIGNED
    assert L.nvfp4_global_scale(P, 1, 16, BAD, None) == MISALIGNED
    # sizes that overflow
    assert L.nvfp4_scale_search_max(P, 1, 1 << 40, 1 << 24, P, P, None) == SHAPE
    assert L.nvfp4_scale_search_max(P, 70000, 4, 16, P, P, None) == TOOLARGE
    # the NVFP4 product: K a multiple of 32, N of 8, aligned operands
    assert L.nvfp4_gemm(P, P, P, P, P, P, 128, 64, 48, P, None) == SHAPE
    assert L.nvfp4_gemm(P, P, P, P, P, P, 128, 60, 64, P, None) == SHAPE
    assert L.nvfp4_gemm(BAD, P, P, P, P, P, 128, 64, 64, P, None) == MISALIGNED
    assert L.nvfp4_gemm(P, P, P, P, P, P, 128, 64, 64, None, None) == INVALID
    # activation-range calibration
    assert L.nvfp4_abs_histogram(BAD, 64, P, None) == MISALIGNED
    assert L.nvfp4_static_scale_from_histogram(P, ctypes.c_double(0.0), P, None) == INVALID
    assert L.nvfp4_static_scale_from_histogram(P, ctypes.c_double(1.5), P, None) == INVALID
    assert L.nvfp4_fake_quant_static(P, 4, 20, P, P, None, None, None) == SHAPE
    assert L.nvfp4_quant_error(P, 4, 16, P, None, None) == INVALID
    # full Gram and GPTQ
    assert L.nvfp4_hessian_full_accumulate(P, 10, 24, P, None) == SHAPE
    assert L.nvfp4_hessian_full_accumulate(P, 10, 32, BAD, None) == MISALIGNED
    assert L.nvfp4_hessian_full_accumulate(P, 10, 32, None, None) == INVALID
    d = ctypes.c_double
    assert L.nvfp4_gptq(P, 1, 4, 24, P, P, P, d(0.01), P, None) == SHAPE
    assert L.nvfp4_gptq(P, 1, 4, 32, P, P, None, d(0.01), P, None) == INVALID
    assert L.nvfp4_gptq(P, 1, 4, 32, P, P, P, d(-1.0), P, None) == INVALID
    assert L.nvfp4_gptq(P, 1, 4, 32, P, P, P, d(float("nan")), P, None) == INVALID
    assert L.nvfp4_gptq(BAD, 1, 4, 32, P, P, P, d(0.01), P, None) == MISALIGNED
    assert L.nvfp4_gptq(P, 1, 4, 32, P, P, BAD, d(0.01), P, None) == MISALIGNED
    assert L.nvfp4_gptq(P, 70000, 4, 32, P, P, P, d(0.01), P, None) == TOOLARGE
    # the statistics call needs somewhere to write
    assert L.nvfp4_search_evaluations(None, 0, None) == INVALID


def test_binding_rejects_cpu_tensors():
    import torch
    from scale_calibration_nvfp4_b200 import nvfp4
    w = torch.zeros(4, 16, dtype=torch.bfloat16)
    with pytest.raises(ValueError):
        nvfp4.scale_search_max(w, torch.ones(1))
    with pytest.raises(TypeError):
        nvfp4.scale_search_max(w.float(), torch.ones(1))
