"""The C ABI boundary on a host without a GPU: the library builds and loads,
exports every function include/rfq.h declares, and rejects bad arguments before
touching the device (these calls make no CUDA call)."""
import ctypes
import os
import re

import pytest

import block_scaled_gemm_rfq_b200 as rfq
from block_scaled_gemm_rfq_b200 import build as rfq_build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    rfq_build.build()
    return rfq.load_library()


def header_functions():
    src = open(os.path.join(ROOT, "include", "rfq.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return set(re.findall(r"\b(rfq_[a-z_0-9]+)\s*\(", src))


def test_header_declares_what_the_binding_binds():
    assert header_functions() == set(rfq.EXPORTED_SYMBOLS)


def test_library_exports_every_declared_symbol(lib):
    for name in header_functions():
        assert hasattr(lib, name), name


def test_status_strings(lib):
    for code, name in rfq.STATUS.items():
        assert lib.rfq_status_string(code).decode() == name
    assert lib.rfq_status_string(99).decode() == "RFQ_ERR_UNKNOWN"


def test_size_functions(lib):
    assert rfq.codes_bytes(128, 256) == 128 * 128
    assert rfq.scales_bytes(128, 256) == 128 * 8
    assert rfq.scales_bytes(129, 256) == 256 * 8           # rows padded to 128
    assert rfq.scales_bytes(1, 32) == 128 * 4               # blocks padded to 4
    assert rfq.scales_bytes(8192, 4096) == 8192 * 128
    assert rfq.codes_bytes(10, 33) == 0 and rfq.scales_bytes(10, 33) == 0
    assert rfq.codes_bytes(-1, 64) == 0
    one = (128 * 128 + 255) // 256 * 256 + (128 * 8 + 255) // 256 * 256
    assert rfq.linear_workspace_bytes(128, 256, True) == 2 * one
    assert rfq.linear_workspace_bytes(128, 256, False) == one


def _vp(v):
    return ctypes.c_void_p(v)


def test_argument_errors_return_before_launch(lib):
    A = 1 << 20  # an aligned fake address: never dereferenced because the checks fail first
    # K not a multiple of 32
    assert lib.rfq_quantize_mxfp4(_vp(A), 4, 48, _vp(A), _vp(A), None, None, None) == 2
    # only one of the residual pointers
    assert lib.rfq_quantize_mxfp4(_vp(A), 4, 64, _vp(A), _vp(A), _vp(A), None, None) == 1
    # misaligned input
    assert lib.rfq_quantize_mxfp4(_vp(A + 2), 4, 64, _vp(A), _vp(A), None, None, None) == 3
    # negative sizes
    assert lib.rfq_quantize_weight(_vp(A), -1, 64, _vp(A), _vp(A), None) == 1
    # N not a multiple of 8
    assert lib.rfq_gemm(_vp(A), _vp(A), None, None, _vp(A), _vp(A), 16, 12, 64, _vp(A), 0, None) == 2
    # bad output type
    assert lib.rfq_gemm(_vp(A), _vp(A), None, None, _vp(A), _vp(A), 16, 16, 64, _vp(A), 7, None) == 1
    # misaligned output
    assert lib.rfq_gemm(_vp(A), _vp(A), None, None, _vp(A), _vp(A), 16, 16, 64, _vp(A + 4), 0, None) in (3, 4, 5)
    # workspace too small / missing
    assert lib.rfq_linear(_vp(A), 16, 64, _vp(A), _vp(A), 16, _vp(A), 0, 1, None, 0, None) == 7
    assert lib.rfq_linear(_vp(A), 16, 64, _vp(A), _vp(A), 16, _vp(A), 0, 1, _vp(A), 10, None) == 7
    # fused layer: more rows than it takes, N not a multiple of 8, bad output type, bad split
    assert lib.rfq_linear_fused(_vp(A), 65, 64, _vp(A), _vp(A), 16, _vp(A), 0, 1, None) == 2
    assert lib.rfq_linear_fused(_vp(A), 16, 64, _vp(A), _vp(A), 12, _vp(A), 0, 1, None) == 2
    assert lib.rfq_linear_fused(_vp(A), 16, 64, _vp(A), _vp(A), 16, _vp(A), 9, 1, None) == 1
    assert lib.rfq_debug_fused_split(9) == 1 and lib.rfq_debug_fused_split(-1) == 1
    assert lib.rfq_debug_fused_split(0) == 0
    assert lib.rfq_linear_fused(None, 0, 64, None, None, 16, None, 0, 1, None) == 0
    # tensor-core rate probe: bad variant, iteration count, pointers, alignment
    f, n = ctypes.c_double(0.0), ctypes.c_int(0)
    assert lib.rfq_mma_rate_probe(3, 10, _vp(A), 1024, ctypes.byref(f), ctypes.byref(n), None) == 1
    assert lib.rfq_mma_rate_probe(0, 0, _vp(A), 1024, ctypes.byref(f), ctypes.byref(n), None) == 1
    assert lib.rfq_mma_rate_probe(0, 100001, _vp(A), 1024, ctypes.byref(f), ctypes.byref(n), None) == 1
    assert lib.rfq_mma_rate_probe(0, 10, None, 1024, ctypes.byref(f), ctypes.byref(n), None) == 1
    assert lib.rfq_mma_rate_probe(0, 10, _vp(A), 1024, None, ctypes.byref(n), None) == 1
    assert lib.rfq_mma_rate_probe(0, 10, _vp(A + 4), 1024, ctypes.byref(f), ctypes.byref(n), None) == 3
    # empty problems are valid no-ops (no device needed)
    assert lib.rfq_quantize_mxfp4(None, 0, 64, None, None, None, None, None) == 0
    assert lib.rfq_gemm(None, None, None, None, None, None, 0, 16, 64, None, 0, None) == 0
    assert lib.rfq_gemm(None, None, None, None, None, None, 16, 0, 64, None, 0, None) == 0


def test_binding_fails_loudly_without_library(tmp_path, monkeypatch):
    import importlib
    mod = importlib.import_module("block_scaled_gemm_rfq_b200")
    monkeypatch.setattr(mod, "_lib", None)
    monkeypatch.setattr(mod, "_LIB_PATH", str(tmp_path / "missing.so"))
    with pytest.raises(RuntimeError, match="missing"):
        mod.load_library()
