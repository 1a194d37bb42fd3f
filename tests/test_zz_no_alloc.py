"""rfq_linear_static_workspace, the RFQ linear layer for callers that cannot allocate
device memory (a plug-in inside an application that owns the device memory pool,
or a loop where allocating is not allowed): its quantized activation lives in the
library's fixed scratch array instead of a caller-provided workspace.

The entry point runs exactly the kernels of rfq_linear, in the same order, on the
same inputs; only the address of the quantized activation differs.  So its output
must be bit-identical to rfq_linear's, and both must be within the oracle's
tolerance.  The calls come in a row with different problems (a larger one, then a
smaller one that must fully overwrite what the first left in the array), with and
without the residual path, and with M <= 32, where rfq_linear runs the
single-kernel layer and never touches the array.  This file is collected last on
purpose.
"""
import ctypes

import pytest

from block_scaled_gemm_rfq_b200 import workloads as wl
from helpers import assert_y_close, dev_bf16, y_to_numpy

pytestmark = pytest.mark.gpu


def _static_call(rfq, x, qw, N, y, residual, y_type=None):
    import torch
    lib = rfq.load_library()
    M, K = x.shape
    if y_type is None:
        y_type = rfq.OUT_BF16 if y.dtype == torch.bfloat16 else rfq.OUT_F32
    return lib.rfq_linear_static_workspace(
        ctypes.c_void_p(x.data_ptr()), M, K, ctypes.c_void_p(qw.codes.data_ptr()),
        ctypes.c_void_p(qw.scales.data_ptr()), N, ctypes.c_void_p(y.data_ptr()), y_type, int(residual),
        ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))


def _compare_once(rfq, oracle, M, N, K, residual, out_dtype, seed):
    import torch
    x_bits = wl.random_matrix(M, K, seed=seed, scale=2.0)
    w_bits = wl.random_matrix(N, K, seed=seed + 1, scale=0.05)
    x, w = dev_bf16(x_bits), dev_bf16(w_bits)
    qw = rfq.quantize_weight_alloc(w)
    y_ref = torch.empty((M, N), dtype=out_dtype, device="cuda")
    ws = torch.empty(rfq.linear_workspace_bytes(M, K, residual), dtype=torch.uint8, device="cuda")
    rfq.linear(x, qw.codes, qw.scales, N, y_ref, ws, residual)
    y_new = torch.full((M, N), float("nan"), dtype=out_dtype, device="cuda")
    assert _static_call(rfq, x, qw, N, y_new, residual) == 0
    torch.cuda.synchronize()
    rfq.check_device_error()
    bits = torch.int16 if out_dtype == torch.bfloat16 else torch.int32
    assert torch.equal(y_new.view(bits), y_ref.view(bits)), \
        f"static workspace {M}x{N}x{K} residual={residual}: output differs from rfq_linear's"
    Y, S, _ = oracle.rfq_linear(x_bits, w_bits, residual=residual)
    assert_y_close(y_to_numpy(y_new), Y, S, bf16_out=(out_dtype == torch.bfloat16),
                   what=f"static workspace {M}x{N}x{K} residual={residual}")


def test_static_workspace_matches_rfq_linear_two_calls(rfq, oracle):
    import torch
    # first a larger problem, then a smaller one that reuses (and must fully overwrite) the array
    _compare_once(rfq, oracle, 640, 264, 2048, True, torch.float32, seed=11)
    _compare_once(rfq, oracle, 200, 136, 1024, True, torch.bfloat16, seed=12)


def test_static_workspace_without_residual_and_short_batch(rfq, oracle):
    import torch
    _compare_once(rfq, oracle, 520, 136, 1536, False, torch.float32, seed=21)   # half-size workspace
    _compare_once(rfq, oracle, 16, 136, 1024, True, torch.float32, seed=22)    # single-kernel layer
    _compare_once(rfq, oracle, 24, 264, 512, False, torch.bfloat16, seed=23)


def test_static_workspace_rejects_oversized_problems(rfq):
    import torch
    M, K = 8192, 4096          # needs ~34 MiB of quantized activation with the residual path
    assert rfq.linear_workspace_bytes(M, K, True) > rfq.STATIC_WORKSPACE_BYTES
    x = torch.zeros((M, K), dtype=torch.bfloat16, device="cuda")
    w = torch.zeros((16, K), dtype=torch.bfloat16, device="cuda")
    qw = rfq.quantize_weight_alloc(w)
    y = torch.full((M, 16), 3.0, device="cuda")
    assert _static_call(rfq, x, qw, 16, y, True) == 2       # RFQ_ERR_UNSUPPORTED_SHAPE, nothing launched
    # a bad output type is reported as rfq_linear reports it (RFQ_ERR_INVALID_ARG), size or not
    assert _static_call(rfq, x, qw, 16, y, True, y_type=7) == 1
    torch.cuda.synchronize()
    assert torch.all(y == 3.0).item()
