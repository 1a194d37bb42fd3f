"""The quantized operands in the standard OCP MX layout, checked with an independent
MXFP4 GEMM: cuBLASLt's block-scaled GEMM (through torch's scaled_mm, 1x32 E8M0
scales in the 32x4x4 swizzled layout) reads the codes and scales our quantizer wrote
and must give the oracle's Y; with RFQ written as one GEMM over the operands
concatenated along K ([QX | QR] . [QW | QW]^T) it must agree with rfq_gemm's bf16 Y
to within one bf16 ulp + 1e-5 * S as well.

A library kernel here is only a second reader of the operand format; the product
path never calls it.  Skipped where torch has no MXFP4 scaled_mm for the device.
"""
import numpy as np
import pytest

import bench
from block_scaled_gemm_rfq_b200 import workloads as wl
from helpers import REL_TOL, assert_y_close, bf16_ulp, dev_bf16, y_to_numpy

pytestmark = pytest.mark.gpu


def _lib_mm(a, b, sa, sb, M, N, kb):
    import torch
    import torch.nn.functional as F
    return F.scaled_mm(a.view(M, kb).view(torch.float4_e2m1fn_x2), b.view(N, kb).view(torch.float4_e2m1fn_x2).t(),
                       sa.view(torch.float8_e8m0fnu), F.ScalingType.BlockWise1x32,
                       sb.view(torch.float8_e8m0fnu), F.ScalingType.BlockWise1x32,
                       swizzle_a=F.SwizzleType.SWIZZLE_32_4_4, swizzle_b=F.SwizzleType.SWIZZLE_32_4_4,
                       output_dtype=torch.bfloat16)


@pytest.mark.parametrize("M,N,K", [(304, 272, 1024), (1008, 528, 2304), (4096, 1024, 4096)])
def test_library_gemm_reads_our_operands(rfq, oracle, M, N, K):
    import torch
    if not hasattr(torch.nn.functional, "scaled_mm") or not hasattr(torch, "float4_e2m1fn_x2"):
        pytest.skip("torch has no MX scaled_mm")
    x_bits = wl.random_matrix(M, K, seed=M + 5, scale=2.0)
    w_bits = wl.random_matrix(N, K, seed=N + 6, scale=0.05)
    qa = rfq.quantize_mxfp4_alloc(dev_bf16(x_bits), residual=True)
    qw = rfq.quantize_weight_alloc(dev_bf16(w_bits))
    kb = K // 2
    a2 = torch.cat([qa.codes.view(M, kb), qa.r_codes.view(M, kb)], dim=1)
    b2 = torch.cat([qw.codes.view(N, kb), qw.codes.view(N, kb)], dim=1)
    sa2 = bench.concat_scales_along_k(qa.scales, qa.r_scales, M, K)
    sb2 = bench.concat_scales_along_k(qw.scales, qw.scales, N, K)
    try:
        y_plain = _lib_mm(qa.codes, qw.codes, qa.scales, qw.scales, M, N, kb)
        y_lib = _lib_mm(a2, b2, sa2, sb2, M, N, 2 * kb)
    except (RuntimeError, ValueError) as e:
        pytest.skip(f"no MXFP4 scaled_mm here: {str(e)[:120]}")
    y_ours = rfq.gemm_alloc(qa, qw, out_dtype=torch.bfloat16, use_residual=True)
    torch.cuda.synchronize()
    rfq.check_device_error()
    Y_off, S_off, _ = oracle.rfq_linear(x_bits, w_bits, residual=False)
    Y, S, _ = oracle.rfq_linear(x_bits, w_bits, residual=True)
    assert_y_close(y_to_numpy(y_plain), Y_off, S_off, bf16_out=True, what=f"library plain {M}x{N}x{K}")
    assert_y_close(y_to_numpy(y_lib), Y, S, bf16_out=True, what=f"library RFQ (2K) {M}x{N}x{K}")
    a, b = y_to_numpy(y_ours).astype(np.float64), y_to_numpy(y_lib).astype(np.float64)
    assert np.all(np.abs(a - b) <= bf16_ulp(b) + REL_TOL * S), f"rfq_gemm vs library {M}x{N}x{K}"
