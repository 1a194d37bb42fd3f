"""Activation fidelity of RFQ vs plain MXFP4, measured with the CUDA path.

The RFQ paper (abstract; section 1) claims that activation quantization dominates the
FP4 error and that the residual path recovers most of it.  A GEMM against the K x K
identity (represented exactly by MXFP4) returns DQ(QX) [+ DQ(QR)]: first checked
against the oracle's dequantization, then used to compare the relative activation
error with and without the residual path on the heavy-tailed synthetic workloads.
"""
import numpy as np
import pytest

from block_scaled_gemm_rfq_b200 import workloads as wl
from helpers import dev_bf16

pytestmark = pytest.mark.gpu


def _xhat(rfq, x, residual):
    import torch
    K = x.shape[1]
    qe = rfq.quantize_weight_alloc(torch.eye(K, dtype=torch.bfloat16, device="cuda"))
    qa = rfq.quantize_mxfp4_alloc(x, residual=residual)
    y = rfq.gemm_alloc(qa, qe, out_dtype=torch.float32, use_residual=residual)
    torch.cuda.synchronize()
    rfq.check_device_error()
    return y


def test_identity_gemm_returns_dequantized_activation(rfq, oracle):
    w = wl.tiny(0)
    xhat = _xhat(rfq, dev_bf16(w.x_bits), True).cpu().numpy().astype(np.float64)
    q = oracle.quantize_bf16(w.x_bits, residual=True)
    want = oracle.dequantize(q["codes_x"], q["scales_x"]) + oracle.dequantize(q["codes_r"], q["scales_r"])
    np.testing.assert_allclose(xhat, want, rtol=2 ** -23, atol=0)


@pytest.mark.parametrize("make", [lambda: wl.tiny(0), lambda: wl.quantize_bandwidth(0, M=512),
                                  lambda: wl.ffn_up(0, M=512, N=256), lambda: wl.dit_ffn(0, M=512, N=256)])
def test_residual_path_recovers_activation_error(rfq, make):
    import torch
    wk = make()
    x = dev_bf16(wk.x_bits)
    xf = x.float()
    err = {}
    for res in (True, False):
        err[res] = float(torch.linalg.norm(_xhat(rfq, x, res) - xf) / torch.linalg.norm(xf))
    assert err[True] < 0.25 * err[False], err
    if wk.w_bits is not None:
        w = dev_bf16(wk.w_bits)
        yref = xf @ w.float().t()
        qw = rfq.quantize_weight_alloc(w)
        yerr = {}
        for res in (True, False):
            qa = rfq.quantize_mxfp4_alloc(x, residual=res)
            y = rfq.gemm_alloc(qa, qw, out_dtype=torch.float32, use_residual=res)
            yerr[res] = float(torch.linalg.norm(y - yref) / torch.linalg.norm(yref))
        assert yerr[True] < yerr[False], yerr
