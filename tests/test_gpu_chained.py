"""Layers chained on one stream with no host synchronisation in between.

Every kernel is launched with programmatic stream serialization: it may start
while the previous kernel on the stream is still running, prefetches its first
input tiles into L2, and waits for the previous kernel only before its first
real load.  A kernel that reads the previous kernel's output must still see all
of it.  A chain of RFQ linear layers (Y of layer i is X of layer i + 1) is run
back to back and compared bit for bit with the same layers run one at a time,
with a device synchronisation around every call.  The three row counts take the
three paths of rfq_linear: the single kernel, quantize + short-batch GEMM, and
quantize + tiled GEMM.
"""
import pytest

from block_scaled_gemm_rfq_b200 import workloads as wl
from helpers import dev_bf16

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("M", [16, 200, 1024])
def test_chained_layers_match_one_at_a_time(rfq, M):
    import torch
    K = 1024
    layers = 4
    # W ~ N(0, 1/K): the activations keep unit scale through the chain
    qws = [rfq.quantize_weight_alloc(dev_bf16(wl.random_matrix(K, K, seed=40 + i, scale=K ** -0.5)))
           for i in range(layers)]
    x0 = dev_bf16(wl.random_matrix(M, K, seed=M, scale=1.0))
    ys = [torch.empty((M, K), dtype=torch.bfloat16, device="cuda") for _ in range(layers)]
    ws = torch.empty(rfq.linear_workspace_bytes(M, K, True), dtype=torch.uint8, device="cuda")

    x = x0
    for qw, y in zip(qws, ys):
        rfq.linear(x, qw.codes, qw.scales, K, y, ws, True)
        x = y
    torch.cuda.synchronize()
    rfq.check_device_error()
    chained = [y.clone() for y in ys]

    x = x0
    for qw, y in zip(qws, ys):
        y.fill_(7.0)
        torch.cuda.synchronize()
        rfq.linear(x, qw.codes, qw.scales, K, y, ws, True)
        torch.cuda.synchronize()
        x = y
    rfq.check_device_error()
    for i, (a, b) in enumerate(zip(chained, ys)):
        assert torch.isfinite(b.float()).all(), f"layer {i}"
        assert float(b.float().abs().max()) > 0.1, f"layer {i}: activations vanished"
        assert torch.equal(a.view(torch.int16), b.view(torch.int16)), f"layer {i} differs when chained"


def test_quantizer_right_after_the_gemm_that_writes_its_input(rfq):
    """rfq_gemm writes Y; rfq_quantize_mxfp4 of Y follows at once on the stream."""
    import torch
    M, K, N = 512, 1024, 2048
    qw = rfq.quantize_weight_alloc(dev_bf16(wl.random_matrix(N, K, seed=3, scale=K ** -0.5)))
    qa = rfq.quantize_mxfp4_alloc(dev_bf16(wl.random_matrix(M, K, seed=4, scale=1.0)))
    y = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
    q1 = rfq.quantize_mxfp4_alloc(torch.zeros((M, N), dtype=torch.bfloat16, device="cuda"))
    q2 = rfq.quantize_mxfp4_alloc(torch.zeros((M, N), dtype=torch.bfloat16, device="cuda"))
    torch.cuda.synchronize()
    for _ in range(3):
        y.fill_(-3.0)
        rfq.gemm(qa.codes, qa.scales, qa.r_codes, qa.r_scales, qw.codes, qw.scales, M, N, K, y)
        rfq.quantize_mxfp4(y, q1.codes, q1.scales, q1.r_codes, q1.r_scales)
        torch.cuda.synchronize()
        rfq.quantize_mxfp4(y, q2.codes, q2.scales, q2.r_codes, q2.r_scales)
        torch.cuda.synchronize()
        rfq.check_device_error()
        for a, b in ((q1.codes, q2.codes), (q1.scales, q2.scales), (q1.r_codes, q2.r_codes),
                     (q1.r_scales, q2.r_scales)):
            assert torch.equal(a, b)
