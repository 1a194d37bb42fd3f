"""The C ABI is stream-ordered and allocation-free, so its calls can be captured in
a CUDA graph: a captured sequence (quantize W, the fused short-batch layer, the
two-kernel layer, the backward GEMMs) replays to the same bits as eager calls,
also after the inputs change in place."""
import pytest

from block_scaled_gemm_rfq_b200 import workloads as wl
from helpers import dev_bf16

pytestmark = pytest.mark.gpu


def test_graph_replay_matches_eager(rfq):
    import torch
    K, N = 1024, 768
    w = dev_bf16(wl.random_matrix(N, K, seed=1, scale=0.05))
    x16 = dev_bf16(wl.random_matrix(16, K, seed=2, scale=2.0))
    x300 = dev_bf16(wl.random_matrix(320, K, seed=3, scale=2.0))
    dy = dev_bf16(wl.random_matrix(320, N, seed=4, scale=1e-3))
    qw = rfq.quantize_weight_alloc(w)
    ws = torch.empty(rfq.linear_workspace_bytes(320, K, True), dtype=torch.uint8, device="cuda")
    wsg = torch.empty(rfq.linear_wgrad_workspace_bytes(320, K, N, True), dtype=torch.uint8, device="cuda")
    y16 = torch.empty((16, N), dtype=torch.bfloat16, device="cuda")
    y300 = torch.empty((320, N), dtype=torch.bfloat16, device="cuda")
    dw = torch.empty((N, K), dtype=torch.float32, device="cuda")

    def run(stream=None):
        rfq.quantize_weight(w, qw.codes, qw.scales, stream)
        rfq.linear(x16, qw.codes, qw.scales, N, y16, ws, True, stream)      # fused kernel (M <= 64)
        rfq.linear(x300, qw.codes, qw.scales, N, y300, ws, True, stream)    # quantize + GEMM
        rfq.linear_wgrad(x300, dy, dw, wsg, True, stream)                   # transposed quantizers + Y^T GEMM

    run()
    torch.cuda.synchronize()
    rfq.check_device_error()
    eager = [t.clone() for t in (y16, y300, dw)]
    for t in (y16, y300, dw):
        t.zero_()

    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    g = torch.cuda.CUDAGraph()
    with torch.cuda.stream(s):
        run()                      # warm-up on the capture stream (first-call setup outside the capture)
        torch.cuda.synchronize()
        with torch.cuda.graph(g, stream=s):
            run()
    for t in (y16, y300, dw):
        t.zero_()
    g.replay()
    torch.cuda.synchronize()
    rfq.check_device_error()
    for got, want in zip((y16, y300, dw), eager):
        assert torch.equal(got, want)

    # new inputs in place: the replay follows them
    x16.mul_(-1.0)
    g.replay()
    torch.cuda.synchronize()
    assert torch.equal(y16, -eager[0])
    del g
