"""The single-kernel RFQ linear layer (quantizer inside the GEMM, M <= 64) against
the CPU oracle.

Same bar as the two-kernel path: max|Y_gpu - Y_ref| <= 1e-5 * S (+ one bf16 ulp
for bf16 output), Y_ref and S from the oracle's own quantization of the seeded
bf16 inputs.  The fused kernel also splits K over a cluster of CTAs and adds
the partial sums in a fixed order: every split must pass, and repeated runs
must agree bit for bit.
"""
import numpy as np
import pytest

from block_scaled_gemm_rfq_b200 import workloads as wl
from helpers import assert_y_close, dev_bf16, y_to_numpy

pytestmark = pytest.mark.gpu


def run_fused(rfq, x_bits, w_bits, residual, out_dtype, split=0):
    import torch
    x, w = dev_bf16(x_bits), dev_bf16(w_bits)
    qw = rfq.quantize_weight_alloc(w)
    rfq.debug_fused_split(split)
    try:
        y = rfq.linear_fused_alloc(x, qw, out_dtype=out_dtype, use_residual=residual)
        torch.cuda.synchronize()
    finally:
        rfq.debug_fused_split(0)
    rfq.check_device_error()
    return y_to_numpy(y)


@pytest.mark.parametrize("M,N,K", [(1, 8, 32), (16, 128, 256), (7, 136, 288), (17, 264, 1024), (33, 520, 544),
                                   (48, 256, 2080), (64, 1000, 4096), (64, 4096, 4096), (2, 12288, 512)])
@pytest.mark.parametrize("residual", [True, False])
def test_fused_edge_shapes(rfq, oracle, M, N, K, residual):
    import torch
    x = wl.random_matrix(M, K, seed=11 * M + 3 * N + K, scale=2.0)
    w = wl.random_matrix(N, K, seed=M + 5 * N + 7 * K, scale=0.05)
    Y, S, _ = oracle.rfq_linear(x, w, residual=residual)
    y = run_fused(rfq, x, w, residual, torch.float32)
    assert_y_close(y, Y, S, bf16_out=False, what=f"fused Y[{M}x{N}x{K}]")


@pytest.mark.parametrize("split", [1, 2, 3, 5, 8])
@pytest.mark.parametrize("M", [12, 24])
def test_fused_every_split(rfq, oracle, split, M):
    """Each cluster size (ragged k-ranges included: 9 k-tiles over 2, 3, 5, 8 CTAs), with
    8 quantizer warps (up to 16 rows) and with 16 (17-32 rows)."""
    import torch
    N, K = 384, 2304
    x = wl.random_matrix(M, K, seed=21 + M, scale=3.0)
    w = wl.random_matrix(N, K, seed=22, scale=0.05)
    Y, S, _ = oracle.rfq_linear(x, w, residual=True)
    for out in (torch.float32, torch.bfloat16):
        y = run_fused(rfq, x, w, True, out, split=split)
        assert_y_close(y, Y, S, bf16_out=(out == torch.bfloat16), what=f"split {split} {out}")


def test_fused_is_deterministic(rfq):
    import torch
    M, N, K = 40, 2048, 4096
    x = wl.random_matrix(M, K, seed=5, scale=2.0)
    w = wl.random_matrix(N, K, seed=6, scale=0.05)
    a = run_fused(rfq, x, w, True, torch.float32)
    b = run_fused(rfq, x, w, True, torch.float32)
    assert np.array_equal(a.view(np.uint32), b.view(np.uint32))


def test_fused_outlier_rows(rfq, oracle):
    """Outlier channels x1000 and tiny channels inside each row, bf16 output."""
    import torch
    rng = np.random.default_rng(8)
    X = rng.standard_t(3.0, (16, 1024))
    X[:, rng.choice(1024, 12, replace=False)] *= 1000.0
    X[:, rng.choice(1024, 12, replace=False)] *= 1e-6
    W = rng.normal(0, 0.02, (512, 1024))
    xb, wb = wl.f64_to_bf16_bits(X), wl.f64_to_bf16_bits(W)
    Y, S, _ = oracle.rfq_linear(xb, wb, residual=True)
    y = run_fused(rfq, xb, wb, True, torch.bfloat16)
    assert_y_close(y, Y, S, bf16_out=True)


def test_rfq_linear_dispatches_short_batches_to_fused(rfq):
    """rfq_linear with M <= 32 runs the fused kernel: bit-identical to rfq_linear_fused
    (same automatic split), and the workspace is left untouched."""
    import torch
    M, N, K = 32, 1024, 2048
    x = dev_bf16(wl.random_matrix(M, K, seed=31, scale=2.0))
    qw = rfq.quantize_weight_alloc(dev_bf16(wl.random_matrix(N, K, seed=32, scale=0.05)))
    y1 = torch.empty((M, N), dtype=torch.float32, device="cuda")
    ws = torch.full((rfq.linear_workspace_bytes(M, K, True),), 0xA5, dtype=torch.uint8, device="cuda")
    rfq.linear(x, qw.codes, qw.scales, N, y1, ws, True)
    y2 = rfq.linear_fused_alloc(x, qw, out_dtype=torch.float32)
    torch.cuda.synchronize()
    rfq.check_device_error()
    assert torch.equal(y1.view(torch.int32), y2.view(torch.int32))
    assert bool((ws == 0xA5).all())


def test_fused_rejects_long_batches_and_writes_zeros_for_k0(rfq):
    import torch
    x = torch.zeros((rfq.FUSED_MAX_M + 1, 64), dtype=torch.bfloat16, device="cuda")
    qw = rfq.quantize_weight_alloc(torch.zeros((16, 64), dtype=torch.bfloat16, device="cuda"))
    y = torch.empty((rfq.FUSED_MAX_M + 1, 16), dtype=torch.float32, device="cuda")
    with pytest.raises(rfq.RFQError) as e:
        rfq.linear_fused(x, qw.codes, qw.scales, 16, y)
    assert e.value.status == 2
    y0 = torch.full((8, 16), 3.0, device="cuda")
    rfq.linear_fused(torch.empty((8, 0), dtype=torch.bfloat16, device="cuda"), qw.codes, qw.scales, 16, y0)
    torch.cuda.synchronize()
    assert torch.count_nonzero(y0).item() == 0
