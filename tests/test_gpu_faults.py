"""Failure detection without a GPU fault: every spin-wait inside the GEMM is bounded.

The library's test hook makes the producer of the first CTA skip one stage fill, so
the MMA warp's wait for that stage runs out (after about 1.5 s).  The skipped fill
is the last one of the CTA's only tile: the producer then has nothing left to wait
for, so the MMA warp's wait is the one that runs out (skipping an early fill would
also leave the producer waiting for a free stage, and either wait may expire first;
the epilogue's wait for the accumulator, which starts earlier, has twice the limit).  The kernel then
records the wait in the device error word, drains its own copies and MMAs, frees its
TMEM and returns; rfq_check_device_error reports RFQ_ERR_TIMEOUT with detail 1 (the
stage wait) and the context stays usable: the next GEMM is correct.  Both the
single-CTA path (M <= 128 with enough columns to fill the GPU), the CTA-pair
path (M > 256) and the short-batch split-K path (few tiles; K unsplit here so
that the skipped fill is again the CTA's last) are exercised.
"""
import pytest

from block_scaled_gemm_rfq_b200 import workloads as wl
from helpers import assert_y_close, dev_bf16, y_to_numpy

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("M,N", [(128, 256), (384, 256), (100, 19200)])
def test_skipped_fill_times_out_and_context_survives(rfq, oracle, M, N):
    import torch
    K = 1024
    x_bits = wl.random_matrix(M, K, seed=M, scale=2.0)
    w_bits = wl.random_matrix(N, K, seed=M + 1, scale=0.05)
    qa = rfq.quantize_mxfp4_alloc(dev_bf16(x_bits), residual=True)
    qw = rfq.quantize_weight_alloc(dev_bf16(w_bits))
    torch.cuda.synchronize()
    rfq.check_device_error()

    rfq.debug_skip_next_fill(K // 256 - 1)   # the last of the tile's 256-K stage fills
    rfq.debug_fused_split(1)
    y = torch.empty((M, N), dtype=torch.float32, device="cuda")
    rfq.gemm(qa.codes, qa.scales, qa.r_codes, qa.r_scales, qw.codes, qw.scales, M, N, K, y)
    try:
        with pytest.raises(rfq.RFQError) as info:
            rfq.check_device_error()
    finally:
        rfq.debug_fused_split(0)
    assert info.value.status == 6          # RFQ_ERR_TIMEOUT
    assert info.value.detail == 1          # the MMA warp's wait for a loaded stage
    rfq.check_device_error()               # the error word was cleared

    # the context is still usable and the hook is one-shot
    y2 = rfq.gemm_alloc(qa, qw, out_dtype=torch.float32)
    torch.cuda.synchronize()
    rfq.check_device_error()
    Y, S, _ = oracle.rfq_linear(x_bits, w_bits, residual=True)
    assert_y_close(y_to_numpy(y2), Y, S, bf16_out=False)


def test_short_batch_exchange_survives_an_aborted_cta(rfq, oracle):
    """Split-K over a cluster of 4 (one k-tile each): the first CTA's only stage fill
    is skipped, so its MMA warp's wait runs out while its three peers finish and wait
    for it at the reduction's cluster barriers.  The aborted CTA still takes part in
    both barriers (every thread reaches them on the error path too), so the cluster
    completes, the error word names the stage wait, and the next call is correct."""
    import torch
    M, N, K = 40, 256, 1024
    x_bits = wl.random_matrix(M, K, seed=41, scale=2.0)
    w_bits = wl.random_matrix(N, K, seed=42, scale=0.05)
    qa = rfq.quantize_mxfp4_alloc(dev_bf16(x_bits), residual=True)
    qw = rfq.quantize_weight_alloc(dev_bf16(w_bits))
    torch.cuda.synchronize()
    rfq.check_device_error()
    rfq.debug_skip_next_fill(0)
    rfq.debug_fused_split(4)
    try:
        y = torch.empty((M, N), dtype=torch.float32, device="cuda")
        rfq.gemm(qa.codes, qa.scales, qa.r_codes, qa.r_scales, qw.codes, qw.scales, M, N, K, y)
        with pytest.raises(rfq.RFQError) as info:
            rfq.check_device_error()
        assert info.value.status == 6 and info.value.detail == 1
        rfq.check_device_error()
        y2 = rfq.gemm_alloc(qa, qw, out_dtype=torch.float32)
        torch.cuda.synchronize()
        rfq.check_device_error()
    finally:
        rfq.debug_fused_split(0)
    Y, S, _ = oracle.rfq_linear(x_bits, w_bits, residual=True)
    assert_y_close(y_to_numpy(y2), Y, S, bf16_out=False)
