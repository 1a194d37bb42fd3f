"""Kernel 2 (RFQ block-scaled GEMM on tcgen05) and rfq_linear against the CPU oracle.

Y_gpu must satisfy max|Y_gpu - Y_ref| <= 1e-5 * S (fp32 output), plus one bf16
ulp for bf16 output, where Y_ref and S come from the oracle's own quantization
of the same seeded bf16 inputs (nothing the GPU computed is fed to the oracle).
"""
import numpy as np
import pytest

from block_scaled_gemm_rfq_b200 import workloads as wl
from helpers import assert_y_close, dev_bf16, y_to_numpy

pytestmark = pytest.mark.gpu


def run_gemm(rfq, x_bits, w_bits, residual, out_dtype):
    import torch
    x, w = dev_bf16(x_bits), dev_bf16(w_bits)
    qa = rfq.quantize_mxfp4_alloc(x, residual=residual)
    qw = rfq.quantize_weight_alloc(w)
    y = rfq.gemm_alloc(qa, qw, out_dtype=out_dtype, use_residual=residual)
    torch.cuda.synchronize()
    rfq.check_device_error()
    return y_to_numpy(y)


def run_linear(rfq, x_bits, w_bits, residual, out_dtype):
    import torch
    x, w = dev_bf16(x_bits), dev_bf16(w_bits)
    qw = rfq.quantize_weight_alloc(w)
    y = rfq.linear_alloc(x, qw, out_dtype=out_dtype, use_residual=residual)
    torch.cuda.synchronize()
    rfq.check_device_error()
    return y_to_numpy(y)


def test_tiny_rfq_linear_fp32(rfq, oracle):
    import torch
    w = wl.tiny(0)
    Y, S, _ = oracle.rfq_linear(w.x_bits, w.w_bits, residual=True)
    for runner in (run_gemm, run_linear):
        y = runner(rfq, w.x_bits, w.w_bits, True, torch.float32)
        assert_y_close(y, Y, S, bf16_out=False)


def test_tiny_rfq_off(rfq, oracle):
    import torch
    w = wl.tiny(0)
    Y, S, _ = oracle.rfq_linear(w.x_bits, w.w_bits, residual=False)
    y = run_gemm(rfq, w.x_bits, w.w_bits, False, torch.float32)
    assert_y_close(y, Y, S, bf16_out=False)


def test_tiny_bf16_output(rfq, oracle):
    import torch
    w = wl.tiny(1)
    Y, S, _ = oracle.rfq_linear(w.x_bits, w.w_bits, residual=True)
    y = run_linear(rfq, w.x_bits, w.w_bits, True, torch.bfloat16)
    assert_y_close(y, Y, S, bf16_out=True)


# Paths: M <= 256 with few tiles -> the short-batch split-K kernel; (100, 19200) the
# single-CTA tiled GEMM (75 tiles); (200, 9472) and M > 256 the CTA-pair GEMM.
@pytest.mark.parametrize("M,N,K", [(1, 8, 64), (16, 16, 64), (127, 136, 96), (129, 264, 160), (300, 520, 1024),
                                   (256, 256, 4096), (64, 512, 32), (200, 1000, 2080), (100, 19200, 256),
                                   (200, 9472, 288), (240, 4096, 1056), (300, 8, 64), (333, 136, 128),
                                   (1000, 72, 256)])
@pytest.mark.parametrize("residual", [True, False])
def test_edge_shapes(rfq, oracle, M, N, K, residual):
    """fp32 and bf16 Y, ragged M, N and K on every GEMM path."""
    import torch
    x = wl.random_matrix(M, K, seed=M + 3 * N + 7 * K, scale=2.0)
    w = wl.random_matrix(N, K, seed=M * N + K, scale=0.05)
    Y, S, _ = oracle.rfq_linear(x, w, residual=residual)
    for out in (torch.float32, torch.bfloat16):
        y = run_gemm(rfq, x, w, residual, out)
        assert_y_close(y, Y, S, bf16_out=(out == torch.bfloat16), what=f"Y[{M}x{N}x{K}] {out}")


@pytest.mark.parametrize("M,N,K", [(2000, 2456, 256), (2048, 2560, 512), (4096, 4096, 256), (1800, 2696, 288)])
@pytest.mark.parametrize("residual", [True, False])
def test_partial_last_wave(rfq, oracle, M, N, K, residual):
    """Tile counts (80, 80, 256, 88 pair tiles on 74 pairs) that leave a partial last
    wave of the persistent schedule, with ragged M and N in the last tiles (the last
    shape's final tile holds 136 real columns)."""
    import torch
    x = wl.random_matrix(M, K, seed=M + K, scale=2.0)
    w = wl.random_matrix(N, K, seed=N + 3 * K, scale=0.05)
    Y, S, _ = oracle.rfq_linear(x, w, residual=residual)
    for out in (torch.float32, torch.bfloat16):
        y = run_gemm(rfq, x, w, residual, out)
        assert_y_close(y, Y, S, bf16_out=(out == torch.bfloat16), what=f"Y[{M}x{N}x{K}] {out}")


def test_outlier_heavy_inputs(rfq, oracle):
    """Large dynamic range inside a row: outlier channels x1000 and tiny channels."""
    import torch
    rng = np.random.default_rng(4)
    X = rng.standard_t(3.0, (192, 512))
    X[:, rng.choice(512, 10, replace=False)] *= 1000.0
    X[:, rng.choice(512, 10, replace=False)] *= 1e-6
    W = rng.normal(0, 0.02, (264, 512))
    xb, wb = wl.f64_to_bf16_bits(X), wl.f64_to_bf16_bits(W)
    Y, S, _ = oracle.rfq_linear(xb, wb, residual=True)
    y = run_gemm(rfq, xb, wb, True, torch.float32)
    assert_y_close(y, Y, S, bf16_out=False)


def test_k_zero_writes_zeros(rfq):
    import torch
    y = torch.full((16, 16), 7.0, device="cuda")
    empty = torch.empty(16, dtype=torch.uint8, device="cuda")
    rfq.gemm(empty, empty, None, None, empty, empty, 16, 16, 0, y)
    torch.cuda.synchronize()
    assert torch.count_nonzero(y).item() == 0


@pytest.mark.parametrize("split", [1, 2, 3, 5, 8])
@pytest.mark.parametrize("M", [40, 100, 200])
def test_short_batch_gemm_every_split(rfq, oracle, split, M):
    """rfq_gemm on a short batch with few tiles runs the split-K kernel on the
    quantizer's operands: each cluster size (9 k-tiles over 1..8 CTAs, ragged
    ranges), the layouts (up to 64 and up to 128 rows with Q(R) stacked under Q(X)
    in one B operand; above 128 rows two 128-row blocks of X on two grid rows per
    weight tile, the second one ragged), bit-identical repeats."""
    import torch
    N, K = 384, 2304
    x = wl.random_matrix(M, K, seed=M + split, scale=3.0)
    w = wl.random_matrix(N, K, seed=17, scale=0.05)
    Y, S, _ = oracle.rfq_linear(x, w, residual=True)
    qa = rfq.quantize_mxfp4_alloc(dev_bf16(x))
    qw = rfq.quantize_weight_alloc(dev_bf16(w))
    rfq.debug_fused_split(split)
    try:
        ys = [rfq.gemm_alloc(qa, qw, out_dtype=out) for out in (torch.float32, torch.bfloat16, torch.float32)]
        torch.cuda.synchronize()
    finally:
        rfq.debug_fused_split(0)
    rfq.check_device_error()
    assert_y_close(y_to_numpy(ys[0]), Y, S, bf16_out=False, what=f"short M={M} split {split}")
    assert_y_close(y_to_numpy(ys[1]), Y, S, bf16_out=True, what=f"short M={M} split {split} bf16")
    assert torch.equal(ys[0].view(torch.int32), ys[2].view(torch.int32))


@pytest.mark.parametrize("M,N,K", [(4096, 4096, 512), (1000, 2056, 768), (200, 1032, 2304), (24, 520, 1024)])
@pytest.mark.parametrize("residual", [True, False])
def test_repeat_and_output_types_agree_bitwise(rfq, M, N, K, residual):
    """Every path (the persistent CTA-pair kernel over several waves, ragged tiles, the
    short-batch split-K kernel) gives bit-identical Y on a repeat call, and its bf16 Y is
    exactly the round-to-nearest-even of its fp32 Y: both come from the same fp32
    accumulation, whatever warp issues the scale copies or the MMAs."""
    import torch
    x = wl.random_matrix(M, K, seed=M + K + 1, scale=2.0)
    w = wl.random_matrix(N, K, seed=N + K + 2, scale=0.05)
    qa = rfq.quantize_mxfp4_alloc(dev_bf16(x), residual=residual)
    qw = rfq.quantize_weight_alloc(dev_bf16(w))
    y32a = rfq.gemm_alloc(qa, qw, out_dtype=torch.float32, use_residual=residual)
    y32b = rfq.gemm_alloc(qa, qw, out_dtype=torch.float32, use_residual=residual)
    y16 = rfq.gemm_alloc(qa, qw, out_dtype=torch.bfloat16, use_residual=residual)
    torch.cuda.synchronize()
    rfq.check_device_error()
    assert torch.equal(y32a.view(torch.int32), y32b.view(torch.int32)), "repeat differs"
    assert torch.equal(y16.view(torch.int16), y32a.to(torch.bfloat16).view(torch.int16)), "bf16 Y != rne(fp32 Y)"
