"""Training-side path against the CPU oracle: the transposed quantizer (bit-exact),
the transposed-output GEMM, and the straight-through backward GEMMs dgrad
(dX = dY . W) and wgrad (dW = dY^T . X) on MXFP4 operands quantized along each
GEMM's contraction axis (tolerance 1e-5 * S, as the forward)."""
import numpy as np
import pytest

from block_scaled_gemm_rfq_b200 import workloads as wl
from helpers import assert_quant_parity, assert_y_close, dev_bf16, y_to_numpy

pytestmark = pytest.mark.gpu


def gpu_quantize_t(rfq, bits, residual):
    import torch
    q = rfq.quantize_mxfp4_t_alloc(dev_bf16(bits), residual=residual)
    torch.cuda.synchronize()
    rfq.check_device_error()
    R, C = bits.shape
    cb, sb = rfq.codes_bytes(C, R), rfq.scales_bytes(C, R)
    out = {"codes_x": q.codes.cpu().numpy()[:cb].reshape(C, R // 2), "scales_x": q.scales.cpu().numpy()[:sb]}
    if residual:
        out["codes_r"] = q.r_codes.cpu().numpy()[:cb].reshape(C, R // 2)
        out["scales_r"] = q.r_scales.cpu().numpy()[:sb]
    return out


@pytest.mark.parametrize("R,C", [(32, 8), (64, 72), (96, 200), (256, 520), (1024, 512), (160, 4096)])
@pytest.mark.parametrize("residual", [True, False])
def test_transposed_quantizer_bit_exact(rfq, oracle, R, C, residual):
    bits = wl.random_matrix(R, C, seed=R + C, scale=3.0)
    got = gpu_quantize_t(rfq, bits, residual)
    assert_quant_parity(oracle, np.ascontiguousarray(bits.T), got, residual=residual)


def test_transposed_quantizer_outliers_and_specials(rfq, oracle):
    """Heavy tails, outlier rows (the blocks run down the rows), tiny values,
    signed zeros and one non-finite block."""
    rng = np.random.default_rng(7)
    X = rng.standard_t(3.0, (256, 136))
    X[rng.choice(256, 5, replace=False), :] *= 1000.0
    X[rng.random(X.shape) < 0.02] *= 1e-30
    X[:32, 0] = -0.0
    bits = wl.f64_to_bf16_bits(X)
    bits[40, 3] = 0x7FC0                         # NaN: block (column 3, rows 32..63) gets scale 0xFF
    got = gpu_quantize_t(rfq, bits, True)
    assert_quant_parity(oracle, np.ascontiguousarray(bits.T), got, residual=True)


def test_gemm_yt_is_the_transpose(rfq):
    import torch
    x = dev_bf16(wl.random_matrix(300, 256, seed=1, scale=2.0))
    w = dev_bf16(wl.random_matrix(264, 256, seed=2, scale=0.05))
    qa = rfq.quantize_mxfp4_alloc(x)
    qw = rfq.quantize_weight_alloc(w)
    for out in (torch.float32, torch.bfloat16):
        y = rfq.gemm_alloc(qa, qw, out_dtype=out)
        yt = torch.empty((264, 300), dtype=out, device="cuda")
        rfq.gemm_yt(qa.codes, qa.scales, qa.r_codes, qa.r_scales, qw.codes, qw.scales, 300, 264, 256, yt)
        torch.cuda.synchronize()
        rfq.check_device_error()
        assert torch.equal(y.t().contiguous(), yt)


@pytest.mark.parametrize("M,N,K", [(16, 256, 128), (128, 256, 192), (300, 512, 264), (1024, 1024, 512)])
@pytest.mark.parametrize("residual", [True, False])
def test_dgrad_parity(rfq, oracle, M, N, K, residual):
    import torch
    dy = wl.random_matrix(M, N, seed=M + N, scale=1e-3)
    w = wl.random_matrix(N, K, seed=N + K, scale=0.02)
    qwt = rfq.quantize_mxfp4_t_alloc(dev_bf16(w), residual=False)      # W^T [K][N], blocks along N
    dx = rfq.linear_dgrad_alloc(dev_bf16(dy), qwt, out_dtype=torch.float32, use_residual=residual)
    torch.cuda.synchronize()
    rfq.check_device_error()
    ref, S, _ = oracle.rfq_dgrad(dy, w, residual=residual)
    assert_y_close(y_to_numpy(dx), ref, S, bf16_out=False, what=f"dX[{M}x{K}] over N={N}")


@pytest.mark.parametrize("M,K,N", [(32, 64, 8), (256, 128, 136), (1024, 512, 264), (96, 4096, 520)])
@pytest.mark.parametrize("residual", [True, False])
def test_wgrad_parity(rfq, oracle, M, K, N, residual):
    import torch
    x = wl.random_matrix(M, K, seed=3 * M + K, scale=2.0)
    dy = wl.random_matrix(M, N, seed=M + 5 * N, scale=1e-3)
    for out in (torch.float32, torch.bfloat16):
        dw = rfq.linear_wgrad_alloc(dev_bf16(x), dev_bf16(dy), out_dtype=out, use_residual=residual)
        torch.cuda.synchronize()
        rfq.check_device_error()
        ref, S, _ = oracle.rfq_wgrad(x, dy, residual=residual)
        assert_y_close(y_to_numpy(dw), ref, S, bf16_out=(out == torch.bfloat16), what=f"dW[{N}x{K}] over M={M}")


def test_wgrad_ffn_shape_sampled(rfq, oracle):
    """dW of the FFN up-projection (M = 4096 tokens, K = 4096, N = 12288) on the GPU;
    the oracle recomputes sampled rows of dW (columns n of dY) against all of X^T."""
    import torch
    wk = wl.ffn_up(0)
    rng = np.random.default_rng(3)
    dy = wl.f64_to_bf16_bits(rng.normal(0, 1e-3, (wk.M, wk.N)))
    dw = rfq.linear_wgrad_alloc(dev_bf16(wk.x_bits), dev_bf16(dy), out_dtype=torch.float32)
    torch.cuda.synchronize()
    rfq.check_device_error()
    cols = np.array(sorted(set(rng.choice(wk.N, 24, replace=False).tolist()) | {0, wk.N - 1}))
    qx = oracle.quantize_transposed(wk.x_bits, residual=True)
    qd = oracle.quantize_transposed(np.ascontiguousarray(dy[:, cols]), residual=False)
    A, B = oracle.rfq_operands(qx, qd, True)            # A = [X^T | R^T] (K x 2M), B = dY^T cols
    Yt, absY = oracle.gemm_blas(A, B)                  # [K, len(cols)]
    assert_y_close(y_to_numpy(dw)[cols], Yt.T, float(absY.max()), bf16_out=False, what="ffn dW rows")


def test_wgrad_rejects_ragged_token_count(rfq):
    import torch
    x = torch.zeros((48, 64), dtype=torch.bfloat16, device="cuda")
    dy = torch.zeros((48, 16), dtype=torch.bfloat16, device="cuda")
    dw = torch.empty((16, 64), dtype=torch.float32, device="cuda")
    ws = torch.empty(1 << 20, dtype=torch.uint8, device="cuda")
    with pytest.raises(rfq.RFQError) as e:
        rfq.linear_wgrad(x, dy, dw, ws)
    assert e.value.status == 2
