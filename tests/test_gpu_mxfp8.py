"""The MXFP8 (E4M3) comparator path against the CPU oracle: quantizer codes and
scales bit for bit, GEMM within 1e-5 * S (fp32 accumulation of exact E4M3 x E4M3
products), plus one bf16 ulp for bf16 output."""
import numpy as np
import pytest

from block_scaled_gemm_rfq_b200 import workloads as wl
from helpers import assert_y_close, dev_bf16, nonfinite_blocks, y_to_numpy

pytestmark = pytest.mark.gpu


def gpu_quantize8(rfq, bits):
    import torch
    q = rfq.quantize_mxfp8_alloc(dev_bf16(bits))
    torch.cuda.synchronize()
    rfq.check_device_error()
    M, K = bits.shape
    return q.codes.cpu().numpy()[: M * K].reshape(M, K), q.scales.cpu().numpy()[: rfq.scales_bytes(M, K)], q


def assert_quant8_parity(oracle, bits, codes, scales):
    ref = oracle.quantize_mxfp8_bf16(bits)
    mask = np.repeat(nonfinite_blocks(bits), 32, axis=1)
    want_c = np.where(mask, 0, ref["codes"])
    got_c = np.where(mask, 0, codes)
    bad = np.argwhere(want_c != got_c)
    assert bad.size == 0, f"{len(bad)} codes differ, first {bad[:4].tolist()}: got {got_c[tuple(bad[0])]:#04x} " \
                          f"want {want_c[tuple(bad[0])]:#04x}"
    want_s = oracle.scales_to_mma_layout(ref["scales"])
    bad = np.nonzero(want_s != scales)[0]
    assert bad.size == 0, f"{bad.size} scale bytes differ, first {bad[:4].tolist()}"


@pytest.mark.parametrize("M,K", [(1, 32), (7, 96), (128, 256), (300, 1056), (1000, 4096)])
def test_mxfp8_quantizer_bit_exact(rfq, oracle, M, K):
    bits = wl.random_matrix(M, K, seed=M * 7 + K, scale=3.0)
    codes, scales, _ = gpu_quantize8(rfq, bits)
    assert_quant8_parity(oracle, bits, codes, scales)


def test_mxfp8_quantizer_saturation_subnormals_specials(rfq, oracle):
    """Block maxima just below a power of two (scaled values in (448, 512) saturate),
    elements far below the block max (E4M3 subnormals and zeros), signed zeros, and
    one block with an infinity."""
    rng = np.random.default_rng(11)
    X = rng.normal(0, 1, (64, 512))
    X[:, ::32] = np.ldexp(1.99, rng.integers(-30, 30, (64, 16)))       # amax ~ 2^(t+1): v up to ~510
    X[rng.random(X.shape) < 0.05] *= 1e-4
    X[3, :32] = -0.0
    bits = wl.f64_to_bf16_bits(X)
    bits[5, 70] = 0x7F80                                               # +inf
    codes, scales, _ = gpu_quantize8(rfq, bits)
    assert_quant8_parity(oracle, bits, codes, scales)


@pytest.mark.parametrize("M,N,K", [(1, 8, 32), (128, 128, 128), (129, 264, 160), (300, 520, 1024), (64, 512, 32),
                                   (256, 256, 4096)])
def test_mxfp8_gemm_parity(rfq, oracle, M, N, K):
    import torch
    x = wl.random_matrix(M, K, seed=M + 3 * N + 7 * K, scale=2.0)
    w = wl.random_matrix(N, K, seed=M * N + K, scale=0.05)
    qa = rfq.quantize_mxfp8_alloc(dev_bf16(x))
    qw = rfq.quantize_mxfp8_alloc(dev_bf16(w))
    Y, S, _ = oracle.mxfp8_linear(x, w)
    for out in (torch.float32, torch.bfloat16):
        y = rfq.gemm_mxfp8_alloc(qa, qw, out_dtype=out)
        torch.cuda.synchronize()
        rfq.check_device_error()
        assert_y_close(y_to_numpy(y), Y, S, bf16_out=(out == torch.bfloat16), what=f"mxfp8 Y[{M}x{N}x{K}] {out}")


def test_mxfp8_gemm_ffn_shape_sampled(rfq, oracle):
    import torch
    wk = wl.ffn_up(0)
    rng = np.random.default_rng(5)
    rows = np.array(sorted(set(rng.choice(wk.M, 24, replace=False).tolist()) | {0, 127, 128, wk.M - 1}))
    qa = rfq.quantize_mxfp8_alloc(dev_bf16(wk.x_bits))
    qw = rfq.quantize_mxfp8_alloc(dev_bf16(wk.w_bits))
    y = rfq.gemm_mxfp8_alloc(qa, qw, out_dtype=torch.float32)
    torch.cuda.synchronize()
    rfq.check_device_error()
    qx = oracle.quantize_mxfp8_bf16(wk.x_bits[rows])
    qwo = oracle.quantize_mxfp8_bf16(wk.w_bits)
    A = oracle.dequantize_mxfp8(qx["codes"], qx["scales"])
    B = oracle.dequantize_mxfp8(qwo["codes"], qwo["scales"])
    Y, absY = oracle.gemm_blas(A, B)
    assert_y_close(y_to_numpy(y)[rows], Y, float(absY.max()), bf16_out=False, what="mxfp8 ffn rows")
