"""Full-size parity on every benchmark workload: the CUDA path against the oracle on
whole matrices, not samples.

* Codes and E8M0 scales (MMA layout, padding included) of Q(X), Q(R) and Q(W) are
  compared byte for byte with the oracle's for the LLM FFN up-projection
  (X 4096 x 4096, W 12288 x 4096), the video-DiT FFN (X 32768 x 5120,
  W 13824 x 5120) and every point of the rfq_linear M sweep (K = N = 4096).
* Y is compared in fp32 against the oracle's float64 product within 1e-5 * S on
  every row of the FFN and DiT GEMMs and of every M-sweep layer (with and without
  the residual path), and bf16 Y within one bf16 ulp + 1e-5 * S.  The DiT product
  (32768 x 13824 outputs over 2 x 5120 terms) is recomputed in row chunks; S is
  taken over each chunk's rows, which is never more than the whole matrix's S, so
  the bound is if anything stricter.

Nothing the GPU computed is fed to the oracle: both sides quantize the same seeded
bf16 bytes.
"""
import numpy as np
import pytest

from block_scaled_gemm_rfq_b200 import workloads as wl
from helpers import assert_quant_parity, assert_y_close, dev_bf16, gpu_quantize, y_to_numpy

pytestmark = pytest.mark.gpu

CHUNK = 2048   # rows of the oracle's float64 product per step


@pytest.fixture(scope="module")
def ffn():
    return wl.ffn_up(0)


@pytest.fixture(scope="module")
def dit():
    return wl.dit_ffn(0)


def _gpu_y(rfq, x_bits, w_bits, residual, out_dtype, linear=False):
    import torch
    x, w = dev_bf16(x_bits), dev_bf16(w_bits)
    qw = rfq.quantize_weight_alloc(w)
    if linear:
        y = rfq.linear_alloc(x, qw, out_dtype=out_dtype, use_residual=residual)
    else:
        qa = rfq.quantize_mxfp4_alloc(x, residual=residual)
        y = rfq.gemm_alloc(qa, qw, out_dtype=out_dtype, use_residual=residual)
    torch.cuda.synchronize()
    rfq.check_device_error()
    out = y_to_numpy(y)
    del x, w, qw, y
    torch.cuda.empty_cache()
    return out


def _compare_rows(oracle, y_by_dtype, x_bits, qw, residual, rows, what):
    """The oracle's Y for X[rows] (quantized by the oracle) against each GPU Y."""
    qa = oracle.quantize_bf16(np.ascontiguousarray(x_bits[rows]), residual=residual)
    A, B = oracle.rfq_operands(qa, qw, residual)
    Y, absY = oracle.gemm_blas(A, B)
    S = float(absY.max())
    for bf16_out, y in y_by_dtype.items():
        assert_y_close(y[rows], Y, S, bf16_out=bf16_out, what=f"{what} rows {rows[0]}..{rows[-1]}")


def _compare_all_rows(oracle, y_by_dtype, x_bits, w_bits, residual, what):
    qw = oracle.quantize_bf16(w_bits, residual=False)
    M = x_bits.shape[0]
    for r0 in range(0, M, CHUNK):
        _compare_rows(oracle, y_by_dtype, x_bits, qw, residual, np.arange(r0, min(M, r0 + CHUNK)), what)


def _one_row_per_tile(M, seed):
    rng = np.random.default_rng(seed)
    rows = [t + int(rng.integers(0, min(128, M - t))) for t in range(0, M, 128)]
    return np.array(sorted(set(rows) | {0, M - 1}))


# --------------------------------------------------------------------------- codes and scales
def test_ffn_activation_codes_full(rfq, oracle, ffn):
    got, _ = gpu_quantize(rfq, ffn.x_bits, residual=True)
    assert_quant_parity(oracle, ffn.x_bits, got, residual=True)


@pytest.mark.parametrize("seed", [1, 2])
def test_activation_codes_full_other_seeds(rfq, oracle, seed):
    """The repeat-parity seeds of the FFN and DiT activations (and the FFN weight)."""
    wk = wl.ffn_up(seed)
    got, _ = gpu_quantize(rfq, wk.x_bits, residual=True)
    assert_quant_parity(oracle, wk.x_bits, got, residual=True)
    got, _ = gpu_quantize(rfq, wk.w_bits, residual=False, weight=True)
    assert_quant_parity(oracle, wk.w_bits, got, residual=False)
    dk = wl.dit_ffn(seed)
    got, _ = gpu_quantize(rfq, dk.x_bits, residual=True)
    assert_quant_parity(oracle, dk.x_bits, got, residual=True)


def test_ffn_weight_codes_full(rfq, oracle, ffn):
    got, _ = gpu_quantize(rfq, ffn.w_bits, residual=False, weight=True)
    assert_quant_parity(oracle, ffn.w_bits, got, residual=False)


def test_dit_activation_codes_full(rfq, oracle, dit):
    got, _ = gpu_quantize(rfq, dit.x_bits, residual=True)
    assert_quant_parity(oracle, dit.x_bits, got, residual=True)


def test_dit_weight_codes_full(rfq, oracle, dit):
    got, _ = gpu_quantize(rfq, dit.w_bits, residual=False, weight=True)
    assert_quant_parity(oracle, dit.w_bits, got, residual=False)


@pytest.mark.parametrize("M", wl.SWEEP_M)
def test_m_sweep_codes_full(rfq, oracle, M):
    wk = wl.m_sweep(M)
    got, _ = gpu_quantize(rfq, wk.x_bits, residual=True)
    assert_quant_parity(oracle, wk.x_bits, got, residual=True)
    got, _ = gpu_quantize(rfq, wk.x_bits, residual=False)
    assert_quant_parity(oracle, wk.x_bits, got, residual=False)
    if M == wl.SWEEP_M[0]:
        got, _ = gpu_quantize(rfq, wk.w_bits, residual=False, weight=True)
        assert_quant_parity(oracle, wk.w_bits, got, residual=False)


# --------------------------------------------------------------------------- Y
@pytest.mark.parametrize("residual", [True, False])
def test_ffn_y_every_row(rfq, oracle, ffn, residual):
    import torch
    ys = {False: _gpu_y(rfq, ffn.x_bits, ffn.w_bits, residual, torch.float32),
          True: _gpu_y(rfq, ffn.x_bits, ffn.w_bits, residual, torch.bfloat16)}
    _compare_all_rows(oracle, ys, ffn.x_bits, ffn.w_bits, residual, f"FFN residual={residual}")


def test_dit_y_every_row_fp32(rfq, oracle, dit):
    """Every one of the 32768 rows (all 128 pair-tile rows of the persistent schedule)."""
    import torch
    ys = {False: _gpu_y(rfq, dit.x_bits, dit.w_bits, True, torch.float32)}
    _compare_all_rows(oracle, ys, dit.x_bits, dit.w_bits, True, "DiT fp32")


@pytest.mark.parametrize("residual", [True, False])
def test_dit_y_bf16_and_off_every_tile(rfq, oracle, dit, residual):
    """bf16 Y with the residual path, and both outputs without it, on one row of every
    128-row tile (plus the first and last rows)."""
    import torch
    ys = {True: _gpu_y(rfq, dit.x_bits, dit.w_bits, residual, torch.bfloat16)}
    if not residual:
        ys[False] = _gpu_y(rfq, dit.x_bits, dit.w_bits, residual, torch.float32)
    qw = oracle.quantize_bf16(dit.w_bits, residual=False)
    _compare_rows(oracle, ys, dit.x_bits, qw, residual, _one_row_per_tile(dit.M, 7 + residual),
                  f"DiT residual={residual}")


@pytest.mark.parametrize("M", wl.SWEEP_M)
@pytest.mark.parametrize("residual", [True, False])
def test_m_sweep_linear_every_row(rfq, oracle, M, residual):
    """rfq_linear (the single-kernel layer for M <= 32, the quantizer and the split-K
    or tiled GEMM above) in fp32 and bf16, every row."""
    import torch
    wk = wl.m_sweep(M)
    ys = {False: _gpu_y(rfq, wk.x_bits, wk.w_bits, residual, torch.float32, linear=True),
          True: _gpu_y(rfq, wk.x_bits, wk.w_bits, residual, torch.bfloat16, linear=True)}
    _compare_all_rows(oracle, ys, wk.x_bits, wk.w_bits, residual, f"sweep M={M} residual={residual}")
