"""Kernel 1 (fused RFQ quantizer) against the CPU oracle: codes and scales bit-exact.

Covers the tiny and quantize-bandwidth workloads, ragged shapes (M not a
multiple of 128, K not a multiple of 128), every finite bf16 bit pattern, every
E2M1 tie point at several scales, subnormals, values near the bf16 maximum,
+-0 blocks and NaN/infinity blocks.
"""
import numpy as np
import pytest

from block_scaled_gemm_rfq_b200 import workloads as wl
from helpers import assert_quant_parity, gpu_quantize

pytestmark = pytest.mark.gpu


def test_tiny_rfq_quantize(rfq, oracle):
    w = wl.tiny(0)
    got, _ = gpu_quantize(rfq, w.x_bits, residual=True)
    assert_quant_parity(oracle, w.x_bits, got, residual=True)


def test_tiny_weight_quantize(rfq, oracle):
    w = wl.tiny(0)
    got, _ = gpu_quantize(rfq, w.w_bits, weight=True)
    assert_quant_parity(oracle, w.w_bits, got, residual=False)


@pytest.mark.parametrize("M,K", [(1, 32), (1, 64), (16, 96), (127, 160), (129, 256), (200, 384), (257, 1056),
                                 (33, 4096)])
def test_ragged_shapes(rfq, oracle, M, K):
    bits = wl.random_matrix(M, K, seed=M * 7 + K, scale=3.0)
    for residual in (True, False):
        got, _ = gpu_quantize(rfq, bits, residual=residual)
        assert_quant_parity(oracle, bits, got, residual=residual)


def test_every_finite_bf16_pattern(rfq, oracle):
    """All finite bf16 patterns, (a) shuffled into random blocks and (b) sorted by
    magnitude into consecutive blocks (so scaled values sweep the whole grid)."""
    bits = np.arange(1 << 16, dtype=np.uint32).astype(np.uint16)
    bits = bits[((bits >> 7) & 0xFF) != 0xFF]
    rng = np.random.default_rng(99)
    pad = (-bits.size) % 256
    a = np.concatenate([rng.permutation(bits), np.zeros(pad, np.uint16)]).reshape(-1, 256)
    mag = np.sort(bits & 0x7FFF)
    signs = rng.integers(0, 2, mag.size).astype(np.uint16) << 15
    b = np.concatenate([mag | signs, np.zeros(pad, np.uint16)]).reshape(-1, 256)
    for m in (a, b):
        got, _ = gpu_quantize(rfq, m, residual=True)
        assert_quant_parity(oracle, m, got, residual=True)


def test_tie_points_at_many_scales(rfq, oracle):
    """Blocks with amax exactly 4*2^t holding every E2M1 midpoint times 2^t, and the
    bf16 neighbours just below and above each midpoint."""
    mids = np.array([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0])
    rows = []
    for t in [-126, -100, -20, -3, 0, 1, 7, 50, 120, 124]:
        vals = np.ldexp(mids, t)
        vb = wl.f64_to_bf16_bits(vals)
        blk = np.concatenate([vb, vb - 1, vb + 1, vb | 0x8000, (vb - 1) | 0x8000, (vb + 1) | 0x8000,
                              wl.f64_to_bf16_bits(np.array([4.0 * 2.0 ** t])), np.array([0x8000], np.uint16),
                              np.array([0], np.uint16), wl.f64_to_bf16_bits(np.array([-6.0 * 2.0 ** t]))])
        blk = blk[:32] if blk.size >= 32 else np.concatenate([blk, np.zeros(32 - blk.size, np.uint16)])
        rows.append(np.tile(blk, 4))
    m = np.array(rows, dtype=np.uint16)
    got, _ = gpu_quantize(rfq, m, residual=True)
    assert_quant_parity(oracle, m, got, residual=True)


def test_special_blocks(rfq, oracle):
    rng = np.random.default_rng(5)
    m = wl.random_matrix(8, 256, seed=1)
    m[0, :32] = 0                                              # all +0
    m[0, 32:64] = 0x8000                                       # all -0
    m[1, :32] = rng.integers(1, 0x80, 32).astype(np.uint16)     # positive subnormals
    m[1, 32:64] = rng.integers(0x8001, 0x8080, 32).astype(np.uint16)  # negative subnormals
    m[2, :32] = 0x7F7F                                         # bf16 max
    m[2, 32:64] = rng.integers(0x7E00, 0x7F80, 32).astype(np.uint16)  # huge
    m[3, 5] = 0x7F80                                           # +inf
    m[3, 40] = 0xFF80                                          # -inf
    m[4, 70] = 0x7FC0                                          # NaN
    m[5, :32] = 0x0001                                         # smallest subnormal
    m[6, :32] = np.where(np.arange(32) % 2 == 0, 0x0080, 0x0001)   # smallest normal and subnormal
    got, _ = gpu_quantize(rfq, m, residual=True)
    ref = assert_quant_parity(oracle, m, got, residual=True)
    assert ref["scales_x"][3, 0] == 0xFF and ref["scales_x"][3, 1] == 0xFF and ref["scales_x"][4, 2] == 0xFF


@pytest.mark.parametrize("seed", [0, 1])
def test_quantize_bandwidth_workload_full(rfq, oracle, seed):
    """The 8192 x 4096 heavy-tailed workload, every byte compared."""
    w = wl.quantize_bandwidth(seed)
    got, _ = gpu_quantize(rfq, w.x_bits, residual=True)
    assert_quant_parity(oracle, w.x_bits, got, residual=True)


def test_repeated_calls_are_deterministic(rfq):
    import torch
    w = wl.tiny(2)
    a, qa = gpu_quantize(rfq, w.x_bits)
    b, qb = gpu_quantize(rfq, w.x_bits)
    for k in a:
        assert np.array_equal(a[k], b[k])
    assert torch.equal(qa.codes, qb.codes)
