"""Seeded synthetic inputs for the RFQ MXFP4 linear layer.

This module holds only input generation: no quantization, scaling or GEMM
arithmetic.  It is the one piece shared by the CUDA path's tests/benchmarks and by
the CPU oracle, so both see the same bf16 bytes.

Recipe (all host-side ``numpy.random.default_rng(seed)``, PCG64):
  * draws are float64, cast to float32 (round to nearest even) and then rounded
    to bf16 (round to nearest even) -> uint16 bit patterns;
  * an "outlier channel" is a column of X (a K index); the columns are picked by
    ``rng.choice(K, n, replace=False)`` and multiplied by the stated factor;
  * "spikes" are single (token, channel) elements picked by
    ``rng.choice(M*K, n, replace=False)`` and multiplied;
  * the draw order is: X body, outlier channels, spikes, then W.

The heavy-tailed bodies (Student-t, Laplace) plus outlier channels stand in for
the heavy-tailed activations with outlier channels that the RFQ paper
("Activation Outliers Matter: Robust Recovery for Quantized Multimodal LLMs",
section 1) identifies as the source of FP4 activation error; no dataset items
are used.
"""
from __future__ import annotations

from dataclasses import dataclass
from typing import Optional

import numpy as np


def f64_to_bf16_bits(a: np.ndarray) -> np.ndarray:
    """float64 -> float32 (RNE) -> bf16 (RNE) bit patterns as uint16.  Finite inputs only."""
    u = np.ascontiguousarray(a, dtype=np.float32).view(np.uint32)
    # finite float32 bit patterns are <= 0xFF7FFFFF, so the rounding add cannot wrap
    rounded = (u + np.uint32(0x7FFF) + ((u >> np.uint32(16)) & np.uint32(1))) >> np.uint32(16)
    return rounded.astype(np.uint16)


def bf16_bits_to_f32(bits: np.ndarray) -> np.ndarray:
    """bf16 bit patterns -> float32 values (exact)."""
    return (np.ascontiguousarray(bits, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


@dataclass
class Workload:
    name: str
    M: int
    K: int
    N: Optional[int]
    x_bits: np.ndarray                  # [M, K] uint16 (bf16 bits)
    w_bits: Optional[np.ndarray]        # [N, K] uint16 (bf16 bits) or None (quantize-only)
    y_fp32: bool                        # output type of the linear layer
    seed: int


def _outlier_channels(rng, X, count, factor):
    ch = rng.choice(X.shape[1], count, replace=False)
    X[:, ch] *= factor
    return ch


def tiny(seed: int = 0) -> Workload:
    """X 128x256 N(0,1) with channels 7 and 100 scaled x64; W 128x256 N(0, 0.02); Y fp32."""
    rng = np.random.default_rng(seed)
    X = rng.standard_normal((128, 256))
    X[:, [7, 100]] *= 64.0
    W = rng.normal(0.0, 0.02, (128, 256))
    return Workload("tiny_rfq_linear_M128_K256_N128", 128, 256, 128,
                    f64_to_bf16_bits(X), f64_to_bf16_bits(W), True, seed)


def quantize_bandwidth(seed: int = 0, M: int = 8192, K: int = 4096) -> Workload:
    """X 8192x4096, 0.5 * Student-t(nu=3), 1% of channels scaled x100; quantize only."""
    rng = np.random.default_rng(seed)
    X = 0.5 * rng.standard_t(3.0, (M, K))
    _outlier_channels(rng, X, int(round(0.01 * K)), 100.0)
    return Workload(f"rfq_quantize_M{M}_K{K}", M, K, None, f64_to_bf16_bits(X), None, False, seed)


def ffn_up(seed: int = 0, M: int = 4096, K: int = 4096, N: int = 12288) -> Workload:
    """LLM FFN up-projection: X N(0,1) + 0.5% channels x50 + 0.01% spikes x500; W N(0,0.02); Y bf16."""
    rng = np.random.default_rng(seed)
    X = rng.standard_normal((M, K))
    _outlier_channels(rng, X, int(round(0.005 * K)), 50.0)
    n_spikes = int(round(1e-4 * M * K))
    idx = rng.choice(M * K, n_spikes, replace=False)
    X.reshape(-1)[idx] *= 500.0
    W = rng.normal(0.0, 0.02, (N, K))
    return Workload(f"rfq_linear_ffn_up_M{M}_K{K}_N{N}", M, K, N,
                    f64_to_bf16_bits(X), f64_to_bf16_bits(W), False, seed)


def dit_ffn(seed: int = 0, M: int = 32768, K: int = 5120, N: int = 13824) -> Workload:
    """Video-DiT FFN: X Laplace(0,1) + 8 channels x80; W N(0, 0.015); Y bf16."""
    rng = np.random.default_rng(seed)
    X = rng.laplace(0.0, 1.0, (M, K))
    _outlier_channels(rng, X, 8, 80.0)
    W = rng.normal(0.0, 0.015, (N, K))
    return Workload(f"rfq_linear_dit_ffn_M{M}_K{K}_N{N}", M, K, N,
                    f64_to_bf16_bits(X), f64_to_bf16_bits(W), False, seed)


SWEEP_M = (16, 64, 256, 1024, 4096, 16384)


def m_sweep(M: int, seed: int = 0, K: int = 4096, N: int = 4096) -> Workload:
    """rfq_linear sweep point: X Student-t(nu=3) + 1% channels x100; W N(0, 0.02); Y bf16."""
    rng = np.random.default_rng(seed)
    X = rng.standard_t(3.0, (M, K))
    _outlier_channels(rng, X, int(round(0.01 * K)), 100.0)
    W = rng.normal(0.0, 0.02, (N, K))
    return Workload(f"rfq_linear_sweep_M{M}_K{K}_N{N}", M, K, N,
                    f64_to_bf16_bits(X), f64_to_bf16_bits(W), False, seed)


def random_matrix(rows: int, K: int, seed: int, scale: float = 1.0) -> np.ndarray:
    """Plain N(0, scale) bf16 matrix for edge-shape tests."""
    rng = np.random.default_rng(seed)
    return f64_to_bf16_bits(scale * rng.standard_normal((rows, K)))
