"""The seeded input generators follow their stated recipe: bf16 rounding, seeds,
outlier channels (count and factor) and spikes, checked on reduced sizes from the
values themselves (not by replaying the draws)."""
import numpy as np

from block_scaled_gemm_rfq_b200 import workloads as wl


def _values(bits):
    return wl.bf16_bits_to_f32(bits).astype(np.float64)


def _outlier_columns(X, ratio=10.0):
    """Columns whose median magnitude exceeds `ratio` times the median column's."""
    med = np.median(np.abs(X), axis=0)
    return np.flatnonzero(med > ratio * np.median(med)), med


def test_bf16_rounding_matches_torch_rne():
    import torch
    rng = np.random.default_rng(3)
    a = np.concatenate([rng.standard_normal(100000) * 10.0 ** rng.integers(-30, 30, 100000),
                        [0.0, -0.0, 1.0 + 2.0 ** -8, 1.0 + 3 * 2.0 ** -8, -(1.0 + 2.0 ** -8), 3.0e38, -3.0e38]])
    ref = torch.from_numpy(a.astype(np.float32)).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(wl.f64_to_bf16_bits(a), ref)


def test_generators_are_deterministic_per_seed():
    a, b, c = wl.m_sweep(16, seed=0), wl.m_sweep(16, seed=0), wl.m_sweep(16, seed=1)
    assert np.array_equal(a.x_bits, b.x_bits) and np.array_equal(a.w_bits, b.w_bits)
    assert not np.array_equal(a.x_bits, c.x_bits)


def test_tiny_recipe():
    w = wl.tiny(0)
    assert (w.M, w.K, w.N, w.y_fp32) == (128, 256, 128, True)
    cols, med = _outlier_columns(_values(w.x_bits))
    assert cols.tolist() == [7, 100]
    assert 30 < med[7] / np.median(med) < 130
    W = _values(w.w_bits)
    assert abs(W.std() - 0.02) < 0.002


def test_quantize_bandwidth_recipe():
    w = wl.quantize_bandwidth(0, M=512, K=4096)
    X = _values(w.x_bits)
    cols, med = _outlier_columns(X)
    assert cols.size == round(0.01 * 4096)                     # 41 channels
    assert 60 < np.median(med[cols]) / np.median(med) < 160    # scaled x100
    body = np.delete(X, cols, axis=1)
    assert 0.3 < np.median(np.abs(body)) < 0.5                 # 0.5 * t(3): median |t3| ~ 0.765


def test_ffn_up_recipe():
    M, K, N = 1024, 4096, 256
    w = wl.ffn_up(0, M=M, K=K, N=N)
    X = _values(w.x_bits)
    cols, med = _outlier_columns(X)
    assert cols.size == round(0.005 * K)                       # 20 channels x50
    assert 30 < np.median(med[cols]) / np.median(med) < 80
    body = np.delete(X, cols, axis=1)
    n_spikes = round(1e-4 * M * K)
    big = int((np.abs(body) > 20.0).sum())                    # spikes x500 of N(0,1); the body stays < 7
    assert 0.85 * n_spikes <= big <= n_spikes
    assert abs(_values(w.w_bits).std() - 0.02) < 0.001


def test_dit_and_sweep_recipes():
    w = wl.dit_ffn(0, M=512, K=5120, N=128)
    cols, med = _outlier_columns(_values(w.x_bits))
    assert cols.size == 8 and 50 < np.median(med[cols]) / np.median(med) < 120
    assert abs(_values(w.w_bits).std() - 0.015) < 0.001
    s = wl.m_sweep(64, seed=0)
    assert (s.M, s.K, s.N) == (64, 4096, 4096)
    cols, _ = _outlier_columns(_values(s.x_bits))
    assert cols.size == round(0.01 * 4096)
