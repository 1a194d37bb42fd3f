"""Pins of the CPU oracle against things other than itself (CPU only).

Each test ties one oracle function to a third-party codec, a brute-force search,
a closed form or an invariant that the mathematics of RFQ fixes, so that a
dropped term, a wrong sign or index, or a transposed operand in the oracle fails
at least one of them.  The method is from "Activation Outliers Matter: Robust
Recovery for Quantized Multimodal LLMs" (section 1, RFQ contribution paragraph;
abstract); the MXFP4 element/scale rule is OCP MX v1.0 (the pages stop before
defining it, at section 3.1).
"""
import math

import ml_dtypes
import numpy as np
import pytest

from block_scaled_gemm_rfq_b200 import workloads as wl

F4 = ml_dtypes.float4_e2m1fn


# --------------------------------------------------------------------------- E2M1 decode
def test_e2m1_decode_matches_ml_dtypes(oracle):
    third_party = np.arange(16, dtype=np.uint8).view(F4).astype(np.float64)
    mine = np.array([oracle.e2m1_value(c) for c in range(16)])
    np.testing.assert_array_equal(mine, third_party)
    # sign of zero is carried by code 8
    assert math.copysign(1.0, oracle.e2m1_value(8)) == -1.0


def test_e2m1_decode_matches_transformers_table(oracle):
    mx = pytest.importorskip("transformers.integrations.mxfp4")
    mine = [oracle.e2m1_value(c) for c in range(16)]
    assert mine == list(mx.FP4_VALUES)


# --------------------------------------------------------------------------- E8M0 decode
def test_e8m0_decode_matches_torch_and_ml_dtypes(oracle):
    import torch
    bytes_ = np.arange(256, dtype=np.uint8)
    want_torch = torch.from_numpy(bytes_.copy()).view(torch.float8_e8m0fnu).to(torch.float64).numpy()
    want_mld = bytes_.view(ml_dtypes.float8_e8m0fnu).astype(np.float64)
    # dequantize a row whose every code is 2 (value 1.0): DQ = 2^(scale-127)
    codes = np.full((256, 16), 0x22, np.uint8)          # 32 elements, all code 2
    scales = bytes_.reshape(256, 1)
    dq = oracle.dequantize(codes, scales)[:, 0]
    np.testing.assert_array_equal(dq[:255], want_torch[:255])
    np.testing.assert_array_equal(dq[:255], want_mld[:255])
    assert math.isnan(dq[255]) and math.isnan(want_torch[255])


# --------------------------------------------------------------------------- scale rule
def _brute_exponent(amax: float) -> int:
    """The unique e in [-127, 127] with 4 <= amax * 2^-e < 8, by search; -127 if amax is below range."""
    if amax == 0.0:
        return -127
    for e in range(-127, 128):
        v = math.ldexp(amax, -e)
        if 4.0 <= v < 8.0:
            return e
    assert amax < math.ldexp(4.0, -127), amax
    return -127


def test_block_exponent_brute_force(oracle):
    rng = np.random.default_rng(123)
    cands = [0.0, 1.0, 4.0, 6.0, 7.999, 8.0, 2.0 ** -126, 2.0 ** -133, 2.0 ** -125,
             2.0 ** -125 * 0.999, 3.0e38, 2.0 ** 127, np.nextafter(2.0, 0), np.nextafter(2.0, 3)]
    cands += list(np.exp(rng.uniform(-90, 88, 2000)))
    # every finite positive bf16 value
    bits = np.arange(1, 0x7F80, dtype=np.uint16)
    cands += list(wl.bf16_bits_to_f32(bits).astype(np.float64)[::7])
    for a in cands:
        assert oracle.block_exponent(a) == _brute_exponent(float(a)), a
    assert oracle.block_exponent(float("inf")) == 128
    assert oracle.block_exponent(float("nan")) == 128


# --------------------------------------------------------------------------- element rounding
def _all_finite_bf16():
    bits = np.arange(0, 1 << 16, dtype=np.uint32).astype(np.uint16)
    vals = wl.bf16_bits_to_f32(bits)
    keep = np.isfinite(vals)
    return bits[keep], vals[keep].astype(np.float64)


@pytest.mark.parametrize("e", [-127, -20, -1, 0, 3, 60, 125])
def test_element_encode_exhaustive_vs_ml_dtypes(oracle, e):
    """Every finite bf16 x that fits a block with exponent e (|x| 2^-e < 8):
    the oracle's code equals ml_dtypes' RNE/saturating float4_e2m1fn cast of the
    exactly scaled value."""
    _, x = _all_finite_bf16()
    v = np.ldexp(x, -e)                   # exact in float64
    keep = np.abs(v) < 8.0
    x, v = x[keep], v[keep]
    want = v.astype(np.float32).astype(F4).view(np.uint8)
    got = np.array([oracle.e2m1_encode(xi, e) for xi in x], dtype=np.uint8)
    bad = np.nonzero(got != want)[0]
    assert bad.size == 0, (x[bad[:5]], got[bad[:5]], want[bad[:5]])


def test_element_encode_matches_rint_formulation(oracle):
    """Round-half-even onto the E2M1 grid written as a different algorithm: the grid
    spacing is 0.5 below 2, 1 in [2, 4), 2 from 4; round v/spacing with numpy's
    rint (half to even integer = even mantissa) and clamp to 6."""
    v = np.linspace(0.0, 7.999, 40001)
    v = np.concatenate([v, [0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0, 6.0, 7.0]])
    spacing = np.where(v < 2.0, 0.5, np.where(v < 4.0, 1.0, 2.0))
    q = np.minimum(np.rint(v / spacing) * spacing, 6.0)
    got = np.array([oracle.e2m1_value(oracle.e2m1_encode(vi, 0)) for vi in v])
    np.testing.assert_array_equal(got, q)


def test_ties_and_saturation_table(oracle):
    # midpoints go to the neighbour with mantissa bit 0; >= 6 saturates; sign kept
    table = {0.25: 0.0, 0.75: 1.0, 1.25: 1.0, 1.75: 2.0, 2.5: 2.0, 3.5: 4.0, 5.0: 4.0,
             6.0: 6.0, 7.0: 6.0, 7.99: 6.0, 0.2499: 0.0, 0.2501: 0.5}
    for v, q in table.items():
        assert oracle.e2m1_value(oracle.e2m1_encode(v, 0)) == q
        assert oracle.e2m1_value(oracle.e2m1_encode(-v, 0)) == -q
    assert oracle.e2m1_encode(-0.0, 0) == 0x8
    assert oracle.e2m1_encode(-0.1, 0) == 0x8
    assert oracle.e2m1_encode(0.0, 0) == 0x0


# --------------------------------------------------------------------------- block quantizer
def test_qdq_identity_on_representable_blocks(oracle):
    """Blocks of grid values times 2^t whose amax is 4*2^t or 6*2^t are reproduced
    exactly by DQ(Q(x)); their residual is zero, so Q(R) is all code 0, scale 0."""
    rng = np.random.default_rng(7)
    grid = np.array([0, 0.5, 1, 1.5, 2, 3, 4, 6])
    rows = []
    for t in [-120, -30, -3, 0, 2, 40, 100]:
        for top in (4.0, 6.0):
            g = rng.choice(grid[grid <= top], 32) * rng.choice([-1.0, 1.0], 32)
            g[rng.integers(32)] = top * rng.choice([-1.0, 1.0])
            rows.append(np.ldexp(g, t))
    X = np.array(rows)
    bits = wl.f64_to_bf16_bits(X)
    assert np.array_equal(wl.bf16_bits_to_f32(bits).astype(np.float64), X)
    q = oracle.quantize_bf16(bits)
    np.testing.assert_array_equal(oracle.dequantize(q["codes_x"], q["scales_x"]), X)
    assert not (q["codes_r"] & 0x7).any()
    assert not q["scales_r"].any()


def _rand_heavy(rows, K, seed):
    rng = np.random.default_rng(seed)
    X = rng.standard_t(3.0, (rows, K))
    X[:, rng.choice(K, max(1, K // 50), replace=False)] *= 100.0
    X[rng.random((rows, K)) < 0.01] *= 1e-30          # tiny values next to large ones
    return wl.f64_to_bf16_bits(X)


def test_residual_is_full_error_and_requantized_by_same_rule(oracle):
    """Q(R) from the bf16 quantizer equals the plain-float64 quantizer applied to
    R = X - DQ(Q(X)) computed here by dequantization (two code paths)."""
    bits = _rand_heavy(64, 512, 11)
    X = wl.bf16_bits_to_f32(bits).astype(np.float64)
    q = oracle.quantize_bf16(bits)
    R = X - oracle.dequantize(q["codes_x"], q["scales_x"])
    codes_r, scales_r = oracle.quantize_f64(R)
    np.testing.assert_array_equal(codes_r, q["codes_r"])
    np.testing.assert_array_equal(scales_r, q["scales_r"])
    # R is exactly representable in fp32 (and in bf16: test_residual_is_exact_in_bf16)
    np.testing.assert_array_equal(R.astype(np.float32).astype(np.float64), R)


def test_residual_is_exact_in_bf16(oracle):
    """|r| <= |x| elementwise (0 is a grid point) and r is a multiple of x's bf16 ulp
    (DQ is a multiple of 2^(e-1), e >= e_x - 2), so R = X - DQ(Q(X)) is itself a bf16
    value: computing it with one bf16 FMA involves no rounding."""
    for seed in (14, 15):
        bits = _rand_heavy(128, 1024, seed)
        X = wl.bf16_bits_to_f32(bits).astype(np.float64)
        q = oracle.quantize_bf16(bits)
        R = X - oracle.dequantize(q["codes_x"], q["scales_x"])
        assert np.all(np.abs(R) <= np.abs(X))
        r32 = R.astype(np.float32)
        np.testing.assert_array_equal(r32.astype(np.float64), R)
        assert np.all((r32.view(np.uint32) & 0xFFFF) == 0), "a residual needs more than bf16 precision"
    # every bf16 magnitude in [2^-8, 8) against scale 2^0 (block amax fixed at 7.5 -> e = 0)
    mags = np.arange(0x3B80, 0x4100, dtype=np.uint16)            # 2^-8 .. just below 8
    mags = mags[(mags & 0x7F80) != 0x7F80]
    n = (len(mags) + 30) // 31 * 31
    blk = np.full(n, mags[0], np.uint16)
    blk[: len(mags)] = mags
    blk = blk.reshape(-1, 31)
    rows = np.concatenate([blk, np.full((blk.shape[0], 1), 0x40F0, np.uint16)], axis=1)  # 7.5 sets e = 0
    q = oracle.quantize_bf16(rows)
    assert np.all(q["scales_x"] == 127)
    X = wl.bf16_bits_to_f32(rows).astype(np.float64)
    R = X - oracle.dequantize(q["codes_x"], q["scales_x"])
    assert np.all((R.astype(np.float32).view(np.uint32) & 0xFFFF) == 0)


def test_residual_never_increases_error(oracle):
    """Elementwise |r - DQ(Q(r))| <= |r| (0 is on the grid), hence on every block
    ||X - DQ(QX) - DQ(QR)|| <= ||X - DQ(QX)||."""
    bits = _rand_heavy(128, 1024, 12)
    X = wl.bf16_bits_to_f32(bits).astype(np.float64)
    q = oracle.quantize_bf16(bits)
    DX = oracle.dequantize(q["codes_x"], q["scales_x"])
    DR = oracle.dequantize(q["codes_r"], q["scales_r"])
    R = X - DX
    assert np.all(np.abs(R - DR) <= np.abs(R))
    e1 = ((R) ** 2).reshape(128, -1, 32).sum(-1)
    e2 = ((R - DR) ** 2).reshape(128, -1, 32).sum(-1)
    assert np.all(e2 <= e1)
    assert e2.sum() < 0.1 * e1.sum()          # the residual path recovers most of the error


def test_residual_scale_invariant(oracle):
    """|r| < 2^(e_X + 1) so the residual scale byte is <= max(byte_X - 2, 0)."""
    bits = _rand_heavy(128, 1024, 13)
    q = oracle.quantize_bf16(bits)
    sx = q["scales_x"].astype(int)
    sr = q["scales_r"].astype(int)
    assert np.all(sr <= np.maximum(sx - 2, 0))


def test_all_zero_and_signed_zero_blocks(oracle):
    bits = np.zeros((2, 64), np.uint16)
    bits[1, :] = 0x8000                                    # -0.0
    q = oracle.quantize_bf16(bits)
    assert not q["scales_x"].any() and not q["scales_r"].any()
    assert not q["codes_x"][0].any()
    assert np.all(q["codes_x"][1] == 0x88)
    # IEEE: r = (-0) - (-0) = +0, so the residual of a -0 block is +0
    assert not q["codes_r"][1].any()


def test_nonfinite_block_gets_nan_scale(oracle):
    bits = wl.random_matrix(2, 64, seed=3)
    bits[0, 5] = 0x7F80          # +inf in block 0 of row 0
    bits[1, 40] = 0x7FC0         # NaN in block 1 of row 1
    q = oracle.quantize_bf16(bits)
    assert q["scales_x"][0, 0] == 0xFF and q["scales_r"][0, 0] == 0xFF
    assert q["scales_x"][1, 1] == 0xFF and q["scales_r"][1, 1] == 0xFF
    assert q["scales_x"][0, 1] != 0xFF and q["scales_x"][1, 0] != 0xFF


def test_subnormal_blocks(oracle):
    """bf16 subnormals: the exponent clamps to -127 (byte 0) and nothing is flushed."""
    bits = np.zeros((1, 32), np.uint16)
    bits[0, :] = np.arange(1, 33, dtype=np.uint16)        # 1..32 x 2^-133
    q = oracle.quantize_bf16(bits)
    assert q["scales_x"][0, 0] == 0
    X = wl.bf16_bits_to_f32(bits).astype(np.float64)
    dx = oracle.dequantize(q["codes_x"], q["scales_x"])
    # scaled values are 2^-6 .. 2^-1: 2^127 * 32 * 2^-133 = 0.5, the largest becomes code 1
    assert dx[0, -1] == X[0, -1]
    assert q["codes_x"][0, -1] >> 4 == 1


# --------------------------------------------------------------------------- reference GEMM
def test_gemm_loops_match_blas_and_closed_forms(oracle):
    rng = np.random.default_rng(5)
    A = rng.standard_normal((37, 96))
    B = rng.standard_normal((23, 96))
    Y, absY = oracle.gemm_loops(A, B)
    Yb, absYb = oracle.gemm_blas(A, B)
    np.testing.assert_allclose(Y, Yb, rtol=0, atol=1e-12)
    np.testing.assert_allclose(absY, absYb, rtol=1e-14)
    # closed form: B = identity rows picks columns of A
    I = np.eye(96)[:23]
    Yi, _ = oracle.gemm_loops(A, I)
    np.testing.assert_array_equal(Yi, A[:, :23])
    # transposition check: swapping operands transposes Y
    Yt, _ = oracle.gemm_loops(B, A)
    np.testing.assert_array_equal(Yt, Y.T)


def test_rfq_gemm_is_sum_of_two_terms(oracle):
    """Y = DQ(QX).DQ(QW)^T + DQ(QR).DQ(QW)^T, and with RFQ off the first term alone."""
    w = wl.tiny(0)
    Y, S, _ = oracle.rfq_linear(w.x_bits, w.w_bits, residual=True)
    Yoff, Soff, _ = oracle.rfq_linear(w.x_bits, w.w_bits, residual=False)
    qa = oracle.quantize_bf16(w.x_bits)
    qw = oracle.quantize_bf16(w.w_bits, residual=False)
    DX = oracle.dequantize(qa["codes_x"], qa["scales_x"])
    DR = oracle.dequantize(qa["codes_r"], qa["scales_r"])
    DW = oracle.dequantize(qw["codes_x"], qw["scales_x"])
    np.testing.assert_allclose(Y, DX @ DW.T + DR @ DW.T, rtol=0, atol=1e-9 * S)
    np.testing.assert_allclose(Yoff, DX @ DW.T, rtol=0, atol=1e-9 * Soff)
    assert S >= Soff


def test_rfq_recovers_activation_fidelity(oracle):
    """The paper's central claim on synthetic heavy-tailed inputs: adding the
    residual term brings Y much closer to the unquantized product X.W^T."""
    w = wl.tiny(0)
    X = wl.bf16_bits_to_f32(w.x_bits).astype(np.float64)
    W = wl.bf16_bits_to_f32(w.w_bits).astype(np.float64)
    exact = X @ W.T
    Y, _, _ = oracle.rfq_linear(w.x_bits, w.w_bits, residual=True)
    Yoff, _, _ = oracle.rfq_linear(w.x_bits, w.w_bits, residual=False)
    assert np.linalg.norm(Y - exact) < 0.8 * np.linalg.norm(Yoff - exact)
    # activation error alone (weights held at DQ(QW)): the residual path removes most of it
    qw = oracle.quantize_bf16(w.w_bits, residual=False)
    act_only = X @ oracle.dequantize(qw["codes_x"], qw["scales_x"]).T
    assert np.linalg.norm(Y - act_only) < 0.3 * np.linalg.norm(Yoff - act_only)


# --------------------------------------------------------------------------- scale layout
def _representable(rows, cols, seed, axis):
    """bf16 matrix whose 32-element blocks along `axis` are exactly MXFP4: grid
    values times a per-block power of two (block max on the grid's top codes)."""
    rng = np.random.default_rng(seed)
    grid = np.array([0, .5, 1, 1.5, 2, 3, 4, 6])
    vals = rng.choice(grid, (rows, cols)) * rng.choice([-1.0, 1.0], (rows, cols))
    if axis == 1:
        v = vals.reshape(rows, cols // 32, 32)
        v[:, :, 0] = 6.0
        v *= np.exp2(rng.integers(-20, 20, (rows, cols // 32, 1)))
        vals = v.reshape(rows, cols)
    else:
        v = vals.reshape(rows // 32, 32, cols)
        v[:, 0, :] = 6.0
        v *= np.exp2(rng.integers(-20, 20, (rows // 32, 1, cols)))
        vals = v.reshape(rows, cols)
    return wl.f64_to_bf16_bits(vals), vals


def test_transposed_quantizer_definition_and_identity(oracle):
    """quantize_transposed(X) is the row rule on X^T; on blocks exactly
    representable along the rows of X it dequantizes to X^T exactly, with an
    all-zero residual."""
    bits, vals = _representable(96, 40, 31, axis=0)
    q = oracle.quantize_transposed(bits)
    np.testing.assert_array_equal(oracle.dequantize(q["codes_x"], q["scales_x"]), vals.T)
    assert not q["codes_r"].any() and not q["scales_r"].any()
    q2 = oracle.quantize_bf16(np.ascontiguousarray(bits.T))
    for k in q:
        np.testing.assert_array_equal(q[k], q2[k])


def test_backward_gemms_straight_through_closed_form(oracle):
    """With operands exactly MXFP4 along each GEMM's contraction axis, the
    straight-through backward GEMMs are the plain products dX = dY . W and
    dW = dY^T . X (float64, exact inputs)."""
    M, N, K = 64, 64, 96
    dy_bits, dy = _representable(M, N, 41, axis=1)     # dgrad: dY along N (its rows)
    w_bits, w = _representable(N, K, 42, axis=0)       # dgrad: W along N (its columns)
    dX, S, _ = oracle.rfq_dgrad(dy_bits, w_bits)
    np.testing.assert_allclose(dX, dy @ w, rtol=0, atol=1e-12 * S)
    x_bits, x = _representable(M, K, 43, axis=0)       # wgrad: X along M (its columns)
    dy2_bits, dy2 = _representable(M, N, 44, axis=0)   # wgrad: dY along M
    dW, S2, _ = oracle.rfq_wgrad(x_bits, dy2_bits)
    np.testing.assert_allclose(dW, dy2.T @ x, rtol=0, atol=1e-12 * S2)
    # and on general inputs the wgrad residual term is the RFQ term of X^T
    xg = _rand_heavy(64, 96, 45)
    dW_on, _, _ = oracle.rfq_wgrad(xg, dy2_bits, residual=True)
    dW_off, _, _ = oracle.rfq_wgrad(xg, dy2_bits, residual=False)
    exact = dy2.T @ wl.bf16_bits_to_f32(xg).astype(np.float64)
    assert np.linalg.norm(dW_on - exact) < np.linalg.norm(dW_off - exact)


def test_mma_scale_layout_known_offsets_and_bijection(oracle):
    Kb = 10                                   # Kb_pad = 12 -> 3 atoms per 128-row tile
    assert oracle.mma_scale_offset(0, 0, Kb) == 0
    assert oracle.mma_scale_offset(0, 1, Kb) == 1
    assert oracle.mma_scale_offset(0, 3, Kb) == 3
    assert oracle.mma_scale_offset(1, 0, Kb) == 16
    assert oracle.mma_scale_offset(31, 0, Kb) == 31 * 16
    assert oracle.mma_scale_offset(32, 0, Kb) == 4
    assert oracle.mma_scale_offset(96, 2, Kb) == 14
    assert oracle.mma_scale_offset(0, 4, Kb) == 512
    assert oracle.mma_scale_offset(128, 0, Kb) == 3 * 512
    rows = 200
    offs = {oracle.mma_scale_offset(r, c, Kb) for r in range(256) for c in range(12)}
    assert offs == set(range(256 * 12))
    plain = np.random.default_rng(0).integers(1, 255, (rows, Kb), dtype=np.uint8)
    lay = oracle.scales_to_mma_layout(plain)
    assert lay.size == 256 * 12
    back = np.array([[lay[oracle.mma_scale_offset(r, c, Kb)] for c in range(Kb)] for r in range(rows)])
    np.testing.assert_array_equal(back, plain)
    assert int(lay.astype(np.int64).sum()) == int(plain.astype(np.int64).sum())   # padding is 0


def test_workload_generators_are_seeded():
    a = wl.tiny(0)
    b = wl.tiny(0)
    c = wl.tiny(1)
    assert np.array_equal(a.x_bits, b.x_bits) and np.array_equal(a.w_bits, b.w_bits)
    assert not np.array_equal(a.x_bits, c.x_bits)
    X = wl.bf16_bits_to_f32(a.x_bits)
    assert np.abs(X[:, 7]).mean() > 20 and np.abs(X[:, 8]).mean() < 2


# --------------------------------------------------------------------------- regression + isolation
def test_oracle_matches_committed_golden_digest(oracle):
    """tests/golden/tiny_oracle_digest.json was written by tests/golden/make_golden.py
    (oracle only); a change of the oracle's arithmetic must regenerate it knowingly."""
    import json
    import os
    import sys
    sys.path.insert(0, os.path.join(os.path.dirname(__file__), "golden"))
    import make_golden
    with open(os.path.join(os.path.dirname(__file__), "golden", "tiny_oracle_digest.json")) as f:
        want = json.load(f)
    got = make_golden.compute()
    for k, v in want.items():
        if isinstance(v, float):
            assert got[k] == pytest.approx(v, rel=1e-12, abs=1e-300), k
        else:
            assert got[k] == v, k


def test_oracle_shares_nothing_with_cuda_path():
    import os
    import re
    here = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    for name in os.listdir(os.path.join(here, "oracle")):
        if name.endswith((".py", ".c", ".h")):
            src = open(os.path.join(here, "oracle", name)).read()
            assert not re.search(r"^\s*(from|import)\s+block_scaled_gemm_rfq_b200", src, re.M), name
            assert "#include \"rfq.h\"" not in src and "csrc" not in src, name


# --------------------------------------------------------------------------- MXFP8 comparator
F8 = ml_dtypes.float8_e4m3fn


def test_e4m3_decode_matches_ml_dtypes_and_torch(oracle):
    import torch
    codes = np.arange(256, dtype=np.uint8)
    mine = np.array([oracle.e4m3_value(int(c)) for c in codes])
    mld = codes.view(F8).astype(np.float64)
    tch = torch.from_numpy(codes.copy()).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    np.testing.assert_array_equal(np.isnan(mine), np.isnan(mld))
    ok = ~np.isnan(mine)
    np.testing.assert_array_equal(mine[ok], mld[ok])
    np.testing.assert_array_equal(mine[ok], tch[ok])
    assert mine[0x7E] == 448.0 and math.copysign(1.0, mine[0x80]) == -1.0


@pytest.mark.parametrize("e", [-127, -3, 0, 5, 117])
def test_e4m3_encode_exhaustive_vs_ml_dtypes(oracle, e):
    """Every finite bf16 x with |x| 2^-e < 512: the oracle's code equals ml_dtypes'
    round-to-nearest-even float8_e4m3fn cast of the exactly scaled value where that
    cast is finite (below 464); from 464 the oracle saturates to 448."""
    _, x = _all_finite_bf16()
    v = np.ldexp(x, -e)
    keep = np.abs(v) < 512.0
    x, v = x[keep], v[keep]
    got = np.array([oracle.e4m3_encode(float(xi), e) for xi in x], dtype=np.uint8)
    small = np.abs(v) < 464.0
    want = v[small].astype(np.float32).astype(F8).view(np.uint8)
    bad = np.nonzero(got[small] != want)[0]
    assert bad.size == 0, (x[small][bad[:5]], got[small][bad[:5]], want[bad[:5]])
    big = ~small
    np.testing.assert_array_equal(got[big] & 0x7F, np.full(big.sum(), 0x7E, np.uint8))
    np.testing.assert_array_equal(got[big] >> 7, (np.signbit(x[big])).astype(np.uint8))


def test_e4m3_block_exponent_brute_force(oracle):
    """The unique e in [-127, 127] with 256 <= amax 2^-e < 512 (E4M3's largest
    exponent is 8), by search; -127 below the range, 128 for non-finite."""
    rng = np.random.default_rng(21)
    amaxes = np.concatenate([np.ldexp(rng.uniform(1, 2, 400), rng.integers(-140, 127, 400)),
                             np.ldexp(1.0, np.arange(-130, 127)), [0.0, 448.0, 449.0, 511.9, 512.0]])
    for a in amaxes:
        want = -127
        if a > 0:
            for e in range(-127, 128):
                if 256.0 <= math.ldexp(float(a), -e) < 512.0:
                    want = e
                    break
        assert oracle.block_exponent_e4m3(float(a)) == want, a
    assert oracle.block_exponent_e4m3(math.inf) == 128


def test_mxfp8_qdq_identity_and_gemm_closed_form(oracle):
    """Blocks of E4M3 values times 2^t with amax >= 256 * 2^t are reproduced exactly;
    the MXFP8 GEMM of such operands is the plain float64 product."""
    rng = np.random.default_rng(23)
    vals = np.arange(0x7F, dtype=np.uint8).view(F8).astype(np.float64)     # all finite magnitudes
    def block_matrix(rows, K):
        m = rng.choice(vals, (rows, K)) * rng.choice([-1.0, 1.0], (rows, K))
        m = m.reshape(rows, K // 32, 32)
        m[:, :, 0] = rng.choice([256.0, 320.0, 448.0], (rows, K // 32))
        m *= np.exp2(rng.integers(-30, 30, (rows, K // 32, 1)))
        return m.reshape(rows, K)
    X = block_matrix(48, 128)
    W = block_matrix(40, 128)
    xb, wb = wl.f64_to_bf16_bits(X), wl.f64_to_bf16_bits(W)
    # every E4M3 value has <= 4 significant bits, so bf16 holds X and W exactly
    np.testing.assert_array_equal(wl.bf16_bits_to_f32(xb).astype(np.float64), X)
    q = oracle.quantize_mxfp8_bf16(xb)
    np.testing.assert_array_equal(oracle.dequantize_mxfp8(q["codes"], q["scales"]), X)
    Y, S, _ = oracle.mxfp8_linear(xb, wb)
    np.testing.assert_allclose(Y, X @ W.T, rtol=0, atol=1e-12 * S)
