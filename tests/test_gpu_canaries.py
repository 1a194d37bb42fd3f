"""Guard bands around every output: the out-of-bounds check of the CUDA path.

Each output buffer (Y, Y^T, codes, scales, workspaces) is carved out of a larger
allocation whose first and last 4 KiB hold a known byte pattern.  After every call
the pattern must be intact: a store past the end of an output (the Y epilogue's
last row and column stores, the transposed quantizer's tile stores, the
scale-padding fill, the split-K reduction stores) or before its start would change
it.  The
shapes are ragged in M and N (and K where the path allows) so that the stores near
the ends of the buffers are exercised.  Every call's result is also checked against
the oracle (Y within 1e-5 * S, codes and scales bit for bit), so a guard that stays
intact because nothing was written cannot pass either.
"""
import numpy as np
import pytest

from block_scaled_gemm_rfq_b200 import workloads as wl
from helpers import assert_quant_parity, assert_y_close, dev_bf16, y_to_numpy

pytestmark = pytest.mark.gpu

GUARD = 4096          # bytes on each side (keeps the output's 256-byte alignment)
PATTERN = 0xA5


class Guarded:
    """An output buffer of `nbytes` with guard bands before and after it."""

    def __init__(self, nbytes, dtype=None, shape=None):
        import torch
        self.n = int(nbytes)
        self.whole = torch.full((self.n + 2 * GUARD,), PATTERN, dtype=torch.uint8, device="cuda")
        self.bytes = self.whole[GUARD:GUARD + self.n]
        self.t = self.bytes if dtype is None else self.bytes.view(dtype).view(*shape)

    def check(self, what):
        import torch
        torch.cuda.synchronize()
        head = self.whole[:GUARD].cpu().numpy()
        tail = self.whole[GUARD + self.n:].cpu().numpy()
        for name, band in (("before", head), ("after", tail)):
            bad = np.nonzero(band != PATTERN)[0]
            assert bad.size == 0, f"{what}: {bad.size} guard bytes {name} the buffer changed, first at offset " \
                                  f"{int(bad[0]) - (GUARD if name == 'before' else 0)}"


def _y(M, N, dtype):
    import torch
    size = 2 if dtype == torch.bfloat16 else 4
    return Guarded(M * N * size, dtype, (M, N))


def _quant_outputs(rfq, rows, K, residual):
    c = [Guarded(rfq.codes_bytes(rows, K)), Guarded(rfq.scales_bytes(rows, K))]
    r = [Guarded(rfq.codes_bytes(rows, K)), Guarded(rfq.scales_bytes(rows, K))] if residual else [None, None]
    return c + r


def _gather(rfq, bufs, rows, K):
    out = {"codes_x": bufs[0].bytes.cpu().numpy().reshape(rows, K // 2), "scales_x": bufs[1].bytes.cpu().numpy()}
    if bufs[2] is not None:
        out["codes_r"] = bufs[2].bytes.cpu().numpy().reshape(rows, K // 2)
        out["scales_r"] = bufs[3].bytes.cpu().numpy()
    return out


@pytest.mark.parametrize("M,K,residual", [(300, 96, True), (129, 4128, True), (77, 224, False), (1, 32, True)])
def test_quantizer_guards(rfq, oracle, M, K, residual):
    """Forward quantizer: codes, and the scale array whose padding rows/blocks the
    kernel fills with zeros (the last atom ends exactly at the buffer end)."""
    x_bits = wl.random_matrix(M, K, seed=M * 7 + K, scale=3.0)
    bufs = _quant_outputs(rfq, M, K, residual)
    rfq.quantize_mxfp4(dev_bf16(x_bits), *(b.t if b is not None else None for b in bufs))
    for i, b in enumerate(bufs):
        if b is not None:
            b.check(f"quantize {M}x{K} output {i}")
    assert_quant_parity(oracle, x_bits, _gather(rfq, bufs, M, K), residual=residual)


def test_weight_quantizer_guards(rfq, oracle):
    N, K = 136, 1056
    w_bits = wl.random_matrix(N, K, seed=5, scale=0.05)
    c, s = Guarded(rfq.codes_bytes(N, K)), Guarded(rfq.scales_bytes(N, K))
    rfq.quantize_weight(dev_bf16(w_bits), c.t, s.t)
    c.check("weight codes")
    s.check("weight scales")
    assert_quant_parity(oracle, w_bits, {"codes_x": c.bytes.cpu().numpy().reshape(N, K // 2),
                                         "scales_x": s.bytes.cpu().numpy()}, residual=False)


# (M, N, K): (100, 19200, 256) single-CTA tiled kernel with many tiles; (300, 520, 1024)
# CTA pairs with ragged M and N (the epilogue's guarded row and column stores);
# (40, 384, 2304), (96, 520, 2304) and (200, 264, 2304) the short-batch split-K
# kernel at 64 rows, 128 rows and two 128-row blocks (ragged reduction slices and a
# ragged second block); (1000, 72, 256) a single ragged column tile.
@pytest.mark.parametrize("M,N,K", [(100, 19200, 256), (300, 520, 1024), (40, 384, 2304), (96, 520, 2304),
                                   (200, 264, 2304), (1000, 72, 256)])
@pytest.mark.parametrize("residual", [True, False])
def test_gemm_guards(rfq, oracle, M, N, K, residual):
    import torch
    x_bits = wl.random_matrix(M, K, seed=M + N, scale=2.0)
    w_bits = wl.random_matrix(N, K, seed=N + K, scale=0.05)
    qa = rfq.quantize_mxfp4_alloc(dev_bf16(x_bits), residual=residual)
    qw = rfq.quantize_weight_alloc(dev_bf16(w_bits))
    Y, S, _ = oracle.rfq_linear(x_bits, w_bits, residual=residual)
    for dt in (torch.float32, torch.bfloat16):
        y = _y(M, N, dt)
        rfq.gemm(qa.codes, qa.scales, qa.r_codes if residual else None, qa.r_scales if residual else None,
                 qw.codes, qw.scales, M, N, K, y.t)
        y.check(f"Y {M}x{N}x{K} {dt} residual={residual}")
        assert_y_close(y_to_numpy(y.t), Y, S, bf16_out=(dt == torch.bfloat16), what=f"Y {M}x{N}x{K} {dt}")
    rfq.check_device_error()


@pytest.mark.parametrize("M,N,K", [(300, 136, 512), (96, 264, 256)])
def test_gemm_transposed_output_guards(rfq, oracle, M, N, K):
    """The Y^T epilogue (weight gradient): per-column stores of 32 neighbouring rows."""
    import torch
    x_bits = wl.random_matrix(M, K, seed=3 * M, scale=2.0)
    w_bits = wl.random_matrix(N, K, seed=3 * N, scale=0.05)
    qa = rfq.quantize_mxfp4_alloc(dev_bf16(x_bits))
    qw = rfq.quantize_weight_alloc(dev_bf16(w_bits))
    Y, S, _ = oracle.rfq_linear(x_bits, w_bits, residual=True)
    for dt in (torch.float32, torch.bfloat16):
        yt = _y(N, M, dt)
        rfq.gemm_yt(qa.codes, qa.scales, qa.r_codes, qa.r_scales, qw.codes, qw.scales, M, N, K, yt.t)
        yt.check(f"Y^T {M}x{N}x{K} {dt}")
        assert_y_close(y_to_numpy(yt.t).T, Y, S, bf16_out=(dt == torch.bfloat16), what=f"Y^T {M}x{N}x{K}")


@pytest.mark.parametrize("M,N,K,split", [(24, 264, 1024, 0), (64, 136, 2304, 3), (1, 8, 64, 0)])
def test_single_kernel_layer_guards(rfq, oracle, M, N, K, split):
    """rfq_linear_fused: quantizer inside the GEMM, split-K reduction through the
    cluster's shared memory, Y stored by the reducing CTAs."""
    import torch
    x_bits = wl.random_matrix(M, K, seed=M + 11, scale=2.0)
    w_bits = wl.random_matrix(N, K, seed=N + 13, scale=0.05)
    qw = rfq.quantize_weight_alloc(dev_bf16(w_bits))
    Y, S, _ = oracle.rfq_linear(x_bits, w_bits, residual=True)
    rfq.debug_fused_split(split)
    try:
        for dt in (torch.float32, torch.bfloat16):
            y = _y(M, N, dt)
            rfq.linear_fused(dev_bf16(x_bits), qw.codes, qw.scales, N, y.t)
            y.check(f"fused Y {M}x{N}x{K} {dt}")
            assert_y_close(y_to_numpy(y.t), Y, S, bf16_out=(dt == torch.bfloat16), what=f"fused {M}x{N}x{K}")
    finally:
        rfq.debug_fused_split(0)


@pytest.mark.parametrize("M,N,K", [(200, 136, 1024), (16, 72, 512)])
def test_linear_workspace_guards(rfq, oracle, M, N, K):
    """rfq_linear writes only inside its workspace (and Y)."""
    import torch
    x_bits = wl.random_matrix(M, K, seed=M + 21, scale=2.0)
    w_bits = wl.random_matrix(N, K, seed=N + 23, scale=0.05)
    qw = rfq.quantize_weight_alloc(dev_bf16(w_bits))
    ws = Guarded(rfq.linear_workspace_bytes(M, K, True))
    y = _y(M, N, torch.float32)
    rfq.linear(dev_bf16(x_bits), qw.codes, qw.scales, N, y.t, ws.t, True)
    ws.check(f"workspace {M}x{K}")
    y.check(f"linear Y {M}x{N}")
    Y, S, _ = oracle.rfq_linear(x_bits, w_bits, residual=True)
    assert_y_close(y_to_numpy(y.t), Y, S, bf16_out=False, what=f"linear {M}x{N}x{K}")


@pytest.mark.parametrize("R,C,residual", [(320, 136, True), (96, 8, False), (1056, 264, True)])
def test_transposed_quantizer_guards(rfq, oracle, R, C, residual):
    """The operand of X^T: 64-row x 8-block shared-memory tiles stored by TMA, the
    last tile clipped at the ragged end of X's columns."""
    x_bits = wl.random_matrix(R, C, seed=R + C, scale=2.0)
    bufs = _quant_outputs(rfq, C, R, residual)
    rfq.quantize_mxfp4_t(dev_bf16(x_bits), *(b.t if b is not None else None for b in bufs))
    for i, b in enumerate(bufs):
        if b is not None:
            b.check(f"quantize_t {R}x{C} output {i}")
    got = _gather(rfq, bufs, C, R)
    assert_quant_parity(oracle, np.ascontiguousarray(x_bits.T), got, residual=residual)


def test_mxfp8_guards(rfq, oracle):
    import torch
    M, N, K = 300, 136, 512
    x_bits = wl.random_matrix(M, K, seed=31, scale=2.0)
    w_bits = wl.random_matrix(N, K, seed=32, scale=0.05)
    qc, qs = Guarded(rfq.mxfp8_codes_bytes(M, K)), Guarded(rfq.scales_bytes(M, K))
    rfq.quantize_mxfp8(dev_bf16(x_bits), qc.t, qs.t)
    qc.check("mxfp8 codes")
    qs.check("mxfp8 scales")
    ref = oracle.quantize_mxfp8_bf16(x_bits)
    assert np.array_equal(qc.bytes.cpu().numpy().reshape(M, K), ref["codes"])
    assert np.array_equal(qs.bytes.cpu().numpy(), oracle.scales_to_mma_layout(ref["scales"]))
    qw = rfq.quantize_mxfp8_alloc(dev_bf16(w_bits))
    Y, S, _ = oracle.mxfp8_linear(x_bits, w_bits)
    y = _y(M, N, torch.float32)
    rfq.gemm_mxfp8(qc.t, qs.t, qw.codes, qw.scales, M, N, K, y.t)
    y.check("mxfp8 Y")
    assert_y_close(y_to_numpy(y.t), Y, S, bf16_out=False, what="mxfp8 Y")
