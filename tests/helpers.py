"""Shared helpers of the GPU parity tests: move the seeded bf16 inputs to the
device, run the CUDA path through the C ABI binding, and compare with the oracle.

Tolerance (stated with the method's arithmetic): the GEMM sums 2K exact FP4 x FP4
products (each product of two E2M1 values times two powers of two is exact) in
fp32, so |Y_gpu - Y_ref| <= 1e-5 * S with S = max_{i,j} sum_k |a_ik b_jk| over the
concatenated K; a bf16 output adds one bf16 ulp of |Y_ref| (round to nearest
even of the fp32 result).  Codes and scales must match bit for bit.
"""
import numpy as np

from block_scaled_gemm_rfq_b200 import workloads as wl

REL_TOL = 1e-5


def dev_bf16(bits: np.ndarray):
    import torch
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16).copy()).view(torch.bfloat16).cuda()


def gpu_quantize(rfq, bits: np.ndarray, residual: bool = True, weight: bool = False):
    """Run the quantizer on the device; returns codes [M, K/2] and MMA-layout scale bytes."""
    import torch
    x = dev_bf16(bits)
    q = rfq.quantize_weight_alloc(x) if weight else rfq.quantize_mxfp4_alloc(x, residual=residual)
    torch.cuda.synchronize()
    M, K = bits.shape
    cb, sb = rfq.codes_bytes(M, K), rfq.scales_bytes(M, K)
    out = {
        "codes_x": q.codes.cpu().numpy()[:cb].reshape(M, K // 2),
        "scales_x": q.scales.cpu().numpy()[:sb],
    }
    if q.has_residual:
        out["codes_r"] = q.r_codes.cpu().numpy()[:cb].reshape(M, K // 2)
        out["scales_r"] = q.r_scales.cpu().numpy()[:sb]
    return out, q


def nonfinite_blocks(bits: np.ndarray) -> np.ndarray:
    """[M, K/32] mask of blocks holding a NaN or infinity (their codes are unspecified)."""
    exp = (bits >> 7) & 0xFF
    return (exp == 0xFF).reshape(bits.shape[0], -1, 32).any(-1)


def _mask_codes(codes: np.ndarray, mask: np.ndarray) -> np.ndarray:
    c = codes.copy()
    m = np.repeat(mask, 16, axis=1)   # 16 code bytes per 32-element block
    c[m] = 0
    return c


def assert_quant_parity(oracle, bits: np.ndarray, got: dict, residual: bool = True):
    ref = oracle.quantize_bf16(bits, residual=residual)
    mask = nonfinite_blocks(bits)
    keys = ["x", "r"] if residual else ["x"]
    for k in keys:
        want_c = _mask_codes(ref[f"codes_{k}"], mask)
        got_c = _mask_codes(got[f"codes_{k}"], mask)
        bad = np.argwhere(want_c != got_c)
        assert bad.size == 0, f"codes_{k}: {len(bad)} bytes differ, first at {bad[:4].tolist()}: " \
                              f"got {got_c[tuple(bad[0])]:#04x} want {want_c[tuple(bad[0])]:#04x}"
        want_s = oracle.scales_to_mma_layout(ref[f"scales_{k}"])
        bad = np.nonzero(want_s != got[f"scales_{k}"])[0]
        assert bad.size == 0, f"scales_{k}: {bad.size} bytes differ, first at {bad[:4].tolist()}"
    return ref


def bf16_ulp(v: np.ndarray) -> np.ndarray:
    a = np.abs(v)
    e = np.floor(np.log2(np.where(a > 0, a, 1.0)))
    return np.where(a > 0, np.exp2(np.maximum(e, -126) - 7), 2.0 ** -133)


def assert_y_close(y_gpu: np.ndarray, y_ref: np.ndarray, S: float, bf16_out: bool, what: str = "Y"):
    y_gpu = y_gpu.astype(np.float64)
    err = np.abs(y_gpu - y_ref)
    bound = REL_TOL * S + (bf16_ulp(y_ref) if bf16_out else 0.0)
    worst = np.unravel_index(np.argmax(err - bound), err.shape)
    assert np.all(err <= bound), (f"{what}: max excess at {worst}: gpu {y_gpu[worst]!r} ref {y_ref[worst]!r} "
                                  f"err {err[worst]:.3e} bound {np.broadcast_to(bound, err.shape)[worst]:.3e} "
                                  f"S {S:.3e}")
    return float(err.max() / S) if S > 0 else 0.0


def y_to_numpy(y):
    import torch
    return y.float().cpu().numpy() if y.dtype == torch.bfloat16 else y.cpu().numpy()


def bits_to_f64(bits):
    return wl.bf16_bits_to_f32(bits).astype(np.float64)
