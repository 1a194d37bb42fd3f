"""CPU oracle for RFQ (Residual Fallback Quantization) with MXFP4 blocks.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
benchmark's ``cpu_baseline`` / ``--impl reference`` legs may import this package.
It shares no code with the CUDA path (``block_scaled_gemm_rfq_b200``) and imports
nothing from it.

What it computes, and where it comes from:

* "Activation Outliers Matter: Robust Recovery for Quantized Multimodal LLMs"
  (arXiv 2608.26581), abstract and section 1, RFQ contribution paragraph: the
  activation X is quantized to FP4, the *full* quantization error
  R = X - DQ(Q(X)) is requantized by a second low-bit path, and the GEMM
  accumulates both contributions: Y = (DQ(Q(X)) + DQ(Q(R))) . DQ(Q(W))^T.
  Weights get a plain MXFP4 quantization (section 1: weight quantization is the
  secondary error source; the residual path is for activations).
* The pages stop at section 3.1 before defining MXFP4; the format follows the OCP
  MX v1.0 MXFP4 rule (32-element blocks along K, E8M0 scale exponent
  floor(log2 amax) - 2, E2M1 round-half-even with saturation to +-6, byte 0
  for an all-zero block).  See ``rfq_oracle.c`` for the per-element steps.

The element/scale arithmetic is plain C (``rfq_oracle.c``, built with gcc on
first use).  The reference GEMM is the textbook float64 product, by plain C loops
(``gemm_loops``) or, for large shapes, numpy's float64 matmul (``gemm_blas``),
the one library primitive used; the two are cross-checked by the pin tests.

Parity status: every function here is pinned by ``tests/test_oracle_pins.py``
(third-party FP4/E8M0 codecs, brute force, closed forms, invariants).  The pages
themselves print no worked example, so no pin comes from them.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "rfq_oracle.c")
_LIB_PATH = os.path.join(_HERE, "librfq_oracle.so")
_lock = threading.Lock()
_lib = None

BLOCK = 32


def build(force: bool = False) -> str:
    """Compile rfq_oracle.c into librfq_oracle.so (gcc, strict IEEE: no fast-math;
    OpenMP spreads independent rows over the host cores and changes no result)."""
    stale = (not os.path.exists(_LIB_PATH)) or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC)
    if force or stale:
        tmp = _LIB_PATH + f".tmp{os.getpid()}"
        cmd = ["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-fno-fast-math",
               "-ffp-contract=off", "-fopenmp", "-Wall", "-Wextra", "-o", tmp, _SRC, "-lm"]
        subprocess.run(cmd, check=True)
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _load():
    global _lib
    with _lock:
        if _lib is None:
            build()
            lib = ctypes.CDLL(_LIB_PATH)
            P = ctypes.c_void_p
            I64 = ctypes.c_int64
            lib.oracle_e2m1_value.restype = ctypes.c_double
            lib.oracle_e2m1_value.argtypes = [ctypes.c_uint8]
            lib.oracle_e2m1_encode.restype = ctypes.c_uint8
            lib.oracle_e2m1_encode.argtypes = [ctypes.c_double, ctypes.c_int]
            lib.oracle_block_exponent.restype = ctypes.c_int
            lib.oracle_block_exponent.argtypes = [ctypes.c_double]
            lib.oracle_bf16_value.restype = ctypes.c_double
            lib.oracle_bf16_value.argtypes = [ctypes.c_uint16]
            lib.oracle_quantize_bf16.restype = None
            lib.oracle_quantize_bf16.argtypes = [P, I64, I64, P, P, P, P]
            lib.oracle_quantize_f64.restype = None
            lib.oracle_quantize_f64.argtypes = [P, I64, I64, P, P]
            lib.oracle_dequantize.restype = None
            lib.oracle_dequantize.argtypes = [P, P, I64, I64, P]
            lib.oracle_gemm_nt.restype = None
            lib.oracle_gemm_nt.argtypes = [P, P, I64, I64, I64, P, P]
            lib.oracle_mma_scale_offset.restype = I64
            lib.oracle_mma_scale_offset.argtypes = [I64, I64, I64]
            lib.oracle_scales_to_mma_layout.restype = None
            lib.oracle_scales_to_mma_layout.argtypes = [P, I64, I64, P]
            lib.oracle_e4m3_value.restype = ctypes.c_double
            lib.oracle_e4m3_value.argtypes = [ctypes.c_uint8]
            lib.oracle_e4m3_encode.restype = ctypes.c_uint8
            lib.oracle_e4m3_encode.argtypes = [ctypes.c_double, ctypes.c_int]
            lib.oracle_block_exponent_e4m3.restype = ctypes.c_int
            lib.oracle_block_exponent_e4m3.argtypes = [ctypes.c_double]
            lib.oracle_quantize_mxfp8_bf16.restype = None
            lib.oracle_quantize_mxfp8_bf16.argtypes = [P, I64, I64, P, P]
            lib.oracle_dequantize_mxfp8.restype = None
            lib.oracle_dequantize_mxfp8.argtypes = [P, P, I64, I64, P]
            lib.oracle_threads.restype = ctypes.c_int
            lib.oracle_threads.argtypes = []
            _lib = lib
    return _lib


def _ptr(a: np.ndarray):
    assert a.flags["C_CONTIGUOUS"]
    return a.ctypes.data_as(ctypes.c_void_p)


# --------------------------------------------------------------------------- scalar pieces
def e2m1_value(code: int) -> float:
    """Value of one 4-bit E2M1 code (sign bit 3, exponent bits 2..1, mantissa bit 0)."""
    return _load().oracle_e2m1_value(int(code) & 0xF)


def e2m1_encode(x: float, e: int) -> int:
    """E2M1 code of x under block exponent e (RNE on |x|*2^-e, saturate to 6, keep sign)."""
    return int(_load().oracle_e2m1_encode(float(x), int(e)))


def block_exponent(amax: float) -> int:
    """floor(log2 amax) - 2 clamped to [-127, 127]; -127 for 0; 128 means non-finite (0xFF)."""
    return int(_load().oracle_block_exponent(float(amax)))


def threads() -> int:
    """Host threads the C row loops run on (OpenMP; OMP_NUM_THREADS caps it)."""
    return int(_load().oracle_threads())


def bf16_value(bits: int) -> float:
    return _load().oracle_bf16_value(int(bits) & 0xFFFF)


# --------------------------------------------------------------------------- matrices
def quantize_bf16(x_bits: np.ndarray, residual: bool = True):
    """MXFP4 quantization of a [rows, K] bf16 matrix given as uint16 bit patterns.

    Returns a dict with plain-layout ``codes_x`` [rows, K/2] uint8 (element 2j in
    the low nibble), ``scales_x`` [rows, K/32] uint8 (E8M0), and, when ``residual``,
    ``codes_r`` / ``scales_r`` for Q(R), R = X - DQ(Q(X)).
    """
    x_bits = np.ascontiguousarray(x_bits, dtype=np.uint16)
    rows, K = x_bits.shape
    if K % BLOCK:
        raise ValueError("K must be a multiple of 32")
    out = {
        "codes_x": np.zeros((rows, K // 2), np.uint8),
        "scales_x": np.zeros((rows, K // BLOCK), np.uint8),
    }
    if residual:
        out["codes_r"] = np.zeros((rows, K // 2), np.uint8)
        out["scales_r"] = np.zeros((rows, K // BLOCK), np.uint8)
    _load().oracle_quantize_bf16(
        _ptr(x_bits), rows, K, _ptr(out["codes_x"]), _ptr(out["scales_x"]),
        _ptr(out["codes_r"]) if residual else None, _ptr(out["scales_r"]) if residual else None)
    return out


def quantize_f64(x: np.ndarray):
    """MXFP4 quantization (same rule) of a float64 [rows, K] matrix -> (codes, scales)."""
    x = np.ascontiguousarray(x, dtype=np.float64)
    rows, K = x.shape
    codes = np.zeros((rows, K // 2), np.uint8)
    scales = np.zeros((rows, K // BLOCK), np.uint8)
    _load().oracle_quantize_f64(_ptr(x), rows, K, _ptr(codes), _ptr(scales))
    return codes, scales


def dequantize(codes: np.ndarray, scales: np.ndarray) -> np.ndarray:
    """DQ: float64 [rows, K] with value(code) * 2^(scale-127)."""
    codes = np.ascontiguousarray(codes, dtype=np.uint8)
    scales = np.ascontiguousarray(scales, dtype=np.uint8)
    rows, half = codes.shape
    K = 2 * half
    out = np.empty((rows, K), np.float64)
    _load().oracle_dequantize(_ptr(codes), _ptr(scales), rows, K, _ptr(out))
    return out


def gemm_loops(A: np.ndarray, B: np.ndarray):
    """Textbook Y = A . B^T in float64 by plain loops; also sum_k |A||B| per output."""
    A = np.ascontiguousarray(A, dtype=np.float64)
    B = np.ascontiguousarray(B, dtype=np.float64)
    M, K = A.shape
    N = B.shape[0]
    Y = np.empty((M, N), np.float64)
    absY = np.empty((M, N), np.float64)
    _load().oracle_gemm_nt(_ptr(A), _ptr(B), M, N, K, _ptr(Y), _ptr(absY))
    return Y, absY


def gemm_blas(A: np.ndarray, B: np.ndarray):
    """The same product by numpy's float64 matmul (for shapes the loops cannot finish)."""
    return A @ B.T, np.abs(A) @ np.abs(B).T


def mma_scale_offset(r: int, c: int, Kb: int) -> int:
    return int(_load().oracle_mma_scale_offset(r, c, Kb))


def scales_to_mma_layout(plain: np.ndarray) -> np.ndarray:
    """Plain [rows, Kb] E8M0 bytes -> the block-scaled MMA's 128x4-atom byte layout (1-D)."""
    plain = np.ascontiguousarray(plain, dtype=np.uint8)
    rows, Kb = plain.shape
    rows_pad = (rows + 127) // 128 * 128
    kb_pad = (Kb + 3) // 4 * 4
    out = np.zeros(rows_pad * kb_pad, np.uint8)
    _load().oracle_scales_to_mma_layout(_ptr(plain), rows, Kb, _ptr(out))
    return out


# --------------------------------------------------------------------------- the RFQ linear
def rfq_operands(q_act: dict, q_w: dict, residual: bool = True):
    """Concatenated operands of the RFQ GEMM in float64 (exact):
    A_cat = [DQ(QX) | DQ(QR)]  (M x 2K),  B_cat = [DQ(QW) | DQ(QW)]  (N x 2K).
    With ``residual=False`` they are DQ(QX) and DQ(QW) (plain MXFP4 GEMM)."""
    ax = dequantize(q_act["codes_x"], q_act["scales_x"])
    bw = dequantize(q_w["codes_x"], q_w["scales_x"])
    if not residual:
        return ax, bw
    ar = dequantize(q_act["codes_r"], q_act["scales_r"])
    return np.concatenate([ax, ar], axis=1), np.concatenate([bw, bw], axis=1)


def rfq_linear(x_bits: np.ndarray, w_bits: np.ndarray, residual: bool = True, use_loops=None):
    """Reference RFQ linear layer.

    Returns (Y_ref float64 [M, N], S, absY) where S = max_{i,j} sum_k |A_cat[i,k]| |B_cat[j,k]|
    is the scalar the tolerance 1e-5 * S is stated against.
    """
    qa = quantize_bf16(x_bits, residual=residual)
    qw = quantize_bf16(w_bits, residual=False)
    A, B = rfq_operands(qa, qw, residual)
    if use_loops is None:
        use_loops = A.shape[0] * B.shape[0] * A.shape[1] <= 64 * 1024 * 1024
    Y, absY = gemm_loops(A, B) if use_loops else gemm_blas(A, B)
    return Y, float(absY.max()) if absY.size else 0.0, absY


# ----------------------------------------------------------------------------- backward GEMMs
# The paper frames RFQ as a differentiable method meant for FP4 *training* (section 1,
# the RFQ paragraph) but states no backward rule.  The
# plainest reading is the straight-through estimator: the quantizers pass the
# gradient unchanged, and the two backward GEMMs of Y = X W^T are themselves run on
# MXFP4 operands quantized along *their* contraction axis, with the residual
# pathway on the activation-side operand as in the forward.


def quantize_transposed(x_bits: np.ndarray, residual: bool = True):
    """MXFP4 quantization of X^T for a [R, C] bf16 matrix: blocks of 32 run down the
    rows of X (the definition: transpose, then the row rule of ``quantize_bf16``)."""
    return quantize_bf16(np.ascontiguousarray(np.asarray(x_bits, dtype=np.uint16).T), residual=residual)


def rfq_dgrad(dy_bits: np.ndarray, w_bits: np.ndarray, residual: bool = True, use_loops=None):
    """dX [M, K] = (DQ(Q(dY)) + DQ(Q(R_dY))) . DQ(Q(W^T))^T: the contraction runs over N,
    so dY [M, N] is quantized along its rows and W [N, K] along its columns.
    Returns (dX, S, absY) as ``rfq_linear``."""
    wt = np.ascontiguousarray(np.asarray(w_bits, dtype=np.uint16).T)
    return rfq_linear(dy_bits, wt, residual=residual, use_loops=use_loops)


def rfq_wgrad(x_bits: np.ndarray, dy_bits: np.ndarray, residual: bool = True, use_loops=None):
    """dW [N, K] = sum over the M tokens of dY[m, n] (X^[m, k]), both operands quantized
    along M; X carries the residual pathway.  Computed as the RFQ product of X^T [K, M]
    (activation, with residual) and dY^T [N, M], transposed.  Returns (dW, S, absY^T)."""
    xt = np.ascontiguousarray(np.asarray(x_bits, dtype=np.uint16).T)
    dyt = np.ascontiguousarray(np.asarray(dy_bits, dtype=np.uint16).T)
    Y, S, absY = rfq_linear(xt, dyt, residual=residual, use_loops=use_loops)
    return np.ascontiguousarray(Y.T), S, np.ascontiguousarray(absY.T)


# ----------------------------------------------------------------------------- MXFP8 comparator
# The paper finds MXFP8 nearly free of accuracy loss (abstract; section 1, first contribution)
# and gives it as the reference point for the 4-bit formats.  OCP MX v1.0 MXFP8 with
# E4M3 elements: 32-element blocks, E8M0 exponent floor(log2 amax) - 8, elements
# rounded to nearest-even and saturated to +-448 (rfq_oracle.c).


def e4m3_value(code: int) -> float:
    """Value of one 8-bit E4M3 code (NaN for 0x7F / 0xFF)."""
    return _load().oracle_e4m3_value(code)


def e4m3_encode(x: float, e: int) -> int:
    """E4M3 code of x under block exponent e (RNE on |x|*2^-e, saturate to 448, keep sign)."""
    return _load().oracle_e4m3_encode(x, e)


def block_exponent_e4m3(amax: float) -> int:
    """floor(log2 amax) - 8 clamped to [-127, 127]; -127 for 0; 128 means non-finite."""
    return _load().oracle_block_exponent_e4m3(amax)


def quantize_mxfp8_bf16(x_bits: np.ndarray):
    """MXFP8 quantization of a [rows, K] bf16 matrix (uint16 bit patterns): ``codes``
    [rows, K] uint8 (one E4M3 code per element) and ``scales`` [rows, K/32] E8M0."""
    x_bits = np.ascontiguousarray(x_bits, dtype=np.uint16)
    rows, K = x_bits.shape
    if K % BLOCK:
        raise ValueError("K must be a multiple of 32")
    out = {"codes": np.zeros((rows, K), np.uint8), "scales": np.zeros((rows, K // BLOCK), np.uint8)}
    _load().oracle_quantize_mxfp8_bf16(_ptr(x_bits), rows, K, _ptr(out["codes"]), _ptr(out["scales"]))
    return out


def dequantize_mxfp8(codes: np.ndarray, scales: np.ndarray) -> np.ndarray:
    codes = np.ascontiguousarray(codes, dtype=np.uint8)
    scales = np.ascontiguousarray(scales, dtype=np.uint8)
    rows, K = codes.shape
    out = np.empty((rows, K), np.float64)
    _load().oracle_dequantize_mxfp8(_ptr(codes), _ptr(scales), rows, K, _ptr(out))
    return out


def mxfp8_linear(x_bits: np.ndarray, w_bits: np.ndarray, use_loops=None):
    """Reference MXFP8 (W8A8) linear layer: Y = DQ(Q8(X)) . DQ(Q8(W))^T in float64.
    Returns (Y, S, absY) with S = max_{i,j} sum_k |a_ik| |b_jk| as ``rfq_linear``."""
    qa = quantize_mxfp8_bf16(x_bits)
    qw = quantize_mxfp8_bf16(w_bits)
    A = dequantize_mxfp8(qa["codes"], qa["scales"])
    B = dequantize_mxfp8(qw["codes"], qw["scales"])
    if use_loops is None:
        use_loops = A.shape[0] * B.shape[0] * A.shape[1] <= 64 * 1024 * 1024
    Y, absY = gemm_loops(A, B) if use_loops else gemm_blas(A, B)
    return Y, float(absY.max()) if absY.size else 0.0, absY
