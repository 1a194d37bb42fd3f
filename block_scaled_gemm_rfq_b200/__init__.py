"""B200 (sm_100a) Residual Fallback Quantization: MXFP4 W4A4 linear layers.

Python binding of the C ABI in include/rfq.h (``librfq.so``, built in-tree by
``block_scaled_gemm_rfq_b200.build``).  This module only marshals arguments:
every step of the path (quantization, residual, requantization, GEMM) runs in the
library's CUDA kernels.  PyTorch is used for device memory and streams.  There is
no CPU fallback: if the library is missing, every call raises.

Method: "Activation Outliers Matter: Robust Recovery for Quantized Multimodal
LLMs" (arXiv 2608.26581), section 1 (RFQ): Y = (DQ(QX) + DQ(QR)) DQ(QW)^T with
R = X - DQ(QX) requantized by the same MXFP4 rule.
"""
from __future__ import annotations

import ctypes
import os
import threading

__all__ = [
    "RFQError", "load_library", "library_path", "codes_bytes", "scales_bytes", "linear_workspace_bytes",
    "quantize_mxfp4", "quantize_weight", "gemm", "linear", "linear_static_workspace", "check_device_error",
    "debug_skip_next_fill", "STATIC_WORKSPACE_BYTES", "linear_fused", "linear_fused_alloc", "debug_fused_split",
    "FUSED_MAX_M", "quantize_mxfp4_t", "gemm_yt", "linear_dgrad", "linear_wgrad", "linear_wgrad_workspace_bytes",
    "quantize_mxfp4_t_alloc", "linear_wgrad_alloc", "linear_dgrad_alloc",
    "mxfp8_codes_bytes", "quantize_mxfp8", "gemm_mxfp8", "quantize_mxfp8_alloc", "gemm_mxfp8_alloc",
    "QuantizedTensor", "quantize_mxfp4_alloc", "quantize_weight_alloc", "gemm_alloc", "linear_alloc",
    "EXPORTED_SYMBOLS", "OUT_F32", "OUT_BF16", "mma_rate_probe", "MMA_PROBE_MAX_ITERATIONS",
]

_HERE = os.path.dirname(os.path.abspath(__file__))
_LIB_PATH = os.path.join(_HERE, "librfq.so")
_lock = threading.Lock()
_lib = None

OUT_F32 = 0
OUT_BF16 = 1

STATUS = {0: "RFQ_OK", 1: "RFQ_ERR_INVALID_ARG", 2: "RFQ_ERR_UNSUPPORTED_SHAPE", 3: "RFQ_ERR_MISALIGNED",
          4: "RFQ_ERR_UNSUPPORTED_DEVICE", 5: "RFQ_ERR_CUDA", 6: "RFQ_ERR_TIMEOUT", 7: "RFQ_ERR_WORKSPACE"}

# Every function include/rfq.h declares (checked against the built library by the CPU tests).
EXPORTED_SYMBOLS = (
    "rfq_status_string", "rfq_codes_bytes", "rfq_scales_bytes", "rfq_quantize_mxfp4", "rfq_quantize_weight",
    "rfq_gemm", "rfq_linear_workspace_bytes", "rfq_linear", "rfq_check_device_error", "rfq_debug_skip_next_fill",
    "rfq_linear_static_workspace", "rfq_linear_fused", "rfq_debug_fused_split", "rfq_quantize_mxfp4_t",
    "rfq_gemm_yt", "rfq_linear_dgrad", "rfq_linear_wgrad_workspace_bytes", "rfq_linear_wgrad",
    "rfq_mxfp8_codes_bytes", "rfq_quantize_mxfp8", "rfq_gemm_mxfp8", "rfq_mma_rate_probe",
)

# Largest iteration count of the tensor-core rate probe (RFQ_MMA_PROBE_MAX_ITERATIONS).
MMA_PROBE_MAX_ITERATIONS = 100000

# Size of the library's fixed scratch array (RFQ_STATIC_WORKSPACE_BYTES in include/rfq.h).
STATIC_WORKSPACE_BYTES = 32 << 20

# Largest M of the single-kernel linear layer (RFQ_FUSED_MAX_M in include/rfq.h).
FUSED_MAX_M = 64


class RFQError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {STATUS.get(status, status)}")


def library_path() -> str:
    """Path of the in-tree librfq.so this binding loads."""
    return _LIB_PATH


def load_library():
    """Load librfq.so (raises if it has not been built)."""
    global _lib
    with _lock:
        if _lib is None:
            if not os.path.exists(_LIB_PATH):
                raise RuntimeError(f"CUDA library {_LIB_PATH} is missing; build it with "
                                   "`python -m block_scaled_gemm_rfq_b200.build`")
            lib = ctypes.CDLL(_LIB_PATH)
            P, I64, SZ, I = ctypes.c_void_p, ctypes.c_int64, ctypes.c_size_t, ctypes.c_int
            sig = {
                "rfq_status_string": (ctypes.c_char_p, [I]),
                "rfq_codes_bytes": (SZ, [I64, I64]),
                "rfq_scales_bytes": (SZ, [I64, I64]),
                "rfq_quantize_mxfp4": (I, [P, I64, I64, P, P, P, P, P]),
                "rfq_quantize_weight": (I, [P, I64, I64, P, P, P]),
                "rfq_gemm": (I, [P, P, P, P, P, P, I64, I64, I64, P, I, P]),
                "rfq_linear_workspace_bytes": (SZ, [I64, I64, I]),
                "rfq_linear": (I, [P, I64, I64, P, P, I64, P, I, I, P, SZ, P]),
                "rfq_check_device_error": (I, [P, ctypes.POINTER(ctypes.c_int)]),
                "rfq_debug_skip_next_fill": (I, [I]),
                "rfq_linear_static_workspace": (I, [P, I64, I64, P, P, I64, P, I, I, P]),
                "rfq_linear_fused": (I, [P, I64, I64, P, P, I64, P, I, I, P]),
                "rfq_debug_fused_split": (I, [I]),
                "rfq_quantize_mxfp4_t": (I, [P, I64, I64, P, P, P, P, P]),
                "rfq_gemm_yt": (I, [P, P, P, P, P, P, I64, I64, I64, P, I, P]),
                "rfq_linear_dgrad": (I, [P, I64, I64, P, P, I64, P, I, I, P, SZ, P]),
                "rfq_linear_wgrad_workspace_bytes": (SZ, [I64, I64, I64, I]),
                "rfq_linear_wgrad": (I, [P, P, I64, I64, I64, P, I, I, P, SZ, P]),
                "rfq_mxfp8_codes_bytes": (SZ, [I64, I64]),
                "rfq_quantize_mxfp8": (I, [P, I64, I64, P, P, P]),
                "rfq_gemm_mxfp8": (I, [P, P, P, P, I64, I64, I64, P, I, P]),
                "rfq_mma_rate_probe": (I, [I, I64, P, I64, ctypes.POINTER(ctypes.c_double),
                                           ctypes.POINTER(ctypes.c_int), P]),
            }
            for name, (res, args) in sig.items():
                fn = getattr(lib, name)
                fn.restype = res
                fn.argtypes = args
            _lib = lib
    return _lib


def _check(status: int, where: str):
    if status != 0:
        raise RFQError(status, where)


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    import torch
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream))


# ----------------------------------------------------------------------------- sizes
def codes_bytes(rows: int, K: int) -> int:
    """rfq_codes_bytes: bytes of packed E2M1 codes for [rows, K] (rows * K / 2)."""
    return int(load_library().rfq_codes_bytes(rows, K))


def scales_bytes(rows: int, K: int) -> int:
    """rfq_scales_bytes: bytes of E8M0 scales for [rows, K] in the MMA layout (padded to 128 rows x 4 blocks)."""
    return int(load_library().rfq_scales_bytes(rows, K))


def linear_workspace_bytes(M: int, K: int, use_residual: bool = True) -> int:
    """rfq_linear_workspace_bytes: workspace rfq_linear needs for an [M, K] activation."""
    return int(load_library().rfq_linear_workspace_bytes(M, K, int(bool(use_residual))))


# ----------------------------------------------------------------------------- raw calls (caller-owned buffers)
def quantize_mxfp4(x, qx_codes, qx_scales, qr_codes=None, qr_scales=None, stream=None):
    """rfq_quantize_mxfp4 on torch tensors: x [M, K] bf16 (CUDA), outputs uint8 buffers."""
    M, K = x.shape
    _check(load_library().rfq_quantize_mxfp4(_ptr(x), M, K, _ptr(qx_codes), _ptr(qx_scales), _ptr(qr_codes),
                                             _ptr(qr_scales), _stream(stream)), "rfq_quantize_mxfp4")


def quantize_weight(w, qw_codes, qw_scales, stream=None):
    """rfq_quantize_weight on torch tensors: w [N, K] bf16 (CUDA) -> Q(W) codes and scales (no residual)."""
    N, K = w.shape
    _check(load_library().rfq_quantize_weight(_ptr(w), N, K, _ptr(qw_codes), _ptr(qw_scales), _stream(stream)),
           "rfq_quantize_weight")


def gemm(qx_codes, qx_scales, qr_codes, qr_scales, qw_codes, qw_scales, M, N, K, y, stream=None):
    """rfq_gemm; y's dtype (float32 or bfloat16) selects the output type."""
    import torch
    y_type = OUT_BF16 if y.dtype == torch.bfloat16 else OUT_F32
    _check(load_library().rfq_gemm(_ptr(qx_codes), _ptr(qx_scales), _ptr(qr_codes), _ptr(qr_scales),
                                   _ptr(qw_codes), _ptr(qw_scales), M, N, K, _ptr(y), y_type, _stream(stream)),
           "rfq_gemm")


def linear(x, qw_codes, qw_scales, N, y, workspace, use_residual=True, stream=None):
    """rfq_linear: quantize x into `workspace`, then the RFQ GEMM against the
    pre-quantized weight (the single-kernel layer for M <= 32); y's dtype selects
    the output type."""
    import torch
    M, K = x.shape
    y_type = OUT_BF16 if y.dtype == torch.bfloat16 else OUT_F32
    _check(load_library().rfq_linear(_ptr(x), M, K, _ptr(qw_codes), _ptr(qw_scales), N, _ptr(y), y_type,
                                     int(bool(use_residual)), _ptr(workspace), workspace.numel(), _stream(stream)),
           "rfq_linear")


def linear_static_workspace(x, qw_codes, qw_scales, N, y, use_residual=True, stream=None):
    """rfq_linear_static_workspace: the RFQ linear layer for callers that cannot allocate
    device memory; the quantized activation goes into the library's fixed 32 MiB scratch
    array (see include/rfq.h for the size limit and the no-overlap rule)."""
    import torch
    M, K = x.shape
    y_type = OUT_BF16 if y.dtype == torch.bfloat16 else OUT_F32
    _check(load_library().rfq_linear_static_workspace(_ptr(x), M, K, _ptr(qw_codes), _ptr(qw_scales), N, _ptr(y),
                                                      y_type, int(bool(use_residual)), _stream(stream)),
           "rfq_linear_static_workspace")


def linear_fused(x, qw_codes, qw_scales, N, y, use_residual=True, stream=None):
    """rfq_linear_fused: the RFQ linear layer in one kernel (quantizer inside the GEMM)
    for M <= FUSED_MAX_M rows; no workspace."""
    import torch
    M, K = x.shape
    y_type = OUT_BF16 if y.dtype == torch.bfloat16 else OUT_F32
    _check(load_library().rfq_linear_fused(_ptr(x), M, K, _ptr(qw_codes), _ptr(qw_scales), N, _ptr(y), y_type,
                                           int(bool(use_residual)), _stream(stream)),
           "rfq_linear_fused")


def debug_fused_split(split: int):
    """Force rfq_linear_fused's split of K over a cluster (1..8); 0 = automatic."""
    _check(load_library().rfq_debug_fused_split(int(split)), "rfq_debug_fused_split")


def quantize_mxfp4_t(x, qt_codes, qt_scales, qr_codes=None, qr_scales=None, stream=None):
    """rfq_quantize_mxfp4_t: the MXFP4 operand of x^T (x is [R][C]; blocks along R)."""
    R, C = x.shape
    _check(load_library().rfq_quantize_mxfp4_t(_ptr(x), R, C, _ptr(qt_codes), _ptr(qt_scales), _ptr(qr_codes),
                                               _ptr(qr_scales), _stream(stream)), "rfq_quantize_mxfp4_t")


def gemm_yt(qx_codes, qx_scales, qr_codes, qr_scales, qw_codes, qw_scales, M, N, K, yt, stream=None):
    """rfq_gemm_yt: rfq_gemm writing Y^T ([N][M])."""
    import torch
    y_type = OUT_BF16 if yt.dtype == torch.bfloat16 else OUT_F32
    _check(load_library().rfq_gemm_yt(_ptr(qx_codes), _ptr(qx_scales), _ptr(qr_codes), _ptr(qr_scales),
                                      _ptr(qw_codes), _ptr(qw_scales), M, N, K, _ptr(yt), y_type, _stream(stream)),
           "rfq_gemm_yt")


def linear_dgrad(dy, qwt_codes, qwt_scales, K, dx, workspace, use_residual=True, stream=None):
    """rfq_linear_dgrad: dX = dY . W (W^T pre-quantized along N by quantize_mxfp4_t)."""
    import torch
    M, N = dy.shape
    y_type = OUT_BF16 if dx.dtype == torch.bfloat16 else OUT_F32
    _check(load_library().rfq_linear_dgrad(_ptr(dy), M, N, _ptr(qwt_codes), _ptr(qwt_scales), K, _ptr(dx), y_type,
                                           int(bool(use_residual)), _ptr(workspace), workspace.numel(),
                                           _stream(stream)), "rfq_linear_dgrad")


def linear_wgrad_workspace_bytes(M: int, K: int, N: int, use_residual: bool = True) -> int:
    """rfq_linear_wgrad_workspace_bytes: workspace of rfq_linear_wgrad for x [M, K], dy [M, N]."""
    return int(load_library().rfq_linear_wgrad_workspace_bytes(M, K, N, int(bool(use_residual))))


def linear_wgrad(x, dy, dw, workspace, use_residual=True, stream=None):
    """rfq_linear_wgrad: dW [N][K] = dY^T . X with both quantized along the M tokens."""
    import torch
    M, K = x.shape
    N = dy.shape[1]
    y_type = OUT_BF16 if dw.dtype == torch.bfloat16 else OUT_F32
    _check(load_library().rfq_linear_wgrad(_ptr(x), _ptr(dy), M, K, N, _ptr(dw), y_type, int(bool(use_residual)),
                                           _ptr(workspace), workspace.numel(), _stream(stream)), "rfq_linear_wgrad")


def mxfp8_codes_bytes(rows: int, K: int) -> int:
    """rfq_mxfp8_codes_bytes: bytes of E4M3 codes for [rows, K] (one byte per element)."""
    return int(load_library().rfq_mxfp8_codes_bytes(rows, K))


def quantize_mxfp8(x, codes, scales, stream=None):
    """rfq_quantize_mxfp8: the MXFP8 (E4M3) comparator quantizer."""
    M, K = x.shape
    _check(load_library().rfq_quantize_mxfp8(_ptr(x), M, K, _ptr(codes), _ptr(scales), _stream(stream)),
           "rfq_quantize_mxfp8")


def gemm_mxfp8(qx_codes, qx_scales, qw_codes, qw_scales, M, N, K, y, stream=None):
    """rfq_gemm_mxfp8: Y = DQ(QX) . DQ(QW)^T on kind::mxf8f6f4 MMAs."""
    import torch
    y_type = OUT_BF16 if y.dtype == torch.bfloat16 else OUT_F32
    _check(load_library().rfq_gemm_mxfp8(_ptr(qx_codes), _ptr(qx_scales), _ptr(qw_codes), _ptr(qw_scales),
                                         M, N, K, _ptr(y), y_type, _stream(stream)), "rfq_gemm_mxfp8")


def check_device_error(stream=None):
    """Synchronize and report a bounded-wait timeout inside a kernel (raises RFQError)."""
    detail = ctypes.c_int(0)
    st = load_library().rfq_check_device_error(_stream(stream), ctypes.byref(detail))
    if st != 0:
        err = RFQError(st, f"rfq_check_device_error (detail {detail.value})")
        err.detail = detail.value
        raise err
    return 0


def debug_skip_next_fill(fill_index: int):
    """rfq_debug_skip_next_fill: test hook; the next GEMM's first CTA skips stage
    fill `fill_index` (its bounded wait then runs out)."""
    load_library().rfq_debug_skip_next_fill(int(fill_index))


# ----------------------------------------------------------------------------- allocating conveniences
class QuantizedTensor:
    """Codes and MMA-layout scales of an MXFP4 matrix [rows, K] (plus Q(R) when present)."""

    def __init__(self, rows, K, codes, scales, r_codes=None, r_scales=None):
        self.rows, self.K = rows, K
        self.codes, self.scales = codes, scales
        self.r_codes, self.r_scales = r_codes, r_scales

    @property
    def has_residual(self):
        return self.r_codes is not None


def _empty_u8(n, device):
    import torch
    # over-allocate by nothing; torch's caching allocator returns 512-byte aligned blocks
    return torch.empty(max(int(n), 1), dtype=torch.uint8, device=device)


def quantize_mxfp4_alloc(x, residual=True, stream=None) -> QuantizedTensor:
    """quantize_mxfp4 into freshly allocated buffers; Q(R) too when `residual`."""
    M, K = x.shape
    cb, sb = codes_bytes(M, K), scales_bytes(M, K)
    q = QuantizedTensor(M, K, _empty_u8(cb, x.device), _empty_u8(sb, x.device),
                        _empty_u8(cb, x.device) if residual else None, _empty_u8(sb, x.device) if residual else None)
    quantize_mxfp4(x, q.codes, q.scales, q.r_codes, q.r_scales, stream)
    return q


def quantize_weight_alloc(w, stream=None) -> QuantizedTensor:
    """quantize_weight into freshly allocated buffers."""
    N, K = w.shape
    q = QuantizedTensor(N, K, _empty_u8(codes_bytes(N, K), w.device), _empty_u8(scales_bytes(N, K), w.device))
    quantize_weight(w, q.codes, q.scales, stream)
    return q


def gemm_alloc(qa: QuantizedTensor, qw: QuantizedTensor, out_dtype=None, use_residual=True, stream=None):
    """rfq_gemm of two QuantizedTensors into a new [qa.rows, qw.rows] tensor (bf16 unless `out_dtype`)."""
    import torch
    out_dtype = out_dtype or torch.bfloat16
    y = torch.empty((qa.rows, qw.rows), dtype=out_dtype, device=qa.codes.device)
    res = use_residual and qa.has_residual
    gemm(qa.codes, qa.scales, qa.r_codes if res else None, qa.r_scales if res else None, qw.codes, qw.scales,
         qa.rows, qw.rows, qa.K, y, stream)
    return y


def linear_fused_alloc(x, qw: QuantizedTensor, out_dtype=None, use_residual=True, stream=None):
    """rfq_linear_fused into a new [M, qw.rows] tensor (bf16 unless `out_dtype`)."""
    import torch
    out_dtype = out_dtype or torch.bfloat16
    y = torch.empty((x.shape[0], qw.rows), dtype=out_dtype, device=x.device)
    linear_fused(x, qw.codes, qw.scales, qw.rows, y, use_residual, stream)
    return y


def quantize_mxfp4_t_alloc(x, residual=True, stream=None) -> QuantizedTensor:
    """The operand of x^T: rows = x's columns, K = x's rows."""
    R, C = x.shape
    cb, sb = codes_bytes(C, R), scales_bytes(C, R)
    q = QuantizedTensor(C, R, _empty_u8(cb, x.device), _empty_u8(sb, x.device),
                        _empty_u8(cb, x.device) if residual else None, _empty_u8(sb, x.device) if residual else None)
    quantize_mxfp4_t(x, q.codes, q.scales, q.r_codes, q.r_scales, stream)
    return q


def linear_dgrad_alloc(dy, qwt: QuantizedTensor, out_dtype=None, use_residual=True, stream=None):
    """rfq_linear_dgrad with a fresh workspace: dX [M, K] for dy [M, N] and Q(W^T) `qwt` (rows K)."""
    import torch
    M, N = dy.shape
    dx = torch.empty((M, qwt.rows), dtype=out_dtype or torch.bfloat16, device=dy.device)
    ws = _empty_u8(linear_workspace_bytes(M, N, use_residual), dy.device)
    linear_dgrad(dy, qwt.codes, qwt.scales, qwt.rows, dx, ws, use_residual, stream)
    return dx


def linear_wgrad_alloc(x, dy, out_dtype=None, use_residual=True, stream=None):
    """rfq_linear_wgrad with a fresh workspace: dW [N, K] for x [M, K] and dy [M, N]."""
    import torch
    M, K = x.shape
    N = dy.shape[1]
    dw = torch.empty((N, K), dtype=out_dtype or torch.bfloat16, device=x.device)
    ws = _empty_u8(linear_wgrad_workspace_bytes(M, K, N, use_residual), x.device)
    linear_wgrad(x, dy, dw, ws, use_residual, stream)
    return dw


def quantize_mxfp8_alloc(x, stream=None) -> QuantizedTensor:
    """quantize_mxfp8 into freshly allocated buffers."""
    M, K = x.shape
    q = QuantizedTensor(M, K, _empty_u8(mxfp8_codes_bytes(M, K), x.device), _empty_u8(scales_bytes(M, K), x.device))
    quantize_mxfp8(x, q.codes, q.scales, stream)
    return q


def gemm_mxfp8_alloc(qa: QuantizedTensor, qw: QuantizedTensor, out_dtype=None, stream=None):
    """rfq_gemm_mxfp8 of two MXFP8 QuantizedTensors into a new tensor (bf16 unless `out_dtype`)."""
    import torch
    y = torch.empty((qa.rows, qw.rows), dtype=out_dtype or torch.bfloat16, device=qa.codes.device)
    gemm_mxfp8(qa.codes, qa.scales, qw.codes, qw.scales, qa.rows, qw.rows, qa.K, y, stream)
    return y


def linear_alloc(x, qw: QuantizedTensor, out_dtype=None, use_residual=True, stream=None):
    """rfq_linear with a fresh workspace and output (bf16 unless `out_dtype`)."""
    import torch
    M, K = x.shape
    out_dtype = out_dtype or torch.bfloat16
    y = torch.empty((M, qw.rows), dtype=out_dtype, device=x.device)
    ws = _empty_u8(linear_workspace_bytes(M, K, use_residual), x.device)
    linear(x, qw.codes, qw.scales, qw.rows, y, ws, use_residual, stream)
    return y


def mma_rate_probe(variant, iterations, cycles, stream=None):
    """rfq_mma_rate_probe: issue `iterations` x 8 MMAs of the GEMM's shape on every SM
    with shared-memory-resident operands (variant 0 = kind::mxf4 CTA pairs, 1 = kind::mxf4
    single CTAs, 2 = kind::mxf8f6f4 CTA pairs).  `cycles` is an int64 device tensor with
    one word per cluster; returns (flops the launch executes, SMs it ran on)."""
    flops = ctypes.c_double(0.0)
    sms = ctypes.c_int(0)
    _check(load_library().rfq_mma_rate_probe(int(variant), int(iterations), _ptr(cycles), cycles.numel(),
                                             ctypes.byref(flops), ctypes.byref(sms), _stream(stream)),
           "rfq_mma_rate_probe")
    return flops.value, sms.value
