// rfq_api.cu -- the C ABI declared in include/rfq.h: argument validation, device
// checks, status codes and launch sequencing.  No allocation, no exceptions.
#include <cuda.h>
#include <cuda_runtime.h>

#include <atomic>
#include <cstdint>
#include <cstring>
#include <mutex>

#include "rfq.h"
#include "rfq_internal.h"

namespace {

constexpr int kMaxDevices = 64;

struct DeviceInfo {
  std::atomic<int> state{0};  // 0 unknown, 1 supported, 2 unsupported
  int num_sms = 0;
};

DeviceInfo g_devices[kMaxDevices];
std::mutex g_init_mutex;
void* g_encode_tiled = nullptr;
std::atomic<int> g_skip_fill{-1};

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

rfq_status_t from_cuda(cudaError_t e) { return e == cudaSuccess ? RFQ_OK : RFQ_ERR_CUDA; }

// Checks the current device (compute capability 10.0) and returns its SM count.
rfq_status_t current_device(int* num_sms) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return RFQ_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return RFQ_ERR_UNSUPPORTED_DEVICE;
  DeviceInfo& d = g_devices[dev];
  int st = d.state.load(std::memory_order_acquire);
  if (st == 0) {
    std::lock_guard<std::mutex> lock(g_init_mutex);
    st = d.state.load(std::memory_order_relaxed);
    if (st == 0) {
      int major = 0, minor = 0, sms = 0;
      if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
          cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess ||
          cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
        return RFQ_ERR_CUDA;
      if (g_encode_tiled == nullptr) {
        cudaDriverEntryPointQueryResult q;
        void* fn = nullptr;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) != cudaSuccess ||
            q != cudaDriverEntryPointSuccess || fn == nullptr)
          return RFQ_ERR_CUDA;
        g_encode_tiled = fn;
      }
      d.num_sms = sms;
      st = (major == 10 && minor == 0) ? 1 : 2;
      d.state.store(st, std::memory_order_release);
    }
  }
  if (st != 1) return RFQ_ERR_UNSUPPORTED_DEVICE;
  *num_sms = d.num_sms;
  return RFQ_OK;
}

size_t align256(size_t v) { return (v + 255) & ~size_t(255); }

// Limits: rows and K fit the kernels' 32-bit tile coordinates, a matrix holds at
// most 2^31 - 64 blocks of 32 elements (the quantizer's 32-bit block indices and
// TMA row coordinate, which runs up to a span past the last block), and a scale
// array stays below 2^32 bytes (32-bit offsets).
bool shape_ok(int64_t rows, int64_t K) {
  if (rows < 0 || K < 0 || (K % 32) != 0 || rows > (int64_t(1) << 31) - 1 || K > (int64_t(1) << 31) - 32) return false;
  if (K == 0) return true;
  const int64_t kb = K / 32;
  if (rows > ((int64_t(1) << 31) - 64) / kb) return false;
  // the scale array (rows padded to 128, blocks to 4) stays below 2^32 bytes
  return (rows + 127) / 128 * 128 * ((kb + 3) / 4 * 4) < (int64_t(1) << 32);
}

rfq_status_t check_quantize_args(const void* x, int64_t M, int64_t K, const void* qc, const void* qs, const void* rc,
                                 const void* rs) {
  if (M < 0 || K < 0) return RFQ_ERR_INVALID_ARG;
  if (!shape_ok(M, K)) return RFQ_ERR_UNSUPPORTED_SHAPE;
  if ((rc == nullptr) != (rs == nullptr)) return RFQ_ERR_INVALID_ARG;
  if (M == 0 || K == 0) return RFQ_OK;
  if (!x || !qc || !qs) return RFQ_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned16(qc) || !aligned16(qs) || (rc && (!aligned16(rc) || !aligned16(rs))))
    return RFQ_ERR_MISALIGNED;
  return RFQ_OK;
}

rfq_status_t quantize_impl(const void* x, int64_t M, int64_t K, void* qc, void* qs, void* rc, void* rs,
                           cudaStream_t stream) {
  rfq_status_t st = check_quantize_args(x, M, K, qc, qs, rc, rs);
  if (st != RFQ_OK) return st;
  if (M == 0) return RFQ_OK;
  int sms = 0;
  if ((st = current_device(&sms)) != RFQ_OK) return st;
  if (K == 0) {
    // No blocks: the scale arrays have no bytes (rfq_scales_bytes == 0); nothing to do.
    return RFQ_OK;
  }
  return from_cuda(rfq::launch_quantize(x, M, K, qc, qs, rc, rs, sms, g_encode_tiled, stream));
}

rfq_status_t gemm_impl(const void* qxc, const void* qxs, const void* qrc, const void* qrs, const void* qwc,
                       const void* qws, int64_t M, int64_t N, int64_t K, void* y, rfq_out_t y_type,
                       cudaStream_t stream, bool y_transposed = false) {
  if (M < 0 || N < 0 || K < 0) return RFQ_ERR_INVALID_ARG;
  if (y_type != RFQ_OUT_F32 && y_type != RFQ_OUT_BF16) return RFQ_ERR_INVALID_ARG;
  if ((qrc == nullptr) != (qrs == nullptr)) return RFQ_ERR_INVALID_ARG;
  if (!shape_ok(M, K) || !shape_ok(N, K) || (N % 8) != 0) return RFQ_ERR_UNSUPPORTED_SHAPE;
  if (M == 0 || N == 0) return RFQ_OK;
  if (!y) return RFQ_ERR_INVALID_ARG;
  if (!aligned16(y)) return RFQ_ERR_MISALIGNED;
  int sms = 0;
  rfq_status_t st = current_device(&sms);
  if (st != RFQ_OK) return st;
  const size_t y_bytes = static_cast<size_t>(M) * static_cast<size_t>(N) * (y_type == RFQ_OUT_BF16 ? 2u : 4u);
  if (K == 0) return from_cuda(cudaMemsetAsync(y, 0, y_bytes, stream));
  if (!qxc || !qxs || !qwc || !qws) return RFQ_ERR_INVALID_ARG;
  if (!aligned16(qxc) || !aligned16(qxs) || !aligned16(qwc) || !aligned16(qws) ||
      (qrc && (!aligned16(qrc) || !aligned16(qrs))))
    return RFQ_ERR_MISALIGNED;
  const int skip = g_skip_fill.exchange(-1);
  // Short batches whose tiles would fill less than half the SMs (M <= 128: one
  // CTA per 256 columns; M <= 256: one CTA pair) go to the split-K kernel.
  const int64_t tile_ctas = (M <= 128 ? 1 : 2) * ((N + 255) / 256);
  if (!y_transposed && M <= rfq::kShortGemmMaxM && tile_ctas < sms / 2)
    return from_cuda(rfq::launch_gemm_short(qxc, qxs, qrc, qrs, qwc, qws, M, N, K, y, y_type == RFQ_OUT_BF16, sms,
                                            g_encode_tiled, skip, stream));
  return from_cuda(rfq::launch_gemm(qxc, qxs, qrc, qrs, qwc, qws, M, N, K, y, y_type == RFQ_OUT_BF16,
                                    y_transposed, sms, g_encode_tiled, skip, stream));
}

rfq_status_t quantize8_impl(const void* x, int64_t M, int64_t K, void* qc, void* qs, cudaStream_t stream) {
  rfq_status_t st = check_quantize_args(x, M, K, qc, qs, nullptr, nullptr);
  if (st != RFQ_OK) return st;
  if (M == 0 || K == 0) return RFQ_OK;
  int sms = 0;
  if ((st = current_device(&sms)) != RFQ_OK) return st;
  return from_cuda(rfq::launch_quantize_mxfp8(x, M, K, qc, qs, sms, g_encode_tiled, stream));
}

rfq_status_t quantize_t_impl(const void* x, int64_t R, int64_t C, void* qc, void* qs, void* rc, void* rs,
                             cudaStream_t stream) {
  if (R < 0 || C < 0) return RFQ_ERR_INVALID_ARG;
  if (!shape_ok(C, R) || (C % 8) != 0) return RFQ_ERR_UNSUPPORTED_SHAPE;
  if ((rc == nullptr) != (rs == nullptr)) return RFQ_ERR_INVALID_ARG;
  if (R == 0 || C == 0) return RFQ_OK;
  if (!x || !qc || !qs) return RFQ_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned16(qc) || !aligned16(qs) || (rc && (!aligned16(rc) || !aligned16(rs))))
    return RFQ_ERR_MISALIGNED;
  int sms = 0;
  rfq_status_t st = current_device(&sms);
  if (st != RFQ_OK) return st;
  return from_cuda(rfq::launch_quantize_t(x, R, C, qc, qs, rc, rs, sms, g_encode_tiled, stream));
}

rfq_status_t fused_impl(const void* x, int64_t M, int64_t K, const void* qwc, const void* qws, int64_t N, void* y,
                        rfq_out_t y_type, int use_residual, cudaStream_t stream) {
  if (M < 0 || N < 0 || K < 0) return RFQ_ERR_INVALID_ARG;
  if (y_type != RFQ_OUT_F32 && y_type != RFQ_OUT_BF16) return RFQ_ERR_INVALID_ARG;
  if (!shape_ok(M, K) || !shape_ok(N, K) || (N % 8) != 0 || M > RFQ_FUSED_MAX_M) return RFQ_ERR_UNSUPPORTED_SHAPE;
  if (M == 0 || N == 0) return RFQ_OK;
  if (!y) return RFQ_ERR_INVALID_ARG;
  if (!aligned16(y)) return RFQ_ERR_MISALIGNED;
  int sms = 0;
  rfq_status_t st = current_device(&sms);
  if (st != RFQ_OK) return st;
  const size_t y_bytes = static_cast<size_t>(M) * static_cast<size_t>(N) * (y_type == RFQ_OUT_BF16 ? 2u : 4u);
  if (K == 0) return from_cuda(cudaMemsetAsync(y, 0, y_bytes, stream));
  if (!x || !qwc || !qws) return RFQ_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned16(qwc) || !aligned16(qws)) return RFQ_ERR_MISALIGNED;
  return from_cuda(rfq::launch_linear_fused(x, M, K, qwc, qws, N, y, y_type == RFQ_OUT_BF16, use_residual != 0, sms,
                                            g_encode_tiled, stream));
}

}  // namespace

extern "C" {

const char* rfq_status_string(rfq_status_t status) {
  switch (status) {
    case RFQ_OK: return "RFQ_OK";
    case RFQ_ERR_INVALID_ARG: return "RFQ_ERR_INVALID_ARG";
    case RFQ_ERR_UNSUPPORTED_SHAPE: return "RFQ_ERR_UNSUPPORTED_SHAPE";
    case RFQ_ERR_MISALIGNED: return "RFQ_ERR_MISALIGNED";
    case RFQ_ERR_UNSUPPORTED_DEVICE: return "RFQ_ERR_UNSUPPORTED_DEVICE";
    case RFQ_ERR_CUDA: return "RFQ_ERR_CUDA";
    case RFQ_ERR_TIMEOUT: return "RFQ_ERR_TIMEOUT";
    case RFQ_ERR_WORKSPACE: return "RFQ_ERR_WORKSPACE";
  }
  return "RFQ_ERR_UNKNOWN";
}

size_t rfq_codes_bytes(int64_t rows, int64_t K) {
  if (!shape_ok(rows, K)) return 0;
  return static_cast<size_t>(rows) * static_cast<size_t>(K / 2);
}

size_t rfq_scales_bytes(int64_t rows, int64_t K) {
  if (!shape_ok(rows, K)) return 0;
  const size_t rows_pad = static_cast<size_t>((rows + 127) / 128 * 128);
  const size_t kb_pad = static_cast<size_t>((K / 32 + 3) / 4 * 4);
  return rows_pad * kb_pad;
}

rfq_status_t rfq_quantize_mxfp4(const void* x_bf16, int64_t M, int64_t K, void* qx_codes, void* qx_scales,
                                void* qr_codes, void* qr_scales, cudaStream_t stream) {
  return quantize_impl(x_bf16, M, K, qx_codes, qx_scales, qr_codes, qr_scales, stream);
}

rfq_status_t rfq_quantize_weight(const void* w_bf16, int64_t N, int64_t K, void* qw_codes, void* qw_scales,
                                 cudaStream_t stream) {
  return quantize_impl(w_bf16, N, K, qw_codes, qw_scales, nullptr, nullptr, stream);
}

rfq_status_t rfq_gemm(const void* qx_codes, const void* qx_scales, const void* qr_codes, const void* qr_scales,
                      const void* qw_codes, const void* qw_scales, int64_t M, int64_t N, int64_t K, void* y,
                      rfq_out_t y_type, cudaStream_t stream) {
  return gemm_impl(qx_codes, qx_scales, qr_codes, qr_scales, qw_codes, qw_scales, M, N, K, y, y_type, stream);
}

size_t rfq_linear_workspace_bytes(int64_t M, int64_t K, int use_residual) {
  if (!shape_ok(M, K)) return 0;
  const size_t one = align256(rfq_codes_bytes(M, K)) + align256(rfq_scales_bytes(M, K));
  return use_residual ? 2 * one : one;
}

rfq_status_t rfq_linear(const void* x_bf16, int64_t M, int64_t K, const void* qw_codes, const void* qw_scales,
                        int64_t N, void* y, rfq_out_t y_type, int use_residual, void* workspace,
                        size_t workspace_bytes, cudaStream_t stream) {
  if (M < 0 || N < 0 || K < 0) return RFQ_ERR_INVALID_ARG;
  if (y_type != RFQ_OUT_F32 && y_type != RFQ_OUT_BF16) return RFQ_ERR_INVALID_ARG;
  if (!shape_ok(M, K) || !shape_ok(N, K) || (N % 8) != 0) return RFQ_ERR_UNSUPPORTED_SHAPE;
  if (M == 0 || N == 0) return RFQ_OK;
  const size_t need = rfq_linear_workspace_bytes(M, K, use_residual);
  if (K > 0 && (workspace == nullptr || workspace_bytes < need)) return RFQ_ERR_WORKSPACE;
  if (K > 0 && (reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return RFQ_ERR_MISALIGNED;
  if (K > 0 && (!x_bf16 || !qw_codes || !qw_scales)) return RFQ_ERR_INVALID_ARG;
  // Up to 32 rows the single kernel wins; from ~48 rows its repeated quantization
  // of X per weight tile costs more than the quantizer launch it saves, and the
  // quantizer + split-K short-batch GEMM pair is as fast or faster (measured).
  if (M <= 32) return fused_impl(x_bf16, M, K, qw_codes, qw_scales, N, y, y_type, use_residual, stream);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  const size_t cb = align256(rfq_codes_bytes(M, K));
  const size_t sb = align256(rfq_scales_bytes(M, K));
  void* qxc = ws;
  void* qxs = ws ? ws + cb : nullptr;
  void* qrc = (use_residual && ws) ? ws + cb + sb : nullptr;
  void* qrs = (use_residual && ws) ? ws + 2 * cb + sb : nullptr;
  rfq_status_t st = quantize_impl(x_bf16, M, K, qxc, qxs, qrc, qrs, stream);
  if (st != RFQ_OK) return st;
  return gemm_impl(qxc, qxs, qrc, qrs, qw_codes, qw_scales, M, N, K, y, y_type, stream);
}

rfq_status_t rfq_linear_fused(const void* x_bf16, int64_t M, int64_t K, const void* qw_codes, const void* qw_scales,
                              int64_t N, void* y, rfq_out_t y_type, int use_residual, cudaStream_t stream) {
  return fused_impl(x_bf16, M, K, qw_codes, qw_scales, N, y, y_type, use_residual, stream);
}

rfq_status_t rfq_quantize_mxfp4_t(const void* x_bf16, int64_t R, int64_t C, void* qt_codes, void* qt_scales,
                                  void* qr_codes, void* qr_scales, cudaStream_t stream) {
  return quantize_t_impl(x_bf16, R, C, qt_codes, qt_scales, qr_codes, qr_scales, stream);
}

rfq_status_t rfq_gemm_yt(const void* qx_codes, const void* qx_scales, const void* qr_codes, const void* qr_scales,
                         const void* qw_codes, const void* qw_scales, int64_t M, int64_t N, int64_t K, void* yt,
                         rfq_out_t y_type, cudaStream_t stream) {
  return gemm_impl(qx_codes, qx_scales, qr_codes, qr_scales, qw_codes, qw_scales, M, N, K, yt, y_type, stream, true);
}

rfq_status_t rfq_linear_dgrad(const void* dy_bf16, int64_t M, int64_t N, const void* qwt_codes,
                              const void* qwt_scales, int64_t K, void* dx, rfq_out_t dx_type, int use_residual,
                              void* workspace, size_t workspace_bytes, cudaStream_t stream) {
  return rfq_linear(dy_bf16, M, N, qwt_codes, qwt_scales, K, dx, dx_type, use_residual, workspace, workspace_bytes,
                    stream);
}

size_t rfq_linear_wgrad_workspace_bytes(int64_t M, int64_t K, int64_t N, int use_residual) {
  if (!shape_ok(K, M) || !shape_ok(N, M)) return 0;
  const size_t xt = align256(rfq_codes_bytes(K, M)) + align256(rfq_scales_bytes(K, M));
  const size_t dyt = align256(rfq_codes_bytes(N, M)) + align256(rfq_scales_bytes(N, M));
  return (use_residual ? 2 * xt : xt) + dyt;
}

rfq_status_t rfq_linear_wgrad(const void* x_bf16, const void* dy_bf16, int64_t M, int64_t K, int64_t N, void* dw,
                              rfq_out_t dw_type, int use_residual, void* workspace, size_t workspace_bytes,
                              cudaStream_t stream) {
  if (M < 0 || N < 0 || K < 0) return RFQ_ERR_INVALID_ARG;
  if (dw_type != RFQ_OUT_F32 && dw_type != RFQ_OUT_BF16) return RFQ_ERR_INVALID_ARG;
  if (!shape_ok(K, M) || !shape_ok(N, M) || (K % 32) != 0 || (N % 8) != 0) return RFQ_ERR_UNSUPPORTED_SHAPE;
  if (N == 0 || K == 0) return RFQ_OK;
  if (M == 0) return gemm_impl(nullptr, nullptr, nullptr, nullptr, nullptr, nullptr, K, N, 0, dw, dw_type, stream,
                               true);
  const size_t need = rfq_linear_wgrad_workspace_bytes(M, K, N, use_residual);
  if (workspace == nullptr || workspace_bytes < need) return RFQ_ERR_WORKSPACE;
  if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return RFQ_ERR_MISALIGNED;
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  const size_t xcb = align256(rfq_codes_bytes(K, M)), xsb = align256(rfq_scales_bytes(K, M));
  const size_t ycb = align256(rfq_codes_bytes(N, M));
  void* qxc = ws;
  void* qxs = ws + xcb;
  void* qrc = use_residual ? ws + xcb + xsb : nullptr;
  void* qrs = use_residual ? ws + 2 * xcb + xsb : nullptr;
  uint8_t* yt = ws + (use_residual ? 2 * (xcb + xsb) : xcb + xsb);
  rfq_status_t st = quantize_t_impl(x_bf16, M, K, qxc, qxs, qrc, qrs, stream);
  if (st != RFQ_OK) return st;
  st = quantize_t_impl(dy_bf16, M, N, yt, yt + ycb, nullptr, nullptr, stream);
  if (st != RFQ_OK) return st;
  // dW^T [K][N] = (X^T)^ . (dY^T)^T, written transposed: dW [N][K]
  return gemm_impl(qxc, qxs, qrc, qrs, yt, yt + ycb, K, N, M, dw, dw_type, stream, true);
}

size_t rfq_mxfp8_codes_bytes(int64_t rows, int64_t K) {
  if (!shape_ok(rows, K)) return 0;
  return static_cast<size_t>(rows) * static_cast<size_t>(K);
}

rfq_status_t rfq_quantize_mxfp8(const void* x_bf16, int64_t M, int64_t K, void* q_codes, void* q_scales,
                                cudaStream_t stream) {
  return quantize8_impl(x_bf16, M, K, q_codes, q_scales, stream);
}

rfq_status_t rfq_gemm_mxfp8(const void* qx_codes, const void* qx_scales, const void* qw_codes, const void* qw_scales,
                            int64_t M, int64_t N, int64_t K, void* y, rfq_out_t y_type, cudaStream_t stream) {
  if (M < 0 || N < 0 || K < 0) return RFQ_ERR_INVALID_ARG;
  if (y_type != RFQ_OUT_F32 && y_type != RFQ_OUT_BF16) return RFQ_ERR_INVALID_ARG;
  if (!shape_ok(M, K) || !shape_ok(N, K) || (N % 8) != 0) return RFQ_ERR_UNSUPPORTED_SHAPE;
  if (M == 0 || N == 0) return RFQ_OK;
  if (!y) return RFQ_ERR_INVALID_ARG;
  if (!aligned16(y)) return RFQ_ERR_MISALIGNED;
  int sms = 0;
  rfq_status_t st = current_device(&sms);
  if (st != RFQ_OK) return st;
  const size_t y_bytes = static_cast<size_t>(M) * static_cast<size_t>(N) * (y_type == RFQ_OUT_BF16 ? 2u : 4u);
  if (K == 0) return from_cuda(cudaMemsetAsync(y, 0, y_bytes, stream));
  if (!qx_codes || !qx_scales || !qw_codes || !qw_scales) return RFQ_ERR_INVALID_ARG;
  if (!aligned16(qx_codes) || !aligned16(qx_scales) || !aligned16(qw_codes) || !aligned16(qw_scales))
    return RFQ_ERR_MISALIGNED;
  return from_cuda(rfq::launch_gemm_mxfp8(qx_codes, qx_scales, qw_codes, qw_scales, M, N, K, y,
                                          y_type == RFQ_OUT_BF16, sms, g_encode_tiled, stream));
}

rfq_status_t rfq_mma_rate_probe(int variant, int64_t iterations, unsigned long long* cycles, int64_t cycles_len,
                                double* flops, int* sms_used, cudaStream_t stream) {
  if (variant < 0 || variant > 2 || iterations < 1 || iterations > RFQ_MMA_PROBE_MAX_ITERATIONS || !cycles ||
      !flops || !sms_used)
    return RFQ_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(cycles) & 7u) != 0) return RFQ_ERR_MISALIGNED;
  int sms = 0;
  rfq_status_t st = current_device(&sms);
  if (st != RFQ_OK) return st;
  const int pair = variant == 1 ? 1 : 2;
  const int clusters = sms / pair;
  if (cycles_len < clusters) return RFQ_ERR_INVALID_ARG;
  int used = 0;
  st = from_cuda(rfq::launch_mma_rate_probe(variant, static_cast<int>(iterations), cycles, clusters, &used, stream));
  if (st != RFQ_OK) return st;
  const double mma_k = variant == 2 ? 32.0 : 64.0;   // K of one kind::mxf8f6f4 / kind::mxf4 MMA
  *flops = static_cast<double>(used) * static_cast<double>(iterations) * 8.0 * 2.0 * (128.0 * pair) * 256.0 * mma_k;
  *sms_used = used * pair;
  return RFQ_OK;
}

rfq_status_t rfq_check_device_error(cudaStream_t stream, int* detail) {
  if (detail) *detail = 0;
  if (cudaStreamSynchronize(stream) != cudaSuccess) return RFQ_ERR_CUDA;
  unsigned int v = 0, q = 0;
  if (rfq::read_and_clear_device_error(&v) != cudaSuccess) return RFQ_ERR_CUDA;
  unsigned int f = 0;
  if (rfq::read_and_clear_quant_error(&q) != cudaSuccess) return RFQ_ERR_CUDA;
  if (rfq::read_and_clear_fused_error(&f) != cudaSuccess) return RFQ_ERR_CUDA;
  if (v == 0) v = q;
  if (v == 0) v = f;
  if (detail) *detail = static_cast<int>(v);
  return v ? RFQ_ERR_TIMEOUT : RFQ_OK;
}

// Test hook: the next rfq_gemm launch on this process makes CTA 0's producer skip
// its fill number `fill_index` (so a bounded wait runs out); -1 clears it.
rfq_status_t rfq_debug_skip_next_fill(int fill_index) {
  g_skip_fill.store(fill_index < 0 ? -1 : fill_index);
  return RFQ_OK;
}

rfq_status_t rfq_debug_fused_split(int split) {
  if (split < 0 || split > 8) return RFQ_ERR_INVALID_ARG;
  rfq::set_fused_split_override(split);
  return RFQ_OK;
}

}  // extern "C"
