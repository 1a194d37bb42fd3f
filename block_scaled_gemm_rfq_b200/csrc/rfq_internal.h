// rfq_internal.h -- launchers shared between the kernels' .cu files and the C ABI.
// Arguments are validated by the C ABI (rfq_api.cu) before these are called.
#pragma once

#include <cuda_runtime.h>

#include <cstdint>

namespace rfq {

// Kernel 1: fused quantizer.  qr_codes == nullptr selects plain MXFP4.
// `encode_tiled` is the driver's cuTensorMapEncodeTiled.
cudaError_t launch_quantize(const void* x, int64_t M, int64_t K, void* qx_codes, void* qx_scales, void* qr_codes,
                            void* qr_scales, int num_sms, void* encode_tiled, cudaStream_t stream);

// Kernel 1 as the MXFP8 (E4M3) comparator quantizer: codes one byte per element.
cudaError_t launch_quantize_mxfp8(const void* x, int64_t M, int64_t K, void* codes, void* scales, int num_sms,
                                  void* encode_tiled, cudaStream_t stream);

// Kernel 1t: quantizer of X^T for a row-major X [R][C] (blocks along R).
cudaError_t launch_quantize_t(const void* x, int64_t R, int64_t C, void* qt_codes, void* qt_scales, void* qr_codes,
                              void* qr_scales, int num_sms, void* encode_tiled, cudaStream_t stream);

// Kernel 2: RFQ GEMM (y_transposed: Y written as [N][M]).  qr_codes == nullptr selects the plain MXFP4 GEMM.
// `encode_tiled` is the driver's cuTensorMapEncodeTiled.  `skip_fill` >= 0 makes
// the producer of CTA 0 skip that stage fill (fault injection for the bounded
// waits; -1 in normal use).
cudaError_t launch_gemm(const void* qx_codes, const void* qx_scales, const void* qr_codes, const void* qr_scales,
                        const void* qw_codes, const void* qw_scales, int64_t M, int64_t N, int64_t K, void* y,
                        bool y_bf16, bool y_transposed, int num_sms, void* encode_tiled, int skip_fill,
                        cudaStream_t stream);

// Single-kernel RFQ linear layer for M <= 64 (quantizer inside the GEMM).
cudaError_t launch_linear_fused(const void* x, int64_t M, int64_t K, const void* qw_codes, const void* qw_scales,
                                int64_t N, void* y, bool y_bf16, bool residual, int num_sms, void* encode_tiled,
                                cudaStream_t stream);
void set_fused_split_override(int split);   // 0 = automatic

// The same kernel for pre-quantized operands (M <= 256): Q(X), Q(R) as written by
// the quantizer come in by TMA; the GEMM's M <= 256 path when its tiles are few.
cudaError_t launch_gemm_short(const void* qx_codes, const void* qx_scales, const void* qr_codes,
                              const void* qr_scales, const void* qw_codes, const void* qw_scales, int64_t M,
                              int64_t N, int64_t K, void* y, bool y_bf16, int num_sms, void* encode_tiled,
                              int skip_fill, cudaStream_t stream);
constexpr int64_t kShortGemmMaxM = 256;

// The MXFP8 comparator GEMM: E4M3 codes (one byte per element) with E8M0 scales in
// the same MMA layout, plain (no residual term).
cudaError_t launch_gemm_mxfp8(const void* qx_codes, const void* qx_scales, const void* qw_codes,
                              const void* qw_scales, int64_t M, int64_t N, int64_t K, void* y, bool y_bf16,
                              int num_sms, void* encode_tiled, cudaStream_t stream);

// Tensor-core rate probe: up to `max_clusters` clusters (of 2 CTAs for variants 0
// and 2), no more than can be resident at once, issue `iters` x 8 MMAs of the
// GEMM's shapes on shared-memory-resident operands; variant 0 = kind::mxf4 CTA
// pair (M 256), 1 = kind::mxf4 single CTA (M 128), 2 = kind::mxf8f6f4 CTA pair.
// cycles[cluster] = the issuing thread's clock64 span; *clusters_used = clusters launched.
cudaError_t launch_mma_rate_probe(int variant, int iters, unsigned long long* cycles, int max_clusters,
                                  int* clusters_used, cudaStream_t stream);

// Read and clear the device error words (GEMM and quantizer) of the current device.
cudaError_t read_and_clear_device_error(unsigned int* value);
cudaError_t read_and_clear_quant_error(unsigned int* value);
cudaError_t read_and_clear_fused_error(unsigned int* value);

}  // namespace rfq
