/*
 * rfq.h -- C ABI of the B200 (sm_100a) Residual Fallback Quantization library.
 *
 * The operation (from "Activation Outliers Matter: Robust Recovery for Quantized
 * Multimodal LLMs", abstract and section 1, the RFQ contribution paragraph):
 * a linear layer's activation X is quantized to FP4, the full quantization error
 * R = X - DQ(Q(X)) is quantized again by a second low-bit path, and the GEMM
 * accumulates both contributions:
 *
 *     Y = (DQ(Q(X)) + DQ(Q(R))) . DQ(Q(W))^T
 *
 * with no threshold, nothing dropped and no architectural change to the layer.
 * The FP4 format is MXFP4 (OCP Microscaling v1.0; the pages name it but stop
 * before defining it, at section 3.1):
 *   - blocks of 32 consecutive elements along K share one E8M0 scale byte
 *     s = clamp(floor(log2(amax)) - 2, -127, 127) + 127 (0 for an all-zero block,
 *     0xFF when the block holds a NaN or infinity);
 *   - each element is an E2M1 code: bit 3 sign (copied from the input, so -0
 *     encodes as 0x8), bits 2..0 the magnitude |x| * 2^-(s-127) rounded to the
 *     nearest of {0, .5, 1, 1.5, 2, 3, 4, 6}, ties to even mantissa, values >= 6
 *     saturating to 6;
 *   - R is formed in fp32, where it is exact, and quantized by the same rule.
 *
 * Data layouts (all row-major, K contiguous, caller-owned device memory):
 *   bf16 inputs   X [M][K], W [N][K]                      (2 bytes per element)
 *   codes         [rows][K/2] bytes; element 2j in bits 3..0, 2j+1 in bits 7..4
 *   scales        the layout the Blackwell block-scaled MMA reads: the plain
 *                 [rows][K/32] scale matrix padded to rows_pad = ceil(rows/128)*128
 *                 and kb_pad = ceil(K/32/4)*4 (padding bytes 0), cut into 512-byte
 *                 atoms of 128 rows x 4 blocks stored with the block-tile index
 *                 fastest; inside an atom (r, c) is at (r%32)*16 + (r/32)*4 + c.
 *                 Size: rfq_scales_bytes(rows, K).
 *   Y [M][N]      fp32 or bf16 (rfq_out_t), fully overwritten.
 *
 * Conventions for every call:
 *   - Pointers are device pointers (cudaMalloc'd or equivalent) owned by the
 *     caller; the library allocates no device memory and keeps no pointer after
 *     returning.  Outputs must not alias inputs.
 *   - Work is enqueued asynchronously on `stream` (0 = legacy default stream) on
 *     the current device, which must be compute capability 10.0 (B200/B100).
 *   - Arguments are checked before anything is launched; a failed check returns
 *     a status and launches nothing.  RFQ_ERR_CUDA reports a launch error from
 *     the CUDA runtime.  Faults inside a kernel surface at the caller's next
 *     synchronization.  Spin-waits inside the GEMM are bounded; a wait that runs
 *     out sets a device error word that rfq_check_device_error() reports.
 *   - No C++ exception crosses this boundary.  All functions are thread-safe
 *     (no global mutable host state besides a per-process cache of the device's
 *     properties).
 */
#ifndef RFQ_H_
#define RFQ_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Same type as the CUDA runtime's stream handle; NULL means the default stream. */
typedef struct CUstream_st* cudaStream_t;

typedef enum {
  RFQ_OK = 0,
  RFQ_ERR_INVALID_ARG = 1,       /* NULL pointer, negative size, inconsistent pair */
  RFQ_ERR_UNSUPPORTED_SHAPE = 2, /* K not a multiple of 32, N not a multiple of 8, too large */
  RFQ_ERR_MISALIGNED = 3,        /* a pointer is not 16-byte aligned */
  RFQ_ERR_UNSUPPORTED_DEVICE = 4,/* current device is not compute capability 10.0 */
  RFQ_ERR_CUDA = 5,              /* CUDA runtime error at launch */
  RFQ_ERR_TIMEOUT = 6,           /* a bounded device-side wait ran out (from rfq_check_device_error) */
  RFQ_ERR_WORKSPACE = 7          /* workspace NULL or smaller than rfq_linear_workspace_bytes() */
} rfq_status_t;

typedef enum { RFQ_OUT_F32 = 0, RFQ_OUT_BF16 = 1 } rfq_out_t;

/* Human-readable name of a status (static string, never NULL). */
const char* rfq_status_string(rfq_status_t status);

/* Bytes of a packed code array for a [rows][K] matrix: rows * K / 2.
 * Returns 0 for negative sizes or K not a multiple of 32. */
size_t rfq_codes_bytes(int64_t rows, int64_t K);

/* Bytes of a scale array in the MMA layout: ceil(rows/128)*128 * ceil(K/128)*4.
 * Returns 0 for negative sizes or K not a multiple of 32. */
size_t rfq_scales_bytes(int64_t rows, int64_t K);

/*
 * rfq_quantize_mxfp4 -- the fused single-pass RFQ activation quantizer.
 * Reads X once and writes Q(X) and, when the residual pointers are given, Q(R)
 * with R = X - DQ(Q(X)): the whole quantization error, quantized again by a second
 * low-bit path (section 1).
 *
 *   x_bf16              [M][K] bf16, 16-byte aligned
 *   qx_codes, qx_scales Q(X): rfq_codes_bytes(M, K) and rfq_scales_bytes(M, K) bytes
 *   qr_codes, qr_scales Q(R): same sizes; both NULL = residual path off (plain
 *                       MXFP4); exactly one NULL is RFQ_ERR_INVALID_ARG
 * K must be a multiple of 32; M >= 0 (M == 0 or K == 0 launches nothing).
 * Every byte of the scale arrays, padding included, is written.
 */
rfq_status_t rfq_quantize_mxfp4(const void* x_bf16, int64_t M, int64_t K,
                                void* qx_codes, void* qx_scales,
                                void* qr_codes, void* qr_scales,
                                cudaStream_t stream);

/*
 * rfq_quantize_weight -- plain MXFP4 quantization of W [N][K] (no residual path:
 * weight quantization is the secondary error source, section 1).  Same layouts
 * and rules as rfq_quantize_mxfp4 with rows = N.  Done once per weight.
 */
rfq_status_t rfq_quantize_weight(const void* w_bf16, int64_t N, int64_t K,
                                 void* qw_codes, void* qw_scales,
                                 cudaStream_t stream);

/*
 * rfq_gemm -- the RFQ GEMM: Y = DQ(QX).DQ(QW)^T + DQ(QR).DQ(QW)^T, both terms
 * accumulated in fp32 into one accumulator (equivalently one GEMM over the
 * concatenated K, [QX | QR] against [QW | QW]): the residual's product is added
 * inside the GEMM (section 1).
 * qr_codes == qr_scales == NULL gives the plain MXFP4 GEMM (residual path off).
 *
 *   qx_*, qr_*   [M][K] operands as written by rfq_quantize_mxfp4
 *   qw_*         [N][K] operand as written by rfq_quantize_weight
 *   y            [M][N], y_type fp32 or bf16 (round to nearest even), 16-byte aligned
 * K multiple of 32; N multiple of 8.  M == 0 or N == 0 launches nothing;
 * K == 0 writes zeros.  Tensor cores: tcgen05 kind::mxf4 block-scaled MMAs.
 * Short batches (M <= 256) whose output tiles would occupy less than half the
 * SMs run a split-K kernel instead: 128 weight rows and up to 128 rows of X per
 * CTA (two row blocks above 128 rows), K split over a cluster of up to 8 CTAs,
 * the Q(X) and Q(R) products in separate accumulator columns added per output,
 * partial sums added in a fixed order (the result differs from the tiled
 * kernel's only by fp32 summation order).
 */
rfq_status_t rfq_gemm(const void* qx_codes, const void* qx_scales,
                      const void* qr_codes, const void* qr_scales,
                      const void* qw_codes, const void* qw_scales,
                      int64_t M, int64_t N, int64_t K,
                      void* y, rfq_out_t y_type, cudaStream_t stream);

/*
 * rfq_quantize_mxfp4_t -- quantize the transpose of a row-major bf16 matrix, for the
 * backward GEMMs of a training step (whose contractions run over a different axis
 * than the forward's; the paper frames RFQ as FP4 *training*-aware, section 1, and
 * gives no backward rule, so gradients pass the quantizers unchanged: straight
 * through).  X is [R][C]; the output is the operand of X^T ([C][R], 32-element
 * blocks along R) in exactly the layouts rfq_quantize_mxfp4 writes for a [C][R]
 * matrix: codes rfq_codes_bytes(C, R), scales rfq_scales_bytes(C, R).  Same rules
 * (scale, rounding, residual R^T = X^T - DQ(Q(X^T)) when qr_* are given).
 *
 *   x_bf16   [R][C] bf16, 16-byte aligned; R a multiple of 32, C a multiple of 8
 * R == 0 or C == 0 launches nothing.  Every byte of the scale arrays is written.
 */
rfq_status_t rfq_quantize_mxfp4_t(const void* x_bf16, int64_t R, int64_t C,
                                  void* qt_codes, void* qt_scales,
                                  void* qr_codes, void* qr_scales,
                                  cudaStream_t stream);

/*
 * rfq_gemm_yt -- rfq_gemm writing the transposed product: yt is [N][M] with
 * yt[n][m] = Y[m][n].  Same operands, rules and accumulation as rfq_gemm.
 */
rfq_status_t rfq_gemm_yt(const void* qx_codes, const void* qx_scales,
                         const void* qr_codes, const void* qr_scales,
                         const void* qw_codes, const void* qw_scales,
                         int64_t M, int64_t N, int64_t K,
                         void* yt, rfq_out_t y_type, cudaStream_t stream);

/* Workspace bytes rfq_linear needs for an [M][K] activation: codes and scales
 * of Q(X) and, when use_residual, of Q(R), each sub-buffer 256-byte aligned. */
size_t rfq_linear_workspace_bytes(int64_t M, int64_t K, int use_residual);

/*
 * rfq_linear -- the RFQ linear layer: rfq_quantize_mxfp4 of X into the caller's
 * workspace, then rfq_gemm against the pre-quantized weight, on one stream
 * (the method leaves the network unchanged: a drop-in for the layer's GEMM).
 * For 1 <= M <= 32 it runs rfq_linear_fused instead (same arguments checked;
 * the workspace is then left untouched).
 *
 *   x_bf16          [M][K] bf16
 *   qw_codes/scales the weight as written by rfq_quantize_weight for [N][K]
 *   y               [M][N] in y_type
 *   use_residual    1 = RFQ (both terms), 0 = plain MXFP4
 *   workspace       device buffer of at least rfq_linear_workspace_bytes(M, K,
 *                   use_residual) bytes, 256-byte aligned; its contents on
 *                   return are the quantized activation (unspecified layout)
 */
rfq_status_t rfq_linear(const void* x_bf16, int64_t M, int64_t K,
                        const void* qw_codes, const void* qw_scales, int64_t N,
                        void* y, rfq_out_t y_type, int use_residual,
                        void* workspace, size_t workspace_bytes,
                        cudaStream_t stream);

/*
 * Backward GEMMs of the layer Y = X W^T (straight-through: dL/dX ~ dL/dX^, dL/dW ~
 * dL/dW^).  The residual pathway stays on the activation-side operand of each
 * GEMM, as in the forward (section 1: activation quantization is the dominant
 * error; weights stay plain MXFP4).
 *
 * rfq_linear_dgrad -- dX [M][K] = (DQ(Q(dY)) [+ DQ(Q(R_dY))]) . DQ(Q(W^T))^T: the
 * contraction runs over N, so W enters as W^T quantized along N
 * (rfq_quantize_mxfp4_t of W [N][K], no residual: qwt_* with rows K, K-dimension
 * N).  This is rfq_linear with X := dY and the weight operand := W^T; arguments
 * and workspace (rfq_linear_workspace_bytes(M, N, use_residual)) as there.
 */
rfq_status_t rfq_linear_dgrad(const void* dy_bf16, int64_t M, int64_t N,
                              const void* qwt_codes, const void* qwt_scales, int64_t K,
                              void* dx, rfq_out_t dx_type, int use_residual,
                              void* workspace, size_t workspace_bytes,
                              cudaStream_t stream);

/* Workspace bytes of rfq_linear_wgrad: Q(X^T) [and Q(R^T)] [K][M] and Q(dY^T) [N][M],
 * each sub-buffer 256-byte aligned; 0 for unsupported shapes. */
size_t rfq_linear_wgrad_workspace_bytes(int64_t M, int64_t K, int64_t N, int use_residual);

/*
 * rfq_linear_wgrad -- dW [N][K] = sum over the M tokens of dY[m][n] . X^[m][k], with
 * both operands quantized along M (the contraction): X^T with the residual pathway
 * (the forward activation), dY^T plain.  Runs rfq_quantize_mxfp4_t on X and dY and
 * rfq_gemm_yt (A = X^T, B = dY^T, so the [K][N] product is written as [N][K]).
 *
 *   x_bf16 [M][K], dy_bf16 [M][N], bf16, 16-byte aligned; dw [N][K] in dw_type
 * M a multiple of 32, K a multiple of 32, N a multiple of 8.  M == 0 writes zeros.
 */
rfq_status_t rfq_linear_wgrad(const void* x_bf16, const void* dy_bf16, int64_t M, int64_t K, int64_t N,
                              void* dw, rfq_out_t dw_type, int use_residual,
                              void* workspace, size_t workspace_bytes,
                              cudaStream_t stream);

/* Largest M that rfq_linear_fused accepts (rfq_linear uses it for 1 <= M <= 32). */
#define RFQ_FUSED_MAX_M 64

/*
 * rfq_linear_fused -- the RFQ linear layer in one kernel for short batches
 * (M <= RFQ_FUSED_MAX_M): the quantizer runs inside the GEMM kernel, so Q(X)
 * and Q(R) exist only in shared memory (the residual is requantized inside the
 * GEMM, section 1).  Same codes, scales and accumulation as rfq_linear;
 * K is split across a cluster of CTAs per 128 columns of Y and the partial
 * sums are added in a fixed order, so Y differs from rfq_linear's only by fp32
 * summation order.  Needs no workspace.
 *
 *   x_bf16          [M][K] bf16, 16-byte aligned
 *   qw_codes/scales the weight as written by rfq_quantize_weight for [N][K]
 *   y               [M][N] in y_type, 16-byte aligned
 * K multiple of 32; N multiple of 8; M > RFQ_FUSED_MAX_M is
 * RFQ_ERR_UNSUPPORTED_SHAPE.  M == 0 or N == 0 launches nothing; K == 0 writes
 * zeros.
 */
rfq_status_t rfq_linear_fused(const void* x_bf16, int64_t M, int64_t K,
                              const void* qw_codes, const void* qw_scales, int64_t N,
                              void* y, rfq_out_t y_type, int use_residual,
                              cudaStream_t stream);

/*
 * Size of the fixed scratch array used by rfq_linear_static_workspace: 32 MiB of
 * device memory, reserved on every GPU that loads this library and kept until
 * the process exits.
 */
#define RFQ_STATIC_WORKSPACE_BYTES (32u << 20)

/*
 * rfq_linear_static_workspace -- rfq_linear without a caller-provided workspace
 * (the paper has no counterpart; this is a deployment convenience).
 *
 * For callers that cannot allocate device memory when they run the layer, e.g. a
 * plug-in inside a host application that owns the device's memory pool and
 * forbids raw cudaMalloc, or a latency-critical loop where allocating (which can
 * synchronize the device) is not allowed.  The quantized activation goes into a
 * fixed scratch array inside this library's own device memory instead; this
 * call allocates nothing.  Arguments, layouts and results are those of
 * rfq_linear; the caller still provides X, the quantized weight and Y.
 *
 *   - Size limit: rfq_linear_workspace_bytes(M, K, use_residual) must not exceed
 *     RFQ_STATIC_WORKSPACE_BYTES.  That workspace is 1.0625 bytes per element of X
 *     with the residual path (codes and scales of Q(X) and Q(R)) and half of that
 *     without, plus padding, so the limit is about M*K <= 30.1 Mi elements with the
 *     residual (e.g. 4096 x 7680) and 60.2 Mi without.  Larger problems return
 *     RFQ_ERR_UNSUPPORTED_SHAPE and launch nothing.  Bad arguments return the
 *     status rfq_linear returns for them.
 *   - Every call looks up the array's device address on the current device
 *     (nothing is cached).  On a device's first call that lookup can load this
 *     library's device code, so make the first call on each device before any
 *     stream capture on it.
 *   - Every call on a device shares the one array and it keeps the last call's
 *     contents.  Calls whose GPU work can overlap (different streams without
 *     ordering between them, or several host threads) race on it and corrupt
 *     each other's results; serialize them, e.g. on one stream.
 */
rfq_status_t rfq_linear_static_workspace(const void* x_bf16, int64_t M, int64_t K,
                                         const void* qw_codes, const void* qw_scales, int64_t N,
                                         void* y, rfq_out_t y_type, int use_residual,
                                         cudaStream_t stream);

/*
 * MXFP8 comparator path (OCP MX v1.0 MXFP8 with E4M3 elements; the paper reports
 * this format as nearly free of accuracy loss, abstract and section 1, first
 * contribution): a
 * reference point in accuracy and throughput for the 4-bit RFQ path.  No residual.
 *
 * rfq_mxfp8_codes_bytes -- rows * K (one E4M3 code byte per element); 0 for bad sizes.
 * Scales use rfq_scales_bytes(rows, K) and the same MMA layout as MXFP4.
 *
 * rfq_quantize_mxfp8 -- x [M][K] bf16 (16-byte aligned, K a multiple of 32) ->
 * codes [M][K] (element k in byte k) and E8M0 scales: exponent floor(log2 amax) - 8,
 * elements rounded to nearest even and saturated to +-448; 0xFF for a block with a
 * NaN or infinity.  Every byte of the scale array is written.
 *
 * rfq_gemm_mxfp8 -- Y = DQ(QX) . DQ(QW)^T on tcgen05 kind::mxf8f6f4 block-scaled
 * MMAs, fp32 accumulation; operands as written by rfq_quantize_mxfp8 ([M][K] and
 * [N][K]); y [M][N] fp32 or bf16, 16-byte aligned; N a multiple of 8.
 */
size_t rfq_mxfp8_codes_bytes(int64_t rows, int64_t K);
rfq_status_t rfq_quantize_mxfp8(const void* x_bf16, int64_t M, int64_t K,
                                void* q_codes, void* q_scales, cudaStream_t stream);
rfq_status_t rfq_gemm_mxfp8(const void* qx_codes, const void* qx_scales,
                            const void* qw_codes, const void* qw_scales,
                            int64_t M, int64_t N, int64_t K,
                            void* y, rfq_out_t y_type, cudaStream_t stream);

/*
 * rfq_mma_rate_probe -- measurement support (no counterpart in the paper): the rate
 * at which this GPU's tensor cores retire the MMA instructions rfq_gemm issues,
 * with the operands resident in shared memory (no loads, no epilogue).  It is the
 * ceiling against which the GEMM's tensor-pipe fraction is stated.
 *
 *   variant     0 = kind::mxf4 block-scaled (E2M1, E8M0 per 32), CTA pair, M 256 x N 256 x K 64
 *               1 = the same on single CTAs, M 128 x N 256 x K 64
 *               2 = kind::mxf8f6f4 block-scaled (E4M3), CTA pair, M 256 x N 256 x K 32
 *   iterations  1 .. RFQ_MMA_PROBE_MAX_ITERATIONS; each issues the 8 MMAs of one RFQ GEMM
 *               stage (4 on the activation tile, 4 on the residual tile, one weight tile)
 *   cycles      device buffer of at least cycles_len 8-byte words (8-byte aligned); word c
 *               receives cluster c's clock64 span from its first MMA to the completion of
 *               its last (SM clock cycles); words past the clusters launched are untouched
 *   cycles_len  at least SM count / 2 for variants 0 and 2, the SM count for variant 1
 *   flops       host pointer; receives the MMA flops the launch executes (2*M*N*K per MMA)
 *   sms_used    host pointer; receives the SMs the launch ran on: one CTA per SM, and only
 *               as many clusters as can be resident at once (on a GPU whose SM count does
 *               not split evenly into pairs, a few SMs stay idle)
 *
 * Time the launch with events on `stream`; flops / time is the rate of sms_used SMs, and
 * flops / (max cycles * sms_used) the rate per SM per clock.  The MMA results are not
 * meaningful and nothing but `cycles` is written.  Errors: RFQ_ERR_INVALID_ARG for a bad
 * variant, iteration count or pointer, RFQ_ERR_MISALIGNED, RFQ_ERR_UNSUPPORTED_DEVICE.
 */
#define RFQ_MMA_PROBE_MAX_ITERATIONS 100000
rfq_status_t rfq_mma_rate_probe(int variant, int64_t iterations, unsigned long long* cycles, int64_t cycles_len,
                                double* flops, int* sms_used, cudaStream_t stream);

/*
 * rfq_check_device_error -- synchronize `stream`, then read and clear the current
 * device's error word that bounded waits inside the kernels set.  Returns
 * RFQ_OK, RFQ_ERR_TIMEOUT (a wait ran out; the kernel wrote no complete result),
 * or RFQ_ERR_CUDA (the synchronization itself failed).  When detail is non-NULL
 * it receives the raw word (0 = none; 1..5 a wait inside rfq_gemm: 1 stage
 * load, 2 free stage, 3 accumulator ready, 4 accumulator free, 5 teardown;
 * 6 a wait of the quantizer for its TMA load; the same codes 1, 2, 3, 5 for
 * the corresponding waits of rfq_linear_fused, and 7 its quantizer warps
 * waiting for a staged tile of X).
 */
rfq_status_t rfq_check_device_error(cudaStream_t stream, int* detail);

/*
 * Testing hook for the bounded waits (no counterpart in the paper): the next
 * rfq_gemm launched by this process makes the producer of its first CTA skip
 * stage fill number `fill_index` (counted from 0 over that CTA's k-tiles), so
 * the MMA warp's wait for that stage runs out after about 1.5 s; the kernel then
 * drains its own copies and MMAs, frees its TMEM and returns, and
 * rfq_check_device_error() reports RFQ_ERR_TIMEOUT.  fill_index < 0 clears a
 * pending request.  Always returns RFQ_OK.
 */
rfq_status_t rfq_debug_skip_next_fill(int fill_index);

/*
 * Tuning hook: make rfq_linear_fused and the short-batch path of rfq_gemm split
 * K over `split` CTAs (1..8, capped at the number of 256-element k-tiles)
 * instead of choosing from the device's occupancy; 0 restores the automatic
 * choice.  Process-wide.
 */
rfq_status_t rfq_debug_fused_split(int split);

#ifdef __cplusplus
}
#endif

#endif /* RFQ_H_ */
