// rfq_quantize.cu -- kernel 1: the fused single-pass RFQ quantizer for sm_100a.
//
// "Activation Outliers Matter: Robust Recovery for Quantized Multimodal LLMs",
// section 1 (RFQ contribution paragraph): X is quantized to FP4 (here MXFP4), the
// full quantization error R = X - DQ(Q(X)) is formed, and R is quantized again by
// the same rule ("a second low-bit quantization path").  This kernel does all of
// it in one pass over X: every bf16 element is read from HBM exactly once and the
// codes and E8M0 scales of Q(X) and Q(R) are written once, the scales directly in
// the layout the block-scaled tensor-core MMA consumes.  R lives only in
// registers, in fp32, where it is exact.
//
// Work decomposition (HBM-bound streaming kernel, no tensor cores):
//   * X is viewed as a flat sequence of 32-element blocks (64 bytes each; a block
//     never crosses a row because K is a multiple of 32);
//   * a warp owns spans of 32 consecutive blocks (2 KiB) and each lane one block,
//     so the block amax needs no shuffles;
//   * every warp keeps kStages spans in flight with its own TMA ring (2-D tensor
//     map over [blocks][64 bytes], 64-byte swizzle so that the lanes' 16-byte
//     shared-memory reads are bank-conflict free) and mbarriers with bounded waits;
//   * pairs of fp32 values go through packed f32x2 multiplies / FMAs, codes
//     through cvt.rn.satfinite.e2m1x2.f32 (2 per instruction);
//   * scale bytes: when K is a multiple of 128 the 4 lanes holding blocks
//     4j..4j+3 of a row gather them into one 32-bit word of the MMA layout;
//     otherwise each lane stores its byte.  The padding bytes of the scale
//     arrays (rows up to a multiple of 128, blocks up to a multiple of 4) are
//     zeroed by the same launch.
#include <cuda.h>
#include <cuda_runtime.h>

#include <cstdint>

#include "rfq_internal.h"
#include "rfq_ptx.cuh"

namespace rfq {

__device__ unsigned int g_quant_error = 0;

namespace {

constexpr int kWarps = 8;
constexpr int kThreads = kWarps * 32;
constexpr int kStages = 4;
constexpr int kSpanBlocks = 32;                  // one block per lane
constexpr int kSpanBytes = kSpanBlocks * 64;     // 2 KiB
constexpr unsigned int kErrQuantWait = 6;        // a warp's wait for its TMA span ran out
constexpr uint32_t kSmemBytes = kWarps * kStages * kSpanBytes + kWarps * kStages * 8 + 1024;

struct QuantParams {
  uint8_t* qx_codes;
  uint8_t* qx_scales;
  uint8_t* qr_codes;
  uint8_t* qr_scales;
  int64_t M;             // rows
  int64_t Kb;            // 32-element blocks per row
  int64_t kb4_per_tile;  // 4-block words per row in the scale layout = ceil(Kb / 4)
  int64_t rows_pad;      // ceil(M / 128) * 128
  int64_t total_blocks;  // M * Kb
  int64_t num_spans;     // ceil(total_blocks / 32)
};

// ---------------------------------------------------------------- arithmetic helpers
__device__ __forceinline__ void mul2(float& o0, float& o1, float i0, float i1, float s) {
  asm("{\n\t.reg .b64 p, q, r;\n\t"
      "mov.b64 p, {%2, %3};\n\t"
      "mov.b64 q, {%4, %4};\n\t"
      "mul.rn.f32x2 r, p, q;\n\t"
      "mov.b64 {%0, %1}, r;\n\t}"
      : "=f"(o0), "=f"(o1)
      : "f"(i0), "f"(i1), "f"(s));
}

// (o0, o1) = (a0, a1) * s + (c0, c1), each rounded once.
__device__ __forceinline__ void fma2(float& o0, float& o1, float a0, float a1, float s, float c0, float c1) {
  asm("{\n\t.reg .b64 p, q, c, r;\n\t"
      "mov.b64 p, {%2, %3};\n\t"
      "mov.b64 q, {%4, %4};\n\t"
      "mov.b64 c, {%5, %6};\n\t"
      "fma.rn.f32x2 r, p, q, c;\n\t"
      "mov.b64 {%0, %1}, r;\n\t}"
      : "=f"(o0), "=f"(o1)
      : "f"(a0), "f"(a1), "f"(s), "f"(c0), "f"(c1));
}

// 8 fp32 values -> 8 E2M1 codes in one word (element i in bits 4i+3..4i), round
// to nearest even, saturating to +-6.
__device__ __forceinline__ uint32_t encode8(const float* v) {
  uint32_t out;
  asm("{\n\t.reg .b8 b0, b1, b2, b3;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b0, %2, %1;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b1, %4, %3;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b2, %6, %5;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b3, %8, %7;\n\t"
      "mov.b32 %0, {b0, b1, b2, b3};\n\t}"
      : "=r"(out)
      : "f"(v[0]), "f"(v[1]), "f"(v[2]), "f"(v[3]), "f"(v[4]), "f"(v[5]), "f"(v[6]), "f"(v[7]));
  return out;
}

__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t b, uint32_t sel) {
  uint32_t d;
  asm("prmt.b32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(sel));
  return d;
}

// One word of 8 E2M1 codes -> their exact values as fp32.  The magnitudes
// {0, .5, 1, 1.5, 2, 3, 4, 6} are bf16 0x0000, 0x3F00, 0x3F80, 0x3FC0, 0x4000,
// 0x4040, 0x4080, 0x40C0: two 8-entry byte tables (high and low bytes) indexed by
// the 3 magnitude bits of 4 codes at a time through byte permutes, then
// interleaved into bf16 pairs.  The sign of a code is the sign of the element it
// was encoded from, so it is copied from the input pair `xw[j]` (bf16 sign bits
// 15 and 31) instead of being decoded.
__device__ __forceinline__ void decode8(uint32_t cw, const uint32_t* xw, float* v) {
  const uint32_t mags = cw & 0x77777777u;
  const uint32_t sel_lo = mags & 0xffffu, sel_hi = mags >> 16;
  const uint32_t hi0 = prmt(0x3F3F3F00u, 0x40404040u, sel_lo), lo0 = prmt(0xC0800000u, 0xC0804000u, sel_lo);
  const uint32_t hi1 = prmt(0x3F3F3F00u, 0x40404040u, sel_hi), lo1 = prmt(0xC0800000u, 0xC0804000u, sel_hi);
  const uint32_t pr[4] = {prmt(lo0, hi0, 0x5140u), prmt(lo0, hi0, 0x7362u), prmt(lo1, hi1, 0x5140u),
                          prmt(lo1, hi1, 0x7362u)};
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const uint32_t bf2 = pr[j] | (xw[j] & 0x80008000u);
    v[2 * j] = __uint_as_float(bf2 << 16);
    v[2 * j + 1] = __uint_as_float(bf2 & 0xffff0000u);
  }
}

// Per half: max(|a|, |b|) (with the XOR of the signs as sign, cleared by the
// caller), NaN-propagating.
__device__ __forceinline__ uint32_t bmax2_abs(uint32_t a, uint32_t b) {
  uint32_t d;
  asm("max.NaN.xorsign.abs.bf16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
  return d;
}

// E8M0 byte from a biased exponent field: max(bexp - 2, 0) = clamp(floor(log2 amax)
// - 2, -127, 127) + 127; 0xFF (NaN) for a NaN/infinite amax.
__device__ __forceinline__ uint32_t scale_byte(uint32_t bexp) {
  return bexp == 0xFFu ? 0xFFu : (bexp >= 2u ? bexp - 2u : 0u);
}

// 2^(127 - s) and 2^(s - 127) as fp32 for a scale byte s in [0, 254].
__device__ __forceinline__ float inv_scale(uint32_t s) { return __uint_as_float((254u - s) << 23); }
__device__ __forceinline__ float scale_value(uint32_t s) {
  return s == 0u ? __uint_as_float(0x00400000u) : __uint_as_float(s << 23);
}

// Byte offset in the MMA scale layout of (row r, 4-block word kb4): atoms of 128
// rows x 4 blocks with the block-tile index fastest; row r inside its atom at
// (r % 32) * 16 + ((r / 32) % 4) * 4.
__device__ __forceinline__ int64_t scale_word_offset(int64_t r, int64_t kb4, int64_t kb4_per_tile) {
  return ((r >> 7) * kb4_per_tile + kb4) * 512 + (r & 31) * 16 + ((r >> 5) & 3) * 4;
}

// Store one block's scale byte: as a gathered 32-bit word of 4 lanes (word mode)
// or as a byte.  Called by all 32 lanes (the gather shuffles).
template <bool kWordScales>
__device__ __forceinline__ void store_scale(uint8_t* scales, uint32_t s, bool valid, int64_t row, int64_t kb,
                                            int64_t kb4_per_tile, int lane) {
  if constexpr (kWordScales) {
    const int base = lane & ~3;
    const uint32_t w = __shfl_sync(0xffffffffu, s, base) | (__shfl_sync(0xffffffffu, s, base + 1) << 8) |
                       (__shfl_sync(0xffffffffu, s, base + 2) << 16) | (__shfl_sync(0xffffffffu, s, base + 3) << 24);
    if (valid && (lane & 3) == 0) *reinterpret_cast<uint32_t*>(scales + scale_word_offset(row, kb >> 2, kb4_per_tile)) = w;
  } else {
    if (valid) scales[scale_word_offset(row, kb >> 2, kb4_per_tile) + (kb & 3)] = static_cast<uint8_t>(s);
  }
}

template <bool kResidual, bool kWordScales>
__global__ void __launch_bounds__(kThreads, 2)
    rfq_quantize_kernel(const __grid_constant__ CUtensorMap tm_x, const QuantParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  uint8_t* ring = smem + warp * (kStages * kSpanBytes);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kWarps * kStages * kSpanBytes) + warp * kStages;
  volatile int abort_flag = 0;   // per warp: each warp's ring is independent

  const int64_t gw = static_cast<int64_t>(blockIdx.x) * kWarps + warp;
  const int64_t GW = static_cast<int64_t>(gridDim.x) * kWarps;
  const int64_t n_my = p.num_spans > gw ? (p.num_spans - gw + GW - 1) / GW : 0;

  if (lane == 0) {
    for (int s = 0; s < kStages; ++s) mbar_init(&bars[s], 1);
    fence_mbar_init();
    for (int s = 0; s < kStages && s < n_my; ++s) {
      mbar_arrive_expect_tx(&bars[s], kSpanBytes);
      tma_load_2d(ring + s * kSpanBytes, &tm_x, &bars[s], 0, static_cast<int>((gw + s * GW) * kSpanBlocks));
    }
  }
  __syncwarp();

  // Block coordinates of lane 0's block, advanced incrementally span by span.
  const int64_t stride_blocks = GW * kSpanBlocks;
  const int64_t d_row = stride_blocks / p.Kb, d_kb = stride_blocks - (stride_blocks / p.Kb) * p.Kb;
  int64_t row0 = (gw * kSpanBlocks) / p.Kb;
  int64_t kb0 = gw * kSpanBlocks - row0 * p.Kb;
  const int swz = (lane >> 1) & 3;   // 64-byte swizzle of this lane's row in the span

  int64_t i = 0;
  for (; i < n_my; ++i) {
    const int s = static_cast<int>(i % kStages);
    const bool ok = mbar_wait(&bars[s], static_cast<uint32_t>((i / kStages) & 1), &abort_flag, &g_quant_error,
                              kErrQuantWait);
    if (!__all_sync(0xffffffffu, ok)) break;   // every lane returns from its bounded wait: a uniform decision
    const int64_t gb = (gw + i * GW) * kSpanBlocks + lane;
    const bool valid = gb < p.total_blocks;
    // lane's block: row, block-in-row
    int64_t row, kb;
    {
      const int64_t t = kb0 + lane;
      int64_t q;
      if (p.Kb >= kSpanBlocks) q = t >= p.Kb ? 1 : 0;
      else q = static_cast<int64_t>(static_cast<uint32_t>(t) / static_cast<uint32_t>(p.Kb));
      row = row0 + q;
      kb = t - q * p.Kb;
    }

    uint32_t w[16];
    const uint8_t* src = ring + s * kSpanBytes + lane * 64;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const uint4 c = *reinterpret_cast<const uint4*>(src + ((j ^ swz) << 4));
      w[4 * j + 0] = c.x;
      w[4 * j + 1] = c.y;
      w[4 * j + 2] = c.z;
      w[4 * j + 3] = c.w;
    }
    __syncwarp();
    // This lane's data are now in registers: refill the stage with the span
    // kStages ahead (the reads above are ordered before the async-proxy write).
    if (lane == 0 && i + kStages < n_my) {
      asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
      mbar_arrive_expect_tx(&bars[s], kSpanBytes);
      tma_load_2d(ring + s * kSpanBytes, &tm_x, &bars[s], 0,
                  static_cast<int>((gw + (i + kStages) * GW) * kSpanBlocks));
    }

    // ---- Q(X): block amax on bf16 magnitudes (NaN-propagating), E8M0 byte
    uint32_t m[8];
#pragma unroll
    for (int k = 0; k < 8; ++k) m[k] = bmax2_abs(w[2 * k], w[2 * k + 1]);
#pragma unroll
    for (int k = 0; k < 4; ++k) m[k] = bmax2_abs(m[k], m[k + 4]);
    m[0] = bmax2_abs(bmax2_abs(m[0], m[2]), bmax2_abs(m[1], m[3])) & 0x7fff7fffu;
    const uint32_t amax = max(m[0] & 0xffffu, m[0] >> 16);
    const uint32_t sx = scale_byte(amax >> 7);
    const uint32_t sx_eff = sx == 0xFFu ? 127u : sx;   // codes of a non-finite block are unspecified
    const float inv_x = inv_scale(sx_eff);
    const float neg_sc = -scale_value(sx_eff);

    // Per group of 8 elements: unpack bf16 -> fp32, scale (exact), encode; then
    // decode and form the residual R = X - DQ(Q(X)) in fp32 (exact).
    uint32_t cx[4];
    float r[32];
    float ra = 0.0f, rb = 0.0f;
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      float xv[8], v[8];
#pragma unroll
      for (int h = 0; h < 4; ++h) {
        xv[2 * h] = __uint_as_float(w[4 * k + h] << 16);
        xv[2 * h + 1] = __uint_as_float(w[4 * k + h] & 0xffff0000u);
        mul2(v[2 * h], v[2 * h + 1], xv[2 * h], xv[2 * h + 1], inv_x);
      }
      cx[k] = encode8(v);
      if constexpr (kResidual) {
        float dq[8];
        decode8(cx[k], w + 4 * k, dq);
#pragma unroll
        for (int h = 0; h < 4; ++h) {
          const int e = 8 * k + 2 * h;
          fma2(r[e], r[e + 1], dq[2 * h], dq[2 * h + 1], neg_sc, xv[2 * h], xv[2 * h + 1]);
          ra = fmaxf(ra, fabsf(r[e]));
          rb = fmaxf(rb, fabsf(r[e + 1]));
        }
      }
    }
    if (valid) *reinterpret_cast<uint4*>(p.qx_codes + gb * 16) = make_uint4(cx[0], cx[1], cx[2], cx[3]);
    store_scale<kWordScales>(p.qx_scales, sx, valid, row, kb, p.kb4_per_tile, lane);

    if constexpr (kResidual) {
      // ---- Q(R) by the same rule
      uint32_t sr = scale_byte(__float_as_uint(fmaxf(ra, rb)) >> 23);
      if (sx == 0xFFu) sr = 0xFFu;
      const float inv_r = inv_scale(sr == 0xFFu ? 127u : sr);
      uint32_t cr[4];
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        float v[8];
#pragma unroll
        for (int h = 0; h < 4; ++h) mul2(v[2 * h], v[2 * h + 1], r[8 * k + 2 * h], r[8 * k + 2 * h + 1], inv_r);
        cr[k] = encode8(v);
      }
      if (valid) *reinterpret_cast<uint4*>(p.qr_codes + gb * 16) = make_uint4(cr[0], cr[1], cr[2], cr[3]);
      store_scale<kWordScales>(p.qr_scales, sr, valid, row, kb, p.kb4_per_tile, lane);
    }

    kb0 += d_kb;
    row0 += d_row;
    if (kb0 >= p.Kb) {
      kb0 -= p.Kb;
      row0 += 1;
    }
  }

  if (i < n_my && lane == 0) {
    // A wait ran out: let this warp's outstanding copies land before leaving.
    int never = 0;
    for (int64_t k = i; k < n_my && k < i + kStages; ++k)
      mbar_wait(&bars[k % kStages], static_cast<uint32_t>((k / kStages) & 1), &never, &g_quant_error, kErrQuantWait);
  }

  // ---- zero padding of the scale arrays: rows [M, rows_pad) and blocks [Kb, 4*kb4) of real rows
  const int64_t tid = static_cast<int64_t>(blockIdx.x) * kThreads + threadIdx.x;
  const int64_t nthreads = static_cast<int64_t>(gridDim.x) * kThreads;
  const int64_t pad_rows = p.rows_pad - p.M;
  const int64_t pad_words = pad_rows * p.kb4_per_tile;
  for (int64_t t = tid; t < pad_words; t += nthreads) {
    const int64_t r = p.M + t / p.kb4_per_tile, kb4 = t % p.kb4_per_tile;
    const int64_t off = scale_word_offset(r, kb4, p.kb4_per_tile);
    *reinterpret_cast<uint32_t*>(p.qx_scales + off) = 0u;
    if (kResidual) *reinterpret_cast<uint32_t*>(p.qr_scales + off) = 0u;
  }
  const int64_t tail = p.kb4_per_tile * 4 - p.Kb;   // 0..3 pad blocks per real row
  if (tail > 0) {
    for (int64_t t = tid; t < p.M * tail; t += nthreads) {
      const int64_t r = t / tail, kb = p.Kb + t % tail;
      const int64_t off = scale_word_offset(r, kb >> 2, p.kb4_per_tile) + (kb & 3);
      p.qx_scales[off] = 0;
      if (kResidual) p.qr_scales[off] = 0;
    }
  }
}

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

template <bool kResidual, bool kWord>
cudaError_t launch_typed(const CUtensorMap& tm, const QuantParams& p, int grid, cudaStream_t stream) {
  auto kernel = rfq_quantize_kernel<kResidual, kWord>;
  cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
  if (e != cudaSuccess) return e;
  kernel<<<grid, kThreads, kSmemBytes, stream>>>(tm, p);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_quantize(const void* x, int64_t M, int64_t K, void* qx_codes, void* qx_scales, void* qr_codes,
                            void* qr_scales, int num_sms, void* encode_tiled, cudaStream_t stream) {
  QuantParams p;
  p.qx_codes = static_cast<uint8_t*>(qx_codes);
  p.qx_scales = static_cast<uint8_t*>(qx_scales);
  p.qr_codes = static_cast<uint8_t*>(qr_codes);
  p.qr_scales = static_cast<uint8_t*>(qr_scales);
  p.M = M;
  p.Kb = K / 32;
  p.kb4_per_tile = (p.Kb + 3) / 4;
  p.rows_pad = (M + 127) / 128 * 128;
  p.total_blocks = M * p.Kb;
  p.num_spans = (p.total_blocks + kSpanBlocks - 1) / kSpanBlocks;

  // X as [total_blocks][64 bytes]; 32-row boxes, 64-byte swizzle, zero fill past the end.
  CUtensorMap tm;
  cuuint64_t dims[2] = {64, static_cast<cuuint64_t>(p.total_blocks)};
  cuuint64_t strides[1] = {64};
  cuuint32_t box[2] = {64, static_cast<cuuint32_t>(kSpanBlocks)};
  cuuint32_t elem_strides[2] = {1, 1};
  EncodeTiledFn encode = reinterpret_cast<EncodeTiledFn>(encode_tiled);
  if (encode(&tm, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(x), dims, strides, box, elem_strides,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_64B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
    return cudaErrorInvalidValue;

  const int64_t warps_needed = p.num_spans;
  int64_t grid = (warps_needed + kWarps - 1) / kWarps;
  const int64_t cap = static_cast<int64_t>(num_sms) * 2;
  if (grid > cap) grid = cap;
  if (grid < 1) grid = 1;
  const bool word = (p.Kb % 4) == 0;
  if (qr_codes) {
    return word ? launch_typed<true, true>(tm, p, static_cast<int>(grid), stream)
                : launch_typed<true, false>(tm, p, static_cast<int>(grid), stream);
  }
  return word ? launch_typed<false, true>(tm, p, static_cast<int>(grid), stream)
              : launch_typed<false, false>(tm, p, static_cast<int>(grid), stream);
}

cudaError_t read_and_clear_quant_error(unsigned int* value) {
  unsigned int zero = 0;
  cudaError_t e = cudaMemcpyFromSymbol(value, g_quant_error, sizeof(unsigned int));
  if (e != cudaSuccess) return e;
  return cudaMemcpyToSymbol(g_quant_error, &zero, sizeof(unsigned int));
}

}  // namespace rfq
