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
//   chunk  = 8 consecutive elements of one row (one 16-byte load per thread);
//   block  = 32 elements = 4 consecutive lanes; the block amax is a two-step
//            xor-shuffle reduction inside those 4 lanes;
//   a half-warp = 16 chunks = 4 blocks = one 4-byte word of the scale layout.
// The matrix is walked as [rows_pad][K_pad] with rows_pad = ceil(M/128)*128 and
// K_pad = ceil(K/128)*128, so the same pass also writes the zero padding bytes of
// the scale arrays (an all-zero block gets scale byte 0); codes are stored only
// inside [M][K].  Each thread keeps kUnroll independent 16-byte loads in flight.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cstdint>

#include "rfq_internal.h"
#include "rfq_ptx.cuh"

namespace rfq {

namespace {

constexpr int kThreads = 256;
constexpr int kUnroll = 4;

// 8 fp32 values -> 8 E2M1 codes in one word (element i in bits 4i+3..4i).
__device__ __forceinline__ uint32_t encode8(const float (&v)[8]) {
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

// One word of 8 E2M1 codes -> their values (exact: +-0, .5, 1, 1.5, 2, 3, 4, 6) as
// fp32, built from the code's fields: magnitude 0 -> 0, 1 -> 0.5, and for
// 2..7 (exponent E = mag >> 1 >= 1, mantissa m = mag & 1) 2^(E-1) * (1 + m/2),
// whose fp32 pattern is (mag + 252) << 22; bit 3 is the sign.
__device__ __forceinline__ void decode8(uint32_t w, float (&v)[8]) {
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const uint32_t c = (w >> (4 * i)) & 0xFu;
    const uint32_t mag = c & 7u;
    uint32_t bits = (mag + 252u) << 22;
    bits = (mag == 1u) ? 0x3F000000u : bits;
    bits = (mag == 0u) ? 0u : bits;
    v[i] = __uint_as_float(bits | ((c & 8u) << 28));
  }
}

// E8M0 byte of a block from the bit pattern of its amax, given the position of
// the exponent field: max(biased_exponent - 2, 0) = clamp(floor(log2 amax) - 2,
// -127, 127) + 127, and 0xFF for a NaN/infinite amax.
template <int kMantBits, uint32_t kExpMask>
__device__ __forceinline__ uint32_t scale_byte_from_amax_bits(uint32_t amax_bits) {
  const uint32_t bexp = (amax_bits >> kMantBits) & kExpMask;
  if (bexp == kExpMask) return 0xFFu;
  return bexp >= 2u ? bexp - 2u : 0u;
}

// 2^(127 - s) and 2^(s - 127) as fp32 for a scale byte s in [0, 254].
__device__ __forceinline__ float inv_scale(uint32_t s) { return __uint_as_float((254u - s) << 23); }
__device__ __forceinline__ float scale_value(uint32_t s) {
  return s == 0u ? __uint_as_float(0x00400000u) : __uint_as_float(s << 23);
}

// Gather the scale bytes of the 4 blocks of this half-warp into one word (block
// j in byte j) and return it; valid in every lane.
__device__ __forceinline__ uint32_t gather_scale_word(uint32_t s) {
  const int base = threadIdx.x & 16;
  const uint32_t b0 = __shfl_sync(0xffffffffu, s, base + 0);
  const uint32_t b1 = __shfl_sync(0xffffffffu, s, base + 4);
  const uint32_t b2 = __shfl_sync(0xffffffffu, s, base + 8);
  const uint32_t b3 = __shfl_sync(0xffffffffu, s, base + 12);
  return b0 | (b1 << 8) | (b2 << 16) | (b3 << 24);
}

// Byte offset, in the MMA scale layout, of the word holding blocks 4*kb4..4*kb4+3
// of row r (atoms of 128 rows x 4 blocks, block-tile index fastest; inside an
// atom row r sits at (r%32)*16 + ((r/32)%4)*4).
__device__ __forceinline__ int64_t scale_word_offset(int64_t r, int64_t kb4, int64_t atoms_per_row_tile) {
  return ((r >> 7) * atoms_per_row_tile + kb4) * 512 + (r & 31) * 16 + ((r >> 5) & 3) * 4;
}

template <bool kResidual>
__global__ void __launch_bounds__(kThreads) rfq_quantize_kernel(const uint4* __restrict__ x, int64_t M, int64_t K,
                                                                int64_t total_chunks, int64_t chunks_per_row_pad,
                                                                uint32_t* __restrict__ qx_codes,
                                                                uint8_t* __restrict__ qx_scales,
                                                                uint32_t* __restrict__ qr_codes,
                                                                uint8_t* __restrict__ qr_scales) {
  const int64_t chunks_per_row = K >> 3;                       // 8 elements per chunk
  const int64_t atoms_per_row_tile = chunks_per_row_pad >> 4;  // 16 chunks (128 elements) per atom column
  const int64_t span = static_cast<int64_t>(kThreads) * kUnroll;

  for (int64_t base = static_cast<int64_t>(blockIdx.x) * span; base < total_chunks;
       base += static_cast<int64_t>(gridDim.x) * span) {
    uint4 raw[kUnroll];
    int64_t row[kUnroll], cc[kUnroll];
    bool inside[kUnroll];
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
      const int64_t g = base + u * kThreads + threadIdx.x;
      row[u] = g / chunks_per_row_pad;
      cc[u] = g - row[u] * chunks_per_row_pad;
      inside[u] = (g < total_chunks) && (row[u] < M) && (cc[u] < chunks_per_row);
      raw[u] = inside[u] ? __ldcs(x + row[u] * chunks_per_row + cc[u]) : make_uint4(0u, 0u, 0u, 0u);
    }
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
      const int64_t g = base + u * kThreads + threadIdx.x;
      const uint32_t w[4] = {raw[u].x, raw[u].y, raw[u].z, raw[u].w};

      // --- Q(X): block amax on the bf16 magnitude bits (monotone in |x|; NaN > inf > finite)
      uint32_t m2 = __vmaxu2(__vmaxu2(w[0] & 0x7fff7fffu, w[1] & 0x7fff7fffu),
                             __vmaxu2(w[2] & 0x7fff7fffu, w[3] & 0x7fff7fffu));
      uint32_t amax = max(m2 & 0xffffu, m2 >> 16);
      amax = max(amax, __shfl_xor_sync(0xffffffffu, amax, 1));
      amax = max(amax, __shfl_xor_sync(0xffffffffu, amax, 2));
      const uint32_t sx = scale_byte_from_amax_bits<7, 0xffu>(amax);
      const uint32_t sx_eff = sx == 0xFFu ? 127u : sx;   // codes of a non-finite block are unspecified
      const float inv_x = inv_scale(sx_eff);

      float xv[8], v[8];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        xv[2 * i] = __uint_as_float(w[i] << 16);
        xv[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
      }
#pragma unroll
      for (int i = 0; i < 8; ++i) v[i] = xv[i] * inv_x;  // exact: a power-of-two scaling, |v| < 8
      const uint32_t cx = encode8(v);

      const uint32_t wx = gather_scale_word(sx);
      if (g < total_chunks) {
        if (inside[u]) qx_codes[row[u] * chunks_per_row + cc[u]] = cx;
        if ((threadIdx.x & 15) == 0)
          *reinterpret_cast<uint32_t*>(qx_scales + scale_word_offset(row[u], cc[u] >> 4, atoms_per_row_tile)) = wx;
      }

      if constexpr (kResidual) {
        // --- R = X - DQ(Q(X)) in fp32 (exact: |r| < 2^(e+1) on a 2^(e-9) grid)
        float dq[8], r[8];
        decode8(cx, dq);
        const float sc = scale_value(sx_eff);
        uint32_t ramax = 0u;
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          r[i] = __fmaf_rn(-dq[i], sc, xv[i]);
          ramax = max(ramax, __float_as_uint(r[i]) & 0x7fffffffu);
        }
        ramax = max(ramax, __shfl_xor_sync(0xffffffffu, ramax, 1));
        ramax = max(ramax, __shfl_xor_sync(0xffffffffu, ramax, 2));
        uint32_t sr = scale_byte_from_amax_bits<23, 0xffu>(ramax);
        if (sx == 0xFFu) sr = 0xFFu;
        const float inv_r = inv_scale(sr == 0xFFu ? 127u : sr);
#pragma unroll
        for (int i = 0; i < 8; ++i) v[i] = r[i] * inv_r;
        const uint32_t cr = encode8(v);
        const uint32_t wr = gather_scale_word(sr);
        if (g < total_chunks) {
          if (inside[u]) qr_codes[row[u] * chunks_per_row + cc[u]] = cr;
          if ((threadIdx.x & 15) == 0)
            *reinterpret_cast<uint32_t*>(qr_scales + scale_word_offset(row[u], cc[u] >> 4, atoms_per_row_tile)) = wr;
        }
      }
    }
  }
}

}  // namespace

cudaError_t launch_quantize(const void* x, int64_t M, int64_t K, void* qx_codes, void* qx_scales, void* qr_codes,
                            void* qr_scales, int num_sms, cudaStream_t stream) {
  const int64_t rows_pad = (M + 127) / 128 * 128;
  const int64_t k_pad = (K + 127) / 128 * 128;
  const int64_t chunks_per_row_pad = k_pad / 8;
  const int64_t total = rows_pad * chunks_per_row_pad;
  const int64_t span = static_cast<int64_t>(kThreads) * kUnroll;
  int64_t blocks = (total + span - 1) / span;
  const int64_t cap = static_cast<int64_t>(num_sms) * 8;
  if (blocks > cap) blocks = cap;
  if (blocks < 1) blocks = 1;
  if (qr_codes) {
    rfq_quantize_kernel<true><<<static_cast<unsigned>(blocks), kThreads, 0, stream>>>(
        static_cast<const uint4*>(x), M, K, total, chunks_per_row_pad, static_cast<uint32_t*>(qx_codes),
        static_cast<uint8_t*>(qx_scales), static_cast<uint32_t*>(qr_codes), static_cast<uint8_t*>(qr_scales));
  } else {
    rfq_quantize_kernel<false><<<static_cast<unsigned>(blocks), kThreads, 0, stream>>>(
        static_cast<const uint4*>(x), M, K, total, chunks_per_row_pad, static_cast<uint32_t*>(qx_codes),
        static_cast<uint8_t*>(qx_scales), nullptr, nullptr);
  }
  return cudaGetLastError();
}

}  // namespace rfq
