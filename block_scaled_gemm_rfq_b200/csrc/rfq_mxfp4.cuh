// rfq_mxfp4.cuh -- per-block MXFP4 / RFQ arithmetic shared by the stand-alone
// quantizer (rfq_quantize.cu) and the fused quantize-and-multiply kernel
// (rfq_linear_fused.cu).
//
// "Activation Outliers Matter: Robust Recovery for Quantized Multimodal LLMs",
// section 1 (RFQ contribution paragraph): a 32-element block of X gets an E8M0
// scale and E2M1 codes (OCP MX v1.0, section 6.3: scale exponent
// floor(log2 amax) - emax_elem, emax_elem = 2 for E2M1; elements X / scale rounded
// to nearest even, saturating to +-6); the residual R = X - DQ(Q(X)) is formed
// exactly (in bf16 pairs, see quantize_block) and quantized by the same rule.
#pragma once

#include <cstdint>

namespace rfq {

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

// bf16 pair word -> the two fp32 values (element 2j from the low half; exact).
__device__ __forceinline__ void unpack_bf16x2(uint32_t w, float& lo, float& hi) {
  lo = __uint_as_float(w << 16);
  hi = __uint_as_float(w & 0xffff0000u);
}

// One word of 8 E2M1 codes -> their exact values as 4 bf16 pairs (element 2j in
// the low half of word j).  The magnitudes {0, .5, 1, 1.5, 2, 3, 4, 6} are bf16
// 0x0000, 0x3F00, 0x3F80, 0x3FC0, 0x4000, 0x4040, 0x4080, 0x40C0: two 8-entry
// byte tables (high and low bytes) indexed by the 3 magnitude bits of 4 codes at
// a time through byte permutes, then interleaved into pairs.  The sign of a code
// is the sign of the element it was encoded from, so it is copied from the input
// pair `xw[j]` (bf16 sign bits 15 and 31) instead of being decoded.
__device__ __forceinline__ void decode8(uint32_t cw, const uint32_t* xw, uint32_t* out) {
  const uint32_t mags = cw & 0x77777777u;
  const uint32_t sel_lo = mags & 0xffffu, sel_hi = mags >> 16;
  const uint32_t hi0 = prmt(0x3F3F3F00u, 0x40404040u, sel_lo), lo0 = prmt(0xC0800000u, 0xC0804000u, sel_lo);
  const uint32_t hi1 = prmt(0x3F3F3F00u, 0x40404040u, sel_hi), lo1 = prmt(0xC0800000u, 0xC0804000u, sel_hi);
  out[0] = prmt(lo0, hi0, 0x5140u) | (xw[0] & 0x80008000u);
  out[1] = prmt(lo0, hi0, 0x7362u) | (xw[1] & 0x80008000u);
  out[2] = prmt(lo1, hi1, 0x5140u) | (xw[2] & 0x80008000u);
  out[3] = prmt(lo1, hi1, 0x7362u) | (xw[3] & 0x80008000u);
}

// a * b + c on bf16 pairs with one rounding (exact when the result is a bf16 value).
__device__ __forceinline__ uint32_t bfma2(uint32_t a, uint32_t b, uint32_t c) {
  uint32_t d;
  asm("fma.rn.bf16x2 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(c));
  return d;
}

// Per half: max(|a|, |b|) (with the XOR of the signs as sign, cleared by the
// caller), NaN-propagating.
__device__ __forceinline__ uint32_t bmax2_abs(uint32_t a, uint32_t b) {
  uint32_t d;
  asm("max.NaN.xorsign.abs.bf16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
  return d;
}

// bf16 bits of the largest magnitude among 32 bf16 values (16 pair words);
// NaN-propagating.
__device__ __forceinline__ uint32_t block_amax_bits(const uint32_t (&w)[16]) {
  uint32_t m[8];
#pragma unroll
  for (int k = 0; k < 8; ++k) m[k] = bmax2_abs(w[2 * k], w[2 * k + 1]);
#pragma unroll
  for (int k = 0; k < 4; ++k) m[k] = bmax2_abs(m[k], m[k + 4]);
  m[0] = bmax2_abs(bmax2_abs(m[0], m[2]), bmax2_abs(m[1], m[3])) & 0x7fff7fffu;
  return max(m[0] & 0xffffu, m[0] >> 16);
}

// E8M0 byte from a biased exponent field: max(bexp - 2, 0) = clamp(floor(log2 amax)
// - 2, -127, 127) + 127; 0xFF (NaN) for a NaN/infinite amax.
__device__ __forceinline__ uint32_t scale_byte(uint32_t bexp) {
  return bexp == 0xFFu ? 0xFFu : (bexp >= 2u ? bexp - 2u : 0u);
}

// 2^(127 - s) as fp32 for a scale byte s in [0, 254].
__device__ __forceinline__ float inv_scale(uint32_t s) { return __uint_as_float((254u - s) << 23); }

// Quantize one 32-element bf16 block (16 words, element 2i in the low half of
// word i).  Outputs the E2M1 codes of Q(X) (4 words, element i in bits
// 4(i%8)+3..4(i%8) of word i/8) and its E8M0 byte, and, with kResidual, the codes
// and byte of Q(R), R = X - DQ(Q(X)).  A non-finite block gets scale byte 0xFF
// for both terms (its codes are unspecified).
//
// R is formed in bf16 pairs, exactly: with x an element (exponent e, so a
// multiple of its bf16 ulp 2^(e-7)) and s the block's scale exponent (s >=
// e - 2), DQ(Q(x)) is a multiple of 2^(s-1), hence of ulp(x), and the nearest
// grid point is no farther from x than 0 is, so |x - DQ| <= |x|.  x - DQ is thus
// a multiple of ulp(x) below 2^(e+1): a bf16 value, which one bf16 FMA returns
// unrounded (saturated elements, |x| < 8 * 2^s against 6 * 2^s, too).
template <bool kResidual>
__device__ __forceinline__ void quantize_block(const uint32_t (&w)[16], uint32_t (&cx)[4], uint32_t& sx_out,
                                               uint32_t (&cr)[4], uint32_t& sr_out) {
  // ---- Q(X): block amax on bf16 magnitudes (NaN-propagating), E8M0 byte
  const uint32_t sx = scale_byte(block_amax_bits(w) >> 7);
  const uint32_t sx_eff = sx == 0xFFu ? 127u : sx;   // codes of a non-finite block are unspecified
  const float inv_x = inv_scale(sx_eff);
  // -2^(sx-127) as a bf16 pair (byte 0: -2^-127, a bf16 subnormal)
  const uint32_t neg_sc = sx_eff == 0u ? 0x8040u : (0x8000u | (sx_eff << 7));
  const uint32_t neg_sc2 = neg_sc | (neg_sc << 16);

  // Per group of 8 elements: unpack bf16 -> fp32, scale (exact), encode; then
  // decode and form the residual pairs.
  uint32_t r2[16];
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    float v[8];
#pragma unroll
    for (int h = 0; h < 4; ++h) {
      float x0, x1;
      unpack_bf16x2(w[4 * k + h], x0, x1);
      mul2(v[2 * h], v[2 * h + 1], x0, x1, inv_x);
    }
    cx[k] = encode8(v);
    if constexpr (kResidual) {
      uint32_t dq[4];
      decode8(cx[k], w + 4 * k, dq);
#pragma unroll
      for (int h = 0; h < 4; ++h) r2[4 * k + h] = bfma2(dq[h], neg_sc2, w[4 * k + h]);
    }
  }
  sx_out = sx;

  if constexpr (kResidual) {
    // ---- Q(R) by the same rule
    uint32_t sr = scale_byte(block_amax_bits(r2) >> 7);
    if (sx == 0xFFu) sr = 0xFFu;
    const float inv_r = inv_scale(sr == 0xFFu ? 127u : sr);
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      float v[8];
#pragma unroll
      for (int h = 0; h < 4; ++h) {
        float r0, r1;
        unpack_bf16x2(r2[4 * k + h], r0, r1);
        mul2(v[2 * h], v[2 * h + 1], r0, r1, inv_r);
      }
      cr[k] = encode8(v);
    }
    sr_out = sr;
  }
}

// ---------------------------------------------------------------- MXFP8 (comparator)
// OCP MX v1.0 MXFP8 with E4M3 elements: E8M0 exponent floor(log2 amax) - 8 (8 = the
// E4M3 largest exponent; 448 = 1.75 * 2^8), elements rounded to nearest even and
// saturated to +-448.  The paper finds this format nearly free of accuracy loss (abstract;
// section 1, first contribution).

// 4 fp32 values -> 4 E4M3 codes in one word (element i in byte i).
__device__ __forceinline__ uint32_t encode4_e4m3(float a0, float a1, float a2, float a3) {
  uint32_t out;
  asm("{\n\t.reg .b16 h0, h1;\n\t"
      "cvt.rn.satfinite.e4m3x2.f32 h0, %2, %1;\n\t"
      "cvt.rn.satfinite.e4m3x2.f32 h1, %4, %3;\n\t"
      "mov.b32 %0, {h0, h1};\n\t}"
      : "=r"(out)
      : "f"(a0), "f"(a1), "f"(a2), "f"(a3));
  return out;
}

// MXFP8 quantization of one 32-element bf16 block: 8 words of E4M3 codes
// (element i in byte i%4 of word i/4) and the E8M0 byte (0xFF for a non-finite
// block, whose codes are unspecified).  x * 2^-e is exact in fp32 (or below
// E4M3's resolution, where it encodes to 0 either way).
__device__ __forceinline__ void quantize_block_e4m3(const uint32_t (&w)[16], uint32_t (&codes)[8], uint32_t& s_out) {
  const uint32_t bexp = block_amax_bits(w) >> 7;
  const uint32_t s = bexp == 0xFFu ? 0xFFu : (bexp >= 8u ? bexp - 8u : 0u);
  const float inv = inv_scale(s == 0xFFu ? 127u : s);
#pragma unroll
  for (int k = 0; k < 8; ++k) {
    float x0, x1, x2, x3, v0, v1, v2, v3;
    unpack_bf16x2(w[2 * k], x0, x1);
    unpack_bf16x2(w[2 * k + 1], x2, x3);
    mul2(v0, v1, x0, x1, inv);
    mul2(v2, v3, x2, x3, inv);
    codes[k] = encode4_e4m3(v0, v1, v2, v3);
  }
  s_out = s;
}

}  // namespace rfq
