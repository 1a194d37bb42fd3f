// rfq_mxfp4.cuh -- per-block MXFP4 / RFQ arithmetic shared by the stand-alone
// quantizer (rfq_quantize.cu) and the fused quantize-and-multiply kernel
// (rfq_linear_fused.cu).
//
// "Activation Outliers Matter: Robust Recovery for Quantized Multimodal LLMs",
// section 1 (RFQ contribution paragraph): a 32-element block of X gets an E8M0
// scale and E2M1 codes (OCP MX v1.0, section 6.3: scale exponent
// floor(log2 amax) - emax_elem, emax_elem = 2 for E2M1; elements X / scale rounded
// to nearest even, saturating to +-6); the residual R = X - DQ(Q(X)) is formed
// exactly (in fp32, see quantize_block) and quantized by the same rule.
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

// a * b + c on fp32 pairs (b shared by both), one rounding each.
__device__ __forceinline__ void fma2(float& o0, float& o1, float a0, float a1, float b, float c0, float c1) {
  asm("{\n\t.reg .b64 p, q, c, r;\n\t"
      "mov.b64 p, {%2, %3};\n\t"
      "mov.b64 q, {%4, %4};\n\t"
      "mov.b64 c, {%5, %6};\n\t"
      "fma.rn.f32x2 r, p, q, c;\n\t"
      "mov.b64 {%0, %1}, r;\n\t}"
      : "=f"(o0), "=f"(o1)
      : "f"(a0), "f"(a1), "f"(b), "f"(c0), "f"(c1));
}

// encode8, also returning the grid values the codes stand for (signed, exact) as
// fp32: each code byte is decoded back by the hardware E2M1x2 -> f16x2
// conversion (element 2j in the low half) and widened to fp32.
__device__ __forceinline__ uint32_t encode8_dq(const float* v, float* q) {
  uint32_t out, h[4];
  asm("{\n\t.reg .b8 b0, b1, b2, b3;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b0, %6, %5;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b1, %8, %7;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b2, %10, %9;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b3, %12, %11;\n\t"
      "mov.b32 %0, {b0, b1, b2, b3};\n\t"
      "cvt.rn.f16x2.e2m1x2 %1, b0;\n\t"
      "cvt.rn.f16x2.e2m1x2 %2, b1;\n\t"
      "cvt.rn.f16x2.e2m1x2 %3, b2;\n\t"
      "cvt.rn.f16x2.e2m1x2 %4, b3;\n\t}"
      : "=r"(out), "=r"(h[0]), "=r"(h[1]), "=r"(h[2]), "=r"(h[3])
      : "f"(v[0]), "f"(v[1]), "f"(v[2]), "f"(v[3]), "f"(v[4]), "f"(v[5]), "f"(v[6]), "f"(v[7]));
#pragma unroll
  for (int j = 0; j < 4; ++j)
    asm("{\n\t.reg .f16 l, u;\n\tmov.b32 {l, u}, %2;\n\tcvt.f32.f16 %0, l;\n\tcvt.f32.f16 %1, u;\n\t}"
        : "=f"(q[2 * j]), "=f"(q[2 * j + 1])
        : "r"(h[j]));
  return out;
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
// R is formed in fp32, exactly: with x an element (exponent e, so a multiple of
// its bf16 ulp 2^(e-7)) and s the block's scale exponent (s >= e - 2), DQ(Q(x)) =
// q * 2^s is a multiple of 2^(s-1), hence of ulp(x), and the nearest grid point
// is no farther from x than 0 is, so |x - DQ| <= |x|.  x - DQ is thus a multiple
// of ulp(x) below 2^(e+1), a bf16 (so also fp32) value; q * 2^s is exact too (q
// has 2 significant bits, 2^-127 is an fp32 subnormal), so one fp32 FMA
// q * (-2^s) + x returns R unrounded (saturated elements, |x| < 8 * 2^s against
// 6 * 2^s, too).  R's elements being bf16 values, its amax has the exponent field
// the bf16 rule reads.
template <bool kResidual>
__device__ __forceinline__ void quantize_block(const uint32_t (&w)[16], uint32_t (&cx)[4], uint32_t& sx_out,
                                               uint32_t (&cr)[4], uint32_t& sr_out) {
  // ---- Q(X): block amax on bf16 magnitudes (NaN-propagating), E8M0 byte
  const uint32_t sx = scale_byte(block_amax_bits(w) >> 7);
  const uint32_t sx_eff = sx == 0xFFu ? 127u : sx;   // codes of a non-finite block are unspecified
  const float inv_x = inv_scale(sx_eff);
  const float neg_sc = -__uint_as_float(sx_eff == 0u ? 0x00400000u : sx_eff << 23);   // -2^(sx-127)

  // Per group of 8 elements: unpack bf16 -> fp32, scale (exact), encode; with
  // the residual, decode the codes and form R = x - q * 2^s.
  float r[32];
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    float x[8], v[8];
#pragma unroll
    for (int h = 0; h < 4; ++h) {
      unpack_bf16x2(w[4 * k + h], x[2 * h], x[2 * h + 1]);
      mul2(v[2 * h], v[2 * h + 1], x[2 * h], x[2 * h + 1], inv_x);
    }
    if constexpr (kResidual) {
      float q[8];
      cx[k] = encode8_dq(v, q);
#pragma unroll
      for (int h = 0; h < 4; ++h)
        fma2(r[8 * k + 2 * h], r[8 * k + 2 * h + 1], q[2 * h], q[2 * h + 1], neg_sc, x[2 * h], x[2 * h + 1]);
    } else {
      cx[k] = encode8(v);
    }
  }
  sx_out = sx;

  if constexpr (kResidual) {
    // ---- Q(R) by the same rule (R is finite when X is; a non-finite X block
    // forces byte 0xFF)
    float m[16];
#pragma unroll
    for (int i = 0; i < 16; ++i) m[i] = fmaxf(fabsf(r[2 * i]), fabsf(r[2 * i + 1]));
#pragma unroll
    for (int n = 8; n >= 1; n >>= 1)
#pragma unroll
      for (int i = 0; i < n; ++i) m[i] = fmaxf(m[i], m[i + n]);
    uint32_t sr = scale_byte(__float_as_uint(m[0]) >> 23);
    if (sx == 0xFFu) sr = 0xFFu;
    const float inv_r = inv_scale(sr == 0xFFu ? 127u : sr);
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      float v[8];
#pragma unroll
      for (int h = 0; h < 4; ++h) mul2(v[2 * h], v[2 * h + 1], r[8 * k + 2 * h], r[8 * k + 2 * h + 1], inv_r);
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
