/*
 * rfq_oracle.c -- plain, slow CPU oracle for Residual Fallback Quantization (RFQ)
 * with MXFP4 blocks.  TEST INFRASTRUCTURE ONLY: only the tests, the smoke check and
 * the benchmark's CPU-baseline leg may load this file's library.  It shares no
 * code, header, table or helper with the CUDA path.
 *
 * What it follows:
 *   "Activation Outliers Matter: Robust Recovery for Quantized Multimodal LLMs"
 *   (arXiv 2608.26581), abstract and section 1 (Introduction, the RFQ contribution
 *   paragraph): the activation is split into a primary FP4 quantization and an
 *   explicit residual, the *full* quantization error, which a second low-bit
 *   path requantizes; nothing is thresholded or dropped, and the residual's
 *   contribution is accumulated in the GEMM together with the primary term.
 *
 *   The pages stop at section 3.1 before defining MXFP4, so the format is the
 *   OCP Microscaling (MX) v1.0 MXFP4 rule: 32-element blocks along K, one E8M0
 *   power-of-two scale per block with exponent floor(log2(amax)) - 2, E2M1
 *   elements rounded to nearest with ties to even and saturated to +-6, and the
 *   smallest scale (byte 0) for an all-zero block.
 *
 * Every number is carried in IEEE double.  Every value that reaches the
 * quantizer (bf16 inputs, the exact residual) is exactly representable in
 * double, and the scaled value |x| * 2^-e is formed with ldexp, which is exact,
 * so every rounding decision below is taken on the exact real number.
 *
 * Parity of each function is pinned by tests/test_oracle_pins.py against
 * third-party decoders/encoders, brute force and closed forms.
 */
#include <math.h>
#include <stdint.h>
#include <stddef.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define RFQ_BLOCK 32        /* elements that share one E8M0 scale */
#define E8M0_NAN 0xFF       /* E8M0 encoding of NaN */

/* ------------------------------------------------------------------------- */
/* E2M1 element format: bit 3 sign, bits 2..1 exponent E (bias 1), bit 0 mantissa m. */

/* Value of a 4-bit E2M1 code (closed form: subnormal 0.5*m when E == 0,
 * otherwise 2^(E-1) * (1 + m/2)). */
double oracle_e2m1_value(uint8_t code)
{
    int sign = (code >> 3) & 1;
    int E = (code >> 1) & 3;
    int m = code & 1;
    double mag = (E == 0) ? 0.5 * m : ldexp(1.0 + 0.5 * m, E - 1);
    return sign ? -mag : mag;
}

/* Round a non-negative real v onto the E2M1 magnitude grid: the nearest of the
 * eight magnitudes, ties to the candidate with mantissa bit 0 (round half to
 * even), which for v above the largest magnitude (6) is 6 (saturation). */
static uint8_t e2m1_round_magnitude(double v)
{
    uint8_t best = 0;
    double best_d = fabs(v - oracle_e2m1_value(0));
    for (uint8_t c = 1; c < 8; ++c) {
        double d = fabs(v - oracle_e2m1_value(c));
        if (d < best_d || (d == best_d && (c & 1) == 0)) {
            best = c;
            best_d = d;
        }
    }
    return best;
}

/* E2M1 code of x under the block exponent e: magnitude |x| * 2^-e rounded as
 * above, with the sign bit copied from x (so -0 and negatives that round to
 * zero encode as 0x8). */
uint8_t oracle_e2m1_encode(double x, int e)
{
    double v = ldexp(fabs(x), -e);
    uint8_t mag = e2m1_round_magnitude(v);
    return (uint8_t)((signbit(x) ? 0x8 : 0x0) | mag);
}

/* ------------------------------------------------------------------------- */
/* E8M0 block scale: an 8-bit biased exponent, value 2^(byte - 127), 0xFF = NaN. */

/* Block exponent for a block amax (amax >= 0): floor(log2(amax)) - 2, with the
 * E2M1 largest exponent 2, clamped to the E8M0 range [-127, 127]; 0 gives -127.
 * Returns 128 for a non-finite amax (the caller encodes 0xFF). */
int oracle_block_exponent(double amax)
{
    if (!isfinite(amax))
        return 128;
    if (amax == 0.0)
        return -127;
    int p;
    (void)frexp(amax, &p);         /* amax = f * 2^p with 0.5 <= f < 1 */
    int e = (p - 1) - 2;           /* floor(log2(amax)) = p - 1 */
    if (e < -127) e = -127;
    if (e > 127) e = 127;
    return e;
}

/* ------------------------------------------------------------------------- */
/* One block of up to 32 reals -> E8M0 byte and 32 codes. */

static void quantize_block(const double* v, int n, uint8_t* codes, uint8_t* scale_byte, int* exponent)
{
    double amax = 0.0;
    int finite = 1;
    for (int i = 0; i < n; ++i) {
        if (!isfinite(v[i])) finite = 0;
        double a = fabs(v[i]);
        if (a > amax) amax = a;
    }
    if (!finite) {
        *scale_byte = E8M0_NAN;
        *exponent = 128;
        for (int i = 0; i < n; ++i) codes[i] = 0;   /* unspecified; written 0 */
        return;
    }
    int e = oracle_block_exponent(amax);
    *scale_byte = (uint8_t)(e + 127);
    *exponent = e;
    for (int i = 0; i < n; ++i)
        codes[i] = oracle_e2m1_encode(v[i], e);
}

/* bf16 bit pattern -> its exact value. */
double oracle_bf16_value(uint16_t bits)
{
    uint32_t u = ((uint32_t)bits) << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

static uint8_t get_code(const uint8_t* packed, size_t k)
{
    uint8_t b = packed[k >> 1];
    return (k & 1) ? (uint8_t)(b >> 4) : (uint8_t)(b & 0xF);
}

static void put_code(uint8_t* packed, size_t k, uint8_t c)
{
    uint8_t* b = &packed[k >> 1];
    if (k & 1) *b = (uint8_t)((*b & 0x0F) | (c << 4));
    else       *b = (uint8_t)((*b & 0xF0) | (c & 0xF));
}

/*
 * MXFP4 quantization of a row-major bf16 matrix x[rows][K] (K a multiple of 32),
 * optionally followed by the RFQ residual path.
 *
 *   codes_x  [rows][K/2]   element 2j in bits 3..0 of byte j, element 2j+1 in bits 7..4
 *   scales_x [rows][K/32]  E8M0 bytes, plain row-major
 *   codes_r / scales_r     the same for Q(R), R = X - DQ(Q(X)); both NULL = no residual
 *
 * The residual of every element is x - value(code) * 2^e, taken in double.  It is
 * exact: either the code is 0 (r = x), or |x| > 2^(e-2) so x is a multiple of
 * 2^(e-9) (bf16 carries 8 significant bits; below the bf16 normal range, of
 * 2^-133), value(code) * 2^e is a multiple of 2^(e-1), and |r| < 2^(e+1) (the
 * widest gap, saturation from [6, 8) to 6, is 2 * 2^e): at most ten significant
 * bits, so r is exact even in fp32.  R is then quantized with exactly the rule
 * used for X.  A block of X
 * that holds a NaN or infinity gets scale 0xFF in both Q(X) and Q(R).
 */
void oracle_quantize_bf16(const uint16_t* x, int64_t rows, int64_t K,
                          uint8_t* codes_x, uint8_t* scales_x,
                          uint8_t* codes_r, uint8_t* scales_r)
{
    const int64_t Kb = K / RFQ_BLOCK;
    memset(codes_x, 0, (size_t)(rows * K / 2));
    if (codes_r) memset(codes_r, 0, (size_t)(rows * K / 2));
    /* Rows are independent; OpenMP only spreads them over the host cores. */
    #pragma omp parallel for schedule(static)
    for (int64_t m = 0; m < rows; ++m) {
        double v[RFQ_BLOCK], r[RFQ_BLOCK];
        uint8_t cx[RFQ_BLOCK], cr[RFQ_BLOCK];
        for (int64_t kb = 0; kb < Kb; ++kb) {
            const uint16_t* src = x + m * K + kb * RFQ_BLOCK;
            for (int i = 0; i < RFQ_BLOCK; ++i) v[i] = oracle_bf16_value(src[i]);
            uint8_t sx; int ex;
            quantize_block(v, RFQ_BLOCK, cx, &sx, &ex);
            scales_x[m * Kb + kb] = sx;
            for (int i = 0; i < RFQ_BLOCK; ++i)
                put_code(codes_x + m * K / 2, (size_t)(kb * RFQ_BLOCK + i), cx[i]);
            if (!codes_r) continue;
            uint8_t sr; int er;
            if (sx == E8M0_NAN) {
                sr = E8M0_NAN;
                for (int i = 0; i < RFQ_BLOCK; ++i) cr[i] = 0;
            } else {
                for (int i = 0; i < RFQ_BLOCK; ++i)
                    r[i] = v[i] - ldexp(oracle_e2m1_value(cx[i]), ex);
                quantize_block(r, RFQ_BLOCK, cr, &sr, &er);
            }
            scales_r[m * Kb + kb] = sr;
            for (int i = 0; i < RFQ_BLOCK; ++i)
                put_code(codes_r + m * K / 2, (size_t)(kb * RFQ_BLOCK + i), cr[i]);
        }
    }
}

/* The same quantizer on a matrix of doubles (used to pin the residual path on
 * arbitrary reals, e.g. residuals that bf16 cannot hold). */
void oracle_quantize_f64(const double* x, int64_t rows, int64_t K,
                         uint8_t* codes, uint8_t* scales)
{
    const int64_t Kb = K / RFQ_BLOCK;
    memset(codes, 0, (size_t)(rows * K / 2));
    #pragma omp parallel for schedule(static)
    for (int64_t m = 0; m < rows; ++m)
        for (int64_t kb = 0; kb < Kb; ++kb) {
            uint8_t c[RFQ_BLOCK];
            uint8_t s; int e;
            quantize_block(x + m * K + kb * RFQ_BLOCK, RFQ_BLOCK, c, &s, &e);
            scales[m * Kb + kb] = s;
            for (int i = 0; i < RFQ_BLOCK; ++i)
                put_code(codes + m * K / 2, (size_t)(kb * RFQ_BLOCK + i), c[i]);
        }
}

/* DQ: out[m][k] = value(code) * 2^(scale - 127); a 0xFF scale gives NaN. */
void oracle_dequantize(const uint8_t* codes, const uint8_t* scales, int64_t rows, int64_t K, double* out)
{
    const int64_t Kb = K / RFQ_BLOCK;
    #pragma omp parallel for schedule(static)
    for (int64_t m = 0; m < rows; ++m)
        for (int64_t k = 0; k < K; ++k) {
            uint8_t s = scales[m * Kb + k / RFQ_BLOCK];
            double val = oracle_e2m1_value(get_code(codes + m * K / 2, (size_t)k));
            out[m * K + k] = (s == E8M0_NAN) ? NAN : ldexp(val, (int)s - 127);
        }
}

/* Textbook GEMM in double: Y[i][j] = sum_k A[i][k] * B[j][k] (both K-contiguous).
 * Also returns, per output, sum_k |A[i][k]| * |B[j][k]| in absY when non-NULL. */
void oracle_gemm_nt(const double* A, const double* B, int64_t M, int64_t N, int64_t K,
                    double* Y, double* absY)
{
    #pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < M; ++i)
        for (int64_t j = 0; j < N; ++j) {
            double acc = 0.0, aacc = 0.0;
            for (int64_t k = 0; k < K; ++k) {
                acc += A[i * K + k] * B[j * K + k];
                aacc += fabs(A[i * K + k]) * fabs(B[j * K + k]);
            }
            Y[i * N + j] = acc;
            if (absY) absY[i * N + j] = aacc;
        }
}

/*
 * Scale bytes as the Blackwell block-scaled MMA reads them (the cuBLAS/PTX
 * documented 128x4 scale-factor tile): the plain [rows][Kb] matrix is padded to
 * rows_pad = ceil(rows/128)*128 and Kb_pad = ceil(Kb/4)*4 (pad bytes 0) and cut
 * into 512-byte atoms of 128 rows x 4 blocks, stored row-tile-major with the
 * block-tile index fastest; inside an atom, (r, c) sits at
 * (r % 32) * 16 + (r / 32) * 4 + c.
 */
int64_t oracle_mma_scale_offset(int64_t r, int64_t c, int64_t Kb)
{
    int64_t Kb_pad = (Kb + 3) / 4 * 4;
    int64_t atom = (r / 128) * (Kb_pad / 4) + (c / 4);
    int64_t rr = r % 128, cc = c % 4;
    return atom * 512 + (rr % 32) * 16 + (rr / 32) * 4 + cc;
}

void oracle_scales_to_mma_layout(const uint8_t* plain, int64_t rows, int64_t Kb, uint8_t* out)
{
    int64_t rows_pad = (rows + 127) / 128 * 128;
    int64_t Kb_pad = (Kb + 3) / 4 * 4;
    memset(out, 0, (size_t)(rows_pad * Kb_pad));
    for (int64_t r = 0; r < rows; ++r)
        for (int64_t c = 0; c < Kb; ++c)
            out[oracle_mma_scale_offset(r, c, Kb)] = plain[r * Kb + c];
}

/* ------------------------------------------------------------------------- */
/* MXFP8 (E4M3 elements) comparator.  The paper finds MXFP8 nearly free of accuracy loss
 * (abstract; section 1, the first contribution); the format is the OCP MX v1.0
 * MXFP8 E4M3 rule: 32-element blocks along K, E8M0 scale exponent
 * floor(log2(amax)) - 8 (8 = the E4M3 largest exponent), elements rounded to the
 * nearest E4M3 value with ties to even and saturated to +-448.
 *
 * E4M3 ("fn": no infinities): bit 7 sign, bits 6..3 exponent E (bias 7), bits 2..0
 * mantissa m.  E == 0: subnormal 2^-6 * m/8; otherwise 2^(E-7) * (1 + m/8);
 * E == 15 and m == 7 is NaN, so the largest finite magnitude is 2^8 * 1.75 = 448. */

double oracle_e4m3_value(uint8_t code)
{
    int sign = (code >> 7) & 1;
    int E = (code >> 3) & 15;
    int m = code & 7;
    if (E == 15 && m == 7) return NAN;
    double mag = (E == 0) ? ldexp(m / 8.0, -6) : ldexp(1.0 + m / 8.0, E - 7);
    return sign ? -mag : mag;
}

/* Round a non-negative real v onto the E4M3 magnitudes (codes 0x00..0x7E, which
 * increase with the code): the nearest, ties to the even code (mantissa bit 0
 * clear); v beyond 448 gets 448 (saturation). */
static uint8_t e4m3_round_magnitude(double v)
{
    if (v >= 448.0) return 0x7E;
    /* largest code whose value is <= v (binary search over the increasing table) */
    int lo = 0, hi = 0x7E;
    while (lo < hi) {
        int mid = (lo + hi + 1) / 2;
        if (oracle_e4m3_value((uint8_t)mid) <= v) lo = mid; else hi = mid - 1;
    }
    if (lo == 0x7E) return 0x7E;
    double below = oracle_e4m3_value((uint8_t)lo), above = oracle_e4m3_value((uint8_t)(lo + 1));
    double db = v - below, da = above - v;
    if (db < da) return (uint8_t)lo;
    if (da < db) return (uint8_t)(lo + 1);
    return (lo & 1) ? (uint8_t)(lo + 1) : (uint8_t)lo;
}

uint8_t oracle_e4m3_encode(double x, int e)
{
    double v = ldexp(fabs(x), -e);
    uint8_t mag = e4m3_round_magnitude(v);
    return (uint8_t)((signbit(x) ? 0x80 : 0x00) | mag);
}

/* floor(log2(amax)) - 8 clamped to [-127, 127]; 0 gives -127; 128 = non-finite. */
int oracle_block_exponent_e4m3(double amax)
{
    if (!isfinite(amax))
        return 128;
    if (amax == 0.0)
        return -127;
    int p;
    (void)frexp(amax, &p);
    int e = (p - 1) - 8;
    if (e < -127) e = -127;
    if (e > 127) e = 127;
    return e;
}

/* MXFP8 quantization of a row-major bf16 x[rows][K]: codes [rows][K] one byte per
 * element, scales [rows][K/32] E8M0 plain row-major.  A block holding a NaN or
 * infinity gets scale 0xFF and codes 0 (unspecified). */
void oracle_quantize_mxfp8_bf16(const uint16_t* x, int64_t rows, int64_t K, uint8_t* codes, uint8_t* scales)
{
    const int64_t Kb = K / RFQ_BLOCK;
    #pragma omp parallel for schedule(static)
    for (int64_t m = 0; m < rows; ++m)
        for (int64_t kb = 0; kb < Kb; ++kb) {
            const uint16_t* src = x + m * K + kb * RFQ_BLOCK;
            double v[RFQ_BLOCK], amax = 0.0;
            int finite = 1;
            for (int i = 0; i < RFQ_BLOCK; ++i) {
                v[i] = oracle_bf16_value(src[i]);
                if (!isfinite(v[i])) finite = 0;
                if (fabs(v[i]) > amax) amax = fabs(v[i]);
            }
            uint8_t* dst = codes + m * K + kb * RFQ_BLOCK;
            if (!finite) {
                scales[m * Kb + kb] = E8M0_NAN;
                memset(dst, 0, RFQ_BLOCK);
                continue;
            }
            int e = oracle_block_exponent_e4m3(amax);
            scales[m * Kb + kb] = (uint8_t)(e + 127);
            for (int i = 0; i < RFQ_BLOCK; ++i) dst[i] = oracle_e4m3_encode(v[i], e);
        }
}

/* DQ of MXFP8: out[m][k] = value(code) * 2^(scale - 127); a 0xFF scale gives NaN. */
void oracle_dequantize_mxfp8(const uint8_t* codes, const uint8_t* scales, int64_t rows, int64_t K, double* out)
{
    const int64_t Kb = K / RFQ_BLOCK;
    #pragma omp parallel for schedule(static)
    for (int64_t m = 0; m < rows; ++m)
        for (int64_t k = 0; k < K; ++k) {
            uint8_t s = scales[m * Kb + k / RFQ_BLOCK];
            double val = oracle_e4m3_value(codes[m * K + k]);
            out[m * K + k] = (s == E8M0_NAN) ? NAN : ldexp(val, (int)s - 127);
        }
}

/* Host threads the row loops above run on (1 without OpenMP). */
int oracle_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}
