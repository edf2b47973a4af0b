/*
 * nvq_oracle.c -- plain, slow CPU oracle for the microscaling-quantized
 * linear layer: NVFP4 / MXFP8 activation quantization, dequantization and
 * the block-scaled GEMM that consumes the quantized operands.
 *
 * TEST INFRASTRUCTURE.  Only the test suite, the smoke check and the
 * benchmark's CPU-baseline leg load this library.  It shares no code, table,
 * header or constant generator with the CUDA library, and neither side
 * imports the other.
 *
 * Sources (the pages this follows):
 *   [P1] "NVIDIA量化推理：5步极速优化显存+成功率翻倍" (nmedialink.com),
 *        section "MXFP8和NVFP4技术背景解析": microscaling groups small blocks
 *        (16 or 32 values) under one high-precision scale; MXFP8 is the OCP
 *        8-bit format with E4M3/E5M2 elements; NVFP4 is E2M1 in 16-value
 *        blocks with an FP8 scale, ~3.5x smaller than BF16.
 *   [P2] "NVIDIA Blackwell平台FP4量化技术解析与图像生成优化" (jsqmd.com),
 *        section 3.1: dynamic quantization returns FP4 data, FP8 block
 *        scales and one FP32 global scale; block scales FP8, global FP32.
 *   [P5] "FP8量化技术提升SD3.5在低带宽环境下的响应速度" (blog.csdn.net),
 *        section "量化映射": q = round(x / scale), x_dequant = q * scale;
 *        section "Fake Quantization": store low precision, compute after
 *        up-casting (the GEMM definition used here).
 *
 * Readings where the pages are silent (each listed in the design notes):
 *   - E2M1 = 1 sign, 2 exponent, 1 mantissa bit, bias 1 (the name, not the
 *     garbled "1 exponent + 2 mantissa" of [P2] section 1).
 *   - E4M3 is the FN variant (max 448, no infinities, S.1111.111 = NaN).
 *   - E8M0 is an unsigned biased exponent, value 2^(c-127), 0xFF = NaN.
 *   - round() is round-to-nearest, ties to even, saturating at the largest
 *     finite value; the sign is kept, so a negative value that rounds to
 *     zero gives -0.
 *   - NVFP4 global scale: g_enc = 2688 / amax_t, g_dec = amax_t / 2688
 *     (2688 = 6 * 448 maps the tensor maximum onto the largest E2M1 value
 *     times the largest E4M3 value); the stored FP32 global scale is g_dec.
 *     Scale decisions are taken in FP32 (the pages fix FP32 for the global
 *     scale), in exactly the order written below, with no fused multiply-add.
 *   - A tensor whose amax_t is below 2^-100 (zero included) quantizes to all
 *     zero codes and scales with g_dec = 0.
 *   - MXFP8 block scale: OCP MX rule X = floor(log2(block amax)) - emax, emax
 *     the exponent of the element type's largest normal (8 for E4M3, 15 for
 *     E5M2); the "ceil" variant takes the smallest X with block amax <=
 *     max_elem * 2^X instead, so no element saturates.
 *   - E5M2 is the IEEE-like variant: s.eeeee.mm, bias 15, max finite 57344,
 *     S.11111.00 = infinity, S.11111.xx = NaN; encoding saturates at 57344.
 *   - Ragged row counts: codes are dense over the M rows; the scale tiles
 *     are padded to a multiple of 128 rows with zero bytes.
 *   - The activation between the two linears of a feed-forward block is GELU
 *     with the exact error function, 0.5 x (1 + erf(x / sqrt 2)), evaluated in
 *     binary64 on the BF16 output of the first linear and rounded once to BF16.
 *   - Scale bytes are stored in the 128x4 tensor-core tile order (see
 *     oracle_sf_offset).
 *   - Codes are K-contiguous; two E2M1 codes per byte, even element in the
 *     low nibble.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define ORACLE_EXPORT __attribute__((visibility("default")))

/* ------------------------------------------------------------------ */
/* Element formats: decode straight from the bit fields.              */
/* ------------------------------------------------------------------ */

/* E2M1 ([P1] "NVFP4量化格式"): s.ee.m, bias 1; e == 0 is subnormal (m * 0.5). */
ORACLE_EXPORT double oracle_e2m1_value(int code) {
    int s = (code >> 3) & 1, e = (code >> 1) & 3, m = code & 1;
    double mag = (e == 0) ? 0.5 * m : ldexp(1.0 + 0.5 * m, e - 1);
    return s ? -mag : mag;
}

/* E4M3 FN ([P1] "MXFP8量化格式", [P5] "E4M3"): s.eeee.mmm, bias 7. */
ORACLE_EXPORT double oracle_e4m3_value(int code) {
    int s = (code >> 7) & 1, e = (code >> 3) & 15, m = code & 7;
    if (e == 15 && m == 7) return NAN;
    double mag = (e == 0) ? ldexp((double)m, -9) : ldexp(1.0 + m / 8.0, e - 7);
    return s ? -mag : mag;
}

/* E5M2 ([P1] "MXFP8量化格式" names E4M3 and E5M2): s.eeeee.mm, bias 15;
 * e == 0 is subnormal (m * 2^-16); e == 31 is infinity (m == 0) or NaN. */
ORACLE_EXPORT double oracle_e5m2_value(int code) {
    int s = (code >> 7) & 1, e = (code >> 2) & 31, m = code & 3;
    double mag;
    if (e == 31) mag = (m == 0) ? INFINITY : NAN;
    else mag = (e == 0) ? ldexp((double)m, -16) : ldexp(1.0 + m / 4.0, e - 15);
    return s ? -mag : mag;
}

/* E8M0: 2^(c - 127); 0xFF is NaN. */
ORACLE_EXPORT double oracle_e8m0_value(int code) {
    if (code == 255) return NAN;
    return ldexp(1.0, code - 127);
}

/* ------------------------------------------------------------------ */
/* Rounding: nearest representable value, ties to the even code,      */
/* saturating.  Written as a search over the value table so that it   */
/* follows the definition, not a bit trick.                           */
/* ------------------------------------------------------------------ */

/* Generic nearest-even search over the non-negative codes 0..max_code,
 * whose values increase with the code. */
static int round_to_table(double a, int max_code, double (*value)(int)) {
    if (a >= value(max_code)) return max_code;          /* saturate */
    int lo = 0, hi = max_code;                           /* value(lo) <= a < value(hi) */
    while (hi - lo > 1) {
        int mid = (lo + hi) / 2;
        if (value(mid) <= a) lo = mid; else hi = mid;
    }
    double vlo = value(lo), vhi = value(hi);
    if (a == vlo) return lo;
    double mid = 0.5 * (vlo + vhi);                     /* exact in binary64 */
    if (a < mid) return lo;
    if (a > mid) return hi;
    return (lo % 2 == 0) ? lo : hi;                      /* tie: even code */
}

static int g_nan_seen = 0;

/* E2M1 encode of an FP32 value: RNE, saturate to 6, sign kept. */
ORACLE_EXPORT int oracle_e2m1_encode(float v) {
    if (isnan(v)) { g_nan_seen = 1; return 0x7; }
    int sign = signbit(v) ? 0x8 : 0x0;
    return sign | round_to_table(fabs((double)v), 7, oracle_e2m1_value);
}

/* E4M3 encode of an FP32 value: RNE, saturate to 448, sign kept. */
ORACLE_EXPORT int oracle_e4m3_encode(float v) {
    if (isnan(v)) { g_nan_seen = 1; return 0x7F; }
    int sign = signbit(v) ? 0x80 : 0x00;
    return sign | round_to_table(fabs((double)v), 0x7E, oracle_e4m3_value);
}

/* E5M2 encode of an FP32 value: RNE, saturate to 57344 (code 0x7B), sign kept. */
ORACLE_EXPORT int oracle_e5m2_encode(float v) {
    if (isnan(v)) { g_nan_seen = 1; return 0x7F; }
    int sign = signbit(v) ? 0x80 : 0x00;
    return sign | round_to_table(fabs((double)v), 0x7B, oracle_e5m2_value);
}

/* Elementwise oracle_e4m3_encode of n FP32 values: the array form that a
 * test uses to bound MXFP8 element codes (E4M3 elements, page "NVIDIA量化推理：
 * 5步极速优化显存+成功率翻倍", section MXFP8量化格式). */
ORACLE_EXPORT void oracle_e4m3_encode_array(const float* in, int64_t n, uint8_t* out) {
    for (int64_t i = 0; i < n; ++i) out[i] = (uint8_t)oracle_e4m3_encode(in[i]);
}

/* Returns 1 if any NaN input reached an encoder since the last call. */
ORACLE_EXPORT int oracle_take_nan_flag(void) { int f = g_nan_seen; g_nan_seen = 0; return f; }

/* ------------------------------------------------------------------ */
/* Scale-factor storage order: the 128x4 tile of the sm_100 block-    */
/* scaled tensor-core operand.  A logical scale matrix S[R][C] (R     */
/* rows, C = K / block scale columns), with R padded to 128 and C to  */
/* 4, is stored as tiles of 128 rows x 4 columns, 512 bytes each,     */
/* ordered row-tile major then column-tile; inside a tile, row r and  */
/* column c sit at (r % 32) * 16 + ((r % 128) / 32) * 4 + (c % 4).    */
/* Padding bytes are zero.                                            */
/* ------------------------------------------------------------------ */

static int64_t round_up(int64_t x, int64_t m) { return (x + m - 1) / m * m; }

ORACLE_EXPORT int64_t oracle_sf_bytes(int64_t rows, int64_t cols) {
    return round_up(rows, 128) * round_up(cols, 4);
}

ORACLE_EXPORT int64_t oracle_sf_offset(int64_t r, int64_t c, int64_t cols) {
    int64_t col_tiles = round_up(cols, 4) / 4;
    int64_t tile = (r / 128) * col_tiles + (c / 4);
    return tile * 512 + (r % 32) * 16 + ((r % 128) / 32) * 4 + (c % 4);
}

/* ------------------------------------------------------------------ */
/* BF16 input                                                          */
/* ------------------------------------------------------------------ */

static float bf16_to_float(uint16_t h) {
    uint32_t u = (uint32_t)h << 16;
    float f;
    memcpy(&f, &u, 4);
    return f;
}

/* binary64 -> BF16 bits, round to nearest (one rounding; overflow to
 * infinity, NaN kept quiet).  A value exactly half-way between two BF16
 * values goes to the even one (tie = 0), or toward +infinity (tie > 0) or
 * -infinity (tie < 0).  Written from the binary64 fields. */
static uint16_t bf16_round_tie(double v, int tie) {
    uint64_t u;
    memcpy(&u, &v, 8);
    const uint16_t sign = (uint16_t)((u >> 48) & 0x8000u);
    if (isnan(v)) return (uint16_t)(sign | 0x7FC0u);
    double a = fabs(v);
    if (a == 0.0) return sign;
    /* a = m * 2^e with m in [1, 2) */
    int e;
    (void)frexp(a, &e);                  /* a = f * 2^e, f in [0.5, 1) */
    e -= 1;                              /* a = (2f) * 2^e */
    if (e > 127) return (uint16_t)(sign | 0x7F80u);
    /* quantum of the BF16 grid at this exponent: 2^(e-7) for normals,
     * 2^-133 for subnormals (e < -126) */
    int qexp = (e < -126) ? -133 : e - 7;
    double units = ldexp(a, -qexp);      /* exact: a / quantum */
    double fl = floor(units), rem = units - fl;
    double r = fl;
    int up;                              /* round the magnitude up */
    if (rem != 0.5) up = rem > 0.5;
    else if (tie == 0) up = fmod(fl, 2.0) != 0.0;
    else up = (tie > 0) == (sign == 0); /* toward +inf grows a positive magnitude */
    if (up) r = fl + 1.0;
    double rounded = ldexp(r, qexp);     /* exact */
    if (rounded >= 0x1p128) return (uint16_t)(sign | 0x7F80u);
    float rf = (float)rounded;           /* exact: rounded is on the BF16 grid */
    uint32_t b;
    memcpy(&b, &rf, 4);
    return (uint16_t)(sign | (uint16_t)((b >> 16) & 0x7FFFu));
}

ORACLE_EXPORT uint16_t oracle_double_to_bf16(double v) { return bf16_round_tie(v, 0); }

/* GELU of a BF16 value, x * Phi(x) with Phi the standard normal CDF (the
 * exact-erf form), rounded once to BF16.
 *   |x| >= 1:  x * erfc(-x / sqrt 2) / 2 in binary64; the same function as
 *              x (1 + erf(x / sqrt 2)) / 2 without its cancellation for
 *              negative x (GELU(-10) is -7.6e-23, not 0).
 *   |x| < 1:   x/2 + (x/2) erf(x / sqrt 2), the exact sum of the two binary64
 *              terms (TwoSum: s + err).  For a subnormal x, x/2 can fall
 *              exactly half-way between two BF16 values; the second term,
 *              about x^2 / sqrt(2 pi) > 0, then decides, although it is far
 *              below binary64 resolution at x/2.
 * GELU(+-0) = +-0; GELU(+inf) = +inf; GELU(-inf) is its limit, -0. */
ORACLE_EXPORT uint16_t oracle_gelu_bf16(uint16_t in) {
    const double x = (double)bf16_to_float(in);
    const double c = 0.70710678118654752440;
    if (isnan(x)) return oracle_double_to_bf16(x);
    if (isinf(x)) return x > 0 ? 0x7F80u : 0x8000u;
    if (x == 0.0) return in;
    if (fabs(x) >= 1.0) return oracle_double_to_bf16(0.5 * x * erfc(-x * c));
    const double h = 0.5 * x;            /* exact */
    const double t = h * erf(x * c);
    const double s = h + t;
    const double bb = s - h;
    const double err = (h - (s - bb)) + (t - bb);
    /* s + err = h + t exactly; s is the binary64 nearest to it, so only
     * when s is itself a BF16 tie can err change the rounding */
    return bf16_round_tie(s, err > 0 ? 1 : (err < 0 ? -1 : 0));
}

/* Elementwise forms of the two functions above, over n values. */
ORACLE_EXPORT void oracle_double_to_bf16_array(const double* v, int64_t n, uint16_t* out) {
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < n; ++i) out[i] = oracle_double_to_bf16(v[i]);
}

ORACLE_EXPORT void oracle_gelu_bf16_array(const uint16_t* in, int64_t n, uint16_t* out) {
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < n; ++i) out[i] = oracle_gelu_bf16(in[i]);
}

/* ------------------------------------------------------------------ */
/* NVFP4 quantization ([P1] NVFP4; [P2] 3.1 three outputs)            */
/* ------------------------------------------------------------------ */

#define NVFP4_BLOCK 16
#define MXFP8_BLOCK 32

/* amax_t = max |x| over the M x K region (x row-major, row pitch ldx elements). */
ORACLE_EXPORT float oracle_amax(const uint16_t* x, int64_t M, int64_t K, int64_t ldx) {
    float amax = 0.0f;
    for (int64_t m = 0; m < M; ++m)
        for (int64_t k = 0; k < K; ++k) {
            float a = fabsf(bf16_to_float(x[m * ldx + k]));
            if (a > amax) amax = a;
        }
    return amax;
}

/*
 * Quantize one BF16 tensor to NVFP4.
 *   codes:  rows M, K/2 bytes per row (dense), element 2j in the low nibble.
 *   sf:     oracle_sf_bytes(M, K/16) bytes, 128x4 tile order, zero padding.
 *   g_dec:  out, the FP32 global (decode) scale.
 *   calib_amax: if non-NULL, the per-tensor amax to use instead of the
 *     tensor's own (a calibrated, static range; [P5] "校准").
 * Steps, all in FP32 round-to-nearest-even:
 *   1. amax_t = max |x|                          (or *calib_amax)
 *   2. g_enc = 2688 / amax_t, g_dec = amax_t / 2688
 *   3. per 16-block along K: b = max |x_i|; s = (b / 6) * g_enc;
 *      sc = E4M3(s)
 *   4. if decode(sc) == 0 the block's codes are 0; else
 *      r = g_enc / decode(sc), q_i = E2M1(x_i * r)
 */
ORACLE_EXPORT void oracle_nvfp4_quantize(const uint16_t* x, int64_t M, int64_t K, int64_t ldx,
                                         const float* calib_amax,
                                         uint8_t* codes, uint8_t* sf, float* g_dec_out) {
    const int64_t nblk = K / NVFP4_BLOCK;
    memset(sf, 0, (size_t)oracle_sf_bytes(M, nblk));
    memset(codes, 0, (size_t)(M * (K / 2)));

    float amax_t = calib_amax ? *calib_amax : oracle_amax(x, M, K, ldx);
    if (!(amax_t >= 0x1p-100f)) { *g_dec_out = 0.0f; return; }
    float g_enc = 2688.0f / amax_t;
    float g_dec = amax_t / 2688.0f;
    *g_dec_out = g_dec;

#pragma omp parallel for schedule(static)
    for (int64_t m = 0; m < M; ++m) {
        for (int64_t j = 0; j < nblk; ++j) {
            const uint16_t* blk = x + m * ldx + j * NVFP4_BLOCK;
            float b = 0.0f;
            for (int i = 0; i < NVFP4_BLOCK; ++i) {
                float a = fabsf(bf16_to_float(blk[i]));
                if (a > b) b = a;
            }
            float b6 = b / 6.0f;
            float s = b6 * g_enc;
            int sc = oracle_e4m3_encode(s);
            sf[oracle_sf_offset(m, j, nblk)] = (uint8_t)sc;
            float sc_val = (float)oracle_e4m3_value(sc);
            if (sc_val == 0.0f) continue;                   /* codes stay 0 */
            float r = g_enc / sc_val;
            for (int i = 0; i < NVFP4_BLOCK; ++i) {
                float v = bf16_to_float(blk[i]) * r;
                int q = oracle_e2m1_encode(v);
                int64_t e = j * NVFP4_BLOCK + i;            /* element index along K */
                uint8_t* byte = codes + m * (K / 2) + e / 2;
                *byte |= (uint8_t)((e % 2 == 0) ? q : (q << 4));
            }
        }
    }
}

/* x_hat = E2M1(q) * decode(sc) * g_dec, binary64, row-major [rows][K]. */
ORACLE_EXPORT void oracle_nvfp4_dequantize(const uint8_t* codes, const uint8_t* sf, float g_dec,
                                           int64_t rows, int64_t K, double* out) {
    const int64_t nblk = K / NVFP4_BLOCK;
#pragma omp parallel for schedule(static)
    for (int64_t m = 0; m < rows; ++m)
        for (int64_t k = 0; k < K; ++k) {
            uint8_t byte = codes[m * (K / 2) + k / 2];
            int q = (k % 2 == 0) ? (byte & 0xF) : (byte >> 4);
            double s = oracle_e4m3_value(sf[oracle_sf_offset(m, k / NVFP4_BLOCK, nblk)]);
            out[m * K + k] = oracle_e2m1_value(q) * s * (double)g_dec;
        }
}

/* ------------------------------------------------------------------ */
/* MXFP8 quantization ([P1] MXFP8 = OCP standard; E4M3 elements,      */
/* 32-element blocks, E8M0 shared scale)                              */
/* ------------------------------------------------------------------ */

/* floor(log2(b)) for a finite b > 0, from the binary64 exponent (exact). */
static int floor_log2(double b) {
    int e;
    double f = frexp(b, &e);    /* b = f * 2^e, f in [0.5, 1) */
    (void)f;
    return e - 1;
}

/* The element types of MXFP8: code -> value, value -> code, the largest
 * finite value and the exponent emax of that value. */
typedef struct {
    double (*value)(int);
    int (*encode)(float);
    double max_value;
    int emax;
} mx_elem;

static mx_elem mx_element(int elem) {
    mx_elem e;
    if (elem == 1) { e.value = oracle_e5m2_value; e.encode = oracle_e5m2_encode; e.max_value = 57344.0; e.emax = 15; }
    else { e.value = oracle_e4m3_value; e.encode = oracle_e4m3_encode; e.max_value = 448.0; e.emax = 8; }
    return e;
}

/* Shared block exponent X for block amax b > 0.
 *   rule 0 (OCP "floor"): X = floor(log2 b) - emax.
 *   rule 1 ("ceil"): the smallest X with b <= max_value * 2^X, found by
 *   stepping from the floor value (so that the definition is what runs).
 * Clamped to [-127, 127]; b == 0 gives -127. */
static int mx_block_exponent(float b, const mx_elem* e, int rule) {
    if (b == 0.0f) return -127;
    int X = floor_log2((double)b) - e->emax;
    if (rule == 1) {
        while ((double)b > ldexp(e->max_value, X)) ++X;
        while ((double)b <= ldexp(e->max_value, X - 1)) --X;
    }
    if (X < -127) X = -127;
    if (X > 127) X = 127;
    return X;
}

/*
 * Quantize one BF16 tensor to MXFP8.
 *   elem:  0 = E4M3 elements, 1 = E5M2 elements.
 *   rule:  0 = floor block exponent (OCP), 1 = ceil (no saturation).
 *   codes: rows M, K bytes per row (dense).
 *   sf:    oracle_sf_bytes(M, K/32) bytes of E8M0, 128x4 tile order, zero padding.
 * Per 32-block along K: b = max |x_i|; X as in mx_block_exponent; scale
 * byte = X + 127; q_i = ELEM(x_i * 2^-X)  (FP32 multiply by a power of two).
 */
ORACLE_EXPORT void oracle_mxfp8_quantize_ex(const uint16_t* x, int64_t M, int64_t K, int64_t ldx,
                                            int elem, int rule, uint8_t* codes, uint8_t* sf) {
    const int64_t nblk = K / MXFP8_BLOCK;
    const mx_elem e = mx_element(elem);
    memset(sf, 0, (size_t)oracle_sf_bytes(M, nblk));
#pragma omp parallel for schedule(static)
    for (int64_t m = 0; m < M; ++m) {
        for (int64_t j = 0; j < nblk; ++j) {
            const uint16_t* blk = x + m * ldx + j * MXFP8_BLOCK;
            float b = 0.0f;
            for (int i = 0; i < MXFP8_BLOCK; ++i) {
                float a = fabsf(bf16_to_float(blk[i]));
                if (a > b) b = a;
            }
            int X = mx_block_exponent(b, &e, rule);
            sf[oracle_sf_offset(m, j, nblk)] = (uint8_t)(X + 127);
            float mult = (float)ldexp(1.0, -X);   /* exact: 2^-X fits FP32 */
            for (int i = 0; i < MXFP8_BLOCK; ++i) {
                float v = bf16_to_float(blk[i]) * mult;
                codes[m * K + j * MXFP8_BLOCK + i] = (uint8_t)e.encode(v);
            }
        }
    }
}

/* The default MXFP8 quantizer: E4M3 elements, floor block exponent. */
ORACLE_EXPORT void oracle_mxfp8_quantize(const uint16_t* x, int64_t M, int64_t K, int64_t ldx,
                                         uint8_t* codes, uint8_t* sf) {
    oracle_mxfp8_quantize_ex(x, M, K, ldx, 0, 0, codes, sf);
}

/* x_hat = ELEM(q) * 2^X, binary64, row-major [rows][K]. */
ORACLE_EXPORT void oracle_mxfp8_dequantize_ex(const uint8_t* codes, const uint8_t* sf, int64_t rows, int64_t K,
                                              int elem, double* out) {
    const int64_t nblk = K / MXFP8_BLOCK;
    const mx_elem e = mx_element(elem);
#pragma omp parallel for schedule(static)
    for (int64_t m = 0; m < rows; ++m)
        for (int64_t k = 0; k < K; ++k) {
            double s = oracle_e8m0_value(sf[oracle_sf_offset(m, k / MXFP8_BLOCK, nblk)]);
            out[m * K + k] = e.value(codes[m * K + k]) * s;
        }
}

ORACLE_EXPORT void oracle_mxfp8_dequantize(const uint8_t* codes, const uint8_t* sf,
                                           int64_t rows, int64_t K, double* out) {
    oracle_mxfp8_dequantize_ex(codes, sf, rows, K, 0, out);
}

/* ------------------------------------------------------------------ */
/* GEMM over dequantized operands ([P5] fake quantization: compute    */
/* after up-casting), binary64.                                       */
/*   out[i][n] = sum_k A[rows[i]][k] * B[n][k]  (+ bias[n])           */
/* A is [*, K] and B is [N, K], both row-major; rows lists the A rows */
/* to evaluate (all of them, or a sample).                             */
/* ------------------------------------------------------------------ */
ORACLE_EXPORT void oracle_gemm_rows(const double* A, const double* B, int64_t N, int64_t K,
                                    const int64_t* rows, int64_t nrows,
                                    const uint16_t* bias_bf16, double* out) {
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t i = 0; i < nrows; ++i) {
        const double* a = A + rows[i] * K;
        for (int64_t n = 0; n < N; ++n) {
            const double* b = B + n * K;
            double acc = 0.0;
            for (int64_t k = 0; k < K; ++k) acc += a[k] * b[k];
            if (bias_bf16) acc += (double)bf16_to_float(bias_bf16[n]);
            out[i * N + n] = acc;
        }
    }
}

ORACLE_EXPORT int oracle_num_threads(void) {
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}
