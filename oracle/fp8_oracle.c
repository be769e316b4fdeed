/*
 * fp8_oracle.c -- plain, slow CPU oracle for the FP8 delayed-scaling linear path.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product library links, includes or
 * calls this file; only the test suite, the smoke check and the CPU-baseline leg
 * of the benchmark use it.  It shares no code, header, table or constant with the
 * CUDA path.
 *
 * Every function below is the definition of the operation written out directly,
 * single-threaded, with no blocking, fusion or reordering:
 *
 *   - FP8 formats (E4M3FN, E5M2): the field layouts whose extreme values the
 *     finfo table of "Accelerating PyTorch Training Workloads with FP8 -- Part 2"
 *     (section "PyTorch-native FP8 data types") prints: max 448 / 57344,
 *     smallest normal 2^-6 / 2^-14, eps 2^-3 / 2^-2.
 *   - Cast: the same page's worked example casts fp32 values to both formats
 *     with round-to-nearest; the cast here is round-to-nearest-even on the exact
 *     value, saturating to +-max (the plain reading of "saturating cast").
 *   - Per-tensor scaling: q = cast(fl32(x * scale)); the FP8 tensor carries the
 *     private scale_inv = fl32(1 / scale) it was cast with ("[PyTorch] Refactor
 *     FP8 workspaces in linear modules": Float8Tensor keeps a private copy of the
 *     scale-inverse that later scale updates do not touch).
 *   - Delayed scaling update (recipe DelayedScaling(amax_history_len=16,
 *     amax_compute_algo="max") in "CPU Overhead of te.Linear FP8 Layers", repro
 *     script): scale = fp8_max / max(amax window), history rolled by one slot.
 *   - GEMM: D = (sum_k dec(A[m,k]) dec(B[n,k])) * a_scale_inv * b_scale_inv
 *     + bias[n], the torch._scaled_mm contract shown on the PyTorch FP8 page.
 *
 * Floating point: fp64 throughout.  Where the method fixes fp32 (the scaled
 * value, the scale, the scale inverse) the fp64 result is rounded once to fp32.
 * For a product of two fp32 values the fp64 product is exact (48 <= 53 bits), so
 * one rounding to fp32 equals the IEEE fp32 product.  For a quotient of two fp32
 * values, rounding the correctly rounded fp64 quotient to fp32 equals the
 * correctly rounded fp32 quotient, because 53 >= 2*24 + 2 (double rounding is
 * innocuous for division under that condition).
 */
#include <math.h>
#include <stdint.h>
#include <string.h>

#define ORC_E4M3 0
#define ORC_E5M2 1

#define ORC_F32 0
#define ORC_BF16 1

/* ---------------------------------------------------------------- decode -- */

/* Value of one FP8 code, exactly, as a double (NaN for NaN codes). */
double orc_decode(uint8_t code, int fmt)
{
    int s = (code >> 7) & 1;
    double sign = s ? -1.0 : 1.0;
    if (fmt == ORC_E4M3) {
        /* 1 sign, 4 exponent (bias 7), 3 mantissa bits; no infinities; the
         * only NaN encodings are S.1111.111. */
        int e = (code >> 3) & 0xF;
        int m = code & 0x7;
        if (e == 15 && m == 7) return NAN;
        if (e == 0) return sign * ldexp((double)m / 8.0, 1 - 7);
        return sign * ldexp(1.0 + (double)m / 8.0, e - 7);
    } else {
        /* 1 sign, 5 exponent (bias 15), 2 mantissa bits; IEEE-style specials. */
        int e = (code >> 2) & 0x1F;
        int m = code & 0x3;
        if (e == 31) return m == 0 ? sign * INFINITY : NAN;
        if (e == 0) return sign * ldexp((double)m / 4.0, 1 - 15);
        return sign * ldexp(1.0 + (double)m / 4.0, e - 15);
    }
}

void orc_decode_table(int fmt, double *out256)
{
    for (int c = 0; c < 256; ++c) out256[c] = orc_decode((uint8_t)c, fmt);
}

/* Largest finite positive code: 0x7E (448) for E4M3FN, 0x7B (57344) for E5M2. */
static int max_finite_code(int fmt) { return fmt == ORC_E4M3 ? 0x7E : 0x7B; }

/* ---------------------------------------------------------------- encode -- */

/*
 * Saturating round-to-nearest-even of an fp32 value to FP8.
 *
 * Positive finite codes 0..max_code decode to strictly increasing values, so
 * the two codes that bracket |v| are found by binary search over the codes and
 * the nearer one is taken; on an exact tie the code with an even last bit (the
 * even mantissa) is taken.  |v| >= max (including +inf) gives the max code.
 * The sign bit is copied, so a negative value that rounds to zero gives the
 * negative-zero code 0x80.  NaN gives the canonical positive NaN code 0x7F in
 * both formats.  All differences below are exact in double (v has 24
 * significant bits, the decoded values at most 4).
 */
static uint8_t encode_with_table(float v, const double *dec, int top)
{
    if (isnan(v)) return 0x7F;
    uint8_t sign = signbit(v) ? 0x80 : 0x00;
    double a = fabs((double)v);
    if (a >= dec[top]) return (uint8_t)(sign | top);
    int lo = 0, hi = top; /* invariant: dec[lo] <= a < dec[hi] */
    while (hi - lo > 1) {
        int mid = (lo + hi) / 2;
        if (dec[mid] <= a) lo = mid; else hi = mid;
    }
    double dlo = a - dec[lo];
    double dhi = dec[hi] - a;
    int c;
    if (dlo < dhi) c = lo;
    else if (dhi < dlo) c = hi;
    else c = (lo % 2 == 0) ? lo : hi;
    return (uint8_t)(sign | c);
}

uint8_t orc_encode(float v, int fmt)
{
    double dec[256];
    orc_decode_table(fmt, dec);
    return encode_with_table(v, dec, max_finite_code(fmt));
}

void orc_encode_array(const float *v, int64_t n, int fmt, uint8_t *out)
{
    double dec[256];
    orc_decode_table(fmt, dec);
    int top = max_finite_code(fmt);
    for (int64_t i = 0; i < n; ++i) out[i] = encode_with_table(v[i], dec, top);
}

/* ------------------------------------------------------------- quantize -- */

static float load_elem(const void *x, int xdtype, int64_t i)
{
    if (xdtype == ORC_F32) return ((const float *)x)[i];
    /* bf16 is the top half of an fp32: widening is exact. */
    uint32_t bits = (uint32_t)((const uint16_t *)x)[i] << 16;
    float f;
    memcpy(&f, &bits, sizeof f);
    return f;
}

/* max(m, v) where a NaN v (quiet or signalling) is ignored.  The amax and the
 * history window skip NaN entries; libm fmaxf is not used because for a
 * signalling NaN it returns NaN. */
static float max_ignoring_nan(float m, float v)
{
    if (isnan(v)) return m;
    if (isnan(m)) return v;
    return v > m ? v : m;
}

/* fl32(x * scale): exact fp64 product, rounded once to fp32. */
float orc_scaled(float x, float scale) { return (float)((double)x * (double)scale); }

/* fl32(1 / scale). */
float orc_reciprocal(float s) { return (float)(1.0 / (double)s); }

/*
 * Per-tensor cast of a row-major [rows, cols] tensor with one scale.
 *   y[i,j]  = encode(fl32(x[i,j] * scale))
 *   yt[j,i] = y[i,j]                  (if yt is not NULL)
 *   *amax   = max(*amax, max |x|)     (unscaled input; NaN ignored; if amax != NULL)
 *   *scale_inv_out = fl32(1 / scale)  (if not NULL)
 */
void orc_cast_transpose_amax(const void *x, int xdtype, int64_t rows, int64_t cols, int fmt,
                             float scale, uint8_t *y, uint8_t *yt, float *amax,
                             float *scale_inv_out)
{
    double dec[256];
    orc_decode_table(fmt, dec);
    int top = max_finite_code(fmt);
    float m = amax ? *amax : 0.0f;
    for (int64_t i = 0; i < rows; ++i) {
        for (int64_t j = 0; j < cols; ++j) {
            float v = load_elem(x, xdtype, i * cols + j);
            uint8_t q = encode_with_table(orc_scaled(v, scale), dec, top);
            if (y) y[i * cols + j] = q;
            if (yt) yt[j * rows + i] = q;
            m = max_ignoring_nan(m, fabsf(v));
        }
    }
    if (amax) *amax = m;
    if (scale_inv_out) *scale_inv_out = orc_reciprocal(scale);
}

/* Flat quantize (no transpose): the rows = 1 case of the above. */
void orc_quantize(const void *x, int xdtype, int64_t n, int fmt, float scale, uint8_t *y,
                  float *amax, float *scale_inv_out)
{
    orc_cast_transpose_amax(x, xdtype, 1, n, fmt, scale, y, NULL, amax, scale_inv_out);
}

/*
 * The amax alone: *amax = max(*amax, max |x|) over n elements, NaN ignored --
 * the reduction the cast above records, without producing codes.  Full-size
 * checks use it for tensors whose complete cast would take minutes here.
 */
void orc_amax(const void *x, int xdtype, int64_t n, float *amax)
{
    float m = *amax;
    for (int64_t i = 0; i < n; ++i) m = max_ignoring_nan(m, fabsf(load_elem(x, xdtype, i)));
    *amax = m;
}

/* --------------------------------------------------------------- update -- */

/*
 * Delayed-scaling update of T meta tensors.
 * History layout: hist[h * T + t], h = 0..H-1 (slot 0 holds the amax recorded
 * in the current step).  Per tensor t:
 *   a      = max_h hist[h][t]            amax_compute_algo = "max" (algo 0)
 *            hist[0][t]                   "most_recent" (algo 1): the current
 *                                         step's amax alone
 *   scale' = fl32(fp8_max / a)  if a > 0, a finite and the quotient finite;
 *            otherwise the previous scale is kept
 *   scale_inv = fl32(1 / scale')
 *   roll:  hist'[h] = hist[(h + 1) mod H], then hist'[0] = 0
 * After the roll slot H-1 holds the current amax and slot 0 is clear for the
 * next step, so each max is over exactly the last H recorded amaxes.
 */
void orc_update_scales_algo(int64_t T, int H, float *hist, float *scale, float *scale_inv,
                            const uint8_t *fmts, int algo)
{
    for (int64_t t = 0; t < T; ++t) {
        float a = hist[t];
        if (algo == 0)
            for (int h = 1; h < H; ++h) a = max_ignoring_nan(a, hist[(int64_t)h * T + t]);
        double fp8_max = orc_decode((uint8_t)max_finite_code(fmts[t]), fmts[t]);
        float s = scale[t];
        if (a > 0.0f && isfinite(a)) {
            float q = (float)(fp8_max / (double)a);
            if (isfinite(q)) s = q;
        }
        scale[t] = s;
        scale_inv[t] = orc_reciprocal(s);
        float first = hist[t];
        for (int h = 0; h < H - 1; ++h) hist[(int64_t)h * T + t] = hist[(int64_t)(h + 1) * T + t];
        hist[(int64_t)(H - 1) * T + t] = first;
        hist[t] = 0.0f;
    }
}

void orc_update_scales(int64_t T, int H, float *hist, float *scale, float *scale_inv,
                       const uint8_t *fmts)
{
    orc_update_scales_algo(T, H, hist, scale, scale_inv, fmts, 0);
}

/* ----------------------------------------------------------- bf16 output -- */

/*
 * Round-to-nearest-even of an exact (fp64) value to bf16, returned as its 16
 * raw bits.  bf16 keeps 8 significant bits, normal exponents down to 2^-126 and
 * subnormals down to 2^-133; a value whose rounded magnitude reaches 2^128
 * overflows to infinity.  The quantum for |d| in [2^(e-1), 2^e) is
 * 2^max(e-8, -133); scaling by it is exact, nearbyint() rounds to even in the
 * default rounding mode, and the rounded value is exact in fp32.
 */
uint16_t orc_round_bf16(double d)
{
    if (isnan(d)) return 0x7FC0;
    uint16_t sign = signbit(d) ? 0x8000 : 0x0000;
    double a = fabs(d);
    if (a == 0.0) return sign;
    if (isinf(a)) return (uint16_t)(sign | 0x7F80);
    int e;
    frexp(a, &e);
    int qexp = e - 8 < -133 ? -133 : e - 8;
    double r = ldexp(nearbyint(ldexp(a, -qexp)), qexp);
    if (r >= ldexp(1.0, 128)) return (uint16_t)(sign | 0x7F80);
    float f = (float)r;
    uint32_t bits;
    memcpy(&bits, &f, sizeof bits);
    return (uint16_t)(sign | (bits >> 16));
}

void orc_round_bf16_array(const double *d, int64_t n, uint16_t *out)
{
    for (int64_t i = 0; i < n; ++i) out[i] = orc_round_bf16(d[i]);
}

/* ----------------------------------------------------------------- GEMM -- */

/*
 * D[m,n] = (sum_k dec(A[m,k]) * dec(B[n,k])) * a_scale_inv * b_scale_inv + bias[n]
 * A is [M,K] row-major, B is [N,K] row-major (both contraction-major), bias is
 * NULL or [N].  Computed for the rows listed in `row_idx` (all rows if NULL,
 * n_rows = M); D is [n_rows, N] in fp64.
 */
void orc_gemm_rows(const uint8_t *A, int fa, const uint8_t *B, int fb, float a_scale_inv,
                   float b_scale_inv, const float *bias, int64_t M, int64_t N, int64_t K,
                   const int64_t *row_idx, int64_t n_rows, double *D)
{
    double da[256], db[256];
    orc_decode_table(fa, da);
    orc_decode_table(fb, db);
    for (int64_t r = 0; r < n_rows; ++r) {
        int64_t m = row_idx ? row_idx[r] : r;
        if (m < 0 || m >= M) continue;
        for (int64_t n = 0; n < N; ++n) {
            double acc = 0.0;
            for (int64_t k = 0; k < K; ++k) acc += da[A[m * K + k]] * db[B[n * K + k]];
            double d = acc * (double)a_scale_inv * (double)b_scale_inv;
            if (bias) d += (double)bias[n];
            D[r * N + n] = d;
        }
    }
}

void orc_gemm(const uint8_t *A, int fa, const uint8_t *B, int fb, float a_scale_inv,
              float b_scale_inv, const float *bias, int64_t M, int64_t N, int64_t K, double *D)
{
    orc_gemm_rows(A, fa, B, fb, a_scale_inv, b_scale_inv, bias, M, N, K, NULL, M, D);
}
