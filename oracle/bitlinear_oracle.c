/*
 * CPU oracle for the BitLinear forward path of BitNet a4.8
 * ("BitNet a4.8: 4-bit Activations for 1-bit LLMs", arXiv 2411.04965).
 *
 * TEST INFRASTRUCTURE ONLY.  This file is the plain, slow, obviously-correct
 * definition that the CUDA kernels are checked against.  It shares no code,
 * header, table or constant with the CUDA path, and only the test-suite, the
 * smoke check and the benchmark's CPU-baseline leg may build or call it.
 *
 * Build: gcc -O2 -ffp-contract=off -fno-fast-math -shared -fPIC (no SIMD
 * intrinsics, no FMA contraction, so every fp32 operation below is one IEEE
 * round-to-nearest-even operation in the order written).
 *
 * Conventions
 *   - bf16 values arrive as raw uint16 bit patterns; fp32 latent weights as float.
 *   - All quantizers work per token (one row of X), the reading the paper's
 *     per-tensor wording takes for a token-wise forward.
 *   - round() is round-half-to-even (rint under the default rounding mode).
 *   - Return value: 0 on success, a negative number when an input violates a
 *     stated precondition (see each function).
 */
#include <fenv.h>
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define ORC_OK 0
#define ORC_ERR_INEXACT_SUM (-2)   /* a row's |x| sum is not exact in fp64 */
#define ORC_ERR_ARG (-3)
#define ORC_ERR_NONFINITE (-4)
#define ORC_ERR_OVERFLOW (-5)

static float bf16_value(uint16_t h) {
    uint32_t u = (uint32_t)h << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return f;
}

static uint32_t f32_bits(float f) {
    uint32_t u;
    memcpy(&u, &f, sizeof u);
    return u;
}

/* fp64 -> bf16, rounded once to nearest even: 8 significant bits for normal
 * results, a fixed quantum of 2^-133 in bf16's subnormal range. */
static uint16_t bf16_round(double v) {
    if (v == 0.0) return (uint16_t)(signbit(v) ? 0x8000u : 0u);
    int e;
    frexp(v, &e);                         /* |v| = f * 2^e, f in [0.5, 1) */
    int lsb = (e - 1 >= -126) ? e - 8 : -133;
    double r = ldexp(rint(ldexp(v, -lsb)), lsb);   /* both ldexp calls are exact */
    if (fabs(r) >= ldexp(1.0, 128)) r = copysign(INFINITY, v);
    float f = (float)r;                   /* exact: r has <= 8 significant bits */
    return (uint16_t)(f32_bits(f) >> 16);
}

/* RoundClip(x, a, b) = min(max(round(x), a), b)
 * (§3.4 "Ternary Weight Quantization", the RoundClip definition). */
static float round_clip(float x, float a, float b) {
    float r = rintf(x);
    if (r < a) r = a;
    if (r > b) r = b;
    return r;
}

/* Sum of |x| over a bf16 row in fp64, with an error-free check that every
 * addition was exact (Knuth's TwoSum).  An exact sum does not depend on the
 * order of the additions, which is what lets the GPU reduce in any order. */
static int exact_abs_sum_bf16(const uint16_t* x, int64_t k, double* out) {
    double s = 0.0, err = 0.0;
    for (int64_t i = 0; i < k; ++i) {
        double a = fabs((double)bf16_value(x[i]));
        if (!isfinite(a)) return ORC_ERR_NONFINITE;
        double t = s + a;
        double bp = t - s;
        double e = (s - (t - bp)) + (a - bp);
        err += fabs(e);
        s = t;
    }
    if (err != 0.0) return ORC_ERR_INEXACT_SUM;
    *out = s;
    return ORC_OK;
}

/* ---------------------------------------------------------------------------
 * INT4 absmean activation quantizer (§3.4 "4-Bit Activation Quantization",
 * Eq. 6-7):   Q(X) = beta/sqrt7 * RoundClip(sqrt7/(beta+eps) * X, -8, 7),
 *             beta = mean(|X|), per token.
 * Outputs per element the integer code, per row beta and the dequant scale
 * beta/sqrt7 (fp32).
 * ------------------------------------------------------------------------- */
int orc_quant_int4(const uint16_t* x, int64_t M, int64_t K, int64_t ldx, float eps,
                   int8_t* codes, float* beta_out, float* scale_out) {
    if (M < 0 || K <= 0 || ldx < K) return ORC_ERR_ARG;
    const float sqrt7 = (float)sqrt(7.0);
    for (int64_t m = 0; m < M; ++m) {
        const uint16_t* row = x + m * ldx;
        double s;
        int rc = exact_abs_sum_bf16(row, K, &s);
        if (rc) return rc;
        float beta = (float)(s / (double)K);
        float mult = sqrt7 / (beta + eps);
        for (int64_t k = 0; k < K; ++k) {
            float v = bf16_value(row[k]) * mult;
            codes[m * K + k] = (int8_t)round_clip(v, -8.0f, 7.0f);
        }
        beta_out[m] = beta;
        scale_out[m] = beta / sqrt7;
    }
    return ORC_OK;
}

/* ---------------------------------------------------------------------------
 * FP4 E2M1 MinMax activation quantizer (§3.4 "FP4 Quantizer", Eq. 8-9).
 * The printed formula is garbled; the reading used: a per-token power-of-two
 * scale 2^p with p the smallest integer such that max|x| <= 6 * 2^p (6 is the
 * largest E2M1 magnitude, so nothing clips), then each x / 2^p is rounded to
 * the nearest E2M1 value {0, .5, 1, 1.5, 2, 3, 4, 6} (ties to the even
 * encoding).  A row of zeros takes p = 0.
 * Outputs: the E2M1 4-bit code per element (sign bit 3, value bits 0..2), the
 * value doubled as an exact integer in [-12, 12], p per row, and the dequant
 * scale 2^p as fp32.  A magnitude that rounds to 0 is encoded as +0 (code 0).
 * ------------------------------------------------------------------------- */
static const double e2m1_grid[8] = {0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0};

static int e2m1_nearest_index(double mag) {
    /* Nearest grid magnitude; on an exact tie take the even index, which is
     * the encoding whose mantissa bit is 0.  Magnitudes above 6 saturate. */
    int best = 0;
    double best_d = fabs(mag - e2m1_grid[0]);
    for (int i = 1; i < 8; ++i) {
        double d = fabs(mag - e2m1_grid[i]);
        if (d < best_d || (d == best_d && (i % 2 == 0) && (best % 2 == 1))) {
            best = i;
            best_d = d;
        }
    }
    return best;
}

int orc_quant_fp4(const uint16_t* x, int64_t M, int64_t K, int64_t ldx,
                  uint8_t* code4, int8_t* twice_value, int32_t* p_out, float* scale_out) {
    if (M < 0 || K <= 0 || ldx < K) return ORC_ERR_ARG;
    for (int64_t m = 0; m < M; ++m) {
        const uint16_t* row = x + m * ldx;
        double g = 0.0;
        for (int64_t k = 0; k < K; ++k) {
            double a = fabs((double)bf16_value(row[k]));
            if (!isfinite(a)) return ORC_ERR_NONFINITE;
            if (a > g) g = a;
        }
        int p = 0;
        if (g > 0.0) {
            while (g > 6.0 * ldexp(1.0, p)) ++p;
            while (g <= 6.0 * ldexp(1.0, p - 1)) --p;
        }
        for (int64_t k = 0; k < K; ++k) {
            double v = (double)bf16_value(row[k]) * ldexp(1.0, -p);   /* exact */
            int idx = e2m1_nearest_index(fabs(v));
            int neg = (v < 0.0) && idx != 0;
            code4[m * K + k] = (uint8_t)((neg ? 8 : 0) | idx);
            int tv = (int)(2.0 * e2m1_grid[idx]);
            twice_value[m * K + k] = (int8_t)(neg ? -tv : tv);
        }
        p_out[m] = p;
        scale_out[m] = (float)ldexp(1.0, p);
    }
    return ORC_OK;
}

/* ---------------------------------------------------------------------------
 * Quantizer variants of the ablation figures (Fig. 5: INT4 absmean with
 * beta = 2 mean(|X|); Fig. 6: INT4 absmax and FP4 E1M2 beside INT4 absmean and
 * FP4 E2M1).  The pages name them without formulas; the readings used:
 *   INT4 absmax:   Q(X) = gamma/7 * RoundClip(7/(gamma+eps) * X, -8, 7),
 *                  gamma = max|X| per token -- the absmax quantizer of Eq. 1
 *                  with the 4-bit range (7 = 2^(4-1) - 1).
 *   INT4 absmean, beta = 2 mean(|X|):  Eq. 6-7 with that beta.
 *   FP4 E1M2:      1 exponent bit (bias 1, no inf/nan) and 2 mantissa bits,
 *                  magnitudes {0, .25, .5, .75, 1, 1.25, 1.5, 1.75}; a per-token
 *                  power-of-two scale 2^p, p the smallest integer with
 *                  max|x| <= 1.75 * 2^p (the MinMax reading of the E2M1 case);
 *                  x / 2^p rounded to the nearest magnitude, ties to the even
 *                  encoding; code = sign bit 3 + magnitude index bits 0..2.
 * ------------------------------------------------------------------------- */
int orc_quant_int4_absmax(const uint16_t* x, int64_t M, int64_t K, int64_t ldx, float eps,
                          int8_t* codes, float* gamma_out, float* scale_out) {
    if (M < 0 || K <= 0 || ldx < K) return ORC_ERR_ARG;
    for (int64_t m = 0; m < M; ++m) {
        const uint16_t* row = x + m * ldx;
        float gamma = 0.0f;
        for (int64_t k = 0; k < K; ++k) {
            float a = fabsf(bf16_value(row[k]));
            if (!isfinite(a)) return ORC_ERR_NONFINITE;
            if (a > gamma) gamma = a;
        }
        float mult = 7.0f / (gamma + eps);
        for (int64_t k = 0; k < K; ++k) {
            float v = bf16_value(row[k]) * mult;
            codes[m * K + k] = (int8_t)round_clip(v, -8.0f, 7.0f);
        }
        gamma_out[m] = gamma;
        scale_out[m] = gamma / 7.0f;
    }
    return ORC_OK;
}

int orc_quant_int4_absmean2(const uint16_t* x, int64_t M, int64_t K, int64_t ldx, float eps,
                            int8_t* codes, float* beta_out, float* scale_out) {
    if (M < 0 || K <= 0 || ldx < K) return ORC_ERR_ARG;
    const float sqrt7 = (float)sqrt(7.0);
    for (int64_t m = 0; m < M; ++m) {
        const uint16_t* row = x + m * ldx;
        double s;
        int rc = exact_abs_sum_bf16(row, K, &s);
        if (rc) return rc;
        float beta = (float)((2.0 * s) / (double)K);   /* beta = 2 mean|x| */
        float mult = sqrt7 / (beta + eps);
        for (int64_t k = 0; k < K; ++k) {
            float v = bf16_value(row[k]) * mult;
            codes[m * K + k] = (int8_t)round_clip(v, -8.0f, 7.0f);
        }
        beta_out[m] = beta;
        scale_out[m] = beta / sqrt7;
    }
    return ORC_OK;
}

static const double e1m2_grid[8] = {0.0, 0.25, 0.5, 0.75, 1.0, 1.25, 1.5, 1.75};

static int e1m2_nearest_index(double mag) {
    /* nearest magnitude; an exact tie goes to the even index (mantissa bit 0) */
    int best = 0;
    double best_d = fabs(mag - e1m2_grid[0]);
    for (int i = 1; i < 8; ++i) {
        double d = fabs(mag - e1m2_grid[i]);
        if (d < best_d || (d == best_d && (i % 2 == 0) && (best % 2 == 1))) {
            best = i;
            best_d = d;
        }
    }
    return best;
}

/* Outputs: the 4-bit code, four times the value (an exact integer in [-7, 7]),
 * p per row and the dequant scale 2^p of the code's value. */
int orc_quant_fp4_e1m2(const uint16_t* x, int64_t M, int64_t K, int64_t ldx,
                       uint8_t* code4, int8_t* four_value, int32_t* p_out, float* scale_out) {
    if (M < 0 || K <= 0 || ldx < K) return ORC_ERR_ARG;
    for (int64_t m = 0; m < M; ++m) {
        const uint16_t* row = x + m * ldx;
        double g = 0.0;
        for (int64_t k = 0; k < K; ++k) {
            double a = fabs((double)bf16_value(row[k]));
            if (!isfinite(a)) return ORC_ERR_NONFINITE;
            if (a > g) g = a;
        }
        int p = 0;
        if (g > 0.0) {
            while (g > 1.75 * ldexp(1.0, p)) ++p;
            while (g <= 1.75 * ldexp(1.0, p - 1)) --p;
        }
        for (int64_t k = 0; k < K; ++k) {
            double v = (double)bf16_value(row[k]) * ldexp(1.0, -p);   /* exact */
            int idx = e1m2_nearest_index(fabs(v));
            int neg = (v < 0.0) && idx != 0;
            code4[m * K + k] = (uint8_t)((neg ? 8 : 0) | idx);
            four_value[m * K + k] = (int8_t)(neg ? -idx : idx);
        }
        p_out[m] = p;
        scale_out[m] = (float)ldexp(1.0, p);
    }
    return ORC_OK;
}

/* ---------------------------------------------------------------------------
 * Top-K mask (§3.4 "Sparsification Pipeline", Eq. 1: M = Top_k(|X|)).
 * Exactly `keep` survivors per row; the ranking key is (|x| descending,
 * index ascending), so ties at the threshold go to the lower index.
 * ------------------------------------------------------------------------- */
typedef struct { double mag; int64_t idx; } rank_item;

static int rank_cmp(const void* pa, const void* pb) {
    const rank_item* a = (const rank_item*)pa;
    const rank_item* b = (const rank_item*)pb;
    if (a->mag > b->mag) return -1;
    if (a->mag < b->mag) return 1;
    return (a->idx < b->idx) ? -1 : (a->idx > b->idx);
}

static void topk_mask_row(const double* mag, int64_t K, int64_t keep, rank_item* tmp, uint8_t* mask) {
    for (int64_t k = 0; k < K; ++k) { tmp[k].mag = mag[k]; tmp[k].idx = k; mask[k] = 0; }
    qsort(tmp, (size_t)K, sizeof(rank_item), rank_cmp);
    for (int64_t i = 0; i < keep; ++i) mask[tmp[i].idx] = 1;
}

/* INT8 absmax quantizer (§3.4, Q_INT8 next to Eq. 1):
 *   Q(X) = gamma/127 * RoundClip(127/(gamma+eps) * X, -128, 127), gamma = max|X|,
 * followed by the Top-K mask:  codes = RoundClip(...) * M. */
static void int8_absmax_masked(const float* xr, int64_t K, float eps, const uint8_t* mask,
                               int8_t* codes, float* gamma_out, float* scale_out) {
    float gamma = 0.0f;
    for (int64_t k = 0; k < K; ++k) {
        float a = fabsf(xr[k]);
        if (a > gamma) gamma = a;
    }
    float mult = 127.0f / (gamma + eps);
    for (int64_t k = 0; k < K; ++k) {
        float c = round_clip(xr[k] * mult, -128.0f, 127.0f);
        codes[k] = mask[k] ? (int8_t)c : (int8_t)0;
    }
    *gamma_out = gamma;
    *scale_out = gamma / 127.0f;
}

/* Sparsify-then-quantize for the outlier-heavy inputs (§3.4 "Sparsification
 * Pipeline", Eq. 1): Y-input = Q_INT8(X) (.) Top_k(|X|), per token. */
int orc_sparsify_a8(const uint16_t* x, int64_t M, int64_t K, int64_t ldx, int64_t keep, float eps,
                    int8_t* codes, uint8_t* mask, float* gamma_out, float* scale_out) {
    if (M < 0 || K <= 0 || ldx < K || keep < 1 || keep > K) return ORC_ERR_ARG;
    float* xr = (float*)malloc(sizeof(float) * (size_t)K);
    double* mag = (double*)malloc(sizeof(double) * (size_t)K);
    rank_item* tmp = (rank_item*)malloc(sizeof(rank_item) * (size_t)K);
    if (!xr || !mag || !tmp) { free(xr); free(mag); free(tmp); return ORC_ERR_ARG; }
    int rc = ORC_OK;
    for (int64_t m = 0; m < M && rc == ORC_OK; ++m) {
        for (int64_t k = 0; k < K; ++k) {
            xr[k] = bf16_value(x[m * ldx + k]);
            if (!isfinite(xr[k])) { rc = ORC_ERR_NONFINITE; break; }
            mag[k] = fabs((double)xr[k]);
        }
        if (rc) break;
        topk_mask_row(mag, K, keep, tmp, mask + m * K);
        int8_absmax_masked(xr, K, eps, mask + m * K, codes + m * K, gamma_out + m, scale_out + m);
    }
    free(xr); free(mag); free(tmp);
    return rc;
}

/* ---------------------------------------------------------------------------
 * ReLU^2-GLU (§3.4 "Squared ReLU Gating", Eq. 5):
 *   h = (X W_up^T) (.) ReLU^2(X W_gate^T),  ReLU^2(z) = max(0, z)^2,
 * in fp32 with two roundings in this order: g2 = g*g, h = u*g2.  The result
 * feeds the down projection through the same Top-K + INT8 step as above; the
 * ranking key is |h| in fp32.  `h_out` (nullable) receives h.
 * ------------------------------------------------------------------------- */
int orc_relu2_glu(const uint16_t* gate, const uint16_t* up, int64_t M, int64_t F, int64_t ld,
                  int64_t keep, float eps, int8_t* codes, uint8_t* mask, float* h_out,
                  float* gamma_out, float* scale_out) {
    if (M < 0 || F <= 0 || ld < F || keep < 1 || keep > F) return ORC_ERR_ARG;
    float* h = (float*)malloc(sizeof(float) * (size_t)F);
    double* mag = (double*)malloc(sizeof(double) * (size_t)F);
    rank_item* tmp = (rank_item*)malloc(sizeof(rank_item) * (size_t)F);
    if (!h || !mag || !tmp) { free(h); free(mag); free(tmp); return ORC_ERR_ARG; }
    int rc = ORC_OK;
    for (int64_t m = 0; m < M && rc == ORC_OK; ++m) {
        for (int64_t f = 0; f < F; ++f) {
            float gv = bf16_value(gate[m * ld + f]);
            float uv = bf16_value(up[m * ld + f]);
            if (!isfinite(gv) || !isfinite(uv)) { rc = ORC_ERR_NONFINITE; break; }
            float r = gv > 0.0f ? gv : 0.0f;
            float g2 = r * r;
            h[f] = uv * g2;
            if (!isfinite(h[f])) { rc = ORC_ERR_NONFINITE; break; }
            mag[f] = fabs((double)h[f]);
            if (h_out) h_out[m * F + f] = h[f];
        }
        if (rc) break;
        topk_mask_row(mag, F, keep, tmp, mask + m * F);
        int8_absmax_masked(h, F, eps, mask + m * F, codes + m * F, gamma_out + m, scale_out + m);
    }
    free(h); free(mag); free(tmp);
    return rc;
}

/* ---------------------------------------------------------------------------
 * Ternary weight quantizer (§3.4 "Ternary Weight Quantization", Eq. 2):
 *   Q_w(W) = alpha * RoundClip(W/(alpha+eps), -1, 1),  alpha = mean(|W|) per tensor.
 *
 * alpha is the exact mean rounded once to fp32.  The exact sum of |w| is kept
 * as one integer accumulator per fp32 biased exponent:
 *   |w| = m * 2^(max(E,1) - 150), m the 24-bit significand (hidden bit set when
 *   E > 0), so  sum|w| = sum_E bins[E] * 2^(max(E,1) - 150)  exactly.
 * orc_ternary_abs_bins fills the 256 bins (the caller finishes the rational
 * division and the single rounding with arbitrary-precision integers).
 * ------------------------------------------------------------------------- */
int orc_ternary_abs_bins(const float* w, int64_t N, int64_t K, int64_t ldw, uint64_t* bins) {
    if (N < 0 || K <= 0 || ldw < K) return ORC_ERR_ARG;
    for (int i = 0; i < 256; ++i) bins[i] = 0;
    for (int64_t n = 0; n < N; ++n) {
        for (int64_t k = 0; k < K; ++k) {
            float v = w[n * ldw + k];
            if (!isfinite(v)) return ORC_ERR_NONFINITE;
            uint32_t u = f32_bits(v) & 0x7FFFFFFFu;
            uint32_t e = u >> 23;
            uint64_t mant = (uint64_t)(u & 0x7FFFFFu) | (e ? 0x800000u : 0u);
            if (bins[e] > UINT64_MAX - mant) return ORC_ERR_OVERFLOW;
            bins[e] += mant;
        }
    }
    return ORC_OK;
}

/* Ternary codes given alpha:  t = RoundClip(w / (alpha + eps), -1, 1). */
int orc_ternary_codes(const float* w, int64_t N, int64_t K, int64_t ldw, float alpha, float eps,
                      int8_t* t) {
    if (N < 0 || K <= 0 || ldw < K) return ORC_ERR_ARG;
    float denom = alpha + eps;
    for (int64_t n = 0; n < N; ++n)
        for (int64_t k = 0; k < K; ++k)
            t[n * K + k] = (int8_t)round_clip(w[n * ldw + k] / denom, -1.0f, 1.0f);
    return ORC_OK;
}

/* ---------------------------------------------------------------------------
 * BitLinear matmul (§3.4, Y = Q_x(X) . Q_w(W)^T, Eq. 1 and the equation above
 * Eq. 6): integer accumulation of codes, then per-token x per-tensor dequant.
 *   acc[m,n] = sum_k a[m,k] * t[n,k]            (exact, int64, checked to fit int32)
 *   y[m,n]   = bf16( acc * a_scale[m] * alpha[n / alpha_group] )   (fp64, rounded once)
 * `rows` (nullable) selects which rows of A to compute; outputs are then
 * [n_rows x N].  acc_out / y_out are nullable.
 * ------------------------------------------------------------------------- */
int orc_gemm(const int8_t* a, int64_t lda, const float* a_scale, const int8_t* t, const float* alpha,
             int64_t alpha_group, int64_t M, int64_t N, int64_t K, const int64_t* rows, int64_t n_rows,
             int32_t* acc_out, uint16_t* y_out) {
    if (M < 0 || N <= 0 || K <= 0 || lda < K || alpha_group <= 0) return ORC_ERR_ARG;
    int64_t R = rows ? n_rows : M;
    for (int64_t r = 0; r < R; ++r) {
        int64_t m = rows ? rows[r] : r;
        if (m < 0 || m >= M) return ORC_ERR_ARG;
        const int8_t* ar = a + m * lda;
        for (int64_t n = 0; n < N; ++n) {
            const int8_t* tr = t + n * K;
            int64_t acc = 0;
            for (int64_t k = 0; k < K; ++k) acc += (int64_t)ar[k] * (int64_t)tr[k];
            if (acc > INT32_MAX || acc < INT32_MIN) return ORC_ERR_OVERFLOW;
            if (acc_out) acc_out[r * N + n] = (int32_t)acc;
            if (y_out) {
                double yv = (double)acc * (double)a_scale[m] * (double)alpha[n / alpha_group];
                y_out[r * N + n] = bf16_round(yv);
            }
        }
    }
    return ORC_OK;
}

/* ---------------------------------------------------------------------------
 * Post-RoPE low-bit KV quantizer (§3.4 "Low-Bit KV Cache Quantization"):
 * absmax per (position, head) vector of D values, to unsigned b-bit integers.
 * Reading: symmetric absmax with Q = 2^(b-1) - 1,
 *   c = RoundClip(Q/(gamma+eps) * x, -Q-1, Q),  stored unsigned as c + 2^(b-1),
 *   dequant scale gamma/Q.
 * For 3-bit caches the beginning-of-sequence position `bos_pos` is kept at 4
 * bits (bos_pos = -1: none).  kv is [T x H x D] with a stride of `ldt` values
 * between consecutive positions.  codes_u: [T x H x D] unsigned codes (the
 * BOS row carries its 4-bit codes); scale: [T x H].
 * ------------------------------------------------------------------------- */
int orc_kv_quant(const uint16_t* kv, int64_t T, int64_t H, int64_t D, int64_t ldt, int bits,
                 int64_t bos_pos, float eps, uint8_t* codes_u, float* scale) {
    if (T < 0 || H <= 0 || D <= 0 || ldt < H * D || (bits != 3 && bits != 4)) return ORC_ERR_ARG;
    for (int64_t t = 0; t < T; ++t) {
        int b = (t == bos_pos) ? 4 : bits;
        float q = (float)((1 << (b - 1)) - 1);
        int offset = 1 << (b - 1);
        for (int64_t h = 0; h < H; ++h) {
            const uint16_t* v = kv + t * ldt + h * D;
            float gamma = 0.0f;
            for (int64_t d = 0; d < D; ++d) {
                float a = fabsf(bf16_value(v[d]));
                if (!isfinite(a)) return ORC_ERR_NONFINITE;
                if (a > gamma) gamma = a;
            }
            float mult = q / (gamma + eps);
            for (int64_t d = 0; d < D; ++d) {
                float c = round_clip(bf16_value(v[d]) * mult, -q - 1.0f, q);
                codes_u[(t * H + h) * D + d] = (uint8_t)((int)c + offset);
            }
            scale[t * H + h] = gamma / q;
        }
    }
    return ORC_OK;
}

/* ---------------------------------------------------------------------------
 * RMSNorm ahead of the 4-bit quantizer (§3.2's per-layer data flow: RMSNorm ->
 * 4-bit quantize -> QKV / Up|Gate BitLinear).  The pages name the step without
 * a formula; the reading used is the usual root-mean-square normalization with
 * a per-channel weight, its output an activation tensor in bf16 like every
 * other one:
 *   ms = mean(x^2) over the row,  s = sqrt(ms + eps_n),  r = 1 / s,
 *   y_k = bf16( (x_k * r) * g_k )      (g_k = 1 without a weight).
 * The arithmetic is fixed so that it can be reproduced exactly: ms is the exact
 * mean of the squares rounded once to fp32 (order-free); ms + eps_n, the square
 * root, 1 / s and the two products are single IEEE fp32 operations, each
 * rounded to nearest even; the last result is rounded once to bf16.
 *
 * orc_rmsnorm_sumsq gives the exact sum of squares of each row as an unevaluated
 * pair hi + lo of doubles (the caller divides and rounds with exact rationals).
 * Each x^2 is exact in fp64; the pair is a double-double accumulation whose
 * every step is checked to be exact (TwoSum), and the row is rejected unless
 * the squares, as multiples of the smallest one's last significant bit, stay
 * below 2^90 in sum -- then a double-double accumulation in any order (and any
 * grouping, up to 16384 terms) is exact as well.
 * orc_rmsnorm_apply takes ms and forms y and r.
 * ------------------------------------------------------------------------- */
static void two_sum(double a, double b, double* s, double* e) {
    double t = a + b;
    double bp = t - a;
    *e = (a - (t - bp)) + (b - bp);
    *s = t;
}

int orc_rmsnorm_sumsq(const uint16_t* x, int64_t M, int64_t K, int64_t ldx, double* hi_out, double* lo_out) {
    if (M < 0 || K <= 0 || ldx < K) return ORC_ERR_ARG;
    for (int64_t m = 0; m < M; ++m) {
        const uint16_t* row = x + m * ldx;
        double hi = 0.0, lo = 0.0;
        int lowbit = INT32_MAX;            /* exponent of the lowest significant bit over the squares */
        for (int64_t k = 0; k < K; ++k) {
            double v = (double)bf16_value(row[k]);
            if (!isfinite(v)) return ORC_ERR_NONFINITE;
            double a = v * v;              /* exact: an 8-bit significand squared, within fp64's range */
            if (a != 0.0) {
                int e;
                double f = frexp(a, &e);   /* a = f * 2^e, f in [0.5, 1) */
                int b = e - 53;            /* a = (f * 2^53) * 2^b with f * 2^53 an integer */
                double n = ldexp(f, 53);
                while (fmod(n, 2.0) == 0.0) { n /= 2.0; ++b; }
                if (b < lowbit) lowbit = b;
            }
            double t, e1, e2;
            two_sum(hi, a, &t, &e1);
            two_sum(lo, e1, &lo, &e2);
            if (e2 != 0.0) return ORC_ERR_INEXACT_SUM;
            hi = t;
        }
        if (hi != 0.0) {
            int e;
            frexp(hi + lo, &e);            /* the sum is below 2^e (within a rounding) */
            if (e - lowbit > 90) return ORC_ERR_INEXACT_SUM;
        }
        hi_out[m] = hi;
        lo_out[m] = lo;
    }
    return ORC_OK;
}

int orc_rmsnorm_apply(const uint16_t* x, int64_t M, int64_t K, int64_t ldx, const float* ms, const float* g,
                      float eps_n, uint16_t* y, float* r_out) {
    if (M < 0 || K <= 0 || ldx < K || !(eps_n > 0.0f)) return ORC_ERR_ARG;
    for (int64_t m = 0; m < M; ++m) {
        const uint16_t* row = x + m * ldx;
        float s = sqrtf(ms[m] + eps_n);
        float r = 1.0f / s;
        for (int64_t k = 0; k < K; ++k) {
            float t = bf16_value(row[k]) * r;
            if (g) t = t * g[k];
            y[m * K + k] = bf16_round((double)t);
        }
        r_out[m] = r;
    }
    return ORC_OK;
}

/* ---------------------------------------------------------------------------
 * INT4 absmean with one scale for the whole tensor (the per-tensor scaling of
 * the ablations, Fig. 5 / Fig. 6; also the literal reading of Eq. 6-7, whose
 * mean runs over all entries of X): the same codes as orc_quant_int4 but with
 * a given beta, the exact mean of |X| over all M*K entries rounded once to fp32
 * (the caller forms it from orc_ternary_abs_bins on the exact fp32 values).
 * ------------------------------------------------------------------------- */
int orc_quant_int4_given_beta(const uint16_t* x, int64_t M, int64_t K, int64_t ldx, float beta, float eps,
                              int8_t* codes, float* scale_out) {
    if (M < 0 || K <= 0 || ldx < K) return ORC_ERR_ARG;
    const float sqrt7 = (float)sqrt(7.0);
    const float mult = sqrt7 / (beta + eps);
    for (int64_t m = 0; m < M; ++m) {
        const uint16_t* row = x + m * ldx;
        for (int64_t k = 0; k < K; ++k) {
            float v = bf16_value(row[k]);
            if (!isfinite(v)) return ORC_ERR_NONFINITE;
            codes[m * K + k] = (int8_t)round_clip(v * mult, -8.0f, 7.0f);
        }
        scale_out[m] = beta / sqrt7;
    }
    return ORC_OK;
}

/* The rounding mode every function above assumes. */
int orc_rounding_is_nearest(void) { return fegetround() == FE_TONEAREST; }
