/*
 * nf4_oracle.c -- plain, slow, obviously-correct CPU oracle for QLoRA's NF4
 * blockwise quantization, double quantization, dequantization and the
 * frozen-base LoRA linear.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product path links, loads or
 * calls this file: only the tests, the package's smoke check and the
 * benchmark's CPU-baseline leg do.  It shares no code, header, table or
 * constant generator with the CUDA library; the two are compared on the same
 * seeded inputs.
 *
 * Sources (web pages; cited by title and section):
 *   [MF] "QLoRA: Mathematical Foundations of 4-Bit NormalFloat Quantization,
 *        Double Quantization, and Paged Optimizers" (llms.blog)
 *   [L15] "Lesson 15. NF4 and Double Quantisation" (tokencemetery)
 *   [QP] "QLoRA in Production: 4-bit NormalFloat & Double Quantization Deep
 *        Dive" (devtechtools.org)
 *   [AD] "QLoRA: quantising the part you are not training" (addaly.com)
 *
 * Arithmetic: strict IEEE binary32/binary64, round-to-nearest-even.  Build
 * with -O2 -ffp-contract=off and no fast-math; the only fused multiply-add is
 * the explicit fmaf() of the double-quantization decode.  Where the pages fix
 * the precision (fp32 block constants, fp32 codebook, bf16 compute) that
 * precision is used; everything else (sums, the linear) is fp64.
 *
 * Readings of points the pages leave open are marked READING and listed in
 * the design notes: tie rule, all-zero block, nibble order, FP8 format,
 * centring mean and its summation order, decode rounding.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

/* ------------------------------------------------------------------------ */
/* Codebook                                                                  */
/* ------------------------------------------------------------------------ */

/* [MF] section "4-Bit NormalFloat (NF4): Information-Theoretic Quantile
 * Quantization", the list of the sixteen codebook values q_0..q_15.  Typed in
 * from the page; every printed decimal is an exact binary32 value. */
static const float NF4_LEVELS[16] = {
    -1.0f,
    -0.6961928009986877f,
    -0.5250730514526367f,
    -0.39491748809814453f,
    -0.28444138169288635f,
    -0.18477343022823334f,
    -0.09105003625154495f,
    0.0f,
    0.07958029955625534f,
    0.16093020141124725f,
    0.24611230194568634f,
    0.33791524171829224f,
    0.44070982933044434f,
    0.5626170039176941f,
    0.7229568362236023f,
    1.0f,
};

void nf4o_codebook(float out[16]) { memcpy(out, NF4_LEVELS, sizeof NF4_LEVELS); }

/* Standard normal CDF, Phi(x) = erfc(-x / sqrt 2) / 2 (textbook identity; the
 * C library's erfc is the primitive). */
static double std_normal_cdf(double x) { return 0.5 * erfc(-x / sqrt(2.0)); }

/* Inverse standard normal CDF Q(p) for 0 < p < 1 by plain bisection on the
 * monotone Phi over the lower half [-40, 0], where erfc is evaluated at a
 * non-negative argument and keeps full relative accuracy; the upper half
 * follows from the symmetry Q(p) = -Q(1 - p) (1 - p is exact for p >= 1/2).
 * The loop stops when the bracket can no longer shrink. */
double nf4o_norm_ppf(double p) {
    if (p == 0.5) return 0.0;
    double tail = p < 0.5 ? p : 1.0 - p;
    double lo = -40.0, hi = 0.0;
    for (int it = 0; it < 2000; ++it) {
        double mid = 0.5 * (lo + hi);
        if (mid == lo || mid == hi) break;
        if (std_normal_cdf(mid) < tail) lo = mid; else hi = mid;
    }
    double x = 0.5 * (lo + hi);
    return p < 0.5 ? x : -x;
}

/* Construction of the sixteen levels, [MF] section "4-Bit NormalFloat (NF4)",
 * the asymmetric partition: 8 positive levels from quantiles of the positive
 * half split into 16 intervals, 7 negative levels from the negative half
 * split into 14 intervals, an exact zero, all divided by the largest
 * magnitude so the ends are -1 and +1.
 * READING: the pages do not give the outermost probability (Q(1) is
 * infinite).  With delta the outermost probability, the quantile points are
 * p_j = delta - j (delta - 1/2) / 8, j = 0..7 (positive side) and
 * p_j = delta - j (delta - 1/2) / 7, j = 0..6 (negative side, mirrored).
 * The caller passes delta; the tests use delta = 1 - (1/30 + 1/32) / 2, the
 * mean of the outermost half-bin points of 15- and 16-way equal-mass splits,
 * and check the result against the printed table. */
void nf4o_codebook_construct(double delta, double out[16]) {
    double v[16], neg[7], pos[8];
    for (int j = 0; j < 7; ++j) neg[j] = -nf4o_norm_ppf(delta - j * (delta - 0.5) / 7.0);
    for (int j = 0; j < 8; ++j) pos[j] = nf4o_norm_ppf(delta - j * (delta - 0.5) / 8.0);
    /* ascending order: j = 0 is the outermost point on each side */
    int k = 0;
    for (int j = 0; j < 7; ++j) v[k++] = neg[j];
    v[k++] = 0.0;
    for (int j = 7; j >= 0; --j) v[k++] = pos[j];
    double vmax = 0.0;
    for (int i = 0; i < 16; ++i) if (fabs(v[i]) > vmax) vmax = fabs(v[i]);
    for (int i = 0; i < 16; ++i) out[i] = v[i] / vmax;
}

/* ------------------------------------------------------------------------ */
/* bf16 and FP8 E4M3 scalar formats                                          */
/* ------------------------------------------------------------------------ */

static float f32_of_bits(uint32_t u) { float f; memcpy(&f, &u, 4); return f; }
static uint32_t bits_of_f32(float f) { uint32_t u; memcpy(&u, &f, 4); return u; }

float nf4o_bf16_to_f32(uint16_t h) { return f32_of_bits((uint32_t)h << 16); }

/* binary32 -> bfloat16, round to nearest, ties to even (finite inputs; NaN
 * maps to a quiet NaN).  bfloat16 keeps the top 16 bits of binary32; the
 * discarded 16 bits decide the rounding. */
uint16_t nf4o_f32_to_bf16(float f) {
    uint32_t u = bits_of_f32(f);
    if ((u & 0x7F800000u) == 0x7F800000u && (u & 0x007FFFFFu)) return (uint16_t)((u >> 16) | 0x40u);
    uint32_t keep = u >> 16, rest = u & 0xFFFFu;
    if (rest > 0x8000u || (rest == 0x8000u && (keep & 1u))) keep += 1u;
    return (uint16_t)keep;
}

/* OCP 8-bit floating point E4M3 ("FN" variant: no infinities, one NaN
 * pattern per sign): 1 sign bit, 4 exponent bits with bias 7, 3 mantissa
 * bits; exponent field 0 is subnormal (m/8 * 2^-6); S.1111.111 is NaN; the
 * largest finite magnitude is 448.  Decoded exactly in binary64. */
double nf4o_e4m3_decode(uint8_t c) {
    int s = c >> 7, e = (c >> 3) & 15, m = c & 7;
    double v;
    if (e == 15 && m == 7) return NAN;
    if (e == 0) v = ldexp((double)m, -9);
    else v = ldexp(1.0 + m / 8.0, e - 7);
    return s ? -v : v;
}

/* Encode to E4M3 by brute force: the finite magnitude nearest to |y|, ties to
 * the code with an even mantissa, magnitudes above 448 saturate to 448
 * (READING: "quantize_FP8" of [MF] section "Double Quantization (DQ)" taken as
 * round-to-nearest-even E4M3 with saturation; its inputs lie in [-1, 1] so
 * saturation never occurs in the method).  The sign of y (zero included) is
 * kept. */
uint8_t nf4o_e4m3_encode(float y) {
    double a = fabs((double)y);
    int best = 0;
    double bd = INFINITY;
    for (int c = 0; c <= 126; ++c) {
        double d = fabs(a - nf4o_e4m3_decode((uint8_t)c));
        if (d < bd || (d == bd && (c & 1) == 0)) { bd = d; best = c; }
    }
    if (a > 448.0) best = 126;
    return (uint8_t)((signbit(y) ? 0x80 : 0) | best);
}

/* ------------------------------------------------------------------------ */
/* Blockwise NF4 quantization                                                */
/* ------------------------------------------------------------------------ */

/* Nearest codebook level, [MF] section "Block-Wise Quantization Mechanics",
 * the arg-min equation over i in 0..15 of |w_j / c1 - q_i|.
 * READING: an exact tie between two levels goes to the lower index (first
 * minimum).  Distances are formed in binary64, which is exact here: for
 * |x| >= 2^-29 both x and every q_i are multiples of 2^-52 below 2, and for
 * smaller |x| the nearest level is the exact zero by a margin of 0.079. */
int nf4o_code_of(float x) {
    int best = 0;
    double bd = fabs((double)x - (double)NF4_LEVELS[0]);
    for (int i = 1; i < 16; ++i) {
        double d = fabs((double)x - (double)NF4_LEVELS[i]);
        if (d < bd) { bd = d; best = i; }
    }
    return best;
}

/* Quantize a flattened fp32 tensor w[0..n) in contiguous blocks of bs
 * elements ([MF] section "Block-Wise Quantization Mechanics": contiguous 1-D
 * blocks, c1 = max_j |w_j| kept in fp32, code = nearest level of w_j / c1 with
 * the quotient rounded to binary32).  The final block may be shorter.
 * READING: an all-zero block (c1 = 0) codes every element as the exact zero,
 * level 7.  READING (packing): two codes per byte, element 2j in the high
 * nibble and element 2j+1 in the low nibble; n must be even.
 * packed[n/2], absmax[ceil(n/bs)]. */
void nf4o_quantize_f32(const float *w, int64_t n, int bs, uint8_t *packed, float *absmax) {
    int64_t nb = (n + bs - 1) / bs;
    for (int64_t b = 0; b < nb; ++b) {
        int64_t lo = b * bs, hi = lo + bs < n ? lo + bs : n;
        float c1 = 0.0f;
        for (int64_t j = lo; j < hi; ++j) {
            float a = fabsf(w[j]);
            if (a > c1) c1 = a;
        }
        absmax[b] = c1;
        for (int64_t j = lo; j < hi; ++j) {
            int code = (c1 == 0.0f) ? 7 : nf4o_code_of(w[j] / c1);
            if ((j & 1) == 0) packed[j >> 1] = (uint8_t)(code << 4);
            else packed[j >> 1] = (uint8_t)(packed[j >> 1] | code);
        }
    }
}

/* Same, for a bfloat16 tensor (each element widened exactly to binary32). */
void nf4o_quantize_bf16(const uint16_t *w, int64_t n, int bs, uint8_t *packed, float *absmax) {
    float *wf = (float *)malloc((size_t)(n > 0 ? n : 1) * sizeof(float));
    for (int64_t j = 0; j < n; ++j) wf[j] = nf4o_bf16_to_f32(w[j]);
    nf4o_quantize_f32(wf, n, bs, packed, absmax);
    free(wf);
}

/* ------------------------------------------------------------------------ */
/* Double quantization of the block constants                                */
/* ------------------------------------------------------------------------ */

/* Centring mean of the first-level constants.
 * READING: [MF] section "Double Quantization (DQ)" speaks of "an asymmetric
 * bias/mean subtraction" without a formula; the reading is one fp32 mean per
 * tensor, mu = RN_f32( S / nb ), with S a fixed-order binary64 sum:
 *   1. each run of dqbs consecutive constants (the last may be shorter) is
 *      summed sequentially in index order starting from 0;
 *   2. the run sums are combined level by level, s[j] = s[2j] + s[2j+1], an
 *      odd last element carried up unchanged, until one value remains;
 *   3. S / nb is rounded to binary64, then to binary32. */
/* Step 1 alone: s[d] = sequential binary64 sum of run d, d < ceil(nb/dqbs).
 * For a tensor split into shards on run boundaries, the concatenation of the
 * shards' run sums is the run-sum array of the whole tensor. */
void nf4o_dq_run_sums(const float *c1, int64_t nb, int dqbs, double *s) {
    int64_t nd = (nb + dqbs - 1) / dqbs;
    for (int64_t d = 0; d < nd; ++d) {
        int64_t lo = d * dqbs, hi = lo + dqbs < nb ? lo + dqbs : nb;
        double acc = 0.0;
        for (int64_t k = lo; k < hi; ++k) acc += (double)c1[k];
        s[d] = acc;
    }
}

/* Steps 2 and 3 on a run-sum array of nd entries (not modified) for a
 * tensor of nb constants. */
float nf4o_dq_mean_from_run_sums(const double *run_sums, int64_t nd, int64_t nb) {
    if (nb <= 0 || nd <= 0) return 0.0f;
    double *s = (double *)malloc((size_t)nd * sizeof(double));
    memcpy(s, run_sums, (size_t)nd * sizeof(double));
    int64_t len = nd;
    while (len > 1) {
        int64_t half = len / 2;
        for (int64_t j = 0; j < half; ++j) s[j] = s[2 * j] + s[2 * j + 1];
        if (len & 1) s[half] = s[len - 1];
        len = half + (len & 1);
    }
    double mean = s[0] / (double)nb;
    free(s);
    return (float)mean;
}

float nf4o_dq_mean(const float *c1, int64_t nb, int dqbs) {
    if (nb <= 0) return 0.0f;
    int64_t nd = (nb + dqbs - 1) / dqbs;
    double *s = (double *)malloc((size_t)nd * sizeof(double));
    nf4o_dq_run_sums(c1, nb, dqbs, s);
    float mu = nf4o_dq_mean_from_run_sums(s, nd, nb);
    free(s);
    return mu;
}

/* Double quantization, [MF] section "Double Quantization (DQ)": the fp32
 * constants are grouped in runs of dqbs (the last may be shorter); per run
 * c2 = max |c1 - mu| in fp32, and each constant is stored as the 8-bit float
 * code of (c1 - mu) / c2 (both operations binary32, round to nearest).
 * centre = 0 gives mu = 0 (the displayed formula taken literally);
 * centre = 1 subtracts the mean above.  A run whose centred values are all
 * zero (c2 = 0) stores code 0x00.  codes[nb], absmax2[ceil(nb/dqbs)],
 * *offset = mu (if offset is not NULL). */
/* The runs of the double quantization with a given mean mu (the tensor's
 * mean; for a shard of a tensor, the whole tensor's). */
void nf4o_double_quantize_with_mean(const float *c1, int64_t nb, int dqbs, float mu, uint8_t *codes,
                                    float *absmax2) {
    int64_t nd = (nb + dqbs - 1) / dqbs;
    for (int64_t d = 0; d < nd; ++d) {
        int64_t lo = d * dqbs, hi = lo + dqbs < nb ? lo + dqbs : nb;
        float c2 = 0.0f;
        for (int64_t k = lo; k < hi; ++k) {
            float a = fabsf(c1[k] - mu);
            if (a > c2) c2 = a;
        }
        absmax2[d] = c2;
        for (int64_t k = lo; k < hi; ++k)
            codes[k] = (c2 == 0.0f) ? 0x00 : nf4o_e4m3_encode((c1[k] - mu) / c2);
    }
}

void nf4o_double_quantize(const float *c1, int64_t nb, int dqbs, int centre,
                          uint8_t *codes, float *absmax2, float *offset) {
    float mu = centre ? nf4o_dq_mean(c1, nb, dqbs) : 0.0f;
    if (offset) *offset = mu;
    nf4o_double_quantize_with_mean(c1, nb, dqbs, mu, codes, absmax2);
}

/* ------------------------------------------------------------------------ */
/* Dequantization                                                            */
/* ------------------------------------------------------------------------ */

/* Reconstructed first-level constant of block b.
 * With double quantization (codes != NULL): READING, the stored 8-bit value
 * times c2 plus the mean, with one rounding: c1' = fma(dec(code), c2, mu);
 * without a mean (offset == NULL) c1' = dec(code) * c2.  Without double
 * quantization (codes == NULL) scales[] holds the fp32 c1 themselves. */
static float block_constant(const uint8_t *codes, const float *scales, const float *offset,
                            int64_t b, int dqbs) {
    if (!codes) return scales[b];
    float dec = (float)nf4o_e4m3_decode(codes[b]);
    float c2 = scales[b / dqbs];
    if (offset) return fmaf(dec, c2, *offset);
    return dec * c2;
}

/* [MF] section "Block-Wise Quantization Mechanics", the dequantization
 * equation w~_j = c1 * q[code_j], one binary32 multiply.  out[n] fp32. */
void nf4o_dequantize_f32(const uint8_t *packed, const uint8_t *codes, const float *scales,
                         const float *offset, int64_t n, int bs, int dqbs, float *out) {
    int64_t nb = (n + bs - 1) / bs;
    for (int64_t b = 0; b < nb; ++b) {
        float c = block_constant(codes, scales, offset, b, dqbs);
        int64_t lo = b * bs, hi = lo + bs < n ? lo + bs : n;
        for (int64_t j = lo; j < hi; ++j) {
            int code = (j & 1) ? (packed[j >> 1] & 15) : (packed[j >> 1] >> 4);
            out[j] = NF4_LEVELS[code] * c;
        }
    }
}

/* bf16 output: the fp32 reconstruction rounded to nearest-even bfloat16
 * (compute dtype bf16: [MF] "Forward Pass Computation"; [AD] "What it costs",
 * weights dequantised to bf16 on the fly). */
void nf4o_dequantize_bf16(const uint8_t *packed, const uint8_t *codes, const float *scales,
                          const float *offset, int64_t n, int bs, int dqbs, uint16_t *out) {
    float *f = (float *)malloc((size_t)(n > 0 ? n : 1) * sizeof(float));
    nf4o_dequantize_f32(packed, codes, scales, offset, n, bs, dqbs, f);
    for (int64_t j = 0; j < n; ++j) out[j] = nf4o_f32_to_bf16(f[j]);
    free(f);
}

/* ------------------------------------------------------------------------ */
/* Frozen-base LoRA linear                                                   */
/* ------------------------------------------------------------------------ */

/* [MF] section "Forward Pass Computation":
 *   Y = X dequant(W) + (alpha / r) (X L1) L2
 * in the weight layout W[N, K] (row n is output feature n), A[r, K] (= L1
 * transposed), B[N, r] (= L2 transposed), s = alpha / r:
 *   y[m, n] = sum_k x[m, k] w[n, k] + s * sum_j (sum_k x[m, k] A[j, k]) B[n, j]
 * with w the bf16-rounded dequantized weight (compute dtype bf16) and every
 * sum formed in binary64 (the products of bf16 values are exact there).
 * Only the rows listed in rows[0..nrows) are computed; y is [nrows, N].
 * A or B NULL (or r = 0) drops the low-rank term. */
void nf4o_lora_linear(const uint16_t *x, int64_t M, int64_t K, int64_t N,
                      const uint8_t *packed, const uint8_t *codes, const float *scales,
                      const float *offset, int bs, int dqbs,
                      const uint16_t *A, const uint16_t *B, int r, float s,
                      const int64_t *rows, int64_t nrows, double *y) {
    (void)M;
    int lora = (A != NULL && B != NULL && r > 0);
    double *xr = (double *)malloc((size_t)(nrows * K > 0 ? nrows * K : 1) * sizeof(double));
    for (int64_t i = 0; i < nrows; ++i)
        for (int64_t k = 0; k < K; ++k) xr[i * K + k] = nf4o_bf16_to_f32(x[rows[i] * K + k]);
    double *t = NULL;
    if (lora) {
        t = (double *)malloc((size_t)(nrows * r > 0 ? nrows * r : 1) * sizeof(double));
        for (int64_t i = 0; i < nrows; ++i)
            for (int j = 0; j < r; ++j) {
                double acc = 0.0;
                for (int64_t k = 0; k < K; ++k) acc += xr[i * K + k] * nf4o_bf16_to_f32(A[(int64_t)j * K + k]);
                t[i * r + j] = acc;
            }
    }
#pragma omp parallel
    {
        float *wf = (float *)malloc((size_t)(K > 0 ? K : 1) * sizeof(float));
        double *wb = (double *)malloc((size_t)(K > 0 ? K : 1) * sizeof(double));
#pragma omp for schedule(static)
        for (int64_t nn = 0; nn < N; ++nn) {
            /* dequantize row nn: K is a multiple of bs, so the row starts a block */
            int64_t base = nn * K;
            for (int64_t k = 0; k < K; ++k) {
                int64_t j = base + k, b = j / bs;
                float c = block_constant(codes, scales, offset, b, dqbs);
                int code = (j & 1) ? (packed[j >> 1] & 15) : (packed[j >> 1] >> 4);
                wf[k] = NF4_LEVELS[code] * c;
                wb[k] = nf4o_bf16_to_f32(nf4o_f32_to_bf16(wf[k]));
            }
            for (int64_t i = 0; i < nrows; ++i) {
                double acc = 0.0;
                for (int64_t k = 0; k < K; ++k) acc += xr[i * K + k] * wb[k];
                if (lora) {
                    double lo = 0.0;
                    for (int j = 0; j < r; ++j) lo += t[i * r + j] * nf4o_bf16_to_f32(B[nn * r + j]);
                    acc += (double)s * lo;
                }
                y[i * N + nn] = acc;
            }
        }
        free(wf);
        free(wb);
    }
    free(xr);
    free(t);
}

/* ------------------------------------------------------------------------ */
/* Backward pass through the frozen base                                     */
/* ------------------------------------------------------------------------ */

/* [MF] section "Gradient Computation" (after "Forward Pass Computation"):
 * gradients go to the adapter only, and the activation gradient flows through
 * both paths.  In the weight layout used here (W[N, K], L1 = A^T, L2 = B^T,
 * w the bf16 dequantized weight) and with g = dL/dy [M, N]:
 *   dx[m, k] = sum_n g[m, n] w[n, k] + s sum_j u[m, j] A[j, k],
 *              u[m, j] = sum_n g[m, n] B[n, j]
 *   dA[j, k] = s sum_m u[m, j] x[m, k]
 *   dB[n, j] = s sum_m g[m, n] t[m, j],  t[m, j] = sum_k x[m, k] A[j, k]
 * Every sum in binary64 (products of bf16 values are exact there); u and t are
 * kept unrounded.  dx is computed for the token rows rows[0..nrows) only
 * ([nrows, K]); dA ([r, K]) and dB ([N, r]) use all M rows; any output may be
 * NULL.  x may be NULL when dA and dB are. */
void nf4o_lora_linear_bwd(const uint16_t *g, const uint16_t *x, int64_t M, int64_t K, int64_t N,
                          const uint8_t *packed, const uint8_t *codes, const float *scales,
                          const float *offset, int bs, int dqbs,
                          const uint16_t *A, const uint16_t *B, int r, float s,
                          const int64_t *rows, int64_t nrows, double *dx, double *dA, double *dB) {
    int lora = (A != NULL && B != NULL && r > 0);
    double *u = NULL, *t = NULL;
    if (lora) {
        u = (double *)calloc((size_t)(M * r > 0 ? M * r : 1), sizeof(double));
#pragma omp parallel for schedule(static)
        for (int64_t m = 0; m < M; ++m)
            for (int64_t n = 0; n < N; ++n) {
                double gv = nf4o_bf16_to_f32(g[m * N + n]);
                for (int j = 0; j < r; ++j) u[m * r + j] += gv * nf4o_bf16_to_f32(B[n * r + j]);
            }
    }
    if (dx) {
        for (int64_t i = 0; i < nrows * K; ++i) dx[i] = 0.0;
        float *wf = (float *)malloc((size_t)(K > 0 ? K : 1) * sizeof(float));
        for (int64_t n = 0; n < N; ++n) {
            for (int64_t k = 0; k < K; ++k) {
                int64_t j = n * K + k;
                float c = block_constant(codes, scales, offset, j / bs, dqbs);
                int code = (j & 1) ? (packed[j >> 1] & 15) : (packed[j >> 1] >> 4);
                wf[k] = nf4o_bf16_to_f32(nf4o_f32_to_bf16(NF4_LEVELS[code] * c));
            }
#pragma omp parallel for schedule(static)
            for (int64_t i = 0; i < nrows; ++i) {
                double gv = nf4o_bf16_to_f32(g[rows[i] * N + n]);
                if (gv != 0.0)
                    for (int64_t k = 0; k < K; ++k) dx[i * K + k] += gv * (double)wf[k];
            }
        }
        free(wf);
        if (lora)
#pragma omp parallel for schedule(static)
            for (int64_t i = 0; i < nrows; ++i)
                for (int64_t k = 0; k < K; ++k) {
                    double acc = 0.0;
                    for (int j = 0; j < r; ++j) acc += u[rows[i] * r + j] * nf4o_bf16_to_f32(A[(int64_t)j * K + k]);
                    dx[i * K + k] += (double)s * acc;
                }
    }
    if (lora && dA)
#pragma omp parallel for schedule(static)
        for (int64_t k = 0; k < K; ++k)
            for (int j = 0; j < r; ++j) {
                double acc = 0.0;
                for (int64_t m = 0; m < M; ++m) acc += u[m * r + j] * nf4o_bf16_to_f32(x[m * K + k]);
                dA[(int64_t)j * K + k] = (double)s * acc;
            }
    if (lora && dB) {
        t = (double *)malloc((size_t)(M * r > 0 ? M * r : 1) * sizeof(double));
#pragma omp parallel for schedule(static)
        for (int64_t m = 0; m < M; ++m)
            for (int j = 0; j < r; ++j) {
                double acc = 0.0;
                for (int64_t k = 0; k < K; ++k) acc += nf4o_bf16_to_f32(x[m * K + k]) * nf4o_bf16_to_f32(A[(int64_t)j * K + k]);
                t[m * r + j] = acc;
            }
#pragma omp parallel for schedule(static)
        for (int64_t n = 0; n < N; ++n)
            for (int j = 0; j < r; ++j) {
                double acc = 0.0;
                for (int64_t m = 0; m < M; ++m) acc += nf4o_bf16_to_f32(g[m * N + n]) * t[m * r + j];
                dB[n * r + j] = (double)s * acc;
            }
    }
    free(u);
    free(t);
}

/* ------------------------------------------------------------------------ */
/* Merging the adapter into the quantized base, then requantizing            */
/* ------------------------------------------------------------------------ */

/* [QP] section "Step 4: Merging and Inference" merges the trained adapter into
 * the quantized base for deployment; [AD] section "What it costs" (item 3,
 * "Merging is awkward") notes that a merge into the quantized base must be
 * requantized, with its own error.  The pages give no arithmetic.  READING:
 * the merge is formed in binary32 on the exact dequantized weight,
 *   d[n, k]  = B[n, 0] A[0, k] + ... + B[n, r-1] A[r-1, k] as the chain
 *              d <- fma(B[n, j], A[j, k], d), j = 0, 1, ..., r - 1, from +0
 *   W'[n, k] = fma(s, d[n, k], w~[n, k])
 * (A, B bf16 widened exactly; w~ as in nf4o_dequantize_f32).  Rows
 * row0 .. row0 + nrows - 1 of W[N, K]; out is [nrows, K]. */
void nf4o_merge_weight(const uint8_t *packed, const uint8_t *codes, const float *scales,
                       const float *offset, int64_t K, int bs, int dqbs,
                       const uint16_t *A, const uint16_t *B, int r, float s,
                       int64_t row0, int64_t nrows, float *out) {
    for (int64_t i = 0; i < nrows; ++i) {
        int64_t nn = row0 + i;
        for (int64_t k = 0; k < K; ++k) {
            int64_t j = nn * K + k;
            float c = block_constant(codes, scales, offset, j / bs, dqbs);
            int code = (j & 1) ? (packed[j >> 1] & 15) : (packed[j >> 1] >> 4);
            float w = NF4_LEVELS[code] * c;
            float d = 0.0f;
            for (int q = 0; q < r; ++q)
                d = fmaf(nf4o_bf16_to_f32(B[nn * r + q]), nf4o_bf16_to_f32(A[(int64_t)q * K + k]), d);
            out[i * K + k] = fmaf(s, d, w);
        }
    }
}

/* The merged rows quantized again by the blockwise NF4 of nf4o_quantize_f32
 * (K is a multiple of bs, so every block lies inside one row):
 * packed_out [nrows K / 2], absmax_out [nrows K / bs], the fp32 constants of
 * W' (double-quantizing them is the separate step nf4o_double_quantize). */
void nf4o_merge_requantize(const uint8_t *packed, const uint8_t *codes, const float *scales,
                           const float *offset, int64_t K, int bs, int dqbs,
                           const uint16_t *A, const uint16_t *B, int r, float s,
                           int64_t row0, int64_t nrows, uint8_t *packed_out, float *absmax_out) {
    float *wm = (float *)malloc((size_t)(nrows * K > 0 ? nrows * K : 1) * sizeof(float));
    nf4o_merge_weight(packed, codes, scales, offset, K, bs, dqbs, A, B, r, s, row0, nrows, wm);
    nf4o_quantize_f32(wm, nrows * K, bs, packed_out, absmax_out);
    free(wm);
}

/* ------------------------------------------------------------------------ */
/* Array forms of the scalar routines (loops only, for the tests)           */
/* ------------------------------------------------------------------------ */

void nf4o_e4m3_encode_array(const float *y, int64_t n, uint8_t *out) {
    for (int64_t i = 0; i < n; ++i) out[i] = nf4o_e4m3_encode(y[i]);
}

void nf4o_f32_to_bf16_array(const float *f, int64_t n, uint16_t *out) {
    for (int64_t i = 0; i < n; ++i) out[i] = nf4o_f32_to_bf16(f[i]);
}

void nf4o_code_of_array(const float *x, int64_t n, uint8_t *out) {
    for (int64_t i = 0; i < n; ++i) out[i] = (uint8_t)nf4o_code_of(x[i]);
}
