/*
 * Reference oracle for the smoothed, outlier-split W4A4 linear layer.
 *
 * TEST INFRASTRUCTURE ONLY. This file is a plain, slow, single-purpose CPU
 * restatement of what the layer computes, written from the method's
 * description in "W4A4 Quantization for Inference on Wan2.2-I2V-A14B"
 * (ICME 2026 challenge paper) and from the OCP Microscaling (MX) v1.0
 * definition of MXFP4. Only the test suite, the smoke check and the CPU
 * baseline leg of the benchmark may load it. It shares no code, header,
 * table or constant generator with the CUDA library.
 *
 * Conventions (each one is a reading of the paper; the list of readings is
 * kept with the design notes):
 *   - BF16 values travel as uint16 bit patterns; FP32 arithmetic is IEEE
 *     single precision, round-to-nearest-even, no contraction
 *     (compiled with -ffp-contract=off).
 *   - Accumulation of the dual-branch product is in FP64; every product of
 *     two dequantised 4-bit values (times their power-of-two scales) or of
 *     two BF16 values is exact in FP64.
 *   - J (bulk channels) and O (outlier channels) are both in ascending
 *     original channel order; bulk blocks of 32 run over the compacted
 *     bulk index p = 0..Kb-1.
 *   - Kbp = Kb rounded up to 128, kp = k rounded up to 64; padded
 *     positions hold code 0 / BF16 zero, and a 32-block with no real
 *     element gets scale code 0.
 *
 * NVFP4 (a second 4-bit block format on the same dual product) has its
 * own section at the end of the file.
 *
 * Parity pins: see tests/test_oracle_*.py. Every function below is pinned.
 */
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#include <math.h>

/* ------------------------------------------------------------------ */
/* Scalar helpers                                                       */
/* ------------------------------------------------------------------ */

static float u32_as_f32(uint32_t u) { float f; memcpy(&f, &u, 4); return f; }
static uint32_t f32_as_u32(float f) { uint32_t u; memcpy(&u, &f, 4); return u; }

/* BF16 is the upper half of an IEEE binary32 word. */
double oracle_bf16_to_f64(uint16_t h) { return (double)u32_as_f32((uint32_t)h << 16); }
float oracle_bf16_to_f32(uint16_t h) { return u32_as_f32((uint32_t)h << 16); }

/*
 * Round a binary32 value to the nearest BF16 value, ties to the even
 * significand (IEEE 754 roundTiesToEven). Written from the definition:
 * take the two BF16 neighbours of |f| (truncation and the next value up),
 * pick the nearer, and on a tie the one whose last significand bit is 0.
 * Overflow follows IEEE: the value just above the largest finite BF16 is
 * treated as 2^128 when measuring distance.
 */
uint16_t oracle_f32_to_bf16(float f)
{
    uint32_t u = f32_as_u32(f);
    uint32_t sign = u & 0x80000000u;
    uint32_t mag = u & 0x7FFFFFFFu;
    if (mag > 0x7F800000u) return (uint16_t)((u >> 16) | 0x0040u); /* NaN stays NaN (quiet) */
    if (mag == 0x7F800000u) return (uint16_t)(u >> 16);              /* +-inf */
    uint16_t lo = (uint16_t)(mag >> 16);         /* truncation toward zero */
    uint16_t hi = (uint16_t)(lo + 1);            /* next magnitude up */
    double v = (double)u32_as_f32(mag);
    double vlo = oracle_bf16_to_f64(lo);
    double vhi = (hi == 0x7F80u) ? ldexp(1.0, 128) : oracle_bf16_to_f64(hi);
    double dlo = v - vlo, dhi = vhi - v;
    uint16_t pick;
    if (dlo < dhi) pick = lo;
    else if (dhi < dlo) pick = hi;
    else pick = (lo & 1u) ? hi : lo;
    return (uint16_t)(pick | (sign >> 16));
}

/* binary16 (IEEE half) -> FP64: sign, 5-bit exponent (bias 15), 10-bit
 * significand, subnormals below 2^-14. */
double oracle_f16_to_f64(uint16_t h)
{
    int sign = (h >> 15) & 1, e = (h >> 10) & 31, m = h & 1023;
    double v;
    if (e == 31) v = m ? NAN : INFINITY;
    else if (e == 0) v = ldexp((double)m, -24);
    else v = ldexp((double)(m + 1024), e - 25);
    return sign ? -v : v;
}

/*
 * Round a binary32 value to the nearest binary16 value, ties to the even
 * significand, written from the definition as for BF16: the truncated
 * magnitude code and the next code up are the two neighbours, the nearer
 * wins, a tie goes to the even code. Magnitudes from 65520 (halfway between
 * the largest finite half, 65504, and 2^16) round to infinity.
 */
uint16_t oracle_f32_to_f16(float f)
{
    uint16_t sign = (f32_as_u32(f) >> 16) & 0x8000u;
    double v = fabs((double)f);
    if (isnan(f)) return (uint16_t)(sign | 0x7E00u);
    if (v >= 65520.0) return (uint16_t)(sign | 0x7C00u);
    uint16_t lo;
    if (v < ldexp(1.0, -14)) {
        lo = (uint16_t)floor(v / ldexp(1.0, -24));                /* subnormal grid */
    } else {
        int e;
        frexp(v, &e);                                             /* v in [2^(e-1), 2^e) */
        double q = ldexp(1.0, (e - 1) - 10);
        uint16_t mant = (uint16_t)(floor(v / q) - 1024.0);
        lo = (uint16_t)(((e - 1 + 15) << 10) | mant);
    }
    uint16_t hi = (uint16_t)(lo + 1);
    double dlo = v - oracle_f16_to_f64(lo);
    double dhi = oracle_f16_to_f64(hi) - v;   /* hi may be 0x7C00 = inf only for v >= 65504 + ... (excluded above) */
    uint16_t pick;
    if (dlo < dhi) pick = lo;
    else if (dhi < dlo) pick = hi;
    else pick = (lo & 1u) ? hi : lo;
    return (uint16_t)(pick | sign);
}

/* Round an FP64 value to binary32 (C conversion is round-to-nearest-even). */
float oracle_f64_to_f32(double v) { return (float)v; }

/* ------------------------------------------------------------------ */
/* OCP MXFP4: E2M1 elements with one E8M0 scale per block               */
/* ------------------------------------------------------------------ */

/* The eight non-negative E2M1 magnitudes, indexed by the 3-bit code
 * (exponent bias 1, one mantissa bit, no inf/NaN). */
static const double E2M1_MAG[8] = {0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0};

double oracle_e2m1_decode(uint8_t code)
{
    double m = E2M1_MAG[code & 7u];
    return (code & 8u) ? -m : m;
}

/*
 * Encode one real value v (already divided by the block scale) to E2M1:
 * nearest representable magnitude, ties to the even code (last mantissa
 * bit 0), magnitudes above 6 saturate to 6. The sign bit copies the sign
 * of v, so -0 and small negatives that round to zero give code 0x8.
 */
uint8_t oracle_e2m1_encode(double v, int negative)
{
    double a = fabs(v);
    int best = 0;
    double bestd = fabs(a - E2M1_MAG[0]);
    for (int c = 1; c < 8; ++c) {
        double d = fabs(a - E2M1_MAG[c]);
        if (d < bestd || (d == bestd && (c & 1) == 0 && (best & 1) == 1)) {
            best = c;
            bestd = d;
        }
    }
    return (uint8_t)(best | (negative ? 8 : 0));
}

/*
 * Shared-scale exponent of an MX block (OCP MX v1.0 conversion rule):
 * X = floor(log2(amax)) - emax, with emax = 2 for E2M1, clamped to the
 * E8M0 range [-127, 127]. A block whose amax is 0 gets X = -127.
 * Returns X; the stored E8M0 code is X + 127.
 */
int oracle_mx_scale_exponent(double amax)
{
    if (!(amax > 0.0)) return -127;
    int e;
    (void)frexp(amax, &e);        /* amax = m * 2^e, m in [0.5, 1) */
    int X = (e - 1) - 2;          /* floor(log2 amax) - emax */
    if (X < -127) X = -127;
    if (X > 127) X = 127;
    return X;
}

/* Quantise n values (given as BF16 words) with shared exponent X.
 * Writes one 4-bit code per value into codes[]. */
static void mx_encode_values(const uint16_t* v16, int n, int X, uint8_t* codes)
{
    double inv = ldexp(1.0, -X);
    for (int i = 0; i < n; ++i) {
        double v = oracle_bf16_to_f64(v16[i]);
        int neg = (v16[i] & 0x8000u) != 0;
        codes[i] = oracle_e2m1_encode(v * inv, neg);
    }
}

/* ------------------------------------------------------------------ */
/* Sizes                                                                */
/* ------------------------------------------------------------------ */

static int64_t round_up(int64_t a, int64_t b) { return (a + b - 1) / b * b; }
int64_t oracle_kbp(int64_t K, int64_t k) { return round_up(K - k, 128); }
int64_t oracle_kp(int64_t k) { return round_up(k, 64); }

/* ------------------------------------------------------------------ */
/* Calibration: Eq. (2) and Eq. (4)                                     */
/* ------------------------------------------------------------------ */

/* act_scale_j = max_t |x_tj| over calibration tokens (Eq. (4) score and the
 * activation statistic of Eq. (2)). X is [T][K] BF16, row-major. */
void oracle_act_amax(const uint16_t* X, int64_t T, int64_t K, float* amax)
{
    for (int64_t j = 0; j < K; ++j) amax[j] = 0.0f;
    for (int64_t t = 0; t < T; ++t)
        for (int64_t j = 0; j < K; ++j) {
            float a = fabsf(oracle_bf16_to_f32(X[t * K + j]));
            if (a > amax[j]) amax[j] = a;
        }
}

/* weight_scale_j = max_n |W_jn|: the range of input channel j of W [K][N]. */
void oracle_weight_amax(const uint16_t* W, int64_t K, int64_t N, float* wmax)
{
    for (int64_t j = 0; j < K; ++j) {
        float m = 0.0f;
        for (int64_t n = 0; n < N; ++n) {
            float a = fabsf(oracle_bf16_to_f32(W[j * N + n]));
            if (a > m) m = a;
        }
        wmax[j] = m;
    }
}

static const int64_t* g_sort_keys_idx;
static const float* g_sort_amax;
static int cmp_score_desc(const void* pa, const void* pb)
{
    int64_t a = *(const int64_t*)pa, b = *(const int64_t*)pb;
    float sa = g_sort_amax[a], sb = g_sort_amax[b];
    if (sa > sb) return -1;
    if (sa < sb) return 1;
    return (a < b) ? -1 : (a > b);
}
static int cmp_i32(const void* pa, const void* pb)
{
    int32_t a = *(const int32_t*)pa, b = *(const int32_t*)pb;
    return (a > b) - (a < b);
}

/*
 * Eq. (2): s_j = act_scale_j^alpha / weight_scale_j^(1-alpha), evaluated in
 * FP64 with both statistics floored at 1e-5, then rounded to FP32;
 * inv_s_j = 1/s_j in FP32. Eq. (4): O = the k channels with the largest
 * score (ties: lower channel index first), returned ascending; the paper's
 * score is act_scale itself (oracle_calibrate), the tail-aware variant a
 * percentile of |x| (oracle_act_percentile). Returns 0, or 1 if a
 * statistic is not finite.
 */
int oracle_calibrate_scored(const float* amax, const float* score, const float* wmax, int64_t K, float alpha,
                            int64_t k, float* s, float* inv_s, int32_t* O)
{
    for (int64_t j = 0; j < K; ++j)
        if (!isfinite(amax[j]) || !isfinite(wmax[j]) || !isfinite(score[j])) return 1;
    double a = (double)alpha;
    for (int64_t j = 0; j < K; ++j) {
        double am = (double)amax[j] < 1e-5 ? 1e-5 : (double)amax[j];
        double wm = (double)wmax[j] < 1e-5 ? 1e-5 : (double)wmax[j];
        double sj = pow(am, a) / pow(wm, 1.0 - a);
        s[j] = (float)sj;
        inv_s[j] = 1.0f / s[j];
    }
    if (k > 0) {
        int64_t* idx = (int64_t*)malloc(sizeof(int64_t) * (size_t)K);
        for (int64_t j = 0; j < K; ++j) idx[j] = j;
        g_sort_amax = score;
        qsort(idx, (size_t)K, sizeof(int64_t), cmp_score_desc);
        for (int64_t i = 0; i < k; ++i) O[i] = (int32_t)idx[i];
        qsort(O, (size_t)k, sizeof(int32_t), cmp_i32);
        free(idx);
    }
    return 0;
}

int oracle_calibrate(const float* amax, const float* wmax, int64_t K, float alpha,
                     int64_t k, float* s, float* inv_s, int32_t* O)
{
    return oracle_calibrate_scored(amax, amax, wmax, K, alpha, k, s, inv_s, O);
}

/*
 * Tail-aware channel score (the activation-tail-aware percentile
 * calibration of the Tail-Aware HiFloat4 page, used to build the channel
 * mask): the nearest-rank q-percentile of |x_tj| over the T calibration
 * tokens, i.e. the value of rank r in ascending order with
 * r = ceil(q T) clamped to [1, T], evaluated in FP64. q = 1 gives the
 * maximum, the score of Eq. (4).
 */
int64_t oracle_percentile_rank(double q, int64_t T)
{
    double r = ceil(q * (double)T);
    if (r < 1.0) r = 1.0;
    if (r > (double)T) r = (double)T;
    return (int64_t)r;
}

static int cmp_f32_asc(const void* pa, const void* pb)
{
    float a = *(const float*)pa, b = *(const float*)pb;
    return (a > b) - (a < b);
}

/* score[j] = the rank-th smallest |x_tj| over t (rank 1-based). */
void oracle_act_percentile(const uint16_t* X, int64_t T, int64_t K, int64_t rank, float* score)
{
    float* col = (float*)malloc(sizeof(float) * (size_t)T);
    for (int64_t j = 0; j < K; ++j) {
        for (int64_t t = 0; t < T; ++t) col[t] = fabsf(oracle_bf16_to_f32(X[t * K + j]));
        qsort(col, (size_t)T, sizeof(float), cmp_f32_asc);
        score[j] = col[rank - 1];
    }
    free(col);
}

/* J = ascending complement of O in [0, K). Returns Kb. */
static int64_t build_J(const int32_t* O, int64_t K, int64_t k, int32_t* J)
{
    char* is_out = (char*)calloc((size_t)K, 1);
    for (int64_t i = 0; i < k; ++i) is_out[O[i]] = 1;
    int64_t p = 0;
    for (int64_t j = 0; j < K; ++j)
        if (!is_out[j]) J[p++] = (int32_t)j;
    free(is_out);
    return p;
}

/* ------------------------------------------------------------------ */
/* Eq. (1): smoothing of activations and folding into weights           */
/* ------------------------------------------------------------------ */

/* x'_tj = bf16(fp32(x_tj) * inv_s_j): the activations divided by s, by
 * one FP32 multiply with the FP32 reciprocal, rounded to BF16. */
void oracle_smooth_act(const uint16_t* X, int64_t M, int64_t K, const float* inv_s, uint16_t* Xs)
{
    for (int64_t t = 0; t < M; ++t)
        for (int64_t j = 0; j < K; ++j) {
            float p = oracle_bf16_to_f32(X[t * K + j]) * inv_s[j];
            Xs[t * K + j] = oracle_f32_to_bf16(p);
        }
}

/* w'_jn = bf16(fp32(w_jn) * s_j): s folded into the master weights. */
void oracle_fold_weights(const uint16_t* W, int64_t K, int64_t N, const float* s, uint16_t* Ws)
{
    for (int64_t j = 0; j < K; ++j)
        for (int64_t n = 0; n < N; ++n) {
            float p = oracle_bf16_to_f32(W[j * N + n]) * s[j];
            Ws[j * N + n] = oracle_f32_to_bf16(p);
        }
}

/* ------------------------------------------------------------------ */
/* Runtime activation path: smooth, split, MXFP4-encode                 */
/* ------------------------------------------------------------------ */

/*
 * For each row t of X [M][K]:
 *   x' = smoothed row;
 *   a_hp[t][i] = x'[O_i] (i < k), zero for k <= i < kp;
 *   bulk row = x'[J_p] for p < Kb, zero for Kb <= p < Kbp;
 *   for each 32-block b of the bulk row: X_b from the amax of its real
 *   elements, scale code X_b + 127 (0 if the block has no real element),
 *   codes E2M1(x'/2^X_b), two per byte, low nibble = even position.
 * Outputs: codes [M][Kbp/2], scales (logical) [M][Kbp/32], a_hp [M][kp].
 */
/* hp_fp16 != 0: the outlier slots hold the same FP32 products x * inv_s
 * rounded to binary16 instead of BF16 (the FP16 outlier branch). */
void oracle_quantize_act_ex(const uint16_t* X, int64_t M, int64_t K, int64_t k,
                            const float* inv_s, const int32_t* O,
                            uint8_t* codes, uint8_t* scales, uint16_t* a_hp, int hp_fp16)
{
    int64_t Kbp = oracle_kbp(K, k), kp = oracle_kp(k);
    int64_t nb = Kbp / 32;
    int32_t* J = (int32_t*)malloc(sizeof(int32_t) * (size_t)(K > 0 ? K : 1));
    int64_t Kb = build_J(O, K, k, J);
#pragma omp parallel for schedule(static)
    for (int64_t t = 0; t < M; ++t) {
        uint16_t* row = (uint16_t*)malloc(sizeof(uint16_t) * (size_t)(K > 0 ? K : 1));
        uint8_t c4[32];
        for (int64_t j = 0; j < K; ++j) {
            float p = oracle_bf16_to_f32(X[t * K + j]) * inv_s[j];
            row[j] = oracle_f32_to_bf16(p);
        }
        for (int64_t i = 0; i < kp; ++i) {
            if (i >= k) a_hp[t * kp + i] = 0;
            else if (!hp_fp16) a_hp[t * kp + i] = row[O[i]];
            else a_hp[t * kp + i] = oracle_f32_to_f16(oracle_bf16_to_f32(X[t * K + O[i]]) * inv_s[O[i]]);
        }
        for (int64_t b = 0; b < nb; ++b) {
            int64_t p0 = 32 * b;
            int n_real = (int)(p0 >= Kb ? 0 : (Kb - p0 < 32 ? Kb - p0 : 32));
            uint16_t vals[32];
            double amax = 0.0;
            for (int i = 0; i < n_real; ++i) {
                vals[i] = row[J[p0 + i]];
                double a = fabs(oracle_bf16_to_f64(vals[i]));
                if (a > amax) amax = a;
            }
            int Xe = oracle_mx_scale_exponent(amax);
            scales[t * nb + b] = (uint8_t)(n_real ? Xe + 127 : 0);
            memset(c4, 0, sizeof c4);
            mx_encode_values(vals, n_real, Xe, c4);
            for (int i = 0; i < 16; ++i)
                codes[t * (Kbp / 2) + p0 / 2 + i] = (uint8_t)(c4[2 * i] | (c4[2 * i + 1] << 4));
        }
        free(row);
    }
    free(J);
}

void oracle_quantize_act(const uint16_t* X, int64_t M, int64_t K, int64_t k,
                         const float* inv_s, const int32_t* O,
                         uint8_t* codes, uint8_t* scales, uint16_t* a_hp)
{
    oracle_quantize_act_ex(X, M, K, k, inv_s, O, codes, scales, a_hp, 0);
}

/* ------------------------------------------------------------------ */
/* Offline weight packing with block-wise scales                         */
/* ------------------------------------------------------------------ */

/*
 * W [K][N] BF16 row-major (input channel j, output channel n).
 * w' = folded weights. Outputs are K-major per output channel:
 *   w_hp [N][kp]: w'[O_i][n], zero padded;
 *   codes [N][Kbp/2], scales (logical) [N][Kbp/32] over the compacted bulk
 *   index p, with the block exponent taken from the amax of
 *     mode 0 (1x32):   the 32 positions of the block of row n;
 *     mode 1 (32x32):  the 32x32 tile (32 positions x 32 output channels);
 *     mode 2 (128x1):  the 128-position K-strip of row n;
 *   and replicated to every 32-block inside the tile or strip. Only real
 *   elements (p < Kb, n < N) enter an amax; a block with no real element
 *   gets scale code 0.
 */
/* hp_fp16 != 0: w_hp holds the folded outlier weights fp32(w) * s rounded
 * to binary16 instead of BF16. */
void oracle_pack_weights_ex(const uint16_t* W, int64_t K, int64_t N, int64_t k,
                            const float* s, const int32_t* O, int mode,
                            uint8_t* codes, uint8_t* scales, uint16_t* w_hp, int hp_fp16)
{
    int64_t Kbp = oracle_kbp(K, k), kp = oracle_kp(k);
    int64_t nb = Kbp / 32;
    int32_t* J = (int32_t*)malloc(sizeof(int32_t) * (size_t)(K > 0 ? K : 1));
    int64_t Kb = build_J(O, K, k, J);
    /* folded weights, transposed to [N][K] for convenience */
    uint16_t* Wt = (uint16_t*)malloc(sizeof(uint16_t) * (size_t)(N * (K > 0 ? K : 1)));
#pragma omp parallel for schedule(static)
    for (int64_t n = 0; n < N; ++n)
        for (int64_t j = 0; j < K; ++j) {
            float p = oracle_bf16_to_f32(W[j * N + n]) * s[j];
            Wt[n * K + j] = oracle_f32_to_bf16(p);
        }
    for (int64_t n = 0; n < N; ++n)
        for (int64_t i = 0; i < kp; ++i) {
            if (i >= k) w_hp[n * kp + i] = 0;
            else if (!hp_fp16) w_hp[n * kp + i] = Wt[n * K + O[i]];
            else w_hp[n * kp + i] = oracle_f32_to_f16(oracle_bf16_to_f32(W[(int64_t)O[i] * N + n]) * s[O[i]]);
        }

    /* block amax of row n, block b (real elements only) */
    double* bam = (double*)calloc((size_t)(N * (nb > 0 ? nb : 1)), sizeof(double));
#pragma omp parallel for schedule(static)
    for (int64_t n = 0; n < N; ++n)
        for (int64_t b = 0; b < nb; ++b) {
            double m = 0.0;
            for (int64_t p = 32 * b; p < 32 * b + 32 && p < Kb; ++p) {
                double a = fabs(oracle_bf16_to_f64(Wt[n * K + J[p]]));
                if (a > m) m = a;
            }
            bam[n * nb + b] = m;
        }
#pragma omp parallel for schedule(static)
    for (int64_t n = 0; n < N; ++n) {
        uint8_t c4[32];
        uint16_t vals[32];
        for (int64_t b = 0; b < nb; ++b) {
            int64_t p0 = 32 * b;
            int n_real = (int)(p0 >= Kb ? 0 : (Kb - p0 < 32 ? Kb - p0 : 32));
            double amax = 0.0;
            if (mode == 0) {
                amax = bam[n * nb + b];
            } else if (mode == 1) {
                int64_t n0 = n / 32 * 32;
                for (int64_t nn = n0; nn < n0 + 32 && nn < N; ++nn)
                    if (bam[nn * nb + b] > amax) amax = bam[nn * nb + b];
            } else {
                int64_t b0 = b / 4 * 4;
                for (int64_t bb = b0; bb < b0 + 4 && bb < nb; ++bb)
                    if (bam[n * nb + bb] > amax) amax = bam[n * nb + bb];
            }
            int Xe = oracle_mx_scale_exponent(amax);
            scales[n * nb + b] = (uint8_t)(n_real ? Xe + 127 : 0);
            for (int i = 0; i < n_real; ++i) vals[i] = Wt[n * K + J[p0 + i]];
            memset(c4, 0, sizeof c4);
            mx_encode_values(vals, n_real, Xe, c4);
            for (int i = 0; i < 16; ++i)
                codes[n * (Kbp / 2) + p0 / 2 + i] = (uint8_t)(c4[2 * i] | (c4[2 * i + 1] << 4));
        }
    }
    free(bam);
    free(Wt);
    free(J);
}

void oracle_pack_weights(const uint16_t* W, int64_t K, int64_t N, int64_t k,
                         const float* s, const int32_t* O, int mode,
                         uint8_t* codes, uint8_t* scales, uint16_t* w_hp)
{
    oracle_pack_weights_ex(W, K, N, k, s, O, mode, codes, scales, w_hp, 0);
}

/* ------------------------------------------------------------------ */
/* Eq. (5) / Eq. (3): the dual-branch product                            */
/* ------------------------------------------------------------------ */

/*
 * For each requested activation row r (index rows[r] into the packed
 * activations) and every output channel n:
 *   y = sum_b 2^(Xa+Xw) sum_{p in b} e2m1(a) e2m1(w)     (bulk, W4A4)
 *     + sum_{i<kp} a_hp * w_hp                            (outliers, BF16 or FP16)
 *     + bias[n]                                            (if bias != NULL)
 *   T = the same sum over absolute values of every term (no bias).
 * Every term is exact in FP64; the sum is accumulated in FP64 in the
 * order bulk blocks, then outlier slots.
 * Outputs y, T: [nrows][N].
 */
void oracle_dual_gemm_rows_ex(const uint8_t* a_codes, const uint8_t* a_scales, const uint16_t* a_hp,
                              const int64_t* rows, int64_t nrows,
                              const uint8_t* w_codes, const uint8_t* w_scales, const uint16_t* w_hp,
                              int64_t N, int64_t Kbp, int64_t kp, const float* bias,
                              double* y, double* T, int hp_fp16)
{
    int64_t nb = Kbp / 32;
    /* dequantise all weight rows once: value * 2^Xw, exact in FP64 */
    double* wd = (double*)malloc(sizeof(double) * (size_t)(N * (Kbp > 0 ? Kbp : 1)));
#pragma omp parallel for schedule(static)
    for (int64_t n = 0; n < N; ++n)
        for (int64_t p = 0; p < Kbp; ++p) {
            uint8_t byte = w_codes[n * (Kbp / 2) + p / 2];
            uint8_t c = (p & 1) ? (byte >> 4) : (byte & 15u);
            int Xw = (int)w_scales[n * nb + p / 32] - 127;
            wd[n * Kbp + p] = oracle_e2m1_decode(c) * ldexp(1.0, Xw);
        }
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t r = 0; r < nrows; ++r) {
        int64_t t = rows[r];
        double* ad = (double*)malloc(sizeof(double) * (size_t)(Kbp > 0 ? Kbp : 1));
        double* hd = (double*)malloc(sizeof(double) * (size_t)(kp > 0 ? kp : 1));
        for (int64_t p = 0; p < Kbp; ++p) {
            uint8_t byte = a_codes[t * (Kbp / 2) + p / 2];
            uint8_t c = (p & 1) ? (byte >> 4) : (byte & 15u);
            int Xa = (int)a_scales[t * nb + p / 32] - 127;
            ad[p] = oracle_e2m1_decode(c) * ldexp(1.0, Xa);
        }
        for (int64_t i = 0; i < kp; ++i)
            hd[i] = hp_fp16 ? oracle_f16_to_f64(a_hp[t * kp + i]) : oracle_bf16_to_f64(a_hp[t * kp + i]);
        for (int64_t n = 0; n < N; ++n) {
            double acc = 0.0, mag = 0.0;
            const double* wr = wd + n * Kbp;
            for (int64_t p = 0; p < Kbp; ++p) {
                double term = ad[p] * wr[p];
                acc += term;
                mag += fabs(term);
            }
            for (int64_t i = 0; i < kp; ++i) {
                double wv = hp_fp16 ? oracle_f16_to_f64(w_hp[n * kp + i]) : oracle_bf16_to_f64(w_hp[n * kp + i]);
                double term = hd[i] * wv;
                acc += term;
                mag += fabs(term);
            }
            if (bias) acc += (double)bias[n];
            y[r * N + n] = acc;
            T[r * N + n] = mag;
        }
        free(ad);
        free(hd);
    }
    free(wd);
}

void oracle_dual_gemm_rows(const uint8_t* a_codes, const uint8_t* a_scales, const uint16_t* a_hp,
                           const int64_t* rows, int64_t nrows,
                           const uint8_t* w_codes, const uint8_t* w_scales, const uint16_t* w_hp,
                           int64_t N, int64_t Kbp, int64_t kp, const float* bias,
                           double* y, double* T)
{
    oracle_dual_gemm_rows_ex(a_codes, a_scales, a_hp, rows, nrows, w_codes, w_scales, w_hp, N, Kbp, kp, bias, y, T, 0);
}

/* ------------------------------------------------------------------ */
/* GELU (tanh form) of the FFN, by its definition in FP64               */
/* ------------------------------------------------------------------ */

/*
 * GELU in the tanh form that the FFN uses: 0.5 x (1 + tanh(u)) with
 * u = sqrt(2/pi) (x + 0.044715 x^3), evaluated in FP64 with libm's tanh.
 * The pages fix no bits for it; this is the plain definition, and the CUDA
 * epilogue's own FP32 routine is held to it by an error bound.
 */
double oracle_gelu_tanh(double x)
{
    const double c = sqrt(2.0 / 3.14159265358979323846);
    double u = c * (x + 0.044715 * x * x * x);
    return 0.5 * x * (1.0 + tanh(u));
}

/*
 * Round an FP64 value to the nearest BF16 value (8 significant bits,
 * binary32's exponent range), ties to the even significand, in one step
 * (no intermediate binary32 rounding). From the definition: with
 * |v| = m 2^e, m in [1/2, 1), the BF16 quantum is 2^(e-8) for normal
 * results and 2^-133 below 2^-126; v / quantum is rounded to an integer
 * by rint (round-half-even in the default rounding mode) and scaled back,
 * both exactly. Results of magnitude 2^128 or more are infinite.
 */
uint16_t oracle_f64_to_bf16(double v)
{
    if (isnan(v)) return 0x7fc0;
    double a = fabs(v);
    double r;
    if (a == 0.0 || isinf(a)) {
        r = a;
    } else {
        int e;
        frexp(a, &e);                       /* a = m 2^e, m in [0.5, 1) */
        int qexp = e - 8;                   /* quantum of an 8-bit significand */
        if (qexp < -133) qexp = -133;       /* BF16 subnormal quantum */
        r = ldexp(rint(ldexp(a, -qexp)), qexp);
        if (r >= ldexp(1.0, 128)) r = INFINITY;
    }
    float f = (float)r;                     /* exact: r is a BF16 value (or inf) */
    uint16_t h = (uint16_t)(f32_as_u32(f) >> 16);
    return signbit(v) ? (uint16_t)(h | 0x8000u) : h;
}

/* GELU of FP64 accumulators: g[i] = GELU(y[i]) in FP64. */
void oracle_gelu_rows(const double* y, int64_t n, double* g)
{
    for (int64_t i = 0; i < n; ++i) g[i] = oracle_gelu_tanh(y[i]);
}

/* FFN hidden activations from FP64 accumulators: h = bf16(GELU(y)),
 * rounded once from FP64. */
void oracle_gelu_bf16_rows(const double* y, int64_t n, uint16_t* h)
{
    for (int64_t i = 0; i < n; ++i) h[i] = oracle_f64_to_bf16(oracle_gelu_tanh(y[i]));
}

/* ------------------------------------------------------------------ */
/* NVFP4: E2M1 elements, one UE4M3 scale per 16, a per-tensor 2^g      */
/* ------------------------------------------------------------------ */

/*
 * The pages ask for other 4-bit block formats on the same dual product
 * (Sec. "Implementation" of "W4A4 Quantization for Inference on
 * Wan2.2-I2V-A14B" names block formats as the thing to explore). NVFP4
 * as read here:
 *   - elements E2M1 (the same codec as MXFP4), blocks of 16 consecutive
 *     compacted bulk positions;
 *   - one scale per block in unsigned FP8 E4M3 (bias 7, 3 mantissa bits,
 *     largest finite 448, no infinities);
 *   - one power-of-two factor 2^g per tensor, g the smallest integer in
 *     [-100, 100] with tensor amax <= 6 * 448 * 2^g (g = 0 for amax 0), so
 *     that the largest block scale fits E4M3;
 *   - block scale S = E4M3_RNE_satfinite(fp32(amax_b * k)), k = fp32(1/6) * 2^-g;
 *   - element code = E2M1_RNE_sat(fp32(x * R)), R = fp32(1 / (S * 2^g))
 *     (R = 0 when S = 0: the block encodes as signed zeros);
 *   - decoded element = e2m1 * S * 2^g;
 *   - the BF16 outlier branch shares the accumulator, so its stored
 *     operands carry 2^-g: a_hp = bf16(fp32(x' * 2^-g_a)) and
 *     w_hp = bf16(fp32(w' * 2^-g_w)), and the product is multiplied by
 *     2^(g_a + g_w) after accumulation.
 */

/* E4M3 code -> value (sign, 4-bit exponent bias 7, 3-bit mantissa;
 * exponent field 0 is subnormal 2^-6 * m/8; S.1111.111 is NaN). */
double oracle_e4m3_decode(uint8_t code)
{
    int sign = (code >> 7) & 1, e = (code >> 3) & 15, m = code & 7;
    double v;
    if (e == 15 && m == 7) v = NAN;
    else if (e == 0) v = ldexp((double)m, -9);
    else v = ldexp(8.0 + m, e - 10);
    return sign ? -v : v;
}

/* Nearest E4M3 value to f, ties to the even code (mantissa LSB 0),
 * magnitudes above 448 (and infinities) saturate to 448, NaN -> 0x7F.
 * Written as a search over all 127 finite non-negative codes. */
uint8_t oracle_e4m3_encode_satfinite(float f)
{
    if (isnan(f)) return 0x7Fu;
    uint8_t sign = signbit(f) ? 0x80u : 0u;
    double a = fabs((double)f);
    if (a >= 448.0) return (uint8_t)(sign | 0x7Eu);
    int best = 0;
    double bestd = a;
    for (int c = 1; c < 127; ++c) {
        double d = fabs(a - oracle_e4m3_decode((uint8_t)c));
        if (d < bestd || (d == bestd && (c & 1) == 0 && (best & 1) == 1)) {
            best = c;
            bestd = d;
        }
    }
    return (uint8_t)(sign | best);
}

/* Smallest g in [-100, 100] with amax <= 2688 * 2^g (2688 = 6 * 448); 0 for
 * amax 0. amax must be finite and non-negative. */
int oracle_nvfp4_tensor_exponent(double amax)
{
    if (!(amax > 0.0)) return 0;
    int g = -100;
    while (g < 100 && amax > ldexp(2688.0, g)) ++g;
    return g;
}

/* fp32(1/6) * 2^-g, exact (a power-of-two scaling of a normal number). */
static float nvfp4_k(int g) { return (float)ldexp((double)(float)(1.0 / 6.0), -g); }

/* Block scale code for a block maximum amax (a BF16 value). */
uint8_t oracle_nvfp4_scale(double amax, int g)
{
    float sc = (float)(amax * (double)nvfp4_k(g));   /* exact product, one rounding to FP32 */
    return oracle_e4m3_encode_satfinite(sc);
}

/* Element multiplier R = fp32(1 / (S * 2^g)) for scale code S, 0 for S = 0. */
float oracle_nvfp4_recip(uint8_t S, int g)
{
    double D = oracle_e4m3_decode(S) * ldexp(1.0, g);
    if (!(D > 0.0)) return 0.0f;
    return (float)(1.0 / D);
}

/* Encode n BF16 values with scale code S (multiplier R). */
static void nv_encode_values(const uint16_t* v16, int n, uint8_t S, int g, uint8_t* codes)
{
    float R = oracle_nvfp4_recip(S, g);
    for (int i = 0; i < n; ++i) {
        double v = oracle_bf16_to_f64(v16[i]);
        float q = (float)(v * (double)R);             /* exact product, one rounding */
        codes[i] = oracle_e2m1_encode((double)q, (v16[i] & 0x8000u) != 0);
    }
}

/* bf16(fp32(h * 2^-g)) for a BF16 value h. */
static uint16_t nv_hp_scaled(uint16_t h, int g)
{
    return oracle_f32_to_bf16((float)ldexp(oracle_bf16_to_f64(h), -g));
}

/*
 * Per-tensor exponents of a plan from its calibration: the activations'
 * tensor amax is max over bulk channels of bf16(fp32(amax_j * inv_s_j))
 * (the largest smoothed calibration value: both roundings are monotone),
 * the weights' is max over bulk channels of bf16(fp32(wmax_j * s_j)).
 */
void oracle_nvfp4_plan_exponents(const float* amax, const float* wmax, const float* s, const float* inv_s,
                                 const int32_t* O, int64_t K, int64_t k, int* g_act, int* g_w)
{
    char* is_out = (char*)calloc((size_t)(K > 0 ? K : 1), 1);
    for (int64_t i = 0; i < k; ++i) is_out[O[i]] = 1;
    double am = 0.0, wm = 0.0;
    for (int64_t j = 0; j < K; ++j) {
        if (is_out[j]) continue;
        double a = fabs(oracle_bf16_to_f64(oracle_f32_to_bf16(amax[j] * inv_s[j])));
        double w = fabs(oracle_bf16_to_f64(oracle_f32_to_bf16(wmax[j] * s[j])));
        if (a > am) am = a;
        if (w > wm) wm = w;
    }
    free(is_out);
    *g_act = oracle_nvfp4_tensor_exponent(am);
    *g_w = oracle_nvfp4_tensor_exponent(wm);
}

/* One row of bulk values (BF16, compacted, Kb real of Kbp) -> codes
 * [Kbp/2] and logical scales [Kbp/16]. */
static void nv_encode_row(const uint16_t* bulk, int64_t Kb, int64_t Kbp, int g, uint8_t* codes, uint8_t* scales)
{
    uint8_t c4[16];
    for (int64_t b = 0; b < Kbp / 16; ++b) {
        int64_t p0 = 16 * b;
        int n_real = (int)(p0 >= Kb ? 0 : (Kb - p0 < 16 ? Kb - p0 : 16));
        double amax = 0.0;
        for (int i = 0; i < n_real; ++i) {
            double a = fabs(oracle_bf16_to_f64(bulk[p0 + i]));
            if (a > amax) amax = a;
        }
        uint8_t S = n_real ? oracle_nvfp4_scale(amax, g) : 0;
        scales[b] = S;
        memset(c4, 0, sizeof c4);
        nv_encode_values(bulk + p0, n_real, S, g, c4);
        for (int i = 0; i < 8; ++i) codes[p0 / 2 + i] = (uint8_t)(c4[2 * i] | (c4[2 * i + 1] << 4));
    }
}

/* quantize_act in NVFP4: as the MXFP4 form, with 16-blocks, UE4M3 scales
 * (logical [M][Kbp/16]) and the outlier slots scaled by 2^-g_act. */
void oracle_quantize_act_nv(const uint16_t* X, int64_t M, int64_t K, int64_t k, const float* inv_s,
                            const int32_t* O, int g_act, uint8_t* codes, uint8_t* scales, uint16_t* a_hp)
{
    int64_t Kbp = oracle_kbp(K, k), kp = oracle_kp(k);
    int32_t* J = (int32_t*)malloc(sizeof(int32_t) * (size_t)(K > 0 ? K : 1));
    int64_t Kb = build_J(O, K, k, J);
#pragma omp parallel for schedule(static)
    for (int64_t t = 0; t < M; ++t) {
        uint16_t* row = (uint16_t*)malloc(sizeof(uint16_t) * (size_t)(K > 0 ? K : 1));
        uint16_t* bulk = (uint16_t*)calloc((size_t)(Kbp > 0 ? Kbp : 1), sizeof(uint16_t));
        for (int64_t j = 0; j < K; ++j) {
            float p = oracle_bf16_to_f32(X[t * K + j]) * inv_s[j];
            row[j] = oracle_f32_to_bf16(p);
        }
        for (int64_t i = 0; i < kp; ++i) a_hp[t * kp + i] = i < k ? nv_hp_scaled(row[O[i]], g_act) : 0;
        for (int64_t p = 0; p < Kb; ++p) bulk[p] = row[J[p]];
        nv_encode_row(bulk, Kb, Kbp, g_act, codes + t * (Kbp / 2), scales + t * (Kbp / 16));
        free(bulk);
        free(row);
    }
    free(J);
}

/* pack_weights in NVFP4: folded weights w', 16-blocks along the compacted
 * bulk index of each output channel, w_hp scaled by 2^-g_w. */
void oracle_pack_weights_nv(const uint16_t* W, int64_t K, int64_t N, int64_t k, const float* s,
                            const int32_t* O, int g_w, uint8_t* codes, uint8_t* scales, uint16_t* w_hp)
{
    int64_t Kbp = oracle_kbp(K, k), kp = oracle_kp(k);
    int32_t* J = (int32_t*)malloc(sizeof(int32_t) * (size_t)(K > 0 ? K : 1));
    int64_t Kb = build_J(O, K, k, J);
#pragma omp parallel for schedule(static)
    for (int64_t n = 0; n < N; ++n) {
        uint16_t* bulk = (uint16_t*)calloc((size_t)(Kbp > 0 ? Kbp : 1), sizeof(uint16_t));
        for (int64_t i = 0; i < kp; ++i) {
            if (i >= k) { w_hp[n * kp + i] = 0; continue; }
            float p = oracle_bf16_to_f32(W[(int64_t)O[i] * N + n]) * s[O[i]];
            w_hp[n * kp + i] = nv_hp_scaled(oracle_f32_to_bf16(p), g_w);
        }
        for (int64_t p = 0; p < Kb; ++p) {
            float v = oracle_bf16_to_f32(W[(int64_t)J[p] * N + n]) * s[J[p]];
            bulk[p] = oracle_f32_to_bf16(v);
        }
        nv_encode_row(bulk, Kb, Kbp, g_w, codes + n * (Kbp / 2), scales + n * (Kbp / 16));
        free(bulk);
    }
    free(J);
}

/* Eq. (5) with NVFP4 operands: y = 2^(g_a + g_w) * (sum_b Sa Sw sum e2m1 e2m1
 * + sum a_hp w_hp) (+ bias); T the same over absolute values of every term
 * (times 2^(g_a + g_w)). Every term is exact in FP64. */
void oracle_dual_gemm_rows_nv(const uint8_t* a_codes, const uint8_t* a_scales, const uint16_t* a_hp,
                              const int64_t* rows, int64_t nrows,
                              const uint8_t* w_codes, const uint8_t* w_scales, const uint16_t* w_hp,
                              int64_t N, int64_t Kbp, int64_t kp, int g_act, int g_w, const float* bias,
                              double* y, double* T)
{
    int64_t nb = Kbp / 16;
    double f = ldexp(1.0, g_act + g_w);
    double* wd = (double*)malloc(sizeof(double) * (size_t)(N * (Kbp > 0 ? Kbp : 1)));
#pragma omp parallel for schedule(static)
    for (int64_t n = 0; n < N; ++n)
        for (int64_t p = 0; p < Kbp; ++p) {
            uint8_t byte = w_codes[n * (Kbp / 2) + p / 2];
            uint8_t c = (p & 1) ? (byte >> 4) : (byte & 15u);
            wd[n * Kbp + p] = oracle_e2m1_decode(c) * oracle_e4m3_decode(w_scales[n * nb + p / 16]);
        }
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t r = 0; r < nrows; ++r) {
        int64_t t = rows[r];
        double* ad = (double*)malloc(sizeof(double) * (size_t)(Kbp > 0 ? Kbp : 1));
        for (int64_t p = 0; p < Kbp; ++p) {
            uint8_t byte = a_codes[t * (Kbp / 2) + p / 2];
            uint8_t c = (p & 1) ? (byte >> 4) : (byte & 15u);
            ad[p] = oracle_e2m1_decode(c) * oracle_e4m3_decode(a_scales[t * nb + p / 16]);
        }
        for (int64_t n = 0; n < N; ++n) {
            double acc = 0.0, mag = 0.0;
            for (int64_t p = 0; p < Kbp; ++p) {
                double term = ad[p] * wd[n * Kbp + p];
                acc += term;
                mag += fabs(term);
            }
            for (int64_t i = 0; i < kp; ++i) {
                double term = oracle_bf16_to_f64(a_hp[t * kp + i]) * oracle_bf16_to_f64(w_hp[n * kp + i]);
                acc += term;
                mag += fabs(term);
            }
            acc *= f;
            if (bias) acc += (double)bias[n];
            y[r * N + n] = acc;
            T[r * N + n] = mag * f;
        }
        free(ad);
    }
    free(wd);
}
