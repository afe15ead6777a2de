/*
 * sage_oracle_sa2.c -- plain, slow CPU oracle for the FP8 P.V variant of the 8-bit
 * attention forward pass.
 *
 * TEST INFRASTRUCTURE ONLY (like sage_oracle.c, which it is linked with): nothing in the
 * product path links, loads or calls it, and it shares no code with the CUDA library.
 *
 * What it computes follows the SageAttention2 abstract ("SageAttention2: Efficient Attention
 * with Thorough Outlier Smoothing and Per-thread INT4 Quantization", author pages of Jia Wei
 * and Haofeng Huang): the matrices (P~, V) are quantized to
 * FP8, V (and Q) are smoothed, and P~V is accumulated in an FP32 buffer.  Q.K^T stays the
 * INT8 product of sage_oracle.c (smoothed K, absmax INT8 Q and K): the INT4 Q.K^T of that
 * abstract is not part of this variant.  The abstract leaves the formats open; the readings:
 *
 *   FP8 format      E4M3 (1 sign, 4 exponent bits with bias 7, 3 mantissa bits, no
 *                   infinities, largest finite 448, subnormals down to 2^-9), round to
 *                   nearest even, values beyond +-448 saturate to +-448.
 *   V               per (batch, head): optional smoothing by the channel mean over the N
 *                   tokens (exact fixed-point sum, as for K); x = fl32(V - vm);
 *                   one scale per channel c, sv = fl32(a_c / 448), a_c = max_t |x[t][c]|,
 *                   codes e4m3(fl32(x * fl32(448 / a_c))).  A per-channel scale is constant
 *                   along the P.V contraction (the tokens), so it factors out of the sum.
 *   P~              u_j = s_j * log2(e) (fp64 scores in log2 units), M = ceil(max_j u_j), an
 *                   integer; P~_j = e4m3(2^(u_j - M + 8)), so the row's largest weight lies in
 *                   (128, 256] and every weight is rounded on the E4M3 grid of a power-of-two
 *                   scaling of exp(s_j - max s).  The row sum uses the unrounded 2^(u_j - M + 8).
 *   O_i             (sum_j P~_j * dec(v8_j) * sv) / l + vm, accumulated in fp64 (the
 *                   abstract's FP32 buffer; a wider buffer here).
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define ORACLE_OK 0
#define ORACLE_ERR_ARG -1
#define ORACLE_ERR_NOMEM -5

static double h2d_sa2(uint16_t bits) {
    _Float16 h;
    memcpy(&h, &bits, sizeof h);
    return (double)h;
}

static uint16_t d2h_sa2(double v) {
    _Float16 h = (_Float16)v;
    uint16_t bits;
    memcpy(&bits, &h, sizeof bits);
    return bits;
}

/* ---------------------------------------------------------------------------
 * E4M3 from the format definition.  Encoding: bits 7 sign, 6-3 exponent field E,
 * 2-0 mantissa field F.  E = 0: value F * 2^-9 (subnormal, F = 0 is zero);
 * E = 1..15: (1 + F/8) * 2^(E - 7), except E = 15, F = 7, which is NaN.
 * ------------------------------------------------------------------------- */
double oracle_e4m3_decode(uint8_t b) {
    const int sign = b >> 7, E = (b >> 3) & 15, F = b & 7;
    double v;
    if (E == 15 && F == 7) return NAN;
    if (E == 0) v = ldexp((double)F, -9);
    else v = ldexp(1.0 + F / 8.0, E - 7);
    return sign ? -v : v;
}

/* Round to the nearest E4M3 value, ties to the even mantissa, saturating at +-448. */
uint8_t oracle_e4m3_encode(double x) {
    const uint8_t sign = signbit(x) ? 0x80 : 0;
    double a = fabs(x);
    if (isnan(x)) return 0x7F;
    if (a >= 448.0) return sign | 0x7E; /* 448 = 1.75 * 2^8: E = 15, F = 6 */
    if (a < ldexp(1.0, -6)) {           /* subnormal range: steps of 2^-9 */
        const double m = nearbyint(ldexp(a, 9)); /* exact scaling; ties to even */
        return sign | (uint8_t)m;                 /* m = 8 encodes 2^-6, the smallest normal */
    }
    int e;
    frexp(a, &e); /* a = f * 2^e, f in [0.5, 1): the binade is 2^(e-1) */
    const int eb = e - 1;                          /* -6 .. 8 */
    double m = nearbyint(ldexp(a, 3 - eb));        /* 8 .. 16, steps of 2^(eb-3) */
    int E = eb + 7;
    if (m == 16.0) { m = 8.0; E += 1; }
    if (E > 15 || (E == 15 && m - 8.0 > 6.0)) return sign | 0x7E; /* above 448 after rounding */
    return sign | (uint8_t)((E << 3) | (int)(m - 8.0));
}

void oracle_e4m3_encode_n(const double* x, int64_t n, uint8_t* out) {
    for (int64_t i = 0; i < n; ++i) out[i] = oracle_e4m3_encode(x[i]);
}

void oracle_e4m3_decode_n(const uint8_t* b, int64_t n, double* out) {
    for (int64_t i = 0; i < n; ++i) out[i] = oracle_e4m3_decode(b[i]);
}

/* ---------------------------------------------------------------------------
 * V to FP8 with one scale per (batch, head, channel); smoothing optional (vm = NULL:
 * none).  vm[c] = fl32(fl32(S_c) / fl32(N)) * 2^-24 from the exact sum S_c of
 * V[t][c] * 2^24 (as the K mean); x = fl32(V - vm); a = max_t |x|; sv = fl32(a / 448);
 * inv = fl32(448 / a) (a = 0: both 0); v8 = e4m3(fl32(x * inv)).
 * v: fp16 [BH][N][d]; v8: e4m3 bits [BH][N][d]; sv, vm: fp32 [BH][d].
 * ------------------------------------------------------------------------- */
int oracle_quant_v_fp8(const uint16_t* v, int64_t BH, int64_t N, int64_t d, float* vm, float* sv, uint8_t* v8) {
    if (!v || !sv || !v8 || BH < 0 || N <= 0 || d <= 0 || N >= ((int64_t)1 << 23)) return ORACLE_ERR_ARG;
#pragma omp parallel for schedule(static)
    for (int64_t bh = 0; bh < BH; ++bh) {
        const uint16_t* vh = v + bh * N * d;
        for (int64_t c = 0; c < d; ++c) {
            float mean = 0.0f;
            if (vm) {
                int64_t s = 0;
                for (int64_t t = 0; t < N; ++t) s += (int64_t)(h2d_sa2(vh[t * d + c]) * 16777216.0);
                mean = ((float)s / (float)N) * 0x1p-24f;
                vm[bh * d + c] = mean;
            }
            float a = 0.0f;
            for (int64_t t = 0; t < N; ++t) {
                const float x = (float)h2d_sa2(vh[t * d + c]) - mean;
                if (fabsf(x) > a) a = fabsf(x);
            }
            float s = 0.0f, inv = 0.0f;
            if (a > 0.0f) {
                s = a / 448.0f;
                inv = 448.0f / a;
            }
            sv[bh * d + c] = s;
            for (int64_t t = 0; t < N; ++t) {
                const float x = (float)h2d_sa2(vh[t * d + c]) - mean;
                const float y = x * inv;
                v8[(bh * N + t) * d + c] = oracle_e4m3_encode((double)y);
            }
        }
    }
    return ORACLE_OK;
}

/* One query row i of the FP8 P.V attention (readings at the top of this file), written to
 * orow64[0..d) (may be NULL) and its fp16 rounding to orow16[0..d) (may be NULL).  vm may be
 * NULL (V not smoothed).  acc: d doubles of scratch; u: N doubles of scratch. */
static void attn_fp8pv_row(const int8_t* q8h, const int8_t* k8h, const float* sqh, const float* skh,
                           const uint8_t* v8h, const float* svh, const float* vmh, int64_t N, int64_t d,
                           int causal, double sm_scale, int64_t gq, int64_t gk, int64_t i, double* u,
                           double* acc, double* orow64, uint16_t* orow16) {
    const int64_t jend = causal ? i + 1 : N;
    const int8_t* qi = q8h + i * d;
    const double sqi = (double)sqh[i / gq];
    double umax = -INFINITY;
    for (int64_t j = 0; j < jend; ++j) {
        const int8_t* kj = k8h + j * d;
        int64_t dot = 0;
        for (int64_t c = 0; c < d; ++c) dot += (int64_t)qi[c] * (int64_t)kj[c];
        const double s = (double)dot * sqi * (double)skh[j / gk] * sm_scale;
        u[j] = s * 1.4426950408889634; /* log2(e) */
        if (u[j] > umax) umax = u[j];
    }
    const double M = ceil(umax);
    double l = 0.0;
    for (int64_t c = 0; c < d; ++c) acc[c] = 0.0;
    for (int64_t j = 0; j < jend; ++j) {
        const double p = exp2(u[j] - M + 8.0);
        l += p;
        const double pt = oracle_e4m3_decode(oracle_e4m3_encode(p));
        const uint8_t* vj = v8h + j * d;
        for (int64_t c = 0; c < d; ++c) acc[c] += pt * oracle_e4m3_decode(vj[c]);
    }
    for (int64_t c = 0; c < d; ++c) {
        const double o = acc[c] * (double)svh[c] / l + (vmh ? (double)vmh[c] : 0.0);
        if (orow64) orow64[c] = o;
        if (orow16) orow16[c] = d2h_sa2(o);
    }
}

/* All heads.  q8/k8/sq/sk as in oracle_attn; v8 [BH][N][d] e4m3; sv, vm [BH][d] (vm may be
 * NULL).  Writes o64 (may be NULL) and its fp16 rounding o16 (may be NULL). */
int oracle_attn_fp8pv(const int8_t* q8, const int8_t* k8, const float* sq, const float* sk, const uint8_t* v8,
                      const float* sv, const float* vm, int64_t BH, int64_t N, int64_t d, int causal,
                      double sm_scale, int64_t gq, int64_t gk, double* o64, uint16_t* o16) {
    if (!q8 || !k8 || !sq || !sk || !v8 || !sv || BH < 0 || N <= 0 || d <= 0 || gq <= 0 || gk <= 0)
        return ORACLE_ERR_ARG;
    const int64_t nsq = (N + gq - 1) / gq, nsk = (N + gk - 1) / gk;
    int err = ORACLE_OK;
#pragma omp parallel
    {
        double* u = (double*)malloc(sizeof(double) * (size_t)N);
        double* acc = (double*)malloc(sizeof(double) * (size_t)d);
        if (!u || !acc) {
#pragma omp atomic write
            err = ORACLE_ERR_NOMEM;
        } else {
#pragma omp for collapse(2) schedule(dynamic, 16)
            for (int64_t bh = 0; bh < BH; ++bh) {
                for (int64_t i = 0; i < N; ++i) {
                    attn_fp8pv_row(q8 + bh * N * d, k8 + bh * N * d, sq + bh * nsq, sk + bh * nsk, v8 + bh * N * d,
                                   sv + bh * d, vm ? vm + bh * d : NULL, N, d, causal, sm_scale, gq, gk, i, u, acc,
                                   o64 ? o64 + (bh * N + i) * d : NULL, o16 ? o16 + (bh * N + i) * d : NULL);
                }
            }
        }
        free(u);
        free(acc);
    }
    return err;
}

/* Selected query rows of one head (rows[r] in [0, N)); row r of the output is rows[r]. */
int oracle_attn_fp8pv_rows(const int8_t* q8h, const int8_t* k8h, const float* sqh, const float* skh,
                           const uint8_t* v8h, const float* svh, const float* vmh, int64_t N, int64_t d,
                           int causal, double sm_scale, int64_t gq, int64_t gk, const int64_t* rows,
                           int64_t nrows, double* o64) {
    if (!q8h || !k8h || !sqh || !skh || !v8h || !svh || !rows || !o64 || N <= 0 || d <= 0 || gq <= 0 || gk <= 0)
        return ORACLE_ERR_ARG;
    for (int64_t r = 0; r < nrows; ++r)
        if (rows[r] < 0 || rows[r] >= N) return ORACLE_ERR_ARG;
    int err = ORACLE_OK;
#pragma omp parallel
    {
        double* u = (double*)malloc(sizeof(double) * (size_t)N);
        double* acc = (double*)malloc(sizeof(double) * (size_t)d);
        if (!u || !acc) {
#pragma omp atomic write
            err = ORACLE_ERR_NOMEM;
        } else {
#pragma omp for schedule(dynamic, 1)
            for (int64_t r = 0; r < nrows; ++r) {
                attn_fp8pv_row(q8h, k8h, sqh, skh, v8h, svh, vmh, N, d, causal, sm_scale, gq, gk, rows[r], u, acc,
                               o64 + r * d, NULL);
            }
        }
        free(u);
        free(acc);
    }
    return err;
}
