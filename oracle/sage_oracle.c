/*
 * sage_oracle.c -- plain, slow CPU oracle for the SageAttention-style 8-bit
 * attention forward pass.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product path links, loads or calls
 * this file; only the tests, the package's smoke check and the benchmark's CPU
 * baseline leg do.  It shares no code, header or constant with the CUDA library.
 *
 * What it computes follows "SageAttention: Accurate 8-Bit Attention for
 * Plug-and-play Inference Acceleration" (research.elamur.ai summary page):
 *   - Summary, first bullet: K is smoothed, then Q and K are quantized to INT8;
 *   - Summary, second bullet: the P.V product stays in 16-bit floating point;
 *   - Interesting idea I1: the smoothing subtracts a component shared by all
 *     tokens of K, which leaves every softmax row unchanged;
 *   - Key points, "Effect of smoothing K": per-token quantization granularity.
 * Steps the page leaves open are fixed by the readings written next to each
 * function (symmetric absmax scale, round-half-to-even, mean over the tokens of
 * one (batch, head), per-block groups of 128 Q / 64 K tokens, P rounded to fp16).
 *
 * Arithmetic rules: IEEE-754 binary32/binary64, round-to-nearest-even, built
 * with -ffp-contract=off (no fused multiply-add) and without fast-math.
 * Layout: every tensor is contiguous [BH][N][d] (BH = batch x heads), scales are
 * [BH][ceil(N/g)].  Loops run over heads (and rows) in parallel with OpenMP;
 * heads and rows are independent, so the results do not depend on the thread
 * count.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define ORACLE_OK 0
#define ORACLE_ERR_ARG -1
#define ORACLE_ERR_NOMEM -5

/* fp16 <-> fp64.  _Float16 conversions are exact (fp16 -> fp64) and correctly
 * rounded to nearest-even (fp64 -> fp16, one rounding, no detour via fp32). */
static double h2d(uint16_t bits) {
    _Float16 h;
    memcpy(&h, &bits, sizeof h);
    return (double)h;
}

static uint16_t d2h(double v) {
    _Float16 h = (_Float16)v;
    uint16_t bits;
    memcpy(&bits, &h, sizeof bits);
    return bits;
}

static int64_t ceil_div(int64_t a, int64_t b) { return (a + b - 1) / b; }

/* ---------------------------------------------------------------------------
 * Step 1: K smoothing (Summary bullet 1; idea I1).
 * Reading: the shared component is the mean of K over the N tokens of the same
 * (batch, head), per channel c.  Every fp16 value is an integer multiple of
 * 2^-24, so sum_t K[t][c] * 2^24 is an exact int64 (|K| < 2^16, N <= 2^31/...,
 * |sum| < 2^63 for N < 2^23).  The mean is that exact sum, rounded to fp32, divided
 * by N in fp32, then scaled by 2^-24 (exact for normal results):
 *     km[c] = fl32( fl32(S_c) / fl32(N) ) * 2^-24.
 * ------------------------------------------------------------------------- */
int oracle_smooth_k(const uint16_t* k, int64_t BH, int64_t N, int64_t d, float* km) {
    if (!k || !km || BH < 0 || N <= 0 || d <= 0 || N >= ((int64_t)1 << 23)) return ORACLE_ERR_ARG;
#pragma omp parallel for schedule(static)
    for (int64_t bh = 0; bh < BH; ++bh) {
        const uint16_t* kh = k + bh * N * d;
        for (int64_t c = 0; c < d; ++c) {
            int64_t s = 0;
            for (int64_t t = 0; t < N; ++t) {
                double scaled = h2d(kh[t * d + c]) * 16777216.0; /* exact integer */
                s += (int64_t)scaled;
            }
            float sum32 = (float)s;
            float mean32 = sum32 / (float)N;
            km[bh * d + c] = mean32 * 0x1p-24f;
        }
    }
    return ORACLE_OK;
}

/* ---------------------------------------------------------------------------
 * Step 2: symmetric INT8 quantization (Summary bullet 1; Key points: per-token).
 * Group = g consecutive tokens x all d channels of one (batch, head); g = 1 is
 * per-token, g = 128 (Q) / 64 (K) is per-block.  The last group of a head holds
 * whatever tokens remain.  For K, mu (the smoothing mean) is subtracted in fp32
 * first: x = fl32(K - mu); for Q, mu is NULL and x = Q.
 * Reading (the page names INT8 without the rounding rule):
 *     a   = max |x| over the group           (exact)
 *     s   = fl32(a / 127)                    (dequantization scale)
 *     inv = fl32(127 / a)                    (a = 0: s = inv = 0, all codes 0)
 *     q   = clamp(round_half_even(fl32(x * inv)), -127, 127)
 * ------------------------------------------------------------------------- */
static void quant_scale(float a, float* s, float* inv) {
    *s = 0.0f;
    *inv = 0.0f;
    if (a > 0.0f) {
        *s = a / 127.0f;   /* one fp32 division: the correctly rounded a/127 */
        *inv = 127.0f / a; /* one fp32 division: the correctly rounded 127/a */
    }
}

/* The scale and inverse of groups with the given absmax values a[i] (exported so
 * that the tests can pin the two roundings against exact rational arithmetic). */
void oracle_quant_scale(const float* a, int64_t n, float* s, float* inv) {
    for (int64_t i = 0; i < n; ++i) quant_scale(a[i], s + i, inv + i);
}

int oracle_quant(const uint16_t* x16, const float* mu, int64_t BH, int64_t N, int64_t d,
                 int64_t g, int8_t* q, float* scale) {
    if (!x16 || !q || !scale || BH < 0 || N <= 0 || d <= 0 || g <= 0) return ORACLE_ERR_ARG;
    const int64_t ngroups = ceil_div(N, g);
#pragma omp parallel for schedule(static)
    for (int64_t bh = 0; bh < BH; ++bh) {
        for (int64_t gi = 0; gi < ngroups; ++gi) {
            const int64_t t0 = gi * g;
            const int64_t t1 = (t0 + g < N) ? t0 + g : N;
            float a = 0.0f;
            for (int64_t t = t0; t < t1; ++t) {
                for (int64_t c = 0; c < d; ++c) {
                    float x = (float)h2d(x16[(bh * N + t) * d + c]);
                    if (mu) x = x - mu[bh * d + c];
                    float ax = fabsf(x);
                    if (ax > a) a = ax;
                }
            }
            float s, inv;
            quant_scale(a, &s, &inv);
            scale[bh * ngroups + gi] = s;
            for (int64_t t = t0; t < t1; ++t) {
                for (int64_t c = 0; c < d; ++c) {
                    float x = (float)h2d(x16[(bh * N + t) * d + c]);
                    if (mu) x = x - mu[bh * d + c];
                    float y = x * inv;
                    float r = nearbyintf(y); /* default rounding mode: to nearest, ties to even */
                    if (r > 127.0f) r = 127.0f;
                    if (r < -127.0f) r = -127.0f;
                    q[(bh * N + t) * d + c] = (int8_t)r;
                }
            }
        }
    }
    return ORACLE_OK;
}

/* ---------------------------------------------------------------------------
 * Step 3: the integer product q8 . k8^T (Summary bullet 1: QK^T in INT8),
 * exact in int64.  S has N*N entries per head.
 * ------------------------------------------------------------------------- */
int oracle_qk_int(const int8_t* q8, const int8_t* k8, int64_t BH, int64_t N, int64_t d, int64_t* S) {
    if (!q8 || !k8 || !S || BH < 0 || N <= 0 || d <= 0) return ORACLE_ERR_ARG;
#pragma omp parallel for collapse(2) schedule(static)
    for (int64_t bh = 0; bh < BH; ++bh) {
        for (int64_t i = 0; i < N; ++i) {
            const int8_t* qi = q8 + (bh * N + i) * d;
            for (int64_t j = 0; j < N; ++j) {
                const int8_t* kj = k8 + (bh * N + j) * d;
                int64_t acc = 0;
                for (int64_t c = 0; c < d; ++c) acc += (int64_t)qi[c] * (int64_t)kj[c];
                S[(bh * N + i) * N + j] = acc;
            }
        }
    }
    return ORACLE_OK;
}

/* The same products for selected query rows of one head only (rows[r] in [0,N)):
 * S[r][j] = sum_c q8h[rows[r]][c] * k8h[j][c] for all N keys. */
int oracle_qk_int_rows(const int8_t* q8h, const int8_t* k8h, int64_t N, int64_t d, const int64_t* rows,
                       int64_t nrows, int64_t* S) {
    if (!q8h || !k8h || !rows || !S || N <= 0 || d <= 0) return ORACLE_ERR_ARG;
    for (int64_t r = 0; r < nrows; ++r)
        if (rows[r] < 0 || rows[r] >= N) return ORACLE_ERR_ARG;
#pragma omp parallel for collapse(2) schedule(static)
    for (int64_t r = 0; r < nrows; ++r) {
        for (int64_t j = 0; j < N; ++j) {
            const int8_t* qi = q8h + rows[r] * d;
            const int8_t* kj = k8h + j * d;
            int64_t acc = 0;
            for (int64_t c = 0; c < d; ++c) acc += (int64_t)qi[c] * (int64_t)kj[c];
            S[r * N + j] = acc;
        }
    }
    return ORACLE_OK;
}

/* ---------------------------------------------------------------------------
 * Steps 4-6 for one query row: dequantized scores, softmax, P.V.
 *   s_j  = S_int[i][j] * sq(i) * sk(j) * sm_scale           (fp64)
 *   causal: keys j > i are masked (top-left aligned, N_q == N_k)
 *   m    = max_j s_j,  e_j = exp(s_j - m),  l = sum_j e_j   (fp64, e unrounded)
 *   Pt_j = fp16(e_j)   (Summary bullet 2: P.V runs in 16-bit floating point;
 *                       reading: the unnormalized probabilities are rounded to
 *                       fp16 relative to the row's final maximum)
 *   O_i  = (sum_j Pt_j * V_j) / l                            (fp64)
 * Writes the fp64 row to o64 (may be NULL) and its fp16 rounding to o16
 * (may be NULL).  probs (may be NULL) receives e_j / l for every j (0 if masked).
 * ------------------------------------------------------------------------- */
static void attn_row(const int8_t* q8h, const int8_t* k8h, const float* sqh, const float* skh,
                     const uint16_t* vh, int64_t N, int64_t d, int causal, double sm_scale,
                     int64_t gq, int64_t gk, int64_t i, double* s, double* acc,
                     double* o64, uint16_t* o16, double* probs) {
    const int64_t jend = causal ? i + 1 : N;
    const int8_t* qi = q8h + i * d;
    const double sqi = (double)sqh[i / gq];
    double m = -INFINITY;
    for (int64_t j = 0; j < jend; ++j) {
        const int8_t* kj = k8h + j * d;
        int64_t dot = 0;
        for (int64_t c = 0; c < d; ++c) dot += (int64_t)qi[c] * (int64_t)kj[c];
        s[j] = (double)dot * sqi * (double)skh[j / gk] * sm_scale;
        if (s[j] > m) m = s[j];
    }
    double l = 0.0;
    for (int64_t c = 0; c < d; ++c) acc[c] = 0.0;
    for (int64_t j = 0; j < jend; ++j) {
        const double e = exp(s[j] - m);
        l += e;
        const double pt = h2d(d2h(e));
        const uint16_t* vj = vh + j * d;
        for (int64_t c = 0; c < d; ++c) acc[c] += pt * h2d(vj[c]);
        s[j] = e;
    }
    for (int64_t c = 0; c < d; ++c) {
        const double o = acc[c] / l;
        if (o64) o64[i * d + c] = o;
        if (o16) o16[i * d + c] = d2h(o);
    }
    if (probs) {
        for (int64_t j = 0; j < N; ++j) probs[i * N + j] = (j < jend) ? s[j] / l : 0.0;
    }
}

/* Quantized attention forward for all heads.  gq / gk are the quantization
 * group sizes (1 = per-token, 128 / 64 = per-block) that index sq / sk. */
int oracle_attn(const int8_t* q8, const int8_t* k8, const float* sq, const float* sk,
                const uint16_t* v, int64_t BH, int64_t N, int64_t d, int causal, double sm_scale,
                int64_t gq, int64_t gk, double* o64, uint16_t* o16) {
    if (!q8 || !k8 || !sq || !sk || !v || BH < 0 || N <= 0 || d <= 0 || gq <= 0 || gk <= 0)
        return ORACLE_ERR_ARG;
    const int64_t nsq = ceil_div(N, gq), nsk = ceil_div(N, gk);
    int err = ORACLE_OK;
#pragma omp parallel
    {
        double* s = (double*)malloc(sizeof(double) * (size_t)N);
        double* acc = (double*)malloc(sizeof(double) * (size_t)d);
        if (!s || !acc) {
#pragma omp atomic write
            err = ORACLE_ERR_NOMEM;
        } else {
#pragma omp for collapse(2) schedule(dynamic, 16)
            for (int64_t bh = 0; bh < BH; ++bh) {
                for (int64_t i = 0; i < N; ++i) {
                    attn_row(q8 + bh * N * d, k8 + bh * N * d, sq + bh * nsq, sk + bh * nsk,
                             v + bh * N * d, N, d, causal, sm_scale, gq, gk, i, s, acc,
                             o64 ? o64 + bh * N * d : NULL, o16 ? o16 + bh * N * d : NULL, NULL);
                }
            }
        }
        free(s);
        free(acc);
    }
    return err;
}

/* Only the given query rows of one head (rows[r] in [0, N)); output row r goes
 * to o64[r*d] / o16[r*d].  Used to check sampled outputs of large problems. */
int oracle_attn_rows(const int8_t* q8h, const int8_t* k8h, const float* sqh, const float* skh,
                     const uint16_t* vh, int64_t N, int64_t d, int causal, double sm_scale,
                     int64_t gq, int64_t gk, const int64_t* rows, int64_t nrows,
                     double* o64, uint16_t* o16) {
    if (!q8h || !k8h || !sqh || !skh || !vh || !rows || N <= 0 || d <= 0 || gq <= 0 || gk <= 0)
        return ORACLE_ERR_ARG;
    for (int64_t r = 0; r < nrows; ++r)
        if (rows[r] < 0 || rows[r] >= N) return ORACLE_ERR_ARG;
    int err = ORACLE_OK;
#pragma omp parallel
    {
        double* s = (double*)malloc(sizeof(double) * (size_t)N);
        double* acc = (double*)malloc(sizeof(double) * (size_t)d);
        double* row64 = (double*)malloc(sizeof(double) * (size_t)(N * d));
        uint16_t* row16 = (uint16_t*)malloc(sizeof(uint16_t) * (size_t)(N * d));
        if (!s || !acc || !row64 || !row16) {
#pragma omp atomic write
            err = ORACLE_ERR_NOMEM;
        } else {
#pragma omp for schedule(dynamic, 1)
            for (int64_t r = 0; r < nrows; ++r) {
                const int64_t i = rows[r];
                attn_row(q8h, k8h, sqh, skh, vh, N, d, causal, sm_scale, gq, gk, i, s, acc,
                         row64, row16, NULL);
                for (int64_t c = 0; c < d; ++c) {
                    if (o64) o64[r * d + c] = row64[i * d + c];
                    if (o16) o16[r * d + c] = row16[i * d + c];
                }
            }
        }
        free(s);
        free(acc);
        free(row64);
        free(row16);
    }
    return err;
}

/* Normalized softmax probabilities e_ij / l_i of one head (N x N, fp64), for
 * the invariant "every row sums to one".  Small N only. */
int oracle_attn_probs(const int8_t* q8h, const int8_t* k8h, const float* sqh, const float* skh,
                      const uint16_t* vh, int64_t N, int64_t d, int causal, double sm_scale,
                      int64_t gq, int64_t gk, double* probs) {
    if (!q8h || !k8h || !sqh || !skh || !vh || !probs || N <= 0 || d <= 0) return ORACLE_ERR_ARG;
    double* s = (double*)malloc(sizeof(double) * (size_t)N);
    double* acc = (double*)malloc(sizeof(double) * (size_t)d);
    double* o64 = (double*)malloc(sizeof(double) * (size_t)(N * d));
    if (!s || !acc || !o64) {
        free(s); free(acc); free(o64);
        return ORACLE_ERR_NOMEM;
    }
    for (int64_t i = 0; i < N; ++i)
        attn_row(q8h, k8h, sqh, skh, vh, N, d, causal, sm_scale, gq, gk, i, s, acc, o64, NULL, probs);
    free(s); free(acc); free(o64);
    return ORACLE_OK;
}

/* ---------------------------------------------------------------------------
 * Unquantized attention in fp64, softmax(Q K^T sm_scale) V, straight from the
 * definition, for the "how close is the 8-bit method to exact attention"
 * metrics (idea I5: cosine similarity, relative L1, RMSE at the tensor level).
 * ------------------------------------------------------------------------- */
int oracle_attn_fp64(const uint16_t* q, const uint16_t* k, const uint16_t* v, int64_t BH,
                     int64_t N, int64_t d, int causal, double sm_scale, double* o) {
    if (!q || !k || !v || !o || BH < 0 || N <= 0 || d <= 0) return ORACLE_ERR_ARG;
    int err = ORACLE_OK;
#pragma omp parallel
    {
        double* s = (double*)malloc(sizeof(double) * (size_t)N);
        if (!s) {
#pragma omp atomic write
            err = ORACLE_ERR_NOMEM;
        } else {
#pragma omp for collapse(2) schedule(dynamic, 16)
            for (int64_t bh = 0; bh < BH; ++bh) {
                for (int64_t i = 0; i < N; ++i) {
                    const uint16_t* qi = q + (bh * N + i) * d;
                    const int64_t jend = causal ? i + 1 : N;
                    double m = -INFINITY;
                    for (int64_t j = 0; j < jend; ++j) {
                        const uint16_t* kj = k + (bh * N + j) * d;
                        double dot = 0.0;
                        for (int64_t c = 0; c < d; ++c) dot += h2d(qi[c]) * h2d(kj[c]);
                        s[j] = dot * sm_scale;
                        if (s[j] > m) m = s[j];
                    }
                    double l = 0.0;
                    for (int64_t j = 0; j < jend; ++j) {
                        s[j] = exp(s[j] - m);
                        l += s[j];
                    }
                    for (int64_t c = 0; c < d; ++c) {
                        double acc = 0.0;
                        for (int64_t j = 0; j < jend; ++j) acc += s[j] * h2d(v[(bh * N + j) * d + c]);
                        o[(bh * N + i) * d + c] = acc / l;
                    }
                }
            }
        }
        free(s);
    }
    return err;
}

/* fp64 -> fp16 rounding, exported so the tests can check it against an
 * independent implementation. */
void oracle_round_fp16(const double* x, int64_t n, uint16_t* out) {
    for (int64_t i = 0; i < n; ++i) out[i] = d2h(x[i]);
}
