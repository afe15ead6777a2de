/*
 * sage_oracle_sa3.c -- plain, slow CPU oracle for the microscaling FP4 variant of the
 * attention forward pass.
 *
 * TEST INFRASTRUCTURE ONLY (like sage_oracle.c and sage_oracle_sa2.c, which it is linked
 * with): nothing in the product path links, loads or calls it, and it shares no code with the
 * CUDA library.
 *
 * What it computes follows the SageAttention3 abstract ("SageAttention3: Microscaling FP4
 * Attention for Inference and An Exploration of 8-Bit Training", author pages of Jia Wei and
 * Haofeng Huang): attention whose two products run on FP4 tensor cores with microscaling.  The
 * abstract fixes neither the formats nor the block sizes; the readings, the plainest ones that
 * Blackwell's block-scaled FP4 products accept:
 *
 *   FP4 format      E2M1 (1 sign, 2 exponent bits with bias 1, 1 mantissa bit): 0, 0.5, 1,
 *                   1.5, 2, 3, 4, 6 and their negatives; round to nearest, ties to the even
 *                   mantissa bit; beyond +-6 saturate; the sign of a value that rounds to zero
 *                   is kept.
 *   microscaling    one UE4M3 scale per 16 consecutive elements along the contraction
 *                   dimension (the E4M3 format of sage_oracle_sa2.c, never negative here), chosen as
 *                   e4m3(fl32(max|z| / 6)); codes e2m1(fl32(z * fl32(1 / scale))) (a zero scale
 *                   gives zero codes).
 *   Q, K            a second, fp32 scale per 128-token tile of a head lifts the range: K is
 *                   smoothed first (x = fl32(K - km), km the exact channel mean of sage_oracle.c),
 *                   a = max |x| over the tile, g = fl32(a / 2688), z = fl32(x * fl32(2688 / a))
 *                   (2688 = 6 * 448, the largest E2M1 code times the largest E4M3 scale), then
 *                   microscaling along the d channels.  Dequantized: code * scale * g.
 *   V               smoothed by its exact channel mean vm (as in the FP8 variant); per channel c
 *                   a = max_t |x|, g_c = fl32(a / 2688), z = fl32(x * fl32(2688 / a)); microscaling
 *                   along the tokens (the P.V contraction), 16 tokens per scale, groups aligned to
 *                   token 0 of the head.
 *   scores          S_ij = sum_c (q code * scale)(k code * scale) exactly, s = S * gq * gk *
 *                   sm_scale, u = s * log2(e).
 *   P~              per key tile of 64 keys, in the online softmax's order: the row offset m is
 *                   the integer ceil(max u) over the key tiles seen so far (it only grows; when it
 *                   grows, the running sum and output are scaled by 2^(m_old - m_new), exactly);
 *                   p_j = 2^(u_j - m + 10) (so every p lies in (0, 1024]); the row sum takes the
 *                   unrounded p; P~ = the microscaled FP4 of fl32(p) along the keys, 16 keys per
 *                   scale.  Because m is an integer, a tile's P~ is a power-of-two scaling of the
 *                   one any other integer offset would give, as long as its scales stay normal.
 *   O               (sum_j P~_j * v code_j * v scale_j) * g_c / l + vm_c, accumulated in fp64.
 *
 * Because the kernel computes p in fp32 (exp2 approximations, fp32 scores), a decision taken
 * within a relative 1e-4 of a rounding midpoint may go either way there.  The row functions
 * therefore also return, per output element, an envelope: the sum over such keys of the largest
 * change the other rounding makes (a P~ code one E2M1 step away, or the group's other UE4M3
 * scale), times |v^| / l; and per row an "unsure" flag when a tile's offset decision (the ceil of
 * its maximum) lies within 1e-4 of an integer.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define ORACLE_OK 0
#define ORACLE_ERR_ARG -1
#define ORACLE_ERR_NOMEM -5

#define FP4_TILE 128    /* tokens per fp32 scale of Q and K */
#define FP4_KTILE 64    /* keys per online-softmax tile */
#define FP4_GROUP 16    /* elements per UE4M3 scale */
#define FP4_RANGE 2688.0f
#define P_SHIFT 10.0
#define NEAR_REL 1e-4

double oracle_e4m3_decode(uint8_t b);  /* sage_oracle_sa2.c */
uint8_t oracle_e4m3_encode(double x);

static double h2d_sa3(uint16_t bits) {
    _Float16 h;
    memcpy(&h, &bits, sizeof h);
    return (double)h;
}

static uint16_t d2h_sa3(double v) {
    _Float16 h = (_Float16)v;
    uint16_t bits;
    memcpy(&bits, &h, sizeof bits);
    return bits;
}

/* ---------------------------------------------------------------------------
 * E2M1 from the format definition: bit 3 sign, bits 2-1 exponent field E, bit 0 mantissa
 * field F.  E = 0: F * 0.5 (zero or the subnormal 0.5); E = 1..3: (1 + F/2) * 2^(E - 1).
 * ------------------------------------------------------------------------- */
static const double kE2M1[8] = {0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0};

double oracle_e2m1_decode(uint8_t c) {
    const double v = kE2M1[c & 7];
    return (c & 8) ? -v : v;
}

/* Nearest of the eight magnitudes, ties to the even code (the even mantissa bit), saturating
 * at 6; the sign bit follows the input's sign (also for results of zero). */
uint8_t oracle_e2m1_encode(double x) {
    const uint8_t sign = signbit(x) ? 8 : 0;
    const double a = fabs(x);
    if (isnan(x)) return 7;
    if (a >= 6.0) return sign | 7;
    int best = 0;
    for (int k = 1; k < 8; ++k) {
        const double dk = fabs(a - kE2M1[k]), db = fabs(a - kE2M1[best]);
        if (dk < db || (dk == db && (k & 1) == 0)) best = k;
    }
    return sign | (uint8_t)best;
}

void oracle_e2m1_encode_n(const double* x, int64_t n, uint8_t* out) {
    for (int64_t i = 0; i < n; ++i) out[i] = oracle_e2m1_encode(x[i]);
}

void oracle_e2m1_decode_n(const uint8_t* c, int64_t n, double* out) {
    for (int64_t i = 0; i < n; ++i) out[i] = oracle_e2m1_decode(c[i]);
}

/* Microscaling of n (<= 16) fp32 values z: one UE4M3 scale s8, codes c[0..n). */
static uint8_t microscale(const float* z, int n, uint8_t* c) {
    float gm = 0.0f;
    for (int i = 0; i < n; ++i)
        if (fabsf(z[i]) > gm) gm = fabsf(z[i]);
    const float t = gm / 6.0f;
    const uint8_t s8 = oracle_e4m3_encode((double)t);
    const float sd = (float)oracle_e4m3_decode(s8);
    const float inv = sd > 0.0f ? 1.0f / sd : 0.0f;
    for (int i = 0; i < n; ++i) {
        const float y = z[i] * inv;
        c[i] = oracle_e2m1_encode((double)y);
    }
    return s8;
}

/* Exposed for the pins: the scale and codes of one group. */
uint8_t oracle_fp4_microscale(const float* z, int n, uint8_t* codes) {
    if (n < 0 || n > FP4_GROUP) return 0;
    return microscale(z, n, codes);
}

/* ---------------------------------------------------------------------------
 * Q (km = NULL) or K (km = its channel means, fp32 [BH][d]) to FP4.
 * x: fp16 [BH][N][d]; codes: one E2M1 code per byte [BH][N][d]; s8: UE4M3 [BH][N][d/16];
 * g: fp32 [BH][ceil(N/128)].  d a multiple of 16.
 * ------------------------------------------------------------------------- */
int oracle_quant_fp4(const uint16_t* x, const float* km, int64_t BH, int64_t N, int64_t d, uint8_t* codes,
                     uint8_t* s8, float* g) {
    if (!x || !codes || !s8 || !g || BH < 0 || N <= 0 || d <= 0 || d % FP4_GROUP) return ORACLE_ERR_ARG;
    const int64_t nt = (N + FP4_TILE - 1) / FP4_TILE, ng = d / FP4_GROUP;
#pragma omp parallel for collapse(2) schedule(static)
    for (int64_t bh = 0; bh < BH; ++bh) {
        for (int64_t t = 0; t < nt; ++t) {
            const int64_t r0 = t * FP4_TILE, r1 = r0 + FP4_TILE < N ? r0 + FP4_TILE : N;
            float a = 0.0f;
            for (int64_t i = r0; i < r1; ++i)
                for (int64_t c = 0; c < d; ++c) {
                    const float v = (float)h2d_sa3(x[(bh * N + i) * d + c]) - (km ? km[bh * d + c] : 0.0f);
                    if (fabsf(v) > a) a = fabsf(v);
                }
            const float gt = a / FP4_RANGE;
            const float r = a > 0.0f ? FP4_RANGE / a : 0.0f;
            g[bh * nt + t] = gt;
            float z[FP4_GROUP];
            for (int64_t i = r0; i < r1; ++i) {
                for (int64_t gi = 0; gi < ng; ++gi) {
                    for (int k = 0; k < FP4_GROUP; ++k) {
                        const int64_t c = gi * FP4_GROUP + k;
                        const float v = (float)h2d_sa3(x[(bh * N + i) * d + c]) - (km ? km[bh * d + c] : 0.0f);
                        z[k] = v * r;
                    }
                    s8[(bh * N + i) * ng + gi] = microscale(z, FP4_GROUP, codes + (bh * N + i) * d + gi * FP4_GROUP);
                }
            }
        }
    }
    return ORACLE_OK;
}

/* ---------------------------------------------------------------------------
 * V to FP4, groups of 16 tokens per channel.  smooth = 0: vm is not computed and V is not
 * smoothed.  codes [BH][N][d] (token-major, one per byte); s8 [BH][ceil(N/16)][d];
 * vm, gv fp32 [BH][d].
 * ------------------------------------------------------------------------- */
int oracle_quant_v_fp4(const uint16_t* v, int64_t BH, int64_t N, int64_t d, int smooth, float* vm, float* gv,
                       uint8_t* codes, uint8_t* s8) {
    if (!v || !gv || !codes || !s8 || (smooth && !vm) || BH < 0 || N <= 0 || d <= 0 || N >= ((int64_t)1 << 23))
        return ORACLE_ERR_ARG;
    const int64_t ngt = (N + FP4_GROUP - 1) / FP4_GROUP;
#pragma omp parallel for collapse(2) schedule(static)
    for (int64_t bh = 0; bh < BH; ++bh) {
        for (int64_t c = 0; c < d; ++c) {
            const uint16_t* vh = v + bh * N * d;
            float mean = 0.0f;
            if (smooth) {
                int64_t s = 0;  /* exact: fp16 * 2^24 is an integer */
                for (int64_t t = 0; t < N; ++t) s += (int64_t)(h2d_sa3(vh[t * d + c]) * 16777216.0);
                mean = ((float)s / (float)N) * 0x1p-24f;
                vm[bh * d + c] = mean;
            }
            float a = 0.0f;
            for (int64_t t = 0; t < N; ++t) {
                const float x = (float)h2d_sa3(vh[t * d + c]) - mean;
                if (fabsf(x) > a) a = fabsf(x);
            }
            gv[bh * d + c] = a / FP4_RANGE;
            const float r = a > 0.0f ? FP4_RANGE / a : 0.0f;
            for (int64_t gt = 0; gt < ngt; ++gt) {
                float z[FP4_GROUP];
                uint8_t cc[FP4_GROUP];
                const int64_t t0 = gt * FP4_GROUP;
                const int n = (int)(t0 + FP4_GROUP <= N ? FP4_GROUP : N - t0);
                for (int k = 0; k < n; ++k) z[k] = ((float)h2d_sa3(vh[(t0 + k) * d + c]) - mean) * r;
                s8[(bh * ngt + gt) * d + c] = microscale(z, n, cc);
                for (int k = 0; k < n; ++k) codes[(bh * N + t0 + k) * d + c] = cc[k];
            }
        }
    }
    return ORACLE_OK;
}

/* ---------------------------------------------------------------------------
 * Attention rows.
 * ------------------------------------------------------------------------- */
/* distance of x > 0 to the nearest rounding midpoint of the E2M1 magnitudes, relative to x */
static int e2m1_near_midpoint(double x) {
    static const double mid[7] = {0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0};
    for (int k = 0; k < 7; ++k)
        if (fabs(x - mid[k]) <= NEAR_REL * x) return 1;
    return 0;
}

/* the E4M3 value next to a positive t on the other side of its nearest rounding midpoint,
 * or -1 when t is not within NEAR_REL of a midpoint */
static double e4m3_other_rounding(double t) {
    const uint8_t b = oracle_e4m3_encode(t);
    const double v = oracle_e4m3_decode(b);
    const double up = (b & 0x7F) < 0x7E ? oracle_e4m3_decode((uint8_t)(b + 1)) : v;
    const double dn = (b & 0x7F) > 0 ? oracle_e4m3_decode((uint8_t)(b - 1)) : v;
    if (up > v && fabs(t - 0.5 * (v + up)) <= NEAR_REL * t) return up;
    if (dn < v && fabs(t - 0.5 * (v + dn)) <= NEAR_REL * t) return dn;
    return -1.0;
}

/* P~ of one value z' = fl32(p * fl32(1/s)) at the scale s (as a double) */
static double pt_at_scale(float p32, double s) {
    const float inv = s > 0.0 ? 1.0f / (float)s : 0.0f;
    return oracle_e2m1_decode(oracle_e2m1_encode((double)(p32 * inv))) * s;
}

typedef struct {
    const uint8_t *q4, *qs, *k4, *ks, *v4, *vs; /* one head */
    const float *gq, *gk, *gv, *vm;
    int64_t N, d;
    int causal;
    double sm_scale;
} fp4_head;

/* One query row i: o64[0..d) (may be NULL), o16 (may be NULL), env[0..d) (may be NULL);
 * returns 1 when the row is unsure (an offset decision within 1e-4 of an integer).
 * Scratch: u [N], acc [d], eacc [d]. */
static int attn_fp4_row(const fp4_head* h, int64_t i, double* u, double* acc, double* eacc, double* o64,
                        uint16_t* o16, double* env) {
    const int64_t N = h->N, d = h->d, ng = d / FP4_GROUP, ngt = (N + FP4_GROUP - 1) / FP4_GROUP;
    const int64_t nt = (N + FP4_KTILE - 1) / FP4_KTILE;
    const int64_t jend = h->causal ? i + 1 : N;
    const double gqi = (double)h->gq[i / FP4_TILE];
    int unsure = 0;
    /* exact scores */
    for (int64_t j = 0; j < jend; ++j) {
        double S = 0.0;
        for (int64_t c = 0; c < d; ++c) {
            const double qa = oracle_e2m1_decode(h->q4[i * d + c]) * oracle_e4m3_decode(h->qs[i * ng + c / FP4_GROUP]);
            const double kb = oracle_e2m1_decode(h->k4[j * d + c]) * oracle_e4m3_decode(h->ks[j * ng + c / FP4_GROUP]);
            S += qa * kb;
        }
        u[j] = S * gqi * (double)h->gk[j / FP4_TILE] * h->sm_scale * 1.4426950408889634;
    }
    double m = -INFINITY, l = 0.0;
    for (int64_t c = 0; c < d; ++c) acc[c] = eacc[c] = 0.0;
    for (int64_t t = 0; t < nt && t * FP4_KTILE < jend; ++t) {
        const int64_t j0 = t * FP4_KTILE, j1 = (j0 + FP4_KTILE < jend) ? j0 + FP4_KTILE : jend;
        double tmax = -INFINITY;
        for (int64_t j = j0; j < j1; ++j)
            if (u[j] > tmax) tmax = u[j];
        if (fabs(tmax - nearbyint(tmax)) <= 1e-4) unsure = 1;
        const double mt = ceil(tmax);
        if (mt > m) {
            if (m != -INFINITY) {
                const double f = exp2(m - mt);
                l *= f;
                for (int64_t c = 0; c < d; ++c) { acc[c] *= f; eacc[c] *= f; }
            }
            m = mt;
        }
        /* 16-key groups of this tile (the tile's last group may be cut by jend) */
        for (int64_t jg = j0; jg < j1; jg += FP4_GROUP) {
            const int n = (int)(jg + FP4_GROUP <= j1 ? FP4_GROUP : j1 - jg);
            double p[FP4_GROUP];
            float p32[FP4_GROUP];
            double gm = 0.0;
            float gm32 = 0.0f;
            for (int k = 0; k < n; ++k) {
                p[k] = exp2(u[jg + k] - m + P_SHIFT);
                p32[k] = (float)p[k];
                l += p[k];
                if (p[k] > gm) gm = p[k];
                if (p32[k] > gm32) gm32 = p32[k];
            }
            uint8_t cc[FP4_GROUP];
            const uint8_t s8 = microscale(p32, n, cc);
            const double sd = oracle_e4m3_decode(s8);
            const double s_other = e4m3_other_rounding(gm / 6.0);
            for (int k = 0; k < n; ++k) {
                const int64_t j = jg + k;
                const double pt = oracle_e2m1_decode(cc[k]) * sd;
                /* envelope weight of this key: the other group scale, or the other code */
                double b = 0.0;
                if (s_other >= 0.0) {
                    b = fabs(pt - pt_at_scale(p32[k], s_other));
                    if (e2m1_near_midpoint(p[k] / s_other)) b += 2.0 * s_other;
                    if (e2m1_near_midpoint(p[k] / sd)) b += 2.0 * sd;
                } else if (sd > 0.0 && e2m1_near_midpoint(p[k] / sd)) {
                    b = 2.0 * sd;  /* at most one E2M1 step (the largest is 2) */
                }
                const int64_t grow = j / FP4_GROUP;
                for (int64_t c = 0; c < d; ++c) {
                    const double vh = oracle_e2m1_decode(h->v4[j * d + c]) * oracle_e4m3_decode(h->vs[grow * d + c]);
                    acc[c] += pt * vh;
                    if (b > 0.0) eacc[c] += b * fabs(vh);
                }
            }
        }
    }
    (void)ngt;
    for (int64_t c = 0; c < d; ++c) {
        const double gvc = (double)h->gv[c];
        const double o = acc[c] * gvc / l + (h->vm ? (double)h->vm[c] : 0.0);
        if (o64) o64[c] = o;
        if (o16) o16[c] = d2h_sa3(o);
        if (env) env[c] = eacc[c] * gvc / l;
    }
    return unsure;
}

static void head_at(fp4_head* h, const uint8_t* q4, const uint8_t* qs, const float* gq, const uint8_t* k4,
                    const uint8_t* ks, const float* gk, const uint8_t* v4, const uint8_t* vs, const float* gv,
                    const float* vm, int64_t bh, int64_t N, int64_t d, int causal, double sm_scale) {
    const int64_t ng = d / FP4_GROUP, nt = (N + FP4_TILE - 1) / FP4_TILE, ngt = (N + FP4_GROUP - 1) / FP4_GROUP;
    h->q4 = q4 + bh * N * d;
    h->qs = qs + bh * N * ng;
    h->gq = gq + bh * nt;
    h->k4 = k4 + bh * N * d;
    h->ks = ks + bh * N * ng;
    h->gk = gk + bh * nt;
    h->v4 = v4 + bh * N * d;
    h->vs = vs + bh * ngt * d;
    h->gv = gv + bh * d;
    h->vm = vm ? vm + bh * d : NULL;
    h->N = N;
    h->d = d;
    h->causal = causal;
    h->sm_scale = sm_scale;
}

/* All heads.  Layouts as oracle_quant_fp4 (q, k) and oracle_quant_v_fp4 (v); vm may be NULL.
 * o64, o16, env [BH][N][d] and unsure [BH][N] may each be NULL. */
int oracle_attn_fp4(const uint8_t* q4, const uint8_t* qs, const float* gq, const uint8_t* k4, const uint8_t* ks,
                    const float* gk, const uint8_t* v4, const uint8_t* vs, const float* gv, const float* vm,
                    int64_t BH, int64_t N, int64_t d, int causal, double sm_scale, double* o64, uint16_t* o16,
                    double* env, uint8_t* unsure) {
    if (!q4 || !qs || !gq || !k4 || !ks || !gk || !v4 || !vs || !gv || BH < 0 || N <= 0 || d <= 0 || d % FP4_GROUP)
        return ORACLE_ERR_ARG;
    int err = ORACLE_OK;
#pragma omp parallel
    {
        double* u = (double*)malloc(sizeof(double) * (size_t)N);
        double* acc = (double*)malloc(sizeof(double) * (size_t)d * 2);
        if (!u || !acc) {
#pragma omp atomic write
            err = ORACLE_ERR_NOMEM;
        } else {
#pragma omp for collapse(2) schedule(dynamic, 16)
            for (int64_t bh = 0; bh < BH; ++bh) {
                for (int64_t i = 0; i < N; ++i) {
                    fp4_head h;
                    head_at(&h, q4, qs, gq, k4, ks, gk, v4, vs, gv, vm, bh, N, d, causal, sm_scale);
                    const int64_t row = bh * N + i;
                    const int un = attn_fp4_row(&h, i, u, acc, acc + d, o64 ? o64 + row * d : NULL,
                                                o16 ? o16 + row * d : NULL, env ? env + row * d : NULL);
                    if (unsure) unsure[row] = (uint8_t)un;
                }
            }
        }
        free(u);
        free(acc);
    }
    return err;
}

/* Selected query rows of head bh (rows[r] in [0, N)): row r of o64 / env / unsure is rows[r]. */
int oracle_attn_fp4_rows(const uint8_t* q4, const uint8_t* qs, const float* gq, const uint8_t* k4, const uint8_t* ks,
                         const float* gk, const uint8_t* v4, const uint8_t* vs, const float* gv, const float* vm,
                         int64_t bh, int64_t N, int64_t d, int causal, double sm_scale, const int64_t* rows,
                         int64_t nrows, double* o64, double* env, uint8_t* unsure) {
    if (!q4 || !qs || !gq || !k4 || !ks || !gk || !v4 || !vs || !gv || !rows || !o64 || bh < 0 || N <= 0 || d <= 0 ||
        d % FP4_GROUP)
        return ORACLE_ERR_ARG;
    for (int64_t r = 0; r < nrows; ++r)
        if (rows[r] < 0 || rows[r] >= N) return ORACLE_ERR_ARG;
    int err = ORACLE_OK;
#pragma omp parallel
    {
        double* u = (double*)malloc(sizeof(double) * (size_t)N);
        double* acc = (double*)malloc(sizeof(double) * (size_t)d * 2);
        if (!u || !acc) {
#pragma omp atomic write
            err = ORACLE_ERR_NOMEM;
        } else {
#pragma omp for schedule(dynamic, 1)
            for (int64_t r = 0; r < nrows; ++r) {
                fp4_head h;
                head_at(&h, q4, qs, gq, k4, ks, gk, v4, vs, gv, vm, bh, N, d, causal, sm_scale);
                const int un = attn_fp4_row(&h, rows[r], u, acc, acc + d, o64 + r * d, NULL, env ? env + r * d : NULL);
                if (unsure) unsure[r] = (uint8_t)un;
            }
        }
        free(u);
        free(acc);
    }
    return err;
}
