/*
 * sage_oracle_sparse.c -- plain, slow CPU oracle for the block-sparse variant of the 8-bit
 * attention forward pass.
 *
 * TEST INFRASTRUCTURE ONLY (linked with sage_oracle.c): nothing in the product path links,
 * loads or calls it, and it shares no code with the CUDA library.
 *
 * What it computes follows the SpargeAttn abstract ("SpargeAttention: Accurate and Training-
 * free Sparse Attention Accelerating Any Model Inference", author pages of Jia Wei and Haofeng
 * Huang): a sparse and quantized attention with a two-stage online filter --
 * the first stage predicts the attention map quickly, so that some matrix products are skipped;
 * the second, a softmax-aware filter inside the online softmax, skips further products.  The
 * abstract gives no formulas; the readings:
 *
 *   Blocks      query blocks of BQ = 256 tokens, key blocks of BK = 128 tokens, tiling each
 *               (batch, head) from token 0 (the last block of each kind may be partial).
 *   Stage 1     Each block is represented by the mean of its tokens (q_bar, k_bar).  The
 *               predicted map of query block i is P^_i = softmax_j(q_bar_i . k_bar_j * sm_scale)
 *               over the key blocks it may see (causal: blocks j with j * BK <= the block's
 *               last query).  It keeps the fewest key blocks, taken in decreasing P^, whose
 *               probabilities sum to at least tau (ties in P^ broken by the lower index).
 *               A block's mean represents it only if its tokens point alike: its self-
 *               similarity, the mean cosine over all ordered pairs of its tokens (self-pairs
 *               included, a zero token counting as cosine 0), |sum_t x_t / |x_t||^2 / n^2, must
 *               be at least theta; a query block below theta keeps every key block it may
 *               see, a key block below theta is kept by every query block that may see it.
 *               Causal: the diagonal key blocks (those holding one of the block's own queries)
 *               are always kept, so every query keeps its own key.
 *   Stage 2     Within a kept block pair, query tiles of 128 rows visit their kept key blocks
 *               in increasing order; m_run(r) is the largest score (log2 units) of row r over
 *               the key blocks visited so far.  A key block is skipped for the whole query
 *               tile when, for every row r of the tile (rows past N excluded), its largest
 *               score is below m_run(r) - lambda: its weights are all below 2^-lambda of the
 *               running maximum.  The first visited block is never skipped.
 *   Attention   The 8-bit attention of sage_oracle.c (INT8 scores, fp64 softmax, P~ rounded to
 *               fp16, fp64 P.V) over the keys of the blocks that are kept and not skipped.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define ORACLE_OK 0
#define ORACLE_ERR_ARG -1
#define ORACLE_ERR_NOMEM -5

static double h2d_sp(uint16_t bits) {
    _Float16 h;
    memcpy(&h, &bits, sizeof h);
    return (double)h;
}

static uint16_t d2h_sp(double v) {
    _Float16 h = (_Float16)v;
    uint16_t bits;
    memcpy(&bits, &h, sizeof bits);
    return bits;
}

/* Mean (fp64) and self-similarity of the n token rows of x [n][d] (fp16 bits). */
static double block_stats(const uint16_t* x, int64_t n, int64_t d, double* mean, double* unit_sum) {
    for (int64_t c = 0; c < d; ++c) mean[c] = 0.0, unit_sum[c] = 0.0;
    for (int64_t t = 0; t < n; ++t) {
        double nrm = 0.0;
        for (int64_t c = 0; c < d; ++c) {
            const double v = h2d_sp(x[t * d + c]);
            mean[c] += v;
            nrm += v * v;
        }
        nrm = sqrt(nrm);
        if (nrm > 0.0)
            for (int64_t c = 0; c < d; ++c) unit_sum[c] += h2d_sp(x[t * d + c]) / nrm;
    }
    double s2 = 0.0;
    for (int64_t c = 0; c < d; ++c) {
        mean[c] /= (double)n;
        s2 += unit_sum[c] * unit_sum[c];
    }
    return s2 / ((double)n * (double)n);
}

/* Stage 1.  q, k: fp16 [BH][N][d].  mask: uint8 [BH][NQB][NKB] (1 = kept), NQB = ceil(N/256),
 * NKB = ceil(N/128).  unsure (may be NULL): 1 where the decision sits within eps of flipping
 * (a self-similarity within eps of theta, a cumulative probability within eps of tau at the
 * cut, or probabilities within eps of each other across the cut); qsim / ksim (may be NULL):
 * the blocks' self-similarities [BH][NQB] / [BH][NKB]. */
int oracle_sparse_predict(const uint16_t* q, const uint16_t* k, int64_t BH, int64_t N, int64_t d, int causal,
                          double sm_scale, double tau, double theta, double eps, uint8_t* mask, uint8_t* unsure,
                          double* qsim_out, double* ksim_out) {
    if (!q || !k || !mask || BH < 0 || N <= 0 || d <= 0) return ORACLE_ERR_ARG;
    const int64_t BQ = 256, BK = 128;
    const int64_t NQB = (N + BQ - 1) / BQ, NKB = (N + BK - 1) / BK;
    int err = ORACLE_OK;
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t bh = 0; bh < BH; ++bh) {
        double* qbar = (double*)malloc(sizeof(double) * (size_t)(NQB * d));
        double* kbar = (double*)malloc(sizeof(double) * (size_t)(NKB * d));
        double* qs = (double*)malloc(sizeof(double) * (size_t)NQB);
        double* ks = (double*)malloc(sizeof(double) * (size_t)NKB);
        double* tmp = (double*)malloc(sizeof(double) * (size_t)d);
        double* p = (double*)malloc(sizeof(double) * (size_t)NKB);
        int64_t* order = (int64_t*)malloc(sizeof(int64_t) * (size_t)NKB);
        if (!qbar || !kbar || !qs || !ks || !tmp || !p || !order) {
#pragma omp atomic write
            err = ORACLE_ERR_NOMEM;
        } else {
            const uint16_t* qh = q + bh * N * d;
            const uint16_t* kh = k + bh * N * d;
            for (int64_t i = 0; i < NQB; ++i) {
                const int64_t t0 = i * BQ, n = (t0 + BQ < N ? BQ : N - t0);
                qs[i] = block_stats(qh + t0 * d, n, d, qbar + i * d, tmp);
            }
            for (int64_t j = 0; j < NKB; ++j) {
                const int64_t t0 = j * BK, n = (t0 + BK < N ? BK : N - t0);
                ks[j] = block_stats(kh + t0 * d, n, d, kbar + j * d, tmp);
            }
            if (qsim_out) memcpy(qsim_out + bh * NQB, qs, sizeof(double) * (size_t)NQB);
            if (ksim_out) memcpy(ksim_out + bh * NKB, ks, sizeof(double) * (size_t)NKB);
            for (int64_t i = 0; i < NQB; ++i) {
                uint8_t* mrow = mask + (bh * NQB + i) * NKB;
                uint8_t* urow = unsure ? unsure + (bh * NQB + i) * NKB : NULL;
                const int64_t last_q = (i + 1) * BQ < N ? (i + 1) * BQ - 1 : N - 1;
                const int64_t nvis = causal ? last_q / BK + 1 : NKB;  /* key blocks this block may see */
                for (int64_t j = 0; j < NKB; ++j) {
                    mrow[j] = 0;
                    if (urow) urow[j] = 0;
                }
                /* compressed map and its softmax over the visible key blocks */
                double mx = -INFINITY;
                for (int64_t j = 0; j < nvis; ++j) {
                    double s = 0.0;
                    for (int64_t c = 0; c < d; ++c) s += qbar[i * d + c] * kbar[j * d + c];
                    p[j] = s * sm_scale;
                    if (p[j] > mx) mx = p[j];
                }
                double z = 0.0;
                for (int64_t j = 0; j < nvis; ++j) z += (p[j] = exp(p[j] - mx));
                for (int64_t j = 0; j < nvis; ++j) p[j] /= z;
                /* key blocks in decreasing probability (insertion sort; ties: lower index first) */
                for (int64_t a = 0; a < nvis; ++a) {
                    int64_t b = a;
                    order[a] = a;
                    while (b > 0 && (p[order[b - 1]] < p[a] || (p[order[b - 1]] == p[a] && order[b - 1] > a))) {
                        order[b] = order[b - 1];
                        --b;
                    }
                    order[b] = a;
                }
                double cum = 0.0;
                int64_t cut = 0; /* blocks order[0..cut) are kept by the cumulative rule */
                while (cut < nvis && cum < tau) cum += p[order[cut++]];
                for (int64_t a = 0; a < cut; ++a) mrow[order[a]] = 1;
                if (urow) {
                    /* the cut moves if the sum before the last kept block (or the sum with the
                     * first dropped one) is within eps of tau, or the probabilities on both sides
                     * of the cut are within eps of each other */
                    double before_last = cum - p[order[cut - 1]];
                    const int near_cut = fabs(before_last - tau) < eps || fabs(cum - tau) < eps ||
                                         (cut < nvis && fabs(p[order[cut - 1]] - p[order[cut]]) < eps);
                    if (near_cut) {
                        urow[order[cut - 1]] = 1;
                        if (cut < nvis) urow[order[cut]] = 1;
                    }
                }
                /* self-similarity overrides and the causal diagonal */
                const int q_alike = qs[i] >= theta;
                for (int64_t j = 0; j < nvis; ++j) {
                    if (!q_alike || ks[j] < theta) mrow[j] = 1;
                    if (causal && (j + 1) * BK > i * BQ) mrow[j] = 1; /* block j holds a query of block i */
                    if (urow && (fabs(qs[i] - theta) < eps || fabs(ks[j] - theta) < eps)) urow[j] = 1;
                }
            }
        }
        free(qbar); free(kbar); free(qs); free(ks); free(tmp); free(p); free(order);
    }
    return err;
}

/* Stage 2 and the attention of one query tile of 128 rows (rows r0 .. r0+127 that exist) of
 * one head.  Writes O rows; skipped (optional, uint8 [NKB]) receives 1 for each kept key block
 * stage 2 skipped for this tile.  s: N doubles of scratch per row of the tile (128 * N). */
static void sparse_tile(const int8_t* q8h, const int8_t* k8h, const float* sqh, const float* skh, const uint16_t* vh,
                        int64_t N, int64_t d, int causal, double sm_scale, int64_t gq, int64_t gk,
                        const uint8_t* mrow, double lambda, int64_t r0, double* s, double* acc, double* mrun,
                        uint8_t* used, double* o64, uint16_t* o16, uint8_t* skipped) {
    const int64_t BK = 128, NKB = (N + BK - 1) / BK;
    const int64_t r1 = r0 + 128 < N ? r0 + 128 : N;
    /* scores of the whole tile (log2 units for the filter; natural units kept in s) */
    for (int64_t i = r0; i < r1; ++i) {
        mrun[i - r0] = -INFINITY;
        const int8_t* qi = q8h + i * d;
        for (int64_t j = 0; j < N; ++j) {
            const int8_t* kj = k8h + j * d;
            int64_t dot = 0;
            for (int64_t c = 0; c < d; ++c) dot += (int64_t)qi[c] * (int64_t)kj[c];
            s[(i - r0) * N + j] = (double)dot * (double)sqh[i / gq] * (double)skh[j / gk] * sm_scale;
        }
    }
    for (int64_t b = 0; b < NKB; ++b) {
        used[b] = 0;
        if (skipped) skipped[b] = 0;
    }
    for (int64_t b = 0; b < NKB; ++b) {
        if (!mrow[b]) continue;
        const int64_t j0 = b * BK, j1 = j0 + BK < N ? j0 + BK : N;
        if (causal && j0 > r1 - 1) continue; /* no row of the tile sees this block */
        int skip = 1; /* m_run starts at -inf, so the first visited block is never skipped */
        double bmax[128];
        for (int64_t i = r0; i < r1; ++i) {
            double m = -INFINITY;
            for (int64_t j = j0; j < j1; ++j)
                if (!causal || j <= i) {
                    const double u = s[(i - r0) * N + j] * 1.4426950408889634;
                    if (u > m) m = u;
                }
            bmax[i - r0] = m;
            if (!(m < mrun[i - r0] - lambda)) skip = 0;
        }
        if (skip) {
            if (skipped) skipped[b] = 1;
            continue;
        }
        used[b] = 1;
        for (int64_t i = r0; i < r1; ++i)
            if (bmax[i - r0] > mrun[i - r0]) mrun[i - r0] = bmax[i - r0];
    }
    /* softmax and P.V of every row over the keys of the used blocks */
    for (int64_t i = r0; i < r1; ++i) {
        const double* si = s + (i - r0) * N;
        double m = -INFINITY;
        for (int64_t j = 0; j < N; ++j)
            if (used[j / BK] && (!causal || j <= i) && si[j] > m) m = si[j];
        double l = 0.0;
        for (int64_t c = 0; c < d; ++c) acc[c] = 0.0;
        for (int64_t j = 0; j < N; ++j) {
            if (!used[j / BK] || (causal && j > i)) continue;
            const double e = exp(si[j] - m);
            l += e;
            const double pt = h2d_sp(d2h_sp(e));
            for (int64_t c = 0; c < d; ++c) acc[c] += pt * h2d_sp(vh[j * d + c]);
        }
        for (int64_t c = 0; c < d; ++c) {
            const double o = acc[c] / l;
            if (o64) o64[i * d + c] = o;
            if (o16) o16[i * d + c] = d2h_sp(o);
        }
    }
}

/* Block-sparse 8-bit attention for all heads: mask [BH][ceil(N/256)][ceil(N/128)] from stage 1
 * (any 0/1 map with every query's own diagonal block kept when causal), lambda the stage-2
 * threshold in log2 units (INFINITY: no stage 2).  skipped (may be NULL): uint8
 * [BH][ceil(N/128)][ceil(N/128)], 1 where stage 2 skipped key block b for query tile t. */
int oracle_attn_sparse(const int8_t* q8, const int8_t* k8, const float* sq, const float* sk, const uint16_t* v,
                       int64_t BH, int64_t N, int64_t d, int causal, double sm_scale, int64_t gq, int64_t gk,
                       const uint8_t* mask, double lambda, double* o64, uint16_t* o16, uint8_t* skipped) {
    if (!q8 || !k8 || !sq || !sk || !v || !mask || BH < 0 || N <= 0 || d <= 0 || gq <= 0 || gk <= 0)
        return ORACLE_ERR_ARG;
    const int64_t NQB = (N + 255) / 256, NKB = (N + 127) / 128, NQT = (N + 127) / 128;
    const int64_t nsq = (N + gq - 1) / gq, nsk = (N + gk - 1) / gk;
    int err = ORACLE_OK;
#pragma omp parallel
    {
        double* s = (double*)malloc(sizeof(double) * (size_t)(128 * N));
        double* acc = (double*)malloc(sizeof(double) * (size_t)d);
        double* mrun = (double*)malloc(sizeof(double) * 128);
        uint8_t* used = (uint8_t*)malloc((size_t)NKB);
        if (!s || !acc || !mrun || !used) {
#pragma omp atomic write
            err = ORACLE_ERR_NOMEM;
        } else {
#pragma omp for collapse(2) schedule(dynamic, 1)
            for (int64_t bh = 0; bh < BH; ++bh) {
                for (int64_t t = 0; t < NQT; ++t) {
                    sparse_tile(q8 + bh * N * d, k8 + bh * N * d, sq + bh * nsq, sk + bh * nsk, v + bh * N * d, N, d,
                                causal, sm_scale, gq, gk, mask + (bh * NQB + t / 2) * NKB, lambda, t * 128, s, acc,
                                mrun, used, o64 ? o64 + bh * N * d : NULL, o16 ? o16 + bh * N * d : NULL,
                                skipped ? skipped + (bh * NQT + t) * NKB : NULL);
                }
            }
        }
        free(s); free(acc); free(mrun); free(used);
    }
    return err;
}

/* Only the listed query tiles (128 rows each, tiles[r] in [0, ceil(N/128))) of one head: row i
 * of tile r goes to o64[(r * 128 + i) * d] (rows past N untouched); skipped (may be NULL): uint8
 * [ntiles][ceil(N/128)] as in oracle_attn_sparse.  mask: this head's [ceil(N/256)][ceil(N/128)]. */
int oracle_attn_sparse_tiles(const int8_t* q8h, const int8_t* k8h, const float* sqh, const float* skh,
                             const uint16_t* vh, int64_t N, int64_t d, int causal, double sm_scale, int64_t gq,
                             int64_t gk, const uint8_t* maskh, double lambda, const int64_t* tiles, int64_t ntiles,
                             double* o64, uint8_t* skipped) {
    if (!q8h || !k8h || !sqh || !skh || !vh || !maskh || !tiles || !o64 || N <= 0 || d <= 0 || gq <= 0 || gk <= 0)
        return ORACLE_ERR_ARG;
    const int64_t NKB = (N + 127) / 128, NQT = (N + 127) / 128;
    for (int64_t r = 0; r < ntiles; ++r)
        if (tiles[r] < 0 || tiles[r] >= NQT) return ORACLE_ERR_ARG;
    int err = ORACLE_OK;
#pragma omp parallel
    {
        double* s = (double*)malloc(sizeof(double) * (size_t)(128 * N));
        double* acc = (double*)malloc(sizeof(double) * (size_t)d);
        double* mrun = (double*)malloc(sizeof(double) * 128);
        uint8_t* used = (uint8_t*)malloc((size_t)NKB);
        double* rows64 = (double*)malloc(sizeof(double) * (size_t)(N * d));
        if (!s || !acc || !mrun || !used || !rows64) {
#pragma omp atomic write
            err = ORACLE_ERR_NOMEM;
        } else {
#pragma omp for schedule(dynamic, 1)
            for (int64_t r = 0; r < ntiles; ++r) {
                const int64_t t = tiles[r];
                sparse_tile(q8h, k8h, sqh, skh, vh, N, d, causal, sm_scale, gq, gk, maskh + (t / 2) * NKB, lambda,
                            t * 128, s, acc, mrun, used, rows64, NULL, skipped ? skipped + r * NKB : NULL);
                const int64_t r1 = t * 128 + 128 < N ? t * 128 + 128 : N;
                for (int64_t i = t * 128; i < r1; ++i)
                    for (int64_t c = 0; c < d; ++c) o64[(r * 128 + (i - t * 128)) * d + c] = rows64[i * d + c];
            }
        }
        free(s); free(acc); free(mrun); free(used); free(rows64);
    }
    return err;
}
