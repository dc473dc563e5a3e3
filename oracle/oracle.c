/*
 * oracle.c - plain fp64 CPU oracle of the MoBA (Mixture of Block Attention)
 * causal prefill forward.
 *
 * TEST INFRASTRUCTURE ONLY. Nothing on the product path may link, load or call
 * this file; only the tests, the smoke check and the benchmark's CPU baseline
 * leg use it. It shares no code with the CUDA library.
 *
 * What it computes, step by step (page citations name the web page and the
 * part of it that states the step):
 *   1. Block partition: the context of N tokens is cut into blocks of
 *      block_size consecutive tokens; token t lies in block c = floor(t / B)
 *      ("MoBA tech-report summary", section 2, block partition paragraph;
 *      "MoBA project hub", Step 1).
 *   2. Mean pooling: the representative of block j is the mean of its keys
 *      (blog "KIMI MoBA", section 3 config field score_pooling = mean, and the
 *      section 4 block-selection simulation that averages each block's keys).
 *      Variants (the same blog, section 6, suggests trying max pooling or
 *      weighted pooling instead of the mean): max pooling takes, feature by
 *      feature, the largest key value of the block; weighted pooling takes
 *      sum_u w[u - jB] K[u] / sum_p w[p] with one caller-given non-negative
 *      weight per position inside a block.
 *   3. Parameter-less gating: the score of block j for query q is <q, Kbar_j>,
 *      no learned weights and no scaling ("MoBA project hub", Step 2; tech-
 *      report summary, section 2, relevance score s_i).
 *   4. Causality: blocks after the query's own block are never selected, the
 *      own block is always selected and masked causally inside (blog section
 *      3, causal_mask and current_block_force; tech-report summary, section 2,
 *      causality paragraph). The own block counts toward top_k, so k - 1 past
 *      blocks are chosen by score; ties go to the lower block index.
 *   5. Attention over the union of the selected blocks' keys (the own block
 *      only up to and including t), with logits q.k / sqrt(d) ("NSA vs MoBA"
 *      blog, section 1, the softmax(QK^T / sqrt(d)) V formula).
 *   6. The same result formed blockwise: one partial (O_j, lse_j) per selected
 *      block merged by log-sum-exp ("MoBA project hub", Step 3; tech-report
 *      summary, section 2, step 5 online-softmax combination).
 *
 * Layouts: Q [B, N, Hq, d], K and V [B, N, Hkv, d], bf16 bit patterns; query
 * head h reads kv head floor(h / (Hq / Hkv)). All arithmetic is in double.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

static inline double bf16_to_double(uint16_t h) {
    uint32_t u = (uint32_t)h << 16;
    float f;
    memcpy(&f, &u, 4);
    return (double)f;
}

/* Step 2: Kbar[b, h, j, :] = mean of K[b, jB .. jB+B-1, h, :] for every full block j. */
void oracle_pool(const uint16_t* K, int64_t B, int64_t N, int64_t Hkv, int64_t d, int64_t bs,
                 double* Kbar) {
    int64_t nfull = N / bs;
#pragma omp parallel for collapse(2) schedule(dynamic)
    for (int64_t b = 0; b < B; ++b)
        for (int64_t h = 0; h < Hkv; ++h)
            for (int64_t j = 0; j < nfull; ++j) {
                double* dst = Kbar + ((b * Hkv + h) * nfull + j) * d;
                for (int64_t e = 0; e < d; ++e) dst[e] = 0.0;
                for (int64_t u = j * bs; u < (j + 1) * bs; ++u) {
                    const uint16_t* src = K + ((b * N + u) * Hkv + h) * d;
                    for (int64_t e = 0; e < d; ++e) dst[e] += bf16_to_double(src[e]);
                }
                for (int64_t e = 0; e < d; ++e) dst[e] /= (double)bs;
            }
}

/* Step 2, variants. mode 1: Kbar[b, h, j, e] = max over the block's keys of K[u, e].
 * mode 2: Kbar[b, h, j, :] = sum_p w[p] K[jB + p] / sum_p w[p] (w: bs non-negative weights with a
 * positive sum). mode 0 is the mean (oracle_pool). */
void oracle_pool_mode(const uint16_t* K, int64_t B, int64_t N, int64_t Hkv, int64_t d, int64_t bs,
                      int64_t mode, const double* w, double* Kbar) {
    if (mode == 0) {
        oracle_pool(K, B, N, Hkv, d, bs, Kbar);
        return;
    }
    int64_t nfull = N / bs;
    double wsum = 0.0;
    if (mode == 2)
        for (int64_t p = 0; p < bs; ++p) wsum += w[p];
#pragma omp parallel for collapse(2) schedule(dynamic)
    for (int64_t b = 0; b < B; ++b)
        for (int64_t h = 0; h < Hkv; ++h)
            for (int64_t j = 0; j < nfull; ++j) {
                double* dst = Kbar + ((b * Hkv + h) * nfull + j) * d;
                for (int64_t e = 0; e < d; ++e) dst[e] = (mode == 1) ? -INFINITY : 0.0;
                for (int64_t u = j * bs; u < (j + 1) * bs; ++u) {
                    const uint16_t* src = K + ((b * N + u) * Hkv + h) * d;
                    for (int64_t e = 0; e < d; ++e) {
                        double x = bf16_to_double(src[e]);
                        if (mode == 1) {
                            if (x > dst[e]) dst[e] = x;
                        } else {
                            dst[e] += w[u - j * bs] * x;
                        }
                    }
                }
                if (mode == 2)
                    for (int64_t e = 0; e < d; ++e) dst[e] /= wsum;
            }
}

typedef struct {
    double s;
    int64_t j;
} cand_t;

/* Order of step 4: higher score first, lower block index among equal scores. */
static int cand_cmp(const void* a, const void* b) {
    const cand_t* x = (const cand_t*)a;
    const cand_t* y = (const cand_t*)b;
    if (x->s > y->s) return -1;
    if (x->s < y->s) return 1;
    return (x->j < y->j) ? -1 : (x->j > y->j);
}

static int i32_cmp(const void* a, const void* b) {
    int32_t x = *(const int32_t*)a, y = *(const int32_t*)b;
    return (x > y) - (x < y);
}

/*
 * Steps 1-4 for the listed rows (each row a triple b, hq, t).
 *   sel[r, 0..topk)  ascending selected block ids (own block last), -1 padded.
 *   s_last[r]        score of the lowest-ranked selected past block,
 *   s_next[r]        score of the best unselected past block,
 *                    both NaN when every past block is selected.
 *   scores (optional, may be NULL): [nrows, max_past] score of past block j,
 *                    NaN where j >= c.
 */
void oracle_select(const uint16_t* Q, const double* Kbar, int64_t B, int64_t N, int64_t Hq,
                   int64_t Hkv, int64_t d, int64_t bs, int64_t topk, const int64_t* rows,
                   int64_t nrows, int32_t* sel, double* s_last, double* s_next, double* scores,
                   int64_t max_past) {
    (void)B;
    int64_t nfull = N / bs;
    int64_t G = Hq / Hkv;
#pragma omp parallel
    {
        cand_t* cand = (cand_t*)malloc(sizeof(cand_t) * (size_t)(nfull + 1));
#pragma omp for schedule(dynamic, 16)
        for (int64_t r = 0; r < nrows; ++r) {
            int64_t b = rows[3 * r], hq = rows[3 * r + 1], t = rows[3 * r + 2];
            int64_t hk = hq / G;
            int64_t c = t / bs;
            const uint16_t* q = Q + ((b * N + t) * Hq + hq) * d;
            for (int64_t j = 0; j < c; ++j) {
                const double* kb = Kbar + ((b * Hkv + hk) * nfull + j) * d;
                double s = 0.0;
                for (int64_t e = 0; e < d; ++e) s += bf16_to_double(q[e]) * kb[e];
                cand[j].s = s;
                cand[j].j = j;
            }
            if (scores) {
                for (int64_t j = 0; j < max_past; ++j) scores[r * max_past + j] = (j < c) ? cand[j].s : NAN;
            }
            int64_t npast = c < topk - 1 ? c : topk - 1;
            s_last[r] = NAN;
            s_next[r] = NAN;
            if (c > topk - 1) {
                qsort(cand, (size_t)c, sizeof(cand_t), cand_cmp);
                if (npast > 0) s_last[r] = cand[npast - 1].s;
                s_next[r] = cand[npast].s;
            }
            int32_t* out = sel + r * topk;
            for (int64_t i = 0; i < npast; ++i) out[i] = (int32_t)cand[i].j;
            qsort(out, (size_t)npast, sizeof(int32_t), i32_cmp);
            out[npast] = (int32_t)c;
            for (int64_t i = npast + 1; i < topk; ++i) out[i] = -1;
        }
        free(cand);
    }
}

/* Key range of selected block j for query t: full for a past block, [cB, t] for the own block. */
static inline int block_range(int64_t j, int64_t t, int64_t bs, int64_t* lo, int64_t* hi) {
    int64_t c = t / bs;
    if (j < 0) return 0;
    if (j > c) return -1; /* a future block: never allowed */
    *lo = j * bs;
    *hi = (j == c) ? t + 1 : (j + 1) * bs;
    return 1;
}

/*
 * Step 5 for the listed rows with a given selection sel[nrows, topk] (-1 = none):
 * lse = ln sum_u exp(l_u), out = sum_u exp(l_u - lse) v_u over the allowed keys u,
 * l_u = q.k_u / sqrt(d). Returns the number of rows whose selection named a
 * future block or lacked the own block (those rows are left untouched).
 */
int64_t oracle_attend(const uint16_t* Q, const uint16_t* K, const uint16_t* V, int64_t B, int64_t N,
                      int64_t Hq, int64_t Hkv, int64_t d, int64_t bs, int64_t topk,
                      const int64_t* rows, int64_t nrows, const int32_t* sel, double* out, double* lse) {
    (void)B;
    int64_t G = Hq / Hkv;
    int64_t bad = 0;
    double scale = 1.0 / sqrt((double)d);
#pragma omp parallel
    {
        double* qv = (double*)malloc(sizeof(double) * (size_t)d);
        double* acc = (double*)malloc(sizeof(double) * (size_t)d);
        double* logit = (double*)malloc(sizeof(double) * (size_t)(topk * bs + 1));
        int64_t* key = (int64_t*)malloc(sizeof(int64_t) * (size_t)(topk * bs + 1));
#pragma omp for schedule(dynamic, 4) reduction(+ : bad)
        for (int64_t r = 0; r < nrows; ++r) {
            int64_t b = rows[3 * r], hq = rows[3 * r + 1], t = rows[3 * r + 2];
            int64_t hk = hq / G;
            int64_t c = t / bs;
            const int32_t* sr = sel + r * topk;
            int has_own = 0, ok = 1;
            for (int64_t i = 0; i < topk; ++i) {
                if (sr[i] == c) has_own = 1;
                if (sr[i] > c) ok = 0;
                for (int64_t i2 = 0; i2 < i; ++i2)
                    if (sr[i] >= 0 && sr[i2] == sr[i]) ok = 0; /* a block named twice */
            }
            if (!ok || !has_own) {
                bad += 1;
                continue;
            }
            for (int64_t e = 0; e < d; ++e) qv[e] = bf16_to_double(Q[((b * N + t) * Hq + hq) * d + e]);
            int64_t n = 0;
            double m = -INFINITY;
            for (int64_t i = 0; i < topk; ++i) {
                int64_t lo, hi;
                if (block_range(sr[i], t, bs, &lo, &hi) != 1) continue;
                for (int64_t u = lo; u < hi; ++u) {
                    const uint16_t* kr = K + ((b * N + u) * Hkv + hk) * d;
                    double s = 0.0;
                    for (int64_t e = 0; e < d; ++e) s += qv[e] * bf16_to_double(kr[e]);
                    logit[n] = s * scale;
                    key[n] = u;
                    if (logit[n] > m) m = logit[n];
                    ++n;
                }
            }
            double z = 0.0;
            for (int64_t i = 0; i < n; ++i) z += exp(logit[i] - m);
            double L = m + log(z);
            for (int64_t e = 0; e < d; ++e) acc[e] = 0.0;
            for (int64_t i = 0; i < n; ++i) {
                double p = exp(logit[i] - L);
                const uint16_t* vr = V + ((b * N + key[i]) * Hkv + hk) * d;
                for (int64_t e = 0; e < d; ++e) acc[e] += p * bf16_to_double(vr[e]);
            }
            for (int64_t e = 0; e < d; ++e) out[r * d + e] = acc[e];
            lse[r] = L;
        }
        free(qv);
        free(acc);
        free(logit);
        free(key);
    }
    return bad;
}

/*
 * Step 6: the same rows formed blockwise. Each selected block j gives a partial
 * (O_j normalised by its own sum, lse_j); the partials are merged with weights
 * exp(lse_j - LSE), LSE = ln sum_j exp(lse_j).
 */
int64_t oracle_attend_blockwise(const uint16_t* Q, const uint16_t* K, const uint16_t* V, int64_t B,
                                int64_t N, int64_t Hq, int64_t Hkv, int64_t d, int64_t bs,
                                int64_t topk, const int64_t* rows, int64_t nrows, const int32_t* sel,
                                double* out, double* lse) {
    (void)B;
    int64_t G = Hq / Hkv;
    int64_t bad = 0;
    double scale = 1.0 / sqrt((double)d);
#pragma omp parallel
    {
        double* qv = (double*)malloc(sizeof(double) * (size_t)d);
        double* po = (double*)malloc(sizeof(double) * (size_t)(topk * d));
        double* pl = (double*)malloc(sizeof(double) * (size_t)topk);
        double* logit = (double*)malloc(sizeof(double) * (size_t)bs);
#pragma omp for schedule(dynamic, 4) reduction(+ : bad)
        for (int64_t r = 0; r < nrows; ++r) {
            int64_t b = rows[3 * r], hq = rows[3 * r + 1], t = rows[3 * r + 2];
            int64_t hk = hq / G;
            const int32_t* sr = sel + r * topk;
            for (int64_t e = 0; e < d; ++e) qv[e] = bf16_to_double(Q[((b * N + t) * Hq + hq) * d + e]);
            int64_t np = 0, rowbad = 0;
            for (int64_t i = 0; i < topk; ++i) {
                int64_t lo, hi;
                int k = block_range(sr[i], t, bs, &lo, &hi);
                if (k < 0) rowbad = 1;
                if (k != 1) continue;
                double m = -INFINITY;
                for (int64_t u = lo; u < hi; ++u) {
                    const uint16_t* kr = K + ((b * N + u) * Hkv + hk) * d;
                    double s = 0.0;
                    for (int64_t e = 0; e < d; ++e) s += qv[e] * bf16_to_double(kr[e]);
                    logit[u - lo] = s * scale;
                    if (logit[u - lo] > m) m = logit[u - lo];
                }
                double z = 0.0;
                for (int64_t u = lo; u < hi; ++u) z += exp(logit[u - lo] - m);
                double Lj = m + log(z);
                double* o = po + np * d;
                for (int64_t e = 0; e < d; ++e) o[e] = 0.0;
                for (int64_t u = lo; u < hi; ++u) {
                    double p = exp(logit[u - lo] - Lj);
                    const uint16_t* vr = V + ((b * N + u) * Hkv + hk) * d;
                    for (int64_t e = 0; e < d; ++e) o[e] += p * bf16_to_double(vr[e]);
                }
                pl[np++] = Lj;
            }
            if (rowbad || np == 0) {
                bad += 1;
                continue;
            }
            double m = -INFINITY;
            for (int64_t i = 0; i < np; ++i)
                if (pl[i] > m) m = pl[i];
            double z = 0.0;
            for (int64_t i = 0; i < np; ++i) z += exp(pl[i] - m);
            double L = m + log(z);
            for (int64_t e = 0; e < d; ++e) out[r * d + e] = 0.0;
            for (int64_t i = 0; i < np; ++i) {
                double w = exp(pl[i] - L);
                for (int64_t e = 0; e < d; ++e) out[r * d + e] += w * po[i * d + e];
            }
            lse[r] = L;
        }
        free(qv);
        free(po);
        free(pl);
        free(logit);
    }
    return bad;
}

/*
 * Step 7 (the backward of steps 5-6, for training: "MoBA tech-report summary", section 3
 * trains and continues pre-training models with MoBA). With the selection fixed (the top-k
 * choice is discrete, so the block representatives receive no gradient; only the attention is
 * differentiated), for the loss sum over rows of <dO_t, out_t>:
 *   P_tu = exp(l_u - lse_t) over the row's allowed keys u, l_u = q_t.k_u / sqrt(d)
 *   D_t  = sum_e dO_t[e] out_t[e]
 *   dP_tu = dO_t . v_u,   dS_tu = P_tu (dP_tu - D_t)
 *   dQ_t = sum_u dS_tu k_u / sqrt(d),  dK_u += dS_tu q_t / sqrt(d),  dV_u += P_tu dO_t
 * with out_t and lse_t the row's own forward (recomputed here in fp64). GQA: a kv head sums the
 * contributions of its query heads. sel: [B, Hq, N, topk] for every row. Outputs in fp64:
 * dQ [B, N, Hq, d], dK and dV [B, N, Hkv, d] (zeroed here). Returns the number of rows whose
 * selection was malformed (left without contributions).
 */
int64_t oracle_backward(const uint16_t* Q, const uint16_t* K, const uint16_t* V, const uint16_t* dO,
                        int64_t B, int64_t N, int64_t Hq, int64_t Hkv, int64_t d, int64_t bs,
                        int64_t topk, const int32_t* sel, double* dQ, double* dK, double* dV) {
    int64_t G = Hq / Hkv;
    double scale = 1.0 / sqrt((double)d);
    int64_t bad = 0;
    memset(dQ, 0, sizeof(double) * (size_t)(B * N * Hq * d));
    memset(dK, 0, sizeof(double) * (size_t)(B * N * Hkv * d));
    memset(dV, 0, sizeof(double) * (size_t)(B * N * Hkv * d));
#pragma omp parallel for collapse(2) schedule(dynamic) reduction(+ : bad)
    for (int64_t b = 0; b < B; ++b)
        for (int64_t hk = 0; hk < Hkv; ++hk) {
            /* one (b, kv head) per thread: its dK / dV rows are written by this thread only */
            double* qv = (double*)malloc(sizeof(double) * (size_t)d);
            double* gv = (double*)malloc(sizeof(double) * (size_t)d);
            double* ov = (double*)malloc(sizeof(double) * (size_t)d);
            double* logit = (double*)malloc(sizeof(double) * (size_t)(topk * bs + 1));
            int64_t* key = (int64_t*)malloc(sizeof(int64_t) * (size_t)(topk * bs + 1));
            for (int64_t g = 0; g < G; ++g) {
                int64_t hq = hk * G + g;
                for (int64_t t = 0; t < N; ++t) {
                    int64_t c = t / bs;
                    const int32_t* sr = sel + ((b * Hq + hq) * N + t) * topk;
                    int has_own = 0, ok = 1;
                    for (int64_t i = 0; i < topk; ++i) {
                        if (sr[i] == c) has_own = 1;
                        if (sr[i] > c) ok = 0;
                        for (int64_t i2 = 0; i2 < i; ++i2)
                            if (sr[i] >= 0 && sr[i2] == sr[i]) ok = 0;
                    }
                    if (!ok || !has_own) {
                        bad += 1;
                        continue;
                    }
                    for (int64_t e = 0; e < d; ++e) {
                        qv[e] = bf16_to_double(Q[((b * N + t) * Hq + hq) * d + e]);
                        gv[e] = bf16_to_double(dO[((b * N + t) * Hq + hq) * d + e]);
                    }
                    int64_t n = 0;
                    double m = -INFINITY;
                    for (int64_t i = 0; i < topk; ++i) {
                        int64_t lo, hi;
                        if (block_range(sr[i], t, bs, &lo, &hi) != 1) continue;
                        for (int64_t u = lo; u < hi; ++u) {
                            const uint16_t* kr = K + ((b * N + u) * Hkv + hk) * d;
                            double s = 0.0;
                            for (int64_t e = 0; e < d; ++e) s += qv[e] * bf16_to_double(kr[e]);
                            logit[n] = s * scale;
                            key[n] = u;
                            if (logit[n] > m) m = logit[n];
                            ++n;
                        }
                    }
                    double z = 0.0;
                    for (int64_t i = 0; i < n; ++i) z += exp(logit[i] - m);
                    double L = m + log(z);
                    /* the row's output and D */
                    for (int64_t e = 0; e < d; ++e) ov[e] = 0.0;
                    for (int64_t i = 0; i < n; ++i) {
                        double p = exp(logit[i] - L);
                        const uint16_t* vr = V + ((b * N + key[i]) * Hkv + hk) * d;
                        for (int64_t e = 0; e < d; ++e) ov[e] += p * bf16_to_double(vr[e]);
                    }
                    double D = 0.0;
                    for (int64_t e = 0; e < d; ++e) D += gv[e] * ov[e];
                    double* dq = dQ + ((b * N + t) * Hq + hq) * d;
                    for (int64_t i = 0; i < n; ++i) {
                        double p = exp(logit[i] - L);
                        const uint16_t* kr = K + ((b * N + key[i]) * Hkv + hk) * d;
                        const uint16_t* vr = V + ((b * N + key[i]) * Hkv + hk) * d;
                        double dp = 0.0;
                        for (int64_t e = 0; e < d; ++e) dp += gv[e] * bf16_to_double(vr[e]);
                        double ds = p * (dp - D);
                        double* dk = dK + ((b * N + key[i]) * Hkv + hk) * d;
                        double* dv = dV + ((b * N + key[i]) * Hkv + hk) * d;
                        for (int64_t e = 0; e < d; ++e) {
                            dq[e] += ds * bf16_to_double(kr[e]) * scale;
                            dk[e] += ds * qv[e] * scale;
                            dv[e] += p * gv[e];
                        }
                    }
                }
            }
            free(qv);
            free(gv);
            free(ov);
            free(logit);
            free(key);
        }
    return bad;
}
