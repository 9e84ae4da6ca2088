/*
 * CPU oracle for the Rectified Sparse Attention (ReSA) decode hot path.
 *
 * TEST INFRASTRUCTURE ONLY.  This file is the plain, slow, obviously correct
 * statement of what the CUDA library computes.  It shares no code, header,
 * table or helper with the CUDA path; only the tests, the smoke check and the
 * benchmark's CPU-baseline leg may load it.  The product path never calls it.
 *
 * Source ("ReSA summary"): the page "Rectified Sparse Attention" of the
 * paper-graph-ui summary of arXiv 2506.04108.  Section / equation numbers
 * below refer to that page.
 *
 * Precision (each choice is stated where it is made):
 *   - K, V, q arrive as bf16 bit patterns; widening bf16 -> float is exact.
 *   - Descriptors are min/max of bf16 values, so they are exact bf16.
 *   - The pooled query and the block scores are fp32, summed in index order:
 *     they decide an integer (the selected block set), so they are computed in
 *     the precision the kernels use for the same decision.
 *   - Attention logits, softmax and the weighted value sum accumulate in fp64.
 *
 * Readings of points the pages leave open (listed again in the design notes):
 *   - seq_len counts the decode token, which is appended before attending;
 *     the current block c = (L-1)/b holds positions c*b .. L-1 and is always
 *     attended (local window, n_local = 1) but never scored.
 *   - complete blocks are 0 .. M-1 with M = (L-1)/b; only they are scored.
 *   - k_eff = min(topk, M); ties in score go to the lower block index.
 *   - positions >= L are excluded outright (zero weight) instead of the
 *     pages' -1e6 padding logit; both give a zero softmax weight.
 *   - rectification writes the fresh K/V first, then runs causal attention:
 *     chunk row r (position L-f+r) sees positions 0 .. L-f+r.
 *
 * Layouts (caller's buffers, one layer):
 *   K, V        [num_pages][Hkv][bs][d]      bf16 bits (uint16)
 *   desc        [num_pages][Hkv][2][d]       bf16 bits, row 0 = min, row 1 = max
 *   page_table  [B][max_pages]               int32
 *   seq_len     [B]                          int32
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

static float bf16_to_float(uint16_t x) {
    uint32_t u = ((uint32_t)x) << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return f;
}

static size_t kv_index(const int32_t *page_table, int max_pages, int b, int h, int t,
                       int j, int hkv, int bs, int d) {
    int page = page_table[(size_t)b * max_pages + t / bs];
    return ((((size_t)page * hkv + h) * bs + (t % bs)) * d) + j;
}

static size_t desc_index(int page, int h, int which, int j, int hkv, int d) {
    return (((size_t)page * hkv + h) * 2 + which) * d + j;
}

/* Eq. 3 (ReSA summary §3.4.1): element-wise min and max over the keys of one
 * block, taken over the block's valid tokens t < L in position order.  The
 * comparison keeps the earlier value on equality, so the result is a bit
 * pattern of one of the keys. */
static void describe_block(const uint16_t *K, uint16_t *desc, const int32_t *page_table,
                           int max_pages, int b, int h, int blk, int L, int hkv, int bs,
                           int d) {
    int t0 = blk * bs;
    int t1 = t0 + bs < L ? t0 + bs : L;
    if (t1 <= t0) return;
    int page = page_table[(size_t)b * max_pages + blk];
    for (int j = 0; j < d; ++j) {
        uint16_t mn = K[kv_index(page_table, max_pages, b, h, t0, j, hkv, bs, d)];
        uint16_t mx = mn;
        for (int t = t0 + 1; t < t1; ++t) {
            uint16_t x = K[kv_index(page_table, max_pages, b, h, t, j, hkv, bs, d)];
            if (bf16_to_float(x) < bf16_to_float(mn)) mn = x;
            if (bf16_to_float(x) > bf16_to_float(mx)) mx = x;
        }
        desc[desc_index(page, h, 0, j, hkv, d)] = mn;
        desc[desc_index(page, h, 1, j, hkv, d)] = mx;
    }
}

/* Block key cache construction after prefill (Algorithm 1, initialisation):
 * descriptors of every block that holds at least one token, the partial last
 * block over its valid tokens only.  first_block (nullable) skips blocks
 * below first_block[b]. */
void oracle_build_descriptors(const uint16_t *K, uint16_t *desc, const int32_t *page_table,
                              const int32_t *seq_len, const int32_t *first_block, int B,
                              int hkv, int d, int bs, int max_pages) {
#pragma omp parallel for collapse(2) schedule(dynamic)
    for (int b = 0; b < B; ++b)
        for (int h = 0; h < hkv; ++h) {
            int L = seq_len[b];
            int nblk = (L + bs - 1) / bs;
            int from = first_block ? first_block[b] : 0;
            for (int blk = from; blk < nblk; ++blk)
                describe_block(K, desc, page_table, max_pages, b, h, blk, L, hkv, bs, d);
        }
}

/* Algorithm 1, incremental cache update: the decode token (position L-1,
 * seq_len already counts it) is written to K/V; its key is folded into the
 * last block's min/max, or starts a new block when L-1 is a block boundary. */
void oracle_append(uint16_t *K, uint16_t *V, uint16_t *desc, const uint16_t *k_new,
                   const uint16_t *v_new, const int32_t *page_table, const int32_t *seq_len,
                   int B, int hkv, int d, int bs, int max_pages) {
    for (int b = 0; b < B; ++b) {
        int pos = seq_len[b] - 1;
        int page = page_table[(size_t)b * max_pages + pos / bs];
        for (int h = 0; h < hkv; ++h)
            for (int j = 0; j < d; ++j) {
                uint16_t kx = k_new[((size_t)b * hkv + h) * d + j];
                uint16_t vx = v_new[((size_t)b * hkv + h) * d + j];
                K[kv_index(page_table, max_pages, b, h, pos, j, hkv, bs, d)] = kx;
                V[kv_index(page_table, max_pages, b, h, pos, j, hkv, bs, d)] = vx;
                uint16_t *mn = &desc[desc_index(page, h, 0, j, hkv, d)];
                uint16_t *mx = &desc[desc_index(page, h, 1, j, hkv, d)];
                if (pos % bs == 0) {
                    *mn = kx;
                    *mx = kx;
                } else {
                    if (bf16_to_float(kx) < bf16_to_float(*mn)) *mn = kx;
                    if (bf16_to_float(kx) > bf16_to_float(*mx)) *mx = kx;
                }
            }
    }
}

/* Group query pooling (ReSA summary §3.4.1, "Group pooling and pattern
 * sharing"): the g query heads of a GQA group are averaged into one query,
 * fp32, summed in head order then divided by g. */
void oracle_pooled_query(const uint16_t *q, float *qbar, int B, int hq, int hkv, int d) {
    int g = hq / hkv;
    for (int b = 0; b < B; ++b)
        for (int h = 0; h < hkv; ++h)
            for (int j = 0; j < d; ++j) {
                float s = 0.0f;
                for (int r = 0; r < g; ++r) s += bf16_to_float(q[((size_t)b * hq + h * g + r) * d + j]);
                qbar[((size_t)b * hkv + h) * d + j] = s / (float)g;
            }
}

/* Eq. 4 (ReSA summary §3.4.1): score_i = sum_j max(q_j * max_ij, q_j * min_ij)
 * for every complete block i < M, fp32, summed in j order.  Entries i >= M of
 * scores[b][h][*] are left untouched. */
void oracle_block_scores(const float *qbar, const uint16_t *desc, const int32_t *page_table,
                         const int32_t *seq_len, float *scores, int B, int hkv, int d, int bs,
                         int max_pages) {
    for (int b = 0; b < B; ++b) {
        int M = (seq_len[b] - 1) / bs;
#pragma omp parallel for collapse(2) schedule(static)
        for (int h = 0; h < hkv; ++h)
            for (int i = 0; i < M; ++i) {
                int page = page_table[(size_t)b * max_pages + i];
                const float *qv = &qbar[((size_t)b * hkv + h) * d];
                float s = 0.0f;
                for (int j = 0; j < d; ++j) {
                    float lo = qv[j] * bf16_to_float(desc[desc_index(page, h, 0, j, hkv, d)]);
                    float hi = qv[j] * bf16_to_float(desc[desc_index(page, h, 1, j, hkv, d)]);
                    s += (hi > lo ? hi : lo);
                }
                scores[((size_t)b * hkv + h) * max_pages + i] = s;
            }
    }
}

typedef struct {
    float score;
    int32_t idx;
} scored_block;

/* Higher score first; equal scores: lower block index first. */
static int by_score_then_index(const void *a, const void *b) {
    const scored_block *x = (const scored_block *)a, *y = (const scored_block *)b;
    if (x->score > y->score) return -1;
    if (x->score < y->score) return 1;
    return (x->idx > y->idx) - (x->idx < y->idx);
}

static int ascending_int(const void *a, const void *b) {
    int32_t x = *(const int32_t *)a, y = *(const int32_t *)b;
    return (x > y) - (x < y);
}

/* Top-n block selection (Eq. 5 count supplied by the caller as topk[b]) with
 * the local window n_local = 1 (ReSA summary §3.4.1, "Dynamic top-n with
 * guards"): the k_eff = min(topk, M) best complete blocks, listed in
 * ascending block order, followed by the current block c = M.  The same set
 * serves every query head of the group.  block_idx is [B][hkv][max_topk+1];
 * block_cnt[b][h] = k_eff + 1. */
void oracle_select(const float *scores, const int32_t *topk, const int32_t *seq_len,
                   int32_t *block_idx, int32_t *block_cnt, int max_topk, int B, int hkv,
                   int bs, int max_pages) {
    for (int b = 0; b < B; ++b) {
        int M = (seq_len[b] - 1) / bs;
        int k = topk[b] < M ? topk[b] : M;
        if (k < 0) k = 0;
        for (int h = 0; h < hkv; ++h) {
            scored_block *all = (scored_block *)malloc(sizeof(scored_block) * (M > 0 ? M : 1));
            for (int i = 0; i < M; ++i) {
                all[i].score = scores[((size_t)b * hkv + h) * max_pages + i];
                all[i].idx = i;
            }
            qsort(all, (size_t)M, sizeof(scored_block), by_score_then_index);
            int32_t *out = &block_idx[((size_t)b * hkv + h) * (max_topk + 1)];
            for (int i = 0; i < k; ++i) out[i] = all[i].idx;
            qsort(out, (size_t)k, sizeof(int32_t), ascending_int);
            out[k] = M;
            block_cnt[(size_t)b * hkv + h] = k + 1;
            free(all);
        }
    }
}

/* Softmax attention of one query vector over a list of token positions, fp64:
 * logits z_t = sm_scale * q.k_t, weights exp(z_t - max) / sum, output the
 * weighted sum of v_t; lse = max + log(sum).  Eq. 1 when the list is every
 * position, Eq. 2 (GBSA) when it is the positions of the selected blocks. */
static void attend(const uint16_t *qv, const uint16_t *K, const uint16_t *V,
                   const int32_t *page_table, int max_pages, int b, int h, const int32_t *pos,
                   int npos, double sm_scale, int hkv, int bs, int d, double *out,
                   double *lse) {
    double *z = (double *)malloc(sizeof(double) * (npos > 0 ? npos : 1));
    double zmax = -INFINITY;
    for (int n = 0; n < npos; ++n) {
        double s = 0.0;
        for (int j = 0; j < d; ++j)
            s += (double)bf16_to_float(qv[j]) *
                 (double)bf16_to_float(K[kv_index(page_table, max_pages, b, h, pos[n], j, hkv, bs, d)]);
        z[n] = s * sm_scale;
        if (z[n] > zmax) zmax = z[n];
    }
    double sum = 0.0;
    for (int n = 0; n < npos; ++n) {
        z[n] = exp(z[n] - zmax);
        sum += z[n];
    }
    for (int j = 0; j < d; ++j) out[j] = 0.0;
    for (int n = 0; n < npos; ++n) {
        double w = z[n] / sum;
        for (int j = 0; j < d; ++j)
            out[j] += w * (double)bf16_to_float(V[kv_index(page_table, max_pages, b, h, pos[n], j, hkv, bs, d)]);
    }
    if (lse) *lse = npos > 0 ? zmax + log(sum) : -INFINITY;
    free(z);
}

/* Eq. 2 (GBSA, ReSA summary §3.4.1): each query head (h, r) of sequence b
 * attends to the token positions t < L of the blocks listed in
 * block_idx[b][h][0 .. block_cnt-1].  out is [B][hq][d] fp64, lse [B][hq]. */
void oracle_sparse_attention(const uint16_t *q, const uint16_t *K, const uint16_t *V,
                             const int32_t *page_table, const int32_t *seq_len,
                             const int32_t *block_idx, const int32_t *block_cnt, int max_topk,
                             float sm_scale, double *out, double *lse, int B, int hq, int hkv,
                             int d, int bs, int max_pages) {
    int g = hq / hkv;
#pragma omp parallel for collapse(2) schedule(dynamic)
    for (int b = 0; b < B; ++b)
        for (int qh = 0; qh < hq; ++qh) {
            int h = qh / g;
            int L = seq_len[b];
            int cnt = block_cnt[(size_t)b * hkv + h];
            const int32_t *blocks = &block_idx[((size_t)b * hkv + h) * (max_topk + 1)];
            int32_t *pos = (int32_t *)malloc(sizeof(int32_t) * (size_t)(cnt > 0 ? cnt : 1) * bs);
            int npos = 0;
            for (int c = 0; c < cnt; ++c)
                for (int t = blocks[c] * bs; t < blocks[c] * bs + bs; ++t)
                    if (t < L) pos[npos++] = t;
            attend(&q[((size_t)b * hq + qh) * d], K, V, page_table, max_pages, b, h, pos, npos,
                   (double)sm_scale, hkv, bs, d, &out[((size_t)b * hq + qh) * d],
                   lse ? &lse[(size_t)b * hq + qh] : NULL);
            free(pos);
        }
}

/* Dense rectification (ReSA summary §3.4.2, "Operational mechanics"; Algorithm
 * 1, rectification check):
 *   1. overwrite K/V at positions L-f .. L-1 with the freshly computed
 *      entries k_new/v_new [B][f][hkv][d];
 *   2. recompute the descriptors of every block those positions touch;
 *   3. causal dense attention of the chunk queries q_chunk [B][f][hq][d]:
 *      row r (position L-f+r) attends to positions 0 .. L-f+r.
 * out is [B][f][hq][d] fp64, lse [B][f][hq] (nullable). */
void oracle_rectify(const uint16_t *q_chunk, const uint16_t *k_new, const uint16_t *v_new,
                    uint16_t *K, uint16_t *V, uint16_t *desc, const int32_t *page_table,
                    const int32_t *seq_len, int f, float sm_scale, double *out, double *lse,
                    int B, int hq, int hkv, int d, int bs, int max_pages) {
    int g = hq / hkv;
    for (int b = 0; b < B; ++b) {
        int L = seq_len[b];
        if (f > L) continue; /* a chunk longer than the sequence leaves it untouched */
        for (int r = 0; r < f; ++r)
            for (int h = 0; h < hkv; ++h)
                for (int j = 0; j < d; ++j) {
                    size_t src = (((size_t)b * f + r) * hkv + h) * d + j;
                    size_t dst = kv_index(page_table, max_pages, b, h, L - f + r, j, hkv, bs, d);
                    K[dst] = k_new[src];
                    V[dst] = v_new[src];
                }
        for (int h = 0; h < hkv; ++h)
            for (int blk = (L - f) / bs; blk <= (L - 1) / bs; ++blk)
                describe_block(K, desc, page_table, max_pages, b, h, blk, L, hkv, bs, d);
    }
#pragma omp parallel for collapse(3) schedule(dynamic)
    for (int b = 0; b < B; ++b)
        for (int r = 0; r < f; ++r)
            for (int qh = 0; qh < hq; ++qh) {
                int L = seq_len[b];
                if (f > L) continue;
                int last = L - f + r;
                int32_t *pos = (int32_t *)malloc(sizeof(int32_t) * (size_t)(last + 1));
                for (int t = 0; t <= last; ++t) pos[t] = t;
                size_t row = ((size_t)b * f + r) * hq + qh;
                attend(&q_chunk[row * d], K, V, page_table, max_pages, b, qh / g, pos, last + 1,
                       (double)sm_scale, hkv, bs, d, &out[row * d], lse ? &lse[row] : NULL);
                free(pos);
            }
}

/* Eq. 1 (ReSA summary §3.4.1): dense decode attention of q [B][hq][d] over
 * every position 0 .. L-1.  The baseline the sparse path is compared with. */
void oracle_dense_attention(const uint16_t *q, const uint16_t *K, const uint16_t *V,
                            const int32_t *page_table, const int32_t *seq_len, float sm_scale,
                            double *out, double *lse, int B, int hq, int hkv, int d, int bs,
                            int max_pages) {
    int g = hq / hkv;
#pragma omp parallel for collapse(2) schedule(dynamic)
    for (int b = 0; b < B; ++b)
        for (int qh = 0; qh < hq; ++qh) {
            int L = seq_len[b];
            int32_t *pos = (int32_t *)malloc(sizeof(int32_t) * (size_t)(L > 0 ? L : 1));
            for (int t = 0; t < L; ++t) pos[t] = t;
            attend(&q[((size_t)b * hq + qh) * d], K, V, page_table, max_pages, b, qh / g, pos, L,
                   (double)sm_scale, hkv, bs, d, &out[((size_t)b * hq + qh) * d],
                   lse ? &lse[(size_t)b * hq + qh] : NULL);
            free(pos);
        }
}

int oracle_num_threads(void) {
#ifdef _OPENMP
    extern int omp_get_max_threads(void);
    return omp_get_max_threads();
#else
    return 1;
#endif
}

/* Thread count of the parallel loops above (timing harness control only; the
 * results do not depend on it: every output element is computed by one thread
 * in the same order). */
void oracle_set_num_threads(int n) {
#ifdef _OPENMP
    extern void omp_set_num_threads(int);
    if (n > 0) omp_set_num_threads(n);
#else
    (void)n;
#endif
}
