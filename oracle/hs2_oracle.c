/*
 * hs2_oracle.c -- plain, slow, fp64 CPU oracle for HySparse2's Cross-Decoder
 * attention hot path.  TEST INFRASTRUCTURE ONLY: the product path (the CUDA
 * library and its Python binding) never links, loads or calls this file.
 * Only the tests, the smoke check and the benchmark's CPU-baseline leg use it.
 *
 * What it computes, per query token ("row") at absolute position t of one
 * sequence, following the HySparse2 pages:
 *   - "KV Reuse" (xiawanshe.com report, section "两级KV共享", second level):
 *     one full-attention layer of the Cross-Decoder produces the KV cache AND
 *     a token-selection result; several following sparse-attention layers
 *     reuse both.
 *   - "Token-level selection" (same report, section "Token级选择"): tokens are
 *     picked one by one; the most recent 128 tokens are always kept and 1024
 *     tokens are picked from the older context; local and global attention
 *     share one KV cache.  The davidyin.dev video notes (section "HySparse2
 *     的解法") add that no extra indexer is trained.
 *
 * Where the pages are silent this file takes the readings below (each one is
 * the plainest reading the pages support):
 *   - softmax scale 1/sqrt(D), causal row j in [0, t], natural-log LSE;
 *   - heads map to KV groups contiguously: g = h / G, G = H_q / H_kv;
 *   - window(t) = [max(0, t-W+1), t] (W tokens including t itself);
 *     candidates are j in [0, t-W], n_cand = max(0, t-W+1);
 *   - selection score of candidate j for group g = sum over the G heads of the
 *     group of the causal softmax probability p_{h,t,j} (normalised over the
 *     whole causal row, window included);
 *   - the selection takes the min(K, n_cand) candidates first in the order
 *     (score descending, j ascending) -- ties go to the lower index -- and is
 *     emitted sorted ascending by j, padded with -1;
 *   - a sparse layer attends, per head, to the set idx_g(t) U window(t) with
 *     its own query, same K/V, same 1/sqrt(D) scale;
 *   - block-level selection (the predecessor design the "Token级选择" section
 *     contrasts with) keeps whole blocks of blk contiguous candidate tokens,
 *     blocks ranked by the sum of their tokens' scores, at the same budget;
 *   - the predecessor design's sparse layer had two branches, a sliding-window
 *     attention over its own cache and an attention over the selected tokens
 *     of the shared cache; both are returned, uncombined (the pages do not
 *     say how they were combined);
 *   - "KV Bridging" (same report and section, first level) computes a token's
 *     K and V from its Self-Decoder hidden state with one projection (no
 *     bias, no normalisation or position encoding: the pages name none); the
 *     projection's output features are [K heads 0..H_kv-1 | V heads], each
 *     head D contiguous features.
 *
 * Every quantity is computed in double precision from the bf16 inputs widened
 * exactly (bf16 bits << 16 is an exact fp32, and fp32 -> fp64 is exact).
 * No blocking, no online softmax, no fusion: each step is the textbook
 * definition written out.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define HS2O_OK 0
#define HS2O_EINVAL 1
#define HS2O_ENOMEM 2
#define HS2O_EIDX 3

static double bf16_to_double(uint16_t b) {
    uint32_t u = ((uint32_t)b) << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

typedef struct {
    double score;
    int64_t j;
} cand_t;

/* Order "first is better": larger score first, then smaller j. */
static int cand_cmp(const void* a, const void* b) {
    const cand_t* x = (const cand_t*)a;
    const cand_t* y = (const cand_t*)b;
    if (x->score > y->score) return -1;
    if (x->score < y->score) return 1;
    if (x->j < y->j) return -1;
    if (x->j > y->j) return 1;
    return 0;
}

static int i32_cmp(const void* a, const void* b) {
    int32_t x = *(const int32_t*)a, y = *(const int32_t*)b;
    return (x > y) - (x < y);
}

/* s[j] = scale * <q_h, k_{g,j}> for j in [0, n). */
static void dot_scores(const uint16_t* qh, const uint16_t* kg, int64_t n, int d,
                       double scale, double* s) {
    double qd[512];
    for (int e = 0; e < d; ++e) qd[e] = bf16_to_double(qh[e]);
    for (int64_t j = 0; j < n; ++j) {
        const uint16_t* kj = kg + j * (int64_t)d;
        double acc = 0.0;
        for (int e = 0; e < d; ++e) acc += qd[e] * bf16_to_double(kj[e]);
        s[j] = acc * scale;
    }
}

/*
 * Full causal attention + selection for n_rows query tokens of ONE sequence.
 *
 * q      [n_rows, h_q, d]        bf16 bits, the full-attention layer's queries
 * t      [n_rows]                absolute position of each query (0 <= t < kv_len)
 * k, v   [h_kv, kv_stride, d]    bf16 bits, the shared cache of the sequence
 * out    [n_rows, h_q, d]        softmax(s) . v, fp64
 * lse    [n_rows, h_q]           ln sum_j exp(s_j), fp64
 * idx    [n_rows, h_kv, topk]    selection, ascending, -1 padded
 * kth    [n_rows, h_kv]          score of the last selected candidate in rank
 *                                order (NAN when nothing is selected)
 * next   [n_rows, h_kv]          score of the best unselected candidate
 *                                (-1 when every candidate is selected)
 * scores [n_rows, h_kv, score_stride] or NULL: score of every candidate
 *                                j in [0, t-window] (entries beyond n_cand untouched)
 */
int hs2o_full_select(int h_q, int h_kv, int d, int window, int topk, double scale,
                     int64_t n_rows, const int64_t* t, const uint16_t* q,
                     const uint16_t* k, const uint16_t* v, int64_t kv_len, int64_t kv_stride,
                     double* out, double* lse, int32_t* idx, double* kth, double* next,
                     double* scores, int64_t score_stride, int n_threads) {
    if (h_q <= 0 || h_kv <= 0 || h_q % h_kv != 0 || d <= 0 || d > 512 || window < 1 ||
        topk < 0 || n_rows < 0 || kv_len > kv_stride)
        return HS2O_EINVAL;
    for (int64_t r = 0; r < n_rows; ++r)
        if (t[r] < 0 || t[r] >= kv_len) return HS2O_EINVAL;
    const int G = h_q / h_kv;
    int err = HS2O_OK;
    const int64_t n_work = n_rows * h_kv;
#ifdef _OPENMP
    if (n_threads > 0) omp_set_num_threads(n_threads);
#pragma omp parallel for schedule(dynamic, 1)
#endif
    for (int64_t w = 0; w < n_work; ++w) {
        const int64_t r = w / h_kv;
        const int g = (int)(w % h_kv);
        const int64_t tr = t[r];
        const int64_t n_causal = tr + 1;
        const int64_t n_cand = tr - window + 1 > 0 ? tr - window + 1 : 0;
        double* s = (double*)malloc(sizeof(double) * (size_t)n_causal);
        double* grp = (double*)calloc((size_t)(n_cand > 0 ? n_cand : 1), sizeof(double));
        cand_t* cand = (cand_t*)malloc(sizeof(cand_t) * (size_t)(n_cand > 0 ? n_cand : 1));
        if (!s || !grp || !cand) {
            free(s); free(grp); free(cand);
#ifdef _OPENMP
#pragma omp atomic write
#endif
            err = HS2O_ENOMEM;
            continue;
        }
        const uint16_t* kg = k + (int64_t)g * kv_stride * d;
        const uint16_t* vg = v + (int64_t)g * kv_stride * d;
        for (int hh = 0; hh < G; ++hh) {
            const int h = g * G + hh;
            const uint16_t* qh = q + (r * h_q + h) * (int64_t)d;
            /* step 1: scaled dot products over the causal row */
            dot_scores(qh, kg, n_causal, d, scale, s);
            /* step 2: lse = m + ln sum exp(s - m) */
            double m = -INFINITY;
            for (int64_t j = 0; j < n_causal; ++j) m = s[j] > m ? s[j] : m;
            double z = 0.0;
            for (int64_t j = 0; j < n_causal; ++j) z += exp(s[j] - m);
            const double l = m + log(z);
            lse[r * h_q + h] = l;
            /* out_h = sum_j exp(s_j - lse) v_j */
            double* o = out + (r * h_q + h) * (int64_t)d;
            for (int e = 0; e < d; ++e) o[e] = 0.0;
            for (int64_t j = 0; j < n_causal; ++j) {
                const double p = exp(s[j] - l);
                const uint16_t* vj = vg + j * (int64_t)d;
                for (int e = 0; e < d; ++e) o[e] += p * bf16_to_double(vj[e]);
            }
            /* step 3: group score = sum over the group's heads of p_{h,j} */
            for (int64_t j = 0; j < n_cand; ++j) grp[j] += exp(s[j] - l);
        }
        /* step 4: rank candidates by (score desc, j asc), keep the first n */
        for (int64_t j = 0; j < n_cand; ++j) {
            cand[j].score = grp[j];
            cand[j].j = j;
        }
        if (scores)
            for (int64_t j = 0; j < n_cand; ++j) scores[(r * h_kv + g) * score_stride + j] = grp[j];
        qsort(cand, (size_t)n_cand, sizeof(cand_t), cand_cmp);
        const int64_t n_sel = n_cand < topk ? n_cand : topk;
        int32_t* row_idx = idx + (r * h_kv + g) * (int64_t)topk;
        for (int64_t i = 0; i < n_sel; ++i) row_idx[i] = (int32_t)cand[i].j;
        qsort(row_idx, (size_t)n_sel, sizeof(int32_t), i32_cmp);
        for (int64_t i = n_sel; i < topk; ++i) row_idx[i] = -1;
        kth[r * h_kv + g] = n_sel > 0 ? cand[n_sel - 1].score : NAN;
        next[r * h_kv + g] = n_sel < n_cand ? cand[n_sel].score : -1.0;
        free(s);
        free(grp);
        free(cand);
    }
    return err;
}

/*
 * One sparse (KV-reuse) layer for n_rows query tokens of ONE sequence:
 * per head h, softmax attention of the layer's own query over the set
 * idx_{g}(t) U window(t), g = h / G.
 *
 * idx [n_rows, h_kv, topk]: entries are -1 (unused) or a candidate index in
 * [0, t-window]; duplicates are rejected (HS2O_EIDX).
 */
int hs2o_sparse(int h_q, int h_kv, int d, int window, int topk, double scale,
                int64_t n_rows, const int64_t* t, const uint16_t* q,
                const uint16_t* k, const uint16_t* v, int64_t kv_len, int64_t kv_stride,
                const int32_t* idx, double* out, int n_threads) {
    if (h_q <= 0 || h_kv <= 0 || h_q % h_kv != 0 || d <= 0 || d > 512 || window < 1 ||
        topk < 0 || n_rows < 0 || kv_len > kv_stride)
        return HS2O_EINVAL;
    for (int64_t r = 0; r < n_rows; ++r)
        if (t[r] < 0 || t[r] >= kv_len) return HS2O_EINVAL;
    const int G = h_q / h_kv;
    int err = HS2O_OK;
    const int64_t n_work = n_rows * h_kv;
#ifdef _OPENMP
    if (n_threads > 0) omp_set_num_threads(n_threads);
#pragma omp parallel for schedule(dynamic, 1)
#endif
    for (int64_t w = 0; w < n_work; ++w) {
        const int64_t r = w / h_kv;
        const int g = (int)(w % h_kv);
        const int64_t tr = t[r];
        const int64_t w0 = tr - window + 1 > 0 ? tr - window + 1 : 0;
        /* the attended set: selected candidates, then the window */
        int64_t* set = (int64_t*)malloc(sizeof(int64_t) * (size_t)(topk + window));
        double* s = (double*)malloc(sizeof(double) * (size_t)(topk + window));
        if (!set || !s) {
            free(set); free(s);
#ifdef _OPENMP
#pragma omp atomic write
#endif
            err = HS2O_ENOMEM;
            continue;
        }
        int64_t n = 0;
        int bad = 0;
        const int32_t* ir = idx + (r * h_kv + g) * (int64_t)topk;
        for (int i = 0; i < topk; ++i) {
            const int64_t j = ir[i];
            if (j == -1) continue;
            if (j < 0 || j > tr - window) { bad = 1; break; }
            for (int64_t u = 0; u < n; ++u)
                if (set[u] == j) { bad = 1; break; }
            if (bad) break;
            set[n++] = j;
        }
        if (bad) {
            free(set); free(s);
#ifdef _OPENMP
#pragma omp atomic write
#endif
            err = HS2O_EIDX;
            continue;
        }
        for (int64_t j = w0; j <= tr; ++j) set[n++] = j;
        const uint16_t* kg = k + (int64_t)g * kv_stride * d;
        const uint16_t* vg = v + (int64_t)g * kv_stride * d;
        for (int hh = 0; hh < G; ++hh) {
            const int h = g * G + hh;
            const uint16_t* qh = q + (r * h_q + h) * (int64_t)d;
            double qd[512];
            for (int e = 0; e < d; ++e) qd[e] = bf16_to_double(qh[e]);
            double m = -INFINITY;
            for (int64_t u = 0; u < n; ++u) {
                const uint16_t* kj = kg + set[u] * (int64_t)d;
                double acc = 0.0;
                for (int e = 0; e < d; ++e) acc += qd[e] * bf16_to_double(kj[e]);
                s[u] = acc * scale;
                m = s[u] > m ? s[u] : m;
            }
            double z = 0.0;
            for (int64_t u = 0; u < n; ++u) z += exp(s[u] - m);
            double* o = out + (r * h_q + h) * (int64_t)d;
            for (int e = 0; e < d; ++e) o[e] = 0.0;
            for (int64_t u = 0; u < n; ++u) {
                const double p = exp(s[u] - m) / z;
                const uint16_t* vj = vg + set[u] * (int64_t)d;
                for (int e = 0; e < d; ++e) o[e] += p * bf16_to_double(vj[e]);
            }
        }
        free(set);
        free(s);
    }
    return err;
}

/* Softmax attention of one fp64 query over the n rows set[] of one head's K/V:
 * out = sum_u p_u v_{set[u]}, p_u = exp(s_u - lse), s_u = scale <q, k_{set[u]}>,
 * lse = ln sum_u exp(s_u).  n = 0 gives out = 0 and lse = -inf. */
static void attend_rows(const double* qd, const uint16_t* kg, const uint16_t* vg, const int64_t* set, int64_t n,
                        int d, double scale, double* s, double* out, double* lse) {
    for (int e = 0; e < d; ++e) out[e] = 0.0;
    if (n == 0) {
        *lse = -INFINITY;
        return;
    }
    double m = -INFINITY;
    for (int64_t u = 0; u < n; ++u) {
        const uint16_t* kj = kg + set[u] * (int64_t)d;
        double acc = 0.0;
        for (int e = 0; e < d; ++e) acc += qd[e] * bf16_to_double(kj[e]);
        s[u] = acc * scale;
        m = s[u] > m ? s[u] : m;
    }
    double z = 0.0;
    for (int64_t u = 0; u < n; ++u) z += exp(s[u] - m);
    for (int64_t u = 0; u < n; ++u) {
        const double pu = exp(s[u] - m) / z;
        const uint16_t* vj = vg + set[u] * (int64_t)d;
        for (int e = 0; e < d; ++e) out[e] += pu * bf16_to_double(vj[e]);
    }
    *lse = m + log(z);
}

/* The two attention branches of a sparse layer in the predecessor design
 * (xiawanshe.com report, section "Token级选择": HySparse2 drops the separate
 * sliding-window branch of the Cross-Decoder and keeps the recent tokens in
 * the one shared cache instead).  Per row and head h (g = h / G):
 *   window branch:   softmax attention over window(t) = [max(0, t-W+1), t] of
 *                    the branch's OWN cache k_swa, v_swa;
 *   selected branch: softmax attention over the selected set idx_g(t) alone
 *                    (no window) of the shared cache k, v.
 * Each writes its output [n_rows, h_q, d] and natural-log LSE [n_rows, h_q];
 * a row with no selected key gets a zero output and LSE -inf.  The pages do
 * not say how the predecessor combined the two branches, so both are
 * returned.  idx entries are -1 or a candidate index in [0, t-W], no
 * duplicates (HS2O_EIDX otherwise). */
int hs2o_branches(int h_q, int h_kv, int d, int window, int topk, double scale, int64_t n_rows, const int64_t* t,
                  const uint16_t* q, const uint16_t* k_swa, const uint16_t* v_swa, const uint16_t* k,
                  const uint16_t* v, int64_t kv_len, const int32_t* idx, double* out_swa, double* lse_swa,
                  double* out_sel, double* lse_sel, int n_threads) {
    if (h_q <= 0 || h_kv <= 0 || h_q % h_kv != 0 || d <= 0 || d > 512 || window < 1 || topk < 0 || n_rows < 0)
        return HS2O_EINVAL;
    for (int64_t r = 0; r < n_rows; ++r)
        if (t[r] < 0 || t[r] >= kv_len) return HS2O_EINVAL;
    const int G = h_q / h_kv;
    int err = HS2O_OK;
#ifdef _OPENMP
    if (n_threads > 0) omp_set_num_threads(n_threads);
#pragma omp parallel for schedule(dynamic, 1)
#endif
    for (int64_t w = 0; w < n_rows * h_kv; ++w) {
        const int64_t r = w / h_kv;
        const int g = (int)(w % h_kv);
        const int64_t tr = t[r];
        const int64_t w0 = tr - window + 1 > 0 ? tr - window + 1 : 0;
        const int64_t cap = (topk > window ? topk : window) + 1;
        int64_t* wset = (int64_t*)malloc(sizeof(int64_t) * (size_t)cap);
        int64_t* sset = (int64_t*)malloc(sizeof(int64_t) * (size_t)cap);
        double* s = (double*)malloc(sizeof(double) * (size_t)cap);
        if (!wset || !sset || !s) {
            free(wset); free(sset); free(s);
#ifdef _OPENMP
#pragma omp atomic write
#endif
            err = HS2O_ENOMEM;
            continue;
        }
        int64_t nw = 0, ns = 0;
        for (int64_t j = w0; j <= tr; ++j) wset[nw++] = j;
        int bad = 0;
        const int32_t* ir = idx + (r * h_kv + g) * (int64_t)topk;
        for (int i = 0; i < topk && !bad; ++i) {
            const int64_t j = ir[i];
            if (j == -1) continue;
            if (j < 0 || j > tr - window) bad = 1;
            for (int64_t u = 0; u < ns && !bad; ++u)
                if (sset[u] == j) bad = 1;
            if (!bad) sset[ns++] = j;
        }
        if (bad) {
            free(wset); free(sset); free(s);
#ifdef _OPENMP
#pragma omp atomic write
#endif
            err = HS2O_EIDX;
            continue;
        }
        const int64_t off = (int64_t)g * kv_len * d;
        for (int hh = 0; hh < G; ++hh) {
            const int h = g * G + hh;
            const uint16_t* qh = q + (r * h_q + h) * (int64_t)d;
            double qd[512];
            for (int e = 0; e < d; ++e) qd[e] = bf16_to_double(qh[e]);
            const int64_t o = (r * h_q + h) * (int64_t)d;
            attend_rows(qd, k_swa + off, v_swa + off, wset, nw, d, scale, s, out_swa + o, lse_swa + r * h_q + h);
            attend_rows(qd, k + off, v + off, sset, ns, d, scale, s, out_sel + o, lse_sel + r * h_q + h);
        }
        free(wset);
        free(sset);
        free(s);
    }
    return err;
}

/* Block-level selection, the predecessor design (xiawanshe.com report, section
 * "Token级选择": the previous HySparse picked whole contiguous blocks of
 * tokens).  From the per-candidate group scores written by hs2o_full_select:
 * block b holds tokens [b*blk, (b+1)*blk); the candidate blocks are those lying
 * entirely in [0, t-window], n_blk = (t - window + 1) / blk of them; a block's
 * score is the sum of its tokens' scores; the first min(topk / blk, n_blk)
 * blocks in the order (score desc, b asc) are kept and their tokens emitted
 * ascending, -1 padded to topk.  kth_block (or NULL) gets the score of the last
 * kept block in rank order (NAN when none is kept).
 * scores [n_rows, h_kv, score_stride]; idx [n_rows, h_kv, topk]. */
int hs2o_block_select(int64_t n_rows, int h_kv, int window, int topk, int blk, const int64_t* t,
                      const double* scores, int64_t score_stride, int32_t* idx, double* kth_block,
                      double* next_block) {
    if (n_rows < 0 || h_kv <= 0 || window < 1 || topk < 0 || blk <= 0) return HS2O_EINVAL;
    int err = HS2O_OK;
    for (int64_t w = 0; w < n_rows * h_kv; ++w) {
        const int64_t r = w / h_kv;
        const int64_t n_cand = t[r] - window + 1 > 0 ? t[r] - window + 1 : 0;
        const int64_t n_blk = n_cand / blk;
        const int64_t keep = n_blk < topk / blk ? n_blk : topk / blk;
        cand_t* cb = (cand_t*)malloc(sizeof(cand_t) * (size_t)(n_blk > 0 ? n_blk : 1));
        if (!cb) {
            err = HS2O_ENOMEM;
            continue;
        }
        const double* row = scores + w * score_stride;
        for (int64_t bb = 0; bb < n_blk; ++bb) {
            double acc = 0.0;
            for (int64_t u = 0; u < blk; ++u) acc += row[bb * blk + u];
            cb[bb].score = acc;
            cb[bb].j = bb;
        }
        qsort(cb, (size_t)n_blk, sizeof(cand_t), cand_cmp);
        int32_t* row_idx = idx + w * (int64_t)topk;
        int32_t* blocks = (int32_t*)malloc(sizeof(int32_t) * (size_t)(keep > 0 ? keep : 1));
        if (!blocks) {
            free(cb);
            err = HS2O_ENOMEM;
            continue;
        }
        for (int64_t i = 0; i < keep; ++i) blocks[i] = (int32_t)cb[i].j;
        qsort(blocks, (size_t)keep, sizeof(int32_t), i32_cmp);
        for (int64_t i = 0; i < keep; ++i)
            for (int64_t u = 0; u < blk; ++u) row_idx[i * blk + u] = (int32_t)(blocks[i] * blk + u);
        for (int64_t i = keep * blk; i < topk; ++i) row_idx[i] = -1;
        if (kth_block) kth_block[w] = keep > 0 ? cb[keep - 1].score : NAN;
        if (next_block) next_block[w] = keep < n_blk ? cb[keep].score : -1.0;
        free(blocks);
        free(cb);
    }
    return err;
}

/* KV bridging (xiawanshe.com report, section "两级KV共享", first level "KV
 * Bridging"): the Cross-Decoder's K and V of a token are computed from the
 * Self-Decoder hidden state of that token by one projection,
 *     kv[f] = sum_c hidden[c] * w[f][c],   f < 2 * h_kv * d,
 * features [0, h_kv*d) being K (head f / d, dim f % d) and [h_kv*d, 2*h_kv*d)
 * being V.  hidden [n_rows][d_model], w [2*h_kv*d][d_model] (bf16 bits);
 * out_k, out_v [n_rows][h_kv][d] fp64. */
int hs2o_kv_bridge(int64_t n_rows, int d_model, int h_kv, int d, const uint16_t* hidden, const uint16_t* w,
                   double* out_k, double* out_v, int n_threads) {
    if (n_rows < 0 || d_model <= 0 || h_kv <= 0 || d <= 0) return HS2O_EINVAL;
    const int64_t hd = (int64_t)h_kv * d;
#ifdef _OPENMP
    if (n_threads > 0) omp_set_num_threads(n_threads);
#pragma omp parallel for schedule(dynamic, 4)
#endif
    for (int64_t r = 0; r < n_rows; ++r) {
        const uint16_t* x = hidden + r * (int64_t)d_model;
        for (int64_t f = 0; f < 2 * hd; ++f) {
            const uint16_t* wf = w + f * (int64_t)d_model;
            double acc = 0.0;
            for (int c = 0; c < d_model; ++c) acc += bf16_to_double(x[c]) * bf16_to_double(wf[c]);
            if (f < hd)
                out_k[r * hd + f] = acc;
            else
                out_v[r * hd + (f - hd)] = acc;
        }
    }
    return HS2O_OK;
}

int hs2o_max_threads(void) {
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}
