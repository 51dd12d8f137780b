/*
 * moba_oracle.c -- plain, slow, fp64 CPU oracle for MoBA block-sparse attention
 * prefill and sliding-window attention.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product path links, loads or calls this
 * file: only the tests, the smoke check and the benchmark's CPU-baseline leg do.  It
 * shares no code, header, table or helper with the CUDA library.
 *
 * Sources (cited by page title and section):
 *   [MoBA]  "MoBA: 어텐션에 전문가 혼합을 적용해 긴 문맥을 효율적으로 처리하는 블록 어텐션
 *           (feat. MoonshotAI)" (PyTorch KR forum summary of the MoBA paper).
 *   [SWA]   "SWA + MoE: 어텐션과 희소 전문가" (Bit-Axon architecture page).
 *
 * Everything is computed in double precision from the exact bf16 input values.
 * Inputs are contiguous [batch, heads, N, d] arrays of raw bf16 bit patterns.
 * Block and position indices are 0-based (the MoBA page numbers blocks from 1).
 *
 * Readings taken where the pages are silent (each one is pinned by a test):
 *   - top-k counts the forced current block: a row keeps its own block plus the
 *     k-1 best past blocks (the page's sparsity arithmetic, k*B keys per query,
 *     only fits this reading);
 *   - gate scores are unscaled inner products; attention logits use 1/sqrt(d);
 *   - score ties go to the lower block index;
 *   - with fewer than k-1 past blocks every past block is kept;
 *   - each GQA query head selects on its own; head h reads KV head h / (Hq/Hkv);
 *   - the optional causal window is a set union with the selected blocks;
 *   - lse is the natural log of the sum of exp(scaled logits) over the key set;
 *   - when B does not divide N, the last block holds the remaining N mod B
 *     positions and is pooled by the mean of those keys (it is only ever a row's
 *     own block, never a past block of any row).
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define ORC_OK 0
#define ORC_ERR_ARG -1
#define ORC_ERR_IDX -2
#define ORC_ERR_MEM -3

/* Exact widening of a bf16 bit pattern (the upper half of an IEEE binary32). */
static double bf16_to_double(uint16_t x)
{
    uint32_t u = (uint32_t)x << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

int orc_num_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

/* Number of blocks: ceil(N / B).  When B does not divide N the last block is
   partial: it holds the N mod B remaining positions. */
static int n_blocks(int N, int B) { return (N + B - 1) / B; }

/*
 * [MoBA] §"블록 분할과 top-k 게이팅" (block partition and top-k gating): block j covers
 * key positions [j*B, min((j+1)*B, N)) and is represented by the mean of its keys,
 * MeanPool(K[I_j]) (a partial last block: the mean of the keys it holds).
 *   k    : bf16 [b, hkv, N, d]
 *   kbar : double [b, hkv, ceil(N/B), d]
 */
int orc_pool_keys(const uint16_t *k, int b, int hkv, int N, int d, int B, double *kbar)
{
    if (b < 1 || hkv < 1 || N < 1 || d < 1 || B < 1)
        return ORC_ERR_ARG;
    const int n = n_blocks(N, B);
    const long total = (long)b * hkv * n;
#pragma omp parallel for schedule(static)
    for (long u = 0; u < total; ++u) {
        const long bh = u / n;
        const int j = (int)(u % n);
        const int len = (N - j * B < B) ? N - j * B : B;
        const uint16_t *kb = k + (bh * N + (long)j * B) * d;
        double *dst = kbar + u * d;
        for (int t = 0; t < d; ++t) {
            double sum = 0.0;
            for (int r = 0; r < len; ++r)
                sum += bf16_to_double(kb[(long)r * d + t]);
            dst[t] = sum / (double)len;
        }
    }
    return ORC_OK;
}

/*
 * [MoBA] §"블록 분할과 top-k 게이팅": gate score s_j = <q, MeanPool(K[I_j])>, no scale.
 * [MoBA] §"인과성 보존" (causality): only blocks wholly before the query's own block
 * c = i / B compete; the own block is forced and later blocks are excluded, so only
 * j < c gets a score.  Entries j >= c are written as -INFINITY.
 *   q      : bf16 [b, hq, N, d]
 *   kbar   : double [b, hkv, ceil(N/B), d]
 *   rows   : nrows query positions (applied to every batch and head)
 *   scores : double [b, hq, nrows, ceil(N/B)]
 */
int orc_gate_scores(const uint16_t *q, const double *kbar, int b, int hq, int hkv, int N,
                    int d, int B, const int32_t *rows, int nrows, double *scores)
{
    if (b < 1 || hq < 1 || hkv < 1 || hq % hkv != 0 || N < 1 || d < 1 || B < 1)
        return ORC_ERR_ARG;
    const int n = n_blocks(N, B), G = hq / hkv;
    const long total = (long)b * hq * nrows;
    int bad = 0;
#pragma omp parallel for schedule(static) reduction(| : bad)
    for (long u = 0; u < total; ++u) {
        const long bh = u / nrows;
        const int bb = (int)(bh / hq), h = (int)(bh % hq), r = (int)(u % nrows);
        const int i = rows[r];
        double *s = scores + u * n;
        if (i < 0 || i >= N) {
            bad = 1;
            continue;
        }
        const int c = i / B;
        const uint16_t *qi = q + (bh * N + i) * (long)d;
        const double *kb = kbar + ((long)bb * hkv + h / G) * n * (long)d;
        for (int j = 0; j < n; ++j) {
            if (j >= c) {
                s[j] = -INFINITY;
                continue;
            }
            double acc = 0.0;
            for (int t = 0; t < d; ++t)
                acc += bf16_to_double(qi[t]) * kb[(long)j * d + t];
            s[j] = acc;
        }
    }
    return bad ? ORC_ERR_ARG : ORC_OK;
}

/* Order for the top-k: higher score first, lower block index on ties. */
typedef struct {
    double s;
    int j;
} scored_block;

static int by_score_desc(const void *a, const void *b)
{
    const scored_block *x = (const scored_block *)a, *y = (const scored_block *)b;
    if (x->s > y->s) return -1;
    if (x->s < y->s) return 1;
    return (x->j > y->j) - (x->j < y->j);
}

/*
 * [MoBA] §"블록 분할과 top-k 게이팅": g_j = 1 iff s_j is among the top-k scores, with
 * §"인과성 보존": the current block is always attended (it takes one of the k
 * places) and future blocks never are.  The past blocks are fully sorted, so this
 * is the plain definition, not a selection algorithm.
 *   scores : double [b, hq, nrows, n] as written by orc_gate_scores
 *   idx    : int32 [b, hq, nrows, topk] chosen blocks ascending, -1 padded
 *   gap    : double [b, hq, nrows]  s_(k-1) - s_(k) over the past blocks sorted
 *            descending (1-based ranks), +INFINITY when no past block is left out
 */
int orc_select_topk(const double *scores, int b, int hq, int N, int B, int topk,
                    const int32_t *rows, int nrows, int32_t *idx, double *gap)
{
    if (b < 1 || hq < 1 || N < 1 || B < 1 || topk < 1)
        return ORC_ERR_ARG;
    const int n = n_blocks(N, B);
    const long total = (long)b * hq * nrows;
    int bad = 0;
#pragma omp parallel reduction(| : bad)
    {
        scored_block *past = (scored_block *)malloc(sizeof(scored_block) * (size_t)(n > 0 ? n : 1));
        char *keep = (char *)malloc((size_t)n);
        if (!past || !keep) {
            bad = 1;
        } else {
#pragma omp for schedule(static)
            for (long u = 0; u < total; ++u) {
                const int i = rows[u % nrows];
                int32_t *out = idx + u * topk;
                if (i < 0 || i >= N) {
                    bad = 1;
                    continue;
                }
                const int c = i / B;
                const double *s = scores + u * n;
                memset(keep, 0, (size_t)n);
                keep[c] = 1;
                if (c <= topk - 1) {
                    for (int j = 0; j < c; ++j) keep[j] = 1;
                    gap[u] = INFINITY;
                } else {
                    for (int j = 0; j < c; ++j) {
                        past[j].s = s[j];
                        past[j].j = j;
                    }
                    qsort(past, (size_t)c, sizeof(scored_block), by_score_desc);
                    for (int t = 0; t < topk - 1; ++t) keep[past[t].j] = 1;
                    gap[u] = (topk >= 2) ? past[topk - 2].s - past[topk - 1].s : INFINITY;
                }
                int w = 0;
                for (int j = 0; j <= c; ++j)
                    if (keep[j]) out[w++] = j;
                while (w < topk) out[w++] = -1;
            }
        }
        free(past);
        free(keep);
    }
    return bad ? ORC_ERR_ARG : ORC_OK;
}

#define ORC_MODE_MOBA 0  /* keys of the blocks listed in idx (causal), union the window */
#define ORC_MODE_SWA 1   /* [SWA] causal band: j <= i and i - j < window            */
#define ORC_MODE_DENSE 2 /* plain causal attention, j <= i                          */

/*
 * Softmax attention over each row's key set J:
 *   [MoBA] §"표준 어텐션에서 블록 어텐션으로": MoBA(q,K,V) = Softmax(q K[I]^T) V[I];
 *   [MoBA] §"MoBA의 구현": the current block is causal, past blocks are whole;
 *   [SWA]  §"어텐션 공식" and §"슬라이딩 윈도우 마스크": softmax(QK^T/sqrt(d_k) + M) V with
 *          M_ij = 0 iff j <= i and i - j < w.
 * J for MODE_MOBA = { j <= i : j / B is listed in idx } U { j : 0 <= i - j < window }
 * (window <= 0 means no window).  Logits z_j = scale * <q_i, k_j>.
 *   q      : bf16 [b, hq, N, d];  k, v : bf16 [b, hkv, N, d]
 *   idx    : int32 [b, hq, nrows, topk] (MODE_MOBA only; entries -1 or in [0, i/B])
 *   out    : double [b, hq, nrows, d];  lse : double [b, hq, nrows]
 * Returns ORC_ERR_IDX when an idx entry names a block the row may not see.
 */
int orc_attention(const uint16_t *q, const uint16_t *k, const uint16_t *v, int b, int hq,
                  int hkv, int N, int d, int mode, int B, int topk, const int32_t *idx,
                  int window, double scale, const int32_t *rows, int nrows, double *out,
                  double *lse)
{
    if (b < 1 || hq < 1 || hkv < 1 || hq % hkv != 0 || N < 1 || d < 1)
        return ORC_ERR_ARG;
    if (mode == ORC_MODE_MOBA && (B < 1 || topk < 1 || !idx))
        return ORC_ERR_ARG;
    if (mode == ORC_MODE_SWA && window < 1)
        return ORC_ERR_ARG;
    if (mode < 0 || mode > 2)
        return ORC_ERR_ARG;
    const int G = hq / hkv;
    const int n = (mode == ORC_MODE_MOBA) ? n_blocks(N, B) : 1;
    const long total = (long)b * hq * nrows;
    int bad = 0;
#pragma omp parallel reduction(| : bad)
    {
        double *z = (double *)malloc(sizeof(double) * (size_t)N);
        int32_t *key = (int32_t *)malloc(sizeof(int32_t) * (size_t)N);
        char *sel = (char *)malloc((size_t)n);
        double *qd = (double *)malloc(sizeof(double) * (size_t)d);
        double *acc = (double *)malloc(sizeof(double) * (size_t)d);
        if (!z || !key || !sel || !qd || !acc) {
            bad |= 4;
        } else {
#pragma omp for schedule(dynamic, 16)
            for (long u = 0; u < total; ++u) {
                const long bh = u / nrows;
                const int bb = (int)(bh / hq), h = (int)(bh % hq);
                const int i = rows[u % nrows];
                if (i < 0 || i >= N) {
                    bad |= 1;
                    continue;
                }
                /* Build the key set J in ascending key order. */
                int nk = 0;
                if (mode == ORC_MODE_DENSE) {
                    for (int j = 0; j <= i; ++j) key[nk++] = j;
                } else if (mode == ORC_MODE_SWA) {
                    for (int j = (i - window + 1 > 0 ? i - window + 1 : 0); j <= i; ++j) key[nk++] = j;
                } else {
                    const int c = i / B;
                    memset(sel, 0, (size_t)n);
                    const int32_t *ir = idx + u * topk;
                    for (int t = 0; t < topk; ++t) {
                        if (ir[t] == -1) continue;
                        if (ir[t] < 0 || ir[t] > c) {
                            bad |= 2;
                            continue;
                        }
                        sel[ir[t]] = 1;
                    }
                    /* Walk the blocks up to the own one: a listed block gives all of
                       its keys up to i, any other block only its keys inside the
                       window. */
                    for (int blk = 0; blk <= c; ++blk) {
                        const int lo = blk * B;
                        const int hi = (blk * B + B - 1 < i) ? blk * B + B - 1 : i;
                        int from = lo;
                        if (!sel[blk]) {
                            if (window <= 0) continue;
                            from = (i - window + 1 > lo) ? i - window + 1 : lo;
                        }
                        for (int j = from; j <= hi; ++j) key[nk++] = j;
                    }
                }
                const uint16_t *qi = q + (bh * N + i) * (long)d;
                const long kvh = (long)bb * hkv + h / G;
                const uint16_t *kh = k + kvh * N * (long)d;
                const uint16_t *vh = v + kvh * N * (long)d;
                for (int t = 0; t < d; ++t) qd[t] = bf16_to_double(qi[t]);
                double m = -INFINITY;
                for (int e = 0; e < nk; ++e) {
                    const uint16_t *kj = kh + (long)key[e] * d;
                    double dot = 0.0;
                    for (int t = 0; t < d; ++t) dot += qd[t] * bf16_to_double(kj[t]);
                    z[e] = scale * dot;
                    if (z[e] > m) m = z[e];
                }
                double l = 0.0;
                for (int t = 0; t < d; ++t) acc[t] = 0.0;
                for (int e = 0; e < nk; ++e) {
                    const double p = exp(z[e] - m);
                    const uint16_t *vj = vh + (long)key[e] * d;
                    l += p;
                    for (int t = 0; t < d; ++t) acc[t] += p * bf16_to_double(vj[t]);
                }
                double *o = out + u * d;
                for (int t = 0; t < d; ++t) o[t] = acc[t] / l;
                lse[u] = m + log(l);
            }
        }
        free(z);
        free(key);
        free(sel);
        free(qd);
        free(acc);
    }
    if (bad & 4) return ORC_ERR_MEM;
    if (bad & 1) return ORC_ERR_ARG;
    if (bad & 2) return ORC_ERR_IDX;
    return ORC_OK;
}

/*
 * Key set J_i of row i under MoBA with block choice `ir` (topk entries, -1 padded)
 * and an optional causal window, in ascending key order: the keys j <= i whose block
 * is listed, and (window > 0) the keys with 0 <= i - j < window.  `sel` is scratch of
 * n bytes.  Returns the key count, or -1 when an entry names a block the row may not
 * see.
 */
static int moba_keys(int i, int B, int n, int topk, const int32_t *ir, int window, char *sel,
                     int32_t *key)
{
    const int c = i / B;
    memset(sel, 0, (size_t)n);
    for (int t = 0; t < topk; ++t) {
        if (ir[t] == -1) continue;
        if (ir[t] < 0 || ir[t] > c) return -1;
        sel[ir[t]] = 1;
    }
    int nk = 0;
    for (int blk = 0; blk <= c; ++blk) {
        const int lo = blk * B;
        const int hi = (blk * B + B - 1 < i) ? blk * B + B - 1 : i;
        int from = lo;
        if (!sel[blk]) {
            if (window <= 0) continue;
            from = (i - window + 1 > lo) ? i - window + 1 : lo;
        }
        for (int j = from; j <= hi; ++j) key[nk++] = j;
    }
    return nk;
}

/*
 * Gradients of MoBA attention for a fixed block choice.  [MoBA] §"MoBA와 전체 어텐션의
 * 하이브리드" trains models whose layers are MoBA attention, so gradients flow through
 * it; the gate is a parameter-free top-k and passes no gradient, so for the choice in
 * idx the layer is plain softmax attention over each row's key set J_i (§"MoBA의 구현",
 * unioned with the optional causal window).  With z_ij = scale q_i . k_j on J_i,
 * p_ij = exp(z_ij - lse_i), o_i = sum_j p_ij v_j and the upstream gradient dO:
 *     D_i = dO_i . o_i,   dp_ij = dO_i . v_j,   dz_ij = p_ij (dp_ij - D_i)
 *     dQ_i = scale sum_j dz_ij k_j
 *     dK_j = scale sum_i dz_ij q_i,   dV_j = sum_i p_ij dO_i
 * where a KV head's dK and dV sum over the q-heads that read it (GQA).
 * dQ is computed at the listed rows (every q-head), dK and dV at the listed key
 * positions (every KV head): a key's sums run over every row of every q-head of its
 * group whose key set holds it, each with that row's own lse_i and D_i.
 *   q, dout : bf16 [b, hq, N, d];  k, v : bf16 [b, hkv, N, d]
 *   idx     : int32 [b, hq, N, topk], the choice of EVERY row
 *   rows    : R row positions -> dq double [b, hq, R, d]
 *   keys    : K key positions -> dk, dv double [b, hkv, K, d]
 */
int orc_attention_bwd(const uint16_t *q, const uint16_t *k, const uint16_t *v,
                      const uint16_t *dout, int b, int hq, int hkv, int N, int d, int B, int topk,
                      const int32_t *idx, int window, double scale, const int32_t *rows, int R,
                      double *dq, const int32_t *keys, int K, double *dk, double *dv)
{
    if (b < 1 || hq < 1 || hkv < 1 || hq % hkv != 0 || N < 1 || d < 1 || B < 1 || topk < 1 ||
        !idx || R < 0 || K < 0)
        return ORC_ERR_ARG;
    for (int r = 0; r < R; ++r)
        if (rows[r] < 0 || rows[r] >= N) return ORC_ERR_ARG;
    for (int e = 0; e < K; ++e)
        if (keys[e] < 0 || keys[e] >= N) return ORC_ERR_ARG;
    const int G = hq / hkv;
    const int n = n_blocks(N, B);
    const long nrows_all = (long)b * hq * N;
    /* Row statistics (lse_i, D_i) of the rows a listed key's sums need. */
    char *need = (char *)calloc((size_t)nrows_all, 1);
    double *lse = (double *)malloc(sizeof(double) * (size_t)nrows_all);
    double *D = (double *)malloc(sizeof(double) * (size_t)nrows_all);
    if (!need || !lse || !D) {
        free(need);
        free(lse);
        free(D);
        return ORC_ERR_MEM;
    }
    int bad = 0;
    /* A row needs its statistics when it is a listed row or when its key set holds a
       listed key of its KV head. */
#pragma omp parallel for schedule(dynamic, 64)
    for (long u = 0; u < nrows_all; ++u) {
        const long bh = u / N;
        const int bb = (int)(bh / hq), h = (int)(bh % hq), i = (int)(u % N);
        const int32_t *ir = idx + u * topk;
        char hit = 0;
        for (int e = 0; e < K && !hit; ++e) {
            const int j = keys[e];
            if (j > i) continue;
            const int cj = j / B;
            if (window > 0 && i - j < window) hit = 1;
            for (int t = 0; t < topk && !hit; ++t) hit = (ir[t] == cj);
        }
        (void)bb;
        (void)h;
        need[u] = hit;
    }
    for (long bh = 0; bh < (long)b * hq; ++bh)
        for (int r = 0; r < R; ++r) need[bh * N + rows[r]] = 1;

#pragma omp parallel reduction(| : bad)
    {
        double *z = (double *)malloc(sizeof(double) * (size_t)N);
        int32_t *key = (int32_t *)malloc(sizeof(int32_t) * (size_t)N);
        char *sel = (char *)malloc((size_t)n);
        double *qd = (double *)malloc(sizeof(double) * (size_t)d);
        double *od = (double *)malloc(sizeof(double) * (size_t)d);
        double *acc = (double *)malloc(sizeof(double) * (size_t)d);
        if (!z || !key || !sel || !qd || !od || !acc) {
            bad |= 4;
        } else {
#pragma omp for schedule(dynamic, 16)
            for (long u = 0; u < nrows_all; ++u) {
                if (!need[u]) continue;
                const long bh = u / N;
                const int bb = (int)(bh / hq), h = (int)(bh % hq), i = (int)(u % N);
                const int nk = moba_keys(i, B, n, topk, idx + u * topk, window, sel, key);
                if (nk < 0) {
                    bad |= 2;
                    continue;
                }
                const long kvh = (long)bb * hkv + h / G;
                const uint16_t *kh = k + kvh * N * (long)d;
                const uint16_t *vh = v + kvh * N * (long)d;
                for (int t = 0; t < d; ++t) {
                    qd[t] = bf16_to_double(q[u * d + t]);
                    od[t] = bf16_to_double(dout[u * d + t]);
                }
                double m = -INFINITY;
                for (int e = 0; e < nk; ++e) {
                    const uint16_t *kj = kh + (long)key[e] * d;
                    double dot = 0.0;
                    for (int t = 0; t < d; ++t) dot += qd[t] * bf16_to_double(kj[t]);
                    z[e] = scale * dot;
                    if (z[e] > m) m = z[e];
                }
                double l = 0.0;
                for (int t = 0; t < d; ++t) acc[t] = 0.0;
                for (int e = 0; e < nk; ++e) {
                    const double p = exp(z[e] - m);
                    const uint16_t *vj = vh + (long)key[e] * d;
                    l += p;
                    for (int t = 0; t < d; ++t) acc[t] += p * bf16_to_double(vj[t]);
                }
                double Di = 0.0;
                for (int t = 0; t < d; ++t) Di += od[t] * (acc[t] / l);
                lse[u] = m + log(l);
                D[u] = Di;
            }
        }
        free(z);
        free(key);
        free(sel);
        free(qd);
        free(od);
        free(acc);
    }
    if (bad) {
        free(need);
        free(lse);
        free(D);
        return (bad & 4) ? ORC_ERR_MEM : ORC_ERR_IDX;
    }

    /* dQ at the listed rows. */
#pragma omp parallel reduction(| : bad)
    {
        int32_t *key = (int32_t *)malloc(sizeof(int32_t) * (size_t)N);
        char *sel = (char *)malloc((size_t)n);
        double *qd = (double *)malloc(sizeof(double) * (size_t)d);
        double *od = (double *)malloc(sizeof(double) * (size_t)d);
        if (!key || !sel || !qd || !od) {
            bad |= 4;
        } else {
#pragma omp for schedule(dynamic, 4)
            for (long w = 0; w < (long)b * hq * R; ++w) {
                const long bh = w / R;
                const int bb = (int)(bh / hq), h = (int)(bh % hq), i = rows[w % R];
                const long u = bh * N + i;
                const int nk = moba_keys(i, B, n, topk, idx + u * topk, window, sel, key);
                const long kvh = (long)bb * hkv + h / G;
                const uint16_t *kh = k + kvh * N * (long)d;
                const uint16_t *vh = v + kvh * N * (long)d;
                for (int t = 0; t < d; ++t) {
                    qd[t] = bf16_to_double(q[u * d + t]);
                    od[t] = bf16_to_double(dout[u * d + t]);
                }
                double *g = dq + w * d;
                for (int t = 0; t < d; ++t) g[t] = 0.0;
                for (int e = 0; e < nk; ++e) {
                    const uint16_t *kj = kh + (long)key[e] * d;
                    const uint16_t *vj = vh + (long)key[e] * d;
                    double zq = 0.0, dp = 0.0;
                    for (int t = 0; t < d; ++t) {
                        zq += qd[t] * bf16_to_double(kj[t]);
                        dp += od[t] * bf16_to_double(vj[t]);
                    }
                    const double p = exp(scale * zq - lse[u]);
                    const double dz = p * (dp - D[u]);
                    for (int t = 0; t < d; ++t) g[t] += scale * dz * bf16_to_double(kj[t]);
                }
            }
        }
        free(key);
        free(sel);
        free(qd);
        free(od);
    }

    /* dK and dV at the listed keys: every row of the group whose key set holds it. */
#pragma omp parallel reduction(| : bad)
    {
        char *sel = (char *)malloc((size_t)n);
        if (!sel) {
            bad |= 4;
        } else {
#pragma omp for schedule(dynamic, 1)
            for (long w = 0; w < (long)b * hkv * K; ++w) {
                const long bk = w / K;
                const int bb = (int)(bk / hkv), hk = (int)(bk % hkv), j = keys[w % K];
                const int cj = j / B;
                const uint16_t *kj = k + (bk * N + j) * (long)d;
                const uint16_t *vj = v + (bk * N + j) * (long)d;
                double *gk = dk + w * d, *gv = dv + w * d;
                for (int t = 0; t < d; ++t) gk[t] = gv[t] = 0.0;
                for (int g = 0; g < G; ++g) {
                    const long bh = (long)bb * hq + (long)hk * G + g;
                    for (int i = j; i < N; ++i) {
                        const long u = bh * N + i;
                        const int32_t *ir = idx + u * topk;
                        int in = (window > 0 && i - j < window);
                        for (int t = 0; t < topk && !in; ++t) in = (ir[t] == cj);
                        if (!in) continue;
                        const uint16_t *qi = q + u * d;
                        const uint16_t *oi = dout + u * d;
                        double zq = 0.0, dp = 0.0;
                        for (int t = 0; t < d; ++t) {
                            zq += bf16_to_double(qi[t]) * bf16_to_double(kj[t]);
                            dp += bf16_to_double(oi[t]) * bf16_to_double(vj[t]);
                        }
                        const double p = exp(scale * zq - lse[u]);
                        const double dz = p * (dp - D[u]);
                        for (int t = 0; t < d; ++t) {
                            gk[t] += scale * dz * bf16_to_double(qi[t]);
                            gv[t] += p * bf16_to_double(oi[t]);
                        }
                    }
                }
            }
        }
        free(sel);
    }
    free(need);
    free(lse);
    free(D);
    return (bad & 4) ? ORC_ERR_MEM : ORC_OK;
}
