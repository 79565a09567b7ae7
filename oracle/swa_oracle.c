/*
 * swa_oracle.c -- plain, slow, fp64 CPU oracle for banded sparse self-attention
 * (sliding window with optional dilation and causal mask, global tokens, appended
 * side keys with an additive bias, grouped KV heads).
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path may link, load or call
 * this file: only the tests, the graft smoke check and the bench's CPU-baseline
 * leg use it.  It shares no code, header, table or helper with the CUDA library.
 *
 * Every function states the definition it writes out.  Sources (page title and
 * section; the pages are web articles about Longformer, LongT5, BigBird,
 * SWAN-GPT and a SWA fine-tuning recipe):
 *   [BB-3.2.1]  "精读笔记：Big Bird" §3.2.1 Local Window Attention: a query at i
 *               attends to keys i-w/2 .. i+w/2; worked example w=6: position 5
 *               sees positions 2..8.
 *   [BB-3.2.3]  same page §3.2.3 Global Attention (ITC): chosen existing tokens
 *               attend over the whole sequence and are attended by every token.
 *   [LF-2]      "Longformer 如何打破 512 token 魔咒" §二: sliding window + global
 *               attention + dilated attention (skip tokens inside the window, like
 *               a dilated convolution, widening the span at equal cost).
 *   [LT5-TG]    "LongT5 长序列模型完全指南" section "两种高效注意力机制": Local
 *               attention (r on each side) and Transient-Global (block summaries
 *               of k=16 tokens become extra keys every token attends to).
 *   [LT5-SRC]   same page, section "源码级证据": side key/values are concatenated
 *               after the local keys, and a global relative-position bias is
 *               added to the scores; padding tokens get block id -1.
 *   [LT5-RPE]   same page, section "相对位置编码": relative distance
 *               memory_position - query_position is bucketed: half the buckets
 *               per direction, exact below half of that, log-spaced above,
 *               everything beyond max_distance in the last bucket;
 *               section "LongT5Config 参数全解": num_buckets 32, max_distance 128.
 *   [SWAN-3.3]  "SWAN-GPT：无需长文本训练" §3.3(1): decoder SWA-RoPE layers with
 *               a fixed 512-token causal window.
 *   [LT5-LOCAL] LongT5 guide, "相对位置编码" section: the local attention adds a
 *               relative-position bias bucketed on memory_position -
 *               query_position, computed once over the local window.
 *   [BB-3.2.2]  "精读笔记：Big Bird" §3.2.2: every query also attends to r
 *               randomly chosen keys.  Here the random keys come in blocks: the
 *               rows of query block q = floor(i / bs) share rand_blocks[b][h][q][:],
 *               each naming a block of bs consecutive keys (the draws are inputs).
 *
 * Readings where the pages are silent (each is listed in the design notes):
 *   window bounds inclusive (2r+1 keys, non-causal); causal window t in [-r,0];
 *   dilation d: keys i + d*t; window and global sets are merged as a SET;
 *   padded query rows (i >= valid_len) give o = 0 and lse = -inf; padded keys
 *   are never attended; side keys are attended by every valid query, global
 *   queries included; score = scale*<q,k> (+ bias on side keys only);
 *   lse is the natural log; KV head of query head h is h / (Hq/Hkv).
 *
 * Layouts (row-major, contiguous): q/out [B,Hq,n,D]; k/v [B,Hkv,n,D];
 * side_k/side_v [B,Hkv,S,D]; bias [Hq, S + nblk - 1] with nblk = ceil(n/kb);
 * global_idx [B,g] sorted ascending, unique, each < valid_len[b].
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#ifdef _OPENMP
#include <omp.h>
#endif

#define ORACLE_OK 0
#define ORACLE_EINVAL 1
#define ORACLE_ENOMEM 2

typedef struct {
    int B, Hq, Hkv, n, D;
    const float *q, *k, *v;
    const int32_t *global_idx;
    int g;
    const float *side_k, *side_v;
    int S, side_block;
    const float *bias;
    const int32_t *window, *dilation;
    int causal;
    const int32_t *valid_len;
    double scale;
    const float *local_bias;   /* [Hq, 2R+1] or NULL: bias of window keys by j - i */
    int local_radius;          /* R */
    const int32_t *rand_blocks; /* [B, Hq, ceil(n / bs), num_rand] or NULL */
    int num_rand;
    int rand_block;            /* bs */
} oracle_problem;

/* Optional terms of the score and the key set, passed by pointer (NULL: none). */
typedef struct {
    const float *local_bias;
    int local_radius;
    const int32_t *rand_blocks;
    int num_rand;
    int rand_block;
} oracle_extras;

static void apply_extras(oracle_problem *P, const oracle_extras *ex) {
    if (!ex) return;
    P->local_bias = ex->local_bias;
    P->local_radius = ex->local_radius;
    if (ex->rand_blocks && ex->num_rand > 0 && ex->rand_block > 0) {
        P->rand_blocks = ex->rand_blocks;
        P->num_rand = ex->num_rand;
        P->rand_block = ex->rand_block;
    }
}

static int num_blocks(int n, int kb) { return kb > 0 ? (n + kb - 1) / kb : 0; }

/* Membership of position i in the sorted global list of batch b. */
static int is_global(const oracle_problem *P, int b, int i) {
    for (int t = 0; t < P->g; ++t)
        if (P->global_idx[(int64_t)b * P->g + t] == i) return 1;
    return 0;
}

/*
 * The explicit key set K(i) of one query row, in increasing key order, without
 * duplicates [BB-3.2.1, BB-3.2.2, BB-3.2.3, LF-2, SWAN-3.3]:
 *   i >= V            -> empty (padded query row)
 *   i global          -> {0, .., V-1}
 *   otherwise         -> W(i) U G U R(i), W(i) = {i + d t : -r <= t <= r (t <= 0
 *                        if causal), 0 <= i + d t < V}, R(i) = the keys below V
 *                        of the random blocks of i's query block
 * W and G are merged as two ascending lists with repeats dropped; random blocks,
 * when present, are added through a mark per key.  Returns the number of keys
 * written to keys[] (capacity n).
 */
static int key_set(const oracle_problem *P, int b, int h, int i, int32_t *keys,
                   int32_t *wbuf) {
    int V = P->valid_len ? P->valid_len[b] : P->n;
    if (i >= V) return 0;
    if (P->g > 0 && is_global(P, b, i)) {
        for (int j = 0; j < V; ++j) keys[j] = j;
        return V;
    }
    int r = P->window[h], d = P->dilation[h];
    int nw = 0;
    int tmax = P->causal ? 0 : r;
    for (int t = -r; t <= tmax; ++t) {
        int64_t j = (int64_t)i + (int64_t)d * t;
        if (j >= 0 && j < V) wbuf[nw++] = (int32_t)j;
    }
    /* merge W(i) (ascending) with G (ascending) as a set */
    const int32_t *G = P->global_idx ? P->global_idx + (int64_t)b * P->g : NULL;
    int a = 0, c = 0, m = 0;
    while (a < nw || c < P->g) {
        int32_t next;
        if (c >= P->g || (a < nw && wbuf[a] <= G[c])) {
            next = wbuf[a++];
        } else {
            next = G[c++];
            if (next >= V) continue; /* never attend a padded key */
        }
        if (m == 0 || keys[m - 1] != next) keys[m++] = next;
    }
    if (P->rand_blocks) {
        unsigned char *mark = (unsigned char *)calloc((size_t)V + 1, 1);
        if (!mark) return -1;
        for (int t = 0; t < m; ++t) mark[keys[t]] = 1;
        const int bs = P->rand_block;
        const int nqb = (P->n + bs - 1) / bs;
        const int32_t *rb = P->rand_blocks + (((int64_t)b * P->Hq + h) * nqb + i / bs) * P->num_rand;
        for (int t = 0; t < P->num_rand; ++t) {
            int64_t lo = (int64_t)rb[t] * bs, hi = lo + bs;
            if (lo < 0) lo = 0;
            if (hi > V) hi = V;
            for (int64_t j = lo; j < hi; ++j) mark[j] = 1;
        }
        m = 0;
        for (int j = 0; j < V; ++j)
            if (mark[j]) keys[m++] = j;
        free(mark);
    }
    return m;
}

/*
 * Side-key bias index for query position i and side key s [LT5-SRC]:
 * relative block distance delta = s - floor(i / kb) (memory minus query),
 * stored at column delta + nblk - 1 of the per-head table.
 */
static double side_bias(const oracle_problem *P, int h, int i, int s) {
    if (!P->bias) return 0.0;
    int nblk = num_blocks(P->n, P->side_block);
    int cols = P->S + nblk - 1;
    int delta = s - i / P->side_block;
    return (double)P->bias[(int64_t)h * cols + delta + nblk - 1];
}

/*
 * Local relative-position bias of a window key [LT5-LOCAL]: added to s_ij when j
 * is in the window W(i) of a non-global query, read from column (j - i) + R of
 * the head's table.  Global query rows and global / side keys get none.
 */
static int in_window(const oracle_problem *P, int h, int i, int j) {
    int64_t diff = (int64_t)i - j;
    int64_t rd = (int64_t)P->window[h] * P->dilation[h];
    int band = P->causal ? (diff >= 0 && diff <= rd) : (diff >= -rd && diff <= rd);
    return band && (diff % P->dilation[h] == 0);
}

static double local_bias(const oracle_problem *P, int b, int h, int i, int j) {
    if (!P->local_bias) return 0.0;
    if (P->g > 0 && is_global(P, b, i)) return 0.0;
    if (!in_window(P, h, i, j)) return 0.0;
    return (double)P->local_bias[(int64_t)h * (2 * P->local_radius + 1) + (j - i) + P->local_radius];
}

static double dot(const float *a, const float *b, int D) {
    double acc = 0.0;
    for (int x = 0; x < D; ++x) acc += (double)a[x] * (double)b[x];
    return acc;
}

/*
 * Softmax attention of one query row over an explicit key list plus all side
 * keys: s_j = scale <q_i, k_j> (+ side bias), m = max s, l = sum exp(s - m),
 * o = sum exp(s - m) v_j / l, lse = m + ln l.  An empty list gives o = 0 and
 * lse = -inf.
 */
static void attend_row(const oracle_problem *P, int b, int h, int i,
                       const int32_t *keys, int nk, double *scores, double *o,
                       double *lse) {
    int D = P->D;
    int hk = h / (P->Hq / P->Hkv);
    int V = P->valid_len ? P->valid_len[b] : P->n;
    int S = (i < V) ? P->S : 0;
    const float *qi = P->q + (((int64_t)b * P->Hq + h) * P->n + i) * D;
    const float *kb = P->k + ((int64_t)b * P->Hkv + hk) * P->n * D;
    const float *vb = P->v + ((int64_t)b * P->Hkv + hk) * P->n * D;
    const float *skb = S ? P->side_k + ((int64_t)b * P->Hkv + hk) * P->S * D : NULL;
    const float *svb = S ? P->side_v + ((int64_t)b * P->Hkv + hk) * P->S * D : NULL;
    int tot = nk + S;
    for (int x = 0; x < D; ++x) o[x] = 0.0;
    if (tot == 0) {
        *lse = -INFINITY;
        return;
    }
    double m = -INFINITY;
    for (int t = 0; t < nk; ++t) {
        scores[t] = P->scale * dot(qi, kb + (int64_t)keys[t] * D, D) + local_bias(P, b, h, i, keys[t]);
        if (scores[t] > m) m = scores[t];
    }
    for (int s = 0; s < S; ++s) {
        scores[nk + s] = P->scale * dot(qi, skb + (int64_t)s * D, D) + side_bias(P, h, i, s);
        if (scores[nk + s] > m) m = scores[nk + s];
    }
    if (m == -INFINITY) { /* every score is -inf (only possible through bias) */
        *lse = -INFINITY;
        return;
    }
    double l = 0.0;
    for (int t = 0; t < tot; ++t) {
        double p = exp(scores[t] - m);
        scores[t] = p;
        l += p;
    }
    for (int t = 0; t < nk; ++t) {
        const float *vj = vb + (int64_t)keys[t] * D;
        for (int x = 0; x < D; ++x) o[x] += scores[t] * (double)vj[x];
    }
    for (int s = 0; s < S; ++s) {
        const float *vj = svb + (int64_t)s * D;
        for (int x = 0; x < D; ++x) o[x] += scores[nk + s] * (double)vj[x];
    }
    for (int x = 0; x < D; ++x) o[x] /= l;
    *lse = m + log(l);
}

static int check_problem(const oracle_problem *P) {
    if (P->rand_blocks) {
        const int nqb = (P->n + P->rand_block - 1) / P->rand_block;
        for (int64_t t = 0; t < (int64_t)P->B * P->Hq * nqb * P->num_rand; ++t)
            if (P->rand_blocks[t] < 0 || P->rand_blocks[t] >= nqb) return ORACLE_EINVAL;
    }
    if (P->B <= 0 || P->Hq <= 0 || P->Hkv <= 0 || P->n < 0 || P->D <= 0) return ORACLE_EINVAL;
    if (P->Hq % P->Hkv) return ORACLE_EINVAL;
    if (!P->q || !P->k || !P->v || !P->window || !P->dilation) return ORACLE_EINVAL;
    if (P->g < 0 || (P->g > 0 && !P->global_idx)) return ORACLE_EINVAL;
    if (P->S < 0 || (P->S > 0 && (!P->side_k || !P->side_v || P->side_block <= 0))) return ORACLE_EINVAL;
    for (int h = 0; h < P->Hq; ++h)
        if (P->window[h] < 0 || P->dilation[h] < 1) return ORACLE_EINVAL;
    if (P->local_bias) {
        /* the table must cover every offset j - i a window key can take */
        for (int h = 0; h < P->Hq; ++h) {
            int64_t reach = (int64_t)P->window[h] * P->dilation[h];
            if (reach > P->n - 1) reach = P->n - 1;
            if (P->local_radius < reach) return ORACLE_EINVAL;
        }
    }
    return ORACLE_OK;
}

/*
 * oracle_forward: for each requested row (flat id (b*Hq + h)*n + i; rows == NULL
 * means every row in that order) write o (fp64, D values), lse and
 * count = |K(i)| + (number of side keys attended) -- the attended pairs.
 */
int oracle_forward_ex(int B, int Hq, int Hkv, int n, int D, const float *q, const float *k,
                      const float *v, const int32_t *global_idx, int g, const float *side_k,
                      const float *side_v, int S, int side_block, const float *bias,
                      const int32_t *window, const int32_t *dilation, int causal,
                      const int32_t *valid_len, double scale, const int64_t *rows,
                      int64_t nrows, double *out, double *lse, int64_t *count,
                      const oracle_extras *ex) {
    oracle_problem P = {B, Hq, Hkv, n, D, q, k, v, global_idx, g, side_k, side_v,
                        S, side_block, bias, window, dilation, causal, valid_len, scale,
                        NULL, 0, NULL, 0, 0};
    apply_extras(&P, ex);
    int rc = check_problem(&P);
    if (rc) return rc;
    int64_t total = rows ? nrows : (int64_t)B * Hq * n;
    int failed = 0;
#pragma omp parallel
    {
        int32_t *keys = (int32_t *)malloc(sizeof(int32_t) * (size_t)(n + 1));
        int32_t *wbuf = (int32_t *)malloc(sizeof(int32_t) * (size_t)(n + 1));
        double *scores = (double *)malloc(sizeof(double) * (size_t)(n + S + 1));
        if (!keys || !wbuf || !scores) {
#pragma omp atomic write
            failed = 1;
        } else {
#pragma omp for schedule(dynamic, 64)
            for (int64_t t = 0; t < total; ++t) {
                int64_t id = rows ? rows[t] : t;
                int i = (int)(id % n);
                int h = (int)((id / n) % Hq);
                int b = (int)(id / ((int64_t)n * Hq));
                int nk = key_set(&P, b, h, i, keys, wbuf);
                if (nk < 0) {
#pragma omp atomic write
                    failed = 1;
                    nk = 0;
                }
                int Vb = valid_len ? valid_len[b] : n;
                attend_row(&P, b, h, i, keys, nk, scores, out + t * D, lse + t);
                if (count) count[t] = (i < Vb) ? (int64_t)nk + S : 0;
            }
        }
        free(keys);
        free(wbuf);
        free(scores);
    }
    return failed ? ORACLE_ENOMEM : ORACLE_OK;
}

int oracle_forward(int B, int Hq, int Hkv, int n, int D, const float *q, const float *k,
                   const float *v, const int32_t *global_idx, int g, const float *side_k,
                   const float *side_v, int S, int side_block, const float *bias,
                   const int32_t *window, const int32_t *dilation, int causal,
                   const int32_t *valid_len, double scale, const int64_t *rows,
                   int64_t nrows, double *out, double *lse, int64_t *count) {
    return oracle_forward_ex(B, Hq, Hkv, n, D, q, k, v, global_idx, g, side_k, side_v, S, side_block,
                             bias, window, dilation, causal, valid_len, scale, rows, nrows, out, lse,
                             count, NULL);
}

/*
 * oracle_key_counts: |K(i)| + S for every row (flat order), without touching
 * q/k/v -- the attended-pair count that defines the useful FLOPs 4*D*pairs.
 */
int oracle_key_counts_ex(int B, int Hq, int n, const int32_t *global_idx, int g, int S,
                         const int32_t *window, const int32_t *dilation, int causal,
                         const int32_t *valid_len, int64_t *count, const oracle_extras *ex) {
    oracle_problem P;
    memset(&P, 0, sizeof(P));
    P.B = B; P.Hq = Hq; P.Hkv = Hq; P.n = n; P.D = 1; P.global_idx = global_idx; P.g = g;
    P.S = S; P.window = window; P.dilation = dilation; P.causal = causal; P.valid_len = valid_len;
    apply_extras(&P, ex);
    int failed = 0;
#pragma omp parallel
    {
        int32_t *keys = (int32_t *)malloc(sizeof(int32_t) * (size_t)(n + 1));
        int32_t *wbuf = (int32_t *)malloc(sizeof(int32_t) * (size_t)(n + 1));
        if (!keys || !wbuf) {
#pragma omp atomic write
            failed = 1;
        } else {
#pragma omp for schedule(dynamic, 256)
            for (int64_t t = 0; t < (int64_t)B * Hq * n; ++t) {
                int i = (int)(t % n);
                int h = (int)((t / n) % Hq);
                int b = (int)(t / ((int64_t)n * Hq));
                int Vb = valid_len ? valid_len[b] : n;
                int nk = key_set(&P, b, h, i, keys, wbuf);
                if (nk < 0) {
#pragma omp atomic write
                    failed = 1;
                    nk = 0;
                }
                count[t] = (i < Vb) ? (int64_t)nk + S : 0;
            }
        }
        free(keys);
        free(wbuf);
    }
    return failed ? ORACLE_ENOMEM : ORACLE_OK;
}

int oracle_key_counts(int B, int Hq, int n, const int32_t *global_idx, int g, int S,
                      const int32_t *window, const int32_t *dilation, int causal,
                      const int32_t *valid_len, int64_t *count) {
    return oracle_key_counts_ex(B, Hq, n, global_idx, g, S, window, dilation, causal, valid_len,
                                count, NULL);
}

/*
 * oracle_key_list: the explicit key set K(i) of one row (no side keys), for
 * support checks.  Returns the count; keys[] must hold n entries.
 */
int oracle_key_list_ex(int B, int Hq, int n, const int32_t *global_idx, int g,
                       const int32_t *window, const int32_t *dilation, int causal,
                       const int32_t *valid_len, int b, int h, int i, int32_t *keys,
                       const oracle_extras *ex) {
    oracle_problem P;
    memset(&P, 0, sizeof(P));
    P.B = B; P.Hq = Hq; P.Hkv = Hq; P.n = n; P.D = 1; P.global_idx = global_idx; P.g = g;
    P.window = window; P.dilation = dilation; P.causal = causal; P.valid_len = valid_len;
    apply_extras(&P, ex);
    int32_t *wbuf = (int32_t *)malloc(sizeof(int32_t) * (size_t)(n + 1));
    if (!wbuf) return -1;
    int nk = key_set(&P, b, h, i, keys, wbuf);
    free(wbuf);
    return nk;
}

int oracle_key_list(int B, int Hq, int n, const int32_t *global_idx, int g,
                    const int32_t *window, const int32_t *dilation, int causal,
                    const int32_t *valid_len, int b, int h, int i, int32_t *keys) {
    return oracle_key_list_ex(B, Hq, n, global_idx, g, window, dilation, causal, valid_len, b, h,
                              i, keys, NULL);
}

/*
 * oracle_dense_bruteforce: an independent second statement of the same
 * attention, with no key lists at all.  It builds the n x n boolean "allowed"
 * matrix from the closed form
 *   non-causal: |i-j| <= r d  and  (i-j) mod d == 0
 *   causal:     0 <= i-j <= r d  and  (i-j) mod d == 0
 *   OR j global OR i global OR floor(j / bs) is a random block of floor(i / bs);
 *   AND i < V AND j < V,
 * appends every side column for valid rows, and runs a dense masked softmax
 * over all n + S columns.  Every row is written (flat order).
 */
int oracle_dense_bruteforce_ex(int B, int Hq, int Hkv, int n, int D, const float *q,
                               const float *k, const float *v, const int32_t *global_idx, int g,
                               const float *side_k, const float *side_v, int S, int side_block,
                               const float *bias, const int32_t *window, const int32_t *dilation,
                               int causal, const int32_t *valid_len, double scale, double *out,
                               double *lse, const oracle_extras *ex) {
    const float *local_bias_tab = ex ? ex->local_bias : NULL;
    const int local_radius = ex ? ex->local_radius : 0;
    const int32_t *rblk = (ex && ex->rand_blocks && ex->num_rand > 0) ? ex->rand_blocks : NULL;
    const int nrand = rblk ? ex->num_rand : 0, bs = rblk ? ex->rand_block : 1;
    if (B <= 0 || Hq <= 0 || Hkv <= 0 || Hq % Hkv || D <= 0 || n < 0) return ORACLE_EINVAL;
    if (rblk && bs <= 0) return ORACLE_EINVAL;
    if (local_bias_tab) {
        for (int h = 0; h < Hq; ++h) {
            int64_t reach = (int64_t)window[h] * dilation[h];
            if (reach > n - 1) reach = n - 1;
            if (local_radius < reach) return ORACLE_EINVAL;
        }
    }
    int G = Hq / Hkv;
    int nblk = side_block > 0 ? (n + side_block - 1) / side_block : 0;
    int cols = n + S;
    unsigned char *isg = (unsigned char *)calloc((size_t)n + 1, 1);
    unsigned char *allow = (unsigned char *)malloc((size_t)cols + 1);
    unsigned char *inband = (unsigned char *)malloc((size_t)n + 1);
    double *s = (double *)malloc(sizeof(double) * ((size_t)cols + 1));
    if (!isg || !allow || !s || !inband) {
        free(isg); free(allow); free(s); free(inband);
        return ORACLE_ENOMEM;
    }
    for (int b = 0; b < B; ++b) {
        int V = valid_len ? valid_len[b] : n;
        memset(isg, 0, (size_t)n + 1);
        for (int t = 0; t < g; ++t) isg[global_idx[(int64_t)b * g + t]] = 1;
        for (int h = 0; h < Hq; ++h) {
            int hk = h / G;
            int64_t rd = (int64_t)window[h] * dilation[h];
            for (int i = 0; i < n; ++i) {
                int64_t row = ((int64_t)b * Hq + h) * n + i;
                double *o = out + row * D;
                int any = 0;
                for (int j = 0; j < n; ++j) {
                    int64_t diff = (int64_t)i - j;
                    int band = causal ? (diff >= 0 && diff <= rd) : (llabs(diff) <= rd);
                    band = band && (diff % dilation[h] == 0);
                    int rnd = 0;
                    for (int t = 0; t < nrand; ++t)
                        rnd |= (j / bs == rblk[(((int64_t)b * Hq + h) * ((n + bs - 1) / bs) + i / bs) * nrand + t]);
                    int a = (band || isg[j] || isg[i] || rnd) && i < V && j < V;
                    inband[j] = (unsigned char)(band && !isg[i]);
                    allow[j] = (unsigned char)a;
                    any |= a;
                }
                for (int c = 0; c < S; ++c) {
                    allow[n + c] = (unsigned char)(i < V);
                    any |= (i < V);
                }
                for (int x = 0; x < D; ++x) o[x] = 0.0;
                if (!any) {
                    lse[row] = -INFINITY;
                    continue;
                }
                const float *qi = q + row * D;
                double m = -INFINITY;
                for (int c = 0; c < cols; ++c) {
                    if (!allow[c]) continue;
                    const float *kk = c < n ? k + (((int64_t)b * Hkv + hk) * n + c) * D
                                            : side_k + (((int64_t)b * Hkv + hk) * S + (c - n)) * D;
                    double acc = 0.0;
                    for (int x = 0; x < D; ++x) acc += (double)qi[x] * (double)kk[x];
                    acc *= scale;
                    if (c < n && local_bias_tab && inband[c])
                        acc += (double)local_bias_tab[(int64_t)h * (2 * local_radius + 1) + (c - i) + local_radius];
                    if (c >= n && bias) {
                        int delta = (c - n) - i / side_block;
                        acc += (double)bias[(int64_t)h * (S + nblk - 1) + delta + nblk - 1];
                    }
                    s[c] = acc;
                    if (acc > m) m = acc;
                }
                double l = 0.0;
                for (int c = 0; c < cols; ++c) {
                    if (!allow[c]) continue;
                    s[c] = exp(s[c] - m);
                    l += s[c];
                }
                for (int c = 0; c < cols; ++c) {
                    if (!allow[c]) continue;
                    const float *vv = c < n ? v + (((int64_t)b * Hkv + hk) * n + c) * D
                                            : side_v + (((int64_t)b * Hkv + hk) * S + (c - n)) * D;
                    for (int x = 0; x < D; ++x) o[x] += s[c] / l * (double)vv[x];
                }
                lse[row] = m + log(l);
            }
        }
    }
    free(isg);
    free(allow);
    free(s);
    free(inband);
    return ORACLE_OK;
}

int oracle_dense_bruteforce(int B, int Hq, int Hkv, int n, int D, const float *q,
                            const float *k, const float *v, const int32_t *global_idx, int g,
                            const float *side_k, const float *side_v, int S, int side_block,
                            const float *bias, const int32_t *window, const int32_t *dilation,
                            int causal, const int32_t *valid_len, double scale, double *out,
                            double *lse) {
    return oracle_dense_bruteforce_ex(B, Hq, Hkv, n, D, q, k, v, global_idx, g, side_k, side_v, S,
                                      side_block, bias, window, dilation, causal, valid_len, scale,
                                      out, lse, NULL);
}

/*
 * oracle_relative_bucket: the T5 bidirectional relative-position bucket as the
 * LongT5 page describes it [LT5-RPE], for num_buckets = 32 and
 * max_distance = 128 (the LongT5Config defaults):
 *   16 buckets per direction, +16 when delta > 0 (memory after query);
 *   a = |delta|; a < 8 -> bucket a (exact);
 *   otherwise 8 + m, m = floor(8 * log(a/8) / log(128/8)) = floor(log2(a^2/64))
 *   clamped to 7, so every a >= 91 (in particular >= max_distance) shares the
 *   last bucket.  The log is evaluated exactly in integers: m is the largest
 *   value in [0,7] with a*a >= 64 * 2^m.
 */
int oracle_relative_bucket(int delta) {
    int ret = delta > 0 ? 16 : 0;
    int64_t a = delta < 0 ? -(int64_t)delta : delta;
    if (a < 8) return ret + (int)a;
    int m = 0;
    while (m < 7 && a * a >= ((int64_t)64 << (m + 1))) ++m;
    return ret + 8 + m;
}

/*
 * oracle_expand_side_bias: per-head bias over relative block distances
 * delta = s - qb, s in [0,S), qb in [0,nblk): out[h][delta + nblk - 1] =
 * table[h][bucket(delta)], table being [Hq][32].
 */
int oracle_expand_side_bias(int Hq, int S, int nblk, const float *table, float *out) {
    if (Hq <= 0 || S <= 0 || nblk <= 0 || !table || !out) return ORACLE_EINVAL;
    int cols = S + nblk - 1;
    for (int h = 0; h < Hq; ++h)
        for (int c = 0; c < cols; ++c) {
            int delta = c - (nblk - 1);
            out[(int64_t)h * cols + c] = table[h * 32 + oracle_relative_bucket(delta)];
        }
    return ORACLE_OK;
}

/*
 * oracle_side_aggregate: Transient-Global block summaries used as side keys or
 * values [LT5-TG, LT5-SRC], read as a plain mean: token j < V belongs to block
 * floor(j / kb); padded tokens (j >= V) belong to no block; S = floor(n / kb)
 * blocks, and a trailing partial block joins the block before it.  Block s is
 * the mean of its member rows (all-zero when it has none).
 * x: [B,H,n,D] -> out: [B,H,S,D] (fp64).
 */
int oracle_side_aggregate(int B, int H, int n, int D, int kb, const float *x,
                          const int32_t *valid_len, double *out) {
    if (B <= 0 || H <= 0 || n <= 0 || D <= 0 || kb <= 0 || n < kb) return ORACLE_EINVAL;
    int S = n / kb;
    for (int b = 0; b < B; ++b) {
        int V = valid_len ? valid_len[b] : n;
        for (int h = 0; h < H; ++h) {
            const float *xb = x + ((int64_t)b * H + h) * n * D;
            double *ob = out + ((int64_t)b * H + h) * S * D;
            for (int s = 0; s < S; ++s) {
                int lo = s * kb;
                int hi = (s == S - 1) ? n : lo + kb;
                if (hi > V) hi = V;
                int cnt = hi > lo ? hi - lo : 0;
                for (int x0 = 0; x0 < D; ++x0) {
                    double acc = 0.0;
                    for (int j = lo; j < hi; ++j) acc += (double)xb[(int64_t)j * D + x0];
                    ob[(int64_t)s * D + x0] = cnt ? acc / cnt : 0.0;
                }
            }
        }
    }
    return ORACLE_OK;
}

/*
 * oracle_backward_ex: gradients of the attention with respect to q, k, v and the
 * side keys / values, for an upstream gradient dout = dL/do, by the chain rule
 * through the softmax of each row [definition of softmax attention; the key sets
 * are those of oracle_forward, side keys appended to every valid row]:
 *   p_j  = exp(s_j - lse),  s_j = scale <q_i, k_j> (+ local bias / side bias)
 *   dp_j = <dout_i, v_j>,   Delta_i = sum_j p_j dp_j,   ds_j = p_j (dp_j - Delta_i)
 *   dq_i = scale sum_j ds_j k_j,  dk_j += scale ds_j q_i,  dv_j += p_j dout_i
 * with j running over K(i) and the side keys (whose rows of dk / dv are dside_k /
 * dside_v).  The biases are inputs, not differentiated.  Padded rows contribute
 * nothing.  dq [B,Hq,n,D], dk/dv [B,Hkv,n,D], dside_k/dside_v [B,Hkv,S,D] (fp64,
 * may be NULL when S = 0) are overwritten.  Work is split over (batch, KV head)
 * pairs, so the accumulations into dk/dv and dside_k/dside_v never race.
 */
int oracle_backward_ex(int B, int Hq, int Hkv, int n, int D, const float *q, const float *k,
                       const float *v, const float *dout, const int32_t *global_idx, int g,
                       const float *side_k, const float *side_v, int S, int side_block,
                       const float *bias, const int32_t *window, const int32_t *dilation,
                       int causal, const int32_t *valid_len, double scale,
                       const oracle_extras *ex, double *dq, double *dk, double *dv,
                       double *dside_k, double *dside_v) {
    oracle_problem P = {B, Hq, Hkv, n, D, q, k, v, global_idx, g, side_k, side_v,
                        S, side_block, bias, window, dilation, causal, valid_len, scale,
                        NULL, 0, NULL, 0, 0};
    apply_extras(&P, ex);
    int rc = check_problem(&P);
    if (rc) return rc;
    if (!dout || !dq || !dk || !dv) return ORACLE_EINVAL;
    if (S > 0 && (!dside_k || !dside_v)) return ORACLE_EINVAL;
    const int G = Hq / Hkv;
    memset(dq, 0, sizeof(double) * (size_t)B * Hq * n * D);
    memset(dk, 0, sizeof(double) * (size_t)B * Hkv * n * D);
    memset(dv, 0, sizeof(double) * (size_t)B * Hkv * n * D);
    if (S > 0) {
        memset(dside_k, 0, sizeof(double) * (size_t)B * Hkv * S * D);
        memset(dside_v, 0, sizeof(double) * (size_t)B * Hkv * S * D);
    }
    int failed = 0;
#pragma omp parallel
    {
        const size_t cap = (size_t)n + 1 + (size_t)(S > 0 ? S : 0);
        int32_t *keys = (int32_t *)malloc(sizeof(int32_t) * (size_t)(n + 1));
        int32_t *wbuf = (int32_t *)malloc(sizeof(int32_t) * (size_t)(n + 1));
        double *sc = (double *)malloc(sizeof(double) * cap);
        double *dp = (double *)malloc(sizeof(double) * cap);
        if (!keys || !wbuf || !sc || !dp) {
#pragma omp atomic write
            failed = 1;
        } else {
#pragma omp for schedule(dynamic, 1)
            for (int bk = 0; bk < B * Hkv; ++bk) {
                const int b = bk / Hkv, hk = bk % Hkv;
                const int V = valid_len ? valid_len[b] : n;
                const float *kb = k + ((int64_t)b * Hkv + hk) * n * D;
                const float *vb = v + ((int64_t)b * Hkv + hk) * n * D;
                const float *skb = S > 0 ? side_k + ((int64_t)b * Hkv + hk) * S * D : NULL;
                const float *svb = S > 0 ? side_v + ((int64_t)b * Hkv + hk) * S * D : NULL;
                double *dkb = dk + ((int64_t)b * Hkv + hk) * n * D;
                double *dvb = dv + ((int64_t)b * Hkv + hk) * n * D;
                double *dskb = S > 0 ? dside_k + ((int64_t)b * Hkv + hk) * S * D : NULL;
                double *dsvb = S > 0 ? dside_v + ((int64_t)b * Hkv + hk) * S * D : NULL;
                for (int h = hk * G; h < (hk + 1) * G; ++h) {
                    for (int i = 0; i < V && i < n; ++i) {
                        int nk = key_set(&P, b, h, i, keys, wbuf);
                        if (nk < 0) continue;
                        const int total = nk + S;
                        if (total <= 0) continue;
                        const int64_t row = ((int64_t)b * Hq + h) * n + i;
                        const float *qi = q + row * D;
                        const float *doi = dout + row * D;
                        double m = -INFINITY;
                        for (int t = 0; t < total; ++t) {
                            if (t < nk)
                                sc[t] = scale * dot(qi, kb + (int64_t)keys[t] * D, D) +
                                        local_bias(&P, b, h, i, keys[t]);
                            else
                                sc[t] = scale * dot(qi, skb + (int64_t)(t - nk) * D, D) +
                                        side_bias(&P, h, i, t - nk);
                            if (sc[t] > m) m = sc[t];
                        }
                        double l = 0.0;
                        for (int t = 0; t < total; ++t) l += exp(sc[t] - m);
                        const double lse = m + log(l);
                        double delta = 0.0;
                        for (int t = 0; t < total; ++t) {
                            const float *vj = t < nk ? vb + (int64_t)keys[t] * D : svb + (int64_t)(t - nk) * D;
                            sc[t] = exp(sc[t] - lse);                        /* p */
                            dp[t] = dot(doi, vj, D);
                            delta += sc[t] * dp[t];
                        }
                        double *dqi = dq + row * D;
                        for (int t = 0; t < total; ++t) {
                            const double ds = sc[t] * (dp[t] - delta);
                            const float *kj;
                            double *dkj, *dvj;
                            if (t < nk) {
                                kj = kb + (int64_t)keys[t] * D;
                                dkj = dkb + (int64_t)keys[t] * D;
                                dvj = dvb + (int64_t)keys[t] * D;
                            } else {
                                kj = skb + (int64_t)(t - nk) * D;
                                dkj = dskb + (int64_t)(t - nk) * D;
                                dvj = dsvb + (int64_t)(t - nk) * D;
                            }
                            for (int x = 0; x < D; ++x) {
                                dqi[x] += scale * ds * (double)kj[x];
                                dkj[x] += scale * ds * (double)qi[x];
                                dvj[x] += sc[t] * (double)doi[x];
                            }
                        }
                    }
                }
            }
        }
        free(keys);
        free(wbuf);
        free(sc);
        free(dp);
    }
    return failed ? ORACLE_ENOMEM : ORACLE_OK;
}

/* oracle_backward_ex without side keys. */
int oracle_backward(int B, int Hq, int Hkv, int n, int D, const float *q, const float *k,
                    const float *v, const float *dout, const int32_t *global_idx, int g,
                    const int32_t *window, const int32_t *dilation, int causal,
                    const int32_t *valid_len, double scale, const oracle_extras *ex,
                    double *dq, double *dk, double *dv) {
    return oracle_backward_ex(B, Hq, Hkv, n, D, q, k, v, dout, global_idx, g, NULL, NULL, 0, 0,
                              NULL, window, dilation, causal, valid_len, scale, ex, dq, dk, dv,
                              NULL, NULL);
}

int oracle_num_threads(void) {
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}
