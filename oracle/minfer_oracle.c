/*
 * minfer_oracle.c -- plain, slow CPU oracle for MInference dynamic sparse
 * prefill (MInference 1.0, arXiv 2407.02490).
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path may load this file:
 * only the tests, the smoke check and the benchmark's CPU-baseline leg call
 * it.  It shares no code, header, table or helper with the CUDA library.
 *
 * Every quantity is computed in fp64 from the same bf16 values the GPU gets
 * (widened exactly to fp32 by the caller), with plain loops and no tiling,
 * blocking or reordering beyond what each definition states.  OpenMP only
 * spreads independent rows / columns over threads; every sum runs in a fixed
 * order, so results do not depend on the thread count.
 *
 * Layout: q [Hq][N][d], k and v [Hkv][N][d], row-major float32.
 * Query head h reads KV head g(h) = floor(h * Hkv / Hq) (grouped-query
 * attention with contiguous groups).
 *
 * Sources (web pages about MInference 1.0):
 *  - hotpaper.ai summary, "key idea": Vertical-Slash heads estimate their
 *    index from the last `last_q` queries against all keys; Block-Sparse heads
 *    mean-pool queries and keys over 64-token blocks to get block-level
 *    attention weights.
 *  - aifetchly "MInference 1.0 Guide", "The Three Fundamental Attention
 *    Topologies": A-shape = initial sink tokens + local causal band;
 *    Vertical-Slash = key columns + diagonals at fixed offsets i - j;
 *    Block-Sparse = B x B tiles, B = 64.
 *  - same guide, "Block-Sparse Kernel Mechanics": block score = query block
 *    against the mean key of each 64-token key block, keep the top-k blocks.
 *  - same guide, "Vertical-Slash Kernel Mechanics": online-softmax attention
 *    over only the selected entries.
 *
 * Readings where the pages leave a step open:
 *  - softmax scale is 1/sqrt(d) (guide, "Calibration Forward Pass");
 *  - Vertical-Slash index: row softmax over the causal keys j <= i of each
 *    of the last `last_q` rows, summed per column j (vertical) and per
 *    diagonal o = i - j (slash); no forced entries;
 *  - top-k ranks by score descending, then index ascending, and returns the
 *    selected indices sorted ascending; k is clamped to the candidate count;
 *  - a slash offset o selects every 64x64 tile (bq, bk) it touches, i.e.
 *    block-diagonal delta = bq - bk with |o - 64 delta| <= 63; such tiles are
 *    computed whole (with the causal mask);
 *  - A-shape: key j is kept for row i iff j <= i and (j < sink or
 *    i - j < window) -- the window counts the query itself;
 *  - a row with no allowed key outputs 0 and lse = -inf.
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

static int kv_head(int h, int Hq, int Hkv) { return (int)(((int64_t)h * Hkv) / Hq); }

static const float* row_ptr(const float* base, int head, int64_t N, int d, int64_t i) {
    return base + ((int64_t)head * N + i) * d;
}

/* scale * <a, b> in fp64 */
static double dot_scaled(const float* a, const float* b, int d, double scale) {
    double acc = 0.0;
    for (int t = 0; t < d; ++t) acc += (double)a[t] * (double)b[t];
    return scale * acc;
}

int oracle_num_threads(void) {
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

/* ------------------------------------------------------------------------ */
/* Vertical-Slash index scores (hotpaper.ai "key idea"; guide, "2. The      */
/* Vertical-Slash Pattern").                                                 */
/*                                                                          */
/* For r = 0..L-1, row i = N - L + r:                                        */
/*   s_j = scale * q_i . k_j for j <= i;  p_j = exp(s_j - m) / sum exp(.)   */
/*   vertical[j] += p_j;   slash[i - j] += p_j.                             */
/* The L x N probability matrix is materialised, then reduced per column    */
/* and per diagonal, rows in ascending order.                               */
/* ------------------------------------------------------------------------ */
int oracle_vs_scores(const float* q, const float* k, int Hq, int Hkv, int N, int d,
                     double scale, int last_q, int h, double* vertical, double* slash) {
    if (!q || !k || !vertical || !slash || Hq <= 0 || Hkv <= 0 || Hq % Hkv || N <= 0 ||
        d <= 0 || last_q <= 0 || h < 0 || h >= Hq)
        return ORACLE_EINVAL;
    const int L = last_q < N ? last_q : N;
    const int g = kv_head(h, Hq, Hkv);
    double* P = (double*)calloc((size_t)L * (size_t)N, sizeof(double));
    if (!P) return ORACLE_ENOMEM;

    #pragma omp parallel for schedule(dynamic, 1)
    for (int r = 0; r < L; ++r) {
        const int64_t i = (int64_t)N - L + r;
        const float* qi = row_ptr(q, h, N, d, i);
        double* Pr = P + (size_t)r * N;
        double m = -INFINITY;
        for (int64_t j = 0; j <= i; ++j) {
            Pr[j] = dot_scaled(qi, row_ptr(k, g, N, d, j), d, scale);
            if (Pr[j] > m) m = Pr[j];
        }
        double l = 0.0;
        for (int64_t j = 0; j <= i; ++j) {
            Pr[j] = exp(Pr[j] - m);
            l += Pr[j];
        }
        for (int64_t j = 0; j <= i; ++j) Pr[j] /= l;
        /* entries j > i stay 0 (causal) */
    }

    #pragma omp parallel for schedule(static)
    for (int64_t j = 0; j < N; ++j) {
        double acc = 0.0;
        for (int r = 0; r < L; ++r) acc += P[(size_t)r * N + j];
        vertical[j] = acc;
    }

    #pragma omp parallel for schedule(static)
    for (int64_t o = 0; o < N; ++o) {
        double acc = 0.0;
        for (int r = 0; r < L; ++r) {
            const int64_t i = (int64_t)N - L + r;
            const int64_t j = i - o;
            if (j >= 0) acc += P[(size_t)r * N + j];
        }
        slash[o] = acc;
    }
    free(P);
    return ORACLE_OK;
}

/* ------------------------------------------------------------------------ */
/* Top-k selection: full sort by (score descending, index ascending), keep   */
/* the first min(k, n), return them sorted ascending.  Returns the count.    */
/* ------------------------------------------------------------------------ */
typedef struct {
    double s;
    int64_t i;
} scored_t;

static int cmp_scored(const void* a, const void* b) {
    const scored_t* x = (const scored_t*)a;
    const scored_t* y = (const scored_t*)b;
    if (x->s > y->s) return -1;
    if (x->s < y->s) return 1;
    return (x->i > y->i) - (x->i < y->i);
}

static int cmp_i64(const void* a, const void* b) {
    int64_t x = *(const int64_t*)a, y = *(const int64_t*)b;
    return (x > y) - (x < y);
}

int64_t oracle_topk(const double* score, int64_t n, int64_t k, int64_t* out) {
    if (!score || !out || n < 0 || k < 0) return -1;
    const int64_t m = k < n ? k : n;
    scored_t* a = (scored_t*)malloc((size_t)(n > 0 ? n : 1) * sizeof(scored_t));
    if (!a) return -1;
    for (int64_t i = 0; i < n; ++i) {
        a[i].s = score[i];
        a[i].i = i;
    }
    qsort(a, (size_t)n, sizeof(scored_t), cmp_scored);
    for (int64_t t = 0; t < m; ++t) out[t] = a[t].i;
    qsort(out, (size_t)m, sizeof(int64_t), cmp_i64);
    free(a);
    return m;
}

/* ------------------------------------------------------------------------ */
/* Block-Sparse index (hotpaper.ai "key idea": 64-token mean pooling of      */
/* queries and keys gives block-level weights; guide, "Block-Sparse Kernel  */
/* Mechanics": score each key block by its mean key, keep the top-k).        */
/*                                                                          */
/* Qm[b] = mean of q rows block*b .. block*b+block-1 (query head h), Km[b]   */
/* likewise for KV head g(h); S[bq][bk] = scale * Qm[bq] . Km[bk], bk <= bq.  */
/* Per row bq keep min(topk, bq+1) blocks by (S desc, bk asc), ascending.    */
/* blk_idx [nB][topk] (unused entries -1), blk_cnt [nB]; scores_opt          */
/* [nB][nB] receives S (NAN above the diagonal) when non-NULL.               */
/* ------------------------------------------------------------------------ */
int oracle_bs_index(const float* q, const float* k, int Hq, int Hkv, int N, int d,
                    double scale, int block, int topk, int h, int32_t* blk_idx,
                    int32_t* blk_cnt, double* scores_opt) {
    if (!q || !k || !blk_idx || !blk_cnt || Hq <= 0 || Hkv <= 0 || Hq % Hkv || N <= 0 ||
        d <= 0 || block <= 0 || N % block || topk < 0 || h < 0 || h >= Hq)
        return ORACLE_EINVAL;
    const int g = kv_head(h, Hq, Hkv);
    const int nB = N / block;
    double* Qm = (double*)calloc((size_t)nB * d, sizeof(double));
    double* Km = (double*)calloc((size_t)nB * d, sizeof(double));
    if (!Qm || !Km) {
        free(Qm);
        free(Km);
        return ORACLE_ENOMEM;
    }
    #pragma omp parallel for schedule(static)
    for (int b = 0; b < nB; ++b) {
        for (int t = 0; t < d; ++t) {
            double sq = 0.0, sk = 0.0;
            for (int r = 0; r < block; ++r) {
                const int64_t i = (int64_t)b * block + r;
                sq += (double)row_ptr(q, h, N, d, i)[t];
                sk += (double)row_ptr(k, g, N, d, i)[t];
            }
            Qm[(size_t)b * d + t] = sq / block;
            Km[(size_t)b * d + t] = sk / block;
        }
    }
    int fail = 0;
    #pragma omp parallel for schedule(dynamic, 4)
    for (int bq = 0; bq < nB; ++bq) {
        scored_t* cand = (scored_t*)malloc((size_t)(bq + 1) * sizeof(scored_t));
        int64_t* sel = (int64_t*)malloc((size_t)(bq + 1) * sizeof(int64_t));
        if (!cand || !sel) {
            free(cand);
            free(sel);
            #pragma omp atomic write
            fail = 1;
            continue;
        }
        for (int bk = 0; bk <= bq; ++bk) {
            double acc = 0.0;
            for (int t = 0; t < d; ++t) acc += Qm[(size_t)bq * d + t] * Km[(size_t)bk * d + t];
            cand[bk].s = scale * acc;
            cand[bk].i = bk;
            if (scores_opt) scores_opt[(size_t)bq * nB + bk] = cand[bk].s;
        }
        if (scores_opt)
            for (int bk = bq + 1; bk < nB; ++bk) scores_opt[(size_t)bq * nB + bk] = NAN;
        qsort(cand, (size_t)bq + 1, sizeof(scored_t), cmp_scored);
        const int cnt = topk < bq + 1 ? topk : bq + 1;
        for (int t = 0; t < cnt; ++t) sel[t] = cand[t].i;
        qsort(sel, (size_t)cnt, sizeof(int64_t), cmp_i64);
        for (int t = 0; t < topk; ++t) blk_idx[(size_t)bq * topk + t] = t < cnt ? (int32_t)sel[t] : -1;
        blk_cnt[bq] = cnt;
        free(cand);
        free(sel);
    }
    free(Qm);
    free(Km);
    return fail ? ORACLE_ENOMEM : ORACLE_OK;
}

/* ------------------------------------------------------------------------ */
/* Slash offsets -> block diagonals.  A diagonal o (key j = i - o) meets the */
/* 64x64 tile (bq, bk) iff some i in that query block has i - o in that key  */
/* block, i.e. |o - block*(bq - bk)| <= block - 1.  D[delta] = 1 iff some    */
/* selected o meets diagonal-block delta.  Offsets outside [0, N) are        */
/* ignored.  Evaluated straight from the definition: every delta against     */
/* every offset.                                                             */
/* ------------------------------------------------------------------------ */
int oracle_slash_deltas(const int32_t* s_idx, int64_t ks, int N, int block, uint8_t* D) {
    if ((!s_idx && ks > 0) || !D || N <= 0 || block <= 0 || N % block || ks < 0)
        return ORACLE_EINVAL;
    const int nB = N / block;
    for (int delta = 0; delta < nB; ++delta) {
        uint8_t hit = 0;
        for (int64_t t = 0; t < ks && !hit; ++t) {
            const int64_t o = s_idx[t];
            if (o < 0 || o >= N) continue;
            const int64_t diff = o - (int64_t)block * delta;
            if (diff <= block - 1 && diff >= -(block - 1)) hit = 1;
        }
        D[delta] = hit;
    }
    return ORACLE_OK;
}

/* ------------------------------------------------------------------------ */
/* Masked softmax attention for selected rows of query head h (guide,       */
/* "Vertical-Slash Kernel Mechanics": softmax over only the selected keys). */
/* For row i: allowed keys j <= i passing the pattern's predicate;          */
/* s_j = scale q_i.k_j; m = max s; l = sum exp(s - m);                      */
/* out_i = sum_j exp(s_j - m)/l * v_j; lse_i = m + ln l.  Two passes, fp64.  */
/* ------------------------------------------------------------------------ */
typedef int (*allow_fn)(const void* ctx, int64_t i, int64_t j);

static int attn_rows(const float* q, const float* k, const float* v, int Hq, int Hkv, int N,
                     int d, double scale, int h, allow_fn allow, const void* ctx,
                     const int64_t* rows, int64_t n_rows, double* out, double* lse) {
    const int g = kv_head(h, Hq, Hkv);
    int fail = 0;
    #pragma omp parallel
    {
        double* s = (double*)malloc((size_t)N * sizeof(double));
        int64_t* js = (int64_t*)malloc((size_t)N * sizeof(int64_t));
        if (!s || !js) {
            #pragma omp atomic write
            fail = 1;
        }
        #pragma omp for schedule(dynamic, 1)
        for (int64_t r = 0; r < n_rows; ++r) {
            if (!s || !js) continue;
            const int64_t i = rows[r];
            double* o = out + (size_t)r * d;
            for (int t = 0; t < d; ++t) o[t] = 0.0;
            if (i < 0 || i >= N) {
                lse[r] = NAN;
                continue;
            }
            const float* qi = row_ptr(q, h, N, d, i);
            int64_t n = 0;
            double m = -INFINITY;
            for (int64_t j = 0; j <= i; ++j) {
                if (!allow(ctx, i, j)) continue;
                js[n] = j;
                s[n] = dot_scaled(qi, row_ptr(k, g, N, d, j), d, scale);
                if (s[n] > m) m = s[n];
                ++n;
            }
            if (n == 0) {
                lse[r] = -INFINITY;
                continue;
            }
            double l = 0.0;
            for (int64_t t = 0; t < n; ++t) {
                s[t] = exp(s[t] - m);
                l += s[t];
            }
            for (int64_t t = 0; t < n; ++t) {
                const double p = s[t] / l;
                const float* vj = row_ptr(v, g, N, d, js[t]);
                for (int c = 0; c < d; ++c) o[c] += p * (double)vj[c];
            }
            lse[r] = m + log(l);
        }
        free(s);
        free(js);
    }
    return fail ? ORACLE_ENOMEM : ORACLE_OK;
}

static int check_attn_args(const float* q, const float* k, const float* v, int Hq, int Hkv,
                           int N, int d, int h, const int64_t* rows, int64_t n_rows,
                           const double* out, const double* lse) {
    return !q || !k || !v || Hq <= 0 || Hkv <= 0 || Hq % Hkv || N <= 0 || d <= 0 || h < 0 ||
           h >= Hq || (!rows && n_rows > 0) || n_rows < 0 || !out || !lse;
}

/* dense causal: every j <= i */
static int allow_all(const void* ctx, int64_t i, int64_t j) {
    (void)ctx;
    (void)i;
    (void)j;
    return 1;
}

int oracle_attn_dense_rows(const float* q, const float* k, const float* v, int Hq, int Hkv,
                           int N, int d, double scale, int h, const int64_t* rows,
                           int64_t n_rows, double* out, double* lse) {
    if (check_attn_args(q, k, v, Hq, Hkv, N, d, h, rows, n_rows, out, lse)) return ORACLE_EINVAL;
    return attn_rows(q, k, v, Hq, Hkv, N, d, scale, h, allow_all, NULL, rows, n_rows, out, lse);
}

/* A-shape (guide, "1. The A-Shape Pattern"): sink keys plus a local band. */
typedef struct {
    int64_t sink, window;
} ashape_ctx;

static int allow_ashape(const void* ctx, int64_t i, int64_t j) {
    const ashape_ctx* c = (const ashape_ctx*)ctx;
    return j < c->sink || i - j < c->window;
}

int oracle_attn_ashape_rows(const float* q, const float* k, const float* v, int Hq, int Hkv,
                            int N, int d, double scale, int h, int sink, int window,
                            const int64_t* rows, int64_t n_rows, double* out, double* lse) {
    if (check_attn_args(q, k, v, Hq, Hkv, N, d, h, rows, n_rows, out, lse) || sink < 0 ||
        window < 0)
        return ORACLE_EINVAL;
    ashape_ctx c = {sink, window};
    return attn_rows(q, k, v, Hq, Hkv, N, d, scale, h, allow_ashape, &c, rows, n_rows, out, lse);
}

/* Vertical-Slash: key j kept for row i iff j is a selected column or the   */
/* block diagonal bq(i) - bk(j) is in D (slash offsets -> tiles, above).     */
typedef struct {
    const uint8_t* in_v; /* [N] */
    const uint8_t* D;    /* [nB] */
    int block;
} vs_ctx;

static int allow_vs(const void* ctx, int64_t i, int64_t j) {
    const vs_ctx* c = (const vs_ctx*)ctx;
    if (c->in_v[j]) return 1;
    return c->D[i / c->block - j / c->block] != 0;
}

int oracle_attn_vs_rows(const float* q, const float* k, const float* v, int Hq, int Hkv, int N,
                        int d, double scale, int h, const int32_t* v_idx, int64_t kv,
                        const int32_t* s_idx, int64_t ks, int block, const int64_t* rows,
                        int64_t n_rows, double* out, double* lse) {
    if (check_attn_args(q, k, v, Hq, Hkv, N, d, h, rows, n_rows, out, lse) || kv < 0 ||
        ks < 0 || (!v_idx && kv > 0) || (!s_idx && ks > 0) || block <= 0 || N % block)
        return ORACLE_EINVAL;
    uint8_t* in_v = (uint8_t*)calloc((size_t)N, 1);
    uint8_t* D = (uint8_t*)calloc((size_t)(N / block), 1);
    if (!in_v || !D) {
        free(in_v);
        free(D);
        return ORACLE_ENOMEM;
    }
    for (int64_t t = 0; t < kv; ++t)
        if (v_idx[t] >= 0 && v_idx[t] < N) in_v[v_idx[t]] = 1;
    int rc = oracle_slash_deltas(s_idx, ks, N, block, D);
    if (rc == ORACLE_OK) {
        vs_ctx c = {in_v, D, block};
        rc = attn_rows(q, k, v, Hq, Hkv, N, d, scale, h, allow_vs, &c, rows, n_rows, out, lse);
    }
    free(in_v);
    free(D);
    return rc;
}

/* Vertical-Slash with range-based slash tiles (aifetchly guide, "2. The   */
/* Vertical-Slash Pattern": the diagonals cost O(N (k_v + k_s)) rather than */
/* whole tiles).  For the 64-row query block bq of row i, diagonal o covers  */
/* the unaligned 64-key range [64 bq - o, 64 bq + 63 - o]; key j is kept     */
/* for row i iff j is a selected column or j lies in the range of some       */
/* selected diagonal.                                                        */
typedef struct {
    const uint8_t* in_v;   /* [N] selected columns */
    const int64_t* s_cnt;  /* [N + 1]: s_cnt[x] = number of selected diagonals o < x */
    int64_t N;
    int block;
} vsr_ctx;

static int allow_vs_range(const void* ctx, int64_t i, int64_t j) {
    const vsr_ctx* c = (const vsr_ctx*)ctx;
    if (c->in_v[j]) return 1;
    const int64_t base = (i / c->block) * c->block; /* 64 bq */
    /* j in [base - o, base + block - 1 - o]  <=>  o in [base - j, base + block - 1 - j] */
    int64_t lo = base - j, hi = base + c->block - 1 - j;
    if (lo < 0) lo = 0;
    if (hi > c->N - 1) hi = c->N - 1;
    if (lo > hi) return 0;
    return c->s_cnt[hi + 1] - c->s_cnt[lo] > 0;
}

/* in_v [N] and s_cnt [N + 1] from the index lists (entries outside [0, N) ignored). */
static int vs_range_tables(int N, const int32_t* v_idx, int64_t kv, const int32_t* s_idx,
                           int64_t ks, uint8_t** in_v, int64_t** s_cnt) {
    *in_v = (uint8_t*)calloc((size_t)N, 1);
    *s_cnt = (int64_t*)calloc((size_t)N + 1, sizeof(int64_t));
    uint8_t* in_s = (uint8_t*)calloc((size_t)N, 1);
    if (!*in_v || !*s_cnt || !in_s) {
        free(*in_v);
        free(*s_cnt);
        free(in_s);
        return ORACLE_ENOMEM;
    }
    for (int64_t t = 0; t < kv; ++t)
        if (v_idx[t] >= 0 && v_idx[t] < N) (*in_v)[v_idx[t]] = 1;
    for (int64_t t = 0; t < ks; ++t)
        if (s_idx[t] >= 0 && s_idx[t] < N) in_s[s_idx[t]] = 1;
    for (int64_t x = 0; x < N; ++x) (*s_cnt)[x + 1] = (*s_cnt)[x] + in_s[x];
    free(in_s);
    return ORACLE_OK;
}

int oracle_attn_vs_range_rows(const float* q, const float* k, const float* v, int Hq, int Hkv,
                              int N, int d, double scale, int h, const int32_t* v_idx,
                              int64_t kv, const int32_t* s_idx, int64_t ks, int block,
                              const int64_t* rows, int64_t n_rows, double* out, double* lse) {
    if (check_attn_args(q, k, v, Hq, Hkv, N, d, h, rows, n_rows, out, lse) || kv < 0 ||
        ks < 0 || (!v_idx && kv > 0) || (!s_idx && ks > 0) || block <= 0 || N % block)
        return ORACLE_EINVAL;
    uint8_t* in_v;
    int64_t* s_cnt;
    int rc = vs_range_tables(N, v_idx, kv, s_idx, ks, &in_v, &s_cnt);
    if (rc) return rc;
    vsr_ctx c = {in_v, s_cnt, N, block};
    rc = attn_rows(q, k, v, Hq, Hkv, N, d, scale, h, allow_vs_range, &c, rows, n_rows, out, lse);
    free(in_v);
    free(s_cnt);
    return rc;
}

/* The causal Vertical-Slash mask itself, mask[i][j] for 0 <= i, j < N (1 =    */
/* kept): whole 64x64 tiles (range = 0) or range-based slash tiles            */
/* (range = 1).  For the pins only (N x N bytes).                              */
int oracle_vs_mask(int N, const int32_t* v_idx, int64_t kv, const int32_t* s_idx, int64_t ks,
                   int block, int range, uint8_t* mask) {
    if (N <= 0 || block <= 0 || N % block || kv < 0 || ks < 0 || (!v_idx && kv > 0) ||
        (!s_idx && ks > 0) || !mask)
        return ORACLE_EINVAL;
    uint8_t* in_v;
    int64_t* s_cnt;
    int rc = vs_range_tables(N, v_idx, kv, s_idx, ks, &in_v, &s_cnt);
    if (rc) return rc;
    uint8_t* D = (uint8_t*)calloc((size_t)(N / block), 1);
    if (!D) {
        free(in_v);
        free(s_cnt);
        return ORACLE_ENOMEM;
    }
    rc = oracle_slash_deltas(s_idx, ks, N, block, D);
    if (rc == ORACLE_OK) {
        vs_ctx ca = {in_v, D, block};
        vsr_ctx cr = {in_v, s_cnt, N, block};
        for (int64_t i = 0; i < N; ++i)
            for (int64_t j = 0; j < N; ++j)
                mask[(size_t)i * N + j] =
                    (uint8_t)(j <= i && (range ? allow_vs_range(&cr, i, j) : allow_vs(&ca, i, j)));
    }
    free(in_v);
    free(s_cnt);
    free(D);
    return rc;
}

/* Block-Sparse: key j kept for row i iff bk(j) is listed for bq(i). */
typedef struct {
    const uint8_t* sel; /* [nB][nB], sel[bq*nB + bk] */
    int block, nB;
} bs_ctx;

static int allow_bs(const void* ctx, int64_t i, int64_t j) {
    const bs_ctx* c = (const bs_ctx*)ctx;
    return c->sel[(size_t)(i / c->block) * c->nB + (size_t)(j / c->block)] != 0;
}

int oracle_attn_bs_rows(const float* q, const float* k, const float* v, int Hq, int Hkv, int N,
                        int d, double scale, int h, const int32_t* blk_idx,
                        const int32_t* blk_cnt, int topk, int block, const int64_t* rows,
                        int64_t n_rows, double* out, double* lse) {
    if (check_attn_args(q, k, v, Hq, Hkv, N, d, h, rows, n_rows, out, lse) || !blk_idx ||
        !blk_cnt || topk < 0 || block <= 0 || N % block)
        return ORACLE_EINVAL;
    const int nB = N / block;
    uint8_t* sel = (uint8_t*)calloc((size_t)nB * nB, 1);
    if (!sel) return ORACLE_ENOMEM;
    for (int bq = 0; bq < nB; ++bq) {
        const int cnt = blk_cnt[bq] < topk ? blk_cnt[bq] : topk;
        for (int t = 0; t < cnt; ++t) {
            const int bk = blk_idx[(size_t)bq * topk + t];
            if (bk >= 0 && bk < nB) sel[(size_t)bq * nB + bk] = 1;
        }
    }
    bs_ctx c = {sel, block, nB};
    int rc = attn_rows(q, k, v, Hq, Hkv, N, d, scale, h, allow_bs, &c, rows, n_rows, out, lse);
    free(sel);
    return rc;
}
