/*
 * oracle.c -- plain fp64 CPU reference for shared-prefix attention.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path may link, load or
 * call this file; only the tests, the smoke check and the CPU-baseline leg
 * of the benchmark do.  It shares no code, header or table with the CUDA
 * library.
 *
 * Every function here is the *definition* of the quantity, written out with
 * no blocking, fusion or reordering: for each (query row, query head) the
 * logits of every visible key are formed in fp64, then the softmax-weighted
 * sum of the value rows and the natural-log log-sum-exp of the logits.
 * Subtracting the row maximum before exponentiating is the only
 * rearrangement, and it is exact in real arithmetic.
 *
 * Sources (web pages, by title and section):
 *  - "KV-0 redundancy prefix sharing attention mask design" (PrefixSharing
 *    PR #50), design summary: the prefix K/V is stored once in a flat,
 *    deduplicated layout [prefix; s_1; ...; s_N]; visibility comes from a
 *    block-causal mask; one forward pass is mathematically equivalent to
 *    running every [prefix; s_i] on its own.  Key changes, section 2: the
 *    mask for the flat GRPO case and for multi-level tree / chain cases.
 *  - "Split-KV flash-decode attention for EAGLE target-verify" (sglang PR
 *    #27382), implementation breakdown item 1: verify queries attend to the
 *    whole cached prefix plus a small causal draft-draft block.
 *  - "SM8x sparse-MLA prefill fallback re-reads the shared MLA latent once
 *    per head" (vLLM issue), environment: one shared 512-wide latent serves
 *    as both K and V for all 64 heads; every query attends to its own top-k
 *    index list (index_topk = 2048).
 *
 * Readings where the pages are silent (also listed in the design notes):
 *  - Segments form a tree in flat order, parents before children.  A query
 *    in segment s sees key k iff k <= q and the segment of k is s or one of
 *    its ancestors.  Flat GRPO is the depth-2 tree; a chain is a path.
 *  - GQA maps query head h to KV head h / (Hq / Hkv).
 *  - LSE is the natural log of the sum of exp(scaled logits).
 *  - A row with no visible key gets O = 0 and LSE = -inf.
 *
 * Inputs are fp32 arrays that hold the exact values the GPU reads (bf16
 * inputs are widened without rounding); all arithmetic is fp64.
 * Threads split the list of rows; each (row, head) is computed by one thread
 * in one pass, so threading changes no arithmetic.
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#ifndef ORACLE_MUTANT
#define ORACLE_MUTANT 0 /* tests build deliberately broken copies with 1..N */
#endif

/* ------------------------------------------------------------------ */
/* segment-tree visibility                                              */
/* ------------------------------------------------------------------ */

/* Segment index of every flat token.  seg_start is ascending. */
static void token_segments(const int32_t *seg_start, const int32_t *seg_len,
                           int nseg, int T, int32_t *tok_seg) {
    for (int t = 0; t < T; ++t) tok_seg[t] = -1;
    for (int s = 0; s < nseg; ++s)
        for (int t = seg_start[s]; t < seg_start[s] + seg_len[s]; ++t)
            if (t >= 0 && t < T) tok_seg[t] = s;
}

/* 1 iff segment a is segment s or one of its ancestors. */
static int ancestor_or_self(const int32_t *parent, int a, int s) {
    while (s >= 0) {
        if (s == a) return 1;
        s = parent[s];
    }
    return 0;
}

static int visible(const int32_t *tok_seg, const int32_t *parent, int q, int k) {
#if ORACLE_MUTANT == 2
    if (k >= q) return 0;         /* planted: strict causality drops the diagonal */
#else
    if (k > q) return 0;
#endif
    int sq = tok_seg[q], sk = tok_seg[k];
    if (sq < 0 || sk < 0) return 0;
#if ORACLE_MUTANT == 4
    return sq == sk;              /* planted: suffixes no longer see the prefix */
#else
    return ancestor_or_self(parent, sk, sq);
#endif
}

/* Dense visibility rows [row0, row0 + nrows) x [0, T) as bytes. */
int oracle_visibility(const int32_t *seg_start, const int32_t *seg_len,
                      const int32_t *parent, int nseg, int T, int row0,
                      int nrows, uint8_t *out) {
    int32_t *tok_seg = (int32_t *)malloc(sizeof(int32_t) * (size_t)(T > 0 ? T : 1));
    if (!tok_seg) return -1;
    token_segments(seg_start, seg_len, nseg, T, tok_seg);
    for (int r = 0; r < nrows; ++r)
        for (int k = 0; k < T; ++k)
            out[(size_t)r * T + k] = (uint8_t)visible(tok_seg, parent, row0 + r, k);
    free(tok_seg);
    return 0;
}

/* ------------------------------------------------------------------ */
/* one softmax-attention row: the definition                            */
/* ------------------------------------------------------------------ */

/* Given the logits z[0..n) of the visible keys and pointers to their value
 * rows, write O (length d) and return the LSE. */
static double softmax_row(const double *z, const float *const *vrows, int n,
                          int d, double *o) {
    for (int c = 0; c < d; ++c) o[c] = 0.0;
    if (n == 0) return -INFINITY;
    double m = -INFINITY;
    for (int i = 0; i < n; ++i) if (z[i] > m) m = z[i];
    double l = 0.0;
    for (int i = 0; i < n; ++i) l += exp(z[i] - m);
    for (int i = 0; i < n; ++i) {
        double p = exp(z[i] - m) / l;
        for (int c = 0; c < d; ++c) o[c] += p * (double)vrows[i][c];
    }
#if ORACLE_MUTANT == 5
    return log(l);                /* planted: LSE forgets the row maximum */
#else
    return m + log(l);
#endif
}

static double dot(const float *a, const float *b, int d) {
    double s = 0.0;
    for (int c = 0; c < d; ++c) s += (double)a[c] * (double)b[c];
    return s;
}

static double apply_scale(double qk, double scale) {
#if ORACLE_MUTANT == 1
    (void)scale;
    return qk;                    /* planted: the softmax scale is dropped */
#else
    return scale * qk;
#endif
}

static int kv_head_of(int h, int Hq, int Hkv) {
#if ORACLE_MUTANT == 3
    (void)Hq;
    return h % Hkv;               /* planted: interleaved instead of contiguous GQA */
#else
    return h / (Hq / Hkv);
#endif
}

/* ------------------------------------------------------------------ */
/* threading helper: rows are split into contiguous ranges               */
/* ------------------------------------------------------------------ */

typedef void (*row_fn)(void *ctx, int r, double *zbuf, const float **vbuf, double *obuf);

typedef struct {
    row_fn fn;
    void *ctx;
    int r0, r1;
    int zcap, d;
} worker_arg;

static void *worker(void *p) {
    worker_arg *w = (worker_arg *)p;
    double *z = (double *)malloc(sizeof(double) * (size_t)(w->zcap > 0 ? w->zcap : 1));
    const float **vr = (const float **)malloc(sizeof(float *) * (size_t)(w->zcap > 0 ? w->zcap : 1));
    double *o = (double *)malloc(sizeof(double) * (size_t)w->d);
    if (z && vr && o)
        for (int r = w->r0; r < w->r1; ++r) w->fn(w->ctx, r, z, vr, o);
    free(z);
    free((void *)vr);
    free(o);
    return NULL;
}

static void run_rows(row_fn fn, void *ctx, int nrows, int zcap, int d, int nthreads) {
    if (nthreads < 1) nthreads = 1;
    if (nthreads > nrows) nthreads = nrows > 0 ? nrows : 1;
    pthread_t *th = (pthread_t *)malloc(sizeof(pthread_t) * (size_t)nthreads);
    worker_arg *args = (worker_arg *)malloc(sizeof(worker_arg) * (size_t)nthreads);
    for (int i = 0; i < nthreads; ++i) {
        args[i].fn = fn;
        args[i].ctx = ctx;
        args[i].r0 = (int)((int64_t)nrows * i / nthreads);
        args[i].r1 = (int)((int64_t)nrows * (i + 1) / nthreads);
        args[i].zcap = zcap;
        args[i].d = d;
        pthread_create(&th[i], NULL, worker, &args[i]);
    }
    for (int i = 0; i < nthreads; ++i) pthread_join(th[i], NULL);
    free(th);
    free(args);
}

/* ------------------------------------------------------------------ */
/* prefill over the flat packed layout                                  */
/* ------------------------------------------------------------------ */

typedef struct {
    const float *q, *k, *v;
    int T, Hq, Hkv, d;
    double scale;
    const int32_t *tok_seg, *parent;
    const int32_t *rows;
    double *o, *lse;
} prefill_ctx;

static void prefill_row(void *p, int r, double *z, const float **vr, double *o) {
    prefill_ctx *c = (prefill_ctx *)p;
    int qi = c->rows[r];
    for (int h = 0; h < c->Hq; ++h) {
        int kvh = kv_head_of(h, c->Hq, c->Hkv);
        const float *qrow = c->q + ((size_t)qi * c->Hq + h) * c->d;
        int n = 0;
        for (int kj = 0; kj < c->T; ++kj) {
            if (!visible(c->tok_seg, c->parent, qi, kj)) continue;
            const float *krow = c->k + ((size_t)kj * c->Hkv + kvh) * c->d;
            z[n] = apply_scale(dot(qrow, krow, c->d), c->scale);
            vr[n] = c->v + ((size_t)kj * c->Hkv + kvh) * c->d;
            ++n;
        }
        double l = softmax_row(z, vr, n, c->d, o);
        memcpy(c->o + ((size_t)r * c->Hq + h) * c->d, o, sizeof(double) * (size_t)c->d);
        c->lse[(size_t)r * c->Hq + h] = l;
    }
}

/*
 * q [T, Hq, d], k/v [T, Hkv, d] (fp32 holding the exact input values),
 * segments (seg_start, seg_len, parent) over the flat token range [0, T),
 * rows[nrows] = the flat query rows to evaluate.
 * o [nrows, Hq, d], lse [nrows, Hq] (fp64).
 */
int oracle_prefill(const float *q, const float *k, const float *v, int T, int Hq,
                   int Hkv, int d, double scale, const int32_t *seg_start,
                   const int32_t *seg_len, const int32_t *parent, int nseg,
                   const int32_t *rows, int nrows, double *o, double *lse,
                   int nthreads) {
    if (Hkv <= 0 || Hq % Hkv != 0 || d <= 0 || T < 0) return -1;
    int32_t *tok_seg = (int32_t *)malloc(sizeof(int32_t) * (size_t)(T > 0 ? T : 1));
    if (!tok_seg) return -1;
    token_segments(seg_start, seg_len, nseg, T, tok_seg);
    prefill_ctx c = {q, k, v, T, Hq, Hkv, d, scale, tok_seg, parent, rows, o, lse};
    run_rows(prefill_row, &c, nrows, T, d, nthreads);
    free(tok_seg);
    return 0;
}

/* ------------------------------------------------------------------ */
/* backward of the prefill: gradients of O = softmax(scale Q K^T) V      */
/* ------------------------------------------------------------------ */

/*
 * "KV-0 redundancy prefix sharing attention mask design", design summary and
 * test plan: the flat layout must give the same gradients as running every
 * [prefix; s_i] on its own, so the prefix K/V collect the gradients of all
 * suffixes that see them.  Written out from the definition of softmax
 * attention for one query row q with visible keys k:
 *   P_k = softmax_k(scale q.k_k), O = sum_k P_k v_k, D = dO . O,
 *   dV_k += P_k dO, dP_k = dO . v_k, dS_k = P_k (dP_k - D),
 *   dQ += scale sum_k dS_k k_k, dK_k += scale dS_k q.
 * A query head h contributes to KV head h / (Hq / Hkv).
 */
typedef struct {
    const float *q, *k, *v, *dout;
    int T, Hq, Hkv, d;
    double scale;
    const int32_t *tok_seg, *parent;
    double *dq, *dk, *dv;
    int kvh0, kvh1;
} bwd_ctx;

static void *bwd_worker(void *p) {
    bwd_ctx *c = (bwd_ctx *)p;
    int G = c->Hq / c->Hkv, d = c->d, T = c->T;
    double *z = (double *)malloc(sizeof(double) * (size_t)(T > 0 ? T : 1));
    int32_t *ks = (int32_t *)malloc(sizeof(int32_t) * (size_t)(T > 0 ? T : 1));
    double *o = (double *)malloc(sizeof(double) * (size_t)d);
    for (int kvh = c->kvh0; kvh < c->kvh1; ++kvh) {
        for (int g = 0; g < G; ++g) {
            int h = kvh * G + g;
            for (int qi = 0; qi < T; ++qi) {
                const float *qrow = c->q + ((size_t)qi * c->Hq + h) * d;
                const float *dorow = c->dout + ((size_t)qi * c->Hq + h) * d;
                int n = 0;
                for (int kj = 0; kj < T; ++kj) {
                    if (!visible(c->tok_seg, c->parent, qi, kj)) continue;
                    const float *krow = c->k + ((size_t)kj * c->Hkv + kvh) * d;
                    z[n] = c->scale * dot(qrow, krow, d);
                    ks[n++] = kj;
                }
                if (n == 0) continue;
                double m = -INFINITY, l = 0.0;
                for (int i = 0; i < n; ++i) if (z[i] > m) m = z[i];
                for (int i = 0; i < n; ++i) { z[i] = exp(z[i] - m); l += z[i]; }
                for (int i = 0; i < n; ++i) z[i] /= l; /* z now holds P */
                for (int e = 0; e < d; ++e) o[e] = 0.0;
                for (int i = 0; i < n; ++i) {
                    const float *vrow = c->v + ((size_t)ks[i] * c->Hkv + kvh) * d;
                    for (int e = 0; e < d; ++e) o[e] += z[i] * (double)vrow[e];
                }
                double D = 0.0;
                for (int e = 0; e < d; ++e) D += (double)dorow[e] * o[e];
                double *dqrow = c->dq + ((size_t)qi * c->Hq + h) * d;
                for (int i = 0; i < n; ++i) {
                    const float *krow = c->k + ((size_t)ks[i] * c->Hkv + kvh) * d;
                    const float *vrow = c->v + ((size_t)ks[i] * c->Hkv + kvh) * d;
                    double dp = dot(dorow, vrow, d);
#if ORACLE_MUTANT == 8
                    double dsc = z[i] * dp;     /* planted: the softmax Jacobian loses D */
#else
                    double dsc = z[i] * (dp - D);
#endif
                    double *dkrow = c->dk + ((size_t)ks[i] * c->Hkv + kvh) * d;
                    double *dvrow = c->dv + ((size_t)ks[i] * c->Hkv + kvh) * d;
                    for (int e = 0; e < d; ++e) {
                        dqrow[e] += c->scale * dsc * (double)krow[e];
#if ORACLE_MUTANT == 9
                        dkrow[e] += dsc * (double)qrow[e]; /* planted: dk loses the scale */
#else
                        dkrow[e] += c->scale * dsc * (double)qrow[e];
#endif
                        dvrow[e] += z[i] * (double)dorow[e];
                    }
                }
            }
        }
    }
    free(z);
    free(ks);
    free(o);
    return NULL;
}

/*
 * q, dout [T, Hq, d]; k, v [T, Hkv, d] (fp32 holding the exact input values);
 * segments as for oracle_prefill.  dq [T, Hq, d], dk, dv [T, Hkv, d] (fp64,
 * written).  Threads split the KV heads, so no two threads write one output.
 */
int oracle_prefill_bwd(const float *q, const float *k, const float *v, const float *dout,
                       int T, int Hq, int Hkv, int d, double scale,
                       const int32_t *seg_start, const int32_t *seg_len,
                       const int32_t *parent, int nseg, double *dq, double *dk, double *dv,
                       int nthreads) {
    if (Hkv <= 0 || Hq % Hkv != 0 || d <= 0 || T < 0) return -1;
    int32_t *tok_seg = (int32_t *)malloc(sizeof(int32_t) * (size_t)(T > 0 ? T : 1));
    if (!tok_seg) return -1;
    token_segments(seg_start, seg_len, nseg, T, tok_seg);
    memset(dq, 0, sizeof(double) * (size_t)T * Hq * d);
    memset(dk, 0, sizeof(double) * (size_t)T * Hkv * d);
    memset(dv, 0, sizeof(double) * (size_t)T * Hkv * d);
    if (nthreads < 1) nthreads = 1;
    if (nthreads > Hkv) nthreads = Hkv;
    pthread_t *th = (pthread_t *)malloc(sizeof(pthread_t) * (size_t)nthreads);
    bwd_ctx *cs = (bwd_ctx *)malloc(sizeof(bwd_ctx) * (size_t)nthreads);
    for (int i = 0; i < nthreads; ++i) {
        bwd_ctx c = {q, k, v, dout, T, Hq, Hkv, d, scale, tok_seg, parent, dq, dk, dv,
                     Hkv * i / nthreads, Hkv * (i + 1) / nthreads};
        cs[i] = c;
        pthread_create(&th[i], NULL, bwd_worker, &cs[i]);
    }
    for (int i = 0; i < nthreads; ++i) pthread_join(th[i], NULL);
    free(th);
    free(cs);
    free(tok_seg);
    return 0;
}

/*
 * dq of selected rows only (dq of a row depends on that row's softmax
 * alone): dq[r] = scale sum_k P_k (dO . v_k - dO . O) k_k for row rows[r].
 * dq [nrows, Hq, d] (fp64, written).
 */
typedef struct {
    const float *q, *k, *v, *dout;
    int T, Hq, Hkv, d;
    double scale;
    const int32_t *tok_seg, *parent, *rows;
    double *dq;
} bwdq_ctx;

static void bwdq_row(void *p, int r, double *z, const float **vr, double *o) {
    bwdq_ctx *c = (bwdq_ctx *)p;
    int qi = c->rows[r], d = c->d;
    for (int h = 0; h < c->Hq; ++h) {
        int kvh = kv_head_of(h, c->Hq, c->Hkv);
        const float *qrow = c->q + ((size_t)qi * c->Hq + h) * d;
        const float *dorow = c->dout + ((size_t)qi * c->Hq + h) * d;
        double *dqrow = c->dq + ((size_t)r * c->Hq + h) * d;
        for (int e = 0; e < d; ++e) dqrow[e] = 0.0;
        int n = 0;
        for (int kj = 0; kj < c->T; ++kj) {
            if (!visible(c->tok_seg, c->parent, qi, kj)) continue;
            z[n] = c->scale * dot(qrow, c->k + ((size_t)kj * c->Hkv + kvh) * d, d);
            vr[n++] = c->k + ((size_t)kj * c->Hkv + kvh) * d; /* the key row, for dq */
        }
        if (n == 0) continue;
        double m = -INFINITY, l = 0.0;
        for (int i = 0; i < n; ++i) if (z[i] > m) m = z[i];
        for (int i = 0; i < n; ++i) { z[i] = exp(z[i] - m); l += z[i]; }
        for (int e = 0; e < d; ++e) o[e] = 0.0;
        for (int i = 0; i < n; ++i) {
            size_t kj = (size_t)(vr[i] - c->k) / ((size_t)c->Hkv * d);
            const float *vrow = c->v + (kj * c->Hkv + kvh) * d;
            for (int e = 0; e < d; ++e) o[e] += z[i] / l * (double)vrow[e];
        }
        double D = 0.0;
        for (int e = 0; e < d; ++e) D += (double)dorow[e] * o[e];
        for (int i = 0; i < n; ++i) {
            size_t kj = (size_t)(vr[i] - c->k) / ((size_t)c->Hkv * d);
            const float *vrow = c->v + (kj * c->Hkv + kvh) * d;
            double dsc = z[i] / l * (dot(dorow, vrow, d) - D);
            for (int e = 0; e < d; ++e) dqrow[e] += c->scale * dsc * (double)vr[i][e];
        }
    }
}

int oracle_prefill_bwd_dq(const float *q, const float *k, const float *v, const float *dout,
                          int T, int Hq, int Hkv, int d, double scale,
                          const int32_t *seg_start, const int32_t *seg_len,
                          const int32_t *parent, int nseg, const int32_t *rows, int nrows,
                          double *dq, int nthreads) {
    if (Hkv <= 0 || Hq % Hkv != 0 || d <= 0 || T < 0) return -1;
    int32_t *tok_seg = (int32_t *)malloc(sizeof(int32_t) * (size_t)(T > 0 ? T : 1));
    if (!tok_seg) return -1;
    token_segments(seg_start, seg_len, nseg, T, tok_seg);
    bwdq_ctx c = {q, k, v, dout, T, Hq, Hkv, d, scale, tok_seg, parent, rows, dq};
    run_rows(bwdq_row, &c, nrows, T, d, nthreads);
    free(tok_seg);
    return 0;
}

/* ------------------------------------------------------------------ */
/* speculative verify: cached prefix plus a causal draft block          */
/* ------------------------------------------------------------------ */

typedef struct {
    const float *qd, *kd, *vd, *kc, *vc;
    const int64_t *indptr; /* NULL: every request shares cache tokens [0, shared_len) */
    int64_t shared_len;
    int Ld, Hq, Hkv, d;
    double scale;
    const int32_t *rows;
    double *o, *lse;
    const uint8_t *dmask;  /* NULL: causal draft block; else [B*Ld, Ld], draft j sees i */
    /* extend form (all three NULL for the uniform, contiguous case):
     * qo_indptr   request b's draft rows are [qo_indptr[b], qo_indptr[b+1])
     * kv_indices  prefix position t of the flat kv_indptr range is cache row
     *             kv_indices[t] (a page table with one token per page)
     * mask_indptr request b's draft mask starts at dmask[mask_indptr[b]] */
    const int64_t *qo_indptr;
    const int32_t *kv_indices;
    const int64_t *mask_indptr;
} verify_ctx;

static void verify_row(void *p, int r, double *z, const float **vr, double *o) {
    verify_ctx *c = (verify_ctx *)p;
    int row = c->rows[r]; /* flat draft row: request b, draft j */
    int b, j, Lb;
    int64_t q0;
    if (c->qo_indptr) {
        b = 0;
        while (row >= c->qo_indptr[b + 1]) ++b;
        q0 = c->qo_indptr[b];
        Lb = (int)(c->qo_indptr[b + 1] - q0);
    } else {
        b = row / c->Ld;
        q0 = (int64_t)b * c->Ld;
        Lb = c->Ld;
    }
    j = (int)(row - q0);
    /* request b's mask is Lb x Lb, row-major, draft j's row first at mrow */
    const uint8_t *mrow = NULL;
    if (c->dmask)
        mrow = c->dmask + (c->mask_indptr ? c->mask_indptr[b] : q0 * Lb) + (int64_t)j * Lb;
    int64_t p0 = c->indptr ? c->indptr[b] : 0;
#if ORACLE_MUTANT == 13
    int64_t p1 = c->indptr ? c->indptr[b + 1] : c->shared_len - 1; /* planted: shared prefix short by one */
#else
    int64_t p1 = c->indptr ? c->indptr[b + 1] : c->shared_len;
#endif
    for (int h = 0; h < c->Hq; ++h) {
        int kvh = kv_head_of(h, c->Hq, c->Hkv);
        const float *qrow = c->qd + ((size_t)row * c->Hq + h) * c->d;
        int n = 0;
        for (int64_t t = p0; t < p1; ++t) { /* the whole cached prefix */
#if ORACLE_MUTANT == 7
            int64_t slot = t;  /* planted: the page table is ignored */
#else
            int64_t slot = c->kv_indices ? c->kv_indices[t] : t;
#endif
            const float *krow = c->kc + ((size_t)slot * c->Hkv + kvh) * c->d;
            z[n] = apply_scale(dot(qrow, krow, c->d), c->scale);
            vr[n] = c->vc + ((size_t)slot * c->Hkv + kvh) * c->d;
            ++n;
        }
#if ORACLE_MUTANT == 6
        for (int i = 0; i < Lb; ++i) {  /* planted: the draft block is not causal */
#else
        for (int i = 0; i < Lb; ++i) {
            /* drafts 0..j (the causal draft block), or the tree mask's row j */
            if (mrow ? !mrow[i] : i > j) continue;
#endif
            size_t dr = (size_t)q0 + i;
            const float *krow = c->kd + (dr * c->Hkv + kvh) * c->d;
            z[n] = apply_scale(dot(qrow, krow, c->d), c->scale);
            vr[n] = c->vd + (dr * c->Hkv + kvh) * c->d;
            ++n;
        }
        double l = softmax_row(z, vr, n, c->d, o);
        memcpy(c->o + ((size_t)r * c->Hq + h) * c->d, o, sizeof(double) * (size_t)c->d);
        c->lse[(size_t)r * c->Hq + h] = l;
    }
}

/*
 * q_draft [B*Ld, Hq, d]; k_draft/v_draft [B*Ld, Hkv, d];
 * k_cache/v_cache [Ntok, Hkv, d]; request b's prefix is cache tokens
 * [indptr[b], indptr[b+1]).  rows = draft rows b*Ld + j to evaluate.
 */
int oracle_verify(const float *qd, const float *kd, const float *vd,
                  const float *kc, const float *vc, const int64_t *indptr,
                  int B, int Ld, int Hq, int Hkv, int d, double scale,
                  const int32_t *rows, int nrows, double *o, double *lse,
                  int nthreads) {
    if (Hkv <= 0 || Hq % Hkv != 0 || d <= 0 || B < 0 || Ld <= 0) return -1;
    int64_t maxlen = 0;
    for (int b = 0; b < B; ++b)
        if (indptr[b + 1] - indptr[b] > maxlen) maxlen = indptr[b + 1] - indptr[b];
    verify_ctx c = {qd, kd, vd, kc, vc, indptr, 0, Ld, Hq, Hkv, d, scale, rows, o, lse, NULL,
                     NULL, NULL, NULL};
    run_rows(verify_row, &c, nrows, (int)maxlen + Ld, d, nthreads);
    return 0;
}

/*
 * Tree verify: "Split-KV flash-decode attention for EAGLE target-verify"
 * (can_handle: topk > 1 brings a custom draft mask; the prefix is skipped by
 * the custom mask, so every draft still sees the whole cached prefix).
 * dmask [B*Ld, Ld] uint8: draft j of request b sees draft i of b iff
 * dmask[(b*Ld + j)*Ld + i] != 0.  Otherwise as oracle_verify.
 */
int oracle_verify_tree(const float *qd, const float *kd, const float *vd,
                       const float *kc, const float *vc, const int64_t *indptr,
                       const uint8_t *dmask, int B, int Ld, int Hq, int Hkv, int d,
                       double scale, const int32_t *rows, int nrows, double *o,
                       double *lse, int nthreads) {
    if (Hkv <= 0 || Hq % Hkv != 0 || d <= 0 || B < 0 || Ld <= 0 || !dmask) return -1;
    int64_t maxlen = 0;
    for (int b = 0; b < B; ++b)
        if (indptr[b + 1] - indptr[b] > maxlen) maxlen = indptr[b + 1] - indptr[b];
    verify_ctx c = {qd, kd, vd, kc, vc, indptr, 0, Ld, Hq, Hkv, d, scale, rows, o, lse, dmask,
                     NULL, NULL, NULL};
    run_rows(verify_row, &c, nrows, (int)maxlen + Ld, d, nthreads);
    return 0;
}

/*
 * Verify in the general extend form of "Split-KV flash-decode attention for
 * EAGLE target-verify" (the verify entry's signature: qo_indptr, kv_indptr,
 * kv_indices, custom_mask, mask_indptr; can_handle names ragged extend and
 * the custom mask as the cases its split path leaves out).
 *   qo_indptr [B+1]   request b's draft rows are [qo_indptr[b], qo_indptr[b+1])
 *                     of q/k/v_draft; Lb = their count (0 allowed)
 *   kv_indptr [B+1]   request b's prefix positions are [kv_indptr[b], kv_indptr[b+1])
 *   kv_indices        NULL, or prefix position t is cache row kv_indices[t]
 *   dmask             NULL: causal draft block; else request b's Lb x Lb mask
 *                     starts at dmask[mask_indptr[b]], draft j sees draft i
 *                     iff its (j, i) byte is non-zero
 * Every draft row sees its whole prefix.  rows: flat draft rows to evaluate.
 */
int oracle_verify_extend(const float *qd, const float *kd, const float *vd,
                         const float *kc, const float *vc, const int64_t *qo_indptr,
                         const int64_t *kv_indptr, const int32_t *kv_indices,
                         const uint8_t *dmask, const int64_t *mask_indptr, int B, int Hq,
                         int Hkv, int d, double scale, const int32_t *rows, int nrows,
                         double *o, double *lse, int nthreads) {
    if (Hkv <= 0 || Hq % Hkv != 0 || d <= 0 || B < 0 || !qo_indptr || !kv_indptr) return -1;
    if (dmask && !mask_indptr) return -1;
    int64_t maxlen = 0, maxld = 1;
    for (int b = 0; b < B; ++b) {
        if (kv_indptr[b + 1] - kv_indptr[b] > maxlen) maxlen = kv_indptr[b + 1] - kv_indptr[b];
        if (qo_indptr[b + 1] - qo_indptr[b] > maxld) maxld = qo_indptr[b + 1] - qo_indptr[b];
    }
    for (int r = 0; r < nrows; ++r)
        if (rows[r] < 0 || rows[r] >= qo_indptr[B]) return -1;
    verify_ctx c = {qd, kd, vd, kc, vc, kv_indptr, 0, 1, Hq, Hkv, d, scale, rows, o, lse, dmask,
                    qo_indptr, kv_indices, mask_indptr};
    run_rows(verify_row, &c, nrows, (int)(maxlen + maxld), d, nthreads);
    return 0;
}

/*
 * Verify against one prefix shared by every request: the prefix K/V is
 * stored once ("KV-0 redundancy prefix sharing attention mask design",
 * design summary) and every draft row of every request sees all of it plus
 * its own causal draft block ("Split-KV flash-decode attention for EAGLE
 * target-verify", implementation item 1).  k_prefix/v_prefix [L, Hkv, d];
 * the other arguments are those of oracle_verify.  By definition this
 * equals oracle_verify on a cache holding B copies of the prefix.
 */
int oracle_verify_shared(const float *qd, const float *kd, const float *vd,
                         const float *kp, const float *vp, int64_t L,
                         int B, int Ld, int Hq, int Hkv, int d, double scale,
                         const int32_t *rows, int nrows, double *o, double *lse,
                         int nthreads) {
    if (Hkv <= 0 || Hq % Hkv != 0 || d <= 0 || B < 0 || Ld <= 0 || L < 0) return -1;
    verify_ctx c = {qd, kd, vd, kp, vp, NULL, L, Ld, Hq, Hkv, d, scale, rows, o, lse, NULL,
                     NULL, NULL, NULL};
    run_rows(verify_row, &c, nrows, (int)L + Ld, d, nthreads);
    return 0;
}

/*
 * Tree verify against one shared prefix: oracle_verify_shared with the draft
 * block given by dmask [B*Ld, Ld] as in oracle_verify_tree (the prefix stays
 * fully visible).  By definition this equals oracle_verify_tree on a cache
 * holding B copies of the prefix.
 */
int oracle_verify_shared_tree(const float *qd, const float *kd, const float *vd,
                              const float *kp, const float *vp, int64_t L,
                              const uint8_t *dmask, int B, int Ld, int Hq, int Hkv, int d,
                              double scale, const int32_t *rows, int nrows, double *o,
                              double *lse, int nthreads) {
    if (Hkv <= 0 || Hq % Hkv != 0 || d <= 0 || B < 0 || Ld <= 0 || L < 0 || !dmask) return -1;
    verify_ctx c = {qd, kd, vd, kp, vp, NULL, L, Ld, Hq, Hkv, d, scale, rows, o, lse, dmask,
                    NULL, NULL, NULL};
    run_rows(verify_row, &c, nrows, (int)L + Ld, d, nthreads);
    return 0;
}

/* ------------------------------------------------------------------ */
/* verify with an fp8 (e4m3) prefix cache and per-tensor scales         */
/* ------------------------------------------------------------------ */

/*
 * "Split-KV flash-decode attention for EAGLE target-verify", implementation
 * item 1 and the entry's signature: stage 1 reads the cached prefix and
 * applies the fp8 scales k_scale / v_scale.  Reading: a cached key is
 * k_scale * e4m3(byte), a cached value is v_scale * e4m3(byte); draft keys
 * and values are not scaled.
 *
 * e4m3 (the "E4M3FN" variant): 1 sign bit, 4 exponent bits with bias 7,
 * 3 mantissa bits; exponent field 0 holds subnormals m/8 * 2^-6; the codes
 * S.1111.111 are NaN; there is no infinity.
 */
static double decode_e4m3(uint8_t b) {
    int sgn = b >> 7, e = (b >> 3) & 15, m = b & 7;
    if (e == 15 && m == 7) return NAN;
#if ORACLE_MUTANT == 10
    double v = e == 0 ? ldexp(m / 8.0, -6) : ldexp(1.0 + m / 8.0, e - 8); /* planted: bias 8 */
#else
    double v = e == 0 ? ldexp(m / 8.0, -6) : ldexp(1.0 + m / 8.0, e - 7);
#endif
    return sgn ? -v : v;
}

int oracle_decode_e4m3(const uint8_t *in, double *out, int64_t n) {
    for (int64_t i = 0; i < n; ++i) out[i] = decode_e4m3(in[i]);
    return 0;
}

typedef struct {
    const float *qd, *kd, *vd;
    const uint8_t *kc, *vc;
    const int64_t *indptr;
    int Ld, Hq, Hkv, d;
    double scale, kscale, vscale;
    const int32_t *rows;
    double *o, *lse;
    const int32_t *kv_indices; /* NULL, or prefix position t is cache row kv_indices[t] */
} verify8_ctx;

static void verify8_row(void *p, int r, double *z, const float **vr, double *o) {
    verify8_ctx *c = (verify8_ctx *)p;
    (void)vr;
    int row = c->rows[r]; /* row = b * Ld + j */
    int b = row / c->Ld, j = row % c->Ld;
    int64_t p0 = c->indptr[b], p1 = c->indptr[b + 1];
    for (int h = 0; h < c->Hq; ++h) {
        int kvh = kv_head_of(h, c->Hq, c->Hkv);
        const float *qrow = c->qd + ((size_t)row * c->Hq + h) * c->d;
        int n = 0;
        for (int64_t t = p0; t < p1; ++t) { /* the whole cached prefix, scaled keys */
#if ORACLE_MUTANT == 7
            int64_t slot = t;  /* planted: the page table is ignored */
#else
            int64_t slot = c->kv_indices ? c->kv_indices[t] : t;
#endif
            const uint8_t *krow = c->kc + ((size_t)slot * c->Hkv + kvh) * c->d;
            double sdot = 0.0;
            for (int e = 0; e < c->d; ++e) sdot += (double)qrow[e] * decode_e4m3(krow[e]);
            z[n++] = apply_scale(c->kscale * sdot, c->scale);
        }
        for (int i = 0; i <= j; ++i) {     /* drafts 0..j, unscaled */
            const float *krow = c->kd + (((size_t)b * c->Ld + i) * c->Hkv + kvh) * c->d;
            z[n++] = apply_scale(dot(qrow, krow, c->d), c->scale);
        }
        double m = -INFINITY, l = 0.0;
        for (int i = 0; i < n; ++i) if (z[i] > m) m = z[i];
        for (int i = 0; i < n; ++i) l += exp(z[i] - m);
        for (int e = 0; e < c->d; ++e) o[e] = 0.0;
        n = 0;
        for (int64_t t = p0; t < p1; ++t) {
            double w = exp(z[n++] - m) / l;
            int64_t slot = c->kv_indices ? c->kv_indices[t] : t;
            const uint8_t *vrow = c->vc + ((size_t)slot * c->Hkv + kvh) * c->d;
#if ORACLE_MUTANT == 11
            for (int e = 0; e < c->d; ++e) o[e] += w * decode_e4m3(vrow[e]); /* planted: no v_scale */
#else
            for (int e = 0; e < c->d; ++e) o[e] += w * c->vscale * decode_e4m3(vrow[e]);
#endif
        }
        for (int i = 0; i <= j; ++i) {
            double w = exp(z[n++] - m) / l;
            const float *vrow = c->vd + (((size_t)b * c->Ld + i) * c->Hkv + kvh) * c->d;
            for (int e = 0; e < c->d; ++e) o[e] += w * (double)vrow[e];
        }
        memcpy(c->o + ((size_t)r * c->Hq + h) * c->d, o, sizeof(double) * (size_t)c->d);
        c->lse[(size_t)r * c->Hq + h] = m + log(l);
    }
}

/* As oracle_verify, with k_cache / v_cache holding e4m3 bytes that stand
 * for k_scale * e4m3 and v_scale * e4m3. */
int oracle_verify_fp8(const float *qd, const float *kd, const float *vd,
                      const uint8_t *kc, const uint8_t *vc, double kscale, double vscale,
                      const int64_t *indptr, int B, int Ld, int Hq, int Hkv, int d,
                      double scale, const int32_t *rows, int nrows, double *o, double *lse,
                      int nthreads) {
    if (Hkv <= 0 || Hq % Hkv != 0 || d <= 0 || B < 0 || Ld <= 0) return -1;
    int64_t maxlen = 0;
    for (int b = 0; b < B; ++b)
        if (indptr[b + 1] - indptr[b] > maxlen) maxlen = indptr[b + 1] - indptr[b];
    verify8_ctx c = {qd, kd, vd, kc, vc, indptr, Ld, Hq, Hkv, d, scale, kscale, vscale,
                     rows, o, lse, NULL};
    run_rows(verify8_row, &c, nrows, (int)maxlen + Ld, d, nthreads);
    return 0;
}

/* As oracle_verify_fp8 with the prefix read through a page table of one
 * token per page ("Split-KV flash-decode attention for EAGLE target-verify",
 * the verify entry's kv_indptr / kv_indices): prefix position t of the flat
 * indptr range is cache row kv_indices[t]. */
int oracle_verify_fp8_paged(const float *qd, const float *kd, const float *vd,
                            const uint8_t *kc, const uint8_t *vc, double kscale, double vscale,
                            const int64_t *indptr, const int32_t *kv_indices, int B, int Ld,
                            int Hq, int Hkv, int d, double scale, const int32_t *rows,
                            int nrows, double *o, double *lse, int nthreads) {
    if (Hkv <= 0 || Hq % Hkv != 0 || d <= 0 || B < 0 || Ld <= 0 || !kv_indices) return -1;
    int64_t maxlen = 0;
    for (int b = 0; b < B; ++b)
        if (indptr[b + 1] - indptr[b] > maxlen) maxlen = indptr[b + 1] - indptr[b];
    verify8_ctx c = {qd, kd, vd, kc, vc, indptr, Ld, Hq, Hkv, d, scale, kscale, vscale,
                     rows, o, lse, kv_indices};
    run_rows(verify8_row, &c, nrows, (int)maxlen + Ld, d, nthreads);
    return 0;
}

/* ------------------------------------------------------------------ */
/* shared-latent sparse attention over per-query index lists            */
/* ------------------------------------------------------------------ */

typedef struct {
    const float *q, *lat;
    const int32_t *idx;
    int H, dl, topk;
    double scale;
    const int32_t *rows;
    double *o, *lse;
} sparse_ctx;

static void sparse_row(void *p, int r, double *z, const float **vr, double *o) {
    sparse_ctx *c = (sparse_ctx *)p;
    int t = c->rows[r];
    const int32_t *list = c->idx + (size_t)t * c->topk;
    for (int h = 0; h < c->H; ++h) {
        const float *qrow = c->q + ((size_t)t * c->H + h) * c->dl;
        int n = 0;
        for (int i = 0; i < c->topk; ++i) {
            int32_t kj = list[i];
#if ORACLE_MUTANT == 12
            if (kj <= 0) continue;       /* planted: latent row 0 is taken for a pad */
#else
            if (kj < 0) continue;        /* -1 pads a short list */
#endif
            const float *lrow = c->lat + (size_t)kj * c->dl; /* K = V = latent */
            z[n] = apply_scale(dot(qrow, lrow, c->dl), c->scale);
            vr[n] = lrow;
            ++n;
        }
        double l = softmax_row(z, vr, n, c->dl, o);
        memcpy(c->o + ((size_t)r * c->H + h) * c->dl, o, sizeof(double) * (size_t)c->dl);
        c->lse[(size_t)r * c->H + h] = l;
    }
}

/* q [T, H, dl]; latent [Tk, dl]; idx [T, topk] (-1 = pad).  An entry
 * outside [-1, Tk) names no latent row: the call is refused (returns -2)
 * before anything is read through it, as is a requested row outside [0, T). */
int oracle_sparse_latent(const float *q, const float *lat, const int32_t *idx,
                         int T, int Tk, int H, int dl, int topk, double scale,
                         const int32_t *rows, int nrows, double *o, double *lse,
                         int nthreads) {
    if (T < 0 || Tk < 0 || H <= 0 || dl <= 0 || topk < 0 || nrows < 0) return -1;
    for (int r = 0; r < nrows; ++r) {
        if (rows[r] < 0 || rows[r] >= T) return -2;
        const int32_t *list = idx + (size_t)rows[r] * topk;
        for (int i = 0; i < topk; ++i)
            if (list[i] < -1 || list[i] >= Tk) return -2;
    }
    sparse_ctx c = {q, lat, idx, H, dl, topk, scale, rows, o, lse};
    run_rows(sparse_row, &c, nrows, topk, dl, nthreads);
    return 0;
}
