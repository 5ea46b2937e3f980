/*
 * sas_oracle.c -- plain fp64 CPU oracle for SAS gated block-sparse attention.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path may link, load or call
 * this file: only the tests, the smoke check and the benchmark's CPU-baseline leg
 * use it.  It shares no code, header, table or helper with the CUDA library.
 *
 * Every function below writes out a definition from the reviews of SAS ("SAS: Simple
 * Attention Sparsification via End-to-End Optimization of Context Ranking"):
 *   - block partition, C = n/b blocks (jaehun.me review, Background, Eq. 3 text);
 *   - gate g = softmax(s) over the history blocks, log g_m = s_m - LSE(s)
 *     (jaehun.me review, section 4.2.2 "Gate activation"; shibing624 review,
 *     method section under the SAS equation);
 *   - hard Top-K of s, plus the always-kept current block B_0 with gate 1
 *     (jaehun.me review, Eq. 4 text and walkthrough Steps 3-4);
 *   - o = softmax(q K_S^T + log g_S) V_S (shibing624 review, SAS equation;
 *     jaehun.me review, Eq. 9);
 *   - the backward of that expression by the chain rule, with the log-gate
 *     gradient of a block equal to the sum of the logit gradients of its tokens
 *     (jaehun.me review, Kernel implementation paragraph) and carried to s
 *     through log g = s - LSE(s);
 *   - the inference rule I = Top-K(s, K) with no gate (jaehun.me review,
 *     walkthrough Step 6);
 *   - the ablated gates: log sigmoid(s) and raw logits inside the softmax, the
 *     outer gate weighting the values, and the hard STE gate (jaehun.me review,
 *     "Why the Four Design Choices Matter", Eq. 5 and Eq. 7; shibing624 review,
 *     Fig. 2);
 *   - a weight-free pooled-key scorer: mean-pooled query and key block summaries
 *     and their scaled dot product (jaehun.me review, walkthrough Step 1 and
 *     Limitations: pooling-based block summaries).
 * Readings where the reviews are silent:
 *   softmax scale sigma (default 1/sqrt(d)); one score row per (kv head, query
 *   block) shared by the query heads of a GQA group; 0-based blocks, history of
 *   query block c is m < c, current block causally masked token by token; ties in
 *   Top-K go to the lower block index (-0.0 == +0.0); selected lists ascending,
 *   padded with -1; ds = dlogg - g * sum(dlogg) over the history blocks; the
 *   backward may read o as a bf16 tensor stores it (o_store); the STE passes
 *   dL/dh straight through to g; the scorer pools by plain means.
 *
 * Everything is computed in double.  Inputs may be given as double, float or
 * bfloat16 bits; they are widened exactly on load.  Parallelism (OpenMP) only
 * splits independent output units; each unit's arithmetic is the plain loop.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

enum { ORC_F64 = 0, ORC_F32 = 1, ORC_BF16 = 2 };

enum {
    ORC_OK = 0,
    ORC_ERR_ARG = 1,
    ORC_ERR_MISSING_ROW_STATS = 2,
    ORC_ERR_NOMEM = 3
};

/* widen one element of an input tensor to double (exact for all three types) */
static double ld(const void* p, int dt, size_t i) {
    if (dt == ORC_F64) return ((const double*)p)[i];
    if (dt == ORC_F32) return (double)((const float*)p)[i];
    uint32_t u = ((uint32_t)((const uint16_t*)p)[i]) << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

/* x rounded to the nearest bfloat16 value (8 significant bits, ties to even),
 * kept as a double: the value a bf16 tensor holds after storing x.  Exponents
 * below bf16's normal range keep its subnormal spacing of 2^-133. */
static double round_bf16(double x) {
    if (x == 0.0 || !isfinite(x)) return x;
    int e;
    frexp(x, &e); /* |x| = f 2^e, f in [0.5, 1) */
    int sh = e - 8;
    if (sh < -133) sh = -133;
    return ldexp(nearbyint(ldexp(x, -sh)), sh);
}

int oracle_num_threads(void) {
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

/* ------------------------------------------------------------------------- */
/* Gate and Top-K selection for one score row.                               */
/* ------------------------------------------------------------------------- */

/* LSE over the c history scores of a row: the log of the softmax denominator,
 * so that log g_m = s_m - LSE (jaehun.me review, section 4.2.2). Empty row: -inf. */
static double row_lse(const double* s, int c) {
    if (c <= 0) return -INFINITY;
    double mx = s[0];
    for (int m = 1; m < c; ++m)
        if (s[m] > mx) mx = s[m];
    double acc = 0.0;
    for (int m = 0; m < c; ++m) acc += exp(s[m] - mx);
    return mx + log(acc);
}

typedef struct {
    double v;
    int m;
} scored_t;

/* larger score first; equal scores: lower block index first */
static int cmp_desc(const void* a, const void* b) {
    const scored_t* x = (const scored_t*)a;
    const scored_t* y = (const scored_t*)b;
    if (x->v > y->v) return -1;
    if (x->v < y->v) return 1;
    return (x->m < y->m) ? -1 : (x->m > y->m);
}

static int cmp_int(const void* a, const void* b) {
    int x = *(const int*)a, y = *(const int*)b;
    return (x > y) - (x < y);
}

/* The hard Top-K of Eq. 3 (jaehun.me review, Background; walkthrough Step 3):
 * the min(K, c) highest-scoring history blocks.  Full scope (shibing624 review,
 * Fig. 2(d)) keeps every history block.  Writes the chosen blocks ascending and
 * returns their count. */
static int select_row(const double* s, int c, int K, int full_scope, int* out) {
    if (c <= 0) return 0;
    if (full_scope || K >= c) {
        for (int m = 0; m < c; ++m) out[m] = m;
        return c;
    }
    if (K <= 0) return 0;
    scored_t* buf = (scored_t*)malloc(sizeof(scored_t) * (size_t)c);
    if (!buf) return -1;
    for (int m = 0; m < c; ++m) {
        buf[m].v = s[m];
        buf[m].m = m;
    }
    qsort(buf, (size_t)c, sizeof(scored_t), cmp_desc);
    for (int r = 0; r < K; ++r) out[r] = buf[r].m;
    free(buf);
    qsort(out, (size_t)K, sizeof(int), cmp_int);
    return K;
}

/* Selection over many rows.  Row r has ncand[r] candidates (the first ncand[r]
 * entries of its score row, stride row_stride).  idx gets idx_cols entries per
 * row: the chosen blocks ascending, then -1.  lse (nullable) gets the row LSE. */
int oracle_select(const void* s, int s_dt, long nrows, long row_stride, const int* ncand,
                  int top_k, int full_scope, int* idx, int idx_cols, double* lse) {
    if (!s || !ncand || nrows < 0 || row_stride <= 0 || top_k < 0 || !idx || idx_cols < 0)
        return ORC_ERR_ARG;
    int err = ORC_OK;
#pragma omp parallel for schedule(dynamic, 16)
    for (long r = 0; r < nrows; ++r) {
        int c = ncand[r];
        if (c > row_stride) c = (int)row_stride;
        double* row = (double*)malloc(sizeof(double) * (size_t)(c > 0 ? c : 1));
        int* sel = (int*)malloc(sizeof(int) * (size_t)(c > 0 ? c : 1));
        if (!row || !sel) {
            free(row);
            free(sel);
            err = ORC_ERR_NOMEM;
            continue;
        }
        for (int m = 0; m < c; ++m) row[m] = ld(s, s_dt, (size_t)r * (size_t)row_stride + (size_t)m);
        int cnt = select_row(row, c, top_k, full_scope, sel);
        for (int k = 0; k < idx_cols; ++k) idx[r * (long)idx_cols + k] = (k < cnt) ? sel[k] : -1;
        if (lse) lse[r] = row_lse(row, c);
        free(row);
        free(sel);
    }
    return err;
}

/* ------------------------------------------------------------------------- */
/* Training-shape gated attention (forward and backward).                    */
/* ------------------------------------------------------------------------- */

/* Problem description.  Layouts (row-major, last index fastest):
 *   q, o, dO, dq : [B, n, Hq, d]      k, v, dk, dv : [B, n, Hkv, d]
 *   s, ds        : [B, Hkv, Cq, Cq]   with Cq = n / bs; row c uses entries m < c
 *   lse          : [B, Hq, n]         natural log, including the gate bias */
typedef struct {
    int B, Hq, Hkv, d, n, bs, top_k;
    int full_scope; /* 1: every history block is attended (gated) */
    int gate;       /* 0: plain block-sparse attention (no bias);
                       1: log g = s - LSE(s) (softmax gate, the method);
                       2: log g = log sigmoid(s); 3: log g = s (raw logit) -- the
                       gate-activation variants SAS ablates (jaehun.me review,
                       "Why the Four Design Choices Matter", gate activation);
                       4: outer gate, o = sum_j g_{m(j)} p_j v_j with p the gate-free
                       softmax (gate placement, section 4.2.2 Eq. 5);
                       5: hard STE gate, the forward a plain hard Top-K and the
                       backward straight through to g (ranking preservation,
                       section 4.2.2 Eq. 7).  4 and 5 use g = softmax(s). */
    double sigma;   /* softmax scale applied to q.k */
} orc_desc;

/* Per (b, h, c) gate quantities: the attended history blocks and log g over them. */
typedef struct {
    int cnt;      /* number of attended history blocks */
    int* blocks;  /* [cnt], ascending */
    double* logg; /* [c] log g_m for every history block m < c */
    double* g;    /* [c] g_m */
    double lse_s; /* LSE of the row */
} gate_row_t;

static void gate_row_free(gate_row_t* r) {
    free(r->blocks);
    free(r->logg);
    free(r->g);
    r->blocks = NULL;
    r->logg = NULL;
    r->g = NULL;
}

static int gate_row_make(const orc_desc* D, const void* s, int s_dt, int b, int h, int c, gate_row_t* out) {
    int Cq = D->n / D->bs;
    size_t base = (((size_t)b * D->Hkv + h) * Cq + c) * (size_t)Cq;
    int cc = c > 0 ? c : 1;
    double* row = (double*)malloc(sizeof(double) * cc);
    out->blocks = (int*)malloc(sizeof(int) * cc);
    out->logg = (double*)malloc(sizeof(double) * cc);
    out->g = (double*)malloc(sizeof(double) * cc);
    if (!row || !out->blocks || !out->logg || !out->g) {
        free(row);
        gate_row_free(out);
        return ORC_ERR_NOMEM;
    }
    row[0] = 0.0;
    for (int m = 0; m < c; ++m) row[m] = ld(s, s_dt, base + (size_t)m);
    out->lse_s = row_lse(row, c);
    for (int m = 0; m < c; ++m) {
        double lg;
        if (D->gate == 2)
            lg = row[m] >= 0.0 ? -log1p(exp(-row[m])) : row[m] - log1p(exp(row[m])); /* log sigmoid(s_m) */
        else if (D->gate == 3)
            lg = row[m];                                                             /* raw logit */
        else
            lg = row[m] - out->lse_s;                                                /* s_m - LSE(s) */
        out->logg[m] = lg;
        out->g[m] = exp(lg);
    }
    out->cnt = select_row(row, c, D->top_k, D->full_scope, out->blocks);
    free(row);
    return out->cnt < 0 ? ORC_ERR_NOMEM : ORC_OK;
}

/* Does the gate enter the logits (inner gate, Eq. 9)?  Not for the outer gate,
 * which weights the values, nor for the hard STE gate, whose forward value is 1. */
static int gate_in_logits(const orc_desc* D) { return D->gate >= 1 && D->gate <= 3; }

/* The logits of query row i (block c) of head hq against its attended keys
 * (Eq. 9): z_j = sigma q_i.k_j + log g_{m(j)} for tokens of selected history
 * blocks, z_j = sigma q_i.k_j for tokens j <= i of the current block.
 * Fills keys[], z[] and wv[], the weight of each key's value in o (g_{m(j)} for
 * history keys under the outer gate, else 1); returns the number of keys. */
static int row_logits(const orc_desc* D, const void* q, const void* k, int dt, int b, int hq, int i,
                      const gate_row_t* gr, int* keys, double* z, double* biasv, double* wv) {
    int G = D->Hq / D->Hkv, h = hq / G, c = i / D->bs, d = D->d;
    size_t qoff = (((size_t)b * D->n + i) * D->Hq + hq) * (size_t)d;
    int nk = 0;
    for (int t = 0; t < gr->cnt; ++t) {
        int m = gr->blocks[t];
        double bias = gate_in_logits(D) ? gr->logg[m] : 0.0;
        double w = D->gate == 4 ? gr->g[m] : 1.0;
        for (int j = m * D->bs; j < (m + 1) * D->bs; ++j) {
            keys[nk] = j;
            biasv[nk] = bias;
            wv[nk] = w;
            ++nk;
        }
    }
    for (int j = c * D->bs; j <= i; ++j) {
        keys[nk] = j;
        biasv[nk] = 0.0; /* current block: gate 1, bias log 1 = 0 */
        wv[nk] = 1.0;
        ++nk;
    }
    for (int t = 0; t < nk; ++t) {
        size_t koff = (((size_t)b * D->n + keys[t]) * D->Hkv + h) * (size_t)d;
        double dot = 0.0;
        for (int e = 0; e < d; ++e) dot += ld(q, dt, qoff + e) * ld(k, dt, koff + e);
        z[t] = D->sigma * dot + biasv[t];
    }
    return nk;
}

static double lse_of(const double* z, int nk) {
    double mx = z[0];
    for (int t = 1; t < nk; ++t)
        if (z[t] > mx) mx = z[t];
    double acc = 0.0;
    for (int t = 0; t < nk; ++t) acc += exp(z[t] - mx);
    return mx + log(acc);
}

static int max_keys(const orc_desc* D) {
    int Cq = D->n / D->bs;
    int hist = D->full_scope ? Cq : (D->top_k < Cq ? D->top_k : Cq);
    return (hist + 1) * D->bs;
}

static int check_desc(const orc_desc* D) {
    if (!D || D->B <= 0 || D->Hq <= 0 || D->Hkv <= 0 || D->d <= 0 || D->n <= 0 || D->bs <= 0) return 0;
    if (D->Hq % D->Hkv || D->n % D->bs || D->top_k < 0) return 0;
    return 1;
}

/* Forward over the query blocks whose (b, h, c) entry of qmask is non-zero
 * (NULL: all).  o: [B,n,Hq,d], lse: [B,Hq,n]. */
int oracle_attn_fwd(const orc_desc* D, const void* q, const void* k, const void* v, int dt, const void* s,
                    int s_dt, const unsigned char* qmask, double* o, double* lse) {
    if (!check_desc(D) || !q || !k || !v || !s || !o || !lse) return ORC_ERR_ARG;
    int Cq = D->n / D->bs, G = D->Hq / D->Hkv, d = D->d, MK = max_keys(D);
    long units = (long)D->B * D->Hkv * Cq;
    int err = ORC_OK;
#pragma omp parallel for schedule(dynamic, 1)
    for (long u = 0; u < units; ++u) {
        if (qmask && !qmask[u]) continue;
        int c = (int)(u % Cq), h = (int)((u / Cq) % D->Hkv), b = (int)(u / ((long)Cq * D->Hkv));
        gate_row_t gr;
        int* keys = (int*)malloc(sizeof(int) * MK);
        double* z = (double*)malloc(sizeof(double) * MK);
        double* bv = (double*)malloc(sizeof(double) * MK);
        double* wv = (double*)malloc(sizeof(double) * MK);
        if (!keys || !z || !bv || !wv || gate_row_make(D, s, s_dt, b, h, c, &gr) != ORC_OK) {
            free(keys);
            free(z);
            free(bv);
            free(wv);
            err = ORC_ERR_NOMEM;
            continue;
        }
        for (int g = 0; g < G; ++g) {
            int hq = h * G + g;
            for (int i = c * D->bs; i < (c + 1) * D->bs; ++i) {
                int nk = row_logits(D, q, k, dt, b, hq, i, &gr, keys, z, bv, wv);
                double L = lse_of(z, nk);
                size_t ooff = (((size_t)b * D->n + i) * D->Hq + hq) * (size_t)d;
                for (int e = 0; e < d; ++e) o[ooff + e] = 0.0;
                for (int t = 0; t < nk; ++t) {
                    double p = exp(z[t] - L);
                    size_t voff = (((size_t)b * D->n + keys[t]) * D->Hkv + h) * (size_t)d;
                    for (int e = 0; e < d; ++e) o[ooff + e] += p * wv[t] * ld(v, dt, voff + e);
                }
                lse[((size_t)b * D->Hq + hq) * D->n + i] = L;
            }
        }
        gate_row_free(&gr);
        free(keys);
        free(z);
        free(bv);
        free(wv);
    }
    return err;
}

/* Backward of L = sum(dO * o) through Eq. 9.
 *   D_i   = dO_i . o_i   (o_i as the forward stored it: rounded to bf16 when
 *                         o_store == 1, the exact value when o_store == 0)
 *   dS_ij = p_ij (dO_i . v_j - D_i)           (gradient of the logit z_ij)
 *   dq_i  = sigma sum_j dS_ij k_j
 *   dk_j  = sigma sum_{hq in group, i} dS_ij q_i,   dv_j = sum p_ij dO_i
 *   dlogg[b,h,c,m] = sum over the group's heads, rows i of block c and tokens j
 *                    of block m of dS_ij   (block-wise log-gate gradient)
 *   ds[b,h,c,m] = dlogg_m - g_m sum_{m' < c} dlogg_{m'}  for m < c, else 0
 *                 (chain rule through log g_m = s_m - LSE(s)).
 * Gate variants: sigmoid / raw change log g and its chain rule.  The outer gate
 * weights v_j by w_j = g_{m(j)}: dS_ij = p_ij (w_j dO_i.v_j - D_i), dv_j gets
 * w_j p_ij dO_i, and dlogg_m = g_m sum_{i, j in m} p_ij dO_i.v_j.  The hard STE
 * gate is plain block-sparse attention forward; its dlogg_m is g_m times
 * sum_{i, j in m} exp(z_ij - lse_i) (dO_i.v_j - D_i) over every history block,
 * dropped ones included.
 * Phase 1 runs per query block (b, h, c) selected by qmask and yields dq, ds,
 * dlogg and each row's lse and D.  Phase 2 runs per key block (b, h, m) selected
 * by kvmask and yields dk, dv; every query block that attends a requested key
 * block must be in qmask (else ORC_ERR_MISSING_ROW_STATS).
 * dlogg (nullable): [B,Hkv,Cq,Cq] like ds.  Outputs outside the masks are 0. */
int oracle_attn_bwd(const orc_desc* D, const void* q, const void* k, const void* v, const void* dO, int dt,
                    const void* s, int s_dt, const unsigned char* qmask, const unsigned char* kvmask, int o_store,
                    double* o, double* lse, double* dq, double* dk, double* dv, double* ds, double* dlogg) {
    if (!check_desc(D) || !q || !k || !v || !dO || !s || !o || !lse || !dq || !dk || !dv || !ds) return ORC_ERR_ARG;
    int Cq = D->n / D->bs, G = D->Hq / D->Hkv, d = D->d, MK = max_keys(D);
    long units = (long)D->B * D->Hkv * Cq;
    size_t nq = (size_t)D->B * D->n * D->Hq * d, nkv = (size_t)D->B * D->n * D->Hkv * d;
    memset(dq, 0, nq * sizeof(double));
    memset(dk, 0, nkv * sizeof(double));
    memset(dv, 0, nkv * sizeof(double));
    memset(o, 0, nq * sizeof(double));
    memset(ds, 0, (size_t)units * Cq * sizeof(double));
    if (dlogg) memset(dlogg, 0, (size_t)units * Cq * sizeof(double));
    size_t nrows = (size_t)D->B * D->Hq * D->n;
    double* Drow = (double*)malloc(nrows * sizeof(double));
    double* logg_all = (double*)malloc((size_t)units * Cq * sizeof(double)); /* logit bias of block m in row c */
    double* w_all = (double*)malloc((size_t)units * Cq * sizeof(double));    /* value weight (outer gate) */
    int* sel_all = (int*)calloc((size_t)units * Cq, sizeof(int)); /* 1 if history block m is attended by c */
    unsigned char* have = (unsigned char*)calloc((size_t)units, 1);
    if (!Drow || !logg_all || !w_all || !sel_all || !have) {
        free(Drow);
        free(w_all);
        free(logg_all);
        free(sel_all);
        free(have);
        return ORC_ERR_NOMEM;
    }
    for (size_t r = 0; r < nrows; ++r) lse[r] = NAN;
    int err = ORC_OK;

    /* phase 0: the gate and the selection of every query block (needed by phase 2 even
     * for query blocks outside qmask, to know which of them attend a key block) */
#pragma omp parallel for schedule(dynamic, 4)
    for (long u = 0; u < units; ++u) {
        int c = (int)(u % Cq), h = (int)((u / Cq) % D->Hkv), b = (int)(u / ((long)Cq * D->Hkv));
        gate_row_t gr;
        if (gate_row_make(D, s, s_dt, b, h, c, &gr) != ORC_OK) {
            err = ORC_ERR_NOMEM;
            continue;
        }
        for (int m = 0; m < Cq; ++m) {
            logg_all[u * Cq + m] = (m < c && gate_in_logits(D)) ? gr.logg[m] : 0.0;
            w_all[u * Cq + m] = (m < c && D->gate == 4) ? gr.g[m] : 1.0;
        }
        for (int t = 0; t < gr.cnt; ++t) sel_all[u * Cq + gr.blocks[t]] = 1;
        gate_row_free(&gr);
    }
    if (err != ORC_OK) goto done;

    /* phase 1: per query block */
#pragma omp parallel for schedule(dynamic, 1)
    for (long u = 0; u < units; ++u) {
        if (qmask && !qmask[u]) continue;
        int c = (int)(u % Cq), h = (int)((u / Cq) % D->Hkv), b = (int)(u / ((long)Cq * D->Hkv));
        gate_row_t gr;
        int* keys = (int*)malloc(sizeof(int) * MK);
        double* z = (double*)malloc(sizeof(double) * MK);
        double* bv = (double*)malloc(sizeof(double) * MK);
        double* wv = (double*)malloc(sizeof(double) * MK);
        double* dlg = (double*)calloc((size_t)Cq, sizeof(double));
        unsigned char* selm = (unsigned char*)calloc((size_t)Cq, 1);
        if (!keys || !z || !bv || !wv || !dlg || !selm || gate_row_make(D, s, s_dt, b, h, c, &gr) != ORC_OK) {
            free(keys);
            free(z);
            free(bv);
            free(wv);
            free(dlg);
            free(selm);
            err = ORC_ERR_NOMEM;
            continue;
        }
        for (int t = 0; t < gr.cnt; ++t) selm[gr.blocks[t]] = 1;
        for (int g = 0; g < G; ++g) {
            int hq = h * G + g;
            for (int i = c * D->bs; i < (c + 1) * D->bs; ++i) {
                int nk = row_logits(D, q, k, dt, b, hq, i, &gr, keys, z, bv, wv);
                double L = lse_of(z, nk);
                size_t ooff = (((size_t)b * D->n + i) * D->Hq + hq) * (size_t)d;
                for (int t = 0; t < nk; ++t) {
                    double p = exp(z[t] - L);
                    size_t voff = (((size_t)b * D->n + keys[t]) * D->Hkv + h) * (size_t)d;
                    for (int e = 0; e < d; ++e) o[ooff + e] += p * wv[t] * ld(v, dt, voff + e);
                }
                double Di = 0.0;
                for (int e = 0; e < d; ++e)
                    Di += ld(dO, dt, ooff + e) * (o_store == 1 ? round_bf16(o[ooff + e]) : o[ooff + e]);
                size_t rix = ((size_t)b * D->Hq + hq) * D->n + i;
                lse[rix] = L;
                Drow[rix] = Di;
                for (int t = 0; t < nk; ++t) {
                    double p = exp(z[t] - L);
                    size_t kvoff = (((size_t)b * D->n + keys[t]) * D->Hkv + h) * (size_t)d;
                    double dp = 0.0;
                    for (int e = 0; e < d; ++e) dp += ld(dO, dt, ooff + e) * ld(v, dt, kvoff + e);
                    /* o = sum_j w_j p_j v_j: dz_j = p_j (w_j dp_j - D) */
                    double dS = p * (wv[t] * dp - Di);
                    for (int e = 0; e < d; ++e) dq[ooff + e] += D->sigma * dS * ld(k, dt, kvoff + e);
                    int m = keys[t] / D->bs;
                    if (m == c) continue;
                    /* history token: its block's log-gate gradient; the outer gate's
                       dg_m = sum p_j dp_j (Eq. 5), times g_m for the log */
                    dlg[m] += D->gate == 4 ? wv[t] * p * dp : dS;
                }
                if (D->gate == 5) {
                    /* hard STE: dropped blocks get d h_m = sum_j exp(z_j - LSE_S) do.(v_j - o)
                       with z_j = sigma q.k_j, normalised by the selected set's LSE (Eq. 7) */
                    for (int m = 0; m < c; ++m) {
                        if (selm[m]) continue;
                        for (int j = m * D->bs; j < (m + 1) * D->bs; ++j) {
                            size_t kvoff = (((size_t)b * D->n + j) * D->Hkv + h) * (size_t)d;
                            double dot = 0.0, dp = 0.0;
                            for (int e = 0; e < d; ++e) {
                                dot += ld(q, dt, ooff + e) * ld(k, dt, kvoff + e);
                                dp += ld(dO, dt, ooff + e) * ld(v, dt, kvoff + e);
                            }
                            dlg[m] += exp(D->sigma * dot - L) * (dp - Di);
                        }
                    }
                }
            }
        }
        if (D->gate == 5) /* straight through: dL/dg = dL/dh; as a log-gate gradient, g dL/dg */
            for (int m = 0; m < c; ++m) dlg[m] *= gr.g[m];
        if (D->gate) {
            /* chain rule through log g: softmax d(log g_m)/ds_m' = [m = m'] - g_m';
               log sigmoid: [m = m'] (1 - g_m); raw logit: [m = m'].  The outer and
               STE gates use g = softmax(s) too, dlg holding g dL/dg */
            double tot = 0.0;
            for (int m = 0; m < c; ++m) tot += dlg[m];
            size_t rowoff = (size_t)u * Cq;
            for (int m = 0; m < c; ++m) {
                if (D->gate == 2)
                    ds[rowoff + m] = dlg[m] * (1.0 - gr.g[m]);
                else if (D->gate == 3)
                    ds[rowoff + m] = dlg[m];
                else
                    ds[rowoff + m] = dlg[m] - gr.g[m] * tot;
                if (dlogg) dlogg[rowoff + m] = dlg[m];
            }
        }
        have[u] = 1;
        gate_row_free(&gr);
        free(keys);
        free(z);
        free(bv);
        free(wv);
        free(dlg);
        free(selm);
    }
    if (err != ORC_OK) goto done;

    /* phase 2: per key block; gathers over every query row that attends each key */
#pragma omp parallel for schedule(dynamic, 1)
    for (long u = 0; u < units; ++u) {
        if (kvmask && !kvmask[u]) continue;
        int m = (int)(u % Cq), h = (int)((u / Cq) % D->Hkv), b = (int)(u / ((long)Cq * D->Hkv));
        long ubase = ((long)b * D->Hkv + h) * Cq;
        for (int c = m; c < Cq; ++c) {
            int attends = (c == m) || sel_all[(ubase + c) * Cq + m];
            if (!attends) continue;
            if (!have[ubase + c]) {
                err = ORC_ERR_MISSING_ROW_STATS;
                continue;
            }
            double bias = (c == m) ? 0.0 : logg_all[(ubase + c) * Cq + m];
            double w = (c == m) ? 1.0 : w_all[(ubase + c) * Cq + m];
            for (int g = 0; g < G; ++g) {
                int hq = h * G + g;
                for (int i = c * D->bs; i < (c + 1) * D->bs; ++i) {
                    size_t qoff = (((size_t)b * D->n + i) * D->Hq + hq) * (size_t)d;
                    size_t rix = ((size_t)b * D->Hq + hq) * D->n + i;
                    for (int j = m * D->bs; j < (m + 1) * D->bs; ++j) {
                        if (c == m && j > i) continue; /* causal inside the current block */
                        size_t kvoff = (((size_t)b * D->n + j) * D->Hkv + h) * (size_t)d;
                        double dot = 0.0, dp = 0.0;
                        for (int e = 0; e < d; ++e) {
                            dot += ld(q, dt, qoff + e) * ld(k, dt, kvoff + e);
                            dp += ld(dO, dt, qoff + e) * ld(v, dt, kvoff + e);
                        }
                        double p = exp(D->sigma * dot + bias - lse[rix]);
                        double dS = p * (w * dp - Drow[rix]);
                        for (int e = 0; e < d; ++e) {
                            dk[kvoff + e] += D->sigma * dS * ld(q, dt, qoff + e);
                            dv[kvoff + e] += p * w * ld(dO, dt, qoff + e);
                        }
                    }
                }
            }
        }
    }
done:
    free(Drow);
    free(w_all);
    free(logg_all);
    free(sel_all);
    free(have);
    return err;
}

/* ------------------------------------------------------------------------- */
/* Decode: one new token per sequence, gate-free hard Top-K (walkthrough Step 6) */
/* ------------------------------------------------------------------------- */

/* q: [B, Hq, d]; caches: [B, Hkv, Tmax, d]; ctx_len[b] = T, the number of
 * cached tokens including the new one, so the query sits at t = T - 1.
 * History blocks: Cb = floor(t / bs) full blocks before the current (partial)
 * block [Cb*bs, t].  s: [B, Hkv, s_cols], row (b,h) scores blocks 0..Cb-1.
 * dense != 0: attend every token 0..t (the full-attention comparator).
 * o: [B, Hq, d].  idx (nullable): [B, Hkv, top_k] chosen blocks ascending, -1 pad. */
int oracle_decode(int B, int Hq, int Hkv, int d, int bs, int Tmax, int top_k, double sigma, const void* q,
                  const void* kc, const void* vc, int dt, const int* ctx_len, const void* s, int s_dt, int s_cols,
                  int dense, double* o, int* idx) {
    if (B <= 0 || Hq <= 0 || Hkv <= 0 || Hq % Hkv || d <= 0 || bs <= 0 || Tmax <= 0 || top_k < 0 || !q || !kc ||
        !vc || !ctx_len || !o || (!dense && !s))
        return ORC_ERR_ARG;
    int G = Hq / Hkv;
    int err = ORC_OK;
#pragma omp parallel for schedule(dynamic, 1)
    for (long u = 0; u < (long)B * Hkv; ++u) {
        int b = (int)(u / Hkv), h = (int)(u % Hkv);
        int T = ctx_len[b];
        if (T <= 0 || T > Tmax) {
            err = ORC_ERR_ARG;
            continue;
        }
        int t = T - 1, Cb = t / bs;
        if (!dense && Cb > s_cols) {
            err = ORC_ERR_ARG;
            continue;
        }
        int* sel = (int*)malloc(sizeof(int) * (size_t)(Cb > 0 ? Cb : 1));
        double* row = (double*)malloc(sizeof(double) * (size_t)(Cb > 0 ? Cb : 1));
        int* keys = (int*)malloc(sizeof(int) * (size_t)T);
        double* z = (double*)malloc(sizeof(double) * (size_t)T);
        if (!sel || !row || !keys || !z) {
            free(sel);
            free(row);
            free(keys);
            free(z);
            err = ORC_ERR_NOMEM;
            continue;
        }
        int cnt;
        if (dense) {
            cnt = 0;
        } else {
            for (int m = 0; m < Cb; ++m) row[m] = ld(s, s_dt, ((size_t)b * Hkv + h) * (size_t)s_cols + m);
            cnt = select_row(row, Cb, top_k, 0, sel);
            if (idx)
                for (int r = 0; r < top_k; ++r) idx[u * (long)top_k + r] = (r < cnt) ? sel[r] : -1;
        }
        int nk = 0;
        if (dense) {
            for (int j = 0; j <= t; ++j) keys[nk++] = j;
        } else {
            for (int r = 0; r < cnt; ++r)
                for (int j = sel[r] * bs; j < (sel[r] + 1) * bs; ++j) keys[nk++] = j;
            for (int j = Cb * bs; j <= t; ++j) keys[nk++] = j;
        }
        for (int g = 0; g < G; ++g) {
            int hq = h * G + g;
            size_t qoff = ((size_t)b * Hq + hq) * (size_t)d;
            for (int r = 0; r < nk; ++r) {
                size_t koff = (((size_t)b * Hkv + h) * (size_t)Tmax + keys[r]) * (size_t)d;
                double dot = 0.0;
                for (int e = 0; e < d; ++e) dot += ld(q, dt, qoff + e) * ld(kc, dt, koff + e);
                z[r] = sigma * dot;
            }
            double L = lse_of(z, nk);
            for (int e = 0; e < d; ++e) o[qoff + e] = 0.0;
            for (int r = 0; r < nk; ++r) {
                double p = exp(z[r] - L);
                size_t voff = (((size_t)b * Hkv + h) * (size_t)Tmax + keys[r]) * (size_t)d;
                for (int e = 0; e < d; ++e) o[qoff + e] += p * ld(vc, dt, voff + e);
            }
        }
        free(sel);
        free(row);
        free(keys);
        free(z);
    }
    return err;
}

/* ------------------------------------------------------------------------- */
/* Parameter-free pooled-key scorer: block summaries by mean pooling          */
/* (jaehun.me review, walkthrough Step 1 and Limitations: the selector scores  */
/* a query against per-block key summaries, pooling-based).                   */
/* ------------------------------------------------------------------------- */

/* Training shape.  q [B,n,Hq,d], k [B,n,Hkv,d]; s [B,Hkv,Cq,Cq] out:
 *   qbar[b,h,c] = mean over the b tokens of block c and the G heads of group h of q
 *   kbar[b,h,m] = mean over the b tokens of block m of k
 *   s[b,h,c,m]  = sigma qbar[b,h,c] . kbar[b,h,m]  for m < c, 0 for m >= c. */
int oracle_pool_scores(int B, int n, int Hq, int Hkv, int d, int bs, double sigma, const void* q, const void* k,
                       int dt, double* s) {
    if (B <= 0 || n <= 0 || Hq <= 0 || Hkv <= 0 || Hq % Hkv || d <= 0 || bs <= 0 || n % bs || !q || !k || !s)
        return ORC_ERR_ARG;
    int G = Hq / Hkv, Cq = n / bs;
    int err = ORC_OK;
#pragma omp parallel for schedule(dynamic, 1)
    for (long u = 0; u < (long)B * Hkv; ++u) {
        int b = (int)(u / Hkv), h = (int)(u % Hkv);
        double* qbar = (double*)calloc((size_t)Cq * d, sizeof(double));
        double* kbar = (double*)calloc((size_t)Cq * d, sizeof(double));
        if (!qbar || !kbar) {
            free(qbar);
            free(kbar);
            err = ORC_ERR_NOMEM;
            continue;
        }
        for (int c = 0; c < Cq; ++c) {
            for (int i = c * bs; i < (c + 1) * bs; ++i) {
                for (int g = 0; g < G; ++g) {
                    size_t qoff = (((size_t)b * n + i) * Hq + h * G + g) * (size_t)d;
                    for (int e = 0; e < d; ++e) qbar[(size_t)c * d + e] += ld(q, dt, qoff + e);
                }
                size_t koff = (((size_t)b * n + i) * Hkv + h) * (size_t)d;
                for (int e = 0; e < d; ++e) kbar[(size_t)c * d + e] += ld(k, dt, koff + e);
            }
            for (int e = 0; e < d; ++e) {
                qbar[(size_t)c * d + e] /= (double)bs * G;
                kbar[(size_t)c * d + e] /= (double)bs;
            }
        }
        for (int c = 0; c < Cq; ++c)
            for (int m = 0; m < Cq; ++m) {
                double dot = 0.0;
                if (m < c)
                    for (int e = 0; e < d; ++e) dot += qbar[(size_t)c * d + e] * kbar[(size_t)m * d + e];
                s[(u * Cq + c) * (size_t)Cq + m] = m < c ? sigma * dot : 0.0;
            }
        free(qbar);
        free(kbar);
    }
    return err;
}

/* Decode shape.  Key summaries of the full blocks [m0, m1) of a cache
 * [B,Hkv,Tmax,d]: ksum[b,h,m] = mean over the block's b tokens, kept in the
 * summary array's dtype (rounded to bf16 when round_out != 0).  ksum is
 * [B,Hkv,nsum,d] doubles; blocks outside [m0, m1) are left as they are. */
int oracle_pool_keys(int B, int Hkv, int Tmax, int d, int bs, const void* kc, int dt, int m0, int m1, int nsum,
                     int round_out, double* ksum) {
    if (B <= 0 || Hkv <= 0 || Tmax <= 0 || d <= 0 || bs <= 0 || !kc || !ksum || m0 < 0 || m1 < m0 || m1 > nsum ||
        (long)m1 * bs > Tmax)
        return ORC_ERR_ARG;
#pragma omp parallel for schedule(static)
    for (long u = 0; u < (long)B * Hkv; ++u) {
        for (int m = m0; m < m1; ++m) {
            for (int e = 0; e < d; ++e) {
                double acc = 0.0;
                for (int j = m * bs; j < (m + 1) * bs; ++j) acc += ld(kc, dt, ((size_t)u * Tmax + j) * (size_t)d + e);
                acc /= (double)bs;
                ksum[((size_t)u * nsum + m) * (size_t)d + e] = round_out ? round_bf16(acc) : acc;
            }
        }
    }
    return ORC_OK;
}

/* Decode scores: q [B,Hq,d]; ksum [B,Hkv,nsum,d] doubles; ctx_len[b] = T:
 *   s[b,h,m] = sigma qbar[b,h] . ksum[b,h,m] for the Cb = floor((T-1)/b) full
 *   history blocks, 0 for m >= Cb; qbar = mean of q over the group's G heads.
 * s: [B,Hkv,s_cols], s_cols >= every Cb. */
int oracle_decode_scores(int B, int Hq, int Hkv, int d, int bs, double sigma, const void* q, int dt,
                         const double* ksum, int nsum, const int* ctx_len, int s_cols, double* s) {
    if (B <= 0 || Hq <= 0 || Hkv <= 0 || Hq % Hkv || d <= 0 || bs <= 0 || !q || !ksum || !ctx_len || !s)
        return ORC_ERR_ARG;
    int G = Hq / Hkv;
    int err = ORC_OK;
    for (long u = 0; u < (long)B * Hkv; ++u) {
        int b = (int)(u / Hkv), h = (int)(u % Hkv);
        int T = ctx_len[b];
        int Cb = T > 0 ? (T - 1) / bs : 0;
        if (T <= 0 || Cb > s_cols || Cb > nsum) {
            err = ORC_ERR_ARG;
            continue;
        }
        for (int m = 0; m < s_cols; ++m) {
            double dot = 0.0;
            if (m < Cb)
                for (int e = 0; e < d; ++e) {
                    double qb = 0.0;
                    for (int g = 0; g < G; ++g) qb += ld(q, dt, ((size_t)b * Hq + h * G + g) * (size_t)d + e);
                    dot += qb / G * ksum[((size_t)u * nsum + m) * (size_t)d + e];
                }
            s[u * (size_t)s_cols + m] = m < Cb ? sigma * dot : 0.0;
        }
    }
    return err;
}
