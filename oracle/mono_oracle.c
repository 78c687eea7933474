/*
 * mono_oracle.c -- the oracle: a plain, slow, single-threaded CPU statement of
 * the Monodratic mixer forward pass (learned product-hash routing followed by
 * exact causal softmax over the selected token set).
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path may link, load or
 * call this file: only the test-suite, the smoke check and the benchmark's
 * CPU-baseline leg use it.  It shares no code, header, table or constant
 * generator with the CUDA library.
 *
 * Sources (page title, section):
 *   [P1] "Monodratic Routes Sparse Attention with Learned Product Hashes"
 *        (setupai.cc), Key Points.
 *   [P2] aitechinspire.com Monodratic article, "Snapshot: key facts from the
 *        report" and "What's the core idea?".
 *   [P4] "Monodratic 声称学习式路由可让稀疏因果注意力更具选择性" (remio.ai, zh),
 *        section "Monodratic 将稀疏注意力转化为检索决策".
 *   [P5] the German translation of [P4] (remio.ai, de), section
 *        "Monodratic macht aus Sparse Attention eine Abrufentscheidung".
 *
 * Arithmetic:
 *   - Values (projections, RoPE, attention, output projection) are computed
 *     in fp64 from the stored inputs upcast exactly.
 *   - Every floating-point quantity that decides an integer (block summary,
 *     codeword scores, grid scores, rerank scores) is computed in fp32 in the
 *     plain order this library specifies: sums in ascending index order, dot
 *     products as a chain of fused multiply-adds starting from +0.0f in
 *     ascending element order, except the rerank score <q, kbar_j>, which is
 *     eight such chains over the eight contiguous runs of the vector added as
 *     a balanced tree (dot_tree8).  Build with -ffp-contract=off so that no
 *     other contraction happens.
 *   - A second statement of the routing (orc_summary_assign64,
 *     orc_route_queries64) takes the same decisions in fp64 from the stored
 *     Q, K and codebooks: the plain-precision reference against which the
 *     fp32 decisions are measured (they may differ only where an fp64 margin
 *     is within fp32 rounding of zero).
 *
 * Every function returns 0 on success and a negative value on bad arguments.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

typedef struct {
    int B, S, W, H, d;
    int Bs, L, R, E, M, C, T, cap;
    double theta;
} orc_cfg;

static int cfg_ok(const orc_cfg *c)
{
    if (!c) return 0;
    if (c->B < 0 || c->S < 0 || c->W < 1 || c->H < 1 || c->d < 2 || (c->d & 1)) return 0;
    if (c->Bs < 1 || c->S % c->Bs) return 0;
    if (c->L < 1 || c->R < 0 || c->E < c->R || c->M < 1 || c->C < 1 || c->T < 1 || c->cap < 1) return 0;
    if (c->d % c->M) return 0;
    if (c->M > 16) return 0;
    long a = 1;
    for (int m = 0; m < c->M; ++m) { a *= c->C; if (a > (1L << 26)) return 0; }
    return 1;
}

static long n_addr(const orc_cfg *c)
{
    long a = 1;
    for (int m = 0; m < c->M; ++m) a *= c->C;
    return a;
}

/* ------------------------------------------------------------------------ */
/* Q/K/V projection followed by RoPE ([P2] Snapshot: "After RoPE, source     */
/* blocks are assigned ..."; [P4]/[P5] RoPE rotates query and key before     */
/* scores are formed).  Linear maps without bias, weights in the              */
/* [out_features, in_features] layout: q[t, n] = sum_k x[t, k] * Wq[n, k].   */
/* RoPE pairs are interleaved (2i, 2i+1), angle = t * theta^(-2i/d), t the    */
/* 0-based position; (a, b) -> (a cos - b sin, a sin + b cos).               */
/* rows: optional list of flat token indices b*S + t (NULL = every token);   */
/* outputs are [nrows, H, d] in that case, else [B, H, S, d].                */
/* ------------------------------------------------------------------------ */
static void rope_pair(double *a, double *b, long t, int i, int d, double theta)
{
    double inv_freq = pow(theta, -(2.0 * (double)i) / (double)d);
    double ang = (double)t * inv_freq;
    double c = cos(ang), s = sin(ang);
    double x0 = *a, x1 = *b;
    *a = x0 * c - x1 * s;
    *b = x0 * s + x1 * c;
}

int orc_project(const orc_cfg *c, const double *x, const double *Wq, const double *Wk,
                const double *Wv, long nrows, const int64_t *rows,
                double *Q, double *K, double *V)
{
    if (!cfg_ok(c) || !x || !Wq || !Wk || !Wv) return -1;
    const int W = c->W, H = c->H, d = c->d, S = c->S;
    const long total = (long)c->B * S;
    const long n = rows ? nrows : total;
    const double *Wm[3] = {Wq, Wk, Wv};
    double *Out[3] = {Q, K, V};
    for (long r = 0; r < n; ++r) {
        long flat = rows ? (long)rows[r] : r;
        if (flat < 0 || flat >= total) return -2;
        long b = flat / S, t = flat % S;
        const double *xr = x + flat * W;
        for (int which = 0; which < 3; ++which) {
            if (!Out[which]) continue;
            for (int h = 0; h < H; ++h) {
                double *dst = rows ? Out[which] + ((r * H + h) * (long)d)
                                   : Out[which] + (((b * H + h) * (long)S + t) * d);
                for (int i = 0; i < d; ++i) {
                    const double *wr = Wm[which] + (long)(h * d + i) * W;
                    double acc = 0.0;
                    for (int k = 0; k < W; ++k) acc += xr[k] * wr[k];
                    dst[i] = acc;
                }
                if (which < 2)
                    for (int i = 0; i < d / 2; ++i) rope_pair(&dst[2 * i], &dst[2 * i + 1], t, i, d, c->theta);
            }
        }
    }
    return 0;
}

/* ------------------------------------------------------------------------ */
/* Block summary and product address ([P2] "source blocks are assigned to    */
/* bounded causal posting lists"; [P4]/[P5] each product address combines   */
/* the decisions of several learned code components).                        */
/* kbar[j] = (sum of the Bs post-RoPE keys of block j, fp32, ascending t)/Bs.*/
/* Subspace m = dims [m*d/M, (m+1)*d/M).  Code c_m = argmax_c <kbar_m, cw>   */
/* (fp32 fma chain), ties -> lowest c.  addr = sum_m c_m * C^(M-1-m).        */
/* margin = min over m of (best - second best) fp32 score (C>1, else +inf). */
/* K [B,H,S,d] fp32, cb [H,M,C,d/M] fp32, kbar [B,H,nb,d], addr [B,H,nb].    */
/* ------------------------------------------------------------------------ */
static float dot_fma(const float *a, const float *b, int n)
{
    float acc = 0.0f;
    for (int i = 0; i < n; ++i) acc = fmaf(a[i], b[i], acc);
    return acc;
}

/* The rerank score's order: run l = elements [l*n/8, (l+1)*n/8) (integer     */
/* division) as an fma chain from +0.0f (dot_fma), then the eight run values */
/* added as ((c0 + c1) + (c2 + c3)) + ((c4 + c5) + (c6 + c7)) in fp32.      */
static float dot_tree8(const float *a, const float *b, int n)
{
    float c[8];
    for (int l = 0; l < 8; ++l) {
        const int lo = (int)((long)l * n / 8), hi = (int)((long)(l + 1) * n / 8);
        c[l] = dot_fma(a + lo, b + lo, hi - lo);
    }
    return ((c[0] + c[1]) + (c[2] + c[3])) + ((c[4] + c[5]) + (c[6] + c[7]));
}

int orc_summary_assign(const orc_cfg *c, const float *K, const float *cb,
                       float *kbar, int32_t *addr, float *margin)
{
    if (!cfg_ok(c) || !K || !cb || !kbar || !addr) return -1;
    const int S = c->S, d = c->d, Bs = c->Bs, M = c->M, C = c->C, dm = d / M;
    const int nb = S / Bs;
    for (long bh = 0; bh < (long)c->B * c->H; ++bh) {
        const int h = (int)(bh % c->H);
        for (int j = 0; j < nb; ++j) {
            float *kb = kbar + (bh * nb + j) * d;
            for (int i = 0; i < d; ++i) {
                float acc = 0.0f;
                for (int t = j * Bs; t < (j + 1) * Bs; ++t) acc = acc + K[(bh * S + t) * d + i];
                kb[i] = acc / (float)Bs;
            }
            long a = 0;
            float mg = INFINITY;
            for (int m = 0; m < M; ++m) {
                const float *cwm = cb + ((long)(h * M + m) * C) * dm;
                int best_c = 0;
                float best = dot_fma(kb + m * dm, cwm, dm);
                float second = -INFINITY;
                for (int cc = 1; cc < C; ++cc) {
                    float s = dot_fma(kb + m * dm, cwm + (long)cc * dm, dm);
                    if (s > best) { second = best; best = s; best_c = cc; }
                    else if (s > second) second = s;
                }
                if (C > 1 && best - second < mg) mg = best - second;
                a = a * C + best_c;
            }
            addr[bh * nb + j] = (int32_t)a;
            if (margin) margin[bh * nb + j] = mg;
        }
    }
    return 0;
}

/* ------------------------------------------------------------------------ */
/* Bounded causal posting lists ([P2] Snapshot; [P4]/[P5] strict capacity;   */
/* overflow may drop or redirect -- this library drops and counts).          */
/* Scanning blocks j = 0..nb-1 in order, block j is appended to the list of  */
/* addr[j] if that list holds fewer than cap blocks, else dropped and the    */
/* (b,h) overflow counter is incremented.                                    */
/* Export in canonical form: ids sorted by (addr, j); sorted_addr the        */
/* address of each entry; rank the entry's position among blocks of its      */
/* address (kept <=> rank < cap).                                            */
/* ------------------------------------------------------------------------ */
typedef struct { int32_t a, j; } aj_pair;

static int cmp_aj(const void *x, const void *y)
{
    const aj_pair *p = (const aj_pair *)x, *q = (const aj_pair *)y;
    if (p->a != q->a) return p->a < q->a ? -1 : 1;
    return (p->j > q->j) - (p->j < q->j);
}

int orc_posting(const orc_cfg *c, const int32_t *addr, int32_t *ids, int32_t *sorted_addr,
                int32_t *rank, int64_t *overflow)
{
    if (!cfg_ok(c) || !addr) return -1;
    const int nb = c->S / c->Bs;
    const long A = n_addr(c);
    aj_pair *tmp = (aj_pair *)malloc(sizeof(aj_pair) * (nb > 0 ? nb : 1));
    int32_t *len = (int32_t *)calloc((size_t)A, sizeof(int32_t));
    if (!tmp || !len) { free(tmp); free(len); return -3; }
    for (long bh = 0; bh < (long)c->B * c->H; ++bh) {
        const int32_t *ad = addr + bh * nb;
        int64_t ov = 0;
        memset(len, 0, sizeof(int32_t) * (size_t)A);
        for (int j = 0; j < nb; ++j) {
            if (ad[j] < 0 || ad[j] >= A) { free(tmp); free(len); return -2; }
            if (len[ad[j]] < c->cap) len[ad[j]]++;
            else ov++;
        }
        if (overflow) overflow[bh] = ov;
        for (int j = 0; j < nb; ++j) { tmp[j].a = ad[j]; tmp[j].j = j; }
        qsort(tmp, (size_t)nb, sizeof(aj_pair), cmp_aj);
        for (int k = 0; k < nb; ++k) {
            if (ids) ids[bh * nb + k] = tmp[k].j;
            if (sorted_addr) sorted_addr[bh * nb + k] = tmp[k].a;
            if (rank) rank[bh * nb + k] = (k > 0 && tmp[k - 1].a == tmp[k].a) ? rank[bh * nb + k - 1] + 1 : 0;
        }
    }
    free(tmp);
    free(len);
    return 0;
}

/* ------------------------------------------------------------------------ */
/* Bounded causal posting lists with redirect-on-overflow ([P4]/[P5]: a     */
/* strict capacity bounds each list, and overflow handling may drop or      */
/* redirect blocks; the pages give no redirect rule).  This library's        */
/* reading: scanning blocks j = 0..nb-1 in order, block j goes to the list  */
/* of its own address if that list holds fewer than cap blocks, else to the */
/* first list with room among the next addresses in mixed-radix order,      */
/* addr+1, addr+2, ... (mod C^M); only when every list is full is it        */
/* dropped, and the (b,h) overflow counter incremented.  The lists stay     */
/* causal: block j's placement depends on blocks 0..j only.                 */
/* list_addr[j] = the address of the list holding block j, or -1 (dropped). */
/* Export in canonical form as orc_posting, over the list addresses: ids    */
/* sorted by (list address, j), the dropped blocks last under the address   */
/* C^M (outside the grid); rank = position within the list address.         */
/* ------------------------------------------------------------------------ */
int orc_posting_redirect(const orc_cfg *c, const int32_t *addr, int32_t *list_addr, int32_t *ids,
                         int32_t *sorted_addr, int32_t *rank, int64_t *overflow)
{
    if (!cfg_ok(c) || !addr || !list_addr) return -1;
    const int nb = c->S / c->Bs;
    const long A = n_addr(c);
    aj_pair *tmp = (aj_pair *)malloc(sizeof(aj_pair) * (nb > 0 ? nb : 1));
    int32_t *len = (int32_t *)calloc((size_t)A, sizeof(int32_t));
    if (!tmp || !len) { free(tmp); free(len); return -3; }
    for (long bh = 0; bh < (long)c->B * c->H; ++bh) {
        const int32_t *ad = addr + bh * nb;
        int32_t *la = list_addr + bh * nb;
        int64_t ov = 0;
        memset(len, 0, sizeof(int32_t) * (size_t)A);
        for (int j = 0; j < nb; ++j) {
            if (ad[j] < 0 || ad[j] >= A) { free(tmp); free(len); return -2; }
            la[j] = -1;
            for (long step = 0; step < A; ++step) {
                const long a = (ad[j] + step) % A;
                if (len[a] < c->cap) { len[a]++; la[j] = (int32_t)a; break; }
            }
            if (la[j] < 0) ov++;
        }
        if (overflow) overflow[bh] = ov;
        for (int j = 0; j < nb; ++j) { tmp[j].a = la[j] >= 0 ? la[j] : (int32_t)A; tmp[j].j = j; }
        qsort(tmp, (size_t)nb, sizeof(aj_pair), cmp_aj);
        for (int k = 0; k < nb; ++k) {
            if (ids) ids[bh * nb + k] = tmp[k].j;
            if (sorted_addr) sorted_addr[bh * nb + k] = tmp[k].a;
            if (rank) rank[bh * nb + k] = (k > 0 && tmp[k - 1].a == tmp[k].a) ? rank[bh * nb + k - 1] + 1 : 0;
        }
    }
    free(tmp);
    free(len);
    return 0;
}

/* ------------------------------------------------------------------------ */
/* Per-query routing ([P2] Snapshot: each query probes product addresses,    */
/* reranks returned candidates and selects a fixed number of remote source   */
/* blocks; [P1] Key Points: two remote blocks out of five eligible;          */
/* [P4]/[P5] no source block may become visible to an earlier query).        */
/*  1. s_m[c] = <q_m, cw[h,m,c]> (fp32 fma chain).                            */
/*  2. grid score g(a) = s_0[c_0] + s_1[c_1] + ... (fp32, ascending m),       */
/*     every one of the C^M addresses scored; order (g desc, a asc); the     */
/*     first T are the probes.                                               */
/*  3. walk the probes in rank order, each kept list in ascending block id;  */
/*     keep block j iff j <= bq - L (bq = t / Bs); stop after E candidates.  */
/*  4. rerank score <q, kbar_j> (fp32, dot_tree8); order (score desc, j asc);*/
/*     keep the first R; optional forced block (see below); emit ascending, */
/*     pad with -1.                                                          */
/* Forced block ([P1] Key Points, forcing the labelled target under the      */
/* same maximum R budget): f = forced[b,h,t] >= 0 and eligible (f <= bq-L):  */
/* if f is not selected it is appended when fewer than R blocks are          */
/* selected, else it replaces the lowest-ranked selected block; with R = 0   */
/* nothing is selected.  An ineligible forced id is ignored and counted.     */
/* Lists are rebuilt here from addr by the plain append-if-room scan; addr  */
/* holds each block's list address, -1 for a block that no list holds.     */
/* qidx: optional flat query-head indices ((b*H+h)*S + t), NULL = all.       */
/* Outputs per listed query: sel [n,R], ncand [n] (eligible candidates       */
/* after the E cap), probe_margin [n] = g(T-th) - g((T+1)-th) (or +inf),     */
/* rerank_margin [n] = score(R-th) - score((R+1)-th) over the candidates     */
/* (+inf if ncand <= R or R = 0).  forced_ignored: count (may be NULL).      */
/* ------------------------------------------------------------------------ */
typedef struct { float g; int32_t a; } ga_pair;

static int cmp_ga(const void *x, const void *y)
{
    const ga_pair *p = (const ga_pair *)x, *q = (const ga_pair *)y;
    if (p->g != q->g) return p->g > q->g ? -1 : 1;
    return (p->a > q->a) - (p->a < q->a);
}

/* The first k entries of v[0..n) under the order cmp, in that order: one scan
 * that keeps the best k seen so far sorted by insertion.  The order is total
 * (ties on the score go to the lower index), so this is exactly the first k
 * of the fully sorted array.  Returns min(k, n). */
static int first_k(const void *v, long n, int k, size_t size, int (*cmp)(const void *, const void *), void *best)
{
    int got = 0;
    char *b = (char *)best;
    for (long i = 0; i < n; ++i) {
        const char *e = (const char *)v + (size_t)i * size;
        if (got == k && cmp(e, b + (size_t)(k - 1) * size) >= 0) continue;
        int pos = got < k ? got++ : k - 1;
        while (pos > 0 && cmp(e, b + (size_t)(pos - 1) * size) < 0) {
            memcpy(b + (size_t)pos * size, b + (size_t)(pos - 1) * size, size);
            --pos;
        }
        memcpy(b + (size_t)pos * size, e, size);
    }
    return got;
}

int orc_route_queries(const orc_cfg *c, const float *Q, const float *kbar, const float *cb,
                      const int32_t *addr, const int32_t *forced, long nq, const int64_t *qidx,
                      int32_t *sel, int32_t *ncand, float *probe_margin, float *rerank_margin,
                      int64_t *forced_ignored)
{
    if (!cfg_ok(c) || !Q || !kbar || !cb || !addr || !sel) return -1;
    const int S = c->S, H = c->H, d = c->d, Bs = c->Bs, M = c->M, C = c->C, dm = d / M;
    const int nb = S / Bs, T = c->T, R = c->R, E = c->E, L = c->L, cap = c->cap;
    const long A = n_addr(c);
    if (T > A) return -1;
    const long total = (long)c->B * H * S;
    const long n = qidx ? nq : total;

    float *s = (float *)malloc(sizeof(float) * (size_t)M * C);
    ga_pair *grid = (ga_pair *)malloc(sizeof(ga_pair) * (size_t)A);
    ga_pair *top = (ga_pair *)malloc(sizeof(ga_pair) * (size_t)(T + 1));
    int32_t *list = (int32_t *)malloc(sizeof(int32_t) * (size_t)A * cap);
    int32_t *len = (int32_t *)malloc(sizeof(int32_t) * (size_t)A);
    int32_t *cand = (int32_t *)malloc(sizeof(int32_t) * (size_t)(E > 0 ? E : 1));
    ga_pair *rr = (ga_pair *)malloc(sizeof(ga_pair) * (size_t)(E > 0 ? E : 1));
    if (!s || !grid || !top || !list || !len || !cand || !rr) {
        free(s); free(grid); free(top); free(list); free(len); free(cand); free(rr);
        return -3;
    }
    long cur_bh = -1;
    int64_t ignored = 0;
    for (long qi = 0; qi < n; ++qi) {
        long flat = qidx ? (long)qidx[qi] : qi;
        if (flat < 0 || flat >= total) { ignored = -1; break; }
        long bh = flat / S;
        int t = (int)(flat % S), h = (int)(bh % H);
        if (bh != cur_bh) {
            /* rebuild the bounded lists of this (b, h) */
            memset(len, 0, sizeof(int32_t) * (size_t)A);
            for (int j = 0; j < nb; ++j) {
                int32_t a = addr[bh * nb + j];
                if (a < 0) continue;  /* a block that no list holds (redirect mode: dropped) */
                if (len[a] < cap) list[(long)a * cap + len[a]++] = j;
            }
            cur_bh = bh;
        }
        const float *q = Q + flat * d;
        const int bq = t / Bs;
        /* 1. subspace scores */
        for (int m = 0; m < M; ++m)
            for (int cc = 0; cc < C; ++cc)
                s[m * C + cc] = dot_fma(q + m * dm, cb + ((long)(h * M + m) * C + cc) * dm, dm);
        /* 2. score every address of the product grid, rank, take T */
        for (long a = 0; a < A; ++a) {
            long rem = a;
            int code[16];
            for (int m = M - 1; m >= 0; --m) { code[m] = (int)(rem % C); rem /= C; }
            float g = s[0 * C + code[0]];
            for (int m = 1; m < M; ++m) g = g + s[m * C + code[m]];
            grid[a].g = g;
            grid[a].a = (int32_t)a;
        }
        first_k(grid, A, T + 1, sizeof(ga_pair), cmp_ga, top);   /* = grid sorted, first T+1 */
        if (probe_margin) probe_margin[qi] = (T < A) ? top[T - 1].g - top[T].g : INFINITY;
        /* 3. union of the probed lists, causal filter, E cap */
        int nc = 0;
        for (int r = 0; r < T && nc < E; ++r) {
            int32_t a = top[r].a;
            for (int k = 0; k < len[a] && nc < E; ++k) {
                int32_t j = list[(long)a * cap + k];
                if (j <= bq - L) cand[nc++] = j;
            }
        }
        if (ncand) ncand[qi] = nc;
        /* 4. rerank */
        for (int k = 0; k < nc; ++k) {
            rr[k].g = dot_tree8(q, kbar + (bh * nb + cand[k]) * (long)d, d);
            rr[k].a = cand[k];
        }
        qsort(rr, (size_t)nc, sizeof(ga_pair), cmp_ga);
        if (rerank_margin) rerank_margin[qi] = (R > 0 && nc > R) ? rr[R - 1].g - rr[R].g : INFINITY;
        int ns = nc < R ? nc : R;
        int32_t chosen[64];
        if (R > 64) { ignored = -1; break; }
        for (int k = 0; k < ns; ++k) chosen[k] = rr[k].a;
        if (forced && R > 0) {
            int32_t f = forced[flat];
            if (f >= 0) {
                if (f <= bq - L) {
                    int present = 0;
                    for (int k = 0; k < ns; ++k) present |= (chosen[k] == f);
                    if (!present) {
                        if (ns < R) chosen[ns++] = f;
                        else chosen[R - 1] = f;
                    }
                } else {
                    ignored++;
                }
            }
        }
        /* ascending id, pad -1 */
        for (int x = 1; x < ns; ++x)
            for (int y = x; y > 0 && chosen[y - 1] > chosen[y]; --y) {
                int32_t tmp = chosen[y]; chosen[y] = chosen[y - 1]; chosen[y - 1] = tmp;
            }
        for (int k = 0; k < R; ++k) sel[qi * R + k] = k < ns ? chosen[k] : -1;
    }
    free(s); free(grid); free(top); free(list); free(len); free(cand); free(rr);
    if (ignored < 0) return -2;
    if (forced_ignored) *forced_ignored = ignored;
    return 0;
}

/* ------------------------------------------------------------------------ */
/* Exact causal softmax over the selected token set ([P2] Snapshot: exact    */
/* causal softmax over the selected tokens; [P4]/[P5] the attention is not   */
/* approximated once candidates are chosen).                                 */
/* Sel(t) = tokens of the remote blocks in sel[t] plus the local tokens      */
/* s in [max(0, bq-L+1)*Bs, t].  o_t = sum_s softmax_s(<q_t,k_s>/sqrt(d)) v_s */
/* in fp64 (max-subtracted exp).  Q, K, V [B,H,S,d] fp64, sel [B,H,S,R].    */
/* O: [n, d] for the listed query-heads (qidx) or [B,H,S,d] for all.        */
/* ------------------------------------------------------------------------ */
int orc_attend(const orc_cfg *c, const double *Q, const double *K, const double *V,
               const int32_t *sel, long nq, const int64_t *qidx, double *O)
{
    if (!cfg_ok(c) || !Q || !K || !V || !sel || !O) return -1;
    const int S = c->S, H = c->H, d = c->d, Bs = c->Bs, R = c->R, L = c->L;
    const long total = (long)c->B * H * S;
    const long n = qidx ? nq : total;
    const long maxkeys = (long)R * Bs + (long)L * Bs;
    int32_t *keys = (int32_t *)malloc(sizeof(int32_t) * (size_t)(maxkeys > 0 ? maxkeys : 1));
    double *sc = (double *)malloc(sizeof(double) * (size_t)(maxkeys > 0 ? maxkeys : 1));
    if (!keys || !sc) { free(keys); free(sc); return -3; }
    const double scale = 1.0 / sqrt((double)d);
    for (long qi = 0; qi < n; ++qi) {
        long flat = qidx ? (long)qidx[qi] : qi;
        if (flat < 0 || flat >= total) { free(keys); free(sc); return -2; }
        long bh = flat / S;
        int t = (int)(flat % S), bq = t / Bs;
        int nk = 0;
        for (int r = 0; r < R; ++r) {
            int32_t j = sel[flat * R + r];
            if (j < 0) continue;
            if (j > bq - L) { free(keys); free(sc); return -4; } /* not a remote block */
            for (int u = 0; u < Bs; ++u) keys[nk++] = j * Bs + u;
        }
        int lo = bq - L + 1;
        if (lo < 0) lo = 0;
        for (int u = lo * Bs; u <= t; ++u) keys[nk++] = u;
        const double *q = Q + flat * d;
        double mx = -INFINITY;
        for (int k = 0; k < nk; ++k) {
            const double *kr = K + (bh * S + keys[k]) * d;
            double acc = 0.0;
            for (int i = 0; i < d; ++i) acc += q[i] * kr[i];
            sc[k] = acc * scale;
            if (sc[k] > mx) mx = sc[k];
        }
        double l = 0.0;
        for (int k = 0; k < nk; ++k) { sc[k] = exp(sc[k] - mx); l += sc[k]; }
        double *o = O + qi * d;
        for (int i = 0; i < d; ++i) o[i] = 0.0;
        for (int k = 0; k < nk; ++k) {
            const double *vr = V + (bh * S + keys[k]) * d;
            for (int i = 0; i < d; ++i) o[i] += sc[k] * vr[i];
        }
        for (int i = 0; i < d; ++i) o[i] /= l;
    }
    free(keys);
    free(sc);
    return 0;
}

/* ------------------------------------------------------------------------ */
/* Output projection: delta[t, n] = sum_k O[t, k] * Wo[n, k], fp64.          */
/* ([P2] Snapshot: the mixer maps [batch, sequence, width] to an attention   */
/* delta; the host adds the residual.)  O [B,S,H*d], Wo [W, H*d].            */
/* rows: optional flat token list (b*S+t); delta [nrows, W] or [B,S,W].     */
/* ------------------------------------------------------------------------ */
int orc_out_project(const orc_cfg *c, const double *O, const double *Wo, long nrows,
                    const int64_t *rows, double *delta)
{
    if (!cfg_ok(c) || !O || !Wo || !delta) return -1;
    const int W = c->W, HD = c->H * c->d;
    const long total = (long)c->B * c->S;
    const long n = rows ? nrows : total;
    for (long r = 0; r < n; ++r) {
        long flat = rows ? (long)rows[r] : r;
        if (flat < 0 || flat >= total) return -2;
        const double *orow = O + flat * HD;
        for (int o = 0; o < W; ++o) {
            const double *wr = Wo + (long)o * HD;
            double acc = 0.0;
            for (int k = 0; k < HD; ++k) acc += orow[k] * wr[k];
            delta[r * W + o] = acc;
        }
    }
    return 0;
}


/* ------------------------------------------------------------------------ */
/* Routing in fp64: the same steps as orc_summary_assign and                */
/* orc_route_queries ([P2] Snapshot; [P4]/[P5] product addresses, strict     */
/* capacity, causality), with every score, sum and mean in double precision */
/* on the stored inputs upcast exactly.  The plain reading of the method:    */
/* the decision each step names, taken on the real-valued scores as closely */
/* as fp64 allows, with the same tie rules (lowest code, lowest address,     */
/* lowest block id).  Margins are reported so that a caller can tell which  */
/* decisions fp32 rounding could flip.                                       */
/*                                                                            */
/* orc_summary_assign64: kbar[j] = (sum of the block's keys) / Bs in fp64;   */
/* code c_m = argmax_c <kbar_m, cw[h,m,c]>; margin = min over m of          */
/* best - second best (+inf when C = 1).                                     */
/* ------------------------------------------------------------------------ */
static double dot64(const double *a, const double *b, int n)
{
    double acc = 0.0;
    for (int i = 0; i < n; ++i) acc += a[i] * b[i];
    return acc;
}

int orc_summary_assign64(const orc_cfg *c, const double *K, const double *cb,
                         double *kbar, int32_t *addr, double *margin)
{
    if (!cfg_ok(c) || !K || !cb || !kbar || !addr) return -1;
    const int S = c->S, d = c->d, Bs = c->Bs, M = c->M, C = c->C, dm = d / M;
    const int nb = S / Bs;
    for (long bh = 0; bh < (long)c->B * c->H; ++bh) {
        const int h = (int)(bh % c->H);
        for (int j = 0; j < nb; ++j) {
            double *kb = kbar + (bh * nb + j) * d;
            for (int i = 0; i < d; ++i) {
                double acc = 0.0;
                for (int t = j * Bs; t < (j + 1) * Bs; ++t) acc += K[(bh * S + t) * d + i];
                kb[i] = acc / (double)Bs;
            }
            long a = 0;
            double mg = INFINITY;
            for (int m = 0; m < M; ++m) {
                const double *cwm = cb + ((long)(h * M + m) * C) * dm;
                int best_c = 0;
                double best = dot64(kb + m * dm, cwm, dm);
                double second = -INFINITY;
                for (int cc = 1; cc < C; ++cc) {
                    double sc = dot64(kb + m * dm, cwm + (long)cc * dm, dm);
                    if (sc > best) { second = best; best = sc; best_c = cc; }
                    else if (sc > second) second = sc;
                }
                if (C > 1 && best - second < mg) mg = best - second;
                a = a * C + best_c;
            }
            addr[bh * nb + j] = (int32_t)a;
            if (margin) margin[bh * nb + j] = mg;
        }
    }
    return 0;
}

/* orc_route_queries64: per query-head, subspace scores and the grid score   */
/* of every address in fp64; probes = the first T under (g desc, a asc);     */
/* union in probe order over the kept lists (rebuilt from addr), causal      */
/* filter j <= bq - L, E cap; rerank <q, kbar_j> in fp64 under (score desc,  */
/* j asc), first R; forced block as in orc_route_queries; ascending, -1 pad. */
/* probe_margin[n] = the smallest gap between neighbours among grid ranks    */
/* 1..T+1 (the probe set and its order, which the E cap reads);              */
/* rerank_margin[n] = the smallest gap between neighbours among rerank       */
/* ranks 1..R+1 of the candidates (+inf where there is no such pair).        */
typedef struct { double g; int32_t a; } ga64_pair;

static int cmp_ga64(const void *x, const void *y)
{
    const ga64_pair *p = (const ga64_pair *)x, *q = (const ga64_pair *)y;
    if (p->g != q->g) return p->g > q->g ? -1 : 1;
    return (p->a > q->a) - (p->a < q->a);
}

static double min_gap(const ga64_pair *v, int n)
{
    double mg = INFINITY;
    for (int k = 0; k + 1 < n; ++k)
        if (v[k].g - v[k + 1].g < mg) mg = v[k].g - v[k + 1].g;
    return mg;
}

int orc_route_queries64(const orc_cfg *c, const double *Q, const double *kbar, const double *cb,
                        const int32_t *addr, const int32_t *forced, long nq, const int64_t *qidx,
                        int32_t *sel, int32_t *ncand, double *probe_margin, double *rerank_margin,
                        int64_t *forced_ignored)
{
    if (!cfg_ok(c) || !Q || !kbar || !cb || !addr || !sel) return -1;
    const int S = c->S, H = c->H, d = c->d, Bs = c->Bs, M = c->M, C = c->C, dm = d / M;
    const int nb = S / Bs, T = c->T, R = c->R, E = c->E, L = c->L, cap = c->cap;
    const long A = n_addr(c);
    if (T > A || R > 64) return -1;
    const long total = (long)c->B * H * S;
    const long n = qidx ? nq : total;

    double *s = (double *)malloc(sizeof(double) * (size_t)M * C);
    ga64_pair *grid = (ga64_pair *)malloc(sizeof(ga64_pair) * (size_t)A);
    ga64_pair *top = (ga64_pair *)malloc(sizeof(ga64_pair) * (size_t)(T + 1));
    int32_t *list = (int32_t *)malloc(sizeof(int32_t) * (size_t)A * cap);
    int32_t *len = (int32_t *)malloc(sizeof(int32_t) * (size_t)A);
    int32_t *cand = (int32_t *)malloc(sizeof(int32_t) * (size_t)(E > 0 ? E : 1));
    ga64_pair *rr = (ga64_pair *)malloc(sizeof(ga64_pair) * (size_t)(E > 0 ? E : 1));
    if (!s || !grid || !top || !list || !len || !cand || !rr) {
        free(s); free(grid); free(top); free(list); free(len); free(cand); free(rr);
        return -3;
    }
    long cur_bh = -1;
    int64_t ignored = 0;
    int bad = 0;
    for (long qi = 0; qi < n; ++qi) {
        long flat = qidx ? (long)qidx[qi] : qi;
        if (flat < 0 || flat >= total) { bad = 1; break; }
        long bh = flat / S;
        int t = (int)(flat % S), h = (int)(bh % H);
        if (bh != cur_bh) {
            memset(len, 0, sizeof(int32_t) * (size_t)A);
            for (int j = 0; j < nb; ++j) {
                int32_t a = addr[bh * nb + j];
                if (a < 0) continue;  /* a block that no list holds (redirect mode: dropped) */
                if (a >= A) { bad = 1; break; }
                if (len[a] < cap) list[(long)a * cap + len[a]++] = j;
            }
            if (bad) break;
            cur_bh = bh;
        }
        const double *q = Q + flat * d;
        const int bq = t / Bs;
        for (int m = 0; m < M; ++m)
            for (int cc = 0; cc < C; ++cc)
                s[m * C + cc] = dot64(q + m * dm, cb + ((long)(h * M + m) * C + cc) * dm, dm);
        for (long a = 0; a < A; ++a) {
            long rem = a;
            int code[16];
            for (int m = M - 1; m >= 0; --m) { code[m] = (int)(rem % C); rem /= C; }
            double g = 0.0;
            for (int m = 0; m < M; ++m) g += s[m * C + code[m]];
            grid[a].g = g;
            grid[a].a = (int32_t)a;
        }
        const int ntop = first_k(grid, A, T + 1, sizeof(ga64_pair), cmp_ga64, top);  /* = sorted, first T+1 */
        if (probe_margin) probe_margin[qi] = min_gap(top, ntop);
        int nc = 0;
        for (int r = 0; r < T && nc < E; ++r) {
            int32_t a = top[r].a;
            for (int k = 0; k < len[a] && nc < E; ++k) {
                int32_t j = list[(long)a * cap + k];
                if (j <= bq - L) cand[nc++] = j;
            }
        }
        if (ncand) ncand[qi] = nc;
        for (int k = 0; k < nc; ++k) {
            rr[k].g = dot64(q, kbar + (bh * nb + cand[k]) * (long)d, d);
            rr[k].a = cand[k];
        }
        qsort(rr, (size_t)nc, sizeof(ga64_pair), cmp_ga64);
        if (rerank_margin) rerank_margin[qi] = R > 0 ? min_gap(rr, nc < R + 1 ? nc : R + 1) : INFINITY;
        int ns = nc < R ? nc : R;
        int32_t chosen[64];
        for (int k = 0; k < ns; ++k) chosen[k] = rr[k].a;
        if (forced && R > 0) {
            int32_t f = forced[flat];
            if (f >= 0) {
                if (f <= bq - L) {
                    int present = 0;
                    for (int k = 0; k < ns; ++k) present |= (chosen[k] == f);
                    if (!present) {
                        if (ns < R) chosen[ns++] = f;
                        else chosen[R - 1] = f;
                    }
                } else {
                    ignored++;
                }
            }
        }
        for (int x = 1; x < ns; ++x)
            for (int y = x; y > 0 && chosen[y - 1] > chosen[y]; --y) {
                int32_t tmp = chosen[y]; chosen[y] = chosen[y - 1]; chosen[y - 1] = tmp;
            }
        for (int k = 0; k < R; ++k) sel[qi * R + k] = k < ns ? chosen[k] : -1;
    }
    free(s); free(grid); free(top); free(list); free(len); free(cand); free(rr);
    if (bad) return -2;
    if (forced_ignored) *forced_ignored = ignored;
    return 0;
}
