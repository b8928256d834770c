/*
 * rr_oracle.c -- plain, slow, CPU reference of the RouteRelay routing path.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product library links, loads or
 * calls this file; only the tests, the package smoke check and the benchmark's
 * CPU-baseline leg do.  It shares no code, header, table or constant
 * generator with the CUDA path.
 *
 * Source of every step: the page "RouteRelay: Event-Triggered Cross-Layer
 * Route Reuse for Efficient Dynamic Sparse Attention" (arXiv 2609.07306),
 * abbreviated "RouteRelay" below.  Each function names the section/equation
 * it follows.  Where the page leaves a step open, the reading taken is
 * stated at the function (the full list is kept with the design notes).
 *
 * Arithmetic: every score is an fp64 sum of fp64 products of the fp32 inputs
 * (bf16 inputs arrive already widened to fp32, which is exact).  Ranking,
 * alpha/beta and the challenge test are all done in fp64.
 *
 * Parity status: every exported function is pinned by CPU tests against
 * brute force, closed forms, invariants from the page (Lemma 1, Eq. 10) and
 * an independent Philox implementation; none is "parity unpinned".
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

/* ------------------------------------------------------------------------ */
/* Scores: RouteRelay §2.1 Eq. 1, S = Qc Kc^T (raw dot product, no 1/sqrt(d);
 * the 1/sqrt(d) of Eq. 3 belongs to attention, not to routing).            */
/* ------------------------------------------------------------------------ */
void rro_scores(const float *q, const float *k, int32_t nq, int32_t nk,
                int32_t d, double *S)
{
    for (int32_t i = 0; i < nq; ++i) {
        for (int32_t j = 0; j < nk; ++j) {
            double acc = 0.0;
            for (int32_t t = 0; t < d; ++t)
                acc += (double)q[(int64_t)i * d + t] * (double)k[(int64_t)j * d + t];
            S[(int64_t)i * nk + j] = acc;
        }
    }
}

/* Number of key chunks query row i may route to.  The causal mask (query
 * chunk i sees key chunks 0..i) belongs to the underlying router
 * (RouteRelay §4.3); non-causal rows see all nk chunks. */
int32_t rro_valid_count(int32_t i, int32_t nk, int32_t causal)
{
    if (!causal) return nk;
    return (i + 1 < nk) ? (i + 1) : nk;
}

/* ------------------------------------------------------------------------ */
/* Full route of one row: RouteRelay §2.1 Eq. 2 (TopK) and §3.1 item 1
 * (near-miss sentinels = the m chunks ranked just below the top-k cutoff).
 * Reading: ties are broken by ascending chunk index; the stored order is
 * (score descending, index ascending).  Brute force: the whole valid row is
 * sorted, no partial selection.                                            */
/* ------------------------------------------------------------------------ */
typedef struct { double s; int32_t j; } rro_pair;

static int rro_cmp_desc(const void *a, const void *b)
{
    const rro_pair *x = (const rro_pair *)a, *y = (const rro_pair *)b;
    if (x->s > y->s) return -1;
    if (x->s < y->s) return 1;
    return (x->j < y->j) ? -1 : (x->j > y->j);
}

/* route[k] and near[m] receive chunk ids (-1 where the row has fewer valid
 * chunks); *alpha receives min over the route of S (RouteRelay Eq. 6 at the
 * row's own layer), i.e. the score at rank |R|.  Returns |R|. */
int32_t rro_route_row(const double *s_row, int32_t n_valid, int32_t k,
                      int32_t m, int32_t *route, int32_t *near, double *alpha)
{
    rro_pair *v = (rro_pair *)malloc(sizeof(rro_pair) * (size_t)(n_valid > 0 ? n_valid : 1));
    for (int32_t j = 0; j < n_valid; ++j) { v[j].s = s_row[j]; v[j].j = j; }
    qsort(v, (size_t)n_valid, sizeof(rro_pair), rro_cmp_desc);
    int32_t nr = n_valid < k ? n_valid : k;
    int32_t nm = (n_valid - nr) < m ? (n_valid - nr) : m;
    for (int32_t a = 0; a < k; ++a) route[a] = a < nr ? v[a].j : -1;
    for (int32_t a = 0; a < m; ++a) near[a] = a < nm ? v[nr + a].j : -1;
    *alpha = nr > 0 ? v[nr - 1].s : INFINITY;
    free(v);
    return nr;
}

/* ------------------------------------------------------------------------ */
/* Philox4x32-10, written from Salmon, Moraes, Dror, Shaw, "Parallel Random
 * Numbers: As Easy as 1, 2, 3" (SC'11): ten rounds of the Philox S-box on a
 * 4x32-bit counter; each round multiplies words 0 and 2 by the two round
 * multipliers, mixes the high halves with words 1/3 and the key, and the key
 * is bumped by the two Weyl constants between rounds.                      */
/* ------------------------------------------------------------------------ */
#define RRO_PHILOX_M0 0xD2511F53u
#define RRO_PHILOX_M1 0xCD9E8D57u
#define RRO_PHILOX_W0 0x9E3779B9u
#define RRO_PHILOX_W1 0xBB67AE85u

void rro_philox4x32_10(const uint32_t ctr_in[4], const uint32_t key_in[2],
                       uint32_t out[4])
{
    uint32_t c0 = ctr_in[0], c1 = ctr_in[1], c2 = ctr_in[2], c3 = ctr_in[3];
    uint32_t k0 = key_in[0], k1 = key_in[1];
    for (int round = 0; round < 10; ++round) {
        if (round > 0) { k0 += RRO_PHILOX_W0; k1 += RRO_PHILOX_W1; }
        uint64_t p0 = (uint64_t)RRO_PHILOX_M0 * (uint64_t)c0;
        uint64_t p1 = (uint64_t)RRO_PHILOX_M1 * (uint64_t)c2;
        uint32_t hi0 = (uint32_t)(p0 >> 32), lo0 = (uint32_t)p0;
        uint32_t hi1 = (uint32_t)(p1 >> 32), lo1 = (uint32_t)p1;
        uint32_t n0 = hi1 ^ c1 ^ k0;
        uint32_t n1 = lo1;
        uint32_t n2 = hi0 ^ c3 ^ k1;
        uint32_t n3 = lo0;
        c0 = n0; c1 = n1; c2 = n2; c3 = n3;
    }
    out[0] = c0; out[1] = c1; out[2] = c2; out[3] = c3;
}

/* ------------------------------------------------------------------------ */
/* Random sentinels: RouteRelay §3.1 item 2 (r chunks drawn uniformly from
 * the omitted chunks) and §3.4 (drawn without replacement from the residual
 * pool outside the deterministic near-miss set).
 * Readings: pool P = valid chunks minus (route U near-miss).  If |P| <= r
 * every pool chunk is taken in ascending order (padded with -1).  Otherwise
 * draw t = 0,1,2,...: word t%4 of Philox4x32-10 with key (seed lo, seed hi)
 * and counter (bh, row, layer, t/4) maps to chunk (w * n_valid) >> 32; a
 * draw is accepted when it is not in route U near-miss U already accepted.
 * After max_draws draws, remaining slots are filled from P in ascending
 * order.  Sentinels are stored in acceptance order.  Returns the number of
 * draws consumed.                                                          */
/* ------------------------------------------------------------------------ */
static int rro_contains(const int32_t *a, int32_t n, int32_t x)
{
    for (int32_t t = 0; t < n; ++t) if (a[t] == x) return 1;
    return 0;
}

int32_t rro_random_sentinels(uint64_t seed, int32_t bh, int32_t row,
                             int32_t layer, int32_t n_valid,
                             const int32_t *excl, int32_t n_excl, int32_t r,
                             int32_t max_draws, int32_t *out)
{
    /* excl holds route U near-miss (entries of -1 are ignored) */
    int32_t n_taken = 0;
    for (int32_t t = 0; t < n_excl; ++t) if (excl[t] >= 0) ++n_taken;
    int32_t np = n_valid - n_taken;
    for (int32_t a = 0; a < r; ++a) out[a] = -1;
    if (np <= r) {
        int32_t w = 0;
        for (int32_t j = 0; j < n_valid; ++j)
            if (!rro_contains(excl, n_excl, j)) out[w++] = j;
        return 0;
    }
    uint32_t key[2] = { (uint32_t)(seed & 0xffffffffu), (uint32_t)(seed >> 32) };
    int32_t acc = 0, t = 0;
    uint32_t words[4];
    for (; acc < r && t < max_draws; ++t) {
        if ((t & 3) == 0) {
            uint32_t ctr[4] = { (uint32_t)bh, (uint32_t)row, (uint32_t)layer, (uint32_t)(t >> 2) };
            rro_philox4x32_10(ctr, key, words);
        }
        uint32_t w = words[t & 3];
        int32_t j = (int32_t)(((uint64_t)w * (uint64_t)(uint32_t)n_valid) >> 32);
        if (rro_contains(excl, n_excl, j)) continue;
        if (rro_contains(out, acc, j)) continue;
        out[acc++] = j;
    }
    for (int32_t j = 0; j < n_valid && acc < r; ++j)
        if (!rro_contains(excl, n_excl, j) && !rro_contains(out, acc, j)) out[acc++] = j;
    return t;
}

/* ------------------------------------------------------------------------ */
/* Ledger row rebuild: RouteRelay §3.1 Eq. 4, L_i = (R_i, C_i, a); the row
 * is laid out as c = k+m+r ids: route | near-miss | random.               */
/* ------------------------------------------------------------------------ */
typedef struct {
    int32_t nq, nk, d, k, m, r, causal, max_draws;
    double gamma;
    uint64_t seed;
    int32_t max_age;   /* 0: off; else a row whose ledger is max_age layers old refreshes */
    int32_t min_reuse; /* 0: off; else a row is reused for min_reuse layers after it was built */
    int32_t g_sink;    /* mandatory global sentinels: sink chunks 0..g_sink-1 */
    int32_t g_recent;  /* ... and the row's recent chunks i-g_recent+1..i */
    double gamma_h;    /* 0: off; else the larger guard margin of a refreshed row */
} rro_params;

static void rro_rebuild_row(const rro_params *p, int32_t bh, int32_t layer,
                            int32_t i, const double *s_row, int32_t *ids,
                            double *alpha)
{
    int32_t n_valid = rro_valid_count(i, p->nk, p->causal);
    const int32_t ksel = p->k + p->m, g = p->g_sink + p->g_recent;
    rro_route_row(s_row, n_valid, p->k, p->m, ids, ids + p->k, alpha);
    /* Mandatory global candidates (RouteRelay §3.1 item 3, "sink and recent
     * chunks"): the sink chunks 0..g_sink-1, then the row's recent chunks
     * i-g_recent+1..i, each kept if valid, not in route U near-miss and not
     * already listed (a recent chunk below g_sink is a sink chunk); stored in
     * that order after the random block, -1 padded. */
    int32_t *glob = ids + ksel + p->r;
    int32_t ng = 0;
    for (int32_t t = 0; t < g; ++t) {
        const int32_t j = t < p->g_sink ? t : i - p->g_recent + 1 + (t - p->g_sink);
        if (j < 0 || j >= n_valid) continue;
        if (t >= p->g_sink && j < p->g_sink) continue;
        if (rro_contains(ids, ksel, j)) continue;
        glob[ng++] = j;
    }
    for (int32_t t = ng; t < g; ++t) glob[t] = -1;
    /* random sentinels from the valid chunks outside route U near-miss U the
     * global candidates */
    int32_t *excl = (int32_t *)malloc(sizeof(int32_t) * (size_t)(ksel + g + 1));
    memcpy(excl, ids, sizeof(int32_t) * (size_t)ksel);
    memcpy(excl + ksel, glob, sizeof(int32_t) * (size_t)ng);
    rro_random_sentinels(p->seed, bh, i, layer, n_valid, excl, ksel + ng,
                         p->r, p->max_draws, ids + ksel);
    free(excl);
}

/* ------------------------------------------------------------------------ */
/* One layer of one head.
 *  anchor != 0: full routing of every row (RouteRelay §4.1, "an anchor layer
 *     constructs this state from a complete chunk-score matrix"; forced
 *     anchors, §3.2).
 *  anchor == 0: relay (RouteRelay §3.2 Eq. 5-8 and §4.1-4.2): candidate set
 *     A_i = R_i U C_i, alpha = min over R, beta = max over C, reuse iff
 *     alpha > beta + gamma_i; otherwise the row computes all its scores,
 *     replaces its route and rebuilds its sentinels (anchor_layer <- layer).
 *     Stable rows keep ids; their age advances implicitly (age = layer -
 *     anchor_layer); their stored alpha becomes this layer's alpha.
 *     gamma_i (Eq. 8, "a configurable guard margin" per row) is
 *     gamma_rows[i], or p->gamma for every row when gamma_rows is NULL.
 *     Per-row lifetime bound (reading of §3.2 "Forced anchors ... bound the
 *     lifetime of stale random sentinels", applied per row): with
 *     p->max_age > 0, a row with layer - anchor_layer >= max_age refreshes
 *     whatever the test says, so no ledger row is reused max_age or more
 *     layers after it was built.  A forced row is rescored first, like any
 *     relay row, and counted like a challenged one.
 *     Hysteresis (reading of §3.2 "a refreshed row receives a minimum reuse
 *     horizon of one layer", the horizon made configurable): with
 *     p->min_reuse = h > 0, a row built at layer a is reused without the
 *     test at layers a+1 .. a+h (ids kept, alpha stored).  The lifetime bound
 *     takes precedence where the two meet.
 *     Elevated margin (reading of the same passage, "may use a larger guard
 *     margin until its anchor margin recovers"): with p->gamma_h > 0, a row
 *     rebuilt at a relay layer is marked elevated (elevated[i] = 1; a row
 *     built at an anchor layer is not).  An elevated row's test uses
 *     max(gamma_i, gamma_h) in place of gamma_i; the first time it passes
 *     (alpha - beta > that margin: its margin has recovered) the mark is
 *     cleared and later tests use gamma_i again.  A row kept by the horizon
 *     without a test keeps its mark.
 * Outputs: ids [nq*c] (in/out), alpha [nq] (in/out), anchor_layer [nq]
 * (in/out), elevated [nq] (in/out; may be NULL when gamma_h is 0), flags
 * [nq] (out: 1 = row was fully routed at this layer),
 * beta_out [nq] (out, may be NULL; relay only), counts[2] (out: rows fully
 * routed, score pairs evaluated under the counting rule below).
 * Counting rule (reading of RouteRelay §5.2 "evaluated query-key score
 * pairs"): an anchor row costs its n_valid scores; a relay row costs its
 * non-padding candidates plus n_valid if it is refreshed.
 * Returns 0, or -1 when a ledger id is out of range.                       */
/* ------------------------------------------------------------------------ */
int32_t rro_head_layer(const rro_params *p, int32_t bh, int32_t layer,
                       int32_t anchor, const float *q, const float *kc,
                       int32_t *ids, double *alpha, int32_t *anchor_layer,
                       uint8_t *flags, double *beta_out, int64_t *counts,
                       const double *gamma_rows, uint8_t *elevated)
{
    const int32_t use_h = p->gamma_h > 0.0 && elevated != NULL;
    const int32_t c = p->k + p->m + p->r + p->g_sink + p->g_recent;
    double *S = (double *)malloc(sizeof(double) * (size_t)p->nq * (size_t)p->nk);
    rro_scores(q, kc, p->nq, p->nk, p->d, S);
    int64_t refreshed = 0, pairs = 0;
    int32_t status = 0;
    for (int32_t i = 0; i < p->nq; ++i) {
        const double *s_row = S + (int64_t)i * p->nk;
        int32_t *row = ids + (int64_t)i * c;
        int32_t n_valid = rro_valid_count(i, p->nk, p->causal);
        if (anchor) {
            rro_rebuild_row(p, bh, layer, i, s_row, row, &alpha[i]);
            anchor_layer[i] = layer;
            flags[i] = 1;
            if (use_h) elevated[i] = 0;
            refreshed += 1;
            pairs += n_valid;
            if (beta_out) beta_out[i] = NAN;
            continue;
        }
        /* A_i = R_i U C_i (Eq. 5): rescore the candidates at this layer */
        double a = INFINITY, b = -INFINITY;
        int32_t n_cand = 0;
        for (int32_t t = 0; t < c; ++t) {
            int32_t j = row[t];
            if (j < 0) continue;
            if (j >= n_valid) { status = -1; continue; }
            ++n_cand;
            if (t < p->k) { if (s_row[j] < a) a = s_row[j]; }  /* Eq. 6 */
            else          { if (s_row[j] > b) b = s_row[j]; }  /* Eq. 7 */
        }
        pairs += n_cand;
        if (beta_out) beta_out[i] = b;
        double g = gamma_rows ? gamma_rows[i] : p->gamma;
        if (use_h && elevated[i] && p->gamma_h > g) g = p->gamma_h;   /* elevated margin */
        int refresh;
        int tested = 0;
        if (p->max_age > 0 && layer - anchor_layer[i] >= p->max_age) {
            refresh = 1;                                        /* lifetime bound */
        } else if (p->min_reuse > 0 && layer - anchor_layer[i] <= p->min_reuse) {
            refresh = 0;                                        /* hysteresis horizon */
        } else {
            refresh = !(a > b + g);                             /* Eq. 8 */
            tested = 1;
        }
        flags[i] = (uint8_t)refresh;
        if (refresh) {
            rro_rebuild_row(p, bh, layer, i, s_row, row, &alpha[i]);
            anchor_layer[i] = layer;
            if (use_h) elevated[i] = 1;                         /* refreshed at a relay layer */
            refreshed += 1;
            pairs += n_valid;
        } else {
            alpha[i] = a;
            if (use_h && tested) elevated[i] = 0;               /* passed: the margin recovered */
        }
    }
    free(S);
    counts[0] = refreshed;
    counts[1] = pairs;
    return status;
}

/* Exact per-layer top-k of every row of one head (the "route every layer"
 * reference of RouteRelay §5.1, used as the recall denominator).
 * out [nq*k], -1 padded. */
void rro_exact_topk(const rro_params *p, const float *q, const float *kc,
                    int32_t *out)
{
    double *S = (double *)malloc(sizeof(double) * (size_t)p->nq * (size_t)p->nk);
    rro_scores(q, kc, p->nq, p->nk, p->d, S);
    for (int32_t i = 0; i < p->nq; ++i) {
        double a;
        rro_route_row(S + (int64_t)i * p->nk, rro_valid_count(i, p->nk, p->causal),
                      p->k, 0, out + (int64_t)i * p->k, NULL, &a);
    }
    free(S);
}
