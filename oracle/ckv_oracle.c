/*
 * ckv_oracle.c -- CPU oracle for CommunityKV decode and prefill graph.
 *
 * TEST INFRASTRUCTURE ONLY: called by tests/, the smoke check and the
 * benchmark's CPU-baseline leg; never by the CUDA library, with which it
 * shares no code.  Plain single-threaded C, compiled without FMA
 * contraction (-ffp-contract=off) so every rounding below is the one the
 * source states.
 *
 * Source: "CommunityKV: Efficient Long-Context Decoding via Graph
 * Partitioning": abstract, Figure 1 caption steps (1)-(3), Table 1.
 * Each function names the passage it follows and the reading it takes
 * where the pages are silent.
 */
#include "ckv_oracle.h"

#include <math.h>
#include <stdlib.h>
#include <string.h>

struct ckvo_graph {
    int n_comm, D, n_max;
    int ntok;          /* positions [0, ntok) are sinks or assigned members */
    int n_sinks;
    float* mu;         /* [n_comm][D] centroids (float storage)            */
    int32_t* size;     /* [n_comm]                                          */
    int32_t* cap;      /* [n_comm] allocated length of mem[c]               */
    int32_t** mem;     /* [n_comm] ascending member positions               */
};

/* ---- element access --------------------------------------------------- */
static double elem(const void* base, int dtype, int64_t i)
{
    if (dtype == CKVO_BF16) {
        /* bfloat16 is the top half of an IEEE single: widening is exact. */
        uint32_t u = (uint32_t)((const uint16_t*)base)[i] << 16;
        float f;
        memcpy(&f, &u, sizeof f);
        return (double)f;
    }
    return (double)((const float*)base)[i];
}

static double relgap(double a, double b)
{
    double m = fmax(fabs(a), fabs(b));
    if (m == 0.0) return 0.0;
    return fabs(a - b) / m;
}

/* ---- state ------------------------------------------------------------ */
ckvo_graph* ckvo_graph_new(int n_comm, int head_dim, int n_max)
{
    if (n_comm <= 0 || head_dim <= 0 || n_max <= 0) return NULL;
    ckvo_graph* g = (ckvo_graph*)calloc(1, sizeof *g);
    g->n_comm = n_comm;
    g->D = head_dim;
    g->n_max = n_max;
    g->mu = (float*)calloc((size_t)n_comm * head_dim, sizeof(float));
    g->size = (int32_t*)calloc((size_t)n_comm, sizeof(int32_t));
    g->cap = (int32_t*)calloc((size_t)n_comm, sizeof(int32_t));
    g->mem = (int32_t**)calloc((size_t)n_comm, sizeof(int32_t*));
    return g;
}

void ckvo_graph_free(ckvo_graph* g)
{
    if (!g) return;
    for (int c = 0; c < g->n_comm; ++c) free(g->mem[c]);
    free(g->mem);
    free(g->cap);
    free(g->size);
    free(g->mu);
    free(g);
}

int ckvo_graph_ntok(const ckvo_graph* g) { return g->ntok; }

static void append_member(ckvo_graph* g, int c, int32_t j)
{
    if (g->size[c] == g->cap[c]) {
        int nc = g->cap[c] ? 2 * g->cap[c] : 16;
        g->mem[c] = (int32_t*)realloc(g->mem[c], (size_t)nc * sizeof(int32_t));
        g->cap[c] = nc;
    }
    g->mem[c][g->size[c]++] = j;
}

/* Figure 1, step (2) "Initial Partitioning": the Leiden partition arrives as
 * a label per position; each community gets a centroid.  Reading: the
 * centroid is the mean of the member keys; sink positions [0, S) belong to
 * no community (they are attended at every step instead, step (3)).
 * The sum runs over members in ascending position, in double, and the mean
 * is rounded once to float. */
int ckvo_init(ckvo_graph* g, int n, int n_sinks, const int32_t* labels,
              const void* K, int kv_dtype)
{
    if (n < n_sinks || n > g->n_max) return -1;
    for (int j = n_sinks; j < n; ++j)
        if (labels[j] < 0 || labels[j] >= g->n_comm) return -1;
    for (int c = 0; c < g->n_comm; ++c) g->size[c] = 0;
    for (int j = n_sinks; j < n; ++j) append_member(g, labels[j], j);
    const int D = g->D;
    for (int c = 0; c < g->n_comm; ++c) {
        for (int d = 0; d < D; ++d) {
            double sum = 0.0;
            for (int r = 0; r < g->size[c]; ++r)
                sum += elem(K, kv_dtype, (int64_t)g->mem[c][r] * D + d);
            g->mu[(size_t)c * D + d] =
                g->size[c] ? (float)(sum / (double)g->size[c]) : 0.0f;
        }
    }
    g->ntok = n;
    g->n_sinks = n_sinks;
    return 0;
}

void ckvo_get_centroids(const ckvo_graph* g, float* mu)
{
    memcpy(mu, g->mu, (size_t)g->n_comm * g->D * sizeof(float));
}

void ckvo_get_sizes(const ckvo_graph* g, int32_t* size)
{
    memcpy(size, g->size, (size_t)g->n_comm * sizeof(int32_t));
}

int ckvo_get_members(const ckvo_graph* g, int32_t* members)
{
    int k = 0;
    for (int c = 0; c < g->n_comm; ++c)
        for (int r = 0; r < g->size[c]; ++r) members[k++] = g->mem[c][r];
    return k;
}

int ckvo_set_state(ckvo_graph* g, int n_tok, const float* mu, const int32_t* size,
                   const int32_t* members)
{
    int k = 0;
    for (int c = 0; c < g->n_comm; ++c) {
        if (size[c] < 0) return -1;
        g->size[c] = 0;
    }
    for (int c = 0; c < g->n_comm; ++c)
        for (int r = 0; r < size[c]; ++r) append_member(g, c, members[k++]);
    memcpy(g->mu, mu, (size_t)g->n_comm * g->D * sizeof(float));
    g->ntok = n_tok;
    return 0;
}

/* ---- a1: centroid scoring ---------------------------------------------- */
/* Figure 1, step (3): "score the query against community centroids";
 * Table 1 puts this retrieval at O(sqrt(n) d).  Reading for a query-group
 * graph (abstract: "query-group graph aggregation"): the score is the sum
 * over the group's query heads of q_h . mu_c.  Empty communities have no
 * centroid and score -inf. */
void ckvo_score(const ckvo_graph* g, int n_heads, const void* q, int q_dtype, float* s)
{
    const int D = g->D;
    for (int c = 0; c < g->n_comm; ++c) {
        if (g->size[c] == 0) {
            s[c] = -INFINITY;
            continue;
        }
        double acc = 0.0;
        for (int h = 0; h < n_heads; ++h)
            for (int i = 0; i < D; ++i)
                acc += elem(q, q_dtype, (int64_t)h * D + i) * (double)g->mu[(size_t)c * D + i];
        s[c] = (float)acc;
    }
}

/* ---- a2: top-C communities up to the token budget ---------------------- */
typedef struct { float s; int32_t id; } scored;

static int cmp_scored(const void* a, const void* b)
{
    const scored* x = (const scored*)a;
    const scored* y = (const scored*)b;
    if (x->s > y->s) return -1;
    if (x->s < y->s) return 1;
    return (x->id < y->id) ? -1 : (x->id > y->id);
}

/* Figure 1, step (3) "retrieve a candidate subset"; the token budgets of
 * Tables 2-3.  Reading: greedy prefix in (score desc, id asc) order that
 * stops at the first community that does not fit, and keeps at least one. */
int ckvo_select(int n_comm, const float* s, const int32_t* size, int budget,
                int32_t* sel, float* gap_lo, float* gap_hi)
{
    scored* o = (scored*)malloc((size_t)(n_comm > 0 ? n_comm : 1) * sizeof *o);
    int cnt = 0;
    for (int c = 0; c < n_comm; ++c)
        if (size[c] > 0) { o[cnt].s = s[c]; o[cnt].id = c; ++cnt; }
    qsort(o, (size_t)cnt, sizeof *o, cmp_scored);
    long long acc = 0;
    int C = 0;
    while (C < cnt && acc + size[o[C].id] <= budget) {
        acc += size[o[C].id];
        ++C;
    }
    if (C == 0 && cnt > 0) { C = 1; acc = size[o[0].id]; }
    *gap_lo = INFINITY;
    *gap_hi = INFINITY;
    if (C < cnt) {
        *gap_lo = (float)relgap(o[C - 1].s, o[C].s);
        /* The next community only matters if it would have fit. */
        if (C + 1 < cnt && acc + size[o[C + 1].id] <= budget)
            *gap_hi = (float)relgap(o[C].s, o[C + 1].s);
    }
    for (int k = 0; k < C; ++k) sel[k] = o[k].id;
    free(o);
    return C;
}

/* ---- a3: exact attention over sinks, the subset and the new token ------- */
/* Figure 1, step (3): "run exact attention on this subset together with sink
 * tokens".  z = q.k / sqrt(D); softmax over the listed rows; all in double. */
void ckvo_attend(int n_heads, int D, const void* q, int q_dtype,
                 const void* K, const void* V, int kv_dtype,
                 const int32_t* rows, int R, float* out, double* p,
                 double* m_out, double* l_out)
{
    double* z = (double*)malloc((size_t)(R > 0 ? R : 1) * sizeof(double));
    const double inv_sqrt_d = 1.0 / sqrt((double)D);
    for (int h = 0; h < n_heads; ++h) {
        double m = -INFINITY;
        for (int r = 0; r < R; ++r) {
            double dot = 0.0;
            for (int i = 0; i < D; ++i)
                dot += elem(q, q_dtype, (int64_t)h * D + i) *
                       elem(K, kv_dtype, (int64_t)rows[r] * D + i);
            z[r] = dot * inv_sqrt_d;
            if (z[r] > m) m = z[r];
        }
        double l = 0.0;
        for (int r = 0; r < R; ++r) l += exp(z[r] - m);
        for (int i = 0; i < D; ++i) {
            double o = 0.0;
            for (int r = 0; r < R; ++r)
                o += exp(z[r] - m) / l * elem(V, kv_dtype, (int64_t)rows[r] * D + i);
            out[(size_t)h * D + i] = (float)o;
        }
        if (p)
            for (int r = 0; r < R; ++r) p[(size_t)h * R + r] = exp(z[r] - m) / l;
        if (m_out) m_out[h] = m;
        if (l_out) l_out[h] = l;
    }
    free(z);
}

/* ---- NEXT f3: attention-mass recall of the retrieved set ---------------- */
/* Figure 3 (right) caption: the share of the full attention mass that the
 * retrieved set captures.  Reading: per query head, with the dense softmax
 * over every cached position [0, n) (the new token included), recall =
 * sum over the step's attended rows (sinks, kept members, the new token) of
 * the dense probabilities = l_sel * exp(m_sel - m_den) / l_den, where
 * (m_sel, l_sel) are the subset softmax statistics of ckvo_attend.  This
 * function returns the dense statistics (m_den, l_den), in double. */
void ckvo_dense_stats(int n_heads, int D, const void* q, int q_dtype, const void* K, int kv_dtype, int n,
                      double* m_out, double* l_out)
{
    double* z = (double*)malloc((size_t)(n > 0 ? n : 1) * sizeof(double));
    const double inv_sqrt_d = 1.0 / sqrt((double)D);
    for (int h = 0; h < n_heads; ++h) {
        double m = -INFINITY;
        for (int j = 0; j < n; ++j) {
            double dot = 0.0;
            for (int i = 0; i < D; ++i)
                dot += elem(q, q_dtype, (int64_t)h * D + i) * elem(K, kv_dtype, (int64_t)j * D + i);
            z[j] = dot * inv_sqrt_d;
            if (z[j] > m) m = z[j];
        }
        double l = 0.0;
        for (int j = 0; j < n; ++j) l += exp(z[j] - m);
        m_out[h] = m;
        l_out[h] = l;
    }
    free(z);
}

/* ---- a4: top-kappa edges ------------------------------------------------ */
typedef struct { float w; int32_t tok; int32_t idx; } cand;

static int cmp_cand(const void* a, const void* b)
{
    const cand* x = (const cand*)a;
    const cand* y = (const cand*)b;
    if (x->w > y->w) return -1;
    if (x->w < y->w) return 1;
    return (x->tok < y->tok) ? -1 : (x->tok > y->tok);
}

/* Figure 1, step (3): "use the resulting top-kappa keys to update the new
 * token's edges".  Ranking by (w desc, token asc) on the float w. */
int ckvo_topk(int R, const float* w, const int32_t* tok, int kappa,
              int32_t* out_idx, float* gap)
{
    cand* o = (cand*)malloc((size_t)(R > 0 ? R : 1) * sizeof *o);
    for (int r = 0; r < R; ++r) { o[r].w = w[r]; o[r].tok = tok[r]; o[r].idx = r; }
    qsort(o, (size_t)R, sizeof *o, cmp_cand);
    int E = R < kappa ? R : kappa;
    for (int k = 0; k < E; ++k) out_idx[k] = o[k].idx;
    *gap = (R > kappa) ? (float)relgap(o[kappa - 1].w, o[kappa].w) : INFINITY;
    free(o);
    return E;
}

/* ---- a5: constant-time community assignment ----------------------------- */
/* Abstract: "a local update rule assigns newly generated tokens to
 * communities in constant time"; Figure 1: the new token's top-kappa edges
 * are used to "assign it to a community".  The rule is not stated.
 * Reading: weighted plurality -- each edge votes its weight for its
 * endpoint's community, summed in rank order in double; the largest vote
 * wins, ties to the lower community id.  Returns -1 when there are no
 * edges. */
int ckvo_vote(int n_edges, const int32_t* edge_comm, const float* edge_w, double* gap)
{
    int32_t ids[CKVO_KMAX];
    double v[CKVO_KMAX];
    int nd = 0;
    for (int e = 0; e < n_edges; ++e) {
        int k = 0;
        while (k < nd && ids[k] != edge_comm[e]) ++k;
        if (k == nd) { ids[nd] = edge_comm[e]; v[nd] = 0.0; ++nd; }
        v[k] += (double)edge_w[e];
    }
    *gap = INFINITY;
    if (nd == 0) return -1;
    int best = 0;
    for (int k = 1; k < nd; ++k)
        if (v[k] > v[best] || (v[k] == v[best] && ids[k] < ids[best])) best = k;
    int second = -1;
    for (int k = 0; k < nd; ++k) {
        if (k == best) continue;
        if (second < 0 || v[k] > v[second] || (v[k] == v[second] && ids[k] < ids[second]))
            second = k;
    }
    if (second >= 0) *gap = relgap(v[best], v[second]);
    return ids[best];
}

/* ---- a6: running-mean centroid update ----------------------------------- */
/* Table 1: the per-step update costs O(d) -- one centroid changes.  Reading:
 * the centroid stays the mean of its members, updated as a running mean
 * mu + (k_t - mu) / (m + 1) in double and rounded once to float; the new
 * token is appended to the community's members. */
int ckvo_update(ckvo_graph* g, int c, int t, const void* k_t, int kv_dtype)
{
    if (c < 0 || c >= g->n_comm) return -1;
    const int D = g->D;
    const double m1 = (double)(g->size[c] + 1);
    for (int d = 0; d < D; ++d) {
        double mu = (double)g->mu[(size_t)c * D + d];
        double k = elem(k_t, kv_dtype, d);
        g->mu[(size_t)c * D + d] = (float)(mu + (k - mu) / m1);
    }
    append_member(g, c, t);
    return 0;
}

/* ---- the decode step ------------------------------------------------------ */
/* Figure 1, step (3), in the caption's order: score, retrieve, attend over
 * subset + sinks (+ the new token itself, as a causal query always sees its
 * own key), top-kappa edges (sinks and self excluded, as in step (1)),
 * assign, update. */
int ckvo_decode_step(ckvo_graph* g, int n_heads, int n_sinks, int kappa, int budget,
                     int n, const void* q, const void* K, const void* V, int dtype,
                     float* out, int32_t* sel, ckvo_step_info* info)
{
    if (n != g->ntok + 1 || n > g->n_max || kappa > CKVO_KMAX || n_heads > CKVO_KMAX)
        return -1;
    const int D = g->D;
    const int t = n - 1;
    float* s = (float*)malloc((size_t)g->n_comm * sizeof(float));
    ckvo_score(g, n_heads, q, dtype, s);
    int C = ckvo_select(g->n_comm, s, g->size, budget, sel, &info->cut_gap_lo, &info->cut_gap_hi);
    free(s);

    int T = 0;
    for (int k = 0; k < C; ++k) T += g->size[sel[k]];
    const int R = n_sinks + T + 1;
    int32_t* rows = (int32_t*)malloc((size_t)R * sizeof(int32_t));
    int32_t* comm = (int32_t*)malloc((size_t)(T > 0 ? T : 1) * sizeof(int32_t));
    int r = 0;
    for (int j = 0; j < n_sinks; ++j) rows[r++] = j;
    for (int k = 0; k < C; ++k)
        for (int i = 0; i < g->size[sel[k]]; ++i) {
            comm[r - n_sinks] = sel[k];
            rows[r++] = g->mem[sel[k]][i];
        }
    rows[r++] = t;

    double* p = (double*)malloc((size_t)n_heads * R * sizeof(double));
    ckvo_attend(n_heads, D, q, dtype, K, V, dtype, rows, R, out, p, info->m, info->l);

    float* w = (float*)malloc((size_t)(T > 0 ? T : 1) * sizeof(float));
    for (int i = 0; i < T; ++i) {
        double acc = 0.0;
        for (int h = 0; h < n_heads; ++h) acc += p[(size_t)h * R + n_sinks + i];
        w[i] = (float)acc;
    }
    int32_t idx[CKVO_KMAX];
    int E = ckvo_topk(T, w, rows + n_sinks, kappa, idx, &info->edge_gap);
    for (int e = 0; e < E; ++e) {
        info->edge_col[e] = rows[n_sinks + idx[e]];
        info->edge_w[e] = w[idx[e]];
        info->edge_comm[e] = comm[idx[e]];
    }
    int cs = ckvo_vote(E, info->edge_comm, info->edge_w, &info->vote_gap);
    /* Reading: with no selected member there is nothing to vote on, which
     * only happens when every community is empty; the token then joins 0. */
    if (cs < 0) cs = 0;
    ckvo_update(g, cs, t, (const char*)K + (size_t)t * D * (dtype == CKVO_BF16 ? 2 : 4), dtype);
    g->ntok = n;

    info->C = C;
    info->T = T;
    info->n_edges = E;
    info->assigned = cs;
    free(w);
    free(p);
    free(comm);
    free(rows);
    return 0;
}

/* ---- prefill graph -------------------------------------------------------- */
/* Figure 1, step (1): each query connects to its top-kappa keys of the
 * attention matrix; sink tokens are excluded from the pool.  Reading: the
 * causal row i attends j in [0, i]; candidates are j in [S, i-1] (no sink,
 * no self loop), so row i has min(kappa, max(0, i - S)) edges. */
int64_t ckvo_row_ptr(int64_t i, int n_sinks, int kappa)
{
    int64_t total = 0;
    for (int64_t r = 0; r < i; ++r) {
        int64_t e = r - n_sinks;
        if (e < 0) e = 0;
        if (e > kappa) e = kappa;
        total += e;
    }
    return total;
}

void ckvo_prefill_rows(int n, int D, int n_sinks, int kappa, const void* Q, const void* K,
                       int dtype, const int32_t* rows, int n_rows,
                       int32_t* col, float* w, int32_t* deg, float* gap)
{
    double* z = (double*)malloc((size_t)n * sizeof(double));
    const double inv_sqrt_d = 1.0 / sqrt((double)D);
    for (int rr = 0; rr < n_rows; ++rr) {
        const int i = rows[rr];
        double m = -INFINITY;
        for (int j = 0; j <= i; ++j) {
            double dot = 0.0;
            for (int d = 0; d < D; ++d)
                dot += elem(Q, dtype, (int64_t)i * D + d) * elem(K, dtype, (int64_t)j * D + d);
            z[j] = dot * inv_sqrt_d;
            if (z[j] > m) m = z[j];
        }
        double l = 0.0;
        for (int j = 0; j <= i; ++j) l += exp(z[j] - m);
        /* Keep the best kappa+1 candidates by (float z desc, j asc): the
         * extra one gives the cutoff gap. */
        float bz[CKVO_KMAX + 1];
        int32_t bj[CKVO_KMAX + 1];
        int nb = 0;
        for (int j = n_sinks; j < i; ++j) {
            float zf = (float)z[j];
            int pos = nb;
            while (pos > 0 && bz[pos - 1] < zf) --pos;   /* equal z: earlier j stays ahead */
            if (pos > kappa) continue;
            int last = nb < kappa + 1 ? nb : kappa;
            for (int k = last; k > pos; --k) { bz[k] = bz[k - 1]; bj[k] = bj[k - 1]; }
            bz[pos] = zf;
            bj[pos] = j;
            if (nb < kappa + 1) ++nb;
        }
        int e = nb < kappa ? nb : kappa;
        deg[rr] = e;
        for (int k = 0; k < e; ++k) {
            col[(size_t)rr * kappa + k] = bj[k];
            w[(size_t)rr * kappa + k] = (float)(exp(z[bj[k]] - m) / l);
        }
        gap[rr] = (nb > kappa) ? (float)relgap(bz[kappa - 1], bz[kappa]) : INFINITY;
    }
    free(z);
}

/* ---- NEXT f2: query-group aggregated prefill graph ---------------------- */
/* The abstract contrasts one graph per query head with query-group graph
 * aggregation.  Reading for the prefill graph of a group: one graph per KV
 * head, shared by its nh query heads; for row i every head h has its own
 * causal softmax p_hij over j in [0, i] (z_hij = q_hi.k_j / sqrt(D)), the
 * edge weight is their sum w_ij = sum_h p_hij (rounded to float, the value
 * ranked), and the row's edges are the top-kappa j in [S, i-1] by
 * (w desc, j asc) -- the prefill counterpart of the decode edge rule.
 * Q holds the group's heads [nh][n][D]; K is the KV head's keys [n][D]. */
void ckvo_prefill_rows_grouped(int n, int D, int n_sinks, int kappa, int nh, const void* Q, const void* K,
                               int dtype, const int32_t* rows, int n_rows,
                               int32_t* col, float* w, int32_t* deg, float* gap)
{
    double* z = (double*)malloc((size_t)(n > 0 ? n : 1) * sizeof(double));
    double* ws = (double*)malloc((size_t)(n > 0 ? n : 1) * sizeof(double));
    const double inv_sqrt_d = 1.0 / sqrt((double)D);
    for (int rr = 0; rr < n_rows; ++rr) {
        const int i = rows[rr];
        for (int j = 0; j <= i; ++j) ws[j] = 0.0;
        for (int h = 0; h < nh; ++h) {
            const int64_t qrow = ((int64_t)h * n + i) * D;
            double m = -INFINITY;
            for (int j = 0; j <= i; ++j) {
                double dot = 0.0;
                for (int d = 0; d < D; ++d)
                    dot += elem(Q, dtype, qrow + d) * elem(K, dtype, (int64_t)j * D + d);
                z[j] = dot * inv_sqrt_d;
                if (z[j] > m) m = z[j];
            }
            double l = 0.0;
            for (int j = 0; j <= i; ++j) l += exp(z[j] - m);
            for (int j = 0; j <= i; ++j) ws[j] += exp(z[j] - m) / l;
        }
        float bw[CKVO_KMAX + 1];
        int32_t bj[CKVO_KMAX + 1];
        int nb = 0;
        for (int j = n_sinks; j < i; ++j) {
            const float wf = (float)ws[j];
            int pos = nb;
            while (pos > 0 && bw[pos - 1] < wf) --pos;   /* equal w: earlier j stays ahead */
            if (pos > kappa) continue;
            int last = nb < kappa + 1 ? nb : kappa;
            for (int k = last; k > pos; --k) { bw[k] = bw[k - 1]; bj[k] = bj[k - 1]; }
            bw[pos] = wf;
            bj[pos] = j;
            if (nb < kappa + 1) ++nb;
        }
        int e = nb < kappa ? nb : kappa;
        deg[rr] = e;
        for (int k = 0; k < e; ++k) {
            col[(size_t)rr * kappa + k] = bj[k];
            w[(size_t)rr * kappa + k] = bw[k];
        }
        gap[rr] = (nb > kappa) ? (float)relgap(bw[kappa - 1], bw[kappa]) : INFINITY;
    }
    free(ws);
    free(z);
}
