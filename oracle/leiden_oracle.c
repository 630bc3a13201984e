/*
 * leiden_oracle.c -- CPU oracle of the Leiden partition and the modularity
 * of a token graph.
 *
 * TEST INFRASTRUCTURE ONLY (see ckv_oracle.h): plain, slow and single
 * threaded; it shares no code with the library.
 *
 * "CommunityKV: Efficient Long-Context Decoding via Graph Partitioning",
 * Figure 1 caption step (2): the prefill token graph is partitioned with the
 * Leiden algorithm; Figure 2: the community count grows like sqrt(n);
 * Figure 3 (left): the modularity Q of the partition.  The pages name the
 * algorithm and its resolution only.  Readings taken here:
 *
 *  - Graph: undirected and weighted.  A directed edge (i -> j, w) of the
 *    top-kappa graph adds w to A_ij and A_ji; an edge i -> i adds w to the
 *    self-loop of i.  Node degree k_i = sum_j A_ij + 2 self_i, m = sum k / 2.
 *  - Quality: modularity with resolution gamma, H = sum_c [in_c -
 *    gamma K_c^2 / (4m)] (in_c: weight inside c, K_c: degree of c);
 *    Q = H / m.
 *  - Leiden steps as in the method's original description (local moving with
 *    a queue, refinement inside each community, aggregation of the refined
 *    partition with the unrefined one as the start, until local moving
 *    leaves every node alone), made deterministic:
 *      * nodes are queued and visited in ascending id;
 *      * a node moves only to the community of a neighbour, to the one of
 *        largest gain, ties to its own community, then to the lower id;
 *      * refinement is the zero-randomness limit: a well-connected
 *        singleton joins the well-connected refined community of largest
 *        positive gain (ties to the lower id);
 *      * community ids are renumbered by first appearance after every
 *        local moving, aggregate nodes follow ascending refined ids;
 *      * every sum runs in ascending node, then neighbour, order in double;
 *      * the loop also stops when aggregation no longer shrinks the graph;
 *      * the whole algorithm is iterated, each run starting from the
 *        previous run's partition, until a run returns its start (the
 *        iteration under which the original description's guarantees hold).
 */
#include "ckv_oracle.h"

#include <math.h>
#include <stdlib.h>
#include <string.h>

typedef struct {
    int n;
    int64_t* off;    /* [n+1] */
    int32_t* nbr;    /* neighbours, ascending per node */
    double* wt;
    double* self;    /* [n] self-loop weight */
    double* deg;     /* [n] */
} lgraph;

typedef struct {
    int32_t to;
    int64_t seq;
    double w;
} lentry;

static int cmp_entry(const void* a, const void* b)
{
    const lentry* x = (const lentry*)a;
    const lentry* y = (const lentry*)b;
    if (x->to != y->to) return x->to < y->to ? -1 : 1;
    return x->seq < y->seq ? -1 : (x->seq > y->seq ? 1 : 0);
}

static void lg_free(lgraph* g)
{
    free(g->off); free(g->nbr); free(g->wt); free(g->self); free(g->deg);
    memset(g, 0, sizeof(*g));
}

/* Adjacency from per-node entry lists (each sorted by (to, seq), equal `to`
 * summed in seq order).  cnt[v] entries of node v start at start[v]. */
static void lg_build(lgraph* g, int n, lentry* ent, const int64_t* start, const int64_t* cnt, const double* self)
{
    g->n = n;
    g->off = (int64_t*)calloc((size_t)n + 1, sizeof(int64_t));
    g->self = (double*)calloc((size_t)n + 1, sizeof(double));
    g->deg = (double*)calloc((size_t)n + 1, sizeof(double));
    int64_t total = 0;
    for (int v = 0; v < n; ++v) total += cnt[v];
    g->nbr = (int32_t*)malloc((size_t)(total > 0 ? total : 1) * sizeof(int32_t));
    g->wt = (double*)malloc((size_t)(total > 0 ? total : 1) * sizeof(double));
    int64_t k = 0;
    for (int v = 0; v < n; ++v) {
        lentry* e = ent + start[v];
        qsort(e, (size_t)cnt[v], sizeof(lentry), cmp_entry);
        g->off[v] = k;
        for (int64_t a = 0; a < cnt[v];) {
            int64_t b = a;
            double s = 0.0;
            while (b < cnt[v] && e[b].to == e[a].to) s += e[b++].w;
            g->nbr[k] = e[a].to;
            g->wt[k] = s;
            ++k;
            a = b;
        }
        g->self[v] = self[v];
    }
    g->off[n] = k;
    for (int v = 0; v < n; ++v) {
        double d = 0.0;
        for (int64_t a = g->off[v]; a < g->off[v + 1]; ++a) d += g->wt[a];
        g->deg[v] = d + 2.0 * g->self[v];
    }
}

static void lg_from_csr(lgraph* g, int n, const int64_t* row_ptr, const int32_t* col, const float* w)
{
    int64_t* cnt = (int64_t*)calloc((size_t)n + 1, sizeof(int64_t));
    int64_t* start = (int64_t*)calloc((size_t)n + 1, sizeof(int64_t));
    double* self = (double*)calloc((size_t)n + 1, sizeof(double));
    for (int i = 0; i < n; ++i)
        for (int64_t e = row_ptr[i]; e < row_ptr[i + 1]; ++e)
            if (col[e] != i) { cnt[i]++; cnt[col[e]]++; }
    for (int v = 1; v <= n; ++v) start[v] = start[v - 1] + cnt[v - 1];
    lentry* ent = (lentry*)malloc((size_t)(start[n] > 0 ? start[n] : 1) * sizeof(lentry));
    int64_t* fill = (int64_t*)calloc((size_t)n + 1, sizeof(int64_t));
    int64_t seq = 0;
    for (int i = 0; i < n; ++i)
        for (int64_t e = row_ptr[i]; e < row_ptr[i + 1]; ++e) {
            const int j = col[e];
            if (j == i) { self[i] += (double)w[e]; continue; }
            lentry a = {j, seq, (double)w[e]}, b = {i, seq, (double)w[e]};
            ent[start[i] + fill[i]++] = a;
            ent[start[j] + fill[j]++] = b;
            ++seq;
        }
    lg_build(g, n, ent, start, cnt, self);
    free(ent); free(fill); free(self); free(start); free(cnt);
}

/* community ids by first appearance over ascending nodes; returns the count */
static int renumber(int n, int* comm)
{
    int* map = (int*)malloc((size_t)(n > 0 ? n : 1) * sizeof(int));
    for (int i = 0; i < n; ++i) map[i] = -1;
    int nc = 0;
    for (int v = 0; v < n; ++v) {
        if (map[comm[v]] < 0) map[comm[v]] = nc++;
        comm[v] = map[comm[v]];
    }
    free(map);
    return nc;
}

/* local moving with a FIFO queue (all nodes, ascending, at the start) */
static void move_nodes(const lgraph* g, int* comm, double m, double gamma)
{
    const int n = g->n;
    double* K = (double*)calloc((size_t)n + 1, sizeof(double));
    for (int v = 0; v < n; ++v) K[comm[v]] += g->deg[v];
    int* q = (int*)malloc((size_t)(n > 0 ? n : 1) * sizeof(int));
    char* inq = (char*)calloc((size_t)n + 1, 1);
    int* pos = (int*)malloc((size_t)(n > 0 ? n : 1) * sizeof(int));
    int* lc = (int*)malloc((size_t)(n > 0 ? n : 1) * sizeof(int));
    double* lw = (double*)malloc((size_t)(n > 0 ? n : 1) * sizeof(double));
    for (int i = 0; i < n; ++i) { q[i] = i; inq[i] = 1; pos[i] = -1; }
    int head = 0, size = n;
    while (size > 0) {
        const int v = q[head];
        head = (head + 1) % n;
        --size;
        inq[v] = 0;
        const int a = comm[v];
        double wa = 0.0;
        int nl = 0;
        for (int64_t e = g->off[v]; e < g->off[v + 1]; ++e) {
            const int c = comm[g->nbr[e]];
            if (c == a) { wa += g->wt[e]; continue; }
            if (pos[c] < 0) { pos[c] = nl; lc[nl] = c; lw[nl] = 0.0; ++nl; }
            lw[pos[c]] += g->wt[e];
        }
        const double kv = g->deg[v];
        int best = a;
        double best_gain = wa - gamma * kv * (K[a] - kv) / (2.0 * m);
        for (int t = 0; t < nl; ++t) {
            const double gain = lw[t] - gamma * kv * K[lc[t]] / (2.0 * m);
            if (gain > best_gain || (gain == best_gain && best != a && lc[t] < best)) {
                best_gain = gain;
                best = lc[t];
            }
        }
        for (int t = 0; t < nl; ++t) pos[lc[t]] = -1;
        if (best != a) {
            K[a] -= kv;
            K[best] += kv;
            comm[v] = best;
            for (int64_t e = g->off[v]; e < g->off[v + 1]; ++e) {
                const int u = g->nbr[e];
                if (comm[u] != best && !inq[u]) {
                    q[(head + size) % n] = u;
                    ++size;
                    inq[u] = 1;
                }
            }
        }
    }
    free(lw); free(lc); free(pos); free(inq); free(q); free(K);
}

typedef struct { int c; int v; } cv_pair;
static int cmp_cv(const void* a, const void* b)
{
    const cv_pair* x = (const cv_pair*)a;
    const cv_pair* y = (const cv_pair*)b;
    if (x->c != y->c) return x->c < y->c ? -1 : 1;
    return x->v < y->v ? -1 : (x->v > y->v ? 1 : 0);
}

/* refinement of each community of comm; rcomm gets refined ids (node ids) */
static void refine(const lgraph* g, const int* comm, int nc, double m, double gamma, int* rcomm)
{
    const int n = g->n;
    double* KC = (double*)calloc((size_t)nc + 1, sizeof(double));
    for (int v = 0; v < n; ++v) KC[comm[v]] += g->deg[v];
    double* RK = (double*)malloc((size_t)(n > 0 ? n : 1) * sizeof(double));
    double* eS = (double*)malloc((size_t)(n > 0 ? n : 1) * sizeof(double));
    double* ev = (double*)malloc((size_t)(n > 0 ? n : 1) * sizeof(double));
    int* rsize = (int*)malloc((size_t)(n > 0 ? n : 1) * sizeof(int));
    for (int v = 0; v < n; ++v) {
        rcomm[v] = v;
        RK[v] = g->deg[v];
        rsize[v] = 1;
        double s = 0.0;
        for (int64_t e = g->off[v]; e < g->off[v + 1]; ++e)
            if (comm[g->nbr[e]] == comm[v]) s += g->wt[e];
        ev[v] = s;
        eS[v] = s;
    }
    cv_pair* order = (cv_pair*)malloc((size_t)(n > 0 ? n : 1) * sizeof(cv_pair));
    for (int v = 0; v < n; ++v) { order[v].c = comm[v]; order[v].v = v; }
    qsort(order, (size_t)n, sizeof(cv_pair), cmp_cv);
    int* pos = (int*)malloc((size_t)(n > 0 ? n : 1) * sizeof(int));
    int* lS = (int*)malloc((size_t)(n > 0 ? n : 1) * sizeof(int));
    double* lw = (double*)malloc((size_t)(n > 0 ? n : 1) * sizeof(double));
    for (int i = 0; i < n; ++i) pos[i] = -1;
    for (int t = 0; t < n; ++t) {
        const int v = order[t].v, c = order[t].c;
        if (rsize[rcomm[v]] != 1) continue;
        const double kv = g->deg[v];
        if (!(ev[v] >= gamma * kv * (KC[c] - kv) / (2.0 * m))) continue;
        int nl = 0;
        for (int64_t e = g->off[v]; e < g->off[v + 1]; ++e) {
            const int u = g->nbr[e];
            if (comm[u] != c || rcomm[u] == rcomm[v]) continue;
            const int S = rcomm[u];
            if (pos[S] < 0) { pos[S] = nl; lS[nl] = S; lw[nl] = 0.0; ++nl; }
            lw[pos[S]] += g->wt[e];
        }
        int best = -1;
        double best_gain = 0.0;
        for (int k = 0; k < nl; ++k) {
            const int S = lS[k];
            if (!(eS[S] >= gamma * RK[S] * (KC[c] - RK[S]) / (2.0 * m))) continue;
            const double gain = lw[k] - gamma * kv * RK[S] / (2.0 * m);
            if (gain > 0.0 && (best < 0 || gain > best_gain || (gain == best_gain && S < best))) {
                best = S;
                best_gain = gain;
            }
        }
        double wvS = 0.0;
        for (int k = 0; k < nl; ++k) {
            if (lS[k] == best) wvS = lw[k];
            pos[lS[k]] = -1;
        }
        if (best >= 0) {
            eS[best] = eS[best] - wvS + (ev[v] - wvS);
            RK[best] += kv;
            rsize[best] += 1;
            rsize[rcomm[v]] = 0;
            rcomm[v] = best;
        }
    }
    free(lw); free(lS); free(pos); free(order); free(rsize); free(ev); free(eS); free(RK); free(KC);
}

/* aggregate graph of the refined partition; returns its node count and
 * fills newidx[refined id] */
static int aggregate(const lgraph* g, const int* rcomm, int* newidx, lgraph* out)
{
    const int n = g->n;
    char* used = (char*)calloc((size_t)n + 1, 1);
    for (int v = 0; v < n; ++v) used[rcomm[v]] = 1;
    int nn = 0;
    for (int r = 0; r < n; ++r) newidx[r] = used[r] ? nn++ : -1;
    int64_t* cnt = (int64_t*)calloc((size_t)nn + 1, sizeof(int64_t));
    int64_t* start = (int64_t*)calloc((size_t)nn + 1, sizeof(int64_t));
    double* self = (double*)calloc((size_t)nn + 1, sizeof(double));
    for (int u = 0; u < n; ++u) {
        const int ru = newidx[rcomm[u]];
        for (int64_t e = g->off[u]; e < g->off[u + 1]; ++e)
            if (newidx[rcomm[g->nbr[e]]] != ru) cnt[ru]++;
    }
    for (int v = 1; v <= nn; ++v) start[v] = start[v - 1] + cnt[v - 1];
    lentry* ent = (lentry*)malloc((size_t)(start[nn] > 0 ? start[nn] : 1) * sizeof(lentry));
    int64_t* fill = (int64_t*)calloc((size_t)nn + 1, sizeof(int64_t));
    int64_t seq = 0;
    for (int u = 0; u < n; ++u) {
        const int ru = newidx[rcomm[u]];
        self[ru] += g->self[u];
        for (int64_t e = g->off[u]; e < g->off[u + 1]; ++e) {
            const int rx = newidx[rcomm[g->nbr[e]]];
            if (rx == ru) { self[ru] += g->wt[e] / 2.0; continue; }
            lentry a = {rx, seq++, g->wt[e]};
            ent[start[ru] + fill[ru]++] = a;
        }
    }
    lg_build(out, nn, ent, start, cnt, self);
    /* degrees of aggregate nodes: the members' degrees, summed in node order */
    for (int r = 0; r < nn; ++r) out->deg[r] = 0.0;
    for (int u = 0; u < n; ++u) out->deg[newidx[rcomm[u]]] += g->deg[u];
    free(fill); free(ent); free(self); free(start); free(cnt); free(used);
    return nn;
}

/* one run of the Leiden loop from the partition comm0 of the original
 * graph (labels renumbered by first appearance, count returned) */
static int leiden_run(const lgraph* g0, const int* comm0, double m, double gamma, int max_levels, int32_t* labels)
{
    const int n = g0->n;
    lgraph g;
    /* the working graph starts as a copy of the original */
    {
        int64_t* cnt = (int64_t*)calloc((size_t)n + 1, sizeof(int64_t));
        int64_t* start = (int64_t*)calloc((size_t)n + 1, sizeof(int64_t));
        for (int v = 0; v < n; ++v) { cnt[v] = g0->off[v + 1] - g0->off[v]; start[v] = g0->off[v]; }
        lentry* ent = (lentry*)malloc((size_t)(g0->off[n] > 0 ? g0->off[n] : 1) * sizeof(lentry));
        for (int64_t e = 0; e < g0->off[n]; ++e) { ent[e].to = g0->nbr[e]; ent[e].seq = e; ent[e].w = g0->wt[e]; }
        lg_build(&g, n, ent, start, cnt, g0->self);
        for (int v = 0; v < n; ++v) g.deg[v] = g0->deg[v];
        free(ent); free(start); free(cnt);
    }
    int* node_of = (int*)malloc((size_t)n * sizeof(int));
    for (int i = 0; i < n; ++i) node_of[i] = i;
    int* comm = (int*)malloc((size_t)n * sizeof(int));
    for (int v = 0; v < n; ++v) comm[v] = comm0[v];
    for (int level = 0; level < max_levels; ++level) {
        move_nodes(&g, comm, m, gamma);
        const int nc = renumber(g.n, comm);
        if (nc == g.n) break;
        int* rcomm = (int*)malloc((size_t)g.n * sizeof(int));
        refine(&g, comm, nc, m, gamma, rcomm);
        int* newidx = (int*)malloc((size_t)g.n * sizeof(int));
        lgraph h;
        const int nn = aggregate(&g, rcomm, newidx, &h);
        if (nn == g.n) {   /* refinement merged nothing: no coarser level */
            free(newidx); free(rcomm); lg_free(&h);
            break;
        }
        int* hcomm = (int*)malloc((size_t)nn * sizeof(int));
        for (int u = 0; u < g.n; ++u) hcomm[newidx[rcomm[u]]] = comm[u];
        renumber(nn, hcomm);
        for (int i = 0; i < n; ++i) node_of[i] = newidx[rcomm[node_of[i]]];
        free(comm);
        comm = hcomm;
        lg_free(&g);
        g = h;
        free(newidx); free(rcomm);
    }
    for (int i = 0; i < n; ++i) labels[i] = comm[node_of[i]];
    const int nc = renumber(n, labels);
    free(comm); free(node_of);
    lg_free(&g);
    return nc;
}

/* Leiden iterated to a fixed point: every run starts from the previous
 * run's partition (the first from singletons) until a run returns the
 * partition it started from, at most max_levels runs of at most
 * max_levels levels each. */
int ckvo_leiden(int n, const int64_t* row_ptr, const int32_t* col, const float* w, double gamma, int max_levels,
                int32_t* labels)
{
    if (n <= 0) return 0;
    lgraph g;
    lg_from_csr(&g, n, row_ptr, col, w);
    double m2 = 0.0;
    for (int v = 0; v < n; ++v) m2 += g.deg[v];
    const double m = m2 / 2.0;
    int* cur = (int*)malloc((size_t)n * sizeof(int));
    int32_t* next = (int32_t*)malloc((size_t)n * sizeof(int32_t));
    for (int v = 0; v < n; ++v) cur[v] = v;
    int nc = n;
    if (m > 0.0) {
        for (int it = 0; it < max_levels; ++it) {
            nc = leiden_run(&g, cur, m, gamma, max_levels, next);
            int same = 1;
            for (int v = 0; v < n; ++v) if (next[v] != cur[v]) { same = 0; break; }
            for (int v = 0; v < n; ++v) cur[v] = next[v];
            if (same) break;
        }
    }
    for (int v = 0; v < n; ++v) labels[v] = cur[v];
    nc = renumber(n, (int*)labels);
    free(next); free(cur);
    lg_free(&g);
    return nc;
}

double ckvo_modularity(int n, const int64_t* row_ptr, const int32_t* col, const float* w, const int32_t* labels,
                       double gamma)
{
    int nc = 0;
    for (int i = 0; i < n; ++i) if (labels[i] + 1 > nc) nc = labels[i] + 1;
    double* K = (double*)calloc((size_t)nc + 1, sizeof(double));
    double m = 0.0, in = 0.0;
    for (int i = 0; i < n; ++i)
        for (int64_t e = row_ptr[i]; e < row_ptr[i + 1]; ++e) {
            const int j = col[e];
            const double we = (double)w[e];
            m += we;
            K[labels[i]] += we;
            K[labels[j]] += we;
            if (labels[i] == labels[j]) in += we;
        }
    double kk = 0.0;
    for (int c = 0; c < nc; ++c) kk += K[c] * K[c];
    free(K);
    if (m <= 0.0) return 0.0;
    return (in - gamma * kk / (4.0 * m)) / m;
}
