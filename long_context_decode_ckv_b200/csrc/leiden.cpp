// leiden.cpp -- Leiden partition of the prefill token graph (host, C++).
//
// "CommunityKV: Efficient Long-Context Decoding via Graph Partitioning",
// Figure 1 caption step (2): the token graph built in prefill is
// partitioned with the Leiden algorithm (resolution gamma), and the
// communities become the retrieval units of the decode steps; the pages run
// it on the host.  Figure 2: the community count grows like sqrt(n).
//
// The graph is the directed top-kappa CSR of ckv_build_graph read as an
// undirected weighted graph (an edge i -> j of weight w adds w between i and
// j); the quality is modularity with resolution gamma,
// H = sum_c [in_c - gamma K_c^2 / (4m)].  Leiden's three phases (local
// moving with a work queue, refinement of every community from singletons,
// aggregation of the refined partition started from the unrefined one) run
// until local moving leaves every node alone, and the whole loop is repeated
// from its own result until that result no longer changes.  Every choice is
// deterministic: ascending node order for the queue and the refinement,
// moves only to neighbouring communities (largest gain, ties to staying,
// then to the lower id), refinement at zero randomness (largest positive
// gain among well-connected refined communities, ties to the lower id),
// communities renumbered by first appearance, and all sums in double in
// ascending node then neighbour order.
#include <stdint.h>

#include <algorithm>
#include <utility>
#include <vector>

#include "leiden.h"

namespace ckv {

namespace {

struct Adj {
    int n = 0;
    std::vector<int64_t> off;    // [n + 1]
    std::vector<int32_t> to;     // ascending per node
    std::vector<double> wt;
    std::vector<double> loop;    // self-loop weight
    std::vector<double> k;       // degree: sum of wt + 2 loop
};

// Half-edges of every node, grouped by node: node v's are [hoff[v],
// hoff[v + 1]) in the order they were emitted.
struct Halves {
    std::vector<int64_t> hoff;   // [n + 1]
    std::vector<int32_t> to;
    std::vector<double> w;
};

// Collects half-edges in two passes: `emit(sink)` calls sink(node, to, w) for
// every half-edge in increasing order, once to count and once to place.
template <typename Emit>
Halves collect_halves(int n, Emit emit)
{
    Halves h;
    h.hoff.assign((size_t)n + 1, 0);
    emit([&](int a, int32_t, double) { ++h.hoff[(size_t)a + 1]; });
    for (int v = 0; v < n; ++v) h.hoff[(size_t)v + 1] += h.hoff[(size_t)v];
    h.to.resize((size_t)h.hoff[(size_t)n]);
    h.w.resize((size_t)h.hoff[(size_t)n]);
    std::vector<int64_t> pos(h.hoff.begin(), h.hoff.end() - 1);
    emit([&](int a, int32_t b, double x) {
        const int64_t p = pos[(size_t)a]++;
        h.to[(size_t)p] = b;
        h.w[(size_t)p] = x;
    });
    return h;
}

// Adjacency lists from each node's half-edges: each(v, add) calls add(to, w)
// for node v's half-edges in their order.  A neighbour's weights are summed
// in that order (the same sums as summing after a stable sort by
// neighbour), and the distinct (node, neighbour) pairs are put in ascending
// neighbour order by two counting-sort transpositions: node -> neighbour
// lists scattered by neighbour (nodes ascending), then back.
template <typename Each>
Adj merge_adj(int n, Each each, const std::vector<double>& loop)
{
    Adj a;
    a.n = n;
    a.loop = loop;
    a.k.assign((size_t)n, 0.0);
    std::vector<int32_t> slot((size_t)n, -1);
    std::vector<int64_t> uoff((size_t)n + 1, 0);
    std::vector<int32_t> uto;
    std::vector<double> uw;
    for (int v = 0; v < n; ++v) {
        const int64_t u0 = (int64_t)uto.size();
        each(v, [&](int32_t t, double x) {
            if (slot[(size_t)t] < 0) {
                slot[(size_t)t] = (int32_t)(uto.size() - (size_t)u0);
                uto.push_back(t);
                uw.push_back(0.0);
            }
            uw[(size_t)u0 + (size_t)slot[(size_t)t]] += x;
        });
        for (int64_t i = u0; i < (int64_t)uto.size(); ++i) slot[(size_t)uto[(size_t)i]] = -1;
        uoff[(size_t)v + 1] = (int64_t)uto.size();
    }
    const size_t U = uto.size();
    // transpose: by neighbour, nodes ascending
    std::vector<int64_t> toff((size_t)n + 1, 0);
    for (size_t i = 0; i < U; ++i) ++toff[(size_t)uto[i] + 1];
    for (int v = 0; v < n; ++v) toff[(size_t)v + 1] += toff[(size_t)v];
    std::vector<int32_t> tfrom(U);
    std::vector<double> tw(U);
    {
        std::vector<int64_t> pos(toff.begin(), toff.end() - 1);
        for (int v = 0; v < n; ++v)
            for (int64_t i = uoff[(size_t)v]; i < uoff[(size_t)v + 1]; ++i) {
                const int64_t p = pos[(size_t)uto[(size_t)i]]++;
                tfrom[(size_t)p] = v;
                tw[(size_t)p] = uw[(size_t)i];
            }
    }
    // and back: every node's neighbours ascending
    a.to.resize(U);
    a.wt.resize(U);
    a.off = uoff;
    {
        std::vector<int64_t> pos(uoff.begin(), uoff.end() - 1);
        for (int t = 0; t < n; ++t)
            for (int64_t i = toff[(size_t)t]; i < toff[(size_t)t + 1]; ++i) {
                const int64_t p = pos[(size_t)tfrom[(size_t)i]]++;
                a.to[(size_t)p] = t;
                a.wt[(size_t)p] = tw[(size_t)i];
            }
    }
    for (int v = 0; v < n; ++v) {
        double s = 0.0;
        for (int64_t e = a.off[(size_t)v]; e < a.off[(size_t)v + 1]; ++e) s += a.wt[(size_t)e];
        a.k[(size_t)v] = s + 2.0 * a.loop[(size_t)v];
    }
    return a;
}

Adj from_topk(int n, const int64_t* rp, const int32_t* col, const float* w)
{
    std::vector<double> loop((size_t)n, 0.0);
    for (int i = 0; i < n; ++i)
        for (int64_t e = rp[i]; e < rp[i + 1]; ++e)
            if (col[e] == i) loop[(size_t)i] += (double)w[e];
    const Halves h = collect_halves(n, [&](auto&& sink) {
        for (int i = 0; i < n; ++i)
            for (int64_t e = rp[i]; e < rp[i + 1]; ++e) {
                const int32_t j = col[e];
                if (j == i) continue;
                const double x = (double)w[e];
                sink(i, j, x);
                sink(j, i, x);
            }
    });
    return merge_adj(n, [&](int v, auto&& add) {
        for (int64_t i = h.hoff[(size_t)v]; i < h.hoff[(size_t)v + 1]; ++i) add(h.to[(size_t)i], h.w[(size_t)i]);
    }, loop);
}

// first-appearance renumbering; returns the number of communities
int compact(std::vector<int>& c)
{
    std::vector<int> id(c.size(), -1);
    int next = 0;
    for (int& x : c) {
        if (id[(size_t)x] < 0) id[(size_t)x] = next++;
        x = id[(size_t)x];
    }
    return next;
}

// weights from node v to the communities of its neighbours, in order of
// first appearance (own community kept apart)
struct NeighbourWeights {
    std::vector<int> slot;       // community -> position, -1 when absent
    std::vector<int> comm;
    std::vector<double> w;
    explicit NeighbourWeights(size_t n) : slot(n, -1) {}
    void add(int c, double x)
    {
        if (slot[(size_t)c] < 0) {
            slot[(size_t)c] = (int)comm.size();
            comm.push_back(c);
            w.push_back(0.0);
        }
        w[(size_t)slot[(size_t)c]] += x;
    }
    void clear()
    {
        for (int c : comm) slot[(size_t)c] = -1;
        comm.clear();
        w.clear();
    }
};

void local_moving(const Adj& g, std::vector<int>& comm, double m, double gamma)
{
    const int n = g.n;
    std::vector<double> K((size_t)n, 0.0);
    for (int v = 0; v < n; ++v) K[(size_t)comm[(size_t)v]] += g.k[(size_t)v];
    std::vector<int> ring((size_t)std::max(n, 1));
    std::vector<char> queued((size_t)n, 1);
    for (int v = 0; v < n; ++v) ring[(size_t)v] = v;
    size_t front = 0, count = (size_t)n;
    NeighbourWeights nb((size_t)n);
    const double two_m = 2.0 * m;
    while (count) {
        const int v = ring[front];
        front = (front + 1) % (size_t)n;
        --count;
        queued[(size_t)v] = 0;
        const int own = comm[(size_t)v];
        double w_own = 0.0;
        for (int64_t e = g.off[(size_t)v]; e < g.off[(size_t)v + 1]; ++e) {
            const int c = comm[(size_t)g.to[(size_t)e]];
            if (c == own) w_own += g.wt[(size_t)e];
            else nb.add(c, g.wt[(size_t)e]);
        }
        const double kv = g.k[(size_t)v];
        int pick = own;
        double pick_gain = w_own - gamma * kv * (K[(size_t)own] - kv) / two_m;
        for (size_t t = 0; t < nb.comm.size(); ++t) {
            const int c = nb.comm[t];
            const double gain = nb.w[t] - gamma * kv * K[(size_t)c] / two_m;
            const bool better = gain > pick_gain || (gain == pick_gain && pick != own && c < pick);
            if (better) { pick = c; pick_gain = gain; }
        }
        nb.clear();
        if (pick == own) continue;
        K[(size_t)own] -= kv;
        K[(size_t)pick] += kv;
        comm[(size_t)v] = pick;
        for (int64_t e = g.off[(size_t)v]; e < g.off[(size_t)v + 1]; ++e) {
            const int u = g.to[(size_t)e];
            if (comm[(size_t)u] == pick || queued[(size_t)u]) continue;
            ring[(front + count) % (size_t)n] = u;
            ++count;
            queued[(size_t)u] = 1;
        }
    }
}

// refined partition of every community (ids: the node a refined community
// grew from)
std::vector<int> refinement(const Adj& g, const std::vector<int>& comm, int nc, double m, double gamma)
{
    const int n = g.n;
    const double two_m = 2.0 * m;
    std::vector<double> Kc((size_t)nc, 0.0);
    for (int v = 0; v < n; ++v) Kc[(size_t)comm[(size_t)v]] += g.k[(size_t)v];
    std::vector<int> ref((size_t)n), members((size_t)n, 1);
    std::vector<double> Kr(g.k), ext((size_t)n), single_ext((size_t)n);
    for (int v = 0; v < n; ++v) {
        ref[(size_t)v] = v;
        double s = 0.0;
        for (int64_t e = g.off[(size_t)v]; e < g.off[(size_t)v + 1]; ++e)
            if (comm[(size_t)g.to[(size_t)e]] == comm[(size_t)v]) s += g.wt[(size_t)e];
        ext[(size_t)v] = single_ext[(size_t)v] = s;
    }
    // nodes by community, ascending node order within one (a stable counting sort)
    std::vector<int> byc((size_t)n), cstart((size_t)nc + 1, 0);
    for (int v = 0; v < n; ++v) ++cstart[(size_t)comm[(size_t)v] + 1];
    for (int c = 0; c < nc; ++c) cstart[(size_t)c + 1] += cstart[(size_t)c];
    for (int v = 0; v < n; ++v) byc[(size_t)cstart[(size_t)comm[(size_t)v]]++] = v;
    NeighbourWeights nb((size_t)n);
    for (int v : byc) {
        const int c = comm[(size_t)v];
        if (members[(size_t)ref[(size_t)v]] != 1) continue;           // v is no longer alone
        const double kv = g.k[(size_t)v];
        if (!(single_ext[(size_t)v] >= gamma * kv * (Kc[(size_t)c] - kv) / two_m)) continue;
        for (int64_t e = g.off[(size_t)v]; e < g.off[(size_t)v + 1]; ++e) {
            const int u = g.to[(size_t)e];
            if (comm[(size_t)u] == c && ref[(size_t)u] != ref[(size_t)v]) nb.add(ref[(size_t)u], g.wt[(size_t)e]);
        }
        int into = -1;
        double into_gain = 0.0, into_w = 0.0;
        for (size_t t = 0; t < nb.comm.size(); ++t) {
            const int S = nb.comm[t];
            if (!(ext[(size_t)S] >= gamma * Kr[(size_t)S] * (Kc[(size_t)c] - Kr[(size_t)S]) / two_m)) continue;
            const double gain = nb.w[t] - gamma * kv * Kr[(size_t)S] / two_m;
            if (!(gain > 0.0)) continue;
            if (into < 0 || gain > into_gain || (gain == into_gain && S < into)) {
                into = S;
                into_gain = gain;
                into_w = nb.w[t];
            }
        }
        nb.clear();
        if (into < 0) continue;
        ext[(size_t)into] = ext[(size_t)into] - into_w + (single_ext[(size_t)v] - into_w);
        Kr[(size_t)into] += kv;
        members[(size_t)into] += 1;
        members[(size_t)ref[(size_t)v]] = 0;
        ref[(size_t)v] = into;
    }
    return ref;
}

// graph of the refined communities (numbered by ascending refined id)
Adj coarsen(const Adj& g, const std::vector<int>& ref, std::vector<int>& node_of_ref)
{
    const int n = g.n;
    node_of_ref.assign((size_t)n, -1);
    std::vector<char> present((size_t)n, 0);
    for (int v = 0; v < n; ++v) present[(size_t)ref[(size_t)v]] = 1;
    int nn = 0;
    for (int r = 0; r < n; ++r)
        if (present[(size_t)r]) node_of_ref[(size_t)r] = nn++;
    // coarse node of every node, and each coarse node's members ascending (a
    // stable counting sort): a coarse node's half-edges are its members'
    // edges in ascending member order, as they come in one pass over the nodes
    std::vector<int> cn((size_t)n), mstart((size_t)nn + 1, 0), mem((size_t)n);
    for (int u = 0; u < n; ++u) cn[(size_t)u] = node_of_ref[(size_t)ref[(size_t)u]];
    for (int u = 0; u < n; ++u) ++mstart[(size_t)cn[(size_t)u] + 1];
    for (int a = 0; a < nn; ++a) mstart[(size_t)a + 1] += mstart[(size_t)a];
    {
        std::vector<int> pos(mstart.begin(), mstart.end() - 1);
        for (int u = 0; u < n; ++u) mem[(size_t)pos[(size_t)cn[(size_t)u]]++] = u;
    }
    std::vector<double> loop((size_t)nn, 0.0);
    for (int a = 0; a < nn; ++a)
        for (int i = mstart[(size_t)a]; i < mstart[(size_t)a + 1]; ++i) {
            const int u = mem[(size_t)i];
            loop[(size_t)a] += g.loop[(size_t)u];
            for (int64_t e = g.off[(size_t)u]; e < g.off[(size_t)u + 1]; ++e)
                if (cn[(size_t)g.to[(size_t)e]] == a) loop[(size_t)a] += g.wt[(size_t)e] / 2.0;
        }
    Adj h = merge_adj(nn, [&](int a, auto&& add) {
        for (int i = mstart[(size_t)a]; i < mstart[(size_t)a + 1]; ++i) {
            const int u = mem[(size_t)i];
            for (int64_t e = g.off[(size_t)u]; e < g.off[(size_t)u + 1]; ++e) {
                const int b = cn[(size_t)g.to[(size_t)e]];
                if (b != a) add(b, g.wt[(size_t)e]);
            }
        }
    }, loop);
    std::fill(h.k.begin(), h.k.end(), 0.0);
    for (int u = 0; u < n; ++u) h.k[(size_t)node_of_ref[(size_t)ref[(size_t)u]]] += g.k[(size_t)u];
    return h;
}

// one Leiden run from the partition `start` of the original graph
std::vector<int> leiden_once(const Adj& base, const std::vector<int>& start, double m, double gamma, int max_levels)
{
    Adj g = base;
    std::vector<int> comm = start;
    std::vector<int> level_node((size_t)base.n);
    for (int i = 0; i < base.n; ++i) level_node[(size_t)i] = i;
    for (int level = 0; level < max_levels; ++level) {
        local_moving(g, comm, m, gamma);
        const int nc = compact(comm);
        if (nc == g.n) break;
        const std::vector<int> ref = refinement(g, comm, nc, m, gamma);
        std::vector<int> node_of_ref;
        Adj h = coarsen(g, ref, node_of_ref);
        if (h.n == g.n) break;                               // nothing merged: no coarser level
        std::vector<int> hcomm((size_t)h.n);
        for (int u = 0; u < g.n; ++u) hcomm[(size_t)node_of_ref[(size_t)ref[(size_t)u]]] = comm[(size_t)u];
        compact(hcomm);
        for (int& x : level_node) x = node_of_ref[(size_t)ref[(size_t)x]];
        comm.swap(hcomm);
        g = std::move(h);
    }
    std::vector<int> out((size_t)base.n);
    for (int i = 0; i < base.n; ++i) out[(size_t)i] = comm[(size_t)level_node[(size_t)i]];
    compact(out);
    return out;
}

}  // namespace

int leiden_partition(int n, const int64_t* row_ptr, const int32_t* col, const float* w, double gamma,
                     int max_levels, int32_t* labels)
{
    if (n <= 0) return 0;
    const Adj g = from_topk(n, row_ptr, col, w);
    double deg_sum = 0.0;
    for (int v = 0; v < n; ++v) deg_sum += g.k[(size_t)v];
    const double m = deg_sum / 2.0;
    std::vector<int> part((size_t)n);
    for (int v = 0; v < n; ++v) part[(size_t)v] = v;
    if (m > 0.0) {
        for (int run = 0; run < max_levels; ++run) {
            std::vector<int> next = leiden_once(g, part, m, gamma, max_levels);
            const bool fixed = next == part;
            part.swap(next);
            if (fixed) break;
        }
    }
    const int nc = compact(part);
    for (int v = 0; v < n; ++v) labels[v] = part[(size_t)v];
    return nc;
}

}  // namespace ckv
