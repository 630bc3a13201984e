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

// Half-edges of every node, grouped by node: node v's are he[hoff[v] ..
// hoff[v + 1]) in the order they were added (their `order`), so a stable
// sort of a group by neighbour gives the (neighbour, order) order.
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

// merges each node's half-edges, summed in (neighbour, order) order, into
// adjacency lists
Adj merge_halves(int n, const Halves& h, const std::vector<double>& loop)
{
    Adj a;
    a.n = n;
    a.off.assign((size_t)n + 1, 0);
    a.loop = loop;
    a.k.assign((size_t)n, 0.0);
    a.to.reserve(h.to.size());
    a.wt.reserve(h.to.size());
    // (neighbour, position in the group) of each half-edge: unique keys, so
    // any sort by them is the stable sort by neighbour
    std::vector<std::pair<int32_t, int32_t>> key;
    for (int v = 0; v < n; ++v) {
        const int64_t b = h.hoff[(size_t)v], e = h.hoff[(size_t)v + 1];
        const size_t d = (size_t)(e - b);
        key.resize(d);
        for (size_t i = 0; i < d; ++i) key[i] = {h.to[(size_t)b + i], (int32_t)i};
        if (d <= 32) {
            for (size_t i = 1; i < d; ++i) {   // insertion sort (already ordered by position)
                const auto x = key[i];
                size_t j = i;
                for (; j > 0 && key[j - 1].first > x.first; --j) key[j] = key[j - 1];
                key[j] = x;
            }
        } else {
            std::sort(key.begin(), key.end());
        }
        size_t i = 0;
        while (i < d) {
            double s = 0.0;
            const int32_t t = key[i].first;
            for (; i < d && key[i].first == t; ++i) s += h.w[(size_t)b + (size_t)key[i].second];
            a.to.push_back(t);
            a.wt.push_back(s);
        }
        a.off[(size_t)v + 1] = (int64_t)a.to.size();
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
    return merge_halves(n, h, loop);
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
    std::vector<double> loop((size_t)nn, 0.0);
    for (int u = 0; u < n; ++u) {
        const int a = node_of_ref[(size_t)ref[(size_t)u]];
        loop[(size_t)a] += g.loop[(size_t)u];
        for (int64_t e = g.off[(size_t)u]; e < g.off[(size_t)u + 1]; ++e)
            if (node_of_ref[(size_t)ref[(size_t)g.to[(size_t)e]]] == a) loop[(size_t)a] += g.wt[(size_t)e] / 2.0;
    }
    const Halves hv = collect_halves(nn, [&](auto&& sink) {
        for (int u = 0; u < n; ++u) {
            const int a = node_of_ref[(size_t)ref[(size_t)u]];
            for (int64_t e = g.off[(size_t)u]; e < g.off[(size_t)u + 1]; ++e) {
                const int b = node_of_ref[(size_t)ref[(size_t)g.to[(size_t)e]]];
                if (a != b) sink(a, b, g.wt[(size_t)e]);
            }
        }
    });
    Adj h = merge_halves(nn, hv, loop);
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
