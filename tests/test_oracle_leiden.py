"""Pins of the CPU oracle's Leiden partition and modularity.

"CommunityKV: Efficient Long-Context Decoding via Graph Partitioning",
Figure 1 caption step (2) (Leiden partition of the token graph), Figure 2
(community count against n) and Figure 3 left (modularity Q).  The
modularity is checked against its textbook definition on a dense matrix;
the partition against planted communities, local optimality by brute force
(no single node move raises the quality), connectedness of every community,
and its ordering against trivial partitions.
"""
import numpy as np
import pytest

import oracle


def _csr(n, edges):
    rows = [[] for _ in range(n)]
    for i, j, w in edges:
        rows[i].append((j, w))
    rp = np.zeros(n + 1, np.int64)
    col, ww = [], []
    for i in range(n):
        rp[i + 1] = rp[i] + len(rows[i])
        col += [j for j, _ in rows[i]]
        ww += [w for _, w in rows[i]]
    return rp, np.array(col, np.int32), np.array(ww, np.float32)


def _dense(n, rp, col, w):
    A = np.zeros((n, n))
    for i in range(n):
        for e in range(rp[i], rp[i + 1]):
            A[i, col[e]] += w[e]
            if col[e] != i:
                A[col[e], i] += w[e]
    return A


def _q_dense(A, labels, gamma):
    """(1 / 2m) sum_ij [A_ij - gamma k_i k_j / 2m] delta(c_i, c_j) (self-loops
    on the diagonal count twice in the degree, as the textbook's A_ii = 2 w)."""
    A2 = A + np.diag(np.diag(A))
    k = A2.sum(1)
    two_m = k.sum()
    same = labels[:, None] == labels[None, :]
    return float(((A2 - gamma * np.outer(k, k) / two_m) * same).sum() / two_m)


def _random_knn(n, kap, seed, S=0):
    """A directed top-kappa style graph: row i points to up to kappa earlier rows."""
    rng = np.random.default_rng(seed)
    edges = []
    for i in range(n):
        cand = np.arange(S, i)
        if len(cand) == 0:
            continue
        pick = rng.choice(cand, size=min(kap, len(cand)), replace=False)
        for j in pick:
            edges.append((i, int(j), float(rng.uniform(0.01, 1.0))))
    return _csr(n, edges)


@pytest.mark.parametrize("gamma", [0.5, 1.0, 2.0])
@pytest.mark.parametrize("seed", range(5))
def test_modularity_matches_textbook_definition(oracle_lib, seed, gamma):
    n = 40
    rp, col, w = _random_knn(n, 4, seed)
    rng = np.random.default_rng(100 + seed)
    for labels in (rng.integers(0, 5, n), np.arange(n), np.zeros(n, int)):
        q = oracle.modularity(rp, col, w, labels.astype(np.int32), gamma)
        assert q == pytest.approx(_q_dense(_dense(n, rp, col, w), labels, gamma), rel=1e-9, abs=1e-12)


def test_planted_cliques_are_found(oracle_lib):
    s, k = 8, 6
    n = s * k
    edges = []
    for c in range(k):
        for a in range(s):
            for b in range(a):
                edges.append((c * s + a, c * s + b, 1.0))
    for c in range(k - 1):                                   # weak bridges
        edges.append(((c + 1) * s, c * s + s - 1, 0.05))
    rp, col, w = _csr(n, sorted(edges))
    labels, C = oracle.leiden(rp, col, w, n)
    assert C == k
    np.testing.assert_array_equal(labels, np.repeat(np.arange(k), s))
    q = oracle.modularity(rp, col, w, labels)
    assert q > oracle.modularity(rp, col, w, np.zeros(n, np.int32))
    assert q > oracle.modularity(rp, col, w, np.arange(n, dtype=np.int32))


def _quality(A2, k, two_m, labels, gamma):
    same = labels[:, None] == labels[None, :]
    return ((A2 - gamma * np.outer(k, k) / two_m) * same).sum()


@pytest.mark.parametrize("seed", range(6))
def test_partition_is_locally_optimal_and_connected(oracle_lib, seed):
    n = 60
    rp, col, w = _random_knn(n, 3, seed)
    gamma = [0.7, 1.0, 1.5][seed % 3]
    labels, C = oracle.leiden(rp, col, w, n, gamma)
    assert labels.min() == 0 and labels.max() == C - 1 and len(set(labels.tolist())) == C
    A = _dense(n, rp, col, w)
    A2 = A + np.diag(np.diag(A))
    k = A2.sum(1)
    two_m = k.sum()
    base = _quality(A2, k, two_m, labels, gamma)
    # no single node move to a neighbouring community raises the quality
    for v in range(n):
        for c in set(labels[np.nonzero(A[v])[0]].tolist()) - {labels[v]}:
            moved = labels.copy()
            moved[v] = c
            assert _quality(A2, k, two_m, moved, gamma) <= base + 1e-9 * abs(base) + 1e-12, (v, c)
    # every community induces a connected subgraph
    for c in range(C):
        members = np.nonzero(labels == c)[0]
        seen = {members[0]}
        stack = [members[0]]
        while stack:
            u = stack.pop()
            for x in np.nonzero(A[u])[0]:
                if labels[x] == c and x not in seen:
                    seen.add(x)
                    stack.append(x)
        assert len(seen) == len(members), f"community {c} is not connected"
    # and the result beats the trivial partitions
    q = oracle.modularity(rp, col, w, labels, gamma)
    assert q >= oracle.modularity(rp, col, w, np.arange(n, dtype=np.int32), gamma)
    assert q >= oracle.modularity(rp, col, w, np.zeros(n, np.int32), gamma)


def test_resolution_and_determinism(oracle_lib):
    n = 300
    rp, col, w = _random_knn(n, 6, 7)
    counts = [oracle.leiden(rp, col, w, n, g)[1] for g in (0.25, 1.0, 4.0)]
    assert counts[0] <= counts[1] <= counts[2]
    a, _ = oracle.leiden(rp, col, w, n, 1.0)
    b, _ = oracle.leiden(rp, col, w, n, 1.0)
    np.testing.assert_array_equal(a, b)


def test_edge_cases(oracle_lib):
    # no edges: every node alone; isolated nodes next to an edge
    rp = np.zeros(6, np.int64)
    labels, C = oracle.leiden(rp, np.zeros(0, np.int32), np.zeros(0, np.float32), 5)
    assert C == 5 and list(labels) == [0, 1, 2, 3, 4]
    rp, col, w = _csr(4, [(2, 1, 1.0)])
    labels, C = oracle.leiden(rp, col, w, 4)
    assert C == 3 and labels[1] == labels[2] and len({labels[0], labels[1], labels[3]}) == 3
    assert oracle.modularity(rp, col, w, labels) == pytest.approx(0.0, abs=1e-12)  # one edge inside: 1 - 1


def test_two_triangles_closed_form(oracle_lib):
    # two triangles {0,1,2} and {3,4,5} joined by the edge 2-3, unit weights:
    # m = 7; each triangle holds 3 edges and a degree sum of 7, so
    # Q = 2 * (3/7 - (7/14)^2) = 5/14 at gamma = 1, and at gamma:
    # Q = 6/7 - gamma / 2
    edges = [(1, 0, 1.0), (2, 0, 1.0), (2, 1, 1.0), (3, 2, 1.0), (4, 3, 1.0), (5, 3, 1.0), (5, 4, 1.0)]
    rp, col, w = _csr(6, edges)
    labels, C = oracle.leiden(rp, col, w, 6, 1.0)
    assert C == 2 and list(labels) == [0, 0, 0, 1, 1, 1]
    assert oracle.modularity(rp, col, w, labels) == pytest.approx(5 / 14, abs=1e-12)
    assert oracle.modularity(rp, col, w, labels, 0.5) == pytest.approx(6 / 7 - 0.25, abs=1e-12)
    # everything in one community: Q = 1 - gamma
    assert oracle.modularity(rp, col, w, np.zeros(6, np.int32)) == pytest.approx(0.0, abs=1e-12)
