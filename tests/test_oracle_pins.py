"""Pins of the CPU oracle against things other than itself.

Each test checks one oracle function against brute force on tiny inputs, a
library routine (torch softmax / scaled_dot_product_attention, numpy sorts
and means), a closed form, an invariant, or a hand-derived fixture in
tests/golden/.  The cases are chosen so that a dropped term, a wrong sign or
index, a flipped tie-break or a transposed operand fails at least one.

Source: "CommunityKV: Efficient Long-Context Decoding via Graph
Partitioning" -- Figure 1 caption steps (1)-(3), abstract, Table 1.
"""
import json
import math
import os

import numpy as np
import pytest
import torch

import oracle
from long_context_decode_ckv_b200 import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _sdpa64(q, K, V):
    """Library attention (torch SDPA, float64) of q [H][D] over all rows."""
    qt = torch.from_numpy(np.asarray(q, np.float64))[None, :, None, :]        # [1,H,1,D]
    kt = torch.from_numpy(np.asarray(K, np.float64))[None, None].expand(1, qt.shape[1], -1, -1)
    vt = torch.from_numpy(np.asarray(V, np.float64))[None, None].expand(1, qt.shape[1], -1, -1)
    return torch.nn.functional.scaled_dot_product_attention(qt, kt, vt)[0, :, 0, :].numpy()


def _probs64(q, K):
    """Library softmax (torch, float64) of q K^T / sqrt(D): [H][n]."""
    qt = torch.from_numpy(np.asarray(q, np.float64))
    kt = torch.from_numpy(np.asarray(K, np.float64))
    return torch.softmax(qt @ kt.T / math.sqrt(qt.shape[1]), dim=1).numpy()


def _f32(a):
    return synth.bf16_bits_to_f32(a) if a.dtype == np.uint16 else a.astype(np.float32)


# --------------------------------------------------------------- a2 select
def _select_brute(s, size, budget):
    """Largest k whose first k communities (score desc, id asc) fit the
    budget, searched from the top; at least one."""
    ids = sorted((c for c in range(len(s)) if size[c] > 0), key=lambda c: (-float(s[c]), c))
    for k in range(len(ids), 0, -1):
        if sum(int(size[c]) for c in ids[:k]) <= budget:
            return ids[:k]
    return ids[:1]


@pytest.mark.parametrize("seed", range(40))
def test_select_matches_brute_force(oracle_lib, seed):
    rng = np.random.default_rng(seed)
    n = int(rng.integers(1, 40))
    s = rng.integers(-3, 4, size=n).astype(np.float32)       # many exact ties
    if seed % 3 == 0:
        s = rng.standard_normal(n).astype(np.float32)
    size = rng.integers(0, 9, size=n).astype(np.int32)
    budget = int(rng.integers(0, 60))
    sel, _, _ = oracle.select(s, size, budget)
    assert list(sel) == _select_brute(s, size, budget)


def test_select_properties(oracle_lib):
    rng = np.random.default_rng(7)
    s = rng.standard_normal(300).astype(np.float32)
    size = rng.integers(1, 30, size=300).astype(np.int32)
    # budget covering everything keeps every non-empty community
    sel, lo, hi = oracle.select(s, size, int(size.sum()))
    assert sorted(sel) == list(range(300)) and math.isinf(lo)
    # a budget smaller than every community still keeps the best one
    sel, _, _ = oracle.select(s, size, 0)
    assert list(sel) == [int(np.argmax(s))]
    # kept communities outrank every dropped one, and the first dropped one
    # would overflow the budget
    sel, lo, _ = oracle.select(s, size, 700)
    kept = set(sel.tolist())
    drop = [c for c in range(300) if c not in kept]
    assert min(s[list(kept)]) >= max(s[drop])
    first_drop = max(drop, key=lambda c: (s[c], -c))
    assert size[list(kept)].sum() + size[first_drop] > 700
    assert lo == pytest.approx(abs(min(s[list(kept)]) - s[first_drop]) /
                               max(abs(min(s[list(kept)])), abs(s[first_drop])), rel=1e-6)
    # empty communities are never kept
    size[::2] = 0
    sel, _, _ = oracle.select(s, size, 10 ** 9)
    assert all(size[c] > 0 for c in sel)


# ---------------------------------------------------------------- a1 score
def test_score_matches_library_and_basis(oracle_lib):
    rng = np.random.default_rng(3)
    D, Nc, n = 128, 12, 200
    K = rng.standard_normal((n, D)).astype(np.float32)
    labels = rng.integers(0, Nc - 1, size=n).astype(np.int32)   # community Nc-1 stays empty
    g = oracle.Graph(Nc, D, n)
    g.init(n, 4, labels, K)
    q = rng.standard_normal((3, D)).astype(np.float32)
    s = oracle.score(g, q)
    mu = g.centroids().astype(np.float64)
    ref = (q.astype(np.float64).sum(0) @ mu.T).astype(np.float32)   # library matmul
    assert np.isneginf(s[Nc - 1])
    np.testing.assert_allclose(s[:Nc - 1], ref[:Nc - 1], rtol=1e-6, atol=1e-5)
    # basis queries pick out one centroid coordinate each
    for i in (0, 5, 127):
        e = np.zeros((1, D), np.float32)
        e[0, i] = 1.0
        np.testing.assert_array_equal(oracle.score(g, e)[:Nc - 1], g.centroids()[:Nc - 1, i])


# ------------------------------------------------------- a8 init / a6 update
def test_init_centroids_are_member_means(oracle_lib):
    w = synth.make_workload(synth.scaled(synth.TINY, n0=512, n_clusters=16, steps=0))
    K = w.K[0, 0]
    labels = w.labels[0]
    g = oracle.Graph(w.cfg.n_comm, 128, w.cfg.n_max)
    g.init(w.cfg.n0, 4, labels, K)
    size, mu, mem = g.sizes(), g.centroids(), g.members()
    assert size.sum() + 4 == w.cfg.n0                    # sinks are no community's
    assert not np.isin(np.arange(4), mem).any()
    k = 0
    for c in range(w.cfg.n_comm):
        m = mem[k:k + size[c]]
        k += size[c]
        assert np.all(np.diff(m) > 0)                      # ascending positions
        assert np.all(labels[m] == c)
        ref = K[m].astype(np.float64).mean(0).astype(np.float32)   # numpy mean
        np.testing.assert_allclose(mu[c], ref, rtol=2e-7, atol=1e-7)


def test_running_mean_stays_member_mean(oracle_lib):
    rng = np.random.default_rng(11)
    D, Nc, n0, steps = 128, 8, 64, 400
    K = (rng.standard_normal((n0 + steps, D)) * 3).astype(np.float32)
    labels = (np.arange(n0) % Nc).astype(np.int32)
    g = oracle.Graph(Nc, D, n0 + steps)
    g.init(n0, 4, labels, K)
    for t in range(n0, n0 + steps):
        before = g.centroids()
        c = int(rng.integers(0, Nc))
        g.update(c, t, K[t])
        after = g.centroids()
        changed = np.nonzero(np.any(before != after, axis=1))[0]
        assert set(changed.tolist()) <= {c}                # one O(d) update (Table 1)
    size, mu, mem = g.sizes(), g.centroids(), g.members()
    assert size.sum() + 4 == n0 + steps
    k = 0
    for c in range(Nc):
        m = mem[k:k + size[c]]
        k += size[c]
        ref = K[m].astype(np.float64).mean(0)
        np.testing.assert_allclose(mu[c], ref, rtol=1e-5, atol=1e-5)


# -------------------------------------------------------------- a3 attend
def test_attend_matches_sdpa_and_special_cases(oracle_lib):
    rng = np.random.default_rng(5)
    n, D, H = 97, 128, 4
    K = rng.standard_normal((n, D)).astype(np.float32)
    V = rng.standard_normal((n, D)).astype(np.float32)
    q = (rng.standard_normal((H, D)) * 2).astype(np.float32)
    rows = np.arange(n, dtype=np.int32)
    out, p, m, l = oracle.attend(q, K, V, rows)
    np.testing.assert_allclose(out, _sdpa64(q, K, V), rtol=0, atol=2e-6)
    np.testing.assert_allclose(p, _probs64(q, K), rtol=1e-12, atol=1e-15)
    np.testing.assert_allclose(p.sum(1), 1.0, rtol=1e-12)
    # row order does not matter (a set, not a sequence)
    perm = rng.permutation(n).astype(np.int32)
    out2, _, _, _ = oracle.attend(q, K, V, perm)
    np.testing.assert_allclose(out2, out, rtol=0, atol=1e-6)
    # a zero query averages the values
    out3, _, _, _ = oracle.attend(np.zeros((1, D), np.float32), K, V, rows[:10])
    np.testing.assert_allclose(out3[0], V[:10].astype(np.float64).mean(0), rtol=0, atol=1e-6)
    # bf16 path widens exactly
    Kb, Vb, qb = synth.to_bf16_bits(K), synth.to_bf16_bits(V), synth.to_bf16_bits(q)
    out4, _, _, _ = oracle.attend(qb, Kb, Vb, rows)
    np.testing.assert_allclose(out4, _sdpa64(_f32(qb), _f32(Kb), _f32(Vb)), rtol=0, atol=2e-6)


# ---------------------------------------------------------------- a4 top-k
@pytest.mark.parametrize("seed", range(30))
def test_topk_matches_lexsort(oracle_lib, seed):
    rng = np.random.default_rng(100 + seed)
    R = int(rng.integers(0, 50))
    w = (rng.integers(0, 6, size=R) / 8).astype(np.float32)     # heavy ties
    tok = rng.permutation(1000)[:R].astype(np.int32)
    kappa = int(rng.integers(1, 12))
    idx, _ = oracle.topk(w, tok, kappa)
    ref = np.lexsort((tok, -w))[:kappa]                       # library sort
    assert list(idx) == list(ref)


# ------------------------------------------------------------------ a5 vote
def test_vote_hand_tables(oracle_lib):
    cases = json.load(open(os.path.join(GOLDEN, "vote_cases.json")))["cases"]
    for c in cases:
        winner, _ = oracle.vote(np.array(c["comm"], np.int32), np.array(c["w"], np.float32))
        assert winner == c["winner"], c["why"]


# --------------------------------------------------------- golden decode
def _golden_graph(case, common):
    D, n0 = common["head_dim"], common["n0"]
    n = common["n"]
    K = np.zeros((n, D), np.float32)
    V = np.zeros((n, D), np.float32)
    K[:, 0], K[:, 1], V[:, 0] = case["k_dim0"], case["k_dim1"], case["v_dim0"]
    g = oracle.Graph(case["n_comm"], D, n)
    g.init(n0, common["n_sinks"], np.array(common["labels"], np.int32), K)
    q = np.zeros((1, D), np.float32)
    q[0, 0] = case["q_dim0"]
    return g, q, K, V


def test_golden_decode_cases(oracle_lib):
    data = json.load(open(os.path.join(GOLDEN, "decode_cases.json")))
    common = data["common"]
    for case in data["cases"]:
        g, q, K, V = _golden_graph(case, common)
        e = case["expect"]
        s = oracle.score(g, q)
        exp_s = [-np.inf if v == "-inf" else v for v in e["scores"]]
        np.testing.assert_array_equal(s, np.array(exp_s, np.float32))
        r = oracle.decode_step(g, q, K, V, common["n"], common["n_sinks"], common["kappa"],
                               case["budget"])
        assert list(r.sel) == e["selected"], case["why"]
        assert r.T == e["T"]
        assert list(r.edge_col) == e["edges"], case["why"]
        assert r.assigned == e["assigned"]
        if "out_dim0" in e:
            assert r.out[0, 0] == e["out_dim0"]
            assert np.all(r.out[0, 1:] == 0)
        if "edge_w" in e:
            np.testing.assert_allclose(r.edge_w, e["edge_w"], rtol=1e-7)
        if "cut_gap_lo" in e:
            assert r.cut_gap_lo == pytest.approx(e["cut_gap_lo"])
        c = e["assigned"]
        np.testing.assert_array_equal(g.centroids()[c, :2], e[f"new_centroid_c{c}"])
        assert g.sizes()[c] == e[f"new_size_c{c}"]


# ------------------------------------------------- whole step, dense special case
@pytest.mark.parametrize("mode", [synth.PER_HEAD, synth.QUERY_GROUP])
def test_step_with_full_budget_is_dense_attention(oracle_lib, mode):
    """Budget >= every member: the step is dense causal attention of the new
    token, and its edges are the top-kappa of the dense probabilities."""
    cfg = synth.scaled(synth.LLAMA, batch=1, n_q_heads=8, n_kv_heads=2, n0=384, steps=3,
                       n_clusters=24, budget=10 ** 6, mode=mode, bf16=True)
    w = synth.make_workload(cfg)
    for g_id in (0, cfg.n_graphs - 1):
        b, kvh, heads = cfg.graph_heads(g_id)
        K, V = w.K[b, kvh], w.V[b, kvh]
        g = oracle.Graph(cfg.n_comm, 128, cfg.n_max)
        g.init(cfg.n0, cfg.n_sinks, w.labels[g_id], K)
        for step in range(cfg.steps):
            n = cfg.n0 + step + 1
            q = np.ascontiguousarray(w.q[step, b, heads])
            r = oracle.decode_step(g, q, K, V, n, cfg.n_sinks, cfg.kappa, cfg.budget)
            assert r.T == n - 1 - cfg.n_sinks
            np.testing.assert_allclose(r.out, _sdpa64(_f32(q), _f32(K[:n]), _f32(V[:n])),
                                       rtol=0, atol=5e-6)
            p = _probs64(_f32(q), _f32(K[:n])).sum(0)          # summed over the graph's heads
            cand = np.arange(cfg.n_sinks, n - 1)
            wc = p[cand].astype(np.float32)
            ref = cand[np.lexsort((cand, -wc))[:cfg.kappa]]
            assert list(r.edge_col) == list(ref)
            np.testing.assert_allclose(r.edge_w, wc[np.lexsort((cand, -wc))[:cfg.kappa]],
                                       rtol=1e-6)
            assert not np.isin(r.edge_col, list(range(cfg.n_sinks)) + [n - 1]).any()


def test_step_assigns_one_selected_community(oracle_lib):
    cfg = synth.scaled(synth.TINY, n0=1024, n_clusters=32, steps=12, budget=128)
    w = synth.make_workload(cfg)
    K, V = w.K[0, 0], w.V[0, 0]
    g = oracle.Graph(cfg.n_comm, 128, cfg.n_max)
    g.init(cfg.n0, cfg.n_sinks, w.labels[0], K)
    for step in range(cfg.steps):
        n = cfg.n0 + step + 1
        before_mu, before_size = g.centroids(), g.sizes()
        r = oracle.decode_step(g, w.q[step, 0], K, V, n, cfg.n_sinks, cfg.kappa, cfg.budget)
        assert r.assigned in set(r.sel.tolist())
        assert before_size[r.sel].sum() <= cfg.budget or r.C == 1
        after_mu, after_size = g.centroids(), g.sizes()
        diff = np.nonzero(np.any(before_mu != after_mu, axis=1))[0]
        assert set(diff.tolist()) <= {r.assigned}
        assert after_size.sum() + cfg.n_sinks == n
        assert after_size[r.assigned] == before_size[r.assigned] + 1
        assert set(r.edge_comm.tolist()) <= set(r.sel.tolist())
        assert np.all(np.diff(r.edge_w) <= 0)
    with pytest.raises(ValueError):   # the next step must be n + 1
        oracle.decode_step(g, w.q[0, 0], K, V, cfg.n_max + 5, 4, 8, 128)


# ------------------------------------------------------------ a7 prefill
def test_prefill_golden(oracle_lib):
    c = json.load(open(os.path.join(GOLDEN, "prefill_case.json")))
    n = len(c["k_dim0"])
    K = np.zeros((n, c["head_dim"]), np.float32)
    K[:, 0] = c["k_dim0"]
    Q = np.zeros_like(K)
    Q[:, 0] = c["q_dim0"]
    col, _, deg, _ = oracle.prefill_rows(Q, K, np.arange(n), c["n_sinks"], c["kappa"])
    for i, e in enumerate(c["expect_edges"]):
        assert deg[i] == len(e) and list(col[i, :deg[i]]) == e, c["why"]


def test_prefill_matches_library_softmax(oracle_lib):
    P = synth.PREFILL
    Q, K = synth.make_prefill(P, n=96)
    S, kap = P.n_sinks, P.kappa
    for h in (0, 7):
        Qf, Kf = _f32(Q[h]).astype(np.float64), _f32(K[h]).astype(np.float64)
        z = torch.from_numpy(Qf @ Kf.T / math.sqrt(128))
        z = z.masked_fill(torch.triu(torch.ones(96, 96, dtype=torch.bool), 1), -math.inf)
        prob = torch.softmax(z, dim=1).numpy()
        zf = z.numpy().astype(np.float32)
        col, w, deg, _ = oracle.prefill_rows(Q[h], K[h], np.arange(96), S, kap)
        for i in range(96):
            cand = np.arange(S, i)
            order = cand[np.lexsort((cand, -zf[i, cand]))][:kap]
            assert deg[i] == min(kap, max(0, i - S))
            assert list(col[i, :deg[i]]) == list(order)
            np.testing.assert_allclose(w[i, :deg[i]], prob[i, order], rtol=1e-6, atol=1e-12)
            assert w[i, :deg[i]].sum() <= 1.0 + 1e-6


def test_row_ptr_closed_form(oracle_lib):
    for S, kap in ((4, 8), (1, 2), (0, 3)):
        for i in (0, 1, S, S + 1, S + kap, S + kap + 1, 1000):
            # closed form: rows S+1 .. S+kappa contribute 1..kappa, later rows kappa each
            a = max(0, min(i, S + kap + 1) - S - 1)          # rows with degree < kappa
            closed = a * (a + 1) // 2 + max(0, i - (S + kap + 1)) * kap
            assert oracle.row_ptr(i, S, kap) == closed


# ------------------------------------------------ NEXT f3 attention-mass recall
def test_dense_stats_match_library_logsumexp(oracle_lib):
    rng = np.random.default_rng(11)
    n, D, H = 131, 128, 3
    K = rng.standard_normal((n, D)).astype(np.float32)
    q = (rng.standard_normal((H, D)) * 3).astype(np.float32)
    for cut in (1, 7, n):
        m, l = oracle.dense_stats(q, K, cut)
        z = torch.from_numpy(q.astype(np.float64)) @ torch.from_numpy(K[:cut].astype(np.float64)).T
        z = z / math.sqrt(D)
        np.testing.assert_allclose(m, z.max(1).values.numpy(), rtol=0, atol=1e-12)
        np.testing.assert_allclose(m + np.log(l), torch.logsumexp(z, 1).numpy(), rtol=0, atol=1e-12)
    # identical keys: m is the single logit, l counts the rows
    Kc = np.tile(K[:1], (9, 1))
    m, l = oracle.dense_stats(q, Kc, 9)
    np.testing.assert_allclose(m, q.astype(np.float64) @ K[0].astype(np.float64) / math.sqrt(D), atol=1e-12)
    np.testing.assert_allclose(l, 9.0, rtol=1e-15)
    # bf16 operands widen exactly
    qb, Kb = synth.to_bf16_bits(q), synth.to_bf16_bits(K)
    mb, lb = oracle.dense_stats(qb, Kb, n)
    m2, l2 = oracle.dense_stats(_f32(qb), _f32(Kb), n)
    np.testing.assert_array_equal(mb, m2)
    np.testing.assert_array_equal(lb, l2)


@pytest.mark.parametrize("budget", [40, 160, 10 ** 6])
def test_recall_is_dense_mass_of_attended_rows(oracle_lib, budget):
    cfg = synth.scaled(synth.TINY, n0=512, n_clusters=24, steps=4, budget=budget, bf16=True)
    w = synth.make_workload(cfg)
    K, V = w.K[0, 0], w.V[0, 0]
    g = oracle.Graph(cfg.n_comm, 128, cfg.n_max)
    g.init(cfg.n0, cfg.n_sinks, w.labels[0], K)
    for step in range(cfg.steps):
        n = cfg.n0 + step + 1
        q = np.ascontiguousarray(w.q[step, 0])                        # [H][D], one head
        sizes_before, mem_before = g.sizes(), g.members()           # state before the step
        r = oracle.decode_step(g, q, K, V, n, cfg.n_sinks, cfg.kappa, cfg.budget)
        g_rows = _attended_rows_from(sizes_before, mem_before, r.sel, n, cfg.n_sinks)
        rec = oracle.recall(r.m, r.l, *oracle.dense_stats(q, K, n))
        ref = _probs64(_f32(q), _f32(K[:n]))[:, g_rows].sum(1)      # brute force, library softmax
        np.testing.assert_allclose(rec, ref, rtol=1e-12, atol=0)
        assert np.all(rec <= 1.0 + 1e-12) and np.all(rec > 0)
        if budget >= n:
            assert len(g_rows) == n
            np.testing.assert_allclose(rec, 1.0, rtol=1e-12)


def _attended_rows_from(sizes, mem, sel, n, n_sinks):
    start = np.concatenate([[0], np.cumsum(sizes)])
    rows = list(range(n_sinks)) + [n - 1]
    for c in sel:
        rows += mem[start[c]:start[c + 1]].tolist()
    assert len(set(rows)) == len(rows)
    return np.array(sorted(rows), np.int64)


def test_recall_grows_with_budget(oracle_lib):
    """A larger budget keeps a longer prefix of the same order, so the
    attended set only grows and recall never falls."""
    cfg0 = synth.scaled(synth.TINY, n0=600, n_clusters=30, steps=1, budget=1, bf16=True)
    w = synth.make_workload(cfg0)
    K, V = w.K[0, 0], w.V[0, 0]
    q = np.ascontiguousarray(w.q[0, 0])
    n = cfg0.n0 + 1
    den = oracle.dense_stats(q, K, n)
    prev = None
    for budget in (1, 20, 50, 100, 200, 400, 600):
        g = oracle.Graph(cfg0.n_comm, 128, cfg0.n_max)
        g.init(cfg0.n0, cfg0.n_sinks, w.labels[0], K)
        r = oracle.decode_step(g, q, K, V, n, cfg0.n_sinks, cfg0.kappa, budget)
        rec = oracle.recall(r.m, r.l, *den)
        if prev is not None:
            assert np.all(rec >= prev - 1e-12)
        prev = rec
    np.testing.assert_allclose(prev, 1.0, rtol=1e-12)


# ------------------------------------- NEXT f2 query-group aggregated prefill
def _grouped_brute(Q, K, S, kap):
    """Library softmax per head (torch, float64, causal), summed over the
    heads, rounded to float32; lexsort by (w desc, j asc) per row."""
    nh, n, D = Q.shape
    Qt = torch.from_numpy(_f32(Q).astype(np.float64))
    Kt = torch.from_numpy(_f32(K).astype(np.float64))
    z = Qt @ Kt.T / math.sqrt(D)                                          # [nh][n][n]
    z = z.masked_fill(torch.triu(torch.ones(n, n, dtype=torch.bool), 1), -math.inf)
    wsum = torch.softmax(z, dim=2).sum(0).numpy().astype(np.float32)      # [n][n]
    out = []
    for i in range(n):
        cand = np.arange(S, i)
        order = cand[np.lexsort((cand, -wsum[i, cand]))][:kap]
        out.append((order, wsum[i, order]))
    return out


@pytest.mark.parametrize("nh,bf16", [(1, False), (2, True), (4, True), (4, False)])
def test_grouped_prefill_matches_library_softmax(oracle_lib, nh, bf16):
    rng = np.random.default_rng(40 + nh)
    n, D, S, kap = 70, 128, 4, 8
    Q = (rng.standard_normal((nh, n, D)) * 1.5).astype(np.float32)
    K = rng.standard_normal((n, D)).astype(np.float32)
    if bf16:
        Q, K = synth.to_bf16_bits(Q), synth.to_bf16_bits(K)
    col, w, deg, _ = oracle.prefill_rows_grouped(Q, K, np.arange(n), S, kap)
    ref = _grouped_brute(Q, K, S, kap)
    for i in range(n):
        order, wr = ref[i]
        assert deg[i] == min(kap, max(0, i - S))
        assert list(col[i, :deg[i]]) == list(order), i
        np.testing.assert_allclose(w[i, :deg[i]], wr, rtol=1e-6, atol=0)
        assert w[i, :deg[i]].sum() <= nh * (1 + 1e-6)


def test_grouped_prefill_special_cases(oracle_lib):
    rng = np.random.default_rng(9)
    n, D, S, kap = 90, 128, 3, 6
    q = (rng.standard_normal((n, D)) * 2).astype(np.float32)
    K = rng.standard_normal((n, D)).astype(np.float32)
    rows = np.arange(n)
    # one head: the per-head prefill graph (weights are that head's p)
    c1, w1, d1, g1 = oracle.prefill_rows(q, K, rows, S, kap)
    cg, wg, dg, _ = oracle.prefill_rows_grouped(q[None], K, rows, S, kap)
    np.testing.assert_array_equal(dg, d1)
    for i in range(n):
        if g1[i] > 1e-5:                      # no near-tie at the cutoff
            assert set(cg[i, :dg[i]].tolist()) == set(c1[i, :d1[i]].tolist())
    np.testing.assert_allclose(np.sort(wg, 1), np.sort(w1, 1), rtol=1e-6)
    # the same head twice: the same edges, every weight doubled
    c2, w2, d2, _ = oracle.prefill_rows_grouped(np.stack([q, q]), K, rows, S, kap)
    np.testing.assert_array_equal(c2, cg)
    np.testing.assert_allclose(w2, 2 * wg, rtol=1e-6)
