"""Refresh mechanics (ckv_set_token_graph, ckv_refresh, ckv_graph_modularity)
on the GPU against the oracle.

"CommunityKV: Efficient Long-Context Decoding via Graph Partitioning",
Tables 8-9 (periodic re-partitioning, "refresh", against the incremental
update) and Figure 3 (left, the modularity of the partition over
generation).  Mechanics only: the token graph is the prefill graph plus the
decode-time edges; a refresh re-runs Leiden on it and re-initialises the
communities; decoding then continues in lockstep with the oracle.
"""
import numpy as np
import pytest

import oracle
import long_context_decode_ckv_b200 as ckv
from long_context_decode_ckv_b200 import build as ckv_build
from long_context_decode_ckv_b200 import state as ckv_state
from long_context_decode_ckv_b200 import synth
from tests.conftest import gpu_available
from tests.lockstep import Lockstep

pytestmark = [pytest.mark.gpu,
              pytest.mark.skipif(not gpu_available(), reason="needs a CUDA device")]


@pytest.fixture(scope="module", autouse=True)
def _built():
    ckv_build.build()


def _prefill_graph(K0, S, kap):
    """Prefill graph of the keys over themselves (queries = keys: the
    workload carries no prefill queries) for one KV head: host CSR."""
    import torch
    n = K0.shape[0]
    dev = torch.device("cuda", 0)
    k = torch.from_numpy(np.ascontiguousarray(K0)).view(torch.bfloat16).to(dev)[None]
    E = int(np.clip(np.arange(n) - S, 0, kap).sum())
    rp = torch.empty((1, n + 1), dtype=torch.int64, device=dev)
    col = torch.empty((1, E), dtype=torch.int32, device=dev)
    w = torch.empty((1, E), dtype=torch.float32, device=dev)
    ckv.ckv_build_graph(1, n, 128, S, kap, ckv.CKV_BF16, k, k, rp, col, w)
    torch.cuda.synchronize()
    return rp[0].cpu().numpy(), col[0].cpu().numpy(), w[0].cpu().numpy()


def _combined(rp, col, w, st: ckv_state.State, g):
    """Token graph of graph g: the prefill rows, then its decode-time rows."""
    rows = [(col[rp[i]:rp[i + 1]], w[rp[i]:rp[i + 1]]) for i in range(len(rp) - 1)]
    for r in range(st.deg.shape[1]):
        d = st.deg[g, r]
        rows.append((st.col[g, r, :d], st.w[g, r, :d]))
    nrp = np.concatenate([[0], np.cumsum([len(c) for c, _ in rows])]).astype(np.int64)
    ncol = np.concatenate([c for c, _ in rows]).astype(np.int32)
    nw = np.concatenate([x for _, x in rows]).astype(np.float32)
    return nrp, ncol, nw


def _labels_of(st: ckv_state.State, g, n, S):
    lab = np.full(n, st.sizes.shape[1], np.int32)           # sinks: one extra label
    start = np.concatenate([[0], np.cumsum(st.sizes[g])])
    for c in range(st.sizes.shape[1]):
        lab[st.members[g][start[c]:start[c + 1]]] = c
    return lab


def _setup(steps=24):
    cfg = synth.scaled(synth.LLAMA, batch=1, n_q_heads=2, n_kv_heads=1, n0=1024, n_clusters=32, steps=steps,
                       budget=160)
    wl = synth.make_workload(cfg)
    S, kap = cfg.n_sinks, cfg.kappa
    rp, col, w = _prefill_graph(wl.K[0, 0, :cfg.n0], S, kap)
    labels = np.empty(cfg.n0, np.int32)
    C = ckv.ckv_leiden(cfg.n0, rp, col, w, 1.0, labels)
    assert C <= cfg.n_comm
    for g in range(cfg.n_graphs):
        wl.labels[g] = labels
    ls = Lockstep(wl)
    G = cfg.n_graphs
    ckv.ckv_set_token_graph(ls.ctx, np.tile(rp, (G, 1)), np.tile(col, (G, 1)), np.tile(w, (G, 1)), cfg.n0)
    return cfg, wl, ls, (rp, col, w)


def test_refresh_is_leiden_on_the_token_graph_and_decoding_continues():
    cfg, wl, ls, (rp, col, w) = _setup()
    try:
        for i in range(12):
            ls.step(i)
        n = ls.n
        before = ckv_state.parse(ckv.ckv_export_state(ls.ctx))
        counts = np.zeros(cfg.n_graphs, np.int32)
        ckv.ckv_refresh(ls.ctx, ls.K, 1.0, counts)
        after = ckv_state.parse(ckv.ckv_export_state(ls.ctx))
        assert after.n_tok == n and after.deg.shape[1] == 0
        nc = after.sizes.shape[1]
        assert nc == counts.max()
        K = wl.K[0, 0]
        for g in range(cfg.n_graphs):
            trp, tcol, tw = _combined(rp, col, w, before, g)
            lab = np.empty(n, np.int32)
            C = ckv.ckv_leiden(n, trp, tcol, tw, 1.0, lab)
            ref, Cr = oracle.leiden(trp, tcol, tw, n, 1.0)
            assert C == Cr == counts[g]
            np.testing.assert_array_equal(lab, ref)
            # the new communities: Leiden's labels, centroids = member means (oracle init)
            o = oracle.Graph(nc, 128, cfg.n_max)
            o.init(n, cfg.n_sinks, lab, K)
            np.testing.assert_array_equal(after.sizes[g], o.sizes())
            np.testing.assert_array_equal(after.members[g], o.members())
            assert np.array_equal(after.centroids[g].view(np.uint32), o.centroids().view(np.uint32))
            ls.og[g] = o
            ls.oracle_edges[g] = []
        for i in range(12, cfg.steps):                        # decoding continues from the refreshed state
            ls.step(i)
        ls.compare_state()
    finally:
        ls.close()


def test_graph_modularity_matches_oracle():
    cfg, wl, ls, (rp, col, w) = _setup(steps=10)
    try:
        q0 = np.zeros(cfg.n_graphs)
        ckv.ckv_graph_modularity(ls.ctx, 1.0, q0)
        for i in range(10):
            ls.step(i)
        q = np.zeros(cfg.n_graphs)
        ckv.ckv_graph_modularity(ls.ctx, 1.0, q)
        st = ckv_state.parse(ckv.ckv_export_state(ls.ctx))
        for g in range(cfg.n_graphs):
            trp, tcol, tw = _combined(rp, col, w, st, g)
            ref = oracle.modularity(trp, tcol, tw, _labels_of(st, g, ls.n, cfg.n_sinks))
            assert q[g] == pytest.approx(ref, rel=1e-9)
            assert 0.2 < q[g] < 1.0 and abs(q[g] - q0[g]) < 0.1   # the incremental update keeps Q
    finally:
        ls.close()


def test_refresh_call_order_checked():
    cfg = synth.scaled(synth.TINY, n0=256, n_clusters=8, steps=4, bf16=True)
    wl = synth.make_workload(cfg)
    ls = Lockstep(wl)
    try:
        q = np.zeros(1)
        for fn in (lambda: ckv.ckv_refresh(ls.ctx, ls.K, 1.0),                 # no token graph registered
                   lambda: ckv.ckv_graph_modularity(ls.ctx, 1.0, q)):
            with pytest.raises(ckv.CkvError) as e:
                fn()
            assert e.value.status == ckv.CKV_ERR_STATE
        ls.step(0)
        rp = np.zeros((1, ls.n + 1), np.int64)
        with pytest.raises(ckv.CkvError) as e:                                # not right after init
            ckv.ckv_set_token_graph(ls.ctx, rp, np.zeros((1, 1), np.int32), np.zeros((1, 1), np.float32), ls.n)
        assert e.value.status == ckv.CKV_ERR_STATE
    finally:
        ls.close()
