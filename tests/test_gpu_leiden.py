"""GPU modularity (ckv_modularity) against the oracle's, and the pages'
pipeline end to end: prefill graph on the GPU (ckv_build_graph) -> Leiden on
the host (ckv_leiden) -> communities initialised from its labels
(ckv_init_communities) -> decode steps.

"CommunityKV: Efficient Long-Context Decoding via Graph Partitioning",
Figure 1 caption steps (1)-(3), Figure 3 (left).  Modularity: double on both
sides, the GPU's atomic sums in any order: relative 1e-9.
"""
import numpy as np
import pytest

import oracle
import long_context_decode_ckv_b200 as ckv
from long_context_decode_ckv_b200 import build as ckv_build
from long_context_decode_ckv_b200 import synth
from tests.conftest import gpu_available
from tests.lockstep import Lockstep
from tests.test_oracle_leiden import _random_knn

pytestmark = [pytest.mark.gpu,
              pytest.mark.skipif(not gpu_available(), reason="needs a CUDA device")]

Q_RTOL = 1e-9


@pytest.fixture(scope="module", autouse=True)
def _built():
    ckv_build.build()


def _gpu_modularity(rp, col, w, labels, nc, gamma=1.0):
    import torch
    dev = torch.device("cuda", 0)
    t = lambda a, dt: torch.from_numpy(np.ascontiguousarray(a, dt)).to(dev)
    ws = torch.empty(ckv.ckv_modularity_workspace(nc), dtype=torch.uint8, device=dev)
    return ckv.ckv_modularity(len(rp) - 1, t(rp, np.int64), t(col, np.int32), t(w, np.float32),
                              t(labels, np.int32), nc, gamma, ws)


@pytest.mark.parametrize("seed", range(4))
def test_modularity_matches_oracle(seed):
    n = [100, 1000, 5000, 20000][seed]
    rp, col, w = _random_knn(n, 8, seed)
    rng = np.random.default_rng(seed)
    for gamma in (0.5, 1.0):
        for labels in (rng.integers(0, 37, n).astype(np.int32), np.arange(n, dtype=np.int32)):
            nc = int(labels.max()) + 1
            q = _gpu_modularity(rp, col, w, labels, nc, gamma)
            assert q == pytest.approx(oracle.modularity(rp, col, w, labels, gamma), rel=Q_RTOL, abs=1e-12)


def test_modularity_rejects_bad_labels():
    rp, col, w = _random_knn(50, 3, 1)
    labels = np.zeros(50, np.int32)
    labels[7] = 9                                           # outside [0, 4)
    with pytest.raises(ckv.CkvError) as e:
        _gpu_modularity(rp, col, w, labels, 4)
    assert e.value.status == ckv.CKV_ERR_INVALID_ARG


def test_prefill_leiden_modularity_pipeline():
    import torch
    P = synth.PREFILL
    n, S, kap = 4096, P.n_sinks, P.kappa
    Q, K = synth.make_prefill(P, n=n)
    dev = torch.device("cuda", 0)
    q = torch.from_numpy(Q[:2]).view(torch.bfloat16).to(dev)
    k = torch.from_numpy(K[:2]).view(torch.bfloat16).to(dev)
    E = int(np.clip(np.arange(n) - S, 0, kap).sum())
    rp = torch.empty((2, n + 1), dtype=torch.int64, device=dev)
    col = torch.empty((2, E), dtype=torch.int32, device=dev)
    w = torch.empty((2, E), dtype=torch.float32, device=dev)
    ckv.ckv_build_graph(2, n, 128, S, kap, ckv.CKV_BF16, q, k, rp, col, w)
    torch.cuda.synchronize()
    for h in range(2):
        rph, colh, wh = rp[h].cpu().numpy(), col[h].cpu().numpy(), w[h].cpu().numpy()
        labels = np.empty(n, np.int32)
        C = ckv.ckv_leiden(n, rph, colh, wh, 1.0, labels)
        ref, Cr = oracle.leiden(rph, colh, wh, n, 1.0)          # the oracle on the GPU's graph
        assert C == Cr
        np.testing.assert_array_equal(labels, ref)
        qg = ckv.ckv_modularity(n, rp[h], col[h], w[h], torch.from_numpy(labels).to(dev), C, 1.0,
                                torch.empty(ckv.ckv_modularity_workspace(C), dtype=torch.uint8, device=dev))
        assert qg == pytest.approx(oracle.modularity(rph, colh, wh, labels), rel=Q_RTOL)
        assert 0.3 < qg < 1.0
        print(f"head {h}: n {n}, {C} communities, modularity {qg:.4f}")


def test_leiden_labels_drive_the_decode_step():
    # Figure 1 end to end: the communities of the decode steps come from Leiden
    # on the prefill graph of the same keys (one graph, per-head mode)
    import torch
    cfg = synth.scaled(synth.TINY, n0=1024, n_clusters=32, steps=6, budget=160, bf16=True)
    wl = synth.make_workload(cfg)
    dev = torch.device("cuda", 0)
    K = torch.from_numpy(np.ascontiguousarray(wl.K[0, 0, :cfg.n0])).view(torch.bfloat16).to(dev)[None]
    Qp = K.clone()                                           # prefill queries: the keys themselves
    n, S, kap = cfg.n0, cfg.n_sinks, cfg.kappa
    E = int(np.clip(np.arange(n) - S, 0, kap).sum())
    rp = torch.empty((1, n + 1), dtype=torch.int64, device=dev)
    col = torch.empty((1, E), dtype=torch.int32, device=dev)
    w = torch.empty((1, E), dtype=torch.float32, device=dev)
    ckv.ckv_build_graph(1, n, 128, S, kap, ckv.CKV_BF16, Qp, K, rp, col, w)
    torch.cuda.synchronize()
    labels = np.empty(n, np.int32)
    C = ckv.ckv_leiden(n, rp[0].cpu().numpy(), col[0].cpu().numpy(), w[0].cpu().numpy(), 1.0, labels)
    assert 1 < C <= cfg.n_comm
    wl.labels[0] = labels                                   # the partition the steps start from
    ls = Lockstep(wl)
    try:
        for i in range(cfg.steps):
            ls.step(i)
        ls.compare_state()
    finally:
        ls.close()
