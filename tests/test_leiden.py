"""The library's host Leiden (ckv_leiden, native C++) against the CPU oracle's
(leiden_oracle.c): the same deterministic algorithm, so the labels must be
identical, on random top-kappa graphs, tie-heavy graphs (equal weights) and
prefill graphs of the synthetic workload computed by the oracle.

"CommunityKV: Efficient Long-Context Decoding via Graph Partitioning",
Figure 1 caption step (2).  Host code only: no GPU is needed.
"""
import numpy as np
import pytest

import oracle
import long_context_decode_ckv_b200 as ckv
from long_context_decode_ckv_b200 import build as ckv_build
from long_context_decode_ckv_b200 import synth
from tests.test_oracle_leiden import _csr, _random_knn


@pytest.fixture(scope="module", autouse=True)
def _built():
    ckv_build.build()


def _lib_leiden(rp, col, w, n, gamma):
    labels = np.full(n, -1, np.int32)
    C = ckv.ckv_leiden(n, np.ascontiguousarray(rp, np.int64), np.ascontiguousarray(col, np.int32),
                       np.ascontiguousarray(w, np.float32), gamma, labels)
    return labels, C


@pytest.mark.parametrize("gamma", [0.5, 1.0, 2.0])
@pytest.mark.parametrize("seed", range(6))
def test_same_labels_as_oracle_on_random_graphs(oracle_lib, seed, gamma):
    n = [50, 200, 700][seed % 3]
    rp, col, w = _random_knn(n, 1 + seed % 8, seed)
    lab, C = _lib_leiden(rp, col, w, n, gamma)
    ref, Cr = oracle.leiden(rp, col, w, n, gamma)
    assert C == Cr
    np.testing.assert_array_equal(lab, ref)


@pytest.mark.parametrize("seed", range(3))
def test_same_labels_on_larger_graphs(oracle_lib, seed):
    # coarse levels whose nodes have hundreds of neighbours (the adjacency
    # merge's sorted path as well as its insertion-sort path)
    n = [3000, 6000, 12000][seed]
    rp, col, w = _random_knn(n, 8, 100 + seed)
    for gamma in (0.7, 1.0):
        lab, C = _lib_leiden(rp, col, w, n, gamma)
        ref, Cr = oracle.leiden(rp, col, w, n, gamma)
        assert C == Cr
        np.testing.assert_array_equal(lab, ref)


def test_same_labels_on_equal_weights(oracle_lib):
    # every weight 1: gains tie everywhere, so the tie rules decide
    rng = np.random.default_rng(3)
    n = 400
    edges = [(i, int(j), 1.0) for i in range(1, n) for j in rng.choice(i, size=min(3, i), replace=False)]
    rp, col, w = _csr(n, edges)
    for gamma in (0.8, 1.0, 1.3):
        lab, C = _lib_leiden(rp, col, w, n, gamma)
        ref, Cr = oracle.leiden(rp, col, w, n, gamma)
        assert C == Cr
        np.testing.assert_array_equal(lab, ref)


@pytest.mark.slow
def test_same_labels_on_prefill_graph(oracle_lib):
    # the prefill top-kappa graph of one head of the synthetic workload
    P = synth.PREFILL
    n = 1500
    Q, K = synth.make_prefill(P, n=n)
    col, w, deg, _ = oracle.prefill_rows(Q[0], K[0], np.arange(n), P.n_sinks, P.kappa)
    rp = np.concatenate([[0], np.cumsum(deg)]).astype(np.int64)
    cc = np.concatenate([col[i, :deg[i]] for i in range(n)]).astype(np.int32)
    ww = np.concatenate([w[i, :deg[i]] for i in range(n)]).astype(np.float32)
    lab, C = _lib_leiden(rp, cc, ww, n, 1.0)
    ref, Cr = oracle.leiden(rp, cc, ww, n, 1.0)
    assert C == Cr
    np.testing.assert_array_equal(lab, ref)
    assert oracle.modularity(rp, cc, ww, lab) > 0.3


def test_edge_cases_match_oracle(oracle_lib):
    empty = (np.zeros(0, np.int32), np.zeros(0, np.float32))
    cases = [
        (1, np.array([0, 0], np.int64), *empty),                                  # one node
        (5, np.zeros(6, np.int64), *empty),                                       # no edges
        (5, np.array([0, 1, 1, 1, 2, 2], np.int64), np.array([3, 0], np.int32),  # isolated nodes
         np.array([1.0, 2.0], np.float32)),
        (2, np.array([0, 1, 2], np.int64), np.array([0, 0], np.int32),           # a self-loop
         np.array([1.0, 1.0], np.float32)),
        (2, np.array([0, 1, 2], np.int64), np.array([1, 0], np.int32),           # zero weights
         np.array([0.0, 0.0], np.float32)),
    ]
    expect = {0: [0], 1: [0, 1, 2, 3, 4], 2: [0, 1, 2, 0, 3], 4: [0, 1]}       # hand-derived
    for k, (n, rp, col, w) in enumerate(cases):
        lab, C = _lib_leiden(rp, col, w, n, 1.0)
        ref, Cr = oracle.leiden(rp, col, w, n, 1.0)
        assert C == Cr
        np.testing.assert_array_equal(lab, ref)
        if k in expect:
            assert list(lab) == expect[k] and C == max(expect[k]) + 1


def test_arguments_checked():
    rp = np.array([0, 1, 1], np.int64)
    lab = np.zeros(2, np.int32)
    for args in ((2, rp, np.array([5], np.int32), np.array([1.0], np.float32), 1.0),      # column out of range
                 (2, rp, np.array([0], np.int32), np.array([-1.0], np.float32), 1.0),     # negative weight
                 (2, rp, np.array([0], np.int32), np.array([1.0], np.float32), 0.0),      # gamma
                 (2, np.array([0, 2, 1], np.int64), np.array([0, 1], np.int32),
                  np.array([1.0, 1.0], np.float32), 1.0),                                 # row_ptr not monotone
                 (2, rp, np.array([0], np.int32), np.array([np.nan], np.float32), 1.0),   # NaN weight
                 (2, rp, np.array([0], np.int32), np.array([np.inf], np.float32), 1.0),   # infinite weight
                 (2, rp, np.array([0], np.int32), np.array([1.0], np.float32), np.inf),   # infinite gamma
                 (2, rp, np.array([0], np.int32), np.array([1.0], np.float32), np.nan)):  # NaN gamma
        with pytest.raises(ckv.CkvError) as e:
            ckv.ckv_leiden(*args, lab)
        assert e.value.status == ckv.CKV_ERR_INVALID_ARG
    with pytest.raises(ckv.CkvError) as e:                                          # n < 1
        ckv.ckv_leiden(0, np.zeros(1, np.int64), np.zeros(0, np.int32), np.zeros(0, np.float32), 1.0,
                       np.zeros(0, np.int32))
    assert e.value.status == ckv.CKV_ERR_INVALID_ARG


def test_binding_checks_host_arrays():
    rp = np.array([0, 1, 1], np.int64)
    col = np.array([0], np.int32)
    w = np.array([1.0], np.float32)
    with pytest.raises(TypeError):
        ckv.ckv_leiden(2, rp.astype(np.int32), col, w, 1.0, np.zeros(2, np.int32))   # wrong row_ptr dtype
    with pytest.raises(TypeError):
        ckv.ckv_leiden(2, rp, col, w, 1.0, np.zeros(2, np.int64))                  # wrong labels dtype
    with pytest.raises(ValueError):
        ckv.ckv_leiden(3, rp, col, w, 1.0, np.zeros(3, np.int32))                  # row_ptr too short


def test_two_triangles(oracle_lib):
    # the oracle's closed-form case: the library finds the same two triangles
    rp = np.array([0, 0, 1, 3, 4, 5, 7], np.int64)
    col = np.array([0, 0, 1, 2, 3, 3, 4], np.int32)
    w = np.ones(7, np.float32)
    lab, C = _lib_leiden(rp, col, w, 6, 1.0)
    assert C == 2 and list(lab) == [0, 0, 0, 1, 1, 1]
