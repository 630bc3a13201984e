"""GPU parity of ckv_build_graph_grouped (query-group aggregated prefill
graph: per-head row statistics, then one graph per KV head on the tcgen05
tensor cores) against the CPU oracle.

"CommunityKV: Efficient Long-Context Decoding via Graph Partitioning":
Figure 1 caption step (1) with the abstract's query-group graph
aggregation.  Edge sets bit-exact except at a near-tie (the oracle's float
gap between the kappa-th and the next summed weight below 1e-5 relative);
weights within 1e-4 relative (fp32 tensor-core scores and exp2 against the
double oracle, as for the per-head graph).
"""
import numpy as np
import pytest

import long_context_decode_ckv_b200 as ckv
import oracle
from long_context_decode_ckv_b200 import build as ckv_build
from long_context_decode_ckv_b200 import synth
from tests.conftest import gpu_available

pytestmark = [pytest.mark.gpu,
              pytest.mark.skipif(not gpu_available(), reason="needs a CUDA device")]

W_RTOL = 1e-4
GAP_EXEMPT = 1e-5


@pytest.fixture(scope="module", autouse=True)
def _built():
    ckv_build.build()


def closed_row_ptr(n, S, kap):
    deg = np.clip(np.arange(n) - S, 0, kap)
    return np.concatenate([[0], np.cumsum(deg)]).astype(np.int64)


def run_grouped(Q, K, group, S, kap):
    import torch
    Hq, n, D = Q.shape
    Hkv = Hq // group
    dev = torch.device("cuda", 0)
    q = torch.from_numpy(np.ascontiguousarray(Q)).view(torch.bfloat16).to(dev)
    k = torch.from_numpy(np.ascontiguousarray(K)).view(torch.bfloat16).to(dev)
    E = int(closed_row_ptr(n, S, kap)[-1])
    ws = torch.full((ckv.ckv_build_graph_grouped_workspace(Hkv, group, n),), 0x7f, dtype=torch.uint8, device=dev)
    row_ptr = torch.full((Hkv, n + 1), -7, dtype=torch.int64, device=dev)
    col = torch.full((Hkv, max(E, 1)), -7, dtype=torch.int32, device=dev)
    w = torch.full((Hkv, max(E, 1)), -7.0, dtype=torch.float32, device=dev)
    ckv.ckv_build_graph_grouped(Hkv, group, n, D, S, kap, ckv.CKV_BF16, q, k, ws, row_ptr, col, w)
    torch.cuda.synchronize()
    return row_ptr.cpu().numpy(), col.cpu().numpy(), w.cpu().numpy()


def check_grouped(Q, K, group, S, kap, rows=None):
    Hq, n, _ = Q.shape
    Hkv = Hq // group
    rp, col, w = run_grouped(Q, K, group, S, kap)
    ref_rp = closed_row_ptr(n, S, kap)
    rows = np.arange(n) if rows is None else rows
    exempt = 0
    for u in range(Hkv):
        np.testing.assert_array_equal(rp[u], ref_rp, err_msg=f"kv head {u} row_ptr")
        ocol, ow, odeg, ogap = oracle.prefill_rows_grouped(Q[u * group:(u + 1) * group], K[u], rows, S, kap)
        for t, i in enumerate(rows):
            a, b = rp[u, i], rp[u, i + 1]
            assert b - a == odeg[t]
            gc, gw = col[u, a:b], w[u, a:b]
            rc, rw = ocol[t, :odeg[t]], ow[t, :odeg[t]]
            if set(gc.tolist()) != set(rc.tolist()):
                assert ogap[t] < GAP_EXEMPT, f"kv head {u} row {i}: edges {gc} vs {rc} (gap {ogap[t]:.3g})"
                exempt += 1
                continue
            ref = dict(zip(rc.tolist(), rw.tolist()))
            for j, wv in zip(gc.tolist(), gw.tolist()):
                assert abs(wv - ref[j]) <= W_RTOL * ref[j] + 1e-12, f"kv head {u} row {i} edge {j}: {wv} vs {ref[j]}"
            assert np.all(np.diff(gw) <= 1e-6 * np.abs(gw[:-1]))
            assert not np.isin(gc, np.arange(S)).any() and np.all(gc < i)
            assert gw.sum() <= group * (1 + 1e-4)
    return exempt


@pytest.mark.parametrize("group", [1, 2, 4])
def test_grouped_full_graph_n2048(group):
    Q, K = synth.make_prefill(synth.PREFILL, n=2048)
    check_grouped(Q[:2 * group], K[:2], group, 4, 8)


@pytest.mark.parametrize("group,n,S,kap", [(4, 1, 4, 8), (4, 5, 4, 8), (4, 63, 4, 8), (4, 65, 4, 8),
                                           (4, 127, 4, 8), (4, 129, 4, 8), (2, 300, 0, 1), (4, 777, 17, 16),
                                           (4, 640, 4, 32), (1, 129, 4, 3), (2, 1000, 4, 32)])
def test_grouped_ragged_and_kappa_variants(group, n, S, kap):
    Q, K = synth.make_prefill(synth.PREFILL, n=n)
    check_grouped(Q[:2 * group], K[:2], group, S, kap)


def test_grouped_full_size_n16384_sampled_rows():
    # the prefill workload's 8 query heads as 2 KV heads of 4
    P = synth.PREFILL
    Q, K = synth.make_prefill(P)
    rng = np.random.default_rng(1)
    edge = [0, 1, 3, 4, 5, 12, 13, 63, 64, 127, 128, 129, 255, 256, 8191, 8192, P.n - 129, P.n - 65,
            P.n - 64, P.n - 2, P.n - 1]
    rows = np.unique(np.concatenate([edge, rng.integers(0, P.n, 120)])).astype(np.int32)
    check_grouped(Q, K[:2], 4, P.n_sinks, P.kappa, rows=rows)


def test_grouped_bad_arguments():
    import torch
    dev = torch.device("cuda", 0)
    x = torch.zeros((8, 64, 128), dtype=torch.bfloat16, device=dev)
    ws = torch.zeros(ckv.ckv_build_graph_grouped_workspace(1, 8, 64) + 64, dtype=torch.uint8, device=dev)
    rp = torch.zeros((2, 65), dtype=torch.int64, device=dev)
    c = torch.zeros(1024, dtype=torch.int32, device=dev)
    w = torch.zeros(1024, dtype=torch.float32, device=dev)
    for kw in (dict(group=8), dict(group=3), dict(kap=0), dict(ws_off=4)):
        with pytest.raises(ckv.CkvError) as e:
            g = kw.get("group", 4)
            ckv.ckv_build_graph_grouped(8 // g if 8 % g == 0 else 2, g, 64, 128, 4, kw.get("kap", 8), ckv.CKV_BF16,
                                        x, x, ws[kw.get("ws_off", 0):], rp, c, w)
        assert e.value.status == ckv.CKV_ERR_INVALID_ARG
