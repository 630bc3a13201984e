"""GPU parity of ckv_build_graph (prefill top-kappa graph on tcgen05 tensor
cores) against the CPU oracle.

"CommunityKV: Efficient Long-Context Decoding via Graph Partitioning",
Figure 1 caption, step (1): each query row connects to its top-kappa keys,
sinks excluded.  Edge sets are bit-exact except at a near-tie (the oracle's
float score gap at the cutoff below 1e-5 relative); weights within 1e-4
relative (fp32 tensor-core scores and exp2 against the double oracle).
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


def run_gpu(Q, K, S, kap):
    import torch
    H, n, D = Q.shape
    dev = torch.device("cuda", 0)
    q = torch.from_numpy(Q).view(torch.bfloat16).to(dev)
    k = torch.from_numpy(K).view(torch.bfloat16).to(dev)
    E = int(closed_row_ptr(n, S, kap)[-1])
    row_ptr = torch.full((H, n + 1), -7, dtype=torch.int64, device=dev)
    col = torch.full((H, max(E, 1)), -7, dtype=torch.int32, device=dev)
    w = torch.full((H, max(E, 1)), -7.0, dtype=torch.float32, device=dev)
    ckv.ckv_build_graph(H, n, D, S, kap, ckv.CKV_BF16, q, k, row_ptr, col, w)
    torch.cuda.synchronize()
    return row_ptr.cpu().numpy(), col.cpu().numpy(), w.cpu().numpy()


def check(Q, K, S, kap, rows_per_head=None, heads=None):
    H, n, _ = Q.shape
    rp, col, w = run_gpu(Q, K, S, kap)
    ref_rp = closed_row_ptr(n, S, kap)
    exempt = 0
    for h in (range(H) if heads is None else heads):
        np.testing.assert_array_equal(rp[h], ref_rp, err_msg=f"head {h} row_ptr")
        rows = np.arange(n) if rows_per_head is None else rows_per_head
        ocol, ow, odeg, ogap = oracle.prefill_rows(Q[h], K[h], rows, S, kap)
        for t, i in enumerate(rows):
            a, b = rp[h, i], rp[h, i + 1]
            assert b - a == odeg[t]
            gc, gw = col[h, a:b], w[h, a:b]
            rc, rw = ocol[t, :odeg[t]], ow[t, :odeg[t]]
            if set(gc.tolist()) != set(rc.tolist()):
                assert ogap[t] < GAP_EXEMPT, f"head {h} row {i}: edges {gc} vs {rc} (gap {ogap[t]:.3g})"
                exempt += 1
                continue
            ref = dict(zip(rc.tolist(), rw.tolist()))
            for j, wv in zip(gc.tolist(), gw.tolist()):
                assert abs(wv - ref[j]) <= W_RTOL * ref[j] + 1e-12, f"head {h} row {i} edge {j}: {wv} vs {ref[j]}"
            assert np.all(np.diff(gw) <= 0) or np.all(np.diff(gw) <= 1e-6 * gw[:-1])
            assert not np.isin(gc, np.arange(S)).any() and np.all(gc < i)
    return exempt


def test_full_graph_n2048_two_heads():
    Q, K = synth.make_prefill(synth.PREFILL, n=2048)
    check(Q[:2], K[:2], 4, 8)


@pytest.mark.parametrize("n,S,kap", [(1, 4, 8), (5, 4, 8), (127, 4, 8), (129, 4, 8), (1000, 0, 1),
                                     (777, 17, 16), (640, 4, 32), (300, 4, 3)])
def test_ragged_and_kappa_variants(n, S, kap):
    Q, K = synth.make_prefill(synth.PREFILL, n=n)
    check(Q[:3], K[:3], S, kap)


def test_full_size_n16384_sampled_rows():
    P = synth.PREFILL
    Q, K = synth.make_prefill(P)
    rng = np.random.default_rng(0)
    edge = [0, 1, 3, 4, 5, 12, 13, 127, 128, 129, 255, 256, 8191, 8192, P.n - 129, P.n - 128,
            P.n - 2, P.n - 1]
    rows = np.unique(np.concatenate([edge, rng.integers(0, P.n, 200)])).astype(np.int32)
    check(Q, K, P.n_sinks, P.kappa, rows_per_head=rows)


def test_bad_arguments():
    import torch
    dev = torch.device("cuda", 0)
    x = torch.zeros((2, 64, 128), dtype=torch.bfloat16, device=dev)
    rp = torch.zeros((2, 65), dtype=torch.int64, device=dev)
    c = torch.zeros(1024, dtype=torch.int32, device=dev)
    w = torch.zeros(1024, dtype=torch.float32, device=dev)
    with pytest.raises(ckv.CkvError):
        ckv.ckv_build_graph(2, 64, 128, 4, 8, ckv.CKV_BF16, x[:, :, 1:], x, rp, c, w)   # misaligned
    with pytest.raises(ckv.CkvError):
        ckv.ckv_build_graph(2, 64, 128, 4, 0, ckv.CKV_BF16, x, x, rp, c, w)
