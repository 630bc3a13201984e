"""The allocation-free attention entry point against the oracle.

ckv_attend_rows_static serves hosts that cannot call cudaMalloc where the
attention runs (a plugin-style custom op with no workspace, for instance):
its scratch is the library's file-scope device array.  Each graph's query
heads attend over the sinks, the caller's rows and the new token -- the
exact attention with sinks of "CommunityKV: Efficient Long-Context Decoding
via Graph Partitioning", Figure 1 caption step (3), over a given row set.
The output must match oracle.attend on the same rows within the decode
parity tolerance (2e-3 max relative error per (batch, head)), on two calls
in a row with different rows, for bf16 query groups of 4 and 8 heads, bf16
per-head graphs and fp32.  Ragged row counts (0, 1, one item's worth, a
ragged tail) are in every case.  This file is collected last and needs no
state from the other tests.
"""
import numpy as np
import pytest

import oracle
import long_context_decode_ckv_b200 as ckv
from long_context_decode_ckv_b200 import build as ckv_build
from long_context_decode_ckv_b200 import synth
from tests.conftest import gpu_available
from tests.lockstep import _torch_view, config_for

pytestmark = [pytest.mark.gpu,
              pytest.mark.skipif(not gpu_available(), reason="needs a CUDA device")]

OUT_RTOL = 2e-3
# row counts per graph, cycled: empty, one row, one attention item's worth
# (264) and its neighbours, a longer ragged list
ROW_COUNTS = [0, 1, 263, 264, 265, 700, 1500, 37]

CASES = {
    "bf16_group4": synth.scaled(synth.LLAMA, batch=2, n_q_heads=8, n_kv_heads=2, n0=3000, n_clusters=150,
                                budget=256, steps=2, mode=synth.QUERY_GROUP),
    "bf16_group8": synth.scaled(synth.LLAMA, batch=1, n_q_heads=16, n_kv_heads=2, n0=2500, n_clusters=150,
                                budget=256, steps=2, mode=synth.QUERY_GROUP),
    "bf16_per_head": synth.scaled(synth.LLAMA, batch=1, n_q_heads=8, n_kv_heads=2, n0=3000, n_clusters=150,
                                  budget=256, steps=2, mode=synth.PER_HEAD),
    "f32_tiny": synth.scaled(synth.TINY, steps=2),
}


def _rows_for(cfg, n, call, rng):
    """Per graph: a row list of [S, n-1) (sorted, except graph 1 of call 1)."""
    G = cfg.n_graphs
    pool = np.arange(cfg.n_sinks, n - 1, dtype=np.int32)
    rows = []
    for g in range(G):
        T = min(ROW_COUNTS[(g + 3 * call) % len(ROW_COUNTS)], len(pool))
        r = rng.choice(pool, T, replace=False)
        rows.append(r if (call == 1 and g == 1) else np.sort(r))
    max_rows = max(1, max(len(r) for r in rows))
    rows_host = np.full((G, max_rows), -1, np.int32)     # the padding is never read
    for g, r in enumerate(rows):
        rows_host[g, :len(r)] = r
    return rows, rows_host, np.array([len(r) for r in rows], np.int32), max_rows


@pytest.mark.parametrize("case", list(CASES))
def test_static_scratch_attention_matches_oracle(case):
    import torch
    ckv_build.build()
    cfg = CASES[case]
    wl = synth.make_workload(cfg)
    dev = torch.device("cuda", 0)
    K, V, q = _torch_view(wl.K, dev), _torch_view(wl.V, dev), _torch_view(wl.q, dev)
    c = config_for(cfg)
    rng = np.random.default_rng(synth.BASE_SEED + 77)
    S = cfg.n_sinks
    for call in range(2):                                 # two calls in a row
        n = cfg.n0 + call + 1
        rows, rows_host, n_rows, max_rows = _rows_for(cfg, n, call, rng)
        out = torch.full((cfg.batch, cfg.n_q_heads, cfg.head_dim), float("nan"), dtype=torch.float32,
                         device=dev)
        ckv.ckv_attend_rows_static(c, q[call], K, V, n, rows_host, n_rows, max_rows, out)
        got = out.cpu().numpy()
        for g in range(cfg.n_graphs):
            b, kvh, heads = cfg.graph_heads(g)
            all_rows = np.concatenate([np.arange(S, dtype=np.int32), rows[g],
                                       np.array([n - 1], np.int32)])
            ref, _, _, _ = oracle.attend(np.ascontiguousarray(wl.q[call, b, heads]), wl.K[b, kvh],
                                         wl.V[b, kvh], all_rows)
            for h_i, h in enumerate(heads):
                err = float(np.max(np.abs(got[b, h] - ref[h_i])) / np.max(np.abs(ref[h_i])))
                assert err <= OUT_RTOL, (f"{case} call {call} graph {g} ({len(rows[g])} rows) head {h}: "
                                         f"rel err {err:.3g}")


def test_static_scratch_arguments_checked():
    import torch
    ckv_build.build()
    cfg = CASES["bf16_group4"]
    wl = synth.make_workload(cfg)
    dev = torch.device("cuda", 0)
    K, V, q = _torch_view(wl.K, dev), _torch_view(wl.V, dev), _torch_view(wl.q, dev)
    c = config_for(cfg)
    n = cfg.n0 + 1
    rows, rows_host, n_rows, max_rows = _rows_for(cfg, n, 0, np.random.default_rng(5))
    out = torch.zeros((cfg.batch, cfg.n_q_heads, cfg.head_dim), dtype=torch.float32, device=dev)

    def status_of(*args):
        with pytest.raises(ckv.CkvError) as e:
            ckv.ckv_attend_rows_static(*args)
        return e.value.status

    # a sink or the new token as a row, and a row count above max_rows
    for bad_row in (0, n - 1):
        bad = rows_host.copy()
        g = int(np.argmax(n_rows > 0))
        bad[g, 0] = bad_row
        assert status_of(c, q[0], K, V, n, bad, n_rows, max_rows, out) == ckv.CKV_ERR_INVALID_ARG
    too_many = n_rows.copy()
    too_many[0] = max_rows + 1
    assert status_of(c, q[0], K, V, n, rows_host, too_many, max_rows, out) == ckv.CKV_ERR_INVALID_ARG
    # a device the machine does not have
    c_bad = config_for(cfg, device=999)
    assert status_of(c_bad, q[0], K, V, n, rows_host, n_rows, max_rows, out) == ckv.CKV_ERR_INVALID_ARG
    # row lists larger than the static array: refused before any device work
    big = 2_000_000
    assert status_of(c, q[0], K, V, n, np.zeros((cfg.n_graphs, big), np.int32),
                     np.zeros(cfg.n_graphs, np.int32), big, out) == ckv.CKV_ERR_CAPACITY
    # the array is still usable afterwards
    ckv.ckv_attend_rows_static(c, q[0], K, V, n, rows_host, n_rows, max_rows, out)
    assert torch.isfinite(out).all()
