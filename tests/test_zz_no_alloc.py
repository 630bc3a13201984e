"""The allocation-free attention entry point against the decode step.

ckv_attend_rows_static serves hosts that cannot call cudaMalloc where the
attention runs (a plugin-style custom op with no workspace, for instance):
its scratch is the library's file-scope device array.  Given the rows a
ckv_decode_step kept, it must reproduce that step's attention output within
the tolerance of the decode parity tests (2e-3 max relative error per
(batch, head)), on two calls in a row.  This file is collected last and
needs no state from the other tests.
"""
import numpy as np
import pytest

import long_context_decode_ckv_b200 as ckv
from long_context_decode_ckv_b200 import build as ckv_build
from long_context_decode_ckv_b200 import state as ckv_state
from long_context_decode_ckv_b200 import synth
from tests.conftest import gpu_available
from tests.lockstep import _torch_view, config_for

pytestmark = [pytest.mark.gpu,
              pytest.mark.skipif(not gpu_available(), reason="needs a CUDA device")]

OUT_RTOL = 2e-3


@pytest.mark.parametrize("mode", [synth.QUERY_GROUP, synth.PER_HEAD])
def test_static_scratch_attention_matches_decode_step(mode):
    import torch
    ckv_build.build()
    cfg = synth.scaled(synth.LLAMA, batch=2, n_q_heads=8, n_kv_heads=2, n0=3000, n_clusters=150,
                       budget=256, steps=2, mode=mode)
    wl = synth.make_workload(cfg)
    dev = torch.device("cuda", 0)
    K, V, q = _torch_view(wl.K, dev), _torch_view(wl.V, dev), _torch_view(wl.q, dev)
    c = config_for(cfg)
    ctx = ckv.ckv_create(c)
    try:
        ckv.ckv_init_communities(ctx, wl.labels, 0, cfg.n_comm, K, cfg.n0)
        G = cfg.n_graphs
        for i in range(2):                                   # two calls in a row
            n = cfg.n0 + i + 1
            st = ckv_state.parse(ckv.ckv_export_state(ctx))  # members as the step sees them
            ref = torch.empty((cfg.batch, cfg.n_q_heads, 128), dtype=torch.float32, device=dev)
            ckv.ckv_decode_step(ctx, q[i], K, V, n, ref)
            ckv.ckv_assign_update(ctx, K, n)
            n_sel = np.zeros(G, np.int32)
            sel = np.zeros((G, cfg.n_comm), np.int32)
            ckv.ckv_get_step_debug(ctx, n_sel=n_sel, sel=sel)
            rows = [np.concatenate([st.community_members(g, int(cc)) for cc in sel[g, :n_sel[g]]])
                    for g in range(G)]
            max_rows = max(len(r) for r in rows)
            rows_host = np.zeros((G, max_rows), np.int32)
            for g, r in enumerate(rows):
                rows_host[g, :len(r)] = r
            n_rows = np.array([len(r) for r in rows], np.int32)
            out = torch.full_like(ref, float("nan"))
            ckv.ckv_attend_rows_static(c, q[i], K, V, n, rows_host, n_rows, max_rows, out)
            torch.cuda.synchronize()
            a, b = out.cpu().numpy(), ref.cpu().numpy()
            for bb in range(cfg.batch):
                for h in range(cfg.n_q_heads):
                    err = np.max(np.abs(a[bb, h] - b[bb, h])) / np.max(np.abs(b[bb, h]))
                    assert err <= OUT_RTOL, f"call {i} batch {bb} head {h}: rel err {err:.3g}"
        # rows that are sinks or the new token are rejected before any launch
        bad = rows_host.copy()
        bad[0, 0] = n - 1
        with pytest.raises(ckv.CkvError) as e:
            ckv.ckv_attend_rows_static(c, q[1], K, V, n, bad, n_rows, max_rows, out)
        assert e.value.status == ckv.CKV_ERR_INVALID_ARG
    finally:
        ckv.ckv_destroy(ctx)
