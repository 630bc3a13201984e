"""The range-checked build (libckv_debug.so, -DCKV_DEBUG_BOUNDS) turns
corrupt community state into CKV_ERR_STATE instead of a memory fault.

A child process loads the range-checked library (CKV_DEBUG_BOUNDS=1), runs
a normal decode step, then overwrites device state through the debug-only
ckv_debug_poke -- the first member of every community of graph 0 becomes a
token far outside the cache, or every community's segment offset points far
outside the member pool -- and runs the next step.  The gather, the row copy
and the centroid update each check the index before the access, so the step
reports CKV_ERR_STATE through ckv_last_error and the device stays usable: a
fresh context then steps normally.  Both decode paths (three kernels, and
the single persistent kernel selected by CKV_STEP=fused) are covered.
"""
import json
import os
import subprocess
import sys

import pytest

from tests.conftest import gpu_available

pytestmark = [pytest.mark.gpu,
              pytest.mark.skipif(not gpu_available(), reason="needs a CUDA device")]

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
FAR = 1 << 30          # far outside any cache length or pool capacity of the test


def child():
    """Runs in the child process (CKV_DEBUG_BOUNDS=1); prints one JSON line."""
    import numpy as np
    import torch

    import long_context_decode_ckv_b200 as ckv
    from long_context_decode_ckv_b200 import build as ckv_build
    from long_context_decode_ckv_b200 import state as ckv_state
    from long_context_decode_ckv_b200 import synth
    from tests.lockstep import _torch_view, config_for

    assert ckv.DEBUG_BOUNDS and ckv.LIB_PATH == ckv_build.LIB_DEBUG
    ckv_build.build(debug=True)
    cfg = synth.scaled(synth.LLAMA, batch=1, n_q_heads=8, n_kv_heads=2, n0=3000, n_clusters=150,
                       budget=256, steps=3, mode=synth.QUERY_GROUP)
    wl = synth.make_workload(cfg)
    dev = torch.device("cuda", 0)
    K, V, q = _torch_view(wl.K, dev), _torch_view(wl.V, dev), _torch_view(wl.q, dev)
    out = torch.empty((cfg.batch, cfg.n_q_heads, cfg.head_dim), dtype=torch.float32, device=dev)

    def step(ctx, i):
        n = cfg.n0 + i + 1
        ckv.ckv_decode_step(ctx, q[i], K, V, n, out)
        ckv.ckv_assign_update(ctx, K, n)
        return ckv.ckv_last_error(ctx)

    res = {}
    for mode in ("split", "fused"):
        os.environ["CKV_STEP"] = mode
        for what in (0, 1):
            ctx = ckv.ckv_create(config_for(cfg))
            try:
                ckv.ckv_init_communities(ctx, wl.labels, 0, cfg.n_comm, K, cfg.n0)
                first = step(ctx, 0)
                sizes = ckv_state.parse(ckv.ckv_export_state(ctx)).sizes[0]
                for c in range(cfg.n_comm):
                    if sizes[c] > 0:
                        ckv.ckv_debug_poke(ctx, what, 0, c, 0, FAR)
                res[f"{mode}_{what}"] = [first, step(ctx, 1)]
            finally:
                ckv.ckv_destroy(ctx)
        # the device still answers: a fresh context steps normally
        ctx = ckv.ckv_create(config_for(cfg))
        try:
            ckv.ckv_init_communities(ctx, wl.labels, 0, cfg.n_comm, K, cfg.n0)
            res[f"{mode}_fresh"] = [step(ctx, 0), step(ctx, 1)]
            res[f"{mode}_launches"] = ckv.ckv_step_launches(ctx)
        finally:
            ckv.ckv_destroy(ctx)
        assert np.isfinite(out.cpu().numpy()).all()
    print("RESULT " + json.dumps(res), flush=True)


def test_corrupt_state_reports_error_without_fault():
    import long_context_decode_ckv_b200 as ckv
    from long_context_decode_ckv_b200 import build as ckv_build
    ckv_build.build(debug=True)
    env = dict(os.environ, CKV_DEBUG_BOUNDS="1")
    p = subprocess.run([sys.executable, "-c", "from tests.test_gpu_debug_bounds import child; child()"],
                       cwd=ROOT, env=env, capture_output=True, text=True, timeout=600)
    assert p.returncode == 0, p.stdout[-2000:] + p.stderr[-4000:]
    line = [ln for ln in p.stdout.splitlines() if ln.startswith("RESULT ")][-1]
    res = json.loads(line[len("RESULT "):])
    OK, STATE = ckv.CKV_OK, ckv.CKV_ERR_STATE
    assert res["split_launches"] == 4 and res["fused_launches"] == 1
    for mode in ("split", "fused"):
        for what in (0, 1):
            assert res[f"{mode}_{what}"] == [OK, STATE], (mode, what, res)
        assert res[f"{mode}_fresh"] == [OK, OK], (mode, res)
