"""Failure handling through the C ABI, made without any GPU fault.

* A bounded device wait that runs out: the single-launch decode step waits
  across CTAs (a selection for its graph's score items, an attention item
  for its graph's selection, a finish for its attention items).  With the
  wait bound cut to one poll (ckv_set_wait_limit) those waits give up, the
  kernel sets CKV_ERR_TIMEOUT in the context's error word and returns; the
  context reports it, stays failed until a state import, and then steps
  exactly as a fresh context does.
* A forced allocation failure on the host side: CKV_FAULT_ALLOC=k makes the
  k-th device allocation inside a call fail as out of memory.  ckv_create
  then returns CKV_ERR_OOM without leaking, and ckv_import_state /
  ckv_init_communities return it with the context's state untouched.
"""
import numpy as np
import pytest

import long_context_decode_ckv_b200 as ckv
from long_context_decode_ckv_b200 import build as ckv_build
from long_context_decode_ckv_b200 import synth
from tests.conftest import gpu_available
from tests.lockstep import _torch_view, config_for

pytestmark = [pytest.mark.gpu,
              pytest.mark.skipif(not gpu_available(), reason="needs a CUDA device")]

CFG = synth.scaled(synth.LLAMA, batch=2, n_q_heads=8, n_kv_heads=2, n0=8000, n_clusters=250,
                   budget=512, steps=3, mode=synth.QUERY_GROUP)


@pytest.fixture(scope="module")
def setup():
    import torch
    ckv_build.build()
    wl = synth.make_workload(CFG)
    dev = torch.device("cuda", 0)
    return wl, _torch_view(wl.K, dev), _torch_view(wl.V, dev), _torch_view(wl.q, dev), dev


def _out(dev):
    import torch
    return torch.empty((CFG.batch, CFG.n_q_heads, CFG.head_dim), dtype=torch.float32, device=dev)


def _step(ctx, q, K, V, n, out):
    ckv.ckv_decode_step(ctx, q, K, V, n, out)
    ckv.ckv_assign_update(ctx, K, n)
    return ckv.ckv_last_error(ctx)


def test_bounded_wait_runs_out_and_reports_timeout(setup, monkeypatch):
    wl, K, V, q, dev = setup
    monkeypatch.setenv("CKV_STEP", "fused")
    ctx = ckv.ckv_create(config_for(CFG))
    fresh = ckv.ckv_create(config_for(CFG))
    try:
        assert ckv.ckv_step_launches(ctx) == 1
        ckv.ckv_init_communities(ctx, wl.labels, 0, CFG.n_comm, K, CFG.n0)
        blob = ckv.ckv_export_state(ctx)
        n = CFG.n0 + 1
        ckv.ckv_set_wait_limit(ctx, 1)
        out = _out(dev)
        assert _step(ctx, q[0], K, V, n, out) == ckv.CKV_ERR_TIMEOUT
        # the failure is sticky: the next step is refused on the host
        with pytest.raises(ckv.CkvError) as e:
            ckv.ckv_decode_step(ctx, q[0], K, V, n, out)
        assert e.value.status == ckv.CKV_ERR_TIMEOUT
        # an import clears it; with the default bound the step is the same
        # as a fresh context's, bit for bit
        ckv.ckv_set_wait_limit(ctx, 0)
        ckv.ckv_import_state(ctx, blob)
        ckv.ckv_init_communities(fresh, wl.labels, 0, CFG.n_comm, K, CFG.n0)
        out_f = _out(dev)
        for i in range(2):
            n = CFG.n0 + i + 1
            assert _step(ctx, q[i], K, V, n, out) == ckv.CKV_OK
            assert _step(fresh, q[i], K, V, n, out_f) == ckv.CKV_OK
            assert bool((out == out_f).all()), f"step {i}: output differs from a fresh context's"
        assert ckv.ckv_export_state(ctx) == ckv.ckv_export_state(fresh)
    finally:
        ckv.ckv_destroy(ctx)
        ckv.ckv_destroy(fresh)


def test_forced_allocation_failure_in_create_leaks_nothing(setup, monkeypatch):
    import torch
    torch.cuda.synchronize()
    free0 = torch.cuda.mem_get_info()[0]
    for k in (1, 2, 9, 25):
        monkeypatch.setenv("CKV_FAULT_ALLOC", str(k))
        with pytest.raises(ckv.CkvError) as e:
            ckv.ckv_create(config_for(CFG))
        assert e.value.status == ckv.CKV_ERR_OOM, k
    monkeypatch.delenv("CKV_FAULT_ALLOC")
    torch.cuda.synchronize()
    free1 = torch.cuda.mem_get_info()[0]
    assert abs(free1 - free0) <= 8 << 20, f"{(free0 - free1) / 2**20:.1f} MiB not released"
    ckv.ckv_destroy(ckv.ckv_create(config_for(CFG)))   # no fault armed: creation works


def test_forced_allocation_failure_keeps_state(setup, monkeypatch):
    wl, K, V, q, dev = setup
    ctx = ckv.ckv_create(config_for(CFG))
    twin = ckv.ckv_create(config_for(CFG))
    try:
        ckv.ckv_init_communities(ctx, wl.labels, 0, CFG.n_comm, K, CFG.n0)
        out = _out(dev)
        assert _step(ctx, q[0], K, V, CFG.n0 + 1, out) == ckv.CKV_OK
        blob = ckv.ckv_export_state(ctx)
        # import allocates the new edge store (3 allocations) before it
        # touches the state; init also a staging buffer for host labels
        for call, ks in (("import", (1, 2, 3)), ("init", (1, 2, 3, 4))):
            for k in ks:
                monkeypatch.setenv("CKV_FAULT_ALLOC", str(k))
                with pytest.raises(ckv.CkvError) as e:
                    if call == "import":
                        ckv.ckv_import_state(ctx, blob)
                    else:
                        ckv.ckv_init_communities(ctx, wl.labels, 0, CFG.n_comm, K, CFG.n0)
                assert e.value.status == ckv.CKV_ERR_OOM, (call, k)
                monkeypatch.delenv("CKV_FAULT_ALLOC")
                assert ckv.ckv_export_state(ctx) == blob, f"{call} k={k} changed the state"
        # the context carries on exactly like one that never saw the failures
        ckv.ckv_import_state(twin, blob)
        out_t = _out(dev)
        for i in (1, 2):
            n = CFG.n0 + i + 1
            assert _step(ctx, q[i], K, V, n, out) == ckv.CKV_OK
            assert _step(twin, q[i], K, V, n, out_t) == ckv.CKV_OK
            assert bool((out == out_t).all()), f"step {i}: output differs from the twin's"
        assert ckv.ckv_export_state(ctx) == ckv.ckv_export_state(twin)
    finally:
        ckv.ckv_destroy(ctx)
        ckv.ckv_destroy(twin)
