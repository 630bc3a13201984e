"""GPU parity of the attention-mass recall (ckv_step_recall) and of the dense
decode comparator (ckv_dense_decode) against the CPU oracle, through the C
ABI.

"CommunityKV: Efficient Long-Context Decoding via Graph Partitioning",
Figure 3 (right): the share of the dense attention mass that the retrieved
set captures, per query head.  Rules: recall |r_gpu - r_ref| <= 1e-3 r_ref +
1e-6 (derivation in lockstep.py); dense output max |o - o_ref| / max |o_ref|
<= 2e-3 per head, the same bound as the sparse attention; log-sum-exp within
1e-3 absolute (the relative error of the sum plus the logit error of the max).
"""
import os

import numpy as np
import pytest

import oracle
import long_context_decode_ckv_b200 as ckv
from long_context_decode_ckv_b200 import build as ckv_build
from long_context_decode_ckv_b200 import synth
from tests.conftest import gpu_available
from tests.lockstep import OUT_RTOL, Lockstep, _torch_view, config_for

pytestmark = [pytest.mark.gpu,
              pytest.mark.skipif(not gpu_available(), reason="needs a CUDA device")]

WORKERS = min(8, os.cpu_count() or 1)
LSE_ATOL = 1e-3


@pytest.fixture(scope="module", autouse=True)
def _built():
    ckv_build.build()


def _run(cfg, tracked=None, steps=None, recall_every=1):
    wl = synth.make_workload(cfg, workers=WORKERS)
    ls = Lockstep(wl, tracked=tracked, recall_every=recall_every)
    try:
        for i in range(cfg.steps if steps is None else steps):
            ls.step(i)
    finally:
        ls.close()
    rec = [r for l in ls.logs for r in l.recalls]
    print(f"{cfg.name}: recall checks {len(rec)}, oracle recall min {min(rec):.4f} "
          f"mean {np.mean(rec):.4f}, max |err| {max(l.max_recall_err for l in ls.logs):.3g}")
    return ls, rec


@pytest.mark.parametrize("cfg", [
    synth.scaled(synth.TINY, n0=1000, n_clusters=25, budget=200),                 # fp32, ragged tiles
    synth.scaled(synth.LLAMA, batch=2, n_q_heads=8, n_kv_heads=2, n0=4000, n_clusters=125,
                 budget=300, steps=6),                                           # bf16, per head
    synth.scaled(synth.LLAMA, batch=2, n_q_heads=8, n_kv_heads=2, n0=4000, n_clusters=125,
                 budget=300, steps=6, mode=synth.QUERY_GROUP),                   # bf16, query group
    synth.scaled(synth.LLAMA, batch=1, n_q_heads=8, n_kv_heads=1, n0=3001, n_clusters=100,
                 budget=500, steps=4, bf16=False),                               # fp32, 8 heads per unit
    synth.scaled(synth.LLAMA, batch=1, n_q_heads=32, n_kv_heads=1, n0=2003, n_clusters=64,
                 budget=256, steps=3),                                           # bf16, 32 heads per unit
], ids=["tiny_f32", "gqa_per_head", "gqa_query_group", "f32_group8", "bf16_group32"])
def test_recall_matches_oracle(cfg):
    _, rec = _run(cfg)
    assert len(rec) > 0 and all(0.0 < r <= 1.0 + 1e-12 for r in rec)


def test_recall_is_one_when_every_token_is_attended():
    cfg = synth.scaled(synth.LLAMA, batch=1, n_q_heads=4, n_kv_heads=1, n0=1500, n_clusters=40,
                       budget=10 ** 6, steps=3, mode=synth.QUERY_GROUP)
    _, rec = _run(cfg)
    np.testing.assert_allclose(rec, 1.0, rtol=1e-12)


def test_recall_qwen8b_full_size_sampled():
    # full size (n = 131072 + steps), budget 4096; the oracle follows 2 graphs
    cfg = synth.scaled(synth.QWEN8B, steps=17)
    _run(cfg, tracked=[0, 31], recall_every=8)


def _dense_check(wl, n, dev, heads_sample=None):
    import torch
    cfg = wl.cfg
    K, V, q = _torch_view(wl.K, dev), _torch_view(wl.V, dev), _torch_view(wl.q[0], dev)
    ctx = ckv.ckv_create(config_for(cfg))
    try:
        out = torch.full((cfg.batch, cfg.n_q_heads, 128), float("nan"), dtype=torch.float32, device=dev)
        lse = torch.full((cfg.batch, cfg.n_q_heads), float("nan"), dtype=torch.float32, device=dev)
        ckv.ckv_dense_decode(ctx, q, K, V, n, out, lse)
        torch.cuda.synchronize()
        out, lse = out.cpu().numpy(), lse.cpu().numpy()
    finally:
        ckv.ckv_destroy(ctx)
    pairs = heads_sample or [(b, h) for b in range(cfg.batch) for h in range(cfg.n_q_heads)]
    rows = np.arange(n, dtype=np.int32)
    worst = 0.0
    for b, h in pairs:
        kvh = h // cfg.group
        qh = np.ascontiguousarray(wl.q[0, b, h:h + 1])
        ref, _, m, l = oracle.attend(qh, wl.K[b, kvh], wl.V[b, kvh], rows)
        err = float(np.max(np.abs(out[b, h] - ref[0])) / max(np.max(np.abs(ref[0])), 1e-30))
        worst = max(worst, err)
        assert err <= OUT_RTOL, f"n={n} b={b} h={h}: out rel err {err:.3g}"
        assert abs(float(lse[b, h]) - (m[0] + np.log(l[0]))) <= LSE_ATOL
    return worst


@pytest.mark.parametrize("bf16", [False, True])
@pytest.mark.parametrize("group", [1, 4, 8])
def test_dense_decode_matches_oracle(bf16, group):
    import torch
    cfg = synth.scaled(synth.LLAMA, batch=2, n_q_heads=2 * group, n_kv_heads=2, n0=1500,
                       n_clusters=40, steps=2, bf16=bf16)
    wl = synth.make_workload(cfg, workers=WORKERS)
    dev = torch.device("cuda", 0)
    for n in (1, 7, 17, 1000, cfg.n_max):   # single row, ragged tiles, the full cache
        _dense_check(wl, n, dev)


def test_dense_decode_qwen8b_full_size_sampled():
    import torch
    cfg = synth.scaled(synth.QWEN8B, steps=1)
    wl = synth.make_workload(cfg, workers=WORKERS)
    worst = _dense_check(wl, cfg.n_max, torch.device("cuda", 0),
                         heads_sample=[(0, 0), (1, 13), (2, 22), (3, 31)])
    print(f"dense decode n={cfg.n_max}: worst out rel err {worst:.3g}")


def test_recall_and_dense_arguments_checked():
    import torch
    cfg = synth.scaled(synth.TINY, n0=256, n_clusters=8, steps=4)
    wl = synth.make_workload(cfg)
    dev = torch.device("cuda", 0)
    K, V, q = _torch_view(wl.K, dev), _torch_view(wl.V, dev), _torch_view(wl.q, dev)
    rec = torch.empty((1, 1), dtype=torch.float32, device=dev)
    out = torch.empty((1, 1, 128), dtype=torch.float32, device=dev)
    ctx = ckv.ckv_create(config_for(cfg))
    try:
        def status(fn):
            with pytest.raises(ckv.CkvError) as e:
                fn()
            return e.value.status
        n = cfg.n0 + 1
        assert status(lambda: ckv.ckv_step_recall(ctx, q[0], K, n, rec)) == ckv.CKV_ERR_STATE  # no init
        ckv.ckv_init_communities(ctx, wl.labels, 0, cfg.n_comm, K, cfg.n0)
        assert status(lambda: ckv.ckv_step_recall(ctx, q[0], K, n, rec)) == ckv.CKV_ERR_STATE  # no step
        ckv.ckv_decode_step(ctx, q[0], K, V, n, out)
        assert status(lambda: ckv.ckv_step_recall(ctx, q[0], K, n + 1, rec)) == ckv.CKV_ERR_STATE
        assert status(lambda: ckv.ckv_step_recall(ctx, q[0], K, n, None)) == ckv.CKV_ERR_INVALID_ARG
        ckv.ckv_step_recall(ctx, q[0], K, n, rec)         # before the assign call
        ckv.ckv_assign_update(ctx, K, n)
        ckv.ckv_step_recall(ctx, q[0], K, n, rec)         # and after it
        assert ckv.ckv_last_error(ctx) == ckv.CKV_OK
        r = float(rec.cpu()[0, 0])
        assert 0.0 < r <= 1.0 + 1e-6
        assert status(lambda: ckv.ckv_dense_decode(ctx, q[0], K, V, 0, out)) == ckv.CKV_ERR_INVALID_ARG
        assert status(lambda: ckv.ckv_dense_decode(ctx, q[0], K, V, cfg.n_max + 1, out)) == \
            ckv.CKV_ERR_INVALID_ARG
        assert status(lambda: ckv.ckv_dense_decode(ctx, q[0], K, None, 5, out)) == ckv.CKV_ERR_INVALID_ARG
        ckv.ckv_import_state(ctx, ckv.ckv_export_state(ctx))
        assert status(lambda: ckv.ckv_step_recall(ctx, q[0], K, n, rec)) == ckv.CKV_ERR_STATE  # after import
    finally:
        ckv.ckv_destroy(ctx)
