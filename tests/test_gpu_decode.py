"""GPU parity of the decode path (ckv_init_communities, ckv_decode_step,
ckv_assign_update) against the CPU oracle, through the C ABI.

"CommunityKV: Efficient Long-Context Decoding via Graph Partitioning",
Figure 1 caption steps (2)-(3).  The comparison rules are in lockstep.py.
"""
import dataclasses
import os

import numpy as np
import pytest

import long_context_decode_ckv_b200 as ckv
from long_context_decode_ckv_b200 import build as ckv_build
from long_context_decode_ckv_b200 import state as ckv_state
from long_context_decode_ckv_b200 import synth
from tests.conftest import gpu_available
from tests.lockstep import Lockstep, config_for, _torch_view

pytestmark = [pytest.mark.gpu,
              pytest.mark.skipif(not gpu_available(), reason="needs a CUDA device")]

WORKERS = min(8, os.cpu_count() or 1)


@pytest.fixture(scope="module", autouse=True)
def _built():
    ckv_build.build()


def run_lockstep(cfg, tracked=None, steps=None, compare_every=1, slack=16, wl=None):
    wl = synth.make_workload(cfg, workers=WORKERS) if wl is None else wl
    ls = Lockstep(wl, tracked=tracked, slack=slack)
    try:
        ls.compare_state()
        steps = cfg.steps if steps is None else steps
        for i in range(steps):
            ls.step(i)
            if compare_every and (i + 1) % compare_every == 0:
                ls.compare_state()
        ls.compare_state()
    finally:
        ls.close()
    if ls.logs:
        print(f"{cfg.name}: max out err {max(l.max_out_err for l in ls.logs):.3g}")
        ls.check_exempt_cap()
    return ls


def test_tiny_fp32_all_steps():
    run_lockstep(synth.TINY)


@pytest.mark.parametrize("kw", [
    dict(n0=1000, n_clusters=25, budget=200),          # ragged tiles, uneven clusters
    dict(budget=8),                                     # no community fits: forced C = 1
    dict(budget=10 ** 6),                               # every community kept: dense attention
    dict(kappa=1), dict(kappa=32), dict(n_sinks=0), dict(n_sinks=17),
    dict(n0=5, n_clusters=1, steps=6, comm_size=16),    # one community, a few members
])
def test_tiny_edge_cases(kw):
    cfg = synth.scaled(synth.TINY, **kw)
    run_lockstep(cfg)


def test_tied_scores_take_the_radix_passes():
    # a zero query scores every community 0: the boundary bin of the linear
    # pass holds all 1500 communities, so the selection narrows it by radix
    # passes down to the ids (equal scores keep the lower ids first)
    cfg = synth.scaled(synth.TINY, n0=24000, n_clusters=1500, budget=6000, steps=3)
    assert cfg.n_comm > 1024
    wl = synth.make_workload(cfg, workers=WORKERS)
    wl.q[:] = 0
    ls = Lockstep(wl)
    try:
        for i in range(cfg.steps):
            ls.step(i)
        ls.compare_state()
    finally:
        ls.close()


def test_one_community_far_above_the_rest():
    # one community's keys far along the query direction: its score sits far
    # above every other, so the upper half of the score range holds only it
    # (less than the budget) and the linear histogram crowds every other
    # community into its lowest bins; the boundary lies among them.
    cfg = synth.scaled(synth.TINY, n0=8000, n_clusters=400, budget=600, steps=4)
    wl = synth.make_workload(cfg, workers=WORKERS)
    S, D = cfg.n_sinks, cfg.head_dim
    rng = np.random.default_rng(synth.BASE_SEED + 91)
    u = rng.standard_normal(D)
    u /= np.linalg.norm(u)
    lab = wl.labels[0]
    c_star = int(lab[S])
    members = np.nonzero(lab[S:cfg.n0] == c_star)[0] + S
    wl.K[0, 0, members] = (30.0 * u).astype(np.float32)
    wl.q[:, 0, 0] = (u + 0.01 * rng.standard_normal((cfg.steps, D))).astype(np.float32)
    # the case holds at the first step: the initial centroids (member means)
    # that score in the upper half of the range hold no more than the budget
    pos = np.arange(S, cfg.n0)
    mu = np.zeros((cfg.n_comm, D))
    size = np.zeros(cfg.n_comm, np.int64)
    np.add.at(mu, lab[pos], wl.K[0, 0, pos].astype(np.float64))
    np.add.at(size, lab[pos], 1)
    live = size > 0
    sc = (mu[live] / size[live, None]) @ wl.q[0, 0, 0].astype(np.float64)
    upper = sc >= sc.min() + 0.5 * (sc.max() - sc.min())
    assert size[live][upper].sum() <= cfg.budget < size.sum()
    ls = Lockstep(wl)
    try:
        for i in range(cfg.steps):
            ls.step(i)
        ls.compare_state()
    finally:
        ls.close()


def test_small_slack_relocates_segments():
    # slack 0: every append past the initial size moves the community segment
    cfg = synth.scaled(synth.TINY, n0=512, n_clusters=2, steps=40)
    run_lockstep(cfg, slack=0)


@pytest.mark.parametrize("mode", [synth.PER_HEAD, synth.QUERY_GROUP])
def test_small_gqa_both_modes(mode):
    cfg = synth.scaled(synth.LLAMA, batch=2, n_q_heads=8, n_kv_heads=2, n0=4000, n_clusters=125,
                       budget=300, steps=12, mode=mode)
    run_lockstep(cfg)


@pytest.mark.parametrize("group,bf16", [(2, True), (8, True), (4, False), (8, False)])
def test_query_group_sizes(group, bf16):
    # query groups of 2 and 8 heads per graph (the tensor-core path) and the
    # fp32 CUDA-core path with 4 and 8 heads per graph
    cfg = synth.scaled(synth.LLAMA, batch=2, n_q_heads=2 * group, n_kv_heads=2, n0=3000, n_clusters=100,
                       budget=300, steps=10, mode=synth.QUERY_GROUP, bf16=bf16)
    run_lockstep(cfg)


@pytest.mark.parametrize("name", ["tiny_fp32", "gqa_bf16", "qwen8b_sampled"])
def test_single_launch_step(name, monkeypatch):
    """The whole step as one persistent kernel (CKV_STEP=fused: score items,
    selection and finish workers, attention items) in lockstep with the
    oracle."""
    monkeypatch.setenv("CKV_STEP", "fused")
    if name == "tiny_fp32":
        run_lockstep(synth.TINY)
    elif name == "gqa_bf16":
        run_lockstep(synth.scaled(synth.LLAMA, batch=2, n_q_heads=8, n_kv_heads=2, n0=4000, n_clusters=125,
                                  budget=300, steps=12, mode=synth.QUERY_GROUP))
    else:
        run_lockstep(synth.scaled(synth.QWEN8B, steps=16), tracked=[0, 13, 26, 31], compare_every=0)


def test_llama_per_head_full():
    run_lockstep(synth.LLAMA, compare_every=16)


def test_qwen8b_query_group_full_size_sampled():
    # full size, all 128 steps on the GPU; the oracle follows 8 of the 32
    # graphs: two KV heads of each of the 4 sequences
    run_lockstep(synth.QWEN8B, tracked=[0, 5, 10, 15, 17, 22, 27, 30], compare_every=0)


# the batch-16 sweep: every (n, budget) point, all 32 steps, 16 of the 128
# graphs tracked (every sequence once, every KV head twice).  The workload
# does not depend on the budget, so the four budgets of one n share one
# draw.
SWEEP_TRACKED = [8 * i + (i % 8) if i < 8 else 8 * i + ((i + 3) % 8) for i in range(16)]
_sweep_wl = {}


def _sweep_workload(n):
    if n not in _sweep_wl:
        _sweep_wl.clear()                                # one n resident at a time
        _sweep_wl[n] = synth.make_workload(synth.sweep_config(n, 128), workers=WORKERS)
    return _sweep_wl[n]


@pytest.mark.parametrize("n,budget", [(n, t) for n in (8192, 32768, 131072) for t in (128, 512, 1024, 4096)])
def test_sweep_point(n, budget):
    cfg = synth.sweep_config(n, budget)
    base = _sweep_workload(n)
    assert dataclasses.replace(base.cfg, budget=budget, name=cfg.name) == cfg
    wl = synth.Workload(cfg, base.K, base.V, base.q, base.labels)
    ls = run_lockstep(cfg, tracked=SWEEP_TRACKED, compare_every=0, wl=wl)
    assert len(ls.logs) == 32
    if n == 131072 and budget == 4096:
        _sweep_wl.clear()


# ----------------------------------------------------------------- boundary
def _small_ctx(slack=16, pool_capacity=0, cfg=None):
    import torch
    cfg = cfg or synth.scaled(synth.TINY, n0=256, n_clusters=8, steps=4)
    wl = synth.make_workload(cfg)
    dev = torch.device("cuda", 0)
    K, V, q = _torch_view(wl.K, dev), _torch_view(wl.V, dev), _torch_view(wl.q, dev)
    ctx = ckv.ckv_create(config_for(cfg, 0, slack, pool_capacity))
    out = torch.empty((cfg.batch, cfg.n_q_heads, 128), dtype=torch.float32, device=dev)
    return cfg, wl, ctx, K, V, q, out


def test_call_order_and_arguments_checked():
    cfg, wl, ctx, K, V, q, out = _small_ctx()
    try:
        with pytest.raises(ckv.CkvError) as e:          # step before init
            ckv.ckv_decode_step(ctx, q[0], K, V, cfg.n0 + 1, out)
        assert e.value.status == ckv.CKV_ERR_STATE
        bad = wl.labels.copy()
        bad[0, 100] = cfg.n_comm                        # label out of range
        with pytest.raises(ckv.CkvError) as e:
            ckv.ckv_init_communities(ctx, bad, 0, cfg.n_comm, K, cfg.n0)
        assert e.value.status == ckv.CKV_ERR_INVALID_ARG
        ckv.ckv_init_communities(ctx, wl.labels, 0, cfg.n_comm, K, cfg.n0)
        with pytest.raises(ckv.CkvError) as e:          # wrong n
            ckv.ckv_decode_step(ctx, q[0], K, V, cfg.n0 + 2, out)
        assert e.value.status == ckv.CKV_ERR_STATE
        with pytest.raises(ckv.CkvError) as e:          # update without a step
            ckv.ckv_assign_update(ctx, K, cfg.n0 + 1)
        assert e.value.status == ckv.CKV_ERR_STATE
        ckv.ckv_decode_step(ctx, q[0], K, V, cfg.n0 + 1, out)
        with pytest.raises(ckv.CkvError) as e:          # second step before the update
            ckv.ckv_decode_step(ctx, q[1], K, V, cfg.n0 + 2, out)
        assert e.value.status == ckv.CKV_ERR_STATE
        ckv.ckv_assign_update(ctx, K, cfg.n0 + 1)
        assert ckv.ckv_last_error(ctx) == ckv.CKV_OK
        with pytest.raises(ckv.CkvError):               # corrupt checkpoint
            blob = bytearray(ckv.ckv_export_state(ctx))
            blob[36 + 4 * cfg.n_comm * 128] = 0xFF      # first size -> negative
            blob[36 + 4 * cfg.n_comm * 128 + 3] = 0xFF
            ckv.ckv_import_state(ctx, bytes(blob))
    finally:
        ckv.ckv_destroy(ctx)


def test_capacity_error_is_sticky_and_state_unchanged():
    cfg = synth.scaled(synth.TINY, n0=256, n_clusters=1, steps=20)
    # pool just large enough for the initial segments: the first relocation fails
    cfg_, wl, ctx, K, V, q, out = _small_ctx(slack=0, pool_capacity=256, cfg=cfg)
    try:
        ckv.ckv_init_communities(ctx, wl.labels, 0, cfg.n_comm, K, cfg.n0)
        before = ckv_state.parse(ckv.ckv_export_state(ctx))
        ckv.ckv_decode_step(ctx, q[0], K, V, cfg.n0 + 1, out)
        ckv.ckv_assign_update(ctx, K, cfg.n0 + 1)
        assert ckv.ckv_last_error(ctx) == ckv.CKV_ERR_CAPACITY
        with pytest.raises(ckv.CkvError) as e:          # sticky
            ckv.ckv_decode_step(ctx, q[1], K, V, cfg.n0 + 2, out)
        assert e.value.status == ckv.CKV_ERR_CAPACITY
        ckv.ckv_import_state(ctx, ckv_state.pack(before))   # import clears it
        assert ckv.ckv_last_error(ctx) == ckv.CKV_OK
        after = ckv_state.parse(ckv.ckv_export_state(ctx))
        np.testing.assert_array_equal(after.sizes, before.sizes)
        np.testing.assert_array_equal(after.centroids, before.centroids)
    finally:
        ckv.ckv_destroy(ctx)


def test_deterministic_and_checkpoint_roundtrip():
    import torch
    cfg = synth.scaled(synth.LLAMA, batch=1, n_q_heads=8, n_kv_heads=2, n0=3000, n_clusters=150,
                       budget=256, steps=6, mode=synth.QUERY_GROUP)
    wl = synth.make_workload(cfg)
    dev = torch.device("cuda", 0)
    K, V, q = _torch_view(wl.K, dev), _torch_view(wl.V, dev), _torch_view(wl.q, dev)
    outs, blobs = [], []
    for rep in range(2):
        ctx = ckv.ckv_create(config_for(cfg))
        o = torch.empty((1, 8, 128), dtype=torch.float32, device=dev)
        ckv.ckv_init_communities(ctx, wl.labels, 0, cfg.n_comm, K, cfg.n0)
        got = []
        mid = None
        for i in range(cfg.steps):
            if i == 3:
                mid = ckv.ckv_export_state(ctx)
            ckv.ckv_decode_step(ctx, q[i], K, V, cfg.n0 + i + 1, o)
            ckv.ckv_assign_update(ctx, K, cfg.n0 + i + 1)
            got.append(o.cpu().numpy().copy())
        blobs.append(ckv.ckv_export_state(ctx))
        outs.append(np.stack(got))
        # resume from the mid-run checkpoint and replay the last steps
        ckv.ckv_import_state(ctx, mid)
        for i in range(3, cfg.steps):
            ckv.ckv_decode_step(ctx, q[i], K, V, cfg.n0 + i + 1, o)
            ckv.ckv_assign_update(ctx, K, cfg.n0 + i + 1)
            assert np.array_equal(o.cpu().numpy(), got[i])
        assert ckv.ckv_export_state(ctx) == blobs[-1]
        ckv.ckv_destroy(ctx)
    assert np.array_equal(outs[0], outs[1])
    assert blobs[0] == blobs[1]


def test_host_buffer_step_matches_device_step():
    import torch
    cfg = synth.scaled(synth.LLAMA, batch=2, n_q_heads=8, n_kv_heads=2, n0=2000, n_clusters=100,
                       budget=256, steps=5, mode=synth.QUERY_GROUP)
    wl = synth.make_workload(cfg)
    dev = torch.device("cuda", 0)
    K, V, q = _torch_view(wl.K, dev), _torch_view(wl.V, dev), _torch_view(wl.q, dev)
    K2 = K.clone()
    V2 = V.clone()
    K2[:, :, cfg.n0:] = 0                                   # the host path writes these rows
    V2[:, :, cfg.n0:] = 0
    a = ckv.ckv_create(config_for(cfg))
    b = ckv.ckv_create(config_for(cfg))
    try:
        ckv.ckv_init_communities(a, wl.labels, 0, cfg.n_comm, K, cfg.n0)
        ckv.ckv_init_communities(b, wl.labels, 0, cfg.n_comm, K2, cfg.n0)
        o = torch.empty((2, 8, 128), dtype=torch.float32, device=dev)
        oh = torch.empty((2, 8, 128), dtype=torch.float32).pin_memory()
        for i in range(cfg.steps):
            n = cfg.n0 + i + 1
            ckv.ckv_decode_step(a, q[i], K, V, n, o)
            ckv.ckv_assign_update(a, K, n)
            qh = torch.from_numpy(wl.q[i].copy()).pin_memory()
            kh = torch.from_numpy(np.ascontiguousarray(wl.K[:, :, n - 1])).pin_memory()
            vh = torch.from_numpy(np.ascontiguousarray(wl.V[:, :, n - 1])).pin_memory()
            ckv.ckv_decode_host(b, qh, kh, vh, K2, V2, n, oh)
            assert np.array_equal(oh.numpy(), o.cpu().numpy())
        assert torch.equal(K2, K) and torch.equal(V2, V)
        assert ckv.ckv_export_state(a) == ckv.ckv_export_state(b)
    finally:
        ckv.ckv_destroy(a)
        ckv.ckv_destroy(b)


@pytest.mark.parametrize("captured", [False, True])
def test_per_kernel_profile_eager_and_captured(captured):
    """ckv_profile_begin/end time each kernel of eager and graph-captured steps;
    profiling changes no result."""
    import torch
    cfg, wl, ctx, K, V, q, out = _small_ctx()
    ref_ctx = ckv.ckv_create(config_for(cfg))
    try:
        ckv.ckv_init_communities(ctx, wl.labels, 0, cfg.n_comm, K, cfg.n0)
        ckv.ckv_init_communities(ref_ctx, wl.labels, 0, cfg.n_comm, K, cfg.n0)
        ref = torch.empty_like(out)
        ckv.ckv_profile_begin(ctx)
        steps = range(cfg.steps)
        if captured:
            side = torch.cuda.Stream()
            graph = torch.cuda.CUDAGraph()
            with torch.cuda.stream(side), torch.cuda.graph(graph, stream=side, capture_error_mode="relaxed"):
                for i in steps:
                    ckv.ckv_decode_step(ctx, q[i], K, V, cfg.n0 + i + 1, out, side.cuda_stream)
                    ckv.ckv_assign_update(ctx, K, cfg.n0 + i + 1, side.cuda_stream)
            graph.replay()
        else:
            for i in steps:
                ckv.ckv_decode_step(ctx, q[i], K, V, cfg.n0 + i + 1, out)
                ckv.ckv_assign_update(ctx, K, cfg.n0 + i + 1)
        torch.cuda.synchronize()
        ms, n = ckv.ckv_profile_end(ctx)
        assert n == cfg.steps
        # the fused step has one kernel: its time is ms[0], the selection
        # and attention spans are then empty; ms[3] is the update kernel's
        # when ckv_assign_update launches one
        launches = ckv.ckv_step_launches(ctx)
        timed = ms[:1] if launches == 1 else ms[:launches]
        assert all(m > 0.0 for m in timed) and all(m >= 0.0 for m in ms) and sum(ms) < 1000.0 * n
        for i in steps:
            ckv.ckv_decode_step(ref_ctx, q[i], K, V, cfg.n0 + i + 1, ref)
            ckv.ckv_assign_update(ref_ctx, K, cfg.n0 + i + 1)
        torch.cuda.synchronize()
        assert torch.equal(out, ref)
        assert ckv.ckv_export_state(ctx) == ckv.ckv_export_state(ref_ctx)
    finally:
        ckv.ckv_destroy(ctx)
        ckv.ckv_destroy(ref_ctx)


def test_update_on_a_second_stream_matches_inline(monkeypatch):
    """ckv_assign_update's kernel run on a second stream, each step of the
    context waiting for the previous update by an event (as a decoder
    overlapping it with the next layer does), gives bit for bit the outputs
    and state of the inline update (CKV_UPDATE=inline: the attention
    kernel's last slice runs the edges, assignment and update)."""
    import torch
    cfg = synth.scaled(synth.LLAMA, batch=2, n_q_heads=8, n_kv_heads=2, n0=4000, n_clusters=125,
                       budget=300, steps=8, mode=synth.QUERY_GROUP)
    wl = synth.make_workload(cfg)
    dev = torch.device("cuda", 0)
    K, V, q = _torch_view(wl.K, dev), _torch_view(wl.V, dev), _torch_view(wl.q, dev)
    # the same attention kernel in both (the cluster variant slices the rows
    # differently, so its sums round differently)
    monkeypatch.setenv("CKV_ATT_CLUSTER", "0")
    deferred = ckv.ckv_create(config_for(cfg))
    monkeypatch.setenv("CKV_UPDATE", "inline")
    inline = ckv.ckv_create(config_for(cfg))
    try:
        assert ckv.ckv_step_launches(deferred) == 4 and ckv.ckv_step_launches(inline) == 3
        for c in (deferred, inline):
            ckv.ckv_init_communities(c, wl.labels, 0, cfg.n_comm, K, cfg.n0)
        main, side = torch.cuda.Stream(), torch.cuda.Stream()
        ev_a, ev_u = torch.cuda.Event(), torch.cuda.Event()
        out_d = torch.empty((cfg.batch, cfg.n_q_heads, 128), dtype=torch.float32, device=dev)
        out_i = torch.empty_like(out_d)
        for i in range(cfg.steps):
            n = cfg.n0 + i + 1
            if i:
                main.wait_event(ev_u)
            ckv.ckv_decode_step(deferred, q[i], K, V, n, out_d, main.cuda_stream)
            ev_a.record(main)
            side.wait_event(ev_a)
            ckv.ckv_assign_update(deferred, K, n, side.cuda_stream)
            ev_u.record(side)
            ckv.ckv_decode_step(inline, q[i], K, V, n, out_i)
            ckv.ckv_assign_update(inline, K, n)
            main.synchronize()
            torch.cuda.synchronize()
            assert torch.equal(out_d, out_i), f"step {i}: outputs differ"
        torch.cuda.synchronize()
        assert ckv.ckv_last_error(deferred) == ckv.CKV_OK and ckv.ckv_last_error(inline) == ckv.CKV_OK
        assert ckv.ckv_export_state(deferred) == ckv.ckv_export_state(inline)
    finally:
        ckv.ckv_destroy(deferred)
        ckv.ckv_destroy(inline)

