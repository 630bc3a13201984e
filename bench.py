#!/usr/bin/env python
"""Decode-step throughput of libckv on B200 (CommunityKV community-retrieval
sparse decode, "CommunityKV: Efficient Long-Context Decoding via Graph
Partitioning", Figure 1 step (3)).

Workload: Qwen3-8B-shaped decode with query-group graphs -- batch 4, 32 query
heads over 8 KV heads, head_dim 128, bf16 K/V, n = 131072 context tokens,
communities of 16 (8192 per graph), 4 sinks, budget 4096, kappa 8; seeded
synthetic clustered keys (long_context_decode_ckv_b200.synth).

A step = ckv_decode_step + ckv_assign_update for all 32 graphs of one layer.
The timed loop rotates over `--replicas` independent copies of the layer
(separate K/V caches and community state, > 18 GB in total), so no step finds
its working set in the 126 MB L2: inputs larger than L2, no flush.

After the timed steps it also reports, outside the timed region, the
attention-mass recall of each replica's last step (Figure 3 right: the dense
softmax mass of the attended rows, per query head) and the time of a dense
decode attention over the whole cache (the comparator of the sparse step).

Prints one JSON line (rank 0).  `--impl reference` times the CPU oracle
(test infrastructure; the only other code here that runs it is the
cpu_baseline leg) on the same workload instead.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from long_context_decode_ckv_b200 import synth  # noqa: E402

CFG = synth.QWEN8B
WORKLOAD = "qwen3_8b_shape_query_group_b4_h32kv8_d128_n131072_budget4096_k8_s4_bf16"
METRIC = "decode steps/s"
NOMINAL_HBM_GBS = 8000.0


def algorithmic_bytes(cfg, T):
    """Bytes one step must move, per graph (T = member tokens kept):
    centroids N_c*D*4, community offset+size N_c*8, member ids T*4, K and V
    rows (T+S+1)*D*2*2, queries in and outputs out |H(g)|*D*(2+4)."""
    Nc, D, S, hg = cfg.n_comm, cfg.head_dim, cfg.n_sinks, cfg.heads_per_graph
    eb = 2 if cfg.bf16 else 4
    return (Nc * D * 4 + Nc * 8 + T * 4 + (T + S + 1) * D * eb * 2 + hg * D * (eb + 4))


def kernel_bytes(cfg, T):
    """Algorithmic bytes of the two streaming kernels per graph."""
    Nc, D, S, hg = cfg.n_comm, cfg.head_dim, cfg.n_sinks, cfg.heads_per_graph
    eb = 2 if cfg.bf16 else 4
    return {
        "score": Nc * D * 4 + Nc * 4 + Nc * 4,                         # centroids, sizes, scores out
        "attend": (T + S + 1) * D * eb * 2 + T * 4 + hg * D * (eb + 4),  # K/V rows, ids, q, out
    }


# DRAM bytes read + written per launch from one ncu capture (profiles/), each
# valid only while the sources that define that kernel are the ones the
# capture was taken on (source_hash over KERNEL_SOURCES of the kernel)
KERNEL_SOURCES = {
    "k_score": ("k_decode.cu", "warp_mma.cuh", "dev_async.cuh", "ckv_internal.cuh"),
    "k_attend": ("k_decode.cu", "warp_mma.cuh", "dev_async.cuh", "ckv_internal.cuh"),
    "k_dense_stats": ("k_dense.cu", "warp_mma.cuh", "dev_async.cuh", "ckv_internal.cuh"),
    "k_dense_attention": ("k_dense.cu", "warp_mma.cuh", "dev_async.cuh", "ckv_internal.cuh"),
}
PROFILED_TRAFFIC = {
    "k_score": ("88429c0b21494fe5", 138.591232e6),
    "k_attend": ("88429c0b21494fe5", 67.92192e6),
    "k_dense_stats": ("1674ed41fb19dce3", 1079.90176e6),
}


def source_hash(files):
    """First 16 hex digits of the SHA-256 over the given CUDA sources of the
    library (in order, each with its name)."""
    import hashlib
    h = hashlib.sha256()
    for f in files:
        h.update(f.encode())
        h.update(open(os.path.join(ROOT, "long_context_decode_ckv_b200", "csrc", f), "rb").read())
    return h.hexdigest()[:16]


def profiled_traffic(kernel):
    """DRAM bytes per launch from the ncu capture, only while the kernel's
    sources are the ones it was taken on."""
    if kernel not in PROFILED_TRAFFIC:
        return None
    try:
        h = source_hash(KERNEL_SOURCES[kernel])
    except OSError:
        return None
    sha, traffic = PROFILED_TRAFFIC[kernel]
    return traffic if h == sha else None


def measured_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return float(d["hbm_gbs"]), "measured"
    return 6650.0, "fallback"


class Clocks:
    """nvidia-smi samples during the timed region."""

    def __init__(self, index: int):
        self.index, self.rows, self.proc = index, [], None

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.index}",
                 "--query-gpu=clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
                 "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
                 "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
        except OSError:
            self.proc = None
        time.sleep(0.25)
        return self

    def _read(self):
        for line in self.proc.stdout:
            self.rows.append([c.strip() for c in line.split(",")])

    def __exit__(self, *exc):
        time.sleep(0.15)
        if self.proc:
            self.proc.terminate()
            self.proc.wait(timeout=5)
            self.thread.join(timeout=2)

    def summary(self):
        if not self.rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        sm = [float(r[0]) for r in self.rows if r[0].replace(".", "").isdigit()]
        mx = [float(r[1]) for r in self.rows if r[1].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[k] for r in self.rows for k in range(4)
                          if len(r) > 4 + k and r[4 + k].lower() == "active"})
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(mx) if mx else None, "reasons": reasons,
                "samples": len(self.rows)}


# ------------------------------------------------------------ ranks (N > 1)
def rank_env():
    """(rank, world size, local rank) from the launcher's environment."""
    return (int(os.environ.get("RANK", 0)), int(os.environ.get("WORLD_SIZE", 1)),
            int(os.environ.get("LOCAL_RANK", 0)))


def max_over_ranks(dist, value, device):
    """The largest of every rank's value (each rank's device time: the job
    takes as long as its slowest replica)."""
    if dist is None:
        return value
    import torch
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_rate(world, steps, ms):
    """Whole-job steps/s: every rank ran `steps` steps of its own replica in
    at most `ms` milliseconds (weak scaling)."""
    return world * steps / (ms / 1e3)


# ------------------------------------------------------------------ oracle
def host_cores():
    return len(os.sched_getaffinity(0)) if hasattr(os, "sched_getaffinity") else (os.cpu_count() or 1)


class OracleSteps:
    """The CPU oracle on the decode workload, graph by graph.  The graphs of
    a step are independent, so with threads > 1 they run on a thread pool
    (each oracle call is one C call that releases the GIL); a step ends when
    all its graphs are done."""

    def __init__(self, wl, threads=1, graphs=None):
        import oracle
        from concurrent.futures import ThreadPoolExecutor
        self.oracle, self.wl, self.cfg = oracle, wl, wl.cfg
        cfg = wl.cfg
        self.graphs = list(range(cfg.n_graphs)) if graphs is None else list(graphs)
        self.og = {}
        for g in self.graphs:
            b, kvh, _ = cfg.graph_heads(g)
            self.og[g] = oracle.Graph(cfg.n_comm, cfg.head_dim, cfg.n_max)
            self.og[g].init(cfg.n0, cfg.n_sinks, wl.labels[g], wl.K[b, kvh])
        self.threads = max(1, min(threads, len(self.graphs)))
        self.pool = ThreadPoolExecutor(self.threads) if self.threads > 1 else None

    def _one(self, i, g):
        cfg, wl = self.cfg, self.wl
        b, kvh, heads = cfg.graph_heads(g)
        self.oracle.decode_step(self.og[g], np.ascontiguousarray(wl.q[i, b, heads]), wl.K[b, kvh],
                                wl.V[b, kvh], cfg.n0 + i + 1, cfg.n_sinks, cfg.kappa, cfg.budget)

    def step(self, i):
        if self.pool is None:
            for g in self.graphs:
                self._one(i, g)
        else:
            list(self.pool.map(lambda g: self._one(i, g), self.graphs))

    def close(self):
        if self.pool is not None:
            self.pool.shutdown()


def run_oracle_steps(wl, n_steps, threads=1, first=0):
    """Time the CPU oracle on decode steps [first, first + n_steps) of the
    workload (steps before `first` run untimed); returns seconds."""
    o = OracleSteps(wl, threads)
    try:
        for i in range(first):
            o.step(i)
        t0 = time.perf_counter()
        for i in range(first, first + n_steps):
            o.step(i)
        return time.perf_counter() - t0
    finally:
        o.close()


def prefill_oracle_time(P, Q, K, rows_per_head=2048, threads=1):
    """The prefill oracle (top-kappa rows of every head) on a bounded sample:
    `rows_per_head` rows spread evenly over [0, n) of each head, split over
    `threads` threads.  A row i costs (i + 1) key dots, so the time is scaled
    to all n rows by the ratio of summed row lengths.  Returns (seconds
    measured, seconds extrapolated to the whole prefill, sample note)."""
    import oracle
    from concurrent.futures import ThreadPoolExecutor
    n, H = P.n, P.n_heads
    rows = np.unique(np.linspace(0, n - 1, rows_per_head).round().astype(np.int32))
    chunks = [(h, c) for h in range(H) for c in np.array_split(rows, max(1, threads // H + 1))]

    def work(hc):
        h, r = hc
        oracle.prefill_rows(Q[h], K[h], r, P.n_sinks, P.kappa)

    t0 = time.perf_counter()
    with ThreadPoolExecutor(max(1, threads)) as ex:
        list(ex.map(work, chunks))
    secs = time.perf_counter() - t0
    scale = (n * (n + 1) / 2) / float((rows.astype(np.float64) + 1).sum())
    return secs, secs * scale, (f"{len(rows)} rows evenly spread over n={n} x {H} heads, "
                                f"{threads} threads, scaled x{scale:.2f} by summed row length")


def reference_arm(args, rank, world):
    if rank != 0:
        return 0
    wl = synth.make_workload(CFG, workers=max(1, min(16, os.cpu_count() or 1)))
    steps = args.warmup + args.steps
    if steps > CFG.steps:
        raise SystemExit(f"--impl reference supports at most {CFG.steps} steps")
    cores = host_cores()
    dt = run_oracle_steps(wl, args.steps, threads=cores, first=args.warmup)
    v = args.steps / dt
    sample = (f"{args.steps} full decode steps (all {CFG.n_graphs} graphs, one thread per graph on "
              f"{min(cores, CFG.n_graphs)} of {cores} host cores) after {args.warmup} warm-up steps")
    print(json.dumps({
        "impl": "reference", "metric": METRIC, "value": v, "unit": "steps/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * dt / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic", "config": {"workload": WORKLOAD},
        "cpu_baseline": {"value": v, "unit": "steps/s", "cores": min(cores, CFG.n_graphs), "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": v, "unit": "steps/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }), flush=True)
    return 0


# ------------------------------------------------------------------ GPU arm
class Stepper:
    """Decode steps over layer replicas: ckv_decode_step on the caller's
    stream, ckv_assign_update (the edges, assignment and update kernel) on a
    side stream, so that it overlaps the next replica's step the way a
    decoder overlaps it with the next layer; a replica's next step waits for
    its previous update (events; also inside CUDA graph capture)."""

    def __init__(self, reps, q, out, cfg, dev, side=True):
        import torch
        import long_context_decode_ckv_b200 as ckv
        self.ckv, self.reps, self.q, self.out, self.cfg = ckv, reps, q, out, cfg
        self.side = torch.cuda.Stream(device=dev) if side else None
        self.ev_a = [torch.cuda.Event() for _ in reps]
        self.ev_u = [torch.cuda.Event() for _ in reps]
        self.pending = [False] * len(reps)

    def step(self, s, st):
        ckv, cfg = self.ckv, self.cfg
        r = s % len(self.reps)
        rep = self.reps[r]
        i = rep["i"]
        n = cfg.n0 + i + 1
        if self.side is None:   # both calls on the caller's stream
            ckv.ckv_decode_step(rep["ctx"], self.q[i], rep["K"], rep["V"], n, self.out, st)
            ckv.ckv_assign_update(rep["ctx"], rep["K"], n, st)
            rep["i"] = i + 1
            return
        if self.pending[r]:
            st.wait_event(self.ev_u[r])
        ckv.ckv_decode_step(rep["ctx"], self.q[i], rep["K"], rep["V"], n, self.out, st)
        self.ev_a[r].record(st)
        self.side.wait_event(self.ev_a[r])
        ckv.ckv_assign_update(rep["ctx"], rep["K"], n, self.side)
        self.ev_u[r].record(self.side)
        self.pending[r] = True
        rep["i"] = i + 1

    def join(self, st):
        """The caller's stream waits for every update still outstanding."""
        for r, p in enumerate(self.pending):
            if p:
                st.wait_event(self.ev_u[r])
                self.pending[r] = False


def hold(stream, us=500.0):
    """Enqueues a spin kernel of about `us` microseconds (torch's) on
    `stream`, ahead of a start event: the host's submission of the timed
    launches overlaps it, so that the events time the device work and not
    an idle device waiting for the host."""
    import torch
    with torch.cuda.stream(stream):
        torch.cuda._sleep(int(us * 2000))   # cycles, at about 2 GHz


def upload_graph(g, stream):
    """Uploads an instantiated CUDA graph to the device ahead of its first
    launch (a one-time setup cost, like the instantiation), so that the
    timed replay runs only the captured steps."""
    from cuda.bindings import runtime as cudart
    err, = cudart.cudaGraphUpload(g.raw_cuda_graph_exec(), stream.cuda_stream)
    if int(err) != 0:
        raise RuntimeError(f"cudaGraphUpload failed: {err}")
    stream.synchronize()


def bf16_peak_tflops():
    pp = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(pp):
        v = float(json.load(open(pp)).get("bf16_tflops", 0) or 0)
        if v:
            return v, "measured"
    return 1590.0, "fallback"


def prefill_measure(steps, warmup, P=synth.PREFILL):
    """Figure 1 step (1): the prefill top-kappa graph of the 8-head n=16384
    workload, per head (ckv_build_graph) and per KV head of 4 query heads
    (ckv_build_graph_grouped); device time per call with CUDA events over
    `steps` calls after `warmup`, and the causal Q K^T flops it implies
    against the measured bf16 peak (burst: each call is timed alone)."""
    import torch
    import long_context_decode_ckv_b200 as ckv
    from long_context_decode_ckv_b200 import build as ckv_build
    Q, K = synth.make_prefill(P)
    ckv_build.build()
    dev = torch.device("cuda", torch.cuda.current_device())
    q = torch.from_numpy(Q).view(torch.bfloat16).to(dev)
    k = torch.from_numpy(K).view(torch.bfloat16).to(dev)
    n, H, S, kap = P.n, P.n_heads, P.n_sinks, P.kappa
    E = int(np.clip(np.arange(n) - S, 0, kap).sum())
    causal_flops = 2.0 * 128 * n * (n + 1) / 2 * H          # one Q K^T over the causal triangle, all heads
    stream = torch.cuda.current_stream(dev)

    def timed(fn):
        for _ in range(warmup):
            fn()
        torch.cuda.synchronize(dev)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        hold(stream)
        e0.record(stream)
        for _ in range(steps):
            fn()
        e1.record(stream)
        torch.cuda.synchronize(dev)
        return e0.elapsed_time(e1) / steps

    rp = torch.empty((H, n + 1), dtype=torch.int64, device=dev)
    col = torch.empty((H, E), dtype=torch.int32, device=dev)
    w = torch.empty((H, E), dtype=torch.float32, device=dev)
    ms_head = timed(lambda: ckv.ckv_build_graph(H, n, 128, S, kap, ckv.CKV_BF16, q, k, rp, col, w))
    Hkv, g = H // 4, 4
    ws = torch.empty(ckv.ckv_build_graph_grouped_workspace(Hkv, g, n), dtype=torch.uint8, device=dev)
    kk = k[:Hkv].contiguous()
    ms_group = timed(lambda: ckv.ckv_build_graph_grouped(Hkv, g, n, 128, S, kap, ckv.CKV_BF16, q, kk, ws,
                                                         rp[:Hkv], col[:Hkv], w[:Hkv]))
    peak, peak_kind = bf16_peak_tflops()
    tf_head = causal_flops / (ms_head / 1e3) / 1e12
    tf_group = 2 * causal_flops / (ms_group / 1e3) / 1e12   # statistics pass + grouped pass
    res = {
        "workload": "prefill_8h_n16384_k8_s4_bf16", "steps": steps, "warmup": warmup,
        "ms": ms_head, "kernel": "k_prefill_topk",
        "roofline": {"bound": "tensor", "achieved": tf_head, "peak": peak, "unit": "TFLOP/s",
                     "frac": tf_head / peak, "peak_kind": peak_kind + " bf16 burst",
                     "flops_per_launch": causal_flops},
        "query_group_4": {"ms": ms_group, "tflops_both_passes": tf_group, "frac": tf_group / peak},
        "exp2_count": n * (n + 1) / 2 * H,
    }
    del q, k, rp, col, w, ws, kk
    torch.cuda.empty_cache()
    return res, (Q, K)


def prefill_bench(args):
    res, _ = prefill_measure(args.steps, args.warmup)
    print(json.dumps({"metric": "prefill graph ms", **res}), flush=True)
    return 0


def decode_rate(cfg, wl, warmup, steps, replicas, profile_steps=0):
    """Decode steps/s of one more workload (cfg, wl already drawn): `replicas`
    independent layer copies rotated (inputs larger than L2), `warmup`
    eager steps, then `steps` steps captured into a CUDA graph and timed
    with events on the launching stream; optionally `profile_steps` more
    with per-kernel events.  Returns a dict with the rate, GB/s and the
    dominant kernel's roofline."""
    import torch
    import long_context_decode_ckv_b200 as ckv
    dev = torch.device("cuda", torch.cuda.current_device())
    stream = torch.cuda.current_stream(dev)
    L = replicas
    if -(-(warmup + steps + profile_steps) // L) > cfg.steps:
        raise SystemExit(f"{cfg.name}: not enough decode tokens for these steps")

    def upload(a):
        t = torch.from_numpy(a)
        return (t.view(torch.bfloat16) if a.dtype == np.uint16 else t).to(dev)

    K0, V0, q = upload(wl.K), upload(wl.V), upload(wl.q)
    reps = []
    c = ckv.ckv_config()
    c.batch, c.n_q_heads, c.n_kv_heads, c.head_dim = cfg.batch, cfg.n_q_heads, cfg.n_kv_heads, cfg.head_dim
    c.n_max, c.max_communities, c.n_sinks = cfg.n_max, cfg.n_comm, cfg.n_sinks
    c.kappa, c.budget, c.slack = cfg.kappa, cfg.budget, 16
    c.kv_dtype = ckv.CKV_BF16 if cfg.bf16 else ckv.CKV_F32
    c.mode = ckv.CKV_QUERY_GROUP if cfg.mode == synth.QUERY_GROUP else ckv.CKV_PER_HEAD
    c.device, c.pool_capacity = dev.index, 0
    try:
        for r in range(L):
            K = K0 if r == 0 else K0.clone()
            V = V0 if r == 0 else V0.clone()
            ctx = ckv.ckv_create(c)
            reps.append({"ctx": ctx, "K": K, "V": V, "i": 0})
            ckv.ckv_init_communities(ctx, wl.labels, 0, cfg.n_comm, K, cfg.n0)
        aux, kvb = ckv.ckv_aux_bytes(reps[0]["ctx"])
        out = torch.empty((cfg.batch, cfg.n_q_heads, cfg.head_dim), dtype=torch.float32, device=dev)
        stepper = Stepper(reps, q, out, cfg, dev)

        def graph_of(first, count):
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, capture_error_mode="relaxed"):
                cap = torch.cuda.current_stream(dev)
                for s in range(first, first + count):
                    stepper.step(s, cap)
                stepper.join(cap)
            upload_graph(g, stream)
            return g

        for s in range(warmup):
            stepper.step(s, stream)
        stepper.join(stream)
        torch.cuda.synchronize(dev)
        g = graph_of(warmup, steps)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        torch.cuda.synchronize(dev)
        hold(stream)
        e0.record(stream)
        g.replay()
        e1.record(stream)
        torch.cuda.synchronize(dev)
        ms = e0.elapsed_time(e1) / steps
        del g
        avg = None
        if profile_steps:
            for r in reps:
                ckv.ckv_profile_begin(r["ctx"])
            g = graph_of(warmup + steps, profile_steps)
            g.replay()
            torch.cuda.synchronize(dev)
            tot, ks = [0.0] * 4, 0
            for r in reps:
                m, k = ckv.ckv_profile_end(r["ctx"])
                tot = [a + b for a, b in zip(tot, m)]
                ks += k
            del g
            avg = [t / ks for t in tot] if ks else None
        for r in reps:
            assert ckv.ckv_last_error(r["ctx"]) == ckv.CKV_OK
        launches = ckv.ckv_step_launches(reps[0]["ctx"])
        sel_tok = np.zeros(cfg.n_graphs, np.int32)
        ckv.ckv_get_step_debug(reps[(warmup + steps - 1) % L]["ctx"], n_tok_sel=sel_tok)
    finally:
        for r in reps:
            ckv.ckv_destroy(r["ctx"])
        del reps
        torch.cuda.empty_cache()
    T_mean = float(sel_tok.mean())
    step_bytes = algorithmic_bytes(cfg, T_mean) * cfg.n_graphs
    peak, peak_kind = measured_peaks()
    res = {"workload": cfg.name, "steps_per_s": 1e3 / ms, "ms_per_step": ms, "steps": steps,
           "warmup": warmup, "layer_replicas": L, "graphs": cfg.n_graphs, "mean_tokens_kept": T_mean,
           "algorithmic_bytes_per_step": step_bytes, "hbm_gbs": step_bytes / (ms / 1e3) / 1e9,
           "hbm_frac_of_measured": step_bytes / (ms / 1e3) / 1e9 / peak, "gpu_launches": launches * steps,
           "aux_bytes": aux, "kv_bytes": kvb, "aux_over_kv": aux / kvb}
    if avg is not None:
        res["kernel_ms_per_step"] = {k: v for k, v in zip(kernel_names(launches), avg) if k != "-"}
        res["roofline"] = roofline_of(cfg, T_mean, avg, launches, peak, peak_kind)
    return res


def kernel_names(launches):
    """Names of the four per-kernel spans ckv_profile_end reports."""
    if launches == 1:
        return ["step", "-", "-", "step_close"]
    if launches == 4:
        return ["score", "select", "attend_output", "edges_assign_update"]
    return ["score", "select", "attend_edges_update", "step_close"]


def roofline_of(cfg, T_mean, avg, launches, peak, peak_kind):
    """The dominant kernel's algorithmic bytes over its average event time.
    avg: per-kernel ms per step (score, select, attend, close) or, for the
    single-launch step, the step kernel's in avg[0]."""
    if launches == 1:
        kb = algorithmic_bytes(cfg, T_mean) * cfg.n_graphs
        kname, t = "k_step", avg[0]
    else:
        dom = 0 if avg[0] >= avg[2] else 2
        kb = kernel_bytes(cfg, T_mean)["score" if dom == 0 else "attend"] * cfg.n_graphs
        kname, t = ("k_score" if dom == 0 else "k_attend"), avg[dom]
    achieved = kb / (t / 1e3) / 1e9
    return {"bound": "hbm", "kernel": kname, "achieved": achieved, "peak": peak, "unit": "GB/s",
            "frac": achieved / peak, "peak_kind": peak_kind, "traffic": profiled_traffic(kname),
            "algorithmic_bytes_per_launch": kb, "avg_launch_ms": t}


def sweep_bench(args):
    """The batch-16 Qwen3-4B-shaped sweep: decode steps/s at every (n, budget)
    point (n in 8K/32K/128K, budget 128..4096), one JSON line per point plus
    a summary line.  The workload of one n serves its four budgets."""
    import torch
    from long_context_decode_ckv_b200 import build as ckv_build
    ckv_build.build()
    torch.cuda.set_device(0)
    workers = max(1, min(16, os.cpu_count() or 1))
    rows = []
    with Clocks(0) as clk:
        for n in (8192, 32768, 131072):
            base = synth.make_workload(synth.sweep_config(n, 128), workers=workers)
            for t in (128, 512, 1024, 4096):
                cfg = synth.sweep_config(n, t)
                wl = synth.Workload(cfg, base.K, base.V, base.q, base.labels)
                # enough replicas that the rotated step data exceeds L2 4 times over
                sb = algorithmic_bytes(cfg, min(t, cfg.n0)) * cfg.n_graphs
                kvb = cfg.batch * cfg.n_kv_heads * cfg.n_max * cfg.head_dim * 2 * 2
                L = int(min(max(2, -(-4 * 126e6 // sb)), max(1, 48e9 // kvb)))
                L = max(L, -(-(args.warmup + args.steps) // cfg.steps))
                r = decode_rate(cfg, wl, args.warmup, args.steps, L, profile_steps=0)
                r.update(n=n, budget=t)
                rows.append(r)
                print(json.dumps({"sweep_point": r}), flush=True)
            del base
    print(json.dumps({"metric": "decode steps/s (sweep)", "points": len(rows),
                      "table": [{k: r[k] for k in ("n", "budget", "steps_per_s", "ms_per_step", "hbm_gbs",
                                                    "mean_tokens_kept", "layer_replicas")} for r in rows],
                      "clocks": clk.summary()}), flush=True)
    return 0


def leiden_bench(args):
    """Figure 1 step (2) and Figure 2: the prefill graph (GPU, ckv_build_graph)
    of the 8-head workload at growing n, partitioned by the host Leiden
    (ckv_leiden, gamma 1); community count, mean size, modularity (GPU,
    ckv_modularity) and the host time per graph."""
    import torch
    import long_context_decode_ckv_b200 as ckv
    from long_context_decode_ckv_b200 import build as ckv_build
    P = synth.PREFILL
    ckv_build.build()
    dev = torch.device("cuda", 0)
    rows = []
    for n in (1024, 2048, 4096, 8192, 16384):
        Q, K = synth.make_prefill(P, n=n)
        q = torch.from_numpy(Q).view(torch.bfloat16).to(dev)
        k = torch.from_numpy(K).view(torch.bfloat16).to(dev)
        H, S, kap = P.n_heads, P.n_sinks, P.kappa
        E = int(np.clip(np.arange(n) - S, 0, kap).sum())
        rp = torch.empty((H, n + 1), dtype=torch.int64, device=dev)
        col = torch.empty((H, E), dtype=torch.int32, device=dev)
        w = torch.empty((H, E), dtype=torch.float32, device=dev)
        ckv.ckv_build_graph(H, n, 128, S, kap, ckv.CKV_BF16, q, k, rp, col, w)
        torch.cuda.synchronize(dev)
        counts, qs, secs = [], [], []
        for h in range(H):
            rph, colh, wh = rp[h].cpu().numpy(), col[h].cpu().numpy(), w[h].cpu().numpy()
            labels = np.empty(n, np.int32)
            t0 = time.perf_counter()
            C = ckv.ckv_leiden(n, rph, colh, wh, 1.0, labels)
            secs.append(time.perf_counter() - t0)
            ws = torch.empty(ckv.ckv_modularity_workspace(C), dtype=torch.uint8, device=dev)
            qs.append(ckv.ckv_modularity(n, rp[h], col[h], w[h], torch.from_numpy(labels).to(dev), C, 1.0, ws))
            counts.append(C)
        rows.append({"n": n, "communities_mean": float(np.mean(counts)),
                     "communities_over_sqrt_n": float(np.mean(counts) / np.sqrt(n)),
                     "mean_size": float(n / np.mean(counts)), "modularity_mean": float(np.mean(qs)),
                     "leiden_host_ms_per_graph": 1e3 * float(np.mean(secs))})
    print(json.dumps({"leiden_vs_n": rows, "workload": "prefill_8h_k8_s4_bf16 (per-head graphs, gamma 1)",
                      "data": "synthetic clustered keys (2048 clusters)"}), flush=True)
    return 0


def refresh_bench(args):
    """Tables 8-9 and Figure 3 (left), mechanics: two contexts decode the same
    steps from the same Leiden partition of the prefill graph; one updates
    incrementally only, the other also refreshes (ckv_refresh) every R steps.
    Every R/2 steps both report the modularity of their partition on the
    token graph (ckv_graph_modularity).  Workload: batch 1, 8 query heads
    over 2 KV heads, per-head graphs, n0 = 8192, budget 1024; the prefill
    graph is the keys over themselves (the synthetic workload has no
    prefill queries)."""
    import torch
    import long_context_decode_ckv_b200 as ckv
    from long_context_decode_ckv_b200 import build as ckv_build
    R = args.refresh
    steps = min(args.steps, 4 * R) if args.steps else 4 * R
    cfg = synth.scaled(synth.LLAMA, batch=1, n_q_heads=8, n_kv_heads=2, n0=8192, n_clusters=512, steps=steps,
                       budget=1024)
    wl = synth.make_workload(cfg, workers=max(1, min(16, os.cpu_count() or 1)))
    ckv_build.build()
    dev = torch.device("cuda", 0)

    def upload(a):
        return torch.from_numpy(np.ascontiguousarray(a)).view(torch.bfloat16).to(dev)

    K, V, q = upload(wl.K), upload(wl.V), upload(wl.q)
    S, kap, n0, G = cfg.n_sinks, cfg.kappa, cfg.n0, cfg.n_graphs
    E = int(np.clip(np.arange(n0) - S, 0, kap).sum())
    graphs, labels = [], np.empty((G, n0), np.int32)
    t0 = time.perf_counter()
    for kvh in range(cfg.n_kv_heads):
        kk = K[0, kvh, :n0][None].contiguous()
        rp = torch.empty((1, n0 + 1), dtype=torch.int64, device=dev)
        col = torch.empty((1, E), dtype=torch.int32, device=dev)
        w = torch.empty((1, E), dtype=torch.float32, device=dev)
        ckv.ckv_build_graph(1, n0, 128, S, kap, ckv.CKV_BF16, kk, kk, rp, col, w)
        graphs.append((rp[0].cpu().numpy(), col[0].cpu().numpy(), w[0].cpu().numpy()))
    lab_kv = []
    for rp, col, w in graphs:
        lab = np.empty(n0, np.int32)
        ckv.ckv_leiden(n0, rp, col, w, 1.0, lab)
        lab_kv.append(lab)
    init_s = time.perf_counter() - t0
    nc0 = 0
    for g in range(G):
        labels[g] = lab_kv[cfg.graph_heads(g)[1]]
        nc0 = max(nc0, int(labels[g].max()) + 1)
    Nc = max(4 * nc0, 256)
    c = ckv.ckv_config()
    c.batch, c.n_q_heads, c.n_kv_heads, c.head_dim = 1, cfg.n_q_heads, cfg.n_kv_heads, 128
    c.n_max, c.max_communities, c.n_sinks = cfg.n_max, Nc, S
    c.kappa, c.budget, c.slack = kap, cfg.budget, 16
    c.kv_dtype, c.mode, c.device, c.pool_capacity = ckv.CKV_BF16, ckv.CKV_PER_HEAD, 0, 0
    rp_all = np.stack([graphs[cfg.graph_heads(g)[1]][0] for g in range(G)])
    col_all = np.stack([graphs[cfg.graph_heads(g)[1]][1] for g in range(G)])
    w_all = np.stack([graphs[cfg.graph_heads(g)[1]][2] for g in range(G)])
    arms = {}
    for name in ("incremental", "refresh"):
        ctx = ckv.ckv_create(c)
        ckv.ckv_init_communities(ctx, labels, 0, nc0, K, n0)
        ckv.ckv_set_token_graph(ctx, rp_all, col_all, w_all, n0)
        arms[name] = ctx
    out = torch.empty((1, cfg.n_q_heads, 128), dtype=torch.float32, device=dev)
    qv = np.zeros(G)
    traj = {"incremental": [], "refresh": []}
    refresh_ms, counts = [], []
    cnt = np.zeros(G, np.int32)
    for i in range(steps + 1):
        if i % max(1, R // 2) == 0:
            for name, ctx in arms.items():
                ckv.ckv_graph_modularity(ctx, 1.0, qv)
                traj[name].append({"generated": i, "modularity_mean": float(qv.mean()),
                                   "modularity_min": float(qv.min())})
        if i == steps:
            break
        if i and i % R == 0:
            t1 = time.perf_counter()
            ckv.ckv_refresh(arms["refresh"], K, 1.0, cnt)
            refresh_ms.append(1e3 * (time.perf_counter() - t1))
            counts.append(float(cnt.mean()))
        n = n0 + i + 1
        for ctx in arms.values():
            ckv.ckv_decode_step(ctx, q[i], K, V, n, out)
            ckv.ckv_assign_update(ctx, K, n)
    for ctx in arms.values():
        assert ckv.ckv_last_error(ctx) == ckv.CKV_OK
        ckv.ckv_destroy(ctx)
    print(json.dumps({"refresh_period": R, "steps": steps, "n0": n0, "graphs": G,
                      "initial_communities": nc0, "prefill_graph_and_leiden_s": init_s,
                      "modularity": traj, "refresh_ms": refresh_ms, "communities_after_refresh": counts,
                      "data": "synthetic clustered keys; prefill graph = keys over keys"}), flush=True)
    return 0


def recall_sweep(args, budgets):
    """Figure 3 (right): attention-mass recall of the retrieved set versus the
    token budget, on the throughput workload, every 8th of --steps steps."""
    import torch
    import long_context_decode_ckv_b200 as ckv
    from long_context_decode_ckv_b200 import build as ckv_build
    cfg = CFG
    wl = synth.make_workload(cfg, workers=max(1, min(16, os.cpu_count() or 1)))
    ckv_build.build()
    dev = torch.device("cuda", 0)

    def upload(a):
        t = torch.from_numpy(a)
        return (t.view(torch.bfloat16) if a.dtype == np.uint16 else t).to(dev)

    K, V, q = upload(wl.K), upload(wl.V), upload(wl.q)
    out = torch.empty((cfg.batch, cfg.n_q_heads, 128), dtype=torch.float32, device=dev)
    rec = torch.empty((cfg.batch, cfg.n_q_heads), dtype=torch.float32, device=dev)
    steps = min(args.steps, cfg.steps)
    rows = []
    for budget in budgets:
        c = ckv.ckv_config()
        c.batch, c.n_q_heads, c.n_kv_heads, c.head_dim = cfg.batch, cfg.n_q_heads, cfg.n_kv_heads, 128
        c.n_max, c.max_communities, c.n_sinks = cfg.n_max, cfg.n_comm, cfg.n_sinks
        c.kappa, c.budget, c.slack = cfg.kappa, budget, 16
        c.kv_dtype, c.mode, c.device, c.pool_capacity = ckv.CKV_BF16, ckv.CKV_QUERY_GROUP, 0, 0
        ctx = ckv.ckv_create(c)
        Kr, Vr = K.clone(), V.clone()        # the steps' community updates stay per budget
        ckv.ckv_init_communities(ctx, wl.labels, 0, cfg.n_comm, Kr, cfg.n0)
        vals, kept = [], []
        sel_tok = np.zeros(cfg.n_graphs, np.int32)
        for i in range(steps):
            n = cfg.n0 + i + 1
            ckv.ckv_decode_step(ctx, q[i], Kr, Vr, n, out)
            ckv.ckv_assign_update(ctx, Kr, n)
            if i % 8 == 0:
                ckv.ckv_step_recall(ctx, q[i], Kr, n, rec)
                vals.append(rec.cpu().numpy().copy())
                ckv.ckv_get_step_debug(ctx, n_tok_sel=sel_tok)
                kept.append(float(sel_tok.mean()))
        assert ckv.ckv_last_error(ctx) == ckv.CKV_OK
        ckv.ckv_destroy(ctx)
        del Kr, Vr
        v = np.stack(vals)
        rows.append({"budget": budget, "mean_tokens_kept": float(np.mean(kept)), "recall_mean": float(v.mean()),
                     "recall_p10": float(np.quantile(v, 0.1)), "recall_min": float(v.min()),
                     "checks": int(v.size)})
    print(json.dumps({"recall_vs_budget": rows, "workload": WORKLOAD, "steps": steps,
                      "data": "synthetic clustered keys (not a model's attention)"}), flush=True)
    return 0


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=8)
    ap.add_argument("--impl", default="ckv", choices=["ckv", "reference"])
    ap.add_argument("--replicas", type=int, default=0, help="layer copies rotated (0 = auto)")
    ap.add_argument("--e2e-steps", type=int, default=40)
    ap.add_argument("--cpu-steps", type=int, default=8)
    ap.add_argument("--no-cpu", action="store_true")
    ap.add_argument("--no-graph", action="store_true", help="launch the timed steps eagerly")
    ap.add_argument("--profile-steps", type=int, default=40,
                    help="further steps replayed with per-kernel events (0 = none)")
    ap.add_argument("--recall-sweep", default="",
                    help="comma-separated budgets: print the mean attention-mass recall per budget "
                         "over --steps decode steps instead of timing")
    ap.add_argument("--refresh", type=int, default=0,
                    help="refresh period R: decode with and without a refresh every R steps and report the "
                         "modularity over generation instead (Tables 8-9, Figure 3 left)")
    ap.add_argument("--leiden", action="store_true",
                    help="partition prefill graphs of growing n with the host Leiden and report the community "
                         "count and modularity instead")
    ap.add_argument("--prefill", action="store_true",
                    help="time the prefill graph construction (per-head and query-group) instead")
    ap.add_argument("--dense-steps", type=int, default=20,
                    help="dense decode comparator launches timed after the sparse steps (0 = none)")
    ap.add_argument("--sweep", action="store_true",
                    help="decode steps/s at every point of the batch-16 (n, budget) sweep instead")
    ap.add_argument("--update-stream", default="side", choices=["side", "main"],
                    help="stream of ckv_assign_update: a side stream overlapping the next replica's step "
                         "(default), or the step's own stream")
    ap.add_argument("--no-extras", action="store_true",
                    help="skip the prefill and Llama per-head measurements of the default line")
    args = ap.parse_args()
    rank, world, local = rank_env()
    if args.warmup < 3:
        raise SystemExit("--warmup must be >= 3")
    if args.impl == "reference":
        return reference_arm(args, rank, world)
    if args.recall_sweep:
        return recall_sweep(args, [int(b) for b in args.recall_sweep.split(",")])
    if args.prefill:
        return prefill_bench(args)
    if args.sweep:
        return sweep_bench(args)
    if args.leiden:
        return leiden_bench(args)
    if args.refresh:
        return refresh_bench(args)

    # host-side generation first (spawned pool, before any CUDA call)
    workers = max(1, min(16, (os.cpu_count() or 1) // max(1, world)))
    t_gen = time.perf_counter()
    wl = synth.make_workload(CFG, workers=workers)
    wl_llama = synth.make_workload(synth.LLAMA, workers=workers) if not args.no_extras else None
    t_gen = time.perf_counter() - t_gen

    import torch
    import long_context_decode_ckv_b200 as ckv
    from long_context_decode_ckv_b200 import build as ckv_build
    ckv_build.build()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    pg = None
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=dev)
        pg = dist

    cfg = CFG
    total_steps = args.warmup + args.steps + args.profile_steps + args.e2e_steps
    L = args.replicas or max(4, -(-total_steps // cfg.steps))
    if -(-total_steps // L) > cfg.steps:
        raise SystemExit("not enough decode tokens in the workload for these steps; raise --replicas")

    def upload(a):
        t = torch.from_numpy(a)
        return (t.view(torch.bfloat16) if a.dtype == np.uint16 else t).to(dev)

    K0, V0, q = upload(wl.K), upload(wl.V), upload(wl.q)
    reps = []
    for r in range(L):
        K = K0 if r == 0 else K0.clone()
        V = V0 if r == 0 else V0.clone()
        c = ckv.ckv_config()
        c.batch, c.n_q_heads, c.n_kv_heads, c.head_dim = cfg.batch, cfg.n_q_heads, cfg.n_kv_heads, 128
        c.n_max, c.max_communities, c.n_sinks = cfg.n_max, cfg.n_comm, cfg.n_sinks
        c.kappa, c.budget, c.slack = cfg.kappa, cfg.budget, 16
        c.kv_dtype, c.mode, c.device, c.pool_capacity = ckv.CKV_BF16, ckv.CKV_QUERY_GROUP, local, 0
        ctx = ckv.ckv_create(c)
        ckv.ckv_init_communities(ctx, wl.labels, 0, cfg.n_comm, K, cfg.n0)
        reps.append({"ctx": ctx, "K": K, "V": V, "i": 0})
    out = torch.empty((cfg.batch, cfg.n_q_heads, 128), dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream(dev)
    sel_tok = np.zeros(cfg.n_graphs, np.int32)
    stepper = Stepper(reps, q, out, cfg, dev, side=args.update_stream == "side")
    step = stepper.step

    for s in range(args.warmup):
        step(s, stream)
    stepper.join(stream)
    torch.cuda.synchronize(dev)

    def capture(first, count):
        """The steps [first, first + count) captured into one CUDA graph (the
        launches of a real decoder are), or None when capture is refused."""
        if args.no_graph:
            return None
        saved = [r["i"] for r in reps]
        try:
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, capture_error_mode="relaxed"):
                cap = torch.cuda.current_stream(dev)
                for s in range(first, first + count):
                    step(s, cap)
                stepper.join(cap)
            try:
                upload_graph(g, stream)
            except Exception as exc:   # the first replay then uploads it
                print(f"graph upload skipped ({exc})", file=sys.stderr)
            return g
        except Exception as exc:   # capture refused: time the same steps eagerly
            print(f"CUDA graph capture failed ({exc}); timing eager launches", file=sys.stderr)
            for r, i in zip(reps, saved):
                r["i"] = i
            stepper.pending = [False] * len(reps)
            return None

    def run(first, count, g):
        if g is not None:
            g.replay()
        else:
            for s in range(first, first + count):
                step(s, stream)
            stepper.join(stream)

    # timed steps: no profiling events inside
    s_timed = args.warmup
    graph = capture(s_timed, args.steps)
    launch_mode = "cuda-graph" if graph is not None else "eager"
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if pg:
        pg.barrier()
    torch.cuda.synchronize(dev)
    with Clocks(local) as clk:
        hold(stream)
        start.record(stream)
        run(s_timed, args.steps, graph)
        end.record(stream)
        torch.cuda.synchronize(dev)
    if pg:
        pg.barrier()
    ms = start.elapsed_time(end)
    del graph

    # per-kernel device time: the next steps again, with an event pair
    # around every kernel (recorded on the launching stream)
    s_prof = s_timed + args.steps
    kern_ms, kern_steps = [0.0] * 4, 0
    if args.profile_steps:
        for r in reps:
            ckv.ckv_profile_begin(r["ctx"])
        pgraph = capture(s_prof, args.profile_steps)
        run(s_prof, args.profile_steps, pgraph)
        torch.cuda.synchronize(dev)
        for r in reps:
            try:
                m, k = ckv.ckv_profile_end(r["ctx"])
            except ckv.CkvError as exc:
                print(f"per-kernel profile unavailable: {exc}", file=sys.stderr)
                kern_ms, kern_steps = None, 0
                break
            kern_ms = [a + b for a, b in zip(kern_ms, m)]
            kern_steps += k
        del pgraph
    else:
        kern_ms = None
    for r in reps:
        assert ckv.ckv_last_error(r["ctx"]) == ckv.CKV_OK
    launches_per_step = ckv.ckv_step_launches(reps[0]["ctx"])
    aux_b, kv_b = ckv.ckv_aux_bytes(reps[0]["ctx"])
    ckv.ckv_get_step_debug(reps[(args.warmup + args.steps - 1) % L]["ctx"], n_tok_sel=sel_tok)
    T_mean = float(sel_tok.mean())
    ms = max_over_ranks(pg, ms, dev)

    # end-to-end through the host-buffer entry point: per step H2D of q and
    # the new token's K/V rows from pinned memory, D2H of the output
    e2e = None
    if args.e2e_steps:
        qh = torch.from_numpy(wl.q).pin_memory()
        kh = torch.from_numpy(np.ascontiguousarray(wl.K[:, :, cfg.n0:])).pin_memory()
        vh = torch.from_numpy(np.ascontiguousarray(wl.V[:, :, cfg.n0:])).pin_memory()
        oh = torch.empty((cfg.batch, cfg.n_q_heads, 128), dtype=torch.float32).pin_memory()
        qstep = [qh[i] for i in range(cfg.steps)]   # each step's pinned host buffers
        kstep = [kh[:, :, i].contiguous() for i in range(cfg.steps)]
        vstep = [vh[:, :, i].contiguous() for i in range(cfg.steps)]
        s0 = s_prof + args.profile_steps
        if pg:
            pg.barrier()
        torch.cuda.synchronize(dev)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for s in range(s0, s0 + args.e2e_steps):
            r = reps[s % L]
            i = r["i"]
            ckv.ckv_decode_host(r["ctx"], qstep[i], kstep[i], vstep[i], r["K"], r["V"], cfg.n0 + i + 1,
                                oh, stream)
            r["i"] = i + 1
        e1.record(stream)
        torch.cuda.synchronize(dev)
        ems = e0.elapsed_time(e1)
        ems = max_over_ranks(pg, ems, dev)
        eb = 2
        e2e = {"value": job_rate(world, args.e2e_steps, ems), "unit": "steps/s",
               "h2d_bytes_per_step": cfg.batch * (cfg.n_q_heads + 2 * cfg.n_kv_heads) * 128 * eb,
               "d2h_bytes_per_step": cfg.batch * cfg.n_q_heads * 128 * 4}

    # attention-mass recall of each replica's last step (Figure 3 right),
    # one dense statistics pass over K per replica
    rec_t = torch.empty((cfg.batch, cfg.n_q_heads), dtype=torch.float32, device=dev)
    recalls, rec_ms = [], 0.0
    for r in reps:
        i = r["i"] - 1
        # a first call loads the kernel and sizes its grid; the second is timed
        ckv.ckv_step_recall(r["ctx"], q[i], r["K"], cfg.n0 + i + 1, rec_t, stream)
        r0, r1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        hold(stream)
        r0.record(stream)
        ckv.ckv_step_recall(r["ctx"], q[i], r["K"], cfg.n0 + i + 1, rec_t, stream)
        r1.record(stream)
        torch.cuda.synchronize(dev)
        rec_ms += r0.elapsed_time(r1)
        recalls.append(rec_t.cpu().numpy().copy())
    recalls = np.stack(recalls)
    recall = {"mean": float(recalls.mean()), "min": float(recalls.min()), "heads": int(recalls.size),
              "budget": cfg.budget, "n": int(cfg.n0 + reps[0]["i"]),
              "kernel_ms": rec_ms / len(reps), "kernel": "k_dense (statistics only)",
              "achieved_gbs": cfg.batch * cfg.n_kv_heads * (cfg.n0 + reps[0]["i"]) * 256 / (rec_ms / len(reps) / 1e3) / 1e9,
              "traffic": profiled_traffic("k_dense_stats")}

    # dense decode comparator: every head over the whole cache, same replicas
    dense = None
    if args.dense_steps:
        dout = torch.empty((cfg.batch, cfg.n_q_heads, 128), dtype=torch.float32, device=dev)
        for s in range(3):
            r = reps[s % L]
            ckv.ckv_dense_decode(r["ctx"], q[r["i"] - 1], r["K"], r["V"], cfg.n0 + r["i"], dout, None, stream)
        torch.cuda.synchronize(dev)
        d0, d1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        hold(stream)
        d0.record(stream)
        for s in range(args.dense_steps):
            r = reps[s % L]
            ckv.ckv_dense_decode(r["ctx"], q[r["i"] - 1], r["K"], r["V"], cfg.n0 + r["i"], dout, None, stream)
        d1.record(stream)
        torch.cuda.synchronize(dev)
        dms = d0.elapsed_time(d1) / args.dense_steps
        n_d = cfg.n0 + reps[0]["i"]
        dbytes = cfg.batch * cfg.n_kv_heads * n_d * 128 * 2 * 2 + cfg.batch * cfg.n_q_heads * 128 * (2 + 4)
        dense = {"kernel": "k_dense", "ms_per_step": dms, "steps_per_s": 1e3 / dms,
                 "algorithmic_bytes": dbytes, "achieved_gbs": dbytes / (dms / 1e3) / 1e9,
                 "frac": dbytes / (dms / 1e3) / 1e9 / measured_peaks()[0],
                 "traffic": profiled_traffic("k_dense_attention"),
                 "sparse_step_speedup": dms / (ms / args.steps)}

    for r in reps:
        ckv.ckv_destroy(r["ctx"])
    del reps, K0, V0
    torch.cuda.empty_cache()
    if pg:
        pg.barrier()
        pg.destroy_process_group()
    if rank != 0:
        return 0

    # the other headline numbers, each timed on its own after the step:
    # the Llama-3.1-8B per-head decode workload and the prefill graph
    llama, prefill, prefill_qk = None, None, None
    if not args.no_extras:
        lc = synth.LLAMA
        llama = decode_rate(lc, wl_llama, 5, 40, max(4, -(-(5 + 40 + 16) // lc.steps)), profile_steps=16)
        del wl_llama
        prefill, prefill_qk = prefill_measure(10, 3)

    steps_per_s = job_rate(world, args.steps, ms)
    per_graph = algorithmic_bytes(cfg, T_mean)
    step_bytes = per_graph * cfg.n_graphs
    gbs = step_bytes * args.steps / (ms / 1e3) / 1e9
    peak, peak_kind = measured_peaks()
    avg, roofline = None, None
    if kern_ms is not None and kern_steps:
        per = [k / kern_steps for k in kern_ms]
        avg = {k: v for k, v in zip(kernel_names(launches_per_step), per) if k != "-"}
        roofline = roofline_of(cfg, T_mean, per, launches_per_step, peak, peak_kind)

    # the oracle on the host: all cores (one thread per graph), one core,
    # and the prefill oracle on sampled rows
    cpu = None
    if not args.no_cpu:
        cores = host_cores()
        secs = run_oracle_steps(wl, args.cpu_steps, threads=cores)
        secs1 = run_oracle_steps(wl, max(1, args.cpu_steps // 4), threads=1)
        cpu = {"value": args.cpu_steps / secs, "unit": "steps/s", "cores": min(cores, cfg.n_graphs),
               "kind": "oracle",
               "sample": f"{args.cpu_steps} decode steps x {cfg.n_graphs} graphs of the same workload, C oracle, "
                         f"one thread per graph on {min(cores, cfg.n_graphs)} of {cores} host cores ({secs:.1f} s)",
               "single_core": {"value": max(1, args.cpu_steps // 4) / secs1, "unit": "steps/s", "cores": 1,
                               "sample": f"{max(1, args.cpu_steps // 4)} decode steps x {cfg.n_graphs} graphs, "
                                         f"one thread ({secs1:.1f} s)"}}
        if prefill_qk is not None:
            pm, pe, note = prefill_oracle_time(synth.PREFILL, *prefill_qk, threads=cores)
            cpu["prefill"] = {"value": pe * 1e3, "unit": "ms (extrapolated)", "cores": cores,
                              "measured_s": pm, "sample": note,
                              "gpu_speedup": (pe * 1e3) / prefill["ms"] if prefill else None}
    line = {
        "metric": METRIC, "value": steps_per_s, "unit": "steps/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic",
        "config": {"workload": WORKLOAD, "graphs": cfg.n_graphs, "layer_replicas": L,
                   "l2": f"{L} layer replicas rotated (inputs larger than L2), no flush",
                   "parallelism": "replicas" if world > 1 else "single",
                   "launch": launch_mode,
                   "update": ("inside the step's last kernel" if launches_per_step != 4 else
                              "side stream: each ckv_assign_update overlaps the next replica's step"
                              if args.update_stream == "side" else "own kernel on the step's stream")},
        "hbm_gbs": gbs, "hbm_frac_of_8000": gbs / NOMINAL_HBM_GBS, "hbm_frac_of_measured": gbs / peak,
        "algorithmic_bytes_per_step": step_bytes, "mean_tokens_kept": T_mean,
        "kernel_ms_per_step": avg,
        "roofline": roofline, "cpu_baseline": cpu, "e2e": e2e,
        "aux_bytes": aux_b, "kv_bytes": kv_b, "aux_over_kv": aux_b / kv_b,
        "prefill": prefill, "llama_per_head": llama,
        "recall": recall, "dense_decode": dense,
        "gpu_launches": launches_per_step * args.steps, "clocks": clk.summary(),
        "gen_seconds": t_gen,
    }
    print(json.dumps(line), flush=True)
    return 0


if __name__ == "__main__":
    sys.exit(main())
