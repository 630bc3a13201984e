"""Seeded synthetic workloads for CommunityKV decode and prefill.

This module only draws inputs: clustered keys, values, queries, the initial
partition labels and the new tokens' K/V.  It holds none of the method's
arithmetic, so both the CUDA library's tests and the CPU oracle read the same
bytes from it.

Recipe (stands in for LongBench v2 / BABILong / RULER activations, which need
model weights and datasets; none of their items is reproduced):

* per (batch, KV head) slab, its own numpy PCG64 stream seeded by
  (config seed, tag, b, kv head);
* ``n_clusters`` cluster centres ~ N(0, I_D); every position gets a cluster
  through a seeded balanced permutation, so clusters are spread over the
  context;
* key = centre + 0.3 N(0, I); in bf16 workloads 4 seeded channels of the key
  are then scaled by 8 (per-channel outliers); value ~ N(0, I);
* labels (the initial partition): each cluster's positions ascending,
  chunked into communities of ``comm_size``; community ids in
  (cluster, chunk) order.  Labels at sink positions are ignored by the
  method;
* decode step s: each query group (QUERY_GROUP) or head (PER_HEAD) draws a
  cluster c; q = centre_c + 0.3 N(0, I) per head (no outlier scale); the new
  token's key is drawn like a context key of cluster c (PER_HEAD: the first
  head's cluster of the group) and its value ~ N(0, I); they sit at row
  n0 + s of the cache;
* bf16 conversion rounds to nearest even.
"""
from __future__ import annotations

from dataclasses import dataclass, replace

import numpy as np

PER_HEAD, QUERY_GROUP = 0, 1
BASE_SEED = 20261202


@dataclass(frozen=True)
class DecodeConfig:
    name: str
    batch: int
    n_q_heads: int
    n_kv_heads: int
    head_dim: int
    n0: int             # context tokens present before the first decode step
    steps: int
    n_sinks: int
    kappa: int
    budget: int
    comm_size: int
    n_clusters: int
    bf16: bool
    mode: int           # PER_HEAD or QUERY_GROUP
    seed: int

    @property
    def group(self) -> int:
        return self.n_q_heads // self.n_kv_heads

    @property
    def n_graphs(self) -> int:
        return self.batch * (self.n_kv_heads if self.mode == QUERY_GROUP else self.n_q_heads)

    @property
    def heads_per_graph(self) -> int:
        return self.group if self.mode == QUERY_GROUP else 1

    @property
    def n_max(self) -> int:
        return self.n0 + self.steps

    @property
    def n_comm(self) -> int:
        per = -(-(-(-self.n0 // self.n_clusters)) // self.comm_size)
        return self.n_clusters * per

    def graph_heads(self, g: int):
        """(batch, kv head, [query heads]) of graph g."""
        if self.mode == QUERY_GROUP:
            b, kvh = divmod(g, self.n_kv_heads)
            return b, kvh, list(range(kvh * self.group, (kvh + 1) * self.group))
        b, h = divmod(g, self.n_q_heads)
        return b, h // self.group, [h]


@dataclass(frozen=True)
class PrefillConfig:
    name: str
    n_heads: int
    head_dim: int
    n: int
    n_sinks: int
    kappa: int
    n_clusters: int
    seed: int


# The five workloads: tiny single head; Llama-3.1-8B-shaped per-head graphs;
# Qwen3-8B-shaped query-group graphs at n=128K (the throughput workload);
# prefill graph construction; and the Qwen3-4B-shaped batch-16 sweep.
TINY = DecodeConfig("tiny_1h_n2k", 1, 1, 1, 128, 2048, 16, 4, 8, 256, 16, 64, False, PER_HEAD,
                    BASE_SEED + 0)
LLAMA = DecodeConfig("llama31_8b_perhead_n32k", 1, 32, 8, 128, 32768, 64, 4, 8, 1024, 16, 2048,
                     True, PER_HEAD, BASE_SEED + 1)
QWEN8B = DecodeConfig("qwen3_8b_qgroup_b4_n128k", 4, 32, 8, 128, 131072, 128, 4, 8, 4096, 16,
                      2048, True, QUERY_GROUP, BASE_SEED + 2)
PREFILL = PrefillConfig("prefill_8h_n16k", 8, 128, 16384, 4, 8, 2048, BASE_SEED + 3)


def sweep_config(n: int, budget: int, steps: int = 32) -> DecodeConfig:
    return DecodeConfig(f"qwen3_4b_sweep_b16_n{n}_t{budget}", 16, 32, 8, 128, n, steps, 4, 8,
                        budget, 16, min(2048, n // 16), True, QUERY_GROUP, BASE_SEED + 4)


SWEEP = [sweep_config(n, t) for n in (8192, 32768, 131072) for t in (128, 512, 1024, 4096)]


def scaled(cfg: DecodeConfig, **kw) -> DecodeConfig:
    """A smaller copy of a workload (same recipe), for tests."""
    return replace(cfg, **kw)


# ------------------------------------------------------------------ helpers
def to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """float32 -> bfloat16 bit patterns (uint16), round to nearest even."""
    u = np.ascontiguousarray(x, np.float32).view(np.uint32)
    return ((u + (((u >> 16) & 1) + 0x7FFF)) >> 16).astype(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    return (b.astype(np.uint32) << 16).view(np.float32)


def _rng(seed: int, *tag: int) -> np.random.Generator:
    return np.random.default_rng([seed, *tag])


@dataclass
class Slab:
    """One (batch, KV head) slab: keys, values and the initial partition."""
    K: np.ndarray        # [n_max][D] float32 or bf16 bits
    V: np.ndarray
    labels: np.ndarray   # [n0] int32
    centers: np.ndarray  # [n_clusters][D] float32 (pre-outlier)
    outl: np.ndarray     # outlier channel ids (empty for fp32 workloads)


def _key_rows(rng, centers, clus, outl, D):
    k = centers[clus] + np.float32(0.3) * rng.standard_normal((len(clus), D), dtype=np.float32)
    if len(outl):
        k[:, outl] *= np.float32(8.0)
    return k


def make_slab(cfg: DecodeConfig, b: int, kvh: int) -> Slab:
    """Context K/V (rows [0, n0)), labels, plus decode-token rows [n0, n_max)."""
    D, n0 = cfg.head_dim, cfg.n0
    rng = _rng(cfg.seed, 1, b, kvh)
    centers = rng.standard_normal((cfg.n_clusters, D), dtype=np.float32)
    outl = (np.sort(rng.choice(D, 4, replace=False)).astype(np.int64) if cfg.bf16
            else np.zeros(0, np.int64))
    perm = rng.permutation(n0)
    clus = np.empty(n0, np.int64)
    clus[perm] = np.arange(n0) % cfg.n_clusters
    K = np.empty((cfg.n_max, D), np.float32)
    V = np.empty((cfg.n_max, D), np.float32)
    K[:n0] = _key_rows(rng, centers, clus, outl, D)
    V[:n0] = rng.standard_normal((n0, D), dtype=np.float32)
    # initial partition: cluster members ascending, chunks of comm_size
    per = cfg.n_comm // cfg.n_clusters
    order = np.lexsort((np.arange(n0), clus))          # by cluster, then position
    rank = np.empty(n0, np.int64)
    starts = np.searchsorted(clus[order], np.arange(cfg.n_clusters))
    rank[order] = np.arange(n0) - starts[clus[order]]
    labels = (clus * per + rank // cfg.comm_size).astype(np.int32)
    # decode tokens: their clusters follow the queries (see queries())
    qc = query_clusters(cfg, b, kvh)
    if cfg.steps:
        rng_t = _rng(cfg.seed, 3, b, kvh)
        K[n0:] = _key_rows(rng_t, centers, qc[:, 0], outl, D)
        V[n0:] = rng_t.standard_normal((cfg.steps, D), dtype=np.float32)
    if cfg.bf16:
        return Slab(to_bf16_bits(K), to_bf16_bits(V), labels, centers, outl)
    return Slab(K, V, labels, centers, outl)


def query_clusters(cfg: DecodeConfig, b: int, kvh: int) -> np.ndarray:
    """[steps][group] cluster drawn by each query head of the KV head's group."""
    rng = _rng(cfg.seed, 2, b, kvh)
    if cfg.mode == QUERY_GROUP:
        c = rng.integers(0, cfg.n_clusters, size=cfg.steps)
        return np.repeat(c[:, None], cfg.group, axis=1)
    return rng.integers(0, cfg.n_clusters, size=(cfg.steps, cfg.group))


def make_queries(cfg: DecodeConfig, slab: Slab, b: int, kvh: int) -> np.ndarray:
    """[steps][group][D] queries of the KV head's query heads."""
    qc = query_clusters(cfg, b, kvh)
    rng = _rng(cfg.seed, 4, b, kvh)
    q = slab.centers[qc] + np.float32(0.3) * rng.standard_normal(
        (cfg.steps, cfg.group, cfg.head_dim), dtype=np.float32)
    return to_bf16_bits(q) if cfg.bf16 else q.astype(np.float32)


@dataclass
class Workload:
    cfg: DecodeConfig
    K: np.ndarray        # [B][H_kv][n_max][D]
    V: np.ndarray
    q: np.ndarray        # [steps][B][H_q][D]
    labels: np.ndarray   # [n_graphs][n0] int32


def _slab_job(args):
    cfg, b, kvh = args
    s = make_slab(cfg, b, kvh)
    return b, kvh, s.K, s.V, s.labels, make_queries(cfg, s, b, kvh)


def make_workload(cfg: DecodeConfig, workers: int = 1) -> Workload:
    """Whole workload on the host (all slabs).  workers > 1 draws the slabs
    in a pool of spawned processes (same bytes as workers = 1)."""
    dt = np.uint16 if cfg.bf16 else np.float32
    K = np.empty((cfg.batch, cfg.n_kv_heads, cfg.n_max, cfg.head_dim), dt)
    V = np.empty_like(K)
    q = np.empty((cfg.steps, cfg.batch, cfg.n_q_heads, cfg.head_dim), dt)
    lab_kv = np.empty((cfg.batch, cfg.n_kv_heads, cfg.n0), np.int32)
    jobs = [(cfg, b, kvh) for b in range(cfg.batch) for kvh in range(cfg.n_kv_heads)]
    if workers > 1 and len(jobs) > 1:
        import multiprocessing as mp
        from concurrent.futures import ProcessPoolExecutor
        with ProcessPoolExecutor(min(workers, len(jobs)), mp_context=mp.get_context("spawn")) as ex:
            results = ex.map(_slab_job, jobs)
            for b, kvh, sk, sv, sl, sq in results:
                K[b, kvh], V[b, kvh], lab_kv[b, kvh] = sk, sv, sl
                q[:, b, kvh * cfg.group:(kvh + 1) * cfg.group] = sq
    else:
        for job in jobs:
            b, kvh, sk, sv, sl, sq = _slab_job(job)
            K[b, kvh], V[b, kvh], lab_kv[b, kvh] = sk, sv, sl
            q[:, b, kvh * cfg.group:(kvh + 1) * cfg.group] = sq
    labels = np.empty((cfg.n_graphs, cfg.n0), np.int32)
    for g in range(cfg.n_graphs):
        b, kvh, _ = cfg.graph_heads(g)
        labels[g] = lab_kv[b, kvh]
    return Workload(cfg, K, V, q, labels)


def make_prefill(cfg: PrefillConfig, n: int | None = None):
    """Q, K [H][n][D] bf16 bits: clustered keys (outliers as above) and
    queries near random cluster centres."""
    n = cfg.n if n is None else n
    D = cfg.head_dim
    Q = np.empty((cfg.n_heads, n, D), np.uint16)
    K = np.empty((cfg.n_heads, n, D), np.uint16)
    for h in range(cfg.n_heads):
        rng = _rng(cfg.seed, 5, h)
        centers = rng.standard_normal((cfg.n_clusters, D), dtype=np.float32)
        outl = np.sort(rng.choice(D, 4, replace=False))
        clus = rng.integers(0, cfg.n_clusters, size=n)
        K[h] = to_bf16_bits(_key_rows(rng, centers, clus, outl, D))
        qc = rng.integers(0, cfg.n_clusters, size=n)
        Q[h] = to_bf16_bits(centers[qc] + np.float32(0.3) *
                            rng.standard_normal((n, D), dtype=np.float32))
    return Q, K
