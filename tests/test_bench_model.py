"""bench.py's byte model and roofline arithmetic, on CPU.

The bench line's GB/s and roofline fractions divide algorithmic bytes by
measured times.  These tests pin the byte model to its closed form at the
Qwen3-8B-shaped workload (batch 4, 8 KV heads: 32 query-group graphs of 4
heads; 8192 communities of 16 members, D = 128, 4 sinks, budget 4096, bf16
K/V, fp32 centroids), check which kernel the roofline names, and check that
an ncu traffic figure is reported only while the sources it was captured on
are unchanged.
"""
import pytest

import bench
from long_context_decode_ckv_b200 import synth

CFG = synth.QWEN8B
T = 4096          # kept member tokens per graph


def test_workload_shape():
    assert (CFG.n_graphs, CFG.n_comm, CFG.head_dim, CFG.n_sinks, CFG.heads_per_graph) == (32, 8192, 128, 4, 4)
    assert CFG.bf16


def test_step_bytes_closed_form():
    # per graph: fp32 centroids, offset + size per community, member ids,
    # K and V rows of the kept members, the sinks and the new token (bf16),
    # bf16 queries in and fp32 outputs out
    per_graph = 8192 * 128 * 4 + 8192 * 8 + T * 4 + (T + 4 + 1) * 128 * 2 * 2 + 4 * 128 * (2 + 4)
    assert per_graph == 6_379_008
    assert bench.algorithmic_bytes(CFG, T) == per_graph
    assert bench.algorithmic_bytes(CFG, T) * CFG.n_graphs == 204_128_256


def test_kernel_bytes_closed_form():
    kb = bench.kernel_bytes(CFG, T)
    assert kb["score"] * CFG.n_graphs == 136_314_880           # centroids, sizes in, scores out
    assert kb["attend"] == (T + 5) * 128 * 4 + T * 4 + 4 * 128 * 6
    # the two streams plus the selection's reads make up the step's bytes
    # (the step model counts the offsets where the scan model counts the
    # scores it writes: same 4 bytes per community)
    assert kb["score"] + kb["attend"] == bench.algorithmic_bytes(CFG, T)


@pytest.mark.parametrize("score_ms,attend_ms,kernel", [(0.028, 0.024, "k_score"), (0.020, 0.026, "k_attend")])
def test_roofline_names_the_longer_stream(score_ms, attend_ms, kernel):
    r = bench.roofline_of(CFG, T, [score_ms, 0.017, attend_ms, 0.027], 4, 6523.3, "measured")
    assert r["kernel"] == kernel and r["bound"] == "hbm" and r["unit"] == "GB/s"
    stream = "score" if kernel == "k_score" else "attend"
    t = score_ms if kernel == "k_score" else attend_ms
    kb = bench.kernel_bytes(CFG, T)[stream] * CFG.n_graphs
    assert r["algorithmic_bytes_per_launch"] == kb and r["avg_launch_ms"] == t
    assert r["achieved"] == pytest.approx(kb / (t * 1e-3) / 1e9)
    assert r["frac"] == pytest.approx(r["achieved"] / 6523.3)


def test_single_launch_roofline_takes_the_whole_step():
    r = bench.roofline_of(CFG, T, [0.050, 0.0, 0.0, 0.001], 1, 6523.3, "measured")
    assert r["kernel"] == "k_step"
    assert r["algorithmic_bytes_per_launch"] == bench.algorithmic_bytes(CFG, T) * CFG.n_graphs


def test_traffic_reported_only_for_the_captured_sources(monkeypatch):
    h = bench.source_hash(bench.KERNEL_SOURCES["k_score"])
    monkeypatch.setitem(bench.PROFILED_TRAFFIC, "k_score", (h, 1.25e8))
    assert bench.profiled_traffic("k_score") == 1.25e8
    monkeypatch.setitem(bench.PROFILED_TRAFFIC, "k_score", ("0" * 16, 1.25e8))
    assert bench.profiled_traffic("k_score") is None
    assert bench.profiled_traffic("k_select") is None            # never captured


def test_job_rate_counts_every_rank():
    # N ranks of K steps each over the slowest rank's milliseconds
    assert bench.job_rate(4, 20, 1.0) == pytest.approx(80_000.0)
