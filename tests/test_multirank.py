"""bench.py's multi-rank host logic on CPU: two gloo ranks.

With N GPUs the bench runs one independent replica of the workload per rank
(replicas only: the decode step has no exchange between graphs), times each
rank on its own device, and reports the whole job as N x steps over the
slowest rank's time.  These tests run that logic with the gloo backend,
world size 2, without a GPU.
"""
import os
import socket
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as sk:
        sk.bind(("127.0.0.1", 0))
        return sk.getsockname()[1]


def _rank_main(rank, world, port, results):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    sys.path.insert(0, ROOT)
    import datetime
    import torch.distributed as dist
    import bench
    try:
        dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
        r, w, lr = bench.rank_env()
        own_ms = 5.0 + 3.0 * rank                       # rank 1 is the slower replica
        ms = bench.max_over_ranks(dist, own_ms, "cpu")
        rate = bench.job_rate(w, 100, ms)
        dist.barrier()
        dist.destroy_process_group()
        results.put((rank, r, w, lr, ms, rate, None))
    except Exception as exc:                            # reported to the parent
        results.put((rank, None, None, None, None, None, repr(exc)))


def test_max_over_ranks_and_job_rate_two_gloo_ranks():
    import torch.multiprocessing as mp
    ctx = mp.get_context("spawn")
    results = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, results)) for r in range(2)]
    for p in procs:
        p.start()
    got = [results.get(timeout=120) for _ in procs]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    got.sort()
    for rank, r, w, lr, ms, rate, err in got:
        assert err is None, err
        assert (r, w, lr) == (rank, 2, rank)
        assert ms == 8.0                                # the slowest rank's time, on every rank
        assert rate == pytest.approx(2 * 100 / 8e-3)    # whole job: both replicas' steps


def test_single_process_defaults():
    sys.path.insert(0, ROOT)
    import bench
    for k in ("RANK", "WORLD_SIZE", "LOCAL_RANK"):
        os.environ.pop(k, None)
    assert bench.rank_env() == (0, 1, 0)
    assert bench.max_over_ranks(None, 3.5, "cpu") == 3.5
    assert bench.job_rate(1, 200, 100.0) == pytest.approx(2000.0)


def test_reference_arm_runs_on_rank_zero_only():
    sys.path.insert(0, ROOT)
    import argparse
    import bench
    args = argparse.Namespace(warmup=3, steps=1)
    assert bench.reference_arm(args, rank=1, world=2) == 0   # other ranks exit without work
