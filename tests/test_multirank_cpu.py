"""The bench's multi-rank host logic on CPU: two gloo ranks, no GPU.

The path shards nothing (every rank runs a full replica), so the only
cross-rank steps are the timing reduction and the whole-job value.  Each rank
must report the slowest rank's times, and the value must be the work of all
ranks over that time.  The reference arm runs on rank 0 alone."""
import argparse
import os
import socket
import sys
from datetime import timedelta

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    import torch.distributed as dist

    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=timedelta(seconds=60))
    try:
        import bench

        # rank r measured (1 + r) ms for the step and (5 - r) ms end to end
        got = bench.max_over_ranks([1.0 + rank, 5.0 - rank], dist, "cpu")
        dist.barrier()
        q.put((rank, got))
    finally:
        dist.destroy_process_group()


def test_timings_are_max_over_two_gloo_ranks():
    import multiprocessing as mp

    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    try:
        results = sorted(q.get(timeout=120) for _ in procs)
    finally:
        for p in procs:
            p.join(timeout=60)
            if p.is_alive():
                p.kill()
    assert [r for r, _ in results] == [0, 1]
    for _, got in results:
        assert got == [2.0, 5.0]  # max of (1, 2) and of (5, 4)
    assert all(p.exitcode == 0 for p in procs)


def test_single_rank_reduction_is_identity_and_value_is_weak_scaling():
    sys.path.insert(0, ROOT)
    import bench

    assert bench.max_over_ranks([0.25, 3], None, "cpu") == [0.25, 3.0]
    # 1.374e11 FLOP per rank in 0.2 ms: 687 TOPS on one GPU, 8x that on eight
    one = bench.whole_job_tops(1, 1.374e11, 0.2)
    assert one == pytest.approx(687.0)
    assert bench.whole_job_tops(8, 1.374e11, 0.2) == pytest.approx(8 * one)


def test_reference_arm_runs_on_rank_zero_only(capsys):
    sys.path.insert(0, ROOT)
    import bench
    from bit_quantized_attention_channel_b200 import workloads as wl

    args = argparse.Namespace(steps=1, warmup=3, mode="max")
    assert bench.run_reference(args, wl.WORKLOADS["llm"], rank=1, world=2) is None
    assert capsys.readouterr().out == ""


def test_reference_arm_reports_the_steps_it_ran(capsys):
    """The reference arm runs W untimed and K timed oracle samples; its line
    carries K and W and a per-step time that the run's own wall time covers."""
    import json
    import time

    sys.path.insert(0, ROOT)
    import bench
    from bit_quantized_attention_channel_b200 import workloads as wl

    args = argparse.Namespace(steps=2, warmup=3, mode="max")
    t0 = time.perf_counter()
    bench.run_reference(args, wl.WORKLOADS["tiny"], rank=0, world=1)
    wall = time.perf_counter() - t0
    line = json.loads(capsys.readouterr().out.strip().splitlines()[-1])
    assert line["impl"] == "reference" and line["steps"] == 2 and line["warmup"] == 3
    assert 0 < line["ms_per_step"] * line["steps"] / 1e3 <= wall
    assert line["value"] > 0 and line["cpu_baseline"]["kind"] == "oracle"
