"""The multi-rank bench path on CPU: two gloo ranks run the replica helpers.

With N > 1 GPUs every rank runs an independent replica of the workload (the
decoder has no exchange step); the ranks only line up the timed region and take
the slowest rank's time, and the whole-job throughput is the units of all ranks
over that time. Here two CPU processes with the gloo backend stand in for the
GPU ranks (the helpers take the process group and a device, nothing else).
"""
import datetime
import os
import socket

import pytest
import torch
import torch.multiprocessing as mp

import bench

WORLD = 2


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, port, seconds, out):
    import torch.distributed as dist
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=WORLD, timeout=datetime.timedelta(seconds=60))
    try:
        bench.replica_barrier(WORLD)
        t = bench.replica_max(seconds[rank], WORLD, torch.device("cpu"))
        v = bench.replica_throughput(WORLD, 3, 2304, t)
        bench.replica_barrier(WORLD)
        out.put((rank, t, v))
    finally:
        dist.destroy_process_group()


def _run(seconds):
    ctx = mp.get_context("spawn")
    out = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, port, seconds, out)) for r in range(WORLD)]
    for p in procs:
        p.start()
    res = [out.get(timeout=120) for _ in range(WORLD)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    return sorted(res)


def test_every_rank_gets_the_slowest_rank_time_and_the_whole_job_throughput():
    seconds = [1.25, 2.5]
    res = _run(seconds)
    assert [r for r, _, _ in res] == [0, 1]
    for _, t, v in res:
        assert t == max(seconds)
        assert v == pytest.approx(WORLD * 3 * 2304 / max(seconds))


def test_single_rank_needs_no_process_group():
    assert bench.replica_max(1.5, 1, torch.device("cpu")) == 1.5
    bench.replica_barrier(1)
    assert bench.replica_throughput(1, 5, 2304, 2.0) == pytest.approx(5 * 2304 / 2.0)


def test_reference_arm_runs_on_rank_zero_only(capsys):
    class Args:
        steps, warmup, gpus = 1, 0, 2
    bench.run_reference(Args, rank=1)  # the other ranks exit without work or output
    assert capsys.readouterr().out == ""
