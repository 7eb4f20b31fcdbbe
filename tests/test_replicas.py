"""The multi-GPU mode of bench.py is replicas only: every rank runs the whole
block step on its own GPU, no collective touches the data path, and the job's
time is the slowest rank's.  This covers that host-side plumbing with two
gloo ranks on the CPU: rank environment, the max-over-ranks reduction and
the whole-job throughput.
"""
import os
import socket

import pytest
import torch.multiprocessing as mp

import bench


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, times, out_q):
    import datetime

    import torch.distributed as dist

    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        ws, r, local = bench.dist_env()
        worst = bench.max_over_ranks(times[rank], dist, "cpu")
        dist.barrier()
        out_q.put((r, ws, local, worst))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_agree_on_the_slowest_replica():
    world, port = 2, _free_port()
    times = [12.5, 17.25]            # ms of timed steps on each rank
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, times, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    got = sorted(q.get(timeout=10) for _ in range(world))
    assert [g[0] for g in got] == [0, 1]
    assert all(g[1] == world and g[2] == g[0] for g in got)
    assert all(g[3] == pytest.approx(max(times)) for g in got)


def test_job_throughput_counts_every_replica():
    flops, steps, ms = 6.04e10, 200, 22.0
    one = bench.job_tflops(1, flops, steps, ms)
    assert one == pytest.approx(flops * steps / (ms * 1e-3) / 1e12)
    # N replicas doing the same work in the same (max-over-ranks) time: N times the job rate
    assert bench.job_tflops(4, flops, steps, ms) == pytest.approx(4 * one)


def test_single_process_needs_no_collective():
    assert bench.max_over_ranks(3.5, None, "cpu") == 3.5
