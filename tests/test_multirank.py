"""The bench's multi-rank plumbing on CPU: two gloo ranks (one process per
rank, as torchrun starts them on GPUs).  Every rank runs an independent
replica of the layer; the only cross-rank steps are the barrier around the
timed region and the max of the ranks' times, and only rank 0 prints."""
import os
import socket
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    sys.path.insert(0, ROOT)
    import datetime

    import torch.distributed as dist

    import bench
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank,
                            world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        bench.barrier(world)
        # each rank's own step time; the job's time is the slowest rank's
        t = bench.max_over_ranks(1.5 + rank, world)
        bench.barrier(world)
        out.put((rank, t))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_share_the_max_time():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
    codes = [p.exitcode for p in procs]
    for p in procs:
        if p.is_alive():
            p.kill()
    assert codes == [0, 0], codes
    got = dict(q.get(timeout=10) for _ in range(2))
    assert got == {0: 2.5, 1: 2.5}


def test_reference_arm_runs_on_rank_zero_only(capsys):
    # under torchrun the reference arm (the CPU oracle) runs once, on rank 0
    sys.path.insert(0, ROOT)
    import bench

    class A:
        workload = "decode"
        steps = 1
        warmup = 3
    bench.run_reference(A(), world=2, rank=1)
    assert capsys.readouterr().out == ""
