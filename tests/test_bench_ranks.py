"""The multi-rank host logic of bench.py on CPU: two gloo ranks on
127.0.0.1 take the element-wise maximum of their timings (the slowest rank
sets the whole job's time), and the whole-job rate counts every rank's
images."""
import os
import socket

import pytest


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank(rank, world, port, q):
    import torch.distributed as dist
    import bench
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        # rank 0 is slower on the first timing, rank 1 on the second
        got = bench.max_over_ranks([10.0 - rank, 3.0 + 4.0 * rank], world, "cpu")
        q.put((rank, got))
    finally:
        dist.barrier()
        dist.destroy_process_group()


def test_max_over_two_gloo_ranks():
    import torch.multiprocessing as mp
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    out = dict(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    assert out[0] == [10.0, 7.0] and out[1] == [10.0, 7.0]


def test_whole_job_rate_counts_every_rank():
    import bench
    # two ranks x 128 images x 10 steps in 20 ms on the slowest rank
    assert bench.whole_job_rate(128, 2, 10, 20.0) == pytest.approx(128_000.0)
    assert bench.max_over_ranks([1.5, 2.5], 1, "cpu") == [1.5, 2.5]
