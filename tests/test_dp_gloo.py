"""The data-parallel step's host logic on CPU ranks (gloo, 127.0.0.1).

Each rank's engine here is the oracle: its gradients come from the oracle's
step of the rank's images (their rows of the whole batch's dropout masks),
and its slice update is the oracle's update rule.  Two (and three) ranks
running deep_cnn_image_b200.dp.DataParallelStep must end with the parameters
of one oracle step on the concatenated batch, and each rank's momentum slice
must be that step's momentum there: this checks the bucketing, the slice
offsets, the reduce-scatter arithmetic (sum, then the 1 / ranks scale), the
dropout row offsets and the in-place all-gather.  The GPU engine runs the
same host logic with NCCL."""
import os
import socket

import numpy as np
import pytest

import oracle

SEED, STEP, LR = 17, 3, 0.05


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _problem(B):
    net = oracle.small_net()
    n = oracle.param_count(net)
    r = np.random.default_rng(41)
    params = r.standard_normal(n) * 0.2
    for (wo, wl, bo, bl) in oracle.param_layout(net):
        params[bo:bo + bl] = r.uniform(0.05, 0.3, bl)
    vel = r.standard_normal(n) * 1e-3
    x = r.standard_normal((B, 67, 67, 3))
    y = r.integers(0, 10, B).astype(np.int32)
    return net, params, vel, x, y


class OracleEngine:
    """The engine interface of DataParallelStep on the CPU oracle."""

    def __init__(self, net, params, vel):
        import torch
        self.net = net
        self.p = torch.from_numpy(params.astype(np.float32).copy())
        self.v = torch.from_numpy(vel.astype(np.float32).copy())
        self.g = torch.zeros_like(self.p)
        self.steps = 0

    def device_buffer(self, which):
        return {0: self.p, 1: self.v, 2: self.g}[which]

    def train_grads(self, x, labels, B, image_offset, loss=None):
        _, _, _, g, _ = oracle.train_step_rows(self.net, self.p.numpy().astype(np.float64),
                                               np.zeros(self.p.numel()), x, labels,
                                               image_offset, lr=0.0, seed=SEED, step=STEP)
        self.g.copy_(__import__("torch").from_numpy(g.astype(np.float32)))

    def stream_wait_fc_grads(self, stream):
        pass

    def sgd_range(self, offset, count, gsum, scale, lr):
        w = self.p[offset:offset + count].numpy().astype(np.float64)
        v = self.v[offset:offset + count].numpy().astype(np.float64)
        w2, v2 = oracle.sgd(w, v, scale * gsum.numpy().astype(np.float64), lr)
        self.p[offset:offset + count] = __import__("torch").from_numpy(w2.astype(np.float32))
        self.v[offset:offset + count] = __import__("torch").from_numpy(v2.astype(np.float32))

    def params_updated(self):
        self.steps += 1


def _rank(rank, world, port, B, fc_start, q):
    import torch.distributed as dist
    from deep_cnn_image_b200.dp import DataParallelStep
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        net, params, vel, x, y = _problem(B * world)
        eng = OracleEngine(net, params, vel)
        dp = DataParallelStep(eng, fc_start=fc_start)
        mine = slice(rank * B, rank * B + B)
        dp.step(x[mine], y[mine], B, LR)
        slices = [(bk.start + bk.mine[0], bk.start + bk.mine[1]) for bk in dp.buckets]
        q.put((rank, eng.p.numpy().copy(), eng.v.numpy().copy(), slices, eng.steps))
    finally:
        dist.barrier()
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 3])
def test_data_parallel_step_equals_one_step_on_the_whole_batch(world):
    import torch.multiprocessing as mp
    B = 2
    net, params, vel, x, y = _problem(B * world)
    n = oracle.param_count(net)
    lay = oracle.param_layout(net)
    fc_start = lay[5][0]  # the FC layers are the blob's tail
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank, args=(r, world, port, B, fc_start, q))
             for r in range(world)]
    for p in procs:
        p.start()
    out = {}
    for _ in procs:
        r, p_, v_, sl, steps = q.get(timeout=300)
        out[r] = (p_, v_, sl, steps)
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    # one oracle step on the whole batch, from the same fp32 starting values
    p32 = params.astype(np.float32).astype(np.float64)
    v32 = vel.astype(np.float32).astype(np.float64)
    _, want_p, want_v, _, _ = oracle.train_step(net, p32, v32, x, y, lr=LR, seed=SEED,
                                                step=STEP)
    covered = np.zeros(n, bool)
    for r in range(world):
        got_p, got_v, slices, steps = out[r]
        assert steps == 1
        np.testing.assert_allclose(got_p, want_p, rtol=0, atol=2e-6)
        for a, b in slices:
            np.testing.assert_allclose(got_v[a:b], want_v[a:b], rtol=1e-5, atol=1e-9)
            covered[a:b] = True
    assert covered.all()
    # the update moved the parameters (the check is not vacuous)
    assert np.abs(want_p - p32).max() > 1e-3
