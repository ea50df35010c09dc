"""The data-parallel step on one GPU (a one-rank NCCL group, in a child
process so that its NCCL state ends with it).

  * One rank: DataParallelStep (gradient-only step, reduce-scatter, slice
    update, all-gather, operand refresh) must give the gradients of the fused
    single-GPU step bit for bit, and its parameters up to fp32 rounding of
    the update, over two steps (the second with momentum).
  * The dropout rows: a gradient-only step of images k .. k + B - 1 with
    image_offset = k drops exactly the units the oracle's mask rows k .. of
    the whole batch drop.
More ranks run the same host logic; tests/test_dp_gloo.py checks it on CPU
ranks against the oracle's step on the whole batch."""
import os
import socket

import numpy as np
import pytest

pytestmark = pytest.mark.gpu


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _child(port, q):
    import datetime

    import torch
    import torch.distributed as dist
    torch.cuda.set_device(0)
    dist.init_process_group("nccl", init_method="tcp://127.0.0.1:%d" % port, rank=0,
                            world_size=1, timeout=datetime.timedelta(seconds=120),
                            device_id=torch.device("cuda", 0))
    out = {}
    try:
        _run(out)
    except Exception as e:  # reported to the parent instead of a silent queue timeout
        out["error"] = repr(e)
    finally:
        dist.barrier()
        dist.destroy_process_group()
    q.put(out)


def _run(out):
    import numpy as np
    import torch

    import oracle
    from deep_cnn_image_b200 import alexnet as ax
    from deep_cnn_image_b200 import synthetic
    from deep_cnn_image_b200.dp import DataParallelStep
    B = 8
    xs = [synthetic.to_bf16(synthetic.images(300 + i, B))[0].cuda() for i in range(2)]
    ys = [torch.from_numpy(synthetic.labels(310 + i, B)).cuda() for i in range(2)]
    a = ax.AlexNet(batch_max=B, keep_grads=1, seed=77)
    b = ax.AlexNet(batch_max=B, keep_grads=1, seed=77)
    dp = DataParallelStep(a)
    n = ax.param_count(a.cfg)
    gerr, perr = [], []
    for i in range(2):
        dp.step(xs[i], ys[i], B, 0.01)
        b.train_step(xs[i], ys[i], B, 0.01)
        torch.cuda.synchronize()
        ga = a.device_buffer(2).cpu().numpy()
        gb = torch.zeros(n, dtype=torch.float32)
        b.get_grads(gb)
        gerr.append(float(np.abs(ga - gb.numpy()).max()))
        pa = a.device_buffer(0).cpu().numpy()
        pb = b.device_buffer(0).cpu().numpy()
        perr.append(float(np.abs(pa - pb).max() / np.abs(pb).max()))
    out["grad_max_diff"] = gerr
    out["param_rel_diff"] = perr
    out["status"] = (a.get_status(), b.get_status())
    # dropout rows of the whole batch: images 4..7 with image_offset 4
    c = ax.AlexNet(batch_max=4, keep_grads=1, seed=91)
    c.train_grads(xs[0][4:].clone(), ys[0][4:].clone(), 4, 4)
    f6 = torch.empty((4, 4096), dtype=torch.bfloat16, device="cuda")
    c.debug_copy(30, f6)
    torch.cuda.synchronize()
    got = f6.float().cpu().numpy()
    step = 0
    keep = oracle.dropout_mask(91, 6, step, 4, 4096, row0=4)
    out["dropped_nonzero"] = int(np.count_nonzero(got[keep == 0]))
    out["kept_nonzero"] = int(np.count_nonzero(got[keep == 1]))
    other = oracle.dropout_mask(91, 6, step, 4, 4096, row0=0)
    out["rows0_dropped_nonzero"] = int(np.count_nonzero(got[other == 0]))


def test_one_rank_data_parallel_step_matches_the_fused_step():
    import torch.multiprocessing as mp
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    p = ctx.Process(target=_child, args=(_free_port(), q))
    p.start()
    out = q.get(timeout=600)
    p.join(timeout=120)
    print("data-parallel one-rank check: %s" % out)
    assert "error" not in out, out["error"]
    assert p.exitcode == 0
    assert out["status"] == (0, 0)
    assert out["grad_max_diff"] == [0.0, 0.0]
    assert max(out["param_rel_diff"]) < 1e-6
    assert out["dropped_nonzero"] == 0 and out["kept_nonzero"] > 1000
    # the offset matters: the first rows' mask would drop units that are on
    assert out["rows0_dropped_nonzero"] > 1000
