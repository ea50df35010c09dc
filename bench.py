#!/usr/bin/env python
"""Benchmark: one AlexNet bf16 training step (forward, backward, SGD update)
of the grouped network on a batch of 128 synthetic 227x227x3 images per GPU.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

Prints one JSON line (rank 0).  For N > 1 launch one process per GPU with
torch.distributed.run: data-parallel training, each rank 128 images of its
own per step, the gradients averaged over the ranks with NCCL
(reduce-scatter, per-slice update, all-gather of the parameters), so the
scaling is weak and `value` is the images of all ranks divided by the
slowest rank's device time.

Timing: W untimed steps; then K steps back to back between two CUDA events
on the library's stream, barrier + synchronize on both sides; max over
ranks.  A step's working set (about 1.2 GB of activations, gradients and
weights) is far larger than the 126 MB L2, so no step finds the previous
step's data there and no flush is needed.  The GEMM roofline comes from a
separate pass with per-GEMM events (L2 flushed before each step).  `e2e`
times the same steps through the public call with every batch copied from
pinned host memory and every loss copied back inside the timed span (the
copy of batch i+1 overlaps step i on a second stream).

`--mode forward|augment|tencrop|fp32|ensemble|knn|train_variant` times the
other workloads instead (not the headline): the batch-128 inference
forward, the batch-512 training step fed by on-device augmentation of
256x256 uint8 sources, batch-256 ten-crop inference, the fp32 ungrouped
batch-1 forward, a five-network batch-128 ensemble, 128 nearest-neighbour
queries against a million 4096-d features, and the batch-128 training step
of one of the pages' ablations (`--variant pool2|nolrn|nodropout|ungrouped`).

`--impl reference` times the CPU oracle (the plain fp64 C implementation
under oracle/) as it stands on the host cores: each step is a training step
on one image of the same workload.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "images/sec, AlexNet bf16 train step, batch 128, 1×B200; % of bf16 tensor roofline"
# DRAM bytes (read + written) per batch-128 step of the GEMM class's 20
# launches, summed from the per-launch ncu counters recorded in
# profiles/train_step_counters_b128.md (None once those kernels change)
GEMM_CLASS_TRAFFIC_BYTES = 813034496
UNIT = "images/s"
WORKLOAD = "AlexNet (grouped conv2/4/5) bf16 training step: forward + backward + SGD-momentum, " \
           "227x227x3 NHWC inputs ~N(0,1), labels U[0,1000)"
# Per-image FLOPs of one training step (2 x multiply-adds of the forward
# convolutions and FC layers, their data gradients except conv1's, and their
# weight gradients), from the layer shapes of the network.
FWD_MACS_PER_IMAGE = 724406816
CONV1_MACS_PER_IMAGE = 55 * 55 * 96 * 363


def step_flops_per_image():
    return 2.0 * (3 * FWD_MACS_PER_IMAGE - CONV1_MACS_PER_IMAGE)


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return {"hbm_gbs": float(p["hbm_gbs"]), "bf16_tflops": float(p["bf16_tflops"]),
                "bf16_tflops_sustained": float(p.get("bf16_tflops_sustained", p["bf16_tflops"])),
                "source": "measured"}
    except Exception:
        return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0,
                "source": "fallback"}


class ClockSampler:
    """nvidia-smi samples of SM clock and throttle reasons while running."""
    QUERY = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index):
        self.proc = None
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "--query-gpu=" + self.QUERY, "--format=csv,noheader,nounits",
                 "-lms", "200", "-i", str(gpu_index)],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        time.sleep(0.25)
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=5)
        except Exception:
            self.proc.kill()
            return None
        sm, smax, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in out.strip().splitlines():
            f = [x.strip() for x in line.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                smax.append(float(f[2]))
            except ValueError:
                continue
            for name, v in zip(names, f[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(name)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(smax),
                "reasons": sorted(reasons), "samples": len(sm)}


def max_over_ranks(values, world, device):
    """Element-wise maximum over all ranks of this rank's timings (ms): the
    whole job is as slow as its slowest rank."""
    import torch
    t = torch.tensor(values, dtype=torch.float64, device=device)
    if world > 1:
        import torch.distributed as dist
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return t.tolist()


def whole_job_rate(images_per_rank_step, world, steps, ms_max):
    """Images per second of all ranks together over `steps` steps that took
    ms_max milliseconds on the slowest rank."""
    return world * images_per_rank_step * steps / (ms_max / 1e3)


def dist_setup():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


def cpu_baseline_oracle(images_per_step, steps):
    """Time the oracle's training step (fp64 C loops, OpenMP over the batch)
    on the host cores; returns (images/s, cores, seconds)."""
    cores = len(os.sched_getaffinity(0)) if hasattr(os, "sched_getaffinity") else os.cpu_count()
    os.environ["OMP_NUM_THREADS"] = str(cores)
    import numpy as np

    import oracle
    from deep_cnn_image_b200 import synthetic
    net = oracle.alexnet(grouped=True)
    n = oracle.param_count(net)
    params = synthetic.params(1).astype(np.float64)
    vel = np.zeros(n)
    x = synthetic.images(2, images_per_step).astype(np.float64)
    y = synthetic.labels(3, images_per_step)
    t0 = time.perf_counter()
    for i in range(steps):
        _, params, vel, _, _ = oracle.train_step(net, params, vel, x, y, lr=0.01, seed=1, step=i)
    dt = time.perf_counter() - t0
    return images_per_step * steps / dt, cores, dt


def run_reference(args):
    world, rank, _ = dist_setup()
    if rank != 0:
        return 0
    # the oracle trains on one image per step: the same network, input shape
    # and update; warm-up steps are run and not timed
    cpu_baseline_oracle(1, args.warmup) if args.warmup > 0 else None
    value, cores, dt = cpu_baseline_oracle(1, args.steps)
    sample = "%d training steps on 1 image each (the batch-128 workload's per-image work)" % args.steps
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * dt / max(args.steps, 1),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic",
        # our arm's workload; each timed step is a bounded sample of it
        "config": {"workload": WORKLOAD, "global_batch": 128, "batch_per_gpu": 128,
                   "parallelism": "single", "sampled_images_per_step": 1},
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": cores, "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


def run_ours(args):
    from datetime import timedelta

    import torch
    import torch.distributed as dist

    world, rank, local = dist_setup()
    torch.cuda.set_device(local)
    if world > 1:
        dist.init_process_group("nccl", timeout=timedelta(seconds=300),
                                device_id=torch.device("cuda", local))
    from deep_cnn_image_b200 import alexnet as ax
    from deep_cnn_image_b200 import synthetic

    B = args.batch
    # every rank starts from the same parameters (same seed); each trains on
    # its own images.  One GPU: the fused single-GPU step.  N GPUs: the
    # data-parallel step (gradients reduce-scattered, the update applied per
    # slice, parameters all-gathered; deep_cnn_image_b200/dp.py).
    net = ax.AlexNet(batch_max=B, seed=1234, keep_grads=1 if world > 1 else 0)
    x_host, _ = synthetic.to_bf16(synthetic.images(100 + rank, B))
    y_np = synthetic.labels(200 + rank, B)
    x = x_host.cuda()
    y = torch.from_numpy(y_np).cuda()
    loss = torch.zeros(1, dtype=torch.float32, device="cuda")
    flush = torch.empty(256 << 20, dtype=torch.uint8, device="cuda")
    stream = torch.cuda.current_stream()
    if world > 1:
        from deep_cnn_image_b200.dp import DataParallelStep
        dp_step = DataParallelStep(net)

        def train(xb, yb, lo=loss):
            dp_step.step(xb, yb, B, 0.01, lo)
    else:
        def train(xb, yb, lo=loss):
            net.train_step(xb, yb, B, 0.01, lo)

    def barrier():
        torch.cuda.synchronize()
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()

    for _ in range(args.warmup):
        train(x, y)
    barrier()

    # ---- device-timed steps (inputs resident in HBM), back to back: one
    # step's working set (activations, gradients, weights: about 1.2 GB)
    # is far larger than the 126 MB L2, so nothing survives in L2 from one
    # step to the next and no flush is needed
    sampler = ClockSampler(local) if rank == 0 else None
    e_start = torch.cuda.Event(enable_timing=True)
    e_end = torch.cuda.Event(enable_timing=True)
    barrier()
    t_wall = time.perf_counter()
    e_start.record(stream)
    for _ in range(args.steps):
        train(x, y)
    e_end.record(stream)
    barrier()
    t_wall = time.perf_counter() - t_wall
    clocks = sampler.stop() if sampler else None
    ms = e_start.elapsed_time(e_end)
    assert net.get_status() == ax.OK, "device status after the timed steps"
    loss_val = float(loss.item())

    # ---- per-GEMM timing for the roofline: event pairs recorded inside the
    # replayed step graph around every GEMM launch (a separate pass, L2
    # flushed before each step)
    stats = {"launches": 0, "gemm_launches": 0, "gemm_flops": 0.0, "gemm_ms": 0.0}
    # the class split by kind: convolutions (tensor-bound) and the FC forward
    # and data-gradient products (HBM-bound at batch 128: every weight is
    # read once per launch for 2 x 128 FLOPs)
    by_kind = {0: [0.0, 0.0], 1: [0.0, 0.0]}
    stat_steps = min(args.steps, 20)
    net.stats_enable(True)
    for _ in range(2):
        net.train_step(x, y, B, 0.01, loss)
    net.stats_read()
    for _ in range(stat_steps):
        flush.zero_()
        net.train_step(x, y, B, 0.01, loss)
        st = net.stats_read()  # this step's GEMM times (synchronises the stream)
        for k in stats:
            stats[k] += st[k]
        for kind, fl, t in net.stats_launches():
            if kind in by_kind:
                by_kind[kind][0] += fl
                by_kind[kind][1] += t
    net.stats_enable(False)
    for _ in range(2):  # the step graph without timing nodes
        net.train_step(x, y, B, 0.01, loss)
    barrier()

    # ---- end to end through the public call, host buffers: every step's
    # batch is copied from pinned host memory and its loss read back inside
    # the timed span; the copy of batch i+1 (its own stream, into the other
    # of two device buffers) overlaps step i, and so does the read-back of
    # step i's loss (from one of two device loss slots, on the copy stream,
    # so that the compute stream does not wait for it).  The step's
    # activations (about 1 GB) exceed the L2, so no flush is needed between
    # steps.
    x_pin = x_host.pin_memory()
    y_pin = torch.from_numpy(y_np).pin_memory()
    loss_pin = torch.zeros(args.steps, dtype=torch.float32).pin_memory()
    xs = [x, torch.empty_like(x)]
    ys = [y, torch.empty_like(y)]
    losses = [torch.zeros(1, dtype=torch.float32, device="cuda") for _ in range(2)]
    copy_stream = torch.cuda.Stream()
    copied = [torch.cuda.Event(), torch.cuda.Event()]
    consumed = [torch.cuda.Event(), torch.cuda.Event()]
    e_start = torch.cuda.Event(enable_timing=True)
    e_end = torch.cuda.Event(enable_timing=True)

    def stage(i):
        buf = i % 2
        with torch.cuda.stream(copy_stream):
            if i >= 2:
                copy_stream.wait_event(consumed[buf])
            xs[buf].copy_(x_pin, non_blocking=True)
            ys[buf].copy_(y_pin, non_blocking=True)
            copied[buf].record(copy_stream)

    barrier()
    e_start.record(stream)
    copy_stream.wait_event(e_start)
    stage(0)
    for i in range(args.steps):
        buf = i % 2
        if i + 1 < args.steps:
            stage(i + 1)
        stream.wait_event(copied[buf])
        train(xs[buf], ys[buf], losses[buf])
        consumed[buf].record(stream)
        # step i's loss, read back on the copy stream: queued before the copy
        # that refills this buffer pair, which step i + 2 (the next writer of
        # the slot) waits for
        with torch.cuda.stream(copy_stream):
            copy_stream.wait_event(consumed[buf])
            loss_pin[i:i + 1].copy_(losses[buf], non_blocking=True)
    stream.wait_stream(copy_stream)
    e_end.record(stream)
    barrier()
    ms_e2e = e_start.elapsed_time(e_end)

    ms_max, ms_e2e_max = max_over_ranks([ms, ms_e2e], world, "cuda")
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    if rank != 0:
        return 0

    peaks = load_peaks()
    images = world * B * args.steps
    value = whole_job_rate(B, world, args.steps, ms_max)
    step_ms = ms_max / args.steps
    step_tflops = step_flops_per_image() * B / (step_ms / 1e3) / 1e12
    gemm_tflops = stats["gemm_flops"] / (stats["gemm_ms"] / 1e3) / 1e12 if stats["gemm_ms"] else None
    # each GEMM launch is timed alone (event pair, milliseconds at most) and
    # the timed steps span tens of milliseconds, not the seconds-long run the
    # sustained figure describes: the burst peak is the denominator
    peak = peaks["bf16_tflops"]
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": step_ms, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": WORKLOAD, "global_batch": world * B, "batch_per_gpu": B,
                   "parallelism": ("dp%d" % world) if world > 1 else "single",
                   "l2": "no flush: a step's ~1.2 GB working set exceeds the 126 MB L2"},
        "roofline": {
            "kernel": "tcgen05 GEMM (conv forward, data- and weight-gradient, FC forward and data-"
                      "gradient launches; the FC weight-gradient launches apply the SGD update in "
                      "their epilogue, are HBM-bound and are not counted here)",
            "bound": "tensor", "achieved": gemm_tflops, "peak": peak, "unit": "TFLOP/s",
            "frac": gemm_tflops / peak if gemm_tflops else None,
            "traffic": GEMM_CLASS_TRAFFIC_BYTES if B == 128 and world == 1 else None,
            "traffic_unit": "bytes per step (DRAM read + write of the class's launches, ncu)",
            "peak_source": peaks["source"] + " bf16_tflops (burst)",
            "gemm_launches_per_step": stats["gemm_launches"] / stat_steps,
            "gemm_ms_per_step": stats["gemm_ms"] / stat_steps,
            "gemm_timing": f"{stat_steps} separate steps with per-GEMM events, L2 flushed before each",
        },
        "roofline_by_kind": {
            "conv": {"bound": "tensor",
                     "achieved": by_kind[0][0] / (by_kind[0][1] / 1e3) / 1e12 if by_kind[0][1] else None,
                     "peak": peak, "unit": "TFLOP/s",
                     "frac": by_kind[0][0] / (by_kind[0][1] / 1e3) / 1e12 / peak if by_kind[0][1] else None,
                     "ms_per_step": by_kind[0][1] / stat_steps},
            "fc": {"bound": "hbm",
                   # bf16 weights read once per launch: FLOPs / batch bytes
                   "achieved": by_kind[1][0] / B / (by_kind[1][1] / 1e3) / 1e9 if by_kind[1][1] else None,
                   "peak": peaks["hbm_gbs"], "unit": "GB/s",
                   "frac": by_kind[1][0] / B / (by_kind[1][1] / 1e3) / 1e9 / peaks["hbm_gbs"]
                   if by_kind[1][1] else None,
                   "ms_per_step": by_kind[1][1] / stat_steps},
        },
        "step_roofline": {"achieved": step_tflops, "peak": peak, "unit": "TFLOP/s",
                          "frac": step_tflops / peak,
                          "flops_per_image": step_flops_per_image()},
        "e2e": {"value": images / (ms_e2e_max / 1e3), "unit": UNIT,
                "h2d_bytes_per_step": x_pin.numel() * 2 + y_pin.numel() * 4,
                "overlap": "batch i+1 copied on a second stream during step i",
                "d2h_bytes_per_step": 4},
        "gpu_launches": int(round(stats["launches"] / stat_steps)) * args.steps,
        "clocks": clocks,
        "loss_last": loss_val,
        "wall_s_timed": t_wall,
    }
    if world == 1 and not args.no_cpu_baseline:
        v, cores, dt = cpu_baseline_oracle(args.cpu_images, 1)
        line["cpu_baseline"] = {"value": v, "unit": UNIT, "cores": cores, "kind": "oracle",
                                "sample": "one training step of the oracle on %d images "
                                          "(fp64 C loops), %.1f s" % (args.cpu_images, dt)}
    print(json.dumps(line), flush=True)
    return 0


def run_mode(args):
    """The non-headline workloads: forward (batch 128, inference),
    augment (batch 512: augmentation + training step), tencrop (batch 256
    source images, 10 crops each).  Device-timed, inputs resident."""
    import numpy as np
    import torch
    from deep_cnn_image_b200 import alexnet as ax
    from deep_cnn_image_b200 import synthetic

    torch.cuda.set_device(0)
    stream = torch.cuda.current_stream()
    # the pages' ablations (throughput only): non-overlapping 2x2 pooling, no
    # LRN, no dropout, ungrouped convolutions
    variant = {"pool2": {"pool_size": 2}, "nolrn": {"lrn_on": 0}, "nodropout": {"dropout_on": 0},
               "ungrouped": {"grouped": 0}, "none": {}}[args.variant]
    if args.mode == "fp32":
        # batch 1, fp32, ungrouped, inference: latency-bound, reads the fp32
        # weights once per image
        B = 1
        net = ax.AlexNet(batch_max=1, seed=1, dtype=ax.FP32, grouped=0)
        x = torch.from_numpy(synthetic.images(100, 1)).cuda()
        logits = torch.empty((1, 1000), dtype=torch.float32, device="cuda")
        probs = torch.empty_like(logits)
        def step():
            net.forward(x, 1, ax.INFERENCE, logits, probs)
        images, metric = 1, "images/sec, AlexNet fp32 ungrouped inference forward, batch 1"
        flops = 2.0 * 1135256096
    elif args.mode == "train_variant":
        B = 128
        net = ax.AlexNet(batch_max=B, seed=1, **variant)
        x = synthetic.to_bf16(synthetic.images(100, B))[0].cuda()
        y = torch.from_numpy(synthetic.labels(200, B)).cuda()
        loss = torch.zeros(1, dtype=torch.float32, device="cuda")
        def step():
            net.train_step(x, y, B, 0.01, loss)
        images = B
        metric = "images/sec, AlexNet bf16 train step, batch 128, variant " + args.variant
        flops = step_flops_per_image()
    elif args.mode == "ensemble":
        # five networks averaged ([S] ILSVRC-2012 results): every image goes
        # through five inference forwards, then the mean softmax and top 5
        B, M = 128, 5
        nets = [ax.AlexNet(batch_max=B, seed=1 + m) for m in range(M)]
        net = nets[0]
        x = synthetic.to_bf16(synthetic.images(100, B))[0].cuda()
        probs = torch.empty((B, 1000), dtype=torch.float32, device="cuda")
        top5 = torch.empty((B, 5), dtype=torch.int32, device="cuda")
        ws = torch.empty(ax.ensemble_workspace_bytes(M, B), dtype=torch.uint8, device="cuda")
        def step():
            ax.ensemble_forward(nets, x, B, probs, top5, ws)
        images = B
        metric = "images/sec, AlexNet bf16 five-network ensemble inference, batch 128"
        flops = M * 2.0 * FWD_MACS_PER_IMAGE
    elif args.mode == "knn":
        # Euclidean retrieval over 4096-d feature vectors ([S] "Qualitative
        # Evaluation"): 128 queries against a base of one million synthetic
        # ReLU-like bf16 features (a stand-in for last-hidden-layer
        # activations of a million images); the base is read once per call
        Q, N, D, K = 128, 1_000_000, 4096, 10
        B = Q
        g = torch.Generator(device="cuda").manual_seed(7)
        base = torch.randn((N, D), device="cuda", dtype=torch.bfloat16, generator=g).relu_()
        qs = torch.randn((Q, D), device="cuda", dtype=torch.bfloat16, generator=g).relu_()
        dist = torch.empty((Q, K), dtype=torch.float32, device="cuda")
        idx = torch.empty((Q, K), dtype=torch.int32, device="cuda")
        ws = torch.empty(ax.knn_workspace_bytes(Q, N), dtype=torch.uint8, device="cuda")
        # a fixed base: its squared norms computed once, outside the timing
        bnorm = torch.empty(N, dtype=torch.float32, device="cuda")
        ax.knn_sqnorms(base, bnorm)
        net = None
        def step():
            ax.knn(qs, base, K, dist, idx, ws, base_sqnorm=bnorm)
        images = Q
        metric = "queries/sec, Euclidean 10-NN of 4096-d bf16 features in a base of 1,000,000"
        flops = 2.0 * N * D
        hbm_bytes = 2.0 * N * D
    elif args.mode == "forward":
        B = 128
        net = ax.AlexNet(batch_max=B, seed=1)
        x = synthetic.to_bf16(synthetic.images(100, B))[0].cuda()
        logits = torch.empty((B, 1000), dtype=torch.float32, device="cuda")
        probs = torch.empty_like(logits)
        def step():
            net.forward(x, B, ax.INFERENCE, logits, probs)
        images, metric = B, "images/sec, AlexNet bf16 inference forward (logits + softmax), batch 128"
        flops = 2.0 * FWD_MACS_PER_IMAGE
    elif args.mode == "augment":
        B = 512
        net = ax.AlexNet(batch_max=B, seed=1)
        src_np = synthetic.source_images(8, B)
        src = torch.from_numpy(src_np).cuda()
        mean = torch.from_numpy(synthetic.mean_image(src_np)).cuda()
        vec, val = synthetic.pca(9)
        vec, val = torch.from_numpy(vec).cuda(), torch.from_numpy(val).cuda()
        x = torch.empty((B, 227, 227, 3), dtype=torch.bfloat16, device="cuda")
        y = torch.from_numpy(synthetic.labels(200, B)).cuda()
        loss = torch.zeros(1, dtype=torch.float32, device="cuda")
        def step():
            net.augment(src, B, mean, vec, val, x)
            net.train_step(x, y, B, 0.01, loss)
        images = B
        metric = "images/sec, AlexNet bf16 train step with on-device augmentation, batch 512"
        flops = step_flops_per_image()
    else:
        B = 256
        net = ax.AlexNet(batch_max=10 * B, seed=1)
        src_np = synthetic.source_images(42, B)
        src = torch.from_numpy(src_np).cuda()
        mean = torch.from_numpy(synthetic.mean_image(src_np)).cuda()
        probs = torch.empty((B, 1000), dtype=torch.float32, device="cuda")
        top5 = torch.empty((B, 5), dtype=torch.int32, device="cuda")
        def step():
            net.tencrop(src, B, mean, probs, top5)
        images = B
        metric = "source images/sec, AlexNet bf16 ten-crop inference (10 forwards each), batch 256"
        flops = 10 * 2.0 * FWD_MACS_PER_IMAGE
    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(args.steps):
        step()
    e1.record(stream)
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1)
    if net is not None:
        assert net.get_status() == ax.OK
    peak = load_peaks()["bf16_tflops"]  # short runs: the burst peak
    value = images * args.steps / (ms / 1e3)
    line = {"metric": metric, "value": value, "unit": "images/s", "n_gpus": 1,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms / args.steps,
            "higher_is_better": True, "dtype": "f32" if args.mode == "fp32" else "bf16",
            "data": "synthetic",
            "config": {"workload": args.mode, "batch": B, "variant": args.variant},
            "step_roofline": {"achieved": flops * value / 1e12, "peak": peak,
                              "unit": "TFLOP/s", "frac": flops * value / 1e12 / peak}}
    if args.mode == "augment":
        # the augmentation kernel alone (HBM-bound): per image the 256x256x3
        # u8 source read once and the 227x227x3 bf16 crop written once (the
        # mean image is shared by the batch)
        a0 = torch.cuda.Event(enable_timing=True)
        a1 = torch.cuda.Event(enable_timing=True)
        reps = 50
        a0.record(stream)
        for _ in range(reps):
            net.augment(src, B, mean, vec, val, x)
        a1.record(stream)
        torch.cuda.synchronize()
        aug_ms = a0.elapsed_time(a1) / reps
        aug_bytes = B * (256 * 256 * 3 + 227 * 227 * 3 * 2)
        hbm = load_peaks()["hbm_gbs"]
        gbs = aug_bytes / (aug_ms / 1e3) / 1e9
        line["augment_kernel"] = {"ms": aug_ms, "bytes": aug_bytes, "achieved": gbs, "peak": hbm,
                                  "unit": "GB/s", "frac": gbs / hbm}
    if args.mode == "knn":
        # the base is streamed once per call: HBM-bound
        gbs = hbm_bytes * args.steps / (ms / 1e3) / 1e9
        hbm = load_peaks()["hbm_gbs"]
        line["unit"] = "queries/s"
        line["config"].update({"base_rows": N, "dims": D, "k": K})
        line["roofline"] = {"bound": "hbm", "achieved": gbs, "peak": hbm, "unit": "GB/s",
                            "frac": gbs / hbm, "traffic": None,
                            "kernel": "base rows read by the dot-product GEMM (N x D bf16)"}
    print(json.dumps(line), flush=True)
    return 0


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--batch", type=int, default=128)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--cpu-images", type=int, default=24)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--mode", choices=["train", "forward", "augment", "tencrop", "fp32",
                                       "ensemble", "knn", "train_variant"], default="train")
    ap.add_argument("--variant", choices=["none", "pool2", "nolrn", "nodropout", "ungrouped"],
                    default="none")
    args = ap.parse_args()
    if args.warmup < 3 and args.impl == "ours":
        args.warmup = 3
    if args.impl == "reference":
        return run_reference(args)
    if args.mode != "train":
        return run_mode(args)
    return run_ours(args)


if __name__ == "__main__":
    sys.exit(main())
