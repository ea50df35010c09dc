"""Data-parallel training step: one process per GPU, the minibatch split
across the ranks, the gradient averaged with collectives of
torch.distributed (NCCL over NVLink on GPUs).

The pages train one network split across two GPUs by its channels
("ImageNet Classification with Deep Convolutional Neural Networks", 3.4
"Training on Multiple GPUs"); that split is kept inside one GPU here (the
grouped convolutions), and more GPUs take more images instead.  Per step:

  1. every rank runs the forward and backward of its own B images without an
     update (dropout rows drawn for the images' places in the whole batch);
  2. the gradients are reduce-scattered (summed) in two buckets: the FC
     layers' (about 96% of the parameters, complete first: their reduction
     starts on a second stream while the convolutions' backward still runs)
     and the convolutions';
  3. each rank applies the SGD update of 3.4 "Training Procedure Details" to
     its slice of each bucket, the gradient scaled by 1 / ranks (the mean of
     the ranks' batch means, i.e. the mean over the whole batch);
  4. the updated fp32 parameters are all-gathered in place, and each rank
     rebuilds its bf16 operand copies.

The momentum lives per slice: a rank's momentum values outside its own
slices are not updated.

`engine` is the network (deep_cnn_image_b200.alexnet.AlexNet created with
keep_grads=1 on a GPU); it provides train_grads, stream_wait_fc_grads,
sgd_range, params_updated and device_buffer.  Collectives that a backend
lacks (reduce-scatter on gloo) are replaced by the all-reduce they are
defined from, so the host logic also runs on CPU ranks.
"""
from __future__ import annotations

import torch
import torch.distributed as dist

# Blob order: conv1.W conv1.b ... conv5.W conv5.b fc6.W fc6.b ... fc8.b; the
# FC layers' parameters are the blob's tail from this index on (grouped
# network: 60,965,224 parameters, of which 58,631,144 are FC).
FC_PARAMS = 9216 * 4096 + 4096 + 4096 * 4096 + 4096 + 4096 * 1000 + 1000


class _Bucket:
    """A contiguous range [start, start + length) of the blob, split into
    `world` equal slices (the last one padded when length % world != 0)."""

    def __init__(self, start, length, world, rank, device):
        self.start, self.length = start, length
        self.slice = -(-length // world)
        self.world, self.rank = world, rank
        self.padded = self.slice * world != length
        self.mine = (rank * self.slice, min(length, (rank + 1) * self.slice))
        self.recv = torch.empty(self.slice, dtype=torch.float32, device=device)
        if self.padded:
            self.stage = torch.zeros(self.slice * world, dtype=torch.float32, device=device)

    def reduce_scatter(self, grads, group):
        """recv <- this rank's slice of the sum over ranks of grads[range]."""
        src = grads[self.start:self.start + self.length]
        if self.padded:
            self.stage[:self.length].copy_(src)
            src = self.stage
        if _has_reduce_scatter(group):
            dist.reduce_scatter_tensor(self.recv, src, op=dist.ReduceOp.SUM, group=group)
        else:
            full = src.clone()
            dist.all_reduce(full, op=dist.ReduceOp.SUM, group=group)
            self.recv.copy_(full[self.rank * self.slice:(self.rank + 1) * self.slice])

    def all_gather(self, params, group):
        """params[range] <- every rank's updated slice."""
        dst = params[self.start:self.start + self.length]
        if not self.padded and _has_reduce_scatter(group):
            # in place: this rank's input is its own slice of the output
            mine = dst[self.rank * self.slice:(self.rank + 1) * self.slice]
            dist.all_gather_into_tensor(dst, mine, group=group)
            return
        a, b = self.mine
        out = [torch.empty(self.slice, dtype=params.dtype, device=params.device)
               for _ in range(self.world)]
        mine = torch.zeros(self.slice, dtype=params.dtype, device=params.device)
        mine[:b - a].copy_(dst[a:b])
        dist.all_gather(out, mine, group=group)
        dst.copy_(torch.cat(out)[:self.length])


def _has_reduce_scatter(group):
    return dist.get_backend(group) == "nccl"


class DataParallelStep:
    """One data-parallel training step per call (see the module docstring)."""

    def __init__(self, engine, group=None, fc_start=None):
        self.engine = engine
        self.group = group
        self.world = dist.get_world_size(group)
        self.rank = dist.get_rank(group)
        params = engine.device_buffer(0)
        self.params = params
        self.grads = engine.device_buffer(2)
        n = params.numel()
        fc_start = n - FC_PARAMS if fc_start is None else fc_start
        dev = params.device
        # the FC bucket first: its gradients are complete first
        self.buckets = [_Bucket(fc_start, n - fc_start, self.world, self.rank, dev),
                        _Bucket(0, fc_start, self.world, self.rank, dev)]
        self.comm = torch.cuda.Stream() if dev.type == "cuda" else None

    def step(self, x, labels, B, lr, loss=None):
        """x, labels: this rank's B images (every rank the same B); they are
        images rank * B .. rank * B + B - 1 of the whole batch."""
        e = self.engine
        e.train_grads(x, labels, B, self.rank * B, loss)
        fc, conv = self.buckets
        if self.comm is not None:
            main = torch.cuda.current_stream()
            e.stream_wait_fc_grads(self.comm)
            with torch.cuda.stream(self.comm):
                fc.reduce_scatter(self.grads, self.group)
            conv.reduce_scatter(self.grads, self.group)
            main.wait_stream(self.comm)
        else:
            fc.reduce_scatter(self.grads, self.group)
            conv.reduce_scatter(self.grads, self.group)
        scale = 1.0 / self.world
        for bk in self.buckets:
            a, b = bk.mine
            if b > a:
                e.sgd_range(bk.start + a, b - a, bk.recv[:b - a], scale, lr)
        for bk in self.buckets:
            bk.all_gather(self.params, self.group)
        e.params_updated()
