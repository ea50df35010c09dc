"""Bounds evidence without a sanitiser: guard regions around what the kernels
write.

  * Inside the workspace, every buffer the handle carves is followed by a
    256-byte guard (filled at create; alexnet_debug_canaries counts the bytes
    that changed).  A full training step at the benchmark's batch (and the
    other network calls, and the ablation variants) must leave all of them
    intact.
  * Past the end of the workspace, and past the end of every output of the
    single-op entry points, the tests place their own guard (1 MiB, resp.
    64 KiB of the byte 0x5A) and check it afterwards.

A kernel that wrote out of bounds would change a guard; none of these checks
needs a fault to see it, and none can cause one (the guards are ordinary
memory inside the tensors the tests allocate)."""
import ctypes

import numpy as np
import pytest

from deep_cnn_image_b200 import synthetic
from tests._gpu import dev, workspace

pytestmark = pytest.mark.gpu

GUARD = 0x5A


@pytest.fixture(scope="module")
def ax():
    from deep_cnn_image_b200 import alexnet
    return alexnet


class Guarded:
    """A device tensor followed by a guard of `tail` bytes of 0x5A."""

    def __init__(self, n, dtype, tail=64 << 10):
        import torch
        esz = torch.empty((), dtype=dtype).element_size()
        self.nbytes = n * esz
        self.buf = torch.empty(self.nbytes + tail, dtype=torch.uint8, device="cuda")
        self.buf.fill_(GUARD)
        self.t = self.buf[:self.nbytes].view(dtype)
        self.tail = tail

    def intact(self):
        import torch
        torch.cuda.synchronize()
        return bool(torch.all(self.buf[self.nbytes:] == GUARD).item())


def _step_inputs(B, seed=3):
    import torch
    xt, _ = synthetic.to_bf16(synthetic.images(seed, B))
    y = synthetic.labels(seed + 1, B)
    return xt.cuda(), torch.from_numpy(y).cuda()


def test_full_batch_step_keeps_every_workspace_guard(ax):
    """Batch 128, default options: training steps, both forward modes, the
    parameter accessors; then the guards after every workspace buffer and a
    1 MiB guard past the workspace's end are checked."""
    import torch
    cfg = ax.default_config(batch_max=128, keep_grads=1)
    nbytes = ax.workspace_bytes(cfg)
    tail = 1 << 20
    ws = torch.empty(nbytes + 256 + tail, dtype=torch.uint8, device="cuda")
    base = (ws.data_ptr() + 255) & ~255
    off = base - ws.data_ptr()
    ws[off + nbytes:].fill_(GUARD)
    h = ctypes.c_void_p()
    ax.check(ax.lib.alexnet_create(ctypes.byref(cfg), base, nbytes, None, ctypes.byref(h)))
    try:
        x, y = _step_inputs(128)
        loss = torch.zeros(1, dtype=torch.float32, device="cuda")
        for _ in range(2):
            ax.check(ax.lib.alexnet_train_step(h, x.data_ptr(), y.data_ptr(), 128, 0.01,
                                               loss.data_ptr(), None), h)
        logits = torch.empty((128, 1000), dtype=torch.float32, device="cuda")
        probs = torch.empty_like(logits)
        for mode in (ax.TRAIN, ax.INFERENCE):
            ax.check(ax.lib.alexnet_forward(h, x.data_ptr(), 128, mode, logits.data_ptr(),
                                            probs.data_ptr(), None), h)
        # a smaller batch on the same handle (its own plan and graph)
        ax.check(ax.lib.alexnet_train_step(h, x.data_ptr(), y.data_ptr(), 37, 0.01,
                                           loss.data_ptr(), None), h)
        assert ax.lib.alexnet_get_status(h) == ax.OK
        bad = ctypes.c_int64(-1)
        ax.check(ax.lib.alexnet_debug_canaries(h, ctypes.byref(bad)), h)
        assert bad.value == 0
        torch.cuda.synchronize()
        assert bool(torch.all(ws[off + nbytes:] == GUARD).item())
    finally:
        ax.lib.alexnet_destroy(h)


@pytest.mark.parametrize("opts", [dict(keep_grads=1), dict(pool_size=2), dict(lrn_on=0),
                                  dict(grouped=0), dict(dropout_on=0)])
def test_variant_steps_keep_every_workspace_guard(ax, opts):
    """Small odd batches through the other code paths: the debug stores
    (normalised maps), the separate FC update kernel, the ablations."""
    import torch
    net = ax.AlexNet(batch_max=5, seed=11, **opts)
    net.debug_keep(True)
    x, y = _step_inputs(5, 21)
    for fused in (True, False):
        net.debug_fc_update(fused)
        net.train_step(x, y, 5, 0.01)
        net.train_step(x, y, 3, 0.01)
    logits = torch.empty((5, 1000), dtype=torch.float32, device="cuda")
    net.forward(x, 5, ax.INFERENCE, logits)
    assert net.get_status() == ax.OK
    assert net.debug_canaries() == 0
    net.close()


def test_single_op_outputs_keep_their_guards(ax):
    """Every single-op entry point at the network's layer shapes (batch 2,
    plus an odd one), each output followed by a 64 KiB guard."""
    import torch
    ws = workspace(512)
    r = np.random.default_rng(5)
    B = 2

    def rnd(*shape, relu=False):
        a = r.standard_normal(shape)
        return dev(np.maximum(a, 0) if relu else a, "bf16")

    checks = []

    def out(n, dtype=torch.bfloat16):
        g = Guarded(n, dtype)
        checks.append(g)
        return g.t

    # convolutions (conv2..conv5 shapes), conv1, data and weight gradients
    for (H, Cin, Cout, K, pad, groups) in ((27, 96, 256, 5, 2, 2), (13, 256, 384, 3, 1, 1),
                                           (13, 384, 384, 3, 1, 2), (13, 384, 256, 3, 1, 2)):
        x = rnd(B, H, H, Cin, relu=True)
        w = rnd(Cout, K, K, Cin // groups) * 0.05
        bias = torch.zeros(Cout, dtype=torch.float32, device="cuda")
        y = out(B * H * H * Cout)
        ax.op_conv_fwd(x, B, H, H, Cin, w, bias, Cout, K, pad, groups, 1, y, ws)
        dy = rnd(B, H, H, Cout)
        dx = out(B * H * H * Cin)
        ax.op_conv_dgrad(dy, B, H, H, Cin, w, Cout, K, pad, groups, x, dx, ws)
        dw = out(Cout * K * K * (Cin // groups), torch.float32)
        ax.op_conv_wgrad(x, B, H, H, Cin, dy, Cout, K, pad, groups, 0, dw, ws)
        dw2 = out(Cout * K * K * (Cin // groups), torch.float32)
        ax.op_conv_wgrad_noalloc(x, B, H, H, Cin, dy, Cout, K, pad, groups, 0, dw2)
    x1 = rnd(B, 227, 227, 3)
    w1 = rnd(96, 11, 11, 3) * 0.05
    b1 = torch.zeros(96, dtype=torch.float32, device="cuda")
    y1 = out(B * 55 * 55 * 96)
    ax.op_conv1_fwd(x1, B, w1, b1, y1, ws)
    dw1 = out(96 * 11 * 11 * 3, torch.float32)
    ax.op_conv1_wgrad(x1, B, rnd(B, 55, 55, 96), 0, dw1, ws)
    # FC products at FC6's shape, an odd batch
    Bf = 3
    xf = rnd(Bf, 9216)
    wf = rnd(4096, 9216) * 0.01
    yf = out(Bf * 4096, torch.float32)
    ax.op_fc_fwd(xf, Bf, 9216, wf, 4096, 0, yf, ws)
    dzf = rnd(Bf, 4096)
    dxf = out(Bf * 9216, torch.float32)
    ax.op_fc_dgrad(dzf, Bf, 4096, wf, 9216, 0, dxf, ws)
    dwf = out(4096 * 9216, torch.float32)
    ax.op_fc_wgrad(dzf, xf, Bf, 4096, 9216, dwf, ws)
    # normalisation, pooling and their fused forms (conv1 / conv2 maps)
    for (H, C) in ((55, 96), (27, 256)):
        a = rnd(B, H, H, C, relu=True)
        P = (H - 3) // 2 + 1
        b = out(B * H * H * C)
        ax.op_lrn_fwd(a, B * H * H, C, 2.0, 1e-4, 0.75, b)
        da = out(B * H * H * C)
        ax.op_lrn_bwd(a, rnd(B, H, H, C), B * H * H, C, 2.0, 1e-4, 0.75, da)
        yp = out(B * P * P * C)
        am = out(B * P * P * C, torch.uint8)
        ax.op_pool_fwd(a, B, H, H, C, 3, 2, yp, am)
        dxp = out(B * H * H * C)
        ax.op_pool_bwd(rnd(B, P, P, C), am, yp, B, H, H, C, 3, 2, 1, dxp)
        lo = out(B * H * H * C)
        yl = out(B * P * P * C)
        aml = out(B * P * P * C, torch.uint8)
        ax.op_lrn_pool_fwd(a, B, H, H, C, 3, 2.0, 1e-4, 0.75, lo, yl, aml)
        dl = out(B * H * H * C)
        dal = out(B * H * H * C)
        ax.op_pool_lrn_bwd(rnd(B, P, P, C), aml, a, B, H, H, C, 3, 2.0, 1e-4, 0.75, dl, dal)
    # softmax + cross-entropy, dropout mask
    logits = torch.randn((5, 1000), dtype=torch.float32, device="cuda")
    labels = torch.arange(5, dtype=torch.int32, device="cuda")
    probs = out(5 * 1000, torch.float32)
    dlog = out(5 * 1000)
    loss = out(1, torch.float32)
    ax.op_softmax_ce(logits, labels, 5, 1000, probs, dlog, loss, ws)
    keep = out(7 * 4096, torch.uint8)
    ax.op_dropout_mask(5, 6, 1, 0.5, 7, 4096, keep, ws)
    torch.cuda.synchronize()
    bad = [i for i, g in enumerate(checks) if not g.intact()]
    assert not bad, bad
