"""The allocation-free weight-gradient entry point
(alexnet_op_conv_wgrad_noalloc) against the scratch-taking one.

Callers that can neither hand the library scratch memory nor let it allocate
use the no-allocation variant; it must give the same gradients.  Two calls in
a row (different shapes, then the first shape again with new data) check that
the shared array's leftover contents never leak into a result.  This file is
collected last so that a run stopping at the first failure has already run
every other test."""
import ctypes

import numpy as np
import pytest

from tests._gpu import bf16_round, dev, host, rel_l2, workspace

pytestmark = pytest.mark.gpu

TOL_F32_ACC = 1e-3  # the bound of the other fp32 weight-gradient tests


def _call_noalloc(lib, x, B, H, Cin, dy, Cout, K, pad, groups, splits, dw):
    import torch
    fn = lib.alexnet_op_conv_wgrad_noalloc
    fn.restype = ctypes.c_int
    fn.argtypes = [ctypes.c_void_p, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                   ctypes.c_void_p, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                   ctypes.c_int, ctypes.c_void_p, ctypes.c_void_p]
    return fn(x.data_ptr(), B, H, H, Cin, dy.data_ptr(), Cout, K, pad, groups, splits,
              dw.data_ptr(), torch.cuda.current_stream().cuda_stream)


@pytest.mark.parametrize("order", [0, 1])
def test_noalloc_weight_gradient_matches_scratch_version(order):
    import torch
    from deep_cnn_image_b200 import alexnet as ax
    ws = workspace(512)
    shapes = [(13, 384, 256, 3, 1, 2, 4, 0, 11),   # conv5 shape
              (27, 96, 256, 5, 2, 2, 2, 0, 12),    # conv2 shape
              (13, 384, 256, 3, 1, 2, 4, 3, 13),   # conv5 again, new data, 3 splits
              # conv2 shape asking for 16 K-slices: 23 K blocks, but only 10
              # slices of partial sums fit in the array, so the call lowers
              # the count and the summing kernel sees the lowered one
              (27, 96, 256, 5, 2, 2, 2, 16, 14)]
    if order:
        shapes = shapes[::-1]
    for (H, Cin, Cout, K, pad, groups, B, splits, seed) in shapes:
        r = np.random.default_rng(seed)
        x = bf16_round(np.maximum(r.standard_normal((B, H, H, Cin)), 0.0))
        dy = bf16_round(r.standard_normal((B, H + 2 * pad - K + 1, H + 2 * pad - K + 1, Cout)))
        xt, dyt = dev(x, "bf16"), dev(dy, "bf16")
        shape = (Cout, K, K, Cin // groups)
        want = torch.empty(shape, dtype=torch.float32, device="cuda")
        ax.op_conv_wgrad(xt, B, H, H, Cin, dyt, Cout, K, pad, groups, splits, want, ws)
        got = torch.full(shape, float("nan"), dtype=torch.float32, device="cuda")
        st = _call_noalloc(ax.lib, xt, B, H, Cin, dyt, Cout, K, pad, groups, splits, got)
        assert st == ax.OK
        assert rel_l2(host(got), host(want)) < TOL_F32_ACC


def test_noalloc_weight_gradient_matches_oracle():
    """The allocation-free call runs the im2col GEMM, which the scratch-taking
    call may not: one small grouped shape against the oracle's fp64 weight
    gradient, within the fp32-accumulation bound of the other weight-gradient
    tests (two calls, so the second one finds the first one's leftovers)."""
    import torch
    import oracle
    from deep_cnn_image_b200 import alexnet as ax
    H, Cin, Cout, K, pad, groups, B = 13, 128, 64, 3, 1, 2, 3
    for seed in (21, 22):
        r = np.random.default_rng(seed)
        x = bf16_round(np.maximum(r.standard_normal((B, H, H, Cin)), 0.0))
        dy = bf16_round(r.standard_normal((B, H, H, Cout)))
        got = torch.full((Cout, K, K, Cin // groups), float("nan"), dtype=torch.float32,
                         device="cuda")
        st = _call_noalloc(ax.lib, dev(x, "bf16"), B, H, Cin, dev(dy, "bf16"), Cout, K, pad,
                           groups, 0, got)
        assert st == ax.OK
        _, want, _ = oracle.conv_bwd(x, np.zeros((Cout, K, K, Cin // groups)), dy, 1, pad, groups,
                                     need_dx=False)
        assert rel_l2(host(got), want) < TOL_F32_ACC


def test_noalloc_rejects_sizes_beyond_the_array():
    import torch
    from deep_cnn_image_b200 import alexnet as ax
    # one K-slice of a 1024 -> 2048 3x3 convolution is 75 MB of partial sums
    x = torch.zeros((1, 3, 3, 1024), dtype=torch.bfloat16, device="cuda")
    dy = torch.zeros((1, 3, 3, 2048), dtype=torch.bfloat16, device="cuda")
    dw = torch.zeros((2048, 3, 3, 1024), dtype=torch.float32, device="cuda")
    st = _call_noalloc(ax.lib, x, 1, 3, 1024, dy, 2048, 3, 1, 1, 0, dw)
    assert st == ax.ERR_UNSUPPORTED
