"""Per-operation parity: each CUDA kernel of the hot path, called through the
C ABI, against the CPU oracle fed the very same (bf16-rounded) inputs.

Tolerances: integer and index results (pool argmax, dropout masks, Philox
words) bit-exact; bf16 outputs of one op within rel-L2 1e-2 (their only
error is the final bf16 rounding, about 2^-9 per element); fp32 outputs
(weight gradients, FC products) within rel-L2 1e-3 (fp32 accumulation of
exact bf16 products)."""
import zlib

import numpy as np
import pytest

import oracle
from tests._gpu import TOL_OP, bf16_round, dev, host, rel_l2, workspace

pytestmark = pytest.mark.gpu

TOL_F32_ACC = 1e-3


@pytest.fixture(scope="module")
def ax():
    from deep_cnn_image_b200 import alexnet
    return alexnet


@pytest.fixture(scope="module")
def ws():
    return workspace(1024)


def _rng(seed):
    return np.random.default_rng(seed)


# ------------------------------------------------------------------ Philox / dropout
def test_philox_known_answers_on_device(ax):
    import torch
    kat = [([0, 0, 0, 0], [0, 0], [0x6627e8d5, 0xe169c58d, 0xbc57ac4c, 0x9b00dbd8]),
           ([0xffffffff] * 4, [0xffffffff] * 2, [0x408f276d, 0x41c83b0e, 0xa20bc7c6, 0x6d5451fd]),
           ([0x243f6a88, 0x85a308d3, 0x13198a2e, 0x03707344], [0xa4093822, 0x299f31d0],
            [0xd16cfe09, 0x94fdcceb, 0x5001e420, 0x24126ea1])]
    r = _rng(1)
    rand = [(list(r.integers(0, 2**32, 4)), list(r.integers(0, 2**32, 2))) for _ in range(61)]
    cases = [(c, k) for c, k, _ in kat] + rand
    ctr = np.array([c for c, _ in cases], dtype=np.uint32).ravel()
    key = np.array([k for _, k in cases], dtype=np.uint32).ravel()
    out = torch.zeros(4 * len(cases), dtype=torch.int32, device="cuda")
    ax.op_philox(dev(ctr.view(np.int32)), dev(key.view(np.int32)), len(cases), out)
    got = host(out).view(np.uint32).reshape(-1, 4)
    for i, (c, k) in enumerate(cases):
        assert list(got[i]) == oracle.philox4x32_10(c, k)
    for i, (_, _, want) in enumerate(kat):
        assert list(got[i]) == want


@pytest.mark.parametrize("layer,step,seed", [(6, 0, 0x5EED), (7, 3, 12345), (6, 77, 2**40 + 9)])
def test_dropout_mask_bit_exact(ax, ws, layer, step, seed):
    import torch
    keep = torch.zeros(128 * 4096, dtype=torch.uint8, device="cuda")
    ax.op_dropout_mask(seed, layer, step, 0.5, 128, 4096, keep, ws)
    got = host(keep).reshape(128, 4096)
    want = oracle.dropout_mask(seed, layer, step, 128, 4096)
    np.testing.assert_array_equal(got, want)


# ------------------------------------------------------------------ LRN
@pytest.mark.parametrize("C", [96, 256])
def test_lrn_forward_backward(ax, C):
    import torch
    r = _rng(C)
    P = 2 * 27 * 27 + 5
    a = bf16_round(np.maximum(r.standard_normal((P, C)) * 20.0, 0.0))
    g = bf16_round(r.standard_normal((P, C)))
    da_ = dev(a, "bf16")
    b = torch.empty_like(da_)
    ax.op_lrn_fwd(da_, P, C, 2.0, 1e-4, 0.75, b)
    want = oracle.lrn_fwd(a)
    assert rel_l2(host(b), want) < 4e-3
    dgrad = torch.empty_like(da_)
    ax.op_lrn_bwd(da_, dev(g, "bf16"), P, C, 2.0, 1e-4, 0.75, dgrad)
    want_d = oracle.lrn_bwd(a, g) * (a > 0)
    assert rel_l2(host(dgrad), want_d) < 4e-3


# ------------------------------------------------------------------ pooling
@pytest.mark.parametrize("shape,z", [((3, 55, 55, 96), 3), ((2, 27, 27, 256), 3),
                                     ((2, 13, 13, 256), 3), ((2, 55, 55, 96), 2)])
def test_pool_forward_bit_exact_with_ties(ax, shape, z):
    import torch
    r = _rng(sum(shape) + z)
    x = r.standard_normal(shape)
    x[0] = np.round(x[0] * 2) / 2  # image 0 on a coarse grid: many exact ties
    x = bf16_round(x)
    B, H, W, C = shape
    Ho = (H - z) // 2 + 1
    y = torch.empty((B, Ho, Ho, C), dtype=torch.bfloat16, device="cuda")
    am = torch.empty((B, Ho, Ho, C), dtype=torch.uint8, device="cuda")
    ax.op_pool_fwd(dev(x, "bf16"), B, H, W, C, z, 2, y, am)
    wy, wam = oracle.maxpool_fwd(x, z, 2)
    np.testing.assert_array_equal(host(am), wam)
    np.testing.assert_array_equal(host(y), wy)


@pytest.mark.parametrize("relu_mask", [0, 1])
def test_pool_backward(ax, relu_mask):
    import torch
    r = _rng(5 + relu_mask)
    B, H, C = 2, 13, 256
    x = bf16_round(np.maximum(r.standard_normal((B, H, H, C)), 0.0) if relu_mask
                   else r.standard_normal((B, H, H, C)))
    wy, wam = oracle.maxpool_fwd(x)
    g = bf16_round(r.standard_normal(wy.shape))
    dx = torch.empty((B, H, H, C), dtype=torch.bfloat16, device="cuda")
    ax.op_pool_bwd(dev(g, "bf16"), dev(wam), dev(wy, "bf16"), B, H, H, C, 3, 2, relu_mask, dx)
    gm = g * (wy > 0) if relu_mask else g
    want = oracle.maxpool_bwd(gm, wam, H, H)
    assert rel_l2(host(dx), want) < 4e-3


# ------------------------------------------------------------------ normalisation + pooling, fused
FUSED_SHAPES = [((3, 55, 55, 96), 3), ((2, 27, 27, 256), 3), ((2, 13, 13, 64), 3),
                ((2, 55, 55, 96), 2), ((1, 20, 17, 32), 3), ((1, 18, 18, 32), 3), ((1, 9, 9, 32), 2),
                # many channels: four pixels per block in the backward
                ((1, 40, 40, 512), 3)]


def _lrn_input(seed, shape):
    r = _rng(seed)
    a = np.maximum(r.standard_normal(shape) * 20.0, 0.0)
    # image 0 has one channel vector at every pixel: every window is a tie
    a[0] = a[0, :1, :1, :]
    return bf16_round(a)


@pytest.mark.parametrize("shape,z", FUSED_SHAPES)
def test_lrn_pool_forward_fused(ax, shape, z):
    """Bit-identical to the separate normalisation and pooling kernels; the
    normalised map within the bf16 bound of the oracle's; the window choices
    the oracle's first maxima of that map, bit-exact."""
    import torch
    B, H, W, C = shape
    a = _lrn_input(sum(shape) + z, shape)
    Ho, Wo = (H - z) // 2 + 1, (W - z) // 2 + 1
    da_ = dev(a, "bf16")
    lo = torch.empty_like(da_)
    y = torch.empty((B, Ho, Wo, C), dtype=torch.bfloat16, device="cuda")
    am = torch.empty((B, Ho, Wo, C), dtype=torch.uint8, device="cuda")
    ax.op_lrn_pool_fwd(da_, B, H, W, C, z, 2.0, 1e-4, 0.75, lo, y, am)
    lo_ref = torch.empty_like(da_)
    ax.op_lrn_fwd(da_, B * H * W, C, 2.0, 1e-4, 0.75, lo_ref)
    y_ref = torch.empty_like(y)
    am_ref = torch.empty_like(am)
    ax.op_pool_fwd(lo_ref, B, H, W, C, z, 2, y_ref, am_ref)
    torch.cuda.synchronize()
    assert torch.equal(lo.view(torch.int16), lo_ref.view(torch.int16))
    assert torch.equal(y.view(torch.int16), y_ref.view(torch.int16))
    assert torch.equal(am, am_ref)
    glo = host(lo)
    assert rel_l2(glo, oracle.lrn_fwd(a)) < 4e-3
    wy, wam = oracle.maxpool_fwd(glo, z, 2)
    np.testing.assert_array_equal(host(am), wam)
    np.testing.assert_array_equal(host(y), wy)
    assert np.all(host(am)[0] == 0)
    # without the normalised map: same pooled output
    y2 = torch.empty_like(y)
    am2 = torch.empty_like(am)
    ax.op_lrn_pool_fwd(da_, B, H, W, C, z, 2.0, 1e-4, 0.75, None, y2, am2)
    torch.cuda.synchronize()
    assert torch.equal(y2.view(torch.int16), y.view(torch.int16)) and torch.equal(am2, am)


@pytest.mark.parametrize("shape,z", FUSED_SHAPES)
def test_pool_lrn_backward_fused(ax, shape, z):
    """da = ReLU'(a) * LRN-backward(a, pool-backward(dy)) against the oracle
    on the GPU's own window choices; dl = the pool backward alone."""
    import torch
    B, H, W, C = shape
    a = _lrn_input(sum(shape) + 7 * z, shape)
    Ho, Wo = (H - z) // 2 + 1, (W - z) // 2 + 1
    da_ = dev(a, "bf16")
    y = torch.empty((B, Ho, Wo, C), dtype=torch.bfloat16, device="cuda")
    am = torch.empty((B, Ho, Wo, C), dtype=torch.uint8, device="cuda")
    ax.op_lrn_pool_fwd(da_, B, H, W, C, z, 2.0, 1e-4, 0.75, None, y, am)
    g = bf16_round(_rng(sum(shape)).standard_normal((B, Ho, Wo, C)))
    dl = torch.empty_like(da_)
    dout = torch.empty_like(da_)
    ax.op_pool_lrn_bwd(dev(g, "bf16"), am, da_, B, H, W, C, z, 2.0, 1e-4, 0.75, dl, dout)
    gam = host(am)
    want_dl = oracle.maxpool_bwd(g, gam, H, W, z, 2)
    assert rel_l2(host(dl), want_dl) < 4e-3
    want = oracle.lrn_bwd(a, want_dl) * (a > 0)
    assert rel_l2(host(dout), want) < 4e-3
    d2 = torch.empty_like(da_)
    ax.op_pool_lrn_bwd(dev(g, "bf16"), am, da_, B, H, W, C, z, 2.0, 1e-4, 0.75, None, d2)
    torch.cuda.synchronize()
    assert torch.equal(d2.view(torch.int16), dout.view(torch.int16))


def test_fused_pool_rejects_bad_shapes(ax):
    import torch
    t = torch.zeros(4 * 9 * 9 * 48, dtype=torch.bfloat16, device="cuda")
    am = torch.zeros(4 * 4 * 4 * 48, dtype=torch.uint8, device="cuda")
    with pytest.raises(Exception):
        ax.op_lrn_pool_fwd(t, 4, 9, 9, 48, 3, 2.0, 1e-4, 0.75, None, t, am)  # C % 32
    with pytest.raises(Exception):
        ax.op_pool_lrn_bwd(t, am, t, 1, 9, 9, 32, 4, 2.0, 1e-4, 0.75, None, t)  # z = 4


# ------------------------------------------------------------------ nearest neighbours
@pytest.mark.parametrize("Q,N,D,k", [(8, 1000, 4096, 10), (3, 136, 64, 1), (130, 520, 128, 32)])
def test_knn_matches_oracle(ax, Q, N, D, k):
    """Squared distances within the fp32 bound of the oracle's direct fp64
    sums; neighbour indices equal wherever the oracle's ranking is separated
    by more than that bound; a planted duplicate of query 0 is its nearest."""
    import torch
    r = _rng(Q * 7 + N)
    base = bf16_round(np.maximum(r.standard_normal((N, D)), 0.0))  # ReLU-like features
    q = bf16_round(np.maximum(r.standard_normal((Q, D)), 0.0))
    base[N // 3] = q[0]
    dist = torch.empty((Q, k), dtype=torch.float32, device="cuda")
    idx = torch.empty((Q, k), dtype=torch.int32, device="cuda")
    ws = torch.empty(ax.knn_workspace_bytes(Q, N), dtype=torch.uint8, device="cuda")
    ax.knn(dev(q, "bf16"), dev(base, "bf16"), k, dist, idx, ws)
    torch.cuda.synchronize()
    wd, wi = oracle.knn(q, base, k)
    gd, gi = host(dist), host(idx)
    # fp32 accumulation of D products of size ~1 and the norm expansion
    tol = 1e-5 * (np.sum(q * q, axis=1).max() + np.sum(base * base, axis=1).max())
    assert np.abs(gd - wd).max() <= tol
    assert gi[0, 0] == N // 3 and gd[0, 0] <= tol
    # with the base norms precomputed: identical results
    bn = torch.empty(N, dtype=torch.float32, device="cuda")
    ax.knn_sqnorms(dev(base, "bf16"), bn)
    d2 = torch.empty_like(dist)
    i2 = torch.empty_like(idx)
    ax.knn(dev(q, "bf16"), dev(base, "bf16"), k, d2, i2, ws, base_sqnorm=bn)
    torch.cuda.synchronize()
    assert torch.equal(d2, dist) and torch.equal(i2, idx)
    np.testing.assert_allclose(host(bn), np.sum(base * base, axis=1), rtol=1e-5)
    full, _ = oracle.knn(q, base, min(N, k + 1))
    for i in range(Q):
        for j in range(k):
            gap_lo = full[i, j] - full[i, j - 1] if j > 0 else np.inf
            gap_hi = full[i, j + 1] - full[i, j] if j + 1 < full.shape[1] else np.inf
            if min(gap_lo, gap_hi) > 2 * tol:
                assert gi[i, j] == wi[i, j], (i, j)


def test_knn_rejects_bad_arguments(ax):
    import torch
    q = torch.zeros((2, 64), dtype=torch.bfloat16, device="cuda")
    base = torch.zeros((16, 64), dtype=torch.bfloat16, device="cuda")
    dist = torch.empty((2, 40), dtype=torch.float32, device="cuda")
    idx = torch.empty((2, 40), dtype=torch.int32, device="cuda")
    ws = torch.empty(ax.knn_workspace_bytes(2, 16), dtype=torch.uint8, device="cuda")
    with pytest.raises(Exception):
        ax.knn(q, base, 33, dist, idx, ws)  # k above 32
    with pytest.raises(Exception):
        ax.knn(q, base, 17, dist, idx, ws)  # k above N
    with pytest.raises(Exception):
        ax.knn(q, base[:12], 4, dist, idx, ws)  # N not a multiple of 8


# ------------------------------------------------------------------ failure detection
def test_bounded_wait_runs_out_and_reports_timeout(ax, ws):
    """A device wait that nothing completes (the pipelined kernels' bounded
    mbarrier wait, limited to about a millisecond) returns with the TIMEOUT
    bit set instead of hanging, and the context stays usable."""
    import torch
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    ax.op_wait_probe(status, 2_000_000)
    torch.cuda.synchronize()
    assert int(status.item()) & 1 == 1
    # the next launch on the same context still works
    z = torch.zeros((2, 1000), dtype=torch.float32, device="cuda")
    probs = torch.empty_like(z)
    ax.op_softmax_ce(z, None, 2, 1000, probs, None, None, ws)
    torch.cuda.synchronize()
    np.testing.assert_allclose(host(probs), np.full((2, 1000), 1e-3), rtol=1e-6)
    with pytest.raises(Exception):
        ax.op_wait_probe(status, 0)


# ------------------------------------------------------------------ softmax + CE
def test_softmax_cross_entropy(ax, ws):
    import torch
    r = _rng(9)
    B, N = 128, 1000
    z = (r.standard_normal((B, N)) * 3).astype(np.float32)
    y = r.integers(0, N, B).astype(np.int32)
    probs = torch.empty((B, N), dtype=torch.float32, device="cuda")
    dl = torch.empty((B, N), dtype=torch.bfloat16, device="cuda")
    loss = torch.zeros(1, dtype=torch.float32, device="cuda")
    ax.op_softmax_ce(dev(z), dev(y), B, N, probs, dl, loss, ws)
    wl, wp, wd = oracle.softmax_ce(z.astype(np.float64), y)
    assert abs(host(loss)[0] - wl) / wl < 1e-5
    assert rel_l2(host(probs), wp) < 1e-5
    assert rel_l2(host(dl), wd) < 4e-3


# ------------------------------------------------------------------ convolutions
CONVS = [  # (name, H, Cin, Cout, K, pad, groups, B)
    ("conv2", 27, 96, 256, 5, 2, 2, 2),
    ("conv2_ungrouped", 27, 96, 256, 5, 2, 1, 1),
    ("conv3", 13, 256, 384, 3, 1, 1, 3),
    ("conv4", 13, 384, 384, 3, 1, 2, 3),
    ("conv4_ungrouped", 13, 384, 384, 3, 1, 1, 2),
    ("conv5", 13, 384, 256, 3, 1, 2, 3),
    ("conv5_ungrouped", 13, 384, 256, 3, 1, 1, 2),
    ("ragged_5x5", 20, 64, 128, 5, 2, 1, 2),
    # 64 input channels per group and a 3 x 3 kernel: the data gradient's
    # tap pairs with an odd last tap beside the zero slab in every row
    ("pair_3x3", 15, 128, 128, 3, 1, 2, 2),
    ("one_by_one", 9, 32, 64, 1, 0, 1, 2),
    ("wide_im2col_fallback", 258, 64, 64, 3, 1, 1, 1),
]
# 96 output channels per group (conv1's count): N = 96 weight-gradient tiles.
# The data gradient of such a layer is not supported (its input channels per
# group must be a multiple of 64 there) and the network never needs it.
CONVS_FWD_WGRAD = CONVS + [("og96", 15, 64, 96, 3, 1, 1, 2)]


def _conv_inputs(seed, B, H, Cin, Cout, K, groups):
    r = _rng(seed)
    x = bf16_round(np.maximum(r.standard_normal((B, H, H, Cin)), 0.0))
    w = bf16_round(r.standard_normal((Cout, K, K, Cin // groups)) * 0.05)
    b = (r.standard_normal(Cout) * 0.1).astype(np.float32)
    return x, w, b


@pytest.mark.parametrize("name,H,Cin,Cout,K,pad,groups,B", CONVS_FWD_WGRAD)
def test_conv_forward(ax, ws, name, H, Cin, Cout, K, pad, groups, B):
    import torch
    x, w, b = _conv_inputs(zlib.crc32(name.encode()) % 1000, B, H, Cin, Cout, K, groups)
    Ho = H + 2 * pad - K + 1
    y = torch.empty((B, Ho, Ho, Cout), dtype=torch.bfloat16, device="cuda")
    ax.op_conv_fwd(dev(x, "bf16"), B, H, H, Cin, dev(w, "bf16"), dev(b), Cout, K, pad, groups, 1, y,
                   ws)
    want = np.maximum(oracle.conv_fwd(x, w, b.astype(np.float64), 1, pad, groups), 0.0)
    err = rel_l2(host(y), want)
    assert err < TOL_OP, err


def test_conv1_forward(ax, ws):
    import torch
    r = _rng(31)
    B = 3
    x = bf16_round(r.standard_normal((B, 227, 227, 3)))
    w = bf16_round(r.standard_normal((96, 11, 11, 3)) * 0.05)
    b = (r.standard_normal(96) * 0.1).astype(np.float32)
    y = torch.empty((B, 55, 55, 96), dtype=torch.bfloat16, device="cuda")
    ax.op_conv1_fwd(dev(x, "bf16"), B, dev(w, "bf16"), dev(b), y, ws)
    want = np.maximum(oracle.conv_fwd(x, w, b.astype(np.float64), 4, 0, 1), 0.0)
    err = rel_l2(host(y), want)
    assert err < TOL_OP, err


@pytest.mark.parametrize("name,H,Cin,Cout,K,pad,groups,B", CONVS)
@pytest.mark.parametrize("masked", [0, 1])
def test_conv_data_gradient(ax, ws, name, H, Cin, Cout, K, pad, groups, B, masked):
    import torch
    x, w, _ = _conv_inputs(zlib.crc32(name.encode()) % 1000 + 7, B, H, Cin, Cout, K, groups)
    r = _rng(zlib.crc32(name.encode()) % 1000 + 8)
    dy = bf16_round(r.standard_normal((B, H, H, Cout)))
    dx = torch.empty((B, H, H, Cin), dtype=torch.bfloat16, device="cuda")
    mask = dev(x, "bf16") if masked else None
    ax.op_conv_dgrad(dev(dy, "bf16"), B, H, H, Cin, dev(w, "bf16"), Cout, K, pad, groups, mask, dx,
                     ws)
    want, _, _ = oracle.conv_bwd(x, w, dy, 1, pad, groups)
    if masked:
        want = want * (x > 0)
    err = rel_l2(host(dx), want)
    assert err < TOL_OP, err


@pytest.mark.parametrize("name,H,Cin,Cout,K,pad,groups,B", CONVS_FWD_WGRAD)
def test_conv_weight_gradient(ax, ws, name, H, Cin, Cout, K, pad, groups, B):
    import torch
    x, w, _ = _conv_inputs(zlib.crc32(name.encode()) % 1000 + 11, B, H, Cin, Cout, K, groups)
    r = _rng(zlib.crc32(name.encode()) % 1000 + 12)
    dy = bf16_round(r.standard_normal((B, H, H, Cout)))
    _, want, _ = oracle.conv_bwd(x, w, dy, 1, pad, groups, need_dx=False)
    dxt, dyt = dev(x, "bf16"), dev(dy, "bf16")
    results = []
    for splits in (1, 3, 0):
        dw = torch.empty(w.shape, dtype=torch.float32, device="cuda")
        ax.op_conv_wgrad(dxt, B, H, H, Cin, dyt, Cout, K, pad, groups, splits, dw, ws)
        got = host(dw)
        results.append(got)
        err = rel_l2(got, want)
        assert err < TOL_F32_ACC, (splits, err)
    # Both results sum the same exact bf16 products in fp32 on the tensor core:
    # T = terms / 16 + S accumulation steps (16 products each, terms =
    # B * Ho * Wo positions; S <= 16 split partial sums), each rounding the running sum by at most one
    # fp32 unit (2^-23) in either direction; the rounding mode of the tensor
    # core's accumulation is not documented, so the errors may all lean one
    # way and add up linearly: at most T * 2^-23 of the running sums, which
    # for these zero-mean inputs stay within about twice the final one (in
    # L2).  Measured: 1e-7 .. 1e-6 for the box kernels (short chains), 7e-5
    # for the 66,564-position im2col case, against bounds of 7e-6 .. 1e-3.
    terms = B * H * H
    bound = 2.0 * (np.ceil(terms / 16.0) + 16) * 2.0**-23
    split_err = rel_l2(results[1], results[0])
    print("conv wgrad %s: oracle rel-L2 %.3g, split 3 vs 1 rel-L2 %.3g (bound %.3g)" %
          (name, rel_l2(results[0], want), split_err, bound))
    for got in results:
        assert rel_l2(got, want) < bound
    assert split_err < 2.0 * bound


def test_conv1_weight_gradient(ax, ws):
    import torch
    r = _rng(41)
    B = 2
    x = bf16_round(r.standard_normal((B, 227, 227, 3)))
    dy = bf16_round(r.standard_normal((B, 55, 55, 96)))
    w0 = np.zeros((96, 11, 11, 3))
    _, want, _ = oracle.conv_bwd(x, w0, dy, 4, 0, 1, need_dx=False)
    for splits in (0, 5):
        dw = torch.empty((96, 11, 11, 3), dtype=torch.float32, device="cuda")
        ax.op_conv1_wgrad(dev(x, "bf16"), B, dev(dy, "bf16"), splits, dw, ws)
        err = rel_l2(host(dw), want)
        assert err < TOL_F32_ACC, (splits, err)


# ------------------------------------------------------------------ FC
FCS = [(64, 9216, 4096), (128, 4096, 4096), (128, 4096, 1000), (37, 4096, 1000), (5, 9216, 4096)]


@pytest.mark.parametrize("B,In,Out", FCS)
def test_fc_products(ax, ws, B, In, Out):
    import torch
    r = _rng(B + In + Out)
    x = bf16_round(np.maximum(r.standard_normal((B, In)), 0))
    w = bf16_round(r.standard_normal((Out, In)) * 0.01)
    dz = bf16_round(r.standard_normal((B, Out)))
    xt, wt, dzt = dev(x, "bf16"), dev(w, "bf16"), dev(dz, "bf16")
    y = torch.empty((B, Out), dtype=torch.float32, device="cuda")
    ax.op_fc_fwd(xt, B, In, wt, Out, 0, y, ws)
    assert rel_l2(host(y), oracle.fc_fwd(x, w, None)) < TOL_F32_ACC
    dx = torch.empty((B, In), dtype=torch.float32, device="cuda")
    ax.op_fc_dgrad(dzt, B, Out, wt, In, 0, dx, ws)
    dw = torch.empty((Out, In), dtype=torch.float32, device="cuda")
    ax.op_fc_wgrad(dzt, xt, B, Out, In, dw, ws)
    want_dx, want_dw, _ = oracle.fc_bwd(x, w, dz)
    assert rel_l2(host(dx), want_dx) < TOL_F32_ACC
    assert rel_l2(host(dw), want_dw) < TOL_F32_ACC
