"""Pins of the oracle's intermediate-map accessors (forward_probe,
forward_trace, train_probe) on the shrunken network.

The GPU tests compare the library's internal tensors with these accessors, so
a mislabelled code (a gradient taken after the pool backward instead of
before it, say) would otherwise pass unnoticed on both sides.  Each map is
rebuilt here from its neighbours with the single ops (themselves pinned
against torch, brute force and finite differences in test_oracle_pins.py)
by the chain rule of the network's layer order ([S] 3.4 "Overall
Architecture"; [W] the training-step listing), and the bias gradients of the
probes are tied to the step's finite-difference-pinned parameter gradients.
"""
import numpy as np

import oracle

SEED, STEP = 31, 4


def _setup(B=2):
    net = oracle.small_net()
    n = oracle.param_count(net)
    r = np.random.default_rng(5)
    params = r.standard_normal(n) * 0.2
    for (wo, wl, bo, bl) in oracle.param_layout(net):
        params[bo:bo + bl] = r.uniform(0.05, 0.3, bl)
    x = r.standard_normal((B, 67, 67, 3))
    y = np.array([3, 8, 1, 5][:B], np.int32)
    return net, params, x, y


def _w(net, params, l):
    wo, wl, bo, bl = oracle.param_layout(net)[l]
    if l < 5:
        Cin = net.in_c if l == 0 else net.conv_c[l - 1]
        shape = (net.conv_c[l], net.conv_k[l], net.conv_k[l], Cin // net.conv_g[l])
    else:
        In = oracle.map_sizes(net)[4][2] ** 2 * net.conv_c[4] if l == 5 else net.fc_n[l - 6]
        shape = (net.fc_n[l - 5], In)
    return params[wo:wo + wl].reshape(shape), params[bo:bo + bl]


def test_forward_trace_equals_probes_and_preactivations():
    net, params, x, _ = _setup()
    B = x.shape[0]
    codes = [0, 1, 2, 3, 4, 10, 11, 20, 21, 24, 30, 31, 40, 100, 101, 102, 103, 104, 105, 106]
    t = oracle.forward_trace(net, params, x, codes, mode=0, seed=SEED, step=STEP)
    for c in codes:
        if c < 100:
            np.testing.assert_array_equal(
                t[c], oracle.forward_probe(net, params, x, c, mode=0, seed=SEED, step=STEP))
    for l in range(5):
        np.testing.assert_array_equal(np.maximum(t[100 + l], 0.0), t[l])
    # conv1's pre-activation is the single op on the input
    w, b = _w(net, params, 0)
    np.testing.assert_array_equal(t[100], oracle.conv_fwd(x, w, b, 4, 0, 1).ravel())
    # FC6 / FC7: ReLU then the step's dropout mask
    for f in range(2):
        keep = oracle.dropout_mask(SEED, 6 + f, STEP, B, net.fc_n[f]).ravel()
        np.testing.assert_array_equal(np.maximum(t[105 + f], 0.0) * keep, t[30 + f])
    # FC6's pre-activation from the flattened pool5 map
    w6, b6 = _w(net, params, 5)
    np.testing.assert_allclose(t[105].reshape(B, -1), oracle.fc_fwd(t[24].reshape(B, -1), w6, b6),
                               rtol=0, atol=1e-13)


def test_train_probes_follow_the_chain_rule():
    net, params, x, y = _setup()
    B = x.shape[0]
    ms = oracle.map_sizes(net)
    fw = oracle.forward_trace(net, params, x, [0, 1, 2, 3, 4, 10, 11, 20, 21, 24, 30, 31, 40,
                                               105, 106], mode=0, seed=SEED, step=STEP)
    g = {w: oracle.train_probe(net, params, x, y, w, seed=SEED, step=STEP)
         for w in (80, 81, 82, 50, 51, 52, 53, 54, 60, 61, 64, 70, 71)}
    # 80: the mean cross-entropy's gradient of the forward's logits
    _, _, dlog = oracle.softmax_ce(fw[40].reshape(B, -1), y)
    np.testing.assert_allclose(g[80].reshape(B, -1), dlog, rtol=0, atol=1e-15)
    # 81, 82: back through FC8 / FC7, the dropout mask and the ReLU
    keep = [oracle.dropout_mask(SEED, 6 + f, STEP, B, net.fc_n[f]) for f in range(2)]
    w8, _ = _w(net, params, 7)
    dz7 = (dlog @ w8) * keep[1] * (fw[106].reshape(B, -1) > 0)
    np.testing.assert_allclose(g[81].reshape(B, -1), dz7, rtol=1e-12, atol=1e-15)
    w7, _ = _w(net, params, 6)
    dz6 = (dz7 @ w7) * keep[0] * (fw[105].reshape(B, -1) > 0)
    np.testing.assert_allclose(g[82].reshape(B, -1), dz6, rtol=1e-12, atol=1e-15)
    # 64: the gradient of the pooled conv5 map, i.e. of FC6's input
    w6, _ = _w(net, params, 5)
    np.testing.assert_allclose(g[64].reshape(B, -1), dz6 @ w6, rtol=1e-12, atol=1e-15)
    # 54: through pool5 (the forward's own window choices) and conv5's ReLU
    side5 = ms[4][1]
    a5 = fw[4].reshape(B, side5, side5, -1)
    _, am5 = oracle.maxpool_fwd(a5)
    d54 = oracle.maxpool_bwd(g[64].reshape(am5.shape), am5, side5, side5) * (a5 > 0)
    np.testing.assert_allclose(g[54], d54.ravel(), rtol=1e-12, atol=1e-15)
    # 70+l, 50+l (conv1, conv2): pool backward, then the normalisation's
    # backward and the ReLU
    for l in (0, 1):
        side = ms[l][1]
        a = fw[l].reshape(B, side, side, -1)
        lo = fw[10 + l].reshape(a.shape)
        _, am = oracle.maxpool_fwd(lo)
        dl = oracle.maxpool_bwd(g[60 + l].reshape(am.shape), am, side, side)
        np.testing.assert_allclose(g[70 + l], dl.ravel(), rtol=1e-12, atol=1e-15)
        da = oracle.lrn_bwd(a, dl) * (a > 0)
        np.testing.assert_allclose(g[50 + l], da.ravel(), rtol=1e-12, atol=1e-15)
    # 60 (pooled conv1 map) and 61 (pooled conv2 map) are the data gradients
    # of conv2 and conv3; 52, 53 come from conv4's and conv5's data gradients
    # through the ReLU of conv3 and conv4
    inputs = {1: fw[20], 2: fw[21], 3: fw[2], 4: fw[3]}
    for l in (1, 2, 3, 4):
        side_in = ms[l][0]
        xin = inputs[l].reshape(B, side_in, side_in, -1)
        w, _ = _w(net, params, l)
        dz = g[50 + l].reshape(B, ms[l][1], ms[l][1], -1)
        dx, _, _ = oracle.conv_bwd(xin, w, dz, net.conv_s[l], net.conv_p[l], net.conv_g[l])
        if l <= 2:
            np.testing.assert_allclose(g[60 + l - 1], dx.ravel(), rtol=1e-12, atol=1e-15)
        else:
            np.testing.assert_allclose(g[50 + l - 1], (dx * (xin > 0)).ravel(), rtol=1e-12,
                                       atol=1e-15)
    # the bias gradients of the step (pinned by finite differences) are the
    # column sums of the pre-activation gradients
    _, _, _, grads, _ = oracle.train_step(net, params, np.zeros_like(params), x, y, lr=0.0,
                                          seed=SEED, step=STEP)
    lay = oracle.param_layout(net)
    for l in range(5):
        bo, bl = lay[l][2], lay[l][3]
        np.testing.assert_allclose(g[50 + l].reshape(-1, bl).sum(0), grads[bo:bo + bl],
                                   rtol=1e-12, atol=1e-15)
    for f, code in ((5, 82), (6, 81), (7, 80)):
        bo, bl = lay[f][2], lay[f][3]
        np.testing.assert_allclose(g[code].reshape(B, bl).sum(0), grads[bo:bo + bl], rtol=1e-12,
                                   atol=1e-15)
