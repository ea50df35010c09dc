"""Validity of the decisions the bf16 path takes on rounded values: the ReLU's
sign and the max-pools' window choices.

Both sides compute the same network; the GPU stores every activation in bf16
and accumulates every sum in fp32, the oracle keeps fp64.  Where a unit's
pre-activation, or a pooling window's two largest values, sit closer together
than that rounding, the two sides may legitimately decide differently, and
every later gradient then takes a different path.  The end-to-end gradient
tests therefore hand the GPU's own decisions to the oracle; this module checks
first that each of those decisions is one the rounding allows, unit by unit,
in both directions.

The bounds are local to a layer.  For layer l the GPU's own input map x^ is
read back, and the oracle computes in fp64 (single ops, pinned on the CPU)

    z' = conv(x^, w) + b          A = conv(|x^|, |w|)

with the same bf16 weights.  The GPU's fp32 sum of the n exact bf16 products,
in any order, plus the bias add, lies within

    tau = gamma_n A + 2u (|z'| + |b|),   gamma_n = n u / (1 - n u),  u = 2^-23

of z' (u is twice fp32's unit roundoff, so adders that truncate are covered
too).  A bf16 store rounds to nearest: relative error <= U = 2^-8.  Hence, for
every unit:

  * decision: the GPU's unit is active iff z' > 0, except where |z'| <= tau;
  * value: the stored output a^ satisfies |a^ - relu(z')| <= (1 + U) tau + U relu(z');
  * normalisation map b^ (conv1, conv2): |b^ - LRN(a^)| <= (U + 2^-18) |LRN(a^)|
    (fp32 arithmetic with approximate reciprocal square roots, then the store);
  * window choice: the first maximum of the GPU's own pooled-from map, exactly.

End to end, against the oracle's own forward (z_o, its maps m_o): a differing
ReLU decision needs |z_o| <= |z_o - z'| + tau, and a window choice c of the
GPU needs m_o[c] >= max(window of m_o) - eps[c] - eps[m*], eps being the
exactly computed difference between the oracle's map and the map it computes
from the GPU's inputs, plus the local rounding bound above.  The rates of
differing decisions are returned so that the tests can bound and print them.
"""
import numpy as np

import oracle

U_BF16 = 2.0 ** -8
U_ACC = 2.0 ** -23
LRN_REL = U_BF16 + 2.0 ** -18


def gamma(n):
    return n * U_ACC / (1.0 - n * U_ACC)


def _weights(net, op, l):
    lay = oracle.param_layout(net)
    wo, wl, bo, bl = lay[l]
    if l < 5:
        Cin = net.in_c if l == 0 else net.conv_c[l - 1]
        shape = (net.conv_c[l], net.conv_k[l], net.conv_k[l], Cin // net.conv_g[l])
    else:
        In = oracle.map_sizes(net)[4][2] ** 2 * net.conv_c[4] if l == 5 else net.fc_n[l - 6]
        shape = (net.fc_n[l - 5], In)
    return op[wo:wo + wl].reshape(shape), op[bo:bo + bl]


def local_sum(net, op, l, x_hat):
    """z' (fp64 pre-activation from the GPU's input) and tau (the fp32
    accumulation + bias rounding bound) of layer l (0..4 conv, 5/6 FC6/FC7)."""
    w, b = _weights(net, op, l)
    if l < 5:
        s, p = net.conv_s[l], net.conv_p[l]
        g = net.conv_g[l]
        z = oracle.conv_fwd(x_hat, w, b, s, p, g)
        A = oracle.conv_fwd(np.abs(x_hat), np.abs(w), None, s, p, g)
        n = w.shape[1] * w.shape[2] * w.shape[3]
    else:
        z = oracle.fc_fwd(x_hat, w, b)
        A = oracle.fc_fwd(np.abs(x_hat), np.abs(w), None)
        n = w.shape[1]
    tau = gamma(n) * A + 2 * U_ACC * (np.abs(z) + np.abs(b))
    return z, tau


def check_layer(z_loc, tau, a_hat, z_own, keep=None):
    """Decision and value checks of one layer's ReLU output (see the module
    docstring).  keep: optional dropout keep mask (FC6/FC7): dropped units must
    be exactly 0 and take no decision.  Returns (local mismatch rate,
    end-to-end flip rate)."""
    z_loc = z_loc.ravel()
    tau = tau.ravel()
    a_hat = a_hat.ravel()
    z_own = z_own.ravel()
    live = np.ones(z_loc.shape, bool) if keep is None else keep.ravel().astype(bool)
    if keep is not None:
        assert np.all(a_hat[~live] == 0.0), "dropped units must be exactly zero"
    gpu_on = (a_hat > 0) & live
    loc_on = (z_loc > 0) & live
    mism = gpu_on != loc_on
    assert np.all(np.abs(z_loc[mism]) <= tau[mism]), \
        "a GPU ReLU decision contradicts the fp64 sum of its own inputs beyond fp32 rounding"
    rz = np.maximum(z_loc, 0.0)
    bound = (1 + U_BF16) * tau + U_BF16 * rz
    err = np.abs(a_hat - rz)
    assert np.all(err[live] <= bound[live]), \
        "stored output outside the rounding bound of its own inputs: max excess %g" % \
        float(np.max((err - bound)[live]))
    own_on = (z_own > 0) & live
    flip = gpu_on != own_on
    assert np.all(np.abs(z_own[flip]) <= np.abs(z_own - z_loc)[flip] + tau[flip])
    n = max(int(live.sum()), 1)
    return float(mism.sum()) / n, float(flip.sum()) / n


def check_lrn_map(b_hat, a_hat, n=5, k=2.0, alpha=1e-4, beta=0.75):
    """The GPU's normalised map against the oracle's normalisation of the
    GPU's own input; returns the fp64 map LRN(a^)."""
    want = oracle.lrn_fwd(a_hat, n, k, alpha, beta)
    assert np.all(np.abs(b_hat - want) <= LRN_REL * np.abs(want) + 1e-30), \
        "normalised map outside the rounding bound of its own input"
    return want


def check_windows(m_own, m_loc, eps_loc, choice, z=3, s=2):
    """End-to-end window check: m_own is the oracle's pooled-from map, m_loc
    the one the oracle computes from the GPU's inputs, eps_loc the local
    rounding bound of the GPU's map around m_loc (all [B, H, W, C]); choice
    the GPU's window offsets [B, P, P, C].  Returns the fraction of windows
    whose GPU choice differs from the oracle's own first maximum."""
    eps = np.abs(m_own - m_loc) + eps_loc
    B, H, W, C = m_own.shape
    P = (H - z) // s + 1
    best = None
    arg = None
    at_choice = np.zeros((B, P, P, C))
    eps_choice = np.zeros((B, P, P, C))
    for dy in range(z):
        for dx in range(z):
            v = m_own[:, dy:dy + s * (P - 1) + 1:s, dx:dx + s * (P - 1) + 1:s, :]
            e = eps[:, dy:dy + s * (P - 1) + 1:s, dx:dx + s * (P - 1) + 1:s, :]
            off = dy * z + dx
            if best is None:
                best, arg, eps_best = v.copy(), np.zeros(v.shape, np.uint8), e.copy()
            else:
                gt = v > best
                best = np.where(gt, v, best)
                arg = np.where(gt, off, arg).astype(np.uint8)
                eps_best = np.where(gt, e, eps_best)
            sel = choice == off
            at_choice[sel] = v[sel]
            eps_choice[sel] = e[sel]
    assert np.all(at_choice >= best - eps_choice - eps_best), \
        "a GPU window choice is below the oracle's window maximum by more than the bound"
    return float(np.mean(arg != choice))


def validate(net, params, x, g, seed, step):
    """Every check above on one training-mode forward of `net`.

    g: the implementation's maps by the library's debug codes (flat or
    shaped): 0..4 conv outputs after the ReLU, 10+l the normalised maps (where
    the network normalises), 20+l the pooled maps, 30/31 FC6/FC7 outputs after
    dropout, 90+l the window choices.  params: the weights both sides use
    (bf16 values), x the input (bf16 values).  Returns (choices, relu, rates):
    the window choices and ReLU sign decisions to hand to the oracle's step,
    and per layer (local mismatch rate, end-to-end flip rate) plus
    "pool<l>": the fraction of windows whose choice differs from the
    oracle's own."""
    B = x.shape[0]
    ms = oracle.map_sizes(net)

    def shaped(code, l, side):
        return np.asarray(g[code], dtype=np.float64).reshape(B, side, side, net.conv_c[l])

    A = {l: shaped(l, l, ms[l][1]) for l in range(5)}
    pooled = {l: shaped(20 + l, l, ms[l][2]) for l in range(5) if net.pool_after[l]}
    codes = [100, 101, 102, 103, 104, 105, 106]
    for l in range(5):
        if net.pool_after[l]:
            codes.append(10 + l if net.lrn_after[l] else l)
    t = oracle.forward_trace(net, params, x, sorted(set(codes)), mode=0, seed=seed, step=step)
    inputs = {0: x}
    for l in range(1, 5):
        inputs[l] = pooled[l - 1] if net.pool_after[l - 1] else A[l - 1]
    inputs[5] = (pooled[4] if net.pool_after[4] else A[4]).reshape(B, -1)
    inputs[6] = np.asarray(g[30], dtype=np.float64).reshape(B, -1)
    rates, loc = {}, {}
    for l in range(7):
        z_loc, tau = local_sum(net, params, l, inputs[l])
        loc[l] = (z_loc, tau)
        own = t[100 + l] if l < 5 else t[105 + l - 5]
        keep = None
        if l >= 5 and net.dropout_on:
            keep = oracle.dropout_mask(seed, l + 1, step, B, net.fc_n[l - 5])
        a_hat = A[l] if l < 5 else np.asarray(g[30 + l - 5], dtype=np.float64).reshape(B, -1)
        rates[l] = check_layer(z_loc, tau, a_hat, own, keep)
    choices = {}
    for l in range(5):
        if not net.pool_after[l]:
            continue
        side = ms[l][1]
        if net.lrn_after[l]:
            m_hat = shaped(10 + l, l, side)
            m_loc = check_lrn_map(m_hat, A[l], net.lrn_n, net.lrn_k, net.lrn_alpha, net.lrn_beta)
            eps_loc = LRN_REL * np.abs(m_loc)
            m_own = t[10 + l].reshape(m_hat.shape)
        else:
            m_hat = A[l]
            z_loc, tau = loc[l]
            m_loc = np.maximum(z_loc, 0).reshape(m_hat.shape)
            eps_loc = (1 + U_BF16) * tau.reshape(m_hat.shape) + U_BF16 * m_loc
            m_own = t[l].reshape(m_hat.shape)
        P = ms[l][2]
        ch = np.asarray(g[90 + l], dtype=np.uint8).reshape(B, P, P, net.conv_c[l])
        # the choice is the first maximum of the implementation's own map, and
        # the pooled map is the value it chose (both exact)
        _, own_choice = oracle.maxpool_fwd(m_hat, net.pool_z, net.pool_s)
        np.testing.assert_array_equal(own_choice, ch)
        np.testing.assert_array_equal(oracle.maxpool_select(m_hat, ch, net.pool_z, net.pool_s),
                                      pooled[l])
        rates["pool%d" % l] = check_windows(m_own, m_loc, eps_loc, ch, net.pool_z, net.pool_s)
        choices[l] = ch
    relu = {l: (A[l] > 0).astype(np.uint8) for l in range(5)}
    for f in range(2):
        relu[5 + f] = (np.asarray(g[30 + f]).reshape(B, -1) > 0).astype(np.uint8)
    return choices, relu, rates
