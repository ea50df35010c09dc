"""The decision checker of tests/_decisions.py, pinned on the CPU.

A stand-in for the GPU's arithmetic -- every activation rounded to bf16,
every sum accumulated in fp32 (torch's CPU float32 convolution and matrix
product), the normalisation in float32 -- runs the shrunken network; its maps
must pass every check.  Planted mistakes (a unit switched off whose
pre-activation is far from zero, a pooling choice of a clearly smaller
element, an output off by 5%) must each fail one.  Nothing here touches the
CUDA library.
"""
import numpy as np
import pytest
import torch
import torch.nn.functional as F

import oracle
from tests import _decisions as D

SEED, STEP = 9, 2


def _bf16(a):
    return torch.as_tensor(a, dtype=torch.float32).to(torch.bfloat16).to(torch.float64).numpy()


def _weights(net, params):
    ws = []
    for l in range(8):
        ws.append(D._weights(net, params, l))
    return ws


def _simulate(net, params, x, mode=0):
    """bf16-storage / fp32-accumulation forward; returns the maps under the
    library's debug codes (0..4 conv outputs, 10/11 normalised maps, 20/21/24
    pooled maps, 30/31 FC outputs, 90/91/94 window choices)."""
    B = x.shape[0]
    ws = _weights(net, params)
    out = {}
    cur = x
    for l in range(5):
        w, b = ws[l]
        xt = torch.from_numpy(cur.astype(np.float32)).permute(0, 3, 1, 2)
        wt = torch.from_numpy(w.astype(np.float32)).permute(0, 3, 1, 2).contiguous()
        z = F.conv2d(xt, wt, torch.from_numpy(b.astype(np.float32)), stride=net.conv_s[l],
                     padding=net.conv_p[l], groups=net.conv_g[l])
        a = _bf16(torch.relu(z).permute(0, 2, 3, 1).numpy())
        out[l] = a
        m = a
        if net.lrn_after[l]:
            a32 = torch.from_numpy(a.astype(np.float32))
            sq = F.pad(a32 * a32, (2, 2))
            s = sum(sq[..., i:i + a.shape[-1]] for i in range(5))
            m = _bf16((a32 * (net.lrn_k + net.lrn_alpha * s) ** -net.lrn_beta).numpy())
            out[10 + l] = m
        cur = m
        if net.pool_after[l]:
            cur, am = oracle.maxpool_fwd(m)
            out[20 + l] = cur
            out[90 + l] = am
    h = cur.reshape(B, -1)
    for f in range(3):
        w, b = ws[5 + f]
        z = (torch.from_numpy(h.astype(np.float32)) @ torch.from_numpy(w.astype(np.float32)).T
             + torch.from_numpy(b.astype(np.float32))).numpy()
        if f == 2:
            out[40] = z
            break
        a = np.maximum(z, 0)
        if mode == 0:
            a = a * oracle.dropout_mask(SEED, 6 + f, STEP, B, net.fc_n[f])
        else:
            a = a * 0.5
        h = _bf16(a)
        out[30 + f] = h
    return out


def _setup():
    net = oracle.small_net()
    n = oracle.param_count(net)
    r = np.random.default_rng(23)
    params = _bf16(r.standard_normal(n) * 0.15)
    for (wo, wl, bo, bl) in oracle.param_layout(net):
        params[bo:bo + bl] = r.uniform(-0.05, 0.2, bl)
    x = _bf16(r.standard_normal((3, 67, 67, 3)))
    return net, params, x


def _run_checks(net, params, x, g):
    return D.validate(net, params, x, g, SEED, STEP)[2]


def test_checks_accept_a_bf16_fp32_pipeline():
    net, params, x = _setup()
    g = _simulate(net, params, x)
    rates = _run_checks(net, params, x, g)
    for l in range(7):
        assert rates[l][0] < 0.01  # local mismatches: only units within fp32 rounding of 0


def test_checks_reject_a_unit_switched_off():
    net, params, x = _setup()
    g = _simulate(net, params, x)
    a = g[2].copy().ravel()
    i = int(np.argmax(a))  # the most active unit of conv3
    a[i] = 0.0
    g[2] = a.reshape(g[2].shape)
    with pytest.raises(AssertionError):
        _run_checks(net, params, x, g)


def test_checks_reject_an_output_off_by_five_percent():
    net, params, x = _setup()
    g = _simulate(net, params, x)
    a = g[1].copy().ravel()
    i = int(np.argmax(a))
    a[i] *= 1.05
    g[1] = a.reshape(g[1].shape)
    with pytest.raises(AssertionError):
        _run_checks(net, params, x, g)


def test_checks_reject_a_wrong_window_choice():
    net, params, x = _setup()
    g = _simulate(net, params, x)
    m = g[10]
    am = g[90].copy()
    # pick the window whose maximum stands furthest above its smallest element
    # and choose the smallest element instead
    P = am.shape[1]
    best, where = -1.0, None
    for oh in range(P):
        for ow in range(P):
            win = m[:, 2 * oh:2 * oh + 3, 2 * ow:2 * ow + 3, :]
            gap = win.max(axis=(1, 2)) - win.min(axis=(1, 2))
            b, c = np.unravel_index(np.argmax(gap), gap.shape)
            if gap[b, c] > best:
                flat = win[b, :, :, c].ravel()
                best, where = gap[b, c], (b, oh, ow, c, int(np.argmin(flat)))
    b, oh, ow, c, off = where
    am[b, oh, ow, c] = off
    m_own = oracle.forward_trace(net, params, x, [10], mode=0, seed=SEED, step=STEP)[10]
    with pytest.raises(AssertionError):
        D.check_windows(m_own.reshape(m.shape), m, D.LRN_REL * np.abs(m), am)
