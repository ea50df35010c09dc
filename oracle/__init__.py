"""CPU oracle for the AlexNet training hot path (test infrastructure only).

The oracle is a plain C library (``alexnet_oracle.c``: fp64 storage and
accumulation, direct nested loops) wrapped here with ctypes and numpy.  Only
the tests, ``__graft_entry__.smoke()`` and the benchmark's CPU-baseline leg use
it.  It shares no code with the CUDA library in ``deep_cnn_image_b200`` and
neither side imports the other.

Pages cited (title, section):
  [S]  "ImageNet Classification with Deep Convolutional Neural Networks",
       paper-graph-ui summary page.
  [W]  "AlexNet and Deep CNNs" (fermi.ai wiki page).
  [P2] "AlexNet Part 2: Turning the Training Recipe into Testable Design
       Choices" (bloss0m page).
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from ctypes import POINTER, c_double, c_int, c_int64, c_uint8, c_uint32, c_uint64

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "alexnet_oracle.c")
_LIB_PATH = os.path.join(_HERE, "liboracle.so")
_lib = None


def build(force: bool = False) -> str:
    """Compile the C oracle into ``oracle/liboracle.so`` (gcc, OpenMP)."""
    if force or not os.path.exists(_LIB_PATH) or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC):
        tmp = _LIB_PATH + ".tmp%d" % os.getpid()
        subprocess.check_call(["gcc", "-O2", "-std=c11", "-fopenmp", "-fPIC", "-shared",
                               "-fvisibility=hidden", "-ffp-contract=off", _SRC, "-o", tmp, "-lm"])
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


class Net(ctypes.Structure):
    """Network description (mirrors ``oracle_net`` in the C source)."""
    _fields_ = [
        ("in_hw", c_int), ("in_c", c_int),
        ("conv_c", c_int * 5), ("conv_k", c_int * 5), ("conv_s", c_int * 5),
        ("conv_p", c_int * 5), ("conv_g", c_int * 5),
        ("lrn_after", c_int * 5), ("pool_after", c_int * 5),
        ("fc_n", c_int * 3),
        ("pool_z", c_int), ("pool_s", c_int),
        ("lrn_n", c_int),
        ("lrn_k", c_double), ("lrn_alpha", c_double), ("lrn_beta", c_double),
        ("dropout_on", c_int),
        ("dropout_p", c_double),
    ]


def _ivec(t, n):
    return (c_int * n)(*t)


def alexnet(grouped: bool = True, lrn: bool = True, dropout: bool = True,
            pool_z: int = 3) -> Net:
    """The eight-layer network of [S] 3.4 "Overall Architecture" and [W]
    "Layer-by-layer structure" on a 227x227x3 input.  grouped=True gives
    conv2/4/5 two groups (the two-GPU restricted connectivity)."""
    g = 2 if grouped else 1
    return Net(227, 3, _ivec((96, 256, 384, 384, 256), 5), _ivec((11, 5, 3, 3, 3), 5),
               _ivec((4, 1, 1, 1, 1), 5), _ivec((0, 2, 1, 1, 1), 5), _ivec((1, g, 1, g, g), 5),
               _ivec((1, 1, 0, 0, 0) if lrn else (0, 0, 0, 0, 0), 5), _ivec((1, 1, 0, 0, 1), 5),
               _ivec((4096, 4096, 1000), 3), pool_z, 2, 5, 2.0, 1e-4, 0.75,
               1 if dropout else 0, 0.5)


def small_net() -> Net:
    """A shrunken instance with AlexNet's op sequence (67x67 input gives
    15 -> 7 -> 7 -> 3 -> 3 -> 3 -> 3 -> 1), for finite-difference checks."""
    return Net(67, 3, _ivec((8, 8, 12, 12, 8), 5), _ivec((11, 5, 3, 3, 3), 5),
               _ivec((4, 1, 1, 1, 1), 5), _ivec((0, 2, 1, 1, 1), 5), _ivec((1, 2, 1, 2, 2), 5),
               _ivec((1, 1, 0, 0, 0), 5), _ivec((1, 1, 0, 0, 1), 5), _ivec((16, 16, 10), 3),
               3, 2, 5, 2.0, 1e-4, 0.75, 1, 0.5)


def lib():
    global _lib
    if _lib is None:
        path = build()
        L = ctypes.CDLL(path)
        dp, ip, u8p, i32p, i64p = POINTER(c_double), POINTER(c_int), POINTER(c_uint8), \
            POINTER(ctypes.c_int32), POINTER(c_int64)
        u32p = POINTER(c_uint32)
        netp = POINTER(Net)
        sig = {
            "oracle_philox4x32_10": (None, [u32p, u32p, u32p]),
            "oracle_conv_out_size": (c_int, [c_int] * 4),
            "oracle_conv_fwd": (None, [dp, c_int, c_int, c_int, c_int, dp, dp, c_int, c_int,
                                       c_int, c_int, c_int, dp]),
            "oracle_conv_bwd": (None, [dp, c_int, c_int, c_int, c_int, dp, c_int, c_int, c_int,
                                       c_int, c_int, dp, dp, dp, dp]),
            "oracle_conv_fwd_sampled": (None, [dp, c_int, c_int, c_int, c_int, dp, dp, c_int, c_int,
                                               c_int, c_int, c_int, i64p, c_int, dp]),
            "oracle_conv_wgrad_sampled": (None, [dp, c_int, c_int, c_int, c_int, c_int, c_int,
                                                 c_int, c_int, c_int, dp, i64p, c_int, dp]),
            "oracle_relu": (None, [dp, c_int64]),
            "oracle_relu_bwd": (None, [dp, dp, c_int64]),
            "oracle_lrn_fwd": (None, [dp, c_int64, c_int, c_int, c_double, c_double, c_double, dp]),
            "oracle_lrn_bwd": (None, [dp, dp, c_int64, c_int, c_int, c_double, c_double, c_double,
                                      dp]),
            "oracle_pool_out_size": (c_int, [c_int] * 3),
            "oracle_maxpool_fwd": (None, [dp, c_int, c_int, c_int, c_int, c_int, c_int, dp, u8p]),
            "oracle_maxpool_bwd": (None, [dp, u8p, c_int, c_int, c_int, c_int, c_int, c_int, dp]),
            "oracle_fc_fwd": (None, [dp, c_int, c_int, dp, dp, c_int, dp]),
            "oracle_fc_bwd": (None, [dp, c_int, c_int, dp, c_int, dp, dp, dp, dp]),
            "oracle_dropout_mask": (None, [c_uint64, c_uint32, c_uint32, c_int, c_int, c_double,
                                           u8p]),
            "oracle_softmax_ce": (c_double, [dp, i32p, c_int, c_int, dp, dp]),
            "oracle_sgd": (None, [dp, dp, dp, c_int64, c_double, c_double, c_double]),
            "oracle_param_count": (c_int64, [netp]),
            "oracle_param_layout": (None, [netp, i64p]),
            "oracle_forward_macs": (c_int64, [netp]),
            "oracle_neuron_counts": (None, [netp, i64p]),
            "oracle_forward": (None, [netp, dp, dp, c_int, c_int, c_uint64, c_uint32, dp, dp]),
            "oracle_forward_probe": (None, [netp, dp, dp, c_int, c_int, c_uint64, c_uint32, c_int,
                                            dp]),
            "oracle_forward_trace": (None, [netp, dp, dp, c_int, c_int, c_uint64, c_uint32, c_int,
                                            ip, POINTER(dp)]),
            "oracle_train_step": (c_double, [netp, dp, dp, dp, i32p, c_int, c_double, c_double,
                                             c_double, c_uint64, c_uint32, dp, dp]),
            "oracle_train_step_rows": (c_double, [netp, dp, dp, dp, i32p, c_int, c_double,
                                                  c_double, c_double, c_uint64, c_uint32, c_int,
                                                  dp, dp]),
            "oracle_dropout_mask_rows": (None, [c_uint64, c_uint32, c_uint32, c_int, c_int, c_int,
                                                c_double, u8p]),
            "oracle_loss": (c_double, [netp, dp, dp, i32p, c_int, c_uint64, c_uint32]),
            "oracle_train_probe": (None, [netp, dp, dp, i32p, c_int, c_uint64, c_uint32, c_int,
                                          dp, u8p, u8p, u8p, POINTER(u8p)]),
            "oracle_train_step_given": (c_double, [netp, dp, dp, dp, i32p, c_int, c_double,
                                                   c_double, c_double, c_uint64, c_uint32, dp, dp,
                                                   u8p, u8p, u8p, POINTER(u8p)]),
            "oracle_maxpool_select": (None, [dp, u8p, c_int, c_int, c_int, c_int, c_int, c_int,
                                             dp]),
            "oracle_aug_draws": (None, [c_uint64, c_uint32, c_uint32, i32p, dp]),
            "oracle_augment": (None, [u8p, c_int, dp, dp, dp, c_uint64, c_uint32, dp]),
            "oracle_tencrop_inputs": (None, [u8p, c_int, dp, dp]),
            "oracle_topk": (None, [dp, c_int, c_int, c_int, i32p]),
            "oracle_tencrop": (None, [netp, dp, u8p, c_int, dp, dp, i32p]),
        }
        for name, (res, args) in sig.items():
            f = getattr(L, name)
            f.restype = res
            f.argtypes = args
        _lib = L
    return _lib


def _d(a):
    a = np.ascontiguousarray(a, dtype=np.float64)
    return a, a.ctypes.data_as(POINTER(c_double))


def _p(a, ctype):
    return a.ctypes.data_as(POINTER(ctype))


# --------------------------------------------------------------------------
# Philox4x32-10 (Salmon et al., SC'11) and the draws built on it
# --------------------------------------------------------------------------
def philox4x32_10(ctr, key):
    c = (c_uint32 * 4)(*[int(v) & 0xFFFFFFFF for v in ctr])
    k = (c_uint32 * 2)(*[int(v) & 0xFFFFFFFF for v in key])
    o = (c_uint32 * 4)()
    lib().oracle_philox4x32_10(c, k, o)
    return [int(v) for v in o]


def dropout_mask(seed, layer, step, B, out, p=0.5, row0=0):
    """[S] 3.4 "Dropout": keep mask (uint8 0/1) of FC layer 6 or 7; row0: the
    first image's index in the whole minibatch."""
    m = np.zeros((B, out), np.uint8)
    lib().oracle_dropout_mask_rows(seed, layer, step, row0, B, out, p, _p(m, c_uint8))
    return m


def aug_draws(seed, img, step):
    o = np.zeros(3, np.int32)
    a = np.zeros(3, np.float64)
    lib().oracle_aug_draws(seed, img, step, _p(o, ctypes.c_int32), _p(a, c_double))
    return int(o[0]), int(o[1]), int(o[2]), a


# --------------------------------------------------------------------------
# Single ops (NHWC numpy arrays, fp64)
# --------------------------------------------------------------------------
def conv_fwd(x, w, b, stride, pad, groups):
    """[S] 3.4 "Overall Architecture": y = bias + sum over the kernel taps."""
    x, xp = _d(x)
    w, wp = _d(w)
    B, H, W, C = x.shape
    Cout, K = w.shape[0], w.shape[1]
    Ho = (H + 2 * pad - K) // stride + 1
    Wo = (W + 2 * pad - K) // stride + 1
    y = np.zeros((B, Ho, Wo, Cout))
    bp = None
    if b is not None:
        b, bp = _d(b)
    lib().oracle_conv_fwd(xp, B, H, W, C, w.ctypes.data_as(POINTER(c_double)), bp, Cout, K,
                          stride, pad, groups, _p(y, c_double))
    return y


def conv_bwd(x, w, dy, stride, pad, groups, need_dx=True):
    x, xp = _d(x)
    w, wp = _d(w)
    dy, dyp = _d(dy)
    B, H, W, C = x.shape
    Cout, K = w.shape[0], w.shape[1]
    dx = np.zeros_like(x) if need_dx else None
    dw = np.zeros_like(w)
    db = np.zeros(Cout)
    lib().oracle_conv_bwd(xp, B, H, W, C, wp, Cout, K, stride, pad, groups, dyp,
                          _p(dx, c_double) if need_dx else None, _p(dw, c_double), _p(db, c_double))
    return dx, dw, db


def conv_fwd_sampled(x, w, b, stride, pad, groups, idx):
    x, xp = _d(x)
    w, wp = _d(w)
    B, H, W, C = x.shape
    Cout, K = w.shape[0], w.shape[1]
    idx = np.ascontiguousarray(idx, dtype=np.int64)
    out = np.zeros(len(idx))
    bp = None
    if b is not None:
        b, bp = _d(b)
    lib().oracle_conv_fwd_sampled(xp, B, H, W, C, wp, bp, Cout, K, stride, pad, groups,
                                  _p(idx, c_int64), len(idx), _p(out, c_double))
    return out


def conv_wgrad_sampled(x, dy, Cout, K, stride, pad, groups, idx):
    x, xp = _d(x)
    dy, dyp = _d(dy)
    B, H, W, C = x.shape
    idx = np.ascontiguousarray(idx, dtype=np.int64)
    out = np.zeros(len(idx))
    lib().oracle_conv_wgrad_sampled(xp, B, H, W, C, Cout, K, stride, pad, groups, dyp,
                                    _p(idx, c_int64), len(idx), _p(out, c_double))
    return out


def relu(x):
    x = np.array(x, dtype=np.float64, copy=True)
    lib().oracle_relu(_p(x, c_double), x.size)
    return x


def lrn_fwd(a, n=5, k=2.0, alpha=1e-4, beta=0.75):
    """[S] 3.4 "Local Response Normalization" over the last (channel) axis."""
    a, ap = _d(a)
    N = a.shape[-1]
    b = np.zeros_like(a)
    lib().oracle_lrn_fwd(ap, a.size // N, N, n, k, alpha, beta, _p(b, c_double))
    return b


def lrn_bwd(a, g, n=5, k=2.0, alpha=1e-4, beta=0.75):
    a, ap = _d(a)
    g, gp = _d(g)
    N = a.shape[-1]
    da = np.zeros_like(a)
    lib().oracle_lrn_bwd(ap, gp, a.size // N, N, n, k, alpha, beta, _p(da, c_double))
    return da


def maxpool_fwd(x, z=3, s=2):
    """[S] 3.4 "Overlapping Pooling": returns (pooled, argmax offsets)."""
    x, xp = _d(x)
    B, H, W, C = x.shape
    Ho, Wo = (H - z) // s + 1, (W - z) // s + 1
    y = np.zeros((B, Ho, Wo, C))
    am = np.zeros((B, Ho, Wo, C), np.uint8)
    lib().oracle_maxpool_fwd(xp, B, H, W, C, z, s, _p(y, c_double), _p(am, c_uint8))
    return y, am


def maxpool_bwd(dy, argmax, H, W, z=3, s=2):
    dy, dyp = _d(dy)
    argmax = np.ascontiguousarray(argmax, dtype=np.uint8)
    B, _, _, C = dy.shape
    dx = np.zeros((B, H, W, C))
    lib().oracle_maxpool_bwd(dyp, _p(argmax, c_uint8), B, H, W, C, z, s, _p(dx, c_double))
    return dx


def fc_fwd(x, w, b):
    x, xp = _d(x)
    w, wp = _d(w)
    B, In = x.shape
    Out = w.shape[0]
    y = np.zeros((B, Out))
    bp = None
    if b is not None:
        b, bp = _d(b)
    lib().oracle_fc_fwd(xp, B, In, wp, bp, Out, _p(y, c_double))
    return y


def fc_bwd(x, w, dz, need_dx=True):
    x, xp = _d(x)
    w, wp = _d(w)
    dz, dzp = _d(dz)
    B, In = x.shape
    Out = w.shape[0]
    dx = np.zeros_like(x) if need_dx else None
    dw = np.zeros_like(w)
    db = np.zeros(Out)
    lib().oracle_fc_bwd(xp, B, In, wp, Out, dzp, _p(dx, c_double) if need_dx else None,
                        _p(dw, c_double), _p(db, c_double))
    return dx, dw, db


def softmax_ce(z, labels=None):
    """Returns (loss, probs, dlogits) ([S] 3.4 "Objective function")."""
    z, zp = _d(z)
    B, N = z.shape
    probs = np.zeros_like(z)
    dz = np.zeros_like(z)
    lp = None
    if labels is not None:
        labels = np.ascontiguousarray(labels, dtype=np.int32)
        lp = _p(labels, ctypes.c_int32)
    loss = lib().oracle_softmax_ce(zp, lp, B, N, _p(probs, c_double), _p(dz, c_double))
    return loss, probs, dz


def sgd(w, v, g, lr, momentum=0.9, wd=5e-4):
    """[S] 3.4 "Training Procedure Details", update rule.  Returns new (w, v)."""
    w = np.array(w, dtype=np.float64, copy=True)
    v = np.array(v, dtype=np.float64, copy=True)
    g, gp = _d(g)
    lib().oracle_sgd(_p(w, c_double), _p(v, c_double), gp, w.size, lr, momentum, wd)
    return w, v


def topk(probs, k=5):
    probs, pp = _d(probs)
    B, N = probs.shape
    idx = np.zeros((B, k), np.int32)
    lib().oracle_topk(pp, B, N, k, _p(idx, ctypes.c_int32))
    return idx


def knn(queries, base, k):
    """[S] "Qualitative Evaluation" (Figure 4, right): retrieval by the
    Euclidean distance between feature vectors.  For every query row the k
    base rows of smallest squared distance sum_d (q_d - x_d)^2, in fp64 and
    written out directly (no norm expansion); ties go to the lower base
    index.  Returns (squared distances [Q, k], indices [Q, k])."""
    q = np.asarray(queries, dtype=np.float64)
    x = np.asarray(base, dtype=np.float64)
    Q, N = q.shape[0], x.shape[0]
    dist = np.zeros((Q, k))
    idx = np.zeros((Q, k), np.int64)
    for i in range(Q):
        diff = x - q[i]
        d = np.einsum("nd,nd->n", diff, diff)
        order = np.lexsort((np.arange(N), d))[:k]  # by distance, then index
        dist[i] = d[order]
        idx[i] = order
    return dist, idx


# --------------------------------------------------------------------------
# Whole network
# --------------------------------------------------------------------------
def param_count(net):
    return int(lib().oracle_param_count(ctypes.byref(net)))


def param_layout(net):
    """[(w_off, w_len, b_off, b_len)] for the 8 learned layers."""
    o = np.zeros(32, np.int64)
    lib().oracle_param_layout(ctypes.byref(net), _p(o, c_int64))
    return [(int(o[l]), int(o[8 + l]), int(o[16 + l]), int(o[24 + l])) for l in range(8)]


def forward_macs(net):
    return int(lib().oracle_forward_macs(ctypes.byref(net)))


def neuron_counts(net):
    o = np.zeros(8, np.int64)
    lib().oracle_neuron_counts(ctypes.byref(net), _p(o, c_int64))
    return [int(v) for v in o]


def forward(net, params, x, mode=1, seed=0, step=0):
    """Returns (logits, probs).  mode 0 = training (dropout drawn), 1 = inference."""
    params, pp = _d(params)
    x, xp = _d(x)
    B = x.shape[0]
    N = net.fc_n[2]
    logits = np.zeros((B, N))
    probs = np.zeros((B, N))
    lib().oracle_forward(ctypes.byref(net), pp, xp, B, mode, seed, step, _p(logits, c_double),
                         _p(probs, c_double))
    return logits, probs


PROBE_RELU, PROBE_LRN, PROBE_POOL, PROBE_FC, PROBE_LOGITS = 0, 10, 20, 30, 40


def map_sizes(net):
    """Per conv layer: (input side, conv output side, side after pooling)."""
    out = []
    hw = net.in_hw
    for l in range(5):
        o = (hw + 2 * net.conv_p[l] - net.conv_k[l]) // net.conv_s[l] + 1
        p = (o - net.pool_z) // net.pool_s + 1 if net.pool_after[l] else o
        out.append((hw, o, p))
        hw = p
    return out


def probe_size(net, which):
    """Elements per image of the map forward_probe returns for `which`."""
    ms = map_sizes(net)
    if which < 20:
        l = which % 10
        return ms[l][1] ** 2 * net.conv_c[l]
    if which < 30:
        l = which - 20
        return ms[l][2] ** 2 * net.conv_c[l]
    if which < 40:
        return net.fc_n[which - 30]
    return net.fc_n[2]


def forward_probe(net, params, x, which, mode=1, seed=0, step=0):
    """One intermediate map of a forward pass, flat (see oracle_forward_probe)."""
    params, pp = _d(params)
    x, xp = _d(x)
    B = x.shape[0]
    out = np.zeros(B * probe_size(net, which))
    lib().oracle_forward_probe(ctypes.byref(net), pp, xp, B, mode, seed, step, which,
                               _p(out, c_double))
    return out


# forward_trace codes beyond forward_probe's: pre-activations (before the ReLU)
TRACE_PRE, TRACE_FC_PRE = 100, 105


def trace_size(net, which):
    """Elements per image of the map forward_trace returns for `which`."""
    if which < 100:
        return probe_size(net, which)
    if which in (105, 106):
        return net.fc_n[which - 105]
    return map_sizes(net)[which - 100][1] ** 2 * net.conv_c[which - 100]


def forward_trace(net, params, x, which, mode=1, seed=0, step=0):
    """Several maps of ONE forward pass (codes of forward_probe, plus the
    pre-activations TRACE_PRE + l and TRACE_FC_PRE + f), as {code: flat array}."""
    params, pp = _d(params)
    x, xp = _d(x)
    B = x.shape[0]
    which = [int(w) for w in which]
    outs = [np.zeros(B * trace_size(net, w)) for w in which]
    arr = (POINTER(c_double) * len(which))(*[_p(o, c_double) for o in outs])
    wv = (c_int * len(which))(*which)
    lib().oracle_forward_trace(ctypes.byref(net), pp, xp, B, mode, seed, step, len(which), wv,
                               arr)
    return dict(zip(which, outs))


def train_step_rows(net, params, velocity, x, labels, row0, lr=0.01, momentum=0.9, wd=5e-4,
                    seed=0, step=0):
    """The step of images row0 .. row0 + B - 1 of a minibatch (their rows of
    the dropout masks; the loss averaged over these B).  Returns (loss,
    new_params, new_velocity, grads, logits)."""
    params = np.array(params, dtype=np.float64, copy=True)
    velocity = np.array(velocity, dtype=np.float64, copy=True)
    x, xp = _d(x)
    labels = np.ascontiguousarray(labels, dtype=np.int32)
    B = x.shape[0]
    grads = np.zeros_like(params)
    logits = np.zeros((B, net.fc_n[2]))
    loss = lib().oracle_train_step_rows(ctypes.byref(net), _p(params, c_double),
                                        _p(velocity, c_double), xp, _p(labels, ctypes.c_int32),
                                        B, lr, momentum, wd, seed, step, row0,
                                        _p(grads, c_double), _p(logits, c_double))
    return loss, params, velocity, grads, logits


def train_step(net, params, velocity, x, labels, lr=0.01, momentum=0.9, wd=5e-4, seed=0,
               step=0, given_argmax=None, given_relu=None):
    """One step of [W] TRAIN_STEP.  Returns (loss, new_params, new_velocity,
    grads, logits).  given_argmax: optional {0|1|4: uint8 map} of pool window
    choices (for instance an implementation's own) used instead of the
    oracle's; given_relu: optional {0..4 conv, 5 FC6, 6 FC7: uint8 mask} of
    ReLU sign decisions used instead of the oracle's own (z > 0)."""
    params = np.array(params, dtype=np.float64, copy=True)
    velocity = np.array(velocity, dtype=np.float64, copy=True)
    x, xp = _d(x)
    labels = np.ascontiguousarray(labels, dtype=np.int32)
    B = x.shape[0]
    grads = np.zeros_like(params)
    logits = np.zeros((B, net.fc_n[2]))
    keep, ptrs = _am_ptrs(given_argmax)
    keep2, relu = _relu_ptrs(given_relu)
    loss = lib().oracle_train_step_given(ctypes.byref(net), _p(params, c_double),
                                         _p(velocity, c_double), xp, _p(labels, ctypes.c_int32),
                                         B, lr, momentum, wd, seed, step, _p(grads, c_double),
                                         _p(logits, c_double), *ptrs, relu)
    return loss, params, velocity, grads, logits


GPROBE_DZ, GPROBE_DPOOL, GPROBE_DLRN, GPROBE_DLOGITS, GPROBE_DZ7, GPROBE_DZ6 = 50, 60, 70, 80, 81, 82


def gprobe_size(net, which):
    """Elements per image of the gradient train_probe returns for `which`."""
    ms = map_sizes(net)
    if 50 <= which < 60 or 70 <= which < 80:
        l = which % 10
        return ms[l][1] ** 2 * net.conv_c[l]
    if 60 <= which < 70:
        l = which - 60
        return ms[l][2] ** 2 * net.conv_c[l]
    return {80: net.fc_n[2], 81: net.fc_n[1], 82: net.fc_n[0]}[which]


def _am_ptrs(given):
    """given: None or dict {0: am1, 1: am2, 4: am5} of uint8 window choices."""
    given = given or {}
    keep, ptrs = [], []
    for l in (0, 1, 4):
        a = given.get(l)
        if a is None:
            ptrs.append(None)
        else:
            a = np.ascontiguousarray(a, dtype=np.uint8)
            keep.append(a)
            ptrs.append(_p(a, c_uint8))
    return keep, ptrs


def _relu_ptrs(given):
    """given: None or dict {0..4: conv mask, 5: FC6 mask, 6: FC7 mask} (uint8)."""
    if not given:
        return [], None
    keep = []
    arr = (POINTER(c_uint8) * 7)()
    for i in range(7):
        a = given.get(i)
        if a is None:
            arr[i] = None
        else:
            a = np.ascontiguousarray(a, dtype=np.uint8)
            keep.append(a)
            arr[i] = _p(a, c_uint8)
    return keep, arr


def train_probe(net, params, x, labels, which, seed=0, step=0, given_argmax=None,
                given_relu=None):
    """One intermediate gradient of a training step (see oracle_train_probe), flat.
    given_argmax: optional {0|1|4: uint8 map} of pool window choices to use;
    given_relu: optional {0..4, 5, 6: uint8 mask} of ReLU sign decisions."""
    params, pp = _d(params)
    x, xp = _d(x)
    labels = np.ascontiguousarray(labels, dtype=np.int32)
    B = x.shape[0]
    out = np.zeros(B * gprobe_size(net, which))
    keep, ptrs = _am_ptrs(given_argmax)
    keep2, relu = _relu_ptrs(given_relu)
    lib().oracle_train_probe(ctypes.byref(net), pp, xp, _p(labels, ctypes.c_int32), B, seed, step,
                             which, _p(out, c_double), *ptrs, relu)
    return out


def maxpool_select(x, argmax, z=3, s=2):
    """Pooled map taking the given window choice (argmax) in every window."""
    x, xp = _d(x)
    argmax = np.ascontiguousarray(argmax, dtype=np.uint8)
    B, H, W, C = x.shape
    Ho, Wo = (H - z) // s + 1, (W - z) // s + 1
    y = np.zeros((B, Ho, Wo, C))
    lib().oracle_maxpool_select(xp, _p(argmax, c_uint8), B, H, W, C, z, s, _p(y, c_double))
    return y


def loss(net, params, x, labels, seed=0, step=0):
    params, pp = _d(params)
    x, xp = _d(x)
    labels = np.ascontiguousarray(labels, dtype=np.int32)
    return lib().oracle_loss(ctypes.byref(net), pp, xp, _p(labels, ctypes.c_int32), x.shape[0],
                             seed, step)


def augment(src, mean, pca_vec, pca_val, seed, step):
    """[S] 3.4 "Data Augmentation" Forms 1 and 2 -> [B, 227, 227, 3] fp64."""
    src = np.ascontiguousarray(src, dtype=np.uint8)
    B = src.shape[0]
    mean, mp = _d(mean)
    pv, pvp = _d(pca_vec)
    pl, plp = _d(pca_val)
    out = np.zeros((B, 227, 227, 3))
    lib().oracle_augment(_p(src, c_uint8), B, mp, pvp, plp, seed, step, _p(out, c_double))
    return out


def tencrop_inputs(src, mean):
    src = np.ascontiguousarray(src, dtype=np.uint8)
    B = src.shape[0]
    mean, mp = _d(mean)
    out = np.zeros((B * 10, 227, 227, 3))
    lib().oracle_tencrop_inputs(_p(src, c_uint8), B, mp, _p(out, c_double))
    return out


def tencrop(net, params, src, mean):
    """Ten-patch averaged probabilities and top-5 ([S] 3.4 "Data Augmentation")."""
    params, pp = _d(params)
    src = np.ascontiguousarray(src, dtype=np.uint8)
    B = src.shape[0]
    mean, mp = _d(mean)
    N = net.fc_n[2]
    probs = np.zeros((B, N))
    top5 = np.zeros((B, 5), np.int32)
    lib().oracle_tencrop(ctypes.byref(net), pp, _p(src, c_uint8), B, mp, _p(probs, c_double),
                         _p(top5, ctypes.c_int32))
    return probs, top5
