"""ctypes binding of libalexnet.so (include/alexnet.h, include/alexnet_ops.h).

Argument marshalling only: every computation runs in the library's CUDA
kernels.  Tensors are torch tensors (their data pointers are passed); streams
default to torch's current CUDA stream.  Importing this module loads the
library and raises if it is missing: there is no fallback.
"""
from __future__ import annotations

import ctypes
import os
from ctypes import POINTER, byref, c_float, c_int, c_int64, c_size_t, c_uint32, c_uint64, c_void_p

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libalexnet.so")

OK, ERR_INVALID_ARG, ERR_UNSUPPORTED, ERR_CUDA, ERR_TIMEOUT, ERR_LABEL_RANGE = range(6)
FP32, BF16 = 0, 1
TRAIN, INFERENCE = 0, 1
STATUS_NAMES = {0: "OK", 1: "INVALID_ARG", 2: "UNSUPPORTED", 3: "CUDA", 4: "TIMEOUT",
                5: "LABEL_RANGE"}


class Config(ctypes.Structure):
    """alexnet_config."""
    _fields_ = [
        ("batch_max", c_int), ("dtype", c_int), ("grouped", c_int), ("seed", c_uint64),
        ("momentum", c_float), ("weight_decay", c_float), ("dropout_p", c_float),
        ("lrn_k", c_float), ("lrn_alpha", c_float), ("lrn_beta", c_float), ("lrn_n", c_int),
        ("lrn_on", c_int), ("pool_size", c_int), ("dropout_on", c_int), ("keep_grads", c_int),
    ]


class Stats(ctypes.Structure):
    """alexnet_stats."""
    _fields_ = [("launches", ctypes.c_int64), ("gemm_launches", ctypes.c_int64),
                ("gemm_flops", ctypes.c_double), ("gemm_ms", ctypes.c_double)]


class AlexNetError(RuntimeError):
    def __init__(self, status, msg=""):
        super().__init__("alexnet status %s: %s" % (STATUS_NAMES.get(status, status), msg))
        self.status = status


def _load():
    if not os.path.exists(LIB_PATH):
        raise ImportError("libalexnet.so is not built (python -m deep_cnn_image_b200.build)")
    L = ctypes.CDLL(LIB_PATH)
    vp, st, i, sz = c_void_p, c_int, c_int, c_size_t
    cfgp = POINTER(Config)
    sig = {
        "alexnet_default_config": (None, [cfgp]),
        "alexnet_param_count": (c_int64, [cfgp]),
        "alexnet_workspace_bytes": (sz, [cfgp]),
        "alexnet_create": (st, [cfgp, vp, sz, vp, POINTER(vp)]),
        "alexnet_forward": (st, [vp, vp, i, i, vp, vp, vp]),
        "alexnet_train_step": (st, [vp, vp, vp, i, c_float, vp, vp]),
        "alexnet_augment": (st, [vp, vp, i, vp, vp, vp, vp, vp]),
        "alexnet_tencrop": (st, [vp, vp, i, vp, vp, vp, vp]),
        "alexnet_ensemble_workspace_bytes": (sz, [i, i]),
        "alexnet_knn_workspace_bytes": (sz, [i, i]),
        "alexnet_knn": (st, [vp, i, vp, i, i, i, vp, vp, vp, vp, sz, vp]),
        "alexnet_knn_sqnorms": (st, [vp, i, i, vp, vp]),
        "alexnet_ensemble_forward": (st, [vp, i, vp, i, vp, vp, vp, sz, vp]),
        "alexnet_train_grads": (st, [vp, vp, vp, i, c_int64, vp, vp]),
        "alexnet_stream_wait_fc_grads": (st, [vp, vp]),
        "alexnet_sgd_range": (st, [vp, c_int64, c_int64, vp, c_float, c_float, vp]),
        "alexnet_params_updated": (st, [vp, vp]),
        "alexnet_device_buffer": (st, [vp, i, POINTER(vp), POINTER(c_int64)]),
        "alexnet_params_bytes": (sz, [vp]),
        "alexnet_get_params": (st, [vp, vp, sz, vp]),
        "alexnet_set_params": (st, [vp, vp, sz, vp]),
        "alexnet_get_grads": (st, [vp, vp, sz, vp]),
        "alexnet_get_status": (st, [vp]),
        "alexnet_last_error": (ctypes.c_char_p, [vp]),
        "alexnet_destroy": (st, [vp]),
        "alexnet_op_conv_fwd": (st, [vp, i, i, i, i, vp, vp, i, i, i, i, i, vp, vp, sz, vp]),
        "alexnet_op_conv1_fwd": (st, [vp, i, vp, vp, vp, vp, sz, vp]),
        "alexnet_op_conv_dgrad": (st, [vp, i, i, i, i, vp, i, i, i, i, vp, vp, vp, sz, vp]),
        "alexnet_op_conv_wgrad": (st, [vp, i, i, i, i, vp, i, i, i, i, i, vp, vp, sz, vp]),
        "alexnet_op_conv1_wgrad": (st, [vp, i, vp, i, vp, vp, sz, vp]),
        "alexnet_op_conv_wgrad_noalloc": (st, [vp, i, i, i, i, vp, i, i, i, i, i, vp, vp]),
        "alexnet_op_fc_fwd": (st, [vp, i, i, vp, i, i, vp, vp, sz, vp]),
        "alexnet_op_fc_dgrad": (st, [vp, i, i, vp, i, i, vp, vp, sz, vp]),
        "alexnet_op_fc_wgrad": (st, [vp, vp, i, i, i, vp, vp, sz, vp]),
        "alexnet_op_lrn_fwd": (st, [vp, c_int64, i, c_float, c_float, c_float, vp, vp]),
        "alexnet_op_lrn_bwd": (st, [vp, vp, c_int64, i, c_float, c_float, c_float, vp, vp]),
        "alexnet_op_pool_fwd": (st, [vp, i, i, i, i, i, i, vp, vp, vp]),
        "alexnet_op_pool_bwd": (st, [vp, vp, vp, i, i, i, i, i, i, i, vp, vp]),
        "alexnet_op_lrn_pool_fwd": (st, [vp, i, i, i, i, i, c_float, c_float, c_float, vp, vp, vp,
                                         vp]),
        "alexnet_op_pool_lrn_bwd": (st, [vp, vp, vp, i, i, i, i, i, c_float, c_float, c_float, vp,
                                         vp, vp]),
        "alexnet_op_softmax_ce": (st, [vp, vp, i, i, vp, vp, vp, vp, sz, vp]),
        "alexnet_op_dropout_mask": (st, [c_uint64, c_uint32, c_uint32, c_float, i, i, vp, vp, sz,
                                         vp]),
        "alexnet_op_philox": (st, [vp, vp, i, vp, vp]),
        "alexnet_op_wait_probe": (st, [vp, c_int64, vp]),
        "alexnet_debug_copy": (st, [vp, i, vp, sz, vp]),
        "alexnet_debug_keep": (st, [vp, i]),
        "alexnet_debug_fc_update": (st, [vp, i]),
        "alexnet_debug_overlap": (st, [vp, i]),
        "alexnet_debug_canaries": (st, [vp, POINTER(c_int64)]),
        "alexnet_conv_algo": (st, [vp, i, i, i, POINTER(c_int)]),
        "alexnet_stats_enable": (st, [vp, i]),
        "alexnet_stats_read": (st, [vp, POINTER(Stats)]),
        "alexnet_stats_launch": (st, [vp, i, POINTER(c_int), POINTER(ctypes.c_double),
                                      POINTER(ctypes.c_double)]),
    }
    for name, (res, args) in sig.items():
        f = getattr(L, name)
        f.restype = res
        f.argtypes = args
    return L, sorted(sig)


lib, EXPORTED = _load()


def _ptr(t):
    if t is None:
        return None
    if isinstance(t, int):
        return t
    return t.data_ptr()


def _stream(stream):
    if stream is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def check(status, handle=None):
    if status != OK:
        msg = lib.alexnet_last_error(handle)
        raise AlexNetError(status, msg.decode() if msg else "")
    return status


def default_config(**overrides) -> Config:
    c = Config()
    lib.alexnet_default_config(ctypes.byref(c))
    for k, v in overrides.items():
        setattr(c, k, v)
    return c


def param_count(cfg: Config) -> int:
    return lib.alexnet_param_count(ctypes.byref(cfg))


def workspace_bytes(cfg: Config) -> int:
    return lib.alexnet_workspace_bytes(ctypes.byref(cfg))


class AlexNet:
    """Owns a handle; the workspace is a torch uint8 CUDA tensor it keeps alive."""

    def __init__(self, cfg: Config | None = None, stream=None, **overrides):
        import torch
        self.cfg = cfg if cfg is not None else default_config(**overrides)
        nbytes = workspace_bytes(self.cfg)
        if nbytes == 0:
            raise AlexNetError(ERR_INVALID_ARG, "invalid config")
        self.workspace = torch.empty(nbytes + 256, dtype=torch.uint8, device="cuda")
        base = self.workspace.data_ptr()
        aligned = (base + 255) & ~255
        h = c_void_p()
        check(lib.alexnet_create(ctypes.byref(self.cfg), aligned, nbytes, _stream(stream),
                                 ctypes.byref(h)))
        self.h = h

    def close(self):
        # at interpreter exit the module globals may already be gone
        if getattr(self, "h", None) and lib is not None:
            lib.alexnet_destroy(self.h)
            self.h = None

    def __del__(self):
        self.close()

    # -- the C calls, same names ------------------------------------------
    def forward(self, x, B, mode, logits, probs=None, stream=None):
        return check(lib.alexnet_forward(self.h, _ptr(x), B, mode, _ptr(logits), _ptr(probs),
                                         _stream(stream)), self.h)

    def train_step(self, x, labels, B, lr, loss=None, stream=None):
        return check(lib.alexnet_train_step(self.h, _ptr(x), _ptr(labels), B, lr, _ptr(loss),
                                            _stream(stream)), self.h)

    def augment(self, src, B, mean, pca_vec, pca_val, x_out, stream=None):
        return check(lib.alexnet_augment(self.h, _ptr(src), B, _ptr(mean), _ptr(pca_vec),
                                         _ptr(pca_val), _ptr(x_out), _stream(stream)), self.h)

    def tencrop(self, src, B, mean, probs_avg, top5, stream=None):
        return check(lib.alexnet_tencrop(self.h, _ptr(src), B, _ptr(mean), _ptr(probs_avg),
                                         _ptr(top5), _stream(stream)), self.h)

    # -- data-parallel step (see alexnet.h) ------------------------------
    def train_grads(self, x, labels, B, image_offset, loss=None, stream=None):
        return check(lib.alexnet_train_grads(self.h, _ptr(x), _ptr(labels), B, image_offset,
                                             _ptr(loss), _stream(stream)), self.h)

    def stream_wait_fc_grads(self, stream):
        return check(lib.alexnet_stream_wait_fc_grads(self.h, _stream(stream)), self.h)

    def sgd_range(self, offset, count, gsum, grad_scale, lr, stream=None):
        return check(lib.alexnet_sgd_range(self.h, offset, count, _ptr(gsum), grad_scale, lr,
                                           _stream(stream)), self.h)

    def params_updated(self, stream=None):
        return check(lib.alexnet_params_updated(self.h, _stream(stream)), self.h)

    def device_buffer(self, which):
        """The handle's fp32 parameters (0), momentum (1) or gradients (2) as
        a torch view of the workspace (blob order)."""
        import torch
        p = c_void_p()
        n = c_int64()
        check(lib.alexnet_device_buffer(self.h, which, byref(p), byref(n)), self.h)
        off = p.value - self.workspace.data_ptr()
        return self.workspace[off:off + 4 * n.value].view(torch.float32)

    def params_bytes(self):
        return lib.alexnet_params_bytes(self.h)

    def get_params(self, dst, stream=None):
        return check(lib.alexnet_get_params(self.h, _ptr(dst), dst.numel() * dst.element_size(),
                                            _stream(stream)), self.h)

    def set_params(self, src, stream=None):
        return check(lib.alexnet_set_params(self.h, _ptr(src), src.numel() * src.element_size(),
                                            _stream(stream)), self.h)

    def get_grads(self, dst, stream=None):
        return check(lib.alexnet_get_grads(self.h, _ptr(dst), dst.numel(), _stream(stream)), self.h)

    def get_status(self):
        return lib.alexnet_get_status(self.h)

    def stats_enable(self, enable=True):
        return check(lib.alexnet_stats_enable(self.h, 1 if enable else 0), self.h)

    def stats_read(self):
        st_ = Stats()
        check(lib.alexnet_stats_read(self.h, ctypes.byref(st_)), self.h)
        return {"launches": st_.launches, "gemm_launches": st_.gemm_launches,
                "gemm_flops": st_.gemm_flops, "gemm_ms": st_.gemm_ms}

    def stats_launches(self):
        """(kind, flops, ms) of every GEMM launch stats_read reports: kind 0
        a convolution, 1 an FC forward or data gradient, 2 an FC weight
        gradient written to memory."""
        out = []
        k, f, m = c_int(), ctypes.c_double(), ctypes.c_double()
        for idx in range(self.stats_read()["gemm_launches"]):
            check(lib.alexnet_stats_launch(self.h, idx, ctypes.byref(k), ctypes.byref(f),
                                           ctypes.byref(m)), self.h)
            out.append((k.value, f.value, m.value))
        return out

    def conv_algo(self, batch, layer, pass_):
        """1 if convolution `layer` runs the shifted-box kernel for this batch
        size in pass 0 (forward), 1 (data gradient) or 2 (weight gradient)."""
        v = c_int(-1)
        check(lib.alexnet_conv_algo(self.h, batch, layer, pass_, byref(v)))
        return v.value

    def debug_keep(self, keep=True):
        """Also store the normalised maps and their gradients (debug_copy
        10/11, 70/71) in later calls."""
        return check(lib.alexnet_debug_keep(self.h, 1 if keep else 0))

    def debug_overlap(self, on=True):
        """Weight gradients on a second stream beside the data gradients (default on)."""
        return check(lib.alexnet_debug_overlap(self.h, 1 if on else 0))

    def debug_fc_update(self, fused=True):
        """FC weights updated by the weight-gradient GEMM's epilogue (True,
        the default) or by a separate kernel (False); identical results."""
        return check(lib.alexnet_debug_fc_update(self.h, 1 if fused else 0))

    def debug_canaries(self):
        """Bytes changed in the guard regions after the workspace's buffers
        (0 unless some kernel wrote past the end of a buffer); synchronises."""
        v = c_int64(-1)
        check(lib.alexnet_debug_canaries(self.h, byref(v)), self.h)
        return v.value

    def debug_copy(self, which, dst, stream=None):
        return check(lib.alexnet_debug_copy(self.h, which, _ptr(dst), dst.numel() * dst.element_size(),
                                            _stream(stream)), self.h)


# -- single-op entry points (alexnet_ops.h), same names ------------------------
def _op(name, *args):
    return check(getattr(lib, name)(*args))


def op_conv_fwd(x, B, H, W, Cin, w, bias, Cout, K, pad, groups, relu, y, ws, stream=None):
    return _op("alexnet_op_conv_fwd", _ptr(x), B, H, W, Cin, _ptr(w), _ptr(bias), Cout, K, pad,
               groups, relu, _ptr(y), _ptr(ws), ws.numel(), _stream(stream))


def op_conv1_fwd(x, B, w, bias, y, ws, stream=None):
    return _op("alexnet_op_conv1_fwd", _ptr(x), B, _ptr(w), _ptr(bias), _ptr(y), _ptr(ws),
               ws.numel(), _stream(stream))


def op_conv_dgrad(dy, B, H, W, Cin, w, Cout, K, pad, groups, mask, dx, ws, stream=None):
    return _op("alexnet_op_conv_dgrad", _ptr(dy), B, H, W, Cin, _ptr(w), Cout, K, pad, groups,
               _ptr(mask), _ptr(dx), _ptr(ws), ws.numel(), _stream(stream))


def op_conv_wgrad(x, B, H, W, Cin, dy, Cout, K, pad, groups, splits, dw, ws, stream=None):
    return _op("alexnet_op_conv_wgrad", _ptr(x), B, H, W, Cin, _ptr(dy), Cout, K, pad, groups,
               splits, _ptr(dw), _ptr(ws), ws.numel(), _stream(stream))


def op_conv_wgrad_noalloc(x, B, H, W, Cin, dy, Cout, K, pad, groups, splits, dw, stream=None):
    """alexnet_op_conv_wgrad without scratch: for callers that can neither pass
    scratch memory nor let the library allocate (see alexnet_ops.h)."""
    return _op("alexnet_op_conv_wgrad_noalloc", _ptr(x), B, H, W, Cin, _ptr(dy), Cout, K, pad,
               groups, splits, _ptr(dw), _stream(stream))


def op_conv1_wgrad(x, B, dy, splits, dw, ws, stream=None):
    return _op("alexnet_op_conv1_wgrad", _ptr(x), B, _ptr(dy), splits, _ptr(dw), _ptr(ws),
               ws.numel(), _stream(stream))


def op_fc_fwd(x, B, In, w, Out, splits, y, ws, stream=None):
    return _op("alexnet_op_fc_fwd", _ptr(x), B, In, _ptr(w), Out, splits, _ptr(y), _ptr(ws),
               ws.numel(), _stream(stream))


def op_fc_dgrad(dz, B, Out, w, In, splits, dx, ws, stream=None):
    return _op("alexnet_op_fc_dgrad", _ptr(dz), B, Out, _ptr(w), In, splits, _ptr(dx), _ptr(ws),
               ws.numel(), _stream(stream))


def op_fc_wgrad(dz, x, B, Out, In, dw, ws, stream=None):
    return _op("alexnet_op_fc_wgrad", _ptr(dz), _ptr(x), B, Out, In, _ptr(dw), _ptr(ws),
               ws.numel(), _stream(stream))


def op_lrn_fwd(a, P, C, k, alpha, beta, b, stream=None):
    return _op("alexnet_op_lrn_fwd", _ptr(a), P, C, k, alpha, beta, _ptr(b), _stream(stream))


def op_lrn_bwd(a, g, P, C, k, alpha, beta, da, stream=None):
    return _op("alexnet_op_lrn_bwd", _ptr(a), _ptr(g), P, C, k, alpha, beta, _ptr(da),
               _stream(stream))


def op_pool_fwd(x, B, H, W, C, z, st, y, argmax, stream=None):
    return _op("alexnet_op_pool_fwd", _ptr(x), B, H, W, C, z, st, _ptr(y), _ptr(argmax),
               _stream(stream))


def op_pool_bwd(dy, argmax, pooled, B, H, W, C, z, st, relu_mask, dx, stream=None):
    return _op("alexnet_op_pool_bwd", _ptr(dy), _ptr(argmax), _ptr(pooled), B, H, W, C, z, st,
               relu_mask, _ptr(dx), _stream(stream))


def op_lrn_pool_fwd(a, B, H, W, C, z, k, alpha, beta, lo, y, argmax, stream=None):
    return _op("alexnet_op_lrn_pool_fwd", _ptr(a), B, H, W, C, z, k, alpha, beta, _ptr(lo),
               _ptr(y), _ptr(argmax), _stream(stream))


def op_pool_lrn_bwd(dy, argmax, a, B, H, W, C, z, k, alpha, beta, dl, da, stream=None):
    return _op("alexnet_op_pool_lrn_bwd", _ptr(dy), _ptr(argmax), _ptr(a), B, H, W, C, z, k,
               alpha, beta, _ptr(dl), _ptr(da), _stream(stream))


def op_softmax_ce(logits, labels, B, N, probs, dlogits, loss, ws, stream=None):
    return _op("alexnet_op_softmax_ce", _ptr(logits), _ptr(labels), B, N, _ptr(probs),
               _ptr(dlogits), _ptr(loss), _ptr(ws), ws.numel(), _stream(stream))


def ensemble_workspace_bytes(n_models, B):
    return lib.alexnet_ensemble_workspace_bytes(n_models, B)


def ensemble_forward(nets, x, B, probs_avg, top5, ws, stream=None):
    """Mean of the softmax outputs of several networks on one batch (and its
    top 5); ws: a device byte tensor of ensemble_workspace_bytes(len(nets), B)."""
    arr = (c_void_p * len(nets))(*[n.h for n in nets])
    return _op("alexnet_ensemble_forward", arr, len(nets), _ptr(x), B, _ptr(probs_avg),
               _ptr(top5), _ptr(ws), ws.numel() * ws.element_size(), _stream(stream))


def knn_workspace_bytes(Q, N):
    return lib.alexnet_knn_workspace_bytes(Q, N)


def knn(queries, base, k, dist, idx, ws, base_sqnorm=None, stream=None):
    """k nearest base rows (squared Euclidean distance) of every query row;
    queries [Q, D] and base [N, D] bf16 on the device; base_sqnorm: the base
    rows' squared norms (knn_sqnorms), computed per call when None."""
    Q, D = queries.shape
    N = base.shape[0]
    return _op("alexnet_knn", _ptr(queries), Q, _ptr(base), N, D, k, _ptr(base_sqnorm),
               _ptr(dist), _ptr(idx), _ptr(ws), ws.numel() * ws.element_size(), _stream(stream))


def knn_sqnorms(x, out, stream=None):
    rows, D = x.shape
    return _op("alexnet_knn_sqnorms", _ptr(x), rows, D, _ptr(out), _stream(stream))


def op_wait_probe(status, limit_cycles, stream=None):
    """A bounded device wait that nothing completes: sets the TIMEOUT bit of
    the int32 device tensor `status` after limit_cycles clocks."""
    return _op("alexnet_op_wait_probe", _ptr(status), limit_cycles, _stream(stream))


def op_dropout_mask(seed, layer, step, p, rows, cols, keep, ws, stream=None):
    return _op("alexnet_op_dropout_mask", seed, layer, step, p, rows, cols, _ptr(keep), _ptr(ws),
               ws.numel(), _stream(stream))


def op_philox(ctr, key, n, out, stream=None):
    return _op("alexnet_op_philox", _ptr(ctr), _ptr(key), n, _ptr(out), _stream(stream))
