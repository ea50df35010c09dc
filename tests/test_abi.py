"""Host-side checks of the C-ABI library (no GPU needed): it loads, exports
every entry point the public headers declare, and its host logic (parameter
counts, workspace sizing, config validation) agrees with the oracle."""
import ctypes
import os
import re

import pytest

import oracle

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared():
    names = set()
    for h in ("alexnet.h", "alexnet_ops.h"):
        src = open(os.path.join(ROOT, "include", h)).read()
        names.update(re.findall(r"ALEXNET_API\s+[\w\s\*]+?\b(alexnet_\w+)\s*\(", src))
    return names


def test_library_exports_every_declared_symbol():
    from deep_cnn_image_b200 import alexnet as ax
    lib = ctypes.CDLL(ax.LIB_PATH)
    declared = _declared()
    assert len(declared) >= 30
    for name in declared:
        assert hasattr(lib, name), name
    # the binding wraps exactly the declared names
    assert set(ax.EXPORTED) == declared


def test_param_counts_match_oracle():
    from deep_cnn_image_b200 import alexnet as ax
    for grouped in (1, 0):
        cfg = ax.default_config(grouped=grouped)
        assert ax.param_count(cfg) == oracle.param_count(oracle.alexnet(grouped=bool(grouped)))


def test_workspace_sizing_and_validation():
    from deep_cnn_image_b200 import alexnet as ax
    cfg = ax.default_config()
    n = ax.workspace_bytes(cfg)
    # parameters + momentum alone are 8 bytes per parameter
    assert n > 8 * 60965224
    # larger batches need more workspace, fp32 inference less than bf16 training
    assert ax.workspace_bytes(ax.default_config(batch_max=512)) > n
    assert ax.workspace_bytes(ax.default_config(batch_max=1, dtype=ax.FP32, grouped=0)) > 0
    for bad in (dict(batch_max=0), dict(lrn_n=3), dict(pool_size=4), dict(dropout_p=1.0),
                dict(dtype=7)):
        assert ax.workspace_bytes(ax.default_config(**bad)) == 0
        assert ax.param_count(ax.default_config(**bad)) == -1


def test_invalid_arguments_return_before_any_launch():
    from deep_cnn_image_b200 import alexnet as ax
    lib = ax.lib
    h = ctypes.c_void_p()
    cfg = ax.default_config()
    # null workspace / undersized workspace / null out pointer
    assert lib.alexnet_create(ctypes.byref(cfg), None, 1 << 30, None, ctypes.byref(h)) == ax.ERR_INVALID_ARG
    assert lib.alexnet_create(ctypes.byref(cfg), 256, 16, None, ctypes.byref(h)) == ax.ERR_INVALID_ARG
    assert lib.alexnet_create(ctypes.byref(cfg), 256, 1 << 40, None, None) == ax.ERR_INVALID_ARG
    assert lib.alexnet_last_error(None)
    # calls on a NULL handle
    assert lib.alexnet_forward(None, 256, 1, 1, 256, None, None) == ax.ERR_INVALID_ARG
    assert lib.alexnet_train_step(None, 256, 256, 1, 0.01, None, None) == ax.ERR_INVALID_ARG
    assert lib.alexnet_destroy(None) == ax.OK
    # op argument checks
    assert lib.alexnet_op_lrn_fwd(None, 10, 96, 2.0, 1e-4, 0.75, None, None) == ax.ERR_INVALID_ARG
    assert lib.alexnet_op_pool_fwd(256, 1, 2, 2, 8, 3, 2, 256, 256, None) == ax.ERR_INVALID_ARG
    assert lib.alexnet_op_fc_wgrad(256, 256, 1, 8, 60, 256, 256, 1024, None) == ax.ERR_INVALID_ARG
