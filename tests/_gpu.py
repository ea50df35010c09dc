"""Helpers shared by the GPU tests: device buffers, bf16 round trips and the
error measures the tolerances are stated in."""
import numpy as np

TOL_BF16 = 2e-2   # relative L2 bound on the bf16 path (logits, gradients)
TOL_FP32 = 1e-4   # relative L2 bound on the fp32 path
TOL_OP = 1e-2     # one bf16 op on identical inputs: output rounding only


def torch():
    import torch as t
    return t


def dev(a, dtype=None):
    """numpy -> CUDA tensor (bf16 when dtype == 'bf16')."""
    t = torch()
    if dtype == "bf16":
        return t.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(t.bfloat16).cuda()
    return t.from_numpy(np.ascontiguousarray(a)).cuda()


def host(t_):
    t = torch()
    t.cuda.synchronize()
    if t_.dtype == t.bfloat16:
        return t_.float().cpu().numpy().astype(np.float64)
    return t_.cpu().numpy()


def bf16_round(a):
    """Values of `a` rounded to bf16 (torch's conversion), as float64."""
    t = torch()
    return t.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(t.bfloat16).to(
        t.float64).numpy()


def rel_l2(got, want):
    got = np.asarray(got, dtype=np.float64).ravel()
    want = np.asarray(want, dtype=np.float64).ravel()
    den = np.linalg.norm(want)
    return float(np.linalg.norm(got - want) / (den if den > 0 else 1.0))


def workspace(mb=512):
    t = torch()
    return t.empty(mb << 20, dtype=t.uint8, device="cuda")
