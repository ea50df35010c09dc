"""Seeded synthetic inputs shared by the CUDA library's tests, the oracle's
tests and the benchmark.

This module holds no arithmetic of the method itself: it only draws random
numbers (numpy's PCG64 generator, seeded) in the shapes and distributions of
the workloads, and rounds them to bf16 with torch's own conversion.  ImageNet
is not available, so these draws stand in for it:

* network inputs x ~ N(0, 1), [B, 227, 227, 3] NHWC;
* labels uniform in [0, 1000);
* source images for augmentation: uint8 uniform in [0, 255], [B, 256, 256, 3];
  their per-pixel mean image is the fp32 mean over the drawn pool;
* an RGB covariance C = A A^T / 3 + 0.1 I with A ~ N(0, 1) (3 x 3), and its
  eigen-pairs from numpy's symmetric eigensolver (fp64), passed to both sides;
* parameters: weights ~ N(0, 0.01^2); biases 1 on conv2, conv4, conv5, FC6,
  FC7 and 0 on conv1, conv3, FC8 (the initialisation the pages state).
"""
from __future__ import annotations

import numpy as np

# (Cout, k, Cin_per_group) of the five convolutions and (out, in) of the FC
# layers, for the grouped and ungrouped network on a 227 x 227 x 3 input.
CONV_SHAPES = {
    True: [(96, 11, 3), (256, 5, 48), (384, 3, 256), (384, 3, 192), (256, 3, 192)],
    False: [(96, 11, 3), (256, 5, 96), (384, 3, 256), (384, 3, 384), (256, 3, 384)],
}
FC_SHAPES = [(4096, 9216), (4096, 4096), (1000, 4096)]
BIAS_ONE = [False, True, False, True, True, True, True, False]


def rng(seed: int) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(seed))


def param_shapes(grouped: bool = True):
    """[(weight shape, bias length)] of the 8 learned layers, canonical order."""
    out = [((co, k, k, ci), co) for (co, k, ci) in CONV_SHAPES[grouped]]
    out += [((o, i), o) for (o, i) in FC_SHAPES]
    return out


def param_count(grouped: bool = True) -> int:
    return sum(int(np.prod(w)) + b for w, b in param_shapes(grouped))


def params(seed: int, grouped: bool = True, std: float = 0.01) -> np.ndarray:
    """Flat fp32 parameter blob: W1 b1 W2 b2 ... W8 b8."""
    g = rng(seed)
    parts = []
    for l, (ws, bl) in enumerate(param_shapes(grouped)):
        parts.append((g.standard_normal(int(np.prod(ws))) * std).astype(np.float32))
        parts.append(np.full(bl, 1.0 if BIAS_ONE[l] else 0.0, np.float32))
    return np.concatenate(parts)


def images(seed: int, B: int, hw: int = 227) -> np.ndarray:
    return rng(seed).standard_normal((B, hw, hw, 3), dtype=np.float32)


def labels(seed: int, B: int, classes: int = 1000) -> np.ndarray:
    return rng(seed).integers(0, classes, size=B, dtype=np.int32)


def source_images(seed: int, B: int) -> np.ndarray:
    return rng(seed).integers(0, 256, size=(B, 256, 256, 3), dtype=np.uint8)


def mean_image(src: np.ndarray) -> np.ndarray:
    return src.astype(np.float64).mean(axis=0).astype(np.float32)


def pca(seed: int):
    """(eigenvectors as columns [3,3] fp32, eigenvalues [3] fp32)."""
    A = rng(seed).standard_normal((3, 3))
    C = A @ A.T / 3.0 + 0.1 * np.eye(3)
    val, vec = np.linalg.eigh(C)
    return vec.astype(np.float32), val.astype(np.float32)


def to_bf16(x: np.ndarray):
    """Round fp32 values to bf16 (torch's round-to-nearest-even conversion).
    Returns (bf16 torch tensor, the rounded values as float64 numpy)."""
    import torch
    t = torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32)).to(torch.bfloat16)
    return t, t.to(torch.float64).numpy()
