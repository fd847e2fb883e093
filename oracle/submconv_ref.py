"""Python CPU oracle for SubMConv3d (test infrastructure only).

Written from the trellis_sparse_mlx README:

* "What's in it" -- SubMConv3d is the submanifold 3x3x3 (and 1x1x1) sparse
  convolution over a SparseTensor of coords [N, 4] = (b, x, y, z) and feats
  [N, C]; the output has exactly the input's coordinates.
* "Correctness" -- the convention is cross-correlation: the output at voxel c
  sums feats[c + d] @ W[d] over the kernel offsets d, over active neighbours
  only; this oracle is the "deliberately naive" form that section describes
  (a dict lookup and a per-voxel loop).

Readings where the pages are silent:

* tap order: for K = 3, k = 9 (dx + 1) + 3 (dy + 1) + (dz + 1), x slowest;
  for general odd K the same mixed-radix order with radius K // 2;
* neighbours are looked up at c + stride * d (stride = 1 in every workload);
* a missing neighbour is written as -1 in the neighbour map;
* voxels of different batch index b are never neighbours;
* duplicate coordinates are an error.

Every value is accumulated in float64 from inputs that were already rounded
to the workload dtype, so the result is the exact sum for those inputs up to
float64 rounding.  ``scale`` is sum_d |feats[c+d]| @ |W[d]|, the magnitude
the tolerance of the half-precision comparison is measured against.

Pins (tests/test_oracle_pins.py): dense conv3d on a zero-filled grid with
outputs taken at active sites (brute force), K = 1 equals a Linear layer, an
isolated voxel gives feats @ W[centre], a hand-worked two-voxel case
(tests/golden/hand_worked.json) that separates c + d from c - d, and
neighbour-map invariants (centre tap is the voxel itself, symmetry).
"""
from __future__ import annotations

import numpy as np


def tap_offsets(K: int) -> list:
    """Kernel offsets d = (dx, dy, dz) in tap order (x slowest)."""
    if K < 1 or K % 2 == 0:
        raise ValueError("kernel size must be odd and positive")
    r = K // 2
    return [(dx, dy, dz)
            for dx in range(-r, r + 1)
            for dy in range(-r, r + 1)
            for dz in range(-r, r + 1)]


def coord_dict(coords) -> dict:
    """(b, x, y, z) -> row index; duplicate coordinates raise ValueError."""
    table = {}
    for i, row in enumerate(np.asarray(coords).tolist()):
        key = tuple(int(v) for v in row)
        if key in table:
            raise ValueError(f"duplicate coordinate {key} at rows {table[key]} and {i}")
        table[key] = i
    return table


def neighbor_map(coords, K: int = 3, stride: int = 1) -> np.ndarray:
    """int64 [N, K^3]: entry (i, k) is the row j with coords[j] = coords[i] +
    stride * d_k in the same batch, or -1 when that site is not active."""
    table = coord_dict(coords)
    offs = tap_offsets(K)
    rows = np.asarray(coords).tolist()
    out = np.full((len(rows), len(offs)), -1, dtype=np.int64)
    for i, (b, x, y, z) in enumerate(rows):
        for k, (dx, dy, dz) in enumerate(offs):
            j = table.get((b, x + stride * dx, y + stride * dy, z + stride * dz))
            if j is not None:
                out[i, k] = j
    return out


def submconv(coords, feats, W, K: int = 3, stride: int = 1, nbr=None):
    """Submanifold convolution, output sites = input sites.

    feats: [N, Cin] (any float type; widened to float64), W: [K^3, Cin, Cout].
    Returns (out, scale), both float64 [N, Cout].
    """
    f = np.asarray(feats, dtype=np.float64)
    w = np.asarray(W, dtype=np.float64)
    if w.shape[0] != K ** 3 or w.shape[1] != f.shape[1]:
        raise ValueError("weight shape does not match K and Cin")
    if nbr is None:
        nbr = neighbor_map(coords, K, stride)
    n, cout = f.shape[0], w.shape[2]
    out = np.zeros((n, cout), dtype=np.float64)
    scale = np.zeros((n, cout), dtype=np.float64)
    aw = np.abs(w)
    for i in range(n):
        acc = np.zeros(cout, dtype=np.float64)
        mag = np.zeros(cout, dtype=np.float64)
        for k in range(K ** 3):
            j = nbr[i, k]
            if j < 0:
                continue
            acc += f[j] @ w[k]
            mag += np.abs(f[j]) @ aw[k]
        out[i] = acc
        scale[i] = mag
    return out, scale


# ----------------------------------------------------------------------------
# Backward passes ("Metal-native replacement for flex_gemm bottleneck?",
# "Fixed" / "Open": fwd / bwd-input / bwd-weight, each with its own parity).
# The forward map is linear in feats and in W; these are its two adjoints,
# written straight from the forward sum: every term feats[j] @ W[k] that the
# forward adds to out[i] (j = nbr[i, k]) sends grad_out[i] @ W[k]^T back to
# feats[j] and outer(feats[j], grad_out[i]) to W[k].
# ----------------------------------------------------------------------------
def submconv_backward_input(coords, grad_out, W, K: int = 3, stride: int = 1, nbr=None):
    """grad_feats float64 [N, Cin] and its error scale (the same sum over
    |grad_out[i]| @ |W[k]|^T), for loss gradient grad_out [N, Cout]."""
    g = np.asarray(grad_out, dtype=np.float64)
    w = np.asarray(W, dtype=np.float64)
    if nbr is None:
        nbr = neighbor_map(coords, K, stride)
    n, cin = g.shape[0], w.shape[1]
    gin = np.zeros((n, cin), dtype=np.float64)
    scale = np.zeros((n, cin), dtype=np.float64)
    aw = np.abs(w)
    for i in range(n):
        for k in range(K ** 3):
            j = nbr[i, k]
            if j < 0:
                continue
            gin[j] += w[k] @ g[i]
            scale[j] += aw[k] @ np.abs(g[i])
    return gin, scale


def submconv_backward_weight(coords, feats, grad_out, K: int = 3, stride: int = 1, nbr=None):
    """dW float64 [K^3, Cin, Cout] and its error scale (the same sum of
    outer(|feats[j]|, |grad_out[i]|))."""
    f = np.asarray(feats, dtype=np.float64)
    g = np.asarray(grad_out, dtype=np.float64)
    if nbr is None:
        nbr = neighbor_map(coords, K, stride)
    taps = K ** 3
    dW = np.zeros((taps, f.shape[1], g.shape[1]), dtype=np.float64)
    scale = np.zeros_like(dW)
    for i in range(f.shape[0]):
        for k in range(taps):
            j = nbr[i, k]
            if j < 0:
                continue
            dW[k] += np.outer(f[j], g[i])
            scale[k] += np.outer(np.abs(f[j]), np.abs(g[i]))
    return dW, scale


# ----------------------------------------------------------------------------
# x2 coordinate ops (trellis_sparse_mlx README, "What's in it": subdivide /
# downsample -- x2 coordinate expansion; x2 max-pool, upstream passing
# reduce="amax" although its docstring says "average").
# Readings: the parent of (b, x, y, z) is (b, x // 2, y // 2, z // 2); the
# downsampled tensor lists each parent once, in lexicographic (b, x, y, z)
# order (batch-contiguous, like every SparseTensor here), with the element-wise
# maximum of its children's rows; subdivision gives every voxel its 8 children
# (b, 2x + dx, 2y + dy, 2z + dz), child c = 4 dx + 2 dy + dz, parents in input
# order, each child carrying its parent's row.
# ----------------------------------------------------------------------------
def downsample2(coords, feats):
    """(parent coords int32 [M, 4], float64 feats [M, C]) of the x2 max-pool."""
    f = np.asarray(feats, dtype=np.float64)
    groups = {}
    for i, (b, x, y, z) in enumerate(np.asarray(coords).tolist()):
        groups.setdefault((b, x // 2, y // 2, z // 2), []).append(i)
    keys = sorted(groups)
    out_c = np.array(keys, dtype=np.int32).reshape(-1, 4)
    out_f = np.zeros((len(keys), f.shape[1]), dtype=np.float64)
    for p, key in enumerate(keys):
        rows = groups[key]
        acc = f[rows[0]].copy()
        for r in rows[1:]:
            acc = np.maximum(acc, f[r])
        out_f[p] = acc
    return out_c, out_f


def subdivide2(coords, feats):
    """(child coords int32 [8N, 4], float64 feats [8N, C]) of the x2 expansion."""
    f = np.asarray(feats, dtype=np.float64)
    rows = np.asarray(coords).tolist()
    out_c = np.zeros((8 * len(rows), 4), dtype=np.int32)
    out_f = np.zeros((8 * len(rows), f.shape[1]), dtype=np.float64)
    for i, (b, x, y, z) in enumerate(rows):
        for dx in (0, 1):
            for dy in (0, 1):
                for dz in (0, 1):
                    c = 8 * i + 4 * dx + 2 * dy + dz
                    out_c[c] = (b, 2 * x + dx, 2 * y + dy, 2 * z + dz)
                    out_f[c] = f[i]
    return out_c, out_f


# ----------------------------------------------------------------------------
# Fused epilogue of a convolution layer inside a sparse ResBlock
# (trellis_sparse_mlx README, "What's in it": SparseLinear, SparseSiLU/GELU,
# SparseResBlock).  Reading: out = act(conv + bias) + residual, every term
# optional; SiLU(v) = v / (1 + exp(-v)); GELU is the exact (erf) form,
# v / 2 * (1 + erf(v / sqrt(2))); ReLU(v) = max(v, 0).
# ----------------------------------------------------------------------------
ACTIVATIONS = ("none", "relu", "silu", "gelu")


def activation(v: np.ndarray, act: str) -> np.ndarray:
    v = np.asarray(v, dtype=np.float64)
    if act == "none":
        return v
    if act == "relu":
        return np.maximum(v, 0.0)
    if act == "silu":
        return v / (1.0 + np.exp(-v))
    if act == "gelu":
        from math import erf, sqrt
        return 0.5 * v * (1.0 + np.vectorize(erf)(v / sqrt(2.0)))
    raise ValueError(act)


def epilogue(conv_out, bias=None, act: str = "none", residual=None) -> np.ndarray:
    """act(conv_out + bias) + residual in float64 (bias [Cout], residual [N, Cout])."""
    v = np.asarray(conv_out, dtype=np.float64)
    if bias is not None:
        v = v + np.asarray(bias, dtype=np.float64)[None, :]
    v = activation(v, act)
    if residual is not None:
        v = v + np.asarray(residual, dtype=np.float64)
    return v
