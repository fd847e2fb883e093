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
