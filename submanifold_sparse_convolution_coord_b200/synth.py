"""Seeded synthetic inputs for the submanifold sparse 3-D convolution.

This module only draws inputs: active-voxel coordinates, feature rows and
weights.  It holds none of the convolution's arithmetic (no neighbour search,
no gather, no accumulation), so both the CUDA path and the CPU oracle can take
their inputs from here without sharing any of the method.

Workloads (named by what they are):

* ``tiny16``       batch 1, 16^3 grid, each cell active independently with
                   p = 0.10, Cin = Cout = 16, fp32.
* ``uniform64``    batch 1, 64^3 grid, exactly floor(0.10 * 64^3) = 26,214
                   cells drawn without replacement, Cin = Cout = 64, fp16.
* ``uniform128``   batch 1, 128^3 grid, exactly 209,715 cells (10 %),
                   Cin = Cout = 128, fp16.  This is the layer the
                   trellis_sparse_mlx README times in its "Performance"
                   section (128^3 grid, 128 channels, ~10 % occupancy).
* ``shells512``    batch 2 (two distinct scenes), 512^3 grid, active cells are
                   the 2-voxel-thick shell of the union of 8 random
                   axis-aligned ellipsoids (semi-axes U(40, 160), centres
                   U[0, 512)^3), Cin = Cout = 64, bf16.
* ``resblock64``   batch 1, 64^3 grid, the same shell construction with
                   semi-axes U(10, 40); a 3x3x3 512 -> 512 convolution followed
                   by a 1x1x1 512 -> 1024 convolution, bf16.

Random draws: ``numpy.random.default_rng(seed)`` (PCG64), drawn in the order
coordinates (scene 0, then scene 1), features, then each weight tensor.
Normals are drawn in float64 and rounded to the workload dtype.  ``N(0, v)``
means variance ``v``.  Coordinates are int32 rows ``(b, x, y, z)`` sorted
lexicographically (batch-contiguous, as the README's SparseTensor keeps them).
"""
from __future__ import annotations

import dataclasses
import math
from typing import Optional

import numpy as np
import torch

DTYPES = {"f32": torch.float32, "f16": torch.float16, "bf16": torch.bfloat16}


@dataclasses.dataclass(frozen=True)
class Layer:
    K: int
    cin: int
    cout: int
    weight_var: float  # variance of the normal the weights are drawn from


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    batch: int
    grid: int
    sparsity: str  # "bernoulli" | "exact" | "shells"
    dtype: str  # "f32" | "f16" | "bf16"
    layers: tuple
    p: float = 0.10
    n_ellipsoids: int = 8
    semi_axes: tuple = (40.0, 160.0)
    shell_thickness: int = 2
    description: str = ""


def _layer3(c_in: int, c_out: int) -> Layer:
    return Layer(3, c_in, c_out, 1.0 / (27 * c_in))


WORKLOADS = {
    "tiny16": Workload(
        "tiny16", 1, 16, "bernoulli", "f32", (_layer3(16, 16),),
        description="16^3, Bernoulli(0.10) cells, C16, fp32"),
    "uniform64": Workload(
        "uniform64", 1, 64, "exact", "f16", (_layer3(64, 64),),
        description="64^3, exactly 10% cells, C64, fp16"),
    "uniform128": Workload(
        "uniform128", 1, 128, "exact", "f16", (_layer3(128, 128),),
        description="128^3, exactly 10% cells (209,715), C128, fp16"),
    "shells512": Workload(
        "shells512", 2, 512, "shells", "bf16", (_layer3(64, 64),),
        semi_axes=(40.0, 160.0),
        description="2 scenes x 512^3, 2-voxel ellipsoid shells, C64, bf16"),
    "resblock64": Workload(
        "resblock64", 1, 64, "shells", "bf16",
        (_layer3(512, 512), Layer(1, 512, 1024, 1.0 / 512)),
        semi_axes=(10.0, 40.0),
        description="64^3 shells, 3x3x3 512->512 then 1x1x1 512->1024, bf16"),
}


# ----------------------------------------------------------------------------
# coordinates
# ----------------------------------------------------------------------------
def erode_cube(mask: np.ndarray) -> np.ndarray:
    """One binary erosion by the 3x3x3 cube; cells outside the grid count as
    empty.  The cube is separable, so this is three 1-D 3-wide erosions."""
    out = mask.copy()
    for axis in range(3):
        src = out
        cur = src.copy()
        sl_lo = [slice(None)] * 3
        sl_hi = [slice(None)] * 3
        # neighbour at -1 along axis
        sl_lo[axis] = slice(1, None)
        sl_hi[axis] = slice(None, -1)
        cur[tuple(sl_lo)] &= src[tuple(sl_hi)]
        edge = [slice(None)] * 3
        edge[axis] = slice(0, 1)
        cur[tuple(edge)] = False
        # neighbour at +1 along axis
        cur[tuple(sl_hi)] &= src[tuple(sl_lo)]
        edge[axis] = slice(-1, None)
        cur[tuple(edge)] = False
        out = cur
    return out


def ellipsoid_union(grid: int, centres: np.ndarray, axes: np.ndarray) -> np.ndarray:
    """Boolean grid: cell p (integer index) is inside when, for some ellipsoid
    e, sum(((p - c_e) / a_e)^2) <= 1."""
    inside = np.zeros((grid, grid, grid), dtype=bool)
    for c, a in zip(centres, axes):
        lo = np.maximum(np.floor(c - a).astype(np.int64), 0)
        hi = np.minimum(np.ceil(c + a).astype(np.int64) + 1, grid)
        if np.any(hi <= lo):
            continue
        xs = (np.arange(lo[0], hi[0], dtype=np.float64) - c[0]) / a[0]
        ys = (np.arange(lo[1], hi[1], dtype=np.float64) - c[1]) / a[1]
        zs = (np.arange(lo[2], hi[2], dtype=np.float64) - c[2]) / a[2]
        yz = ys[:, None] ** 2 + zs[None, :] ** 2
        for ix, xv in enumerate(xs):
            inside[lo[0] + ix, lo[1]:hi[1], lo[2]:hi[2]] |= (xv * xv + yz) <= 1.0
    return inside


def shell_cells(rng: np.random.Generator, grid: int, n_ellipsoids: int,
                semi_axes: tuple, thickness: int) -> np.ndarray:
    centres = rng.uniform(0.0, float(grid), size=(n_ellipsoids, 3))
    axes = rng.uniform(semi_axes[0], semi_axes[1], size=(n_ellipsoids, 3))
    inside = ellipsoid_union(grid, centres, axes)
    core = inside
    for _ in range(thickness):
        core = erode_cube(core)
    shell = inside & ~core
    return np.argwhere(shell).astype(np.int32)  # C order: x slowest


def draw_coords(w: Workload, rng: np.random.Generator) -> np.ndarray:
    scenes = []
    g = w.grid
    for b in range(w.batch):
        if w.sparsity == "bernoulli":
            flat = np.flatnonzero(rng.random(g ** 3) < w.p)
        elif w.sparsity == "exact":
            n = int(math.floor(w.p * g ** 3))
            flat = np.sort(rng.choice(g ** 3, size=n, replace=False))
        elif w.sparsity == "shells":
            xyz = shell_cells(rng, g, w.n_ellipsoids, w.semi_axes, w.shell_thickness)
            flat = None
        else:
            raise ValueError(w.sparsity)
        if flat is not None:
            xyz = np.stack(np.unravel_index(flat, (g, g, g)), axis=1).astype(np.int32)
        bcol = np.full((xyz.shape[0], 1), b, dtype=np.int32)
        scenes.append(np.concatenate([bcol, xyz], axis=1))
    coords = np.concatenate(scenes, axis=0)
    order = np.lexsort(coords.T[::-1])
    return np.ascontiguousarray(coords[order])


# ----------------------------------------------------------------------------
# features and weights
# ----------------------------------------------------------------------------
def round_to(x: np.ndarray, dtype: str) -> torch.Tensor:
    """float64 array -> torch tensor of ``dtype`` (round to nearest even)."""
    return torch.from_numpy(np.ascontiguousarray(x, dtype=np.float64)).to(DTYPES[dtype])


@dataclasses.dataclass
class Inputs:
    workload: Workload
    coords: np.ndarray  # int32 [N, 4]
    feats: torch.Tensor  # [N, Cin] in the workload dtype (CPU)
    weights: list  # one [K^3, Cin, Cout] tensor per layer (CPU)

    @property
    def n(self) -> int:
        return int(self.coords.shape[0])


def make_inputs(name: str, seed: int = 0, n_layers: Optional[int] = None) -> Inputs:
    w = WORKLOADS[name]
    rng = np.random.default_rng(seed)
    coords = draw_coords(w, rng)
    n = coords.shape[0]
    cin0 = w.layers[0].cin
    feats = round_to(rng.standard_normal((n, cin0)), w.dtype)
    weights = []
    layers = w.layers if n_layers is None else w.layers[:n_layers]
    for layer in layers:
        shape = (layer.K ** 3, layer.cin, layer.cout)
        weights.append(round_to(rng.standard_normal(shape) * math.sqrt(layer.weight_var), w.dtype))
    return Inputs(w, coords, feats, weights)


def random_case(seed: int, n_target: int, grid: int, batch: int, cin: int, cout: int,
                K: int, dtype: str, shuffle: bool = False) -> tuple:
    """A small random case for parity tests: ``n_target`` distinct cells per
    scene (clipped to the grid), standard-normal features, weights of variance
    1/(K^3 cin).  Returns (coords int32 [N,4], feats, W)."""
    rng = np.random.default_rng(seed)
    rows = []
    for b in range(batch):
        n = min(n_target, grid ** 3)
        flat = np.sort(rng.choice(grid ** 3, size=n, replace=False))
        xyz = np.stack(np.unravel_index(flat, (grid, grid, grid)), axis=1).astype(np.int32)
        rows.append(np.concatenate([np.full((n, 1), b, np.int32), xyz], axis=1))
    coords = np.concatenate(rows, axis=0)
    if shuffle:
        coords = coords[rng.permutation(coords.shape[0])]
    coords = np.ascontiguousarray(coords)
    feats = round_to(rng.standard_normal((coords.shape[0], cin)), dtype)
    W = round_to(rng.standard_normal((K ** 3, cin, cout)) / math.sqrt(K ** 3 * cin), dtype)
    return coords, feats, W
