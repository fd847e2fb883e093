"""The seeded input generators (no GPU): the workloads have the sizes and
structure the recipe states, are reproducible, and hold values that the
workload dtype represents exactly."""
import math

import numpy as np
import pytest
import torch

from submanifold_sparse_convolution_coord_b200 import synth

EXPECTED_N = {"tiny16": 424, "uniform64": 26214, "uniform128": 209715, "resblock64": 55100}


def _check_coords(coords: np.ndarray, w: synth.Workload):
    assert coords.dtype == np.int32 and coords.ndim == 2 and coords.shape[1] == 4
    assert coords[:, 0].min() >= 0 and coords[:, 0].max() < w.batch
    assert coords[:, 1:].min() >= 0 and coords[:, 1:].max() < w.grid
    # lexicographic (b, x, y, z) order, hence batch-contiguous, and no duplicates
    keys = ((coords[:, 0].astype(np.int64) * w.grid + coords[:, 1]) * w.grid
            + coords[:, 2]) * w.grid + coords[:, 3]
    assert np.all(np.diff(keys) > 0)


@pytest.mark.parametrize("name", sorted(EXPECTED_N))
def test_sizes_order_and_reproducibility(name):
    a = synth.make_inputs(name)
    b = synth.make_inputs(name)
    w = synth.WORKLOADS[name]
    assert a.n == EXPECTED_N[name]
    _check_coords(a.coords, w)
    assert np.array_equal(a.coords, b.coords)
    assert torch.equal(a.feats, b.feats)
    assert all(torch.equal(x, y) for x, y in zip(a.weights, b.weights))
    assert a.feats.dtype == synth.DTYPES[w.dtype] and a.feats.shape == (a.n, w.layers[0].cin)
    for layer, W in zip(w.layers, a.weights):
        assert W.shape == (layer.K ** 3, layer.cin, layer.cout)
        assert W.dtype == a.feats.dtype
    # another seed gives another draw
    c = synth.make_inputs(name, seed=1)
    assert not (c.coords.shape == a.coords.shape and np.array_equal(c.coords, a.coords))


def test_exact_occupancy_of_uniform_workloads():
    for name in ("uniform64", "uniform128"):
        w = synth.WORKLOADS[name]
        assert synth.make_inputs(name, n_layers=0).n == math.floor(w.p * w.grid ** 3)


def test_weight_and_feature_statistics():
    inp = synth.make_inputs("uniform128")
    f = inp.feats.double().numpy()
    assert abs(f.mean()) < 0.01 and abs(f.var() - 1.0) < 0.01
    W = inp.weights[0].double().numpy()
    assert abs(W.var() * 27 * 128 - 1.0) < 0.02  # N(0, 1 / (27 Cin)), variance


def test_values_are_exact_in_the_dtype():
    rng = np.random.default_rng(3)
    x = rng.standard_normal(1000)
    for dt in ("f16", "bf16", "f32"):
        t = synth.round_to(x, dt)
        back = t.double()
        assert torch.equal(back.to(synth.DTYPES[dt]).double(), back)
        # rounded to nearest: within half an ulp (bounded loosely for |x| < 4)
        assert float((back - torch.from_numpy(x)).abs().max()) <= {"f16": 2 ** -11 * 4,
                                                                   "bf16": 2 ** -8 * 4,
                                                                   "f32": 2 ** -24 * 4}[dt]


def test_erode_cube_matches_scipy():
    ndimage = pytest.importorskip("scipy.ndimage")
    rng = np.random.default_rng(5)
    m = rng.random((20, 17, 23)) < 0.8
    ref = ndimage.binary_erosion(m, structure=np.ones((3, 3, 3), bool), border_value=0)
    assert np.array_equal(synth.erode_cube(m), ref)


def test_ellipsoid_union_brute_force():
    rng = np.random.default_rng(6)
    g = 24
    centres = rng.uniform(0, g, size=(3, 3))
    axes = rng.uniform(2, 9, size=(3, 3))
    got = synth.ellipsoid_union(g, centres, axes)
    p = np.stack(np.meshgrid(*([np.arange(g)] * 3), indexing="ij"), axis=-1).astype(np.float64)
    ref = np.zeros((g, g, g), bool)
    for c, a in zip(centres, axes):
        ref |= (((p - c) / a) ** 2).sum(-1) <= 1.0
    assert np.array_equal(got, ref)


def test_shell_cells_lie_within_two_cells_of_the_outside():
    """The shell is the union minus its double 3x3x3 erosion, so every active
    cell has, within Chebyshev distance 2, a cell outside the union or the
    grid; this checks the consequence that can be seen from the active cells
    alone: an inactive or out-of-grid cell within distance 2."""
    inp = synth.make_inputs("resblock64", n_layers=0)
    g = synth.WORKLOADS["resblock64"].grid
    grid = np.zeros((g + 4, g + 4, g + 4), bool)  # 2-cell empty border
    xyz = inp.coords[:, 1:] + 2
    grid[xyz[:, 0], xyz[:, 1], xyz[:, 2]] = True
    near_outside = np.zeros(len(xyz), bool)
    for dx in range(-2, 3):
        for dy in range(-2, 3):
            for dz in range(-2, 3):
                near_outside |= ~grid[xyz[:, 0] + dx, xyz[:, 1] + dy, xyz[:, 2] + dz]
    assert near_outside.all()
