"""The allocation-free neighbour map (smc_build_neighbor_map_static).

Some callers cannot allocate device memory themselves (a framework that owns
the GPU's memory through its own pool, a latency-sensitive loop that must not
let cudaMalloc synchronise the device).  For them libsmc has one entry point
whose scratch (the coordinate hash table) is a fixed static device array.
These tests call it through the C ABI and compare its map with the map the
regular index build produces, bit for bit, on calls made back to back (the
array keeps the previous call's contents, so the second call must not see
them).  This file is collected last so that a failure here stops a run only
after every other test has run.
"""
import ctypes

import numpy as np
import pytest
import torch

from submanifold_sparse_convolution_coord_b200 import binding, synth

pytestmark = pytest.mark.gpu

DEV = "cuda:0"
MAX_VOXELS = 524288  # SMC_STATIC_MAX_VOXELS in include/smc.h


def _static_map(coords: torch.Tensor, stride: int = 1) -> tuple:
    n = coords.shape[0]
    out = torch.full((n, 27), 7, dtype=torch.int32, device=DEV)
    stream = torch.cuda.current_stream(torch.device(DEV)).cuda_stream
    rc = binding.lib().smc_build_neighbor_map_static(
        ctypes.c_void_p(coords.data_ptr()), n, stride, ctypes.c_void_p(out.data_ptr()),
        ctypes.c_void_p(stream))
    return rc, out


def _regular_map(coords: torch.Tensor, stride: int = 1) -> torch.Tensor:
    idx = binding.SubMIndex(coords, stride=stride)
    m = idx.neighbor_map()
    torch.cuda.synchronize()
    idx.close()
    return m


def _coords(seed: int, n: int, grid: int, batch: int) -> torch.Tensor:
    co, _, _ = synth.random_case(seed, n, grid, batch, 64, 64, 3, "f16", shuffle=True)
    return torch.from_numpy(co).to(DEV)


def test_matches_regular_entry_point_on_consecutive_calls():
    cases = [
        (torch.from_numpy(synth.make_inputs("uniform64", n_layers=0).coords).to(DEV), 1),
        (_coords(1, 3000, 18, 2), 1),   # smaller than the previous call
        (_coords(2, 3000, 18, 2), 2),
        (_coords(2, 3000, 18, 2), 2),   # the same input twice in a row
    ]
    for coords, stride in cases:
        rc, got = _static_map(coords, stride)
        assert rc == 0, binding.status_string(rc)
        want = _regular_map(coords, stride)
        assert torch.equal(got, want)


def test_largest_accepted_size_and_rejection_beyond_it():
    g = 128
    rng = np.random.default_rng(5)
    flat = np.sort(rng.choice(g ** 3, size=MAX_VOXELS, replace=False))
    xyz = np.stack(np.unravel_index(flat, (g, g, g)), 1)
    co = np.concatenate([np.zeros((MAX_VOXELS, 1)), xyz], 1).astype(np.int32)
    coords = torch.from_numpy(co).to(DEV)
    rc, got = _static_map(coords)
    assert rc == 0
    assert torch.equal(got, _regular_map(coords))
    # one voxel more than the static table holds: rejected before any launch
    big = torch.zeros((MAX_VOXELS + 1, 4), dtype=torch.int32, device=DEV)
    rc, _ = _static_map(big)
    assert rc == -6  # SMC_ERR_UNSUPPORTED


def test_errors_then_recovery():
    dup = torch.tensor([[0, 1, 2, 3], [0, 1, 2, 3]], dtype=torch.int32, device=DEV)
    rc, _ = _static_map(dup)
    assert rc == -2  # SMC_ERR_DUPLICATE
    bad = torch.tensor([[0, 1, 2, 3], [0, 70000, 0, 0]], dtype=torch.int32, device=DEV)
    rc, _ = _static_map(bad)
    assert rc == -3  # SMC_ERR_RANGE
    coords = _coords(3, 500, 12, 1)
    rc, got = _static_map(coords)
    assert rc == 0
    assert torch.equal(got, _regular_map(coords))
