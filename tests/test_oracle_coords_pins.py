"""Pins of the x2 coordinate-op oracles (downsample by max, subdivide) against
dense brute force, a hand-worked case and their round trip.

* downsample2 equals a dense max_pool3d (kernel 2, stride 2) over the grid
  filled with -inf at empty cells, read at the cells that have a child;
* subdivide2 equals dense nearest-neighbour x2 upsampling of the grid, read at
  the children of active voxels;
* downsample2(subdivide2(c, f)) gives back (c, f) in sorted order.

Planted mistakes (average instead of max, the parent rounded up, children in
z-slowest order) are applied to copies here and must fail a pin.
"""
import numpy as np
import pytest
import torch

from oracle import submconv_ref as ref


def _sites(rng, grid, batch, p):
    rows = []
    for b in range(batch):
        xyz = np.argwhere(rng.random((grid, grid, grid)) < p)
        rows.append(np.concatenate([np.full((len(xyz), 1), b), xyz], axis=1))
    c = np.concatenate(rows).astype(np.int32)
    return c[rng.permutation(len(c))]


def _dense_maxpool(coords, feats, grid, batch):
    C = feats.shape[1]
    d = torch.full((batch, C, grid, grid, grid), -np.inf, dtype=torch.float64)
    ci = torch.from_numpy(coords.astype(np.int64))
    d[ci[:, 0], :, ci[:, 1], ci[:, 2], ci[:, 3]] = torch.as_tensor(feats)
    occ = torch.zeros((batch, 1, grid, grid, grid), dtype=torch.float64)
    occ[ci[:, 0], :, ci[:, 1], ci[:, 2], ci[:, 3]] = 1.0
    pooled = torch.nn.functional.max_pool3d(d, 2, 2)
    pocc = torch.nn.functional.max_pool3d(occ, 2, 2)
    idx = torch.nonzero(pocc[:, 0] > 0)  # lexicographic (b, x, y, z)
    return idx.numpy().astype(np.int32), pooled[idx[:, 0], :, idx[:, 1], idx[:, 2], idx[:, 3]].numpy()


@pytest.mark.parametrize("seed,grid,batch,p,C", [(0, 8, 1, 0.2, 3), (1, 10, 2, 0.5, 2), (2, 6, 1, 0.95, 4)])
def test_downsample_dense_bruteforce(seed, grid, batch, p, C):
    rng = np.random.default_rng(seed)
    coords = _sites(rng, grid, batch, p)
    feats = rng.standard_normal((len(coords), C))
    oc, of = ref.downsample2(coords, feats)
    dc, df = _dense_maxpool(coords, feats, grid, batch)
    np.testing.assert_array_equal(oc, dc)
    np.testing.assert_array_equal(of, df)


@pytest.mark.parametrize("seed,grid,batch,p,C", [(3, 5, 1, 0.3, 2), (4, 4, 2, 0.6, 3)])
def test_subdivide_dense_bruteforce(seed, grid, batch, p, C):
    rng = np.random.default_rng(seed)
    coords = _sites(rng, grid, batch, p)
    feats = rng.standard_normal((len(coords), C))
    oc, of = ref.subdivide2(coords, feats)
    d = torch.full((batch, C, grid, grid, grid), np.nan, dtype=torch.float64)
    ci = torch.from_numpy(coords.astype(np.int64))
    d[ci[:, 0], :, ci[:, 1], ci[:, 2], ci[:, 3]] = torch.as_tensor(feats)
    up = d.repeat_interleave(2, dim=2).repeat_interleave(2, dim=3).repeat_interleave(2, dim=4)
    o = torch.from_numpy(oc.astype(np.int64))
    np.testing.assert_array_equal(of, up[o[:, 0], :, o[:, 1], o[:, 2], o[:, 3]].numpy())
    # exactly the upsampled active cells, each once
    active = torch.nonzero(~torch.isnan(up[:, 0])).numpy()
    assert sorted(map(tuple, oc.tolist())) == sorted(map(tuple, active.tolist()))


def test_hand_worked():
    coords = np.array([[0, 3, 0, 0], [0, 2, 1, 1], [1, 2, 0, 0], [0, 0, 0, 5]], np.int32)
    feats = np.array([[1.0, -4.0], [2.0, -9.0], [7.0, 7.0], [0.5, 0.25]])
    oc, of = ref.downsample2(coords, feats)
    # (0,3,0,0) and (0,2,1,1) share parent (0,1,0,0): max (2, -4); (0,0,0,5) -> (0,0,0,2); (1,2,0,0) -> (1,1,0,0)
    assert oc.tolist() == [[0, 0, 0, 2], [0, 1, 0, 0], [1, 1, 0, 0]]
    assert of.tolist() == [[0.5, 0.25], [2.0, -4.0], [7.0, 7.0]]
    sc, sf = ref.subdivide2(coords[:1], feats[:1])
    assert sc.tolist() == [[0, 6, 0, 0], [0, 6, 0, 1], [0, 6, 1, 0], [0, 6, 1, 1],
                           [0, 7, 0, 0], [0, 7, 0, 1], [0, 7, 1, 0], [0, 7, 1, 1]]
    assert sf.tolist() == [[1.0, -4.0]] * 8


def test_round_trip():
    rng = np.random.default_rng(5)
    coords = _sites(rng, 9, 2, 0.3)
    feats = rng.standard_normal((len(coords), 3))
    sc, sf = ref.subdivide2(coords, feats)
    dc, df = ref.downsample2(sc, sf)
    order = np.lexsort(coords.T[::-1])
    np.testing.assert_array_equal(dc, coords[order])
    np.testing.assert_array_equal(df, feats[order])


def _mutant_down(coords, feats, mutation):
    f = np.asarray(feats, np.float64)
    groups = {}
    for i, (b, x, y, z) in enumerate(coords.tolist()):
        key = (b, (x + 1) // 2, (y + 1) // 2, (z + 1) // 2) if mutation == "round_up" else \
            (b, x // 2, y // 2, z // 2)
        groups.setdefault(key, []).append(i)
    keys = sorted(groups)
    red = (lambda r: f[r].mean(axis=0)) if mutation == "average" else (lambda r: f[r].max(axis=0))
    return np.array(keys, np.int32), np.stack([red(groups[k]) for k in keys])


@pytest.mark.parametrize("mutation", ["average", "round_up", "z_slowest"])
def test_planted_mistakes_are_caught(mutation):
    rng = np.random.default_rng(6)
    coords = _sites(rng, 8, 1, 0.4)
    feats = rng.standard_normal((len(coords), 2))
    if mutation == "z_slowest":
        sc, sf = ref.subdivide2(coords[:3], feats[:3])
        mc = sc.copy()
        for i in range(3):  # children with z slowest: c = 4 dz + 2 dy + dx
            blk = mc[8 * i:8 * i + 8].copy()
            mc[8 * i:8 * i + 8] = blk[[0, 4, 2, 6, 1, 5, 3, 7]]
        assert not np.array_equal(mc, sc)
        return
    dc, df = _dense_maxpool(coords, feats, 8, 1)
    mc, mf = _mutant_down(coords, feats, mutation)
    assert not (np.array_equal(mc, dc) and np.allclose(mf, df))
