"""GPU coordinate operations against the CPU oracle: the sort-based neighbour
lookup (bit-exact against the hash lookup and the oracle's dict), x2
downsample by maximum and x2 subdivision (both exact: they only move and
compare values)."""
import numpy as np
import pytest
import torch

from oracle import native, submconv_ref as ref
from submanifold_sparse_convolution_coord_b200 import binding, synth
from submanifold_sparse_convolution_coord_b200.binding import SmcError, SubMIndex

pytestmark = pytest.mark.gpu

DEV = "cuda:0"


@pytest.mark.parametrize("wl", ["tiny16", "uniform64", "uniform128", "resblock64", "shells512"])
def test_sorted_lookup_matches_hash_and_oracle(wl):
    coords = synth.make_inputs(wl, n_layers=0).coords
    c = torch.from_numpy(coords).to(DEV)
    a = SubMIndex(c, lookup="sort")
    b = SubMIndex(c, lookup="hash")
    ma, mb = a.neighbor_map().cpu().numpy(), b.neighbor_map().cpu().numpy()
    assert np.array_equal(ma, mb)
    assert np.array_equal(ma, native.neighbor_map(coords))
    assert a.plan_stats() == b.plan_stats()
    a.close()
    b.close()


def test_sorted_lookup_shuffled_stride_and_conv():
    coords, feats, W = synth.random_case(3, 3000, 20, 2, 64, 128, 3, "f16", shuffle=True)
    c = torch.from_numpy(coords).to(DEV)
    for stride in (1, 2):
        idx = SubMIndex(c, stride=stride, lookup="sort")
        assert np.array_equal(idx.neighbor_map().cpu().numpy(),
                              native.neighbor_map(coords, 3, stride))
        out = idx.forward(feats.to(DEV), W.to(DEV))
        ref_out, scale = native.submconv(feats.double().numpy(), W.double().numpy(),
                                         native.neighbor_map(coords, 3, stride))
        err = np.abs(out.double().cpu().numpy() - ref_out)
        assert np.all(err <= 2e-3 * scale + 2.0 ** -11 * np.abs(ref_out))
        idx.close()


def test_sorted_lookup_errors():
    dup = torch.tensor([[0, 1, 2, 3], [0, 5, 5, 5], [0, 1, 2, 3]], dtype=torch.int32, device=DEV)
    with pytest.raises(SmcError) as e:
        SubMIndex(dup, lookup="sort")
    assert e.value.status == -2
    bad = torch.tensor([[0, 1, 2, 3], [0, 70000, 0, 0], [0, 70001, 0, 0]], dtype=torch.int32,
                       device=DEV)
    with pytest.raises(SmcError) as e:
        SubMIndex(bad, lookup="sort")
    assert e.value.status == -3


def _rand_sites(seed, grid, batch, p):
    rng = np.random.default_rng(seed)
    rows = []
    for b in range(batch):
        xyz = np.argwhere(rng.random((grid, grid, grid)) < p)
        rows.append(np.concatenate([np.full((len(xyz), 1), b), xyz], axis=1))
    c = np.concatenate(rows).astype(np.int32)
    return c[rng.permutation(len(c))], rng


@pytest.mark.parametrize("dt", ["f32", "f16", "bf16"])
@pytest.mark.parametrize("seed,grid,batch,p,C", [(0, 12, 1, 0.3, 8), (1, 20, 2, 0.1, 3), (2, 9, 1, 0.9, 64)])
def test_downsample_matches_oracle(dt, seed, grid, batch, p, C):
    coords, rng = _rand_sites(seed, grid, batch, p)
    feats = synth.round_to(rng.standard_normal((len(coords), C)), dt)
    oc, of = binding.smc_downsample2(torch.from_numpy(coords).to(DEV), feats.to(DEV))
    rc, rf = ref.downsample2(coords, feats.double().numpy())
    assert np.array_equal(oc.cpu().numpy(), rc)
    assert np.array_equal(of.double().cpu().numpy(), rf)  # the maximum is one of the inputs


@pytest.mark.parametrize("dt", ["f32", "bf16"])
def test_subdivide_matches_oracle_and_round_trips(dt):
    coords, rng = _rand_sites(4, 14, 2, 0.2, )
    feats = synth.round_to(rng.standard_normal((len(coords), 5)), dt)
    c, f = torch.from_numpy(coords).to(DEV), feats.to(DEV)
    sc, sf = binding.smc_subdivide2(c, f)
    rc, rf = ref.subdivide2(coords, feats.double().numpy())
    assert np.array_equal(sc.cpu().numpy(), rc)
    assert np.array_equal(sf.double().cpu().numpy(), rf)
    dc, df = binding.smc_downsample2(sc, sf)
    order = np.lexsort(coords.T[::-1])
    assert np.array_equal(dc.cpu().numpy(), coords[order])
    assert torch.equal(df.cpu(), feats[torch.from_numpy(order)])


def test_coords_ops_on_workloads():
    for wl in ("uniform64", "resblock64"):
        inp = synth.make_inputs(wl)
        c, f = torch.from_numpy(inp.coords).to(DEV), inp.feats[:, :16].contiguous()
        oc, of = binding.smc_downsample2(c, f.to(DEV))
        rc, rf = ref.downsample2(inp.coords, f.double().numpy())
        assert np.array_equal(oc.cpu().numpy(), rc) and np.array_equal(of.double().cpu().numpy(), rf)


def test_coords_ops_errors_and_empty():
    big = torch.tensor([[0, 40000, 0, 0]], dtype=torch.int32, device=DEV)
    f = torch.ones((1, 4), dtype=torch.float16, device=DEV)
    with pytest.raises(SmcError) as e:
        binding.smc_subdivide2(big, f)
    assert e.value.status == -3
    empty = torch.zeros((0, 4), dtype=torch.int32, device=DEV)
    oc, of = binding.smc_downsample2(empty, torch.zeros((0, 4), dtype=torch.float16, device=DEV))
    assert oc.shape[0] == 0 and of.shape[0] == 0
