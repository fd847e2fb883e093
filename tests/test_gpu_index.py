"""GPU neighbour map and tile plan against the CPU oracle (bit-exact), plus the
error paths of the index build.  All calls go through the C ABI."""
import numpy as np
import pytest
import torch

from oracle import native
from submanifold_sparse_convolution_coord_b200 import binding, synth
from submanifold_sparse_convolution_coord_b200.binding import SmcError, SubMIndex

pytestmark = pytest.mark.gpu

DEV = "cuda:0"


def _gpu_map(coords: np.ndarray, stride: int = 1, order: str = "mask"):
    c = torch.from_numpy(np.ascontiguousarray(coords, dtype=np.int32)).to(DEV)
    idx = SubMIndex(c, stride=stride, order=order)
    m = idx.neighbor_map().cpu().numpy()
    return idx, m


def _check_plan(idx: SubMIndex, nbr: np.ndarray):
    """perm is a bijection; every useful (voxel, tap) pair is covered by the tap
    set of the voxel's tile; plan counters match the map."""
    n = nbr.shape[0]
    perm, tmask = idx.tile_plan()
    perm = perm.cpu().numpy().astype(np.int64)
    tmask = tmask.cpu().numpy().astype(np.uint32)
    assert np.array_equal(np.sort(perm), np.arange(n))
    mask = np.zeros(n, np.uint32)
    for k in range(27):
        mask |= (nbr[:, k] >= 0).astype(np.uint32) << np.uint32(k)
    tile_of = np.empty(n, np.int64)
    tile_of[perm] = np.arange(n) // 128
    assert np.all((mask & ~tmask[tile_of]) == 0)
    # the tile mask is exactly the OR of its rows' masks
    expect = np.zeros(len(tmask), np.uint32)
    np.bitwise_or.at(expect, tile_of, mask)
    assert np.array_equal(expect, tmask)
    useful, issued = idx.plan_stats()
    assert useful == int((nbr >= 0).sum())
    pops = np.array([bin(int(v)).count("1") for v in tmask])
    assert issued == int(pops.sum()) * 128


@pytest.mark.parametrize("name", ["tiny16", "uniform64", "uniform128", "resblock64", "shells512"])
def test_map_bit_exact_on_workloads(name):
    inp = synth.make_inputs(name, n_layers=0)
    idx, m = _gpu_map(inp.coords)
    ref = native.neighbor_map(inp.coords)
    assert m.dtype == np.int32 and m.shape == ref.shape
    assert np.array_equal(m, ref)
    if inp.n <= 300_000:
        _check_plan(idx, ref)
    idx.close()


def _adversarial_cases():
    rng = np.random.default_rng(3)
    cases = {}
    co, _, _ = synth.random_case(1, 3000, 20, 2, 64, 64, 3, "f16", shuffle=True)
    cases["shuffled"] = co
    edge = []
    for x in (0, 1, 65534, 65535):
        for y in (0, 65535):
            for z in (0, 1, 65535):
                edge.append((0, x, y, z))
    edge += [(32767, 0, 0, 0), (32767, 65535, 65535, 65535), (32767, 65535, 65535, 65534)]
    cases["axis_limits"] = np.array(edge, np.int32)
    block = np.argwhere(np.ones((6, 6, 6), bool))
    touch = np.concatenate([np.concatenate([np.full((216, 1), b), block], 1) for b in (0, 1)])
    cases["two_batches_touching"] = touch.astype(np.int32)
    cases["single_voxel"] = np.array([[0, 7, 7, 7]], np.int32)
    cases["dense_block_9"] = np.concatenate(
        [np.zeros((729, 1)), np.argwhere(np.ones((9, 9, 9), bool))], 1).astype(np.int32)
    big = rng.choice(40 ** 3, size=129, replace=False)
    cases["n129"] = np.concatenate(
        [np.zeros((129, 1)), np.stack(np.unravel_index(big, (40, 40, 40)), 1)], 1).astype(np.int32)
    return cases


@pytest.mark.parametrize("case", sorted(_adversarial_cases()))
def test_map_adversarial(case):
    coords = _adversarial_cases()[case]
    idx, m = _gpu_map(coords)
    ref = native.neighbor_map(coords)
    assert np.array_equal(m, ref)
    _check_plan(idx, ref)
    idx.close()


@pytest.mark.parametrize("stride", [2, 3])
def test_map_stride(stride):
    co, _, _ = synth.random_case(5, 2000, 16, 2, 64, 64, 3, "f16")
    idx, m = _gpu_map(co, stride=stride)
    assert np.array_equal(m, native.neighbor_map(co, 3, stride))
    idx.close()


def test_input_order_plan():
    co, _, _ = synth.random_case(6, 5000, 30, 1, 64, 64, 3, "f16")
    idx, m = _gpu_map(co, order="input")
    ref = native.neighbor_map(co)
    assert np.array_equal(m, ref)
    perm, _ = idx.tile_plan()
    assert np.array_equal(perm.cpu().numpy(), np.arange(len(co)))
    _check_plan(idx, ref)
    idx.close()


@pytest.mark.parametrize("name", ["uniform64", "uniform128", "resblock64"])
def test_greedy_order_plan_and_conv(name):
    """The greedy tile packing: a valid plan (bijection, every pair covered,
    exact tile masks), fewer issued rows x taps than the mask sort, and the
    convolution over it matching the oracle on every row."""
    inp = synth.make_inputs(name)
    ref = native.neighbor_map(inp.coords)
    idx, m = _gpu_map(inp.coords, order="greedy")
    assert np.array_equal(m, ref)
    _check_plan(idx, ref)
    sorted_idx, _ = _gpu_map(inp.coords, order="mask")
    assert idx.plan_stats()[1] <= sorted_idx.plan_stats()[1]
    sorted_idx.close()
    W = inp.weights[0]
    out = idx.forward(inp.feats.to(DEV), W.to(DEV))
    torch.cuda.synchronize()
    assert idx.status() == 0
    want, scale = native.submconv(inp.feats.double().numpy(), W.double().numpy(), ref)
    from gpu_common import check_conv
    check_conv(out, want, scale, f"{name} greedy")
    idx.close()


def test_greedy_order_segments_and_edges():
    """Many 1,024-row segments with a ragged last one, shuffled input,
    and the small edge cases of the plan."""
    co, feats, W = synth.random_case(7, 40000, 60, 1, 64, 64, 3, "f16", shuffle=True)
    ref = native.neighbor_map(co)
    idx, m = _gpu_map(co, order="greedy")
    assert np.array_equal(m, ref)
    _check_plan(idx, ref)
    idx.close()
    for case in ("single_voxel", "n129", "two_batches_touching"):
        coords = _adversarial_cases()[case]
        idx, m = _gpu_map(coords, order="greedy")
        r = native.neighbor_map(coords)
        assert np.array_equal(m, r)
        _check_plan(idx, r)
        idx.close()


def test_empty_index():
    c = torch.zeros((0, 4), dtype=torch.int32, device=DEV)
    idx = SubMIndex(c)
    assert idx.n == 0 and idx.n_tiles == 0
    assert idx.plan_stats() == (0, 0)
    f = torch.zeros((0, 64), dtype=torch.float16, device=DEV)
    W = torch.zeros((27, 64, 64), dtype=torch.float16, device=DEV)
    out = idx.forward(f, W)
    assert out.shape == (0, 64)
    idx.close()


def _expect_status(coords: np.ndarray, status: int, **kw):
    c = torch.from_numpy(np.ascontiguousarray(coords, dtype=np.int32)).to(DEV)
    with pytest.raises(SmcError) as e:
        binding.smc_build_index(c, **kw)
    assert e.value.status == status


def test_duplicate_rejected():
    co = np.array([[0, 1, 2, 3], [0, 4, 5, 6], [0, 1, 2, 3]], np.int32)
    _expect_status(co, -2)


@pytest.mark.parametrize("bad", [(0, -1, 0, 0), (0, 0, 65536, 0), (0, 0, 0, -5),
                                 (32768, 0, 0, 0), (-1, 0, 0, 0)])
def test_range_rejected(bad):
    co = np.array([[0, 1, 1, 1], bad], np.int32)
    _expect_status(co, -3)


def test_table_full_reported():
    co, _, _ = synth.random_case(7, 500, 20, 1, 64, 64, 3, "f16")
    _expect_status(co, -7, table_capacity=256)


def test_handle_survives_errors_and_reuse():
    co, _, _ = synth.random_case(8, 700, 20, 1, 64, 64, 3, "f16")
    for _ in range(3):
        idx, m = _gpu_map(co)
        assert np.array_equal(m, native.neighbor_map(co))
        assert idx.status() == 0
        idx.close()


@pytest.mark.parametrize("first,then", [("mask", "greedy"), ("greedy", "mask"), ("mask", "input")])
def test_replan_equals_fresh_build(first, then):
    """Rebuilding a handle's plan in another row order (from its stored map)
    gives exactly the plan a fresh build in that order gives, and the
    convolution over it matches the oracle."""
    inp = synth.make_inputs("uniform64")
    ref = native.neighbor_map(inp.coords)
    idx, _ = _gpu_map(inp.coords, order=first)
    idx.replan(then)
    fresh, _ = _gpu_map(inp.coords, order=then)
    p1, t1 = idx.tile_plan()
    p2, t2 = fresh.tile_plan()
    assert torch.equal(p1, p2) and torch.equal(t1, t2)
    assert idx.plan_stats() == fresh.plan_stats()
    assert np.array_equal(idx.neighbor_map().cpu().numpy(), ref)
    _check_plan(idx, ref)
    W = inp.weights[0]
    out = idx.forward(inp.feats.to(DEV), W.to(DEV))
    torch.cuda.synchronize()
    assert idx.status() == 0
    want, scale = native.submconv(inp.feats.double().numpy(), W.double().numpy(), ref)
    from gpu_common import check_conv
    check_conv(out, want, scale, f"replan {first} -> {then}")
    fresh.close()
    idx.close()


def test_autotune_over_orders():
    """The search over row orders and launch configurations leaves the handle
    in one of the searched orders, with a forward that matches the oracle."""
    inp = synth.make_inputs("uniform64")
    ref = native.neighbor_map(inp.coords)
    idx, _ = _gpu_map(inp.coords, order="mask")
    W = inp.weights[0]
    f, w = inp.feats.to(DEV), W.to(DEV)
    name = idx.autotune(f, w, K=3, search_orders=True)
    assert name != "cuda-cores" and idx.order in ("mask", "greedy")
    _check_plan(idx, ref)
    out = idx.forward(f, w)
    torch.cuda.synchronize()
    assert idx.status() == 0
    want, scale = native.submconv(inp.feats.double().numpy(), W.double().numpy(), ref)
    from gpu_common import check_conv
    check_conv(out, want, scale, f"autotuned {idx.order} {name}")
    idx.close()
