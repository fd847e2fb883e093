"""Pins of the CPU oracle against things other than itself.

* brute force: a dense float64 conv3d (PyTorch, cross-correlation) over the
  zero-filled grid, read at the active sites, must equal the submanifold
  convolution there (trellis_sparse_mlx README, "What's in it" / "Correctness");
* closed forms: 1x1x1 is a Linear layer, an isolated voxel gives
  feats @ W[centre], the interior of a dense block of ones gives the sum of
  all weights;
* the hand-worked fixtures in tests/golden/hand_worked.json, which separate
  feats[c+d] from feats[c-d], fix the tap order, and fix the error scale
  S = sum |feats[c+d]| |W[d]| (equal to the output when no terms cancel, above
  |out| in the mixed-sign case);
* neighbour-map invariants and an O(N^2) brute-force neighbour search;
* the C++ oracle against the Python one.

Planted mistakes (a flipped offset, a dropped tap, a transposed weight; for S:
absent taps counted, a product of sums, |out| in place of S) are applied to a
copy of the oracle here, on the CPU, to show the pins catch them.
"""
import json
import os

import numpy as np
import pytest
import torch

from oracle import native, submconv_ref as ref

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "hand_worked.json")


def _random_sites(rng, grid, batch, p):
    rows = []
    for b in range(batch):
        occ = rng.random((grid, grid, grid)) < p
        xyz = np.argwhere(occ)
        rows.append(np.concatenate([np.full((len(xyz), 1), b), xyz], axis=1))
    return np.concatenate(rows).astype(np.int32)


def _dense_conv(coords, feats, W, K, stride, grid, batch):
    """Dense float64 conv3d over the zero-filled grid, read at active sites."""
    cin, cout = W.shape[1], W.shape[2]
    dense = torch.zeros((batch, cin, grid, grid, grid), dtype=torch.float64)
    c = torch.from_numpy(coords.astype(np.int64))
    dense[c[:, 0], :, c[:, 1], c[:, 2], c[:, 3]] = torch.as_tensor(feats, dtype=torch.float64)
    # weight[co, ci, a, b, c] = W[k(a-r, b-r, c-r)][ci, co]
    w = torch.as_tensor(W, dtype=torch.float64).reshape(K, K, K, cin, cout)
    weight = w.permute(4, 3, 0, 1, 2).contiguous()
    r = K // 2
    y = torch.nn.functional.conv3d(dense, weight, padding=r * stride, dilation=stride)
    return y[c[:, 0], :, c[:, 1], c[:, 2], c[:, 3]].numpy()


@pytest.mark.parametrize("seed,grid,batch,p,K,stride,cin,cout", [
    (0, 8, 1, 0.10, 3, 1, 3, 4),
    (1, 9, 2, 0.30, 3, 1, 4, 2),
    (2, 7, 2, 0.90, 3, 1, 2, 3),
    (3, 10, 1, 0.25, 3, 2, 3, 3),
    (4, 8, 2, 0.40, 1, 1, 5, 3),
    (5, 9, 1, 0.20, 5, 1, 2, 2),
])
def test_bruteforce_dense_conv3d(seed, grid, batch, p, K, stride, cin, cout):
    rng = np.random.default_rng(seed)
    coords = _random_sites(rng, grid, batch, p)
    feats = rng.standard_normal((len(coords), cin))
    W = rng.standard_normal((K ** 3, cin, cout))
    out, scale = ref.submconv(coords, feats, W, K=K, stride=stride)
    dense = _dense_conv(coords, feats, W, K, stride, grid, batch)
    np.testing.assert_allclose(out, dense, rtol=1e-12, atol=1e-12)
    assert np.all(scale >= np.abs(out) - 1e-12)


def test_linear_closed_form():
    rng = np.random.default_rng(7)
    coords = _random_sites(rng, 6, 2, 0.5)
    feats = rng.standard_normal((len(coords), 6))
    W = rng.standard_normal((1, 6, 5))
    out, _ = ref.submconv(coords, feats, W, K=1)
    np.testing.assert_allclose(out, feats @ W[0], rtol=1e-13, atol=1e-13)


def test_isolated_voxel_is_centre_tap():
    rng = np.random.default_rng(8)
    coords = np.array([[0, 5, 5, 5], [0, 9, 9, 9], [1, 5, 5, 5], [0, 5, 5, 7]], np.int32)
    feats = rng.standard_normal((4, 3))
    W = rng.standard_normal((27, 3, 2))
    out, _ = ref.submconv(coords, feats, W)
    np.testing.assert_allclose(out, feats @ W[13], rtol=1e-13, atol=1e-13)


def test_dense_block_of_ones():
    g = 5
    xyz = np.argwhere(np.ones((g, g, g), bool))
    coords = np.concatenate([np.zeros((len(xyz), 1)), xyz], axis=1).astype(np.int32)
    rng = np.random.default_rng(9)
    W = rng.standard_normal((27, 2, 3))
    feats = np.ones((len(coords), 2))
    out, _ = ref.submconv(coords, feats, W)
    centre = np.flatnonzero((coords[:, 1:] == 2).all(axis=1))[0]
    np.testing.assert_allclose(out[centre], W.sum(axis=(0, 1)), rtol=1e-13)
    corner = np.flatnonzero((coords[:, 1:] == 0).all(axis=1))[0]
    # the corner voxel only sees offsets with every component in {0, +1}
    taps = [9 * (dx + 1) + 3 * (dy + 1) + (dz + 1)
            for dx in (0, 1) for dy in (0, 1) for dz in (0, 1)]
    np.testing.assert_allclose(out[corner], W[taps].sum(axis=(0, 1)), rtol=1e-13)


def _golden_cases():
    with open(GOLDEN) as fh:
        return json.load(fh)["cases"]


def _golden_weights(case) -> np.ndarray:
    """W[k] = k + 1, or (-1)^k (k + 1) for the 'alternating' cases (Cin = Cout = 1)."""
    k = np.arange(27, dtype=np.float64)
    w = k + 1.0
    if case.get("weights") == "alternating":
        w = np.where(k % 2 == 0, 1.0, -1.0) * w
    return w.reshape(27, 1, 1)


@pytest.mark.parametrize("case", _golden_cases(), ids=lambda c: c["name"])
def test_hand_worked_golden(case):
    """Output and error scale S of both oracles equal the hand-worked values
    (exactly: every product and sum is a small integer)."""
    coords = np.array(case["coords"], np.int32)
    feats = np.array(case["feats"], np.float64)[:, None]
    W = _golden_weights(case)
    out, scale = ref.submconv(coords, feats, W)
    assert out[:, 0].tolist() == case["expected"]
    assert scale[:, 0].tolist() == case["expected_scale"]
    nbr = native.neighbor_map(coords)
    out_c, scale_c = native.submconv(feats, W, nbr)
    assert out_c[:, 0].tolist() == case["expected"]
    assert scale_c[:, 0].tolist() == case["expected_scale"]


def test_scale_bounds_and_reaches_output():
    """S >= |out| always (triangle inequality), with equality exactly when no
    terms cancel: all-positive inputs give S == out, element by element."""
    rng = np.random.default_rng(13)
    coords = _random_sites(rng, 8, 2, 0.3)
    feats = rng.standard_normal((len(coords), 4))
    W = rng.standard_normal((27, 4, 3))
    out, scale = ref.submconv(coords, feats, W)
    assert np.all(scale >= np.abs(out) - 1e-12)
    assert np.any(scale > np.abs(out) + 1e-6)  # random signs do cancel somewhere
    out_p, scale_p = ref.submconv(coords, np.abs(feats), np.abs(W))
    np.testing.assert_allclose(scale_p, out_p, rtol=1e-13, atol=0)
    np.testing.assert_allclose(scale_p, scale, rtol=1e-13, atol=0)  # S depends on |f|, |W| only


def test_map_invariants_and_bruteforce_search():
    rng = np.random.default_rng(10)
    coords = _random_sites(rng, 7, 2, 0.35)
    nbr = ref.neighbor_map(coords)
    n = len(coords)
    assert np.all(nbr[:, 13] == np.arange(n))
    for i in range(n):
        for k in range(27):
            j = nbr[i, k]
            if j >= 0:
                assert nbr[j, 26 - k] == i
    offs = np.array(ref.tap_offsets(3))
    # O(N^2) search: for each pair (i, j) in the same batch, the offset j - i
    brute = np.full((n, 27), -1, np.int64)
    for i in range(n):
        d = coords[:, 1:] - coords[i, 1:]
        same = coords[:, 0] == coords[i, 0]
        for k, o in enumerate(offs):
            hit = np.flatnonzero(same & (d == o).all(axis=1))
            assert len(hit) <= 1
            if len(hit):
                brute[i, k] = hit[0]
    np.testing.assert_array_equal(nbr, brute)


def test_duplicates_rejected():
    coords = np.array([[0, 1, 2, 3], [0, 1, 2, 3]], np.int32)
    with pytest.raises(ValueError):
        ref.neighbor_map(coords)
    with pytest.raises(ValueError):
        native.neighbor_map(coords)


@pytest.mark.parametrize("K,stride", [(3, 1), (3, 2), (1, 1), (5, 1)])
def test_native_matches_python(K, stride):
    rng = np.random.default_rng(11 + K + stride)
    coords = _random_sites(rng, 9, 2, 0.3)
    coords = coords[rng.permutation(len(coords))]
    feats = rng.standard_normal((len(coords), 5))
    W = rng.standard_normal((K ** 3, 5, 6))
    nbr_py = ref.neighbor_map(coords, K, stride)
    nbr_c = native.neighbor_map(coords, K, stride)
    np.testing.assert_array_equal(nbr_py, nbr_c)
    out_py, s_py = ref.submconv(coords, feats, W, K=K, stride=stride, nbr=nbr_py)
    out_c, s_c = native.submconv(feats, W, nbr_c)
    np.testing.assert_allclose(out_c, out_py, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(s_c, s_py, rtol=1e-12, atol=1e-12)
    rows = np.array([3, 0, len(coords) - 1])
    out_r = native.submconv(feats, W, nbr_c, rows=rows, want_scale=False)
    np.testing.assert_allclose(out_r, out_py[rows], rtol=1e-12, atol=1e-12)


def test_uniform_pair_count_matches_expectation():
    """Exactly-n uniform occupancy: the expected number of (voxel, active
    neighbour) pairs is n + sum_{d != 0} prod_a (G - |d_a|) * n (n-1) / (G^3 (G^3-1))."""
    from submanifold_sparse_convolution_coord_b200 import synth
    inp = synth.make_inputs("uniform64")
    g, n = inp.workload.grid, inp.n
    nbr = native.neighbor_map(inp.coords)
    pairs = int((nbr >= 0).sum())
    cells = g ** 3
    expect = n + sum(np.prod([g - abs(v) for v in d]) for d in ref.tap_offsets(3) if d != (0, 0, 0)) \
        * n * (n - 1) / (cells * (cells - 1))
    # hypergeometric-like fluctuation is ~sqrt(expect); allow 5 sigma
    assert abs(pairs - expect) < 5 * np.sqrt(expect), (pairs, expect)


# ----------------------------------------------------------------------------
# planted mistakes: each mutant of the oracle must fail at least one pin
# ----------------------------------------------------------------------------
def _mutant_submconv(coords, feats, W, mutation):
    if mutation == "flip":
        nbr = ref.neighbor_map(coords)[:, ::-1]  # tap k reads the neighbour at c - d_k
    else:
        nbr = ref.neighbor_map(coords)
    if mutation == "drop_tap":
        nbr = nbr.copy()
        nbr[:, 26] = -1
    f = np.asarray(feats, np.float64)
    w = np.asarray(W, np.float64)
    if mutation == "transpose":
        w = np.ascontiguousarray(np.transpose(w, (0, 2, 1)))
    out = np.zeros((len(f), w.shape[2]))
    for k in range(27):
        j = nbr[:, k]
        ok = j >= 0
        out[ok] += f[j[ok]] @ w[k]
    return out


@pytest.mark.parametrize("mutation", ["flip", "drop_tap", "transpose"])
def test_planted_mistakes_are_caught(mutation):
    caught = False
    for case in _golden_cases():
        coords = np.array(case["coords"], np.int32)
        feats = np.array(case["feats"])[:, None]
        W = _golden_weights(case)
        if _mutant_submconv(coords, feats, W, mutation)[:, 0].tolist() != case["expected"]:
            caught = True
        assert _mutant_submconv(coords, feats, W, "none")[:, 0].tolist() == case["expected"]
    rng = np.random.default_rng(12)
    coords = _random_sites(rng, 8, 1, 0.5)
    feats = rng.standard_normal((len(coords), 3))
    W = rng.standard_normal((27, 3, 3))
    dense = _dense_conv(coords, feats, W, 3, 1, 8, 1)
    if not np.allclose(_mutant_submconv(coords, feats, W, mutation), dense, rtol=1e-9, atol=1e-9):
        caught = True
    # the unmutated form agrees with brute force
    assert np.allclose(_mutant_submconv(coords, feats, W, "none"), dense, rtol=1e-9, atol=1e-9)
    assert caught


def _mutant_scale(coords, feats, W, mutation):
    """The error scale S with a planted mistake."""
    nbr = ref.neighbor_map(coords)
    f = np.abs(np.asarray(feats, np.float64))
    w = np.abs(np.asarray(W, np.float64))
    n = len(f)
    S = np.zeros((n, w.shape[2]))
    for i in range(n):
        for k in range(27):
            j = nbr[i, k]
            if mutation == "all_taps":  # absent neighbours counted with the voxel's own row
                S[i] += f[j if j >= 0 else i] @ w[k]
            elif j >= 0:
                S[i] += f[j] @ w[k]
    if mutation == "product_of_sums":  # (sum |f|) * (sum |W|) over the active taps
        for i in range(n):
            ks = [k for k in range(27) if nbr[i, k] >= 0]
            S[i] = f[nbr[i, ks]].sum(axis=0) @ w[ks].sum(axis=0)
    if mutation == "abs_of_sum":  # |out| instead of sum |f| |W|
        S = np.abs(ref.submconv(coords, feats, W)[0])
    return S


@pytest.mark.parametrize("mutation", ["all_taps", "product_of_sums", "abs_of_sum"])
def test_planted_scale_mistakes_are_caught(mutation):
    caught = False
    for case in _golden_cases():
        coords = np.array(case["coords"], np.int32)
        feats = np.array(case["feats"])[:, None]
        W = _golden_weights(case)
        if _mutant_scale(coords, feats, W, mutation)[:, 0].tolist() != case["expected_scale"]:
            caught = True
        # the unmutated form reproduces the hand-worked values
        assert _mutant_scale(coords, feats, W, "none")[:, 0].tolist() == case["expected_scale"]
    assert caught
