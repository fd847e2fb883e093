"""Pins of the backward oracles (input and weight gradients) against things
other than themselves.

* brute force: the dense float64 conv3d over the zero-filled grid, read at the
  active sites, differentiated by PyTorch autograd with respect to the active
  features and to the weights;
* the hand-worked fixture tests/golden/hand_worked_backward.json;
* closed forms: for K = 1 the gradients of a Linear layer (grad_out @ W^T and
  feats^T @ grad_out); isolated voxels see only the centre tap;
* the adjoint identities <conv(f), g> = <f, bwd_input(g)> = sum_k <W[k], dW[k]>;
* the C++ oracle against the Python one.

Planted mistakes (W[k] not transposed, the mirrored tap 26 - k, the weight
gradient's outer product taken the wrong way round) are applied to copies of
the oracle here, on the CPU, to show the pins catch them.
"""
import json
import os

import numpy as np
import pytest
import torch

from oracle import native, submconv_ref as ref

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "hand_worked_backward.json")


def _random_sites(rng, grid, batch, p):
    rows = []
    for b in range(batch):
        xyz = np.argwhere(rng.random((grid, grid, grid)) < p)
        rows.append(np.concatenate([np.full((len(xyz), 1), b), xyz], axis=1))
    return np.concatenate(rows).astype(np.int32)


def _dense_grads(coords, feats, W, G, K, stride, grid, batch):
    """Autograd of sum(conv3d(dense(feats)) at the active sites * G)."""
    cin, cout = W.shape[1], W.shape[2]
    f = torch.tensor(feats, dtype=torch.float64, requires_grad=True)
    w = torch.tensor(W, dtype=torch.float64, requires_grad=True)
    c = torch.from_numpy(coords.astype(np.int64))
    dense = torch.zeros((batch, cin, grid, grid, grid), dtype=torch.float64)
    dense[c[:, 0], :, c[:, 1], c[:, 2], c[:, 3]] = f  # differentiable scatter of the active rows
    weight = w.reshape(K, K, K, cin, cout).permute(4, 3, 0, 1, 2)
    r = K // 2
    y = torch.nn.functional.conv3d(dense, weight, padding=r * stride, dilation=stride)
    out = y[c[:, 0], :, c[:, 1], c[:, 2], c[:, 3]]
    (out * torch.as_tensor(G)).sum().backward()
    return f.grad.numpy(), w.grad.numpy()


@pytest.mark.parametrize("seed,grid,batch,p,K,stride,cin,cout", [
    (0, 8, 1, 0.15, 3, 1, 3, 4),
    (1, 9, 2, 0.35, 3, 1, 4, 2),
    (2, 7, 1, 0.90, 3, 1, 2, 3),
    (3, 10, 1, 0.25, 3, 2, 3, 3),
    (4, 8, 2, 0.40, 1, 1, 5, 3),
])
def test_backward_dense_autograd_bruteforce(seed, grid, batch, p, K, stride, cin, cout):
    rng = np.random.default_rng(100 + seed)
    coords = _random_sites(rng, grid, batch, p)
    feats = rng.standard_normal((len(coords), cin))
    W = rng.standard_normal((K ** 3, cin, cout))
    G = rng.standard_normal((len(coords), cout))
    gf, gw = _dense_grads(coords, feats, W, G, K, stride, grid, batch)
    gin, s_in = ref.submconv_backward_input(coords, G, W, K=K, stride=stride)
    dW, s_w = ref.submconv_backward_weight(coords, feats, G, K=K, stride=stride)
    np.testing.assert_allclose(gin, gf, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(dW, gw, rtol=1e-12, atol=1e-12)
    assert np.all(s_in >= np.abs(gin) - 1e-12) and np.all(s_w >= np.abs(dW) - 1e-12)


def _golden():
    with open(GOLDEN) as fh:
        return json.load(fh)["cases"]


@pytest.mark.parametrize("case", _golden(), ids=lambda c: c["name"])
def test_backward_hand_worked_golden(case):
    coords = np.array(case["coords"], np.int32)
    feats = np.array(case["feats"])[:, None]
    G = np.array(case["grad_out"])[:, None]
    W = (np.arange(27, dtype=np.float64) + 1.0).reshape(27, 1, 1)
    want_dW = np.zeros(27)
    for k, v in case["expected_dW_nonzero"].items():
        want_dW[int(k)] = v
    gin, s_in = ref.submconv_backward_input(coords, G, W)
    dW, _ = ref.submconv_backward_weight(coords, feats, G)
    assert gin[:, 0].tolist() == case["expected_grad_in"]
    assert s_in[:, 0].tolist() == case["expected_grad_in"]  # all terms positive
    assert dW[:, 0, 0].tolist() == want_dW.tolist()
    nbr = native.neighbor_map(coords)
    assert native.submconv_backward_input(G, W, nbr, want_scale=False)[:, 0].tolist() == \
        case["expected_grad_in"]
    assert native.submconv_backward_weight(feats, G, nbr, want_scale=False)[:, 0, 0].tolist() == \
        want_dW.tolist()


def test_backward_closed_forms():
    rng = np.random.default_rng(7)
    coords = _random_sites(rng, 6, 2, 0.5)
    f = rng.standard_normal((len(coords), 6))
    G = rng.standard_normal((len(coords), 5))
    W1 = rng.standard_normal((1, 6, 5))
    gin, _ = ref.submconv_backward_input(coords, G, W1, K=1)
    dW, _ = ref.submconv_backward_weight(coords, f, G, K=1)
    np.testing.assert_allclose(gin, G @ W1[0].T, rtol=1e-13, atol=1e-13)
    np.testing.assert_allclose(dW[0], f.T @ G, rtol=1e-13, atol=1e-13)
    iso = np.array([[0, 2, 2, 2], [0, 7, 7, 7], [1, 2, 2, 2]], np.int32)
    f3 = rng.standard_normal((3, 4))
    G3 = rng.standard_normal((3, 2))
    W3 = rng.standard_normal((27, 4, 2))
    gin3, _ = ref.submconv_backward_input(iso, G3, W3)
    dW3, _ = ref.submconv_backward_weight(iso, f3, G3)
    np.testing.assert_allclose(gin3, G3 @ W3[13].T, rtol=1e-13, atol=1e-13)
    np.testing.assert_allclose(dW3[13], f3.T @ G3, rtol=1e-13, atol=1e-13)
    assert not np.any(np.delete(dW3, 13, axis=0))


def test_adjoint_identities():
    rng = np.random.default_rng(8)
    coords = _random_sites(rng, 8, 2, 0.3)
    f = rng.standard_normal((len(coords), 3))
    G = rng.standard_normal((len(coords), 4))
    W = rng.standard_normal((27, 3, 4))
    out, _ = ref.submconv(coords, f, W)
    gin, _ = ref.submconv_backward_input(coords, G, W)
    dW, _ = ref.submconv_backward_weight(coords, f, G)
    a = float(np.sum(out * G))
    assert abs(a - float(np.sum(f * gin))) < 1e-9 * max(1.0, abs(a))
    assert abs(a - float(np.sum(W * dW))) < 1e-9 * max(1.0, abs(a))


@pytest.mark.parametrize("K,stride", [(3, 1), (3, 2), (1, 1)])
def test_native_backward_matches_python(K, stride):
    rng = np.random.default_rng(20 + K + stride)
    coords = _random_sites(rng, 9, 2, 0.3)
    coords = coords[rng.permutation(len(coords))]
    f = rng.standard_normal((len(coords), 5))
    G = rng.standard_normal((len(coords), 6))
    W = rng.standard_normal((K ** 3, 5, 6))
    nbr = native.neighbor_map(coords, K, stride)
    gin, s_in = ref.submconv_backward_input(coords, G, W, K=K, stride=stride)
    dW, s_w = ref.submconv_backward_weight(coords, f, G, K=K, stride=stride)
    gin_c, s_in_c = native.submconv_backward_input(G, W, nbr)
    dW_c, s_w_c = native.submconv_backward_weight(f, G, nbr)
    np.testing.assert_allclose(gin_c, gin, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(s_in_c, s_in, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(dW_c, dW, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(s_w_c, s_w, rtol=1e-12, atol=1e-12)


# ----------------------------------------------------------------------------
# planted mistakes
# ----------------------------------------------------------------------------
def _mutant_backward(coords, f, G, W, mutation):
    nbr = ref.neighbor_map(coords)
    n = len(coords)
    gin = np.zeros((n, W.shape[1]))
    dW = np.zeros_like(W)
    for i in range(n):
        for k in range(27):
            j = nbr[i, k]
            if j < 0:
                continue
            kk = 26 - k if mutation == "mirrored_tap" else k
            if mutation == "no_transpose":  # grad_out[i] @ W[k] instead of W[k] @ grad_out[i]
                gin[j] += W[kk].T @ G[i]
            else:
                gin[j] += W[kk] @ G[i]
            if mutation == "outer_swapped":  # outer(grad_out, feats): dW[k] transposed
                dW[k] += np.outer(G[i], f[j])
            else:
                dW[k] += np.outer(f[j], G[i])
    return gin, dW


@pytest.mark.parametrize("mutation", ["no_transpose", "mirrored_tap", "outer_swapped"])
def test_backward_planted_mistakes_are_caught(mutation):
    rng = np.random.default_rng(12)
    coords = _random_sites(rng, 7, 1, 0.5)
    f = rng.standard_normal((len(coords), 3))
    G = rng.standard_normal((len(coords), 3))
    W = rng.standard_normal((27, 3, 3))
    gf, gw = _dense_grads(coords, f, W, G, 3, 1, 7, 1)
    ok_in, ok_w = _mutant_backward(coords, f, G, W, "none")
    assert np.allclose(ok_in, gf, atol=1e-9) and np.allclose(ok_w, gw, atol=1e-9)
    m_in, m_w = _mutant_backward(coords, f, G, W, mutation)
    caught = not (np.allclose(m_in, gf, atol=1e-9) and np.allclose(m_w, gw, atol=1e-9))
    case = _golden()[0]
    c1 = np.array(case["coords"], np.int32)
    W1 = (np.arange(27, dtype=np.float64) + 1.0).reshape(27, 1, 1)
    g_in, _ = _mutant_backward(c1, np.array(case["feats"])[:, None], np.array(case["grad_out"])[:, None],
                               W1, mutation)
    caught = caught or g_in[:, 0].tolist() != case["expected_grad_in"]
    assert caught
