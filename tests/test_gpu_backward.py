"""GPU backward passes (input and weight gradients) against the CPU oracle,
element by element, through the C ABI.

Bounds: the input gradient is a convolution of grad_out and is held to the
forward's bounds (tests/gpu_common.py); the weight gradient is returned in
fp32 and, for fp16/bf16 inputs, must satisfy |dW - ref| <= 2e-3 * S with
S = sum over pairs of |feats[j]| |grad_out[i]| (products of half-precision
values are exact in fp32; the bound covers the fp32 accumulation), and for
fp32 inputs |dW - ref| <= 1e-5 |ref| + 1e-12 S (fp64 accumulation)."""
import numpy as np
import pytest
import torch

from oracle import native
from submanifold_sparse_convolution_coord_b200 import synth
from submanifold_sparse_convolution_coord_b200.binding import SubMIndex

from gpu_common import as_f64, check_conv

pytestmark = pytest.mark.gpu

DEV = "cuda:0"


def _grads(coords, feats, G, W, K, stride=1, order="mask"):
    c = torch.from_numpy(np.ascontiguousarray(coords, dtype=np.int32)).to(DEV)
    idx = SubMIndex(c, stride=stride, order=order)
    gin = idx.backward_input(G.to(DEV), W.to(DEV), K=K)
    dW = idx.backward_weight(feats.to(DEV), G.to(DEV), K=K)
    torch.cuda.synchronize()
    assert idx.status() == 0
    return idx, gin, dW


def _oracle(coords, feats, G, W, K, stride=1, nbr=None):
    if nbr is None:
        nbr = native.neighbor_map(coords, K, stride)
    gin, s_in = native.submconv_backward_input(as_f64(G), as_f64(W), nbr)
    dW, s_w = native.submconv_backward_weight(as_f64(feats), as_f64(G), nbr)
    return gin, s_in, dW, s_w


def _check(idx, gin, dW, ref, feats, what):
    r_in, s_in, r_w, s_w = ref
    check_conv(gin, r_in, s_in, what + " grad_in")
    taps, cin, cout = r_w.shape
    check_conv(dW.reshape(taps * cin, cout), r_w.reshape(taps * cin, cout),
               s_w.reshape(taps * cin, cout), what + " dW", input_dtype=feats.dtype)


def _case(seed, n, grid, batch, cin, cout, K, dt, shuffle=False):
    coords, feats, W = synth.random_case(seed, n, grid, batch, cin, cout, K, dt, shuffle)
    G = synth.round_to(np.random.default_rng(seed + 1000).standard_normal((len(coords), cout)), dt)
    return coords, feats, G, W


# (seed, n per scene, grid, batch, cin, cout, K, dtype, shuffle)
CASES = [
    (0, 1, 8, 1, 64, 64, 3, "f16", False),
    (1, 300, 10, 1, 64, 64, 3, "bf16", False),
    (2, 2000, 16, 2, 128, 128, 3, "f16", True),
    (3, 3000, 20, 1, 128, 64, 3, "bf16", False),
    (4, 1500, 14, 1, 64, 256, 3, "f16", False),
    (5, 700, 12, 1, 192, 320, 3, "bf16", False),
    (6, 500, 12, 1, 512, 128, 3, "bf16", False),
    (7, 1000, 20, 1, 512, 1024, 1, "bf16", False),
    (8, 257, 20, 2, 64, 64, 1, "f16", False),
    (9, 400, 12, 2, 16, 16, 3, "f32", True),
    (10, 300, 10, 1, 3, 5, 3, "f32", False),
    (11, 300, 10, 1, 48, 80, 3, "f16", False),
    (12, 500, 12, 1, 8, 8, 1, "f32", False),
]


@pytest.mark.parametrize("case", CASES, ids=lambda c: "s{}_n{}_{}x{}_K{}_{}".format(
    c[0], c[1], c[4], c[5], c[6], c[7]))
def test_backward_small(case):
    seed, n, grid, batch, cin, cout, K, dt, shuffle = case
    coords, feats, G, W = _case(seed, n, grid, batch, cin, cout, K, dt, shuffle)
    idx, gin, dW = _grads(coords, feats, G, W, K)
    _check(idx, gin, dW, _oracle(coords, feats, G, W, K), feats, f"case {case}")
    idx.close()


def test_backward_stride2_and_input_order():
    coords, feats, G, W = _case(30, 3000, 20, 1, 64, 128, 3, "f16")
    for order, stride in (("input", 1), ("mask", 2)):
        idx, gin, dW = _grads(coords, feats, G, W, 3, stride=stride, order=order)
        _check(idx, gin, dW, _oracle(coords, feats, G, W, 3, stride=stride), feats,
               f"{order} stride {stride}")
        idx.close()


def test_backward_deterministic_repeat():
    coords, feats, G, W = _case(32, 5000, 24, 1, 128, 128, 3, "f16")
    idx, gin, dW = _grads(coords, feats, G, W, 3)
    gin2 = idx.backward_input(G.to(DEV), W.to(DEV))
    dW2 = idx.backward_weight(feats.to(DEV), G.to(DEV))
    torch.cuda.synchronize()
    assert torch.equal(gin, gin2) and torch.equal(dW, dW2)
    idx.close()


def test_backward_empty_index():
    c = torch.zeros((0, 4), dtype=torch.int32, device=DEV)
    idx = SubMIndex(c)
    dW = torch.full((27, 64, 64), 7.0, device=DEV)
    idx.backward_weight(torch.zeros((0, 64), dtype=torch.float16, device=DEV),
                        torch.zeros((0, 64), dtype=torch.float16, device=DEV), out=dW)
    torch.cuda.synchronize()
    assert torch.count_nonzero(dW) == 0
    idx.close()


@pytest.mark.parametrize("wl", ["uniform64", "uniform128"])
def test_backward_workload_full(wl):
    inp = synth.make_inputs(wl)
    W = inp.weights[0]
    G = synth.round_to(np.random.default_rng(7).standard_normal((inp.n, W.shape[2])),
                       inp.workload.dtype)
    idx, gin, dW = _grads(inp.coords, inp.feats, G, W, 3)
    _check(idx, gin, dW, _oracle(inp.coords, inp.feats, G, W, 3), inp.feats, wl)
    idx.close()


def test_backward_resblock64_full():
    """The channel-heavy block's 3x3x3 512->512 layer and 1x1x1 512->1024
    layer, every row and every weight."""
    inp = synth.make_inputs("resblock64")
    nbr = native.neighbor_map(inp.coords)
    for layer, K in ((0, 3), (1, 1)):
        W = inp.weights[layer]
        cin, cout = W.shape[1], W.shape[2]
        rng = np.random.default_rng(8 + layer)
        feats = synth.round_to(rng.standard_normal((inp.n, cin)), "bf16")
        G = synth.round_to(rng.standard_normal((inp.n, cout)), "bf16")
        idx, gin, dW = _grads(inp.coords, feats, G, W, K)
        m = nbr if K == 3 else np.arange(inp.n, dtype=np.int32)[:, None]
        _check(idx, gin, dW, _oracle(inp.coords, feats, G, W, K, nbr=m), feats, f"resblock L{layer}")
        idx.close()
