"""Fused epilogue out = act(conv + bias) + residual against the oracle
(conv in float64, then submconv_ref.epilogue).

Bound: the activations are Lipschitz with constant at most 1.13 (GELU; SiLU
1.10, ReLU 1), so the accumulator's error 2e-3 * S grows to at most
1.2 * 2e-3 * S through them; bias and residual are exact in fp32 and add one
fp32 rounding each (the 1e-6 term); the stored result adds u * |ref|.  fp32
features (fp64 accumulation and epilogue): 1e-5 * |ref| + 1e-12 * (S + |b| + |r|).
"""
import numpy as np
import pytest
import torch

from oracle import native, submconv_ref as ref
from submanifold_sparse_convolution_coord_b200 import synth
from submanifold_sparse_convolution_coord_b200.binding import SubMIndex

from gpu_common import UNIT_ROUNDOFF, as_f64

pytestmark = pytest.mark.gpu

DEV = "cuda:0"


def _check(out, want, S, mag, dtype, what):
    got = as_f64(out)
    err = np.abs(got - want)
    if dtype == torch.float32:
        bound = 1e-5 * np.abs(want) + 1e-12 * (S + mag)
    else:
        bound = 1.2 * 2e-3 * S + UNIT_ROUNDOFF[dtype] * np.abs(want) + 1e-6 * mag
    bad = err > bound
    assert not bad.any(), f"{what}: {int(bad.sum())} out of tolerance, max err {err.max()}"


# (seed, n, grid, cin, cout, K, dtype)
SHAPES = [(0, 3000, 20, 128, 128, 3, "f16"), (1, 2000, 16, 64, 256, 3, "bf16"),
          (2, 1500, 20, 256, 128, 1, "bf16"), (3, 500, 10, 16, 24, 3, "f32"),
          (4, 600, 12, 48, 80, 3, "f16")]


@pytest.mark.parametrize("act", ["none", "relu", "silu", "gelu"])
@pytest.mark.parametrize("shape", SHAPES, ids=lambda s: "s{}_{}x{}_K{}_{}".format(s[0], s[3], s[4], s[5], s[6]))
def test_fused_epilogue(act, shape):
    seed, n, grid, cin, cout, K, dt = shape
    coords, feats, W = synth.random_case(seed, n, grid, 1, cin, cout, K, dt)
    rng = np.random.default_rng(seed + 500)
    bias = synth.round_to(rng.standard_normal(cout) * 0.5, dt)
    res = synth.round_to(rng.standard_normal((len(coords), cout)), dt)
    idx = SubMIndex(torch.from_numpy(coords).to(DEV))
    nbr = native.neighbor_map(coords, K) if K == 3 else np.arange(len(coords), dtype=np.int32)[:, None]
    conv, S = native.submconv(as_f64(feats), as_f64(W), nbr)
    for use_b, use_r in ((True, False), (False, True), (True, True)):
        b = bias.to(DEV) if use_b else None
        r = res.to(DEV) if use_r else None
        out = idx.forward(feats.to(DEV), W.to(DEV), K=K, bias=b, residual=r, activation=act)
        torch.cuda.synchronize()
        want = ref.epilogue(conv, as_f64(bias) if use_b else None, act,
                            as_f64(res) if use_r else None)
        mag = (np.abs(as_f64(bias))[None, :] if use_b else 0) + (np.abs(as_f64(res)) if use_r else 0)
        _check(out, want, S, mag, feats.dtype, f"{shape} {act} b={use_b} r={use_r}")
    assert idx.status() == 0
    idx.close()


def test_resblock_pair_with_fused_skip_sum():
    """The block's closing layer: conv3x3x3(h) + skip, with the skip computed by
    the 1x1x1 layer first; checked layer by layer on the GPU's own inputs."""
    coords, x, W1 = synth.random_case(9, 3000, 20, 1, 128, 256, 1, "bf16")
    _, _, W3 = synth.random_case(10, 10, 4, 1, 128, 256, 3, "bf16")
    idx = SubMIndex(torch.from_numpy(coords).to(DEV))
    skip = idx.forward(x.to(DEV), W1.to(DEV), K=1)
    out = idx.forward(x.to(DEV), W3.to(DEV), K=3, residual=skip)
    torch.cuda.synchronize()
    conv, S = native.submconv(as_f64(x), as_f64(W3), native.neighbor_map(coords))
    want = ref.epilogue(conv, None, "none", as_f64(skip))
    _check(out, want, S, np.abs(as_f64(skip)), torch.bfloat16, "conv + skip")
    idx.close()
