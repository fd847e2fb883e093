"""GPU SubMConv3d against the CPU oracle, element by element, through the C
ABI.  Tolerances are the ones stated in tests/gpu_common.py."""
import numpy as np
import pytest
import torch

from oracle import native
from submanifold_sparse_convolution_coord_b200 import synth
from submanifold_sparse_convolution_coord_b200.binding import SubMIndex

from gpu_common import check_conv, oracle_conv, sample_rows

pytestmark = pytest.mark.gpu

DEV = "cuda:0"


def _run(coords, feats, W, K, order="mask", stride=1):
    c = torch.from_numpy(np.ascontiguousarray(coords, dtype=np.int32)).to(DEV)
    idx = SubMIndex(c, stride=stride, order=order)
    out = idx.forward(feats.to(DEV), W.to(DEV), K=K)
    torch.cuda.synchronize()
    assert idx.status() == 0
    return idx, out


# (seed, n per scene, grid, batch, cin, cout, K, dtype, shuffle)
SMALL = [
    (0, 1, 8, 1, 64, 64, 3, "f16", False),
    (1, 100, 10, 1, 64, 64, 3, "f16", False),
    (2, 129, 12, 1, 64, 128, 3, "bf16", True),
    (3, 1000, 16, 2, 128, 128, 3, "f16", True),
    (4, 3000, 20, 1, 128, 64, 3, "bf16", False),
    (5, 2500, 24, 2, 64, 256, 3, "f16", False),
    (6, 1500, 14, 1, 256, 192, 3, "bf16", False),
    (7, 700, 12, 1, 512, 512, 3, "bf16", False),
    (8, 300, 16, 1, 192, 320, 3, "f16", False),
    (9, 5000, 17, 1, 64, 64, 3, "f16", True),
    (10, 1000, 20, 1, 512, 1024, 1, "bf16", False),
    (11, 257, 20, 2, 64, 64, 1, "f16", False),
    (12, 4000, 30, 1, 128, 384, 1, "bf16", True),
]


@pytest.mark.parametrize("case", SMALL, ids=lambda c: "s{}_n{}_b{}_{}x{}_K{}_{}".format(
    c[0], c[1], c[3], c[4], c[5], c[6], c[7]))
def test_tensor_core_small(case):
    seed, n, grid, batch, cin, cout, K, dt, shuffle = case
    coords, feats, W = synth.random_case(seed, n, grid, batch, cin, cout, K, dt, shuffle)
    idx, out = _run(coords, feats, W, K)
    ref, scale = oracle_conv(coords, feats, W, K)
    check_conv(out, ref, scale, f"case {case}")
    idx.close()


@pytest.mark.parametrize("cin,cout,dt", [(16, 16, "f32"), (3, 5, "f32"), (64, 64, "f32"),
                                         (16, 48, "f16"), (32, 64, "bf16"), (64, 40, "f16")])
@pytest.mark.parametrize("K", [1, 3])
def test_cuda_core_path(cin, cout, dt, K):
    coords, feats, W = synth.random_case(20 + cin, 600, 12, 2, cin, cout, K, dt, True)
    idx, out = _run(coords, feats, W, K)
    ref, scale = oracle_conv(coords, feats, W, K)
    check_conv(out, ref, scale, f"simt {cin}x{cout} {dt} K{K}")
    idx.close()


def test_stride2_and_input_order():
    coords, feats, W = synth.random_case(30, 3000, 20, 1, 64, 128, 3, "f16")
    for order, stride in (("input", 1), ("mask", 2)):
        idx, out = _run(coords, feats, W, 3, order=order, stride=stride)
        ref, scale = oracle_conv(coords, feats, W, 3, stride=stride)
        check_conv(out, ref, scale, f"{order} stride {stride}")
        idx.close()


def test_deterministic_repeat():
    coords, feats, W = synth.random_case(31, 4000, 24, 1, 128, 128, 3, "bf16", True)
    c = torch.from_numpy(coords).to(DEV)
    idx = SubMIndex(c)
    f, w = feats.to(DEV), W.to(DEV)
    a = idx.forward(f, w)
    b = idx.forward(f, w)
    torch.cuda.synchronize()
    assert torch.equal(a, b)
    idx.close()


def test_isolated_voxels_closed_form():
    """Isolated voxels: out = feats @ W[13] (only the centre tap is active)."""
    pts = np.array([[0, 4 * i, 4 * j, 4 * k] for i in range(6) for j in range(6) for k in range(6)],
                   np.int32)
    rng = np.random.default_rng(40)
    feats = synth.round_to(rng.standard_normal((len(pts), 64)), "f16")
    W = synth.round_to(rng.standard_normal((27, 64, 128)) / 40.0, "f16")
    idx, out = _run(pts, feats, W, 3)
    ref = feats.double().numpy() @ W[13].double().numpy()
    scale = np.abs(feats.double().numpy()) @ np.abs(W[13].double().numpy())
    check_conv(out, ref, scale, "isolated")
    idx.close()


def test_workload_tiny16_full():
    inp = synth.make_inputs("tiny16")
    idx, out = _run(inp.coords, inp.feats, inp.weights[0], 3)
    ref, scale = oracle_conv(inp.coords, inp.feats, inp.weights[0], 3)
    check_conv(out, ref, scale, "tiny16")
    idx.close()


def test_workload_uniform64_full():
    inp = synth.make_inputs("uniform64")
    idx, out = _run(inp.coords, inp.feats, inp.weights[0], 3)
    ref, scale = oracle_conv(inp.coords, inp.feats, inp.weights[0], 3)
    check_conv(out, ref, scale, "uniform64")
    idx.close()


def test_workload_uniform128_full():
    inp = synth.make_inputs("uniform128")
    idx, out = _run(inp.coords, inp.feats, inp.weights[0], 3)
    ref, scale = oracle_conv(inp.coords, inp.feats, inp.weights[0], 3)
    check_conv(out, ref, scale, "uniform128")
    useful, issued = idx.plan_stats()
    assert useful == int((native.neighbor_map(inp.coords) >= 0).sum())
    idx.close()


def test_workload_shells512_sampled():
    inp = synth.make_inputs("shells512")
    idx, out = _run(inp.coords, inp.feats, inp.weights[0], 3)
    rows = sample_rows(inp.n, 40_000, seed=1)
    ref, scale = oracle_conv(inp.coords, inp.feats, inp.weights[0], 3, rows=rows)
    check_conv(out[torch.from_numpy(rows).to(DEV)], ref, scale, "shells512")
    idx.close()


def test_workload_resblock64_pair_sampled():
    inp = synth.make_inputs("resblock64")
    c = torch.from_numpy(inp.coords).to(DEV)
    idx = SubMIndex(c)
    h = idx.forward(inp.feats.to(DEV), inp.weights[0].to(DEV), K=3)
    y = idx.forward(h, inp.weights[1].to(DEV), K=1)
    torch.cuda.synchronize()
    assert idx.status() == 0
    nbr = native.neighbor_map(inp.coords)
    rows = sample_rows(inp.n, 3000, seed=2)
    r_idx = torch.from_numpy(rows).to(DEV)
    ref, scale = native.submconv(inp.feats.double().numpy(), inp.weights[0].double().numpy(), nbr,
                                 rows=rows)
    check_conv(h[r_idx], ref, scale, "resblock 3x3x3")
    # the 1x1x1 layer is checked on the exact bf16 input the GPU produced
    h_cpu = h.double().cpu().numpy()
    ident = np.arange(inp.n, dtype=np.int32)[:, None]
    ref1, scale1 = native.submconv(h_cpu, inp.weights[1].double().numpy(), ident, rows=rows)
    check_conv(y[r_idx], ref1, scale1, "resblock 1x1x1")
    idx.close()


@pytest.mark.parametrize("cout", [64, 128, 256])
def test_many_single_stage_work_items(cout):
    """Isolated voxels give one-tap tiles (one or two pipeline stages per work
    item); the kernel must hand items to every role without waiting on later
    items."""
    pts = np.array([[b, 3 * i, 3 * j, 3 * k] for b in range(2) for i in range(12)
                    for j in range(12) for k in range(12)], np.int32)
    rng = np.random.default_rng(41 + cout)
    feats = synth.round_to(rng.standard_normal((len(pts), 64)), "bf16")
    W = synth.round_to(rng.standard_normal((27, 64, cout)) / 8.0, "bf16")
    idx, out = _run(pts, feats, W, 3)
    ref, scale = oracle_conv(pts, feats, W, 3)
    check_conv(out, ref, scale, f"isolated cout={cout}")
    idx.close()


_GROUP1_SCRIPT = r"""
import sys, numpy as np, torch
sys.path.insert(0, {root!r}); sys.path.insert(0, {tests!r})
from submanifold_sparse_convolution_coord_b200 import synth
from submanifold_sparse_convolution_coord_b200.binding import SubMIndex
from gpu_common import check_conv, oracle_conv
cases = [(0, 3000, 20, 1, 128, 128, "f16"), (1, 800, 40, 2, 64, 64, "bf16"), (2, 2000, 16, 1, 64, 128, "f16"),
         (3, 900, 14, 1, 192, 256, "bf16"), (4, 1500, 30, 2, 128, 64, "f16")]
for seed, n, grid, batch, cin, cout, dt in cases:
    coords, feats, W = synth.random_case(seed, n, grid, batch, cin, cout, 3, dt, True)
    idx = SubMIndex(torch.from_numpy(coords).cuda())
    out = idx.forward(feats.cuda(), W.cuda())
    W1 = synth.round_to(np.random.default_rng(seed).standard_normal((1, cin, cout)) / cin ** 0.5, dt)
    out1 = idx.forward(feats.cuda(), W1.cuda(), K=1)
    torch.cuda.synchronize()
    assert idx.status() == 0
    ref, scale = oracle_conv(coords, feats, W, 3)
    check_conv(out, ref, scale, str((seed, cin, cout)))
    ref1, scale1 = oracle_conv(coords, feats, W1, 1)
    check_conv(out1, ref1, scale1, str((seed, cin, cout, "K1")))
    idx.close()
print("ok")
"""


@pytest.mark.parametrize("override", [("SMC_TC_GROUP", "1"), ("SMC_TC_GROUP", "2"),
                                      ("SMC_TC_BK", "32")])
def test_tuning_override_configurations(override):
    """The kernel configurations behind the tuning overrides (one tile per work
    item; 32-channel stages with 64-byte swizzle), each in a fresh process
    since the settings are read once per process."""
    import os
    import subprocess
    import sys
    here = os.path.dirname(os.path.abspath(__file__))
    code = _GROUP1_SCRIPT.format(root=os.path.dirname(here), tests=here)
    env = dict(os.environ, **{override[0]: override[1]})
    r = subprocess.run([sys.executable, "-c", code], env=env, capture_output=True, text=True,
                       timeout=600)
    assert r.returncode == 0 and "ok" in r.stdout, r.stdout + r.stderr
