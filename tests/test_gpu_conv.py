"""GPU SubMConv3d against the CPU oracle, element by element, through the C
ABI.  Tolerances are the ones stated in tests/gpu_common.py."""
import numpy as np
import pytest
import torch

from oracle import native
from submanifold_sparse_convolution_coord_b200 import synth
from submanifold_sparse_convolution_coord_b200.binding import SubMIndex

from gpu_common import check_conv, oracle_conv

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


def test_workload_shells512_full():
    """Every row of the 4.75 M-voxel two-scene shell layer against the oracle."""
    inp = synth.make_inputs("shells512")
    idx, out = _run(inp.coords, inp.feats, inp.weights[0], 3)
    ref, scale = oracle_conv(inp.coords, inp.feats, inp.weights[0], 3)
    check_conv(out, ref, scale, "shells512")
    useful, _ = idx.plan_stats()
    assert useful == int(np.count_nonzero(native.neighbor_map(inp.coords) >= 0))
    idx.close()


def test_workload_resblock64_pair_full():
    """Both layers of the channel-heavy block, every row: the 3x3x3 512->512
    conv, then the 1x1x1 512->1024 conv checked on the exact bf16 input the
    GPU produced for it."""
    inp = synth.make_inputs("resblock64")
    c = torch.from_numpy(inp.coords).to(DEV)
    idx = SubMIndex(c)
    h = idx.forward(inp.feats.to(DEV), inp.weights[0].to(DEV), K=3)
    y = idx.forward(h, inp.weights[1].to(DEV), K=1)
    torch.cuda.synchronize()
    assert idx.status() == 0
    nbr = native.neighbor_map(inp.coords)
    ref, scale = native.submconv(inp.feats.double().numpy(), inp.weights[0].double().numpy(), nbr)
    check_conv(h, ref, scale, "resblock 3x3x3")
    h_cpu = h.double().cpu().numpy()
    ident = np.arange(inp.n, dtype=np.int32)[:, None]
    ref1, scale1 = native.submconv(h_cpu, inp.weights[1].double().numpy(), ident)
    check_conv(y, ref1, scale1, "resblock 1x1x1")
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


@pytest.mark.parametrize("override", [("SMC_TC_GROUP", "1"), ("SMC_TC_GROUP", "2")])
def test_tuning_override_configurations(override):
    """The kernel configurations behind the tuning override (one or two tiles
    per work item), each in a fresh process since the setting is read once per
    process."""
    import os
    import subprocess
    import sys
    here = os.path.dirname(os.path.abspath(__file__))
    code = _GROUP1_SCRIPT.format(root=os.path.dirname(here), tests=here)
    env = dict(os.environ, **{override[0]: override[1]})
    r = subprocess.run([sys.executable, "-c", code], env=env, capture_output=True, text=True,
                       timeout=600)
    assert r.returncode == 0 and "ok" in r.stdout, r.stdout + r.stderr


def test_close_right_after_forward_on_side_stream():
    """Releasing a handle while its forward is still queued on a non-blocking
    side stream: the release waits for the device, so the output is intact
    and the memory handed back afterwards is not read by the finished kernel."""
    coords, feats, W = synth.random_case(50, 20000, 48, 1, 128, 128, 3, "f16")
    c = torch.from_numpy(coords).to(DEV)
    f, w = feats.to(DEV), W.to(DEV)
    side = torch.cuda.Stream()
    idx = SubMIndex(c)
    out = torch.empty((len(coords), 128), dtype=torch.float16, device=DEV)
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        for _ in range(3):
            idx.forward(f, w, out=out)
    idx.close()  # no synchronisation with the side stream before this
    junk = [torch.full((1 << 22,), -1, dtype=torch.int32, device=DEV) for _ in range(8)]
    torch.cuda.synchronize()
    ref, scale = oracle_conv(coords, feats, W, 3)
    check_conv(out, ref, scale, "close after side-stream forward")
    del junk


_ABORT_SCRIPT = r"""
import sys, numpy as np, torch
sys.path.insert(0, {root!r})
from submanifold_sparse_convolution_coord_b200 import synth
from submanifold_sparse_convolution_coord_b200.binding import SubMIndex
statuses = []
for seed, n, grid, cin, cout, K, dt in [(0, 20000, 48, 128, 128, 3, "f16"), (1, 3000, 24, 64, 64, 3, "bf16"),
                                        (2, 4000, 32, 512, 256, 1, "bf16")]:
    coords, feats, W = synth.random_case(seed, n, grid, 1, cin, cout, K, dt)
    idx = SubMIndex(torch.from_numpy(coords).cuda())
    for _ in range(3):
        idx.forward(feats.cuda(), W.cuda(), K=K)
    torch.cuda.synchronize()
    statuses.append(idx.status())
    idx.close()
print("statuses", statuses)
"""


@pytest.mark.parametrize("limit_ns,must_abort", [(200, True), (20000, False)])
def test_bounded_wait_abort_path(limit_ns, must_abort):
    """With the kernels' wait limit cut to a debug value (read once per
    process), waits give up mid-pipeline: the kernel must drain what it issued,
    free tensor memory, return, and report SMC_ERR_TIMEOUT through the status
    word, leaving the process's CUDA context usable.  A 200 ns limit makes the
    first unready wait give up; 20 us makes some CTAs give up and others not."""
    import os
    import subprocess
    import sys
    here = os.path.dirname(os.path.abspath(__file__))
    code = _ABORT_SCRIPT.format(root=os.path.dirname(here))
    env = dict(os.environ, SMC_DEBUG_WAIT_LIMIT_NS=str(limit_ns))
    r = subprocess.run([sys.executable, "-c", code], env=env, capture_output=True, text=True,
                       timeout=600)
    assert r.returncode == 0, r.stdout + r.stderr
    line = [ln for ln in r.stdout.splitlines() if ln.startswith("statuses")][0]
    statuses = eval(line.split(" ", 1)[1])
    assert all(s in (0, -8) for s in statuses), statuses  # SMC_OK or SMC_ERR_TIMEOUT only
    if must_abort:
        assert all(s == -8 for s in statuses), statuses
    # the normal limit, in this process: full parity
    coords, feats, W = synth.random_case(0, 20000, 48, 1, 128, 128, 3, "f16")
    idx, out = _run(coords, feats, W, 3)
    ref, scale = oracle_conv(coords, feats, W, 3)
    check_conv(out, ref, scale, "after abort runs")
    idx.close()


# (cin, cout, dtype, K): every launch configuration family appears in one of these
AUTOTUNE_SHAPES = [(128, 128, "f16", 3), (64, 64, "bf16", 3), (64, 128, "f16", 3),
                   (128, 256, "bf16", 3), (256, 256, "bf16", 1), (64, 256, "f16", 1)]


@pytest.mark.parametrize("shape", AUTOTUNE_SHAPES, ids=lambda s: "{}x{}_{}_K{}".format(*s))
def test_every_launch_configuration(shape, monkeypatch):
    """Each tensor-core launch configuration valid for the shape (forced
    through SMC_TC_CONFIG, read at every call) matches the oracle, and the
    configuration search picks a valid one whose forward matches too."""
    from submanifold_sparse_convolution_coord_b200 import binding
    cin, cout, dt, K = shape
    coords, feats, W = synth.random_case(50 + cin + cout, 3000, 24, 1, cin, cout, K, dt, True)
    ref, scale = oracle_conv(coords, feats, W, K)
    c = torch.from_numpy(np.ascontiguousarray(coords, dtype=np.int32)).to(DEV)
    idx = SubMIndex(c)
    f, w = feats.to(DEV), W.to(DEV)
    for cfg in range(11):
        monkeypatch.setenv("SMC_TC_CONFIG", str(cfg))
        out = idx.forward(f, w, K=K)
        torch.cuda.synchronize()
        assert idx.status() == 0
        check_conv(out, ref, scale, f"{shape} config {binding.conv_config_name(cfg)}")
    monkeypatch.delenv("SMC_TC_CONFIG")
    name = idx.autotune(f, w, K=K)
    assert name not in ("cuda-cores", "")
    out = idx.forward(f, w, K=K)
    torch.cuda.synchronize()
    assert idx.status() == 0
    check_conv(out, ref, scale, f"{shape} tuned {name}")
    idx.close()


def test_autotune_cuda_core_shapes():
    """fp32 (and off-grid channel counts) run on the CUDA cores: nothing to
    choose, and the forward is unchanged."""
    coords, feats, W = synth.random_case(61, 800, 12, 1, 16, 16, 3, "f32", True)
    c = torch.from_numpy(np.ascontiguousarray(coords, dtype=np.int32)).to(DEV)
    idx = SubMIndex(c)
    assert idx.autotune(feats.to(DEV), W.to(DEV), K=3) == "cuda-cores"
    ref, scale = oracle_conv(coords, feats, W, 3)
    check_conv(idx.forward(feats.to(DEV), W.to(DEV), K=3), ref, scale, "f32 after autotune")
    idx.close()
