"""Pins of the fused-epilogue oracle (act(conv + bias) + residual) against
PyTorch's own float64 activations and hand values."""
import numpy as np
import pytest
import torch

from oracle import submconv_ref as ref

TORCH_ACT = {"none": lambda t: t, "relu": torch.relu, "silu": torch.nn.functional.silu,
             "gelu": lambda t: torch.nn.functional.gelu(t, approximate="none")}


@pytest.mark.parametrize("act", ref.ACTIVATIONS)
def test_activation_matches_torch(act):
    v = np.linspace(-8.0, 8.0, 1601)
    want = TORCH_ACT[act](torch.tensor(v, dtype=torch.float64)).numpy()
    np.testing.assert_allclose(ref.activation(v, act), want, rtol=1e-14, atol=1e-15)


def test_hand_values():
    assert ref.activation(np.array([0.0]), "silu")[0] == 0.0
    assert ref.activation(np.array([0.0]), "gelu")[0] == 0.0
    assert ref.activation(np.array([-2.0, 3.0]), "relu").tolist() == [0.0, 3.0]
    # silu(1) = 1 / (1 + e^-1), gelu(1) = (1 + erf(1/sqrt 2)) / 2
    assert abs(ref.activation(np.array([1.0]), "silu")[0] - 0.7310585786300049) < 1e-15
    assert abs(ref.activation(np.array([1.0]), "gelu")[0] - 0.8413447460685429) < 1e-15


def test_epilogue_order():
    conv = np.array([[-1.0, 2.0]])
    bias = np.array([0.5, -3.0])
    res = np.array([[10.0, 20.0]])
    # relu(conv + bias) + residual = relu([-0.5, -1.0]) + [10, 20] = [10, 20]
    assert ref.epilogue(conv, bias, "relu", res).tolist() == [[10.0, 20.0]]
    # relu applied after the residual would give [9.5, 19.0]: the order is pinned
    assert ref.epilogue(conv, None, "none", res).tolist() == [[9.0, 22.0]]
    assert ref.epilogue(conv, bias).tolist() == [[-0.5, -1.0]]
