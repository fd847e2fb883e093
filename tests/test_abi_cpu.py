"""C-ABI checks that need no GPU: the library loads, exports every symbol the
header declares, and rejects bad arguments on the host before touching CUDA."""
import ctypes
import os
import re

import pytest

from submanifold_sparse_convolution_coord_b200 import binding

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "smc.h")


def _declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    names = re.findall(r"\b(smc_[a-z_0-9]+)\s*\(", text)
    return sorted(set(names))


@pytest.fixture(scope="module")
def L():
    from submanifold_sparse_convolution_coord_b200.csrc import build
    build.build()
    return binding.lib()


def test_header_and_binding_agree():
    assert sorted(binding.EXPORTS) == _declared_functions()


def test_every_declared_symbol_is_exported(L):
    for name in _declared_functions():
        assert hasattr(L, name), name


def test_status_strings(L):
    for code in binding.STATUS:
        s = binding.status_string(code)
        assert isinstance(s, str) and s
    assert binding.status_string(0) == "ok"
    assert binding.status_string(12345) == "unknown status"


def test_version(L):
    assert L.smc_version() >= 100


def test_host_side_argument_checks(L):
    h = ctypes.c_void_p()
    # null out_handle, negative n, zero stride: rejected before any CUDA call
    assert L.smc_build_index(None, 4, 1, None) == -1
    assert L.smc_build_index(None, -1, 1, ctypes.byref(h)) == -1
    assert h.value is None
    assert L.smc_build_index(None, 4, 1, ctypes.byref(h)) == -1
    assert L.smc_build_index(ctypes.c_void_p(0x1000), 4, 0, ctypes.byref(h)) == -1
    # misaligned coordinate pointer
    assert L.smc_build_index(ctypes.c_void_p(0x1004), 4, 1, ctypes.byref(h)) == -1
    # null handle
    assert L.smc_forward(None, None, None, None, 3, 64, 64, 1, None) == -1
    assert L.smc_get_neighbor_map(None, None, None) == -1
    assert L.smc_get_plan_stats(None, None, None) == -1
    assert L.smc_get_sizes(None, None, None) == -1
    assert L.smc_get_tile_plan(None, None, None, None) == -1
    assert L.smc_device_status(None, None) == -1
    L.smc_destroy(None)  # ignored


def test_no_cpu_fallback_in_binding():
    """The binding refuses CPU tensors instead of computing anything."""
    import torch
    with pytest.raises(ValueError):
        binding.smc_build_index(torch.zeros((3, 4), dtype=torch.int32))
