"""ctypes wrapper of the C++ oracle (``submconv_oracle.cpp``).

TEST INFRASTRUCTURE ONLY (see the package docstring).  ``build()`` compiles
the shared object with g++ and OpenMP next to the source; ``load()`` builds
on first use if it is missing or older than the source.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "submconv_oracle.cpp")
_LIB = os.path.join(_HERE, "libsubmconv_oracle.so")
_lib = None


def build(force: bool = False) -> str:
    if (not force and os.path.exists(_LIB)
            and os.path.getmtime(_LIB) >= os.path.getmtime(_SRC)):
        return _LIB
    cmd = ["g++", "-O2", "-std=c++17", "-fopenmp", "-shared", "-fPIC", _SRC, "-o", _LIB + ".tmp"]
    subprocess.run(cmd, check=True)
    os.replace(_LIB + ".tmp", _LIB)
    return _LIB


def load():
    global _lib
    if _lib is not None:
        return _lib
    build()
    lib = ctypes.CDLL(_LIB)
    i64, i32, p = ctypes.c_int64, ctypes.c_int32, ctypes.c_void_p
    lib.oracle_num_threads.restype = ctypes.c_int
    lib.oracle_neighbor_map.argtypes = [p, i64, i32, i32, p, p, p]
    lib.oracle_neighbor_map.restype = ctypes.c_int
    lib.oracle_submconv.argtypes = [p, p, p, i64, i32, i32, i32, p, i64, p, p, p]
    lib.oracle_submconv.restype = ctypes.c_int
    lib.oracle_submconv_backward_input.argtypes = [p, p, p, i64, i32, i32, i32, p, p, p]
    lib.oracle_submconv_backward_input.restype = ctypes.c_int
    lib.oracle_submconv_backward_weight.argtypes = [p, p, p, i64, i32, i32, i32, p, p, p]
    lib.oracle_submconv_backward_weight.restype = ctypes.c_int
    _lib = lib
    return lib


def _ptr(a: np.ndarray):
    return a.ctypes.data_as(ctypes.c_void_p)


def num_threads() -> int:
    return int(load().oracle_num_threads())


def neighbor_map(coords, K: int = 3, stride: int = 1, timings: dict | None = None) -> np.ndarray:
    """int32 [N, K^3] neighbour map (-1 = absent).  Raises on duplicates."""
    lib = load()
    c = np.ascontiguousarray(coords, dtype=np.int32)
    n = c.shape[0]
    out = np.empty((n, K ** 3), dtype=np.int32)
    t_dict = ctypes.c_double(0.0)
    t_query = ctypes.c_double(0.0)
    rc = lib.oracle_neighbor_map(_ptr(c), n, K, stride, _ptr(out),
                                 ctypes.byref(t_dict), ctypes.byref(t_query))
    if rc == -2:
        raise ValueError("duplicate coordinate")
    if rc != 0:
        raise ValueError(f"oracle_neighbor_map failed ({rc})")
    if timings is not None:
        timings["dict_ms"] = t_dict.value
        timings["query_ms"] = t_query.value
    return out


def submconv(feats, W, nbr, rows=None, want_scale: bool = True,
             timings: dict | None = None):
    """out (and scale) float64 [len(rows) or N, Cout] for the given rows."""
    lib = load()
    f = np.ascontiguousarray(feats, dtype=np.float64)
    w = np.ascontiguousarray(W, dtype=np.float64)
    m = np.ascontiguousarray(nbr, dtype=np.int32)
    n, cin = f.shape
    taps, wcin, cout = w.shape
    if wcin != cin or m.shape != (n, taps):
        raise ValueError("shape mismatch")
    if rows is None:
        nrows, rp = n, None
    else:
        r = np.ascontiguousarray(rows, dtype=np.int64)
        nrows, rp = r.shape[0], _ptr(r)
    out = np.empty((nrows, cout), dtype=np.float64)
    scale = np.empty((nrows, cout), dtype=np.float64) if want_scale else None
    t_conv = ctypes.c_double(0.0)
    rc = lib.oracle_submconv(_ptr(f), _ptr(w), _ptr(m), n, taps, cin, cout, rp, nrows,
                             _ptr(out), _ptr(scale) if want_scale else None,
                             ctypes.byref(t_conv))
    if rc != 0:
        raise ValueError(f"oracle_submconv failed ({rc})")
    if timings is not None:
        timings["conv_ms"] = t_conv.value
    return (out, scale) if want_scale else out


def submconv_backward_input(grad_out, W, nbr, want_scale: bool = True,
                            timings: dict | None = None):
    """Input gradient float64 [N, Cin] (and its error scale) of the
    convolution with weights W [taps, Cin, Cout] over the neighbour map nbr."""
    lib = load()
    g = np.ascontiguousarray(grad_out, dtype=np.float64)
    w = np.ascontiguousarray(W, dtype=np.float64)
    m = np.ascontiguousarray(nbr, dtype=np.int32)
    n, cout = g.shape
    taps, cin, wcout = w.shape
    if wcout != cout or m.shape != (n, taps):
        raise ValueError("shape mismatch")
    gin = np.empty((n, cin), dtype=np.float64)
    scale = np.empty((n, cin), dtype=np.float64) if want_scale else None
    t = ctypes.c_double(0.0)
    rc = lib.oracle_submconv_backward_input(_ptr(g), _ptr(w), _ptr(m), n, taps, cin, cout,
                                            _ptr(gin), _ptr(scale) if want_scale else None,
                                            ctypes.byref(t))
    if rc != 0:
        raise ValueError(f"oracle_submconv_backward_input failed ({rc})")
    if timings is not None:
        timings["bwd_input_ms"] = t.value
    return (gin, scale) if want_scale else gin


def submconv_backward_weight(feats, grad_out, nbr, want_scale: bool = True,
                             timings: dict | None = None):
    """Weight gradient float64 [taps, Cin, Cout] (and its error scale)."""
    lib = load()
    f = np.ascontiguousarray(feats, dtype=np.float64)
    g = np.ascontiguousarray(grad_out, dtype=np.float64)
    m = np.ascontiguousarray(nbr, dtype=np.int32)
    n, cin = f.shape
    gn, cout = g.shape
    taps = m.shape[1]
    if gn != n or m.shape[0] != n:
        raise ValueError("shape mismatch")
    dW = np.empty((taps, cin, cout), dtype=np.float64)
    scale = np.empty((taps, cin, cout), dtype=np.float64) if want_scale else None
    t = ctypes.c_double(0.0)
    rc = lib.oracle_submconv_backward_weight(_ptr(f), _ptr(g), _ptr(m), n, taps, cin, cout,
                                             _ptr(dW), _ptr(scale) if want_scale else None,
                                             ctypes.byref(t))
    if rc != 0:
        raise ValueError(f"oracle_submconv_backward_weight failed ({rc})")
    if timings is not None:
        timings["bwd_weight_ms"] = t.value
    return (dW, scale) if want_scale else dW
