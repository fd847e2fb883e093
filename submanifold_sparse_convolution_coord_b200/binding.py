"""Thin ctypes binding of libsmc (C ABI in include/smc.h).

Every function here only marshals arguments: it checks tensor properties,
takes raw device pointers and the current CUDA stream from PyTorch, and calls
the C entry point of the same name.  All computation runs in libsmc's CUDA
kernels; there is no CPU path.  Importing works without a GPU (so the symbol
table can be checked anywhere); calls need the CUDA device the tensors live on.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libsmc.so")

SMC_OK = 0
STATUS = {
    0: "SMC_OK", -1: "SMC_ERR_INVALID", -2: "SMC_ERR_DUPLICATE", -3: "SMC_ERR_RANGE",
    -4: "SMC_ERR_OOM", -5: "SMC_ERR_CUDA", -6: "SMC_ERR_UNSUPPORTED", -7: "SMC_ERR_TABLE_FULL",
    -8: "SMC_ERR_TIMEOUT",
}
DTYPE_CODE = {torch.float32: 0, torch.float16: 1, torch.bfloat16: 2}
ORDER_CODE = {"mask": 0, "input": 1, "greedy": 2}
LOOKUP_CODE = {"hash": 0, "sort": 1}

# every symbol include/smc.h declares
EXPORTS = (
    "smc_build_index", "smc_build_index_ex", "smc_forward", "smc_get_neighbor_map",
    "smc_get_plan_stats", "smc_get_sizes", "smc_get_tile_plan", "smc_device_status",
    "smc_destroy", "smc_status_string", "smc_version", "smc_build_neighbor_map_static",
    "smc_backward_input", "smc_backward_weight", "smc_downsample2", "smc_subdivide2",
    "smc_forward_ex", "smc_autotune", "smc_conv_config_name", "smc_autotune_ex", "smc_replan",
)


class SmcError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {STATUS.get(status, status)} ({status_string(status)})")


ACT_CODE = {"none": 0, "relu": 1, "silu": 2, "gelu": 3}


class _Epilogue(ctypes.Structure):
    _fields_ = [("bias", ctypes.c_void_p), ("residual", ctypes.c_void_p),
                ("activation", ctypes.c_int32), ("reserved", ctypes.c_int32)]


class _Options(ctypes.Structure):
    _fields_ = [("table_capacity", ctypes.c_int64), ("order", ctypes.c_int32),
                ("lookup", ctypes.c_int32)]


_lib = None


def lib() -> ctypes.CDLL:
    """Load libsmc.so; raises if the library has not been built."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise RuntimeError(
            f"libsmc.so not found at {LIB_PATH}; build it with "
            "`python -m submanifold_sparse_convolution_coord_b200.csrc.build`")
    L = ctypes.CDLL(LIB_PATH)
    p, i64, i32, i = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int32, ctypes.c_int
    L.smc_build_index.argtypes = [p, i64, i32, ctypes.POINTER(p)]
    L.smc_build_index_ex.argtypes = [p, i64, i32, ctypes.POINTER(_Options), p, ctypes.POINTER(p)]
    L.smc_forward.argtypes = [p, p, p, p, i, i, i, i, p]
    L.smc_forward_ex.argtypes = [p, p, p, p, i, i, i, i, ctypes.POINTER(_Epilogue), p]
    L.smc_backward_input.argtypes = [p, p, p, p, i, i, i, i, p]
    L.smc_backward_weight.argtypes = [p, p, p, p, i, i, i, i, p]
    L.smc_downsample2.argtypes = [p, i64, p, i, i, p, p, ctypes.POINTER(i64), p]
    L.smc_subdivide2.argtypes = [p, i64, p, i, i, p, p, p]
    L.smc_get_neighbor_map.argtypes = [p, p, p]
    L.smc_get_plan_stats.argtypes = [p, ctypes.POINTER(i64), ctypes.POINTER(i64)]
    L.smc_get_sizes.argtypes = [p, ctypes.POINTER(i64), ctypes.POINTER(i64)]
    L.smc_get_tile_plan.argtypes = [p, p, p, p]
    L.smc_device_status.argtypes = [p, p]
    L.smc_destroy.argtypes = [p]
    L.smc_destroy.restype = None
    L.smc_status_string.argtypes = [i]
    L.smc_status_string.restype = ctypes.c_char_p
    L.smc_version.argtypes = []
    L.smc_build_neighbor_map_static.argtypes = [p, i64, i32, p, p]
    L.smc_autotune.argtypes = [p, p, p, p, i, i, i, i, p, ctypes.POINTER(i)]
    L.smc_autotune_ex.argtypes = [p, p, p, p, i, i, i, i, i, p, ctypes.POINTER(i),
                                  ctypes.POINTER(i)]
    L.smc_replan.argtypes = [p, i, p]
    L.smc_conv_config_name.argtypes = [i]
    L.smc_conv_config_name.restype = ctypes.c_char_p
    for name in EXPORTS:
        fn = getattr(L, name)
        if name not in ("smc_destroy", "smc_status_string", "smc_conv_config_name"):
            fn.restype = ctypes.c_int
    _lib = L
    return L


def status_string(status: int) -> str:
    return lib().smc_status_string(int(status)).decode()


def _check(rc: int, where: str) -> None:
    if rc != SMC_OK:
        raise SmcError(rc, where)


def _stream(stream: Optional[torch.cuda.Stream], device: torch.device) -> ctypes.c_void_p:
    s = stream if stream is not None else torch.cuda.current_stream(device)
    return ctypes.c_void_p(s.cuda_stream)


def _dev_ptr(t: torch.Tensor, name: str, dtype=None) -> int:
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if dtype is not None and t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, got {t.dtype}")
    return t.data_ptr()


# ----------------------------------------------------------------------------
# same-name wrappers
# ----------------------------------------------------------------------------
def smc_build_index(coords: torch.Tensor, stride: int = 1, table_capacity: int = 0,
                    order: str = "mask", stream: Optional[torch.cuda.Stream] = None,
                    lookup: str = "hash") -> int:
    """coords: CUDA int32 [N, 4] (b, x, y, z).  Returns the raw handle (int)."""
    if coords.dim() != 2 or coords.shape[1] != 4:
        raise ValueError("coords must be [N, 4]")
    ptr = _dev_ptr(coords, "coords", torch.int32)
    opts = _Options(int(table_capacity), ORDER_CODE[order], LOOKUP_CODE[lookup])
    h = ctypes.c_void_p()
    with torch.cuda.device(coords.device):  # the handle belongs to the coordinates' device
        rc = lib().smc_build_index_ex(ctypes.c_void_p(ptr), coords.shape[0], int(stride),
                                      ctypes.byref(opts), _stream(stream, coords.device),
                                      ctypes.byref(h))
    _check(rc, "smc_build_index")
    return h.value


def smc_forward(handle: int, feats: torch.Tensor, W: torch.Tensor, out: torch.Tensor, K: int,
                cin: int, cout: int, stream: Optional[torch.cuda.Stream] = None) -> None:
    dtype = feats.dtype
    if dtype not in DTYPE_CODE:
        raise ValueError(f"unsupported dtype {dtype}")
    fp = _dev_ptr(feats, "feats", dtype)
    wp = _dev_ptr(W, "W", dtype)
    op = _dev_ptr(out, "out", dtype)
    if W.device != feats.device or out.device != feats.device:
        raise ValueError("feats, W and out must be on one device")
    with torch.cuda.device(feats.device):  # the library checks it is the handle's device
        rc = lib().smc_forward(ctypes.c_void_p(handle), ctypes.c_void_p(fp), ctypes.c_void_p(wp),
                               ctypes.c_void_p(op), int(K), int(cin), int(cout),
                               DTYPE_CODE[dtype], _stream(stream, feats.device))
    _check(rc, "smc_forward")


def smc_autotune(handle: int, feats: torch.Tensor, W: torch.Tensor, out: torch.Tensor, K: int,
                 cin: int, cout: int, stream: Optional[torch.cuda.Stream] = None) -> int:
    """Time the valid launch configurations on these buffers and keep the
    fastest in the handle; returns its id (-1: CUDA cores).  out is
    overwritten with the forward result."""
    dtype = feats.dtype
    if dtype not in DTYPE_CODE:
        raise ValueError(f"unsupported dtype {dtype}")
    fp = _dev_ptr(feats, "feats", dtype)
    wp = _dev_ptr(W, "W", dtype)
    op = _dev_ptr(out, "out", dtype)
    if W.device != feats.device or out.device != feats.device:
        raise ValueError("feats, W and out must be on one device")
    chosen = ctypes.c_int(-1)
    with torch.cuda.device(feats.device):
        rc = lib().smc_autotune(ctypes.c_void_p(handle), ctypes.c_void_p(fp), ctypes.c_void_p(wp),
                                ctypes.c_void_p(op), int(K), int(cin), int(cout),
                                DTYPE_CODE[dtype], _stream(stream, feats.device),
                                ctypes.byref(chosen))
    _check(rc, "smc_autotune")
    return chosen.value


def smc_autotune_ex(handle: int, feats: torch.Tensor, W: torch.Tensor, out: torch.Tensor, K: int,
                    cin: int, cout: int, search_orders: bool = True,
                    stream: Optional[torch.cuda.Stream] = None) -> tuple:
    """smc_autotune, with the plan's row order searched as well; returns
    (configuration id, order name)."""
    dtype = feats.dtype
    if dtype not in DTYPE_CODE:
        raise ValueError(f"unsupported dtype {dtype}")
    fp = _dev_ptr(feats, "feats", dtype)
    wp = _dev_ptr(W, "W", dtype)
    op = _dev_ptr(out, "out", dtype)
    if W.device != feats.device or out.device != feats.device:
        raise ValueError("feats, W and out must be on one device")
    cfg, order = ctypes.c_int(-1), ctypes.c_int(-1)
    with torch.cuda.device(feats.device):
        rc = lib().smc_autotune_ex(ctypes.c_void_p(handle), ctypes.c_void_p(fp),
                                   ctypes.c_void_p(wp), ctypes.c_void_p(op), int(K), int(cin),
                                   int(cout), DTYPE_CODE[dtype], int(bool(search_orders)),
                                   _stream(stream, feats.device), ctypes.byref(cfg),
                                   ctypes.byref(order))
    _check(rc, "smc_autotune_ex")
    names = {v: k for k, v in ORDER_CODE.items()}
    return cfg.value, names.get(order.value, str(order.value))


def smc_replan(handle: int, order: str, device: torch.device,
               stream: Optional[torch.cuda.Stream] = None) -> None:
    with torch.cuda.device(device):
        rc = lib().smc_replan(ctypes.c_void_p(handle), ORDER_CODE[order], _stream(stream, device))
    _check(rc, "smc_replan")


def conv_config_name(config: int) -> str:
    return lib().smc_conv_config_name(int(config)).decode()


def smc_forward_ex(handle: int, feats: torch.Tensor, W: torch.Tensor, out: torch.Tensor, K: int,
                   cin: int, cout: int, bias: Optional[torch.Tensor] = None,
                   residual: Optional[torch.Tensor] = None, activation: str = "none",
                   stream: Optional[torch.cuda.Stream] = None) -> None:
    """smc_forward with the fused epilogue out = act(conv + bias) + residual."""
    dtype = feats.dtype
    if dtype not in DTYPE_CODE:
        raise ValueError(f"unsupported dtype {dtype}")
    fp = _dev_ptr(feats, "feats", dtype)
    wp = _dev_ptr(W, "W", dtype)
    op = _dev_ptr(out, "out", dtype)
    bp = _dev_ptr(bias, "bias", dtype) if bias is not None else None
    rp = _dev_ptr(residual, "residual", dtype) if residual is not None else None
    ep = _Epilogue(bp, rp, ACT_CODE[activation], 0)
    with torch.cuda.device(feats.device):
        rc = lib().smc_forward_ex(ctypes.c_void_p(handle), ctypes.c_void_p(fp), ctypes.c_void_p(wp),
                                  ctypes.c_void_p(op), int(K), int(cin), int(cout),
                                  DTYPE_CODE[dtype], ctypes.byref(ep), _stream(stream, feats.device))
    _check(rc, "smc_forward_ex")


def smc_backward_input(handle: int, grad_out: torch.Tensor, W: torch.Tensor,
                       grad_in: torch.Tensor, K: int, cin: int, cout: int,
                       stream: Optional[torch.cuda.Stream] = None) -> None:
    dtype = grad_out.dtype
    if dtype not in DTYPE_CODE:
        raise ValueError(f"unsupported dtype {dtype}")
    gp = _dev_ptr(grad_out, "grad_out", dtype)
    wp = _dev_ptr(W, "W", dtype)
    ip = _dev_ptr(grad_in, "grad_in", dtype)
    with torch.cuda.device(grad_out.device):
        rc = lib().smc_backward_input(ctypes.c_void_p(handle), ctypes.c_void_p(gp),
                                      ctypes.c_void_p(wp), ctypes.c_void_p(ip), int(K), int(cin),
                                      int(cout), DTYPE_CODE[dtype], _stream(stream, grad_out.device))
    _check(rc, "smc_backward_input")


def smc_backward_weight(handle: int, feats: torch.Tensor, grad_out: torch.Tensor,
                        dW: torch.Tensor, K: int, cin: int, cout: int,
                        stream: Optional[torch.cuda.Stream] = None) -> None:
    dtype = feats.dtype
    if dtype not in DTYPE_CODE:
        raise ValueError(f"unsupported dtype {dtype}")
    fp = _dev_ptr(feats, "feats", dtype)
    gp = _dev_ptr(grad_out, "grad_out", dtype)
    wp = _dev_ptr(dW, "dW", torch.float32)
    with torch.cuda.device(feats.device):
        rc = lib().smc_backward_weight(ctypes.c_void_p(handle), ctypes.c_void_p(fp),
                                       ctypes.c_void_p(gp), ctypes.c_void_p(wp), int(K), int(cin),
                                       int(cout), DTYPE_CODE[dtype], _stream(stream, feats.device))
    _check(rc, "smc_backward_weight")


def smc_downsample2(coords: torch.Tensor, feats: torch.Tensor,
                    stream: Optional[torch.cuda.Stream] = None) -> tuple:
    """x2 downsample by maximum: (parent coords int32 [M, 4], feats [M, C])."""
    if coords.dim() != 2 or coords.shape[1] != 4 or feats.dim() != 2 or \
            feats.shape[0] != coords.shape[0]:
        raise ValueError("coords must be [N, 4] and feats [N, C]")
    n, c = feats.shape
    cp = _dev_ptr(coords, "coords", torch.int32)
    fp = _dev_ptr(feats, "feats", feats.dtype)
    out_c = torch.empty((max(n, 1), 4), dtype=torch.int32, device=coords.device)
    out_f = torch.empty((max(n, 1), c), dtype=feats.dtype, device=coords.device)
    m = ctypes.c_int64(0)
    with torch.cuda.device(coords.device):
        rc = lib().smc_downsample2(ctypes.c_void_p(cp), n, ctypes.c_void_p(fp), int(c),
                                   DTYPE_CODE[feats.dtype], ctypes.c_void_p(out_c.data_ptr()),
                                   ctypes.c_void_p(out_f.data_ptr()), ctypes.byref(m),
                                   _stream(stream, coords.device))
    _check(rc, "smc_downsample2")
    return out_c[:m.value], out_f[:m.value]


def smc_subdivide2(coords: torch.Tensor, feats: torch.Tensor,
                   stream: Optional[torch.cuda.Stream] = None) -> tuple:
    """x2 subdivision: (child coords int32 [8N, 4], feats [8N, C])."""
    if coords.dim() != 2 or coords.shape[1] != 4 or feats.dim() != 2 or \
            feats.shape[0] != coords.shape[0]:
        raise ValueError("coords must be [N, 4] and feats [N, C]")
    n, c = feats.shape
    cp = _dev_ptr(coords, "coords", torch.int32)
    fp = _dev_ptr(feats, "feats", feats.dtype)
    out_c = torch.empty((max(8 * n, 1), 4), dtype=torch.int32, device=coords.device)
    out_f = torch.empty((max(8 * n, 1), c), dtype=feats.dtype, device=coords.device)
    with torch.cuda.device(coords.device):
        rc = lib().smc_subdivide2(ctypes.c_void_p(cp), n, ctypes.c_void_p(fp), int(c),
                                  DTYPE_CODE[feats.dtype], ctypes.c_void_p(out_c.data_ptr()),
                                  ctypes.c_void_p(out_f.data_ptr()), _stream(stream, coords.device))
    _check(rc, "smc_subdivide2")
    return out_c[:8 * n], out_f[:8 * n]


def smc_get_neighbor_map(handle: int, map_out: torch.Tensor,
                         stream: Optional[torch.cuda.Stream] = None) -> None:
    rc = lib().smc_get_neighbor_map(ctypes.c_void_p(handle),
                                    ctypes.c_void_p(_dev_ptr(map_out, "map", torch.int32)),
                                    _stream(stream, map_out.device))
    _check(rc, "smc_get_neighbor_map")


def smc_get_plan_stats(handle: int) -> tuple:
    u, s = ctypes.c_int64(), ctypes.c_int64()
    _check(lib().smc_get_plan_stats(ctypes.c_void_p(handle), ctypes.byref(u), ctypes.byref(s)),
           "smc_get_plan_stats")
    return u.value, s.value


def smc_get_sizes(handle: int) -> tuple:
    n, t = ctypes.c_int64(), ctypes.c_int64()
    _check(lib().smc_get_sizes(ctypes.c_void_p(handle), ctypes.byref(n), ctypes.byref(t)),
           "smc_get_sizes")
    return n.value, t.value


def smc_get_tile_plan(handle: int, perm: Optional[torch.Tensor], tile_mask: Optional[torch.Tensor],
                      stream: Optional[torch.cuda.Stream] = None) -> None:
    dev = (perm if perm is not None else tile_mask).device
    pp = _dev_ptr(perm, "perm", torch.int32) if perm is not None else None
    mp = _dev_ptr(tile_mask, "tile_mask", torch.int32) if tile_mask is not None else None
    rc = lib().smc_get_tile_plan(ctypes.c_void_p(handle), ctypes.c_void_p(pp),
                                 ctypes.c_void_p(mp), _stream(stream, dev))
    _check(rc, "smc_get_tile_plan")


def smc_device_status(handle: int, device=None, stream: Optional[torch.cuda.Stream] = None) -> int:
    dev = torch.device("cuda", torch.cuda.current_device()) if device is None else device
    return lib().smc_device_status(ctypes.c_void_p(handle), _stream(stream, dev))


def smc_destroy(handle: int) -> None:
    if handle:
        lib().smc_destroy(ctypes.c_void_p(handle))


def smc_version() -> int:
    return lib().smc_version()


# ----------------------------------------------------------------------------
# convenience object
# ----------------------------------------------------------------------------
class SubMIndex:
    """Owns one handle: the neighbour map and tile plan of a coordinate set
    (the cached indice map of the README's SparseTensor)."""

    def __init__(self, coords: torch.Tensor, stride: int = 1, table_capacity: int = 0,
                 order: str = "mask", lookup: str = "hash"):
        self.device = coords.device
        self.order = order
        self.handle = smc_build_index(coords, stride, table_capacity, order, lookup=lookup)
        self.n, self.n_tiles = smc_get_sizes(self.handle)

    def close(self) -> None:
        if getattr(self, "handle", None):
            smc_destroy(self.handle)
            self.handle = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    def __enter__(self):
        return self

    def __exit__(self, *exc):
        self.close()

    def neighbor_map(self) -> torch.Tensor:
        out = torch.empty((self.n, 27), dtype=torch.int32, device=self.device)
        smc_get_neighbor_map(self.handle, out)
        return out

    def plan_stats(self) -> tuple:
        return smc_get_plan_stats(self.handle)

    def tile_plan(self) -> tuple:
        perm = torch.empty(self.n, dtype=torch.int32, device=self.device)
        tmask = torch.empty(self.n_tiles, dtype=torch.int32, device=self.device)
        smc_get_tile_plan(self.handle, perm, tmask)
        return perm, tmask

    def status(self) -> int:
        return smc_device_status(self.handle, self.device)

    def autotune(self, feats: torch.Tensor, W: torch.Tensor, K: int = 3,
                 search_orders: bool = False) -> str:
        """Choose the fastest launch configuration for this layer shape on
        these inputs (kept for later forwards of the shape); with
        search_orders the plan's row order too (for the whole handle).
        Returns the configuration's name."""
        taps, cin, cout = W.shape
        if taps != K ** 3 or cin != feats.shape[1] or feats.shape[0] != self.n:
            raise ValueError("feats must be [N, Cin] and W [K^3, Cin, Cout]")
        out = torch.empty((self.n, cout), dtype=feats.dtype, device=feats.device)
        if search_orders:
            cfg, self.order = smc_autotune_ex(self.handle, feats, W, out, K, cin, cout, True)
            return conv_config_name(cfg)
        return conv_config_name(smc_autotune(self.handle, feats, W, out, K, cin, cout))

    def replan(self, order: str) -> None:
        """Rebuild the tile plan in another row order (the map is kept)."""
        smc_replan(self.handle, order, self.device)
        self.order = order

    def forward(self, feats: torch.Tensor, W: torch.Tensor, K: int = 3,
                out: Optional[torch.Tensor] = None, bias: Optional[torch.Tensor] = None,
                residual: Optional[torch.Tensor] = None, activation: str = "none") -> torch.Tensor:
        """act(conv(feats, W) + bias) + residual (the epilogue parts are optional)."""
        if feats.dim() != 2 or feats.shape[0] != self.n:
            raise ValueError("feats must be [N, Cin] for this index")
        taps, cin, cout = W.shape
        if taps != K ** 3 or cin != feats.shape[1]:
            raise ValueError("W must be [K^3, Cin, Cout]")
        if out is None:
            out = torch.empty((self.n, cout), dtype=feats.dtype, device=feats.device)
        if bias is None and residual is None and activation == "none":
            smc_forward(self.handle, feats, W, out, K, cin, cout)
        else:
            smc_forward_ex(self.handle, feats, W, out, K, cin, cout, bias, residual, activation)
        return out


    def backward_input(self, grad_out: torch.Tensor, W: torch.Tensor, K: int = 3,
                       out: Optional[torch.Tensor] = None) -> torch.Tensor:
        """Gradient of the forward with respect to feats, [N, Cin]."""
        taps, cin, cout = W.shape
        if taps != K ** 3 or grad_out.dim() != 2 or grad_out.shape != (self.n, cout):
            raise ValueError("grad_out must be [N, Cout] and W [K^3, Cin, Cout]")
        if out is None:
            out = torch.empty((self.n, cin), dtype=grad_out.dtype, device=grad_out.device)
        smc_backward_input(self.handle, grad_out, W, out, K, cin, cout)
        return out

    def backward_weight(self, feats: torch.Tensor, grad_out: torch.Tensor, K: int = 3,
                        out: Optional[torch.Tensor] = None) -> torch.Tensor:
        """Gradient of the forward with respect to W, float32 [K^3, Cin, Cout]."""
        if feats.dim() != 2 or grad_out.dim() != 2 or feats.shape[0] != self.n or \
                grad_out.shape[0] != self.n:
            raise ValueError("feats must be [N, Cin] and grad_out [N, Cout]")
        cin, cout = feats.shape[1], grad_out.shape[1]
        if out is None:
            out = torch.empty((K ** 3, cin, cout), dtype=torch.float32, device=feats.device)
        smc_backward_weight(self.handle, feats, grad_out, out, K, cin, cout)
        return out


def submconv3d(index: SubMIndex, feats: torch.Tensor, W: torch.Tensor, K: int = 3,
               out: Optional[torch.Tensor] = None) -> torch.Tensor:
    return index.forward(feats, W, K, out)
