"""Submanifold sparse 3-D convolution (SubMConv3d) for NVIDIA B200 (sm_100a).

The product is ``libsmc.so`` (C ABI: ``include/smc.h``); :mod:`.binding` is a
thin ctypes layer over it with the same function names, and :mod:`.synth`
draws the seeded synthetic inputs.
"""
from .binding import (SmcError, SubMIndex, lib, smc_backward_input,  # noqa: F401
                      smc_backward_weight, smc_build_index, smc_destroy, smc_device_status,
                      smc_downsample2, smc_forward, smc_forward_ex, smc_get_neighbor_map,
                      smc_get_plan_stats,
                      smc_get_sizes, smc_get_tile_plan, smc_subdivide2, smc_version, submconv3d)

__all__ = [
    "SmcError", "SubMIndex", "lib", "smc_backward_input", "smc_backward_weight",
    "smc_build_index", "smc_destroy", "smc_device_status", "smc_downsample2", "smc_subdivide2",
    "smc_forward", "smc_forward_ex", "smc_get_neighbor_map", "smc_get_plan_stats", "smc_get_sizes",
    "smc_get_tile_plan", "smc_version", "submconv3d",
]
