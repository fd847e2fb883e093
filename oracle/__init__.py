"""CPU oracle for the submanifold sparse 3-D convolution (SubMConv3d).

TEST INFRASTRUCTURE ONLY.  Nothing in the product path may import, call, link
or execute anything in this package; only ``tests/``, ``__graft_entry__.smoke``
and ``bench.py``'s CPU-baseline / reference arm use it.  It shares no code with
the CUDA library: no kernels, headers, tables, packing or helpers.

Two implementations of the same plain definition:

* :mod:`oracle.submconv_ref`  -- Python, a dict of coordinate tuples and a
  per-voxel, per-offset loop accumulating in float64 (small inputs).
* :mod:`oracle.native`        -- C++ (``submconv_oracle.cpp``), the same
  algorithm written separately with ``std::unordered_map`` and OpenMP over
  voxels, for the full-size workloads and for the timed CPU baseline.

The definition both follow is the one the trellis_sparse_mlx README gives in
"What's in it" (SubMConv3d, submanifold 3x3x3 and 1x1x1, output sites are the
input sites) and "Correctness" (cross-correlation: the output at voxel c
gathers feats[c + d] for offset d).
"""
