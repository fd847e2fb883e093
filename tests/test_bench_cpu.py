"""Host-side arithmetic of bench.py (no GPU): the algorithmic byte counts the
roofline numbers are built from."""
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402


def test_conv_bytes_uniform128():
    # feats + out (209,715 x 128 fp16 each), 13,943 gather-index slots, W
    n, c, slots = 209715, 128, 13943
    expect = 2 * n * c * 2 + slots * 128 * 4 + 27 * c * c * 2
    assert bench.conv_bytes(n, c, c, 2, slots) == expect == 115397632


def test_index_build_bytes_counts_each_part():
    n, slots = 209715, 13943
    per_voxel = 28 + 128 + 92 + 16
    cap = 1 << 19  # smallest power of two >= 2 n
    assert bench.index_build_bytes(n, slots) == n * per_voxel + cap * 20 + slots * 1024
    # the greedy order adds one read of each sorted row and mask and the permutation write
    assert bench.index_build_bytes(n, slots, "greedy") - bench.index_build_bytes(n, slots) == 12 * n
    # the table never drops below 64 slots, and every part grows with its input
    assert bench.index_build_bytes(0, 0) == 64 * 20
    assert bench.index_build_bytes(n + 1, slots) > bench.index_build_bytes(n, slots)
    assert bench.index_build_bytes(n, slots + 1) - bench.index_build_bytes(n, slots) == 1024


def test_index_build_summary():
    s = bench.index_build_summary(1000, 10, 0.5, 6545.0)
    b = bench.index_build_bytes(1000, 10)
    assert s["algorithmic_bytes"] == b
    assert abs(s["gbs"] - b / 0.5e-3 / 1e9) < 1e-9
    assert abs(s["hbm_frac"] - s["gbs"] / 6545.0) < 1e-12
    assert bench.index_build_summary(1000, 10, 0.0, 6545.0)["gbs"] is None
