"""Helpers for the GPU parity tests: tolerance checks and oracle calls.

Tolerances (the bar each parity test applies):

* fp16 / bf16 features, fp32 accumulation, output in the feature dtype:
  |out - ref| <= 2e-3 * S + u * |ref| element-wise, S = sum_d |feats[c+d]| @
  |W[d]|.  2e-3 * S bounds the products and the fp32 accumulation; u * |ref|
  is the one rounding of the stored result to the output dtype (unit
  roundoff u = 2^-11 for fp16, 2^-8 for bf16), which 2e-3 * S alone does not
  cover for bf16 when |ref| > 0.51 S (few-term sums, e.g. isolated voxels);
* fp32 features: |out - ref| <= 1e-5 * |ref| + 1e-12 * S element-wise
  (the CUDA-core kernel accumulates in fp64 and rounds once to fp32).

``ref`` and ``S`` come from the C++ oracle fed the very values the GPU saw,
widened to float64.
"""
import numpy as np
import torch

from oracle import native

HALF_TOL = 2e-3
UNIT_ROUNDOFF = {torch.float16: 2.0 ** -11, torch.bfloat16: 2.0 ** -8}
F32_RTOL = 1e-5
F32_FLOOR = 1e-12


def as_f64(t: torch.Tensor) -> np.ndarray:
    return t.detach().to("cpu", torch.float64).numpy()


def check_conv(out_gpu: torch.Tensor, ref: np.ndarray, scale: np.ndarray, what: str = "") -> dict:
    out = as_f64(out_gpu)
    assert out.shape == ref.shape, (out.shape, ref.shape)
    assert np.all(np.isfinite(out)), f"{what}: non-finite output"
    err = np.abs(out - ref)
    if out_gpu.dtype == torch.float32:
        bound = F32_RTOL * np.abs(ref) + F32_FLOOR * scale
    else:
        bound = HALF_TOL * scale + UNIT_ROUNDOFF[out_gpu.dtype] * np.abs(ref)
    bad = err > bound
    if bad.any():
        idx = np.argwhere(bad)[:5]
        detail = [(tuple(int(v) for v in i), float(out[tuple(i)]), float(ref[tuple(i)]),
                   float(scale[tuple(i)])) for i in idx]
        raise AssertionError(f"{what}: {int(bad.sum())} elements out of tolerance, e.g. {detail}")
    with np.errstate(divide="ignore", invalid="ignore"):
        ratio = np.where(scale > 0, err / scale, 0.0)
    return {"max_err_over_scale": float(ratio.max()) if ratio.size else 0.0}


def oracle_conv(coords: np.ndarray, feats: torch.Tensor, W: torch.Tensor, K: int, rows=None,
                nbr: np.ndarray | None = None, stride: int = 1):
    if nbr is None:
        nbr = native.neighbor_map(coords, K, stride)
    return native.submconv(as_f64(feats), as_f64(W), nbr, rows=rows)


def sample_rows(n: int, count: int, seed: int = 0) -> np.ndarray:
    """Sorted sample of row ids that always includes the first and last rows."""
    if count >= n:
        return np.arange(n, dtype=np.int64)
    rng = np.random.default_rng(seed)
    rows = rng.choice(n, size=count, replace=False)
    rows = np.unique(np.concatenate([rows, [0, n - 1]]))
    return rows.astype(np.int64)
