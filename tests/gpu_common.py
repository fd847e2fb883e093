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


def check_conv(out_gpu: torch.Tensor, ref: np.ndarray, scale: np.ndarray, what: str = "",
               chunk: int = 1 << 18, input_dtype=None) -> dict:
    """Element-wise tolerance check of a GPU result against the oracle, in row
    chunks (full-size workloads hold millions of rows).  input_dtype, when the
    result is fp32 but its inputs were half precision (the weight gradient),
    selects the half-precision bound without an output-rounding term."""
    assert tuple(out_gpu.shape) == ref.shape, (tuple(out_gpu.shape), ref.shape)
    worst = 0.0
    n_bad = 0
    detail = []
    for r0 in range(0, ref.shape[0], chunk):
        out = as_f64(out_gpu[r0:r0 + chunk])
        rf, sc = ref[r0:r0 + chunk], scale[r0:r0 + chunk]
        assert np.all(np.isfinite(out)), f"{what}: non-finite output"
        err = np.abs(out - rf)
        if input_dtype in (torch.float16, torch.bfloat16):
            bound = HALF_TOL * sc  # fp32 result: its own rounding is far below the bound
        elif out_gpu.dtype == torch.float32:
            bound = F32_RTOL * np.abs(rf) + F32_FLOOR * sc
        else:
            bound = HALF_TOL * sc + UNIT_ROUNDOFF[out_gpu.dtype] * np.abs(rf)
        bad = err > bound
        if bad.any():
            n_bad += int(bad.sum())
            for i in np.argwhere(bad)[:5 - len(detail)]:
                detail.append(((r0 + int(i[0]), int(i[1])), float(out[tuple(i)]),
                               float(rf[tuple(i)]), float(sc[tuple(i)])))
        with np.errstate(divide="ignore", invalid="ignore"):
            ratio = np.where(sc > 0, err / sc, 0.0)
        if ratio.size:
            worst = max(worst, float(ratio.max()))
    if n_bad:
        raise AssertionError(f"{what}: {n_bad} elements out of tolerance, e.g. {detail}")
    return {"max_err_over_scale": worst}


def oracle_conv(coords: np.ndarray, feats: torch.Tensor, W: torch.Tensor, K: int, rows=None,
                nbr: np.ndarray | None = None, stride: int = 1):
    if nbr is None:
        nbr = native.neighbor_map(coords, K, stride)
    return native.submconv(as_f64(feats), as_f64(W), nbr, rows=rows)
