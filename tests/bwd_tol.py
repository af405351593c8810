"""Tolerances for the bf16 tensor-core backward products (dX, dW).

Two criteria, both checked:

* the stated limit for bf16 GEMMs: max|gpu - ref| <= 2e-2 * max|ref| per
  output tensor;
* an elementwise bound from fp32 accumulation: the products of bf16 (or
  ternary) operands are exact in fp32, so each output may differ from the
  fp64 reference only by the rounding of its sums,
      |gpu - ref| <= K * u * sum|a||b| + u * |ref|,   u = 2^-24,
  with sum|a||b| the sum of the absolute products behind that output.  K
  covers the tensor core's internal adds, the fp32 running sum over the
  K blocks and split-K atomics; it is far below the size of a dropped
  block of the reduction, a wrong split-K partial or a wrong row.

The elementwise median relative error over outputs with ref != 0 is returned
and recorded, and must stay below MEDIAN_REL_MAX.
"""
import numpy as np

import oracle

REL_BWD = 2e-2
U32 = 2.0 ** -24
K_ACC = 512
MEDIAN_REL_MAX = 1e-4


def abs_dx(dy_bits: np.ndarray, weff: np.ndarray, gamma) -> np.ndarray:
    """gamma * |dY| . |W_eff| (fp64): the absolute products behind dX."""
    dy = np.abs(oracle.bf16_to_f32(dy_bits).astype(np.float64))
    return float(gamma) * (dy @ np.abs(weff.astype(np.float64)))


def abs_dw(dy_bits: np.ndarray, x_bits: np.ndarray) -> np.ndarray:
    """|dY|^T . |X| (fp64): the absolute products behind dW."""
    dy = np.abs(oracle.bf16_to_f32(dy_bits).astype(np.float64))
    x = np.abs(oracle.bf16_to_f32(x_bits).astype(np.float64))
    return dy.T @ x


def check_bwd(gpu: np.ndarray, ref: np.ndarray, absb: np.ndarray, what: str, record=None) -> float:
    g = gpu.astype(np.float64)
    r = ref.astype(np.float64)
    d = np.abs(g - r)
    scale = np.abs(r).max() if r.size else 0.0
    assert d.max(initial=0.0) <= REL_BWD * scale, f"{what}: max err {d.max()} vs {REL_BWD} * {scale}"
    lim = K_ACC * U32 * absb + U32 * np.abs(r) + 1e-30
    bad = d > lim
    if bad.any():
        i = np.unravel_index(np.argmax(d / lim), d.shape)
        raise AssertionError(f"{what}: {int(bad.sum())} outputs outside the accumulation bound; worst at {i}: "
                             f"gpu {g[i]} ref {r[i]} bound {lim[i]}")
    nz = r != 0
    med = float(np.median(d[nz] / np.abs(r[nz]))) if nz.any() else 0.0
    assert med <= MEDIAN_REL_MAX, f"{what}: median relative error {med}"
    if record is not None:
        record(f"median_rel_err {what}", med)
    return med
