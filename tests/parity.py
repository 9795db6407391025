"""Comparison metrics for the CUDA path against the fp64 oracle.

Tolerances (the stated bar for this method): 1e-4 for fp32 inputs, 2e-2 for
bf16 inputs with fp32 state.  "Relative error" is taken row-wise in the
infinity norm, because elementwise ratios are unbounded where an entry is ~0:

* out: for each token row i, max_c |out_gpu - out_ref| / max_c |out_ref|, over
  rows whose denominator is well conditioned, |den_i| >= 1e-2 * sum_j |T(s_ij)|
  (T_P < 0 for some s when P is even, so den_i can cancel to ~0; the excluded
  count is reported and is small);
* state: for each (b, h, column), max over basis rows |dS| / max |S_ref|.
"""
import numpy as np

TOL = {"f32": 1e-4, "bf16": 2e-2}
KAPPA = 1e-2


def out_row_error(out_gpu, out_ref, den_ref, cond_ref, kappa=KAPPA):
    out_gpu = np.asarray(out_gpu, dtype=np.float64)
    diff = np.max(np.abs(out_gpu - out_ref), axis=-1)
    scale = np.max(np.abs(out_ref), axis=-1)
    rel = diff / np.maximum(scale, 1e-300)
    good = np.abs(den_ref) >= kappa * cond_ref
    finite = np.isfinite(out_gpu).all(axis=-1)
    assert finite[good].all(), "non-finite output on a well-conditioned row"
    return float(rel[good].max()) if good.any() else 0.0, int((~good).sum())


def state_col_error(S_gpu, S_ref):
    S_gpu = np.asarray(S_gpu, dtype=np.float64)
    diff = np.max(np.abs(S_gpu - S_ref), axis=-2)
    scale = np.max(np.abs(S_ref), axis=-2)
    return float(np.max(diff / np.maximum(scale, 1e-300)))
