"""Tolerances used by every parity test.

* bf16 outputs (Y, dX, dA, dB), per element:
      |y - y_ref| <= 1e-2 * max|y_ref| + 1.6e-2 * |y_ref|
  with max taken over the whole reference tensor (or over the sampled part
  of it, when only rows are checked).
* merge: the merged bf16 weight is within one bf16 ULP of the exact value,
  plus the forward error bound of an fp32 accumulation of the r-term rank
  product and the add:  (r + 2) * 2**-24 * (|W| + |s| * (|B| @ |A|)).
  That second term only matters where W and s*B@A cancel to a value whose
  own bf16 ULP is below the fp32 rounding of the summands; everywhere else
  (|exact| >= (r+2) 2^-14 (|W| + |s| |B| @ |A|)) one ULP is required.
"""
from __future__ import annotations

import numpy as np

from oracle import ulp_bf16

ATOL_FRAC = 1e-2
RTOL = 1.6e-2


def lora_tol_check(y, y_ref, atol_frac: float = ATOL_FRAC, rtol: float = RTOL):
    """Return (ok, info) for the per-element bf16 output tolerance."""
    y = np.asarray(y, dtype=np.float64)
    y_ref = np.asarray(y_ref, dtype=np.float64)
    assert y.shape == y_ref.shape, (y.shape, y_ref.shape)
    if y_ref.size == 0:
        return True, dict(n=0)
    err = np.abs(y - y_ref)
    ymax = float(np.max(np.abs(y_ref)))
    bound = atol_frac * ymax + rtol * np.abs(y_ref)
    bad = ~(err <= bound)              # NaN in y counts as bad
    info = dict(n=int(y.size), n_bad=int(bad.sum()), max_err=float(np.nanmax(err)) if err.size else 0.0,
                max_ref=ymax, worst_ratio=float(np.nanmax(err / np.maximum(bound, 1e-300))))
    if bad.any():
        i = np.unravel_index(int(np.argmax(bad)), bad.shape)
        info["first_bad"] = dict(index=[int(v) for v in i], got=float(y[i]), ref=float(y_ref[i]))
    return (not bad.any()) and np.isfinite(y).all(), info


def merge_tol_check(w, w_exact, W_src, A, B, scale: float):
    """Return (ok, info) for the merge bound (all arguments float64 values)."""
    w = np.asarray(w, dtype=np.float64)
    w_exact = np.asarray(w_exact, dtype=np.float64)
    r = A.shape[0]
    acc_mag = np.abs(W_src) + abs(scale) * (np.abs(B) @ np.abs(A))
    bound = ulp_bf16(w_exact) + (r + 2) * 2.0 ** -24 * acc_mag
    err = np.abs(w - w_exact)
    bad = ~(err <= bound)
    ulps = err / ulp_bf16(w_exact)
    # where |exact| >= (r+2) 2^-14 acc_mag the fp32 accumulation error is at
    # most half a bf16 ULP of the result, so one ULP must hold there
    noncancel = np.abs(w_exact) >= (r + 2) * 2.0 ** -14 * acc_mag
    info = dict(n=int(w.size), n_bad=int(bad.sum()), max_err=float(err.max()) if err.size else 0.0,
                max_err_in_ulps=float(ulps.max()) if err.size else 0.0,
                max_ulps_noncancel=float(ulps[noncancel].max()) if noncancel.any() else 0.0,
                frac_noncancel=float(noncancel.mean()) if err.size else 1.0)
    return not bad.any(), info
