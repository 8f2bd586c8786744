"""fp64 CPU oracle for the fused LoRA linear layer.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` may import this module.  The product path
(the C-ABI library and its Python binding) never calls it, and it shares no
code with the CUDA kernels.

Every function is the plain definition written out in float64 with numpy; a
matrix product is the only library primitive used.  Inputs are the exact bf16
values the GPU sees, widened to float64 by this module's own bit conversion.

Sources (page title, section):

* fastaf 0.1.0, "Minimal LoRA fine-tuning with hand-written Triton kernels",
  section "FWD kernel speedup": the layer computes
  ``out = X @ W.T + (X @ A.T) @ B.T * scale`` with ``scale = alpha / r``.
* Same page, section "BWD kernel speedup": the backward produces the three
  gradients dA, dB, dX (W is frozen).  The page prints no formula; the
  gradients below follow from the forward formula by the chain rule.
* unsloth fork commit log, scripts/benchmarks/qwen3_flex_inference.py, the
  commit that replaces copy + merge_adapter with one ``addmm``: the merged
  weight is ``pristine + scaling * (B @ A)`` accumulated in fp32 and rounded
  once to bf16; the base weight stays bit-identical across perturb+refresh
  cycles when every refresh restores from the pristine copy, while a bf16
  merge/unmerge pair drifts.

Pins: every function here is checked in ``tests/test_oracle.py`` against
brute-force loops, a hand-computed example, finite differences, closed forms
and the invariants of the pages (B = 0, merged == unmerged, restore is
bit-identical, merge/unmerge drifts).  No function is unpinned.
"""
from __future__ import annotations

import numpy as np

__all__ = [
    "bf16_bits_to_f64", "f64_to_bf16_bits", "bf16_round", "scale_of",
    "lora_down", "lora_forward", "lora_backward", "lora_merge",
    "lora_merge_bf16", "peft_merge_unmerge_bf16", "restore_and_merge_bf16",
    "ulp_bf16",
]


# --------------------------------------------------------------------------
# bf16 <-> float64.  bf16 is the upper half of an IEEE float32.
# --------------------------------------------------------------------------

def bf16_bits_to_f64(bits) -> np.ndarray:
    """uint16 bf16 bit patterns -> float64 (exact widening)."""
    b = np.asarray(bits).astype(np.uint16).astype(np.uint32) << np.uint32(16)
    return b.view(np.float32).astype(np.float64)


def bf16_round(x) -> np.ndarray:
    """Round float64 values to the nearest bf16 value, ties to even.

    bf16 keeps 8 significant bits.  With x = m * 2**e and 0.5 <= |m| < 1
    (frexp), the rounded value is round_half_even(m * 2**8) * 2**(e - 8).
    Values here stay in the normal range (no overflow / subnormal handling).
    """
    x = np.asarray(x, dtype=np.float64)
    m, e = np.frexp(x)
    q = np.round(m * 256.0)            # numpy rounds half to even
    return np.ldexp(q, e - 8)


def f64_to_bf16_bits(x) -> np.ndarray:
    """float64 -> bf16 bit patterns, via bf16_round (exactly representable)."""
    y = bf16_round(x).astype(np.float32)           # exact: 8-bit significand
    return (y.view(np.uint32) >> np.uint32(16)).astype(np.uint16)


def ulp_bf16(x) -> np.ndarray:
    """Spacing of bf16 numbers at |x|: 2**(floor(log2|x|) - 7); 2**-133 at 0."""
    x = np.abs(np.asarray(x, dtype=np.float64))
    _, e = np.frexp(x)                 # x = m * 2**e, 0.5 <= m < 1
    u = np.ldexp(1.0, e - 8)
    return np.where(x == 0, np.ldexp(1.0, -133), u)


def _f64(a) -> np.ndarray:
    a = np.asarray(a)
    if a.dtype == np.uint16:
        return bf16_bits_to_f64(a)
    return a.astype(np.float64)


def scale_of(alpha: float, r: int) -> float:
    """scale = alpha / r (fastaf, "FWD kernel speedup")."""
    return float(alpha) / float(r)


# --------------------------------------------------------------------------
# Forward: out = X @ W.T + (X @ A.T) @ B.T * scale   (fastaf, FWD section)
# --------------------------------------------------------------------------

def lora_down(X, A, rows=None) -> np.ndarray:
    """T = X @ A.T, shape [M, r] (the LoRA down-projection, step 2 of the
    unfused forward in the fastaf FWD section)."""
    X = _f64(X)
    if rows is not None:
        X = X[np.asarray(rows)]
    return X @ _f64(A).T


def lora_forward(X, W, A, B, alpha: float, rows=None) -> np.ndarray:
    """Y = X @ W.T + scale * (X @ A.T) @ B.T in float64.

    ``rows`` restricts the result to those rows of X (the formula is row-wise
    in X, so this is the same definition evaluated on a subset).
    """
    X = _f64(X)
    if rows is not None:
        X = X[np.asarray(rows)]
    W, A, B = _f64(W), _f64(A), _f64(B)
    s = scale_of(alpha, A.shape[0])
    base = X @ W.T                      # step 1: base projection
    T = X @ A.T                         # step 2: down-projection
    up = T @ B.T                        # step 4: up-projection
    return base + up * s                # steps 5-6: scale, add


# --------------------------------------------------------------------------
# Backward for frozen W (chain rule on the forward formula)
#   dT = s * dY @ B,  dB = s * dY.T @ T,  dA = dT.T @ X,  dX = dY @ W + dT @ A
# --------------------------------------------------------------------------

def lora_backward(X, W, A, B, dY, alpha: float, dx_rows=None):
    """Return (dX, dA, dB) in float64.

    With Y = X W^T + s (X A^T) B^T and upstream gradient dY:
      T  = X A^T                      [M, r]   (recomputed, nothing saved)
      dT = s dY B                     [M, r]
      dB = s dY^T T                   [d_out, r]
      dA = dT^T X                     [r, d_in]
      dX = dY W + dT A                [M, d_in]
    ``dx_rows`` restricts dX to those rows; dA and dB always reduce over all M.
    """
    X, W, A, B, dY = _f64(X), _f64(W), _f64(A), _f64(B), _f64(dY)
    s = scale_of(alpha, A.shape[0])
    T = X @ A.T
    dT = s * (dY @ B)
    dB = s * (dY.T @ T)
    dA = dT.T @ X
    if dx_rows is None:
        dX = dY @ W + dT @ A
    else:
        idx = np.asarray(dx_rows)
        dX = dY[idx] @ W + dT[idx] @ A
    return dX, dA, dB


# --------------------------------------------------------------------------
# Merge (unsloth fork commit log: fused restore+merge via one addmm)
# --------------------------------------------------------------------------

def lora_merge(W_src, A, B, alpha: float) -> np.ndarray:
    """W' = W_src + scale * (B @ A), exact in float64 (before any rounding)."""
    W_src, A, B = _f64(W_src), _f64(A), _f64(B)
    s = scale_of(alpha, A.shape[0])
    return W_src + s * (B @ A)


def lora_merge_bf16(W_src, A, B, alpha: float) -> np.ndarray:
    """The merged weight rounded once to bf16 (returned as float64 values)."""
    return bf16_round(lora_merge(W_src, A, B, alpha))


def peft_merge_unmerge_bf16(W, A, B, alpha: float):
    """One merge + unmerge cycle done in bf16, the way the commit log says
    PEFT's pair behaves: add the delta and round, subtract it and round.

    Returns (W_merged, W_after_unmerge), both bf16 values as float64.  The
    second generally differs from W by an ULP here and there (the drift).
    """
    W = _f64(W)
    A, B = _f64(A), _f64(B)
    s = scale_of(alpha, A.shape[0])
    delta = s * (B @ A)
    merged = bf16_round(W + delta)
    back = bf16_round(merged - delta)
    return merged, back


def restore_and_merge_bf16(pristine, A, B, alpha: float):
    """Restore protocol: W_inf <- pristine (bit copy), then merge fresh from
    the pristine copy.  Returns (W_inf after restore, W_inf after merge);
    the pristine array itself is never written."""
    pristine = _f64(pristine)
    restored = pristine.copy()
    merged = lora_merge_bf16(restored, A, B, alpha)
    return restored, merged
