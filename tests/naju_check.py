"""Comparison helpers shared by the GPU parity tests.

Tolerances (max|err| / max|ref| over each output tensor):
  * fp32 inputs:                                     1e-4
  * bf16 inputs, fp32 state, fp32 outputs:           3e-3
  * bf16 inputs with bf16 outputs: 3e-3 of max|ref| plus, per element, the
    half-ULP that storing the exact value in bf16 costs (at most 2^-8 |ref|).
    No bf16-output implementation can avoid that rounding: an exact result
    lying midway between two bf16 numbers just above a power of two already
    errs by 2^-8 relative, which is more than 3e-3.
"""
from __future__ import annotations

import numpy as np
import torch

TOL_F32 = 1e-4
TOL_BF16 = 3e-3
BF16_HALF_ULP = 2.0 ** -8


def to_np(t) -> np.ndarray:
    if isinstance(t, torch.Tensor):
        return t.detach().float().cpu().numpy().astype(np.float64)
    return np.asarray(t, dtype=np.float64)


def rel_err(got, ref) -> float:
    got, ref = to_np(got), to_np(ref)
    m = float(np.max(np.abs(ref))) if ref.size else 0.0
    if m == 0.0:
        return float(np.max(np.abs(got))) if got.size else 0.0
    return float(np.max(np.abs(got - ref))) / m


def assert_close(got, ref, tol: float, bf16_out: bool = False, name: str = ""):
    g, r = to_np(got), to_np(ref)
    assert g.shape == r.shape, f"{name}: shape {g.shape} vs {r.shape}"
    assert np.all(np.isfinite(g)), f"{name}: non-finite values"
    if r.size == 0:
        return 0.0
    m = float(np.max(np.abs(r)))
    allowed = tol * m + (BF16_HALF_ULP * np.abs(r) if bf16_out else 0.0)
    err = np.abs(g - r)
    bad = err > allowed
    if np.any(bad):
        i = np.unravel_index(np.argmax(err - allowed), err.shape)
        raise AssertionError(
            f"{name}: max|err|/max|ref| = {float(err.max()) / max(m, 1e-300):.3e} (tol {tol}); "
            f"worst at {i}: got {g[i]!r} ref {r[i]!r}")
    return float(err.max()) / max(m, 1e-300)
