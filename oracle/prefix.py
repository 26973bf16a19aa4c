"""Second fp64 evaluation of the Naju scan, by parallel prefix over affine maps.

Test infrastructure (part of the oracle).  The Naju reproduction README,
section "Scope", states that the sequential recurrence is mathematically
equivalent to the paper's affine scan.  This module evaluates that affine
scan directly: each token is the affine map x -> f_n (.) x + i_n h_n B_n^T
(README, "Core equations"), maps are composed by a Hillis-Steele inclusive
prefix, and the readout is applied to the composed result.  It shares no
arithmetic with the sequential loop in ``naju_oracle.c``, so agreement of the
two pins the loop's indexing and the order of the gate products.
"""
from __future__ import annotations

import numpy as np


def _sigmoid(v):
    return 1.0 / (1.0 + np.exp(-v))


def scan_fwd_prefix(h, a, b, B, C, z=None, D=None, x0=None):
    """Returns (out, xL) like ``oracle.scan_fwd``; inputs float64 numpy."""
    h, a, b, B, C = (np.asarray(v, dtype=np.float64) for v in (h, a, b, B, C))
    Bt, L, d = h.shape
    N = B.shape[-1]
    f = _sigmoid(a)                                   # [Bt, L, d]
    i = _sigmoid(b)
    # Each token's map: multiplier A_n (per channel, broadcast over N) and
    # offset U_n = i_n h_n B_n^T.
    A = f[..., None] * np.ones((1, 1, 1, N))          # [Bt, L, d, N]
    U = (i * h)[..., None] * B[:, :, None, :]         # [Bt, L, d, N]
    # Inclusive prefix: after the loop, (A[n], U[n]) is map_n o ... o map_0.
    off = 1
    while off < L:
        A_prev = A[:, :-off]
        U_prev = U[:, :-off]
        A_new = A.copy()
        U_new = U.copy()
        # (later) o (earlier): x -> A_l (A_e x + U_e) + U_l
        A_new[:, off:] = A[:, off:] * A_prev
        U_new[:, off:] = A[:, off:] * U_prev + U[:, off:]
        A, U = A_new, U_new
        off *= 2
    init = np.zeros((Bt, d, N)) if x0 is None else np.asarray(x0, dtype=np.float64)
    x = A * init[:, None, :, :] + U                   # x_n for every n
    y = np.einsum("bldn,bln->bld", x, C) / np.sqrt(N)
    if D is not None:
        y = y + np.asarray(D, dtype=np.float64)[None, None, :] * h
    if z is not None:
        z = np.asarray(z, dtype=np.float64)
        y = y * (z * _sigmoid(z))
    return y, x[:, -1]
