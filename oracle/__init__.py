"""Naju fp64 oracle -- test infrastructure, not part of the product.

A plain sequential double-precision CPU implementation of the Naju scan path
(causal depthwise conv + SiLU, the native-discrete selective recurrence, the
readout with feedthrough, the SiLU output modulation, their gradients and the
single-token decode step), written from the "Core equations" section and the
block flowchart of the Naju reproduction README (arXiv 2607.21000).

Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline
leg may import this package.  It shares no code with the CUDA path: the C
source here is compiled with gcc into its own shared library.

Every function takes and returns float64 numpy arrays in the layouts of
``naju_oracle.c``.  Optional inputs are ``None``.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "naju_oracle.c")
_LIB = os.path.join(_HERE, "_naju_oracle.so")
_lock = threading.Lock()
_lib = None


def build(force: bool = False) -> str:
    """Compile the oracle with gcc (-O2, OpenMP, strict IEEE: no fast-math)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(
            ["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-std=c11", "-fno-fast-math",
             "-ffp-contract=off", _SRC, "-o", tmp, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    with _lock:
        if _lib is None:
            lib = ctypes.CDLL(build())
            i64, dp = ctypes.c_int64, ctypes.c_void_p
            lib.naju_oracle_num_threads.restype = ctypes.c_int
            lib.naju_oracle_conv_silu_fwd.argtypes = [i64] * 4 + [dp] * 5
            lib.naju_oracle_conv_silu_bwd.argtypes = [i64] * 4 + [dp] * 7
            lib.naju_oracle_scan_fwd.argtypes = [i64] * 4 + [dp] * 11
            lib.naju_oracle_scan_bwd.argtypes = [i64] * 4 + [dp] * 18
            lib.naju_oracle_scan_step.argtypes = [i64] * 3 + [dp] * 9
            lib.naju_oracle_conv_silu_step.argtypes = [i64] * 3 + [dp] * 5
            for f in ("conv_silu_fwd", "conv_silu_bwd", "scan_fwd", "scan_bwd", "scan_step",
                      "conv_silu_step"):
                getattr(lib, "naju_oracle_" + f).restype = None
            _lib = lib
    return _lib


def _d(x):
    """Contiguous float64 copy (or None)."""
    if x is None:
        return None
    if hasattr(x, "detach"):  # torch tensor
        x = x.detach().to("cpu").double().numpy()
    return np.ascontiguousarray(x, dtype=np.float64)


def _p(x):
    return None if x is None else x.ctypes.data


def num_threads() -> int:
    return _load().naju_oracle_num_threads()


def conv_silu_fwd(u, w, bias=None, return_p: bool = False):
    """h = SiLU(causal depthwise conv(u)); u [Bt,L,d], w [d,W], bias [d]."""
    u, w, bias = _d(u), _d(w), _d(bias)
    Bt, L, d = u.shape
    W = w.shape[1]
    h = np.empty_like(u)
    p = np.empty_like(u) if return_p else None
    _load().naju_oracle_conv_silu_fwd(Bt, L, d, W, _p(u), _p(w), _p(bias), _p(p), _p(h))
    return (h, p) if return_p else h


def conv_silu_step(conv_state, u, w, bias=None):
    """One decode token of conv + SiLU.  conv_state [Bt,d,W-1] (previous
    inputs, oldest first), u [Bt,d].  Returns (h, new_conv_state); the input
    state is not modified."""
    cs = _d(conv_state).copy()
    u, w, bias = _d(u), _d(w), _d(bias)
    Bt, d = u.shape
    W = w.shape[1]
    h = np.empty_like(u)
    _load().naju_oracle_conv_silu_step(Bt, d, W, _p(u), _p(w), _p(bias), _p(cs), _p(h))
    return h, cs


def block_step(state, conv_state, u, conv_w, conv_b, a, b, B, C, z=None, D=None):
    """One decode token of the fused path: conv + SiLU step, then the scan
    step.  Returns (out, new_state, new_conv_state)."""
    h, cs = conv_silu_step(conv_state, u, conv_w, conv_b)
    out, st = scan_step(state, h, a, b, B, C, z, D)
    return out, st, cs


def conv_silu_bwd(u, w, bias, dh):
    """Returns (du, dw, dbias) for h = SiLU(conv(u)) given dh."""
    u, w, bias, dh = _d(u), _d(w), _d(bias), _d(dh)
    Bt, L, d = u.shape
    W = w.shape[1]
    du = np.empty_like(u)
    dw = np.empty_like(w)
    dbias = np.empty(d)
    _load().naju_oracle_conv_silu_bwd(Bt, L, d, W, _p(u), _p(w), _p(bias), _p(dh),
                                      _p(du), _p(dw), _p(dbias))
    return du, dw, dbias


def scan_fwd(h, a, b, B, C, z=None, D=None, x0=None, return_y_pre: bool = False):
    """Naju scan with readout and modulation.  Returns (out, xL) or
    (out, xL, y_pre)."""
    h, a, b, B, C, z, D, x0 = map(_d, (h, a, b, B, C, z, D, x0))
    Bt, L, d = h.shape
    N = B.shape[-1]
    out = np.empty_like(h)
    xL = np.empty((Bt, d, N))
    y_pre = np.empty_like(h) if return_y_pre else None
    _load().naju_oracle_scan_fwd(Bt, L, d, N, _p(h), _p(a), _p(b), _p(B), _p(C), _p(z),
                                 _p(D), _p(x0), _p(y_pre), _p(out), _p(xL))
    return (out, xL, y_pre) if return_y_pre else (out, xL)


def scan_bwd(h, a, b, B, C, z, D, x0, dout, dxL=None):
    """Gradients of scan_fwd.  Returns a dict with dh, da, db, dB, dC, dz, dD,
    dx0 (dz is None when z is None, dD is None when D is None)."""
    h, a, b, B, C, z, D, x0, dout, dxL = map(_d, (h, a, b, B, C, z, D, x0, dout, dxL))
    Bt, L, d = h.shape
    N = B.shape[-1]
    g = {k: np.empty_like(h) for k in ("dh", "da", "db")}
    g["dB"] = np.empty_like(B)
    g["dC"] = np.empty_like(C)
    g["dz"] = np.empty_like(h) if z is not None else None
    g["dD"] = np.empty(d) if D is not None else None
    g["dx0"] = np.empty((Bt, d, N))
    _load().naju_oracle_scan_bwd(Bt, L, d, N, _p(h), _p(a), _p(b), _p(B), _p(C), _p(z), _p(D),
                                 _p(x0), _p(dout), _p(dxL), _p(g["dh"]), _p(g["da"]),
                                 _p(g["db"]), _p(g["dB"]), _p(g["dC"]), _p(g["dz"]),
                                 _p(g["dD"]), _p(g["dx0"]))
    return g


def scan_step(state, h, a, b, B, C, z=None, D=None):
    """One decode step.  state [Bt,d,N]; h,a,b,z [Bt,d]; B,C [Bt,N].
    Returns (out, new_state); the input state is not modified."""
    state = _d(state).copy()
    h, a, b, B, C, z, D = map(_d, (h, a, b, B, C, z, D))
    Bt, d = h.shape
    N = B.shape[-1]
    out = np.empty_like(h)
    _load().naju_oracle_scan_step(Bt, d, N, _p(h), _p(a), _p(b), _p(B), _p(C), _p(z), _p(D),
                                  _p(state), _p(out))
    return out, state


def block_fwd(u, conv_w, conv_b, a, b, B, C, z=None, D=None, x0=None):
    """Fused block path: h = SiLU(conv(u)), then the scan.  Returns
    (out, xL, h)."""
    h = conv_silu_fwd(u, conv_w, conv_b)
    out, xL = scan_fwd(h, a, b, B, C, z, D, x0)
    return out, xL, h


def block_bwd(u, conv_w, conv_b, a, b, B, C, z, D, x0, dout, dxL=None):
    """Gradients of block_fwd: the scan gradients with dh replaced by du,
    plus dconv_w and dconv_b."""
    h = conv_silu_fwd(u, conv_w, conv_b)
    g = scan_bwd(h, a, b, B, C, z, D, x0, dout, dxL)
    du, dw, dbias = conv_silu_bwd(u, conv_w, conv_b, g["dh"])
    g["du"], g["dconv_w"], g["dconv_b"] = du, dw, dbias
    return g
