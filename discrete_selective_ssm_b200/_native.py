"""ctypes binding of libnaju.so (include/naju.h, include/naju_testing.h).

Argument marshalling only: every function here checks tensor placement,
dtype and contiguity, allocates outputs with torch on the inputs' device,
passes raw device pointers and the current CUDA stream to the C ABI, and
raises NajuError on a non-OK status.  All arithmetic runs in the library's
CUDA kernels; there is no host or PyTorch fallback.
"""
from __future__ import annotations

import ctypes
import os
import re
import threading
from typing import Optional

import torch

from . import build as _build

_HERE = os.path.dirname(os.path.abspath(__file__))
_ROOT = os.path.dirname(_HERE)
HEADERS = [os.path.join(_ROOT, "include", "naju.h"), os.path.join(_ROOT, "include",
                                                                  "naju_testing.h")]

F32, BF16 = 0, 1
_STATUS = {0: "ok", 1: "invalid argument", 2: "unsupported configuration", 3: "CUDA error",
           4: "inter-block wait timed out"}


class NajuError(RuntimeError):
    def __init__(self, status: int, where: str):
        super().__init__(f"{where}: {_STATUS.get(status, status)} (status {status})")
        self.status = status


class Dims(ctypes.Structure):
    _fields_ = [("batch", ctypes.c_int64), ("seqlen", ctypes.c_int64),
                ("d_inner", ctypes.c_int64), ("d_state", ctypes.c_int64),
                ("conv_width", ctypes.c_int32), ("dtype", ctypes.c_int32),
                ("out_dtype", ctypes.c_int32), ("reserved", ctypes.c_int32)]


_lock = threading.Lock()
_lib = None


def library_path() -> str:
    return _build.LIB


def lib(build_if_missing: bool = True):
    """The loaded library.  Raises if it is not built (never falls back)."""
    global _lib
    with _lock:
        if _lib is None:
            path = _build.LIB
            if not os.path.exists(path):
                if not build_if_missing:
                    raise RuntimeError(f"Naju CUDA library missing: {path}")
                _build.build()
            L = ctypes.CDLL(path)
            vp, i64, i32, sz = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int32, ctypes.c_size_t
            dp = ctypes.POINTER(Dims)
            L.naju_scan_workspace_bytes.argtypes = [dp]
            L.naju_scan_workspace_bytes.restype = sz
            L.naju_conv_silu_fwd.argtypes = [dp] + [vp] * 5
            L.naju_conv_silu_bwd.argtypes = [dp] + [vp] * 8
            L.naju_scan_fwd.argtypes = [dp] + [vp] * 13 + [sz, vp]
            L.naju_scan_bwd.argtypes = [dp] + [vp] * 23 + [sz, vp]
            L.naju_scan_step.argtypes = [i64, i64, i64, i32] + [vp] * 10
            L.naju_conv_silu_step.argtypes = [i64, i64, i32] + [vp] * 6
            L.naju_scan_step_conv.argtypes = [i64, i64, i64, i32] + [vp] * 13
            L.naju_last_device_status.argtypes = [vp, vp]
            L.naju_status_string.argtypes = [ctypes.c_int]
            L.naju_status_string.restype = ctypes.c_char_p
            L.naju_testing_set_wait_limit.argtypes = [i64]
            L.naju_testing_set_skip_publish.argtypes = [i32]
            L.naju_testing_set_fwd_groups.argtypes = [i32]
            L.naju_testing_fwd_groups.argtypes = [vp]
            L.naju_testing_fwd_groups.restype = i32
            L.naju_testing_set_bwd_groups.argtypes = [i32]
            L.naju_testing_set_fwd_impl.argtypes = [i32]
            L.naju_testing_fwd_impl.argtypes = [vp]
            L.naju_testing_fwd_impl.restype = i32
            L.naju_testing_set_bwd_impl.argtypes = [i32]
            L.naju_testing_bwd_impl.argtypes = [vp]
            L.naju_testing_bwd_impl.restype = i32
            L.naju_testing_bwd_groups.argtypes = [vp]
            L.naju_testing_bwd_groups.restype = i32
            L.naju_testing_set_bwd_pieces.argtypes = [i32]
            L.naju_testing_set_fwd_pieces.argtypes = [i32]
            L.naju_testing_fwd_pieces.argtypes = [vp]
            L.naju_testing_fwd_pieces.restype = i32
            L.naju_testing_bwd_pieces.argtypes = [vp]
            L.naju_testing_bwd_pieces.restype = i32
            for name in ("naju_conv_silu_fwd", "naju_conv_silu_bwd", "naju_scan_fwd",
                         "naju_scan_bwd", "naju_scan_step", "naju_conv_silu_step",
                         "naju_scan_step_conv", "naju_last_device_status"):
                getattr(L, name).restype = ctypes.c_int
            _lib = L
    return _lib


def declared_symbols() -> list[str]:
    """Function names declared in the public headers."""
    names = []
    for h in HEADERS:
        txt = open(h).read()
        txt = re.sub(r"/\*.*?\*/", "", txt, flags=re.S)
        names += re.findall(r"\b(naju_\w+)\s*\(", txt)
    return sorted(set(names))


# --------------------------------------------------------------- helpers
def _dt(t: torch.Tensor) -> int:
    if t.dtype == torch.float32:
        return F32
    if t.dtype == torch.bfloat16:
        return BF16
    raise TypeError(f"unsupported dtype {t.dtype}")


def _torch_dt(code: int):
    return torch.float32 if code == F32 else torch.bfloat16


def _ptr(t: Optional[torch.Tensor], name: str = "", dtype=None, device=None):
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if dtype is not None and t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if device is not None and t.device != device:
        raise ValueError(f"{name} is on {t.device}, expected {device}")
    return ctypes.c_void_p(t.data_ptr())


def _stream(stream=None):
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


def _check(st: int, where: str):
    if st != 0:
        raise NajuError(st, where)


def make_dims(batch, seqlen, d_inner, d_state, dtype: int, out_dtype: Optional[int] = None,
              conv_width: int = 4) -> Dims:
    return Dims(batch, seqlen, d_inner, d_state, conv_width, dtype,
                dtype if out_dtype is None else out_dtype, 0)


def workspace_bytes(dims: Dims) -> int:
    return int(lib().naju_scan_workspace_bytes(ctypes.byref(dims)))


def alloc_workspace(dims: Dims, device) -> torch.Tensor:
    n = workspace_bytes(dims)
    if n == 0:
        raise NajuError(1, "naju_scan_workspace_bytes")
    ws = torch.empty(n + 256, dtype=torch.uint8, device=device)
    off = (-ws.data_ptr()) % 256
    ws = ws[off:off + n]
    ws.zero_()
    return ws


# ------------------------------------------------------------- entry points
def conv_silu_fwd(u, conv_w, conv_b=None, out_dtype=None, stream=None):
    Bt, L, d = u.shape
    dims = make_dims(Bt, L, d, 16, _dt(u), out_dtype, conv_w.shape[1])
    h = torch.empty(u.shape, dtype=_torch_dt(dims.out_dtype), device=u.device)
    _check(lib().naju_conv_silu_fwd(ctypes.byref(dims), _ptr(u, "u"),
                                    _ptr(conv_w, "conv_w", torch.float32),
                                    _ptr(conv_b, "conv_b", torch.float32), _ptr(h), _stream(stream)),
           "naju_conv_silu_fwd")
    return h


def conv_silu_bwd(u, conv_w, conv_b, dh, stream=None):
    Bt, L, d = u.shape
    dims = make_dims(Bt, L, d, 16, _dt(u), None, conv_w.shape[1])
    du = torch.empty_like(u)
    dw = torch.empty_like(conv_w)
    db = torch.empty(d, dtype=torch.float32, device=u.device)
    _check(lib().naju_conv_silu_bwd(ctypes.byref(dims), _ptr(u, "u"),
                                    _ptr(conv_w, "conv_w", torch.float32),
                                    _ptr(conv_b, "conv_b", torch.float32),
                                    _ptr(dh, "dh", u.dtype), _ptr(du), _ptr(dw), _ptr(db),
                                    _stream(stream)), "naju_conv_silu_bwd")
    return du, dw, db


def scan_fwd(hu, a, b, B, C, *, conv_w=None, conv_b=None, z=None, D=None, x0=None,
             out_dtype=None, workspace=None, want_final=True, y=None, x_final=None,
             stream=None):
    """Returns (y, x_final, workspace).  `hu` is u when conv_w is given."""
    Bt, L, d = hu.shape
    N = B.shape[-1]
    dt = _dt(hu)
    dims = make_dims(Bt, L, d, N, dt, out_dtype)
    dev = hu.device
    for name, t in (("a", a), ("b", b), ("B", B), ("C", C), ("z", z)):
        if t is not None and t.dtype != hu.dtype:
            raise TypeError(f"{name} must have the activation dtype {hu.dtype}")
    if workspace is None:
        workspace = alloc_workspace(dims, dev)
    if y is None:
        y = torch.empty((Bt, L, d), dtype=_torch_dt(dims.out_dtype), device=dev)
    if x_final is None and want_final:
        x_final = torch.empty((Bt, d, N), dtype=torch.float32, device=dev)
    _check(lib().naju_scan_fwd(
        ctypes.byref(dims), _ptr(hu, "hu"), _ptr(conv_w, "conv_w", torch.float32),
        _ptr(conv_b, "conv_b", torch.float32), _ptr(a, "a"), _ptr(b, "b"), _ptr(B, "B"),
        _ptr(C, "C"), _ptr(z, "z"), _ptr(D, "D", torch.float32), _ptr(x0, "x0", torch.float32),
        _ptr(y, "y"), _ptr(x_final, "x_final", torch.float32), _ptr(workspace, "workspace"),
        ctypes.c_size_t(workspace.numel()), _stream(stream)), "naju_scan_fwd")
    return y, x_final, workspace


def scan_bwd(dy, hu, a, b, B, C, workspace, *, conv_w=None, conv_b=None, z=None, D=None,
             x0=None, dx_final=None, out_dtype=None, want_dx0=True, grads=None, stream=None):
    """Gradients of scan_fwd; `workspace` must hold that forward's checkpoints.
    Returns a dict: dhu, da, db, dB, dC, dz, dD, dconv_w, dconv_b, dx0."""
    Bt, L, d = hu.shape
    N = B.shape[-1]
    dims = make_dims(Bt, L, d, N, _dt(hu), out_dtype)
    dev = hu.device
    if grads is None:
        ot = _torch_dt(dims.out_dtype)
        grads = {
            "dhu": torch.empty((Bt, L, d), dtype=ot, device=dev),
            "da": torch.empty((Bt, L, d), dtype=ot, device=dev),
            "db": torch.empty((Bt, L, d), dtype=ot, device=dev) if b is not None else None,
            "dB": torch.empty((Bt, L, N), dtype=ot, device=dev),
            "dC": torch.empty((Bt, L, N), dtype=ot, device=dev),
            "dz": torch.empty((Bt, L, d), dtype=ot, device=dev) if z is not None else None,
            "dD": torch.empty(d, dtype=torch.float32, device=dev) if D is not None else None,
            "dconv_w": torch.empty_like(conv_w) if conv_w is not None else None,
            "dconv_b": torch.empty(d, dtype=torch.float32, device=dev)
            if conv_w is not None else None,
            "dx0": torch.empty((Bt, d, N), dtype=torch.float32, device=dev) if want_dx0 else None,
        }
    g = grads
    _check(lib().naju_scan_bwd(
        ctypes.byref(dims), _ptr(hu, "hu"), _ptr(conv_w, "conv_w", torch.float32),
        _ptr(conv_b, "conv_b", torch.float32), _ptr(a, "a"), _ptr(b, "b"), _ptr(B, "B"),
        _ptr(C, "C"), _ptr(z, "z"), _ptr(D, "D", torch.float32), _ptr(x0, "x0", torch.float32),
        _ptr(dy, "dy", hu.dtype), _ptr(dx_final, "dx_final", torch.float32), _ptr(g["dhu"]),
        _ptr(g["da"]), _ptr(g["db"]), _ptr(g["dB"]), _ptr(g["dC"]), _ptr(g["dz"]),
        _ptr(g["dD"]), _ptr(g["dconv_w"]), _ptr(g["dconv_b"]), _ptr(g["dx0"]),
        _ptr(workspace, "workspace"), ctypes.c_size_t(workspace.numel()), _stream(stream)),
        "naju_scan_bwd")
    return g


def scan_step(state, h, a, b, B, C, z=None, D=None, y=None, stream=None):
    """One decode step; `state` [Bt, d, N] fp32 is updated in place.  Returns y."""
    Bt, d = h.shape
    N = B.shape[-1]
    if y is None:
        y = torch.empty_like(h)
    _check(lib().naju_scan_step(Bt, d, N, _dt(h), _ptr(h, "h"), _ptr(a, "a"), _ptr(b, "b"),
                                _ptr(B, "B"), _ptr(C, "C"), _ptr(z, "z"),
                                _ptr(D, "D", torch.float32), _ptr(state, "state", torch.float32),
                                _ptr(y, "y"), _stream(stream)), "naju_scan_step")
    return y


def conv_silu_step(conv_state, u, conv_w, conv_b=None, h=None, stream=None):
    """Decode step of conv + SiLU; `conv_state` [Bt, d, 3] fp32 is updated in
    place (previous three inputs, oldest first).  Returns h."""
    Bt, d = u.shape
    if h is None:
        h = torch.empty_like(u)
    _check(lib().naju_conv_silu_step(Bt, d, _dt(u), _ptr(u, "u"),
                                     _ptr(conv_w, "conv_w", torch.float32),
                                     _ptr(conv_b, "conv_b", torch.float32),
                                     _ptr(conv_state, "conv_state", torch.float32),
                                     _ptr(h, "h"), _stream(stream)), "naju_conv_silu_step")
    return h


def scan_step_conv(state, conv_state, u, a, b, B, C, conv_w, conv_b=None, z=None, D=None,
                   y=None, stream=None):
    """One decode step from the pre-conv input u (conv + SiLU fused); `state`
    and `conv_state` are updated in place.  Returns y."""
    Bt, d = u.shape
    N = B.shape[-1]
    if y is None:
        y = torch.empty_like(u)
    _check(lib().naju_scan_step_conv(Bt, d, N, _dt(u), _ptr(u, "u"),
                                     _ptr(conv_w, "conv_w", torch.float32),
                                     _ptr(conv_b, "conv_b", torch.float32),
                                     _ptr(conv_state, "conv_state", torch.float32),
                                     _ptr(a, "a"), _ptr(b, "b"), _ptr(B, "B"), _ptr(C, "C"),
                                     _ptr(z, "z"), _ptr(D, "D", torch.float32),
                                     _ptr(state, "state", torch.float32), _ptr(y, "y"),
                                     _stream(stream)), "naju_scan_step_conv")
    return y


def last_device_status(workspace, stream=None) -> int:
    return int(lib().naju_last_device_status(_ptr(workspace, "workspace"), _stream(stream)))


def testing_set_wait_limit(polls: int):
    lib().naju_testing_set_wait_limit(int(polls))


def testing_set_skip_publish(skip: bool):
    lib().naju_testing_set_skip_publish(1 if skip else 0)


def testing_set_fwd_groups(groups: int):
    lib().naju_testing_set_fwd_groups(int(groups))


def testing_fwd_groups(dims: Dims) -> int:
    return int(lib().naju_testing_fwd_groups(ctypes.byref(dims)))


def testing_set_fwd_impl(impl: int):
    lib().naju_testing_set_fwd_impl(int(impl))


def testing_fwd_impl(dims: Dims) -> int:
    return int(lib().naju_testing_fwd_impl(ctypes.byref(dims)))


def testing_set_bwd_impl(impl: int):
    lib().naju_testing_set_bwd_impl(int(impl))


def testing_bwd_impl(dims: Dims) -> int:
    return int(lib().naju_testing_bwd_impl(ctypes.byref(dims)))


def testing_set_bwd_groups(groups: int):
    lib().naju_testing_set_bwd_groups(int(groups))


def testing_bwd_groups(dims: Dims) -> int:
    return int(lib().naju_testing_bwd_groups(ctypes.byref(dims)))


def testing_set_bwd_pieces(pieces: int):
    lib().naju_testing_set_bwd_pieces(int(pieces))


def testing_bwd_pieces(dims: Dims) -> int:
    return int(lib().naju_testing_bwd_pieces(ctypes.byref(dims)))


def testing_set_fwd_pieces(pieces: int):
    lib().naju_testing_set_fwd_pieces(int(pieces))


def testing_fwd_pieces(dims: Dims) -> int:
    return int(lib().naju_testing_fwd_pieces(ctypes.byref(dims)))


def testing_set_sm_count(sms: int):
    lib().naju_testing_set_sm_count(int(sms))


def testing_sm_count() -> int:
    return int(lib().naju_testing_sm_count())
