"""The allocation-free forward entry point.

naju_scan_fwd_noalloc exists for callers that cannot allocate device memory
(code running where no allocator is available, or a plugin that is handed
only its input and output buffers): its scratch is a fixed array inside the
library instead of a caller-allocated workspace.  These tests call it through
the C ABI and check that it reproduces naju_scan_fwd and the fp64 oracle on
two calls in a row (the second call must not see a stale ticket or flags left
by the first), over the optional inputs (coupled gate, unfused h input, no z)
and both output dtypes, and that a problem larger than the fixed scratch is
refused before any launch.

Collected last on purpose (file name), so that a failure here cannot stop a
run before the other tests have run.
"""
import ctypes

import pytest
import torch

import discrete_selective_ssm_b200 as naju
import oracle
from discrete_selective_ssm_b200 import _native
from discrete_selective_ssm_b200.workloads import WORKLOADS, make_inputs, scaled
from naju_check import TOL_BF16, TOL_F32, assert_close

pytestmark = pytest.mark.gpu
DEV = "cuda:0"


def _fn():
    L = naju.lib()
    f = L.naju_scan_fwd_noalloc
    f.argtypes = [ctypes.POINTER(_native.Dims)] + [ctypes.c_void_p] * 13
    f.restype = ctypes.c_int
    return f


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _case(N, dtype, Bt, L, d, seed, coupled=False, conv=True, use_z=True):
    w = scaled(WORKLOADS["mid_lm"], batch=Bt, seqlen=L, d_inner=d, d_state=N, dtype=dtype)
    t = make_inputs(w, which=("u", "a", "b", "B", "C", "z", "D", "conv_w", "conv_b", "x0"),
                    seed_offset=seed)
    if coupled:
        t["b"] = None
    if not conv:  # unfused: the input is h itself
        t["conv_w"] = t["conv_b"] = None
    if not use_z:
        t["z"] = None
    return {k: (None if v is None else v.to(DEV).contiguous()) for k, v in t.items()}


def _oracle(t):
    cpu = {k: (None if v is None else v.cpu()) for k, v in t.items()}
    if cpu["conv_w"] is not None:
        ro, rx, _ = oracle.block_fwd(cpu["u"], cpu["conv_w"], cpu["conv_b"], cpu["a"], cpu["b"],
                                     cpu["B"], cpu["C"], cpu["z"], cpu["D"], cpu["x0"])
    else:
        ro, rx = oracle.scan_fwd(cpu["u"], cpu["a"], cpu["b"], cpu["B"], cpu["C"], cpu["z"],
                                 cpu["D"], cpu["x0"])
    return ro, rx


def _noalloc(t, out_dtype):
    Bt, L, d = t["u"].shape
    N = t["B"].shape[-1]
    dims = naju.make_dims(Bt, L, d, N, naju.BF16 if t["u"].dtype == torch.bfloat16 else naju.F32,
                          out_dtype)
    y = torch.full((Bt, L, d), float("nan"), device=DEV,
                   dtype=torch.float32 if out_dtype == naju.F32 else torch.bfloat16)
    xf = torch.full((Bt, d, N), float("nan"), device=DEV)
    st = _fn()(ctypes.byref(dims), _ptr(t["u"]), _ptr(t["conv_w"]), _ptr(t["conv_b"]),
               _ptr(t["a"]), _ptr(t["b"]), _ptr(t["B"]), _ptr(t["C"]), _ptr(t["z"]),
               _ptr(t["D"]), _ptr(t["x0"]), _ptr(y), _ptr(xf),
               ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert st == 0, f"naju_scan_fwd_noalloc returned {st}"
    return y, xf


def _reference(t, out_dtype):
    y, xf, _ = naju.scan_fwd(t["u"], t["a"], t["b"], t["B"], t["C"], conv_w=t["conv_w"],
                             conv_b=t["conv_b"], z=t["z"], D=t["D"], x0=t["x0"],
                             out_dtype=out_dtype)
    return y, xf


@pytest.mark.parametrize("dtype,out_dtype,tol", [("bf16", naju.F32, TOL_BF16),
                                                 ("bf16", naju.BF16, TOL_BF16),
                                                 ("f32", naju.F32, TOL_F32)])
@pytest.mark.parametrize("variant", ["full", "coupled", "unfused", "no_z"])
def test_noalloc_matches_workspace_forward_and_oracle_twice(dtype, out_dtype, tol, variant):
    kw = {"coupled": variant == "coupled", "conv": variant != "unfused",
          "use_z": variant != "no_z"}
    first = _case(64, dtype, 2, 300, 200, seed=1, **kw)
    second = _case(128, dtype, 3, 170, 96, seed=2, **kw)
    bo = out_dtype == naju.BF16
    for t in (first, second):  # two calls in a row, different shapes
        y, xf = _noalloc(t, out_dtype)
        ry, rxf = _reference(t, out_dtype)
        torch.cuda.synchronize()
        assert_close(y, ry, tol, bf16_out=bo, name="y vs naju_scan_fwd")
        assert_close(xf, rxf, tol, name="x_final vs naju_scan_fwd")
        oy, ox = _oracle(t)
        assert_close(y, oy, tol, bf16_out=bo, name="y vs oracle")
        assert_close(xf, ox, tol, name="x_final vs oracle")
    # the first problem again, after the second has reused the scratch
    y, xf = _noalloc(first, out_dtype)
    torch.cuda.synchronize()
    oy, ox = _oracle(first)
    assert_close(y, oy, tol, bf16_out=bo, name="y (repeat) vs oracle")
    assert_close(xf, ox, tol, name="x_final (repeat) vs oracle")


def test_noalloc_refuses_problems_beyond_its_scratch():
    # 2^20 batch x 8 channel tiles (1024 channels, d_state 16) = 2^23 flags of
    # 4 bytes, plus the header: more than the 32 MiB scratch
    dims = naju.make_dims(1 << 20, 1, 1024, 16, naju.BF16)
    fake = ctypes.c_void_p(1 << 20)  # never dereferenced: refused on the host
    st = _fn()(ctypes.byref(dims), fake, None, None, fake, fake, fake, fake, None, None, None,
               fake, None, None)
    assert st == 2
