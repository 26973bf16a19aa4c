"""Parity at each workload's own stated size, in the launch configuration the
library picks for that shape by itself (no group, piece or implementation
override).

The scan (Naju reproduction README, "Core equations") is independent per
(batch element, channel) given B and C, so every per-channel output and
gradient (y, du, da, db, dz, dD, dconv) is checked on sampled channels across
all batch elements, the oracle computing those channels alone; the
cross-channel dB and dC are checked completely for batch element 0.  The two
smallest workloads are compared in full.

Each large workload runs once with fp32 outputs, which holds the arithmetic
itself to the plain tolerance (no bf16 storage rounding allowance), and the
bench workload once more with bf16 outputs, as the bench runs it.
"""
import numpy as np
import pytest
import torch

import discrete_selective_ssm_b200 as naju
import oracle
from discrete_selective_ssm_b200.workloads import (WORKLOADS, decode_D, decode_state0,
                                                   decode_step_inputs, make_inputs)
from naju_check import TOL_BF16, TOL_F32, assert_close

pytestmark = pytest.mark.gpu

KEYS = ("u", "a", "b", "B", "C", "z", "D", "conv_w", "conv_b", "dout")


def _sample_channels(d):
    """Channels spanning 128-channel tiles, tile edges and both ends."""
    cand = [0, 1, 127, 128, d // 2 - 1, d // 2, d - 129, d - 128, d - 2, d - 1]
    return sorted({c for c in cand if 0 <= c < d})


def _run(w, out_dtype):
    t = make_inputs(w, which=KEYS)
    g = {k: v.cuda() for k, v in t.items()}
    y, xf, ws = naju.scan_fwd(g["u"], g["a"], g["b"], g["B"], g["C"], conv_w=g["conv_w"],
                              conv_b=g["conv_b"], z=g["z"], D=g["D"], out_dtype=out_dtype)
    gr = None
    if w.backward:
        gr = naju.scan_bwd(g["dout"], g["u"], g["a"], g["b"], g["B"], g["C"], ws,
                           conv_w=g["conv_w"], conv_b=g["conv_b"], z=g["z"], D=g["D"],
                           out_dtype=out_dtype)
    torch.cuda.synchronize()
    assert naju.last_device_status(ws) == 0
    return t, y, xf, gr


def _tol(w):
    return TOL_F32 if w.dtype == "f32" else TOL_BF16


def _check_full(w, out_dtype):
    """Every output of the whole workload against the oracle."""
    t, y, xf, gr = _run(w, out_dtype)
    tol, bo = _tol(w), out_dtype == naju.BF16
    ro, rx, _ = oracle.block_fwd(t["u"], t["conv_w"], t["conv_b"], t["a"], t["b"], t["B"],
                                 t["C"], t["z"], t["D"])
    assert_close(y, ro, tol, bf16_out=bo, name="y")
    assert_close(xf, rx, tol, name="x_final")
    if gr is None:
        return
    r = oracle.block_bwd(t["u"], t["conv_w"], t["conv_b"], t["a"], t["b"], t["B"], t["C"],
                         t["z"], t["D"], None, t["dout"])
    for k, rk in (("dhu", "du"), ("da", "da"), ("db", "db"), ("dz", "dz"), ("dB", "dB"),
                  ("dC", "dC")):
        assert_close(gr[k], r[rk], tol, bf16_out=bo, name=k)
    for k in ("dD", "dconv_w", "dconv_b", "dx0"):
        assert_close(gr[k], r[k], tol, name=k)


def _check_sampled(w, out_dtype):
    """Per-channel outputs on sampled channels (all batch elements), dB / dC
    for batch element 0 in full, the final state on the sampled channels."""
    t, y, xf, gr = _run(w, out_dtype)
    tol, bo = _tol(w), out_dtype == naju.BF16
    ch = _sample_channels(w.d_inner)
    sl = lambda v: v[..., ch].contiguous()  # noqa: E731
    ro, rx, _ = oracle.block_fwd(sl(t["u"]), t["conv_w"][ch], t["conv_b"][ch], sl(t["a"]),
                                 sl(t["b"]), t["B"], t["C"], sl(t["z"]), t["D"][ch])
    assert_close(y[..., ch], ro, tol, bf16_out=bo, name="y")
    assert_close(xf[:, ch], rx, tol, name="x_final")
    r = oracle.block_bwd(sl(t["u"]), t["conv_w"][ch], t["conv_b"][ch], sl(t["a"]), sl(t["b"]),
                         t["B"], t["C"], sl(t["z"]), t["D"][ch], None, sl(t["dout"]))
    for k, rk in (("dhu", "du"), ("da", "da"), ("db", "db"), ("dz", "dz")):
        assert_close(gr[k][..., ch], r[rk], tol, bf16_out=bo, name=k)
    for k in ("dD", "dconv_w", "dconv_b"):
        assert_close(gr[k][ch], r[k], tol, name=k)
    assert_close(gr["dx0"][:, ch], r["dx0"], tol, name="dx0")
    b0 = lambda v: v[:1].contiguous()  # noqa: E731
    r0 = oracle.block_bwd(b0(t["u"]), t["conv_w"], t["conv_b"], b0(t["a"]), b0(t["b"]),
                          b0(t["B"]), b0(t["C"]), b0(t["z"]), t["D"], None, b0(t["dout"]))
    assert_close(gr["dB"][:1], r0["dB"], tol, bf16_out=bo, name="dB")
    assert_close(gr["dC"][:1], r0["dC"], tol, bf16_out=bo, name="dC")


def test_tiny_fwd_f32_full():
    """1 x 256 x 64 x 16, fp32, forward only: every output."""
    _check_full(WORKLOADS["tiny_fwd_f32"], naju.F32)


@pytest.mark.parametrize("out", ["f32", "bf16"])
def test_small_lm_full(out):
    """8 x 512 x 192 x 16, bf16, forward and backward: every output."""
    _check_full(WORKLOADS["small_lm"], naju.F32 if out == "f32" else naju.BF16)


def test_mid_lm_full_size_sampled():
    """8 x 2048 x 1536 x 64, bf16 (a wave-model group count)."""
    _check_sampled(WORKLOADS["mid_lm"], naju.F32)


def test_long_retention_full_size_sampled():
    """2 x 8192 x 2048 x 128, bf16, 5 % overwrite events (the longest
    accumulation chain and the most sequence groups)."""
    _check_sampled(WORKLOADS["long_retention"], naju.F32)


@pytest.mark.parametrize("out", ["f32", "bf16"])
def test_throughput_train_full_size_sampled(out):
    """16 x 4096 x 2048 x 64, bf16: the bench workload (piece mode)."""
    _check_sampled(WORKLOADS["throughput_train"], naju.F32 if out == "f32" else naju.BF16)


@pytest.mark.parametrize("conv", [False, True])
def test_throughput_decode_1024_steps(conv):
    """256 x 2048 x 64, 1024 sequential decode steps from the seeded N(0, 0.1)
    state: the final state and the last step's y on sampled batch rows (rows
    are independent) against the oracle's own 1024 steps.  conv=False is the
    plain step on h; conv=True the fused step on u with the conv state."""
    w = WORKLOADS["throughput_decode"]
    rows = [0, 1, 127, 128, 254, 255]
    state0 = decode_state0(w)
    D = decode_D(w)
    cw = make_inputs(w, which=("conv_w", "conv_b"))
    st = state0.cuda()
    cs = torch.zeros(w.batch, w.d_inner, 3, device="cuda")
    Dg = D.cuda()
    cwg = {k: v.cuda() for k, v in cw.items()}
    ref_st = state0[rows].double().numpy()
    ref_cs = np.zeros((len(rows), w.d_inner, 3))
    y = yo = None
    for k in range(w.decode_steps):
        s = decode_step_inputs(w, k)
        g = {kk: v.cuda(non_blocking=True) for kk, v in s.items()}
        if conv:
            y = naju.scan_step_conv(st, cs, g["h"], g["a"], g["b"], g["B"], g["C"],
                                    cwg["conv_w"], cwg["conv_b"], g["z"], Dg)
            yo, ref_st, ref_cs = oracle.block_step(ref_st, ref_cs, s["h"][rows], cw["conv_w"],
                                                   cw["conv_b"], s["a"][rows], s["b"][rows],
                                                   s["B"][rows], s["C"][rows], s["z"][rows], D)
        else:
            y = naju.scan_step(st, g["h"], g["a"], g["b"], g["B"], g["C"], g["z"], Dg)
            yo, ref_st = oracle.scan_step(ref_st, s["h"][rows], s["a"][rows], s["b"][rows],
                                          s["B"][rows], s["C"][rows], s["z"][rows], D)
    torch.cuda.synchronize()
    assert_close(st[rows], ref_st, TOL_BF16, name="state after 1024 steps")
    assert_close(y[rows], yo, TOL_BF16, bf16_out=True, name="y of step 1024")
    if conv:
        assert_close(cs[rows], ref_cs, 0.0, name="conv state")
