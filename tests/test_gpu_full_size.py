"""Parity at the bench workload's full size (16 x 4096 x 2048 x 64, bf16,
fused conv and gating, the launch configuration bench.py times), on outputs
the oracle can compute separately: every per-channel output and gradient
(y, du, da, db, dz, dD, dconv) on sampled channels across all batch
elements (channels are independent given B and C), and the cross-channel
dB, dC completely for one batch element."""
import numpy as np
import pytest
import torch

import discrete_selective_ssm_b200 as naju
import oracle
from discrete_selective_ssm_b200.workloads import WORKLOADS, make_inputs
from naju_check import TOL_BF16, assert_close

pytestmark = pytest.mark.gpu

# channels spanning tiles, tile edges and both ends of d_inner
CHANNELS = [0, 1, 127, 128, 777, 1023, 1024, 2047]


def test_throughput_train_full_size_sampled():
    w = WORKLOADS["throughput_train"]
    t = make_inputs(w, which=("u", "a", "b", "B", "C", "z", "D", "conv_w", "conv_b", "dout"))
    g = {k: v.cuda() for k, v in t.items()}
    y, _, ws = naju.scan_fwd(g["u"], g["a"], g["b"], g["B"], g["C"], conv_w=g["conv_w"],
                             conv_b=g["conv_b"], z=g["z"], D=g["D"], out_dtype=naju.BF16)
    gr = naju.scan_bwd(g["dout"], g["u"], g["a"], g["b"], g["B"], g["C"], ws,
                       conv_w=g["conv_w"], conv_b=g["conv_b"], z=g["z"], D=g["D"],
                       out_dtype=naju.BF16)
    torch.cuda.synchronize()
    assert naju.last_device_status(ws) == 0
    ch = CHANNELS
    sl = lambda v: v[..., ch].contiguous()  # noqa: E731
    ro, _, _ = oracle.block_fwd(sl(t["u"]), t["conv_w"][ch], t["conv_b"][ch], sl(t["a"]),
                                sl(t["b"]), t["B"], t["C"], sl(t["z"]), t["D"][ch])
    assert_close(y[..., ch], ro, TOL_BF16, bf16_out=True, name="y")
    r = oracle.block_bwd(sl(t["u"]), t["conv_w"][ch], t["conv_b"][ch], sl(t["a"]), sl(t["b"]),
                         t["B"], t["C"], sl(t["z"]), t["D"][ch], None, sl(t["dout"]))
    for k, rk in (("dhu", "du"), ("da", "da"), ("db", "db"), ("dz", "dz")):
        assert_close(gr[k][..., ch], r[rk], TOL_BF16, bf16_out=True, name=k)
    assert_close(gr["dD"][ch], r["dD"], TOL_BF16, name="dD")
    assert_close(gr["dconv_w"][ch], r["dconv_w"], TOL_BF16, name="dconv_w")
    assert_close(gr["dconv_b"][ch], r["dconv_b"], TOL_BF16, name="dconv_b")
    # dB, dC sum over all 2048 channels: batch element 0 in full
    b0 = lambda v: v[:1].contiguous()  # noqa: E731
    r0 = oracle.block_bwd(b0(t["u"]), t["conv_w"], t["conv_b"], b0(t["a"]), b0(t["b"]),
                          b0(t["B"]), b0(t["C"]), b0(t["z"]), t["D"], None, b0(t["dout"]))
    assert_close(gr["dB"][:1], r0["dB"], TOL_BF16, bf16_out=True, name="dB")
    assert_close(gr["dC"][:1], r0["dC"], TOL_BF16, bf16_out=True, name="dC")
