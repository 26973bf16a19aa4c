"""The full Naju block around the library (Naju reproduction README, block
flowchart): normalized token -> input projection (u, z) -> causal depthwise
conv + SiLU (h) -> gate logits a, b and token directions B, C projected from
h -> native-discrete state scan with readout and feedthrough -> SiLU(z)
output modulation -> output projection -> residual.

The dense parts (RMSNorm, the projections: cuBLAS GEMMs through torch) are
plain library calls; the conv, the scan and their gradients run in this
package's kernels (h-mode scan, so the projections of h can add their own
gradient to dh before the conv backward).  Readings where the pages are
silent: RMSNorm with eps 1e-6; a, b, B, C are linear maps of h, with the
preserve-first biases forget_bias = 5 on a and write_bias = -2 on b (README
"Core equations") and no bias on B, C or the output projection.
`coupled=True` drops the b projection: i = 1 - f.
"""
from __future__ import annotations

import math

import torch

from . import _native as nj

EPS = 1e-6
PARAMS = ("norm_w", "W_in", "conv_w", "conv_b", "W_a", "b_a", "W_b", "b_b", "W_B", "W_C",
          "D", "W_out")
# parameters kept in fp32 whatever the activation dtype
_FP32 = ("norm_w", "conv_w", "conv_b", "b_a", "b_b", "D")


class NajuBlock:
    """Parameters live in `self.p` (CUDA tensors).  forward(x) returns
    (out, ctx); backward(ctx, dout) returns (dx, grads) with one gradient per
    parameter (fp32 for the fp32 parameters, the activation dtype otherwise)."""

    def __init__(self, d_model: int, d_inner: int, d_state: int, device, dtype=torch.bfloat16,
                 params: dict | None = None, seed: int = 0, coupled: bool = False):
        self.d_model, self.d_inner, self.d_state = d_model, d_inner, d_state
        self.dtype, self.coupled = dtype, coupled
        if params is None:
            params = init_params(d_model, d_inner, d_state, seed)
        self.p = {k: torch.as_tensor(v).to(device=device,
                                           dtype=torch.float32 if k in _FP32 else dtype)
                  .contiguous() for k, v in params.items()}

    # ------------------------------------------------------------ forward
    def forward(self, x: torch.Tensor):
        p, dt = self.p, self.dtype
        xf = x.float()
        r = torch.rsqrt(xf.pow(2).mean(-1, keepdim=True) + EPS)
        n = xf * r
        xn = (n * p["norm_w"]).to(dt)
        uz = xn @ p["W_in"]
        di = self.d_inner
        u, z = uz[..., :di].contiguous(), uz[..., di:].contiguous()
        h = nj.conv_silu_fwd(u, p["conv_w"], p["conv_b"])
        a = (h @ p["W_a"] + p["b_a"]).to(dt)
        b = None if self.coupled else (h @ p["W_b"] + p["b_b"]).to(dt)
        B = (h @ p["W_B"]).contiguous()
        C = (h @ p["W_C"]).contiguous()
        y, _, ws = nj.scan_fwd(h, a, b, B, C, z=z, D=p["D"], want_final=False)
        out = (xf + (y @ p["W_out"]).float()).to(x.dtype)
        ctx = dict(x=x, r=r, n=n, xn=xn, u=u, z=z, h=h, a=a, b=b, B=B, C=C, y=y, ws=ws)
        return out, ctx

    # ----------------------------------------------------------- backward
    def backward(self, ctx: dict, dout: torch.Tensor):
        p, dt, c = self.p, self.dtype, ctx
        flat = lambda t: t.reshape(-1, t.shape[-1])  # noqa: E731
        g = {}
        do = dout.to(dt)
        g["W_out"] = flat(c["y"]).t() @ flat(do)
        dy = (do @ p["W_out"].t()).contiguous()
        sg = nj.scan_bwd(dy, c["h"], c["a"], c["b"], c["B"], c["C"], c["ws"], z=c["z"],
                         D=p["D"], want_dx0=False)
        g["D"] = sg["dD"]
        dh = sg["dhu"].float() + (sg["da"] @ p["W_a"].t()).float() \
            + (sg["dB"] @ p["W_B"].t()).float() + (sg["dC"] @ p["W_C"].t()).float()
        g["W_a"] = flat(c["h"]).t() @ flat(sg["da"])
        g["b_a"] = flat(sg["da"]).float().sum(0)
        if self.coupled:
            g["W_b"] = torch.zeros_like(p["W_b"])
            g["b_b"] = torch.zeros_like(p["b_b"])
        else:
            dh = dh + (sg["db"] @ p["W_b"].t()).float()
            g["W_b"] = flat(c["h"]).t() @ flat(sg["db"])
            g["b_b"] = flat(sg["db"]).float().sum(0)
        g["W_B"] = flat(c["h"]).t() @ flat(sg["dB"])
        g["W_C"] = flat(c["h"]).t() @ flat(sg["dC"])
        du, g["conv_w"], g["conv_b"] = nj.conv_silu_bwd(c["u"], p["conv_w"], p["conv_b"],
                                                        dh.to(dt).contiguous())
        duz = torch.cat([du, sg["dz"]], dim=-1)
        g["W_in"] = flat(c["xn"]).t() @ flat(duz)
        dxn = (duz @ p["W_in"].t()).float()
        g["norm_w"] = flat(dxn * c["n"]).sum(0)
        dn = dxn * p["norm_w"]
        dx = c["r"] * (dn - c["n"] * (dn * c["n"]).mean(-1, keepdim=True))
        return (dout.float() + dx).to(dout.dtype), g


def init_params(d_model: int, d_inner: int, d_state: int, seed: int = 0) -> dict:
    """Seeded fp32 parameters (CPU tensors), scaled so activations stay O(1)."""
    gen = torch.Generator().manual_seed(seed)
    s_in, s_h = 1.0 / math.sqrt(d_model), 1.0 / math.sqrt(d_inner)
    rn = lambda *s: torch.randn(*s, generator=gen)  # noqa: E731
    return {
        "norm_w": 1.0 + 0.1 * rn(d_model),
        "W_in": rn(d_model, 2 * d_inner) * s_in,
        "conv_w": rn(d_inner, 4) * 0.5,
        "conv_b": rn(d_inner) * 0.1,
        "W_a": rn(d_inner, d_inner) * s_h,
        "b_a": torch.full((d_inner,), 5.0),
        "W_b": rn(d_inner, d_inner) * s_h,
        "b_b": torch.full((d_inner,), -2.0),
        "W_B": rn(d_inner, d_state) * s_h,
        "W_C": rn(d_inner, d_state) * s_h,
        "D": rn(d_inner),
        "W_out": rn(d_inner, d_model) * s_h,
    }
