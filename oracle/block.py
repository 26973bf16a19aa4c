"""fp64 oracle of the full Naju block (test infrastructure only).

Block (Naju reproduction README, block flowchart): normalized token ->
input projection (u, z) -> causal depthwise conv + SiLU (h) -> gate logits
a, b and token directions B, C projected from h -> native-discrete state scan
with readout and feedthrough -> SiLU(z) output modulation -> output projection
-> residual.  Readings: RMSNorm (eps 1e-6) for the normalisation; a, b, B, C
are linear maps of h with biases forget_bias = 5 on a and write_bias = -2 on
b (README "Core equations"), none on B and C; the output projection has no
bias.  The conv and scan steps call this package's oracle; the rest is plain
numpy matrix algebra, and the backward is the chain rule written out.
"""
from __future__ import annotations

import numpy as np

from . import conv_silu_bwd, conv_silu_fwd, scan_bwd, scan_fwd

EPS = 1e-6
PARAMS = ("norm_w", "W_in", "conv_w", "conv_b", "W_a", "b_a", "W_b", "b_b", "W_B", "W_C",
          "D", "W_out")


def _f(v):
    return None if v is None else np.asarray(v, dtype=np.float64)


def block_fwd(x, p, coupled=False):
    """x [Bt, L, d_model]; p: dict of PARAMS.  Returns (out, cache)."""
    x = _f(x)
    p = {k: _f(v) for k, v in p.items()}
    ms = np.mean(x * x, axis=-1, keepdims=True)
    r = 1.0 / np.sqrt(ms + EPS)
    n = x * r
    xn = n * p["norm_w"]
    uz = xn @ p["W_in"]
    di = p["W_in"].shape[1] // 2
    u, z = uz[..., :di], uz[..., di:]
    h = conv_silu_fwd(u, p["conv_w"], p["conv_b"])
    a = h @ p["W_a"] + p["b_a"]
    b = None if coupled else h @ p["W_b"] + p["b_b"]
    B = h @ p["W_B"]
    C = h @ p["W_C"]
    y, _ = scan_fwd(h, a, b, B, C, z, p["D"])
    out = x + y @ p["W_out"]
    cache = dict(x=x, r=r, n=n, xn=xn, u=u, z=z, h=h, a=a, b=b, B=B, C=C, y=y, p=p)
    return out, cache


def block_bwd(cache, dout, coupled=False):
    """Gradients of block_fwd: returns (dx, dict of parameter gradients)."""
    c = cache
    p = c["p"]
    dout = _f(dout)
    g = {}
    flat = lambda t: t.reshape(-1, t.shape[-1])  # noqa: E731
    g["W_out"] = flat(c["y"]).T @ flat(dout)
    dy = dout @ p["W_out"].T
    sg = scan_bwd(c["h"], c["a"], c["b"], c["B"], c["C"], c["z"], p["D"], None, dy)
    g["D"] = sg["dD"]
    dh = sg["dh"] + sg["da"] @ p["W_a"].T + sg["dB"] @ p["W_B"].T + sg["dC"] @ p["W_C"].T
    g["W_a"] = flat(c["h"]).T @ flat(sg["da"])
    g["b_a"] = flat(sg["da"]).sum(0)
    if coupled:
        g["W_b"] = np.zeros_like(p["W_b"])
        g["b_b"] = np.zeros_like(p["b_b"])
    else:
        dh = dh + sg["db"] @ p["W_b"].T
        g["W_b"] = flat(c["h"]).T @ flat(sg["db"])
        g["b_b"] = flat(sg["db"]).sum(0)
    g["W_B"] = flat(c["h"]).T @ flat(sg["dB"])
    g["W_C"] = flat(c["h"]).T @ flat(sg["dC"])
    du, g["conv_w"], g["conv_b"] = conv_silu_bwd(c["u"], p["conv_w"], p["conv_b"], dh)
    duz = np.concatenate([du, sg["dz"]], axis=-1)
    g["W_in"] = flat(c["xn"]).T @ flat(duz)
    dxn = duz @ p["W_in"].T
    g["norm_w"] = flat(dxn * c["n"]).sum(0)
    dn = dxn * p["norm_w"]
    dx = c["r"] * (dn - c["n"] * np.mean(dn * c["n"], axis=-1, keepdims=True))
    return dout + dx, g


def init_params(d_model, d_inner, d_state, seed=0):
    """Seeded fp32 parameters (numpy), scaled so activations stay O(1)."""
    rng = np.random.default_rng(seed)
    s_in, s_h = 1.0 / np.sqrt(d_model), 1.0 / np.sqrt(d_inner)
    f32 = np.float32
    return {
        "norm_w": (1.0 + 0.1 * rng.normal(size=(d_model,))).astype(f32),
        "W_in": (rng.normal(size=(d_model, 2 * d_inner)) * s_in).astype(f32),
        "conv_w": (rng.normal(size=(d_inner, 4)) * 0.5).astype(f32),
        "conv_b": (rng.normal(size=(d_inner,)) * 0.1).astype(f32),
        "W_a": (rng.normal(size=(d_inner, d_inner)) * s_h).astype(f32),
        "b_a": np.full((d_inner,), 5.0, dtype=f32),
        "W_b": (rng.normal(size=(d_inner, d_inner)) * s_h).astype(f32),
        "b_b": np.full((d_inner,), -2.0, dtype=f32),
        "W_B": (rng.normal(size=(d_inner, d_state)) * s_h).astype(f32),
        "W_C": (rng.normal(size=(d_inner, d_state)) * s_h).astype(f32),
        "D": rng.normal(size=(d_inner,)).astype(f32),
        "W_out": (rng.normal(size=(d_inner, d_model)) * s_h).astype(f32),
    }
