"""Seeded synthetic inputs for the Naju scan, shared by tests and the bench.

This module holds no arithmetic of the method: it only draws random numbers
with the shapes and distributions of the workloads below and casts them to the
activation dtype.  The CUDA path and the fp64 oracle both consume exactly the
tensors it returns (the oracle reads the already-rounded bf16 values).

Distributions (second argument of N(.,.) is the standard deviation):
  u, h, z ~ N(0,1); a ~ N(mu_a, sd_a); b ~ N(mu_b, sd_b); B, C ~ N(0,1)
  [batch, L, d_state]; D ~ N(0,1) [d_inner]; conv weight ~ N(0, 0.25)
  [d_inner, 4]; conv bias 0; dout ~ N(0,1); zero initial state.
  mu_a = 5 and mu_b = -2 are the preserve-first biases of the Naju
  reproduction README (forget_bias=5, write_bias=-2).
  The long-horizon workload replaces a seeded 5% of (batch, token, channel)
  entries ("overwrite events") with a ~ N(-4,1), b ~ N(3,1).

Every tensor has its own generator seed (base seed, workload index, tensor
name), so any subset can be drawn without changing the others.
"""
from __future__ import annotations

import dataclasses
import zlib
from typing import Optional

import torch

BASE_SEED = 20261202


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    index: int
    batch: int
    seqlen: int
    d_inner: int
    d_state: int
    dtype: str                 # "f32" or "bf16": activation storage dtype
    a_mean: float = 5.0
    a_std: float = 1.0
    b_mean: float = -2.0
    b_std: float = 1.0
    overwrite_frac: float = 0.0
    backward: bool = True
    conv_width: int = 4
    decode_steps: int = 0      # > 0: single-token decode workload
    state0_std: float = 0.0    # decode initial state N(0, state0_std)

    @property
    def torch_dtype(self):
        return torch.float32 if self.dtype == "f32" else torch.bfloat16

    @property
    def tokens(self) -> int:
        return self.batch * max(self.seqlen, 1)


WORKLOADS = {
    w.name: w
    for w in [
        Workload("tiny_fwd_f32", 0, 1, 256, 64, 16, "f32", backward=False),
        Workload("small_lm", 1, 8, 512, 192, 16, "bf16"),
        Workload("mid_lm", 2, 8, 2048, 1536, 64, "bf16", a_std=1.5, b_std=1.5),
        Workload("long_retention", 3, 2, 8192, 2048, 128, "bf16", a_mean=6.0, a_std=0.5,
                 overwrite_frac=0.05),
        Workload("throughput_train", 4, 16, 4096, 2048, 64, "bf16"),
        Workload("throughput_decode", 4, 256, 0, 2048, 64, "bf16", backward=False,
                 decode_steps=1024, state0_std=0.1),
    ]
}


def _gen(w: Workload, what: str, seed_offset: int = 0) -> torch.Generator:
    g = torch.Generator(device="cpu")
    tag = zlib.crc32(f"{w.name}/{what}".encode())
    g.manual_seed((BASE_SEED + w.index) * 1_000_003 + tag + seed_offset * 7919)
    return g


def _normal(shape, mean, std, g) -> torch.Tensor:
    x = torch.randn(shape, generator=g, dtype=torch.float32)
    if std != 1.0:
        x.mul_(std)
    if mean != 0.0:
        x.add_(mean)
    return x


def scaled(w: Workload, **changes) -> Workload:
    """Same distributions, other sizes (parity tests at reduced size)."""
    return dataclasses.replace(w, **changes)


def make_inputs(w: Workload, which=("u", "a", "b", "B", "C", "z", "D", "conv_w", "conv_b", "dout"),
                seed_offset: int = 0) -> dict:
    """CPU tensors of the workload.  Activations are in the workload dtype;
    D, conv_w, conv_b, x0 are fp32."""
    Bt, L, d, N = w.batch, w.seqlen, w.d_inner, w.d_state
    act = (Bt, L, d)
    out = {}
    mask = None
    if w.overwrite_frac > 0 and ("a" in which or "b" in which):
        mask = torch.rand(act, generator=_gen(w, "mask", seed_offset)) < w.overwrite_frac
    for k in which:
        g = _gen(w, k, seed_offset)
        if k in ("u", "h", "z", "dout"):
            t = _normal(act, 0.0, 1.0, g)
        elif k == "a":
            t = _normal(act, w.a_mean, w.a_std, g)
            if mask is not None:
                t = torch.where(mask, _normal(act, -4.0, 1.0, _gen(w, "a_ow", seed_offset)), t)
        elif k == "b":
            t = _normal(act, w.b_mean, w.b_std, g)
            if mask is not None:
                t = torch.where(mask, _normal(act, 3.0, 1.0, _gen(w, "b_ow", seed_offset)), t)
        elif k in ("B", "C"):
            t = _normal((Bt, L, N), 0.0, 1.0, g)
        elif k == "D":
            out[k] = _normal((d,), 0.0, 1.0, g)
            continue
        elif k == "conv_w":
            out[k] = _normal((d, w.conv_width), 0.0, 0.25, g)
            continue
        elif k == "conv_b":
            out[k] = torch.zeros(d, dtype=torch.float32)
            continue
        elif k == "x0":
            out[k] = _normal((Bt, d, N), 0.0, 1.0, g)
            continue
        elif k == "dxL":
            out[k] = _normal((Bt, d, N), 0.0, 1.0, g)
            continue
        else:
            raise KeyError(k)
        out[k] = t.to(w.torch_dtype)
    return out


def decode_state0(w: Workload) -> torch.Tensor:
    """Initial fp32 state [batch, d_inner, d_state] of a decode workload."""
    return _normal((w.batch, w.d_inner, w.d_state), 0.0, w.state0_std, _gen(w, "state0"))


def decode_step_inputs(w: Workload, step: int) -> dict:
    """Per-token inputs of decode step ``step``: h, a, b, z [batch, d_inner]
    in the workload dtype, B, C [batch, d_state]."""
    Bt, d, N = w.batch, w.d_inner, w.d_state
    out = {}
    for k in ("h", "a", "b", "B", "C", "z"):
        g = _gen(w, f"step{k}", step + 1)
        if k == "a":
            t = _normal((Bt, d), w.a_mean, w.a_std, g)
        elif k == "b":
            t = _normal((Bt, d), w.b_mean, w.b_std, g)
        elif k in ("B", "C"):
            t = _normal((Bt, N), 0.0, 1.0, g)
        else:
            t = _normal((Bt, d), 0.0, 1.0, g)
        out[k] = t.to(w.torch_dtype)
    return out


def decode_D(w: Workload) -> torch.Tensor:
    return _normal((w.d_inner,), 0.0, 1.0, _gen(w, "D"))
