"""Pins of the fp64 oracle against facts the Naju pages and mathematics fix.

None of these tests uses the oracle's own loop as its expected value: each
expected value comes from a special case with a closed form, an unrolled sum
written independently of the recurrence, a library routine (torch conv1d), an
invariant stated on the pages, a second evaluation by affine prefix, or central
finite differences of the forward.
"""
import math
import os

import numpy as np
import pytest
import torch

import oracle
from oracle.prefix import scan_fwd_prefix

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def rnd(seed, *shape, mean=0.0, std=1.0):
    return np.random.default_rng(seed).normal(mean, std, size=shape)


def tiny(seed=0, Bt=2, L=7, d=3, N=4, x0=True):
    r = np.random.default_rng(seed)
    t = {
        "h": r.normal(size=(Bt, L, d)),
        "a": r.normal(2.0, 1.5, size=(Bt, L, d)),
        "b": r.normal(-1.0, 1.5, size=(Bt, L, d)),
        "B": r.normal(size=(Bt, L, N)),
        "C": r.normal(size=(Bt, L, N)),
        "z": r.normal(size=(Bt, L, d)),
        "D": r.normal(size=(d,)),
        "x0": r.normal(size=(Bt, d, N)) if x0 else None,
    }
    return t


def sig(v):
    return 1.0 / (1.0 + np.exp(-v))


def silu(v):
    return v * sig(v)


# ---------------------------------------------------------------- gate values
def test_preserve_first_gate_values():
    """sigma(5) and sigma(-2), the preserve-first biases (README, Core
    equations), read through the oracle's scan: with i == 0 (b = -800) a unit
    state decays once by f, and with f == 0 a unit write gives i."""
    rows = {}
    with open(os.path.join(GOLDEN, "preserve_first_gates.txt")) as fh:
        for line in fh:
            if line.strip() and not line.startswith("#"):
                name, logit, val = line.split()
                rows[name] = (float(logit), float(val))
    one = np.ones((1, 1, 1))
    # retain: x_1 = f * x0 with no write; y = x_1 * C / sqrt(1)
    out, _ = oracle.scan_fwd(0 * one, rows["forget_gate"][0] * one, -800 * one, one, one,
                             x0=np.ones((1, 1, 1)))
    assert out[0, 0, 0] == pytest.approx(rows["forget_gate"][1], rel=1e-15)
    # write: x_1 = i * h * B with f = 0; y = x_1 * C
    out, _ = oracle.scan_fwd(one, -800 * one, rows["write_gate"][0] * one, one, one)
    assert out[0, 0, 0] == pytest.approx(rows["write_gate"][1], rel=1e-15)
    assert round(rows["forget_gate"][1], 3) == 0.993  # README: trained mean retain 0.993


# ------------------------------------------------------------- special cases
def test_forget_zero_is_pure_write():
    """f == 0: x_n = i_n h_n B_n^T, so y_n = i_n h_n (B_n . C_n)/sqrt(N) + D h_n."""
    t = tiny(1)
    N = t["B"].shape[-1]
    a = np.full_like(t["a"], -800.0)
    out, xL = oracle.scan_fwd(t["h"], a, t["b"], t["B"], t["C"], t["z"], t["D"], t["x0"])
    i = sig(t["b"])
    BC = np.einsum("bln,bln->bl", t["B"], t["C"])[..., None]
    y = i * t["h"] * BC / math.sqrt(N) + t["D"] * t["h"]
    np.testing.assert_allclose(out, y * silu(t["z"]), rtol=1e-12, atol=1e-12)
    want_xL = (i * t["h"])[:, -1, :, None] * t["B"][:, -1, None, :]
    np.testing.assert_allclose(xL, want_xL, rtol=1e-12, atol=1e-12)


def test_write_zero_is_geometric_decay():
    """i == 0: x_n = (prod_{k<=n} f_k) x0."""
    t = tiny(2)
    N = t["B"].shape[-1]
    b = np.full_like(t["b"], -800.0)
    out, xL = oracle.scan_fwd(t["h"], t["a"], b, t["B"], t["C"], None, None, t["x0"])
    P = np.cumprod(sig(t["a"]), axis=1)                       # [Bt, L, d]
    x0C = np.einsum("bdn,bln->bld", t["x0"], t["C"])
    np.testing.assert_allclose(out, P * x0C / math.sqrt(N), rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(xL, P[:, -1, :, None] * t["x0"], rtol=1e-12, atol=1e-14)


def test_full_retain_full_write_is_running_sum():
    """f == i == 1 (a = b = 40, sigma = 1 in fp64): x_n = x0 + sum_m h_m B_m^T."""
    t = tiny(3)
    N = t["B"].shape[-1]
    big = np.full_like(t["a"], 40.0)
    assert sig(40.0) == 1.0
    out, xL = oracle.scan_fwd(t["h"], big, big, t["B"], t["C"], None, t["D"], t["x0"])
    S = np.cumsum(t["h"][..., None] * t["B"][:, :, None, :], axis=1)   # [Bt,L,d,N]
    x = t["x0"][:, None] + S
    y = np.einsum("bldn,bln->bld", x, t["C"]) / math.sqrt(N) + t["D"] * t["h"]
    np.testing.assert_allclose(out, y, rtol=1e-11, atol=1e-11)
    np.testing.assert_allclose(xL, x[:, -1], rtol=1e-12, atol=1e-12)


def test_unrolled_closed_form_brute_force():
    """y_n[d] = sum_{m<=n} (prod_{k=m+1..n} f_k[d]) i_m[d] h_m[d] (B_m . C_n)/sqrt(N)
               + (prod_{k<=n} f_k[d]) (x0[d] . C_n)/sqrt(N) + D[d] h_n[d]."""
    for seed, (Bt, L, d, N) in enumerate([(1, 1, 1, 1), (2, 12, 3, 4), (1, 9, 2, 3)]):
        t = tiny(10 + seed, Bt, L, d, N)
        out, _ = oracle.scan_fwd(t["h"], t["a"], t["b"], t["B"], t["C"], t["z"], t["D"], t["x0"])
        f, i = sig(t["a"]), sig(t["b"])
        want = np.zeros((Bt, L, d))
        for bb in range(Bt):
            for n in range(L):
                for c in range(d):
                    acc = 0.0
                    for m in range(n + 1):
                        prod = 1.0
                        for k in range(m + 1, n + 1):
                            prod *= f[bb, k, c]
                        acc += prod * i[bb, m, c] * t["h"][bb, m, c] * float(
                            np.dot(t["B"][bb, m], t["C"][bb, n]))
                    prod0 = float(np.prod(f[bb, : n + 1, c]))
                    acc += prod0 * float(np.dot(t["x0"][bb, c], t["C"][bb, n]))
                    y = acc / math.sqrt(N) + t["D"][c] * t["h"][bb, n, c]
                    want[bb, n, c] = y * silu(t["z"][bb, n, c])
        np.testing.assert_allclose(out, want, rtol=1e-11, atol=1e-12)


def test_linear_in_h():
    t = tiny(4, x0=False)
    h2 = rnd(99, *t["h"].shape)
    al, be = 0.7, -1.3
    o1, _ = oracle.scan_fwd(t["h"], t["a"], t["b"], t["B"], t["C"], t["z"], t["D"])
    o2, _ = oracle.scan_fwd(h2, t["a"], t["b"], t["B"], t["C"], t["z"], t["D"])
    o3, _ = oracle.scan_fwd(al * t["h"] + be * h2, t["a"], t["b"], t["B"], t["C"], t["z"], t["D"])
    np.testing.assert_allclose(o3, al * o1 + be * o2, rtol=1e-10, atol=1e-12)


def test_bibo_bound():
    """Fading memory (abstract: 0 < f < 1 gives a BIBO bound):
    |x_n| <= |x0| + max|i h B| / (1 - max f), elementwise per (batch, channel)."""
    t = tiny(5, Bt=2, L=200, d=4, N=5)
    a = rnd(6, 2, 200, 4, mean=3.0, std=1.0)
    b, B, h = rnd(7, 2, 200, 4), rnd(8, 2, 200, 5), rnd(9, 2, 200, 4)
    for L in (1, 50, 200):
        _, xL = oracle.scan_fwd(h[:, :L], a[:, :L], b[:, :L], B[:, :L], B[:, :L], None, None,
                                t["x0"][:, :4])
        w = np.abs(sig(b[:, :L]) * h[:, :L])[..., None] * np.abs(B[:, :L, None, :])
        fmax = sig(a[:, :L]).max(axis=1)[..., None]
        bound = np.abs(t["x0"][:, :4]) + w.max(axis=1) / (1 - fmax)
        assert np.all(np.abs(xL) <= bound + 1e-12)


def test_affine_prefix_matches_loop():
    for seed, (Bt, L, d, N) in enumerate([(2, 33, 3, 4), (1, 64, 5, 8), (3, 17, 2, 16)]):
        t = tiny(20 + seed, Bt, L, d, N)
        o1, x1 = oracle.scan_fwd(t["h"], t["a"], t["b"], t["B"], t["C"], t["z"], t["D"], t["x0"])
        o2, x2 = scan_fwd_prefix(t["h"], t["a"], t["b"], t["B"], t["C"], t["z"], t["D"], t["x0"])
        np.testing.assert_allclose(o1, o2, rtol=1e-12, atol=1e-12)
        np.testing.assert_allclose(x1, x2, rtol=1e-12, atol=1e-12)


def test_decode_steps_equal_forward():
    """L single-token steps from x0 give the forward's outputs and final state."""
    t = tiny(30, Bt=3, L=24, d=5, N=8)
    out, xL = oracle.scan_fwd(t["h"], t["a"], t["b"], t["B"], t["C"], t["z"], t["D"], t["x0"])
    state = t["x0"]
    for n in range(24):
        o, state = oracle.scan_step(state, t["h"][:, n], t["a"][:, n], t["b"][:, n],
                                    t["B"][:, n], t["C"][:, n], t["z"][:, n], t["D"])
        np.testing.assert_allclose(o, out[:, n], rtol=1e-13, atol=1e-13)
    np.testing.assert_allclose(state, xL, rtol=1e-13, atol=1e-13)


# ------------------------------------------------------------------ the conv
def test_conv_matches_torch_conv1d():
    """Causal depthwise conv = torch conv1d with groups=d and W-1 left zeros."""
    r = np.random.default_rng(40)
    Bt, L, d, W = 2, 19, 5, 4
    u, w, bias = r.normal(size=(Bt, L, d)), r.normal(size=(d, W)), r.normal(size=(d,))
    h, p = oracle.conv_silu_fwd(u, w, bias, return_p=True)
    ut = torch.tensor(u).transpose(1, 2)                       # [Bt, d, L]
    pt = torch.nn.functional.conv1d(ut, torch.tensor(w)[:, None, :], torch.tensor(bias),
                                    padding=W - 1, groups=d)[..., :L].transpose(1, 2)
    np.testing.assert_allclose(p, pt.numpy(), rtol=1e-13, atol=1e-13)
    np.testing.assert_allclose(h, torch.nn.functional.silu(pt).numpy(), rtol=1e-13, atol=1e-13)


def test_conv_steps_match_torch_conv1d():
    """L decode steps of the conv from a zero conv state = torch conv1d over the
    sequence (the state holds the previous W-1 inputs, oldest first)."""
    r = np.random.default_rng(41)
    Bt, L, d, W = 2, 13, 5, 4
    u, w, bias = r.normal(size=(Bt, L, d)), r.normal(size=(d, W)), r.normal(size=(d,))
    ut = torch.tensor(u).transpose(1, 2)
    pt = torch.nn.functional.conv1d(ut, torch.tensor(w)[:, None, :], torch.tensor(bias),
                                    padding=W - 1, groups=d)[..., :L].transpose(1, 2)
    ref = torch.nn.functional.silu(pt).numpy()
    cs = np.zeros((Bt, d, W - 1))
    for t in range(L):
        h, cs = oracle.conv_silu_step(cs, u[:, t], w, bias)
        np.testing.assert_allclose(h, ref[:, t], rtol=1e-13, atol=1e-13)
    np.testing.assert_allclose(cs, u[:, L - (W - 1):].transpose(0, 2, 1), rtol=0, atol=0)


# ------------------------------------------------------ finite differences
def _loss_scan(t, dout, dxL):
    out, xL = oracle.scan_fwd(t["h"], t["a"], t["b"], t["B"], t["C"], t["z"], t["D"], t["x0"])
    return float(np.sum(out * dout) + np.sum(xL * dxL))


def _fd_check(loss, t, key, grad, eps=1e-6, rtol=1e-6):
    x = t[key]
    num = np.zeros_like(x)
    it = np.nditer(x, flags=["multi_index"])
    for _ in it:
        idx = it.multi_index
        old = x[idx]
        x[idx] = old + eps
        lp = loss(t)
        x[idx] = old - eps
        lm = loss(t)
        x[idx] = old
        num[idx] = (lp - lm) / (2 * eps)
    err = np.max(np.abs(num - grad)) / max(np.max(np.abs(num)), 1e-30)
    assert err < rtol, f"d{key}: rel err {err:.2e}"


def test_scan_gradients_finite_differences():
    t = tiny(50, Bt=2, L=6, d=3, N=4)
    r = np.random.default_rng(51)
    dout, dxL = r.normal(size=t["h"].shape), r.normal(size=t["x0"].shape)
    g = oracle.scan_bwd(t["h"], t["a"], t["b"], t["B"], t["C"], t["z"], t["D"], t["x0"], dout,
                        dxL)
    loss = lambda tt: _loss_scan(tt, dout, dxL)  # noqa: E731
    for key, gk in [("h", "dh"), ("a", "da"), ("b", "db"), ("B", "dB"), ("C", "dC"),
                    ("z", "dz"), ("D", "dD"), ("x0", "dx0")]:
        _fd_check(loss, t, key, g[gk])


def test_block_gradients_finite_differences():
    """Fused path: conv + SiLU feeding the scan; du, dconv_w, dconv_b."""
    r = np.random.default_rng(60)
    Bt, L, d, N, W = 2, 9, 3, 4, 4
    t = tiny(61, Bt, L, d, N)
    t["u"], t["w"], t["bias"] = r.normal(size=(Bt, L, d)), r.normal(0, .5, (d, W)), r.normal(
        size=(d,))
    dout, dxL = r.normal(size=(Bt, L, d)), r.normal(size=(Bt, d, N))

    def loss(tt):
        out, xL, _ = oracle.block_fwd(tt["u"], tt["w"], tt["bias"], tt["a"], tt["b"], tt["B"],
                                      tt["C"], tt["z"], tt["D"], tt["x0"])
        return float(np.sum(out * dout) + np.sum(xL * dxL))

    g = oracle.block_bwd(t["u"], t["w"], t["bias"], t["a"], t["b"], t["B"], t["C"], t["z"],
                         t["D"], t["x0"], dout, dxL)
    for key, gk in [("u", "du"), ("w", "dconv_w"), ("bias", "dconv_b"), ("a", "da"),
                    ("B", "dB"), ("C", "dC")]:
        _fd_check(loss, t, key, g[gk])


def test_gradients_without_optional_inputs():
    """No z, no D, no x0, no dxL: gradients still match finite differences."""
    t = tiny(70, Bt=1, L=5, d=2, N=3, x0=False)
    t["z"], t["D"] = None, None
    dout = np.random.default_rng(71).normal(size=t["h"].shape)

    def loss(tt):
        out, _ = oracle.scan_fwd(tt["h"], tt["a"], tt["b"], tt["B"], tt["C"])
        return float(np.sum(out * dout))

    g = oracle.scan_bwd(t["h"], t["a"], t["b"], t["B"], t["C"], None, None, None, dout)
    assert g["dz"] is None and g["dD"] is None
    for key, gk in [("h", "dh"), ("a", "da"), ("b", "db"), ("B", "dB"), ("C", "dC")]:
        _fd_check(loss, t, key, g[gk])


# ------------------------------------------- coupled single gate (i = 1 - f)
def test_coupled_gate_equals_write_gate_minus_a():
    """Coupled gate (b absent) = the two-gate scan with b = -a, since
    1 - sigma(a) = sigma(-a)."""
    t = tiny(80, Bt=2, L=7, d=3, N=4)
    o1, x1 = oracle.scan_fwd(t["h"], t["a"], None, t["B"], t["C"], t["z"], t["D"], t["x0"])
    o2, x2 = oracle.scan_fwd(t["h"], t["a"], -t["a"], t["B"], t["C"], t["z"], t["D"], t["x0"])
    np.testing.assert_allclose(o1, o2, rtol=1e-14, atol=1e-14)
    np.testing.assert_allclose(x1, x2, rtol=1e-14, atol=1e-14)


def test_coupled_gate_fixed_point_and_bound():
    """With i = 1 - f the update is a convex combination: a state equal to
    h B stays there for constant h and B, and |x_n| never exceeds
    max(|x0|, max |h B|) (the abstract's |r| + w <= 1 bound)."""
    r = np.random.default_rng(81)
    Bt, L, d, N = 1, 30, 3, 4
    hc, Bc = r.normal(size=(d,)), r.normal(size=(N,))
    h = np.broadcast_to(hc, (Bt, L, d)).copy()
    B = np.broadcast_to(Bc, (Bt, L, N)).copy()
    a = r.normal(0, 3, size=(Bt, L, d))
    C = r.normal(size=(Bt, L, N))
    x0 = np.einsum("d,n->dn", hc, Bc)[None]
    _, xL = oracle.scan_fwd(h, a, None, B, C, None, None, x0)
    np.testing.assert_allclose(xL, x0, rtol=1e-12, atol=1e-12)
    hr = r.normal(size=(Bt, L, d))
    Br = r.normal(size=(Bt, L, N))
    x0r = r.normal(size=(Bt, d, N))
    bound = np.maximum(np.abs(x0r), np.max(np.abs(np.einsum("btd,btn->btdn", hr, Br)),
                                           axis=1))
    for Lk in (1, 5, 30):
        _, xk = oracle.scan_fwd(hr[:, :Lk], a[:, :Lk], None, Br[:, :Lk], C[:, :Lk], None,
                                None, x0r)
        assert np.all(np.abs(xk) <= bound + 1e-12)


def test_coupled_gate_gradients_finite_differences():
    """Coupled gate: a enters through f and i = 1 - f; no b."""
    t = tiny(82, Bt=2, L=6, d=3, N=4)
    r = np.random.default_rng(83)
    dout, dxL = r.normal(size=t["h"].shape), r.normal(size=t["x0"].shape)
    g = oracle.scan_bwd(t["h"], t["a"], None, t["B"], t["C"], t["z"], t["D"], t["x0"], dout, dxL)

    def loss(tt):
        out, xL = oracle.scan_fwd(tt["h"], tt["a"], None, tt["B"], tt["C"], tt["z"], tt["D"],
                                  tt["x0"])
        return float(np.sum(out * dout) + np.sum(xL * dxL))

    for key, gk in [("h", "dh"), ("a", "da"), ("B", "dB"), ("C", "dC"), ("z", "dz"),
                    ("D", "dD"), ("x0", "dx0")]:
        _fd_check(loss, t, key, g[gk])


# ------------------------------------------------------ the full block
@pytest.mark.parametrize("coupled", [False, True])
def test_block_oracle_finite_differences(coupled):
    """Full block (norm, projections, conv, scan, modulation, residual): every
    gradient against central finite differences."""
    from oracle import block as ob
    r = np.random.default_rng(90)
    Bt, L, dm, di, N = 1, 5, 4, 3, 4
    p = {k: v.astype(np.float64) for k, v in ob.init_params(dm, di, N, seed=91).items()}
    x = r.normal(size=(Bt, L, dm))
    dout = r.normal(size=(Bt, L, dm))
    out, cache = ob.block_fwd(x, p, coupled)
    dx, g = ob.block_bwd(cache, dout, coupled)
    t = dict(p, x=x)

    def loss(tt):
        pp = {k: tt[k] for k in ob.PARAMS}
        o, _ = ob.block_fwd(tt["x"], pp, coupled)
        return float(np.sum(o * dout))

    _fd_check(loss, t, "x", dx, rtol=1e-5)
    for k in ob.PARAMS:
        if coupled and k in ("W_b", "b_b"):
            continue
        _fd_check(loss, t, k, g[k], rtol=1e-5)


@pytest.mark.parametrize("coupled", [False, True])
def test_block_oracle_forward_independent_composition(coupled):
    """The block oracle's forward (README block flowchart: normalized token ->
    input projection -> conv + SiLU -> projections of h -> scan -> SiLU(z)
    modulation -> output projection -> residual) equals a composition of
    library routines written independently of it, in fp64: torch rms_norm,
    linear maps, a depthwise conv1d with left zero padding, torch silu, and
    the affine-prefix evaluation of the scan (coupled gate: b = -a, since
    sigma(-a) = 1 - sigma(a)).  Pins the norm (RMS with eps 1e-6 and a
    learned scale), the order of the u / z split, the bias placement and the
    residual."""
    import torch.nn.functional as F
    from oracle import block as ob
    r = np.random.default_rng(95)
    Bt, L, dm, di, N = 2, 9, 6, 5, 4
    p = {k: v.astype(np.float64) for k, v in ob.init_params(dm, di, N, seed=96).items()}
    x = r.normal(size=(Bt, L, dm))
    out, _ = ob.block_fwd(x, p, coupled)

    T = {k: torch.from_numpy(v) for k, v in p.items()}
    xt = torch.from_numpy(x)
    xn = F.rms_norm(xt, (dm,), weight=T["norm_w"], eps=1e-6)
    uz = F.linear(xn, T["W_in"].T)
    u, z = uz[..., :di], uz[..., di:]
    pre = F.conv1d(u.transpose(1, 2), T["conv_w"][:, None, :], bias=T["conv_b"],
                   padding=3, groups=di)[..., :L].transpose(1, 2)
    h = F.silu(pre)
    a = F.linear(h, T["W_a"].T, T["b_a"])
    b = -a if coupled else F.linear(h, T["W_b"].T, T["b_b"])
    B = F.linear(h, T["W_B"].T)
    C = F.linear(h, T["W_C"].T)
    y, _ = scan_fwd_prefix(h.numpy(), a.numpy(), b.numpy(), B.numpy(), C.numpy(),
                           z.numpy(), p["D"])
    ref = xt + F.linear(torch.from_numpy(y), T["W_out"].T)
    np.testing.assert_allclose(out, ref.numpy(), rtol=1e-12, atol=1e-12)
