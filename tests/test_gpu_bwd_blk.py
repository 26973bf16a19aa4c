"""The block-form tensor-core backward (64-token blocks, bf16 activations,
d_state 64, and 128 as two passes over state halves) against the fp64
oracle, forced through the testing hook so it runs whatever the automatic
choice is: every optional input, the coupled gate, both output dtypes,
sequence groups, piece mode with cuts inside units, the exact path for
blocks outside the factorisation's range, and ragged lengths and widths."""
import pytest
import torch

import discrete_selective_ssm_b200 as naju
from naju_check import TOL_BF16
from test_gpu_parity import compare_grads, gpu, inputs, oracle_bwd, run_bwd, run_fwd, wl

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def block_backward():
    naju.testing_set_bwd_impl(3)
    yield
    naju.testing_set_bwd_impl(0)
    naju.testing_set_bwd_groups(0)
    naju.testing_set_bwd_pieces(0)


def _check(t, conv, out_dtype=naju.F32, **kw):
    g = run_bwd(t, conv, out_dtype=out_dtype)
    compare_grads(g, oracle_bwd(t, conv), conv, TOL_BF16, bf16_out=out_dtype == naju.BF16, **kw)


@pytest.mark.parametrize("N", [64, 128])
@pytest.mark.parametrize("conv", [True, False])
def test_blk_basic(conv, N):
    w = wl(N, "bf16", Bt=2, L=333, d=264)
    t = inputs(w, conv, use_x0=True, use_dxL=True)
    assert naju.testing_bwd_impl(naju.make_dims(2, 333, 264, N, naju.BF16)) == 3
    _check(t, conv)


@pytest.mark.parametrize("N", [64, 128])
def test_blk_bf16_outputs(N):
    w = wl(N, "bf16", Bt=2, L=200, d=136)
    _check(inputs(w, True), True, out_dtype=naju.BF16)


@pytest.mark.parametrize("N", [64, 128])
def test_blk_no_optional_inputs(N):
    w = wl(N, "bf16", Bt=1, L=150, d=128)
    t = inputs(w, False, use_z=False, use_D=False)
    _check(t, False, has_z=False, has_D=False)


@pytest.mark.parametrize("N", [64, 128])
@pytest.mark.parametrize("conv", [True, False])
def test_blk_coupled_gate(conv, N):
    w = wl(N, "bf16", Bt=2, L=260, d=136)
    t = inputs(w, conv, use_x0=True, use_dxL=True)
    t["b"] = None
    g = run_bwd(t, conv, out_dtype=naju.F32)
    r = oracle_bwd(t, conv)
    from naju_check import assert_close
    assert_close(g["dhu"], r["du"] if conv else r["dh"], TOL_BF16, name="du")
    for k in ("da", "dB", "dC", "dz", "dx0"):
        assert_close(g[k], r[k], TOL_BF16, name=k)


@pytest.mark.parametrize("N", [64, 128])
@pytest.mark.parametrize("L", [1, 5, 63, 64, 65, 130])
def test_blk_lengths(L, N):
    w = wl(N, "bf16", Bt=2, L=L, d=136)
    _check(inputs(w, True, use_x0=True, use_dxL=True), True)


@pytest.mark.parametrize("N", [64, 128])
@pytest.mark.parametrize("groups", [2, 3, 5])
def test_blk_sequence_groups(groups, N):
    w = wl(N, "bf16", Bt=2, L=600, d=136)
    t = inputs(w, True, use_x0=True, use_dxL=True)
    naju.testing_set_bwd_groups(groups)
    _check(t, True)


@pytest.mark.parametrize("N", [64, 128])
@pytest.mark.parametrize("conv", [True, False])
@pytest.mark.parametrize("pieces", [2, 4, 7])
def test_blk_pieces(pieces, conv, N):
    w = wl(N, "bf16", Bt=3, L=333, d=264)
    t = inputs(w, conv, use_x0=True, use_dxL=True)
    naju.testing_set_bwd_pieces(pieces)
    assert naju.testing_bwd_pieces(naju.make_dims(3, 333, 264, N, naju.BF16)) == pieces
    _check(t, conv)


@pytest.mark.parametrize("N", [64, 128])
def test_blk_exact_path(N):
    """Runs of vanishing forget gates push blocks outside the factorisation's
    range (decay below 2^-90 over 64 tokens): those blocks take the exact
    token-by-token path; f = 0 exactly and f = 1 exactly included."""
    w = wl(N, "bf16", Bt=1, L=300, d=136)
    t = inputs(w, True, use_x0=True, use_dxL=True)
    a = t["a"].float().clone()
    a[:, 40:60] = -60.0
    a[:, 100:200:2] = -25.0
    a[:, 220:240] = 60.0
    a[:, 250, 7] = -200.0
    t["a"] = a.to(torch.bfloat16)
    _check(t, True)


@pytest.mark.parametrize("N", [64, 128])
def test_blk_exact_path_in_groups(N):
    """The exact path inside the early (adjoint-only) pass of sequence groups."""
    w = wl(N, "bf16", Bt=2, L=600, d=136)
    t = inputs(w, True, use_x0=True, use_dxL=True)
    a = t["a"].float().clone()
    a[:, 330:350] = -60.0
    t["a"] = a.to(torch.bfloat16)
    naju.testing_set_bwd_groups(3)
    _check(t, True)


def test_blk_moderate_decay_runs():
    """Quarter products above 2^22 (the conservative test fires) while no
    block product exceeds 2^90: the factorised path stays exact enough."""
    w = wl(64, "bf16", Bt=2, L=300, d=136)
    t = inputs(w, True, use_x0=True, use_dxL=True)
    a = t["a"].float().clone()
    a[:, 36:46] = -3.0
    a[0, 130:136] = -2.9
    t["a"] = a.to(torch.bfloat16)
    _check(t, True)


@pytest.mark.parametrize("N", [64, 128])
def test_blk_overwrite_events(N):
    """The long-horizon distribution (5 % overwrite events)."""
    w = wl(N, "bf16", Bt=2, L=700, d=136, base="long_retention")
    _check(inputs(w, True, use_x0=True, use_dxL=True), True)


@pytest.mark.parametrize("N", [64, 128])
def test_blk_pieces_timeout_is_reported(N):
    w = wl(N, "bf16", Bt=2, L=320, d=256)
    t = inputs(w, True)
    naju.testing_set_bwd_pieces(3)
    y, xf, ws = run_fwd(t, True)
    naju.testing_set_wait_limit(2000)
    naju.testing_set_skip_publish(True)
    try:
        naju.scan_bwd(gpu(t["dout"]), gpu(t["u"]), gpu(t["a"]), gpu(t["b"]), gpu(t["B"]),
                      gpu(t["C"]), ws, conv_w=gpu(t["conv_w"]), conv_b=gpu(t["conv_b"]),
                      z=gpu(t["z"]), D=gpu(t["D"]))
        assert naju.last_device_status(ws) == 4
    finally:
        naju.testing_set_skip_publish(False)
        naju.testing_set_wait_limit(0)
    _check(t, True)
