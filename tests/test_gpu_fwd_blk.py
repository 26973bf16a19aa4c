"""The block-form tensor-core forward (64-token blocks, bf16 activations,
d_state 64 and 128) against the fp64 oracle, forced through the testing hook:
optional inputs, the coupled gate, both output dtypes, sequence groups,
piece mode with cuts inside units, the exact path, ragged sizes; and its
checkpoints driving the backward."""
import pytest
import torch

import discrete_selective_ssm_b200 as naju
from naju_check import TOL_BF16, assert_close
from test_gpu_parity import (compare_grads, inputs, oracle_bwd, oracle_fwd, run_bwd, run_fwd,
                             wl)

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def block_forward():
    naju.testing_set_fwd_impl(3)
    yield
    naju.testing_set_fwd_impl(0)
    naju.testing_set_bwd_impl(0)
    naju.testing_set_fwd_groups(0)
    naju.testing_set_fwd_pieces(0)


def _check(t, conv, out_dtype=naju.F32, groups=0):
    y, xf, _ = run_fwd(t, conv, out_dtype=out_dtype, groups=groups)
    ro, rx = oracle_fwd(t, conv)
    assert_close(y, ro, TOL_BF16, bf16_out=out_dtype == naju.BF16, name="y")
    assert_close(xf, rx, TOL_BF16, name="x_final")


@pytest.mark.parametrize("N", [64, 128])
@pytest.mark.parametrize("conv", [True, False])
def test_fblk_basic(N, conv):
    w = wl(N, "bf16", Bt=2, L=333, d=264)
    assert naju.testing_fwd_impl(naju.make_dims(2, 333, 264, N, naju.BF16)) == 3
    _check(inputs(w, conv, use_x0=True), conv)


@pytest.mark.parametrize("N", [64, 128])
def test_fblk_bf16_outputs(N):
    w = wl(N, "bf16", Bt=3, L=257, d=136)
    _check(inputs(w, True), True, out_dtype=naju.BF16)


def test_fblk_no_optional_inputs():
    w = wl(64, "bf16", Bt=1, L=150, d=128)
    _check(inputs(w, False, use_z=False, use_D=False), False)


@pytest.mark.parametrize("N", [64, 128])
def test_fblk_coupled_gate(N):
    w = wl(N, "bf16", Bt=2, L=260, d=136)
    t = inputs(w, True, use_x0=True)
    t["b"] = None
    _check(t, True)


@pytest.mark.parametrize("L", [1, 5, 63, 64, 65, 130])
def test_fblk_lengths(L):
    w = wl(64, "bf16", Bt=2, L=L, d=136)
    _check(inputs(w, True, use_x0=True), True)


@pytest.mark.parametrize("N", [64, 128])
@pytest.mark.parametrize("groups", [2, 3, 7])
def test_fblk_sequence_groups(N, groups):
    w = wl(N, "bf16", Bt=2, L=1000, d=136)
    _check(inputs(w, True, use_x0=True), True, groups=groups)


@pytest.mark.parametrize("N", [64, 128])
@pytest.mark.parametrize("conv", [True, False])
@pytest.mark.parametrize("pieces", [2, 4, 7])
def test_fblk_pieces(pieces, conv, N):
    w = wl(N, "bf16", Bt=3, L=333, d=264)
    t = inputs(w, conv, use_x0=True)
    naju.testing_set_fwd_pieces(pieces)
    assert naju.testing_fwd_pieces(naju.make_dims(3, 333, 264, N, naju.BF16)) == pieces
    _check(t, conv)


@pytest.mark.parametrize("N", [64, 128])
def test_fblk_exact_path(N):
    w = wl(N, "bf16", Bt=1, L=300, d=136)
    t = inputs(w, True, use_x0=True)
    a = t["a"].float().clone()
    a[:, 40:60] = -60.0
    a[:, 100:200:2] = -25.0
    a[:, 220:240] = 60.0
    a[:, 250, 7] = -200.0
    t["a"] = a.to(torch.bfloat16)
    _check(t, True)


def test_fblk_exact_path_in_update_pass():
    w = wl(64, "bf16", Bt=2, L=1000, d=136)
    t = inputs(w, True, use_x0=True)
    a = t["a"].float().clone()
    a[:, 100:130] = -60.0
    t["a"] = a.to(torch.bfloat16)
    _check(t, True, groups=3)


@pytest.mark.parametrize("N", [64, 128])
def test_fblk_overwrite_events(N):
    w = wl(N, "bf16", Bt=2, L=700, d=136, base="long_retention")
    _check(inputs(w, True, use_x0=True), True)


@pytest.mark.parametrize("bwd_impl", [0, 1, 3])
def test_fblk_checkpoints_drive_the_backward(bwd_impl):
    """The backward (automatic choice, CUDA cores, block form) from this
    forward's checkpoints."""
    w = wl(64, "bf16", Bt=2, L=333, d=264)
    t = inputs(w, True, use_x0=True, use_dxL=True)
    naju.testing_set_bwd_impl(bwd_impl)
    g = run_bwd(t, True, out_dtype=naju.F32)
    compare_grads(g, oracle_bwd(t, True), True, TOL_BF16)
