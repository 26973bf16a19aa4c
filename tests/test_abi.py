"""Host-side checks of the C ABI: the library loads, exports every declared
symbol, sizes workspaces, and rejects bad arguments before touching a GPU."""
import ctypes

import pytest

import discrete_selective_ssm_b200 as naju
from discrete_selective_ssm_b200 import _native


@pytest.fixture(scope="module")
def L():
    return naju.lib()


@pytest.fixture
def b200_sms(L):
    """Tiling rules below are stated for a B200's 148 SMs."""
    naju.testing_set_sm_count(148)
    yield
    naju.testing_set_sm_count(0)


def test_exports_every_declared_symbol(L):
    names = naju.declared_symbols()
    assert "naju_scan_fwd" in names and "naju_scan_bwd" in names and "naju_scan_step" in names
    for n in names:
        assert hasattr(L, n), f"{n} declared in include/ but not exported"


def test_workspace_bytes(L):
    d = naju.make_dims(2, 300, 200, 64, naju.BF16)
    n = naju.workspace_bytes(d)
    # at least the checkpoints: Bt * (ceil(L/128)+1) * d * N fp32
    assert n >= 2 * 4 * 200 * 64 * 4
    assert n % 256 == 0
    bad = naju.make_dims(2, 300, 200, 48, naju.BF16)
    assert naju.workspace_bytes(bad) == 0
    assert L.naju_scan_workspace_bytes(None) == 0


def test_rejects_bad_arguments_on_host(L):
    d = naju.make_dims(1, 8, 8, 16, naju.F32)
    null = None
    # null dims / null required pointers -> INVALID_ARG (1), never reaches CUDA
    assert L.naju_scan_fwd(None, *([null] * 13), 0, null) == 1
    assert L.naju_scan_fwd(ctypes.byref(d), *([null] * 13), 0, null) == 1
    assert L.naju_scan_bwd(ctypes.byref(d), *([null] * 23), 0, null) == 1
    # unsupported d_state -> UNSUPPORTED (2)
    d2 = naju.make_dims(1, 8, 8, 24, naju.F32)
    assert L.naju_scan_fwd(ctypes.byref(d2), *([null] * 13), 0, null) == 2
    # f32 inputs with bf16 outputs -> UNSUPPORTED
    d3 = naju.make_dims(1, 8, 8, 16, naju.F32, naju.BF16)
    assert L.naju_scan_fwd(ctypes.byref(d3), *([null] * 13), 0, null) == 2
    # conv width other than 4 in fused mode -> UNSUPPORTED
    d4 = naju.make_dims(1, 8, 8, 16, naju.F32, conv_width=3)
    fake = ctypes.c_void_p(256)
    assert L.naju_scan_fwd(ctypes.byref(d4), fake, fake, *([null] * 11), 0, null) == 2
    # misaligned activation pointer -> INVALID_ARG
    mis = ctypes.c_void_p(258)
    assert L.naju_scan_fwd(ctypes.byref(d), mis, null, null, fake, fake, fake, fake, null, null,
                           null, fake, null, fake, 1 << 30, null) == 1
    # workspace too small -> INVALID_ARG
    assert L.naju_scan_fwd(ctypes.byref(d), fake, null, null, fake, fake, fake, fake, null, null,
                           null, fake, null, fake, 16, null) == 1
    # step: bad d_state / null pointers
    assert L.naju_scan_step(1, 8, 24, 0, *([null] * 10)) == 2
    assert L.naju_scan_step(1, 8, 16, 0, *([null] * 10)) == 1
    assert L.naju_last_device_status(None, None) == 1
    # conv decode steps: null pointers / bad d_state
    assert L.naju_conv_silu_step(1, 8, 0, *([null] * 6)) == 1
    assert L.naju_conv_silu_step(1, 8, 7, *([null] * 6)) == 2
    assert L.naju_scan_step_conv(1, 8, 24, 0, *([null] * 13)) == 2
    assert L.naju_scan_step_conv(1, 8, 16, 0, *([null] * 13)) == 1


def test_status_strings(L):
    for code in range(5):
        assert L.naju_status_string(code)


def test_fwd_group_policy(L, b200_sms):
    # Few (batch x tile) items split the sequence; many do not.
    few = naju.make_dims(2, 8192, 2048, 128, naju.BF16)
    many = naju.make_dims(64, 4096, 2048, 64, naju.BF16)
    assert naju.testing_fwd_groups(few) > 1
    assert naju.testing_fwd_groups(many) == 1
    naju.testing_set_fwd_groups(3)
    try:
        assert naju.testing_fwd_groups(many) == 3
    finally:
        naju.testing_set_fwd_groups(0)


def test_binding_refuses_cpu_tensors():
    import torch
    with pytest.raises(ValueError):
        _native._ptr(torch.zeros(4), "x")


def test_empty_and_oversized_dims_are_rejected(L):
    """Empty inputs (batch, length or width 0) and sizes past the documented
    limits are rejected on the host before any launch."""
    null = None
    for dims in (naju.make_dims(0, 8, 8, 16, naju.F32), naju.make_dims(1, 0, 8, 16, naju.F32),
                 naju.make_dims(1, 8, 0, 16, naju.F32),
                 naju.make_dims(1 << 21, 8, 8, 16, naju.F32),
                 naju.make_dims(1, 1 << 27, 8, 16, naju.F32),
                 naju.make_dims(1 << 20, 1 << 12, 1 << 10, 16, naju.F32)):
        assert naju.workspace_bytes(dims) == 0
        assert L.naju_scan_fwd(ctypes.byref(dims), *([null] * 13), 0, null) == 1
        assert L.naju_scan_bwd(ctypes.byref(dims), *([null] * 23), 0, null) == 1
    assert L.naju_scan_step(0, 8, 16, 0, *([null] * 10)) == 1
    assert L.naju_scan_step_conv(0, 8, 16, 0, *([null] * 13)) == 1
    assert L.naju_conv_silu_step(0, 8, 0, *([null] * 6)) == 1


def test_tensor_core_dispatch_rules(L):
    """Tensor-core kernels for bf16 with d_state 64/128 and d_inner % 8 == 0
    (block form, forward and backward); CUDA-core kernels otherwise (fp32,
    d_state 16/32, other widths).  Forcing impl 2 selects the sub-chunk
    kernels."""
    assert naju.testing_fwd_impl(naju.make_dims(2, 64, 256, 64, naju.BF16)) == 3
    assert naju.testing_fwd_impl(naju.make_dims(2, 64, 256, 128, naju.BF16)) == 3
    assert naju.testing_bwd_impl(naju.make_dims(2, 64, 256, 64, naju.BF16)) == 3
    assert naju.testing_bwd_impl(naju.make_dims(2, 64, 256, 128, naju.BF16)) == 3
    assert naju.testing_fwd_impl(naju.make_dims(2, 64, 264, 64, naju.BF16)) == 3
    naju.testing_set_fwd_impl(2)
    naju.testing_set_bwd_impl(2)
    try:
        assert naju.testing_fwd_impl(naju.make_dims(2, 64, 256, 64, naju.BF16)) == 2
        assert naju.testing_bwd_impl(naju.make_dims(2, 64, 256, 64, naju.BF16)) == 2
    finally:
        naju.testing_set_fwd_impl(0)
        naju.testing_set_bwd_impl(0)
    assert naju.testing_fwd_impl(naju.make_dims(2, 64, 258, 64, naju.BF16)) == 1
    assert naju.testing_bwd_impl(naju.make_dims(2, 64, 258, 64, naju.BF16)) == 1
    assert naju.testing_fwd_impl(naju.make_dims(2, 64, 256, 32, naju.BF16)) == 1
    assert naju.testing_bwd_impl(naju.make_dims(2, 64, 256, 64, naju.F32)) == 1


def test_backward_piece_mode_rules(L, b200_sms):
    """The tensor-core backward cuts the units' blocks into one range per SM
    (148) when there are at least that many 128-channel units but not a whole
    number of waves; otherwise it keeps sequence groups."""
    dm = naju.make_dims(16, 4096, 2048, 64, naju.BF16)  # 256 units
    assert naju.testing_bwd_pieces(dm) == 148
    assert naju.testing_bwd_groups(dm) == 2  # the two carry slots
    assert naju.testing_bwd_pieces(naju.make_dims(8, 2048, 1536, 64, naju.BF16)) == 0  # 96
    assert naju.testing_bwd_pieces(naju.make_dims(37, 512, 1024, 64, naju.BF16)) == 0  # 296
    assert naju.testing_bwd_pieces(naju.make_dims(16, 4096, 2048, 64, naju.F32)) == 0
    assert naju.testing_bwd_pieces(naju.make_dims(160, 64, 128, 64, naju.BF16)) == 0  # 1 block
    naju.testing_set_bwd_pieces(-1)
    try:
        assert naju.testing_bwd_pieces(dm) == 0
    finally:
        naju.testing_set_bwd_pieces(0)
    naju.testing_set_bwd_pieces(5)
    try:
        assert naju.testing_bwd_pieces(naju.make_dims(1, 512, 512, 64, naju.BF16)) == 0  # 4 units
        assert naju.testing_bwd_pieces(naju.make_dims(2, 512, 512, 64, naju.BF16)) == 5
    finally:
        naju.testing_set_bwd_pieces(0)


def test_forward_piece_mode_rules(L, b200_sms):
    """The tensor-core forward takes piece mode under the backward's rule."""
    dm = naju.make_dims(16, 4096, 2048, 64, naju.BF16)
    assert naju.testing_fwd_pieces(dm) == 148
    assert naju.testing_fwd_groups(dm) == 1
    assert naju.testing_fwd_pieces(naju.make_dims(8, 2048, 1536, 64, naju.BF16)) == 0
    assert naju.testing_fwd_pieces(naju.make_dims(16, 4096, 2048, 64, naju.F32)) == 0
    naju.testing_set_fwd_pieces(-1)
    try:
        assert naju.testing_fwd_pieces(dm) == 0
    finally:
        naju.testing_set_fwd_pieces(0)


def test_tensor_core_group_counts_follow_the_wave_model(L, b200_sms):
    """Fewer 128-channel units than SMs: the sequence-group count with the
    least modelled time (mid_lm: 96 units -> 3 backward groups, 288 blocks,
    two full waves, but 1 forward group, whose update-only pass would cost
    more than the idle SMs; long_retention: 32 units -> 9 groups, 288
    blocks)."""
    mid = naju.make_dims(8, 2048, 1536, 64, naju.BF16)
    lr = naju.make_dims(2, 8192, 2048, 128, naju.BF16)
    assert naju.testing_fwd_groups(mid) == 1 and naju.testing_bwd_groups(mid) == 3
    assert naju.testing_fwd_groups(lr) == 9 and naju.testing_bwd_groups(lr) == 9
    one = naju.make_dims(148, 1024, 128, 64, naju.BF16)  # exactly one wave
    assert naju.testing_fwd_groups(one) == 1 and naju.testing_bwd_groups(one) == 1
    assert naju.testing_bwd_pieces(one) == 0
    big = naju.make_dims(16, 4096, 2048, 64, naju.BF16)  # 256 units, piece mode off
    naju.testing_set_fwd_pieces(-1)
    naju.testing_set_bwd_pieces(-1)
    try:
        assert naju.testing_fwd_groups(big) == 1 and naju.testing_bwd_groups(big) == 1
    finally:
        naju.testing_set_fwd_pieces(0)
        naju.testing_set_bwd_pieces(0)


def test_tiling_follows_the_sm_count(L):
    """Piece mode and the wave model use the SM count of the device (queried
    once per device; forced here): 256 units of the bench workload are cut
    into one range per SM unless they fill whole waves."""
    dm = naju.make_dims(16, 4096, 2048, 64, naju.BF16)  # 256 units of 128 channels
    mid = naju.make_dims(8, 2048, 1536, 64, naju.BF16)  # 96 units
    try:
        naju.testing_set_sm_count(132)
        assert naju.testing_sm_count() == 132
        assert naju.testing_fwd_pieces(dm) == 132 and naju.testing_bwd_pieces(dm) == 132
        naju.testing_set_sm_count(128)  # two whole waves: no cut
        assert naju.testing_fwd_pieces(dm) == 0 and naju.testing_bwd_pieces(dm) == 0
        assert naju.testing_fwd_groups(dm) == 1
        naju.testing_set_sm_count(96)   # mid_lm fills exactly one wave
        assert naju.testing_fwd_groups(mid) == 1 and naju.testing_bwd_groups(mid) == 1
        naju.testing_set_sm_count(1000)  # 96 units on 1000 SMs: more sequence groups
        assert naju.testing_fwd_groups(mid) > 3 and naju.testing_bwd_groups(mid) > 3
        # the workspace is sized for the tiling in force
        assert naju.workspace_bytes(mid) > 0
    finally:
        naju.testing_set_sm_count(0)
    assert naju.testing_sm_count() > 0
