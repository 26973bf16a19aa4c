"""Tensor-core building blocks: tf32 MMAs with A in tensor memory or shared
memory and shared operands in the no-swizzle or 128-byte swizzled K-major
layouts, against a host product."""
import ctypes

import numpy as np
import pytest
import torch

import discrete_selective_ssm_b200 as naju

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("N,K", [(16, 16), (16, 80), (64, 16), (128, 16), (16, 144), (32, 96),
                                 (128, 128)])
def test_tc_mma_tf32(N, K):
    L = naju.lib()
    f = L.naju_testing_tc_mma
    f.argtypes = [ctypes.c_int32, ctypes.c_int32] + [ctypes.c_void_p] * 5
    f.restype = ctypes.c_int
    g = torch.Generator().manual_seed(N * 1000 + K)
    A = torch.randn(128, K, generator=g)
    B = torch.randn(N, K, generator=g)
    dA, dB = A.cuda(), B.cuda()
    dD = torch.full((128, N), float("nan"), device="cuda")
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    rc = f(N, K, ctypes.c_void_p(dA.data_ptr()), ctypes.c_void_p(dB.data_ptr()),
           ctypes.c_void_p(dD.data_ptr()), ctypes.c_void_p(st.data_ptr()),
           ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert rc == 0
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    ref = A.double().numpy() @ B.double().numpy().T
    got = dD.cpu().double().numpy()
    # tf32 operands: ~2^-11 relative per element, sums of K terms
    err = np.max(np.abs(got - ref)) / np.max(np.abs(ref))
    assert err < 4e-3, err


@pytest.mark.parametrize("N,K,rows_a,swz_a,swz_b", [
    (16, 128, 128, 1, 1), (16, 128, 64, 1, 1), (64, 128, 128, 1, 1), (128, 128, 128, 1, 0),
    (16, 16, 64, 0, 0), (16, 16, 128, 0, 0), (32, 64, 64, 1, 1), (16, 32, 128, 0, 1)])
def test_tc_mma_tf32_shared_operands(N, K, rows_a, swz_a, swz_b):
    L = naju.lib()
    f = L.naju_testing_tc_mma_ss
    f.argtypes = [ctypes.c_int32] * 5 + [ctypes.c_void_p] * 5
    f.restype = ctypes.c_int
    g = torch.Generator().manual_seed(N * 1000 + K * 10 + rows_a + swz_a * 2 + swz_b)
    A = torch.randn(rows_a, K, generator=g)
    B = torch.randn(N, K, generator=g)
    dA, dB = A.cuda(), B.cuda()
    dD = torch.full((128, N), float("nan"), device="cuda")
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    rc = f(N, K, rows_a, swz_a, swz_b, ctypes.c_void_p(dA.data_ptr()),
           ctypes.c_void_p(dB.data_ptr()), ctypes.c_void_p(dD.data_ptr()),
           ctypes.c_void_p(st.data_ptr()), ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert rc == 0
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    ref = A.double().numpy() @ B.double().numpy().T
    got = dD.cpu().double().numpy()[:rows_a]
    err = np.max(np.abs(got - ref)) / np.max(np.abs(ref))
    assert err < 4e-3, err


def _tmem_rows(M, d_lane):
    """TMEM lane of each result row: M = 128 fills lanes 0-127 in order; M = 64
    fills 16 lanes of each 32-lane sub-partition (rows 16 s + i -> lane
    32 s + i + d_lane)."""
    if M == 128:
        return list(range(128))
    return [32 * (r // 16) + (r % 16) + d_lane for r in range(64)]


@pytest.mark.parametrize("M,N,K,a_mn,b_mn,d_lane,kind", [
    # tf32: K-major 128-byte swizzle, MN-major 32-byte swizzle atoms
    (128, 64, 64, 0, 0, 0, 0), (128, 64, 64, 1, 0, 0, 0), (128, 64, 64, 0, 1, 0, 0),
    (128, 64, 128, 1, 1, 0, 0), (128, 128, 64, 0, 1, 0, 0), (128, 32, 96, 1, 0, 0, 0),
    (64, 64, 64, 0, 0, 0, 0), (64, 64, 64, 1, 1, 0, 0), (64, 64, 128, 1, 0, 16, 0),
    (64, 64, 64, 0, 1, 16, 0), (64, 32, 32, 1, 1, 16, 0), (64, 128, 64, 1, 1, 0, 0),
    # bf16 hi/lo split (kind::f16), the block-form backward's products
    (128, 64, 64, 0, 0, 0, 1), (128, 64, 64, 0, 1, 0, 1), (64, 64, 128, 1, 1, 0, 1),
    (64, 64, 128, 1, 1, 16, 1), (64, 64, 64, 1, 0, 0, 1), (64, 64, 64, 1, 1, 16, 1)])
def test_tc_mma_mn_major_m64_and_split(M, N, K, a_mn, b_mn, d_lane, kind):
    """MN-major (transposed) shared operands, M = 64 accumulators and their
    placement at lane offset 16, tf32 and bf16 hi/lo split products, against a
    host product."""
    L = naju.lib()
    f = L.naju_testing_tc_mma_gen
    f.argtypes = [ctypes.c_int32] * 7 + [ctypes.c_void_p] * 5
    f.restype = ctypes.c_int
    g = torch.Generator().manual_seed(M * 7 + N * 1000 + K * 10 + a_mn * 2 + b_mn + d_lane + kind)
    A = torch.randn(M, K, generator=g)
    B = torch.randn(N, K, generator=g)
    dA, dB = A.cuda(), B.cuda()
    dD = torch.full((128, N), float("nan"), device="cuda")
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    rc = f(M, N, K, a_mn, b_mn, d_lane, kind, ctypes.c_void_p(dA.data_ptr()),
           ctypes.c_void_p(dB.data_ptr()), ctypes.c_void_p(dD.data_ptr()),
           ctypes.c_void_p(st.data_ptr()), ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert rc == 0
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    ref = A.double().numpy() @ B.double().numpy().T
    raw = dD.cpu().double().numpy()
    lanes = _tmem_rows(M, d_lane)
    got = raw[lanes]
    err = np.max(np.abs(got - ref)) / np.max(np.abs(ref))
    # tf32 operands: ~2^-11 per element; bf16 hi/lo split: ~2^-16
    assert err < (4e-3 if kind == 0 else 5e-5), err
    others = sorted(set(range(128)) - set(lanes))
    if others:  # lanes outside the result keep the zeros written before the MMA
        assert np.all(raw[others] == 0.0)


def test_fast_math_against_fp64_and_cuda_expf():
    """The block-form kernels compute e^x as 2^(x log2 e) on the MUFU base-2
    unit (PTX ex2.approx.ftz) and sigma(x) = 1 / (1 + e^{-x}) with the
    approximate reciprocal; the forward shares one reciprocal among three
    sigmoids with each e^{-v} capped at 2^36.  Bounds, derived: rounding
    x log2 e costs |x| log2(e) 2^-24 in the exponent, i.e. a relative error
    of at most 88 * 1.4427 * 2^-24 * ln 2 < 5.3e-6 in e^x for |x| <= 88, plus
    the base-2 unit's few ulp; results below the normal range (x < -87.33)
    may flush to zero.  sigma(x) then errs by < 2e-6 absolute; the capped
    form also moves sigma(x) for x < -24.95 to 1 / (1 + 2^36) < 1.46e-11.
    The output gate's SiLU(x) = h + h tanh(h), h = x / 2, on the MUFU tanh
    (PTX tanh.approx.f32, relative error below 2^-10.98): an error of at most
    |h| |tanh(h)| 2^-10.98 < 2.5e-4 |x| plus the fp32 rounding of h + h t."""
    L = naju.lib()
    f = L.naju_testing_fast_math
    f.argtypes = [ctypes.c_void_p] * 5 + [ctypes.c_int64, ctypes.c_void_p]
    f.restype = ctypes.c_int
    g = torch.Generator().manual_seed(7)
    x = torch.cat([torch.linspace(-100.0, 100.0, 200001), 5.0 * torch.randn(100000, generator=g),
                   torch.tensor([0.0, 1e-30, -1e-30, 88.0, -87.3, -87.4, 40.0, -40.0, 24.9, -24.9,
                                 -25.0, 25.0])])
    dx = x.cuda()
    ex = torch.empty_like(dx)
    sig = torch.empty_like(dx)
    sig3 = torch.empty_like(dx)
    silut = torch.empty_like(dx)
    rc = f(ctypes.c_void_p(dx.data_ptr()), ctypes.c_void_p(ex.data_ptr()),
           ctypes.c_void_p(sig.data_ptr()), ctypes.c_void_p(sig3.data_ptr()),
           ctypes.c_void_p(silut.data_ptr()), x.numel(),
           ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert rc == 0
    cuda_exp = torch.exp(dx).cpu().double().numpy()  # CUDA's expf
    torch.cuda.synchronize()
    xd = x.double().numpy()
    e64 = np.exp(xd)
    got = ex.cpu().double().numpy()
    normal = (xd > -87.3) & (xd < 88.5)
    rel = np.abs(got[normal] - e64[normal]) / e64[normal]
    assert rel.max() < 6e-6, rel.max()
    rel_cuda = np.abs(got[normal] - cuda_exp[normal]) / cuda_exp[normal]
    assert rel_cuda.max() < 6e-6, rel_cuda.max()
    assert np.all(got[xd <= -87.3] <= 1.22e-38)  # e^-87.3 = 1.2193e-38
    s64 = 1.0 / (1.0 + np.exp(-xd))
    s = sig.cpu().double().numpy()
    assert np.max(np.abs(s - s64)) < 2e-6
    big = s64 > 1e-30
    assert np.max(np.abs(s[big] - s64[big]) / s64[big]) < 1e-5
    s3 = sig3.cpu().double().numpy()
    assert np.all(np.isfinite(s3))
    assert np.max(np.abs(s3 - s64)) < 2e-6
    unc = xd > -24.9
    assert np.max(np.abs(s3[unc] - s64[unc]) / s64[unc]) < 2e-5
    assert np.max(np.abs(s3[~unc] - s64[~unc])) < 1.46e-11
    st = silut.cpu().double().numpy()
    silu64 = xd * s64
    err_t = np.abs(st - silu64)
    assert np.all(err_t <= 2.5e-4 * np.abs(xd) + 2e-7 * np.abs(silu64) + 1e-30), \
        (err_t / np.maximum(np.abs(xd), 1e-30)).max()
