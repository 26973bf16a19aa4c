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
