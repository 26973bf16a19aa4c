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
