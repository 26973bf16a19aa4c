// Self-tests of the tensor-core building blocks used by the tensor-core scan:
// D[128 x N] = A[128 x K] * B[N x K]^T, kind::tf32, K = 8 per instruction,
// D in tensor memory; A either in tensor memory or in shared memory, shared
// operands either no-swizzle K-major core matrices or the 128-byte swizzled
// K-major layout.  Exposed through naju_testing.h so the test suite can check
// the operand conventions against a host product.
#include <cuda_bf16.h>

#include "naju.h"
#include "naju_common.cuh"
#include "naju_tc.cuh"
#include "naju_testing.h"

namespace naju {

__global__ void __launch_bounds__(128, 1)
tc_selftest_kernel(const float* __restrict__ A, const float* __restrict__ B,
                   float* __restrict__ D, int N, int K, uint32_t ncols, int* status) {
    extern __shared__ float4 smem4[];
    unsigned char* sb = reinterpret_cast<unsigned char*>(smem4);
    __shared__ uint64_t mbar;
    __shared__ uint32_t taddr_s;
    const int tid = threadIdx.x, warp = tid / 32;

    if (warp == 0) {
        tc::tmem_alloc(&taddr_s, ncols);
        tc::tmem_relinquish();
    }
    if (tid == 0) tc::mbar_init(&mbar, 1);
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    const uint32_t tbase = taddr_s;
    const uint32_t lane_off = (uint32_t)(warp * 32) << 16;

    // A row `tid` -> TMEM lane `tid`, columns [0, K).
    for (int k0 = 0; k0 < K; k0 += 16) {
        float v[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) v[i] = A[tid * K + k0 + i];
        tc::tmem_st16(tbase + lane_off + k0, v);
    }
    // B [N x K] -> shared memory, K-major core matrices.
    for (int e = tid; e < N * K; e += 128) {
        const int row = e / K, k = e % K;
        *reinterpret_cast<float*>(sb + tc::kmajor_offset(row, k, K)) = B[e];
    }
    tc::tmem_st_wait();
    tc::fence_proxy_async();
    tc::fence_before_sync();
    __syncthreads();
    if (tid == 0) {
        tc::fence_after_sync();
        const uint32_t idesc = tc::idesc_tf32(128, N);
        const uint32_t sbase = tc::smem_u32(sb);
        for (int ks = 0; ks < K / 8; ++ks) {
            const uint64_t bdesc = tc::sdesc(sbase + ks * 256, 128, 32 * K);
            tc::mma_tf32_ts(tbase + K, tbase + ks * 8, bdesc, idesc, ks > 0 ? 1u : 0u);
        }
        tc::mma_commit(&mbar);
    }
    const bool done = tc::mbar_wait(&mbar, 0, 1LL << 22);
    if (!done && tid == 0) atomicOr(status, 1 << NAJU_ERR_TIMEOUT);
    tc::fence_after_sync();
    for (int n0 = 0; n0 < N; n0 += 16) {
        float v[16];
        tc::tmem_ld16(tbase + lane_off + K + n0, v);
        tc::tmem_ld_wait();
#pragma unroll
        for (int i = 0; i < 16; ++i) D[tid * N + n0 + i] = done ? v[i] : __int_as_float(0x7fc00000);
    }
    tc::fence_before_sync();
    __syncthreads();
    if (warp == 0) tc::tmem_dealloc(tbase, ncols);
}


// Both operands from shared memory.  A is stored as an R x K tile (R = 64 or
// 128) while the MMA always reads 128 rows: rows past R read other bytes of
// the A region (zeros here), which is how a 64-row operand rides an M = 128
// MMA.  swz_a / swz_b select the 128-byte swizzled layout (K % 32 == 0).
__global__ void __launch_bounds__(128, 1)
tc_selftest_ss_kernel(const float* __restrict__ A, const float* __restrict__ B,
                      float* __restrict__ D, int N, int K, int R, int swz_a, int swz_b,
                      uint32_t ncols, int* status) {
    extern __shared__ __align__(1024) float4 smem4[];
    unsigned char* sa = reinterpret_cast<unsigned char*>(smem4);
    unsigned char* sb = sa + (size_t)128 * K * 4;
    __shared__ uint64_t mbar;
    __shared__ uint32_t taddr_s;
    const int tid = threadIdx.x, warp = tid / 32;

    if (warp == 0) {
        tc::tmem_alloc(&taddr_s, ncols);
        tc::tmem_relinquish();
    }
    if (tid == 0) tc::mbar_init(&mbar, 1);
    for (int e = tid; e < 128 * K; e += 128) reinterpret_cast<float*>(sa)[e] = 0.f;
    __syncthreads();
    for (int e = tid; e < R * K; e += 128) {
        const int row = e / K, k = e % K;
        const uint32_t off = swz_a ? tc::sw128_offset(row, k, R) : tc::kmajor_offset(row, k, K);
        *reinterpret_cast<float*>(sa + off) = A[e];
    }
    for (int e = tid; e < N * K; e += 128) {
        const int row = e / K, k = e % K;
        const uint32_t off = swz_b ? tc::sw128_offset(row, k, N) : tc::kmajor_offset(row, k, K);
        *reinterpret_cast<float*>(sb + off) = B[e];
    }
    tc::fence_proxy_async();
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    const uint32_t tbase = taddr_s;
    const uint32_t lane_off = (uint32_t)(warp * 32) << 16;
    if (tid == 0) {
        const uint32_t idesc = tc::idesc_tf32(128, N);
        const uint32_t abase = tc::smem_u32(sa), bbase = tc::smem_u32(sb);
        for (int ks = 0; ks < K / 8; ++ks) {
            const uint64_t ad = swz_a ? tc::sdesc_sw128(abase + (ks >> 2) * R * 128 + (ks & 3) * 32)
                                      : tc::sdesc(abase + ks * 256, 128, 32 * K);
            const uint64_t bd = swz_b ? tc::sdesc_sw128(bbase + (ks >> 2) * N * 128 + (ks & 3) * 32)
                                      : tc::sdesc(bbase + ks * 256, 128, 32 * K);
            tc::mma_tf32_ss(tbase, ad, bd, idesc, ks > 0 ? 1u : 0u);
        }
        tc::mma_commit(&mbar);
    }
    const bool done = tc::mbar_wait(&mbar, 0, 1LL << 22);
    if (!done && tid == 0) atomicOr(status, 1 << NAJU_ERR_TIMEOUT);
    tc::fence_after_sync();
    for (int n0 = 0; n0 < N; n0 += 16) {
        float v[16];
        tc::tmem_ld16(tbase + lane_off + n0, v);
        tc::tmem_ld_wait();
#pragma unroll
        for (int i = 0; i < 16; ++i) D[tid * N + n0 + i] = done ? v[i] : __int_as_float(0x7fc00000);
    }
    tc::fence_before_sync();
    __syncthreads();
    if (warp == 0) tc::tmem_dealloc(tbase, ncols);
}

// General form: D = A[M x K] * B[N x K]^T with both operands in shared
// memory, in the layouts the block-form kernels use.
//  kind 0 (tf32): a_mn = 0 stores A as its [M x K] tile in the 128-byte
//    swizzled layout (K-major operand); a_mn = 1 as the transposed [K x M]
//    tile with 32-byte swizzle atoms (MN-major operand).  Likewise B.
//  kind 1 (bf16, kind::f16): A and B are split into bf16 hi + lo tiles (one
//    128-byte swizzled row tile serves both majors: a_mn selects whether the
//    tile holds [M x K] or [K x M]) and D = hi.hi + hi.lo + lo.hi.
// M = 64 or 128; d_lane (0 or 16) is the lane offset of D in tensor memory.
// Every lane of the D columns is copied out raw (D_out[128][N]).
__global__ void __launch_bounds__(128, 1)
tc_selftest_gen_kernel(const float* __restrict__ A, const float* __restrict__ B,
                       float* __restrict__ D, int M, int N, int K, int a_mn, int b_mn,
                       int d_lane, int kind, uint32_t ncols, int* status) {
    extern __shared__ __align__(1024) float4 smem4[];
    unsigned char* sa = reinterpret_cast<unsigned char*>(smem4);
    unsigned char* sb = sa + (size_t)M * K * 4;  // tf32 A, or bf16 A hi + lo
    __shared__ uint64_t mbar;
    __shared__ uint32_t taddr_s;
    const int tid = threadIdx.x, warp = tid / 32;

    if (warp == 0) {
        tc::tmem_alloc(&taddr_s, ncols);
        tc::tmem_relinquish();
    }
    if (tid == 0) tc::mbar_init(&mbar, 1);
    if (kind == 0) {
        for (int e = tid; e < M * K; e += 128) {
            const int m = e / K, k = e % K;
            const uint32_t off = a_mn ? tc::mn32_offset(k, m, K) : tc::sw128_offset(m, k, M);
            *reinterpret_cast<float*>(sa + off) = A[e];
        }
        for (int e = tid; e < N * K; e += 128) {
            const int n = e / K, k = e % K;
            const uint32_t off = b_mn ? tc::mn32_offset(k, n, K) : tc::sw128_offset(n, k, N);
            *reinterpret_cast<float*>(sb + off) = B[e];
        }
    } else {
        // bf16 tiles hold at most 64 columns: the stored tile is [rows][64]
        const size_t ha = (size_t)M * K * 2, hb = (size_t)N * K * 2;
        for (int e = tid; e < M * K; e += 128) {
            const int m = e / K, k = e % K;
            const uint32_t off = a_mn ? tc::bf_offset(k, m) : tc::bf_offset(m, k);
            const __nv_bfloat16 h = __float2bfloat16_rn(A[e]);
            *reinterpret_cast<__nv_bfloat16*>(sa + off) = h;
            *reinterpret_cast<__nv_bfloat16*>(sa + ha + off) =
                __float2bfloat16_rn(A[e] - __bfloat162float(h));
        }
        for (int e = tid; e < N * K; e += 128) {
            const int n = e / K, k = e % K;
            const uint32_t off = b_mn ? tc::bf_offset(k, n) : tc::bf_offset(n, k);
            const __nv_bfloat16 h = __float2bfloat16_rn(B[e]);
            *reinterpret_cast<__nv_bfloat16*>(sb + off) = h;
            *reinterpret_cast<__nv_bfloat16*>(sb + hb + off) =
                __float2bfloat16_rn(B[e] - __bfloat162float(h));
        }
    }
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    const uint32_t tbase = taddr_s;
    const uint32_t lane_off = (uint32_t)(warp * 32) << 16;
    // zero the D columns of every lane (the MMA overwrites only its own lanes)
    for (int n0 = 0; n0 < N; n0 += 16) {
        float z[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) z[i] = 0.f;
        tc::tmem_st16(tbase + lane_off + n0, z);
    }
    tc::tmem_st_wait();
    tc::fence_proxy_async();
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    if (tid == 0) {
        const uint32_t abase = tc::smem_u32(sa), bbase = tc::smem_u32(sb);
        const uint32_t dcol = tbase + ((uint32_t)d_lane << 16);
        if (kind == 0) {
            const uint32_t idesc = tc::idesc_tf32(M, N, a_mn != 0, b_mn != 0);
            for (int ks = 0; ks < K / 8; ++ks) {
                const uint64_t ad = a_mn ? tc::sdesc_mn32(abase, K, ks)
                                         : tc::sdesc_sw128(abase + (ks >> 2) * M * 128 + (ks & 3) * 32);
                const uint64_t bd = b_mn ? tc::sdesc_mn32(bbase, K, ks)
                                         : tc::sdesc_sw128(bbase + (ks >> 2) * N * 128 + (ks & 3) * 32);
                tc::mma_tf32_ss(dcol, ad, bd, idesc, ks > 0 ? 1u : 0u);
            }
        } else {
            const uint32_t idesc = tc::idesc_bf16(M, N, a_mn != 0, b_mn != 0);
            const uint32_t ha = (uint32_t)M * K * 2, hb = (uint32_t)N * K * 2;
            const uint32_t pa[3] = {0, 0, ha}, pb[3] = {0, hb, 0};
            bool first = true;
            for (int pr = 0; pr < 3; ++pr)
                for (int ks = 0; ks < K / 16; ++ks) {
                    const uint64_t ad = a_mn ? tc::sdesc_bf_mn(abase + pa[pr], ks)
                                             : tc::sdesc_bf_k(abase + pa[pr], ks);
                    const uint64_t bd = b_mn ? tc::sdesc_bf_mn(bbase + pb[pr], ks)
                                             : tc::sdesc_bf_k(bbase + pb[pr], ks);
                    tc::mma_bf16_ss(dcol, ad, bd, idesc, first ? 0u : 1u);
                    first = false;
                }
        }
        tc::mma_commit(&mbar);
    }
    const bool done = tc::mbar_wait(&mbar, 0, 1LL << 22);
    if (!done && tid == 0) atomicOr(status, 1 << NAJU_ERR_TIMEOUT);
    tc::fence_after_sync();
    for (int n0 = 0; n0 < N; n0 += 16) {
        float v[16];
        tc::tmem_ld16(tbase + lane_off + n0, v);
        tc::tmem_ld_wait();
#pragma unroll
        for (int i = 0; i < 16; ++i) D[tid * N + n0 + i] = done ? v[i] : __int_as_float(0x7fc00000);
    }
    tc::fence_before_sync();
    __syncthreads();
    if (warp == 0) tc::tmem_dealloc(tbase, ncols);
}

}  // namespace naju

extern "C" naju_status naju_testing_tc_mma_gen(int32_t M, int32_t N, int32_t K, int32_t a_mn,
                                               int32_t b_mn, int32_t d_lane, int32_t kind,
                                               const float* A, const float* B, float* D,
                                               int* status, void* stream) {
    if (!A || !B || !D || !status) return NAJU_ERR_INVALID_ARG;
    if ((M != 64 && M != 128) || N < 16 || N > 128 || N % 16 != 0 || K < 32 || K > 128 ||
        K % 32 != 0 || (kind != 0 && kind != 1))
        return NAJU_ERR_UNSUPPORTED;
    if (kind == 0 && b_mn && N % 32 != 0) return NAJU_ERR_UNSUPPORTED;  // 32-column blocks
    // bf16 tiles: exactly 64 columns (one 128-byte line per row)
    if (kind == 1 && ((a_mn ? M : K) != 64 || (b_mn ? N : K) != 64)) return NAJU_ERR_UNSUPPORTED;
    if (d_lane != 0 && !(d_lane == 16 && M == 64)) return NAJU_ERR_UNSUPPORTED;
    uint32_t ncols = 32;
    while (ncols < (uint32_t)N) ncols <<= 1;
    const size_t smem = sizeof(float) * ((size_t)M * K + (size_t)N * K);
    cudaError_t e = cudaFuncSetAttribute(naju::tc_selftest_gen_kernel,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return NAJU_ERR_CUDA;
    naju::tc_selftest_gen_kernel<<<1, 128, smem, static_cast<cudaStream_t>(stream)>>>(
        A, B, D, M, N, K, a_mn, b_mn, d_lane, kind, ncols, status);
    return cudaGetLastError() == cudaSuccess ? NAJU_OK : NAJU_ERR_CUDA;
}

extern "C" naju_status naju_testing_tc_mma(int32_t N, int32_t K, const float* A, const float* B,
                                           float* D, int* status, void* stream) {
    if (!A || !B || !D || !status) return NAJU_ERR_INVALID_ARG;
    if (N < 16 || N > 256 || N % 16 != 0 || K < 16 || K % 16 != 0 || K + N > 512)
        return NAJU_ERR_UNSUPPORTED;
    uint32_t ncols = 32;
    while (ncols < (uint32_t)(K + N)) ncols <<= 1;
    const size_t smem = sizeof(float) * (size_t)N * K;
    cudaError_t e = cudaFuncSetAttribute(naju::tc_selftest_kernel,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return NAJU_ERR_CUDA;
    naju::tc_selftest_kernel<<<1, 128, smem, static_cast<cudaStream_t>(stream)>>>(A, B, D, N, K,
                                                                                 ncols, status);
    return cudaGetLastError() == cudaSuccess ? NAJU_OK : NAJU_ERR_CUDA;
}

extern "C" naju_status naju_testing_tc_mma_ss(int32_t N, int32_t K, int32_t rows_a,
                                              int32_t swz_a, int32_t swz_b, const float* A,
                                              const float* B, float* D, int* status,
                                              void* stream) {
    if (!A || !B || !D || !status) return NAJU_ERR_INVALID_ARG;
    if (N < 16 || N > 128 || N % 16 != 0 || K < 16 || K > 128 || K % 16 != 0 ||
        (rows_a != 64 && rows_a != 128))
        return NAJU_ERR_UNSUPPORTED;
    if ((swz_a || swz_b) && K % 32 != 0) return NAJU_ERR_UNSUPPORTED;
    if (swz_b && N % 8 != 0) return NAJU_ERR_UNSUPPORTED;
    uint32_t ncols = 32;
    while (ncols < (uint32_t)N) ncols <<= 1;
    const size_t smem = sizeof(float) * ((size_t)128 * K + (size_t)N * K);
    cudaError_t e = cudaFuncSetAttribute(naju::tc_selftest_ss_kernel,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return NAJU_ERR_CUDA;
    naju::tc_selftest_ss_kernel<<<1, 128, smem, static_cast<cudaStream_t>(stream)>>>(
        A, B, D, N, K, rows_a, swz_a, swz_b, ncols, status);
    return cudaGetLastError() == cudaSuccess ? NAJU_OK : NAJU_ERR_CUDA;
}

namespace naju {
// The block-form kernels' exponential and sigmoids, element by element: e^x
// as 2^(x log2 e) on the MUFU base-2 unit, sigma(x) = 1 / (1 + e^{-x}), and
// the forward's shared-reciprocal form for three arguments (x, x / 2, -x):
// q_i = 1 + min(e^{-v_i}, 2^36), r = 1 / (q0 q1 q2), sigma(x) = r q1 q2.
__global__ void fast_math_kernel(const float* __restrict__ x, float* __restrict__ ex,
                                 float* __restrict__ sig, float* __restrict__ sig3,
                                 float* __restrict__ silut, int64_t n) {
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n;
         i += (int64_t)gridDim.x * blockDim.x) {
        const float v = x[i];
        ex[i] = expa_(v);
        sig[i] = sigmoidx_(v);
        constexpr float kL2e = 1.4426950408889634f;
        const float q0 = 1.f + exp2a_(fminf(-kL2e * v, 36.f));
        const float q1 = 1.f + exp2a_(fminf(-kL2e * (0.5f * v), 36.f));
        const float q2 = 1.f + exp2a_(fminf(kL2e * v, 36.f));
        const float r = rcpa_(q0 * (q1 * q2));
        sig3[i] = r * (q1 * q2);
        silut[i] = siluta_(v);
    }
}
}  // namespace naju

extern "C" naju_status naju_testing_fast_math(const float* x, float* ex, float* sig, float* sig3,
                                              float* silut, int64_t n, void* stream) {
    if (!x || !ex || !sig || !sig3 || !silut || n < 0) return NAJU_ERR_INVALID_ARG;
    if (n == 0) return NAJU_OK;
    const int blocks = (int)((n + 255) / 256 < 1184 ? (n + 255) / 256 : 1184);
    naju::fast_math_kernel<<<blocks, 256, 0, static_cast<cudaStream_t>(stream)>>>(x, ex, sig, sig3,
                                                                                silut, n);
    return cudaGetLastError() == cudaSuccess ? NAJU_OK : NAJU_ERR_CUDA;
}
