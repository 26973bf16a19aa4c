// Shared device helpers for the Naju scan kernels (sm_100a).
#pragma once
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "naju.h"

namespace naju {

__host__ __device__ __forceinline__ int64_t min64(int64_t a, int64_t b) { return a < b ? a : b; }
__host__ __device__ __forceinline__ int64_t max64(int64_t a, int64_t b) { return a > b ? a : b; }

// ----------------------------------------------------------------- dtypes
__device__ __forceinline__ float to_f(float v) { return v; }
__device__ __forceinline__ float to_f(__nv_bfloat16 v) { return __bfloat162float(v); }
template <typename T> __device__ __forceinline__ T from_f(float v);
template <> __device__ __forceinline__ float from_f<float>(float v) { return v; }
template <> __device__ __forceinline__ __nv_bfloat16 from_f<__nv_bfloat16>(float v) {
    return __float2bfloat16_rn(v);
}

// Load 8 consecutive activations as fp32 (16-byte aligned for bf16, two
// 16-byte loads for fp32).
__device__ __forceinline__ void load8(const __nv_bfloat16* p, float* o) {
    uint4 r = *reinterpret_cast<const uint4*>(p);
    const __nv_bfloat162* h2 = reinterpret_cast<const __nv_bfloat162*>(&r);
#pragma unroll
    for (int k = 0; k < 4; ++k) {
        float2 f = __bfloat1622float2(h2[k]);
        o[2 * k] = f.x;
        o[2 * k + 1] = f.y;
    }
}
__device__ __forceinline__ void load8(const float* p, float* o) {
    float4 a = reinterpret_cast<const float4*>(p)[0];
    float4 b = reinterpret_cast<const float4*>(p)[1];
    o[0] = a.x; o[1] = a.y; o[2] = a.z; o[3] = a.w;
    o[4] = b.x; o[5] = b.y; o[6] = b.z; o[7] = b.w;
}
__device__ __forceinline__ void store8(__nv_bfloat16* p, const float* v) {
    uint4 r;
    __nv_bfloat162* h2 = reinterpret_cast<__nv_bfloat162*>(&r);
#pragma unroll
    for (int k = 0; k < 4; ++k) h2[k] = __floats2bfloat162_rn(v[2 * k], v[2 * k + 1]);
    *reinterpret_cast<uint4*>(p) = r;
}
__device__ __forceinline__ void store8(float* p, const float* v) {
    reinterpret_cast<float4*>(p)[0] = make_float4(v[0], v[1], v[2], v[3]);
    reinterpret_cast<float4*>(p)[1] = make_float4(v[4], v[5], v[6], v[7]);
}

// ------------------------------------------------------------ activations
// CUDA's fast exponential and its round-to-nearest reciprocal (inf -> 0, so
// sigmoid saturates cleanly); the accuracy of each use is covered by the
// parity tests against the fp64 oracle.
__device__ __forceinline__ float rcpf_(float v) { return __frcp_rn(v); }
// Single-instruction approximate reciprocal (PTX rcp.approx.ftz.f32; about
// one ulp), for the tensor-core path whose operands are tf32 anyway.
__device__ __forceinline__ float rcpa_(float v) {
    float r;
    asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(r) : "f"(v));
    return r;
}
__device__ __forceinline__ float sigmoida_(float v) { return rcpa_(1.0f + __expf(-v)); }
// e^v as 2^(v log2 e) on the MUFU unit (PTX ex2.approx.ftz.f32: a few ulp,
// results below the normal range flushed to zero), and the sigmoid on it.
// The block-form tensor-core kernels use these; the parity tests against the
// fp64 oracle bound their effect.
__device__ __forceinline__ float exp2a_(float v) {
    float r;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(r) : "f"(v));
    return r;
}
__device__ __forceinline__ float expa_(float v) { return exp2a_(v * 1.4426950408889634f); }
__device__ __forceinline__ float sigmoidx_(float v) { return rcpa_(1.0f + expa_(-v)); }
// tanh on the MUFU unit (PTX tanh.approx.f32: relative error about 2^-11) and
// SiLU through it, v sigma(v) = h + h tanh(h) with h = v / 2 (absolute error
// at most about 2^-12 |v|).  Used only where the result is rounded to bf16
// right after (the forward's output gate with bf16 outputs).
__device__ __forceinline__ float tanha_(float v) {
    float r;
    asm("tanh.approx.f32 %0, %1;" : "=f"(r) : "f"(v));
    return r;
}
__device__ __forceinline__ float siluta_(float v) {
    const float h = 0.5f * v;
    return fmaf(h, tanha_(h), h);
}
__device__ __forceinline__ float silua_(float v) { return v * sigmoida_(v); }
__device__ __forceinline__ float sigmoidf_(float v) { return rcpf_(1.0f + __expf(-v)); }
__device__ __forceinline__ float siluf_(float v) { return v * sigmoidf_(v); }
// d/dv SiLU(v) = s (1 + v (1 - s)), s = sigmoid(v)
__device__ __forceinline__ float dsiluf_(float v) {
    float s = sigmoidf_(v);
    return s * (1.0f + v * (1.0f - s));
}

// ------------------------------------------------ inter-block signalling
__device__ __forceinline__ int ld_acquire(const int* p) {
    int v;
    asm volatile("ld.acquire.gpu.global.b32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}
__device__ __forceinline__ void st_release(int* p, int v) {
    asm volatile("st.release.gpu.global.b32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}

// Bounded wait for *flag == 1 by one thread.  Returns false after
// `limit` polls (~limit * 0.5 us) and records NAJU_ERR_TIMEOUT.
__device__ __forceinline__ bool wait_flag(const int* flag, int* status, long long limit) {
    long long it = 0;
    unsigned ns = 32;
    while (ld_acquire(flag) != 1) {
        if (++it > limit) {
            atomicOr(status, 1 << NAJU_ERR_TIMEOUT);
            return false;
        }
        __nanosleep(ns);
        if (ns < 512) ns <<= 1;
    }
    return true;
}

// Workspace header: the status word and the per-launch work tickets.  The
// forward clears fwd_ticket (with its flags, which follow it) before each
// launch and the backward clears bwd_ticket; status persists until read.
struct WsHeader {
    int status;
    int pad0[31];
    int fwd_ticket;
    int pad1[31];
    int bwd_ticket;
    int pad2[31];
    int pad3[32];
};
static_assert(sizeof(WsHeader) == 512, "header is two 256-byte blocks");

}  // namespace naju

namespace naju {

// ------------------------------------------------------ async staging
// 16-byte global -> shared copy; src_bytes = 0 zero-fills the destination
// (no global bytes are read; `src` must still be a valid address).
__device__ __forceinline__ void cp_async16(void* dst, const void* src, int src_bytes) {
    const unsigned d = static_cast<unsigned>(__cvta_generic_to_shared(dst));
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;\n" ::"r"(d), "l"(src),
                 "r"(src_bytes)
                 : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;\n" ::); }
template <int N_>
__device__ __forceinline__ void cp_async_wait() {
    asm volatile("cp.async.wait_group %0;\n" ::"n"(N_) : "memory");
}

// Stage `rows` rows (token t0 + r, r in [0, rows)) of a [Bt, L, width]
// tensor, columns [col0, col0 + cols), into dst[rows][cols] (element type T).
// Rows outside [0, tlim) and columns past `width` are zero.  vec: the 16-byte
// path is legal (width * sizeof(T) and col0 * sizeof(T) multiples of 16,
// cols * sizeof(T) multiple of 16); otherwise plain loads are used.
template <typename T>
__device__ __forceinline__ void stage_rows(T* dst, const T* src_b, int64_t width, int64_t t0,
                                           int rows, int64_t tlim, int64_t col0, int cols,
                                           bool vec, int tid, int nthreads) {
    constexpr int G = 16 / sizeof(T);  // elements per granule
    if (vec) {
        const int gpr = cols / G;      // granules per row
        for (int e = tid; e < rows * gpr; e += nthreads) {
            const int r = e / gpr, gi = e % gpr;
            const int64_t t = t0 + r;
            const int64_t col = col0 + (int64_t)gi * G;
            const bool ok = t >= 0 && t < tlim && col < width;
            const T* s = ok ? src_b + t * width + col : src_b;
            cp_async16(dst + r * cols + gi * G, s, ok ? 16 : 0);
        }
    } else {
        for (int e = tid; e < rows * cols; e += nthreads) {
            const int r = e / cols, ci = e % cols;
            const int64_t t = t0 + r;
            const int64_t col = col0 + ci;
            T v = T(0.f);
            if (t >= 0 && t < tlim && col < width) v = src_b[t * width + col];
            dst[r * cols + ci] = v;
        }
    }
}

}  // namespace naju
