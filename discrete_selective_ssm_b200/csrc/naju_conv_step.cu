// Standalone causal depthwise conv + SiLU (forward and backward) and the
// single-token decode step (sm_100a, CUDA cores; both are memory-bound).
//
// Conv (Naju reproduction README flowchart, "causal depthwise conv + SiLU"):
//   p_t = bias + sum_{k<4} w[k] u_{t-3+k} (zero left padding), h_t = SiLU(p_t).
// Decode step (README, "Core equations", one token on a carried state):
//   x <- sigmoid(a) x + sigmoid(b) h B^T,  y = (x . C)/sqrt(N) + D h,  y *= SiLU(z).
#include <algorithm>

#include "naju_common.cuh"
#include "naju_kernels.h"

namespace naju {

constexpr int kConvRun = 32;      // tokens per thread, forward
constexpr int kConvRunBwd = 64;   // tokens per thread, backward

// One thread per (channel, run of tokens); a warp covers 32 consecutive
// channels of a token row, so every load and store is a coalesced row slice.
template <typename Tin, typename Tout>
__global__ void __launch_bounds__(128)
conv_fwd_kernel(int64_t L, int64_t d, const Tin* __restrict__ u, const float* __restrict__ w,
                const float* __restrict__ bias, Tout* __restrict__ h) {
    const int64_t c = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (c >= d) return;
    const int64_t t0 = (int64_t)blockIdx.y * kConvRun;
    const int64_t bb = blockIdx.z;
    const float w0 = w[c * 4], w1 = w[c * 4 + 1], w2 = w[c * 4 + 2], w3 = w[c * 4 + 3];
    const float wb = bias ? bias[c] : 0.f;
    const Tin* col = u + bb * L * d + c;
    Tout* hc = h + bb * L * d + c;
    float u0 = t0 >= 3 ? to_f(col[(t0 - 3) * d]) : 0.f;
    float u1 = t0 >= 2 ? to_f(col[(t0 - 2) * d]) : 0.f;
    float u2 = t0 >= 1 ? to_f(col[(t0 - 1) * d]) : 0.f;
    const int n = (int)min64(kConvRun, L - t0);
#pragma unroll 8
    for (int k = 0; k < n; ++k) {
        const float u3 = to_f(col[(t0 + k) * d]);
        const float pre = wb + w0 * u0 + w1 * u1 + w2 * u2 + w3 * u3;
        hc[(t0 + k) * d] = from_f<Tout>(siluf_(pre));
        u0 = u1; u1 = u2; u2 = u3;
    }
}

// Backward: dp_t = dh_t SiLU'(p_t); du_s = sum_k w[k] dp_{s+3-k};
// dw[k] = sum_t dp_t u_{t-3+k}; dbias = sum_t dp_t.  Each thread recomputes
// dp on its run plus three tokens of look-ahead, writes du for its run and
// adds its run's share of dw, dbias with one atomic per value (the caller
// zeroes dw, dbias first).
template <typename Tin, typename Tout>
__global__ void __launch_bounds__(128)
conv_bwd_kernel(int64_t L, int64_t d, const Tin* __restrict__ u, const float* __restrict__ w,
                const float* __restrict__ bias, const Tin* __restrict__ dh,
                Tout* __restrict__ du, float* __restrict__ dw, float* __restrict__ dbias) {
    const int64_t c = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (c >= d) return;
    const int64_t t0 = (int64_t)blockIdx.y * kConvRunBwd;
    const int64_t bb = blockIdx.z;
    const float w0 = w[c * 4], w1 = w[c * 4 + 1], w2 = w[c * 4 + 2], w3 = w[c * 4 + 3];
    const float wb = bias ? bias[c] : 0.f;
    const Tin* col = u + bb * L * d + c;
    const Tin* dhc = dh + bb * L * d + c;
    Tout* duc = du + bb * L * d + c;
    auto uat = [&](int64_t t) { return (t >= 0 && t < L) ? to_f(col[t * d]) : 0.f; };
    auto dpat = [&](int64_t t) {
        if (t >= L) return 0.f;
        const float pre = wb + w0 * uat(t - 3) + w1 * uat(t - 2) + w2 * uat(t - 1) + w3 * uat(t);
        return to_f(dhc[t * d]) * dsiluf_(pre);
    };
    const int n = (int)min64(kConvRunBwd, L - t0);
    // Sliding window over dp_{s+3}, dp_{s+2}, dp_{s+1}, dp_s, walking s downward.
    const int64_t tl = t0 + n - 1;
    float dp1 = dpat(tl + 1), dp2 = dpat(tl + 2), dp3 = dpat(tl + 3);
    float sw0 = 0.f, sw1 = 0.f, sw2 = 0.f, sw3 = 0.f, sb = 0.f;
    float um3 = uat(tl - 3), um2 = uat(tl - 2), um1 = uat(tl - 1), u0v = uat(tl);
    for (int k = n - 1; k >= 0; --k) {
        const int64_t s = t0 + k;
        const float pre = wb + w0 * um3 + w1 * um2 + w2 * um1 + w3 * u0v;
        const float dp0 = to_f(dhc[s * d]) * dsiluf_(pre);
        duc[s * d] = from_f<Tout>(w3 * dp0 + w2 * dp1 + w1 * dp2 + w0 * dp3);
        sw0 += dp0 * um3; sw1 += dp0 * um2; sw2 += dp0 * um1; sw3 += dp0 * u0v;
        sb += dp0;
        dp3 = dp2; dp2 = dp1; dp1 = dp0;
        u0v = um1; um1 = um2; um2 = um3; um3 = uat(s - 4);
    }
    atomicAdd(dw + c * 4 + 0, sw0);
    atomicAdd(dw + c * 4 + 1, sw1);
    atomicAdd(dw + c * 4 + 2, sw2);
    atomicAdd(dw + c * 4 + 3, sw3);
    if (dbias) atomicAdd(dbias + c, sb);
}

template <typename Tin, typename Tout>
static cudaError_t conv_fwd_t(int64_t Bt, int64_t L, int64_t d, const void* u, const float* w,
                              const float* bias, void* h, cudaStream_t st) {
    dim3 grid((unsigned)((d + 127) / 128), (unsigned)((L + kConvRun - 1) / kConvRun),
              (unsigned)Bt);
    conv_fwd_kernel<Tin, Tout><<<grid, 128, 0, st>>>(L, d, static_cast<const Tin*>(u), w, bias,
                                                     static_cast<Tout*>(h));
    return cudaGetLastError();
}

cudaError_t launch_conv_fwd(int64_t Bt, int64_t L, int64_t d, const void* u, const float* w,
                            const float* bias, void* h, int dtype, int out_dtype,
                            cudaStream_t st) {
    if (dtype == NAJU_F32) return conv_fwd_t<float, float>(Bt, L, d, u, w, bias, h, st);
    if (out_dtype == NAJU_BF16)
        return conv_fwd_t<__nv_bfloat16, __nv_bfloat16>(Bt, L, d, u, w, bias, h, st);
    return conv_fwd_t<__nv_bfloat16, float>(Bt, L, d, u, w, bias, h, st);
}

template <typename Tin, typename Tout>
static cudaError_t conv_bwd_t(int64_t Bt, int64_t L, int64_t d, const void* u, const float* w,
                              const float* bias, const void* dh, void* du, float* dw,
                              float* dbias, cudaStream_t st) {
    cudaError_t e = cudaMemsetAsync(dw, 0, sizeof(float) * d * 4, st);
    if (e == cudaSuccess && dbias) e = cudaMemsetAsync(dbias, 0, sizeof(float) * d, st);
    if (e != cudaSuccess) return e;
    dim3 grid((unsigned)((d + 127) / 128), (unsigned)((L + kConvRunBwd - 1) / kConvRunBwd),
              (unsigned)Bt);
    conv_bwd_kernel<Tin, Tout><<<grid, 128, 0, st>>>(
        L, d, static_cast<const Tin*>(u), w, bias, static_cast<const Tin*>(dh),
        static_cast<Tout*>(du), dw, dbias);
    return cudaGetLastError();
}

cudaError_t launch_conv_bwd(int64_t Bt, int64_t L, int64_t d, const void* u, const float* w,
                            const float* bias, const void* dh, void* du, float* dw,
                            float* dbias, int dtype, int out_dtype, cudaStream_t st) {
    if (dtype == NAJU_F32)
        return conv_bwd_t<float, float>(Bt, L, d, u, w, bias, dh, du, dw, dbias, st);
    if (out_dtype == NAJU_BF16)
        return conv_bwd_t<__nv_bfloat16, __nv_bfloat16>(Bt, L, d, u, w, bias, dh, du, dw,
                                                        dbias, st);
    return conv_bwd_t<__nv_bfloat16, float>(Bt, L, d, u, w, bias, dh, du, dw, dbias, st);
}

// ------------------------------------------------------------ decode step
// S = N/4 threads share a channel, each holding 4 consecutive state entries,
// so a warp's float4 accesses cover whole contiguous state rows.
// One decode token: x <- f x + i h B^T, y = (x.C s + D h) SiLU(z).  With CONV,
// h = SiLU(bias + w0 s0 + w1 s1 + w2 s2 + w3 u) from the conv state
// s = (s0, s1, s2) (the previous three inputs, oldest first), which then
// becomes (s1, s2, u).
//
// A warp owns 32 consecutive channels.  Lane l first computes the gates of
// channel l once (coalesced per-channel loads); then the warp streams the 32
// state rows, Q = N/4 lanes per row (one float4 each), so every load and
// store instruction covers 128/N whole contiguous rows; the gate values
// reach the row lanes by shuffles, the readout is a shuffle reduction over
// the row's lanes, and y returns to lane l for one coalesced store.
template <typename T, int N, bool CONV>
__global__ void __launch_bounds__(256)
step_kernel(int64_t d, const T* __restrict__ h, const T* __restrict__ a,
            const T* __restrict__ b, const T* __restrict__ B, const T* __restrict__ C,
            const T* __restrict__ z, const float* __restrict__ D, float* __restrict__ state,
            T* __restrict__ y, float scale, const float* __restrict__ conv_w,
            const float* __restrict__ conv_b, float* __restrict__ conv_state) {
    constexpr int Q = N / 4;        // lanes per state row
    constexpr int CPI = 32 / Q;     // rows per warp instruction
    constexpr int ITER = 32 / CPI;  // instructions per 32 rows (= Q)
    constexpr int BATCH = ITER < 8 ? ITER : 8;  // loads in flight per lane
    const int64_t bb = blockIdx.y;
    const int lane = threadIdx.x & 31;
    const int64_t cw0 = ((int64_t)blockIdx.x * 8 + (threadIdx.x >> 5)) * 32;  // warp's first channel
    if (cw0 >= d) return;
    // ---- gates of channel cw0 + lane
    const int64_t cg = cw0 + lane;
    const bool gvalid = cg < d;
    const int64_t eg = bb * d + cg;
    float f = 0.f, v = 0.f, dh = 0.f, gz = 1.f;
    if (gvalid) {
        float hh = to_f(h[eg]);
        if (CONV) {
            const float s0 = conv_state[eg * 3], s1 = conv_state[eg * 3 + 1],
                        s2 = conv_state[eg * 3 + 2];
            const float p = (conv_b ? conv_b[cg] : 0.f) + conv_w[cg * 4] * s0 +
                            conv_w[cg * 4 + 1] * s1 + conv_w[cg * 4 + 2] * s2 +
                            conv_w[cg * 4 + 3] * hh;
            conv_state[eg * 3] = s1;
            conv_state[eg * 3 + 1] = s2;
            conv_state[eg * 3 + 2] = hh;
            hh = siluf_(p);
        }
        const float ea = __expf(-to_f(a[eg]));
        f = rcpf_(1.f + ea);
        // b absent: coupled single gate i = 1 - f
        v = (b ? sigmoidf_(to_f(b[eg])) : ea * f) * hh;
        dh = D ? D[cg] * hh : 0.f;
        if (z) gz = siluf_(to_f(z[eg]));
    }
    // ---- B, C slice of this lane's float4 position
    const int q = lane % Q, grp = lane / Q;
    float4 Bv, Cv;
    {
        float t4[4], u4[4];
#pragma unroll
        for (int r = 0; r < 4; ++r) {
            t4[r] = to_f(B[bb * N + q * 4 + r]);
            u4[r] = to_f(C[bb * N + q * 4 + r]);
        }
        Bv = make_float4(t4[0], t4[1], t4[2], t4[3]);
        Cv = make_float4(u4[0], u4[1], u4[2], u4[3]);
    }
    // ---- stream the 32 rows
    float yl = 0.f;  // y of channel cw0 + lane, gathered below
#pragma unroll
    for (int r0 = 0; r0 < ITER; r0 += BATCH) {
        float4 x[BATCH];
#pragma unroll
        for (int k = 0; k < BATCH; ++k) {
            const int64_t c = cw0 + (int64_t)(r0 + k) * CPI + grp;
            x[k] = c < d ? reinterpret_cast<const float4*>(state + (bb * d + c) * N)[q]
                         : make_float4(0.f, 0.f, 0.f, 0.f);
        }
#pragma unroll
        for (int k = 0; k < BATCH; ++k) {
            const int r = r0 + k;
            const int src = r * CPI + grp;  // lane holding this row's gates
            const int64_t c = cw0 + src;
            const float fr = __shfl_sync(0xffffffffu, f, src);
            const float vr = __shfl_sync(0xffffffffu, v, src);
            float4 xk = x[k];
            xk.x = fmaf(fr, xk.x, vr * Bv.x);
            xk.y = fmaf(fr, xk.y, vr * Bv.y);
            xk.z = fmaf(fr, xk.z, vr * Bv.z);
            xk.w = fmaf(fr, xk.w, vr * Bv.w);
            if (c < d) reinterpret_cast<float4*>(state + (bb * d + c) * N)[q] = xk;
            float part = (xk.x * Cv.x + xk.y * Cv.y) + (xk.z * Cv.z + xk.w * Cv.w);
#pragma unroll
            for (int o = 1; o < Q; o <<= 1) part += __shfl_xor_sync(0xffffffffu, part, o);
            // lanes r*CPI .. r*CPI + CPI - 1 collect the sums of rows r*CPI + g
            const float got = __shfl_sync(0xffffffffu, part, (lane - r * CPI) * Q & 31);
            if (lane >= r * CPI && lane < r * CPI + CPI) yl = got;
        }
    }
    if (gvalid) y[eg] = from_f<T>(fmaf(yl, scale, dh) * gz);
}

template <typename T, bool CONV>
static cudaError_t step_t(int64_t Bt, int64_t d, int64_t N, const void* h, const void* a,
                          const void* b, const void* B, const void* C, const void* z,
                          const float* D, float* state, void* y, const float* conv_w,
                          const float* conv_b, float* conv_state, cudaStream_t st) {
    const float scale = 1.0f / sqrtf((float)N);
    dim3 grid((unsigned)((d + 255) / 256), (unsigned)Bt);  // 8 warps x 32 channels
#define NAJU_STEP(NN)                                                                     \
    step_kernel<T, NN, CONV><<<grid, 256, 0, st>>>(                                      \
        d, static_cast<const T*>(h), static_cast<const T*>(a), static_cast<const T*>(b), \
        static_cast<const T*>(B), static_cast<const T*>(C), static_cast<const T*>(z), D,  \
        state, static_cast<T*>(y), scale, conv_w, conv_b, conv_state)
    switch (N) {
        case 16: NAJU_STEP(16); break;
        case 32: NAJU_STEP(32); break;
        case 64: NAJU_STEP(64); break;
        case 128: NAJU_STEP(128); break;
        default: return cudaErrorInvalidValue;
    }
#undef NAJU_STEP
    return cudaGetLastError();
}

cudaError_t launch_scan_step(int64_t Bt, int64_t d, int64_t N, const void* h, const void* a,
                             const void* b, const void* B, const void* C, const void* z,
                             const float* D, float* state, void* y, int dtype,
                             const float* conv_w, const float* conv_b, float* conv_state,
                             cudaStream_t st) {
    const bool conv = conv_w != nullptr;
    if (dtype == NAJU_F32)
        return conv ? step_t<float, true>(Bt, d, N, h, a, b, B, C, z, D, state, y, conv_w,
                                          conv_b, conv_state, st)
                    : step_t<float, false>(Bt, d, N, h, a, b, B, C, z, D, state, y, nullptr,
                                           nullptr, nullptr, st);
    return conv ? step_t<__nv_bfloat16, true>(Bt, d, N, h, a, b, B, C, z, D, state, y, conv_w,
                                              conv_b, conv_state, st)
                : step_t<__nv_bfloat16, false>(Bt, d, N, h, a, b, B, C, z, D, state, y, nullptr,
                                               nullptr, nullptr, st);
}

// Standalone conv decode step: h = SiLU(bias + w . (s0, s1, s2, u)), state shift.
template <typename T>
__global__ void conv_step_kernel(int64_t n, int64_t d, const T* __restrict__ u,
                                 const float* __restrict__ w, const float* __restrict__ bias,
                                 float* __restrict__ cs, T* __restrict__ h) {
    for (int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; e < n;
         e += (int64_t)gridDim.x * blockDim.x) {
        const int64_t c = e % d;
        const float uv = to_f(u[e]);
        const float s0 = cs[e * 3], s1 = cs[e * 3 + 1], s2 = cs[e * 3 + 2];
        const float p = (bias ? bias[c] : 0.f) + w[c * 4] * s0 + w[c * 4 + 1] * s1 +
                        w[c * 4 + 2] * s2 + w[c * 4 + 3] * uv;
        h[e] = from_f<T>(siluf_(p));
        cs[e * 3] = s1;
        cs[e * 3 + 1] = s2;
        cs[e * 3 + 2] = uv;
    }
}

cudaError_t launch_conv_step(int64_t Bt, int64_t d, const void* u, const float* w,
                             const float* bias, float* conv_state, void* h, int dtype,
                             cudaStream_t st) {
    const int64_t n = Bt * d;
    const unsigned blocks = (unsigned)std::min<int64_t>((n + 255) / 256, 148 * 16);
    if (dtype == NAJU_F32)
        conv_step_kernel<float><<<blocks, 256, 0, st>>>(n, d, static_cast<const float*>(u), w,
                                                        bias, conv_state,
                                                        static_cast<float*>(h));
    else
        conv_step_kernel<__nv_bfloat16><<<blocks, 256, 0, st>>>(
            n, d, static_cast<const __nv_bfloat16*>(u), w, bias, conv_state,
            static_cast<__nv_bfloat16*>(h));
    return cudaGetLastError();
}

}  // namespace naju
