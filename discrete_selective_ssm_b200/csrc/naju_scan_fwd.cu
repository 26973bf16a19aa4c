// Naju forward scan on CUDA cores (sm_100a).
//
// Computes, per (batch, channel) row (Naju reproduction README, "Core
// equations"; flowchart nodes "causal depthwise conv + SiLU" and "SiLU output
// modulation"):
//   h_n = SiLU(conv(u)_n)                    (fused mode) or h_n given
//   x_n = f_n x_{n-1} + i_n h_n B_n^T,       f = sigmoid(a), i = sigmoid(b)
//   y_n = x_n . C_n / sqrt(N) + D h_n,       out_n = y_n SiLU(z_n)
//
// Work decomposition.  A thread block owns P channels of one batch element
// and one group of consecutive checkpoint segments.  Each channel's d_state
// row is split over S threads that keep NS state entries in registers.  The
// sequence is streamed in chunks of T tokens: the block first computes the
// per-(token, channel) scalars of the chunk into shared memory (conv, gates,
// feedthrough, modulation), then every thread advances its state slice token
// by token, and the chunk's outputs are written back coalesced.
//
// Rescaled state.  Each thread keeps xs = x * Q with Q = prod 1/f since the
// last renormalisation, so one token costs one FMA for the write
// (xs += (i h Q) B) and one FMA for the readout (y = (xs . C) / Q).  Q only
// grows (1/f = 1 + e^{-a} >= 1); when it would pass 2^64 in any lane of a
// warp, the warp folds Q back into its states.
//
// Sequence groups.  When batch x channel tiles alone do not fill the GPU,
// the sequence is split into G groups handled by different blocks.  A block
// of group g > 0 first runs its group with a zero initial state to get the
// group's local end state and decay product, then waits (bounded) for group
// g-1 to publish its end state, publishes its own, and finally runs the group
// again from the true initial state producing outputs (a decoupled
// look-back along the sequence).  Work items are taken from an atomic ticket
// in group order, so every awaited block has already started.
#include "naju_common.cuh"
#include "naju_kernels.h"

namespace naju {

constexpr float kRenorm = 18446744073709551616.0f;  // 2^64

template <typename Tin, typename Tout, int NS, int S, bool CONV>
__global__ void __launch_bounds__(128)
scan_fwd_kernel(const FwdParams p) {
    constexpr int NT = 128;
    constexpr int P = NT / S;        // channels per block
    constexpr int N = NS * S;        // d_state
    constexpr int T = kFwdChunk;     // tokens per chunk
    constexpr int R = T / S;         // tokens per prep run (NT / P = S runs)
    static_assert(NS % 4 == 0 && T % S == 0, "tile shape");

    extern __shared__ float4 smem4[];
    float* sm = reinterpret_cast<float*>(smem4);
    float* sB = sm;                  // [T][N]
    float* sC = sB + T * N;          // [T][N]
    float* sQ = sC + T * N;          // [T][P]  1/f
    float* sF = sQ + T * P;          // [T][P]  f
    float* sV = sF + T * P;          // [T][P]  i*h
    float* sHD = sV + T * P;         // [T][P]  D*h
    float* sG = sHD + T * P;         // [T][P]  SiLU(z) (or 1)
    float* sY = sG + T * P;          // [T][P]  x.C (unscaled readout)
    __shared__ int s_item;

    const int tid = threadIdx.x;
    const int js = tid % S;
    const int pl = tid / S;
    const int64_t Bt = p.Bt, L = p.L, d = p.d;

    if (tid == 0) s_item = atomicAdd(&p.hdr->fwd_ticket, 1);
    __syncthreads();
    const int item = s_item;
    const int per_g = (int)(Bt * p.ntiles);
    const int g = item / per_g;
    const int bb = (item % per_g) / p.ntiles;
    const int tile = item % p.ntiles;
    const int64_t c0 = (int64_t)tile * P;
    const int64_t c = c0 + pl;
    const bool cvalid = c < d;

    const int seg0 = g * p.seg_per_group;
    const int seg1 = min(seg0 + p.seg_per_group, p.nck);
    const int64_t tbeg = (int64_t)seg0 * p.T_ck;
    const int64_t tend = min64(L, (int64_t)seg1 * p.T_ck);
    const bool last_group = (g == p.ngroups - 1);

    const Tin* hu = static_cast<const Tin*>(p.hu);
    const Tin* ga = static_cast<const Tin*>(p.a);
    const Tin* gb = static_cast<const Tin*>(p.b);
    const Tin* gB = static_cast<const Tin*>(p.B);
    const Tin* gC = static_cast<const Tin*>(p.C);
    const Tin* gz = static_cast<const Tin*>(p.z);
    Tout* gy = static_cast<Tout*>(p.y);

    // Per-thread prep assignment: channel column pp, token run rr.
    const int pp = tid % P;
    const int rr = tid / P;
    const int64_t cp = c0 + pp;
    const bool cpvalid = cp < d;
    float w0 = 0.f, w1 = 0.f, w2 = 0.f, w3 = 0.f, wb = 0.f, Dc = 0.f;
    if (cpvalid) {
        if (CONV) {
            w0 = p.conv_w[cp * 4 + 0];
            w1 = p.conv_w[cp * 4 + 1];
            w2 = p.conv_w[cp * 4 + 2];
            w3 = p.conv_w[cp * 4 + 3];
            wb = p.conv_b ? p.conv_b[cp] : 0.f;
        }
        Dc = p.D ? p.D[cp] : 0.f;
    }

    float* ck_b = p.ckpt + (int64_t)bb * (p.nck + 1) * d * N;  // [nck+1][d][N]

    // ------------------------------------------------ chunk staging helpers
    auto prep_chunk = [&](int64_t t0, bool full) {
        // B, C rows of the chunk -> fp32 smem (zeros past L).
        for (int e = tid; e < T * N; e += NT) {
            const int tt = e / N;
            const int64_t t = t0 + tt;
            float vb = 0.f, vc = 0.f;
            if (t < tend) {
                vb = to_f(gB[((int64_t)bb * L + t) * N + (e % N)]);
                if (full) vc = to_f(gC[((int64_t)bb * L + t) * N + (e % N)]);
            }
            sB[e] = vb;
            sC[e] = vc;
        }
        // Per-(token, channel) scalars; run rr covers tokens [rr*R, rr*R+R).
        const int64_t tr = t0 + rr * R;
        float u0 = 0.f, u1 = 0.f, u2 = 0.f;  // u_{t-3}, u_{t-2}, u_{t-1}
        if (CONV && cpvalid) {
            const Tin* col = hu + (int64_t)bb * L * d + cp;
            if (tr - 3 >= 0 && tr - 3 < L) u0 = to_f(col[(tr - 3) * d]);
            if (tr - 2 >= 0 && tr - 2 < L) u1 = to_f(col[(tr - 2) * d]);
            if (tr - 1 >= 0 && tr - 1 < L) u2 = to_f(col[(tr - 1) * d]);
        }
#pragma unroll 4
        for (int k = 0; k < R; ++k) {
            const int tt = rr * R + k;
            const int64_t t = tr + k;
            float q = 1.f, f = 1.f, v = 0.f, hd = 0.f, gg = 1.f;
            if (cpvalid && t < tend) {
                const int64_t e = ((int64_t)bb * L + t) * d + cp;
                float h;
                if (CONV) {
                    const float u3 = to_f(hu[e]);
                    const float pre = wb + w0 * u0 + w1 * u1 + w2 * u2 + w3 * u3;
                    h = siluf_(pre);
                    u0 = u1; u1 = u2; u2 = u3;
                } else {
                    h = to_f(hu[e]);
                }
                const float ea = __expf(-to_f(ga[e]));
                q = 1.f + ea;
                f = 1.f / q;
                v = sigmoidf_(to_f(gb[e])) * h;
                if (full) {
                    hd = Dc * h;
                    if (gz) gg = siluf_(to_f(gz[e]));
                }
            }
            sQ[tt * P + pp] = q;
            sF[tt * P + pp] = f;
            sV[tt * P + pp] = v;
            if (full) {
                sHD[tt * P + pp] = hd;
                sG[tt * P + pp] = gg;
            }
        }
    };

    // ------------------------------------------------------- state in regs
    float xs[NS];
    float Q = 1.f, invQ = 1.f;      // x = xs * invQ; Q ~ 1/invQ
    float logPf = 0.f;              // log of prod f folded by renormalisation

    auto load_state = [&](const float* src, bool cg) {
#pragma unroll
        for (int m = 0; m < NS / 4; ++m) {
            float4 v4 = make_float4(0.f, 0.f, 0.f, 0.f);
            if (src && cvalid) {
                const float4* s4 = reinterpret_cast<const float4*>(src + c * N) + m * S + js;
                v4 = cg ? __ldcg(s4) : *s4;
            }
            xs[4 * m + 0] = v4.x; xs[4 * m + 1] = v4.y;
            xs[4 * m + 2] = v4.z; xs[4 * m + 3] = v4.w;
        }
        Q = 1.f; invQ = 1.f; logPf = 0.f;
    };
    auto store_state = [&](float* dst) {
        if (!cvalid) return;
#pragma unroll
        for (int m = 0; m < NS / 4; ++m) {
            float4 v4 = make_float4(xs[4 * m] * invQ, xs[4 * m + 1] * invQ,
                                    xs[4 * m + 2] * invQ, xs[4 * m + 3] * invQ);
            reinterpret_cast<float4*>(dst + c * N)[m * S + js] = v4;
        }
    };

    // One token of the recurrence for this thread's state slice.  Returns the
    // unscaled readout partial x.C when READ.
    auto step = [&](int tt, bool READ) -> float {
        const float q = sQ[tt * P + pl];
        const float f = sF[tt * P + pl];
        const float v = sV[tt * P + pl];
        float Qn = Q * q;
        float iQn = invQ * f;
        const bool need = !(Qn <= kRenorm);
        if (__any_sync(0xffffffffu, need)) {
            // Fold: xs <- x_{t-1} * f_t, i.e. xs * invQ * f.
            logPf += __logf(iQn);
#pragma unroll
            for (int j = 0; j < NS; ++j) xs[j] *= iQn;
            Qn = 1.f;
            iQn = 1.f;
        }
        Q = Qn;
        invQ = iQn;
        const float wv = v * Q;
        const float4* b4 = reinterpret_cast<const float4*>(sB + tt * N);
        const float4* c4 = reinterpret_cast<const float4*>(sC + tt * N);
        float a0 = 0.f, a1 = 0.f, a2 = 0.f, a3 = 0.f;
#pragma unroll
        for (int m = 0; m < NS / 4; ++m) {
            const float4 bv = b4[m * S + js];
            xs[4 * m + 0] = fmaf(wv, bv.x, xs[4 * m + 0]);
            xs[4 * m + 1] = fmaf(wv, bv.y, xs[4 * m + 1]);
            xs[4 * m + 2] = fmaf(wv, bv.z, xs[4 * m + 2]);
            xs[4 * m + 3] = fmaf(wv, bv.w, xs[4 * m + 3]);
            if (READ) {
                const float4 cv = c4[m * S + js];
                a0 = fmaf(xs[4 * m + 0], cv.x, a0);
                a1 = fmaf(xs[4 * m + 1], cv.y, a1);
                a2 = fmaf(xs[4 * m + 2], cv.z, a2);
                a3 = fmaf(xs[4 * m + 3], cv.w, a3);
            }
        }
        return (a0 + a1) + (a2 + a3);
    };

    // --------------------------------------------- local pass (groups > 0)
    const bool do_local = (g > 0) && !last_group;
    if (do_local) {
        load_state(nullptr, false);
        for (int64_t t0 = tbeg; t0 < tend; t0 += T) {
            prep_chunk(t0, false);
            __syncthreads();
            for (int tt = 0; tt < T; ++tt) step(tt, false);
            __syncthreads();
        }
    }
    // Local end state (zero start) and log prod f of the group.
    const float logPf_loc = logPf + __logf(invQ);

    // ----------------------------------------------- carry in / publish
    const int* flag_prev = (g > 0) ? p.flags + ((int64_t)(g - 1) * Bt + bb) * p.ntiles + tile
                                   : nullptr;
    int* flag_mine = p.flags + ((int64_t)g * Bt + bb) * p.ntiles + tile;
    float* ck_start = ck_b + (int64_t)seg0 * d * N;
    float* ck_end = ck_b + (int64_t)seg1 * d * N;
    __shared__ int s_ok;
    if (g > 0) {
        if (tid == 0) s_ok = wait_flag(flag_prev, &p.hdr->status, p.wait_limit) ? 1 : 0;
        __syncthreads();
        if (do_local) {
            // X_end = prod f * X_start + local state.
            const float Pf = __expf(logPf_loc);
#pragma unroll
            for (int m = 0; m < NS / 4; ++m) {
                float4 v4 = make_float4(0.f, 0.f, 0.f, 0.f);
                if (s_ok && cvalid)
                    v4 = __ldcg(reinterpret_cast<const float4*>(ck_start + c * N) + m * S + js);
                xs[4 * m + 0] = fmaf(Pf, v4.x, xs[4 * m + 0] * invQ);
                xs[4 * m + 1] = fmaf(Pf, v4.y, xs[4 * m + 1] * invQ);
                xs[4 * m + 2] = fmaf(Pf, v4.z, xs[4 * m + 2] * invQ);
                xs[4 * m + 3] = fmaf(Pf, v4.w, xs[4 * m + 3] * invQ);
            }
            invQ = 1.f;
            store_state(ck_end);
            __threadfence();
            __syncthreads();
            if (tid == 0) st_release(flag_mine, 1);
        }
        load_state(s_ok ? ck_start : nullptr, true);
    } else {
        load_state(p.x0 ? p.x0 + (int64_t)bb * d * N : nullptr, false);
        store_state(ck_b);  // checkpoint 0 = initial state
    }

    // ------------------------------------------------------- full pass
    const float scale = p.scale;
    for (int64_t t0 = tbeg; t0 < tend; t0 += T) {
        prep_chunk(t0, true);
        __syncthreads();
        for (int tt = 0; tt < T; ++tt) {
            float part = step(tt, true);
#pragma unroll
            for (int o = 1; o < S; o <<= 1) part += __shfl_xor_sync(0xffffffffu, part, o);
            if (js == 0) sY[tt * P + pl] = part * invQ;
        }
        // Interior checkpoints at segment boundaries inside this group.
        const int64_t tnext = t0 + T;
        if (tnext < tend && tnext % p.T_ck == 0) store_state(ck_b + (tnext / p.T_ck) * d * N);
        __syncthreads();
        // Epilogue: out = (scale * x.C + D h) * SiLU(z), coalesced over channels.
        if (cpvalid) {
            for (int k = 0; k < R; ++k) {
                const int tt = rr * R + k;
                const int64_t t = t0 + tt;
                if (t < tend) {
                    const float yv = fmaf(scale, sY[tt * P + pp], sHD[tt * P + pp]);
                    gy[((int64_t)bb * L + t) * d + cp] = from_f<Tout>(yv * sG[tt * P + pp]);
                }
            }
        }
        __syncthreads();
    }

    // -------------------------------------------------- group end state
    if (g == 0 && p.ngroups > 1) {
        store_state(ck_end);
        __threadfence();
        __syncthreads();
        if (tid == 0 && !p.fault_skip_publish) st_release(flag_mine, 1);
    }
    if (last_group) {
        store_state(ck_b + (int64_t)p.nck * d * N);
        if (p.x_final) store_state(p.x_final + (int64_t)bb * d * N);
    }
}

template <typename Tin, typename Tout, int NS, int S, bool CONV>
static cudaError_t launch_fwd_t(const FwdParams& p, cudaStream_t st) {
    constexpr int P = 128 / S;
    constexpr int N = NS * S;
    constexpr int T = kFwdChunk;
    const size_t smem = sizeof(float) * (2 * T * N + 6 * T * P);
    auto kern = scan_fwd_kernel<Tin, Tout, NS, S, CONV>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)smem);
    if (e != cudaSuccess) return e;
    const int grid = p.ngroups * (int)p.Bt * p.ntiles;
    kern<<<grid, 128, smem, st>>>(p);
    return cudaGetLastError();
}

template <typename Tin, typename Tout, bool CONV>
static cudaError_t launch_fwd_n(const FwdParams& p, cudaStream_t st) {
    switch (p.N) {
        case 16: return launch_fwd_t<Tin, Tout, 16, 1, CONV>(p, st);
        case 32: return launch_fwd_t<Tin, Tout, 32, 1, CONV>(p, st);
        case 64: return launch_fwd_t<Tin, Tout, 32, 2, CONV>(p, st);
        case 128: return launch_fwd_t<Tin, Tout, 32, 4, CONV>(p, st);
        default: return cudaErrorInvalidValue;
    }
}

int fwd_channels_per_block(int64_t N) {
    return N <= 32 ? 128 : (N == 64 ? 64 : 32);
}

cudaError_t launch_scan_fwd(const FwdParams& p, int dtype, int out_dtype, cudaStream_t st) {
    const bool conv = p.conv_w != nullptr;
    if (dtype == NAJU_F32) {
        return conv ? launch_fwd_n<float, float, true>(p, st)
                    : launch_fwd_n<float, float, false>(p, st);
    }
    if (out_dtype == NAJU_BF16) {
        return conv ? launch_fwd_n<__nv_bfloat16, __nv_bfloat16, true>(p, st)
                    : launch_fwd_n<__nv_bfloat16, __nv_bfloat16, false>(p, st);
    }
    return conv ? launch_fwd_n<__nv_bfloat16, float, true>(p, st)
                : launch_fwd_n<__nv_bfloat16, float, false>(p, st);
}

}  // namespace naju
