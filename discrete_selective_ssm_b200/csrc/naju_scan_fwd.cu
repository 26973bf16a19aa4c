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
// sequence is streamed in chunks of T tokens through a double-buffered
// shared-memory stage filled by cp.async (the next chunk's raw rows are in
// flight while the current chunk is scanned).  Per chunk the block first
// computes the per-(token, channel) scalars (conv, gates) into shared memory,
// then every thread advances its state slice token by token, and the
// chunk's outputs are written back coalesced.
//
// Rescaled state.  Each thread keeps xs = x * Q with Q = prod 1/f since the
// last renormalisation, so one token costs one FMA for the write
// (xs += (i h Q) B) and one FMA for the readout (y = (xs . C) / Q); both run
// as packed two-wide FP32 FMAs.  Q only grows (1/f = 1 + e^{-a} >= 1); when it
// would pass 2^64 in any lane of a warp, the warp folds Q back into its states.
//
// Sequence groups.  When batch x channel tiles alone do not fill the GPU,
// the sequence is split into G groups handled by different blocks.  Every
// group but the last first runs its tokens without readout: group 0 from x0,
// the others from a zero state, after which they wait (bounded) for group
// g-1's end state, fold it in with the group's decay product and publish
// their own end state.  All groups then run their full pass from the true
// initial state concurrently (a decoupled look-back along the sequence).
// Work items are taken from an atomic ticket in group order, so every
// awaited block has already started.
#include <type_traits>

#include "naju_common.cuh"
#include "naju_kernels.h"

namespace naju {

constexpr float kRenorm = 18446744073709551616.0f;  // 2^64

template <typename Tin, int P, int N>
struct FwdRaw {
    static constexpr int T = kFwdChunk;
    Tin u[T + 3][P];   // rows t0-3 .. t0+T-1 (conv input, or h in rows 3..)
    Tin a[T][P], b[T][P], z[T][P];
    Tin Bm[T][N], Cm[T][N];
};

template <typename Tin, int P, int N>
struct FwdSmem {
    static constexpr int T = kFwdChunk;
    FwdRaw<Tin, P, N> raw[2];
    float sB[T][N], sC[T][N];
    float sQ[T][P], sF[T][P], sV[T][P], sH[T][P], sY[T][P];
    int item, ok;
};

template <typename Tin, typename Tout, int NS, int S, bool CONV>
__global__ void __launch_bounds__(128, 4)
scan_fwd_kernel(const FwdParams p) {
    constexpr int NT = 128;
    constexpr int P = NT / S;        // channels per block
    constexpr int N = NS * S;        // d_state
    constexpr int T = kFwdChunk;     // tokens per chunk
    constexpr int R = T / S;         // tokens per prep run (NT / P = S runs)
    static_assert(NS % 4 == 0 && T % S == 0, "tile shape");
    using Sm = FwdSmem<Tin, P, N>;
    extern __shared__ float4 smem4[];
    Sm& sm = *reinterpret_cast<Sm*>(smem4);

    const int tid = threadIdx.x;
    const int js = tid % S;
    const int pl = tid / S;
    const int64_t Bt = p.Bt, L = p.L, d = p.d;

    if (tid == 0) sm.item = atomicAdd(&p.hdr->fwd_ticket, 1);
    __syncthreads();
    const int item = sm.item;
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

    const int64_t boff = (int64_t)bb * L;
    const Tin* hu = static_cast<const Tin*>(p.hu) + boff * d;
    const Tin* ga = static_cast<const Tin*>(p.a) + boff * d;
    // b absent: coupled single gate i = 1 - f.
    const Tin* gb = p.b ? static_cast<const Tin*>(p.b) + boff * d : nullptr;
    const Tin* gz = p.z ? static_cast<const Tin*>(p.z) + boff * d : nullptr;
    const Tin* gB = static_cast<const Tin*>(p.B) + boff * N;
    const Tin* gC = static_cast<const Tin*>(p.C) + boff * N;
    Tout* gy = static_cast<Tout*>(p.y) + boff * d;
    const bool vec = ((d * (int64_t)sizeof(Tin)) % 16) == 0;

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

    // [nck+1][d][N]; no checkpoints at all when p.ckpt is null (one group only)
    float* ck_b = p.ckpt ? p.ckpt + (int64_t)bb * (p.nck + 1) * d * N : nullptr;

    // ------------------------------------------------ chunk staging
    auto issue = [&](int64_t t0, int buf, bool full) {
        FwdRaw<Tin, P, N>& r = sm.raw[buf];
        stage_rows(&r.u[0][0], hu, d, t0 - 3, T + 3, L, c0, P, vec, tid, NT);
        stage_rows(&r.a[0][0], ga, d, t0, T, tend, c0, P, vec, tid, NT);
        if (gb) stage_rows(&r.b[0][0], gb, d, t0, T, tend, c0, P, vec, tid, NT);
        if (full && gz) stage_rows(&r.z[0][0], gz, d, t0, T, tend, c0, P, vec, tid, NT);
        stage_rows(&r.Bm[0][0], gB, N, t0, T, tend, 0, N, true, tid, NT);
        if (full) stage_rows(&r.Cm[0][0], gC, N, t0, T, tend, 0, N, true, tid, NT);
        cp_async_commit();
    };
    auto prep = [&](int64_t t0, int buf, bool full) {
        const FwdRaw<Tin, P, N>& r = sm.raw[buf];
        for (int e = tid; e < T * N; e += NT) {
            (&sm.sB[0][0])[e] = to_f((&r.Bm[0][0])[e]);
            if (full) (&sm.sC[0][0])[e] = to_f((&r.Cm[0][0])[e]);
        }
#pragma unroll
        for (int k = 0; k < R; ++k) {
            const int tt = rr * R + k;
            const int64_t t = t0 + tt;
            float q = 1.f, f = 1.f, v = 0.f, h = 0.f;
            if (cpvalid && t < tend) {
                if (CONV) {
                    const float pre = wb + w0 * to_f(r.u[tt][pp]) + w1 * to_f(r.u[tt + 1][pp]) +
                                      w2 * to_f(r.u[tt + 2][pp]) + w3 * to_f(r.u[tt + 3][pp]);
                    h = siluf_(pre);
                } else {
                    h = to_f(r.u[tt + 3][pp]);
                }
                const float ea = __expf(-to_f(r.a[tt][pp]));
                q = 1.f + ea;
                f = rcpf_(q);
                v = (gb ? sigmoidf_(to_f(r.b[tt][pp])) : ea * f) * h;
            }
            sm.sQ[tt][pp] = q;
            sm.sF[tt][pp] = f;
            sm.sV[tt][pp] = v;
            sm.sH[tt][pp] = h;
        }
    };

    // ------------------------------------------------------- state in regs
    float2 xs[NS / 2];
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
            xs[2 * m] = make_float2(v4.x, v4.y);
            xs[2 * m + 1] = make_float2(v4.z, v4.w);
        }
        Q = 1.f; invQ = 1.f; logPf = 0.f;
    };
    auto store_state = [&](float* dst) {
        if (!cvalid) return;
#pragma unroll
        for (int m = 0; m < NS / 4; ++m) {
            float4 v4 = make_float4(xs[2 * m].x * invQ, xs[2 * m].y * invQ,
                                    xs[2 * m + 1].x * invQ, xs[2 * m + 1].y * invQ);
            reinterpret_cast<float4*>(dst + c * N)[m * S + js] = v4;
        }
    };

    // One token of the recurrence for this thread's state slice.  Returns the
    // readout partial x.C (true scale) when READ.  CHECK tests Q against the
    // renormalisation bound (slow path only).
    auto step = [&](int tt, auto read, auto check) -> float {
        const float q = sm.sQ[tt][pl];
        const float f = sm.sF[tt][pl];
        const float v = sm.sV[tt][pl];
        float Qn = Q * q;
        float iQn = invQ * f;
        if constexpr (decltype(check)::value) {
            if (__any_sync(0xffffffffu, !(Qn <= kRenorm))) {
                // Fold: xs <- x_{t-1} * f_t, i.e. xs * invQ * f.
                logPf += __logf(iQn);
                const float2 s2 = make_float2(iQn, iQn);
#pragma unroll
                for (int j = 0; j < NS / 2; ++j) xs[j] = __fmul2_rn(xs[j], s2);
                Qn = 1.f;
                iQn = 1.f;
            }
        }
        Q = Qn;
        invQ = iQn;
        const float wv = v * Q;
        const float2 w2v = make_float2(wv, wv);
        const float4* b4 = reinterpret_cast<const float4*>(sm.sB[tt]);
        const float4* c4 = reinterpret_cast<const float4*>(sm.sC[tt]);
        float2 a[4] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f),
                       make_float2(0.f, 0.f)};
#pragma unroll
        for (int m = 0; m < NS / 4; ++m) {
            const float4 bv = b4[m * S + js];
            xs[2 * m] = __ffma2_rn(w2v, make_float2(bv.x, bv.y), xs[2 * m]);
            xs[2 * m + 1] = __ffma2_rn(w2v, make_float2(bv.z, bv.w), xs[2 * m + 1]);
            if constexpr (decltype(read)::value) {
                const float4 cv = c4[m * S + js];
                a[(2 * m) & 3] = __ffma2_rn(xs[2 * m], make_float2(cv.x, cv.y), a[(2 * m) & 3]);
                a[(2 * m + 1) & 3] =
                    __ffma2_rn(xs[2 * m + 1], make_float2(cv.z, cv.w), a[(2 * m + 1) & 3]);
            }
        }
        const float2 a01 = __fadd2_rn(a[0], a[1]), a23 = __fadd2_rn(a[2], a[3]);
        return ((a01.x + a01.y) + (a23.x + a23.y)) * invQ;
    };
    using Yes = std::integral_constant<bool, true>;
    using No = std::integral_constant<bool, false>;
    // Whether the chunk's T tokens can run without renormalisation checks
    // (Q times the chunk's product of 1/f stays below the bound in every lane
    // of the warp); otherwise fold Q into the state first and test again.
    auto fast_chunk = [&]() -> bool {
        float pq = 1.f;
#pragma unroll
        for (int tt = 0; tt < T; ++tt) pq *= sm.sQ[tt][pl];
        if (!__any_sync(0xffffffffu, !(Q * pq <= kRenorm))) return true;
        logPf += __logf(invQ);
        const float2 s2 = make_float2(invQ, invQ);
#pragma unroll
        for (int j = 0; j < NS / 2; ++j) xs[j] = __fmul2_rn(xs[j], s2);
        Q = 1.f;
        invQ = 1.f;
        return !__any_sync(0xffffffffu, !(pq <= kRenorm));
    };

    // One pass over the group's chunks: FULL = readout, outputs, checkpoints.
    auto run_pass = [&](bool full) {
        const int nch = (int)((tend - tbeg + T - 1) / T);
        issue(tbeg, 0, full);
        const float scale = p.scale;
        for (int k = 0; k < nch; ++k) {
            const int buf = k & 1;
            const int64_t t0 = tbeg + (int64_t)k * T;
            if (k + 1 < nch) {
                issue(t0 + T, buf ^ 1, full);
                cp_async_wait<1>();
            } else {
                cp_async_wait<0>();
            }
            __syncthreads();
            prep(t0, buf, full);
            __syncthreads();
            const bool fast = fast_chunk();
            if (full) {
                auto tok = [&](int tt, auto check) {
                    float part = step(tt, Yes{}, check);
#pragma unroll
                    for (int o = 1; o < S; o <<= 1) part += __shfl_xor_sync(0xffffffffu, part, o);
                    if (js == 0) sm.sY[tt][pl] = part;
                };
                if (fast) {
#pragma unroll 2
                    for (int tt = 0; tt < T; ++tt) tok(tt, No{});
                } else {
                    for (int tt = 0; tt < T; ++tt) tok(tt, Yes{});
                }
                const int64_t tnext = t0 + T;
                if (ck_b && tnext < tend && tnext % p.T_ck == 0)
                    store_state(ck_b + (tnext / p.T_ck) * d * N);
            } else if (fast) {
#pragma unroll 2
                for (int tt = 0; tt < T; ++tt) step(tt, No{}, No{});
            } else {
                for (int tt = 0; tt < T; ++tt) step(tt, No{}, Yes{});
            }
            __syncthreads();
            if (full && cpvalid) {
                const FwdRaw<Tin, P, N>& r = sm.raw[buf];
#pragma unroll
                for (int kk = 0; kk < R; ++kk) {
                    const int tt = rr * R + kk;
                    const int64_t t = t0 + tt;
                    if (t < tend) {
                        float yv = fmaf(scale, sm.sY[tt][pp], Dc * sm.sH[tt][pp]);
                        if (gz) yv *= siluf_(to_f(r.z[tt][pp]));
                        gy[t * d + cp] = from_f<Tout>(yv);
                    }
                }
            }
            __syncthreads();
        }
    };

    // ------------------------------------------ early pass and carry chain
    // Every group with a successor first runs its tokens without readout to
    // get its end state and publishes it, so that all full passes can run
    // concurrently: group 0 starts from x0, later groups from a zero state
    // and fold in the predecessor's end state once it is published.
    const float* x0b = p.x0 ? p.x0 + (int64_t)bb * d * N : nullptr;
    const int* flag_prev = (g > 0) ? p.flags + ((int64_t)(g - 1) * Bt + bb) * p.ntiles + tile
                                   : nullptr;
    int* flag_mine = p.flags + ((int64_t)g * Bt + bb) * p.ntiles + tile;
    float* ck_start = ck_b + (int64_t)seg0 * d * N;
    float* ck_end = ck_b + (int64_t)seg1 * d * N;
    bool ok = true;
    if (!last_group) {
        load_state(g == 0 ? x0b : nullptr, false);
        run_pass(false);
        if (g > 0) {
            const float Pf = __expf(logPf + __logf(invQ));  // prod f over the group
            if (tid == 0) sm.ok = wait_flag(flag_prev, &p.hdr->status, p.wait_limit) ? 1 : 0;
            __syncthreads();
            ok = sm.ok != 0;
#pragma unroll
            for (int m = 0; m < NS / 4; ++m) {
                float4 v4 = make_float4(0.f, 0.f, 0.f, 0.f);
                if (ok && cvalid)
                    v4 = __ldcg(reinterpret_cast<const float4*>(ck_start + c * N) + m * S + js);
                xs[2 * m].x = fmaf(Pf, v4.x, xs[2 * m].x * invQ);
                xs[2 * m].y = fmaf(Pf, v4.y, xs[2 * m].y * invQ);
                xs[2 * m + 1].x = fmaf(Pf, v4.z, xs[2 * m + 1].x * invQ);
                xs[2 * m + 1].y = fmaf(Pf, v4.w, xs[2 * m + 1].y * invQ);
            }
            invQ = 1.f;
        }
        store_state(ck_end);
        __threadfence();
        __syncthreads();
        if (tid == 0 && !(g == 0 && p.fault_skip_publish)) st_release(flag_mine, 1);
    } else if (g > 0) {
        if (tid == 0) sm.ok = wait_flag(flag_prev, &p.hdr->status, p.wait_limit) ? 1 : 0;
        __syncthreads();
        ok = sm.ok != 0;
    }
    if (g > 0) {
        load_state(ok ? ck_start : nullptr, true);
    } else {
        load_state(x0b, false);
        if (ck_b) store_state(ck_b);  // checkpoint 0 = initial state
    }

    // ------------------------------------------------------- full pass
    run_pass(true);
    if (last_group) {
        if (ck_b) store_state(ck_b + (int64_t)p.nck * d * N);
        if (p.x_final) store_state(p.x_final + (int64_t)bb * d * N);
    }
}

template <typename Tin, typename Tout, int NS, int S, bool CONV>
static cudaError_t launch_fwd_t(const FwdParams& p, cudaStream_t st) {
    constexpr int P = 128 / S;
    constexpr int N = NS * S;
    const size_t smem = sizeof(FwdSmem<Tin, P, N>);
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
        case 32: return launch_fwd_t<Tin, Tout, 16, 2, CONV>(p, st);
        case 64: return launch_fwd_t<Tin, Tout, 32, 2, CONV>(p, st);
        case 128: return launch_fwd_t<Tin, Tout, 32, 4, CONV>(p, st);
        default: return cudaErrorInvalidValue;
    }
}

int fwd_channels_per_block(int64_t N) {
    return N == 16 ? 128 : (N <= 64 ? 64 : 32);
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
