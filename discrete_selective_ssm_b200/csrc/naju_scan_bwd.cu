// Naju backward scan on CUDA cores (sm_100a).
//
// Reverse-mode gradient of the forward in naju_scan_fwd.cu, derived by hand
// from the recurrence of the Naju reproduction README ("Core equations").
// For one (batch, channel) row, with G_t = dLoss/dx_t and s = 1/sqrt(N):
//   dy_t   = dout_t SiLU(z_t),   dz_t = dout_t y_t SiLU'(z_t)
//   G_t    = s dy_t C_t + f_{t+1} G_{t+1}          (the last G also gets dx_final)
//   GB_t   = G_t . B_t
//   dh_t   = D dy_t + i_t GB_t,  db_t = h_t GB_t i_t (1 - i_t)
//   da_t   = (f_t df_t)(1 - f_t) with
//   f_t df_t = G_t . (f_t x_{t-1}) = sum_{t' >= t} dL_{t'} + dx_final . x_L,
//   dL_t   = s dy_t (x_t . C_t) - i_t h_t GB_t
//   dB_t   = sum_d G_t[d] i_t[d] h_t[d],   dC_t = s sum_d dy_t[d] x_t[d]
//   dD     = sum dy h,   dx0 = f_0 G_0,    conv: dp = dh SiLU'(p), du, dw, dbias.
//
// Work decomposition.  A thread block owns P channels of one batch element
// and one sequence group of consecutive 64-token blocks; the blocks of a
// cluster (consecutive channel tiles) share batch element and group.  The
// group's blocks are walked from the last to the first with the adjoint
// carry in registers.  For each block:
//  * the forward checkpoint at the block start gives its initial state;
//  * a forward sweep over 16-token sub-blocks recomputes the readout
//    (kept for dz and dL) and forms dC as a contraction over the block's
//    channels: dC_t = s[(dy E)_t X_b + sum_{m<=t} A[t,m] B_m], with X_b the
//    state entering the sub-block, E_t the decay since then and
//    A[t,m] = sum_d dy_t E_t/E_m i_m h_m;
//  * a backward sweep runs the adjoint, writes the per-channel gradients and
//    forms dB_m = s sum_{t>=m} A[t,m] C_t + (i h F)_m H_e, with H_e the
//    carry entering the sub-block's end and F_m the decay to that end.
// The dB/dC partial sums over each block's channels are summed across the
// cluster through distributed shared memory and written once per cluster.
//
// Sequence groups.  When batch x channel tiles alone do not fill the GPU,
// the sequence is split into groups.  The carry entering a group's end comes
// from the next group: every group with a predecessor first runs a cheap
// reverse pass (adjoint only) - from dx_final for the last group, from a zero
// carry for the others, which then wait (bounded) for the carry of the next
// group - and publishes the carry leaving its start before its main work
// (a decoupled look-back running backwards in time).  Groups are taken from
// an atomic ticket starting with the last, so every awaited block has started.
// Small kernels then sum the cluster partials, the per-channel partials
// (dD, dconv) and the conv's group-boundary terms.
#include <cooperative_groups.h>

#include <type_traits>

#include "naju_common.cuh"
#include "naju_kernels.h"

namespace cg = cooperative_groups;

namespace naju {

constexpr float kRenormB = 18446744073709551616.0f;  // 2^64
constexpr float kLogFloor = -10.0f;  // per-token log f floor inside the pivot factors of A
constexpr int kCluster = 8;

template <int N> struct BwdShape;
template <> struct BwdShape<16> { static constexpr int NS = 16, S = 1; };
template <> struct BwdShape<32> { static constexpr int NS = 32, S = 1; };
template <> struct BwdShape<64> { static constexpr int NS = 32, S = 2; };
template <> struct BwdShape<128> { static constexpr int NS = 32, S = 4; };

int bwd_channels_per_block(int64_t N) { return N <= 32 ? 128 : (N == 64 ? 64 : 32); }
// Cluster of channel tiles sharing one dB/dC partial set: 2 when the tiles
// fit (no padding blocks for narrow d_inner), else 8.
int bwd_cluster_size(int tiles) { return tiles <= 2 ? 2 : kCluster; }

template <typename Tin, int N, int P>
struct BwdSmem {
    static constexpr int T = kBwdChunk;   // 16
    static constexpr int K = kBwdSub;     // 64
    // raw rows of the current sub-block (cp.async destination)
    Tin u[T + 3][P], a[T][P], b[T][P], z[T][P], dout[T][P];
    Tin Bm[T][N], Cm[T][N];
    // unpacked per-(token, channel) values
    float f[T][P], q[T][P], v[T][P], dy[T][P];
    float x1[T][P];       // forward: clamped log-prefix   backward: G . B
    float x2[T][P + 1];   // forward: dy * decay prefix    backward: i h * decay to end
    float x3[T][P + 1];   // forward: A factor (dy side)   backward: f df
    float x4[T][P + 1];   // forward: A factor (i h side)
    float dp[T + 3][P];
    float ys[K][P];       // unscaled readout x_t . C_t of the block
    float Bf[T][N], Cf[T][N];
    float snap[P][N];     // X_b (forward) or H_e (backward)
    float A[K / T][T][T];
    float acc[K][N];      // dC (forward sweep) then dB (backward sweep) partials
    int item, ok;
};

template <typename Tin, typename Tout, int N, bool CONV, int CL>
__global__ void __launch_bounds__(128, 2)
scan_bwd_kernel(const BwdParams p) {
    constexpr int NS = BwdShape<N>::NS, S = BwdShape<N>::S;
    constexpr int NT = 128, P = NT / S;
    constexpr int T = kBwdChunk, K = kBwdSub, NSUB = K / T;
    constexpr int R = T / S;              // prep run length per thread
    using Sm = BwdSmem<Tin, N, P>;
    extern __shared__ float4 smem4[];
    Sm& sm = *reinterpret_cast<Sm*>(smem4);
    cg::cluster_group cluster = cg::this_cluster();
    const int crank = (int)cluster.block_rank();

    const int tid = threadIdx.x;
    const int js = tid % S, pl = tid / S;
    const int pp = tid % P, rr = tid / P;
    const int64_t Bt = p.Bt, L = p.L, d = p.d;
    const float s = p.scale;

    // ---------------------------------------------------- work item
    if (crank == 0 && tid == 0) sm.item = atomicAdd(&p.hdr->bwd_ticket, 1);
    cluster.sync();
    const int item = *cluster.map_shared_rank(&sm.item, 0);
    const int per_g = (int)(Bt * p.nclus);
    const int g = p.ngroups - 1 - item / per_g;
    const int bb = (item % per_g) / p.nclus;
    const int cgi = item % p.nclus;
    const int tile = cgi * CL + crank;
    const int64_t c0 = (int64_t)tile * P;
    const int64_t c = c0 + pl;
    const bool cvalid = c < d;
    const int64_t cp = c0 + pp;
    const bool cpvalid = cp < d;
    const int kb0 = g * p.blk_per_group;
    const int kb1 = min(kb0 + p.blk_per_group, p.nsub);
    const int64_t tg0 = (int64_t)kb0 * K;
    const int64_t tg1 = min64(L, (int64_t)kb1 * K);
    const bool lastg = (g == p.ngroups - 1);
    const bool firstg = (g == 0);

    const int64_t boff = (int64_t)bb * L;
    const Tin* hu = static_cast<const Tin*>(p.hu) + boff * d;
    const Tin* ga = static_cast<const Tin*>(p.a) + boff * d;
    // b absent: coupled single gate i = 1 - f (a also reaches i; no db).
    const Tin* gbp = p.b ? static_cast<const Tin*>(p.b) + boff * d : nullptr;
    const Tin* gz = p.z ? static_cast<const Tin*>(p.z) + boff * d : nullptr;
    const Tin* gdy = static_cast<const Tin*>(p.dy) + boff * d;
    const Tin* gB = static_cast<const Tin*>(p.B) + boff * N;
    const Tin* gC = static_cast<const Tin*>(p.C) + boff * N;
    const bool vec = ((d * (int64_t)sizeof(Tin)) % 16) == 0;

    float w0 = 0.f, w1 = 0.f, w2 = 0.f, w3 = 0.f, wb = 0.f, Dc = 0.f;
    if (cpvalid) {
        if (CONV) {
            w0 = p.conv_w[cp * 4]; w1 = p.conv_w[cp * 4 + 1];
            w2 = p.conv_w[cp * 4 + 2]; w3 = p.conv_w[cp * 4 + 3];
            wb = p.conv_b ? p.conv_b[cp] : 0.f;
        }
        Dc = p.D ? p.D[cp] : 0.f;
    }

    // Stage the raw rows of sub-block [t0, t0+T) (tokens >= tlim are zero).
    auto issue = [&](int64_t t0, int64_t tlim) {
        stage_rows(&sm.u[0][0], hu, d, t0 - 3, T + 3, L, c0, P, vec, tid, NT);
        stage_rows(&sm.a[0][0], ga, d, t0, T, tlim, c0, P, vec, tid, NT);
        if (gbp) stage_rows(&sm.b[0][0], gbp, d, t0, T, tlim, c0, P, vec, tid, NT);
        if (gz) stage_rows(&sm.z[0][0], gz, d, t0, T, tlim, c0, P, vec, tid, NT);
        stage_rows(&sm.dout[0][0], gdy, d, t0, T, tlim, c0, P, vec, tid, NT);
        stage_rows(&sm.Bm[0][0], gB, N, t0, T, tlim, 0, N, true, tid, NT);
        stage_rows(&sm.Cm[0][0], gC, N, t0, T, tlim, 0, N, true, tid, NT);
        cp_async_commit();
    };
    // Unpack the staged rows into fp32 per-(token, channel) values.
    auto prep = [&](int64_t t0, int64_t tlim) {
        for (int e = tid; e < T * N; e += NT) {
            (&sm.Bf[0][0])[e] = to_f((&sm.Bm[0][0])[e]);
            (&sm.Cf[0][0])[e] = to_f((&sm.Cm[0][0])[e]);
        }
#pragma unroll
        for (int kk = 0; kk < R; ++kk) {
            const int tt = rr * R + kk;
            const int64_t t = t0 + tt;
            float f = 1.f, q = 1.f, v = 0.f, dyv = 0.f;
            if (cpvalid && t < tlim) {
                float h;
                if (CONV) {
                    h = siluf_(wb + w0 * to_f(sm.u[tt][pp]) + w1 * to_f(sm.u[tt + 1][pp]) +
                               w2 * to_f(sm.u[tt + 2][pp]) + w3 * to_f(sm.u[tt + 3][pp]));
                } else {
                    h = to_f(sm.u[tt + 3][pp]);
                }
                const float ea = __expf(-to_f(sm.a[tt][pp]));
                q = 1.f + ea;
                f = rcpf_(q);
                v = (gbp ? sigmoidf_(to_f(sm.b[tt][pp])) : ea * f) * h;
                dyv = to_f(sm.dout[tt][pp]);
                if (gz) dyv *= siluf_(to_f(sm.z[tt][pp]));
            }
            sm.f[tt][pp] = f; sm.q[tt][pp] = q; sm.v[tt][pp] = v; sm.dy[tt][pp] = dyv;
        }
    };
    // Sub-block sequence of a pass: sub-block i starts at first + dir * i * T.
    // The raw buffer is refilled with sub-block i+1 right after sub-block i
    // is unpacked unless `late` (the body reads raw rows), in which case the
    // refill follows the body.
    auto pass = [&](int64_t first, int count, int dir, int64_t tlim, bool late, auto&& body) {
        if (count <= 0) return;
        issue(first, tlim);
        for (int i = 0; i < count; ++i) {
            const int64_t t0 = first + (int64_t)dir * i * T;
            cp_async_wait<0>();
            __syncthreads();
            prep(t0, tlim);
            __syncthreads();
            if (!late && i + 1 < count) issue(t0 + dir * T, tlim);
            body(i, t0);
            __syncthreads();
            if (late && i + 1 < count) issue(t0 + dir * T, tlim);
        }
    };

    // ----------------------------------------------------- register state
    float2 xs[NS / 2], gs[NS / 2];
    float Q = 1.f, iQ = 1.f;   // forward: x = xs * iQ
    float Rr = 1.f, iR = 1.f;  // backward: G = gs * iR
    float logF = 0.f;          // log of decay folded out of the backward state

    auto load_rows = [&](float2* dst, const float* src, bool cg_) {
#pragma unroll
        for (int m = 0; m < NS / 4; ++m) {
            float4 v4 = make_float4(0.f, 0.f, 0.f, 0.f);
            if (src && cvalid) {
                const float4* s4 = reinterpret_cast<const float4*>(src + c * N) + m * S + js;
                v4 = cg_ ? __ldcg(s4) : *s4;
            }
            dst[2 * m] = make_float2(v4.x, v4.y);
            dst[2 * m + 1] = make_float2(v4.z, v4.w);
        }
    };
    auto store_rows = [&](float* dst, const float2* src, float sc) {
        if (!cvalid) return;
#pragma unroll
        for (int m = 0; m < NS / 4; ++m)
            reinterpret_cast<float4*>(dst + c * N)[m * S + js] =
                make_float4(src[2 * m].x * sc, src[2 * m].y * sc, src[2 * m + 1].x * sc,
                            src[2 * m + 1].y * sc);
    };
    auto snap_rows = [&](const float2* src, float sc) {
        if (cvalid) {
#pragma unroll
            for (int m = 0; m < NS / 4; ++m)
                reinterpret_cast<float4*>(sm.snap[pl])[m * S + js] =
                    make_float4(src[2 * m].x * sc, src[2 * m].y * sc, src[2 * m + 1].x * sc,
                                src[2 * m + 1].y * sc);
        } else {
#pragma unroll
            for (int m = 0; m < NS / 4; ++m)
                reinterpret_cast<float4*>(sm.snap[pl])[m * S + js] = make_float4(0.f, 0.f, 0.f, 0.f);
        }
    };
    auto scale_rows = [&](float2* v, float sc) {
        const float2 s2 = make_float2(sc, sc);
#pragma unroll
        for (int j = 0; j < NS / 2; ++j) v[j] = __fmul2_rn(v[j], s2);
    };
    auto red = [&](float v) {
#pragma unroll
        for (int o = 1; o < S; o <<= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
        return v;
    };
    // Forward token: xs <- xs + (v Q) B (rescaled); returns the readout x.C.
    // CHECK: test Q against the renormalisation bound (slow path only).
    auto fstep = [&](int tt, auto check) -> float {
        const float qv = sm.q[tt][pl], fv = sm.f[tt][pl], vv = sm.v[tt][pl];
        float Qn = Q * qv, iQn = iQ * fv;
        if constexpr (decltype(check)::value) {
            if (__any_sync(0xffffffffu, !(Qn <= kRenormB))) {
                scale_rows(xs, iQn);
                Qn = 1.f; iQn = 1.f;
            }
        }
        Q = Qn; iQ = iQn;
        const float wv = vv * Q;
        const float2 w2v = make_float2(wv, wv);
        const float4* b4 = reinterpret_cast<const float4*>(sm.Bf[tt]);
        const float4* c4 = reinterpret_cast<const float4*>(sm.Cf[tt]);
        float2 a[4] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f),
                       make_float2(0.f, 0.f)};
#pragma unroll
        for (int m = 0; m < NS / 4; ++m) {
            const float4 bv = b4[m * S + js];
            const float4 cv = c4[m * S + js];
            xs[2 * m] = __ffma2_rn(w2v, make_float2(bv.x, bv.y), xs[2 * m]);
            xs[2 * m + 1] = __ffma2_rn(w2v, make_float2(bv.z, bv.w), xs[2 * m + 1]);
            a[(2 * m) & 3] = __ffma2_rn(xs[2 * m], make_float2(cv.x, cv.y), a[(2 * m) & 3]);
            a[(2 * m + 1) & 3] =
                __ffma2_rn(xs[2 * m + 1], make_float2(cv.z, cv.w), a[(2 * m + 1) & 3]);
        }
        const float2 a01 = __fadd2_rn(a[0], a[1]), a23 = __fadd2_rn(a[2], a[3]);
        return ((a01.x + a01.y) + (a23.x + a23.y)) * iQ;
    };
    // Backward token t (after the carry from t+1 is in gs): G_t = G + s dy C.
    auto bstep = [&](int tt, bool dotB) -> float {
        const float wv = s * sm.dy[tt][pl] * Rr;
        const float2 w2v = make_float2(wv, wv);
        const float4* b4 = reinterpret_cast<const float4*>(sm.Bf[tt]);
        const float4* c4 = reinterpret_cast<const float4*>(sm.Cf[tt]);
        float2 a[4] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f),
                       make_float2(0.f, 0.f)};
#pragma unroll
        for (int m = 0; m < NS / 4; ++m) {
            const float4 cv = c4[m * S + js];
            gs[2 * m] = __ffma2_rn(w2v, make_float2(cv.x, cv.y), gs[2 * m]);
            gs[2 * m + 1] = __ffma2_rn(w2v, make_float2(cv.z, cv.w), gs[2 * m + 1]);
            if (dotB) {
                const float4 bv = b4[m * S + js];
                a[(2 * m) & 3] = __ffma2_rn(gs[2 * m], make_float2(bv.x, bv.y), a[(2 * m) & 3]);
                a[(2 * m + 1) & 3] =
                    __ffma2_rn(gs[2 * m + 1], make_float2(bv.z, bv.w), a[(2 * m + 1) & 3]);
            }
        }
        const float2 a01 = __fadd2_rn(a[0], a[1]), a23 = __fadd2_rn(a[2], a[3]);
        return ((a01.x + a01.y) + (a23.x + a23.y)) * iR;
    };
    // Multiply the backward state by f_t (moving from t to t-1).
    auto bdecay = [&](int tt, auto check) {
        const float qv = sm.q[tt][pl], fv = sm.f[tt][pl];
        float Rn = Rr * qv, iRn = iR * fv;
        if constexpr (decltype(check)::value) {
            if (__any_sync(0xffffffffu, !(Rn <= kRenormB))) {
                logF += __logf(iRn);
                scale_rows(gs, iRn);
                Rn = 1.f; iRn = 1.f;
            }
        }
        Rr = Rn; iR = iRn;
    };
    // Whether the next T tokens can run without renormalisation checks: the
    // scale (Q forward, R backward) times the sub-block's product of 1/f stays
    // below the bound in every lane of the warp.  If not, fold the scale into
    // the state first and test again; if it still fails (a sub-block whose own
    // decay exceeds 2^64), the caller takes the checked path.
    auto fast_fwd = [&]() -> bool {
        float pq = 1.f;
#pragma unroll
        for (int tt = 0; tt < T; ++tt) pq *= sm.q[tt][pl];
        if (!__any_sync(0xffffffffu, !(Q * pq <= kRenormB))) return true;
        scale_rows(xs, iQ);
        Q = 1.f; iQ = 1.f;
        return !__any_sync(0xffffffffu, !(pq <= kRenormB));
    };
    auto fast_bwd = [&]() -> bool {
        float pq = 1.f;
#pragma unroll
        for (int tt = 0; tt < T; ++tt) pq *= sm.q[tt][pl];
        if (!__any_sync(0xffffffffu, !(Rr * pq <= kRenormB))) return true;
        logF += __logf(iR);
        scale_rows(gs, iR);
        Rr = 1.f; iR = 1.f;
        return !__any_sync(0xffffffffu, !(pq <= kRenormB));
    };
    using Checked = std::integral_constant<bool, true>;
    using Unchecked = std::integral_constant<bool, false>;
    // Cluster sum of acc[K][N] into the dB (slot 0) or dC (slot 1) partials.
    auto cluster_reduce = [&](int slot, int64_t tb, int64_t te) {
        cluster.sync();
        constexpr int ROWS = K / CL;
        const int r0 = crank * ROWS;
        float* out = p.dBCp + (((int64_t)cgi * Bt + bb) * L) * 2 * N + slot * N;
        for (int e = tid; e < ROWS * N; e += NT) {
            const int tt = r0 + e / N;
            const int j = e % N;
            float a = 0.f;
#pragma unroll
            for (int qr = 0; qr < CL; ++qr)
                a += cluster.map_shared_rank(&sm.acc[0][0], qr)[tt * N + j];
            const int64_t t = tb + tt;
            if (t < te) out[t * 2 * N + j] = a;
        }
        cluster.sync();
    };

    // ------------------------------------ carry entering the group's end
    float2 H[NS / 2];
    float* carry_in = p.carry + ((int64_t)g * Bt + bb) * d * N;
    float* carry_out = g > 0 ? p.carry + ((int64_t)(g - 1) * Bt + bb) * d * N : nullptr;
    int* flag_in = p.flags + ((int64_t)g * Bt + bb) * p.ntiles + tile;
    int* flag_out = g > 0 ? p.flags + ((int64_t)(g - 1) * Bt + bb) * p.ntiles + tile : nullptr;
    if (lastg) load_rows(H, p.dx_final ? p.dx_final + (int64_t)bb * d * N : nullptr, false);
    if (!firstg) {
        // Early reverse pass over the group: adjoint only, to publish the carry
        // leaving the group's start before the main work.
        if (lastg) {
#pragma unroll
            for (int j = 0; j < NS / 2; ++j) gs[j] = H[j];
        } else {
#pragma unroll
            for (int j = 0; j < NS / 2; ++j) gs[j] = make_float2(0.f, 0.f);
        }
        Rr = 1.f; iR = 1.f; logF = 0.f;
        const int nsb = (int)((tg1 - tg0 + T - 1) / T);
        pass(tg0 + (int64_t)(nsb - 1) * T, nsb, -1, tg1, false, [&](int, int64_t) {
            if (fast_bwd()) {
#pragma unroll 2
                for (int tt = T - 1; tt >= 0; --tt) {
                    bstep(tt, false);
                    bdecay(tt, Unchecked{});
                }
            } else {
                for (int tt = T - 1; tt >= 0; --tt) {
                    bstep(tt, false);
                    bdecay(tt, Checked{});
                }
            }
        });
        if (!lastg) {
            if (tid == 0) sm.ok = wait_flag(flag_in, &p.hdr->status, p.wait_limit) ? 1 : 0;
            __syncthreads();
            load_rows(H, sm.ok ? carry_in : nullptr, true);
            // carry out = decay(group) * H + local contribution
            const float Pf = __expf(logF + __logf(iR));
            const float2 P2 = make_float2(Pf, Pf);
            const float2 r2 = make_float2(iR, iR);
#pragma unroll
            for (int j = 0; j < NS / 2; ++j) gs[j] = __ffma2_rn(P2, H[j], __fmul2_rn(gs[j], r2));
            iR = 1.f;
        }
        store_rows(carry_out, gs, iR);
        __threadfence();
        __syncthreads();
        if (tid == 0 && !(lastg && p.fault_skip_publish)) st_release(flag_out, 1);
    } else if (!lastg) {
        if (tid == 0) sm.ok = wait_flag(flag_in, &p.hdr->status, p.wait_limit) ? 1 : 0;
        __syncthreads();
        load_rows(H, sm.ok ? carry_in : nullptr, true);
    }

    // ------------------------------------------------ main: blocks in reverse
#pragma unroll
    for (int j = 0; j < NS / 2; ++j) gs[j] = H[j];
    Rr = 1.f; iR = 1.f; logF = 0.f;
    float dD_acc = 0.f, dw0 = 0.f, dw1 = 0.f, dw2 = 0.f, dw3 = 0.f, dbias = 0.f;
    Tout* gdhu = static_cast<Tout*>(p.dhu) + boff * d;
    Tout* gda = static_cast<Tout*>(p.da) + boff * d;
    Tout* gdb = p.db ? static_cast<Tout*>(p.db) + boff * d : nullptr;
    Tout* gdz = p.dz ? static_cast<Tout*>(p.dz) + boff * d : nullptr;
    float* edge = p.conv_edge + ((int64_t)bb * p.ngroups + g) * 2 * 3 * d;
    if (tid < P) {  // dp beyond the group: zero (the next group's terms go via the edge fixup)
        sm.dp[T][tid] = 0.f; sm.dp[T + 1][tid] = 0.f; sm.dp[T + 2][tid] = 0.f;
    }
    for (int k = kb1 - 1; k >= kb0; --k) {
        const int64_t tb = (int64_t)k * K;
        const int64_t te = min64(L, tb + K);
        // carry entering this block's end, true scale (gs is unchanged by the
        // forward sweep and serves as H in the tail below)
        scale_rows(gs, iR);
        Rr = 1.f; iR = 1.f;
        // state entering the block
        load_rows(xs, p.ckpt + ((int64_t)bb * (p.nck + 1) + k) * d * N, false);
        Q = 1.f; iQ = 1.f;

        // --------------------------------------------- forward sweep
        pass(tb, NSUB, +1, te, false, [&](int sb, int64_t) {
            snap_rows(xs, 1.f);  // state entering the sub-block (xs unscaled here)
            float lg = 0.f, E = 1.f;
            auto tok = [&](int tt, auto check) {
                const float yv = red(fstep(tt, check));
                const float fv = sm.f[tt][pl];
                lg += fmaxf(__logf(fv), kLogFloor);
                E *= fv;
                if (js == 0) {
                    sm.ys[sb * T + tt][pl] = yv;
                    sm.x1[tt][pl] = lg;
                    sm.x2[tt][pl] = E;
                }
            };
            if (fast_fwd()) {
#pragma unroll 2
                for (int tt = 0; tt < T; ++tt) tok(tt, Unchecked{});
            } else {
                for (int tt = 0; tt < T; ++tt) tok(tt, Checked{});
            }
            scale_rows(xs, iQ);
            Q = 1.f; iQ = 1.f;
            __syncthreads();
            // Pivot factors of A around token T/2 of the sub-block.
#pragma unroll
            for (int kk = 0; kk < R; ++kk) {
                const int tt = rr * R + kk;
                const float piv = sm.x1[T / 2][pp];
                const float l = sm.x1[tt][pp];
                sm.x3[tt][pp] = sm.dy[tt][pp] * __expf(l - piv);
                sm.x4[tt][pp] = sm.v[tt][pp] * __expf(piv - l);
                sm.x2[tt][pp] *= sm.dy[tt][pp];  // dy_t E_t
            }
            __syncthreads();
            // A[t][m] = sum_p fa[t][p] fb[m][p] for m <= t (two outputs per thread).
#pragma unroll
            for (int h2 = 0; h2 < 2; ++h2) {
                const int e = tid + h2 * NT;
                const int tt = e / T, mm = e % T;
                float a = 0.f;
                if (mm <= tt) {
#pragma unroll 8
                    for (int q2 = 0; q2 < P; ++q2) a = fmaf(sm.x3[tt][q2], sm.x4[mm][q2], a);
                }
                sm.A[sb][tt][mm] = a;
            }
            __syncthreads();
            // dC[t][j] = s [ sum_p (dy E)[t][p] X_b[p][j] + sum_{m<=t} A[t][m] B[m][j] ].
            {
                constexpr int JB = (N * T) / NT;  // outputs per thread
                const int tt = tid % T;
                const int j0 = (tid / T) * JB;
                float o[JB];
#pragma unroll
                for (int r = 0; r < JB; ++r) o[r] = 0.f;
#pragma unroll 4
                for (int q2 = 0; q2 < P; ++q2) {
                    const float a = sm.x2[tt][q2];
#pragma unroll
                    for (int r = 0; r < JB; ++r) o[r] = fmaf(a, sm.snap[q2][j0 + r], o[r]);
                }
                for (int mm = 0; mm <= tt; ++mm) {
                    const float a = sm.A[sb][tt][mm];
#pragma unroll
                    for (int r = 0; r < JB; ++r) o[r] = fmaf(a, sm.Bf[mm][j0 + r], o[r]);
                }
#pragma unroll
                for (int r = 0; r < JB; ++r) sm.acc[sb * T + tt][j0 + r] = s * o[r];
            }
        });
        cluster_reduce(1, tb, te);

        // tail of f df over this block: H . x_end (per channel)
        float tail = 0.f;
#pragma unroll
        for (int j = 0; j < NS / 2; ++j) tail = fmaf(gs[j].x, xs[j].x, fmaf(gs[j].y, xs[j].y, tail));
        tail = red(tail);

        // --------------------------------------------- backward sweep
        float cum = 0.f;  // sum of dL over later tokens of the block
        const bool group_end_block = (k == kb1 - 1);
        pass(tb + (NSUB - 1) * T, NSUB, -1, te, true, [&](int i, int64_t t0) {
            const int sb = NSUB - 1 - i;
            snap_rows(gs, iR);  // H_e: carry entering the sub-block's end, true scale
            float F = 1.f;      // prod f_{m+1..end of sub-block}
            auto tok = [&](int tt, auto check) {
                const float gbv = red(bstep(tt, true));
                const float vv = sm.v[tt][pl];
                const float dL = s * sm.dy[tt][pl] * sm.ys[sb * T + tt][pl] - vv * gbv;
                cum += dL;
                if (js == 0) {
                    sm.x1[tt][pl] = gbv;
                    sm.x3[tt][pl] = cum + tail;
                    sm.x2[tt][pl] = vv * F;  // (i h F)_m
                }
                F *= sm.f[tt][pl];
                bdecay(tt, check);
            };
            if (fast_bwd()) {
#pragma unroll 2
                for (int tt = T - 1; tt >= 0; --tt) tok(tt, Unchecked{});
            } else {
                for (int tt = T - 1; tt >= 0; --tt) tok(tt, Checked{});
            }
            __syncthreads();
            // dB[m][j] = sum_p (i h F)[m][p] H_e[p][j] + s sum_{t>=m} A[t][m] C[t][j].
            {
                constexpr int JB = (N * T) / NT;
                const int mm = tid % T;
                const int j0 = (tid / T) * JB;
                float o[JB], o2[JB];
#pragma unroll
                for (int r = 0; r < JB; ++r) { o[r] = 0.f; o2[r] = 0.f; }
#pragma unroll 4
                for (int q2 = 0; q2 < P; ++q2) {
                    const float a = sm.x2[mm][q2];
#pragma unroll
                    for (int r = 0; r < JB; ++r) o[r] = fmaf(a, sm.snap[q2][j0 + r], o[r]);
                }
                for (int tt = mm; tt < T; ++tt) {
                    const float a = sm.A[sb][tt][mm];
#pragma unroll
                    for (int r = 0; r < JB; ++r) o2[r] = fmaf(a, sm.Cf[tt][j0 + r], o2[r]);
                }
#pragma unroll
                for (int r = 0; r < JB; ++r) sm.acc[sb * T + mm][j0 + r] = fmaf(s, o2[r], o[r]);
            }
            // Per-channel gradients of the sub-block (thread pp, run rr).
#pragma unroll
            for (int kk = 0; kk < R; ++kk) {
                const int tt = rr * R + kk;
                const int64_t t = t0 + tt;
                float dpv = 0.f;
                if (cpvalid && t < te) {
                    float h, pre = 0.f;
                    if (CONV) {
                        pre = wb + w0 * to_f(sm.u[tt][pp]) + w1 * to_f(sm.u[tt + 1][pp]) +
                              w2 * to_f(sm.u[tt + 2][pp]) + w3 * to_f(sm.u[tt + 3][pp]);
                        h = siluf_(pre);
                    } else {
                        h = to_f(sm.u[tt + 3][pp]);
                    }
                    const float fv = sm.f[tt][pp];
                    const float iv = gbp ? sigmoidf_(to_f(sm.b[tt][pp]))
                                         : __expf(-to_f(sm.a[tt][pp])) * fv;
                    const float gbv = sm.x1[tt][pp];
                    const float dyv = sm.dy[tt][pp];
                    const float dh = Dc * dyv + iv * gbv;
                    if (gbp) {
                        gda[t * d + cp] = from_f<Tout>(sm.x3[tt][pp] * (1.f - fv));
                        gdb[t * d + cp] = from_f<Tout>(h * gbv * iv * (1.f - iv));
                    } else {  // da = (f df - f di)(1 - f), di = h G.B
                        gda[t * d + cp] = from_f<Tout>((sm.x3[tt][pp] - fv * h * gbv) * iv);
                    }
                    if (gz) {
                        const float zv = to_f(sm.z[tt][pp]);
                        const float yv = fmaf(s, sm.ys[sb * T + tt][pp], Dc * h);
                        gdz[t * d + cp] = from_f<Tout>(to_f(sm.dout[tt][pp]) * yv * dsiluf_(zv));
                    }
                    dD_acc = fmaf(dyv, h, dD_acc);
                    if (CONV) {
                        dpv = dh * dsiluf_(pre);
                        dw0 = fmaf(dpv, to_f(sm.u[tt][pp]), dw0);
                        dw1 = fmaf(dpv, to_f(sm.u[tt + 1][pp]), dw1);
                        dw2 = fmaf(dpv, to_f(sm.u[tt + 2][pp]), dw2);
                        dw3 = fmaf(dpv, to_f(sm.u[tt + 3][pp]), dw3);
                        dbias += dpv;
                    } else {
                        gdhu[t * d + cp] = from_f<Tout>(dh);
                    }
                }
                if (CONV) sm.dp[tt][pp] = dpv;
            }
            if (CONV) {
                __syncthreads();
                // du_t = w3 dp_t + w2 dp_{t+1} + w1 dp_{t+2} + w0 dp_{t+3}
#pragma unroll
                for (int kk = 0; kk < R; ++kk) {
                    const int tt = rr * R + kk;
                    const int64_t t = t0 + tt;
                    if (cpvalid && t < te) {
                        const float duv = w3 * sm.dp[tt][pp] + w2 * sm.dp[tt + 1][pp] +
                                          w1 * sm.dp[tt + 2][pp] + w0 * sm.dp[tt + 3][pp];
                        if (!lastg && group_end_block && t >= te - 3) {
                            edge[(3 + (t - (te - 3))) * d + cp] = duv;  // partial, fixed up later
                        } else {
                            gdhu[t * d + cp] = from_f<Tout>(duv);
                        }
                        if (k == kb0 && sb == 0 && tt < 3) edge[tt * d + cp] = sm.dp[tt][pp];
                    }
                }
                __syncthreads();
                if (tid < P) {  // carry the first three dp rows to the earlier sub-block
                    sm.dp[T][tid] = sm.dp[0][tid];
                    sm.dp[T + 1][tid] = sm.dp[1][tid];
                    sm.dp[T + 2][tid] = sm.dp[2][tid];
                }
            }
        });
        cluster_reduce(0, tb, te);
    }

    // ------------------------------------------------ carries and partials
    if (firstg && p.dx0) store_rows(p.dx0 + (int64_t)bb * d * N, gs, iR);
    // Per-channel partial sums (runs of the same channel add through shared atomics).
    {
        float* cpart = p.chan_part + ((int64_t)bb * p.ngroups + g) * d * 8;
        float* red6 = &sm.x1[0][0];  // reuse: [6][P] (T >= 6)
        __syncthreads();
        for (int i = tid; i < 6 * P; i += NT) red6[i] = 0.f;
        __syncthreads();
        if (cpvalid) {
            atomicAdd(&red6[0 * P + pp], dD_acc);
            atomicAdd(&red6[1 * P + pp], dw0);
            atomicAdd(&red6[2 * P + pp], dw1);
            atomicAdd(&red6[3 * P + pp], dw2);
            atomicAdd(&red6[4 * P + pp], dw3);
            atomicAdd(&red6[5 * P + pp], dbias);
        }
        __syncthreads();
        if (tid < P && c0 + tid < d) {
#pragma unroll
            for (int r = 0; r < 6; ++r) cpart[(c0 + tid) * 8 + r] = red6[r * P + tid];
        }
    }
}

// Sum the cluster partials of dB, dC and write them in the output dtype.
template <typename Tout>
__global__ void reduce_dBC_kernel(const float* __restrict__ part, int nclus, int64_t BtL,
                                  int64_t N, Tout* __restrict__ dB, Tout* __restrict__ dC) {
    // Four consecutive d_state entries per thread (N % 4 == 0): 16-byte loads,
    // four partial sets in flight.
    const int64_t n4 = BtL * N / 4;
    for (int64_t i4 = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i4 < n4;
         i4 += (int64_t)gridDim.x * blockDim.x) {
        const int64_t i = i4 * 4, row = i / N, j = i % N;
        float4 sb = make_float4(0.f, 0.f, 0.f, 0.f), sc = sb;
#pragma unroll 4
        for (int q = 0; q < nclus; ++q) {
            const float* pr = part + ((int64_t)q * BtL + row) * 2 * N;
            const float4 b4 = *reinterpret_cast<const float4*>(pr + j);
            const float4 c4 = *reinterpret_cast<const float4*>(pr + N + j);
            sb.x += b4.x; sb.y += b4.y; sb.z += b4.z; sb.w += b4.w;
            sc.x += c4.x; sc.y += c4.y; sc.z += c4.z; sc.w += c4.w;
        }
        dB[i] = from_f<Tout>(sb.x); dB[i + 1] = from_f<Tout>(sb.y);
        dB[i + 2] = from_f<Tout>(sb.z); dB[i + 3] = from_f<Tout>(sb.w);
        dC[i] = from_f<Tout>(sc.x); dC[i + 1] = from_f<Tout>(sc.y);
        dC[i + 2] = from_f<Tout>(sc.z); dC[i + 3] = from_f<Tout>(sc.w);
    }
}

// Sum per-(batch, block) channel partials: dD, dconv_w[4], dconv_b.
__global__ void reduce_chan_kernel(const float* __restrict__ part, int64_t rows, int64_t d,
                                   float* dD, float* dw, float* dbias) {
    const int64_t c = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (c >= d) return;
    float acc[6] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
    for (int64_t r = 0; r < rows; ++r) {
        const float* pr = part + (r * d + c) * 8;
#pragma unroll
        for (int q = 0; q < 6; ++q) acc[q] += pr[q];
    }
    if (dD) dD[c] = acc[0];
    if (dw) {
        dw[c * 4] = acc[1]; dw[c * 4 + 1] = acc[2]; dw[c * 4 + 2] = acc[3]; dw[c * 4 + 3] = acc[4];
    }
    if (dbias) dbias[c] = acc[5];
}

// Piece mode of the tensor-core backward: the same fixup at the cut of each
// cut unit (128 channels of one batch element).  The units' blocks, laid end
// to end (Wb in all), are cut at k Wb / npieces; unit u holds blocks
// [u nsub, (u + 1) nsub) and at most one cut.  Head edges are group slot 0,
// tail edges slot 1.
template <typename Tout>
__global__ void conv_edge_pieces_kernel(const float* __restrict__ edge,
                                        const float* __restrict__ w, int64_t Bt, int ntiles,
                                        int nsub, int npieces, int64_t L, int64_t d,
                                        Tout* __restrict__ du) {
    const int64_t n = Bt * 3 * d;
    const int64_t Wb = Bt * ntiles * (int64_t)nsub;
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n;
         i += (int64_t)gridDim.x * blockDim.x) {
        const int64_t c = i % d;
        const int r = (int)((i / d) % 3);
        const int64_t bb = i / (3 * d);
        const int64_t x = (bb * ntiles + c / 128) * nsub;  // the unit's first block
        // first cut after x: smallest k with k Wb / npieces > x
        const int64_t k = ((x + 1) * npieces + Wb - 1) / Wb;
        if (k >= npieces) continue;
        const int64_t cut = k * Wb / npieces;
        if (cut >= x + nsub) continue;  // uncut unit
        const int64_t tend = (cut - x) * kBwdSub;
        const int64_t t = tend - 3 + r;
        const float* mine = edge + ((bb * 2 + 0) * 2 + 1) * 3 * d;
        const float* next = edge + ((bb * 2 + 1) * 2 + 0) * 3 * d;
        float v = mine[r * d + c];
        for (int kk = 0; kk < 4; ++kk) {
            const int64_t ts = t + 3 - kk - tend;
            if (ts >= 0 && ts < 3) v += w[c * 4 + kk] * next[ts * d + c];
        }
        du[(bb * L + t) * d + c] = from_f<Tout>(v);
    }
}

// du of the last three tokens of each non-final sequence group: the group's
// own partial plus the terms from the first three dp of the next group.
template <typename Tout>
__global__ void conv_edge_kernel(const float* __restrict__ edge, const float* __restrict__ w,
                                 int64_t Bt, int ngroups, int64_t group_tokens, int64_t L,
                                 int64_t d, Tout* __restrict__ du) {
    const int64_t n = Bt * (int64_t)(ngroups - 1) * 3 * d;
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n;
         i += (int64_t)gridDim.x * blockDim.x) {
        const int64_t c = i % d;
        const int r = (int)((i / d) % 3);
        const int64_t gb = (i / (3 * d)) % (ngroups - 1);
        const int64_t bb = i / (3 * d * (ngroups - 1));
        const int64_t tend = (gb + 1) * group_tokens;
        const int64_t t = tend - 3 + r;
        const float* mine = edge + ((bb * ngroups + gb) * 2 + 1) * 3 * d;
        const float* next = edge + ((bb * ngroups + gb + 1) * 2 + 0) * 3 * d;
        float v = mine[r * d + c];
        // du_t += sum_k w[k] dp_{t+3-k} over the next group's tokens.
        for (int kk = 0; kk < 4; ++kk) {
            const int64_t ts = t + 3 - kk - tend;
            if (ts >= 0 && ts < 3) v += w[c * 4 + kk] * next[ts * d + c];
        }
        du[(bb * L + t) * d + c] = from_f<Tout>(v);
    }
}

// The follow-up kernels of a backward: dB / dC from the channel-tile partials
// (p.nclus partial sets), the per-channel sums, the conv group-boundary fixups.
// acc: dB / dC are already summed in an fp32 accumulator (one set).
template <typename Tout>
static cudaError_t reductions_t(const BwdParams& p, void* dB, void* dC, float* dD, float* dw,
                                float* dbias, cudaStream_t st, bool acc = false) {
    const bool conv = p.conv_w != nullptr;
    const int64_t BtL = p.Bt * p.L;
    if (acc) {
        cudaError_t e = launch_finish_dBC(p, std::is_same<Tout, float>::value ? NAJU_F32 : NAJU_BF16,
                                          dB, dC, st);
        if (e != cudaSuccess) return e;
    } else {
        reduce_dBC_kernel<Tout><<<592, 256, 0, st>>>(p.dBCp, p.nclus, BtL, p.N,
                                                      static_cast<Tout*>(dB),
                                                      static_cast<Tout*>(dC));
    }
    reduce_chan_kernel<<<(unsigned)((p.d + 127) / 128), 128, 0, st>>>(
        p.chan_part, p.Bt * p.ngroups, p.d, dD, conv ? dw : nullptr, conv ? dbias : nullptr);
    if (conv && p.npieces > 0)
        conv_edge_pieces_kernel<Tout><<<296, 256, 0, st>>>(p.conv_edge, p.conv_w, p.Bt, p.ntiles,
                                                            p.nsub, p.npieces, p.L, p.d,
                                                            static_cast<Tout*>(p.dhu));
    else if (conv && p.ngroups > 1)
        conv_edge_kernel<Tout><<<296, 256, 0, st>>>(p.conv_edge, p.conv_w, p.Bt, p.ngroups,
                                                     (int64_t)p.blk_per_group * kBwdSub, p.L,
                                                     p.d, static_cast<Tout*>(p.dhu));
    return cudaGetLastError();
}

cudaError_t launch_bwd_reductions_acc(const BwdParams& p, int out_dtype, void* dB, void* dC,
                                      float* dD, float* dw, float* dbias, cudaStream_t st) {
    if (out_dtype == NAJU_BF16)
        return reductions_t<__nv_bfloat16>(p, dB, dC, dD, dw, dbias, st, true);
    return reductions_t<float>(p, dB, dC, dD, dw, dbias, st, true);
}

cudaError_t launch_bwd_reductions(const BwdParams& p, int out_dtype, void* dB, void* dC,
                                  float* dD, float* dw, float* dbias, cudaStream_t st) {
    if (out_dtype == NAJU_BF16)
        return reductions_t<__nv_bfloat16>(p, dB, dC, dD, dw, dbias, st);
    return reductions_t<float>(p, dB, dC, dD, dw, dbias, st);
}

template <typename Tin, typename Tout, int N, bool CONV, int CL>
static cudaError_t launch_bwd_t(const BwdParams& p, void* dB, void* dC, float* dD, float* dw,
                                float* dbias, cudaStream_t st) {
    constexpr int S = BwdShape<N>::S;
    constexpr int P = 128 / S;
    const size_t smem = sizeof(BwdSmem<Tin, N, P>);
    auto kern = scan_bwd_kernel<Tin, Tout, N, CONV, CL>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)smem);
    if (e != cudaSuccess) return e;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)(p.nclus * CL), (unsigned)p.Bt, (unsigned)p.ngroups);
    cfg.blockDim = dim3(128);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = CL;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    e = cudaLaunchKernelEx(&cfg, kern, p);
    if (e != cudaSuccess) return e;
    return reductions_t<Tout>(p, dB, dC, dD, dw, dbias, st);
}

template <typename Tin, typename Tout, bool CONV>
static cudaError_t launch_bwd_n(const BwdParams& p, void* dB, void* dC, float* dD, float* dw,
                                float* dbias, cudaStream_t st) {
    const int cl = p.ntiles / p.nclus;  // blocks per cluster (bwd_cluster_size)
#define NAJU_BWD_N(NN)                                                                     \
    return cl == 2 ? launch_bwd_t<Tin, Tout, NN, CONV, 2>(p, dB, dC, dD, dw, dbias, st)  \
                   : launch_bwd_t<Tin, Tout, NN, CONV, kCluster>(p, dB, dC, dD, dw, dbias, st)
    if (cl != 2 && cl != kCluster) return cudaErrorInvalidValue;
    switch (p.N) {
        case 16: NAJU_BWD_N(16);
        case 32: NAJU_BWD_N(32);
        case 64: NAJU_BWD_N(64);
        case 128: NAJU_BWD_N(128);
        default: return cudaErrorInvalidValue;
    }
#undef NAJU_BWD_N
}

cudaError_t launch_scan_bwd(const BwdParams& p, int dtype, int out_dtype, void* dB, void* dC,
                            float* dD, float* dw, float* dbias, cudaStream_t st) {
    const bool conv = p.conv_w != nullptr;
    if (dtype == NAJU_F32)
        return conv ? launch_bwd_n<float, float, true>(p, dB, dC, dD, dw, dbias, st)
                    : launch_bwd_n<float, float, false>(p, dB, dC, dD, dw, dbias, st);
    if (out_dtype == NAJU_BF16)
        return conv ? launch_bwd_n<__nv_bfloat16, __nv_bfloat16, true>(p, dB, dC, dD, dw, dbias, st)
                    : launch_bwd_n<__nv_bfloat16, __nv_bfloat16, false>(p, dB, dC, dD, dw, dbias,
                                                                         st);
    return conv ? launch_bwd_n<__nv_bfloat16, float, true>(p, dB, dC, dD, dw, dbias, st)
                : launch_bwd_n<__nv_bfloat16, float, false>(p, dB, dC, dD, dw, dbias, st);
}

}  // namespace naju
