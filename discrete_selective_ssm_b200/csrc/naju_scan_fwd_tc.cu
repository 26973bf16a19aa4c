// Naju forward scan with the d_state contractions on the 5th-generation
// tensor cores (sm_100a, tcgen05, kind::tf32), for bf16 activations.
//
// Same computation as naju_scan_fwd.cu (Naju reproduction README, "Core
// equations"):  x_n = f_n x_{n-1} + i_n h_n B_n^T,  y_n = x_n.C_n/sqrt(N) + D h_n,
// out_n = y_n SiLU(z_n), h = SiLU(conv(u)).
//
// Chunked form.  A thread block owns 128 channels of one batch element (one
// channel per thread = one tensor-memory lane) and walks its tokens in
// sub-chunks of T = 16.  With X the state entering a sub-chunk,
// E_t = prod_{k<=t} f_k (inclusive, from the sub-chunk start),
// W_m = i_m h_m / E_m and G[t][m] = C_t.B_m (m <= t, else 0):
//   y_t  = s E_t ( X.C_t + sum_m W_m G[t][m] ) + D h_t         (readout MMA)
//   X'   = E_T X + sum_m (i_m h_m E_T / E_m) B_m                (state MMA)
// Both contractions run on the tensor core with the per-channel operands in
// tensor memory (X resident there for the whole sequence; W and the state
// weights written per sub-chunk) and the per-token operands (C, G, B) in
// shared memory; everything per (token, channel) - conv, gates, SiLU, decay
// prefixes, the outputs - runs on the CUDA cores.  The state chain from one
// sub-chunk to the next is only the elementwise X' = E_T X + D_state.
//
// Exactness.  W_m carries 1/E_m; a sub-chunk whose product of 1/f exceeds
// 2^64 in any channel of the block is run on the CUDA cores instead (the
// plain recurrence token by token, exact), so no input can overflow.  tf32
// operands give about 1e-3 relative error on the contractions; the fp32
// activations path uses the CUDA-core kernel.
//
// Threads.  256 threads: channel p is TMEM lane p; the two threads of a
// channel (warps w and w+4 share a lane quadrant) each unpack 8 of the 16
// tokens, exchanging their decay products through shared memory, and each
// update half of the state columns.
//
// Pipeline.  While the tensor core runs sub-chunk i, the CUDA cores unpack
// sub-chunk i+1 (double-buffered operands) and cp.async stages sub-chunk i+2.
// Sequence groups work as in the CUDA-core kernel: an update-only pass and a
// decoupled look-back publish each group's end state before the full pass.
#include <type_traits>

#include "naju_common.cuh"
#include "naju_kernels.h"
#include "naju_tc.cuh"

namespace naju {

namespace {

constexpr int kTS = 16;                               // tokens per sub-chunk
constexpr float kTcBound = 18446744073709551616.0f;   // 2^64

template <int N>
struct TcCols {
    static constexpr uint32_t X = 0;                  // state [N]
    static constexpr uint32_t W = N;                  // 2 x kTS (parity)
    static constexpr uint32_t V = N + 2 * kTS;        // 2 x kTS (parity)
    static constexpr uint32_t DR = N + 4 * kTS;       // readout result [kTS]
    static constexpr uint32_t DS = N + 5 * kTS;       // state result [N]
    static constexpr uint32_t USED = 2 * N + 5 * kTS;
    static constexpr uint32_t ALLOC = USED <= 256 ? 256 : 512;
};

template <int N>
struct FwdTcSmem {
    static constexpr int T = kTS, P = 128;
    struct Raw {
        __nv_bfloat16 u[T + 3][P];
        __nv_bfloat16 a[T][P], b[T][P], z[T][P];
        __nv_bfloat16 Bm[T][N], Cm[T][N];
    };
    alignas(128) Raw raw[2];
    alignas(128) float bc[2][T * N];   // C: rows t, K = j      (readout B operand, part 1)
    alignas(128) float bg[2][T * T];   // G: rows t, K = m      (readout B operand, part 2)
    alignas(128) float bs[2][N * T];   // B^T: rows j, K = m    (state B operand)
    alignas(16) float brow[2][T][N];   // B rows, fp32, for the Gram
    float eg[2][T][P];                 // s E_t SiLU(z_t)  (s SiLU(z_t) on the exact path)
    float dhg[2][T][P];                // D h_t SiLU(z_t)
    float yacc[T][P];                  // exact path: readout of the first column half
    float xq0[P], xe0[P], xe1[P];      // per-half decay products of a sub-chunk
    float elast[2][P];                 // E over the whole sub-chunk
    int slow[2];
    uint64_t mbar;
    uint32_t taddr;
    int item, ok;
};

}  // namespace

template <typename Tout, int N, bool CONV>
__global__ void __launch_bounds__(256, (N == 64 ? 2 : 1))
scan_fwd_tc_kernel(const FwdParams p) {
    using Tin = __nv_bfloat16;
    using Cols = TcCols<N>;
    using Sm = FwdTcSmem<N>;
    constexpr int T = kTS, P = 128, NT = 256, H = T / 2, NH = N / 2;
    extern __shared__ float4 smem4[];
    Sm& sm = *reinterpret_cast<Sm*>(smem4);

    const int tid = threadIdx.x;
    const int warp = tid >> 5;
    const int ch = tid & (P - 1);   // channel within the block = TMEM lane
    const int half = tid >> 7;      // token half (unpacking) / column half (state)
    const int64_t Bt = p.Bt, L = p.L, d = p.d;

    // ------------------------------------------------------------ set-up
    if (warp == 0) {
        tc::tmem_alloc(&sm.taddr, Cols::ALLOC);
        tc::tmem_relinquish();
    }
    if (tid == 0) {
        sm.item = atomicAdd(&p.hdr->fwd_ticket, 1);
        tc::mbar_init(&sm.mbar, 1);
    }
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    const uint32_t tbase = sm.taddr;
    const uint32_t lane = (uint32_t)((warp & 3) * 32) << 16;  // this warp's TMEM lanes
    const int item = sm.item;
    const int per_g = (int)(Bt * p.ntiles);
    const int g = item / per_g;
    const int bb = (item % per_g) / p.ntiles;
    const int tile = item % p.ntiles;
    const int64_t c0 = (int64_t)tile * P;
    const int64_t c = c0 + ch;
    const bool cvalid = c < d;

    const int seg0 = g * p.seg_per_group;
    const int seg1 = min(seg0 + p.seg_per_group, p.nck);
    const int64_t tbeg = (int64_t)seg0 * p.T_ck;
    const int64_t tend = min64(L, (int64_t)seg1 * p.T_ck);
    const bool last_group = (g == p.ngroups - 1);

    const int64_t boff = (int64_t)bb * L;
    const Tin* hu = static_cast<const Tin*>(p.hu) + boff * d;
    const Tin* ga = static_cast<const Tin*>(p.a) + boff * d;
    const Tin* gb = static_cast<const Tin*>(p.b) + boff * d;
    const Tin* gz = p.z ? static_cast<const Tin*>(p.z) + boff * d : nullptr;
    const Tin* gB = static_cast<const Tin*>(p.B) + boff * N;
    const Tin* gC = static_cast<const Tin*>(p.C) + boff * N;
    Tout* gy = static_cast<Tout*>(p.y) + boff * d;
    const bool vec = ((d * (int64_t)sizeof(Tin)) % 16) == 0;

    float w0 = 0.f, w1 = 0.f, w2 = 0.f, w3 = 0.f, wb = 0.f, Dc = 0.f;
    if (cvalid) {
        if (CONV) {
            w0 = p.conv_w[c * 4 + 0];
            w1 = p.conv_w[c * 4 + 1];
            w2 = p.conv_w[c * 4 + 2];
            w3 = p.conv_w[c * 4 + 3];
            wb = p.conv_b ? p.conv_b[c] : 0.f;
        }
        Dc = p.D ? p.D[c] : 0.f;
    }
    const float scale = p.scale;
    float* ck_b = p.ckpt + (int64_t)bb * (p.nck + 1) * d * N;
    bool timed_out = false;

    // ---------------------------------------------------------- helpers
    auto issue = [&](int64_t t0, int buf, bool full) {
        typename Sm::Raw& r = sm.raw[buf];
        stage_rows(&r.u[0][0], hu, d, t0 - 3, T + 3, L, c0, P, vec, tid, NT);
        stage_rows(&r.a[0][0], ga, d, t0, T, tend, c0, P, vec, tid, NT);
        stage_rows(&r.b[0][0], gb, d, t0, T, tend, c0, P, vec, tid, NT);
        if (full && gz) stage_rows(&r.z[0][0], gz, d, t0, T, tend, c0, P, vec, tid, NT);
        stage_rows(&r.Bm[0][0], gB, N, t0, T, tend, 0, N, true, tid, NT);
        if (full) stage_rows(&r.Cm[0][0], gC, N, t0, T, tend, 0, N, true, tid, NT);
        cp_async_commit();
    };
    // Unpack sub-chunk (t0, raw buffer `buf`) into operand set `pr`.
    auto prep = [&](int64_t t0, int buf, int pr, bool full) {
        const typename Sm::Raw& r = sm.raw[buf];
        // Per-token operands: four consecutive d_state entries per step.
        for (int e = tid; e < T * N / 4; e += NT) {
            const int tt = e / (N / 4), j = (e % (N / 4)) * 4;
            const uint2 braw = *reinterpret_cast<const uint2*>(&r.Bm[tt][j]);
            const float2 b01 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&braw.x));
            const float2 b23 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&braw.y));
            *reinterpret_cast<float4*>(&sm.brow[pr][tt][j]) = make_float4(b01.x, b01.y, b23.x, b23.y);
            sm.bs[pr][tc::kmajor_offset(j + 0, tt, T) >> 2] = b01.x;
            sm.bs[pr][tc::kmajor_offset(j + 1, tt, T) >> 2] = b01.y;
            sm.bs[pr][tc::kmajor_offset(j + 2, tt, T) >> 2] = b23.x;
            sm.bs[pr][tc::kmajor_offset(j + 3, tt, T) >> 2] = b23.y;
            if (full) {
                const uint2 craw = *reinterpret_cast<const uint2*>(&r.Cm[tt][j]);
                const float2 c01 =
                    __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&craw.x));
                const float2 c23 =
                    __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&craw.y));
                *reinterpret_cast<float4*>(&sm.bc[pr][tc::kmajor_offset(tt, j, N) >> 2]) =
                    make_float4(c01.x, c01.y, c23.x, c23.y);
            }
        }
        // Per-channel values: this thread's 8 tokens.
        float qv[H], fv[H], hv[H];
        float Qh = 1.f, Eh = 1.f;
#pragma unroll
        for (int k = 0; k < H; ++k) {
            const int tt = half * H + k;
            const bool valid = cvalid && (t0 + tt < tend);
            qv[k] = valid ? 1.f + __expf(-to_f(r.a[tt][ch])) : 1.f;
            fv[k] = rcpa_(qv[k]);
            Qh *= qv[k];
            Eh *= fv[k];
            float h = 0.f;
            if (valid) {
                if (CONV) {
                    h = silua_(wb + w0 * to_f(r.u[tt][ch]) + w1 * to_f(r.u[tt + 1][ch]) +
                               w2 * to_f(r.u[tt + 2][ch]) + w3 * to_f(r.u[tt + 3][ch]));
                } else {
                    h = to_f(r.u[tt + 3][ch]);
                }
            }
            hv[k] = h;
        }
        if (half == 0) {
            sm.xq0[ch] = Qh;
            sm.xe0[ch] = Eh;
        } else {
            sm.xe1[ch] = Eh;
        }
        __syncthreads();
        const float Q0 = sm.xq0[ch], E0 = sm.xe0[ch], E1 = sm.xe1[ch];
        const int slow = __syncthreads_or((half == 1 && !(Q0 * Qh <= kTcBound)) ? 1 : 0);
        const float Elast = E0 * E1;
        float Q = half ? Q0 : 1.f, E = half ? E0 : 1.f;
        float Wv[H], Vv[H];
#pragma unroll
        for (int k = 0; k < H; ++k) {
            const int tt = half * H + k;
            const bool valid = cvalid && (t0 + tt < tend);
            const float v = valid ? sigmoida_(to_f(r.b[tt][ch])) * hv[k] : 0.f;
            E *= fv[k];
            Q *= qv[k];
            if (slow) {
                Wv[k] = v;        // the exact path reads i h and f back from TMEM
                Vv[k] = fv[k];
            } else {
                Wv[k] = v * Q;           // v_m / E_m
                Vv[k] = v * Q * Elast;   // v_m E_T / E_m
            }
            if (full) {
                const float gg = (valid && gz) ? silua_(to_f(r.z[tt][ch])) : 1.f;
                sm.eg[pr][tt][ch] = slow ? scale * gg : scale * E * gg;
                sm.dhg[pr][tt][ch] = Dc * hv[k] * gg;
            }
        }
        if (half == 0) sm.elast[pr][ch] = Elast;
        if (tid == 0) sm.slow[pr] = slow;
        tc::tmem_st8(tbase + lane + Cols::W + pr * T + half * H, Wv);
        tc::tmem_st8(tbase + lane + Cols::V + pr * T + half * H, Vv);
        tc::tmem_st_wait();
        if (full && !slow) {
            __syncthreads();  // bc, brow complete
            // G[t][m] = C_t . B_m for m <= t (one entry per thread).
            const int tt = tid / T, mm = tid % T;
            float a = 0.f;
            if (mm <= tt) {
#pragma unroll 4
                for (int j = 0; j < N; j += 4) {
                    const float4 cv = *reinterpret_cast<const float4*>(
                        &sm.bc[pr][tc::kmajor_offset(tt, j, N) >> 2]);
                    const float4 bv = *reinterpret_cast<const float4*>(&sm.brow[pr][mm][j]);
                    a = fmaf(cv.x, bv.x, fmaf(cv.y, bv.y, fmaf(cv.z, bv.z, fmaf(cv.w, bv.w, a))));
                }
            }
            sm.bg[pr][tc::kmajor_offset(tt, mm, T) >> 2] = a;
        }
    };
    // Issue the sub-chunk's MMAs (one thread) and commit them to the barrier.
    auto issue_mma = [&](int pr, bool full) {
        const uint32_t id_r = tc::idesc_tf32(128, T);
        const uint32_t id_s = tc::idesc_tf32(128, N);
        if (full) {
            const uint32_t sc = tc::smem_u32(&sm.bc[pr][0]);
#pragma unroll
            for (int ks = 0; ks < N / 8; ++ks)
                tc::mma_tf32_ts(tbase + Cols::DR, tbase + Cols::X + ks * 8,
                                tc::sdesc(sc + ks * 256, 128, 32 * N), id_r, ks > 0 ? 1u : 0u);
            const uint32_t sg = tc::smem_u32(&sm.bg[pr][0]);
#pragma unroll
            for (int ks = 0; ks < T / 8; ++ks)
                tc::mma_tf32_ts(tbase + Cols::DR, tbase + Cols::W + pr * T + ks * 8,
                                tc::sdesc(sg + ks * 256, 128, 32 * T), id_r, 1u);
        }
        const uint32_t ss = tc::smem_u32(&sm.bs[pr][0]);
#pragma unroll
        for (int ks = 0; ks < T / 8; ++ks)
            tc::mma_tf32_ts(tbase + Cols::DS, tbase + Cols::V + pr * T + ks * 8,
                            tc::sdesc(ss + ks * 256, 128, 32 * T), id_s, ks > 0 ? 1u : 0u);
        tc::mma_commit(&sm.mbar);
    };
    // TMEM state row <-> global row (each thread moves its column half).
    auto state_from = [&](const float* src, bool cg) {
#pragma unroll
        for (int n0 = half * NH; n0 < half * NH + NH; n0 += 16) {
            float v[16];
#pragma unroll
            for (int k = 0; k < 16; k += 4) {
                float4 v4 = make_float4(0.f, 0.f, 0.f, 0.f);
                if (src && cvalid) {
                    const float4* s4 = reinterpret_cast<const float4*>(src + c * N + n0 + k);
                    v4 = cg ? __ldcg(s4) : *s4;
                }
                v[k] = v4.x; v[k + 1] = v4.y; v[k + 2] = v4.z; v[k + 3] = v4.w;
            }
            tc::tmem_st16(tbase + lane + Cols::X + n0, v);
        }
        tc::tmem_st_wait();
    };
    auto state_to = [&](float* dst) {
#pragma unroll
        for (int n0 = half * NH; n0 < half * NH + NH; n0 += 16) {
            float v[16];
            tc::tmem_ld16(tbase + lane + Cols::X + n0, v);
            tc::tmem_ld_wait();
            if (cvalid) {
#pragma unroll
                for (int k = 0; k < 16; k += 4)
                    *reinterpret_cast<float4*>(dst + c * N + n0 + k) =
                        make_float4(v[k], v[k + 1], v[k + 2], v[k + 3]);
            }
        }
    };
    // Sub-chunk i's results: outputs (full) and the next state.
    float logP = 0.f;  // log of the decay product over the pass
    auto epilogue = [&](int64_t t0, int pr, bool full) {
        const float El = sm.elast[pr][ch];
        if (!sm.slow[pr]) {
            if (full) {
                float dr[H];
                tc::tmem_ld8(tbase + lane + Cols::DR + half * H, dr);
                tc::tmem_ld_wait();
                if (cvalid) {
#pragma unroll
                    for (int k = 0; k < H; ++k) {
                        const int tt = half * H + k;
                        const int64_t t = t0 + tt;
                        if (t < tend)
                            gy[t * d + c] =
                                from_f<Tout>(fmaf(sm.eg[pr][tt][ch], dr[k], sm.dhg[pr][tt][ch]));
                    }
                }
            }
#pragma unroll
            for (int n0 = half * NH; n0 < half * NH + NH; n0 += 16) {
                float x[16], s2[16];
                tc::tmem_ld16(tbase + lane + Cols::X + n0, x);
                tc::tmem_ld16(tbase + lane + Cols::DS + n0, s2);
                tc::tmem_ld_wait();
#pragma unroll
                for (int k = 0; k < 16; ++k) x[k] = fmaf(El, x[k], s2[k]);
                tc::tmem_st16(tbase + lane + Cols::X + n0, x);
            }
            logP += __logf(El);
        } else {
            // Exact path: x <- f x + (i h) B token by token, y from x . C, each
            // thread on its column half; the halves' readouts meet in yacc.
            float vv[16], ff[16], yp[16];
            tc::tmem_ld16(tbase + lane + Cols::W + pr * T, vv);
            tc::tmem_ld16(tbase + lane + Cols::V + pr * T, ff);
            tc::tmem_ld_wait();
#pragma unroll
            for (int tt = 0; tt < T; ++tt) yp[tt] = 0.f;
            for (int n0 = half * NH; n0 < half * NH + NH; n0 += 16) {
                float x[16];
                tc::tmem_ld16(tbase + lane + Cols::X + n0, x);
                tc::tmem_ld_wait();
#pragma unroll
                for (int tt = 0; tt < T; ++tt) {
                    float acc = 0.f;
#pragma unroll
                    for (int k = 0; k < 16; ++k) {
                        x[k] = fmaf(ff[tt], x[k], vv[tt] * sm.brow[pr][tt][n0 + k]);
                        if (full)
                            acc = fmaf(x[k], sm.bc[pr][tc::kmajor_offset(tt, n0 + k, N) >> 2], acc);
                    }
                    yp[tt] += acc;
                }
                tc::tmem_st16(tbase + lane + Cols::X + n0, x);
            }
            if (full) {
                if (half == 0) {
#pragma unroll
                    for (int tt = 0; tt < T; ++tt) sm.yacc[tt][ch] = yp[tt];
                }
                __syncthreads();
                if (half == 1 && cvalid) {
#pragma unroll
                    for (int tt = 0; tt < T; ++tt) {
                        const int64_t t = t0 + tt;
                        if (t < tend)
                            gy[t * d + c] = from_f<Tout>(fmaf(
                                sm.eg[pr][tt][ch], yp[tt] + sm.yacc[tt][ch], sm.dhg[pr][tt][ch]));
                    }
                }
            }
            float lp = 0.f;
#pragma unroll
            for (int tt = 0; tt < T; ++tt) lp += __logf(ff[tt]);
            logP += lp;
        }
        tc::tmem_st_wait();
    };
    uint32_t phase = 0;
    // One pass over the group's sub-chunks (full: readout, outputs, checkpoints).
    auto run_pass = [&](bool full) {
        const int nsc = (int)((tend - tbeg + T - 1) / T);
        issue(tbeg, 0, full);
        if (nsc > 1) {
            issue(tbeg + T, 1, full);
            cp_async_wait<1>();
        } else {
            cp_async_wait<0>();
        }
        __syncthreads();
        prep(tbeg, 0, 0, full);
        tc::fence_proxy_async();
        tc::fence_before_sync();
        __syncthreads();
        if (tid == 0) {
            tc::fence_after_sync();
            if (!sm.slow[0]) issue_mma(0, full);
        }
        for (int i = 0; i < nsc; ++i) {
            const int pr = i & 1;
            const int64_t t0 = tbeg + (int64_t)i * T;
            const bool more = i + 1 < nsc;
            if (more) {
                cp_async_wait<0>();
                __syncthreads();  // raw (i+1) visible; raw (i) free
                if (i + 2 < nsc) issue(t0 + 2 * T, i & 1, full);
                prep(t0 + T, (i + 1) & 1, pr ^ 1, full);
            }
            if (!sm.slow[pr]) {
                if (!tc::mbar_wait(&sm.mbar, phase, 1LL << 24)) timed_out = true;
                phase ^= 1u;
            }
            tc::fence_after_sync();
            epilogue(t0, pr, full);
            if (full) {
                const int64_t tnext = t0 + T;
                if (tnext < tend && tnext % p.T_ck == 0) state_to(ck_b + (tnext / p.T_ck) * d * N);
            }
            tc::fence_proxy_async();
            tc::fence_before_sync();
            __syncthreads();
            if (more && tid == 0) {
                tc::fence_after_sync();
                if (!sm.slow[pr ^ 1]) issue_mma(pr ^ 1, full);
            }
        }
    };

    // ------------------------------------------ early pass and carry chain
    const float* x0b = p.x0 ? p.x0 + (int64_t)bb * d * N : nullptr;
    const int* flag_prev = (g > 0) ? p.flags + ((int64_t)(g - 1) * Bt + bb) * p.ntiles + tile
                                   : nullptr;
    int* flag_mine = p.flags + ((int64_t)g * Bt + bb) * p.ntiles + tile;
    float* ck_start = ck_b + (int64_t)seg0 * d * N;
    float* ck_end = ck_b + (int64_t)seg1 * d * N;
    bool ok = true;
    if (!last_group) {
        state_from(g == 0 ? x0b : nullptr, false);
        tc::fence_before_sync();
        __syncthreads();
        tc::fence_after_sync();
        logP = 0.f;
        run_pass(false);
        if (g > 0) {
            const float Pf = __expf(logP);
            if (tid == 0) sm.ok = wait_flag(flag_prev, &p.hdr->status, p.wait_limit) ? 1 : 0;
            __syncthreads();
            ok = sm.ok != 0;
#pragma unroll
            for (int n0 = half * NH; n0 < half * NH + NH; n0 += 16) {
                float x[16];
                tc::tmem_ld16(tbase + lane + Cols::X + n0, x);
                tc::tmem_ld_wait();
#pragma unroll
                for (int k = 0; k < 16; k += 4) {
                    float4 v4 = make_float4(0.f, 0.f, 0.f, 0.f);
                    if (ok && cvalid)
                        v4 = __ldcg(reinterpret_cast<const float4*>(ck_start + c * N + n0 + k));
                    x[k] = fmaf(Pf, v4.x, x[k]);
                    x[k + 1] = fmaf(Pf, v4.y, x[k + 1]);
                    x[k + 2] = fmaf(Pf, v4.z, x[k + 2]);
                    x[k + 3] = fmaf(Pf, v4.w, x[k + 3]);
                }
                tc::tmem_st16(tbase + lane + Cols::X + n0, x);
            }
            tc::tmem_st_wait();
        }
        state_to(ck_end);
        __threadfence();
        __syncthreads();
        if (tid == 0 && !(g == 0 && p.fault_skip_publish)) st_release(flag_mine, 1);
    } else if (g > 0) {
        if (tid == 0) sm.ok = wait_flag(flag_prev, &p.hdr->status, p.wait_limit) ? 1 : 0;
        __syncthreads();
        ok = sm.ok != 0;
    }
    if (g > 0) {
        state_from(ok ? ck_start : nullptr, true);
    } else {
        state_from(x0b, false);
        state_to(ck_b);  // checkpoint 0 = initial state
    }
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();

    // ------------------------------------------------------- full pass
    run_pass(true);
    if (last_group) {
        state_to(ck_b + (int64_t)p.nck * d * N);
        if (p.x_final) state_to(p.x_final + (int64_t)bb * d * N);
    }
    if (timed_out && tid == 0) atomicOr(&p.hdr->status, 1 << NAJU_ERR_TIMEOUT);

    // ---------------------------------------------------------- teardown
    tc::fence_before_sync();
    __syncthreads();
    if (warp == 0) tc::tmem_dealloc(tbase, Cols::ALLOC);
}

template <typename Tout, int N, bool CONV>
static cudaError_t launch_fwd_tc_t(const FwdParams& p, cudaStream_t st) {
    // At least enough shared memory that no more blocks share an SM than its
    // 512 tensor-memory columns can hold.
    const size_t need = sizeof(FwdTcSmem<N>);
    const size_t floor_bytes = TcCols<N>::ALLOC == 512 ? (size_t)120 * 1024 : (size_t)80 * 1024;
    const size_t smem = need > floor_bytes ? need : floor_bytes;
    auto kern = scan_fwd_tc_kernel<Tout, N, CONV>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)smem);
    if (e != cudaSuccess) return e;
    const int grid = p.ngroups * (int)p.Bt * p.ntiles;
    kern<<<grid, 256, smem, st>>>(p);
    return cudaGetLastError();
}

int fwd_tc_channels_per_block() { return 128; }

bool fwd_tc_supported(int dtype, int64_t N) {
    return dtype == NAJU_BF16 && (N == 64 || N == 128);
}

cudaError_t launch_scan_fwd_tc(const FwdParams& p, int out_dtype, cudaStream_t st) {
    const bool conv = p.conv_w != nullptr;
#define NAJU_TC_FWD(TO, NN)                                                     \
    return conv ? launch_fwd_tc_t<TO, NN, true>(p, st) : launch_fwd_tc_t<TO, NN, false>(p, st)
    if (out_dtype == NAJU_BF16) {
        if (p.N == 64) NAJU_TC_FWD(__nv_bfloat16, 64);
        if (p.N == 128) NAJU_TC_FWD(__nv_bfloat16, 128);
    } else {
        if (p.N == 64) NAJU_TC_FWD(float, 64);
        if (p.N == 128) NAJU_TC_FWD(float, 128);
    }
#undef NAJU_TC_FWD
    return cudaErrorInvalidValue;
}

}  // namespace naju
