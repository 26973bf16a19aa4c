// Naju forward scan with the d_state contractions on the 5th-generation
// tensor cores (sm_100a, tcgen05, kind::tf32), for bf16 activations.
//
// Same computation as naju_scan_fwd.cu (Naju reproduction README, "Core
// equations"):  x_n = f_n x_{n-1} + i_n h_n B_n^T,  y_n = x_n.C_n/sqrt(N) + D h_n,
// out_n = y_n SiLU(z_n), h = SiLU(conv(u)).
//
// Chunked form.  A thread block owns 128 channels of one batch element (one
// channel = one tensor-memory lane) and walks its tokens in sub-chunks of
// T = 16.  With X the state entering a sub-chunk,
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
// Warp roles.  Warps 0-15 produce: one thread issues TMA loads of raw
// sub-chunks two ahead into three buffers (an mbarrier each), refilling a
// buffer once every producer has unpacked it (its stage's full barrier), and
// all 512 unpack each sub-chunk into one of three operand stages (shared
// memory + tensor-memory columns); channel p is handled by threads p + 128 q,
// q = 0..3, each taking 4 of the 16 tokens.  Warps 16-19 consume: thread 512 + p owns channel p;
// one of them issues the MMAs of a stage, all of them run the epilogue
// (outputs, X' = E_T X + D_state, checkpoints) and release the stage.  Stages
// hand over through mbarriers (full: 512 producer arrivals; empty: 128
// consumer arrivals; one MMA-completion barrier), so unpacking overlaps the
// tensor core and the epilogue.
//
// Sequence groups work as in the CUDA-core kernel: an update-only pass and a
// decoupled look-back publish each group's end state before the full pass.
// Piece mode (at least one wave of 128-channel units, not a whole number of
// waves) instead gives each block one equal range of all units' 64-token
// checkpoint segments; a unit cut in two hands the state at the cut from its
// head to its tail.
#include <string.h>

#include <type_traits>

#include "naju_common.cuh"
#include "naju_kernels.h"
#include "naju_tc.cuh"
#include "naju_tma.h"

namespace naju {

namespace {

constexpr int kTS = 16;                               // tokens per sub-chunk
constexpr int kStages = 3;                            // operand stages = raw buffers
constexpr float kTcBound = 18446744073709551616.0f;   // 2^64
// No quarter (4 tokens) above 2^16 means no channel's sub-chunk above 2^64.
constexpr float kTcQuarter = 65536.0f;
constexpr long long kMbarSpin = 1LL << 24;            // polls before giving up

// Tensor-memory columns (lane = channel).  Per stage: W (readout weights,
// or i h on the exact path), V (state weights, or f), EG (s E_t SiLU(z_t),
// or s SiLU(z_t) on the exact path), DH (D h_t SiLU(z_t)).
template <int N>
struct TcCols {
    static constexpr uint32_t X = 0;                           // state [N]
    static constexpr uint32_t W = N;                           // kStages x kTS each
    static constexpr uint32_t V = W + kStages * kTS;
    static constexpr uint32_t EG = V + kStages * kTS;
    static constexpr uint32_t DH = EG + kStages * kTS;
    static constexpr uint32_t DR = DH + kStages * kTS;         // readout result [kTS]
    static constexpr uint32_t DS = DR + kTS;                   // state result [N]
    static constexpr uint32_t USED = DS + N;
    static constexpr uint32_t ALLOC = USED <= 256 ? 256 : 512;
    static_assert(USED <= 512, "tensor memory");
};

struct alignas(64) FwdTmaps {
    CUtensorMap u, a, b, z, B, C;
};

template <int N>
struct FwdTcSmem {
    static constexpr int T = kTS, P = 128, S = kStages, NP = N + 4;
    // TMA destinations (each 128-byte aligned; rows of 256 bytes).
    struct Raw {
        alignas(128) __nv_bfloat16 u[T + 3][P];
        alignas(128) __nv_bfloat16 a[T][P];
        alignas(128) __nv_bfloat16 b[T][P];
        alignas(128) __nv_bfloat16 z[T][P];
        alignas(128) __nv_bfloat16 Bm[T][N];
        alignas(128) __nv_bfloat16 Cm[T][N];
    };
    // One stage of unpacked sub-chunk operands.
    struct Stage {
        alignas(128) float bc[T * N];   // C: rows t, K = j      (readout B operand, part 1)
        alignas(128) float bg[T * T];   // G: rows t, K = m      (readout B operand, part 2)
        alignas(128) float bs[N * T];   // B^T: rows j, K = m    (state B operand)
        alignas(16) float brow[T][NP];  // B rows, fp32, padded against bank conflicts
        alignas(16) float crow[T][NP];  // C rows, fp32, padded
        float elast[P];                 // E over the whole sub-chunk
        int slow;
    };
    Raw raw[S];
    Stage st[S];
    float xq[4][P], xe[4][P];           // per-quarter decay products of a sub-chunk
    uint64_t loaded[S], full[S], empty[S], mma;
    uint32_t taddr;
    int item, ok;
};

}  // namespace

template <typename Tout, int N, bool CONV, bool PIECES>
__global__ void __launch_bounds__(640, 1)
scan_fwd_tc_kernel(const FwdParams p, const __grid_constant__ FwdTmaps tm) {
    using Tin = __nv_bfloat16;
    using Cols = TcCols<N>;
    using Sm = FwdTcSmem<N>;
    constexpr int T = kTS, P = 128, TQ = T / 4, S = kStages;
    constexpr int NPROD = 512, NCONS = 128;
    extern __shared__ __align__(1024) float4 smem4[];
    Sm& sm = *reinterpret_cast<Sm*>(smem4);

    const int tid = threadIdx.x;
    const int warp = tid >> 5;
    const bool prod = tid < NPROD;
    const bool cons = !prod;
    // Producers: channel pch, token quarter pq.  Consumers: channel cch.
    const int pch = tid & (P - 1);
    const int pq = (tid >> 7) & 3;
    const int cch = tid - NPROD;
    const int ch = prod ? pch : cch;
    const int64_t Bt = p.Bt, L = p.L, d = p.d;

    // ------------------------------------------------------------ set-up
    if (warp == 0) {
        tc::tmem_alloc(&sm.taddr, Cols::ALLOC);
        tc::tmem_relinquish();
    }
    if (tid == 0) {
        sm.item = atomicAdd(&p.hdr->fwd_ticket, 1);
        for (int s = 0; s < S; ++s) {
            tc::mbar_init(&sm.loaded[s], 1);
            tc::mbar_init(&sm.full[s], NPROD);
            tc::mbar_init(&sm.empty[s], NCONS);
        }
        tc::mbar_init(&sm.mma, 1);
        tma::prefetch_map(&tm.u);
        tma::prefetch_map(&tm.a);
        if (p.b) tma::prefetch_map(&tm.b);
        if (p.z) tma::prefetch_map(&tm.z);
        tma::prefetch_map(&tm.B);
        tma::prefetch_map(&tm.C);
    }
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    const uint32_t tbase = sm.taddr;
    const uint32_t lane = (uint32_t)((warp & 3) * 32) << 16;  // this warp's TMEM lanes
    const int item = sm.item;
    const bool has_z = p.z != nullptr;
    const bool has_b = p.b != nullptr;  // absent: coupled single gate i = 1 - f
    // Work unit u = bb * ntiles + tile: 128 channels of one batch element,
    // over checkpoint segments [seg0, seg1).  Group mode: one (sequence group,
    // unit) per block.  Piece mode (PIECES): the units' segments, laid end to
    // end, are cut into npieces equal ranges, one per block; a block takes its
    // range's unit segments last first, so the head of a unit cut in two (the
    // last segment of the earlier range) runs first and publishes the state at
    // the cut for the tail (the first segment of the later range), which runs
    // last in a block that started after it.
    int g = 0, bb = 0, tile = 0, seg0 = 0, seg1 = 0;
    int64_t c0 = 0, c = 0, tbeg = 0, tend = 0;
    bool cvalid = false, last_group = true;
    Tout* gy = nullptr;
    float* ck_b = nullptr;
    float w0 = 0.f, w1 = 0.f, w2 = 0.f, w3 = 0.f, wb = 0.f, Dc = 0.f;
    auto set_unit = [&](int u, int g_, int s0, int s1) {
        g = g_;
        bb = u / p.ntiles;
        tile = u % p.ntiles;
        c0 = (int64_t)tile * P;
        c = c0 + ch;
        cvalid = c < d;
        seg0 = s0;
        seg1 = s1;
        tbeg = (int64_t)seg0 * p.T_ck;
        tend = min64(L, (int64_t)seg1 * p.T_ck);
        last_group = seg1 == p.nck;
        gy = static_cast<Tout*>(p.y) + (int64_t)bb * L * d;
        ck_b = p.ckpt + (int64_t)bb * (p.nck + 1) * d * N;
        w0 = w1 = w2 = w3 = wb = Dc = 0.f;
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
    };
    if (!PIECES) {
        const int per_g = (int)(Bt * p.ntiles);
        const int gg = item / per_g;
        const int s0 = gg * p.seg_per_group;
        set_unit(item % per_g, gg, s0, min(s0 + p.seg_per_group, p.nck));
    }
    const float scale = p.scale;
    bool timed_out = false;

    // ======================================================= producer side
    // One thread: TMA loads of sub-chunk t0 into raw buffer `buf`.
    auto issue = [&](int64_t t0, int buf, bool full) {
        typename Sm::Raw& r = sm.raw[buf];
        uint64_t* mb = &sm.loaded[buf];
        const bool zz = full && has_z;
        const uint32_t bytes =
            (uint32_t)sizeof(Tin) * ((T + 3) * P + (has_b ? 2 : 1) * T * P + (zz ? T * P : 0) +
                                     (full ? 2 : 1) * T * N);
        tma::expect_tx(mb, bytes);
        const int x = (int)c0, y = (int)t0, zb = bb;
        tma::load_3d(&r.u[0][0], &tm.u, x, y - 3, zb, mb);
        tma::load_3d(&r.a[0][0], &tm.a, x, y, zb, mb);
        if (has_b) tma::load_3d(&r.b[0][0], &tm.b, x, y, zb, mb);
        if (zz) tma::load_3d(&r.z[0][0], &tm.z, x, y, zb, mb);
        tma::load_3d(&r.Bm[0][0], &tm.B, 0, y, zb, mb);
        if (full) tma::load_3d(&r.Cm[0][0], &tm.C, 0, y, zb, mb);
    };
    auto bf4 = [](const __nv_bfloat16* src) {
        const uint2 raw = *reinterpret_cast<const uint2*>(src);
        const float2 lo = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&raw.x));
        const float2 hi = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&raw.y));
        return make_float4(lo.x, lo.y, hi.x, hi.y);
    };
    // Unpack sub-chunk (t0, raw buffer `buf`) into stage `s` (producers only).
    auto prep = [&](int64_t t0, int buf, int s, bool full) {
        const typename Sm::Raw& r = sm.raw[buf];
        typename Sm::Stage& stg = sm.st[s];
        // B and C rows to fp32 (padded rows: conflict-free reads below).
        for (int e = tid; e < T * N / 4; e += NPROD) {
            const int tt = e / (N / 4), j = (e % (N / 4)) * 4;
            *reinterpret_cast<float4*>(&stg.brow[tt][j]) = bf4(&r.Bm[tt][j]);
            if (full) *reinterpret_cast<float4*>(&stg.crow[tt][j]) = bf4(&r.Cm[tt][j]);
        }
        // Tokens of this thread's quarter inside [t0, tend) (0 for a padding channel).
        const int nv = cvalid ? (int)max((int64_t)0, min64((int64_t)TQ, tend - t0 - pq * TQ)) : 0;
        // Per-channel values: this thread's 4 tokens.
        float qv[TQ], fv[TQ], hv[TQ], ev[TQ];
        float Qh = 1.f, Eh = 1.f;
#pragma unroll
        for (int k = 0; k < TQ; ++k) {
            const int tt = pq * TQ + k;
            const bool valid = k < nv;
            ev[k] = valid ? __expf(-to_f(r.a[tt][pch])) : 0.f;
            qv[k] = 1.f + ev[k];
            fv[k] = rcpa_(qv[k]);
            Qh *= qv[k];
            Eh *= fv[k];
            float h;
            if (CONV) {
                h = silua_(wb + w0 * to_f(r.u[tt][pch]) + w1 * to_f(r.u[tt + 1][pch]) +
                           w2 * to_f(r.u[tt + 2][pch]) + w3 * to_f(r.u[tt + 3][pch]));
            } else {
                h = to_f(r.u[tt + 3][pch]);
            }
            hv[k] = valid ? h : 0.f;
        }
        sm.xq[pq][pch] = Qh;
        sm.xe[pq][pch] = Eh;
        // The exchange barrier also ORs a conservative per-quarter test; only
        // when it fires does the exact per-sub-chunk test below take a barrier.
        const bool maybe_slow = tc::named_bar_or(1, NPROD, !(Qh <= kTcQuarter));
        // decay products of the earlier quarters and of the whole sub-chunk
        float Qb = 1.f, Eb = 1.f, Qa = 1.f, Ea = 1.f;
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            const float xq = sm.xq[q][pch], xe = sm.xe[q][pch];
            if (q < pq) {
                Qb *= xq;
                Eb *= xe;
            }
            Qa *= xq;
            Ea *= xe;
        }
        const bool slow =
            maybe_slow && tc::named_bar_or(1, NPROD, pq == 0 && !(Qa <= kTcBound));
        if (!slow) {
            if (full && warp == 0) {
                // G[t][m] = C_t . B_m for m <= t: one warp, tf32 warp-level MMAs.
                float dd[2][4];
                tc::warp_gram16<N, N + 4>(&stg.crow[0][0], &stg.brow[0][0], dd);
                const int lane = tid & 31, gq = lane >> 2, kq = lane & 3;
#pragma unroll
                for (int n = 0; n < 2; ++n)
#pragma unroll
                    for (int r = 0; r < 4; ++r) {
                        const int row = gq + (r >> 1) * 8, col = 8 * n + 2 * kq + (r & 1);
                        stg.bg[tc::kmajor_offset(row, col, T) >> 2] = col <= row ? dd[n][r] : 0.f;
                    }
            } else {
                // K-major operand tiles (the other warps).  bc: a quarter warp
                // fills one 8-row core matrix; bs: one thread gathers 4
                // consecutive m of one row j.
                const int t2 = full ? tid - 32 : tid, n2 = full ? NPROD - 32 : NPROD;
                for (int e = t2; e < T * N / 4; e += n2) {
                    if (full) {
                        const int rest = e >> 3;
                        const int tt = (rest & 1) * 8 + (e & 7), j = (rest >> 1) * 4;
                        *reinterpret_cast<float4*>(&stg.bc[tc::kmajor_offset(tt, j, N) >> 2]) =
                            *reinterpret_cast<const float4*>(&stg.crow[tt][j]);
                    }
                    const int jj = e % N, m0 = (e / N) * 4;
                    *reinterpret_cast<float4*>(&stg.bs[tc::kmajor_offset(jj, m0, T) >> 2]) =
                        make_float4(stg.brow[m0][jj], stg.brow[m0 + 1][jj], stg.brow[m0 + 2][jj],
                                    stg.brow[m0 + 3][jj]);
                }
            }
        }
        const float Elast = Ea;
        float Q = Qb, E = Eb;
        float Wv[TQ], Vv[TQ], Gv[TQ], Dv[TQ];
#pragma unroll
        for (int k = 0; k < TQ; ++k) {
            const int tt = pq * TQ + k;
            const float iw = has_b ? sigmoida_(to_f(r.b[tt][pch])) : ev[k] * fv[k];
            const float v = iw * hv[k];  // 0 past the end (h = 0)
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
                const float gg = has_z ? silua_(to_f(r.z[tt][pch])) : 1.f;
                Gv[k] = slow ? scale * gg : scale * E * gg;
                Dv[k] = Dc * hv[k] * gg;
            }
        }
        if (pq == 0) stg.elast[pch] = Elast;
        if (tid == 0) stg.slow = slow ? 1 : 0;
        const uint32_t col = tbase + lane + s * T + pq * TQ;
        tc::tmem_st4(col + Cols::W, Wv);
        tc::tmem_st4(col + Cols::V, Vv);
        if (full) {
            tc::tmem_st4(col + Cols::EG, Gv);
            tc::tmem_st4(col + Cols::DH, Dv);
        }
        tc::tmem_st_wait();
    };

    // ======================================================= consumer side
    // Issue the sub-chunk's MMAs (one consumer thread) and commit them.
    auto issue_mma = [&](int s, bool full) {
        const typename Sm::Stage& stg = sm.st[s];
        constexpr uint32_t id_r = tc::idesc_tf32(128, T);
        constexpr uint32_t id_s = tc::idesc_tf32(128, N);
        if (full) {
            const uint32_t sc = tc::smem_u32(&stg.bc[0]);
#pragma unroll
            for (int ks = 0; ks < N / 8; ++ks)
                tc::mma_tf32_ts(tbase + Cols::DR, tbase + Cols::X + ks * 8,
                                tc::sdesc(sc + ks * 256, 128, 32 * N), id_r, ks > 0 ? 1u : 0u);
            const uint32_t sg = tc::smem_u32(&stg.bg[0]);
#pragma unroll
            for (int ks = 0; ks < T / 8; ++ks)
                tc::mma_tf32_ts(tbase + Cols::DR, tbase + Cols::W + s * T + ks * 8,
                                tc::sdesc(sg + ks * 256, 128, 32 * T), id_r, 1u);
        }
        const uint32_t ss = tc::smem_u32(&stg.bs[0]);
#pragma unroll
        for (int ks = 0; ks < T / 8; ++ks)
            tc::mma_tf32_ts(tbase + Cols::DS, tbase + Cols::V + s * T + ks * 8,
                            tc::sdesc(ss + ks * 256, 128, 32 * T), id_s, ks > 0 ? 1u : 0u);
        tc::mma_commit(&sm.mma);
    };
    // TMEM state row <-> global row (consumers; full rows).
    auto state_from = [&](const float* src, bool cg) {
#pragma unroll
        for (int n0 = 0; n0 < N; n0 += 16) {
            float v[16];
#pragma unroll
            for (int k = 0; k < 16; k += 4) {
                float4 v4 = make_float4(0.f, 0.f, 0.f, 0.f);
                if (src && cvalid) {
                    const float4* s4 = reinterpret_cast<const float4*>(src + c * N + n0 + k);
                    v4 = cg ? __ldcg(s4) : *s4;
                }
                v[k] = v4.x;
                v[k + 1] = v4.y;
                v[k + 2] = v4.z;
                v[k + 3] = v4.w;
            }
            tc::tmem_st16(tbase + lane + Cols::X + n0, v);
        }
        tc::tmem_st_wait();
    };
    auto state_to = [&](float* dst) {
#pragma unroll
        for (int n0 = 0; n0 < N; n0 += 16) {
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
    float logP = 0.f;  // log of the decay product over the pass (consumers)
    auto epilogue = [&](int64_t t0, int s, bool full) {
        const typename Sm::Stage& stg = sm.st[s];
        const int ny = cvalid ? (int)min64((int64_t)T, tend - t0) : 0;  // outputs to write
        Tout* yrow = gy + t0 * d + c;
        if (!stg.slow) {
            const float El = stg.elast[cch];
            if (full) {
                float dr[16], eg[16], dh[16];
                tc::tmem_ld16(tbase + lane + Cols::DR, dr);
                tc::tmem_ld16(tbase + lane + Cols::EG + s * T, eg);
                tc::tmem_ld16(tbase + lane + Cols::DH + s * T, dh);
                tc::tmem_ld_wait();
#pragma unroll
                for (int tt = 0; tt < T; ++tt)
                    if (tt < ny) yrow[tt * d] = from_f<Tout>(fmaf(eg[tt], dr[tt], dh[tt]));
            }
#pragma unroll
            for (int n0 = 0; n0 < N; n0 += 16) {
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
            // Exact path: x <- f x + (i h) B token by token, y from x . C.
            float vv[16], ff[16], yp[16];
            tc::tmem_ld16(tbase + lane + Cols::W + s * T, vv);
            tc::tmem_ld16(tbase + lane + Cols::V + s * T, ff);
            tc::tmem_ld_wait();
#pragma unroll
            for (int tt = 0; tt < T; ++tt) yp[tt] = 0.f;
            for (int n0 = 0; n0 < N; n0 += 16) {
                float x[16];
                tc::tmem_ld16(tbase + lane + Cols::X + n0, x);
                tc::tmem_ld_wait();
#pragma unroll
                for (int tt = 0; tt < T; ++tt) {
                    float acc = 0.f;
#pragma unroll
                    for (int k = 0; k < 16; ++k) {
                        x[k] = fmaf(ff[tt], x[k], vv[tt] * stg.brow[tt][n0 + k]);
                        if (full) acc = fmaf(x[k], stg.crow[tt][n0 + k], acc);
                    }
                    yp[tt] += acc;
                }
                tc::tmem_st16(tbase + lane + Cols::X + n0, x);
            }
            if (full) {
                float eg[16], dh[16];
                tc::tmem_ld16(tbase + lane + Cols::EG + s * T, eg);
                tc::tmem_ld16(tbase + lane + Cols::DH + s * T, dh);
                tc::tmem_ld_wait();
#pragma unroll
                for (int tt = 0; tt < T; ++tt)
                    if (tt < ny) yrow[tt * d] = from_f<Tout>(fmaf(eg[tt], yp[tt], dh[tt]));
            }
            float lp = 0.f;
#pragma unroll
            for (int tt = 0; tt < T; ++tt) lp += __logf(ff[tt]);
            logP += lp;
        }
        tc::tmem_st_wait();
    };

    // ============================================================ one pass
    int gbase = 0;           // sub-chunks through the stage ring so far
    uint32_t mma_phase = 0;  // consumers: parity of the next MMA completion
    auto run_pass = [&](bool full) {
        const int nsc = (int)((tend - tbeg + T - 1) / T);
        if (prod) {
            // Raw buffer and operand stage of sub-chunk gi are both gi % S.
            if (tid == 0) {
                issue(tbeg, gbase % S, full);
                if (nsc > 1) issue(tbeg + T, (gbase + 1) % S, full);
            }
            for (int i = 0; i < nsc; ++i) {
                const int gi = gbase + i, s = gi % S, u = gi / S;
                const int64_t t0 = tbeg + (int64_t)i * T;
                if (tid == 0 && i + 2 < nsc) {
                    // Buffer (gi + 2) % S held sub-chunk gi - 1: refill it once
                    // every producer has unpacked that one (its full barrier).
                    if (i > 0 && !tc::mbar_wait(&sm.full[(gi - 1) % S], ((gi - 1) / S) & 1,
                                                kMbarSpin))
                        timed_out = true;
                    issue(t0 + 2 * T, (gi + 2) % S, full);
                }
                if (!tc::mbar_wait(&sm.loaded[s], u & 1, kMbarSpin)) timed_out = true;
                if (u > 0 && !tc::mbar_wait(&sm.empty[s], (u - 1) & 1, kMbarSpin)) timed_out = true;
                prep(t0, s, s, full);
                tc::fence_proxy_async();
                tc::fence_before_sync();
                tc::mbar_arrive(&sm.full[s]);
            }
        } else {
            for (int i = 0; i < nsc; ++i) {
                const int gi = gbase + i, s = gi % S;
                const int64_t t0 = tbeg + (int64_t)i * T;
                if (i == 0) {
                    if (!tc::mbar_wait(&sm.full[s], (gi / S) & 1, kMbarSpin)) timed_out = true;
                    tc::fence_after_sync();
                    if (cch == 0 && !sm.st[s].slow) issue_mma(s, full);
                }
                if (!sm.st[s].slow) {
                    if (!tc::mbar_wait(&sm.mma, mma_phase, kMbarSpin)) timed_out = true;
                    mma_phase ^= 1u;
                }
                tc::fence_after_sync();
                epilogue(t0, s, full);
                if (full) {
                    const int64_t tnext = t0 + T;
                    if (tnext < tend && tnext % p.T_ck == 0)
                        state_to(ck_b + (tnext / p.T_ck) * d * N);
                }
                tc::fence_before_sync();
                tc::mbar_arrive(&sm.empty[s]);
                if (i + 1 < nsc) {
                    const int gn = gi + 1, sn = gn % S;
                    if (!tc::mbar_wait(&sm.full[sn], (gn / S) & 1, kMbarSpin)) timed_out = true;
                    tc::named_bar(2, NCONS);  // every X row updated
                    if (cch == 0) {
                        tc::fence_after_sync();
                        if (!sm.st[sn].slow) issue_mma(sn, full);
                    }
                }
            }
        }
        gbase += nsc;
        tc::fence_before_sync();
        __syncthreads();
        tc::fence_after_sync();
    };

    auto sync_all = [&]() {
        tc::fence_before_sync();
        __syncthreads();
        tc::fence_after_sync();
    };
    if (PIECES) {
        // ----------------------------------------------- piece mode
        const int64_t Wb = Bt * p.ntiles * (int64_t)p.nck;
        const int64_t F0 = (int64_t)item * Wb / p.npieces;
        const int64_t F1 = (int64_t)(item + 1) * Wb / p.npieces;
        const int64_t ub_lo = (F0 / p.nck) * p.nck;
        for (int64_t ub = ((F1 - 1) / p.nck) * p.nck; ub >= ub_lo; ub -= p.nck) {
            const int s0 = (int)(max64(F0, ub) - ub), s1 = (int)(min64(F1, ub + p.nck) - ub);
            set_unit((int)(ub / p.nck), 0, s0, s1);
            int* flag_cut = p.flags + (int64_t)bb * p.ntiles + tile;
            if (s0 == 0) {
                if (cons) {
                    state_from(p.x0 ? p.x0 + (int64_t)bb * d * N : nullptr, false);
                    state_to(ck_b);  // checkpoint 0 = initial state
                }
            } else {
                // tail of a cut unit: the state at the cut from its head
                if (tid == 0) sm.ok = wait_flag(flag_cut, &p.hdr->status, p.wait_limit) ? 1 : 0;
                __syncthreads();
                if (cons) state_from(sm.ok ? ck_b + (int64_t)s0 * d * N : nullptr, true);
            }
            sync_all();
            run_pass(true);
            if (cons) {
                state_to(ck_b + (int64_t)s1 * d * N);
                if (s1 == p.nck && p.x_final) state_to(p.x_final + (int64_t)bb * d * N);
            }
            if (s1 < p.nck) {  // head of a cut unit: publish the state at the cut
                __threadfence();
                __syncthreads();
                if (tid == 0 && !p.fault_skip_publish) st_release(flag_cut, 1);
            }
            sync_all();
        }
    } else {
        // ------------------------------------------ early pass and carry chain
        const float* x0b = p.x0 ? p.x0 + (int64_t)bb * d * N : nullptr;
        const int* flag_prev = (g > 0) ? p.flags + ((int64_t)(g - 1) * Bt + bb) * p.ntiles + tile
                                       : nullptr;
        int* flag_mine = p.flags + ((int64_t)g * Bt + bb) * p.ntiles + tile;
        float* ck_start = ck_b + (int64_t)seg0 * d * N;
        float* ck_end = ck_b + (int64_t)seg1 * d * N;
        bool ok = true;
        if (!last_group) {
            if (cons) state_from(g == 0 ? x0b : nullptr, false);
            sync_all();
            run_pass(false);
            if (g > 0) {
                if (tid == 0) sm.ok = wait_flag(flag_prev, &p.hdr->status, p.wait_limit) ? 1 : 0;
                __syncthreads();
                ok = sm.ok != 0;
                if (cons) {
                    // X_end += (product of f over the group) X_start
                    const float Pf = __expf(logP);
#pragma unroll
                    for (int n0 = 0; n0 < N; n0 += 16) {
                        float x[16];
                        tc::tmem_ld16(tbase + lane + Cols::X + n0, x);
                        tc::tmem_ld_wait();
#pragma unroll
                        for (int k = 0; k < 16; k += 4) {
                            float4 v4 = make_float4(0.f, 0.f, 0.f, 0.f);
                            if (ok && cvalid)
                                v4 = __ldcg(reinterpret_cast<const float4*>(ck_start + c * N +
                                                                            n0 + k));
                            x[k] = fmaf(Pf, v4.x, x[k]);
                            x[k + 1] = fmaf(Pf, v4.y, x[k + 1]);
                            x[k + 2] = fmaf(Pf, v4.z, x[k + 2]);
                            x[k + 3] = fmaf(Pf, v4.w, x[k + 3]);
                        }
                        tc::tmem_st16(tbase + lane + Cols::X + n0, x);
                    }
                    tc::tmem_st_wait();
                }
            }
            if (cons) state_to(ck_end);
            __threadfence();
            __syncthreads();
            if (tid == 0 && !(g == 0 && p.fault_skip_publish)) st_release(flag_mine, 1);
        } else if (g > 0) {
            if (tid == 0) sm.ok = wait_flag(flag_prev, &p.hdr->status, p.wait_limit) ? 1 : 0;
            __syncthreads();
            ok = sm.ok != 0;
        }
        if (cons) {
            if (g > 0) {
                state_from(ok ? ck_start : nullptr, true);
            } else {
                state_from(x0b, false);
                state_to(ck_b);  // checkpoint 0 = initial state
            }
        }
        sync_all();

        // ------------------------------------------------------- full pass
        run_pass(true);
        if (last_group && cons) {
            state_to(ck_b + (int64_t)p.nck * d * N);
            if (p.x_final) state_to(p.x_final + (int64_t)bb * d * N);
        }
    }
    if (timed_out) atomicOr(&p.hdr->status, 1 << NAJU_ERR_TIMEOUT);

    // ---------------------------------------------------------- teardown
    sync_all();
    if (warp == 0) tc::tmem_dealloc(tbase, Cols::ALLOC);
}

template <typename Tout, int N, bool CONV, bool PIECES>
static cudaError_t launch_fwd_tc_t(const FwdParams& p, cudaStream_t st) {
    FwdTmaps tm;
    memset(&tm, 0, sizeof(tm));
    const int T = kTS;
    bool ok = tma_encode_bf16_3d(&tm.u, p.hu, p.Bt, p.L, p.d, T + 3, 128) &&
              tma_encode_bf16_3d(&tm.a, p.a, p.Bt, p.L, p.d, T, 128) &&
              (!p.b || tma_encode_bf16_3d(&tm.b, p.b, p.Bt, p.L, p.d, T, 128)) &&
              tma_encode_bf16_3d(&tm.B, p.B, p.Bt, p.L, N, T, N) &&
              tma_encode_bf16_3d(&tm.C, p.C, p.Bt, p.L, N, T, N);
    if (ok && p.z) ok = tma_encode_bf16_3d(&tm.z, p.z, p.Bt, p.L, p.d, T, 128);
    if (!ok) return cudaErrorInvalidValue;
    const size_t smem = sizeof(FwdTcSmem<N>);
    auto kern = scan_fwd_tc_kernel<Tout, N, CONV, PIECES>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)smem);
    if (e != cudaSuccess) return e;
    const int grid = PIECES ? p.npieces : p.ngroups * (int)p.Bt * p.ntiles;
    kern<<<grid, 640, smem, st>>>(p, tm);
    return cudaGetLastError();
}

int fwd_tc_channels_per_block() { return 128; }

bool fwd_tc_supported(int dtype, int64_t N, int64_t d) {
    // TMA rows must be a multiple of 16 bytes: d_inner % 8 == 0.
    return dtype == NAJU_BF16 && (N == 64 || N == 128) && d % 8 == 0;
}

cudaError_t launch_scan_fwd_tc(const FwdParams& p, int out_dtype, cudaStream_t st) {
    const bool conv = p.conv_w != nullptr;
    const bool pc = p.npieces > 0;
#define NAJU_TC_FWD(TO, NN)                                                          \
    return conv ? (pc ? launch_fwd_tc_t<TO, NN, true, true>(p, st)                   \
                      : launch_fwd_tc_t<TO, NN, true, false>(p, st))                 \
                : (pc ? launch_fwd_tc_t<TO, NN, false, true>(p, st)                  \
                      : launch_fwd_tc_t<TO, NN, false, false>(p, st))
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
