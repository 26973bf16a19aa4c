// Naju forward scan in block form on the 5th-generation tensor cores
// (sm_100a, tcgen05, kind::f16 with fp32 accumulation), for bf16 activations
// with d_state 64 or 128.
//
// Same computation as the CUDA-core forward (Naju reproduction README, "Core
// equations"): x_n = f_n x_{n-1} + i_n h_n B_n^T, y_n = x_n.C_n/sqrt(N) + D h_n,
// out_n = y_n SiLU(z_n), h = SiLU(conv(u)).
//
// A thread block owns 128 channels of one batch element (one channel per
// tensor-memory lane) and walks its tokens in blocks of 64, the spacing of
// the checkpoints it writes for the backward.  With X the state entering a
// block (kept in tensor memory for the whole pass), per channel
// E_t = prod_{k<=t} f_k from the block start, Q_t = 1/E_t, W_t = i_t h_t Q_t and
// G[t][m] = C_t.B_m kept for m <= t:
//   y_t  = s E_t R_t SiLU(z_t) + D h_t SiLU(z_t),   R = X C^T + W G^T
//   X'   = E_63 (X + S),                            S = W B
// All three products run on the tensor core.  Each fp32 operand (X, W, G) is
// a pair of bf16 tiles hi = bf16(v), lo = bf16(v - hi) and a product takes
// hi.hi + hi.lo + lo.hi (about 2^-16 relative error; B and C are bf16 inputs,
// exact in one tile), so the state handed from block to block - and the
// checkpoints the backward starts from - keep nearly fp32 accuracy.  The
// tiles are 128-byte swizzled row tiles; for 16-bit data the same bytes serve
// as the K-major operand and as the MN-major one (B in S = W B).
//
// The raw inputs of a block (u with its 3-token conv halo, a, b, z) arrive by
// TMA into one shared buffer, requested once the previous block has read its
// own and issued its products; B and C arrive by TMA straight into their
// swizzled tiles once the previous block's products are done.  With d_state
// 64 a block's y and fp32 checkpoint leave through staging tiles and TMA
// stores (a warp's checkpoint rows are 256 bytes apart: direct stores would
// cost one memory transaction per lane); with d_state 128 the checkpoint is
// stored directly in 32-byte pieces.  Everything per (token, channel) runs on
// the CUDA cores, 512 threads: warp w handles channels 32 (w % 4) + lane and
// tokens [16 q, 16 q + 16) of the block, q = w / 4, and the state columns
// [q N / 4, (q + 1) N / 4).
//
// Exactness.  A block where some channel's decay product over the block
// falls below 2^-90 runs the plain recurrence token by token instead.
//
// Work split: piece mode (at least one wave of 128-channel units) gives each
// thread block one equal range of the units' 64-token blocks, a unit cut in
// two handing the state at the cut from its head to its tail; below one wave
// sequence groups run an update-only pass and a decoupled look-back first.
#include <stddef.h>
#include <string.h>

#include <type_traits>

#include "naju_common.cuh"
#include "naju_kernels.h"
#include "naju_tc.cuh"
#include "naju_tma.h"

namespace naju {

namespace {

constexpr int kK = 64;
constexpr int kP = 128;
constexpr int kNT = 512;
constexpr float kBound = 1.2379400392853803e27f;  // 2^90
constexpr float kQuarter = 4194304.f;             // 2^22
constexpr long long kSpin = 1LL << 24;
constexpr float kLog2e = 1.4426950408889634f;

template <int N>
struct FkCols {
    static constexpr uint32_t X = 0;             // state [ch][j]
    static constexpr uint32_t S = N;             // W B   [ch][j]
    static constexpr uint32_t R = 2 * N;         // R     [ch][t]
    static constexpr uint32_t G = 2 * N + 64;    // G^T (M = 64): t' < 32 at lanes +0, >= 32 at +16
    static constexpr uint32_t SV = 2 * N + 128;  // s E SiLU(z), D h SiLU(z)  [ch][t] x 2
    static constexpr uint32_t USED = 2 * N + 256;
    static constexpr uint32_t ALLOC = USED <= 256 ? 256 : 512;
    static_assert(USED <= 512, "tensor memory");
};

struct alignas(64) FkTmaps {
    CUtensorMap u, a, b, z;  // bf16 [Bt][L][d], plain boxes of 128 channels
    CUtensorMap B, C;        // bf16 [Bt][L][N], swizzled boxes of 64 columns
    CUtensorMap y;           // bf16 output [Bt][L][d] (bf16 outputs only), store boxes
    CUtensorMap ck;          // fp32 checkpoints [Bt (nck + 1)][d][N], swizzled boxes of
                             // 128 x 32 (d_state 64 only)
};

template <int N>
struct FkSmem {
    alignas(1024) __nv_bfloat16 Wh[kP * kK], Wl[kP * kK];  // rows ch, cols t
    alignas(1024) __nv_bfloat16 Xh[kP * N], Xl[kP * N];    // rows ch, cols j
    // B (rows t, cols j) and the hi tile of G^T (rows m, cols t', m <= t') side by
    // side: one MN-major operand [B | G^T] of N + 64 columns for S and R together
    alignas(1024) __nv_bfloat16 Bs[kK * N], GTh[kK * kK];
    alignas(1024) __nv_bfloat16 Cs[kK * N], GTl[kK * kK];  // C: rows t, cols j
    alignas(1024) __nv_bfloat16 ru[(kK + 3) * kP];         // u of tokens tb - 3 ..
    alignas(128) __nv_bfloat16 ra[kK * kP], rb[kK * kP], rz[kK * kP];
    // d_state 64: a block's fp32 checkpoint (two swizzled 128 x 32 boxes) and
    // its bf16 y are staged here and leave by TMA stores after the next
    // block's first barrier (d_state 128: y staged over the W tiles, the
    // checkpoint stored directly)
    alignas(1024) float ck[N == 64 ? kP * N : 32];
    alignas(128) __nv_bfloat16 ys[N == 64 ? kK * kP : 64];
    float xq[4][kP], xe[4][kP];
    uint64_t mb_raw, mb_bc, mb0, mb2;
    uint32_t taddr;
    int item, ok;
};

__device__ __forceinline__ float bf2f(__nv_bfloat16 v) {
    return __uint_as_float((uint32_t)__bfloat16_as_ushort(v) << 16);
}
// hi = bf16(v), lo = bf16(v - hi) for two values, packed.
__device__ __forceinline__ void split2(float a, float b, uint32_t& hi, uint32_t& lo) {
    const __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
    const float2 hf = __bfloat1622float2(h);
    const __nv_bfloat162 l = __floats2bfloat162_rn(a - hf.x, b - hf.y);
    hi = *reinterpret_cast<const uint32_t*>(&h);
    lo = *reinterpret_cast<const uint32_t*>(&l);
}
// Eight consecutive values (row, col .. col + 7; col % 8 == 0) into a tile
// pair of R rows: one 16-byte chunk in each.
__device__ __forceinline__ void st8(__nv_bfloat16* th, __nv_bfloat16* tl, int row, int col, int R,
                                    const float* v) {
    uint4 h, l;
    split2(v[0], v[1], h.x, l.x);
    split2(v[2], v[3], h.y, l.y);
    split2(v[4], v[5], h.z, l.z);
    split2(v[6], v[7], h.w, l.w);
    const uint32_t o = tc::bf_offset_w(row, col, R);
    *reinterpret_cast<uint4*>(reinterpret_cast<char*>(th) + o) = h;
    *reinterpret_cast<uint4*>(reinterpret_cast<char*>(tl) + o) = l;
}
// Eight floats to global memory in one 32-byte store (p 32-byte aligned):
// a warp's state rows are N * 4 bytes apart, so each lane's store is a
// transaction of its own, and whole 32-byte sectors halve their count.
__device__ __forceinline__ void st_v8(float* p, const float* v) {
    asm volatile("st.global.v8.f32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8};" ::"l"(p), "f"(v[0]),
                 "f"(v[1]), "f"(v[2]), "f"(v[3]), "f"(v[4]), "f"(v[5]), "f"(v[6]), "f"(v[7])
                 : "memory");
}
__device__ __forceinline__ float ld1(const __nv_bfloat16* t, int row, int col, int R) {
    return bf2f(*reinterpret_cast<const __nv_bfloat16*>(reinterpret_cast<const char*>(t) +
                                                          tc::bf_offset_w(row, col, R)));
}

}  // namespace

template <typename Tout, int N, bool CONV, bool PIECES>
__global__ void __launch_bounds__(512, 1)
scan_fwd_blk_kernel(const FwdParams p, const __grid_constant__ FkTmaps tm) {
    using Cols = FkCols<N>;
    using Sm = FkSmem<N>;
    constexpr int NQ = N / 4;  // state columns per thread
    // bf16 outputs are staged in shared memory and leave by one TMA store per
    // block; fp32 outputs are stored directly
    constexpr bool kStageY = std::is_same<Tout, __nv_bfloat16>::value;
    // d_state 64: own staging buffers for y and the checkpoint (room in shared
    // memory), so neither waits on the W tiles nor stores 256-byte-strided rows
    constexpr bool kOwnStage = N == 64;
    static_assert(offsetof(Sm, GTh) == offsetof(Sm, Bs) + sizeof(Sm::Bs) &&
                      sizeof(Sm::Bs) == (size_t)(N / 64) * kK * 128,
                  "B and G^T are one MN-major operand: 64-column blocks kK * 128 bytes apart");
    static_assert(Cols::R == Cols::S + N, "S and R are one accumulator [S | R]");
    const float kZero16[16] = {};
    static_assert(sizeof(Sm::Xh) + sizeof(Sm::Xl) >= kK * kP * sizeof(float),
                  "the exact path's row sums live over the X tiles");
    extern __shared__ __align__(1024) float4 smem4[];
    Sm& sm = *reinterpret_cast<Sm*>(smem4);

    const int tid = threadIdx.x;
    const int warp = tid >> 5, lid = tid & 31;
    const int s4 = warp & 3, q = warp >> 2;
    const int ch = s4 * 32 + lid;
    const int64_t Bt = p.Bt, L = p.L, d = p.d;
    const float sc = p.scale;
    const bool has_z = p.z != nullptr;
    const bool has_b = p.b != nullptr;

    if (warp == 0) {
        tc::tmem_alloc(&sm.taddr, Cols::ALLOC);
        tc::tmem_relinquish();
    }
    if (tid == 0) {
        sm.item = atomicAdd(&p.hdr->fwd_ticket, 1);
        tc::mbar_init(&sm.mb_raw, 1);
        tc::mbar_init(&sm.mb_bc, 1);
        tc::mbar_init(&sm.mb0, 1);
        tc::mbar_init(&sm.mb2, 1 + N / 64);  // R (warp 0), S by 64 columns (warps 1, 2)
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        tma::prefetch_map(&tm.u);
        tma::prefetch_map(&tm.a);
        if (has_b) tma::prefetch_map(&tm.b);
        if (has_z) tma::prefetch_map(&tm.z);
        tma::prefetch_map(&tm.B);
        tma::prefetch_map(&tm.C);
        if (kStageY) tma::prefetch_map(&tm.y);
    }
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    const uint32_t tbase = sm.taddr;
    const uint32_t trow = tbase + ((uint32_t)(s4 * 32) << 16);
    const int item = sm.item;
    const uint32_t sbase = tc::smem_u32(&sm);
// tile start addresses / 16 (the base is 1024-byte aligned: checked below)
#define NAJU_SA(f) (sb4 + (uint32_t)(offsetof(Sm, f) >> 4))
    const uint32_t sb4 = sbase >> 4;
    uint32_t ph_raw = 0, ph_bc = 0, ph0 = 0, ph2 = 0;
    bool timed_out = false;

    int bb = 0, tile = 0, seg0 = 0, seg1 = 0;
    int64_t c0 = 0, c = 0;
    bool cvalid = false;
    float w0 = 0.f, w1 = 0.f, w2 = 0.f, w3 = 0.f, wb = 0.f, Dc = 0.f;
    auto set_unit = [&](int u, int s0, int s1) {
        bb = u / p.ntiles;
        tile = u % p.ntiles;
        c0 = (int64_t)tile * kP;
        c = c0 + ch;
        cvalid = c < d;
        seg0 = s0;
        seg1 = s1;
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
    auto ck_at = [&](int k) { return p.ckpt + ((int64_t)bb * (p.nck + 1) + k) * d * N; };
    auto sync = [&]() {
        tc::fence_before_sync();
        __syncthreads();
        tc::fence_after_sync();
    };
    auto wait_mb = [&](uint64_t* mb, uint32_t& ph) {
        // one warp polls (until a first time-out); the others wait at the barrier
        if (warp == kNT / 32 - 1 && !timed_out && !tc::mbar_wait(mb, ph, kSpin)) timed_out = true;
        __syncthreads();
        ph ^= 1u;
        tc::fence_after_sync();
    };

    // ------------------------------------------------------- TMA issue
    // Raw per-token inputs of block k (thread 0; z only when full).
    auto load_raw = [&](int k, bool full) {
        const bool zz = full && has_z;
        const uint32_t rows = (kK + 3) + kK * (1 + (has_b ? 1 : 0) + (zz ? 1 : 0));
        tma::expect_tx(&sm.mb_raw, rows * kP * 2u);
        const int x = (int)c0, y = k * kK, zb = bb;
        tma::load_3d(sm.ru, &tm.u, x, y - 3, zb, &sm.mb_raw);
        tma::load_3d(sm.ra, &tm.a, x, y, zb, &sm.mb_raw);
        if (has_b) tma::load_3d(sm.rb, &tm.b, x, y, zb, &sm.mb_raw);
        if (zz) tma::load_3d(sm.rz, &tm.z, x, y, zb, &sm.mb_raw);
    };
    // B (and C when full) of block k into their tiles (thread 0).
    auto load_bc = [&](int k, bool full) {
        tma::expect_tx(&sm.mb_bc, (uint32_t)(2 * kK * N * (full ? 2 : 1)));
        const int y = k * kK, zb = bb;
#pragma unroll
        for (int jb = 0; jb < N / 64; ++jb) {
            tma::load_3d(sm.Bs + jb * kK * 64, &tm.B, jb * 64, y, zb, &sm.mb_bc);
            if (full) tma::load_3d(sm.Cs + jb * kK * 64, &tm.C, jb * 64, y, zb, &sm.mb_bc);
        }
    };

    // This thread's state columns: global [d][N] row -> tensor memory.
    auto state_from = [&](const float* src, bool cg) {
        float v[NQ];
#pragma unroll
        for (int k = 0; k < NQ; k += 4) {
            float4 v4 = make_float4(0.f, 0.f, 0.f, 0.f);
            if (src && cvalid) {
                const float4* s4p = reinterpret_cast<const float4*>(src + c * N + NQ * q + k);
                v4 = cg ? __ldcg(s4p) : *s4p;
            }
            v[k] = v4.x; v[k + 1] = v4.y; v[k + 2] = v4.z; v[k + 3] = v4.w;
        }
#pragma unroll
        for (int k = 0; k < NQ; k += 16) tc::tmem_st16(trow + Cols::X + NQ * q + k, &v[k]);
        tc::tmem_st_wait();
    };
    // This thread's state columns from tensor memory to a global [d][N] row
    // (dst != null) and to the X tile pair (tiles).
    auto state_out = [&](float* dst, bool tiles) {
#pragma unroll
        for (int k = 0; k < NQ; k += 16) {
            float v[16];
            tc::tmem_ld16(trow + Cols::X + NQ * q + k, v);
            tc::tmem_ld_wait();
            if (dst && cvalid) {
                st_v8(dst + c * N + NQ * q + k, v);
                st_v8(dst + c * N + NQ * q + k + 8, v + 8);
            }
            if (tiles) {
                st8(sm.Xh, sm.Xl, ch, NQ * q + k, kP, v);
                st8(sm.Xh, sm.Xl, ch, NQ * q + k + 8, kP, v + 8);
            }
        }
    };

    // ------------------------------------------------- decays (loop 1)
    float fv[16], qv[16];
    float Eb = 1.f, Qb = 1.f, E63 = 1.f;
    // Tokens past the end (last block only) decay by 1; channels past d
    // read zeros (their values are finite and never stored).
    auto decays = [&](int nv) -> bool {
        const __nv_bfloat16* rap = sm.ra + 16 * q * kP + ch;
        float Qh = 1.f, Eh = 1.f;
        if (nv == kK) {
#pragma unroll
            for (int k = 0; k < 16; ++k) {
                qv[k] = 1.f + expa_(-bf2f(rap[k * kP]));
                fv[k] = rcpa_(qv[k]);
                Qh *= qv[k];
                Eh *= fv[k];
            }
        } else {
            const int nq = nv - 16 * q;
#pragma unroll
            for (int k = 0; k < 16; ++k) {
                qv[k] = k < nq ? 1.f + expa_(-bf2f(rap[k * kP])) : 1.f;
                fv[k] = k < nq ? rcpa_(qv[k]) : 1.f;
                Qh *= qv[k];
                Eh *= fv[k];
            }
        }
        sm.xq[q][ch] = Qh;
        sm.xe[q][ch] = Eh;
        const bool maybe = __syncthreads_or(!(Qh <= kQuarter)) != 0;
        float Qa = 1.f, Ea = 1.f;
        Qb = 1.f;
        Eb = 1.f;
#pragma unroll
        for (int qq = 0; qq < 4; ++qq) {
            const float xq = sm.xq[qq][ch], xe = sm.xe[qq][ch];
            if (qq < q) {
                Qb *= xq;
                Eb *= xe;
            }
            Qa *= xq;
            Ea *= xe;
        }
        E63 = Ea;
        return maybe && __syncthreads_or(!(Qa <= kBound)) != 0;
    };
    // ------------------------------------------------- unpack (loop 2)
    // W to its tile pair; full: s E SiLU(z) and D h SiLU(z) to tensor memory.
    // slow (exact path): E = Q = 1, so W = i h.  W of a token past the end
    // meets only zero rows of B (and of G), so no token mask is needed here.
    auto unpack_v = [&](bool slow, bool full, auto hb_c, auto hz_c) {
        constexpr bool has_b = decltype(hb_c)::value;
        constexpr bool has_z = decltype(hz_c)::value;  // (z read only in a full pass)
        const __nv_bfloat16* rup = sm.ru + 16 * q * kP + ch;  // row i: token 16 q - 3 + i
        const __nv_bfloat16* rbp = sm.rb + 16 * q * kP + ch;
        const __nv_bfloat16* rzp = sm.rz + 16 * q * kP + ch;
        float E = slow ? sc : sc * Eb, Q = slow ? 1.f : Qb;  // E carries the scale s
        float u0 = 0.f, u1 = 0.f, u2 = 0.f;
        if (CONV) {
            u0 = bf2f(rup[0]);
            u1 = bf2f(rup[kP]);
            u2 = bf2f(rup[2 * kP]);
        }
#pragma unroll
        for (int g8 = 0; g8 < 2; ++g8) {
            float Wv[8], s0[8], s1[8];
#pragma unroll
            for (int h4 = 0; h4 < 2; ++h4) {
                const int kb = 8 * g8 + 4 * h4;  // first of four tokens
                // SiLU(conv), sigma(b) and SiLU(z) share one reciprocal:
                // q = 1 + e^{-v} with e^{-v} capped at 2^36 (the product stays
                // finite; a sigmoid below 1.5e-11 moves by at most that much),
                // r = 1 / (qp qb qz), sigma_p = r qb qz and so on.  With bf16
                // outputs SiLU(z), which only scales y, comes from the MUFU tanh
                // instead (error at most about 2^-12 |z|, below y's own bf16
                // rounding) and leaves the reciprocal to the other two.
                float pv[4], qp[4], qb[4], qz[4], zv[4], gz[4];
#pragma unroll
                for (int k4 = 0; k4 < 4; ++k4) {
                    const float u3 = bf2f(rup[(kb + k4 + 3) * kP]);
                    if (CONV) {
                        pv[k4] = fmaf(w3, u3, fmaf(w2, u2, fmaf(w1, u1, fmaf(w0, u0, wb))));
                        qp[k4] = 1.f + exp2a_(fminf(-kLog2e * pv[k4], 36.f));
                        u0 = u1;
                        u1 = u2;
                        u2 = u3;
                    } else {
                        pv[k4] = u3;
                        qp[k4] = 1.f;
                    }
                }
                if (has_b) {
#pragma unroll
                    for (int k4 = 0; k4 < 4; ++k4)
                        qb[k4] = 1.f + exp2a_(fminf(-kLog2e * bf2f(rbp[(kb + k4) * kP]), 36.f));
                } else {
#pragma unroll
                    for (int k4 = 0; k4 < 4; ++k4) qb[k4] = 1.f;
                }
                if (full && has_z) {
#pragma unroll
                    for (int k4 = 0; k4 < 4; ++k4) {
                        zv[k4] = bf2f(rzp[(kb + k4) * kP]);
                        if (kStageY) {
                            gz[k4] = siluta_(zv[k4]);
                            qz[k4] = 1.f;
                        } else {
                            qz[k4] = 1.f + exp2a_(fminf(-kLog2e * zv[k4], 36.f));
                        }
                    }
                } else {
#pragma unroll
                    for (int k4 = 0; k4 < 4; ++k4) {
                        zv[k4] = 1.f;
                        qz[k4] = 1.f;
                    }
                }
                float hv[4], iw[4], gg[4];
#pragma unroll
                for (int k4 = 0; k4 < 4; ++k4) {
                    const float qbz = qb[k4] * qz[k4];
                    const float r = rcpa_(qp[k4] * qbz);
                    hv[k4] = CONV ? pv[k4] * (r * qbz) : pv[k4];
                    const float rp = r * qp[k4];
                    if (has_b) {
                        iw[k4] = rp * qz[k4];
                    } else {
                        // coupled: i = 1 - f = (1/f - 1) f (1 where exp(-a) overflowed)
                        const float qq = qv[kb + k4];
                        iw[k4] = qq < 3.0e38f ? (qq - 1.f) * fv[kb + k4] : 1.f;
                    }
                    gg[k4] = (full && has_z) ? (kStageY ? gz[k4] : zv[k4] * (rp * qb[k4])) : 1.f;
                }
#pragma unroll
                for (int k4 = 0; k4 < 4; ++k4) {
                    const int k = kb + k4;
                    if (!slow) {
                        E *= fv[k];
                        Q *= qv[k];
                    }
                    Wv[4 * h4 + k4] = iw[k4] * hv[k4] * Q;
                    s0[4 * h4 + k4] = E * gg[k4];
                    s1[4 * h4 + k4] = Dc * hv[k4] * gg[k4];
                }
            }
            const int col = 16 * q + 8 * g8;
            st8(sm.Wh, sm.Wl, ch, col, kP, Wv);
            if (full) {
                tc::tmem_st8(trow + Cols::SV + col, s0);
                tc::tmem_st8(trow + Cols::SV + 64 + col, s1);
            }
        }
    };
    // (four variants: b present or not, z used or not)
    auto unpack = [&](bool slow, bool full) {
        const bool uz = full && p.z != nullptr;
        if (p.b != nullptr) {
            if (uz) unpack_v(slow, full, std::true_type{}, std::true_type{});
            else unpack_v(slow, full, std::true_type{}, std::false_type{});
        } else {
            if (uz) unpack_v(slow, full, std::false_type{}, std::true_type{});
            else unpack_v(slow, full, std::false_type{}, std::false_type{});
        }
    };

    // --------------------------------------------------------- the MMAs
    // D (+)= A B over nks K steps of 16, A and B bf16 tiles in the layout of
    // tc::bf_offset_w (a_rows, b_rows: their row counts).
    // (a, b: tile start addresses / 16; K-major steps walk 32 bytes along a
    // 128-byte row, then the next 64-column block R * 128 bytes on; MN-major
    // steps walk 16 rows = 2048 bytes)
    auto kstep = [](int rows, int ks) { return (uint32_t)((ks >> 2) * rows * 8 + (ks & 3) * 2); };
    auto prod = [&](uint32_t dcol, uint32_t a, int a_rows, uint32_t b, int b_rows, bool b_mn,
                    int nks, uint32_t idesc, bool& first) {
#pragma unroll
        for (int ks = 0; ks < nks; ++ks) {
            const uint64_t bd = b_mn ? tc::sdesc_sw128_mn_a4(b + ks * 128u, (uint32_t)b_rows * 128)
                                     : tc::sdesc_sw128_a4(b + kstep(b_rows, ks));
            tc::mma_bf16_ss(dcol, tc::sdesc_sw128_a4(a + kstep(a_rows, ks)), bd, idesc,
                            first ? 0u : 1u);
            first = false;
        }
    };
    // S = W B: W (rows ch, K = t) against B (rows t = K, columns j = N),
    // one 64-column block of j per product.
    // (one 64-column block of S per issuing thread: lane 0 of warp 1 + jb;
    // on the exact path those threads arrive instead)
    auto issue_S = [&](int jb) {
        constexpr uint32_t id = tc::idesc_bf16(128, 64, false, true);
        const uint32_t bsrc = NAJU_SA(Bs) + (uint32_t)(jb * kK * 8);
        bool f = true;
        prod(tbase + Cols::S + 64 * jb, NAJU_SA(Wh), kP, bsrc, kK, true, kK / 16, id, f);
        prod(tbase + Cols::S + 64 * jb, NAJU_SA(Wl), kP, bsrc, kK, true, kK / 16, id, f);
        tc::mma_commit(&sm.mb2);
    };

    // Exact path: the plain recurrence over the block on this thread's state
    // columns (f recomputed from the raw a); full: x . C summed over the
    // quarters (in the X tiles' bytes, rewritten after the block), then R.
    auto exact_block = [&](int nv, bool full) {
        float* rsum = reinterpret_cast<float*>(sm.Xh);  // [64 t][128 ch]
        if (full) {
            for (int e = tid; e < kK * kP; e += kNT) rsum[e] = 0.f;
            __syncthreads();
        }
        float x[NQ];
#pragma unroll
        for (int k = 0; k < NQ; k += 16) tc::tmem_ld16(trow + Cols::X + NQ * q + k, &x[k]);
        tc::tmem_ld_wait();
        for (int tt = 0; tt < nv; ++tt) {
            const float f = sigmoidf_(bf2f(sm.ra[tt * kP + ch]));
            const float v = ld1(sm.Wh, ch, tt, kP) + ld1(sm.Wl, ch, tt, kP);
            float rp = 0.f;
#pragma unroll
            for (int j = 0; j < NQ; ++j) {
                x[j] = fmaf(f, x[j], v * ld1(sm.Bs, tt, NQ * q + j, kK));
                if (full) rp = fmaf(x[j], ld1(sm.Cs, tt, NQ * q + j, kK), rp);
            }
            if (full) atomicAdd(&rsum[tt * kP + ch], rp);
        }
#pragma unroll
        for (int k = 0; k < NQ; k += 16) tc::tmem_st16(trow + Cols::X + NQ * q + k, &x[k]);
        if (full) {
            __syncthreads();
            float rv[16];
#pragma unroll
            for (int k = 0; k < 16; ++k) rv[k] = rsum[(16 * q + k) * kP + ch];
            tc::tmem_st16(trow + Cols::R + 16 * q, rv);
        }
        tc::tmem_st_wait();
        sync();
    };
    // After a block: X <- E_63 (X + S) on this thread's columns (the exact
    // path has updated X already), then the new state to a global [d][N] row
    // (dst != null), to the checkpoint staging tile (stage; d_state 64) and to
    // the X tile pair (tiles), from the same registers.
    auto advance = [&](bool slow, float* dst, bool stage, bool tiles) {
#pragma unroll
        for (int k = 0; k < NQ; k += 16) {
            float v[16], sv[16];
            tc::tmem_ld16(trow + Cols::X + NQ * q + k, v);
            if (!slow) tc::tmem_ld16(trow + Cols::S + NQ * q + k, sv);
            tc::tmem_ld_wait();
            if (!slow) {
#pragma unroll
                for (int j = 0; j < 16; ++j) v[j] = E63 * (v[j] + sv[j]);
                tc::tmem_st16(trow + Cols::X + NQ * q + k, v);
                tc::tmem_st16(trow + Cols::S + NQ * q + k, kZero16);  // S accumulates from zero
            }
            if (dst && cvalid) {
                st_v8(dst + c * N + NQ * q + k, v);
                st_v8(dst + c * N + NQ * q + k + 8, v + 8);
            }
            if (kOwnStage && stage) {
                // box col / 32 of 128 rows x 128 bytes, row ch, 16-byte chunk
                // (col % 32) / 4 XOR-permuted by ch % 8 (the TMA store's layout)
#pragma unroll
                for (int j = 0; j < 16; j += 4) {
                    const int col = NQ * q + k + j;
                    const uint32_t o = (uint32_t)((col >> 5) * kP * 128 + ch * 128 +
                                                  ((((col & 31) >> 2) ^ (ch & 7)) << 4));
                    *reinterpret_cast<float4*>(reinterpret_cast<char*>(sm.ck) + o) =
                        make_float4(v[j], v[j + 1], v[j + 2], v[j + 3]);
                }
            }
            if (tiles) {
                st8(sm.Xh, sm.Xl, ch, NQ * q + k, kP, v);
                st8(sm.Xh, sm.Xl, ch, NQ * q + k + 8, kP, v + 8);
            }
        }
        tc::tmem_st_wait();
    };

    // One block: full (outputs) or update-only.  On entry the block's raw
    // inputs and B (and C) are on their way and, when full, the X tile pair
    // holds the state entering it; on exit the state in tensor memory is
    // updated and, for next >= 0, block next's loads are issued.
    float logP = 0.f;  // log of the decay product over an update-only pass
    // The staged y of a block and its staged checkpoint leave after the next
    // block's first barrier (no barrier of their own): the block whose y is
    // pending and the checkpoint index pending, or -1.
    int y_pending = -1, ck_pending = -1;
    auto store_out = [&]() {
        if (tid == 0) {
            bool any = false;
            if (kStageY && y_pending >= 0) {
                tma::store_3d(&tm.y, (int)c0, y_pending * kK, bb, kOwnStage ? sm.ys : sm.Wh);
                any = true;
            }
            if (kOwnStage && ck_pending >= 0) {
                const int z = bb * (p.nck + 1) + ck_pending;
#pragma unroll
                for (int jb = 0; jb < N / 32; ++jb)
                    tma::store_3d(&tm.ck, 32 * jb, (int)c0, z, sm.ck + jb * kP * 32);
                any = true;
            }
            if (any) tma::store_commit();
        }
        y_pending = -1;
        ck_pending = -1;
    };
    auto run_block = [&](int k, bool full, int next) {
        const int64_t tb = (int64_t)k * kK;
        const int nv = (int)min64((int64_t)kK, L - tb);
        constexpr uint32_t idR = tc::idesc_bf16(128, 64);
        wait_mb(&sm.mb_raw, ph_raw);
        store_out();
        // Once this block's B and C have landed, two threads on different
        // warps issue the two products that overlap the CUDA-core work below
        // (each MMA holds its issuing warp for some 50 cycles): thread 32
        // G^T = B C^T (M = 64: rows m, columns t'; B and C exact) as two
        // halves of 32 columns t' in the two lane halves of the same tensor
        // memory columns, so all lanes share the copy below; thread 0
        // R = X C^T (the X tiles hold the state entering the block since the
        // barrier above; R += W G^T follows on the same thread).  Thread 32
        // also waits in an update-only pass, whose S reads B.
        if (tid == 32 || (full && tid == 0)) {
            if (!timed_out && !tc::mbar_wait(&sm.mb_bc, ph_bc, kSpin)) timed_out = true;
        }
        ph_bc ^= 1u;
        if (full && tid == 32) {
            constexpr uint32_t idG = tc::idesc_bf16(64, 32);
            bool fg = true;
            prod(tbase + Cols::G, NAJU_SA(Bs), kK, NAJU_SA(Cs), kK, false, N / 16, idG, fg);
            fg = true;  // rows t' 32.. of C: four 8-row groups (4096 bytes) on
            prod(tbase + (16u << 16) + Cols::G, NAJU_SA(Bs), kK, NAJU_SA(Cs) + 4096 / 16, kK, false,
                 N / 16, idG, fg);
            tc::mma_commit(&sm.mb0);
        }
        if (full && tid == 0) {
            bool fr = true;
            prod(tbase + Cols::R, NAJU_SA(Xh), kP, NAJU_SA(Cs), kK, false, N / 16, idR, fr);
            prod(tbase + Cols::R, NAJU_SA(Xl), kP, NAJU_SA(Cs), kK, false, N / 16, idR, fr);
        }
        // d_state 128: the previous block's y (staged over W) must have left
        // before unpack rewrites W (the decays' barrier orders this wait)
        if (!kOwnStage && kStageY && tid == 0) tma::store_wait_read();
        const bool slow = decays(nv);
        unpack(slow, full);
        tc::tmem_st_wait();
        tc::fence_proxy_async();
        if (full) {
            wait_mb(&sm.mb0, ph0);
        } else {
            sync();
        }
        // update-only pass: S = W B, one 64-column block per issuing thread
        // (a full pass has S in the chain below; those threads arrive)
        if (lid == 0 && warp >= 1 && warp <= N / 64) {
            if (!slow && !full) issue_S(warp - 1);
            else tc::mbar_arrive(&sm.mb2);
        }
        if (!slow) {
            if (full) {
                {   // masked G^T to its tile pair, kept where t' >= m: lane l of
                    // sub-partition s4 holds row m = 16 s4 + l % 16, columns
                    // t' = 32 (l / 16) + [0, 32); this warp copies 8 of them
                    float v[8];
                    tc::tmem_ld8(trow + Cols::G + 8 * q, v);
                    tc::tmem_ld_wait();
                    const int row = 16 * s4 + (lid & 15), t0 = 32 * (lid >> 4) + 8 * q;
#pragma unroll
                    for (int j = 0; j < 8; ++j)
                        if (t0 + j < row) v[j] = 0.f;
                    st8(sm.GTh, sm.GTl, row, t0, kK, v);
                }
                tc::fence_proxy_async();
                sync();
            }
            if (tid == 0) {
                if (full) {
                    // [S | R] += W_hi [B | G^T_hi] + W_lo [B | G^T_hi], R += W_hi G^T_lo
                    // (S starts at zero, R holds X C^T)
                    constexpr uint32_t idSR = tc::idesc_bf16(128, N + 64, false, true);
                    constexpr uint32_t idR2 = tc::idesc_bf16(128, 64, false, true);
                    bool f = false;
                    prod(tbase + Cols::S, NAJU_SA(Wh), kP, NAJU_SA(Bs), kK, true, kK / 16, idSR, f);
                    prod(tbase + Cols::S, NAJU_SA(Wl), kP, NAJU_SA(Bs), kK, true, kK / 16, idSR, f);
                    prod(tbase + Cols::R, NAJU_SA(Wh), kP, NAJU_SA(GTl), kK, true, kK / 16, idR2, f);
                    tc::mma_commit(&sm.mb2);
                } else {
                    tc::mbar_arrive(&sm.mb2);  // no R in an update-only pass
                }
                // the raw buffer is read: the next block's inputs load while
                // the products run
                if (next >= 0) load_raw(next, full);
                // d_state 64: the staged y and checkpoint of the previous
                // block have left before this block's are staged
                if (kOwnStage) tma::store_wait_read();
            }
            wait_mb(&sm.mb2, ph2);
        } else {
            // R = X C^T may still read the X tiles, whose bytes the exact path reuses
            if (tid == 0) {
                if (full) tc::mma_commit(&sm.mb2);
                else tc::mbar_arrive(&sm.mb2);
                if (kOwnStage) tma::store_wait_read();
            }
            wait_mb(&sm.mb2, ph2);
            exact_block(nv, full);
            if (tid == 0 && next >= 0) load_raw(next, full);
        }
        // the B and C tiles are free
        if (tid == 0 && next >= 0) load_bc(next, full);
        if (full) {
            float r[16], e[16], dh[16];
            tc::tmem_ld16(trow + Cols::R + 16 * q, r);
            tc::tmem_ld16(trow + Cols::SV + 16 * q, e);
            tc::tmem_ld16(trow + Cols::SV + 64 + 16 * q, dh);
            tc::tmem_ld_wait();
            if constexpr (kStageY) {
                // [64 t][128 ch], d_state 128 over W
                __nv_bfloat16* ys = (kOwnStage ? sm.ys : sm.Wh) + 16 * q * kP + ch;
#pragma unroll
                for (int kk = 0; kk < 16; ++kk)
                    ys[kk * kP] = __float2bfloat16_rn(fmaf(e[kk], r[kk], dh[kk]));
            } else {
                Tout* gy = static_cast<Tout*>(p.y) + ((int64_t)bb * L + tb + 16 * q) * d + c;
                const int nk = cvalid ? min(16, nv - 16 * q) : 0;
#pragma unroll
                for (int kk = 0; kk < 16; ++kk)
                    if (kk < nk) gy[(int64_t)kk * d] = from_f<Tout>(fmaf(e[kk], r[kk], dh[kk]));
            }
        }
        logP += __logf(E63);  // decay over the block (for the look-back)
        return slow;
    };

    // ============================================================ passes
    // Blocks [s0, s1) of the current unit from the state in tensor memory:
    // full passes write the checkpoint after every block but the last (and
    // after the last when end_ckpt) and the outputs.
    auto run_segment = [&](int s0, int s1, bool full, bool end_ckpt) {
        if (tid == 0) {
            load_raw(s0, full);
            load_bc(s0, full);
        }
        if (full) state_out(nullptr, true);
#pragma unroll
        for (int k = 0; k < NQ; k += 16) tc::tmem_st16(trow + Cols::S + NQ * q + k, kZero16);
        tc::tmem_st_wait();
        tc::fence_proxy_async();
        sync();
        for (int k = s0; k < s1; ++k) {
            const bool last = k + 1 == s1;
            const bool slow = run_block(k, full, last ? -1 : k + 1);
            // checkpoint after every block but the last (and the last when
            // end_ckpt; that one is stored directly, as a successor may read
            // it in this launch)
            const bool ck = full && (!last || end_ckpt);
            const bool stage = kOwnStage && ck && !last;
            advance(slow, ck && !stage ? ck_at(k + 1) : nullptr, stage, full && !last);
            // X tiles and the staged y / checkpoint -> async proxy; the next
            // block's first barrier orders them before its MMAs and stores
            tc::fence_proxy_async();
            if (full) y_pending = k;
            if (stage) ck_pending = k + 1;
        }
        sync();
        store_out();
    };
    if (sbase & 1023u) {  // the swizzled tiles need 1024-byte alignment
        if (tid == 0) atomicOr(&p.hdr->status, 1 << NAJU_ERR_INVALID_ARG);
    } else if (PIECES) {
        const int64_t Wb = Bt * p.ntiles * (int64_t)p.nck;
        const int64_t F0 = (int64_t)item * Wb / p.npieces;
        const int64_t F1 = (int64_t)(item + 1) * Wb / p.npieces;
        const int64_t ub_lo = (F0 / p.nck) * p.nck;
        for (int64_t ub = ((F1 - 1) / p.nck) * p.nck; ub >= ub_lo; ub -= p.nck) {
            const int s0 = (int)(max64(F0, ub) - ub), s1 = (int)(min64(F1, ub + p.nck) - ub);
            set_unit((int)(ub / p.nck), s0, s1);
            int* flag_cut = p.flags + (int64_t)bb * p.ntiles + tile;
            if (s0 == 0) {
                state_from(p.x0 ? p.x0 + (int64_t)bb * d * N : nullptr, false);
                state_out(ck_at(0), false);
            } else {
                if (tid == 0) sm.ok = wait_flag(flag_cut, &p.hdr->status, p.wait_limit) ? 1 : 0;
                __syncthreads();
                state_from(sm.ok ? ck_at(s0) : nullptr, true);
            }
            run_segment(s0, s1, true, true);
            if (s1 == p.nck && p.x_final) state_out(p.x_final + (int64_t)bb * d * N, false);
            if (s1 < p.nck) {  // head of a cut unit: the state at the cut is published
                __threadfence();
                __syncthreads();
                if (tid == 0 && !p.fault_skip_publish) st_release(flag_cut, 1);
            }
            sync();
        }
    } else {
        const int per_g = (int)(Bt * p.ntiles);
        const int g = item / per_g;
        const int s0 = g * p.seg_per_group;
        set_unit(item % per_g, s0, min(s0 + p.seg_per_group, p.nck));
        const bool last_group = seg1 == p.nck;
        const float* x0b = p.x0 ? p.x0 + (int64_t)bb * d * N : nullptr;
        const int* flag_prev = (g > 0) ? p.flags + ((int64_t)(g - 1) * Bt + bb) * p.ntiles + tile
                                       : nullptr;
        int* flag_mine = p.flags + ((int64_t)g * Bt + bb) * p.ntiles + tile;
        bool ok = true;
        if (!last_group) {
            // update-only pass from x0 (first group) or zero, then the look-back
            state_from(g == 0 ? x0b : nullptr, false);
            logP = 0.f;
            run_segment(seg0, seg1, false, false);
            if (g > 0) {
                if (tid == 0) sm.ok = wait_flag(flag_prev, &p.hdr->status, p.wait_limit) ? 1 : 0;
                __syncthreads();
                ok = sm.ok != 0;
                const float Pf = __expf(logP);
                const float* xs = ck_at(seg0);
#pragma unroll
                for (int k = 0; k < NQ; k += 16) {
                    float xv[16];
                    tc::tmem_ld16(trow + Cols::X + NQ * q + k, xv);
                    tc::tmem_ld_wait();
#pragma unroll
                    for (int j = 0; j < 16; j += 4) {
                        float4 v4 = make_float4(0.f, 0.f, 0.f, 0.f);
                        if (ok && cvalid)
                            v4 = __ldcg(reinterpret_cast<const float4*>(xs + c * N + NQ * q + k + j));
                        xv[j] = fmaf(Pf, v4.x, xv[j]);
                        xv[j + 1] = fmaf(Pf, v4.y, xv[j + 1]);
                        xv[j + 2] = fmaf(Pf, v4.z, xv[j + 2]);
                        xv[j + 3] = fmaf(Pf, v4.w, xv[j + 3]);
                    }
                    tc::tmem_st16(trow + Cols::X + NQ * q + k, xv);
                }
                tc::tmem_st_wait();
            }
            state_out(ck_at(seg1), false);
            __threadfence();
            __syncthreads();
            if (tid == 0 && !(g == 0 && p.fault_skip_publish)) st_release(flag_mine, 1);
        } else if (g > 0) {
            if (tid == 0) sm.ok = wait_flag(flag_prev, &p.hdr->status, p.wait_limit) ? 1 : 0;
            __syncthreads();
            ok = sm.ok != 0;
        }
        if (g > 0) {
            state_from(ok ? ck_at(seg0) : nullptr, true);
        } else {
            state_from(x0b, false);
            state_out(ck_at(0), false);
        }
        run_segment(seg0, seg1, true, last_group);
        if (last_group && p.x_final) state_out(p.x_final + (int64_t)bb * d * N, false);
    }
#undef NAJU_SA
    if (tid == 0) tma::store_wait_all();
    if (timed_out) atomicOr(&p.hdr->status, 1 << NAJU_ERR_TIMEOUT);
    sync();
    if (warp == 0) tc::tmem_dealloc(tbase, Cols::ALLOC);
}

template <typename Tout, int N, bool CONV, bool PIECES>
static cudaError_t launch_fwd_blk_t(const FwdParams& p, cudaStream_t st) {
    FkTmaps tm;
    memset(&tm, 0, sizeof(tm));
    bool ok = tma_encode_bf16_3d(&tm.u, p.hu, p.Bt, p.L, p.d, kK + 3, kP) &&
              tma_encode_bf16_3d(&tm.a, p.a, p.Bt, p.L, p.d, kK, kP) &&
              (!p.b || tma_encode_bf16_3d(&tm.b, p.b, p.Bt, p.L, p.d, kK, kP)) &&
              (!p.z || tma_encode_bf16_3d(&tm.z, p.z, p.Bt, p.L, p.d, kK, kP)) &&
              tma_encode_bf16_3d_sw128(&tm.B, p.B, p.Bt, p.L, N, kK) &&
              tma_encode_bf16_3d_sw128(&tm.C, p.C, p.Bt, p.L, N, kK);
    if (ok && std::is_same<Tout, __nv_bfloat16>::value)
        ok = tma_encode_bf16_3d(&tm.y, p.y, p.Bt, p.L, p.d, kK, kP);
    if (ok && N == 64)
        ok = p.ckpt != nullptr &&
             tma_encode_f32_3d_sw128(&tm.ck, p.ckpt, p.Bt * (p.nck + 1), p.d, N, kP);
    if (!ok) return cudaErrorInvalidValue;
    const size_t smem = sizeof(FkSmem<N>);
    auto kern = scan_fwd_blk_kernel<Tout, N, CONV, PIECES>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)smem);
    if (e != cudaSuccess) return e;
    const int grid = PIECES ? p.npieces : p.ngroups * (int)p.Bt * p.ntiles;
    kern<<<grid, kNT, smem, st>>>(p, tm);
    return cudaGetLastError();
}

bool fwd_blk_supported(int dtype, int64_t N, int64_t d, int T_ck) {
    return dtype == NAJU_BF16 && (N == 64 || N == 128) && d % 8 == 0 && T_ck == kK;
}

cudaError_t launch_scan_fwd_blk(const FwdParams& p, int out_dtype, cudaStream_t st) {
    const bool conv = p.conv_w != nullptr, pc = p.npieces > 0;
#define NAJU_FWD_BLK(TO, NN)                                                           \
    return conv ? (pc ? launch_fwd_blk_t<TO, NN, true, true>(p, st)                    \
                      : launch_fwd_blk_t<TO, NN, true, false>(p, st))                  \
                : (pc ? launch_fwd_blk_t<TO, NN, false, true>(p, st)                   \
                      : launch_fwd_blk_t<TO, NN, false, false>(p, st))
    if (out_dtype == NAJU_BF16) {
        if (p.N == 64) NAJU_FWD_BLK(__nv_bfloat16, 64);
        if (p.N == 128) NAJU_FWD_BLK(__nv_bfloat16, 128);
    } else {
        if (p.N == 64) NAJU_FWD_BLK(float, 64);
        if (p.N == 128) NAJU_FWD_BLK(float, 128);
    }
#undef NAJU_FWD_BLK
    return cudaErrorInvalidValue;
}

}  // namespace naju
