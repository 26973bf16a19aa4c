// Naju forward scan in block form on the 5th-generation tensor cores
// (sm_100a, tcgen05, kind::tf32), for bf16 activations with d_state 64 or 128.
//
// Same computation as the CUDA-core forward (Naju reproduction README, "Core
// equations"): x_n = f_n x_{n-1} + i_n h_n B_n^T, y_n = x_n.C_n/sqrt(N) + D h_n,
// out_n = y_n SiLU(z_n), h = SiLU(conv(u)).
//
// A thread block owns 128 channels of one batch element (one channel per
// tensor-memory lane) and walks its tokens in blocks of 64, the spacing of
// the checkpoints it writes for the backward.  With X the state entering a
// block (resident in tensor memory for the whole pass), per channel
// E_t = prod_{k<=t} f_k from the block start, Q_t = 1/E_t, W_t = i_t h_t Q_t and
// G[t][m] = C_t.B_m kept for m <= t:
//   y_t  = s E_t R_t SiLU(z_t) + D h_t SiLU(z_t),   R = X C^T + W G^T
//   X'   = E_63 (X + S),                            S = W B
// G = C B^T (M = 64) goes from tensor memory to a masked shared tile; R and S
// run with X from tensor memory and the other operands from shared memory
// (tf32: fp32 tiles in the 128-byte swizzled row layout; S reads B MN-major,
// which for tf32 needs a second copy of B with 32-byte swizzle atoms).
// The state chain from one block to the next is the per-channel update X';
// everything per (token, channel) runs on the CUDA cores, 512 threads: warp w
// handles channels 32 (w % 4) + lane and tokens [16 q, 16 q + 16) of the
// block, q = w / 4, and the state columns [q N / 4, (q + 1) N / 4).
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

template <int N>
struct FkCols {
    static constexpr uint32_t X = 0;            // state [ch][j]
    static constexpr uint32_t S = N;            // W B   [ch][j]
    static constexpr uint32_t R = 2 * N;        // R     [ch][t]
    static constexpr uint32_t G = 2 * N + 64;   // G (M = 64)
    static constexpr uint32_t SV = 2 * N + 128; // s E SiLU(z), D h SiLU(z)  [ch][t] x 2
    static constexpr uint32_t USED = 2 * N + 256;
    static constexpr uint32_t ALLOC = USED <= 256 ? 256 : 512;
    static_assert(USED <= 512, "tensor memory");
};

struct alignas(64) FkTmaps {
    CUtensorMap u, a, b, z, B, C;  // bf16, for L2 prefetches
};

template <int N>
struct FkSmem {
    alignas(1024) float W[kP * kK];   // rows ch, cols t
    alignas(1024) float Bf[kK * N];   // rows t, cols j
    alignas(1024) float Cf[kK * N];   // rows t, cols j
    alignas(1024) float G[kK * kK];   // rows t, cols m (m <= t)
    alignas(1024) float Bm[kK * N];   // B again, MN-major layout for S = W B
    alignas(1024) float F[kP * kK];   // f of the block (exact path), rows ch, cols t
    alignas(1024) float rsum[kK * kP];// exact path: x_t . C_t [t][ch]
    float xq[4][kP], xe[4][kP];
    uint64_t mb0, mb2;
    uint32_t taddr;
    int item, ok;
};

__device__ __forceinline__ float ldbf(const __nv_bfloat16* p) {
    return __uint_as_float((uint32_t)__ldg(reinterpret_cast<const unsigned short*>(p)) << 16);
}
__device__ __forceinline__ float bf_lo(uint32_t v) { return __uint_as_float(v << 16); }
__device__ __forceinline__ float bf_hi(uint32_t v) { return __uint_as_float(v & 0xffff0000u); }

}  // namespace

template <typename Tout, int N, bool CONV, bool PIECES>
__global__ void __launch_bounds__(512, 1)
scan_fwd_blk_kernel(const FwdParams p, const __grid_constant__ FkTmaps tm) {
    using Cols = FkCols<N>;
    using Sm = FkSmem<N>;
    using Tin = __nv_bfloat16;
    constexpr int NQ = N / 4;  // state columns per thread
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
        tc::mbar_init(&sm.mb0, 1);
        tc::mbar_init(&sm.mb2, 1);
        tma::prefetch_map(&tm.u);
        tma::prefetch_map(&tm.a);
        if (has_b) tma::prefetch_map(&tm.b);
        if (has_z) tma::prefetch_map(&tm.z);
        tma::prefetch_map(&tm.B);
        tma::prefetch_map(&tm.C);
    }
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    const uint32_t tbase = sm.taddr;
    const uint32_t trow = tbase + ((uint32_t)(s4 * 32) << 16);
    const int item = sm.item;
    const uint32_t sbase = tc::smem_u32(&sm);
    const uint32_t aW = sbase + (uint32_t)offsetof(Sm, W), aB = sbase + (uint32_t)offsetof(Sm, Bf),
                   aC = sbase + (uint32_t)offsetof(Sm, Cf), aG = sbase + (uint32_t)offsetof(Sm, G),
                   aBm = sbase + (uint32_t)offsetof(Sm, Bm);
    uint32_t ph0 = 0, ph2 = 0;
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
    auto gin = [&](const void* base) {
        return static_cast<const Tin*>(base) + (int64_t)bb * L * d + c;
    };
    auto ck_at = [&](int k) { return p.ckpt + ((int64_t)bb * (p.nck + 1) + k) * d * N; };
    auto sync = [&]() {
        tc::fence_before_sync();
        __syncthreads();
        tc::fence_after_sync();
    };
    auto sw = [](int row, int col, int R) { return tc::sw128_offset(row, col, R) >> 2; };

    // This thread's state columns of the TMEM state <-> a global [d][N] row.
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
    auto state_to = [&](float* dst) {
        float v[NQ];
#pragma unroll
        for (int k = 0; k < NQ; k += 16) tc::tmem_ld16(trow + Cols::X + NQ * q + k, &v[k]);
        tc::tmem_ld_wait();
        if (cvalid) {
#pragma unroll
            for (int k = 0; k < NQ; k += 4)
                *reinterpret_cast<float4*>(dst + c * N + NQ * q + k) =
                    make_float4(v[k], v[k + 1], v[k + 2], v[k + 3]);
        }
    };
    auto prefetch_block = [&](int k) {
        const int x = (int)c0, y = k * kK, zb = bb;
        tma::prefetch_l2_3d(&tm.u, x, y > 3 ? y - 3 : 0, zb);
        tma::prefetch_l2_3d(&tm.a, x, y, zb);
        if (has_b) tma::prefetch_l2_3d(&tm.b, x, y, zb);
        if (has_z) tma::prefetch_l2_3d(&tm.z, x, y, zb);
        tma::prefetch_l2_3d(&tm.B, 0, y, zb);
        tma::prefetch_l2_3d(&tm.C, 0, y, zb);
    };

    // ------------------------------------------------- decays (loop 1)
    float fv[16], qv[16];
    float Eb = 1.f, Qb = 1.f, E63 = 1.f;
    auto decays = [&](int64_t tb, int nv) -> bool {
        const Tin* ga = gin(p.a);
        float Qh = 1.f, Eh = 1.f;
#pragma unroll
        for (int k = 0; k < 16; ++k) {
            const int tt = 16 * q + k;
            const bool valid = cvalid && tt < nv;
            const float av = valid ? ldbf(ga + (tb + tt) * d) : 0.f;
            const float ea = __expf(-av);
            qv[k] = valid ? 1.f + ea : 1.f;
            fv[k] = valid ? rcpa_(qv[k]) : 1.f;
            Qh *= qv[k];
            Eh *= fv[k];
        }
#pragma unroll
        for (int k = 0; k < 16; k += 4)
            *reinterpret_cast<float4*>(&sm.F[sw(ch, 16 * q + k, kP)]) =
                make_float4(fv[k], fv[k + 1], fv[k + 2], fv[k + 3]);
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
    // W (shared tile); full: s E SiLU(z) and D h SiLU(z) (tensor memory).
    auto unpack = [&](int64_t tb, int nv, bool slow, bool full) {
        const Tin* gu = gin(p.hu);
        const Tin* gbp = has_b ? gin(p.b) : nullptr;
        const Tin* gz = has_z ? gin(p.z) : nullptr;
        auto ubits = [&](int i) -> uint32_t {
            const int tt = 16 * q - 3 + i;
            const int64_t t = tb + tt;
            const bool ok = cvalid && tt < nv && t >= 0 && (CONV || i >= 3);
            return ok ? (uint32_t)__ldg(reinterpret_cast<const unsigned short*>(gu + t * d)) : 0u;
        };
        uint32_t upk[10];
#pragma unroll
        for (int i = 0; i < 10; ++i) upk[i] = ubits(2 * i) | (i < 9 ? ubits(2 * i + 1) << 16 : 0u);
        auto uwin = [&](int m) { return (m & 1) ? bf_hi(upk[m >> 1]) : bf_lo(upk[m >> 1]); };
        float E = slow ? 1.f : Eb, Q = slow ? 1.f : Qb;
#pragma unroll
        for (int g4 = 0; g4 < 4; ++g4) {
            float Wv[4], s0[4], s1[4];
#pragma unroll
            for (int k4 = 0; k4 < 4; ++k4) {
                const int k = 4 * g4 + k4;
                const int tt = 16 * q + k;
                const int64_t t = tb + tt;
                const bool valid = cvalid && tt < nv;
                float h;
                if (CONV) {
                    const float pp = fmaf(w3, uwin(k + 3), fmaf(w2, uwin(k + 2),
                                         fmaf(w1, uwin(k + 1), fmaf(w0, uwin(k), wb))));
                    h = pp * sigmoida_(pp);
                } else {
                    h = uwin(k + 3);
                }
                if (!valid) h = 0.f;
                const float f = fv[k], qq = qv[k];
                // coupled: i = 1 - f = (1/f - 1) f (1 where exp(-a) overflowed)
                const float iw = has_b ? (valid ? sigmoida_(ldbf(gbp + t * d)) : 0.f)
                                       : (qq < 3.0e38f ? (qq - 1.f) * f : 1.f);
                if (!slow) {
                    E *= f;
                    Q *= qq;
                }
                Wv[k4] = iw * h * Q;
                if (full) {
                    float gg = 1.f;
                    if (has_z) {
                        const float zv = valid ? ldbf(gz + t * d) : 0.f;
                        gg = zv * sigmoida_(zv);
                    }
                    s0[k4] = sc * E * gg;
                    s1[k4] = Dc * h * gg;
                }
            }
            const int col = 16 * q + 4 * g4;
            *reinterpret_cast<float4*>(&sm.W[sw(ch, col, kP)]) = make_float4(Wv[0], Wv[1], Wv[2], Wv[3]);
            if (full) {
                tc::tmem_st4(trow + Cols::SV + col, s0);
                tc::tmem_st4(trow + Cols::SV + 64 + col, s1);
            }
        }
    };
    auto load_bc = [&](int64_t tb, int nv, bool want_c) {
#pragma unroll
        for (int e0 = tid * 8; e0 < kK * N; e0 += kNT * 8) {
            const int tt = e0 / N, j = e0 % N;
            float4 lo = make_float4(0.f, 0.f, 0.f, 0.f), hi = lo, clo = lo, chi = lo;
            if (tt < nv) {
                const int64_t off = ((int64_t)bb * L + tb + tt) * N + j;
                const uint4 br = __ldg(reinterpret_cast<const uint4*>(static_cast<const Tin*>(p.B) + off));
                lo = make_float4(bf_lo(br.x), bf_hi(br.x), bf_lo(br.y), bf_hi(br.y));
                hi = make_float4(bf_lo(br.z), bf_hi(br.z), bf_lo(br.w), bf_hi(br.w));
                if (want_c) {
                    const uint4 cr = __ldg(reinterpret_cast<const uint4*>(static_cast<const Tin*>(p.C) + off));
                    clo = make_float4(bf_lo(cr.x), bf_hi(cr.x), bf_lo(cr.y), bf_hi(cr.y));
                    chi = make_float4(bf_lo(cr.z), bf_hi(cr.z), bf_lo(cr.w), bf_hi(cr.w));
                }
            }
            *reinterpret_cast<float4*>(&sm.Bf[sw(tt, j, kK)]) = lo;
            *reinterpret_cast<float4*>(&sm.Bf[sw(tt, j + 4, kK)]) = hi;
            *reinterpret_cast<float4*>(&sm.Bm[tc::mn32_offset(tt, j, kK) >> 2]) = lo;
            *reinterpret_cast<float4*>(&sm.Bm[tc::mn32_offset(tt, j + 4, kK) >> 2]) = hi;
            if (want_c) {
                *reinterpret_cast<float4*>(&sm.Cf[sw(tt, j, kK)]) = clo;
                *reinterpret_cast<float4*>(&sm.Cf[sw(tt, j + 4, kK)]) = chi;
            }
        }
    };
    auto kd = [](uint32_t base, int rows, int ks) {
        return tc::sdesc_sw128(base + (ks >> 2) * rows * 128 + (ks & 3) * 32);
    };
    auto wait_mb = [&](uint64_t* mb, uint32_t& ph) {
        if (warp == kNT / 32 - 1 && !tc::mbar_wait(mb, ph, kSpin)) timed_out = true;
        __syncthreads();
        ph ^= 1u;
        tc::fence_after_sync();
    };
    // S = W B (the state update's product), on its own (update-only pass).
    auto mma_S = [&]() {
        constexpr uint32_t idS = tc::idesc_tf32(128, N, false, true);
#pragma unroll
        for (int ks = 0; ks < kK / 8; ++ks)
            tc::mma_tf32_ss(tbase + Cols::S, kd(aW, kP, ks), tc::sdesc_mn32(aBm, kK, ks), idS, ks > 0);
    };
    // Exact path: plain recurrence over the block on this thread's state
    // columns; full: x . C summed over the quarters into rsum, then R.
    auto exact_block = [&](int nv, bool full) {
        if (full) {
            for (int e = tid; e < kK * kP; e += kNT) sm.rsum[e] = 0.f;
            __syncthreads();
        }
        float x[NQ];
#pragma unroll
        for (int k = 0; k < NQ; k += 16) tc::tmem_ld16(trow + Cols::X + NQ * q + k, &x[k]);
        tc::tmem_ld_wait();
        for (int tt = 0; tt < nv; ++tt) {
            const float f = sm.F[sw(ch, tt, kP)], v = sm.W[sw(ch, tt, kP)];
            float rp = 0.f;
#pragma unroll
            for (int j = 0; j < NQ; ++j) {
                x[j] = fmaf(f, x[j], v * sm.Bf[sw(tt, NQ * q + j, kK)]);
                if (full) rp = fmaf(x[j], sm.Cf[sw(tt, NQ * q + j, kK)], rp);
            }
            if (full) atomicAdd(&sm.rsum[tt * kP + ch], rp);
        }
#pragma unroll
        for (int k = 0; k < NQ; k += 16) tc::tmem_st16(trow + Cols::X + NQ * q + k, &x[k]);
        if (full) {
            __syncthreads();
            float rv[16];
#pragma unroll
            for (int k = 0; k < 16; ++k) rv[k] = sm.rsum[(16 * q + k) * kP + ch];
            tc::tmem_st16(trow + Cols::R + 16 * q, rv);
        }
        tc::tmem_st_wait();
        sync();
    };
    // X <- E_63 (X + S) on this thread's columns.
    auto update_state = [&]() {
#pragma unroll
        for (int k = 0; k < NQ; k += 16) {
            float xv[16], sv[16];
            tc::tmem_ld16(trow + Cols::X + NQ * q + k, xv);
            tc::tmem_ld16(trow + Cols::S + NQ * q + k, sv);
            tc::tmem_ld_wait();
#pragma unroll
            for (int j = 0; j < 16; ++j) xv[j] = E63 * (xv[j] + sv[j]);
            tc::tmem_st16(trow + Cols::X + NQ * q + k, xv);
        }
        tc::tmem_st_wait();
    };

    // One block: full (outputs) or update-only.  The state X in tensor
    // memory enters the block and leaves it updated.
    float logP = 0.f;  // log of the decay product over an update-only pass
    auto run_block = [&](int k, bool full) {
        const int64_t tb = (int64_t)k * kK;
        const int nv = (int)min64((int64_t)kK, L - tb);
        const bool slow = decays(tb, nv);
        unpack(tb, nv, slow, full);
        load_bc(tb, nv, full);
        tc::fence_proxy_async();
        sync();
        if (!slow) {
            if (full) {
                if (tid == 0) {
                    constexpr uint32_t id64 = tc::idesc_tf32(64, 64);
                    constexpr uint32_t idR = tc::idesc_tf32(128, 64);
#pragma unroll
                    for (int ks = 0; ks < N / 8; ++ks)
                        tc::mma_tf32_ss(tbase + Cols::G, kd(aC, kK, ks), kd(aB, kK, ks), id64, ks > 0);
                    tc::mma_commit(&sm.mb0);
                    mma_S();
#pragma unroll
                    for (int ks = 0; ks < N / 8; ++ks)
                        tc::mma_tf32_ts(tbase + Cols::R, tbase + Cols::X + ks * 8, kd(aC, kK, ks), idR,
                                        ks > 0);
                }
                wait_mb(&sm.mb0, ph0);
                {   // masked G to its tile: lanes +0 of each sub-partition hold rows
                    float v[16];
                    tc::tmem_ld16(trow + Cols::G + 16 * q, v);
                    tc::tmem_ld_wait();
                    if (lid < 16) {
                        const int row = 16 * s4 + lid;
#pragma unroll
                        for (int j = 0; j < 16; j += 4) {
                            const int col = 16 * q + j;
                            float4 o;
                            o.x = col + 0 <= row ? v[j] : 0.f;
                            o.y = col + 1 <= row ? v[j + 1] : 0.f;
                            o.z = col + 2 <= row ? v[j + 2] : 0.f;
                            o.w = col + 3 <= row ? v[j + 3] : 0.f;
                            *reinterpret_cast<float4*>(&sm.G[sw(row, col, kK)]) = o;
                        }
                    }
                }
                tc::fence_proxy_async();
                sync();
                if (tid == 0) {
                    constexpr uint32_t idR = tc::idesc_tf32(128, 64);
#pragma unroll
                    for (int ks = 0; ks < kK / 8; ++ks)
                        tc::mma_tf32_ss(tbase + Cols::R, kd(aW, kP, ks), kd(aG, kK, ks), idR, 1u);
                    tc::mma_commit(&sm.mb2);
                }
            } else if (tid == 0) {
                mma_S();
                tc::mma_commit(&sm.mb2);
            }
            wait_mb(&sm.mb2, ph2);
        } else {
            exact_block(nv, full);
        }
        if (full) {
            Tout* gy = static_cast<Tout*>(p.y) + (int64_t)bb * L * d + c;
            float r[16], e[16], dh[16];
            tc::tmem_ld16(trow + Cols::R + 16 * q, r);
            tc::tmem_ld16(trow + Cols::SV + 16 * q, e);
            tc::tmem_ld16(trow + Cols::SV + 64 + 16 * q, dh);
            tc::tmem_ld_wait();
#pragma unroll
            for (int kk = 0; kk < 16; ++kk) {
                const int tt = 16 * q + kk;
                if (cvalid && tt < nv) gy[(tb + tt) * d] = from_f<Tout>(fmaf(e[kk], r[kk], dh[kk]));
            }
        }
        if (!slow) update_state();
        logP += __logf(E63);  // decay over the block (for the look-back)
        sync();
    };

    // ============================================================ passes
    if (PIECES) {
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
                state_to(ck_at(0));
            } else {
                if (tid == 0) sm.ok = wait_flag(flag_cut, &p.hdr->status, p.wait_limit) ? 1 : 0;
                __syncthreads();
                state_from(sm.ok ? ck_at(s0) : nullptr, true);
            }
            if (tid == 0) prefetch_block(s0);
            sync();
            for (int k = s0; k < s1; ++k) {
                if (tid == 0 && k + 1 < s1) prefetch_block(k + 1);
                run_block(k, true);
                state_to(ck_at(k + 1));
            }
            if (s1 == p.nck && p.x_final) state_to(p.x_final + (int64_t)bb * d * N);
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
            sync();
            logP = 0.f;
            for (int k = seg0; k < seg1; ++k) {
                if (tid == 0 && k + 1 < seg1) prefetch_block(k + 1);
                run_block(k, false);
            }
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
            state_to(ck_at(seg1));
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
            state_to(ck_at(0));
        }
        if (tid == 0) prefetch_block(seg0);
        sync();
        for (int k = seg0; k < seg1; ++k) {
            if (tid == 0 && k + 1 < seg1) prefetch_block(k + 1);
            run_block(k, true);
            if (k + 1 < seg1 || last_group) state_to(ck_at(k + 1));
        }
        if (last_group && p.x_final) state_to(p.x_final + (int64_t)bb * d * N);
    }
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
              tma_encode_bf16_3d(&tm.B, p.B, p.Bt, p.L, N, kK, N) &&
              tma_encode_bf16_3d(&tm.C, p.C, p.Bt, p.L, N, kK, N);
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
