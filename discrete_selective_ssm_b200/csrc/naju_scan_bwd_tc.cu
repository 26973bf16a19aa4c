// Naju backward scan with the d_state contractions on the 5th-generation
// tensor cores (sm_100a, tcgen05, kind::tf32), for bf16 activations.
//
// Same gradient as naju_scan_bwd.cu (derived from the recurrence of the Naju
// reproduction README, "Core equations"); with G_t = dLoss/dx_t,
// s = 1/sqrt(N), f = sigmoid(a), i = sigmoid(b), v = i h:
//   G_t = s dy_t C_t + f_{t+1} G_{t+1},  GB_t = G_t . B_t,
//   dh_t = D dy_t + i_t GB_t,  db_t = h_t GB_t i_t (1 - i_t),
//   da_t = (f df)_t (1 - f_t),  (f df)_t = sum_{t'>=t} dL_t' + (carry . state),
//   dL_t = s dy_t (x_t . C_t) - v_t GB_t,
//   dB_t = sum_ch v_t G_t,  dC_t = s sum_ch dy_t x_t.
//
// Chunked form.  A block owns 128 channels (tensor-memory lanes) of one batch
// element and one sequence group; it walks the group's 64-token blocks from
// the last to the first, each in two sweeps over 16-token sub-chunks.  With
// E_t the decay product from the sub-chunk start (inclusive), Elast = E_15:
//  forward sweep (from the block's forward checkpoint X):
//   readout   R[ch][t] = X.C_t + sum_m W_m G[t][m],   W_m = v_m / E_m,
//             x_t.C_t = E_t R (for dz and dL),
//   state     X' = Elast X + sum_m (v_m Elast / E_m) B_m,
//   dC        dC_t = sum_ch Y_t X + sum_{m<=t} A_C[t][m] B_m,  Y_t = s dy_t E_t,
//             A_C[t][m] = sum_ch Y_t W_m   (contractions over channels);
//  backward sweep (carry H = the adjoint entering the sub-chunk's end):
//   dv        GB_t = (Elast / E_t) [H.B_t + sum_{t'>=t} U_t' (C_t'.B_t)],
//             U_t' = s dy_t' E_t' / Elast,
//   adjoint   H' = Elast H + sum_t' (s dy_t' E_t') C_t',
//   dB        dB_t = sum_ch P_t H + sum_{t'>=t} A_B[t][t'] C_t',
//             P_t = v_t Elast / E_t,  A_B[t][t'] = sum_ch P_t U_t'.
// Readout, state, dv and adjoint run with the per-channel operand (X, H, W,
// U, ...) in tensor memory; the channel contractions for dB and dC run with
// both operands in shared memory, X or H written transposed into a 128-byte
// swizzled tile (K = channels) - for d_state 64 the 64-row operand rides an
// M = 128 MMA whose upper rows are ignored.  The small A_C / A_B products and
// everything per (token, channel) run on the CUDA cores.
//
// Threads.  512 per block: channel p (TMEM lane p) is handled by threads
// p + 128 q, q = 0..3, each taking 4 of the 16 tokens and a quarter of the
// state columns; one thread issues the MMAs.  Raw inputs arrive by TMA one
// or two sub-chunks ahead (two or three buffers), issued while the MMAs run.
//
// Exactness.  A sub-chunk whose product of 1/f exceeds 2^64 in any channel of
// the block takes an exact token-by-token path on the CUDA cores (states in
// tensor memory, channel sums of dB / dC through warp shuffles).
//
// Outputs.  dB and dC partial sums over each block's 128 channels go to a
// per-tile buffer that a small kernel sums; dD and the conv parameter
// gradients go through per-(batch, group) channel partials; sequence groups
// exchange the adjoint carry by a decoupled look-back backwards in time
// (an adjoint-only early pass, bounded waits), as in the CUDA-core kernel.
// Piece mode (at least one wave of 128-channel units, not a whole number
// of waves) instead gives each block one equal range of all units' 64-token
// blocks; a unit cut in two hands its carry from its tail to its head.
#include <string.h>

#include <type_traits>

#include "naju_common.cuh"
#include "naju_kernels.h"
#include "naju_tc.cuh"
#include "naju_tma.h"

namespace naju {

namespace {

constexpr int kBT = 16;                              // tokens per sub-chunk
constexpr float kBBound = 18446744073709551616.0f;   // 2^64
// No quarter (4 tokens) above 2^16 means no channel's sub-chunk above 2^64.
constexpr float kBQuarter = 65536.0f;
constexpr long long kBSpin = 1LL << 24;

template <int N>
struct BCols {
    static constexpr uint32_t X = 0;            // forward state [N]
    static constexpr uint32_t G = N;            // adjoint carry [N]
    static constexpr uint32_t D = 2 * N;        // state / adjoint MMA result [N]
    static constexpr uint32_t R = 3 * N;        // readout / dv MMA result [16]
    static constexpr uint32_t BC = 3 * N + 16;  // dC / dB MMA result [16] (lanes = d_state)
    static constexpr uint32_t WU = 3 * N + 32;  // W or U [16]
    static constexpr uint32_t VV = 3 * N + 48;  // state weights or s dy E [16]
    static constexpr uint32_t DL = 3 * N + 64;  // s dy_t x_t.C_t of the block [64]
    // d_state 64 has room to split the dC / dB chain over two accumulators
    // (second half of the channel sum), shortening the longest MMA chain.
    static constexpr bool SPLIT = 3 * N + 144 <= 512;
    static constexpr uint32_t BC2 = 3 * N + 128;
    // d_state 64 also has room to keep h and SiLU'(conv pre-activation) of the
    // block's 64 tokens from the forward sweep for the backward sweep.
    static constexpr bool GCACHE = 3 * N + 272 <= 512;
    static constexpr uint32_t GH = 3 * N + 144;   // h [64]
    static constexpr uint32_t GA = 3 * N + 208;   // SiLU'(pre) [64]
    static constexpr uint32_t USED = GCACHE ? 3 * N + 272 : SPLIT ? 3 * N + 144 : 3 * N + 128;
    static constexpr uint32_t ALLOC = 512;
    static_assert(USED <= ALLOC, "tensor memory");
};

struct alignas(64) BwdTmaps {
    CUtensorMap u, a, b, z, dy, B, C;
};

template <int N>
struct BwdTcSmem {
    static constexpr int T = kBT, P = 128;
    // Transposed state tile (X or H), 128-byte swizzled, rows = d_state,
    // K = channels; for N = 64 the M = 128 MMA also reads 8 KB past it.
    static constexpr int ST_FLOATS = N * 128 > 10240 ? N * 128 : 10240;
    // B^T / C^T tile (rows = d_state, K = 16), with the same overrun for N = 64.
    static constexpr int TS_FLOATS = N * 16 > 2048 ? N * 16 : 2048;
    struct Raw {
        alignas(128) __nv_bfloat16 u[T + 3][P];
        alignas(128) __nv_bfloat16 a[T][P];
        alignas(128) __nv_bfloat16 b[T][P];
        alignas(128) __nv_bfloat16 z[T][P];
        alignas(128) __nv_bfloat16 dy[T][P];
        alignas(128) __nv_bfloat16 Bm[T][N];
        alignas(128) __nv_bfloat16 Cm[T][N];
    };
    alignas(1024) float st[ST_FLOATS];
    alignas(1024) float pk[T * P];     // Y or P, swizzled, rows t, K = channels
    // Raw-input buffers: TMA runs up to NRAW - 1 sub-chunks ahead (three for
    // d_state 64; shared memory allows two for 128).
    static constexpr int NRAW = N <= 64 ? 3 : 2;
    Raw raw[NRAW];
    alignas(128) float ta[T * N];      // C (forward) / B (backward) rows t, K = d_state
    alignas(128) float ts[TS_FLOATS];  // B^T (forward) / C^T (backward): rows d_state, K = 16
    // G[t][m] (forward) / G^T (backward) and A_C (forward) / A_B (backward),
    // each as two partial sums over halves of the contraction (two warps each;
    // the MMAs accumulate both halves).
    alignas(128) float tg[2][T * T];
    alignas(128) float ta2[2][T * T];
    alignas(16) float y1[T][P + 4];    // Y / P rows (slow path: s dy or v)
    alignas(16) float w1[T][P + 4];    // W / U rows (slow path: sums over quarters)
    alignas(16) float brow[T][N + 4];
    alignas(16) float crow[T][N + 4];
    float dp[2][T][P];                 // conv dp of the last two backward sub-chunks
    float acc[T][N];                   // slow path channel sums
    float xq[4][P], xe[4][P], xs[4][P];  // exchanges between a channel's four threads
    uint64_t loaded[3], mma;
    uint32_t taddr;
    int item, ok;
    int slowf[4];                      // exact-path decision of the block's sub-chunks
};

enum { kSweepFwd = 0, kSweepBwd = 1, kSweepEarly = 2 };

}  // namespace

template <typename Tout, int N, bool CONV, bool PIECES>
__global__ void __launch_bounds__(512, 1)
scan_bwd_tc_kernel(const BwdParams p, const __grid_constant__ BwdTmaps tm) {
    using Tin = __nv_bfloat16;
    using Cols = BCols<N>;
    using Sm = BwdTcSmem<N>;
    constexpr int T = kBT, P = 128, NT = 512, TQ = T / 4, NC = N / 4;
    constexpr int K = kBwdSub;  // tokens per block (forward checkpoint spacing)
    extern __shared__ __align__(1024) float4 smem4[];
    Sm& sm = *reinterpret_cast<Sm*>(smem4);

    const int tid = threadIdx.x;
    const int warp = tid >> 5;
    const int ch = tid & (P - 1);   // channel within the block = TMEM lane
    const int qd = tid >> 7;        // tokens [4 qd, 4 qd + 4), state columns [N/4 qd, ...)
    const int64_t Bt = p.Bt, L = p.L, d = p.d;
    const float s = p.scale;
    const bool has_z = p.z != nullptr;
    const bool has_b = p.b != nullptr;  // absent: coupled single gate i = 1 - f

    // ------------------------------------------------------------ set-up
    if (warp == 0) {
        tc::tmem_alloc(&sm.taddr, Cols::ALLOC);
        tc::tmem_relinquish();
    }
    if (tid == 0) {
        sm.item = atomicAdd(&p.hdr->bwd_ticket, 1);
        for (int q = 0; q < Sm::NRAW; ++q) tc::mbar_init(&sm.loaded[q], 1);
        tc::mbar_init(&sm.mma, 3);  // three committing (or arriving) lanes per item
        tma::prefetch_map(&tm.u);
        tma::prefetch_map(&tm.a);
        if (p.b) tma::prefetch_map(&tm.b);
        if (has_z) tma::prefetch_map(&tm.z);
        tma::prefetch_map(&tm.dy);
        tma::prefetch_map(&tm.B);
        tma::prefetch_map(&tm.C);
    }
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    const uint32_t tbase = sm.taddr;
    const uint32_t lane = (uint32_t)((warp & 3) * 32) << 16;
    const uint32_t trow = tbase + lane;  // this thread's TMEM row (channel)
    const int item = sm.item;
    // Work unit u = bb * ntiles + tile: 128 channels of one batch element.
    // Group mode: one (sequence group, unit) per block.  Piece mode: the
    // units' 64-token blocks, laid end to end, are cut into npieces equal
    // ranges; a block walks its range in order, so a unit cut in two has its
    // later part (tail) at the start of one range and its earlier part (head)
    // at the end of the previous range, and the tail's adjoint carry reaches
    // the head through the workspace (slot g = 0; head g = 0, tail g = 1).
    // Group mode is its own instantiation (no per-unit state to carry: it
    // keeps the register budget); the piece instantiation still reads the
    // mode at run time, which measured faster than folding it.
    const bool pieces = PIECES ? p.npieces > 0 : false;
    int g = 0, bb = 0, tile = 0, kb0 = 0, kb1 = 0;
    int64_t c0 = 0, c = 0, tg0 = 0, tg1 = 0;
    bool cvalid = false, lastg = true, firstg = true;
    float w0 = 0.f, w1 = 0.f, w2 = 0.f, w3 = 0.f, wb = 0.f, Dc = 0.f;
    int64_t goff = 0;  // (bb L) d + c: this thread's channel in the [Bt][L][d] outputs
    auto set_unit = [&](int u, int g_, int k0, int k1) {
        g = g_;
        bb = u / p.ntiles;
        tile = u % p.ntiles;
        c0 = (int64_t)tile * P;
        c = c0 + ch;
        cvalid = c < d;
        kb0 = k0;
        kb1 = k1;
        tg0 = (int64_t)kb0 * K;
        tg1 = min64(L, (int64_t)kb1 * K);
        lastg = kb1 == p.nsub;
        firstg = kb0 == 0;
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
        goff = (int64_t)bb * L * d + c;
    };
    // Per-unit output rows, formed where used (fewer live registers).
    auto gout = [&](void* base) { return static_cast<Tout*>(base) + goff; };
    auto part_row = [&]() {  // [L][2][N] dB / dC partials of this tile
        return p.dBCp + (((int64_t)tile * Bt + bb) * L) * 2 * N;
    };
    auto edge_row = [&]() { return p.conv_edge + ((int64_t)bb * p.ngroups + g) * 2 * 3 * d; };
    bool timed_out = false;

    // ------------------------------------------------ the item sequence
    // Per unit segment [k0, k1) of blocks: blocks last first; per block the
    // forward sweep's sub-chunks in order, then the backward sweep's in
    // reverse.  Group mode puts an early pass (the group's sub-chunks, last
    // first) in front when the group has a predecessor.
    const int nsbL = (int)((L - (int64_t)(p.nsub - 1) * K + T - 1) / T);  // last block's
    auto seg_items = [&](int k0, int k1) {
        return 2 * (4 * (k1 - k0) - (k1 == p.nsub ? 4 - nsbL : 0));
    };
    auto seg_t0 = [&](int j, int k0, int k1) -> int64_t {
        int k = k1 - 1, nsb = k1 == p.nsub ? nsbL : 4;
        if (j >= 2 * nsb) {
            j -= 2 * nsb;
            k = k1 - 2 - j / 8;
            j %= 8;
            nsb = 4;
        }
        const int sb = j < nsb ? j : 2 * nsb - 1 - j;
        return (int64_t)k * K + (int64_t)sb * T;
    };
    // Piece mode: this block's range [F0, F1) of the units' blocks.  Ranges
    // are taken in reverse ticket order, so the range holding a cut unit's
    // tail started before the one waiting for it.
    const int64_t Wb = Bt * p.ntiles * (int64_t)p.nsub;
    const int piece = pieces ? p.npieces - 1 - item : 0;
    const int64_t F0 = pieces ? (int64_t)piece * Wb / p.npieces : 0;
    const int64_t F1 = pieces ? (int64_t)(piece + 1) * Wb / p.npieces : 0;
    // Segment holding item li of the range: unit u, blocks [k0, k1); returns
    // the item's index inside the segment.
    auto piece_seg = [&](int li, int& u, int& k0, int& k1) -> int {
        u = (int)(F0 / p.nsub);
        for (;;) {
            const int64_t ub = (int64_t)u * p.nsub;
            k0 = (int)(max64(F0, ub) - ub);
            k1 = (int)(min64(F1, ub + p.nsub) - ub);
            const int n = seg_items(k0, k1);
            if (li < n || ub + p.nsub >= F1) return li;
            li -= n;
            ++u;
        }
    };
    int nE = 0, nitems = 0;
    if (pieces) {
        for (int64_t ub = (F0 / p.nsub) * p.nsub; ub < F1; ub += p.nsub)
            nitems += seg_items((int)(max64(F0, ub) - ub), (int)(min64(F1, ub + p.nsub) - ub));
    } else {
        const int per_g = (int)(Bt * p.ntiles);
        const int gg = p.ngroups - 1 - item / per_g;
        const int k0 = gg * p.blk_per_group;
        set_unit(item % per_g, gg, k0, min(k0 + p.blk_per_group, p.nsub));
        nE = firstg ? 0 : (int)((tg1 - tg0 + T - 1) / T);
        nitems = nE + seg_items(kb0, kb1);
    }
    // Input coordinates of item li: batch element, first channel, first token.
    auto item_at = [&](int li, int& zb, int& x) -> int64_t {
        if (pieces) {
            int u, k0, k1;
            const int j = piece_seg(li, u, k0, k1);
            zb = u / p.ntiles;
            x = (u % p.ntiles) * P;
            return seg_t0(j, k0, k1);
        }
        zb = bb;
        x = (int)c0;
        if (li < nE) return tg0 + (int64_t)(nE - 1 - li) * T;
        return seg_t0(li - nE, kb0, kb1);
    };
    auto issue = [&](int li) {  // one thread
        const int buf = li % Sm::NRAW;
        typename Sm::Raw& r = sm.raw[buf];
        uint64_t* mb = &sm.loaded[buf];
        const uint32_t bytes =
            (uint32_t)sizeof(Tin) *
            ((T + 3) * P + (2 + (has_z ? 1 : 0) + (has_b ? 1 : 0)) * T * P + 2 * T * N);
        tma::expect_tx(mb, bytes);
        int zb, x;
        const int y = (int)item_at(li, zb, x);
        tma::load_3d(&r.u[0][0], &tm.u, x, y - 3, zb, mb);
        tma::load_3d(&r.a[0][0], &tm.a, x, y, zb, mb);
        if (has_b) tma::load_3d(&r.b[0][0], &tm.b, x, y, zb, mb);
        if (has_z) tma::load_3d(&r.z[0][0], &tm.z, x, y, zb, mb);
        tma::load_3d(&r.dy[0][0], &tm.dy, x, y, zb, mb);
        tma::load_3d(&r.Bm[0][0], &tm.B, 0, y, zb, mb);
        tma::load_3d(&r.Cm[0][0], &tm.C, 0, y, zb, mb);
    };
    int li = 0;            // current item
    uint32_t mma_phase = 0;
    if (tid == 0)
        for (int q = 0; q < Sm::NRAW - 1 && q < nitems; ++q) issue(q);

    auto bf4 = [](const __nv_bfloat16* src) {
        const uint2 raw = *reinterpret_cast<const uint2*>(src);
        const float2 lo = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&raw.x));
        const float2 hi = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&raw.y));
        return make_float4(lo.x, lo.y, hi.x, hi.y);
    };
    auto sync = [&]() {
        tc::fence_before_sync();
        __syncthreads();
        tc::fence_after_sync();
    };
    // Transposed copy of TMEM columns [col, col + N) into the swizzled tile:
    // element (row j, k = channel).
    auto to_st = [&](uint32_t col) {
#pragma unroll
        for (int n0 = 0; n0 < NC; n0 += 16) {
            float v[16];
            tc::tmem_ld16(trow + col + qd * NC + n0, v);
            tc::tmem_ld_wait();
#pragma unroll
            for (int k = 0; k < 16; ++k)
                sm.st[tc::sw128_offset(qd * NC + n0 + k, ch, N) >> 2] = cvalid ? v[k] : 0.f;
        }
    };
    // TMEM columns [col, col + N) of this row <-> global rows (a quarter each).
    auto tmem_from = [&](uint32_t col, const float* src, bool cg) {
#pragma unroll
        for (int n0 = 0; n0 < NC; n0 += 16) {
            float v[16];
#pragma unroll
            for (int k = 0; k < 16; k += 4) {
                float4 v4 = make_float4(0.f, 0.f, 0.f, 0.f);
                if (src && cvalid) {
                    const float4* s4 =
                        reinterpret_cast<const float4*>(src + c * N + qd * NC + n0 + k);
                    v4 = cg ? __ldcg(s4) : *s4;
                }
                v[k] = v4.x;
                v[k + 1] = v4.y;
                v[k + 2] = v4.z;
                v[k + 3] = v4.w;
            }
            tc::tmem_st16(trow + col + qd * NC + n0, v);
        }
        tc::tmem_st_wait();
    };
    auto tmem_to = [&](uint32_t col, float* dst) {
#pragma unroll
        for (int n0 = 0; n0 < NC; n0 += 16) {
            float v[16];
            tc::tmem_ld16(trow + col + qd * NC + n0, v);
            tc::tmem_ld_wait();
            if (cvalid) {
#pragma unroll
                for (int k = 0; k < 16; k += 4)
                    *reinterpret_cast<float4*>(dst + c * N + qd * NC + n0 + k) =
                        make_float4(v[k], v[k + 1], v[k + 2], v[k + 3]);
            }
        }
    };
    // Dot of TMEM columns [ca, ca + N) and [cb, cb + N) of this row (all quarters).
    auto tmem_dot = [&](uint32_t ca, uint32_t cb) -> float {
        float acc = 0.f;
#pragma unroll
        for (int n0 = 0; n0 < NC; n0 += 16) {
            float va[16], vb[16];
            tc::tmem_ld16(trow + ca + qd * NC + n0, va);
            tc::tmem_ld16(trow + cb + qd * NC + n0, vb);
            tc::tmem_ld_wait();
#pragma unroll
            for (int k = 0; k < 16; ++k) acc = fmaf(va[k], vb[k], acc);
        }
        sm.xs[qd][ch] = acc;
        __syncthreads();
        acc = (sm.xs[0][ch] + sm.xs[1][ch]) + (sm.xs[2][ch] + sm.xs[3][ch]);
        __syncthreads();
        return acc;
    };
    // Scale-and-add on TMEM: col_a <- m * col_a + (col_b or a global row).
    auto tmem_axpy = [&](uint32_t ca, float m, uint32_t cb) {
#pragma unroll
        for (int n0 = 0; n0 < NC; n0 += 16) {
            float va[16], vb[16];
            tc::tmem_ld16(trow + ca + qd * NC + n0, va);
            tc::tmem_ld16(trow + cb + qd * NC + n0, vb);
            tc::tmem_ld_wait();
#pragma unroll
            for (int k = 0; k < 16; ++k) va[k] = fmaf(m, va[k], vb[k]);
            tc::tmem_st16(trow + ca + qd * NC + n0, va);
        }
        tc::tmem_st_wait();
    };

    // ------------------------------------------------- per-item state
    // Per (token, channel) values of this thread's 4 tokens; aux is SiLU'(z)
    // in the forward sweep and SiLU'(conv pre-activation) in the backward.
    float fv[TQ], qv[TQ], hv[TQ], iv[TQ], dyv[TQ], aux[TQ], Ev[TQ], Qv[TQ];
    float Elast = 1.f;
    bool slow = false;
    int nvh = 0;  // valid tokens of this thread's quarter

    // Unpack item `li` (raw buffer li % NRAW) for a sweep; fills the registers
    // above, the TMEM operand columns and the per-token tiles.  Returns after
    // a block-wide barrier.
    // sb: the sub-chunk's index in its 64-token block (main phase).  The
    // backward sweep reuses the forward sweep's decision and, with GCACHE and
    // the fused conv, its h and SiLU'(pre).
    auto prep = [&](int64_t t0, int64_t te, int sweep, int sb) {
        const typename Sm::Raw& r = sm.raw[li % Sm::NRAW];
        const bool fwd = sweep == kSweepFwd;
        constexpr bool CACHE = CONV && Cols::GCACHE;
        float hc[TQ], ac[TQ];
        if (CACHE && sweep == kSweepBwd) {
            tc::tmem_ld4(trow + Cols::GH + sb * T + qd * TQ, hc);
            tc::tmem_ld4(trow + Cols::GA + sb * T + qd * TQ, ac);
            tc::tmem_ld_wait();
        }
        // B and C rows to fp32.
        for (int e = tid; e < T * N / 4; e += NT) {
            const int tt = e / (N / 4), j = (e % (N / 4)) * 4;
            *reinterpret_cast<float4*>(&sm.brow[tt][j]) = bf4(&r.Bm[tt][j]);
            *reinterpret_cast<float4*>(&sm.crow[tt][j]) = bf4(&r.Cm[tt][j]);
        }
        nvh = cvalid ? (int)max((int64_t)0, min64((int64_t)TQ, te - t0 - qd * TQ)) : 0;
        float Qh = 1.f, Eh = 1.f;
#pragma unroll
        for (int k = 0; k < TQ; ++k) {
            const int tt = qd * TQ + k;
            const bool valid = k < nvh;
            const float ea = valid ? __expf(-to_f(r.a[tt][ch])) : 0.f;
            qv[k] = 1.f + ea;
            fv[k] = rcpa_(qv[k]);
            Qh *= qv[k];
            Eh *= fv[k];
            float hh, ax = 0.f;
            if (CACHE && sweep == kSweepBwd) {
                hh = hc[k];
                ax = ac[k];
            } else if (CONV) {
                const float pp = wb + w0 * to_f(r.u[tt][ch]) + w1 * to_f(r.u[tt + 1][ch]) +
                                 w2 * to_f(r.u[tt + 2][ch]) + w3 * to_f(r.u[tt + 3][ch]);
                const float sp = sigmoida_(pp);
                hh = pp * sp;
                ax = sp * fmaf(pp, 1.f - sp, 1.f);
                if (CACHE && fwd) {
                    hc[k] = valid ? hh : 0.f;
                    ac[k] = ax;
                }
            } else {
                hh = to_f(r.u[tt + 3][ch]);
            }
            hv[k] = valid ? hh : 0.f;
            iv[k] = has_b ? sigmoida_(to_f(r.b[tt][ch])) : ea * fv[k];
            float gg = 1.f;
            if (has_z) {
                const float zv = to_f(r.z[tt][ch]);
                const float sz = sigmoida_(zv);
                gg = zv * sz;
                if (fwd) ax = sz * fmaf(zv, 1.f - sz, 1.f);
            }
            aux[k] = ax;
            dyv[k] = valid ? to_f(r.dy[tt][ch]) * gg : 0.f;
        }
        if (CACHE && fwd) {
            tc::tmem_st4(trow + Cols::GH + sb * T + qd * TQ, hc);
            tc::tmem_st4(trow + Cols::GA + sb * T + qd * TQ, ac);
        }
        sm.xq[qd][ch] = Qh;
        sm.xe[qd][ch] = Eh;
        // The exchange barrier also ORs a conservative per-quarter test (not
        // needed by the backward sweep, which reuses the forward sweep's
        // decision); only when it fires does the exact test take a barrier.
        const bool maybe_slow = __syncthreads_or(sweep != kSweepBwd && !(Qh <= kBQuarter)) != 0;
        {
            // decay products of the earlier quarters and of the whole sub-chunk
            float Qb = 1.f, Eb = 1.f, Qa = 1.f, Ea = 1.f;
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                const float xq = sm.xq[q][ch], xe = sm.xe[q][ch];
                if (q < qd) {
                    Qb *= xq;
                    Eb *= xe;
                }
                Qa *= xq;
                Ea *= xe;
            }
            if (sweep == kSweepBwd) {
                slow = sm.slowf[sb] != 0;  // same sub-chunk as the forward sweep's
            } else {
                slow = maybe_slow && __syncthreads_or(qd == 0 && !(Qa <= kBBound)) != 0;
                if (fwd && tid == 0) sm.slowf[sb] = slow ? 1 : 0;
            }
            Elast = Ea;
            float Q = Qb, E = Eb;
#pragma unroll
            for (int k = 0; k < TQ; ++k) {
                E *= fv[k];
                Q *= qv[k];
                Ev[k] = E;
                Qv[k] = Q;
            }
        }
        // Per-(token, channel) operands.
        float c1[TQ], c2[TQ];
        const float QL = rcpa_(Elast);  // product of q over the sub-chunk (fast path)
#pragma unroll
        for (int k = 0; k < TQ; ++k) {
            const int tt = qd * TQ + k;
            const float v = iv[k] * hv[k];
            if (fwd) {
                // W (readout weights), V (state weights), Y = s dy E.
                const float W = slow ? v : v * Qv[k];
                c1[k] = W;
                c2[k] = slow ? fv[k] : W * Elast;
                const float Y = slow ? s * dyv[k] : s * dyv[k] * Ev[k];
                sm.y1[tt][ch] = Y;
                sm.w1[tt][ch] = W;
                if (!slow) sm.pk[tc::sw128_offset(tt, ch, T) >> 2] = cvalid ? Y : 0.f;
            } else {
                // U = s dy E / Elast, s dy E (adjoint weights), P = v Elast / E.
                const float sdy = s * dyv[k];
                c1[k] = slow ? sdy : sdy * Ev[k] * QL;
                c2[k] = slow ? fv[k] : sdy * Ev[k];
                if (sweep == kSweepBwd) {
                    const float Pv = slow ? v : v * Elast * Qv[k];
                    sm.y1[tt][ch] = Pv;
                    sm.w1[tt][ch] = c1[k];
                    if (!slow) sm.pk[tc::sw128_offset(tt, ch, T) >> 2] = cvalid ? Pv : 0.f;
                }
            }
        }
        tc::tmem_st4(trow + Cols::WU + qd * TQ, c1);
        tc::tmem_st4(trow + Cols::VV + qd * TQ, c2);
        tc::tmem_st_wait();
        if (!slow) {
            // K-major per-token tiles (all threads; brow / crow are complete
            // since the exchange barrier).
            for (int e = tid; e < T * N / 4; e += NT) {
                const int rest = e >> 3;
                const int tt = (rest & 1) * 8 + (e & 7), j = (rest >> 1) * 4;
                // ta: rows t, K = d_state (C forward, B backward)
                *reinterpret_cast<float4*>(&sm.ta[tc::kmajor_offset(tt, j, N) >> 2]) =
                    fwd ? *reinterpret_cast<const float4*>(&sm.crow[tt][j])
                        : *reinterpret_cast<const float4*>(&sm.brow[tt][j]);
                // ts: rows d_state, K = 16 (B^T forward, C^T backward)
                const int jj = e % N, m0 = (e / N) * 4;
                const float(*src)[N + 4] = fwd ? sm.brow : sm.crow;
                *reinterpret_cast<float4*>(&sm.ts[tc::kmajor_offset(jj, m0, T) >> 2]) =
                    make_float4(src[m0][jj], src[m0 + 1][jj], src[m0 + 2][jj], src[m0 + 3][jj]);
            }
        }
        tc::fence_proxy_async();
        sync();  // y1, w1, pk, tiles and the TMEM operand columns complete
        // Prefetch: buffer (li + NRAW - 1) % NRAW was last read by item li - 1.
        // Issued here, by a thread that neither computes the small products nor
        // issues MMAs, so it overlaps the MMA wait.
        if (tid == 160 && li + Sm::NRAW - 1 < nitems) issue(li + Sm::NRAW - 1);
    };

    // The small per-sub-chunk products on warps 0-3 (warp-level tf32 MMAs):
    // warps 0, 1 take halves (64 channels each) of A_C[t][m] = sum_ch Y_t W_m
    // (m <= t) or A_B[t][t'] = sum_ch P_t U_t' (t' >= t) -> ta2; warps 2, 3
    // halves (d_state / 2 each) of the Gram, forward G[t][m] = C_t . B_m
    // (m <= t), backward G^T[t][t'] = C_t' . B_t (t' >= t) -> tg.  The MMAs
    // accumulate both halves.
    auto small_products = [&](bool fwd) {
        float dd[2][4];
        float* dst;
        const int h = warp & 1;
        if (warp < 2) {
            tc::warp_gram16<P / 2, P + 4>(&sm.y1[0][h * (P / 2)], &sm.w1[0][h * (P / 2)], dd);
            dst = sm.ta2[h];
        } else {
            const int k0 = h * (N / 2);
            tc::warp_gram16<N / 2, N + 4>(fwd ? &sm.crow[0][k0] : &sm.brow[0][k0],
                                          fwd ? &sm.brow[0][k0] : &sm.crow[0][k0], dd);
            dst = sm.tg[h];
        }
        const int lane = tid & 31, gq = lane >> 2, kq = lane & 3;
#pragma unroll
        for (int n = 0; n < 2; ++n)
#pragma unroll
            for (int r = 0; r < 4; ++r) {
                const int row = gq + (r >> 1) * 8, col = 8 * n + 2 * kq + (r & 1);
                const bool live = fwd ? (col <= row) : (col >= row);
                dst[tc::kmajor_offset(row, col, T) >> 2] = live ? dd[n][r] : 0.f;
            }
    };

    // MMAs of the current item, in independent accumulation chains: chain 0,
    // readout (forward: X . C + W G) or dv (backward: H . B + U G^T) into R;
    // chain 1, state (forward: V B^T) or adjoint (backward: (s dy E) C^T)
    // into D; chain 2, dC or dB ((state^T)(Y or P) over channels + (B^T or
    // C^T)(A_C or A_B)) into BC; chain 3 (d_state 64), the second half of
    // the channel sum into BC2.
    auto issue_chain = [&](int chain, int sweep) {
        constexpr uint32_t id16 = tc::idesc_tf32(128, T);
        constexpr uint32_t idN = tc::idesc_tf32(128, N);
        if (chain == 3) {  // second half of the dC / dB channel sum into BC2
            const uint32_t a_st = tc::smem_u32(sm.st), a_pk = tc::smem_u32(sm.pk);
#pragma unroll
            for (int i = P / 16; i < P / 8; ++i)
                tc::mma_tf32_ss(tbase + Cols::BC2,
                                tc::sdesc_sw128(a_st + (i >> 2) * N * 128 + (i & 3) * 32),
                                tc::sdesc_sw128(a_pk + (i >> 2) * T * 128 + (i & 3) * 32), id16,
                                i > P / 16 ? 1u : 0u);
            return;
        }
        if (chain == 0) {
            const uint32_t a_ta = tc::smem_u32(sm.ta), a_tg = tc::smem_u32(&sm.tg[0][0]);
            const uint32_t Acol = sweep == kSweepFwd ? Cols::X : Cols::G;
#pragma unroll
            for (int i = 0; i < N / 8; ++i)
                tc::mma_tf32_ts(tbase + Cols::R, tbase + Acol + i * 8,
                                tc::sdesc(a_ta + i * 256, 128, 32 * N), id16, i > 0 ? 1u : 0u);
#pragma unroll
            for (int i = 0; i < 2 * (T / 8); ++i)  // both partial Gram tiles
                tc::mma_tf32_ts(tbase + Cols::R, tbase + Cols::WU + (i % (T / 8)) * 8,
                                tc::sdesc(a_tg + (i / (T / 8)) * T * T * 4 + (i % (T / 8)) * 256,
                                          128, 32 * T),
                                id16, 1u);
        } else if (chain == 1) {
            const uint32_t a_ts = tc::smem_u32(sm.ts);
#pragma unroll
            for (int i = 0; i < T / 8; ++i)
                tc::mma_tf32_ts(tbase + Cols::D, tbase + Cols::VV + i * 8,
                                tc::sdesc(a_ts + i * 256, 128, 32 * T), idN, i > 0 ? 1u : 0u);
        } else {
            const uint32_t a_ts = tc::smem_u32(sm.ts), a_t2 = tc::smem_u32(&sm.ta2[0][0]);
            const uint32_t a_st = tc::smem_u32(sm.st), a_pk = tc::smem_u32(sm.pk);
            constexpr int KE = Cols::SPLIT ? P / 16 : P / 8;  // K steps of this chain
#pragma unroll
            for (int i = 0; i < KE; ++i)
                tc::mma_tf32_ss(tbase + Cols::BC,
                                tc::sdesc_sw128(a_st + (i >> 2) * N * 128 + (i & 3) * 32),
                                tc::sdesc_sw128(a_pk + (i >> 2) * T * 128 + (i & 3) * 32), id16,
                                i > 0 ? 1u : 0u);
#pragma unroll
            for (int i = 0; i < 2 * (T / 8); ++i) {  // both partial A_C / A_B tiles
                const int kk = i % (T / 8), hh = i / (T / 8);
                tc::mma_tf32_ss(tbase + Cols::BC, tc::sdesc(a_ts + kk * 256, 128, 32 * T),
                                tc::sdesc(a_t2 + hh * T * T * 4 + kk * 256, 128, 32 * T), id16,
                                1u);
            }
        }
    };

    // Start item li: prefetch the next one, wait for this one's inputs.
    auto begin_item = [&]() {
        if (!tc::mbar_wait(&sm.loaded[li % Sm::NRAW], (uint32_t)((li / Sm::NRAW) & 1), kBSpin))
            timed_out = true;
    };
    // Three arrivals on sm.mma per item.  Warp 4 issues the chains that need
    // no small product (1, and 3 for d_state 64) at once; warps 0-3 compute
    // the small products meanwhile, meet on named barrier 1, and lanes 0 of
    // warps 0 and 1 issue chains 0 and 2.  The early sweep runs chain 1 only.
    auto run_mma = [&](int sweep) {
        const bool full = sweep != kSweepEarly;
        if (full && warp < 4) {
            small_products(sweep == kSweepFwd);
            tc::fence_proxy_async();
            tc::named_bar(1, 128);
        }
        if ((tid & 31) == 0) {
            if (warp == 4) {
                tc::fence_after_sync();
                issue_chain(1, sweep);
                if (Cols::SPLIT && full) issue_chain(3, sweep);
                tc::mma_commit(&sm.mma);
            } else if (warp < 2) {
                if (full) {
                    tc::fence_after_sync();
                    issue_chain(warp == 0 ? 0 : 2, sweep);
                    tc::mma_commit(&sm.mma);
                } else {
                    tc::mbar_arrive(&sm.mma);
                }
            }
        }
        // One warp (it issues nothing) polls the completion barrier; the rest
        // wait on the block barrier instead of spinning.
        if (warp == NT / 32 - 1 && !tc::mbar_wait(&sm.mma, mma_phase, kBSpin)) timed_out = true;
        __syncthreads();
        mma_phase ^= 1u;
        tc::fence_after_sync();
    };
    // Write a [16][N] channel-sum tile (slot 0 dB, 1 dC) from TMEM BC (lanes
    // = d_state rows, columns = tokens) to the per-tile partial buffer.
    auto write_bc_tmem = [&](int slot, int64_t t0, int64_t te) {
        if ((warp & 3) * 32 < N) {
            float v[TQ];
            tc::tmem_ld4(tbase + lane + Cols::BC + qd * TQ, v);
            if (Cols::SPLIT) {
                float v2[TQ];
                tc::tmem_ld4(tbase + lane + Cols::BC2 + qd * TQ, v2);
                tc::tmem_ld_wait();
#pragma unroll
                for (int k = 0; k < TQ; ++k) v[k] += v2[k];
            }
            tc::tmem_ld_wait();
            const int j = ch;  // lane = d_state row
#pragma unroll
            for (int k = 0; k < TQ; ++k) {
                const int64_t t = t0 + qd * TQ + k;
                if (t < te) part_row()[t * 2 * N + slot * N + j] = v[k];
            }
        } else {
            // keep the warp's tcgen05.ld count uniform per lane quadrant
        }
    };
    auto write_bc_smem = [&](int slot, int64_t t0, int64_t te) {
        for (int e = tid; e < T * N; e += NT) {
            const int tt = e / N, j = e % N;
            const int64_t t = t0 + tt;
            if (t < te) part_row()[t * 2 * N + slot * N + j] = sm.acc[tt][j];
        }
    };
    auto warp_sum = [](float v) {
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
        return v;
    };

    // ----------------------------------------------------------------
    // Exact forward sub-chunk: token recurrence on this thread's quarter of
    // the state columns; x.C partial sums added over the quarters in sm.w1;
    // dC channel sums into sm.acc.  Requires sm.acc and sm.w1 zeroed.
    auto fwd_exact = [&](float* ydot) {
        float vv[16], ff[16];
        tc::tmem_ld16(trow + Cols::WU, vv);
        tc::tmem_ld16(trow + Cols::VV, ff);
        tc::tmem_ld_wait();
        float yp[16];
#pragma unroll
        for (int tt = 0; tt < T; ++tt) yp[tt] = 0.f;
        for (int n0 = qd * NC; n0 < qd * NC + NC; n0 += 16) {
            float x[16];
            tc::tmem_ld16(trow + Cols::X + n0, x);
            tc::tmem_ld_wait();
            for (int tt = 0; tt < T; ++tt) {
                const float sdy = cvalid ? sm.y1[tt][ch] : 0.f;
                float a = 0.f;
#pragma unroll
                for (int k = 0; k < 16; ++k) {
                    x[k] = fmaf(ff[tt], x[k], vv[tt] * sm.brow[tt][n0 + k]);
                    a = fmaf(x[k], sm.crow[tt][n0 + k], a);
                    const float r = warp_sum(sdy * x[k]);
                    if ((tid & 31) == 0) atomicAdd(&sm.acc[tt][n0 + k], r);
                }
                yp[tt] += a;
            }
            tc::tmem_st16(trow + Cols::X + n0, x);
        }
        tc::tmem_st_wait();
#pragma unroll
        for (int tt = 0; tt < T; ++tt) atomicAdd(&sm.w1[tt][ch], yp[tt]);
        __syncthreads();
#pragma unroll
        for (int k = 0; k < TQ; ++k) ydot[k] = sm.w1[qd * TQ + k][ch];
        float lp = 0.f;
#pragma unroll
        for (int tt = 0; tt < T; ++tt) lp += __logf(ff[tt]);
        return lp;
    };
    // Exact backward sub-chunk: adjoint recurrence over this quarter of the
    // columns, G.B summed over the quarters in sm.w1, dB channel sums into
    // sm.acc.  Requires sm.acc and sm.w1 zeroed when `grads`.
    auto bwd_exact = [&](float* gbv, bool grads) {
        float sd[16], ff[16];
        tc::tmem_ld16(trow + Cols::WU, sd);
        tc::tmem_ld16(trow + Cols::VV, ff);
        tc::tmem_ld_wait();
        float gp[16];
#pragma unroll
        for (int tt = 0; tt < T; ++tt) gp[tt] = 0.f;
        for (int n0 = qd * NC; n0 < qd * NC + NC; n0 += 16) {
            float hx[16];
            tc::tmem_ld16(trow + Cols::G + n0, hx);
            tc::tmem_ld_wait();
            for (int tt = T - 1; tt >= 0; --tt) {
                const float v = (grads && cvalid) ? sm.y1[tt][ch] : 0.f;
                float a = 0.f;
#pragma unroll
                for (int k = 0; k < 16; ++k) {
                    const float gk = fmaf(sd[tt], sm.crow[tt][n0 + k], hx[k]);
                    if (grads) {
                        a = fmaf(gk, sm.brow[tt][n0 + k], a);
                        const float r = warp_sum(v * gk);
                        if ((tid & 31) == 0) atomicAdd(&sm.acc[tt][n0 + k], r);
                    }
                    hx[k] = ff[tt] * gk;
                }
                gp[tt] += a;
            }
            tc::tmem_st16(trow + Cols::G + n0, hx);
        }
        tc::tmem_st_wait();
        if (grads) {
#pragma unroll
            for (int tt = 0; tt < T; ++tt) atomicAdd(&sm.w1[tt][ch], gp[tt]);
            __syncthreads();
#pragma unroll
            for (int k = 0; k < TQ; ++k) gbv[k] = sm.w1[qd * TQ + k][ch];
        }
        float lp = 0.f;
#pragma unroll
        for (int tt = 0; tt < T; ++tt) lp += __logf(ff[tt]);
        return lp;
    };

    // ====================================================== early pass
    // Adjoint only over the group (last sub-chunk first) to publish the
    // carry leaving the group's start.
    // (Group mode.)  Carry slots: group mode, the carry entering group g's
    // end in slot g; piece mode, a cut unit's carry in slot 0.
    auto carry_slot = [&](int slot) { return p.carry + ((int64_t)slot * Bt + bb) * d * N; };
    auto flag_slot = [&](int slot) { return p.flags + ((int64_t)slot * Bt + bb) * p.ntiles + tile; };
    if (!pieces && !firstg) {
        float* carry_in = carry_slot(g);
        const float* dxf = p.dx_final ? p.dx_final + (int64_t)bb * d * N : nullptr;
        tmem_from(Cols::G, lastg ? dxf : nullptr, false);
        float logF = 0.f;
        for (int e = 0; e < nE; ++e, ++li) {
            int zb_, x_;
            const int64_t t0 = item_at(li, zb_, x_);
            begin_item();
            prep(t0, tg1, kSweepEarly, 0);
            if (!slow) {
                run_mma(kSweepEarly);
                tmem_axpy(Cols::G, Elast, Cols::D);
                logF += __logf(Elast);
            } else {
                float dummy[TQ];
                logF += bwd_exact(dummy, false);
            }
            sync();
        }
        if (!lastg) {
            if (tid == 0) sm.ok = wait_flag(flag_slot(g), &p.hdr->status, p.wait_limit) ? 1 : 0;
            __syncthreads();
            const bool okc = sm.ok != 0;
            // carry out = (decay over the group) H + local contribution
            const float Pf = __expf(logF);
#pragma unroll
            for (int n0 = 0; n0 < NC; n0 += 16) {
                float hx[16];
                tc::tmem_ld16(trow + Cols::G + qd * NC + n0, hx);
                tc::tmem_ld_wait();
#pragma unroll
                for (int k = 0; k < 16; k += 4) {
                    float4 v4 = make_float4(0.f, 0.f, 0.f, 0.f);
                    if (okc && cvalid)
                        v4 = __ldcg(reinterpret_cast<const float4*>(carry_in + c * N + qd * NC +
                                                                    n0 + k));
                    hx[k] = fmaf(Pf, v4.x, hx[k]);
                    hx[k + 1] = fmaf(Pf, v4.y, hx[k + 1]);
                    hx[k + 2] = fmaf(Pf, v4.z, hx[k + 2]);
                    hx[k + 3] = fmaf(Pf, v4.w, hx[k + 3]);
                }
                tc::tmem_st16(trow + Cols::G + qd * NC + n0, hx);
            }
            tc::tmem_st_wait();
        }
        tmem_to(Cols::G, carry_slot(g - 1));
        __threadfence();
        __syncthreads();
        if (tid == 0 && !(lastg && p.fault_skip_publish)) st_release(flag_slot(g - 1), 1);
    }

    // ====================================================== main phase
    // Per unit segment [kb0, kb1) (group mode: the one set above), from the
    // carry entering its end.
    const int64_t ub_first = pieces ? (F0 / p.nsub) * p.nsub : 0;
    const int64_t ub_end = pieces ? F1 : 1;
    for (int64_t ub = ub_first; ub < ub_end; ub += pieces ? p.nsub : 1) {
    if (pieces) {
        const int k0 = (int)(max64(F0, ub) - ub), k1 = (int)(min64(F1, ub + p.nsub) - ub);
        set_unit((int)(ub / p.nsub), k0 > 0 ? 1 : 0, k0, k1);
    }
    if (lastg) {
        tmem_from(Cols::G, p.dx_final ? p.dx_final + (int64_t)bb * d * N : nullptr, false);
    } else {
        const int slot = pieces ? 0 : g;
        if (tid == 0) sm.ok = wait_flag(flag_slot(slot), &p.hdr->status, p.wait_limit) ? 1 : 0;
        __syncthreads();
        tmem_from(Cols::G, sm.ok ? carry_slot(slot) : nullptr, true);
    }
    // dp beyond the group: zero (the next group's terms go via the edge fixup)
    for (int i = tid; i < 3 * P; i += NT) (&sm.dp[1][0][0])[i] = 0.f;
    int bi = 0;  // backward-sweep items so far (dp buffer bi & 1; the later sub-chunk's in the other)
    sync();

    // ====================================================== main: blocks
    float dD_acc = 0.f, dw0 = 0.f, dw1 = 0.f, dw2 = 0.f, dw3 = 0.f, dbias = 0.f;
    for (int k = kb1 - 1; k >= kb0; --k) {
        const int64_t tb = (int64_t)k * K;
        const int64_t te = min64(L, tb + K);
        const int nsb = (int)((te - tb + T - 1) / T);
        const bool group_end_block = (k == kb1 - 1);
        // state entering the block (forward checkpoint)
        tmem_from(Cols::X, p.ckpt + ((int64_t)bb * (p.nck + 1) + k) * d * N, false);
        to_st(Cols::X);
        sync();

        // --------------------------------------------- forward sweep
        for (int sb = 0; sb < nsb; ++sb, ++li) {
            const int64_t t0 = tb + (int64_t)sb * T;
            begin_item();
            prep(t0, te, kSweepFwd, sb);
            float yd[TQ];  // x_t . C_t of this thread's tokens
            if (!slow) {
                run_mma(kSweepFwd);
                float r[TQ];
                tc::tmem_ld4(trow + Cols::R + qd * TQ, r);
                tc::tmem_ld_wait();
#pragma unroll
                for (int q = 0; q < TQ; ++q) yd[q] = Ev[q] * r[q];
                write_bc_tmem(1, t0, te);
                tmem_axpy(Cols::X, Elast, Cols::D);
            } else {
                for (int e = tid; e < T * N; e += NT) (&sm.acc[0][0])[e] = 0.f;
                for (int e = tid; e < T * (P + 4); e += NT) (&sm.w1[0][0])[e] = 0.f;
                __syncthreads();
                fwd_exact(yd);
                __syncthreads();
                write_bc_smem(1, t0, te);
            }
            // dz and s dy (x.C) for the backward sweep
            {
                const typename Sm::Raw& r = sm.raw[li % Sm::NRAW];
                float dl[TQ];
#pragma unroll
                for (int q = 0; q < TQ; ++q) {
                    const int tt = qd * TQ + q;
                    dl[q] = s * dyv[q] * yd[q];
                    if (has_z && q < nvh) {
                        const float yv = fmaf(s, yd[q], Dc * hv[q]);
                        gout(p.dz)[(t0 + tt) * d] = from_f<Tout>(to_f(r.dy[tt][ch]) * yv * aux[q]);
                    }
                }
                tc::tmem_st4(trow + Cols::DL + sb * T + qd * TQ, dl);
                tc::tmem_st_wait();
            }
            // State entering the next sub-chunk: each thread copies its own TMEM
            // columns (no barrier needed; the next item's MMAs follow its
            // unpacking barriers).
            to_st(Cols::X);
        }
        // (f df) tail of this block: carry entering the block's end . state at its end
        const float tail = tmem_dot(Cols::G, Cols::X);

        // --------------------------------------------- backward sweep
        to_st(Cols::G);
        sync();
        float cum = 0.f;  // sum of dL over the later tokens of the block
        for (int sb = nsb - 1; sb >= 0; --sb, ++li) {
            const int64_t t0 = tb + (int64_t)sb * T;
            begin_item();
            prep(t0, te, kSweepBwd, sb);
            float gbv[TQ];
            if (!slow) {
                run_mma(kSweepBwd);
                float r[TQ];
                tc::tmem_ld4(trow + Cols::R + qd * TQ, r);
                tc::tmem_ld_wait();
#pragma unroll
                for (int q = 0; q < TQ; ++q) gbv[q] = Elast * Qv[q] * r[q];
                write_bc_tmem(0, t0, te);
                tmem_axpy(Cols::G, Elast, Cols::D);
            } else {
                for (int e = tid; e < T * N; e += NT) (&sm.acc[0][0])[e] = 0.f;
                for (int e = tid; e < T * (P + 4); e += NT) (&sm.w1[0][0])[e] = 0.f;
                __syncthreads();
                bwd_exact(gbv, true);
                __syncthreads();
                write_bc_smem(0, t0, te);
            }
            // per-(token, channel) gradients
            const typename Sm::Raw& r = sm.raw[li % Sm::NRAW];
            float dl[TQ];
            tc::tmem_ld4(trow + Cols::DL + sb * T + qd * TQ, dl);
            tc::tmem_ld_wait();
            float sfx[TQ];
            float run = 0.f;
#pragma unroll
            for (int q = TQ - 1; q >= 0; --q) {
                run += dl[q] - iv[q] * hv[q] * gbv[q];
                sfx[q] = run;
            }
            // conv dp (needs no suffix sums) into this item's buffer
            float(*dpc)[P] = sm.dp[bi & 1];
            const float(*dpl)[P] = sm.dp[(bi & 1) ^ 1];  // the later sub-chunk's (halo)
            float dhv[TQ];
#pragma unroll
            for (int q = 0; q < TQ; ++q) {
                const int tt = qd * TQ + q;
                dhv[q] = fmaf(Dc, dyv[q], iv[q] * gbv[q]);
                if (CONV) {
                    float dpv = 0.f;
                    if (q < nvh) {
                        dpv = dhv[q] * aux[q];
                        dw0 = fmaf(dpv, to_f(r.u[tt][ch]), dw0);
                        dw1 = fmaf(dpv, to_f(r.u[tt + 1][ch]), dw1);
                        dw2 = fmaf(dpv, to_f(r.u[tt + 2][ch]), dw2);
                        dw3 = fmaf(dpv, to_f(r.u[tt + 3][ch]), dw3);
                        dbias += dpv;
                    }
                    dpc[tt][ch] = dpv;
                }
            }
            sm.xs[qd][ch] = run;
            __syncthreads();  // suffix partials and dp complete
            float later = 0.f, total = 0.f;  // sums of dL over later quarters / all
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                const float v = sm.xs[q][ch];
                if (q > qd) later += v;
                total += v;
            }
            const float base = cum + tail + later;
            cum += total;
#pragma unroll
            for (int q = 0; q < TQ; ++q) {
                const int tt = qd * TQ + q;
                const int64_t t = t0 + tt;
                if (q < nvh) {
                    if (has_b) {
                        gout(p.da)[t * d] = from_f<Tout>((base + sfx[q]) * (1.f - fv[q]));
                        gout(p.db)[t * d] = from_f<Tout>(hv[q] * gbv[q] * iv[q] * (1.f - iv[q]));
                    } else {  // da = (f df - f di)(1 - f), di = h G.B; 1 - f = i
                        gout(p.da)[t * d] =
                            from_f<Tout>((base + sfx[q] - fv[q] * hv[q] * gbv[q]) * iv[q]);
                    }
                    dD_acc = fmaf(dyv[q], hv[q], dD_acc);
                    if (CONV) {
                        // du_t = w3 dp_t + w2 dp_{t+1} + w1 dp_{t+2} + w0 dp_{t+3}
                        auto dpat = [&](int row) {
                            return row < T ? dpc[row][ch] : dpl[row - T][ch];
                        };
                        const float duv = w3 * dpc[tt][ch] + w2 * dpat(tt + 1) +
                                          w1 * dpat(tt + 2) + w0 * dpat(tt + 3);
                        if (!lastg && group_end_block && t >= te - 3) {
                            edge_row()[(3 + (t - (te - 3))) * d + c] = duv;  // partial, fixed up later
                        } else {
                            gout(p.dhu)[t * d] = from_f<Tout>(duv);
                        }
                        if (k == kb0 && sb == 0 && tt < 3) edge_row()[tt * d + c] = dpc[tt][ch];
                    } else {
                        gout(p.dhu)[t * d] = from_f<Tout>(dhv[q]);
                    }
                }
            }
            ++bi;
            // Carry entering the earlier sub-chunk's end: own TMEM columns, no
            // barrier needed (see the forward sweep).
            to_st(Cols::G);
        }
    }

    // ------------------------------------------------ carries and partials
    if (firstg) {
        if (p.dx0) tmem_to(Cols::G, p.dx0 + (int64_t)bb * d * N);
    } else if (pieces) {
        // the tail of a cut unit: publish the carry leaving its start
        tmem_to(Cols::G, carry_slot(0));
        __threadfence();
        __syncthreads();
        if (tid == 0 && !p.fault_skip_publish) st_release(flag_slot(0), 1);
    }
    {
        float* cpart = p.chan_part + ((int64_t)bb * p.ngroups + g) * d * 8;
        float* red6 = &sm.acc[0][0];  // [6][P] (T * N >= 6 * P)
        __syncthreads();
        for (int i = tid; i < 6 * P; i += NT) red6[i] = 0.f;
        __syncthreads();
        if (cvalid) {
            atomicAdd(&red6[0 * P + ch], dD_acc);
            atomicAdd(&red6[1 * P + ch], dw0);
            atomicAdd(&red6[2 * P + ch], dw1);
            atomicAdd(&red6[3 * P + ch], dw2);
            atomicAdd(&red6[4 * P + ch], dw3);
            atomicAdd(&red6[5 * P + ch], dbias);
        }
        __syncthreads();
        if (tid < P && c0 + tid < d) {
#pragma unroll
            for (int q = 0; q < 6; ++q) cpart[(c0 + tid) * 8 + q] = red6[q * P + tid];
            if (pieces && firstg && lastg) {  // uncut unit: its tail slot stays empty
                float* cp1 = p.chan_part + ((int64_t)bb * p.ngroups + 1) * d * 8;
#pragma unroll
                for (int q = 0; q < 6; ++q) cp1[(c0 + tid) * 8 + q] = 0.f;
            }
        }
    }
    }  // unit segments

    if (timed_out) atomicOr(&p.hdr->status, 1 << NAJU_ERR_TIMEOUT);
    sync();
    if (warp == 0) tc::tmem_dealloc(tbase, Cols::ALLOC);
}

template <typename Tout, int N, bool CONV, bool PIECES>
static cudaError_t launch_bwd_tc_t(const BwdParams& p, cudaStream_t st) {
    BwdTmaps tm;
    memset(&tm, 0, sizeof(tm));
    const int T = kBT;
    bool ok = tma_encode_bf16_3d(&tm.u, p.hu, p.Bt, p.L, p.d, T + 3, 128) &&
              tma_encode_bf16_3d(&tm.a, p.a, p.Bt, p.L, p.d, T, 128) &&
              (!p.b || tma_encode_bf16_3d(&tm.b, p.b, p.Bt, p.L, p.d, T, 128)) &&
              tma_encode_bf16_3d(&tm.dy, p.dy, p.Bt, p.L, p.d, T, 128) &&
              tma_encode_bf16_3d(&tm.B, p.B, p.Bt, p.L, N, T, N) &&
              tma_encode_bf16_3d(&tm.C, p.C, p.Bt, p.L, N, T, N);
    if (ok && p.z) ok = tma_encode_bf16_3d(&tm.z, p.z, p.Bt, p.L, p.d, T, 128);
    if (!ok) return cudaErrorInvalidValue;
    const size_t smem = sizeof(BwdTcSmem<N>);
    auto kern = scan_bwd_tc_kernel<Tout, N, CONV, PIECES>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)smem);
    if (e != cudaSuccess) return e;
    const int grid = p.npieces > 0 ? p.npieces : p.ngroups * (int)p.Bt * p.ntiles;
    kern<<<grid, 512, smem, st>>>(p, tm);
    return cudaGetLastError();
}

bool bwd_tc_supported(int dtype, int64_t N, int64_t d) {
    return dtype == NAJU_BF16 && (N == 64 || N == 128) && d % 8 == 0;
}

cudaError_t launch_scan_bwd_tc_main(const BwdParams& p, int out_dtype, cudaStream_t st) {
    const bool conv = p.conv_w != nullptr;
    const bool pc = p.npieces > 0;
#define NAJU_TC_BWD(TO, NN)                                                          \
    return conv ? (pc ? launch_bwd_tc_t<TO, NN, true, true>(p, st)                   \
                      : launch_bwd_tc_t<TO, NN, true, false>(p, st))                 \
                : (pc ? launch_bwd_tc_t<TO, NN, false, true>(p, st)                  \
                      : launch_bwd_tc_t<TO, NN, false, false>(p, st))
    if (out_dtype == NAJU_BF16) {
        if (p.N == 64) NAJU_TC_BWD(__nv_bfloat16, 64);
        if (p.N == 128) NAJU_TC_BWD(__nv_bfloat16, 128);
    } else {
        if (p.N == 64) NAJU_TC_BWD(float, 64);
        if (p.N == 128) NAJU_TC_BWD(float, 128);
    }
#undef NAJU_TC_BWD
    return cudaErrorInvalidValue;
}

}  // namespace naju
