// Naju backward scan in block form on the 5th-generation tensor cores
// (sm_100a, tcgen05, kind::f16 with fp32 accumulation), for bf16 activations
// with d_state 64 (d_state 128 as two passes over 64-column state halves).
//
// Gradient of the Naju recurrence (Naju reproduction README, "Core
// equations"): x_n = f_n x_{n-1} + i_n h_n B_n^T, y_n = x_n.C_n/sqrt(N) + D h_n,
// out = y SiLU(z), h = SiLU(conv(u)); s = 1/sqrt(N), v = i h, dy = dout SiLU(z).
//
// A thread block owns 128 channels of one batch element (one channel per
// tensor-memory lane) and walks its 64-token blocks from the last to the
// first.  A block needs only the state X entering it (the forward pass's
// checkpoint) and the adjoint carry H entering its end (H = f_next lambda_next,
// from the later block).  Relative to the block start, per channel, with
// E_t = prod_{k<=t} f_k, Q_t = 1/E_t, W_t = v_t Q_t, U_t = s dy_t E_t,
// H' = E_63 H and G[t][m] = C_t.B_m kept for m <= t:
//   x_t . C_t       = E_t R_t,   R  = X C^T + W G^T
//   lambda_t . B_t  = Q_t GB_t,  GB = H' B^T + U G      (G read transposed)
//   carry out       = U C + H'   (the adjoint carry entering the earlier block)
//   dC_t = sum_ch U_t X + sum_{m<=t} P[t][m] B_m,     P = U^T W (over channels)
//   dB_t = sum_ch W_t H' + sum_{t'>=t} P[t'][t] C_t'
//   dL_t = U_t R_t - W_t GB_t,  (f df)_t = sum_{t'>=t} dL_t' + H . x_63,
//   da = (f df)(1 - f), dz = dout y SiLU'(z), dh = D dy + i lambda.B,
//   db = h (lambda.B) i (1 - i), and the conv backward from dp = dh SiLU'(p).
// Every product runs on the tensor core (kind::f16, fp32 accumulation).  Each
// fp32 operand is held as a pair of bf16 tiles, hi = bf16(v) and
// lo = bf16(v - hi), and a product takes the three terms hi.hi + hi.lo + lo.hi
// (about 2^-16 relative error, finer than tf32); B and C are bf16 inputs and
// exact in one tile.  The tiles are 128-byte swizzled row tiles (rows =
// channels or tokens); for 16-bit elements the same bytes serve as the K-major
// operand (contraction over the columns) and as the MN-major operand
// (contraction over the rows: over channels for P, dC, dB, over tokens for
// the carry and for GB), so no thread ever transposes an operand.  The 64 x 64
// products G and P (M = 64) share tensor-memory columns at lane offsets 0 and
// 16, and later dC^T and dB^T do the same.
//
// Data movement.  Every input of a block arrives by TMA while the block
// before it (the later one) finishes: the per-token inputs u (with its 3-token
// conv halo), a, b, z and dout into shared memory that the carry, G and P tiles
// occupy only between the two phases that need them; B and C straight into
// their swizzled tiles; the fp32 checkpoint into the X tiles' bytes, which the
// block turns into its hi / lo pair.  bf16 gradients dz, db, da and dh (du)
// are written to shared memory in the W and U tiles' bytes once the block no
// longer reads them and leave by TMA stores, which clip the ragged edges.
//
// Threads.  512: warp w handles tensor-memory lanes 32 (w % 4) .. + 31, i.e.
// channels 32 (w % 4) + lane, and the 16 tokens [16 q, 16 q + 16) of the
// block, q = w / 4 (and the state columns [16 q, 16 q + 16) where a channel's
// state row is split); the per-token coefficients the gradients need after
// the MMAs wait in tensor memory and registers.
//
// Exactness.  A block in which some channel's decay product over the block
// falls below 2^-90 (the factorisation's range) runs an exact token-by-token
// recurrence instead, on the CUDA cores, and hands its results to the same
// epilogue through tensor memory.
//
// dB and dC: each block adds its channels' partial sums into an fp32
// accumulator with red.global.add (a small kernel converts it to the output
// dtype), so no per-tile partial sets go through HBM.  Sequence groups
// (below one wave of 128-channel units) and piece mode (at least one wave)
// split the work exactly as in the sub-chunk tensor-core backward.
#include <stddef.h>
#include <string.h>

#include <type_traits>

#include "naju_common.cuh"
#include "naju_kernels.h"
#include "naju_tc.cuh"
#include "naju_tma.h"
namespace naju {

namespace {

constexpr int kK = 64;    // tokens per block (the forward's checkpoint spacing)
constexpr int kP = 128;   // channels per unit
constexpr int kN = 64;    // d_state
constexpr int kNT = 512;  // threads
constexpr float kBound = 1.2379400392853803e27f;  // 2^90
constexpr float kQuarter = 4194304.f;             // 2^22: four quarters below it stay below 2^88
constexpr long long kSpin = 1LL << 24;
// The tensor-core chains of a block are issued by lanes 0 of warps 0..5 (one
// accumulator per thread, so each chain keeps its order): committing
// threads per completion barrier.
constexpr int kIss0 = 2;  // G (warp 0), P (warp 5); the exact path arrives for P
constexpr int kIss2 = 3;  // R (1), GB (2), carry (3)
constexpr int kIss3 = 2;  // dC (1), dB (2)
// the thread that stores a block's staged gradients (not an MMA issuer)
constexpr int kStoreTid = 7 * 32;

// Tensor-memory columns (lane = channel unless stated).
struct BkCols {
    static constexpr uint32_t R = 0;     // R[ch][t]           (64)
    static constexpr uint32_t GB = 64;   // GB[ch][t]          (64)
    static constexpr uint32_t H = 128;   // carry [ch][j]      (64)
    static constexpr uint32_t BC = 192;  // G / P, then dC^T / dB^T (M = 64 at lanes +0 / +16)
    // four per-token coefficients [ch][t]: s dzc E, dzc D h, the db (coupled:
    // da) coefficient, 1 - f; slots 2 and 3 first hold f and 1/f
    static constexpr uint32_t SV = 256;
};

struct alignas(64) BkTmaps {
    CUtensorMap u, a, b, z, dy;  // bf16 [Bt][L][d]: 64 tokens (u: 67) x 128 channels
    CUtensorMap B, C;            // bf16 [Bt][L][N]: 64 tokens x 64 columns, swizzled
    CUtensorMap X;               // fp32 checkpoints [Bt (nck+1)][d][N]: 128 x 32, swizzled
    CUtensorMap oz, ob, oa, ou;  // bf16 outputs dz, db, da, dh (du): 64 tokens x 128 channels
    CUtensorMap pr, pg;          // second d_state-128 pass: partial R, GB [Bt][L][d] fp32 (L2 prefetch)
};

// Shared memory, 1024-byte aligned tiles.  Region A (the carry, G and P tile
// pairs) is dead from the end of one block's products to the next block's
// carry scaling and takes that block's per-token inputs in between; the W and
// U pairs take the staged bf16 outputs once the second-to-last pass is done;
// the X pair takes the next fp32 checkpoint once the block's tail sum has
// read it.
struct BkSmem {
    alignas(1024) __nv_bfloat16 Xh[kP * kN], Xl[kP * kN];  // checkpoint: rows ch, cols j
    alignas(1024) __nv_bfloat16 Wh[kP * kK], Wl[kP * kK];  // rows ch, cols t
    alignas(1024) __nv_bfloat16 Uh[kP * kK], Ul[kP * kK];  // rows ch, cols t
    alignas(1024) __nv_bfloat16 Bs[kK * kN], Cs[kK * kN];  // rows t, cols j (exact)
    // region A
    alignas(1024) __nv_bfloat16 Hh[kP * kN], Hl[kP * kN];  // H' = E_63 H: rows ch, cols j
    __nv_bfloat16 Gh[kK * kK], Gl[kK * kK];                // rows t, cols m (m <= t)
    __nv_bfloat16 Ph[kK * kK], Pl[kK * kK];                // rows t, cols m (m <= t)
    alignas(1024) __nv_bfloat16 ru[(kK + 3) * kP];         // u of tokens tb - 3 .. tb + 63
    float xq[4][kP], xe[4][kP];   // per-quarter decay products
    float xs[4][kP];              // per-quarter sums of dL
    float tailp[2][4][kP];        // partial H . x_63 of the next block to run
    float dph[4][3][kP];          // first three dp of each quarter
    float dnext[2][3][kP];        // first three dp of the later block
    float red6[6][kP];            // per-channel parameter sums
    uint64_t mb_in, mb_bc, mb_x, mb0, mb2, mb3, mb_e;
    uint32_t taddr;
    int item, ok;
};
static_assert(offsetof(BkSmem, Pl) + sizeof(BkSmem::Pl) - offsetof(BkSmem, Hh) == 4 * kK * kP * 2,
              "region A holds the four raw per-token inputs");
static_assert(sizeof(BkSmem::Xh) + sizeof(BkSmem::Xl) == kP * kN * 4, "fp32 checkpoint");
static_assert(sizeof(BkSmem) <= 232448, "shared memory");

__device__ __forceinline__ float bf2f(__nv_bfloat16 v) {
    return __uint_as_float((uint32_t)__bfloat16_as_ushort(v) << 16);
}
__device__ __forceinline__ float bf_lo(uint32_t v) { return __uint_as_float(v << 16); }
__device__ __forceinline__ float bf_hi(uint32_t v) { return __uint_as_float(v & 0xffff0000u); }
__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}
__device__ __forceinline__ void red_add(float* p, float v) {
    asm volatile("red.global.add.f32 [%0], %1;" ::"l"(p), "f"(v) : "memory");
}
// Four consecutive floats (p 16-byte aligned) in one reduction.
__device__ __forceinline__ void red_add4(float* p, float a, float b, float c, float d) {
    asm volatile("red.global.add.v4.f32 [%0], {%1, %2, %3, %4};" ::"l"(p), "f"(a), "f"(b),
                 "f"(c), "f"(d)
                 : "memory");
}
// The dB / dC accumulator holds tokens in chunks of four, innermost:
// [Bt][ceil(L / 4)][2][N][4] (slot 0 dB, 1 dC), so one thread's four
// consecutive tokens of a state column are one 16-byte reduction.
__host__ __device__ __forceinline__ int64_t dbc_index(int64_t b, int64_t t, int slot, int64_t col,
                                                       int64_t L, int64_t N) {
    const int64_t L4 = (L + 3) >> 2;
    return (((b * L4 + (t >> 2)) * 2 + slot) * N + col) * 4 + (t & 3);
}
// hi = bf16(a, b) (round to nearest), lo = bf16 of the remainders.
__device__ __forceinline__ void split2(float a, float b, uint32_t& hi, uint32_t& lo) {
    const __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
    const float2 hf = __bfloat1622float2(h);
    const __nv_bfloat162 l = __floats2bfloat162_rn(a - hf.x, b - hf.y);
    hi = *reinterpret_cast<const uint32_t*>(&h);
    lo = *reinterpret_cast<const uint32_t*>(&l);
}
// Eight consecutive values into a tile pair at byte offset o (one 16-byte
// chunk of each).
__device__ __forceinline__ void st8o(__nv_bfloat16* th, __nv_bfloat16* tl, uint32_t o,
                                     const float* v) {
    uint4 h, l;
    split2(v[0], v[1], h.x, l.x);
    split2(v[2], v[3], h.y, l.y);
    split2(v[4], v[5], h.z, l.z);
    split2(v[6], v[7], h.w, l.w);
    *reinterpret_cast<uint4*>(reinterpret_cast<char*>(th) + o) = h;
    *reinterpret_cast<uint4*>(reinterpret_cast<char*>(tl) + o) = l;
}
// Four consecutive values (hi + lo) from a tile pair at byte offset o.
__device__ __forceinline__ void ld4o(const __nv_bfloat16* th, const __nv_bfloat16* tl, uint32_t o,
                                     float* v) {
    const uint2 h = *reinterpret_cast<const uint2*>(reinterpret_cast<const char*>(th) + o);
    const uint2 l = *reinterpret_cast<const uint2*>(reinterpret_cast<const char*>(tl) + o);
    v[0] = bf_lo(h.x) + bf_lo(l.x);
    v[1] = bf_hi(h.x) + bf_hi(l.x);
    v[2] = bf_lo(h.y) + bf_lo(l.y);
    v[3] = bf_hi(h.y) + bf_hi(l.y);
}
// One value (hi + lo) of a tile pair, and one value of an exact tile.
__device__ __forceinline__ float ld1(const __nv_bfloat16* th, const __nv_bfloat16* tl, int row,
                                     int col) {
    const uint32_t o = tc::bf_offset(row, col);
    return bf2f(*reinterpret_cast<const __nv_bfloat16*>(reinterpret_cast<const char*>(th) + o)) +
           bf2f(*reinterpret_cast<const __nv_bfloat16*>(reinterpret_cast<const char*>(tl) + o));
}
__device__ __forceinline__ float ld1(const __nv_bfloat16* t, int row, int col) {
    return bf2f(*reinterpret_cast<const __nv_bfloat16*>(reinterpret_cast<const char*>(t) +
                                                          tc::bf_offset(row, col)));
}

}  // namespace

// MODE 0: d_state 64.  d_state 128 runs twice over 64-column halves of the
// state (the columns evolve independently; only R, GB and the tail sums
// couple them, and linearly): MODE 1 takes columns 0..63 and writes its
// partial R, GB and tails to p.rgb_part / p.tail_part (no gradients of the
// per-token inputs), MODE 2 takes columns 64..127, adds them and finishes.
// The carry, dB, dC and the initial-state gradient split by columns.
template <typename Tout, bool CONV, bool PIECES, int MODE>
__global__ void __launch_bounds__(512, 1)
scan_bwd_blk_kernel(const BwdParams p, const __grid_constant__ BkTmaps tm) {
    constexpr int NS = MODE == 0 ? kN : 2 * kN;  // d_state (row stride of states)
    constexpr int JH = MODE == 2 ? kN : 0;    // this pass's first state column
    constexpr bool kExport = MODE == 1;
    constexpr bool kImport = MODE == 2;
    // bf16 gradients leave through shared memory and TMA stores; fp32 ones
    // are stored directly
    constexpr bool kStage = !kExport && std::is_same<Tout, __nv_bfloat16>::value;
    using Cols = BkCols;
    using Sm = BkSmem;
    extern __shared__ __align__(1024) float4 smem4[];
    Sm& sm = *reinterpret_cast<Sm*>(smem4);

    const int tid = threadIdx.x;
    const int warp = tid >> 5, lid = tid & 31;
    const int s4 = warp & 3;       // tensor-memory sub-partition
    const int q = warp >> 2;       // token quarter / state-column quarter
    const int ch = s4 * 32 + lid;  // channel within the unit = TMEM lane
    const int64_t Bt = p.Bt, L = p.L, d = p.d;
    const float sc = p.scale;
    const bool has_z = p.z != nullptr;
    const bool has_b = p.b != nullptr;

    // ------------------------------------------------------------ set-up
    if (warp == 0) {
        tc::tmem_alloc(&sm.taddr, 512);
        tc::tmem_relinquish();
    }
    if (tid == 0) {
        sm.item = atomicAdd(&p.hdr->bwd_ticket, 1);
        tc::mbar_init(&sm.mb_in, 1);
        tc::mbar_init(&sm.mb_bc, 1);
        tc::mbar_init(&sm.mb_x, 1);
        tc::mbar_init(&sm.mb0, kIss0);  // G and P
        tc::mbar_init(&sm.mb2, kIss2);  // the chains the epilogue reads
        tc::mbar_init(&sm.mb3, kIss3);  // dB and dC
        tc::mbar_init(&sm.mb_e, 1);     // the early pass's carry
        tma::prefetch_map(&tm.X);
        tma::prefetch_map(&tm.u);
        tma::prefetch_map(&tm.a);
        if (has_b) tma::prefetch_map(&tm.b);
        if (has_z) tma::prefetch_map(&tm.z);
        tma::prefetch_map(&tm.dy);
        tma::prefetch_map(&tm.B);
        tma::prefetch_map(&tm.C);
        if constexpr (kStage) {
            tma::prefetch_map(&tm.oa);
            tma::prefetch_map(&tm.ou);
            if (has_z) tma::prefetch_map(&tm.oz);
            if (has_b) tma::prefetch_map(&tm.ob);
        }
    }
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    const uint32_t tbase = sm.taddr;
    const uint32_t trow = tbase + ((uint32_t)(s4 * 32) << 16);  // this warp's lanes
    const int item = sm.item;
    const uint32_t sbase = tc::smem_u32(&sm);
// tile start addresses / 16 (the base is 1024-byte aligned: checked below)
#define NAJU_SA(f) (sb4 + (uint32_t)(offsetof(Sm, f) >> 4))
    const uint32_t sb4 = sbase >> 4;
    const bool aligned1k = (sbase & 1023u) == 0;  // the swizzled tiles need it
    if (!aligned1k && tid == 0) atomicOr(&p.hdr->status, 1 << NAJU_ERR_INVALID_ARG);
    uint32_t ph_in = 0, ph_bc = 0, ph_x = 0, ph0 = 0, ph2 = 0, ph3 = 0, ph_e = 0;  // mbarrier parities
    bool timed_out = false;

    // This thread's two 16-byte chunks (columns [16 q, 16 q + 8) and
    // [16 q + 8, 16 q + 16) of row ch) in every row tile with rows = channels.
    const uint32_t oc0 = tc::bf_offset(ch, 16 * q), oc1 = tc::bf_offset(ch, 16 * q + 8);
    // Element offset of (token 16 q, channel ch) in a [64][128] per-token
    // buffer (raw inputs, staged outputs).
    const int ro = 16 * q * kP + ch;
    // the raw per-token inputs in region A
    auto region_a = [&](int i) {
        return reinterpret_cast<__nv_bfloat16*>(reinterpret_cast<char*>(&sm) + offsetof(Sm, Hh) +
                                                (size_t)i * kK * kP * 2);
    };
    __nv_bfloat16* const ra = region_a(0);
    __nv_bfloat16* const rb = region_a(1);
    __nv_bfloat16* const rz = region_a(2);
    __nv_bfloat16* const rdy = region_a(3);

    // ------------------------------------------------------------ work units
    constexpr bool pieces = PIECES;  // the launch picks the instantiation by p.npieces
    int g = 0, bb = 0, tile = 0, kb0 = 0, kb1 = 0;
    int64_t c0 = 0, c = 0;
    bool cvalid = false, lastg = true, firstg = true;
    float w0 = 0.f, w1 = 0.f, w2 = 0.f, w3 = 0.f, wb = 0.f, Dc = 0.f;
    auto set_unit = [&](int u, int g_, int k0, int k1) {
        g = g_;
        bb = u / p.ntiles;
        tile = u % p.ntiles;
        c0 = (int64_t)tile * kP;
        c = c0 + ch;
        cvalid = c < d;
        kb0 = k0;
        kb1 = k1;
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
    };
    const int64_t Wb = Bt * p.ntiles * (int64_t)p.nsub;
    const int piece = pieces ? p.npieces - 1 - item : 0;
    const int64_t F0 = pieces ? (int64_t)piece * Wb / p.npieces : 0;
    const int64_t F1 = pieces ? (int64_t)(piece + 1) * Wb / p.npieces : 0;
    if (!pieces) {
        const int per_g = (int)(Bt * p.ntiles);
        const int gg = p.ngroups - 1 - item / per_g;
        const int k0 = gg * p.blk_per_group;
        set_unit(item % per_g, gg, k0, min(k0 + p.blk_per_group, p.nsub));
    }
    auto carry_slot = [&](int slot) { return p.carry + ((int64_t)slot * Bt + bb) * d * NS; };
    auto flag_slot = [&](int slot) {
        return p.flags + ((int64_t)slot * Bt + bb) * p.ntiles + tile;
    };
    auto edge_row = [&]() { return p.conv_edge + ((int64_t)bb * p.ngroups + g) * 2 * 3 * d; };
    auto ck_at = [&](int k) { return p.ckpt + ((int64_t)bb * (p.nck + 1) + k) * d * NS; };

    auto sync = [&]() {
        tc::fence_before_sync();
        __syncthreads();
        tc::fence_after_sync();
    };
    // Bounded mbarrier waits: one warp polls (until a first time-out), the
    // others wait at the block barrier.
    auto wait_mb = [&](uint64_t* mb, uint32_t& ph) {
        if (warp == kNT / 32 - 1 && !timed_out && !tc::mbar_wait(mb, ph, kSpin)) timed_out = true;
        __syncthreads();
        ph ^= 1u;
        tc::fence_after_sync();
    };
    auto wait_mb2 = [&](uint64_t* ma, uint32_t& pa, uint64_t* mb, uint32_t& pb) {
        if (warp == kNT / 32 - 1 && !timed_out &&
            !(tc::mbar_wait(ma, pa, kSpin) && tc::mbar_wait(mb, pb, kSpin)))
            timed_out = true;
        __syncthreads();
        pa ^= 1u;
        pb ^= 1u;
        tc::fence_after_sync();
    };
    // TMEM carry columns of this thread (state columns [16 q, 16 q + 16)) <->
    // a global [d][N] state row.
    auto carry_from = [&](const float* src, bool cg) {
        float v[16];
#pragma unroll
        for (int k = 0; k < 16; k += 4) {
            float4 v4 = make_float4(0.f, 0.f, 0.f, 0.f);
            if (src && cvalid) {
                const float4* s4p = reinterpret_cast<const float4*>(src + c * NS + JH + 16 * q + k);
                v4 = cg ? __ldcg(s4p) : *s4p;
            }
            v[k] = v4.x; v[k + 1] = v4.y; v[k + 2] = v4.z; v[k + 3] = v4.w;
        }
        tc::tmem_st16(trow + Cols::H + 16 * q, v);
        tc::tmem_st_wait();
    };
    auto carry_to = [&](float* dst) {
        float v[16];
        tc::tmem_ld16(trow + Cols::H + 16 * q, v);
        tc::tmem_ld_wait();
        if (cvalid) {
#pragma unroll
            for (int k = 0; k < 16; k += 4)
                *reinterpret_cast<float4*>(dst + c * NS + JH + 16 * q + k) =
                    make_float4(v[k], v[k + 1], v[k + 2], v[k + 3]);
        }
    };

    // ------------------------------------------------------- TMA loads
    // Per-token inputs of block k (thread 0): full: u, a, b, z, dout;
    // adjoint only: a, z, dout.
    auto load_raw = [&](int k, bool full) {
        const int x = (int)c0, y = k * kK, zb = bb;
        uint32_t rows = kK * (2 + (has_z ? 1 : 0));
        if (full) rows += (kK + 3) + (has_b ? kK : 0);
        tma::expect_tx(&sm.mb_in, rows * kP * 2u);
        tma::load_3d(ra, &tm.a, x, y, zb, &sm.mb_in);
        tma::load_3d(rdy, &tm.dy, x, y, zb, &sm.mb_in);
        if (has_z) tma::load_3d(rz, &tm.z, x, y, zb, &sm.mb_in);
        if (full) {
            tma::load_3d(sm.ru, &tm.u, x, y - 3, zb, &sm.mb_in);
            if (has_b) tma::load_3d(rb, &tm.b, x, y, zb, &sm.mb_in);
        }
    };
    // The same inputs of a full block in two steps: u (its own buffer) with
    // the expected bytes of all five, then the four in region A.
    auto load_raw_u = [&](int k) {
        const uint32_t rows = kK * (2 + (has_z ? 1 : 0) + (has_b ? 1 : 0)) + (kK + 3);
        tma::expect_tx(&sm.mb_in, rows * kP * 2u);
        tma::load_3d(sm.ru, &tm.u, (int)c0, k * kK - 3, bb, &sm.mb_in);
    };
    auto load_raw_a = [&](int k) {
        const int x = (int)c0, y = k * kK, zb = bb;
        tma::load_3d(ra, &tm.a, x, y, zb, &sm.mb_in);
        tma::load_3d(rdy, &tm.dy, x, y, zb, &sm.mb_in);
        if (has_z) tma::load_3d(rz, &tm.z, x, y, zb, &sm.mb_in);
        if (has_b) tma::load_3d(rb, &tm.b, x, y, zb, &sm.mb_in);
    };
    // C (and B when full) of block k into their tiles (thread 0).
    auto load_bc = [&](int k, bool full) {
        tma::expect_tx(&sm.mb_bc, (uint32_t)(2 * kK * kN * (full ? 2 : 1)));
        tma::load_3d(sm.Cs, &tm.C, JH, k * kK, bb, &sm.mb_bc);
        if (full) tma::load_3d(sm.Bs, &tm.B, JH, k * kK, bb, &sm.mb_bc);
    };
    // The fp32 checkpoint entering block k into the X tiles' bytes (thread 0):
    // two swizzled boxes of 32 state columns.
    auto load_x = [&](int k) {
        tma::expect_tx(&sm.mb_x, (uint32_t)(kP * kN * 4));
        const int zz = (int)((int64_t)bb * (p.nck + 1) + k);
        tma::load_3d(sm.Xh, &tm.X, JH, (int)c0, zz, &sm.mb_x);
        tma::load_3d(sm.Xl, &tm.X, JH + 32, (int)c0, zz, &sm.mb_x);
    };
    // This thread's 16 checkpoint values from the fp32 landing layout (box
    // q / 2, chunks 4 (q % 2) .. + 3 of row ch, XOR-permuted by ch % 8).
    auto read_x = [&](float* xr) {
        const char* base = reinterpret_cast<const char*>(sm.Xh) + (q >> 1) * 16384 + ch * 128;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const float4 v =
                *reinterpret_cast<const float4*>(base + ((((q & 1) * 4 + i) ^ (ch & 7)) << 4));
            xr[4 * i] = v.x; xr[4 * i + 1] = v.y; xr[4 * i + 2] = v.z; xr[4 * i + 3] = v.w;
        }
    };

    // ---------------------------------------------------- loop 1: decays
    // f and 1/f of this thread's 16 tokens, parked in tensor memory (slots 2
    // and 3); exchange of the quarter products; the exact-path decision.
    float Eb = 1.f, Qb = 1.f, E63 = 1.f;
    // Tokens past the end (last block only) decay by 1; channels past d
    // read zeros (finite values that are never stored).
    auto decays = [&](int nv) -> bool {
        const __nv_bfloat16* rap = ra + ro;
        float fv[16], qv[16];
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
        tc::tmem_st16(trow + Cols::SV + 2 * 64 + 16 * q, fv);
        tc::tmem_st16(trow + Cols::SV + 3 * 64 + 16 * q, qv);
        sm.xq[q][ch] = Qh;
        sm.xe[q][ch] = Eh;
        // the previous block's staged gradients must have left the W / U bytes
        // before unpack rewrites them (this barrier orders the wait)
        if (kStage && tid == kStoreTid) tma::store_wait_read();
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
        tc::tmem_st_wait();
        return maybe && __syncthreads_or(!(Qa <= kBound)) != 0;
    };

    // ------------------------------------------------ full unpack (loop 2)
    // Writes the W, U tile pairs, four coefficients per token (tensor memory)
    // and keeps c0v, c1v (dp = c0 + c1 GB) and the u window in registers.
    float c0v[16], c1v[16];
    uint32_t upk[10] = {};  // u at tokens 16q-3 .. 16q+15 (bf16 pairs)
    float dD_acc = 0.f;     // this block's sum of dy h (added to red6 in phase C)
    // u of window entry m (token 16q - 3 + m of the block)
    auto uwin = [&](int m) { return (m & 1) ? bf_hi(upk[m >> 1]) : bf_lo(upk[m >> 1]); };
    // No token masks: past the end, dout, B and C read zero, so U, GB and
    // dp = c0 + c1 GB vanish and W meets only zero rows; the decays mask.
    auto unpack_v = [&](bool slow, auto hb_c, auto hz_c) {
        constexpr bool has_b = decltype(hb_c)::value;
        constexpr bool has_z = decltype(hz_c)::value;
        const unsigned short* rup = reinterpret_cast<const unsigned short*>(sm.ru) + ro;
        const __nv_bfloat16* rbp = rb + ro;
        const __nv_bfloat16* rzp = rz + ro;
        const __nv_bfloat16* rdp = rdy + ro;
#pragma unroll
        for (int i = 0; i < 10; ++i)
            upk[i] = (uint32_t)rup[(2 * i) * kP] |
                     (i < 9 ? (uint32_t)rup[(2 * i + 1) * kP] << 16 : 0u);
        float E = slow ? sc : sc * Eb, Q = slow ? 1.f : Qb;  // E carries the scale s
        dD_acc = 0.f;
        uint32_t pk[8];  // packed W, U hi / lo of the previous group of four
#pragma unroll
        for (int g4 = 0; g4 < 4; ++g4) {
            float Wv[4], Uv[4], s0[4], s1[4], s2[4], s3[4], fa[4], qa[4];
            float hv[4], spd[4], iw[4], gg[4], gd[4], dout[4];
            const int col = 16 * q + 4 * g4;
            tc::tmem_ld4(trow + Cols::SV + 2 * 64 + col, fa);
            tc::tmem_ld4(trow + Cols::SV + 3 * 64 + col, qa);
#pragma unroll
            for (int k4 = 0; k4 < 4; ++k4) {
                const int k = 4 * g4 + k4;
                if (CONV) {
                    const float pp = fmaf(w3, uwin(k + 3), fmaf(w2, uwin(k + 2),
                                         fmaf(w1, uwin(k + 1), fmaf(w0, uwin(k), wb))));
                    const float sp = sigmoidx_(pp);
                    hv[k4] = pp * sp;
                    spd[k4] = sp * fmaf(pp, 1.f - sp, 1.f);
                } else {
                    hv[k4] = uwin(k + 3);
                    spd[k4] = 1.f;
                }
                dout[k4] = bf2f(rdp[k * kP]);
            }
            if (has_b) {
#pragma unroll
                for (int k4 = 0; k4 < 4; ++k4) iw[k4] = sigmoidx_(bf2f(rbp[(4 * g4 + k4) * kP]));
            }
            if (has_z) {
#pragma unroll
                for (int k4 = 0; k4 < 4; ++k4) {
                    const float zv = bf2f(rzp[(4 * g4 + k4) * kP]);
                    const float sz = sigmoidx_(zv);
                    gg[k4] = zv * sz;
                    gd[k4] = sz * fmaf(zv, 1.f - sz, 1.f);
                }
            } else {
#pragma unroll
                for (int k4 = 0; k4 < 4; ++k4) {
                    gg[k4] = 1.f;
                    gd[k4] = 0.f;
                }
            }
            tc::tmem_ld_wait();
#pragma unroll
            for (int k4 = 0; k4 < 4; ++k4) {
                const int k = 4 * g4 + k4;
                const float f = fa[k4], qq = qa[k4], h = hv[k4];
                // 1 - f = (1/f - 1) f, exact for f near 1; 1 where exp(-a) overflowed
                const float omf = qq < 3.0e38f ? (qq - 1.f) * f : 1.f;
                const float i = has_b ? iw[k4] : omf;
                const float dyv = dout[k4] * gg[k4];
                const float dzc = dout[k4] * gd[k4];
                if (!slow) {
                    E *= f;
                    Q *= qq;
                }
                const float iQ = i * Q;
                Wv[k4] = iQ * h;
                Uv[k4] = dyv * E;
                s0[k4] = dzc * E;                                        // dz = s0 R + s1
                s1[k4] = dzc * Dc * h;
                s2[k4] = has_b ? Wv[k4] * (1.f - i) : f * h * Q;         // db = s2 GB
                s3[k4] = omf;
                c1v[k] = iQ * spd[k4];                                   // dp = c0 + c1 GB
                c0v[k] = Dc * dyv * spd[k4];
                dD_acc = fmaf(dyv, h, dD_acc);
            }
            {   // W and U hi / lo: one 16-byte chunk per tile every second group
                uint32_t wh0, wl0, wh1, wl1, uh0, ul0, uh1, ul1;
                split2(Wv[0], Wv[1], wh0, wl0);
                split2(Wv[2], Wv[3], wh1, wl1);
                split2(Uv[0], Uv[1], uh0, ul0);
                split2(Uv[2], Uv[3], uh1, ul1);
                if ((g4 & 1) == 0) {
                    pk[0] = wh0; pk[1] = wh1; pk[2] = wl0; pk[3] = wl1;
                    pk[4] = uh0; pk[5] = uh1; pk[6] = ul0; pk[7] = ul1;
                } else {
                    const uint32_t o = g4 < 2 ? oc0 : oc1;
                    auto st = [&](__nv_bfloat16* t, uint4 v) {
                        *reinterpret_cast<uint4*>(reinterpret_cast<char*>(t) + o) = v;
                    };
                    st(sm.Wh, make_uint4(pk[0], pk[1], wh0, wh1));
                    st(sm.Wl, make_uint4(pk[2], pk[3], wl0, wl1));
                    st(sm.Uh, make_uint4(pk[4], pk[5], uh0, uh1));
                    st(sm.Ul, make_uint4(pk[6], pk[7], ul0, ul1));
                }
            }
            if constexpr (!kExport) {
                tc::tmem_st4(trow + Cols::SV + 0 * 64 + col, s0);
                tc::tmem_st4(trow + Cols::SV + 1 * 64 + col, s1);
                tc::tmem_st4(trow + Cols::SV + 2 * 64 + col, s2);
            }
            tc::tmem_st4(trow + Cols::SV + 3 * 64 + col, s3);
        }
    };
    // (four variants: b and z present or not)
    auto unpack = [&](bool slow) {
        if (p.b != nullptr) {
            if (p.z != nullptr) unpack_v(slow, std::true_type{}, std::true_type{});
            else unpack_v(slow, std::true_type{}, std::false_type{});
        } else {
            if (p.z != nullptr) unpack_v(slow, std::false_type{}, std::true_type{});
            else unpack_v(slow, std::false_type{}, std::false_type{});
        }
    };

    // H' = E_63 H into tensor memory and (tiles) into the H tile pair (its
    // initial value: carry out = U C + H').
    auto scale_carry = [&](bool tiles) {
        float hv[16];
        tc::tmem_ld16(trow + Cols::H + 16 * q, hv);
        tc::tmem_ld_wait();
#pragma unroll
        for (int j = 0; j < 16; ++j) hv[j] *= E63;
        if (tiles) {
            st8o(sm.Hh, sm.Hl, oc0, hv);
            st8o(sm.Hh, sm.Hl, oc1, hv + 8);
        }
        tc::tmem_st16(trow + Cols::H + 16 * q, hv);
    };

    // --------------------------------------------------------- the MMAs
    const uint32_t lane16 = 16u << 16;
    // one product A.B over K steps ks < nks, into d (accumulating unless first)
    // (a, b: tile start addresses / 16; a K step of 16 elements is 32 bytes
    // along a K-major row, 16 rows = 2048 bytes of an MN-major tile)
    auto prod = [&](uint32_t dcol, uint32_t a, bool a_mn, uint32_t b, bool b_mn, int nks,
                    uint32_t idesc, bool& first) {
#pragma unroll
        for (int ks = 0; ks < nks; ++ks) {
            const uint64_t ad = a_mn ? tc::sdesc_sw128_mn_a4(a + ks * 128u, 1024)
                                     : tc::sdesc_sw128_a4(a + ks * 2u);
            const uint64_t bd = b_mn ? tc::sdesc_sw128_mn_a4(b + ks * 128u, 1024)
                                     : tc::sdesc_sw128_a4(b + ks * 2u);
            tc::mma_bf16_ss(dcol, ad, bd, idesc, first ? 0u : 1u);
            first = false;
        }
    };
    // the three terms of a split product (hi.hi + hi.lo + lo.hi)
    auto prod3 = [&](uint32_t dcol, uint32_t ah, uint32_t al, bool a_mn, uint32_t bh, uint32_t bl,
                     bool b_mn, int nks, uint32_t idesc, bool& first) {
        prod(dcol, ah, a_mn, bh, b_mn, nks, idesc, first);
        prod(dcol, ah, a_mn, bl, b_mn, nks, idesc, first);
        prod(dcol, al, a_mn, bh, b_mn, nks, idesc, first);
    };
    // and of a product with an exact operand B (hi.B + lo.B)
    auto prod2 = [&](uint32_t dcol, uint32_t ah, uint32_t al, bool a_mn, uint32_t b, bool b_mn,
                     int nks, uint32_t idesc, bool& first) {
        prod(dcol, ah, a_mn, b, b_mn, nks, idesc, first);
        prod(dcol, al, a_mn, b, b_mn, nks, idesc, first);
    };
    // Batch 0: G = C B^T (lanes +0), P = U^T W (lanes +16), M = 64.
    // Batch 1: R = X C^T, GB = H' B^T, carry += U C.
    // Each accumulator's chain is issued by one thread (lane 0 of warp
    // `issuer`), so the chains run side by side and keep their own order.
    const int issuer = lid == 0 ? warp : -1;
    // G as soon as B and C have landed (thread 0 waits for them), at the start
    // of phase A; P and R once W, U and X are in their tiles; GB and the
    // carry once H' is.
    auto issue_g = [&]() {
        if (issuer == 0) {
            if (!timed_out && !tc::mbar_wait(&sm.mb_bc, ph_bc, kSpin)) timed_out = true;
            bool f = true;
            prod(tbase + Cols::BC, NAJU_SA(Cs), false, NAJU_SA(Bs), false, kN / 16,
                 tc::idesc_bf16(64, 64), f);
            tc::mma_commit(&sm.mb0);
        }
    };
    auto issue_pr = [&]() {
        if (issuer == 5) {
            bool f = true;
            prod3(tbase + lane16 + Cols::BC, NAJU_SA(Uh), NAJU_SA(Ul), true, NAJU_SA(Wh),
                  NAJU_SA(Wl), true, kP / 16, tc::idesc_bf16(64, 64, true, true), f);
            tc::mma_commit(&sm.mb0);
        } else if (issuer == 1) {
            bool f = true;
            prod2(tbase + Cols::R, NAJU_SA(Xh), NAJU_SA(Xl), false, NAJU_SA(Cs), false, kN / 16,
                  tc::idesc_bf16(128, 64), f);
        }
    };
    auto issue_gbh = [&]() {
        if (issuer == 2) {
            bool f = true;
            prod2(tbase + Cols::GB, NAJU_SA(Hh), NAJU_SA(Hl), false, NAJU_SA(Bs), false, kN / 16,
                  tc::idesc_bf16(128, 64), f);
        } else if (issuer == 3) {
            bool f = false;
            prod2(tbase + Cols::H, NAJU_SA(Uh), NAJU_SA(Ul), false, NAJU_SA(Cs), true, kK / 16,
                  tc::idesc_bf16(128, kN, false, true), f);
            tc::mma_commit(&sm.mb2);
        }
    };
    // Batch 2: R += W G^T, GB += U G (G transposed), dC^T = X^T U + B^T Pm^T
    // (lanes +0), dB^T = H'^T W + C^T Pm (lanes +16), all over the masked tiles.
    // R, GB (and the carry) complete on mb2, which the epilogue waits for;
    // dC and dB on mb3, waited for halfway through the epilogue, so these
    // chains run beside its first pass.  dC follows R on one thread and dB
    // follows GB on another (two issuing threads measured best: the tensor
    // core then takes R and GB first).
    auto issue_b2 = [&]() {
        if (issuer == 1) {
            bool f = false;
            prod3(tbase + Cols::R, NAJU_SA(Wh), NAJU_SA(Wl), false, NAJU_SA(Gh), NAJU_SA(Gl), false,
                  kK / 16, tc::idesc_bf16(128, 64), f);
            tc::mma_commit(&sm.mb2);
            f = true;
            prod3(tbase + Cols::BC, NAJU_SA(Xh), NAJU_SA(Xl), true, NAJU_SA(Uh), NAJU_SA(Ul), true,
                  kP / 16, tc::idesc_bf16(64, 64, true, true), f);
            // B^T Pm^T: B (rows m = K) against Pm (rows t, K = m): hi and lo of Pm
            prod(tbase + Cols::BC, NAJU_SA(Bs), true, NAJU_SA(Ph), false, kK / 16,
                 tc::idesc_bf16(64, 64, true, false), f);
            prod(tbase + Cols::BC, NAJU_SA(Bs), true, NAJU_SA(Pl), false, kK / 16,
                 tc::idesc_bf16(64, 64, true, false), f);
            tc::mma_commit(&sm.mb3);
        } else if (issuer == 2) {
            bool f = false;
            prod3(tbase + Cols::GB, NAJU_SA(Uh), NAJU_SA(Ul), false, NAJU_SA(Gh), NAJU_SA(Gl), true,
                  kK / 16, tc::idesc_bf16(128, 64, false, true), f);
            tc::mma_commit(&sm.mb2);
            f = true;
            prod3(tbase + lane16 + Cols::BC, NAJU_SA(Hh), NAJU_SA(Hl), true, NAJU_SA(Wh),
                  NAJU_SA(Wl), true, kP / 16, tc::idesc_bf16(64, 64, true, true), f);
            prod(tbase + lane16 + Cols::BC, NAJU_SA(Cs), true, NAJU_SA(Ph), true, kK / 16,
                 tc::idesc_bf16(64, 64, true, true), f);
            prod(tbase + lane16 + Cols::BC, NAJU_SA(Cs), true, NAJU_SA(Pl), true, kK / 16,
                 tc::idesc_bf16(64, 64, true, true), f);
            tc::mma_commit(&sm.mb3);
        }
    };
    // G (lanes +0) and P (lanes +16) from tensor memory to their tile pairs,
    // lower triangle kept: this warp's lanes, columns [16 q, 16 q + 16).
    auto copy_gp = [&]() {
        float v[16];
        tc::tmem_ld16(trow + Cols::BC + 16 * q, v);
        tc::tmem_ld_wait();
        const int row = 16 * s4 + (lid & 15);
#pragma unroll
        for (int j = 0; j < 16; ++j)
            if (16 * q + j > row) v[j] = 0.f;
        __nv_bfloat16* dh = lid < 16 ? sm.Gh : sm.Ph;
        __nv_bfloat16* dl = lid < 16 ? sm.Gl : sm.Pl;
        st8o(dh, dl, tc::bf_offset(row, 16 * q), v);
        st8o(dh, dl, tc::bf_offset(row, 16 * q + 8), v + 8);
    };

    // ---------------------------------------------------- exact path
    // Token-by-token recurrences for a block outside the factorisation's
    // range.  W holds v, U holds s dy (E = Q = 1), f = 1 - (saved 1 - f).
    // Results go where the MMAs would have put them: R <- x.C, GB <- lambda.B,
    // carry <- f_0 lambda_0; dB and dC are added to the accumulator directly.
    // Its row sums live in region A (the per-token inputs are read by now).
    auto exact_block = [&](int64_t tb, int nv) {
        float* rsum = reinterpret_cast<float*>(sm.Gh);  // [64 t][128 ch] over G and P
        float* gsum = reinterpret_cast<float*>(sm.Hh);  // [64 t][128 ch] over the H pair
        for (int e = tid; e < kK * kP; e += kNT) {
            rsum[e] = 0.f;
            gsum[e] = 0.f;
        }
        auto f_at = [&](int tt) {
            const float om = tc::tmem_ld1(trow + Cols::SV + 3 * 64 + tt);
            return 1.f - om;
        };
        float hx[16];
        tc::tmem_ld16(trow + Cols::H + 16 * q, hx);  // carry entering the block end
        tc::tmem_ld_wait();
        float x[16];
#pragma unroll
        for (int j = 0; j < 16; j += 4) ld4o(sm.Xh, sm.Xl, (j < 8 ? oc0 : oc1) + (j & 4) * 2, x + j);
        __syncthreads();
        for (int tt = 0; tt < nv; ++tt) {
            const float f = f_at(tt), v = ld1(sm.Wh, sm.Wl, ch, tt), sdy = ld1(sm.Uh, sm.Ul, ch, tt);
            float rp = 0.f;
#pragma unroll
            for (int j = 0; j < 16; ++j) {
                x[j] = fmaf(f, x[j], v * ld1(sm.Bs, tt, 16 * q + j));
                rp = fmaf(x[j], ld1(sm.Cs, tt, 16 * q + j), rp);
            }
            atomicAdd(&rsum[tt * kP + ch], rp);
#pragma unroll
            for (int j = 0; j < 16; ++j) {
                const float r = warp_sum(sdy * x[j]);
                if (lid == 0) red_add(p.dBCp + dbc_index(bb, tb + tt, 1, JH + 16 * q + j, L, NS), r);
            }
        }
        for (int tt = nv - 1; tt >= 0; --tt) {
            const float f = f_at(tt), v = ld1(sm.Wh, sm.Wl, ch, tt), sdy = ld1(sm.Uh, sm.Ul, ch, tt);
            float gp = 0.f;
#pragma unroll
            for (int j = 0; j < 16; ++j) {
                hx[j] = fmaf(sdy, ld1(sm.Cs, tt, 16 * q + j), hx[j]);
                gp = fmaf(hx[j], ld1(sm.Bs, tt, 16 * q + j), gp);
            }
            atomicAdd(&gsum[tt * kP + ch], gp);
#pragma unroll
            for (int j = 0; j < 16; ++j) {
                const float r = warp_sum(v * hx[j]);
                if (lid == 0) red_add(p.dBCp + dbc_index(bb, tb + tt, 0, JH + 16 * q + j, L, NS), r);
                hx[j] *= f;
            }
        }
        tc::tmem_st16(trow + Cols::H + 16 * q, hx);
        __syncthreads();
        float rv[16], gv[16];
#pragma unroll
        for (int k = 0; k < 16; ++k) {
            rv[k] = rsum[(16 * q + k) * kP + ch];
            gv[k] = gsum[(16 * q + k) * kP + ch];
        }
        tc::tmem_st16(trow + Cols::R + 16 * q, rv);
        tc::tmem_st16(trow + Cols::GB + 16 * q, gv);
        tc::tmem_st_wait();
        sync();
    };
    // Adjoint-only exact block (early pass): f from tensor memory (slot 2),
    // U holds s dy.
    auto exact_carry = [&](int nv) {
        float hx[16];
        tc::tmem_ld16(trow + Cols::H + 16 * q, hx);
        tc::tmem_ld_wait();
        for (int tt = nv - 1; tt >= 0; --tt) {
            const float f = tc::tmem_ld1(trow + Cols::SV + 2 * 64 + tt);
            const float sdy = ld1(sm.Uh, sm.Ul, ch, tt);
#pragma unroll
            for (int j = 0; j < 16; ++j)
                hx[j] = f * fmaf(sdy, ld1(sm.Cs, tt, 16 * q + j), hx[j]);
        }
        tc::tmem_st16(trow + Cols::H + 16 * q, hx);
        tc::tmem_st_wait();
        sync();
    };

    // ============================================================ early pass
    // Group mode, every group but the first: the adjoint alone over the
    // group (last block first) from a zero carry (the sequence's dx_final for
    // the last group), then the carry leaving the group's start is published
    // after adding the decayed carry of the later group (bounded wait).
    if (aligned1k && !pieces && !firstg) {
        const float* dxf = p.dx_final ? p.dx_final + (int64_t)bb * d * NS : nullptr;
        carry_from(lastg ? dxf : nullptr, false);
        if (tid == 0) {
            load_raw(kb1 - 1, false);
            load_bc(kb1 - 1, false);
        }
        float logF = 0.f;
        for (int k = kb1 - 1; k >= kb0; --k) {
            const int64_t tb = (int64_t)k * kK;
            const int nv = (int)min64((int64_t)kK, L - tb);
            wait_mb(&sm.mb_in, ph_in);
            const bool slow = decays(nv);
            // U = s dy E (slow: s dy)
            {
                const __nv_bfloat16* rzp = rz + ro;
                const __nv_bfloat16* rdp = rdy + ro;
                float E = slow ? 1.f : Eb;
#pragma unroll
                for (int g4 = 0; g4 < 4; ++g4) {
                    float Uv[4], fa[4];
                    const int col = 16 * q + 4 * g4;
                    tc::tmem_ld4(trow + Cols::SV + 2 * 64 + col, fa);
                    tc::tmem_ld_wait();
#pragma unroll
                    for (int k4 = 0; k4 < 4; ++k4) {
                        const int kk = 4 * g4 + k4;
                        float gg = 1.f;
                        if (has_z) {
                            const float zv = bf2f(rzp[kk * kP]);
                            gg = zv * sigmoidx_(zv);
                        }
                        const float dout = bf2f(rdp[kk * kP]);  // zero outside the tensor
                        if (!slow) E *= fa[k4];
                        Uv[k4] = sc * dout * gg * E;
                    }
                    uint32_t h0, l0, h1, l1;
                    split2(Uv[0], Uv[1], h0, l0);
                    split2(Uv[2], Uv[3], h1, l1);
                    const uint32_t o = (g4 < 2 ? oc0 : oc1) + (g4 & 1) * 8;
                    *reinterpret_cast<uint2*>(reinterpret_cast<char*>(sm.Uh) + o) = make_uint2(h0, h1);
                    *reinterpret_cast<uint2*>(reinterpret_cast<char*>(sm.Ul) + o) = make_uint2(l0, l1);
                }
            }
            tc::tmem_st_wait();
            tc::fence_proxy_async();
            sync();  // the per-token inputs are read
            if (tid == 0 && k > kb0) load_raw(k - 1, false);
            wait_mb(&sm.mb_bc, ph_bc);
            logF += __logf(E63);
            if (!slow) {
                scale_carry(false);
                tc::tmem_st_wait();
                sync();
                if (tid == 0) {
                    bool fh = false;
                    prod2(tbase + Cols::H, NAJU_SA(Uh), NAJU_SA(Ul), false, NAJU_SA(Cs), true, kK / 16,
                          tc::idesc_bf16(128, kN, false, true), fh);
                    tc::mma_commit(&sm.mb_e);
                }
                wait_mb(&sm.mb_e, ph_e);
            } else {
                exact_carry(nv);
            }
            if (tid == 0 && k > kb0) load_bc(k - 1, false);  // the C tile is free
        }
        if (!lastg) {
            if (tid == 0) sm.ok = wait_flag(flag_slot(g), &p.hdr->status, p.wait_limit) ? 1 : 0;
            __syncthreads();
            const bool okc = sm.ok != 0;
            const float Pf = __expf(logF);  // decay over the whole group
            const float* cin = carry_slot(g);
            float hx[16];
            tc::tmem_ld16(trow + Cols::H + 16 * q, hx);
            tc::tmem_ld_wait();
#pragma unroll
            for (int k = 0; k < 16; k += 4) {
                float4 v4 = make_float4(0.f, 0.f, 0.f, 0.f);
                if (okc && cvalid)
                    v4 = __ldcg(reinterpret_cast<const float4*>(cin + c * NS + JH + 16 * q + k));
                hx[k] = fmaf(Pf, v4.x, hx[k]);
                hx[k + 1] = fmaf(Pf, v4.y, hx[k + 1]);
                hx[k + 2] = fmaf(Pf, v4.z, hx[k + 2]);
                hx[k + 3] = fmaf(Pf, v4.w, hx[k + 3]);
            }
            tc::tmem_st16(trow + Cols::H + 16 * q, hx);
            tc::tmem_st_wait();
        }
        carry_to(carry_slot(g - 1));
        __threadfence();
        __syncthreads();
        if (tid == 0 && !(lastg && p.fault_skip_publish)) st_release(flag_slot(g - 1), 1);
        sync();
    }

    // ============================================================ main phase
    const int64_t ub_first = pieces ? (F0 / p.nsub) * p.nsub : 0;
    const int64_t ub_end = !aligned1k ? ub_first : pieces ? F1 : 1;
    for (int64_t ub = ub_first; ub < ub_end; ub += pieces ? p.nsub : 1) {
        if (pieces) {
            const int k0 = (int)(max64(F0, ub) - ub), k1 = (int)(min64(F1, ub + p.nsub) - ub);
            set_unit((int)(ub / p.nsub), k0 > 0 ? 1 : 0, k0, k1);
        }
        // carry entering the segment's end, and the tail H . x at that end
        if (lastg) {
            carry_from(p.dx_final ? p.dx_final + (int64_t)bb * d * NS : nullptr, false);
        } else {
            const int slot = pieces ? 0 : g;
            if (tid == 0) sm.ok = wait_flag(flag_slot(slot), &p.hdr->status, p.wait_limit) ? 1 : 0;
            __syncthreads();
            carry_from(sm.ok ? carry_slot(slot) : nullptr, true);
        }
        int par = 0;  // parity of the block within the segment (double buffers)
        // The staged gradients of a block leave after the next block's first
        // barrier (no barrier of their own): that block's first token, or -1.
        int out_pending = -1;
        auto store_out = [&]() {
            if (kStage && tid == kStoreTid && out_pending >= 0) {
                const int x = (int)c0, y = out_pending;
                if (has_z) tma::store_3d(&tm.oz, x, y, bb, sm.Wh);
                if (has_b) tma::store_3d(&tm.ob, x, y, bb, sm.Wl);
                tma::store_3d(&tm.oa, x, y, bb, sm.Uh);
                tma::store_3d(&tm.ou, x, y, bb, sm.Ul);
                tma::store_commit();
            }
            out_pending = -1;
        };
        {
            float hx[16];
            tc::tmem_ld16(trow + Cols::H + 16 * q, hx);
            tc::tmem_ld_wait();
            const float* xe = ck_at(kb1);
            float tp = 0.f;
            if (cvalid) {
#pragma unroll
                for (int k = 0; k < 16; k += 4) {
                    const float4 x4 =
                        __ldcg(reinterpret_cast<const float4*>(xe + c * NS + JH + 16 * q + k));
                    tp = fmaf(hx[k], x4.x, tp);
                    tp = fmaf(hx[k + 1], x4.y, tp);
                    tp = fmaf(hx[k + 2], x4.z, tp);
                    tp = fmaf(hx[k + 3], x4.w, tp);
                }
            }
            sm.tailp[par][q][ch] = tp;
            if (q == 0) {
#pragma unroll
                for (int i = 0; i < 3; ++i) sm.dnext[par][i][ch] = 0.f;
#pragma unroll
                for (int v = 0; v < 6; ++v) sm.red6[v][ch] = 0.f;
            }
        }
        if (tid == 0) {
            load_raw(kb1 - 1, true);
            load_bc(kb1 - 1, true);
            load_x(kb1 - 1);
        }
        sync();

        for (int k = kb1 - 1; k >= kb0; --k, par ^= 1) {
            const int64_t tb = (int64_t)k * kK;
            const int nv = (int)min64((int64_t)kK, L - tb);
            const int nq = cvalid ? nv - 16 * q : 0;  // valid tokens of this thread
            // ------------------------------------------------ phase A
            if (kImport && tid == 0) {
#pragma unroll
                for (int i = 0; i < kP; i += 32) {
                    tma::prefetch_l2_3d(&tm.pr, (int)c0 + i, (int)tb, bb);
                    tma::prefetch_l2_3d(&tm.pg, (int)c0 + i, (int)tb, bb);
                }
            }
            wait_mb2(&sm.mb_in, ph_in, &sm.mb_x, ph_x);
            store_out();  // the previous block's staged gradients (after that barrier)
            issue_g();    // (the exact path waits for it too, to keep the barrier phases)
            float xr[16];
            read_x(xr);
            const bool slow = decays(nv);  // (its barriers end the reads of the fp32 checkpoint)
            st8o(sm.Xh, sm.Xl, oc0, xr);
            st8o(sm.Xh, sm.Xl, oc1, xr + 8);
            unpack(slow);
            tc::tmem_st_wait();
            tc::fence_proxy_async();
            wait_mb(&sm.mb_bc, ph_bc);  // and region A's per-token inputs are read
            if (!slow) {
                issue_pr();
                scale_carry(true);
            } else if (issuer == 5) {
                tc::mbar_arrive(&sm.mb0);  // no P on the exact path
            }
            tc::tmem_st_wait();
            tc::fence_proxy_async();
            sync();
            // ------------------------------------------------ phase B
            if (!slow) {
                issue_gbh();
                wait_mb(&sm.mb0, ph0);
                copy_gp();
                tc::fence_proxy_async();
                sync();
                issue_b2();
                wait_mb(&sm.mb2, ph2);
            } else {
                wait_mb(&sm.mb0, ph0);  // G (unused here)
                exact_block(tb, nv);
            }
            // ------------------------------------------------ phase C
            // The u buffer is free: the earlier block's u is requested.
            if (tid == 0 && k > kb0) load_raw_u(k - 1);
            // Halfway through the epilogue: dB and dC are complete, so region A,
            // the B, C tiles and the X tiles (their operands) take the earlier
            // block's inputs and checkpoint.
            auto mid_barrier = [&]() {
                if (!slow) wait_mb(&sm.mb3, ph3);
                else __syncthreads();
                if (tid == 0 && k > kb0) {
                    load_raw_a(k - 1);
                    load_bc(k - 1, true);
                    load_x(k - 1);
                }
            };
            if constexpr (kImport) {
                // the first pass's R and GB of this block (state columns 0..63)
                const float* rp = p.rgb_part + ((int64_t)bb * L + tb + 16 * q) * d + c;
                const float* gp = rp + Bt * L * d;
                float r[16], gv[16];
                tc::tmem_ld16(trow + Cols::R + 16 * q, r);
                tc::tmem_ld16(trow + Cols::GB + 16 * q, gv);
                tc::tmem_ld_wait();
#pragma unroll
                for (int kk = 0; kk < 16; ++kk) {
                    if (kk < nq) {
                        r[kk] += __ldcg(rp + (int64_t)kk * d);
                        gv[kk] += __ldcg(gp + (int64_t)kk * d);
                    }
                }
                tc::tmem_st16(trow + Cols::R + 16 * q, r);
                tc::tmem_st16(trow + Cols::GB + 16 * q, gv);
                tc::tmem_st_wait();
            }
            // tail of the earlier block: (carry entering it) . (this block's X)
            {
                float hx[16], xv[16];
                tc::tmem_ld16(trow + Cols::H + 16 * q, hx);
#pragma unroll
                for (int j = 0; j < 16; j += 4)
                    ld4o(sm.Xh, sm.Xl, (j < 8 ? oc0 : oc1) + (j & 4) * 2, xv + j);
                tc::tmem_ld_wait();
                float tp = 0.f;
#pragma unroll
                for (int j = 0; j < 16; ++j) tp = fmaf(hx[j], xv[j], tp);
                sm.tailp[par ^ 1][q][ch] = tp;
            }
            if constexpr (kExport) {
                // partial R, GB and this block's tail go to the second pass
                float* rp = p.rgb_part + ((int64_t)bb * L + tb + 16 * q) * d + c;
                float* gp = rp + Bt * L * d;
                float r[16], gv[16];
                tc::tmem_ld16(trow + Cols::R + 16 * q, r);
                tc::tmem_ld16(trow + Cols::GB + 16 * q, gv);
                tc::tmem_ld_wait();
#pragma unroll
                for (int kk = 0; kk < 16; ++kk) {
                    if (kk < nq) {
                        rp[(int64_t)kk * d] = r[kk];
                        gp[(int64_t)kk * d] = gv[kk];
                    }
                }
                if (q == 0 && cvalid) {
                    float ts = 0.f;
#pragma unroll
                    for (int qq = 0; qq < 4; ++qq) ts += sm.tailp[par][qq][ch];
                    p.tail_part[((int64_t)bb * p.nsub + k) * d + c] = ts;
                }
                mid_barrier();
            } else {
            // The epilogue in four variants (b and z present or not), so no
            // per-token branch tests them.
            auto epilogue = [&](auto hb_c, auto hz_c) {
                constexpr bool hb = decltype(hb_c)::value;
                constexpr bool hz = decltype(hz_c)::value;
                // Pass 1 (tokens in order): dL; the quarter's sum of dL and its
                // first three dp for the neighbouring quarter.
                float dL[16];
                float qsum = 0.f, dpf0 = 0.f, dpf1 = 0.f, dpf2 = 0.f;
                uint4 uh4, ul4, wh4, wl4;  // 8 tokens of U and W hi / lo
#pragma unroll
                for (int g4 = 0; g4 < 4; ++g4) {
                    const int col = 16 * q + 4 * g4;
                    float R4[4], G4[4], b2[4], Ua[4], Wa[4];
                    tc::tmem_ld4(trow + Cols::R + col, R4);
                    tc::tmem_ld4(trow + Cols::GB + col, G4);
                    if (!hb) tc::tmem_ld4(trow + Cols::SV + 2 * 64 + col, b2);
                    if ((g4 & 1) == 0) {
                        const uint32_t o = g4 < 2 ? oc0 : oc1;
                        auto ld = [&](const __nv_bfloat16* t) {
                            return *reinterpret_cast<const uint4*>(reinterpret_cast<const char*>(t) + o);
                        };
                        uh4 = ld(sm.Uh);
                        ul4 = ld(sm.Ul);
                        wh4 = ld(sm.Wh);
                        wl4 = ld(sm.Wl);
                    }
                    {
                        const bool hi = (g4 & 1) != 0;
                        const uint32_t a0 = hi ? uh4.z : uh4.x, a1 = hi ? uh4.w : uh4.y;
                        const uint32_t b0 = hi ? ul4.z : ul4.x, b1 = hi ? ul4.w : ul4.y;
                        const uint32_t c0_ = hi ? wh4.z : wh4.x, c1_ = hi ? wh4.w : wh4.y;
                        const uint32_t d0 = hi ? wl4.z : wl4.x, d1 = hi ? wl4.w : wl4.y;
                        Ua[0] = bf_lo(a0) + bf_lo(b0); Ua[1] = bf_hi(a0) + bf_hi(b0);
                        Ua[2] = bf_lo(a1) + bf_lo(b1); Ua[3] = bf_hi(a1) + bf_hi(b1);
                        Wa[0] = bf_lo(c0_) + bf_lo(d0); Wa[1] = bf_hi(c0_) + bf_hi(d0);
                        Wa[2] = bf_lo(c1_) + bf_lo(d1); Wa[3] = bf_hi(c1_) + bf_hi(d1);
                    }
                    tc::tmem_ld_wait();
#pragma unroll
                    for (int k4 = 0; k4 < 4; ++k4) {
                        const int kk = 4 * g4 + k4;
                        float dl = Ua[k4] * R4[k4] - Wa[k4] * G4[k4];
                        if (hb) {
                            qsum += dl;
                        } else {
                            // coupled gate: the sums over later tokens keep the plain dL,
                            // this token's da loses f h lambda.B (kept in dL[kk])
                            qsum += dl;
                            dl = fmaf(-b2[k4], G4[k4], dl);
                        }
                        dL[kk] = dl;
                        if (kk == 0) dpf0 = fmaf(c1v[0], G4[k4], c0v[0]);
                        if (kk == 1) dpf1 = fmaf(c1v[1], G4[k4], c0v[1]);
                        if (kk == 2) dpf2 = fmaf(c1v[2], G4[k4], c0v[2]);
                    }
                }
                sm.xs[q][ch] = qsum;
                sm.dph[q][0][ch] = dpf0;
                sm.dph[q][1][ch] = dpf1;
                sm.dph[q][2][ch] = dpf2;
                mid_barrier();
                float base = 0.f;  // dL over the later quarters, plus the tail
#pragma unroll
                for (int qq = 0; qq < 4; ++qq) {
                    if (qq > q) base += sm.xs[qq][ch];
                    base += sm.tailp[par][qq][ch];
                }
                if (kImport && cvalid) base += __ldcg(p.tail_part + ((int64_t)bb * p.nsub + k) * d + c);
                float n1, n2, n3;  // dp of the three tokens after the current one
                if (q < 3) {
                    n1 = sm.dph[q + 1][0][ch];
                    n2 = sm.dph[q + 1][1][ch];
                    n3 = sm.dph[q + 1][2][ch];
                } else {
                    n1 = sm.dnext[par][0][ch];
                    n2 = sm.dnext[par][1][ch];
                    n3 = sm.dnext[par][2][ch];
                }
                // Pass 2 (tokens in reverse): da from the suffix sums of dL, dz, db;
                // dp, the conv backward (du, dw, dbias) from a window of later dp.
                // bf16 gradients go to the staging buffers over the W and U tiles
                // (dz, db, da, dh or du), fp32 ones straight to global memory.
                {
                    [[maybe_unused]] const int64_t gofs = ((int64_t)bb * L + tb + 16 * q) * d + c;
                    auto put = [&](__nv_bfloat16* stage, void* gbase, int kk, float v) {
                        if constexpr (kStage) {
                            stage[ro + kk * kP] = __float2bfloat16_rn(v);
                        } else {
                            if (kk < nq) static_cast<float*>(gbase)[gofs + (int64_t)kk * d] = v;
                        }
                    };
                    float dw0 = 0.f, dw1 = 0.f, dw2 = 0.f, dw3 = 0.f, dbias = 0.f;
                    float run = base;
                    const bool seg_end = !lastg && k == kb1 - 1;  // a full block
#pragma unroll
                    for (int g4 = 3; g4 >= 0; --g4) {
                        const int col = 16 * q + 4 * g4;
                        float G4[4], om[4], b2[4], R4[4], z1[4], z0[4];
                        tc::tmem_ld4(trow + Cols::GB + col, G4);
                        tc::tmem_ld4(trow + Cols::SV + 3 * 64 + col, om);
                        tc::tmem_ld4(trow + Cols::SV + 2 * 64 + col, b2);
                        if (hz) {
                            tc::tmem_ld4(trow + Cols::R + col, R4);
                            tc::tmem_ld4(trow + Cols::SV + 0 * 64 + col, z1);
                            tc::tmem_ld4(trow + Cols::SV + 1 * 64 + col, z0);
                        }
                        tc::tmem_ld_wait();
#pragma unroll
                        for (int k4 = 3; k4 >= 0; --k4) {
                            const int kk = 4 * g4 + k4;
                            float fdf;
                            if (hb) {
                                run += dL[kk];
                                fdf = run;
                            } else {  // dL[kk] holds dL - f h lambda.B
                                fdf = run + dL[kk];
                                run += fmaf(b2[k4], G4[k4], dL[kk]);
                            }
                            put(sm.Uh, p.da, kk, fdf * om[k4]);
                            if (hz) put(sm.Wh, p.dz, kk, fmaf(z1[k4], R4[k4], z0[k4]));
                            if (hb) put(sm.Wl, p.db, kk, b2[k4] * G4[k4]);
                            const float dpv = fmaf(c1v[kk], G4[k4], c0v[kk]);  // 0 outside
                            if (CONV) {
                                const float duv = fmaf(w3, dpv, fmaf(w2, n1, fmaf(w1, n2, w0 * n3)));
                                // u and dp vanish outside the tensor: no masks
                                dw0 = fmaf(dpv, uwin(kk), dw0);
                                dw1 = fmaf(dpv, uwin(kk + 1), dw1);
                                dw2 = fmaf(dpv, uwin(kk + 2), dw2);
                                dw3 = fmaf(dpv, uwin(kk + 3), dw3);
                                dbias += dpv;
                                put(sm.Ul, p.dhu, kk, duv);
                                // the segment's last three du are partial (fixed up later)
                                if (kk >= 13 && q == 3 && seg_end && cvalid)
                                    edge_row()[(3 + (kk - 13)) * d + c] = duv;
                                if (kk < 3 && q == 0 && k == kb0 && kk < nq) edge_row()[kk * d + c] = dpv;
                                n3 = n2;
                                n2 = n1;
                                n1 = dpv;
                            } else {
                                put(sm.Ul, p.dhu, kk, dpv);
                            }
                        }
                    }
                    if (q == 0) {
                        sm.dnext[par ^ 1][0][ch] = dpf0;
                        sm.dnext[par ^ 1][1][ch] = dpf1;
                        sm.dnext[par ^ 1][2][ch] = dpf2;
                    }
                    if (cvalid) {
                        atomicAdd(&sm.red6[0][ch], dD_acc);
                        if (CONV) {
                            atomicAdd(&sm.red6[1][ch], dw0);
                            atomicAdd(&sm.red6[2][ch], dw1);
                            atomicAdd(&sm.red6[3][ch], dw2);
                            atomicAdd(&sm.red6[4][ch], dw3);
                            atomicAdd(&sm.red6[5][ch], dbias);
                        }
                    }
                }
            };
            if (has_b) {
                if (has_z) epilogue(std::true_type{}, std::true_type{});
                else epilogue(std::true_type{}, std::false_type{});
            } else {
                if (has_z) epilogue(std::false_type{}, std::true_type{});
                else epilogue(std::false_type{}, std::false_type{});
            }
            }  // (gradients of the per-token inputs)
            // dC^T (lanes +0) and dB^T (lanes +16): this warp's lanes, columns
            // [16 q, 16 q + 16), added into the accumulator four tokens at a
            // time (the tokens of a chunk past the end land in its padding)
            if (!slow) {
                float v[16];
                tc::tmem_ld16(trow + Cols::BC + 16 * q, v);
                tc::tmem_ld_wait();
                const int j = 16 * s4 + (lid & 15);
                const int slot = lid < 16 ? 1 : 0;  // slot 0 dB, 1 dC
                float* acc = p.dBCp + dbc_index(bb, tb + 16 * q, slot, JH + j, L, NS);
                const int nvq = nv - 16 * q;
#pragma unroll
                for (int i = 0; i < 4; ++i)
                    if (4 * i < nvq)
                        red_add4(acc + (int64_t)i * 2 * NS * 4, v[4 * i], v[4 * i + 1], v[4 * i + 2],
                                 v[4 * i + 3]);
            }
            // staged outputs -> async proxy; the next block's first barrier
            // orders them (and this block's reads of tiles and tensor memory)
            // before its stores and writes
            if (kStage) tc::fence_proxy_async();
            out_pending = (int)tb;
        }
        sync();
        store_out();

        // ------------------------------------------- carries and partials
        if (firstg) {
            if (p.dx0) carry_to(p.dx0 + (int64_t)bb * d * NS);
        } else if (pieces) {
            carry_to(carry_slot(0));
            __threadfence();
            __syncthreads();
            if (tid == 0 && !p.fault_skip_publish) st_release(flag_slot(0), 1);
        }
        if constexpr (!kExport) {
            float* cpart = p.chan_part + ((int64_t)bb * p.ngroups + g) * d * 8;
            __syncthreads();
            if (tid < kP && c0 + tid < d) {
#pragma unroll
                for (int v = 0; v < 6; ++v) cpart[(c0 + tid) * 8 + v] = sm.red6[v][tid];
                if (pieces && firstg && lastg) {  // uncut unit: its tail slot stays empty
                    float* cp1 = p.chan_part + ((int64_t)bb * p.ngroups + 1) * d * 8;
#pragma unroll
                    for (int v = 0; v < 6; ++v) cp1[(c0 + tid) * 8 + v] = 0.f;
                }
            }
            sync();
        }
    }
#undef NAJU_SA

    if (kStage && tid == kStoreTid) tma::store_wait_all();
    if (timed_out) atomicOr(&p.hdr->status, 1 << NAJU_ERR_TIMEOUT);
    sync();
    if (warp == 0) tc::tmem_dealloc(tbase, 512);
}

// dB, dC from the fp32 accumulator [Bt][ceil(L / 4)][2][N][4]: one thread per
// (batch, four-token chunk, state column), consecutive threads on consecutive
// columns (16-byte loads, coalesced stores).
template <typename Tout>
__global__ void finish_dBC_kernel(const float* __restrict__ acc, int64_t Bt, int64_t L, int64_t N,
                                  Tout* __restrict__ dB, Tout* __restrict__ dC) {
    const int64_t L4 = (L + 3) >> 2, n = Bt * L4 * N;
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n;
         i += (int64_t)gridDim.x * blockDim.x) {
        const int64_t j = i % N, row = i / N, b = row / L4, t0 = (row % L4) * 4;
        const float4 b4 = *reinterpret_cast<const float4*>(acc + (row * 2 * N + j) * 4);
        const float4 c4 = *reinterpret_cast<const float4*>(acc + (row * 2 * N + N + j) * 4);
        const float bv[4] = {b4.x, b4.y, b4.z, b4.w}, cv[4] = {c4.x, c4.y, c4.z, c4.w};
#pragma unroll
        for (int tt = 0; tt < 4; ++tt) {
            if (t0 + tt < L) {
                const int64_t o = (b * L + t0 + tt) * N + j;
                dB[o] = from_f<Tout>(bv[tt]);
                dC[o] = from_f<Tout>(cv[tt]);
            }
        }
    }
}

template <typename Tout, bool CONV, bool PIECES, int MODE>
static cudaError_t launch_blk_t(const BwdParams& p, cudaStream_t st) {
    constexpr int NS = MODE == 0 ? kN : 2 * kN;
    BkTmaps tm;
    memset(&tm, 0, sizeof(tm));
    bool ok = tma_encode_bf16_3d(&tm.u, p.hu, p.Bt, p.L, p.d, kK + 3, kP) &&
              tma_encode_bf16_3d(&tm.a, p.a, p.Bt, p.L, p.d, kK, kP) &&
              (!p.b || tma_encode_bf16_3d(&tm.b, p.b, p.Bt, p.L, p.d, kK, kP)) &&
              (!p.z || tma_encode_bf16_3d(&tm.z, p.z, p.Bt, p.L, p.d, kK, kP)) &&
              tma_encode_bf16_3d(&tm.dy, p.dy, p.Bt, p.L, p.d, kK, kP) &&
              tma_encode_bf16_3d_sw128(&tm.B, p.B, p.Bt, p.L, NS, kK) &&
              tma_encode_bf16_3d_sw128(&tm.C, p.C, p.Bt, p.L, NS, kK) &&
              tma_encode_f32_3d_sw128(&tm.X, p.ckpt, p.Bt * (int64_t)(p.nck + 1), p.d, NS, kP);
    if (ok && MODE == 2)
        ok = tma_encode_f32_3d_sw128(&tm.pr, p.rgb_part, p.Bt, p.L, p.d, kK) &&
             tma_encode_f32_3d_sw128(&tm.pg, p.rgb_part + p.Bt * p.L * p.d, p.Bt, p.L, p.d, kK);
    if (ok && MODE != 1 && std::is_same<Tout, __nv_bfloat16>::value) {
        ok = tma_encode_bf16_3d(&tm.oa, p.da, p.Bt, p.L, p.d, kK, kP) &&
             tma_encode_bf16_3d(&tm.ou, p.dhu, p.Bt, p.L, p.d, kK, kP) &&
             (!p.z || tma_encode_bf16_3d(&tm.oz, p.dz, p.Bt, p.L, p.d, kK, kP)) &&
             (!p.b || tma_encode_bf16_3d(&tm.ob, p.db, p.Bt, p.L, p.d, kK, kP));
    }
    if (!ok) return cudaErrorInvalidValue;
    const size_t smem = sizeof(BkSmem);
    auto kern = scan_bwd_blk_kernel<Tout, CONV, PIECES, MODE>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)smem);
    if (e != cudaSuccess) return e;
    const int grid = p.npieces > 0 ? p.npieces : p.ngroups * (int)p.Bt * p.ntiles;
    kern<<<grid, kNT, smem, st>>>(p, tm);
    return cudaGetLastError();
}

bool bwd_blk_supported(int dtype, int64_t N, int64_t d) {
    return dtype == NAJU_BF16 && (N == kN || N == 2 * kN) && d % 8 == 0;
}

template <int MODE>
static cudaError_t launch_blk_mode(const BwdParams& p, int out_dtype, cudaStream_t st) {
    const bool conv = p.conv_w != nullptr, pc = p.npieces > 0;
    if (out_dtype == NAJU_BF16) {
        using T = __nv_bfloat16;
        return conv ? (pc ? launch_blk_t<T, true, true, MODE>(p, st)
                          : launch_blk_t<T, true, false, MODE>(p, st))
                    : (pc ? launch_blk_t<T, false, true, MODE>(p, st)
                          : launch_blk_t<T, false, false, MODE>(p, st));
    }
    return conv ? (pc ? launch_blk_t<float, true, true, MODE>(p, st)
                      : launch_blk_t<float, true, false, MODE>(p, st))
                : (pc ? launch_blk_t<float, false, true, MODE>(p, st)
                      : launch_blk_t<float, false, false, MODE>(p, st));
}

cudaError_t launch_scan_bwd_blk(const BwdParams& p, int out_dtype, cudaStream_t st) {
    // the dB / dC accumulator starts at zero
    cudaError_t e = cudaMemsetAsync(
        p.dBCp, 0, sizeof(float) * (size_t)p.Bt * ((p.L + 3) / 4 * 4) * 2 * p.N, st);
    if (e != cudaSuccess) return e;
    if (p.N == kN) return launch_blk_mode<0>(p, out_dtype, st);
    // d_state 128: state columns 0..63, then 64..127 with fresh tickets and flags
    e = launch_blk_mode<1>(p, out_dtype, st);
    if (e == cudaSuccess) e = cudaMemsetAsync(&p.hdr->bwd_ticket, 0, sizeof(int), st);
    if (e == cudaSuccess)
        e = cudaMemsetAsync(p.flags, 0, sizeof(int) * (size_t)p.ngroups * p.Bt * p.ntiles, st);
    if (e == cudaSuccess) e = launch_blk_mode<2>(p, out_dtype, st);
    return e;
}

cudaError_t launch_finish_dBC(const BwdParams& p, int out_dtype, void* dB, void* dC,
                              cudaStream_t st) {
    if (out_dtype == NAJU_BF16)
        finish_dBC_kernel<__nv_bfloat16><<<592, 256, 0, st>>>(
            p.dBCp, p.Bt, p.L, p.N, static_cast<__nv_bfloat16*>(dB), static_cast<__nv_bfloat16*>(dC));
    else
        finish_dBC_kernel<float><<<592, 256, 0, st>>>(p.dBCp, p.Bt, p.L, p.N,
                                                       static_cast<float*>(dB), static_cast<float*>(dC));
    return cudaGetLastError();
}

}  // namespace naju
