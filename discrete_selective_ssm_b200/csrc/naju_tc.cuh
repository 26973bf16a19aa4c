// Blackwell (sm_100a) tensor-core primitives: tensor memory (TMEM), the
// 5th-generation MMA (tcgen05.mma, kind::tf32, one CTA), its completion
// barrier, and the shared-memory operand layout.  Inline PTX only.
//
// Operand layout used throughout (no swizzle, K-major): a matrix of R rows
// and K fp32 elements is stored as 8-row x 16-byte "core matrices"
// (8 rows x 4 elements, 128 contiguous bytes, row r at byte 16 r).  Core
// matrix (row group g, K group k) sits at byte g * SBO + k * LBO with
// LBO = 128 (K groups adjacent) and SBO = 128 * K / 4.
#pragma once
#include <cuda_runtime.h>
#include <stdint.h>

namespace naju {
namespace tc {

// Byte offset of element (row, k) of an R x K K-major tile.
__host__ __device__ __forceinline__ uint32_t kmajor_offset(int row, int k, int K) {
    return (uint32_t)((row >> 3) * (K * 32) + (k >> 2) * 128 + (row & 7) * 16 + (k & 3) * 4);
}

// Shared-memory matrix descriptor (tcgen05 format): start address, leading
// byte offset (between K groups), stride byte offset (between 8-row
// groups), descriptor version 1, no swizzle.
__device__ __forceinline__ uint64_t sdesc(uint32_t saddr, uint32_t lbo, uint32_t sbo) {
    uint64_t d = 0;
    d |= (uint64_t)((saddr >> 4) & 0x3FFFu);
    d |= (uint64_t)((lbo >> 4) & 0x3FFFu) << 16;
    d |= (uint64_t)((sbo >> 4) & 0x3FFFu) << 32;
    d |= (uint64_t)1 << 46;
    return d;
}

// Byte offset of element (row, k) of an R x 128 K-major tile in the 128-byte
// swizzled layout: 8-row x 128-byte atoms (1024 bytes; rows 128 bytes apart,
// the 16-byte chunks of row r XOR-permuted by r % 8), 8-row groups 1024 bytes
// apart, the four 32-element K atoms R * 128 bytes apart.  The tile base must
// be 1024-byte aligned.  A warp writing one row's 32 consecutive k (or one k
// of 32 consecutive rows of an atom column) touches 32 distinct banks.
__host__ __device__ __forceinline__ uint32_t sw128_offset(int row, int k, int R) {
    const int r = row & 7;
    return (uint32_t)((k >> 5) * (R * 128) + (row >> 3) * 1024 + r * 128 +
                      ((((k >> 2) & 7) ^ r) << 4) + (k & 3) * 4);
}

// Descriptor of the 128-byte swizzled K-major layout above (SBO 1024; the
// leading offset is not used by swizzled K-major operands).  For K step ks
// (8 tf32) the start address is base + (ks / 4) * R * 128 + (ks % 4) * 32.
__device__ __forceinline__ uint64_t sdesc_sw128(uint32_t saddr) {
    uint64_t d = 0;
    d |= (uint64_t)((saddr >> 4) & 0x3FFFu);
    d |= (uint64_t)1 << 16;
    d |= (uint64_t)(1024 >> 4) << 32;
    d |= (uint64_t)1 << 46;
    d |= (uint64_t)2 << 61;
    return d;
}

// Descriptor of a 128-byte swizzled operand with explicit leading and
// stride byte offsets.  Used for the MN-major form of a row tile (see
// sw128_offset): the tile's rows are the operand's K index and its columns
// the M (or N) index, so one MMA K step (8 tf32) is one 8-row group at
// base + ks * 1024, the 32-element M / N blocks are LBO = rows * 128 bytes
// apart and successive 8-row groups SBO = 1024 bytes apart.
__device__ __forceinline__ uint64_t sdesc_sw128_mn(uint32_t saddr, uint32_t lbo) {
    uint64_t d = 0;
    d |= (uint64_t)((saddr >> 4) & 0x3FFFu);
    d |= (uint64_t)((lbo >> 4) & 0x3FFFu) << 16;
    d |= (uint64_t)(1024 >> 4) << 32;
    d |= (uint64_t)1 << 46;
    d |= (uint64_t)2 << 61;
    return d;
}

// MN-major tf32 operands need the 128-byte swizzle with 32-byte atoms: a tile
// with rows = the operand's K index (R rows) and columns = its M or N index,
// 32-column blocks R * 128 bytes apart, 4-row groups 512 bytes apart, each
// 128-byte row's 32-byte chunks (8 elements) XOR-permuted by row % 4.
__host__ __device__ __forceinline__ uint32_t mn32_offset(int row, int col, int R) {
    return (uint32_t)((col >> 5) * (R * 128) + (row >> 2) * 512 + (row & 3) * 128 +
                      ((((col >> 3) & 3) ^ (row & 3)) << 5) + (col & 7) * 4);
}
// Its descriptor for K step ks (8 rows = two 4-row groups).
__device__ __forceinline__ uint64_t sdesc_mn32(uint32_t base, int R, int ks) {
    const uint32_t saddr = base + (uint32_t)ks * 1024;
    uint64_t d = 0;
    d |= (uint64_t)((saddr >> 4) & 0x3FFFu);
    d |= (uint64_t)(((uint32_t)R * 128 >> 4) & 0x3FFFu) << 16;
    d |= (uint64_t)(512 >> 4) << 32;
    d |= (uint64_t)1 << 46;
    d |= (uint64_t)1 << 61;
    return d;
}

// Instruction descriptor: D fp32, A and B tf32, M x N; a_mn / b_mn select the
// MN-major form of the shared-memory A / B operand (K-major otherwise).
__host__ __device__ constexpr uint32_t idesc_tf32(int M, int N, bool a_mn = false,
                                                  bool b_mn = false) {
    return (1u << 4) | (2u << 7) | (2u << 10) | ((a_mn ? 1u : 0u) << 15) |
           ((b_mn ? 1u : 0u) << 16) | ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// ------------------------------------------------------- bf16 operand tiles
// A bf16 row tile of R rows and at most 64 columns in the 128-byte swizzled
// layout: one 128-byte line per row, its 16-byte chunks (8 elements)
// XOR-permuted by row % 8, 8-row groups 1024 bytes apart (base 1024-byte
// aligned).  For 16-bit operands the same bytes are the K-major operand with
// rows = M or N (K = columns) and the MN-major operand with rows = K
// (M or N = columns): one tile serves both contractions.
__host__ __device__ __forceinline__ uint32_t bf_offset(int row, int col) {
    return (uint32_t)((row >> 3) * 1024 + (row & 7) * 128 + ((((col >> 3) & 7) ^ (row & 7)) << 4) +
                      (col & 7) * 2);
}
// Descriptors of such a tile for one kind::f16 K step (16 elements):
// K-major, step ks < 4 (32 bytes of each line); MN-major, step ks (16 rows =
// two 8-row groups).
__device__ __forceinline__ uint64_t sdesc_bf_k(uint32_t base, int ks) {
    return sdesc_sw128(base + (uint32_t)ks * 32);
}
__device__ __forceinline__ uint64_t sdesc_bf_mn(uint32_t base, int ks) {
    return sdesc_sw128_mn(base + (uint32_t)ks * 2048, 1024);
}
// Wider bf16 tiles (R rows, up to 128 columns): 64-column blocks R * 128
// bytes apart, each in the layout above.
__host__ __device__ __forceinline__ uint32_t bf_offset_w(int row, int col, int R) {
    return (uint32_t)((col >> 6) * (R * 128)) + bf_offset(row, col & 63);
}
__device__ __forceinline__ uint64_t sdesc_bfw_k(uint32_t base, int R, int ks) {
    return sdesc_sw128(base + (uint32_t)((ks >> 2) * R * 128 + (ks & 3) * 32));
}
__device__ __forceinline__ uint64_t sdesc_bfw_mn(uint32_t base, int R, int ks) {
    return sdesc_sw128_mn(base + (uint32_t)ks * 2048, (uint32_t)R * 128);
}
// The same two descriptors from the start address already divided by 16
// (shared-memory addresses below 256 KB fit the 14-bit field): with the
// tile base 1024-byte aligned, (base + offset) / 16 = base / 16 + offset / 16,
// so a descriptor for a compile-time offset costs one add.
__device__ __forceinline__ uint64_t sdesc_sw128_a4(uint32_t a4) {
    return ((uint64_t)((1024u >> 4) | (1u << 14) | (2u << 29)) << 32) | (uint64_t)(a4 | (1u << 16));
}
__device__ __forceinline__ uint64_t sdesc_sw128_mn_a4(uint32_t a4, uint32_t lbo) {
    return ((uint64_t)((1024u >> 4) | (1u << 14) | (2u << 29)) << 32) |
           (uint64_t)(a4 | ((lbo >> 4) << 16));
}
// Instruction descriptor: D fp32, A and B bf16 (kind::f16), M x N.
__host__ __device__ constexpr uint32_t idesc_bf16(int M, int N, bool a_mn = false,
                                                  bool b_mn = false) {
    return (1u << 4) | (1u << 7) | (1u << 10) | ((a_mn ? 1u : 0u) << 15) |
           ((b_mn ? 1u : 0u) << 16) | ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}

// ------------------------------------------------------------------ TMEM
// Warp-wide: allocate `ncols` columns (power of two >= 32); the base address
// is written to *dst (shared memory).
__device__ __forceinline__ void tmem_alloc(uint32_t* dst, uint32_t ncols) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_u32(dst)),
                 "r"(ncols)
                 : "memory");
}
__device__ __forceinline__ void tmem_relinquish() {
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols)
                 : "memory");
}
__device__ __forceinline__ void fence_before_sync() {
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void fence_after_sync() {
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}
// Make generic-proxy shared-memory writes visible to the tensor core.
__device__ __forceinline__ void fence_proxy_async() {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// 16 consecutive 32-bit columns of this warp's 32 lanes <-> 16 registers.
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, float* v) {
    uint32_t r[16];
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,"
        "%14,%15}, [%16];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
          "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]),
          "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
        : "r"(taddr)
        : "memory");
#pragma unroll
    for (int i = 0; i < 16; ++i) v[i] = __uint_as_float(r[i]);
}
// 8 consecutive 32-bit columns of this warp's 32 lanes <-> 8 registers.
__device__ __forceinline__ void tmem_ld8(uint32_t taddr, float* v) {
    uint32_t r[8];
    asm volatile("tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]),
                   "=r"(r[6]), "=r"(r[7])
                 : "r"(taddr)
                 : "memory");
#pragma unroll
    for (int i = 0; i < 8; ++i) v[i] = __uint_as_float(r[i]);
}
__device__ __forceinline__ void tmem_st8(uint32_t taddr, const float* v) {
    asm volatile("tcgen05.st.sync.aligned.32x32b.x8.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8};" ::"r"(
                     taddr),
                 "r"(__float_as_uint(v[0])), "r"(__float_as_uint(v[1])),
                 "r"(__float_as_uint(v[2])), "r"(__float_as_uint(v[3])),
                 "r"(__float_as_uint(v[4])), "r"(__float_as_uint(v[5])),
                 "r"(__float_as_uint(v[6])), "r"(__float_as_uint(v[7]))
                 : "memory");
}
// One 32-bit column of this warp's 32 lanes (waits for the load).
__device__ __forceinline__ float tmem_ld1(uint32_t taddr) {
    uint32_t r;
    asm volatile("tcgen05.ld.sync.aligned.32x32b.x1.b32 {%0}, [%1];\n\t"
                 "tcgen05.wait::ld.sync.aligned;"
                 : "=r"(r)
                 : "r"(taddr)
                 : "memory");
    return __uint_as_float(r);
}
// 4 consecutive 32-bit columns of this warp's 32 lanes <-> 4 registers.
__device__ __forceinline__ void tmem_ld4(uint32_t taddr, float* v) {
    uint32_t r[4];
    asm volatile("tcgen05.ld.sync.aligned.32x32b.x4.b32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
                 : "r"(taddr)
                 : "memory");
#pragma unroll
    for (int i = 0; i < 4; ++i) v[i] = __uint_as_float(r[i]);
}
__device__ __forceinline__ void tmem_st4(uint32_t taddr, const float* v) {
    asm volatile("tcgen05.st.sync.aligned.32x32b.x4.b32 [%0], {%1,%2,%3,%4};" ::"r"(taddr),
                 "r"(__float_as_uint(v[0])), "r"(__float_as_uint(v[1])),
                 "r"(__float_as_uint(v[2])), "r"(__float_as_uint(v[3]))
                 : "memory");
}
__device__ __forceinline__ void tmem_ld_wait() {
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_st16(uint32_t taddr, const float* v) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,"
        "%13,%14,%15,%16};" ::"r"(taddr),
        "r"(__float_as_uint(v[0])), "r"(__float_as_uint(v[1])), "r"(__float_as_uint(v[2])),
        "r"(__float_as_uint(v[3])), "r"(__float_as_uint(v[4])), "r"(__float_as_uint(v[5])),
        "r"(__float_as_uint(v[6])), "r"(__float_as_uint(v[7])), "r"(__float_as_uint(v[8])),
        "r"(__float_as_uint(v[9])), "r"(__float_as_uint(v[10])), "r"(__float_as_uint(v[11])),
        "r"(__float_as_uint(v[12])), "r"(__float_as_uint(v[13])), "r"(__float_as_uint(v[14])),
        "r"(__float_as_uint(v[15]))
        : "memory");
}
__device__ __forceinline__ void tmem_st_wait() {
    asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}

// ------------------------------------------------------------------- MMA
// D[tmem] (+)= A[tmem] * B[smem]^T for one K = 8 step (tf32), issued by one
// thread.  accumulate = 0 overwrites D.
__device__ __forceinline__ void mma_tf32_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc,
                                            uint32_t idesc, uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::tf32 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
        "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
        : "memory");
}
// D[tmem] (+)= A[smem] * B[smem]^T for one K = 8 step (tf32), issued by one thread.
__device__ __forceinline__ void mma_tf32_ss(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                            uint32_t idesc, uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::tf32 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
        "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
        : "memory");
}
// D[tmem] (+)= A[smem] * B[smem]^T for one K = 16 step, bf16 operands
// (kind::f16, fp32 accumulate), issued by one thread.
__device__ __forceinline__ void mma_bf16_ss(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                            uint32_t idesc, uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
        "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
        : "memory");
}
// Arrive on an mbarrier when all previously issued MMAs of this thread finish.
__device__ __forceinline__ void mma_commit(uint64_t* mbar) {
    asm volatile(
        "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
            smem_u32(mbar))
        : "memory");
}

// --------------------------------------------------- warp-level products
// D[16 x 8] += A[16 x 8] * B[8 x 8] (tf32 operands as fp32 bits, fp32
// accumulate), one warp.  Fragments (g = lane / 4, k = lane % 4):
// a = {A[g][k], A[g+8][k], A[g][k+4], A[g+8][k+4]}, b = {B[k][g], B[k+4][g]},
// d = {D[g][2k], D[g][2k+1], D[g+8][2k], D[g+8][2k+1]}.
__device__ __forceinline__ void mma_16x8x8_tf32(float* d, const float* a, const float* b) {
    asm volatile(
        "mma.sync.aligned.m16n8k8.row.col.f32.tf32.tf32.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
        "{%8,%9}, {%0,%1,%2,%3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(__float_as_uint(a[0])), "r"(__float_as_uint(a[1])), "r"(__float_as_uint(a[2])),
          "r"(__float_as_uint(a[3])), "r"(__float_as_uint(b[0])), "r"(__float_as_uint(b[1])));
}

// One warp: D[t][m] = sum_k X[t][k] Y[m][k] for t, m < 16, with X and Y
// row-major in shared memory (row stride LD floats, LD % 32 == 4 keeps the
// fragment loads conflict-free).  Lane (g, k) ends with
// d[n][0..3] = D[g][8n+2k], D[g][8n+2k+1], D[g+8][8n+2k], D[g+8][8n+2k+1].
template <int K, int LD>
__device__ __forceinline__ void warp_gram16(const float* X, const float* Y, float (&d)[2][4]) {
    const int lane = threadIdx.x & 31, g = lane >> 2, k = lane & 3;
#pragma unroll
    for (int n = 0; n < 2; ++n)
#pragma unroll
        for (int r = 0; r < 4; ++r) d[n][r] = 0.f;
#pragma unroll 4
    for (int k0 = 0; k0 < K; k0 += 8) {
        const float a[4] = {X[g * LD + k0 + k], X[(g + 8) * LD + k0 + k], X[g * LD + k0 + k + 4],
                            X[(g + 8) * LD + k0 + k + 4]};
#pragma unroll
        for (int n = 0; n < 2; ++n) {
            const float b[2] = {Y[(8 * n + g) * LD + k0 + k], Y[(8 * n + g) * LD + k0 + k + 4]};
            mma_16x8x8_tf32(d[n], a, b);
        }
    }
}

// -------------------------------------------------------------- mbarrier
__device__ __forceinline__ void mbar_init(uint64_t* mbar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(mbar)), "r"(count)
                 : "memory");
}
__device__ __forceinline__ bool mbar_try_wait(uint64_t* mbar, uint32_t phase) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\tmbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.b32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(smem_u32(mbar)), "r"(phase)
        : "memory");
    return ok != 0;
}
__device__ __forceinline__ void mbar_arrive(uint64_t* mbar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(mbar)) : "memory");
}
// Bounded wait for the completion of `phase`; false after `limit` polls.
__device__ __forceinline__ bool mbar_wait(uint64_t* mbar, uint32_t phase, long long limit) {
    for (long long i = 0; i < limit; ++i)
        if (mbar_try_wait(mbar, phase)) return true;
    return false;
}

// ------------------------------------------------------- named barriers
// Barrier among `count` threads (a multiple of 32) of the block, id 1..15.
__device__ __forceinline__ void named_bar(int id, int count) {
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(count) : "memory");
}
// Same, returning whether `pred` holds in any participating thread.
__device__ __forceinline__ bool named_bar_or(int id, int count, bool pred) {
    uint32_t r;
    asm volatile(
        "{\n\t.reg .pred p, q;\n\tsetp.ne.b32 p, %1, 0;\n\t"
        "barrier.red.or.pred q, %2, %3, p;\n\tselp.b32 %0, 1, 0, q;\n\t}"
        : "=r"(r)
        : "r"(pred ? 1u : 0u), "r"(id), "r"(count)
        : "memory");
    return r != 0;
}

}  // namespace tc
}  // namespace naju
