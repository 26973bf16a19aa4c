// Tensor Memory Accelerator (TMA) support: host-side tensor-map encoding and
// the device-side bulk tensor load into shared memory with an mbarrier
// transaction count, and the bulk tensor store back.  Never with cluster
// multicast.
//
// A tensor map describes a row-major bf16 tensor [outer][rows][cols] and a
// box [box_rows][box_cols]; a load copies the box at (col, row, outer) into
// shared memory as box_rows x box_cols contiguous elements.  Out-of-range
// elements (negative rows included) read as zero.
#pragma once
#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace naju {

// Encode a 3-D bf16 tensor map.  Requirements (checked): base 16-byte
// aligned, cols * 2 a multiple of 16, box_cols * 2 a multiple of 16,
// boxes of at most 256 per dimension.  Returns false when the driver entry
// point is unavailable or the encoding is rejected.
bool tma_encode_bf16_3d(CUtensorMap* map, const void* base, int64_t outer, int64_t rows,
                        int64_t cols, int box_rows, int box_cols);

// Encode a 3-D bf16 tensor map whose box is box_rows rows of 64 columns (128
// bytes), written to shared memory in the 128-byte swizzled layout (box row r
// at byte 128 r, its 16-byte chunks XOR-permuted by r % 8; destination
// 1024-byte aligned).  Same checks as tma_encode_bf16_3d.
bool tma_encode_bf16_3d_sw128(CUtensorMap* map, const void* base, int64_t outer, int64_t rows,
                              int64_t cols, int box_rows);

// Encode a 3-D fp32 tensor map [outer][rows][cols] whose box is box_rows rows
// of 32 columns (128 bytes), written to shared memory in the 128-byte swizzled
// layout: box row r lands at byte 128 r with its 16-byte chunks XOR-permuted
// by r % 8 (the destination must be 1024-byte aligned).  Requirements
// (checked): base 16-byte aligned, cols * 4 a multiple of 16, box_rows <= 256.
bool tma_encode_f32_3d_sw128(CUtensorMap* map, const void* base, int64_t outer, int64_t rows,
                             int64_t cols, int box_rows);

#ifdef __CUDACC__
namespace tma {

__device__ __forceinline__ void prefetch_map(const CUtensorMap* map) {
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}

// Arrive on the mbarrier and add `bytes` to its expected transaction count.
__device__ __forceinline__ void expect_tx(uint64_t* mbar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(
                     static_cast<uint32_t>(__cvta_generic_to_shared(mbar))),
                 "r"(bytes)
                 : "memory");
}

// Box load at coordinates (x = col, y = row, z = outer); x * 2 bytes must be
// a multiple of 16.  Completion is signalled on `mbar` as transaction bytes.
__device__ __forceinline__ void load_3d(void* dst, const CUtensorMap* map, int x, int y, int z,
                                        uint64_t* mbar) {
    asm volatile(
        "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%2, %3, %4}], [%5];" ::"r"(
            static_cast<uint32_t>(__cvta_generic_to_shared(dst))),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(z),
        "r"(static_cast<uint32_t>(__cvta_generic_to_shared(mbar)))
        : "memory");
}

// Box store from shared memory (the layout a load of the same map writes) to
// (x, y, z); elements outside the tensor are not written.  x * 2 bytes must
// be a multiple of 16 and no coordinate may be negative.  Generic writes to
// the source must be fenced (fence.proxy.async) and synchronised first; the
// store joins the issuing thread's current bulk group.
__device__ __forceinline__ void store_3d(const CUtensorMap* map, int x, int y, int z,
                                         const void* src) {
    asm volatile(
        "cp.async.bulk.tensor.3d.global.shared::cta.tile.bulk_group [%0, {%1, %2, %3}], [%4];" ::"l"(
            reinterpret_cast<uint64_t>(map)),
        "r"(x), "r"(y), "r"(z), "r"(static_cast<uint32_t>(__cvta_generic_to_shared(src)))
        : "memory");
}
__device__ __forceinline__ void store_commit() {
    asm volatile("cp.async.bulk.commit_group;" ::: "memory");
}
// Wait until the issuing thread's committed stores have read their shared
// memory (the source may be rewritten), or have completed entirely.
__device__ __forceinline__ void store_wait_read() {
    asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");
}
__device__ __forceinline__ void store_wait_all() {
    asm volatile("cp.async.bulk.wait_group 0;" ::: "memory");
}

// Hint: bring the box at (x, y, z) into L2 (no shared memory, no completion
// signal).  Coordinates outside the tensor are ignored.
__device__ __forceinline__ void prefetch_l2_3d(const CUtensorMap* map, int x, int y, int z) {
    asm volatile(
        "cp.async.bulk.prefetch.tensor.3d.L2.global.tile [%0, {%1, %2, %3}];" ::"l"(
            reinterpret_cast<uint64_t>(map)),
        "r"(x), "r"(y), "r"(z)
        : "memory");
}

}  // namespace tma
#endif

}  // namespace naju
