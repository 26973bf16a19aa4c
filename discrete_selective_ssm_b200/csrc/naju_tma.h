// Tensor Memory Accelerator (TMA) support: host-side tensor-map encoding and
// the device-side bulk tensor load into shared memory with an mbarrier
// transaction count.  Loads only, never with cluster multicast.
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

}  // namespace tma
#endif

}  // namespace naju
