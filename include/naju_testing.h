/*
 * naju_testing.h -- process-wide test and tuning hooks of the Naju library.
 *
 * These hooks exist so that the library's failure handling can be exercised
 * without faulting a GPU: a forward whose first sequence group never
 * publishes its carry makes the next group's bounded wait run out, which must
 * surface as NAJU_ERR_TIMEOUT from naju_last_device_status() while the kernel
 * still returns.  They are not part of the numerical interface and default to
 * off.  Not thread-safe: set them before launching work.
 */
#ifndef NAJU_TESTING_H_
#define NAJU_TESTING_H_

#include <stdint.h>

#include "naju.h"

#ifdef __cplusplus
extern "C" {
#endif

/* Polls before an inter-block wait gives up (each poll sleeps <= 0.5 us).
 * polls <= 0 restores the default (about one second). */
void naju_testing_set_wait_limit(int64_t polls);

/* skip != 0: the forward's first sequence group and the backward's last
 * sequence group do not publish their carries (their successors time out). */
void naju_testing_set_skip_publish(int32_t skip);

/* Forces the number of sequence groups of the forward (<= 0: automatic).
 * More groups than checkpoint segments are clamped. */
void naju_testing_set_fwd_groups(int32_t groups);

/* The forward's number of sequence groups for these dims (after the
 * automatic choice and any forced value). */
int32_t naju_testing_fwd_groups(const void* dims);

/* Forces the number of sequence groups of the backward (<= 0: automatic);
 * more groups than 64-token blocks are clamped. */
void naju_testing_set_bwd_groups(int32_t groups);

/* The backward's number of sequence groups for these dims. */
int32_t naju_testing_bwd_groups(const void* dims);

/* Piece mode of the tensor-core backward: 0 = automatic (one range per SM
 * when there are at least as many 128-channel units as SMs but not a whole
 * number of waves), < 0 = never, > 0 = that many ranges (used when there
 * are at least that many units and no forced group count). */
void naju_testing_set_bwd_pieces(int32_t pieces);

/* The backward's number of piece-mode ranges for these dims (0: group mode). */
int32_t naju_testing_bwd_pieces(const void* dims);

/* Piece mode of the tensor-core forward, with the same values and rule as
 * the backward's (ranges of 64-token checkpoint segments). */
void naju_testing_set_fwd_pieces(int32_t pieces);

/* The forward's number of piece-mode ranges for these dims (0: group mode). */
int32_t naju_testing_fwd_pieces(const void* dims);

/* Forces the streaming-multiprocessor count that the automatic tiling
 * (piece mode, the wave model of the sequence-group count) is computed for;
 * sms <= 0 restores the current device's own count, queried once per device
 * (148 when no device can be queried). */
void naju_testing_set_sm_count(int32_t sms);

/* The SM count the tiling currently uses. */
int32_t naju_testing_sm_count(void);

/* Forward implementation: 0 = automatic (the tensor-core block-form kernel
 * for bf16 activations with d_state 64 or 128 and d_inner % 8 == 0, CUDA
 * cores otherwise), 1 = always CUDA cores, 2 = the tensor-core sub-chunk
 * kernel, 3 = the tensor-core block-form kernel, where tensor cores apply. */
void naju_testing_set_fwd_impl(int32_t impl);

/* The forward implementation for these dims: 1 = CUDA cores, 2 = tensor-core
 * sub-chunk kernel, 3 = tensor-core block-form kernel (0 for invalid dims). */
int32_t naju_testing_fwd_impl(const void* dims);

/* Backward implementation: 0 = automatic (the tensor-core block-form kernel
 * for bf16 activations with d_state 64 or 128 and d_inner % 8 == 0, d_state
 * 128 as two passes over 64-column state halves; CUDA cores otherwise),
 * 1 = always CUDA cores, 2 = the tensor-core sub-chunk kernel, 3 = the
 * block-form kernel (as automatic), where tensor cores apply. */
void naju_testing_set_bwd_impl(int32_t impl);

/* The backward implementation for these dims: 1 = CUDA cores, 2 = tensor-core
 * sub-chunk kernel, 3 = tensor-core block-form kernel (0 for invalid dims). */
int32_t naju_testing_bwd_impl(const void* dims);

/* Self-test of the tensor-core building block of the tensor-core scans:
 * D[128 x N] = A[128 x K] * B[N x K]^T (device pointers, row-major fp32)
 * computed with A in tensor memory, B in shared memory and kind::tf32 MMAs
 * (one thread block).  N, K multiples of 16, N <= 256, K + N <= 512.  A
 * completion wait that runs out sets NAJU_ERR_TIMEOUT in *status (device
 * int) and writes NaN to D. */
naju_status naju_testing_tc_mma(int32_t N, int32_t K, const float* A, const float* B, float* D,
                                int* status, void* stream);

/* Same product with both operands in shared memory.  A [rows_a x K] is staged
 * as a rows_a-row tile (rows_a 64 or 128) and the MMA reads 128 rows; only
 * the first rows_a rows of D are meaningful.  swz_a / swz_b select the
 * 128-byte swizzled K-major layout for A / B (K % 32 == 0), else no-swizzle
 * core matrices.  N in [16, 128], K in [16, 128], multiples of 16. */
naju_status naju_testing_tc_mma_ss(int32_t N, int32_t K, int32_t rows_a, int32_t swz_a,
                                   int32_t swz_b, const float* A, const float* B, float* D,
                                   int* status, void* stream);

/* General form of the same product, both operands in shared memory, in the
 * forms the block-form kernels use.  kind 0 (tf32): a_mn = 0 stores A as its
 * [M x K] tile, 128-byte swizzled (K-major operand); a_mn = 1 as the
 * transposed [K x M] tile with 32-byte swizzle atoms (MN-major operand, the
 * only layout tf32 accepts for it); likewise b_mn for B.  kind 1 (bf16): A and
 * B are split into bf16 hi + lo tiles in the 128-byte swizzled layout (one
 * tile serves both majors for 16-bit data) and D = hi.hi + hi.lo + lo.hi
 * (kind::f16 MMAs); the stored tiles are exactly 64 columns wide.  M is 64 or
 * 128; d_lane (0, or 16 with M = 64) is the tensor-memory lane offset of D.
 * D receives all 128 tensor-memory lanes of the N result columns, row-major
 * [128 x N], so the caller can check where an M = 64 result lands.  K in
 * {32, 64, 96, 128}; N a multiple of 16 up to 128 (of 32 for a tf32 MN-major
 * B). */
naju_status naju_testing_tc_mma_gen(int32_t M, int32_t N, int32_t K, int32_t a_mn, int32_t b_mn,
                                    int32_t d_lane, int32_t kind, const float* A, const float* B,
                                    float* D, int* status, void* stream);

/* The block-form kernels' fast exponential and sigmoids, for n device fp32
 * inputs x: ex = e^x computed as 2^(x log2 e) with the MUFU base-2 unit (PTX
 * ex2.approx.ftz; results below the normal range flush to zero), sig =
 * 1 / (1 + e^{-x}) with the approximate reciprocal, sig3 = the forward's
 * shared-reciprocal form of sigma(x) taken together with sigma(x / 2) and
 * sigma(-x) (each e^{-v} capped at 2^36), and silut = SiLU(x) = x sigma(x) as
 * h + h tanh(h), h = x / 2, with the MUFU tanh (PTX tanh.approx.f32; the
 * forward's output gate with bf16 outputs).  Device pointers, n >= 0. */
naju_status naju_testing_fast_math(const float* x, float* ex, float* sig, float* sig3,
                                   float* silut, int64_t n, void* stream);

#ifdef __cplusplus
}
#endif
#endif /* NAJU_TESTING_H_ */
