/*
 * naju.h -- C ABI of the B200 (sm_100a) Naju scan library.
 *
 * Naju (arXiv 2607.21000; Naju reproduction README, "Core equations" and the
 * block flowchart) is a native-discrete selective state-space block.  This
 * library implements its data-parallel hot path:
 *
 *   h_n   = SiLU(causal depthwise conv(u)_n)                    (optional)
 *   x_n   = f_n (.) x_{n-1} + i_n (.) (h_n B_n^T),  f = sigmoid(a), i = sigmoid(b)
 *   y_n   = x_n C_n / sqrt(d_state) + D (.) h_n
 *   out_n = y_n * SiLU(z_n)                                       (optional)
 *
 * its gradients, and a single-token decode step on a carried state.
 *
 * Shapes (row-major, contiguous; Bt = batch, L = seqlen, d = d_inner,
 * N = d_state, W = conv_width):
 *   u or h, a, b, z, y (out), dy, du/dh, da, db, dz : [Bt, L, d]  activation dtype
 *   B, C, dB, dC                                   : [Bt, L, N]  activation dtype
 *   x0, x_final, dx_final, dx0, decode state       : [Bt, d, N]  fp32
 *   D, dD, conv_b, dconv_b                         : [d]         fp32
 *   conv_w, dconv_w                                : [d, W]      fp32
 * Gates f, i are per (token, channel) and broadcast over the N state columns;
 * B and C are one N-vector per (batch, token), shared by all channels.  The
 * conv is a cross-correlation over the W most recent tokens with zero left
 * padding: p_t = conv_b + sum_k conv_w[k] u_{t-(W-1)+k}.
 *
 * Ownership and ordering.  The caller allocates every device buffer (inputs,
 * outputs and the workspace); the library never allocates, frees or
 * synchronises (except naju_last_device_status), and every call is enqueued
 * on the given CUDA stream (`stream` is a cudaStream_t; NULL = the legacy
 * default stream).  All pointers are device pointers unless stated.
 *
 * Errors.  Every entry point validates its arguments on the host before any
 * launch and returns NAJU_ERR_INVALID_ARG (null required pointer, bad size,
 * misaligned pointer: activations need 16-byte alignment) or
 * NAJU_ERR_UNSUPPORTED (d_state not in {16, 32, 64, 128}, conv_width != 4,
 * unknown dtype) without touching the GPU.  A failed launch returns
 * NAJU_ERR_CUDA.  Waits between thread blocks are bounded: when one gives up
 * it records NAJU_ERR_TIMEOUT in the workspace's status word (read with
 * naju_last_device_status) and the kernel returns instead of hanging.
 */
#ifndef NAJU_H_
#define NAJU_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    NAJU_OK = 0,
    NAJU_ERR_INVALID_ARG = 1,
    NAJU_ERR_UNSUPPORTED = 2,
    NAJU_ERR_CUDA = 3,
    NAJU_ERR_TIMEOUT = 4
} naju_status;

typedef enum { NAJU_F32 = 0, NAJU_BF16 = 1 } naju_dtype;

typedef struct {
    int64_t batch;      /* Bt >= 1                                        */
    int64_t seqlen;     /* L >= 1                                         */
    int64_t d_inner;    /* d >= 1                                         */
    int64_t d_state;    /* N in {16, 32, 64, 128}                         */
    int32_t conv_width; /* W; must be 4 when conv weights are passed      */
    int32_t dtype;      /* naju_dtype of the activation inputs            */
    int32_t out_dtype;  /* naju_dtype of y and of the activation grads;
                           bf16 inputs may write f32 or bf16 outputs,
                           f32 inputs write f32                            */
    int32_t reserved;   /* must be 0                                      */
} naju_dims;

/* Bytes of device workspace that naju_scan_fwd / naju_scan_bwd need for
 * these dims: state checkpoints written by the forward and read by the
 * backward, inter-block carry flags, the status word, and the backward's
 * partial sums.  0 if dims are invalid.  The workspace must be 256-byte
 * aligned, must not be shared by calls that may run concurrently, and must
 * be passed unchanged from a forward to the backward of the same inputs. */
size_t naju_scan_workspace_bytes(const naju_dims* dims);

/* Causal depthwise conv + SiLU (README flowchart, "causal depthwise conv +
 * SiLU"): h = SiLU(conv(u)).  u, h in dims->dtype (h in out_dtype);
 * conv_b may be NULL (zero bias).  Uses no workspace. */
naju_status naju_conv_silu_fwd(const naju_dims* dims, const void* u, const float* conv_w,
                               const float* conv_b, void* h, void* stream);

/* Gradient of naju_conv_silu_fwd given dh: writes du (out_dtype) and
 * overwrites dconv_w [d, W], dconv_b [d] (fp32, summed over batch and time;
 * dconv_b may be NULL). */
naju_status naju_conv_silu_bwd(const naju_dims* dims, const void* u, const float* conv_w,
                               const float* conv_b, const void* dh, void* du, float* dconv_w,
                               float* dconv_b, void* stream);

/* Forward scan (README, "Core equations"), fused with the conv + SiLU that
 * produces h when conv_w != NULL (then `hu` is u; otherwise `hu` is h) and
 * with the SiLU(z) output modulation when z != NULL.  D == NULL means no
 * feedthrough; x0 == NULL means a zero initial state.  b == NULL selects the
 * coupled single gate i = 1 - sigmoid(a) (the complementary gating analysed in
 * the paper's abstract) instead of i = sigmoid(b); the same holds for every
 * entry point below that takes b.  Writes y (out_dtype), optionally x_final,
 * and the state checkpoints the backward needs into the workspace. */
naju_status naju_scan_fwd(const naju_dims* dims, const void* hu, const float* conv_w,
                          const float* conv_b, const void* a, const void* b, const void* B,
                          const void* C, const void* z, const float* D, const float* x0,
                          void* y, float* x_final, void* workspace, size_t workspace_bytes,
                          void* stream);

/* Allocation-free forward for callers that cannot allocate device memory
 * (for example code running where no allocator is available, or a plugin
 * that is handed only its input and output buffers).  The Naju pages have no
 * counterpart: this is a library convenience.  Same arguments, checks and
 * results (y, optional x_final) as naju_scan_fwd, but no workspace: the
 * scratch is a fixed 32 MiB device array inside the library, reserved on
 * every GPU that loads the library until the process exits.
 * It always runs the CUDA-core forward kernel with the whole sequence as one
 * sequence group, whatever the dtype and d_state: bf16 calls with d_state 64
 * or 128 do not get the tensor-core kernel of naju_scan_fwd, and a small
 * batch leaves most of the GPU idle, so it is slower than naju_scan_fwd.  It
 * writes no checkpoints, so naju_scan_bwd cannot follow it.  The scratch
 * holds a work ticket and one flag per (batch element, channel tile):
 * batch * ceil(d_inner / P) <= about 8.4 million (P = 128, 64, 64, 32
 * channels for d_state 16, 32, 64, 128); larger problems return
 * NAJU_ERR_UNSUPPORTED before any launch.
 * The first call on each device looks up the array's device address (with
 * that device current) and keeps it until the process exits; make that first
 * call before any stream capture, and do not call it after a
 * cudaDeviceReset.  Every call shares the one array, and each call clears
 * what must start at zero; calls that may overlap on the GPU (other streams,
 * other threads) race on it and must be serialised by the caller. */
naju_status naju_scan_fwd_noalloc(const naju_dims* dims, const void* hu, const float* conv_w,
                                  const float* conv_b, const void* a, const void* b,
                                  const void* B, const void* C, const void* z, const float* D,
                                  const float* x0, void* y, float* x_final, void* stream);

/* Backward of naju_scan_fwd for a loss with gradient dy w.r.t. y and,
 * optionally, dx_final w.r.t. x_final.  Same inputs as the forward; the
 * workspace must hold that forward's checkpoints.  Writes dhu (du in fused
 * mode, dh otherwise), da, db, dB, dC and dz (when z != NULL) in out_dtype,
 * and overwrites dD (when D != NULL), dconv_w and dconv_b (fused mode) and
 * dx0 (when not NULL) in fp32.  With b == NULL (coupled gate) da includes the
 * write-gate path, db is not written and may be NULL. */
naju_status naju_scan_bwd(const naju_dims* dims, const void* hu, const float* conv_w,
                          const float* conv_b, const void* a, const void* b, const void* B,
                          const void* C, const void* z, const float* D, const float* x0,
                          const void* dy, const float* dx_final, void* dhu, void* da, void* db,
                          void* dB, void* dC, void* dz, float* dD, float* dconv_w,
                          float* dconv_b, float* dx0, void* workspace, size_t workspace_bytes,
                          void* stream);

/* One decode step (README, "Core equations", one token): h, a, b, z, y are
 * [batch, d_inner] in `dtype` (y too); B, C are [batch, d_state]; state
 * [batch, d_inner, d_state] fp32 is read and overwritten in place.  h is the
 * post-conv activation.  z and D may be NULL.  Uses no workspace. */
naju_status naju_scan_step(int64_t batch, int64_t d_inner, int64_t d_state, int32_t dtype,
                           const void* h, const void* a, const void* b, const void* B,
                           const void* C, const void* z, const float* D, float* state, void* y,
                           void* stream);

/* Decode step of the causal depthwise conv + SiLU (README flowchart, "causal
 * depthwise conv + SiLU", one token at a time).  u and h are [batch, d_inner]
 * in `dtype`; conv_w [d_inner, 4] and conv_b [d_inner] (NULL: no bias) fp32;
 * conv_state [batch, d_inner, 3] fp32 holds the previous three inputs of each
 * channel, oldest first (zeros at the start of a sequence, matching the
 * forward's left zero padding), and is updated in place to end with u.
 *   h = SiLU(conv_b + w[0] s[0] + w[1] s[1] + w[2] s[2] + w[3] u).
 * Uses no workspace.  Errors: INVALID_ARG for null or misaligned pointers or
 * bad sizes, UNSUPPORTED for another dtype, CUDA for launch errors. */
naju_status naju_conv_silu_step(int64_t batch, int64_t d_inner, int32_t dtype, const void* u,
                                const float* conv_w, const float* conv_b, float* conv_state,
                                void* h, void* stream);

/* naju_conv_silu_step fused into naju_scan_step: one decode token of the
 * whole path from the pre-conv input u [batch, d_inner] (same layouts and
 * in-place updates of conv_state and state as the two calls; no h round trip
 * through memory).  Uses no workspace. */
naju_status naju_scan_step_conv(int64_t batch, int64_t d_inner, int64_t d_state, int32_t dtype,
                                const void* u, const float* conv_w, const float* conv_b,
                                float* conv_state, const void* a, const void* b, const void* B,
                                const void* C, const void* z, const float* D, float* state,
                                void* y, void* stream);

/* Synchronises `stream`, reads the workspace's status word (NAJU_OK or
 * NAJU_ERR_TIMEOUT) and clears it.  Returns NAJU_ERR_CUDA if the stream
 * itself reports an error. */
naju_status naju_last_device_status(void* workspace, void* stream);

/* Static description of a status code. */
const char* naju_status_string(naju_status s);

#ifdef __cplusplus
}
#endif
#endif /* NAJU_H_ */
