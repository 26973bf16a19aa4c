// Internal launch interface between the C ABI layer and the kernels.
#pragma once
#include <cuda_runtime.h>
#include <stdint.h>

#include "naju.h"

namespace naju {

struct WsHeader;

// Host-side validation of the dims shared by every sequence entry point:
// NAJU_OK, NAJU_ERR_INVALID_ARG (sizes out of range) or NAJU_ERR_UNSUPPORTED.
naju_status check_dims(const naju_dims* dm);

constexpr int kFwdChunk = 16;   // tokens staged per forward chunk
constexpr int kBwdSub = 64;     // tokens per backward work item
constexpr int kBwdChunk = 16;   // tokens per backward contraction block

struct FwdParams {
    const void* hu;
    const float* conv_w;
    const float* conv_b;
    const void* a;
    const void* b;
    const void* B;
    const void* C;
    const void* z;
    const float* D;
    const float* x0;
    void* y;
    float* x_final;
    float* ckpt;        // [Bt][nck+1][d][N] fp32 state at segment starts (+ final);
                        // CUDA-core kernel, one group: may be null (no checkpoints)
    int* flags;         // [ngroups][Bt][ntiles]
    WsHeader* hdr;
    int64_t Bt, L, d, N;
    int T_ck;           // tokens per checkpoint segment
    int nck;            // number of segments = ceil(L / T_ck)
    int seg_per_group;  // segments per sequence group
    int ngroups;
    int ntiles;         // channel tiles = ceil(d / P)
    float scale;        // 1 / sqrt(N)
    long long wait_limit;
    int fault_skip_publish;
    int npieces;        // tensor-core kernel: > 0 for piece mode (ngroups == 1)
};

struct BwdParams {
    const void* hu;
    const float* conv_w;
    const float* conv_b;
    const void* a;
    const void* b;
    const void* B;
    const void* C;
    const void* z;
    const float* D;
    const void* dy;
    const float* dx_final;
    void* dhu;
    void* da;
    void* db;
    void* dz;
    float* dx0;
    const float* ckpt;     // written by the forward, one state per kBwdSub tokens
    float* carry;          // [ngroups][Bt][d][N] adjoint carries between groups
    int* flags;            // [ngroups][Bt][ntiles]
    float* dBCp;           // [nclus][Bt][L][2][N] partial dB, dC over channel clusters
                           // (block backward: one accumulator [Bt][ceil(L/4)][2][N][4])
    float* chan_part;      // [Bt*ngroups][d][8] partial dD, dconv_w[4], dconv_b
    float* conv_edge;      // [Bt][ngroups][2][3][d]: first 3 dp / last 3 partial du
    float* rgb_part;       // block backward, d_state 128: [2][Bt][L][d] partial R, GB of
                           // state columns 0..63 (first pass), read by the second
    float* tail_part;      // same: [Bt][nsub][d] partial H . x_63 of each block
    WsHeader* hdr;
    int64_t Bt, L, d, N;
    int T_ck, nck;         // forward checkpoint spacing (== kBwdSub) and count
    int nsub;              // ceil(L / kBwdSub) blocks
    int blk_per_group;     // blocks per sequence group
    int ngroups;
    int ntiles;
    int nclus;             // ceil(ntiles / cluster size)
    int npieces;           // tensor-core kernel: > 0 for piece mode (ngroups == 2)
    float scale;
    long long wait_limit;
    int fault_skip_publish;
};

int fwd_channels_per_block(int64_t N);
int bwd_channels_per_block(int64_t N);
int bwd_cluster_size(int tiles);

cudaError_t launch_scan_fwd(const FwdParams& p, int dtype, int out_dtype, cudaStream_t st);
// Tensor-core forward (bf16 activations, d_state 64 or 128, 128 channels per block).
bool fwd_tc_supported(int dtype, int64_t N, int64_t d);
int fwd_tc_channels_per_block();
cudaError_t launch_scan_fwd_tc(const FwdParams& p, int out_dtype, cudaStream_t st);
cudaError_t launch_scan_bwd(const BwdParams& p, int dtype, int out_dtype, void* dB, void* dC,
                            float* dD, float* dconv_w, float* dconv_b, cudaStream_t st);
// Tensor-core backward (bf16 activations, d_state 64 or 128, 128 channels per
// block, one dB/dC partial set per channel tile), then the reductions.
bool bwd_tc_supported(int dtype, int64_t N, int64_t d);
cudaError_t launch_scan_bwd_tc_main(const BwdParams& p, int out_dtype, cudaStream_t st);
cudaError_t launch_bwd_reductions(const BwdParams& p, int out_dtype, void* dB, void* dC,
                                  float* dD, float* dw, float* dbias, cudaStream_t st);
// Block-form tensor-core forward (bf16 activations, d_state 64 or 128,
// checkpoints every 64 tokens).
bool fwd_blk_supported(int dtype, int64_t N, int64_t d, int T_ck);
cudaError_t launch_scan_fwd_blk(const FwdParams& p, int out_dtype, cudaStream_t st);
// Block-form tensor-core backward (bf16 activations, d_state 64 or 128; 128 as
// two passes over 64-column state halves through p.rgb_part / p.tail_part):
// dB / dC go into an fp32 accumulator [Bt][ceil(L/4)][2][N][4] at p.dBCp (zeroed by the
// launch); launch_bwd_reductions_acc then finishes dB, dC and the per-channel
// sums.
bool bwd_blk_supported(int dtype, int64_t N, int64_t d);
cudaError_t launch_scan_bwd_blk(const BwdParams& p, int out_dtype, cudaStream_t st);
cudaError_t launch_finish_dBC(const BwdParams& p, int out_dtype, void* dB, void* dC,
                              cudaStream_t st);
cudaError_t launch_bwd_reductions_acc(const BwdParams& p, int out_dtype, void* dB, void* dC,
                                      float* dD, float* dw, float* dbias, cudaStream_t st);
cudaError_t launch_conv_fwd(int64_t Bt, int64_t L, int64_t d, const void* u, const float* w,
                            const float* bias, void* h, int dtype, int out_dtype,
                            cudaStream_t st);
cudaError_t launch_conv_bwd(int64_t Bt, int64_t L, int64_t d, const void* u, const float* w,
                            const float* bias, const void* dh, void* du, float* dw,
                            float* dbias, int dtype, int out_dtype, cudaStream_t st);
cudaError_t launch_scan_step(int64_t Bt, int64_t d, int64_t N, const void* h, const void* a,
                             const void* b, const void* B, const void* C, const void* z,
                             const float* D, float* state, void* y, int dtype,
                             const float* conv_w, const float* conv_b, float* conv_state,
                             cudaStream_t st);
cudaError_t launch_conv_step(int64_t Bt, int64_t d, const void* u, const float* w,
                             const float* bias, float* conv_state, void* h, int dtype,
                             cudaStream_t st);

}  // namespace naju
