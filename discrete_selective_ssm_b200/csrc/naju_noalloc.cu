// Allocation-free forward scan.
//
// naju_scan_fwd needs a caller-allocated workspace.  Some callers cannot
// allocate device memory at the point where they run the scan: code executed
// inside a memory-pool-less runtime, plugins handed only input and output
// buffers by a host framework, or a step that must not grow the allocator's
// footprint.  naju_scan_fwd_noalloc serves them: its only scratch memory is a
// fixed array in this file, reserved on every GPU when the library's module
// is loaded and kept until the process exits.
//
// The whole sequence runs as one group on the CUDA-core forward kernel (no
// sequence split, so no waits between thread blocks), and without
// checkpoints (nothing can follow with a backward).  The scratch then holds
// only the work ticket and one ready-flag per (batch, channel tile): problems
// with more flags than fit in kScratchBytes are rejected.
#include <mutex>

#include "naju.h"
#include "naju_common.cuh"
#include "naju_kernels.h"

namespace {

constexpr size_t kScratchBytes = (size_t)32 << 20;  // 32 MiB, stated in naju.h
constexpr int kMaxDevices = 64;

// The scratch: one copy per GPU that loads the library.  Host code never
// dereferences this name; it only asks the runtime for its device address.
static __device__ __align__(256) unsigned char g_scratch[kScratchBytes];

std::mutex g_mu;
void* g_addr[kMaxDevices] = {};

// Device address of g_scratch on the current device (looked up once per
// device, with that device current, and kept for the life of the process: a
// cudaDeviceReset invalidates it).
cudaError_t scratch_address(void** out) {
    int dev = -1;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> lk(g_mu);
    if (!g_addr[dev]) {
        void* p = nullptr;
        e = cudaGetSymbolAddress(&p, g_scratch);
        if (e != cudaSuccess) return e;
        g_addr[dev] = p;
    }
    *out = g_addr[dev];
    return cudaSuccess;
}

inline size_t up256(size_t x) { return (x + 255) & ~size_t(255); }
inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) % 16) == 0; }

}  // namespace

extern "C" {

naju_status naju_scan_fwd_noalloc(const naju_dims* dims, const void* hu, const float* conv_w,
                                  const float* conv_b, const void* a, const void* b,
                                  const void* B, const void* C, const void* z, const float* D,
                                  const float* x0, void* y, float* x_final, void* stream) {
    using namespace naju;
    const naju_status chk = check_dims(dims);  // the workspace forward's own checks
    if (chk != NAJU_OK) return chk;
    const int64_t N = dims->d_state;
    if (conv_w && dims->conv_width != 4) return NAJU_ERR_UNSUPPORTED;
    if (!hu || !a || !B || !C || !y) return NAJU_ERR_INVALID_ARG;  // b NULL: coupled gate
    const void* required[] = {hu, a, b, B, C, y};
    for (const void* q : required)
        if (!aligned16(q)) return NAJU_ERR_INVALID_ARG;
    const void* optional[] = {z, x0, x_final};
    for (const void* q : optional)
        if (q && !aligned16(q)) return NAJU_ERR_INVALID_ARG;

    const int64_t Bt = dims->batch, L = dims->seqlen, d = dims->d_inner;
    const int ntiles = (int)((d + fwd_channels_per_block(N) - 1) / fwd_channels_per_block(N));
    // One sequence group covering the whole sequence (a single segment of L
    // rounded up to the chunk), no checkpoints: the header and the flags.
    const size_t off_flags = sizeof(WsHeader);
    const size_t need = up256(off_flags + sizeof(int) * (size_t)Bt * ntiles);
    if (need > kScratchBytes) return NAJU_ERR_UNSUPPORTED;  // beyond the fixed scratch

    void* base = nullptr;
    if (scratch_address(&base) != cudaSuccess) return NAJU_ERR_CUDA;
    char* ws = static_cast<char*>(base);
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    // The scratch keeps the previous call's contents: clear the ticket and
    // the flags (the status word is unused: nothing waits).
    WsHeader* hdr = reinterpret_cast<WsHeader*>(ws);
    if (cudaMemsetAsync(&hdr->fwd_ticket, 0, sizeof(int), s) != cudaSuccess ||
        cudaMemsetAsync(ws + off_flags, 0, sizeof(int) * (size_t)Bt * ntiles, s) != cudaSuccess)
        return NAJU_ERR_CUDA;

    FwdParams p{};
    p.hu = hu; p.conv_w = conv_w; p.conv_b = conv_b; p.a = a; p.b = b; p.B = B; p.C = C;
    p.z = z; p.D = D; p.x0 = x0; p.y = y; p.x_final = x_final;
    p.ckpt = nullptr;  // no checkpoints
    p.flags = reinterpret_cast<int*>(ws + off_flags);
    p.hdr = hdr;
    p.Bt = Bt; p.L = L; p.d = d; p.N = N;
    p.T_ck = (int)(((L + kFwdChunk - 1) / kFwdChunk) * kFwdChunk);
    p.nck = 1;
    p.seg_per_group = 1;
    p.ngroups = 1;
    p.ntiles = ntiles;
    p.scale = 1.0f / sqrtf((float)N);
    p.wait_limit = 1;
    p.fault_skip_publish = 0;
    return launch_scan_fwd(p, dims->dtype, dims->out_dtype, s) == cudaSuccess ? NAJU_OK
                                                                               : NAJU_ERR_CUDA;
}

}  // extern "C"
