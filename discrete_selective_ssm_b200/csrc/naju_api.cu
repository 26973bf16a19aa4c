// C ABI of the Naju scan library: argument checks, workspace layout and
// kernel launches.  See include/naju.h for the contract of each entry point.
#include <stdint.h>
#include <string.h>

#include <algorithm>
#include <atomic>
#include <cmath>

#include "naju.h"
#include "naju_common.cuh"
#include "naju_kernels.h"
#include "naju_testing.h"

using namespace naju;

namespace {

constexpr int kTck = kBwdSub;      // tokens per forward checkpoint segment (= backward block)
constexpr long long kDefaultWait = 1LL << 21;

long long g_wait_limit = kDefaultWait;
int g_skip_publish = 0;
int g_fwd_groups = 0;
int g_bwd_groups = 0;
int g_bwd_pieces = 0;  // 0 automatic, < 0 never, > 0 that many ranges
int g_fwd_pieces = 0;  // the same for the tensor-core forward
int g_fwd_impl = 0;  // 0 automatic, 1 CUDA cores, 2 tensor-core sub-chunk, 3 block form
int g_bwd_impl = 0;  // 0 automatic, 1 CUDA cores, 2 tensor-core sub-chunk, 3 block form
int g_sm_override = 0;  // > 0: SM count used by the tiling (tests)

// Streaming multiprocessors of the current device, queried once per device
// ordinal (the tensor-core kernels run one block per SM, so the tiling below
// depends on it).  148 (B200) when no device can be queried.
constexpr int kMaxDevices = 64;
std::atomic<int> g_sm_cache[kMaxDevices];

int sm_count() {
    if (g_sm_override > 0) return g_sm_override;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0) {
        cudaGetLastError();
        return 148;
    }
    if (dev < kMaxDevices) {
        const int c = g_sm_cache[dev].load(std::memory_order_relaxed);
        if (c > 0) return c;
    }
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n < 1) {
        cudaGetLastError();
        return 148;
    }
    if (dev < kMaxDevices) g_sm_cache[dev].store(n, std::memory_order_relaxed);
    return n;
}

inline bool aligned(const void* ptr, size_t a) {
    return (reinterpret_cast<uintptr_t>(ptr) % a) == 0;
}
inline int64_t cdiv(int64_t a, int64_t b) { return (a + b - 1) / b; }
inline size_t up256(size_t x) { return (x + 255) & ~size_t(255); }

// Workspace layout (every region 256-byte aligned).
struct Layout {
    bool fwd_tc, bwd_tc;
    int nck, ngroups, seg_per_group, ntiles_f, npieces_f;
    int nsub, nclus, ntiles_b, bgroups, blk_per_group, npieces;
    size_t off_fflags, off_bflags, off_ckpt, off_carry, off_dbc, off_chan, off_edge, off_rgb,
        off_tail, total;
};

bool use_fwd_tc(const naju_dims* dm) {
    if (g_fwd_impl == 1) return false;
    return fwd_tc_supported(dm->dtype, dm->d_state, dm->d_inner);
}
bool use_bwd_tc(const naju_dims* dm) {
    if (g_bwd_impl == 1) return false;
    return bwd_tc_supported(dm->dtype, dm->d_state, dm->d_inner);
}
// The block-form kernels are the automatic choice wherever they apply; the
// sub-chunk kernels stay reachable for testing (impl 2).
bool use_fwd_blk(const naju_dims* dm) {
    return use_fwd_tc(dm) && g_fwd_impl != 2 &&
           fwd_blk_supported(dm->dtype, dm->d_state, dm->d_inner, kTck);
}
bool use_bwd_blk(const naju_dims* dm) {
    return use_bwd_tc(dm) && g_bwd_impl != 2 &&
           bwd_blk_supported(dm->dtype, dm->d_state, dm->d_inner);
}

// Tensor-core kernels run one block per SM, so the launch's last wave
// decides the time.  Sequence-group count for `units` blocks' worth of work
// per group over `nseg` 64-token segments: the g (at most 16) with the least
// modelled time: waves of units * G blocks, G the groups after rounding to
// whole segments, each over ceil(nseg / g) segments, plus `extra` (a share of
// a full pass) for the early (backward) or update-only (forward) pass that
// all but the last group run.  Fitted on sweeps of the group count: 0.17 for
// the backward's early pass, 0.7 for the forward's update-only pass (it runs
// most of the forward's per-token work); for 8 x 2048 x 1536 x 64 these pick
// 3 backward groups and 1 forward group, for 2 x 8192 x 2048 x 128 9 and 9.
constexpr double kBwdEarlyPass = 0.17, kFwdUpdatePass = 0.7;
int tc_groups(int64_t units, int nseg, int sms, double extra) {
    if (units >= sms) return 1;  // a wave or more: piece mode, or whole waves already
    int best = 1;
    double best_cost = 1e30;
    for (int g = 1; g <= nseg && g <= 16; ++g) {
        const int64_t per = cdiv(nseg, g), groups = cdiv(nseg, per);
        const double waves = (double)cdiv(units * groups, sms);
        const double cost =
            waves * (double)per / nseg * (1.0 + extra * (double)(groups - 1) / groups);
        if (cost < best_cost - 1e-12) {
            best_cost = cost;
            best = g;
        }
    }
    return best;
}

// Backward tiling: channel tiles, dB/dC partial sets, sequence groups.
struct BwdTiling {
    int ntiles, nparts, bgroups, blk_per_group, npieces;
};
BwdTiling bwd_tiling(const naju_dims* dm, int nsub, bool tc, int sms) {
    BwdTiling b{};
    const int64_t d = dm->d_inner;
    if (tc) {
        // 128 channels per block (one per tensor-memory lane), one partial set
        // per tile; one block per SM.
        b.ntiles = (int)cdiv(d, 128);
        b.nparts = b.ntiles;
    } else {
        // Clusters of channel tiles share one partial set; two blocks per SM.
        const int tiles = (int)cdiv(d, bwd_channels_per_block(dm->d_state));
        const int cl = bwd_cluster_size(tiles);
        b.nparts = (int)cdiv(tiles, cl);
        b.ntiles = b.nparts * cl;
    }
    // Tensor-core piece mode: with at least one unit (128 channels of one
    // batch element) per SM but not a whole number of waves, cut the units'
    // blocks into one equal range per SM instead of leaving the last wave
    // part-empty.  Sequence groups are not used then (two carry slots).
    if (tc && g_bwd_groups <= 0 && g_bwd_pieces >= 0 && nsub >= 2) {
        const int64_t units = dm->batch * (int64_t)b.ntiles;
        int np = 0;
        if (g_bwd_pieces > 0) {
            np = units >= g_bwd_pieces ? g_bwd_pieces : 0;
        } else if (units >= sms && units % sms != 0) {
            np = sms;
        }
        if (np > 0) {
            b.npieces = np;
            b.bgroups = 2;
            b.blk_per_group = nsub;
            return b;
        }
    }
    int gb = g_bwd_groups;
    if (gb <= 0) {
        const int64_t ctas = dm->batch * (int64_t)b.ntiles;
        if (tc) {
            gb = tc_groups(ctas, nsub, sms, kBwdEarlyPass);
        } else {
            const int64_t want = 4 * (int64_t)sms;
            gb = ctas >= want ? 1 : (int)cdiv(want, ctas);
        }
    }
    if (gb > nsub) gb = nsub;
    b.blk_per_group = (int)cdiv(nsub, gb);
    b.bgroups = (int)cdiv(nsub, b.blk_per_group);
    return b;
}

int auto_groups(const naju_dims* dm, int nck, int ntiles_f, bool tc, int sms) {
    if (g_fwd_groups > 0) return g_fwd_groups < nck ? g_fwd_groups : nck;
    const int64_t items = dm->batch * (int64_t)ntiles_f;
    // One tensor-core block per SM (its operand stages fill most of the
    // shared memory): the wave model; three CUDA-core blocks per SM.
    if (tc) return tc_groups(items, nck, sms, kFwdUpdatePass);
    const int64_t want = 3 * (int64_t)sms;
    if (items >= want) return 1;
    int64_t g = cdiv(want, items);
    return (int)(g < nck ? g : nck);
}

// Tensor-core forward piece mode: the rule of the backward's (one range of
// checkpoint segments per SM when the 128-channel units fill at least one
// wave but not a whole number of them); one flag slot per unit.
int fwd_pieces(const naju_dims* dm, int nck, int ntiles_f, bool tc, int sms) {
    if (!tc || g_fwd_groups > 0 || g_fwd_pieces < 0 || nck < 2) return 0;
    const int64_t units = dm->batch * (int64_t)ntiles_f;
    if (g_fwd_pieces > 0) return units >= g_fwd_pieces ? g_fwd_pieces : 0;
    return (units >= sms && units % sms != 0) ? sms : 0;
}

Layout layout(const naju_dims* dm) {
    Layout l{};
    const int sms = sm_count();
    const int64_t Bt = dm->batch, L = dm->seqlen, d = dm->d_inner, N = dm->d_state;
    l.nck = (int)cdiv(L, kTck);
    l.fwd_tc = use_fwd_tc(dm);
    l.ntiles_f = (int)cdiv(d, l.fwd_tc ? fwd_tc_channels_per_block() : fwd_channels_per_block(N));
    l.npieces_f = fwd_pieces(dm, l.nck, l.ntiles_f, l.fwd_tc, sms);
    int g = l.npieces_f > 0 ? 1 : auto_groups(dm, l.nck, l.ntiles_f, l.fwd_tc, sms);
    l.seg_per_group = (int)cdiv(l.nck, g);
    l.ngroups = (int)cdiv(l.nck, l.seg_per_group);
    l.nsub = (int)cdiv(L, kBwdSub);
    l.bwd_tc = use_bwd_tc(dm);
    const BwdTiling bt = bwd_tiling(dm, l.nsub, l.bwd_tc, sms);
    l.ntiles_b = bt.ntiles;
    l.nclus = bt.nparts;
    l.bgroups = bt.bgroups;
    l.blk_per_group = bt.blk_per_group;
    l.npieces = bt.npieces;
    // Regions sized for the larger of the two backward tilings, so the
    // workspace size does not depend on which backward kernel runs.
    const BwdTiling bo = bwd_tiling(dm, l.nsub, !l.bwd_tc, sms);
    const bool other_ok = l.bwd_tc || bwd_tc_supported(dm->dtype, N, d);
    const int64_t flags_n = std::max<int64_t>((int64_t)bt.bgroups * bt.ntiles,
                                              other_ok ? (int64_t)bo.bgroups * bo.ntiles : 0);
    const int64_t groups_n = std::max(bt.bgroups, other_ok ? bo.bgroups : 0);
    const int64_t parts_n = std::max(bt.nparts, other_ok ? bo.nparts : 0);
    size_t off = sizeof(WsHeader);
    l.off_fflags = off;
    // Flags for the larger of the two forward tilings (at most nck groups), so
    // the workspace size does not depend on which forward kernel runs.
    off = up256(off + sizeof(int) * (size_t)l.nck * Bt * cdiv(d, 32));
    l.off_bflags = off;
    off = up256(off + sizeof(int) * (size_t)flags_n * Bt);
    l.off_ckpt = off;
    off = up256(off + sizeof(float) * (size_t)Bt * (l.nck + 1) * d * N);
    l.off_carry = off;
    off = up256(off + sizeof(float) * (size_t)groups_n * Bt * d * N);
    l.off_dbc = off;
    // (the block backward's accumulator pads the tokens to a multiple of four)
    off = up256(off + sizeof(float) * (size_t)parts_n * Bt * ((L + 3) / 4 * 4) * 2 * N);
    l.off_chan = off;
    off = up256(off + sizeof(float) * (size_t)Bt * groups_n * d * 8);
    l.off_edge = off;
    off = up256(off + sizeof(float) * (size_t)Bt * groups_n * 2 * 3 * d);
    // d_state 128 block backward: the first pass's partial R, GB and tails
    const bool halves = N == 128 && bwd_blk_supported(dm->dtype, N, d);
    l.off_rgb = off;
    off = up256(off + (halves ? sizeof(float) * (size_t)2 * Bt * L * d : 0));
    l.off_tail = off;
    off = up256(off + (halves ? sizeof(float) * (size_t)Bt * l.nsub * d : 0));
    l.total = off;
    return l;
}

inline naju_status cuda_status(cudaError_t e) { return e == cudaSuccess ? NAJU_OK : NAJU_ERR_CUDA; }

#define NAJU_REQUIRE(cond) \
    do {                   \
        if (!(cond)) return NAJU_ERR_INVALID_ARG; \
    } while (0)

inline bool ok_act(const void* p) { return p && aligned(p, 16); }
inline bool ok_opt(const void* p) { return !p || aligned(p, 16); }

}  // namespace

namespace naju {

naju_status check_dims(const naju_dims* dm) {
    if (!dm) return NAJU_ERR_INVALID_ARG;
    if (dm->batch < 1 || dm->seqlen < 1 || dm->d_inner < 1 || dm->reserved != 0)
        return NAJU_ERR_INVALID_ARG;
    if (dm->batch > (1 << 20) || dm->seqlen > (1LL << 26) || dm->d_inner > (1 << 20))
        return NAJU_ERR_INVALID_ARG;
    if (dm->batch * dm->seqlen * dm->d_inner > (1LL << 40)) return NAJU_ERR_INVALID_ARG;
    if (dm->d_state != 16 && dm->d_state != 32 && dm->d_state != 64 && dm->d_state != 128)
        return NAJU_ERR_UNSUPPORTED;
    if (dm->dtype != NAJU_F32 && dm->dtype != NAJU_BF16) return NAJU_ERR_UNSUPPORTED;
    if (dm->out_dtype != NAJU_F32 && dm->out_dtype != NAJU_BF16) return NAJU_ERR_UNSUPPORTED;
    if (dm->dtype == NAJU_F32 && dm->out_dtype != NAJU_F32) return NAJU_ERR_UNSUPPORTED;
    return NAJU_OK;
}

}  // namespace naju

extern "C" {

size_t naju_scan_workspace_bytes(const naju_dims* dims) {
    if (check_dims(dims) != NAJU_OK) return 0;
    return layout(dims).total;
}

naju_status naju_conv_silu_fwd(const naju_dims* dims, const void* u, const float* conv_w,
                               const float* conv_b, void* h, void* stream) {
    naju_status st = check_dims(dims);
    if (st != NAJU_OK) return st;
    if (dims->conv_width != 4) return NAJU_ERR_UNSUPPORTED;
    NAJU_REQUIRE(ok_act(u) && ok_act(h) && conv_w && ok_opt(conv_b));
    return cuda_status(launch_conv_fwd(dims->batch, dims->seqlen, dims->d_inner, u, conv_w,
                                       conv_b, h, dims->dtype, dims->out_dtype,
                                       static_cast<cudaStream_t>(stream)));
}

naju_status naju_conv_silu_bwd(const naju_dims* dims, const void* u, const float* conv_w,
                               const float* conv_b, const void* dh, void* du, float* dconv_w,
                               float* dconv_b, void* stream) {
    naju_status st = check_dims(dims);
    if (st != NAJU_OK) return st;
    if (dims->conv_width != 4) return NAJU_ERR_UNSUPPORTED;
    if (dims->dtype != dims->out_dtype) return NAJU_ERR_UNSUPPORTED;  // dh arrives in dtype
    NAJU_REQUIRE(ok_act(u) && ok_act(dh) && ok_act(du) && conv_w && dconv_w);
    return cuda_status(launch_conv_bwd(dims->batch, dims->seqlen, dims->d_inner, u, conv_w,
                                       conv_b, dh, du, dconv_w, dconv_b, dims->dtype,
                                       dims->out_dtype, static_cast<cudaStream_t>(stream)));
}

naju_status naju_scan_fwd(const naju_dims* dims, const void* hu, const float* conv_w,
                          const float* conv_b, const void* a, const void* b, const void* B,
                          const void* C, const void* z, const float* D, const float* x0,
                          void* y, float* x_final, void* workspace, size_t workspace_bytes,
                          void* stream) {
    naju_status st = check_dims(dims);
    if (st != NAJU_OK) return st;
    if (conv_w && dims->conv_width != 4) return NAJU_ERR_UNSUPPORTED;
    NAJU_REQUIRE(ok_act(hu) && ok_act(a) && ok_opt(b) && ok_act(B) && ok_act(C) && ok_act(y));
    NAJU_REQUIRE(ok_opt(z) && ok_opt(x0) && ok_opt(x_final));
    NAJU_REQUIRE(workspace && aligned(workspace, 256));
    const Layout l = layout(dims);
    NAJU_REQUIRE(workspace_bytes >= l.total);
    NAJU_REQUIRE((int64_t)l.ngroups * dims->batch * l.ntiles_f < (1LL << 31));
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    char* ws = static_cast<char*>(workspace);
    WsHeader* hdr = reinterpret_cast<WsHeader*>(ws);
    cudaError_t e = cudaMemsetAsync(&hdr->fwd_ticket, 0, sizeof(int), s);
    if (e == cudaSuccess)
        e = cudaMemsetAsync(ws + l.off_fflags, 0,
                            sizeof(int) * (size_t)l.ngroups * dims->batch * l.ntiles_f, s);
    if (e != cudaSuccess) return NAJU_ERR_CUDA;
    FwdParams p{};
    p.hu = hu; p.conv_w = conv_w; p.conv_b = conv_b; p.a = a; p.b = b; p.B = B; p.C = C;
    p.z = z; p.D = D; p.x0 = x0; p.y = y; p.x_final = x_final;
    p.ckpt = reinterpret_cast<float*>(ws + l.off_ckpt);
    p.flags = reinterpret_cast<int*>(ws + l.off_fflags);
    p.hdr = hdr;
    p.Bt = dims->batch; p.L = dims->seqlen; p.d = dims->d_inner; p.N = dims->d_state;
    p.T_ck = kTck; p.nck = l.nck; p.seg_per_group = l.seg_per_group; p.ngroups = l.ngroups;
    p.ntiles = l.ntiles_f;
    p.npieces = l.npieces_f;
    p.scale = 1.0f / std::sqrt((float)dims->d_state);
    p.wait_limit = g_wait_limit;
    p.fault_skip_publish = g_skip_publish;
    if (use_fwd_blk(dims))
        return cuda_status(launch_scan_fwd_blk(p, dims->out_dtype, s));
    if (l.fwd_tc) return cuda_status(launch_scan_fwd_tc(p, dims->out_dtype, s));
    return cuda_status(launch_scan_fwd(p, dims->dtype, dims->out_dtype, s));
}

naju_status naju_scan_bwd(const naju_dims* dims, const void* hu, const float* conv_w,
                          const float* conv_b, const void* a, const void* b, const void* B,
                          const void* C, const void* z, const float* D, const float* x0,
                          const void* dy, const float* dx_final, void* dhu, void* da, void* db,
                          void* dB, void* dC, void* dz, float* dD, float* dconv_w,
                          float* dconv_b, float* dx0, void* workspace, size_t workspace_bytes,
                          void* stream) {
    (void)x0;  // the forward's checkpoint 0 holds the initial state
    naju_status st = check_dims(dims);
    if (st != NAJU_OK) return st;
    if (conv_w && dims->conv_width != 4) return NAJU_ERR_UNSUPPORTED;
    NAJU_REQUIRE(ok_act(hu) && ok_act(a) && ok_opt(b) && ok_act(B) && ok_act(C) && ok_act(dy));
    NAJU_REQUIRE(ok_act(dhu) && ok_act(da) && ok_act(dB) && ok_act(dC));
    NAJU_REQUIRE(b ? ok_act(db) : ok_opt(db));
    NAJU_REQUIRE(ok_opt(z) && ok_opt(dx_final) && ok_opt(dx0));
    NAJU_REQUIRE(!z || ok_act(dz));
    NAJU_REQUIRE(!conv_w || dconv_w);
    NAJU_REQUIRE(workspace && aligned(workspace, 256));
    const Layout l = layout(dims);
    NAJU_REQUIRE(workspace_bytes >= l.total);
    NAJU_REQUIRE((int64_t)l.bgroups * dims->batch * l.ntiles_b < (1LL << 31));
    NAJU_REQUIRE(l.bgroups <= 65535 && dims->batch <= 65535);
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    char* ws = static_cast<char*>(workspace);
    WsHeader* hdr = reinterpret_cast<WsHeader*>(ws);
    cudaError_t e = cudaMemsetAsync(&hdr->bwd_ticket, 0, sizeof(int), s);
    if (e == cudaSuccess)
        e = cudaMemsetAsync(ws + l.off_bflags, 0,
                            sizeof(int) * (size_t)l.bgroups * dims->batch * l.ntiles_b, s);
    if (e != cudaSuccess) return NAJU_ERR_CUDA;
    BwdParams p{};
    p.hu = hu; p.conv_w = conv_w; p.conv_b = conv_b; p.a = a; p.b = b; p.B = B; p.C = C;
    p.z = z; p.D = D; p.dy = dy; p.dx_final = dx_final;
    p.dhu = dhu; p.da = da; p.db = db; p.dz = dz; p.dx0 = dx0;
    p.ckpt = reinterpret_cast<const float*>(ws + l.off_ckpt);
    p.carry = reinterpret_cast<float*>(ws + l.off_carry);
    p.flags = reinterpret_cast<int*>(ws + l.off_bflags);
    p.dBCp = reinterpret_cast<float*>(ws + l.off_dbc);
    p.chan_part = reinterpret_cast<float*>(ws + l.off_chan);
    p.conv_edge = reinterpret_cast<float*>(ws + l.off_edge);
    p.rgb_part = reinterpret_cast<float*>(ws + l.off_rgb);
    p.tail_part = reinterpret_cast<float*>(ws + l.off_tail);
    p.hdr = hdr;
    p.Bt = dims->batch; p.L = dims->seqlen; p.d = dims->d_inner; p.N = dims->d_state;
    p.T_ck = kTck; p.nck = l.nck; p.nsub = l.nsub; p.ntiles = l.ntiles_b; p.nclus = l.nclus;
    p.blk_per_group = l.blk_per_group; p.ngroups = l.bgroups; p.npieces = l.npieces;
    p.scale = 1.0f / std::sqrt((float)dims->d_state);
    p.wait_limit = g_wait_limit;
    p.fault_skip_publish = g_skip_publish;
    if (use_bwd_blk(dims)) {
        e = launch_scan_bwd_blk(p, dims->out_dtype, s);
        if (e == cudaSuccess)
            e = launch_bwd_reductions_acc(p, dims->out_dtype, dB, dC, dD, dconv_w, dconv_b, s);
        return cuda_status(e);
    }
    if (l.bwd_tc) {
        e = launch_scan_bwd_tc_main(p, dims->out_dtype, s);
        if (e == cudaSuccess)
            e = launch_bwd_reductions(p, dims->out_dtype, dB, dC, dD, dconv_w, dconv_b, s);
        return cuda_status(e);
    }
    return cuda_status(launch_scan_bwd(p, dims->dtype, dims->out_dtype, dB, dC, dD, dconv_w,
                                       dconv_b, s));
}

naju_status naju_scan_step(int64_t batch, int64_t d_inner, int64_t d_state, int32_t dtype,
                           const void* h, const void* a, const void* b, const void* B,
                           const void* C, const void* z, const float* D, float* state, void* y,
                           void* stream) {
    if (batch < 1 || d_inner < 1 || batch > 65535) return NAJU_ERR_INVALID_ARG;
    if (d_state != 16 && d_state != 32 && d_state != 64 && d_state != 128)
        return NAJU_ERR_UNSUPPORTED;
    if (dtype != NAJU_F32 && dtype != NAJU_BF16) return NAJU_ERR_UNSUPPORTED;
    NAJU_REQUIRE(ok_act(h) && ok_act(a) && ok_opt(b) && ok_act(B) && ok_act(C) && ok_act(y));
    NAJU_REQUIRE(ok_opt(z) && ok_act(state));
    return cuda_status(launch_scan_step(batch, d_inner, d_state, h, a, b, B, C, z, D, state, y,
                                        dtype, nullptr, nullptr, nullptr,
                                        static_cast<cudaStream_t>(stream)));
}

naju_status naju_conv_silu_step(int64_t batch, int64_t d_inner, int32_t dtype, const void* u,
                                const float* conv_w, const float* conv_b, float* conv_state,
                                void* h, void* stream) {
    if (batch < 1 || d_inner < 1 || batch > (1 << 20) || d_inner > (1 << 20))
        return NAJU_ERR_INVALID_ARG;
    if (dtype != NAJU_F32 && dtype != NAJU_BF16) return NAJU_ERR_UNSUPPORTED;
    NAJU_REQUIRE(ok_act(u) && ok_act(h) && conv_w && ok_act(conv_state) && ok_opt(conv_b));
    return cuda_status(launch_conv_step(batch, d_inner, u, conv_w, conv_b, conv_state, h, dtype,
                                        static_cast<cudaStream_t>(stream)));
}

naju_status naju_scan_step_conv(int64_t batch, int64_t d_inner, int64_t d_state, int32_t dtype,
                                const void* u, const float* conv_w, const float* conv_b,
                                float* conv_state, const void* a, const void* b, const void* B,
                                const void* C, const void* z, const float* D, float* state,
                                void* y, void* stream) {
    if (batch < 1 || d_inner < 1 || batch > 65535) return NAJU_ERR_INVALID_ARG;
    if (d_state != 16 && d_state != 32 && d_state != 64 && d_state != 128)
        return NAJU_ERR_UNSUPPORTED;
    if (dtype != NAJU_F32 && dtype != NAJU_BF16) return NAJU_ERR_UNSUPPORTED;
    NAJU_REQUIRE(ok_act(u) && ok_act(a) && ok_opt(b) && ok_act(B) && ok_act(C) && ok_act(y));
    NAJU_REQUIRE(ok_opt(z) && ok_act(state) && conv_w && ok_act(conv_state) && ok_opt(conv_b));
    return cuda_status(launch_scan_step(batch, d_inner, d_state, u, a, b, B, C, z, D, state, y,
                                        dtype, conv_w, conv_b, conv_state,
                                        static_cast<cudaStream_t>(stream)));
}

naju_status naju_last_device_status(void* workspace, void* stream) {
    if (!workspace || !aligned(workspace, 256)) return NAJU_ERR_INVALID_ARG;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (cudaStreamSynchronize(s) != cudaSuccess) return NAJU_ERR_CUDA;
    int v = 0;
    WsHeader* hdr = static_cast<WsHeader*>(workspace);
    if (cudaMemcpy(&v, &hdr->status, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess)
        return NAJU_ERR_CUDA;
    if (cudaMemset(&hdr->status, 0, sizeof(int)) != cudaSuccess) return NAJU_ERR_CUDA;
    if (v & (1 << NAJU_ERR_TIMEOUT)) return NAJU_ERR_TIMEOUT;
    return NAJU_OK;
}

const char* naju_status_string(naju_status s) {
    switch (s) {
        case NAJU_OK: return "ok";
        case NAJU_ERR_INVALID_ARG: return "invalid argument";
        case NAJU_ERR_UNSUPPORTED: return "unsupported configuration";
        case NAJU_ERR_CUDA: return "CUDA error";
        case NAJU_ERR_TIMEOUT: return "inter-block wait timed out";
    }
    return "unknown status";
}

void naju_testing_set_wait_limit(int64_t polls) {
    g_wait_limit = polls > 0 ? (long long)polls : kDefaultWait;
}
void naju_testing_set_skip_publish(int32_t skip) { g_skip_publish = skip ? 1 : 0; }
void naju_testing_set_fwd_groups(int32_t groups) { g_fwd_groups = groups > 0 ? groups : 0; }
void naju_testing_set_bwd_groups(int32_t groups) { g_bwd_groups = groups > 0 ? groups : 0; }
void naju_testing_set_bwd_pieces(int32_t pieces) { g_bwd_pieces = pieces; }
void naju_testing_set_fwd_pieces(int32_t pieces) { g_fwd_pieces = pieces; }
int32_t naju_testing_fwd_pieces(const void* dims) {
    const naju_dims* dm = static_cast<const naju_dims*>(dims);
    if (check_dims(dm) != NAJU_OK) return 0;
    return layout(dm).npieces_f;
}
int32_t naju_testing_bwd_pieces(const void* dims) {
    const naju_dims* dm = static_cast<const naju_dims*>(dims);
    if (check_dims(dm) != NAJU_OK) return 0;
    return layout(dm).npieces;
}
void naju_testing_set_sm_count(int32_t sms) { g_sm_override = sms > 0 ? sms : 0; }
int32_t naju_testing_sm_count(void) { return sm_count(); }
void naju_testing_set_fwd_impl(int32_t impl) {
    g_fwd_impl = (impl >= 1 && impl <= 3) ? impl : 0;
}
void naju_testing_set_bwd_impl(int32_t impl) {
    g_bwd_impl = (impl >= 1 && impl <= 3) ? impl : 0;
}
int32_t naju_testing_bwd_impl(const void* dims) {
    const naju_dims* dm = static_cast<const naju_dims*>(dims);
    if (check_dims(dm) != NAJU_OK) return 0;
    if (!use_bwd_tc(dm)) return 1;
    return use_bwd_blk(dm) ? 3 : 2;
}
int32_t naju_testing_fwd_impl(const void* dims) {
    const naju_dims* dm = static_cast<const naju_dims*>(dims);
    if (check_dims(dm) != NAJU_OK) return 0;
    if (!use_fwd_tc(dm)) return 1;
    return use_fwd_blk(dm) ? 3 : 2;
}
int32_t naju_testing_bwd_groups(const void* dims) {
    const naju_dims* dm = static_cast<const naju_dims*>(dims);
    if (check_dims(dm) != NAJU_OK) return 0;
    return layout(dm).bgroups;
}
int32_t naju_testing_fwd_groups(const void* dims) {
    const naju_dims* dm = static_cast<const naju_dims*>(dims);
    if (check_dims(dm) != NAJU_OK) return 0;
    return layout(dm).ngroups;
}

}  // extern "C"
