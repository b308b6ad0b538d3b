// moe_dispatch_noalloc: the capacity-bounded dispatch (histogram -> scan ->
// stable scatter + row gather) for callers that cannot allocate device memory.
//
// Who needs it: code that runs where cudaMalloc is not available or not
// allowed -- a plugin or custom op inside a host framework that owns every
// device allocation and hands the plugin only its input and output buffers;
// a real-time loop that forbids allocation after start-up; code that must
// not trigger the implicit synchronisation a cudaMalloc/cudaFree can cause.
// Such a caller cannot provide the workspace that moe_dispatch needs for its
// per-chunk histograms and rank bases.  This entry point keeps that scratch
// in a fixed-size array in the library's own device memory instead
// (`g_dispatch_scratch`, 632 KiB on every GPU that loads the library, held
// until the process exits).
//
// Limits and rules:
//   - ceil(T / 32) * E must not exceed 131072 (for E = 64: T <= 65536 tokens);
//     larger shapes return MOE_ERR_UNSUPPORTED before anything is launched.
//   - The first call on each device looks up the array's device address
//     (cudaGetSymbolAddress) with that device current; make that first call
//     before any stream capture.
//   - Every call on a device shares the one array, which keeps what the last
//     call wrote.  Nothing in it has to start at zero: each call clears the
//     per-group counts it adds into (a cudaMemsetAsync on the array, no
//     allocation) and writes every other entry it later reads.  Calls that
//     overlap on the GPU -- two streams, or two host threads -- race on it and
//     give wrong results.  Serialise them.
//   - No cudaMalloc, cudaFree or allocating library routine is called.
#include <mutex>

#include "internal.h"
#include "moe.h"

namespace {

constexpr int64_t kNoAllocMaxEntries = 131072;  // ceil(T/32) * E
constexpr int kMaxDevices = 64;

// [0, kNoAllocMaxEntries): per-chunk expert histogram; then per-group expert
// counts and per-group rank bases, moe::kMaxGroupEntries each.
constexpr int64_t kScratchEntries = kNoAllocMaxEntries + 2 * (int64_t)moe::kMaxGroupEntries;
static __device__ __align__(256) int32_t g_dispatch_scratch[kScratchEntries];

std::mutex g_setup_mutex;
int32_t* g_scratch_on_device[kMaxDevices] = {nullptr};

// Device address of g_dispatch_scratch for the current device (the host-side
// name is only a stand-in and must never be passed to a kernel).
moe_status_t scratch_address(int32_t** out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return MOE_ERR_CUDA;
    if (dev < 0 || dev >= kMaxDevices) return MOE_ERR_UNSUPPORTED;
    std::lock_guard<std::mutex> lock(g_setup_mutex);
    if (g_scratch_on_device[dev] == nullptr) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_dispatch_scratch) != cudaSuccess || p == nullptr) return MOE_ERR_CUDA;
        g_scratch_on_device[dev] = static_cast<int32_t*>(p);
    }
    *out = g_scratch_on_device[dev];
    return MOE_OK;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

}  // namespace

extern "C" moe_status_t moe_dispatch_noalloc(const moe_config_t* cfg, const void* x, const int32_t* topk_idx,
                                             int32_t* counts, int32_t* offsets, int32_t* slot, int32_t* src_assign,
                                             void* x_perm, cudaStream_t stream) {
    size_t ws_bytes = 0;
    moe_status_t st = moe_workspace_size(cfg, &ws_bytes);  // validates the config
    if (st != MOE_OK) return st;
    if (counts == nullptr || offsets == nullptr) return MOE_ERR_INVALID_ARG;
    if (cfg->T > 0 && (x == nullptr || topk_idx == nullptr || slot == nullptr || src_assign == nullptr ||
                       x_perm == nullptr || !aligned16(x) || !aligned16(x_perm)))
        return MOE_ERR_INVALID_ARG;
    const int64_t nchunk = (cfg->T + moe::kChunkTokens - 1) / moe::kChunkTokens;
    if (nchunk * cfg->E > kNoAllocMaxEntries) return MOE_ERR_UNSUPPORTED;
    int64_t cap = 0;
    if ((st = moe_capacity(cfg, &cap)) != MOE_OK) return st;
    if (cap > cfg->T) cap = cfg->T;

    int32_t* scratch = nullptr;
    if ((st = scratch_address(&scratch)) != MOE_OK) return st;
    int32_t* hist = scratch;
    int32_t* group_hist = scratch + kNoAllocMaxEntries;
    int32_t* group_base = group_hist + moe::kMaxGroupEntries;
    const int group_chunks = moe::group_chunks_for(cfg->E, nchunk);
    const int ngroups = moe::ngroups_for(cfg->E, nchunk);

    if (cudaMemsetAsync(group_hist, 0, (size_t)ngroups * cfg->E * sizeof(int32_t), stream) != cudaSuccess)
        return MOE_ERR_CUDA;
    if (moe::launch_dispatch_hist(topk_idx, hist, group_hist, cfg->T, cfg->E, cfg->k, group_chunks, ngroups, stream) !=
        cudaSuccess)
        return MOE_ERR_CUDA;
    moe::ScanArgs sa;
    sa.group_hist = group_hist;
    sa.psum = nullptr;
    sa.group_base = group_base;
    sa.counts = counts;
    sa.offsets = offsets;
    sa.f = nullptr;
    sa.p = nullptr;
    sa.l_aux = nullptr;
    sa.psum_total = nullptr;
    sa.T = cfg->T;
    sa.ngroups = ngroups;
    sa.npsum = 0;
    sa.E = cfg->E;
    sa.k = cfg->k;
    sa.cap = (int)cap;
    sa.alpha = cfg->aux_alpha;
    if (moe::launch_dispatch_scan(sa, stream) != cudaSuccess) return MOE_ERR_CUDA;
    moe::ScatterArgs xa;
    xa.topk_idx = topk_idx;
    xa.hist = hist;
    xa.group_base = group_base;
    xa.group_chunks = group_chunks;
    xa.ngroups = ngroups;
    xa.offsets = offsets;
    xa.slot = slot;
    xa.src_assign = src_assign;
    xa.x = x;
    xa.x_perm = x_perm;
    xa.cap_e = nullptr;
    xa.T = cfg->T;
    xa.E = cfg->E;
    xa.k = cfg->k;
    xa.cap = (int)cap;
    xa.nchunk = (int)nchunk;
    xa.row_bytes = (int)(cfg->d * (cfg->dtype == MOE_DT_BF16 ? 2 : 4));
    if (moe::launch_dispatch_scatter(xa, stream) != cudaSuccess) return MOE_ERR_CUDA;
    return MOE_OK;
}
