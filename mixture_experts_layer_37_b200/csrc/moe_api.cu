// libmoe C ABI: argument validation, capacity and workspace planning, and the
// kernel launch sequence of the MoE layer forward.  No allocation, no host
// synchronisation (except moe_check_device_status), no CPU fallback.
#include <math.h>
#include <string.h>

#include <nvtx3/nvToolsExt.h>

#include "internal.h"
#include "moe.h"

namespace moe {

int sm_count() {
    static std::atomic<int> cached[64];  // per device, 0 until queried
    int dev = 0;
    cudaGetDevice(&dev);
    int n = dev < 64 ? cached[dev].load(std::memory_order_relaxed) : 0;
    if (n == 0) {
        cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
        if (n <= 0) n = 1;
        if (dev < 64) cached[dev].store(n, std::memory_order_relaxed);
    }
    return n;
}

namespace {
thread_local bool t_pdl = false;
}
bool pdl_enabled() { return t_pdl; }
PdlScope::PdlScope() : prev(t_pdl) { t_pdl = true; }
PdlScope::~PdlScope() { t_pdl = prev; }

}  // namespace moe

namespace {

using namespace moe;

uint32_t g_timeout_ms = 2000;

constexpr size_t kStatusBytes = kStatusBlockBytes;
constexpr int kMaxShared = 8;

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }
size_t elem_size(const moe_config_t* c) { return c->dtype == MOE_DT_BF16 ? 2 : 4; }

moe_status_t check_config(const moe_config_t* c) {
    if (c == nullptr) return MOE_ERR_INVALID_ARG;
    if (c->T < 0 || c->d <= 0 || c->ffn <= 0 || c->E <= 0 || c->k <= 0) return MOE_ERR_INVALID_ARG;
    if (c->k > c->E) return MOE_ERR_INVALID_ARG;
    if (c->dtype != MOE_DT_F32 && c->dtype != MOE_DT_BF16) return MOE_ERR_INVALID_ARG;
    if (c->act != MOE_ACT_SWIGLU && c->act != MOE_ACT_GELU_BIAS) return MOE_ERR_INVALID_ARG;
    if (isnan(c->capacity_factor) || isnan(c->aux_alpha) || c->router_kernel < MOE_ROUTER_AUTO ||
        c->router_kernel > MOE_ROUTER_WARP_MMA_STAGED || c->gemm_kernel < MOE_GEMM_AUTO || c->gemm_kernel > MOE_GEMM_CTA_PAIR ||
        c->dispatch < MOE_DISPATCH_AUTO || c->dispatch > MOE_DISPATCH_GATHER || c->n_shared < 0 ||
        c->weight_format < MOE_WEIGHTS_NATIVE || c->weight_format > MOE_WEIGHTS_INT8 ||
        c->weighting < MOE_WEIGHTING_AUTO || c->weighting > MOE_WEIGHTING_EPILOGUE)
        return MOE_ERR_INVALID_ARG;
    if (c->n_shared > kMaxShared) return MOE_ERR_UNSUPPORTED;
    if (c->weight_format == MOE_WEIGHTS_INT8 && c->dtype != MOE_DT_BF16) return MOE_ERR_UNSUPPORTED;
    if (c->router_kernel == MOE_ROUTER_TCGEN05 &&
        (c->dtype != MOE_DT_BF16 || c->E % 8 != 0 || c->d % 64 != 0))
        return MOE_ERR_UNSUPPORTED;
    if (c->E > kMaxExperts || c->k > kMaxTopK) return MOE_ERR_UNSUPPORTED;
    if (c->T * (int64_t)c->k >= ((int64_t)1 << 31)) return MOE_ERR_UNSUPPORTED;
    if (c->dtype == MOE_DT_BF16) {
        if (c->d % 64 != 0 || c->ffn % 64 != 0) return MOE_ERR_UNSUPPORTED;
        if ((int64_t)c->E * c->d >= ((int64_t)1 << 31) || (int64_t)c->E * c->ffn >= ((int64_t)1 << 31))
            return MOE_ERR_UNSUPPORTED;
    } else {
        if (c->d % 4 != 0 || c->ffn % 4 != 0) return MOE_ERR_UNSUPPORTED;
    }
    return MOE_OK;
}

// Formula value of the capacity (may exceed T) and the clamped value the
// kernels use (an expert can receive at most T assignments).
int64_t capacity_formula(const moe_config_t* c) {
    if (!(c->capacity_factor > 0.0)) return c->T;
    const double v = ceil(((double)c->T * (double)c->k / (double)c->E) * c->capacity_factor);
    if (v >= 9.0e18) return INT64_MAX;
    return (int64_t)v;
}
int64_t capacity_used(const moe_config_t* c) {
    const int64_t cap = capacity_formula(c);
    return cap < c->T ? cap : c->T;
}
int64_t max_rows(const moe_config_t* c) {
    const int64_t cap = capacity_used(c);
    const int64_t a = c->T * c->k, b = (int64_t)c->E * cap;
    return a < b ? a : b;
}

struct Plan {
    int nchunk, group_chunks, ngroups, psum_cols;
    int64_t rows;
    size_t hist, psum, gbase, cap_e, shared_off, ep_dest, xperm, h, yperm, hs, ys, total;
};

// perm_buffers = false: no x_perm / y_perm (the expert-parallel calls use the
// caller's receive buffers instead).
Plan plan_rows(const moe_config_t* c, int64_t rows, bool perm_buffers = true) {
    Plan p;
    p.nchunk = (int)((c->T + kChunkTokens - 1) / kChunkTokens);
    p.group_chunks = group_chunks_for(c->E, p.nchunk);
    p.ngroups = ngroups_for(c->E, p.nchunk);
    // probability sums per chunk, or per CTA of the resident-weight router
    p.psum_cols = p.nchunk > router_v2_psum_columns() ? p.nchunk : router_v2_psum_columns();
    p.rows = rows;
    const size_t s = elem_size(c);
    const size_t E = (size_t)c->E;
    size_t off = kStatusBytes;
    p.hist = off;
    off = align_up(off + (size_t)p.nchunk * E * 4, 1024);
    p.psum = off;
    off = align_up(off + (size_t)p.psum_cols * E * 8, 1024);
    p.gbase = off;
    off = align_up(off + (size_t)p.ngroups * E * 4, 1024);
    p.cap_e = off;
    off = align_up(off + E * 4, 1024);
    p.shared_off = off;
    off = align_up(off + 2 * 4, 1024);
    p.ep_dest = off;
    off = align_up(off + E * 4, 1024);
    const size_t perm_rows = perm_buffers ? (size_t)p.rows : 0;
    p.xperm = off;
    off = align_up(off + perm_rows * c->d * s, 1024);
    p.h = off;
    off = align_up(off + (size_t)p.rows * c->ffn * s, 1024);
    p.yperm = off;
    off = align_up(off + perm_rows * c->d * s, 1024);
    // shared experts: one [T, ffn] intermediate reused in turn, and each one's [T, d] output
    p.hs = off;
    off = align_up(off + (c->n_shared > 0 ? (size_t)c->T * c->ffn * s : 0), 1024);
    p.ys = off;
    off = align_up(off + (size_t)c->n_shared * c->T * c->d * s, 1024);
    p.total = off;
    return p;
}

Plan plan_of(const moe_config_t* c) { return plan_rows(c, max_rows(c)); }

// Data-parallel shard of a batch of T_global tokens: capacity of the whole
// batch, and the most rows this shard can keep.
int64_t dp_cap_used(const moe_config_t* c, int64_t T_global) {
    moe_config_t g = *c;
    g.T = T_global;
    const int64_t cap = capacity_formula(&g);
    return cap < T_global ? cap : T_global;
}
int64_t dp_rows(const moe_config_t* c, int64_t T_global) {
    int64_t cap = dp_cap_used(c, T_global);
    if (cap > c->T) cap = c->T;
    const int64_t a = c->T * c->k, b = (int64_t)c->E * cap;
    return a < b ? a : b;
}
moe_status_t check_dp(const moe_config_t* c, int64_t T_global) {
    if (T_global < c->T) return MOE_ERR_INVALID_ARG;
    if (T_global * (int64_t)c->k >= ((int64_t)1 << 31)) return MOE_ERR_UNSUPPORTED;
    return MOE_OK;
}

// Expert-parallel shard over `world` ranks: rows of every receive buffer
// (the most rows E/world experts can keep of the whole batch).
int64_t ep_recv_rows(const moe_config_t* c, int64_t T_global, int world) {
    const int64_t cap = dp_cap_used(c, T_global);
    const int64_t a = T_global * c->k, b = (int64_t)(c->E / world) * cap;
    return a < b ? a : b;
}
moe_status_t check_ep(const moe_config_t* c, int64_t T_global, int world) {
    moe_status_t st = check_dp(c, T_global);
    if (st != MOE_OK) return st;
    if (world < 1 || c->E % world != 0) return MOE_ERR_INVALID_ARG;
    if (world > kMaxRanks) return MOE_ERR_UNSUPPORTED;
    return MOE_OK;
}
Plan plan_ep(const moe_config_t* c, int64_t T_global, int world) {
    return plan_rows(c, ep_recv_rows(c, T_global, world), false);
}

moe_status_t check_ws_plan(const Plan& pl, const void* ws, size_t ws_bytes) {
    if (ws == nullptr || ws_bytes < pl.total) return MOE_ERR_WORKSPACE;
    if ((reinterpret_cast<uintptr_t>(ws) & 1023u) != 0) return MOE_ERR_INVALID_ARG;
    return MOE_OK;
}

moe_status_t check_ws(const moe_config_t* c, const void* ws, size_t ws_bytes, Plan* p) {
    *p = plan_of(c);
    if (ws == nullptr || ws_bytes < p->total) return MOE_ERR_WORKSPACE;
    if ((reinterpret_cast<uintptr_t>(ws) & 1023u) != 0) return MOE_ERR_INVALID_ARG;
    return MOE_OK;
}

DevStatus status_of(void* ws) {
    DevStatus st;
    st.word = static_cast<uint32_t*>(ws);
    st.timeout_ns = (uint64_t)g_timeout_ms * 1000000ull;
    return st;
}

uint8_t* at(void* ws, size_t off) { return static_cast<uint8_t*>(ws) + off; }

// A named NVTX range over the host-side launches of one stage, for profilers
// (for example `ncu --nvtx --nvtx-include "moe_forward/"`); without an
// attached tool each call returns at once.
struct NvtxRange {
    explicit NvtxRange(const char* name) { nvtxRangePushA(name); }
    ~NvtxRange() { nvtxRangePop(); }
    NvtxRange(const NvtxRange&) = delete;
    NvtxRange& operator=(const NvtxRange&) = delete;
};

moe_status_t from_cuda(cudaError_t e) { return e == cudaSuccess ? MOE_OK : MOE_ERR_CUDA; }

moe_status_t check_weights(const moe_config_t* c, const moe_weights_t* w, bool need_router, bool need_experts) {
    if (w == nullptr) return MOE_ERR_INVALID_ARG;
    if (need_router && (w->w_router == nullptr || !aligned16(w->w_router))) return MOE_ERR_INVALID_ARG;
    if (need_experts) {
        if (w->w_gate_or_w1 == nullptr || w->w_down_or_w2 == nullptr) return MOE_ERR_INVALID_ARG;
        if (!aligned16(w->w_gate_or_w1) || !aligned16(w->w_down_or_w2)) return MOE_ERR_INVALID_ARG;
        if (c->act == MOE_ACT_SWIGLU) {
            if (w->w_up == nullptr || !aligned16(w->w_up)) return MOE_ERR_INVALID_ARG;
        } else {
            if (w->b1 == nullptr || w->b2 == nullptr || !aligned16(w->b1) || !aligned16(w->b2))
                return MOE_ERR_INVALID_ARG;
        }
        if (c->weight_format == MOE_WEIGHTS_INT8 &&
            (w->gate_or_w1_scale == nullptr || w->down_or_w2_scale == nullptr ||
             (c->act == MOE_ACT_SWIGLU && w->up_scale == nullptr)))
            return MOE_ERR_INVALID_ARG;
        if (c->n_shared > 0) {
            if (w->shared_gate_or_w1 == nullptr || w->shared_down_or_w2 == nullptr ||
                !aligned16(w->shared_gate_or_w1) || !aligned16(w->shared_down_or_w2))
                return MOE_ERR_INVALID_ARG;
            if (c->act == MOE_ACT_SWIGLU) {
                if (w->shared_up == nullptr || !aligned16(w->shared_up)) return MOE_ERR_INVALID_ARG;
            } else if (w->shared_b1 == nullptr || w->shared_b2 == nullptr || !aligned16(w->shared_b1) ||
                       !aligned16(w->shared_b2)) {
                return MOE_ERR_INVALID_ARG;
            }
        }
    }
    return MOE_OK;
}

ScanArgs scan_args(const moe_config_t* c, int32_t* counts, int32_t* offsets, float* f, float* p, float* l_aux,
                   bool with_stats, void* ws, const Plan& pl) {
    ScanArgs sa;
    sa.group_hist = reinterpret_cast<int32_t*>(at(ws, kGroupHistOffset));
    sa.psum = with_stats ? reinterpret_cast<const double*>(at(ws, pl.psum)) : nullptr;
    sa.group_base = reinterpret_cast<int32_t*>(at(ws, pl.gbase));
    sa.counts = counts;
    sa.offsets = offsets;
    sa.f = f;
    sa.p = p;
    sa.l_aux = l_aux;
    sa.psum_total = nullptr;
    sa.real_counter = nullptr;
    sa.shared_off = c->n_shared > 0 ? reinterpret_cast<int32_t*>(at(ws, pl.shared_off)) : nullptr;
    sa.T = c->T;
    sa.ngroups = pl.ngroups;
    sa.npsum = pl.nchunk;
    sa.E = c->E;
    sa.k = c->k;
    sa.cap = (int)capacity_used(c);
    sa.alpha = c->aux_alpha;
    return sa;
}

// Router; with `fused` set, its last CTA also runs the scan described by `sa`.
moe_status_t run_router(const moe_config_t* c, const void* x, const void* w_router, const float* bias,
                        const float* logits_in, const uint8_t* mask, int32_t* idx, float* w, float* logits_out,
                        float* probs_out, void* ws, const Plan& pl, cudaStream_t s, const ScanArgs* fused = nullptr) {
    // the tensor-core router is a GEMM kernel: with fed logits there is no GEMM
    // for it to run, and silently running the warp router instead would hide
    // which kernel produced the routing
    if (logits_in != nullptr && c->router_kernel == MOE_ROUTER_TCGEN05) return MOE_ERR_UNSUPPORTED;
    RouterArgs a;
    a.x = x;
    a.w_router = w_router;
    a.bias = bias;
    a.logits_in = logits_in;
    a.topk_idx = idx;
    a.topk_w = w;
    a.logits_out = logits_out;
    a.probs_out = probs_out;
    a.hist = reinterpret_cast<int32_t*>(at(ws, pl.hist));
    a.psum = reinterpret_cast<double*>(at(ws, pl.psum));
    a.mask = mask;
    a.T = c->T;
    a.d = c->d;
    a.E = c->E;
    a.k = c->k;
    a.nchunk = pl.nchunk;
    a.group_chunks = pl.group_chunks;
    a.ngroups = pl.ngroups;
    a.psum_cap = pl.psum_cols;
    a.fuse_scan = fused != nullptr ? 1 : 0;
    a.counter = static_cast<unsigned int*>(ws) + kStatusCounterWord;
    if (fused != nullptr) {
        // counters that only a fused scan reads and returns to zero
        a.group_hist = reinterpret_cast<int32_t*>(at(ws, kGroupHistOffset));
        a.scan = *fused;
        if (mask != nullptr) {
            a.real_counter = static_cast<int32_t*>(ws) + kStatusRealWord;
            a.scan.real_counter = a.real_counter;  // statistics over the real tokens
        }
    }
    a.st = status_of(ws);
    a.kernel = c->router_kernel;
    return from_cuda(launch_router(a, c->dtype == MOE_DT_BF16, s));
}

moe_status_t run_scatter(const moe_config_t* c, const void* x, const int32_t* idx, const int32_t* offsets,
                         int32_t* slot, int32_t* src_assign, void* x_perm, void* ws, const Plan& pl, cudaStream_t s,
                         const int32_t* cap_e = nullptr) {
    ScatterArgs xa;
    xa.topk_idx = idx;
    xa.hist = reinterpret_cast<const int32_t*>(at(ws, pl.hist));
    xa.group_base = reinterpret_cast<const int32_t*>(at(ws, pl.gbase));
    xa.group_chunks = pl.group_chunks;
    xa.ngroups = pl.ngroups;
    xa.offsets = offsets;
    xa.slot = slot;
    xa.src_assign = src_assign;
    xa.x = x;
    xa.x_perm = x_perm;
    xa.cap_e = cap_e;
    xa.T = c->T;
    xa.E = c->E;
    xa.k = c->k;
    xa.cap = (int)capacity_used(c);
    xa.nchunk = pl.nchunk;
    xa.row_bytes = (int)(c->d * elem_size(c));
    return from_cuda(launch_dispatch_scatter(xa, s));
}

// Whether moe_forward / moe_dp_finish gather the first GEMM's rows from x
// (on request only: the copy is faster end to end on B200; never with INT8 weights).
bool gathers(const moe_config_t* c) {
    return c->dtype == MOE_DT_BF16 && c->dispatch == MOE_DISPATCH_GATHER && c->weight_format == MOE_WEIGHTS_NATIVE;
}

// Whether moe_forward / moe_dp_finish weight the expert rows in the second
// GEMM's epilogue (then the combine is a plain sum of the k rows).
bool weights_in_epilogue(const moe_config_t* c) {
    return c->dtype == MOE_DT_BF16 && c->weight_format == MOE_WEIGHTS_NATIVE && c->weighting != MOE_WEIGHTING_COMBINE;
}

moe_status_t run_ffn(const moe_config_t* c, const moe_weights_t* w, const void* x_perm, const int32_t* offsets,
                     void* y_perm, void* ws, const Plan& pl, cudaStream_t s, cudaEvent_t between = nullptr,
                     const void* gather_x = nullptr, const int32_t* src_assign = nullptr,
                     const float* row_w = nullptr) {
    FfnArgs f;
    f.act = c->act;
    f.E = c->E;
    f.d = c->d;
    f.ffn = c->ffn;
    f.rows_cap = pl.rows;
    f.offsets = offsets;
    f.x_perm = x_perm;
    f.h = at(ws, pl.h);
    f.y_perm = y_perm;
    f.w1 = w->w_gate_or_w1;
    f.w_up = w->w_up;
    f.w2 = w->w_down_or_w2;
    f.b1 = w->b1;
    f.b2 = w->b2;
    f.st = status_of(ws);
    f.between = between;
    f.gemm_kernel = c->gemm_kernel;
    f.gather_x = gather_x;
    f.src_assign = src_assign;
    f.gather_rows = c->T;
    f.k = c->k;
    f.row_w = row_w;
    if ((row_w != nullptr || gather_x != nullptr) && src_assign == nullptr) return MOE_ERR_INVALID_ARG;
    if (row_w != nullptr && !weights_in_epilogue(c)) return MOE_ERR_INVALID_ARG;
    if (c->weight_format == MOE_WEIGHTS_INT8) {
        // INT8 routed experts: rows always come from the sorted copy
        if (x_perm == nullptr) return MOE_ERR_INVALID_ARG;
        f.int8 = true;
        f.gather_x = nullptr;
        f.w1_scale = w->gate_or_w1_scale;
        f.w_up_scale = w->up_scale;
        f.w2_scale = w->down_or_w2_scale;
        return from_cuda(launch_ffn_int8(f, s));
    }
    return from_cuda(c->dtype == MOE_DT_BF16 ? launch_ffn_bf16_sm100(f, s) : launch_ffn_f32(f, s));
}

moe_status_t run_combine(const moe_config_t* c, const void* y_perm, const int32_t* slot, const float* w, void* out,
                         cudaStream_t s, const void* y_shared = nullptr) {
    CombineArgs a;
    a.y_perm = y_perm;
    a.slot = slot;
    a.topk_w = w;
    a.out = out;
    a.y_shared = y_shared;
    a.n_shared = y_shared != nullptr ? c->n_shared : 0;
    a.T = c->T;
    a.d = c->d;
    a.k = c->k;
    return from_cuda(launch_combine(a, c->dtype == MOE_DT_BF16, s));
}

// The shared experts (LLaMA4-MoE §5.2): each one's two GEMMs over all T token
// rows (one group of T rows, offsets {0, T} written by the scan), its output in
// ys[s].  `mark` records the stage events of moe_forward_profiled.
template <class Mark>
moe_status_t run_shared(const moe_config_t* c, const moe_weights_t* w, const void* x, void* ws, const Plan& pl,
                        cudaStream_t s, Mark&& mark, cudaEvent_t* ev, int* n) {
    const size_t es = elem_size(c);
    const size_t wsz = (size_t)c->d * c->ffn * es;
    for (int i = 0; i < c->n_shared; ++i) {
        FfnArgs f;
        f.act = c->act;
        f.E = 1;
        f.d = c->d;
        f.ffn = c->ffn;
        f.rows_cap = c->T;
        f.offsets = reinterpret_cast<const int32_t*>(at(ws, pl.shared_off));
        f.x_perm = x;
        f.h = at(ws, pl.hs);
        f.y_perm = at(ws, pl.ys + (size_t)i * c->T * c->d * es);
        f.w1 = static_cast<const uint8_t*>(w->shared_gate_or_w1) + i * wsz;
        f.w_up = w->shared_up != nullptr ? static_cast<const uint8_t*>(w->shared_up) + i * wsz : nullptr;
        f.w2 = static_cast<const uint8_t*>(w->shared_down_or_w2) + i * wsz;
        f.b1 = w->shared_b1 != nullptr ? static_cast<const uint8_t*>(w->shared_b1) + (size_t)i * c->ffn * es : nullptr;
        f.b2 = w->shared_b2 != nullptr ? static_cast<const uint8_t*>(w->shared_b2) + (size_t)i * c->d * es : nullptr;
        f.st = status_of(ws);
        f.between = ev != nullptr ? ev[(*n)++] : nullptr;
        f.gemm_kernel = c->gemm_kernel;
        f.gather_x = nullptr;
        f.src_assign = nullptr;
        f.k = 1;
        const cudaError_t e = c->dtype == MOE_DT_BF16 ? launch_ffn_bf16_sm100(f, s) : launch_ffn_f32(f, s);
        if (e != cudaSuccess) return MOE_ERR_CUDA;
        if (!mark()) return MOE_ERR_CUDA;
    }
    return MOE_OK;
}

}  // namespace

extern "C" {

const char* moe_status_string(moe_status_t status) {
    switch (status) {
        case MOE_OK: return "MOE_OK";
        case MOE_ERR_INVALID_ARG: return "MOE_ERR_INVALID_ARG: null, misaligned or out-of-range argument";
        case MOE_ERR_UNSUPPORTED: return "MOE_ERR_UNSUPPORTED: shape outside what this build runs";
        case MOE_ERR_WORKSPACE: return "MOE_ERR_WORKSPACE: workspace missing or smaller than moe_workspace_size";
        case MOE_ERR_CUDA: return "MOE_ERR_CUDA: a CUDA call or kernel launch failed";
        case MOE_ERR_TIMEOUT: return "MOE_ERR_TIMEOUT: a bounded device wait gave up";
        case MOE_ERR_RANGE: return "MOE_ERR_RANGE: a device-side bounds check refused a row (inconsistent counts)";
    }
    return "MOE_ERR_UNKNOWN";
}

moe_status_t moe_capacity(const moe_config_t* cfg, int64_t* cap) {
    moe_status_t st = check_config(cfg);
    if (st != MOE_OK) return st;
    if (cap == nullptr) return MOE_ERR_INVALID_ARG;
    *cap = capacity_formula(cfg);
    return MOE_OK;
}

moe_status_t moe_max_rows(const moe_config_t* cfg, int64_t* rows) {
    moe_status_t st = check_config(cfg);
    if (st != MOE_OK) return st;
    if (rows == nullptr) return MOE_ERR_INVALID_ARG;
    *rows = max_rows(cfg);
    return MOE_OK;
}

moe_status_t moe_workspace_size(const moe_config_t* cfg, size_t* bytes) {
    moe_status_t st = check_config(cfg);
    if (st != MOE_OK) return st;
    if (bytes == nullptr) return MOE_ERR_INVALID_ARG;
    *bytes = plan_of(cfg).total;
    return MOE_OK;
}

moe_status_t moe_workspace_init(void* ws, size_t ws_bytes, cudaStream_t stream) {
    if (ws == nullptr || ws_bytes < kStatusBytes) return MOE_ERR_WORKSPACE;
    return from_cuda(cudaMemsetAsync(ws, 0, kStatusBytes, stream));
}

moe_status_t moe_router_topk(const moe_config_t* cfg, const void* x, const void* w_router, const float* logit_bias,
                             const float* logits_in, const uint8_t* token_mask, int32_t* topk_idx, float* topk_w,
                             float* logits_out, float* probs_out, void* ws, size_t ws_bytes, cudaStream_t stream) {
    moe_status_t st = check_config(cfg);
    if (st != MOE_OK) return st;
    if (topk_idx == nullptr || topk_w == nullptr) return MOE_ERR_INVALID_ARG;
    if (logits_in == nullptr) {
        if (x == nullptr || w_router == nullptr || !aligned16(x) || !aligned16(w_router)) return MOE_ERR_INVALID_ARG;
    }
    Plan pl;
    if ((st = check_ws(cfg, ws, ws_bytes, &pl)) != MOE_OK) return st;
    if (cfg->T == 0) return MOE_OK;
    return run_router(cfg, x, w_router, logit_bias, logits_in, token_mask, topk_idx, topk_w, logits_out, probs_out, ws,
                      pl, stream);
}

moe_status_t moe_quantize_int8(const moe_config_t* cfg, const void* w, int64_t K, int64_t N, int8_t* q, float* scale,
                               cudaStream_t stream) {
    moe_status_t st = check_config(cfg);
    if (st != MOE_OK) return st;
    if (K <= 0 || N <= 0 || N % 4 != 0) return MOE_ERR_INVALID_ARG;
    if (w == nullptr || q == nullptr || scale == nullptr) return MOE_ERR_INVALID_ARG;
    return from_cuda(launch_quantize_int8(w, cfg->dtype == MOE_DT_BF16, cfg->E, K, N, q, scale, stream));
}

moe_status_t moe_dispatch(const moe_config_t* cfg, const void* x, const int32_t* topk_idx, int32_t* counts,
                          int32_t* offsets, int32_t* slot, int32_t* src_assign, void* x_perm, void* ws,
                          size_t ws_bytes, cudaStream_t stream) {
    moe_status_t st = check_config(cfg);
    if (st != MOE_OK) return st;
    if (counts == nullptr || offsets == nullptr) return MOE_ERR_INVALID_ARG;
    if (cfg->T > 0 && (x == nullptr || topk_idx == nullptr || slot == nullptr || src_assign == nullptr ||
                       x_perm == nullptr || !aligned16(x) || !aligned16(x_perm)))
        return MOE_ERR_INVALID_ARG;
    Plan pl;
    if ((st = check_ws(cfg, ws, ws_bytes, &pl)) != MOE_OK) return st;
    if (launch_dispatch_hist(topk_idx, reinterpret_cast<int32_t*>(at(ws, pl.hist)),
                             reinterpret_cast<int32_t*>(at(ws, kGroupHistOffset)), cfg->T, cfg->E, cfg->k,
                             pl.group_chunks, pl.ngroups, stream) != cudaSuccess)
        return MOE_ERR_CUDA;
    const ScanArgs sa = scan_args(cfg, counts, offsets, nullptr, nullptr, nullptr, false, ws, pl);
    if (launch_dispatch_scan(sa, stream) != cudaSuccess) return MOE_ERR_CUDA;
    return run_scatter(cfg, x, topk_idx, offsets, slot, src_assign, x_perm, ws, pl, stream);
}

moe_status_t moe_expert_ffn(const moe_config_t* cfg, const moe_weights_t* weights, const void* x_perm,
                            const int32_t* offsets, void* y_perm, void* ws, size_t ws_bytes, cudaStream_t stream) {
    moe_status_t st = check_config(cfg);
    if (st != MOE_OK) return st;
    if ((st = check_weights(cfg, weights, false, true)) != MOE_OK) return st;
    if (offsets == nullptr || x_perm == nullptr || y_perm == nullptr || !aligned16(x_perm) || !aligned16(y_perm))
        return MOE_ERR_INVALID_ARG;
    Plan pl;
    if ((st = check_ws(cfg, ws, ws_bytes, &pl)) != MOE_OK) return st;
    if (pl.rows == 0) return MOE_OK;
    return run_ffn(cfg, weights, x_perm, offsets, y_perm, ws, pl, stream);
}

moe_status_t moe_combine(const moe_config_t* cfg, const void* y_perm, const int32_t* slot, const float* topk_w,
                         void* out, cudaStream_t stream) {
    moe_status_t st = check_config(cfg);
    if (st != MOE_OK) return st;
    if (cfg->T == 0) return MOE_OK;
    if (y_perm == nullptr || slot == nullptr || topk_w == nullptr || out == nullptr || !aligned16(y_perm) ||
        !aligned16(out))
        return MOE_ERR_INVALID_ARG;
    return run_combine(cfg, y_perm, slot, topk_w, out, stream);
}

moe_status_t moe_aux_stats(const moe_config_t* cfg, const int32_t* counts, const float* probs, float* f, float* p,
                           float* l_aux, cudaStream_t stream) {
    moe_status_t st = check_config(cfg);
    if (st != MOE_OK) return st;
    if (counts == nullptr || f == nullptr || p == nullptr || l_aux == nullptr) return MOE_ERR_INVALID_ARG;
    if (cfg->T > 0 && probs == nullptr) return MOE_ERR_INVALID_ARG;
    return from_cuda(launch_aux_from_probs(counts, probs, f, p, l_aux, cfg->T, cfg->E, cfg->k, cfg->aux_alpha, stream));
}

static moe_status_t forward_impl(const moe_config_t* cfg, const moe_weights_t* weights, const void* x,
                                 const float* logits_in, const uint8_t* token_mask, moe_outputs_t* o, void* ws,
                                 size_t ws_bytes, cudaStream_t stream, cudaEvent_t* ev) {
    moe_status_t st = check_config(cfg);
    if (st != MOE_OK) return st;
    if ((st = check_weights(cfg, weights, logits_in == nullptr, true)) != MOE_OK) return st;
    if (o == nullptr || o->counts == nullptr || o->offsets == nullptr || o->f == nullptr || o->p == nullptr ||
        o->l_aux == nullptr)
        return MOE_ERR_INVALID_ARG;
    if (cfg->T > 0 && (x == nullptr || !aligned16(x) || o->out == nullptr || !aligned16(o->out) ||
                       o->topk_idx == nullptr || o->topk_w == nullptr || o->slot == nullptr ||
                       o->src_assign == nullptr))
        return MOE_ERR_INVALID_ARG;
    Plan pl;
    if ((st = check_ws(cfg, ws, ws_bytes, &pl)) != MOE_OK) return st;
    int n = 0;
    auto mark = [&]() -> bool { return ev == nullptr || record_mark(ev[n++], stream) == cudaSuccess; };
    const ScanArgs sa = scan_args(cfg, o->counts, o->offsets, o->f, o->p, o->l_aux, true, ws, pl);
    if (cfg->T == 0) {
        // nothing to route: one launch writes the zero counts, offsets and statistics
        if (!mark()) return MOE_ERR_CUDA;
        if (launch_dispatch_scan(sa, stream) != cudaSuccess) return MOE_ERR_CUDA;
        return mark() ? MOE_OK : MOE_ERR_CUDA;
    }
    void* x_perm = at(ws, pl.xperm);
    void* y_perm = at(ws, pl.yperm);
    const NvtxRange whole("moe_forward");
    if (!mark()) return MOE_ERR_CUDA;
    {
        const NvtxRange r("moe_forward/router");
        st = run_router(cfg, x, weights->w_router, weights->router_logit_bias, logits_in, token_mask, o->topk_idx,
                        o->topk_w, o->logits_out, o->probs_out, ws, pl, stream, &sa);
    }
    if (st != MOE_OK) return st;
    if (!mark()) return MOE_ERR_CUDA;
    const bool gather = gathers(cfg);
    const bool weighted = weights_in_epilogue(cfg);
    // the launches after the router overlap each predecessor's tail (programmatic dependent launch)
    const PdlScope pdl;
    {
        const NvtxRange r("moe_forward/scatter");
        st = run_scatter(cfg, x, o->topk_idx, o->offsets, o->slot, o->src_assign, gather ? nullptr : x_perm, ws, pl,
                         stream);
    }
    if (st != MOE_OK) return st;
    if (!mark()) return MOE_ERR_CUDA;
    {
        const NvtxRange r("moe_forward/expert_ffn");
        st = run_ffn(cfg, weights, x_perm, o->offsets, y_perm, ws, pl, stream, ev ? ev[n++] : nullptr,
                     gather ? x : nullptr, o->src_assign, weighted ? o->topk_w : nullptr);
    }
    if (st != MOE_OK) return st;
    if (!mark()) return MOE_ERR_CUDA;
    {
        const NvtxRange r("moe_forward/shared_experts");
        if ((st = run_shared(cfg, weights, x, ws, pl, stream, mark, ev, &n)) != MOE_OK) return st;
    }
    {
        const NvtxRange r("moe_forward/combine");
        st = run_combine(cfg, y_perm, o->slot, weighted ? nullptr : o->topk_w, o->out, stream,
                         cfg->n_shared > 0 ? at(ws, pl.ys) : nullptr);
    }
    if (st != MOE_OK) return st;
    return mark() ? MOE_OK : MOE_ERR_CUDA;
}

moe_status_t moe_forward(const moe_config_t* cfg, const moe_weights_t* weights, const void* x, const float* logits_in,
                         const uint8_t* token_mask, moe_outputs_t* o, void* ws, size_t ws_bytes, cudaStream_t stream) {
    return forward_impl(cfg, weights, x, logits_in, token_mask, o, ws, ws_bytes, stream, nullptr);
}

moe_status_t moe_forward_profiled(const moe_config_t* cfg, const moe_weights_t* weights, const void* x,
                                  const float* logits_in, const uint8_t* token_mask, moe_outputs_t* o, void* ws,
                                  size_t ws_bytes, cudaStream_t stream, cudaEvent_t* stage_events) {
    if (stage_events == nullptr) return MOE_ERR_INVALID_ARG;
    return forward_impl(cfg, weights, x, logits_in, token_mask, o, ws, ws_bytes, stream, stage_events);
}

moe_status_t moe_dp_workspace_size(const moe_config_t* cfg, int64_t T_global, size_t* bytes) {
    moe_status_t st = check_config(cfg);
    if (st != MOE_OK) return st;
    if ((st = check_dp(cfg, T_global)) != MOE_OK) return st;
    if (bytes == nullptr) return MOE_ERR_INVALID_ARG;
    *bytes = plan_rows(cfg, dp_rows(cfg, T_global)).total;
    return MOE_OK;
}

moe_status_t moe_dp_max_rows(const moe_config_t* cfg, int64_t T_global, int64_t* rows) {
    moe_status_t st = check_config(cfg);
    if (st != MOE_OK) return st;
    if ((st = check_dp(cfg, T_global)) != MOE_OK) return st;
    if (rows == nullptr) return MOE_ERR_INVALID_ARG;
    *rows = dp_rows(cfg, T_global);
    return MOE_OK;
}

}  // extern "C"

namespace {

// Router and top-k of one slice of a sharded batch, with the slice's
// per-expert counts and probability sums (the data- and expert-parallel calls).
moe_status_t route_slice(const moe_config_t* cfg, const moe_weights_t* weights, const void* x, const float* logits_in,
                         const uint8_t* token_mask, moe_outputs_t* o, int32_t* local_counts, double* local_psum,
                         int32_t* local_real, void* ws, size_t ws_bytes, const Plan& pl, cudaStream_t stream) {
    moe_status_t st = check_weights(cfg, weights, logits_in == nullptr, false);
    if (st != MOE_OK) return st;
    if (o == nullptr || o->offsets == nullptr || local_counts == nullptr || local_psum == nullptr)
        return MOE_ERR_INVALID_ARG;
    if (token_mask != nullptr && local_real == nullptr) return MOE_ERR_INVALID_ARG;  // the count must be exchanged
    if (cfg->T > 0 && (x == nullptr || !aligned16(x) || o->topk_idx == nullptr || o->topk_w == nullptr))
        return MOE_ERR_INVALID_ARG;
    if ((st = check_ws_plan(pl, ws, ws_bytes)) != MOE_OK) return st;
    ScanArgs sa = scan_args(cfg, local_counts, o->offsets, nullptr, nullptr, nullptr, true, ws, pl);
    sa.cap = 0x7fffffff;        // local totals only; the capacity is applied by the second phase
    sa.psum_total = local_psum;
    sa.t_real_out = local_real;
    if (cfg->T == 0) return from_cuda(launch_dispatch_scan(sa, stream));
    return run_router(cfg, x, weights->w_router, weights->router_logit_bias, logits_in, token_mask, o->topk_idx,
                      o->topk_w, o->logits_out, o->probs_out, ws, pl, stream, &sa);
}

}  // namespace

extern "C" {

moe_status_t moe_dp_route(const moe_config_t* cfg, int64_t T_global, const moe_weights_t* weights, const void* x,
                          const float* logits_in, const uint8_t* token_mask, moe_outputs_t* o, int32_t* local_counts,
                          double* local_psum, int32_t* local_real, void* ws, size_t ws_bytes, cudaStream_t stream) {
    moe_status_t st = check_config(cfg);
    if (st != MOE_OK) return st;
    if ((st = check_dp(cfg, T_global)) != MOE_OK) return st;
    return route_slice(cfg, weights, x, logits_in, token_mask, o, local_counts, local_psum, local_real, ws, ws_bytes,
                       plan_rows(cfg, dp_rows(cfg, T_global)), stream);
}

moe_status_t moe_dp_finish(const moe_config_t* cfg, int64_t T_global, const int32_t* all_counts,
                           const double* all_psum, const int32_t* all_real, int32_t world, int32_t rank,
                           const moe_weights_t* weights,
                           const void* x, moe_outputs_t* o, void* ws, size_t ws_bytes, cudaStream_t stream) {
    moe_status_t st = check_config(cfg);
    if (st != MOE_OK) return st;
    if ((st = check_dp(cfg, T_global)) != MOE_OK) return st;
    if ((st = check_weights(cfg, weights, false, true)) != MOE_OK) return st;
    if (world < 1 || rank < 0 || rank >= world || all_counts == nullptr || all_psum == nullptr)
        return MOE_ERR_INVALID_ARG;
    if (o == nullptr || o->counts == nullptr || o->offsets == nullptr || o->f == nullptr || o->p == nullptr ||
        o->l_aux == nullptr)
        return MOE_ERR_INVALID_ARG;
    if (cfg->T > 0 && (x == nullptr || !aligned16(x) || o->out == nullptr || !aligned16(o->out) ||
                       o->topk_idx == nullptr || o->topk_w == nullptr || o->slot == nullptr ||
                       o->src_assign == nullptr))
        return MOE_ERR_INVALID_ARG;
    const Plan pl = plan_rows(cfg, dp_rows(cfg, T_global));
    if ((st = check_ws_plan(pl, ws, ws_bytes)) != MOE_OK) return st;
    DpPrepareArgs dp;
    dp.all_counts = all_counts;
    dp.all_psum = all_psum;
    dp.all_real = all_real;
    dp.world = world;
    dp.rank = rank;
    dp.E = cfg->E;
    dp.k = cfg->k;
    dp.cap = (int)dp_cap_used(cfg, T_global);
    dp.T_global = T_global;
    dp.alpha = cfg->aux_alpha;
    dp.cap_e = reinterpret_cast<int32_t*>(at(ws, pl.cap_e));
    dp.offsets = o->offsets;
    dp.counts = o->counts;
    dp.f = o->f;
    dp.p = o->p;
    dp.l_aux = o->l_aux;
    dp.shared_off = cfg->n_shared > 0 ? reinterpret_cast<int32_t*>(at(ws, pl.shared_off)) : nullptr;
    dp.T_local = cfg->T;
    if (launch_dp_prepare(dp, stream) != cudaSuccess) return MOE_ERR_CUDA;
    if (cfg->T == 0) return MOE_OK;
    void* x_perm = at(ws, pl.xperm);
    void* y_perm = at(ws, pl.yperm);
    const bool gather = gathers(cfg);
    const bool weighted = weights_in_epilogue(cfg);
    st = run_scatter(cfg, x, o->topk_idx, o->offsets, o->slot, o->src_assign, gather ? nullptr : x_perm, ws, pl,
                     stream, dp.cap_e);
    if (st != MOE_OK) return st;
    st = run_ffn(cfg, weights, x_perm, o->offsets, y_perm, ws, pl, stream, nullptr, gather ? x : nullptr,
                 o->src_assign, weighted ? o->topk_w : nullptr);
    if (st != MOE_OK) return st;
    if (cfg->n_shared > 0) {
        // the shared experts' row offsets {0, T} were written by the prepare kernel
        auto nomark = []() { return true; };
        int n = 0;
        if ((st = run_shared(cfg, weights, x, ws, pl, stream, nomark, nullptr, &n)) != MOE_OK) return st;
    }
    return run_combine(cfg, y_perm, o->slot, weighted ? nullptr : o->topk_w, o->out, stream,
                       cfg->n_shared > 0 ? at(ws, pl.ys) : nullptr);
}

moe_status_t moe_ep_recv_rows(const moe_config_t* cfg, int64_t T_global, int32_t world, int64_t* rows) {
    moe_status_t st = check_config(cfg);
    if (st != MOE_OK) return st;
    if ((st = check_ep(cfg, T_global, world)) != MOE_OK) return st;
    if (rows == nullptr) return MOE_ERR_INVALID_ARG;
    *rows = ep_recv_rows(cfg, T_global, world);
    return MOE_OK;
}

moe_status_t moe_ep_workspace_size(const moe_config_t* cfg, int64_t T_global, int32_t world, size_t* bytes) {
    moe_status_t st = check_config(cfg);
    if (st != MOE_OK) return st;
    if ((st = check_ep(cfg, T_global, world)) != MOE_OK) return st;
    if (bytes == nullptr) return MOE_ERR_INVALID_ARG;
    *bytes = plan_ep(cfg, T_global, world).total;
    return MOE_OK;
}

moe_status_t moe_ep_route(const moe_config_t* cfg, int64_t T_global, int32_t world, const moe_weights_t* weights,
                          const void* x, const float* logits_in, const uint8_t* token_mask, moe_outputs_t* o,
                          int32_t* local_counts, double* local_psum, int32_t* local_real, void* ws, size_t ws_bytes,
                          cudaStream_t stream) {
    moe_status_t st = check_config(cfg);
    if (st != MOE_OK) return st;
    if ((st = check_ep(cfg, T_global, world)) != MOE_OK) return st;
    return route_slice(cfg, weights, x, logits_in, token_mask, o, local_counts, local_psum, local_real, ws, ws_bytes,
                       plan_ep(cfg, T_global, world), stream);
}

moe_status_t moe_ep_dispatch(const moe_config_t* cfg, int64_t T_global, const int32_t* all_counts,
                             const double* all_psum, const int32_t* all_real, int32_t world, int32_t rank,
                             const void* x,
                             void* const* x_recv, moe_outputs_t* o, int32_t* recv_offsets, void* ws,
                             size_t ws_bytes, cudaStream_t stream) {
    moe_status_t st = check_config(cfg);
    if (st != MOE_OK) return st;
    if ((st = check_ep(cfg, T_global, world)) != MOE_OK) return st;
    if (rank < 0 || rank >= world || all_counts == nullptr || all_psum == nullptr || x_recv == nullptr ||
        recv_offsets == nullptr)
        return MOE_ERR_INVALID_ARG;
    for (int r = 0; r < world; ++r)
        if (x_recv[r] == nullptr || !aligned16(x_recv[r])) return MOE_ERR_INVALID_ARG;
    if (o == nullptr || o->counts == nullptr || o->offsets == nullptr || o->f == nullptr || o->p == nullptr ||
        o->l_aux == nullptr)
        return MOE_ERR_INVALID_ARG;
    if (cfg->T > 0 && (x == nullptr || !aligned16(x) || o->topk_idx == nullptr || o->slot == nullptr))
        return MOE_ERR_INVALID_ARG;
    const Plan pl = plan_ep(cfg, T_global, world);
    if ((st = check_ws_plan(pl, ws, ws_bytes)) != MOE_OK) return st;
    const NvtxRange range("moe_ep_dispatch");
    int32_t* dest_off = reinterpret_cast<int32_t*>(at(ws, pl.ep_dest));
    int32_t* cap_e = reinterpret_cast<int32_t*>(at(ws, pl.cap_e));
    EpPrepareArgs ep;
    ep.all_counts = all_counts;
    ep.all_psum = all_psum;
    ep.all_real = all_real;
    ep.world = world;
    ep.rank = rank;
    ep.E = cfg->E;
    ep.e_per_rank = cfg->E / world;
    ep.k = cfg->k;
    ep.cap = (int)dp_cap_used(cfg, T_global);
    ep.T_global = T_global;
    ep.T_local = cfg->T;
    ep.recv_rows = pl.rows;
    ep.alpha = cfg->aux_alpha;
    ep.cap_e = cap_e;
    ep.dest_off = dest_off;
    ep.recv_offsets = recv_offsets;
    ep.offsets = o->offsets;
    ep.counts = o->counts;
    ep.f = o->f;
    ep.p = o->p;
    ep.l_aux = o->l_aux;
    ep.shared_off = cfg->n_shared > 0 ? reinterpret_cast<int32_t*>(at(ws, pl.shared_off)) : nullptr;
    ep.st = status_of(ws);
    if (launch_ep_prepare(ep, stream) != cudaSuccess) return MOE_ERR_CUDA;
    if (cfg->T == 0) return MOE_OK;
    ScatterArgs xa;
    xa.topk_idx = o->topk_idx;
    xa.hist = reinterpret_cast<const int32_t*>(at(ws, pl.hist));
    xa.group_base = reinterpret_cast<const int32_t*>(at(ws, pl.gbase));
    xa.group_chunks = pl.group_chunks;
    xa.ngroups = pl.ngroups;
    xa.offsets = dest_off;
    xa.slot = o->slot;
    xa.src_assign = nullptr;
    xa.x = x;
    xa.x_perm = nullptr;
    xa.cap_e = cap_e;
    xa.T = cfg->T;
    xa.E = cfg->E;
    xa.k = cfg->k;
    xa.cap = 0;
    xa.nchunk = pl.nchunk;
    xa.row_bytes = (int)(cfg->d * elem_size(cfg));
    for (int r = 0; r < world; ++r) xa.x_dst[r] = x_recv[r];
    xa.e_per_rank = cfg->E / world;
    xa.row_limit = pl.rows;
    xa.st = status_of(ws);
    return from_cuda(launch_dispatch_scatter(xa, stream));
}

moe_status_t moe_ep_expert_ffn(const moe_config_t* cfg, int64_t T_global, int32_t world,
                               const moe_weights_t* weights, const void* x, const void* x_recv,
                               const int32_t* recv_offsets, void* y_recv, void* ws, size_t ws_bytes,
                               cudaStream_t stream) {
    moe_status_t st = check_config(cfg);
    if (st != MOE_OK) return st;
    if ((st = check_ep(cfg, T_global, world)) != MOE_OK) return st;
    moe_config_t local = *cfg;   // this rank's experts: a pool of E/world
    local.E = cfg->E / world;
    if ((st = check_weights(&local, weights, false, true)) != MOE_OK) return st;
    if (x_recv == nullptr || y_recv == nullptr || recv_offsets == nullptr || !aligned16(x_recv) || !aligned16(y_recv))
        return MOE_ERR_INVALID_ARG;
    if (cfg->n_shared > 0 && cfg->T > 0 && (x == nullptr || !aligned16(x))) return MOE_ERR_INVALID_ARG;
    const Plan pl = plan_ep(cfg, T_global, world);
    if ((st = check_ws_plan(pl, ws, ws_bytes)) != MOE_OK) return st;
    const NvtxRange range("moe_ep_expert_ffn");
    if (pl.rows > 0) {
        st = run_ffn(&local, weights, x_recv, recv_offsets, y_recv, ws, pl, stream);
        if (st != MOE_OK) return st;
    }
    if (cfg->n_shared > 0 && cfg->T > 0) {
        // the shared experts' row offsets {0, T} were written by moe_ep_dispatch
        auto nomark = []() { return true; };
        int n = 0;
        if ((st = run_shared(cfg, weights, x, ws, pl, stream, nomark, nullptr, &n)) != MOE_OK) return st;
    }
    return MOE_OK;
}

moe_status_t moe_ep_combine(const moe_config_t* cfg, int64_t T_global, int32_t world, const void* const* y_recv,
                            moe_outputs_t* o, void* ws, size_t ws_bytes, cudaStream_t stream) {
    moe_status_t st = check_config(cfg);
    if (st != MOE_OK) return st;
    if ((st = check_ep(cfg, T_global, world)) != MOE_OK) return st;
    if (y_recv == nullptr || o == nullptr) return MOE_ERR_INVALID_ARG;
    for (int r = 0; r < world; ++r)
        if (y_recv[r] == nullptr || !aligned16(y_recv[r])) return MOE_ERR_INVALID_ARG;
    const Plan pl = plan_ep(cfg, T_global, world);
    if ((st = check_ws_plan(pl, ws, ws_bytes)) != MOE_OK) return st;
    if (cfg->T == 0) return MOE_OK;
    if (o->out == nullptr || !aligned16(o->out) || o->slot == nullptr || o->topk_w == nullptr ||
        o->topk_idx == nullptr)
        return MOE_ERR_INVALID_ARG;
    const NvtxRange range("moe_ep_combine");
    CombineArgs a;
    a.y_perm = nullptr;
    a.slot = o->slot;
    a.topk_w = o->topk_w;
    a.out = o->out;
    a.y_shared = cfg->n_shared > 0 ? at(ws, pl.ys) : nullptr;
    a.n_shared = cfg->n_shared;
    a.T = cfg->T;
    a.d = cfg->d;
    a.k = cfg->k;
    for (int r = 0; r < world; ++r) a.y_src[r] = y_recv[r];
    a.topk_idx = o->topk_idx;
    a.e_per_rank = cfg->E / world;
    a.row_limit = pl.rows;
    a.st = status_of(ws);
    return from_cuda(launch_combine(a, cfg->dtype == MOE_DT_BF16, stream));
}

moe_status_t moe_ipc_export(const void* dev_ptr, moe_ipc_buffer_t* rec) {
    if (dev_ptr == nullptr || rec == nullptr) return MOE_ERR_INVALID_ARG;
    using AddressRangeFn = CUresult (*)(CUdeviceptr*, size_t*, CUdeviceptr);
    static std::atomic<AddressRangeFn> cached{nullptr};
    AddressRangeFn fn = cached.load(std::memory_order_acquire);
    if (fn == nullptr) {
        void* ptr = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuMemGetAddressRange", &ptr, cudaEnableDefault, &q) != cudaSuccess ||
            q != cudaDriverEntryPointSuccess || ptr == nullptr)
            return MOE_ERR_CUDA;
        fn = reinterpret_cast<AddressRangeFn>(ptr);
        cached.store(fn, std::memory_order_release);
    }
    CUdeviceptr base = 0;
    size_t size = 0;
    const CUdeviceptr p = reinterpret_cast<CUdeviceptr>(dev_ptr);
    if (fn(&base, &size, p) != CUDA_SUCCESS || p < base || p >= base + size) return MOE_ERR_CUDA;
    cudaIpcMemHandle_t h;
    if (cudaIpcGetMemHandle(&h, reinterpret_cast<void*>(base)) != cudaSuccess) return MOE_ERR_CUDA;
    static_assert(sizeof(h) == sizeof(rec->handle), "IPC handle size");
    memcpy(rec->handle, &h, sizeof(h));
    rec->offset = (uint64_t)(p - base);
    rec->bytes = (uint64_t)(base + size - p);
    return MOE_OK;
}

moe_status_t moe_ipc_open(const moe_ipc_buffer_t* rec, void** dev_ptr) {
    if (rec == nullptr || dev_ptr == nullptr) return MOE_ERR_INVALID_ARG;
    cudaIpcMemHandle_t h;
    memcpy(&h, rec->handle, sizeof(h));
    void* base = nullptr;
    if (cudaIpcOpenMemHandle(&base, h, cudaIpcMemLazyEnablePeerAccess) != cudaSuccess) return MOE_ERR_CUDA;
    *dev_ptr = static_cast<uint8_t*>(base) + rec->offset;
    return MOE_OK;
}

moe_status_t moe_ipc_close(void* dev_ptr, const moe_ipc_buffer_t* rec) {
    if (dev_ptr == nullptr || rec == nullptr) return MOE_ERR_INVALID_ARG;
    return from_cuda(cudaIpcCloseMemHandle(static_cast<uint8_t*>(dev_ptr) - rec->offset));
}

moe_status_t moe_forward_hostio(const moe_config_t* cfg, const moe_weights_t* weights, const void* x_host,
                                void* x_dev, moe_outputs_t* o, void* out_host, float* l_aux_host, void* ws,
                                size_t ws_bytes, cudaStream_t stream) {
    moe_status_t st = check_config(cfg);
    if (st != MOE_OK) return st;
    if (o == nullptr || l_aux_host == nullptr) return MOE_ERR_INVALID_ARG;
    const size_t bytes = (size_t)cfg->T * cfg->d * elem_size(cfg);
    if (cfg->T > 0 && (x_host == nullptr || x_dev == nullptr || out_host == nullptr)) return MOE_ERR_INVALID_ARG;
    if (bytes && cudaMemcpyAsync(x_dev, x_host, bytes, cudaMemcpyHostToDevice, stream) != cudaSuccess)
        return MOE_ERR_CUDA;
    st = moe_forward(cfg, weights, x_dev, nullptr, nullptr, o, ws, ws_bytes, stream);
    if (st != MOE_OK) return st;
    if (bytes && cudaMemcpyAsync(out_host, o->out, bytes, cudaMemcpyDeviceToHost, stream) != cudaSuccess)
        return MOE_ERR_CUDA;
    if (cudaMemcpyAsync(l_aux_host, o->l_aux, sizeof(float), cudaMemcpyDeviceToHost, stream) != cudaSuccess)
        return MOE_ERR_CUDA;
    return MOE_OK;
}

moe_status_t moe_check_device_status(void* ws, size_t ws_bytes, cudaStream_t stream, uint32_t* site) {
    if (ws == nullptr || ws_bytes < kStatusBytes) return MOE_ERR_WORKSPACE;
    if (cudaStreamSynchronize(stream) != cudaSuccess) return MOE_ERR_CUDA;
    uint32_t words[3] = {0, 0, 0};
    if (cudaMemcpyAsync(words, ws, sizeof(words), cudaMemcpyDeviceToHost, stream) != cudaSuccess) return MOE_ERR_CUDA;
    if (cudaStreamSynchronize(stream) != cudaSuccess) return MOE_ERR_CUDA;
    if (site) *site = words[1];
    if (words[0] & (kErrTimeout | kErrRange)) {
        if (cudaMemsetAsync(ws, 0, kStatusBytes, stream) != cudaSuccess) return MOE_ERR_CUDA;
        if (cudaStreamSynchronize(stream) != cudaSuccess) return MOE_ERR_CUDA;
        return (words[0] & kErrTimeout) ? MOE_ERR_TIMEOUT : MOE_ERR_RANGE;
    }
    return MOE_OK;
}

void moe_set_wait_timeout_ms(uint32_t ms) { g_timeout_ms = ms == 0 ? 1 : ms; }

moe_status_t moe_selftest_bounded_wait(void* ws, size_t ws_bytes, uint32_t timeout_ms, cudaStream_t stream) {
    if (ws == nullptr || ws_bytes < kStatusBytes) return MOE_ERR_WORKSPACE;
    DevStatus st;
    st.word = static_cast<uint32_t*>(ws);
    st.timeout_ns = (uint64_t)(timeout_ms == 0 ? 1 : timeout_ms) * 1000000ull;
    return from_cuda(launch_selftest_wait(st, stream));
}

int32_t moe_forward_launch_count(const moe_config_t* cfg) {
    if (check_config(cfg) != MOE_OK) return 0;
    if (cfg->T == 0) return 1;
    return 5 + 2 * cfg->n_shared;  // router, scatter, two GEMMs, combine; two GEMMs per shared expert
}

}  // extern "C"
