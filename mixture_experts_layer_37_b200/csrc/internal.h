// Host-side launch interfaces between the C ABI (moe_api.cu) and the kernel
// translation units.  Internal to libmoe.
#pragma once

#include <atomic>
#include <utility>

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "common.cuh"

namespace moe {

// Chunks of kChunkTokens tokens are grouped kGroupChunks at a time for the
// dispatch scan: the smallest power-of-two multiple of 32 chunks that keeps
// E * ngroups within the status block's group counts.
inline int group_chunks_for(int E, int64_t nchunk) {
    int g = 32;
    while ((int64_t)E * ((nchunk + g - 1) / g) > kMaxGroupEntries) g *= 2;
    return g;
}
inline int ngroups_for(int E, int64_t nchunk) {
    const int g = group_chunks_for(E, nchunk);
    return (int)((nchunk + g - 1) / g);
}

struct ScanArgs {
    int32_t* group_hist = nullptr;   // [E, ngroups] per-group expert counts (status block); read, then reset to 0
    const double* psum = nullptr;    // [E, npsum] partial sums of the probabilities, or null (no aux stats)
    int32_t* group_base = nullptr;   // [E, ngroups] out: assignments to e in earlier groups
    int32_t* counts = nullptr;       // [E] out
    int32_t* offsets = nullptr;      // [E+1] out
    float* f = nullptr;              // [E] out or null
    float* p = nullptr;              // [E] out or null
    float* l_aux = nullptr;          // [1] out or null
    double* psum_total = nullptr;    // [E] out or null: sum over this batch's tokens of p[t,e] (not divided)
    int32_t* real_counter = nullptr; // [1] real (unmasked) tokens counted by the router (read, then reset to 0),
                                     // or null: every token is real
    int32_t* shared_off = nullptr;   // [2] out or null: {0, T}, the row offsets of the shared experts' GEMMs
    int32_t* t_real_out = nullptr;   // [1] out or null: the number of real (unmasked) tokens
    int64_t T = 0;
    int ngroups = 0, npsum = 0, E = 0, k = 0, cap = 0;
    float alpha = 0;
};

struct RouterArgs {
    const void* x = nullptr;           // [T, d] act dtype
    const void* w_router = nullptr;    // [d, E] act dtype
    const float* bias = nullptr;       // [E] or null
    const float* logits_in = nullptr;  // [T, E] or null
    int32_t* topk_idx = nullptr;       // [T, k]
    float* topk_w = nullptr;           // [T, k]
    float* logits_out = nullptr;       // [T, E] or null
    float* probs_out = nullptr;        // [T, E] or null
    int32_t* hist = nullptr;           // [E, nchunk] out: per-chunk expert histogram
    int32_t* group_hist = nullptr;     // [E, ngroups] per-group counts, added atomically (zero on entry)
    double* psum = nullptr;            // [E, npsum] out: partial probability sums (per chunk, or per CTA)
    const uint8_t* mask = nullptr;     // [T] 0 = padding token (selects nothing, not in the sums), or null
    int32_t* real_counter = nullptr;   // [1] real tokens, added atomically (when mask != null)
    int64_t T = 0;
    int d = 0, E = 0, k = 0, nchunk = 0;
    int group_chunks = 32, ngroups = 0;
    int psum_cap = 0;            // columns of psum available (>= nchunk)
    int tpc = 0;                 // tokens per CTA (set by the launcher; multiple of the chunk)
    // when fuse_scan != 0: the last CTA to finish (counted on `counter`) runs
    // the dispatch scan and the aux statistics described by `scan`
    int fuse_scan = 0;
    unsigned int* counter = nullptr;
    ScanArgs scan;
    DevStatus st;            // status word and wait limit
    int kernel = 0;              // moe_router_kernel_t
};
cudaError_t launch_router(const RouterArgs& a, bool bf16, cudaStream_t s);
// Tensor-core router (TMA + tcgen05 + TMEM): bf16, E % 8 == 0, no logits feed.
bool router_tc_supported(const RouterArgs& a);
cudaError_t launch_router_tc(const RouterArgs& a, DevStatus st, cudaStream_t s);
// Warp-MMA router with the router weight resident across a CTA cluster (bf16):
// same logits as the slab-staged warp-MMA router; shapes whose weight slices
// do not fit in shared memory are not supported (the staged router takes them).
bool router_v2_supported(const RouterArgs& a);
cudaError_t launch_router_v2(const RouterArgs& a, cudaStream_t s);
int router_v2_psum_columns();  // probability-sum columns the v2 router may write per expert

cudaError_t launch_dispatch_hist(const int32_t* topk_idx, int32_t* hist, int32_t* group_hist, int64_t T, int E, int k,
                                 int group_chunks, int ngroups, cudaStream_t s);
cudaError_t launch_dispatch_scan(const ScanArgs& a, cudaStream_t s);

struct ScatterArgs {
    const int32_t* topk_idx = nullptr;    // [T, k]
    const int32_t* hist = nullptr;        // [E, nchunk] per-chunk expert histogram
    const int32_t* group_base = nullptr;  // [E, ngroups] assignments to e in earlier groups of group_chunks chunks
    const int32_t* offsets = nullptr;     // [E+1]
    int32_t* slot = nullptr;              // [T, k]
    int32_t* src_assign = nullptr;        // [R_max]
    const void* x = nullptr;              // [T, d]
    void* x_perm = nullptr;               // [R_max, d], or null: no row copies (slot / src_assign only)
    const int32_t* cap_e = nullptr;       // [E] per-expert capacity left for this batch, or null (use cap)
    int64_t T = 0;
    int E = 0, k = 0, cap = 0, nchunk = 0, group_chunks = 32, ngroups = 0;
    int row_bytes = 0;              // d * element size (multiple of 16)
    // expert parallelism (e_per_rank > 0): the rows of expert e go to
    // x_dst[e / e_per_rank] (the receive buffer of the rank holding e, possibly
    // a peer's memory), slot = row there; rows at or past row_limit are refused
    // (slot -1, kErrRange in st); src_assign may be null
    void* x_dst[kMaxRanks] = {};
    int e_per_rank = 0;
    int64_t row_limit = 0;          // > 0: bound of every destination row
    DevStatus st;
};
cudaError_t launch_dispatch_scatter(const ScatterArgs& a, cudaStream_t s);

// Data-parallel shard of one logical batch: from every rank's counts and
// probability sums ([world, E], gathered in rank order) compute this rank's
// per-expert capacity left, kept offsets, and the global counts / f / p / L_aux.
struct DpPrepareArgs {
    const int32_t* all_counts = nullptr;  // [world, E]
    const double* all_psum = nullptr;     // [world, E]
    const int32_t* all_real = nullptr;    // [world] real tokens per rank, or null: every token is real
    int world = 0, rank = 0, E = 0, k = 0, cap = 0;
    int64_t T_global = 0;
    float alpha = 0;
    int32_t* cap_e = nullptr;             // [E] out
    int32_t* offsets = nullptr;           // [E+1] out (this rank's kept rows)
    int32_t* counts = nullptr;            // [E] out (global)
    float* f = nullptr;                   // [E] out
    float* p = nullptr;                   // [E] out
    float* l_aux = nullptr;               // [1] out
    int32_t* shared_off = nullptr;        // [2] out or null: {0, T_local}, the shared experts' row offsets
    int64_t T_local = 0;
};
cudaError_t launch_dp_prepare(const DpPrepareArgs& a, cudaStream_t s);

// Expert-parallel shard: rank `rank` holds the tokens of its slice and the
// experts [rank*e_per_rank, (rank+1)*e_per_rank).  From every rank's counts
// and probability sums ([world, E], gathered in rank order): the capacity
// left for this slice, the first row in its owner's receive buffer of this
// slice's kept rows of each expert, this rank's receive offsets as an owner,
// and the whole batch's counts, offsets, f, p, L_aux.
struct EpPrepareArgs {
    const int32_t* all_counts = nullptr;  // [world, E]
    const double* all_psum = nullptr;     // [world, E]
    const int32_t* all_real = nullptr;    // [world] real tokens per rank, or null: every token is real
    int world = 0, rank = 0, E = 0, e_per_rank = 0, k = 0, cap = 0;
    int64_t T_global = 0, T_local = 0;
    int64_t recv_rows = 0;                // rows of every receive buffer
    float alpha = 0;
    int32_t* cap_e = nullptr;             // [E] out
    int32_t* dest_off = nullptr;          // [E] out: row in owner(e)'s buffer of this slice's first kept row of e
    int32_t* recv_offsets = nullptr;      // [e_per_rank + 1] out: this rank's received rows per local expert
    int32_t* offsets = nullptr;           // [E+1] out: the whole batch's kept-row offsets (single-device layout)
    int32_t* counts = nullptr;            // [E] out (global)
    float* f = nullptr;                   // [E] out
    float* p = nullptr;                   // [E] out
    float* l_aux = nullptr;               // [1] out
    int32_t* shared_off = nullptr;        // [2] out or null: {0, T_local}
    DevStatus st;
};
cudaError_t launch_ep_prepare(const EpPrepareArgs& a, cudaStream_t s);

struct CombineArgs {
    const void* y_perm = nullptr;    // [R_max, d]
    const int32_t* slot = nullptr;   // [T, k]
    const float* topk_w = nullptr;   // [T, k], or null: rows already weighted (plain sum)
    void* out = nullptr;             // [T, d]
    const void* y_shared = nullptr;  // [n_shared, T, d] shared experts' outputs, added with weight 1, or null
    int n_shared = 0;
    int64_t T = 0;
    int d = 0, k = 0;
    // expert parallelism (e_per_rank > 0): row slot[t,j] of y_src[topk_idx[t,j] / e_per_rank]
    // (the output buffer of the rank holding the expert, possibly a peer's memory); slots at or
    // past row_limit are refused (kErrRange in st)
    const void* y_src[kMaxRanks] = {};
    const int32_t* topk_idx = nullptr;
    int e_per_rank = 0;
    int64_t row_limit = 0;
    DevStatus st;
};
cudaError_t launch_combine(const CombineArgs& a, bool bf16, cudaStream_t s);
cudaError_t launch_aux_from_probs(const int32_t* counts, const float* probs, float* f, float* p, float* l_aux,
                                  int64_t T, int E, int k, float alpha, cudaStream_t s);

// Expert FFN (grouped GEMMs over the expert-sorted rows).
struct FfnArgs {
    int act = 0;                 // 0 swiglu, 1 gelu+bias
    int E = 0, d = 0, ffn = 0;
    int64_t rows_cap = 0;        // R_max (rows allocated in x_perm / h / y_perm)
    const int32_t* offsets = nullptr;  // [E+1]
    const void* x_perm = nullptr;      // [rows_cap, d]
    void* h = nullptr;                 // [rows_cap, ffn] (workspace)
    void* y_perm = nullptr;            // [rows_cap, d]
    const void* w1 = nullptr;          // [E, d, ffn] (gate or W1)
    const void* w_up = nullptr;        // [E, d, ffn] or null
    const void* w2 = nullptr;          // [E, ffn, d]
    const void* b1 = nullptr;          // [E, ffn] or null
    const void* b2 = nullptr;          // [E, d] or null
    DevStatus st;
    cudaEvent_t between = nullptr;  // recorded between the two GEMM launches, or null
    int gemm_kernel = 0;         // moe_gemm_kernel_t
    // when gather_x != null the first GEMM reads its rows straight from the
    // tokens (row s = token src_assign[s] / k) and x_perm is not used
    const void* gather_x = nullptr;    // [gather_rows, d] or null
    const int32_t* src_assign = nullptr;
    int64_t gather_rows = 0;           // T: rows of gather_x
    int k = 0;
    // bf16 only: when row_w != null the second GEMM multiplies output row s by
    // row_w[src_assign[s]] (its routing weight) before rounding
    const float* row_w = nullptr;      // [T*k] or null
    // INT8 weights (w1 / w_up / w2 hold codes): per-expert, per-output-column scales
    bool int8 = false;
    const float* w1_scale = nullptr;   // [E, ffn]
    const float* w_up_scale = nullptr; // [E, ffn] or null
    const float* w2_scale = nullptr;   // [E, d]
};
// bf16: tcgen05 grouped GEMMs (two launches).  Returns cudaErrorInvalidValue
// when a tensor map cannot be encoded.
cudaError_t launch_ffn_bf16_sm100(const FfnArgs& a, cudaStream_t s);
// f32: SIMT FMA grouped GEMMs (two launches).
cudaError_t launch_ffn_f32(const FfnArgs& a, cudaStream_t s);
// bf16 activations, INT8 weights (two launches), and the quantiser.
cudaError_t launch_ffn_int8(const FfnArgs& a, cudaStream_t s);
cudaError_t launch_quantize_int8(const void* w, bool bf16, int64_t E, int64_t K, int64_t N, int8_t* q, float* scale,
                                 cudaStream_t s);

cudaError_t launch_selftest_wait(DevStatus st, cudaStream_t s);

int sm_count();

// Programmatic dependent launch inside one forward.  While a PdlScope lives on
// this host thread, launch_kernel starts kernels with programmatic stream
// serialization: a kernel's launch and prologue overlap the tail of the kernel
// before it on the stream.  Every kernel launched that way executes
// griddep_wait() before it reads anything an earlier kernel wrote (for a
// kernel launched without the attribute that wait returns at once).
bool pdl_enabled();
struct PdlScope {
    PdlScope();
    ~PdlScope();
    PdlScope(const PdlScope&) = delete;
    PdlScope& operator=(const PdlScope&) = delete;
    bool prev;
};
template <class... KArgs, class... Args>
cudaError_t launch_kernel(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t s,
                          Args&&... args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    if (pdl_enabled()) {
        attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        attr[0].val.programmaticStreamSerializationAllowed = 1;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
    }
    return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

// Raises a kernel's dynamic shared-memory limit once per device.  Safe from
// several host threads: concurrent first calls may both set it (idempotent).
template <class Kernel>
cudaError_t ensure_smem_attr(std::atomic<bool> (&done)[64], Kernel kernel, int bytes) {
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev < 64 && done[dev].load(std::memory_order_acquire)) return cudaSuccess;
    const cudaError_t err = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
    if (err == cudaSuccess && dev < 64) done[dev].store(true, std::memory_order_release);
    return err;
}

// Records `ev` on `s`; while `s` is being captured into a CUDA graph, as an
// external record, so that the event still marks (and times) each replay.
inline cudaError_t record_mark(cudaEvent_t ev, cudaStream_t s) {
    cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
    cudaError_t err = cudaStreamIsCapturing(s, &cs);
    if (err != cudaSuccess) return err;
    return cs == cudaStreamCaptureStatusActive ? cudaEventRecordWithFlags(ev, s, cudaEventRecordExternal)
                                                : cudaEventRecord(ev, s);
}

}  // namespace moe
