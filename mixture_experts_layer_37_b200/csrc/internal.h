// Host-side launch interfaces between the C ABI (moe_api.cu) and the kernel
// translation units.  Internal to libmoe.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "common.cuh"

namespace moe {

struct ScanArgs {
    const int32_t* hist;   // [E, nchunk] per-chunk expert histogram
    const double* psum;    // [E, nchunk] per-chunk probability sums, or null (no aux stats)
    int32_t* chunk_base;   // [E, nchunk] out: assignments to e in earlier chunks
    int32_t* counts;       // [E] out
    int32_t* offsets;      // [E+1] out
    float* f;              // [E] out or null
    float* p;              // [E] out or null
    float* l_aux;          // [1] out or null
    double* psum_total;    // [E] out or null: sum over this batch's tokens of p[t,e] (not divided)
    int64_t T;
    int nchunk, E, k, cap;
    float alpha;
};

struct RouterArgs {
    const void* x;           // [T, d] act dtype
    const void* w_router;    // [d, E] act dtype
    const float* bias;       // [E] or null
    const float* logits_in;  // [T, E] or null
    int32_t* topk_idx;       // [T, k]
    float* topk_w;           // [T, k]
    float* logits_out;       // [T, E] or null
    float* probs_out;        // [T, E] or null
    int32_t* hist;           // [E, nchunk] per-chunk expert histogram
    double* psum;            // [E, nchunk] per-chunk sum of probabilities
    int64_t T;
    int d, E, k, nchunk;
    int tpc;                 // tokens per CTA (set by the launcher; multiple of the chunk)
    // when fuse_scan != 0: the last CTA to finish (counted on `counter`) runs
    // the dispatch scan and the aux statistics described by `scan`
    int fuse_scan;
    unsigned int* counter;
    ScanArgs scan;
    DevStatus st;            // status word and wait limit (tensor-core router)
    int kernel;              // moe_router_kernel_t
};
cudaError_t launch_router(const RouterArgs& a, bool bf16, cudaStream_t s);
// Tensor-core router (TMA + tcgen05 + TMEM): bf16, E % 8 == 0, no logits feed.
bool router_tc_supported(const RouterArgs& a);
cudaError_t launch_router_tc(const RouterArgs& a, DevStatus st, cudaStream_t s);

cudaError_t launch_dispatch_hist(const int32_t* topk_idx, int32_t* hist, int64_t T, int E, int k, cudaStream_t s);
cudaError_t launch_dispatch_scan(const ScanArgs& a, cudaStream_t s);

struct ScatterArgs {
    const int32_t* topk_idx;    // [T, k]
    const int32_t* chunk_base;  // [E, nchunk]
    const int32_t* offsets;     // [E+1]
    int32_t* slot;              // [T, k]
    int32_t* src_assign;        // [R_max]
    const void* x;              // [T, d]
    void* x_perm;               // [R_max, d], or null: no row copies (slot / src_assign only)
    const int32_t* cap_e;       // [E] per-expert capacity left for this batch, or null (use cap)
    int64_t T;
    int E, k, cap, nchunk;
    int row_bytes;              // d * element size (multiple of 16)
};
cudaError_t launch_dispatch_scatter(const ScatterArgs& a, cudaStream_t s);

// Data-parallel shard of one logical batch: from every rank's counts and
// probability sums ([world, E], gathered in rank order) compute this rank's
// per-expert capacity left, kept offsets, and the global counts / f / p / L_aux.
struct DpPrepareArgs {
    const int32_t* all_counts;  // [world, E]
    const double* all_psum;     // [world, E]
    int world, rank, E, k, cap;
    int64_t T_global;
    float alpha;
    int32_t* cap_e;             // [E] out
    int32_t* offsets;           // [E+1] out (this rank's kept rows)
    int32_t* counts;            // [E] out (global)
    float* f;                   // [E] out
    float* p;                   // [E] out
    float* l_aux;               // [1] out
};
cudaError_t launch_dp_prepare(const DpPrepareArgs& a, cudaStream_t s);

struct CombineArgs {
    const void* y_perm;    // [R_max, d]
    const int32_t* slot;   // [T, k]
    const float* topk_w;   // [T, k]
    void* out;             // [T, d]
    int64_t T;
    int d, k;
};
cudaError_t launch_combine(const CombineArgs& a, bool bf16, cudaStream_t s);
cudaError_t launch_aux_from_probs(const int32_t* counts, const float* probs, float* f, float* p, float* l_aux,
                                  int64_t T, int E, int k, float alpha, cudaStream_t s);

// Expert FFN (grouped GEMMs over the expert-sorted rows).
struct FfnArgs {
    int act;                 // 0 swiglu, 1 gelu+bias
    int E, d, ffn;
    int64_t rows_cap;        // R_max (rows allocated in x_perm / h / y_perm)
    const int32_t* offsets;  // [E+1]
    const void* x_perm;      // [rows_cap, d]
    void* h;                 // [rows_cap, ffn] (workspace)
    void* y_perm;            // [rows_cap, d]
    const void* w1;          // [E, d, ffn] (gate or W1)
    const void* w_up;        // [E, d, ffn] or null
    const void* w2;          // [E, ffn, d]
    const void* b1;          // [E, ffn] or null
    const void* b2;          // [E, d] or null
    DevStatus st;
    cudaEvent_t between;     // recorded between the two GEMM launches, or null
    int gemm_kernel;         // moe_gemm_kernel_t
    // when gather_x != null the first GEMM reads its rows straight from the
    // tokens (row s = token src_assign[s] / k) and x_perm is not used
    const void* gather_x;    // [T, d] or null
    const int32_t* src_assign;
    int k;
};
// bf16: tcgen05 grouped GEMMs (two launches).  Returns cudaErrorInvalidValue
// when a tensor map cannot be encoded.
cudaError_t launch_ffn_bf16_sm100(const FfnArgs& a, cudaStream_t s);
// f32: SIMT FMA grouped GEMMs (two launches).
cudaError_t launch_ffn_f32(const FfnArgs& a, cudaStream_t s);

cudaError_t launch_selftest_wait(DevStatus st, cudaStream_t s);

int sm_count();

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
