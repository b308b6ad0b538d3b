// Capacity-bounded dispatch: expert histogram -> scan -> stable scatter and
// row gather.
//
// Method: the per-expert capacity and the rule that tokens beyond it are
// dropped ("MoE: gating, experts, load balancing, capacity factor"
// (dpshk.com/news/6005940) §2.4), applied in token order; grouping of the
// top-k assignments into one contiguous block of rows per expert ("Hand-
// building a LLaMA4-MoE" (dpshk.com/news/5809432) §2.4: sort by expert id,
// per-expert counts, split).
//
// Deterministic by construction: the rank of assignment (t, j) among the
// assignments to its expert is computed from per-chunk histograms and an
// exclusive scan (over chunks, per expert), then within a chunk from warp
// match/ballot masks and a scan over warps; no atomic decides an order.
#include "internal.h"

namespace moe {
namespace {

constexpr int kScatterThreads = 256;
constexpr int kScatterWarps = kScatterThreads / 32;

__global__ void __launch_bounds__(256) hist_kernel(const int32_t* __restrict__ idx, int32_t* __restrict__ hist,
                                                   int64_t T, int E, int k) {
    __shared__ int sHist[kMaxExperts];
    const int tid = threadIdx.x;
    if (tid < E) sHist[tid] = 0;
    __syncthreads();
    const int64_t a0 = (int64_t)blockIdx.x * kChunkTokens * k;
    const int64_t a1 = min64(a0 + (int64_t)kChunkTokens * k, T * k);
    for (int64_t a = a0 + tid; a < a1; a += blockDim.x) {
        const int e = idx[a];
        if (e >= 0 && e < E) atomicAdd(&sHist[e], 1);
    }
    __syncthreads();
    if (tid < E) hist[(int64_t)blockIdx.x * E + tid] = sHist[tid];
}

__device__ __forceinline__ int warp_inclusive_scan(int v, int lane) {
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int n = __shfl_up_sync(0xffffffffu, v, o);
        if (lane >= o) v += n;
    }
    return v;
}

// One CTA: per-expert exclusive scan of the chunk histograms (chunk bases),
// totals (counts), kept offsets, and the load-balance statistics.
__global__ void __launch_bounds__(1024) scan_kernel(ScanArgs a) {
    __shared__ int sCount[kMaxExperts];
    __shared__ double sP[kMaxExperts];
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int E = a.E;
    for (int e = warp; e < E; e += 32) {
        int run = 0;
        for (int c0 = 0; c0 < a.nchunk; c0 += 32) {
            const int c = c0 + lane;
            const int v = c < a.nchunk ? a.hist[(int64_t)c * E + e] : 0;
            const int incl = warp_inclusive_scan(v, lane);
            if (c < a.nchunk) a.chunk_base[(int64_t)c * E + e] = run + incl - v;
            run += __shfl_sync(0xffffffffu, incl, 31);
        }
        if (lane == 0) sCount[e] = run;
    }
    if (a.psum != nullptr && tid < E) {
        double s = 0.0;
        for (int c = 0; c < a.nchunk; ++c) s += a.psum[(int64_t)c * E + tid];
        sP[tid] = a.T > 0 ? s / (double)a.T : 0.0;
    }
    __syncthreads();
    if (tid == 0) {
        int off = 0;
        double l = 0.0;
        for (int e = 0; e < E; ++e) {
            a.counts[e] = sCount[e];
            a.offsets[e] = off;
            off += min(sCount[e], a.cap);
            if (a.psum != nullptr) {
                const double f = a.T > 0 ? (double)sCount[e] / ((double)a.T * a.k) : 0.0;
                if (a.f) a.f[e] = (float)f;
                if (a.p) a.p[e] = (float)sP[e];
                l += f * sP[e];
            }
        }
        a.offsets[E] = off;
        if (a.psum != nullptr && a.l_aux) a.l_aux[0] = (float)((double)a.alpha * E * l);
    }
}

// One CTA per chunk of kChunkTokens tokens: ranks, capacity test, slot and
// src_assign, then the row copies x[t] -> x_perm[slot] (16-byte vectors,
// one warp per row).
__global__ void __launch_bounds__(kScatterThreads) scatter_kernel(ScatterArgs a) {
    __shared__ int sRun[kMaxExperts];
    __shared__ int sWarpBase[kScatterWarps][kMaxExperts];
    __shared__ int sSlot[kScatterThreads];
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int E = a.E, k = a.k;
    const int chunk = blockIdx.x;
    const int64_t t0 = (int64_t)chunk * kChunkTokens;
    const int ntok = (int)min64(kChunkTokens, a.T - t0);
    const int nA = ntok * k;
    const int64_t a_base = t0 * k;
    if (tid < E) sRun[tid] = a.chunk_base[(int64_t)chunk * E + tid];
    const uint32_t lt_mask = (1u << lane) - 1u;
    const int vecs = a.row_bytes / 16;
    for (int g0 = 0; g0 < nA; g0 += kScatterThreads) {
        for (int i = tid; i < kScatterWarps * kMaxExperts; i += kScatterThreads) (&sWarpBase[0][0])[i] = 0;
        __syncthreads();
        const int i = g0 + tid;
        int e = -1;
        if (i < nA) {
            e = a.topk_idx[a_base + i];
            if (e < 0 || e >= E) e = -1;
        }
        const uint32_t peers = __match_any_sync(0xffffffffu, e);
        const int lrank = __popc(peers & lt_mask);
        if (e >= 0 && lrank == 0) sWarpBase[warp][e] = __popc(peers);
        __syncthreads();
        if (tid < E) {
            int run = sRun[tid];
            for (int w = 0; w < kScatterWarps; ++w) {
                const int c = sWarpBase[w][tid];
                sWarpBase[w][tid] = run;
                run += c;
            }
            sRun[tid] = run;
        }
        __syncthreads();
        int s = -1;
        if (e >= 0) {
            const int rank = sWarpBase[warp][e] + lrank;
            if (rank < a.cap) {
                s = a.offsets[e] + rank;
                a.src_assign[s] = (int32_t)(a_base + i);
            }
        }
        if (i < nA) a.slot[a_base + i] = s;
        sSlot[tid] = s;
        __syncthreads();
        // row gather for this group of assignments
        const int ng = min(kScatterThreads, nA - g0);
        for (int q = warp; q < ng; q += kScatterWarps) {
            const int sq = sSlot[q];
            if (sq < 0) continue;
            const int64_t t = (a_base + g0 + q) / k;
            const uint4* src = reinterpret_cast<const uint4*>(static_cast<const uint8_t*>(a.x) + t * a.row_bytes);
            uint4* dst = reinterpret_cast<uint4*>(static_cast<uint8_t*>(a.x_perm) + (int64_t)sq * a.row_bytes);
            for (int v = lane; v < vecs; v += 32) dst[v] = src[v];
        }
        __syncthreads();
    }
}

}  // namespace

cudaError_t launch_dispatch_hist(const int32_t* topk_idx, int32_t* hist, int64_t T, int E, int k, cudaStream_t s) {
    const int nchunk = (int)((T + kChunkTokens - 1) / kChunkTokens);
    if (nchunk == 0) return cudaSuccess;
    hist_kernel<<<nchunk, 256, 0, s>>>(topk_idx, hist, T, E, k);
    return cudaGetLastError();
}

cudaError_t launch_dispatch_scan(const ScanArgs& a, cudaStream_t s) {
    scan_kernel<<<1, 1024, 0, s>>>(a);
    return cudaGetLastError();
}

cudaError_t launch_dispatch_scatter(const ScatterArgs& a, cudaStream_t s) {
    const int nchunk = (int)((a.T + kChunkTokens - 1) / kChunkTokens);
    if (nchunk == 0) return cudaSuccess;
    scatter_kernel<<<nchunk, kScatterThreads, 0, s>>>(a);
    return cudaGetLastError();
}

}  // namespace moe
