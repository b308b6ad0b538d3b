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
// assignments to its expert is the chunk's base (an exclusive scan over
// chunks of per-chunk histograms) plus the rank inside the chunk, taken from
// warp match masks and a scan over warps; no atomic decides an order.
#include "scan.cuh"

namespace moe {
namespace {

constexpr int kScatterThreads = 256;
constexpr int kScatterWarps = kScatterThreads / 32;
static_assert(kChunkTokens * kMaxTopK <= kScatterThreads, "one scatter CTA covers a chunk's assignments");

__global__ void __launch_bounds__(256) hist_kernel(const int32_t* __restrict__ idx, int32_t* __restrict__ hist,
                                                   int64_t T, int E, int k, int nchunk) {
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
    if (tid < E) hist[(int64_t)tid * nchunk + blockIdx.x] = sHist[tid];
}

__global__ void __launch_bounds__(1024) scan_kernel(ScanArgs a) {
    __shared__ int sCount[kMaxExperts];
    __shared__ double sP[kMaxExperts];
    scan_block(a, sCount, sP);
}

// One CTA per chunk of kChunkTokens tokens (<= 256 assignments): ranks,
// capacity test, slot and src_assign, then the row copies x[t] -> x_perm[slot]
// (each warp copies two rows at a time with 16-byte vectors).
__global__ void __launch_bounds__(kScatterThreads) scatter_kernel(ScatterArgs a) {
    __shared__ int sWarpBase[kScatterWarps][kMaxExperts];
    __shared__ int sSlot[kScatterThreads];
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int E = a.E, k = a.k;
    const int chunk = blockIdx.x;
    const int64_t t0 = (int64_t)chunk * kChunkTokens;
    const int ntok = (int)min64(kChunkTokens, a.T - t0);
    const int nA = ntok * k;
    const int64_t a_base = t0 * k;
    for (int i = tid; i < kScatterWarps * kMaxExperts; i += kScatterThreads) (&sWarpBase[0][0])[i] = 0;
    int e = -1;
    if (tid < nA) {
        e = a.topk_idx[a_base + tid];
        if (e < 0 || e >= E) e = -1;
    }
    __syncthreads();
    const uint32_t peers = __match_any_sync(0xffffffffu, e);
    const int lrank = __popc(peers & ((1u << lane) - 1u));
    if (e >= 0 && lrank == 0) sWarpBase[warp][e] = __popc(peers);
    __syncthreads();
    if (tid < E) {
        int run = a.chunk_base[(int64_t)tid * a.nchunk + chunk];
        for (int w = 0; w < kScatterWarps; ++w) {
            const int c = sWarpBase[w][tid];
            sWarpBase[w][tid] = run;
            run += c;
        }
    }
    __syncthreads();
    int s = -1;
    if (e >= 0) {
        const int rank = sWarpBase[warp][e] + lrank;
        const int cap = a.cap_e != nullptr ? a.cap_e[e] : a.cap;
        if (rank < cap) {
            s = a.offsets[e] + rank;
            a.src_assign[s] = (int32_t)(a_base + tid);
        }
    }
    if (tid < nA) a.slot[a_base + tid] = s;
    if (a.x_perm == nullptr) return;  // rows gathered by the first GEMM instead
    sSlot[tid] = s;
    __syncthreads();
    // row gather: each warp copies two rows at a time (16-byte vectors, up to
    // 16 loads in flight per lane); dropped assignments copy nothing
    const int vecs = a.row_bytes / 16;
    const uint4* X = static_cast<const uint4*>(a.x);
    uint4* XP = static_cast<uint4*>(a.x_perm);
    for (int q = warp; q < nA; q += 2 * kScatterWarps) {
        const int q1 = q + kScatterWarps;
        const int s0 = sSlot[q];
        const int s1 = q1 < nA ? sSlot[q1] : -1;
        const uint4* src0 = X + ((a_base + q) / k) * vecs;
        const uint4* src1 = X + ((a_base + (q1 < nA ? q1 : q)) / k) * vecs;
        for (int v0 = lane; v0 < vecs; v0 += 32 * 8) {
            uint4 b0[8], b1[8];
#pragma unroll
            for (int u = 0; u < 8; ++u) {
                const int v = v0 + 32 * u;
                if (v < vecs) {
                    if (s0 >= 0) b0[u] = src0[v];
                    if (s1 >= 0) b1[u] = src1[v];
                }
            }
#pragma unroll
            for (int u = 0; u < 8; ++u) {
                const int v = v0 + 32 * u;
                if (v < vecs) {
                    if (s0 >= 0) XP[(int64_t)s0 * vecs + v] = b0[u];
                    if (s1 >= 0) XP[(int64_t)s1 * vecs + v] = b1[u];
                }
            }
        }
    }
}

// One CTA: data-parallel shard preparation (see DpPrepareArgs).  The
// assignment rank of this rank's tokens in the whole batch is the number of
// assignments to the same expert on lower ranks plus the local rank, so this
// rank may keep max(0, cap - base_e) more rows of expert e.  Sums over ranks
// run in rank order.
__global__ void __launch_bounds__(64) dp_prepare_kernel(DpPrepareArgs a) {
    __shared__ int sKept[kMaxExperts];
    __shared__ int sCount[kMaxExperts];
    __shared__ double sP[kMaxExperts];
    const int e = threadIdx.x;
    if (e < a.E) {
        int base = 0, total = 0;
        double ps = 0.0;
        for (int r = 0; r < a.world; ++r) {
            const int c = a.all_counts[(int64_t)r * a.E + e];
            if (r < a.rank) base += c;
            total += c;
            ps += a.all_psum[(int64_t)r * a.E + e];
        }
        const int mine = a.all_counts[(int64_t)a.rank * a.E + e];
        const int left = a.cap - base > 0 ? a.cap - base : 0;
        a.cap_e[e] = left;
        sKept[e] = mine < left ? mine : left;
        sCount[e] = total;
        sP[e] = a.T_global > 0 ? ps / (double)a.T_global : 0.0;
    }
    __syncthreads();
    if (e == 0) {
        int off = 0;
        double l = 0.0;
        for (int i = 0; i < a.E; ++i) {
            a.offsets[i] = off;
            off += sKept[i];
            a.counts[i] = sCount[i];
            const double f = a.T_global > 0 ? (double)sCount[i] / ((double)a.T_global * a.k) : 0.0;
            a.f[i] = (float)f;
            a.p[i] = (float)sP[i];
            l += f * sP[i];
        }
        a.offsets[a.E] = off;
        a.l_aux[0] = (float)((double)a.alpha * a.E * l);
        if (a.shared_off != nullptr) {
            a.shared_off[0] = 0;
            a.shared_off[1] = (int32_t)a.T_local;
        }
    }
}

}  // namespace

cudaError_t launch_dp_prepare(const DpPrepareArgs& a, cudaStream_t s) {
    dp_prepare_kernel<<<1, 64, 0, s>>>(a);
    return cudaGetLastError();
}

cudaError_t launch_dispatch_hist(const int32_t* topk_idx, int32_t* hist, int64_t T, int E, int k, cudaStream_t s) {
    const int nchunk = (int)((T + kChunkTokens - 1) / kChunkTokens);
    if (nchunk == 0) return cudaSuccess;
    hist_kernel<<<nchunk, 256, 0, s>>>(topk_idx, hist, T, E, k, nchunk);
    return cudaGetLastError();
}

cudaError_t launch_dispatch_scan(const ScanArgs& a, cudaStream_t s) {
    scan_kernel<<<1, 1024, 0, s>>>(a);
    return cudaGetLastError();
}

cudaError_t launch_dispatch_scatter(const ScatterArgs& a, cudaStream_t s) {
    if (a.nchunk == 0) return cudaSuccess;
    scatter_kernel<<<a.nchunk, kScatterThreads, 0, s>>>(a);
    return cudaGetLastError();
}

}  // namespace moe
