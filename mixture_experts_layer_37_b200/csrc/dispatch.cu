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
// assignments to its expert is the chunk's base (the exclusive scan over
// groups of chunks, plus the counts of the earlier chunks of its group) plus
// the rank inside the chunk, taken from warp match masks and a scan over
// warps; no atomic decides an order (the group counts are integer sums).
#include "scan.cuh"

namespace moe {
namespace {

constexpr int kScatterThreads = 256;
constexpr int kScatterWarps = kScatterThreads / 32;
static_assert(kChunkTokens * kMaxTopK <= kScatterThreads, "one scatter CTA covers a chunk's assignments");

__global__ void __launch_bounds__(256) hist_kernel(const int32_t* __restrict__ idx, int32_t* __restrict__ hist,
                                                   int32_t* __restrict__ group_hist, int64_t T, int E, int k,
                                                   int nchunk, int group_chunks, int ngroups) {
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
    if (tid < E) {
        const int n = sHist[tid];
        hist[(int64_t)tid * nchunk + blockIdx.x] = n;
        if (n) atomicAdd(group_hist + (int64_t)tid * ngroups + blockIdx.x / group_chunks, n);
    }
}

__global__ void __launch_bounds__(1024) scan_kernel(ScanArgs a) {
    __shared__ int sCount[kMaxExperts];
    __shared__ double sP[kMaxExperts];
    scan_block(a, sCount, sP);
}

// `nsplit` CTAs per chunk of kChunkTokens tokens (<= 256 assignments): each
// computes the chunk's ranks, capacity test and slots (the first one writes
// slot and src_assign), then copies its share of the rows x[t] -> x_perm[slot]
// (each warp copies two rows at a time with 16-byte vectors; splitting a
// chunk's copies over several CTAs keeps every SM busy when chunks are few).
// Under expert parallelism the destination is the receive buffer of the
// expert's rank, so the copies are this step's all-to-all: stores into peer
// memory over NVLink.
__global__ void __launch_bounds__(kScatterThreads) scatter_kernel(ScatterArgs a, int nsplit) {
    __shared__ int sWarpBase[kScatterWarps][kMaxExperts];
    __shared__ uint4* sDst[kScatterThreads];
    griddep_wait();  // the routing of the launch before
    griddep_launch_dependents();
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int E = a.E, k = a.k;
    const int chunk = blockIdx.x / nsplit, part = blockIdx.x - chunk * nsplit;
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
        int run = chunk_base_of(a.hist, a.group_base, tid, chunk, a.nchunk, a.group_chunks, a.ngroups);
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
            if (a.row_limit > 0 && (s < 0 || s >= a.row_limit)) {
                if (a.st.word != nullptr) report_range(a.st, SITE_EP_SCATTER_ROW);
                s = -1;
            } else if (a.src_assign != nullptr && part == 0) {
                a.src_assign[s] = (int32_t)(a_base + tid);
            }
        }
    }
    if (tid < nA && part == 0) a.slot[a_base + tid] = s;
    const bool ep = a.e_per_rank > 0;
    if (a.x_perm == nullptr && !ep) return;  // rows gathered by the first GEMM instead
    uint4* dst = nullptr;
    if (s >= 0) {
        void* base = ep ? a.x_dst[e / a.e_per_rank] : a.x_perm;
        dst = reinterpret_cast<uint4*>(static_cast<uint8_t*>(base) + (int64_t)s * a.row_bytes);
    }
    sDst[tid] = dst;
    __syncthreads();
    // row gather: each warp copies two rows at a time (16-byte vectors, up to
    // 16 loads in flight per lane); dropped assignments copy nothing
    const int vecs = a.row_bytes / 16;
    const uint4* X = static_cast<const uint4*>(a.x);
    const int qb = part * nA / nsplit, qe = (part + 1) * nA / nsplit;  // this CTA's assignments
    for (int q = qb + warp; q < qe; q += 2 * kScatterWarps) {
        const int q1 = q + kScatterWarps;
        uint4* d0 = sDst[q];
        uint4* d1 = q1 < qe ? sDst[q1] : nullptr;
        const uint4* src0 = X + ((a_base + q) / k) * vecs;
        const uint4* src1 = X + ((a_base + (q1 < qe ? q1 : q)) / k) * vecs;
        for (int v0 = lane; v0 < vecs; v0 += 32 * 8) {
            uint4 b0[8], b1[8];
#pragma unroll
            for (int u = 0; u < 8; ++u) {
                const int v = v0 + 32 * u;
                if (v < vecs) {
                    if (d0 != nullptr) b0[u] = src0[v];
                    if (d1 != nullptr) b1[u] = src1[v];
                }
            }
#pragma unroll
            for (int u = 0; u < 8; ++u) {
                const int v = v0 + 32 * u;
                if (v < vecs) {
                    if (d0 != nullptr) d0[v] = b0[u];
                    if (d1 != nullptr) d1[v] = b1[u];
                }
            }
        }
    }
}

// The batch's real tokens (padding masked out): the ranks' counts summed in
// rank order, or every token when no count is given.
__device__ __forceinline__ int64_t real_tokens(const int32_t* all_real, int world, int64_t T_global) {
    if (all_real == nullptr) return T_global;
    int64_t n = 0;
    for (int r = 0; r < world; ++r) n += all_real[r];
    return n;
}

// One CTA: data-parallel shard preparation (see DpPrepareArgs).  The
// assignment rank of this rank's tokens in the whole batch is the number of
// assignments to the same expert on lower ranks plus the local rank, so this
// rank may keep max(0, cap - base_e) more rows of expert e.  Sums over ranks
// run in rank order.  f and p divide by the batch's real tokens (padding
// masked out); the capacity is that of all T_global tokens.
__global__ void __launch_bounds__(64) dp_prepare_kernel(DpPrepareArgs a) {
    __shared__ int sKept[kMaxExperts];
    __shared__ int sCount[kMaxExperts];
    __shared__ double sP[kMaxExperts];
    const int e = threadIdx.x;
    const int64_t t_real = real_tokens(a.all_real, a.world, a.T_global);
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
        sP[e] = t_real > 0 ? ps / (double)t_real : 0.0;
    }
    __syncthreads();
    if (e == 0) {
        int off = 0;
        double l = 0.0;
        for (int i = 0; i < a.E; ++i) {
            a.offsets[i] = off;
            off += sKept[i];
            a.counts[i] = sCount[i];
            const double f = t_real > 0 ? (double)sCount[i] / ((double)t_real * a.k) : 0.0;
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

// One CTA: expert-parallel shard preparation (see EpPrepareArgs).  Ranks
// before this one keep min(base_e, cap) rows of expert e, so this slice's
// kept rows of e start there within e's block in its owner's buffer; an
// owner's blocks follow its experts in ascending id, each of size
// min(total_e, cap), so every expert's rows sit in the batch's token order.
// The capacity left for this slice is also capped by the slice's own
// gathered count, so that a slice can never write past its part of e's block.
// If the gathered counts are negative or would overflow any owner's receive
// buffer, nothing is kept (cap_e = 0, all offsets 0) and kErrRange is set.
__global__ void __launch_bounds__(64) ep_prepare_kernel(EpPrepareArgs a) {
    __shared__ int64_t sBefore[kMaxExperts];
    __shared__ int64_t sTotal[kMaxExperts];
    __shared__ int64_t sMine[kMaxExperts];
    __shared__ double sP[kMaxExperts];
    __shared__ int sBad;
    const int e = threadIdx.x;
    const int64_t t_real = real_tokens(a.all_real, a.world, a.T_global);
    if (e == 0) sBad = 0;
    __syncthreads();
    if (e < a.E) {
        int64_t base = 0, total = 0;
        double ps = 0.0;
        for (int r = 0; r < a.world; ++r) {
            const int c = a.all_counts[(int64_t)r * a.E + e];
            if (c < 0) sBad = 1;
            if (r < a.rank) base += c;
            total += c;
            ps += a.all_psum[(int64_t)r * a.E + e];
        }
        sBefore[e] = base;
        sTotal[e] = total;
        sMine[e] = a.all_counts[(int64_t)a.rank * a.E + e];
        sP[e] = t_real > 0 ? ps / (double)t_real : 0.0;
    }
    __syncthreads();
    if (e == 0) {
        for (int o = 0; o < a.world; ++o) {
            int64_t rows = 0;
            for (int el = 0; el < a.e_per_rank; ++el) rows += min64(sTotal[o * a.e_per_rank + el], a.cap);
            if (rows > a.recv_rows) sBad = 1;
        }
        if (sBad) report_range(a.st, SITE_EP_PREPARE_ROWS);
    }
    __syncthreads();
    const bool ok = sBad == 0;
    if (e < a.E) {
        const int64_t left = min64(a.cap - sBefore[e], sMine[e]);
        a.cap_e[e] = ok && left > 0 ? (int32_t)left : 0;
    }
    if (e == 0) {
        int64_t off = 0, owner_off = 0;
        double l = 0.0;
        for (int i = 0; i < a.E; ++i) {
            const int el = i % a.e_per_rank;
            const bool mine = i / a.e_per_rank == a.rank;
            if (el == 0) owner_off = 0;
            const int64_t kept = ok ? min64(sTotal[i], a.cap) : 0;
            a.dest_off[i] = (int32_t)(owner_off + (ok ? min64(sBefore[i], a.cap) : 0));
            if (mine) a.recv_offsets[el] = (int32_t)owner_off;
            owner_off += kept;
            if (mine && el == a.e_per_rank - 1) a.recv_offsets[a.e_per_rank] = (int32_t)owner_off;
            a.offsets[i] = (int32_t)off;
            off += kept;
            const int32_t cnt = ok ? (int32_t)sTotal[i] : 0;
            a.counts[i] = cnt;
            const double f = t_real > 0 ? (double)cnt / ((double)t_real * a.k) : 0.0;
            a.f[i] = (float)f;
            a.p[i] = (float)sP[i];
            l += f * sP[i];
        }
        a.offsets[a.E] = (int32_t)off;
        a.l_aux[0] = (float)((double)a.alpha * a.E * l);
        if (a.shared_off != nullptr) {
            a.shared_off[0] = 0;
            a.shared_off[1] = (int32_t)a.T_local;
        }
    }
}

}  // namespace

cudaError_t launch_ep_prepare(const EpPrepareArgs& a, cudaStream_t s) {
    ep_prepare_kernel<<<1, 64, 0, s>>>(a);
    return cudaGetLastError();
}

cudaError_t launch_dp_prepare(const DpPrepareArgs& a, cudaStream_t s) {
    dp_prepare_kernel<<<1, 64, 0, s>>>(a);
    return cudaGetLastError();
}

cudaError_t launch_dispatch_hist(const int32_t* topk_idx, int32_t* hist, int32_t* group_hist, int64_t T, int E, int k,
                                 int group_chunks, int ngroups, cudaStream_t s) {
    const int nchunk = (int)((T + kChunkTokens - 1) / kChunkTokens);
    if (nchunk == 0) return cudaSuccess;
    hist_kernel<<<nchunk, 256, 0, s>>>(topk_idx, hist, group_hist, T, E, k, nchunk, group_chunks, ngroups);
    return cudaGetLastError();
}

cudaError_t launch_dispatch_scan(const ScanArgs& a, cudaStream_t s) {
    scan_kernel<<<1, 1024, 0, s>>>(a);
    return cudaGetLastError();
}

cudaError_t launch_dispatch_scatter(const ScatterArgs& a, cudaStream_t s) {
    if (a.nchunk == 0) return cudaSuccess;
    // with row copies to do and fewer than two chunks per SM, each chunk's copies go to several CTAs
    int nsplit = 1;
    const bool copies = a.x_perm != nullptr || a.e_per_rank > 0;
    while (copies && nsplit < 4 && (int64_t)a.nchunk * nsplit < 2 * (int64_t)sm_count()) nsplit *= 2;
    return launch_kernel(scatter_kernel, dim3((unsigned)(a.nchunk * nsplit)), dim3(kScatterThreads), 0, s, a, nsplit);
}

}  // namespace moe
