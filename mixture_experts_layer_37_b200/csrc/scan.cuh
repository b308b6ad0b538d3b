// Dispatch scan + load-balance statistics, as a block-level device function
// shared by the standalone scan kernel and the routers' last CTA.
//
// For each expert e: exclusive scan of the per-group counts over groups (the
// rank base of every group of chunks; the scatter adds the counts of the
// earlier chunks inside the group), the total n_e (counts, before the
// capacity cut), and the sum of the partial probability sums.  Then the kept
// offsets offsets[e] = sum_{e'<e} min(n_e', cap) ("MoE: gating, experts, load
// balancing, capacity factor" (dpshk.com/news/6005940) §2.4; groups per
// expert as in "Hand-building a LLaMA4-MoE" (dpshk.com/news/5809432) §2.4)
// and f_e = n_e/(T*k), p_e = (1/T) sum_t p[t,e], L_aux = alpha*E*sum_e f_e p_e
// (MoE-basics §2.3, §3.1), with T the number of real tokens when padding is
// masked (LLaMA4-MoE §4.1).
//
// The per-group counts were added with integer atomics (exact in any order);
// every floating-point sum has a fixed order, so results do not depend on
// scheduling.  The counters the producers accumulated (group counts, real
// tokens) are returned to zero here for the next launch.
#pragma once

#include "internal.h"

namespace moe {

__device__ __forceinline__ int warp_inclusive_scan(int v, int lane) {
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int n = __shfl_up_sync(0xffffffffu, v, o);
        if (lane >= o) v += n;
    }
    return v;
}

// Copies n values global -> shared, eight loads in flight per thread.
template <class T>
__device__ __forceinline__ void stage_to_smem(T* dst, const T* src, int n) {
    for (int i0 = threadIdx.x; i0 < n; i0 += 8 * blockDim.x) {
        T v[8];
#pragma unroll
        for (int u = 0; u < 8; ++u) {
            const int i = i0 + u * blockDim.x;
            v[u] = i < n ? __ldcg(src + i) : T(0);
        }
#pragma unroll
        for (int u = 0; u < 8; ++u) {
            const int i = i0 + u * blockDim.x;
            if (i < n) dst[i] = v[u];
        }
    }
}

// All threads of the CTA call this; sCount / sP are shared arrays of kMaxExperts.
// Inputs written by other CTAs of the same grid are read with .cg loads.
// With `scratch` (shared memory) large enough for the group counts and the
// probability sums, every input is first copied there in a few round trips,
// and the per-expert work reads shared memory.  The experts are handled side by
// side: P threads per expert (the largest power of two with P*E threads in the
// block, at most 32) sum the expert's probability-sum columns (thread j takes
// columns j, j+P, ..., then a fixed xor tree over the P threads), and the first
// of them scans the expert's groups in order.
__device__ __forceinline__ void scan_block(const ScanArgs& a, int* sCount, double* sP, void* scratch = nullptr,
                                           int scratch_bytes = 0) {
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31, nthreads = blockDim.x;
    // every argument in a register: no reloads from the parameter block after the stores
    const int E = a.E, ng = a.ngroups, k = a.k, cap = a.cap;
    const int64_t T = a.T;
    const int npsum = a.psum != nullptr ? a.npsum : 0;
    int32_t* __restrict__ group_hist = a.group_hist;
    int32_t* __restrict__ group_base = a.group_base;
    double* __restrict__ psum_total = a.psum_total;
    int32_t* __restrict__ real_counter = a.real_counter;
    const bool staged = scratch != nullptr && (int64_t)E * npsum * 8 + (int64_t)E * ng * 4 <= scratch_bytes;
    const double* psum = a.psum;
    const int32_t* ghist = group_hist;
    if (staged) {
        double* sPs = static_cast<double*>(scratch);
        int32_t* sG = reinterpret_cast<int32_t*>(sPs + (int64_t)E * npsum);
        stage_to_smem(sG, group_hist, E * ng);
        if (npsum > 0) stage_to_smem(sPs, a.psum, E * npsum);
        __syncthreads();
        for (int i = tid; i < E * ng; i += nthreads) group_hist[i] = 0;
        psum = sPs;
        ghist = sG;
    }
    int P = 32;
    while (P > 1 && P * E > nthreads) P >>= 1;
    const int ex = tid / P, jx = tid - (tid / P) * P;  // this thread's expert and its place in the expert's group
    double ps = 0.0;
    if (ex < E && npsum > 0) {
        const double* pp = psum + (int64_t)ex * npsum;
        for (int i = jx; i < npsum; i += P) ps += staged ? pp[i] : __ldcg(pp + i);
    }
    // P lanes of one warp per expert (P divides 32): a fixed xor tree
    for (int o = P >> 1; o > 0; o >>= 1) ps += __shfl_xor_sync(0xffffffffu, ps, o);
    if (ex < E && jx == 0) {
        // group bases and the expert's total, in group order (integer sums); the
        // group counts go back to zero
        const int32_t* gh = ghist + (int64_t)ex * ng;
        int32_t* gb = group_base + (int64_t)ex * ng;
        int run = 0;
        for (int g0 = 0; g0 < ng; g0 += 8) {
            int v[8];
#pragma unroll
            for (int u = 0; u < 8; ++u) v[u] = g0 + u < ng ? (staged ? gh[g0 + u] : __ldcg(gh + g0 + u)) : 0;
#pragma unroll
            for (int u = 0; u < 8; ++u)
                if (g0 + u < ng) {
                    gb[g0 + u] = run;
                    run += v[u];
                    if (!staged) group_hist[(int64_t)ex * ng + g0 + u] = 0;
                }
        }
        sCount[ex] = run;
        sP[ex] = ps;  // divided by the real-token count below
        if (psum_total != nullptr) psum_total[ex] = ps;
    }
    __syncthreads();
    // two warps side by side: warp 0 the kept offsets, warp 1 (warp 0 in a one-warp block) the statistics,
    // whose fp64 divisions are the longest chain left
    const int stats_warp = nthreads > 32 ? 1 : 0;
    if (warp == stats_warp && a.psum != nullptr) {
        float* __restrict__ fo = a.f;
        float* __restrict__ po = a.p;
        float* __restrict__ lo = a.l_aux;
        // the real-token count is final: every producer added to it before the scan started
        const int64_t t_real = real_counter != nullptr ? (int64_t)__ldcg(real_counter) : T;
        // statistics in a fixed order: lane-strided partial sums, then a fixed xor tree
        double l = 0.0;
        for (int e = lane; e < E; e += 32) {
            const double f = t_real > 0 ? (double)sCount[e] / ((double)t_real * k) : 0.0;
            const double pe = t_real > 0 ? sP[e] / (double)t_real : 0.0;
            if (fo) fo[e] = (float)f;
            if (po) po[e] = (float)pe;
            l += f * pe;
        }
        double tot = l;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) tot += __shfl_xor_sync(0xffffffffu, tot, o);
        if (lane == 0 && lo) lo[0] = (float)((double)a.alpha * E * tot);
    }
    if (warp == 0) {
        int32_t* __restrict__ counts = a.counts;
        int32_t* __restrict__ offsets = a.offsets;
        int32_t* __restrict__ t_real_out = a.t_real_out;
        int32_t* __restrict__ shared_off = a.shared_off;
        // real tokens: every token, or the router's count of unmasked tokens
        int64_t t_real = T;
        if (real_counter != nullptr) t_real = __ldcg(real_counter);
        if (lane == 0 && t_real_out != nullptr) t_real_out[0] = (int32_t)t_real;
        if (lane == 0 && shared_off != nullptr) {
            shared_off[0] = 0;
            shared_off[1] = (int32_t)T;
        }
        // kept offsets: exclusive scan of min(n_e, cap) over experts, 32 at a time
        int run = 0;
        for (int e0 = 0; e0 < E; e0 += 32) {
            const int e = e0 + lane;
            const int kept = e < E ? min(sCount[e], cap) : 0;
            const int incl = warp_inclusive_scan(kept, lane);
            if (e < E) {
                counts[e] = sCount[e];
                offsets[e] = run + incl - kept;
            }
            run += __shfl_sync(0xffffffffu, incl, 31);
        }
        if (lane == 0) offsets[E] = run;
    }
    // the real-token counter goes back to zero once both warps have read it
    __syncthreads();
    if (tid == 0 && real_counter != nullptr) *real_counter = 0;
}

// The rank base of chunk `chunk` for expert e: its group's base plus the
// chunk counts of the earlier chunks of the same group (integer sums, exact),
// read 32 at a time with every load of a batch in flight together.
__device__ __forceinline__ int chunk_base_of(const int32_t* __restrict__ hist, const int32_t* __restrict__ group_base,
                                             int e, int chunk, int nchunk, int group_chunks, int ngroups) {
    const int g = chunk / group_chunks;
    int run = group_base[(int64_t)e * ngroups + g];
    const int32_t* h = hist + (int64_t)e * nchunk;
    for (int c0 = g * group_chunks; c0 < chunk; c0 += 32) {
        int v[32];
#pragma unroll
        for (int i = 0; i < 32; ++i) v[i] = c0 + i < chunk ? h[c0 + i] : 0;
#pragma unroll
        for (int i = 0; i < 32; ++i) run += v[i];
    }
    return run;
}

}  // namespace moe
