// Dispatch scan + load-balance statistics, as a block-level device function
// shared by the standalone scan kernel and the router's last CTA.
//
// For each expert e: exclusive scan of the per-chunk histogram over chunks
// (the rank base of every chunk), the total n_e (counts, before the capacity
// cut), and the sum of the per-chunk probability sums.  Then, in one thread,
// the kept offsets offsets[e] = sum_{e'<e} min(n_e', cap) ("MoE: gating,
// experts, load balancing, capacity factor" (dpshk.com/news/6005940) §2.4;
// groups per expert as in "Hand-building a LLaMA4-MoE" (dpshk.com/news/
// 5809432) §2.4) and f_e = n_e/(T*k), p_e = (1/T) sum_t p[t,e],
// L_aux = alpha*E*sum_e f_e p_e (MoE-basics §2.3, §3.1), with T the number of
// real tokens when padding is masked (LLaMA4-MoE §4.1).
// Every sum has a fixed order, so results do not depend on scheduling.
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

// All threads of the CTA call this; sCount / sP are shared arrays of kMaxExperts.
// Partials are read with .cg loads (they may come from other CTAs of the same
// grid); each lane first loads all of its chunks, so one round trip covers up
// to 32 * kScanRegs chunks.
constexpr int kScanRegs = 8;
__device__ __forceinline__ void scan_block(const ScanArgs& a, int* sCount, double* sP) {
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31, nwarps = blockDim.x >> 5;
    const int E = a.E, nc = a.nchunk;
    for (int e = warp; e < E; e += nwarps) {
        const int32_t* h = a.hist + (int64_t)e * nc;
        int32_t* cb = a.chunk_base + (int64_t)e * nc;
        const double* pp = a.psum != nullptr ? a.psum + (int64_t)e * nc : nullptr;
        int run = 0;
        double ps = 0.0;
        // lane owns chunks [c0 + lane*per, c0 + (lane+1)*per) of each 32*per span
        for (int c0 = 0; c0 < nc; c0 += 32 * kScanRegs) {
            const int per = min(kScanRegs, (nc - c0 + 31) / 32);
            const int cbeg = c0 + lane * per;
            int v[kScanRegs];
            double q[kScanRegs];
#pragma unroll
            for (int i = 0; i < kScanRegs; ++i) {
                const int c = cbeg + i;
                const bool in = i < per && c < nc;
                v[i] = in ? __ldcg(h + c) : 0;
                q[i] = (in && pp != nullptr) ? __ldcg(pp + c) : 0.0;
            }
            int local = 0;
#pragma unroll
            for (int i = 0; i < kScanRegs; ++i) local += v[i];
            const int incl = warp_inclusive_scan(local, lane);
            int base = run + incl - local;
#pragma unroll
            for (int i = 0; i < kScanRegs; ++i) {
                const int c = cbeg + i;
                if (i < per && c < nc) cb[c] = base;
                base += v[i];
                ps += q[i];
            }
            run += __shfl_sync(0xffffffffu, incl, 31);
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) ps += __shfl_xor_sync(0xffffffffu, ps, o);
        if (lane == 0) {
            sCount[e] = run;
            sP[e] = pp != nullptr ? ps : 0.0;  // divided by the real-token count below
            if (a.psum_total != nullptr) a.psum_total[e] = ps;
        }
    }
    __syncthreads();
    if (warp == 0) {
        // real tokens: every token, or the per-chunk counts of unmasked tokens summed in chunk order
        int64_t t_real = a.T;
        if (a.nreal != nullptr) {
            int64_t run = 0;
            for (int c0 = 0; c0 < nc; c0 += 32) {
                int v = c0 + lane < nc ? __ldcg(a.nreal + c0 + lane) : 0;
#pragma unroll
                for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
                run += v;
            }
            t_real = run;
        }
        if (lane == 0 && a.t_real_out != nullptr) a.t_real_out[0] = (int32_t)t_real;
        if (lane == 0 && a.shared_off != nullptr) {
            a.shared_off[0] = 0;
            a.shared_off[1] = (int32_t)a.T;
        }
        // kept offsets: exclusive scan of min(n_e, cap) over experts, 32 at a time
        int run = 0;
        for (int e0 = 0; e0 < E; e0 += 32) {
            const int e = e0 + lane;
            const int kept = e < E ? min(sCount[e], a.cap) : 0;
            const int incl = warp_inclusive_scan(kept, lane);
            if (e < E) {
                a.counts[e] = sCount[e];
                a.offsets[e] = run + incl - kept;
            }
            run += __shfl_sync(0xffffffffu, incl, 31);
        }
        if (lane == 0) a.offsets[E] = run;
        if (a.psum != nullptr) {
            // statistics in a fixed order: lane-strided partial sums, then lane 0 adds them in lane order
            double l = 0.0;
            for (int e = lane; e < E; e += 32) {
                const double f = t_real > 0 ? (double)sCount[e] / ((double)t_real * a.k) : 0.0;
                const double pe = t_real > 0 ? sP[e] / (double)t_real : 0.0;
                if (a.f) a.f[e] = (float)f;
                if (a.p) a.p[e] = (float)pe;
                l += f * pe;
            }
            double tot = 0.0;
            for (int i = 0; i < 32; ++i) tot += __shfl_sync(0xffffffffu, l, i);
            if (lane == 0 && a.l_aux) a.l_aux[0] = (float)((double)a.alpha * E * tot);
        }
    }
}

}  // namespace moe
