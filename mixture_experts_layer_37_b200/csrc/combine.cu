// Weighted combine back to token order, load-balance statistics from a full
// probability matrix, and the bounded-wait self-test kernel.
//
// Combine: out[t] = sum_j w[t,j] * expert_j(x[t]) ("Hand-building a
// LLaMA4-MoE" (dpshk.com/news/5809432) §2.4; "MoE: gating, experts, load
// balancing, capacity factor" (dpshk.com/news/6005940) §3.1), over the kept
// assignments only, fp32 accumulation in ascending j.  One warp per token,
// 16-byte vector loads of the expert rows, no atomics.
//
// Statistics: f_e = n_e / (T*k), p_e = mean_t softmax[t,e],
// L_aux = alpha * E * sum_e f_e p_e (MoE-basics §2.3 and §3.1).
#include "internal.h"

namespace moe {
namespace {

template <bool BF16>
__global__ void __launch_bounds__(256) combine_kernel(CombineArgs a) {
    const int warps_per_cta = blockDim.x >> 5;
    const int lane = threadIdx.x & 31;
    const int64_t warp_g = (int64_t)blockIdx.x * warps_per_cta + (threadIdx.x >> 5);
    const int64_t nwarps = (int64_t)gridDim.x * warps_per_cta;
    constexpr int VEC = BF16 ? 8 : 4;  // elements per 16-byte vector
    const int nvec = a.d / VEC;
    for (int64_t t = warp_g; t < a.T; t += nwarps) {
        int s_l = -1;
        float w_l = 0.f;
        if (lane < a.k) {
            s_l = a.slot[t * a.k + lane];
            w_l = a.topk_w[t * a.k + lane];
        }
        int sj[kMaxTopK];
        float wj[kMaxTopK];
#pragma unroll
        for (int j = 0; j < kMaxTopK; ++j) {
            sj[j] = __shfl_sync(0xffffffffu, s_l, j);
            wj[j] = __shfl_sync(0xffffffffu, w_l, j);
        }
        for (int v = lane; v < nvec; v += 32) {
            float acc[VEC];
#pragma unroll
            for (int q = 0; q < VEC; ++q) acc[q] = 0.f;
#pragma unroll
            for (int j = 0; j < kMaxTopK; ++j) {
                if (j >= a.k) break;
                const int s = sj[j];
                const float w = wj[j];
                if (s < 0) continue;
                const uint4 y = reinterpret_cast<const uint4*>(a.y_perm)[(int64_t)s * nvec + v];
                if constexpr (BF16) {
                    const uint32_t ys[4] = {y.x, y.y, y.z, y.w};
#pragma unroll
                    for (int q = 0; q < 4; ++q) {
                        acc[2 * q] = fmaf(w, bf16_lo(ys[q]), acc[2 * q]);
                        acc[2 * q + 1] = fmaf(w, bf16_hi(ys[q]), acc[2 * q + 1]);
                    }
                } else {
                    acc[0] = fmaf(w, __uint_as_float(y.x), acc[0]);
                    acc[1] = fmaf(w, __uint_as_float(y.y), acc[1]);
                    acc[2] = fmaf(w, __uint_as_float(y.z), acc[2]);
                    acc[3] = fmaf(w, __uint_as_float(y.w), acc[3]);
                }
            }
            uint4 o;
            if constexpr (BF16) {
                o = make_uint4(pack_bf16x2(acc[0], acc[1]), pack_bf16x2(acc[2], acc[3]), pack_bf16x2(acc[4], acc[5]),
                               pack_bf16x2(acc[6], acc[7]));
            } else {
                o = make_uint4(__float_as_uint(acc[0]), __float_as_uint(acc[1]), __float_as_uint(acc[2]),
                               __float_as_uint(acc[3]));
            }
            reinterpret_cast<uint4*>(a.out)[t * nvec + v] = o;
        }
    }
}

// One CTA; p_e summed in fp64 in a fixed order (strided partial sums, then a
// fixed tree), so the result does not depend on scheduling.
__global__ void __launch_bounds__(1024) aux_probs_kernel(const int32_t* counts, const float* probs, float* f, float* p,
                                                         float* l_aux, int64_t T, int E, int k, float alpha) {
    __shared__ double sRed[1024];
    __shared__ double sP[kMaxExperts];
    const int tid = threadIdx.x;
    for (int e = 0; e < E; ++e) {
        double s = 0.0;
        for (int64_t t = tid; t < T; t += blockDim.x) s += (double)probs[t * E + e];
        sRed[tid] = s;
        __syncthreads();
        for (int o = blockDim.x / 2; o > 0; o >>= 1) {
            if (tid < o) sRed[tid] += sRed[tid + o];
            __syncthreads();
        }
        if (tid == 0) sP[e] = T > 0 ? sRed[0] / (double)T : 0.0;
        __syncthreads();
    }
    if (tid == 0) {
        double l = 0.0;
        for (int e = 0; e < E; ++e) {
            const double fe = T > 0 ? (double)counts[e] / ((double)T * k) : 0.0;
            f[e] = (float)fe;
            p[e] = (float)sP[e];
            l += fe * sP[e];
        }
        l_aux[0] = (float)((double)alpha * E * l);
    }
}

// Waits on an mbarrier phase that never completes and on a status-block flag
// that nothing sets, both bounded; each gives up and records a timeout.
__global__ void selftest_wait_kernel(DevStatus st) {
    __shared__ __align__(8) uint64_t bar;
    if (threadIdx.x == 0) {
        mbar_init(&bar, 1);
        fence_barrier_init();
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        if (!mbar_wait_bounded(&bar, 0, st.timeout_ns)) report_timeout(st, SITE_SELFTEST_MBAR);
        volatile uint32_t* flag = st.word + 2;
        const uint64_t t0 = globaltimer_ns();
        bool ok = false;
        while (true) {
            if (*flag != 0u) { ok = true; break; }
            if (globaltimer_ns() - t0 > st.timeout_ns) break;
            __nanosleep(1000);
        }
        if (!ok) report_timeout(st, SITE_SELFTEST_FLAG);
    }
}

}  // namespace

cudaError_t launch_combine(const CombineArgs& a, bool bf16, cudaStream_t s) {
    if (a.T == 0) return cudaSuccess;
    const int64_t blocks = min64((a.T + 7) / 8, (int64_t)sm_count() * 16);
    if (bf16)
        combine_kernel<true><<<(unsigned)blocks, 256, 0, s>>>(a);
    else
        combine_kernel<false><<<(unsigned)blocks, 256, 0, s>>>(a);
    return cudaGetLastError();
}

cudaError_t launch_aux_from_probs(const int32_t* counts, const float* probs, float* f, float* p, float* l_aux,
                                  int64_t T, int E, int k, float alpha, cudaStream_t s) {
    aux_probs_kernel<<<1, 1024, 0, s>>>(counts, probs, f, p, l_aux, T, E, k, alpha);
    return cudaGetLastError();
}

cudaError_t launch_selftest_wait(DevStatus st, cudaStream_t s) {
    selftest_wait_kernel<<<1, 32, 0, s>>>(st);
    return cudaGetLastError();
}

}  // namespace moe
