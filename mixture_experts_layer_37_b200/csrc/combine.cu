// Weighted combine back to token order, load-balance statistics from a full
// probability matrix, and the bounded-wait self-test kernel.
//
// Combine: out[t] = sum_j w[t,j] * expert_j(x[t]) ("Hand-building a
// LLaMA4-MoE" (dpshk.com/news/5809432) §2.4; "MoE: gating, experts, load
// balancing, capacity factor" (dpshk.com/news/6005940) §3.1), over the kept
// assignments only, fp32 accumulation in ascending j, then plus each shared
// expert's output (LLaMA4-MoE §5.2: fixed experts in every token's
// computation), rounded once.  Without weights (topk_w null) the expert rows
// were already multiplied by their routing weights in the second GEMM's
// epilogue and the combine is their plain sum.  One warp per token, 16-byte
// vector loads of the expert rows, no atomics.
//
// Statistics: f_e = n_e / (T*k), p_e = mean_t softmax[t,e],
// L_aux = alpha * E * sum_e f_e p_e (MoE-basics §2.3 and §3.1).
#include "internal.h"

namespace moe {
namespace {

// EP: the expert rows are read from the output buffer of the rank holding
// each expert (peer memory over NVLink), so the gather back to token order is
// this step's all-to-all, fused with the weighted sum.
template <bool BF16, bool EP, int U>  // U: 16-byte vectors per lane per expert row (x2 rows in flight)
__global__ void __launch_bounds__(256, 8 / U) combine_kernel(CombineArgs a) {
    griddep_wait();  // the expert rows of the launches before
    griddep_launch_dependents();
    constexpr int VEC = BF16 ? 8 : 4;  // elements per 16-byte vector
    const int warps_per_cta = blockDim.x >> 5;
    const int lane = threadIdx.x & 31;
    const int64_t warp_g = (int64_t)blockIdx.x * warps_per_cta + (threadIdx.x >> 5);
    const int64_t nwarps = (int64_t)gridDim.x * warps_per_cta;
    const int nvec = a.d / VEC;
    const uint4* Y = reinterpret_cast<const uint4*>(a.y_perm);
    uint4* O = reinterpret_cast<uint4*>(a.out);
    for (int64_t t = warp_g; t < a.T; t += nwarps) {
        int s_l = -1;
        float w_l = 0.f;
        [[maybe_unused]] const uint4* y_l = Y;
        if (lane < a.k) {
            s_l = a.slot[t * a.k + lane];
            w_l = a.topk_w != nullptr ? a.topk_w[t * a.k + lane] : 1.0f;
            if constexpr (EP) {
                if (s_l >= 0) {
                    const int e = a.topk_idx[t * a.k + lane];
                    const int r = e >= 0 ? e / a.e_per_rank : kMaxRanks;
                    y_l = r < kMaxRanks ? static_cast<const uint4*>(a.y_src[r]) : nullptr;
                    if (y_l == nullptr || s_l >= a.row_limit) {
                        report_range(a.st, SITE_EP_COMBINE_ROW);
                        s_l = -1;
                    }
                }
            }
        }
        int sj[kMaxTopK];
        float wj[kMaxTopK];
#pragma unroll
        for (int j = 0; j < kMaxTopK; ++j) {
            sj[j] = __shfl_sync(0xffffffffu, s_l, j);
            wj[j] = __shfl_sync(0xffffffffu, w_l, j);
        }
        [[maybe_unused]] const uint4* yj[EP ? kMaxTopK : 1];
        if constexpr (EP) {
#pragma unroll
            for (int j = 0; j < kMaxTopK; ++j)
                yj[j] = reinterpret_cast<const uint4*>(
                    __shfl_sync(0xffffffffu, reinterpret_cast<unsigned long long>(y_l), j));
        }
        for (int v0 = lane; v0 < nvec; v0 += 32 * U) {
            float acc[U][VEC];
#pragma unroll
            for (int u = 0; u < U; ++u)
#pragma unroll
                for (int q = 0; q < VEC; ++q) acc[u][q] = 0.f;
            // experts in pairs: 2*U loads in flight, then the FMAs in ascending j
            for (int j = 0; j < a.k; j += 2) {
                const int s0 = sj[j];
                const int s1 = (j + 1 < a.k) ? sj[j + 1] : -1;
                uint4 y0[U], y1[U];
                if constexpr (EP) {
                    const uint4* Y0 = yj[j];
                    const uint4* Y1 = (j + 1 < a.k) ? yj[j + 1] : Y;
#pragma unroll
                    for (int u = 0; u < U; ++u) {
                        const bool in = v0 + 32 * u < nvec;
                        if (in && s0 >= 0) y0[u] = Y0[(int64_t)s0 * nvec + v0 + 32 * u];
                        if (in && s1 >= 0) y1[u] = Y1[(int64_t)s1 * nvec + v0 + 32 * u];
                    }
                } else {
#pragma unroll
                    for (int u = 0; u < U; ++u) {
                        const bool in = v0 + 32 * u < nvec;
                        if (in && s0 >= 0) y0[u] = Y[(int64_t)s0 * nvec + v0 + 32 * u];
                        if (in && s1 >= 0) y1[u] = Y[(int64_t)s1 * nvec + v0 + 32 * u];
                    }
                }
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    const int s = h ? s1 : s0;
                    if (s < 0) continue;
                    const float w = h ? wj[j + 1] : wj[j];
#pragma unroll
                    for (int u = 0; u < U; ++u) {
                        if (v0 + 32 * u >= nvec) continue;
                        const uint4 yv = h ? y1[u] : y0[u];
                        if constexpr (BF16) {
                            const uint32_t ys[4] = {yv.x, yv.y, yv.z, yv.w};
#pragma unroll
                            for (int q = 0; q < 4; ++q) {
                                acc[u][2 * q] = fmaf(w, bf16_lo(ys[q]), acc[u][2 * q]);
                                acc[u][2 * q + 1] = fmaf(w, bf16_hi(ys[q]), acc[u][2 * q + 1]);
                            }
                        } else {
                            acc[u][0] = fmaf(w, __uint_as_float(yv.x), acc[u][0]);
                            acc[u][1] = fmaf(w, __uint_as_float(yv.y), acc[u][1]);
                            acc[u][2] = fmaf(w, __uint_as_float(yv.z), acc[u][2]);
                            acc[u][3] = fmaf(w, __uint_as_float(yv.w), acc[u][3]);
                        }
                    }
                }
            }
            // shared experts: every token, weight 1, after the routed terms, in order
            for (int sh = 0; sh < a.n_shared; ++sh) {
                const uint4* YS = reinterpret_cast<const uint4*>(a.y_shared) + ((int64_t)sh * a.T + t) * nvec;
                uint4 ysv[U];
#pragma unroll
                for (int u = 0; u < U; ++u)
                    if (v0 + 32 * u < nvec) ysv[u] = YS[v0 + 32 * u];
#pragma unroll
                for (int u = 0; u < U; ++u) {
                    if (v0 + 32 * u >= nvec) continue;
                    const uint4 yv = ysv[u];
                    if constexpr (BF16) {
                        const uint32_t ys[4] = {yv.x, yv.y, yv.z, yv.w};
#pragma unroll
                        for (int q = 0; q < 4; ++q) {
                            acc[u][2 * q] += bf16_lo(ys[q]);
                            acc[u][2 * q + 1] += bf16_hi(ys[q]);
                        }
                    } else {
                        acc[u][0] += __uint_as_float(yv.x);
                        acc[u][1] += __uint_as_float(yv.y);
                        acc[u][2] += __uint_as_float(yv.z);
                        acc[u][3] += __uint_as_float(yv.w);
                    }
                }
            }
#pragma unroll
            for (int u = 0; u < U; ++u) {
                if (v0 + 32 * u >= nvec) continue;
                uint4 o;
                if constexpr (BF16) {
                    o = make_uint4(pack_bf16x2(acc[u][0], acc[u][1]), pack_bf16x2(acc[u][2], acc[u][3]),
                                   pack_bf16x2(acc[u][4], acc[u][5]), pack_bf16x2(acc[u][6], acc[u][7]));
                } else {
                    o = make_uint4(__float_as_uint(acc[u][0]), __float_as_uint(acc[u][1]), __float_as_uint(acc[u][2]),
                                   __float_as_uint(acc[u][3]));
                }
                O[t * nvec + v0 + 32 * u] = o;
            }
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

template <int U>
cudaError_t launch_combine_u(const CombineArgs& a, bool bf16, int64_t blocks, cudaStream_t s) {
    const bool ep = a.e_per_rank > 0;
    const dim3 grid((unsigned)blocks), block(256);
    if (bf16 && ep) return launch_kernel(combine_kernel<true, true, U>, grid, block, 0, s, a);
    if (bf16) return launch_kernel(combine_kernel<true, false, U>, grid, block, 0, s, a);
    if (ep) return launch_kernel(combine_kernel<false, true, U>, grid, block, 0, s, a);
    return launch_kernel(combine_kernel<false, false, U>, grid, block, 0, s, a);
}

}  // namespace

// Rows in passes of 128 16-byte vectors (4 per lane, both rows of an expert
// pair in flight), two CTAs per SM.  (Whole 2048-wide rows per pass, 8
// vectors per lane, were measured slower: half the warps fit per SM.)
cudaError_t launch_combine(const CombineArgs& a, bool bf16, cudaStream_t s) {
    if (a.T == 0) return cudaSuccess;
    return launch_combine_u<4>(a, bf16, min64((a.T + 7) / 8, (int64_t)sm_count() * 8), s);
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
