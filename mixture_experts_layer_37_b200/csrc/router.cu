// Router kernel: logits = x . W_r (+ bias), fp32 softmax over all experts,
// top-k on the logits (lower id first on ties), renormalised top-k weights,
// and per-chunk partial statistics (expert histogram, sum of probabilities)
// for the dispatch scan and the load-balance loss.
//
// Method: "MoE: gating, experts, load balancing, capacity factor"
// (dpshk.com/news/6005940) §2.1 (score = x . W_r, softmax) and §3.1 (top-k);
// "Llama-MoE架构解析" (coreui.cn/article/2610641) §3.1 (softmax -> top-k ->
// divide by the sum of the k weights).
//
// One CTA per chunk of kChunkTokens tokens.  bf16: each warp computes 16
// tokens x E logits with mma.sync m16n8k16 (fp32 accumulate).  x is streamed
// once from HBM with 16-byte loads; the (small) router weight is staged in
// shared memory, transposed, in K slabs.  The 32 reduction indices of one
// step are assigned to MMA fragment positions so that every thread loads 16
// contiguous bytes of x (the same assignment is used for W_r, so the product
// is unchanged).  f32: one thread per token, fp32 FMA.
#include <math.h>

#include "internal.h"

namespace moe {
namespace {

constexpr int kThreads = 128;          // 4 warps x 16 tokens = kChunkTokens
constexpr int kSlabK = 512;            // K slab of W_r held in shared memory (bf16)
constexpr int kSlabPad = 32;           // row padding (elements): conflict-free 16-byte reads
constexpr int kSlabStride = kSlabK + kSlabPad;
constexpr int kLStride = kMaxExperts + 1;
static_assert(kChunkTokens == 64, "router tiling assumes 64-token chunks");

__device__ __forceinline__ uint4 ldg_stream_128(const void* p) {
    uint4 v;
    asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "l"(p));
    return v;
}

__device__ __forceinline__ void mma_bf16_16816(float (&c)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                               uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
        "{%0, %1, %2, %3};"
        : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// Softmax / top-k / renormalisation / partial statistics for the chunk whose
// logits sit in sL[token][e].  Called by all threads of the CTA.
__device__ void router_finish(const RouterArgs& a, float* sL, int* sHist, bool add_bias) {
    const int tid = threadIdx.x;
    const int E = a.E, k = a.k;
    const int chunk = blockIdx.x;
    const int64_t t0 = (int64_t)chunk * kChunkTokens;
    const int ntok = (int)min64(kChunkTokens, a.T - t0);
    if (tid < E) sHist[tid] = 0;
    __syncthreads();
    if (tid < ntok) {
        const int64_t t = t0 + tid;
        float* row = sL + tid * kLStride;
        float m = -INFINITY;
        for (int e = 0; e < E; ++e) {
            float v = row[e];
            if (add_bias && a.bias) v += a.bias[e];
            row[e] = v;
            m = fmaxf(m, v);
            if (a.logits_out) a.logits_out[t * E + e] = v;
        }
        // top-k on the logits: repeated maximum over the unchosen experts;
        // strict '>' keeps the lower id on equal values.
        int sel_idx[kMaxTopK];
        uint64_t chosen = 0;
        for (int j = 0; j < k; ++j) {
            int best = -1;
            float bv = 0.f;
            for (int e = 0; e < E; ++e) {
                if ((chosen >> e) & 1ull) continue;
                const float v = row[e];
                if (best < 0 || v > bv) { best = e; bv = v; }
            }
            chosen |= 1ull << best;
            sel_idx[j] = best;
        }
        // softmax over all experts, fp32, ascending e
        float s = 0.f;
        for (int e = 0; e < E; ++e) {
            const float z = expf(row[e] - m);
            row[e] = z;
            s += z;
        }
        const float inv = 1.0f / s;
        for (int e = 0; e < E; ++e) {
            const float pe = row[e] * inv;
            row[e] = pe;
            if (a.probs_out) a.probs_out[t * E + e] = pe;
        }
        float ps = 0.f;
        for (int j = 0; j < k; ++j) ps += row[sel_idx[j]];
        for (int j = 0; j < k; ++j) {
            a.topk_idx[t * k + j] = sel_idx[j];
            a.topk_w[t * k + j] = row[sel_idx[j]] / ps;
            atomicAdd(&sHist[sel_idx[j]], 1);
        }
    }
    __syncthreads();
    if (tid < E) {
        double acc = 0.0;
        for (int i = 0; i < ntok; ++i) acc += (double)sL[i * kLStride + tid];
        a.psum[(int64_t)chunk * E + tid] = acc;
        a.hist[(int64_t)chunk * E + tid] = sHist[tid];
    }
}

__device__ void load_logits_in(const RouterArgs& a, float* sL) {
    const int64_t t0 = (int64_t)blockIdx.x * kChunkTokens;
    const int ntok = (int)min64(kChunkTokens, a.T - t0);
    for (int i = threadIdx.x; i < ntok * a.E; i += blockDim.x) {
        const int tok = i / a.E, e = i - tok * a.E;
        sL[tok * kLStride + e] = a.logits_in[(t0 + tok) * a.E + e];
    }
    __syncthreads();
}

template <int NT>  // experts padded to 8*NT
__global__ void __launch_bounds__(kThreads) router_bf16_kernel(RouterArgs a) {
    extern __shared__ __align__(16) uint8_t smem[];
    float* sL = reinterpret_cast<float*>(smem);                                       // [64][65]
    int* sHist = reinterpret_cast<int*>(smem + kChunkTokens * kLStride * 4);          // [64]
    __nv_bfloat16* sW = reinterpret_cast<__nv_bfloat16*>(smem + kChunkTokens * kLStride * 4 + 256);  // [8NT][stride]

    if (a.logits_in) {
        load_logits_in(a, sL);
        router_finish(a, sL, sHist, false);
        return;
    }
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int g = lane >> 2, c = lane & 3;
    const int E = a.E, d = a.d;
    const int64_t t0 = (int64_t)blockIdx.x * kChunkTokens;
    const int64_t r0 = t0 + warp * 16 + g, r1 = r0 + 8;
    const bool v0 = r0 < a.T, v1 = r1 < a.T;
    const __nv_bfloat16* X = static_cast<const __nv_bfloat16*>(a.x);
    const __nv_bfloat16* W = static_cast<const __nv_bfloat16*>(a.w_router);
    const __nv_bfloat16* x0 = X + (v0 ? r0 : 0) * (int64_t)d;
    const __nv_bfloat16* x1 = X + (v1 ? r1 : 0) * (int64_t)d;

    float acc[NT][4];
#pragma unroll
    for (int n = 0; n < NT; ++n) acc[n][0] = acc[n][1] = acc[n][2] = acc[n][3] = 0.f;

    const __nv_bfloat16 zero = __float2bfloat16(0.f);
    for (int k0 = 0; k0 < d; k0 += kSlabK) {
        const int ks = min(kSlabK, d - k0);  // multiple of 64
        __syncthreads();
        // stage W_r[k0:k0+ks, :] transposed: sW[e][kk]
        if ((E & 7) == 0) {
            for (int kk = tid; kk < ks; kk += kThreads) {
                const uint4* src = reinterpret_cast<const uint4*>(W + (int64_t)(k0 + kk) * E);
                for (int e8 = 0; e8 < E / 8; ++e8) {
                    const uint4 v = src[e8];
                    const __nv_bfloat16* h = reinterpret_cast<const __nv_bfloat16*>(&v);
#pragma unroll
                    for (int q = 0; q < 8; ++q) sW[(e8 * 8 + q) * kSlabStride + kk] = h[q];
                }
                for (int e = E; e < 8 * NT; ++e) sW[e * kSlabStride + kk] = zero;
            }
        } else {
            for (int kk = tid; kk < ks; kk += kThreads) {
                for (int e = 0; e < 8 * NT; ++e)
                    sW[e * kSlabStride + kk] = e < E ? W[(int64_t)(k0 + kk) * E + e] : zero;
            }
        }
        __syncthreads();
        for (int kk = 0; kk < ks; kk += 64) {
            uint4 xa[2], xb[2];
#pragma unroll
            for (int u = 0; u < 2; ++u) {
                xa[u] = v0 ? ldg_stream_128(x0 + k0 + kk + 32 * u + 8 * c) : make_uint4(0, 0, 0, 0);
                xb[u] = v1 ? ldg_stream_128(x1 + k0 + kk + 32 * u + 8 * c) : make_uint4(0, 0, 0, 0);
            }
#pragma unroll
            for (int u = 0; u < 2; ++u) {
#pragma unroll
                for (int n = 0; n < NT; ++n) {
                    const uint4 bw = *reinterpret_cast<const uint4*>(sW + (n * 8 + g) * kSlabStride + kk + 32 * u + 8 * c);
                    mma_bf16_16816(acc[n], xa[u].x, xb[u].x, xa[u].y, xb[u].y, bw.x, bw.y);
                    mma_bf16_16816(acc[n], xa[u].z, xb[u].z, xa[u].w, xb[u].w, bw.z, bw.w);
                }
            }
        }
    }
    // accumulators -> sL[token][e]
#pragma unroll
    for (int n = 0; n < NT; ++n) {
        const int e0 = n * 8 + 2 * c;
        float* ra = sL + (warp * 16 + g) * kLStride;
        float* rb = sL + (warp * 16 + g + 8) * kLStride;
        ra[e0] = acc[n][0];
        ra[e0 + 1] = acc[n][1];
        rb[e0] = acc[n][2];
        rb[e0 + 1] = acc[n][3];
    }
    __syncthreads();
    router_finish(a, sL, sHist, true);
}

template <int EP>  // experts padded to EP (8 or 64)
__global__ void __launch_bounds__(kThreads) router_f32_kernel(RouterArgs a) {
    extern __shared__ __align__(16) uint8_t smem[];
    float* sL = reinterpret_cast<float*>(smem);
    int* sHist = reinterpret_cast<int*>(smem + kChunkTokens * kLStride * 4);
    float* sW = reinterpret_cast<float*>(smem + kChunkTokens * kLStride * 4 + 256);  // [slab][EP]
    if (a.logits_in) {
        load_logits_in(a, sL);
        router_finish(a, sL, sHist, false);
        return;
    }
    constexpr int kSlab = 8192 / EP;  // 32 KB of fp32 weights per slab
    const int tid = threadIdx.x;
    const int E = a.E, d = a.d;
    const int64_t t = (int64_t)blockIdx.x * kChunkTokens + tid;
    const bool valid = tid < kChunkTokens && t < a.T;
    const float* X = static_cast<const float*>(a.x);
    const float* W = static_cast<const float*>(a.w_router);
    float acc[EP];
#pragma unroll
    for (int e = 0; e < EP; ++e) acc[e] = 0.f;
    for (int k0 = 0; k0 < d; k0 += kSlab) {
        const int ks = min(kSlab, d - k0);
        __syncthreads();
        for (int i = tid; i < ks * EP; i += kThreads) {
            const int kk = i / EP, e = i - kk * EP;
            sW[i] = e < E ? W[(int64_t)(k0 + kk) * E + e] : 0.f;
        }
        __syncthreads();
        if (valid) {
            const float* xr = X + t * d + k0;
            for (int kk = 0; kk < ks; ++kk) {
                const float xv = xr[kk];
#pragma unroll
                for (int e = 0; e < EP; ++e) acc[e] = fmaf(xv, sW[kk * EP + e], acc[e]);
            }
        }
    }
    if (valid) {
#pragma unroll
        for (int e = 0; e < EP; ++e)
            if (e < E) sL[tid * kLStride + e] = acc[e];
    }
    __syncthreads();
    router_finish(a, sL, sHist, true);
}

template <int NT>
cudaError_t launch_bf16_nt(const RouterArgs& a, int nchunk, cudaStream_t s) {
    const size_t smem = kChunkTokens * kLStride * 4 + 256 + (size_t)8 * NT * kSlabStride * 2;
    cudaError_t err = cudaFuncSetAttribute(router_bf16_kernel<NT>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (err != cudaSuccess) return err;
    router_bf16_kernel<NT><<<nchunk, kThreads, smem, s>>>(a);
    return cudaGetLastError();
}

template <int EP>
cudaError_t launch_f32_ep(const RouterArgs& a, int nchunk, cudaStream_t s) {
    const size_t smem = kChunkTokens * kLStride * 4 + 256 + (size_t)8192 * 4;
    cudaError_t err = cudaFuncSetAttribute(router_f32_kernel<EP>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (err != cudaSuccess) return err;
    router_f32_kernel<EP><<<nchunk, kThreads, smem, s>>>(a);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_router(const RouterArgs& a, bool bf16, cudaStream_t s) {
    const int nchunk = (int)((a.T + kChunkTokens - 1) / kChunkTokens);
    if (nchunk == 0) return cudaSuccess;
    if (bf16) {
        switch ((a.E + 7) / 8) {
            case 1: return launch_bf16_nt<1>(a, nchunk, s);
            case 2: return launch_bf16_nt<2>(a, nchunk, s);
            case 3: return launch_bf16_nt<3>(a, nchunk, s);
            case 4: return launch_bf16_nt<4>(a, nchunk, s);
            case 5: return launch_bf16_nt<5>(a, nchunk, s);
            case 6: return launch_bf16_nt<6>(a, nchunk, s);
            case 7: return launch_bf16_nt<7>(a, nchunk, s);
            default: return launch_bf16_nt<8>(a, nchunk, s);
        }
    }
    if (a.E <= 8) return launch_f32_ep<8>(a, nchunk, s);
    return launch_f32_ep<64>(a, nchunk, s);
}

}  // namespace moe
