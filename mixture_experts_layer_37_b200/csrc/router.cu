// Router kernel: logits = x . W_r (+ bias), fp32 softmax over all experts,
// top-k on the logits (lower id first on ties), renormalised top-k weights,
// and per-chunk partial statistics (expert histogram, sum of probabilities);
// in moe_forward the last CTA to finish also runs the dispatch scan and the
// load-balance statistics.
//
// Method: "MoE: gating, experts, load balancing, capacity factor"
// (dpshk.com/news/6005940) §2.1 (score = x . W_r, softmax) and §3.1 (top-k);
// "Llama-MoE架构解析" (coreui.cn/article/2610641) §3.1 (softmax -> top-k ->
// divide by the sum of the k weights).
//
// bf16: one CTA of 8 warps per `tpc` tokens (32 or 64: enough CTAs to
// fill the GPU, and enough tokens per CTA that re-reading the router weight
// per CTA stays small next to the x stream).  The warps form tpc/16 token
// groups x 128/tpc K-splits; each token's logits are always the same
// fixed-order sum of four K partial sums, so they do not depend on the batch.  Each warp streams its x rows once from HBM with
// 16-byte loads, four 32-column blocks (8 loads per lane) in flight per batch
// and two CTAs per SM, and multiplies on the tensor cores with mma.sync m16n8k16 (bf16 in,
// fp32 accumulate).  The router weight [d, E] is copied into shared memory as
// it lies in HBM (16-byte rows per 8 experts) in K slabs, and ldmatrix.trans
// turns it into MMA B fragments.  Inside each MMA the 32 reduction indices of
// a step are assigned so that a thread's A fragment is 16 contiguous bytes of
// x; the ldmatrix row addresses apply the same assignment to W_r, so the
// product is unchanged.  Slab rows are stored rotated within 32-row blocks and
// padded to an odd number of 16-byte units, so the eight rows of every
// ldmatrix phase fall in eight distinct bank groups.  K-split partial sums
// are added in a fixed order.  f32: one thread per token, fp32 FMA.
#include <math.h>

#include "moe.h"
#include "scan.cuh"
#include "warp_mma.cuh"

namespace moe {
namespace {

constexpr int kThreads = 256;
constexpr int kLStride = kMaxExperts + 1;
constexpr int kSlabBytes = 32 * 1024;  // one of the two router-weight slab buffers
constexpr int kMaxTpc = 64;
constexpr int kSplits = 4;  // K partial sums per token, always (batch-invariant logits)
constexpr int kBatch = 8;  // 32-column blocks of x loaded per batch

__device__ __forceinline__ uint4 ldg_stream_128(const void* p) {
    uint4 v;
    asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "l"(p));
    return v;
}

// Row position of slab row kk: rotated inside its 32-row block.
__device__ __forceinline__ int slab_phys_row(int kk) {
    const int a = (kk >> 3) & 3, b = kk & 7;
    return (kk & ~31) + 8 * a + ((b + 2 * a) & 7);
}

// Softmax / top-k / renormalisation / per-chunk partial statistics for the
// CTA's tokens, whose logits sit in sL[token][e]; then, when fusing, the last
// CTA to arrive runs the dispatch scan.  All threads of the CTA call it.
__device__ void router_finish(const RouterArgs& a, float* sL, int* sHist, bool add_bias) {
    const int tid = threadIdx.x;
    const int E = a.E, k = a.k;
    const int64_t t0 = (int64_t)blockIdx.x * a.tpc;
    const int ntok = (int)min64(a.tpc, a.T - t0);
    const int nchk = (ntok + kChunkTokens - 1) / kChunkTokens;
    const int chunk0 = (int)(t0 / kChunkTokens);
    for (int i = tid; i < nchk * kMaxExperts; i += blockDim.x) sHist[i] = 0;
    __syncthreads();
    if (tid < ntok) {
        const int64_t t = t0 + tid;
        const bool real = a.mask == nullptr || a.mask[t] != 0;  // padding selects nothing
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
                if (best < 0 || v > bv) {
                    best = e;
                    bv = v;
                }
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
        int* hrow = sHist + (tid / kChunkTokens) * kMaxExperts;
        for (int j = 0; j < k; ++j) {
            a.topk_idx[t * k + j] = real ? sel_idx[j] : -1;
            a.topk_w[t * k + j] = real ? row[sel_idx[j]] / ps : 0.f;
            if (real) atomicAdd(&hrow[sel_idx[j]], 1);
        }
        if (!real)
            for (int e = 0; e < E; ++e) row[e] = 0.f;  // out of the probability sums
    }
    __syncthreads();
    // per-chunk statistics: probability sums (psum columns are chunks here),
    // expert counts, and the counts added into the chunk's group
    for (int i = tid; i < nchk * E; i += blockDim.x) {
        const int cl = i / E, e = i - cl * E;
        const int i0 = cl * kChunkTokens, i1 = min(ntok, i0 + kChunkTokens);
        double acc = 0.0;
        for (int r = i0; r < i1; ++r) acc += (double)sL[r * kLStride + e];
        const int chunk = chunk0 + cl;
        a.psum[(int64_t)e * a.nchunk + chunk] = acc;
        const int n = sHist[cl * kMaxExperts + e];
        a.hist[(int64_t)e * a.nchunk + chunk] = n;
        if (n && a.group_hist) atomicAdd(a.group_hist + (int64_t)e * a.ngroups + chunk / a.group_chunks, n);
    }
    if (a.mask != nullptr && a.real_counter != nullptr && tid == 0) {
        int n = 0;
        for (int64_t t = t0; t < t0 + ntok; ++t) n += a.mask[t] != 0;
        if (n) atomicAdd(a.real_counter, n);
    }
    if (!a.fuse_scan) return;
    // last-CTA-done: the CTA that completes the arrival count runs the scan on
    // everyone's partials (fences order the partial stores before the count)
    __shared__ int sLast;
    __threadfence();
    __syncthreads();
    if (tid == 0) sLast = (atomicAdd(a.counter, 1u) == (unsigned)gridDim.x - 1u) ? 1 : 0;
    __syncthreads();
    if (!sLast) return;
    __threadfence();
    __shared__ int sCount[kMaxExperts];
    __shared__ double sP[kMaxExperts];
    scan_block(a.scan, sCount, sP);
    if (tid == 0) *a.counter = 0u;
}

__device__ void load_logits_in(const RouterArgs& a, float* sL) {
    const int64_t t0 = (int64_t)blockIdx.x * a.tpc;
    const int ntok = (int)min64(a.tpc, a.T - t0);
    for (int i = threadIdx.x; i < ntok * a.E; i += blockDim.x) {
        const int tok = i / a.E, e = i - tok * a.E;
        sL[tok * kLStride + e] = a.logits_in[(t0 + tok) * a.E + e];
    }
    __syncthreads();
}

template <int NT>
struct SlabGeom {
    static constexpr int kUnits = (NT & 1) ? NT : NT + 1;   // odd row pitch in 16-byte units
    static constexpr int kPitch = 16 * kUnits;
    static constexpr int kRows = (kSlabBytes / kPitch) / 128 * 128;
    static constexpr int kPartBytes = kSplits * kMaxTpc * 8 * NT * 4;  // [4][tpc][EP] floats
};

// Bytes of the shared region that holds the two weight slab buffers, and
// after the K loop the K-split partial logits.
template <int NT>
__host__ __device__ __forceinline__ int union_bytes_for(int d) {
    const int slab = d <= SlabGeom<NT>::kRows ? ((d * SlabGeom<NT>::kPitch + 127) & ~127) : 2 * kSlabBytes;
    return slab > SlabGeom<NT>::kPartBytes ? slab : SlabGeom<NT>::kPartBytes;
}

__host__ __device__ __forceinline__ int tail_bytes_for(int tpc) {
    return tpc * kLStride * 4 + (kMaxTpc / kChunkTokens) * kMaxExperts * 4;
}

template <int NT, int TPC>  // experts padded to 8*NT; TPC tokens per CTA (32 or 64)
__global__ void __launch_bounds__(kThreads, 2) router_bf16_kernel(RouterArgs a) {
    using G = SlabGeom<NT>;
    constexpr int EP = 8 * NT;
    extern __shared__ __align__(128) uint8_t smem[];
    uint8_t* sW = smem;                                                // slab, then partials
    float* sPart = reinterpret_cast<float*>(smem);                     // [nsplit][tpc][EP]
    float* sL = reinterpret_cast<float*>(smem + union_bytes_for<NT>(a.d));  // [tpc][65]
    int* sHist = reinterpret_cast<int*>(sL + a.tpc * kLStride);        // [tpc/32][64]

    if (a.logits_in) {
        load_logits_in(a, sL);
        router_finish(a, sL, sHist, false);
        return;
    }
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int g = lane >> 2, c = lane & 3;
    constexpr int ngroups = TPC / 16, nsplit = 8 / ngroups, kSets = kSplits / nsplit;
    const int tg = warp % ngroups, ksplit = warp / ngroups;
    const int E = a.E, d = a.d;
    const int64_t t0 = (int64_t)blockIdx.x * a.tpc;
    const int64_t r0 = t0 + tg * 16 + g, r1 = r0 + 8;
    const bool v0 = r0 < a.T, v1 = r1 < a.T;
    const __nv_bfloat16* X = static_cast<const __nv_bfloat16*>(a.x);
    const __nv_bfloat16* W = static_cast<const __nv_bfloat16*>(a.w_router);
    const __nv_bfloat16* x0 = X + (v0 ? r0 : 0) * (int64_t)d + 8 * c;
    const __nv_bfloat16* x1 = X + (v1 ? r1 : 0) * (int64_t)d + 8 * c;
    // ldmatrix lane j = lane/8 (fragment), r = lane%8 (matrix row): logical
    // k = 8*(r/2) + 2j + (r%2) of the 32-row block, stored at its rotated row.
    const int lj = lane >> 3, lr = lane & 7;
    const int la = lr >> 1, lb = 2 * lj + (lr & 1);
    const uint32_t lds_base = smem_u32(sW) + (uint32_t)((8 * la + ((lb + 2 * la) & 7)) * G::kPitch);

    // Every token's logits are the fixed-order sum of kSplits partial sums,
    // partial s accumulating the 32-column blocks b with b % 4 == s in
    // ascending order; a warp owns partials ksplit + nsplit*j.  The result is
    // therefore independent of how tokens are grouped into CTAs (batch size).
    float acc[kSets][NT][4];
#pragma unroll
    for (int j = 0; j < kSets; ++j)
#pragma unroll
        for (int n = 0; n < NT; ++n) acc[j][n][0] = acc[j][n][1] = acc[j][n][2] = acc[j][n][3] = 0.f;

    // Router weight slabs: copied (cp.async, 16-byte units, no register round
    // trip) into two alternating buffers, slab i+1 in flight while slab i is
    // multiplied.
    const bool vec_rows = (E & 7) == 0;
    const int nslabs = (d + G::kRows - 1) / G::kRows;
    auto stage = [&](int slab) {
        const int k0s = slab * G::kRows;
        const int ks = min(G::kRows, d - k0s);  // multiple of 64
        uint8_t* dst = sW + (slab & 1) * kSlabBytes;
        const int nunits = ks * NT;
        for (int i = tid; i < nunits; i += kThreads) {
            const int kk = i / NT, q = i - kk * NT;
            uint8_t* sd = dst + slab_phys_row(kk) * G::kPitch + 16 * q;
            if (vec_rows) {
                cp_async_16(sd, W + (int64_t)(k0s + kk) * E + 8 * q);
            } else {
                __nv_bfloat16 h[8];
#pragma unroll
                for (int w = 0; w < 8; ++w) {
                    const int e = 8 * q + w;
                    h[w] = e < E ? W[(int64_t)(k0s + kk) * E + e] : __float2bfloat16(0.f);
                }
                *reinterpret_cast<uint4*>(sd) = *reinterpret_cast<const uint4*>(h);
            }
        }
        cp_async_commit();
    };
    stage(0);
    for (int slab = 0; slab < nslabs; ++slab) {
        const int k0 = slab * G::kRows;
        const int ks = min(G::kRows, d - k0);
        if (slab + 1 < nslabs)
            stage(slab + 1);
        else
            cp_async_commit();  // empty group: keeps "all but the newest group" meaning slab's copies
        // this warp's 32-row blocks of the slab: ksplit, ksplit + nsplit, ...
        const int nblk = ks / 32;
        uint4 xa[kBatch], xb[kBatch];
        auto load_batch = [&](int b0) {
#pragma unroll
            for (int u = 0; u < kBatch; ++u) {
                const int blk = b0 + u * nsplit;
                const int kx = k0 + 32 * blk;
                xa[u] = (blk < nblk && v0) ? ldg_stream_128(x0 + kx) : make_uint4(0, 0, 0, 0);
                xb[u] = (blk < nblk && v1) ? ldg_stream_128(x1 + kx) : make_uint4(0, 0, 0, 0);
            }
        };
        // the first batch of token fragments is in flight while the slab lands
        load_batch(ksplit);
        cp_async_wait_prev();
        __syncthreads();
        const uint32_t lds_slab = lds_base + (uint32_t)((slab & 1) * kSlabBytes);
        for (int b0 = ksplit; b0 < nblk; b0 += nsplit * kBatch) {
            if (b0 != ksplit) load_batch(b0);
#pragma unroll
            for (int u = 0; u < kBatch; ++u) {
                const int blk = b0 + u * nsplit;
                if (blk >= nblk) break;
                // which of this warp's partials: (blk % 4) = ksplit + nsplit * j.  With
                // kBatch a multiple of kSets, j is fixed by u at compile time.
                const int j = ((u * nsplit) % kSplits) / nsplit;
#pragma unroll
                for (int n = 0; n < NT; ++n) {
                    uint32_t b0r, b1r, b2r, b3r;
                    ldsm_x4_trans(lds_slab + (uint32_t)(32 * blk * G::kPitch + 16 * n), b0r, b1r, b2r, b3r);
                    mma_bf16_16816(acc[j][n], xa[u].x, xb[u].x, xa[u].y, xb[u].y, b0r, b1r);
                    mma_bf16_16816(acc[j][n], xa[u].z, xb[u].z, xa[u].w, xb[u].w, b2r, b3r);
                }
            }
        }
        __syncthreads();  // this buffer is refilled two slabs later
    }
    __syncthreads();  // the slab region is reused for the partials
#pragma unroll
    for (int j = 0; j < kSets; ++j) {
        const int sidx = ksplit + nsplit * j;
#pragma unroll
        for (int n = 0; n < NT; ++n) {
            const int e0 = n * 8 + 2 * c;
            float* pa = sPart + (sidx * a.tpc + tg * 16 + g) * EP;
            float* pb = pa + 8 * EP;
            pa[e0] = acc[j][n][0];
            pa[e0 + 1] = acc[j][n][1];
            pb[e0] = acc[j][n][2];
            pb[e0 + 1] = acc[j][n][3];
        }
    }
    __syncthreads();
    const int split_stride = a.tpc * EP;
    for (int i = tid; i < a.tpc * E; i += kThreads) {
        const int tok = i / E, e = i - tok * E;
        const float* p = sPart + tok * EP + e;
        sL[tok * kLStride + e] = ((p[0] + p[split_stride]) + p[2 * split_stride]) + p[3 * split_stride];
    }
    __syncthreads();
    router_finish(a, sL, sHist, true);
}

template <int EP>  // experts padded to EP (8 or 64); tpc = 32
__global__ void __launch_bounds__(kThreads) router_f32_kernel(RouterArgs a) {
    extern __shared__ __align__(128) uint8_t smem[];
    float* sW = reinterpret_cast<float*>(smem);                                // [slab][EP]
    float* sL = reinterpret_cast<float*>(smem + kSlabBytes);                   // [32][65]
    int* sHist = reinterpret_cast<int*>(sL + kChunkTokens * kLStride);
    if (a.logits_in) {
        load_logits_in(a, sL);
        router_finish(a, sL, sHist, false);
        return;
    }
    constexpr int kSlab = kSlabBytes / 4 / EP;
    const int tid = threadIdx.x;
    const int E = a.E, d = a.d;
    const int64_t t = (int64_t)blockIdx.x * a.tpc + tid;
    const bool valid = tid < a.tpc && t < a.T;
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

// Tokens per CTA: 64 when 16 < E <= 32 (router weight re-read per CTA at most
// half of its x bytes) and there are enough tokens for >= ~1 CTA per SM,
// else 32.
int pick_tpc(int64_t T, int E) {
    if (E > 16 && E <= 32 && (T + 63) / 64 >= sm_count()) return 64;
    return 32;
}

template <int NT, int TPC>
cudaError_t launch_bf16_tpc(RouterArgs a, cudaStream_t s) {
    a.tpc = TPC;
    const size_t smem = (size_t)union_bytes_for<NT>(a.d) + tail_bytes_for(TPC);
    const size_t smem_max = (size_t)union_bytes_for<NT>(1 << 30) + tail_bytes_for(kMaxTpc);
    static std::atomic<bool> attr[64];
    const cudaError_t err = ensure_smem_attr(attr, router_bf16_kernel<NT, TPC>, (int)smem_max);
    if (err != cudaSuccess) return err;
    const int grid = (int)((a.T + TPC - 1) / TPC);
    router_bf16_kernel<NT, TPC><<<grid, kThreads, smem, s>>>(a);
    return cudaGetLastError();
}

template <int NT>
cudaError_t launch_bf16_nt(RouterArgs a, cudaStream_t s) {
    if constexpr (NT == 3 || NT == 4) {
        if (pick_tpc(a.T, a.E) == 64) return launch_bf16_tpc<NT, 64>(a, s);
    }
    return launch_bf16_tpc<NT, 32>(a, s);
}

template <int EP>
cudaError_t launch_f32_ep(RouterArgs a, cudaStream_t s) {
    a.tpc = kChunkTokens;
    const size_t smem = kSlabBytes + tail_bytes_for(a.tpc);
    static std::atomic<bool> attr[64];
    const cudaError_t err = ensure_smem_attr(attr, router_f32_kernel<EP>, (int)smem);
    if (err != cudaSuccess) return err;
    const int grid = (int)((a.T + a.tpc - 1) / a.tpc);
    router_f32_kernel<EP><<<grid, kThreads, smem, s>>>(a);
    return cudaGetLastError();
}

}  // namespace

// Router kernel choice: by the configuration only (never by T), so a token's
// logits are the same whichever batch it is routed in.  The library's choice
// for bf16 is the warp-MMA router with the router weight resident across a
// CTA cluster (same logits bit for bit as the slab-staged one, which takes the
// shapes whose weight slices do not fit in shared memory); the tensor-core
// router on request.  Fed logits (no GEMM) take the warp routers' selection.
bool use_router_tc(const RouterArgs& a) { return a.kernel == MOE_ROUTER_TCGEN05 && router_tc_supported(a); }

cudaError_t launch_router(const RouterArgs& a_in, bool bf16, cudaStream_t s) {
    if (a_in.T == 0) return cudaSuccess;
    RouterArgs a = a_in;
    a.scan.npsum = a.nchunk;  // probability sums per chunk (the resident-weight router sets its own)
    if (bf16 && use_router_tc(a)) return launch_router_tc(a, a.st, s);
    if (bf16 && a.kernel != MOE_ROUTER_WARP_MMA_STAGED && router_v2_supported(a)) return launch_router_v2(a, s);
    if (bf16) {
        switch ((a.E + 7) / 8) {
            case 1: return launch_bf16_nt<1>(a, s);
            case 2: return launch_bf16_nt<2>(a, s);
            case 3: return launch_bf16_nt<3>(a, s);
            case 4: return launch_bf16_nt<4>(a, s);
            case 5: return launch_bf16_nt<5>(a, s);
            case 6: return launch_bf16_nt<6>(a, s);
            case 7: return launch_bf16_nt<7>(a, s);
            default: return launch_bf16_nt<8>(a, s);
        }
    }
    if (a.E <= 8) return launch_f32_ep<8>(a, s);
    return launch_f32_ep<64>(a, s);
}

}  // namespace moe
