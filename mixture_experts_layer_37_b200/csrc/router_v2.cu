// Router with the router weight resident in shared memory across a cluster
// of CTAs, the tokens streamed by TMA, and the products on the warp-level
// tensor-core MMA (bf16).
//
// Method: logits = x . W_r (+ bias), softmax over all experts, top-k on the
// logits (lower id first on ties), weights renormalised over the k chosen
// ("MoE: gating, experts, load balancing, capacity factor" (dpshk.com/news/
// 6005940) §2.1, §3.1; "Llama-MoE架构解析" (coreui.cn/article/2610641) §3.1),
// plus the per-chunk expert histogram and probability sums for the dispatch
// scan and the load-balance statistics; the last CTA runs that scan.
//
// Arithmetic.  A token's logit for expert e is ((P0 + P1) + P2) + P3, where
// P_s accumulates, in ascending order, the 32-column blocks b of x with
// b % 4 == s, each block as two mma.sync m16n8k16 steps whose reduction
// indices are assigned so that a thread's A fragment is 16 contiguous bytes
// of x.  This is exactly the arithmetic of the slab-staged warp-MMA router
// (router.cu), so both give the same logits bit for bit, and a token's logits
// do not depend on the batch it is in.
//
// Parallel structure.  A cluster of 2*ns CTAs works on 64-token tiles.  CTA
// rank r holds partial sums P_{2(r%2)} and P_{2(r%2)+1} for the experts of
// n-tiles [(r/2)*NTL, (r/2+1)*NTL): the rows of W_r for its blocks stay in
// shared memory for the whole kernel (loaded once), laid out so that every
// ldmatrix phase reads eight distinct bank groups.  Per CTA:
//   warp 8    TMA producer: for each tile, the CTA's 64-column block pairs of
//             the tile's 64 rows (one 8 KB box per stage, 128-byte swizzle; as
//             many stages as the shared memory left over holds, up to 16), so x
//             streams without any CTA-wide barrier, starting before the
//             resident weight has landed;
//   warps 0-7 (m-tile w/2, partial w%2): the MMA chain over the CTA's blocks,
//             A from the ring (mma row g of an m-tile takes tile row
//             (g>>1) | ((g&1)<<2), which makes each quarter-warp's 16-byte
//             reads fall in distinct bank groups), B by ldmatrix.trans from the
//             resident weight; then the 16 tokens' partial sums are stored into
//             the exchange buffer of the CTA that finishes their 32-token chunk
//             (rank 0 or 1) through distributed shared memory.
// Exchange buffers are guarded by mbarriers with cluster-scope release and
// acquire (full: every writer lane has stored; empty: the finisher has read),
// so the producer keeps streaming the next tile while the finishers work.
//   warps 9-16 (ranks 0 and 1) finish one 32-token chunk each per tile, while
//             the consumer warps already run the next tile's products: eight
//             lanes per token, shuffle reductions inside each lane group,
//             outputs, and the chunk's statistics; probability sums
//             accumulate per CTA in a fixed order.
// The last CTA runs the dispatch scan with its shared memory as scratch.
// Every wait is bounded in time; on expiry the kernel records the site, skips
// the remaining work, keeps every barrier count, and returns.
#include <math.h>

#include <map>
#include <mutex>
#include <tuple>

#include "gemm_common.cuh"
#include "moe.h"
#include "scan.cuh"
#include "warp_mma.cuh"

namespace moe {
namespace {

constexpr int kQW = 8;                        // consumer warps, and finisher warps
constexpr int kProducerWarp = kQW;            // the TMA producer
constexpr int kFinWarp0 = kQW + 1;            // first finisher warp
constexpr int kV2Threads = (2 * kQW + 1) * 32;
constexpr int kConsumerBar = 1, kFinisherBar = 2;  // named barriers of the two warp groups
constexpr int kTile = 64;                     // tokens per tile: four 16-token m-tiles, two chunks
constexpr int kStageBytes = kTile * 128;      // one 64-column block pair of a tile
constexpr int kMinStages = 4, kMaxStages = 16;
constexpr int kV2SmemLimit = 227 * 1024;
constexpr int kMaxRouterCtas = 512;           // grid cap (the workspace holds this many psum columns)
static_assert(kTile == 2 * kChunkTokens, "a tile is two chunks, one per finisher");

struct V2Args {
    RouterArgs r;
    int ns = 1;           // expert splits: 2 * ns CTAs per cluster
    int nst = kMinStages; // ring stages
    int units = 1;        // 16-byte units per resident weight row
    int slice_bytes = 0;  // resident weight bytes per CTA (0 with fed logits)
    int xs = 0;           // floats per token row of the exchange buffer and the statistics scratch
    int ntiles = 0;
};

__host__ __device__ constexpr bool xor_layout(int ntl) { return ntl == 4 || ntl == 8; }
__host__ __device__ constexpr int units_for(int ntl) { return xor_layout(ntl) ? ntl : (ntl | 1); }

// Byte offset of resident row `row` (32 rows per block, blocks in the CTA's
// order) and 16-byte unit n.  NTL 4 or 8: unpadded rows, units XOR-swizzled by
// the row's position in its block; otherwise rows padded to an odd number of
// units and rotated inside their block.  Either way the eight rows
// 8a + 2j + {0,1} (a = 0..3) that one ldmatrix phase reads fall in eight
// distinct 16-byte bank groups.
template <int NTL>
__host__ __device__ __forceinline__ uint32_t slice_off(int row, int n, int units) {
    if constexpr (xor_layout(NTL)) {
        const int a = (row >> 3) & 3;
        const int h = NTL == 4 ? a : 2 * a + (row & 1);
        return (uint32_t)(row * NTL * 16 + 16 * (n ^ h));
    } else {
        const int a = (row >> 3) & 3, b = row & 7;
        const int prow = (row & ~31) + 8 * a + ((b + 2 * a) & 7);
        return (uint32_t)(prow * units * 16 + 16 * n);
    }
}

__device__ __forceinline__ uint4 lds128(uint32_t addr) {
    uint4 v;
    asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(addr));
    return v;
}
__device__ __forceinline__ void st_cluster_v2(uint32_t addr, float a, float b) {
    asm volatile("st.shared::cluster.v2.f32 [%0], {%1, %2};" ::"r"(addr), "f"(a), "f"(b) : "memory");
}
__device__ __forceinline__ bool mbar_try_wait_acq_cluster(uint64_t* bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity)
        : "memory");
    return ok != 0;
}
__device__ __forceinline__ bool mbar_wait_cluster_bounded(uint64_t* bar, uint32_t parity, uint64_t timeout_ns) {
    if (mbar_try_wait_acq_cluster(bar, parity)) return true;
    const uint64_t t0 = globaltimer_ns();
    uint32_t n = 0;
    while (true) {
        if (mbar_try_wait_acq_cluster(bar, parity)) return true;
        if ((++n & 15u) == 0 && globaltimer_ns() - t0 > timeout_ns) return false;
    }
}
// Split cluster barrier: every thread arrives once, and waits before its next arrival.
__device__ __forceinline__ void cluster_arrive() { asm volatile("barrier.cluster.arrive.release.aligned;" ::: "memory"); }
__device__ __forceinline__ void cluster_wait() { asm volatile("barrier.cluster.wait.acquire.aligned;" ::: "memory"); }

// Finish of one 32-token chunk by the 8 finisher warps (all of them call it;
// `work` false skips the work but keeps the three barriers).  Eight lanes per
// token: warp w takes tokens 4w..4w+3, lane group g = lane/8 one token, lane
// j = lane%8 of the group the experts j, j+8, ..., so every reduction over a
// token's experts is three xor-shuffle levels inside the group and the 32
// tokens of the chunk proceed together.
// Logits: the exchange buffer's four partial sums in the fixed order (or the
// fed logits), plus the bias.  Top-k: k rounds of (each lane's largest
// unchosen logit, lower id first on equal values) reduced over the group,
// larger logit first and the lower id on equal logits.  Softmax in fp32 with
// the sum in a fixed order (the lane's terms ascending, then the tree);
// chosen weights renormalised by their sum in j order.  The exchange buffer
// is released (`release`) as soon as all warps have read it.  Then the
// chunk's statistics: probability sums per expert in a fixed order (fp64),
// expert counts (per-lane counters, no atomics), and the counts added into
// the chunk's group.
// `ft` is the thread's index in the finisher group (0..255).
template <int M, class Release>  // M = experts per lane = ceil(E / 8)
__device__ __forceinline__ void finish_chunk(const RouterArgs& a, int chunk, const float* xb, int xs, const float* sBias,
                                             float* sPc, int* sH, double* sPsum, int* sReal, bool work, int ft,
                                             Release release) {
    const int PS = xs;  // row stride of the statistics scratch, as of the exchange buffer
    constexpr int NONE = 0x7fffffff;
    const int warp = ft >> 5, lane = ft & 31;
    const int grp = lane >> 3, jl = lane & 7;
    // every argument in a register: no reloads from the parameter block after the stores
    const int E = a.E, k = a.k, nchunk = a.nchunk, ngroups = a.ngroups, gchunks = a.group_chunks;
    const int64_t T = a.T;
    const uint8_t* __restrict__ mask = a.mask;
    const float* __restrict__ lin = a.logits_in;
    float* __restrict__ lout = a.logits_out;
    float* __restrict__ pout = a.probs_out;
    int32_t* __restrict__ tidx = a.topk_idx;
    float* __restrict__ tw = a.topk_w;
    int32_t* __restrict__ hist = a.hist;
    int32_t* __restrict__ ghist = a.group_hist;
    const bool fed = lin != nullptr;
    const int tl = 4 * warp + grp;  // this lane group's token in the chunk
    const int64_t t = (int64_t)chunk * kChunkTokens + tl;
    const bool valid = work && t < T;
    const bool real = valid && (mask == nullptr || mask[t] != 0);  // padding selects nothing
    float v[M];
#pragma unroll
    for (int m = 0; m < M; ++m) {
        const int e = jl + 8 * m;
        float x = -INFINITY;
        if (valid && e < E) {
            if (fed) {
                x = lin[t * E + e];
            } else {
                const float* r = xb + tl * xs + e;
                x = ((r[0] + r[kChunkTokens * xs]) + r[2 * kChunkTokens * xs]) + r[3 * kChunkTokens * xs];
                if (sBias != nullptr) x += sBias[e];
            }
        }
        v[m] = x;
    }
    named_barrier_sync(kFinisherBar, kQW * 32);
    release();  // every warp has read the exchange buffer
    int cnt[M];
#pragma unroll
    for (int m = 0; m < M; ++m) cnt[m] = 0;
    if (work) {
        float mx = -INFINITY;
#pragma unroll
        for (int m = 0; m < M; ++m) {
            if (valid && jl + 8 * m < E && lout) lout[t * E + jl + 8 * m] = v[m];
            mx = fmaxf(mx, v[m]);
        }
#pragma unroll
        for (int o = 4; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
        // top-k: k rounds over the group of (value, id), larger value first, lower id on equal values
        uint32_t chosen = 0;
        int sel[kMaxTopK];
#pragma unroll
        for (int j = 0; j < kMaxTopK; ++j) {
            if (j >= k) break;
            float bv = -INFINITY;
            int bi = NONE;
#pragma unroll
            for (int m = 0; m < M; ++m) {
                const int e = jl + 8 * m;
                const bool take = e < E && !((chosen >> m) & 1u) && (bi == NONE || v[m] > bv);
                bv = take ? v[m] : bv;
                bi = take ? e : bi;
            }
#pragma unroll
            for (int o = 4; o > 0; o >>= 1) {
                const float ov = __shfl_xor_sync(0xffffffffu, bv, o);
                const int oi = __shfl_xor_sync(0xffffffffu, bi, o);
                const bool take = oi != NONE && (bi == NONE || ov > bv || (ov == bv && oi < bi));
                bv = take ? ov : bv;
                bi = take ? oi : bi;
            }
            sel[j] = bi;
            if ((bi & 7) == jl) chosen |= 1u << (bi >> 3);
        }
        // softmax over all experts, fp32; the sum in a fixed order (the lane's terms, then the tree)
        float p[M];
        float ssum = 0.f;
#pragma unroll
        for (int m = 0; m < M; ++m) {
            p[m] = (valid && jl + 8 * m < E) ? expf(v[m] - mx) : 0.f;
            ssum += p[m];
        }
#pragma unroll
        for (int o = 4; o > 0; o >>= 1) ssum += __shfl_xor_sync(0xffffffffu, ssum, o);
        const float inv = valid ? 1.0f / ssum : 0.f;
#pragma unroll
        for (int m = 0; m < M; ++m) {
            const int e = jl + 8 * m;
            p[m] *= inv;
            if (e < E) {
                if (valid && pout) pout[t * E + e] = p[m];
                sPc[tl * PS + e] = real ? p[m] : 0.f;  // padding and tokens past T: not in the sums
            }
        }
        // the k chosen probabilities, renormalised by their sum (j ascending); lane j of the group writes choice j
        float pw[kMaxTopK];
        float ps = 0.f;
#pragma unroll
        for (int j = 0; j < kMaxTopK; ++j) {
            if (j >= k) break;
            float own = 0.f;
#pragma unroll
            for (int m = 0; m < M; ++m) own = (m == (sel[j] >> 3)) ? p[m] : own;
            pw[j] = __shfl_sync(0xffffffffu, own, (lane & ~7) | (sel[j] & 7));
            ps += pw[j];
        }
        int my_e = -1;
        float my_w = 0.f;
#pragma unroll
        for (int j = 0; j < kMaxTopK; ++j) {
            if (j >= k) break;
            const float wj = pw[j] / ps;
            my_e = jl == j ? sel[j] : my_e;
            my_w = jl == j ? wj : my_w;
#pragma unroll
            for (int m = 0; m < M; ++m) cnt[m] += (real && sel[j] == jl + 8 * m) ? 1 : 0;
        }
        if (jl < k && valid) {
            tidx[t * k + jl] = real ? my_e : -1;
            tw[t * k + jl] = real ? my_w : 0.f;
        }
        // this warp's counts per expert (its four tokens): lane j of group 0 holds experts j + 8m
#pragma unroll
        for (int m = 0; m < M; ++m) {
            cnt[m] += __shfl_xor_sync(0xffffffffu, cnt[m], 8);
            cnt[m] += __shfl_xor_sync(0xffffffffu, cnt[m], 16);
            if (grp == 0 && jl + 8 * m < E) sH[warp * kMaxExperts + jl + 8 * m] = cnt[m];
        }
        const unsigned nreal = __popc(__ballot_sync(0xffffffffu, real && jl == 0));
        if (lane == 0) atomicAdd(sReal, (int)nreal);
    }
    named_barrier_sync(kFinisherBar, kQW * 32);
    if (work && warp == 0) {
        for (int e = lane; e < E; e += 32) {
            // the chunk's probability sum in a fixed order: four interleaved token chains, then pairwise
            double acc[4] = {0.0, 0.0, 0.0, 0.0};
#pragma unroll
            for (int r = 0; r < kChunkTokens; r += 4) {
#pragma unroll
                for (int u = 0; u < 4; ++u) acc[u] += (double)sPc[(r + u) * PS + e];
            }
            sPsum[e] += (acc[0] + acc[1]) + (acc[2] + acc[3]);
            int n = 0;
#pragma unroll
            for (int w = 0; w < kQW; ++w) n += sH[w * kMaxExperts + e];
            hist[(int64_t)e * nchunk + chunk] = n;
            if (n && ghist) atomicAdd(ghist + (int64_t)e * ngroups + chunk / gchunks, n);
        }
    }
    named_barrier_sync(kFinisherBar, kQW * 32);
}

template <int NTL, int M>
__global__ void __launch_bounds__(kV2Threads, 1)
    router_v2_kernel(const __grid_constant__ CUtensorMap tmX, const __grid_constant__ V2Args va) {
    const RouterArgs& a = va.r;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    const int nst = va.nst;
    uint8_t* ring = smem;
    uint8_t* slice = smem + nst * kStageBytes;
    float* xbuf = reinterpret_cast<float*>(slice + va.slice_bytes);  // [4 partials][32 tokens][xs]
    float* sPc = xbuf + 4 * kChunkTokens * va.xs;                     // [32 tokens][xs]
    int* sH = reinterpret_cast<int*>(sPc + kChunkTokens * va.xs);     // [8 warps][64] expert counts
    float* sBias = reinterpret_cast<float*>(sH + kQW * kMaxExperts);   // [64]
    uint64_t* bars = reinterpret_cast<uint64_t*>(sBias + kMaxExperts);
    uint64_t* full = bars;                     // [nst] a ring stage has landed
    uint64_t* empty = bars + kMaxStages;       // [nst] the consumers have read a stage
    uint64_t* xfull = bars + 2 * kMaxStages;   // [1] every partial of this CTA's chunk has been stored
    uint64_t* xempty = xfull + 1;              // [2] finisher f has read its exchange buffer
    double* sPsum = reinterpret_cast<double*>(xempty + 2);             // [64]
    int* sMisc = reinterpret_cast<int*>(sPsum + kMaxExperts);          // abort, last CTA, real tokens
    volatile int* abort_flag = sMisc;
    __shared__ int sCount[kMaxExperts];
    __shared__ double sP[kMaxExperts];

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int rank = (int)cluster_ctarank();
    const int pr = rank & 1, nsi = rank >> 1;
    const int cs = 2 * va.ns;
    const int cid = blockIdx.x / cs, ncl = gridDim.x / cs;
    const bool fed = a.logits_in != nullptr;
    const int ntiles = va.ntiles, xs = va.xs, units = va.units, nchunk = a.nchunk, E = a.E;
    const int nblk = a.d / 32;
    const int nj = (nblk - 2 * pr + 3) / 4;  // block pairs (stages per tile) holding this CTA's partials
    const uint64_t tmo = a.st.timeout_ns;
    const bool finisher = rank < 2;

    if (threadIdx.x == 0) {
        for (int s = 0; s < nst; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], kQW);
        }
        mbar_init(xfull, 32u * 4u * (uint32_t)cs);  // 4 writer warps per CTA, every lane arrives
        mbar_init(&xempty[0], 1);
        mbar_init(&xempty[1], 1);
        sMisc[0] = 0;
        sMisc[2] = 0;
        fence_barrier_init();
        if (!fed) tma_prefetch_desc(&tmX);
    }
    for (int i = threadIdx.x; i < kMaxExperts; i += blockDim.x) {
        sPsum[i] = 0.0;
        sBias[i] = (a.bias != nullptr && i < a.E) ? a.bias[i] : 0.f;
    }
    __syncthreads();
    cluster_arrive();  // this CTA's barriers exist; waited on before the first remote arrival

    auto give_up = [&](uint32_t site) {
        report_timeout(a.st, site);
        *abort_flag = 1;
    };

    if (warp == kProducerWarp) {
        if (lane == 0 && !fed) {
            // ------------------------------------------------ TMA producer (starts before the weights land)
            int stage = 0;
            uint32_t phase = 0, issued_mask = 0, issued_par = 0;
            bool stop = false;
            for (int tile = cid; tile < ntiles && !stop; tile += ncl) {
                for (int j = 0; j < nj; ++j) {
                    if (*abort_flag) { stop = true; break; }
                    if (!mbar_wait_bounded(&empty[stage], phase ^ 1u, tmo)) {
                        give_up(SITE_ROUTER_RING_EMPTY);
                        stop = true;
                        break;
                    }
                    mbar_arrive_expect_tx(&full[stage], kStageBytes);
                    tma_load_2d(ring + stage * kStageBytes, &tmX, &full[stage], 128 * j + 64 * pr, tile * kTile);
                    issued_mask |= 1u << stage;
                    issued_par = (issued_par & ~(1u << stage)) | (phase << stage);
                    if (++stage == nst) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
            }
            // no copy may still be landing in shared memory when the CTA exits
            for (int s = 0; s < nst; ++s)
                if ((issued_mask >> s) & 1u)
                    if (!mbar_wait_bounded(&full[s], (issued_par >> s) & 1u, tmo)) give_up(SITE_ROUTER_DRAIN);
        }
        __syncwarp();
        cluster_wait();
    } else if (warp < kQW) {
        // ---------------------------------------------------- consumers
        if (!fed) {
            // the resident weight: W_r rows of the CTA's blocks (4j + 2pr + {0,1}), its experts
            const __nv_bfloat16* W = static_cast<const __nv_bfloat16*>(a.w_router);
            const int nunits = 64 * nj * NTL;
            const bool vec = (a.E & 7) == 0;
            for (int i = threadIdx.x; i < nunits; i += kQW * 32) {
                const int row = i / NTL, n = i - row * NTL;
                const int ib = row >> 5, kk = row & 31;
                const int b = 4 * (ib >> 1) + 2 * pr + (ib & 1);
                const int64_t wrow = 32 * (int64_t)b + kk;
                const int e0 = 8 * (nsi * NTL + n);
                uint8_t* dst = slice + slice_off<NTL>(row, n, va.units);
                if (vec) {
                    cp_async_16(dst, W + wrow * a.E + e0);
                } else {
                    __nv_bfloat16 h[8];
#pragma unroll
                    for (int w = 0; w < 8; ++w)
                        h[w] = e0 + w < a.E ? W[wrow * a.E + e0 + w] : __float2bfloat16(0.f);
                    *reinterpret_cast<uint4*>(dst) = *reinterpret_cast<const uint4*>(h);
                }
            }
            cp_async_commit();
            cp_async_wait_all();
        }
        named_barrier_sync(kConsumerBar, kQW * 32);
        cluster_wait();  // every CTA's barriers exist before any remote arrival

        const int u = warp & 1, mt = warp >> 1;
        const int g = lane >> 2, c = lane & 3;
        const int rg = (g >> 1) | ((g & 1) << 2);   // tile row (inside the m-tile) of mma row g
        const int r0 = 16 * mt + rg, r1 = r0 + 8;
        const uint32_t ring_s = smem_u32(ring);
        const uint32_t a0off = (uint32_t)(r0 * 128 + 16 * ((4 * u + c) ^ (r0 & 7)));
        const uint32_t a1off = (uint32_t)(r1 * 128 + 16 * ((4 * u + c) ^ (r1 & 7)));
        // ldmatrix: lane (j = lane/8, r = lane%8) gives row 8*(r/2) + 2j + (r%2) of each 32-row block
        const int lj = lane >> 3, lr = lane & 7;
        const int lrow = 8 * (lr >> 1) + 2 * lj + (lr & 1);
        const int hx = xor_layout(NTL) ? (NTL == 4 ? (lr >> 1) : 2 * (lr >> 1) + (lr & 1)) : 0;
        // XOR layout: this lane's row base (its unit hx sits at unit 0); unit n is then at n ^ hx
        const uint32_t slice_s = smem_u32(slice) + slice_off<NTL>(lrow, hx, units);
        const uint32_t blk_bytes = 32u * (uint32_t)units * 16u;
        const int f = mt >> 1;  // finisher of this warp's chunk
        const uint32_t xbuf_f = mapa_shared(smem_u32(xbuf), (uint32_t)f);
        const uint32_t xfull_f = mapa_shared(smem_u32(xfull), (uint32_t)f);
        const int s_part = 2 * pr + u;
        const int lt0 = 16 * (mt & 1) + rg, lt1 = lt0 + 8;  // token rows inside the chunk
        int stage = 0;
        uint32_t phase = 0, xe_par = 0;
        bool dead = false;
        for (int tile = cid; tile < ntiles; tile += ncl) {
            dead = dead || __shfl_sync(0xffffffffu, *abort_flag, 0) != 0;
            if (!fed) {
                float acc[NTL][4];
#pragma unroll
                for (int n = 0; n < NTL; ++n) acc[n][0] = acc[n][1] = acc[n][2] = acc[n][3] = 0.f;
                for (int j = 0; j < nj; ++j) {
                    if (!dead) {
                        const bool ok = mbar_wait_bounded(&full[stage], phase, tmo);
                        if (!__all_sync(0xffffffffu, ok)) {
                            if (lane == 0) give_up(SITE_ROUTER_RING_FULL);
                            dead = true;
                        }
                    }
                    if (!dead) {
                        const uint4 xa = lds128(ring_s + stage * kStageBytes + a0off);
                        const uint4 xb = lds128(ring_s + stage * kStageBytes + a1off);
                        __syncwarp();
                        if (lane == 0) mbar_arrive(&empty[stage]);
                        const uint32_t bb = slice_s + (uint32_t)(2 * j + u) * blk_bytes;
#pragma unroll
                        for (int n = 0; n < NTL; ++n) {
                            uint32_t b0, b1, b2, b3;
                            const uint32_t un = xor_layout(NTL) ? (uint32_t)(n ^ hx) : (uint32_t)n;
                            ldsm_x4_trans(bb + 16u * un, b0, b1, b2, b3);
                            mma_bf16_16816(acc[n], xa.x, xb.x, xa.y, xb.y, b0, b1);
                            mma_bf16_16816(acc[n], xa.z, xb.z, xa.w, xb.w, b2, b3);
                        }
                    }
                    if (++stage == nst) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
                // the partial sums of this warp's 16 tokens -> the finisher of their chunk
                if (!dead) {
                    const bool ok = mbar_wait_cluster_bounded(&xempty[f], xe_par ^ 1u, tmo);
                    if (!__all_sync(0xffffffffu, ok)) {
                        if (lane == 0) give_up(SITE_ROUTER_XCHG_EMPTY);
                        dead = true;
                    }
                }
                if (!dead) {
#pragma unroll
                    for (int n = 0; n < NTL; ++n) {
                        const int e0 = 8 * (nsi * NTL + n) + 2 * c;
                        st_cluster_v2(xbuf_f + 4u * (uint32_t)((s_part * kChunkTokens + lt0) * xs + e0), acc[n][0],
                                      acc[n][1]);
                        st_cluster_v2(xbuf_f + 4u * (uint32_t)((s_part * kChunkTokens + lt1) * xs + e0), acc[n][2],
                                      acc[n][3]);
                    }
                    mbar_arrive_cluster(xfull_f);
                }
                xe_par ^= 1u;
            }
        }
    } else {
        // ---------------------------------------------------- finishers (ranks 0 and 1)
        // warps kFinWarp0.. finish this CTA's chunk of each tile while the
        // consumers already run the next tile's products
        cluster_wait();  // every CTA's barriers exist before any remote arrival (the releases)
        const int ft = (int)threadIdx.x - kFinWarp0 * 32;
        uint32_t xf_par = 0;
        bool dead = false;
        if (finisher) {
            for (int tile = cid; tile < ntiles; tile += ncl) {
                dead = dead || __shfl_sync(0xffffffffu, *abort_flag, 0) != 0;
                if (!fed && !dead) {
                    const bool ok = mbar_wait_cluster_bounded(xfull, xf_par, tmo);
                    if (!__all_sync(0xffffffffu, ok)) {
                        if (lane == 0) give_up(SITE_ROUTER_XCHG_FULL);
                        dead = true;
                    }
                }
                xf_par ^= 1u;
                const int chunk = tile * 2 + rank;
                // the exchange buffer is free again for every writer of the cluster
                // (finisher thread r signals CTA r: one release each, in parallel)
                auto release = [&]() {
                    if (!fed && ft < cs) mbar_arrive_cluster(mapa_shared(smem_u32(&xempty[rank]), (uint32_t)ft));
                };
                finish_chunk<M>(a, chunk, xbuf, xs, a.bias != nullptr ? sBias : nullptr, sPc, sH, sPsum,
                                &sMisc[2], !dead && chunk < nchunk, ft, release);
            }
        }
    }
    __syncthreads();
    {
        // this CTA's probability sums (zero when it finished no chunk) and real-token count
        if (warp == 0) {
            for (int e = lane; e < E; e += 32) a.psum[(int64_t)e * gridDim.x + blockIdx.x] = sPsum[e];
            if (lane == 0 && a.mask != nullptr && a.real_counter != nullptr && sMisc[2] != 0)
                atomicAdd(a.real_counter, sMisc[2]);
        }
    }
    cluster_sync_all();  // no CTA leaves while a peer may still store into it or arrive on its barriers
    if (!a.fuse_scan) return;
    // the scan on everyone's statistics (its ring and weight slice as scratch): with one cluster, rank 0
    // runs it at once (the cluster barrier's release and acquire already ordered every CTA's results);
    // otherwise the last CTA to finish
    const bool one_cluster = gridDim.x == (unsigned)cs;
    if (one_cluster) {
        if (rank != 0) return;
    } else {
        __threadfence();
        __syncthreads();
        if (threadIdx.x == 0) sMisc[1] = (atomicAdd(a.counter, 1u) == gridDim.x - 1u) ? 1 : 0;
        __syncthreads();
        if (!sMisc[1]) return;
        __threadfence();
    }
    scan_block(a.scan, sCount, sP, smem, nst * kStageBytes + va.slice_bytes);
    if (threadIdx.x == 0 && !one_cluster) *a.counter = 0u;
}

struct V2Plan {
    bool ok = false;
    int ns = 1, ntl = 1, units = 1, slice_bytes = 0, xs = 0, smem = 0, ntiles = 0, nst = kMinStages, m = 1;
};

// shared memory besides the ring: slice, exchange buffer, statistics scratch, barriers and small arrays
int smem_fixed(int slice_bytes, int xs, int m) {
    return 1024 + slice_bytes + 4 * kChunkTokens * xs * 4 + kChunkTokens * xs * 4 +
           kQW * kMaxExperts * 4 + kMaxExperts * 4 + (2 * kMaxStages + 3) * 8 + kMaxExperts * 8 + 16;
}

V2Plan plan_v2(const RouterArgs& a) {
    V2Plan p;
    const int NT = (a.E + 7) / 8;
    const bool fed = a.logits_in != nullptr;
    const int rows = 64 * ((a.d / 32 + 3) / 4);  // rank 0 of the pair holds the most blocks
    const int budget = kV2SmemLimit - 1024;      // the static shared arrays of the scan
    // row stride: an odd multiple of 8 floats, so the four token rows a warp's lane groups
    // read or write at once fall in distinct banks (and 8-byte aligned)
    p.xs = (NT & 1) ? 8 * NT : 8 * NT + 8;
    p.m = NT;
    p.ntiles = (int)((a.T + kTile - 1) / kTile);
    auto fill = [&](int ns) {
        p.ns = ns;
        p.ntl = NT / ns;
        p.units = units_for(p.ntl);
        p.slice_bytes = fed ? 0 : rows * p.units * 16;
        const int fixed = smem_fixed(p.slice_bytes, p.xs, p.m);
        int nst = (budget - fixed) / kStageBytes;
        if (nst > kMaxStages) nst = kMaxStages;
        p.nst = nst;
        p.smem = fixed + nst * kStageBytes;
        return nst >= kMinStages;
    };
    if (fed) {
        p.ok = fill(1);
        return p;
    }
    int ns = 0;
    for (int c = 1; c <= 4; c *= 2)
        if (NT % c == 0 && fill(c)) {
            ns = c;
            break;
        }
    if (ns == 0) return p;
    // more expert splits while the tiles alone cannot occupy the GPU
    while (ns < 4 && NT % (2 * ns) == 0 && (int64_t)p.ntiles * 4 * ns <= sm_count() && fill(2 * ns)) ns *= 2;
    p.ok = fill(ns);
    return p;
}

std::mutex g_occ_mutex;
std::map<std::tuple<int, const void*, int, int>, int> g_occ;  // (device, kernel, cluster size, smem) -> clusters

template <int NTL, int M>
cudaError_t launch_v2(const RouterArgs& a, const V2Plan& p, cudaStream_t s) {
    auto kernel = router_v2_kernel<NTL, M>;
    static std::atomic<bool> attr[64];
    cudaError_t err = ensure_smem_attr(attr, kernel, kV2SmemLimit - 1024);
    if (err != cudaSuccess) return err;
    CUtensorMap mx;
    if (a.logits_in == nullptr) {
        if (!gemm::make_map(&mx, a.x, (uint64_t)a.d, (uint64_t)a.T, (uint64_t)a.d * 2, 64, kTile))
            return cudaErrorInvalidValue;
    } else {
        memset(&mx, 0, sizeof(mx));
    }
    const int cs = 2 * p.ns;
    cudaLaunchConfig_t cfg = {};
    cudaLaunchAttribute attr_c;
    attr_c.id = cudaLaunchAttributeClusterDimension;
    attr_c.val.clusterDim.x = (unsigned)cs;
    attr_c.val.clusterDim.y = 1;
    attr_c.val.clusterDim.z = 1;
    cfg.blockDim = dim3(kV2Threads);
    cfg.dynamicSmemBytes = (size_t)p.smem;
    cfg.stream = s;
    cfg.attrs = &attr_c;
    cfg.numAttrs = 1;
    int dev = 0;
    cudaGetDevice(&dev);
    int resident = 0;
    {
        std::lock_guard<std::mutex> lock(g_occ_mutex);
        const auto key = std::make_tuple(dev, reinterpret_cast<const void*>(kernel), cs, p.smem);
        auto it = g_occ.find(key);
        if (it != g_occ.end()) {
            resident = it->second;
        } else {
            cfg.gridDim = dim3((unsigned)(cs * (sm_count() / cs)));
            if (cudaOccupancyMaxActiveClusters(&resident, kernel, &cfg) != cudaSuccess || resident <= 0)
                resident = sm_count() / cs;
            g_occ[key] = resident;
        }
    }
    int ncl = p.ntiles < resident ? p.ntiles : resident;
    if (ncl * cs > kMaxRouterCtas) ncl = kMaxRouterCtas / cs;
    if (ncl < 1) ncl = 1;
    V2Args va;
    va.r = a;
    va.r.scan.npsum = ncl * cs;  // one probability-sum column per CTA
    va.ns = p.ns;
    va.nst = p.nst;
    va.units = p.units;
    va.slice_bytes = p.slice_bytes;
    va.xs = p.xs;
    va.ntiles = p.ntiles;
    cfg.gridDim = dim3((unsigned)(ncl * cs));
    err = cudaLaunchKernelEx(&cfg, kernel, mx, va);
    if (err != cudaSuccess) return err;
    return cudaGetLastError();
}

// NTL (n-tiles per CTA) divides M (n-tiles of all experts) by 1, 2 or 4
template <int M>
cudaError_t launch_v2_ntl(const RouterArgs& a, const V2Plan& p, cudaStream_t s) {
    if (p.ntl == M) return launch_v2<M, M>(a, p, s);
    if constexpr (M % 2 == 0) {
        if (p.ntl == M / 2) return launch_v2<M / 2, M>(a, p, s);
    }
    if constexpr (M % 4 == 0) {
        if (p.ntl == M / 4) return launch_v2<M / 4, M>(a, p, s);
    }
    return cudaErrorInvalidValue;
}

}  // namespace

bool router_v2_supported(const RouterArgs& a) { return plan_v2(a).ok; }

int router_v2_psum_columns() { return kMaxRouterCtas; }

cudaError_t launch_router_v2(const RouterArgs& a, cudaStream_t s) {
    const V2Plan p = plan_v2(a);
    if (!p.ok) return cudaErrorInvalidValue;
    switch (p.m) {
        case 1: return launch_v2_ntl<1>(a, p, s);
        case 2: return launch_v2_ntl<2>(a, p, s);
        case 3: return launch_v2_ntl<3>(a, p, s);
        case 4: return launch_v2_ntl<4>(a, p, s);
        case 5: return launch_v2_ntl<5>(a, p, s);
        case 6: return launch_v2_ntl<6>(a, p, s);
        case 7: return launch_v2_ntl<7>(a, p, s);
        default: return launch_v2_ntl<8>(a, p, s);
    }
}

}  // namespace moe
