// Router on the tensor cores with TMA and TMEM (bf16, E a multiple of 8).
//
// Method: logits = x . W_r (+ bias), softmax over all experts, top-k on the
// logits (lower id first on ties), weights renormalised over the k chosen
// ("MoE: gating, experts, load balancing, capacity factor" (dpshk.com/news/
// 6005940) §2.1, §3.1; "Llama-MoE架构解析" (coreui.cn/article/2610641) §3.1),
// plus per-chunk expert histograms and probability sums for the dispatch scan
// and the load-balance statistics; the last CTA to finish runs that scan.
//
// One persistent CTA per SM walks 128-token tiles:
//   warp 0   TMA producer: x tile [128 tokens x 64 K] (K-major, 128-byte
//            swizzle) and W_r tile [64 K x 64 experts] (expert-major, columns
//            beyond E zero-filled), 6 stages;
//   warp 1   TMEM allocation and single-thread tcgen05.mma (M=128, N=64,
//            K=16) into one of two accumulators;
//   warps 2-5 one thread per token: its E logits from TMEM (tcgen05.ld) into
//            its row of shared memory, bias, softmax, top-k and
//            renormalisation (compact loops); each warp's
//            32 tokens are one statistics chunk (fixed-order fp64 tree sum of
//            the probabilities, ballot counts of the chosen experts).
// A token's logits are the tensor-core sum over K in a fixed order, so they do
// not depend on the batch the token is in.  All waits are bounded in time.
#include <math.h>

#include "gemm_common.cuh"
#include "scan.cuh"

namespace moe {
namespace {

using gemm::smem_desc_sw128;

constexpr int RBM = 128;                      // tokens per tile
constexpr int RBK = 64;                       // K per stage
constexpr int RBN = 64;                       // expert columns computed (E <= 64)
constexpr int kRStages = 6;
constexpr int kRAStage = RBM * RBK * 2;       // 16 KB
constexpr int kRBStage = RBK * RBN * 2;       // 8 KB
constexpr int kRStage = kRAStage + kRBStage;  // 24 KB
constexpr int kRThreads = 192;
constexpr int kRTmemCols = 128;               // two 64-column accumulators
constexpr int kRLStride = kMaxExperts + 1;     // logits staging row (floats)
constexpr int kRLBytes = RBM * kRLStride * 4;  // 33 KB
constexpr int kRSmem = kRStages * kRStage + 1024 + kRLBytes + 1024;
constexpr uint32_t kRIdesc = gemm::make_idesc(RBM, RBN);

struct RouterTcArgs {
    RouterArgs r;
    DevStatus st;
};

template <int EP>  // experts rounded up to a multiple of 16 (<= 64)
__global__ void __launch_bounds__(kRThreads, 1)
    router_tc_kernel(const __grid_constant__ CUtensorMap tmX, const __grid_constant__ CUtensorMap tmW, RouterTcArgs args) {
    const RouterArgs& a = args.r;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    uint8_t* sA = smem;
    uint8_t* sB = smem + kRStages * kRAStage;
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kRStages * kRStage);
    uint64_t* full = bars;
    uint64_t* empty = bars + kRStages;
    uint64_t* tfull = bars + 2 * kRStages;
    uint64_t* tempty = tfull + 2;
    uint64_t* drain = tempty + 2;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
    int* s_last = reinterpret_cast<int*>(tmem_slot + 2);
    float* sL = reinterpret_cast<float*>(smem + kRStages * kRStage + 1024);  // [128][65]

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int ntiles = (int)((a.T + RBM - 1) / RBM);
    const int kblocks = a.d / RBK;
    const uint64_t tmo = args.st.timeout_ns;

    if (threadIdx.x == 0) {
        for (int s = 0; s < kRStages; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        mbar_init(&tfull[0], 1);
        mbar_init(&tfull[1], 1);
        mbar_init(&tempty[0], 4);
        mbar_init(&tempty[1], 4);
        mbar_init(drain, 1);
        *abort_flag = 0;
        fence_barrier_init();
        fence_proxy_async_smem();
        tma_prefetch_desc(&tmX);
        tma_prefetch_desc(&tmW);
    }
    if (warp == 1) {
        tmem_alloc(tmem_slot, kRTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;
    auto give_up = [&](uint32_t site) {
        report_timeout(args.st, site);
        *abort_flag = 1;
    };

    if (warp == 0) {
        if (lane == 0) {
            int stage = 0;
            uint32_t phase = 0;
            uint32_t issued_mask = 0, issued_par = 0;
            bool stop = false;
            for (int tile = blockIdx.x; tile < ntiles && !stop; tile += gridDim.x) {
                for (int kb = 0; kb < kblocks; ++kb) {
                    if (*abort_flag) { stop = true; break; }
                    if (!mbar_wait_bounded(&empty[stage], phase ^ 1u, tmo)) {
                        give_up(SITE_GEMM_PRODUCER_EMPTY);
                        stop = true;
                        break;
                    }
                    mbar_arrive_expect_tx(&full[stage], kRStage);
                    tma_load_2d(sA + stage * kRAStage, &tmX, &full[stage], kb * RBK, tile * RBM);
                    tma_load_2d(sB + stage * kRBStage, &tmW, &full[stage], 0, kb * RBK);
                    issued_mask |= 1u << stage;
                    issued_par = (issued_par & ~(1u << stage)) | (phase << stage);
                    if (++stage == kRStages) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
            }
            for (int s = 0; s < kRStages; ++s)
                if ((issued_mask >> s) & 1u)
                    if (!mbar_wait_bounded(&full[s], (issued_par >> s) & 1u, tmo)) give_up(SITE_GEMM_PRODUCER_DRAIN);
        }
    } else if (warp == 1) {
        if (lane == 0) {
            int stage = 0;
            uint32_t phase = 0;
            int acc = 0;
            uint32_t acc_phase = 0;
            bool stop = false;
            for (int tile = blockIdx.x; tile < ntiles && !stop; tile += gridDim.x) {
                if (!mbar_wait_bounded(&tempty[acc], acc_phase ^ 1u, tmo)) {
                    give_up(SITE_GEMM_MMA_TMEM_EMPTY);
                    break;
                }
                tc_fence_after();
                const uint32_t d_tmem = tmem_base + (uint32_t)(acc * RBN);
                for (int kb = 0; kb < kblocks; ++kb) {
                    if (*abort_flag) { stop = true; break; }
                    if (!mbar_wait_bounded(&full[stage], phase, tmo)) {
                        give_up(SITE_GEMM_MMA_FULL);
                        stop = true;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t a_addr = smem_u32(sA + stage * kRAStage);
                    const uint32_t b_addr = smem_u32(sB + stage * kRBStage);
#pragma unroll
                    for (int kk = 0; kk < RBK / 16; ++kk) {
                        const uint64_t adesc = smem_desc_sw128(a_addr + kk * 32, 16, 1024);
                        const uint64_t bdesc = smem_desc_sw128(b_addr + kk * 2048, kRBStage, 1024);
                        tc_mma_f16(d_tmem, adesc, bdesc, kRIdesc, (kb | kk) != 0 ? 1u : 0u);
                    }
                    tc_commit(&empty[stage]);
                    if (++stage == kRStages) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
                if (stop) break;
                tc_commit(&tfull[acc]);
                acc ^= 1;
                if (acc == 0) acc_phase ^= 1u;
            }
            tc_commit(drain);
            if (!mbar_wait_bounded(drain, 0, tmo)) give_up(SITE_GEMM_DRAIN);
        }
    } else {
        // ------------------------------------------------ epilogue: one thread per token
        const int q = warp & 3;
        const int E = a.E, k = a.k;
        int acc = 0;
        uint32_t acc_phase = 0;
        for (int tile = blockIdx.x; tile < ntiles; tile += gridDim.x) {
            if (__shfl_sync(0xffffffffu, *abort_flag, 0)) break;
            const bool ok = mbar_wait_bounded(&tfull[acc], acc_phase, tmo);
            if (!__all_sync(0xffffffffu, ok)) {
                if (lane == 0) give_up(SITE_GEMM_EPI_TMEM_FULL);
                break;
            }
            tc_fence_after();
            // this thread's logits: TMEM -> its row of shared memory
            float* row = sL + (q * 32 + lane) * kRLStride;
            const uint32_t tbase = tmem_base + ((uint32_t)(q * 32) << 16) + (uint32_t)(acc * RBN);
#pragma unroll
            for (int c = 0; c < EP; c += 16) {
                uint32_t v[16];
                tmem_ld_16(tbase + c, v);
                tmem_ld_wait();
#pragma unroll
                for (int i = 0; i < 16; ++i) row[c + i] = __uint_as_float(v[i]);
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&tempty[acc]);
            acc ^= 1;
            if (acc == 0) acc_phase ^= 1u;

            const int chunk = tile * (RBM / kChunkTokens) + q;
            const int64_t t = (int64_t)chunk * kChunkTokens + lane;
            const bool valid = t < a.T;
            const bool real = valid && (a.mask == nullptr || a.mask[t] != 0);  // padding selects nothing
            float m = -INFINITY;
#pragma unroll 1
            for (int e = 0; e < E; ++e) {
                float v = row[e];
                if (a.bias) v += a.bias[e];
                row[e] = v;
                m = fmaxf(m, v);
                if (valid && a.logits_out) a.logits_out[t * E + e] = v;
            }
            // top-k on the logits: repeated maximum over unchosen experts,
            // strict '>' keeps the lower id on equal values
            int sel[kMaxTopK];
            uint64_t chosen = 0;
#pragma unroll 1
            for (int j = 0; j < k; ++j) {
                int best = -1;
                float bv = 0.f;
#pragma unroll 1
                for (int e = 0; e < E; ++e) {
                    const float v = row[e];
                    if (!((chosen >> e) & 1ull) && (best < 0 || v > bv)) {
                        best = e;
                        bv = v;
                    }
                }
                chosen |= 1ull << best;
                sel[j] = best;
            }
            // softmax over all experts, fp32, ascending e
            float s = 0.f;
#pragma unroll 1
            for (int e = 0; e < E; ++e) {
                const float z = expf(row[e] - m);
                row[e] = z;
                s += z;
            }
            const float inv = 1.0f / s;
#pragma unroll 1
            for (int e = 0; e < E; ++e) {
                const float pe = row[e] * inv;
                row[e] = pe;
                if (valid && a.probs_out) a.probs_out[t * E + e] = pe;
            }
            float psel = 0.f;
#pragma unroll 1
            for (int j = 0; j < k; ++j) psel += row[sel[j]];
            if (valid) {
#pragma unroll 1
                for (int j = 0; j < k; ++j) {
                    a.topk_idx[t * k + j] = real ? sel[j] : -1;
                    a.topk_w[t * k + j] = real ? row[sel[j]] / psel : 0.f;
                }
            }
            // chunk statistics over the real tokens: fixed-order tree sums in fp64, ballot counts
            if (chunk < a.nchunk) {
#pragma unroll 1
                for (int e = 0; e < E; ++e) {
                    double v = real ? (double)row[e] : 0.0;
#pragma unroll
                    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
                    int cnt = 0;
#pragma unroll 1
                    for (int j = 0; j < k; ++j) cnt += __popc(__ballot_sync(0xffffffffu, real && sel[j] == e));
                    if (lane == 0) {
                        a.psum[(int64_t)e * a.nchunk + chunk] = v;
                        a.hist[(int64_t)e * a.nchunk + chunk] = cnt;
                        if (cnt && a.group_hist) atomicAdd(a.group_hist + (int64_t)e * a.ngroups + chunk / a.group_chunks, cnt);
                    }
                }
                const int nr = __popc(__ballot_sync(0xffffffffu, real));
                if (a.mask != nullptr && a.real_counter != nullptr && lane == 0 && nr) atomicAdd(a.real_counter, nr);
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem_base, kRTmemCols);
    }
    if (!a.fuse_scan) return;
    // last-CTA-done: the CTA that completes the arrival count runs the scan on
    // everyone's partials (fences order the partial stores before the count)
    __threadfence();
    __syncthreads();
    if (threadIdx.x == 0) *s_last = (atomicAdd(a.counter, 1u) == (unsigned)gridDim.x - 1u) ? 1 : 0;
    __syncthreads();
    if (!*s_last) return;
    __threadfence();
    __shared__ int sCount[kMaxExperts];
    __shared__ double sP[kMaxExperts];
    scan_block(a.scan, sCount, sP);
    if (threadIdx.x == 0) *a.counter = 0u;
}

template <int EP>
cudaError_t launch_ep(const CUtensorMap& mx, const CUtensorMap& mw, const RouterTcArgs& args, cudaStream_t s) {
    static std::atomic<bool> attr[64];
    const cudaError_t err = ensure_smem_attr(attr, router_tc_kernel<EP>, kRSmem);
    if (err != cudaSuccess) return err;
    const int ntiles = (int)((args.r.T + RBM - 1) / RBM);
    const int grid = ntiles < sm_count() ? ntiles : sm_count();
    router_tc_kernel<EP><<<grid, kRThreads, kRSmem, s>>>(mx, mw, args);
    return cudaGetLastError();
}

}  // namespace

bool router_tc_supported(const RouterArgs& a) {
    return a.logits_in == nullptr && (a.E % 8) == 0 && a.E <= RBN && (a.d % RBK) == 0 && a.k <= kMaxTopK;
}

cudaError_t launch_router_tc(const RouterArgs& a, DevStatus st, cudaStream_t s) {
    if (a.T == 0) return cudaSuccess;
    CUtensorMap mx, mw;
    bool ok = gemm::make_map(&mx, a.x, (uint64_t)a.d, (uint64_t)a.T, (uint64_t)a.d * 2, RBK, RBM);
    ok = ok && gemm::make_map(&mw, a.w_router, (uint64_t)a.E, (uint64_t)a.d, (uint64_t)a.E * 2, RBN, RBK);
    if (!ok) return cudaErrorInvalidValue;
    RouterTcArgs args;
    args.r = a;
    args.st = st;
    switch ((a.E + 15) / 16) {
        case 1: return launch_ep<16>(mx, mw, args, s);
        case 2: return launch_ep<32>(mx, mw, args, s);
        case 3: return launch_ep<48>(mx, mw, args, s);
        default: return launch_ep<64>(mx, mw, args, s);
    }
}

}  // namespace moe
