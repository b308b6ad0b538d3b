// Grouped expert GEMMs on the 5th-generation tensor cores (tcgen05, TMEM,
// TMA) for sm_100a, with the expert activation fused into the epilogue.
//
// Method: each expert is an FFN over the rows dispatched to it -- SwiGLU
// W_down(silu(x W_gate) * x W_up) ("MoE: gating, experts, load balancing,
// capacity factor" (dpshk.com/news/6005940) §2.2; "Llama-MoE架构解析"
// (coreui.cn/article/2610641) §2.1) or W2(gelu(x W1 + b1)) + b2 (MoE-basics
// §3.1 ExpertFFN) -- with all experts' weights in one flattened [E, d, ffn]
// pool ("How to Loop MoE: Flatten the Experts, Untie the Attention"
// (discosf.com/news/5228035) §2.1), and all tokens of one expert processed as
// one matrix product (MoE-basics §4.4).
//
// Kernel design (one persistent CTA per SM, 192 threads):
//   warp 0   TMA producer: A tile [128 rows x 64 K] of the expert-sorted
//            activations (K-major, 128-byte swizzle) and four [64 K x 64 N]
//            boxes of the expert's weights (N-major, 128-byte swizzle) per
//            stage, 4 stages of 48 KB, mbarrier transaction counts;
//   warp 1   TMEM allocator and single-thread MMA issuer:
//            tcgen05.mma.cta_group::1.kind::f16, M=128, N=256, K=16, fp32
//            accumulators in TMEM, two accumulator buffers (2 x 256 columns)
//            so the epilogue of one tile overlaps the MMAs of the next;
//   warps 2-5 epilogue: tcgen05.ld of the accumulator rows, activation
//            (silu(gate)*up for SwiGLU: the gate and up halves of the N=256
//            accumulator; bias + erf-GELU; or bias), round to bf16 once, and
//            store the rows that belong to the tile's expert.
// Tiles walk the ragged per-expert row groups: the tile list (m-tiles per
// expert) is built on the device from the kept-row offsets, so the host never
// reads the routing result.  A tile that runs past its expert's last row
// reads the next rows (or TMA zero-fill) and masks them at the store.
// Every wait is bounded in time; on expiry the kernel records a timeout,
// drains its own copies and MMAs, frees TMEM and returns.
#include "internal.h"

namespace moe {
namespace {

constexpr int BM = 128;
constexpr int BK = 64;
constexpr int BN_MMA = 256;
constexpr int kStages = 4;
constexpr int kAStageBytes = BM * BK * 2;                  // 16 KB
constexpr int kBBoxBytes = BK * 64 * 2;                    // 8 KB: 64 K-rows x 64 N (128 B)
constexpr int kBStageBytes = 4 * kBBoxBytes;               // 32 KB
constexpr int kStageBytes = kAStageBytes + kBStageBytes;   // 48 KB
constexpr int kTmemCols = 2 * BN_MMA;                      // two fp32 accumulators
constexpr int kThreads = 192;
constexpr int kGroupM = 32;  // m-tiles per raster group
constexpr int kBiasBytes = 4 * BN_MMA * 2;                 // one bf16 bias row per epilogue warp
constexpr int kSmemBytes = kStages * kStageBytes + 1024 /*barriers + tables*/ + kBiasBytes + 1024 /*alignment*/;

enum { MODE_PLAIN = 0, MODE_SWIGLU = 1, MODE_GELU = 2 };

// Instruction descriptor, kind::f16: D fp32 (bits 4-5 = 1), A bf16 (bits 7-9
// = 1), B bf16 (bits 10-12 = 1), A K-major (bit 15 = 0), B MN-major (bit 16
// = 1), N>>3 in bits 17-22, M>>4 in bits 24-28.
constexpr uint32_t kIdesc = (1u << 4) | (1u << 7) | (1u << 10) | (0u << 15) | (1u << 16) |
                            ((uint32_t)(BN_MMA >> 3) << 17) | ((uint32_t)(BM >> 4) << 24);

// Shared-memory matrix descriptor, 128-byte swizzle: start address, leading
// and stride byte offsets (all >> 4), version 1 (bit 46), layout 2 (bits 61-63).
__device__ __forceinline__ uint64_t smem_desc_sw128(uint32_t saddr, uint32_t lbo, uint32_t sbo) {
    uint64_t d = (uint64_t)((saddr >> 4) & 0x3FFFu);
    d |= (uint64_t)((lbo >> 4) & 0x3FFFu) << 16;
    d |= (uint64_t)((sbo >> 4) & 0x3FFFu) << 32;
    d |= (uint64_t)1 << 46;
    d |= (uint64_t)2 << 61;
    return d;
}

struct GemmParams {
    const int32_t* offsets;      // [E+1] kept-row offsets per expert
    __nv_bfloat16* out;          // [rows_cap, N]
    const __nv_bfloat16* bias;   // [E, N] or null
    int E, K, N;
    int bn_out;                  // output columns per tile: 128 (SwiGLU) or 256
    int n_tiles;
    DevStatus st;
};

__device__ __forceinline__ float silu_f(float x) { return x / (1.0f + __expf(-x)); }
__device__ __forceinline__ float gelu_f(float x) { return 0.5f * x * (1.0f + erff(x * 0.70710678118654752f)); }

template <int MODE>
__global__ void __launch_bounds__(kThreads, 1)
    grouped_gemm_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB0,
                        const __grid_constant__ CUtensorMap tmB1, GemmParams p) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    uint8_t* sA = smem;
    uint8_t* sB = smem + kStages * kAStageBytes;
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kStages * kStageBytes);
    uint64_t* full = bars;
    uint64_t* empty = bars + kStages;
    uint64_t* tfull = bars + 2 * kStages;
    uint64_t* tempty = tfull + 2;
    uint64_t* drain = tempty + 2;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
    int* mt_prefix = reinterpret_cast<int*>(tmem_slot + 2);   // [E+1]
    int* s_off = mt_prefix + (kMaxExperts + 1);                // [E+1]
    __nv_bfloat16* s_bias = reinterpret_cast<__nv_bfloat16*>(smem + kStages * kStageBytes + 1024);  // [4][256]

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    if (threadIdx.x == 0) {
        for (int s = 0; s < kStages; ++s) {
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
        tma_prefetch_desc(&tmA);
        tma_prefetch_desc(&tmB0);
        tma_prefetch_desc(&tmB1);
    }
    if (warp == 1) {
        tmem_alloc(tmem_slot, kTmemCols);
        tmem_relinquish();
    }
    if (threadIdx.x == 64) {
        int acc = 0;
        mt_prefix[0] = 0;
        for (int e = 0; e < p.E; ++e) {
            const int o0 = p.offsets[e], o1 = p.offsets[e + 1];
            s_off[e] = o0;
            acc += (o1 - o0 + BM - 1) / BM;
            mt_prefix[e + 1] = acc;
        }
        s_off[p.E] = p.offsets[p.E];
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;
    const int total_tiles = mt_prefix[p.E] * p.n_tiles;
    const int kblocks = p.K / BK;
    const uint64_t tmo = p.st.timeout_ns;

    // Tile order: expert by expert; inside an expert, groups of kGroupM
    // m-tiles, and inside a group n-tile-major.  The CTAs running at the same
    // time then share each weight tile among up to kGroupM of them and each
    // activation tile among the group's n-tiles, which keeps the expert's
    // working set in L2 even when its weights exceed it.
    auto decode = [&](int tile, int& e, int& row0, int& rows, int& nt) {
        e = 0;
        while (mt_prefix[e + 1] * p.n_tiles <= tile) ++e;
        const int local = tile - mt_prefix[e] * p.n_tiles;
        const int mt_e = mt_prefix[e + 1] - mt_prefix[e];
        const int grp = local / (kGroupM * p.n_tiles);
        const int gm = min(kGroupM, mt_e - grp * kGroupM);
        const int r = local - grp * kGroupM * p.n_tiles;
        nt = r / gm;
        const int mt = grp * kGroupM + (r - nt * gm);
        row0 = s_off[e] + mt * BM;
        rows = min(BM, s_off[e + 1] - row0);
    };
    auto give_up = [&](uint32_t site) {
        report_timeout(p.st, site);
        *abort_flag = 1;
    };

    if (warp == 0) {
        if (lane == 0) {
            // ------------------------------------------------ TMA producer
            int stage = 0;
            uint32_t phase = 0;
            uint32_t issued_mask = 0, issued_par = 0;
            bool stop = false;
            for (int tile = blockIdx.x; tile < total_tiles && !stop; tile += gridDim.x) {
                int e, row0, rows, nt;
                decode(tile, e, row0, rows, nt);
                const int n0 = nt * p.bn_out;
                for (int kb = 0; kb < kblocks; ++kb) {
                    if (*abort_flag) { stop = true; break; }
                    if (!mbar_wait_bounded(&empty[stage], phase ^ 1u, tmo)) {
                        give_up(SITE_GEMM_PRODUCER_EMPTY);
                        stop = true;
                        break;
                    }
                    mbar_arrive_expect_tx(&full[stage], kStageBytes);
                    uint8_t* a_dst = sA + stage * kAStageBytes;
                    uint8_t* b_dst = sB + stage * kBStageBytes;
                    tma_load_2d(a_dst, &tmA, &full[stage], kb * BK, row0);
                    const int krow = e * p.K + kb * BK;
                    if (MODE == MODE_SWIGLU) {
                        tma_load_2d(b_dst, &tmB0, &full[stage], n0, krow);
                        tma_load_2d(b_dst + kBBoxBytes, &tmB0, &full[stage], n0 + 64, krow);
                        tma_load_2d(b_dst + 2 * kBBoxBytes, &tmB1, &full[stage], n0, krow);
                        tma_load_2d(b_dst + 3 * kBBoxBytes, &tmB1, &full[stage], n0 + 64, krow);
                    } else {
#pragma unroll
                        for (int i = 0; i < 4; ++i)
                            tma_load_2d(b_dst + i * kBBoxBytes, &tmB0, &full[stage], n0 + 64 * i, krow);
                    }
                    issued_mask |= 1u << stage;
                    issued_par = (issued_par & ~(1u << stage)) | (phase << stage);
                    if (++stage == kStages) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
            }
            // no copy may still be landing in shared memory when the CTA exits
            for (int s = 0; s < kStages; ++s)
                if ((issued_mask >> s) & 1u)
                    if (!mbar_wait_bounded(&full[s], (issued_par >> s) & 1u, tmo)) give_up(SITE_GEMM_PRODUCER_DRAIN);
        }
    } else if (warp == 1) {
        if (lane == 0) {
            // ------------------------------------------------ MMA issuer
            int stage = 0;
            uint32_t phase = 0;
            int acc = 0;
            uint32_t acc_phase = 0;
            bool stop = false;
            for (int tile = blockIdx.x; tile < total_tiles && !stop; tile += gridDim.x) {
                if (!mbar_wait_bounded(&tempty[acc], acc_phase ^ 1u, tmo)) {
                    give_up(SITE_GEMM_MMA_TMEM_EMPTY);
                    break;
                }
                tc_fence_after();
                const uint32_t d_tmem = tmem_base + (uint32_t)(acc * BN_MMA);
                for (int kb = 0; kb < kblocks; ++kb) {
                    if (*abort_flag) { stop = true; break; }
                    if (!mbar_wait_bounded(&full[stage], phase, tmo)) {
                        give_up(SITE_GEMM_MMA_FULL);
                        stop = true;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t a_addr = smem_u32(sA + stage * kAStageBytes);
                    const uint32_t b_addr = smem_u32(sB + stage * kBStageBytes);
#pragma unroll
                    for (int kk = 0; kk < BK / 16; ++kk) {
                        // A: K-major, +32 bytes per K=16 step inside the 128-byte swizzle row.
                        // B: N-major, +2 x 8 K-rows (2048 bytes) per K=16 step; the four
                        //    64-column boxes are 8 KB apart (leading byte offset).
                        const uint64_t adesc = smem_desc_sw128(a_addr + kk * 32, 16, 1024);
                        const uint64_t bdesc = smem_desc_sw128(b_addr + kk * 2048, kBBoxBytes, 1024);
                        tc_mma_f16(d_tmem, adesc, bdesc, kIdesc, (kb | kk) != 0 ? 1u : 0u);
                    }
                    tc_commit(&empty[stage]);
                    if (++stage == kStages) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
                if (stop) break;
                tc_commit(&tfull[acc]);
                acc ^= 1;
                if (acc == 0) acc_phase ^= 1u;
            }
            // every MMA issued by this thread has completed before TMEM is freed
            tc_commit(drain);
            if (!mbar_wait_bounded(drain, 0, tmo)) give_up(SITE_GEMM_DRAIN);
        }
    } else {
        // ---------------------------------------------------- epilogue
        const int q = warp & 3;  // TMEM lanes 32q..32q+31 are reachable from this warp
        int acc = 0;
        uint32_t acc_phase = 0;
        for (int tile = blockIdx.x; tile < total_tiles; tile += gridDim.x) {
            const int ab = __shfl_sync(0xffffffffu, *abort_flag, 0);
            if (ab) break;
            int e, row0, rows, nt;
            decode(tile, e, row0, rows, nt);
            const bool ok = mbar_wait_bounded(&tfull[acc], acc_phase, tmo);
            if (!__all_sync(0xffffffffu, ok)) {
                if (lane == 0) give_up(SITE_GEMM_EPI_TMEM_FULL);
                break;
            }
            tc_fence_after();
            const int r = q * 32 + lane;
            const bool valid = r < rows;
            __nv_bfloat16* orow = p.out + (int64_t)(row0 + (valid ? r : 0)) * p.N;
            const uint32_t tbase = tmem_base + ((uint32_t)(q * 32) << 16) + (uint32_t)(acc * BN_MMA);
            const int n0 = nt * p.bn_out;
            if (MODE == MODE_SWIGLU) {
                for (int c = 0; c < 128; c += 16) {
                    uint32_t g[16], u[16];
                    tmem_ld_16(tbase + c, g);
                    tmem_ld_16(tbase + 128 + c, u);
                    tmem_ld_wait();
                    if (valid && n0 + c < p.N) {
                        uint32_t pk[8];
#pragma unroll
                        for (int i = 0; i < 8; ++i) {
                            const float h0 = silu_f(__uint_as_float(g[2 * i])) * __uint_as_float(u[2 * i]);
                            const float h1 = silu_f(__uint_as_float(g[2 * i + 1])) * __uint_as_float(u[2 * i + 1]);
                            pk[i] = pack_bf16x2(h0, h1);
                        }
                        uint4* dst = reinterpret_cast<uint4*>(orow + n0 + c);
                        dst[0] = make_uint4(pk[0], pk[1], pk[2], pk[3]);
                        dst[1] = make_uint4(pk[4], pk[5], pk[6], pk[7]);
                    }
                }
            } else {
                // this tile's 256 bias values, staged once per tile in the warp's own row
                __nv_bfloat16* wb = s_bias + (warp - 2) * BN_MMA;
                if (p.bias != nullptr) {
                    __syncwarp();
                    const int col = n0 + 8 * lane;
                    uint4 bv = make_uint4(0, 0, 0, 0);
                    if (col < p.N) bv = *reinterpret_cast<const uint4*>(p.bias + (int64_t)e * p.N + col);
                    reinterpret_cast<uint4*>(wb)[lane] = bv;
                    __syncwarp();
                }
                for (int c = 0; c < BN_MMA; c += 16) {
                    uint32_t v[16];
                    tmem_ld_16(tbase + c, v);
                    tmem_ld_wait();
                    if (valid && n0 + c < p.N) {
                        float x[16];
#pragma unroll
                        for (int i = 0; i < 16; ++i) x[i] = __uint_as_float(v[i]);
                        if (p.bias != nullptr) {
                            const __nv_bfloat16* b = wb + c;
#pragma unroll
                            for (int i = 0; i < 16; ++i) x[i] += __bfloat162float(b[i]);
                        }
                        if (MODE == MODE_GELU) {
#pragma unroll
                            for (int i = 0; i < 16; ++i) x[i] = gelu_f(x[i]);
                        }
                        uint32_t pk[8];
#pragma unroll
                        for (int i = 0; i < 8; ++i) pk[i] = pack_bf16x2(x[2 * i], x[2 * i + 1]);
                        uint4* dst = reinterpret_cast<uint4*>(orow + n0 + c);
                        dst[0] = make_uint4(pk[0], pk[1], pk[2], pk[3]);
                        dst[1] = make_uint4(pk[4], pk[5], pk[6], pk[7]);
                    }
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&tempty[acc]);
            acc ^= 1;
            if (acc == 0) acc_phase ^= 1u;
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem_base, kTmemCols);
    }
}

// ------------------------------------------------------------------ host side
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = nullptr;
    if (fn == nullptr) {
        void* ptr = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(ptr);
    }
    return fn;
}

// 2-D bf16 tensor [outer, inner] (inner contiguous, row pitch `pitch` bytes),
// box [box_outer, box_inner], 128-byte swizzle, zero fill out of bounds.
bool make_map(CUtensorMap* m, const void* base, uint64_t inner, uint64_t outer, uint64_t pitch, uint32_t box_inner,
              uint32_t box_outer) {
    EncodeTiledFn enc = encode_fn();
    if (enc == nullptr) return false;
    const cuuint64_t dims[2] = {inner, outer};
    const cuuint64_t strides[1] = {pitch};
    const cuuint32_t box[2] = {box_inner, box_outer};
    const cuuint32_t estr[2] = {1, 1};
    return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int MODE>
cudaError_t launch_mode(const CUtensorMap& a, const CUtensorMap& b0, const CUtensorMap& b1, const GemmParams& p,
                        int64_t rows_cap, cudaStream_t s) {
    static bool attr_set[64] = {false};
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev < 64 && !attr_set[dev]) {
        cudaError_t err =
            cudaFuncSetAttribute(grouped_gemm_kernel<MODE>, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
        if (err != cudaSuccess) return err;
        attr_set[dev] = true;
    }
    const int64_t tiles_upper = (rows_cap / BM + p.E) * (int64_t)p.n_tiles;
    const int grid = (int)min64(tiles_upper, (int64_t)sm_count());
    if (grid <= 0) return cudaSuccess;
    grouped_gemm_kernel<MODE><<<grid, kThreads, kSmemBytes, s>>>(a, b0, b1, p);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_ffn_bf16_sm100(const FfnArgs& a, cudaStream_t s) {
    if (a.rows_cap <= 0) return cudaSuccess;
    const bool swiglu = a.act == 0;
    CUtensorMap mA1, mB1, mB1u, mA2, mB2;
    bool ok = make_map(&mA1, a.x_perm, (uint64_t)a.d, (uint64_t)a.rows_cap, (uint64_t)a.d * 2, 64, BM);
    ok = ok && make_map(&mB1, a.w1, (uint64_t)a.ffn, (uint64_t)a.E * a.d, (uint64_t)a.ffn * 2, 64, BK);
    if (swiglu)
        ok = ok && make_map(&mB1u, a.w_up, (uint64_t)a.ffn, (uint64_t)a.E * a.d, (uint64_t)a.ffn * 2, 64, BK);
    else
        mB1u = mB1;
    ok = ok && make_map(&mA2, a.h, (uint64_t)a.ffn, (uint64_t)a.rows_cap, (uint64_t)a.ffn * 2, 64, BM);
    ok = ok && make_map(&mB2, a.w2, (uint64_t)a.d, (uint64_t)a.E * a.ffn, (uint64_t)a.d * 2, 64, BK);
    if (!ok) return cudaErrorInvalidValue;

    GemmParams p1;
    p1.offsets = a.offsets;
    p1.out = static_cast<__nv_bfloat16*>(a.h);
    p1.bias = swiglu ? nullptr : static_cast<const __nv_bfloat16*>(a.b1);
    p1.E = a.E;
    p1.K = a.d;
    p1.N = a.ffn;
    p1.bn_out = swiglu ? 128 : 256;
    p1.n_tiles = (a.ffn + p1.bn_out - 1) / p1.bn_out;
    p1.st = a.st;
    cudaError_t err = swiglu ? launch_mode<MODE_SWIGLU>(mA1, mB1, mB1u, p1, a.rows_cap, s)
                             : launch_mode<MODE_GELU>(mA1, mB1, mB1u, p1, a.rows_cap, s);
    if (err != cudaSuccess) return err;
    if (a.between != nullptr && (err = cudaEventRecord(a.between, s)) != cudaSuccess) return err;

    GemmParams p2;
    p2.offsets = a.offsets;
    p2.out = static_cast<__nv_bfloat16*>(a.y_perm);
    p2.bias = swiglu ? nullptr : static_cast<const __nv_bfloat16*>(a.b2);
    p2.E = a.E;
    p2.K = a.ffn;
    p2.N = a.d;
    p2.bn_out = 256;
    p2.n_tiles = (a.d + 255) / 256;
    p2.st = a.st;
    return launch_mode<MODE_PLAIN>(mA2, mB2, mB2, p2, a.rows_cap, s);
}

}  // namespace moe
