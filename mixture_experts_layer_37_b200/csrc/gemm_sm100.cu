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
// This file: the one-CTA-per-tile kernel and the host launcher; the CTA-pair
// kernel (cta_group::2, 256-row tiles) is in gemm_sm100_pair.cu.
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
// reads the next rows (or TMA zero-fill) and masks them at the store; an
// expert's last tile of at most 64 rows runs as an M=64 MMA (half the work),
// whose accumulator rows sit in lanes 0-15 of each 32-lane TMEM quarter.
// Every wait is bounded in time; on expiry the kernel records a timeout,
// drains its own copies and MMAs, frees TMEM and returns.
#include "gemm_common.cuh"
#include "moe.h"

namespace moe {
namespace {

using namespace gemm;

constexpr int BM = 128;
constexpr int kStages = 4;
constexpr int kAStageBytes = BM * BK * 2;                  // 16 KB
constexpr int kBStageBytes = 4 * kBBoxBytes;               // 32 KB
constexpr int kStageBytes = kAStageBytes + kBStageBytes;   // 48 KB
constexpr int kSmemBytes =
    kStages * kStageBytes + 1024 /*barriers + tables*/ + kBiasBytes + 1024 /*alignment*/;
constexpr uint32_t kIdesc = make_idesc(BM, BN_MMA);
constexpr uint32_t kIdesc64 = make_idesc(BM / 2, BN_MMA);

template <int MODE, bool GATHER>
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
    // the prologue above overlaps the launch before; from here on its results are read
    griddep_wait();
    griddep_launch_dependents();
    if (threadIdx.x == 64) build_tile_table(p, BM, mt_prefix, s_off);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;
    const int total_tiles = mt_prefix[p.E] * p.n_tiles;
    const int kblocks = p.K / BK;
    const uint64_t tmo = p.st.timeout_ns;

    auto give_up = [&](uint32_t site) {
        report_timeout(p.st, site);
        *abort_flag = 1;
    };

    if (warp == 0 && GATHER) {
        // ------------------------------------------------ gathering producer
        // A tile: 32 TMA gathers of four token rows each (tile::gather4 over
        // the token activations, a one-row box of 64 columns, 128-byte
        // swizzle), lane l copying tile rows 4l..4l+3 into their place in the
        // swizzled tile, all lanes issuing at once; lane 0 arms the stage and
        // loads B as the plain producer does.
        int stage = 0;
        uint32_t phase = 0;
        uint32_t issued_mask = 0, issued_par = 0;
        bool stop = false;
        const int R = s_off[p.E];
        for (int tile = blockIdx.x; tile < total_tiles && !stop; tile += gridDim.x) {
            int e, row0, rows, nt;
            decode_tile(tile, mt_prefix, s_off, p.n_tiles, BM, e, row0, rows, nt);
            const int n0 = nt * p.bn_out;
            int tok[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const int row = row0 + 4 * lane + i;
                tok[i] = row < R ? p.src_assign[row] / p.k : 0;  // rows past R: any valid row, masked later
            }
            for (int kb = 0; kb < kblocks; ++kb) {
                if (lane == 0) {
                    if (*abort_flag) {
                        stop = true;
                    } else if (!mbar_wait_bounded(&empty[stage], phase ^ 1u, tmo)) {
                        give_up(SITE_GEMM_PRODUCER_EMPTY);
                        stop = true;
                    } else {
                        mbar_arrive_expect_tx(&full[stage], kStageBytes);
                        uint8_t* b_dst = sB + stage * kBStageBytes;
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
                    }
                }
                // the stage is armed (or the producer stops) before any lane's copy
                stop = __shfl_sync(0xffffffffu, stop ? 1 : 0, 0) != 0;
                if (stop) break;
                tma_gather4(sA + stage * kAStageBytes + lane * 4 * 128, &tmA, &full[stage], kb * BK, tok[0], tok[1],
                            tok[2], tok[3]);
                if (++stage == kStages) {
                    stage = 0;
                    phase ^= 1u;
                }
            }
        }
        // no copy may still be landing in shared memory when the CTA exits
        if (lane == 0)
            for (int s = 0; s < kStages; ++s)
                if ((issued_mask >> s) & 1u)
                    if (!mbar_wait_bounded(&full[s], (issued_par >> s) & 1u, tmo)) give_up(SITE_GEMM_PRODUCER_DRAIN);
    } else if (warp == 0) {
        if (lane == 0) {
            // ------------------------------------------------ TMA producer
            int stage = 0;
            uint32_t phase = 0;
            uint32_t issued_mask = 0, issued_par = 0;
            bool stop = false;
            for (int tile = blockIdx.x; tile < total_tiles && !stop; tile += gridDim.x) {
                int e, row0, rows, nt;
                decode_tile(tile, mt_prefix, s_off, p.n_tiles, BM, e, row0, rows, nt);
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
                int e, row0, rows, nt;
                decode_tile(tile, mt_prefix, s_off, p.n_tiles, BM, e, row0, rows, nt);
                const uint32_t idesc = rows <= BM / 2 ? kIdesc64 : kIdesc;
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
                        tc_mma_f16(d_tmem, adesc, bdesc, idesc, (kb | kk) != 0 ? 1u : 0u);
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
        __nv_bfloat16* wb = s_bias + (warp - 2) * BN_MMA;
        int acc = 0;
        uint32_t acc_phase = 0;
        for (int tile = blockIdx.x; tile < total_tiles; tile += gridDim.x) {
            const int ab = __shfl_sync(0xffffffffu, *abort_flag, 0);
            if (ab) break;
            int e, row0, rows, nt;
            decode_tile(tile, mt_prefix, s_off, p.n_tiles, BM, e, row0, rows, nt);
            const bool ok = mbar_wait_bounded(&tfull[acc], acc_phase, tmo);
            if (!__all_sync(0xffffffffu, ok)) {
                if (lane == 0) give_up(SITE_GEMM_EPI_TMEM_FULL);
                break;
            }
            tc_fence_after();
            // M=128: row 32q + lane.  M=64 (a last tile of at most 64 rows):
            // rows 16q..16q+15 sit in lanes 0-15 of this warp's quarter
            const bool m64 = rows <= BM / 2;
            const int r = m64 ? 16 * q + lane : q * 32 + lane;
            const bool valid = r < rows && (!m64 || lane < 16);
            __nv_bfloat16* orow = p.out + (int64_t)(row0 + (valid ? r : 0)) * p.N;
            const uint32_t tbase = tmem_base + ((uint32_t)(q * 32) << 16) + (uint32_t)(acc * BN_MMA);
            epilogue_rows<MODE>(p, tbase, orow, valid, nt * p.bn_out, e, wb, lane, row_weight(p, row0 + r, valid));
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
    static std::atomic<EncodeTiledFn> cached{nullptr};
    EncodeTiledFn fn = cached.load(std::memory_order_acquire);
    if (fn == nullptr) {
        void* ptr = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess) {
            fn = reinterpret_cast<EncodeTiledFn>(ptr);
            cached.store(fn, std::memory_order_release);
        }
    }
    return fn;
}

template <int MODE, bool GATHER = false>
cudaError_t launch_mode(const CUtensorMap& a, const CUtensorMap& b0, const CUtensorMap& b1, const GemmParams& p,
                        int64_t rows_cap, cudaStream_t s) {
    static std::atomic<bool> attr_set[64];
    const cudaError_t err = ensure_smem_attr(attr_set, grouped_gemm_kernel<MODE, GATHER>, kSmemBytes);
    if (err != cudaSuccess) return err;
    const int64_t tiles_upper = (rows_cap / BM + p.E) * (int64_t)p.n_tiles;
    const int grid = (int)min64(tiles_upper, (int64_t)sm_count());
    if (grid <= 0) return cudaSuccess;
    return launch_kernel(grouped_gemm_kernel<MODE, GATHER>, dim3(grid), dim3(kThreads), kSmemBytes, s, a, b0, b1, p);
}

}  // namespace

namespace gemm {
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
bool make_map_plain(CUtensorMap* m, CUtensorMapDataType dtype, const void* base, uint64_t inner, uint64_t outer,
                    uint64_t pitch, uint32_t box_inner, uint32_t box_outer) {
    EncodeTiledFn enc = encode_fn();
    if (enc == nullptr) return false;
    const cuuint64_t dims[2] = {inner, outer};
    const cuuint64_t strides[1] = {pitch};
    const cuuint32_t box[2] = {box_inner, box_outer};
    const cuuint32_t estr[2] = {1, 1};
    return enc(m, dtype, 2, const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
               CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}
}  // namespace gemm

// CTA-pair variant (gemm_sm100_pair.cu).
cudaError_t launch_pair_gemm(int mode, const CUtensorMap& a, const CUtensorMap& b0, const CUtensorMap& b1,
                             const gemm::GemmParams& p, int64_t rows_cap, cudaStream_t s);

namespace {
// Kernel choice per GEMM.  The CTA pair halves the weight bytes each SM loads
// and reads per MMA, and its 256-row tiles halve the number of tiles; an
// expert's rows are padded to a multiple of 128 by either kernel (the pair
// runs a last tile of at most 128 rows as an M=128 pair tile).  The library's
// choice, from same-machine measurements of both kernels on every benchmark
// workload: the one-CTA kernel for the first GEMM (the pair was 1-7 % slower
// there); for the second GEMM the pair when an expert is expected to hold at
// least 512 rows and there are at most 16 experts (4096 and 8192 tokens over 8
// experts: 110 vs 115 us and 1.58-1.61 vs 1.61-1.62 ms), else the one-CTA
// kernel (32768 tokens over 32 experts: 1.17 vs 1.19-1.22 ms, where the pair
// fetched its operands 1.45x over from DRAM).
cudaError_t launch_one(int mode, bool pair, const CUtensorMap& a, const CUtensorMap& b0, const CUtensorMap& b1,
                       const GemmParams& p, int64_t rows_cap, cudaStream_t s) {
    if (p.gx != nullptr) {  // first GEMM with its rows gathered from the tokens (one-CTA kernel)
        if (mode == MODE_SWIGLU) return launch_mode<MODE_SWIGLU, true>(a, b0, b1, p, rows_cap, s);
        return launch_mode<MODE_GELU, true>(a, b0, b1, p, rows_cap, s);
    }
    if (pair) return launch_pair_gemm(mode, a, b0, b1, p, rows_cap, s);
    if (mode == MODE_SWIGLU) return launch_mode<MODE_SWIGLU>(a, b0, b1, p, rows_cap, s);
    if (mode == MODE_GELU) return launch_mode<MODE_GELU>(a, b0, b1, p, rows_cap, s);
    return launch_mode<MODE_PLAIN>(a, b0, b1, p, rows_cap, s);
}
}  // namespace

cudaError_t launch_ffn_bf16_sm100(const FfnArgs& a, cudaStream_t s) {
    if (a.rows_cap <= 0) return cudaSuccess;
    const bool swiglu = a.act == 0;
    // A maps use 128-row boxes (one CTA's half of a pair tile, or a whole single-CTA tile); a first
    // GEMM gathering its rows reads the token activations through a one-row box (tile::gather4)
    CUtensorMap mA1, mB1, mB1u, mA2, mB2;
    bool ok = a.gather_x != nullptr
                  ? make_map(&mA1, a.gather_x, (uint64_t)a.d, (uint64_t)a.gather_rows, (uint64_t)a.d * 2, 64, 1)
                  : make_map(&mA1, a.x_perm, (uint64_t)a.d, (uint64_t)a.rows_cap, (uint64_t)a.d * 2, 64, 128);
    ok = ok && make_map(&mB1, a.w1, (uint64_t)a.ffn, (uint64_t)a.E * a.d, (uint64_t)a.ffn * 2, 64, BK);
    if (swiglu)
        ok = ok && make_map(&mB1u, a.w_up, (uint64_t)a.ffn, (uint64_t)a.E * a.d, (uint64_t)a.ffn * 2, 64, BK);
    else
        mB1u = mB1;
    ok = ok && make_map(&mA2, a.h, (uint64_t)a.ffn, (uint64_t)a.rows_cap, (uint64_t)a.ffn * 2, 64, 128);
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
    p1.gx = static_cast<const __nv_bfloat16*>(a.gather_x);
    p1.src_assign = a.src_assign;
    p1.k = a.k;
    // rows an expert is expected to receive (the routing itself stays on the device)
    const bool pair1 = a.gemm_kernel == MOE_GEMM_CTA_PAIR;
    const bool pair2 = a.gemm_kernel == MOE_GEMM_CTA_PAIR ||
                       (a.gemm_kernel == MOE_GEMM_AUTO && a.rows_cap / a.E >= 512 && a.E <= 16);
    cudaError_t err = launch_one(swiglu ? MODE_SWIGLU : MODE_GELU, pair1, mA1, mB1, mB1u, p1, a.rows_cap, s);
    if (err != cudaSuccess) return err;
    if (a.between != nullptr && (err = record_mark(a.between, s)) != cudaSuccess) return err;

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
    p2.gx = nullptr;
    p2.src_assign = a.row_w != nullptr ? a.src_assign : nullptr;
    p2.row_w = a.row_w;
    p2.k = a.k;
    return launch_one(MODE_PLAIN, pair2, mA2, mB2, mB2, p2, a.rows_cap, s);
}

}  // namespace moe
