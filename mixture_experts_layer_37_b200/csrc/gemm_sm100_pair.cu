// Grouped expert GEMM on CTA pairs: tcgen05.mma.cta_group::2, 256-row tiles.
//
// Same method and epilogue as the one-CTA kernel in gemm_sm100.cu (expert FFN
// matrices over the expert-sorted rows, activation fused into the epilogue;
// "MoE: gating, experts, load balancing, capacity factor" (dpshk.com/news/
// 6005940) §2.2, §3.1; "How to Loop MoE: Flatten the Experts, Untie the
// Attention" (discosf.com/news/5228035) §2.1).
//
// Two CTAs of a cluster (on two SMs) compute one 256 x 256 tile: each holds
// 128 rows of A and 128 of the tile's 256 weight columns in its own shared
// memory, and the leader CTA issues M=256, N=256, K=16 MMAs that read both
// CTAs' operands and write each CTA's 128 accumulator rows into that CTA's
// TMEM.  Per SM this halves the weight bytes loaded and read per MMA, and the
// smaller stage (32 KB) allows a 6-deep pipeline.
//   - Loads: both CTAs issue their own TMA loads (no multicast); transaction
//     bytes complete on the leader's `full` barrier, which the leader arms
//     with both CTAs' bytes.
//   - Stage release / accumulator ready: the leader's tcgen05.commit arrives
//     on the `empty` / `tfull` barrier at the same offset in both CTAs.
//   - Accumulator free: each epilogue warp of both CTAs arrives on the
//     leader's `tempty` barrier (8 arrivals).
// An expert's last tile, when it holds at most 128 rows, runs as an M=128
// pair tile instead (64 rows per CTA), which halves its padding: each CTA's
// accumulator then holds its 64 rows twice over, TMEM lanes 0-63 for the
// first 128 of the 256 columns and lanes 64-127 for the other 128, in TMEM
// columns 0-127 (the two-CTA M=128 data-path layout).
// Column order of the 256 accumulator columns: CTA 0's 128 weight columns
// first, then CTA 1's.  SwiGLU: CTA r loads the gate and the up box of output
// columns [64r, 64r+64) of the tile's 128, so every 128-column half holds
// [gate 64 | up 64] of the same 64 outputs, in both tile shapes.
// Every wait is bounded in time, as in the one-CTA kernel.
#include "gemm_common.cuh"

namespace moe {
namespace {

using namespace gemm;

constexpr int BMP = 256;                         // rows per pair tile (128 per CTA)
constexpr int kStagesP = 6;
constexpr int kAStageP = 128 * BK * 2;           // 16 KB
constexpr int kBStageP = 2 * kBBoxBytes;         // 16 KB: this CTA's 128 of the 256 columns
constexpr int kStageP = kAStageP + kBStageP;     // 32 KB
constexpr int kSmemP = kStagesP * kStageP + 1024 + kBiasBytes + 1024;
constexpr uint32_t kIdescP = make_idesc(BMP, BN_MMA);
constexpr uint32_t kIdescPHalf = make_idesc(BMP / 2, BN_MMA);

// Epilogue of one warp for `ncols` accumulator columns starting at TMEM column
// offset 0 of `tbase`, written to output columns [out0, out0 + ncols) (SwiGLU:
// ncols/2 outputs from [gate 64 | up 64] groups).  `wb` is the warp's bias
// staging row; `rw` the row's routing weight (GEMMs with row weights).
// Warp-collective.
template <int MODE>
__device__ __forceinline__ void epilogue_pair(const GemmParams& p, uint32_t tbase, __nv_bfloat16* orow, bool valid,
                                              int out0, int ncols, int e, __nv_bfloat16* wb, int lane,
                                              float rw = 1.0f) {
    if (MODE == MODE_SWIGLU) {
        for (int g = 0; g < ncols; g += 128) {
            const int o = out0 + g / 2;
#pragma unroll 1
            for (int c = 0; c < 64; c += 16) {
                uint32_t gv[16], uv[16];
                tmem_ld_16(tbase + g + c, gv);
                tmem_ld_16(tbase + g + 64 + c, uv);
                tmem_ld_wait();
                if (valid && o + c < p.N) {
                    uint32_t pk[8];
#pragma unroll
                    for (int i = 0; i < 8; ++i) {
                        const float h0 = silu_f(__uint_as_float(gv[2 * i])) * __uint_as_float(uv[2 * i]);
                        const float h1 = silu_f(__uint_as_float(gv[2 * i + 1])) * __uint_as_float(uv[2 * i + 1]);
                        pk[i] = pack_bf16x2(h0, h1);
                    }
                    uint4* dst = reinterpret_cast<uint4*>(orow + o + c);
                    dst[0] = make_uint4(pk[0], pk[1], pk[2], pk[3]);
                    dst[1] = make_uint4(pk[4], pk[5], pk[6], pk[7]);
                }
            }
        }
    } else {
        if (p.bias != nullptr) {
            __syncwarp();
            const int col = out0 + 8 * lane;
            uint4 bv = make_uint4(0, 0, 0, 0);
            if (8 * lane < ncols && col < p.N) bv = *reinterpret_cast<const uint4*>(p.bias + (int64_t)e * p.N + col);
            reinterpret_cast<uint4*>(wb)[lane] = bv;
            __syncwarp();
        }
#pragma unroll 1
        for (int c = 0; c < ncols; c += 16) {
            uint32_t v[16];
            tmem_ld_16(tbase + c, v);
            tmem_ld_wait();
            if (valid && out0 + c < p.N) {
                float x[16];
#pragma unroll
                for (int i = 0; i < 16; ++i) x[i] = __uint_as_float(v[i]);
                if (p.bias != nullptr) {
                    const uint4* b4 = reinterpret_cast<const uint4*>(wb + c);
                    const uint4 bA = b4[0], bB = b4[1];
                    const uint32_t bw[8] = {bA.x, bA.y, bA.z, bA.w, bB.x, bB.y, bB.z, bB.w};
#pragma unroll
                    for (int i = 0; i < 8; ++i) {
                        x[2 * i] += bf16_lo(bw[i]);
                        x[2 * i + 1] += bf16_hi(bw[i]);
                    }
                }
                if (MODE == MODE_GELU) {
#pragma unroll
                    for (int i = 0; i < 16; ++i) x[i] = gelu_f(x[i]);
                }
                if (p.row_w != nullptr) {
#pragma unroll
                    for (int i = 0; i < 16; ++i) x[i] *= rw;
                }
                uint32_t pk[8];
#pragma unroll
                for (int i = 0; i < 8; ++i) pk[i] = pack_bf16x2(x[2 * i], x[2 * i + 1]);
                uint4* dst = reinterpret_cast<uint4*>(orow + out0 + c);
                dst[0] = make_uint4(pk[0], pk[1], pk[2], pk[3]);
                dst[1] = make_uint4(pk[4], pk[5], pk[6], pk[7]);
            }
        }
    }
}

template <int MODE>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kThreads, 1)
    grouped_gemm_pair_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB0,
                             const __grid_constant__ CUtensorMap tmB1, GemmParams p) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    uint8_t* sA = smem;
    uint8_t* sB = smem + kStagesP * kAStageP;
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kStagesP * kStageP);
    uint64_t* full = bars;
    uint64_t* empty = bars + kStagesP;
    uint64_t* tfull = bars + 2 * kStagesP;
    uint64_t* tempty = tfull + 2;
    uint64_t* drain = tempty + 2;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
    int* mt_prefix = reinterpret_cast<int*>(tmem_slot + 2);   // [E+1]
    int* s_off = mt_prefix + (kMaxExperts + 1);                // [E+1]
    __nv_bfloat16* s_bias = reinterpret_cast<__nv_bfloat16*>(smem + kStagesP * kStageP + 1024);  // [4][256]

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t rank = cluster_ctarank();
    const int pair = blockIdx.x >> 1, npairs = gridDim.x >> 1;

    if (threadIdx.x == 0) {
        for (int s = 0; s < kStagesP; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        mbar_init(&tfull[0], 1);
        mbar_init(&tfull[1], 1);
        mbar_init(&tempty[0], 8);
        mbar_init(&tempty[1], 8);
        mbar_init(drain, 1);
        *abort_flag = 0;
        fence_barrier_init();
        fence_proxy_async_smem();
        tma_prefetch_desc(&tmA);
        tma_prefetch_desc(&tmB0);
        tma_prefetch_desc(&tmB1);
    }
    if (warp == 1) {
        tmem_alloc_pair(tmem_slot, kTmemCols);
        tmem_relinquish_pair();
    }
    // the prologue above overlaps the launch before; from here on its results are read
    griddep_wait();
    griddep_launch_dependents();
    if (threadIdx.x == 64) build_tile_table(p, BMP, mt_prefix, s_off);
    tc_fence_before();
    __syncthreads();
    cluster_sync_all();  // both CTAs' barriers exist before any cross-CTA signal
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;
    const int total_tiles = mt_prefix[p.E] * p.n_tiles;
    const int kblocks = p.K / BK;
    const uint64_t tmo = p.st.timeout_ns;
    const uint32_t full_lead = mapa_shared(smem_u32(full), 0);     // leader's full[0]
    const uint32_t tempty_lead = mapa_shared(smem_u32(tempty), 0);  // leader's tempty[0]

    auto give_up = [&](uint32_t site) {
        report_timeout(p.st, site);
        *abort_flag = 1;
    };

    if (warp == 0) {
        if (lane == 0) {
            // ------------------------------------------------ TMA producer (both CTAs)
            int stage = 0;
            uint32_t phase = 0;
            uint32_t issued_mask = 0, issued_par = 0;
            bool stop = false;
            for (int tile = pair; tile < total_tiles && !stop; tile += npairs) {
                int e, row0, rows, nt;
                decode_tile(tile, mt_prefix, s_off, p.n_tiles, BMP, e, row0, rows, nt);
                // this CTA's rows: 128 of a full tile, 64 of a half (M=128) tile
                const int arow = row0 + (rows <= BMP / 2 ? 64 : 128) * (int)rank;
                const int col0 = (MODE == MODE_SWIGLU) ? nt * 128 + 64 * (int)rank : nt * 256 + 128 * (int)rank;
                for (int kb = 0; kb < kblocks; ++kb) {
                    if (*abort_flag) { stop = true; break; }
                    if (!mbar_wait_bounded(&empty[stage], phase ^ 1u, tmo)) {
                        give_up(SITE_GEMM_PRODUCER_EMPTY);
                        stop = true;
                        break;
                    }
                    if (rank == 0) mbar_arrive_expect_tx(&full[stage], 2 * kStageP);
                    const uint32_t bar = full_lead + 8u * stage;
                    uint8_t* a_dst = sA + stage * kAStageP;
                    uint8_t* b_dst = sB + stage * kBStageP;
                    tma_load_2d_pair(a_dst, &tmA, bar, kb * BK, arow);
                    const int krow = e * p.K + kb * BK;
                    if (MODE == MODE_SWIGLU) {
                        tma_load_2d_pair(b_dst, &tmB0, bar, col0, krow);                // gate
                        tma_load_2d_pair(b_dst + kBBoxBytes, &tmB1, bar, col0, krow);   // up
                    } else {
                        tma_load_2d_pair(b_dst, &tmB0, bar, col0, krow);
                        tma_load_2d_pair(b_dst + kBBoxBytes, &tmB0, bar, col0 + 64, krow);
                    }
                    issued_mask |= 1u << stage;
                    issued_par = (issued_par & ~(1u << stage)) | (phase << stage);
                    if (++stage == kStagesP) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
            }
            // the loads land before the MMAs that read them complete; wait for
            // the last consumer release of every stage this CTA filled
            for (int s = 0; s < kStagesP; ++s)
                if ((issued_mask >> s) & 1u)
                    if (!mbar_wait_bounded(&empty[s], (issued_par >> s) & 1u, tmo)) give_up(SITE_GEMM_PRODUCER_DRAIN);
        }
    } else if (warp == 1) {
        if (lane == 0 && rank == 0) {
            // ------------------------------------------------ MMA issuer (leader CTA)
            int stage = 0;
            uint32_t phase = 0;
            int acc = 0;
            uint32_t acc_phase = 0;
            bool stop = false;
            for (int tile = pair; tile < total_tiles && !stop; tile += npairs) {
                int e, row0, rows, nt;
                decode_tile(tile, mt_prefix, s_off, p.n_tiles, BMP, e, row0, rows, nt);
                const uint32_t idesc = rows <= BMP / 2 ? kIdescPHalf : kIdescP;
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
                    const uint32_t a_addr = smem_u32(sA + stage * kAStageP);
                    const uint32_t b_addr = smem_u32(sB + stage * kBStageP);
#pragma unroll
                    for (int kk = 0; kk < BK / 16; ++kk) {
                        const uint64_t adesc = smem_desc_sw128(a_addr + kk * 32, 16, 1024);
                        const uint64_t bdesc = smem_desc_sw128(b_addr + kk * 2048, kBBoxBytes, 1024);
                        tc_mma_f16_pair(d_tmem, adesc, bdesc, idesc, (kb | kk) != 0 ? 1u : 0u);
                    }
                    tc_commit_pair_mc(&empty[stage], 0x3);
                    if (++stage == kStagesP) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
                if (stop) break;
                tc_commit_pair_mc(&tfull[acc], 0x3);
                acc ^= 1;
                if (acc == 0) acc_phase ^= 1u;
            }
            // every pair MMA has completed before either CTA frees its TMEM
            tc_commit_pair_mc(drain, 0x3);
        }
        if (lane == 0) {
            if (!mbar_wait_bounded(drain, 0, tmo)) give_up(SITE_GEMM_DRAIN);
        }
    } else {
        // ---------------------------------------------------- epilogue (both CTAs)
        const int q = warp & 3;  // TMEM lanes 32q..32q+31 are reachable from this warp
        __nv_bfloat16* wb = s_bias + (warp - 2) * BN_MMA;
        int acc = 0;
        uint32_t acc_phase = 0;
        for (int tile = pair; tile < total_tiles; tile += npairs) {
            const int ab = __shfl_sync(0xffffffffu, *abort_flag, 0);
            if (ab) break;
            int e, row0, rows, nt;
            decode_tile(tile, mt_prefix, s_off, p.n_tiles, BMP, e, row0, rows, nt);
            const bool ok = mbar_wait_bounded(&tfull[acc], acc_phase, tmo);
            if (!__all_sync(0xffffffffu, ok)) {
                if (lane == 0) give_up(SITE_GEMM_EPI_TMEM_FULL);
                break;
            }
            tc_fence_after();
            // full tile: this warp's 32 of the CTA's 128 rows, all 256 columns;
            // half tile: rows 32(q&1).. of the CTA's 64, columns [128(q>>1), +128)
            const bool half = rows <= BMP / 2;
            const int r = half ? 64 * (int)rank + 32 * (q & 1) + lane : 128 * (int)rank + q * 32 + lane;
            const int ncols = half ? 128 : 256;
            const int out0 = nt * p.bn_out + (half ? (q >> 1) * (MODE == MODE_SWIGLU ? 64 : 128) : 0);
            const bool valid = r < rows;
            __nv_bfloat16* orow = p.out + (int64_t)(row0 + (valid ? r : 0)) * p.N;
            const uint32_t tbase = tmem_base + ((uint32_t)(q * 32) << 16) + (uint32_t)(acc * BN_MMA);
            epilogue_pair<MODE>(p, tbase, orow, valid, out0, ncols, e, wb, lane, row_weight(p, row0 + r, valid));
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive_cluster(tempty_lead + 8u * acc);
            acc ^= 1;
            if (acc == 0) acc_phase ^= 1u;
        }
    }
    tc_fence_before();
    __syncthreads();
    cluster_sync_all();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc_pair(tmem_base, kTmemCols);
    }
}

template <int MODE>
cudaError_t launch_pair_mode(const CUtensorMap& a, const CUtensorMap& b0, const CUtensorMap& b1, const GemmParams& p,
                             int64_t rows_cap, cudaStream_t s) {
    static std::atomic<int> max_pairs[64];  // resident clusters per device, 0 until measured
    int dev = 0;
    cudaGetDevice(&dev);
    int pairs_cap = dev < 64 ? max_pairs[dev].load(std::memory_order_acquire) : 0;
    if (pairs_cap <= 0) {
        cudaError_t err =
            cudaFuncSetAttribute(grouped_gemm_pair_kernel<MODE>, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemP);
        if (err != cudaSuccess) return err;
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3(2 * (unsigned)(sm_count() / 2));
        cfg.blockDim = dim3(kThreads);
        cfg.dynamicSmemBytes = kSmemP;
        cudaLaunchAttribute attr;
        attr.id = cudaLaunchAttributeClusterDimension;
        attr.val.clusterDim.x = 2;
        attr.val.clusterDim.y = 1;
        attr.val.clusterDim.z = 1;
        cfg.attrs = &attr;
        cfg.numAttrs = 1;
        int n = 0;
        err = cudaOccupancyMaxActiveClusters(&n, grouped_gemm_pair_kernel<MODE>, &cfg);
        if (err != cudaSuccess || n <= 0) n = sm_count() / 2;
        pairs_cap = n;
        if (dev < 64) max_pairs[dev].store(n, std::memory_order_release);
    }
    const int64_t tiles_upper = (rows_cap / BMP + p.E) * (int64_t)p.n_tiles;
    const int pairs = (int)min64(tiles_upper, (int64_t)pairs_cap);
    if (pairs <= 0) return cudaSuccess;
    return launch_kernel(grouped_gemm_pair_kernel<MODE>, dim3(2 * pairs), dim3(kThreads), kSmemP, s, a, b0, b1, p);
}

}  // namespace

cudaError_t launch_pair_gemm(int mode, const CUtensorMap& a, const CUtensorMap& b0, const CUtensorMap& b1,
                             const gemm::GemmParams& p, int64_t rows_cap, cudaStream_t s) {
    if (mode == gemm::MODE_SWIGLU) return launch_pair_mode<gemm::MODE_SWIGLU>(a, b0, b1, p, rows_cap, s);
    if (mode == gemm::MODE_GELU) return launch_pair_mode<gemm::MODE_GELU>(a, b0, b1, p, rows_cap, s);
    return launch_pair_mode<gemm::MODE_PLAIN>(a, b0, b1, p, rows_cap, s);
}

}  // namespace moe
