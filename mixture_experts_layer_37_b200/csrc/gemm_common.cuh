// Pieces shared by the two grouped-GEMM kernels (one CTA per tile, and a CTA
// pair per tile with cta_group::2): UMMA descriptors, the tile order over the
// ragged per-expert row groups, the fused activation epilogue, and the TMA
// tensor maps.
#pragma once

#include "internal.h"

namespace moe {
namespace gemm {

constexpr int BK = 64;                      // K per pipeline stage (128 bytes of bf16)
constexpr int BN_MMA = 256;                 // accumulator columns per tile
constexpr int kBBoxBytes = BK * 64 * 2;     // one [64 K x 64 N] weight box, 8 KB
constexpr int kTmemCols = 2 * BN_MMA;       // two fp32 accumulators
constexpr int kThreads = 192;               // producer warp, MMA warp, 4 epilogue warps
constexpr int kGroupM = 32;                 // m-tiles per raster group
constexpr int kBiasBytes = 4 * BN_MMA * 2;  // one bf16 bias row per epilogue warp

enum { MODE_PLAIN = 0, MODE_SWIGLU = 1, MODE_GELU = 2 };

// Instruction descriptor, kind::f16: D fp32 (bits 4-5 = 1), A bf16 (bits 7-9
// = 1), B bf16 (bits 10-12 = 1), A K-major (bit 15 = 0), B MN-major (bit 16
// = 1), N>>3 in bits 17-22, M>>4 in bits 24-28.
constexpr uint32_t make_idesc(int m, int n) {
    return (1u << 4) | (1u << 7) | (1u << 10) | (0u << 15) | (1u << 16) | ((uint32_t)(n >> 3) << 17) |
           ((uint32_t)(m >> 4) << 24);
}

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
    const int32_t* offsets = nullptr;     // [E+1] kept-row offsets per expert
    __nv_bfloat16* out = nullptr;         // [rows_cap, N]
    const __nv_bfloat16* bias = nullptr;  // [E, N] or null
    int E = 0, K = 0, N = 0;
    int bn_out = 0;                       // output columns per tile: 128 (SwiGLU) or 256
    int n_tiles = 0;
    DevStatus st;
    // A rows gathered from the token activations instead of a sorted copy:
    // row s of the expert-sorted order is token src_assign[s] / k of gx
    const __nv_bfloat16* gx = nullptr;    // [T, K] or null (A read through its tensor map)
    const int32_t* src_assign = nullptr;  // [R]
    int k = 0;
    // routing weights of the output rows (second GEMM): row s is multiplied by
    // row_w[src_assign[s]] in fp32, after the bias, before the one rounding; or null
    const float* row_w = nullptr;         // [T*k]
};

__device__ __forceinline__ float silu_f(float x) { return x / (1.0f + __expf(-x)); }
__device__ __forceinline__ float gelu_f(float x) { return 0.5f * x * (1.0f + erff(x * 0.70710678118654752f)); }

// Builds the per-expert m-tile prefix (tiles of `bm` rows) and a copy of the
// offsets in shared memory.  One thread.
__device__ __forceinline__ void build_tile_table(const GemmParams& p, int bm, int* mt_prefix, int* s_off) {
    int acc = 0;
    mt_prefix[0] = 0;
    for (int e = 0; e < p.E; ++e) {
        const int o0 = p.offsets[e], o1 = p.offsets[e + 1];
        s_off[e] = o0;
        acc += (o1 - o0 + bm - 1) / bm;
        mt_prefix[e + 1] = acc;
    }
    s_off[p.E] = p.offsets[p.E];
}

// Tile order: expert by expert; inside an expert, groups of kGroupM m-tiles,
// and inside a group n-tile-major.  The CTAs running at the same time then
// share each weight tile among the group's m-tiles and each activation tile
// among its n-tiles, which keeps an expert's working set in L2 even when its
// weights exceed it.
__device__ __forceinline__ void decode_tile(int tile, const int* mt_prefix, const int* s_off, int n_tiles, int bm,
                                            int& e, int& row0, int& rows, int& nt) {
    e = 0;
    while (mt_prefix[e + 1] * n_tiles <= tile) ++e;
    const int local = tile - mt_prefix[e] * n_tiles;
    const int mt_e = mt_prefix[e + 1] - mt_prefix[e];
    const int grp = local / (kGroupM * n_tiles);
    const int gm = min(kGroupM, mt_e - grp * kGroupM);
    const int r = local - grp * kGroupM * n_tiles;
    nt = r / gm;
    const int mt = grp * kGroupM + (r - nt * gm);
    row0 = s_off[e] + mt * bm;
    rows = min(bm, s_off[e + 1] - row0);
}

// The routing weight of output row `row` (1 without row weights or for a row
// that is not stored).
__device__ __forceinline__ float row_weight(const GemmParams& p, int row, bool valid) {
    return p.row_w != nullptr && valid ? __ldg(p.row_w + __ldg(p.src_assign + row)) : 1.0f;
}

// Epilogue of one warp for one tile: its 32 accumulator rows (TMEM lanes of
// `tbase`), activation (or bias, times the row's routing weight `rw` when the
// GEMM has row weights), one rounding to bf16, and the store of the rows that
// are valid.  `wb` is the warp's 256-entry bias staging row.  Warp-collective.
template <int MODE>
__device__ __forceinline__ void epilogue_rows(const GemmParams& p, uint32_t tbase, __nv_bfloat16* orow, bool valid,
                                              int n0, int e, __nv_bfloat16* wb, int lane, float rw = 1.0f) {
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
        // the tile's 256 bias values, staged once per tile in the warp's own row
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
                uint4* dst = reinterpret_cast<uint4*>(orow + n0 + c);
                dst[0] = make_uint4(pk[0], pk[1], pk[2], pk[3]);
                dst[1] = make_uint4(pk[4], pk[5], pk[6], pk[7]);
            }
        }
    }
}

// 2-D bf16 tensor [outer, inner] (inner contiguous, row pitch `pitch` bytes),
// box [box_outer, box_inner], 128-byte swizzle, zero fill out of bounds.
bool make_map(CUtensorMap* m, const void* base, uint64_t inner, uint64_t outer, uint64_t pitch, uint32_t box_inner,
              uint32_t box_outer);
// The same for any element type, without swizzle (rows land in shared memory as they are in memory).
bool make_map_plain(CUtensorMap* m, CUtensorMapDataType dtype, const void* base, uint64_t inner, uint64_t outer,
                    uint64_t pitch, uint32_t box_inner, uint32_t box_outer);

}  // namespace gemm
}  // namespace moe
