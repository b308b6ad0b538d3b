// Routed experts with INT8 weights: quantisation, and the expert FFNs on
// INT8 weights with a per-expert, per-output-channel scale.
//
// Method ("Million-token-context MoE memory" (2kiu.com/news/5130654) §3):
// expert weights stored as INT8 codes times a scale computed per expert and
// per dimension, dequantised for use.  Here: s[e,n] = max_k |W[e,k,n]| / 127,
// q = clamp(rint(W / s), -127, 127) (ties to even), both in fp32; the FFN
// computes  s[e,n] * sum_k x[k] q[e,k,n]  (fp32 accumulation), which is the
// product with the dequantised weights q*s.
//
// The FFN kernel is built for decode-sized batches, where an expert holds a
// handful of rows and the layer time is the time to stream the weights.  One
// CTA per (expert, 128-column tile), two CTAs per SM, 288 threads:
//   warp 0, lane 0   producer: per stage one TMA tile of codes [64 K x 128
//                    columns] (two for SwiGLU: gate and up) and one of the
//                    expert's activations [4 rows x 64 K], 4 stages;
//   warps 1-8        each takes 8 of a stage's 64 K rows for all 128 columns
//                    (4 per lane: one 4-byte load of codes per K row), only
//                    as many activation rows as the pass holds (up to 4);
//                    codes become fp32 by a byte permute and one packed
//                    subtraction per two codes, and the FMAs run two at a
//                    time (f32x2, each rounded as a scalar fmaf); the eight
//                    partial sums are added in warp order and the scale (and
//                    bias / activation) applied once per output.
// 128-column tiles give the decode workload's ~57 busy experts 16 tiles each,
// about 6 per SM: the last partial wave costs little.
// Weight bytes per element: 1 instead of 2.  An expert with more than 4 rows
// streams its weights once per 4 rows (correct, slow for large batches).
// Every wait is bounded in time, as in the other kernels.
#include <math.h>

#include "gemm_common.cuh"

namespace moe {
namespace {

constexpr int kQThreads = 288;             // producer warp + 8 consumer warps
constexpr int kQWarps = 8;                  // consumer warps: each takes 8 of a stage's 64 K rows
constexpr int kQCols = 128;                 // output columns per CTA (4 per consumer lane)
constexpr int kQKB = 64;                    // K rows per stage
constexpr int kQRows = 4;                   // expert rows per pass
constexpr int kQStages = 4;
constexpr int kQWTile = kQKB * kQCols;      // 8 KB of codes
constexpr int kQXTile = kQRows * kQKB * 2;  // 512 B of bf16 activations
constexpr int kQStage = 2 * kQWTile + kQXTile;
constexpr int kQRed = kQWarps * kQRows * kQCols * 2 * 4;  // partial sums of the 8 warps (32 KB)
constexpr int kQSmem = kQStages * kQStage + kQRed + 256 + 128;
static_assert(kQKB / kQWarps == 8, "a consumer warp takes 8 K rows: one 16-byte load of activations per row");
static_assert(kQStage % 128 == 0, "stages stay 128-byte aligned");

enum { Q_SWIGLU = 0, Q_GELU = 1, Q_PLAIN = 2, Q_PLAIN_BIAS = 3 };

// One thread per (expert, column): the column's absolute maximum over K, the
// scale, then the codes.
template <bool BF16>
__global__ void __launch_bounds__(256) quantize_kernel(const void* __restrict__ w, int64_t K, int64_t N,
                                                       int8_t* __restrict__ q, float* __restrict__ scale) {
    const int64_t n = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    const int64_t e = blockIdx.y;
    if (n >= N) return;
    auto load = [&](int64_t k) -> float {
        const int64_t i = (e * K + k) * N + n;
        if constexpr (BF16) return __bfloat162float(static_cast<const __nv_bfloat16*>(w)[i]);
        return static_cast<const float*>(w)[i];
    };
    float amax = 0.f;
    for (int64_t k = 0; k < K; ++k) amax = fmaxf(amax, fabsf(load(k)));
    const float s = amax / 127.0f;
    scale[e * N + n] = s;
    for (int64_t k = 0; k < K; ++k) {
        int code = 0;
        if (s > 0.f) {
            const float v = rintf(load(k) / s);
            code = (int)fminf(fmaxf(v, -127.f), 127.f);
        }
        q[(e * K + k) * N + n] = (int8_t)code;
    }
}

struct QArgs {
    const int32_t* offsets = nullptr;     // [E+1] rows of each expert in the activations
    const float* s0 = nullptr;            // [E, N] scales (gate / W1 / W2)
    const float* s1 = nullptr;            // [E, N] scales (up) or null
    const __nv_bfloat16* bias = nullptr;  // [E, N] or null
    __nv_bfloat16* out = nullptr;         // [rows, N]
    int K = 0, N = 0;
    DevStatus st;
};

__device__ __forceinline__ float silu_q(float x) { return x / (1.0f + __expf(-x)); }
__device__ __forceinline__ float gelu_q(float x) { return 0.5f * x * (1.0f + erff(x * 0.70710678118654752f)); }

// Packed pairs of fp32 values (the f32x2 arithmetic of sm_100: two independent
// fp32 operations per instruction, each rounded as its scalar form).
__device__ __forceinline__ uint64_t pack2(uint32_t lo, uint32_t hi) {
    uint64_t r;
    asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "r"(lo), "r"(hi));
    return r;
}
__device__ __forceinline__ void unpack2(uint64_t v, float& lo, float& hi) {
    asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(v));
}
__device__ __forceinline__ uint64_t fma2(uint64_t a, uint64_t b, uint64_t c) {
    uint64_t r;
    asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(r) : "l"(a), "l"(b), "l"(c));
    return r;
}
__device__ __forceinline__ uint64_t sub2(uint64_t a, uint64_t b) {
    uint64_t r;
    asm("sub.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
    return r;
}

// Four int8 codes (one 32-bit word) to exact floats, as two packed pairs,
// without the integer conversion unit: with the sign bit flipped a code b
// becomes the unsigned byte u = b + 128; placed as the low mantissa byte of
// 2^23 (bit pattern 0x4B0000uu) it reads as 2^23 + u, and subtracting
// 2^23 + 128 leaves b exactly.
__device__ __forceinline__ void codes_to_pairs(uint32_t word, uint64_t* f) {
    const uint32_t u = word ^ 0x80808080u;
    uint32_t bits[4];
#pragma unroll
    for (int j = 0; j < 4; ++j)
        // bytes of {0x4B000000 : u}: result = [u.byte j, 0x00, 0x00, 0x4B]
        asm("prmt.b32 %0, %1, %2, %3;" : "=r"(bits[j]) : "r"(u), "r"(0x4B000000u), "r"(0x7540u | (uint32_t)j));
    const uint32_t m = __float_as_uint(8388736.0f);
    const uint64_t magic = pack2(m, m);
    f[0] = sub2(pack2(bits[0], bits[1]), magic);
    f[1] = sub2(pack2(bits[2], bits[3]), magic);
}

// One consumer warp's share of a stage: K rows [8w, 8w+8), all 128 columns
// (4 per lane, as two packed pairs), the first RT activation rows.
template <bool TWO, int RT>
__device__ __forceinline__ void consume_stage(const uint8_t* st, int w, int lane, uint64_t (&acc0)[kQRows][2],
                                              uint64_t (&acc1)[kQRows][2]) {
    const uint32_t* w0 = reinterpret_cast<const uint32_t*>(st) + lane;
    const uint32_t* w1 = reinterpret_cast<const uint32_t*>(st + kQWTile) + lane;
    const __nv_bfloat16* xs = reinterpret_cast<const __nv_bfloat16*>(st + 2 * kQWTile);
    // the warp's 8 activation values of each row, one 16-byte load per row (a bf16
    // value widens to fp32 exactly by moving its bits to the upper half)
    uint32_t xw[RT][4];
#pragma unroll
    for (int r = 0; r < RT; ++r) {
        const uint4 v = *reinterpret_cast<const uint4*>(xs + r * kQKB + w * (kQKB / kQWarps));
        xw[r][0] = v.x;
        xw[r][1] = v.y;
        xw[r][2] = v.z;
        xw[r][3] = v.w;
    }
#pragma unroll
    for (int i = 0; i < kQKB / kQWarps; ++i) {
        const int kk = w * (kQKB / kQWarps) + i;
        const uint32_t q0 = w0[kk * (kQCols / 4)];
        const uint32_t q1 = TWO ? w1[kk * (kQCols / 4)] : 0u;
        uint64_t c0[2], c1[2];
        codes_to_pairs(q0, c0);
        if (TWO) codes_to_pairs(q1, c1);
#pragma unroll
        for (int r = 0; r < RT; ++r) {
            const uint32_t h = xw[r][i >> 1];
            const uint32_t xb = (i & 1) ? (h & 0xFFFF0000u) : (h << 16);
            const uint64_t xv = pack2(xb, xb);
#pragma unroll
            for (int j = 0; j < 2; ++j) {
                acc0[r][j] = fma2(xv, c0[j], acc0[r][j]);
                if (TWO) acc1[r][j] = fma2(xv, c1[j], acc1[r][j]);
            }
        }
    }
}

// tmQ0/tmQ1: codes as a 2-D uint8 tensor [E*K, N], box [64 rows, 128 columns];
// tmA: activations [rows, K] bf16, box [4 rows, 64 K].
template <int MODE>
__global__ void __launch_bounds__(kQThreads, 2) ffn_int8_kernel(const __grid_constant__ CUtensorMap tmQ0,
                                                               const __grid_constant__ CUtensorMap tmQ1,
                                                               const __grid_constant__ CUtensorMap tmA, QArgs p) {
    constexpr bool TWO = MODE == Q_SWIGLU;
    constexpr uint32_t kBytes = (TWO ? 2 : 1) * kQWTile + kQXTile;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = smem_raw + ((128u - (smem_u32(smem_raw) & 127u)) & 127u);
    float* red = reinterpret_cast<float*>(smem + kQStages * kQStage);  // [warp][2][row][kQCols]
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + kQStages * kQStage + kQRed);
    uint64_t* empty = full + kQStages;
    volatile int* abort_flag = reinterpret_cast<volatile int*>(empty + kQStages);
    griddep_wait();  // the rows and offsets of the launches before
    griddep_launch_dependents();
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int e = blockIdx.y;
    const int row_begin = p.offsets[e], row_end = p.offsets[e + 1];
    const int n0 = blockIdx.x * kQCols;
    const int kblocks = p.K / kQKB;
    const uint64_t tmo = p.st.timeout_ns;
    if (row_begin >= row_end) return;  // no rows: nothing loaded, nothing written
    if (threadIdx.x == 0) {
        for (int s = 0; s < kQStages; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], kQWarps);
        }
        *abort_flag = 0;
        fence_barrier_init();
    }
    __syncthreads();
    auto give_up = [&](uint32_t site) {
        report_timeout(p.st, site);
        *abort_flag = 1;
    };

    if (warp == 0) {
        if (lane == 0) {
            int stage = 0;
            uint32_t phase = 0, issued_mask = 0, issued_par = 0;
            bool stop = false;
            for (int r0 = row_begin; r0 < row_end && !stop; r0 += kQRows) {
                for (int kb = 0; kb < kblocks; ++kb) {
                    if (*abort_flag) { stop = true; break; }
                    if (!mbar_wait_bounded(&empty[stage], phase ^ 1u, tmo)) {
                        give_up(SITE_GEMM_PRODUCER_EMPTY);
                        stop = true;
                        break;
                    }
                    uint8_t* st = smem + stage * kQStage;
                    mbar_arrive_expect_tx(&full[stage], kBytes);
                    const int krow = e * p.K + kb * kQKB;
                    tma_load_2d(st, &tmQ0, &full[stage], n0, krow);
                    if (TWO) tma_load_2d(st + kQWTile, &tmQ1, &full[stage], n0, krow);
                    tma_load_2d(st + 2 * kQWTile, &tmA, &full[stage], kb * kQKB, r0);
                    issued_mask |= 1u << stage;
                    issued_par = (issued_par & ~(1u << stage)) | (phase << stage);
                    if (++stage == kQStages) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
            }
            for (int s = 0; s < kQStages; ++s)
                if ((issued_mask >> s) & 1u)
                    if (!mbar_wait_bounded(&full[s], (issued_par >> s) & 1u, tmo)) give_up(SITE_GEMM_PRODUCER_DRAIN);
        }
    } else {
        const int w = warp - 1;  // consumer warp 0..7
        int stage = 0;
        uint32_t phase = 0;
        bool ok = true;  // the same in all four warps: set from the shared abort flag after each barrier
        for (int r0 = row_begin; r0 < row_end && ok; r0 += kQRows) {
            const int nr = min(kQRows, row_end - r0);
            uint64_t acc0[kQRows][2], acc1[kQRows][2];
#pragma unroll
            for (int r = 0; r < kQRows; ++r)
#pragma unroll
                for (int j = 0; j < 2; ++j) acc0[r][j] = acc1[r][j] = 0ull;  // +0.0f pairs
            for (int kb = 0; kb < kblocks; ++kb) {
                if (__shfl_sync(0xffffffffu, *abort_flag, 0)) { ok = false; break; }
                const bool got = mbar_wait_bounded(&full[stage], phase, tmo);
                if (!__all_sync(0xffffffffu, got)) {
                    if (lane == 0) give_up(SITE_GEMM_MMA_FULL);
                    ok = false;
                    break;
                }
                const uint8_t* st = smem + stage * kQStage;
                // only the rows this pass holds (decode: one or two)
                if (nr <= 1) consume_stage<TWO, 1>(st, w, lane, acc0, acc1);
                else if (nr == 2) consume_stage<TWO, 2>(st, w, lane, acc0, acc1);
                else if (nr == 3) consume_stage<TWO, 3>(st, w, lane, acc0, acc1);
                else consume_stage<TWO, 4>(st, w, lane, acc0, acc1);
                __syncwarp();
                if (lane == 0) mbar_arrive(&empty[stage]);
                if (++stage == kQStages) {
                    stage = 0;
                    phase ^= 1u;
                }
            }
            // the eight warps' partial sums, added in warp order, then the epilogue;
            // every consumer warp arrives here whether or not its loop gave up
            named_barrier_sync(1, kQWarps * 32);
            ok = !*abort_flag;
            if (ok) {
                for (int r = 0; r < nr; ++r)
#pragma unroll
                    for (int j = 0; j < 2; ++j) {
                        float* d0 = red + ((w * 2 + 0) * kQRows + r) * kQCols + 4 * lane + 2 * j;
                        unpack2(acc0[r][j], d0[0], d0[1]);
                        if (TWO) {
                            float* d1 = red + ((w * 2 + 1) * kQRows + r) * kQCols + 4 * lane + 2 * j;
                            unpack2(acc1[r][j], d1[0], d1[1]);
                        }
                    }
            }
            named_barrier_sync(1, kQWarps * 32);
            if (ok) {
                // consumer thread t finishes output t of each row
                const int t = w * 32 + lane;
                for (int r = 0; r < nr; ++r) {
                    for (int cc = t; cc < kQCols; cc += kQWarps * 32) {
                        const int n = n0 + cc;
                        if (n >= p.N) continue;
                        float g = 0.f, u = 0.f;
#pragma unroll
                        for (int ww = 0; ww < kQWarps; ++ww) {
                            g += red[((ww * 2 + 0) * kQRows + r) * kQCols + cc];
                            if (TWO) u += red[((ww * 2 + 1) * kQRows + r) * kQCols + cc];
                        }
                        g *= p.s0[(int64_t)e * p.N + n];
                        float v;
                        if (MODE == Q_SWIGLU) v = silu_q(g) * (u * p.s1[(int64_t)e * p.N + n]);
                        else if (MODE == Q_GELU) v = gelu_q(g + __bfloat162float(p.bias[(int64_t)e * p.N + n]));
                        else if (MODE == Q_PLAIN_BIAS) v = g + __bfloat162float(p.bias[(int64_t)e * p.N + n]);
                        else v = g;
                        p.out[(int64_t)(r0 + r) * p.N + n] = __float2bfloat16_rn(v);
                    }
                }
            }
            named_barrier_sync(1, kQWarps * 32);  // the partials are read before the next pass rewrites them
        }
    }
}

template <int MODE>
cudaError_t launch_q(const CUtensorMap& q0, const CUtensorMap& q1, const CUtensorMap& a, const QArgs& p, int E,
                     cudaStream_t s) {
    static std::atomic<bool> attr[64];
    const cudaError_t err = ensure_smem_attr(attr, ffn_int8_kernel<MODE>, kQSmem);
    if (err != cudaSuccess) return err;
    dim3 grid((p.N + kQCols - 1) / kQCols, E);
    return launch_kernel(ffn_int8_kernel<MODE>, grid, dim3(kQThreads), kQSmem, s, q0, q1, a, p);
}

}  // namespace

cudaError_t launch_quantize_int8(const void* w, bool bf16, int64_t E, int64_t K, int64_t N, int8_t* q, float* scale,
                                 cudaStream_t s) {
    if (E == 0 || K == 0 || N == 0) return cudaSuccess;
    dim3 grid((unsigned)((N + 255) / 256), (unsigned)E);
    if (bf16)
        quantize_kernel<true><<<grid, 256, 0, s>>>(w, K, N, q, scale);
    else
        quantize_kernel<false><<<grid, 256, 0, s>>>(w, K, N, q, scale);
    return cudaGetLastError();
}

cudaError_t launch_ffn_int8(const FfnArgs& a, cudaStream_t s) {
    if (a.rows_cap <= 0) return cudaSuccess;
    const bool swiglu = a.act == 0;
    // codes [E*K, N] (uint8 view), activations / intermediate [rows_cap, K] bf16
    CUtensorMap q1a, q1b, x1, q2, x2;
    bool ok = gemm::make_map_plain(&q1a, CU_TENSOR_MAP_DATA_TYPE_UINT8, a.w1, (uint64_t)a.ffn, (uint64_t)a.E * a.d,
                                   (uint64_t)a.ffn, kQCols, kQKB);
    ok = ok && gemm::make_map_plain(&q1b, CU_TENSOR_MAP_DATA_TYPE_UINT8, swiglu ? a.w_up : a.w1, (uint64_t)a.ffn,
                                    (uint64_t)a.E * a.d, (uint64_t)a.ffn, kQCols, kQKB);
    ok = ok && gemm::make_map_plain(&x1, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, a.x_perm, (uint64_t)a.d,
                                    (uint64_t)a.rows_cap, (uint64_t)a.d * 2, kQKB, kQRows);
    ok = ok && gemm::make_map_plain(&q2, CU_TENSOR_MAP_DATA_TYPE_UINT8, a.w2, (uint64_t)a.d, (uint64_t)a.E * a.ffn,
                                    (uint64_t)a.d, kQCols, kQKB);
    ok = ok && gemm::make_map_plain(&x2, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, a.h, (uint64_t)a.ffn, (uint64_t)a.rows_cap,
                                    (uint64_t)a.ffn * 2, kQKB, kQRows);
    if (!ok) return cudaErrorInvalidValue;
    QArgs p1;
    p1.offsets = a.offsets;
    p1.s0 = a.w1_scale;
    p1.s1 = swiglu ? a.w_up_scale : nullptr;
    p1.bias = swiglu ? nullptr : static_cast<const __nv_bfloat16*>(a.b1);
    p1.out = static_cast<__nv_bfloat16*>(a.h);
    p1.K = a.d;
    p1.N = a.ffn;
    p1.st = a.st;
    cudaError_t err = swiglu ? launch_q<Q_SWIGLU>(q1a, q1b, x1, p1, a.E, s) : launch_q<Q_GELU>(q1a, q1b, x1, p1, a.E, s);
    if (err != cudaSuccess) return err;
    if (a.between != nullptr && (err = record_mark(a.between, s)) != cudaSuccess) return err;
    QArgs p2;
    p2.offsets = a.offsets;
    p2.s0 = a.w2_scale;
    p2.bias = swiglu ? nullptr : static_cast<const __nv_bfloat16*>(a.b2);
    p2.out = static_cast<__nv_bfloat16*>(a.y_perm);
    p2.K = a.ffn;
    p2.N = a.d;
    p2.st = a.st;
    return swiglu ? launch_q<Q_PLAIN>(q2, q2, x2, p2, a.E, s) : launch_q<Q_PLAIN_BIAS>(q2, q2, x2, p2, a.E, s);
}

}  // namespace moe
