// fp32 expert FFNs with plain FMA (no TF32): the precision-reference path of
// the layer for float32 configurations.
//
// Same method as the tensor-core path (SwiGLU or bias+GELU experts over the
// expert-sorted rows; "MoE: gating, experts, load balancing, capacity factor"
// (dpshk.com/news/6005940) §2.2 and §3.1), as a tiled 64x64 SIMT GEMM per
// (expert m-tile, n-tile); the tile list is built from the device offsets.
#include "internal.h"

namespace moe {
namespace {

constexpr int TM = 64, TN = 64, TK = 16;

struct SimtParams {
    const float* A;        // [rows_cap, K]
    const float* B0;       // [E, K, N]
    const float* B1;       // [E, K, N] (SwiGLU up) or null
    const float* bias;     // [E, N] or null
    float* out;            // [rows_cap, N]
    const int32_t* offsets;
    int E, K, N, n_tiles;
};

enum { S_PLAIN = 0, S_SWIGLU = 1, S_GELU = 2 };

template <int MODE>
__global__ void __launch_bounds__(256) simt_gemm_kernel(SimtParams p) {
    __shared__ int mt_prefix[kMaxExperts + 1];
    __shared__ float As[TK][TM + 4];
    __shared__ float Bs[2][TK][TN];
    griddep_wait();  // the rows and offsets of the launches before
    griddep_launch_dependents();
    if (threadIdx.x == 0) {
        int acc = 0;
        mt_prefix[0] = 0;
        for (int e = 0; e < p.E; ++e) {
            acc += (p.offsets[e + 1] - p.offsets[e] + TM - 1) / TM;
            mt_prefix[e + 1] = acc;
        }
    }
    __syncthreads();
    const int tile = blockIdx.x;
    if (tile >= mt_prefix[p.E] * p.n_tiles) return;
    const int mt = tile / p.n_tiles, nt = tile - mt * p.n_tiles;
    int e = 0;
    while (mt_prefix[e + 1] <= mt) ++e;
    const int row0 = p.offsets[e] + (mt - mt_prefix[e]) * TM;
    const int rows = min(TM, p.offsets[e + 1] - row0);
    const int n0 = nt * TN;
    const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
    float acc0[4][4], acc1[4][4];
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc0[i][j] = acc1[i][j] = 0.f;
    const float* Be0 = p.B0 + (int64_t)e * p.K * p.N;
    const float* Be1 = MODE == S_SWIGLU ? p.B1 + (int64_t)e * p.K * p.N : nullptr;
    for (int k0 = 0; k0 < p.K; k0 += TK) {
        for (int i = threadIdx.x; i < TM * TK; i += 256) {
            const int m = i / TK, kk = i - m * TK, k = k0 + kk;
            As[kk][m] = (m < rows && k < p.K) ? p.A[(int64_t)(row0 + m) * p.K + k] : 0.f;
        }
        for (int i = threadIdx.x; i < TK * TN; i += 256) {
            const int kk = i / TN, n = i - kk * TN, k = k0 + kk, col = n0 + n;
            const bool in = k < p.K && col < p.N;
            Bs[0][kk][n] = in ? Be0[(int64_t)k * p.N + col] : 0.f;
            if (MODE == S_SWIGLU) Bs[1][kk][n] = in ? Be1[(int64_t)k * p.N + col] : 0.f;
        }
        __syncthreads();
#pragma unroll
        for (int kk = 0; kk < TK; ++kk) {
            float a[4], b0[4], b1[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) a[i] = As[kk][ty * 4 + i];
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                b0[j] = Bs[0][kk][tx * 4 + j];
                if (MODE == S_SWIGLU) b1[j] = Bs[1][kk][tx * 4 + j];
            }
#pragma unroll
            for (int i = 0; i < 4; ++i)
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    acc0[i][j] = fmaf(a[i], b0[j], acc0[i][j]);
                    if (MODE == S_SWIGLU) acc1[i][j] = fmaf(a[i], b1[j], acc1[i][j]);
                }
        }
        __syncthreads();
    }
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const int m = ty * 4 + i;
        if (m >= rows) continue;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const int col = n0 + tx * 4 + j;
            if (col >= p.N) continue;
            float v = acc0[i][j];
            if (MODE == S_SWIGLU) {
                v = (v / (1.0f + expf(-v))) * acc1[i][j];
            } else {
                if (p.bias) v += p.bias[(int64_t)e * p.N + col];
                if (MODE == S_GELU) v = 0.5f * v * (1.0f + erff(v * 0.70710678118654752f));
            }
            p.out[(int64_t)(row0 + m) * p.N + col] = v;
        }
    }
}

template <int MODE>
cudaError_t launch_simt(const SimtParams& p, int64_t rows_cap, cudaStream_t s) {
    const int64_t tiles = (rows_cap / TM + p.E) * (int64_t)p.n_tiles;
    if (tiles <= 0) return cudaSuccess;
    const cudaError_t err = launch_kernel(simt_gemm_kernel<MODE>, dim3((unsigned)tiles), dim3(256), 0, s, p);
    if (err != cudaSuccess) return err;
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_ffn_f32(const FfnArgs& a, cudaStream_t s) {
    if (a.rows_cap <= 0) return cudaSuccess;
    const bool swiglu = a.act == 0;
    SimtParams p1;
    p1.A = static_cast<const float*>(a.x_perm);
    p1.B0 = static_cast<const float*>(a.w1);
    p1.B1 = static_cast<const float*>(a.w_up);
    p1.bias = swiglu ? nullptr : static_cast<const float*>(a.b1);
    p1.out = static_cast<float*>(a.h);
    p1.offsets = a.offsets;
    p1.E = a.E;
    p1.K = a.d;
    p1.N = a.ffn;
    p1.n_tiles = (a.ffn + TN - 1) / TN;
    cudaError_t err = swiglu ? launch_simt<S_SWIGLU>(p1, a.rows_cap, s) : launch_simt<S_GELU>(p1, a.rows_cap, s);
    if (err != cudaSuccess) return err;
    if (a.between != nullptr && (err = record_mark(a.between, s)) != cudaSuccess) return err;
    SimtParams p2;
    p2.A = static_cast<const float*>(a.h);
    p2.B0 = static_cast<const float*>(a.w2);
    p2.B1 = nullptr;
    p2.bias = swiglu ? nullptr : static_cast<const float*>(a.b2);
    p2.out = static_cast<float*>(a.y_perm);
    p2.offsets = a.offsets;
    p2.E = a.E;
    p2.K = a.ffn;
    p2.N = a.d;
    p2.n_tiles = (a.d + TN - 1) / TN;
    return launch_simt<S_PLAIN>(p2, a.rows_cap, s);
}

}  // namespace moe
