/*
 * Seeded synthetic input generator shared by the CUDA tests, the bench and
 * the CPU oracle's tests.  It holds no arithmetic of the MoE layer itself:
 * it only turns (seed, stream, index) into numbers.
 *
 * Counter-based: element i of stream s under seed S is a pure function of
 * (S, s, i), so any slice of any tensor can be generated independently and
 * in parallel, and a token subset can be regenerated without the rest.
 *
 * Bits:    SplitMix64 finaliser (G. Steele, D. Lea, C. Flood, "Fast
 *          splittable pseudorandom number generators", OOPSLA 2014; constants
 *          as published by S. Vigna) applied to key + (i+1)*golden-gamma.
 * Uniform: top 53 bits, centred: u = (bits>>11 + 0.5) * 2^-53, in (0,1).
 * Normal:  Box-Muller (G. Box, M. Muller, Ann. Math. Stat. 1958) on the pair
 *          (u(2m), u(2m+1)); element 2m takes the cosine branch, 2m+1 the sine.
 * Output:  double -> float by C conversion (round to nearest even), and for
 *          bf16 float -> bf16 by round-to-nearest-even on the bit pattern.
 */
#include <math.h>
#include <stdint.h>
#include <string.h>

#define GOLDEN_GAMMA 0x9e3779b97f4a7c15ULL

static inline uint64_t mix64(uint64_t z) {
    z = (z ^ (z >> 30)) * 0xbf58476d1ce4e5b9ULL;
    z = (z ^ (z >> 27)) * 0x94d049bb133111ebULL;
    return z ^ (z >> 31);
}

/* Per-(seed, stream) key: two rounds so that nearby seeds/streams decorrelate. */
uint64_t wl_stream_key(uint64_t seed, uint64_t stream) {
    return mix64(mix64(seed + GOLDEN_GAMMA) ^ (stream * 0xd1b54a32d192ed03ULL + 0x8bb84b93962eacc9ULL));
}

static inline double uniform_at(uint64_t key, uint64_t i) {
    uint64_t b = mix64(key + (i + 1) * GOLDEN_GAMMA);
    return ((double)(b >> 11) + 0.5) * (1.0 / 9007199254740992.0);
}

static inline double normal_at(uint64_t key, uint64_t i) {
    uint64_t m = i >> 1;
    double u1 = uniform_at(key, 2 * m);
    double u2 = uniform_at(key, 2 * m + 1);
    double r = sqrt(-2.0 * log(u1));
    double a = 6.283185307179586476925286766559 * u2;
    return (i & 1) ? r * sin(a) : r * cos(a);
}

static inline uint16_t f32_to_bf16_rne(float f) {
    uint32_t u;
    memcpy(&u, &f, 4);
    if ((u & 0x7f800000u) == 0x7f800000u) {            /* inf / nan: keep, quiet nan */
        return (uint16_t)((u >> 16) | ((u & 0xffffu) ? 0x40u : 0u));
    }
    u += 0x7fffu + ((u >> 16) & 1u);
    return (uint16_t)(u >> 16);
}

void wl_uniform_f64(uint64_t seed, uint64_t stream, uint64_t start, int64_t n, double* out) {
    uint64_t key = wl_stream_key(seed, stream);
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < n; ++i) out[i] = uniform_at(key, start + (uint64_t)i);
}

void wl_normal_f32(uint64_t seed, uint64_t stream, uint64_t start, int64_t n,
                   double mean, double std, float* out) {
    uint64_t key = wl_stream_key(seed, stream);
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < n; ++i) out[i] = (float)(mean + std * normal_at(key, start + (uint64_t)i));
}

void wl_normal_bf16(uint64_t seed, uint64_t stream, uint64_t start, int64_t n,
                    double mean, double std, uint16_t* out) {
    uint64_t key = wl_stream_key(seed, stream);
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < n; ++i)
        out[i] = f32_to_bf16_rne((float)(mean + std * normal_at(key, start + (uint64_t)i)));
}

/* Gather-generation: element idx[r] of a stream, for r < n (used to build
 * token subsets of a [T, d] tensor without generating the rest). */
void wl_normal_bf16_rows(uint64_t seed, uint64_t stream, const int64_t* rows, int64_t nrows,
                         int64_t row_len, double mean, double std, uint16_t* out) {
    uint64_t key = wl_stream_key(seed, stream);
#pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < nrows; ++r)
        for (int64_t c = 0; c < row_len; ++c)
            out[r * row_len + c] = f32_to_bf16_rne(
                (float)(mean + std * normal_at(key, (uint64_t)(rows[r] * row_len + c))));
}
