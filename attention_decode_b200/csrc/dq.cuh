// Double quantization of the NSN byproducts (gist.science "NSNQuant ...",
// Technical Summary, Methodology §3, Double Quantization: o, s1 and the
// codebook entries take 4-bit values). s1 takes one of 16 levels of a
// per-head grid uniform in log2, (lo, step) kept in fp32; the level is
// decided in fp64 from the fp64 s1, and a zero token keeps s1 = 0.
#pragma once

#include <math.h>
#include <stdint.h>

namespace nsnq {

// The level of s1 on the grid (-1 for s1 = 0) and its value 2^(lo + k step).
__device__ __forceinline__ double dq_s1(double s1, double lo, double step, int* level = nullptr) {
    if (!(s1 > 0.0)) {
        if (level) *level = -1;
        return 0.0;
    }
    double k = step > 0.0 ? round((log2(s1) - lo) / step) : 0.0;
    k = fmin(fmax(k, 0.0), 15.0);
    if (level) *level = (int)k;
    return exp2(lo + k * step);
}

// Level value as every reader of a packed cache evaluates it (fp64, then fp32),
// equal to the fp32 s1 an encoder stores for that level.
__device__ __forceinline__ float dq_level_value(const float* s1_grid, int64_t bh, int k) {
    return (float)exp2((double)s1_grid[2 * bh] + (double)k * (double)s1_grid[2 * bh + 1]);
}

// The 4-bit s1 level of token position pos in a packed cache's level words.
__device__ __forceinline__ int dq_packed_level(const uint32_t* levels, int64_t bh, int64_t cap,
                                               int64_t pos) {
    return (int)((levels[bh * ((cap + 7) >> 3) + (pos >> 3)] >> (4 * (int)(pos & 7))) & 15u);
}

// Writes one token's byproducts: the (s1, s2) pair, or in the packed form s2
// alone (sign bit set for a token with s1 = 0, level < 0) and the 4-bit level.
// Two atomics keep the neighbouring tokens' nibbles of the word intact.
__device__ __forceinline__ void store_byproducts(float* scales, uint32_t* levels, int64_t bh,
                                                 int64_t cap, int64_t pos, float s1, float s2,
                                                 int level) {
    const int64_t row = bh * cap + pos;
    if (levels) {
        scales[row] = level < 0 ? __int_as_float(__float_as_int(s2) | (int)0x80000000) : s2;
        uint32_t* w = levels + bh * ((cap + 7) >> 3) + (pos >> 3);
        const int sh = 4 * (int)(pos & 7);
        atomicAnd(w, ~(0xFu << sh));
        atomicOr(w, (uint32_t)(level < 0 ? 0 : level) << sh);
    } else {
        reinterpret_cast<float2*>(scales)[row] = make_float2(s1, s2);
    }
}

// Level tables of a grid, for deciding many tokens of one head without a
// log2/exp2 per token: lvl[k] = 2^(lo + k step) (k < 16), thr[k] =
// 2^(lo + (k + 1/2) step) (k < 15), inv[k] = 1 / lvl[k]. Built by threads
// 0..15 of a block.
__device__ __forceinline__ void dq_table_build(double lo, double step, double* lvl, double* thr,
                                               double* inv) {
    const int k = threadIdx.x;
    if (k < 16) {
        lvl[k] = exp2(lo + (double)k * step);
        inv[k] = 1.0 / lvl[k];
        if (k < 15) thr[k] = exp2(lo + ((double)k + 0.5) * step);
    }
}

// The level dq_s1 picks for s1 > 0, by counting the thresholds at or below
// s1; -1 when s1 lies within a relative 1e-12 of a threshold, where the
// rounding of the log2 form decides (the caller then uses dq_s1). Away from
// the thresholds the two agree exactly: the log2 form's error is ~1e-16.
__device__ __forceinline__ int dq_level(double s1, double step, const double* thr) {
    if (!(step > 0.0)) return 0;
    int k = 0;
#pragma unroll
    for (int i = 0; i < 15; ++i) k += s1 >= thr[i] ? 1 : 0;
    const double lo_t = k > 0 ? thr[k - 1] : 0.0, hi_t = k < 15 ? thr[k] : INFINITY;
    if (s1 - lo_t <= 1e-12 * s1 || hi_t - s1 <= 1e-12 * s1) return -1;
    return k;
}

// The grid of head bh from its fp32 copy.
__device__ __forceinline__ void dq_grid(const float* s1_grid, int64_t bh, double& lo, double& step) {
    lo = (double)s1_grid[2 * bh];
    step = (double)s1_grid[2 * bh + 1];
}

// The grid from the per-chunk least / largest log2 s1 (+inf / -inf for a
// chunk without a non-zero token), rounded to fp32 as it is stored.
__device__ __forceinline__ void dq_grid_from_chunks(const double* minmax, int nchunk, double& lo,
                                                    double& step) {
    double mn = INFINITY, mx = -INFINITY;
    for (int k = 0; k < nchunk; ++k) {
        mn = fmin(mn, minmax[2 * k]);
        mx = fmax(mx, minmax[2 * k + 1]);
    }
    if (!(mn <= mx)) {  // no non-zero token
        lo = 0.0;
        step = 0.0;
        return;
    }
    lo = (double)(float)mn;
    step = (double)(float)((mx - mn) / 15.0);
}

}  // namespace nsnq
