// Double quantization of the NSN byproducts (gist.science "NSNQuant ...",
// Technical Summary, Methodology §3, Double Quantization: o, s1 and the
// codebook entries take 4-bit values). s1 takes one of 16 levels of a
// per-head grid uniform in log2, (lo, step) kept in fp32; the level is
// decided in fp64 from the fp64 s1, and a zero token keeps s1 = 0.
#pragma once

#include <math.h>
#include <stdint.h>

namespace nsnq {

__device__ __forceinline__ double dq_s1(double s1, double lo, double step) {
    if (!(s1 > 0.0)) return 0.0;
    double k = step > 0.0 ? round((log2(s1) - lo) / step) : 0.0;
    k = fmin(fmax(k, 0.0), 15.0);
    return exp2(lo + k * step);
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
