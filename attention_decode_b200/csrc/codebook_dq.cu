// Double quantization of a codebook (gist.science "NSNQuant ...", Technical
// Summary, Methodology §3, Double Quantization: the codebook entries take
// 4-bit values). Every entry of the codebook is put on one shared grid of 16
// uniform levels spanning the entries' least to largest value; the level is
// the nearest one (halves away from zero), decided in fp64.
#include <math.h>

#include "common.cuh"
#include "internal.h"

namespace nsnq {

namespace {

constexpr int kQ4Threads = 256;

__global__ void __launch_bounds__(kQ4Threads) codebook_q4_kernel(const float* in, float* out,
                                                                 uint8_t* levels, double* grid,
                                                                 int n) {
    __shared__ float red_lo[kQ4Threads / 32], red_hi[kQ4Threads / 32];
    const int tid = threadIdx.x, lane = lane_id(), warp = tid >> 5;
    float lo = INFINITY, hi = -INFINITY;
    for (int i = tid; i < n; i += kQ4Threads) {
        lo = fminf(lo, in[i]);
        hi = fmaxf(hi, in[i]);
    }
#pragma unroll
    for (int m = 16; m; m >>= 1) {
        lo = fminf(lo, __shfl_xor_sync(kFull, lo, m));
        hi = fmaxf(hi, __shfl_xor_sync(kFull, hi, m));
    }
    if (lane == 0) { red_lo[warp] = lo; red_hi[warp] = hi; }
    __syncthreads();  // every entry has been read once before any is written (out may be in)
    lo = red_lo[0];
    hi = red_hi[0];
#pragma unroll
    for (int w = 1; w < kQ4Threads / 32; ++w) {
        lo = fminf(lo, red_lo[w]);
        hi = fmaxf(hi, red_hi[w]);
    }
    const double dlo = (double)lo;
    const double step = ((double)hi - dlo) / 15.0;
    // Thread i owns entries 2i and 2i + 1 (one byte of levels).
    for (int p = tid; 2 * p < n; p += kQ4Threads) {
        uint32_t nib = 0;
#pragma unroll
        for (int e = 0; e < 2; ++e) {
            const int i = 2 * p + e;
            if (i >= n) break;
            const double k = step > 0.0 ? round(((double)in[i] - dlo) / step) : 0.0;
            out[i] = (float)(dlo + k * step);
            nib |= (uint32_t)k << (4 * e);
        }
        if (levels) levels[p] = (uint8_t)nib;
    }
    if (grid && tid == 0) {
        grid[0] = dlo;
        grid[1] = step;
    }
}

}  // namespace

cudaError_t launch_codebook_q4(const float* in, float* out, uint8_t* levels, double* grid, int n,
                               cudaStream_t s) {
    codebook_q4_kernel<<<1, kQ4Threads, 0, s>>>(in, out, levels, grid, n);
    return cudaGetLastError();
}

}  // namespace nsnq
