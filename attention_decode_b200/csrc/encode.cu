// NSNQuant encode on sm_100a: Normalize-Shift-Normalize, Hadamard transform
// and nearest-codeword vector quantization (gist.science "NSNQuant ...",
// Technical Summary, Methodology §1-§3).
//
// Two launches per call in shift-compute mode (three with double
// quantization), one in shift-given mode:
//   nsn_s1minmax_kernel per (b, h, chunk), double quantization only: least and
//                      largest log2 s1 (the per-head s1 grid)
//   nsn_stats_kernel   per (b, h, chunk): channel sums of y = x / s1 in fp64;
//                      the last chunk of a (b, h) to finish computes
//                      o = sum / T (fp64, kept in the workspace for the
//                      near-tie path) and its fp32 copy in the cache
//   pass 2             NSN + FWHT + nearest codeword: encode_pruned.cu
//                      (2 bit, search index) or encode1_tc.cu (1 bit, and
//                      2 bit with the tensor-core search: all codewords
//                      scored on the tensor cores); calls of at most
//                      kSmallEncode token-heads: encode_small.cu (one warp
//                      per token-head, fp32 scan, fp64 near ties)
// Pass 2 is a programmatic dependent launch of pass 1 (pass 1 triggers its
// dependents first; pass 2 stages its tables, then waits for the shift).
#include <math.h>

#include "common.cuh"
#include "dq.cuh"
#include "internal.h"

namespace nsnq {

constexpr int kStatsThreads = 256;

// --------------------------------------------------------------- pass 1 --
// Pass-1 lane layout: 16 lanes per token (8 channels each, one 16-byte load
// for bf16), 2 tokens per warp step, stats_depth<XT> steps of loads in
// flight per warp (64 bytes per lane: the kernel streams x once from HBM and
// needs the bytes in flight to cover the latency); at most 64 registers so
// that four CTAs fit on an SM and the usual grids run in one wave.
template <typename XT>
constexpr int stats_depth() { return sizeof(XT) == 2 ? 4 : 2; }

template <typename XT>
struct Raw8;
template <>
struct Raw8<__nv_bfloat16> {
    uint4 u;
    __device__ __forceinline__ void load(const __nv_bfloat16* p) { u = __ldg(reinterpret_cast<const uint4*>(p)); }
    __device__ __forceinline__ void zero() { u = make_uint4(0, 0, 0, 0); }
    __device__ __forceinline__ void unpack(float (&v)[8]) const {
        const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            v[2 * k] = __uint_as_float(w[k] << 16);
            v[2 * k + 1] = __uint_as_float(w[k] & 0xffff0000u);
        }
    }
};
template <>
struct Raw8<float> {
    float4 f[2];
    __device__ __forceinline__ void load(const float* p) {
        f[0] = __ldg(reinterpret_cast<const float4*>(p));
        f[1] = __ldg(reinterpret_cast<const float4*>(p) + 1);
    }
    __device__ __forceinline__ void zero() { f[0] = f[1] = make_float4(0.f, 0.f, 0.f, 0.f); }
    __device__ __forceinline__ void unpack(float (&v)[8]) const {
        v[0] = f[0].x; v[1] = f[0].y; v[2] = f[0].z; v[3] = f[0].w;
        v[4] = f[1].x; v[5] = f[1].y; v[6] = f[1].z; v[7] = f[1].w;
    }
};

// Least and largest log2 s1 of a chunk's non-zero tokens (layout and loads
// as in the stats kernel, fp64 sum of squares). log2(sqrt(ss)/sqrt(d)) is
// increasing in ss, so the chunk keeps the least and largest ss and takes
// the log2 of those two only.
template <typename XT>
__global__ void __launch_bounds__(kStatsThreads, 4) nsn_s1minmax_kernel(EncodeArgs a) {
    const int chunk = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
    const int warp = threadIdx.x >> 5, lane = lane_id();
    const int tk = lane >> 4, cg = lane & 15;
    const int64_t t0 = (int64_t)chunk * a.chunk1;
    const int64_t t1 = min(t0 + a.chunk1, a.T);
    const XT* xb = enc_head<XT>(a, b, h) + 8 * cg;
    constexpr int64_t kStride = 2 * (kStatsThreads / 32);  // tokens per CTA step
    constexpr int kDepth = stats_depth<XT>();
    Raw8<XT> buf[kDepth];
#pragma unroll
    for (int d = 0; d < kDepth; ++d) {
        const int64_t t = t0 + warp * 2 + d * kStride + tk;
        if (t < t1) buf[d].load(xb + t * a.st); else buf[d].zero();
    }
    double mn = INFINITY, mx = -INFINITY;  // of ss > 0 (zero-filled slots give 0)
    for (int64_t base = t0 + warp * 2; base < t1; base += kDepth * kStride) {
#pragma unroll
        for (int d = 0; d < kDepth; ++d) {
            float v[8];
            buf[d].unpack(v);
            const int64_t tn = base + (d + kDepth) * kStride + tk;
            if (tn < t1) buf[d].load(xb + tn * a.st); else buf[d].zero();
            double s0 = 0.0, s1 = 0.0;
#pragma unroll
            for (int c = 0; c < 8; c += 2) {
                s0 = fma((double)v[c], (double)v[c], s0);
                s1 = fma((double)v[c + 1], (double)v[c + 1], s1);
            }
            double ss = s0 + s1;
#pragma unroll
            for (int m = 1; m < 16; m <<= 1) ss += __shfl_xor_sync(kFull, ss, m);
            if (ss > 0.0) {
                mn = fmin(mn, ss);
                mx = fmax(mx, ss);
            }
        }
    }
    mn = fmin(mn, __shfl_xor_sync(kFull, mn, 16));
    mx = fmax(mx, __shfl_xor_sync(kFull, mx, 16));
    __shared__ double red[kStatsThreads / 32][2];
    if (lane == 0) { red[warp][0] = mn; red[warp][1] = mx; }
    __syncthreads();
    if (threadIdx.x == 0) {
        for (int w = 1; w < kStatsThreads / 32; ++w) {
            mn = fmin(mn, red[w][0]);
            mx = fmax(mx, red[w][1]);
        }
        const double sqrt_d = sqrt((double)kD);
        double* out = a.minmax + ((int64_t)(b * a.H + h) * a.nchunk1 + chunk) * 2;
        out[0] = mn <= mx ? log2(sqrt(mn) / sqrt_d) : INFINITY;
        out[1] = mn <= mx ? log2(sqrt(mx) / sqrt_d) : -INFINITY;
    }
}

// o of one (b, h) from its chunk partials, by the CTA whose chunk finished
// last: o = sum / T in fp64 (double quantization: o on 16 uniform levels
// between its least and largest channel value, and the head's s1 grid).
template <bool DQ>
__device__ void shift_of_head(const EncodeArgs& a, int64_t bh, double (*red)[kD]) {
    const int c = threadIdx.x;
    const bool sec = enc_second(a, bh);
    const int64_t cbh = enc_cbh(a, bh);
    double o = 0.0;
    if (c < kD) {
        double s = 0.0;
        for (int k = 0; k < a.nchunk1; ++k) s += __ldcg(a.partial + (bh * a.nchunk1 + k) * kD + c);
        o = a.T > 0 ? s / (double)a.T : 0.0;
    }
    if constexpr (DQ) {
        double mn = o, mx = o;
#pragma unroll
        for (int m = 1; m < 32; m <<= 1) {
            mn = fmin(mn, __shfl_xor_sync(kFull, mn, m));
            mx = fmax(mx, __shfl_xor_sync(kFull, mx, m));
        }
        __syncthreads();  // red is free again
        if (c < kD && (c & 31) == 0) { red[0][c >> 5] = mn; red[1][c >> 5] = mx; }
        __syncthreads();
        mn = red[0][0]; mx = red[1][0];
#pragma unroll
        for (int w = 1; w < kD / 32; ++w) { mn = fmin(mn, red[0][w]); mx = fmax(mx, red[1][w]); }
        const double step = (mx - mn) / 15.0;
        o = mn + (step > 0.0 ? round((o - mn) / step) : 0.0) * step;
        if (c == 0) {
            double lo, st;
            dq_grid_from_chunks(a.minmax + bh * a.nchunk1 * 2, a.nchunk1, lo, st);
            float* grid = enc_s1_grid(a, sec);
            grid[2 * cbh] = (float)lo;
            grid[2 * cbh + 1] = (float)st;
        }
    }
    if (c < kD) {
        a.o64[bh * kD + c] = o;
        enc_shift(a, sec)[cbh * kD + c] = (float)o;
    }
}

template <typename XT, bool DQ>
__global__ void __launch_bounds__(kStatsThreads, 4) nsn_stats_kernel(EncodeArgs a) {
    // pass 2 is a programmatic dependent: it may be scheduled as this grid's
    // CTAs retire (it waits for the whole grid before reading the shift)
    asm volatile("griddepcontrol.launch_dependents;\n" ::: "memory");
    const int chunk = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
    const int64_t bh = (int64_t)b * a.H + h;
    const int warp = threadIdx.x >> 5, lane = lane_id();
    const int tk = lane >> 4, cg = lane & 15;
    const int64_t t0 = (int64_t)chunk * a.chunk1;
    const int64_t t1 = min(t0 + a.chunk1, a.T);
    const XT* xb = enc_head<XT>(a, b, h) + 8 * cg;
    const double sqrt_d = sqrt((double)kD);
    constexpr int64_t kStride = 2 * (kStatsThreads / 32);  // tokens per CTA step
    double glo = 0.0, gstep = 0.0;
    __shared__ double dq_lvl[16], dq_thr[15], dq_inv[16];
    if constexpr (DQ) {
        dq_grid_from_chunks(a.minmax + bh * a.nchunk1 * 2, a.nchunk1, glo, gstep);
        dq_table_build(glo, gstep, dq_lvl, dq_thr, dq_inv);
        __syncthreads();
    }
    double acc[8];
#pragma unroll
    for (int c = 0; c < 8; ++c) acc[c] = 0.0;
    constexpr int kStatsDepth2 = stats_depth<XT>();
    Raw8<XT> buf[kStatsDepth2];
#pragma unroll
    for (int d = 0; d < kStatsDepth2; ++d) {
        const int64_t t = t0 + warp * 2 + d * kStride + tk;
        if (t < t1) buf[d].load(xb + t * a.st); else buf[d].zero();
    }
    for (int64_t base = t0 + warp * 2; base < t1; base += kStatsDepth2 * kStride) {
#pragma unroll
        for (int d = 0; d < kStatsDepth2; ++d) {
            float v[8];
            buf[d].unpack(v);
            // refill this slot kStatsDepth2 steps ahead
            const int64_t tn = base + (d + kStatsDepth2) * kStride + tk;
            if (tn < t1) buf[d].load(xb + tn * a.st); else buf[d].zero();
            double s0 = 0.0, s1 = 0.0;
#pragma unroll
            for (int c = 0; c < 8; c += 2) {
                s0 = fma((double)v[c], (double)v[c], s0);
                s1 = fma((double)v[c + 1], (double)v[c + 1], s1);
            }
            double ss = s0 + s1;
#pragma unroll
            for (int m = 1; m < 16; m <<= 1) ss += __shfl_xor_sync(kFull, ss, m);
            if (ss > 0.0) {
                double inv;  // 1 / s1
                if constexpr (DQ) {
                    const double st = sqrt(ss) / sqrt_d;
                    const int k = dq_level(st, gstep, dq_thr);
                    inv = k >= 0 ? dq_inv[k] : 1.0 / dq_s1(st, glo, gstep);
                } else {
                    inv = rsqrt(ss) * sqrt_d;
                }
#pragma unroll
                for (int c = 0; c < 8; ++c) acc[c] = fma((double)v[c], inv, acc[c]);
            }
        }
    }
    // Sum the two token slots of each channel group, then the warps.
#pragma unroll
    for (int c = 0; c < 8; ++c) acc[c] += __shfl_xor_sync(kFull, acc[c], 16);
    __shared__ double red[kStatsThreads / 32][kD];
    __shared__ unsigned last;
    if (tk == 0) {
#pragma unroll
        for (int c = 0; c < 8; ++c) red[warp][8 * cg + c] = acc[c];
    }
    __syncthreads();
    if (threadIdx.x < kD) {
        double s = 0.0;
#pragma unroll
        for (int w = 0; w < kStatsThreads / 32; ++w) s += red[w][threadIdx.x];
        a.partial[(bh * a.nchunk1 + chunk) * kD + threadIdx.x] = s;
    }
    // The chunk that completes its (b, h) last also derives the shift.
    __threadfence();
    __syncthreads();
    if (threadIdx.x == 0) last = atomicAdd(a.head_done + bh, 1u) == (unsigned)(a.nchunk1 - 1);
    __syncthreads();
    if (last) {
        __threadfence();
        shift_of_head<DQ>(a, bh, red);
    }
}

// ---------------------------------------------------------------- host --
// Pass 1 splits each head's tokens into nchunk1 chunks so that the grid
// (B * H * nchunk1 CTAs, four per SM) fills one wave of a 148-SM B200 as
// evenly as the head count allows; a chunk is at least 64 tokens.
constexpr int64_t kPass1Slots = 148 * 4;

EncodePlan plan_encode(int B, int H, int64_t T) {
    EncodePlan p{};
    const int64_t heads = (int64_t)B * H > 0 ? (int64_t)B * H : 1;
    int64_t n = kPass1Slots / heads;
    const int64_t by_len = (T + 63) / 64;
    if (n > by_len) n = by_len;
    if (n < 1) n = 1;
    p.nchunk1 = (int)n;
    p.chunk1 = (T + n - 1) / n;
    if (p.chunk1 < 1) p.chunk1 = 1;
    p.reset_bytes = kEncodeStatsBytes + (size_t)B * H * sizeof(unsigned);  // stats + per-head counters
    p.partial_off = align_up(p.reset_bytes, kWsAlign);
    const size_t partial_bytes = (size_t)B * H * p.nchunk1 * kD * sizeof(double);
    p.o64_off = align_up(p.partial_off + partial_bytes, kWsAlign);
    p.minmax_off = align_up(p.o64_off + (size_t)B * H * kD * sizeof(double), kWsAlign);
    p.total = align_up(p.minmax_off + (size_t)B * H * p.nchunk1 * 2 * sizeof(double), kWsAlign);
    return p;
}

template <typename XT>
static cudaError_t launch_encode_t(const EncodeArgs& a, cudaStream_t s) {
    if (!a.given_shift) {
        const dim3 grid1(a.nchunk1, a.H, a.B);
        if (a.dq) {
            nsn_s1minmax_kernel<XT><<<grid1, kStatsThreads, 0, s>>>(a);
            nsn_stats_kernel<XT, true><<<grid1, kStatsThreads, 0, s>>>(a);
        } else {
            nsn_stats_kernel<XT, false><<<grid1, kStatsThreads, 0, s>>>(a);
        }
    }
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    if ((int64_t)a.B * a.H * a.T <= kSmallEncode) return launch_encode_small(a, s);
    return (a.sub == 4 && !a.tc_search) ? launch_encode_pruned(a, s) : launch_encode_tc(a, s);
}

cudaError_t launch_encode(const EncodeArgs& a, cudaStream_t s) {
    return a.x_bf16 ? launch_encode_t<__nv_bfloat16>(a, s) : launch_encode_t<float>(a, s);
}

}  // namespace nsnq
