// NSNQuant encode on sm_100a: Normalize-Shift-Normalize, Hadamard transform
// and nearest-codeword vector quantization (gist.science "NSNQuant ...",
// Technical Summary, Methodology §1-§3).
//
// Three launches per call in shift-compute mode, one in shift-given mode:
//   nsn_s1minmax_kernel per (b, h, chunk), double quantization only: least and
//                      largest log2 s1 (the per-head s1 grid)
//   nsn_stats_kernel   per (b, h, chunk): channel sums of y = x / s1 in fp64
//   nsn_shift_kernel   per (b, h): o = sum / T (fp64, kept in the workspace
//                      for the near-tie path) and its fp32 copy in the cache
//   pass 2             NSN + FWHT + nearest codeword: encode_pruned.cu
//                      (2 bit, search index) or encode1_tc.cu (1 bit, all
//                      codewords scored on the tensor cores)
#include <math.h>

#include "common.cuh"
#include "dq.cuh"
#include "internal.h"

namespace nsnq {

constexpr int kStatsThreads = 256;

// --------------------------------------------------------------- pass 1 --
// Lane layout: 8 lanes per token (16 channels each), 4 tokens per warp step.
// Each warp keeps kStatsDepth steps of loads in flight (the kernel streams
// x once from HBM and needs the bytes in flight to cover the latency).
constexpr int kStatsDepth = 4;

template <typename XT>
struct Raw16;
template <>
struct Raw16<__nv_bfloat16> {
    uint4 u[2];
    __device__ __forceinline__ void load(const __nv_bfloat16* p) {
        const uint4* q = reinterpret_cast<const uint4*>(p);
        u[0] = __ldg(q);
        u[1] = __ldg(q + 1);
    }
    __device__ __forceinline__ void zero() { u[0] = u[1] = make_uint4(0, 0, 0, 0); }
    __device__ __forceinline__ void unpack(float (&v)[16]) const {
#pragma unroll
        for (int i = 0; i < 2; ++i) {
            const uint32_t w[4] = {u[i].x, u[i].y, u[i].z, u[i].w};
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                v[8 * i + 2 * k] = __uint_as_float(w[k] << 16);
                v[8 * i + 2 * k + 1] = __uint_as_float(w[k] & 0xffff0000u);
            }
        }
    }
};
template <>
struct Raw16<float> {
    float4 f[4];
    __device__ __forceinline__ void load(const float* p) {
        const float4* q = reinterpret_cast<const float4*>(p);
#pragma unroll
        for (int i = 0; i < 4; ++i) f[i] = __ldg(q + i);
    }
    __device__ __forceinline__ void zero() {
#pragma unroll
        for (int i = 0; i < 4; ++i) f[i] = make_float4(0.f, 0.f, 0.f, 0.f);
    }
    __device__ __forceinline__ void unpack(float (&v)[16]) const {
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            v[4 * i] = f[i].x; v[4 * i + 1] = f[i].y; v[4 * i + 2] = f[i].z; v[4 * i + 3] = f[i].w;
        }
    }
};

// Least and largest log2 s1 of a chunk's non-zero tokens (8 lanes per token,
// fp64 sum of squares as in the stats kernel).
template <typename XT>
__global__ void __launch_bounds__(kStatsThreads) nsn_s1minmax_kernel(EncodeArgs a) {
    const int chunk = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
    const int warp = threadIdx.x >> 5, lane = lane_id();
    const int tk = lane >> 3, cg = lane & 7;
    const int64_t t0 = (int64_t)chunk * a.chunk1;
    const int64_t t1 = min(t0 + a.chunk1, a.T);
    const XT* xb = reinterpret_cast<const XT*>(a.x) + b * a.sb + h * a.sh + 16 * cg;
    const double sqrt_d = sqrt((double)kD);
    constexpr int64_t kStride = 4 * (kStatsThreads / 32);
    double mn = INFINITY, mx = -INFINITY;
    for (int64_t t = t0 + warp * 4 + tk; t - tk < t1; t += kStride) {
        Raw16<XT> r;
        if (t < t1) r.load(xb + t * a.st); else r.zero();
        float v[16];
        r.unpack(v);
        double ss = 0.0;
#pragma unroll
        for (int c = 0; c < 16; ++c) ss = fma((double)v[c], (double)v[c], ss);
        ss += __shfl_xor_sync(kFull, ss, 1);
        ss += __shfl_xor_sync(kFull, ss, 2);
        ss += __shfl_xor_sync(kFull, ss, 4);
        if (t < t1 && ss > 0.0) {
            const double l = log2(sqrt(ss) / sqrt_d);
            mn = fmin(mn, l);
            mx = fmax(mx, l);
        }
    }
#pragma unroll
    for (int m = 8; m < 32; m <<= 1) {
        mn = fmin(mn, __shfl_xor_sync(kFull, mn, m));
        mx = fmax(mx, __shfl_xor_sync(kFull, mx, m));
    }
    __shared__ double red[kStatsThreads / 32][2];
    if (lane == 0) { red[warp][0] = mn; red[warp][1] = mx; }
    __syncthreads();
    if (threadIdx.x == 0) {
        for (int w = 1; w < kStatsThreads / 32; ++w) {
            mn = fmin(mn, red[w][0]);
            mx = fmax(mx, red[w][1]);
        }
        double* out = a.minmax + ((int64_t)(b * a.H + h) * a.nchunk1 + chunk) * 2;
        out[0] = mn;
        out[1] = mx;
    }
}

template <typename XT, bool DQ>
__global__ void __launch_bounds__(kStatsThreads) nsn_stats_kernel(EncodeArgs a) {
    const int chunk = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
    const int warp = threadIdx.x >> 5, lane = lane_id();
    const int tk = lane >> 3, cg = lane & 7;
    const int64_t t0 = (int64_t)chunk * a.chunk1;
    const int64_t t1 = min(t0 + a.chunk1, a.T);
    const XT* xb = reinterpret_cast<const XT*>(a.x) + b * a.sb + h * a.sh + 16 * cg;
    const double sqrt_d = sqrt((double)kD);
    constexpr int64_t kStride = 4 * (kStatsThreads / 32);  // tokens per CTA step
    double glo = 0.0, gstep = 0.0;
    if constexpr (DQ)
        dq_grid_from_chunks(a.minmax + (int64_t)(b * a.H + h) * a.nchunk1 * 2, a.nchunk1, glo, gstep);
    double acc[16];
#pragma unroll
    for (int c = 0; c < 16; ++c) acc[c] = 0.0;
    Raw16<XT> buf[kStatsDepth];
#pragma unroll
    for (int d = 0; d < kStatsDepth; ++d) {
        const int64_t t = t0 + warp * 4 + d * kStride + tk;
        if (t < t1) buf[d].load(xb + t * a.st); else buf[d].zero();
    }
    for (int64_t base = t0 + warp * 4; base < t1; base += kStatsDepth * kStride) {
#pragma unroll
        for (int d = 0; d < kStatsDepth; ++d) {
            float v[16];
            buf[d].unpack(v);
            // refill this slot kStatsDepth steps ahead
            const int64_t tn = base + (d + kStatsDepth) * kStride + tk;
            if (tn < t1) buf[d].load(xb + tn * a.st); else buf[d].zero();
            double ss = 0.0;
#pragma unroll
            for (int c = 0; c < 16; ++c) ss = fma((double)v[c], (double)v[c], ss);
            ss += __shfl_xor_sync(kFull, ss, 1);
            ss += __shfl_xor_sync(kFull, ss, 2);
            ss += __shfl_xor_sync(kFull, ss, 4);
            if (ss > 0.0) {
                double inv;  // 1 / s1
                if constexpr (DQ) {
                    inv = 1.0 / dq_s1(sqrt(ss) / sqrt_d, glo, gstep);
                } else {
                    inv = rsqrt(ss) * sqrt_d;
                }
#pragma unroll
                for (int c = 0; c < 16; ++c) acc[c] = fma((double)v[c], inv, acc[c]);
            }
        }
    }
    // Sum the four token slots of each channel group, then the warps.
#pragma unroll
    for (int c = 0; c < 16; ++c) {
        acc[c] += __shfl_xor_sync(kFull, acc[c], 8);
        acc[c] += __shfl_xor_sync(kFull, acc[c], 16);
    }
    __shared__ double red[kStatsThreads / 32][kD];
    if (tk == 0) {
#pragma unroll
        for (int c = 0; c < 16; ++c) red[warp][16 * cg + c] = acc[c];
    }
    __syncthreads();
    if (threadIdx.x < kD) {
        double s = 0.0;
#pragma unroll
        for (int w = 0; w < kStatsThreads / 32; ++w) s += red[w][threadIdx.x];
        a.partial[((int64_t)(b * a.H + h) * a.nchunk1 + chunk) * kD + threadIdx.x] = s;
    }
}

template <bool DQ>
__global__ void __launch_bounds__(kD) nsn_shift_kernel(EncodeArgs a) {
    const int bh = blockIdx.x;
    const int c = threadIdx.x;
    double s = 0.0;
    for (int k = 0; k < a.nchunk1; ++k) s += a.partial[((int64_t)bh * a.nchunk1 + k) * kD + c];
    double o = a.T > 0 ? s / (double)a.T : 0.0;
    if constexpr (DQ) {
        // o on 16 uniform levels between its least and largest channel value
        __shared__ double red[kD / 32][2];
        double mn = o, mx = o;
#pragma unroll
        for (int m = 1; m < 32; m <<= 1) {
            mn = fmin(mn, __shfl_xor_sync(kFull, mn, m));
            mx = fmax(mx, __shfl_xor_sync(kFull, mx, m));
        }
        if ((c & 31) == 0) { red[c >> 5][0] = mn; red[c >> 5][1] = mx; }
        __syncthreads();
        mn = red[0][0]; mx = red[0][1];
#pragma unroll
        for (int w = 1; w < kD / 32; ++w) { mn = fmin(mn, red[w][0]); mx = fmax(mx, red[w][1]); }
        const double step = (mx - mn) / 15.0;
        o = mn + (step > 0.0 ? round((o - mn) / step) : 0.0) * step;
        if (c == 0) {
            double lo, st;
            dq_grid_from_chunks(a.minmax + (int64_t)bh * a.nchunk1 * 2, a.nchunk1, lo, st);
            a.s1_grid[2 * bh] = (float)lo;
            a.s1_grid[2 * bh + 1] = (float)st;
        }
    }
    a.o64[(int64_t)bh * kD + c] = o;
    a.shift[(int64_t)bh * kD + c] = (float)o;
}

// ---------------------------------------------------------------- host --
EncodePlan plan_encode(int B, int H, int64_t T) {
    EncodePlan p{};
    p.chunk1 = 512;
    p.nchunk1 = (int)((T + p.chunk1 - 1) / p.chunk1);
    if (p.nchunk1 < 1) p.nchunk1 = 1;
    p.partial_off = align_up(kEncodeStatsBytes, kWsAlign);
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
            nsn_shift_kernel<true><<<a.B * a.H, kD, 0, s>>>(a);
        } else {
            nsn_stats_kernel<XT, false><<<grid1, kStatsThreads, 0, s>>>(a);
            nsn_shift_kernel<false><<<a.B * a.H, kD, 0, s>>>(a);
        }
    }
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    return a.sub == 4 ? launch_encode_pruned(a, s) : launch_encode1_tc(a, s);
}

cudaError_t launch_encode(const EncodeArgs& a, cudaStream_t s) {
    return a.x_bf16 ? launch_encode_t<__nv_bfloat16>(a, s) : launch_encode_t<float>(a, s);
}

}  // namespace nsnq
