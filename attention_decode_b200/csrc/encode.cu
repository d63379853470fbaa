// NSNQuant encode on sm_100a: Normalize-Shift-Normalize, Hadamard transform
// and nearest-codeword vector quantization (gist.science "NSNQuant ...",
// Technical Summary, Methodology §1-§3).
//
// Three launches per call in shift-compute mode, one in shift-given mode:
//   nsn_stats_kernel   per (b, h, chunk): channel sums of y = x / s1 in fp64
//   nsn_shift_kernel   per (b, h): o = sum / T (fp64, kept in the workspace
//                      for the near-tie path) and its fp32 copy in the cache
//   nsn_encode_kernel  per (b, h, chunk): fp32 NSN + FWHT + nearest codeword,
//                      with an exact fp64 re-decision of near-tied sub-vectors
#include <math.h>

#include "common.cuh"
#include "internal.h"

namespace nsnq {

// A sub-vector whose best two fp32 distances are closer than this is
// re-decided from an fp64 recomputation of the whole token. fp32 errors in
// the transformed token are ~1e-7 relative, so 1e-4 leaves a wide margin.
constexpr float kTieRel = 1e-4f;
constexpr float kTieAbs = 1e-6f;
// Tokens whose shift residual has s2 below this are re-encoded in fp64: the
// fp32 difference y - o loses too many digits to be trusted.
constexpr float kCancel = 1e-3f;

constexpr int kStatsThreads = 256;
constexpr int kEncodeThreads = 128;
constexpr int64_t kEncodeChunk = 64;  // tokens per pass-2 CTA

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

template <typename XT>
__global__ void __launch_bounds__(kStatsThreads) nsn_stats_kernel(EncodeArgs a) {
    const int chunk = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
    const int warp = threadIdx.x >> 5, lane = lane_id();
    const int tk = lane >> 3, cg = lane & 7;
    const int64_t t0 = (int64_t)chunk * a.chunk1;
    const int64_t t1 = min(t0 + a.chunk1, a.T);
    const XT* xb = reinterpret_cast<const XT*>(a.x) + b * a.sb + h * a.sh + 16 * cg;
    const double sqrt_d = sqrt((double)kD);
    constexpr int64_t kStride = 4 * (kStatsThreads / 32);  // tokens per CTA step
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
                const double inv = rsqrt(ss) * sqrt_d;  // 1 / s1
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

__global__ void __launch_bounds__(kD) nsn_shift_kernel(EncodeArgs a) {
    const int bh = blockIdx.x;
    const int c = threadIdx.x;
    double s = 0.0;
    for (int k = 0; k < a.nchunk1; ++k) s += a.partial[((int64_t)bh * a.nchunk1 + k) * kD + c];
    const double o = a.T > 0 ? s / (double)a.T : 0.0;
    a.o64[(int64_t)bh * kD + c] = o;
    a.shift[(int64_t)bh * kD + c] = (float)o;
}

// --------------------------------------------------------------- pass 2 --
struct Best {
    float d1, d2;
    int i1;
};

// Lane holds 4 coordinates of the transformed token (coordinates 4l..4l+3).
// SUB = 4: the lane's coordinates are sub-vector l; it scans all centroids.
// SUB = 8: lanes 2j, 2j+1 hold sub-vector j; each scans half the centroids.
template <int SUB>
__device__ __forceinline__ Best search_fp32(const float (&w)[4], const float* Cs) {
    Best r{INFINITY, INFINITY, 0};
    const int lane = lane_id();
    if constexpr (SUB == 4) {
        const float4* C4 = reinterpret_cast<const float4*>(Cs);
#pragma unroll 4
        for (int c = 0; c < kNC; ++c) {
            const float4 cv = C4[c];
            const float e0 = w[0] - cv.x, e1 = w[1] - cv.y, e2 = w[2] - cv.z, e3 = w[3] - cv.w;
            const float d = fmaf(e3, e3, fmaf(e2, e2, fmaf(e1, e1, e0 * e0)));
            if (d < r.d1) {
                r.d2 = r.d1; r.d1 = d; r.i1 = c;
            } else {
                r.d2 = fminf(r.d2, d);
            }
        }
    } else {
        float f[8];
        const bool odd = lane & 1;
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            const float p = __shfl_xor_sync(kFull, w[k], 1);
            f[k] = odd ? p : w[k];
            f[4 + k] = odd ? w[k] : p;
        }
        const float4* C4 = reinterpret_cast<const float4*>(Cs);
        const int cbeg = odd ? kNC / 2 : 0;
#pragma unroll 2
        for (int c = cbeg; c < cbeg + kNC / 2; ++c) {
            const float4 a = C4[2 * c], bq = C4[2 * c + 1];
            float d = 0.f;
            float e;
            e = f[0] - a.x; d = fmaf(e, e, d);
            e = f[1] - a.y; d = fmaf(e, e, d);
            e = f[2] - a.z; d = fmaf(e, e, d);
            e = f[3] - a.w; d = fmaf(e, e, d);
            e = f[4] - bq.x; d = fmaf(e, e, d);
            e = f[5] - bq.y; d = fmaf(e, e, d);
            e = f[6] - bq.z; d = fmaf(e, e, d);
            e = f[7] - bq.w; d = fmaf(e, e, d);
            if (d < r.d1) {
                r.d2 = r.d1; r.d1 = d; r.i1 = c;
            } else {
                r.d2 = fminf(r.d2, d);
            }
        }
        const float od1 = __shfl_xor_sync(kFull, r.d1, 1);
        const float od2 = __shfl_xor_sync(kFull, r.d2, 1);
        const int oi1 = __shfl_xor_sync(kFull, r.i1, 1);
        if (od1 < r.d1 || (od1 == r.d1 && oi1 < r.i1)) {
            r.d2 = fminf(r.d1, od2); r.d1 = od1; r.i1 = oi1;
        } else {
            r.d2 = fminf(r.d2, od1);
        }
    }
    return r;
}

// Exact fp64 nearest codeword (full squared distance, lowest index on ties).
template <int SUB>
__device__ __forceinline__ int search_fp64(const double (&w)[4], const float* Cs, bool active) {
    const int lane = lane_id();
    double f[SUB];
    if constexpr (SUB == 4) {
#pragma unroll
        for (int k = 0; k < 4; ++k) f[k] = w[k];
    } else {
        const bool odd = lane & 1;
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            const double p = __shfl_xor_sync(kFull, w[k], 1);
            f[k] = odd ? p : w[k];
            f[4 + k] = odd ? w[k] : p;
        }
    }
    double bd = INFINITY;
    int bi = 0;
    if (active) {
        const int cbeg = (SUB == 8 && (lane & 1)) ? kNC / 2 : 0;
        const int cend = SUB == 8 ? cbeg + kNC / 2 : kNC;
        for (int c = cbeg; c < cend; ++c) {
            double d = 0.0;
#pragma unroll
            for (int k = 0; k < SUB; ++k) {
                const double e = f[k] - (double)Cs[c * SUB + k];
                d += e * e;
            }
            if (d < bd) { bd = d; bi = c; }
        }
    }
    if constexpr (SUB == 8) {
        const double od = __shfl_xor_sync(kFull, bd, 1);
        const int oi = __shfl_xor_sync(kFull, bi, 1);
        if (od < bd || (od == bd && oi < bi)) bi = oi;
    }
    return bi;
}

template <typename XT, int SUB>
__global__ void __launch_bounds__(kEncodeThreads) nsn_encode_kernel(EncodeArgs a) {
    __shared__ __align__(16) float Cs[kNC * SUB];
    __shared__ double o64s[kD];
    const int chunk = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
    const int64_t bh = (int64_t)b * a.H + h;
    for (int i = threadIdx.x; i < kNC * SUB; i += blockDim.x) Cs[i] = a.C[i];
    if (threadIdx.x < kD)
        o64s[threadIdx.x] =
            a.given_shift ? (double)a.shift[bh * kD + threadIdx.x] : a.o64[bh * kD + threadIdx.x];
    __syncthreads();

    constexpr int J = kD / SUB;
    const int lane = lane_id(), warp = threadIdx.x >> 5;
    float o32[4];
#pragma unroll
    for (int r = 0; r < 4; ++r) o32[r] = (float)o64s[4 * lane + r];
    const int64_t t0 = (int64_t)chunk * kEncodeChunk;
    const int64_t t1 = min(t0 + kEncodeChunk, a.T);
    const XT* xb = reinterpret_cast<const XT*>(a.x) + b * a.sb + h * a.sh + 4 * lane;
    const double sqrt_d = sqrt((double)kD);
    const double rsqrt_d = 1.0 / sqrt_d;

    for (int64_t t = t0 + warp; t < t1; t += kEncodeThreads / 32) {
        float x[4];
        load4(xb + t * a.st, x);
        // Normalize: s1 = ||x|| / sqrt(D) (1/D is exact for D = 128).
        const float ss = warp_sum(fmaf(x[3], x[3], fmaf(x[2], x[2], fmaf(x[1], x[1], x[0] * x[0]))));
        float s1 = sqrtf(ss * (1.0f / kD));
        const float inv1 = s1 > 0.f ? 1.0f / s1 : 0.f;
        // Shift, then normalize again: s2 = ||z|| / sqrt(D).
        float z[4];
#pragma unroll
        for (int r = 0; r < 4; ++r) z[r] = fmaf(x[r], inv1, -o32[r]);
        const float ss2 = warp_sum(fmaf(z[3], z[3], fmaf(z[2], z[2], fmaf(z[1], z[1], z[0] * z[0]))));
        float s2 = sqrtf(ss2 * (1.0f / kD));
        const float sc = s2 > 0.f ? kRsqrtD / s2 : 0.f;
        // A small residual (heavy cancellation in y - o) is decided in fp64.
        const bool cancel = s2 < kCancel;
        float w[4];
#pragma unroll
        for (int r = 0; r < 4; ++r) w[r] = z[r] * sc;
        fwht128_lane4(w);  // w = H u, H orthonormal (scale folded into sc)

        const Best best = search_fp32<SUB>(w, Cs);
        int code = best.i1;
        double wsub[4] = {w[0], w[1], w[2], w[3]};  // the transformed coordinates (fp64 if re-decided)
        const bool tie = cancel || (best.d2 - best.d1) <= kTieRel * best.d1 + kTieAbs;
        const unsigned tie_mask = __ballot_sync(kFull, tie);
        if (tie_mask) {
            // Recompute the token in fp64 and re-decide the near-tied sub-vectors.
            double xd[4], zd[4];
#pragma unroll
            for (int r = 0; r < 4; ++r) xd[r] = (double)x[r];
            double ssd = 0.0;
#pragma unroll
            for (int r = 0; r < 4; ++r) ssd = fma(xd[r], xd[r], ssd);
            ssd = warp_sum_d(ssd);
            const double s1d = sqrt(ssd) / sqrt_d;
#pragma unroll
            for (int r = 0; r < 4; ++r)
                zd[r] = (s1d > 0.0 ? xd[r] / s1d : 0.0) - o64s[4 * lane + r];
            double ss2d = 0.0, yy = 0.0, oo = 0.0;
#pragma unroll
            for (int r = 0; r < 4; ++r) {
                const double o = o64s[4 * lane + r];
                ss2d = fma(zd[r], zd[r], ss2d);
                yy = fma(zd[r] + o, zd[r] + o, yy);
                oo = fma(o, o, oo);
            }
            ss2d = warp_sum_d(ss2d);
            yy = warp_sum_d(yy);
            oo = warp_sum_d(oo);
            // residual at or below 2^-20 of the token/shift magnitude counts as zero
            const double s2d = ss2d <= 0x1p-40 * (yy + oo) ? 0.0 : sqrt(ss2d) / sqrt_d;
#pragma unroll
            for (int r = 0; r < 4; ++r) zd[r] = s2d > 0.0 ? zd[r] / s2d : 0.0;
            fwht128_lane4(zd);
#pragma unroll
            for (int r = 0; r < 4; ++r) zd[r] *= rsqrt_d;
            const int c64 = search_fp64<SUB>(zd, Cs, tie);
            if (tie) code = c64;
            s1 = (float)s1d;
            s2 = (float)s2d;
#pragma unroll
            for (int r = 0; r < 4; ++r) wsub[r] = zd[r];
            if (lane == 0 && a.stats) {
                atomicAdd(&a.stats[0], 1ull);
                atomicAdd(&a.stats[1], (unsigned long long)(__popc(tie_mask) / (SUB / 4)));
            }
        }
        if (a.adaptive) {
            // Scale adjustment: s2 *= ||w||^2 / (w . w_hat); lane holds coordinates
            // 4l..4l+3, i.e. the (lane & 1) half of sub-vector lane / 2 when SUB = 8.
            const float* cw = Cs + code * SUB + (SUB == 8 ? 4 * (lane & 1) : 0);
            double ww = 0.0, wq = 0.0;
#pragma unroll
            for (int r = 0; r < 4; ++r) {
                ww += wsub[r] * wsub[r];
                wq += wsub[r] * (double)cw[r];
            }
            ww = warp_sum_d(ww);
            wq = warp_sum_d(wq);
            s2 = (float)((double)s2 * (wq > 0.0 ? ww / wq : 1.0));
        }
        const int64_t row = bh * a.cap + a.t_offset + t;
        if constexpr (SUB == 4) {
            a.codes[row * J + lane] = (uint8_t)code;
        } else {
            if ((lane & 1) == 0) a.codes[row * J + (lane >> 1)] = (uint8_t)code;
        }
        if (lane == 0) reinterpret_cast<float2*>(a.scales)[row] = make_float2(s1, s2);
    }
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
    p.total = align_up(p.o64_off + (size_t)B * H * kD * sizeof(double), kWsAlign);
    return p;
}

template <typename XT>
static cudaError_t launch_encode_t(const EncodeArgs& a, cudaStream_t s) {
    if (!a.given_shift) {
        nsn_stats_kernel<XT><<<dim3(a.nchunk1, a.H, a.B), kStatsThreads, 0, s>>>(a);
        nsn_shift_kernel<<<a.B * a.H, kD, 0, s>>>(a);
    }
    if (a.sub == 4) {
        cudaError_t e = cudaGetLastError();
        if (e != cudaSuccess) return e;
        return launch_encode_pruned(a, s);
    }
    const dim3 grid((unsigned)((a.T + kEncodeChunk - 1) / kEncodeChunk), a.H, a.B);
    nsn_encode_kernel<XT, 8><<<grid, kEncodeThreads, 0, s>>>(a);
    return cudaGetLastError();
}

cudaError_t launch_encode(const EncodeArgs& a, cudaStream_t s) {
    return a.x_bf16 ? launch_encode_t<__nv_bfloat16>(a, s) : launch_encode_t<float>(a, s);
}

}  // namespace nsnq
