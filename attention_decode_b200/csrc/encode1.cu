// Pass 2 of the 1-bit encode (8-dimensional sub-vectors, 256 codewords): NSN,
// Hadamard transform and the exact nearest codeword of every sub-vector
// (gist.science "NSNQuant ...", Technical Summary, Methodology §1-§3).
//
// In 8 dimensions a cell index is out of reach (10^8 cells), so every
// codeword is scored, as cheaply as possible: a warp holds two token-heads,
// sixteen lanes each, and a lane one sub-vector (8 coordinates). For a pair
// of codewords (c, c') the lane evaluates s = ||c||^2 - 2 w.c for both at
// once with packed f32x2 FMAs against a table of (-2c, -2c') coordinate pairs
// that every lane reads at the same address (a shared-memory broadcast), and
// keeps the best and second-best s. Since d = ||w||^2 + s, the nearest
// codeword has the least s. Sub-vectors whose two best distances are within
// kTieRel1 * d1 + kTieAbs1 are re-decided in fp64 by the whole warp.
#include <math.h>

#include "common.cuh"
#include "internal.h"

namespace nsnq {

namespace {

constexpr int kThreads1 = 256;
constexpr float kTieRel1 = 1e-4f;  // fp32 error of s is ~1e-6 relative to d: wide margin
constexpr float kTieAbs1 = 1e-6f;
constexpr float kCancel1 = 1e-3f;  // s2 below this: residual decided in fp64

__device__ __forceinline__ uint64_t pk2(float a, float b) {
    uint64_t r;
    asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(a), "f"(b));
    return r;
}
__device__ __forceinline__ float2 upk2(uint64_t u) {
    float2 r;
    asm("mov.b64 {%0, %1}, %2;" : "=f"(r.x), "=f"(r.y) : "l"(u));
    return r;
}
__device__ __forceinline__ uint64_t ffma2(uint64_t a, uint64_t b, uint64_t c) {
    uint64_t d;
    asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
    return d;
}

template <typename XT>
__device__ __forceinline__ void load8(const XT* p, float (&v)[8]);
template <>
__device__ __forceinline__ void load8<__nv_bfloat16>(const __nv_bfloat16* p, float (&v)[8]) {
    const uint4 a = *reinterpret_cast<const uint4*>(p);
    const uint32_t u[4] = {a.x, a.y, a.z, a.w};
#pragma unroll
    for (int k = 0; k < 4; ++k) {
        v[2 * k] = __uint_as_float(u[k] << 16);
        v[2 * k + 1] = __uint_as_float(u[k] & 0xffff0000u);
    }
}
template <>
__device__ __forceinline__ void load8<float>(const float* p, float (&v)[8]) {
    const float4 a = reinterpret_cast<const float4*>(p)[0], b = reinterpret_cast<const float4*>(p)[1];
    v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
    v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
}

// Sum over the 16 lanes of one token-head.
__device__ __forceinline__ float half_sum(float v) {
#pragma unroll
    for (int m = 1; m < 16; m <<= 1) v += __shfl_xor_sync(kFull, v, m);
    return v;
}

// Exact decision for one token-head by the whole warp: fp64 NSN and fp64
// Hadamard transform (lane l holds coordinates 4l..4l+3), then for each
// flagged sub-vector j (8 coordinates, on lanes 2j and 2j+1) an fp64 scan of
// the 256 codewords split over the lanes and a warp argmin (lowest index on
// exact ties). Returns, on every lane, the new codes packed as code of
// sub-vector j in byte j of the 16-byte result (unflagged: old code), the
// fp64 (s1, s2) and the sums over all sub-vectors of w . C[code] (for the
// scale adjustment).
template <typename XT>
__device__ __noinline__ void exact_warp1(const XT* xtok, const double* o64, const float* o32,
                                         const float* C, uint32_t flags, uint4& codes,
                                         double& s1_out, double& s2_out, double& wq_out) {
    const int lane = lane_id();
    float xf[4];
    load4(xtok + 4 * lane, xf);
    double x[4], o[4];
#pragma unroll
    for (int r = 0; r < 4; ++r) {
        x[r] = (double)xf[r];
        o[r] = o64 ? o64[4 * lane + r] : (double)o32[4 * lane + r];
    }
    const double sqrt_d = sqrt((double)kD);
    const double ss = warp_sum_d(x[0] * x[0] + x[1] * x[1] + x[2] * x[2] + x[3] * x[3]);
    const double s1 = sqrt(ss) / sqrt_d;
    const double inv1 = s1 > 0.0 ? 1.0 / s1 : 0.0;
    double z[4], ss2 = 0.0, yy = 0.0, oo = 0.0;
#pragma unroll
    for (int r = 0; r < 4; ++r) {
        const double y = x[r] * inv1;
        z[r] = y - o[r];
        ss2 = fma(z[r], z[r], ss2);
        yy = fma(y, y, yy);
        oo = fma(o[r], o[r], oo);
    }
    ss2 = warp_sum_d(ss2);
    yy = warp_sum_d(yy);
    oo = warp_sum_d(oo);
    // a residual at or below 2^-20 of the token/shift magnitude counts as zero
    const double s2 = ss2 <= 0x1p-40 * (yy + oo) ? 0.0 : sqrt(ss2) / sqrt_d;
    const double inv2 = s2 > 0.0 ? 1.0 / s2 : 0.0;
#pragma unroll
    for (int r = 0; r < 4; ++r) z[r] *= inv2;
    fwht128_lane4(z);  // unnormalised: w = z / sqrt(d)
    const double hs = 1.0 / sqrt_d;
#pragma unroll
    for (int r = 0; r < 4; ++r) z[r] *= hs;
    uint32_t cw[4] = {codes.x, codes.y, codes.z, codes.w};
    uint32_t todo = flags;
    while (todo) {  // warp-uniform
        const int j = __ffs(todo) - 1;
        todo &= todo - 1;
        double f[8];
#pragma unroll
        for (int r = 0; r < 8; ++r) f[r] = __shfl_sync(kFull, z[r & 3], 2 * j + (r >> 2));
        double bd = INFINITY;
        int bi = 0;
#pragma unroll 2
        for (int k = 0; k < kNC / 32; ++k) {
            const int c = lane + 32 * k;
            double d = 0.0;
#pragma unroll
            for (int r = 0; r < 8; ++r) {
                const double e = f[r] - (double)C[c * 8 + r];
                d = fma(e, e, d);
            }
            if (d < bd) { bd = d; bi = c; }  // c rises with k: ties keep the lower index
        }
#pragma unroll
        for (int m = 1; m < 32; m <<= 1) {
            const double od = __shfl_xor_sync(kFull, bd, m);
            const int oi = __shfl_xor_sync(kFull, bi, m);
            if (od < bd || (od == bd && oi < bi)) { bd = od; bi = oi; }
        }
        const int sh = 8 * (j & 3);
        cw[j >> 2] = (cw[j >> 2] & ~(0xffu << sh)) | ((uint32_t)bi << sh);
    }
    // w . C[code] over the warp: lane l holds half of sub-vector l / 2
    const int j = lane >> 1;
    const int code = (int)((cw[j >> 2] >> (8 * (j & 3))) & 0xffu);
    double q = 0.0;
#pragma unroll
    for (int r = 0; r < 4; ++r) q = fma(z[r], (double)C[code * 8 + 4 * (lane & 1) + r], q);
    wq_out = warp_sum_d(q);
    codes = make_uint4(cw[0], cw[1], cw[2], cw[3]);
    s1_out = s1;
    s2_out = s2;
}

template <typename XT, bool ADAPT>
__global__ void __launch_bounds__(kThreads1) nsn_encode1_kernel(EncodeArgs a) {
    // tbl[q][k] = (-2 C[2q][k], -2 C[2q+1][k]); n2p[q] = (|C[2q]|^2, |C[2q+1]|^2)
    __shared__ __align__(16) float2 tbl[kNC / 2][8];
    __shared__ __align__(16) float2 n2p[kNC / 2];
    __shared__ float Cs[kNC * 8];
    for (int i = threadIdx.x; i < kNC * 8; i += kThreads1) {
        const float c = a.C[i];
        Cs[i] = c;
        const int code = i >> 3, k = i & 7;
        reinterpret_cast<float*>(&tbl[code >> 1][k])[code & 1] = -2.0f * c;
    }
    __syncthreads();
    for (int code = threadIdx.x; code < kNC; code += kThreads1) {
        float n = 0.f;
#pragma unroll
        for (int k = 0; k < 8; ++k) n = fmaf(Cs[code * 8 + k], Cs[code * 8 + k], n);
        reinterpret_cast<float*>(&n2p[code >> 1])[code & 1] = n;
    }
    __syncthreads();

    const int lane = lane_id(), l16 = lane & 15, half = lane >> 4;
    const int64_t pairs_per_head = (a.T + 1) / 2;
    const int64_t npairs = (int64_t)a.B * a.H * pairs_per_head;
    const int64_t warps = (int64_t)gridDim.x * (kThreads1 / 32);
    for (int64_t pi = (int64_t)blockIdx.x * (kThreads1 / 32) + (threadIdx.x >> 5); pi < npairs;
         pi += warps) {
        const int64_t bh = pi / pairs_per_head;
        const int64_t t0 = 2 * (pi - bh * pairs_per_head);  // first token of the warp
        const int64_t t = t0 + half;
        const int b = (int)(bh / a.H), h = (int)(bh - (int64_t)b * a.H);
        const bool valid = t < a.T;
        const XT* xhead = reinterpret_cast<const XT*>(a.x) + b * a.sb + h * a.sh;
        float v[8];
        if (valid) {
            load8<XT>(xhead + t * a.st + 8 * l16, v);
        } else {
#pragma unroll
            for (int k = 0; k < 8; ++k) v[k] = 0.f;
        }
        // ---- normalize, shift, normalize ----
        float ss = 0.f;
#pragma unroll
        for (int k = 0; k < 8; ++k) ss = fmaf(v[k], v[k], ss);
        ss = half_sum(ss);
        const float s1 = sqrtf(ss * (1.0f / kD));
        const float inv1 = s1 > 0.f ? 1.0f / s1 : 0.f;
        const float4* o4 = reinterpret_cast<const float4*>(a.shift + bh * kD + 8 * l16);
        const float4 oa = o4[0], ob = o4[1];
        const float o[8] = {oa.x, oa.y, oa.z, oa.w, ob.x, ob.y, ob.z, ob.w};
        float ss2 = 0.f;
#pragma unroll
        for (int k = 0; k < 8; ++k) {
            v[k] = fmaf(v[k], inv1, -o[k]);
            ss2 = fmaf(v[k], v[k], ss2);
        }
        ss2 = half_sum(ss2);
        const float s2 = sqrtf(ss2 * (1.0f / kD));
        const bool cancel = s2 < kCancel1;
        const float sc = s2 > 0.f ? kRsqrtD / s2 : 0.f;
        // ---- FWHT: bits 0-2 in registers, bits 3-6 across the token's 16 lanes ----
#pragma unroll
        for (int k = 0; k < 8; ++k) v[k] *= sc;
#pragma unroll
        for (int bit = 1; bit < 8; bit <<= 1) {
#pragma unroll
            for (int k = 0; k < 8; ++k) {
                if (k & bit) continue;
                const float x0 = v[k], x1 = v[k | bit];
                v[k] = x0 + x1;
                v[k | bit] = x0 - x1;
            }
        }
#pragma unroll
        for (int m = 1; m < 16; m <<= 1) {
            const float sg = (l16 & m) ? -1.0f : 1.0f;
#pragma unroll
            for (int k = 0; k < 8; ++k) {
                const float p = __shfl_xor_sync(kFull, v[k], m);
                v[k] = fmaf(v[k], sg, p);  // lower index a + b, upper index b - a
            }
        }
        // ---- all 256 codewords, two per step ----
        uint64_t w2[8];
        float ww = 0.f;
#pragma unroll
        for (int k = 0; k < 8; ++k) {
            w2[k] = pk2(v[k], v[k]);
            ww = fmaf(v[k], v[k], ww);
        }
        float b1 = INFINITY, b2 = INFINITY;
        int i1 = 0;
#pragma unroll 4
        for (int q = 0; q < kNC / 2; ++q) {
            const float2 n = n2p[q];
            uint64_t acc = pk2(n.x, n.y);
            const float4* tq = reinterpret_cast<const float4*>(tbl[q]);
#pragma unroll
            for (int k4 = 0; k4 < 4; ++k4) {
                const float4 t4 = tq[k4];
                acc = ffma2(w2[2 * k4], pk2(t4.x, t4.y), acc);
                acc = ffma2(w2[2 * k4 + 1], pk2(t4.z, t4.w), acc);
            }
            const float2 sv = upk2(acc);
            b2 = fminf(b2, fmaxf(b1, sv.x));
            i1 = sv.x < b1 ? 2 * q : i1;
            b1 = fminf(b1, sv.x);
            b2 = fminf(b2, fmaxf(b1, sv.y));
            i1 = sv.y < b1 ? 2 * q + 1 : i1;
            b1 = fminf(b1, sv.y);
        }
        bool tie = cancel || (b2 - b1) <= fmaf(kTieRel1, ww + b1, kTieAbs1);
        if (!valid) tie = false;
        float wq = 0.f;
        if constexpr (ADAPT) {  // w . C[best] = (|C|^2 - s) / 2, summed over the token
            const float2 n = n2p[i1 >> 1];
            wq = half_sum(0.5f * (((i1 & 1) ? n.y : n.x) - b1));
        }
        // ---- codes of the two token-heads, then the exact path ----
        uint32_t cw[4];
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            uint32_t word = 0u;
#pragma unroll
            for (int r = 0; r < 4; ++r)
                word |= (uint32_t)__shfl_sync(kFull, i1, 16 * half + 4 * k + r) << (8 * r);
            cw[k] = word;
        }
        uint4 codes = make_uint4(cw[0], cw[1], cw[2], cw[3]);
        float s1o = s1, s2o = s2;
        double wqd = (double)wq;
        const uint32_t tmask = __ballot_sync(kFull, tie);
        if (tmask) {
            const double* o64 = a.given_shift ? nullptr : a.o64 + bh * kD;
#pragma unroll 1
            for (int hh = 0; hh < 2; ++hh) {
                const uint32_t flags = (tmask >> (16 * hh)) & 0xffffu;  // bit j: sub-vector j
                if (!flags) continue;  // warp-uniform
                uint4 cq = make_uint4(__shfl_sync(kFull, codes.x, 16 * hh), __shfl_sync(kFull, codes.y, 16 * hh),
                                      __shfl_sync(kFull, codes.z, 16 * hh), __shfl_sync(kFull, codes.w, 16 * hh));
                double s1d, s2d, wq64;
                exact_warp1<XT>(xhead + (t0 + hh) * a.st, o64, a.shift + bh * kD, Cs, flags, cq, s1d, s2d,
                                wq64);
                if (half == hh) {
                    codes = cq;
                    s1o = (float)s1d;
                    s2o = (float)s2d;
                    wqd = wq64;
                }
                if (lane == 0 && a.stats) {
                    atomicAdd(&a.stats[0], 1ull);
                    atomicAdd(&a.stats[1], (unsigned long long)__popc(flags));
                }
            }
        }
        if constexpr (ADAPT) {
            if (wqd > 0.0) s2o = (float)((double)s2o * ((double)kD / wqd));
        }
        if (valid && l16 == 0) {
            const int64_t row = bh * a.cap + a.t_offset + t;
            reinterpret_cast<uint4*>(a.codes + row * 16)[0] = codes;
            reinterpret_cast<float2*>(a.scales)[row] = make_float2(s1o, s2o);
        }
    }
}

template <typename XT, bool ADAPT>
cudaError_t launch_t(const EncodeArgs& a, cudaStream_t s) {
    int dev = 0, sms = 148;
    if (cudaGetDevice(&dev) == cudaSuccess)
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const int64_t npairs = (int64_t)a.B * a.H * ((a.T + 1) / 2);
    const int64_t need = (npairs + kThreads1 / 32 - 1) / (kThreads1 / 32);
    const int64_t cap = (int64_t)sms * 3;  // resident blocks per SM at 80 registers per thread
    const int grid = (int)(need < cap ? need : cap);
    nsn_encode1_kernel<XT, ADAPT><<<grid, kThreads1, 0, s>>>(a);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_encode1(const EncodeArgs& a, cudaStream_t s) {
    if (a.adaptive)
        return a.x_bf16 ? launch_t<__nv_bfloat16, true>(a, s) : launch_t<float, true>(a, s);
    return a.x_bf16 ? launch_t<__nv_bfloat16, false>(a, s) : launch_t<float, false>(a, s);
}

}  // namespace nsnq
