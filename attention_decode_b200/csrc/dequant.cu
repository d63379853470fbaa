// NSNQuant dequantization on sm_100a: x_hat = s1 * (s2 * H w_hat + o)
// (gist.science "NSNQuant ...", Technical Summary, Methodology §1: the
// byproducts s1, o, s2 reconstruct the tensor; §2: naive Hadamard).
#include "common.cuh"
#include "dq.cuh"
#include "internal.h"

namespace nsnq {

constexpr int kDequantThreads = 128;

// One warp per token: lane l gathers coordinates 4l..4l+3 of w_hat from its
// codeword, the warp runs the 128-point FWHT, and lane l writes 16 bytes.
template <int SUB>
__global__ void __launch_bounds__(kDequantThreads) nsnq_dequant_kernel(DequantArgs a) {
    __shared__ __align__(16) float Cs[kNC * SUB];
    for (int i = threadIdx.x; i < kNC * SUB; i += blockDim.x) Cs[i] = a.C[i];
    __syncthreads();
    constexpr int J = kD / SUB;
    const int lane = lane_id(), warp = threadIdx.x >> 5;
    const int64_t ntok = (int64_t)a.B * a.H * a.T;
    const float4* C4 = reinterpret_cast<const float4*>(Cs);
    for (int64_t i = (int64_t)blockIdx.x * (kDequantThreads / 32) + warp; i < ntok;
         i += (int64_t)gridDim.x * (kDequantThreads / 32)) {
        const int64_t bh = i / a.T;
        const int64_t row = bh * a.cap + a.t0 + (i - bh * a.T);
        float4 cv;
        if constexpr (SUB == 4) {
            cv = C4[a.codes[row * J + lane]];
        } else {
            cv = C4[2 * a.codes[row * J + (lane >> 1)] + (lane & 1)];
        }
        float v[4] = {cv.x, cv.y, cv.z, cv.w};
        fwht128_lane4(v);
        float2 s;
        if (a.s1_levels) {  // packed: s2 alone (sign bit: s1 = 0) and the 4-bit s1 level
            const float s2 = a.scales[row];
            const int k = dq_packed_level(a.s1_levels, bh, a.cap, a.t0 + (i - bh * a.T));
            s = make_float2(signbit(s2) ? 0.f : dq_level_value(a.s1_grid, bh, k), fabsf(s2));
        } else {
            s = reinterpret_cast<const float2*>(a.scales)[row];
        }
        const float4 o = reinterpret_cast<const float4*>(a.shift + bh * kD)[lane];
        float4 r;
        r.x = s.x * fmaf(s.y, v[0] * kRsqrtD, o.x);
        r.y = s.x * fmaf(s.y, v[1] * kRsqrtD, o.y);
        r.z = s.x * fmaf(s.y, v[2] * kRsqrtD, o.z);
        r.w = s.x * fmaf(s.y, v[3] * kRsqrtD, o.w);
        reinterpret_cast<float4*>(a.out + i * kD)[lane] = r;
    }
}

cudaError_t launch_dequant(const DequantArgs& a, cudaStream_t s) {
    const int64_t ntok = (int64_t)a.B * a.H * a.T;
    const int64_t want = (ntok + (kDequantThreads / 32) - 1) / (kDequantThreads / 32);
    const int grid = (int)(want < 148 * 16 ? want : 148 * 16);
    if (a.sub == 4)
        nsnq_dequant_kernel<4><<<grid, kDequantThreads, 0, s>>>(a);
    else
        nsnq_dequant_kernel<8><<<grid, kDequantThreads, 0, s>>>(a);
    return cudaGetLastError();
}

}  // namespace nsnq
