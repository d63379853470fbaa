// Device helpers shared by the NSNQuant kernels (sm_100a).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace nsnq {

constexpr int kD = 128;            // head_dim supported by the kernels
constexpr int kNC = 256;           // codebook entries (one byte per code)
constexpr unsigned kFull = 0xffffffffu;
constexpr float kRsqrtD = 0.08838834764831845f;      // 1/sqrt(128), fp32
constexpr double kRsqrtDd = 0.088388347648318440550;  // 1/sqrt(128), fp64
constexpr float kLog2e = 1.4426950408889634f;

__device__ __forceinline__ int lane_id() { return threadIdx.x & 31; }

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
    for (int m = 16; m; m >>= 1) v += __shfl_xor_sync(kFull, v, m);
    return v;
}

__device__ __forceinline__ double warp_sum_d(double v) {
#pragma unroll
    for (int m = 16; m; m >>= 1) v += __shfl_xor_sync(kFull, v, m);
    return v;
}

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
    for (int m = 16; m; m >>= 1) v = fmaxf(v, __shfl_xor_sync(kFull, v, m));
    return v;
}

// Four consecutive channels as fp32 (exact for both I/O types).
__device__ __forceinline__ void load4(const float* p, float (&v)[4]) {
    float4 a = *reinterpret_cast<const float4*>(p);
    v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
}
__device__ __forceinline__ void load4(const __nv_bfloat16* p, float (&v)[4]) {
    uint2 a = *reinterpret_cast<const uint2*>(p);
    v[0] = __uint_as_float(a.x << 16);
    v[1] = __uint_as_float(a.x & 0xffff0000u);
    v[2] = __uint_as_float(a.y << 16);
    v[3] = __uint_as_float(a.y & 0xffff0000u);
}

// Unnormalised Walsh-Hadamard transform (Sylvester order) of 128 values held
// four per lane: lane l owns coordinates 4l..4l+3. Coordinate bits 0-1 are
// in registers, bits 2-6 are the lane bits 0-4. Butterfly on bit b: the lower
// index gets a + b, the upper index gets a - b.
template <typename F>
__device__ __forceinline__ void fwht128_lane4(F (&v)[4]) {
    const int lane = lane_id();
    F a0 = v[0] + v[1], a1 = v[0] - v[1], a2 = v[2] + v[3], a3 = v[2] - v[3];
    v[0] = a0 + a2; v[1] = a1 + a3; v[2] = a0 - a2; v[3] = a1 - a3;
#pragma unroll
    for (int m = 1; m < 32; m <<= 1) {
        const bool upper = (lane & m) != 0;
#pragma unroll
        for (int r = 0; r < 4; ++r) {
            F p = __shfl_xor_sync(kFull, v[r], m);
            v[r] = upper ? (p - v[r]) : (v[r] + p);
        }
    }
}

__device__ __forceinline__ uint16_t f32_to_bf16_rn(float f) {
    return __bfloat16_as_ushort(__float2bfloat16_rn(f));
}

}  // namespace nsnq
