// Full-precision residual window: copy of new tokens into the window buffer
// (NSNQuant Technical Summary, Methodology §4, Implementation Details,
// Residuals). The attention over the window runs in the combine kernel of
// attention.cu; the flush is an encode with the stored shift.
//
//   residual_write_kernel  one warp per token row, 4 channels per lane
#include "common.cuh"
#include "internal.h"

namespace nsnq {

constexpr int kWriteThreads = 256;

__device__ __forceinline__ void store4(float* p, const float (&v)[4]) {
    *reinterpret_cast<float4*>(p) = make_float4(v[0], v[1], v[2], v[3]);
}
__device__ __forceinline__ void store4(__nv_bfloat16* p, const float (&v)[4]) {
    uint2 u;
    u.x = (uint32_t)f32_to_bf16_rn(v[0]) | ((uint32_t)f32_to_bf16_rn(v[1]) << 16);
    u.y = (uint32_t)f32_to_bf16_rn(v[2]) | ((uint32_t)f32_to_bf16_rn(v[3]) << 16);
    *reinterpret_cast<uint2*>(p) = u;
}

template <typename XT, typename BT>
__global__ void __launch_bounds__(kWriteThreads) residual_write_kernel(ResWriteArgs a) {
    const int lane = lane_id();
    const int64_t rows = (int64_t)a.B * a.H * a.T;
    const int64_t wpb = kWriteThreads / 32;
    for (int64_t r = (int64_t)blockIdx.x * wpb + (threadIdx.x >> 5); r < rows;
         r += (int64_t)gridDim.x * wpb) {
        const int64_t bh = r / a.T, t = r - bh * a.T;
        const int64_t b = bh / a.H, h = bh - b * a.H;
        const XT* src = reinterpret_cast<const XT*>(a.x) + b * a.sb + h * a.sh + t * a.st;
        BT* dst = reinterpret_cast<BT*>(a.buf) + (bh * a.cap + a.t_offset + t) * kD;
        float v[4];
        load4(src + 4 * lane, v);
        store4(dst + 4 * lane, v);
    }
}

cudaError_t launch_residual_write(const ResWriteArgs& a, cudaStream_t s) {
    const int64_t rows = (int64_t)a.B * a.H * a.T;
    const int64_t wpb = kWriteThreads / 32;
    const int grid = (int)((rows + wpb - 1) / wpb < 4096 ? (rows + wpb - 1) / wpb : 4096);
    if (a.x_bf16) {
        if (a.buf_bf16) residual_write_kernel<__nv_bfloat16, __nv_bfloat16><<<grid, kWriteThreads, 0, s>>>(a);
        else residual_write_kernel<__nv_bfloat16, float><<<grid, kWriteThreads, 0, s>>>(a);
    } else {
        if (a.buf_bf16) residual_write_kernel<float, __nv_bfloat16><<<grid, kWriteThreads, 0, s>>>(a);
        else residual_write_kernel<float, float><<<grid, kWriteThreads, 0, s>>>(a);
    }
    return cudaGetLastError();
}

}  // namespace nsnq
