// Shared by the decode-attention split kernels: the balanced split of the
// flattened (unit, token) space over the CTAs (unit = batch x kv-head x
// head group, L virtual tokens each).
#pragma once

#include <stdint.h>

#include "internal.h"

namespace nsnq {

// Balanced split of the flattened (unit, token) space over the CTAs: CTA c
// covers virtual tokens [cta_begin(c), cta_begin(c + 1)).
__host__ __device__ inline int64_t cta_begin(int c, const AttnPlan& p) {
    const int64_t W = p.units * p.L;
    return (W / p.ctas) * c + ((W % p.ctas) * c) / p.ctas;
}
// The CTA whose range holds virtual token v.
__host__ __device__ inline int first_cta(int64_t v, const AttnPlan& p) {
    const int64_t W = p.units * p.L;
    int c = (int)((double)v * (double)p.ctas / (double)(W > 0 ? W : 1));
    c = c < 0 ? 0 : (c >= p.ctas ? p.ctas - 1 : c);
    while (c + 1 < p.ctas && cta_begin(c + 1, p) <= v) ++c;
    while (c > 0 && cta_begin(c, p) > v) --c;
    return c;
}

// (s1, s2) of token t of head bkv in a cache of either form. Packed form
// (levels != NULL): s2 from scales[t] (sign bit set: s1 = 0) and s1 the
// head's level value k, taken by shuffle from lane k of `lvl` (lanes 0..15
// hold the 16 level values), so every lane of the warp must call this
// together. Invalid lanes read nothing and get (0, 0).
__device__ __forceinline__ float2 load_byproducts(const float* scales, const uint32_t* levels,
                                                  int64_t bkv, int64_t cap, int64_t t, bool valid,
                                                  float lvl) {
    if (levels) {
        float s2 = 0.f;
        uint32_t w = 0u;
        if (valid) {
            s2 = __ldg(scales + bkv * cap + t);
            w = __ldg(levels + bkv * ((cap + 7) >> 3) + (t >> 3));
        }
        const float s1 = __shfl_sync(0xffffffffu, lvl, (int)((w >> (4 * (int)(t & 7))) & 15u));
        return make_float2(signbit(s2) ? 0.f : s1, fabsf(s2));
    }
    return valid ? __ldg(reinterpret_cast<const float2*>(scales) + bkv * cap + t)
                 : make_float2(0.f, 0.f);
}

// Lane k < 16 of a warp: level k of head bkv's s1 grid (packed caches), else 0.
__device__ __forceinline__ float packed_level_lane(const uint32_t* levels, const float* grid,
                                                   int64_t bkv) {
    const int k = threadIdx.x & 31;
    if (!levels || k >= 16) return 0.f;
    return (float)exp2((double)grid[2 * bkv] + (double)k * (double)grid[2 * bkv + 1]);
}

}  // namespace nsnq
