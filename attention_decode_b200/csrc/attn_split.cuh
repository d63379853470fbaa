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

// (s1, s2) of token t of one head in a cache of either form, in two steps so
// that a prefetch does not wait for its loads: fetch_byproducts issues the
// loads (packed form: s2 from scales[t], sign bit set for s1 = 0, and the
// word holding t's 4-bit level; otherwise the (s1, s2) pair), and
// resolve_byproducts, called when the values are needed, turns the level
// into s1 by a shuffle from lane k of `lvl` (lanes 0..15 hold the 16 level
// values), so every lane of the warp must call it together. Invalid lanes
// load nothing and get (0, 0). Token indices are 32-bit (sequence lengths
// are int32); the head's rows are addressed from ByproductSrc.
struct RawByproducts {
    float a;     // s2 (packed) or s1
    uint32_t b;  // level word (packed) or the bits of s2
};
struct ByproductSrc {
    const float* s;       // head's scales: s2 per token (packed) or (s1, s2) pairs
    const uint32_t* lv;   // head's level words (packed), else nullptr
};
__device__ __forceinline__ ByproductSrc byproduct_src(const float* scales, const uint32_t* levels,
                                                      int64_t bkv, int64_t cap) {
    ByproductSrc r;
    if (levels) {
        r.s = scales + bkv * cap;
        r.lv = levels + bkv * ((cap + 7) >> 3);
    } else {
        r.s = scales + 2 * bkv * cap;
        r.lv = nullptr;
    }
    return r;
}
__device__ __forceinline__ RawByproducts fetch_byproducts(const ByproductSrc& src, uint32_t t,
                                                          bool valid) {
    RawByproducts r{0.f, 0u};
    if (!valid) return r;
    if (src.lv) {
        r.a = __ldg(src.s + t);
        r.b = __ldg(src.lv + (t >> 3));
    } else {
        const float2 v = __ldg(reinterpret_cast<const float2*>(src.s) + t);
        r.a = v.x;
        r.b = __float_as_uint(v.y);
    }
    return r;
}
__device__ __forceinline__ float2 resolve_byproducts(RawByproducts r, const ByproductSrc& src,
                                                     uint32_t t, float lvl) {
    if (src.lv) {
        const float s1 = __shfl_sync(0xffffffffu, lvl, (int)((r.b >> (4 * (t & 7u))) & 15u));
        return make_float2(signbit(r.a) ? 0.f : s1, fabsf(r.a));
    }
    return make_float2(r.a, __uint_as_float(r.b));
}
__device__ __forceinline__ float2 load_byproducts(const ByproductSrc& src, uint32_t t, bool valid,
                                                  float lvl) {
    return resolve_byproducts(fetch_byproducts(src, t, valid), src, t, lvl);
}

// A running max may lag the true max by up to 2^kLazy (log2 units) before the
// accumulators are rescaled; weights then stay below 2^kLazy, far from the
// fp32 range.
constexpr float kLazy = 8.0f;

// 2^x by the hardware approximation (relative error ~2^-22; results below
// 2^-126 flush to zero, weights far below the softmax's resolution).
__device__ __forceinline__ float exp2_approx(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// Lane k < 16 of a warp: level k of head bkv's s1 grid (packed caches), else 0.
__device__ __forceinline__ float packed_level_lane(const uint32_t* levels, const float* grid,
                                                   int64_t bkv) {
    const int k = threadIdx.x & 31;
    if (!levels || k >= 16) return 0.f;
    return (float)exp2((double)grid[2 * bkv] + (double)k * (double)grid[2 * bkv + 1]);
}

}  // namespace nsnq
