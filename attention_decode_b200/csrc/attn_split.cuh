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

}  // namespace nsnq
