// Decode attention with keys quantized before RoPE (gist.science "NSNQuant
// ...", Technical Summary, Methodology §4, Implementation Details: NSN runs
// on the keys before the rotary position embedding, so attention rotates the
// dequantized keys).
//
// The rotation depends on the key's position, so the single rotated-query
// table of the plain kernel does not apply: every key is dequantized in
// registers, k_t = s1 (s2 H w_hat + o), rotated to position t, and dotted
// with the query heads (already rotated at their own position by the
// caller). Rotary embedding: channel i pairs with channel i + 64 (i < 64),
// angle t * base^(-i/64). Per lane (= token) the codewords are gathered into
// packed pairs (w_i, w_{i+64}), six FWHT stages run on the pairs and the last
// one (bit 6) combines the two halves, which leaves exactly the rotary pairs.
// cos/sin of t theta_i come from angle addition: a per-warp fp64 seed for the
// batch's first token and a per-lane table for the offset 0..31.
// The value side (online softmax, values in the Hadamard domain, the split
// partials and the combine kernel) is that of the plain decode attention.
#include <math.h>

#include "attn_split.cuh"
#include "common.cuh"
#include "f32x2.cuh"
#include "internal.h"

namespace nsnq {

namespace {

constexpr int kRopeWarps = 8;  // the key (128 values in packed pairs) stays in registers
constexpr int kRopeThreads = kRopeWarps * 32;
constexpr int kHalf = kD / 2;


// Shared-memory map (bytes):
//   krep  K codewords, [256][KSUB/4][8 copies] 16-byte pieces
//   vrep  V codewords, same layout
//   rotL  float2 [64][32]: (cos, sin) of lane * theta_i
//   theta double [64]
//   qp    float2 [64][GC]: (q_h[i], q_h[i+64])
//   op    float2 [64]: (o_i, o_{i+64}) of the unit's K shift
//   per warp: seed float4 [64] (c0, s0, -s0, c0), V codes [32][VJ], weights [32][GC]
//             as duplicated pairs (w, w)
template <int GC, int KSUB, int VSUB>
struct RopeSmem {
    static constexpr int VJ = kD / VSUB;
    static constexpr size_t krep = (size_t)kNC * (KSUB / 4) * 8 * 16;
    static constexpr size_t vrep = (size_t)kNC * (VSUB / 4) * 8 * 16;
    static constexpr size_t rotl = (size_t)kHalf * 32 * 8;
    static constexpr size_t theta = (size_t)kHalf * 8;
    static constexpr size_t qp = (size_t)kHalf * GC * 8;
    static constexpr size_t op = (size_t)kHalf * 8;
    static constexpr size_t seed = (size_t)kHalf * 16;
    static constexpr size_t wcodes = (size_t)32 * VJ;
    static constexpr size_t wweights = (size_t)32 * GC * 8;
    static constexpr size_t per_warp = seed + wcodes + wweights;
    static constexpr size_t merge = (size_t)kRopeWarps * GC * (3 + kD) * 4;
    static constexpr size_t o_vrep = krep;
    static constexpr size_t o_rotl = o_vrep + vrep;
    static constexpr size_t o_theta = o_rotl + rotl;
    static constexpr size_t o_qp = o_theta + theta;
    static constexpr size_t o_op = o_qp + qp;
    static constexpr size_t o_warp = o_op + op;
    static constexpr size_t o_merge = o_warp + per_warp * kRopeWarps;
    static constexpr size_t bytes = o_merge + merge;
    static_assert(bytes <= 232448, "shared memory per block");
};

template <int GC, int KSUB, int VSUB, typename QT>
__global__ void __launch_bounds__(kRopeThreads, 1) attn_rope_split_kernel(AttnArgs a) {
    using S = RopeSmem<GC, KSUB, VSUB>;
    constexpr int KJ = kD / KSUB, VJ = S::VJ;
    constexpr int KW = KJ / 4;  // 32-bit words per K code row
    extern __shared__ __align__(16) uint8_t smb[];
    float4* krep = reinterpret_cast<float4*>(smb);
    float4* vrep = reinterpret_cast<float4*>(smb + S::o_vrep);
    float2* rotL = reinterpret_cast<float2*>(smb + S::o_rotl);
    double* theta = reinterpret_cast<double*>(smb + S::o_theta);
    float2* qp = reinterpret_cast<float2*>(smb + S::o_qp);
    float2* op = reinterpret_cast<float2*>(smb + S::o_op);
    float* mergeb = reinterpret_cast<float*>(smb + S::o_merge);

    const int tid = threadIdx.x, lane = lane_id(), warp = tid >> 5;
    const int G = a.Hq / a.Hkv;
    const int cta = blockIdx.x;
    const int64_t L = a.plan.L;
    const int nslot = a.plan.nslot;
    const int64_t vbeg = cta_begin(cta, a.plan), vend = cta_begin(cta + 1, a.plan);

    for (int i = tid; i < kNC * (KSUB / 4) * 8; i += kRopeThreads)  // [piece][copy]
        krep[i] = reinterpret_cast<const float4*>(a.kC)[i >> 3];
    for (int i = tid; i < kNC * (VSUB / 4) * 8; i += kRopeThreads)
        vrep[i] = reinterpret_cast<const float4*>(a.vC)[i >> 3];
    for (int i = tid; i < kHalf; i += kRopeThreads) theta[i] = pow(a.rope_base, -(double)i / (double)kHalf);
    __syncthreads();
    for (int e = tid; e < kHalf * 32; e += kRopeThreads) {  // [i][lane]
        double sn, cs;
        sincos((double)(e & 31) * theta[e >> 5], &sn, &cs);
        rotL[e] = make_float2((float)cs, (float)sn);
    }

    uint8_t* warp_area = smb + S::o_warp + (size_t)warp * S::per_warp;
    float4* seed = reinterpret_cast<float4*>(warp_area);
    uint8_t* my_codes = warp_area + S::seed;
    uint64_t* my_w = reinterpret_cast<uint64_t*>(my_codes + S::wcodes);  // [32][GC] (w, w)
    constexpr int TPI = 32 / VJ;  // tokens per V step (1 at VSUB=4, 2 at VSUB=8)
    const int jj = lane % VJ, sub_t = lane / VJ;
    const float4* kmy = krep + (lane & 7);
    const ulonglong2* myrep = reinterpret_cast<const ulonglong2*>(vrep) + (lane & 7);

  for (int64_t u = vbeg / L; u < a.plan.units && u * L < vend; ++u) {
    const int64_t per_b = (int64_t)a.Hkv * a.plan.ngroups;
    const int b = (int)(u / per_b);
    const int kvh = (int)((u % per_b) / a.plan.ngroups), hg = (int)(u % a.plan.ngroups);
    const int qh0 = kvh * G + hg * GC;
    const int64_t bkv = (int64_t)b * a.Hkv + kvh;
    const int slot = cta - first_cta(u * L, a.plan);
    int64_t len = a.seq_lens[b];
    len = len < 0 ? 0 : (len > a.max_len ? a.max_len : len);
    const int64_t ts = max(vbeg, u * L) - u * L;
    const int64_t te = min(min(vend, (u + 1) * L) - u * L, len);
    __syncthreads();  // the previous segment is done with qp, op and the merge area

    if (ts >= te) {  // nothing to attend in this segment: neutral partial
        for (int idx = tid; idx < GC * kPartStride; idx += kRopeThreads) {
            const int h = idx / kPartStride, c = idx % kPartStride;
            float* P = a.part + (((int64_t)b * a.Hq + qh0 + h) * nslot + slot) * kPartStride;
            P[c] = (c == kD) ? -INFINITY : 0.f;
        }
        continue;
    }

    // ---- segment prologue: query pairs and shift pairs ----
    for (int e = tid; e < kHalf * GC; e += kRopeThreads) {
        const int i = e / GC, h = e % GC;
        const int64_t qo = ((int64_t)b * a.Hq + qh0 + h) * kD;
        const QT* qq = reinterpret_cast<const QT*>(a.q);
        qp[e] = make_float2((float)qq[qo + i], (float)qq[qo + i + kHalf]);
    }
    for (int i = tid; i < kHalf; i += kRopeThreads)
        op[i] = make_float2(a.kshift[bkv * kD + i], a.kshift[bkv * kD + i + kHalf]);
    __syncthreads();

    float m[GC], l[GC], be[GC];
    uint64_t acc[GC][VSUB / 2];
#pragma unroll
    for (int h = 0; h < GC; ++h) {
        m[h] = -INFINITY; l[h] = 0.f; be[h] = 0.f;
#pragma unroll
        for (int r = 0; r < VSUB / 2; ++r) acc[h][r] = 0ull;
    }
    const uint8_t* kc = a.kcodes + bkv * a.kcap * KJ;
    const uint8_t* vc = a.vcodes + bkv * a.vcap * VJ;
    const float lvlK = packed_level_lane(a.klevels, a.kgrid, bkv);
    const float lvlV = packed_level_lane(a.vlevels, a.vgrid, bkv);
    const ByproductSrc ksrc = byproduct_src(a.kscales, a.klevels, bkv, a.kcap);
    const ByproductSrc vsrc = byproduct_src(a.vscales, a.vlevels, bkv, a.vcap);

    for (int64_t base = ts + warp * 32; base < te; base += kRopeWarps * 32) {
        const int64_t t = base + lane;
        const bool valid = t < te;
        // seed of the batch: (cos, sin) of base * theta_i in fp64
        __syncwarp();
#pragma unroll
        for (int r = 0; r < 2; ++r) {
            const int i = lane + 32 * r;
            double sn, cs;
            sincos((double)base * theta[i], &sn, &cs);
            seed[i] = make_float4((float)cs, (float)sn, (float)-sn, (float)cs);
        }
        uint32_t kw[KW];
        const float2 k2 = load_byproducts(ksrc, (uint32_t)t, valid, lvlK);
        const float2 v2 = load_byproducts(vsrc, (uint32_t)t, valid, lvlV);
        if (valid) {
            const uint4* kr = reinterpret_cast<const uint4*>(kc + t * KJ);
#pragma unroll
            for (int q4 = 0; q4 < KW / 4; ++q4) {
                const uint4 w4 = __ldg(kr + q4);
                kw[4 * q4] = w4.x; kw[4 * q4 + 1] = w4.y; kw[4 * q4 + 2] = w4.z; kw[4 * q4 + 3] = w4.w;
            }
            const uint4* vr = reinterpret_cast<const uint4*>(vc + t * VJ);
            uint4* dst = reinterpret_cast<uint4*>(my_codes + lane * VJ);
#pragma unroll
            for (int q4 = 0; q4 < VJ / 16; ++q4) dst[q4] = __ldg(vr + q4);
        } else {
#pragma unroll
            for (int i = 0; i < KW; ++i) kw[i] = 0u;
        }
        // ---- dequantize the key in packed pairs P[i] = (w_i, w_{i+64}) ----
        uint64_t P[kHalf];
#pragma unroll
        for (int j = 0; j < KJ / 2; ++j) {  // sub-vector j holds i in [j KSUB, (j+1) KSUB), j + KJ/2 the partners
            const int clo = (int)((kw[j >> 2] >> (8 * (j & 3))) & 0xffu);
            const int jh = j + KJ / 2;
            const int chi = (int)((kw[jh >> 2] >> (8 * (jh & 3))) & 0xffu);
#pragma unroll
            for (int k = 0; k < KSUB / 4; ++k) {
                const float4 lo = kmy[(clo * (KSUB / 4) + k) * 8];
                const float4 hi = kmy[(chi * (KSUB / 4) + k) * 8];
                const int i0 = j * KSUB + 4 * k;
                P[i0] = pk2(lo.x, hi.x);
                P[i0 + 1] = pk2(lo.y, hi.y);
                P[i0 + 2] = pk2(lo.z, hi.z);
                P[i0 + 3] = pk2(lo.w, hi.w);
            }
        }
#pragma unroll
        for (int bit = 1; bit < kHalf; bit <<= 1) {  // FWHT bits 0-5 on both halves at once
#pragma unroll
            for (int i = 0; i < kHalf; ++i) {
                if (i & bit) continue;
                const uint64_t x0 = P[i], x1 = P[i | bit];
                P[i] = add2(x0, x1);
                P[i | bit] = sub2(x0, x1);
            }
        }
        __syncwarp();  // the seed is written
        // k = s1 (s2 H w + o): A (unnormalised FWHT) + s1 o; then rotate and dot
        const float A = k2.x * k2.y * kRsqrtD;
        const uint64_t A2 = pk2(A, A), S1 = pk2(k2.x, k2.x);
        uint64_t sacc[GC];
#pragma unroll
        for (int h = 0; h < GC; ++h) sacc[h] = 0ull;
        // seed read as packed pairs (c0, s0), (-s0, c0); shift and query
        // pairs (x_i, x_{i+64}) read as one 64-bit word each
        const float2* myL = rotL + lane;
        const ulonglong2* sd2 = reinterpret_cast<const ulonglong2*>(seed);
        const uint64_t* op2 = reinterpret_cast<const uint64_t*>(op);
        const uint64_t* qp2 = reinterpret_cast<const uint64_t*>(qp);
#pragma unroll
        for (int i = 0; i < kHalf; ++i) {
            const float2 y = upk2(P[i]);
            const uint64_t kk = fma2(pk2(y.x + y.y, y.x - y.y), A2, mul2(op2[i], S1));  // (k_i, k_{i+64})
            const ulonglong2 sd = sd2[i];
            const float2 lr = myL[32 * i];
            const float2 cs = upk2(fma2(sd.x, pk2(lr.x, lr.x), mul2(sd.y, pk2(lr.y, lr.y))));  // angle addition
            const float2 kf = upk2(kk);
            // rotated pair: (k_i c - k_{i+64} s, k_i s + k_{i+64} c)
            const uint64_t rk = fma2(pk2(cs.x, cs.x), kk, mul2(pk2(cs.y, cs.y), pk2(-kf.y, kf.x)));
#pragma unroll
            for (int h = 0; h < GC; ++h) sacc[h] = fma2(rk, qp2[i * GC + h], sacc[h]);
        }
        // ---- online softmax (log2 domain), lazy running max as in the plain
        //      kernel: raised (and the accumulators rescaled) only when a
        //      logit exceeds it by more than kLazy
        float logit[GC];
        bool raise = false;
#pragma unroll
        for (int h = 0; h < GC; ++h) {
            const float2 sp = upk2(sacc[h]);
            logit[h] = valid ? (sp.x + sp.y) * a.scale_log2 : -INFINITY;
            raise |= logit[h] > m[h] + kLazy;
        }
        if (__any_sync(kFull, raise)) {  // warp-uniform, rare
#pragma unroll
            for (int h = 0; h < GC; ++h) {
                if (__any_sync(kFull, logit[h] > m[h] + kLazy)) {
                    const float mx = warp_max(logit[h]);
                    const float alpha = (m[h] == -INFINITY) ? 0.f : exp2_approx(m[h] - mx);
                    l[h] *= alpha;
                    be[h] *= alpha;
                    const uint64_t al = pk2(alpha, alpha);
#pragma unroll
                    for (int r = 0; r < VSUB / 2; ++r) acc[h][r] = mul2(acc[h][r], al);
                    m[h] = mx;
                }
            }
        }
        // every batch holds a valid token: m is finite and invalid lanes get p = 0
        const float vw = v2.x * v2.y;
#pragma unroll
        for (int h = 0; h < GC; ++h) {
            const float p = exp2_approx(logit[h] - m[h]);
            l[h] += p;
            be[h] = fmaf(p, v2.x, be[h]);
            const float w = p * vw;
            my_w[lane * GC + h] = pk2(w, w);
        }
        __syncwarp();
        // ---- values: lane = sub-vector, fp32 codewords, Hadamard domain ----
        const int nt = (int)min((int64_t)32, te - base);
        for (int i = 0; i < nt; i += TPI) {
            const int tt = i + sub_t;
            if (tt < nt) {
                const int code = my_codes[tt * VJ + jj];
                uint64_t c[VSUB / 2];  // codeword as packed pairs
#pragma unroll
                for (int k = 0; k < VSUB / 4; ++k) {
                    const ulonglong2 cv = myrep[(code * (VSUB / 4) + k) * 8];
                    c[2 * k] = cv.x; c[2 * k + 1] = cv.y;
                }
#pragma unroll
                for (int h = 0; h < GC; ++h) {
                    const uint64_t wp = my_w[tt * GC + h];
#pragma unroll
                    for (int r = 0; r < VSUB / 2; ++r) acc[h][r] = fma2(c[r], wp, acc[h][r]);
                }
            }
        }
        __syncwarp();
    }

#pragma unroll
    for (int h = 0; h < GC; ++h) {
        l[h] = warp_sum(l[h]);
        be[h] = warp_sum(be[h]);
        if constexpr (TPI == 2) {
#pragma unroll
            for (int r = 0; r < VSUB / 2; ++r) {
                const float2 v = upk2(acc[h][r]);
                acc[h][r] = pk2(v.x + __shfl_xor_sync(kFull, v.x, 16), v.y + __shfl_xor_sync(kFull, v.y, 16));
            }
        }
    }
    // ---- merge the warps' partials, write this segment's row ----
    float* mw = mergeb;
    float* lw = mw + kRopeWarps * GC;
    float* bw = lw + kRopeWarps * GC;
    float* Aw = bw + kRopeWarps * GC;  // [warp][h][128]
    if (lane == 0) {
#pragma unroll
        for (int h = 0; h < GC; ++h) {
            mw[warp * GC + h] = m[h]; lw[warp * GC + h] = l[h]; bw[warp * GC + h] = be[h];
        }
    }
    if (lane < VJ) {
#pragma unroll
        for (int h = 0; h < GC; ++h)
#pragma unroll
            for (int r = 0; r < VSUB / 2; ++r) {
                const float2 v = upk2(acc[h][r]);
                Aw[(warp * GC + h) * kD + jj * VSUB + 2 * r] = v.x;
                Aw[(warp * GC + h) * kD + jj * VSUB + 2 * r + 1] = v.y;
            }
    }
    __syncthreads();
    for (int idx = tid; idx < GC * (kD + 2); idx += kRopeThreads) {
        const int h = idx / (kD + 2), c = idx % (kD + 2);
        float M = -INFINITY;
#pragma unroll
        for (int w = 0; w < kRopeWarps; ++w) M = fmaxf(M, mw[w * GC + h]);
        float accm = 0.f;
#pragma unroll
        for (int w = 0; w < kRopeWarps; ++w) {
            const float mv = mw[w * GC + h];
            const float f = (mv == -INFINITY) ? 0.f : exp2_approx(mv - M);
            float v;
            if (c < kD) v = Aw[(w * GC + h) * kD + c];
            else if (c == kD) v = lw[w * GC + h];
            else v = bw[w * GC + h];
            accm = fmaf(f, v, accm);
        }
        float* Pp = a.part + (((int64_t)b * a.Hq + qh0 + h) * nslot + slot) * kPartStride;
        if (c < kD) Pp[c] = accm;
        else if (c == kD) { Pp[kD] = M; Pp[kD + 1] = accm; }
        else Pp[kD + 2] = accm;  // c == kD + 1: beta
    }
  }
}

template <int GC, int KSUB, int VSUB, typename QT>
cudaError_t launch_rope_split(const AttnArgs& a, cudaStream_t s) {
    using S = RopeSmem<GC, KSUB, VSUB>;
    static std::atomic<unsigned long long> ready{0};
    return launch_smem(attn_rope_split_kernel<GC, KSUB, VSUB, QT>, ready, dim3(a.plan.ctas),
                       dim3(kRopeThreads), S::bytes, s, a);
}

template <int GC, typename QT>
cudaError_t launch_rope_sub(const AttnArgs& a, cudaStream_t s) {
    if (a.ksub == 4 && a.vsub == 4) return launch_rope_split<GC, 4, 4, QT>(a, s);
    if (a.ksub == 4 && a.vsub == 8) return launch_rope_split<GC, 4, 8, QT>(a, s);
    if (a.ksub == 8 && a.vsub == 4) return launch_rope_split<GC, 8, 4, QT>(a, s);
    return launch_rope_split<GC, 8, 8, QT>(a, s);
}

template <typename QT>
cudaError_t launch_rope_gc(const AttnArgs& a, cudaStream_t s) {
    if (a.plan.gc == 4) return launch_rope_sub<4, QT>(a, s);
    if (a.plan.gc == 2) return launch_rope_sub<2, QT>(a, s);
    return launch_rope_sub<1, QT>(a, s);
}

}  // namespace

cudaError_t launch_attention_rope(const AttnArgs& a, cudaStream_t s) {
    cudaError_t e = a.q_bf16 ? launch_rope_gc<__nv_bfloat16>(a, s) : launch_rope_gc<float>(a, s);
    if (e != cudaSuccess) return e;
    return launch_attn_combine(a, s);
}

}  // namespace nsnq
