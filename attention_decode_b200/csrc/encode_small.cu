// NSNQuant encode pass 2 for small calls (gist.science "NSNQuant ...",
// Technical Summary, Methodology §1-§3): a decode step appends one token per
// sequence and kv-head, a few hundred token-heads, where the persistent
// kernels' fixed costs (staging the search index, one busy warp per tile)
// dominate. Here one warp takes one token-head and does everything in fp64:
// NSN with warp sums, the Hadamard transform across the warp (lane l holds
// coordinates 4l..4l+3), and the nearest codeword of each sub-vector by a
// full scan of the 256 codewords: in fp32 on the fp64 w rounded to fp32,
// keeping the best and second-best distance, and again in fp64 (lowest index
// on exact ties) where the two are within the near-tie band of the indexed
// search (kTieRel d1 + kTieAbs, far above the fp32 scan's error). Stored s1,
// s2 are the fp64 values rounded to fp32, as the persistent kernels store
// them for the tokens they re-decide in fp64.
#include <math.h>

#include "common.cuh"
#include "dq.cuh"
#include "f32x2.cuh"
#include "internal.h"
#include "vq_index.cuh"

namespace nsnq {

namespace {

constexpr int kSmallThreads = 32;  // one warp (one token-head) per CTA: the CTAs spread over the SMs

template <typename XT, int G, bool ADAPT, bool DQ>
__global__ void __launch_bounds__(kSmallThreads) nsn_encode_small_kernel(EncodeArgs a) {
    // a dependent attention kernel (a decode step's) may be scheduled now;
    // it waits for this grid before reading the codes
    asm volatile("griddepcontrol.launch_dependents;\n" ::: "memory");
    __shared__ __align__(16) double Cs[kNC * G];  // the codebook, converted once
    __shared__ __align__(16) float Cf[kNC * G];   // and as given
    for (int i = threadIdx.x; i < kNC * G; i += kSmallThreads) {
        Cf[i] = a.C[i];
        Cs[i] = (double)a.C[i];
    }
    __syncthreads();
    if (a.zero_stats && blockIdx.x == 0 && threadIdx.x < 8) a.stats[threadIdx.x] = 0ull;
    const int lane = lane_id();
    const int64_t th = (int64_t)blockIdx.x * (kSmallThreads / 32) + (threadIdx.x >> 5);
    if (th >= (int64_t)a.B * a.H * a.T) return;  // warp-uniform
    // th < B H T <= kSmallEncode: 32-bit divisions by the launch's invariants
    const uint32_t bh32 = fdiv((uint32_t)th, a.div_items);  // T
    const int64_t bh = bh32, t = th - bh * a.T;
    const uint32_t b32 = fdiv(bh32, a.div_H);
    const int b = (int)b32, h = (int)(bh32 - b32 * (uint32_t)a.H);
    const bool sec = enc_second(a, bh);
    const int64_t cbh = enc_cbh(a, bh);
    const XT* xtok = enc_head<XT>(a, b, h) + t * a.st;

    // ---- NSN in fp64 ----
    float xf[4];
    load4(xtok + 4 * lane, xf);
    double x[4], o[4];
#pragma unroll
    for (int r = 0; r < 4; ++r) {
        x[r] = (double)xf[r];
        o[r] = a.given_shift ? (double)enc_shift(a, sec)[cbh * kD + 4 * lane + r]
                             : a.o64[bh * kD + 4 * lane + r];
    }
    const double sqrt_d = sqrt((double)kD);
    const double ss = warp_sum_d(x[0] * x[0] + x[1] * x[1] + x[2] * x[2] + x[3] * x[3]);
    double s1 = sqrt(ss) / sqrt_d;
    int s1lev = 0;
    if constexpr (DQ) {
        double glo, gstep;
        dq_grid(enc_s1_grid(a, sec), cbh, glo, gstep);
        s1 = dq_s1(s1, glo, gstep, &s1lev);
    }
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
    double w[G];
    int j;  // this lane's sub-vector
    int c0, c1;  // the codewords it scans
    if constexpr (G == 4) {
#pragma unroll
        for (int r = 0; r < 4; ++r) w[r] = z[r] * hs;
        j = lane;
        c0 = 0;
        c1 = kNC;
    } else {
        // sub-vector j = coordinates 8j..8j+7 (lanes 2j, 2j+1); the two
        // halves of the warp scan the two halves of the codebook
        j = lane & 15;
#pragma unroll
        for (int r = 0; r < 4; ++r) {
            w[r] = __shfl_sync(kFull, z[r], 2 * j) * hs;
            w[4 + r] = __shfl_sync(kFull, z[r], 2 * j + 1) * hs;
        }
        c0 = (lane >> 4) * (kNC / 2);
        c1 = c0 + kNC / 2;
    }
    // ---- nearest codeword: fp32 scan with the best and second best ----
    uint64_t wp[G / 2];
#pragma unroll
    for (int r = 0; r < G / 2; ++r) wp[r] = pk2((float)w[2 * r], (float)w[2 * r + 1]);
    float b1 = INFINITY, b2 = INFINITY;
    int bi = c0;
#pragma unroll 4
    for (int c = c0; c < c1; ++c) {
        const float4* cv = reinterpret_cast<const float4*>(Cf + c * G);
        uint64_t acc = 0ull;
#pragma unroll
        for (int r = 0; r < G / 4; ++r) {
            const float4 q = cv[r];
            const uint64_t e0 = sub2(wp[2 * r], pk2(q.x, q.y)), e1 = sub2(wp[2 * r + 1], pk2(q.z, q.w));
            acc = fma2(e1, e1, fma2(e0, e0, acc));
        }
        const float2 dd = upk2(acc);
        const float d = dd.x + dd.y;
        b2 = fminf(b2, fmaxf(b1, d));
        bi = d < b1 ? c : bi;
        b1 = fminf(b1, d);
    }
    if constexpr (G == 8) {  // merge the two codebook halves (the lower wins exact ties)
        const float o1 = __shfl_xor_sync(kFull, b1, 16), o2 = __shfl_xor_sync(kFull, b2, 16);
        const int oi = __shfl_xor_sync(kFull, bi, 16);
        const bool mine = (lane < 16) ? !(o1 < b1) : (b1 < o1);
        b2 = fminf(fmaxf(b1, o1), fminf(b2, o2));
        b1 = fminf(b1, o1);
        bi = mine ? bi : oi;
    }
    // near ties: the exact decision in fp64 (four trackers over the codewords
    // c = k mod 4, in increasing order, strict <; merged lowest distance,
    // then lowest index)
    const bool tie = (b2 - b1) <= fmaf(kTieRel, b1, kTieAbs);
    if (__any_sync(kFull, tie)) {  // warp-uniform
        double bd = INFINITY;
        int bdi = c0;
        if (tie) {
            double bd4[4] = {INFINITY, INFINITY, INFINITY, INFINITY};
            int bi4[4] = {c0, c0 + 1, c0 + 2, c0 + 3};
            for (int c = c0; c < c1; c += 4) {
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                    double d = 0.0;
#pragma unroll
                    for (int r = 0; r < G; ++r) {
                        const double e = w[r] - Cs[(c + k) * G + r];
                        d = fma(e, e, d);
                    }
                    if (d < bd4[k]) { bd4[k] = d; bi4[k] = c + k; }
                }
            }
            bd = bd4[0];
            bdi = bi4[0];
#pragma unroll
            for (int k = 1; k < 4; ++k)
                if (bd4[k] < bd || (bd4[k] == bd && bi4[k] < bdi)) { bd = bd4[k]; bdi = bi4[k]; }
        }
        if constexpr (G == 8) {  // both lanes of a sub-vector share its tie flag
            const double od = __shfl_xor_sync(kFull, bd, 16);
            const int oi = __shfl_xor_sync(kFull, bdi, 16);
            const bool mine = (lane < 16) ? !(od < bd) : (bd < od);
            bdi = mine ? bdi : oi;
        }
        if (tie) bi = bdi;
    }
    float s1o = (float)s1, s2o = (float)s2;
    if constexpr (ADAPT) {  // s2 * d / (w . w_hat), w . w_hat over all sub-vectors in fp64
        double q = 0.0;
        if (G == 4 || lane < 16) {
#pragma unroll
            for (int r = 0; r < G; ++r) q = fma(w[r], Cs[bi * G + r], q);
        }
        q = warp_sum_d(q);
        if (q > 0.0) s2o = (float)((double)s2o * ((double)kD / q));
    }
    const int64_t orow = cbh * a.cap + a.t_offset + t;
    if (G == 4 || lane < 16) enc_codes(a, sec)[orow * (kD / G) + j] = (uint8_t)bi;
    if (lane == 0)
        store_byproducts(enc_scales(a, sec), enc_s1_levels(a, sec), cbh, a.cap,
                         a.t_offset + t, s1o, s2o, s1lev);
}

template <typename XT, int G>
cudaError_t launch_small_t(const EncodeArgs& args, cudaStream_t s) {
    const int64_t n = (int64_t)args.B * args.H * args.T;
    const int grid = (int)((n + kSmallThreads / 32 - 1) / (kSmallThreads / 32));
    EncodeArgs a = args;
    a.div_items = make_fastdiv((uint32_t)args.T);
    a.div_H = make_fastdiv((uint32_t)args.H);
    if (a.dq) {
        if (a.adaptive) nsn_encode_small_kernel<XT, G, true, true><<<grid, kSmallThreads, 0, s>>>(a);
        else nsn_encode_small_kernel<XT, G, false, true><<<grid, kSmallThreads, 0, s>>>(a);
    } else {
        if (a.adaptive) nsn_encode_small_kernel<XT, G, true, false><<<grid, kSmallThreads, 0, s>>>(a);
        else nsn_encode_small_kernel<XT, G, false, false><<<grid, kSmallThreads, 0, s>>>(a);
    }
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_encode_small(const EncodeArgs& a, cudaStream_t s) {
    if (a.x_bf16) return a.sub == 4 ? launch_small_t<__nv_bfloat16, 4>(a, s) : launch_small_t<__nv_bfloat16, 8>(a, s);
    return a.sub == 4 ? launch_small_t<float, 4>(a, s) : launch_small_t<float, 8>(a, s);
}

}  // namespace nsnq
