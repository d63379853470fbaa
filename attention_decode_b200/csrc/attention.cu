// Decode attention over the NSNQuant-quantized KV cache on sm_100a
// (gist.science "NSNQuant ...", Technical Summary, Methodology §4: the score
// folds the NSN byproducts s1, s2, o into a kernel that reads the codes).
//
// With k_hat = s1 (s2 H w_hat + o) and H symmetric orthonormal:
//   q . k_hat = s1 * (s2 * (H q) . w_hat + q . o)
//             = s1 * (s2 * sum_j L[j][code_j] + gamma),  L[j][c] = (Hq)_j . C_c
//   sum_t p_t v_hat_t = H (sum_t p_t s1_t s2_t w_hat_t) + (sum_t p_t s1_t) o_V
// so a CTA rotates q once, builds L in shared memory, streams codes and
// accumulates values in the Hadamard domain; a combine kernel merges the
// context splits (online-softmax rescaling) and applies H once per head.
#include <math.h>

#include "common.cuh"
#include "f32x2.cuh"
#include "internal.h"
#include "attn_split.cuh"

namespace nsnq {

// Split kernel: warps of a CTA (WARPS of them) stream batches of 32 tokens.
// Per warp and batch, K and V codes arrive in shared memory by cp.async (16-byte
// copies issued one batch ahead: K into a single buffer, V into a double buffer),
// scales by register prefetch. Scores take lane = token (LUT gathers in
// lane-xor sub-vector order); values take lane = (token of 4, 16-dimension slice)
// so that a 128-byte row of value codes and the 4 tokens' weights are one
// shared-memory wavefront each.
template <int GC, int KSUB, int VSUB>
struct AttnCfg {
    static constexpr int KJ = kD / KSUB, VJ = kD / VSUB;
    static constexpr size_t lut = (size_t)kNC * KJ * GC * 4;
    static constexpr size_t vrep = (size_t)kNC * (VSUB / 4) * 8 * 16;
    static constexpr size_t qrot = (size_t)GC * kD * 4 + 32;
    static constexpr size_t kbuf = (size_t)32 * KJ;      // K codes of one batch
    static constexpr size_t vbuf = (size_t)2 * 32 * VJ;  // V codes, two batches
    static constexpr size_t wts = (size_t)32 * GC * 8;   // value weights (w, w) of one batch
    static constexpr size_t per_warp = kbuf + vbuf + wts;
    static constexpr size_t fixed = lut + vrep + qrot;
    // as many warps (<= 16) as shared memory allows
    static constexpr int warps_fit = (int)((232448 - fixed) / per_warp);
    static constexpr int WARPS = warps_fit >= 16 ? 16 : (warps_fit >= 12 ? 12 : 8);
    static constexpr size_t o_vrep = lut;
    static constexpr size_t o_qrot = o_vrep + vrep;
    static constexpr size_t o_warp = o_qrot + qrot;
    static constexpr size_t bytes = o_warp + per_warp * WARPS;
    static constexpr size_t merge = (size_t)WARPS * GC * (3 + kD) * 4;
    static_assert(merge <= lut, "merge area must fit in the LUT region");
    static_assert(bytes <= 232448, "shared memory per block");
};

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
    return (uint32_t)__cvta_generic_to_shared(p);
}
// 16-byte global -> shared copy that bypasses L1; src_bytes = 0 writes zeros.
__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src, uint32_t src_bytes) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;\n" ::"r"(dst), "l"(src), "r"(src_bytes)
                 : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;\n" ::: "memory"); }
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_group 0;\n" ::: "memory"); }

template <typename QT>
__device__ __forceinline__ void load_q4(const void* q, int64_t off, float (&v)[4]) {
    load4(reinterpret_cast<const QT*>(q) + off, v);
}



template <int GC, int KSUB, int VSUB, typename QT>
__global__ void __launch_bounds__(AttnCfg<GC, KSUB, VSUB>::WARPS * 32, 1) attn_split_kernel(AttnArgs a) {
    using S = AttnCfg<GC, KSUB, VSUB>;
    constexpr int WARPS = S::WARPS, THREADS = WARPS * 32;
    constexpr int KJ = S::KJ, VJ = S::VJ;
    constexpr int KW = KJ / 4;          // 32-bit words per K code row
    constexpr int SPL = 16 / VSUB;      // value sub-vectors per lane (16 dimensions)
    extern __shared__ __align__(16) uint8_t smb[];
    float* lut = reinterpret_cast<float*>(smb);
    float4* vrep = reinterpret_cast<float4*>(smb + S::o_vrep);
    float* qrot = reinterpret_cast<float*>(smb + S::o_qrot);
    float* gam = qrot + GC * kD;

    const int tid = threadIdx.x, lane = lane_id(), warp = tid >> 5;
    const int G = a.Hq / a.Hkv;
    const int cta = blockIdx.x;
    const int64_t L = a.plan.L;
    const int nslot = a.plan.nslot;
    const int64_t vbeg = cta_begin(cta, a.plan), vend = cta_begin(cta + 1, a.plan);

    uint8_t* warp_area = smb + S::o_warp + (size_t)warp * S::per_warp;
    uint8_t* kbuf = warp_area;                       // [32][KJ], 16-byte halves swizzled
    uint8_t* vbuf = warp_area + S::kbuf;             // [2][32][VJ]
    uint64_t* wts = reinterpret_cast<uint64_t*>(warp_area + S::kbuf + S::vbuf);  // [32][GC] (w, w)

    for (int i = tid; i < kNC * (VSUB / 4) * 8; i += THREADS)  // [piece][copy]
        vrep[i] = reinterpret_cast<const float4*>(a.vC)[i >> 3];

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
    __syncthreads();  // the previous segment is done with the LUT, qrot and merge area

    if (ts >= te) {  // nothing to attend in this segment: neutral partial
        for (int idx = tid; idx < GC * kPartStride; idx += THREADS) {
            const int h = idx / kPartStride, c = idx % kPartStride;
            float* P = a.part + (((int64_t)b * a.Hq + qh0 + h) * nslot + slot) * kPartStride;
            P[c] = (c == kD) ? -INFINITY : 0.f;
        }
        continue;
    }

    const uint8_t* kc = a.kcodes + bkv * a.kcap * KJ;
    const uint8_t* vc = a.vcodes + bkv * a.vcap * VJ;
    const float lvlK = packed_level_lane(a.klevels, a.kgrid, bkv);
    const float lvlV = packed_level_lane(a.vlevels, a.vgrid, bkv);
    const ByproductSrc ksrc = byproduct_src(a.kscales, a.klevels, bkv, a.kcap);
    const ByproductSrc vsrc = byproduct_src(a.vscales, a.vlevels, bkv, a.vcap);
    // Token indices of the loop are 32-bit: lengths are int32, and a batch
    // start stays below te + 32 * WARPS < 2^32.
    const uint32_t ts32 = (uint32_t)ts, te32 = (uint32_t)te;

    // Copies of one batch's codes (lane = token): K row with its 16-byte
    // halves swapped for lanes 4-7 of each group of 8 (conflict-free reads
    // of whole rows), V row into the batch's buffer.
    const uint32_t kb_s = smem_u32(kbuf), vb_s = smem_u32(vbuf);
    const uint32_t kdst = kb_s + lane * KJ, vdst = vb_s + lane * VJ;
    auto issue_codes = [&](uint32_t base, int parity) {
        const uint32_t t = base + lane;
        const bool ok = t < te32;
        const uint32_t tc = ok ? t : ts32;  // any valid row (nothing is read when !ok)
        const uint32_t nb = ok ? 16u : 0u;
        const uint8_t* ks = kc + (size_t)tc * KJ;
        const uint8_t* vs = vc + (size_t)tc * VJ;
#pragma unroll
        for (int p = 0; p < KJ / 16; ++p) {
            const int ps = (KJ == 32) ? (p ^ ((lane >> 2) & 1)) : p;
            cp_async16(kdst + ps * 16, ks + p * 16, nb);
        }
#pragma unroll
        for (int p = 0; p < VJ / 16; ++p) cp_async16(vdst + parity * 32 * VJ + p * 16, vs + p * 16, nb);
        cp_async_commit();
    };

    // ---- segment prologue: rotated queries, q . o_K, LUT ----
    if (warp < GC) {
        float qv[4];
        load_q4<QT>(a.q, ((int64_t)b * a.Hq + qh0 + warp) * kD + 4 * lane, qv);
        const float4 o = reinterpret_cast<const float4*>(a.kshift + bkv * kD)[lane];
        const float g = warp_sum(fmaf(qv[3], o.w, fmaf(qv[2], o.z, fmaf(qv[1], o.y, qv[0] * o.x))));
        fwht128_lane4(qv);
#pragma unroll
        for (int r = 0; r < 4; ++r) qrot[warp * kD + 4 * lane + r] = qv[r] * kRsqrtD;
        if (lane == 0) gam[warp] = g;
    }
    __syncthreads();
    {
        // A thread keeps sub-vector j of the rotated queries in registers and
        // walks the codes c = tid / KJ + k * (threads / KJ): the codeword is
        // one broadcast read per warp and each warp stores whole LUT rows.
        static_assert(THREADS % KJ == 0, "threads must tile the sub-vectors");
        // The softmax scale (log2 domain) is folded into the table and gamma.
        const int j = tid % KJ;
        float qj[GC][KSUB];
#pragma unroll
        for (int h = 0; h < GC; ++h)
#pragma unroll
            for (int r = 0; r < KSUB; ++r) qj[h][r] = qrot[h * kD + j * KSUB + r] * a.scale_log2;
#pragma unroll 4
        for (int c = tid / KJ; c < kNC; c += THREADS / KJ) {
            float ck[KSUB];
#pragma unroll
            for (int k = 0; k < KSUB / 4; ++k) {
                const float4 c4 = __ldg(reinterpret_cast<const float4*>(a.kC) + c * (KSUB / 4) + k);
                ck[4 * k] = c4.x; ck[4 * k + 1] = c4.y; ck[4 * k + 2] = c4.z; ck[4 * k + 3] = c4.w;
            }
            float sum[GC];
#pragma unroll
            for (int h = 0; h < GC; ++h) {
                sum[h] = 0.f;
#pragma unroll
                for (int r = 0; r < KSUB; ++r) sum[h] = fmaf(qj[h][r], ck[r], sum[h]);
            }
            const int e = c * KJ + j;
            if constexpr (GC == 4) {
                reinterpret_cast<float4*>(lut)[e] = make_float4(sum[0], sum[1], sum[2], sum[3]);
            } else {
#pragma unroll
                for (int h = 0; h < GC; ++h) lut[(size_t)e * GC + h] = sum[h];
            }
        }
    }
    __syncthreads();
    // Launched as a programmatic dependent (of the encode that appended to
    // the caches, in a decode step): the prologue above reads only q, o_K and
    // the codebook, so it overlaps that kernel; codes and scales are read
    // after this wait.
    asm volatile("griddepcontrol.wait;\n" ::: "memory");
    const uint32_t first = ts32 + warp * 32;
    if (first < te32) issue_codes(first, 0);
    RawByproducts k2n{0.f, 0u}, v2n{0.f, 0u};  // next batch's byproducts, still raw
    if (first < te32) {  // warp-uniform
        k2n = fetch_byproducts(ksrc, first + lane, first + lane < te32);
        v2n = fetch_byproducts(vsrc, first + lane, first + lane < te32);
    }

    float gm[GC];
#pragma unroll
    for (int h = 0; h < GC; ++h) gm[h] = gam[h] * a.scale_log2;
    float m[GC], l[GC], be[GC];
    uint64_t acc[GC][8];  // dims 16 sl + (2r, 2r + 1)
#pragma unroll
    for (int h = 0; h < GC; ++h) {
        m[h] = -INFINITY; l[h] = 0.f; be[h] = 0.f;
#pragma unroll
        for (int r = 0; r < 8; ++r) acc[h][r] = 0ull;
    }
    const int t7 = lane & 7;
    const int grp = lane >> 3, sl = lane & 7;  // value phase: token of 4, dimension slice
    // codeword (c0, c1, c2, c3) read as two packed pairs (c0, c1), (c2, c3)
    const ulonglong2* myrep = reinterpret_cast<const ulonglong2*>(vrep) + sl;
    int parity = 0;
    // Score gathers visit sub-vector j = s ^ t7 at step s: its code is byte
    // (s ^ t7) & 3 of word (s ^ t7) >> 2 of the row. With the row's words
    // swapped in pairs for t7 >= 4 (kwp), the word index is s >> 2 for every
    // lane and the byte selector is (s & 3) ^ (t7 & 3).
    const uint32_t t3 = (uint32_t)(t7 & 3);

    for (uint32_t base = first; base < te32; base += WARPS * 32) {
        const uint32_t t = base + lane;
        const bool valid = t < te32;
        const RawByproducts k2r = k2n, v2r = v2n;  // resolved where first needed (softmax)
        const uint32_t nbase = base + WARPS * 32;
        cp_async_wait_all();
        __syncwarp();
        // ---- this lane's K code row (from the swizzled buffer) ----
        uint32_t kw[KW];
        {
            const uint4* kr = reinterpret_cast<const uint4*>(kbuf + lane * KJ);
#pragma unroll
            for (int p = 0; p < KJ / 16; ++p) {
                const int ps = (KJ == 32) ? (p ^ ((lane >> 2) & 1)) : p;
                const uint4 w4 = kr[ps];
                kw[4 * p] = w4.x; kw[4 * p + 1] = w4.y; kw[4 * p + 2] = w4.z; kw[4 * p + 3] = w4.w;
            }
        }
        __syncwarp();  // every lane has its K row: the buffer takes the next batch
        if (nbase < te32) {  // warp-uniform
            issue_codes(nbase, parity ^ 1);
            k2n = fetch_byproducts(ksrc, nbase + lane, nbase + lane < te32);
            v2n = fetch_byproducts(vsrc, nbase + lane, nbase + lane < te32);
        }
        // ---- scores: lane = token; sub-vector order s ^ (lane & 7) keeps the
        //      eight lanes of a quarter-warp on eight different bank groups
        uint32_t kwp[KW];
#pragma unroll
        for (int i = 0; i < KW; ++i) kwp[i] = (t7 & 4) ? kw[i ^ 1] : kw[i];
        float sc[GC];
        if constexpr (GC == 4) {
            uint64_t s01 = 0ull, s23 = 0ull;
            // a table row is read as two packed pairs: heads (0, 1) and (2, 3)
            const ulonglong2* lut2 = reinterpret_cast<const ulonglong2*>(lut);
#pragma unroll
            for (int s = 0; s < KJ; ++s) {
                const uint32_t code = __byte_perm(kwp[s >> 2], 0u, (0x4440u | (uint32_t)(s & 3)) ^ t3);
                const ulonglong2 e = lut2[(int)code * KJ + (s ^ t7)];
                s01 = add2(s01, e.x);
                s23 = add2(s23, e.y);
            }
            const float2 a01 = upk2(s01), a23 = upk2(s23);
            sc[0] = a01.x; sc[1] = a01.y; sc[2] = a23.x; sc[3] = a23.y;
        } else {
#pragma unroll
            for (int h = 0; h < GC; ++h) sc[h] = 0.f;
#pragma unroll
            for (int s = 0; s < KJ; ++s) {
                const uint32_t code = __byte_perm(kwp[s >> 2], 0u, (0x4440u | (uint32_t)(s & 3)) ^ t3);
                const float* e = lut + ((int)code * KJ + (s ^ t7)) * GC;
#pragma unroll
                for (int h = 0; h < GC; ++h) sc[h] += e[h];
            }
        }
        // ---- online softmax (log2 domain). The running max m is raised only
        //      when a logit exceeds it by more than kLazy (a warp vote); then
        //      the accumulators are rescaled. Weights stay below 2^kLazy.
        const float2 k2 = resolve_byproducts(k2r, ksrc, t, lvlK);
        const float2 v2 = resolve_byproducts(v2r, vsrc, t, lvlV);
        const float vw = v2.x * v2.y;
        float logit[GC];
        bool raise = false;
#pragma unroll
        for (int h = 0; h < GC; ++h) {
            logit[h] = valid ? k2.x * fmaf(k2.y, sc[h], gm[h]) : -INFINITY;
            raise |= logit[h] > m[h] + kLazy;
        }
        if (__any_sync(kFull, raise)) {  // warp-uniform, rare: one vote for all heads
#pragma unroll
            for (int h = 0; h < GC; ++h) {
                if (__any_sync(kFull, logit[h] > m[h] + kLazy)) {
                    const float mx = warp_max(logit[h]);
                    const float alpha = (m[h] == -INFINITY) ? 0.f : exp2_approx(m[h] - mx);
                    l[h] *= alpha;
                    be[h] *= alpha;
                    const uint64_t al = pk2(alpha, alpha);
#pragma unroll
                    for (int r = 0; r < 8; ++r) acc[h][r] = mul2(acc[h][r], al);
                    m[h] = mx;
                }
            }
        }
        // Every batch holds a valid token, so m is finite here and an invalid
        // lane's logit of -inf gives p = 0.
        uint64_t wpair[GC];
#pragma unroll
        for (int h = 0; h < GC; ++h) {
            const float p = exp2_approx(logit[h] - m[h]);
            l[h] += p;
            be[h] = fmaf(p, v2.x, be[h]);
            const float w = p * vw;
            wpair[h] = pk2(w, w);
        }
        if constexpr (GC % 2 == 0) {
#pragma unroll
            for (int h2 = 0; h2 < GC / 2; ++h2)
                reinterpret_cast<ulonglong2*>(wts + lane * GC)[h2] = make_ulonglong2(wpair[2 * h2], wpair[2 * h2 + 1]);
        } else {
            wts[lane] = wpair[0];
        }
        __syncwarp();
        // ---- values: lane = (token 4i + grp, dimensions 16 sl .. 16 sl + 15) ----
        const uint8_t* vb = vbuf + (size_t)parity * 32 * VJ;
        uint32_t cws[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const int tt = 4 * i + grp;
            if constexpr (VSUB == 4) cws[i] = *reinterpret_cast<const uint32_t*>(vb + tt * VJ + 4 * sl);
            else cws[i] = *reinterpret_cast<const uint16_t*>(vb + tt * VJ + 2 * sl);
        }
        auto vstep = [&](int tt, uint32_t cw) {
            uint64_t wp[GC];
            if constexpr (GC % 2 == 0) {
#pragma unroll
                for (int h2 = 0; h2 < GC / 2; ++h2) {
                    const ulonglong2 w2 = reinterpret_cast<const ulonglong2*>(wts + tt * GC)[h2];
                    wp[2 * h2] = w2.x; wp[2 * h2 + 1] = w2.y;
                }
            } else {
                wp[0] = wts[tt];
            }
#pragma unroll
            for (int s = 0; s < SPL; ++s) {
                const uint32_t code = (cw >> (8 * s)) & 0xffu;
#pragma unroll
                for (int k = 0; k < VSUB / 4; ++k) {
                    const ulonglong2 cv = myrep[(code * (VSUB / 4) + k) * 8];
                    const int r0 = (s * VSUB + 4 * k) / 2;  // packed pair index of dims 4k, 4k+1
                    const uint64_t c01 = cv.x, c23 = cv.y;
#pragma unroll
                    for (int h = 0; h < GC; ++h) {
                        acc[h][r0] = fma2(c01, wp[h], acc[h][r0]);
                        acc[h][r0 + 1] = fma2(c23, wp[h], acc[h][r0 + 1]);
                    }
                }
            }
        };
        // Tokens past the end of a partial batch carry weight 0 and zero-filled
        // codes, so every batch runs the same eight steps.
#pragma unroll
        for (int i = 0; i < 8; ++i) vstep(4 * i + grp, cws[i]);
        __syncwarp();
        parity ^= 1;
    }

    // ---- warp totals: l, beta over lanes; A over the four token groups ----
#pragma unroll
    for (int h = 0; h < GC; ++h) {
        l[h] = warp_sum(l[h]);
        be[h] = warp_sum(be[h]);
#pragma unroll
        for (int r = 0; r < 8; ++r) {
            float2 v = upk2(acc[h][r]);
            v.x += __shfl_xor_sync(kFull, v.x, 8);
            v.y += __shfl_xor_sync(kFull, v.y, 8);
            v.x += __shfl_xor_sync(kFull, v.x, 16);
            v.y += __shfl_xor_sync(kFull, v.y, 16);
            acc[h][r] = pk2(v.x, v.y);
        }
    }
    __syncthreads();  // LUT no longer needed: reuse it for the CTA merge
    float* mw = lut;
    float* lw = mw + WARPS * GC;
    float* bw = lw + WARPS * GC;
    float* Aw = bw + WARPS * GC;  // [warp][h][128]
    if (lane == 0) {
#pragma unroll
        for (int h = 0; h < GC; ++h) {
            mw[warp * GC + h] = m[h]; lw[warp * GC + h] = l[h]; bw[warp * GC + h] = be[h];
        }
    }
    if (grp == 0) {
#pragma unroll
        for (int h = 0; h < GC; ++h)
#pragma unroll
            for (int r = 0; r < 8; ++r)
                reinterpret_cast<float2*>(Aw + (warp * GC + h) * kD + 16 * sl)[r] = upk2(acc[h][r]);
    }
    __syncthreads();
    for (int idx = tid; idx < GC * (kD + 2); idx += THREADS) {
        const int h = idx / (kD + 2), c = idx % (kD + 2);
        float M = -INFINITY;
#pragma unroll
        for (int w = 0; w < WARPS; ++w) M = fmaxf(M, mw[w * GC + h]);
        float accm = 0.f;
#pragma unroll
        for (int w = 0; w < WARPS; ++w) {
            const float mv = mw[w * GC + h];
            const float f = (mv == -INFINITY) ? 0.f : exp2f(mv - M);
            float v;
            if (c < kD) v = Aw[(w * GC + h) * kD + c];
            else if (c == kD) v = lw[w * GC + h];
            else v = bw[w * GC + h];
            accm = fmaf(f, v, accm);
        }
        float* P = a.part + (((int64_t)b * a.Hq + qh0 + h) * nslot + slot) * kPartStride;
        if (c < kD) P[c] = accm;
        else if (c == kD) { P[kD] = M; P[kD + 1] = accm; }
        else P[kD + 2] = accm;  // c == kD + 1: beta
    }
  }
}

// Residual tokens scored per combine pass (one score per token in shared memory).
constexpr int kResChunk = 256;

// Merge the splits of one (batch, query head): rescale by exp2(m_s - M),
// apply H to the rotated-domain sum, add beta * o_V, divide by l. Tokens of
// the full-precision residual window join the same softmax here: their
// scores q . k * scale are taken in fp32 chunk by chunk (an online max over
// the chunks), their values accumulate in the original domain.
template <typename RT>
__device__ __forceinline__ void combine_residual(const AttnArgs& a, int b, int qh, int kvh,
                                                 int64_t rlen, float& M, float& acc, float& L,
                                                 float& Be, float& racc, float* qs, float* ps) {
    const int c = threadIdx.x, lane = lane_id(), warp = c >> 5;
    const int64_t qoff = ((int64_t)b * a.Hq + qh) * kD + c;
    qs[c] = a.q_bf16 ? __bfloat162float(reinterpret_cast<const __nv_bfloat16*>(a.q)[qoff])
                     : reinterpret_cast<const float*>(a.q)[qoff];
    __syncthreads();
    float q4[4];
#pragma unroll
    for (int r = 0; r < 4; ++r) q4[r] = qs[4 * lane + r];
    const int64_t base = ((int64_t)b * a.Hkv + kvh) * a.rcap;
    const RT* K = reinterpret_cast<const RT*>(a.rk) + base * kD;
    const RT* V = reinterpret_cast<const RT*>(a.rv) + base * kD;
    for (int64_t t0 = 0; t0 < rlen; t0 += kResChunk) {
        const int n = (int)(rlen - t0 < kResChunk ? rlen - t0 : kResChunk);
        for (int i = warp; i < n; i += kD / 32) {
            float k4[4];
            load4(K + (t0 + i) * kD + 4 * lane, k4);
            float d = fmaf(q4[3], k4[3], fmaf(q4[2], k4[2], fmaf(q4[1], k4[1], q4[0] * k4[0])));
            d = warp_sum(d);
            if (lane == 0) ps[i] = d * a.scale_log2;
        }
        __syncthreads();
        float mc = -INFINITY;
        for (int i = 0; i < n; ++i) mc = fmaxf(mc, ps[i]);
        const float Mn = fmaxf(M, mc);
        const float f = M == -INFINITY ? 0.f : exp2f(M - Mn);
        acc *= f; L *= f; Be *= f; racc *= f;
        M = Mn;
        __syncthreads();  // every thread has read the scores
        for (int i = c; i < n; i += kD) ps[i] = exp2f(ps[i] - M);
        __syncthreads();
        for (int i = 0; i < n; ++i) {
            const float p = ps[i];
            L += p;
            const RT vv = V[(t0 + i) * kD + c];
            racc = fmaf(p, (float)vv, racc);
        }
        __syncthreads();  // before the next chunk overwrites ps
    }
}

__global__ void __launch_bounds__(kD) attn_combine_kernel(AttnArgs a) {
    __shared__ float As[kD];
    __shared__ float Rs[kD];
    __shared__ float qs[kD];
    __shared__ float ps[kResChunk];
    __shared__ float LB[2];
    const int bq = blockIdx.x;
    const int b = bq / a.Hq, qh = bq % a.Hq;
    const int G = a.Hq / a.Hkv;
    const int kvh = qh / G, hg = (qh % G) / a.plan.gc;
    const int64_t u = ((int64_t)b * a.Hkv + kvh) * a.plan.ngroups + hg;
    const int nslot = a.plan.nslot;
    const int used = a.plan.L > 0
                         ? first_cta(u * a.plan.L + a.plan.L - 1, a.plan) - first_cta(u * a.plan.L, a.plan) + 1
                         : 0;
    const float* P = a.part + (int64_t)bq * nslot * kPartStride;
    const int c = threadIdx.x;
    float M = -INFINITY;
    for (int s = 0; s < used; ++s) M = fmaxf(M, P[(int64_t)s * kPartStride + kD]);
    float acc = 0.f, L = 0.f, Be = 0.f, racc = 0.f;
    if (M != -INFINITY) {
        for (int s = 0; s < used; ++s) {
            const float* Ps = P + (int64_t)s * kPartStride;
            const float ms = Ps[kD];
            const float f = (ms == -INFINITY) ? 0.f : exp2f(ms - M);
            acc = fmaf(f, Ps[c], acc);
            L = fmaf(f, Ps[kD + 1], L);
            Be = fmaf(f, Ps[kD + 2], Be);
        }
    }
    int64_t rlen = a.rcap > 0 ? (int64_t)a.res_lens[b] : 0;
    rlen = rlen < 0 ? 0 : (rlen > a.rcap ? a.rcap : rlen);
    if (rlen > 0) {  // block-uniform
        if (a.r_bf16)
            combine_residual<__nv_bfloat16>(a, b, qh, kvh, rlen, M, acc, L, Be, racc, qs, ps);
        else
            combine_residual<float>(a, b, qh, kvh, rlen, M, acc, L, Be, racc, qs, ps);
    }
    As[c] = acc;
    Rs[c] = racc;
    if (c == 0) { LB[0] = L; LB[1] = Be; }
    __syncthreads();
    if (threadIdx.x >= 32) return;
    const int lane = lane_id();
    float v[4];
#pragma unroll
    for (int r = 0; r < 4; ++r) v[r] = As[4 * lane + r];
    fwht128_lane4(v);
    const float Lt = LB[0], Bt = LB[1];
    const float inv = Lt > 0.f ? 1.0f / Lt : 0.f;
    const float4 o = reinterpret_cast<const float4*>(a.vshift + ((int64_t)b * a.Hkv + kvh) * kD)[lane];
    const float4 rr = reinterpret_cast<const float4*>(Rs)[lane];
    float r4[4];
    r4[0] = (fmaf(Bt, o.x, v[0] * kRsqrtD) + rr.x) * inv;
    r4[1] = (fmaf(Bt, o.y, v[1] * kRsqrtD) + rr.y) * inv;
    r4[2] = (fmaf(Bt, o.z, v[2] * kRsqrtD) + rr.z) * inv;
    r4[3] = (fmaf(Bt, o.w, v[3] * kRsqrtD) + rr.w) * inv;
    if (a.out_bf16) {
        uint2 pk;
        pk.x = (uint32_t)f32_to_bf16_rn(r4[0]) | ((uint32_t)f32_to_bf16_rn(r4[1]) << 16);
        pk.y = (uint32_t)f32_to_bf16_rn(r4[2]) | ((uint32_t)f32_to_bf16_rn(r4[3]) << 16);
        reinterpret_cast<uint2*>(reinterpret_cast<uint16_t*>(a.out) + (int64_t)bq * kD)[lane] = pk;
    } else {
        reinterpret_cast<float4*>(reinterpret_cast<float*>(a.out) + (int64_t)bq * kD)[lane] =
            make_float4(r4[0], r4[1], r4[2], r4[3]);
    }
}

// ---------------------------------------------------------------- host --
// A CTA pays a fixed cost per segment it attends to (rotated queries, table
// build, the CTA merge), counted here in streamed tokens.
constexpr int64_t kSegmentFixedTokens = 1000;

AttnPlan plan_attention(int B, int Hq, int Hkv, int64_t max_len) {
    AttnPlan p{};
    const int G = Hq / Hkv;
    p.gc = (G % 4 == 0) ? 4 : (G % 2 == 0 ? 2 : 1);
    p.ngroups = G / p.gc;
    p.units = (int64_t)B * Hkv * p.ngroups;
    p.L = max_len;
    const int sms = device_sm_count();  // one CTA per SM (the tables fill shared memory)
    p.ctas = sms;
    // Two ways to cut the (unit, token) space: the balanced split gives every
    // CTA the same number of tokens, but a CTA whose share crosses a unit
    // boundary attends to two segments; the unit-aligned split gives each unit
    // nsplit CTAs of one segment each (padding each unit to nsplit equal parts,
    // a multiple of 32 tokens), at the price of idle SMs when units * nsplit <
    // SMs. The cheaper one by the fixed-cost model is taken.
    if (p.units > 0 && p.units <= sms && max_len > 0) {
        const int64_t nsplit = sms / p.units;
        const int64_t seg = (max_len + nsplit - 1) / nsplit;
        const int64_t seg32 = (seg + 31) / 32 * 32;
        const int64_t per_cta = (p.units * max_len + sms - 1) / sms;
        const int64_t balanced = per_cta + (per_cta < max_len ? 2 : 1) * kSegmentFixedTokens;
        const int64_t aligned = seg32 + kSegmentFixedTokens;
        if (aligned < balanced) {
            p.L = nsplit * seg32;
            p.ctas = (int)(p.units * nsplit);
        }
    }
    p.nslot = (int)((p.ctas + p.units - 1) / (p.units > 0 ? p.units : 1)) + 1;
    p.total = align_up((size_t)B * Hq * p.nslot * kPartStride * sizeof(float), kWsAlign);
    return p;
}

template <int GC, int KSUB, int VSUB, typename QT>
static cudaError_t launch_split(const AttnArgs& a, cudaStream_t s) {
    using S = AttnCfg<GC, KSUB, VSUB>;
    static std::atomic<unsigned long long> ready{0};
    return launch_smem_pdl(attn_split_kernel<GC, KSUB, VSUB, QT>, ready, dim3(a.plan.ctas),
                           dim3(S::WARPS * 32), S::bytes, s, a);
}

template <int GC, typename QT>
static cudaError_t launch_split_sub(const AttnArgs& a, cudaStream_t s) {
    if (a.ksub == 4 && a.vsub == 4) return launch_split<GC, 4, 4, QT>(a, s);
    if (a.ksub == 4 && a.vsub == 8) return launch_split<GC, 4, 8, QT>(a, s);
    if (a.ksub == 8 && a.vsub == 4) return launch_split<GC, 8, 4, QT>(a, s);
    return launch_split<GC, 8, 8, QT>(a, s);
}

template <typename QT>
static cudaError_t launch_split_gc(const AttnArgs& a, cudaStream_t s) {
    if (a.plan.gc == 4) return launch_split_sub<4, QT>(a, s);
    if (a.plan.gc == 2) return launch_split_sub<2, QT>(a, s);
    return launch_split_sub<1, QT>(a, s);
}

cudaError_t launch_attn_combine(const AttnArgs& a, cudaStream_t s) {
    attn_combine_kernel<<<a.B * a.Hq, kD, 0, s>>>(a);
    return cudaGetLastError();
}

cudaError_t launch_attention(const AttnArgs& a, cudaStream_t s) {
    cudaError_t e = a.q_bf16 ? launch_split_gc<__nv_bfloat16>(a, s) : launch_split_gc<float>(a, s);
    if (e != cudaSuccess) return e;
    attn_combine_kernel<<<a.B * a.Hq, kD, 0, s>>>(a);
    return cudaGetLastError();
}

}  // namespace nsnq
