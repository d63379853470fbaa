// Pass 2 of the encode with every codeword scored on the 5th-generation
// tensor cores (gist.science "NSNQuant ...", Technical Summary, Methodology
// §1-§3): the 1-bit encode (8-dimensional sub-vectors), and the 2-bit encode
// when the caller asks for the tensor-core search (4-dimensional
// sub-vectors, no search index; slower than the index walk of
// encode_pruned.cu, kept as the index-free path and for comparison).
//
// Every codeword is scored, so the scoring is a dense contraction: for a
// tile of 128 sub-vectors and the 256 codewords, s[m][n] = |C_n|^2 - 2 w_m .
// C_n, and the nearest codeword has the least s (d = |w|^2 + s). The CTA
// computes w by NSN and the Hadamard transform (two token-heads per warp,
// 8 coordinates per lane: one 8-dimensional sub-vector, or two 4-dimensional
// ones taken in two rounds), writes it as the A operand (a 4-dimensional
// sub-vector padded with zeros to K = 8), and one thread issues tcgen05.mma
// (kind::tf32, M 128, N 128, K 8) into a 128-column TMEM accumulator, once
// for each half of the codebook:
//   D  = A_hi B_hi + A_lo B_hi + A_hi B_lo + 1 (|C|^2_hi + |C|^2_lo)
// with x_hi = tf32(x), x_lo = tf32(x - x_hi) (three-term split, about fp32
// accuracy) and B = -2C. Each thread then reads its own row of D (its own
// sub-vector, TMEM lane = row) with tcgen05.ld and finds the best and
// second-best score by groups of 8. Near ties (gap within the near-tie band,
// at least the derived scoring-error bound kScoreErrTc) and tokens with a
// cancelling shift are re-decided in fp64 by the whole warp.
//
// Shared-memory operands use the no-swizzle K-major layout: a row's 8 tf32
// values are two 16-byte pieces, piece p of row r at p * LBO + r * 16
// (8-row groups 128 bytes apart).
#include <math.h>

#include "common.cuh"
#include "dq.cuh"
#include "internal.h"

namespace nsnq {

namespace {

constexpr int kTcThreads = 128;  // 4 warps = the 128 TMEM lanes
constexpr int kRows = 128;       // sub-vectors per tile (8 token-heads)
constexpr int kCols = 128;       // TMEM accumulator columns (one per codeword of a half)
constexpr float kTieRelTc = 1e-4f;
constexpr float kTieAbsTc = 1e-6f;
// Bound on the scoring error of one score s = |C|^2 - 2 w . C, relative to
// |C|^2 + 2 |w| |C| (the sum of the absolute values of its terms):
//  - each tf32 x tf32 product is exact in fp32 (11 + 11 significant bits);
//  - dropping A_lo B_lo and the residuals of the two-term splits of w and
//    -2C leaves at most 3.001 * 2^-22 of each |w_k| |2 C_k| term;
//  - |C|^2 is an fp32 chain of at most 8 fused multiply-adds (8 * 2^-24
//    relative) split into two tf32 parts (2^-22 left over);
//  - the tensor core adds at most 26 terms (3 split MMAs of K = 8 plus the
//    two |C|^2 parts; zero padding adds exact zeros); with every addition
//    rounding or truncating to fp32 (relative error <= 2^-23) the sum is off
//    by at most 25 * 2^-23 of the terms' absolute sum.
// Together: |s_computed - s| <= 3.71e-6 (|C|^2 + 2 |w| |C|). The near-tie band
// of a sub-vector is at least the sum of this bound for its best codeword and
// for the largest codeword (the second best is not tracked by index).
constexpr float kScoreErrTc = 3.71e-6f;
constexpr float kCancelTc = 1e-3f;
constexpr long long kWaitLimit = 1ll << 24;  // spins on the MMA barrier before giving up

// shared-memory map (bytes, from a 1024-aligned base)
constexpr uint32_t kOffAhi = 0;        // [2 pieces][128 rows][16 B]
constexpr uint32_t kOffAlo = 4096;
constexpr uint32_t kOffAone = 8192;
constexpr uint32_t kOffBhi = 12288;    // [2 pieces][256 rows][16 B]
constexpr uint32_t kOffBlo = 20480;
constexpr uint32_t kOffBn2 = 28672;
constexpr uint32_t kOffC = 36864;      // fp32 codebook [256][SUB] (fp64 path)
constexpr uint32_t kOffN2 = 45056;     // fp32 |C|^2 [256]
constexpr uint32_t kOffBar = 46080;    // mbarrier (8 B) + TMEM address (4 B)
// Dynamic shared memory per CTA: above 46 KB so that at most four CTAs share
// an SM, which keeps every CTA's 128 TMEM columns available (512 per SM).
constexpr uint32_t kTcSmem = 50 * 1024;

__device__ __forceinline__ uint32_t smem_addr(const void* p) {
    return (uint32_t)__cvta_generic_to_shared(p);
}
__device__ __forceinline__ uint32_t to_tf32(float x) {
    uint32_t r;
    asm("cvt.rna.tf32.f32 %0, %1;" : "=r"(r) : "f"(x));
    return r;
}
// Shared-memory matrix descriptor: no swizzle, K-major, version 1.
__device__ __forceinline__ uint64_t mat_desc(uint32_t addr, uint32_t lbo, uint32_t sbo) {
    return (uint64_t)((addr >> 4) & 0x3fffu) | ((uint64_t)((lbo >> 4) & 0x3fffu) << 16) |
           ((uint64_t)((sbo >> 4) & 0x3fffu) << 32) | (1ull << 46);
}
// Instruction descriptor: D f32, A and B tf32, both K-major, N = 128, M = 128.
constexpr uint32_t kIdesc = (1u << 4) | (2u << 7) | (2u << 10) | ((uint32_t)(kCols >> 3) << 17) |
                            ((uint32_t)(kRows >> 4) << 24);

__device__ __forceinline__ void mma_tf32(uint32_t d, uint64_t a, uint64_t b, uint32_t acc) {
    asm volatile(
        "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::tf32 [%0], %1, %2, %3, {%5, %6, %7, %8}, p;\n\t}\n" ::"r"(d),
        "l"(a), "l"(b), "r"(kIdesc), "r"(acc), "r"(0), "r"(0), "r"(0), "r"(0));
}
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&r)[32]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, "
        "%12, %13, %14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, "
        "%30, %31}, [%32];\n"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
          "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
          "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]),
          "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]),
          "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
        : "r"(taddr));
    asm volatile("tcgen05.wait::ld.sync.aligned;\n" ::: "memory");
}
__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\tmbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}\n"
        : "=r"(ok)
        : "r"(bar), "r"(parity)
        : "memory");
    return ok != 0;
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

__device__ __forceinline__ float half_sum(float v) {
#pragma unroll
    for (int m = 1; m < 16; m <<= 1) v += __shfl_xor_sync(kFull, v, m);
    return v;
}

// Exact decision for one token-head by the whole warp (see the fp64 path of
// the 2-bit encode): fp64 NSN and Hadamard transform, lane l holding
// coordinates 4l..4l+3; each flagged sub-vector j (lanes (SUB/4) j ..) is
// scored against all 256 codewords in fp64, split over the lanes, with a
// warp argmin (lowest index on exact ties). cw: byte j = code of sub-vector j.
template <typename XT, int SUB>
__device__ __noinline__ void exact_warp_tc(const XT* xtok, const double* o64, const float* o32,
                                           const float* C, uint32_t flags, uint32_t* cw,
                                           double s1_fixed, double& s1_out, double& s2_out,
                                           double& wq_out) {
    constexpr int LPS = SUB / 4;  // lanes per sub-vector
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
    const double s1 = s1_fixed >= 0.0 ? s1_fixed : sqrt(ss) / sqrt_d;  // fixed: quantized s1
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
    uint32_t todo = flags;
    while (todo) {  // warp-uniform
        const int j = __ffs(todo) - 1;
        todo &= todo - 1;
        double f[SUB];
#pragma unroll
        for (int r = 0; r < SUB; ++r) f[r] = __shfl_sync(kFull, z[r & 3], LPS * j + (r >> 2));
        double bd = INFINITY;
        int bi = 0;
#pragma unroll 2
        for (int k = 0; k < kNC / 32; ++k) {
            const int c = lane + 32 * k;
            double d = 0.0;
#pragma unroll
            for (int r = 0; r < SUB; ++r) {
                const double e = f[r] - (double)C[c * SUB + r];
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
    const int j = lane / LPS;
    const int code = (int)((cw[j >> 2] >> (8 * (j & 3))) & 0xffu);
    double q = 0.0;
#pragma unroll
    for (int r = 0; r < 4; ++r) q = fma(z[r], (double)C[code * SUB + 4 * (lane % LPS) + r], q);
    wq_out = warp_sum_d(q);
    s1_out = s1;
    s2_out = s2;
}

// SUB = 8: one sub-vector per lane (1 bit/coordinate); SUB = 4: two per
// lane, scored in two rounds (2 bits/coordinate, the tensor-core search).
template <typename XT, bool ADAPT, bool DQ, int SUB>
__global__ void __launch_bounds__(kTcThreads) nsn_encode_tc_kernel(EncodeArgs a) {
    constexpr int RPL = 8 / SUB;        // rounds (sub-vectors) per lane
    constexpr int NW = 32 / SUB;        // 32-bit code words per token-head
    extern __shared__ __align__(1024) uint8_t smraw[];
    // the base of dynamic shared memory is at least 16-byte aligned; align to 1024
    uint8_t* sm = smraw + ((1024u - (smem_addr(smraw) & 1023u)) & 1023u);
    const uint32_t sbase = smem_addr(sm);
    float* Cs = reinterpret_cast<float*>(sm + kOffC);
    float* n2s = reinterpret_cast<float*>(sm + kOffN2);
    uint64_t* bar = reinterpret_cast<uint64_t*>(sm + kOffBar);
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sm + kOffBar + 8);
    const int tid = threadIdx.x, lane = lane_id(), warp = tid >> 5;

    // ---- constant operands: B = -2C (hi, lo; zero-padded to K = 8), |C|^2
    //      column, ones column ----
    for (int i = tid; i < kNC * SUB; i += kTcThreads) Cs[i] = a.C[i];
    __syncthreads();
    for (int n = tid; n < kNC; n += kTcThreads) {
        float nn = 0.f;
#pragma unroll
        for (int k = 0; k < SUB; ++k) nn = fmaf(Cs[n * SUB + k], Cs[n * SUB + k], nn);
        n2s[n] = nn;
        uint32_t hi[8], lo[8], q2[8];
#pragma unroll
        for (int k = 0; k < 8; ++k) {
            const float c = k < SUB ? -2.0f * Cs[n * SUB + k] : 0.f;
            hi[k] = to_tf32(c);
            lo[k] = to_tf32(c - __uint_as_float(hi[k]));
            q2[k] = 0u;
        }
        q2[0] = to_tf32(nn);
        q2[1] = to_tf32(nn - __uint_as_float(q2[0]));
#pragma unroll
        for (int p = 0; p < 2; ++p) {
            const uint32_t off = (uint32_t)p * (kNC * 16) + (uint32_t)n * 16;
            *reinterpret_cast<uint4*>(sm + kOffBhi + off) = make_uint4(hi[4 * p], hi[4 * p + 1], hi[4 * p + 2], hi[4 * p + 3]);
            *reinterpret_cast<uint4*>(sm + kOffBlo + off) = make_uint4(lo[4 * p], lo[4 * p + 1], lo[4 * p + 2], lo[4 * p + 3]);
            *reinterpret_cast<uint4*>(sm + kOffBn2 + off) = make_uint4(q2[4 * p], q2[4 * p + 1], q2[4 * p + 2], q2[4 * p + 3]);
        }
    }
    {  // ones column: A_one[m] = (1, 1, 0, ..., 0)
        const uint32_t one = __float_as_uint(1.0f);
        *reinterpret_cast<uint4*>(sm + kOffAone + tid * 16) = make_uint4(one, one, 0u, 0u);
        *reinterpret_cast<uint4*>(sm + kOffAone + kRows * 16 + tid * 16) = make_uint4(0u, 0u, 0u, 0u);
    }
    if (tid == 0) {
        asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;\n" ::"r"(smem_addr(bar)));
        asm volatile("fence.mbarrier_init.release.cluster;\n" ::: "memory");
    }
    if (warp == 0) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;\n" ::"r"(smem_addr(tmem_slot)),
                     "r"((uint32_t)kCols));
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;\n");
    }
    asm volatile("fence.proxy.async.shared::cta;\n" ::: "memory");
    asm volatile("tcgen05.fence::before_thread_sync;\n" ::: "memory");
    __syncthreads();
    asm volatile("tcgen05.fence::after_thread_sync;\n" ::: "memory");
    const uint32_t tmem = *tmem_slot;
    float cmax2 = 0.f;  // largest |C|^2 (for the near-tie band)
    for (int n = 0; n < kNC; ++n) cmax2 = fmaxf(cmax2, n2s[n]);
    const float cmax = sqrtf(cmax2) * (1.f + 1e-6f);
    const uint64_t dAhi = mat_desc(sbase + kOffAhi, kRows * 16, 128);
    const uint64_t dAlo = mat_desc(sbase + kOffAlo, kRows * 16, 128);
    const uint64_t dAone = mat_desc(sbase + kOffAone, kRows * 16, 128);
    const uint64_t dBhi = mat_desc(sbase + kOffBhi, kNC * 16, 128);
    const uint64_t dBlo = mat_desc(sbase + kOffBlo, kNC * 16, 128);
    const uint64_t dBn2 = mat_desc(sbase + kOffBn2, kNC * 16, 128);

    // Launched as a programmatic dependent of pass 1: the setup above
    // overlaps its end; the shift it derives is read only after this wait.
    // A dependent attention kernel may then be scheduled (it waits for this
    // grid before reading the codes).
    asm volatile("griddepcontrol.wait;\n" ::: "memory");
    asm volatile("griddepcontrol.launch_dependents;\n" ::: "memory");
    const int l16 = lane & 15, half = lane >> 4;
    const int row = tid;  // = 32 * warp + lane: this thread's sub-vector row and TMEM lane
    const int64_t pairs_per_head = (a.T + 1) / 2;
    const int64_t npairs = (int64_t)a.B * a.H * pairs_per_head;
    const int64_t ntiles = (npairs + 3) / 4;
    uint32_t phase = 0;
    bool failed = false;
    for (int64_t tile = blockIdx.x; tile < ntiles; tile += gridDim.x) {
        const int64_t pi = 4 * tile + warp;
        const bool wvalid = pi < npairs;
        const int64_t pic = wvalid ? pi : 0;
        // pic < npairs < 2^31: 32-bit divisions by the launch's invariants
        const uint32_t pic32 = (uint32_t)pic;
        const uint32_t bh32 = fdiv(pic32, a.div_items);  // pairs_per_head
        const int64_t bh = bh32;
        const int64_t t0 = 2 * (int64_t)(pic32 - bh32 * a.div_items.d);
        const int64_t t = t0 + half;
        const uint32_t b32 = fdiv(bh32, a.div_H);
        const int b = (int)b32, h = (int)(bh32 - b32 * (uint32_t)a.H);
        const bool valid = wvalid && t < a.T;
        const XT* xhead = enc_head<XT>(a, b, h);
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
        float s1 = sqrtf(ss * (1.0f / kD));
        float inv1 = s1 > 0.f ? 1.0f / s1 : 0.f;
        double s1dq = -1.0;
        int s1lev = 0;
        if constexpr (DQ) {  // s1 on the head's 4-bit log2 grid, level decided in fp64
            double ss64 = 0.0;
#pragma unroll
            for (int k = 0; k < 8; ++k) ss64 = fma((double)v[k], (double)v[k], ss64);
#pragma unroll
            for (int m = 1; m < 16; m <<= 1) ss64 += __shfl_xor_sync(kFull, ss64, m);
            double glo, gstep;
            dq_grid(enc_s1_grid(a, enc_second(a, bh)), enc_cbh(a, bh), glo, gstep);
            s1dq = dq_s1(sqrt(ss64) / sqrt((double)kD), glo, gstep, &s1lev);
            s1 = (float)s1dq;
            inv1 = s1dq > 0.0 ? (float)(1.0 / s1dq) : 0.f;
        }
        const float* shift_h = enc_shift(a, enc_second(a, bh)) + enc_cbh(a, bh) * kD;
        const float4* o4 = reinterpret_cast<const float4*>(shift_h + 8 * l16);
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
        const bool cancel = s2 < kCancelTc;
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
        // ---- per round: this thread's sub-vector as the A row, the MMAs over
        //      both halves of the codebook, and the scan of its 256 scores ----
        int i1r[RPL];
        bool tier[RPL];
        float wq = 0.f;
        const uint32_t taddr = tmem + ((uint32_t)(32 * warp) << 16);
#pragma unroll
        for (int rd = 0; rd < RPL; ++rd) {
            float ws[8];
#pragma unroll
            for (int k = 0; k < 8; ++k) ws[k] = k < SUB ? v[SUB * rd + k] : 0.f;
            float ww = 0.f;
#pragma unroll
            for (int k = 0; k < SUB; ++k) ww = fmaf(ws[k], ws[k], ww);
            {
                uint32_t hi[8], lo[8];
#pragma unroll
                for (int k = 0; k < 8; ++k) {
                    hi[k] = to_tf32(ws[k]);
                    lo[k] = to_tf32(ws[k] - __uint_as_float(hi[k]));
                }
#pragma unroll
                for (int p = 0; p < 2; ++p) {
                    const uint32_t off = (uint32_t)p * (kRows * 16) + (uint32_t)row * 16;
                    *reinterpret_cast<uint4*>(sm + kOffAhi + off) = make_uint4(hi[4 * p], hi[4 * p + 1], hi[4 * p + 2], hi[4 * p + 3]);
                    *reinterpret_cast<uint4*>(sm + kOffAlo + off) = make_uint4(lo[4 * p], lo[4 * p + 1], lo[4 * p + 2], lo[4 * p + 3]);
                }
            }
            asm volatile("fence.proxy.async.shared::cta;\n" ::: "memory");
            asm volatile("tcgen05.fence::before_thread_sync;\n" ::: "memory");
            __syncthreads();  // A written; the previous round's TMEM reads are done
            // Scan of the row's 256 scores by groups of 8: the group minimum (no
            // index), the least and second-least group minimum, and a copy of the
            // best group's 8 scores. The best score, its index (lowest on ties)
            // and the second-best score come out exactly as from a full scan: the
            // second best is the better of the best group's second and the second
            // group minimum.
            float gm1 = INFINITY, gm2 = INFINITY;
            float gs[8];
#pragma unroll
            for (int k = 0; k < 8; ++k) gs[k] = INFINITY;
            int gcol = 0;
#pragma unroll 1
            for (int hf = 0; hf < 2; ++hf) {
                if (hf) {  // this half reuses the accumulator: every read of the first is done
                    asm volatile("tcgen05.fence::before_thread_sync;\n" ::: "memory");
                    __syncthreads();
                }
                if (tid == 0) {
                    asm volatile("tcgen05.fence::after_thread_sync;\n" ::: "memory");
                    const uint64_t bo = (uint64_t)((hf * kCols * 16) >> 4);  // rows 128 hf.. of B
                    mma_tf32(tmem, dAhi, dBhi + bo, 0u);
                    mma_tf32(tmem, dAlo, dBhi + bo, 1u);
                    mma_tf32(tmem, dAhi, dBlo + bo, 1u);
                    mma_tf32(tmem, dAone, dBn2 + bo, 1u);
                    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];\n" ::"r"(
                                     smem_addr(bar))
                                 : "memory");
                }
                long long spins = 0;
                while (!mbar_try_wait(smem_addr(bar), phase) && ++spins < kWaitLimit) {
                }
                const bool done = spins < kWaitLimit;
                if (__syncthreads_and(done) == 0) {  // MMA not seen complete: flag and stop
                    if (tid == 0 && a.stats) atomicOr(&a.stats[4], 1ull);
                    failed = true;
                    break;
                }
                phase ^= 1u;
                asm volatile("tcgen05.fence::after_thread_sync;\n" ::: "memory");
#pragma unroll 1
                for (int c0 = 0; c0 < kCols; c0 += 32) {
                    uint32_t r[32];
                    tmem_ld32(taddr + (uint32_t)c0, r);
#pragma unroll
                    for (int g = 0; g < 4; ++g) {
                        float q[8];
#pragma unroll
                        for (int k = 0; k < 8; ++k) q[k] = __uint_as_float(r[8 * g + k]);
                        const float m = fminf(fminf(fminf(q[0], q[1]), fminf(q[2], q[3])),
                                              fminf(fminf(q[4], q[5]), fminf(q[6], q[7])));
                        const bool better = m < gm1;  // strict: the earlier group keeps ties
                        gm2 = fminf(gm2, fmaxf(gm1, m));
                        gm1 = fminf(gm1, m);
#pragma unroll
                        for (int k = 0; k < 8; ++k) gs[k] = better ? q[k] : gs[k];
                        gcol = better ? hf * kCols + c0 + 8 * g : gcol;
                    }
                }
            }
            if (failed) break;
            const float b1 = gm1;
            int k1 = 7;
#pragma unroll
            for (int k = 6; k >= 0; --k) k1 = gs[k] == b1 ? k : k1;
            float bin = INFINITY;
#pragma unroll
            for (int k = 0; k < 8; ++k) bin = k == k1 ? bin : fminf(bin, gs[k]);
            const float b2 = fminf(bin, gm2);
            const int i1 = gcol + k1;
            const float wn = sqrtf(ww), c1 = sqrtf(n2s[i1]);
            const float band_s = kScoreErrTc * (n2s[i1] + cmax * cmax + 2.f * wn * (c1 + cmax));
            tier[rd] = valid && (cancel || (b2 - b1) <= fmaxf(fmaf(kTieRelTc, ww + b1, kTieAbsTc), band_s));
            i1r[rd] = i1;
            if constexpr (ADAPT) wq += 0.5f * (n2s[i1] - b1);  // w . C[best] = (|C|^2 - s) / 2
        }
        if (failed) break;
        if constexpr (ADAPT) wq = half_sum(wq);
        // ---- codes of the warp's two token-heads (lane l16 holds sub-vectors
        //      RPL l16 .. RPL l16 + RPL - 1 of its token), then the exact path ----
        uint32_t mine = 0u;  // this lane's codes, one byte per round
#pragma unroll
        for (int rd = 0; rd < RPL; ++rd) mine |= (uint32_t)i1r[rd] << (8 * rd);
        constexpr int LPW = 4 / RPL;  // lanes per code word
        uint32_t cw[NW];
#pragma unroll
        for (int k = 0; k < NW; ++k) {
            uint32_t word = 0u;
#pragma unroll
            for (int r = 0; r < LPW; ++r)
                word |= __shfl_sync(kFull, mine, 16 * half + LPW * k + r) << (8 * RPL * r);
            cw[k] = word;
        }
        // near-tie flags of the warp's token-heads: bit j of half hh = sub-vector j
        uint32_t tflag[2] = {0u, 0u};
#pragma unroll
        for (int rd = 0; rd < RPL; ++rd) {
            const uint32_t m = __ballot_sync(kFull, tier[rd]);
#pragma unroll
            for (int hh = 0; hh < 2; ++hh) {
                const uint32_t f = (m >> (16 * hh)) & 0xffffu;
#pragma unroll
                for (int i = 0; i < 16; ++i) tflag[hh] |= ((f >> i) & 1u) << (RPL * i + rd);
            }
        }
        float s1o = s1, s2o = s2;
        double wqd = (double)wq;
        if (tflag[0] | tflag[1]) {  // warp-uniform
            const double* o64 = a.given_shift ? nullptr : a.o64 + bh * kD;
#pragma unroll 1
            for (int hh = 0; hh < 2; ++hh) {
                const uint32_t flags = tflag[hh];
                if (!flags) continue;  // warp-uniform
                uint32_t cq[NW];
#pragma unroll
                for (int k = 0; k < NW; ++k) cq[k] = __shfl_sync(kFull, cw[k], 16 * hh);
                double s1d, s2d, wq64;
                const double s1f = __shfl_sync(kFull, s1dq, 16 * hh);
                exact_warp_tc<XT, SUB>(xhead + (t0 + hh) * a.st, o64,
                                       enc_shift(a, enc_second(a, bh)) + enc_cbh(a, bh) * kD, Cs, flags,
                                       cq, s1f, s1d, s2d, wq64);
                if (half == hh) {
#pragma unroll
                    for (int k = 0; k < NW; ++k) cw[k] = cq[k];
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
            const bool sec = enc_second(a, bh);
            const int64_t cbh = enc_cbh(a, bh);
            const int64_t orow = cbh * a.cap + a.t_offset + t;
            uint4* dst = reinterpret_cast<uint4*>(enc_codes(a, sec) + orow * (4 * NW));
#pragma unroll
            for (int k = 0; k < NW / 4; ++k) dst[k] = make_uint4(cw[4 * k], cw[4 * k + 1], cw[4 * k + 2], cw[4 * k + 3]);
            store_byproducts(enc_scales(a, sec), enc_s1_levels(a, sec), cbh, a.cap, a.t_offset + t, s1o,
                             s2o, s1lev);
        }
    }
    // ---- release TMEM (after every thread's last read; after the last MMA) ----
    if (failed) {  // wait, bounded, for the MMA in flight before freeing its columns
        long long spins = 0;
        while (!mbar_try_wait(smem_addr(bar), phase) && ++spins < kWaitLimit) {
        }
    }
    asm volatile("tcgen05.fence::before_thread_sync;\n" ::: "memory");
    __syncthreads();
    if (warp == 0) {
        asm volatile("tcgen05.fence::after_thread_sync;\n" ::: "memory");
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;\n" ::"r"(tmem), "r"((uint32_t)kCols));
    }
}

template <typename XT, bool ADAPT, bool DQ, int SUB>
cudaError_t launch_tc(const EncodeArgs& a, cudaStream_t s) {
    static std::atomic<unsigned long long> ready{0};
    const int sms = device_sm_count();
    const int64_t npairs = (int64_t)a.B * a.H * ((a.T + 1) / 2);
    const int64_t ntiles = (npairs + 3) / 4;
    const int64_t cap = (int64_t)sms * 4;  // four CTAs per SM: all resident, 512 TMEM columns
    const int grid = (int)(ntiles < cap ? ntiles : cap);
    EncodeArgs k = a;
    k.div_items = make_fastdiv((uint32_t)((a.T + 1) / 2));
    k.div_H = make_fastdiv((uint32_t)a.H);
    return launch_smem_pdl(nsn_encode_tc_kernel<XT, ADAPT, DQ, SUB>, ready, dim3(grid), dim3(kTcThreads),
                           (size_t)kTcSmem, s, k);
}

template <int SUB>
cudaError_t launch_tc_sub(const EncodeArgs& a, cudaStream_t s) {
    if (a.x_bf16) {
        if (a.dq) return a.adaptive ? launch_tc<__nv_bfloat16, true, true, SUB>(a, s)
                                    : launch_tc<__nv_bfloat16, false, true, SUB>(a, s);
        return a.adaptive ? launch_tc<__nv_bfloat16, true, false, SUB>(a, s)
                          : launch_tc<__nv_bfloat16, false, false, SUB>(a, s);
    }
    if (a.dq) return a.adaptive ? launch_tc<float, true, true, SUB>(a, s) : launch_tc<float, false, true, SUB>(a, s);
    return a.adaptive ? launch_tc<float, true, false, SUB>(a, s) : launch_tc<float, false, false, SUB>(a, s);
}

}  // namespace

cudaError_t launch_encode_tc(const EncodeArgs& a, cudaStream_t s) {
    return a.sub == 4 ? launch_tc_sub<4>(a, s) : launch_tc_sub<8>(a, s);
}

}  // namespace nsnq
