// NSNQuant encode for 4-dimensional sub-vectors (2 bits/coordinate) on
// sm_100a: normalize-shift-normalize, Hadamard transform and the exact
// nearest codeword found through the grid-cell index of vq_index.cuh
// (gist.science "NSNQuant ...", Technical Summary, Methodology §1-§3).
//
// Persistent CTAs of 512 threads keep the index (cell offsets + candidate
// lists) and an 8-way replicated copy of the codebook in shared memory.
// Two threads share a token-head: each holds 64 of its 128 coordinates, runs
// six FWHT stages in registers (packed f32x2 adds) and one across the pair,
// then searches its 16 sub-vectors: cell -> candidate list (sorted by a
// lower bound of the distance) -> distances until the next lower bound
// exceeds the best distance plus the near-tie band. Near ties and heavily
// cancelled residuals are re-decided from an fp64 recomputation.
#include <math.h>

#include "common.cuh"
#include "f32x2.cuh"
#include "internal.h"
#include "dq.cuh"
#include "vq_index.cuh"

namespace nsnq {

constexpr int kPrunedThreads = 512;
constexpr int kWarps = kPrunedThreads / 32;
constexpr int kWarpTile = 16;              // token-heads per warp tile (2 threads each)
constexpr float kCancel = 1e-3f;           // s2 below this: residual decided in fp64

// shared-memory map (bytes)
constexpr size_t kSmReps = 0;                                  // float4 [256][8]
constexpr size_t kSmShift = kSmReps + size_t(kNC) * 8 * 16;   // float [warps][136]
constexpr size_t kSmHash = kSmShift + size_t(kPrunedThreads / 32) * 136 * 4;
constexpr size_t kSmBinTab = kSmHash + 16;                     // uint8 [kBinTabSize]
constexpr size_t kSmOffsets = kSmBinTab + kBinTabSize;         // uint16 [kCells + 1]
constexpr size_t kSmEntries = kSmOffsets + kIdxSmemOffsetsBytes;
constexpr size_t kSmBytes = kSmEntries + size_t(kMaxPairs) * 4;


__device__ __forceinline__ uint32_t cb_hash_term(uint32_t bits, uint32_t i) {
    uint32_t h = bits * 0x9E3779B1u ^ (i * 0x85EBCA77u + 0x165667B1u);
    h ^= h >> 15;
    h *= 0x2C1B3C6Du;
    h ^= h >> 13;
    return h;
}

template <typename XT>
__device__ __forceinline__ void load64(const XT* p, float (&v)[64]);
template <>
__device__ __forceinline__ void load64<__nv_bfloat16>(const __nv_bfloat16* p, float (&v)[64]) {
    const uint4* q = reinterpret_cast<const uint4*>(p);
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        const uint4 a = __ldg(q + i);
        const uint32_t u[4] = {a.x, a.y, a.z, a.w};
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            v[8 * i + 2 * k] = __uint_as_float(u[k] << 16);
            v[8 * i + 2 * k + 1] = __uint_as_float(u[k] & 0xffff0000u);
        }
    }
}
template <>
__device__ __forceinline__ void load64<float>(const float* p, float (&v)[64]) {
    const float4* q = reinterpret_cast<const float4*>(p);
#pragma unroll
    for (int i = 0; i < 16; ++i) {
        const float4 a = __ldg(q + i);
        v[4 * i] = a.x; v[4 * i + 1] = a.y; v[4 * i + 2] = a.z; v[4 * i + 3] = a.w;
    }
}

// Exact decision for one token-head, by the whole warp: fp64 NSN of the
// token (lane l holds channels 4l..4l+3; s1_fixed >= 0 is a given, double-
// quantized s1), fp64 Hadamard transform across the
// warp, after which lane l holds sub-vector l of w; each flagged lane scans
// its cell list in fp64 (the list holds every codeword that can be nearest
// there; lowest index on exact ties). Returns this lane's code (old_code when
// not flagged), the fp64 (s1, s2) and, summed over the warp, w . C[code] over
// all sub-vectors and w . (C[new] - C[old]) over the flagged ones (for the
// scale adjustment). Kept short and warp-wide: a slow warp holds its SM.
template <typename XT>
__device__ __noinline__ int exact_warp(const XT* xtok, const double* o64, const float* o32,
                                       const float4* reps, const uint16_t* offs,
                                       const uint16_t* ents, uint32_t flags, int old_code,
                                       double s1_fixed, double& s1_out, double& s2_out,
                                       double& wq_all, double& wq_delta) {
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
    double w[4];
#pragma unroll
    for (int r = 0; r < 4; ++r) w[r] = z[r] * hs;
    int code = old_code;
    if ((flags >> lane) & 1u) {
        int cell = 0;
#pragma unroll
        for (int i = 0; i < 4; ++i) cell = cell * kNb + bin_of((float)w[i]);
        double bd = INFINITY;
        int bi = 0;
        // every entry of the list, the padding codeword included (it never wins)
        for (uint32_t q = 2u * offs[cell]; q < 2u * offs[cell + 1]; ++q) {
            const int c = ents[q] & 0xff;
            const float4 cv = reps[c * 8];
            const double e0 = w[0] - (double)cv.x, e1 = w[1] - (double)cv.y;
            const double e2 = w[2] - (double)cv.z, e3 = w[3] - (double)cv.w;
            const double d = e0 * e0 + e1 * e1 + e2 * e2 + e3 * e3;
            if (d < bd || (d == bd && c < bi)) { bd = d; bi = c; }
        }
        code = bi;
    }
    const float4 cn = reps[code * 8], co = reps[old_code * 8];
    const double qn = w[0] * (double)cn.x + w[1] * (double)cn.y + w[2] * (double)cn.z + w[3] * (double)cn.w;
    const double qo = w[0] * (double)co.x + w[1] * (double)co.y + w[2] * (double)co.z + w[3] * (double)co.w;
    wq_all = warp_sum_d(qn);
    wq_delta = warp_sum_d(((flags >> lane) & 1u) ? qn - qo : 0.0);
    s1_out = s1;
    s2_out = s2;
    return code;
}

// Bin of one coordinate through the shared-memory bin table.
__device__ __forceinline__ int bin_fast(float x, const uint8_t* tab) {
    const unsigned t = (unsigned)__float2int_rd(fmaf(x, kBinGrid, (float)kBinTabZero));
    return tab[min(t, (unsigned)kBinTabSize - 1u)];
}

// Candidate walk of one sub-vector w through its cell's list.
struct Walk {
    uint64_t w01, w23;
    uint32_t p, e;
    float d1, d2;
    int i1;

    __device__ __forceinline__ void init(float w0, float w1, float w2, float w3,
                                         const uint16_t* offs, const uint8_t* tab) {
        const int cell = ((bin_fast(w0, tab) * kNb + bin_fast(w1, tab)) * kNb + bin_fast(w2, tab)) * kNb +
                         bin_fast(w3, tab);
        p = offs[cell];
        e = offs[cell + 1];
        w01 = pk2(w0, w1);
        w23 = pk2(w2, w3);
        d1 = INFINITY; d2 = INFINITY; i1 = 0;
    }

    // Evaluate the next pair of entries (p < e); the walk ends (p = e) after
    // a pair whose second lower bound leaves the band of the best distance
    // before the pair, or at the end of the list (entries are sorted by lower
    // bound, so no contender is skipped). Branch-free.
    __device__ __forceinline__ void step(const uint32_t* pairs, const float4* myrep) {
        const uint32_t pr = pairs[p];
        const uint32_t ent0 = pr & 0xffffu, ent1 = pr >> 16;
        // Lower bounds are floor(lb * 64) in the high byte of each entry. The
        // band's limit, 64 d1 (1 + rel) rounded to the nearest integer (never
        // below floor(64 (d1 (1 + rel) + abs)), abs < 1/128), is the low
        // mantissa of y = 2^23 + 64 d1 (1 + rel); a larger y (d1 >= 2^17 or
        // infinite) has larger bits and admits every entry.
        const float y = fmaf(d1, (1.0f + kTieRel) * kLbScale, 8388608.0f);
        const uint32_t lim = __float_as_uint(y);
        const bool take1 = (0x4b000000u | (ent1 >> 8)) <= lim;
        // codewords read as packed pairs (c0, c1), (c2, c3)
        const ulonglong2 cv0 = reinterpret_cast<const ulonglong2*>(myrep)[(ent0 & 0xff) * 8];
        const ulonglong2 cv1 = reinterpret_cast<const ulonglong2*>(myrep)[(ent1 & 0xff) * 8];
        const uint64_t a01 = sub2(w01, cv0.x), a23 = sub2(w23, cv0.y);
        const uint64_t b01 = sub2(w01, cv1.x), b23 = sub2(w23, cv1.y);
        const float2 da = upk2(fma2(a23, a23, mul2(a01, a01)));
        const float2 db = upk2(fma2(b23, b23, mul2(b01, b01)));
        // Both entries count even past the band: they are listed codewords
        // (or the padding, farther than the nearest by the margin), so they
        // can only tighten d1 or reveal a true near-tie.
        const float dA = da.x + da.y;
        const float dB = db.x + db.y;
        d2 = fminf(d2, fmaxf(d1, dA));
        i1 = dA < d1 ? (int)(ent0 & 0xff) : i1;
        d1 = fminf(d1, dA);
        d2 = fminf(d2, fmaxf(d1, dB));
        i1 = dB < d1 ? (int)(ent1 & 0xff) : i1;
        d1 = fminf(d1, dB);
        p = take1 ? p + 1 : e;
    }

    __device__ __forceinline__ bool tie() const { return (d2 - d1) <= fmaf(kTieRel, d1, kTieAbs); }
};

// ADAPT: also apply the scale adjustment s2 *= ||w||^2 / (w . w_hat). Since
// u = z / s2 has ||u||^2 = d and H is orthonormal, ||w||^2 = d; only w . w_hat
// is accumulated, in the search loop. DQ: s1 on the head's 4-bit log2 grid,
// its level decided from an fp64 sum of squares.
template <typename XT, bool ADAPT, bool DQ>
__global__ void __launch_bounds__(kPrunedThreads, 1) nsn_encode_pruned_kernel(EncodeArgs a) {
    extern __shared__ __align__(16) uint8_t sm[];
    float4* reps = reinterpret_cast<float4*>(sm + kSmReps);
    float* shift_s = reinterpret_cast<float*>(sm + kSmShift);
    const uint16_t* offs = reinterpret_cast<const uint16_t*>(sm + kSmOffsets);
    const uint16_t* ents = reinterpret_cast<const uint16_t*>(sm + kSmEntries);
    const uint32_t* pairs = reinterpret_cast<const uint32_t*>(sm + kSmEntries);
    uint8_t* bintab = sm + kSmBinTab;
    const int tid = threadIdx.x, lane = lane_id();
    const int half = lane & 1;
    const float sgn = half ? -1.0f : 1.0f;

    // ---- stage the index and the replicated codebook ----
    const IndexHeader* hdr = reinterpret_cast<const IndexHeader*>(a.index);
    const uint32_t n_pairs = min(hdr->n_pairs, (uint32_t)kMaxPairs);
    unsigned* hash_s = reinterpret_cast<unsigned*>(sm + kSmHash);
    if (tid == 0) *hash_s = 0u;
    __syncthreads();
    {
        const uint4* src = reinterpret_cast<const uint4*>(static_cast<const uint8_t*>(a.index) + kIdxOffsets);
        uint4* dst = reinterpret_cast<uint4*>(sm + kSmOffsets);
        const size_t nbytes = kIdxSmemOffsetsBytes + ((size_t)n_pairs * 4 + 15) / 16 * 16;
        for (size_t i = tid; i < nbytes / 16; i += kPrunedThreads) dst[i] = src[i];
        for (int i = tid; i < kNC * 8; i += kPrunedThreads)
            reps[i] = reinterpret_cast<const float4*>(a.C)[i >> 3];
        for (int t = tid; t < kBinTabSize; t += kPrunedThreads)
            bintab[t] = (uint8_t)bin_of((float)(t - kBinTabZero) * (1.0f / kBinGrid));
        uint32_t h = 0;
        for (int i = tid; i < kNC * 4; i += kPrunedThreads) h ^= cb_hash_term(__float_as_uint(a.C[i]), i);
#pragma unroll
        for (int m = 16; m; m >>= 1) h ^= __shfl_xor_sync(kFull, h, m);
        if (lane == 0) atomicXor(hash_s, h);
    }
    __syncthreads();
    if (tid == 0 && blockIdx.x == 0 && a.stats &&
        (*hash_s != hdr->pad[0] || hdr->magic != kIndexMagic || hdr->overflow))
        atomicOr(&a.stats[2], 1ull);
    // Offsets past the staged entries (an index of other centroids, or not
    // an index at all: flagged above, its codes are void) are clamped, so
    // that every walk stays inside shared memory.
    {
        uint16_t* offs_w = reinterpret_cast<uint16_t*>(sm + kSmOffsets);
        for (int i = tid; i <= kCells; i += kPrunedThreads)
            offs_w[i] = (uint16_t)min((uint32_t)offs_w[i], n_pairs);
    }
    __syncthreads();
    // Launched as a programmatic dependent of pass 1: the staging above
    // overlaps its end; the shift it derives is read only after this wait.
    // The next kernel (decode attention over these caches) may then be
    // scheduled; it waits for this grid before reading the codes.
    asm volatile("griddepcontrol.wait;\n" ::: "memory");
    asm volatile("griddepcontrol.launch_dependents;\n" ::: "memory");

    // Each warp owns tiles of 16 consecutive token-heads of one (batch, head)
    // and keeps its own copy of that head's shift: no CTA barrier in the loop.
    const int warp = tid >> 5;
    float* wshift = shift_s + warp * 136;  // [128 + 4 pad + 4]
    const int64_t tiles_per_bh = (a.T + kWarpTile - 1) / kWarpTile;
    const int64_t ntiles = (int64_t)a.B * a.H * tiles_per_bh;
    const float4* shift4 = reinterpret_cast<const float4*>(wshift);
    int64_t cur_bh = -1;
    // Warp tiles are handed out by a counter in the workspace (reset by the
    // host before the launch), so warps that hit slow tiles do not hold back
    // a static share of the work.
    for (;;) {
        unsigned long long tl = 0;
        if (lane == 0) tl = atomicAdd(&a.stats[3], 1ull);
        const int64_t tile = (int64_t)__shfl_sync(kFull, tl, 0);
        if (tile >= ntiles) break;
        // tile < ntiles < 2^31: 32-bit divisions by the launch's invariants
        const uint32_t tile32 = (uint32_t)tile;
        const uint32_t bh32 = fdiv(tile32, a.div_items);  // tiles_per_bh
        const int64_t bh = bh32;
        const int64_t t = (int64_t)(tile32 - bh32 * a.div_items.d) * kWarpTile + (lane >> 1);
        const uint32_t b32 = fdiv(bh32, a.div_H);
        const int b = (int)b32, h = (int)(bh32 - b32 * (uint32_t)a.H);
        if (bh != cur_bh) {  // warp-uniform
            __syncwarp();
            const float4 o =
                reinterpret_cast<const float4*>(enc_shift(a, enc_second(a, bh)) + enc_cbh(a, bh) * kD)[lane];
            reinterpret_cast<float4*>(wshift)[lane + (lane >= 16 ? 1 : 0)] =
                make_float4(-o.x, -o.y, -o.z, -o.w);  // -o: the shift is subtracted
            __syncwarp();
            cur_bh = bh;
        }
        const bool valid = t < a.T;
        const XT* xrow = enc_head<XT>(a, b, h) + (valid ? t : 0) * a.st;
        float v[64];
        if (valid) {
            load64<XT>(xrow + 64 * half, v);
        } else {
#pragma unroll
            for (int k = 0; k < 64; ++k) v[k] = 0.f;
        }
        // ---- normalize, shift, normalize ----
        uint64_t acc0 = 0, acc1 = 0;
#pragma unroll
        for (int k = 0; k < 64; k += 4) {
            const uint64_t p0 = pk2(v[k], v[k + 1]), p1 = pk2(v[k + 2], v[k + 3]);
            acc0 = fma2(p0, p0, acc0);
            acc1 = fma2(p1, p1, acc1);
        }
        float2 s01 = upk2(add2(acc0, acc1));
        float ss = s01.x + s01.y;
        ss += __shfl_xor_sync(kFull, ss, 1);
        float s1 = sqrtf(ss * (1.0f / kD));
        float inv1 = s1 > 0.f ? 1.0f / s1 : 0.f;
        double s1dq = -1.0;
        int s1lev = 0;
        if constexpr (DQ) {
            double ss64 = 0.0;
#pragma unroll
            for (int k = 0; k < 64; ++k) ss64 = fma((double)v[k], (double)v[k], ss64);
            ss64 += __shfl_xor_sync(kFull, ss64, 1);
            double glo, gstep;
            dq_grid(enc_s1_grid(a, enc_second(a, bh)), enc_cbh(a, bh), glo, gstep);
            s1dq = dq_s1(sqrt(ss64) / sqrt((double)kD), glo, gstep, &s1lev);
            s1 = (float)s1dq;
            inv1 = s1dq > 0.0 ? (float)(1.0 / s1dq) : 0.f;
        }
        const float4* o4 = shift4 + 17 * half;  // upper half stored 4 floats further
        acc0 = 0; acc1 = 0;
        const uint64_t inv2 = pk2(inv1, inv1);
#pragma unroll
        for (int k = 0; k < 64; k += 4) {
            const float4 o = o4[k >> 2];
            const uint64_t z0 = fma2(pk2(v[k], v[k + 1]), inv2, pk2(o.x, o.y));
            const uint64_t z1 = fma2(pk2(v[k + 2], v[k + 3]), inv2, pk2(o.z, o.w));
            acc0 = fma2(z0, z0, acc0);
            acc1 = fma2(z1, z1, acc1);
            const float2 a0 = upk2(z0), a1 = upk2(z1);
            v[k] = a0.x; v[k + 1] = a0.y; v[k + 2] = a1.x; v[k + 3] = a1.y;
        }
        s01 = upk2(add2(acc0, acc1));
        float ss2 = s01.x + s01.y;
        ss2 += __shfl_xor_sync(kFull, ss2, 1);
        const float s2 = sqrtf(ss2 * (1.0f / kD));
        const bool cancel = s2 < kCancel;
        const float sc = s2 > 0.f ? kRsqrtD / s2 : 0.f;
        // ---- FWHT: bits 0..4 on packed pairs (v[i], v[i+32]), bit 5 in-thread, bit 6 across the pair
        uint64_t P[32];
        const uint64_t sc2 = pk2(sc, sc);
#pragma unroll
        for (int i = 0; i < 32; ++i) P[i] = mul2(pk2(v[i], v[i + 32]), sc2);
#pragma unroll
        for (int bit = 1; bit < 32; bit <<= 1) {
#pragma unroll
            for (int i = 0; i < 32; ++i) {
                if (i & bit) continue;
                const uint64_t x0 = P[i], x1 = P[i | bit];
                P[i] = add2(x0, x1);
                P[i | bit] = sub2(x0, x1);
            }
        }
#pragma unroll
        for (int i = 0; i < 32; ++i) {
            const float2 q = upk2(P[i]);
            v[i] = q.x + q.y;
            v[i + 32] = q.x - q.y;
        }
#pragma unroll
        for (int k = 0; k < 64; ++k) {
            const float p = __shfl_xor_sync(kFull, v[k], 1);
            v[k] = fmaf(v[k], sgn, p);  // lower half v + p, upper half p - v
        }
        // ---- nearest codeword of the 16 sub-vectors this thread holds ----
        uint32_t codes[4] = {0u, 0u, 0u, 0u};
        uint32_t tie = 0;
        float wq = 0.f;
        const float4* myrep = reps + (lane & 7);
#pragma unroll
        for (int jj = 0; jj < 16; ++jj) {
            Walk A;
            A.init(v[4 * jj], v[4 * jj + 1], v[4 * jj + 2], v[4 * jj + 3], offs, bintab);
            while (A.p < A.e) A.step(pairs, myrep);
            codes[jj >> 2] |= (uint32_t)A.i1 << (8 * (jj & 3));
            if (cancel || A.tie()) tie |= 1u << jj;
            if constexpr (ADAPT) {
                const float4 c = myrep[A.i1 * 8];
                wq = fmaf(v[4 * jj + 3], c.w, fmaf(v[4 * jj + 2], c.z,
                     fmaf(v[4 * jj + 1], c.y, fmaf(v[4 * jj], c.x, wq))));
            }
        }
        if (!valid) tie = 0;
        // ---- exact fp64 decision where the fp32 search is not conclusive ----
        // Token-heads with a flagged sub-vector are re-done one at a time by
        // the whole warp; results go back to the owning pair of lanes.
        const uint32_t my_mask = tie << (16 * half);
        const uint32_t both = my_mask | __shfl_xor_sync(kFull, my_mask, 1);
        float s1o = s1, s2o = s2;
        double wqd = 0.0;
        if constexpr (ADAPT) wqd = (double)(wq + __shfl_xor_sync(kFull, wq, 1));
        uint32_t pending = __ballot_sync(kFull, both != 0u && half == 0);
        if (pending) {
            const double* o64 = a.given_shift ? nullptr : a.o64 + bh * kD;
            const XT* xhead = enc_head<XT>(a, b, h);
            const int64_t t0 = t - (lane >> 1);  // first token of the tile
            while (pending) {
                const int src = __ffs(pending) - 1;  // even lane of the token-head's pair
                pending &= pending - 1;
                const uint32_t flags = __shfl_sync(kFull, both, src);
                // current code of sub-vector `lane` (held by lane src + lane / 16)
                uint32_t word = 0u;
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                    const uint32_t wk = __shfl_sync(kFull, codes[k], src + (lane >> 4));
                    if (k == ((lane & 15) >> 2)) word = wk;
                }
                const int old_code = (int)((word >> (8 * (lane & 3))) & 0xffu);
                double s1d, s2d, wq_all, wq_delta;
                const double s1f = __shfl_sync(kFull, s1dq, src);
                const int code = exact_warp<XT>(xhead + (t0 + (src >> 1)) * a.st, o64,
                                                enc_shift(a, enc_second(a, bh)) + enc_cbh(a, bh) * kD,
                                                reps, offs, ents, flags,
                                                old_code, s1f, s1d, s2d, wq_all, wq_delta);
                const bool mine = (lane >> 1) == (src >> 1);
#pragma unroll
                for (int jj = 0; jj < 16; ++jj) {
                    const uint32_t c = (uint32_t)__shfl_sync(kFull, code, 16 * half + jj);
                    const int sh = 8 * (jj & 3);
                    if (mine) codes[jj >> 2] = (codes[jj >> 2] & ~(0xffu << sh)) | (c << sh);
                }
                if (mine) {
                    s1o = (float)s1d;
                    s2o = (float)s2d;
                    // all re-decided (always so on cancellation): the fp64 sum
                    wqd = flags == kFull ? wq_all : wqd + wq_delta;
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
        if (valid) {
            const bool sec = enc_second(a, bh);
            const int64_t cbh = enc_cbh(a, bh);
            const int64_t row = cbh * a.cap + a.t_offset + t;
            reinterpret_cast<uint4*>(enc_codes(a, sec) + row * 32)[half] =
                make_uint4(codes[0], codes[1], codes[2], codes[3]);
            if (half == 0)
                store_byproducts(enc_scales(a, sec), enc_s1_levels(a, sec), cbh, a.cap, a.t_offset + t,
                                 s1o, s2o, s1lev);
        }
    }
}

size_t pruned_smem_bytes() { return kSmBytes; }

template <typename XT, bool ADAPT, bool DQ>
static cudaError_t launch_pruned_t(const EncodeArgs& a, cudaStream_t s) {
    static std::atomic<unsigned long long> ready{0};
    const int sms = device_sm_count();
    const int64_t ntiles = (int64_t)a.B * a.H * ((a.T + kWarpTile - 1) / kWarpTile);
    const int64_t ctas = (ntiles + kWarps - 1) / kWarps;
    const int grid = (int)(ctas < sms ? ctas : sms);
    EncodeArgs k = a;
    k.div_items = make_fastdiv((uint32_t)((a.T + kWarpTile - 1) / kWarpTile));
    k.div_H = make_fastdiv((uint32_t)a.H);
    return launch_smem_pdl(nsn_encode_pruned_kernel<XT, ADAPT, DQ>, ready, dim3(grid),
                           dim3(kPrunedThreads), kSmBytes, s, k);
}

cudaError_t launch_encode_pruned(const EncodeArgs& a, cudaStream_t s) {
    if (a.x_bf16) {
        if (a.dq) return a.adaptive ? launch_pruned_t<__nv_bfloat16, true, true>(a, s)
                                    : launch_pruned_t<__nv_bfloat16, false, true>(a, s);
        return a.adaptive ? launch_pruned_t<__nv_bfloat16, true, false>(a, s)
                          : launch_pruned_t<__nv_bfloat16, false, false>(a, s);
    }
    if (a.dq) return a.adaptive ? launch_pruned_t<float, true, true>(a, s) : launch_pruned_t<float, false, true>(a, s);
    return a.adaptive ? launch_pruned_t<float, true, false>(a, s) : launch_pruned_t<float, false, false>(a, s);
}

}  // namespace nsnq
