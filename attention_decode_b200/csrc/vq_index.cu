// Builder of the nearest-codeword search index for 4-dimensional
// sub-vectors (see vq_index.cuh). Runs once per codebook on the device:
//   vq_index_cells_kernel(count)  per grid cell: which codewords survive
//   vq_index_scan_kernel          pair counts -> uint16 pair offsets, header
//   vq_index_cells_kernel(fill)   per grid cell: survivors sorted by lower bound,
//                                 an odd list padded with a dominated codeword
// Dominance tests run in fp64 over cells expanded by kBoxEps.
#include <math.h>

#include "common.cuh"
#include "internal.h"
#include "vq_index.cuh"

namespace nsnq {

__device__ __forceinline__ void cell_box(int cell, double (&lo)[4], double (&hi)[4]) {
    int b[4];
    int r = cell;
#pragma unroll
    for (int i = 3; i >= 0; --i) {
        b[i] = r % kNb;
        r /= kNb;
    }
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        lo[i] = bin_edge(b[i]) - kBoxEps;
        hi[i] = bin_edge(b[i] + 1) + kBoxEps;
    }
}

// 32-bit hash of the codebook bits (order-dependent mix, reduced by xor).
__device__ __forceinline__ uint32_t codebook_hash_term(uint32_t bits, uint32_t i) {
    uint32_t h = bits * 0x9E3779B1u ^ (i * 0x85EBCA77u + 0x165667B1u);
    h ^= h >> 15;
    h *= 0x2C1B3C6Du;
    h ^= h >> 13;
    return h;
}

template <bool kFill>
__global__ void __launch_bounds__(kNC) vq_index_cells_kernel(const float* __restrict__ C,
                                                             uint8_t* __restrict__ index) {
    __shared__ double Cs[kNC][4];
    __shared__ double n2s[kNC];
    __shared__ int surv[kNC];
    __shared__ int lbqs[kNC];
    const int cell = blockIdx.x;
    const int c = threadIdx.x;
    double cc[4], n2 = 0.0;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        cc[i] = (double)C[c * 4 + i];
        Cs[c][i] = cc[i];
        n2 += cc[i] * cc[i];
    }
    n2s[c] = n2;
    double lo[4], hi[4];
    cell_box(cell, lo, hi);
    __syncthreads();
    bool dominated = false;
    for (int c2 = 0; c2 < kNC && !dominated; ++c2) {
        if (c2 == c) continue;
        // min over the cell of d(p, c) - d(p, c2) = ||c||^2 - ||c2||^2 + 2 p.(c2 - c)
        double val = n2 - n2s[c2], dmax = 0.0;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const double df = Cs[c2][i] - cc[i];
            val += fmin(2.0 * lo[i] * df, 2.0 * hi[i] * df);
            const double a = lo[i] - Cs[c2][i], bq = hi[i] - Cs[c2][i];
            dmax += fmax(a * a, bq * bq);
        }
        // margin: the near-tie band at the largest distance in the cell, twice, plus slack
        const double margin = 2.0 * ((double)kTieRel * dmax + (double)kTieAbs) + 1e-4;
        dominated = val > margin;
    }
    double lb = 0.0;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const double e = fmin(fmax(cc[i], lo[i]), hi[i]) - cc[i];
        lb += e * e;
    }
    const int lbq = (int)fmin(floor(lb * (double)kLbScale), 255.0);
    const int alive = dominated ? 0 : 1;
    const int count = __syncthreads_count(alive);
    uint16_t* offsets = reinterpret_cast<uint16_t*>(index + kIdxOffsets);
    if (!kFill) {
        if (c == 0) offsets[cell] = (uint16_t)((count + 1) / 2);
        if (cell == 0) {
            // codebook hash (xor is order-free; the term mixes in the position)
            uint32_t h = 0;
#pragma unroll
            for (int i = 0; i < 4; ++i) h ^= codebook_hash_term(__float_as_uint(C[c * 4 + i]), c * 4 + i);
#pragma unroll
            for (int m = 16; m; m >>= 1) h ^= __shfl_xor_sync(kFull, h, m);
            __shared__ uint32_t hw[kNC / 32];
            if ((c & 31) == 0) hw[c >> 5] = h;
            __syncthreads();
            if (c == 0) {
                uint32_t t = 0;
                for (int w = 0; w < kNC / 32; ++w) t ^= hw[w];
                reinterpret_cast<IndexHeader*>(index)->pad[0] = t;
            }
        }
        return;
    }
    const IndexHeader* hdr = reinterpret_cast<const IndexHeader*>(index);
    if (hdr->overflow) return;
    __shared__ int pad_code;
    if (c == 0) pad_code = kNC;
    surv[c] = alive;
    lbqs[c] = lbq;
    __syncthreads();
    if (!alive) atomicMin(&pad_code, c);  // a dominated codeword exists whenever count < 256
    __syncthreads();
    uint16_t* entries = reinterpret_cast<uint16_t*>(index + kIdxEntries) + 2 * (size_t)offsets[cell];
    if ((count & 1) && c == 0) entries[count] = (uint16_t)(pad_code | (255 << 8));
    if (!alive) return;
    int rank = 0;
    for (int c2 = 0; c2 < kNC; ++c2)
        rank += surv[c2] && (lbqs[c2] < lbq || (lbqs[c2] == lbq && c2 < c));
    entries[rank] = (uint16_t)(c | (lbq << 8));
}

// pair counts (in the offsets array) -> exclusive pair offsets; one CTA.
__global__ void __launch_bounds__(1024) vq_index_scan_kernel(uint8_t* __restrict__ index) {
    __shared__ uint32_t part[1024];
    uint16_t* offsets = reinterpret_cast<uint16_t*>(index + kIdxOffsets);
    constexpr int per = (kCells + 1023) / 1024;
    const int t = threadIdx.x;
    uint32_t local[per];
    uint32_t s = 0;
#pragma unroll
    for (int k = 0; k < per; ++k) {
        const int i = t * per + k;
        local[k] = i < kCells ? offsets[i] : 0;
        s += local[k];
    }
    part[t] = s;
    __syncthreads();
    for (int off = 1; off < 1024; off <<= 1) {
        const uint32_t v = t >= off ? part[t - off] : 0;
        __syncthreads();
        part[t] += v;
        __syncthreads();
    }
    const uint32_t total = part[1023];
    uint32_t run = part[t] - s;
    const bool overflow = total > (uint32_t)kMaxPairs;
#pragma unroll
    for (int k = 0; k < per; ++k) {
        const int i = t * per + k;
        if (i < kCells && !overflow) offsets[i] = (uint16_t)run;
        run += local[k];
    }
    if (t == 0) {
        IndexHeader* hdr = reinterpret_cast<IndexHeader*>(index);
        if (!overflow) offsets[kCells] = (uint16_t)total;
        hdr->n_pairs = total;
        hdr->overflow = overflow ? 1u : 0u;
        hdr->cells = kCells;
        hdr->magic = kIndexMagic;
    }
}

size_t index_bytes() { return kIdxBytes; }

cudaError_t launch_index_build(const float* C, void* index, cudaStream_t s) {
    uint8_t* idx = static_cast<uint8_t*>(index);
    cudaError_t e = cudaMemsetAsync(idx, 0, sizeof(IndexHeader), s);
    if (e != cudaSuccess) return e;
    vq_index_cells_kernel<false><<<kCells, kNC, 0, s>>>(C, idx);
    vq_index_scan_kernel<<<1, 1024, 0, s>>>(idx);
    vq_index_cells_kernel<true><<<kCells, kNC, 0, s>>>(C, idx);
    return cudaGetLastError();
}

}  // namespace nsnq
