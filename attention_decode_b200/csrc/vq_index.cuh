// Layout of the nearest-codeword search index for 4-dimensional sub-vectors
// (2 bits/coordinate), shared by the builder and the encode kernel.
//
// The transformed coordinates are near N(0, 1) (NSN + Hadamard, gist.science
// "NSNQuant ...", Methodology §1-§2), so each coordinate is binned on a grid
// that is fine where the data is dense: kNb = 10 bins per coordinate with
// edges at 0, +-kE1, +-kE2, +-kE3, +-kE4 (about 1.3x the deciles of N(0, 1),
// rounded to multiples of 1/32 so that a table over a 1/32 grid gives the
// bin exactly) and two outer bins reaching to +-kOuter (every coordinate of w satisfies
// |w_i| <= ||w|| = sqrt(128) < kOuter). For every grid cell the index lists
// the codewords that can be nearest (or within the near-tie margin of the
// nearest) for some point of the cell, sorted by a lower bound of their
// squared distance over the cell. A codeword is left out only if another
// codeword is closer by a margin everywhere in the cell (expanded by
// kBoxEps), so the list's best codeword is the exact nearest.
//
// Lists are stored as pairs of 16-bit entries (code | lbq << 8, lbq =
// floor(64 * lower bound) clamped to 255) so that one 32-bit load fetches
// two; an odd list is padded with a codeword that is dominated in the cell
// (never nearest and never within the near-tie margin) and lbq 255.
// Offsets count pairs.
#pragma once

#include <math.h>
#include <stdint.h>

namespace nsnq {

constexpr int kNb = 10;                           // bins per coordinate
constexpr float kE1 = 0.3125f, kE2 = 0.6875f, kE3 = 1.09375f, kE4 = 1.65625f;  // positive inner edges
constexpr double kOuter = 12.0;                   // outer bins end here (> sqrt(128))
constexpr double kBoxEps = 1e-3;                  // cell expansion covering fp32 error in w
constexpr int kCells = kNb * kNb * kNb * kNb;
constexpr int kMaxPairs = 41984;                  // list capacity in entry pairs (shared memory)
// Bin table: entry t is the bin of (t - kBinTabZero) / kBinGrid, so a
// coordinate x has bin table[floor(x * kBinGrid) + kBinTabZero] (|x| < 12).
constexpr float kBinGrid = 32.0f;
constexpr int kBinTabZero = 384;
constexpr int kBinTabSize = 768;
constexpr float kLbScale = 64.0f;                 // lower bounds stored as floor(lb * 64), <= 255
constexpr uint32_t kIndexMagic = 0x4e534e52u;

// Bin of one coordinate: the number of inner edges at or below x (bins are
// closed below, open above, like floor() on the 1/32 grid of the table).
__host__ __device__ __forceinline__ int bin_of(float x) {
    return (x >= -kE4) + (x >= -kE3) + (x >= -kE2) + (x >= -kE1) + (x >= 0.f) + (x >= kE1) +
           (x >= kE2) + (x >= kE3) + (x >= kE4);
}

// Edge k of the bins (k = 0..kNb): bin b covers [bin_edge(b), bin_edge(b + 1)].
__host__ __device__ __forceinline__ double bin_edge(int k) {
    const double e[kNb + 1] = {-kOuter, -(double)kE4, -(double)kE3, -(double)kE2, -(double)kE1, 0.0,
                               (double)kE1, (double)kE2, (double)kE3, (double)kE4, kOuter};
    return e[k];
}

// Near-tie rule of the fp32 search: a sub-vector whose two best distances
// are within kTieRel * d1 + kTieAbs is re-decided in fp64 (the fp32 error of
// a distance is ~1e-6 relative, so the band keeps a 20x margin). The index
// keeps every codeword that can come that close, so the rule sees all
// contenders.
constexpr float kTieRel = 2e-5f;
constexpr float kTieAbs = 1e-6f;

struct IndexHeader {
    uint32_t magic;
    uint32_t n_pairs;    // total list entry pairs
    uint32_t overflow;   // nonzero if the lists did not fit kMaxPairs
    uint32_t cells;
    uint32_t pad[12];    // pad[0]: hash of the codebook the index was built for
};
static_assert(sizeof(IndexHeader) == 64, "index header is 64 bytes");

// byte offsets inside the index buffer
constexpr size_t kIdxOffsets = 64;                                   // uint16[kCells + 1]
constexpr size_t kIdxEntries = 64 + ((size_t(kCells + 1) * 2 + 15) / 16) * 16;  // uint32[] pairs
constexpr size_t kIdxBytes = kIdxEntries + size_t(kMaxPairs) * 4;
// shared-memory image: offsets + entries (without the header)
constexpr size_t kIdxSmemOffsetsBytes = kIdxEntries - kIdxOffsets;

}  // namespace nsnq
