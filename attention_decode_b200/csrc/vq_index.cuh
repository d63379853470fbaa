// Layout of the nearest-codeword search index for 4-dimensional sub-vectors
// (2 bits/coordinate), shared by the builder and the encode kernel.
//
// The transformed coordinates are near N(0, 1) (NSN + Hadamard, gist.science
// "NSNQuant ...", Methodology §1-§2), so each coordinate is binned on a
// uniform grid: kNb bins per coordinate, the inner kNb-2 bins of width kW
// covering [-kR, kR) and two outer bins reaching to +-kOuter (every
// coordinate of w satisfies |w_i| <= ||w|| = sqrt(128) < kOuter). For every
// grid cell the index lists the codewords that can be nearest (or within the
// near-tie margin of the nearest) for some point of the cell, sorted by a
// lower bound of their squared distance over the cell. A codeword is left
// out only if another codeword is closer by a margin everywhere in the cell
// (expanded by kBoxEps), so the list's best codeword is the exact nearest.
#pragma once

#include <stdint.h>

namespace nsnq {

constexpr int kNb = 10;                           // bins per coordinate
constexpr float kR = 2.4f;                        // inner grid covers [-kR, kR)
constexpr float kW = 0.6f;                        // inner bin width
constexpr float kInvW = 1.0f / 0.6f;
constexpr float kBinBias = 2.4f / 0.6f + 1.0f;    // bin = floor(w / kW + kBinBias), clamped
constexpr double kOuter = 12.0;                   // outer bins end here (> sqrt(128))
constexpr double kBoxEps = 1e-3;                  // cell expansion covering fp32 error in w
constexpr int kCells = kNb * kNb * kNb * kNb;
constexpr int kMaxEntries = 65535;                // offsets are uint16
constexpr float kLbScale = 64.0f;                 // lower bounds stored as floor(lb * 64), <= 255
constexpr uint32_t kIndexMagic = 0x4e534e51u;     // "NSNQ"

// Near-tie rule of the fp32 search: a sub-vector whose two best distances
// are within kTieRel * d1 + kTieAbs is re-decided in fp64 (the fp32 error of
// a distance is ~1e-6 relative, so the band keeps a 20x margin). The index
// keeps every codeword that can come that close, so the rule sees all
// contenders.
constexpr float kTieRel = 2e-5f;
constexpr float kTieAbs = 1e-6f;

struct IndexHeader {
    uint32_t magic;
    uint32_t n_entries;  // total list entries
    uint32_t overflow;   // nonzero if the lists did not fit kMaxEntries
    uint32_t cells;
    uint32_t pad[12];
};
static_assert(sizeof(IndexHeader) == 64, "index header is 64 bytes");

// byte offsets inside the index buffer
constexpr size_t kIdxOffsets = 64;                                   // uint16[kCells + 1]
constexpr size_t kIdxEntries = 64 + ((size_t(kCells + 1) * 2 + 15) / 16) * 16;  // uint16[]
constexpr size_t kIdxBytes = kIdxEntries + size_t(kMaxEntries + 1) * 2;
// smem image: offsets + entries (without the header)
constexpr size_t kIdxSmemOffsetsBytes = kIdxEntries - kIdxOffsets;

}  // namespace nsnq
