// The EPL1 lossless tile-ANS blob: header layout and checks shared by the host encoder, the ABI and the
// decode launcher. Byte planes of the elements' raw bit patterns, each stored verbatim or rANS-coded under
// its own 12-bit table, in tiles of 32 interleaved lanes (EntroPack README, Config table: TileANSConfig,
// lossless, several dtypes).
#pragma once

#include <cstdint>

#include "epk_format.h"

namespace epk {
namespace tans {

constexpr uint32_t kHeaderBytes = 96;
constexpr int kMaxDims = 8;
constexpr uint32_t kLanes = 32;
constexpr uint32_t kProbBits = 12;
constexpr uint32_t kScale = 1u << kProbBits;
constexpr uint32_t kDefaultK = 128;  // elements per lane per tile: 4096 a tile
constexpr uint32_t kMaxK = 1024;

struct Header {
    int dtype = 0, e = 0, ndim = 0;
    uint32_t dims[kMaxDims] = {0};
    uint64_t n = 0;       // elements
    uint32_t K = 0;       // elements per lane per tile
    uint32_t mask = 0;    // bit j: byte plane j is rANS-coded
    uint32_t T = 0;       // tiles
    uint32_t off_tables = 0, off_offsets = 0, off_payload = 0;
    uint64_t total = 0;
    uint32_t crc = 0;
    uint64_t per_tile() const { return uint64_t(kLanes) * K; }
    int coded_planes() const { return __builtin_popcount(mask); }
};

// Field checks of the 96-byte header (sizes, ranges, section order); tables, offsets and the CRC are
// checked by validate_tans against the whole blob.
inline bool parse_tans_header(const uint8_t* p, Header& h) {
    if (!(p[0] == 'E' && p[1] == 'P' && p[2] == 'L' && p[3] == '1') || rd16(p + 4) != 1) return false;
    h.dtype = p[6];
    h.e = elem_bytes(h.dtype);
    h.ndim = p[7];
    if (h.e <= 0 || h.ndim > kMaxDims || p[51] != kLanes) return false;
    h.n = rd64(p + 8);
    uint64_t prod = 1;
    for (int d = 0; d < kMaxDims; ++d) {
        h.dims[d] = rd32(p + 16 + 4 * d);
        if (d < h.ndim) {
            prod *= h.dims[d];
        } else if (h.dims[d] != 0) {
            return false;
        }
    }
    if (prod != h.n) return false;
    h.K = rd16(p + 48);
    h.mask = p[50];
    if (h.K < 1 || h.K > kMaxK || (h.mask >> h.e) != 0) return false;
    h.T = rd32(p + 52);
    if (uint64_t(h.T) != (h.n + h.per_tile() - 1) / h.per_tile()) return false;
    h.off_tables = rd32(p + 56);
    h.off_offsets = rd32(p + 60);
    h.off_payload = rd32(p + 64);
    h.total = rd64(p + 72);
    h.crc = rd32(p + 80);
    if (h.off_tables != kHeaderBytes || h.off_offsets < h.off_tables || h.off_offsets % 16 || h.off_payload % 16 ||
        uint64_t(h.off_payload) < uint64_t(h.off_offsets) + 4ull * (uint64_t(h.T) + 1) || h.off_payload > h.total)
        return false;
    return true;
}

}  // namespace tans
}  // namespace epk
