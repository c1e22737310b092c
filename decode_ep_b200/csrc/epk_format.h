// Internal constants and the host-side header reader of the EPK1 blob, used by the host encoder,
// the C ABI and the decode launcher. The byte layout:
//   header (64 B) | scales M x bf16 | tables: lo[9], cnt[9], frequencies packed LSB-first (12-bit in
//   format version 1, 8-bit in version 2) |
//   tile offsets (T+1) x u32 (start/16 | has_esc<<31) | payload: per tile 32 x u32 states,
//   raw low bits (groups*r bytes, padded to 4), u16 word stream, zero padding to 16.
// Every section starts 16-byte aligned; all fields are little-endian.
#pragma once

#include <cstddef>
#include <cstdint>
#include <cstring>

namespace epk {

constexpr uint32_t kHeaderBytes = 64;
constexpr int kLanes = 32;
constexpr int kNumCtx = 9;
// Format version 1: 12-bit tables, the state renormalised after every symbol.
constexpr int kProbBits = 12;
constexpr uint32_t kProbScale = 1u << kProbBits;  // 4096
// Format version 2: 8-bit tables, the state renormalised after every pair of symbols; rare symbols are
// sent as escapes (a symbol seen in fewer than 1/2^kEscShift of its context's coordinates, other than
// hi in [-2, 2]), and a round's escape words follow its last pair.
constexpr int kProbBitsV2 = 8;
constexpr uint32_t kProbScaleV2 = 1u << kProbBitsV2;  // 256
constexpr int kEscShift = 14;
constexpr uint32_t kRansL = 1u << 16;             // state lower bound; 16-bit refills
constexpr int kEscIdx = 63;
constexpr int kMaxG = 1024;

inline int prob_bits_of_version(int version) { return version == 1 ? kProbBits : kProbBitsV2; }

inline uint64_t pad16(uint64_t n) { return (n + 15) & ~uint64_t(15); }
inline uint64_t pad4(uint64_t n) { return (n + 3) & ~uint64_t(3); }

inline uint32_t rd16(const uint8_t* p) { return uint32_t(p[0]) | (uint32_t(p[1]) << 8); }
inline uint32_t rd32(const uint8_t* p) {
    return uint32_t(p[0]) | (uint32_t(p[1]) << 8) | (uint32_t(p[2]) << 16) | (uint32_t(p[3]) << 24);
}
inline uint64_t rd64(const uint8_t* p) { return uint64_t(rd32(p)) | (uint64_t(rd32(p + 4)) << 32); }
inline void wr16(uint8_t* p, uint32_t v) { p[0] = uint8_t(v); p[1] = uint8_t(v >> 8); }
inline void wr32(uint8_t* p, uint32_t v) {
    p[0] = uint8_t(v); p[1] = uint8_t(v >> 8); p[2] = uint8_t(v >> 16); p[3] = uint8_t(v >> 24);
}
inline void wr64(uint8_t* p, uint64_t v) { wr32(p, uint32_t(v)); wr32(p + 4, uint32_t(v >> 32)); }

inline int elem_bytes(int dtype) {
    switch (dtype) {
        case 1: case 2: return 2;
        case 3: return 4;
        case 4: case 5: return 1;
        default: return 0;
    }
}

// Header fields as the decoder needs them.
struct Header {
    int version = 0, dtype = 0, r = 0, G = 0;
    uint32_t M = 0, N = 0, T = 0;
    float alpha = 0.f;
    uint32_t off_scales = 0, off_tables = 0, off_offsets = 0, off_payload = 0;
    uint64_t total = 0;
    uint64_t groups() const { return uint64_t(M) * N / 8; }
};

// Parses and checks the 64-byte header alone (no sections). Returns false if malformed.
inline bool parse_header(const uint8_t* p, Header& h) {
    if (std::memcmp(p, "EPK1", 4) != 0) return false;
    h.version = int(rd16(p + 4));
    if (h.version != 1 && h.version != 2) return false;
    h.dtype = p[6];
    h.r = p[7];
    h.M = rd32(p + 8);
    h.N = rd32(p + 12);
    uint32_t ab = rd32(p + 16);
    std::memcpy(&h.alpha, &ab, 4);
    h.G = int(rd16(p + 20));
    if (p[22] != kLanes || p[23] != 0) return false;
    h.T = rd32(p + 24);
    h.off_scales = rd32(p + 28);
    h.off_tables = rd32(p + 32);
    h.off_offsets = rd32(p + 36);
    h.off_payload = rd32(p + 40);
    h.total = rd64(p + 48);
    if (!elem_bytes(h.dtype) || h.r > 12 || h.M < 1 || h.N < 8 || h.N % 8) return false;
    if (h.groups() > 0xFFFFFFFFull) return false;
    if (!(h.alpha > 0.f) || !(h.alpha < 3.4e38f) || h.G < 1 || h.G > kMaxG) return false;
    uint64_t per_tile = 32ull * uint64_t(h.G);
    if (h.T != (h.groups() + per_tile - 1) / per_tile) return false;
    if (h.off_scales != kHeaderBytes || h.off_tables != h.off_scales + pad16(2ull * h.M)) return false;
    // The tables section is at least pad16(18) bytes: the decode kernel reads lo[9] and cnt[9] unchecked.
    if (h.off_offsets < h.off_tables + 32 || (h.off_offsets & 15) ||
        h.off_payload != h.off_offsets + pad16(4ull * (uint64_t(h.T) + 1)) || h.off_payload > h.total)
        return false;
    return true;
}

}  // namespace epk
