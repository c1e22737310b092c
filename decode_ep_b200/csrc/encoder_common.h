// Host-side pieces shared by the two EPK1 encoders (the multithreaded host encoder and the CUDA
// encoder): table fitting (12-bit for format version 1, 8-bit with rare symbols escaped for version 2),
// the sampled storage estimate, the raw-bit and tile-size choices and the blob's metadata sections. Both encoders call these, so every decision that fixes the blob's
// bytes is taken by the same code.
#pragma once

#include <algorithm>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <vector>

#include "capi_internal.h"
#include "entropack.h"
#include "epk_format.h"

namespace epk {
namespace enc {

inline float bf16_bits_to_float(uint16_t h) {
    uint32_t u = uint32_t(h) << 16;
    float f;
    std::memcpy(&f, &u, 4);
    return f;
}

inline uint16_t float_to_bf16_rne(float f) {
    uint32_t u;
    std::memcpy(&u, &f, 4);
    uint32_t rounding = 0x7FFFu + ((u >> 16) & 1u);  // ties go to the even upper half
    return uint16_t((u + rounding) >> 16);           // inputs here are finite and non-negative
}

// Smallest r in [0, 12] with 8 * 2^r >= alpha: the raw low bits per coordinate.
inline int raw_bits_for(float alpha) {
    int r = 0;
    while (r < 12 && 8.0 * double(int64_t(1) << r) < double(alpha)) ++r;
    return r;
}

// Tile rounds G for a tensor of NG groups. The decode runs one tile per warp at a time, on 148 SMs x
// 32 warps of a B200. With fixed 16-round tiles, a tensor's last wave of tiles can be nearly empty: it
// then runs at the latency of a lone tile. For tensors that fill at least half a wave, G is chosen in
// [12, 24] so that the tiles fill a whole number of waves. Smaller tensors keep G = 16.
inline uint32_t auto_rounds_per_tile(int64_t NG) {
    const double slots = 148.0 * 32.0;
    const double t16 = std::ceil(double(NG) / 512.0);
    if (t16 < 0.5 * slots) return 16;
    const double waves = std::max(1.0, std::floor(t16 / slots + 0.25));
    const double g = std::ceil(double(NG) / (32.0 * slots * waves));
    return uint32_t(std::min(24.0, std::max(12.0, g)));
}

using Counts = std::vector<uint64_t>;  // [kNumCtx][128]

// Normalisation to a total of `scale` (4096 or 256): f = max(1, floor(scale n_s / n)) for present
// symbols. The rounding gap is closed at the largest frequency, or in steps of whole units when there is
// too much. No f exceeds scale - 1: a single present symbol gets scale - 1, and its neighbour (s + 1, or
// s - 1 at the alphabet's end) gets 1.
inline void normalize(const uint64_t* cnt, int A, uint32_t scale, uint32_t* f) {
    uint64_t total = 0;
    int present = 0;
    for (int s = 0; s < A; ++s) { total += cnt[s]; present += cnt[s] != 0; f[s] = 0; }
    if (!present) return;
    if (present == 1) {
        for (int s = 0; s < A; ++s)
            if (cnt[s]) { f[s] = scale - 1; f[s + 1 < A ? s + 1 : s - 1] = 1; }
        return;
    }
    int64_t sum = 0;
    for (int s = 0; s < A; ++s) {
        if (!cnt[s]) continue;
        uint64_t q = cnt[s] * uint64_t(scale) / total;
        f[s] = q ? uint32_t(q) : 1u;
        sum += f[s];
    }
    int64_t d = int64_t(scale) - sum;
    while (d) {
        int best = -1;
        for (int s = 0; s < A; ++s) if (f[s] && (best < 0 || f[s] > f[best])) best = s;
        if (d > 0) { f[best] += uint32_t(d); d = 0; }
        else {
            int64_t take = std::min<int64_t>(-d, int64_t(f[best]) - 1);
            f[best] -= uint32_t(take);
            d += take;
        }
    }
}

// Version 2: the counts of rare symbols move onto their escape symbol (index 63 of the symbol's coset
// half in START, 63 elsewhere). Rare: seen in fewer than 1/2^kEscShift of the context's coordinates; hi in
// [-2, 2] (idx 29..33) is never escaped, so an escaped coordinate always has magnitude class 1.
inline void escape_rare(Counts& c) {
    for (int k = 0; k < kNumCtx; ++k) {
        const int A = k == 0 ? 128 : 64;
        uint64_t* n = &c[size_t(k) * 128];
        uint64_t total = 0;
        for (int s = 0; s < A; ++s) total += n[s];
        for (int s = 0; s < A; ++s) {
            const int idx = s & 63;
            if (idx == kEscIdx || (idx >= 29 && idx <= 33) || n[s] == 0) continue;
            if ((n[s] << kEscShift) < total) {
                n[(s & 64) | kEscIdx] += n[s];
                n[s] = 0;
            }
        }
    }
}

// The counts the tables of format `version` are fitted to.
inline Counts prepared_counts(const Counts& raw, int version) {
    Counts c = raw;
    if (version == 2) escape_rare(c);
    return c;
}

struct Tables {
    int version = 1, bits = kProbBits;
    uint32_t f[kNumCtx][128];
    uint32_t cum[kNumCtx][128];
    int lo[kNumCtx], cnt[kNumCtx];
    uint64_t nsym = 0;

    // c: prepared counts (prepared_counts).
    void build(const Counts& c, int ver) {
        version = ver;
        bits = prob_bits_of_version(ver);
        nsym = 0;
        for (int k = 0; k < kNumCtx; ++k) {
            int A = k == 0 ? 128 : 64;
            normalize(&c[size_t(k) * 128], A, 1u << bits, f[k]);
            for (int s = A; s < 128; ++s) f[k][s] = 0;
            int first = -1, last = -1;
            for (int s = 0; s < A; ++s) if (f[k][s]) { if (first < 0) first = s; last = s; }
            lo[k] = first < 0 ? 0 : first;
            cnt[k] = first < 0 ? 0 : last - first + 1;
            nsym += uint64_t(cnt[k]);
            uint32_t acc = 0;
            for (int s = 0; s < 128; ++s) { cum[k][s] = acc; acc += f[k][s]; }
        }
    }
    uint64_t serialized_bytes() const { return 2 * kNumCtx + (uint64_t(bits) * nsym + 7) / 8; }
    void serialize(uint8_t* out) const {
        for (int k = 0; k < kNumCtx; ++k) { out[k] = uint8_t(lo[k]); out[kNumCtx + k] = uint8_t(cnt[k]); }
        uint8_t* bytes = out + 2 * kNumCtx;
        uint64_t pos = 0;
        for (int k = 0; k < kNumCtx; ++k)
            for (int s = lo[k]; s < lo[k] + cnt[k]; ++s, pos += uint64_t(bits)) {
                uint32_t v = f[k][s];
                uint32_t word = v << (pos & 7);  // 12 + 7 bits fit in three bytes
                bytes[pos >> 3] |= uint8_t(word);
                if (word >> 8) bytes[(pos >> 3) + 1] |= uint8_t(word >> 8);
                if (word >> 16) bytes[(pos >> 3) + 2] |= uint8_t(word >> 16);
            }
    }
    // The table symbol coded for `sym` of context k: itself, or its escape when the tables give it no
    // frequency (a rare symbol of version 2).
    int coded(int k, int sym) const { return f[k][sym] ? sym : ((sym & 64) | kEscIdx); }
};

// Storage estimate in bytes from the symbol counts of a row sample: the ideal code length under the
// tables fitted to the sample, plus escapes and raw bits, scaled to the whole tensor, plus the exact
// metadata and 104 bytes per tile for the final states (their low half carries payload).
inline double estimate_from_counts(const Counts& raw, int version, int r, int64_t Rs, int64_t gpr, int64_t NG,
                                   int64_t M, uint32_t T) {
    const Counts total = prepared_counts(raw, version);
    Tables tab;
    tab.build(total, version);
    uint64_t n_esc = 0;
    for (int k = 0; k < kNumCtx; ++k) n_esc += total[size_t(k) * 128 + kEscIdx] + (k == 0 ? total[64 + kEscIdx] : 0);
    double bits = 0.0;
    for (int k = 0; k < kNumCtx; ++k)
        for (int sy = tab.lo[k]; sy < tab.lo[k] + tab.cnt[k]; ++sy) {
            uint64_t n = total[size_t(k) * 128 + sy];
            if (n) bits += double(n) * (double(tab.bits) - std::log2(double(tab.f[k][sy])));
        }
    double ng_s = double(Rs * gpr);
    bits += 16.0 * double(n_esc) + 8.0 * double(r) * ng_s;
    double bits_full = bits * double(NG) / ng_s;
    double meta = double(kHeaderBytes + pad16(2 * uint64_t(M)) + pad16(tab.serialized_bytes()) +
                         pad16(4 * (uint64_t(T) + 1)) + uint64_t(T) * (128 - 32 + 8));
    return meta + std::ceil(bits_full / 8.0);
}

// Section offsets of a blob with `payload_bytes` of tile payload.
struct BlobLayout {
    uint64_t off_scales, off_tables, off_offsets, off_payload, total;
};

inline BlobLayout blob_layout(int64_t rows, const Tables& tab, uint32_t T, uint64_t payload_bytes) {
    BlobLayout L;
    L.off_scales = kHeaderBytes;
    L.off_tables = L.off_scales + pad16(2 * uint64_t(rows));
    L.off_offsets = L.off_tables + pad16(tab.serialized_bytes());
    L.off_payload = L.off_offsets + pad16(4 * (uint64_t(T) + 1));
    L.total = L.off_payload + payload_bytes;
    return L;
}

// Writes every section but the payload into a zeroed blob of L.total bytes: header, scales, tables
// and tile offsets (start[j] = payload byte offset of tile j, start[T] = payload size; esc[j] marks
// tiles holding an escape). The CRC field is left zero; finish_crc fills it once the metadata is final.
inline void write_metadata(uint8_t* blob, const BlobLayout& L, ep_dtype dt, int r, int64_t rows, int64_t cols,
                           float alpha, uint32_t G, uint32_t T, const uint16_t* sbits, const Tables& tab,
                           const uint64_t* start, const uint8_t* esc) {
    std::memcpy(blob, "EPK1", 4);
    wr16(blob + 4, uint32_t(tab.version));
    blob[6] = uint8_t(dt);
    blob[7] = uint8_t(r);
    wr32(blob + 8, uint32_t(rows));
    wr32(blob + 12, uint32_t(cols));
    uint32_t abits;
    std::memcpy(&abits, &alpha, 4);
    wr32(blob + 16, abits);
    wr16(blob + 20, G);
    blob[22] = kLanes;
    wr32(blob + 24, T);
    wr32(blob + 28, uint32_t(L.off_scales));
    wr32(blob + 32, uint32_t(L.off_tables));
    wr32(blob + 36, uint32_t(L.off_offsets));
    wr32(blob + 40, uint32_t(L.off_payload));
    wr64(blob + 48, L.total);
    for (int64_t i = 0; i < rows; ++i) wr16(blob + L.off_scales + 2 * i, sbits[size_t(i)]);
    tab.serialize(blob + L.off_tables);
    for (uint32_t j = 0; j < T; ++j)
        wr32(blob + L.off_offsets + 4ull * j, uint32_t(start[j] / 16) | (esc[j] ? 0x80000000u : 0u));
    wr32(blob + L.off_offsets + 4ull * T, uint32_t(start[T] / 16));
}

// CRC-32 of the metadata sections, with the CRC field itself still zero.
inline void finish_crc(uint8_t* blob, const BlobLayout& L) { wr32(blob + 56, crc32(blob, L.off_payload)); }

}  // namespace enc
}  // namespace epk
