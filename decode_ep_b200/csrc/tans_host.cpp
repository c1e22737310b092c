// Lossless tile-ANS (EPL1): the multithreaded host encoder, full blob validation, and the ABI entries
// ep_tans_compress and ep_tans_info. The decode kernel is in tans_decode.cuh.
//
// The EntroPack README's Config table lists TileANSConfig(): lossless compression of BF16, FP16, FP32, FP8
// and INT8 tensors, with a ratio that depends on the data. Here the raw bit patterns of the elements are
// cut into byte planes (byte j of every element); a plane whose values cluster (the sign and exponent byte
// of floating-point weights) is rANS-coded under its own 12-bit table, the others are stored verbatim.
#include <algorithm>
#include <atomic>
#include <cmath>
#include <cstdlib>
#include <cstring>
#include <functional>
#include <mutex>
#include <thread>
#include <vector>

#include "capi_internal.h"
#include "encoder_common.h"
#include "entropack.h"
#include "tans_format.h"

namespace epk {
namespace tans {
namespace {

void parallel_for(int64_t n, int threads, const std::function<void(int64_t, int64_t)>& fn) {
    if (n <= 0) return;
    const int nt = int(std::min<int64_t>(threads, n));
    if (nt <= 1) {
        fn(0, n);
        return;
    }
    const int64_t chunk = std::max<int64_t>(1, n / (int64_t(nt) * 8));
    std::atomic<int64_t> next{0};
    std::vector<std::thread> pool;
    pool.reserve(size_t(nt));
    for (int t = 0; t < nt; ++t)
        pool.emplace_back([&] {
            for (;;) {
                const int64_t b = next.fetch_add(chunk);
                if (b >= n) break;
                fn(b, std::min(n, b + chunk));
            }
        });
    for (auto& th : pool) th.join();
}

struct Model {
    int e = 0;
    bool coded[4] = {false, false, false, false};
    int lo[4] = {0}, cnt[4] = {0};
    uint32_t f[4][256] = {{0}};
    uint32_t cum[4][257] = {{0}};
};

// Per plane: counts over the whole tensor, the 12-bit normalisation, and the plane coded when its ideal
// coded size plus its table (4 + 2 cnt bytes) is at most 7 bits a byte.
Model fit(const uint8_t* data, uint64_t n, int e, int threads) {
    Model m;
    m.e = e;
    std::vector<uint64_t> counts(size_t(e) * 256, 0);
    std::mutex mu;
    parallel_for(int64_t(n), threads, [&](int64_t a, int64_t b) {
        std::vector<uint64_t> local(size_t(e) * 256, 0);
        for (int64_t i = a; i < b; ++i)
            for (int j = 0; j < e; ++j) ++local[size_t(j) * 256 + data[uint64_t(i) * uint64_t(e) + uint64_t(j)]];
        std::lock_guard<std::mutex> lk(mu);
        for (size_t k = 0; k < local.size(); ++k) counts[k] += local[k];
    });
    for (int j = 0; j < e; ++j) {
        const uint64_t* c = counts.data() + size_t(j) * 256;
        enc::normalize(c, 256, kScale, m.f[j]);
        if (n == 0) continue;
        int lo = 256, hi = -1;
        for (int s = 0; s < 256; ++s)
            if (m.f[j][s]) {
                lo = std::min(lo, s);
                hi = s;
            }
        double bits = 8.0 * (4 + 2 * (hi - lo + 1));
        for (int s = 0; s < 256; ++s)
            if (c[s]) bits += double(c[s]) * std::log2(double(kScale) / double(m.f[j][s]));
        if (bits <= 7.0 * double(n)) {
            m.coded[j] = true;
            m.lo[j] = lo;
            m.cnt[j] = hi - lo + 1;
            m.cum[j][0] = 0;
            for (int s = 0; s < 256; ++s) m.cum[j][s + 1] = m.cum[j][s] + m.f[j][s];
        }
    }
    return m;
}

// One tile (elements [i0, i0 + ne)): the decode order run backwards (rounds, then coded planes, then lanes,
// all descending), then the tile's layout: states, raw planes padded to 4 bytes, the words in reverse push
// order, zeros to a 16-byte multiple.
std::vector<uint8_t> encode_tile(const uint8_t* data, uint64_t i0, uint64_t ne, const Model& m) {
    const int e = m.e;
    bool any = false;
    for (int j = 0; j < e; ++j) any = any || m.coded[j];
    uint32_t x[kLanes];
    for (uint32_t L = 0; L < kLanes; ++L) x[L] = 1u << 16;
    std::vector<uint16_t> words;
    const int64_t R = int64_t((ne + 31) / 32);
    for (int64_t k = R - 1; k >= 0; --k)
        for (int j = e - 1; j >= 0; --j) {
            if (!m.coded[j]) continue;
            for (int L = int(kLanes) - 1; L >= 0; --L) {
                const uint64_t i = 32 * uint64_t(k) + uint64_t(L);
                if (i >= ne) continue;
                const uint32_t s = data[(i0 + i) * uint64_t(e) + uint64_t(j)];
                const uint32_t f = m.f[j][s], c = m.cum[j][s];
                if (uint64_t(x[L]) >= (uint64_t(f) << 20)) {
                    words.push_back(uint16_t(x[L] & 0xFFFFu));
                    x[L] >>= 16;
                }
                x[L] = (x[L] / f) * kScale + (x[L] % f) + c;
            }
        }
    uint64_t size = any ? 128 : 0;
    for (int j = 0; j < e; ++j)
        if (!m.coded[j]) size += pad4(ne);
    size = pad16(size + 2 * uint64_t(words.size()));
    std::vector<uint8_t> out(size_t(size), 0);
    uint64_t o = 0;
    if (any) {
        for (uint32_t L = 0; L < kLanes; ++L) wr32(out.data() + 4 * L, x[L]);
        o = 128;
    }
    for (int j = 0; j < e; ++j) {
        if (m.coded[j]) continue;
        for (uint64_t i = 0; i < ne; ++i) out[size_t(o + i)] = data[(i0 + i) * uint64_t(e) + uint64_t(j)];
        o += pad4(ne);
    }
    for (size_t w = 0; w < words.size(); ++w) wr16(out.data() + o + 2 * w, words[words.size() - 1 - w]);
    return out;
}

}  // namespace

// Full validation of an EPL1 blob: header, CRC, tables, tile offsets. Fills h.
ep_status validate_tans(const uint8_t* p, uint64_t bytes, Header& h) {
    if (!p) return fail(EP_ERR_ARG, "NULL blob");
    if (bytes < kHeaderBytes) return fail(EP_ERR_CORRUPT, "blob shorter than its 96-byte EPL1 header");
    if (!parse_tans_header(p, h)) return fail(EP_ERR_CORRUPT, "malformed EPL1 header");
    if (h.total != bytes) return fail(EP_ERR_CORRUPT, "header says %llu bytes, have %llu", (unsigned long long)h.total,
                                      (unsigned long long)bytes);
    std::vector<uint8_t> head(p, p + h.off_payload);
    std::memset(head.data() + 80, 0, 4);
    if (crc32(head.data(), h.off_payload) != h.crc) return fail(EP_ERR_CORRUPT, "EPL1 metadata CRC mismatch");
    uint64_t o = h.off_tables;
    for (int j = 0; j < h.e; ++j) {
        if (!((h.mask >> j) & 1)) continue;
        if (o + 4 > h.off_offsets) return fail(EP_ERR_CORRUPT, "EPL1 tables overrun");
        const uint32_t lo = rd16(p + o), cnt = rd16(p + o + 2);
        if (cnt < 2 || lo + cnt > 256 || o + 4 + 2ull * cnt > h.off_offsets)
            return fail(EP_ERR_CORRUPT, "EPL1 table of plane %d out of range", j);
        uint32_t sum = 0;
        for (uint32_t s = 0; s < cnt; ++s) {
            const uint32_t f = rd16(p + o + 4 + 2 * s);
            if (f >= kScale) return fail(EP_ERR_CORRUPT, "EPL1 frequency out of range");
            sum += f;
        }
        if (sum != kScale) return fail(EP_ERR_CORRUPT, "EPL1 table of plane %d does not sum to 4096", j);
        o += 4 + 2ull * cnt;
    }
    const uint8_t* off = p + h.off_offsets;
    const uint64_t payload = bytes - h.off_payload;
    if (rd32(off) != 0 || 16ull * rd32(off + 4ull * h.T) != payload)
        return fail(EP_ERR_CORRUPT, "EPL1 tile offsets do not span the payload");
    for (uint64_t t = 0; t < h.T; ++t)
        if (rd32(off + 4 * (t + 1)) < rd32(off + 4 * t)) return fail(EP_ERR_CORRUPT, "EPL1 tile offsets not ascending");
    return EP_OK;
}

}  // namespace tans
}  // namespace epk

using namespace epk;

extern "C" ep_status ep_tans_compress(const void* data, ep_dtype dtype, int ndim, const int64_t* dims,
                                      uint32_t elems_per_lane, int threads, uint8_t** blob_out, size_t* bytes_out) {
    clear_error();
    if (!blob_out || !bytes_out || ndim < 0 || ndim > tans::kMaxDims || (ndim > 0 && !dims))
        return fail(EP_ERR_ARG, "ep_tans_compress: bad arguments");
    const int e = elem_bytes(int(dtype));
    if (e <= 0) return fail(EP_ERR_DTYPE, "ep_tans_compress: unknown dtype %d", int(dtype));
    const uint32_t K = elems_per_lane ? elems_per_lane : tans::kDefaultK;
    if (K > tans::kMaxK) return fail(EP_ERR_ARG, "ep_tans_compress: elems_per_lane %u above %u", K, tans::kMaxK);
    uint64_t n = 1;
    for (int d = 0; d < ndim; ++d) {
        if (dims[d] < 0 || dims[d] > 0xFFFFFFFFll) return fail(EP_ERR_SHAPE, "ep_tans_compress: dim %d out of range", d);
        n *= uint64_t(dims[d]);
    }
    if (n && !data) return fail(EP_ERR_ARG, "ep_tans_compress: NULL data");
    if (threads <= 0) threads = int(std::max(1u, std::thread::hardware_concurrency()));
    const uint8_t* src = static_cast<const uint8_t*>(data);
    const uint64_t per_tile = uint64_t(tans::kLanes) * K;
    const uint64_t T = (n + per_tile - 1) / per_tile;
    if (T > 0xFFFFFFFFull) return fail(EP_ERR_SHAPE, "ep_tans_compress: too many tiles");
    const auto m = tans::fit(src, n, e, threads);
    std::vector<std::vector<uint8_t>> tiles(static_cast<size_t>(T));
    tans::parallel_for(int64_t(T), threads, [&](int64_t a, int64_t b) {
        for (int64_t t = a; t < b; ++t) {
            const uint64_t i0 = uint64_t(t) * per_tile, ne = std::min<uint64_t>(per_tile, n - i0);
            tiles[size_t(t)] = tans::encode_tile(src, i0, ne, m);
        }
    });
    uint64_t tables = 0;
    for (int j = 0; j < e; ++j)
        if (m.coded[j]) tables += 4 + 2ull * uint64_t(m.cnt[j]);
    const uint64_t off_tables = tans::kHeaderBytes, off_offsets = pad16(off_tables + tables);
    const uint64_t off_payload = pad16(off_offsets + 4 * (T + 1));
    uint64_t payload = 0;
    for (const auto& t : tiles) payload += t.size();
    if (payload / 16 > 0xFFFFFFFFull || off_payload > 0xFFFFFFFFull)
        return fail(EP_ERR_SHAPE, "ep_tans_compress: blob too large");
    const uint64_t total = off_payload + payload;
    uint8_t* p = static_cast<uint8_t*>(std::calloc(size_t(total), 1));
    if (!p) return fail(EP_ERR_NOMEM, "ep_tans_compress: %llu bytes", (unsigned long long)total);
    std::memcpy(p, "EPL1", 4);
    wr16(p + 4, 1);
    p[6] = uint8_t(dtype);
    p[7] = uint8_t(ndim);
    wr64(p + 8, n);
    for (int d = 0; d < ndim; ++d) wr32(p + 16 + 4 * d, uint32_t(dims[d]));
    wr16(p + 48, K);
    uint32_t mask = 0;
    for (int j = 0; j < e; ++j) mask |= uint32_t(m.coded[j]) << j;
    p[50] = uint8_t(mask);
    p[51] = uint8_t(tans::kLanes);
    wr32(p + 52, uint32_t(T));
    wr32(p + 56, uint32_t(off_tables));
    wr32(p + 60, uint32_t(off_offsets));
    wr32(p + 64, uint32_t(off_payload));
    wr64(p + 72, total);
    uint64_t o = off_tables;
    for (int j = 0; j < e; ++j) {
        if (!m.coded[j]) continue;
        wr16(p + o, uint32_t(m.lo[j]));
        wr16(p + o + 2, uint32_t(m.cnt[j]));
        for (int s = 0; s < m.cnt[j]; ++s) wr16(p + o + 4 + 2 * s, m.f[j][m.lo[j] + s]);
        o += 4 + 2ull * uint64_t(m.cnt[j]);
    }
    uint64_t at = 0;
    for (uint64_t t = 0; t < T; ++t) {
        wr32(p + off_offsets + 4 * t, uint32_t(at / 16));
        std::memcpy(p + off_payload + at, tiles[size_t(t)].data(), tiles[size_t(t)].size());
        at += tiles[size_t(t)].size();
    }
    wr32(p + off_offsets + 4 * T, uint32_t(at / 16));
    wr32(p + 80, crc32(p, off_payload));  // the crc field is still zero here
    *blob_out = p;
    *bytes_out = size_t(total);
    return EP_OK;
}

extern "C" ep_status ep_tans_info(const uint8_t* blob, size_t blob_bytes, ep_dtype* dt, int* ndim, int64_t* dims,
                                  uint32_t* coded_mask, uint32_t* elems_per_lane) {
    clear_error();
    tans::Header h;
    const ep_status st = tans::validate_tans(blob, blob_bytes, h);
    if (st != EP_OK) return st;
    if (dt) *dt = ep_dtype(h.dtype);
    if (ndim) *ndim = h.ndim;
    if (dims)
        for (int d = 0; d < h.ndim; ++d) dims[d] = h.dims[d];
    if (coded_mask) *coded_mask = h.mask;
    if (elems_per_lane) *elems_per_lane = h.K;
    return EP_OK;
}
