// C-ABI plumbing of libentropack: error reporting, CRC-32, full blob validation (ep_blob_info).
#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <mutex>
#include <string>

#include <cuda_runtime.h>

#include "capi_internal.h"
#include "entropack.h"
#include "epk_format.h"

namespace epk {

namespace {
thread_local std::string g_last_error;

struct CrcTable {
    uint32_t t[256];
    CrcTable() {
        for (uint32_t i = 0; i < 256; ++i) {
            uint32_t c = i;
            for (int k = 0; k < 8; ++k) c = (c & 1) ? 0xEDB88320u ^ (c >> 1) : c >> 1;
            t[i] = c;
        }
    }
};
const CrcTable kCrc;
}  // namespace

ep_status fail(ep_status st, const char* fmt, ...) {
    char buf[512];
    va_list ap;
    va_start(ap, fmt);
    std::vsnprintf(buf, sizeof(buf), fmt, ap);
    va_end(ap);
    g_last_error = buf;
    return st;
}

void clear_error() { g_last_error.clear(); }

uint32_t crc32(const uint8_t* p, uint64_t n) {
    uint32_t c = 0xFFFFFFFFu;
    for (uint64_t i = 0; i < n; ++i) c = kCrc.t[(c ^ p[i]) & 0xFFu] ^ (c >> 8);
    return c ^ 0xFFFFFFFFu;
}

cudaError_t scratch_pool(cudaMemPool_t* out) {
    static std::mutex mu;
    static cudaMemPool_t pools[64];
    static bool made[64] = {false};
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> lk(mu);
    if (!made[dev]) {
        cudaMemPoolProps props = {};
        props.allocType = cudaMemAllocationTypePinned;
        props.location.type = cudaMemLocationTypeDevice;
        props.location.id = dev;
        e = cudaMemPoolCreate(&pools[dev], &props);
        if (e != cudaSuccess) return e;
        uint64_t keep = uint64_t(1) << 30;
        e = cudaMemPoolSetAttribute(pools[dev], cudaMemPoolAttrReleaseThreshold, &keep);
        if (e != cudaSuccess) return e;
        made[dev] = true;
    }
    *out = pools[dev];
    return cudaSuccess;
}

ep_status validate_blob(const uint8_t* p, uint64_t bytes) {
    if (!p) return fail(EP_ERR_ARG, "NULL blob");
    if (bytes < kHeaderBytes) return fail(EP_ERR_CORRUPT, "blob shorter than its 64-byte header");
    Header h;
    if (!parse_header(p, h)) return fail(EP_ERR_CORRUPT, "malformed EPK1 header");
    if (h.total != bytes) return fail(EP_ERR_CORRUPT, "header says %llu bytes, have %llu", (unsigned long long)h.total,
                                      (unsigned long long)bytes);
    // Tables: lo/cnt bounds, then the frequencies (12-bit in version 1, 8-bit in version 2).
    const int fbits = prob_bits_of_version(h.version);
    const uint32_t scale = 1u << fbits;
    const uint8_t* tb = p + h.off_tables;
    uint64_t avail = h.off_offsets - h.off_tables, nsym = 0;
    if (avail < 2 * kNumCtx) return fail(EP_ERR_CORRUPT, "tables section too short");
    for (int c = 0; c < kNumCtx; ++c) {
        int lo = tb[c], cnt = tb[kNumCtx + c];
        if ((cnt == 0 && lo != 0) || lo + cnt > (c == 0 ? 128 : 64)) return fail(EP_ERR_CORRUPT, "context %d out of range", c);
        nsym += uint64_t(cnt);
    }
    uint64_t used = 2 * kNumCtx + (uint64_t(fbits) * nsym + 7) / 8;
    if (pad16(used) != avail) return fail(EP_ERR_CORRUPT, "tables section size mismatch");
    const uint8_t* bits = tb + 2 * kNumCtx;
    uint64_t pos = 0;
    for (int c = 0; c < kNumCtx; ++c) {
        int cnt = tb[kNumCtx + c];
        uint32_t sum = 0, fmax = 0;
        for (int k = 0; k < cnt; ++k, pos += uint64_t(fbits)) {
            uint32_t v = 0;
            for (int b = 0; b < fbits; ++b) v |= uint32_t((bits[(pos + b) >> 3] >> ((pos + b) & 7)) & 1u) << b;
            sum += v;
            fmax = v > fmax ? v : fmax;
        }
        if (cnt == 1) return fail(EP_ERR_CORRUPT, "context %d: a single symbol must be stored as %u + 1", c, scale - 1);
        if (cnt >= 2 && (sum != scale || fmax > scale - 1))
            return fail(EP_ERR_CORRUPT, "context %d: frequencies do not sum to %u", c, scale);
    }
    // Tile offsets: start at 0, non-decreasing, last one ends the blob.
    uint64_t prev = 0;
    for (uint64_t j = 0; j <= h.T; ++j) {
        uint32_t e = rd32(p + h.off_offsets + 4 * j);
        uint64_t start = uint64_t(e & 0x7FFFFFFFu) * 16;
        if ((j == 0 && start != 0) || start < prev) return fail(EP_ERR_CORRUPT, "tile offset %llu out of order", (unsigned long long)j);
        if (j == h.T && ((e >> 31) || h.off_payload + start != bytes)) return fail(EP_ERR_CORRUPT, "payload size mismatch");
        prev = start;
    }
    // CRC-32 of the metadata, with the crc field read as zero.
    uint32_t c = 0xFFFFFFFFu;
    for (uint64_t i = 0; i < h.off_payload; ++i) {
        uint8_t byte = (i >= 56 && i < 60) ? 0 : p[i];
        c = kCrc.t[(c ^ byte) & 0xFFu] ^ (c >> 8);
    }
    if ((c ^ 0xFFFFFFFFu) != rd32(p + 56)) return fail(EP_ERR_CORRUPT, "metadata CRC mismatch");
    return EP_OK;
}

}  // namespace epk

using namespace epk;

extern "C" ep_status ep_blob_info(const uint8_t* blob, size_t blob_bytes, ep_dtype* dt, int64_t* rows, int64_t* cols,
                                  double* actual_bpp) {
    clear_error();
    ep_status st = validate_blob(blob, blob_bytes);
    if (st != EP_OK) return st;
    Header h;
    parse_header(blob, h);
    if (dt) *dt = ep_dtype(h.dtype);
    if (rows) *rows = h.M;
    if (cols) *cols = h.N;
    if (actual_bpp) *actual_bpp = 8.0 * double(blob_bytes) / (double(h.M) * double(h.N));
    return EP_OK;
}

extern "C" const char* ep_status_string(ep_status st) {
    switch (st) {
        case EP_OK: return "ok";
        case EP_ERR_ARG: return "invalid argument";
        case EP_ERR_DTYPE: return "unsupported dtype";
        case EP_ERR_SHAPE: return "unsupported shape (need 2-D, cols a multiple of 8)";
        case EP_ERR_TARGET: return "target_bpp must be finite and in [0.001, 11]";
        case EP_ERR_NONFINITE: return "non-finite input";
        case EP_ERR_CORRUPT: return "corrupt blob";
        case EP_ERR_CUDA: return "CUDA error";
        case EP_ERR_NOMEM: return "out of memory";
        case EP_ERR_BUFFER: return "buffer too small or misaligned";
    }
    return "unknown status";
}

extern "C" const char* ep_last_error(void) { return g_last_error.c_str(); }
