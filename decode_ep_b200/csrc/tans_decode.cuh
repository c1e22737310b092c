// Lossless tile-ANS (EPL1) decode for sm_100a, and its ABI entry ep_tans_decompress_into. Included by
// decode.cu, so that it shares the device status word.
//
// One warp per tile, tiles dealt round-robin over the CTAs first. A round gives each lane one element:
// for each byte plane in order, a coded plane decodes one symbol from the lane's rANS state (the fused
// entry of slot x mod 4096 in the plane's shared table, then the lanes with x < 2^16 take the next words
// of the tile's stream in lane order), a raw plane reads its byte from the tile's raw section; the bytes
// make the element, which the lane stores. The whole round of a warp stores 32 consecutive elements.
#pragma once

namespace epk {
namespace dev {
namespace tansdev {

constexpr int kWarpsT = 32;
constexpr int kThreadsT = kWarpsT * 32;
constexpr uint32_t kEntries = 4096;                   // slots of a 12-bit table
constexpr uint32_t kTableBytesT = kEntries * 4;       // fused entries of one coded plane: 16 KB
constexpr uint32_t kScratchT = 4 * (256 + 257) * 4;   // f and cum of up to four planes

struct TParams {
    const uint8_t* blob;
    void* dst;
    uint64_t n;            // elements
    uint64_t payload_bytes;
    uint32_t K, T, mask;   // elements per lane per tile, tiles, coded planes
    uint32_t off_tables, off_offsets, off_payload;
};

// Fused entry: symbol (bits 24-31) | slot - cum (bits 12-23) | f (bits 0-11).
// Builds the tables of the coded planes: one warp per coded plane reads its frequencies and scans them into
// cum (a plane that does not sum to 4096 sets EP_DEV_BAD_TABLES); then every thread fills slots, finding
// each slot's symbol by an 8-step binary search over cum.
template <int E>
__device__ void build_tans_tables(const TParams& p, uint32_t* tables, uint32_t* scratch) {
    uint32_t* F = scratch;             // [4][256]
    uint32_t* cum = scratch + 4 * 256; // [4][257]
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    // The table of coded plane number c (the c-th set bit of the mask) starts after those before it.
    int c = 0;
    uint32_t o = p.off_tables;
    for (int j = 0; j < E; ++j) {
        if (!((p.mask >> j) & 1u)) continue;
        // Reads stay inside the tables section; a corrupt one leaves the plane without frequencies.
        const bool in = o + 4 <= p.off_offsets;
        const uint32_t lo = in ? uint32_t(p.blob[o]) | (uint32_t(p.blob[o + 1]) << 8) : 0u;
        const uint32_t cnt = in ? uint32_t(p.blob[o + 2]) | (uint32_t(p.blob[o + 3]) << 8) : 0u;
        if (warp == c) {
            uint32_t f[8], part = 0;
#pragma unroll
            for (int k = 0; k < 8; ++k) {
                const uint32_t s = 8 * lane + k;
                const uint32_t q = o + 4 + 2 * (s - lo);
                f[k] = (s >= lo && s < lo + cnt && q + 2 <= p.off_offsets)
                           ? uint32_t(p.blob[q]) | (uint32_t(p.blob[q + 1]) << 8)
                           : 0u;
                part += f[k];
            }
            uint32_t incl = part;
#pragma unroll
            for (int d = 1; d < 32; d <<= 1) {
                const uint32_t v = __shfl_up_sync(kFullMask, incl, d);
                if (lane >= d) incl += v;
            }
            uint32_t acc = incl - part;
#pragma unroll
            for (int k = 0; k < 8; ++k) {
                F[c * 256 + 8 * lane + k] = f[k];
                cum[c * 257 + 8 * lane + k] = acc;
                acc += f[k];
            }
            const uint32_t total = __shfl_sync(kFullMask, incl, 31);
            if (lane == 0) {
                cum[c * 257 + 256] = total;
                if (total != kEntries && blockIdx.x == 0) atomicOr(&g_status, int(EP_DEV_BAD_TABLES));
            }
        }
        o += 4 + 2 * cnt;
        ++c;
    }
    __syncthreads();
    const int nc = __popc(p.mask);
    for (uint32_t k = threadIdx.x; k < uint32_t(nc) * kEntries; k += kThreadsT) {
        const uint32_t cc = k >> 12, t = k & (kEntries - 1);
        const uint32_t* cu = cum + cc * 257;
        uint32_t s = 0;
#pragma unroll
        for (uint32_t step = 128; step >= 1; step >>= 1)
            if (s + step < 256 && cu[s + step] <= t) s += step;
        const uint32_t f = F[cc * 256 + s];
        // A slot past a corrupt table's end gets f = 0: the tile check flags it.
        tables[k] = (t >= cu[s] && t < cu[s] + f) ? (s << 24) | ((t - cu[s]) << 12) | f : 0u;
    }
    __syncthreads();
}

template <int E>
__global__ void __launch_bounds__(kThreadsT, 1) tans_decode_kernel(const TParams p) {
    extern __shared__ __align__(16) uint8_t smem_t[];
    uint32_t* scratch = reinterpret_cast<uint32_t*>(smem_t);
    uint32_t* tables = scratch + kScratchT / 4;
    build_tans_tables<E>(p, tables, scratch);
    const uint32_t lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const uint32_t lt_mask = (1u << lane) - 1u;
    const uint32_t* toff = reinterpret_cast<const uint32_t*>(p.blob + p.off_offsets);
    const uint8_t* payload = p.blob + p.off_payload;
    const uint32_t t_base = smem_addr(tables);
    const int nc = __popc(p.mask);
    const uint64_t per_tile = 32ull * p.K;
    using Elem = typename std::conditional<E == 4, uint32_t, typename std::conditional<E == 2, uint16_t, uint8_t>::type>::type;
    Elem* out = static_cast<Elem*>(p.dst);
    for (uint32_t tile = warp * gridDim.x + blockIdx.x; tile < p.T; tile += kWarpsT * gridDim.x) {
        const uint64_t start = 16ull * __ldg(toff + tile), end = 16ull * __ldg(toff + tile + 1);
        const uint64_t i0 = uint64_t(tile) * per_tile;
        const uint32_t ne = uint32_t(per_tile < p.n - i0 ? per_tile : p.n - i0);
        const uint32_t raw_run = (ne + 3) & ~3u;
        const uint32_t words_off = (nc ? 128u : 0u) + uint32_t(E - nc) * raw_run;
        if (end < start || end > p.payload_bytes || end - start < words_off) {
            if (lane == 0) atomicOr(&g_status, int(EP_DEV_BAD_OFFSETS));
            continue;
        }
        const uint8_t* tp = payload + start;
        const uint16_t* words = reinterpret_cast<const uint16_t*>(tp + words_off);
        const uint32_t cap = uint32_t((end - start - words_off) / 2);
        uint32_t x = nc ? __ldg(reinterpret_cast<const uint32_t*>(tp) + lane) : 0u;
        uint32_t pw = 0;
        const uint32_t R = (ne + 31) / 32;
        for (uint32_t k = 0; k < R; ++k) {
            const uint32_t i = 32 * k + lane;
            const bool act = i < ne;
            uint32_t val = 0;
            int c = 0, r = 0;
#pragma unroll
            for (int j = 0; j < E; ++j) {
                uint32_t byte = 0;
                if ((p.mask >> j) & 1u) {
                    if (act) {
                        const uint32_t e = ld_shared_u32(t_base + 4 * (uint32_t(c) * kEntries + (x & (kEntries - 1))));
                        x = (e & 0xFFFu) * (x >> 12) + ((e >> 12) & 0xFFFu);
                        byte = e >> 24;
                    }
                    const bool need = act && x < 65536u;
                    const uint32_t m = __ballot_sync(kFullMask, need);
                    if (need) {
                        const uint32_t idx = pw + __popc(m & lt_mask);
                        x = (x << 16) | (idx < cap ? uint32_t(__ldg(words + idx)) : 0u);
                    }
                    pw += __popc(m);
                    ++c;
                } else {
                    if (act) byte = __ldg(tp + (nc ? 128u : 0u) + uint32_t(r) * raw_run + i);
                    ++r;
                }
                val |= byte << (8 * j);
            }
            if (act) out[i0 + i] = Elem(val);
        }
        const bool good = nc == 0 || (__all_sync(kFullMask, x == 65536u) && pw <= cap && cap - pw <= 7);
        if (!good && lane == 0) atomicOr(&g_status, int(EP_DEV_CORRUPT_TILE));
    }
}

}  // namespace tansdev
}  // namespace dev
}  // namespace epk

namespace {
bool g_tans_configured[64][5] = {};
}

extern "C" ep_status ep_tans_decompress_into(const uint8_t* host_hdr, const void* dev_blob, size_t blob_bytes,
                                             void* dst, size_t dst_bytes, void* cuda_stream) {
    using namespace epk;
    using namespace epk::dev::tansdev;
    clear_error();
    if (!host_hdr || !dev_blob) return fail(EP_ERR_ARG, "ep_tans_decompress_into: NULL argument");
    tans::Header h;
    if (!tans::parse_tans_header(host_hdr, h)) return fail(EP_ERR_CORRUPT, "ep_tans_decompress_into: malformed EPL1 header");
    if (!dst && h.n) return fail(EP_ERR_ARG, "ep_tans_decompress_into: NULL dst");
    if (h.total != blob_bytes)
        return fail(EP_ERR_BUFFER, "ep_tans_decompress_into: blob_bytes %zu but header says %llu", blob_bytes,
                    (unsigned long long)h.total);
    if ((reinterpret_cast<uintptr_t>(dev_blob) & 15) || (reinterpret_cast<uintptr_t>(dst) & 15))
        return fail(EP_ERR_BUFFER, "ep_tans_decompress_into: dev_blob and dst must be 16-byte aligned");
    if (dst_bytes < h.n * uint64_t(h.e))
        return fail(EP_ERR_BUFFER, "ep_tans_decompress_into: dst holds %zu bytes, need %llu", dst_bytes,
                    (unsigned long long)(h.n * uint64_t(h.e)));
    if (h.T == 0) return EP_OK;
    int device = 0;
    cudaError_t e = cudaGetDevice(&device);
    if (e != cudaSuccess || device < 0 || device >= 64) return fail(EP_ERR_CUDA, "cudaGetDevice: %s", cudaGetErrorString(e));
    TParams p;
    p.blob = static_cast<const uint8_t*>(dev_blob);
    p.dst = dst;
    p.n = h.n;
    p.payload_bytes = h.total - h.off_payload;
    p.K = h.K;
    p.T = h.T;
    p.mask = h.mask;
    p.off_tables = h.off_tables;
    p.off_offsets = h.off_offsets;
    p.off_payload = h.off_payload;
    const uint32_t smem = kScratchT + uint32_t(h.coded_planes()) * kTableBytesT;
    const void* fn = h.e == 4   ? reinterpret_cast<const void*>(tans_decode_kernel<4>)
                     : h.e == 2 ? reinterpret_cast<const void*>(tans_decode_kernel<2>)
                                : reinterpret_cast<const void*>(tans_decode_kernel<1>);
    int sms = 0;
    {
        std::lock_guard<std::mutex> lk(g_dev_mu);
        if (!g_dev[device].sms) {
            e = cudaDeviceGetAttribute(&g_dev[device].sms, cudaDevAttrMultiProcessorCount, device);
            if (e != cudaSuccess) return fail(EP_ERR_CUDA, "cudaDeviceGetAttribute: %s", cudaGetErrorString(e));
        }
        sms = g_dev[device].sms;
        bool& conf = g_tans_configured[device][h.e];
        if (!conf) {
            e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, int(kScratchT + 4 * kTableBytesT));
            if (e != cudaSuccess) return fail(EP_ERR_CUDA, "cudaFuncSetAttribute: %s", cudaGetErrorString(e));
            conf = true;
        }
    }
    const uint32_t grid = h.T < uint32_t(sms) ? h.T : uint32_t(sms);
    cudaStream_t stream = static_cast<cudaStream_t>(cuda_stream);
    if (h.e == 4) tans_decode_kernel<4><<<grid, kThreadsT, smem, stream>>>(p);
    else if (h.e == 2) tans_decode_kernel<2><<<grid, kThreadsT, smem, stream>>>(p);
    else tans_decode_kernel<1><<<grid, kThreadsT, smem, stream>>>(p);
    e = cudaGetLastError();
    if (e != cudaSuccess) return fail(EP_ERR_CUDA, "tile-ANS decode launch: %s", cudaGetErrorString(e));
    return EP_OK;
}
