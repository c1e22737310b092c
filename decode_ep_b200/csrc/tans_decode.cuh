// Lossless tile-ANS (EPL1) decode for sm_100a, and its ABI entry ep_tans_decompress_into. Included by
// decode.cu, so that it shares the device status word.
//
// One warp per tile, tiles dealt round-robin over the CTAs first; the warp first copies its tile into its
// shared buffer. A round gives each lane one element:
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
constexpr uint32_t kMaxSmemT = 227 * 1024;             // per-CTA limit of sm_100

struct TParams {
    const uint8_t* blob;
    void* dst;
    uint64_t n;            // elements
    uint64_t payload_bytes;
    uint32_t K, T, mask;   // elements per lane per tile, tiles, coded planes
    uint32_t off_tables, off_offsets, off_payload;
    uint32_t buf_bytes;    // per-warp tile buffer (a multiple of 16)
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
    for (uint32_t k = threadIdx.x; k < uint32_t(nc) * kEntries; k += blockDim.x) {
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

__device__ __forceinline__ uint32_t ld_shared_u8(uint32_t addr) {
    uint16_t v;
    asm volatile("ld.shared.u8 %0, [%1];" : "=h"(v) : "r"(addr));
    return v;
}

// The bytes of one tile, in the warp's shared buffer (SMEM) or read from global memory in place.
template <bool SMEM>
struct TileBytes {
    const uint8_t* g;  // the tile in global memory
    uint32_t s;        // its shared-memory copy
    __device__ __forceinline__ uint32_t u32(uint32_t o) const {
        if constexpr (SMEM) return ld_shared_u32(s + o);
        else return __ldg(reinterpret_cast<const uint32_t*>(g + o));
    }
    __device__ __forceinline__ uint32_t u16(uint32_t o) const {
        if constexpr (SMEM) return ld_shared_u16(s + o);
        else return __ldg(reinterpret_cast<const uint16_t*>(g + o));
    }
    __device__ __forceinline__ uint32_t u8(uint32_t o) const {
        if constexpr (SMEM) return ld_shared_u8(s + o);
        else return __ldg(g + o);
    }
};

// One round of a tile: each lane's element i (act: it exists; PARTIAL: some lane's may not). MASK, the coded
// planes, is a compile-time constant, so the planes unroll with no test. A word index past the tile's stream
// reads the last word (shared copy, whose buffer has slack past the tile) or zero (in place): the values then
// come out wrong, and the tile check flags the tile.
template <int E, uint32_t MASK, bool SMEM, bool PARTIAL, class Elem>
__device__ __forceinline__ void tans_round(const TileBytes<SMEM>& tb, uint32_t t_base, uint32_t raw_run,
                                           uint32_t words_off, uint32_t cap, uint32_t capm1, uint32_t& x, uint32_t& pw,
                                           uint32_t i,
                                           bool act, Elem* o, uint32_t lt_mask) {
    constexpr uint32_t raw0 = MASK ? 128u : 0u;
    uint32_t val = 0;
    int c = 0, r = 0;
#pragma unroll
    for (int j = 0; j < E; ++j) {
        uint32_t byte = 0;
        if ((MASK >> j) & 1u) {
            if (!PARTIAL || act) {
                const uint32_t e = ld_shared_u32(t_base + 4 * (uint32_t(c) * kEntries + (x & (kEntries - 1))));
                x = (e & 0xFFFu) * (x >> 12) + ((e >> 12) & 0xFFFu);
                byte = e >> 24;
            }
            const bool need = (!PARTIAL || act) && x < 65536u;
            const uint32_t m = __ballot_sync(kFullMask, need);
            if (need) {
                const uint32_t idx = pw + __popc(m & lt_mask);
                if constexpr (SMEM) x = (x << 16) | tb.u16(words_off + 2 * min(idx, capm1));
                else x = (x << 16) | (idx < cap ? tb.u16(words_off + 2 * idx) : 0u);
            }
            pw += __popc(m);
            ++c;
        } else {
            if (!PARTIAL || act) byte = tb.u8(raw0 + uint32_t(r) * raw_run + i);
            ++r;
        }
        val |= byte << (8 * j);
    }
    if (!PARTIAL || act) o[i] = Elem(val);
}

// One full round of a tile held in shared memory: lane's raw bytes at rp[r] + off, its word stream at words
// (shared addresses). Every lane reads a word, at its clamped index, and only the lanes that refill keep it:
// the refill takes no branch.
template <int E, uint32_t MASK>
__device__ __forceinline__ uint32_t tans_round_smem(uint32_t t_base, const uint32_t* rp, uint32_t off, uint32_t words,
                                                    uint32_t capm1, uint32_t& x, uint32_t& pw, uint32_t lt_mask) {
    uint32_t val = 0;
    int c = 0, r = 0;
#pragma unroll
    for (int j = 0; j < E; ++j) {
        uint32_t byte;
        if ((MASK >> j) & 1u) {
            const uint32_t e = ld_shared_u32(t_base + uint32_t(c) * kTableBytesT + 4u * (x & (kEntries - 1)));
            x = (e & 0xFFFu) * (x >> 12) + ((e >> 12) & 0xFFFu);
            byte = e >> 24;
            const bool need = x < 65536u;
            const uint32_t m = __ballot_sync(kFullMask, need);
            const uint32_t w = ld_shared_u16(words + 2u * min(pw + __popc(m & lt_mask), capm1));
            if (need) x = __byte_perm(w, x, 0x5410);  // (x << 16) | w
            pw += __popc(m);
            ++c;
        } else {
            byte = ld_shared_u8(rp[r] + off);
            ++r;
        }
        val |= byte << (8 * j);
    }
    return val;
}

// The full rounds of a tile held in shared memory, four to a step: the raw planes' shared addresses and the
// output pointer advance once a step, and the rounds inside it use constant offsets from them.
template <int E, uint32_t MASK, class Elem>
__device__ __forceinline__ void tans_rounds_smem(uint32_t t_base, uint32_t raw_lane, uint32_t raw_run, uint32_t words,
                                                 uint32_t capm1, uint32_t& x, uint32_t& pw, uint32_t rounds, Elem* o,
                                                 uint32_t lt_mask) {
    constexpr int NR = E - __builtin_popcount(MASK);
    constexpr uint32_t U = 4;
    uint32_t rp[NR > 0 ? NR : 1];
#pragma unroll
    for (int r = 0; r < (NR > 0 ? NR : 1); ++r) rp[r] = raw_lane + uint32_t(r) * raw_run;
    uint32_t k = 0;
    for (; k + U <= rounds; k += U) {
#pragma unroll
        for (uint32_t u = 0; u < U; ++u)
            o[32 * u] = Elem(tans_round_smem<E, MASK>(t_base, rp, 32 * u, words, capm1, x, pw, lt_mask));
#pragma unroll
        for (int r = 0; r < NR; ++r) rp[r] += 32 * U;
        o += 32 * U;
    }
    for (; k < rounds; ++k) {
        *o = Elem(tans_round_smem<E, MASK>(t_base, rp, 0, words, capm1, x, pw, lt_mask));
#pragma unroll
        for (int r = 0; r < NR; ++r) rp[r] += 32;
        o += 32;
    }
}

// Decodes one tile of ne elements (output o, the tile's first element) whose bytes tb holds; returns whether
// its checks pass.
template <int E, uint32_t MASK, bool SMEM, class Elem>
__device__ __forceinline__ bool tans_tile(const TileBytes<SMEM>& tb, uint32_t t_base, uint32_t size, uint32_t ne,
                                          Elem* o, uint32_t lane, uint32_t lt_mask) {
    constexpr int NC = __builtin_popcount(MASK);
    const uint32_t raw_run = (ne + 3) & ~3u;
    const uint32_t words_off = (NC ? 128u : 0u) + uint32_t(E - NC) * raw_run;
    const uint32_t cap = (size - words_off) / 2;
    const uint32_t capm1 = cap ? cap - 1 : 0u;  // with cap = 0 the clamped read stays inside the tile's slack
    uint32_t x = NC ? tb.u32(4 * lane) : 0u;
    uint32_t pw = 0;
    const uint32_t full = ne / 32;
    if constexpr (SMEM) {
        tans_rounds_smem<E, MASK>(t_base, tb.s + (NC ? 128u : 0u) + lane, raw_run, tb.s + words_off, capm1, x, pw,
                                  full, o + lane, lt_mask);
    } else {
        for (uint32_t k = 0; k < full; ++k)
            tans_round<E, MASK, SMEM, false>(tb, t_base, raw_run, words_off, cap, capm1, x, pw, 32 * k + lane, true,
                                             o, lt_mask);
    }
    if (ne % 32) {
        const uint32_t i = 32 * full + lane;
        tans_round<E, MASK, SMEM, true>(tb, t_base, raw_run, words_off, cap, capm1, x, pw, i, i < ne, o, lt_mask);
    }
    return NC == 0 || (__all_sync(kFullMask, x == 65536u) && pw <= cap && cap - pw <= 7);
}

// tans_tile for the runtime mask: one instantiation per possible set of coded planes.
template <int E, uint32_t M, bool SMEM, class Elem>
__device__ __forceinline__ bool tans_tile_any(uint32_t mask, const TileBytes<SMEM>& tb, uint32_t t_base, uint32_t size,
                                              uint32_t ne, Elem* o, uint32_t lane, uint32_t lt_mask) {
    if (mask == M) return tans_tile<E, M, SMEM>(tb, t_base, size, ne, o, lane, lt_mask);
    if constexpr (M + 1 < (1u << E)) return tans_tile_any<E, M + 1, SMEM>(mask, tb, t_base, size, ne, o, lane, lt_mask);
    return false;
}

// The whole kernel. Each warp copies its tile into its shared buffer (buf_bytes, cp.async, 16 bytes a lane)
// when it fits, and reads it in place from global memory otherwise.
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
    const uint32_t buf = t_base + uint32_t(__popc(p.mask)) * kTableBytesT + warp * p.buf_bytes;
    const int nc = __popc(p.mask);
    const uint64_t per_tile = 32ull * p.K;
    using Elem = typename std::conditional<E == 4, uint32_t, typename std::conditional<E == 2, uint16_t, uint8_t>::type>::type;
    Elem* out = static_cast<Elem*>(p.dst);
    const uint32_t warps = blockDim.x / 32;
    for (uint32_t tile = warp * gridDim.x + blockIdx.x; tile < p.T; tile += warps * gridDim.x) {
        const uint64_t start = 16ull * __ldg(toff + tile), end = 16ull * __ldg(toff + tile + 1);
        const uint64_t i0 = uint64_t(tile) * per_tile;
        const uint32_t ne = uint32_t(per_tile < p.n - i0 ? per_tile : p.n - i0);
        const uint32_t words_off = (nc ? 128u : 0u) + uint32_t(E - nc) * ((ne + 3) & ~3u);
        if (end < start || end > p.payload_bytes || end - start < words_off) {
            if (lane == 0) atomicOr(&g_status, int(EP_DEV_BAD_OFFSETS));
            continue;
        }
        const uint32_t size = uint32_t(end - start);
        Elem* o = out + i0;
        bool good;
        // The buffer keeps 16 bytes past the tile, so that a clamped word read of an empty stream stays inside.
        if (size + 16 <= p.buf_bytes) {
            v2::copy_tile(buf, payload + start, size, lane);
            cp_async_commit();
            cp_async_wait<0>();
            __syncwarp();
            good = tans_tile_any<E, 0>(p.mask, TileBytes<true>{payload + start, buf}, t_base, size, ne, o, lane, lt_mask);
            __syncwarp();  // the buffer's reads are done before the next tile's copy
        } else {
            good = tans_tile_any<E, 0>(p.mask, TileBytes<false>{payload + start, 0u}, t_base, size, ne, o, lane, lt_mask);
        }
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
    // Per-warp tile buffers fill what the tables leave of the CTA's shared memory. The CTA takes as many warps
    // (32 down to 8) as can each hold an average tile with 15 % to spare (a 4096-element tile of 2-byte values
    // takes 6-7 KB, of 4-byte values about 14 KB); tiles that do not fit are read in place.
    const uint32_t fixed = kScratchT + uint32_t(h.coded_planes()) * kTableBytesT;
    const uint64_t avg = (h.total - h.off_payload) / h.T;
    const uint64_t need = ((avg + avg / 7 + 15) & ~uint64_t(15)) + 64;
    uint32_t warps = 8;
    for (uint32_t w = uint32_t(kWarpsT); w >= 8; w -= 4)
        if ((kMaxSmemT - fixed) / w >= need) {
            warps = w;
            break;
        }
    const uint32_t buf = ((kMaxSmemT - fixed) / warps) & ~15u;
    p.buf_bytes = buf;
    const uint32_t smem = fixed + warps * buf;
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
            e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, int(kMaxSmemT));
            if (e != cudaSuccess) return fail(EP_ERR_CUDA, "cudaFuncSetAttribute: %s", cudaGetErrorString(e));
            conf = true;
        }
    }
    const uint32_t grid = h.T < uint32_t(sms) ? h.T : uint32_t(sms);
    cudaStream_t stream = static_cast<cudaStream_t>(cuda_stream);
    const uint32_t threads = warps * 32;
    if (h.e == 4) tans_decode_kernel<4><<<grid, threads, smem, stream>>>(p);
    else if (h.e == 2) tans_decode_kernel<2><<<grid, threads, smem, stream>>>(p);
    else tans_decode_kernel<1><<<grid, threads, smem, stream>>>(p);
    e = cudaGetLastError();
    if (e != cudaSuccess) return fail(EP_ERR_CUDA, "tile-ANS decode launch: %s", cudaGetErrorString(e));
    return EP_OK;
}
