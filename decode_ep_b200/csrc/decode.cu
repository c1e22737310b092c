// Fused EntroPack decode for sm_100a (B200): rANS symbols -> E8 coordinates -> s_row * v / alpha ->
// container. One kernel does all of it. No symbol tensor and no codebook sit in between; the
// arithmetic inverse of the lattice map and the per-row rescale are fused with the symbol decode
// (modelscope paper page, summary; paper page abstract).
//
// Kernel shape: a persistent grid with one 1024-thread CTA per SM.
//   - Each CTA first expands the blob's 17 twelve-bit frequency tables into shared memory. Every
//     context gets a block: a 4096-entry slot -> symbol byte table, then one 16-byte record per
//     symbol {f, -cum, next context block, value}. The next-context pointer and the reconstructed
//     value are baked into the record. The hot loop therefore spends two shared loads per
//     coordinate and does no extra arithmetic for the context chain.
//   - Each warp then decodes whole tiles. Lane L owns the groups 32k + L of the tile. After every
//     symbol step the lanes that must refill take the next 16-bit words of the shared stream in
//     lane order, found with a warp ballot and a popcount prefix.
//   - Each lane reconstructs its 8 values and writes them with one 16-byte store (BF16/FP16), so a
//     warp writes 512 contiguous bytes.
// The loop is bound by integer issue and shared-memory bandwidth, not by tensor cores: decode has
// no dense contraction.
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_fp8.h>
#include <cuda_runtime.h>

#include <mutex>

#include "capi_internal.h"
#include "entropack.h"
#include "epk_format.h"

namespace epk {
namespace dev {

constexpr int kWarps = 32;
constexpr int kThreads = kWarps * 32;
constexpr uint32_t kLutBytes = 4096;
constexpr uint32_t kStartBlock = kLutBytes + 128 * 16;  // START: 128 symbols (coset bit x 64)
constexpr uint32_t kCtxBlock = kLutBytes + 64 * 16;     // other contexts: 64 symbols
constexpr uint32_t kPos7Shift = 8 * kCtxBlock;          // contexts 9..16 sit 8 blocks after 1..8
constexpr uint32_t kTablesBytes = kStartBlock + 16 * kCtxBlock;
constexpr uint32_t kCumBytes = (kNumCtx * 129 * 4 + 15) & ~15u;
constexpr uint32_t kSmemBytes = kTablesBytes + kCumBytes;
constexpr uint32_t kFullMask = 0xFFFFFFFFu;
// Words one round can take in the table-only fast path: 8 positions x 32 lanes, one refill each.
constexpr uint32_t kFastRoundWords = 8 * 32;

__host__ __device__ constexpr uint32_t block_of(int c) {
    return c == 0 ? 0u : kStartBlock + uint32_t(c - 1) * kCtxBlock;
}

enum Mode { kBF16 = 1, kFP16 = 2, kFP32 = 3, kFP8 = 4, kINT8 = 5, kCoords = 6 };

struct Params {
    const uint8_t* blob;
    void* dst;
    uint32_t gpr;  // groups per row, N / 8
    uint32_t T, G, NG, M;
    int r;
    float alpha;
    uint32_t off_scales, off_tables, off_offsets, off_payload, tables_len;
    uint64_t payload_bytes;
};

__device__ int g_status;

// ------------------------------------------------------------------------- table expansion

__device__ void build_tables(const Params& p, uint8_t* smem) {
    __shared__ uint32_t s_lo[kNumCtx], s_cnt[kNumCtx], s_bit[kNumCtx];
    uint32_t* cum = reinterpret_cast<uint32_t*>(smem + kTablesBytes);  // [17][129]
    const uint8_t* tb = p.blob + p.off_tables;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;

    if (tid < kNumCtx) {
        s_lo[tid] = tb[tid];
        s_cnt[tid] = tb[kNumCtx + tid];
    }
    __syncthreads();
    if (tid == 0) {
        uint32_t acc = 0;
        for (int c = 0; c < kNumCtx; ++c) { s_bit[c] = acc; acc += 12 * s_cnt[c]; }
    }
    __syncthreads();

    // Frequencies, indexed by symbol (zero outside [lo, lo + cnt)).
    const uint32_t bits_len = p.tables_len > 2 * kNumCtx ? p.tables_len - 2 * kNumCtx : 0;
    for (int i = tid; i < kNumCtx * 128; i += kThreads) {
        int c = i >> 7, s = i & 127, A = c == 0 ? 128 : 64;
        uint32_t lo = s_lo[c], cnt = s_cnt[c], f = 0;
        if (uint32_t(s) >= lo && uint32_t(s) < lo + cnt && s < A) {
            if (cnt == 1) {
                f = kProbScale;
            } else {
                uint32_t bit = s_bit[c] + 12 * (uint32_t(s) - lo), byte = bit >> 3, w = 0;
                for (int k = 0; k < 3; ++k)
                    if (byte + k < bits_len) w |= uint32_t(tb[2 * kNumCtx + byte + k]) << (8 * k);
                f = (w >> (bit & 7)) & 0xFFFu;
            }
        }
        cum[c * 129 + s] = f;
    }
    __syncthreads();

    // Exclusive prefix sums, one warp per context (4 symbols per lane).
    if (warp < kNumCtx) {
        uint32_t* cc = cum + warp * 129;
        uint32_t f0 = cc[4 * lane], f1 = cc[4 * lane + 1], f2 = cc[4 * lane + 2], f3 = cc[4 * lane + 3];
        uint32_t sum = f0 + f1 + f2 + f3, incl = sum;
#pragma unroll
        for (int d = 1; d < 32; d <<= 1) {
            uint32_t v = __shfl_up_sync(kFullMask, incl, d);
            if (lane >= d) incl += v;
        }
        uint32_t ex = incl - sum;
        __syncwarp();
        cc[4 * lane] = ex;
        cc[4 * lane + 1] = ex + f0;
        cc[4 * lane + 2] = ex + f0 + f1;
        cc[4 * lane + 3] = ex + f0 + f1 + f2;
        if (lane == 31) {
            cc[128] = incl;
            bool ok = s_cnt[warp] == 0 ? incl == 0 : incl == kProbScale;
            if (!ok && blockIdx.x == 0) atomicOr(&g_status, int(EP_DEV_BAD_TABLES));
        }
    }
    __syncthreads();

    // Records: {f, -cum, next block, value}. The value is v = hi + b/2 for positions 0..6 and
    // 2h + b/2 for position 7 (u7 = 2h + parity is completed in the decode loop).
    for (int i = tid; i < kNumCtx * 128; i += kThreads) {
        int c = i >> 7, s = i & 127, A = c == 0 ? 128 : 64;
        if (s >= A) continue;
        const uint32_t* cc = cum + c * 129;
        uint32_t f = cc[s + 1] - cc[s];
        int b = c == 0 ? (s >> 6) : (c <= 8 ? (c - 1) >> 2 : (c - 9) >> 2);
        int idx = s & 63, hi = idx - 31;
        uint32_t next = 0;
        float val;
        if (c <= 8) {
            int m = hi >= 0 ? hi : -hi - b;
            int cls = idx == kEscIdx ? 3 : (m < 3 ? m : 3);
            next = block_of(1 + 4 * b + cls);
            val = float(hi) + 0.5f * float(b);
        } else {
            val = float(2 * hi) + 0.5f * float(b);
        }
        uint4 rec = make_uint4(f, 0u - cc[s], next, __float_as_uint(val));
        *reinterpret_cast<uint4*>(smem + block_of(c) + kLutBytes + 16 * s) = rec;
    }

    // Slot -> symbol bytes, 16 slots per thread: the largest s with cum[s] <= slot (symbols with f = 0
    // share their successor's cum and are skipped).
    for (int i = tid; i < kNumCtx * 256; i += kThreads) {
        int c = i >> 8, A = c == 0 ? 128 : 64;
        uint32_t slot0 = uint32_t(i & 255) * 16;
        const uint32_t* cc = cum + c * 129;
        int lo = 0, hi = A - 1;
        while (lo < hi) {
            int mid = (lo + hi + 1) >> 1;
            if (cc[mid] <= slot0) lo = mid; else hi = mid - 1;
        }
        int s = lo;
        uint32_t out[4] = {0, 0, 0, 0};
#pragma unroll
        for (int j = 0; j < 16; ++j) {
            uint32_t slot = slot0 + j;
            while (s + 1 < A && cc[s + 1] <= slot) ++s;
            out[j >> 2] |= uint32_t(s) << (8 * (j & 3));
        }
        *reinterpret_cast<uint4*>(smem + block_of(c) + slot0) = make_uint4(out[0], out[1], out[2], out[3]);
    }
}

// ------------------------------------------------------------------------------- stores

__device__ __forceinline__ uint32_t pack_bf16(float a, float b) {
    __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
    return *reinterpret_cast<uint32_t*>(&h);
}
__device__ __forceinline__ uint32_t pack_f16(float a, float b) {
    __half2 h = __floats2half2_rn(a, b);
    return *reinterpret_cast<uint32_t*>(&h);
}
__device__ __forceinline__ uint32_t pack_e4m3x4(float a, float b, float c, float d) {
    uint32_t lo = __nv_cvt_float2_to_fp8x2(make_float2(a, b), __NV_SATFINITE, __NV_E4M3);
    uint32_t hi = __nv_cvt_float2_to_fp8x2(make_float2(c, d), __NV_SATFINITE, __NV_E4M3);
    return lo | (hi << 16);
}
__device__ __forceinline__ uint32_t sat_s8(float y) {
    int v = __float2int_rn(y);  // round half to even
    v = v < -128 ? -128 : (v > 127 ? 127 : v);
    return uint32_t(v) & 0xFFu;
}

// Writes the 8 values of group g; y[] are the binary32 values, z[] = 2v for the coordinate mode.
template <int MODE>
__device__ __forceinline__ void store_group(void* dst, uint32_t g, const float* y, const int32_t* z) {
    if constexpr (MODE == kBF16) {
        uint4 q = make_uint4(pack_bf16(y[0], y[1]), pack_bf16(y[2], y[3]), pack_bf16(y[4], y[5]), pack_bf16(y[6], y[7]));
        reinterpret_cast<uint4*>(dst)[g] = q;
    } else if constexpr (MODE == kFP16) {
        uint4 q = make_uint4(pack_f16(y[0], y[1]), pack_f16(y[2], y[3]), pack_f16(y[4], y[5]), pack_f16(y[6], y[7]));
        reinterpret_cast<uint4*>(dst)[g] = q;
    } else if constexpr (MODE == kFP32) {
        float4* o = reinterpret_cast<float4*>(dst) + 2ull * g;
        o[0] = make_float4(y[0], y[1], y[2], y[3]);
        o[1] = make_float4(y[4], y[5], y[6], y[7]);
    } else if constexpr (MODE == kFP8) {
        reinterpret_cast<uint2*>(dst)[g] = make_uint2(pack_e4m3x4(y[0], y[1], y[2], y[3]), pack_e4m3x4(y[4], y[5], y[6], y[7]));
    } else if constexpr (MODE == kINT8) {
        uint32_t a = sat_s8(y[0]) | (sat_s8(y[1]) << 8) | (sat_s8(y[2]) << 16) | (sat_s8(y[3]) << 24);
        uint32_t b = sat_s8(y[4]) | (sat_s8(y[5]) << 8) | (sat_s8(y[6]) << 16) | (sat_s8(y[7]) << 24);
        reinterpret_cast<uint2*>(dst)[g] = make_uint2(a, b);
    } else {
        int4* o = reinterpret_cast<int4*>(dst) + 2ull * g;
        o[0] = make_int4(z[0], z[1], z[2], z[3]);
        o[1] = make_int4(z[4], z[5], z[6], z[7]);
    }
}

// Per-lane state of the row of the current group; c_row = fl32(s_row / alpha) is recomputed only
// when the row changes.
struct RowCursor {
    uint32_t row, col, cached_row;
    float c_row;

    __device__ __forceinline__ float scale(const Params& p, const uint16_t* scales) {
        if (row != cached_row) {
            cached_row = row;
            float s = __uint_as_float(uint32_t(__ldg(scales + row)) << 16);
            c_row = __fdiv_rn(s, p.alpha);
        }
        return c_row;
    }
    __device__ __forceinline__ void advance(uint32_t gpr) {  // next round: 32 groups further
        col += 32;
        while (col >= gpr) { col -= gpr; ++row; }
    }
};

// ------------------------------------------------------------------------------ one round

// Fast round: all 32 lanes hold a group, the tile has no ESC, r = 0, and a full round of reads stays
// inside the payload, so no read needs a bounds check.
template <int MODE>
__device__ __forceinline__ void round_fast(const Params& p, const uint8_t* smem, const uint16_t* words,
                                           const uint16_t* scales, uint32_t& x, uint32_t& pos, uint32_t g,
                                           uint32_t lt_mask, RowCursor& rc) {
    float v[8];
    uint32_t B = 0, par = 0;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        if (i == 7) B += kPos7Shift;
        const uint32_t slot = x & (kProbScale - 1);
        const uint32_t sym = smem[B + slot];
        const uint4 rec = *reinterpret_cast<const uint4*>(smem + B + kLutBytes + 16 * sym);
        x = rec.x * (x >> kProbBits) + slot + rec.y;  // f * (x >> 12) + slot - cum
        const bool need = x < kRansL;
        const uint32_t m = __ballot_sync(kFullMask, need);
        if (need) x = (x << 16) | uint32_t(__ldg(words + pos + __popc(m & lt_mask)));
        pos += __popc(m);
        if (i < 7) par ^= sym;
        v[i] = __uint_as_float(rec.w);
        B = rec.z;
    }
    // u_i = idx_i - 31 flips parity against idx_i; seven flips make pi = 1 when the idx parity is even.
    if (!(par & 1u)) v[7] += 1.0f;
    const float c = rc.scale(p, scales);
    float y[8];
    int32_t z[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        y[i] = __fmul_rn(v[i], c);
        if constexpr (MODE == kCoords) z[i] = __float2int_rn(v[i] * 2.0f);
    }
    store_group<MODE>(p.dst, g, y, z);
}

// General round: partial rounds, ESC words, raw low bits and bounded stream reads.
template <int MODE>
__device__ __noinline__ void round_general(const Params& p, const uint8_t* smem, const uint16_t* words,
                                           uint32_t nwords, const uint8_t* rawsec, uint32_t raw_avail,
                                           const uint16_t* scales, uint32_t& x, uint32_t& pos, uint32_t q,
                                           bool active, uint32_t g, uint32_t lt_mask, RowCursor& rc) {
    const int r = p.r;
    // The group's 8r raw bits start at byte q*r of the raw section; load a 96-bit window.
    uint32_t win0 = 0, win1 = 0, win2 = 0;
    if (r > 0 && active) {
        uint32_t o = q * uint32_t(r), a = o & ~3u, sh = (o & 3u) * 8;
        uint32_t w[4];
#pragma unroll
        for (int j = 0; j < 4; ++j)
            w[j] = (a + 4 * j + 4 <= raw_avail) ? __ldg(reinterpret_cast<const uint32_t*>(rawsec + a) + j) : 0u;
        win0 = __funnelshift_r(w[0], w[1], sh);
        win1 = __funnelshift_r(w[1], w[2], sh);
        win2 = __funnelshift_r(w[2], w[3], sh);
    }
    const uint32_t rmask = (1u << r) - 1u;
    uint32_t B = 0, b = 0;
    int32_t t[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        if (i == 7) B += kPos7Shift;
        uint32_t sym = 0;
        uint4 rec = make_uint4(0, 0, 0, 0);
        if (active) {
            const uint32_t slot = x & (kProbScale - 1);
            sym = smem[B + slot];
            rec = *reinterpret_cast<const uint4*>(smem + B + kLutBytes + 16 * sym);
            x = rec.x * (x >> kProbBits) + slot + rec.y;
        }
        const bool need = active && x < kRansL;
        const uint32_t m = __ballot_sync(kFullMask, need);
        if (need) {
            uint32_t wi = pos + __popc(m & lt_mask);
            x = (x << 16) | (wi < nwords ? uint32_t(__ldg(words + wi)) : 0u);
        }
        pos += __popc(m);
        const uint32_t idx = sym & 63u;
        int32_t hi = int32_t(idx) - 31;
        const bool esc = active && idx == uint32_t(kEscIdx);
        const uint32_t me = __ballot_sync(kFullMask, esc);
        if (me) {
            if (esc) {
                uint32_t wi = pos + __popc(me & lt_mask);
                hi = int32_t(int16_t(wi < nwords ? __ldg(words + wi) : 0));
            }
            pos += __popc(me);
        }
        if (i == 0) b = sym >> 6;
        int32_t lo = 0;
        if (r > 0) {
            uint32_t bp = uint32_t(i) * uint32_t(r), sel = bp >> 5, sh = bp & 31;
            uint32_t wa = sel == 0 ? win0 : (sel == 1 ? win1 : win2);
            uint32_t wb = sel == 0 ? win1 : win2;
            lo = int32_t(__funnelshift_r(wa, wb, sh) & rmask);
        }
        t[i] = hi * (1 << r) + lo;
        B = rec.z;
    }
    if (!active) return;
    int32_t s7 = 0;
#pragma unroll
    for (int i = 0; i < 7; ++i) s7 += t[i];
    const float c = rc.scale(p, scales);
    float y[8];
    int32_t z[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        int32_t u = i < 7 ? t[i] : 2 * t[7] + (s7 & 1);
        z[i] = 2 * u + int32_t(b);
        y[i] = __fmul_rn(__int2float_rn(z[i]) * 0.5f, c);
    }
    store_group<MODE>(p.dst, g, y, z);
}

// ---------------------------------------------------------------------------------- kernel

template <int MODE>
__global__ void __launch_bounds__(kThreads, 1) decode_kernel(const Params p) {
    extern __shared__ __align__(16) uint8_t smem[];
    build_tables(p, smem);
    __syncthreads();

    const uint32_t lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const uint32_t lt_mask = (1u << lane) - 1u;
    const uint16_t* scales = reinterpret_cast<const uint16_t*>(p.blob + p.off_scales);
    const uint32_t* toff = reinterpret_cast<const uint32_t*>(p.blob + p.off_offsets);
    const uint8_t* payload = p.blob + p.off_payload;
    const uint32_t per_tile = 32 * p.G;

    for (uint32_t tile = blockIdx.x * kWarps + warp; tile < p.T; tile += gridDim.x * kWarps) {
        const uint32_t e0 = __ldg(toff + tile), e1 = __ldg(toff + tile + 1);
        const uint64_t start = uint64_t(e0 & 0x7FFFFFFFu) * 16, end = uint64_t(e1 & 0x7FFFFFFFu) * 16;
        const uint32_t g0 = tile * per_tile;
        const uint32_t ng = min(per_tile, p.NG - g0);
        const uint32_t raw = (ng * uint32_t(p.r) + 3u) & ~3u;
        if (end < start || end > p.payload_bytes || end - start < 128ull + raw || end - start > 0xFFFFFFF0ull) {
            if (lane == 0) atomicOr(&g_status, int(EP_DEV_BAD_OFFSETS));
            continue;
        }
        const uint8_t* tp = payload + start;
        const uint32_t tile_bytes = uint32_t(end - start);
        uint32_t x = __ldg(reinterpret_cast<const uint32_t*>(tp) + lane);
        const uint16_t* words = reinterpret_cast<const uint16_t*>(tp + 128 + raw);
        const uint32_t nwords = (tile_bytes - 128 - raw) / 2;
        uint32_t pos = 0;
        const bool fast_tile = !(e0 >> 31) && p.r == 0;
        // The fast round reads without bounds checks. It is allowed while a whole round of reads stays
        // inside the payload: reading past this tile into the next is harmless (the end-of-tile check
        // catches it), reading past the blob is not.
        const uint64_t words_to_payload_end = (p.payload_bytes - start - 128 - raw) / 2;
        const uint32_t fast_limit = words_to_payload_end > 0xFFFFFFFFull ? 0xFFFFFFFFu : uint32_t(words_to_payload_end);

        RowCursor rc;
        rc.row = (g0 + lane) / p.gpr;
        rc.col = (g0 + lane) - rc.row * p.gpr;
        rc.cached_row = 0xFFFFFFFFu;
        rc.c_row = 0.f;

        const uint32_t R = (ng + 31) / 32;
        for (uint32_t k = 0; k < R; ++k) {
            const uint32_t q = 32 * k + lane, g = g0 + q;
            const bool full = 32 * k + 32 <= ng;
            if (fast_tile && full && pos <= fast_limit - kFastRoundWords && fast_limit >= kFastRoundWords)
                round_fast<MODE>(p, smem, words, scales, x, pos, g, lt_mask, rc);
            else
                round_general<MODE>(p, smem, words, nwords, tp + 128, tile_bytes - 128, scales, x, pos, q, q < ng, g,
                                    lt_mask, rc);
            rc.advance(p.gpr);
        }
        const bool ok = __all_sync(kFullMask, x == kRansL) && pos <= nwords && nwords - pos <= 7;
        if (!ok && lane == 0) atomicOr(&g_status, int(EP_DEV_CORRUPT_TILE));
    }
}

}  // namespace dev

// ------------------------------------------------------------------------------- launcher

namespace {

struct DeviceInfo {
    int sms = 0;
    bool configured[8] = {false};
};
std::mutex g_dev_mu;
DeviceInfo g_dev[64];

template <int MODE>
ep_status launch_mode(const dev::Params& p, cudaStream_t stream, int device) {
    {
        std::lock_guard<std::mutex> lk(g_dev_mu);
        DeviceInfo& d = g_dev[device];
        if (!d.configured[MODE]) {
            cudaError_t e = cudaFuncSetAttribute(dev::decode_kernel<MODE>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                                 int(dev::kSmemBytes));
            if (e != cudaSuccess) return fail(EP_ERR_CUDA, "cudaFuncSetAttribute: %s", cudaGetErrorString(e));
            d.configured[MODE] = true;
        }
    }
    uint32_t want = (p.T + dev::kWarps - 1) / dev::kWarps;
    uint32_t grid = want < uint32_t(g_dev[device].sms) ? want : uint32_t(g_dev[device].sms);
    if (grid == 0) grid = 1;
    dev::decode_kernel<MODE><<<grid, dev::kThreads, dev::kSmemBytes, stream>>>(p);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return fail(EP_ERR_CUDA, "decode launch: %s", cudaGetErrorString(e));
    return EP_OK;
}

ep_status launch_decode(const uint8_t* host_hdr, const void* dev_blob, size_t blob_bytes, void* dst, size_t dst_bytes,
                        int mode, void* stream_ptr) {
    if (!host_hdr || !dev_blob || !dst) return fail(EP_ERR_ARG, "decode: NULL argument");
    Header h;
    if (!parse_header(host_hdr, h)) return fail(EP_ERR_CORRUPT, "decode: malformed EPK1 header");
    if (h.total != blob_bytes) return fail(EP_ERR_BUFFER, "decode: blob_bytes %zu but header says %llu", blob_bytes,
                                           (unsigned long long)h.total);
    if ((reinterpret_cast<uintptr_t>(dev_blob) & 15) || (reinterpret_cast<uintptr_t>(dst) & 15))
        return fail(EP_ERR_BUFFER, "decode: dev_blob and dst must be 16-byte aligned");
    uint64_t es = mode == dev::kCoords ? 4 : uint64_t(elem_bytes(h.dtype));
    uint64_t need = uint64_t(h.M) * h.N * es;
    if (dst_bytes < need) return fail(EP_ERR_BUFFER, "decode: dst holds %zu bytes, need %llu", dst_bytes,
                                      (unsigned long long)need);
    int device = 0;
    cudaError_t e = cudaGetDevice(&device);
    if (e != cudaSuccess || device < 0 || device >= 64) return fail(EP_ERR_CUDA, "cudaGetDevice: %s", cudaGetErrorString(e));
    {
        std::lock_guard<std::mutex> lk(g_dev_mu);
        if (!g_dev[device].sms) {
            e = cudaDeviceGetAttribute(&g_dev[device].sms, cudaDevAttrMultiProcessorCount, device);
            if (e != cudaSuccess) return fail(EP_ERR_CUDA, "cudaDeviceGetAttribute: %s", cudaGetErrorString(e));
        }
    }
    dev::Params p;
    p.blob = static_cast<const uint8_t*>(dev_blob);
    p.dst = dst;
    p.gpr = h.N / 8;
    p.T = h.T;
    p.G = uint32_t(h.G);
    p.NG = uint32_t(h.groups());
    p.M = h.M;
    p.r = h.r;
    p.alpha = h.alpha;
    p.off_scales = h.off_scales;
    p.off_tables = h.off_tables;
    p.off_offsets = h.off_offsets;
    p.off_payload = h.off_payload;
    p.tables_len = h.off_offsets - h.off_tables;
    p.payload_bytes = h.total - h.off_payload;
    cudaStream_t stream = static_cast<cudaStream_t>(stream_ptr);
    switch (mode) {
        case dev::kBF16: return launch_mode<dev::kBF16>(p, stream, device);
        case dev::kFP16: return launch_mode<dev::kFP16>(p, stream, device);
        case dev::kFP32: return launch_mode<dev::kFP32>(p, stream, device);
        case dev::kFP8: return launch_mode<dev::kFP8>(p, stream, device);
        case dev::kINT8: return launch_mode<dev::kINT8>(p, stream, device);
        case dev::kCoords: return launch_mode<dev::kCoords>(p, stream, device);
    }
    return fail(EP_ERR_DTYPE, "decode: unknown dtype %d", mode);
}

}  // namespace
}  // namespace epk

using namespace epk;

extern "C" ep_status ep_decompress_into(const uint8_t* host_hdr, const void* dev_blob, size_t blob_bytes, void* dst,
                                        size_t dst_bytes, void* cuda_stream) {
    clear_error();
    if (!host_hdr) return fail(EP_ERR_ARG, "decode: NULL header");
    Header h;
    if (!parse_header(host_hdr, h)) return fail(EP_ERR_CORRUPT, "decode: malformed EPK1 header");
    return launch_decode(host_hdr, dev_blob, blob_bytes, dst, dst_bytes, h.dtype, cuda_stream);
}

extern "C" ep_status ep_decode_coords_into(const uint8_t* host_hdr, const void* dev_blob, size_t blob_bytes,
                                           int32_t* dst_z, size_t dst_bytes, void* cuda_stream) {
    clear_error();
    return launch_decode(host_hdr, dev_blob, blob_bytes, dst_z, dst_bytes, dev::kCoords, cuda_stream);
}

extern "C" ep_status ep_decompress(const uint8_t* host_hdr, const void* dev_blob, size_t blob_bytes, void** dst,
                                   void* cuda_stream) {
    clear_error();
    if (!host_hdr || !dst) return fail(EP_ERR_ARG, "decode: NULL argument");
    Header h;
    if (!parse_header(host_hdr, h)) return fail(EP_ERR_CORRUPT, "decode: malformed EPK1 header");
    size_t bytes = size_t(uint64_t(h.M) * h.N * uint64_t(elem_bytes(h.dtype)));
    void* out = nullptr;
    cudaStream_t stream = static_cast<cudaStream_t>(cuda_stream);
    cudaError_t e = cudaMallocAsync(&out, bytes, stream);
    if (e != cudaSuccess) return fail(EP_ERR_NOMEM, "cudaMallocAsync(%zu): %s", bytes, cudaGetErrorString(e));
    ep_status st = launch_decode(host_hdr, dev_blob, blob_bytes, out, bytes, h.dtype, cuda_stream);
    if (st != EP_OK) {
        cudaFreeAsync(out, stream);
        return st;
    }
    *dst = out;
    return EP_OK;
}

extern "C" ep_status ep_get_device_status(void* cuda_stream, int32_t* flags) {
    clear_error();
    if (!flags) return fail(EP_ERR_ARG, "ep_get_device_status: NULL flags");
    cudaStream_t stream = static_cast<cudaStream_t>(cuda_stream);
    cudaError_t e = cudaStreamSynchronize(stream);
    if (e != cudaSuccess) return fail(EP_ERR_CUDA, "cudaStreamSynchronize: %s", cudaGetErrorString(e));
    int v = 0, zero = 0;
    e = cudaMemcpyFromSymbol(&v, dev::g_status, sizeof(int));
    if (e == cudaSuccess) e = cudaMemcpyToSymbol(dev::g_status, &zero, sizeof(int));
    if (e != cudaSuccess) return fail(EP_ERR_CUDA, "status word: %s", cudaGetErrorString(e));
    *flags = v;
    return EP_OK;
}
