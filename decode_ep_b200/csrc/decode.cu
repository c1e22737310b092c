// Fused EntroPack decode for sm_100a (B200): rANS symbols -> E8 coordinates -> s_row * v / alpha ->
// container, in one pass. No symbol tensor and no codebook sit in between; the arithmetic inverse of the
// lattice map and the per-row rescale are fused with the symbol decode (modelscope paper page, summary;
// paper page abstract). This file holds four kernels and their C-ABI launchers:
//
//   - v2::decode_kernel, one layer of format version 2 (the default; ep_decompress_into). A persistent grid
//     of 1024-thread CTAs, one per SM. Each CTA builds the blob's 9 x 256 fused 32-bit entries in shared
//     memory (value field, escape and class bits, coset bit, f, slot - cum): a symbol step is one random
//     4-byte shared load and a handful of integer operations, and one refill (ballot, popcount prefix, one
//     16-bit word in lane order) serves each pair of coordinates. Each warp copies its whole tile into a 5 KB
//     shared buffer with cp.async, the next tile landing in the other end while it decodes the current one.
//     v = u + b/2 is rebuilt with no conversion instruction (the value field ORed into the mantissa of
//     1.5 * 2^22), rescaled in packed f32x2, and each lane stores its 8 values at once.
//   - v2::prep_tables_kernel and v2::seq_kernel, a list of version-2 layers of one dtype (ep_decompress_many):
//     the tables of every layer built once into global scratch, then one cooperative persistent launch
//     deals all the layers' tiles round-robin over CTAs and warps, keeps four layers' tables per CTA in
//     shared windows refilled by bulk copies, and orders the stores of overlapping outputs tile by tile.
//   - decode_kernel, one layer of format version 1 (12-bit tables, 144 KB of fused entries, a refill per
//     symbol); with expand_tables_kernel for version-1 sequences, chained with programmatic dependent launch.
//   - tans_decode_kernel (tans_decode.cuh, included at the end): the lossless tile-ANS blobs.
//
// The decode is bound by integer issue and shared-memory latency, not by tensor cores: it has no dense
// contraction.
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_fp8.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cstdlib>
#include <cstring>
#include <memory>
#include <type_traits>
#include <mutex>
#include <vector>

#include "capi_internal.h"
#include "entropack.h"
#include "epk_format.h"

namespace epk {
namespace dev {

constexpr int kWarps = 32;
constexpr int kThreads = kWarps * 32;
constexpr uint32_t kFullMask = 0xFFFFFFFFu;

// Fused decode tables: 4096 four-byte entries per context. Blocks: contexts 1..8 at (c-1) * 16 KB,
// so (b, class) selects a block by bits 14 (class) and 15 (b), with +64 KB for position 7; START at
// 128 KB.
constexpr uint32_t kCtxBytes = 4096 * 4;
constexpr uint32_t kPos7Offset = 4 * kCtxBytes;
constexpr uint32_t kStartOffset = 8 * kCtxBytes;
constexpr uint32_t kTablesBytes = 9 * kCtxBytes;
__host__ __device__ constexpr uint32_t block_of(int c) { return c == 0 ? kStartOffset : uint32_t(c - 1) * kCtxBytes; }

// Per-warp stream rings.
constexpr uint32_t kRingBytes = 2048;
constexpr uint32_t kChunkBytes = 512;  // one 16-byte copy per lane
constexpr uint32_t kRingChunks = kRingBytes / kChunkBytes;
constexpr uint32_t kRingsBytes = kWarps * kRingBytes;

// Dynamic shared memory: [alignment pad up to 2 KB][rings][tables][table-build scratch]. The scratch
// is its own region so that the first tile's stream copies can be in flight during the build.
constexpr uint32_t kScratchCum = 0;                                      // u32 [9][129]
constexpr uint32_t kScratchBytes = 4656;                                 // serialised tables
constexpr uint32_t kScratchTableCap = 1024;                              // a valid blob's tables take < 1 KB
constexpr uint32_t kScratchTmpl = kScratchBytes + kScratchTableCap;      // u32 [9][128]: D = template - cum
constexpr uint32_t kScratchWsum = kScratchTmpl + kNumCtx * 128 * 4;      // u32 [32]: per-warp frequency sums
constexpr uint32_t kScratchSize = kScratchWsum + 32 * 4;
static_assert(kScratchCum + kNumCtx * 129 * 4 <= kScratchBytes, "scratch overlap");
// The table region starts on a 32 KB boundary of the shared window. Every (b, position family) base is
// then a multiple of 32 KB, and the class bit selects +16 KB with one OR. Rings fill the gap in front
// of the tables, and the rest go after them: the request covers any starting offset.
constexpr uint32_t kTableAlign = 32 * 1024;
constexpr uint32_t kSmemBytes = kTablesBytes + kRingsBytes + kScratchSize + 2 * kRingBytes;
static_assert(kSmemBytes <= 227 * 1024, "exceeds the per-block shared memory of sm_100");

// Words one round can take: 8 positions x 32 lanes, one refill each, plus as many ESC words.
constexpr uint32_t kRoundWords = 8 * 32;
constexpr uint32_t kRoundWordsEsc = 2 * kRoundWords;

// 1.5 * 2^22: binary32 with a last-place unit of 1/2. ORing a field F < 2^22 into its mantissa gives
// 1.5 * 2^22 + F/2 exactly.
constexpr uint32_t kHalfMagic = 0x4AC00000u;
constexpr float kHalfMagicF = 6291456.0f;

enum Mode { kBF16 = 1, kFP16 = 2, kFP32 = 3, kFP8 = 4, kINT8 = 5, kCoords = 6 };

struct Params {
    const uint8_t* blob;
    void* dst;
    uint32_t gpr;  // groups per row, N / 8
    uint32_t T, G, NG, M;
    int r;
    float alpha, inv_alpha;  // inv_alpha = RN(1 / alpha), computed on the host
    // Multipliers kept out of the compiler's sight (2, 4, -4096, 128), so that the products below are
    // issued as integer multiply-adds instead of ALU shifts: the loop saturates the ALU pipe first.
    uint32_t k2, k4, kneg4096, k128, kneg256;
    uint32_t off_scales, off_tables, off_offsets, off_payload, tables_len;
    uint64_t payload_bytes;
    // The next blob of a sequence (ep_decompress_many), or null: its tables, tile offsets and scales
    // are pulled into L2 while this one decodes.
    const uint8_t* next_blob;
    uint32_t next_meta_off, next_meta_bytes;  // [off_scales, off_payload) of the next blob
    uint32_t test_no_table_copy;              // test hook: leave the prepared-table copies unissued
    // The fused entries of this blob, 9 x 4096 in shared-memory block order, built once for the whole
    // sequence by expand_tables_kernel; null means each CTA builds them (build_tables).
    const uint32_t* pre_tables;
};

__device__ int g_status;

// Acquire load at GPU scope: the memory operations that follow it in this thread are ordered after it.
__device__ __forceinline__ uint32_t ld_acquire(const uint32_t* p) {
    uint32_t v;
    asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}

// ------------------------------------------------------------------------- PTX helpers

__device__ __forceinline__ uint32_t smem_addr(const void* p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}
__device__ __forceinline__ uint32_t ld_shared_u16(uint32_t addr) {
    unsigned short v;
    asm volatile("ld.shared.u16 %0, [%1];" : "=h"(v) : "r"(addr));
    return v;
}
__device__ __forceinline__ uint32_t ld_shared_u32(uint32_t addr) {
    uint32_t v;
    asm volatile("ld.shared.u32 %0, [%1];" : "=r"(v) : "r"(addr));
    return v;
}
// 16-byte asynchronous copy global -> shared; bytes past `src_bytes` (0..16) are zero-filled and
// not read.
__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src, uint32_t src_bytes) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(src_bytes) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }
__device__ __forceinline__ void prefetch_l2(const void* p) { asm volatile("prefetch.global.L2 [%0];" ::"l"(p)); }
__device__ __forceinline__ void prefetch_l1(const void* p) { asm volatile("prefetch.global.L1 [%0];" ::"l"(p)); }
// (a0 - k0, a1 - k1), then times c: two binary32 values per instruction (packed f32x2, sm_100).
__device__ __forceinline__ void sub_mul_f32x2(float a0, float a1, float k0, float k1, float c, float& y0, float& y1) {
    uint64_t a, kk, cc, r;
    asm("mov.b64 %0, {%1, %2};" : "=l"(a) : "f"(a0), "f"(a1));
    asm("mov.b64 %0, {%1, %2};" : "=l"(kk) : "f"(k0), "f"(k1));
    asm("mov.b64 %0, {%1, %1};" : "=l"(cc) : "f"(c));
    asm("sub.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(kk));
    asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(r), "l"(cc));
    asm("mov.b64 {%0, %1}, %2;" : "=f"(y0), "=f"(y1) : "l"(r));
}
// Bulk copies (TMA, no multicast) completed on a shared-memory mbarrier.
__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}
__device__ __forceinline__ void mbar_expect_tx(uint32_t bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes) : "memory");
}
// dst and src 16-byte aligned, bytes a multiple of 16.
__device__ __forceinline__ void bulk_copy_g2s(uint32_t dst, const void* src, uint32_t bytes, uint32_t bar) {
    asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(dst),
                 "l"(src), "r"(bytes), "r"(bar)
                 : "memory");
}
// Polls phase `parity` of the barrier at most `tries` times, each poll suspending the thread for at most
// about 1 us; true once the phase has completed.
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity, uint32_t tries) {
    for (uint32_t i = 0; i < tries; ++i) {
        uint32_t done;
        asm volatile(
            "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, 1000;\n selp.u32 %0, 1, 0, p;\n}"
            : "=r"(done)
            : "r"(bar), "r"(parity)
            : "memory");
        if (done) return true;
    }
    return false;
}
constexpr uint32_t kTableWaitTries = 1u << 14;

__device__ __forceinline__ void grid_dependency_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void grid_dependents_launch() { asm volatile("griddepcontrol.launch_dependents;"); }

// ------------------------------------------------------------------------- table expansion

// Magnitude class of a coded coordinate: 1 when m = floor(|v|), taken on hi, is at least 2.
__device__ __forceinline__ uint32_t mag_class(int hi, int b) {
    int m = hi >= 0 ? hi : -hi - b;
    return m >= 2 ? 1u : 0u;
}

// The fused entry of symbol `sym` of context c without its slot - cum field (bits 20-31).
__device__ __forceinline__ uint32_t entry_template(int c, int sym, uint32_t f) {
    int b = c == 0 ? (sym >> 6) : (c <= 4 ? (c - 1) >> 1 : (c - 5) >> 1);
    int idx = sym & 63, hi = idx - 31;
    uint32_t field, cls = 0;
    if (c <= 4) {
        field = uint32_t(2 * idx + b);                                // v = hi + b/2
        cls = idx == kEscIdx ? 1u : mag_class(hi, b);                 // an escape has |hi| >= 32
    } else {
        field = uint32_t(4 * idx + b);                                // 2h + b/2 (parity added later)
    }
    return ((f & 0xFFFu) << 8) | (c <= 4 ? (cls << 7) | field : field);
}

// A sequence's prepared entries (144 KB) arrive by nine bulk copies, issued by thread 0 and completed on
// the mbarrier `bar` (phase 0). The barrier must have been initialised, and the initialisation seen by
// every thread, before the call.
__device__ __forceinline__ void load_tables_bulk(const Params& p, uint8_t* tables, uint32_t bar) {
    if (threadIdx.x == 0) {
        mbar_expect_tx(bar, kTablesBytes);
        for (uint32_t c = 0; c < (p.test_no_table_copy ? 0u : kTablesBytes / kCtxBytes); ++c)
            bulk_copy_g2s(smem_addr(tables) + c * kCtxBytes, p.pre_tables + c * (kCtxBytes / 4), kCtxBytes, bar);
    }
}

// Starts the copy of the serialised tables (the first kScratchTableCap bytes of the section, zero past
// its end) into scratch, as one copy group. The section start is 16-byte aligned (header check).
__device__ __forceinline__ void stage_tables_async(const Params& p, uint8_t* scratch) {
    const uint32_t tlen = p.tables_len < kScratchTableCap ? p.tables_len : kScratchTableCap;
    const uint32_t off = 16 * threadIdx.x;
    if (off < kScratchTableCap) {
        const uint32_t n = off < tlen ? min(16u, tlen - off) : 0u;
        cp_async16(smem_addr(scratch + kScratchBytes + off), n ? p.blob + p.off_tables + off : p.blob, n);
    }
    cp_async_commit();
}

// Expands the serialised tables into the fused entries. The entry of slot t in a context is
// D[s] + (t << 20), where s is the symbol owning the slot (cum[s] <= t < cum[s] + f[s]) and
// D[s] = template[s] - (cum[s] << 20); D is never 0, since f >= 1 sits in bits 8-19. Three passes, no
// branching per slot:
//   1. zero the 144 KB (the serialised bytes were staged by stage_tables_async);
//   2. one thread per symbol unpacks its 12-bit frequency; warp scans prefix-sum them into cum, and
//      each symbol with f > 0 drops D[s] at slot cum[s] (the marker);
//   3. each thread takes 36 consecutive entries of the 9 x 4096, starts from the marker in force at its
//      first slot (a 7-step binary search over cum) and carries markers forward: entry = D + (slot << 20).
__device__ void build_tables(const Params& p, uint8_t* tables, uint8_t* scratch) {
    uint32_t* cum = reinterpret_cast<uint32_t*>(scratch + kScratchCum);    // [9][129]
    uint8_t* tbytes = scratch + kScratchBytes;
    uint32_t* dval = reinterpret_cast<uint32_t*>(scratch + kScratchTmpl);  // [9][128]: D[s]
    uint32_t* t32 = reinterpret_cast<uint32_t*>(tables);
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;

    // Pass 1. The serialised bytes were staged by stage_tables_async (the older of this thread's two
    // copy groups).
    {
        uint4* t4 = reinterpret_cast<uint4*>(tables);
        for (uint32_t i = tid; i < kTablesBytes / 16; i += kThreads) t4[i] = make_uint4(0u, 0u, 0u, 0u);
    }
    const uint32_t tlen = p.tables_len < kScratchTableCap ? p.tables_len : kScratchTableCap;
    cp_async_wait<1>();
    __syncthreads();

    // Pass 2: one thread per symbol. Threads 0-127 hold START, then 64 threads (two warps) per context
    // 1..8. A warp scan plus the sums of the context's earlier warps give cum.
    uint32_t* wsum = reinterpret_cast<uint32_t*>(scratch + kScratchWsum);
    const bool owner = tid < 128 + 8 * 64;
    const int c = tid < 128 ? 0 : 1 + (tid - 128) / 64;
    const int sym = tid < 128 ? tid : (tid - 128) & 63;
    const int A = c == 0 ? 128 : 64;
    uint32_t f = 0, incl = 0;
    if (owner) {
        const uint32_t lo = tbytes[c], cnt = tbytes[kNumCtx + c];
        uint32_t bit0 = 0;
#pragma unroll
        for (int k = 0; k < kNumCtx - 1; ++k) bit0 += k < c ? 12u * tbytes[kNumCtx + k] : 0u;
        const uint32_t bits_len = tlen > 2 * kNumCtx ? tlen - 2 * kNumCtx : 0;
        if (uint32_t(sym) >= lo && uint32_t(sym) < lo + cnt) {
            const uint32_t bit = bit0 + 12 * (uint32_t(sym) - lo), byte = bit >> 3;
            uint32_t w = 0;
#pragma unroll
            for (int k = 0; k < 3; ++k)
                if (byte + k < bits_len) w |= uint32_t(tbytes[2 * kNumCtx + byte + k]) << (8 * k);
            f = (w >> (bit & 7)) & 0xFFFu;
        }
        incl = f;
#pragma unroll
        for (int d = 1; d < 32; d <<= 1) {
            const uint32_t v = __shfl_up_sync(kFullMask, incl, d);
            if (lane >= d) incl += v;
        }
        if (lane == 31) wsum[warp] = incl;
    }
    __syncthreads();
    if (owner) {
        // Earlier warps of the same context: warps 0..3 hold START, warps 4+2(c-1) and 5+2(c-1) context c.
        const int first = c == 0 ? 0 : 4 + 2 * (c - 1);
        for (int w = first; w < warp; ++w) incl += wsum[w];
        const uint32_t acc = incl - f;  // cum[sym]
        const uint32_t d = entry_template(c, sym, f) - (acc << 20);
        uint32_t* cc = cum + c * 129;
        cc[sym] = acc;
        dval[c * 128 + sym] = d;
        if (f != 0 && acc < kProbScale) t32[block_of(c) / 4 + acc] = d;
        if (sym == A - 1) {
            cc[A] = incl;
            if (A < 128) cc[128] = incl;
            const uint32_t cnt = tbytes[kNumCtx + c];
            const bool ok = cnt == 0 ? incl == 0 : (incl == kProbScale && cnt >= 2);
            if (!ok && blockIdx.x == 0) atomicOr(&g_status, int(EP_DEV_BAD_TABLES));
        }
    }
    __syncthreads();

    // Pass 3. The 9 blocks are contiguous (contexts 1..8, then START): one run of 9 x 4096 entries.
    // Lane stride 144 B = 36 words and 36 = 4 (mod 32), so the 8 lanes of a quarter-warp cover all 32
    // banks once per 16-byte access.
    {
        constexpr uint32_t kPer = kNumCtx * 4096 / kThreads;
        static_assert(kPer * kThreads == kNumCtx * 4096 && kPer % 4 == 0, "fill geometry");
        const uint32_t gfirst = uint32_t(tid) * kPer;
        const uint32_t blk = gfirst >> 12;                   // memory block: contexts 1..8, then START
        const int c = blk == 8 ? 0 : int(blk) + 1, A = c == 0 ? 128 : 64;
        const uint32_t* cc = cum + c * 129;
        const uint32_t slot0 = gfirst & 4095u;
        int s = 0;
#pragma unroll
        for (int step = 64; step >= 1; step >>= 1)           // largest s < A with cum[s] <= slot0
            if (s + step < A && cc[s + step] <= slot0) s += step;
        uint32_t d = dval[c * 128 + s];
        uint4* run = reinterpret_cast<uint4*>(tables + 4 * gfirst);
#pragma unroll 3
        for (uint32_t q = 0; q < kPer / 4; ++q) {
            uint4 v = run[q];
            const uint32_t t = (gfirst + 4 * q) << 20;      // slot of v.x, in bits 20-31
            d = v.x ? v.x : d;
            v.x = d + t;
            d = v.y ? v.y : d;
            v.y = d + t + (1u << 20);
            d = v.z ? v.z : d;
            v.z = d + t + (2u << 20);
            d = v.w ? v.w : d;
            v.w = d + t + (3u << 20);
            run[q] = v;
        }
    }
    __syncthreads();
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

// ------------------------------------------------------------------------- per-warp state

// Row of the lane's current group. c_row = fl32(s_row / alpha) is recomputed only when the row changes.
struct RowCursor {
    uint32_t row, col;
    float c_row;

    // s / alpha correctly rounded: q0 = s * RN(1/alpha) corrected once with the exact residual
    // s - alpha * q0 (Markstein). This matches IEEE division for every bf16 s >= 2^-96 with a quotient
    // in [2^-96, 2^96] (checked exhaustively over all such s for thousands of alphas). Anything else,
    // zero rows included, takes the IEEE division.
    template <class P>
    static __device__ __forceinline__ float scale_of(const P& p, const uint16_t* scales, uint32_t r) {
        const float s = __uint_as_float(uint32_t(__ldg(scales + r)) << 16);
        const float q0 = __fmul_rn(s, p.inv_alpha);
        const float q = __fmaf_rn(__fmaf_rn(-p.alpha, q0, s), p.inv_alpha, q0);
        return (s >= 0x1p-96f && q >= 0x1p-96f && q <= 0x1p96f) ? q : __fdiv_rn(s, p.alpha);
    }
    template <class P>
    __device__ __forceinline__ void load_scale(const P& p, const uint16_t* scales) {
        if (row >= p.M) return;  // lanes past the last group
        c_row = scale_of(p, scales, row);
    }
    template <class P>
    __device__ __forceinline__ void start(const P& p, const uint16_t* scales, uint32_t g) {
        row = g / p.gpr;
        col = g - row * p.gpr;
        c_row = 0.f;
        load_scale(p, scales);
    }
    // Next round: 32 groups further. The scale is reloaded only when the row changes.
    template <class P>
    __device__ __forceinline__ void advance(const P& p, const uint16_t* scales) {
        col += 32;
        if (col >= p.gpr) {
            col -= p.gpr;
            ++row;
            while (col >= p.gpr) { col -= p.gpr; ++row; }  // rows narrower than 32 groups
            load_scale(p, scales);
        }
    }
    __device__ __forceinline__ float scale() const { return c_row; }
};

// The tile's u16 word stream, read either from the warp's shared ring (all but ragged rounds) or
// straight from global memory with a bounds check. `pb` is the byte position of the next word in
// ring coordinates (lead + 2 * words consumed).
struct RingWords {
    uint32_t base;  // shared address of the warp's ring, kRingBytes-aligned
    __device__ __forceinline__ uint32_t at(uint32_t pb) const { return ld_shared_u16((pb & (kRingBytes - 1)) | base); }
};
struct GlobalWords {
    const uint8_t* ring0;  // global address that ring coordinate 0 mirrors
    uint32_t lo, hi;       // valid ring coordinates of the stream: [lo, hi)
    __device__ __forceinline__ uint32_t at(uint32_t pb) const {
        return (pb >= lo && pb + 2 <= hi) ? uint32_t(__ldg(reinterpret_cast<const uint16_t*>(ring0 + pb))) : 0u;
    }
};

struct TileState {
    uint32_t x;   // rANS state of this lane
    uint32_t pb;  // ring coordinate of the next stream word
};

// ------------------------------------------------------------------------------ one round

// One symbol step: the fused entry for the current context block B, the state update and the
// refill from the shared word stream. Returns the entry.
template <bool PARTIAL, class Words>
__device__ __forceinline__ uint32_t symbol_step(uint32_t B, const Words& words, uint32_t& x, uint32_t& pb,
                                                bool active, uint32_t lt_mask) {
    uint32_t e = 0;
    if (!PARTIAL || active) {
        e = ld_shared_u32(B + ((x & (kProbScale - 1)) << 2));
        x = ((e >> 8) & 0xFFFu) * (x >> kProbBits) + (e >> 20);  // f * (x >> 12) + slot - cum
    }
    const bool need = (!PARTIAL || active) && x < kRansL;
    const uint32_t m = __ballot_sync(kFullMask, need);
    const uint32_t w = words.at(pb + 2 * __popc(m & lt_mask));
    // x = need ? (x << 16) | w : x, as one byte permute: bytes (w0, w1, x0, x1) or x unchanged.
    x = __byte_perm(x, w, need ? 0x1054u : 0x3210u);
    pb += 2 * __popc(m);
    return e;
}

// Symbol step of the fast rounds. The refill is a predicated byte permute; address arithmetic runs as
// integer multiply-adds. WRAP = false: the whole stream sits in the warp's ring without wrapping and `pa` is the shared
// address of the next word itself. WRAP = true: `pa` is a ring coordinate, taken modulo the ring.
template <bool WRAP>
__device__ __forceinline__ uint32_t symbol_step_fast(const Params& p, uint32_t B, uint32_t& x, uint32_t& pa,
                                                     uint32_t ring_base, uint32_t lt_mask) {
    const uint32_t q = x >> kProbBits;
    const uint32_t e = ld_shared_u32((x + q * p.kneg4096) * p.k4 + B);  // B + 4 (x mod 4096)
    x = ((e >> 8) & 0xFFFu) * q + (e >> 20);                     // f * (x >> 12) + slot - cum
    const bool need = x < kRansL;
    const uint32_t m = __ballot_sync(kFullMask, need);
    const uint32_t wp = pa + __popc(m & lt_mask) * p.k2;
    const uint32_t w = ld_shared_u16(WRAP ? (wp & (kRingBytes - 1)) | ring_base : wp);
    if (need) x = __byte_perm(x, w, 0x1054u);                    // (x << 16) | w
    pa += __popc(m) * p.k2;
    return e;
}

// Raw low bits of group q: the r bytes at q*r of the tile's raw section, as the four aligned words that
// cover them (zero past the section) and the bit offset of the first one.
struct RawWindow {
    uint32_t w[4], sh;
    __device__ __forceinline__ void load(const uint8_t* rawsec, uint32_t raw_avail, uint32_t q, uint32_t r) {
        const uint32_t o = q * r, a = o & ~3u;
        sh = (o & 3u) * 8;
#pragma unroll
        for (int j = 0; j < 4; ++j)
            w[j] = (a + 4 * j + 4 <= raw_avail) ? __ldg(reinterpret_cast<const uint32_t*>(rawsec + a) + j) : 0u;
    }
    // Bits [i r, i r + r) of the group's 8r-bit field, LSB first.
    __device__ __forceinline__ uint32_t lo(int i, uint32_t r) const {
        const uint32_t bp = uint32_t(i) * r + sh, sel = bp >> 5, s = bp & 31;
        const uint32_t wa = sel == 0 ? w[0] : (sel == 1 ? w[1] : (sel == 2 ? w[2] : w[3]));
        const uint32_t wb = sel == 0 ? w[1] : (sel == 1 ? w[2] : w[3]);
        return __funnelshift_r(wa, wb, s) & ((1u << r) - 1u);
    }
};

// Fast round: every lane holds a group, the tile has no escapes, and the round's words are in the ring.
// Values come from the entries' value fields. RAW: the tile carries r >= 1 raw low bits per coordinate,
// taken from `raw` (loaded a round ahead); then t = hi 2^r + lo and the parity of u_0..u_6 is that of
// the lo's. WAIT: the warp's first stores of the launch; they wait for the previous launch of a sequence.
template <int MODE, bool WRAP, bool RAW = false, bool WAIT = false>
__device__ __forceinline__ void round_fast(const Params& p, uint32_t t0, uint32_t& x, uint32_t& pa, uint32_t ring_base,
                                           uint32_t g, uint32_t lt_mask, const RowCursor& rc,
                                           const RawWindow* raw = nullptr) {
    uint32_t e[8];
    e[0] = symbol_step_fast<WRAP>(p, t0 + kStartOffset, x, pa, ring_base, lt_mask);
    // Entry bits 0 (coset bit b of START) and 7 (class) land on block bits 15 and 14.
    const uint32_t gbase = t0 + ((e[0] << 15) & 0x8000u);
    const uint32_t gbase7 = gbase + kPos7Offset;
    uint32_t par = e[0];
    uint32_t B = gbase | ((e[0] << 7) & 0x4000u);
#pragma unroll
    for (int i = 1; i < 8; ++i) {
        e[i] = symbol_step_fast<WRAP>(p, B, x, pa, ring_base, lt_mask);
        if (i < 7) {
            par ^= e[i];
            B = (i == 6 ? gbase7 : gbase) | ((e[i] * p.k128) & 0x4000u);
        }
    }

    const float c = rc.scale();
    float m[8], y[8];
    int32_t z[8];
    float K, K7;
    if constexpr (!RAW) {
        // Entry bit 1 is the parity of idx; u_i = idx_i - 31 flips it, and seven flips make
        // pi = 1 - (XOR of the idx parities).
        const uint32_t two_pi = ~par & 2u;
#pragma unroll
        for (int i = 0; i < 7; ++i) m[i] = __uint_as_float((e[i] & 0x7Fu) | kHalfMagic);     // 1.5*2^22 + idx + b/2
        m[7] = __uint_as_float(((e[7] & 0xFFu) | kHalfMagic) + two_pi);                      // 1.5*2^22 + 2 idx + b/2 + pi
        // v = m - (1.5*2^22 + 31) for positions 0..6 and m - (1.5*2^22 + 62) for 7: exact.
        K = kHalfMagicF + 31.0f;
        K7 = kHalfMagicF + 62.0f;
    } else {
        // m_i = 1.5*2^22 + idx 2^r + lo + b/2 (i < 7); m_7 = 1.5*2^22 + 2 (idx 2^r + lo_7) + pi + b/2, with
        // pi = XOR of the lo's lowest bits. v = m - (1.5*2^22 + 31 2^r) or m - (1.5*2^22 + 62 2^r): exact,
        // since every field stays below 2^22 for r <= 12.
        const uint32_t r = uint32_t(p.r);
        uint32_t lpar = 0;
#pragma unroll
        for (int i = 0; i < 7; ++i) {
            const uint32_t lo = raw->lo(i, r);
            lpar ^= lo;
            m[i] = __uint_as_float(kHalfMagic + ((e[i] & 0x7Eu) << r) + (lo << 1) + (e[i] & 1u));
        }
        const uint32_t lo7 = raw->lo(7, r);
        m[7] = __uint_as_float(kHalfMagic + ((e[7] & 0xFCu) << r) + (lo7 << 2) + ((lpar & 1u) << 1) + (e[7] & 1u));
        const float sc = float(1u << r);
        K = kHalfMagicF + 31.0f * sc;
        K7 = kHalfMagicF + 62.0f * sc;
    }
    // y = v * c_row, two coordinates per instruction.
#pragma unroll
    for (int i = 0; i < 6; i += 2) sub_mul_f32x2(m[i], m[i + 1], K, K, c, y[i], y[i + 1]);
    sub_mul_f32x2(m[6], m[7], K, K7, c, y[6], y[7]);
    if constexpr (MODE == kCoords) {
#pragma unroll
        for (int i = 0; i < 8; ++i) z[i] = __float2int_rn((m[i] - (i < 7 ? K : K7)) * 2.0f);
    }
    if constexpr (WAIT) grid_dependency_wait();
    store_group<MODE>(p.dst, g, y, z);
}

// General round: escapes, raw low bits and ragged rounds (PARTIAL: some lanes hold no group).
template <int MODE, bool PARTIAL, class Words>
__device__ __forceinline__ void round_general(const Params& p, uint32_t t0, const Words& words, const uint8_t* rawsec,
                                              uint32_t raw_avail, const uint16_t* scales, TileState& st, uint32_t q,
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
    uint32_t x = st.x, pb = st.pb;
    uint32_t B = t0 + kStartOffset, gbase = t0, b = 0;
    int32_t t[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        const uint32_t e = symbol_step<PARTIAL>(B, words, x, pb, active, lt_mask);
        // idx: entry bits 1-6 (field 2 idx + b) for positions 0..6, bits 2-7 (4 idx + b) for 7.
        const uint32_t idx = i < 7 ? (e >> 1) & 63u : (e >> 2) & 63u;
        int32_t hi = int32_t(idx) - 31;
        const bool esc = (!PARTIAL || active) && idx == uint32_t(kEscIdx);
        const uint32_t me = __ballot_sync(kFullMask, esc);
        if (me) {
            const uint32_t ew = words.at(pb + 2 * __popc(me & lt_mask));
            if (esc) hi = int32_t(int16_t(ew));
            pb += 2 * __popc(me);
        }
        if (i == 0) {
            b = e & 1u;
            gbase = t0 + (b << 15);
        }
        int32_t lo = 0;
        if (r > 0) {
            const uint32_t bp = uint32_t(i) * uint32_t(r), sel = bp >> 5, sh = bp & 31;
            const uint32_t wa = sel == 0 ? win0 : (sel == 1 ? win1 : win2);
            const uint32_t wb = sel == 0 ? win1 : win2;
            lo = int32_t(__funnelshift_r(wa, wb, sh) & ((1u << r) - 1u));
        }
        t[i] = hi * (1 << r) + lo;
        if (i < 7) B = (gbase + (i == 6 ? kPos7Offset : 0u)) | ((e << 7) & 0x4000u);
    }
    st.x = x;
    st.pb = pb;
    if (PARTIAL && !active) return;

    int32_t s7 = 0;
#pragma unroll
    for (int i = 0; i < 7; ++i) s7 += t[i];
    const float c = rc.scale();
    float y[8];
    int32_t z[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        const int32_t u = i < 7 ? t[i] : 2 * t[7] + (s7 & 1);
        z[i] = 2 * u + int32_t(b);
        y[i] = __fmul_rn(__int2float_rn(z[i]) * 0.5f, c);
    }
    store_group<MODE>(p.dst, g, y, z);
}

// ------------------------------------------------------------------------------ tiles

// Geometry of one tile, from its payload offsets. Returns false when the offsets are malformed.
struct TileGeom {
    uint64_t start;                  // payload byte offset of the tile
    uint32_t tile_bytes, g0, ng;     // size, first group, groups held
    uint32_t a0, lead, span, chunks;  // ring coordinate 0 mirrors tile byte a0; the stream starts at `lead`
    bool esc, simple, raw;           // escapes present; no escapes and r = 0; no escapes and r > 0
};

__device__ __forceinline__ bool tile_geometry(const Params& p, const uint32_t* toff, uint32_t tile, uint32_t per_tile,
                                              TileGeom& tg) {
    const uint32_t e0 = __ldg(toff + tile), e1 = __ldg(toff + tile + 1);
    const uint64_t start = uint64_t(e0 & 0x7FFFFFFFu) * 16, end = uint64_t(e1 & 0x7FFFFFFFu) * 16;
    tg.g0 = tile * per_tile;
    tg.ng = min(per_tile, p.NG - tg.g0);
    const uint32_t raw = (tg.ng * uint32_t(p.r) + 3u) & ~3u;
    if (end < start || end > p.payload_bytes || end - start < 128ull + raw || end - start > 0x7FFFFFF0ull) return false;
    tg.start = start;
    tg.tile_bytes = uint32_t(end - start);
    const uint32_t s0 = 128 + raw;
    tg.a0 = s0 & ~15u;
    tg.lead = s0 - tg.a0;
    tg.span = tg.tile_bytes - tg.a0;
    tg.chunks = (tg.span + kChunkBytes - 1) / kChunkBytes;
    tg.esc = e0 >> 31;
    tg.simple = !tg.esc && p.r == 0;
    tg.raw = !tg.esc && p.r > 0;
    return true;
}

// Lane L's 16-byte share of ring chunk c of the tile (zero-filled past the tile's end).
__device__ __forceinline__ void issue_chunk(const uint8_t* payload, const TileGeom& tg, uint32_t c, uint32_t ring_base,
                                            uint32_t lane) {
    const uint32_t off = c * kChunkBytes + 16 * lane;
    const uint32_t n = off < tg.span ? min(16u, tg.span - off) : 0u;
    const uint8_t* tp = payload + tg.start;
    cp_async16(ring_base + (off & (kRingBytes - 1)), n ? tp + tg.a0 + off : tp, n);
}

// Fast rounds with no wrap, for tiles without escapes (RAW: with r >= 1 raw low bits). pa is the shared
// address of the next word, and a round reads at most 512 bytes past it. When the stream fits the ring,
// a valid stream ends inside it, and a corrupt one is stopped at the first round boundary past the ring's
// end: reads stay within 512 bytes of it, still inside the CTA's shared memory (the scratch region
// follows the last ring). A longer stream runs here while a round cannot reach the ring's end, and its
// next chunk is copied into the slot the rounds have left behind. The raw window of the next round is
// loaded while the current one decodes. Returns the number of rounds done. If `waited` is false, the
// first round waits for the previous launch of a sequence before its stores, and sets it.
template <int MODE, bool RAW>
__device__ __forceinline__ uint32_t fast_rounds(const Params& p, uint32_t t0, const TileGeom& tg, const uint8_t* payload,
                                                uint32_t ring_base, uint32_t lane, uint32_t lt_mask,
                                                const uint16_t* scales, RowCursor& rc, TileState& st, uint32_t& issued,
                                                const uint8_t* rawsec, uint32_t raw_avail, bool& waited) {
    const uint32_t Rf = tg.ng / 32, r = uint32_t(p.r);
    const uint32_t pa_lim = ring_base + (tg.chunks <= kRingChunks ? kRingBytes : kRingBytes - 2 * kRoundWords);
    uint32_t k = 0, g = tg.g0 + lane, x = st.x, pa = ring_base + st.pb;
    RawWindow cur, nxt;
    if (RAW) cur.load(rawsec, raw_avail, lane, r);
    if (!waited && Rf > 0 && pa <= pa_lim) {
        // Round 0 decodes while the previous launch may still be running; only its stores wait. No chunk
        // is due yet: the first kRingChunks chunks were issued with the tile.
        if (RAW) nxt.load(rawsec, raw_avail, 32 + lane, r);
        round_fast<MODE, false, RAW, true>(p, t0, x, pa, 0, g, lt_mask, rc, &cur);
        rc.advance(p, scales);
        if (RAW) cur = nxt;
        waited = true;
        k = 1;
        g += 32;
    }
    if (tg.chunks <= kRingChunks) {
        for (; k < Rf && pa <= pa_lim; ++k, g += 32) {
            if (RAW) nxt.load(rawsec, raw_avail, 32 * (k + 1) + lane, r);
            round_fast<MODE, false, RAW>(p, t0, x, pa, 0, g, lt_mask, rc, &cur);
            rc.advance(p, scales);
            if (RAW) cur = nxt;
        }
    } else {
        for (; k < Rf && pa <= pa_lim; ++k, g += 32) {
            if (issued < tg.chunks && pa >= ring_base + (issued - (kRingChunks - 1)) * kChunkBytes) {
                __syncwarp();  // every lane is done reading the slot
                issue_chunk(payload, tg, issued, ring_base, lane);
                cp_async_commit();
                ++issued;
            }
            if (RAW) nxt.load(rawsec, raw_avail, 32 * (k + 1) + lane, r);
            round_fast<MODE, false, RAW>(p, t0, x, pa, 0, g, lt_mask, rc, &cur);
            rc.advance(p, scales);
            if (RAW) cur = nxt;
        }
    }
    st.x = x;
    st.pb = pa - ring_base;
    return k;
}

// ---------------------------------------------------------------------------------- kernel

// Fused entries of a sequence of blobs, built once per (blob, context) instead of once per CTA. Block
// (layer, c) unpacks context c's frequencies, accumulates cum, checks the table and writes the 4096
// entries of its block: entry(t) = template[s] + ((t - cum[s]) << 20) for the symbol s owning slot t,
// the same words as build_tables.
constexpr int kMaxExpandJobs = 512;
struct ExpandArgs {
    const uint8_t* tables[kMaxExpandJobs];  // tables section of each blob (16-byte aligned)
    uint32_t tables_len[kMaxExpandJobs];
    uint32_t* out;                          // count x 9 x 4096 words
    int count;
};

__global__ void __launch_bounds__(256) expand_tables_kernel(const ExpandArgs a) {
    __shared__ uint8_t bytes[kScratchTableCap];
    __shared__ uint32_t cum[129], tmpl[128];
    const int layer = blockIdx.x / kNumCtx, c = blockIdx.x % kNumCtx, tid = threadIdx.x;
    if (layer >= a.count) return;
    const uint32_t tlen = a.tables_len[layer] < kScratchTableCap ? a.tables_len[layer] : kScratchTableCap;
    for (uint32_t i = tid; i < kScratchTableCap; i += blockDim.x) bytes[i] = i < tlen ? __ldg(a.tables[layer] + i) : 0;
    __syncthreads();
    const int A = c == 0 ? 128 : 64;
    const uint32_t lo = bytes[c], cnt = bytes[kNumCtx + c];
    if (tid < 128) {
        uint32_t bit0 = 0;
        for (int k = 0; k < c; ++k) bit0 += 12u * bytes[kNumCtx + k];
        const uint32_t bits_len = tlen > 2 * kNumCtx ? tlen - 2 * kNumCtx : 0;
        uint32_t f = 0;
        if (tid < A && uint32_t(tid) >= lo && uint32_t(tid) < lo + cnt) {
            const uint32_t bit = bit0 + 12 * (uint32_t(tid) - lo), byte = bit >> 3;
            uint32_t w = 0;
            for (int k = 0; k < 3; ++k)
                if (byte + k < bits_len) w |= uint32_t(bytes[2 * kNumCtx + byte + k]) << (8 * k);
            f = (w >> (bit & 7)) & 0xFFFu;
        }
        tmpl[tid] = f;  // the frequency for now; the template once cum is known
    }
    __syncthreads();
    if (tid == 0) {
        uint32_t acc = 0;
        for (int s = 0; s < A; ++s) { cum[s] = acc; acc += tmpl[s]; }
        cum[A] = acc;
        const bool ok = cnt == 0 ? acc == 0 : (acc == kProbScale && cnt >= 2);
        if (!ok) atomicOr(&g_status, int(EP_DEV_BAD_TABLES));
    }
    __syncthreads();
    if (tid < A) tmpl[tid] = entry_template(c, tid, tmpl[tid]);
    __syncthreads();
    // 16 consecutive slots per thread: a binary search for the owner of the first, then a walk.
    uint32_t* out = a.out + size_t(layer) * (kTablesBytes / 4) + block_of(c) / 4;
    const uint32_t first = 16 * uint32_t(tid);
    int s = 0;
    for (int step = 64; step >= 1; step >>= 1)
        if (s + step < A && cum[s + step] <= first) s += step;
    for (uint32_t t = first; t < first + 16; ++t) {
        while (s + 1 < A && t >= cum[s + 1]) ++s;
        out[t] = tmpl[s] + ((t - cum[s]) << 20);
    }
}

template <int MODE>
__global__ void __launch_bounds__(kThreads, 1) decode_kernel(const Params p) {
    extern __shared__ __align__(16) uint8_t smem_raw[];
    // Rings must be kRingBytes-aligned in the shared window so that ring addresses are (offset | base).
    const uint32_t raw_base = smem_addr(smem_raw);
    const uint32_t tbl_pad = (kTableAlign - (raw_base & (kTableAlign - 1))) & (kTableAlign - 1);
    uint8_t* tables = smem_raw + tbl_pad;
    const uint32_t gap_lead = (kRingBytes - (raw_base & (kRingBytes - 1))) & (kRingBytes - 1);
    const uint32_t gap_rings = tbl_pad >= gap_lead ? (tbl_pad - gap_lead) / kRingBytes : 0u;
    const uint32_t rings_before = gap_rings < uint32_t(kWarps) ? gap_rings : uint32_t(kWarps);
    uint8_t* rings_after = tables + kTablesBytes;
    uint8_t* scratch = rings_after + (kWarps - rings_before) * kRingBytes;
    const uint32_t t0 = smem_addr(tables);

    const uint32_t lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const uint32_t lt_mask = (1u << lane) - 1u;
    const uint16_t* scales = reinterpret_cast<const uint16_t*>(p.blob + p.off_scales);
    const uint32_t* toff = reinterpret_cast<const uint32_t*>(p.blob + p.off_offsets);
    const uint8_t* payload = p.blob + p.off_payload;
    const uint32_t per_tile = 32 * p.G;
    const RingWords ring{smem_addr(warp < rings_before ? smem_raw + gap_lead + warp * kRingBytes
                                                       : rings_after + (warp - rings_before) * kRingBytes)};

    grid_dependents_launch();  // lets the next launch of a sequence start its prologue early
    const uint32_t bar = smem_addr(scratch);  // the build scratch is unused when the tables are prepared
    if (p.pre_tables) {
        if (threadIdx.x == 0) mbar_init(bar, 1);
        __syncthreads();
        load_tables_bulk(p, tables, bar);
    } else {
        stage_tables_async(p, scratch);
    }

    // The next layer's metadata (tables, tile offsets, scales) goes to L2 now, so its prologue reads L2.
    if (p.next_blob) {
        const uint32_t lines = (p.next_meta_bytes + 127) / 128;
        for (uint32_t l = blockIdx.x + gridDim.x * threadIdx.x; l < lines; l += gridDim.x * kThreads)
            prefetch_l2(p.next_blob + p.next_meta_off + 128ull * l);
    }

    // Tiles are dealt round-robin over the CTAs first, so that consecutive tiles land on different SMs
    // and a partial last wave is spread over the whole GPU: tile = (k * kWarps + warp) * grid + block.
    // The copies of the warp's first tile are issued before the table build, which hides them. Every
    // thread commits exactly one group here (empty without a first tile), behind the tables' group when
    // the tables are built here.
    uint32_t slot = warp;
    bool first_issued = false;
    {
        const uint32_t tile = slot * gridDim.x + blockIdx.x;
        if (tile < p.T) {
            TileGeom tg;
            if (tile_geometry(p, toff, tile, per_tile, tg)) {
                const uint32_t first = min(tg.chunks, kRingChunks);
                for (uint32_t c = 0; c < first; ++c) issue_chunk(payload, tg, c, ring.base, lane);
                first_issued = true;
            }
        }
        cp_async_commit();
    }
    bool tables_ok = true;
    if (p.pre_tables) {
        // The first tile's copies may still be in flight. A copy that has not landed after the bounded
        // wait flags the launch, and the CTA decodes nothing (after a second bounded wait, so that no
        // copy still writes into its shared memory when it exits).
        const bool ok = mbar_wait(bar, 0, kTableWaitTries);
        if (__syncthreads_or(!ok)) {
            if (threadIdx.x == 0) atomicOr(&g_status, int(EP_DEV_TABLE_COPY));
            mbar_wait(bar, 0, kTableWaitTries);
            tables_ok = false;
        }
    } else {
        build_tables(p, tables, scratch);
    }
    // Stores may overwrite what the previous launch of a sequence wrote, so each warp waits for it
    // before its first store: after decoding its first round, when that round is a fast one.
    bool waited = false;

    for (; tables_ok; slot += kWarps) {
        const uint32_t tile = slot * gridDim.x + blockIdx.x;
        if (tile >= p.T) break;
        TileGeom tg;
        if (!tile_geometry(p, toff, tile, per_tile, tg)) {
            if (lane == 0) atomicOr(&g_status, int(EP_DEV_BAD_OFFSETS));
            first_issued = false;
            continue;
        }
        const uint8_t* tp = payload + tg.start;
        TileState st;
        st.x = __ldg(reinterpret_cast<const uint32_t*>(tp) + lane);
        st.pb = tg.lead;
        const GlobalWords gwords{tp + tg.a0, tg.lead, tg.span};

        // Pull the first 4 KB of this warp's next tile toward L2 while this one decodes.
        {
            const uint32_t next = tile + kWarps * gridDim.x;
            if (next < p.T) {
                const uint64_t ns = uint64_t(__ldg(toff + next) & 0x7FFFFFFFu) * 16 + 128ull * lane;
                if (ns < p.payload_bytes) prefetch_l2(payload + ns);
            }
        }

        RowCursor rc;
        rc.start(p, scales, tg.g0 + lane);
        const uint8_t* rawsec = tp + 128;
        const uint32_t raw_avail = tg.tile_bytes - 128;
        const uint32_t R = (tg.ng + 31) / 32;

        // The first 2 KB of the stream (all of it for most tiles at 4 bpp) fill the ring in one batch.
        const uint32_t first = min(tg.chunks, kRingChunks);
        if (!first_issued) {
            for (uint32_t c = 0; c < first; ++c) issue_chunk(payload, tg, c, ring.base, lane);
            cp_async_commit();
        }
        first_issued = false;
        cp_async_wait<0>();
        __syncwarp();
        uint32_t issued = first, k = 0;

        if (!tg.esc) {
            k = tg.raw ? fast_rounds<MODE, true>(p, t0, tg, payload, ring.base, lane, lt_mask, scales, rc, st, issued,
                                                 rawsec, raw_avail, waited)
                       : fast_rounds<MODE, false>(p, t0, tg, payload, ring.base, lane, lt_mask, scales, rc, st, issued,
                                                  rawsec, raw_avail, waited);
        }

        if (k < R) {
            if (!waited) {
                grid_dependency_wait();
                waited = true;
            }
            // Rolling ring: tiles with escapes or raw bits, the last rounds of a stream longer than the
            // ring, and the ragged last round. Up to three chunks in flight; one more per round while the
            // chunk it replaces lies wholly behind pb.
            cp_async_wait<0>();
            __syncwarp();
            uint32_t h0 = issued, h1 = issued, h2 = issued;
            const uint32_t round_bytes = 2 * (tg.esc ? kRoundWordsEsc : kRoundWords);
            for (; k < R; ++k) {
                if (issued < tg.chunks && issued <= st.pb / kChunkBytes + (kRingChunks - 1)) {
                    __syncwarp();  // every lane is done reading the slot
                    issue_chunk(payload, tg, issued, ring.base, lane);
                    ++issued;
                }
                cp_async_commit();
                h2 = h1; h1 = h0; h0 = issued;
                cp_async_wait<2>();  // chunks [0, h2) have landed
                uint32_t ready = h2 == tg.chunks ? 0xFFFFFFFFu : h2 * kChunkBytes;
                if (st.pb + round_bytes > ready) {
                    cp_async_wait<0>();
                    ready = issued == tg.chunks ? 0xFFFFFFFFu : issued * kChunkBytes;
                }
                __syncwarp();
                const uint32_t q = 32 * k + lane, g = tg.g0 + q;
                const bool full = 32 * k + 32 <= tg.ng;
                const bool in_ring = st.pb + round_bytes <= ready;
                if (full && in_ring) {
                    if (tg.simple) {
                        round_fast<MODE, true>(p, t0, st.x, st.pb, ring.base, g, lt_mask, rc);
                    } else if (!tg.esc) {
                        RawWindow rw;
                        rw.load(rawsec, raw_avail, q, uint32_t(p.r));
                        round_fast<MODE, true, true>(p, t0, st.x, st.pb, ring.base, g, lt_mask, rc, &rw);
                    } else {
                        round_general<MODE, false>(p, t0, ring, rawsec, raw_avail, scales, st, q, true, g, lt_mask, rc);
                    }
                } else {
                    round_general<MODE, true>(p, t0, gwords, rawsec, raw_avail, scales, st, q, q < tg.ng, g, lt_mask,
                                              rc);
                }
                rc.advance(p, scales);
            }
        }
        cp_async_wait<0>();  // the ring is reused by this warp's next tile
        __syncwarp();
        const uint32_t used = st.pb - tg.lead, cap = tg.span - tg.lead;  // bytes of stream read / present
        const bool ok = __all_sync(kFullMask, st.x == kRansL) && used <= cap && cap - used <= 14;
        if (!ok && lane == 0) atomicOr(&g_status, int(EP_DEV_CORRUPT_TILE));
    }
    if (first_issued) cp_async_wait<0>();
    // A launch of a sequence ends after the one before it, whether or not this warp stored anything.
    if (!waited) grid_dependency_wait();
}


// ===================================================================== format version 2
//
// Version 2 codes the same coordinates with 8-bit frequencies, so one renormalisation serves a pair of
// symbols (positions 0-1, 2-3, 4-5, 6-7): from a state in [2^16, 2^32), two symbols take at most 16 bits,
// and one 16-bit word restores the range. The tables are 9 contexts x 256 slots of 4-byte fused entries,
// 9 KB, which each CTA builds in about a microsecond. Rare symbols are escapes; their words follow the
// round's fourth pair and are read only when some lane of the warp met one.
namespace v2 {

// Fused entry of one slot: value field (bits 0-7: 2 idx + b at positions 0..6, 4 idx + b at position 7),
// escape flag (bit 9), magnitude class of the coordinate (bit 10, picks the next context's 1 KB block),
// coset bit b (bit 11, START only: picks the b half), f (bits 16-23) and slot - cum (bits 24-31).
constexpr uint32_t kEscBit = 1u << 9;
constexpr uint32_t kClassBit = 1u << 10;
constexpr uint32_t kCosetBit = 1u << 11;
constexpr uint32_t kPos7Bit = 1u << 12;
// Blocks: contexts 1..8 at (c - 1) KB, so (b, class) select bits 11 and 10 and position 7 adds bit 12;
// START at 8 KB. The region sits on a 16 KB boundary of the shared window, so the bits combine by OR.
constexpr uint32_t kCtxBytes = 256 * 4;
constexpr uint32_t kStartOffset = 8 * kCtxBytes;
constexpr uint32_t kTablesBytes = 9 * kCtxBytes;
constexpr uint32_t kTableAlign = 16 * 1024;
__host__ __device__ constexpr uint32_t block_of(int c) { return c == 0 ? kStartOffset : uint32_t(c - 1) * kCtxBytes; }

// Warps per CTA: one CTA per SM.
constexpr int kWarpsV2 = 32;
constexpr int kThreadsV2 = kWarpsV2 * 32;

// Per-warp tile buffers: 5 KB. A tile is copied whole (states, raw bits, word stream) into its warp's buffer,
// at the bottom or the top. While a warp decodes one tile, the copy of its next tile lands at the other end
// when the two fit together (about 4.4 KB at 4 bits per coordinate), so the next tile's data is there when
// the warp gets to it. Tiles larger than the buffer are read from global memory by the general rounds.
constexpr uint32_t kRingBytes = 5 * 1024;
constexpr uint32_t kRingsBytes = kWarpsV2 * kRingBytes;
// Scratch of the table build: f and cum per context and symbol (u16), and the staged table bytes.
constexpr uint32_t kScratchF = 0;                               // u16 [9][128]
constexpr uint32_t kScratchCum = kScratchF + kNumCtx * 128 * 2; // u16 [9][129]
constexpr uint32_t kScratchBytesOff = (kScratchCum + kNumCtx * 129 * 2 + 15) & ~15u;
constexpr uint32_t kScratchTableCap = 1024;                     // a valid blob's tables take 658 bytes at most
constexpr uint32_t kScratchSize = kScratchBytesOff + kScratchTableCap;
// [pad to 16 B][rings][pad to 16 KB][tables][scratch][slack]. At least kOverrunBytes follow the last ring.
constexpr uint32_t kSlackBytes = 6 * 1024;
constexpr uint32_t kSmemBytes = 16 + kRingsBytes + kTableAlign + kTablesBytes + kScratchSize + kSlackBytes;
static_assert(kSmemBytes <= 227 * 1024, "exceeds the per-block shared memory of sm_100");
// Words one round can take: one refill per pair and lane, plus one escape word per coordinate.
constexpr uint32_t kRoundWords = 4 * 32 + 8 * 32;
// Fast rounds run without checking the stream position; they are capped so that a corrupt stream stays in
// the shared allocation: at most kMaxFastRounds * 2 * kRoundWords bytes past a ring's end.
constexpr uint32_t kMaxFastRounds = 24;
constexpr uint32_t kOverrunBytes = kMaxFastRounds * 2 * kRoundWords + 64;

// Words of a stream that sits wholly in the warp's ring, at ring coordinate pb (callers keep a round's reads
// inside the ring).
struct RingWords {
    uint32_t base;
    __device__ __forceinline__ uint32_t at(uint32_t pb) const { return ld_shared_u16(base + pb); }
};

// The fused entry of symbol `sym` of context c without its slot - cum field.
__device__ __forceinline__ uint32_t entry_template_v2(int c, int sym, uint32_t f) {
    const int b = c == 0 ? (sym >> 6) : (c <= 4 ? (c - 1) >> 1 : (c - 5) >> 1);
    const int idx = sym & 63, hi = idx - 31;
    const bool esc = idx == kEscIdx;
    uint32_t e = (f & 0xFFu) << 16;
    if (esc) e |= kEscBit;
    if (c <= 4) {  // START and positions 1..6: v = hi + b/2; the class picks the next context
        e |= uint32_t(2 * idx + b);
        if (esc || mag_class(hi, b)) e |= kClassBit;  // an escape always has |hi| >= 3
        if (c == 0 && b) e |= kCosetBit;
    } else {       // position 7 codes h: 2h + b/2 (the parity is added later)
        e |= uint32_t(4 * idx + b);
    }
    return e;
}

// Builds the 9 x 256 fused entries of the blob's tables in shared memory. Pass 1: one warp per context
// reads its 8-bit frequencies (4 symbols a lane) and prefix-sums them into cum, checking that a used
// context sums to 256. Pass 2: each thread fills slots, finding the symbol that owns each by binary search.
// Byte `threadIdx.x` of the serialised tables (zero past their end): loaded first thing in the kernel, so
// that it does not queue behind the tiles' copies.
template <class P>
__device__ __forceinline__ uint32_t table_byte(const P& p) {
    const uint32_t tlen = p.tables_len < kScratchTableCap ? p.tables_len : kScratchTableCap;
    return threadIdx.x < tlen ? uint32_t(__ldg(p.blob + p.off_tables + threadIdx.x)) : 0u;
}

template <class P>
__device__ void build_tables_v2(const P& p, uint8_t* tables, uint8_t* scratch, uint32_t tbyte, bool report) {
    uint16_t* F = reinterpret_cast<uint16_t*>(scratch + kScratchF);
    uint16_t* cum = reinterpret_cast<uint16_t*>(scratch + kScratchCum);
    uint8_t* tb = scratch + kScratchBytesOff;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    static_assert(kScratchTableCap == kThreadsV2, "one table byte per thread");
    tb[tid] = uint8_t(tbyte);
    __syncthreads();
    if (warp < kNumCtx) {
        const int c = warp, A = c == 0 ? 128 : 64;
        const uint32_t lo = tb[c], cnt = tb[kNumCtx + c];
        uint32_t off = 2 * kNumCtx;
        for (int k = 0; k < c; ++k) off += tb[kNumCtx + k];
        uint32_t f[4], part = 0;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const uint32_t s = 4 * lane + j;
            f[j] = (s < uint32_t(A) && s >= lo && s < lo + cnt && off + s - lo < kScratchTableCap) ? tb[off + s - lo] : 0u;
            part += f[j];
        }
        uint32_t incl = part;
#pragma unroll
        for (int d = 1; d < 32; d <<= 1) {
            const uint32_t v = __shfl_up_sync(kFullMask, incl, d);
            if (lane >= d) incl += v;
        }
        uint32_t acc = incl - part;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const uint32_t s = 4 * lane + j;
            if (s < 128) {
                F[c * 128 + s] = uint16_t(f[j]);
                cum[c * 129 + s] = uint16_t(acc);
            }
            acc += f[j];
        }
        const uint32_t total = __shfl_sync(kFullMask, incl, 31);
        if (lane == 0) {
            cum[c * 129 + 128] = uint16_t(total);
            const bool ok = cnt == 0 ? total == 0 : (total == kProbScaleV2 && cnt >= 2);
            if (!ok && report) atomicOr(&g_status, int(EP_DEV_BAD_TABLES));
        }
    }
    __syncthreads();
    uint32_t* t32 = reinterpret_cast<uint32_t*>(tables);
    for (uint32_t k = tid; k < kNumCtx * 256; k += kThreadsV2) {
        const int c = int(k >> 8), A = c == 0 ? 128 : 64;
        const uint32_t t = k & 255;
        const uint16_t* cc = cum + c * 129;
        int s = 0;
#pragma unroll
        for (int step = 64; step >= 1; step >>= 1)  // largest s < A with cum[s] <= t
            if (s + step < A && cc[s + step] <= t) s += step;
        const uint32_t f = F[c * 128 + s];
        // A slot past the table's end (a corrupt table) gets f = 0: the tile check flags it.
        const uint32_t e = (t >= cc[s] && t < cc[s] + f) ? entry_template_v2(c, s, f) | ((t - cc[s]) << 24) : 0u;
        t32[block_of(c) / 4 + t] = e;
    }
    __syncthreads();
}

// One symbol step: the fused entry of the context block B at slot x & 255, then x <- f (x >> 8) + slot - cum.
template <class K>
__device__ __forceinline__ uint32_t symbol(const K& k, uint32_t B, uint32_t& x) {
    const uint32_t q = x >> 8;
    const uint32_t e = ld_shared_u32((x + q * k.kneg256) * k.k4 + B);  // B + 4 (x mod 256)
    x = __byte_perm(e, 0u, 0x4442u) * q + (e >> 24);
    return e;
}

// The pair's refill from the warp's ring: lanes with x < 2^16 take the next words in lane order. pa is
// the shared address of the next word; k2 = 2 (a multiplier kept in a register so the address arithmetic
// runs as multiply-adds). Every lane loads (the address stays in the ring), and only the lanes that need
// the word merge it, by a predicated byte permute: no branch.
__device__ __forceinline__ void refill(uint32_t& x, uint32_t& pa, uint32_t lt_mask, uint32_t k2) {
    asm volatile(
        "{\n"
        " .reg .pred p;\n"
        " .reg .b32 m, t, c, a, w;\n"
        " setp.lt.u32 p, %0, 65536;\n"
        " vote.sync.ballot.b32 m, p, 0xffffffff;\n"
        " and.b32 t, m, %2;\n"
        " popc.b32 c, t;\n"
        " mad.lo.u32 a, c, %3, %1;\n"
        " ld.shared.u16 w, [a];\n"
        " @p prmt.b32 %0, %0, w, 0x1054;\n"
        " popc.b32 c, m;\n"
        " mad.lo.u32 %1, c, %3, %1;\n"
        "}"
        : "+r"(x), "+r"(pa)
        : "r"(lt_mask), "r"(k2));
}

// Values of one group from the value bits mb[i]: 1.5 * 2^22 + F/2 with F = 2 idx + b at positions 0..6 and
// 4 idx + b at position 7 (before pi is added), built by ORing the entries' value fields into the mantissa
// (see round_fast of version 1). two_pi = 2 pi comes from the XOR of the idx parities.
template <int MODE, bool WAIT, class P>
__device__ __forceinline__ void store_fast(const P& p, const uint32_t* mb, uint32_t two_pi, uint32_t g, float c,
                                           float K = kHalfMagicF + 31.0f, float K7 = kHalfMagicF + 62.0f) {
    float m[8], y[8];
    int32_t z[8];
#pragma unroll
    for (int i = 0; i < 7; ++i) m[i] = __uint_as_float(mb[i]);
    m[7] = __uint_as_float(mb[7] + two_pi);
#pragma unroll
    for (int i = 0; i < 6; i += 2) sub_mul_f32x2(m[i], m[i + 1], K, K, c, y[i], y[i + 1]);
    sub_mul_f32x2(m[6], m[7], K, K7, c, y[6], y[7]);
    if constexpr (MODE == kCoords) {
#pragma unroll
        for (int i = 0; i < 8; ++i) z[i] = __float2int_rn((m[i] - (i < 7 ? K : K7)) * 2.0f);
    }
    if constexpr (WAIT) grid_dependency_wait();
    store_group<MODE>(p.dst, g, y, z);
}

// Values of one group in general: hi from the entries or the escape words, lo from the raw section, then
// t = hi 2^r + lo, u_7 = 2 t_7 + pi, z = 2u + b and y = RN(z/2 * c).
template <int MODE, class P>
__device__ __forceinline__ void store_general(const P& p, const uint32_t* e, const int32_t* hesc, uint32_t escm,
                                              const uint32_t* win, uint32_t g, float c) {
    const int r = p.r;
    int32_t t[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        const uint32_t idx = i < 7 ? (e[i] >> 1) & 63u : (e[i] >> 2) & 63u;
        const int32_t hi = (escm >> i) & 1u ? hesc[i] : int32_t(idx) - 31;
        int32_t lo = 0;
        if (r > 0) {
            const uint32_t bp = uint32_t(i) * uint32_t(r), sel = bp >> 5, sh = bp & 31;
            const uint32_t wa = sel == 0 ? win[0] : (sel == 1 ? win[1] : win[2]);
            const uint32_t wb = sel == 0 ? win[1] : win[2];
            lo = int32_t(__funnelshift_r(wa, wb, sh) & ((1u << r) - 1u));
        }
        t[i] = hi * (1 << r) + lo;
    }
    const int32_t b = int32_t(e[0] & 1u);
    int32_t s7 = 0;
#pragma unroll
    for (int i = 0; i < 7; ++i) s7 += t[i];
    float y[8];
    int32_t z[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        const int32_t u = i < 7 ? t[i] : 2 * t[7] + (s7 & 1);
        z[i] = 2 * u + b;
        y[i] = __fmul_rn(__int2float_rn(z[i]) * 0.5f, c);
    }
    store_group<MODE>(p.dst, g, y, z);
}

// The 96-bit window of raw bits of group q (8r bits at byte q r of the tile's raw section).
__device__ __forceinline__ void raw_window(const uint8_t* rawsec, uint32_t raw_avail, uint32_t q, int r, uint32_t* win) {
    win[0] = win[1] = win[2] = 0;
    if (r <= 0) return;
    const uint32_t o = q * uint32_t(r), a = o & ~3u, sh = (o & 3u) * 8;
    uint32_t w[4];
#pragma unroll
    for (int j = 0; j < 4; ++j)
        w[j] = (a + 4 * j + 4 <= raw_avail) ? __ldg(reinterpret_cast<const uint32_t*>(rawsec + a) + j) : 0u;
    win[0] = __funnelshift_r(w[0], w[1], sh);
    win[1] = __funnelshift_r(w[1], w[2], sh);
    win[2] = __funnelshift_r(w[2], w[3], sh);
}

// Three-input logic in one instruction: (a & b) | c, a ^ b ^ c and a | b | c.
__device__ __forceinline__ uint32_t and_or(uint32_t a, uint32_t b, uint32_t c) {
    uint32_t d;
    asm("lop3.b32 %0, %1, %2, %3, 0xEA;" : "=r"(d) : "r"(a), "r"(b), "r"(c));
    return d;
}
__device__ __forceinline__ uint32_t xor3(uint32_t a, uint32_t b, uint32_t c) {
    uint32_t d;
    asm("lop3.b32 %0, %1, %2, %3, 0x96;" : "=r"(d) : "r"(a), "r"(b), "r"(c));
    return d;
}
__device__ __forceinline__ uint32_t or3(uint32_t a, uint32_t b, uint32_t c) {
    uint32_t d;
    asm("lop3.b32 %0, %1, %2, %3, 0xFE;" : "=r"(d) : "r"(a), "r"(b), "r"(c));
    return d;
}

// Fast round: every lane holds a group, r = 0, and the whole stream sits in the warp's ring (pa is the
// shared address of the next word). Each entry is turned into its value bits at once; the XOR of the entries
// of positions 0..6 carries the idx parities (bit 1) and their OR the escape flag. ESC: the tile holds an
// escape (its offset entry says so). Then, when some lane of the warp met one in this round, its words are
// read after the fourth pair, and each escaped position's value bits and parity are rebuilt from the word's
// hi (an escape's field, 2 * 63 + b or 4 * 63 + b, marks it).
template <int MODE, bool WAIT, bool ESC, class P, class K, bool RAW = false>
__device__ __forceinline__ void round_fast_v2(const P& p, const K& kc, uint32_t t0, uint32_t ts, uint32_t& x, uint32_t& pa, uint32_t g,
                                              uint32_t lt_mask, float c, uint32_t k2, uint32_t rawb = 0, uint32_t q = 0) {
    uint32_t mb[8], e, e2, par, escs;
    e = symbol(kc, ts, x);
    mb[0] = and_or(e, 0x7Fu, kHalfMagic);
    const uint32_t gbase = and_or(e, kCosetBit, t0);
    e2 = symbol(kc, and_or(e, kClassBit, gbase), x);
    mb[1] = and_or(e2, 0x7Fu, kHalfMagic);
    par = e ^ e2;
    escs = e | e2;
    refill(x, pa, lt_mask, k2);
#pragma unroll
    for (int i = 2; i < 6; i += 2) {
        e = symbol(kc, and_or(e2, kClassBit, gbase), x);
        mb[i] = and_or(e, 0x7Fu, kHalfMagic);
        e2 = symbol(kc, and_or(e, kClassBit, gbase), x);
        mb[i + 1] = and_or(e2, 0x7Fu, kHalfMagic);
        par = xor3(par, e, e2);
        escs = or3(escs, e, e2);
        refill(x, pa, lt_mask, k2);
    }
    e = symbol(kc, and_or(e2, kClassBit, gbase), x);
    mb[6] = and_or(e, 0x7Fu, kHalfMagic);
    e2 = symbol(kc, and_or(e, kClassBit, gbase | kPos7Bit), x);
    mb[7] = and_or(e2, 0xFFu, kHalfMagic);
    par ^= e;
    escs = or3(escs, e, e2);
    refill(x, pa, lt_mask, k2);
    if constexpr (RAW && ESC) {
        // A round in which some lane met an escape: its words follow the fourth pair, position by position and
        // lane by lane, as in the general round. Each position's t = hi 2^r + lo (hi from the entry, or any
        // int16 from the escape word; lo from the group's raw bits in shared memory) replaces its value bits,
        // and the values come from the integer formula.
        if (__any_sync(kFullMask, escs & kEscBit)) {
            const uint32_t r = uint32_t(p.r), o = q * r, a = o & ~3u, sh = (o & 3u) * 8, lmask = (1u << r) - 1u;
            uint32_t w[4];
#pragma unroll
            for (int j = 0; j < 4; ++j) w[j] = ld_shared_u32(rawb + a + 4 * j);
            uint32_t A = __funnelshift_r(w[0], w[1], sh), B = __funnelshift_r(w[1], w[2], sh), C = __funnelshift_r(w[2], w[3], sh);
            const int32_t b = int32_t(mb[0] & 1u);
            int32_t s7 = 0;
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                const bool esc = i < 7 ? (mb[i] & 0x7Eu) == 0x7Eu : (mb[7] & 0xFCu) == 0xFCu;
                const uint32_t me = __ballot_sync(kFullMask, esc);
                int32_t hi = int32_t(i < 7 ? (mb[i] >> 1) & 63u : (mb[7] >> 2) & 63u) - 31;
                if (me) {
                    const uint32_t wd = ld_shared_u16(pa + __popc(me & lt_mask) * k2);
                    pa += __popc(me) * k2;
                    if (esc) hi = int32_t(int16_t(wd));
                }
                const int32_t t = hi * (1 << r) + int32_t(A & lmask);
                if (i < 7) {
                    A = __funnelshift_r(A, B, r);
                    B = __funnelshift_r(B, C, r);
                    C >>= r;
                }
                if (i < 7) s7 += t;
                mb[i] = uint32_t(t);
            }
            float y[8];
            int32_t z[8];
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                const int32_t u = i < 7 ? int32_t(mb[i]) : 2 * int32_t(mb[7]) + (s7 & 1);
                z[i] = 2 * u + b;
                y[i] = __fmul_rn(__int2float_rn(z[i]) * 0.5f, c);
            }
            if constexpr (WAIT) grid_dependency_wait();
            store_group<MODE>(p.dst, g, y, z);
            return;
        }
    }
    if (!RAW && ESC && __any_sync(kFullMask, escs & kEscBit)) {
        const uint32_t b = mb[0] & 1u;
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const bool esc = i < 7 ? (mb[i] & 0x7Eu) == 0x7Eu : (mb[7] & 0xFCu) == 0xFCu;
            const uint32_t me = __ballot_sync(kFullMask, esc);
            if (me) {
                const uint32_t w = ld_shared_u16(pa + __popc(me & lt_mask) * k2);
                pa += __popc(me) * k2;
                if (esc) {
                    const int32_t idx = int32_t(int16_t(w)) + 31;  // hi + 31, any int16 hi
                    if (i < 7) {
                        mb[i] = kHalfMagic + uint32_t(2 * idx) + b;
                        par ^= (uint32_t(idx) & 1u) << 1 ^ 2u;      // replace idx 63's parity by idx's
                    } else {
                        mb[7] = kHalfMagic + uint32_t(4 * idx) + b;
                    }
                }
            }
        }
    }
    if constexpr (RAW) {
        // r >= 1 raw low bits a coordinate, in a round where no lane met an escape (so |hi| <= 31 and every field
        // below stays under 2^22): t = hi 2^r + lo, so m_i = 1.5*2^22 + 2 idx 2^r + 2 lo + b (i < 7) and
        // m_7 = 1.5*2^22 + 4 idx 2^r + 4 lo_7 + 2 pi + b, pi the parity of the seven lo's; the group's 8r
        // bits sit at bit 8 r q of the tile's raw section, in shared memory (rawb).
        const uint32_t r = uint32_t(p.r), o = q * r, a = o & ~3u, sh = (o & 3u) * 8, lmask = (1u << r) - 1u;
        const uint32_t pow2r = 1u << r;
        uint32_t w[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) w[j] = ld_shared_u32(rawb + a + 4 * j);
        // The group's 8r bits from bit 0 of (A, B, C): each position takes the low r bits of A, then the three
        // words shift right by r together.
        uint32_t A = __funnelshift_r(w[0], w[1], sh), B = __funnelshift_r(w[1], w[2], sh), C = __funnelshift_r(w[2], w[3], sh);
        uint32_t lpar = 0;
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const uint32_t lo = A & lmask;
            if (i < 7) {
                A = __funnelshift_r(A, B, r);
                B = __funnelshift_r(B, C, r);
                C >>= r;
            }
            // mb & ~0xFE is 1.5*2^22 + b: the entry's value field sits in the low 8 bits.
            if (i < 7) {
                lpar ^= lo;
                mb[i] = (mb[i] & ~0xFEu) + (mb[i] & 0x7Eu) * pow2r + (lo << 1);
            } else {
                mb[7] = (mb[7] & ~0xFEu) + (mb[7] & 0xFCu) * pow2r + (lo << 2) + ((lpar & 1u) << 1);
            }
        }
        const float sc = float(1u << r);
        store_fast<MODE, WAIT>(p, mb, 0u, g, c, kHalfMagicF + 31.0f * sc, kHalfMagicF + 62.0f * sc);
    } else {
        store_fast<MODE, WAIT>(p, mb, ~par & 2u, g, c);
    }
}

// General round: ragged rounds (PARTIAL: some lanes hold no group), raw low bits, and streams read from
// global memory with bounds checks (Words = GlobalWords) or from the ring (RingWords).
template <int MODE, bool PARTIAL, class Words, class P>
__device__ __forceinline__ void round_general_v2(const P& p, uint32_t t0, uint32_t ts, const Words& words, const uint8_t* rawsec,
                                              uint32_t raw_avail, TileState& st, uint32_t q, bool active, uint32_t g,
                                              uint32_t lt_mask, float c) {
    const bool on = !PARTIAL || active;
    uint32_t win[3];
    raw_window(rawsec, raw_avail, q, on ? p.r : 0, win);
    uint32_t x = st.x, pb = st.pb;
    uint32_t e[8];
    uint32_t gbase = t0, B = ts;
#pragma unroll
    for (int pr = 0; pr < 4; ++pr) {
#pragma unroll
        for (int i = 2 * pr; i <= 2 * pr + 1; ++i) {
            e[i] = 0;
            if (on) {
                const uint32_t qq = x >> 8;
                e[i] = ld_shared_u32(B + ((x & 255u) << 2));
                x = ((e[i] >> 16) & 0xFFu) * qq + (e[i] >> 24);
            }
            if (i == 0) gbase = t0 | (e[0] & kCosetBit);
            B = (i == 6 ? (gbase | kPos7Bit) : gbase) | (e[i] & kClassBit);
        }
        const bool need = on && x < kRansL;
        const uint32_t m = __ballot_sync(kFullMask, need);
        const uint32_t w = words.at(pb + 2 * __popc(m & lt_mask));
        x = __byte_perm(x, w, need ? 0x1054u : 0x3210u);
        pb += 2 * __popc(m);
    }
    int32_t hesc[8];
    uint32_t escm = 0;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        const bool esc = on && (e[i] & kEscBit);
        const uint32_t me = __ballot_sync(kFullMask, esc);
        hesc[i] = 0;
        if (me) {
            const uint32_t w = words.at(pb + 2 * __popc(me & lt_mask));
            if (esc) hesc[i] = int32_t(int16_t(w));
            pb += 2 * __popc(me);
        }
        escm |= esc ? 1u << i : 0u;
    }
    st.x = x;
    st.pb = pb;
    if (on) store_general<MODE>(p, e, hesc, escm, win, g, c);
}

static_assert(kTablesBytes + kScratchSize + kSlackBytes >= kOverrunBytes, "a corrupt stream could read past the allocation");

// Rounds [0, Rf) of a tile from the ring, Rf <= kMaxFastRounds. A valid stream ends inside the ring; a corrupt
// one may run past it, by at most 768 bytes a round, into the shared memory that follows (kSmemBytes keeps
// kOverrunBytes after the last ring), and the tile check flags it. If `waited` is false, the first round waits
// for the previous launch of a sequence before its stores, and sets it. Returns the number of rounds done.
//
// UNIFORM: rows hold whole rounds (gpr % 32 == 0), so every lane of a round is in the same row and the row
// changes for all lanes at once, every gpr / 32 rounds. The tile spans at most kMaxFastRounds rows from row0:
// lane i computes the factor of row row0 + i once, and each round takes its row's factor by a shuffle, with
// no load on the round's path. kr: the first round's column in its row, in rounds. Otherwise the lanes'
// rows move on their own (RowCursor).
template <int MODE, bool ESC, bool UNIFORM, class P, class K, bool RAW = false>
__device__ __forceinline__ uint32_t fast_rounds_v2(const P& p, const K& kc, uint32_t t0, uint32_t ts, TileState& st, uint32_t ring_base,
                                                   uint32_t g, uint32_t lt_mask, uint32_t Rf, uint32_t row0, uint32_t kr,
                                                   const uint16_t* scales, RowCursor& rc, bool& waited, uint32_t rawb = 0) {
    uint32_t k = 0, x = st.x, pa = ring_base + st.pb;
    const uint32_t g0 = g - (threadIdx.x & 31);  // the tile's first group: q = g - g0
    if constexpr (UNIFORM) {
        const uint32_t rpr = p.gpr / 32, lane = threadIdx.x & 31;
        const float cvec = row0 + lane < p.M ? RowCursor::scale_of(p, scales, row0 + lane) : 0.f;
        uint32_t ri = 0;
        if (!waited && Rf > 0) {
            round_fast_v2<MODE, true, ESC, P, K, RAW>(p, kc, t0, ts, x, pa, g, lt_mask, __shfl_sync(kFullMask, cvec, 0), kc.k2, rawb, g - g0);
            waited = true;
            k = 1;
            g += 32;
            if (++kr == rpr) {
                kr = 0;
                ++ri;
            }
        }
        // Row by row: the factor is taken once per row, and the inner loop only counts rounds.
        while (k < Rf) {
            const uint32_t run = min(rpr - kr, Rf - k);
            const float c = __shfl_sync(kFullMask, cvec, ri);
            const uint32_t gend = g + 32 * run;
            for (; g != gend; g += 32) round_fast_v2<MODE, false, ESC, P, K, RAW>(p, kc, t0, ts, x, pa, g, lt_mask, c, kc.k2, rawb, g - g0);
            k += run;
            kr = 0;
            ++ri;
        }
    } else {
        if (!waited && Rf > 0) {
            round_fast_v2<MODE, true, ESC, P, K, RAW>(p, kc, t0, ts, x, pa, g, lt_mask, rc.scale(), kc.k2, rawb, g - g0);
            rc.advance(p, scales);
            waited = true;
            k = 1;
            g += 32;
        }
        for (; k < Rf; ++k, g += 32) {
            round_fast_v2<MODE, false, ESC, P, K, RAW>(p, kc, t0, ts, x, pa, g, lt_mask, rc.scale(), kc.k2, rawb, g - g0);
            rc.advance(p, scales);
        }
    }
    st.x = x;
    st.pb = pa - ring_base;
    return k;
}

// Offset entries of a tile (start / 16 with the escape flag, end / 16), or zeros past the last tile.
struct TileOffs {
    uint32_t e0, e1;
};
template <class P>
__device__ __forceinline__ TileOffs load_offs(const P& p, const uint32_t* toff, uint32_t tile) {
    TileOffs o{0u, 0u};
    if (tile < p.T) {
        o.e0 = __ldg(toff + tile);
        o.e1 = __ldg(toff + tile + 1);
    }
    return o;
}
// Byte size of a tile whose offsets are sane (start <= end <= payload, at least its 128 bytes of states), else 0.
template <class P>
__device__ __forceinline__ uint32_t tile_size(const P& p, const TileOffs& o) {
    const uint64_t start = uint64_t(o.e0 & 0x7FFFFFFFu) * 16, end = uint64_t(o.e1 & 0x7FFFFFFFu) * 16;
    return (end >= start + 128 && end <= p.payload_bytes && end - start <= 0x7FFFFFF0ull) ? uint32_t(end - start) : 0u;
}
// Copies a whole tile (sz bytes, a multiple of 16) from global memory to shared address dst: 16 bytes a lane.
__device__ __forceinline__ void copy_tile(uint32_t dst, const uint8_t* src, uint32_t sz, uint32_t lane) {
    for (uint32_t o = 16 * lane; o < sz; o += 512) cp_async16(dst + o, src + o, 16);
}

template <int MODE>
__global__ void __launch_bounds__(kThreadsV2, 1) decode_kernel(const Params p) {
    extern __shared__ __align__(16) uint8_t smem_raw[];
    const uint32_t tbyte = table_byte(p);
    const uint32_t raw_base = smem_addr(smem_raw);
    uint8_t* rings = smem_raw;
    const uint32_t after_rings = raw_base + kRingsBytes;
    const uint32_t tbl_pad = (kTableAlign - (after_rings & (kTableAlign - 1))) & (kTableAlign - 1);
    uint8_t* tables = rings + kRingsBytes + tbl_pad;
    uint8_t* scratch = tables + kTablesBytes;
    const uint32_t t0 = smem_addr(tables);

    const uint32_t lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const uint32_t lt_mask = (1u << lane) - 1u;
    const uint16_t* scales = reinterpret_cast<const uint16_t*>(p.blob + p.off_scales);
    const uint32_t* toff = reinterpret_cast<const uint32_t*>(p.blob + p.off_offsets);
    const uint8_t* payload = p.blob + p.off_payload;
    const uint32_t per_tile = 32 * p.G;
    const uint32_t ring_base = smem_addr(rings + warp * kRingBytes);
    const uint32_t stride = kWarpsV2 * gridDim.x;  // tiles are dealt round-robin over the CTAs first

    grid_dependents_launch();

    if (p.next_blob) {
        const uint32_t lines = (p.next_meta_bytes + 127) / 128;
        for (uint32_t l = blockIdx.x + gridDim.x * threadIdx.x; l < lines; l += gridDim.x * kThreadsV2)
            prefetch_l2(p.next_blob + p.next_meta_off + 128ull * l);
    }

    // The first tile's copy is issued before the table build, which hides it. `pending`: whether a copy group
    // is committed and not yet waited for.
    uint32_t tile = warp * gridDim.x + blockIdx.x;
    TileOffs cur = load_offs(p, toff, tile), nxt = load_offs(p, toff, tile + stride);
    uint32_t place = 0;  // where the current tile sits in the warp's buffer
    uint32_t pending = 0;
    {
        const uint32_t sz = tile_size(p, cur);
        if (tile < p.T && sz && sz <= kRingBytes) {
            copy_tile(ring_base, payload + uint64_t(cur.e0 & 0x7FFFFFFFu) * 16, sz, lane);
            cp_async_commit();
            pending = 1;
        }
    }
    build_tables_v2(p, tables, scratch, tbyte, blockIdx.x == 0);
    bool waited = false;

    // Every decision below is taken for the whole warp (a vote, or values of the tile index and the kernel
    // parameters only), so that the compiler sees warp-uniform control flow in the round loops.
    for (; tile < p.T; tile += stride) {
        const uint32_t ng = min(per_tile, p.NG - tile * per_tile);
        const uint32_t raw = (ng * uint32_t(p.r) + 3u) & ~3u, s0 = 128 + raw;
        const uint32_t sz = __shfl_sync(kFullMask, tile_size(p, cur), 0);
        const bool ok = sz >= s0;
        const bool in_ring = ok && sz <= kRingBytes;
        // The next tile's copy goes to the other end of the buffer now, if both fit.
        const uint32_t ntile = tile + stride;
        const uint32_t nsz = __shfl_sync(kFullMask, tile_size(p, nxt), 0);
        const bool early = ntile < p.T && nsz && (in_ring ? sz + nsz <= kRingBytes : nsz <= kRingBytes);
        const uint32_t nplace = early && in_ring && place == 0 ? kRingBytes - nsz : 0u;
        const TileOffs after = load_offs(p, toff, ntile + stride);
        // Wait for this tile's copy (if any), then start the next tile's: it lands while this one decodes.
        cp_async_wait<0>();
        __syncwarp();
        pending = 0;
        if (early) {
            copy_tile(ring_base + nplace, payload + uint64_t(nxt.e0 & 0x7FFFFFFFu) * 16, nsz, lane);
            cp_async_commit();
            pending = 1;
        }
        if (!ok) {
            if (lane == 0) atomicOr(&g_status, int(EP_DEV_BAD_OFFSETS));
        } else {
            const uint32_t rb = ring_base + place;
            const uint8_t* tp = payload + uint64_t(cur.e0 & 0x7FFFFFFFu) * 16;
            TileState st;
            st.x = in_ring ? ld_shared_u32(rb + 4 * lane) : __ldg(reinterpret_cast<const uint32_t*>(tp) + lane);
            st.pb = s0;
            const GlobalWords gwords{tp, s0, sz};
            if (!early && ntile < p.T) {  // the next tile's copy comes after this one: pull it toward L2
                const uint64_t ns = uint64_t(nxt.e0 & 0x7FFFFFFFu) * 16 + 128ull * lane;
                if (ns < p.payload_bytes) prefetch_l2(payload + ns);
            }
            RowCursor rc;
            const uint8_t* rawsec = tp + 128;
            const uint32_t raw_avail = sz - 128;
            const uint32_t R = (ng + 31) / 32;
            const uint32_t gt0 = tile * per_tile;

            uint32_t k = 0;
            const bool esc = __any_sync(kFullMask, cur.e0 >> 31);
            if (in_ring) {
                const uint32_t Rf = min(ng / 32, kMaxFastRounds);
                const uint32_t row0 = gt0 / p.gpr, kr0 = (gt0 - row0 * p.gpr) / 32;
                if (p.r != 0) {  // raw low bits
                    if (p.gpr % 32 == 0) {
                        k = esc ? fast_rounds_v2<MODE, true, true, Params, Params, true>(p, p, t0, t0 | kStartOffset, st, rb, gt0 + lane, lt_mask, Rf, row0, kr0, scales, rc, waited, rb + 128)
                                : fast_rounds_v2<MODE, false, true, Params, Params, true>(p, p, t0, t0 | kStartOffset, st, rb, gt0 + lane, lt_mask, Rf, row0, kr0, scales, rc, waited, rb + 128);
                    } else {
                        rc.start(p, scales, gt0 + lane);
                        k = esc ? fast_rounds_v2<MODE, true, false, Params, Params, true>(p, p, t0, t0 | kStartOffset, st, rb, gt0 + lane, lt_mask, Rf, row0, kr0, scales, rc, waited, rb + 128)
                                : fast_rounds_v2<MODE, false, false, Params, Params, true>(p, p, t0, t0 | kStartOffset, st, rb, gt0 + lane, lt_mask, Rf, row0, kr0, scales, rc, waited, rb + 128);
                    }
                } else if (p.gpr % 32 == 0) {
                    k = esc ? fast_rounds_v2<MODE, true, true>(p, p, t0, t0 | kStartOffset, st, rb, gt0 + lane, lt_mask, Rf, row0, kr0, scales, rc, waited)
                            : fast_rounds_v2<MODE, false, true>(p, p, t0, t0 | kStartOffset, st, rb, gt0 + lane, lt_mask, Rf, row0, kr0, scales, rc, waited);
                } else {
                    rc.start(p, scales, gt0 + lane);
                    k = esc ? fast_rounds_v2<MODE, true, false>(p, p, t0, t0 | kStartOffset, st, rb, gt0 + lane, lt_mask, Rf, row0, kr0, scales, rc, waited)
                            : fast_rounds_v2<MODE, false, false>(p, p, t0, t0 | kStartOffset, st, rb, gt0 + lane, lt_mask, Rf, row0, kr0, scales, rc, waited);
                }
            }
            if (k < R) {
                rc.start(p, scales, gt0 + 32 * k + lane);
                if (!waited) {
                    grid_dependency_wait();
                    waited = true;
                }
                const RingWords ring{rb};
                for (; k < R; ++k) {
                    const uint32_t q = 32 * k + lane, g = gt0 + q;
                    const bool full = 32 * k + 32 <= ng;
                    // Ring reads of a round stay within the tile's own bytes (a round takes at most 768).
                    if (in_ring && full && __all_sync(kFullMask, st.pb + 2 * kRoundWords <= sz)) {
                        round_general_v2<MODE, false>(p, t0, t0 | kStartOffset, ring, rawsec, raw_avail, st, q, true, g, lt_mask, rc.scale());
                    } else {
                        round_general_v2<MODE, true>(p, t0, t0 | kStartOffset, gwords, rawsec, raw_avail, st, q, q < ng, g, lt_mask,
                                                      rc.scale());
                    }
                    rc.advance(p, scales);
                }
            }
            __syncwarp();
            const uint32_t used = st.pb - s0, cap = sz - s0;  // bytes of stream read / present
            const bool good = __all_sync(kFullMask, st.x == kRansL) && used <= cap && cap - used <= 14;
            if (!good && lane == 0) atomicOr(&g_status, int(EP_DEV_CORRUPT_TILE));
        }
        // The buffer is free now: a next tile that did not fit beside this one is copied to the bottom.
        if (!early && ntile < p.T && nsz && nsz <= kRingBytes) {
            __syncwarp();
            copy_tile(ring_base, payload + uint64_t(nxt.e0 & 0x7FFFFFFFu) * 16, nsz, lane);
            cp_async_commit();
            pending = 1;
        }
        place = early ? nplace : 0u;
        cur = nxt;
        nxt = after;
    }
    if (pending) cp_async_wait<0>();
    if (!waited) grid_dependency_wait();
}


// ------------------------------------------------------------------------- one launch for a sequence
//
// ep_decompress_many of version-2 blobs that share one output type runs as two launches: prep_tables_kernel
// builds every layer's fused entries once into global scratch, and seq_kernel, one CTA per SM for all the
// layers, decodes them. The tiles of all the layers are dealt round-robin as one list: the sequence's k-th
// tile goes to CTA k mod grid, and a CTA's own tiles go to its warps in turn, so a layer with few tiles shares
// the SMs with the next one, and no launch boundary, table build or wait for a whole previous layer sits
// between layers. Each CTA holds the tables of kWindows consecutive layers in shared windows: the window of
// layer L is refilled with layer L + kWindows by bulk copies once all of the CTA's warps are done with L. A tile
// writes only after the tiles of earlier layers that wrote the same bytes are done (per-layer tile-done
// bitmasks in global memory, bounded waits), so the buffer ends as a sequence of separate launches leaves it.

constexpr uint32_t kMaxSeqLayers = 280;
constexpr uint16_t kNoDep = 0xFFFFu;

struct LayerDesc {
    const uint8_t* blob;
    void* dst;
    uint64_t payload_bytes;
    uint32_t gpr, T, G, NG, M;
    int r;
    float alpha, inv_alpha;
    uint32_t off_scales, off_offsets, off_payload, off_tables, tables_len;
    uint32_t tile0;        // the layer's first tile in the sequence's deal order
    uint32_t bits;         // word offset of the layer's tile-done bitmask in the order scratch
    uint32_t need_prefix;  // layers [0, need_prefix) are complete before any store of this layer
    // Groups [seg_lo[d], seg_hi[d]) of this layer were last written, before it, by layer seg_layer[d]
    // (kNoDep: no such segment). Older writers, if any, are covered by need_prefix.
    uint32_t seg_lo[2], seg_hi[2];
    uint16_t seg_layer[2];
};

struct SeqParams {
    uint32_t count;
    uint32_t k2, k4, kneg256;  // multipliers kept out of the compiler's sight (see Params)
    uint32_t ordered;          // some layer overwrites an earlier one's output: tiles wait and publish
    uint32_t use_prefix;       // some layer has need_prefix > 0: tiles are counted per layer
    uint32_t counts_off;       // word offset of the per-layer done counters in the order scratch
    uint32_t prefix_off;       // word offset of the number of leading complete layers
    const uint32_t* tables;    // prepared fused entries, kTablesBytes per layer, in shared-window layout
    uint32_t* order;           // tile-done bitmasks, done counters, prefix (zeroed before the launch)
    LayerDesc L[kMaxSeqLayers];
};
static_assert(sizeof(SeqParams) <= 32764, "kernel parameters are limited to 32764 bytes");

// One CTA per layer: builds the layer's fused entries into global memory.
__global__ void __launch_bounds__(kThreadsV2, 1) prep_tables_kernel(const __grid_constant__ SeqParams sp) {
    extern __shared__ __align__(16) uint8_t smem_raw[];
    const LayerDesc& p = sp.L[blockIdx.x];
    const uint32_t tbyte = table_byte(p);
    uint32_t* out = const_cast<uint32_t*>(sp.tables) + size_t(blockIdx.x) * (kTablesBytes / 4);
    build_tables_v2(p, reinterpret_cast<uint8_t*>(out), smem_raw, tbyte, true);
}

// Table windows: a CTA holds the tables of kWindows consecutive layers. A window is the 8 KB of context
// blocks, on an 8 KB boundary so that the (b, class, position 7) bits combine by OR, plus a 1 KB START block
// of its own. Layout: rings, then the context blocks of every window, their START blocks, then the window
// barriers and done counters. More than kOverrunBytes follow the last ring.
constexpr uint32_t kWindows = 4;  // a power of two
constexpr uint32_t kCtxRegion = kStartOffset;  // contexts 1..8
constexpr uint32_t kSeqSmemBytes = 16 + kRingsBytes + kCtxRegion + kWindows * kTablesBytes + kWindows * 16 +
                                   kMaxSeqLayers * 4;
static_assert(kSeqSmemBytes <= 227 * 1024, "exceeds the per-block shared memory of sm_100");
static_assert(kWindows * kTablesBytes >= kOverrunBytes, "a corrupt stream could read past the allocation");

// Starts the bulk copies of layer L's entries into window (ctx, start); thread 0 only.
__device__ __noinline__ void load_window(const SeqParams& sp, uint32_t L, uint32_t ctx, uint32_t start,
                                            uint32_t bar) {
    mbar_expect_tx(bar, kTablesBytes);
    const uint32_t* src = sp.tables + size_t(L) * (kTablesBytes / 4);
    for (uint32_t c = 0; c < kCtxRegion / kCtxBytes; ++c)
        bulk_copy_g2s(ctx + c * kCtxBytes, src + c * (kCtxBytes / 4), kCtxBytes, bar);
    bulk_copy_g2s(start, src + kStartOffset / 4, kCtxBytes, bar);
}

// The CTA's tiles of layer L: t0, t0 + grid, ... (the return value counts them).
__device__ __forceinline__ uint32_t cta_tiles(const SeqParams& sp, uint32_t L, uint32_t& t0) {
    const uint32_t T = sp.L[L].T, grid = gridDim.x;
    t0 = (blockIdx.x + grid - sp.L[L].tile0 % grid) % grid;
    return t0 < T ? (T - t0 + grid - 1) / grid : 0u;
}
// This warp's first tile of layer L, or T when it has none there. nb: the CTA's tiles in the layers before L,
// which sets where the warps' turns stand.
__device__ __forceinline__ uint32_t first_tile(const SeqParams& sp, uint32_t L, uint32_t nb, uint32_t warp) {
    uint32_t t0;
    const uint32_t cnt = cta_tiles(sp, L, t0);
    const uint32_t j0 = (warp + 32u - nb % 32u) % 32u;
    return j0 < cnt ? t0 + j0 * gridDim.x : sp.L[L].T;
}

// A position in this warp's walk over the sequence; L == count at the end.
struct Pos {
    uint32_t L, tile;
};
// The warp's next tile after q. nbs[L]: the CTA's tiles in the layers before L (shared memory).
__device__ __forceinline__ Pos next_pos(const SeqParams& sp, const uint32_t* nbs, Pos q, uint32_t warp) {
    q.tile += 32u * gridDim.x;
    while (q.L < sp.count && q.tile >= sp.L[q.L].T) {
        ++q.L;
        if (q.L < sp.count) q.tile = first_tile(sp, q.L, nbs[q.L], warp);
    }
    return q;
}
__device__ __forceinline__ const uint32_t* pos_toff(const SeqParams& sp, const Pos& q) {
    const LayerDesc& p = sp.L[q.L];
    return reinterpret_cast<const uint32_t*>(p.blob + p.off_offsets) + q.tile;
}
__device__ __forceinline__ TileOffs pos_offs(const SeqParams& sp, const Pos& q) {
    if (q.L >= sp.count) return TileOffs{0u, 0u};
    const uint32_t* t = pos_toff(sp, q);
    return TileOffs{__ldg(t), __ldg(t + 1)};
}

constexpr uint32_t kDepSpins = 1u << 20;  // bounded waits: about a quarter second, then a status bit

// Before the first store of a tile of layer p (groups [g0, g0 + ng), es bytes an element): the layers before
// need_prefix complete, and, for each segment the tile meets, the tiles of the segment's writer that cover the
// common bytes done. The flags are read in parallel, one word a lane: lane 0 the prefix, lanes 1-15 segment
// 0's bitmask words, lanes 16-31 segment 1's. A lane's acquire orders the warp's stores after it through the
// closing warp barrier.
__device__ __forceinline__ void seq_wait(const SeqParams& sp, const LayerDesc& p, uint32_t g0, uint32_t ng,
                                         uint32_t es) {
    const uint32_t lane = threadIdx.x & 31;
    const uint32_t d = lane >> 4, first = d ? lane - 16 : lane - 1, step = d ? 16u : 15u;
    const uint32_t* bits = nullptr;
    uint32_t k0 = 1, k1 = 0;  // tiles [k0, k1] of the writer (empty unless set below)
    if (lane != 0 && p.seg_layer[d] != kNoDep) {
        const uint32_t a = max(g0, p.seg_lo[d]), b = min(g0 + ng, p.seg_hi[d]);
        if (a < b) {
            const LayerDesc& q = sp.L[p.seg_layer[d]];
            const uint64_t qlo = reinterpret_cast<uint64_t>(q.dst), qhi = qlo + uint64_t(q.NG) * 8 * es;
            const uint64_t base = reinterpret_cast<uint64_t>(p.dst);
            const uint64_t lo = max(base + uint64_t(a) * 8 * es, qlo), hi = min(base + uint64_t(b) * 8 * es, qhi);
            if (lo < hi) {
                const uint64_t tb = uint64_t(32) * q.G * 8 * es;  // output bytes of one full tile of q
                k0 = uint32_t((lo - qlo) / tb);
                k1 = min(uint32_t((hi - qlo - 1) / tb), q.T - 1);
                bits = sp.order + q.bits;
            }
        }
    }
    for (uint32_t n = 0;; ++n) {
        bool ok = true;
        if (lane == 0 && p.need_prefix) ok = ld_acquire(sp.order + sp.prefix_off) >= p.need_prefix;
        if (bits) {
            for (uint32_t w = k0 / 32 + first; w <= k1 / 32; w += step) {
                const uint32_t lo = w * 32 > k0 ? 0u : k0 % 32, hi = w * 32 + 31 < k1 ? 31u : k1 % 32;
                const uint32_t m = (hi == 31 ? ~0u : (2u << hi) - 1u) & ~((1u << lo) - 1u);
                ok = ok && (ld_acquire(bits + w) & m) == m;
            }
        }
        if (__all_sync(kFullMask, ok)) break;
        if (n >= kDepSpins) {
            if (lane == 0) atomicOr(&g_status, int(EP_DEV_DEP_WAIT));
            break;
        }
        __nanosleep(256);
    }
    __syncwarp();
}

// Moves the prefix of complete layers on from j while layer j is complete (an empty layer always is). The
// prefix only moves by compare-and-swap from j to j + 1, so a caller that finds it elsewhere stops. Two
// callers racing over neighbouring layers cannot both stop short: each makes its update, fences, then reads
// the other's, so at least one sees both and moves on.
__device__ __forceinline__ void advance_prefix(const SeqParams& sp, uint32_t j) {
    for (; j < sp.count; ++j) {
        if (ld_acquire(sp.order + sp.counts_off + j) != sp.L[j].T) break;
        if (atomicCAS(sp.order + sp.prefix_off, j, j + 1) != j) break;
        __threadfence();
    }
}

// After the last store of tile `tile` of layer L: publish it, count it, and when it completes its layer,
// advance the prefix of complete layers (a layer that completes while an earlier one is open leaves the
// advance to that layer's last tile).
__device__ __forceinline__ void seq_done(const SeqParams& sp, uint32_t L, uint32_t tile) {
    __syncwarp();
    if ((threadIdx.x & 31) != 0) return;
    __threadfence();
    atomicOr(sp.order + sp.L[L].bits + tile / 32, 1u << (tile % 32));
    if (!sp.use_prefix) return;
    const uint32_t c = atomicAdd(sp.order + sp.counts_off + L, 1u) + 1u;
    if (c != sp.L[L].T) return;
    __threadfence();
    advance_prefix(sp, L);
}

template <int MODE>
__global__ void __launch_bounds__(kThreadsV2, 1) seq_kernel(const __grid_constant__ SeqParams sp) {
    extern __shared__ __align__(16) uint8_t smem_raw[];
    constexpr uint32_t es = MODE == kFP32 ? 4u : (MODE == kBF16 || MODE == kFP16) ? 2u : 1u;
    const uint32_t raw_base = smem_addr(smem_raw);
    const uint32_t rings0 = (raw_base + 15u) & ~15u;
    const uint32_t win0 = (rings0 + kRingsBytes + kCtxRegion - 1) & ~(kCtxRegion - 1);
    const uint32_t starts = win0 + kWindows * kCtxRegion;
    const uint32_t bars = starts + kWindows * kCtxBytes;  // kWindows mbarriers, then kWindows done counters
    uint32_t* done_cnt = reinterpret_cast<uint32_t*>(smem_raw + (bars + 8u * kWindows - raw_base));
    uint32_t* nbs = done_cnt + kWindows;  // per layer: the CTA's tiles in the layers before it
    const uint32_t lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const uint32_t lt_mask = (1u << lane) - 1u;
    const uint32_t ring_base = rings0 + warp * kRingBytes;
    const uint32_t n = sp.count;

    if (threadIdx.x < kWindows) {
        mbar_init(bars + 8 * threadIdx.x, 1);
        done_cnt[threadIdx.x] = 0;
    }
    if (warp == 0) {  // nbs: an exclusive scan of the CTA's tile counts over the layers
        uint32_t carry = 0;
        for (uint32_t base = 0; base < n; base += 32) {
            uint32_t t0c, c = base + lane < n ? cta_tiles(sp, base + lane, t0c) : 0u, incl = c;
#pragma unroll
            for (int dd = 1; dd < 32; dd <<= 1) {
                const uint32_t v = __shfl_up_sync(kFullMask, incl, dd);
                if (lane >= uint32_t(dd)) incl += v;
            }
            if (base + lane < n) nbs[base + lane] = carry + incl - c;
            carry += __shfl_sync(kFullMask, incl, 31);
        }
    }
    __syncthreads();
    if (threadIdx.x == 0)
        for (uint32_t s = 0; s < kWindows && s < n; ++s)
            load_window(sp, s, win0 + s * kCtxRegion, starts + s * kCtxBytes, bars + 8 * s);
    // Leading empty layers never complete a tile: move the prefix over them.
    if (sp.use_prefix && blockIdx.x == 0 && threadIdx.x == 0) advance_prefix(sp, 0);

    Pos cur{0u, n ? first_tile(sp, 0, 0, warp) : 0u};
    if (n && cur.tile >= sp.L[0].T) cur = next_pos(sp, nbs, cur, warp);
    Pos nxt = next_pos(sp, nbs, cur, warp);
    TileOffs co = pos_offs(sp, cur), no = pos_offs(sp, nxt);
    uint32_t place = 0, pending = 0;
    if (cur.L < n) {
        const LayerDesc& p = sp.L[cur.L];
        const uint32_t sz = tile_size(p, co);
        if (sz && sz <= kRingBytes) {
            copy_tile(ring_base, p.blob + p.off_payload + uint64_t(co.e0 & 0x7FFFFFFFu) * 16, sz, lane);
            cp_async_commit();
            pending = 1;
        }
    }
    bool waited = true;  // no launch-level wait: stores wait tile by tile (seq_wait)

    for (uint32_t L = 0; L < n; ++L) {
        const uint32_t s = L % kWindows, t0 = win0 + s * kCtxRegion, ts = starts + s * kCtxBytes;
        if (!mbar_wait(bars + 8 * s, (L / kWindows) & 1u, kTableWaitTries) && lane == 0)
            atomicOr(&g_status, int(EP_DEV_TABLE_COPY));
        const LayerDesc& p = sp.L[L];
        const uint16_t* scales = reinterpret_cast<const uint16_t*>(p.blob + p.off_scales);
        const uint8_t* payload = p.blob + p.off_payload;
        const uint32_t per_tile = 32 * p.G;
        while (cur.L == L) {
            const uint32_t tile = cur.tile;
            const uint32_t ng = min(per_tile, p.NG - tile * per_tile);
            const uint32_t raw = (ng * uint32_t(p.r) + 3u) & ~3u, s0 = 128 + raw;
            const uint32_t sz = __shfl_sync(kFullMask, tile_size(p, co), 0);
            const bool ok = sz >= s0;
            const bool in_ring = ok && sz <= kRingBytes;
            const Pos aft = next_pos(sp, nbs, nxt, warp);
            const LayerDesc& pn = sp.L[nxt.L < n ? nxt.L : L];
            const uint32_t nsz = nxt.L < n ? __shfl_sync(kFullMask, tile_size(pn, no), 0) : 0u;
            const bool early = nsz && (in_ring ? sz + nsz <= kRingBytes : nsz <= kRingBytes);
            const uint32_t nplace = early && in_ring && place == 0 ? kRingBytes - nsz : 0u;
            if (aft.L < n) prefetch_l1(pos_toff(sp, aft));  // read at the end of the tile
            cp_async_wait<0>();
            __syncwarp();
            pending = 0;
            const uint8_t* nsrc = pn.blob + pn.off_payload + uint64_t(no.e0 & 0x7FFFFFFFu) * 16;
            if (early) {
                copy_tile(ring_base + nplace, nsrc, nsz, lane);
                cp_async_commit();
                pending = 1;
            }
            if (!ok) {
                if (lane == 0) atomicOr(&g_status, int(EP_DEV_BAD_OFFSETS));
            } else {
                const uint32_t rb = ring_base + place;
                const uint8_t* tp = payload + uint64_t(co.e0 & 0x7FFFFFFFu) * 16;
                TileState st;
                st.x = in_ring ? ld_shared_u32(rb + 4 * lane) : __ldg(reinterpret_cast<const uint32_t*>(tp) + lane);
                st.pb = s0;
                const GlobalWords gwords{tp, s0, sz};
                RowCursor rc;
                const uint8_t* rawsec = tp + 128;
                const uint32_t raw_avail = sz - 128;
                const uint32_t R = (ng + 31) / 32;
                const uint32_t gt0 = tile * per_tile;
                if (sp.ordered) seq_wait(sp, p, gt0, ng, es);
                uint32_t k = 0;
                if (in_ring && p.r == 0) {  // (tiles with raw low bits take the general rounds here)
                    const uint32_t Rf = min(ng / 32, kMaxFastRounds);
                    const uint32_t row0 = gt0 / p.gpr, kr0 = (gt0 - row0 * p.gpr) / 32;
                    const bool esc = __any_sync(kFullMask, co.e0 >> 31);
                    if (p.gpr % 32 == 0) {
                        k = esc ? fast_rounds_v2<MODE, true, true>(p, sp, t0, ts, st, rb, gt0 + lane, lt_mask, Rf, row0, kr0, scales, rc, waited)
                                : fast_rounds_v2<MODE, false, true>(p, sp, t0, ts, st, rb, gt0 + lane, lt_mask, Rf, row0, kr0, scales, rc, waited);
                    } else {
                        rc.start(p, scales, gt0 + lane);
                        k = esc ? fast_rounds_v2<MODE, true, false>(p, sp, t0, ts, st, rb, gt0 + lane, lt_mask, Rf, row0, kr0, scales, rc, waited)
                                : fast_rounds_v2<MODE, false, false>(p, sp, t0, ts, st, rb, gt0 + lane, lt_mask, Rf, row0, kr0, scales, rc, waited);
                    }
                }
                if (k < R) {
                    rc.start(p, scales, gt0 + 32 * k + lane);
                    const RingWords ring{rb};
                    for (; k < R; ++k) {
                        const uint32_t q = 32 * k + lane, g = gt0 + q;
                        const bool full = 32 * k + 32 <= ng;
                        if (in_ring && full && __all_sync(kFullMask, st.pb + 2 * kRoundWords <= sz)) {
                            round_general_v2<MODE, false>(p, t0, ts, ring, rawsec, raw_avail, st, q, true, g, lt_mask, rc.scale());
                        } else {
                            round_general_v2<MODE, true>(p, t0, ts, gwords, rawsec, raw_avail, st, q, q < ng, g, lt_mask,
                                                          rc.scale());
                        }
                        rc.advance(p, scales);
                    }
                }
                __syncwarp();
                const uint32_t used = st.pb - s0, cap = sz - s0;
                const bool good = __all_sync(kFullMask, st.x == kRansL) && used <= cap && cap - used <= 14;
                if (!good && lane == 0) atomicOr(&g_status, int(EP_DEV_CORRUPT_TILE));
            }
            if (sp.ordered) seq_done(sp, L, tile);  // bad tiles too: nothing may wait for them in vain
            if (!early && nsz && nsz <= kRingBytes) {
                __syncwarp();
                copy_tile(ring_base, nsrc, nsz, lane);
                cp_async_commit();
                pending = 1;
            }
            place = early ? nplace : 0u;
            cur = nxt;
            co = no;
            nxt = aft;
            no = pos_offs(sp, aft);
        }
        // Done with layer L. The last of the CTA's warps to get here refills the window with layer
        // L + kWindows, once every warp's reads of it are ordered before the copy.
        __syncwarp();
        if (lane == 0) {
            __threadfence_block();
            if (atomicAdd(done_cnt + s, 1u) == 31u) {
                __threadfence_block();
                done_cnt[s] = 0;
                if (L + kWindows < n) {
                    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
                    load_window(sp, L + kWindows, t0, ts, bars + 8 * s);
                }
            }
        }
    }
    if (pending) cp_async_wait<0>();
}

}  // namespace v2


}  // namespace dev

// ------------------------------------------------------------------------------- launcher

namespace {

struct DeviceInfo {
    int sms = 0;
    bool configured[8] = {false};     // version 1 kernels, by mode
    bool configured_v2[8] = {false};  // version 2 kernels, by mode
    bool configured_seq[8] = {false}; // version 2 sequence kernels, by mode
};
std::mutex g_dev_mu;
DeviceInfo g_dev[64];

template <int MODE>
ep_status launch_mode(const dev::Params& p, cudaStream_t stream, int device, bool chained, int version) {
    const void* fn = version == 1 ? reinterpret_cast<const void*>(dev::decode_kernel<MODE>)
                                  : reinterpret_cast<const void*>(dev::v2::decode_kernel<MODE>);
    const uint32_t smem = version == 1 ? dev::kSmemBytes : dev::v2::kSmemBytes;
    {
        std::lock_guard<std::mutex> lk(g_dev_mu);
        DeviceInfo& d = g_dev[device];
        bool& configured = version == 1 ? d.configured[MODE] : d.configured_v2[MODE];
        if (!configured) {
            cudaError_t e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem));
            if (e != cudaSuccess) return fail(EP_ERR_CUDA, "cudaFuncSetAttribute: %s", cudaGetErrorString(e));
            configured = true;
        }
    }
    // One CTA per SM, or one per tile when there are fewer tiles than SMs.
    uint32_t grid = p.T < uint32_t(g_dev[device].sms) ? p.T : uint32_t(g_dev[device].sms);
    if (grid == 0) grid = 1;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(grid);
    cfg.blockDim = dim3(version == 1 ? dev::kThreads : dev::v2::kThreadsV2);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = chained ? 1 : 0;
    cudaError_t e = version == 1 ? cudaLaunchKernelEx(&cfg, dev::decode_kernel<MODE>, p)
                                 : cudaLaunchKernelEx(&cfg, dev::v2::decode_kernel<MODE>, p);
    if (e == cudaSuccess) e = cudaGetLastError();
    if (e != cudaSuccess) return fail(EP_ERR_CUDA, "decode launch: %s", cudaGetErrorString(e));
    return EP_OK;
}

// next_hdr / next_dev: the following blob of a sequence (its metadata is prefetched to L2), or null.
ep_status launch_decode(const uint8_t* host_hdr, const void* dev_blob, size_t blob_bytes, void* dst, size_t dst_bytes,
                        int mode, void* stream_ptr, bool chained, const uint8_t* next_hdr = nullptr,
                        const void* next_dev = nullptr, const uint32_t* pre_tables = nullptr,
                        bool test_no_table_copy = false) {
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
    p.inv_alpha = 1.0f / h.alpha;  // IEEE binary32 division: RN(1 / alpha)
    p.k2 = 2;
    p.k4 = 4;
    p.kneg4096 = 0xFFFFF000u;
    p.k128 = 128;
    p.kneg256 = 0xFFFFFF00u;
    p.off_scales = h.off_scales;
    p.off_tables = h.off_tables;
    p.off_offsets = h.off_offsets;
    p.off_payload = h.off_payload;
    p.tables_len = h.off_offsets - h.off_tables;
    p.payload_bytes = h.total - h.off_payload;
    p.next_blob = nullptr;
    p.next_meta_off = p.next_meta_bytes = 0;
    p.pre_tables = pre_tables;
    p.test_no_table_copy = test_no_table_copy ? 1u : 0u;
    Header hn;
    if (next_hdr && next_dev && parse_header(next_hdr, hn)) {  // headers of a sequence are checked up front
        p.next_blob = static_cast<const uint8_t*>(next_dev);
        p.next_meta_off = hn.off_scales;
        p.next_meta_bytes = hn.off_payload - hn.off_scales;
    }
    cudaStream_t stream = static_cast<cudaStream_t>(stream_ptr);
    const int v = h.version;
    switch (mode) {
        case dev::kBF16: return launch_mode<dev::kBF16>(p, stream, device, chained, v);
        case dev::kFP16: return launch_mode<dev::kFP16>(p, stream, device, chained, v);
        case dev::kFP32: return launch_mode<dev::kFP32>(p, stream, device, chained, v);
        case dev::kFP8: return launch_mode<dev::kFP8>(p, stream, device, chained, v);
        case dev::kINT8: return launch_mode<dev::kINT8>(p, stream, device, chained, v);
        case dev::kCoords: return launch_mode<dev::kCoords>(p, stream, device, chained, v);
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
    return launch_decode(host_hdr, dev_blob, blob_bytes, dst, dst_bytes, h.dtype, cuda_stream, false);
}

// ep_decompress_many of version-2 blobs with one output type: prep_tables_kernel, then seq_kernel (see there),
// for up to kMaxSeqLayers blobs a launch pair; longer sequences take several pairs, in stream order. Returns
// EP_ERR_NOMEM, having launched nothing, when the stream-ordered scratch cannot be had.
template <int MODE>
ep_status decompress_seq(int count, const uint8_t* const* host_hdrs, const void* const* dev_blobs, void* const* dsts,
                         cudaStream_t stream, int device) {
    using dev::v2::LayerDesc;
    using dev::v2::SeqParams;
    {
        std::lock_guard<std::mutex> lk(g_dev_mu);
        bool& configured = g_dev[device].configured_seq[MODE];
        if (!configured) {
            cudaError_t e = cudaFuncSetAttribute(dev::v2::seq_kernel<MODE>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                                 int(dev::v2::kSeqSmemBytes));
            if (e != cudaSuccess) return fail(EP_ERR_CUDA, "cudaFuncSetAttribute: %s", cudaGetErrorString(e));
            configured = true;
        }
    }
    auto sp = std::make_unique<SeqParams>();
    for (int c0 = 0; c0 < count; c0 += int(dev::v2::kMaxSeqLayers)) {
        const int n = std::min(count - c0, int(dev::v2::kMaxSeqLayers));
        std::memset(sp.get(), 0, sizeof(SeqParams));
        sp->count = uint32_t(n);
        sp->k2 = 2;
        sp->k4 = 4;
        sp->kneg256 = 0xFFFFFF00u;
        std::vector<uint64_t> lo(static_cast<size_t>(n)), hi(static_cast<size_t>(n));
        uint32_t tiles = 0, words = 0;
        for (int i = 0; i < n; ++i) {
            Header h;
            parse_header(host_hdrs[c0 + i], h);
            LayerDesc& d = sp->L[i];
            d.blob = static_cast<const uint8_t*>(dev_blobs[c0 + i]);
            d.dst = dsts[c0 + i];
            d.payload_bytes = h.total - h.off_payload;
            d.gpr = h.N / 8;
            d.T = h.T;
            d.G = uint32_t(h.G);
            d.NG = uint32_t(h.groups());
            d.M = h.M;
            d.r = h.r;
            d.alpha = h.alpha;
            d.inv_alpha = 1.0f / h.alpha;  // IEEE binary32 division: RN(1 / alpha)
            d.off_scales = h.off_scales;
            d.off_offsets = h.off_offsets;
            d.off_payload = h.off_payload;
            d.off_tables = h.off_tables;
            d.tables_len = h.off_offsets - h.off_tables;
            d.tile0 = tiles;
            d.bits = words;
            tiles += h.T;
            words += (h.T + 31) / 32;
            lo[size_t(i)] = reinterpret_cast<uint64_t>(d.dst);
            hi[size_t(i)] = lo[size_t(i)] + uint64_t(h.M) * h.N * uint64_t(elem_bytes(h.dtype));
            // The latest earlier writer of each byte of this layer's output: split the range by going back
            // through the layers; a writer's pieces merge into their hull (waiting for a few more of its tiles
            // is harmless). The two latest writers are waited for tile by tile, older ones as whole layers.
            d.seg_layer[0] = d.seg_layer[1] = dev::v2::kNoDep;
            const uint64_t gb = 8 * uint64_t(elem_bytes(h.dtype));
            std::vector<std::pair<uint64_t, uint64_t>> open{{lo[size_t(i)], hi[size_t(i)]}};
            int nd = 0;
            for (int j = i - 1; j >= 0 && hi[size_t(i)] > lo[size_t(i)] && !open.empty(); --j) {
                if (hi[size_t(j)] <= lo[size_t(j)]) continue;
                std::vector<std::pair<uint64_t, uint64_t>> rest;
                uint64_t a0 = ~0ull, b0 = 0;
                for (const auto& u : open) {
                    const uint64_t a = std::max(u.first, lo[size_t(j)]), b = std::min(u.second, hi[size_t(j)]);
                    if (a >= b) {
                        rest.push_back(u);
                        continue;
                    }
                    a0 = std::min(a0, a);
                    b0 = std::max(b0, b);
                    if (u.first < a) rest.emplace_back(u.first, a);
                    if (b < u.second) rest.emplace_back(b, u.second);
                }
                open.swap(rest);
                if (b0 == 0) continue;
                if (nd < 2) {
                    d.seg_layer[nd] = uint16_t(j);
                    d.seg_lo[nd] = uint32_t((a0 - lo[size_t(i)]) / gb);
                    d.seg_hi[nd] = uint32_t((b0 - lo[size_t(i)] + gb - 1) / gb);
                    ++nd;
                } else {
                    d.need_prefix = uint32_t(j + 1);  // the latest of the older writers
                    break;
                }
            }
            if (d.need_prefix) sp->use_prefix = 1;
            if (nd) sp->ordered = 1;
        }
        sp->counts_off = words;
        sp->prefix_off = words + uint32_t(n);
        const size_t order_words = size_t(sp->prefix_off) + 1;
        const size_t table_bytes = size_t(n) * dev::v2::kTablesBytes;
        cudaMemPool_t pool;
        uint8_t* scratch = nullptr;
        if (scratch_pool(&pool) != cudaSuccess ||
            cudaMallocFromPoolAsync(reinterpret_cast<void**>(&scratch), table_bytes + order_words * 4, pool, stream) !=
                cudaSuccess) {
            cudaGetLastError();
            return fail(EP_ERR_NOMEM, "ep_decompress_many: no stream-ordered scratch for the sequence tables");
        }
        sp->tables = reinterpret_cast<const uint32_t*>(scratch);
        sp->order = reinterpret_cast<uint32_t*>(scratch + table_bytes);
        cudaError_t e = sp->ordered ? cudaMemsetAsync(sp->order, 0, order_words * 4, stream) : cudaSuccess;
        if (e == cudaSuccess) {
            dev::v2::prep_tables_kernel<<<unsigned(n), dev::v2::kThreadsV2, dev::v2::kScratchSize, stream>>>(*sp);
            e = cudaGetLastError();
        }
        if (e == cudaSuccess) {
            cudaLaunchConfig_t cfg = {};
            cfg.gridDim = dim3(unsigned(g_dev[device].sms));
            cfg.blockDim = dim3(dev::v2::kThreadsV2);
            cfg.dynamicSmemBytes = dev::v2::kSeqSmemBytes;
            cfg.stream = stream;
            // Every CTA is resident at once: a tile may wait for a tile of another CTA.
            cudaLaunchAttribute attr[1];
            attr[0].id = cudaLaunchAttributeCooperative;
            attr[0].val.cooperative = 1;
            cfg.attrs = attr;
            cfg.numAttrs = 1;
            e = cudaLaunchKernelEx(&cfg, dev::v2::seq_kernel<MODE>, *sp);
            if (e == cudaSuccess) e = cudaGetLastError();
        }
        cudaFreeAsync(scratch, stream);
        if (e != cudaSuccess) return fail(EP_ERR_CUDA, "sequence decode launch: %s", cudaGetErrorString(e));
    }
    return EP_OK;
}

extern "C" ep_status ep_decompress_many(int count, const uint8_t* const* host_hdrs, const void* const* dev_blobs,
                                        const size_t* blob_bytes, void* const* dsts, const size_t* dst_bytes,
                                        void* cuda_stream) {
    clear_error();
    if (count < 0 || (count > 0 && (!host_hdrs || !dev_blobs || !blob_bytes || !dsts || !dst_bytes)))
        return fail(EP_ERR_ARG, "ep_decompress_many: bad arguments");
    // Validate every header, size, pointer and alignment before launching anything, so a failure launches
    // nothing, whichever path the list then takes.
    for (int i = 0; i < count; ++i) {
        Header h;
        if (!host_hdrs[i] || !parse_header(host_hdrs[i], h))
            return fail(EP_ERR_CORRUPT, "ep_decompress_many: blob %d has a malformed header", i);
        if (h.total != blob_bytes[i]) return fail(EP_ERR_BUFFER, "ep_decompress_many: blob %d size mismatch", i);
        if (!dev_blobs[i] || !dsts[i]) return fail(EP_ERR_ARG, "ep_decompress_many: NULL blob or dst %d", i);
        if ((reinterpret_cast<uintptr_t>(dev_blobs[i]) & 15) || (reinterpret_cast<uintptr_t>(dsts[i]) & 15))
            return fail(EP_ERR_BUFFER, "ep_decompress_many: blob and dst %d must be 16-byte aligned", i);
        const uint64_t need = uint64_t(h.M) * h.N * uint64_t(elem_bytes(h.dtype));
        if (dst_bytes[i] < need)
            return fail(EP_ERR_BUFFER, "ep_decompress_many: dst %d holds %zu bytes, need %llu", i, dst_bytes[i],
                        (unsigned long long)need);
    }
    // The fused entries of every version-1 blob, built once for the sequence into stream-ordered scratch
    // (144 KB per blob). The first decode launches in plain stream order behind the expand kernel, and every
    // later one starts after it, so all of them read finished tables. Without the scratch, each CTA builds
    // its own tables. (A list of version-2 blobs of one dtype has returned through decompress_seq above; in a
    // mixed list, each version-2 decode builds its 9 KB of tables in each CTA.)
    cudaStream_t stream = static_cast<cudaStream_t>(cuda_stream);
    constexpr size_t kWords = dev::kTablesBytes / 4;
    std::vector<int> v1;  // indices of the version-1 blobs, in order; blob v1[j] takes prepared slot j
    std::vector<int> slot_of(size_t(count), -1);
    for (int i = 0; i < count; ++i) {
        Header h;
        parse_header(host_hdrs[i], h);
        if (h.version == 1) {
            slot_of[size_t(i)] = int(v1.size());
            v1.push_back(i);
        }
    }
    const int n1 = int(v1.size());
    // Version-2 blobs that share one output type: the sequence kernel.
    bool one_type = count >= 2 && n1 == 0;
    int dtype = -1;
    for (int i = 0; one_type && i < count; ++i) {
        Header h;
        parse_header(host_hdrs[i], h);
        if (dtype < 0) dtype = h.dtype;
        one_type = h.dtype == dtype;
    }
    if (one_type) {
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
        switch (dtype) {
            case dev::kBF16: return decompress_seq<dev::kBF16>(count, host_hdrs, dev_blobs, dsts, stream, device);
            case dev::kFP16: return decompress_seq<dev::kFP16>(count, host_hdrs, dev_blobs, dsts, stream, device);
            case dev::kFP32: return decompress_seq<dev::kFP32>(count, host_hdrs, dev_blobs, dsts, stream, device);
            case dev::kFP8: return decompress_seq<dev::kFP8>(count, host_hdrs, dev_blobs, dsts, stream, device);
            case dev::kINT8: return decompress_seq<dev::kINT8>(count, host_hdrs, dev_blobs, dsts, stream, device);
        }
        return fail(EP_ERR_DTYPE, "ep_decompress_many: unknown dtype %d", dtype);
    }
    uint32_t* pre = nullptr;
    if (count >= 2 && n1 >= 1) {
        cudaMemPool_t pool;
        if (scratch_pool(&pool) != cudaSuccess ||
            cudaMallocFromPoolAsync(reinterpret_cast<void**>(&pre), size_t(n1) * dev::kTablesBytes, pool, stream) !=
                cudaSuccess) {
            cudaGetLastError();
            pre = nullptr;
        }
        for (int b = 0; pre && b < n1; b += dev::kMaxExpandJobs) {
            dev::ExpandArgs a;
            a.count = n1 - b < dev::kMaxExpandJobs ? n1 - b : dev::kMaxExpandJobs;
            a.out = pre + size_t(b) * kWords;
            for (int j = 0; j < a.count; ++j) {
                Header h;
                const int i = v1[size_t(b + j)];
                parse_header(host_hdrs[i], h);
                a.tables[j] = static_cast<const uint8_t*>(dev_blobs[i]) + h.off_tables;
                a.tables_len[j] = h.off_offsets - h.off_tables;
            }
            dev::expand_tables_kernel<<<unsigned(a.count) * kNumCtx, 256, 0, stream>>>(a);
            if (cudaGetLastError() != cudaSuccess) {
                cudaFreeAsync(pre, stream);
                pre = nullptr;
            }
        }
    }
    // Test hook (see the header): the prepared-table copies are left unissued, so that every CTA's
    // bounded wait for them runs out.
    const char* hook = std::getenv("EPK_TEST_TABLE_COPY_TIMEOUT");
    const bool no_copy = hook && hook[0] == '1';
    for (int i = 0; i < count; ++i) {
        Header h;
        parse_header(host_hdrs[i], h);
        const int slot = slot_of[size_t(i)];
        ep_status st = launch_decode(host_hdrs[i], dev_blobs[i], blob_bytes[i], dsts[i], dst_bytes[i], h.dtype,
                                     cuda_stream, i > 0, i + 1 < count ? host_hdrs[i + 1] : nullptr,
                                     i + 1 < count ? dev_blobs[i + 1] : nullptr,
                                     (pre && slot >= 0) ? pre + size_t(slot) * kWords : nullptr, no_copy);
        if (st != EP_OK) {
            if (pre) cudaFreeAsync(pre, stream);
            return st;
        }
    }
    if (pre) cudaFreeAsync(pre, stream);
    return EP_OK;
}

extern "C" ep_status ep_decode_coords_into(const uint8_t* host_hdr, const void* dev_blob, size_t blob_bytes,
                                           int32_t* dst_z, size_t dst_bytes, void* cuda_stream) {
    clear_error();
    return launch_decode(host_hdr, dev_blob, blob_bytes, dst_z, dst_bytes, dev::kCoords, cuda_stream, false);
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
    ep_status st = launch_decode(host_hdr, dev_blob, blob_bytes, out, bytes, h.dtype, cuda_stream, false);
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

// Lossless tile-ANS decode (shares the status word and the device table above).
#include "tans_format.h"
#include "tans_decode.cuh"
