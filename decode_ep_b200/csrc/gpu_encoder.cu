// CUDA encoder of the EPK1 blob: ep_compress_cuda. It writes the same bytes as the host encoder
// (ep_compress), from a tensor already in device memory. It runs once per tensor and is not the decode
// hot path.
//
// The method's steps (arXiv 2609.34185, abstract; modelscope summary) map onto kernels:
//   - row scales s_row = bf16(RMS) and max |w|/s: one thread per row, summing in index order;
//   - rate control: bisection on log2(alpha). Each probe quantises the row sample on the GPU and counts
//     (context, symbol) pairs there; the host fits the frequency tables to the counts and takes the storage
//     estimate with the same code as the host encoder;
//   - quantisation of every group to E8 at the final alpha, then the counts of the whole tensor;
//   - rANS coding: one warp per tile, in the exact reverse of the decode order of the blob's format version. The lanes that emit a
//     word at a step place it with a ballot and a popcount, from the end of the tile's word buffer, so
//     the buffer reads forward in decode order;
//   - assembly: one warp per tile copies states, raw low bits and words to the tile's offset.
// The lattice arithmetic is shared with the host encoder (lattice_code.h). This file is compiled with
// --fmad=false, so every double operation is rounded on its own, as on the host.
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include <cmath>
#include <cstdlib>
#include <cstring>
#include <mutex>
#include <vector>

#include "capi_internal.h"
#include "encoder_common.h"
#include "entropack.h"
#include "epk_format.h"
#include "lattice_code.h"

namespace epk {
namespace genc {

using namespace enc;

constexpr int kHistBins = kNumCtx * 128;

// A strided row-major tensor of one of the five container types, read as binary32.
struct Src {
    const uint8_t* base;
    int dtype;
    int64_t N, stride;  // elements
};

__device__ __forceinline__ float e4m3_to_float(uint32_t c) {
    const uint32_t e = (c >> 3) & 15u, m = c & 7u, sign = (c & 0x80u) << 24;
    if (e == 15u && m == 7u) return __uint_as_float(0x7FC00000u);   // the only NaN code
    if (e == 0u) return __uint_as_float(sign | __float_as_uint(float(m) * 0x1p-9f));  // subnormal: m 2^-9
    return __uint_as_float(sign | ((e + 120u) << 23) | (m << 20));  // (1 + m/8) 2^(e-7)
}

__device__ __forceinline__ float load_w(const Src& s, int64_t i, int64_t j) {
    const int64_t k = i * s.stride + j;
    switch (s.dtype) {
        case EP_BF16: return __uint_as_float(uint32_t(reinterpret_cast<const uint16_t*>(s.base)[k]) << 16);
        case EP_FP16: return __half2float(__ushort_as_half(reinterpret_cast<const unsigned short*>(s.base)[k]));
        case EP_FP32: return reinterpret_cast<const float*>(s.base)[k];
        case EP_FP8_E4M3: return e4m3_to_float(s.base[k]);
        default: return float(reinterpret_cast<const int8_t*>(s.base)[k]);
    }
}

__device__ __forceinline__ uint16_t bf16_rne(float f) {
    const uint32_t u = __float_as_uint(f);
    return uint16_t((u + 0x7FFFu + ((u >> 16) & 1u)) >> 16);  // finite, non-negative inputs
}

// Row scales: s_row = bf16(fl32(sqrt(Σ w² / N))), the sum in double and index order, then the largest
// |w| / s over rows with s != 0. A correctly rounded division is monotonic, so the largest quotient is
// the quotient of the largest |w|: one division per row. One thread per row, reading it in index
// order. The chain of N dependent double additions per row sets the kernel's time; a row's values are
// reused from L1, so staging them through shared memory does not help.
constexpr int kScaleWarps = 4;

template <int DT>
__device__ __forceinline__ float load_as(const uint8_t* base, int64_t k) {
    if constexpr (DT == EP_BF16) return __uint_as_float(uint32_t(reinterpret_cast<const uint16_t*>(base)[k]) << 16);
    else if constexpr (DT == EP_FP16) return __half2float(__ushort_as_half(reinterpret_cast<const unsigned short*>(base)[k]));
    else if constexpr (DT == EP_FP32) return reinterpret_cast<const float*>(base)[k];
    else if constexpr (DT == EP_FP8_E4M3) return e4m3_to_float(base[k]);
    else return float(reinterpret_cast<const int8_t*>(base)[k]);
}

template <int DT>
__global__ void __launch_bounds__(32 * kScaleWarps) row_scales_kernel(Src src, int64_t M, uint16_t* sbits, float* s_out,
                                                                     unsigned long long* amax_bits, int* nonfinite) {
    const int64_t i = int64_t(blockIdx.x) * blockDim.x + threadIdx.x;
    if (i >= M) return;
    const uint8_t* row = src.base + i * src.stride * int64_t(DT == EP_FP32 ? 4 : (DT == EP_BF16 || DT == EP_FP16 ? 2 : 1));
    double acc = 0.0;
    float wmax = 0.f;
    bool finite = true;
    for (int64_t j = 0; j < src.N; ++j) {
        const float w = load_as<DT>(row, j);
        finite = finite && isfinite(w);
        acc = __dadd_rn(acc, __dmul_rn(double(w), double(w)));
        wmax = fmaxf(wmax, fabsf(w));
    }
    if (!finite) {
        atomicOr(nonfinite, 1);
        return;
    }
    const float rms = __double2float_rn(__dsqrt_rn(__ddiv_rn(acc, double(src.N))));
    const uint16_t sb = bf16_rne(rms);
    const float s = __uint_as_float(uint32_t(sb) << 16);
    sbits[i] = sb;
    s_out[i] = s;
    const double m = s != 0.f ? __ddiv_rn(double(wmax), double(s)) : 0.0;
    atomicMax(amax_bits, static_cast<unsigned long long>(__double_as_longlong(m)));  // m >= 0: bits order as values
}

// Launches row_scales_kernel for the source's dtype.
inline cudaError_t launch_row_scales(const Src& src, int64_t M, uint16_t* sbits, float* s_out,
                                     unsigned long long* amax_bits, int* nonfinite, cudaStream_t st) {
    const unsigned blocks = unsigned((M + 32 * kScaleWarps - 1) / (32 * kScaleWarps));
    switch (src.dtype) {
        case EP_BF16: row_scales_kernel<EP_BF16><<<blocks, 32 * kScaleWarps, 0, st>>>(src, M, sbits, s_out, amax_bits, nonfinite); break;
        case EP_FP16: row_scales_kernel<EP_FP16><<<blocks, 32 * kScaleWarps, 0, st>>>(src, M, sbits, s_out, amax_bits, nonfinite); break;
        case EP_FP32: row_scales_kernel<EP_FP32><<<blocks, 32 * kScaleWarps, 0, st>>>(src, M, sbits, s_out, amax_bits, nonfinite); break;
        case EP_FP8_E4M3: row_scales_kernel<EP_FP8_E4M3><<<blocks, 32 * kScaleWarps, 0, st>>>(src, M, sbits, s_out, amax_bits, nonfinite); break;
        default: row_scales_kernel<EP_INT8><<<blocks, 32 * kScaleWarps, 0, st>>>(src, M, sbits, s_out, amax_bits, nonfinite); break;
    }
    return cudaGetLastError();
}

// Quantises group q of row i at alpha: x_k = (alpha w_k) / s in double, then the nearest E8 point.
__device__ __forceinline__ int quantize_group(const Src& src, const float* s, int64_t i, int64_t q, float alpha,
                                              int32_t* t) {
    const double sd = double(s[i]), ad = double(alpha);
    double x[8];
#pragma unroll
    for (int k = 0; k < 8; ++k)
        x[k] = (sd == 0.0) ? 0.0 : __ddiv_rn(__dmul_rn(ad, double(load_w(src, i, q * 8 + k))), sd);
    return e8_code(x, t);
}

// Adds a thread's 8 (context, symbol) pairs to the block's shared histogram.
__device__ __forceinline__ void count_group(unsigned int* h, int b, const int32_t* t, int r) {
    uint8_t ctx[8], sym[8];
    int32_t hi[8];
    group_syms(b, t, r, ctx, sym, hi);
#pragma unroll
    for (int k = 0; k < 8; ++k) atomicAdd(&h[ctx[k] * 128 + sym[k]], 1u);
}

__device__ __forceinline__ void flush_hist(const unsigned int* h, unsigned long long* counts) {
    for (int k = threadIdx.x; k < kHistBins; k += blockDim.x)
        if (h[k]) atomicAdd(&counts[k], static_cast<unsigned long long>(h[k]));
}

// Rate-control probes evaluated in one launch: blockIdx.y picks the probe.
constexpr int kProbeDepth = 4;                         // bisection steps resolved per launch
constexpr int kMaxProbes = (1 << kProbeDepth) - 1;     // every midpoint those steps can visit
struct Probes {
    float alpha[kMaxProbes];
    int r[kMaxProbes];
};

// Counts of the row sample at probe blockIdx.y's alpha: rows floor(k M / Rs), k < Rs, every group of
// each. counts holds one histogram per probe.
__global__ void sample_counts_kernel(Src src, int64_t M, int64_t gpr, int64_t Rs, const float* s, Probes pr,
                                     unsigned long long* counts) {
    const float alpha = pr.alpha[blockIdx.y];
    const int r = pr.r[blockIdx.y];
    counts += size_t(blockIdx.y) * kHistBins;
    __shared__ unsigned int h[kHistBins];
    for (int k = threadIdx.x; k < kHistBins; k += blockDim.x) h[k] = 0;
    __syncthreads();
    const int64_t gi = int64_t(blockIdx.x) * blockDim.x + threadIdx.x;
    if (gi < Rs * gpr) {
        const int64_t k = gi / gpr, q = gi - k * gpr, row = (k * M) / Rs;
        int32_t t[8];
        const int b = quantize_group(src, s, row, q, alpha, t);
        count_group(h, b, t, r);
    }
    __syncthreads();
    flush_hist(h, counts);
}

// Every group at the final alpha: coded integers t (8 per group), coset bits, and the largest
// a = (t >= 0 ? t : -t - 1).
__global__ void quantize_kernel(Src src, int64_t NG, int64_t gpr, const float* s, float alpha, int32_t* tq, uint8_t* bq,
                                unsigned long long* tmax) {
    const int64_t g = int64_t(blockIdx.x) * blockDim.x + threadIdx.x;
    int64_t a = 0;
    if (g < NG) {
        const int64_t i = g / gpr, q = g - i * gpr;
        int32_t t[8];
        bq[g] = uint8_t(quantize_group(src, s, i, q, alpha, t));
#pragma unroll
        for (int k = 0; k < 8; ++k) {
            tq[g * 8 + k] = t[k];
            const int64_t v = t[k], m = v >= 0 ? v : -v - 1;
            a = m > a ? m : a;
        }
    }
    for (int d = 16; d; d >>= 1) {
        const int64_t o = __shfl_xor_sync(0xFFFFFFFFu, a, d);
        a = o > a ? o : a;
    }
    if ((threadIdx.x & 31) == 0 && a) atomicMax(tmax, static_cast<unsigned long long>(a));
}

// Counts of the whole tensor from the coded integers.
__global__ void full_counts_kernel(const int32_t* tq, const uint8_t* bq, int64_t NG, int r, unsigned long long* counts) {
    __shared__ unsigned int h[kHistBins];
    for (int k = threadIdx.x; k < kHistBins; k += blockDim.x) h[k] = 0;
    __syncthreads();
    for (int64_t g = int64_t(blockIdx.x) * blockDim.x + threadIdx.x; g < NG; g += int64_t(gridDim.x) * blockDim.x) {
        int32_t t[8];
#pragma unroll
        for (int k = 0; k < 8; ++k) t[k] = tq[g * 8 + k];
        count_group(h, bq[g], t, r);
    }
    __syncthreads();
    flush_hist(h, counts);
}

// rANS coding of one tile per warp, in the exact reverse of the decode order. Word buffer of tile j:
// words[j cap, (j + 1) cap) with cap = 16 words per group (a renorm word and an escape word per
// coordinate at most). Words are placed from the end backwards; at each step the emitting lanes take
// consecutive slots with the highest lane last, so the used part [cap - n, cap) reads forward in decode
// order: per step, renorm words first, then escape words, lanes ascending.
__global__ void encode_tiles_kernel(const int32_t* tq, const uint8_t* bq, int64_t NG, uint32_t T, int G, int r,
                                    const uint32_t* ftab, const uint32_t* ctab, uint16_t* words, uint32_t* states,
                                    uint32_t* nwords, uint8_t* esc_flag) {
    __shared__ uint32_t F[kHistBins], C[kHistBins];
    for (int k = threadIdx.x; k < kHistBins; k += blockDim.x) {
        F[k] = ftab[k];
        C[k] = ctab[k];
    }
    __syncthreads();
    const uint32_t lane = threadIdx.x & 31, tile = blockIdx.x * (blockDim.x / 32) + (threadIdx.x >> 5);
    if (tile >= T) return;
    const int64_t per = 32 * int64_t(G), g0 = int64_t(tile) * per, ng = min(per, NG - g0), cap = 16 * per;
    uint16_t* wbuf = words + int64_t(tile) * cap;
    const uint32_t gt = ~((2u << lane) - 1u);  // lanes above this one
    uint32_t x = kRansL;
    int64_t cur = cap;
    bool any_esc = false;
    for (int64_t k = (ng + 31) / 32 - 1; k >= 0; --k) {
        const int64_t gl = 32 * k + lane;
        const bool active = gl < ng;
        uint8_t ctx[8] = {0}, sym[8] = {0};
        int32_t hi[8] = {0};
        if (active) {
            int32_t t[8];
#pragma unroll
            for (int kk = 0; kk < 8; ++kk) t[kk] = tq[(g0 + gl) * 8 + kk];
            group_syms(bq[g0 + gl], t, r, ctx, sym, hi);
        }
#pragma unroll
        for (int i = 7; i >= 0; --i) {
            const bool e = active && idx_of(hi[i]) == kEscIdx;
            const uint32_t me = __ballot_sync(0xFFFFFFFFu, e);
            if (me) {
                if (e) wbuf[cur - 1 - __popc(me & gt)] = uint16_t(int16_t(hi[i]));
                cur -= __popc(me);
                any_esc = true;
            }
            uint32_t f = 1, c = 0;
            if (active) {
                f = F[ctx[i] * 128 + sym[i]];
                c = C[ctx[i] * 128 + sym[i]];
            }
            const bool emit = active && x >= (f << 20);
            const uint32_t mw = __ballot_sync(0xFFFFFFFFu, emit);
            if (emit) {
                wbuf[cur - 1 - __popc(mw & gt)] = uint16_t(x);
                x >>= 16;
            }
            cur -= __popc(mw);
            if (active) x = (x / f) * kProbScale + (x % f) + c;
        }
    }
    states[int64_t(tile) * 32 + lane] = x;
    if (lane == 0) {
        nwords[tile] = uint32_t(cap - cur);
        esc_flag[tile] = any_esc ? 1 : 0;
    }
}

// Format version 2: rANS coding of one tile per warp, in the exact reverse of its decode order. The words
// are placed from the end of the tile's buffer backwards, as in encode_tiles_kernel. Per round, from the
// last: the round's escape words (positions descending; within a position the highest lane takes the
// highest slot), then each pair of positions from the last: lanes with x >= f1 f2 2^16 place x & 0xFFFF
// and shift x right by 16, then x <- C(s2, x), x <- C(s1, x) in base 256. A symbol the tables give no
// frequency is coded as its escape (ftab is indexed by context * 128 + symbol).
__global__ void encode_tiles_v2_kernel(const int32_t* tq, const uint8_t* bq, int64_t NG, uint32_t T, int G, int r,
                                       const uint32_t* ftab, const uint32_t* ctab, uint16_t* words, uint32_t* states,
                                       uint32_t* nwords, uint8_t* esc_flag) {
    __shared__ uint32_t F[kHistBins], C[kHistBins];
    for (int k = threadIdx.x; k < kHistBins; k += blockDim.x) {
        F[k] = ftab[k];
        C[k] = ctab[k];
    }
    __syncthreads();
    const uint32_t lane = threadIdx.x & 31, tile = blockIdx.x * (blockDim.x / 32) + (threadIdx.x >> 5);
    if (tile >= T) return;
    const int64_t per = 32 * int64_t(G), g0 = int64_t(tile) * per, ng = min(per, NG - g0), cap = 16 * per;
    uint16_t* wbuf = words + int64_t(tile) * cap;
    const uint32_t gt = ~((2u << lane) - 1u);  // lanes above this one
    uint32_t x = kRansL;
    int64_t cur = cap;
    bool any_esc = false;
    for (int64_t k = (ng + 31) / 32 - 1; k >= 0; --k) {
        const int64_t gl = 32 * k + lane;
        const bool active = gl < ng;
        uint8_t ctx[8] = {0}, sym[8] = {0};
        int32_t hi[8] = {0};
        if (active) {
            int32_t t[8];
#pragma unroll
            for (int kk = 0; kk < 8; ++kk) t[kk] = tq[(g0 + gl) * 8 + kk];
            group_syms(bq[g0 + gl], t, r, ctx, sym, hi);
#pragma unroll
            for (int i = 0; i < 8; ++i)
                if (F[ctx[i] * 128 + sym[i]] == 0) sym[i] = uint8_t((sym[i] & 64) | kEscIdx);
        }
#pragma unroll
        for (int i = 7; i >= 0; --i) {
            const bool e = active && (sym[i] & 63) == kEscIdx;
            const uint32_t me = __ballot_sync(0xFFFFFFFFu, e);
            if (me) {
                if (e) wbuf[cur - 1 - __popc(me & gt)] = uint16_t(int16_t(hi[i]));
                cur -= __popc(me);
                any_esc = true;
            }
        }
#pragma unroll
        for (int p = 3; p >= 0; --p) {
            uint32_t f1 = 1, c1 = 0, f2 = 1, c2 = 0;
            if (active) {
                f1 = F[ctx[2 * p] * 128 + sym[2 * p]];
                c1 = C[ctx[2 * p] * 128 + sym[2 * p]];
                f2 = F[ctx[2 * p + 1] * 128 + sym[2 * p + 1]];
                c2 = C[ctx[2 * p + 1] * 128 + sym[2 * p + 1]];
            }
            const bool emit = active && x >= ((f1 * f2) << 16);  // f1 f2 <= 255^2: the product fits 32 bits
            const uint32_t mw = __ballot_sync(0xFFFFFFFFu, emit);
            if (emit) {
                wbuf[cur - 1 - __popc(mw & gt)] = uint16_t(x);
                x >>= 16;
            }
            cur -= __popc(mw);
            if (active) {
                x = (x / f2) * kProbScaleV2 + (x % f2) + c2;
                x = (x / f1) * kProbScaleV2 + (x % f1) + c1;
            }
        }
    }
    states[int64_t(tile) * 32 + lane] = x;
    if (lane == 0) {
        nwords[tile] = uint32_t(cap - cur);
        esc_flag[tile] = any_esc ? 1 : 0;
    }
}

// One warp per tile writes its payload at start[tile] of the zeroed payload: 32 final states, the raw
// section (8 fields of r bits per group, LSB first, r bytes per group, padded to 4), then the words.
__global__ void assemble_kernel(uint8_t* payload, const uint64_t* start, const uint32_t* states, const uint16_t* words,
                                const uint32_t* nwords, const int32_t* tq, int64_t NG, uint32_t T, int G, int r) {
    const uint32_t lane = threadIdx.x & 31, tile = blockIdx.x * (blockDim.x / 32) + (threadIdx.x >> 5);
    if (tile >= T) return;
    const int64_t per = 32 * int64_t(G), g0 = int64_t(tile) * per, ng = min(per, NG - g0), cap = 16 * per;
    uint8_t* dst = payload + start[tile];
    reinterpret_cast<uint32_t*>(dst)[lane] = states[int64_t(tile) * 32 + lane];
    const uint64_t raw = (uint64_t(ng) * uint64_t(r) + 3) & ~uint64_t(3);
    if (r > 0) {
        const uint32_t mask = (1u << r) - 1u;
        for (int64_t q = lane; q < ng; q += 32) {
            uint64_t lo64 = 0, hi64 = 0;
            for (int i = 0; i < 8; ++i) {
                const uint32_t v = uint32_t(tq[(g0 + q) * 8 + i]) & mask;
                const int pos = i * r;
                if (pos < 64) {
                    lo64 |= uint64_t(v) << pos;
                    if (pos + r > 64) hi64 |= uint64_t(v) >> (64 - pos);
                } else {
                    hi64 |= uint64_t(v) << (pos - 64);
                }
            }
            uint8_t* rp = dst + 128 + q * r;
            for (int byte = 0; byte < r; ++byte)
                rp[byte] = byte < 8 ? uint8_t(lo64 >> (8 * byte)) : uint8_t(hi64 >> (8 * (byte - 8)));
        }
    }
    const uint32_t n = nwords[tile];
    const uint16_t* src = words + int64_t(tile) * cap + (cap - n);
    uint16_t* wd = reinterpret_cast<uint16_t*>(dst + 128 + raw);
    for (uint32_t w = lane; w < n; w += 32) wd[w] = src[w];
}

}  // namespace genc
}  // namespace epk

// ----------------------------------------------------------------------------- host side

namespace epk {
namespace {

using namespace enc;

// Stream-ordered device scratch, released on the stream when it goes out of scope.
struct DevBuf {
    void* p = nullptr;
    cudaStream_t s = nullptr;
    cudaError_t alloc(size_t bytes, cudaStream_t st) {
        s = st;
        cudaMemPool_t pool;
        cudaError_t e = scratch_pool(&pool);
        if (e != cudaSuccess) return e;
        return cudaMallocFromPoolAsync(&p, bytes ? bytes : 16, pool, st);
    }
    ~DevBuf() {
        if (p) cudaFreeAsync(p, s);
    }
    template <class T>
    T* as() const { return static_cast<T*>(p); }
};

#define EPK_CUDA_IN(fn, call)                                                                       \
    do {                                                                                             \
        cudaError_t e_ = (call);                                                                     \
        if (e_ != cudaSuccess) return fail(EP_ERR_CUDA, fn ": %s: %s", #call, cudaGetErrorString(e_)); \
    } while (0)
#define EPK_CUDA(call) EPK_CUDA_IN("ep_compress_cuda", call)

unsigned blocks_for(int64_t n, int per) { return unsigned((n + per - 1) / per); }

}  // namespace
}  // namespace epk

using namespace epk;

extern "C" ep_status ep_compress_cuda(const void* dev_data, ep_dtype dt, int64_t rows, int64_t cols, int64_t row_stride,
                                      double target_bpp, const ep_options* opt_in, void* cuda_stream,
                                      uint8_t** blob_out, size_t* blob_bytes, double* actual_bpp) {
    clear_error();
    if (!dev_data || !blob_out || !blob_bytes) return fail(EP_ERR_ARG, "ep_compress_cuda: NULL argument");
    if (!elem_bytes(int(dt))) return fail(EP_ERR_DTYPE, "ep_compress_cuda: unknown dtype %d", int(dt));
    if (rows < 1 || cols < 8 || cols % 8 != 0 || rows > 0xFFFFFFFFll || cols > 0xFFFFFFFFll ||
        (rows * cols) / 8 > 0xFFFFFFFFll)
        return fail(EP_ERR_SHAPE, "ep_compress_cuda: need a 2-D tensor with rows >= 1 and cols a positive multiple of 8 (got %lld x %lld)",
                    (long long)rows, (long long)cols);
    if (row_stride < cols) return fail(EP_ERR_ARG, "ep_compress_cuda: row_stride %lld < cols", (long long)row_stride);
    if (!(target_bpp >= 0.001 && target_bpp <= 11.0))
        return fail(EP_ERR_TARGET, "ep_compress_cuda: target_bpp must be finite and in [0.001, 11]");
    ep_options opt;
    ep_options_default(&opt);
    if (opt_in) opt = *opt_in;
    if (opt.rounds_per_tile == 0) opt.rounds_per_tile = auto_rounds_per_tile(rows * cols / 8);
    if (opt.format_version == 0) opt.format_version = 2;
    if (opt.rounds_per_tile < 1 || opt.rounds_per_tile > uint32_t(kMaxG) || opt.sample_coords < 1 ||
        opt.bisection_iters > 200 || opt.format_version > 2)
        return fail(EP_ERR_ARG, "ep_compress_cuda: bad options");
    const int version = int(opt.format_version);
    cudaPointerAttributes pa;
    if (cudaPointerGetAttributes(&pa, dev_data) != cudaSuccess || pa.type != cudaMemoryTypeDevice) {
        cudaGetLastError();
        return fail(EP_ERR_ARG, "ep_compress_cuda: the input is not device memory");
    }

    cudaStream_t st = static_cast<cudaStream_t>(cuda_stream);
    const int64_t M = rows, N = cols, NG = M * N / 8, gpr = N / 8;
    const int G = int(opt.rounds_per_tile);
    const uint32_t T = uint32_t((NG + 32 * int64_t(G) - 1) / (32 * int64_t(G)));
    const genc::Src src{static_cast<const uint8_t*>(dev_data), int(dt), N, row_stride};
    try {
        // Row scales and max |w| / s.
        DevBuf d_sbits, d_s, d_small, d_counts;
        EPK_CUDA(d_sbits.alloc(size_t(M) * 2, st));
        EPK_CUDA(d_s.alloc(size_t(M) * 4, st));
        EPK_CUDA(d_small.alloc(64, st));  // [0] amax bits, [2] tmax, [3] nonfinite flag
        EPK_CUDA(d_counts.alloc(sizeof(unsigned long long) * genc::kHistBins, st));
        unsigned long long* small = d_small.as<unsigned long long>();
        EPK_CUDA(cudaMemsetAsync(small, 0, 64, st));
        EPK_CUDA(genc::launch_row_scales(src, M, d_sbits.as<uint16_t>(), d_s.as<float>(), small,
                                         reinterpret_cast<int*>(small + 3), st));
        std::vector<uint16_t> sbits(static_cast<size_t>(M));
        unsigned long long hsmall[4];
        EPK_CUDA(cudaMemcpyAsync(sbits.data(), d_sbits.p, size_t(M) * 2, cudaMemcpyDeviceToHost, st));
        EPK_CUDA(cudaMemcpyAsync(hsmall, small, sizeof(hsmall), cudaMemcpyDeviceToHost, st));
        EPK_CUDA(cudaStreamSynchronize(st));
        if (int(hsmall[3])) return fail(EP_ERR_NONFINITE, "ep_compress_cuda: NaN or Inf in the input");
        double amax;
        std::memcpy(&amax, &hsmall[0], 8);

        // Rate control: the same bisection as the host encoder, with the sample counted on the GPU. One
        // launch counts the sample at every midpoint the next kProbeDepth steps can visit (the nodes of a
        // depth-kProbeDepth subtree, heap order: child 2n+1 when the estimate fits, 2n+2 when not). The
        // host then takes the steps one by one, estimating only the nodes on the path taken, so lo and hi
        // follow the exact sequence of the one-probe-per-step bisection.
        const int64_t Rs = std::min<int64_t>(M, (int64_t(opt.sample_coords) + N - 1) / N);
        DevBuf d_pcounts;
        EPK_CUDA(d_pcounts.alloc(sizeof(unsigned long long) * genc::kHistBins * genc::kMaxProbes, st));
        unsigned long long* pcounts = d_pcounts.as<unsigned long long>();
        std::vector<unsigned long long> hcounts(size_t(genc::kHistBins) * genc::kMaxProbes);
        Counts counts(size_t(genc::kHistBins));
        double lo = -12.0, hi = 15.0;
        if (amax > 0.0) hi = std::min(hi, 22.0 - std::log2(amax));
        if (hi < lo) hi = lo;
        const double budget = target_bpp * double(rows) * double(cols);
        for (uint32_t it = 0; it < opt.bisection_iters;) {
            const int depth = int(std::min<uint32_t>(genc::kProbeDepth, opt.bisection_iters - it));
            const int nodes = (1 << depth) - 1;
            double nlo[genc::kMaxProbes], nhi[genc::kMaxProbes], nmid[genc::kMaxProbes];
            genc::Probes pr;
            nlo[0] = lo;
            nhi[0] = hi;
            for (int n = 0; n < nodes; ++n) {
                nmid[n] = 0.5 * (nlo[n] + nhi[n]);
                pr.alpha[n] = float(std::exp2(nmid[n]));
                pr.r[n] = raw_bits_for(pr.alpha[n]);
                if (2 * n + 2 < nodes) {
                    nlo[2 * n + 1] = nmid[n], nhi[2 * n + 1] = nhi[n];  // the estimate fits: lo = mid
                    nlo[2 * n + 2] = nlo[n], nhi[2 * n + 2] = nmid[n];  // it does not: hi = mid
                }
            }
            EPK_CUDA(cudaMemsetAsync(pcounts, 0, sizeof(unsigned long long) * genc::kHistBins * nodes, st));
            genc::sample_counts_kernel<<<dim3(blocks_for(Rs * gpr, 256), unsigned(nodes)), 256, 0, st>>>(
                src, M, gpr, Rs, d_s.as<float>(), pr, pcounts);
            EPK_CUDA(cudaGetLastError());
            EPK_CUDA(cudaMemcpyAsync(hcounts.data(), pcounts, sizeof(unsigned long long) * genc::kHistBins * nodes,
                                     cudaMemcpyDeviceToHost, st));
            EPK_CUDA(cudaStreamSynchronize(st));
            for (int n = 0, step = 0; step < depth; ++step) {
                std::copy(hcounts.begin() + size_t(n) * genc::kHistBins, hcounts.begin() + size_t(n + 1) * genc::kHistBins,
                          counts.begin());
                const double est = estimate_from_counts(counts, version, pr.r[n], Rs, gpr, NG, M, T);
                if (8.0 * est <= budget) { lo = nmid[n]; n = 2 * n + 1; }
                else { hi = nmid[n]; n = 2 * n + 2; }
            }
            it += uint32_t(depth);
        }
        const float alpha = float(std::exp2(lo));

        // Quantise the whole tensor once, then fix r so that every |hi| < 2^15.
        DevBuf d_tq, d_bq;
        EPK_CUDA(d_tq.alloc(size_t(NG) * 8 * 4, st));
        EPK_CUDA(d_bq.alloc(size_t(NG), st));
        EPK_CUDA(cudaMemsetAsync(small + 2, 0, 8, st));
        genc::quantize_kernel<<<blocks_for(NG, 256), 256, 0, st>>>(src, NG, gpr, d_s.as<float>(), alpha, d_tq.as<int32_t>(),
                                                                 d_bq.as<uint8_t>(), small + 2);
        EPK_CUDA(cudaGetLastError());
        unsigned long long tmax_u = 0;
        EPK_CUDA(cudaMemcpyAsync(&tmax_u, small + 2, 8, cudaMemcpyDeviceToHost, st));
        EPK_CUDA(cudaStreamSynchronize(st));
        const int64_t tmax = int64_t(tmax_u);
        int r = raw_bits_for(alpha);
        while (r < 12 && tmax >= (int64_t(1) << (15 + r))) ++r;
        if (tmax >= (int64_t(1) << (15 + r))) return fail(EP_ERR_ARG, "ep_compress_cuda: value range too wide to code");

        // Tables fitted on the whole tensor.
        EPK_CUDA(cudaMemsetAsync(d_counts.p, 0, sizeof(unsigned long long) * genc::kHistBins, st));
        const unsigned cblocks = std::min<unsigned>(blocks_for(NG, 256), 148u * 8u);
        genc::full_counts_kernel<<<cblocks, 256, 0, st>>>(d_tq.as<int32_t>(), d_bq.as<uint8_t>(), NG, r,
                                                         d_counts.as<unsigned long long>());
        EPK_CUDA(cudaGetLastError());
        EPK_CUDA(cudaMemcpyAsync(counts.data(), d_counts.p, sizeof(unsigned long long) * genc::kHistBins,
                                 cudaMemcpyDeviceToHost, st));
        EPK_CUDA(cudaStreamSynchronize(st));
        Tables tab;
        tab.build(prepared_counts(counts, version), version);

        // Tiles: rANS words per tile, then sizes, offsets and the payload.
        DevBuf d_tabs, d_words, d_states, d_nwords, d_esc;
        EPK_CUDA(d_tabs.alloc(2 * sizeof(uint32_t) * genc::kHistBins, st));
        EPK_CUDA(cudaMemcpyAsync(d_tabs.p, tab.f, sizeof(uint32_t) * genc::kHistBins, cudaMemcpyHostToDevice, st));
        EPK_CUDA(cudaMemcpyAsync(d_tabs.as<uint32_t>() + genc::kHistBins, tab.cum, sizeof(uint32_t) * genc::kHistBins,
                                 cudaMemcpyHostToDevice, st));
        EPK_CUDA(d_words.alloc(size_t(T) * 16 * 32 * size_t(G) * 2, st));
        EPK_CUDA(d_states.alloc(size_t(T) * 32 * 4, st));
        EPK_CUDA(d_nwords.alloc(size_t(T) * 4, st));
        EPK_CUDA(d_esc.alloc(size_t(T), st));
        (version == 1 ? genc::encode_tiles_kernel : genc::encode_tiles_v2_kernel)<<<blocks_for(T, 8), 256, 0, st>>>(
            d_tq.as<int32_t>(), d_bq.as<uint8_t>(), NG, T, G, r, d_tabs.as<uint32_t>(),
            d_tabs.as<uint32_t>() + genc::kHistBins, d_words.as<uint16_t>(), d_states.as<uint32_t>(),
            d_nwords.as<uint32_t>(), d_esc.as<uint8_t>());
        EPK_CUDA(cudaGetLastError());
        std::vector<uint32_t> nwords(T);
        std::vector<uint8_t> esc(T);
        EPK_CUDA(cudaMemcpyAsync(nwords.data(), d_nwords.p, size_t(T) * 4, cudaMemcpyDeviceToHost, st));
        EPK_CUDA(cudaMemcpyAsync(esc.data(), d_esc.p, size_t(T), cudaMemcpyDeviceToHost, st));
        EPK_CUDA(cudaStreamSynchronize(st));

        const int64_t per_tile = 32 * int64_t(G);
        std::vector<uint64_t> start(size_t(T) + 1, 0);
        for (uint32_t j = 0; j < T; ++j) {
            const int64_t ng = std::min(per_tile, NG - int64_t(j) * per_tile);
            start[j + 1] = start[j] + pad16(128 + pad4(uint64_t(ng) * uint64_t(r)) + 2 * uint64_t(nwords[j]));
        }
        if (start[T] / 16 >= 0x80000000ull) return fail(EP_ERR_SHAPE, "ep_compress_cuda: payload too large");
        const BlobLayout L = blob_layout(rows, tab, T, start[T]);
        if (L.off_payload > 0xFFFFFFFFull) return fail(EP_ERR_SHAPE, "ep_compress_cuda: metadata too large");

        DevBuf d_start, d_payload;
        EPK_CUDA(d_start.alloc(sizeof(uint64_t) * (size_t(T) + 1), st));
        EPK_CUDA(cudaMemcpyAsync(d_start.p, start.data(), sizeof(uint64_t) * (size_t(T) + 1), cudaMemcpyHostToDevice, st));
        EPK_CUDA(d_payload.alloc(size_t(start[T]), st));
        EPK_CUDA(cudaMemsetAsync(d_payload.p, 0, size_t(start[T]), st));
        genc::assemble_kernel<<<blocks_for(T, 8), 256, 0, st>>>(d_payload.as<uint8_t>(), d_start.as<uint64_t>(),
                                                              d_states.as<uint32_t>(), d_words.as<uint16_t>(),
                                                              d_nwords.as<uint32_t>(), d_tq.as<int32_t>(), NG, T, G, r);
        EPK_CUDA(cudaGetLastError());

        uint8_t* blob = static_cast<uint8_t*>(std::calloc(size_t(L.total), 1));
        if (!blob) return fail(EP_ERR_NOMEM, "ep_compress_cuda: cannot allocate %llu bytes", (unsigned long long)L.total);
        cudaError_t e = cudaMemcpyAsync(blob + L.off_payload, d_payload.p, size_t(start[T]), cudaMemcpyDeviceToHost, st);
        if (e == cudaSuccess) e = cudaStreamSynchronize(st);
        if (e != cudaSuccess) {
            std::free(blob);
            return fail(EP_ERR_CUDA, "ep_compress_cuda: payload copy: %s", cudaGetErrorString(e));
        }
        write_metadata(blob, L, dt, r, rows, cols, alpha, uint32_t(G), T, sbits.data(), tab, start.data(), esc.data());
        finish_crc(blob, L);
        *blob_out = blob;
        *blob_bytes = size_t(L.total);
        if (actual_bpp) *actual_bpp = 8.0 * double(L.total) / (double(rows) * double(cols));
        return EP_OK;
    } catch (const std::bad_alloc&) {
        return fail(EP_ERR_NOMEM, "ep_compress_cuda: out of host memory");
    }
}

// --------------------------------------------------------- variant with static device scratch

namespace epk {
namespace genc {

// Fixed device scratch of ep_compress_cuda_noalloc: 64 MiB per device, zero at module load. With
// lazy module loading it is reserved when this file's kernels are first used.
constexpr size_t kStaticScratchBytes = size_t(64) << 20;
__device__ __align__(256) unsigned char g_static_scratch[kStaticScratchBytes];

}  // namespace genc

namespace {

struct StaticScratch {
    std::mutex mu;  // one call at a time per device: the area has no owner beyond the call
    void* addr = nullptr;
    bool resolved = false;
};
StaticScratch g_static[64];

// Bump carving of the static area, 256-byte aligned. With base == nullptr it only sums the sizes.
struct Carve {
    unsigned char* base;
    size_t used = 0;
    template <class T>
    T* take(size_t bytes) {
        const size_t o = (used + 255) & ~size_t(255);
        used = o + (bytes ? bytes : 1);
        return base ? reinterpret_cast<T*>(base + o) : nullptr;
    }
};

}  // namespace
}  // namespace epk

#define EPK_CUDA_NA(call) EPK_CUDA_IN("ep_compress_cuda_noalloc", call)

extern "C" ep_status ep_compress_cuda_noalloc(const void* dev_data, ep_dtype dt, int64_t rows, int64_t cols,
                                              int64_t row_stride, double target_bpp, const ep_options* opt_in,
                                              void* cuda_stream, uint8_t* blob, size_t blob_capacity,
                                              size_t* blob_bytes, double* actual_bpp) {
    clear_error();
    if (!dev_data || !blob || !blob_bytes) return fail(EP_ERR_ARG, "ep_compress_cuda_noalloc: NULL argument");
    if (!elem_bytes(int(dt))) return fail(EP_ERR_DTYPE, "ep_compress_cuda_noalloc: unknown dtype %d", int(dt));
    if (rows < 1 || cols < 8 || cols % 8 != 0 || rows > 0xFFFFFFFFll || cols > 0xFFFFFFFFll ||
        (rows * cols) / 8 > 0xFFFFFFFFll)
        return fail(EP_ERR_SHAPE, "ep_compress_cuda_noalloc: need a 2-D tensor with rows >= 1 and cols a positive multiple of 8");
    if (row_stride < cols) return fail(EP_ERR_ARG, "ep_compress_cuda_noalloc: row_stride %lld < cols", (long long)row_stride);
    if (!(target_bpp >= 0.001 && target_bpp <= 11.0))
        return fail(EP_ERR_TARGET, "ep_compress_cuda_noalloc: target_bpp must be finite and in [0.001, 11]");
    ep_options opt;
    ep_options_default(&opt);
    if (opt_in) opt = *opt_in;
    if (opt.rounds_per_tile == 0) opt.rounds_per_tile = auto_rounds_per_tile(rows * cols / 8);
    if (opt.format_version == 0) opt.format_version = 2;
    if (opt.rounds_per_tile < 1 || opt.rounds_per_tile > uint32_t(kMaxG) || opt.sample_coords < 1 ||
        opt.bisection_iters > 200 || opt.format_version > 2)
        return fail(EP_ERR_ARG, "ep_compress_cuda_noalloc: bad options");
    const int version = int(opt.format_version);
    cudaPointerAttributes pa;
    if (cudaPointerGetAttributes(&pa, dev_data) != cudaSuccess || pa.type != cudaMemoryTypeDevice) {
        cudaGetLastError();
        return fail(EP_ERR_ARG, "ep_compress_cuda_noalloc: the input is not device memory");
    }
    const int64_t M = rows, N = cols, NG = M * N / 8, gpr = N / 8;
    const int G = int(opt.rounds_per_tile);
    const uint32_t T = uint32_t((NG + 32 * int64_t(G) - 1) / (32 * int64_t(G)));
    const int64_t per_tile = 32 * int64_t(G);

    // Scratch plan (the same buffers as ep_compress_cuda); the payload is sized for r = 12, its largest.
    uint64_t payload_cap = 0;
    for (uint32_t j = 0; j < T; ++j) {
        const int64_t ng = std::min(per_tile, NG - int64_t(j) * per_tile);
        payload_cap += pad16(128 + pad4(uint64_t(ng) * 12) + 2 * 16 * uint64_t(ng));
    }
    auto plan = [&](Carve& c, uint16_t** sb, float** s, unsigned long long** small, unsigned long long** counts,
                    unsigned long long** pcounts, int32_t** tq, uint8_t** bq, uint32_t** tabs, uint16_t** words,
                    uint32_t** states, uint32_t** nw, uint8_t** esc, uint64_t** start, uint8_t** payload) {
        *sb = c.take<uint16_t>(size_t(M) * 2);
        *s = c.take<float>(size_t(M) * 4);
        *small = c.take<unsigned long long>(64);
        *counts = c.take<unsigned long long>(sizeof(unsigned long long) * genc::kHistBins);
        *pcounts = c.take<unsigned long long>(sizeof(unsigned long long) * genc::kHistBins * genc::kMaxProbes);
        *tq = c.take<int32_t>(size_t(NG) * 32);
        *bq = c.take<uint8_t>(size_t(NG));
        *tabs = c.take<uint32_t>(2 * sizeof(uint32_t) * genc::kHistBins);
        *words = c.take<uint16_t>(size_t(T) * 16 * size_t(per_tile) * 2);
        *states = c.take<uint32_t>(size_t(T) * 128);
        *nw = c.take<uint32_t>(size_t(T) * 4);
        *esc = c.take<uint8_t>(size_t(T));
        *start = c.take<uint64_t>(sizeof(uint64_t) * (size_t(T) + 1));
        *payload = c.take<uint8_t>(size_t(payload_cap));
    };
    uint16_t* d_sbits; float* d_s; unsigned long long *small, *d_counts, *pcounts; int32_t* d_tq; uint8_t* d_bq;
    uint32_t* d_tabs; uint16_t* d_words; uint32_t *d_states, *d_nwords; uint8_t* d_esc; uint64_t* d_start;
    uint8_t* d_payload;
    {
        Carve dry{nullptr};
        plan(dry, &d_sbits, &d_s, &small, &d_counts, &pcounts, &d_tq, &d_bq, &d_tabs, &d_words, &d_states, &d_nwords,
             &d_esc, &d_start, &d_payload);
        if (dry.used > genc::kStaticScratchBytes)
            return fail(EP_ERR_ARG, "ep_compress_cuda_noalloc: this tensor needs %llu bytes of device scratch; the static area holds %llu",
                        (unsigned long long)dry.used, (unsigned long long)genc::kStaticScratchBytes);
    }

    int device = 0;
    EPK_CUDA_NA(cudaGetDevice(&device));
    if (device < 0 || device >= 64) return fail(EP_ERR_CUDA, "ep_compress_cuda_noalloc: device %d out of range", device);
    // The static area used is the current device's, so the input must live there too.
    if (pa.device != device)
        return fail(EP_ERR_ARG, "ep_compress_cuda_noalloc: the input is on device %d, the current device is %d",
                    pa.device, device);
    StaticScratch& ss = g_static[device];
    std::lock_guard<std::mutex> lock(ss.mu);
    if (!ss.resolved) {  // once per device, with that device current
        EPK_CUDA_NA(cudaGetSymbolAddress(&ss.addr, genc::g_static_scratch));
        ss.resolved = true;
    }
    cudaStream_t st = static_cast<cudaStream_t>(cuda_stream);
    // Every exit from here on, error paths included, first drains the stream: no kernel or copy of this
    // call may still use the static area once the lock is released. Declared after the lock, so it runs
    // before the unlock.
    struct DrainOnExit {
        cudaStream_t s;
        ~DrainOnExit() {
            cudaStreamSynchronize(s);
            cudaGetLastError();
        }
    } drain{st};
    Carve carve{static_cast<unsigned char*>(ss.addr)};
    plan(carve, &d_sbits, &d_s, &small, &d_counts, &pcounts, &d_tq, &d_bq, &d_tabs, &d_words, &d_states, &d_nwords,
         &d_esc, &d_start, &d_payload);

    const genc::Src src{static_cast<const uint8_t*>(dev_data), int(dt), N, row_stride};
    try {
        EPK_CUDA_NA(cudaMemsetAsync(small, 0, 64, st));
        EPK_CUDA_NA(genc::launch_row_scales(src, M, d_sbits, d_s, small, reinterpret_cast<int*>(small + 3), st));
        std::vector<uint16_t> sbits(static_cast<size_t>(M));
        unsigned long long hsmall[4];
        EPK_CUDA_NA(cudaMemcpyAsync(sbits.data(), d_sbits, size_t(M) * 2, cudaMemcpyDeviceToHost, st));
        EPK_CUDA_NA(cudaMemcpyAsync(hsmall, small, sizeof(hsmall), cudaMemcpyDeviceToHost, st));
        EPK_CUDA_NA(cudaStreamSynchronize(st));
        if (int(hsmall[3])) return fail(EP_ERR_NONFINITE, "ep_compress_cuda_noalloc: NaN or Inf in the input");
        double amax;
        std::memcpy(&amax, &hsmall[0], 8);

        // Rate control, four bisection steps per launch, exactly as ep_compress_cuda.
        const int64_t Rs = std::min<int64_t>(M, (int64_t(opt.sample_coords) + N - 1) / N);
        std::vector<unsigned long long> hcounts(size_t(genc::kHistBins) * genc::kMaxProbes);
        Counts counts(size_t(genc::kHistBins));
        double lo = -12.0, hi = 15.0;
        if (amax > 0.0) hi = std::min(hi, 22.0 - std::log2(amax));
        if (hi < lo) hi = lo;
        const double budget = target_bpp * double(rows) * double(cols);
        for (uint32_t it = 0; it < opt.bisection_iters;) {
            const int depth = int(std::min<uint32_t>(genc::kProbeDepth, opt.bisection_iters - it));
            const int nodes = (1 << depth) - 1;
            double nlo[genc::kMaxProbes], nhi[genc::kMaxProbes], nmid[genc::kMaxProbes];
            genc::Probes pr;
            nlo[0] = lo;
            nhi[0] = hi;
            for (int n = 0; n < nodes; ++n) {
                nmid[n] = 0.5 * (nlo[n] + nhi[n]);
                pr.alpha[n] = float(std::exp2(nmid[n]));
                pr.r[n] = raw_bits_for(pr.alpha[n]);
                if (2 * n + 2 < nodes) {
                    nlo[2 * n + 1] = nmid[n], nhi[2 * n + 1] = nhi[n];
                    nlo[2 * n + 2] = nlo[n], nhi[2 * n + 2] = nmid[n];
                }
            }
            EPK_CUDA_NA(cudaMemsetAsync(pcounts, 0, sizeof(unsigned long long) * genc::kHistBins * nodes, st));
            genc::sample_counts_kernel<<<dim3(blocks_for(Rs * gpr, 256), unsigned(nodes)), 256, 0, st>>>(
                src, M, gpr, Rs, d_s, pr, pcounts);
            EPK_CUDA_NA(cudaGetLastError());
            EPK_CUDA_NA(cudaMemcpyAsync(hcounts.data(), pcounts, sizeof(unsigned long long) * genc::kHistBins * nodes,
                                     cudaMemcpyDeviceToHost, st));
            EPK_CUDA_NA(cudaStreamSynchronize(st));
            for (int n = 0, step = 0; step < depth; ++step) {
                std::copy(hcounts.begin() + size_t(n) * genc::kHistBins, hcounts.begin() + size_t(n + 1) * genc::kHistBins,
                          counts.begin());
                const double est = estimate_from_counts(counts, version, pr.r[n], Rs, gpr, NG, M, T);
                if (8.0 * est <= budget) { lo = nmid[n]; n = 2 * n + 1; }
                else { hi = nmid[n]; n = 2 * n + 2; }
            }
            it += uint32_t(depth);
        }
        const float alpha = float(std::exp2(lo));

        // Quantisation, raw bits, tables.
        EPK_CUDA_NA(cudaMemsetAsync(small + 2, 0, 8, st));
        genc::quantize_kernel<<<blocks_for(NG, 256), 256, 0, st>>>(src, NG, gpr, d_s, alpha, d_tq, d_bq, small + 2);
        EPK_CUDA_NA(cudaGetLastError());
        unsigned long long tmax_u = 0;
        EPK_CUDA_NA(cudaMemcpyAsync(&tmax_u, small + 2, 8, cudaMemcpyDeviceToHost, st));
        EPK_CUDA_NA(cudaStreamSynchronize(st));
        const int64_t tmax = int64_t(tmax_u);
        int r = raw_bits_for(alpha);
        while (r < 12 && tmax >= (int64_t(1) << (15 + r))) ++r;
        if (tmax >= (int64_t(1) << (15 + r))) return fail(EP_ERR_ARG, "ep_compress_cuda_noalloc: value range too wide to code");
        EPK_CUDA_NA(cudaMemsetAsync(d_counts, 0, sizeof(unsigned long long) * genc::kHistBins, st));
        genc::full_counts_kernel<<<std::min<unsigned>(blocks_for(NG, 256), 148u * 8u), 256, 0, st>>>(d_tq, d_bq, NG, r,
                                                                                                   d_counts);
        EPK_CUDA_NA(cudaGetLastError());
        EPK_CUDA_NA(cudaMemcpyAsync(counts.data(), d_counts, sizeof(unsigned long long) * genc::kHistBins,
                                 cudaMemcpyDeviceToHost, st));
        EPK_CUDA_NA(cudaStreamSynchronize(st));
        Tables tab;
        tab.build(prepared_counts(counts, version), version);

        // Tiles.
        EPK_CUDA_NA(cudaMemcpyAsync(d_tabs, tab.f, sizeof(uint32_t) * genc::kHistBins, cudaMemcpyHostToDevice, st));
        EPK_CUDA_NA(cudaMemcpyAsync(d_tabs + genc::kHistBins, tab.cum, sizeof(uint32_t) * genc::kHistBins,
                                 cudaMemcpyHostToDevice, st));
        (version == 1 ? genc::encode_tiles_kernel : genc::encode_tiles_v2_kernel)<<<blocks_for(T, 8), 256, 0, st>>>(d_tq, d_bq, NG, T, G, r, d_tabs,
                                                                   d_tabs + genc::kHistBins, d_words, d_states,
                                                                   d_nwords, d_esc);
        EPK_CUDA_NA(cudaGetLastError());
        std::vector<uint32_t> nwords(T);
        std::vector<uint8_t> esc(T);
        EPK_CUDA_NA(cudaMemcpyAsync(nwords.data(), d_nwords, size_t(T) * 4, cudaMemcpyDeviceToHost, st));
        EPK_CUDA_NA(cudaMemcpyAsync(esc.data(), d_esc, size_t(T), cudaMemcpyDeviceToHost, st));
        EPK_CUDA_NA(cudaStreamSynchronize(st));
        std::vector<uint64_t> start(size_t(T) + 1, 0);
        for (uint32_t j = 0; j < T; ++j) {
            const int64_t ng = std::min(per_tile, NG - int64_t(j) * per_tile);
            start[j + 1] = start[j] + pad16(128 + pad4(uint64_t(ng) * uint64_t(r)) + 2 * uint64_t(nwords[j]));
        }
        if (start[T] / 16 >= 0x80000000ull) return fail(EP_ERR_SHAPE, "ep_compress_cuda_noalloc: payload too large");
        const BlobLayout L = blob_layout(rows, tab, T, start[T]);
        if (L.total > blob_capacity)
            return fail(EP_ERR_BUFFER, "ep_compress_cuda_noalloc: the blob takes %llu bytes, the buffer holds %llu",
                        (unsigned long long)L.total, (unsigned long long)blob_capacity);

        // Payload in the static area (zeroed first: padding bytes stay zero), then into the caller's buffer.
        EPK_CUDA_NA(cudaMemcpyAsync(d_start, start.data(), sizeof(uint64_t) * (size_t(T) + 1), cudaMemcpyHostToDevice, st));
        EPK_CUDA_NA(cudaMemsetAsync(d_payload, 0, size_t(start[T]), st));
        genc::assemble_kernel<<<blocks_for(T, 8), 256, 0, st>>>(d_payload, d_start, d_states, d_words, d_nwords, d_tq,
                                                              NG, T, G, r);
        EPK_CUDA_NA(cudaGetLastError());
        std::memset(blob, 0, size_t(L.off_payload));
        EPK_CUDA_NA(cudaMemcpyAsync(blob + L.off_payload, d_payload, size_t(start[T]), cudaMemcpyDeviceToHost, st));
        EPK_CUDA_NA(cudaStreamSynchronize(st));
        write_metadata(blob, L, dt, r, rows, cols, alpha, uint32_t(G), T, sbits.data(), tab, start.data(), esc.data());
        finish_crc(blob, L);
        *blob_bytes = size_t(L.total);
        if (actual_bpp) *actual_bpp = 8.0 * double(L.total) / (double(rows) * double(cols));
        return EP_OK;
    } catch (const std::bad_alloc&) {
        return fail(EP_ERR_NOMEM, "ep_compress_cuda_noalloc: out of host memory");
    }
}
