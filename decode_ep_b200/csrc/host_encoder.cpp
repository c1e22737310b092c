// Host encoder of the EPK1 blob: ep_compress. This runs once per tensor and is not the hot path.
//
// The steps follow the EntroPack pages (arXiv 2609.34185):
//   - Each row is normalised by its own scale s_row (paper page abstract; modelscope summary).
//   - Each 8-wide group is quantised to the nearest E8 point at one global resolution alpha.
//   - Alpha comes from bisection on log2(alpha) against a storage estimate taken on a sample of
//     rows, so the full stream is never re-encoded (paper page abstract; techmoon article).
//   - The coordinates are rANS-coded under 9 conditional tables (8-bit in format version 2, 12-bit in
//     version 1), in independent tiles of 32 interleaved lanes (abstract; modelscope summary).
// All floating point is IEEE double/binary32, round-to-nearest, with no FMA contraction. The
// build passes -ffp-contract=off, so every estimate and every quantisation decision is a fixed
// function of the input, whatever the thread count.
#include <algorithm>
#include <atomic>
#include <cmath>
#include <cstdlib>
#include <functional>
#include <thread>
#include <vector>

#include <cuda_runtime.h>

#include "capi_internal.h"
#include "encoder_common.h"
#include "lattice_code.h"
#include "entropack.h"
#include "epk_format.h"

namespace epk {
namespace {

using namespace enc;

// ------------------------------------------------------------------------------- threads

void parallel_for(int64_t n, int threads, const std::function<void(int64_t, int64_t, int)>& fn) {
    if (n <= 0) return;
    int nt = int(std::min<int64_t>(threads, n));
    if (nt <= 1) { fn(0, n, 0); return; }
    int64_t chunk = std::max<int64_t>(1, n / (int64_t(nt) * 16));
    std::atomic<int64_t> next{0};
    std::vector<std::thread> pool;
    pool.reserve(nt);
    for (int t = 0; t < nt; ++t)
        pool.emplace_back([&, t] {
            for (;;) {
                int64_t b = next.fetch_add(chunk);
                if (b >= n) break;
                fn(b, std::min(n, b + chunk), t);
            }
        });
    for (auto& th : pool) th.join();
}

// ---------------------------------------------------------------------- number formats

float half_bits_to_float(uint16_t h) {
    int e = (h >> 10) & 31, m = h & 1023;
    float mag;
    if (e == 31) mag = m ? NAN : INFINITY;
    else if (e == 0) mag = std::ldexp(float(m), -24);
    else mag = std::ldexp(float(1024 + m), e - 25);
    return (h & 0x8000) ? -mag : mag;
}

float e4m3_bits_to_float(uint8_t c) {
    int e = (c >> 3) & 15, m = c & 7;
    float mag;
    if (e == 15 && m == 7) mag = NAN;
    else if (e == 0) mag = std::ldexp(float(m), -9);
    else mag = std::ldexp(float(8 + m), e - 10);
    return (c & 0x80) ? -mag : mag;
}

// Reads rows of a strided row-major container tensor as binary32.
struct Source {
    const uint8_t* base;
    int dtype;
    int64_t N, stride;  // elements
    float e4m3[256];

    Source(const void* p, int dt, int64_t n, int64_t st) : base(static_cast<const uint8_t*>(p)), dtype(dt), N(n), stride(st) {
        for (int i = 0; i < 256; ++i) e4m3[i] = e4m3_bits_to_float(uint8_t(i));
    }
    void row(int64_t i, float* out) const {
        const uint8_t* r = base + i * stride * elem_bytes(dtype);
        switch (dtype) {
            case EP_BF16: { const uint16_t* q = reinterpret_cast<const uint16_t*>(r); for (int64_t j = 0; j < N; ++j) out[j] = bf16_bits_to_float(q[j]); break; }
            case EP_FP16: { const uint16_t* q = reinterpret_cast<const uint16_t*>(r); for (int64_t j = 0; j < N; ++j) out[j] = half_bits_to_float(q[j]); break; }
            case EP_FP32: std::memcpy(out, r, sizeof(float) * size_t(N)); break;
            case EP_FP8_E4M3: for (int64_t j = 0; j < N; ++j) out[j] = e4m3[r[j]]; break;
            case EP_INT8: { const int8_t* q = reinterpret_cast<const int8_t*>(r); for (int64_t j = 0; j < N; ++j) out[j] = float(q[j]); break; }
        }
    }
};

// ------------------------------------------------------------------------------ encoder

struct Encoder {
    const Source& src;
    int64_t M, N, NG, gpr;
    int G, threads;
    uint32_t T;
    std::vector<uint16_t> sbits;
    std::vector<float> s;

    Encoder(const Source& sc, int64_t m, int64_t n, int g, int th)
        : src(sc), M(m), N(n), NG(m * n / 8), gpr(n / 8), G(g), threads(th) {
        T = uint32_t((NG + 32 * int64_t(G) - 1) / (32 * int64_t(G)));
    }

    // Row scales (root mean square in double, index order → binary32 → BF16) and max |w|/s.
    // Returns false on a non-finite input.
    bool scales(double& amax) {
        sbits.assign(size_t(M), 0);
        s.assign(size_t(M), 0.f);
        std::vector<double> tmax(size_t(std::max(threads, 1)), 0.0);
        std::atomic<bool> finite{true};
        parallel_for(M, threads, [&](int64_t b, int64_t e, int t) {
            std::vector<float> w(static_cast<size_t>(N));
            for (int64_t i = b; i < e; ++i) {
                src.row(i, w.data());
                double acc = 0.0;
                for (int64_t j = 0; j < N; ++j) {
                    if (!std::isfinite(w[j])) { finite = false; return; }
                    acc += double(w[j]) * double(w[j]);
                }
                float rms = float(std::sqrt(acc / double(N)));
                sbits[size_t(i)] = float_to_bf16_rne(rms);
                s[size_t(i)] = bf16_bits_to_float(sbits[size_t(i)]);
                if (s[size_t(i)] != 0.f)
                    for (int64_t j = 0; j < N; ++j) tmax[size_t(t)] = std::max(tmax[size_t(t)], std::fabs(double(w[j])) / double(s[size_t(i)]));
            }
        });
        amax = *std::max_element(tmax.begin(), tmax.end());
        return finite;
    }

    // Quantises one row (already converted) at alpha: coded integers t and coset bits per group.
    void quantize_row(const float* w, int64_t i, float alpha, int32_t* t, uint8_t* b) const {
        double sd = double(s[size_t(i)]), ad = double(alpha);
        double x[8];
        for (int64_t q = 0; q < gpr; ++q) {
            for (int k = 0; k < 8; ++k) x[k] = (sd == 0.0) ? 0.0 : (ad * double(w[q * 8 + k])) / sd;
            b[q] = uint8_t(e8_code(x, t + 8 * q));
        }
    }

    // Storage estimate in bytes from the row sample (same definition the format fixes).
    double estimate(float alpha, uint32_t sample_coords, int version) const {
        int64_t Rs = std::min<int64_t>(M, (int64_t(sample_coords) + N - 1) / N);
        int r = raw_bits_for(alpha);
        int nt = std::max(1, threads);
        std::vector<Counts> counts(size_t(nt), Counts(size_t(kNumCtx) * 128, 0));
        parallel_for(Rs, threads, [&](int64_t b, int64_t e, int th) {
            std::vector<float> w(static_cast<size_t>(N));
            std::vector<int32_t> t(static_cast<size_t>(N));
            std::vector<uint8_t> cb(static_cast<size_t>(gpr));
            Counts& c = counts[size_t(th)];
            for (int64_t k = b; k < e; ++k) {
                int64_t row = (k * M) / Rs;
                src.row(row, w.data());
                quantize_row(w.data(), row, alpha, t.data(), cb.data());
                for (int64_t q = 0; q < gpr; ++q) {
                    uint8_t ctx[8], sym[8];
                    int32_t hi[8];
                    group_syms(cb[size_t(q)], &t[size_t(q * 8)], r, ctx, sym, hi);
                    for (int i = 0; i < 8; ++i) c[size_t(ctx[i]) * 128 + sym[i]]++;
                }
            }
        });
        Counts total(size_t(kNumCtx) * 128, 0);
        for (int th = 0; th < nt; ++th)
            for (size_t k = 0; k < total.size(); ++k) total[k] += counts[size_t(th)][k];
        return estimate_from_counts(total, version, r, Rs, gpr, NG, M, T);
    }
};

// One tile's bytes: states, raw section, reversed word stream, zero padding.
struct TileBytes {
    std::vector<uint8_t> bytes;
    bool has_esc = false;
};

void write_tile(const std::vector<int32_t>& tq, int64_t g0, int64_t ng, int r, const uint32_t* x,
                const std::vector<uint16_t>& words, bool has_esc, TileBytes& out);

// Version 1 tile: the decode order of the format document, run backwards.
void encode_tile(const std::vector<int32_t>& tq, const std::vector<uint8_t>& bq, int64_t g0, int64_t ng, int r,
                 const Tables& tab, TileBytes& out) {
    uint32_t x[kLanes];
    for (auto& v : x) v = kRansL;
    std::vector<uint16_t> words;
    words.reserve(size_t(ng) * 4);
    int64_t R = (ng + 31) / 32;
    bool has_esc = false;
    uint8_t ctx[kLanes][8], sym[kLanes][8];
    int32_t hi[kLanes][8];
    for (int64_t k = R - 1; k >= 0; --k) {
        int nl = int(std::min<int64_t>(32, ng - 32 * k));
        for (int L = 0; L < nl; ++L) {
            int64_t g = g0 + 32 * k + L;
            group_syms(bq[size_t(g)], &tq[size_t(g * 8)], r, ctx[L], sym[L], hi[L]);
        }
        for (int i = 7; i >= 0; --i) {
            for (int L = nl - 1; L >= 0; --L)
                if (idx_of(hi[L][i]) == kEscIdx) {
                    words.push_back(uint16_t(int16_t(hi[L][i])));
                    has_esc = true;
                }
            for (int L = nl - 1; L >= 0; --L) {
                uint32_t f = tab.f[ctx[L][i]][sym[L][i]], c = tab.cum[ctx[L][i]][sym[L][i]];
                uint32_t xv = x[L];
                if (uint64_t(xv) >= (uint64_t(f) << 20)) { words.push_back(uint16_t(xv)); xv >>= 16; }
                x[L] = (xv / f) * kProbScale + (xv % f) + c;
            }
        }
    }
    write_tile(tq, g0, ng, r, x, words, has_esc, out);
}

// One tile's bytes from its final states and pushed words: states, the raw section (8 fields of r bits per
// group, LSB-first), the words in reverse push order, zero padding to 16 bytes.
void write_tile(const std::vector<int32_t>& tq, int64_t g0, int64_t ng, int r, const uint32_t* x,
                const std::vector<uint16_t>& words, bool has_esc, TileBytes& out) {
    uint64_t raw = pad4(uint64_t(ng) * uint64_t(r));
    uint64_t size = pad16(128 + raw + 2 * uint64_t(words.size()));
    out.bytes.assign(size_t(size), 0);
    uint8_t* p = out.bytes.data();
    for (int L = 0; L < kLanes; ++L) wr32(p + 4 * L, x[L]);
    if (r > 0) {
        uint8_t* rp = p + 128;
        const uint32_t mask = (1u << r) - 1u;
        for (int64_t q = 0; q < ng; ++q) {
            // 8 fields of r bits, LSB-first, starting at bit 8rq (byte rq)
            uint64_t acc_lo = 0, acc_hi = 0;  // up to 96 bits
            for (int i = 0; i < 8; ++i) {
                uint32_t lo = uint32_t(tq[size_t((g0 + q) * 8 + i)]) & mask;
                int pos = i * r;
                if (pos < 64) {
                    acc_lo |= uint64_t(lo) << pos;
                    if (pos + r > 64) acc_hi |= uint64_t(lo) >> (64 - pos);
                } else {
                    acc_hi |= uint64_t(lo) << (pos - 64);
                }
            }
            uint8_t* dst = rp + q * r;
            for (int byte = 0; byte < r; ++byte)
                dst[byte] = byte < 8 ? uint8_t(acc_lo >> (8 * byte)) : uint8_t(acc_hi >> (8 * (byte - 8)));
        }
    }
    uint8_t* sp = p + 128 + raw;
    size_t n = words.size();
    for (size_t i = 0; i < n; ++i) wr16(sp + 2 * i, words[n - 1 - i]);
    out.has_esc = has_esc;
}

// Version 2 tile: pairs of positions (2p, 2p + 1) share one renormalisation, and a round's escape words
// follow its last pair, positions ascending, lanes ascending. Run backwards: the round's escape words
// (positions and lanes descending), then each pair from the last: if x >= f1 f2 2^16 the lane pushes
// x & 0xFFFF and sets x >>= 16, then x <- C(s2, x) and x <- C(s1, x) in base 256.
void encode_tile_v2(const std::vector<int32_t>& tq, const std::vector<uint8_t>& bq, int64_t g0, int64_t ng, int r,
                    const Tables& tab, TileBytes& out) {
    uint32_t x[kLanes];
    for (auto& v : x) v = kRansL;
    std::vector<uint16_t> words;
    words.reserve(size_t(ng) * 4);
    int64_t R = (ng + 31) / 32;
    bool has_esc = false;
    uint8_t ctx[kLanes][8], sym[kLanes][8];
    int32_t hi[kLanes][8];
    for (int64_t k = R - 1; k >= 0; --k) {
        int nl = int(std::min<int64_t>(32, ng - 32 * k));
        for (int L = 0; L < nl; ++L) {
            int64_t g = g0 + 32 * k + L;
            group_syms(bq[size_t(g)], &tq[size_t(g * 8)], r, ctx[L], sym[L], hi[L]);
            for (int i = 0; i < 8; ++i) sym[L][i] = uint8_t(tab.coded(ctx[L][i], sym[L][i]));
        }
        for (int i = 7; i >= 0; --i)
            for (int L = nl - 1; L >= 0; --L)
                if ((sym[L][i] & 63) == kEscIdx) {
                    words.push_back(uint16_t(int16_t(hi[L][i])));
                    has_esc = true;
                }
        for (int pr = 3; pr >= 0; --pr)
            for (int L = nl - 1; L >= 0; --L) {
                const int i1 = 2 * pr, i2 = 2 * pr + 1;
                const uint32_t f1 = tab.f[ctx[L][i1]][sym[L][i1]], c1 = tab.cum[ctx[L][i1]][sym[L][i1]];
                const uint32_t f2 = tab.f[ctx[L][i2]][sym[L][i2]], c2 = tab.cum[ctx[L][i2]][sym[L][i2]];
                uint32_t xv = x[L];
                if (uint64_t(xv) >= (uint64_t(f1 * f2) << 16)) { words.push_back(uint16_t(xv)); xv >>= 16; }
                xv = (xv / f2) * kProbScaleV2 + (xv % f2) + c2;
                x[L] = (xv / f1) * kProbScaleV2 + (xv % f1) + c1;
            }
    }
    write_tile(tq, g0, ng, r, x, words, has_esc, out);
}

}  // namespace
}  // namespace epk

using namespace epk;

extern "C" void ep_options_default(ep_options* opt) {
    if (!opt) return;
    opt->rounds_per_tile = 0;  // automatic
    opt->sample_coords = 1u << 18;
    opt->bisection_iters = 40;
    opt->threads = 0;
    opt->format_version = 2;
}

extern "C" ep_status ep_compress(const void* data, int is_device, ep_dtype dt, int64_t rows, int64_t cols,
                                 int64_t row_stride, double target_bpp, const ep_options* opt_in,
                                 uint8_t** blob_out, size_t* blob_bytes, double* actual_bpp) {
    clear_error();
    if (!data || !blob_out || !blob_bytes) return fail(EP_ERR_ARG, "ep_compress: NULL argument");
    if (!elem_bytes(int(dt))) return fail(EP_ERR_DTYPE, "ep_compress: unknown dtype %d", int(dt));
    if (rows < 1 || cols < 8 || cols % 8 != 0 || rows > 0xFFFFFFFFll || cols > 0xFFFFFFFFll ||
        (rows * cols) / 8 > 0xFFFFFFFFll)
        return fail(EP_ERR_SHAPE, "ep_compress: need a 2-D tensor with rows >= 1 and cols a positive multiple of 8 (got %lld x %lld)",
                    (long long)rows, (long long)cols);
    if (row_stride < cols) return fail(EP_ERR_ARG, "ep_compress: row_stride %lld < cols", (long long)row_stride);
    if (!(target_bpp >= 0.001 && target_bpp <= 11.0))
        return fail(EP_ERR_TARGET, "ep_compress: target_bpp must be finite and in [0.001, 11]");
    ep_options opt;
    ep_options_default(&opt);
    if (opt_in) opt = *opt_in;
    if (opt.rounds_per_tile == 0) opt.rounds_per_tile = auto_rounds_per_tile(rows * cols / 8);
    if (opt.format_version == 0) opt.format_version = 2;
    if (opt.rounds_per_tile < 1 || opt.rounds_per_tile > uint32_t(kMaxG) || opt.sample_coords < 1 ||
        opt.bisection_iters > 200 || opt.format_version > 2)
        return fail(EP_ERR_ARG, "ep_compress: bad options");
    const int version = int(opt.format_version);
    int threads = opt.threads > 0 ? opt.threads : int(std::max(1u, std::thread::hardware_concurrency()));

    // Device input: one copy to the host, rows packed.
    std::vector<uint8_t> staged;
    const void* host = data;
    int64_t stride = row_stride;
    int es = elem_bytes(int(dt));
    if (is_device) {
        staged.resize(size_t(rows * cols * es));
        cudaError_t e = cudaMemcpy2D(staged.data(), size_t(cols * es), data, size_t(row_stride * es), size_t(cols * es),
                                     size_t(rows), cudaMemcpyDeviceToHost);
        if (e != cudaSuccess) return fail(EP_ERR_CUDA, "ep_compress: cudaMemcpy2D: %s", cudaGetErrorString(e));
        host = staged.data();
        stride = cols;
    }

    try {
        Source src(host, int(dt), cols, stride);
        Encoder enc(src, rows, cols, int(opt.rounds_per_tile), threads);
        double amax = 0.0;
        if (!enc.scales(amax)) return fail(EP_ERR_NONFINITE, "ep_compress: NaN or Inf in the input");

        // Rate control: bisection on log2(alpha); the cap keeps |x| <= 2^22 so 2v is exact in binary32.
        double lo = -12.0, hi = 15.0;
        if (amax > 0.0) hi = std::min(hi, 22.0 - std::log2(amax));
        if (hi < lo) hi = lo;
        double budget = target_bpp * double(rows) * double(cols);
        for (uint32_t it = 0; it < opt.bisection_iters; ++it) {
            double mid = 0.5 * (lo + hi);
            float a = float(std::exp2(mid));
            if (8.0 * enc.estimate(a, opt.sample_coords, version) <= budget) lo = mid; else hi = mid;
        }
        float alpha = float(std::exp2(lo));

        // Quantise the whole tensor once.
        int64_t NG = enc.NG, gpr = enc.gpr;
        std::vector<int32_t> tq(size_t(NG) * 8);
        std::vector<uint8_t> bq(static_cast<size_t>(NG));
        std::vector<int64_t> tabs(size_t(std::max(threads, 1)), 0);
        parallel_for(rows, threads, [&](int64_t b, int64_t e, int th) {
            std::vector<float> w(static_cast<size_t>(cols));
            for (int64_t i = b; i < e; ++i) {
                src.row(i, w.data());
                enc.quantize_row(w.data(), i, alpha, &tq[size_t(i * gpr * 8)], &bq[size_t(i * gpr)]);
                for (int64_t j = i * gpr * 8; j < (i + 1) * gpr * 8; ++j) {
                    int64_t v = tq[size_t(j)], a = v >= 0 ? v : -v - 1;
                    tabs[size_t(th)] = std::max(tabs[size_t(th)], a);
                }
            }
        });
        int64_t tmax = *std::max_element(tabs.begin(), tabs.end());
        int r = raw_bits_for(alpha);
        while (r < 12 && tmax >= (int64_t(1) << (15 + r))) ++r;
        if (tmax >= (int64_t(1) << (15 + r))) return fail(EP_ERR_ARG, "ep_compress: value range too wide to code");

        // Tables fitted on the whole tensor.
        int nt = std::max(threads, 1);
        std::vector<Counts> counts(size_t(nt), Counts(size_t(kNumCtx) * 128, 0));
        parallel_for(NG, threads, [&](int64_t b, int64_t e, int th) {
            Counts& c = counts[size_t(th)];
            uint8_t ctx[8], sym[8];
            int32_t hv[8];
            for (int64_t g = b; g < e; ++g) {
                group_syms(bq[size_t(g)], &tq[size_t(g * 8)], r, ctx, sym, hv);
                for (int i = 0; i < 8; ++i) c[size_t(ctx[i]) * 128 + sym[i]]++;
            }
        });
        Counts total(size_t(kNumCtx) * 128, 0);
        for (auto& c : counts) for (size_t k = 0; k < total.size(); ++k) total[k] += c[k];
        Tables tab;
        tab.build(prepared_counts(total, version), version);

        // Tiles, in parallel.
        uint32_t T = enc.T;
        int64_t per_tile = 32 * int64_t(opt.rounds_per_tile);
        std::vector<TileBytes> tiles(T);
        parallel_for(T, threads, [&](int64_t b, int64_t e, int) {
            for (int64_t j = b; j < e; ++j) {
                int64_t g0 = j * per_tile, ng = std::min(per_tile, NG - g0);
                if (version == 1) encode_tile(tq, bq, g0, ng, r, tab, tiles[size_t(j)]);
                else encode_tile_v2(tq, bq, g0, ng, r, tab, tiles[size_t(j)]);
            }
        });
        std::vector<uint64_t> start(size_t(T) + 1, 0);
        for (uint32_t j = 0; j < T; ++j) start[j + 1] = start[j] + tiles[j].bytes.size();
        if (start[T] / 16 >= 0x80000000ull) return fail(EP_ERR_SHAPE, "ep_compress: payload too large");

        const BlobLayout L = blob_layout(rows, tab, T, start[T]);
        if (L.off_payload > 0xFFFFFFFFull) return fail(EP_ERR_SHAPE, "ep_compress: metadata too large");
        uint8_t* blob = static_cast<uint8_t*>(std::calloc(size_t(L.total), 1));
        if (!blob) return fail(EP_ERR_NOMEM, "ep_compress: cannot allocate %llu bytes", (unsigned long long)L.total);
        std::vector<uint8_t> esc(T);
        for (uint32_t j = 0; j < T; ++j) esc[j] = tiles[j].has_esc;
        write_metadata(blob, L, dt, r, rows, cols, alpha, opt.rounds_per_tile, T, enc.sbits.data(), tab, start.data(),
                       esc.data());
        parallel_for(T, threads, [&](int64_t b, int64_t e, int) {
            for (int64_t j = b; j < e; ++j)
                std::memcpy(blob + L.off_payload + start[size_t(j)], tiles[size_t(j)].bytes.data(), tiles[size_t(j)].bytes.size());
        });
        finish_crc(blob, L);
        const uint64_t total_bytes = L.total;

        *blob_out = blob;
        *blob_bytes = size_t(total_bytes);
        if (actual_bpp) *actual_bpp = 8.0 * double(total_bytes) / (double(rows) * double(cols));
        return EP_OK;
    } catch (const std::bad_alloc&) {
        return fail(EP_ERR_NOMEM, "ep_compress: out of host memory");
    }
}

extern "C" void ep_blob_free(uint8_t* blob) { std::free(blob); }
