// Per-layer target bitrates for a set of tensors that share one storage budget (EntroPack README,
// "Pre-quantised models": the "extreme mixed bitrate" packs assign each layer a bitrate by its
// sensitivity and reach 2.3 to 3.0 bits per parameter on average).
//
// The pages give the idea, not the rule. The rule used here is the classic high-rate bit allocation:
// a layer coded at a data rate of R bits per parameter has a squared weight error proportional to
// 2^(-2R) (each extra bit halves the quantiser step). With a per-layer weight w_i on that error
// (sensitivity times mean square weight), minimising sum_i n_i w_i 2^(-2 (b_i - m_i)) under
// sum_i n_i b_i = budget and box bounds on b_i gives, by the KKT conditions, one water level theta
// with b_i = clamp(m_i + log2(w_i)/2 + theta, lo_i, hi_i). Here b_i is the layer's whole-blob bitrate
// (the quantity the encoders aim at) and m_i its metadata bits per parameter, which buy no accuracy.
// theta is found exactly: the budget is a piecewise linear, non-decreasing function of theta, and the
// segment that crosses it is found by sweeping the sorted breakpoints.
#include <algorithm>
#include <cmath>
#include <cstdint>
#include <utility>
#include <vector>

#include "capi_internal.h"
#include "encoder_common.h"
#include "entropack.h"
#include "epk_format.h"

namespace epk {
namespace {

// Largest tables section of format `version`: 9 contexts of lo and count bytes, then one frequency for each
// of 128 + 8 x 64 symbols (12 bits in version 1, 8 in version 2).
uint64_t max_tables_bytes(int version) {
    return 2 * kNumCtx + (uint64_t(prob_bits_of_version(version)) * (128 + 8 * 64) + 7) / 8;
}

// Metadata bytes of an rows x cols blob with G rounds per tile: header, row scales, the largest tables
// section (the only part that depends on the data), tile offsets, and 104 bytes per tile for the final
// rANS states: 128 bytes of states, less the 32 bytes of payload they carry on average, plus 8 of padding.
// These are the charges the encoders' own storage estimate makes.
double metadata_bytes(int64_t rows, int64_t cols, uint32_t G, int version) {
    const uint64_t NG = uint64_t(rows) * uint64_t(cols) / 8;
    const uint64_t T = (NG + 32ull * G - 1) / (32ull * G);
    return double(kHeaderBytes + pad16(2 * uint64_t(rows)) + pad16(max_tables_bytes(version)) + pad16(4 * (T + 1)) +
                  T * (128 - 32 + 8));
}

}  // namespace
}  // namespace epk

extern "C" ep_status ep_plan_bitrates(int64_t n, const int64_t* rows, const int64_t* cols, const double* weight,
                                      double mean_bpp, double min_bpp, double max_bpp, const ep_options* opt_in,
                                      double* bpp_out) {
    using namespace epk;
    clear_error();
    if (n < 1 || !rows || !cols || !weight || !bpp_out) return fail(EP_ERR_ARG, "ep_plan_bitrates: NULL argument or n < 1");
    if (!(mean_bpp >= 0.001 && mean_bpp <= 11.0) || !(min_bpp >= 0.001 && min_bpp <= 11.0) ||
        !(max_bpp >= 0.001 && max_bpp <= 11.0) || min_bpp > max_bpp || mean_bpp > max_bpp)
        return fail(EP_ERR_TARGET, "ep_plan_bitrates: need 0.001 <= min_bpp <= max_bpp <= 11 and mean_bpp in [0.001, max_bpp]");
    ep_options opt;
    ep_options_default(&opt);
    if (opt_in) opt = *opt_in;
    if (opt.format_version == 0) opt.format_version = 2;
    if (opt.rounds_per_tile > uint32_t(kMaxG) || opt.format_version > 2)
        return fail(EP_ERR_ARG, "ep_plan_bitrates: bad rounds_per_tile or format_version");

    const size_t count = static_cast<size_t>(n);
    std::vector<double> c(count), lo(count), hi(count), np(count);
    double total = 0.0, floor_bits = 0.0, ceil_bits = 0.0;
    for (int64_t i = 0; i < n; ++i) {
        const int64_t M = rows[i], N = cols[i];
        if (M < 1 || N < 8 || N % 8 != 0 || M > 0xFFFFFFFFll || N > 0xFFFFFFFFll || (M * N) / 8 > 0xFFFFFFFFll)
            return fail(EP_ERR_SHAPE, "ep_plan_bitrates: layer %lld: need rows >= 1 and cols a positive multiple of 8",
                        (long long)i);
        if (!(weight[i] > 0.0) || !std::isfinite(weight[i]))
            return fail(EP_ERR_ARG, "ep_plan_bitrates: layer %lld: weight must be finite and > 0", (long long)i);
        const uint32_t G = opt.rounds_per_tile ? opt.rounds_per_tile : enc::auto_rounds_per_tile(M * N / 8);
        np[i] = double(M) * double(N);
        const double meta = 8.0 * metadata_bytes(M, N, G, int(opt.format_version)) / np[i];
        c[i] = meta + 0.5 * std::log2(weight[i]);
        hi[i] = max_bpp;
        lo[i] = std::min(std::max(min_bpp, meta), max_bpp);
        total += np[i];
        floor_bits += np[i] * lo[i];
        ceil_bits += np[i] * hi[i];
    }
    const double budget = mean_bpp * total;

    double theta;
    if (budget <= floor_bits) {
        theta = -INFINITY;  // below every layer's floor: each gets its floor, and its blob overshoots
    } else if (budget >= ceil_bits) {
        theta = INFINITY;
    } else {
        // Breakpoints: layer i starts to rise at lo_i - c_i (slope +n_i) and stops at hi_i - c_i (slope -n_i).
        std::vector<std::pair<double, double>> ev;
        ev.reserve(2 * count);
        for (int64_t i = 0; i < n; ++i) {
            ev.emplace_back(lo[i] - c[i], np[i]);
            ev.emplace_back(hi[i] - c[i], -np[i]);
        }
        std::sort(ev.begin(), ev.end());
        double S = floor_bits, slope = 0.0, at = ev[0].first;
        theta = ev.back().first;
        for (size_t k = 0; k < ev.size(); ++k) {
            const double next = ev[k].first;
            if (slope > 0.0 && S + slope * (next - at) >= budget) {
                theta = at + (budget - S) / slope;
                break;
            }
            S += slope * (next - at);
            at = next;
            slope += ev[k].second;
        }
    }
    for (int64_t i = 0; i < n; ++i) bpp_out[i] = std::min(hi[i], std::max(lo[i], c[i] + theta));
    return EP_OK;
}
