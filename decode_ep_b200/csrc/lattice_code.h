// Quantisation of one 8-wide group to E8 and its coding as table symbols. Both EPK1 encoders (host and
// CUDA) compile this same source. Device code that includes it must be built without FMA contraction
// (nvcc --fmad=false), host code with -ffp-contract=off: every operation below is then one IEEE double
// operation, rounded to nearest, in the written order, on either processor.
#pragma once

#include <math.h>
#include <stdint.h>

#include "epk_format.h"

#if defined(__CUDACC__)
#define EPK_HD __host__ __device__ __forceinline__
#else
#define EPK_HD inline
#endif

namespace epk {
namespace enc {

// Nearest point of D8 (integer vectors with even sum), after Conway and Sloane's D_n decoder:
// round each coordinate half away from zero. If the sum is odd, re-round the coordinate that is
// furthest from its rounded value (lowest index on ties) in the other direction.
EPK_HD void nearest_d8(const double* x, int64_t* f) {
    int64_t sum = 0;
    int worst = 0;
    double werr = -1.0;
    for (int k = 0; k < 8; ++k) {
        f[k] = int64_t(::round(x[k]));
        sum += f[k];
        double e = ::fabs(x[k] - double(f[k]));
        if (e > werr) { werr = e; worst = k; }
    }
    if (sum & 1) f[worst] += (x[worst] - double(f[worst]) >= 0.0) ? 1 : -1;
}

// Nearest E8 = D8 ∪ (D8 + 1/2) point. Writes the coset bit and the coded integers t[8]:
// t_i = u_i for i < 7, and t_7 = h, where u_7 = 2h + (Σ_{i<7} u_i mod 2).
EPK_HD int e8_code(const double* x, int32_t* t) {
    int64_t a[8], c[8];
    double xh[8];
    nearest_d8(x, a);
    for (int k = 0; k < 8; ++k) xh[k] = x[k] - 0.5;
    nearest_d8(xh, c);
    double d0 = 0.0, d1 = 0.0;
    for (int k = 0; k < 8; ++k) {
        double e0 = x[k] - double(a[k]);
        double e1 = x[k] - (double(c[k]) + 0.5);
        d0 += e0 * e0;
        d1 += e1 * e1;
    }
    const int64_t* u = (d0 <= d1) ? a : c;
    int64_t s = 0;
    for (int i = 0; i < 7; ++i) { t[i] = int32_t(u[i]); s += u[i]; }
    t[7] = int32_t((u[7] - (s & 1)) / 2);
    return d0 <= d1 ? 0 : 1;
}

EPK_HD int32_t hi_of(int32_t t, int r) { return t >> r; }  // arithmetic shift = floor division by 2^r
EPK_HD int idx_of(int32_t hi) { return (hi >= -31 && hi <= 31) ? hi + 31 : kEscIdx; }
// Magnitude class: 1 when m = floor(|v|), taken on hi, is at least 2.
EPK_HD int cls_of(int32_t hi, int b) {
    int32_t m = hi >= 0 ? hi : -hi - b;
    return m >= 2 ? 1 : 0;
}

// Context and table symbol of each of the 8 positions of one group.
EPK_HD void group_syms(int b, const int32_t* t, int r, uint8_t* ctx, uint8_t* sym, int32_t* hi) {
    for (int i = 0; i < 8; ++i) hi[i] = hi_of(t[i], r);
    ctx[0] = 0;
    sym[0] = uint8_t(64 * b + idx_of(hi[0]));
    for (int i = 1; i < 8; ++i) {
        ctx[i] = uint8_t((i < 7 ? 1 : 5) + 2 * b + cls_of(hi[i - 1], b));
        sym[i] = uint8_t(idx_of(hi[i]));
    }
}

}  // namespace enc
}  // namespace epk
