/*
 * EntroPack oracle — plain, slow CPU encoder and decoder of the EPK1 blob.
 *
 * TEST INFRASTRUCTURE, NOT PRODUCT CODE (see entropack_oracle.h). Built with
 * gcc -O2 -ffp-contract=off so that every float operation is one IEEE
 * binary32/binary64 round-to-nearest-even step, in source order.
 *
 * What it follows (EntroPack, arXiv 2609.34185):
 *  - row normalisation and E8 lattice quantisation — paper page, abstract;
 *  - a conditional probability model of the lattice coordinates, rANS coded
 *    in independently decodable tiles — abstract; modelscope summary;
 *  - the resolution picked from a sampled storage estimate, with no repeated
 *    full encode — abstract; techmoon article on the release;
 *  - target bits per parameter in [0.001, 11], actual size counting metadata
 *    — README, quick-start and Config sections;
 *  - decode = symbol decode, arithmetic inverse of the lattice map, per-row
 *    rescale, with no symbol tensor or codebook — modelscope summary.
 * Every detail the pages leave open is read as the format document states
 * (E8 = D8 ∪ D8+½, 9 contexts of frequency tables conditioned on the coset
 * bit and the previous coordinate's magnitude class, 32-lane interleaved
 * rANS). The format has two versions, and this file follows both:
 *  - version 1: 12-bit tables, the state renormalised after every symbol;
 *  - version 2: 8-bit tables, the state renormalised after every pair of
 *    symbols, rare symbols sent as escapes, and a round's escape words read
 *    after its last pair.
 */
#include "entropack_oracle.h"

#include <math.h>
#include <stdlib.h>
#include <string.h>

enum { OK = 0, E_ARG = -1, E_DTYPE = -2, E_SHAPE = -3, E_TARGET = -4, E_NONFINITE = -5,
       E_CORRUPT = -6, E_NOMEM = -8 };

#define LANES 32
#define NCTX 9
#define PROB_BITS 12      /* version 1 */
#define PROB_SCALE 4096u
#define PROB_BITS_V2 8    /* version 2 */
#define PROB_SCALE_V2 256u
#define RANS_L 65536u
#define ESC_IDX 63
#define HEADER_BYTES 64
/* Version 2: a symbol (other than hi in [-2, 2]) seen in fewer than 1/2^ESC_SHIFT of its
 * context's coordinates is sent as an escape. */
#define ESC_SHIFT 14

/* ---------------------------------------------------------------- helpers */

static uint64_t pad16(uint64_t n) { return (n + 15) & ~(uint64_t)15; }
static uint64_t pad4(uint64_t n) { return (n + 3) & ~(uint64_t)3; }

static void put_u16(uint8_t* p, uint32_t v) { p[0] = (uint8_t)v; p[1] = (uint8_t)(v >> 8); }
static void put_u32(uint8_t* p, uint32_t v) {
    for (int i = 0; i < 4; i++) p[i] = (uint8_t)(v >> (8 * i));
}
static void put_u64(uint8_t* p, uint64_t v) {
    for (int i = 0; i < 8; i++) p[i] = (uint8_t)(v >> (8 * i));
}
static uint32_t get_u16(const uint8_t* p) { return (uint32_t)p[0] | ((uint32_t)p[1] << 8); }
static uint32_t get_u32(const uint8_t* p) {
    uint32_t v = 0;
    for (int i = 0; i < 4; i++) v |= (uint32_t)p[i] << (8 * i);
    return v;
}
static uint64_t get_u64(const uint8_t* p) {
    uint64_t v = 0;
    for (int i = 0; i < 8; i++) v |= (uint64_t)p[i] << (8 * i);
    return v;
}
static float bits_to_f32(uint32_t u) { float f; memcpy(&f, &u, 4); return f; }
static uint32_t f32_to_bits(float f) { uint32_t u; memcpy(&u, &f, 4); return u; }

uint32_t orc_crc32(const uint8_t* p, size_t n) {
    /* Bitwise CRC-32, reflected, polynomial 0xEDB88320, init and final xor ~0. */
    uint32_t c = 0xFFFFFFFFu;
    for (size_t i = 0; i < n; i++) {
        c ^= p[i];
        for (int k = 0; k < 8; k++) c = (c & 1) ? (c >> 1) ^ 0xEDB88320u : (c >> 1);
    }
    return c ^ 0xFFFFFFFFu;
}

/* ------------------------------------------------------ container formats */

static int elem_size(int dtype) {
    switch (dtype) {
        case 1: case 2: return 2;
        case 3: return 4;
        case 4: case 5: return 1;
        default: return 0;
    }
}

/* BF16 keeps the top 16 bits of the binary32 pattern; round to nearest, ties
 * to the even result (IEEE 754 roundTiesToEven). */
static uint16_t f32_to_bf16(float f) {
    uint32_t u = f32_to_bits(f);
    if (isnan(f)) return (uint16_t)((u >> 16) | 0x40);
    uint32_t upper = u >> 16, lower = u & 0xFFFFu;
    if (lower > 0x8000u || (lower == 0x8000u && (upper & 1u))) upper += 1; /* carries into the exponent */
    return (uint16_t)upper;
}
static float bf16_to_f32(uint16_t h) { return bits_to_f32((uint32_t)h << 16); }

/* IEEE binary16: 1 sign, 5 exponent (bias 15), 10 fraction bits. */
static uint16_t f32_to_f16(float f) {
    uint16_t sign = (f32_to_bits(f) >> 16) & 0x8000u;
    if (isnan(f)) return 0x7E00;
    double a = fabs((double)f);
    if (a >= 65520.0) return sign | 0x7C00; /* halfway past 65504 rounds to 2^16: overflow */
    if (a == 0.0) return sign;
    int e;
    frexp(a, &e);
    e -= 1;                                 /* a in [2^e, 2^(e+1)) */
    double quantum = (e < -14) ? ldexp(1.0, -24) : ldexp(1.0, e - 10);
    double n = nearbyint(a / quantum);      /* exact quotient; ties to even */
    if (e < -14) return sign | (uint16_t)n; /* subnormal, or exactly the smallest normal */
    if (n == 2048.0) { e += 1; n = 1024.0; }
    if (e + 15 >= 31) return sign | 0x7C00;
    return sign | (uint16_t)((e + 15) << 10) | (uint16_t)(n - 1024.0);
}
static float f16_to_f32(uint16_t h) {
    int s = (h >> 15) & 1, e = (h >> 10) & 31, m = h & 1023;
    double v;
    if (e == 31) v = m ? NAN : INFINITY;
    else if (e == 0) v = ldexp((double)m, -24);
    else v = ldexp(1024.0 + m, e - 25);
    return (float)(s ? -v : v);
}

/* OCP FP8 E4M3: 1 sign, 4 exponent (bias 7), 3 mantissa bits, max finite 448,
 * S.1111.111 = NaN. Conversion rounds to nearest even and saturates to ±448. */
static uint8_t f32_to_e4m3_sat(float f) {
    uint8_t sign = (f32_to_bits(f) >> 24) & 0x80u;
    if (isnan(f)) return 0x7F;
    double a = fabs((double)f);
    if (a >= 448.0) return sign | 0x7E;
    if (a == 0.0) return sign;
    int e;
    frexp(a, &e);
    e -= 1;
    double quantum = (e < -6) ? ldexp(1.0, -9) : ldexp(1.0, e - 3);
    double n = nearbyint(a / quantum);
    if (e < -6) return sign | (uint8_t)n;   /* subnormal; n == 8 is the smallest normal */
    if (n == 16.0) { e += 1; n = 8.0; }
    return sign | (uint8_t)((e + 7) << 3) | (uint8_t)(n - 8.0);
}
static float e4m3_to_f32(uint8_t c) {
    int s = (c >> 7) & 1, e = (c >> 3) & 15, m = c & 7;
    double v;
    if (e == 15 && m == 7) v = NAN;
    else if (e == 0) v = ldexp((double)m, -9);
    else v = ldexp(8.0 + m, e - 10);
    return (float)(s ? -v : v);
}

static int8_t f32_to_i8(float f) {
    double n = nearbyint((double)f); /* ties to even under the default rounding mode */
    if (n < -128.0) n = -128.0;
    if (n > 127.0) n = 127.0;
    return (int8_t)n;
}

void orc_to_container(const float* y, int64_t n, int dtype, void* out) {
    for (int64_t i = 0; i < n; i++) {
        switch (dtype) {
            case 1: ((uint16_t*)out)[i] = f32_to_bf16(y[i]); break;
            case 2: ((uint16_t*)out)[i] = f32_to_f16(y[i]); break;
            case 3: ((float*)out)[i] = y[i]; break;
            case 4: ((uint8_t*)out)[i] = f32_to_e4m3_sat(y[i]); break;
            case 5: ((int8_t*)out)[i] = f32_to_i8(y[i]); break;
        }
    }
}

int orc_from_container(const void* in, int64_t n, int dtype, float* out) {
    if (!elem_size(dtype)) return E_DTYPE;
    for (int64_t i = 0; i < n; i++) {
        float v = 0;
        switch (dtype) {
            case 1: v = bf16_to_f32(((const uint16_t*)in)[i]); break;
            case 2: v = f16_to_f32(((const uint16_t*)in)[i]); break;
            case 3: v = ((const float*)in)[i]; break;
            case 4: v = e4m3_to_f32(((const uint8_t*)in)[i]); break;
            case 5: v = (float)((const int8_t*)in)[i]; break;
        }
        if (!isfinite(v)) return E_NONFINITE;
        out[i] = v;
    }
    return OK;
}

/* ---------------------------------------------------------------- lattice */

/* Nearest point of D_n = {integer vectors with even sum} (Conway & Sloane,
 * "Fast quantizing and decoding algorithms for lattice quantizers", 1982):
 * round every coordinate; if the sum is odd, round the coordinate that was
 * furthest from its rounded value the other way. Rounding is half away from
 * zero; ties on the worst coordinate go to the lowest index. */
static void nearest_d8(const double x[8], int64_t f[8]) {
    int64_t sum = 0;
    int worst = 0;
    double worst_err = -1.0;
    for (int k = 0; k < 8; k++) {
        f[k] = (int64_t)round(x[k]);
        sum += f[k];
        double err = fabs(x[k] - (double)f[k]);
        if (err > worst_err) { worst_err = err; worst = k; }
    }
    if (sum & 1) f[worst] += (x[worst] - (double)f[worst] >= 0.0) ? 1 : -1;
}

/* E8 = D8 ∪ (D8 + ½): decode x in both cosets, keep the nearer (ties → D8). */
void orc_e8_nearest(const double* x, int32_t* b, int64_t* u) {
    int64_t f0[8], f1[8];
    double xs[8];
    nearest_d8(x, f0);
    for (int k = 0; k < 8; k++) xs[k] = x[k] - 0.5;
    nearest_d8(xs, f1);
    double d0 = 0.0, d1 = 0.0;
    for (int k = 0; k < 8; k++) {
        double e0 = x[k] - (double)f0[k];
        double e1 = x[k] - ((double)f1[k] + 0.5);
        d0 += e0 * e0;
        d1 += e1 * e1;
    }
    if (d0 <= d1) { *b = 0; for (int k = 0; k < 8; k++) u[k] = f0[k]; }
    else          { *b = 1; for (int k = 0; k < 8; k++) u[k] = f1[k]; }
}

/* ---------------------------------------------------- coordinates ↔ symbols */

typedef struct {
    int b;
    int64_t t[8];  /* t_i = u_i (i < 7), t_7 = h with u_7 = 2h + π */
} Group;

static void group_from_point(int b, const int64_t u[8], Group* g) {
    int64_t s = 0;
    for (int i = 0; i < 7; i++) { g->t[i] = u[i]; s += u[i]; }
    int64_t pi = s & 1;
    g->t[7] = (u[7] - pi) / 2; /* exact: u_7 ≡ Σ_{i<7} u_i (mod 2) */
    g->b = b;
}

static int64_t floor_shift(int64_t t, int r) { return (t >= 0) ? (t >> r) : -((-t + ((int64_t)1 << r) - 1) >> r); }

static int sym_index(int64_t hi) { return (hi >= -31 && hi <= 31) ? (int)(hi + 31) : ESC_IDX; }

/* Magnitude class of a coded coordinate: 1 when m = ⌊|v|⌋ (taken on hi) is at least 2, else 0. */
static int mag_class(int64_t hi, int b) {
    int64_t m = (hi >= 0) ? hi : -hi - b;
    return m >= 2 ? 1 : 0;
}

/* Context of position i, given the previous position's hi and the coset bit:
 * START for position 0, 1 + 2b + class for positions 1..6, 5 + 2b + class for position 7. */
static int context_of(int i, int64_t hi_prev, int b) {
    if (i == 0) return 0;
    return (i < 7 ? 1 : 5) + 2 * b + mag_class(hi_prev, b);
}

/* --------------------------------------------------- frequency normalisation */

/* n is the alphabet size, scale = 2^bits the table total (4096 in version 1, 256 in version 2).
 * Every present symbol gets f >= 1 and no f exceeds scale - 1: a context with a single present
 * symbol s gives it scale - 1 and its neighbour (s + 1, or s - 1 at the end of the alphabet) the
 * remaining 1. */
static int normalize_scale(const uint64_t* counts, int n, uint32_t scale, uint32_t* f);

int orc_normalize(const uint64_t* counts, int n, uint32_t* f) { return normalize_scale(counts, n, PROB_SCALE, f); }

int orc_normalize_bits(const uint64_t* counts, int n, int bits, uint32_t* f) {
    if (bits != PROB_BITS && bits != PROB_BITS_V2) return E_ARG;
    return normalize_scale(counts, n, 1u << bits, f);
}

static int normalize_scale(const uint64_t* counts, int n, uint32_t scale, uint32_t* f) {
    uint64_t total = 0;
    int present = 0;
    for (int s = 0; s < n; s++) { total += counts[s]; if (counts[s]) present++; }
    for (int s = 0; s < n; s++) f[s] = 0;
    if (present == 0) return OK;
    if (present == 1) {
        for (int s = 0; s < n; s++)
            if (counts[s]) {
                f[s] = scale - 1;
                f[s + 1 < n ? s + 1 : s - 1] = 1;
            }
        return OK;
    }
    int64_t sum = 0;
    for (int s = 0; s < n; s++) {
        if (!counts[s]) continue;
        uint64_t q = (counts[s] * (uint64_t)scale) / total;
        f[s] = q < 1 ? 1 : (uint32_t)q;
        sum += f[s];
    }
    int64_t d = (int64_t)scale - sum;
    while (d != 0) {
        int best = -1;
        for (int s = 0; s < n; s++)
            if (f[s] && (best < 0 || f[s] > f[best])) best = s;
        if (d > 0) { f[best] += (uint32_t)d; d = 0; }
        else {
            int64_t take = -d < (int64_t)f[best] - 1 ? -d : (int64_t)f[best] - 1;
            f[best] -= (uint32_t)take;
            d += take;
        }
    }
    return OK;
}

/* ------------------------------------------------------- model (17 tables) */

typedef struct {
    int bits;                /* table precision: 12 (version 1) or 8 (version 2) */
    int lo[NCTX], cnt[NCTX];
    uint32_t f[NCTX][128];   /* indexed by symbol */
    uint32_t cum[NCTX][129]; /* cumulative, indexed by symbol */
} Model;

static int ctx_alphabet(int c) { return c == 0 ? 128 : 64; }

/* The escape symbol of a context symbol s: index 63 of s's coset half (START codes 64 b + idx). */
static int esc_symbol_of(int s) { return (s & 64) | ESC_IDX; }

/* Version 2: moves the counts of rare symbols onto their escape symbol. A symbol is rare when it is
 * seen in fewer than 1/2^ESC_SHIFT of its context's coordinates. hi in [-2, 2] (idx 29..33) is never
 * escaped, so an escaped coordinate always has magnitude class 1. */
static void escape_rare(uint64_t counts[NCTX][128]) {
    for (int c = 0; c < NCTX; c++) {
        int A = ctx_alphabet(c);
        uint64_t n = 0;
        for (int s = 0; s < A; s++) n += counts[c][s];
        for (int s = 0; s < A; s++) {
            int idx = s & 63;
            if (idx == ESC_IDX || (idx >= 29 && idx <= 33) || counts[c][s] == 0) continue;
            if ((counts[c][s] << ESC_SHIFT) < n) {
                counts[c][esc_symbol_of(s)] += counts[c][s];
                counts[c][s] = 0;
            }
        }
    }
}

/* The counts a table of precision `bits` is fitted to: version 2 first moves rare symbols onto the
 * escapes. */
static void prepare_counts(uint64_t counts[NCTX][128], int bits) {
    if (bits == PROB_BITS_V2) escape_rare(counts);
}

/* Fits the tables to prepared counts. */
static void model_from_counts(uint64_t counts[NCTX][128], int bits, Model* m) {
    memset(m, 0, sizeof(*m));
    m->bits = bits;
    for (int c = 0; c < NCTX; c++) {
        int A = ctx_alphabet(c), lo = -1, hi = -1;
        normalize_scale(counts[c], A, 1u << bits, m->f[c]);
        for (int s = 0; s < A; s++) if (m->f[c][s]) { if (lo < 0) lo = s; hi = s; }
        m->lo[c] = lo < 0 ? 0 : lo;
        m->cnt[c] = lo < 0 ? 0 : hi - lo + 1;
        uint32_t acc = 0;
        for (int s = 0; s < 128; s++) { m->cum[c][s] = acc; acc += m->f[c][s]; }
        m->cum[c][128] = acc;
    }
}

/* Frequencies are stored as m->bits-bit fields, packed LSB-first (12 bits in version 1, one byte each
 * in version 2). */
static uint64_t tables_bytes(const Model* m) {
    uint64_t nsym = 0;
    for (int c = 0; c < NCTX; c++) nsym += (uint64_t)m->cnt[c];
    return 2 * NCTX + ((uint64_t)m->bits * nsym + 7) / 8;
}

static void write_tables(const Model* m, uint8_t* out) {
    uint64_t bit = 0;
    uint8_t* bits = out + 2 * NCTX;
    for (int c = 0; c < NCTX; c++) { out[c] = (uint8_t)m->lo[c]; out[NCTX + c] = (uint8_t)m->cnt[c]; }
    for (int c = 0; c < NCTX; c++) {
        for (int s = m->lo[c]; s < m->lo[c] + m->cnt[c]; s++) {
            uint32_t v = m->f[c][s];
            for (int k = 0; k < m->bits; k++, bit++)
                if ((v >> k) & 1) bits[bit >> 3] |= (uint8_t)(1u << (bit & 7));
        }
    }
}

/* Returns 0 or E_CORRUPT. avail = bytes available for the tables section; bits = the precision the
 * header's version fixes. */
static int read_tables(const uint8_t* in, uint64_t avail, int bits_per_f, Model* m, uint64_t* used) {
    memset(m, 0, sizeof(*m));
    m->bits = bits_per_f;
    const uint32_t scale = 1u << bits_per_f;
    if (avail < 2 * NCTX) return E_CORRUPT;
    uint64_t nsym = 0;
    for (int c = 0; c < NCTX; c++) {
        m->lo[c] = in[c];
        m->cnt[c] = in[NCTX + c];
        if (m->cnt[c] == 0 && m->lo[c] != 0) return E_CORRUPT;
        if (m->lo[c] + m->cnt[c] > ctx_alphabet(c)) return E_CORRUPT;
        nsym += (uint64_t)m->cnt[c];
    }
    *used = 2 * NCTX + ((uint64_t)bits_per_f * nsym + 7) / 8;
    if (*used > avail) return E_CORRUPT;
    const uint8_t* bits = in + 2 * NCTX;
    uint64_t bit = 0;
    for (int c = 0; c < NCTX; c++) {
        uint32_t total = 0;
        for (int s = m->lo[c]; s < m->lo[c] + m->cnt[c]; s++) {
            uint32_t v = 0;
            for (int k = 0; k < bits_per_f; k++, bit++) v |= (uint32_t)((bits[bit >> 3] >> (bit & 7)) & 1) << k;
            m->f[c][s] = v;
            total += v;
        }
        if (m->cnt[c] == 1) {
            return E_CORRUPT; /* a lone symbol is stored as (scale - 1) + 1 */
        } else if (m->cnt[c] >= 2) {
            if (total != scale) return E_CORRUPT;
            for (int s = m->lo[c]; s < m->lo[c] + m->cnt[c]; s++)
                if (m->f[c][s] > scale - 1) return E_CORRUPT;
        }
        uint32_t acc = 0;
        for (int s = 0; s < 128; s++) { m->cum[c][s] = acc; acc += m->f[c][s]; }
        m->cum[c][128] = acc;
    }
    return OK;
}

/* ------------------------------------------------------------- the tensor */

typedef struct {
    int64_t M, N, NG;
    float* w;        /* values as binary32 */
    uint16_t* sbits; /* bf16 pattern of s_row */
    float* s;        /* s_row as binary32 */
} Tensor;

static void tensor_free(Tensor* t) { free(t->w); free(t->sbits); free(t->s); }

static int tensor_load(const void* data, int dtype, int64_t M, int64_t N, Tensor* t) {
    memset(t, 0, sizeof(*t));
    t->M = M; t->N = N; t->NG = M * N / 8;
    t->w = (float*)malloc(sizeof(float) * (size_t)(M * N));
    t->sbits = (uint16_t*)malloc(sizeof(uint16_t) * (size_t)M);
    t->s = (float*)malloc(sizeof(float) * (size_t)M);
    if (!t->w || !t->sbits || !t->s) { tensor_free(t); return E_NOMEM; }
    int st = orc_from_container(data, M * N, dtype, t->w);
    if (st) { tensor_free(t); return st; }
    /* Row scale: root mean square of the row, the sum taken in double in
     * index order, rounded to binary32 and then to BF16. */
    for (int64_t i = 0; i < M; i++) {
        double acc = 0.0;
        for (int64_t j = 0; j < N; j++) acc += (double)t->w[i * N + j] * (double)t->w[i * N + j];
        float rms = (float)sqrt(acc / (double)N);
        t->sbits[i] = f32_to_bf16(rms);
        t->s[i] = bf16_to_f32(t->sbits[i]);
    }
    return OK;
}

/* Quantise group g at resolution alpha: x = (alpha·w)/s in double. */
static void quantize_group(const Tensor* t, int64_t g, float alpha, Group* out) {
    int64_t gpr = t->N / 8, row = g / gpr, col = (g % gpr) * 8;
    double x[8];
    int64_t u[8];
    int32_t b;
    for (int k = 0; k < 8; k++) {
        double w = (double)t->w[row * t->N + col + k];
        x[k] = (t->s[row] == 0.0f) ? 0.0 : ((double)alpha * w) / (double)t->s[row];
    }
    orc_e8_nearest(x, &b, u);
    group_from_point(b, u, out);
}

/* The symbols of one group at raw-bit count r: ctx, sym (table index) and hi per position. With a
 * model m (NULL while counting), a symbol the tables give no frequency (a rare symbol of version 2) is
 * replaced by its escape; esc[i] (if not NULL) tells whether position i is sent as an escape. The
 * context comes from the previous coordinate's true hi: an escaped coordinate has |hi| >= 3, so its
 * class is 1 either way. */
static void group_symbols_m(const Group* g, int r, const Model* m, int ctx[8], int sym[8], int64_t hi[8], int esc[8]) {
    for (int i = 0; i < 8; i++) {
        hi[i] = floor_shift(g->t[i], r);
        int idx = sym_index(hi[i]);
        ctx[i] = context_of(i, i ? hi[i - 1] : 0, g->b);
        sym[i] = (i == 0) ? 64 * g->b + idx : idx;
        if (m && m->f[ctx[i]][sym[i]] == 0) sym[i] = esc_symbol_of(sym[i]);
        if (esc) esc[i] = (sym[i] & 63) == ESC_IDX;
    }
}

static void group_symbols(const Group* g, int r, int ctx[8], int sym[8], int64_t hi[8]) {
    group_symbols_m(g, r, NULL, ctx, sym, hi, NULL);
}

/* Smallest r with 8·2^r >= alpha, at most 12. */
static int raw_bits_for(float alpha) {
    int r = 0;
    while (r < 12 && 8.0 * (double)((int64_t)1 << r) < (double)alpha) r++;
    return r;
}

static uint64_t num_tiles(int64_t NG, int G) { return (uint64_t)((NG + 32LL * G - 1) / (32LL * G)); }

/* Exact section sizes, plus 104 bytes per tile: 32 four-byte states less the
 * 8 bits of payload a final rANS state carries on average (its value is close
 * to log-uniform on [2^16, 2^32)), plus 8 bytes of expected padding. */
static double metadata_bytes(int64_t M, uint64_t T, const Model* m) {
    return (double)(HEADER_BYTES + pad16(2 * (uint64_t)M) + pad16(tables_bytes(m)) + pad16(4 * (T + 1)) +
                    T * (128 - 32 + 8));
}

/* Sampled storage estimate (format document, encoder choices, item 5). */
static double estimate_bytes(const Tensor* t, int G, float alpha, int pbits) {
    int64_t M = t->M, N = t->N, gpr = N / 8;
    int64_t Rs = (262144 + N - 1) / N;
    if (Rs > M) Rs = M;
    int r = raw_bits_for(alpha);
    uint64_t counts[NCTX][128];
    memset(counts, 0, sizeof(counts));
    uint64_t n_esc = 0, ng_s = 0;
    for (int64_t k = 0; k < Rs; k++) {
        int64_t row = (k * M) / Rs;
        for (int64_t q = 0; q < gpr; q++) {
            Group g;
            int ctx[8], sym[8];
            int64_t hi[8];
            quantize_group(t, row * gpr + q, alpha, &g);
            group_symbols(&g, r, ctx, sym, hi);
            for (int i = 0; i < 8; i++) counts[ctx[i]][sym[i]]++;
            ng_s++;
        }
    }
    prepare_counts(counts, pbits);
    for (int c = 0; c < NCTX; c++) {
        n_esc += counts[c][ESC_IDX];
        if (c == 0) n_esc += counts[c][64 | ESC_IDX];
    }
    Model m;
    model_from_counts(counts, pbits, &m);
    double bits = 0.0;
    for (int c = 0; c < NCTX; c++)
        for (int s = m.lo[c]; s < m.lo[c] + m.cnt[c]; s++)
            if (counts[c][s]) bits += (double)counts[c][s] * ((double)pbits - log2((double)m.f[c][s]));
    bits += 16.0 * (double)n_esc + 8.0 * (double)r * (double)ng_s;
    double bits_full = bits * (double)t->NG / (double)ng_s;
    return metadata_bytes(M, num_tiles(t->NG, G), &m) + ceil(bits_full / 8.0);
}

static int check_shape(int dtype, int64_t M, int64_t N) {
    if (!elem_size(dtype)) return E_DTYPE;
    if (M < 1 || N < 8 || N % 8 != 0 || M > 0xFFFFFFFFLL || N > 0xFFFFFFFFLL) return E_SHAPE;
    if ((M * N) / 8 > 0xFFFFFFFFLL) return E_SHAPE;
    return OK;
}

double orc_estimate_bytes(const void* data, int dtype, int64_t M, int64_t N, int G, float alpha, int prob_bits) {
    Tensor t;
    if (prob_bits != PROB_BITS && prob_bits != PROB_BITS_V2) return -1.0;
    if (check_shape(dtype, M, N) || tensor_load(data, dtype, M, N, &t)) return -1.0;
    double e = estimate_bytes(&t, G, alpha, prob_bits);
    tensor_free(&t);
    return e;
}

int orc_quantize(const void* data, int dtype, int64_t M, int64_t N, float alpha, int32_t* zout,
                 uint16_t* scales_out) {
    int st = check_shape(dtype, M, N);
    if (st) return st;
    Tensor t;
    if ((st = tensor_load(data, dtype, M, N, &t))) return st;
    for (int64_t g = 0; g < t.NG; g++) {
        Group q;
        quantize_group(&t, g, alpha, &q);
        int64_t u[8], s = 0;
        for (int i = 0; i < 7; i++) { u[i] = q.t[i]; s += u[i]; }
        u[7] = 2 * q.t[7] + (s & 1);
        for (int i = 0; i < 8; i++) zout[g * 8 + i] = (int32_t)(2 * u[i] + q.b);
    }
    if (scales_out) memcpy(scales_out, t.sbits, sizeof(uint16_t) * (size_t)M);
    tensor_free(&t);
    return OK;
}

/* ----------------------------------------------------------------- encoder */

typedef struct { uint16_t* w; size_t n, cap; } Words;

static int push_word(Words* ws, uint32_t v) {
    if (ws->n == ws->cap) {
        size_t cap = ws->cap ? 2 * ws->cap : 1024;
        uint16_t* p = (uint16_t*)realloc(ws->w, cap * sizeof(uint16_t));
        if (!p) return E_NOMEM;
        ws->w = p; ws->cap = cap;
    }
    ws->w[ws->n++] = (uint16_t)v;
    return OK;
}

typedef struct { uint8_t* bytes; uint64_t size; int has_esc; } TileOut;

/* Lays out one tile: the 32 final states, the raw low bits (8 fields of r bits per group, LSB-first),
 * the pushed words in reverse push order, zero padding to 16 bytes. Frees the word list. */
static int finish_tile(const Group* groups, int64_t g0, int64_t ng, int r, const uint32_t x[LANES], Words* ws,
                       int has_esc, TileOut* out) {
    uint64_t raw = pad4((uint64_t)ng * (uint64_t)r);
    uint64_t size = pad16(128 + raw + 2 * (uint64_t)ws->n);
    uint8_t* p = (uint8_t*)calloc((size_t)size, 1);
    if (!p) { free(ws->w); return E_NOMEM; }
    for (int L = 0; L < LANES; L++) put_u32(p + 4 * L, x[L]);
    uint8_t* rawp = p + 128;
    for (int64_t q = 0; q < ng && r > 0; q++) {
        for (int i = 0; i < 8; i++) {
            int64_t t = groups[g0 + q].t[i];
            int64_t lo = t - floor_shift(t, r) * ((int64_t)1 << r);
            uint64_t bit = 8 * (uint64_t)r * (uint64_t)q + (uint64_t)(i * r);
            for (int k = 0; k < r; k++, bit++)
                if ((lo >> k) & 1) rawp[bit >> 3] |= (uint8_t)(1u << (bit & 7));
        }
    }
    uint8_t* sp = p + 128 + raw;
    for (size_t n = 0; n < ws->n; n++) put_u16(sp + 2 * n, ws->w[ws->n - 1 - n]); /* reversed */
    out->bytes = p; out->size = size; out->has_esc = has_esc;
    free(ws->w);
    return OK;
}

/* Encode one tile: the decode order of the format document, run backwards. */
static int encode_tile(const Group* groups, int64_t g0, int64_t ng, int r, const Model* m, TileOut* out) {
    uint32_t x[LANES];
    Words ws = {0, 0, 0};
    int64_t R = (ng + 31) / 32;
    int has_esc = 0;
    for (int L = 0; L < LANES; L++) x[L] = RANS_L;
    for (int64_t k = R - 1; k >= 0; k--) {
        for (int i = 7; i >= 0; i--) {
            /* ESC phase, reversed: lanes descending. */
            for (int L = LANES - 1; L >= 0; L--) {
                int64_t q = 32 * k + L;
                if (q >= ng) continue;
                int ctx[8], sym[8];
                int64_t hi[8];
                group_symbols(&groups[g0 + q], r, ctx, sym, hi);
                if (sym_index(hi[i]) == ESC_IDX) {
                    if (push_word(&ws, (uint32_t)(uint16_t)(int16_t)hi[i])) goto nomem;
                    has_esc = 1;
                }
            }
            /* Symbol phase, reversed: renormalise, then C(s, x). */
            for (int L = LANES - 1; L >= 0; L--) {
                int64_t q = 32 * k + L;
                if (q >= ng) continue;
                int ctx[8], sym[8];
                int64_t hi[8];
                group_symbols(&groups[g0 + q], r, ctx, sym, hi);
                uint32_t f = m->f[ctx[i]][sym[i]], c = m->cum[ctx[i]][sym[i]];
                if ((uint64_t)x[L] >= ((uint64_t)f << 20)) {
                    if (push_word(&ws, x[L] & 0xFFFFu)) goto nomem;
                    x[L] >>= 16;
                }
                x[L] = (x[L] / f) * PROB_SCALE + (x[L] % f) + c;
            }
        }
    }
    return finish_tile(groups, g0, ng, r, x, &ws, has_esc, out);
nomem:
    free(ws.w);
    return E_NOMEM;
}

/* Version 2 tile: the decode order of the format document (pairs of positions share one
 * renormalisation; a round's escape words follow its last pair), run backwards. Every coordinate
 * before its pair is encoded: if x >= f1 f2 2^16 the lane first pushes x & 0xFFFF and sets x >>= 16,
 * then x <- C(s2, x), then x <- C(s1, x), with C(s, x) = floor(x/f) 2^8 + (x mod f) + cum. */
static int encode_tile_v2(const Group* groups, int64_t g0, int64_t ng, int r, const Model* m, TileOut* out) {
    uint32_t x[LANES];
    Words ws = {0, 0, 0};
    int64_t R = (ng + 31) / 32;
    int has_esc = 0;
    for (int L = 0; L < LANES; L++) x[L] = RANS_L;
    for (int64_t k = R - 1; k >= 0; k--) {
        int ctx[LANES][8], sym[LANES][8], esc[LANES][8];
        int64_t hi[LANES][8];
        for (int L = 0; L < LANES; L++)
            if (32 * k + L < ng) group_symbols_m(&groups[g0 + 32 * k + L], r, m, ctx[L], sym[L], hi[L], esc[L]);
        /* Escape words of the round, reversed: positions descending, lanes descending. */
        for (int i = 7; i >= 0; i--)
            for (int L = LANES - 1; L >= 0; L--) {
                if (32 * k + L >= ng || !esc[L][i]) continue;
                if (push_word(&ws, (uint32_t)(uint16_t)(int16_t)hi[L][i])) goto nomem;
                has_esc = 1;
            }
        /* Pairs, reversed: renormalise, then C(s2, x), then C(s1, x). */
        for (int p = 3; p >= 0; p--) {
            for (int L = LANES - 1; L >= 0; L--) {
                if (32 * k + L >= ng) continue;
                int i1 = 2 * p, i2 = 2 * p + 1;
                uint32_t f1 = m->f[ctx[L][i1]][sym[L][i1]], c1 = m->cum[ctx[L][i1]][sym[L][i1]];
                uint32_t f2 = m->f[ctx[L][i2]][sym[L][i2]], c2 = m->cum[ctx[L][i2]][sym[L][i2]];
                if ((uint64_t)x[L] >= (((uint64_t)f1 * f2) << 16)) {
                    if (push_word(&ws, x[L] & 0xFFFFu)) goto nomem;
                    x[L] >>= 16;
                }
                x[L] = (x[L] / f2) * PROB_SCALE_V2 + (x[L] % f2) + c2;
                x[L] = (x[L] / f1) * PROB_SCALE_V2 + (x[L] % f1) + c1;
            }
        }
    }
    return finish_tile(groups, g0, ng, r, x, &ws, has_esc, out);
nomem:
    free(ws.w);
    return E_NOMEM;
}

int orc_compress(const void* data, int dtype, int64_t M, int64_t N, double target_bpp, int G,
                 double force_alpha, int prob_bits, uint8_t** blob_out, size_t* bytes_out, double* actual_bpp) {
    int st = check_shape(dtype, M, N);
    if (st) return st;
    if (!(target_bpp >= 0.001 && target_bpp <= 11.0)) return E_TARGET; /* also rejects NaN */
    if (G < 1 || G > 1024 || !blob_out || !bytes_out) return E_ARG;
    if (prob_bits != PROB_BITS && prob_bits != PROB_BITS_V2) return E_ARG;
    Tensor t;
    if ((st = tensor_load(data, dtype, M, N, &t))) return st;

    /* Resolution cap: keeps |x| <= 2^22 so that 2v fits binary32 exactly. */
    double amax = 0.0;
    for (int64_t i = 0; i < M; i++)
        for (int64_t j = 0; j < N && t.s[i] != 0.0f; j++) {
            double a = fabs((double)t.w[i * N + j]) / (double)t.s[i];
            if (a > amax) amax = a;
        }
    float alpha;
    if (force_alpha > 0.0) {
        alpha = (float)force_alpha;
    } else {
        double lo = -12.0, hi = 15.0;
        if (amax > 0.0) { double cap = 22.0 - log2(amax); if (cap < hi) hi = cap; }
        if (hi < lo) hi = lo;
        double budget = target_bpp * (double)M * (double)N;
        for (int it = 0; it < 40; it++) {
            double mid = 0.5 * (lo + hi);
            float a = (float)exp2(mid);
            if (8.0 * estimate_bytes(&t, G, a, prob_bits) <= budget) lo = mid; else hi = mid;
        }
        alpha = (float)exp2(lo);
    }
    if (!(alpha > 0.0f) || !isfinite(alpha)) { tensor_free(&t); return E_ARG; }

    /* Quantise everything; pick r; fit the tables on the whole tensor. */
    Group* groups = (Group*)malloc(sizeof(Group) * (size_t)t.NG);
    if (!groups) { tensor_free(&t); return E_NOMEM; }
    int64_t tabs = 0;
    for (int64_t g = 0; g < t.NG; g++) {
        quantize_group(&t, g, alpha, &groups[g]);
        for (int i = 0; i < 8; i++) {
            int64_t v = groups[g].t[i], a = v >= 0 ? v : -v - 1;
            if (a > tabs) tabs = a;
        }
    }
    int r = raw_bits_for(alpha);
    while (r < 12 && tabs >= ((int64_t)1 << (15 + r))) r++;
    if (tabs >= ((int64_t)1 << (15 + r))) { free(groups); tensor_free(&t); return E_ARG; }

    uint64_t counts[NCTX][128];
    memset(counts, 0, sizeof(counts));
    for (int64_t g = 0; g < t.NG; g++) {
        int ctx[8], sym[8];
        int64_t hi[8];
        group_symbols(&groups[g], r, ctx, sym, hi);
        for (int i = 0; i < 8; i++) counts[ctx[i]][sym[i]]++;
    }
    prepare_counts(counts, prob_bits);
    Model m;
    model_from_counts(counts, prob_bits, &m);

    uint64_t T = num_tiles(t.NG, G);
    TileOut* tiles = (TileOut*)calloc((size_t)T, sizeof(TileOut));
    if (!tiles) { free(groups); tensor_free(&t); return E_NOMEM; }
    uint64_t payload = 0;
    for (uint64_t j = 0; j < T; j++) {
        int64_t g0 = (int64_t)j * 32 * G, ng = t.NG - g0 < 32LL * G ? t.NG - g0 : 32LL * G;
        st = prob_bits == PROB_BITS ? encode_tile(groups, g0, ng, r, &m, &tiles[j])
                                    : encode_tile_v2(groups, g0, ng, r, &m, &tiles[j]);
        if (st) break;
        payload += tiles[j].size;
    }
    uint8_t* blob = NULL;
    uint64_t total = 0;
    if (!st && payload / 16 >= 0x80000000ULL) st = E_SHAPE;
    if (!st) {
        uint64_t off_scales = HEADER_BYTES;
        uint64_t off_tables = off_scales + pad16(2 * (uint64_t)M);
        uint64_t off_offsets = off_tables + pad16(tables_bytes(&m));
        uint64_t off_payload = off_offsets + pad16(4 * (T + 1));
        total = off_payload + payload;
        if (off_payload > 0xFFFFFFFFULL) st = E_SHAPE;
        else if (!(blob = (uint8_t*)calloc((size_t)total, 1))) st = E_NOMEM;
        if (!st) {
            memcpy(blob, "EPK1", 4);
            put_u16(blob + 4, prob_bits == PROB_BITS ? 1 : 2);
            blob[6] = (uint8_t)dtype;
            blob[7] = (uint8_t)r;
            put_u32(blob + 8, (uint32_t)M);
            put_u32(blob + 12, (uint32_t)N);
            put_u32(blob + 16, f32_to_bits(alpha));
            put_u16(blob + 20, (uint32_t)G);
            blob[22] = LANES;
            put_u32(blob + 24, (uint32_t)T);
            put_u32(blob + 28, (uint32_t)off_scales);
            put_u32(blob + 32, (uint32_t)off_tables);
            put_u32(blob + 36, (uint32_t)off_offsets);
            put_u32(blob + 40, (uint32_t)off_payload);
            put_u64(blob + 48, total);
            for (int64_t i = 0; i < M; i++) put_u16(blob + off_scales + 2 * i, t.sbits[i]);
            write_tables(&m, blob + off_tables);
            uint64_t pos = 0;
            for (uint64_t j = 0; j < T; j++) {
                put_u32(blob + off_offsets + 4 * j, (uint32_t)(pos / 16) | (tiles[j].has_esc ? 0x80000000u : 0));
                memcpy(blob + off_payload + pos, tiles[j].bytes, (size_t)tiles[j].size);
                pos += tiles[j].size;
            }
            put_u32(blob + off_offsets + 4 * T, (uint32_t)(pos / 16));
            put_u32(blob + 56, orc_crc32(blob, (size_t)off_payload));
        }
    }
    for (uint64_t j = 0; j < T; j++) free(tiles[j].bytes);
    free(tiles);
    free(groups);
    tensor_free(&t);
    if (st) { free(blob); return st; }
    *blob_out = blob;
    *bytes_out = (size_t)total;
    if (actual_bpp) *actual_bpp = 8.0 * (double)total / ((double)M * (double)N);
    return OK;
}

void orc_free(void* p) { free(p); }

/* ----------------------------------------------------------------- decoder */

typedef struct {
    int version, dtype, r, G;
    int64_t M, N, NG;
    float alpha;
    uint64_t T, off_scales, off_tables, off_offsets, off_payload, total;
    Model m;
} Blob;

static int parse_blob(const uint8_t* p, size_t bytes, Blob* b, int check_crc) {
    memset(b, 0, sizeof(*b));
    if (!p || bytes < HEADER_BYTES) return E_CORRUPT;
    if (memcmp(p, "EPK1", 4) != 0) return E_CORRUPT;
    b->version = (int)get_u16(p + 4);
    if (b->version != 1 && b->version != 2) return E_CORRUPT;
    b->dtype = p[6];
    b->r = p[7];
    b->M = get_u32(p + 8);
    b->N = get_u32(p + 12);
    b->alpha = bits_to_f32(get_u32(p + 16));
    b->G = (int)get_u16(p + 20);
    if (!elem_size(b->dtype)) return E_CORRUPT;
    if (b->r > 12 || p[22] != LANES || p[23] != 0) return E_CORRUPT;
    if (check_shape(b->dtype, b->M, b->N)) return E_CORRUPT;
    if (!(b->alpha > 0.0f) || !isfinite(b->alpha) || b->G < 1 || b->G > 1024) return E_CORRUPT;
    b->NG = b->M * b->N / 8;
    b->T = get_u32(p + 24);
    b->off_scales = get_u32(p + 28);
    b->off_tables = get_u32(p + 32);
    b->off_offsets = get_u32(p + 36);
    b->off_payload = get_u32(p + 40);
    b->total = get_u64(p + 48);
    if (b->T != num_tiles(b->NG, b->G) || b->total != bytes) return E_CORRUPT;
    if (b->off_scales != HEADER_BYTES || b->off_tables != b->off_scales + pad16(2 * (uint64_t)b->M))
        return E_CORRUPT;
    if (b->off_tables >= bytes) return E_CORRUPT;
    uint64_t used;
    if (read_tables(p + b->off_tables, bytes - b->off_tables, b->version == 1 ? PROB_BITS : PROB_BITS_V2, &b->m, &used))
        return E_CORRUPT;
    if (b->off_offsets != b->off_tables + pad16(used)) return E_CORRUPT;
    if (b->off_payload != b->off_offsets + pad16(4 * (b->T + 1)) || b->off_payload > bytes) return E_CORRUPT;
    uint64_t prev = 0;
    for (uint64_t j = 0; j <= b->T; j++) {
        uint32_t e = get_u32(p + b->off_offsets + 4 * j);
        uint64_t start = (uint64_t)(e & 0x7FFFFFFFu) * 16;
        if ((j == 0 && start != 0) || start < prev) return E_CORRUPT;
        if (j == b->T && ((e >> 31) || b->off_payload + start != bytes)) return E_CORRUPT;
        prev = start;
    }
    if (check_crc) {
        uint8_t* copy = (uint8_t*)malloc((size_t)b->off_payload);
        if (!copy) return E_NOMEM;
        memcpy(copy, p, (size_t)b->off_payload);
        memset(copy + 56, 0, 4);
        uint32_t crc = orc_crc32(copy, (size_t)b->off_payload);
        free(copy);
        if (crc != get_u32(p + 56)) return E_CORRUPT;
    }
    return OK;
}

int orc_blob_info(const uint8_t* blob, size_t bytes, int* dtype, int64_t* M, int64_t* N, float* alpha,
                  int* r, int* G, uint32_t* T, int* version) {
    Blob b;
    int st = parse_blob(blob, bytes, &b, 1);
    if (st) return st;
    if (version) *version = b.version;
    if (dtype) *dtype = b.dtype;
    if (M) *M = b.M;
    if (N) *N = b.N;
    if (alpha) *alpha = b.alpha;
    if (r) *r = b.r;
    if (G) *G = b.G;
    if (T) *T = (uint32_t)b.T;
    return OK;
}

/* Symbol whose slot range holds `slot`, by a linear scan; -1 if none. */
static int find_symbol(const Model* m, int c, uint32_t slot) {
    for (int s = m->lo[c]; s < m->lo[c] + m->cnt[c]; s++)
        if (m->f[c][s] && m->cum[c][s] <= slot && slot < m->cum[c][s] + m->f[c][s]) return s;
    return -1;
}

static void store_value(void* dst, int dtype, int64_t idx, float y) {
    int es = elem_size(dtype);
    orc_to_container(&y, 1, dtype, (uint8_t*)dst + idx * es);
}

static int decode_tile(const uint8_t* p, const Blob* b, uint64_t j, void* dst, int32_t* zout) {
    const Model* m = &b->m;
    uint64_t start = (uint64_t)(get_u32(p + b->off_offsets + 4 * j) & 0x7FFFFFFFu) * 16;
    uint64_t end = (uint64_t)(get_u32(p + b->off_offsets + 4 * (j + 1)) & 0x7FFFFFFFu) * 16;
    const uint8_t* tile = p + b->off_payload + start;
    uint64_t tile_bytes = end - start;
    int64_t g0 = (int64_t)j * 32 * b->G;
    int64_t ng = b->NG - g0 < 32LL * b->G ? b->NG - g0 : 32LL * b->G;
    int r = b->r;
    uint64_t raw = pad4((uint64_t)ng * (uint64_t)r);
    if (tile_bytes < 128 + raw) return E_CORRUPT;
    const uint8_t* rawp = tile + 128;
    const uint8_t* wp = tile + 128 + raw;
    uint64_t cap = (tile_bytes - 128 - raw) / 2, pos = 0;
    uint32_t x[LANES];
    for (int L = 0; L < LANES; L++) x[L] = get_u32(tile + 4 * L);
    int64_t gpr = b->N / 8, R = (ng + 31) / 32;

    for (int64_t k = 0; k < R; k++) {
        int b_of[LANES] = {0}, idx[LANES] = {0};
        int64_t t[LANES][8], hi_prev[LANES] = {0};
        for (int i = 0; i < 8; i++) {
            /* Symbol phase. */
            for (int L = 0; L < LANES; L++) {
                if (32 * k + L >= ng) continue;
                int c = context_of(i, hi_prev[L], b_of[L]);
                uint32_t slot = x[L] & (PROB_SCALE - 1);
                int s = find_symbol(m, c, slot);
                if (s < 0) return E_CORRUPT;
                x[L] = m->f[c][s] * (x[L] >> PROB_BITS) + slot - m->cum[c][s];
                if (i == 0) { b_of[L] = s >> 6; idx[L] = s & 63; }
                else idx[L] = s;
            }
            for (int L = 0; L < LANES; L++) {
                if (32 * k + L >= ng || x[L] >= RANS_L) continue;
                if (pos >= cap) return E_CORRUPT;
                x[L] = (x[L] << 16) | get_u16(wp + 2 * pos++);
            }
            /* ESC phase, then the raw low bits. */
            for (int L = 0; L < LANES; L++) {
                int64_t q = 32 * k + L;
                if (q >= ng) continue;
                int64_t hi;
                if (idx[L] == ESC_IDX) {
                    if (pos >= cap) return E_CORRUPT;
                    hi = (int16_t)get_u16(wp + 2 * pos++);
                } else {
                    hi = idx[L] - 31;
                }
                int64_t lo = 0;
                uint64_t bit = 8 * (uint64_t)r * (uint64_t)q + (uint64_t)(i * r);
                for (int kb = 0; kb < r; kb++, bit++) lo |= (int64_t)((rawp[bit >> 3] >> (bit & 7)) & 1) << kb;
                t[L][i] = hi * ((int64_t)1 << r) + lo;
                hi_prev[L] = hi;
            }
        }
        /* Algebraic inverse of the lattice map, then the per-row rescale. */
        for (int L = 0; L < LANES; L++) {
            int64_t q = 32 * k + L;
            if (q >= ng) continue;
            int64_t g = g0 + q, row = g / gpr, col = (g % gpr) * 8;
            int64_t u[8], s = 0;
            for (int i = 0; i < 7; i++) { u[i] = t[L][i]; s += u[i]; }
            u[7] = 2 * t[L][7] + (s & 1);
            float c_row = bf16_to_f32((uint16_t)get_u16(p + b->off_scales + 2 * row)) / b->alpha;
            for (int i = 0; i < 8; i++) {
                int64_t z = 2 * u[i] + b_of[L];
                float v = (float)z * 0.5f;
                float y = v * c_row;
                store_value(dst, b->dtype, row * b->N + col + i, y);
                if (zout) zout[row * b->N + col + i] = (int32_t)z;
            }
        }
    }
    for (int L = 0; L < LANES; L++) if (x[L] != RANS_L) return E_CORRUPT;
    if (pos > cap || cap - pos > 7) return E_CORRUPT;
    return OK;
}

/* Version 2 tile. Per round k, for each pair of positions (2p, 2p + 1): every lane decodes the two
 * symbols, the second in the context the first one's class gives (an escape has class 1), with
 * slot = x & 255 and x <- f (x >> 8) + slot - cum; then, in ascending lane order, every lane with
 * x < 2^16 reads one word: x <- (x << 16) | w. After the fourth pair come the round's escape words:
 * positions ascending, lanes ascending, one int16 hi each. The raw low bits, the inverse lattice map and
 * the rescale are those of version 1. */
static int decode_tile_v2(const uint8_t* p, const Blob* b, uint64_t j, void* dst, int32_t* zout) {
    const Model* m = &b->m;
    uint64_t start = (uint64_t)(get_u32(p + b->off_offsets + 4 * j) & 0x7FFFFFFFu) * 16;
    uint64_t end = (uint64_t)(get_u32(p + b->off_offsets + 4 * (j + 1)) & 0x7FFFFFFFu) * 16;
    const uint8_t* tile = p + b->off_payload + start;
    uint64_t tile_bytes = end - start;
    int64_t g0 = (int64_t)j * 32 * b->G;
    int64_t ng = b->NG - g0 < 32LL * b->G ? b->NG - g0 : 32LL * b->G;
    int r = b->r;
    uint64_t raw = pad4((uint64_t)ng * (uint64_t)r);
    if (tile_bytes < 128 + raw) return E_CORRUPT;
    const uint8_t* rawp = tile + 128;
    const uint8_t* wp = tile + 128 + raw;
    uint64_t cap = (tile_bytes - 128 - raw) / 2, pos = 0;
    uint32_t x[LANES];
    for (int L = 0; L < LANES; L++) x[L] = get_u32(tile + 4 * L);
    int64_t gpr = b->N / 8, R = (ng + 31) / 32;

    for (int64_t k = 0; k < R; k++) {
        int b_of[LANES] = {0}, idx[LANES][8], cls_prev[LANES] = {0};
        for (int pp = 0; pp < 4; pp++) {
            for (int i = 2 * pp; i <= 2 * pp + 1; i++) {
                for (int L = 0; L < LANES; L++) {
                    if (32 * k + L >= ng) continue;
                    int c = (i == 0) ? 0 : (i < 7 ? 1 : 5) + 2 * b_of[L] + cls_prev[L];
                    uint32_t slot = x[L] & (PROB_SCALE_V2 - 1);
                    int s = find_symbol(m, c, slot);
                    if (s < 0) return E_CORRUPT;
                    x[L] = m->f[c][s] * (x[L] >> PROB_BITS_V2) + slot - m->cum[c][s];
                    if (i == 0) b_of[L] = s >> 6;
                    idx[L][i] = s & 63;
                    cls_prev[L] = idx[L][i] == ESC_IDX ? 1 : mag_class(idx[L][i] - 31, b_of[L]);
                }
            }
            for (int L = 0; L < LANES; L++) {
                if (32 * k + L >= ng || x[L] >= RANS_L) continue;
                if (pos >= cap) return E_CORRUPT;
                x[L] = (x[L] << 16) | get_u16(wp + 2 * pos++);
            }
        }
        int64_t hi[LANES][8];
        for (int i = 0; i < 8; i++)
            for (int L = 0; L < LANES; L++) {
                if (32 * k + L >= ng) continue;
                if (idx[L][i] == ESC_IDX) {
                    if (pos >= cap) return E_CORRUPT;
                    hi[L][i] = (int16_t)get_u16(wp + 2 * pos++);
                } else {
                    hi[L][i] = idx[L][i] - 31;
                }
            }
        for (int L = 0; L < LANES; L++) {
            int64_t q = 32 * k + L;
            if (q >= ng) continue;
            int64_t t[8];
            for (int i = 0; i < 8; i++) {
                int64_t lo = 0;
                uint64_t bit = 8 * (uint64_t)r * (uint64_t)q + (uint64_t)(i * r);
                for (int kb = 0; kb < r; kb++, bit++) lo |= (int64_t)((rawp[bit >> 3] >> (bit & 7)) & 1) << kb;
                t[i] = hi[L][i] * ((int64_t)1 << r) + lo;
            }
            /* Algebraic inverse of the lattice map, then the per-row rescale. */
            int64_t g = g0 + q, row = g / gpr, col = (g % gpr) * 8;
            int64_t u[8], sum = 0;
            for (int i = 0; i < 7; i++) { u[i] = t[i]; sum += u[i]; }
            u[7] = 2 * t[7] + (sum & 1);
            float c_row = bf16_to_f32((uint16_t)get_u16(p + b->off_scales + 2 * row)) / b->alpha;
            for (int i = 0; i < 8; i++) {
                int64_t z = 2 * u[i] + b_of[L];
                float v = (float)z * 0.5f;
                float y = v * c_row;
                store_value(dst, b->dtype, row * b->N + col + i, y);
                if (zout) zout[row * b->N + col + i] = (int32_t)z;
            }
        }
    }
    for (int L = 0; L < LANES; L++) if (x[L] != RANS_L) return E_CORRUPT;
    if (pos > cap || cap - pos > 7) return E_CORRUPT;
    return OK;
}

int orc_decode_tiles(const uint8_t* blob, size_t bytes, uint32_t t0, uint32_t t1, void* dst, int32_t* zout) {
    Blob b;
    int st = parse_blob(blob, bytes, &b, 0);
    if (st) return st;
    if (t0 > t1 || t1 > b.T || !dst) return E_ARG;
    for (uint64_t j = t0; j < t1; j++)
        if ((st = (b.version == 1 ? decode_tile : decode_tile_v2)(blob, &b, j, dst, zout))) return st;
    return OK;
}

int orc_decompress(const uint8_t* blob, size_t bytes, void* dst, int32_t* zout) {
    Blob b;
    int st = parse_blob(blob, bytes, &b, 1);
    if (st) return st;
    return orc_decode_tiles(blob, bytes, 0, (uint32_t)b.T, dst, zout);
}
