/*
 * EntroPack oracle, lossless part — plain, slow CPU encoder and decoder of the EPL1 tile-ANS blob.
 *
 * TEST INFRASTRUCTURE, NOT PRODUCT CODE (see entropack_oracle.h). Built with the lossy oracle into
 * liboracle.so; the product library never links, loads or calls it.
 *
 * What it follows: the EntroPack README's Config table lists TileANSConfig(), lossless compression of
 * BF16, FP16, FP32, FP8 and INT8 tensors whose ratio depends on the data (README_zh page, section
 * Config), and its acknowledgements name tile-ANS as prior art. The pages give no format. The format
 * document's EPL1 part fixes one, which this file follows step by step: the raw bit patterns of the
 * elements are cut into byte planes; each plane is stored verbatim or rANS-coded under its own 12-bit
 * frequency table (the coder of lossy version 1), in tiles of 32 interleaved lanes.
 */
#include "entropack_oracle.h"

#include <math.h>
#include <stdlib.h>
#include <string.h>

enum { T_OK = 0, T_ARG = -1, T_DTYPE = -2, T_SHAPE = -3, T_CORRUPT = -6, T_NOMEM = -8 };

#define T_LANES 32
#define T_SCALE 4096u
#define T_RANS_L 65536u
#define T_HEADER 96
#define T_MAXDIM 8
#define T_DEFAULT_K 128

static uint64_t t_pad16(uint64_t n) { return (n + 15) & ~(uint64_t)15; }
static uint64_t t_pad4(uint64_t n) { return (n + 3) & ~(uint64_t)3; }
static void t_put16(uint8_t* p, uint32_t v) { p[0] = (uint8_t)v; p[1] = (uint8_t)(v >> 8); }
static void t_put32(uint8_t* p, uint32_t v) { for (int i = 0; i < 4; i++) p[i] = (uint8_t)(v >> (8 * i)); }
static void t_put64(uint8_t* p, uint64_t v) { for (int i = 0; i < 8; i++) p[i] = (uint8_t)(v >> (8 * i)); }
static uint32_t t_get16(const uint8_t* p) { return (uint32_t)p[0] | ((uint32_t)p[1] << 8); }
static uint32_t t_get32(const uint8_t* p) {
    return (uint32_t)p[0] | ((uint32_t)p[1] << 8) | ((uint32_t)p[2] << 16) | ((uint32_t)p[3] << 24);
}
static uint64_t t_get64(const uint8_t* p) { return (uint64_t)t_get32(p) | ((uint64_t)t_get32(p + 4) << 32); }

/* Bytes of one element: 2 for BF16 and FP16, 4 for FP32, 1 for FP8 e4m3 and INT8. */
static int t_elem(int dtype) {
    switch (dtype) {
        case 1: case 2: return 2;
        case 3: return 4;
        case 4: case 5: return 1;
    }
    return 0;
}

/* ------------------------------------------------------------ the model */

typedef struct {
    int e;                 /* bytes per element = number of byte planes */
    int coded[4];          /* plane j coded? */
    int lo[4], cnt[4];     /* table range of a coded plane */
    uint32_t f[4][256];    /* frequencies, indexed by byte value */
    uint32_t cum[4][257];  /* cumulative frequencies */
} TModel;

static void t_cum(TModel* m, int j) {
    m->cum[j][0] = 0;
    for (int s = 0; s < 256; s++) m->cum[j][s + 1] = m->cum[j][s] + m->f[j][s];
}

/* Format document, EPL1 part L5: counts per plane over the whole tensor, the lossy format's
 * normalisation at M = 4096, and the plane coded when its ideal coded size plus its table is at most
 * 7 bits per byte. */
static void t_fit(const uint8_t* data, uint64_t n, int e, TModel* m) {
    memset(m, 0, sizeof(*m));
    m->e = e;
    for (int j = 0; j < e; j++) {
        uint64_t counts[256] = {0};
        for (uint64_t i = 0; i < n; i++) counts[data[i * (uint64_t)e + (uint64_t)j]]++;
        orc_normalize_bits(counts, 256, 12, m->f[j]);
        if (n == 0) continue;
        int lo = 256, hi = -1;
        for (int s = 0; s < 256; s++)
            if (m->f[j][s]) {
                if (s < lo) lo = s;
                hi = s;
            }
        double bits = 8.0 * (4 + 2 * (hi - lo + 1));
        for (int s = 0; s < 256; s++)
            if (counts[s]) bits += (double)counts[s] * log2((double)T_SCALE / (double)m->f[j][s]);
        if (bits <= 7.0 * (double)n) {
            m->coded[j] = 1;
            m->lo[j] = lo;
            m->cnt[j] = hi - lo + 1;
            t_cum(m, j);
        }
    }
}

/* --------------------------------------------------------------- encoder */

typedef struct { uint16_t* w; size_t n, cap; } TWords;

static int t_push(TWords* ws, uint32_t v) {
    if (ws->n == ws->cap) {
        size_t cap = ws->cap ? 2 * ws->cap : 1024;
        uint16_t* p = (uint16_t*)realloc(ws->w, cap * sizeof(uint16_t));
        if (!p) return T_NOMEM;
        ws->w = p;
        ws->cap = cap;
    }
    ws->w[ws->n++] = (uint16_t)v;
    return T_OK;
}

/* One tile (elements [i0, i0 + ne)): the decode order of the format document run backwards, then the
 * layout: states, raw planes, the pushed words in reverse push order, zero padding to 16 bytes. */
static int t_encode_tile(const uint8_t* data, uint64_t i0, uint64_t ne, const TModel* m, uint8_t** out,
                         uint64_t* out_size) {
    const int e = m->e;
    int any = 0;
    for (int j = 0; j < e; j++) any |= m->coded[j];
    uint32_t x[T_LANES];
    for (int L = 0; L < T_LANES; L++) x[L] = T_RANS_L;
    TWords ws = {0, 0, 0};
    const int64_t R = (int64_t)((ne + 31) / 32);
    for (int64_t k = R - 1; k >= 0; k--) {
        for (int j = e - 1; j >= 0; j--) {
            if (!m->coded[j]) continue;
            for (int L = T_LANES - 1; L >= 0; L--) {
                const uint64_t i = 32 * (uint64_t)k + (uint64_t)L;
                if (i >= ne) continue;
                const int s = data[(i0 + i) * (uint64_t)e + (uint64_t)j];
                const uint32_t f = m->f[j][s], c = m->cum[j][s];
                if ((uint64_t)x[L] >= ((uint64_t)f << 20)) {
                    if (t_push(&ws, x[L] & 0xFFFFu)) { free(ws.w); return T_NOMEM; }
                    x[L] >>= 16;
                }
                x[L] = (x[L] / f) * T_SCALE + (x[L] % f) + c;
            }
        }
    }
    uint64_t size = any ? 128 : 0;
    for (int j = 0; j < e; j++)
        if (!m->coded[j]) size += t_pad4(ne);
    size = t_pad16(size + 2 * (uint64_t)ws.n);
    uint8_t* p = (uint8_t*)calloc(size ? (size_t)size : 1, 1);
    if (!p) { free(ws.w); return T_NOMEM; }
    uint64_t o = 0;
    if (any) {
        for (int L = 0; L < T_LANES; L++) t_put32(p + 4 * L, x[L]);
        o = 128;
    }
    for (int j = 0; j < e; j++) {
        if (m->coded[j]) continue;
        for (uint64_t i = 0; i < ne; i++) p[o + i] = data[(i0 + i) * (uint64_t)e + (uint64_t)j];
        o += t_pad4(ne);
    }
    for (size_t w = 0; w < ws.n; w++) t_put16(p + o + 2 * w, ws.w[ws.n - 1 - w]);
    free(ws.w);
    *out = p;
    *out_size = size;
    return T_OK;
}

int orc_tans_compress(const void* data, int dtype, int ndim, const int64_t* dims, int K, uint8_t** blob,
                      size_t* bytes) {
    if (!blob || !bytes || ndim < 0 || ndim > T_MAXDIM || (ndim > 0 && !dims)) return T_ARG;
    const int e = t_elem(dtype);
    if (!e) return T_DTYPE;
    if (K == 0) K = T_DEFAULT_K;
    if (K < 1 || K > 1024) return T_ARG;
    uint64_t n = 1;
    for (int d = 0; d < ndim; d++) {
        if (dims[d] < 0 || dims[d] > 0xFFFFFFFFLL) return T_SHAPE;
        n *= (uint64_t)dims[d];
    }
    if (n && !data) return T_ARG;
    const uint8_t* src = (const uint8_t*)data;
    TModel m;
    t_fit(src, n, e, &m);
    const uint64_t per_tile = 32 * (uint64_t)K;
    const uint64_t T = (n + per_tile - 1) / per_tile;
    if (T > 0xFFFFFFFFull) return T_SHAPE;

    uint64_t tables = 0;
    for (int j = 0; j < e; j++)
        if (m.coded[j]) tables += 4 + 2 * (uint64_t)m.cnt[j];
    const uint64_t off_tables = T_HEADER;
    const uint64_t off_offsets = t_pad16(off_tables + tables);
    const uint64_t off_payload = t_pad16(off_offsets + 4 * (T + 1));

    uint8_t** tiles = (uint8_t**)calloc(T ? (size_t)T : 1, sizeof(uint8_t*));
    uint64_t* sizes = (uint64_t*)calloc(T ? (size_t)T : 1, sizeof(uint64_t));
    if (!tiles || !sizes) { free(tiles); free(sizes); return T_NOMEM; }
    int st = T_OK;
    uint64_t payload = 0;
    for (uint64_t t = 0; t < T && st == T_OK; t++) {
        const uint64_t i0 = t * per_tile, ne = n - i0 < per_tile ? n - i0 : per_tile;
        st = t_encode_tile(src, i0, ne, &m, &tiles[t], &sizes[t]);
        payload += sizes[t];
    }
    if (st == T_OK && (payload / 16 > 0x7FFFFFFFull || off_payload > 0xFFFFFFFFull)) st = T_SHAPE;
    uint8_t* p = NULL;
    const uint64_t total = off_payload + payload;
    if (st == T_OK) {
        p = (uint8_t*)calloc((size_t)total, 1);
        if (!p) st = T_NOMEM;
    }
    if (st == T_OK) {
        memcpy(p, "EPL1", 4);
        t_put16(p + 4, 1);
        p[6] = (uint8_t)dtype;
        p[7] = (uint8_t)ndim;
        t_put64(p + 8, n);
        for (int d = 0; d < ndim; d++) t_put32(p + 16 + 4 * d, (uint32_t)dims[d]);
        t_put16(p + 48, (uint32_t)K);
        uint32_t mask = 0;
        for (int j = 0; j < e; j++) mask |= (uint32_t)m.coded[j] << j;
        p[50] = (uint8_t)mask;
        p[51] = T_LANES;
        t_put32(p + 52, (uint32_t)T);
        t_put32(p + 56, (uint32_t)off_tables);
        t_put32(p + 60, (uint32_t)off_offsets);
        t_put32(p + 64, (uint32_t)off_payload);
        t_put64(p + 72, total);
        uint64_t o = off_tables;
        for (int j = 0; j < e; j++) {
            if (!m.coded[j]) continue;
            t_put16(p + o, (uint32_t)m.lo[j]);
            t_put16(p + o + 2, (uint32_t)m.cnt[j]);
            for (int s = 0; s < m.cnt[j]; s++) t_put16(p + o + 4 + 2 * s, m.f[j][m.lo[j] + s]);
            o += 4 + 2 * (uint64_t)m.cnt[j];
        }
        uint64_t at = 0;
        for (uint64_t t = 0; t < T; t++) {
            t_put32(p + off_offsets + 4 * t, (uint32_t)(at / 16));
            memcpy(p + off_payload + at, tiles[t], (size_t)sizes[t]);
            at += sizes[t];
        }
        t_put32(p + off_offsets + 4 * T, (uint32_t)(at / 16));
        t_put32(p + 80, orc_crc32(p, (size_t)off_payload));  /* the crc field is still zero here */
    }
    for (uint64_t t = 0; t < T; t++) free(tiles[t]);
    free(tiles);
    free(sizes);
    if (st != T_OK) { free(p); return st; }
    *blob = p;
    *bytes = (size_t)total;
    return T_OK;
}

/* --------------------------------------------------------------- decoder */

typedef struct {
    int dtype, e, ndim, K, mask;
    uint64_t n, T;
    int64_t dims[T_MAXDIM];
    TModel m;
    const uint8_t* offsets;
    const uint8_t* payload;
    uint64_t payload_bytes;
} TBlob;

static int t_parse(const uint8_t* p, size_t bytes, TBlob* b) {
    memset(b, 0, sizeof(*b));
    if (!p || bytes < T_HEADER || memcmp(p, "EPL1", 4) != 0 || t_get16(p + 4) != 1) return T_CORRUPT;
    b->dtype = p[6];
    b->e = t_elem(b->dtype);
    b->ndim = p[7];
    if (!b->e || b->ndim > T_MAXDIM || p[51] != T_LANES) return T_CORRUPT;
    b->n = t_get64(p + 8);
    uint64_t prod = 1;
    for (int d = 0; d < T_MAXDIM; d++) {
        const uint32_t v = t_get32(p + 16 + 4 * d);
        if (d < b->ndim) {
            b->dims[d] = v;
            prod *= v;
        } else if (v != 0) {
            return T_CORRUPT;
        }
    }
    if (prod != b->n) return T_CORRUPT;
    b->K = (int)t_get16(p + 48);
    b->mask = p[50];
    if (b->K < 1 || b->K > 1024 || (b->mask >> b->e) != 0) return T_CORRUPT;
    b->T = t_get32(p + 52);
    const uint64_t per_tile = 32 * (uint64_t)b->K;
    if (b->T != (b->n + per_tile - 1) / per_tile) return T_CORRUPT;
    const uint64_t off_tables = t_get32(p + 56), off_offsets = t_get32(p + 60), off_payload = t_get32(p + 64);
    const uint64_t total = t_get64(p + 72);
    if (total != bytes || off_tables != T_HEADER || off_offsets < off_tables || off_offsets % 16 ||
        off_payload % 16 || off_payload < off_offsets + 4 * (b->T + 1) || off_payload > bytes)
        return T_CORRUPT;
    /* CRC over [0, off_payload) with the crc field zero. */
    uint8_t* tmp = (uint8_t*)malloc((size_t)off_payload);
    if (!tmp) return T_NOMEM;
    memcpy(tmp, p, (size_t)off_payload);
    memset(tmp + 80, 0, 4);
    const uint32_t crc = orc_crc32(tmp, (size_t)off_payload);
    free(tmp);
    if (crc != t_get32(p + 80)) return T_CORRUPT;
    /* Tables. */
    b->m.e = b->e;
    uint64_t o = off_tables;
    for (int j = 0; j < b->e; j++) {
        if (!((b->mask >> j) & 1)) continue;
        if (o + 4 > off_offsets) return T_CORRUPT;
        const int lo = (int)t_get16(p + o), cnt = (int)t_get16(p + o + 2);
        if (cnt < 2 || lo + cnt > 256 || o + 4 + 2 * (uint64_t)cnt > off_offsets) return T_CORRUPT;
        uint32_t sum = 0;
        for (int s = 0; s < cnt; s++) {
            const uint32_t f = t_get16(p + o + 4 + 2 * s);
            if (f >= T_SCALE) return T_CORRUPT;
            b->m.f[j][lo + s] = f;
            sum += f;
        }
        if (sum != T_SCALE) return T_CORRUPT;
        b->m.coded[j] = 1;
        b->m.lo[j] = lo;
        b->m.cnt[j] = cnt;
        t_cum(&b->m, j);
        o += 4 + 2 * (uint64_t)cnt;
    }
    b->offsets = p + off_offsets;
    b->payload = p + off_payload;
    b->payload_bytes = bytes - off_payload;
    if (t_get32(b->offsets) != 0 || 16 * (uint64_t)t_get32(b->offsets + 4 * b->T) != b->payload_bytes) return T_CORRUPT;
    for (uint64_t t = 0; t < b->T; t++)
        if (t_get32(b->offsets + 4 * (t + 1)) < t_get32(b->offsets + 4 * t)) return T_CORRUPT;
    return T_OK;
}

/* One tile, in the decode order of the format document. */
static int t_decode_tile(const TBlob* b, uint64_t t, uint8_t* dst) {
    const int e = b->e;
    const uint64_t per_tile = 32 * (uint64_t)b->K;
    const uint64_t i0 = t * per_tile, ne = b->n - i0 < per_tile ? b->n - i0 : per_tile;
    const uint64_t start = 16 * (uint64_t)t_get32(b->offsets + 4 * t), end = 16 * (uint64_t)t_get32(b->offsets + 4 * (t + 1));
    const uint8_t* tp = b->payload + start;
    const uint64_t size = end - start;
    int any = 0;
    for (int j = 0; j < e; j++) any |= b->m.coded[j];
    uint64_t o = any ? 128 : 0;
    for (int j = 0; j < e; j++) {
        if (b->m.coded[j]) continue;
        if (o + t_pad4(ne) > size) return T_CORRUPT;
        for (uint64_t i = 0; i < ne; i++) dst[(i0 + i) * (uint64_t)e + (uint64_t)j] = tp[o + i];
        o += t_pad4(ne);
    }
    if (!any) return size == t_pad16(o) ? T_OK : T_CORRUPT;
    if (size < o) return T_CORRUPT;
    const uint8_t* words = tp + o;
    const uint64_t cap = (size - o) / 2;
    uint32_t x[T_LANES];
    for (int L = 0; L < T_LANES; L++) x[L] = t_get32(tp + 4 * L);
    uint64_t pw = 0;
    const uint64_t R = (ne + 31) / 32;
    for (uint64_t k = 0; k < R; k++) {
        for (int j = 0; j < e; j++) {
            if (!b->m.coded[j]) continue;
            for (int L = 0; L < T_LANES; L++) {
                const uint64_t i = 32 * k + (uint64_t)L;
                if (i >= ne) continue;
                const uint32_t slot = x[L] & (T_SCALE - 1);
                int s = 0;
                while (!(b->m.cum[j][s] <= slot && slot < b->m.cum[j][s + 1])) s++;  /* the owner of slot */
                x[L] = b->m.f[j][s] * (x[L] >> 12) + slot - b->m.cum[j][s];
                dst[(i0 + i) * (uint64_t)e + (uint64_t)j] = (uint8_t)s;
            }
            for (int L = 0; L < T_LANES; L++) {
                const uint64_t i = 32 * k + (uint64_t)L;
                if (i >= ne || x[L] >= T_RANS_L) continue;
                if (pw >= cap) return T_CORRUPT;
                x[L] = (x[L] << 16) | t_get16(words + 2 * pw);
                pw++;
            }
        }
    }
    for (int L = 0; L < T_LANES; L++)
        if (x[L] != T_RANS_L) return T_CORRUPT;
    return (cap - pw <= 7) ? T_OK : T_CORRUPT;
}

int orc_tans_info(const uint8_t* blob, size_t bytes, int* dtype, int* ndim, int64_t* dims, int* K, uint32_t* T,
                  int* coded_mask) {
    TBlob b;
    const int st = t_parse(blob, bytes, &b);
    if (st) return st;
    if (dtype) *dtype = b.dtype;
    if (ndim) *ndim = b.ndim;
    if (dims) for (int d = 0; d < b.ndim; d++) dims[d] = b.dims[d];
    if (K) *K = b.K;
    if (T) *T = (uint32_t)b.T;
    if (coded_mask) *coded_mask = b.mask;
    return T_OK;
}

int orc_tans_decode_tiles(const uint8_t* blob, size_t bytes, uint32_t t0, uint32_t t1, void* dst) {
    TBlob b;
    const int st = t_parse(blob, bytes, &b);
    if (st) return st;
    if (t0 > t1 || t1 > b.T || (b.n && !dst)) return T_ARG;
    for (uint64_t t = t0; t < t1; t++) {
        const int r = t_decode_tile(&b, t, (uint8_t*)dst);
        if (r) return r;
    }
    return T_OK;
}

int orc_tans_decompress(const uint8_t* blob, size_t bytes, void* dst) {
    TBlob b;
    const int st = t_parse(blob, bytes, &b);
    if (st) return st;
    return orc_tans_decode_tiles(blob, bytes, 0, (uint32_t)b.T, dst);
}
