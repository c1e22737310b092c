/*
 * EntroPack oracle — plain, slow CPU encoders and decoders of the EPK1 (lossy) and EPL1 (lossless
 * tile-ANS) blobs.
 *
 * TEST INFRASTRUCTURE, NOT PRODUCT CODE. The test suite, the smoke check and
 * the benchmark's CPU-baseline leg are its only users; the product library
 * never links, loads or calls it and shares no source, header or table with
 * it. It is written for a reader checking it against the EntroPack pages
 * (arXiv 2609.34185, "EntroPack: Fast and Accurate Entropy-Coded Weight
 * Compression at Arbitrary Bitrates"), not for speed.
 *
 * Status codes: 0 ok, -1 bad argument, -2 bad dtype, -3 bad shape, -4 target
 * out of range, -5 non-finite input, -6 corrupt blob, -8 out of memory.
 * Container dtypes: 1 BF16, 2 FP16, 3 FP32, 4 FP8 e4m3, 5 INT8.
 */
#ifndef ENTROPACK_ORACLE_H
#define ENTROPACK_ORACLE_H
#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* CRC-32 (IEEE 802.3, reflected, polynomial 0xEDB88320). */
uint32_t orc_crc32(const uint8_t* p, size_t n);

/* Nearest E8 point to x[8]: writes the coset bit b and u[8] (v = u + b/2). */
void orc_e8_nearest(const double* x, int32_t* b, int64_t* u);

/* 12-bit normalisation of n <= 128 symbol counts into f[n]; returns 0. */
int orc_normalize(const uint64_t* counts, int n, uint32_t* f);
/* The same at `bits` = 12 (version 1) or 8 (version 2); -1 for any other precision. */
int orc_normalize_bits(const uint64_t* counts, int n, int bits, uint32_t* f);

/* Container conversions (n elements). from_container returns -5 on NaN/Inf. */
void orc_to_container(const float* y, int64_t n, int dtype, void* out);
int orc_from_container(const void* in, int64_t n, int dtype, float* out);

/* Lossy compression of a row-major M x N container tensor. G = rounds per
 * tile. force_alpha > 0 skips rate control and uses that resolution.
 * prob_bits = 12 writes format version 1, 8 writes version 2. The blob is
 * malloc'd; release it with orc_free. */
int orc_compress(const void* data, int dtype, int64_t M, int64_t N, double target_bpp, int G,
                 double force_alpha, int prob_bits, uint8_t** blob, size_t* bytes, double* actual_bpp);
void orc_free(void* p);

/* Sampled storage estimate, in bytes, of coding the tensor at resolution alpha. */
double orc_estimate_bytes(const void* data, int dtype, int64_t M, int64_t N, int G, float alpha, int prob_bits);

/* Full validation (header, sections, tables, CRC) and header fields. */
int orc_blob_info(const uint8_t* blob, size_t bytes, int* dtype, int64_t* M, int64_t* N,
                  float* alpha, int* r, int* G, uint32_t* T, int* version);

/* Decode tiles [t0, t1) into dst (the full M x N container buffer; only the
 * tiles' groups are written). zout, if not NULL, receives z = 2v (int32) for
 * every decoded coordinate at its row-major index. */
int orc_decode_tiles(const uint8_t* blob, size_t bytes, uint32_t t0, uint32_t t1, void* dst,
                     int32_t* zout);

/* Decode the whole tensor (all tiles). */
int orc_decompress(const uint8_t* blob, size_t bytes, void* dst, int32_t* zout);

/* Quantise the tensor at resolution alpha: zout[M*N] = 2v of the chosen E8
 * point per coordinate, scales_out[M] = bf16 bits of s_row. */
int orc_quantize(const void* data, int dtype, int64_t M, int64_t N, float alpha, int32_t* zout,
                 uint16_t* scales_out);

/* Lossless tile-ANS (EPL1 blob, tileans_oracle.c). data: numel = prod(dims) elements of the dtype's
 * size, read as raw bit patterns; ndim 0..8 (ndim 0 is one element). K: elements per lane per tile,
 * 1..1024, or 0 for 128. The blob is malloc'd; release it with orc_free. */
int orc_tans_compress(const void* data, int dtype, int ndim, const int64_t* dims, int K, uint8_t** blob,
                      size_t* bytes);
/* Full validation (header, tables, offsets, CRC) and the header fields; dims receives ndim values. */
int orc_tans_info(const uint8_t* blob, size_t bytes, int* dtype, int* ndim, int64_t* dims, int* K, uint32_t* T,
                  int* coded_mask);
/* Decode tiles [t0, t1) into dst (the whole tensor's buffer; only those tiles' elements are written). */
int orc_tans_decode_tiles(const uint8_t* blob, size_t bytes, uint32_t t0, uint32_t t1, void* dst);
/* Decode every tile. */
int orc_tans_decompress(const uint8_t* blob, size_t bytes, void* dst);

#ifdef __cplusplus
}
#endif
#endif
