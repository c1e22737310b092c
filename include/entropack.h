/*
 * entropack.h: the C ABI of libentropack, a B200-native (sm_100a) EntroPack codec.
 *
 * EntroPack (arXiv 2609.34185, "EntroPack: Fast and Accurate Entropy-Coded Weight Compression at
 * Arbitrary Bitrates") compresses a 2-D weight matrix at any target bits per parameter. It
 * normalises each row, quantises 8-wide groups to the E8 lattice at one global resolution alpha,
 * and rANS-codes the lattice coordinates under a conditional model. The coded coordinates sit in
 * independently decodable tiles. (Paper page abstract; modelscope summary.)
 *
 * Decode is the hot path. One sm_100a kernel turns the tiles back into a dense matrix in the
 * requested container. It runs symbol decode, the arithmetic inverse of the lattice map and the
 * per-row rescale by s_row/alpha as one fused pass, with no symbol tensor and no codebook in
 * between (modelscope summary). The Python API of the pages is compress(tensor, config) ->
 * object with actual_bpp, and decompress(object) -> tensor of the same shape and dtype
 * (README, quick-start section). This header is the same interface as plain C.
 *
 * Conventions:
 *   - Every call returns an ep_status. Nothing throws. Out-parameters are written only on EP_OK.
 *     ep_last_error() gives a thread-local message for the last failure.
 *   - Layout: row-major, shape (rows, cols). A group is 8 consecutive columns of one row, so cols
 *     must be a multiple of 8 (EP_ERR_SHAPE otherwise).
 *   - Blob: a flat little-endian byte string (format "EPK1"). It describes itself fully, so it can
 *     be stored as it is, for example as a uint8 tensor in a state_dict.
 *   - Ownership: the library owns the blob returned by ep_compress until ep_blob_free. The caller
 *     owns every device buffer and every stream. Decode calls are asynchronous on the caller's
 *     stream.
 *   - Threads: every call is thread-safe. Decode calls on different streams may run concurrently.
 */
#ifndef ENTROPACK_H
#define ENTROPACK_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Container dtypes, for the input of ep_compress and the output of decode. Storage bitrate is
 * independent of the container (paper page abstract). */
typedef enum {
    EP_BF16 = 1,
    EP_FP16 = 2,
    EP_FP32 = 3,
    EP_FP8_E4M3 = 4, /* OCP e4m3; decode saturates to +-448 */
    EP_INT8 = 5      /* decode rounds half to even, then clamps to [-128, 127] */
} ep_dtype;

typedef enum {
    EP_OK = 0,
    EP_ERR_ARG = -1,       /* NULL pointer, bad option, or value range too wide to code */
    EP_ERR_DTYPE = -2,     /* unknown container dtype */
    EP_ERR_SHAPE = -3,     /* not 2-D with rows >= 1, cols >= 8, cols % 8 == 0, or too large */
    EP_ERR_TARGET = -4,    /* target_bpp not finite or outside [0.001, 11] (README, Config table) */
    EP_ERR_NONFINITE = -5, /* NaN or Inf in the input */
    EP_ERR_CORRUPT = -6,   /* malformed blob, caught on the host */
    EP_ERR_CUDA = -7,      /* a CUDA runtime call failed; ep_last_error() names it */
    EP_ERR_NOMEM = -8,     /* host or device allocation failed */
    EP_ERR_BUFFER = -9     /* destination too small or misaligned, or blob shorter than its header says */
} ep_status;

/* Bits of the device status word: set by the decode kernel, read by ep_get_device_status. */
#define EP_DEV_CORRUPT_TILE 1u  /* a tile's final rANS states or its word count did not check out */
#define EP_DEV_BAD_OFFSETS 2u   /* a tile offset points outside the payload */
#define EP_DEV_BAD_TABLES 4u    /* a frequency table does not sum to its scale (4096 in version 1, 256 in 2) */
#define EP_DEV_TABLE_COPY 8u    /* a sequence's prepared tables did not reach a CTA in time; in version 1 it
                                   decoded nothing, in version 2 it decoded with whatever the window held */
#define EP_DEV_DEP_WAIT 16u     /* in a version-2 sequence, a tile waited too long for an earlier layer's tile
                                   that writes the same bytes, and stored without it */

/* Encoder options. Start from ep_options_default(). */
typedef struct {
    uint32_t rounds_per_tile; /* G: a tile holds 32 * G * 8 coordinates. Range 1..1024, or 0 (the default)
                                 for automatic: 16 (4096 coordinates) unless the tensor fills at least half a
                                 wave of 16-round tiles on a 148-SM B200 (148 x 32 warps). It then takes the
                                 G in [12, 24] that fills whole waves, which spares the decode a
                                 near-empty last wave. */
    uint32_t sample_coords;   /* rate-control sample: about this many coordinates of whole rows. Default 2^18 */
    uint32_t bisection_iters; /* bisection steps on log2(alpha). Default 40 */
    int32_t threads;          /* encoder threads; 0 = all hardware threads */
    uint32_t format_version;  /* 2 (the default; 0 also means 2): 8-bit frequency tables, the rANS state
                                 renormalised once per pair of symbols, rare symbols sent as escapes. 1:
                                 12-bit frequency tables, the state renormalised after every symbol. Both
                                 decode with the same calls; version 2 decodes faster on B200 at a
                                 slightly higher error for the same storage. */
} ep_options;

void ep_options_default(ep_options* opt);

/*
 * ep_compress: lossy compression of one 2-D tensor to a blob.
 *
 * data        rows x cols elements of container dtype dt; row i starts at element i*row_stride.
 *             is_device != 0 means a CUDA device pointer, which is copied to the host once.
 * target_bpp  target storage in bits per parameter, metadata included. Must be finite and in
 *             [0.001, 11] (README, quick-start section and Config table). The resolution is chosen
 *             by bisection on log2(alpha), against a storage estimate taken from a sample of rows.
 *             The full tensor is never encoded twice (paper page abstract). Below the metadata floor
 *             the smallest alpha is used, and *actual_bpp is reported above the target.
 * opt         NULL means the defaults.
 * blob        receives a malloc'd buffer, released by ep_blob_free; *blob_bytes is its size.
 * actual_bpp  8 * blob_bytes / (rows * cols), metadata included (README, quick-start section).
 * Errors: EP_ERR_ARG, EP_ERR_DTYPE, EP_ERR_SHAPE, EP_ERR_TARGET, EP_ERR_NONFINITE, EP_ERR_NOMEM,
 *         EP_ERR_CUDA (device input).
 */
ep_status ep_compress(const void* data, int is_device, ep_dtype dt, int64_t rows, int64_t cols,
                      int64_t row_stride, double target_bpp, const ep_options* opt, uint8_t** blob,
                      size_t* blob_bytes, double* actual_bpp);

/*
 * ep_compress_cuda: the same compression run on the GPU, for a tensor already in device memory. It
 * writes the same blob bytes as ep_compress for the same input and options: row scales, every probe
 * of the rate-control bisection, the quantisation and the rANS tiles run as kernels, and the host
 * fits the 12-bit tables and takes the storage estimate with the host encoder's code (paper page
 * abstract: sampled storage estimates, independently decodable tiles).
 *
 * dev_data    CUDA device pointer to rows x cols elements of dtype dt; row i starts at element
 *             i*row_stride. Read only.
 * cuda_stream cudaStream_t for every kernel and copy; NULL means the legacy default stream. The call
 *             synchronises this stream several times and returns when the blob is complete.
 * opt         NULL means the defaults; opt->threads is ignored.
 * Other arguments and the ownership of *blob as for ep_compress (release with ep_blob_free).
 * Device scratch (about 10 bytes per parameter) comes stream-ordered from a memory pool that the
 * library creates per device. Each call frees its scratch before it returns. The pool keeps up to
 * 1 GiB of freed scratch mapped for the next call, and releases the rest.
 * Errors: as ep_compress; EP_ERR_ARG also when dev_data is not device memory; EP_ERR_CUDA for a failed
 *         allocation, launch or copy.
 */
ep_status ep_compress_cuda(const void* dev_data, ep_dtype dt, int64_t rows, int64_t cols, int64_t row_stride,
                           double target_bpp, const ep_options* opt, void* cuda_stream, uint8_t** blob,
                           size_t* blob_bytes, double* actual_bpp);

/*
 * ep_compress_cuda_noalloc: ep_compress_cuda with no device allocation. The pages have no counterpart
 * to this entry point: it exists for callers that must not allocate device memory (no cudaMalloc,
 * cudaMallocAsync, cudaFree or cudaFreeAsync happens in it). It runs the same kernels and writes the
 * same blob bytes as ep_compress_cuda.
 *
 * Scratch     every device buffer is carved from one fixed 64 MiB array in device memory (a static
 *             __device__ array of the library, one per device, reserved when the encoder's kernels are
 *             first loaded). That bounds the tensor to about 4.5 M parameters (for example 2048 x 2048);
 *             a larger request is rejected with EP_ERR_ARG before any work. Counters and the payload
 *             area are zeroed by each call.
 * blob        caller-owned host buffer of blob_capacity bytes; the blob is written there and *blob_bytes
 *             receives its size. 8*rows*cols + 2*rows + 4096 bytes always suffice; a smaller buffer that
 *             cannot hold the blob gives EP_ERR_BUFFER.
 * Set-up      the first call on a device looks up the array's device address (cudaGetSymbolAddress) with
 *             that device current, and keeps it for later calls. Make that first call before any stream
 *             capture. A cudaDeviceReset discards the array with the context; calls after one are not
 *             supported. dev_data must be on the current device (EP_ERR_ARG otherwise).
 * Races       the array is shared by every call on a device in the process, and keeps the last call's
 *             contents. Calls on one device are serialised by a lock held for the whole call, and once
 *             a call has queued work it synchronises cuda_stream before it returns, on error paths too,
 *             so no two calls of this library use the array at once. Other processes have their own array.
 * Other arguments and errors as ep_compress_cuda.
 */
ep_status ep_compress_cuda_noalloc(const void* dev_data, ep_dtype dt, int64_t rows, int64_t cols, int64_t row_stride,
                                   double target_bpp, const ep_options* opt, void* cuda_stream, uint8_t* blob,
                                   size_t blob_capacity, size_t* blob_bytes, double* actual_bpp);

/*
 * ep_plan_bitrates: per-layer targets for a set of tensors that share one storage budget.
 *
 * The EntroPack README ("Pre-quantised models") describes packs whose bitrate is allocated layer by
 * layer by sensitivity, at 2.3 to 3.0 bits per parameter on average; it does not give the rule. This
 * function implements the high-rate allocation: layer i, coded at a data rate of R bits per
 * parameter, is taken to have a squared weight error proportional to weight[i] * 2^(-2R). It returns
 * the bpp_out[i] (whole-blob bits per parameter, as ep_compress takes them) that minimise
 *     sum_i rows[i]*cols[i] * weight[i] * 2^(-2 (bpp_out[i] - meta_i))
 * subject to sum_i rows[i]*cols[i]*bpp_out[i] = mean_bpp * sum_i rows[i]*cols[i] and
 * max(min_bpp, meta_i) <= bpp_out[i] <= max_bpp. meta_i is layer i's metadata in bits per parameter
 * (header, row scales, the largest possible tables section, tile offsets and the per-tile state cost
 * of the encoders' storage estimate, at the tile size opt gives or the encoders' automatic one).
 * The solution has one water level theta: bpp_out[i] = clamp(meta_i + log2(weight[i])/2 + theta).
 *
 * n           number of layers, >= 1. rows, cols, weight: host arrays of n entries; bpp_out receives n.
 * weight      > 0 and finite: the cost of a unit of mean squared error in layer i, in the units the
 *             caller cares about. For an error in the weights' own units use sensitivity times the
 *             layer's mean square weight (the encoders normalise each row, so the error of a layer
 *             scales with its mean square).
 * opt         may be NULL; only rounds_per_tile is read (0 = the encoders' automatic choice).
 *
 * Budgets below every layer's floor give each layer its floor (the blobs then overshoot, as
 * ep_compress does for a target below the metadata); budgets above every ceiling give each max_bpp.
 * Pure host arithmetic: no device, no allocation visible to the caller.
 * Errors: EP_ERR_ARG (NULL, n < 1, a weight not finite and > 0, rounds_per_tile > 1024),
 * EP_ERR_SHAPE (a layer that ep_compress would reject), EP_ERR_TARGET (a bound outside [0.001, 11],
 * min_bpp > max_bpp or mean_bpp > max_bpp). bpp_out is written only on EP_OK.
 */
ep_status ep_plan_bitrates(int64_t n, const int64_t* rows, const int64_t* cols, const double* weight,
                           double mean_bpp, double min_bpp, double max_bpp, const ep_options* opt,
                           double* bpp_out);

/* Releases a blob returned by ep_compress or ep_compress_cuda. NULL is accepted. */
void ep_blob_free(uint8_t* blob);

/*
 * ep_blob_info: full host-side validation of a blob, then its description.
 * Checks the header, the section layout, the frequency tables, the tile offsets and the CRC-32 of
 * the metadata. Every out-pointer may be NULL. Errors: EP_ERR_ARG, EP_ERR_CORRUPT.
 */
ep_status ep_blob_info(const uint8_t* blob, size_t blob_bytes, ep_dtype* dt, int64_t* rows, int64_t* cols,
                       double* actual_bpp);

/*
 * ep_decompress_into: fused decode of a blob into a caller-owned device buffer. This is the hot path.
 *
 * host_hdr    host copy of at least the first 64 bytes of the blob (the header). The launch geometry
 *             comes from it, with no device-to-host traffic.
 * dev_blob    device copy of the whole blob, 16-byte aligned, blob_bytes long. Caller-owned, and
 *             read only.
 * dst         device buffer of rows*cols elements of the blob's container dtype, 16-byte aligned,
 *             row-major. dst_bytes is its size. Only those rows*cols elements are written.
 * cuda_stream cudaStream_t to launch on; NULL means the legacy default stream.
 *
 * The call validates the header on the host, launches one kernel and returns. It allocates nothing
 * and does not synchronise. Host-detectable errors come back at once: EP_ERR_ARG, EP_ERR_CORRUPT
 * (bad header), EP_ERR_BUFFER (dst too small or misaligned, blob_bytes too short), EP_ERR_CUDA
 * (launch failure). Payload corruption is found by the kernel itself: it checks every tile's final
 * rANS states and word count, and bounds every read to the tile. It then sets bits of the device
 * status word (see ep_get_device_status) instead of faulting. A corrupt tile's outputs are
 * unspecified.
 */
ep_status ep_decompress_into(const uint8_t* host_hdr, const void* dev_blob, size_t blob_bytes, void* dst,
                             size_t dst_bytes, void* cuda_stream);

/*
 * ep_decompress_many: decodes `count` blobs in order on one stream: blob i into dsts[i], with the
 * argument rules of ep_decompress_into for each one. This is the layer-sequence form of the hot
 * path, for example all linear layers of a model before a forward pass. Overlapping dsts end as if
 * the blobs were decoded one after another in list order. One requirement follows from reads made
 * while earlier decodes run: no blob in the list may be written by the decodes listed before it.
 * Every header, size and alignment is checked before anything launches, so an error launches nothing.
 *
 * Two or more format-version-2 blobs of one container dtype (the usual case) take the sequence path:
 * per group of up to 280 blobs, a table kernel builds every blob's fused tables (9 KB each) into
 * device scratch, then one persistent kernel (one CTA per SM, launched cooperatively, so all of them
 * are resident at once) decodes the whole group. The tiles of all the blobs are dealt round-robin as
 * one list, so a small layer shares the GPU with the next one, and each CTA keeps four blobs' tables in
 * shared memory, refilled by bulk copies (TMA, no multicast). When some dst overlaps an earlier one,
 * each tile waits, before its first store, for the tiles of earlier blobs that last wrote the same
 * bytes (per-tile done flags in the scratch, with release and acquire ordering); the waits are bounded
 * and set EP_DEV_DEP_WAIT if they run out, and a window copy that does not land in time sets
 * EP_DEV_TABLE_COPY. The scratch (9 KB per blob plus a bit per tile) comes stream-ordered from a pool
 * the library keeps per device and is released stream-ordered after the group; if it cannot be had,
 * the call returns EP_ERR_NOMEM with nothing of that group launched (earlier groups stay queued).
 *
 * Other lists (any version-1 blob, or mixed dtypes) launch one decode per blob. With two or more blobs,
 * an expand kernel first builds every version-1 blob's tables (144 KB each) into the same kind of
 * scratch, and those decodes take them by bulk copies; a copy that has not landed in time sets
 * EP_DEV_TABLE_COPY and that CTA decodes nothing. If the scratch cannot be had, each CTA builds its own
 * tables. The first decode is ordered after earlier work on the stream as usual; each later one is a
 * programmatic dependent launch of the one before it that stores nothing until that decode has
 * finished.
 *
 * Errors: as ep_decompress_into, for the first failing blob; EP_ERR_NOMEM as above.
 * Test hook: with the environment variable EPK_TEST_TABLE_COPY_TIMEOUT set to 1 when the call is made,
 * the version-1 table copies are not issued, so every CTA's bounded wait runs out (each poll suspends
 * about 1 us, 2^14 polls twice) and EP_DEV_TABLE_COPY is set. The test suite uses it to check that path.
 */
ep_status ep_decompress_many(int count, const uint8_t* const* host_hdrs, const void* const* dev_blobs,
                             const size_t* blob_bytes, void* const* dsts, const size_t* dst_bytes,
                             void* cuda_stream);

/*
 * ep_decompress: the same decode, into a device buffer that the call allocates with cudaMallocAsync
 * on cuda_stream. *dst receives the pointer, and the caller frees it (cudaFreeAsync or cudaFree).
 * Errors: as ep_decompress_into, plus EP_ERR_NOMEM.
 */
ep_status ep_decompress(const uint8_t* host_hdr, const void* dev_blob, size_t blob_bytes, void** dst,
                        void* cuda_stream);

/*
 * ep_decode_coords_into: test and inspection entry. It runs the same decode, but stores the lattice
 * coordinates instead of rescaled values: z = 2v as int32, rows*cols of them, row-major, where v is
 * the decoded E8 point (v = u + b/2). dst_z must be 16-byte aligned, with dst_bytes >= 4*rows*cols.
 * Errors as ep_decompress_into.
 */
ep_status ep_decode_coords_into(const uint8_t* host_hdr, const void* dev_blob, size_t blob_bytes,
                                int32_t* dst_z, size_t dst_bytes, void* cuda_stream);

/*
 * ep_get_device_status: synchronises cuda_stream, then reads and clears the device status word of the
 * current device. That word is the OR of the EP_DEV_* bits that the decode kernels set since the last
 * read. The read and the clear are two copies: a bit that a decode still running on another stream sets
 * between them is lost, so synchronise the streams whose decodes should be reported before the call.
 * Errors: EP_ERR_ARG, EP_ERR_CUDA.
 */
ep_status ep_get_device_status(void* cuda_stream, int32_t* flags);

/* Static English text for a status code. */
const char* ep_status_string(ep_status st);

/* Message for the calling thread's last failed call ("" if none). Valid until that thread's next call. */
const char* ep_last_error(void);

/*
 * Lossless tile-ANS ("EPL1" blobs; the EntroPack README's Config table, TileANSConfig: exact restoration of
 * BF16, FP16, FP32, FP8 and INT8 tensors of any shape, with a ratio that depends on the data). The raw bit
 * patterns of the elements are cut into byte planes (byte j of every element, little-endian); a plane whose
 * values cluster is rANS-coded under its own 12-bit table in tiles of 32 interleaved lanes, the others are
 * stored verbatim. No value is interpreted: NaN payloads, signed zeros and subnormals come back as they were.
 */
#define EP_TANS_HEADER_BYTES 96

/*
 * ep_tans_compress: host encoder. data: numel = dims[0] x ... x dims[ndim-1] elements of `dtype`, host
 * memory, row-major, read only (ndim 0..8; ndim 0 is one element; a zero dim gives an empty tensor).
 * elems_per_lane: K, a tile holds 32 x K elements (1..1024, or 0 for 128). threads: host threads (0 = all
 * cores); the blob does not depend on it. The blob is malloc'd; release it with ep_blob_free.
 * Errors: EP_ERR_ARG (NULL pointer, K out of range), EP_ERR_DTYPE, EP_ERR_SHAPE (a dim above 2^32 - 1, or a
 * blob above 64 GB), EP_ERR_NOMEM.
 */
ep_status ep_tans_compress(const void* data, ep_dtype dtype, int ndim, const int64_t* dims, uint32_t elems_per_lane,
                           int threads, uint8_t** blob_out, size_t* bytes_out);

/*
 * ep_tans_info: full host validation of an EPL1 blob (header, tables, tile offsets, metadata CRC) and its
 * description. dims receives ndim values (at most 8). Every out-pointer may be NULL.
 * Errors: EP_ERR_ARG, EP_ERR_CORRUPT.
 */
ep_status ep_tans_info(const uint8_t* blob, size_t blob_bytes, ep_dtype* dt, int* ndim, int64_t* dims,
                       uint32_t* coded_mask, uint32_t* elems_per_lane);

/*
 * ep_tans_decompress_into: decode of an EPL1 blob into a caller-owned device buffer, on the GPU.
 * host_hdr    host copy of at least the first 96 bytes of the blob (the header).
 * dev_blob    device copy of the whole blob, 16-byte aligned, blob_bytes long; read only.
 * dst         device buffer of numel elements of the blob's dtype, 16-byte aligned; dst_bytes its size.
 *             It may be NULL for an empty tensor, which launches nothing.
 * cuda_stream cudaStream_t to launch on; NULL means the legacy default stream.
 * One kernel, no allocation, no synchronisation. Host-detectable errors: EP_ERR_ARG, EP_ERR_CORRUPT (bad
 * header), EP_ERR_BUFFER (size or alignment), EP_ERR_CUDA. The kernel checks every tile's final states and
 * word count and bounds its reads; corruption sets EP_DEV_* bits of the device status word
 * (ep_get_device_status) instead of faulting, and a corrupt tile's elements are unspecified.
 */
ep_status ep_tans_decompress_into(const uint8_t* host_hdr, const void* dev_blob, size_t blob_bytes, void* dst,
                                  size_t dst_bytes, void* cuda_stream);

#ifdef __cplusplus
}
#endif

#endif /* ENTROPACK_H */
