/*
 * nwc.h — C ABI of libnwc: lossless BF16 weight compression with a fused
 * decode-GEMV for NVIDIA B200 (sm_100a).
 *
 * The method, with the passages that define it:
 *   - A BF16 weight (sign 1 | exponent 8 | fraction 7; "Efficient ML #1 — Deep
 *     Learning Data Types", §4) is split into two byte planes.  The exponent byte
 *     is entropy-coded and the sign+fraction byte is stored raw ("Unweight: how we
 *     compressed an LLM 22% without sacrificing quality", section "Compressing BF16
 *     Weights"; "NWC — Neural Weight Compression", "How it works > Byte planes").
 *   - The code is one optimal prefix code per matrix, with lengths limited to lmax
 *     (7 by default, so that one 14-bit table peek always holds two complete
 *     codes, as the decoder in "NWC", "How it works > Prefix code instead of
 *     rANS" does with its 12-bit peek).
 *   - The matrix is cut into independently decodable tiles of 8 rows x tile_cols
 *     columns, with one bit stream per lane ("NWC", "How it works > Fused kernel").
 *   - The GPU decodes the tiles in registers and shared memory inside the
 *     matrix-vector kernel; no decompressed weight is written to device memory
 *     ("NWC", "Fused kernel"; "Unweight", "Direct GPU Decompression").
 *
 * Conventions for every call:
 *   - Matrices are row-major [rows x cols] = [out_features x in_features].  BF16
 *     values are passed as their uint16_t bit patterns.
 *   - The caller owns all device memory.  A handle owns only host metadata and
 *     refers to the caller's device buffer, which must outlive it.  No call frees
 *     caller memory, and no device call allocates.
 *   - Device calls are asynchronous on the given stream (0 = legacy default
 *     stream).  They do not synchronize, except where a call says it does.
 *   - Arguments are validated on the host before anything is launched.  Invalid
 *     input returns an error code and launches nothing.
 *   - Errors found on the device (a corrupt tile, a bounded wait that gave up) set
 *     bits in the handle's error word, which lives in its device image;
 *     nwc_get_device_error() reads and clears it.
 *   - Thread safety: distinct handles may be used concurrently.  Device calls on
 *     one handle write its image's scratch area, so they must be ordered by the
 *     caller (one stream, or events between streams).
 */
#ifndef NWC_H
#define NWC_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st* nwc_stream_t; /* same object as cudaStream_t */
typedef struct nwc_plan_s* nwc_plan_t;     /* opaque, host only           */
typedef struct nwc_handle_s* nwc_handle_t; /* opaque, host metadata only  */

typedef enum {
  NWC_OK = 0,
  NWC_ERR_INVALID_ARG = 1,    /* null pointer, bad size, bad alignment, ...     */
  NWC_ERR_UNSUPPORTED = 2,    /* valid but not implemented (e.g. tile geometry) */
  NWC_ERR_CUDA = 3,           /* a CUDA runtime call failed                     */
  NWC_ERR_CORRUPT = 4,        /* a blob or device image does not parse          */
  NWC_ERR_NOMEM = 5,          /* host allocation failed, or buffer too small    */
  NWC_ERR_DEVICE_TIMEOUT = 6, /* the device error word reported a timeout       */
  NWC_ERR_DEVICE_CORRUPT = 7, /* the device error word reported corrupt data    */
  NWC_ERR_SCRATCH_LIMIT = 8   /* nwc_gemv_noalloc: scratch needed > the limit   */
} nwc_status;

/* Exponent codes (nwc_opts.code). */
typedef enum {
  /* "NWB1": exponent bits 14..7 in a length-limited canonical prefix code;
   * sign and fraction raw.  Every call of this library takes it. */
  NWC_CODE_PREFIX = 0,
  /* "NWR1": exponent bits 14..8 ranked by count in a unary code with the sign
   * bit beside it and an escape ("NWC", "How it works > Prefix code instead of
   * rANS", format v9); bits 7..0 raw; one stream per lane.  Every call takes
   * it. */
  NWC_CODE_RANK = 1,
  /* "NWE1": the `keep` most frequent exponent bytes in the length-limited
   * canonical prefix code; a run of 64 weights of a tile row (one row, one
   * 64-column group) that holds any other exponent keeps its exponent bytes
   * verbatim in the tile's chunk, beside a 16-byte flag field ("Unweight",
   * "Compressing BF16 Weights": the 16 most common exponents cover nearly all
   * weights; rare ones are stored with their whole row of 64, so the decoder
   * branches once per run).  Sign and fraction raw; one stream per lane;
   * lmax <= 7.  Every call takes it. */
  NWC_CODE_ESCAPE = 2
} nwc_code;

/* Plan options.  Set struct_size = sizeof(nwc_opts); pass NULL for the defaults
 * (lmax = 0, tile_rows = 8, tile_cols = 512, threads = 0 meaning all cores,
 * code = NWC_CODE_PREFIX).  A struct_size that ends before `code` (the layout
 * without it) means NWC_CODE_PREFIX.
 * lmax, NWC_CODE_PREFIX: 0 = automatic (7, or the smallest limit that admits
 * every distinct exponent when there are more than 128), else in [1, 12] and at
 * least ceil(log2(distinct exponents)).  With lmax <= 7 the decoder peeks 14
 * bits and every peek holds two complete codes; with 8..12 it peeks 12 bits and
 * takes a second lookup when a pair does not fit.
 * lmax, NWC_CODE_RANK: the number of ranks, 0 = 7, else in [1, 7].
 * lmax, NWC_CODE_ESCAPE: 0 = 7, else in [1, 7] and at least ceil(log2(coded
 * exponents)) (8..12 are a valid format that no kernel reads: UNSUPPORTED).
 * keep (a struct_size that ends before it, or 0, means 16): NWC_CODE_ESCAPE's
 * number of coded exponents, 1..256; ignored by the other codes.
 * tile_rows must be 8; tile_cols must be 64, 128, 256 or 512.
 * streams (a struct_size that ends before it means 1): bit streams per lane
 * and tile, each lane's symbol pairs dealt to its streams in turn (header
 * offset 60 holds streams - 1), with NWC_CODE_PREFIX only (others:
 * UNSUPPORTED).  Every kernel reads 1 and 2 (a lane then follows two
 * independent decode chains); 4 is a host-encoder-only layout: nwc_plan_size
 * reports device_bytes = 0 and the calls that need a device image return
 * UNSUPPORTED. */
typedef struct {
  uint32_t struct_size;
  uint32_t lmax;
  uint32_t tile_rows;
  uint32_t tile_cols;
  uint32_t threads; /* host encoder threads; 0 = hardware concurrency */
  uint32_t code;    /* nwc_code */
  uint32_t streams; /* bit streams per lane and tile: 0 or 1, 2, 4 (see below) */
  uint32_t keep;    /* NWC_CODE_ESCAPE: exponents coded, 0 = 16 (see below) */
} nwc_opts;

/* Library version: major * 10000 + minor * 100 + patch. */
int nwc_version(void);

/* Human-readable name of a status code (static storage; never NULL). */
const char* nwc_status_string(nwc_status status);

/* ---- Host encoder ------------------------------------------------------- */

/* Histogram of the exponent bytes, the length-limited canonical code, and the
 * exact compressed sizes ("Unweight", "Compressing BF16 Weights": the exponent
 * byte is Huffman-coded from its histogram, sign and mantissa kept; "NWC",
 * "How it works > Prefix code instead of rANS": one code table per matrix,
 * decoded by a fixed-width table peek).  w_host holds rows x cols BF16
 * patterns, row-major.
 * It is read, not retained.  rows, cols >= 1.  On success *out_plan owns host
 * memory; free it with nwc_plan_destroy.
 * Errors: INVALID_ARG (null, sizes, options, > 64 GiB of tile data), NOMEM. */
nwc_status nwc_plan(const uint16_t* w_host, int64_t rows, int64_t cols,
                    const nwc_opts* opts, nwc_plan_t* out_plan);

/* Exact sizes for a plan.  *device_bytes is what nwc_compress needs in device
 * memory, the "device image": the serialisable blob, then at 256-byte aligned
 * offsets a derived decode table (64 KiB for lmax <= 7, else 16 KiB), the
 * launch schedules (which bytes each bulk copy of the kernels moves and where
 * they land in shared memory, worked out on the host for the device that runs
 * them), and a scratch area that the kernels write: the handle's error word,
 * split-K arrival counters (4 bytes per 8 rows) and partial sums (for a matrix
 * of more than one column tile: 4 bytes x 16 rows of x x rows x column tiles,
 * about 9 % of the compressed size at 512-column tiles, or 1 MiB if that is
 * larger).  *host_blob_bytes is the size of the serialisable blob
 * (nwc_compress_host).  Either pointer may be NULL. */
nwc_status nwc_plan_size(nwc_plan_t plan, uint64_t* device_bytes,
                         uint64_t* host_blob_bytes);

/* Encode w_host (the same matrix given to nwc_plan) and upload it into the
 * caller's device buffer d_buf (>= device_bytes, 256-byte aligned) on `stream`
 * ("NWC", "How it works > Byte planes" and "> Fused kernel": byte planes in
 * independently decodable blocks of 8 rows x 512 columns, one bit stream per
 * lane).  Only the blob, table, schedules and the start of the scratch area
 * are copied; the partial sums need no initial value.
 * The upload is asynchronous: w_host may be reused when the call returns,
 * but d_buf must not be read before the stream reaches this point.  On success
 * *out_handle refers to d_buf.
 * Errors: INVALID_ARG (null, d_bytes too small, misaligned d_buf), NOMEM,
 * CUDA. */
nwc_status nwc_compress(nwc_plan_t plan, const uint16_t* w_host, void* d_buf,
                        uint64_t d_bytes, nwc_stream_t stream,
                        nwc_handle_t* out_handle);

/* Encode into a host buffer (>= host_blob_bytes).  The bytes are the
 * serialisable blob of the plan's code: "NWB1", "NWR1" or "NWE1". */
nwc_status nwc_compress_host(nwc_plan_t plan, const uint16_t* w_host, void* blob,
                             uint64_t blob_bytes);

/* Bytes of device memory needed to upload an existing blob (the device image:
 * blob + decode table + launch schedule).  Host only; the blob is checked as
 * nwc_upload_blob checks it.
 * Errors: INVALID_ARG (null), CORRUPT (the blob does not parse: a header field
 * inconsistent with the others or with blob_bytes, code lengths over lmax or
 * not a prefix code, an index that is not increasing or whose chunk sizes fall
 * outside what the geometry allows), UNSUPPORTED (a valid layout that no kernel
 * reads, as nwc_upload_blob), NOMEM (the host copy of the index). */
nwc_status nwc_blob_device_bytes(const void* blob, uint64_t blob_bytes,
                                 uint64_t* device_bytes);

/* Validate a host blob ("NWB1", "NWR1" or "NWE1"), upload it into d_buf, and
 * build its decode table and launch schedule for the current device.  The call
 * is synchronous: it returns after the copies finish.
 * Errors: CORRUPT (header, code lengths or index do not parse, as for
 * nwc_blob_device_bytes), UNSUPPORTED (a valid layout no kernel reads: NWB1
 * with 4 streams per lane, NWE1 with lmax over 7), INVALID_ARG, NOMEM, CUDA.
 * The tile area is not read on the host: a corrupt chunk (a stream without a
 * valid code, an NWE1 flag field naming a group past the tile or more runs than
 * the chunk holds) is found by the kernels, which stay inside their buffers and
 * set the handle's corrupt bit (nwc_get_device_error). */
nwc_status nwc_upload_blob(const void* blob, uint64_t blob_bytes, void* d_buf,
                           uint64_t d_bytes, nwc_stream_t stream,
                           nwc_handle_t* out_handle);

/* Build a handle for a device buffer that already holds a device image (from
 * nwc_compress or nwc_upload_blob, possibly copied elsewhere).  The call is
 * synchronous: it reads the header, code lengths and index back to the host,
 * then rewrites the image's launch-schedule area for the current device (the
 * blob and the decode table are not written).  Any of the three formats.
 * Errors: CORRUPT, UNSUPPORTED (as nwc_upload_blob), INVALID_ARG, NOMEM, CUDA. */
nwc_status nwc_handle_from_device(void* d_buf, uint64_t d_bytes,
                                  nwc_handle_t* out_handle);

/* ---- Device kernels ---------------------------------------------------- */

/* A handle belongs to the device that was current when it was made (the one
 * holding its image); the calls below return INVALID_ARG when another device is
 * current.
 *
 * nwc_decompress, nwc_gemv and nwc_gemv_noalloc launch one persistent CTA per
 * SM (at most 256).  Should the current device's launch shape differ from the
 * one the image's schedule was written for, the call first rewrites that
 * schedule on `stream` (a host-to-device copy, in stream order).
 *
 * They launch with programmatic stream serialization: a kernel may start while
 * the previous kernel on the stream is still finishing.  Until that kernel has
 * completed it reads only the device image (blob, decode table, schedule);
 * x, y, the workspace and the output are touched only afterwards.  So the
 * kernel launched just before such a call must not write the device image
 * (stream order still holds for copies, memsets and events). */

/* Bit-exact decompression ("NWC", "How it works > Dequantization and embedding
 * lookup": the same decoder writes BF16).  d_w_out: device, rows x cols BF16,
 * row-major, 4-byte aligned.  Asynchronous on `stream`.
 * Errors: INVALID_ARG, CUDA (launch). */
nwc_status nwc_decompress(nwc_handle_t handle, uint16_t* d_w_out, nwc_stream_t stream);

/* Rows of W, bit-exact, straight from the compressed matrix: an embedding
 * lookup, e.g. on a tied lm_head ("NWC", "How it works > Dequantization and
 * embedding lookup").  out[i][k] = W[rows[i]][k] for i < n, k < cols.
 *   d_rows: device, int32 [n], row ids in [0, rows), 4-byte aligned.
 *   d_out: device, BF16 [n x cols] row-major, 2-byte aligned.
 *   n in [1, 2^20].
 * A row id out of range leaves its output row unwritten and sets a bit of the
 * device error word (nwc_get_device_error then returns INVALID_ARG).  Only the
 * tiles that hold the requested rows are read.  Asynchronous on `stream`.
 * Errors: INVALID_ARG, CUDA (launch). */
nwc_status nwc_gather_rows(nwc_handle_t handle, const int32_t* d_rows, int32_t n,
                           uint16_t* d_out, nwc_stream_t stream);

/* Bytes of split-K scratch one GEMV call of `batch` rows uses: u32 arrival
 * counters (one per 8 rows, padded to 256 bytes) and FP32 partial sums: on the
 * CUDA-core kernel one per (column tile, row of x in a launch, output row), on
 * the tensor-core kernel one per (part of its K split, row of x up to 64,
 * output row) when it splits K; 0 when the matrix has a single column tile.
 * nwc_gemv takes them from the device image's scratch area, nwc_gemv_noalloc
 * from the library's static array.  The partials make the reduction
 * deterministic (fixed summation order). */
nwc_status nwc_gemv_scratch_bytes(nwc_handle_t handle, int32_t batch, uint64_t* bytes);

/* The fused decode-GEMV ("NWC", "How it works > Fused kernel": the matrix-vector
 * kernel decodes the compressed blocks itself and keeps partial sums per
 * (row, column block); "Unweight", "Direct GPU Decompression": weights are
 * decompressed in shared memory and fed to the tensor cores, never written
 * back): y[b][n] = sum_k W[n][k] * x[b][k], for b < batch, n < rows, k < cols.
 *   d_x: device, BF16 [batch x cols], row-major, 4-byte aligned (2-byte when
 *     cols is odd).
 *   d_y: FP32 [batch x rows], row-major (overwritten, not accumulated), in
 *     device memory or in pinned host memory that the device can address (the
 *     kernel then stores the result straight into host memory).
 *   batch in [1, 64].
 * The caller passes no workspace: the split-K partial sums and counters live
 * in the scratch area of the handle's device image, so calls on one handle
 * must be ordered (a completed call leaves the counters zero again;
 * nwc_get_device_error clears them after a call that ended with an error).
 * Products and sums are in FP32; the result is the same bit pattern on every
 * run.  Asynchronous on `stream`; allocates nothing.
 * Errors: INVALID_ARG (null, batch, alignment, another device current),
 * UNSUPPORTED, CUDA (launch). */
nwc_status nwc_gemv(nwc_handle_t handle, const uint16_t* d_x, float* d_y,
                    int32_t batch, nwc_stream_t stream);

/* Two kernels compute nwc_gemv.  The CUDA-core kernel multiplies the decoded
 * weights in registers (mma.sync) and handles up to 16 rows of x per launch,
 * decoding the matrix again for every 16 rows.  The tensor-core kernel decodes
 * each tile once into shared memory and multiplies it with every row of x
 * (up to 64) on the tcgen05 tensor cores, accumulating in TMEM ("Unweight",
 * "Direct GPU Decompression": decompress into shared memory, then the tensor
 * cores).  A GEMV takes the tensor-core kernel when batch >= the handle's
 * threshold, cols is a multiple of 8, d_x is 16-byte aligned and the kernel's
 * shared-memory layout fits the device.  The default threshold is 17: on
 * B200 one CUDA-core launch of up to 16 rows is faster than the tensor-core
 * kernel, whose per-chunk synchronization costs more than it saves until a
 * second CUDA-core launch would be needed.
 * nwc_gemv_set_tc_min_batch sets the threshold: 1..64, or 0 for never.
 * Errors: INVALID_ARG. */
nwc_status nwc_gemv_set_tc_min_batch(nwc_handle_t handle, int32_t min_batch);

/* Which kernel a GEMV of `batch` rows with this d_x would take, without
 * launching: *launches (optional) kernel launches, *tensor_cores (optional) 1
 * for the tensor-core kernel, else 0.  Host only.
 * Errors: INVALID_ARG. */
nwc_status nwc_gemv_path(nwc_handle_t handle, const uint16_t* d_x, int32_t batch,
                         int32_t* launches, int32_t* tensor_cores);

/* GEMV for callers that cannot allocate device memory.  The pages describe
 * no such call; it exists for integrations where the host application owns
 * every device allocation and a library may not call cudaMalloc (inference
 * servers with a fixed memory pool, plugins loaded into another framework),
 * and for code that must not allocate while work is being recorded into a
 * CUDA graph, since an allocation there breaks the recording.
 *
 * It computes exactly what nwc_gemv computes, with the same kernels, but takes
 * its scratch (the split-K partial sums and arrival counters) from an array of
 * NWC_NOALLOC_SCRATCH_BYTES bytes that the library defines as a static device
 * variable instead of the device image's scratch area (the handle's error word
 * stays in the image).  Every GPU that loads the library holds that array until the
 * process exits.  The call allocates nothing: no cudaMalloc, no cudaFree, no
 * allocating library routine.
 *   - Set-up: the first call on a device looks up the array's device address
 *     (cudaGetSymbolAddress) with that device current, and caches it.  Make
 *     that first call before any stream capture.
 *   - Limit: when nwc_gemv_scratch_bytes(handle, batch) exceeds
 *     NWC_NOALLOC_SCRATCH_BYTES the call returns NWC_ERR_SCRATCH_LIMIT and
 *     launches nothing; use nwc_gemv instead.
 *   - Sharing: every call uses the same array, which keeps the last call's
 *     contents; each call first clears the counters it needs (an async memset
 *     on `stream`).  Calls whose work overlaps on the GPU (different streams,
 *     or different threads without ordering) race on the array and must not
 *     be issued.
 * Arguments and other errors as nwc_gemv; every argument is checked before
 * anything is enqueued. */
#define NWC_NOALLOC_SCRATCH_BYTES (8u << 20)
nwc_status nwc_gemv_noalloc(nwc_handle_t handle, const uint16_t* d_x, float* d_y,
                            int32_t batch, nwc_stream_t stream);

/* ---- Inspection, errors, teardown ------------------------------------- */

/* Launch shape and schedule the kernels would use for a blob on a device with
 * sm_count SMs and smem_limit bytes of opt-in shared memory per block (B200:
 * 148 and 232448), for a launch handling rows_of_x rows of x (0 for
 * decompression; nwc_gemv launches one kernel per 16 rows).  Launches of up to
 * 4 rows reserve 8,448 bytes of shared memory for x, larger ones 33,024, so
 * the two classes have different rings and schedules.  Host only; touches no
 * GPU.
 *   info: set struct_size = sizeof(nwc_schedule_info).
 *   cta_batch (optional, ctas + 1 entries): first batch of each CTA, and the
 *     total number of batches at the end.  CTA c owns tiles
 *     [tiles * c / ctas, tiles * (c + 1) / ctas) in blob order.
 *   batch (optional, 4 * batches entries): per batch {tile-area offset in
 *     16-byte units, bytes, offset in the CTA's ring, number of the CTA's
 *     earlier batches that must be released before this one is issued}.
 *   tile_ring (optional, tiles entries): ring offset of each tile's chunk.
 * Query info first (arrays NULL) to size the arrays.
 * Errors: INVALID_ARG, CORRUPT, UNSUPPORTED (shared memory too small). */
typedef struct {
  uint32_t struct_size;
  int32_t ctas;          /* persistent CTAs                                  */
  int32_t batch_tiles;   /* consecutive tiles per bulk copy                  */
  int32_t ring_bytes;    /* staging ring in shared memory, per CTA           */
  int64_t tiles;         /* tiles of the matrix                              */
  int64_t batches;       /* bulk copies over all CTAs                        */
  uint64_t smem_bytes;   /* dynamic shared memory per CTA                    */
  uint32_t xstage_bytes; /* shared memory reserved for x, per CTA            */
} nwc_schedule_info;
nwc_status nwc_schedule_describe(const void* blob, uint64_t blob_bytes, int32_t sm_count,
                                 uint64_t smem_limit, int32_t rows_of_x,
                                 nwc_schedule_info* info, uint32_t* cta_batch,
                                 uint32_t* batch, uint32_t* tile_ring);

/* The tensor-core kernel's launch shape and schedule for a blob, a GEMV of
 * rows_of_x rows (1..64; the accumulator has 16, 32 or 64 columns, and each
 * width has its own shape) on a device of sm_count SMs and smem_limit bytes of
 * opt-in shared memory per block.  Host only; touches no GPU.  K is split
 * into `ksplit` column ranges and the row tiles into ctas / ksplit row ranges
 * (range k of n parts of m items: [m k / n, m (k + 1) / n)); CTA
 * c = rs ksplit + ks owns row range rs x column range ks, in M-groups of
 * `rows` row tiles; `teams` teams of `rows` decode warps take the column
 * blocks j_lo + t, j_lo + t + teams, ... of a group.  Each copy moves one
 * tile's lane lengths and streams (batch_tiles = 1); the raw plane is read
 * from global memory.
 *   cta_batch (optional, ctas + 1 entries), batch (optional, 4 * batches):
 *     as nwc_schedule_describe.
 *   tile_ring, tile_batch (optional, tiles entries each), indexed by blob tile
 *     u = j tiles_r + i: the ring offset of the tile's streams, and the CTA's
 *     copy that brings them.
 * Errors: INVALID_ARG, CORRUPT, UNSUPPORTED (no layout fits). */
typedef struct {
  uint32_t struct_size;
  int32_t ctas, rows, teams, batch_tiles, ring_bytes, n, x_stages;
  int64_t tiles, batches;
  uint64_t smem_bytes, a_offset, b_offset, ring_offset;
  int32_t ksplit, a_stages;
} nwc_tc_schedule_info;
nwc_status nwc_tc_schedule_describe(const void* blob, uint64_t blob_bytes, int32_t sm_count,
                                    uint64_t smem_limit, int32_t rows_of_x,
                                    nwc_tc_schedule_info* info, uint32_t* cta_batch,
                                    uint32_t* batch, uint32_t* tile_ring, uint32_t* tile_batch);

/* Any pointer may be NULL.  *blob_bytes is the serialisable part;
 * *compressed_bytes is what holds the matrix (blob, decode table and launch
 * schedules: the offset of the scratch area); *device_bytes is the whole device
 * image (compressed bytes + scratch area). */
nwc_status nwc_handle_info(nwc_handle_t handle, int64_t* rows, int64_t* cols,
                           uint64_t* blob_bytes, uint64_t* device_bytes,
                           uint64_t* compressed_bytes);

/* Reads the handle's device error word in order on `stream` (which it then
 * synchronizes) and clears it, together with the split-K arrival counters, when
 * it is non-zero.  Only this handle's kernels set it.  Returns OK,
 * DEVICE_TIMEOUT, DEVICE_CORRUPT or INVALID_ARG (a gathered row id out of
 * range), in that order of precedence, or CUDA.  *word (optional) receives the
 * raw bits: 1 a bounded wait gave up, 2 corrupt stream, 4 row id out of range. */
nwc_status nwc_get_device_error(nwc_handle_t handle, nwc_stream_t stream, uint32_t* word);

/* Test and diagnostic use only: the number of polls after which a kernel's
 * bounded wait on an mbarrier gives up (sets error bit 1 and returns) for
 * launches made after this call, process-wide; 0 restores the default
 * (2^22 polls).  A small limit makes a wait that would otherwise only be slow
 * give up, so ordinary callers never set it. */
void nwc_test_set_wait_limit(uint32_t polls);

/* Free host metadata.  NULL is accepted.  Device memory is never freed. */
void nwc_plan_destroy(nwc_plan_t plan);
void nwc_handle_destroy(nwc_handle_t handle);

#ifdef __cplusplus
}
#endif
#endif /* NWC_H */
