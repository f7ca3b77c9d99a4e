// kernels.cuh — launch interface of the sm_100a kernels (host side).
#pragma once
#include <cuda_runtime.h>
#include <cstdint>

#include "nwc_format.h"

namespace nwc {

// Barrier slots per CTA: batches in flight or resident at once are fewer.
constexpr int kSlots = 64;
// Most tiles a consumer warp's next wait can lie beyond the last tile it
// released (its warps x tiles decoded at once, over all kernels); the launch
// schedule relies on it.
constexpr int kMaxLag = 48;

// Device error word bits (the first word of a device image's scratch area;
// read and cleared by nwc_get_device_error).
constexpr uint32_t kErrTimeout = 1u;   // a bounded mbarrier wait gave up
constexpr uint32_t kErrCorrupt = 2u;   // a stream held no valid code
constexpr uint32_t kErrRange = 4u;     // a gathered row id was out of range

// Polls of a bounded mbarrier wait before it gives up (TileParams.wait_limit
// 0 means this).
constexpr uint32_t kDefaultWaitLimit = 1u << 22;

struct TileParams {
  const uint8_t* tiles;     // device: tile area of the blob
  const uint32_t* sched_cta;   // device: first batch of each CTA, ctas + 1
  const uint4* sched_batch;    // device: per batch {offset16, bytes, ring offset, need}
  const uint32_t* tile_ring;   // device: per tile, ring offset of its chunk
  const uint32_t* table;    // device: decode table (table_bytes)
  uint32_t table_bytes;     // 64 KiB (14-bit peek) or 16 KiB (12-bit peek)
  uint32_t ring_offset;     // shared-memory offset of the staging ring
  int64_t rows, cols;
  int64_t tiles_r, tiles_c, n_tiles;
  int32_t ring_bytes;       // CTA staging ring in shared memory
  int32_t batch_tiles;      // consecutive tiles moved by one bulk copy
  uint32_t xstage_bytes;    // shared memory reserved for x (GEMV)
  // GEMV
  const uint16_t* x;        // BF16 [batch x cols]
  float* y;                 // FP32 [batch x rows]
  int32_t batch;            // rows of x handled by this launch (<= kMaxPassRows)
  float* partial;           // [tiles_c][batch][rows_pad] split-K partial sums
  uint32_t* counters;       // [tiles_r] arrivals per row tile
  int64_t rows_pad;         // 8 * tiles_r
  // decompress
  uint16_t* out;            // BF16 [rows x cols]
  uint32_t* err;            // device: the handle's error word
  uint32_t wait_limit;      // polls before a bounded wait gives up (0: default)
};

// Shared memory that a CTA reserves for its columns of x, by x-stage class:
// 4 rows (class 0: decompression and GEMV launches of up to 4 rows) or 16 rows
// (class 1), over two column blocks of 512.  A smaller stage leaves a larger
// ring.
constexpr uint32_t kXStageBytes[2] = {8448, 33024};
inline int stage_class(int rows_of_x) { return rows_of_x <= 4 ? 0 : 1; }

struct LaunchShape {
  int ctas;             // one persistent CTA per SM (fewer for small matrices)
  uint32_t table_bytes;
  uint32_t xstage_bytes;  // x stage reserved after the barriers
  size_t ring_offset;
  int ring_bytes;
  int batch_tiles;
  size_t smem_bytes;
};

// Grid and shared-memory layout for n_tiles tiles whose largest chunk is
// max_chunk bytes (typical_chunk on average), within the device's per-block
// shared-memory limit.
LaunchShape launch_shape(int64_t n_tiles, uint64_t max_chunk, uint64_t typical_chunk,
                         uint32_t table_bytes, int sm_count, size_t smem_limit,
                         uint32_t xstage_bytes);

// Launch schedule for one shape (host): for every CTA (tiles [n c / C,
// n (c + 1) / C)) its batches of batch_tiles consecutive tiles, each with its
// tile-area offset (16-byte units), its bytes, its place in the ring (a batch
// never wraps; space is reused first in, first out) and how many of the CTA's
// earlier batches must have been released before it is issued (for room, and
// to keep fewer than kSlots - ceil(kMaxLag / batch_tiles) outstanding).
// `index` holds the tiles + 1 chunk offsets in 16-byte units; `out` receives
// sched_class_bytes(n_tiles) bytes (one class) laid out as nwc_format.h describes.
void build_schedule(const uint32_t* index, int64_t n_tiles, const LaunchShape& s, uint8_t* out);

// fast: lmax <= 7 (14-bit peek, two codes per entry always).
cudaError_t launch_gemv(const TileParams& p, int tile_cols, bool fast, const LaunchShape& s,
                        cudaStream_t stream);
cudaError_t launch_decompress(const TileParams& p, int tile_cols, bool fast,
                              const LaunchShape& s, cudaStream_t stream);
// Row gather (embedding lookup) from the compressed matrix.
struct GatherParams {
  const uint8_t* tiles;     // device: tile area of the blob
  const uint32_t* index;    // device: chunk offsets (16-byte units), tiles + 1
  const uint32_t* table;    // device: decode table
  int32_t peek;             // table peek width (12 or 14)
  int32_t tile_cols;
  int64_t rows, cols, tiles_r, tiles_c;
  const int32_t* row_ids;   // device: n row ids
  int32_t n;
  uint16_t* out;            // device: BF16 [n x cols]
  uint32_t* err;            // device: the handle's error word
};
cudaError_t launch_gather(const GatherParams& g, cudaStream_t stream);

}  // namespace nwc
