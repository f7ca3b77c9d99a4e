// kernels.cuh — launch interface of the sm_100a kernels (host side).
#pragma once
#include <cuda.h>
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
constexpr uint32_t kErrLayout = 8u;    // shared memory not aligned as a kernel needs

// Polls of a bounded mbarrier wait before it gives up (TileParams.wait_limit
// 0 means this).
constexpr uint32_t kDefaultWaitLimit = 1u << 22;

// The exponent code a kernel reads: the prefix code through a 12-bit or a
// 14-bit table peek, the ranked unary code (variant NWR1, no table), or the
// prefix code through the 14-bit peek with runs of rare exponents stored
// verbatim (variant NWE1).
constexpr int kCode12 = 0, kCode14 = 1, kCodeRank = 2, kCodeEsc = 3;

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
  float* partial;           // split-K partial sums: [tiles_c][batch][rows_pad] (CUDA
                            // cores), [ksplit][tiles_r][kMaxTcRows][8] (tensor cores)
  uint32_t* counters;       // [tiles_r] arrivals per row tile
  int64_t rows_pad;         // 8 * tiles_r
  // decompress
  uint16_t* out;            // BF16 [rows x cols]
  uint32_t* err;            // device: the handle's error word
  uint32_t wait_limit;      // polls before a bounded wait gives up (0: default)
  int32_t streams;          // bit streams per lane and tile (1 or 2)
  // tensor-core kernel
  const uint32_t* index;       // device: chunk offsets (16-byte units), tiles + 1
  const uint32_t* tile_batch;  // device: per tile, its copy's place in its CTA's schedule
  int32_t tc_bstages;       // x stages per team (1 or 2)
  int32_t tc_astages;       // A stages per team (2 or 3)
  int32_t tc_rows;          // R: row tiles per M-group (rows of the MMA / 8)
  int32_t tc_teams;         // teams of R decode warps, each on its own column blocks
  int32_t tc_n;             // accumulator columns: rows of x padded to 16, 32 or 64
  int32_t tc_ksplit;        // column ranges; gridDim.x is a multiple of it
  uint32_t tc_tmem_cols;    // TMEM columns allocated (power of two >= 32)
  uint32_t tc_bar_off, tc_a_off, tc_b_off;  // shared-memory offsets
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

// code: kCode12, kCode14 (lmax <= 7: two codes per table entry always),
// kCodeRank or kCodeEsc.
cudaError_t launch_gemv(const TileParams& p, int tile_cols, int code, const LaunchShape& s,
                        cudaStream_t stream);

// ---- tensor-core (tcgen05) GEMV: decode once, multiply every row of x -----
//
// The matrix's tile grid (tiles_r row tiles x tiles_c column blocks) is cut
// into rectangles: K into ksplit column ranges, the rows into C / ksplit row
// ranges; CTA c = rs ksplit + ks owns row range rs x column range ks.  Its row
// tiles form M-groups of R (the MMA's M = 128 rows holds up to 16 row tiles);
// `teams` teams of R decode warps take the column blocks j_lo + t,
// j_lo + t + teams, ... of a group, each team accumulating into its own TMEM
// accumulator.  With ksplit = 1 a CTA owns whole rows and writes y; otherwise
// each part writes its row tiles' sums to a slot of the scratch and the last
// part to arrive adds the slots in order.  The ring holds only each tile's
// lane lengths and streams (one bulk copy per tile); the decode warps read the
// raw plane straight from global memory, so a tile held while it is decoded
// costs about a quarter of its chunk.
constexpr int kTcDecodeWarps = 30;
constexpr int kTcEpilogueWarps = 16;  // 4 per TMEM lane quarter read the accumulators
constexpr int kTcMmaWarp = 30;        // TMEM allocation and x loads (TMA)
constexpr int kTcProducerWarp = 31;   // bulk copies of the compressed streams
constexpr int kTcThreads = 32 * 32;
constexpr uint32_t kTcBarBytes = 2048;  // barriers, MMA-warp state, TMEM address, flags
constexpr uint32_t kTcStageA = 1024;    // one row tile: 8 x 64 BF16
constexpr int kTcMaxTeams = 14;
constexpr int kTcTeamBarrier0 = 1;      // named barrier of team t: 1 + t
constexpr int kTcTeardownBarrier = 15;
constexpr int kTcMaxAStages = 3;        // A stages per team (decoded 64-column chunks)
// Accumulator widths (rows of x padded): one launch shape and schedule each.
constexpr int kTcClasses = 3;
constexpr int kTcColumns[kTcClasses] = {16, 32, 64};
inline int tc_class(int rows_of_x) { return rows_of_x <= 16 ? 0 : rows_of_x <= 32 ? 1 : 2; }

struct TcShape {
  LaunchShape s;       // grid, ring and copies (batch_tiles 1); s.xstage_bytes spans barriers, A, B
  int rows;            // R
  int teams;
  int ksplit;          // column ranges (s.ctas is a multiple of it)
  int n;               // accumulator columns of the class
  int bstages;         // x stages per team (1 or 2)
  int astages;         // A stages per team (2 or 3)
  uint32_t bar_off, a_off, b_off;  // shared-memory offsets
};
// Chooses the K split, R, the team count and the x stages for a matrix of
// tiles_r x tiles_c tiles and an accumulator of n columns on a device of
// sm_count SMs and smem_limit bytes of shared memory per block: among the
// layouts whose ring holds every decode warp's streams (max_streams bytes per
// tile at most), the fewest tile decodes on a decode warp's path (M-groups x
// rounds of column blocks of the largest rectangle), then the smallest split,
// then two x stages, then the largest ring; else the layout with the most
// decode warps whose ring still holds a team's tiles and two more (so that no
// team waits for a tile that cannot be issued).  Returns false when nothing
// fits.
bool tc_shape(int64_t tiles_r, int64_t tiles_c, uint64_t max_streams, uint32_t table_bytes,
              int n, int sm_count, size_t smem_limit, TcShape* out);
// The tensor-core kernel's schedule (layout in nwc_format.h) for shape s:
// one copy per tile of its lane lengths and streams (the chunk after its raw
// plane of raw_bytes); `out` receives sched_tc_bytes(tiles) bytes.
void build_tc_schedule(const uint32_t* index, int64_t tiles_r, int64_t tiles_c,
                       uint32_t raw_bytes, const TcShape& s, uint8_t* out);
// tmap: the TMA descriptor of x (BF16 [rows of x][cols], box 64 columns x
// tc_n rows, 128-byte swizzle).
cudaError_t launch_gemv_tc(const TileParams& p, const CUtensorMap& tmap, int tile_cols,
                           int code, const TcShape& s, cudaStream_t stream);

cudaError_t launch_decompress(const TileParams& p, int tile_cols, int code,
                              const LaunchShape& s, cudaStream_t stream);
// Row gather (embedding lookup) from the compressed matrix.
struct GatherParams {
  const uint8_t* tiles;     // device: tile area of the blob
  const uint32_t* index;    // device: chunk offsets (16-byte units), tiles + 1
  const uint32_t* table;    // device: decode table
  uint32_t table_bytes;
  uint32_t stage_bytes;     // per warp: a tile's lane lengths and streams + slack
  int32_t streams;          // bit streams per lane and tile (1 or 2)
  int32_t code;             // kCode12, kCode14, kCodeRank or kCodeEsc
  int32_t peek;             // table peek width (12 or 14)
  int32_t tile_cols;
  int64_t rows, cols, tiles_r, tiles_c;
  const int32_t* row_ids;   // device: n row ids
  int32_t n;
  uint16_t* out;            // device: BF16 [n x cols]
  uint32_t* err;            // device: the handle's error word
};
cudaError_t launch_gather(const GatherParams& g, int sm_count, cudaStream_t stream);

}  // namespace nwc
