// nwc_format.h — layout of the "NWB1" blob and of the device image, as the
// library reads and writes them (host and device code).
//
// Byte planes and code: "Unweight: how we compressed an LLM 22% without
// sacrificing quality", section "Compressing BF16 Weights" (exponent bytes
// entropy-coded, sign and mantissa kept); "NWC — Neural Weight Compression",
// "How it works" (byte planes; a 12-bit table peek; blocks of 8 rows x 512
// columns with one bit stream per lane).
//
// Blob: 128-byte header | lens u8[256] | index u32[tiles + 1] | tile chunks.
// A chunk is raw u8[8 * tile_cols] | lane byte counts u8[32] | stream words.
// Stream words are little-endian u32 whose bit 31 is the earliest bit; the 32
// lane streams follow one another, each padded to a byte, the whole run padded
// to 16 bytes.  Lane t = 4g + c owns row g of the tile: its k-th symbol is the
// element (row g, column 64 (k/16) + 16c + k%16), so a 64-column group gives the
// lane 16 consecutive columns of its row; the raw byte is at
// (k/16) * 512 + 16 t + k%16.
// Tiles are stored column-block-major: u = j * tiles_r + i.
// The header's u32 at offset 60 (`zero`) holds S - 1 for S bit streams per
// lane: a lane's symbol pairs go to its S streams in turn, the chunk's length
// array has 32 S entries (lane-major) and the streams follow in that order.
// The kernels read S = 1 and 2 (a decoder follows both streams of a lane at
// once); the C ABI answers UNSUPPORTED for 4.
//
// Device image: blob | zero pad to 256 | decode table u32[table_entries(lmax)]
// | zero pad to 256 | launch schedules (sched_bytes(tiles) bytes: one per
// x-stage class, each sched_class_bytes(tiles)) | scratch (scratch_bytes:
// the error word, the split-K arrival counters and partial sums that the
// kernels write).  None of it is part of the blob: the library writes the
// table and schedules for the device that runs the kernels (its SM count and
// shared memory), each schedule as
//   u32 cta_batch[kMaxCtas + 1]   first batch of each CTA (padded to 16 bytes)
//   u32x4 batch[sched_max_batches(tiles)]
//        {tile-area offset in 16-byte units, bytes, ring offset, batches of
//         the same CTA that must be released before this one is issued}
//   u32 tile_ring[tiles]          ring offset of each tile's chunk
#pragma once
#include <cstdint>

namespace nwc {

constexpr uint32_t kMagic = 0x3142574Eu;  // "NWB1"
// Variant "NWR1": the ranked unary code ("NWC", "How it works > Prefix code
// instead of rANS", format v9).  The same header, index, chunk layout and
// stream packing as NWB1, with: the coded field e = exponent bits 14..8 and the
// sign bit, the raw byte = bits 7..0; the header's lmax field holds R, the
// number of ranks (1..7); its 256-byte lens area holds the ranked values of e
// (R bytes in rank order, then zeros); its filler field the rank-0 value.  A
// weight's code is its sign bit, then r zeros and a one for rank r < R, else R
// zeros and the 7 bits of e.  Every kernel reads it (one stream per lane);
// the device image holds a 256-byte rank table in place of the decode table.
constexpr uint32_t kRankMagic = 0x3152574Eu;  // "NWR1"
constexpr int kMaxRanks = 7;
// Variant "NWE1": rare exponents in verbatim runs ("Unweight", "Compressing
// BF16 Weights": the most common exponents are Huffman-coded; a row of 64
// weights holding any other exponent is stored whole).  NWB1's header, lens,
// index and raw plane, with: the K most frequent exponent bytes kept (header
// offset 60 holds K); run (g, m) of a tile = row g, columns 64 m .. 64 m + 63;
// a run holding an exponent outside the kept set is verbatim; the code covers
// the symbols of the other runs only (so a run is verbatim exactly when it
// holds a symbol without a code).  A chunk is raw u8[8 tile_cols] | flags
// u8[16] (bit m of byte g: run (g, m) verbatim) | the verbatim runs' exponent
// bytes u8[64 n] in (g, m) order | lane lengths u8[32] | streams (one per lane,
// the coded symbols only).  Header offset 104 holds the number of verbatim
// runs (u64).  The kernels read it with lmax <= 7 (the 14-bit table).
constexpr uint32_t kEscMagic = 0x3145574Eu;  // "NWE1"
constexpr uint32_t kEscFlagBytes = 16;
constexpr uint32_t kEscRunBytes = 64;
constexpr uint32_t kEscMaxLmax = 7;
constexpr uint32_t kVersion = 1;
constexpr uint32_t kHeaderBytes = 128;
constexpr uint32_t kLensOffset = 128;
constexpr uint32_t kIndexOffset = 384;
constexpr int kLanes = 32;
constexpr int kTileRows = 8;
constexpr int kMaxTileCols = 512;
constexpr int kMaxLmax = 12;
constexpr int kMaxPeekBits = 14;
constexpr int kMaxStreams = 4;  // bit streams per lane and tile: 1, 2 or 4

// Width of the decoder's table peek for a length limit.  With lmax <= 7 the
// peek is 14 bits, so every entry holds two complete codes and the decoder
// never needs a second lookup ("NWC", "Prefix code instead of rANS": a table
// peek yields two complete codes per step).  Longer codes use a 12-bit peek and
// a second lookup when the pair does not fit.
constexpr int peek_bits(uint32_t lmax) { return lmax <= 7 ? 14 : 12; }
constexpr uint32_t table_entries(uint32_t lmax) { return 1u << peek_bits(lmax); }
constexpr uint32_t table_bytes(uint32_t lmax) { return 4u * table_entries(lmax); }
// The ranked unary code needs no decode table; its device image holds, in the
// table's place, u32[4] = {ranked values 0..3 (bytes), values 4..6, R, 0},
// padded to 256 bytes.
constexpr uint32_t kRankTableBytes = 256;
constexpr uint32_t device_table_bytes(uint32_t lmax, bool rank) {
  return rank ? kRankTableBytes : table_bytes(lmax);
}

// Decode-table entry for one peek (most significant bit = next bit):
//   bits  0..3   bits consumed by the step (both codes, or the first only)
//   bits  7..14  first exponent byte  (its BF16 position in the low half)
//   bits 15..18  length of the first code
//   bit  19      the peek starts with no valid code (corrupt stream)
//   bits 23..30  second exponent byte (its BF16 position in the high half)
//   bit  31      the second code did not fit in the peek (12-bit peek only)
// Bits 4..6 stay zero so that a running difference of entries tracks the
// number of consumed bits in its low 7 bits.
constexpr uint32_t kEntryConsumedMask = 0xFu;
constexpr uint32_t kEntryExponentMask = 0x7F807F80u;
constexpr uint32_t kEntryRawMask = 0x807F807Fu;  // complement of the above
constexpr int kEntryLen0Shift = 15;
constexpr uint32_t kEntryInvalid = 1u << 19;
constexpr uint32_t kEntrySingle = 1u << 31;

constexpr uint64_t round_up(uint64_t v, uint64_t m) { return (v + m - 1) / m * m; }

// Launch-schedule area.  At most kMaxCtas persistent CTAs; every batch but a
// CTA's last holds at least two tiles.
constexpr uint32_t kMaxCtas = 256;
constexpr uint64_t sched_max_batches(uint64_t tiles) { return (tiles + 1) / 2 + kMaxCtas; }
constexpr uint64_t sched_batch_off() { return round_up(4ull * (kMaxCtas + 1), 16); }
constexpr uint64_t sched_tile_off(uint64_t tiles) {
  return sched_batch_off() + 16ull * sched_max_batches(tiles);
}
// One schedule per x-stage class (see kernels.cuh): class 0 for decompression
// and GEMV launches of up to 4 rows of x, class 1 for 5 to 16 rows.
constexpr int kStageClasses = 2;
constexpr uint64_t sched_class_bytes(uint64_t tiles) {
  return round_up(sched_tile_off(tiles) + 4ull * tiles, 256);
}
// The tensor-core kernel's schedules (one per accumulator width) follow the
// class schedules.  Their CTAs take their tiles in another order (row panels,
// see kernels.cuh) and a copy moves one tile's lane lengths and streams (the
// raw plane is read from global memory); they add, per tile, the batch that
// brings it:
//   u32 cta_batch[kMaxCtas + 1] | u32x4 batch[tiles + kMaxCtas]
//   | u32 tile_ring[tiles] | u32 tile_batch[tiles]
// tile_batch = batch index | (extra releases << 28): a batch of fewer tiles
// than the launch's batch_tiles has its first tile release it once more for
// each missing one.  Arrays are indexed by blob tile u = j tiles_r + i.
constexpr uint64_t sched_tc_ring_off(uint64_t tiles) {
  return sched_batch_off() + 16ull * (tiles + kMaxCtas);
}
constexpr uint64_t sched_tc_tbatch_off(uint64_t tiles) { return sched_tc_ring_off(tiles) + 4ull * tiles; }
constexpr uint64_t sched_tc_bytes(uint64_t tiles) {
  return round_up(sched_tc_tbatch_off(tiles) + 4ull * tiles, 256);
}
// One tensor-core schedule per accumulator width (16, 32, 64 columns): the x
// stage, and with it the ring, scales with the rows of x.
constexpr int kTcSchedClasses = 3;
constexpr uint64_t sched_bytes(uint64_t tiles) {
  return kStageClasses * sched_class_bytes(tiles) + kTcSchedClasses * sched_tc_bytes(tiles);
}

// Rows of x one launch of the CUDA-core GEMV kernel handles (one 16-row
// tensor-core operand of mma.sync); larger batches run as several launches.
constexpr int kMaxPassRows = 16;
// Rows of x the tensor-core (tcgen05) kernel handles in one launch.
constexpr int kMaxTcRows = 64;

// Scratch area of the device image, written by the kernels of the handle
// (calls on one handle must therefore be ordered):
//   u32 error word (kErr* bits) | pad to 256
//   u32 arrival counters [tiles_r] | pad to 256
//   FP32 partial sums: the split-K partials of one CUDA-core launch
//   [tiles_c][kMaxPassRows][8 tiles_r], or the tensor-core kernel's partial row
//   tiles when it splits K into ksplit parts [ksplit][tiles_r][kMaxTcRows][8],
//   whichever is larger; none when the matrix has one column tile.  The
//   tensor-core split is at most tc_max_ksplit(tiles_c), which keeps its part
//   no larger than the CUDA-core one.
constexpr uint64_t kScratchCountersOff = 256;
constexpr uint64_t scratch_partial_off(uint64_t tiles_r) {
  return kScratchCountersOff + round_up(4ull * tiles_r, 256);
}
constexpr uint64_t split_partial_bytes(uint64_t tiles_r, uint64_t tiles_c, uint64_t rows_of_x) {
  return tiles_c <= 1 ? 0 : 4ull * tiles_c * rows_of_x * 8ull * tiles_r;
}
constexpr int64_t tc_max_ksplit(int64_t tiles_c) { return tiles_c >= 8 ? tiles_c / 4 : 1; }
constexpr uint64_t tc_partial_bytes(uint64_t tiles_r, uint64_t tiles_c) {
  return tc_max_ksplit((int64_t)tiles_c) <= 1
             ? 0
             : 4ull * (uint64_t)tc_max_ksplit((int64_t)tiles_c) * tiles_r * 8ull *
                   (uint64_t)kMaxTcRows;
}
constexpr uint64_t scratch_bytes(uint64_t tiles_r, uint64_t tiles_c) {
  const uint64_t a = split_partial_bytes(tiles_r, tiles_c, kMaxPassRows),
                 b = tc_partial_bytes(tiles_r, tiles_c);
  return round_up(scratch_partial_off(tiles_r) + (a > b ? a : b), 256);
}

// Offsets of the device image's derived parts after a blob of blob_bytes.
struct ImageLayout {
  uint64_t table_off, sched_off, scratch_off, device_bytes;
};
constexpr ImageLayout image_layout(uint64_t blob_bytes, uint32_t lmax, uint64_t tiles_r,
                                   uint64_t tiles_c, bool rank = false) {
  const uint64_t table_off = round_up(blob_bytes, 256);
  const uint64_t sched_off = round_up(table_off + device_table_bytes(lmax, rank), 256);
  const uint64_t scratch_off = round_up(sched_off + sched_bytes(tiles_r * tiles_c), 256);
  return ImageLayout{table_off, sched_off, scratch_off,
                     scratch_off + scratch_bytes(tiles_r, tiles_c)};
}

struct BlobHeader {
  uint32_t magic, version, header_bytes, lmax;
  uint64_t rows, cols;
  uint32_t tile_rows, tile_cols;
  uint64_t tiles_r, tiles_c;
  uint32_t filler, zero;
  uint64_t lens_off, index_off, tiles_off, total_bytes, coded_bits;
  uint8_t pad[24];
};
static_assert(sizeof(BlobHeader) == 128, "header layout");

// Bytes of one tile's raw plane and the worst-case chunk with S bit streams
// per lane (each holding 16 (tile_cols / 64) / S symbols of at most lmax bits,
// padded to a byte).
constexpr uint32_t raw_bytes(uint32_t tile_cols) { return kTileRows * tile_cols; }
constexpr uint32_t max_chunk_bytes(uint32_t tile_cols, uint32_t lmax, uint32_t streams = 1) {
  return raw_bytes(tile_cols) + kLanes * streams +
         (uint32_t)((kLanes * streams *
                         ((2 * kTileRows * (tile_cols / 64) / streams * lmax + 7) / 8) +
                     15) /
                    16 * 16);
}
// Worst-case NWE1 chunk: every run either verbatim (64 bytes) or coded (4
// lanes x 16 symbols of at most lmax bits), plus each lane's byte padding and
// the 16-byte padding of the streams.
constexpr uint32_t max_escape_chunk_bytes(uint32_t tile_cols, uint32_t lmax) {
  return raw_bytes(tile_cols) + kEscFlagBytes + kLanes +
         kTileRows * (tile_cols / 64) * (8 * lmax > kEscRunBytes ? 8 * lmax : kEscRunBytes) +
         kLanes + 16;
}
// Bit streams per lane that the kernels read (1 or 2).
constexpr uint32_t kMaxDeviceStreams = 2;
// Worst-case chunk of the ranked unary code with R ranks (one stream per
// lane): a code has at most 1 + R + 7 bits.
constexpr uint32_t max_rank_chunk_bytes(uint32_t tile_cols, uint32_t ranks) {
  return raw_bytes(tile_cols) + kLanes +
         (uint32_t)((kLanes * ((2 * kTileRows * (tile_cols / 64) * (ranks + 8) + 7) / 8) + 15) /
                    16 * 16);
}

}  // namespace nwc
