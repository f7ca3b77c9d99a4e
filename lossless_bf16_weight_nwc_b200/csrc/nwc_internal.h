// nwc_internal.h — host-side structures shared by the encoder and the C ABI.
#pragma once
#include <cstdint>
#include <vector>

#include "nwc_format.h"

struct nwc_plan_s {
  int64_t rows = 0, cols = 0;
  uint32_t tile_rows = 8, tile_cols = 512, lmax = 7, threads = 0;
  int64_t tiles_r = 0, tiles_c = 0, tiles = 0;
  uint8_t len[256] = {};
  uint32_t code[256] = {};
  uint32_t filler = 0;
  uint64_t coded_bits = 0;
  // Exponent code: 0 = canonical prefix code of bits 14..7 (NWB1), 1 = ranked
  // unary code of bits 14..8 with the sign bit (NWR1), 2 = the prefix code of
  // the kept exponents with verbatim runs for the rest (NWE1).
  uint32_t code_kind = 0;
  uint32_t keep = 0;                         // NWE1: K, the kept exponents
  uint64_t n_escaped = 0;                    // NWE1: verbatim runs
  std::vector<uint8_t> esc_flags;            // NWE1: 8 bytes a tile, bit m of byte g
  uint32_t streams = 1;                      // bit streams per lane and tile (1, 2, 4)
  uint32_t ranks = 0;                        // NWR1: R
  uint8_t rank_table[nwc::kMaxRanks] = {};   // NWR1: ranked values of e
  uint8_t rank_len[128] = {};                // NWR1: bits after the sign bit
  uint32_t rank_code[128] = {};              // NWR1: those bits, right-aligned
  std::vector<uint32_t> index;  // tiles + 1 entries, 16-byte units
  uint64_t tiles_off = 0;       // blob offset of the tile area
  uint64_t blob_bytes = 0;      // serialisable blob
  uint64_t table_off = 0;       // device-image offset of the decode table
  uint64_t sched_off = 0;       // device-image offset of the launch schedule
  uint64_t scratch_off = 0;     // device-image offset of the scratch area
  uint64_t device_bytes = 0;    // blob + padding + decode table + schedules + scratch
};

struct nwc_handle_s {
  uint8_t* d_base = nullptr;  // caller's device buffer
  uint64_t d_bytes = 0;
  int64_t rows = 0, cols = 0;
  uint32_t tile_cols = 512, lmax = 7, filler = 0;
  uint32_t streams = 1;    // bit streams per lane and tile (1 or 2)
  uint32_t code_kind = 0;  // 0: prefix code (NWB1), 1: ranked unary code (NWR1), 2: NWE1
  int64_t tiles_r = 0, tiles_c = 0, tiles = 0;
  uint64_t index_off = 0, tiles_off = 0, blob_bytes = 0, table_off = 0, sched_off = 0,
           scratch_off = 0;
  uint64_t device_bytes = 0;
  uint64_t max_chunk = 0;  // largest chunk in bytes
  int device = 0;
  std::vector<uint32_t> index;  // chunk offsets (16-byte units), tiles + 1
  // Shape each of the device image's launch schedules (one per x-stage
  // class) was written for (0: none yet).
  int sched_ctas[nwc::kStageClasses] = {}, sched_ring[nwc::kStageClasses] = {},
      sched_tiles_per_batch[nwc::kStageClasses] = {};
  // Shape each tensor-core schedule (one per accumulator width) was written
  // for (tc_rows 0: none), and the smallest batch that takes that kernel (0:
  // never).
  int tc_ctas[3] = {}, tc_ring[3] = {}, tc_bstages[3] = {}, tc_rows[3] = {}, tc_teams[3] = {},
      tc_ksplit[3] = {}, tc_astages[3] = {};
  int32_t tc_min_batch = 17;
};

namespace nwc {

// Encoder steps (encoder.cpp).
// streams: bit streams per lane and tile (1, 2 or 4); only 1 has a device
// image (device_bytes = 0 otherwise).
int plan_build(const uint16_t* w, int64_t rows, int64_t cols, uint32_t tile_rows,
               uint32_t tile_cols, uint32_t lmax, uint32_t threads, nwc_plan_s* plan,
               uint32_t streams = 1);
// The ranked unary code (NWR1) with `ranks` ranks (1..7).
int plan_build_rank(const uint16_t* w, int64_t rows, int64_t cols, uint32_t tile_cols,
                    uint32_t ranks, uint32_t threads, nwc_plan_s* plan);
// The kept-exponent prefix code with verbatim runs (NWE1): the `keep` (1..256)
// most frequent exponents coded with lengths <= lmax (0 = 7; at most 7, the
// kernels' 14-bit table).
int plan_build_escape(const uint16_t* w, int64_t rows, int64_t cols, uint32_t tile_cols,
                      uint32_t lmax, uint32_t keep, uint32_t threads, nwc_plan_s* plan);
void encode_blob(const nwc_plan_s& plan, const uint16_t* w, uint8_t* blob);
bool code_lengths(const uint64_t cnt[256], uint32_t lmax, uint8_t len[256]);
void canonical_codes(const uint8_t len[256], uint32_t code[256]);
// Writes table_entries(lmax) entries.
void build_decode_table(const uint8_t len[256], uint32_t lmax, uint32_t* table);
// The device image's table area of a ranked unary code (kRankTableBytes):
// u32[4] = {ranked values 0..3, values 4..6, R, 0}, then zeros.
void build_rank_table(const uint8_t* ranked, uint32_t ranks, uint32_t* out);
// Parses and checks a blob's header, lens and index (the first head_bytes of a
// blob of `bytes` bytes; head_bytes must reach the tile area); fills the
// handle's geometry fields.  Returns false when the blob does not follow the
// format.
bool parse_blob(const uint8_t* blob, uint64_t head_bytes, uint64_t bytes, nwc_handle_s* h,
                const uint8_t** lens_out);
unsigned hardware_threads(uint32_t requested);

}  // namespace nwc
