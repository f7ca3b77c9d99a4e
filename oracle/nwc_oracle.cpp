/*
 * nwc_oracle.cpp — the test oracle (plain single-threaded C++).
 *
 * TEST INFRASTRUCTURE ONLY: loaded by tests/, by the smoke check and by the
 * benchmark's CPU-baseline leg; the product library never links or calls it.
 *
 * What the method computes, and where the pages say it:
 *
 *  1. Byte planes.  A BF16 weight (sign 1 | exponent 8 | fraction 7, "Efficient
 *     ML #1 — Deep Learning Data Types" §4) is split into the exponent byte
 *     s = bits 14..7, which is entropy-coded, and the raw byte r = sign << 7 |
 *     fraction, which is stored as is ("Unweight" page, "Compressing BF16
 *     Weights": Huffman on exponent bytes, sign and mantissa unchanged; "NWC"
 *     page, "How it works > Byte planes").
 *  2. Code.  One optimal prefix code per matrix, lengths limited to lmax
 *     (12 by default, the width of the "12-bit peek" in "NWC", "How it works >
 *     Prefix code instead of rANS"), computed with the package-merge algorithm
 *     (Larmore & Hirschberg, 1990) and assigned canonically.
 *  3. Blocks.  The matrix is cut into tiles of 8 rows x tile_cols columns
 *     ("NWC", "Fused kernel": blocks of 8 rows x 512 columns, one bit stream per
 *     lane); each tile is decodable on its own.  Positions outside the matrix
 *     are filled with the most frequent exponent and a zero raw byte ("NWC",
 *     "Fused kernel": padding makes any shape work).
 *
 * Readings where the pages are silent (each one is also listed in the
 * repository's design notes):
 *  - tie-breaks: leaves sorted by (count, symbol); a leaf precedes a package of
 *    equal weight; canonical codes in (length, symbol) order;
 *  - the filler symbol is the most frequent exponent of the real weights
 *    (smallest symbol on a tie), counted in the histogram, raw byte 0;
 *  - a lone symbol gets a 1-bit code.
 *
 * Blob format "NWB1" (all integers little-endian):
 *
 *   header, 128 bytes
 *     0  u32 magic 0x3142574E      4  u32 version = 1
 *     8  u32 header bytes = 128   12  u32 lmax (1..12)
 *    16  u64 rows                  24  u64 cols
 *    32  u32 tile_rows = 8         36  u32 tile_cols (64, 128, 256 or 512)
 *    40  u64 tiles_r = ceil(rows / tile_rows)
 *    48  u64 tiles_c = ceil(cols / tile_cols)
 *    56  u32 filler symbol         60  u32 zero
 *    64  u64 lens offset = 128     72  u64 index offset = 384
 *    80  u64 tiles offset = index offset + 4 * (tiles + 1), rounded up to 256
 *    88  u64 total bytes
 *    96  u64 coded bits = sum of code lengths over all coded symbols
 *   104  24 zero bytes
 *   lens   u8[256]: code length of each exponent byte, 0 = absent
 *   index  u32[tiles + 1]: tile u's chunk starts at tiles offset + 16 * index[u];
 *          index[tiles] = size of the tile area / 16
 *   tiles  one chunk per tile, in order u = j * tiles_r + i for the tile in
 *          row block i and column block j (column-block-major).
 *
 *   chunk of a tile, with CP = tile_cols / 64 and S = 16 * CP symbols per lane:
 *     raw   u8[8 * tile_cols]: lane t's k-th symbol at (k / 16) * 512 + 16 t + k % 16
 *     lens  u8[32]: bytes of each lane's stream
 *     bits  the 32 lane streams one after the other, each the lane's codes in k
 *           order, most significant bit first, zero-padded to a whole byte; the
 *           whole sequence zero-padded to a multiple of 16 bytes and stored as
 *           little-endian 32-bit words in which bit i of the sequence is bit
 *           31 - (i mod 32) of word i / 32.
 *   Lane t = 4 g + c (g = t / 4, c = t mod 4) owns row g of the tile: its k-th
 *   symbol is the element at row g and column 64 * (k / 16) + 16 c + (k mod 16),
 *   i.e. in every 64-column group the lane's 16 consecutive columns, in order.
 *
 *   Streams per lane.  The header's u32 at offset 60 holds S - 1, S in {1, 2,
 *   4} (0: one stream per lane, as above).  With S streams per lane a tile has
 *   32 S streams, stream t S + j belonging to lane t and carrying the lane's
 *   symbols k with (k / 2) mod S == j, in k order: consecutive symbol pairs
 *   go to the lane's streams in turn, so a decoder can follow S independent
 *   streams at once.  The lens array of a chunk then has 32 S entries, in
 *   stream order, and the streams follow one another in that order.  This is
 *   a B200 layout choice, not the pages' (they give one stream per lane).
 *
 * Variant "NWR1", the ranked unary code ("NWC", "How it works > Prefix code
 * instead of rANS": format v9 ranks the exponent by frequency and writes a
 * unary rank code plus a raw sign bit, with an escape for rare values):
 *
 *  1. Planes of the literal byte split ("NWC", "How it works > Byte planes": the
 *     byte holding the sign and the exponent is coded, the other byte stored):
 *     the coded field e = exponent bits 14..8 (7 bits) with the sign bit 15
 *     beside it; the raw byte is bits 7..0 (the exponent's lowest bit and the
 *     fraction).
 *  2. Ranks: the values of e ordered by count over the real weights and the
 *     fillers, largest count first, smaller value first on a tie; the first
 *     R = min(ranks, number of values present) of them get ranks 0 .. R - 1,
 *     with ranks in 1..7 (a code then has at most 15 bits and a lane's stream
 *     at most 240 bytes).
 *  3. Code of a weight, most significant bit first: its sign bit; then, if its
 *     e has rank r < R, r zero bits and a one bit; otherwise R zero bits and
 *     the 7 bits of e (the escape).
 *  4. Tiles, lanes, chunk layout, index and stream packing are those of NWB1;
 *     the raw plane holds bits 7..0.  Filler positions hold sign 0, the rank-0
 *     value of e and raw byte 0.
 *
 *   header differences from NWB1: magic 0x3152574E ("NWR1"); offset 12 holds
 *   R; offset 56 the rank-0 value of e (the filler's); offset 96 the total
 *   code bits; the 256 bytes at offset 128 hold the ranked values of e, rank
 *   order, then zeros.
 *
 * Readings where the v9 passage is silent: the sign bit comes first, a rank is
 * counted in zero bits ended by a one, the escape is the 7-bit field after R
 * zero bits, R = 7 by default.
 *
 * Variant "NWE1", rare exponents in verbatim runs ("Unweight", "Compressing
 * BF16 Weights": the 16 most common exponents cover nearly all weights of a
 * layer and are Huffman-coded; a row of 64 weights that holds any other
 * exponent is stored verbatim, so the decoder branches once per run, not per
 * weight):
 *
 *  1. Planes and filler as NWB1.
 *  2. Kept symbols: the K most frequent exponent bytes over the real weights
 *     and the fillers (largest count first, smaller symbol first on a tie;
 *     K = min(keep, number present), keep = 16 by default).  The filler is
 *     always kept.
 *  3. Runs: in a tile, run (g, m) is row g and the columns 64 m .. 64 m + 63 of
 *     the tile (64 consecutive weights of one matrix row; fillers past the
 *     edge).  A run is escaped when one of its 64 exponent bytes is not kept.
 *     It is the 16-symbol slice of lanes 4 g .. 4 g + 3 in group m.
 *  4. Code: the optimal code limited to lmax bits over the counts of the
 *     symbols of the runs that are not escaped, assigned canonically as in
 *     NWB1 (all lengths 0 when every run is escaped).  So a run is escaped
 *     exactly when it holds a symbol without a code.
 *  5. Chunk of a tile:
 *       raw    u8[8 * tile_cols], as NWB1 (every position, escaped or not)
 *       flags  u8[16]: bit m of byte g set when run (g, m) is escaped; bits
 *              m >= tile_cols / 64 and bytes 8 .. 15 zero
 *       runs   u8[64 * n]: the exponent bytes of the tile's n escaped runs in
 *              (g, m) order, each run's 64 bytes in column order (lane 4 g + c
 *              finds its 16 at byte 16 c of the run)
 *       lens   u8[32] and bits: as NWB1 with one stream per lane, the streams
 *              holding the codes of the symbols of the runs not escaped only.
 *     An escaped run costs 16 bits per weight (its raw bytes and its exponent
 *     bytes), as a run stored verbatim does.
 *
 *   header differences from NWB1: magic 0x3145574E ("NWE1"); offset 60 holds
 *   K; offset 96 the total code bits; offset 104 the number of escaped runs
 *   (u64).  lens[256] as NWB1.
 *
 * Readings where the passage is silent: the run is aligned to 64 columns of
 * the tile (so to 64 columns of the matrix), the exponent bytes of an escaped
 * run sit in the chunk and its raw bytes stay in the raw plane (16 bits per
 * weight either way), the kept set counts the fillers.
 */
#include "nwc_oracle.h"

#include <algorithm>
#include <cstring>
#include <vector>

namespace {

const uint32_t kMagic = 0x3142574Eu;
const uint32_t kVersion = 1;
const int kHeaderBytes = 128;
const int kLanes = 32;

void put_u32(uint8_t* p, uint32_t v) {
  for (int i = 0; i < 4; ++i) p[i] = (uint8_t)(v >> (8 * i));
}
void put_u64(uint8_t* p, uint64_t v) {
  for (int i = 0; i < 8; ++i) p[i] = (uint8_t)(v >> (8 * i));
}
uint32_t get_u32(const uint8_t* p) {
  uint32_t v = 0;
  for (int i = 0; i < 4; ++i) v |= (uint32_t)p[i] << (8 * i);
  return v;
}
uint64_t get_u64(const uint8_t* p) {
  uint64_t v = 0;
  for (int i = 0; i < 8; ++i) v |= (uint64_t)p[i] << (8 * i);
  return v;
}
uint64_t round_up(uint64_t v, uint64_t m) { return (v + m - 1) / m * m; }

/* Tile element of lane t's k-th symbol ("NWC", "Fused kernel": each lane owns
 * one bit stream of the block; which elements it owns is not fixed there).
 * Here lane t = 4 g + c owns row g and, in every 64-column group, the 16
 * consecutive columns from 16 c on, taken in order. */
void lane_symbol_position(int t, int k, int* r, int* c) {
  *r = t / 4;
  *c = 64 * (k / 16) + 16 * (t % 4) + (k % 16);
}
int raw_position(int t, int k) { return (k / 16) * 512 + 16 * t + (k % 16); }

/* Geometry checks shared by the encoder and the decoder. */
bool geometry_ok(int tile_rows, int tile_cols, int lmax) {
  if (tile_rows != 8) return false;
  if (tile_cols < 64 || tile_cols > 512 || tile_cols % 64 != 0) return false;
  if (lmax < 1 || lmax > 12) return false;
  return true;
}

/* One item of the package-merge lists: its weight and how many times each
 * leaf symbol occurs inside it. */
struct Item {
  uint64_t weight;
  bool leaf;
  int symbol;                  /* leaves only, for ordering */
  std::vector<uint16_t> uses;  /* uses[s] = occurrences of leaf s */
};

/* Most frequent symbol, smallest on a tie. */
int filler_symbol(const uint64_t cnt[256]) {
  int best = 0;
  for (int s = 1; s < 256; ++s)
    if (cnt[s] > cnt[best]) best = s;
  return best;
}

/* Sub-stream of lane t that carries its k-th symbol when each lane has
 * `streams` streams: consecutive symbol pairs go to the lane's streams in
 * turn (see "Streams per lane" in the format statement). */
int stream_of(int t, int k, int streams) { return t * streams + (k / 2) % streams; }

/* The encoder proper; blob == nullptr only measures. */
int encode_impl(const uint16_t* w, int64_t rows, int64_t cols, int tile_rows,
                int tile_cols, int lmax, int streams, uint8_t* blob, int64_t cap,
                int64_t* size) {
  if (!w || rows < 1 || cols < 1 || !size) return ORC_E_ARG;
  if (!geometry_ok(tile_rows, tile_cols, lmax)) return ORC_E_ARG;
  if (streams != 1 && streams != 2 && streams != 4) return ORC_E_ARG;
  const int nstreams = kLanes * streams;

  const int64_t tiles_r = (rows + tile_rows - 1) / tile_rows;
  const int64_t tiles_c = (cols + tile_cols - 1) / tile_cols;
  const int64_t tiles = tiles_r * tiles_c;
  const int lane_syms = 2 * tile_rows * (tile_cols / 64);
  const int raw_bytes = tile_rows * tile_cols;

  /* Histogram of the real weights, then the fillers on the filler symbol. */
  uint64_t cnt[256];
  orc_histogram(w, rows, cols, cnt);
  const int filler = filler_symbol(cnt);
  const uint64_t fillers =
      (uint64_t)(tiles_r * tile_rows) * (uint64_t)(tiles_c * tile_cols) -
      (uint64_t)rows * (uint64_t)cols;
  cnt[filler] += fillers;

  uint8_t len[256];
  int rc = orc_code_lengths(cnt, lmax, len);
  if (rc != ORC_OK) return rc;
  uint32_t code[256];
  orc_canonical_codes(len, code);

  uint64_t coded_bits = 0;
  for (int s = 0; s < 256; ++s) coded_bits += cnt[s] * (uint64_t)len[s];

  const uint64_t lens_off = kHeaderBytes;
  const uint64_t index_off = lens_off + 256;
  const uint64_t tiles_off = round_up(index_off + 4 * (uint64_t)(tiles + 1), 256);

  /* Pass over the tiles: build each chunk, then copy it out. */
  std::vector<uint8_t> chunk;
  std::vector<uint32_t> index((size_t)tiles + 1);
  uint64_t area = 0;
  for (int64_t u = 0; u < tiles; ++u) {
    const int64_t i = u % tiles_r; /* row block */
    const int64_t j = u / tiles_r; /* column block */
    std::vector<uint8_t> raw((size_t)raw_bytes, 0);
    std::vector<std::vector<uint8_t> > lane_bits((size_t)nstreams);  /* one entry per bit */
    for (int t = 0; t < kLanes; ++t) {
      for (int k = 0; k < lane_syms; ++k) {
        int r, c;
        lane_symbol_position(t, k, &r, &c);
        const int64_t row = i * tile_rows + r;
        const int64_t col = j * tile_cols + c;
        uint8_t s = (uint8_t)filler, rb = 0;
        if (row < rows && col < cols) orc_plane_split(w[row * cols + col], &s, &rb);
        raw[(size_t)raw_position(t, k)] = rb;
        for (int b = len[s] - 1; b >= 0; --b)
          lane_bits[(size_t)stream_of(t, k, streams)].push_back((uint8_t)((code[s] >> b) & 1u));
      }
    }
    /* Concatenate the byte-padded streams, in stream order. */
    std::vector<uint8_t> seq;  /* one entry per bit */
    std::vector<uint8_t> lane_bytes((size_t)nstreams);
    for (int t = 0; t < nstreams; ++t) {
      std::vector<uint8_t>& lb = lane_bits[(size_t)t];
      while (lb.size() % 8 != 0) lb.push_back(0);
      if (lb.size() / 8 > 255) return ORC_E_ARG; /* cannot happen for lmax <= 12 */
      lane_bytes[(size_t)t] = (uint8_t)(lb.size() / 8);
      seq.insert(seq.end(), lb.begin(), lb.end());
    }
    while (seq.size() % 128 != 0) seq.push_back(0); /* 16 bytes */
    /* Words: bit i of the sequence -> bit 31 - i % 32 of word i / 32. */
    std::vector<uint8_t> bits(seq.size() / 8, 0);
    for (size_t b = 0; b < seq.size(); ++b) {
      if (!seq[b]) continue;
      const size_t word = b / 32;
      const int bit = 31 - (int)(b % 32);
      bits[word * 4 + (size_t)(bit / 8)] |= (uint8_t)(1u << (bit % 8));
    }
    chunk.clear();
    chunk.insert(chunk.end(), raw.begin(), raw.end());
    chunk.insert(chunk.end(), lane_bytes.begin(), lane_bytes.end());
    chunk.insert(chunk.end(), bits.begin(), bits.end());
    index[(size_t)u] = (uint32_t)(area / 16);
    if (area / 16 > 0xFFFFFFFFull) return ORC_E_ARG;
    if (blob) {
      if ((int64_t)(tiles_off + area + chunk.size()) > cap) return ORC_E_SPACE;
      std::memcpy(blob + tiles_off + area, chunk.data(), chunk.size());
    }
    area += chunk.size();
  }
  if (area / 16 > 0xFFFFFFFFull) return ORC_E_ARG;
  index[(size_t)tiles] = (uint32_t)(area / 16);
  const uint64_t total = tiles_off + area;
  *size = (int64_t)total;
  if (!blob) return ORC_OK;
  if ((int64_t)total > cap) return ORC_E_SPACE;

  std::memset(blob, 0, (size_t)tiles_off);
  put_u32(blob + 0, kMagic);
  put_u32(blob + 4, kVersion);
  put_u32(blob + 8, kHeaderBytes);
  put_u32(blob + 12, (uint32_t)lmax);
  put_u64(blob + 16, (uint64_t)rows);
  put_u64(blob + 24, (uint64_t)cols);
  put_u32(blob + 32, (uint32_t)tile_rows);
  put_u32(blob + 36, (uint32_t)tile_cols);
  put_u64(blob + 40, (uint64_t)tiles_r);
  put_u64(blob + 48, (uint64_t)tiles_c);
  put_u32(blob + 56, (uint32_t)filler);
  put_u32(blob + 60, (uint32_t)(streams - 1));
  put_u64(blob + 64, lens_off);
  put_u64(blob + 72, index_off);
  put_u64(blob + 80, tiles_off);
  put_u64(blob + 88, total);
  put_u64(blob + 96, coded_bits);
  std::memcpy(blob + lens_off, len, 256);
  for (int64_t u = 0; u <= tiles; ++u) put_u32(blob + index_off + 4 * u, index[(size_t)u]);
  return ORC_OK;
}

struct Header {
  int64_t rows, cols, tiles_r, tiles_c;
  int tile_rows, tile_cols, lmax, filler, streams;
  uint64_t lens_off, index_off, tiles_off, total;
};

int read_header(const uint8_t* blob, int64_t size, Header* h) {
  if (!blob || size < kHeaderBytes) return ORC_E_CORRUPT;
  if (get_u32(blob) != kMagic || get_u32(blob + 4) != kVersion ||
      get_u32(blob + 8) != (uint32_t)kHeaderBytes)
    return ORC_E_CORRUPT;
  h->lmax = (int)get_u32(blob + 12);
  h->rows = (int64_t)get_u64(blob + 16);
  h->cols = (int64_t)get_u64(blob + 24);
  h->tile_rows = (int)get_u32(blob + 32);
  h->tile_cols = (int)get_u32(blob + 36);
  h->tiles_r = (int64_t)get_u64(blob + 40);
  h->tiles_c = (int64_t)get_u64(blob + 48);
  h->filler = (int)get_u32(blob + 56);
  h->streams = (int)get_u32(blob + 60) + 1;
  h->lens_off = get_u64(blob + 64);
  h->index_off = get_u64(blob + 72);
  h->tiles_off = get_u64(blob + 80);
  h->total = get_u64(blob + 88);
  if (h->rows < 1 || h->cols < 1) return ORC_E_CORRUPT;
  if (!geometry_ok(h->tile_rows, h->tile_cols, h->lmax)) return ORC_E_CORRUPT;
  if (h->tiles_r != (h->rows + h->tile_rows - 1) / h->tile_rows) return ORC_E_CORRUPT;
  if (h->tiles_c != (h->cols + h->tile_cols - 1) / h->tile_cols) return ORC_E_CORRUPT;
  if (h->filler < 0 || h->filler > 255) return ORC_E_CORRUPT;
  if (h->streams != 1 && h->streams != 2 && h->streams != 4) return ORC_E_CORRUPT;
  const uint64_t tiles = (uint64_t)(h->tiles_r * h->tiles_c);
  if (h->lens_off != (uint64_t)kHeaderBytes || h->index_off != h->lens_off + 256)
    return ORC_E_CORRUPT;
  if (h->tiles_off != round_up(h->index_off + 4 * (tiles + 1), 256)) return ORC_E_CORRUPT;
  if (h->total != (uint64_t)size) return ORC_E_CORRUPT;
  return ORC_OK;
}

/* Decode tiles [u0, u1) into out (full matrix buffer). */
int decode_impl(const uint8_t* blob, int64_t size, int64_t u0, int64_t u1,
                uint16_t* out, int64_t cap_elems) {
  Header h;
  int rc = read_header(blob, size, &h);
  if (rc != ORC_OK) return rc;
  if (!out || cap_elems < h.rows * h.cols) return ORC_E_SPACE;
  const int64_t tiles = h.tiles_r * h.tiles_c;
  if (u0 < 0 || u1 > tiles || u0 > u1) return ORC_E_ARG;

  /* Code table from the lengths: Kraft sum must not exceed one. */
  uint8_t len[256];
  std::memcpy(len, blob + h.lens_off, 256);
  double kraft = 0.0;
  for (int s = 0; s < 256; ++s) {
    if (len[s] > h.lmax) return ORC_E_CORRUPT;
    if (len[s]) kraft += 1.0 / (double)(1u << len[s]);
  }
  if (kraft > 1.0 || kraft == 0.0) return ORC_E_CORRUPT;
  if (len[h.filler] == 0) return ORC_E_CORRUPT;
  uint32_t code[256];
  orc_canonical_codes(len, code);
  /* sym_of[l][v] = symbol whose code has length l and value v, or -1. */
  std::vector<std::vector<int> > sym_of(13);
  for (int l = 1; l <= 12; ++l) sym_of[(size_t)l].assign((size_t)1 << l, -1);
  for (int s = 0; s < 256; ++s)
    if (len[s]) sym_of[len[s]][code[s]] = s;

  const int lane_syms = 2 * h.tile_rows * (h.tile_cols / 64);
  const int raw_bytes = h.tile_rows * h.tile_cols;
  const uint64_t area = (uint64_t)size - h.tiles_off;
  for (int64_t u = u0; u < u1; ++u) {
    const uint64_t c0 = 16ull * get_u32(blob + h.index_off + 4 * u);
    const uint64_t c1 = 16ull * get_u32(blob + h.index_off + 4 * (u + 1));
    if (c1 < c0 || c1 > area) return ORC_E_CORRUPT;
    const uint8_t* chunk = blob + h.tiles_off + c0;
    const uint64_t chunk_bytes = c1 - c0;
    const int nstreams = kLanes * h.streams;
    if (chunk_bytes < (uint64_t)raw_bytes + nstreams) return ORC_E_CORRUPT;
    const uint8_t* raw = chunk;
    const uint8_t* lane_bytes = chunk + raw_bytes;
    const uint8_t* bits = chunk + raw_bytes + nstreams;
    uint64_t stream_bytes = 0;
    for (int t = 0; t < nstreams; ++t) stream_bytes += lane_bytes[t];
    if (chunk_bytes != (uint64_t)raw_bytes + nstreams + round_up(stream_bytes, 16))
      return ORC_E_CORRUPT;
    const uint64_t nbits = 8 * round_up(stream_bytes, 16);
    /* Bit i of the sequence is bit 31 - i % 32 of little-endian word i / 32. */
    auto bit_at = [&](uint64_t i) -> int {
      const uint64_t word = i / 32;
      const int b = 31 - (int)(i % 32);
      return (bits[word * 4 + (uint64_t)(b / 8)] >> (b % 8)) & 1;
    };
    const int64_t i = u % h.tiles_r, j = u / h.tiles_r;
    uint64_t lane_start = 0;
    for (int sigma = 0; sigma < nstreams; ++sigma) {
      /* Stream sigma belongs to lane t and carries the lane's symbols k with
       * stream_of(t, k) == sigma, in k order. */
      const int t = sigma / h.streams;
      uint64_t pos = lane_start;
      const uint64_t end = lane_start + 8ull * lane_bytes[sigma];
      for (int k = 0; k < lane_syms; ++k) {
        if (stream_of(t, k, h.streams) != sigma) continue;
        /* Read bits one at a time until they spell a code. */
        uint32_t v = 0;
        int l = 0, s = -1;
        while (s < 0) {
          if (pos >= end || l >= h.lmax) return ORC_E_CORRUPT;
          v = (v << 1) | (uint32_t)bit_at(pos++);
          ++l;
          s = sym_of[(size_t)l][v];
        }
        const uint8_t rb = raw[raw_position(t, k)];
        int r, c;
        lane_symbol_position(t, k, &r, &c);
        const int64_t row = i * h.tile_rows + r;
        const int64_t col = j * h.tile_cols + c;
        if (row < h.rows && col < h.cols) {
          out[row * h.cols + col] = orc_plane_join((uint8_t)s, rb);
        } else if (s != h.filler || rb != 0) {
          return ORC_E_CORRUPT; /* filler positions hold (filler, 0) */
        }
      }
      /* Stream padding must be zero and must not reach a whole byte. */
      if (end - pos >= 8) return ORC_E_CORRUPT;
      while (pos < end)
        if (bit_at(pos++)) return ORC_E_CORRUPT;
      lane_start = end;
    }
    for (uint64_t p = lane_start; p < nbits; ++p)
      if (bit_at(p)) return ORC_E_CORRUPT;
  }
  return ORC_OK;
}

/* ---- Variant NWR1: the ranked unary code ---------------------------------- */

const uint32_t kRankMagic = 0x3152574Eu;
const int kMaxRanks = 7;

/* Literal byte split: e = exponent bits 14..8, the sign bit 15, raw = bits 7..0. */
void rank_split(uint16_t w, int* e, int* sign, uint8_t* raw) {
  *e = (w >> 8) & 0x7F;
  *sign = (w >> 15) & 1;
  *raw = (uint8_t)(w & 0xFF);
}

uint16_t rank_join(int e, int sign, uint8_t raw) {
  return (uint16_t)(((uint16_t)sign << 15) | ((uint16_t)e << 8) | raw);
}

/* Values of e by count (largest first, smaller value on a tie); at most
 * `ranks` of those present.  Returns how many were ranked. */
int rank_order(const uint64_t cnt[128], int ranks, uint8_t table[kMaxRanks]) {
  std::vector<int> present;
  for (int e = 0; e < 128; ++e)
    if (cnt[e] > 0) present.push_back(e);
  std::stable_sort(present.begin(), present.end(),
                   [&](int a, int b) { return cnt[a] > cnt[b]; });
  const int n = (int)std::min<size_t>(present.size(), (size_t)ranks);
  for (int r = 0; r < n; ++r) table[r] = (uint8_t)present[(size_t)r];
  return n;
}

/* Appends the code of one weight to a lane's bit list. */
void rank_code_bits(int e, int sign, const uint8_t table[kMaxRanks], int ranks,
                    std::vector<uint8_t>* bits) {
  bits->push_back((uint8_t)sign);
  int r = 0;
  while (r < ranks && table[r] != e) ++r;
  for (int z = 0; z < r; ++z) bits->push_back(0);
  if (r < ranks) {
    bits->push_back(1);
  } else {
    for (int b = 6; b >= 0; --b) bits->push_back((uint8_t)((e >> b) & 1));
  }
}

int encode_rank_impl(const uint16_t* w, int64_t rows, int64_t cols, int tile_rows,
                     int tile_cols, int ranks, uint8_t* blob, int64_t cap, int64_t* size) {
  if (!w || rows < 1 || cols < 1 || !size) return ORC_E_ARG;
  if (!geometry_ok(tile_rows, tile_cols, 12) || ranks < 1 || ranks > kMaxRanks)
    return ORC_E_ARG;
  const int64_t tiles_r = (rows + tile_rows - 1) / tile_rows;
  const int64_t tiles_c = (cols + tile_cols - 1) / tile_cols;
  const int64_t tiles = tiles_r * tiles_c;
  const int lane_syms = 2 * tile_rows * (tile_cols / 64);
  const int raw_bytes = tile_rows * tile_cols;

  /* Counts of e over the real weights; the filler takes the most frequent
   * value (smallest on a tie), then the fillers are counted. */
  uint64_t cnt[128] = {};
  for (int64_t q = 0; q < rows * cols; ++q) {
    int e, sign;
    uint8_t raw;
    rank_split(w[q], &e, &sign, &raw);
    cnt[e] += 1;
  }
  int filler = 0;
  for (int e = 1; e < 128; ++e)
    if (cnt[e] > cnt[filler]) filler = e;
  cnt[filler] += (uint64_t)(tiles_r * tile_rows) * (uint64_t)(tiles_c * tile_cols) -
                 (uint64_t)rows * (uint64_t)cols;
  uint8_t table[kMaxRanks] = {};
  const int R = rank_order(cnt, ranks, table);

  const uint64_t table_off = kHeaderBytes;
  const uint64_t index_off = table_off + 256;
  const uint64_t tiles_off = round_up(index_off + 4 * (uint64_t)(tiles + 1), 256);
  std::vector<uint32_t> index((size_t)tiles + 1);
  uint64_t area = 0, code_bits = 0;
  for (int64_t u = 0; u < tiles; ++u) {
    const int64_t i = u % tiles_r, j = u / tiles_r;
    std::vector<uint8_t> raw((size_t)raw_bytes, 0);
    std::vector<uint8_t> seq;  /* one entry per bit */
    uint8_t lane_bytes[kLanes];
    for (int t = 0; t < kLanes; ++t) {
      std::vector<uint8_t> lb;
      for (int k = 0; k < lane_syms; ++k) {
        int r, c;
        lane_symbol_position(t, k, &r, &c);
        const int64_t row = i * tile_rows + r, col = j * tile_cols + c;
        int e = filler, sign = 0;
        uint8_t rb = 0;
        if (row < rows && col < cols) rank_split(w[row * cols + col], &e, &sign, &rb);
        raw[(size_t)raw_position(t, k)] = rb;
        rank_code_bits(e, sign, table, R, &lb);
      }
      code_bits += lb.size();
      while (lb.size() % 8 != 0) lb.push_back(0);
      lane_bytes[t] = (uint8_t)(lb.size() / 8);
      seq.insert(seq.end(), lb.begin(), lb.end());
    }
    while (seq.size() % 128 != 0) seq.push_back(0);
    std::vector<uint8_t> bits(seq.size() / 8, 0);
    for (size_t b = 0; b < seq.size(); ++b) {
      if (!seq[b]) continue;
      const int bit = 31 - (int)(b % 32);
      bits[(b / 32) * 4 + (size_t)(bit / 8)] |= (uint8_t)(1u << (bit % 8));
    }
    index[(size_t)u] = (uint32_t)(area / 16);
    const uint64_t chunk = (uint64_t)raw_bytes + kLanes + bits.size();
    if (blob) {
      if ((int64_t)(tiles_off + area + chunk) > cap) return ORC_E_SPACE;
      uint8_t* p = blob + tiles_off + area;
      std::memcpy(p, raw.data(), raw.size());
      std::memcpy(p + raw_bytes, lane_bytes, kLanes);
      std::memcpy(p + raw_bytes + kLanes, bits.data(), bits.size());
    }
    area += chunk;
    if (area / 16 > 0xFFFFFFFFull) return ORC_E_ARG;
  }
  index[(size_t)tiles] = (uint32_t)(area / 16);
  const uint64_t total = tiles_off + area;
  *size = (int64_t)total;
  if (!blob) return ORC_OK;
  if ((int64_t)total > cap) return ORC_E_SPACE;
  std::memset(blob, 0, (size_t)tiles_off);
  put_u32(blob + 0, kRankMagic);
  put_u32(blob + 4, kVersion);
  put_u32(blob + 8, kHeaderBytes);
  put_u32(blob + 12, (uint32_t)R);
  put_u64(blob + 16, (uint64_t)rows);
  put_u64(blob + 24, (uint64_t)cols);
  put_u32(blob + 32, (uint32_t)tile_rows);
  put_u32(blob + 36, (uint32_t)tile_cols);
  put_u64(blob + 40, (uint64_t)tiles_r);
  put_u64(blob + 48, (uint64_t)tiles_c);
  put_u32(blob + 56, (uint32_t)filler);
  put_u64(blob + 64, table_off);
  put_u64(blob + 72, index_off);
  put_u64(blob + 80, tiles_off);
  put_u64(blob + 88, total);
  put_u64(blob + 96, code_bits);
  std::memcpy(blob + table_off, table, (size_t)R);
  for (int64_t u = 0; u <= tiles; ++u) put_u32(blob + index_off + 4 * u, index[(size_t)u]);
  return ORC_OK;
}

int decode_rank_impl(const uint8_t* blob, int64_t size, uint16_t* out, int64_t cap_elems) {
  if (!blob || size < kHeaderBytes + 256) return ORC_E_CORRUPT;
  if (get_u32(blob) != kRankMagic || get_u32(blob + 4) != kVersion ||
      get_u32(blob + 8) != (uint32_t)kHeaderBytes)
    return ORC_E_CORRUPT;
  const int R = (int)get_u32(blob + 12);
  const int64_t rows = (int64_t)get_u64(blob + 16), cols = (int64_t)get_u64(blob + 24);
  const int tile_rows = (int)get_u32(blob + 32), tile_cols = (int)get_u32(blob + 36);
  const int64_t tiles_r = (int64_t)get_u64(blob + 40), tiles_c = (int64_t)get_u64(blob + 48);
  const int filler = (int)get_u32(blob + 56);
  const uint64_t table_off = get_u64(blob + 64), index_off = get_u64(blob + 72);
  const uint64_t tiles_off = get_u64(blob + 80), total = get_u64(blob + 88);
  if (rows < 1 || cols < 1 || !geometry_ok(tile_rows, tile_cols, 12)) return ORC_E_CORRUPT;
  if (R < 1 || R > kMaxRanks) return ORC_E_CORRUPT;
  if (tiles_r != (rows + tile_rows - 1) / tile_rows ||
      tiles_c != (cols + tile_cols - 1) / tile_cols)
    return ORC_E_CORRUPT;
  const int64_t tiles = tiles_r * tiles_c;
  if (table_off != (uint64_t)kHeaderBytes || index_off != table_off + 256 ||
      tiles_off != round_up(index_off + 4 * (uint64_t)(tiles + 1), 256) ||
      total != (uint64_t)size)
    return ORC_E_CORRUPT;
  /* The ranked values: distinct 7-bit values, then zeros; rank 0 is the filler's. */
  uint8_t table[kMaxRanks] = {};
  for (int r = 0; r < 256; ++r) {
    const uint8_t v = blob[table_off + (uint64_t)r];
    if (r >= R) {
      if (v) return ORC_E_CORRUPT;
      continue;
    }
    if (v > 127) return ORC_E_CORRUPT;
    for (int q = 0; q < r; ++q)
      if (table[q] == v) return ORC_E_CORRUPT;
    table[r] = v;
  }
  if (filler != table[0]) return ORC_E_CORRUPT;
  if (!out || cap_elems < rows * cols) return ORC_E_SPACE;

  const int lane_syms = 2 * tile_rows * (tile_cols / 64);
  const int raw_bytes = tile_rows * tile_cols;
  const uint64_t area = (uint64_t)size - tiles_off;
  for (int64_t u = 0; u < tiles; ++u) {
    const uint64_t c0 = 16ull * get_u32(blob + index_off + 4 * u);
    const uint64_t c1 = 16ull * get_u32(blob + index_off + 4 * (u + 1));
    if (c1 < c0 || c1 > area || c1 - c0 < (uint64_t)raw_bytes + kLanes) return ORC_E_CORRUPT;
    const uint8_t* chunk = blob + tiles_off + c0;
    const uint8_t* raw = chunk;
    const uint8_t* lane_bytes = chunk + raw_bytes;
    const uint8_t* bits = chunk + raw_bytes + kLanes;
    uint64_t stream_bytes = 0;
    for (int t = 0; t < kLanes; ++t) stream_bytes += lane_bytes[t];
    if (c1 - c0 != (uint64_t)raw_bytes + kLanes + round_up(stream_bytes, 16))
      return ORC_E_CORRUPT;
    auto bit_at = [&](uint64_t q) -> int {
      const int b = 31 - (int)(q % 32);
      return (bits[(q / 32) * 4 + (uint64_t)(b / 8)] >> (b % 8)) & 1;
    };
    const int64_t i = u % tiles_r, j = u / tiles_r;
    uint64_t lane_start = 0;
    for (int t = 0; t < kLanes; ++t) {
      uint64_t pos = lane_start;
      const uint64_t end = lane_start + 8ull * lane_bytes[t];
      auto next = [&](int* bit) -> bool {
        if (pos >= end) return false;
        *bit = bit_at(pos++);
        return true;
      };
      for (int k = 0; k < lane_syms; ++k) {
        int sign, b, zeros = 0, e;
        if (!next(&sign)) return ORC_E_CORRUPT;
        bool ended = false;
        while (zeros < R) {
          if (!next(&b)) return ORC_E_CORRUPT;
          if (b) {
            ended = true;
            break;
          }
          ++zeros;
        }
        if (ended) {
          e = table[zeros];
        } else {
          e = 0;
          for (int q = 0; q < 7; ++q) {
            if (!next(&b)) return ORC_E_CORRUPT;
            e = (e << 1) | b;
          }
          for (int q = 0; q < R; ++q)
            if (table[q] == e) return ORC_E_CORRUPT; /* a ranked value is never escaped */
        }
        const uint8_t rb = raw[raw_position(t, k)];
        int r, c;
        lane_symbol_position(t, k, &r, &c);
        const int64_t row = i * tile_rows + r, col = j * tile_cols + c;
        if (row < rows && col < cols) {
          out[row * cols + col] = rank_join(e, sign, rb);
        } else if (sign != 0 || e != filler || rb != 0) {
          return ORC_E_CORRUPT;
        }
      }
      if (end - pos >= 8) return ORC_E_CORRUPT;
      while (pos < end)
        if (bit_at(pos++)) return ORC_E_CORRUPT;
      lane_start = end;
    }
    for (uint64_t q = lane_start; q < 8 * round_up(stream_bytes, 16); ++q)
      if (bit_at(q)) return ORC_E_CORRUPT;
  }
  return ORC_OK;
}

/* ---- Variant NWE1: rare exponents in verbatim runs ------------------------ */

const uint32_t kEscMagic = 0x3145574Eu;

/* The `keep` most frequent symbols (largest count first, smaller symbol on a
 * tie) among those present.  Returns how many were kept. */
int kept_symbols(const uint64_t cnt[256], int keep, bool kept[256]) {
  std::vector<int> present;
  for (int s = 0; s < 256; ++s) {
    kept[s] = false;
    if (cnt[s] > 0) present.push_back(s);
  }
  std::stable_sort(present.begin(), present.end(),
                   [&](int x, int y) { return cnt[x] > cnt[y]; });
  const int n = (int)std::min<size_t>(present.size(), (size_t)keep);
  for (int q = 0; q < n; ++q) kept[present[(size_t)q]] = true;
  return n;
}

/* Exponent byte and raw byte of tile element (r, c) of tile (i, j); the filler
 * outside the matrix. */
void tile_element(const uint16_t* w, int64_t rows, int64_t cols, int64_t i, int64_t j,
                  int tile_rows, int tile_cols, int filler, int r, int c, uint8_t* s,
                  uint8_t* rb) {
  const int64_t row = i * tile_rows + r, col = j * tile_cols + c;
  *s = (uint8_t)filler;
  *rb = 0;
  if (row < rows && col < cols) orc_plane_split(w[row * cols + col], s, rb);
}

int encode_escape_impl(const uint16_t* w, int64_t rows, int64_t cols, int tile_rows,
                       int tile_cols, int lmax, int keep, uint8_t* blob, int64_t cap,
                       int64_t* size) {
  if (!w || rows < 1 || cols < 1 || !size) return ORC_E_ARG;
  if (!geometry_ok(tile_rows, tile_cols, lmax) || keep < 1 || keep > 256) return ORC_E_ARG;
  const int64_t tiles_r = (rows + tile_rows - 1) / tile_rows;
  const int64_t tiles_c = (cols + tile_cols - 1) / tile_cols;
  const int64_t tiles = tiles_r * tiles_c;
  const int groups = tile_cols / 64;
  const int lane_syms = 2 * tile_rows * groups;
  const int raw_bytes = tile_rows * tile_cols;

  /* Step 2: histogram with the fillers, filler, kept symbols. */
  uint64_t cnt[256];
  orc_histogram(w, rows, cols, cnt);
  const int filler = filler_symbol(cnt);
  cnt[filler] += (uint64_t)(tiles_r * tile_rows) * (uint64_t)(tiles_c * tile_cols) -
                 (uint64_t)rows * (uint64_t)cols;
  bool kept[256];
  const int K = kept_symbols(cnt, keep, kept);

  /* Step 3: which runs are escaped; step 4: counts over the other runs. */
  std::vector<uint8_t> escaped((size_t)(tiles * tile_rows * groups), 0);
  uint64_t ccnt[256] = {};
  uint64_t n_escaped = 0;
  for (int64_t u = 0; u < tiles; ++u) {
    const int64_t i = u % tiles_r, j = u / tiles_r;
    for (int g = 0; g < tile_rows; ++g) {
      for (int m = 0; m < groups; ++m) {
        bool rare = false;
        for (int c = 64 * m; c < 64 * m + 64; ++c) {
          uint8_t s, rb;
          tile_element(w, rows, cols, i, j, tile_rows, tile_cols, filler, g, c, &s, &rb);
          if (!kept[s]) rare = true;
        }
        escaped[(size_t)((u * tile_rows + g) * groups + m)] = rare ? 1 : 0;
        if (rare) {
          ++n_escaped;
          continue;
        }
        for (int c = 64 * m; c < 64 * m + 64; ++c) {
          uint8_t s, rb;
          tile_element(w, rows, cols, i, j, tile_rows, tile_cols, filler, g, c, &s, &rb);
          ccnt[s] += 1;
        }
      }
    }
  }
  uint8_t len[256] = {};
  uint64_t any = 0;
  for (int s = 0; s < 256; ++s) any += ccnt[s];
  if (any) {
    const int rc = orc_code_lengths(ccnt, lmax, len);
    if (rc != ORC_OK) return rc;
  }
  uint32_t code[256];
  orc_canonical_codes(len, code);
  uint64_t coded_bits = 0;
  for (int s = 0; s < 256; ++s) coded_bits += ccnt[s] * (uint64_t)len[s];

  /* Step 5: the chunks. */
  const uint64_t lens_off = kHeaderBytes;
  const uint64_t index_off = lens_off + 256;
  const uint64_t tiles_off = round_up(index_off + 4 * (uint64_t)(tiles + 1), 256);
  std::vector<uint32_t> index((size_t)tiles + 1);
  uint64_t area = 0;
  for (int64_t u = 0; u < tiles; ++u) {
    const int64_t i = u % tiles_r, j = u / tiles_r;
    auto is_escaped = [&](int g, int m) {
      return escaped[(size_t)((u * tile_rows + g) * groups + m)] != 0;
    };
    std::vector<uint8_t> raw((size_t)raw_bytes, 0);
    std::vector<uint8_t> flags(16, 0);
    std::vector<uint8_t> runs;
    for (int g = 0; g < tile_rows; ++g) {
      for (int m = 0; m < groups; ++m) {
        if (!is_escaped(g, m)) continue;
        flags[(size_t)g] |= (uint8_t)(1u << m);
        for (int c = 64 * m; c < 64 * m + 64; ++c) {
          uint8_t s, rb;
          tile_element(w, rows, cols, i, j, tile_rows, tile_cols, filler, g, c, &s, &rb);
          runs.push_back(s);
        }
      }
    }
    std::vector<uint8_t> seq; /* one entry per bit */
    uint8_t lane_bytes[kLanes];
    for (int t = 0; t < kLanes; ++t) {
      std::vector<uint8_t> lb;
      for (int k = 0; k < lane_syms; ++k) {
        int r, c;
        lane_symbol_position(t, k, &r, &c);
        uint8_t s, rb;
        tile_element(w, rows, cols, i, j, tile_rows, tile_cols, filler, r, c, &s, &rb);
        raw[(size_t)raw_position(t, k)] = rb;
        if (is_escaped(r, k / 16)) continue;
        for (int b = len[s] - 1; b >= 0; --b) lb.push_back((uint8_t)((code[s] >> b) & 1u));
      }
      while (lb.size() % 8 != 0) lb.push_back(0);
      lane_bytes[t] = (uint8_t)(lb.size() / 8);
      seq.insert(seq.end(), lb.begin(), lb.end());
    }
    while (seq.size() % 128 != 0) seq.push_back(0);
    std::vector<uint8_t> bits(seq.size() / 8, 0);
    for (size_t b = 0; b < seq.size(); ++b) {
      if (!seq[b]) continue;
      const int bit = 31 - (int)(b % 32);
      bits[(b / 32) * 4 + (size_t)(bit / 8)] |= (uint8_t)(1u << (bit % 8));
    }
    std::vector<uint8_t> chunk;
    chunk.insert(chunk.end(), raw.begin(), raw.end());
    chunk.insert(chunk.end(), flags.begin(), flags.end());
    chunk.insert(chunk.end(), runs.begin(), runs.end());
    chunk.insert(chunk.end(), lane_bytes, lane_bytes + kLanes);
    chunk.insert(chunk.end(), bits.begin(), bits.end());
    index[(size_t)u] = (uint32_t)(area / 16);
    if (blob) {
      if ((int64_t)(tiles_off + area + chunk.size()) > cap) return ORC_E_SPACE;
      std::memcpy(blob + tiles_off + area, chunk.data(), chunk.size());
    }
    area += chunk.size();
    if (area / 16 > 0xFFFFFFFFull) return ORC_E_ARG;
  }
  index[(size_t)tiles] = (uint32_t)(area / 16);
  const uint64_t total = tiles_off + area;
  *size = (int64_t)total;
  if (!blob) return ORC_OK;
  if ((int64_t)total > cap) return ORC_E_SPACE;
  std::memset(blob, 0, (size_t)tiles_off);
  put_u32(blob + 0, kEscMagic);
  put_u32(blob + 4, kVersion);
  put_u32(blob + 8, kHeaderBytes);
  put_u32(blob + 12, (uint32_t)lmax);
  put_u64(blob + 16, (uint64_t)rows);
  put_u64(blob + 24, (uint64_t)cols);
  put_u32(blob + 32, (uint32_t)tile_rows);
  put_u32(blob + 36, (uint32_t)tile_cols);
  put_u64(blob + 40, (uint64_t)tiles_r);
  put_u64(blob + 48, (uint64_t)tiles_c);
  put_u32(blob + 56, (uint32_t)filler);
  put_u32(blob + 60, (uint32_t)K);
  put_u64(blob + 64, lens_off);
  put_u64(blob + 72, index_off);
  put_u64(blob + 80, tiles_off);
  put_u64(blob + 88, total);
  put_u64(blob + 96, coded_bits);
  put_u64(blob + 104, n_escaped);
  std::memcpy(blob + lens_off, len, 256);
  for (int64_t u = 0; u <= tiles; ++u) put_u32(blob + index_off + 4 * u, index[(size_t)u]);
  return ORC_OK;
}

int decode_escape_impl(const uint8_t* blob, int64_t size, uint16_t* out, int64_t cap_elems) {
  if (!blob || size < kHeaderBytes + 256) return ORC_E_CORRUPT;
  if (get_u32(blob) != kEscMagic || get_u32(blob + 4) != kVersion ||
      get_u32(blob + 8) != (uint32_t)kHeaderBytes)
    return ORC_E_CORRUPT;
  const int lmax = (int)get_u32(blob + 12);
  const int64_t rows = (int64_t)get_u64(blob + 16), cols = (int64_t)get_u64(blob + 24);
  const int tile_rows = (int)get_u32(blob + 32), tile_cols = (int)get_u32(blob + 36);
  const int64_t tiles_r = (int64_t)get_u64(blob + 40), tiles_c = (int64_t)get_u64(blob + 48);
  const int filler = (int)get_u32(blob + 56);
  const int K = (int)get_u32(blob + 60);
  const uint64_t lens_off = get_u64(blob + 64), index_off = get_u64(blob + 72);
  const uint64_t tiles_off = get_u64(blob + 80), total = get_u64(blob + 88);
  const uint64_t n_escaped = get_u64(blob + 104);
  if (rows < 1 || cols < 1 || !geometry_ok(tile_rows, tile_cols, lmax)) return ORC_E_CORRUPT;
  if (K < 1 || K > 256 || filler < 0 || filler > 255) return ORC_E_CORRUPT;
  if (tiles_r != (rows + tile_rows - 1) / tile_rows ||
      tiles_c != (cols + tile_cols - 1) / tile_cols)
    return ORC_E_CORRUPT;
  const int64_t tiles = tiles_r * tiles_c;
  if (lens_off != (uint64_t)kHeaderBytes || index_off != lens_off + 256 ||
      tiles_off != round_up(index_off + 4 * (uint64_t)(tiles + 1), 256) ||
      total != (uint64_t)size)
    return ORC_E_CORRUPT;
  for (int q = 112; q < kHeaderBytes; ++q)
    if (blob[q]) return ORC_E_CORRUPT;
  /* The code: Kraft sum at most one, no more coded symbols than kept ones. */
  uint8_t len[256];
  std::memcpy(len, blob + lens_off, 256);
  double kraft = 0.0;
  int coded = 0;
  for (int s = 0; s < 256; ++s) {
    if (len[s] > lmax) return ORC_E_CORRUPT;
    if (len[s]) {
      kraft += 1.0 / (double)(1u << len[s]);
      ++coded;
    }
  }
  if (kraft > 1.0 || coded > K) return ORC_E_CORRUPT;
  uint32_t code[256];
  orc_canonical_codes(len, code);
  std::vector<std::vector<int> > sym_of(13);
  for (int l = 1; l <= 12; ++l) sym_of[(size_t)l].assign((size_t)1 << l, -1);
  for (int s = 0; s < 256; ++s)
    if (len[s]) sym_of[len[s]][code[s]] = s;
  if (!out || cap_elems < rows * cols) return ORC_E_SPACE;

  const int groups = tile_cols / 64;
  const int lane_syms = 2 * tile_rows * groups;
  const int raw_bytes = tile_rows * tile_cols;
  const uint64_t area = (uint64_t)size - tiles_off;
  uint64_t escaped_total = 0;
  for (int64_t u = 0; u < tiles; ++u) {
    const uint64_t c0 = 16ull * get_u32(blob + index_off + 4 * u);
    const uint64_t c1 = 16ull * get_u32(blob + index_off + 4 * (u + 1));
    if (c1 < c0 || c1 > area || c1 - c0 < (uint64_t)raw_bytes + 16 + kLanes)
      return ORC_E_CORRUPT;
    const uint8_t* chunk = blob + tiles_off + c0;
    const uint8_t* raw = chunk;
    const uint8_t* flags = chunk + raw_bytes;
    /* Flags: only bits of real groups, bytes 8 .. 15 zero. */
    for (int q = 0; q < 16; ++q) {
      const unsigned allowed = q < tile_rows ? (1u << groups) - 1u : 0u;
      if (flags[q] & ~allowed) return ORC_E_CORRUPT;
    }
    /* Place of every escaped run among the tile's runs, in (g, m) order. */
    std::vector<int> run_at((size_t)(tile_rows * groups), -1);
    int n = 0;
    for (int g = 0; g < tile_rows; ++g)
      for (int m = 0; m < groups; ++m)
        if ((flags[g] >> m) & 1u) run_at[(size_t)(g * groups + m)] = n++;
    escaped_total += (uint64_t)n;
    const uint64_t head = (uint64_t)raw_bytes + 16 + 64ull * (uint64_t)n;
    if (c1 - c0 < head + kLanes) return ORC_E_CORRUPT;
    const uint8_t* runs = chunk + raw_bytes + 16;
    const uint8_t* lane_bytes = chunk + head;
    const uint8_t* bits = chunk + head + kLanes;
    uint64_t stream_bytes = 0;
    for (int t = 0; t < kLanes; ++t) stream_bytes += lane_bytes[t];
    if (c1 - c0 != head + kLanes + round_up(stream_bytes, 16)) return ORC_E_CORRUPT;
    /* An escaped run holds a symbol without a code (otherwise it would have
     * been coded). */
    for (int q = 0; q < n; ++q) {
      bool rare = false;
      for (int b = 0; b < 64; ++b) rare = rare || len[runs[64 * q + b]] == 0;
      if (!rare) return ORC_E_CORRUPT;
    }
    auto bit_at = [&](uint64_t q) -> int {
      const int b = 31 - (int)(q % 32);
      return (bits[(q / 32) * 4 + (uint64_t)(b / 8)] >> (b % 8)) & 1;
    };
    const int64_t i = u % tiles_r, j = u / tiles_r;
    uint64_t lane_start = 0;
    for (int t = 0; t < kLanes; ++t) {
      uint64_t pos = lane_start;
      const uint64_t end = lane_start + 8ull * lane_bytes[t];
      for (int k = 0; k < lane_syms; ++k) {
        int r, c;
        lane_symbol_position(t, k, &r, &c);
        const int at = run_at[(size_t)(r * groups + k / 16)];
        int s = -1;
        if (at >= 0) {
          /* Column c of the tile is byte c - 64 m of its run. */
          s = runs[64 * at + (c - 64 * (k / 16))];
        } else {
          uint32_t v = 0;
          int l = 0;
          while (s < 0) {
            if (pos >= end || l >= lmax) return ORC_E_CORRUPT;
            v = (v << 1) | (uint32_t)bit_at(pos++);
            ++l;
            s = sym_of[(size_t)l][v];
          }
        }
        const uint8_t rb = raw[raw_position(t, k)];
        const int64_t row = i * tile_rows + r, col = j * tile_cols + c;
        if (row < rows && col < cols) {
          out[row * cols + col] = orc_plane_join((uint8_t)s, rb);
        } else if (s != filler || rb != 0) {
          return ORC_E_CORRUPT;
        }
      }
      if (end - pos >= 8) return ORC_E_CORRUPT;
      while (pos < end)
        if (bit_at(pos++)) return ORC_E_CORRUPT;
      lane_start = end;
    }
    for (uint64_t q = lane_start; q < 8 * round_up(stream_bytes, 16); ++q)
      if (bit_at(q)) return ORC_E_CORRUPT;
  }
  if (escaped_total != n_escaped) return ORC_E_CORRUPT;
  return ORC_OK;
}


}  // namespace

extern "C" {

void orc_plane_split(uint16_t w, uint8_t* s, uint8_t* r) {
  /* "Efficient ML #1 — Deep Learning Data Types" §4: bit 15 sign, bits 14..7
   * exponent (bias 127), bits 6..0 fraction. */
  *s = (uint8_t)((w >> 7) & 0xFF);
  *r = (uint8_t)(((w >> 15) & 1) << 7 | (w & 0x7F));
}

uint16_t orc_plane_join(uint8_t s, uint8_t r) {
  return (uint16_t)(((uint16_t)(r >> 7) << 15) | ((uint16_t)s << 7) | (r & 0x7F));
}

int orc_histogram(const uint16_t* w, int64_t rows, int64_t cols, uint64_t cnt[256]) {
  if (!w || !cnt || rows < 0 || cols < 0) return ORC_E_ARG;
  for (int s = 0; s < 256; ++s) cnt[s] = 0;
  for (int64_t n = 0; n < rows * cols; ++n) {
    uint8_t s, r;
    orc_plane_split(w[n], &s, &r);
    cnt[s] += 1;
  }
  return ORC_OK;
}

int orc_code_lengths(const uint64_t cnt[256], int lmax, uint8_t len[256]) {
  if (!cnt || !len || lmax < 1 || lmax > 32) return ORC_E_ARG;
  for (int s = 0; s < 256; ++s) len[s] = 0;
  /* Leaves sorted by (count ascending, symbol ascending). */
  std::vector<Item> leaves;
  for (int s = 0; s < 256; ++s) {
    if (cnt[s] == 0) continue;
    Item it;
    it.weight = cnt[s];
    it.leaf = true;
    it.symbol = s;
    it.uses.assign(256, 0);
    it.uses[(size_t)s] = 1;
    leaves.push_back(it);
  }
  const size_t n = leaves.size();
  if (n == 0) return ORC_E_ARG;
  if (n == 1) {
    len[leaves[0].symbol] = 1;
    return ORC_OK;
  }
  if (lmax < 31 && n > ((size_t)1 << lmax)) return ORC_E_LMAX;
  std::stable_sort(leaves.begin(), leaves.end(), [](const Item& a, const Item& b) {
    if (a.weight != b.weight) return a.weight < b.weight;
    return a.symbol < b.symbol;
  });

  /* Package-merge: start with the coins of the smallest denomination 2^-lmax;
   * at each level pair consecutive items into packages and merge them with a
   * fresh copy of the leaves (leaf first when weights are equal).  At the
   * level of denomination 1/2, keep the 2n - 2 cheapest items; a symbol's code
   * length is the number of its coins among them. */
  std::vector<Item> list = leaves;
  for (int level = lmax; level > 1; --level) {
    std::vector<Item> packages;
    for (size_t p = 0; p + 1 < list.size(); p += 2) {
      Item pk;
      pk.weight = list[p].weight + list[p + 1].weight;
      pk.leaf = false;
      pk.symbol = -1;
      pk.uses.assign(256, 0);
      for (int s = 0; s < 256; ++s)
        pk.uses[(size_t)s] = (uint16_t)(list[p].uses[(size_t)s] + list[p + 1].uses[(size_t)s]);
      packages.push_back(pk);
    }
    std::vector<Item> merged;
    size_t a = 0, b = 0;
    while (a < leaves.size() || b < packages.size()) {
      const bool take_leaf =
          b >= packages.size() ||
          (a < leaves.size() && leaves[a].weight <= packages[b].weight);
      merged.push_back(take_leaf ? leaves[a++] : packages[b++]);
    }
    list.swap(merged);
  }
  if (list.size() < 2 * n - 2) return ORC_E_LMAX;
  for (size_t q = 0; q < 2 * n - 2; ++q)
    for (int s = 0; s < 256; ++s) len[s] = (uint8_t)(len[s] + list[q].uses[(size_t)s]);
  return ORC_OK;
}

int orc_canonical_codes(const uint8_t len[256], uint32_t code[256]) {
  if (!len || !code) return ORC_E_ARG;
  /* Symbols in (length, symbol) order receive consecutive values; moving to a
   * longer length appends zero bits to the running value. */
  uint32_t next = 0;
  int prev_len = 0;
  bool first = true;
  for (int s = 0; s < 256; ++s) code[s] = 0;
  for (int l = 1; l <= 32; ++l) {
    for (int s = 0; s < 256; ++s) {
      if (len[s] != l) continue;
      if (first) {
        next = 0;
        first = false;
      } else {
        next = (next + 1) << (l - prev_len);
      }
      prev_len = l;
      code[s] = next;
    }
  }
  return ORC_OK;
}

int orc_blob_size(const uint16_t* w, int64_t rows, int64_t cols, int tile_rows,
                  int tile_cols, int lmax, int64_t* size) {
  return encode_impl(w, rows, cols, tile_rows, tile_cols, lmax, 1, nullptr, 0, size);
}

int orc_blob_size_streams(const uint16_t* w, int64_t rows, int64_t cols, int tile_rows,
                          int tile_cols, int lmax, int streams, int64_t* size) {
  return encode_impl(w, rows, cols, tile_rows, tile_cols, lmax, streams, nullptr, 0, size);
}

int orc_encode_streams(const uint16_t* w, int64_t rows, int64_t cols, int tile_rows,
                       int tile_cols, int lmax, int streams, uint8_t* blob, int64_t cap,
                       int64_t* size) {
  if (!blob) return ORC_E_ARG;
  return encode_impl(w, rows, cols, tile_rows, tile_cols, lmax, streams, blob, cap, size);
}

int orc_encode(const uint16_t* w, int64_t rows, int64_t cols, int tile_rows,
               int tile_cols, int lmax, uint8_t* blob, int64_t cap, int64_t* size) {
  if (!blob) return ORC_E_ARG;
  return encode_impl(w, rows, cols, tile_rows, tile_cols, lmax, 1, blob, cap, size);
}

int orc_blob_info(const uint8_t* blob, int64_t size, int64_t* rows, int64_t* cols) {
  Header h;
  int rc = read_header(blob, size, &h);
  if (rc != ORC_OK) return rc;
  if (rows) *rows = h.rows;
  if (cols) *cols = h.cols;
  return ORC_OK;
}

int orc_decode(const uint8_t* blob, int64_t size, uint16_t* w_out, int64_t cap_elems) {
  Header h;
  int rc = read_header(blob, size, &h);
  if (rc != ORC_OK) return rc;
  return decode_impl(blob, size, 0, h.tiles_r * h.tiles_c, w_out, cap_elems);
}

int orc_decode_tiles(const uint8_t* blob, int64_t size, int64_t tile_begin,
                     int64_t tile_end, uint16_t* w_out, int64_t cap_elems) {
  return decode_impl(blob, size, tile_begin, tile_end, w_out, cap_elems);
}

static double bf16_to_double(uint16_t v) {
  /* A BF16 value is the upper half of the FP32 with the same bits. */
  uint32_t u = (uint32_t)v << 16;
  float f;
  std::memcpy(&f, &u, 4);
  return (double)f;
}

int orc_gemv(const uint16_t* w, int64_t rows, int64_t cols, const uint16_t* x,
             int batch, int64_t row_begin, int64_t row_end, double* y) {
  if (!w || !x || !y || rows < 1 || cols < 1 || batch < 1) return ORC_E_ARG;
  if (row_begin < 0 || row_end > rows || row_begin > row_end) return ORC_E_ARG;
  for (int b = 0; b < batch; ++b) {
    for (int64_t n = row_begin; n < row_end; ++n) {
      double acc = 0.0;
      for (int64_t k = 0; k < cols; ++k)
        acc += bf16_to_double(w[n * cols + k]) * bf16_to_double(x[(int64_t)b * cols + k]);
      y[(int64_t)b * rows + n] = acc;
    }
  }
  return ORC_OK;
}

int orc_rank_table(const uint16_t* w, int64_t rows, int64_t cols, int tile_rows,
                   int tile_cols, int ranks, uint8_t table[7], int* n) {
  /* The ranked values and their number, read back from an encoded header. */
  int64_t size = 0;
  int rc = encode_rank_impl(w, rows, cols, tile_rows, tile_cols, ranks, nullptr, 0, &size);
  if (rc != ORC_OK) return rc;
  std::vector<uint8_t> blob((size_t)size);
  rc = encode_rank_impl(w, rows, cols, tile_rows, tile_cols, ranks, blob.data(), size, &size);
  if (rc != ORC_OK) return rc;
  *n = (int)get_u32(blob.data() + 12);
  std::memcpy(table, blob.data() + kHeaderBytes, 7);
  return ORC_OK;
}

int orc_rank_blob_size(const uint16_t* w, int64_t rows, int64_t cols, int tile_rows,
                       int tile_cols, int ranks, int64_t* size) {
  return encode_rank_impl(w, rows, cols, tile_rows, tile_cols, ranks, nullptr, 0, size);
}

int orc_rank_encode(const uint16_t* w, int64_t rows, int64_t cols, int tile_rows,
                    int tile_cols, int ranks, uint8_t* blob, int64_t cap, int64_t* size) {
  if (!blob) return ORC_E_ARG;
  return encode_rank_impl(w, rows, cols, tile_rows, tile_cols, ranks, blob, cap, size);
}

int orc_rank_decode(const uint8_t* blob, int64_t size, uint16_t* w_out, int64_t cap_elems) {
  return decode_rank_impl(blob, size, w_out, cap_elems);
}

int orc_escape_blob_size(const uint16_t* w, int64_t rows, int64_t cols, int tile_rows,
                         int tile_cols, int lmax, int keep, int64_t* size) {
  return encode_escape_impl(w, rows, cols, tile_rows, tile_cols, lmax, keep, nullptr, 0, size);
}

int orc_escape_encode(const uint16_t* w, int64_t rows, int64_t cols, int tile_rows,
                      int tile_cols, int lmax, int keep, uint8_t* blob, int64_t cap,
                      int64_t* size) {
  if (!blob) return ORC_E_ARG;
  return encode_escape_impl(w, rows, cols, tile_rows, tile_cols, lmax, keep, blob, cap, size);
}

int orc_escape_decode(const uint8_t* blob, int64_t size, uint16_t* w_out, int64_t cap_elems) {
  return decode_escape_impl(blob, size, w_out, cap_elems);
}

}  // extern "C"
