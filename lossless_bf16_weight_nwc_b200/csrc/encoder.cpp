// encoder.cpp — host encoder of libnwc (multi-threaded C++).
//
// Steps, in the pages' order:
//  1. Byte planes: exponent byte s = bits 14..7 is coded, raw byte r = sign << 7
//     | fraction is stored ("Unweight", "Compressing BF16 Weights"; "NWC", "How
//     it works > Byte planes").
//  2. Histogram of s over the matrix plus the filler positions of ragged tiles.
//  3. Optimal code lengths limited to lmax (package-merge, Larmore & Hirschberg
//     1990), assigned canonically.  Ties: leaves by (count, symbol); a leaf
//     precedes a package of equal weight; codes in (length, symbol) order.  The
//     filler is the most frequent exponent (smallest symbol on a tie).
//  4. Tiles of 8 rows x tile_cols with one MSB-first bit stream per lane ("NWC",
//     "How it works > Fused kernel"), an offset index, and the raw plane laid
//     out so that one 128-bit load gives a lane 16 of its raw bytes.
//  5. A 4096-entry decode table for the GPU ("NWC", "Prefix code instead of
//     rANS": a 12-bit peek yields up to two complete codes).
// The variant NWR1 (plan_build_rank) replaces steps 1-3 with the ranked unary
// code of "NWC", "Prefix code instead of rANS" (format v9): exponent bits
// 14..8 ranked by count, the sign bit raw in the stream, bits 7..0 raw; step 4
// is shared.
// The variant NWE1 (plan_build_escape) follows "Unweight", "Compressing BF16
// Weights": only the K most frequent exponents are coded (step 3 over the runs
// that hold no other exponent); a run of 64 weights of a tile row that holds
// another one keeps its exponent bytes verbatim in the chunk, and its symbols
// leave the lane streams.
#include <algorithm>
#include <cstring>
#include <functional>
#include <thread>
#include <vector>

#include "nwc_internal.h"

namespace nwc {

unsigned hardware_threads(uint32_t requested) {
  if (requested) return requested;
  unsigned n = std::thread::hardware_concurrency();
  return n ? n : 1;
}

namespace {

// Runs f(begin, end) over [0, n) split into `threads` contiguous parts.
void parallel_for(int64_t n, unsigned threads, const std::function<void(int64_t, int64_t)>& f) {
  if (n <= 0) return;
  unsigned parts = (unsigned)std::min<int64_t>(threads, n);
  if (parts <= 1) {
    f(0, n);
    return;
  }
  std::vector<std::thread> pool;
  for (unsigned p = 0; p < parts; ++p) {
    int64_t b = n * p / parts, e = n * (p + 1) / parts;
    pool.emplace_back([&f, b, e] { f(b, e); });
  }
  for (auto& t : pool) t.join();
}

inline uint8_t exponent_byte(uint16_t w) { return (uint8_t)(w >> 7); }
inline uint8_t raw_byte(uint16_t w) { return (uint8_t)(((w >> 8) & 0x80) | (w & 0x7F)); }

// Symbol (exponent byte) of tile element (r, c); the filler outside the matrix.
struct TileView {
  const uint16_t* w;
  int64_t rows, cols, row0, col0;
  uint8_t filler;
  inline bool inside(int r, int c) const { return row0 + r < rows && col0 + c < cols; }
  inline uint16_t at(int r, int c) const { return w[(row0 + r) * cols + col0 + c]; }
};

// NWR1's coded field: exponent bits 14..8.
inline uint32_t rank_field(uint16_t w) { return (w >> 8) & 0x7Fu; }

// Code bits (right-aligned), their number and the raw byte of tile element
// (r, c) under the plan's code; positions outside the matrix hold the filler
// with a zero raw byte (and, for NWR1, sign 0).
inline void symbol_of(const nwc_plan_s& p, const TileView& v, int r, int c, uint32_t* code,
                      int* len, uint8_t* raw) {
  const bool in = v.inside(r, c);
  const uint16_t x = in ? v.at(r, c) : 0;
  *raw = 0;
  if (p.code_kind != 1) {
    uint8_t s = v.filler;
    if (in) {
      s = exponent_byte(x);
      *raw = raw_byte(x);
    }
    *code = p.code[s];
    *len = p.len[s];
    return;
  }
  uint32_t e = p.filler, sign = 0;
  if (in) {
    e = rank_field(x);
    sign = x >> 15;
    *raw = (uint8_t)(x & 0xFF);
  }
  *code = (sign << p.rank_len[e]) | p.rank_code[e];
  *len = p.rank_len[e] + 1;
}

// Stream of lane t that carries the lane's k-th symbol when each lane has S
// streams: consecutive symbol pairs go to the lane's streams in turn.
inline int stream_of(int t, int k, int S) { return t * S + (k / 2) % S; }

// NWE1: whether run (row r, group m) of tile u is verbatim, and how many of
// the tile's runs are.
inline bool escaped(const nwc_plan_s& p, int64_t u, int r, int m) {
  return (p.esc_flags[(size_t)(8 * u + r)] >> m) & 1u;
}
inline uint32_t escaped_runs(const nwc_plan_s& p, int64_t u) {
  uint32_t n = 0;
  for (int r = 0; r < kTileRows; ++r) n += (uint32_t)__builtin_popcount(p.esc_flags[(size_t)(8 * u + r)]);
  return n;
}

// Exponent-byte histogram of the rows x cols weights, one partial per thread.
void exponent_histogram(const uint16_t* w, int64_t rows, int64_t cols, unsigned nt,
                        uint64_t cnt[256]) {
  std::vector<std::vector<uint64_t>> part(nt, std::vector<uint64_t>(256, 0));
  {
    std::vector<std::thread> pool;
    for (unsigned q = 0; q < nt; ++q) {
      pool.emplace_back([&, q] {
        const int64_t b = rows * q / nt, e = rows * (q + 1) / nt;
        uint64_t* h = part[q].data();
        for (int64_t r = b; r < e; ++r) {
          const uint16_t* row = w + r * cols;
          for (int64_t c = 0; c < cols; ++c) h[exponent_byte(row[c])] += 1;
        }
      });
    }
    for (auto& t : pool) t.join();
  }
  for (int s = 0; s < 256; ++s) cnt[s] = 0;
  for (unsigned q = 0; q < nt; ++q)
    for (int s = 0; s < 256; ++s) cnt[s] += part[q][s];
}

// Bits of each stream in tile u (kLanes * p.streams entries).
void lane_bits(const nwc_plan_s& p, const uint16_t* w, int64_t u, uint32_t* bits) {
  const int64_t i = u % p.tiles_r, j = u / p.tiles_r;
  TileView v{w, p.rows, p.cols, i * kTileRows, j * (int64_t)p.tile_cols, (uint8_t)p.filler};
  const int S = (int)p.streams;
  for (int t = 0; t < kLanes * S; ++t) bits[t] = 0;
  for (int r = 0; r < kTileRows; ++r) {
    for (int c = 0; c < (int)p.tile_cols; ++c) {
      const int t = 4 * r + (c % 64) / 16;  // lane t = 4 r + q owns row r, columns 16 q .. of a group
      const int k = 16 * (c / 64) + c % 16;  // the lane's symbol index
      const int sigma = stream_of(t, k, S);
      if (p.code_kind == 2 && escaped(p, u, r, c / 64)) continue;
      if (p.code_kind != 1) {
        const uint8_t s = v.inside(r, c) ? exponent_byte(v.at(r, c)) : v.filler;
        bits[sigma] += p.len[s];
      } else {
        const uint32_t e = v.inside(r, c) ? rank_field(v.at(r, c)) : p.filler;
        bits[sigma] += p.rank_len[e] + 1u;
      }
    }
  }
}

uint32_t stream_bytes_of(const uint32_t* bits, int n) {
  uint32_t total = 0;
  for (int t = 0; t < n; ++t) total += (bits[t] + 7) / 8;
  return total;
}

}  // namespace

bool code_lengths(const uint64_t cnt[256], uint32_t lmax, uint8_t len[256]) {
  // Package-merge over an arena of nodes: a node is a leaf (symbol) or a
  // package of two earlier nodes.  The code length of a symbol is the number of
  // times its leaf occurs below the 2n - 2 cheapest items of the last list.
  struct Node {
    uint64_t weight;
    int32_t a, b;  // children; a < 0 encodes leaf symbol -a - 1
  };
  std::memset(len, 0, 256);
  std::vector<int> syms;
  for (int s = 0; s < 256; ++s)
    if (cnt[s]) syms.push_back(s);
  const size_t n = syms.size();
  if (n == 0) return false;
  if (n == 1) {
    len[syms[0]] = 1;
    return true;
  }
  if (lmax > 30 || n > (size_t(1) << lmax)) return false;
  std::stable_sort(syms.begin(), syms.end(), [&](int x, int y) {
    return cnt[x] != cnt[y] ? cnt[x] < cnt[y] : x < y;
  });
  std::vector<Node> arena;
  std::vector<int32_t> leaves;
  for (int s : syms) {
    leaves.push_back((int32_t)arena.size());
    arena.push_back({cnt[s], -s - 1, -1});
  }
  std::vector<int32_t> cur = leaves, next;
  for (uint32_t level = lmax; level > 1; --level) {
    next.clear();
    size_t li = 0, pi = 0;
    const size_t packages = cur.size() / 2;
    // Merge leaves with packages of consecutive pairs of `cur`, creating each
    // package node when it is taken.
    std::vector<int32_t> pk(packages);
    for (size_t q = 0; q < packages; ++q) {
      pk[q] = (int32_t)arena.size();
      arena.push_back({arena[cur[2 * q]].weight + arena[cur[2 * q + 1]].weight,
                       cur[2 * q], cur[2 * q + 1]});
    }
    while (li < leaves.size() || pi < packages) {
      if (pi >= packages ||
          (li < leaves.size() && arena[leaves[li]].weight <= arena[pk[pi]].weight))
        next.push_back(leaves[li++]);
      else
        next.push_back(pk[pi++]);
    }
    cur.swap(next);
  }
  if (cur.size() < 2 * n - 2) return false;
  std::vector<int32_t> stack;
  std::vector<uint32_t> uses(256, 0);
  for (size_t q = 0; q < 2 * n - 2; ++q) {
    stack.push_back(cur[q]);
    while (!stack.empty()) {
      const Node& nd = arena[stack.back()];
      stack.pop_back();
      if (nd.a < 0) {
        uses[-nd.a - 1] += 1;
      } else {
        stack.push_back(nd.a);
        stack.push_back(nd.b);
      }
    }
  }
  for (int s = 0; s < 256; ++s) len[s] = (uint8_t)uses[s];
  return true;
}

void canonical_codes(const uint8_t len[256], uint32_t code[256]) {
  // Count codes per length, then the first code of each length (shorter codes
  // are prefixes of nothing longer), then hand out codes in symbol order.
  uint32_t per_len[33] = {}, first[33] = {};
  for (int s = 0; s < 256; ++s)
    if (len[s]) per_len[len[s]] += 1;
  uint32_t c = 0;
  for (int l = 1; l <= 32; ++l) {
    c = (c + per_len[l - 1]) << 1;
    first[l] = c;
  }
  for (int s = 0; s < 256; ++s) code[s] = len[s] ? first[len[s]]++ : 0;
}

void build_decode_table(const uint8_t len[256], uint32_t lmax, uint32_t* table) {
  const int peek = peek_bits(lmax);
  const uint32_t entries = table_entries(lmax);
  uint32_t code[256];
  canonical_codes(len, code);
  // sym[l][v]: symbol with code v of length l, or -1.
  std::vector<std::vector<int16_t>> sym(peek + 1);
  for (int l = 1; l <= peek; ++l) sym[l].assign(size_t(1) << l, -1);
  for (int s = 0; s < 256; ++s)
    if (len[s] >= 1 && len[s] <= peek) sym[len[s]][code[s]] = (int16_t)s;
  auto first_code = [&](uint32_t bits, int avail, int* s_out, int* l_out) {
    for (int l = 1; l <= avail; ++l) {
      const int s = sym[l][bits >> (peek - l)];
      if (s >= 0) {
        *s_out = s;
        *l_out = l;
        return true;
      }
    }
    return false;
  };
  for (uint32_t v = 0; v < entries; ++v) {
    int s0, l0, s1, l1;
    if (!first_code(v, peek, &s0, &l0)) {
      table[v] = 2u | kEntryInvalid;  // consume two bits, emit exponent 0
      continue;
    }
    const uint32_t rest = (v << l0) & (entries - 1);
    uint32_t e = ((uint32_t)s0 << 7) | ((uint32_t)l0 << kEntryLen0Shift);
    if (first_code(rest, peek - l0, &s1, &l1))
      e |= (uint32_t)(l0 + l1) | ((uint32_t)s1 << 23);
    else
      e |= (uint32_t)l0 | kEntrySingle;
    table[v] = e;
  }
}

int plan_tiles(const uint16_t* w, nwc_plan_s* p);

int plan_build(const uint16_t* w, int64_t rows, int64_t cols, uint32_t tile_rows,
               uint32_t tile_cols, uint32_t lmax, uint32_t threads, nwc_plan_s* p,
               uint32_t streams) {
  if (streams != 1 && streams != 2 && streams != 4) return -1;
  p->streams = streams;
  p->rows = rows;
  p->cols = cols;
  p->tile_rows = tile_rows;
  p->tile_cols = tile_cols;
  p->lmax = lmax;
  p->threads = hardware_threads(threads);
  p->tiles_r = (rows + kTileRows - 1) / kTileRows;
  p->tiles_c = (cols + tile_cols - 1) / tile_cols;
  p->tiles = p->tiles_r * p->tiles_c;

  uint64_t cnt[256];
  exponent_histogram(w, rows, cols, p->threads, cnt);
  uint32_t filler = 0;
  for (uint32_t s = 1; s < 256; ++s)
    if (cnt[s] > cnt[filler]) filler = s;
  p->filler = filler;
  cnt[filler] += (uint64_t)(p->tiles_r * kTileRows) * (uint64_t)(p->tiles_c * tile_cols) -
                 (uint64_t)rows * (uint64_t)cols;
  if (lmax == 0) {
    // Automatic: 7 (two codes always fit the decoder's 14-bit peek) unless the
    // matrix holds more than 128 distinct exponents; then the smallest limit
    // that admits them all.
    int distinct = 0;
    for (int s = 0; s < 256; ++s) distinct += cnt[s] != 0;
    lmax = 7;
    while ((1 << lmax) < distinct) ++lmax;
    p->lmax = lmax;
  }
  if (!code_lengths(cnt, lmax, p->len)) return -1;
  canonical_codes(p->len, p->code);
  p->coded_bits = 0;
  for (int s = 0; s < 256; ++s) p->coded_bits += cnt[s] * p->len[s];
  const int rc = plan_tiles(w, p);
  if (rc != 0) return rc;
  if (p->streams > kMaxDeviceStreams) {  // no kernel reads four streams per lane
    p->table_off = p->sched_off = p->scratch_off = p->device_bytes = 0;
    return 0;
  }
  const ImageLayout L =
      image_layout(p->blob_bytes, p->lmax, (uint64_t)p->tiles_r, (uint64_t)p->tiles_c);
  p->table_off = L.table_off;
  p->sched_off = L.sched_off;
  p->scratch_off = L.scratch_off;
  p->device_bytes = L.device_bytes;
  return 0;
}

int plan_build_rank(const uint16_t* w, int64_t rows, int64_t cols, uint32_t tile_cols,
                    uint32_t ranks, uint32_t threads, nwc_plan_s* p) {
  if (ranks < 1 || ranks > (uint32_t)kMaxRanks) return -1;
  p->code_kind = 1;
  p->rows = rows;
  p->cols = cols;
  p->tile_rows = kTileRows;
  p->tile_cols = tile_cols;
  p->threads = hardware_threads(threads);
  p->tiles_r = (rows + kTileRows - 1) / kTileRows;
  p->tiles_c = (cols + tile_cols - 1) / tile_cols;
  p->tiles = p->tiles_r * p->tiles_c;

  // Counts of e over the real weights, one partial per thread.
  const unsigned nt = p->threads;
  std::vector<std::vector<uint64_t>> part(nt, std::vector<uint64_t>(128, 0));
  {
    std::vector<std::thread> pool;
    for (unsigned q = 0; q < nt; ++q) {
      pool.emplace_back([&, q] {
        const int64_t b = rows * q / nt, e = rows * (q + 1) / nt;
        uint64_t* h = part[q].data();
        for (int64_t r = b; r < e; ++r) {
          const uint16_t* row = w + r * cols;
          for (int64_t c = 0; c < cols; ++c) h[rank_field(row[c])] += 1;
        }
      });
    }
    for (auto& t : pool) t.join();
  }
  uint64_t cnt[128] = {};
  for (unsigned q = 0; q < nt; ++q)
    for (int e = 0; e < 128; ++e) cnt[e] += part[q][e];
  // The filler is the most frequent value (smallest on a tie), counted too.
  uint32_t filler = 0;
  for (uint32_t e = 1; e < 128; ++e)
    if (cnt[e] > cnt[filler]) filler = e;
  p->filler = filler;
  cnt[filler] += (uint64_t)(p->tiles_r * kTileRows) * (uint64_t)(p->tiles_c * tile_cols) -
                 (uint64_t)rows * (uint64_t)cols;
  // Ranks by count, largest first, smaller value first on a tie.
  std::vector<int> present;
  for (int e = 0; e < 128; ++e)
    if (cnt[e]) present.push_back(e);
  std::stable_sort(present.begin(), present.end(), [&](int a, int b) { return cnt[a] > cnt[b]; });
  p->ranks = (uint32_t)std::min<size_t>(present.size(), ranks);
  p->lmax = p->ranks;
  // Code after the sign bit: rank r -> r zeros and a one; escape -> R zeros and e.
  for (int e = 0; e < 128; ++e) {
    p->rank_len[e] = (uint8_t)(p->ranks + 7);
    p->rank_code[e] = (uint32_t)e;
  }
  for (uint32_t r = 0; r < p->ranks; ++r) {
    const int e = present[r];
    p->rank_table[r] = (uint8_t)e;
    p->rank_len[e] = (uint8_t)(r + 1);
    p->rank_code[e] = 1;
  }
  p->coded_bits = 0;
  for (int e = 0; e < 128; ++e) p->coded_bits += cnt[e] * (uint64_t)(p->rank_len[e] + 1);
  const int rc = plan_tiles(w, p);
  if (rc != 0) return rc;
  const ImageLayout L =
      image_layout(p->blob_bytes, p->lmax, (uint64_t)p->tiles_r, (uint64_t)p->tiles_c, true);
  p->table_off = L.table_off;
  p->sched_off = L.sched_off;
  p->scratch_off = L.scratch_off;
  p->device_bytes = L.device_bytes;
  return 0;
}

int plan_build_escape(const uint16_t* w, int64_t rows, int64_t cols, uint32_t tile_cols,
                      uint32_t lmax, uint32_t keep, uint32_t threads, nwc_plan_s* p) {
  if (keep < 1 || keep > 256) return -1;
  if (lmax == 0) lmax = kEscMaxLmax;
  if (lmax > kEscMaxLmax) return -1;
  p->code_kind = 2;
  p->streams = 1;
  p->rows = rows;
  p->cols = cols;
  p->tile_rows = kTileRows;
  p->tile_cols = tile_cols;
  p->lmax = lmax;
  p->threads = hardware_threads(threads);
  p->tiles_r = (rows + kTileRows - 1) / kTileRows;
  p->tiles_c = (cols + tile_cols - 1) / tile_cols;
  p->tiles = p->tiles_r * p->tiles_c;

  // Histogram with the fillers; the filler is the most frequent exponent.
  uint64_t cnt[256];
  exponent_histogram(w, rows, cols, p->threads, cnt);
  uint32_t filler = 0;
  for (uint32_t s = 1; s < 256; ++s)
    if (cnt[s] > cnt[filler]) filler = s;
  p->filler = filler;
  cnt[filler] += (uint64_t)(p->tiles_r * kTileRows) * (uint64_t)(p->tiles_c * tile_cols) -
                 (uint64_t)rows * (uint64_t)cols;
  // The kept exponents: the `keep` most frequent, smaller symbol first on a tie.
  std::vector<int> present;
  for (int s = 0; s < 256; ++s)
    if (cnt[s]) present.push_back(s);
  std::stable_sort(present.begin(), present.end(), [&](int a, int b) { return cnt[a] > cnt[b]; });
  bool kept[256] = {};
  p->keep = (uint32_t)std::min<size_t>(present.size(), keep);
  for (uint32_t q = 0; q < p->keep; ++q) kept[present[q]] = true;

  // Verbatim runs per tile, and the histogram of the other runs (one partial
  // per part of the tiles).
  const int groups = (int)(tile_cols / 64);
  p->esc_flags.assign((size_t)(8 * p->tiles), 0);
  const unsigned parts = (unsigned)std::min<int64_t>(p->threads, p->tiles);
  std::vector<std::vector<uint64_t>> part(parts, std::vector<uint64_t>(256, 0));
  std::vector<uint64_t> part_runs(parts, 0);
  {
    std::vector<std::thread> pool;
    for (unsigned q = 0; q < parts; ++q) {
      pool.emplace_back([&, q] {
        const int64_t b = p->tiles * q / parts, e = p->tiles * (q + 1) / parts;
        uint64_t* h = part[q].data();
        for (int64_t u = b; u < e; ++u) {
          const int64_t i = u % p->tiles_r, j = u / p->tiles_r;
          TileView v{w, rows, cols, i * kTileRows, j * (int64_t)tile_cols, (uint8_t)filler};
          for (int r = 0; r < kTileRows; ++r) {
            for (int m = 0; m < groups; ++m) {
              uint64_t run[256 / 64] = {};  // exponents present in the run
              for (int c = 64 * m; c < 64 * m + 64; ++c) {
                const uint8_t s = v.inside(r, c) ? exponent_byte(v.at(r, c)) : v.filler;
                run[s / 64] |= 1ull << (s % 64);
              }
              bool rare = false;
              for (int s = 0; s < 256 && !rare; ++s) rare = ((run[s / 64] >> (s % 64)) & 1u) && !kept[s];
              if (rare) {
                p->esc_flags[(size_t)(8 * u + r)] |= (uint8_t)(1u << m);
                part_runs[q] += 1;
                continue;
              }
              for (int c = 64 * m; c < 64 * m + 64; ++c)
                h[v.inside(r, c) ? exponent_byte(v.at(r, c)) : v.filler] += 1;
            }
          }
        }
      });
    }
    for (auto& t : pool) t.join();
  }
  uint64_t ccnt[256] = {};
  p->n_escaped = 0;
  for (unsigned q = 0; q < parts; ++q) {
    for (int s = 0; s < 256; ++s) ccnt[s] += part[q][s];
    p->n_escaped += part_runs[q];
  }
  uint64_t coded = 0;
  for (int s = 0; s < 256; ++s) coded += ccnt[s];
  std::memset(p->len, 0, sizeof(p->len));
  if (coded && !code_lengths(ccnt, lmax, p->len)) return -1;
  canonical_codes(p->len, p->code);
  p->coded_bits = 0;
  for (int s = 0; s < 256; ++s) p->coded_bits += ccnt[s] * p->len[s];
  const int rc = plan_tiles(w, p);
  if (rc != 0) return rc;
  const ImageLayout L =
      image_layout(p->blob_bytes, p->lmax, (uint64_t)p->tiles_r, (uint64_t)p->tiles_c);
  p->table_off = L.table_off;
  p->sched_off = L.sched_off;
  p->scratch_off = L.scratch_off;
  p->device_bytes = L.device_bytes;
  return 0;
}

void build_rank_table(const uint8_t* ranked, uint32_t ranks, uint32_t* out) {
  std::memset(out, 0, kRankTableBytes);
  uint8_t bytes[8] = {};
  for (uint32_t r = 0; r < ranks && r < (uint32_t)kMaxRanks; ++r) bytes[r] = ranked[r];
  std::memcpy(out, bytes, 8);
  out[2] = ranks;
}

// Chunk sizes -> index, tile-area offset and blob size (either code).
int plan_tiles(const uint16_t* w, nwc_plan_s* p) {
  const unsigned nt = p->threads;
  const uint32_t tile_cols = p->tile_cols;
  std::vector<uint32_t> chunk16((size_t)p->tiles);
  const int n = kLanes * (int)p->streams;
  parallel_for(p->tiles, nt, [&](int64_t b, int64_t e) {
    uint32_t bits[kLanes * kMaxStreams];
    for (int64_t u = b; u < e; ++u) {
      lane_bits(*p, w, u, bits);
      uint32_t bytes =
          raw_bytes(tile_cols) + n + (uint32_t)round_up(stream_bytes_of(bits, n), 16);
      if (p->code_kind == 2) bytes += kEscFlagBytes + kEscRunBytes * escaped_runs(*p, u);
      chunk16[(size_t)u] = bytes / 16;
    }
  });
  p->index.assign((size_t)p->tiles + 1, 0);
  uint64_t acc = 0;
  for (int64_t u = 0; u < p->tiles; ++u) {
    p->index[(size_t)u] = (uint32_t)acc;
    acc += chunk16[(size_t)u];
    if (acc > 0xFFFFFFFFull) return -2;  // more than 64 GiB of tile data
  }
  p->index[(size_t)p->tiles] = (uint32_t)acc;
  p->tiles_off = round_up(kIndexOffset + 4ull * (uint64_t)(p->tiles + 1), 256);
  p->blob_bytes = p->tiles_off + 16ull * acc;
  return 0;
}

void encode_blob(const nwc_plan_s& p, const uint16_t* w, uint8_t* blob) {
  BlobHeader h;
  std::memset(&h, 0, sizeof(h));
  h.magic = p.code_kind == 0 ? kMagic : p.code_kind == 1 ? kRankMagic : kEscMagic;
  h.version = kVersion;
  h.header_bytes = kHeaderBytes;
  h.lmax = p.lmax;
  h.rows = (uint64_t)p.rows;
  h.cols = (uint64_t)p.cols;
  h.tile_rows = kTileRows;
  h.tile_cols = p.tile_cols;
  h.tiles_r = (uint64_t)p.tiles_r;
  h.tiles_c = (uint64_t)p.tiles_c;
  h.filler = p.filler;
  h.zero = p.code_kind == 2 ? p.keep : p.streams - 1;  // NWE1: K; else S - 1
  h.lens_off = kLensOffset;
  h.index_off = kIndexOffset;
  h.tiles_off = p.tiles_off;
  h.total_bytes = p.blob_bytes;
  h.coded_bits = p.coded_bits;
  if (p.code_kind == 2) std::memcpy(h.pad, &p.n_escaped, 8);  // offset 104
  std::memset(blob, 0, p.tiles_off);
  std::memcpy(blob, &h, sizeof(h));
  if (p.code_kind != 1)
    std::memcpy(blob + kLensOffset, p.len, 256);
  else
    std::memcpy(blob + kLensOffset, p.rank_table, p.ranks);
  std::memcpy(blob + kIndexOffset, p.index.data(), 4 * p.index.size());

  const uint32_t groups = p.tile_cols / 64;
  const uint32_t raw_n = raw_bytes(p.tile_cols);
  const int S = (int)p.streams;
  const uint32_t nstreams = kLanes * (uint32_t)S;
  parallel_for(p.tiles, p.threads, [&](int64_t b, int64_t e) {
    std::vector<uint8_t> seq;  // big-endian bytes of the stream run
    for (int64_t u = b; u < e; ++u) {
      const int64_t i = u % p.tiles_r, j = u / p.tiles_r;
      TileView v{w, p.rows, p.cols, i * kTileRows, j * (int64_t)p.tile_cols, (uint8_t)p.filler};
      uint8_t* chunk = blob + p.tiles_off + 16ull * p.index[(size_t)u];
      const uint32_t chunk_bytes = 16u * (p.index[(size_t)u + 1] - p.index[(size_t)u]);
      const bool esc = p.code_kind == 2;
      const uint32_t head =
          raw_n + (esc ? kEscFlagBytes + kEscRunBytes * escaped_runs(p, u) : 0u);
      const uint32_t area = chunk_bytes - head - nstreams;
      uint8_t* raw = chunk;
      uint8_t* lane_len = chunk + head;
      uint8_t* words = chunk + head + nstreams;
      if (esc) {
        // Flags, then the verbatim runs' exponent bytes in (row, group) order.
        uint8_t* flags = chunk + raw_n;
        std::memset(flags, 0, kEscFlagBytes);
        uint8_t* run = flags + kEscFlagBytes;
        for (int r = 0; r < kTileRows; ++r) {
          flags[r] = p.esc_flags[(size_t)(8 * u + r)];
          for (uint32_t g = 0; g < groups; ++g) {
            if (!escaped(p, u, r, (int)g)) continue;
            for (int c = (int)(64 * g); c < (int)(64 * g) + 64; ++c)
              *run++ = v.inside(r, c) ? exponent_byte(v.at(r, c)) : v.filler;
          }
        }
      }
      seq.assign(area, 0);
      uint32_t out = 0;
      for (int sigma = 0; sigma < (int)nstreams; ++sigma) {
        const uint32_t lane_start = out;
        uint32_t accb = 0;  // pending bits, right-aligned
        int nacc = 0;
        // Stream sigma belongs to lane t = sigma / S = 4 r + q, which owns row
        // r; group g gives it columns 64 g + 16 q .. 64 g + 16 q + 15, symbols
        // 16 g .. 16 g + 15, of which this stream takes those of its pairs.
        const int t = sigma / S;
        const int r = t / 4;
        for (uint32_t g = 0; g < groups; ++g) {
          for (int kk = 0; kk < 16; ++kk) {
            const int c = (int)(64 * g) + 16 * (t % 4) + kk;
            const int k = (int)(16 * g) + kk;
            if (stream_of(t, k, S) != sigma) continue;
            uint32_t code;
            int len;
            uint8_t rb;
            symbol_of(p, v, r, c, &code, &len, &rb);
            raw[(k / 16) * 512 + 16 * t + (k % 16)] = rb;
            if (esc && escaped(p, u, r, (int)g)) continue;  // verbatim: no bits
            accb = (accb << len) | code;
            nacc += len;
            while (nacc >= 8) {
              seq[out++] = (uint8_t)(accb >> (nacc - 8));
              nacc -= 8;
            }
            accb &= (1u << nacc) - 1u;
          }
        }
        if (nacc > 0) seq[out++] = (uint8_t)(accb << (8 - nacc));
        lane_len[sigma] = (uint8_t)(out - lane_start);
      }
      // Little-endian words with the earliest bit in bit 31.
      for (uint32_t q = 0; q < area; q += 4) {
        words[q + 0] = seq[q + 3];
        words[q + 1] = seq[q + 2];
        words[q + 2] = seq[q + 1];
        words[q + 3] = seq[q + 0];
      }
    }
  });
}

bool parse_blob(const uint8_t* blob, uint64_t head_bytes, uint64_t bytes, nwc_handle_s* hd,
                const uint8_t** lens_out) {
  if (!blob || head_bytes < kHeaderBytes + 256 || head_bytes > bytes) return false;
  BlobHeader h;
  std::memcpy(&h, blob, sizeof(h));
  const bool rank = h.magic == kRankMagic, esc = h.magic == kEscMagic;
  if ((h.magic != kMagic && !rank && !esc) || h.version != kVersion ||
      h.header_bytes != kHeaderBytes)
    return false;
  const uint32_t lmax_cap =
      rank ? (uint32_t)kMaxRanks : esc ? kEscMaxLmax : (uint32_t)kMaxLmax;
  if (h.lmax < 1 || h.lmax > lmax_cap || h.tile_rows != (uint32_t)kTileRows) return false;
  if (h.tile_cols < 64 || h.tile_cols > (uint32_t)kMaxTileCols || h.tile_cols % 64) return false;
  if (h.rows < 1 || h.cols < 1 || h.rows > (1ull << 40) || h.cols > (1ull << 40)) return false;
  if (h.tiles_r != (h.rows + 7) / 8 || h.tiles_c != (h.cols + h.tile_cols - 1) / h.tile_cols)
    return false;
  if (h.lens_off != kLensOffset || h.index_off != kIndexOffset || h.filler > 255) return false;
  // The streams field holds S - 1 for S bit streams per lane (1 or 2 here;
  // the ranked unary code has one); NWE1 has one and holds K there.
  if (esc ? (h.zero < 1 || h.zero > 256) : h.zero + 1 > (rank ? 1u : kMaxDeviceStreams))
    return false;
  const uint32_t S = esc ? 1u : h.zero + 1;
  // Every tile has a 4-byte index entry inside the head, which bounds the tile
  // count before it is formed: no size computed from it below can wrap around.
  const uint64_t max_tiles = head_bytes / 4;
  if (h.tiles_r > max_tiles || h.tiles_c > max_tiles / h.tiles_r) return false;
  const uint64_t tiles = h.tiles_r * h.tiles_c;
  if (h.tiles_off != round_up(kIndexOffset + 4 * (tiles + 1), 256)) return false;
  if (h.total_bytes != bytes || h.tiles_off > head_bytes) return false;
  const uint8_t* lens = blob + kLensOffset;
  if (rank) {
    // R distinct values of the 7-bit field in rank order, then zeros; rank 0
    // is the filler's.
    bool seen[128] = {};
    for (uint32_t r = 0; r < 256; ++r) {
      if (r >= h.lmax) {
        if (lens[r]) return false;
        continue;
      }
      if (lens[r] > 127 || seen[lens[r]]) return false;
      seen[lens[r]] = true;
    }
    if (h.filler != lens[0]) return false;
  } else {
    double kraft = 0;
    uint32_t coded = 0;
    for (int s = 0; s < 256; ++s) {
      if (lens[s] > h.lmax) return false;
      if (lens[s]) {
        kraft += 1.0 / double(1u << lens[s]);
        ++coded;
      }
    }
    if (kraft > 1.0) return false;
    // NWE1: no more codes than kept exponents (none at all when every run is
    // verbatim, so the filler may have none); NWB1: the filler has a code.
    if (esc ? coded > h.zero : lens[h.filler] == 0) return false;
  }
  auto index_at = [&](uint64_t u) {
    uint32_t v;
    std::memcpy(&v, blob + kIndexOffset + 4 * u, 4);
    return v;
  };
  const uint64_t max_chunk = rank  ? max_rank_chunk_bytes(h.tile_cols, h.lmax)
                             : esc ? max_escape_chunk_bytes(h.tile_cols, h.lmax)
                                   : max_chunk_bytes(h.tile_cols, h.lmax, S);
  const uint64_t min_chunk = raw_bytes(h.tile_cols) + kLanes * S + (esc ? kEscFlagBytes : 0u);
  uint64_t largest = 0;
  if (index_at(0) != 0) return false;
  uint32_t prev = 0;
  for (uint64_t u = 0; u < tiles; ++u) {
    const uint32_t nxt = index_at(u + 1);
    if (nxt < prev) return false;
    const uint64_t c = 16ull * (uint64_t)(nxt - prev);
    if (c < min_chunk || c > max_chunk) return false;
    largest = std::max(largest, c);
    prev = nxt;
  }
  if (h.tiles_off + 16ull * prev != bytes) return false;
  hd->rows = (int64_t)h.rows;
  hd->cols = (int64_t)h.cols;
  hd->tile_cols = h.tile_cols;
  hd->lmax = h.lmax;
  hd->streams = S;
  hd->code_kind = rank ? 1u : esc ? 2u : 0u;
  hd->filler = h.filler;
  hd->tiles_r = (int64_t)h.tiles_r;
  hd->tiles_c = (int64_t)h.tiles_c;
  hd->tiles = (int64_t)tiles;
  hd->index_off = kIndexOffset;
  hd->index.resize((size_t)tiles + 1);
  std::memcpy(hd->index.data(), blob + kIndexOffset, 4 * ((size_t)tiles + 1));
  hd->tiles_off = h.tiles_off;
  hd->blob_bytes = bytes;
  const ImageLayout L = image_layout(bytes, h.lmax, h.tiles_r, h.tiles_c, rank);
  hd->table_off = L.table_off;
  hd->sched_off = L.sched_off;
  hd->scratch_off = L.scratch_off;
  hd->device_bytes = L.device_bytes;
  hd->max_chunk = largest;
  if (lens_out) *lens_out = lens;
  return true;
}

}  // namespace nwc
