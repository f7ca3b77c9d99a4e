// schedule.cpp — the launch schedule of the staging pipeline (host side).
//
// A CTA copies its tiles from HBM into a shared-memory ring in batches of
// consecutive tiles, one bulk copy per batch ("NWC — Neural Weight
// Compression", "How it works > Fused kernel": compressed blocks are staged in
// shared memory and decoded there).  Which bytes a batch moves, where it lands
// in the ring and which earlier batches must have been released first depend
// only on the chunk sizes and the launch shape, so they are worked out here
// once per shape instead of by the producer warp on every launch.
#include <algorithm>
#include <cstring>
#include <vector>

#include "kernels.cuh"
#include "nwc_format.h"

namespace nwc {

void build_schedule(const uint32_t* index, int64_t n_tiles, const LaunchShape& s, uint8_t* out) {
  std::memset(out, 0, sched_class_bytes((uint64_t)n_tiles));
  uint32_t* cta_batch = reinterpret_cast<uint32_t*>(out);
  uint32_t* batch = reinterpret_cast<uint32_t*>(out + sched_batch_off());
  uint32_t* tile_ring = reinterpret_cast<uint32_t*>(out + sched_tile_off((uint64_t)n_tiles));
  const int T = s.batch_tiles;
  const uint64_t R = (uint64_t)s.ring_bytes;
  // Outstanding (issued, not yet released) batches stay below kSlots minus the
  // batches that a consumer warp's next wait can lie beyond its last release.
  const int64_t max_outstanding = kSlots - (kMaxLag + T - 1) / T;
  std::vector<uint64_t> vstart;  // virtual ring position of each batch of the CTA
  uint32_t g = 0;                // batches of the CTAs before this one
  for (int c = 0; c < s.ctas; ++c) {
    const int64_t first = n_tiles * c / s.ctas;
    const int64_t n = n_tiles * (c + 1) / s.ctas - first;
    const int64_t nb = (n + T - 1) / T;
    cta_batch[c] = g;
    vstart.assign((size_t)nb, 0);
    uint64_t vhead = 0;  // virtual position after the last placed batch
    int64_t oldest = 0;  // first batch that may still be unreleased
    for (int64_t k = 0; k < nb; ++k) {
      const int64_t q0 = k * T, q1 = q0 + T < n ? q0 + T : n;
      const uint32_t c0 = index[first + q0], c1 = index[first + q1];
      const uint64_t bytes = 16ull * (c1 - c0);
      uint64_t at = vhead;
      if (at % R + bytes > R) at += R - at % R;  // a batch never wraps
      vstart[(size_t)k] = at;
      // Room: every batch that starts less than R before this one's end must
      // have been released (they are released in order).
      while (oldest < k && vstart[(size_t)oldest] + R < at + bytes) ++oldest;
      int64_t need = oldest;
      if (k - max_outstanding + 1 > need) need = k - max_outstanding + 1;
      uint32_t* d = batch + 4 * (size_t)(g + k);
      d[0] = c0;
      d[1] = (uint32_t)bytes;
      d[2] = (uint32_t)(at % R);
      d[3] = (uint32_t)need;
      for (int64_t q = q0; q < q1; ++q)
        tile_ring[first + q] = (uint32_t)(at % R + 16ull * (index[first + q] - c0));
      vhead = at + bytes;
    }
    g += (uint32_t)nb;
  }
  cta_batch[s.ctas] = g;
}

}  // namespace nwc

namespace nwc {

// The tensor-core kernel's CTAs take their tiles by rectangles (see
// kernels.cuh): CTA c = rs ksplit + ks owns row range rs and column range ks;
// for each M-group of R row tiles, round by round, each team's column block,
// its row tiles in order.  Each tile is one copy of its lane lengths and
// streams (the chunk after its raw plane, which the kernel reads from global
// memory).  Copies are placed in the ring first in, first out, as in
// build_schedule, with fewer than kSlots outstanding; the kernel's consumers
// wait until a copy is issued before they poll its slot.
void build_tc_schedule(const uint32_t* index, int64_t tiles_r, int64_t tiles_c,
                       uint32_t raw_bytes, const TcShape& ts, uint8_t* out) {
  const int64_t tiles = tiles_r * tiles_c;
  std::memset(out, 0, sched_tc_bytes((uint64_t)tiles));
  uint32_t* cta_batch = reinterpret_cast<uint32_t*>(out);
  uint32_t* batch = reinterpret_cast<uint32_t*>(out + sched_batch_off());
  uint32_t* tile_ring = reinterpret_cast<uint32_t*>(out + sched_tc_ring_off((uint64_t)tiles));
  uint32_t* tile_batch = reinterpret_cast<uint32_t*>(out + sched_tc_tbatch_off((uint64_t)tiles));
  const LaunchShape& s = ts.s;
  const int R = ts.rows, TT = ts.teams;
  const int64_t KS = ts.ksplit, row_ranges = s.ctas / ts.ksplit;
  const uint64_t ring = (uint64_t)s.ring_bytes;
  const int64_t max_outstanding = kSlots - 16;
  std::vector<int64_t> order;
  std::vector<uint64_t> vstart;
  uint32_t g = 0;  // batches of the CTAs before this one
  for (int c = 0; c < s.ctas; ++c) {
    const int64_t ks = c % KS, rs = c / KS;
    const int64_t i_lo = tiles_r * rs / row_ranges, i_hi = tiles_r * (rs + 1) / row_ranges;
    const int64_t j_lo = tiles_c * ks / KS, j_hi = tiles_c * (ks + 1) / KS;
    order.clear();
    for (int64_t ig = i_lo; ig < i_hi; ig += R) {
      const int64_t rg = std::min<int64_t>(R, i_hi - ig);
      for (int64_t j0 = j_lo; j0 < j_hi; j0 += TT) {
        for (int t = 0; t < TT && j0 + t < j_hi; ++t) {
          for (int64_t r = 0; r < rg; ++r) order.push_back((j0 + t) * tiles_r + ig + r);
        }
      }
    }
    cta_batch[c] = g;
    const int64_t nb = (int64_t)order.size();
    vstart.assign((size_t)nb, 0);
    uint64_t vhead = 0;
    int64_t oldest = 0;
    for (int64_t k = 0; k < nb; ++k) {
      const int64_t u = order[(size_t)k];
      const uint32_t c0 = index[u] + raw_bytes / 16, c1 = index[u + 1];
      const uint64_t bytes = 16ull * (c1 - c0);
      uint64_t at = vhead;
      if (at % ring + bytes > ring) at += ring - at % ring;  // a copy never wraps
      vstart[(size_t)k] = at;
      while (oldest < k && vstart[(size_t)oldest] + ring < at + bytes) ++oldest;
      int64_t need = oldest;
      if (k - max_outstanding + 1 > need) need = k - max_outstanding + 1;
      uint32_t* d = batch + 4 * (size_t)(g + k);
      d[0] = c0;
      d[1] = (uint32_t)bytes;
      d[2] = (uint32_t)(at % ring);
      d[3] = (uint32_t)need;
      tile_ring[u] = (uint32_t)(at % ring);
      tile_batch[u] = (uint32_t)k;
      vhead = at + bytes;
    }
    g += (uint32_t)nb;
  }
  cta_batch[s.ctas] = g;
}

}  // namespace nwc
