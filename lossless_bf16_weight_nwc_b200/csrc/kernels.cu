// kernels.cu — sm_100a kernels: fused decode-GEMV and bit-exact decompress.
//
// What runs where ("NWC — Neural Weight Compression", "How it works > Fused
// kernel"; "Unweight", "Direct GPU Decompression"):
//   * Each warp owns a contiguous range of tiles (8 rows x tile_cols), in the
//     blob's column-block-major order, so it keeps one slice of x for long runs.
//   * Lane 0 of the warp streams the tile chunks (raw plane + lane streams)
//     from HBM into a per-warp shared-memory ring with cp.async.bulk (no
//     multicast), each completion counted by an mbarrier.  Every wait is
//     bounded: a wait that gives up sets the device error word and the warp
//     drains its copies and stops.
//   * Each lane decodes its own bit stream: a 64-bit window, a 12-bit peek into
//     a 4096-entry table in shared memory that yields two exponent bytes at
//     their BF16 positions ("NWC", "Prefix code instead of rANS"), a funnel
//     shift by the consumed length, and a refill from shared memory every two
//     steps.  A peek whose two codes do not fit in 12 bits takes a second
//     lookup.
//   * BF16x2 reassembly is one byte permute of the raw plane and one bitwise
//     select with the table entry; the weights never leave registers.
//   * GEMV: FP32 FMAs into 8 row sums per batch row, a transposed warp-shuffle
//     reduction per tile, and a split-K reduction in a fixed order through the
//     workspace (the last warp to finish a row block sums the partials).
//   * Decompress: the same decode, with a 32-bit store per weight pair, one
//     128-byte line per warp store.
#include <cuda_runtime.h>

#include <cstdint>

#include "kernels.cuh"
#include "nwc_format.h"

namespace nwc {

__device__ unsigned int g_device_error;

namespace {

constexpr int kDepth = 4;                  // tiles in flight per warp
constexpr uint32_t kWaitLimit = 1u << 22;  // bounded mbarrier polls
constexpr int kMaxWarps = 16;
constexpr int kRingSlack = 16;             // lanes may read a few words past a chunk
constexpr unsigned kFull = 0xFFFFFFFFu;

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return (uint32_t)__cvta_generic_to_shared(p);
}
__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count)
               : "memory");
}
__device__ __forceinline__ void mbar_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)),
               "r"(bytes)
               : "memory");
}
__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}
// Bulk copy global -> this CTA's shared memory, completion counted in bytes on
// `bar`.  Plain (non-multicast) form.
__device__ __forceinline__ void bulk_load(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
          smem_u32(dst)),
      "l"(src), "r"(bytes), "r"(smem_u32(bar))
      : "memory");
}
__device__ __forceinline__ void fence_barrier_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}
__device__ __forceinline__ void fence_proxy_async() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// Polls `bar` for `parity` at most kWaitLimit times; on failure records a
// timeout in the device error word.
__device__ bool wait_bounded(uint64_t* bar, uint32_t parity) {
  for (uint32_t it = 0; it < kWaitLimit; ++it)
    if (mbar_try_wait(bar, parity)) return true;
  atomicOr(&g_device_error, kErrTimeout);
  return false;
}

__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

// Per-lane bit reader over the lane's stream in shared memory.  Invariant at
// every refill point: at least 32 valid bits; one step consumes at most 12, so
// two steps always have the 12 valid bits a peek needs.  The low 7 bits of
// `nbacc` count valid bits; subtracting whole table entries keeps them exact
// because entry bits 4..6 are zero and bits 0..3 hold the consumed count.
struct BitReader {
  uint32_t hi, lo, nbacc;
  const uint32_t* wp;

  __device__ __forceinline__ void init(const uint8_t* area, uint32_t start) {
    wp = reinterpret_cast<const uint32_t*>(area) + (start >> 2);
    const uint32_t sh = (start & 3u) * 8u;
    const uint32_t w0 = wp[0], w1 = wp[1];
    hi = __funnelshift_l(w1, w0, sh);
    lo = w1 << sh;
    nbacc = 64u - sh;
    wp += 2;
  }
  __device__ __forceinline__ uint32_t peek() const { return hi >> (32 - kPeekBits); }
  // Consume the count held in bits 0..3 of e (upper bits are ignored by the
  // funnel shifts, which use e & 31).
  __device__ __forceinline__ void consume_entry(uint32_t e) {
    hi = __funnelshift_l(lo, hi, e);
    lo = __funnelshift_l(0u, lo, e);
    nbacc -= e;
  }
  __device__ __forceinline__ void consume_bits(uint32_t n) {
    hi = __funnelshift_l(lo, hi, n);
    lo = lo << n;
    nbacc -= n;
  }
  __device__ __forceinline__ void refill() {
    const uint32_t nb = nbacc & 127u;
    if (nb < 32u) {
      const uint32_t w = *wp++;
      const uint64_t win = ((uint64_t)hi << 32 | lo) | ((uint64_t)w << (32u - nb));
      hi = (uint32_t)(win >> 32);
      lo = (uint32_t)win;
      nbacc += 32u;
    }
  }
};

// Decodes one step: two exponent bytes at their BF16 positions in a table
// entry (bits 7..14 and 23..30).
__device__ __forceinline__ uint32_t decode_pair(BitReader& br, const uint32_t* table) {
  uint32_t e = table[br.peek()];
  br.consume_entry(e);
  if ((int32_t)e < 0) {
    // The second code did not fit in the peek: look it up on its own.
    br.refill();
    const uint32_t e2 = table[br.peek()];
    br.consume_bits((e2 >> kEntryLen0Shift) & 15u);
    e = (e & ~0x7F800000u) | ((e2 << 16) & 0x7F800000u) | (e2 & kEntryInvalid);
  }
  return e;
}

// Raw bytes of step r (row r of a 64-column group) duplicated into both bytes
// of each half: [r0, r0, r1, r1].
template <int R>
__device__ __forceinline__ uint32_t raw_pair(const uint4& rv) {
  const uint32_t w = (R < 2) ? rv.x : (R < 4) ? rv.y : (R < 6) ? rv.z : rv.w;
  return __byte_perm(w, 0u, (R & 1) ? 0x3322u : 0x1100u);
}

__device__ __forceinline__ uint32_t assemble(uint32_t rawdup, uint32_t e) {
  // Select sign+fraction from the raw bytes and the exponents from the entry.
  return (rawdup & kEntryRawMask) | (e & kEntryExponentMask);
}

// Lane-distributed per-warp staging pipeline (all lanes keep identical state;
// lane 0 issues the copies; lane s < kDepth holds the ring position of slot s).
struct Pipeline {
  const uint8_t* tiles;
  const uint32_t* index;
  uint8_t* ring;
  uint64_t* bars;
  int64_t u0, n;          // this warp's tiles [u0, u0 + n)
  int64_t issued, consumed;
  uint32_t ring_bytes;
  uint32_t vhead, vtail;  // virtual ring positions
  uint32_t slot_vpos;     // lane s: virtual start of slot s
  int64_t wb;             // index window base
  uint32_t idx_a, idx_b;  // index[wb + lane], index[wb + 32 + lane]
  int64_t n_index;        // entries in index (tiles + 1)
  int lane;

  __device__ __forceinline__ uint32_t load_index(int64_t e) const {
    return e < n_index ? __ldg(index + e) : 0u;
  }
  __device__ void init(const uint8_t* t, const uint32_t* ix, int64_t n_tiles, uint8_t* r,
                       uint32_t rb, uint64_t* b, int64_t first, int64_t count, int ln) {
    tiles = t;
    index = ix;
    ring = r;
    ring_bytes = rb;
    bars = b;
    u0 = first;
    n = count;
    issued = consumed = 0;
    vhead = vtail = 0;
    slot_vpos = 0;
    lane = ln;
    n_index = n_tiles + 1;
    wb = u0;
    idx_a = load_index(wb + lane);
    idx_b = load_index(wb + 32 + lane);
  }
  __device__ __forceinline__ uint32_t index_at(int64_t e) {
    while (e - wb >= 64) {  // slide the window (uniform across the warp)
      wb += 32;
      idx_a = idx_b;
      idx_b = load_index(wb + 32 + lane);
    }
    const int d = (int)(e - wb);
    const uint32_t va = __shfl_sync(kFull, idx_a, d & 31);
    const uint32_t vb = __shfl_sync(kFull, idx_b, d & 31);
    return d < 32 ? va : vb;
  }
  // Issue copies while the ring has room and fewer than kDepth are in flight.
  __device__ void issue() {
    while (issued < n && issued - consumed < kDepth) {
      const int64_t u = u0 + issued;
      const uint32_t c0 = index_at(u), c1 = index_at(u + 1);
      const uint32_t bytes = (c1 - c0) * 16u;
      uint32_t p = vhead;
      if (p % ring_bytes + bytes > ring_bytes) p = (p / ring_bytes + 1) * ring_bytes;
      const bool empty = issued == consumed;
      if (!empty && p + bytes - vtail > ring_bytes) break;
      if (empty) vtail = p;
      const int slot = (int)(issued % kDepth);
      if (lane == slot) slot_vpos = p;
      if (lane == 0) {
        mbar_expect_tx(&bars[slot], bytes);
        bulk_load(ring + p % ring_bytes, tiles + 16ull * c0, bytes, &bars[slot]);
      }
      vhead = p + bytes;
      ++issued;
    }
  }
  // Waits for tile `consumed`; returns its chunk or nullptr on timeout.
  __device__ const uint8_t* wait_current() {
    const int slot = (int)(consumed % kDepth);
    const uint32_t parity = (uint32_t)((consumed / kDepth) & 1);
    const bool ok = wait_bounded(&bars[slot], parity);
    if (!__all_sync(kFull, ok)) return nullptr;
    const uint32_t p = __shfl_sync(kFull, slot_vpos, slot);
    return ring + p % ring_bytes;
  }
  __device__ void release_current() {
    __syncwarp();
    ++consumed;
    if (issued > consumed)
      vtail = __shfl_sync(kFull, slot_vpos, (int)(consumed % kDepth));
    else
      vtail = vhead;
    if (lane == 0) fence_proxy_async();
    __syncwarp();
  }
  // After a timeout: wait (bounded) for every copy still in flight.
  __device__ void drain() {
    for (int64_t c = consumed; c < issued; ++c)
      wait_bounded(&bars[c % kDepth], (uint32_t)((c / kDepth) & 1));
  }
};

// Shared-memory layout: decode table | table barrier | per-warp barriers |
// per-warp rings.
__host__ __device__ inline size_t ring_offset(int warps) {
  return ((size_t)kTableBytes + 8 + (size_t)warps * kDepth * 8 + 15) / 16 * 16;
}
__host__ __device__ inline size_t smem_bytes_for(int warps, int ring_bytes) {
  return ring_offset(warps) + (size_t)warps * (size_t)(ring_bytes + kRingSlack);
}

// Sums 8 per-lane row values over the 32 lanes.  On return every lane holds the
// total of row (lane >> 2).
__device__ __forceinline__ float reduce_rows8(const float (&v)[8], int lane) {
  float a[4], b[2];
  const bool h16 = lane & 16, h8 = lane & 8, h4 = lane & 4;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float send = h16 ? v[i] : v[4 + i];
    const float keep = h16 ? v[4 + i] : v[i];
    a[i] = keep + __shfl_xor_sync(kFull, send, 16);
  }
#pragma unroll
  for (int i = 0; i < 2; ++i) {
    const float send = h8 ? a[i] : a[2 + i];
    const float keep = h8 ? a[2 + i] : a[i];
    b[i] = keep + __shfl_xor_sync(kFull, send, 8);
  }
  const float send = h4 ? b[0] : b[1];
  const float keep = h4 ? b[1] : b[0];
  float c = keep + __shfl_xor_sync(kFull, send, 4);
  c += __shfl_xor_sync(kFull, c, 2);
  c += __shfl_xor_sync(kFull, c, 1);
  return c;
}

template <int CP, int B>
struct GemvState {
  float acc[8][B];
  float xl[CP][B], xh[CP][B];  // x pairs of this lane's columns
  int64_t xcol_block;          // column block whose x is loaded
};

template <int CP, int B, bool RAGGED>
__device__ __forceinline__ void decode_gemv_tile(const uint8_t* chunk, const uint32_t* table,
                                                 int lane, GemvState<CP, B>& st) {
  constexpr int kRaw = CP * 512;
  const uint32_t my_len = chunk[kRaw + lane];
  uint32_t incl = my_len;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t v = __shfl_up_sync(kFull, incl, o);
    if (lane >= o) incl += v;
  }
  BitReader br;
  br.init(chunk + kRaw + kLanes, incl - my_len);
#pragma unroll
  for (int g = 0; g < CP; ++g) {
    const uint4 rv = *reinterpret_cast<const uint4*>(chunk + g * 512 + lane * 16);
#pragma unroll
    for (int r = 0; r < 8; ++r) {
      const uint32_t e = decode_pair(br, table);
      uint32_t rawdup;
      switch (r) {
        case 0: rawdup = raw_pair<0>(rv); break;
        case 1: rawdup = raw_pair<1>(rv); break;
        case 2: rawdup = raw_pair<2>(rv); break;
        case 3: rawdup = raw_pair<3>(rv); break;
        case 4: rawdup = raw_pair<4>(rv); break;
        case 5: rawdup = raw_pair<5>(rv); break;
        case 6: rawdup = raw_pair<6>(rv); break;
        default: rawdup = raw_pair<7>(rv); break;
      }
      const uint32_t w = assemble(rawdup, e);
      const float wl = bf16_lo(w), wh = bf16_hi(w);
#pragma unroll
      for (int b = 0; b < B; ++b) {
        st.acc[r][b] = fmaf(wl, st.xl[g][b], st.acc[r][b]);
        st.acc[r][b] = fmaf(wh, st.xh[g][b], st.acc[r][b]);
      }
      if (r & 1) br.refill();
    }
  }
}

template <int CP, int B>
__global__ void __launch_bounds__(kMaxWarps * 32, 1) gemv_kernel(TileParams p) {
  extern __shared__ __align__(16) uint8_t smem[];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int warps = blockDim.x >> 5;
  uint32_t* table = reinterpret_cast<uint32_t*>(smem);
  uint64_t* table_bar = reinterpret_cast<uint64_t*>(smem + kTableBytes);
  uint64_t* bars = table_bar + 1 + warp * kDepth;
  uint8_t* ring = smem + ring_offset(warps) + (size_t)warp * (p.ring_bytes + kRingSlack);

  if (threadIdx.x == 0) mbar_init(table_bar, 1);
  if (lane == 0)
    for (int d = 0; d < kDepth; ++d) mbar_init(&bars[d], 1);
  fence_barrier_init();
  __syncthreads();
  if (threadIdx.x == 0) {
    mbar_expect_tx(table_bar, kTableBytes);
    bulk_load(table, p.table, kTableBytes, table_bar);
  }

  const int64_t gw = (int64_t)blockIdx.x * warps + warp;
  const int64_t first = gw < p.total_warps ? p.n_tiles * gw / p.total_warps : 0;
  const int64_t last = gw < p.total_warps ? p.n_tiles * (gw + 1) / p.total_warps : 0;
  Pipeline pl;
  pl.init(p.tiles, p.index, p.n_tiles, ring, (uint32_t)p.ring_bytes, bars, first, last - first,
          lane);
  pl.issue();
  if (!__all_sync(kFull, wait_bounded(table_bar, 0))) {
    if (threadIdx.x == 0) wait_bounded(table_bar, 0);
    pl.drain();
    return;
  }

  GemvState<CP, B> st;
  st.xcol_block = -1;
  const int64_t cols = p.cols;
  for (int64_t c = 0; c < pl.n; ++c) {
    const int64_t u = pl.u0 + c;
    const int64_t i = u % p.tiles_r, j = u / p.tiles_r;
    if (j != st.xcol_block) {  // load this lane's x pairs for column block j
      st.xcol_block = j;
#pragma unroll
      for (int g = 0; g < CP; ++g) {
        const int64_t col = j * (CP * 64) + g * 64 + 2 * lane;
#pragma unroll
        for (int b = 0; b < B; ++b) {
          uint32_t xv = 0;
          if (col + 1 < cols) {
            xv = __ldg(reinterpret_cast<const uint32_t*>(p.x + (int64_t)b * cols + col));
          } else if (col < cols) {
            xv = __ldg(p.x + (int64_t)b * cols + col);
          }
          st.xl[g][b] = bf16_lo(xv);
          st.xh[g][b] = bf16_hi(xv);
        }
      }
    }
#pragma unroll
    for (int r = 0; r < 8; ++r)
#pragma unroll
      for (int b = 0; b < B; ++b) st.acc[r][b] = 0.f;

    const uint8_t* chunk = pl.wait_current();
    if (!chunk) {
      pl.drain();
      return;
    }
    decode_gemv_tile<CP, B, false>(chunk, table, lane, st);
    pl.release_current();
    pl.issue();

    // Row sums of this tile: lane L holds row L >> 2 for every batch row.
    float tot[B];
#pragma unroll
    for (int b = 0; b < B; ++b) {
      float v[8];
#pragma unroll
      for (int r = 0; r < 8; ++r) v[r] = st.acc[r][b];
      tot[b] = reduce_rows8(v, lane);
    }
    const int r = lane >> 2;
    const int64_t row = i * 8 + r;
    if (p.tiles_c == 1) {
      if ((lane & 3) == 0 && row < p.rows)
#pragma unroll
        for (int b = 0; b < B; ++b) p.y[(int64_t)b * p.rows + row] = tot[b];
      continue;
    }
    if ((lane & 3) == 0)
#pragma unroll
      for (int b = 0; b < B; ++b)
        p.partial[((int64_t)j * B + b) * p.rows_pad + row] = tot[b];
    __threadfence();
    __syncwarp();
    uint32_t arrived = 0;
    if (lane == 0) arrived = atomicAdd(&p.counters[i], 1u);
    arrived = __shfl_sync(kFull, arrived, 0);
    if (arrived == (uint32_t)(p.tiles_c - 1)) {
      // Last arrival for row block i: sum the partials in column-block order.
      __threadfence();
      for (int q = lane; q < 8 * B; q += 32) {
        const int b = q >> 3, rr = q & 7;
        const int64_t orow = i * 8 + rr;
        float s = 0.f;
        for (int64_t jj = 0; jj < p.tiles_c; ++jj)
          s += __ldcg(&p.partial[(jj * B + b) * p.rows_pad + orow]);
        if (orow < p.rows) p.y[(int64_t)b * p.rows + orow] = s;
      }
      if (lane == 0) p.counters[i] = 0u;
    }
  }
}

template <int CP>
__global__ void __launch_bounds__(kMaxWarps * 32, 1) decompress_kernel(TileParams p) {
  extern __shared__ __align__(16) uint8_t smem[];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int warps = blockDim.x >> 5;
  uint32_t* table = reinterpret_cast<uint32_t*>(smem);
  uint64_t* table_bar = reinterpret_cast<uint64_t*>(smem + kTableBytes);
  uint64_t* bars = table_bar + 1 + warp * kDepth;
  uint8_t* ring = smem + ring_offset(warps) + (size_t)warp * (p.ring_bytes + kRingSlack);

  if (threadIdx.x == 0) mbar_init(table_bar, 1);
  if (lane == 0)
    for (int d = 0; d < kDepth; ++d) mbar_init(&bars[d], 1);
  fence_barrier_init();
  __syncthreads();
  if (threadIdx.x == 0) {
    mbar_expect_tx(table_bar, kTableBytes);
    bulk_load(table, p.table, kTableBytes, table_bar);
  }
  const int64_t gw = (int64_t)blockIdx.x * warps + warp;
  const int64_t first = gw < p.total_warps ? p.n_tiles * gw / p.total_warps : 0;
  const int64_t last = gw < p.total_warps ? p.n_tiles * (gw + 1) / p.total_warps : 0;
  Pipeline pl;
  pl.init(p.tiles, p.index, p.n_tiles, ring, (uint32_t)p.ring_bytes, bars, first, last - first,
          lane);
  pl.issue();
  if (!__all_sync(kFull, wait_bounded(table_bar, 0))) {
    if (threadIdx.x == 0) wait_bounded(table_bar, 0);
    pl.drain();
    return;
  }
  const int64_t cols = p.cols;
  const bool even_cols = (cols & 1) == 0;
  uint32_t invalid = 0;
  constexpr int kRaw = CP * 512;
  for (int64_t c = 0; c < pl.n; ++c) {
    const int64_t u = pl.u0 + c;
    const int64_t i = u % p.tiles_r, j = u / p.tiles_r;
    const uint8_t* chunk = pl.wait_current();
    if (!chunk) {
      pl.drain();
      return;
    }
    const uint32_t my_len = chunk[kRaw + lane];
    uint32_t incl = my_len;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t v = __shfl_up_sync(kFull, incl, o);
      if (lane >= o) incl += v;
    }
    BitReader br;
    br.init(chunk + kRaw + kLanes, incl - my_len);
    const bool full_tile = (i + 1) * 8 <= p.rows && (j + 1) * (CP * 64) <= cols && even_cols;
#pragma unroll
    for (int g = 0; g < CP; ++g) {
      const uint4 rv = *reinterpret_cast<const uint4*>(chunk + g * 512 + lane * 16);
      const int64_t col = j * (CP * 64) + g * 64 + 2 * lane;
#pragma unroll
      for (int r = 0; r < 8; ++r) {
        const uint32_t e = decode_pair(br, table);
        invalid |= e;
        uint32_t rawdup;
        switch (r) {
          case 0: rawdup = raw_pair<0>(rv); break;
          case 1: rawdup = raw_pair<1>(rv); break;
          case 2: rawdup = raw_pair<2>(rv); break;
          case 3: rawdup = raw_pair<3>(rv); break;
          case 4: rawdup = raw_pair<4>(rv); break;
          case 5: rawdup = raw_pair<5>(rv); break;
          case 6: rawdup = raw_pair<6>(rv); break;
          default: rawdup = raw_pair<7>(rv); break;
        }
        const uint32_t w = assemble(rawdup, e);
        const int64_t row = i * 8 + r;
        if (full_tile) {
          *reinterpret_cast<uint32_t*>(p.out + row * cols + col) = w;
        } else if (row < p.rows) {
          if (col < cols) p.out[row * cols + col] = (uint16_t)w;
          if (col + 1 < cols) p.out[row * cols + col + 1] = (uint16_t)(w >> 16);
        }
        if (r & 1) br.refill();
      }
    }
    pl.release_current();
    pl.issue();
  }
  if (__any_sync(kFull, invalid & kEntryInvalid) && lane == 0)
    atomicOr(&g_device_error, kErrCorrupt);
}

// Raises a kernel's dynamic shared-memory limit on the current device once per
// (kernel, device) to the largest size requested so far.
template <typename Kernel>
cudaError_t ensure_smem(Kernel k, size_t bytes, int (&configured)[64]) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  if ((size_t)configured[dev] >= bytes) return cudaSuccess;
  e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
  if (e == cudaSuccess) configured[dev] = (int)bytes;
  return e;
}

template <int CP, int B>
cudaError_t launch_gemv_cp_b(const TileParams& p, const LaunchShape& s, cudaStream_t stream) {
  static int configured[64] = {};
  cudaError_t e = ensure_smem(gemv_kernel<CP, B>, s.smem_bytes, configured);
  if (e != cudaSuccess) return e;
  gemv_kernel<CP, B><<<s.ctas, s.warps_per_cta * 32, s.smem_bytes, stream>>>(p);
  return cudaGetLastError();
}

template <int CP>
cudaError_t launch_gemv_cp(const TileParams& p, const LaunchShape& s, cudaStream_t stream) {
  switch (p.batch) {
    case 1: return launch_gemv_cp_b<CP, 1>(p, s, stream);
    case 2: return launch_gemv_cp_b<CP, 2>(p, s, stream);
    case 3: return launch_gemv_cp_b<CP, 3>(p, s, stream);
    case 4: return launch_gemv_cp_b<CP, 4>(p, s, stream);
    case 5: return launch_gemv_cp_b<CP, 5>(p, s, stream);
    case 6: return launch_gemv_cp_b<CP, 6>(p, s, stream);
    case 7: return launch_gemv_cp_b<CP, 7>(p, s, stream);
    case 8: return launch_gemv_cp_b<CP, 8>(p, s, stream);
    default: return cudaErrorInvalidValue;
  }
}

template <int CP>
cudaError_t launch_decompress_cp(const TileParams& p, const LaunchShape& s, cudaStream_t stream) {
  static int configured[64] = {};
  cudaError_t e = ensure_smem(decompress_kernel<CP>, s.smem_bytes, configured);
  if (e != cudaSuccess) return e;
  decompress_kernel<CP><<<s.ctas, s.warps_per_cta * 32, s.smem_bytes, stream>>>(p);
  return cudaGetLastError();
}

}  // namespace

LaunchShape launch_shape(int64_t n_tiles, uint64_t max_chunk, int sm_count) {
  LaunchShape s;
  const int64_t target = (int64_t)sm_count * kMaxWarps;
  const int64_t warps = n_tiles < target ? n_tiles : target;
  int per_cta = (int)((warps + sm_count - 1) / sm_count);
  if (per_cta < 1) per_cta = 1;
  if (per_cta > kMaxWarps) per_cta = kMaxWarps;
  s.warps_per_cta = per_cta;
  s.ctas = (int)((warps + per_cta - 1) / per_cta);
  // Room for one worst-case chunk and, typically, two ordinary ones.
  const uint64_t ring = (max_chunk + 15) / 16 * 16;
  s.ring_bytes = (int)(ring > 12288 ? ring : 12288);
  s.smem_bytes = smem_bytes_for(per_cta, s.ring_bytes);
  return s;
}

cudaError_t launch_gemv(const TileParams& p, int tile_cols, const LaunchShape& s,
                        cudaStream_t stream) {
  switch (tile_cols) {
    case 512: return launch_gemv_cp<8>(p, s, stream);
    case 256: return launch_gemv_cp<4>(p, s, stream);
    case 128: return launch_gemv_cp<2>(p, s, stream);
    case 64: return launch_gemv_cp<1>(p, s, stream);
    default: return cudaErrorInvalidValue;
  }
}

cudaError_t launch_decompress(const TileParams& p, int tile_cols, const LaunchShape& s,
                              cudaStream_t stream) {
  switch (tile_cols) {
    case 512: return launch_decompress_cp<8>(p, s, stream);
    case 256: return launch_decompress_cp<4>(p, s, stream);
    case 128: return launch_decompress_cp<2>(p, s, stream);
    case 64: return launch_decompress_cp<1>(p, s, stream);
    default: return cudaErrorInvalidValue;
  }
}

cudaError_t read_and_clear_error(uint32_t* word) {
  uint32_t zero = 0;
  cudaError_t e = cudaMemcpyFromSymbol(word, g_device_error, sizeof(uint32_t));
  if (e != cudaSuccess) return e;
  return cudaMemcpyToSymbol(g_device_error, &zero, sizeof(uint32_t));
}

}  // namespace nwc
