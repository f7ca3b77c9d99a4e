// kernels.cu — sm_100a kernels: fused decode-GEMV and bit-exact decompress.
//
// What runs where ("NWC — Neural Weight Compression", "How it works > Fused
// kernel"; "Unweight", "Direct GPU Decompression"):
//   * One persistent CTA per SM owns a contiguous range of tiles (8 rows x
//     tile_cols), in the blob's column-block-major order.
//   * A producer warp streams the tiles' chunks (raw plane + lane streams) from
//     HBM into one CTA-wide shared-memory ring with cp.async.bulk (no
//     multicast).  Each chunk lands in a slot with a "full" mbarrier (bytes
//     counted) and is handed back through an "empty" mbarrier.  Every wait is
//     bounded: a wait that gives up sets the device error word, and the
//     producer drains its copies before leaving.
//   * 16 consumer warps take the CTA's tiles round-robin.  Each lane decodes its
//     own bit stream with a 64-bit window and a table peek.  With lmax <= 7 the
//     peek is 14 bits and every entry holds two complete codes ("NWC", "Prefix
//     code instead of rANS"), so a step is a lookup plus two funnel shifts.
//     With lmax 8..12 the peek is 12 bits and a pair that does not fit takes a
//     second lookup.  The window is refilled every two steps, without a branch.
//   * BF16x2 reassembly is one byte permute of the raw plane and one bitwise
//     select with the table entry; the weights never leave registers.
//   * GEMV: FP32 accumulation of BF16 x BF16 products (fma.rn.f32.bf16) into 8
//     row sums per batch row, a transposed warp-shuffle reduction per tile, and
//     a split-K reduction in a fixed order through the workspace (the last of a
//     row block's column tiles to finish sums the partials).
//   * Decompress: the same decode, with a 32-bit store per weight pair, one
//     128-byte line per warp store.
#include <cuda_runtime.h>

#include <cstdint>

#include "kernels.cuh"
#include "nwc_format.h"

namespace nwc {

__device__ unsigned int g_device_error;

namespace {

constexpr uint32_t kWaitLimit = 1u << 22;        // bounded mbarrier polls
constexpr int kRingSlack = 16;                   // lanes may read a few words past a chunk
constexpr unsigned kFull = 0xFFFFFFFFu;

// ---- PTX helpers -----------------------------------------------------------

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
__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
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
__device__ __forceinline__ void bulk_load(void* dst, const void* src, uint32_t bytes,
                                          uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
          smem_u32(dst)),
      "l"(src), "r"(bytes), "r"(smem_u32(bar))
      : "memory");
}
__device__ __forceinline__ void fence_barrier_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}
// Polls `bar` for `parity` at most kWaitLimit times; on failure records a
// timeout in the device error word.
__device__ bool wait_bounded(uint64_t* bar, uint32_t parity) {
  for (uint32_t it = 0; it < kWaitLimit; ++it)
    if (mbar_try_wait(bar, parity)) return true;
  atomicOr(&g_device_error, kErrTimeout);
  return false;
}

__device__ __forceinline__ uint32_t lds32(uint32_t addr) {
  uint32_t v;
  asm volatile("ld.shared.u32 %0, [%1];" : "=r"(v) : "r"(addr));
  return v;
}
__device__ __forceinline__ uint4 lds128(uint32_t addr) {
  uint4 v;
  asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "r"(addr));
  return v;
}
// Loads a word only when `need` is non-zero (predicated, no branch); else
// returns 0.
__device__ __forceinline__ uint32_t lds32_if(uint32_t addr, uint32_t need) {
  uint32_t v = 0;
  asm volatile("{\n\t.reg .pred p;\n\tsetp.ne.u32 p, %2, 0;\n\t@p ld.shared.u32 %0, [%1];\n\t}"
               : "+r"(v)
               : "r"(addr), "r"(need));
  return v;
}
// Low word of ({hi, lo} >> (n mod 32)).
__device__ __forceinline__ uint32_t shr_wrap(uint32_t lo, uint32_t hi, uint32_t n) {
  uint32_t r;
  asm("shf.r.wrap.b32 %0, %1, %2, %3;" : "=r"(r) : "r"(lo), "r"(hi), "r"(n));
  return r;
}
// c + bf16(a half) * bf16(b half) in FP32; HI selects the upper halves.
template <bool HI>
__device__ __forceinline__ float fma_bf16(uint32_t a, uint32_t b, float c) {
  float d;
  if (HI)
    asm("{\n\t.reg .b16 al, ah, bl, bh;\n\tmov.b32 {al, ah}, %1;\n\tmov.b32 {bl, bh}, %2;\n\t"
        "fma.rn.f32.bf16 %0, ah, bh, %3;\n\t}"
        : "=f"(d)
        : "r"(a), "r"(b), "f"(c));
  else
    asm("{\n\t.reg .b16 al, ah, bl, bh;\n\tmov.b32 {al, ah}, %1;\n\tmov.b32 {bl, bh}, %2;\n\t"
        "fma.rn.f32.bf16 %0, al, bl, %3;\n\t}"
        : "=f"(d)
        : "r"(a), "r"(b), "f"(c));
  return d;
}

// ---- bit reader --------------------------------------------------------------

// Per-lane reader of the lane's stream in shared memory: a 64-bit window hi:lo
// (next bit = bit 31 of hi) and a valid-bit count.  Invariant at each refill
// point: at least 32 valid bits; a step consumes at most 14 bits, so the two
// steps between refill points always have their peek bits.  The low 7 bits of
// `nbacc` count valid bits; subtracting whole table entries keeps them exact,
// since entry bits 4..6 are zero and bits 0..3 hold the consumed count.
struct BitReader {
  uint32_t hi, lo, nbacc;
  uint32_t wp;  // shared-window address of the next stream word

  __device__ __forceinline__ void init(uint32_t area, uint32_t start) {
    wp = area + (start & ~3u);
    const uint32_t sh = (start & 3u) * 8u;
    const uint32_t w0 = lds32(wp), w1 = lds32(wp + 4);
    hi = __funnelshift_l(w1, w0, sh);
    lo = w1 << sh;
    nbacc = 64u - sh;
    wp += 8;
  }
  // Consumes the count in bits 0..3 of e (the funnel shifts use e & 31).
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
  // With fewer than 32 valid bits (bit 5 of the count clear; the count never
  // reaches 64 at a refill point), append the next word right after the valid
  // bits; the count becomes count | 32 either way.  No branch: the load is
  // predicated and an empty word shifts in nothing.
  __device__ __forceinline__ void refill() {
    const uint32_t need = (~nbacc) & 32u;
    const uint32_t w = lds32_if(wp, need);
    hi |= shr_wrap(w, 0u, nbacc);
    lo |= shr_wrap(0u, w, nbacc);
    wp += need >> 3;
    nbacc |= 32u;
  }
};

// One step: a table entry holding two exponent bytes at their BF16 positions
// (bits 7..14 and 23..30).  FAST: 14-bit peek, both codes always fit.
template <bool FAST>
__device__ __forceinline__ uint32_t decode_pair(BitReader& br, uint32_t table) {
  if (FAST) {
    const uint32_t e = lds32(table + ((br.hi >> 16) & 0xFFFCu));
    br.consume_entry(e);
    return e;
  }
  uint32_t e = lds32(table + ((br.hi >> 18) & 0x3FFCu));
  br.consume_entry(e);
  if (__builtin_expect((int32_t)e < 0, 0)) {
    // The second code did not fit in the 12-bit peek: look it up on its own.
    br.refill();
    const uint32_t e2 = lds32(table + ((br.hi >> 18) & 0x3FFCu));
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
__device__ __forceinline__ uint32_t raw_pair_r(const uint4& rv, int r) {
  switch (r) {
    case 0: return raw_pair<0>(rv);
    case 1: return raw_pair<1>(rv);
    case 2: return raw_pair<2>(rv);
    case 3: return raw_pair<3>(rv);
    case 4: return raw_pair<4>(rv);
    case 5: return raw_pair<5>(rv);
    case 6: return raw_pair<6>(rv);
    default: return raw_pair<7>(rv);
  }
}

__device__ __forceinline__ uint32_t assemble(uint32_t rawdup, uint32_t e) {
  // Sign+fraction from the raw bytes, exponents from the table entry.
  return (rawdup & kEntryRawMask) | (e & kEntryExponentMask);
}

// Start of lane `lane`'s stream: prefix sum of the lane byte counts.
__device__ __forceinline__ uint32_t lane_stream_start(uint32_t chunk, int raw, int lane) {
  const uint32_t b4 = lds32(chunk + raw + (lane & ~3));
  const uint32_t my_len = (b4 >> (8 * (lane & 3))) & 0xFFu;
  uint32_t incl = my_len;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t v = __shfl_up_sync(kFull, incl, o);
    if (lane >= o) incl += v;
  }
  return incl - my_len;
}

// ---- shared-memory layout and the producer ---------------------------------
//
// Tiles move in batches of p.batch_tiles consecutive tiles (consecutive in HBM
// too), one bulk copy per batch, so that each copy is large enough for the copy
// engine to run at full bandwidth.  Where each batch lands in the ring, and how
// many earlier batches must have been released before it may be issued, is
// fixed by the launch schedule that the host computed for this launch shape;
// the producer only follows it.  Batch k of a CTA uses barrier slot k % kSlots:
// a "full" barrier counting its bytes and an "empty" barrier that each of its
// tiles' consumers arrives at once.

struct Smem {
  uint64_t* table_bar;
  uint64_t* full;    // per batch slot: bytes landed
  uint64_t* empty;   // per batch slot: tiles released
  uint8_t* ring;
};

__device__ __forceinline__ Smem carve(uint8_t* smem, const TileParams& p) {
  Smem s;
  s.table_bar = reinterpret_cast<uint64_t*>(smem + p.table_bytes);
  s.full = s.table_bar + 1;
  s.empty = s.full + kSlots;
  s.ring = smem + p.ring_offset;
  return s;
}

// Issues the CTA's nb batches, descriptors desc[0 .. nb): {tile-area offset in
// 16-byte units, bytes, ring offset, batches that must be released first}.
// The whole warp runs the loop (the descriptors travel 32 at a time in its
// registers, the next 32 loaded while the current ones are used); lane 0 waits
// for releases and issues the copies.  The loop body is a handful of
// instructions, so the copies go out as fast as the ring allows.
__device__ void produce(const TileParams& p, uint8_t* smem, const Smem& s, const uint4* desc,
                        int nb, int lane) {
  if (lane == 0) {
    mbar_expect_tx(s.table_bar, p.table_bytes);
    bulk_load(smem, p.table, p.table_bytes, s.table_bar);
  }
  const uint4 none = make_uint4(0u, 0u, 0u, 0u);
  uint4 cur = lane < nb ? __ldg(desc + lane) : none;
  uint4 nxt = 32 + lane < nb ? __ldg(desc + 32 + lane) : none;
  uint32_t released = 0;  // batches whose release lane 0 has observed
  int k = 0;
  for (; k < nb; ++k) {
    const int l = k & 31;
    if (l == 0 && k) {
      cur = nxt;
      nxt = k + 32 + lane < nb ? __ldg(desc + k + 32 + lane) : none;
    }
    const uint32_t src = __shfl_sync(kFull, cur.x, l);
    const uint32_t bytes = __shfl_sync(kFull, cur.y, l);
    const uint32_t at = __shfl_sync(kFull, cur.z, l);
    const uint32_t need = __shfl_sync(kFull, cur.w, l);
    uint32_t ok = 1;
    if (lane == 0) {
      for (; released < need; ++released) {
        if (!wait_bounded(&s.empty[released % kSlots], (released / kSlots) & 1u)) {
          ok = 0;
          break;
        }
      }
      if (ok) {
        uint64_t* bar = &s.full[k % kSlots];
        mbar_expect_tx(bar, bytes);  // arrive (release) + byte count
        bulk_load(s.ring + at, p.tiles + 16ull * src, bytes, bar);
      }
    }
    if (!__shfl_sync(kFull, ok, 0)) break;
  }
  // Leave no copy in flight: batches [0, k) were issued, and those more than
  // kSlots back have been released, hence landed.
  if (lane == 0) {
    for (int j = k - 1; j >= 0 && j >= k - kSlots; --j)
      wait_bounded(&s.full[j % kSlots], (uint32_t)((j / kSlots) & 1));
    wait_bounded(s.table_bar, 0);
  }
}

// Consumer side: wait until tile q's batch k has landed.  The schedule keeps
// fewer than kSlots - ceil(kMaxConsumers / batch_tiles) batches outstanding, so
// by the time a consumer polls slot k % kSlots (after finishing its previous
// tile, at most kMaxConsumers tiles back) the slot's previous batch k - kSlots
// was released long ago: the parity it polls is batch k's.
__device__ __forceinline__ bool wait_batch(const Smem& s, int k) {
  return __all_sync(kFull, wait_bounded(&s.full[k % kSlots], (uint32_t)((k / kSlots) & 1)));
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

__device__ __forceinline__ uint32_t load_x_pair(const uint16_t* x, int64_t cols, int64_t col) {
  if (col + 1 < cols) return __ldg(reinterpret_cast<const uint32_t*>(x + col));
  if (col < cols) return __ldg(x + col);
  return 0u;
}

// One tile of the GEMV: decode the lane's 16 * CP symbols, 8 rows per 64-column
// group, and accumulate acc[r][b] += W[r][c] * x[b][c] in FP32.  The BF16 pair
// of x for each group (columns col0 + 64 g + 2 lane, + 1) is read from L1 one
// group ahead and serves the group's 8 rows.
template <int CP, int B, bool FAST>
__device__ __forceinline__ void decode_gemv_tile(uint32_t chunk, uint32_t table, int lane,
                                                 float (&acc)[8][B], const uint16_t* x,
                                                 int64_t cols, int64_t col0) {
  constexpr int kRaw = CP * 512;
  BitReader br;
  br.init(chunk + kRaw + kLanes, lane_stream_start(chunk, kRaw, lane));
  uint32_t xn[B];
#pragma unroll
  for (int b = 0; b < B; ++b) xn[b] = load_x_pair(x + (int64_t)b * cols, cols, col0 + 2 * lane);
  constexpr int kGroupUnroll = B <= 4 ? 2 : 1;
#pragma unroll kGroupUnroll
  for (int g = 0; g < CP; ++g) {
    const uint4 rv = lds128(chunk + g * 512 + lane * 16);
    uint32_t xg[B];
#pragma unroll
    for (int b = 0; b < B; ++b) xg[b] = xn[b];
    if (g + 1 < CP) {
#pragma unroll
      for (int b = 0; b < B; ++b)
        xn[b] = load_x_pair(x + (int64_t)b * cols, cols, col0 + (g + 1) * 64 + 2 * lane);
    }
#pragma unroll
    for (int r = 0; r < 8; ++r) {
      const uint32_t e = decode_pair<FAST>(br, table);
      const uint32_t w = assemble(raw_pair_r(rv, r), e);
#pragma unroll
      for (int b = 0; b < B; ++b) {
        acc[r][b] = fma_bf16<false>(w, xg[b], acc[r][b]);
        acc[r][b] = fma_bf16<true>(w, xg[b], acc[r][b]);
      }
      if (r & 1) br.refill();
    }
  }
}

// Tile range of this CTA.
__device__ __forceinline__ void cta_range(const TileParams& p, int64_t* first, int* n) {
  const int64_t a = p.n_tiles * (int64_t)blockIdx.x / gridDim.x;
  const int64_t b = p.n_tiles * (int64_t)(blockIdx.x + 1) / gridDim.x;
  *first = a;
  *n = (int)(b - a);
}

// Sets up barriers; returns false for the producer warp (warp NC; its work is
// done) and for consumers when the decode table never arrived.
template <int NC>
__device__ __forceinline__ bool setup(const TileParams& p, uint8_t* smem, const Smem& s) {
  if (threadIdx.x == 0) {
    mbar_init(s.table_bar, 1);
    for (int k = 0; k < kSlots; ++k) {
      mbar_init(&s.full[k], 1);
      mbar_init(&s.empty[k], (uint32_t)p.batch_tiles);
    }
  }
  fence_barrier_init();
  __syncthreads();
  const int warp = threadIdx.x >> 5;
  if (warp == NC) {
    const uint32_t b0 = __ldg(p.sched_cta + blockIdx.x), b1 = __ldg(p.sched_cta + blockIdx.x + 1);
    produce(p, smem, s, p.sched_batch + b0, (int)(b1 - b0), threadIdx.x & 31);
    return false;
  }
  return __all_sync(kFull, wait_bounded(s.table_bar, 0));
}

// Row block i and column block j of tile u = first + q, stepped by NC tiles.
struct TilePos {
  uint32_t i, j, tiles_r;
  __device__ __forceinline__ void init(int64_t u, uint32_t tr) {
    tiles_r = tr;
    i = (uint32_t)(u % tr);
    j = (uint32_t)(u / tr);
  }
  __device__ __forceinline__ void step(uint32_t by) {
    i += by;
    while (i >= tiles_r) {
      i -= tiles_r;
      ++j;
    }
  }
};

template <int NC, int CP, int B, bool FAST>
__global__ void __launch_bounds__((NC + 1) * 32, 1) gemv_kernel(TileParams p) {
  extern __shared__ __align__(128) uint8_t smem[];
  const Smem s = carve(smem, p);
  int64_t first;
  int n;
  cta_range(p, &first, &n);
  if (!setup<NC>(p, smem, s)) return;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t table = smem_u32(smem);
  const uint32_t ring = smem_u32(s.ring);
  const int64_t cols = p.cols;
  const uint32_t* tile_ring = p.tile_ring + first;
  uint32_t at_next = warp < n ? __ldg(tile_ring + warp) : 0u;
  TilePos pos;
  pos.init(first + warp, (uint32_t)p.tiles_r);
  for (int q = warp; q < n; q += NC, pos.step(NC)) {
    const int k = q / p.batch_tiles;
    const uint32_t chunk = ring + at_next;
    if (q + NC < n) at_next = __ldg(tile_ring + q + NC);  // next tile's ring offset, early
    if (!wait_batch(s, k)) return;
    const int64_t i = pos.i, j = pos.j;
    float acc[8][B];
#pragma unroll
    for (int r = 0; r < 8; ++r)
#pragma unroll
      for (int b = 0; b < B; ++b) acc[r][b] = 0.f;
    decode_gemv_tile<CP, B, FAST>(chunk, table, lane, acc, p.x, cols, j * (CP * 64));
    __syncwarp();
    if (lane == 0) mbar_arrive(&s.empty[k % kSlots]);  // release the tile's share of the batch

    // Row sums of this tile: lane L holds row L >> 2 for every batch row.
    float tot[B];
#pragma unroll
    for (int b = 0; b < B; ++b) {
      float v[8];
#pragma unroll
      for (int r = 0; r < 8; ++r) v[r] = acc[r][b];
      tot[b] = reduce_rows8(v, lane);
    }
    const int64_t row = i * 8 + (lane >> 2);
    if ((lane & 3) == 0) {
      if (p.tiles_c == 1) {
        if (row < p.rows)
#pragma unroll
          for (int b = 0; b < B; ++b) p.y[(int64_t)b * p.rows + row] = tot[b];
      } else {
#pragma unroll
        for (int b = 0; b < B; ++b)
          __stcg(&p.partial[((int64_t)j * B + b) * p.rows_pad + row], tot[b]);
      }
    }
  }
  if (p.tiles_c == 1) return;
  // Split-K, once per warp after all its tiles: publish (fence, then count the
  // arrivals of all the warp's tiles at once); the last of a row block's
  // tiles_c arrivals sums its partials in column-block order and writes y.
  __threadfence();
  __syncwarp();
  for (int q0 = warp; q0 < n; q0 += 32 * NC) {
    const int q = q0 + lane * NC;
    uint32_t last = 0;
    if (q < n) {
      const uint32_t i = (uint32_t)(first + q) % (uint32_t)p.tiles_r;
      last = atomicAdd(&p.counters[i], 1u) == (uint32_t)(p.tiles_c - 1);
    }
    uint32_t mask = __ballot_sync(kFull, last);
    if (mask) __threadfence();
    while (mask) {
      const int src = __ffs(mask) - 1;
      mask &= mask - 1;
      const int64_t i = (uint32_t)(first + q0 + src * NC) % (uint32_t)p.tiles_r;
      for (int qq = lane; qq < 8 * B; qq += 32) {
        const int b = qq >> 3, rr = qq & 7;
        const int64_t orow = i * 8 + rr;
        const float* part = p.partial + (int64_t)b * p.rows_pad + orow;
        const int64_t stride = (int64_t)B * p.rows_pad;
        float sum = 0.f;
        int64_t jj = 0;
        for (; jj + 8 <= p.tiles_c; jj += 8) {
          float v[8];
#pragma unroll
          for (int k = 0; k < 8; ++k) v[k] = __ldcg(part + (jj + k) * stride);
#pragma unroll
          for (int k = 0; k < 8; ++k) sum += v[k];
        }
        for (; jj < p.tiles_c; ++jj) sum += __ldcg(part + jj * stride);
        if (orow < p.rows) p.y[(int64_t)b * p.rows + orow] = sum;
      }
      if (lane == 0) p.counters[i] = 0u;
    }
  }
}

template <int NC, int CP, bool FAST>
__global__ void __launch_bounds__((NC + 1) * 32, 1) decompress_kernel(TileParams p) {
  extern __shared__ __align__(128) uint8_t smem[];
  const Smem s = carve(smem, p);
  int64_t first;
  int n;
  cta_range(p, &first, &n);
  if (!setup<NC>(p, smem, s)) return;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t table = smem_u32(smem);
  const uint32_t ring = smem_u32(s.ring);
  const int64_t cols = p.cols;
  const bool even_cols = (cols & 1) == 0;
  constexpr int kRaw = CP * 512;
  uint32_t invalid = 0;
  const uint32_t* tile_ring = p.tile_ring + first;
  uint32_t at_next = warp < n ? __ldg(tile_ring + warp) : 0u;
  TilePos pos;
  pos.init(first + warp, (uint32_t)p.tiles_r);
  for (int q = warp; q < n; q += NC, pos.step(NC)) {
    const int k = q / p.batch_tiles;
    const uint32_t chunk = ring + at_next;
    if (q + NC < n) at_next = __ldg(tile_ring + q + NC);
    if (!wait_batch(s, k)) return;
    const int64_t i = pos.i, j = pos.j;
    BitReader br;
    br.init(chunk + kRaw + kLanes, lane_stream_start(chunk, kRaw, lane));
    const bool full_tile = (i + 1) * 8 <= p.rows && (j + 1) * (CP * 64) <= cols && even_cols;
#pragma unroll 1
    for (int g = 0; g < CP; ++g) {
      const uint4 rv = lds128(chunk + g * 512 + lane * 16);
      const int64_t col = j * (CP * 64) + g * 64 + 2 * lane;
#pragma unroll
      for (int r = 0; r < 8; ++r) {
        const uint32_t e = decode_pair<FAST>(br, table);
        invalid |= e;
        const uint32_t w = assemble(raw_pair_r(rv, r), e);
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
    __syncwarp();
    if (lane == 0) mbar_arrive(&s.empty[k % kSlots]);  // release the tile's share of the batch
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

// Consumer warps per CTA: more warps hide the decoder's dependency chains, as
// long as the batch's accumulators leave registers for them.
// A CTA with W warps puts up to ceil(W / 4) on one SM sub-partition, whose
// register file holds 16K registers: 25 warps leave 72 per thread, 17 leave 96,
// 13 leave 128.
template <int B>
constexpr int consumers_for() { return B <= 2 ? 24 : (B <= 4 ? 16 : 12); }

template <int CP, int B, bool FAST>
cudaError_t launch_gemv_t(const TileParams& p, const LaunchShape& s, cudaStream_t stream) {
  constexpr int NC = consumers_for<B>();
  static_assert(NC <= kMaxConsumers, "the launch schedule assumes at most kMaxConsumers");
  static int configured[64] = {};
  cudaError_t e = ensure_smem(gemv_kernel<NC, CP, B, FAST>, s.smem_bytes, configured);
  if (e != cudaSuccess) return e;
  gemv_kernel<NC, CP, B, FAST><<<s.ctas, (NC + 1) * 32, s.smem_bytes, stream>>>(p);
  return cudaGetLastError();
}

template <int CP, bool FAST>
cudaError_t launch_gemv_cp(const TileParams& p, const LaunchShape& s, cudaStream_t stream) {
  switch (p.batch) {
    case 1: return launch_gemv_t<CP, 1, FAST>(p, s, stream);
    case 2: return launch_gemv_t<CP, 2, FAST>(p, s, stream);
    case 3: return launch_gemv_t<CP, 3, FAST>(p, s, stream);
    case 4: return launch_gemv_t<CP, 4, FAST>(p, s, stream);
    case 5: return launch_gemv_t<CP, 5, FAST>(p, s, stream);
    case 6: return launch_gemv_t<CP, 6, FAST>(p, s, stream);
    case 7: return launch_gemv_t<CP, 7, FAST>(p, s, stream);
    case 8: return launch_gemv_t<CP, 8, FAST>(p, s, stream);
    default: return cudaErrorInvalidValue;
  }
}

template <int CP, bool FAST>
cudaError_t launch_decompress_t(const TileParams& p, const LaunchShape& s, cudaStream_t stream) {
  constexpr int NC = 24;
  static_assert(NC <= kMaxConsumers, "the launch schedule assumes at most kMaxConsumers");
  static int configured[64] = {};
  cudaError_t e = ensure_smem(decompress_kernel<NC, CP, FAST>, s.smem_bytes, configured);
  if (e != cudaSuccess) return e;
  decompress_kernel<NC, CP, FAST><<<s.ctas, (NC + 1) * 32, s.smem_bytes, stream>>>(p);
  return cudaGetLastError();
}

}  // namespace

LaunchShape launch_shape(int64_t n_tiles, uint64_t max_chunk, uint64_t typical_chunk,
                         uint32_t table_bytes, int sm_count, size_t smem_limit) {
  LaunchShape s;
  int64_t ctas = n_tiles < sm_count ? n_tiles : sm_count;
  if (ctas > (int64_t)kMaxCtas) ctas = kMaxCtas;
  s.ctas = ctas < 1 ? 1 : (int)ctas;
  s.table_bytes = table_bytes;
  // table | table barrier | full[kSlots] | empty[kSlots] | ring
  const size_t head = (size_t)table_bytes + 8 + 2 * kSlots * 8;
  s.ring_offset = (head + 127) / 128 * 128;
  const int64_t per_cta = (n_tiles + s.ctas - 1) / s.ctas;
  // Tiles per bulk copy: enough for >= 16 KB of typical chunks, between 2 and 8
  // (at least 2 keeps the schedule's batch count within its area).
  int t = (int)((16384 + typical_chunk - 1) / (typical_chunk ? typical_chunk : 1));
  if (t < 2) t = 2;
  if (t > 8) t = 8;
  s.batch_tiles = t;
  // As much ring as the device allows, but no more than the CTA's tiles need;
  // a batch of worst-case chunks must fit.
  size_t ring = smem_limit > s.ring_offset + kRingSlack + max_chunk
                    ? smem_limit - s.ring_offset - kRingSlack
                    : 0;
  const size_t batch_max = (size_t)s.batch_tiles * (size_t)max_chunk;
  const size_t need = (size_t)per_cta * (size_t)max_chunk;
  if (ring > need) ring = need;
  ring = ring / 16 * 16;
  if (ring < batch_max) ring = (batch_max + 15) / 16 * 16;
  s.ring_bytes = (int)ring;
  s.smem_bytes = s.ring_offset + ring + kRingSlack;
  return s;
}

cudaError_t launch_gemv(const TileParams& p, int tile_cols, bool fast, const LaunchShape& s,
                        cudaStream_t stream) {
  switch (tile_cols) {
    case 512: return fast ? launch_gemv_cp<8, true>(p, s, stream) : launch_gemv_cp<8, false>(p, s, stream);
    case 256: return fast ? launch_gemv_cp<4, true>(p, s, stream) : launch_gemv_cp<4, false>(p, s, stream);
    case 128: return fast ? launch_gemv_cp<2, true>(p, s, stream) : launch_gemv_cp<2, false>(p, s, stream);
    case 64: return fast ? launch_gemv_cp<1, true>(p, s, stream) : launch_gemv_cp<1, false>(p, s, stream);
    default: return cudaErrorInvalidValue;
  }
}

cudaError_t launch_decompress(const TileParams& p, int tile_cols, bool fast,
                              const LaunchShape& s, cudaStream_t stream) {
  switch (tile_cols) {
    case 512: return fast ? launch_decompress_t<8, true>(p, s, stream) : launch_decompress_t<8, false>(p, s, stream);
    case 256: return fast ? launch_decompress_t<4, true>(p, s, stream) : launch_decompress_t<4, false>(p, s, stream);
    case 128: return fast ? launch_decompress_t<2, true>(p, s, stream) : launch_decompress_t<2, false>(p, s, stream);
    case 64: return fast ? launch_decompress_t<1, true>(p, s, stream) : launch_decompress_t<1, false>(p, s, stream);
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
