// kernels.cu — sm_100a kernels: fused decode-GEMV, bit-exact decompress and
// row gather.
//
// What runs where ("NWC — Neural Weight Compression", "How it works > Fused
// kernel"; "Unweight", "Direct GPU Decompression"):
//   * One persistent CTA per SM owns a contiguous range of tiles (8 rows x
//     tile_cols), in the blob's column-block-major order.
//   * A producer warp follows the launch schedule the host wrote into the
//     device image: per batch of consecutive tiles it waits for the releases
//     the schedule names and issues one cp.async.bulk (no multicast) into a
//     CTA-wide shared-memory ring.  Each batch has a "full" mbarrier (bytes
//     counted) and an "empty" one that its tiles' consumers arrive at.  Every
//     wait is bounded: a wait that gives up sets the device error word, and the
//     producer waits for its copies before leaving.
//   * 31 consumer warps take the CTA's tiles round-robin.  Each lane decodes
//     its own bit stream.  With lmax <= 7 the peek is 14 bits and every table
//     entry holds two complete codes ("NWC", "Prefix code instead of rANS"), so
//     two steps take one 32-bit window, two lookups and a predicated word
//     rotation; lmax 8..12 uses a 12-bit peek with a second lookup for a pair
//     that does not fit.
//   * BF16x2 reassembly is one byte permute of the raw plane and one bitwise
//     select with the table entry; the weights never leave registers.
//   * GEMV: lane 4g + c owns row g of a tile, so two decoded pairs are the B
//     operand of one m16n8k16 tensor-core step whose A operand is x (staged in
//     shared memory); FP32 accumulation, then a split-K reduction in a fixed
//     order through the workspace (the last of a row block's column tiles to
//     finish sums the partials).  Launches use programmatic dependent launch.
//   * Decompress: the same decode, two 16-byte stores per lane and group.
//   * Row gather: the four lanes owning a requested row decode it from L1.
#include <cuda_runtime.h>

#include <cstdint>
#include <type_traits>

#include "kernels.cuh"
#include "nwc_format.h"

namespace nwc {

namespace {

constexpr int kRingSlack = 512;                  // readers may run past a chunk (corrupt data)
constexpr int kTablePieces = 8;                  // bulk copies that bring in the decode table
static_assert(kTablePieces <= 32, "one table piece per producer lane");
constexpr int kMaxPairSteps = 32;                // two-step reads per tile (8 groups x 4)
constexpr uint32_t kPairReadSpan = 12 + 4 * kMaxPairSteps + 4;  // bytes one tile's reader may touch
static_assert(kPairReadSpan <= kRingSlack, "a clamped reader must stay inside the ring slack");
// The rank reader advances at most one word per pair (64 pairs per tile).
constexpr uint32_t kRankReadSpan = 12 + 4 * 2 * kMaxPairSteps + 4;
static_assert(kRankReadSpan <= kRingSlack, "a clamped rank reader must stay inside the slack");
constexpr uint64_t kBatchTarget = 12288;          // bytes a bulk copy should move at least
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
// Hint: bring `bytes` (a multiple of 16) of global memory into L2.
__device__ __forceinline__ void bulk_prefetch_l2(const void* src, uint32_t bytes) {
  asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(src), "r"(bytes) : "memory");
}
__device__ __forceinline__ void fence_barrier_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}
// Where a bounded wait reports giving up, and after how many polls.
struct WaitCtl {
  uint32_t* err;
  uint32_t limit;
};
__device__ __forceinline__ WaitCtl wait_ctl(const TileParams& p) {
  return WaitCtl{p.err, p.wait_limit ? p.wait_limit : kDefaultWaitLimit};
}
// Waits for a CTA's own copies and MMAs in flight before it leaves: never
// shorter than the default, whatever limit a test set, so that no CTA exits
// while a copy into its shared memory is still running.
__device__ __forceinline__ WaitCtl drain_ctl(const TileParams& p) {
  return WaitCtl{p.err, p.wait_limit > kDefaultWaitLimit ? p.wait_limit : kDefaultWaitLimit};
}
__device__ __forceinline__ WaitCtl drain_ctl_default(uint32_t* err) {
  return WaitCtl{err, kDefaultWaitLimit};
}
// Polls `bar` for `parity` at most w.limit times; on failure records a
// timeout in the handle's error word.
__device__ bool wait_bounded(uint64_t* bar, uint32_t parity, const WaitCtl& w) {
  for (uint32_t it = 0; it < w.limit; ++it)
    if (mbar_try_wait(bar, parity)) return true;
  atomicOr(w.err, kErrTimeout);
  return false;
}

__device__ __forceinline__ uint32_t lds32(uint32_t addr) {
  uint32_t v;
  asm volatile("ld.shared.u32 %0, [%1];" : "=r"(v) : "r"(addr));
  return v;
}
__device__ __forceinline__ uint2 lds64(uint32_t addr) {
  uint2 v;
  asm volatile("ld.shared.v2.u32 {%0, %1}, [%2];" : "=r"(v.x), "=r"(v.y) : "r"(addr));
  return v;
}
// Programmatic dependent launch: let the next kernel on the stream start its
// prologue now (its CTAs become resident as this grid's CTAs exit), and wait until
// the previous kernel has completed and its writes are visible.
__device__ __forceinline__ void allow_dependents() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}
__device__ __forceinline__ void wait_prerequisites() {
  asm volatile("griddepcontrol.wait;" ::: "memory");
}
__device__ __forceinline__ void named_barrier_sync(int id, int threads) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(threads) : "memory");
}
__device__ __forceinline__ uint4 lds128(uint32_t addr) {
  uint4 v;
  asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "r"(addr));
  return v;
}
// v = [addr] when `need` is non-zero, else v is left as it was (predicated
// load, no branch).
__device__ __forceinline__ void lds32_keep(uint32_t& v, uint32_t addr, uint32_t need) {
  asm volatile("{\n\t.reg .pred p;\n\tsetp.ne.u32 p, %2, 0;\n\t@p ld.shared.u32 %0, [%1];\n\t}"
               : "+r"(v)
               : "r"(addr), "r"(need));
}
// Low word of ({hi, lo} >> (n mod 32)).
__device__ __forceinline__ uint32_t shr_wrap(uint32_t lo, uint32_t hi, uint32_t n) {
  uint32_t r;
  asm("shf.r.wrap.b32 %0, %1, %2, %3;" : "=r"(r) : "r"(lo), "r"(hi), "r"(n));
  return r;
}
// D += A B on the tensor cores, one warp: A is 16 x 16 BF16 (row-major
// fragment a0..a3), B is 16 x 8 BF16 (column-major fragment b0, b1), D is
// 16 x 8 FP32 (d0..d3).  Fragment of lane L (g = L / 4, c = L % 4):
//   a0 = A[g][2c, 2c+1]   a1 = A[g+8][2c, 2c+1]   a2 = A[g][2c+8, 2c+9]   a3 = A[g+8][2c+8, 2c+9]
//   b0 = B[2c, 2c+1][g]   b1 = B[2c+8, 2c+9][g]
//   d0 = D[g][2c]   d1 = D[g][2c+1]   d2 = D[g+8][2c]   d3 = D[g+8][2c+1]
// (the lower 16 bits of a register hold the first of its two elements).
__device__ __forceinline__ void mma_bf16_16816(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                               uint32_t a3, uint32_t b0, uint32_t b1) {
  asm("mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, "
      "{%8, %9}, {%0, %1, %2, %3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// ---- bit reader --------------------------------------------------------------

// Per-lane reader of the lane's stream in shared memory, used with the 12-bit
// peek (lmax 8..12): a 64-bit window hi:lo (next bit = bit 31 of hi) and a
// valid-bit count.  A refill point leaves at least 32 valid bits; a lookup
// consumes at most 12, and a pair that does not fit refills before its second
// lookup, so every lookup has its 12 peek bits.  The low 7 bits of `nbacc`
// count valid bits; subtracting whole table entries keeps them exact, since
// entry bits 4..6 are zero and bits 0..3 hold the consumed count.
struct BitReader {
  uint32_t hi, lo, nbacc;
  uint32_t nw;  // the stream word after the window, loaded ahead
  uint32_t wp;  // shared-window address of the word after nw

  uint32_t last;  // highest word address the reader may touch

  // `limit`: end of the shared memory the reader may read (see PairReader).
  __device__ __forceinline__ void init(uint32_t area, uint32_t start, uint32_t limit) {
    last = limit - 4;
    wp = min(area + (start & ~3u), last - 8);
    const uint32_t sh = (start & 3u) * 8u;
    const uint32_t w0 = lds32(wp), w1 = lds32(wp + 4);
    nw = lds32(wp + 8);
    hi = __funnelshift_l(w1, w0, sh);
    lo = w1 << sh;
    nbacc = 64u - sh;
    wp += 12;
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
  // bits; the count becomes count | 32 either way.  No branch: an empty word
  // shifts in nothing, and the word after it is fetched (predicated) only
  // when this one was used, so the shared-memory load is off the decoder's
  // dependency chain.
  __device__ __forceinline__ void refill() {
    const uint32_t need = (~nbacc) & 32u;
    const uint32_t w = need ? nw : 0u;
    hi |= shr_wrap(w, 0u, nbacc);
    lo |= shr_wrap(0u, w, nbacc);
    nbacc |= 32u;
    lds32_keep(nw, wp, need);
    wp = min(wp + (need >> 3), last);
  }
};

// One step: a table entry holding two exponent bytes at their BF16 positions
// (bits 7..14 and 23..30).  FAST: 14-bit peek, both codes always fit (the
// kernels read that case with PairReader below); else 12-bit peek with a second
// lookup for a pair that does not fit.
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

// Reader for the 14-bit peek (lmax <= 7), two steps at a time: two steps
// consume at most 28 bits, so one 32-bit window taken before them holds both
// peeks.  The stream is kept as three consecutive words a, b, c with bits 0..4
// of p the offset of the next unread bit in a; after two steps the words move
// on by one when the offset passed 32, and the word after c is fetched
// (predicated) at once, two steps before it can be needed, so no shared-memory
// load of the stream lies on the decoder's dependency chain.
struct PairReader {
  uint32_t a, b, c;  // stream words base, base + 1, base + 2
  uint32_t p;        // bits 0..4: next unread bit of a (0 = its bit 31); higher
                     // bits are don't-care
  uint32_t next;     // shared-window address of word base + 3

  // A tile takes at most kMaxPairSteps calls of two(), each reading at most one
  // word past the three it starts with, so the reader never touches more than
  // kPairReadSpan bytes from its first word; `limit` (the end of the memory it
  // may read) clamps that first word, so a corrupt stream start or length can
  // misdecode but never read outside.
  __device__ __forceinline__ void init(uint32_t area, uint32_t start, uint32_t limit) {
    const uint32_t at = min(area + (start & ~3u), limit - kPairReadSpan);
    a = lds32(at);
    b = lds32(at + 4);
    c = lds32(at + 8);
    next = at + 12;
    p = (start & 3u) * 8u;
  }
  // Entries e0, e1 of the next two steps.
  __device__ __forceinline__ void two(uint32_t table, uint32_t& e0, uint32_t& e1) {
    const uint32_t w = __funnelshift_l(b, a, p);  // 32 bits from the next unread one (p & 31)
    e0 = lds32(table + ((w >> 18) << 2));
    const uint32_t w1 = __funnelshift_l(0u, w, e0);  // shift by e0's count (bits 0..3)
    e1 = lds32(table + ((w1 >> 18) << 2));
    // Bits 0..6 of an entry are its count (bits 4..6 zero) and higher bits never
    // carry into them, so bits 0..4 of p + e0 + e1 are the new offset; the two
    // counts add less than 32, so the window passed a word exactly when bit 5
    // flipped.
    const uint32_t q = p + e0 + e1;
    const uint32_t adv = (q ^ p) & 32u;
    p = q;
    advance(adv);
  }
  // When adv is non-zero: a, b, c move on by one word and the word after them
  // is fetched.  One predicate covers the moves, the load and the address.
  __device__ __forceinline__ void advance(uint32_t adv) {
    asm volatile(
        "{\n\t.reg .pred q;\n\tsetp.ne.u32 q, %4, 0;\n\t"
        "@q mov.b32 %0, %1;\n\t@q mov.b32 %1, %2;\n\t"
        "@q ld.shared.u32 %2, [%3];\n\t@q add.u32 %3, %3, 4;\n\t}"
        : "+r"(a), "+r"(b), "+r"(c), "+r"(next)
        : "r"(adv));
  }
};

// Reader of the ranked unary code (variant NWR1; "NWC", "How it works > Prefix
// code instead of rANS", format v9): a weight's code is its sign bit, then r
// zeros and a one for rank r < R, else R zeros and the 7-bit field e (exponent
// bits 14..8).  A code has at most 1 + R + 7 <= 15 bits, so one 32-bit window
// always holds a pair of codes; the words move as in PairReader, one step
// (pair) at a time.  No table: the R ranked values sit in two registers and a
// rank picks its byte with one byte permute.  A step's entry carries the two
// weights' high bytes (sign and e) at bits 8..15 and 24..31.
struct RankReader {
  uint32_t a, b, c, p, next;
  uint32_t rank_lo, rank_hi, R;

  __device__ __forceinline__ void init(uint32_t area, uint32_t start, uint32_t limit,
                                       uint32_t table) {
    const uint32_t at = min(area + (start & ~3u), limit - kRankReadSpan);
    a = lds32(at);
    b = lds32(at + 4);
    c = lds32(at + 8);
    next = at + 12;
    p = (start & 3u) * 8u;
    rank_lo = lds32(table);
    rank_hi = lds32(table + 4);
    R = lds32(table + 8);
  }
  // High byte (sign << 7 | e) of the code at the top of t, and its length.
  __device__ __forceinline__ uint32_t code(uint32_t t, uint32_t& len) const {
    const uint32_t u = t << 1;
    const uint32_t z = __clz(u);  // zeros after the sign bit (32 when none is one)
    const bool ranked = z < R;
    const uint32_t e = ranked ? (__byte_perm(rank_lo, rank_hi, z) & 0xFFu) : ((u << R) >> 25);
    len = ranked ? z + 2u : R + 8u;
    return ((t >> 31) << 7) | e;
  }
  __device__ __forceinline__ uint32_t step() {
    const uint32_t w = __funnelshift_l(b, a, p);
    uint32_t l0, l1;
    const uint32_t h0 = code(w, l0);
    const uint32_t h1 = code(w << l0, l1);
    // The pair took at most 30 bits: a word was passed exactly when bit 5 of
    // the offset flipped.
    const uint32_t q = p + l0 + l1;
    const uint32_t adv = (q ^ p) & 32u;
    p = q;
    asm volatile(
        "{\n\t.reg .pred q;\n\tsetp.ne.u32 q, %4, 0;\n\t"
        "@q mov.b32 %0, %1;\n\t@q mov.b32 %1, %2;\n\t"
        "@q ld.shared.u32 %2, [%3];\n\t@q add.u32 %3, %3, 4;\n\t}"
        : "+r"(a), "+r"(b), "+r"(c), "+r"(next)
        : "r"(adv));
    return (h0 << 8) | (h1 << 24);
  }
};

// The readers behind one interface: two() yields the entries of the next two
// steps.  kCode14 uses the window reader, kCode12 the bit buffer (whose second
// lookup handles a pair that does not fit in the 12-bit peek), kCodeRank the
// rank reader.
template <int CODE>
struct StreamDecoder;
template <>
struct StreamDecoder<kCode14> {
  PairReader r;
  __device__ __forceinline__ void init(uint32_t area, uint32_t start, uint32_t limit,
                                       uint32_t) {
    r.init(area, start, limit);
  }
  __device__ __forceinline__ void two(uint32_t table, uint32_t& e0, uint32_t& e1) {
    r.two(table, e0, e1);
  }
};
template <>
struct StreamDecoder<kCode12> {
  BitReader br;
  __device__ __forceinline__ void init(uint32_t area, uint32_t start, uint32_t limit,
                                       uint32_t) {
    br.init(area, start, limit);
  }
  __device__ __forceinline__ void two(uint32_t table, uint32_t& e0, uint32_t& e1) {
    e0 = decode_pair<false>(br, table);
    e1 = decode_pair<false>(br, table);
    br.refill();
  }
};
// NWE1 codes its kept exponents exactly as the 14-bit prefix code.
template <>
struct StreamDecoder<kCodeEsc> : StreamDecoder<kCode14> {};
template <>
struct StreamDecoder<kCodeRank> {
  RankReader r;
  __device__ __forceinline__ void init(uint32_t area, uint32_t start, uint32_t limit,
                                       uint32_t table) {
    r.init(area, start, limit, table);
  }
  __device__ __forceinline__ void two(uint32_t, uint32_t& e0, uint32_t& e1) {
    e0 = r.step();
    e1 = r.step();
  }
};

// Raw bytes of the lane's step r in a 64-column group (its symbols 2r and
// 2r + 1, bytes 2r and 2r + 1 of the group's 16) duplicated into both bytes of
// each half: [b1, b1, b0, b0] from high to low.
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

template <int CODE>
__device__ __forceinline__ uint32_t assemble(uint32_t rawdup, uint32_t e) {
  if constexpr (CODE == kCodeRank) {
    // The raw bytes are the low bytes (exponent bit 7 and the fraction); the
    // entry holds the high bytes (sign and exponent bits 14..8).
    return (rawdup & 0x00FF00FFu) | e;
  } else {
    // Sign+fraction from the raw bytes, exponents from the table entry.
    return (rawdup & kEntryRawMask) | (e & kEntryExponentMask);
  }
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

// Stream starts of lane `lane` with S bit streams per lane (S = 2: the lengths
// of streams 2t and 2t + 1 are bytes 2t and 2t + 1 of the length array).
template <int S>
__device__ __forceinline__ void lane_stream_starts(uint32_t chunk, int raw, int lane,
                                                   uint32_t (&start)[S]) {
  if constexpr (S == 1) {
    start[0] = lane_stream_start(chunk, raw, lane);
  } else {
    const uint32_t w = lds32(chunk + raw + ((2 * lane) & ~3));
    const uint32_t b = w >> (8 * ((2 * lane) & 3));
    const uint32_t len0 = b & 0xFFu, len1 = (b >> 8) & 0xFFu;
    const uint32_t mine = len0 + len1;
    uint32_t incl = mine;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t v = __shfl_up_sync(kFull, incl, o);
      if (lane >= o) incl += v;
    }
    start[0] = incl - mine;
    start[1] = start[0] + len0;
  }
}

// Verbatim runs of an NWE1 tile ("Unweight", "Compressing BF16 Weights": a
// run of 64 weights of a row holding a rare exponent is stored whole, so the
// decoder branches once per run).  After the raw plane a chunk holds flags
// u8[16] (bit m of byte g: run (row g, group m) is verbatim), the runs'
// exponent bytes (64 each, in (g, m) order), then the lane lengths and
// streams.  Lane 4 g + c reads bytes 16 c .. 16 c + 15 of its row's runs.
struct EscRuns {
  uint32_t mine;  // bit m: this lane's 16 symbols of group m are verbatim;
                  // bit 31: the flag field is corrupt
  uint32_t at;    // shared-memory address of its bytes in its next such run
};
constexpr uint32_t kEscCorrupt = 1u << 31;
// flags: shared-memory address of the flag field of a tile of CP groups;
// limit: end of the readable buffer.  Returns the offset of the lane lengths
// from the flags.  A flag field that names a group past the tile, or more
// runs than the buffer holds, is corrupt: the lane then decodes its streams
// from just after the flags (a wrong result, but every read stays inside the
// buffer, which holds at least the flags and the lane lengths).
template <int CP>
__device__ __forceinline__ uint32_t esc_runs(uint32_t flags, uint32_t limit, int lane,
                                             EscRuns& er) {
  const uint2 f = lds64(flags);
  const int g = lane >> 2;
  const uint32_t lo = g < 4 ? f.x : f.y;
  const int sh = 8 * (g & 3);
  const uint32_t before =
      __popc(lo & ((1u << sh) - 1u)) + (g < 4 ? 0u : (uint32_t)__popc(f.x));
  const uint32_t lens = kEscFlagBytes + kEscRunBytes * (uint32_t)(__popc(f.x) + __popc(f.y));
  constexpr uint32_t kValid = 0x01010101u * ((1u << CP) - 1u);
  if (((f.x | f.y) & ~kValid) != 0u || flags + lens + kLanes > limit) {
    er.mine = kEscCorrupt;
    er.at = flags;
    return kEscFlagBytes;
  }
  er.mine = (lo >> sh) & 0xFFu;
  er.at = flags + kEscFlagBytes + kEscRunBytes * before + 16u * (uint32_t)(lane & 3);
  return lens;
}
// Table-entry form (exponent bytes at their BF16 positions, nothing else) of
// pairs 4 q .. 4 q + 3 of a lane's 16 verbatim exponent bytes.
__device__ __forceinline__ void esc_quad(const uint4& ev, int q, uint32_t (&e)[4]) {
  const uint32_t a = q == 0 ? ev.x : ev.z, b = q == 0 ? ev.y : ev.w;
  e[0] = __byte_perm(a, 0u, 0x4140u) << 7;
  e[1] = __byte_perm(a, 0u, 0x4342u) << 7;
  e[2] = __byte_perm(b, 0u, 0x4140u) << 7;
  e[3] = __byte_perm(b, 0u, 0x4342u) << 7;
}

// A lane's decoder over its S bit streams: quad() yields the table entries of
// the lane's next four symbol pairs in order.  With S = 2 the pairs alternate
// between the streams, so the two streams' dependency chains interleave.
template <int CODE, int S>
struct LaneDecoder;
template <int CODE>
struct LaneDecoder<CODE, 1> {
  StreamDecoder<CODE> d;
  __device__ __forceinline__ void init(uint32_t area, const uint32_t (&start)[1], uint32_t limit,
                                       uint32_t table) {
    d.init(area, start[0], limit, table);
  }
  __device__ __forceinline__ void quad(uint32_t table, uint32_t (&e)[4]) {
    d.two(table, e[0], e[1]);
    d.two(table, e[2], e[3]);
  }
};
template <int CODE>
struct LaneDecoder<CODE, 2> {
  StreamDecoder<CODE> d0, d1;
  __device__ __forceinline__ void init(uint32_t area, const uint32_t (&start)[2], uint32_t limit,
                                       uint32_t table) {
    d0.init(area, start[0], limit, table);
    d1.init(area, start[1], limit, table);
  }
  __device__ __forceinline__ void quad(uint32_t table, uint32_t (&e)[4]) {
    d0.two(table, e[0], e[2]);
    d1.two(table, e[1], e[3]);
  }
};

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
  uint8_t* xstage;   // p.xstage_bytes: the CTA's columns of x (GEMV)
  uint8_t* ring;
};

// table | table barrier | full[kSlots] | empty[kSlots] | x stage (16-byte
// aligned) | ring
__host__ __device__ constexpr size_t xstage_offset(uint32_t table_bytes) {
  return ((size_t)table_bytes + 8 + 2 * kSlots * 8 + 15) / 16 * 16;
}

__device__ __forceinline__ Smem carve(uint8_t* smem, const TileParams& p) {
  Smem s;
  s.table_bar = reinterpret_cast<uint64_t*>(smem + p.table_bytes);
  s.full = s.table_bar + 1;
  s.empty = s.full + kSlots;
  s.xstage = smem + xstage_offset(p.table_bytes);
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
                        int nb, int lane, volatile uint32_t* issued = nullptr,
                        uint32_t raw_prefetch = 0) {
  // The decode table in kTablePieces copies, one per lane, each CTA starting
  // at a different piece, so that the CTAs do not all ask the same L2 lines at
  // once.
  if (lane == 0) mbar_expect_tx(s.table_bar, p.table_bytes);
  __syncwarp();
  if (lane < kTablePieces) {
    const uint32_t piece = p.table_bytes / kTablePieces;
    const uint32_t off = ((blockIdx.x + lane) % kTablePieces) * piece;
    bulk_load(smem + off, reinterpret_cast<const uint8_t*>(p.table) + off, piece, s.table_bar);
  }
  // Lane l holds the descriptor of copy base + l (and the next window's in
  // dn).  Every copy from k on whose releases (`need`) lane 0 has already
  // observed goes out at once, one per lane; otherwise lane 0 waits for the
  // next release.  With raw_prefetch, each copy's tile also has the raw plane
  // before its streams (raw_prefetch bytes) prefetched into L2.
  const WaitCtl wc = wait_ctl(p);
  const uint4 none = make_uint4(0u, 0u, 0u, ~0u);
  uint4 d = lane < nb ? __ldg(desc + lane) : none;
  uint4 dn = 32 + lane < nb ? __ldg(desc + 32 + lane) : none;
  uint32_t released = 0;  // batches whose release lane 0 has observed
  int k = 0, base = 0;
  uint32_t ok = 1;
  while (k < nb) {
    if (k >= base + 32) {
      base += 32;
      d = dn;
      dn = base + 32 + lane < nb ? __ldg(desc + base + 32 + lane) : none;
    }
    const int off = k - base;
    const uint32_t seen = __shfl_sync(kFull, released, 0);
    const uint32_t ready =
        __ballot_sync(kFull, lane >= off && base + lane < nb && d.w <= seen) >> off;
    const int run = ready == (kFull >> off) ? 32 - off : __ffs(~ready) - 1;
    if (run == 0) {  // copy k waits for the releases it needs, in order
      const uint32_t need = __shfl_sync(kFull, d.w, off);
      if (lane == 0) {
        for (; released < need; ++released) {
          if (!wait_bounded(&s.empty[released % kSlots], (released / kSlots) & 1u, wc)) {
            ok = 0;
            break;
          }
        }
      }
      if (!__shfl_sync(kFull, ok, 0)) break;
      continue;
    }
    if (lane >= off && lane < off + run) {
      if (raw_prefetch) bulk_prefetch_l2(p.tiles + 16ull * d.x - raw_prefetch, raw_prefetch);
      uint64_t* bar = &s.full[(base + lane) % kSlots];
      mbar_expect_tx(bar, d.y);  // arrive (release) + byte count
      bulk_load(s.ring + d.z, p.tiles + 16ull * d.x, d.y, bar);
    }
    k += run;
    __syncwarp();
    if (lane == 0 && issued) *issued = (uint32_t)k;
  }
  // Leave no copy in flight: batches [0, k) were issued, and those more than
  // kSlots back have been released, hence landed.
  if (lane == 0) {
    const WaitCtl dc = drain_ctl(p);
    for (int j = k - 1; j >= 0 && j >= k - kSlots; --j)
      wait_bounded(&s.full[j % kSlots], (uint32_t)((j / kSlots) & 1), dc);
    wait_bounded(s.table_bar, 0, dc);
  }
}

// Consumer side: wait until batch k has landed.  The schedule keeps fewer than
// kSlots - ceil(kMaxLag / batch_tiles) batches outstanding, so by the time a
// consumer polls slot k % kSlots (its last released tile at most kMaxLag tiles
// back) the slot's previous batch k - kSlots was released long ago: the parity
// it polls is batch k's.
__device__ __forceinline__ bool wait_batch(const Smem& s, int k, const WaitCtl& wc) {
  return __all_sync(kFull, wait_bounded(&s.full[k % kSlots], (uint32_t)((k / kSlots) & 1), wc));
}

// Four BF16 values x[col .. col + 3] of one row of x as two words, zeros where
// the columns lie past `cols` (for an even cols a word is wholly inside or
// outside; an odd cols is read element by element).  Every lane loads from a
// valid address and selects afterwards, so lanes never diverge.  vec
// (uniform): 8-byte aligned and inside.
__device__ __forceinline__ uint32_t ldg_u16(const uint16_t* p) {
  return (uint32_t)__ldg(reinterpret_cast<const unsigned short*>(p));
}
// x[col] and x[col + 1] of a row as one word, zeros past `cols`, any
// alignment (rows of an odd number of columns start on 2-byte boundaries).
__device__ __forceinline__ uint32_t load_x2_any(const uint16_t* xrow, int64_t cols, int64_t col) {
  const uint32_t lo = col < cols ? ldg_u16(xrow + col) : 0u;
  const uint32_t hi = col + 1 < cols ? ldg_u16(xrow + col + 1) : 0u;
  return lo | (hi << 16);
}

__device__ __forceinline__ uint2 load_x4(const uint16_t* xrow, int64_t cols, int64_t col,
                                         bool vec) {
  uint2 v;
  if (vec) {
    v = __ldg(reinterpret_cast<const uint2*>(xrow + col));
  } else if (cols & 1) {
    v.x = load_x2_any(xrow, cols, col);
    v.y = load_x2_any(xrow, cols, col + 2);
  } else {
    const bool in0 = col < cols, in1 = col + 2 < cols;
    v.x = __ldg(reinterpret_cast<const uint32_t*>(xrow + (in0 ? col : 0)));
    v.y = __ldg(reinterpret_cast<const uint32_t*>(xrow + (in1 ? col + 2 : 0)));
    v.x = in0 ? v.x : 0u;
    v.y = in1 ? v.y : 0u;
  }
  return v;
}

// A whole tile (8 rows x 64 CP columns at column col_tile) on the tensor cores.
// Lane L = 4 g + c decodes row g, columns 64 m + 16 c .. + 15 of every group m.
// In 16-column block s of a group the lane supplies W[row g][16 c + 4 s + 0..1]
// and [.. + 2..3] as B = W^T (k x row), and x[batch g][the same columns] (and
// batch g + 8 when WIDE) as A (batch x k), so D[batch][row] accumulates x W^T;
// the k order inside a block is one column permutation for A and B alike, so
// the sum is unchanged.  On return d[0..1] hold y[batch g][rows 2c, 2c + 1] of
// the tile's contribution and d[2..3] the same for batch g + 8.  Each block's
// x is read one block ahead: from shared memory (XSM: xs = the staged row 0 at
// the tile's first column, rows xrow bytes apart) or else through L1.
template <int CP, bool WIDE, int CODE, int S, bool XSM>
__device__ __forceinline__ void decode_gemv_tile(uint32_t chunk, uint32_t table, uint32_t limit,
                                                 int lane, float (&d)[4], const TileParams& p,
                                                 int64_t col_tile, bool xvec, uint32_t xs,
                                                 uint32_t xrow) {
  constexpr int kRaw = CP * 512;
  LaneDecoder<CODE, S> dec;
  EscRuns er{0u, 0u};
  {
    const uint32_t lens =
        kRaw + (CODE == kCodeEsc ? esc_runs<CP>(chunk + kRaw, limit, lane, er) : 0u);
    uint32_t start[S];
    lane_stream_starts<S>(chunk, lens, lane, start);
    dec.init(chunk + lens + kLanes * S, start, limit, table);
  }
  const int g = lane >> 2, c = lane & 3;
  const int64_t cols = p.cols;
  // Rows past the batch read row 0 (see x_at).
  const bool has0 = g < p.batch, has1 = WIDE && g + 8 < p.batch;
  const uint16_t* xr0 = p.x + (has0 ? (int64_t)g * cols : 0);
  const uint16_t* xr1 = p.x + (has1 ? (int64_t)(g + 8) * cols : 0);
  const uint32_t xs0 = xs + (has0 ? g * xrow : 0u) + 32u * c;
  const uint32_t xs1 = xs + (has1 ? (g + 8) * xrow : 0u) + 32u * c;
  const bool vec = xvec && col_tile + CP * 64 <= cols;  // whole tile inside and aligned
  // x of the block at column offset o (from this lane's first column).  Lanes
  // of batch rows past the batch read row 0 instead: they only feed rows of D
  // that are never stored (row g of D depends on row g of A alone).
  auto x_at = [&](const uint16_t* xr, uint32_t xsr, uint32_t o) -> uint2 {
    if (XSM) return lds64(xsr + 2 * o);
    return load_x4(xr, cols, col_tile + 16 * c + o, vec);
  };
  uint2 xa = x_at(xr0, xs0, 0);
  uint2 xb = WIDE ? x_at(xr1, xs1, 0) : make_uint2(0u, 0u);
#pragma unroll 2
  for (int m = 0; m < CP; ++m) {
    const uint4 rv = lds128(chunk + m * 512 + lane * 16);
    const bool esc = CODE == kCodeEsc && ((er.mine >> m) & 1u);
    uint4 ev = make_uint4(0u, 0u, 0u, 0u);
    if (esc) {
      ev = lds128(er.at);
      er.at += kEscRunBytes;
    }
#pragma unroll
    for (int s2 = 0; s2 < 4; s2 += 2) {
      uint32_t e[4];
      if (esc)
        esc_quad(ev, s2 / 2, e);
      else
        dec.quad(table, e);  // pairs 2 s2 .. 2 s2 + 3: blocks s2 and s2 + 1
      if (CODE == kCodeEsc) __syncwarp();  // the MMAs below are warp-wide
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const int s = s2 + h;
        const uint2 xa_s = xa, xb_s = xb;
        // Next block's x: + 4 columns, or the next group's first block.
        const uint32_t no = s < 3 ? 64 * m + 4 * (s + 1) : 64 * (m + 1);
        if (s < 3 || m + 1 < CP) {
          xa = x_at(xr0, xs0, no);
          if (WIDE) xb = x_at(xr1, xs1, no);
        }
        const uint32_t w0 = assemble<CODE>(raw_pair_r(rv, 2 * s), e[2 * h]);
        const uint32_t w1 = assemble<CODE>(raw_pair_r(rv, 2 * s + 1), e[2 * h + 1]);
        mma_bf16_16816(d, xa_s.x, WIDE ? xb_s.x : 0u, xa_s.y, WIDE ? xb_s.y : 0u, w0, w1);
      }
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

// Sets up barriers and runs the producer warp (warp NC), for which it returns
// false once its work is done.
template <int NC>
__device__ __forceinline__ bool setup(const TileParams& p, uint8_t* smem, const Smem& s) {
  allow_dependents();
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
  return true;
}

// Consumers: wait for the decode table.
__device__ __forceinline__ bool wait_table(const Smem& s, const WaitCtl& wc) {
  return __all_sync(kFull, wait_bounded(s.table_bar, 0, wc));
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

// y[b][n] for up to 8 (16 when WIDE) rows b of x.  Consumer warp w takes
// tiles w, w + NC, ...; each tile's partial sums go straight to y (one column
// block) or to the workspace, reduced after all tiles in a fixed order.
template <int NC, int CP, bool WIDE, int CODE, int S>
__global__ void __launch_bounds__((NC + 1) * 32, 1) gemv_kernel(TileParams p) {
  extern __shared__ __align__(128) uint8_t smem[];
  const Smem s = carve(smem, p);
  int64_t first;
  int n;
  cta_range(p, &first, &n);
  if (!setup<NC>(p, smem, s)) return;
  const WaitCtl wc = wait_ctl(p);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = lane >> 2, c = lane & 3;
  const uint32_t table = smem_u32(smem);
  const uint32_t ring = smem_u32(s.ring);
  const uint32_t limit = ring + (uint32_t)p.ring_bytes + kRingSlack;  // end of the ring's slack
  const int batch = p.batch;
  const bool xvec = ((reinterpret_cast<uintptr_t>(p.x) & 7) == 0) && (p.cols % 4 == 0);
  // The CTA's column blocks j0 .. j1 of x, staged in shared memory while the
  // decode table is on its way, when they fit; else x is read through L1.
  constexpr int kTileCols = CP * 64;
  const int64_t j0 = first / p.tiles_r, j1 = (first + n - 1) / p.tiles_r;
  const int64_t span = (j1 - j0 + 1) * kTileCols;        // columns staged
  const uint32_t xrow = (uint32_t)(span * 2 + 16);       // bytes per row, padded
  const bool xsmem = (uint64_t)batch * xrow <= (uint64_t)p.xstage_bytes;
  // x, y and the workspace may belong to the previous kernel on the stream; the
  // producer only reads the device image, which no kernel writes.
  wait_prerequisites();
  if (xsmem) {
    // 16-byte pieces when rows of x start 16-byte aligned (a piece is then
    // wholly inside or outside the matrix), else words; two loads in flight
    // per thread before their stores.
    if (((reinterpret_cast<uintptr_t>(p.x) & 15) == 0) && (p.cols % 8 == 0)) {
      const uint32_t pieces = (uint32_t)(span / 8), total = (uint32_t)batch * pieces;
#pragma unroll 2
      for (uint32_t t = threadIdx.x; t < total; t += NC * 32) {
        const uint32_t b = t / pieces, w = t - b * pieces;
        const int64_t col = j0 * kTileCols + 8 * (int64_t)w;
        const uint4 v = col < p.cols ? __ldg(reinterpret_cast<const uint4*>(p.x + b * p.cols + col))
                                     : make_uint4(0u, 0u, 0u, 0u);
        *reinterpret_cast<uint4*>(s.xstage + b * xrow + 16 * w) = v;
      }
    } else {
      const uint32_t words = (uint32_t)(span / 2), total = (uint32_t)batch * words;
      const bool odd = (p.cols & 1) != 0;  // rows start on 2-byte boundaries
#pragma unroll 2
      for (uint32_t t = threadIdx.x; t < total; t += NC * 32) {
        const uint32_t b = t / words, w = t - b * words;
        const int64_t col = j0 * kTileCols + 2 * (int64_t)w;
        const uint16_t* xr = p.x + b * p.cols;
        const uint32_t v =
            odd ? load_x2_any(xr, p.cols, col)
                : (col < p.cols ? __ldg(reinterpret_cast<const uint32_t*>(xr + col)) : 0u);
        *reinterpret_cast<uint32_t*>(s.xstage + b * xrow + 4 * w) = v;
      }
    }
    named_barrier_sync(1, NC * 32);  // consumers only
  }
  if (!wait_table(s, wc)) return;
  const uint32_t xst = smem_u32(s.xstage);
  const uint32_t* tile_ring = p.tile_ring + first;
  uint32_t at_next = warp < n ? __ldg(tile_ring + warp) : 0u;
  TilePos pos;
  pos.init(first + warp, (uint32_t)p.tiles_r);
  for (int q = warp; q < n; q += NC, pos.step(NC)) {
    const int k = q / p.batch_tiles;
    const uint32_t chunk = ring + at_next;
    if (q + NC < n) at_next = __ldg(tile_ring + q + NC);  // next tile's ring offset, early
    if (!wait_batch(s, k, wc)) return;
    const int64_t i = pos.i, j = pos.j;
    float d[4] = {0.f, 0.f, 0.f, 0.f};
    if (xsmem)
      decode_gemv_tile<CP, WIDE, CODE, S, true>(chunk, table, limit, lane, d, p, j * kTileCols,
                                                xvec, xst + (uint32_t)((j - j0) * kTileCols * 2),
                                                xrow);
    else
      decode_gemv_tile<CP, WIDE, CODE, S, false>(chunk, table, limit, lane, d, p, j * kTileCols,
                                                 xvec, 0u, 0u);
    __syncwarp();
    if (lane == 0) mbar_arrive(&s.empty[k % kSlots]);  // release the tile's share of the batch
    // Lane (g, c) holds rows 2c, 2c + 1 of the tile for batch rows g and g + 8.
    const int64_t row = i * 8 + 2 * c;
#pragma unroll
    for (int h = 0; h < (WIDE ? 2 : 1); ++h) {
      const int b = g + 8 * h;
      if (b >= batch) continue;
      if (p.tiles_c == 1) {
        float* yb = p.y + (int64_t)b * p.rows;
        if (row < p.rows) yb[row] = d[2 * h];
        if (row + 1 < p.rows) yb[row + 1] = d[2 * h + 1];
      } else {
        __stcg(reinterpret_cast<float2*>(p.partial + ((int64_t)j * batch + b) * p.rows_pad + row),
               make_float2(d[2 * h], d[2 * h + 1]));
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
      for (int qq = lane; qq < 8 * batch; qq += 32) {
        const int b = qq >> 3, rr = qq & 7;
        const int64_t orow = i * 8 + rr;
        const float* part = p.partial + (int64_t)b * p.rows_pad + orow;
        const int64_t stride = (int64_t)batch * p.rows_pad;
        float sum = 0.f;
        int64_t jj = 0;
        for (; jj + 8 <= p.tiles_c; jj += 8) {
          float v[8];
#pragma unroll
          for (int u = 0; u < 8; ++u) v[u] = __ldcg(part + (jj + u) * stride);
#pragma unroll
          for (int u = 0; u < 8; ++u) sum += v[u];
        }
        for (; jj < p.tiles_c; ++jj) sum += __ldcg(part + jj * stride);
        if (orow < p.rows) p.y[(int64_t)b * p.rows + orow] = sum;
      }
      if (lane == 0) p.counters[i] = 0u;
    }
  }
}

template <int NC, int CP, int CODE, int S>
__global__ void __launch_bounds__((NC + 1) * 32, 1) decompress_kernel(TileParams p) {
  extern __shared__ __align__(128) uint8_t smem[];
  const Smem s = carve(smem, p);
  int64_t first;
  int n;
  cta_range(p, &first, &n);
  if (!setup<NC>(p, smem, s)) return;
  wait_prerequisites();  // the output may still be read by the previous kernel
  const WaitCtl wc = wait_ctl(p);
  if (!wait_table(s, wc)) return;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t table = smem_u32(smem);
  const uint32_t ring = smem_u32(s.ring);
  const uint32_t limit = ring + (uint32_t)p.ring_bytes + kRingSlack;  // end of the ring's slack
  const int64_t cols = p.cols;
  // Rows start 16-byte aligned: 16 columns of a row go out as two 16-byte stores.
  const bool vec = (cols % 8 == 0) && ((reinterpret_cast<uintptr_t>(p.out) & 15) == 0);
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
    if (!wait_batch(s, k, wc)) return;
    const int64_t i = pos.i, j = pos.j;
    LaneDecoder<CODE, S> dec;
    EscRuns er{0u, 0u};
    {
      const uint32_t lens =
          kRaw + (CODE == kCodeEsc ? esc_runs<CP>(chunk + kRaw, limit, lane, er) : 0u);
      uint32_t start[S];
      lane_stream_starts<S>(chunk, lens, lane, start);
      dec.init(chunk + lens + kLanes * S, start, limit, table);
    }
    if (er.mine & kEscCorrupt) invalid |= kEntryInvalid;
    // Lane L owns row L / 4 of the tile and 16 consecutive columns per group.
    const int64_t row = i * 8 + (lane >> 2);
    const bool row_in = row < p.rows;
    uint16_t* orow = p.out + row * cols;
#pragma unroll 1
    for (int g = 0; g < CP; ++g) {
      const uint4 rv = lds128(chunk + g * 512 + lane * 16);
      const int64_t col = j * (CP * 64) + g * 64 + 16 * (lane & 3);
      const bool esc = CODE == kCodeEsc && ((er.mine >> g) & 1u);
      uint4 ev = make_uint4(0u, 0u, 0u, 0u);
      if (esc) {
        ev = lds128(er.at);
        er.at += kEscRunBytes;
      }
      uint32_t wv[8];
#pragma unroll
      for (int r = 0; r < 8; r += 4) {
        uint32_t e[4];
        if (esc)
          esc_quad(ev, r / 4, e);
        else
          dec.quad(table, e);
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          invalid |= e[k];
          wv[r + k] = assemble<CODE>(raw_pair_r(rv, r + k), e[k]);
        }
      }
      if (row_in && vec && col + 16 <= cols) {
        uint4* dst = reinterpret_cast<uint4*>(orow + col);
        dst[0] = make_uint4(wv[0], wv[1], wv[2], wv[3]);
        dst[1] = make_uint4(wv[4], wv[5], wv[6], wv[7]);
      } else if (row_in) {
#pragma unroll
        for (int r = 0; r < 8; ++r) {
          const int64_t c0 = col + 2 * r;
          if (c0 < cols) orow[c0] = (uint16_t)wv[r];
          if (c0 + 1 < cols) orow[c0 + 1] = (uint16_t)(wv[r] >> 16);
        }
      }
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&s.empty[k % kSlots]);  // release the tile's share of the batch
  }
  if (__any_sync(kFull, invalid & kEntryInvalid) && lane == 0)
    atomicOr(p.err, kErrCorrupt);
}

// Row gather ("NWC", "How it works > Dequantization and embedding lookup": the
// same decoder serves row lookups).  CTA i takes requested rows i, i + CTAs,
// ...; for a row, warp w takes column blocks w, w + warps, ...  The decode
// table arrives by bulk copy (lanes 0 .. 7 of warp 0 issue its pieces) while
// every warp fetches its first tile: the chunk offsets, the raw plane
// (straight into registers, all of it at once) and the lane lengths and
// streams (into the warp's shared-memory stage with coalesced 16-byte loads).
// A warp prefix sum gives every lane's stream start, and the four lanes that
// own the row's tile row (lane 4g + c owns row g) decode it with the GEMV's
// reader.  Only the tiles of the requested rows are read.
constexpr int kGatherWarps = 8;
constexpr uint32_t kGatherBarBytes = 16;  // table barrier, between table and stages

template <int CP, int CODE, int S>
__global__ void __launch_bounds__(kGatherWarps * 32) gather_kernel(GatherParams p) {
  extern __shared__ __align__(16) uint8_t gsm[];
  constexpr int kRaw = CP * 512;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  uint64_t* tbar = reinterpret_cast<uint64_t*>(gsm + p.table_bytes);
  if (threadIdx.x == 0) {
    mbar_init(tbar, 1);
    fence_barrier_init();
  }
  __syncthreads();
  if (warp == 0) {
    if (lane == 0) mbar_expect_tx(tbar, p.table_bytes);
    __syncwarp();
    if (lane < kTablePieces) {
      const uint32_t piece = p.table_bytes / kTablePieces;
      const uint32_t off = ((blockIdx.x + lane) % kTablePieces) * piece;
      bulk_load(gsm + off, reinterpret_cast<const uint8_t*>(p.table) + off, piece, tbar);
    }
  }
  const WaitCtl wc{p.err, kDefaultWaitLimit};
  const uint32_t table = smem_u32(gsm);
  uint8_t* stage = gsm + p.table_bytes + kGatherBarBytes + (size_t)warp * p.stage_bytes;
  const uint32_t sbase = smem_u32(stage);
  const uint32_t limit = sbase + p.stage_bytes;
  const int g = lane >> 2, c = lane & 3;
  const bool vec = (p.cols % 8 == 0) && ((reinterpret_cast<uintptr_t>(p.out) & 15) == 0);
  uint32_t invalid = 0;
  bool have_table = false, ok = true;
  for (int64_t i = blockIdx.x; i < p.n && ok; i += gridDim.x) {
    const int32_t row = __ldg(p.row_ids + i);
    if (row < 0 || row >= p.rows) {
      if (threadIdx.x == 0) atomicOr(p.err, kErrRange);
      continue;
    }
    uint16_t* orow = p.out + i * p.cols;
    for (int64_t j = warp; j < p.tiles_c; j += kGatherWarps) {
      const int64_t u = j * p.tiles_r + row / kTileRows;
      const uint32_t c0 = __ldg(p.index + u), c1 = __ldg(p.index + u + 1);
      const uint8_t* chunk = p.tiles + 16ull * c0;
      const bool mine = g == row % kTileRows;
      uint4 rv[CP];
      if (mine) {
#pragma unroll
        for (int m = 0; m < CP; ++m)
          rv[m] = __ldg(reinterpret_cast<const uint4*>(chunk + m * 512 + lane * 16));
      }
      // Lane lengths and streams: the chunk after its raw plane, clamped to the
      // stage (a corrupt index can misdecode but not overrun it).
      uint32_t bytes = 16u * (c1 - c0) > (uint32_t)kRaw ? 16u * (c1 - c0) - (uint32_t)kRaw : 0u;
      if (bytes > p.stage_bytes - kRingSlack) bytes = p.stage_bytes - kRingSlack;
      __syncwarp();
      {
        uint4 sv[4];
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const uint32_t o = 16u * lane + 512u * q;
          if (o < bytes) sv[q] = __ldg(reinterpret_cast<const uint4*>(chunk + kRaw + o));
        }
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const uint32_t o = 16u * lane + 512u * q;
          if (o < bytes) *reinterpret_cast<uint4*>(stage + o) = sv[q];
        }
        for (uint32_t o = 16u * lane + 2048u; o < bytes; o += 512u)
          *reinterpret_cast<uint4*>(stage + o) = __ldg(reinterpret_cast<const uint4*>(chunk + kRaw + o));
      }
      __syncwarp();
      EscRuns er{0u, 0u};
      const uint32_t lens = CODE == kCodeEsc ? esc_runs<CP>(sbase, limit, lane, er) : 0u;
      if (er.mine & kEscCorrupt) invalid |= kEntryInvalid;
      uint32_t start[S];
      lane_stream_starts<S>(sbase, lens, lane, start);
      if (!have_table) {
        have_table = __all_sync(kFull, wait_bounded(tbar, 0, wc));
        if (!have_table) {
          ok = false;
          break;
        }
      }
      if (!mine) continue;
      LaneDecoder<CODE, S> dec;
      dec.init(sbase + lens + kLanes * S, start, limit, table);
#pragma unroll
      for (int m = 0; m < CP; ++m) {
        const bool esc = CODE == kCodeEsc && ((er.mine >> m) & 1u);
        uint4 ev = make_uint4(0u, 0u, 0u, 0u);
        if (esc) {
          ev = lds128(er.at);
          er.at += kEscRunBytes;
        }
        uint32_t wv[8];
#pragma unroll
        for (int r = 0; r < 8; r += 4) {
          uint32_t e[4];
          if (esc)
            esc_quad(ev, r / 4, e);
          else
            dec.quad(table, e);
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            invalid |= e[k];
            wv[r + k] = assemble<CODE>(raw_pair_r(rv[m], r + k), e[k]);
          }
        }
        const int64_t col = j * (CP * 64) + m * 64 + 16 * c;
        if (vec && col + 16 <= p.cols) {
          uint4* dst = reinterpret_cast<uint4*>(orow + col);
          dst[0] = make_uint4(wv[0], wv[1], wv[2], wv[3]);
          dst[1] = make_uint4(wv[4], wv[5], wv[6], wv[7]);
        } else {
#pragma unroll
          for (int r = 0; r < 8; ++r) {
            const int64_t c2 = col + 2 * r;
            if (c2 < p.cols) orow[c2] = (uint16_t)wv[r];
            if (c2 + 1 < p.cols) orow[c2 + 1] = (uint16_t)(wv[r] >> 16);
          }
        }
      }
    }
  }
  if (invalid & kEntryInvalid) atomicOr(p.err, kErrCorrupt);
  // The table copy must have landed before the CTA's shared memory is
  // released, also in a CTA that had no valid row to decode.
  if (threadIdx.x == 0 && !have_table) wait_bounded(tbar, 0, drain_ctl_default(p.err));
}

// ---- tensor-core path: decode once into shared memory, tcgen05 MMA ---------
//
// "Unweight", "Direct GPU Decompression": the compressed weights are
// decompressed into shared memory and fed straight to the tensor cores.  Here
// the decoded tile chunks are the A operand (M = 128 rows of W, K-major, 128-
// byte swizzle) of tcgen05.mma kind::f16 with BF16 inputs and FP32
// accumulation in TMEM; B is x (N = rows of x padded to 16, 32 or 64), brought
// in by TMA with the same swizzle.  Each weight is decoded once for every row
// of x.

__device__ __forceinline__ bool mbar_test_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}
__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}
// Shared-memory matrix descriptor of a K-major operand with 128-byte swizzle:
// rows of 128 bytes (64 BF16 of K), 8-row atoms of 1024 bytes one after the
// other (stride 1024), atoms 1024-byte aligned; the leading offset is unused
// for this layout.  A start 32 bytes further selects the next 16 columns.
__device__ __forceinline__ uint64_t umma_desc_sw128(uint32_t saddr) {
  return (uint64_t)((saddr & 0x3FFFFu) >> 4) | ((uint64_t)1 << 16) |
         ((uint64_t)(1024u >> 4) << 32) | ((uint64_t)1 << 46) | ((uint64_t)2 << 61);
}
// Instruction descriptor of kind::f16: D FP32, A and B BF16, both K-major,
// shape M x N (K = 16).
__device__ __forceinline__ constexpr uint32_t umma_idesc_bf16(int m, int n) {
  return (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(n >> 3) << 17) |
         ((uint32_t)(m >> 4) << 24);
}
// D[tmem] (+)= A B, issued by one thread.
__device__ __forceinline__ void umma_bf16(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                          uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}
// `bar` completes one phase when every tcgen05 operation this thread issued
// before has completed.
__device__ __forceinline__ void umma_commit(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                   smem_u32(bar))
               : "memory");
}
// 2-D TMA load (tile mode, no multicast) of the box at (c0, c1) into `dst`.
__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap* map, int32_t c0,
                                            int32_t c1, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], "
      "[%1, {%2, %3}], [%4];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(smem_u32(bar))
      : "memory");
}
__device__ __forceinline__ void sts128(uint32_t addr, uint32_t a, uint32_t b, uint32_t c,
                                       uint32_t d) {
  asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(a), "r"(b), "r"(c),
               "r"(d)
               : "memory");
}
// NCOL consecutive TMEM columns of the warp's 32 lanes: lane l gets the row
// (lane base + l), v[k] = column (col + k), as FP32.
template <int NCOL>
__device__ __forceinline__ void tmem_load(uint32_t taddr, float (&v)[NCOL]);
template <>
__device__ __forceinline__ void tmem_load<4>(uint32_t taddr, float (&v)[4]) {
  uint32_t r[4];
  asm volatile("tcgen05.ld.sync.aligned.32x32b.x4.b32 {%0, %1, %2, %3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(taddr));
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
  for (int k = 0; k < 4; ++k) v[k] = __uint_as_float(r[k]);
}
template <>
__device__ __forceinline__ void tmem_load<8>(uint32_t taddr, float (&v)[8]) {
  uint32_t r[8];
  asm volatile("tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0, %1, %2, %3, %4, %5, %6, %7}, [%8];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]),
                 "=r"(r[6]), "=r"(r[7])
               : "r"(taddr));
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
  for (int k = 0; k < 8; ++k) v[k] = __uint_as_float(r[k]);
}
template <>
__device__ __forceinline__ void tmem_load<16>(uint32_t taddr, float (&v)[16]) {
  uint32_t r[16];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, "
      "%11, %12, %13, %14, %15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
        "=r"(r[14]), "=r"(r[15])
      : "r"(taddr));
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
  for (int k = 0; k < 16; ++k) v[k] = __uint_as_float(r[k]);
}

// Barriers, counters and flags of the tensor-core kernel (at p.tc_bar_off).
struct TcBars {
  uint64_t* xfull;    // [team][2]: the x chunk of the stage landed (TMA bytes)
  uint64_t* sempty;   // [team][kTcMaxAStages]: the MMAs that read the A stage completed
  uint64_t* accfull;  // [team]: the team's accumulator holds its M-group sum
  uint64_t* accempty; // the epilogue warps have read the accumulators
  uint32_t* tmem;     // TMEM base address (tcgen05.alloc writes it)
  volatile uint32_t* abort;     // a wait gave up: leave
  volatile uint32_t* issued;    // copies the producer has issued so far
  volatile uint32_t* mma_next;  // [team]: chunks whose MMAs have been issued
  uint32_t* xs;                 // x loader: [3][team] fetched, next in group, per group
};
__device__ __forceinline__ TcBars tc_bars(uint8_t* smem, const TileParams& p) {
  TcBars b;
  b.xfull = reinterpret_cast<uint64_t*>(smem + p.tc_bar_off);
  b.sempty = b.xfull + 2 * kTcMaxTeams;
  b.accfull = b.sempty + kTcMaxAStages * kTcMaxTeams;
  b.accempty = b.accfull + kTcMaxTeams;
  b.tmem = reinterpret_cast<uint32_t*>(b.accempty + 1);
  b.abort = b.tmem + 1;
  b.issued = b.tmem + 2;
  b.mma_next = b.tmem + 4;
  b.xs = const_cast<uint32_t*>(b.mma_next) + kTcMaxTeams;
  return b;
}
static_assert(8 * ((2 + kTcMaxAStages + 1) * kTcMaxTeams + 1) + 16 + 4 * (1 + 3) * kTcMaxTeams <=
                  (int)kTcBarBytes,
              "tensor-core barrier area");

// A consumer polls batch k's slot only once the producer has issued batch k:
// the schedule keeps fewer than kSlots batches outstanding, so the slot's
// previous batch (k - kSlots) has landed by then and the parity it polls is
// batch k's, however far this warp's tiles lie apart (the row-panel order can
// put them far apart).
__device__ __forceinline__ bool wait_issued(const TcBars& tb, uint32_t k, const WaitCtl& w) {
  for (uint32_t it = 0; it < w.limit; ++it) {
    if (*tb.issued > k) return true;
    if (*tb.abort) break;
    __nanosleep(32);
  }
  atomicOr(w.err, kErrTimeout);
  return false;
}

// The rectangle of tiles this CTA owns: row tiles [i_lo, i_hi) x column
// blocks [j_lo, j_hi), column range ks of the K split.
struct TcWork {
  int64_t i_lo, i_hi, j_lo, j_hi;
  int ks;         // this CTA's column range
  int groups;     // M-groups of R row tiles
  int teams;      // teams with at least one column block (min(TT, j_hi - j_lo))
};
__device__ __forceinline__ TcWork tc_work(const TileParams& p) {
  TcWork w;
  const int64_t ks = blockIdx.x % p.tc_ksplit, rs = blockIdx.x / p.tc_ksplit;
  const int64_t row_ranges = gridDim.x / p.tc_ksplit;
  w.i_lo = p.tiles_r * rs / row_ranges;
  w.i_hi = p.tiles_r * (rs + 1) / row_ranges;
  w.j_lo = p.tiles_c * ks / p.tc_ksplit;
  w.j_hi = p.tiles_c * (ks + 1) / p.tc_ksplit;
  w.ks = (int)ks;
  w.groups = (int)((w.i_hi - w.i_lo + p.tc_rows - 1) / p.tc_rows);
  const int64_t cols = w.j_hi - w.j_lo;
  w.teams = (int)(cols < p.tc_teams ? cols : p.tc_teams);
  return w;
}
// Slot of the scratch that holds column range ks's sums of row tile i:
// [kMaxTcRows][8] floats.
__device__ __forceinline__ float* tc_slot(const TileParams& p, int ks, int64_t i) {
  return p.partial + ((int64_t)ks * p.tiles_r + i) * (8 * kMaxTcRows);
}

// Accumulator columns (N / 4) an epilogue warp reads back: the sum of the
// teams' accumulators for the warp's lane quarter q = warp % 4 and column
// quarter warp / 4, and its store to y or, when K is split, to the slot of
// this CTA's column range.
template <int NQ>
__device__ __forceinline__ void tc_epilogue(const TileParams& p, const TcWork& wk, uint32_t tmem,
                                            int warp, int lane, int64_t ig, int rg) {
  const int q = warp & 3, kq = warp >> 2;
  float acc[NQ];
#pragma unroll
  for (int u = 0; u < NQ; ++u) acc[u] = 0.f;
  const uint32_t base = tmem + ((uint32_t)(32 * q) << 16) + (uint32_t)(kq * NQ);
  for (int t = 0; t < wk.teams; ++t) {
    float v[NQ];
    tmem_load<NQ>(base + (uint32_t)(t * p.tc_n), v);
#pragma unroll
    for (int u = 0; u < NQ; ++u) acc[u] += v[u];
  }
  const int mrow = 32 * q + lane, rr = mrow >> 3;
  if (rr >= rg) return;
  const int64_t i = ig + rr, orow = 8 * i + (lane & 7);
  if (p.tc_ksplit == 1) {
    if (orow >= p.rows) return;
#pragma unroll
    for (int u = 0; u < NQ; ++u) {
      const int bc = kq * NQ + u;
      if (bc >= p.batch) break;
      p.y[(int64_t)bc * p.rows + orow] = acc[u];
    }
  } else {
    float* slot = tc_slot(p, wk.ks, i);
#pragma unroll
    for (int u = 0; u < NQ; ++u) {
      const int bc = kq * NQ + u;
      if (bc >= p.batch) break;
      __stcg(slot + bc * 8 + (lane & 7), acc[u]);
    }
  }
}

// Row tile i when K is split: the last of the ksplit CTAs to deliver its slot
// adds the slots in column-range order and writes y.  One warp.
__device__ void tc_reduce(const TileParams& p, int64_t i, int lane) {
  uint32_t last = 0;
  if (lane == 0) {
    __threadfence();
    last = atomicAdd(&p.counters[i], 1u) == (uint32_t)(p.tc_ksplit - 1);
  }
  if (!__shfl_sync(kFull, last, 0)) return;
  __threadfence();
  for (int idx = lane; idx < 8 * p.batch; idx += 32) {
    const int bc = idx >> 3, r = idx & 7;
    const int64_t orow = 8 * i + r;
    float sum = 0.f;
    for (int ks = 0; ks < p.tc_ksplit; ++ks) sum += __ldcg(tc_slot(p, ks, i) + bc * 8 + r);
    if (orow < p.rows) p.y[(int64_t)bc * p.rows + orow] = sum;
  }
  if (lane == 0) p.counters[i] = 0u;
}

// 16 raw bytes of global memory, read once (not kept in L1).
__device__ __forceinline__ uint4 ldg_stream128(const uint8_t* p) {
  uint4 v;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p));
  return v;
}

// Waits (bounded) for `parity` of `bar`, or gives up at once when another
// warp of the CTA already gave up.
__device__ bool wait_or_abort(uint64_t* bar, uint32_t parity, const WaitCtl& w,
                              volatile uint32_t* abort) {
  for (uint32_t it = 0; it < w.limit; ++it) {
    if (mbar_try_wait(bar, parity)) return true;
    if (*abort) return false;
    if (it >= 2) __nanosleep(64);  // a long wait leaves the issue slots to the decoders
  }
  atomicOr(w.err, kErrTimeout);
  return false;
}

// Issues the MMAs of chunk c of team t: the four K = 16 steps of A stage
// c % astages against x stage c % bstages into the team's accumulator, their
// completion committed to the A stage's barrier (and, for the group's last
// chunk, to the team's accumulator barrier).  Called by lane 0 of the team's
// leader warp once the team's warps have written the chunk, so a team's
// chunks are issued by one thread in order.  w is the chunk's index within its
// M-group gi, per_group the team's chunks per group.
__device__ bool tc_issue(const TileParams& p, const TcBars& tb, uint32_t a_area, uint32_t b_area,
                         int t, uint32_t c, uint32_t st, uint32_t w, uint32_t per_group, int gi,
                         const WaitCtl& wc) {
  const uint32_t SB = (uint32_t)p.tc_bstages, NA = (uint32_t)p.tc_astages;
  // x stage and its phase parity (one or two stages).
  const uint32_t sx = SB == 2u ? (c & 1u) : 0u, phx = SB == 2u ? ((c >> 1) & 1u) : (c & 1u);
  if (!wait_or_abort(&tb.xfull[2 * t + (int)sx], phx, wc, tb.abort)) return false;
  // The group's first MMA overwrites the accumulator: the epilogue of the
  // previous group must have read it.
  if (w == 0 && gi > 0 && !wait_or_abort(tb.accempty, (uint32_t)(gi - 1) & 1u, wc, tb.abort))
    return false;
  tc_fence_after();
  const uint32_t N = (uint32_t)p.tc_n;
  const uint32_t a0 = a_area + ((uint32_t)t * NA + st) * (uint32_t)p.tc_rows * kTcStageA;
  const uint32_t b0 = b_area + ((uint32_t)t * SB + sx) * N * 128u;
  const uint32_t idesc = umma_idesc_bf16(128, (int)N);
  const uint32_t d = *tb.tmem + (uint32_t)t * N;
  // The next 16 columns start 32 bytes further: 2 in the descriptor's start
  // field (address / 16, which stays below 2^14 inside shared memory).
  const uint64_t da = umma_desc_sw128(a0), db = umma_desc_sw128(b0);
  umma_bf16(d, da, db, idesc, w == 0 ? 0u : 1u);
#pragma unroll
  for (int k = 1; k < 4; ++k) umma_bf16(d, da + 2u * k, db + 2u * k, idesc, 1u);
  umma_commit(&tb.sempty[kTcMaxAStages * t + (int)st]);
  if (w + 1 == per_group) umma_commit(&tb.accfull[t]);
  tb.mma_next[t] = c + 1;  // read by the teardown (after a CTA barrier)
  return true;
}

// Decode warps (0 .. 29): warp w < teams R is slot r = w % R of team t = w / R.
// A tile's lane lengths and streams come from the ring; its raw plane straight
// from global memory, two 64-column groups ahead.  Each warp writes its row
// tile's 8 x 64 chunk into the team's A stage; the team's leader (slot 0)
// issues each chunk's MMAs once the whole team has passed the team's named
// barrier (bar.sync by all R warps, once per chunk, in lockstep).
// Warps 0 .. 15 also read the accumulators back after each M-group.
template <int CP, int CODE, int S>
__device__ void tc_decode(const TileParams& p, uint8_t* smem, const Smem& s, const TcBars& tb,
                          const TcWork& wk, int warp, int lane) {
  const WaitCtl wc = wait_ctl(p);
  const int R = p.tc_rows, TT = p.tc_teams;
  const uint32_t NA = (uint32_t)p.tc_astages;
  const bool decoder = warp < TT * R;
  const bool epilogue = warp < kTcEpilogueWarps;
  const int t = warp / R, r = warp % R;
  const int g = lane >> 2, c = lane & 3;
  const uint32_t table = smem_u32(smem);
  const uint32_t ring = smem_u32(s.ring);
  const uint32_t limit = ring + (uint32_t)p.ring_bytes + kRingSlack;
  const uint32_t a_area = smem_u32(smem + p.tc_a_off);
  const uint32_t b_area = smem_u32(smem + p.tc_b_off);
  const int64_t nj = decoder && t < wk.teams ? (wk.j_hi - wk.j_lo - t + TT - 1) / TT : 0;
  const uint32_t per_group = (uint32_t)nj * CP;
  const uint32_t chunk_lo = ((uint32_t)(2 * c) ^ (uint32_t)g) << 4;
  const uint32_t chunk_hi = ((uint32_t)(2 * c + 1) ^ (uint32_t)g) << 4;
  uint32_t seq = 0, st = 0, use = 0;  // chunk count, its A stage (seq % NA) and use (seq / NA)
  bool ok = true;
  // The loops run to the end even after a wait gave up (ok false, abort set):
  // every warp must pass its team's barrier as often as the others.
  for (int gi = 0; gi < wk.groups; ++gi) {
    const int64_t ig = wk.i_lo + (int64_t)gi * R;
    const int rg = (int)min((int64_t)R, wk.i_hi - ig);
    const int64_t i = ig + r;
    for (int64_t jj = 0; jj < nj; ++jj) {
      const int64_t j = wk.j_lo + t + jj * TT;
      const bool present = r < rg;
      LaneDecoder<CODE, S> dec;
      EscRuns er{0u, 0u};
      const uint8_t* raw = nullptr;
      uint4 rv0 = make_uint4(0u, 0u, 0u, 0u), rv1 = rv0;
      uint32_t bw = 0;
      if (ok && present) {
        const int64_t u = j * p.tiles_r + i;
        raw = p.tiles + 16ull * __ldg(p.index + u);
        rv0 = ldg_stream128(raw + lane * 16);  // groups 0 and 1, before the wait
        if (CP > 1) rv1 = ldg_stream128(raw + 512 + lane * 16);
        bw = __ldg(p.tile_batch + u);
        const uint32_t stage = ring + __ldg(p.tile_ring + u);
        ok = __all_sync(kFull, wait_issued(tb, bw, wc) &&
                                   wait_or_abort(&s.full[bw % kSlots], (bw / kSlots) & 1u, wc,
                                                 tb.abort));
        if (ok) {
          const uint32_t lens = CODE == kCodeEsc ? esc_runs<CP>(stage, limit, lane, er) : 0u;
          uint32_t start[S];
          lane_stream_starts<S>(stage, lens, lane, start);
          dec.init(stage + lens + kLanes * S, start, limit, table);
        } else if (lane == 0) {
          *tb.abort = 1u;
        }
      }
      for (int m = 0; m < CP; ++m, ++seq, st = st + 1u == NA ? 0u : st + 1u, use += st == 0u) {
        // The stage's previous chunk (seq - NA) must have been multiplied.
        if (ok && use > 0) {
          ok = __all_sync(kFull, wait_or_abort(&tb.sempty[kTcMaxAStages * t + (int)st],
                                               (use - 1) & 1u, wc, tb.abort));
          if (!ok && lane == 0) *tb.abort = 1u;
        }
        const uint32_t arow =
            a_area + (((uint32_t)t * NA + st) * (uint32_t)R + (uint32_t)r) * kTcStageA +
            (uint32_t)g * 128u;
        if (ok && present) {
          const uint4 rv = rv0;
          rv0 = rv1;
          if (m + 2 < CP) rv1 = ldg_stream128(raw + (m + 2) * 512 + lane * 16);
          const bool esc = CODE == kCodeEsc && ((er.mine >> m) & 1u);
          uint4 ev = make_uint4(0u, 0u, 0u, 0u);
          if (esc) {
            ev = lds128(er.at);
            er.at += kEscRunBytes;
          }
          uint32_t wv[8];
#pragma unroll
          for (int k = 0; k < 8; k += 4) {
            uint32_t e[4];
            if (esc)
              esc_quad(ev, k / 4, e);
            else
              dec.quad(table, e);
#pragma unroll
            for (int q = 0; q < 4; ++q) wv[k + q] = assemble<CODE>(raw_pair_r(rv, k + q), e[q]);
          }
          if (CODE == kCodeEsc) __syncwarp();
          sts128(arow + chunk_lo, wv[0], wv[1], wv[2], wv[3]);
          sts128(arow + chunk_hi, wv[4], wv[5], wv[6], wv[7]);
        }
        // (A slot of a row past the group's last row tile keeps stale data:
        // it only reaches accumulator rows that the epilogue skips.)
        fence_proxy_async_smem();  // this lane's A writes, before the MMAs read them
        // Every warp of the team passes the team's barrier (bar.sync, so no
        // warp can lap it) once per chunk, whatever happened; after it the
        // leader (r = 0) issues the chunk's MMAs.
        named_barrier_sync(kTcTeamBarrier0 + t, R * 32);
        if (r == 0) {
          uint32_t issued_ok = 1u;
          if (lane == 0 && ok && !*tb.abort)
            issued_ok = tc_issue(p, tb, a_area, b_area, t, seq, st,
                                 (uint32_t)jj * CP + (uint32_t)m, per_group, gi, wc)
                            ? 1u
                            : 0u;
          ok = ok && __shfl_sync(kFull, issued_ok, 0);
          if (!ok && lane == 0) *tb.abort = 1u;
        }
      }
      if (present && ok) {
        __syncwarp();
        if (lane == 0) mbar_arrive(&s.empty[bw % kSlots]);
      }
    }
    if (!ok || !epilogue) continue;
    // Epilogue of the group, by warps 0 .. 15 (the others go on decoding).
    for (int tt = 0; tt < wk.teams && ok; ++tt)
      ok = __all_sync(kFull, wait_or_abort(&tb.accfull[tt], (uint32_t)gi & 1u, wc, tb.abort));
    if (!ok) {
      if (lane == 0) *tb.abort = 1u;
      continue;
    }
    tc_fence_after();
    const uint32_t tmem = *tb.tmem;
    switch (p.tc_n) {
      case 16: tc_epilogue<4>(p, wk, tmem, warp, lane, ig, rg); break;
      case 32: tc_epilogue<8>(p, wk, tmem, warp, lane, ig, rg); break;
      default: tc_epilogue<16>(p, wk, tmem, warp, lane, ig, rg); break;
    }
    tc_fence_before();
    __threadfence();  // this warp's y and slot stores, before the arrival below
    __syncwarp();
    if (lane == 0) mbar_arrive(tb.accempty);
    // K split: once every epilogue warp has stored its slots (accempty
    // completes this group's phase after their 16 arrivals), epilogue warp w
    // delivers row tile ig + w.
    if (p.tc_ksplit > 1) {
      ok = __all_sync(kFull, wait_or_abort(tb.accempty, (uint32_t)gi & 1u, wc, tb.abort));
      if (ok && warp < rg) tc_reduce(p, ig + warp, lane);
    }
  }
  if (!ok && lane == 0) *tb.abort = 1u;
}

// The x loader (lane 0 of warp 30): brings each team's x chunks into its x
// stages by TMA, in the team's chunk order, as soon as the stage's previous
// chunk has been multiplied.  It serves the teams in turn without blocking on
// any of them; its per-team counters live in shared memory (tb.xs).
template <int CP>
__device__ void tc_xload(const TileParams& p, const CUtensorMap* tmap, uint8_t* smem,
                         const TcBars& tb, const TcWork& wk) {
  const WaitCtl wc = wait_ctl(p);
  const int TT = p.tc_teams;
  const uint32_t SB = (uint32_t)p.tc_bstages, NA = (uint32_t)p.tc_astages;
  const uint32_t b_area = smem_u32(smem + p.tc_b_off);
  const uint32_t bstage = (uint32_t)p.tc_n * 128u;
  uint32_t* nx = tb.xs;                       // chunks fetched
  uint32_t* xw = nx + kTcMaxTeams;            // within-group index of the next
  uint32_t* per_group = xw + kTcMaxTeams;     // chunks per group
  for (int t = 0; t < TT; ++t) {
    per_group[t] =
        t < wk.teams ? (uint32_t)((wk.j_hi - wk.j_lo - t + TT - 1) / TT) * CP : 0u;
    nx[t] = xw[t] = 0;
  }
  wait_prerequisites();  // x may be written by the previous kernel on the stream
  uint32_t idle = 0;
  for (;;) {
    bool done = true, moved = false;
    for (int t = 0; t < TT; ++t) {
      const uint32_t cx = nx[t], tot = (uint32_t)wk.groups * per_group[t];
      if (cx >= tot) continue;
      done = false;
      // x stage cx % SB is free once chunk cx - SB (A stage (cx - SB) % NA)
      // has been multiplied.
      if (cx >= SB) {
        const uint32_t prev = cx - SB;
        if (!mbar_test_wait(&tb.sempty[kTcMaxAStages * t + (int)(prev % NA)], (prev / NA) & 1u))
          continue;
      }
      const uint32_t w = xw[t];
      const int64_t j = wk.j_lo + t + (int64_t)(w / CP) * TT;
      const int m = (int)(w % CP);
      const uint32_t sx = cx % SB;
      mbar_expect_tx(&tb.xfull[2 * t + (int)sx], bstage);
      tma_load_2d(b_area + ((uint32_t)t * SB + sx) * bstage, tmap, (int32_t)(j * CP * 64 + m * 64),
                  0, &tb.xfull[2 * t + (int)sx]);
      nx[t] = cx + 1;
      xw[t] = w + 1 == per_group[t] ? 0u : w + 1;
      moved = true;
    }
    if (done) break;
    if (moved) {
      idle = 0;
    } else if (++idle >= wc.limit || *tb.abort) {
      if (!*tb.abort) atomicOr(wc.err, kErrTimeout);
      *tb.abort = 1u;
      break;
    } else {
      __nanosleep(64);  // leave the issue slots to the decode warps
    }
  }
}

// After every decode warp has left: wait (bounded) for the x loads that no MMA
// consumed and for the MMAs issued, so that nothing writes this CTA's shared
// memory or TMEM once it is released.  On the ordinary path every load was
// consumed and the epilogue saw every MMA complete; this matters after a wait
// gave up.
__device__ void tc_drain(const TileParams& p, const TcBars& tb) {
  const WaitCtl dc = drain_ctl(p);
  const uint32_t SB = (uint32_t)p.tc_bstages, NA = (uint32_t)p.tc_astages;
  for (int t = 0; t < p.tc_teams; ++t) {
    const uint32_t issued = tb.mma_next[t];
    for (uint32_t k = issued; k < tb.xs[t]; ++k)
      wait_bounded(&tb.xfull[2 * t + (int)(k % SB)], (k / SB) & 1u, dc);
    for (uint32_t k = issued > NA ? issued - NA : 0u; k < issued; ++k)
      wait_bounded(&tb.sempty[kTcMaxAStages * t + (int)(k % NA)], (k / NA) & 1u, dc);
  }
}

// y[b][n] for up to kMaxTcRows rows b of x, every weight decoded once.
// Warps 0..29 decode into the A stages and issue the MMAs (0..15 also read
// the accumulators back), warp 30 allocates TMEM and loads x, warp 31 moves
// the compressed streams into the ring (the same producer as the other
// kernels).
template <int CP, int CODE, int S>
__global__ void __launch_bounds__(kTcThreads, 1)
    gemv_tc_kernel(const TileParams p, const __grid_constant__ CUtensorMap tmap) {
  extern __shared__ __align__(1024) uint8_t smem_tc[];
  uint8_t* smem = smem_tc;
  allow_dependents();
  if (smem_u32(smem) & 1023u) {  // the swizzled stages need 1024-byte alignment
    if (threadIdx.x == 0) atomicOr(p.err, kErrLayout);
    return;
  }
  const Smem s = carve(smem, p);
  const TcBars tb = tc_bars(smem, p);
  const TcWork wk = tc_work(p);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    mbar_init(s.table_bar, 1);
    for (int k = 0; k < kSlots; ++k) {
      mbar_init(&s.full[k], 1);
      mbar_init(&s.empty[k], (uint32_t)p.batch_tiles);
    }
    for (int k = 0; k < 2 * kTcMaxTeams; ++k) mbar_init(&tb.xfull[k], 1);
    for (int k = 0; k < kTcMaxAStages * kTcMaxTeams; ++k) mbar_init(&tb.sempty[k], 1);
    for (int k = 0; k < kTcMaxTeams; ++k) {
      mbar_init(&tb.accfull[k], 1);
      tb.mma_next[k] = 0u;
      tb.xs[k] = 0u;
    }
    mbar_init(tb.accempty, kTcEpilogueWarps);
    *tb.abort = 0u;
    *tb.issued = 0u;
  }
  if (warp == kTcMmaWarp) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_u32(tb.tmem)),
                 "r"(p.tc_tmem_cols));
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  fence_barrier_init();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == kTcProducerWarp) {
    const uint32_t b0 = __ldg(p.sched_cta + blockIdx.x), b1 = __ldg(p.sched_cta + blockIdx.x + 1);
    // Each copy brings a tile's streams; its raw plane (read by the decode
    // warps from global memory) is prefetched into L2 at the same time.
    produce(p, smem, s, p.sched_batch + b0, (int)(b1 - b0), lane, tb.issued, CP * 512u);
    return;
  }
  if (warp < kTcDecodeWarps) {
    wait_prerequisites();  // y and the scratch may belong to the previous kernel
    const WaitCtl wc = wait_ctl(p);
    if (wait_table(s, wc)) {
      tc_decode<CP, CODE, S>(p, smem, s, tb, wk, warp, lane);
    } else if (lane == 0) {
      *tb.abort = 1u;
    }
    __syncwarp();
  } else if (lane == 0) {
    tc_xload<CP>(p, &tmap, smem, tb, wk);
  }
  __syncwarp();
  // Teardown: every decode warp and the x loader, then what is still in
  // flight, then TMEM goes back.
  tc_fence_before();
  named_barrier_sync(kTcTeardownBarrier, (kTcDecodeWarps + 1) * 32);
  if (warp == kTcMmaWarp) {
    // On the ordinary path every x load was consumed and the epilogue saw
    // every MMA complete; only after a wait gave up is there anything to wait
    // for.
    if (lane == 0 && *tb.abort) tc_drain(p, tb);
    __syncwarp();
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(*tb.tmem),
                 "r"(p.tc_tmem_cols)
                 : "memory");
  }
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

// Consumer warps per CTA: as many as the registers allow (32 warps leave 64
// registers a thread); they hide the decoder's dependency chains.
constexpr int kConsumers = 31;
static_assert(kConsumers <= kMaxLag, "the launch schedule assumes a lag of at most kMaxLag");

// One CTA per SM with programmatic stream serialization: the kernel may start
// before the previous one on the stream ends; it waits for it (see
// wait_prerequisites) before it touches anything that kernel could use.
template <typename Kernel>
cudaError_t launch_pdl(Kernel k, const LaunchShape& s, cudaStream_t stream, const TileParams& p) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)s.ctas);
  cfg.blockDim = dim3((unsigned)((kConsumers + 1) * 32));
  cfg.dynamicSmemBytes = s.smem_bytes;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, k, p);
}


template <int CP, bool WIDE, int CODE, int S>
cudaError_t launch_gemv_t(const TileParams& p, const LaunchShape& s, cudaStream_t stream) {
  static int configured[64] = {};
  cudaError_t e =
      ensure_smem(gemv_kernel<kConsumers, CP, WIDE, CODE, S>, s.smem_bytes, configured);
  if (e != cudaSuccess) return e;
  return launch_pdl(gemv_kernel<kConsumers, CP, WIDE, CODE, S>, s, stream, p);
}

template <int CP, int CODE, int S>
cudaError_t launch_gemv_s(const TileParams& p, const LaunchShape& s, cudaStream_t stream) {
  if (p.batch < 1 || p.batch > kMaxPassRows) return cudaErrorInvalidValue;
  return p.batch <= 8 ? launch_gemv_t<CP, false, CODE, S>(p, s, stream)
                      : launch_gemv_t<CP, true, CODE, S>(p, s, stream);
}

template <int CP, int CODE>
cudaError_t launch_gemv_cp(const TileParams& p, const LaunchShape& s, cudaStream_t stream) {
  if constexpr (CODE == kCodeRank || CODE == kCodeEsc) {
    return launch_gemv_s<CP, CODE, 1>(p, s, stream);
  } else {
    return p.streams == 2 ? launch_gemv_s<CP, CODE, 2>(p, s, stream)
                          : launch_gemv_s<CP, CODE, 1>(p, s, stream);
  }
}

template <int CP, int CODE, int S>
cudaError_t launch_gemv_tc_s(const TileParams& p, const CUtensorMap& tmap, const LaunchShape& s,
                             cudaStream_t stream) {
  static int configured[64] = {};
  cudaError_t e = ensure_smem(gemv_tc_kernel<CP, CODE, S>, s.smem_bytes, configured);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)s.ctas);
  cfg.blockDim = dim3((unsigned)kTcThreads);
  cfg.dynamicSmemBytes = s.smem_bytes;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, gemv_tc_kernel<CP, CODE, S>, p, tmap);
}

template <int CP, int CODE>
cudaError_t launch_gemv_tc_t(const TileParams& p, const CUtensorMap& tmap, const LaunchShape& s,
                             cudaStream_t stream) {
  if constexpr (CODE == kCodeRank || CODE == kCodeEsc) {
    return launch_gemv_tc_s<CP, CODE, 1>(p, tmap, s, stream);
  } else {
    return p.streams == 2 ? launch_gemv_tc_s<CP, CODE, 2>(p, tmap, s, stream)
                          : launch_gemv_tc_s<CP, CODE, 1>(p, tmap, s, stream);
  }
}

template <int CP, int CODE, int S>
cudaError_t launch_decompress_s(const TileParams& p, const LaunchShape& s, cudaStream_t stream) {
  static int configured[64] = {};
  cudaError_t e =
      ensure_smem(decompress_kernel<kConsumers, CP, CODE, S>, s.smem_bytes, configured);
  if (e != cudaSuccess) return e;
  return launch_pdl(decompress_kernel<kConsumers, CP, CODE, S>, s, stream, p);
}

template <int CP, int CODE>
cudaError_t launch_decompress_t(const TileParams& p, const LaunchShape& s, cudaStream_t stream) {
  if constexpr (CODE == kCodeRank || CODE == kCodeEsc) {
    return launch_decompress_s<CP, CODE, 1>(p, s, stream);
  } else {
    return p.streams == 2 ? launch_decompress_s<CP, CODE, 2>(p, s, stream)
                          : launch_decompress_s<CP, CODE, 1>(p, s, stream);
  }
}

}  // namespace

LaunchShape launch_shape(int64_t n_tiles, uint64_t max_chunk, uint64_t typical_chunk,
                         uint32_t table_bytes, int sm_count, size_t smem_limit,
                         uint32_t xstage_bytes) {
  LaunchShape s;
  s.xstage_bytes = xstage_bytes;
  int64_t ctas = n_tiles < sm_count ? n_tiles : sm_count;
  if (ctas > (int64_t)kMaxCtas) ctas = kMaxCtas;
  s.ctas = ctas < 1 ? 1 : (int)ctas;
  s.table_bytes = table_bytes;
  const size_t head = xstage_offset(table_bytes) + xstage_bytes;
  s.ring_offset = (head + 127) / 128 * 128;
  const int64_t per_cta = (n_tiles + s.ctas - 1) / s.ctas;
  // Tiles per bulk copy: enough for kBatchTarget bytes of typical chunks,
  // between 2 and 8 (at least 2 keeps the schedule's batch count within its
  // area).
  int t = (int)((kBatchTarget + typical_chunk - 1) / (typical_chunk ? typical_chunk : 1));
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

// Calls f with std::integral_constant<int, code> for a runtime code.
template <typename F>
cudaError_t by_code(int code, F&& f) {
  switch (code) {
    case kCodeRank: return f(std::integral_constant<int, kCodeRank>{});
    case kCodeEsc: return f(std::integral_constant<int, kCodeEsc>{});
    case kCode14: return f(std::integral_constant<int, kCode14>{});
    case kCode12: return f(std::integral_constant<int, kCode12>{});
    default: return cudaErrorInvalidValue;
  }
}

cudaError_t launch_gemv(const TileParams& p, int tile_cols, int code, const LaunchShape& s,
                        cudaStream_t stream) {
  switch (tile_cols) {
    case 512: return by_code(code, [&](auto k) { return launch_gemv_cp<8, decltype(k)::value>(p, s, stream); });
    case 256: return by_code(code, [&](auto k) { return launch_gemv_cp<4, decltype(k)::value>(p, s, stream); });
    case 128: return by_code(code, [&](auto k) { return launch_gemv_cp<2, decltype(k)::value>(p, s, stream); });
    case 64: return by_code(code, [&](auto k) { return launch_gemv_cp<1, decltype(k)::value>(p, s, stream); });
    default: return cudaErrorInvalidValue;
  }
}

cudaError_t launch_decompress(const TileParams& p, int tile_cols, int code,
                              const LaunchShape& s, cudaStream_t stream) {
  switch (tile_cols) {
    case 512: return by_code(code, [&](auto k) { return launch_decompress_t<8, decltype(k)::value>(p, s, stream); });
    case 256: return by_code(code, [&](auto k) { return launch_decompress_t<4, decltype(k)::value>(p, s, stream); });
    case 128: return by_code(code, [&](auto k) { return launch_decompress_t<2, decltype(k)::value>(p, s, stream); });
    case 64: return by_code(code, [&](auto k) { return launch_decompress_t<1, decltype(k)::value>(p, s, stream); });
    default: return cudaErrorInvalidValue;
  }
}

bool tc_shape(int64_t tiles_r, int64_t tiles_c, uint64_t max_streams, uint32_t table_bytes,
              int n, int sm_count, size_t smem_limit, TcShape* out) {
  int64_t cmax = sm_count < (int)kMaxCtas ? (int64_t)sm_count : (int64_t)kMaxCtas;
  if (cmax < 1) cmax = 1;
  int64_t ks_max = tc_max_ksplit(tiles_c);
  if (ks_max > cmax) ks_max = cmax;
  const uint32_t bar_off = (uint32_t)xstage_offset(table_bytes);
  const uint32_t a_off = (bar_off + kTcBarBytes + 1023u) / 1024u * 1024u;
  const uint32_t bstage = (uint32_t)n * 128u;
  // Candidates in order of preference: two x stages (with one, a team's next x
  // chunk can only be fetched once its last MMAs completed, which serialises
  // the TMA latency with every chunk), every decode warp's streams resident
  // (full), fewest rounds, smallest split, three A stages, largest ring.
  bool found = false;
  TcShape best{};
  int64_t best_key[6] = {0, 0, 0, 0, 0, 0};
  for (int64_t KS = 1; KS <= ks_max; ++KS) {
    int64_t row_ranges = cmax / KS;
    if (row_ranges > tiles_r) row_ranges = tiles_r;
    const int64_t ctas = row_ranges * KS;
    const int64_t rows_c = (tiles_r + row_ranges - 1) / row_ranges;  // largest rectangle
    const int64_t cols_c = (tiles_c + KS - 1) / KS;
    const int64_t per_cta = rows_c * cols_c;
    const int rows_max = rows_c < 16 ? (int)rows_c : 16;
    for (int R = rows_max; R >= 1; --R) {
      int tmax = kTcDecodeWarps / R;
      if (tmax > cols_c) tmax = (int)cols_c;
      if (tmax > kTcMaxTeams) tmax = kTcMaxTeams;
      if (tmax > 512 / n) tmax = 512 / n;
      for (int TT = tmax; TT >= 1; --TT) {
        for (int SB = 2; SB >= 1; --SB) {
          for (int NA = kTcMaxAStages; NA >= 2; --NA) {
            const uint32_t b_off = a_off + (uint32_t)(NA * TT * R) * kTcStageA;
            const size_t head = b_off + (size_t)(TT * SB) * bstage;
            const size_t ring_offset = (head + 127) / 128 * 128;
            if (smem_limit < ring_offset + kRingSlack) continue;
            size_t ring = smem_limit - ring_offset - kRingSlack;
            const size_t cap = (size_t)per_cta * (size_t)max_streams;
            if (ring > cap) ring = cap;
            ring = ring / 16 * 16;
            // Deadlock-free: a team's run of R single-tile copies, one more,
            // and the wrap-around of a copy (no more than the CTA's tiles).
            int64_t need = (int64_t)R + 2;
            if (need > per_cta) need = per_cta;
            if (ring < (size_t)need * (size_t)max_streams) continue;
            // The last A stage's 16 KiB operand window stays inside shared
            // memory: the allocation is padded to cover it when the ring ends
            // earlier.
            const size_t window_end =
                (size_t)a_off + (size_t)(NA * TT * R - 1) * kTcStageA + 16384;
            size_t smem_bytes = ring_offset + ring + kRingSlack;
            if (smem_bytes < window_end) smem_bytes = window_end;
            if (smem_bytes > smem_limit) continue;
            int64_t warps_resident = (int64_t)TT * R + 2;
            if (warps_resident > per_cta) warps_resident = per_cta;
            const int64_t full = ring >= (size_t)warps_resident * (size_t)max_streams ? 1 : 0;
            const int64_t rounds = (rows_c + R - 1) / R * ((cols_c + TT - 1) / TT);
            // Larger is better: x stages, resident, -rounds, -split, A stages, ring.
            const int64_t key[6] = {SB, full, -rounds, -KS, NA, (int64_t)ring};
            bool better = !found;
            for (int k = 0; k < 6 && !better; ++k) {
              if (key[k] != best_key[k]) {
                better = key[k] > best_key[k];
                break;
              }
            }
            if (!better) continue;
            found = true;
            for (int k = 0; k < 6; ++k) best_key[k] = key[k];
            best.rows = R;
            best.teams = TT;
            best.ksplit = (int)KS;
            best.n = n;
            best.bstages = SB;
            best.astages = NA;
            best.bar_off = bar_off;
            best.a_off = a_off;
            best.b_off = b_off;
            best.s.ctas = (int)ctas;
            best.s.table_bytes = table_bytes;
            best.s.xstage_bytes = (uint32_t)(head - bar_off);
            best.s.ring_offset = ring_offset;
            best.s.ring_bytes = (int)ring;
            best.s.batch_tiles = 1;
            best.s.smem_bytes = smem_bytes;
          }
        }
      }
    }
  }
  if (found) *out = best;
  return found;
}

cudaError_t launch_gemv_tc(const TileParams& p, const CUtensorMap& tmap, int tile_cols, int code,
                           const TcShape& s, cudaStream_t stream) {
  if (p.batch < 1 || p.batch > kMaxTcRows || p.tc_teams < 1 || p.tc_teams > kTcMaxTeams ||
      p.tc_rows < 1 || p.tc_rows > 16 || p.tc_rows * p.tc_teams > kTcDecodeWarps ||
      p.tc_ksplit < 1 || s.s.ctas % p.tc_ksplit != 0 || p.tc_astages < 2 ||
      p.tc_astages > kTcMaxAStages || p.tc_bstages < 1 || p.tc_bstages > 2 ||
      p.tc_bstages > p.tc_astages ||
      (p.tc_ksplit > 1 && p.tc_ksplit > tc_max_ksplit(p.tiles_c)))
    return cudaErrorInvalidValue;
  switch (tile_cols) {
    case 512: return by_code(code, [&](auto k) { return launch_gemv_tc_t<8, decltype(k)::value>(p, tmap, s.s, stream); });
    case 256: return by_code(code, [&](auto k) { return launch_gemv_tc_t<4, decltype(k)::value>(p, tmap, s.s, stream); });
    case 128: return by_code(code, [&](auto k) { return launch_gemv_tc_t<2, decltype(k)::value>(p, tmap, s.s, stream); });
    case 64: return by_code(code, [&](auto k) { return launch_gemv_tc_t<1, decltype(k)::value>(p, tmap, s.s, stream); });
    default: return cudaErrorInvalidValue;
  }
}

template <int CP, int CODE, int S>
cudaError_t launch_gather_s(const GatherParams& g, int ctas, size_t smem, cudaStream_t stream) {
  static int configured[64] = {};
  cudaError_t e = ensure_smem(gather_kernel<CP, CODE, S>, smem, configured);
  if (e != cudaSuccess) return e;
  gather_kernel<CP, CODE, S><<<(unsigned)ctas, kGatherWarps * 32, smem, stream>>>(g);
  return cudaGetLastError();
}

template <int CP, int CODE>
cudaError_t launch_gather_t(const GatherParams& g, int ctas, size_t smem, cudaStream_t stream) {
  if constexpr (CODE == kCodeRank || CODE == kCodeEsc) {
    return launch_gather_s<CP, CODE, 1>(g, ctas, smem, stream);
  } else {
    return g.streams == 2 ? launch_gather_s<CP, CODE, 2>(g, ctas, smem, stream)
                          : launch_gather_s<CP, CODE, 1>(g, ctas, smem, stream);
  }
}

cudaError_t launch_gather(const GatherParams& g, int sm_count, cudaStream_t stream) {
  if (g.n < 1) return cudaErrorInvalidValue;
  const int64_t want = 2 * (int64_t)(sm_count > 0 ? sm_count : 1);
  const int ctas = (int)(g.n < want ? g.n : want);
  const size_t smem =
      (size_t)g.table_bytes + kGatherBarBytes + (size_t)kGatherWarps * g.stage_bytes;
  const int code = g.code;
  switch (g.tile_cols) {
    case 512: return by_code(code, [&](auto k) { return launch_gather_t<8, decltype(k)::value>(g, ctas, smem, stream); });
    case 256: return by_code(code, [&](auto k) { return launch_gather_t<4, decltype(k)::value>(g, ctas, smem, stream); });
    case 128: return by_code(code, [&](auto k) { return launch_gather_t<2, decltype(k)::value>(g, ctas, smem, stream); });
    case 64: return by_code(code, [&](auto k) { return launch_gather_t<1, decltype(k)::value>(g, ctas, smem, stream); });
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace nwc
