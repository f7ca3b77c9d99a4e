// nwc_api.cu — the C ABI declared in include/nwc.h.
//
// Host-side validation, plans and handles, device images, and kernel launches.
// Every device call runs on the caller's stream and allocates no device memory.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>

#include <cstddef>
#include <cstdlib>
#include <atomic>
#include <cstring>
#include <mutex>
#include <new>
#include <utility>
#include <vector>

#include "../../include/nwc.h"
#include "kernels.cuh"
#include "nwc_internal.h"

namespace {

using nwc::round_up;

constexpr int kMaxDevices = 64;
int g_sm_count[kMaxDevices] = {};
int g_smem_optin[kMaxDevices] = {};
std::mutex g_mu;
// Polls before a bounded wait in a kernel gives up; 0 = the kernels' default.
// Set only by nwc_test_set_wait_limit.
std::atomic<uint32_t> g_wait_limit{0};

nwc_status cuda_status(cudaError_t e) { return e == cudaSuccess ? NWC_OK : NWC_ERR_CUDA; }

// SM count and per-block opt-in shared memory of the current device (cached).
nwc_status current_device(int* dev, int* sms, size_t* smem) {
  cudaError_t e = cudaGetDevice(dev);
  if (e != cudaSuccess) return NWC_ERR_CUDA;
  if (*dev < 0 || *dev >= kMaxDevices) return NWC_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lk(g_mu);
  if (!g_sm_count[*dev]) {
    int v = 0, m = 0;
    e = cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, *dev);
    if (e == cudaSuccess)
      e = cudaDeviceGetAttribute(&m, cudaDevAttrMaxSharedMemoryPerBlockOptin, *dev);
    if (e != cudaSuccess) return NWC_ERR_CUDA;
    g_sm_count[*dev] = v;
    g_smem_optin[*dev] = m;
  }
  *sms = g_sm_count[*dev];
  *smem = (size_t)g_smem_optin[*dev];
  return NWC_OK;
}

// The code kind the kernels read for a handle, and the table bytes a CTA loads.
int code_of(const nwc_handle_s& h) {
  return h.code_kind == 1   ? nwc::kCodeRank
         : h.code_kind == 2 ? nwc::kCodeEsc
         : h.lmax <= 7      ? nwc::kCode14
                            : nwc::kCode12;
}
uint32_t table_bytes_of(const nwc_handle_s& h) {
  return nwc::device_table_bytes(h.lmax, h.code_kind == 1);
}

// Launch geometry for a handle and x-stage class on a device with `sms` SMs
// and `smem` bytes of opt-in shared memory per block.
nwc_status shape_on(const nwc_handle_s& h, int sms, size_t smem, int cls, nwc::LaunchShape* s) {
  const uint64_t typical = (h.blob_bytes - h.tiles_off) / (uint64_t)h.tiles;
  *s = nwc::launch_shape(h.tiles, h.max_chunk, typical, table_bytes_of(h), sms, smem,
                         nwc::kXStageBytes[cls]);
  if (s->smem_bytes > smem) return NWC_ERR_UNSUPPORTED;
  return NWC_OK;
}

bool same_shape(const nwc_handle_s& h, int cls, const nwc::LaunchShape& s) {
  return h.sched_ctas[cls] == s.ctas && h.sched_ring[cls] == s.ring_bytes &&
         h.sched_tiles_per_batch[cls] == s.batch_tiles;
}

void note_schedule(nwc_handle_s* h, int cls, const nwc::LaunchShape& s) {
  h->sched_ctas[cls] = s.ctas;
  h->sched_ring[cls] = s.ring_bytes;
  h->sched_tiles_per_batch[cls] = s.batch_tiles;
}

uint64_t class_off(const nwc_handle_s& h, int cls) {
  return h.sched_off + (uint64_t)cls * nwc::sched_class_bytes((uint64_t)h.tiles);
}

// Writes class cls's launch schedule for shape `s` into the device image on
// `stream` (from pageable memory: the call returns once the bytes are staged).
nwc_status write_schedule(nwc_handle_s* h, int cls, const nwc::LaunchShape& s,
                          cudaStream_t stream) {
  std::vector<uint8_t> sched;
  try {
    sched.resize(nwc::sched_class_bytes((uint64_t)h->tiles));
  } catch (const std::bad_alloc&) {
    return NWC_ERR_NOMEM;
  }
  nwc::build_schedule(h->index.data(), h->tiles, s, sched.data());
  if (cudaMemcpyAsync(h->d_base + class_off(*h, cls), sched.data(), sched.size(),
                      cudaMemcpyHostToDevice, stream) != cudaSuccess)
    return NWC_ERR_CUDA;
  note_schedule(h, cls, s);
  return NWC_OK;
}

uint64_t tc_class_off(const nwc_handle_s& h, int cls) {
  return h.sched_off + (uint64_t)nwc::kStageClasses * nwc::sched_class_bytes((uint64_t)h.tiles) +
         (uint64_t)cls * nwc::sched_tc_bytes((uint64_t)h.tiles);
}

// Tensor-core launch shape of accumulator class cls for a handle on a device
// of `sms` SMs and `smem` bytes of opt-in shared memory per block; false when
// it does not fit.
bool tc_shape_on(const nwc_handle_s& h, int sms, size_t smem, int cls, nwc::TcShape* ts) {
  const uint64_t max_streams = h.max_chunk - nwc::raw_bytes(h.tile_cols);
  return nwc::tc_shape(h.tiles_r, h.tiles_c, max_streams, table_bytes_of(h), nwc::kTcColumns[cls],
                       sms, smem, ts);
}

bool same_tc_shape(const nwc_handle_s& h, int cls, const nwc::TcShape& t) {
  return h.tc_rows[cls] == t.rows && h.tc_teams[cls] == t.teams && h.tc_ctas[cls] == t.s.ctas &&
         h.tc_ring[cls] == t.s.ring_bytes && h.tc_bstages[cls] == t.bstages &&
         h.tc_ksplit[cls] == t.ksplit && h.tc_astages[cls] == t.astages;
}

void note_tc_schedule(nwc_handle_s* h, int cls, const nwc::TcShape& t) {
  h->tc_rows[cls] = t.rows;
  h->tc_teams[cls] = t.teams;
  h->tc_ctas[cls] = t.s.ctas;
  h->tc_ring[cls] = t.s.ring_bytes;
  h->tc_bstages[cls] = t.bstages;
  h->tc_ksplit[cls] = t.ksplit;
  h->tc_astages[cls] = t.astages;
}

// Writes tensor-core schedule cls for shape t into the device image on
// `stream`, or into `image` (a host copy of the device image) when given.
nwc_status write_tc_schedule(nwc_handle_s* h, int cls, const nwc::TcShape& t, uint8_t* image,
                             cudaStream_t stream) {
  const uint32_t raw = nwc::raw_bytes(h->tile_cols);
  if (image) {
    nwc::build_tc_schedule(h->index.data(), h->tiles_r, h->tiles_c, raw, t,
                           image + tc_class_off(*h, cls));
    note_tc_schedule(h, cls, t);
    return NWC_OK;
  }
  std::vector<uint8_t> sched;
  try {
    sched.resize(nwc::sched_tc_bytes((uint64_t)h->tiles));
  } catch (const std::bad_alloc&) {
    return NWC_ERR_NOMEM;
  }
  nwc::build_tc_schedule(h->index.data(), h->tiles_r, h->tiles_c, raw, t, sched.data());
  if (cudaMemcpyAsync(h->d_base + tc_class_off(*h, cls), sched.data(), sched.size(),
                      cudaMemcpyHostToDevice, stream) != cudaSuccess)
    return NWC_ERR_CUDA;
  note_tc_schedule(h, cls, t);
  return NWC_OK;
}

// Launch geometry of class cls on the current device, which must be the
// handle's (the one current when it was made: its image lives there); rewrites
// that class's schedule (in stream order) when it was made for another shape.
nwc_status shape_for(nwc_handle_s* h, int cls, nwc::LaunchShape* s, cudaStream_t stream) {
  int dev, sms;
  size_t smem;
  nwc_status st = current_device(&dev, &sms, &smem);
  if (st != NWC_OK) return st;
  if (dev != h->device) return NWC_ERR_INVALID_ARG;
  st = shape_on(*h, sms, smem, cls, s);
  if (st != NWC_OK) return st;
  std::lock_guard<std::mutex> lk(g_mu);
  if (!same_shape(*h, cls, *s)) st = write_schedule(h, cls, *s, stream);
  return st;
}

bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

// parse_blob with host allocation failures (the index copy) reported as NOMEM:
// no C++ exception leaves the C ABI.
nwc_status parse(const uint8_t* blob, uint64_t head_bytes, uint64_t bytes, nwc_handle_s* h,
                 const uint8_t** lens) {
  // Well-defined layouts that no kernel reads: NWB1 with 4 bit streams per
  // lane (header offset 60 = S - 1), NWE1 with lmax over 7.
  if (blob && head_bytes >= 64) {
    uint32_t magic, streams_m1;
    std::memcpy(&magic, blob, 4);
    std::memcpy(&streams_m1, blob + 60, 4);
    if (magic == nwc::kMagic && streams_m1 == 3) return NWC_ERR_UNSUPPORTED;
    // NWE1 with codes longer than the kernels' 14-bit table allows.
    uint32_t lmax;
    std::memcpy(&lmax, blob + 12, 4);
    if (magic == nwc::kEscMagic && lmax > nwc::kEscMaxLmax && lmax <= (uint32_t)nwc::kMaxLmax)
      return NWC_ERR_UNSUPPORTED;
  }
  try {
    return nwc::parse_blob(blob, head_bytes, bytes, h, lens) ? NWC_OK : NWC_ERR_CORRUPT;
  } catch (const std::bad_alloc&) {
    return NWC_ERR_NOMEM;
  }
}

uint32_t* error_word(const nwc_handle_s& h) {
  return reinterpret_cast<uint32_t*>(h.d_base + h.scratch_off);
}

nwc::TileParams base_params(const nwc_handle_s& h, int cls, const nwc::LaunchShape& s) {
  nwc::TileParams p;
  std::memset(&p, 0, sizeof(p));
  p.tiles = h.d_base + h.tiles_off;
  const uint8_t* sched = h.d_base + class_off(h, cls);
  p.sched_cta = reinterpret_cast<const uint32_t*>(sched);
  p.sched_batch = reinterpret_cast<const uint4*>(sched + nwc::sched_batch_off());
  p.tile_ring = reinterpret_cast<const uint32_t*>(sched + nwc::sched_tile_off((uint64_t)h.tiles));
  p.table = reinterpret_cast<const uint32_t*>(h.d_base + h.table_off);
  p.table_bytes = table_bytes_of(h);
  p.rows = h.rows;
  p.cols = h.cols;
  p.tiles_r = h.tiles_r;
  p.tiles_c = h.tiles_c;
  p.n_tiles = h.tiles;
  p.rows_pad = 8 * h.tiles_r;
  p.ring_offset = (uint32_t)s.ring_offset;
  p.ring_bytes = s.ring_bytes;
  p.batch_tiles = s.batch_tiles;
  p.xstage_bytes = s.xstage_bytes;
  p.err = error_word(h);
  p.wait_limit = g_wait_limit.load(std::memory_order_relaxed);
  p.streams = (int32_t)h.streams;
  return p;
}

constexpr int kChunkBatch = nwc::kMaxPassRows;  // rows of x per kernel launch

// Split-K scratch one GEMV call of `batch` rows uses: the arrival counters
// (padded to 256 bytes) and the partial sums of one launch.
uint64_t scratch_bytes_for(const nwc_handle_s& h, int32_t batch, bool tensor_cores) {
  if (h.tiles_c <= 1) return 0;
  const int b = batch < kChunkBatch ? batch : kChunkBatch;
  return round_up(4ull * (uint64_t)h.tiles_r, 256) +
         (tensor_cores ? nwc::tc_partial_bytes((uint64_t)h.tiles_r, (uint64_t)h.tiles_c)
                       : nwc::split_partial_bytes((uint64_t)h.tiles_r, (uint64_t)h.tiles_c,
                                                  (uint64_t)b));
}

// Zeroes the error word and the arrival counters of a handle's scratch area.
cudaError_t clear_scratch(const nwc_handle_s& h, cudaStream_t stream) {
  return cudaMemsetAsync(h.d_base + h.scratch_off, 0,
                         nwc::scratch_partial_off((uint64_t)h.tiles_r), stream);
}

nwc_status make_handle(const uint8_t* blob_host_header_region, uint64_t bytes, void* d_buf,
                       uint64_t d_bytes, nwc_handle_t* out, const uint8_t** lens) {
  nwc_handle_s tmp;
  const nwc_status st = parse(blob_host_header_region, bytes, bytes, &tmp, lens);
  if (st != NWC_OK) return st;
  if (d_bytes < tmp.device_bytes) return NWC_ERR_INVALID_ARG;
  nwc_handle_s* h = new (std::nothrow) nwc_handle_s(std::move(tmp));
  if (!h) return NWC_ERR_NOMEM;
  h->d_base = static_cast<uint8_t*>(d_buf);
  h->d_bytes = d_bytes;
  cudaGetDevice(&h->device);
  *out = h;
  return NWC_OK;
}

// Geometry and schedules of a new handle on the current device: writes the
// schedules into `image` (a host copy of the device image) when given, else
// into the device image on `stream`.
nwc_status init_schedule(nwc_handle_s* h, uint8_t* image, cudaStream_t stream) {
  int dev, sms;
  size_t smem;
  nwc_status st = current_device(&dev, &sms, &smem);
  if (st != NWC_OK) return st;
  for (int cls = 0; cls < nwc::kStageClasses; ++cls) {
    nwc::LaunchShape s;
    st = shape_on(*h, sms, smem, cls, &s);
    if (st != NWC_OK) return st;
    if (!image) {
      st = write_schedule(h, cls, s, stream);
      if (st != NWC_OK) return st;
      continue;
    }
    nwc::build_schedule(h->index.data(), h->tiles, s, image + class_off(*h, cls));
    note_schedule(h, cls, s);
  }
  for (int cls = 0; cls < nwc::kTcClasses; ++cls) {
    nwc::TcShape ts;
    if (!tc_shape_on(*h, sms, smem, cls, &ts)) continue;
    st = write_tc_schedule(h, cls, ts, image, stream);
    if (st != NWC_OK) return st;
  }
  return NWC_OK;
}

}  // namespace

extern "C" {

int nwc_version(void) { return 100; }

const char* nwc_status_string(nwc_status s) {
  switch (s) {
    case NWC_OK: return "ok";
    case NWC_ERR_INVALID_ARG: return "invalid argument";
    case NWC_ERR_UNSUPPORTED: return "unsupported";
    case NWC_ERR_CUDA: return "CUDA runtime error";
    case NWC_ERR_CORRUPT: return "corrupt blob or device image";
    case NWC_ERR_NOMEM: return "out of memory or buffer too small";
    case NWC_ERR_DEVICE_TIMEOUT: return "device wait timed out";
    case NWC_ERR_DEVICE_CORRUPT: return "device found corrupt data";
    case NWC_ERR_SCRATCH_LIMIT: return "scratch needed exceeds the no-allocation limit";
  }
  return "unknown status";
}

nwc_status nwc_plan(const uint16_t* w_host, int64_t rows, int64_t cols, const nwc_opts* opts,
                    nwc_plan_t* out_plan) {
  if (!w_host || !out_plan || rows < 1 || cols < 1) return NWC_ERR_INVALID_ARG;
  if (rows > (1ll << 40) || cols > (1ll << 40)) return NWC_ERR_INVALID_ARG;
  *out_plan = nullptr;
  uint32_t lmax = 0, tile_rows = 8, tile_cols = 512, threads = 0, code = NWC_CODE_PREFIX;
  uint32_t streams = 1, keep = 16;
  if (opts) {
    if (opts->struct_size < offsetof(nwc_opts, code)) return NWC_ERR_INVALID_ARG;
    lmax = opts->lmax;
    tile_rows = opts->tile_rows;
    tile_cols = opts->tile_cols;
    threads = opts->threads;
    if (opts->struct_size >= offsetof(nwc_opts, streams)) code = opts->code;
    if (opts->struct_size >= offsetof(nwc_opts, keep) && opts->streams) streams = opts->streams;
    if (opts->struct_size >= sizeof(nwc_opts) && opts->keep) keep = opts->keep;
  }
  if (code != NWC_CODE_PREFIX && code != NWC_CODE_RANK && code != NWC_CODE_ESCAPE)
    return NWC_ERR_INVALID_ARG;
  if (streams != 1 && streams != 2 && streams != 4) return NWC_ERR_INVALID_ARG;
  if (code != NWC_CODE_PREFIX && streams != 1) return NWC_ERR_UNSUPPORTED;
  if (code == NWC_CODE_RANK && lmax > (uint32_t)nwc::kMaxRanks) return NWC_ERR_INVALID_ARG;
  if (code == NWC_CODE_ESCAPE && keep > 256) return NWC_ERR_INVALID_ARG;
  if (code == NWC_CODE_ESCAPE && lmax > nwc::kEscMaxLmax && lmax <= (uint32_t)nwc::kMaxLmax)
    return NWC_ERR_UNSUPPORTED;
  if (lmax > (uint32_t)nwc::kMaxLmax) return NWC_ERR_INVALID_ARG;
  if (tile_rows != 8) return NWC_ERR_UNSUPPORTED;
  if (tile_cols != 64 && tile_cols != 128 && tile_cols != 256 && tile_cols != 512)
    return NWC_ERR_UNSUPPORTED;
  nwc_plan_s* p = new (std::nothrow) nwc_plan_s();
  if (!p) return NWC_ERR_NOMEM;
  int rc;
  try {
    rc = code == NWC_CODE_RANK
             ? nwc::plan_build_rank(w_host, rows, cols, tile_cols, lmax ? lmax : nwc::kMaxRanks,
                                    threads, p)
         : code == NWC_CODE_ESCAPE
             ? nwc::plan_build_escape(w_host, rows, cols, tile_cols, lmax, keep, threads, p)
             : nwc::plan_build(w_host, rows, cols, tile_rows, tile_cols, lmax, threads, p,
                               streams);
  } catch (const std::bad_alloc&) {
    delete p;
    return NWC_ERR_NOMEM;
  }
  if (rc != 0) {
    delete p;
    return NWC_ERR_INVALID_ARG;  // too many distinct exponents for lmax, or > 64 GiB
  }
  *out_plan = p;
  return NWC_OK;
}

nwc_status nwc_plan_size(nwc_plan_t plan, uint64_t* device_bytes, uint64_t* host_blob_bytes) {
  if (!plan) return NWC_ERR_INVALID_ARG;
  if (device_bytes) *device_bytes = plan->device_bytes;
  if (host_blob_bytes) *host_blob_bytes = plan->blob_bytes;
  return NWC_OK;
}

nwc_status nwc_compress_host(nwc_plan_t plan, const uint16_t* w_host, void* blob,
                             uint64_t blob_bytes) {
  if (!plan || !w_host || !blob || blob_bytes < plan->blob_bytes) return NWC_ERR_INVALID_ARG;
  try {
    nwc::encode_blob(*plan, w_host, static_cast<uint8_t*>(blob));
  } catch (const std::bad_alloc&) {
    return NWC_ERR_NOMEM;
  }
  return NWC_OK;
}

nwc_status nwc_compress(nwc_plan_t plan, const uint16_t* w_host, void* d_buf, uint64_t d_bytes,
                        nwc_stream_t stream, nwc_handle_t* out_handle) {
  if (!plan || !w_host || !d_buf || !out_handle) return NWC_ERR_INVALID_ARG;
  *out_handle = nullptr;
  // No kernel reads these layouts yet.
  if (plan->streams > nwc::kMaxDeviceStreams || plan->device_bytes == 0)
    return NWC_ERR_UNSUPPORTED;
  if (d_bytes < plan->device_bytes || !aligned(d_buf, 256)) return NWC_ERR_INVALID_ARG;
  uint8_t* img = static_cast<uint8_t*>(std::malloc(
      plan->scratch_off + nwc::scratch_partial_off((uint64_t)plan->tiles_r)));
  if (!img) return NWC_ERR_NOMEM;
  try {
    nwc::encode_blob(*plan, w_host, img);
  } catch (const std::bad_alloc&) {
    std::free(img);
    return NWC_ERR_NOMEM;
  }
  std::memset(img + plan->blob_bytes, 0, plan->table_off - plan->blob_bytes);
  if (plan->code_kind == NWC_CODE_RANK)
    nwc::build_rank_table(plan->rank_table, plan->ranks,
                          reinterpret_cast<uint32_t*>(img + plan->table_off));
  else
    nwc::build_decode_table(plan->len, plan->lmax,
                            reinterpret_cast<uint32_t*>(img + plan->table_off));
  const uint64_t table_end =
      plan->table_off + nwc::device_table_bytes(plan->lmax, plan->code_kind == NWC_CODE_RANK);
  std::memset(img + table_end, 0, plan->sched_off - table_end);
  // The scratch area starts with the error word and the arrival counters,
  // which must be zero; the partial sums are written before they are read.
  const uint64_t scratch_head = nwc::scratch_partial_off((uint64_t)plan->tiles_r);
  std::memset(img + plan->scratch_off, 0, scratch_head);
  const uint64_t upload = plan->scratch_off + scratch_head;
  nwc_handle_t h = nullptr;
  nwc_status st = make_handle(img, plan->blob_bytes, d_buf, d_bytes, &h, nullptr);
  if (st == NWC_OK) st = init_schedule(h, img, nullptr);
  // From pageable memory the call returns once the bytes are staged, so the
  // image can be freed right after.
  if (st == NWC_OK && cudaMemcpyAsync(d_buf, img, upload, cudaMemcpyHostToDevice,
                                      reinterpret_cast<cudaStream_t>(stream)) != cudaSuccess)
    st = NWC_ERR_CUDA;
  std::free(img);
  if (st != NWC_OK) {
    delete h;
    return st;
  }
  *out_handle = h;
  return NWC_OK;
}

nwc_status nwc_blob_device_bytes(const void* blob, uint64_t blob_bytes, uint64_t* device_bytes) {
  if (!blob || !device_bytes) return NWC_ERR_INVALID_ARG;
  nwc_handle_s tmp;
  const nwc_status st = parse(static_cast<const uint8_t*>(blob), blob_bytes, blob_bytes, &tmp,
                              nullptr);
  if (st != NWC_OK) return st;
  *device_bytes = tmp.device_bytes;
  return NWC_OK;
}

nwc_status nwc_upload_blob(const void* blob, uint64_t blob_bytes, void* d_buf, uint64_t d_bytes,
                           nwc_stream_t stream, nwc_handle_t* out_handle) {
  if (!blob || !d_buf || !out_handle || !aligned(d_buf, 256)) return NWC_ERR_INVALID_ARG;
  *out_handle = nullptr;
  const uint8_t* lens = nullptr;
  nwc_handle_t h = nullptr;
  nwc_status st = make_handle(static_cast<const uint8_t*>(blob), blob_bytes, d_buf, d_bytes, &h,
                              &lens);
  if (st != NWC_OK) return st;
  std::vector<uint32_t> table;
  try {
    table.resize(table_bytes_of(*h) / 4);
  } catch (const std::bad_alloc&) {
    delete h;
    return NWC_ERR_NOMEM;
  }
  if (h->code_kind == 1)
    nwc::build_rank_table(lens, h->lmax, table.data());
  else
    nwc::build_decode_table(lens, h->lmax, table.data());
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  cudaError_t e = cudaMemcpyAsync(d_buf, blob, blob_bytes, cudaMemcpyHostToDevice, s);
  if (e == cudaSuccess && h->table_off > blob_bytes)
    e = cudaMemsetAsync(static_cast<uint8_t*>(d_buf) + blob_bytes, 0, h->table_off - blob_bytes, s);
  if (e == cudaSuccess)
    e = cudaMemcpyAsync(static_cast<uint8_t*>(d_buf) + h->table_off, table.data(),
                        table_bytes_of(*h), cudaMemcpyHostToDevice, s);
  if (e == cudaSuccess) e = clear_scratch(*h, s);
  if (e == cudaSuccess) {
    st = init_schedule(h, nullptr, s);
    if (st != NWC_OK) {
      delete h;
      return st;
    }
    e = cudaStreamSynchronize(s);
  }
  if (e != cudaSuccess) {
    delete h;
    return NWC_ERR_CUDA;
  }
  *out_handle = h;
  return NWC_OK;
}

nwc_status nwc_handle_from_device(void* d_buf, uint64_t d_bytes, nwc_handle_t* out_handle) {
  if (!d_buf || !out_handle || d_bytes < nwc::kIndexOffset) return NWC_ERR_INVALID_ARG;
  *out_handle = nullptr;
  nwc::BlobHeader hd;
  if (cudaMemcpy(&hd, d_buf, sizeof(hd), cudaMemcpyDeviceToHost) != cudaSuccess)
    return NWC_ERR_CUDA;
  if (hd.magic == nwc::kMagic && hd.zero == 3) return NWC_ERR_UNSUPPORTED;
  if ((hd.magic != nwc::kMagic && hd.magic != nwc::kRankMagic && hd.magic != nwc::kEscMagic) ||
      hd.total_bytes > d_bytes ||
      hd.tiles_off > hd.total_bytes ||
      hd.tiles_off < nwc::kIndexOffset)
    return NWC_ERR_CORRUPT;
  // Header, lens and index; the tile area is not read back.
  std::vector<uint8_t> head;
  try {
    head.resize(hd.tiles_off);
  } catch (const std::bad_alloc&) {
    return NWC_ERR_NOMEM;
  }
  if (cudaMemcpy(head.data(), d_buf, hd.tiles_off, cudaMemcpyDeviceToHost) != cudaSuccess)
    return NWC_ERR_CUDA;
  nwc_handle_s tmp;
  nwc_status st = parse(head.data(), head.size(), hd.total_bytes, &tmp, nullptr);
  if (st != NWC_OK) return st;
  if (d_bytes < tmp.device_bytes) return NWC_ERR_INVALID_ARG;
  nwc_handle_s* h = new (std::nothrow) nwc_handle_s(std::move(tmp));
  if (!h) return NWC_ERR_NOMEM;
  h->d_base = static_cast<uint8_t*>(d_buf);
  h->d_bytes = d_bytes;
  cudaGetDevice(&h->device);
  st = init_schedule(h, nullptr, nullptr);
  if (st == NWC_OK && clear_scratch(*h, nullptr) != cudaSuccess) st = NWC_ERR_CUDA;
  if (st == NWC_OK && cudaStreamSynchronize(nullptr) != cudaSuccess) st = NWC_ERR_CUDA;
  if (st != NWC_OK) {
    delete h;
    return st;
  }
  *out_handle = h;
  return NWC_OK;
}

nwc_status nwc_decompress(nwc_handle_t h, uint16_t* d_w_out, nwc_stream_t stream) {
  if (!h || !d_w_out || !aligned(d_w_out, 4)) return NWC_ERR_INVALID_ARG;
  nwc::LaunchShape s;
  nwc_status st = shape_for(h, 0, &s, reinterpret_cast<cudaStream_t>(stream));
  if (st != NWC_OK) return st;
  nwc::TileParams p = base_params(*h, 0, s);
  p.out = d_w_out;
  return cuda_status(nwc::launch_decompress(p, (int)h->tile_cols, code_of(*h), s,
                                            reinterpret_cast<cudaStream_t>(stream)));
}

nwc_status nwc_gather_rows(nwc_handle_t h, const int32_t* d_rows, int32_t n, uint16_t* d_out,
                           nwc_stream_t stream) {
  if (!h || !d_rows || !d_out || n < 1 || n > (1 << 20) || !aligned(d_rows, 4) ||
      !aligned(d_out, 2))
    return NWC_ERR_INVALID_ARG;
  int dev = -1, sms = 0;
  size_t smem = 0;
  nwc_status st = current_device(&dev, &sms, &smem);
  if (st != NWC_OK) return st;
  if (dev != h->device) return NWC_ERR_INVALID_ARG;
  nwc::GatherParams g;
  std::memset(&g, 0, sizeof(g));
  g.tiles = h->d_base + h->tiles_off;
  g.index = reinterpret_cast<const uint32_t*>(h->d_base + h->index_off);
  g.table = reinterpret_cast<const uint32_t*>(h->d_base + h->table_off);
  g.table_bytes = table_bytes_of(*h);
  // Lane lengths and the longest streams a tile can hold, plus the readers'
  // slack.
  const uint32_t max_chunk = h->code_kind == 1   ? nwc::max_rank_chunk_bytes(h->tile_cols, h->lmax)
                             : h->code_kind == 2 ? nwc::max_escape_chunk_bytes(h->tile_cols, h->lmax)
                                                 : nwc::max_chunk_bytes(h->tile_cols, h->lmax,
                                                                        h->streams);
  g.stage_bytes = max_chunk - nwc::raw_bytes(h->tile_cols) + 512;
  if ((size_t)g.table_bytes + 8ull * g.stage_bytes > smem) return NWC_ERR_UNSUPPORTED;
  g.peek = nwc::peek_bits(h->lmax);
  g.streams = (int32_t)h->streams;
  g.code = code_of(*h);
  g.tile_cols = (int32_t)h->tile_cols;
  g.rows = h->rows;
  g.cols = h->cols;
  g.tiles_r = h->tiles_r;
  g.tiles_c = h->tiles_c;
  g.row_ids = d_rows;
  g.n = n;
  g.out = d_out;
  g.err = error_word(*h);
  return cuda_status(nwc::launch_gather(g, sms, reinterpret_cast<cudaStream_t>(stream)));
}

nwc_status nwc_gemv_scratch_bytes(nwc_handle_t h, int32_t batch, uint64_t* bytes) {
  if (!h || !bytes || batch < 1 || batch > 64) return NWC_ERR_INVALID_ARG;
  *bytes = scratch_bytes_for(*h, batch, batch >= h->tc_min_batch && h->tc_min_batch > 0 &&
                                              h->tc_rows[nwc::tc_class(batch)] > 0 &&
                                              (h->cols % 8) == 0);
  return NWC_OK;
}

}  // extern "C"

namespace {

// Checks shared by the GEMV entry points, done before anything is enqueued.
nwc_status gemv_check(const nwc_handle_s* h, const uint16_t* d_x, const float* d_y,
                      int32_t batch) {
  if (!h || !d_x || !d_y || batch < 1 || batch > 64) return NWC_ERR_INVALID_ARG;
  // x is read in BF16 pairs (4-byte words) unless cols is odd.
  if (!aligned(d_x, (h->cols & 1) ? 2 : 4) || !aligned(d_y, 4)) return NWC_ERR_INVALID_ARG;
  // A filler exponent of 255 (Inf/NaN) in padded columns would meet x = 0
  // (the ranked code's filler, e with raw byte 0, is always finite).
  if (h->code_kind != 1 && h->filler == 255 && (h->cols % (int64_t)h->tile_cols) != 0)
    return NWC_ERR_UNSUPPORTED;
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess) return NWC_ERR_CUDA;
  if (dev != h->device) return NWC_ERR_INVALID_ARG;
  return NWC_OK;
}

// cuTensorMapEncodeTiled from the driver, looked up once.
PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* f = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(f);
  });
  return fn;
}

// Whether a GEMV of `batch` rows takes the tensor-core kernel: at or above the
// handle's threshold, when its shape fits this device and x can be read by TMA
// (16-byte aligned rows).
bool use_tensor_cores(const nwc_handle_s& h, const uint16_t* d_x, int32_t batch) {
  return h.tc_min_batch > 0 && batch >= h.tc_min_batch && batch <= nwc::kMaxTcRows &&
         h.tc_rows[nwc::tc_class(batch)] > 0 && (h.cols % 8) == 0 && aligned(d_x, 16);
}

// The tensor-core launch: one kernel for up to 64 rows of x, every weight
// decoded once.
nwc_status gemv_run_tc(nwc_handle_s* h, const uint16_t* d_x, float* d_y, int32_t batch,
                       uint32_t* counters, float* partial, cudaStream_t cs) {
  int dev, sms;
  size_t smem;
  nwc_status st = current_device(&dev, &sms, &smem);
  if (st != NWC_OK) return st;
  const int cls = nwc::tc_class(batch);
  nwc::TcShape ts;
  if (!tc_shape_on(*h, sms, smem, cls, &ts)) return NWC_ERR_UNSUPPORTED;
  {
    std::lock_guard<std::mutex> lk(g_mu);
    if (!same_tc_shape(*h, cls, ts)) {
      st = write_tc_schedule(h, cls, ts, nullptr, cs);
      if (st != NWC_OK) return st;
    }
  }
  PFN_cuTensorMapEncodeTiled_v12000 encode = tensor_map_encoder();
  if (!encode) return NWC_ERR_UNSUPPORTED;
  const int n = nwc::kTcColumns[cls];
  CUtensorMap tmap;
  const cuuint64_t dims[2] = {(cuuint64_t)h->cols, (cuuint64_t)batch};
  const cuuint64_t strides[1] = {(cuuint64_t)h->cols * 2};
  const cuuint32_t box[2] = {64, (cuuint32_t)n};
  const cuuint32_t elem[2] = {1, 1};
  if (encode(&tmap, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<uint16_t*>(d_x), dims, strides,
             box, elem, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
    return NWC_ERR_UNSUPPORTED;
  nwc::TileParams p;
  std::memset(&p, 0, sizeof(p));
  const uint8_t* sched = h->d_base + tc_class_off(*h, cls);
  p.tiles = h->d_base + h->tiles_off;
  p.index = reinterpret_cast<const uint32_t*>(h->d_base + h->index_off);
  p.sched_cta = reinterpret_cast<const uint32_t*>(sched);
  p.sched_batch = reinterpret_cast<const uint4*>(sched + nwc::sched_batch_off());
  p.tile_ring = reinterpret_cast<const uint32_t*>(sched + nwc::sched_tc_ring_off((uint64_t)h->tiles));
  p.tile_batch =
      reinterpret_cast<const uint32_t*>(sched + nwc::sched_tc_tbatch_off((uint64_t)h->tiles));
  p.table = reinterpret_cast<const uint32_t*>(h->d_base + h->table_off);
  p.table_bytes = table_bytes_of(*h);
  p.rows = h->rows;
  p.cols = h->cols;
  p.tiles_r = h->tiles_r;
  p.tiles_c = h->tiles_c;
  p.n_tiles = h->tiles;
  p.rows_pad = 8 * h->tiles_r;
  p.ring_offset = (uint32_t)ts.s.ring_offset;
  p.ring_bytes = ts.s.ring_bytes;
  p.batch_tiles = ts.s.batch_tiles;
  p.xstage_bytes = ts.s.xstage_bytes;
  p.err = error_word(*h);
  p.wait_limit = g_wait_limit.load(std::memory_order_relaxed);
  p.streams = (int32_t)h->streams;
  p.x = d_x;
  p.y = d_y;
  p.batch = batch;
  p.counters = counters;
  p.partial = partial;
  p.tc_rows = ts.rows;
  p.tc_teams = ts.teams;
  p.tc_n = n;
  p.tc_bstages = ts.bstages;
  p.tc_ksplit = ts.ksplit;
  p.tc_astages = ts.astages;
  uint32_t cols = 32;
  while (cols < (uint32_t)(ts.teams * n)) cols <<= 1;
  p.tc_tmem_cols = cols;
  p.tc_bar_off = ts.bar_off;
  p.tc_a_off = ts.a_off;
  p.tc_b_off = ts.b_off;
  return cuda_status(nwc::launch_gemv_tc(p, tmap, (int)h->tile_cols, code_of(*h), ts, cs));
}

// The GEMV launches, with split-K scratch at `counters` (u32 [tiles_r], zero
// on entry and left zero) and `partial` (scratch_bytes_for bytes less the
// counters' 256-byte-padded area).
nwc_status gemv_run(nwc_handle_s* h, const uint16_t* d_x, float* d_y, int32_t batch,
                    uint32_t* counters, float* partial, cudaStream_t cs) {
  if (use_tensor_cores(*h, d_x, batch)) return gemv_run_tc(h, d_x, d_y, batch, counters, partial, cs);
  for (int32_t b0 = 0; b0 < batch; b0 += kChunkBatch) {
    const int32_t nb = batch - b0 < kChunkBatch ? batch - b0 : kChunkBatch;
    // The x-stage class (and with it the schedule and ring) follows the rows
    // of x this launch handles.
    const int cls = nwc::stage_class(nb);
    nwc::LaunchShape s;
    nwc_status st = shape_for(h, cls, &s, cs);
    if (st != NWC_OK) return st;
    nwc::TileParams p = base_params(*h, cls, s);
    p.counters = counters;
    p.partial = partial;
    p.x = d_x + (int64_t)b0 * h->cols;
    p.y = d_y + (int64_t)b0 * h->rows;
    p.batch = nb;
    cudaError_t e = nwc::launch_gemv(p, (int)h->tile_cols, code_of(*h), s, cs);
    if (e != cudaSuccess) return NWC_ERR_CUDA;
  }
  return NWC_OK;
}

// Scratch of nwc_gemv_noalloc: a fixed array that lives as long as the module,
// one copy per device.  Host code must not hand `g_noalloc_scratch` itself to a
// kernel (on the host that name is a stand-in, not a device address); the
// device address comes from cudaGetSymbolAddress, looked up once per device.
__device__ __align__(256) unsigned char g_noalloc_scratch[NWC_NOALLOC_SCRATCH_BYTES];
void* g_noalloc_addr[kMaxDevices] = {};

nwc_status noalloc_scratch(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return NWC_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return NWC_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lk(g_mu);
  if (!g_noalloc_addr[dev]) {
    void* addr = nullptr;
    if (cudaGetSymbolAddress(&addr, g_noalloc_scratch) != cudaSuccess || !addr)
      return NWC_ERR_CUDA;
    g_noalloc_addr[dev] = addr;
  }
  *out = g_noalloc_addr[dev];
  return NWC_OK;
}

}  // namespace

extern "C" {

nwc_status nwc_gemv(nwc_handle_t h, const uint16_t* d_x, float* d_y, int32_t batch,
                    nwc_stream_t stream) {
  nwc_status st = gemv_check(h, d_x, d_y, batch);
  if (st != NWC_OK) return st;
  uint8_t* scratch = h->d_base + h->scratch_off;
  return gemv_run(h, d_x, d_y, batch,
                  reinterpret_cast<uint32_t*>(scratch + nwc::kScratchCountersOff),
                  reinterpret_cast<float*>(scratch + nwc::scratch_partial_off((uint64_t)h->tiles_r)),
                  reinterpret_cast<cudaStream_t>(stream));
}

nwc_status nwc_gemv_noalloc(nwc_handle_t h, const uint16_t* d_x, float* d_y, int32_t batch,
                            nwc_stream_t stream) {
  // Every argument is checked before the shared array is touched, so a
  // rejected call enqueues nothing.
  nwc_status st = gemv_check(h, d_x, d_y, batch);
  if (st != NWC_OK) return st;
  const uint64_t need = scratch_bytes_for(*h, batch, use_tensor_cores(*h, d_x, batch));
  if (need > NWC_NOALLOC_SCRATCH_BYTES) return NWC_ERR_SCRATCH_LIMIT;
  uint8_t* ws = nullptr;
  if (need) {
    void* addr = nullptr;
    st = noalloc_scratch(&addr);
    if (st != NWC_OK) return st;
    ws = static_cast<uint8_t*>(addr);
    // The array keeps the previous call's bytes: the arrival counters must
    // start at zero, the partial sums are overwritten before they are read.
    if (cudaMemsetAsync(ws, 0, 4ull * (uint64_t)h->tiles_r,
                        reinterpret_cast<cudaStream_t>(stream)) != cudaSuccess)
      return NWC_ERR_CUDA;
  }
  return gemv_run(h, d_x, d_y, batch, reinterpret_cast<uint32_t*>(ws),
                  ws ? reinterpret_cast<float*>(ws + round_up(4ull * (uint64_t)h->tiles_r, 256))
                     : nullptr,
                  reinterpret_cast<cudaStream_t>(stream));
}

nwc_status nwc_handle_info(nwc_handle_t h, int64_t* rows, int64_t* cols, uint64_t* blob_bytes,
                           uint64_t* device_bytes, uint64_t* compressed_bytes) {
  if (!h) return NWC_ERR_INVALID_ARG;
  if (rows) *rows = h->rows;
  if (cols) *cols = h->cols;
  if (blob_bytes) *blob_bytes = h->blob_bytes;
  if (device_bytes) *device_bytes = h->device_bytes;
  if (compressed_bytes) *compressed_bytes = h->scratch_off;
  return NWC_OK;
}

nwc_status nwc_get_device_error(nwc_handle_t h, nwc_stream_t stream, uint32_t* word) {
  if (!h) return NWC_ERR_INVALID_ARG;
  cudaStream_t cs = reinterpret_cast<cudaStream_t>(stream);
  uint32_t w = 0;
  cudaError_t e = cudaMemcpyAsync(&w, error_word(*h), sizeof(w), cudaMemcpyDeviceToHost, cs);
  if (e == cudaSuccess) e = cudaStreamSynchronize(cs);
  if (e != cudaSuccess) return NWC_ERR_CUDA;
  // A kernel that gave up may have left arrival counters behind: clear them
  // with the word so that the next call starts from zero.
  if (w && (clear_scratch(*h, cs) != cudaSuccess || cudaStreamSynchronize(cs) != cudaSuccess))
    return NWC_ERR_CUDA;
  if (word) *word = w;
  if (w & nwc::kErrTimeout) return NWC_ERR_DEVICE_TIMEOUT;
  if (w & nwc::kErrCorrupt) return NWC_ERR_DEVICE_CORRUPT;
  if (w & nwc::kErrRange) return NWC_ERR_INVALID_ARG;
  if (w & nwc::kErrLayout) return NWC_ERR_UNSUPPORTED;
  return NWC_OK;
}

nwc_status nwc_gemv_set_tc_min_batch(nwc_handle_t h, int32_t min_batch) {
  if (!h || min_batch < 0 || min_batch > nwc::kMaxTcRows) return NWC_ERR_INVALID_ARG;
  h->tc_min_batch = min_batch;
  return NWC_OK;
}

nwc_status nwc_gemv_path(nwc_handle_t h, const uint16_t* d_x, int32_t batch, int32_t* launches,
                         int32_t* tensor_cores) {
  if (!h || batch < 1 || batch > 64) return NWC_ERR_INVALID_ARG;
  const bool tc = use_tensor_cores(*h, d_x, batch);
  if (launches) *launches = tc ? 1 : (batch + kChunkBatch - 1) / kChunkBatch;
  if (tensor_cores) *tensor_cores = tc ? 1 : 0;
  return NWC_OK;
}

void nwc_test_set_wait_limit(uint32_t polls) {
  g_wait_limit.store(polls, std::memory_order_relaxed);
}

nwc_status nwc_schedule_describe(const void* blob, uint64_t blob_bytes, int32_t sm_count,
                                 uint64_t smem_limit, int32_t rows_of_x, nwc_schedule_info* info,
                                 uint32_t* cta_batch, uint32_t* batch, uint32_t* tile_ring) {
  if (!blob || !info || info->struct_size < sizeof(nwc_schedule_info) || sm_count < 1 ||
      rows_of_x < 0 || rows_of_x > nwc::kMaxPassRows)
    return NWC_ERR_INVALID_ARG;
  nwc_handle_s h;
  nwc_status st = parse(static_cast<const uint8_t*>(blob), blob_bytes, blob_bytes, &h, nullptr);
  if (st != NWC_OK) return st;
  const int cls = nwc::stage_class(rows_of_x);
  nwc::LaunchShape s;
  st = shape_on(h, sm_count, (size_t)smem_limit, cls, &s);
  if (st != NWC_OK) return st;
  std::vector<uint8_t> sched;
  try {
    sched.resize(nwc::sched_class_bytes((uint64_t)h.tiles));
  } catch (const std::bad_alloc&) {
    return NWC_ERR_NOMEM;
  }
  nwc::build_schedule(h.index.data(), h.tiles, s, sched.data());
  const uint32_t* cb = reinterpret_cast<const uint32_t*>(sched.data());
  info->ctas = s.ctas;
  info->batch_tiles = s.batch_tiles;
  info->ring_bytes = s.ring_bytes;
  info->tiles = h.tiles;
  info->batches = cb[s.ctas];
  info->smem_bytes = s.smem_bytes;
  info->xstage_bytes = s.xstage_bytes;
  if (cta_batch) std::memcpy(cta_batch, cb, 4 * ((size_t)s.ctas + 1));
  if (batch)
    std::memcpy(batch, sched.data() + nwc::sched_batch_off(), 16 * (size_t)cb[s.ctas]);
  if (tile_ring)
    std::memcpy(tile_ring, sched.data() + nwc::sched_tile_off((uint64_t)h.tiles),
                4 * (size_t)h.tiles);
  return NWC_OK;
}

nwc_status nwc_tc_schedule_describe(const void* blob, uint64_t blob_bytes, int32_t sm_count,
                                    uint64_t smem_limit, int32_t rows_of_x,
                                    nwc_tc_schedule_info* info, uint32_t* cta_batch,
                                    uint32_t* batch, uint32_t* tile_ring, uint32_t* tile_batch) {
  if (!blob || !info || info->struct_size < sizeof(nwc_tc_schedule_info) || sm_count < 1 ||
      rows_of_x < 1 || rows_of_x > nwc::kMaxTcRows)
    return NWC_ERR_INVALID_ARG;
  nwc_handle_s h;
  nwc_status st = parse(static_cast<const uint8_t*>(blob), blob_bytes, blob_bytes, &h, nullptr);
  if (st != NWC_OK) return st;
  nwc::TcShape ts;
  if (!tc_shape_on(h, sm_count, (size_t)smem_limit, nwc::tc_class(rows_of_x), &ts))
    return NWC_ERR_UNSUPPORTED;
  std::vector<uint8_t> sched;
  try {
    sched.resize(nwc::sched_tc_bytes((uint64_t)h.tiles));
  } catch (const std::bad_alloc&) {
    return NWC_ERR_NOMEM;
  }
  nwc::build_tc_schedule(h.index.data(), h.tiles_r, h.tiles_c, nwc::raw_bytes(h.tile_cols), ts,
                         sched.data());
  const uint32_t* cb = reinterpret_cast<const uint32_t*>(sched.data());
  info->ctas = ts.s.ctas;
  info->rows = ts.rows;
  info->teams = ts.teams;
  info->batch_tiles = ts.s.batch_tiles;
  info->ring_bytes = ts.s.ring_bytes;
  info->n = ts.n;
  info->x_stages = ts.bstages;
  info->ksplit = ts.ksplit;
  info->a_stages = ts.astages;
  info->tiles = h.tiles;
  info->batches = cb[ts.s.ctas];
  info->smem_bytes = ts.s.smem_bytes;
  info->a_offset = ts.a_off;
  info->b_offset = ts.b_off;
  info->ring_offset = ts.s.ring_offset;
  const uint64_t tiles = (uint64_t)h.tiles;
  if (cta_batch) std::memcpy(cta_batch, cb, 4 * ((size_t)ts.s.ctas + 1));
  if (batch) std::memcpy(batch, sched.data() + nwc::sched_batch_off(), 16 * (size_t)cb[ts.s.ctas]);
  if (tile_ring) std::memcpy(tile_ring, sched.data() + nwc::sched_tc_ring_off(tiles), 4 * tiles);
  if (tile_batch)
    std::memcpy(tile_batch, sched.data() + nwc::sched_tc_tbatch_off(tiles), 4 * tiles);
  return NWC_OK;
}

void nwc_plan_destroy(nwc_plan_t plan) { delete plan; }
void nwc_handle_destroy(nwc_handle_t h) { delete h; }

}  // extern "C"
