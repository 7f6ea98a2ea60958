// mla_decode_attn_noalloc: decode attention for callers that cannot allocate
// device memory.
//
// Some callers have no way to hand this library a workspace: a host program
// whose device memory is fully owned by another allocator (a framework's
// caching pool that may not be bypassed, or a fixed arena reserved at start-up),
// or a plugin / custom-operator interface that passes in only the tensors of
// the operation and forbids allocation while it runs.  For them this entry
// point keeps its scratch (plan arrays, split-KV partials, error word) in one
// file-scope device array of fixed size, kMaxScratchBytes.  Every GPU on which
// the library is loaded holds that array until the process exits.
//
// The array's name in host code is only a host-side stand-in, so its device
// address is looked up once per device (cudaGetSymbolAddress, with that
// device current) on the first call made on that device, and that address is
// what the kernels receive.  Make the first call on each device before any
// stream capture.  All calls share the one array: two calls whose work
// overlaps on the GPU (different streams, or different host threads on the
// same device) race on it and must be serialised by the caller.
//
// The error word of the scratch is cleared at the start of each call and
// records what the device saw during it (a page entry, length or position out
// of range, or a bounded wait that gave up); mla_noalloc_get_device_error waits
// for the stream and reads and clears it.
#include <cuda_runtime.h>
#include <math.h>

#include <mutex>

#include "api_checks.h"
#include "common.cuh"
#include "kernels.h"
#include "mla.h"
#include "sm100.h"

namespace {

using namespace mla;

constexpr size_t kMaxScratchBytes = 16u << 20;  // 16 MiB per device
constexpr int kMaxDevices = 64;

__device__ __align__(256) unsigned char g_scratch[kMaxScratchBytes];

std::mutex g_lock;
void *g_scratch_ptr[kMaxDevices] = {};

size_t up256(size_t x) { return (x + 255) & ~size_t(255); }

// Scratch regions inside the static array (byte offsets).
struct Regions {
  size_t err, hdr, seq_start, part_base, bad, part_O, part_m, part_l, total;
};

Regions regions(int batch, int n_heads, int d_c, int parts) {
  Regions r{};
  r.err = 0;
  r.hdr = 64;
  size_t off = 256;
  r.seq_start = off; off = up256(off + sizeof(int) * (batch + 1));
  r.part_base = off; off = up256(off + sizeof(int) * batch);
  r.bad = off; off = up256(off + sizeof(int) * batch);
  const size_t slots = 2 * (size_t)parts + 2;
  r.part_O = off; off = up256(off + sizeof(float) * slots * n_heads * d_c);
  r.part_m = off; off = up256(off + sizeof(float) * slots * n_heads);
  r.part_l = off; off = up256(off + sizeof(float) * slots * n_heads);
  r.total = off;
  return r;
}

// Device address of g_scratch on the current device (looked up once per device).
mla_status scratch_address(void **out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return MLA_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return MLA_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> guard(g_lock);
  if (!g_scratch_ptr[dev]) {
    void *p = nullptr;
    if (cudaGetSymbolAddress(&p, g_scratch) != cudaSuccess || !p) return MLA_ERR_CUDA;
    g_scratch_ptr[dev] = p;
  }
  *out = g_scratch_ptr[dev];
  return MLA_OK;
}

}  // namespace

extern "C" mla_status mla_decode_attn_noalloc(const mla_dims *dims, const mla_paged_cache *cache,
                                              int batch, const void *q_lat, void *z, float *lse,
                                              int num_splits, mla_stream_t stream) {
  // the same argument rules as mla_decode_attn
  const mla_status chk = api::check_attn_args(dims, cache, batch, q_lat, z, lse, num_splits);
  if (chk != MLA_OK) return chk;
  const mla_dims &d = *dims;

  // partitions: as requested, or (0) the most that fit, at most one per SM pair
  int parts = num_splits;
  if (parts == 0) {
    int dev = 0, sms = 148;
    if (cudaGetDevice(&dev) == cudaSuccess)
      cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    parts = sms / 2 > 0 ? sms / 2 : 1;
    while (parts > 1 && regions(batch, d.n_heads, d.d_c, parts).total > kMaxScratchBytes) --parts;
  }
  const Regions R = regions(batch, d.n_heads, d.d_c, parts);
  if (R.total > kMaxScratchBytes) return MLA_ERR_WORKSPACE;  // beyond the fixed scratch

  void *base = nullptr;
  const mla_status st = scratch_address(&base);
  if (st != MLA_OK) return st;
  char *ws = static_cast<char *>(base);
  cudaStream_t s = (cudaStream_t)stream;
  // the error word and plan header must start at zero; the rest is written
  // before it is read
  if (cudaMemsetAsync(ws, 0, 256, s) != cudaSuccess) return MLA_ERR_CUDA;

  PlanArgs pa{};
  pa.seq_lens = cache->seq_lens;
  pa.batch = batch;
  pa.page_size = d.page_size;
  pa.max_pages = cache->max_pages_per_seq;
  pa.parts_max = parts;
  pa.min_pages = d.dtype == MLA_BF16 ? sm100::kAttnMinPages : 1;
  pa.gap = d.dtype == MLA_BF16 ? sm100::kAttnSeqGap : 0;
  pa.hdr = reinterpret_cast<PlanHeader *>(ws + R.hdr);
  pa.seq_start = reinterpret_cast<int *>(ws + R.seq_start);
  pa.part_base = reinterpret_cast<int *>(ws + R.part_base);
  pa.bad = reinterpret_cast<int *>(ws + R.bad);
  pa.err = reinterpret_cast<int *>(ws + R.err);
  if (launch_plan(pa, s) != cudaSuccess) return MLA_ERR_CUDA;

  AttnArgs a{};
  a.q_lat = q_lat;
  a.pool = cache->pool;
  a.block_table = cache->block_table;
  a.seq_lens = cache->seq_lens;
  a.z = z;
  a.lse = lse;
  a.batch = batch;
  a.n_heads = d.n_heads;
  a.d_c = d.d_c;
  a.d_rope = d.d_rope;
  a.page_size = d.page_size;
  a.num_pages = cache->num_pages;
  a.max_pages = cache->max_pages_per_seq;
  a.scale = api::softmax_scale(d);
  a.hdr = pa.hdr;
  a.seq_start = pa.seq_start;
  a.part_base = pa.part_base;
  a.bad = pa.bad;
  a.part_O = reinterpret_cast<float *>(ws + R.part_O);
  a.part_m = reinterpret_cast<float *>(ws + R.part_m);
  a.part_l = reinterpret_cast<float *>(ws + R.part_l);
  a.err = pa.err;
  a.int8_rows = d.cache_format == MLA_CACHE_INT8;
  cudaError_t e;
  if (d.dtype == MLA_FP32) {
    e = launch_attn_simt<float>(a, parts, s);
    if (e == cudaSuccess) e = launch_combine<float>(a, s);
  } else {
    e = sm100::launch_attn(a, parts, s);
    if (e == cudaSuccess) e = launch_combine<__nv_bfloat16>(a, s);
  }
  return e == cudaSuccess ? MLA_OK : MLA_ERR_CUDA;
}

extern "C" mla_status mla_noalloc_get_device_error(mla_stream_t stream) {
  void *base = nullptr;
  const mla_status st = scratch_address(&base);
  if (st != MLA_OK) return st;
  if (cudaStreamSynchronize((cudaStream_t)stream) != cudaSuccess) return MLA_ERR_CUDA;
  int word = 0;
  if (cudaMemcpy(&word, base, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess)
    return MLA_ERR_CUDA;
  const int zero = 0;
  if (cudaMemcpy(base, &zero, sizeof(int), cudaMemcpyHostToDevice) != cudaSuccess)
    return MLA_ERR_CUDA;
  if (word & kErrTimeout) return MLA_ERR_TIMEOUT;
  if (word & kErrRange) return MLA_ERR_DEVICE_RANGE;
  return MLA_OK;
}
