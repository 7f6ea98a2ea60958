// Host-side argument checks and derived constants shared by the C-ABI entry
// points (mla_api.cu and no_alloc.cu), so that every entry point applies the
// same shape, cache and alignment rules and the same softmax scale.
#pragma once

#include <math.h>
#include <stdint.h>

#include <mutex>

#include <cuda_runtime.h>

#include "mla.h"

namespace mla {
namespace api {

inline bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15) == 0; }
inline bool aligned4(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 3) == 0; }

// Sizes accepted by every call: any small shape in fp32, the DeepSeek-V2
// attention sizes in bf16 (n_heads 128, d_c 512, d_rope 64, d_nope = d_v = 128,
// 64-row pages).
inline mla_status check_dims(const mla_dims *d) {
  if (!d) return MLA_ERR_INVALID_ARG;
  if (d->n_heads < 1 || d->d_c < 1 || d->d_nope < 1 || d->d_v < 1 || d->page_size < 1)
    return MLA_ERR_INVALID_ARG;
  if (d->d_rope < 2 || (d->d_rope & 1) || d->d_rope > 128) return MLA_ERR_INVALID_ARG;
  if (d->dtype != MLA_BF16 && d->dtype != MLA_FP32) return MLA_ERR_INVALID_ARG;
  if (d->rope_layout != MLA_ROPE_INTERLEAVED && d->rope_layout != MLA_ROPE_HALF)
    return MLA_ERR_INVALID_ARG;
  if (!(d->rope_base > 0.0) || !(d->rms_eps >= 0.0) || !(d->softmax_scale >= 0.0))
    return MLA_ERR_INVALID_ARG;
  if (d->cache_format != MLA_CACHE_NATIVE && d->cache_format != MLA_CACHE_INT8)
    return MLA_ERR_INVALID_ARG;
  if (d->cache_format == MLA_CACHE_INT8 && d->dtype != MLA_BF16) return MLA_ERR_UNSUPPORTED;
  if (d->dtype == MLA_FP32) {
    if (d->n_heads > 256 || d->d_c > 1024 || (d->d_c % 4) || d->d_nope > 256 || d->d_v > 256)
      return MLA_ERR_UNSUPPORTED;
  } else {
    if (d->n_heads != 128 || d->d_c != 512 || d->d_rope != 64 || d->d_nope != 128 ||
        d->d_v != 128 || d->page_size != 64)
      return MLA_ERR_UNSUPPORTED;
  }
  return MLA_OK;
}

inline mla_status check_cache(const mla_paged_cache *c) {
  if (!c || !c->pool || !c->block_table || c->num_pages < 1 || c->max_pages_per_seq < 1)
    return MLA_ERR_INVALID_ARG;
  if (!aligned16(c->pool) || !aligned4(c->block_table)) return MLA_ERR_ALIGNMENT;
  return MLA_OK;
}

// The arguments both decode-attention entry points share (everything but the
// workspace): dims, cache, batch, q_lat, z, lse, num_splits.
inline mla_status check_attn_args(const mla_dims *dims, const mla_paged_cache *cache, int batch,
                                  const void *q_lat, const void *z, const float *lse,
                                  int num_splits) {
  mla_status st = check_dims(dims);
  if (st != MLA_OK) return st;
  st = check_cache(cache);
  if (st != MLA_OK) return st;
  if (batch < 1 || !q_lat || !z || !cache->seq_lens || num_splits < 0) return MLA_ERR_INVALID_ARG;
  if (!aligned16(q_lat) || !aligned16(z) || (lse && !aligned4(lse)) || !aligned4(cache->seq_lens))
    return MLA_ERR_ALIGNMENT;
  return MLA_OK;
}

// 1/sqrt(d_nope + d_rope) unless the caller gives a scale ("从零理解 MLA",
// 解耦 RoPE: the score is divided by sqrt(d_head + d_r)).
inline float softmax_scale(const mla_dims &d) {
  return d.softmax_scale > 0 ? (float)d.softmax_scale
                             : (float)(1.0 / sqrt((double)(d.d_nope + d.d_rope)));
}

// Raises a kernel's dynamic shared-memory limit once per device (the attribute
// is per device, so a process that uses several GPUs sets it on each).
class PerDeviceOnce {
 public:
  template <class F>
  cudaError_t run(F &&f) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> guard(lock_);
    if (done_[dev]) return cudaSuccess;
    e = f();
    if (e == cudaSuccess) done_[dev] = true;
    return e;
  }

 private:
  static constexpr int kMaxDevices = 64;
  std::mutex lock_;
  bool done_[kMaxDevices] = {};
};

}  // namespace api
}  // namespace mla
