// Host side of the C ABI declared in include/mla.h: argument checks,
// workspace layout and kernel dispatch.  No call here allocates device
// memory or synchronises, except mla_get_device_error.
#include <math.h>
#include <string.h>

#include <cuda_runtime.h>

#include "mla.h"
#include "api_checks.h"
#include "common.cuh"
#include "kernels.h"
#include "sm100.h"

namespace {

using namespace mla;
using api::aligned16;
using api::check_cache;
using api::check_dims;
using api::softmax_scale;
using bf16 = __nv_bfloat16;

size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

// Workspace regions (byte offsets).  The first 256 bytes hold the device
// error word (offset 0) and the attention plan header (offset 64).
struct Layout {
  size_t err, hdr, seq_start, part_base, bad, part_O, part_m, part_l, xkv, cq, qc, qr, o, total;
  int slots;
};

int device_sms() {
  int dev = 0, n = 148;
  if (cudaGetDevice(&dev) == cudaSuccess)
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) n = 148;
  return n > 0 ? n : 148;
}

// Partitions of the attention work: one per CTA pair on the tensor-core path,
// one per block column on the CUDA-core path.
int auto_parts(const mla_dims &d) {
  (void)d;
  return device_sms() / 2;
}

int parts_for(const mla_dims &d, int num_splits) {
  return num_splits > 0 ? num_splits : auto_parts(d);
}

Layout make_layout(const mla_dims &d, int batch, int d_model, int d_q, int parts) {
  Layout L{};
  const int H = d.n_heads, row = d.d_c + d.d_rope;
  size_t off = 0;
  L.err = 0;
  L.hdr = 64;
  off = 256;
  L.seq_start = off; off = align256(off + sizeof(int) * (batch + 1));
  L.part_base = off; off = align256(off + sizeof(int) * batch);
  L.bad = off; off = align256(off + sizeof(int) * batch);
  L.slots = 2 * parts + 2;
  L.part_O = off; off = align256(off + sizeof(float) * (size_t)L.slots * H * d.d_c);
  L.part_m = off; off = align256(off + sizeof(float) * (size_t)L.slots * H);
  L.part_l = off; off = align256(off + sizeof(float) * (size_t)L.slots * H);
  L.xkv = off; off = align256(off + sizeof(float) * (size_t)batch * row);
  L.cq = off; off = align256(off + sizeof(float) * (size_t)batch * (d_q > 0 ? d_q : 0));
  L.qc = off; off = align256(off + sizeof(float) * (size_t)batch * H * d.d_nope);
  L.qr = off; off = align256(off + sizeof(float) * (size_t)batch * H * d.d_rope);
  L.o = off; off = align256(off + sizeof(float) * (size_t)batch * H * d.d_v);
  L.total = off;
  (void)d_model;
  return L;
}

mla_status check_width(const mla_dims *d, int w) {
  if (w < 1) return MLA_ERR_INVALID_ARG;
  if (d->dtype == MLA_BF16 && (w % 64)) return MLA_ERR_UNSUPPORTED;
  return MLA_OK;
}

RopeParams rope_params(const mla_dims &d) {
  RopeParams rp;
  memset(&rp, 0, sizeof(rp));
  rp.d_rope = d.d_rope;
  rp.half = d.rope_layout == MLA_ROPE_HALF;
  for (int i = 0; i < d.d_rope / 2; ++i) rp.theta[i] = pow(d.rope_base, -2.0 * i / d.d_rope);
  return rp;
}

char *at(void *ws, size_t off) { return static_cast<char *>(ws) + off; }

mla_status cuda_ok(cudaError_t e) { return e == cudaSuccess ? MLA_OK : MLA_ERR_CUDA; }

#define MLA_TRY(x)                   \
  do {                               \
    mla_status st_ = (x);            \
    if (st_ != MLA_OK) return st_;   \
  } while (0)

template <class TW, class TX, class TY>
mla_status gemv(const void *W, long w_head, long w_m, long w_k, const void *X, long x_head,
                long x_b, void *Y, long y_head, long y_b, int M, int K, int B, int heads,
                cudaStream_t s) {
  GemvArgs a{W, w_head, w_m, w_k, X, x_head, x_b, Y, y_head, y_b, M, K, B};
  return cuda_ok(launch_gemv<TW, TX, TY>(a, heads, s));
}

// Plan, attention and merge: z / lse, or with pO the unnormalised partial
// softmax (O, m, l) of the rows the cache holds.  Arguments already checked.
mla_status decode_attn_impl(const mla_dims *dims, const mla_paged_cache *cache, int batch,
                            const void *q_lat, void *z, float *lse, float *pO, float *pm,
                            float *pl, int num_splits, void *ws, size_t ws_bytes,
                            cudaStream_t s) {
  if (!ws) return MLA_ERR_INVALID_ARG;
  if (!aligned16(ws)) return MLA_ERR_ALIGNMENT;
  const mla_dims &d = *dims;
  const int parts = parts_for(d, num_splits);
  const Layout L = make_layout(d, batch, 64, 0, parts);
  if (ws_bytes < L.total) return MLA_ERR_WORKSPACE;
  PlanArgs pa{};
  pa.seq_lens = cache->seq_lens;
  pa.batch = batch;
  pa.page_size = d.page_size;
  pa.max_pages = cache->max_pages_per_seq;
  pa.parts_max = parts;
  pa.min_pages = d.dtype == MLA_BF16 ? sm100::kAttnMinPages : 1;
  pa.gap = d.dtype == MLA_BF16 ? sm100::kAttnSeqGap : 0;
  pa.allow_empty = pO != nullptr;
  pa.hdr = reinterpret_cast<PlanHeader *>(at(ws, L.hdr));
  pa.seq_start = reinterpret_cast<int *>(at(ws, L.seq_start));
  pa.part_base = reinterpret_cast<int *>(at(ws, L.part_base));
  pa.bad = reinterpret_cast<int *>(at(ws, L.bad));
  pa.err = reinterpret_cast<int *>(at(ws, L.err));
  MLA_TRY(cuda_ok(launch_plan(pa, s)));
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
  a.scale = softmax_scale(d);
  a.hdr = pa.hdr;
  a.seq_start = pa.seq_start;
  a.part_base = pa.part_base;
  a.bad = pa.bad;
  a.part_O = reinterpret_cast<float *>(at(ws, L.part_O));
  a.part_m = reinterpret_cast<float *>(at(ws, L.part_m));
  a.part_l = reinterpret_cast<float *>(at(ws, L.part_l));
  a.err = pa.err;
  a.int8_rows = d.cache_format == MLA_CACHE_INT8;
  a.pout_O = pO;
  a.pout_m = pm;
  a.pout_l = pl;
  if (d.dtype == MLA_FP32) {
    MLA_TRY(cuda_ok(launch_attn_simt<float>(a, parts, s)));
    return cuda_ok(launch_combine<float>(a, s));
  }
  MLA_TRY(cuda_ok(sm100::launch_attn(a, parts, s)));
  return cuda_ok(launch_combine<bf16>(a, s));
}

}  // namespace

extern "C" {

size_t mla_workspace_size(const mla_dims *dims, int batch, int d_model, int d_q, int num_splits) {
  if (check_dims(dims) != MLA_OK || batch < 1 || d_model < 1 || d_q < 0 || num_splits < 0)
    return 0;
  return make_layout(*dims, batch, d_model, d_q, parts_for(*dims, num_splits)).total;
}

mla_status mla_workspace_init(void *ws, size_t ws_bytes, mla_stream_t stream) {
  if (!ws) return MLA_ERR_INVALID_ARG;
  if (ws_bytes < 256) return MLA_ERR_WORKSPACE;
  if (!aligned16(ws)) return MLA_ERR_ALIGNMENT;
  return cuda_ok(cudaMemsetAsync(ws, 0, 256, (cudaStream_t)stream));
}

mla_status mla_cache_append(const mla_dims *dims, const mla_paged_cache *cache, int batch,
                            int d_model, const void *h, const void *W_DKV, const void *W_KR,
                            const void *gamma, const int32_t *positions, void *ws,
                            size_t ws_bytes, mla_stream_t stream) {
  MLA_TRY(check_dims(dims));
  MLA_TRY(check_cache(cache));
  MLA_TRY(check_width(dims, d_model));
  if (batch < 1 || !h || !W_DKV || !W_KR || !gamma || !positions || !ws)
    return MLA_ERR_INVALID_ARG;
  if (!aligned16(h) || !aligned16(W_DKV) || !aligned16(W_KR) || !aligned16(gamma) ||
      !aligned16(ws) || (reinterpret_cast<uintptr_t>(positions) & 3))
    return MLA_ERR_ALIGNMENT;
  const mla_dims &d = *dims;
  const Layout L = make_layout(d, batch, d_model, 0, parts_for(d, 0));
  if (ws_bytes < L.total) return MLA_ERR_WORKSPACE;
  cudaStream_t s = (cudaStream_t)stream;
  const int row = d.d_c + d.d_rope;
  float *xkv = reinterpret_cast<float *>(at(ws, L.xkv));
  int *err = reinterpret_cast<int *>(at(ws, L.err));
  const RopeParams rp = rope_params(d);
  if (d.dtype == MLA_FP32) {
    MLA_TRY((gemv<float, float, float>(W_DKV, 0, d_model, 1, h, 0, d_model, xkv, 0, row, d.d_c,
                                       d_model, batch, 1, s)));
    MLA_TRY((gemv<float, float, float>(W_KR, 0, d_model, 1, h, 0, d_model, xkv + d.d_c, 0, row,
                                       d.d_rope, d_model, batch, 1, s)));
    return cuda_ok(launch_append_finish<float>(
        xkv, 1, batch, d.d_c, rp, static_cast<const float *>(gamma), (float)d.rms_eps, positions,
        static_cast<float *>(cache->pool), cache->num_pages, d.page_size, cache->block_table,
        cache->max_pages_per_seq, err, s));
  }
  MLA_TRY(cuda_ok(sm100::append_proj(static_cast<const bf16 *>(h), static_cast<const bf16 *>(W_DKV),
                                     static_cast<const bf16 *>(W_KR), batch, d_model, xkv, err,
                                     s)));
  if (d.cache_format == MLA_CACHE_INT8)
    return cuda_ok(launch_append_finish_int8(
        xkv, batch, d.d_c, rp, static_cast<const bf16 *>(gamma), (float)d.rms_eps, positions,
        static_cast<uint8_t *>(cache->pool), cache->num_pages, d.page_size, cache->block_table,
        cache->max_pages_per_seq, err, s));
  return cuda_ok(launch_append_finish<bf16>(
      xkv, 1, batch, d.d_c, rp, static_cast<const bf16 *>(gamma), (float)d.rms_eps, positions,
      static_cast<bf16 *>(cache->pool), cache->num_pages, d.page_size, cache->block_table,
      cache->max_pages_per_seq, err, s));
}

mla_status mla_absorb_q(const mla_dims *dims, int batch, int d_in, const void *x,
                        const void *W_DQ, int d_q, const void *W_UQ, const void *W_QR,
                        const void *W_UK, const int32_t *positions, void *q_lat, void *ws,
                        size_t ws_bytes, mla_stream_t stream) {
  MLA_TRY(check_dims(dims));
  MLA_TRY(check_width(dims, d_in));
  if (batch < 1 || !x || !W_UQ || !W_QR || !W_UK || !positions || !q_lat || !ws)
    return MLA_ERR_INVALID_ARG;
  if (!W_DQ) {
    if (d_q == 0) d_q = d_in;
    if (d_q != d_in) return MLA_ERR_INVALID_ARG;
  } else {
    MLA_TRY(check_width(dims, d_q));
  }
  if (!aligned16(x) || (W_DQ && !aligned16(W_DQ)) || !aligned16(W_UQ) || !aligned16(W_QR) ||
      !aligned16(W_UK) || !aligned16(q_lat) || !aligned16(ws) ||
      (reinterpret_cast<uintptr_t>(positions) & 3))
    return MLA_ERR_ALIGNMENT;
  const mla_dims &d = *dims;
  const Layout L = make_layout(d, batch, d_in, W_DQ ? d_q : 0, parts_for(d, 0));
  if (ws_bytes < L.total) return MLA_ERR_WORKSPACE;
  cudaStream_t s = (cudaStream_t)stream;
  const int H = d.n_heads, row = d.d_c + d.d_rope;
  float *cq = reinterpret_cast<float *>(at(ws, L.cq));
  float *qc = reinterpret_cast<float *>(at(ws, L.qc));
  float *qr = reinterpret_cast<float *>(at(ws, L.qr));
  const RopeParams rp = rope_params(d);
  if (d.dtype == MLA_FP32) {
    const void *xin = x;
    if (W_DQ) {
      MLA_TRY((gemv<float, float, float>(W_DQ, 0, d_in, 1, x, 0, d_in, cq, 0, d_q, d_q, d_in,
                                         batch, 1, s)));
      xin = cq;
    }
    MLA_TRY((gemv<float, float, float>(W_UQ, 0, d_q, 1, xin, 0, d_q, qc, 0, H * d.d_nope,
                                       H * d.d_nope, d_q, batch, 1, s)));
    MLA_TRY((gemv<float, float, float>(W_QR, 0, d_q, 1, xin, 0, d_q, qr, 0, H * d.d_rope,
                                       H * d.d_rope, d_q, batch, 1, s)));
    // q~_i[c] = sum_a W_UK[i][a][c] q_C,i[a]: per-head transposed product
    MLA_TRY((gemv<float, float, float>(W_UK, (long)d.d_nope * d.d_c, 1, d.d_c, qc, d.d_nope,
                                       (long)H * d.d_nope, q_lat, row, (long)H * row, d.d_c,
                                       d.d_nope, batch, H, s)));
    return cuda_ok(launch_rope_q<float>(qr, batch, H, d.d_c, rp, positions,
                                        static_cast<float *>(q_lat), s));
  }
  return cuda_ok(sm100::absorb_proj(
      static_cast<const bf16 *>(x), static_cast<const bf16 *>(W_DQ),
      static_cast<const bf16 *>(W_UQ), static_cast<const bf16 *>(W_QR),
      static_cast<const bf16 *>(W_UK), batch, d_in, d_q, rp, positions,
      reinterpret_cast<bf16 *>(cq), static_cast<bf16 *>(q_lat),
      reinterpret_cast<int *>(at(ws, L.err)), s));
}

mla_status mla_decode_attn(const mla_dims *dims, const mla_paged_cache *cache, int batch,
                           const void *q_lat, void *z, float *lse, int num_splits, void *ws,
                           size_t ws_bytes, mla_stream_t stream) {
  MLA_TRY(api::check_attn_args(dims, cache, batch, q_lat, z, lse, num_splits));
  return decode_attn_impl(dims, cache, batch, q_lat, z, lse, nullptr, nullptr, nullptr,
                          num_splits, ws, ws_bytes, (cudaStream_t)stream);
}

mla_status mla_decode_attn_partial(const mla_dims *dims, const mla_paged_cache *cache, int batch,
                                   const void *q_lat, float *O, float *m, float *l, int num_splits,
                                   void *ws, size_t ws_bytes, mla_stream_t stream) {
  if (!O || !m || !l) return MLA_ERR_INVALID_ARG;
  // O takes z's place in the argument rules (16-byte aligned); m and l are fp32 like lse
  MLA_TRY(api::check_attn_args(dims, cache, batch, q_lat, O, m, num_splits));
  if (!api::aligned4(l)) return MLA_ERR_ALIGNMENT;
  return decode_attn_impl(dims, cache, batch, q_lat, nullptr, nullptr, O, m, l, num_splits, ws,
                          ws_bytes, (cudaStream_t)stream);
}

mla_status mla_merge_partials(const mla_dims *dims, int batch, int n_parts, const float *O,
                              const float *m, const float *l, void *z, float *lse,
                              mla_stream_t stream) {
  MLA_TRY(check_dims(dims));
  if (batch < 1 || n_parts < 1 || !O || !m || !l || !z) return MLA_ERR_INVALID_ARG;
  if (!aligned16(O) || !api::aligned4(m) || !api::aligned4(l) || !aligned16(z) ||
      (lse && !api::aligned4(lse)))
    return MLA_ERR_ALIGNMENT;
  const mla_dims &d = *dims;
  cudaStream_t s = (cudaStream_t)stream;
  if (d.dtype == MLA_FP32)
    return cuda_ok(launch_merge_partials<float>(O, m, l, n_parts, batch, d.n_heads, d.d_c,
                                               static_cast<float *>(z), lse, s));
  return cuda_ok(launch_merge_partials<bf16>(O, m, l, n_parts, batch, d.n_heads, d.d_c,
                                            static_cast<bf16 *>(z), lse, s));
}

mla_status mla_unabsorb_out(const mla_dims *dims, int batch, const void *z, const void *W_UV,
                            const void *W_O, int d_model, void *out, void *ws, size_t ws_bytes,
                            mla_stream_t stream) {
  MLA_TRY(check_dims(dims));
  if (batch < 1 || !z || !W_UV || !out || !ws) return MLA_ERR_INVALID_ARG;
  if (W_O) MLA_TRY(check_width(dims, d_model));
  if (!aligned16(z) || !aligned16(W_UV) || (W_O && !aligned16(W_O)) || !aligned16(out) ||
      !aligned16(ws))
    return MLA_ERR_ALIGNMENT;
  const mla_dims &d = *dims;
  const Layout L = make_layout(d, batch, W_O ? d_model : 64, 0, parts_for(d, 0));
  if (ws_bytes < L.total) return MLA_ERR_WORKSPACE;
  cudaStream_t s = (cudaStream_t)stream;
  const int H = d.n_heads;
  float *o = reinterpret_cast<float *>(at(ws, L.o));
  if (d.dtype == MLA_FP32) {
    void *dst = W_O ? static_cast<void *>(o) : out;
    MLA_TRY((gemv<float, float, float>(W_UV, (long)d.d_v * d.d_c, d.d_c, 1, z, d.d_c,
                                       (long)H * d.d_c, dst, d.d_v, (long)H * d.d_v, d.d_v, d.d_c,
                                       batch, H, s)));
    if (!W_O) return MLA_OK;
    return gemv<float, float, float>(W_O, 0, (long)H * d.d_v, 1, o, 0, (long)H * d.d_v, out, 0,
                                     d_model, d_model, H * d.d_v, batch, 1, s);
  }
  return cuda_ok(sm100::unabsorb_proj(
      static_cast<const bf16 *>(z), static_cast<const bf16 *>(W_UV), static_cast<const bf16 *>(W_O),
      batch, d_model, reinterpret_cast<bf16 *>(o), static_cast<bf16 *>(out),
      reinterpret_cast<int *>(at(ws, L.err)), s));
}

mla_status mla_get_device_error(void *ws, mla_stream_t stream) {
  if (!ws) return MLA_ERR_INVALID_ARG;
  if (cudaStreamSynchronize((cudaStream_t)stream) != cudaSuccess) return MLA_ERR_CUDA;
  int word = 0;
  if (cudaMemcpy(&word, ws, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess)
    return MLA_ERR_CUDA;
  const int zero = 0;
  if (cudaMemcpy(ws, &zero, sizeof(int), cudaMemcpyHostToDevice) != cudaSuccess)
    return MLA_ERR_CUDA;
  if (word & kErrTimeout) return MLA_ERR_TIMEOUT;
  if (word & kErrRange) return MLA_ERR_DEVICE_RANGE;
  return MLA_OK;
}

mla_status mla_debug_absorb_timeout(int enable, unsigned wait_limit_us) {
  if (enable && wait_limit_us == 0) return MLA_ERR_INVALID_ARG;
  sm100::absorb_debug_fault(enable ? 1 : 0, enable ? (uint64_t)wait_limit_us * 1000ull : 0);
  return MLA_OK;
}

const char *mla_status_string(mla_status status) {
  switch (status) {
    case MLA_OK: return "ok";
    case MLA_ERR_INVALID_ARG: return "invalid argument";
    case MLA_ERR_UNSUPPORTED: return "unsupported shape";
    case MLA_ERR_ALIGNMENT: return "tensor pointer not 16-byte aligned";
    case MLA_ERR_WORKSPACE: return "workspace missing or too small";
    case MLA_ERR_CUDA: return "CUDA runtime error";
    case MLA_ERR_DEVICE_RANGE: return "device check: page entry, length or position out of range";
    case MLA_ERR_TIMEOUT: return "device check: bounded wait timed out";
  }
  return "unknown status";
}

}  // extern "C"
