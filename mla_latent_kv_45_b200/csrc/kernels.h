// Internal launch interfaces of the MLA decode kernels (not part of the C ABI).
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "common.cuh"

namespace mla {

// Y[b][m] = sum_k W[m][k] X[b][k], for `heads` independent heads.
// Element (m, k) of head z lives at W + z*w_head + m*w_m + k*w_k (one of w_m,
// w_k is 1); X[b][k] at X + z*x_head + b*x_b + k; Y[b][m] at Y + z*y_head + b*y_b + m.
struct GemvArgs {
  const void *W;
  long w_head, w_m, w_k;
  const void *X;
  long x_head, x_b;
  void *Y;
  long y_head, y_b;
  int M, K, B;
};

template <class TW, class TX, class TY>
cudaError_t launch_gemv(const GemvArgs &a, int heads, cudaStream_t s);

template <class T>
cudaError_t launch_append_finish(const float *xkv, int batch, int d_c, const RopeParams &rp,
                                 const T *gamma, float eps, const int32_t *positions, T *pool,
                                 int num_pages, int page_size, const int32_t *block_table,
                                 int max_pages, int *err, cudaStream_t s);

template <class T>
cudaError_t launch_rope_q(const float *qr, int batch, int n_heads, int d_c, const RopeParams &rp,
                          const int32_t *positions, T *q_lat, cudaStream_t s);

struct PlanArgs {
  const int32_t *seq_lens;
  int batch, page_size, max_pages;
  int parts_max, min_pages;
  PlanHeader *hdr;
  int *seq_start;  // [batch + 1]
  int *part_base;  // [batch]
  int *bad;        // [batch]
  int *err;
};

cudaError_t launch_plan(const PlanArgs &a, cudaStream_t s);

struct AttnArgs {
  const void *q_lat;
  const void *pool;
  const int32_t *block_table;
  const int32_t *seq_lens;
  void *z;
  float *lse;
  int batch, n_heads, d_c, d_rope, page_size, num_pages, max_pages;
  float scale;
  const PlanHeader *hdr;
  const int *seq_start;
  const int *part_base;
  int *bad;
  float *part_O;  // [slots][n_heads][d_c]
  float *part_m;  // [slots][n_heads]
  float *part_l;  // [slots][n_heads]
  int *err;
};

template <class T>
cudaError_t launch_attn_simt(const AttnArgs &a, int parts_max, cudaStream_t s);

template <class T>
cudaError_t launch_combine(const AttnArgs &a, cudaStream_t s);

}  // namespace mla
