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

// xkv: `splits` partial sums [splits][batch][d_c + d_rope] of [W_DKV h ; W_KR h].
template <class T>
cudaError_t launch_append_finish(const float *xkv, int splits, int batch, int d_c,
                                 const RopeParams &rp, const T *gamma, float eps,
                                 const int32_t *positions, T *pool, int num_pages, int page_size,
                                 const int32_t *block_table, int max_pages, int *err,
                                 cudaStream_t s);

// The same append into a 656-byte int8 row (MLA_CACHE_INT8, d_c = 512, d_rope = 64).
cudaError_t launch_append_finish_int8(const float *xkv, int batch, int d_c, const RopeParams &rp,
                                      const __nv_bfloat16 *gamma, float eps,
                                      const int32_t *positions, uint8_t *pool, int num_pages,
                                      int page_size, const int32_t *block_table, int max_pages,
                                      int *err, cudaStream_t s);

template <class T>
cudaError_t launch_rope_q(const float *qr, int batch, int n_heads, int d_c, const RopeParams &rp,
                          const int32_t *positions, T *q_lat, cudaStream_t s);

struct PlanArgs {
  const int32_t *seq_lens;
  int batch, page_size, max_pages;
  int parts_max, min_pages;
  int allow_empty;  // seq_len == 0 is an empty share (no rows), not an error
  int gap;          // virtual pages charged per sequence (its fixed cost), 0 = none
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
  // Partial-softmax output (nullptr for z / lse): unnormalised O [batch][n_heads][d_c],
  // m (natural-log max) and l [batch][n_heads], fp32.
  float *pout_O, *pout_m, *pout_l;
  int int8_rows;  // the pool holds 656-byte int8 rows (MLA_CACHE_INT8)
};

template <class T>
cudaError_t launch_attn_simt(const AttnArgs &a, int parts_max, cudaStream_t s);

template <class T>
cudaError_t launch_combine(const AttnArgs &a, cudaStream_t s);

// Merge of n partial softmaxes (unnormalised O, natural-log m, l), laid out
// [n][batch][n_heads](*d_c): z = sum_j w_j O_j / sum_j w_j l_j, w_j = e^(m_j - max m),
// lse = max m + log(sum_j w_j l_j); rows whose parts are all empty get z = 0,
// lse = -inf.
template <class T>
cudaError_t launch_merge_partials(const float *O, const float *m, const float *l, int n_parts,
                                  int batch, int n_heads, int d_c, T *z, float *lse,
                                  cudaStream_t s);

}  // namespace mla

namespace mla {

// One piece of a partition: local pages [lp0, lp1) of sequence b (s0 = the
// virtual index of the sequence's first page, len = its row count).
struct Segment {
  int b, lp0, lp1, len, s0;
};

// Walks the segments of partition p of the plan: virtual pages
// [p*quota, (p+1)*quota) of the batch's concatenated page list, in which each
// sequence's pages are preceded by `gap` virtual pages that hold no rows (they
// stand for the fixed cost of a sequence, so partitions with more sequences
// get fewer pages).  Sequence b's pages are [seq_start[b], seq_start[b+1] - gap).
struct SegmentWalker {
  int g0, g1, b, gap;

  __device__ __forceinline__ void init(const AttnArgs &a, const PlanHeader &h, int p) {
    g0 = p * h.quota;
    g1 = min(h.total_pages, g0 + h.quota);
    gap = h.gap;
    b = 0;
    if (g0 >= g1) return;
    int lo = 0, hi = a.batch;  // the last b with seq_start[b] <= g0 (or 0)
    while (hi - lo > 1) {
      const int mid = (lo + hi) >> 1;
      if (a.seq_start[mid] <= g0) lo = mid; else hi = mid;
    }
    b = lo;
  }

  __device__ __forceinline__ bool next(const AttnArgs &a, Segment &s) {
    while (g0 < g1 && b < a.batch) {
      const int s0 = a.seq_start[b], s1 = a.seq_start[b + 1] - gap;
      const int lo = max(g0, s0);
      if (lo >= g1) return false;        // the range ends before sequence b's pages
      if (s1 <= lo) { ++b; continue; }   // sequence b ends before lo (or has no pages)
      s.b = b;
      s.s0 = s0;
      s.lp0 = lo - s0;
      s.lp1 = min(g1, s1) - s0;
      s.len = a.seq_lens[b];
      g0 = s0 + s.lp1;
      ++b;
      return true;
    }
    return false;
  }
};

}  // namespace mla
