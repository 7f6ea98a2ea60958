// Interface of the skinny tensor-core GEMM used by the decode projections.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>

namespace mla {
namespace sm100 {

constexpr int kMaxGemmStages = 8;
enum : int { kOutBf16 = 1, kOutF32 = 2 };

// One projection Y[n][m] = sum_k A[m][k] X[n][k] (per head when heads > 1).
//   a_mn = 0: A[m][k] = A2d[head * M + m][k]     (A2d is [heads*M][K], an [out][in] weight)
//   a_mn = 1: A[m][k] = A2d[head * K + k][m]     (A2d is [heads*K][M], a transposed view)
// Output: out[n * ldy + head * y_head + m], bf16 or fp32.
// With splits > 1 (at most kMaxClusterSplits; M, ldy and y_head multiples of
// 4, out 16-byte aligned) the K range of each tile is cut into `splits` CTAs
// that form a thread-block cluster and sum their partial tiles through
// distributed shared memory in a fixed order.  Every op of a launch uses the
// same splits.
struct GemmOp {
  const __nv_bfloat16 *A;
  int M, heads, a_mn;
  int out_mode;
  void *out;
  long ldy, y_head;
  int splits;
};

constexpr int kMaxClusterSplits = 8;

// Kernel-side description of one problem of a launch.  Its work items are
// (head, split, m_tile) triples numbered from item_begin.
struct GemmProblem {
  int M, m_tiles, a_mn, a_map, a_rows_per_head, splits, chunks_per_split, item_begin, out_mode;
  void *out;
  long ldy, y_head;
};

struct GemmLaunch {
  GemmProblem p[2];
  int nprob, n, n0, n_total, n_pad, n_cols, k_chunks, x_cols_per_head, stages, tmem_cols;
  int items, items_per_cta;
  int cluster;  // CTAs per cluster (the splits of one tile) in cluster-reduce mode, else 0
  int *err;
};

// Split count for an in-cluster reduction (at most kMaxClusterSplits) of a
// problem with m_tiles x heads tiles, K / 64 chunks and batch n.
int gemm_cluster_splits(int m_tiles, int heads, int k_chunks, int n);

// Split count for a problem of m_tiles x heads tiles and K / 64 chunks.
int gemm_splits(int m_tiles, int heads, int k_chunks);

// Runs 1 or 2 problems that share X ([n][x_cols] bf16, row-major; head h reads
// columns [h * x_cols_per_head, ... + K)).  K must be a multiple of 64.
cudaError_t gemm(const GemmOp *ops, int nops, const __nv_bfloat16 *X, int n, long x_cols, int K,
                 int x_cols_per_head, int *err, cudaStream_t s);

}  // namespace sm100
}  // namespace mla
