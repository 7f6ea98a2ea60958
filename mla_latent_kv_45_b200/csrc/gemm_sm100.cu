// Skinny bf16 GEMMs of the decode projections on sm_100a tensor cores.
//
// Y[n][m] = sum_k A[m][k] X[n][k] with m over the weight's output rows, n over
// the batch (N <= 256) and k over the input width.  Decode projections are
// weight-bandwidth bound (each weight element is used B times), so the design
// streams the weights once through a deep TMA ring with as many CTAs as it
// takes to keep HBM busy:
//  * a work item is one 128-row tile of one problem, one K range (split-K) and
//    one head; D = A_tile . X^T accumulates in TMEM (tcgen05.mma, M = 128,
//    N = batch padded to 16, K = 16 per instruction);
//  * CTAs are persistent over a contiguous range of items: the TMA ring runs
//    on across items and the accumulator is double-buffered in TMEM, so one
//    item's epilogue overlaps the next item's loads and MMAs;
//  * A comes K-major ([out][in] weights) or MN-major (a per-head transposed
//    view such as W_UK,i^T) -- both through 128-byte-swizzled TMA boxes;
//  * X (the activations, bf16) is reloaded from L2 per K chunk;
//  * two problems that share X (e.g. W_DKV and W_KR, W_UQ and W_QR) run in one
//    launch; per-head problems (W_UK, W_UV) index heads in their items;
//  * the epilogue writes bf16 / fp32 outputs directly; where there are too few
//    tiles, the K range of each tile is split across the CTAs of a cluster,
//    which sum their partial tiles through distributed shared memory in a
//    fixed order (deterministic).
// Warp roles: warp 0 TMA producer, warp 1 TMEM allocation + MMA issue,
// warps 2-5 epilogue.  Every wait is bounded (globaltimer).
#include <cuda.h>

#include <mutex>

#include "api_checks.h"
#include "ptx.cuh"
#include "sm100.h"
#include "gemm_sm100.h"

namespace mla {
namespace sm100 {
namespace {

using namespace ptx;

constexpr int kThreads = 192;
constexpr uint64_t kTimeoutNs = 2000000000ull;
constexpr int kABytes = 128 * 128;  // 128 rows x 64 bf16

struct Bars {
  uint64_t full[kMaxGemmStages], empty[kMaxGemmStages], acc_full[2], acc_free[2], drain;
  uint32_t tmem_base;
  volatile int abort;
};

__device__ __forceinline__ bool gwait(Bars *bars, int *err, uint64_t *bar, uint32_t parity) {
  const uint32_t a = smem_u32(bar);
  if (mbar_try_wait(a, parity)) return true;
  const uint64_t t0 = globaltimer();
  while (true) {
    if (mbar_try_wait_sleep(a, parity, 20000)) return true;
    if (bars->abort) return false;
    if (globaltimer() - t0 > kTimeoutNs) {
      set_error(err, kErrTimeout);
      bars->abort = 1;
      return false;
    }
  }
}

struct Item {
  int pi, head, split, m0, kc0, nk;
};

__device__ __forceinline__ Item decode_item(const GemmLaunch &g, int item) {
  Item it;
  it.pi = (g.nprob > 1 && item >= g.p[1].item_begin) ? 1 : 0;
  const GemmProblem &P = g.p[it.pi];
  int t = item - P.item_begin;
  if (g.cluster) {
    // split fastest: the splits of one tile are the consecutive CTAs of a cluster
    it.split = t % P.splits;
    t /= P.splits;
    it.m0 = (t % P.m_tiles) * 128;
    it.head = t / P.m_tiles;
  } else {
    it.m0 = (t % P.m_tiles) * 128;
    t /= P.m_tiles;
    it.split = t % P.splits;
    it.head = t / P.splits;
  }
  it.kc0 = it.split * P.chunks_per_split;
  it.nk = min(g.k_chunks, it.kc0 + P.chunks_per_split) - it.kc0;
  return it;
}

__global__ void __launch_bounds__(kThreads, 2)
    gemm_sm100_kernel(const __grid_constant__ CUtensorMap tm_a0,
                      const __grid_constant__ CUtensorMap tm_a1,
                      const __grid_constant__ CUtensorMap tm_x, const GemmLaunch g) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int stage_bytes = kABytes + g.n_pad * 128;
  Bars *bars = reinterpret_cast<Bars *>(smem + g.stages * stage_bytes);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int item0 = blockIdx.x * g.items_per_cta;
  const int item1 = min(g.items, item0 + g.items_per_cta);

  if (threadIdx.x == 0) {
    for (int s = 0; s < g.stages; ++s) {
      mbar_init(&bars->full[s], 1);
      mbar_init(&bars->empty[s], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&bars->acc_full[i], 1);
      mbar_init(&bars->acc_free[i], 4);
    }
    mbar_init(&bars->drain, 1);
    bars->abort = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tmap(&tm_a0);
    if (g.nprob > 1) prefetch_tmap(&tm_a1);
    prefetch_tmap(&tm_x);
  }
  if (warp == 1) {
    tmem_alloc(&bars->tmem_base, g.tmem_cols);
    tc_fence_before();
  }
  __syncwarp();   // thread 0 alone set up the barriers
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bars->tmem_base;

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      const int tx = kABytes + g.n_pad * 128;
      // The weights do not depend on the previous kernel: the first stages'
      // weight tiles are requested before waiting for it, and their
      // activation tiles (which it may write) after.
      auto load_a = [&](const Item &it, int i, int st) {
        const GemmProblem &P = g.p[it.pi];
        const CUtensorMap *tm_a = it.pi ? &tm_a1 : &tm_a0;
        uint8_t *a_dst = smem + st * stage_bytes;
        const int k = (it.kc0 + i) * 64;
        if (P.a_mn) {
          // A[m][k] = A2d[head * K + k][m]: two 64-wide MN chunks, 64 K rows each
          const int y = it.head * P.a_rows_per_head + k;
          tma_load_2d(a_dst, tm_a, it.m0, y, &bars->full[st]);
          tma_load_2d(a_dst + kABytes / 2, tm_a, it.m0 + 64, y, &bars->full[st]);
        } else {
          tma_load_2d(a_dst, tm_a, k, it.head * P.a_rows_per_head + it.m0, &bars->full[st]);
        }
      };
      int pre = 0;   // chunks whose weight tile was requested before the wait
      for (int item = item0, c = 0; item < item1 && c < g.stages; ++item) {
        const Item it = decode_item(g, item);
        for (int i = 0; i < it.nk && c < g.stages; ++i, ++c, ++pre) {
          mbar_expect_tx(&bars->full[c], tx);
          load_a(it, i, c);
        }
      }
      grid_dep_wait();
      grid_dep_launch();
      int c = 0;
      bool ok = true;
      for (int item = item0; ok && item < item1; ++item) {
        const Item it = decode_item(g, item);
        for (int i = 0; i < it.nk; ++i, ++c) {
          const int st = c % g.stages;
          if (c >= g.stages && !gwait(bars, g.err, &bars->empty[st], ((c / g.stages) - 1) & 1)) {
            ok = false;
            break;
          }
          uint8_t *x_dst = smem + st * stage_bytes + kABytes;
          const int k = (it.kc0 + i) * 64;
          if (c >= pre) {
            mbar_expect_tx(&bars->full[st], tx);
            load_a(it, i, st);
          }
          tma_load_2d(x_dst, &tm_x, it.head * g.x_cols_per_head + k, 0, &bars->full[st]);
        }
      }
      for (int i = c - g.stages; i < c; ++i)
        if (i >= 0) gwait(bars, g.err, &bars->full[i % g.stages], (i / g.stages) & 1);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      int c = 0;
      bool ok = true;
      for (int item = item0, li = 0; ok && item < item1; ++item, ++li) {
        const Item it = decode_item(g, item);
        const GemmProblem &P = g.p[it.pi];
        const uint32_t idesc = idesc_bf16(128, g.n_pad, P.a_mn, 0);
        const int buf = li & 1;
        const uint32_t acc = tmem + buf * g.n_cols;
        if (li >= 2 && !gwait(bars, g.err, &bars->acc_free[buf], ((li >> 1) - 1) & 1)) break;
        tc_fence_after();
        for (int i = 0; i < it.nk; ++i, ++c) {
          const int st = c % g.stages;
          if (!gwait(bars, g.err, &bars->full[st], (c / g.stages) & 1)) { ok = false; break; }
          tc_fence_after();
          const uint32_t a_base = smem_u32(smem + st * stage_bytes);
          const uint32_t x_base = a_base + kABytes;
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            const uint64_t ad = P.a_mn ? sdesc(a_base + 2048 * k, kABytes / 2, 1024, 2)
                                       : sdesc(a_base + 32 * k, 16, 1024, 2);
            const uint64_t bd = sdesc(x_base + 32 * k, 16, 1024, 2);
            umma_bf16(acc, ad, bd, idesc, (i > 0 || k > 0) ? 1u : 0u);
          }
          umma_commit(&bars->empty[st]);
        }
        if (ok) umma_commit(&bars->acc_full[buf]);
      }
      umma_commit(&bars->drain);
      gwait(bars, g.err, &bars->drain, 0);
    }
  } else if (g.cluster) {
    // epilogue of a split: this CTA's partial tile goes straight from TMEM into
    // the shared memory of the CTA that owns its rows (see the reduction below)
    const int quad = warp & 3;
    const int ml = quad * 32 + lane;
    const bool got = __all_sync(0xffffffffu, gwait(bars, g.err, &bars->acc_full[0], 0));
    tc_fence_after();
    cluster_arrive();   // this CTA's MMAs are complete: its stage ring may be overwritten
    const int S = g.cluster, r = (int)cluster_ctarank();
    const int rp = 4 * ((32 + S - 1) / S);           // rows of an owner's share (padded)
    const int slice = g.n_pad * rp;                  // floats of one sender's slice
    const int q = ml >> 2;                           // row quad of this thread's row
    const int o = ((q + 1) * S - 1) / 32;            // owner: q_lo(o) <= q < q_hi(o)
    const int rl = ml - 4 * (32 * o / S);
    const uint32_t dst = mapa(smem_u32(smem) + 4u * (uint32_t)(r * slice + rl), (uint32_t)o);
    const uint32_t taddr = tmem + (static_cast<uint32_t>(quad * 32) << 16);
    cluster_wait();     // every CTA of the cluster is past its MMAs
    if (got) {
      // one float per column: the lanes of a warp (consecutive rows) write
      // consecutive words of the owner's slice
      for (int c = 0; c < g.n_pad; c += 32) {
        uint32_t v[32];
        tmem_ld32(taddr + c, v);
        tmem_wait_ld();
#pragma unroll
        for (int j = 0; j < 32; ++j)
          if (c + j < g.n_pad)   // the accumulator stride rounds n_pad up to 32
            st_cluster_f32(dst + 4u * (uint32_t)((c + j) * rp), __uint_as_float(v[j]));
      }
    }
    tc_fence_before();
  } else {
    // epilogue: warps 2..5 cover TMEM lanes 64..127, 0..63 (lane quadrant = warp % 4)
    const int quad = warp & 3;
    const int ml = quad * 32 + lane;
    for (int item = item0, li = 0; item < item1; ++item, ++li) {
      const Item it = decode_item(g, item);
      const GemmProblem &P = g.p[it.pi];
      const int buf = li & 1;
      if (!gwait(bars, g.err, &bars->acc_full[buf], (li >> 1) & 1)) break;
      tc_fence_after();
      const uint32_t taddr = tmem + buf * g.n_cols + (static_cast<uint32_t>(quad * 32) << 16);
      const int m = it.m0 + ml;
      for (int c = 0; c < g.n_pad; c += 32) {
        uint32_t r[32];
        tmem_ld32(taddr + c, r);
        tmem_wait_ld();
        if (m < P.M) {
#pragma unroll
          for (int j = 0; j < 32; ++j) {
            const int n = c + j;
            if (n < g.n) {
              const float v = __uint_as_float(r[j]);
              const long idx = (long)n * P.ldy + (long)it.head * P.y_head + m;
              if (P.out_mode == kOutBf16)
                static_cast<__nv_bfloat16 *>(P.out)[idx] = __float2bfloat16_rn(v);
              else
                static_cast<float *>(P.out)[idx] = v;
            }
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars->acc_free[buf]);
    }
  }
  if (g.cluster) {
    // In-cluster split-K reduction.  The rows of the tile are cut into 32 quads
    // of 4; CTA r of the S CTAs of this tile owns quads [q_lo, q_hi) =
    // [32 r / S, 32 (r + 1) / S) and receives, in its drained stage ring, one
    // slice [n][row] per split (written by that split's epilogue above).  The
    // owner sums the slices in split order 0..S-1 (deterministic), four rows
    // at a time, and writes the output.
    if (warp < 2) {
      __syncwarp();
      cluster_arrive();
      cluster_wait();
    }
    cluster_arrive();   // release: this CTA's slices are written
    cluster_wait();     // acquire: all slices of this CTA's rows have landed
    const Item it = decode_item(g, item0);
    const GemmProblem &P = g.p[it.pi];
    const int S = g.cluster, r = (int)cluster_ctarank();
    const int q_lo = 32 * r / S, q_hi = 32 * (r + 1) / S, nq = q_hi - q_lo;
    const int rp = 4 * ((32 + S - 1) / S), slice = g.n_pad * rp;
    const float *recv = reinterpret_cast<const float *>(smem);
    for (int u = threadIdx.x; u < g.n * nq; u += kThreads) {
      const int qq = u % nq, n = u / nq;
      const int m = it.m0 + 4 * (q_lo + qq);
      if (m >= P.M) continue;
      const float *p = recv + n * rp + 4 * qq;
      float4 acc = *reinterpret_cast<const float4 *>(p);
      for (int sp = 1; sp < S; ++sp) {
        p += slice;
        const float4 v = *reinterpret_cast<const float4 *>(p);
        acc.x += v.x;
        acc.y += v.y;
        acc.z += v.z;
        acc.w += v.w;
      }
      const long idx = (long)n * P.ldy + (long)it.head * P.y_head + m;
      if (P.out_mode == kOutBf16) {
        __nv_bfloat162 lo = __floats2bfloat162_rn(acc.x, acc.y);
        __nv_bfloat162 hi = __floats2bfloat162_rn(acc.z, acc.w);
        uint2 w;
        w.x = *reinterpret_cast<uint32_t *>(&lo);
        w.y = *reinterpret_cast<uint32_t *>(&hi);
        *reinterpret_cast<uint2 *>(static_cast<__nv_bfloat16 *>(P.out) + idx) = w;
      } else {
        *reinterpret_cast<float4 *>(static_cast<float *>(P.out) + idx) = acc;
      }
    }
  }
  // the warps whose lane 0 alone ran a loop meet again before the CTA barrier
  // (__syncthreads is warp-aligned: a warp must reach it converged)
  __syncwarp();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, g.tmem_cols);
  }
}

typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *,
                                  const cuuint64_t *, const cuuint64_t *, const cuuint32_t *,
                                  const cuuint32_t *, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  if (!fn) {
    void *p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  }
  return fn;
}

// 2-D bf16 row-major [rows][cols] map with a box of box_cols x box_rows, 128B swizzle.
bool map2d(CUtensorMap *m, const void *base, long rows, long cols, int box_cols, int box_rows) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) return false;
  const cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
  const cuuint64_t strides[1] = {(cuuint64_t)cols * 2};
  const cuuint32_t box[2] = {(cuuint32_t)box_cols, (cuuint32_t)box_rows};
  const cuuint32_t estr[2] = {1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(base), dims, strides, box,
             estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) ==
         CUDA_SUCCESS;
}

int sm_count() {
  static int n = 0;
  if (!n) {
    int dev = 0;
    cudaGetDevice(&dev);
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0)
      n = 148;
  }
  return n;
}

}  // namespace

int gemm_splits(int m_tiles, int heads, int k_chunks) {
  // about two resident CTAs per SM, at least 4 K chunks (64 KB of weights) per CTA
  const int tiles = m_tiles * heads;
  int s = 2 * sm_count() / tiles;
  const int max_s = k_chunks / 4 > 0 ? k_chunks / 4 : 1;
  if (s > max_s) s = max_s;
  if (s < 1) s = 1;
  // no empty split: every split gets ceil(k_chunks / s) chunks but the last
  const int per = (k_chunks + s - 1) / s;
  return (k_chunks + per - 1) / per;
}

namespace {

cudaError_t set_smem_attr() {
  static api::PerDeviceOnce smem_attr;
  return smem_attr.run([] {
    const cudaError_t e = cudaFuncSetAttribute(
        gemm_sm100_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, 232448);
    if (e != cudaSuccess) return e;
    // all of the unified L1 / shared array as shared memory: two CTAs per SM
    return cudaFuncSetAttribute(gemm_sm100_kernel,
                                cudaFuncAttributePreferredSharedMemoryCarveout,
                                cudaSharedmemCarveoutMaxShared);
  });
}

// Pipeline stages and dynamic shared memory of a launch with n_pad batch
// columns: two CTAs per SM, each with at most half of the 227 KB.
int stages_for(int n_pad) {
  const int stage_bytes = kABytes + n_pad * 128;
  int st = (232448 / 2 - 1024 - 256) / stage_bytes;
  return st > kMaxGemmStages ? kMaxGemmStages : st;
}
size_t smem_for(int n_pad) {
  return (size_t)stages_for(n_pad) * (kABytes + n_pad * 128) + 256 + 1024;
}

// Clusters of `size` CTAs of a launch with n_pad batch columns that the device
// can hold at once, or 0 if that cannot be determined (queried once per device,
// size and padded batch).
int max_active_clusters(int size, int n_pad) {
  static std::mutex lock;
  static int known[64][kMaxClusterSplits + 1][9];
  static bool init = false;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64 || size < 1 ||
      size > kMaxClusterSplits || n_pad < 16 || n_pad > 128 || n_pad % 16)
    return 0;
  const int ni = n_pad / 16;
  {
    std::lock_guard<std::mutex> g(lock);
    if (!init) {
      for (auto &a : known)
        for (auto &b : a)
          for (int &v : b) v = -1;
      init = true;
    }
    if (known[dev][size][ni] >= 0) return known[dev][size][ni];
  }
  if (set_smem_attr() != cudaSuccess) return 0;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(size);
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = smem_for(n_pad);
  cudaLaunchAttribute at[1];
  at[0].id = cudaLaunchAttributeClusterDimension;
  at[0].val.clusterDim.x = size;
  at[0].val.clusterDim.y = 1;
  at[0].val.clusterDim.z = 1;
  cfg.attrs = at;
  cfg.numAttrs = 1;
  int n = 0;
  if (cudaOccupancyMaxActiveClusters(&n, gemm_sm100_kernel, &cfg) != cudaSuccess) return 0;
  std::lock_guard<std::mutex> g(lock);
  known[dev][size][ni] = n;
  return n;
}

}  // namespace

int gemm_cluster_splits(int m_tiles, int heads, int k_chunks, int n) {
  int s = gemm_splits(m_tiles, heads, k_chunks);
  if (s > kMaxClusterSplits) s = kMaxClusterSplits;
  // one cluster per tile: take the largest split whose clusters all fit on the
  // device at once, for the shared memory these launches use (clusters live
  // inside one GPC, so a size that packs badly would leave some tiles for a
  // second wave)
  const int tiles = m_tiles * heads;
  const int nn = n < 128 ? n : 128;   // cluster launches take the batch in chunks of 128
  const int n_pad = (nn + 15) / 16 * 16;
  // The occupancy query counts one CTA of this kernel per SM (148 clusters of
  // one on B200), while its launch bounds and shared memory place two; measured
  // with 40 tiles, clusters of 6 (240 CTAs) ran in one wave and clusters of 7
  // (280 CTAs, 30 clusters by twice the query's count) did not.
  while (s > 2 && (2 * max_active_clusters(s, n_pad) < tiles || s * tiles > 2 * sm_count())) --s;
  const int per = (k_chunks + s - 1) / s;
  return (k_chunks + per - 1) / per;
}

cudaError_t gemm(const GemmOp *ops, int nops, const __nv_bfloat16 *X, int n, long x_cols, int K,
                 int x_cols_per_head, int *err, cudaStream_t s) {
  if (nops < 1 || nops > 2 || n < 1 || K % 64) return cudaErrorInvalidValue;
  // in-cluster split-K reduction: every op reduces in clusters of the same size
  const bool cluster = ops[0].splits > 1;
  for (int i = 0; i < nops; ++i) {
    const GemmOp &o = ops[i];
    if (o.splits != ops[0].splits || o.splits < 1) return cudaErrorInvalidValue;
    if (cluster && (o.splits > kMaxClusterSplits || (o.M % 4) || (o.ldy % 4) ||
                    (o.y_head % 4) || (reinterpret_cast<uintptr_t>(o.out) & 15)))
      return cudaErrorInvalidValue;
  }
  const int n_step = cluster ? 128 : 256;
  const cudaError_t ea = set_smem_attr();
  if (ea != cudaSuccess) return ea;
  for (int n0 = 0; n0 < n; n0 += n_step) {
    const int nn = n - n0 < n_step ? n - n0 : n_step;
    GemmLaunch g{};
    g.n = nn;
    g.n0 = n0;
    g.n_total = n;
    g.n_pad = (nn + 15) / 16 * 16;
    g.k_chunks = K / 64;
    g.x_cols_per_head = x_cols_per_head;
    g.err = err;
    g.n_cols = (g.n_pad + 31) / 32 * 32;   // accumulator stride: whole 32-column loads
    g.tmem_cols = 32;
    while (g.tmem_cols < 2 * g.n_cols) g.tmem_cols *= 2;
    const int stage_bytes = kABytes + g.n_pad * 128;
    // two CTAs per SM: half of the 227 KB of shared memory each
    g.stages = stages_for(g.n_pad);
    CUtensorMap tm[2], tx;
    int items = 0;
    g.nprob = nops;
    for (int i = 0; i < nops; ++i) {
      const GemmOp &o = ops[i];
      GemmProblem &P = g.p[i];
      P.M = o.M;
      P.m_tiles = (o.M + 127) / 128;
      P.a_mn = o.a_mn;
      P.a_map = i;
      P.a_rows_per_head = o.a_mn ? K : o.M;
      P.splits = o.splits;
      P.chunks_per_split = (g.k_chunks + P.splits - 1) / P.splits;
      P.item_begin = items;
      items += P.m_tiles * P.splits * o.heads;
      P.out_mode = o.out_mode;
      P.ldy = o.ldy;
      P.y_head = o.y_head;
      P.out = static_cast<char *>(o.out) + (long)n0 * o.ldy * (P.out_mode == kOutBf16 ? 2 : 4);
      const long a_rows = o.a_mn ? (long)o.heads * K : (long)o.heads * o.M;
      const long a_cols = o.a_mn ? o.M : K;
      if (!map2d(&tm[i], o.A, a_rows, a_cols, 64, o.a_mn ? 64 : 128)) return cudaErrorInvalidValue;
    }
    if (nops == 1) tm[1] = tm[0];
    if (!map2d(&tx, X + (long)n0 * x_cols, nn, x_cols, 64, g.n_pad)) return cudaErrorInvalidValue;
    g.items = items;
    const size_t smem = smem_for(g.n_pad);
    cudaError_t e;
    if (cluster) {
      // one item per CTA; the splits of a tile form one cluster, and the slices
      // they send each other ([split][n_pad][rows] fp32) reuse the drained stage
      // ring
      const int S = ops[0].splits;
      if ((size_t)g.stages * stage_bytes < (size_t)S * 4 * ((32 + S - 1) / S) * g.n_pad * 4)
        return cudaErrorInvalidValue;
      g.cluster = ops[0].splits;
      g.items_per_cta = 1;
      e = launch_pdl_cluster(gemm_sm100_kernel, dim3(items), dim3(kThreads), smem, s, g.cluster,
                             tm[0], tm[1], tx, g);
    } else {
      // persistent CTAs: at most two per SM, each over a contiguous range of items
      const int max_ctas = 2 * sm_count();
      g.items_per_cta = (items + max_ctas - 1) / max_ctas;
      const int ctas = (items + g.items_per_cta - 1) / g.items_per_cta;
      e = launch_pdl(gemm_sm100_kernel, dim3(ctas), dim3(kThreads), smem, s, tm[0], tm[1], tx, g);
    }
    if (e != cudaSuccess) return e;
  }
  return cudaSuccess;
}

}  // namespace sm100
}  // namespace mla
