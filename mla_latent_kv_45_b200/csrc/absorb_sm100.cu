// Fused query absorption on sm_100a tensor cores: one CTA per head i computes
//   q_C,i = W_UQ,i x        (128 x K times K x B; rounded to bf16),
//   q_R,i = RoPE_pos(W_QR,i x),
//   q~_i  = W_UK,i^T q_C,i  (512 x 128 times 128 x B)
// and writes q_lat[b][i] = [q~_i ; q_R,i] ("从零理解 MLA", 矩阵吸收 and 查询压缩:
// the content query is folded through the key up-projection into latent
// space; 解耦 RoPE: q^R = RoPE(W^QR c_Q)).  x is c_Q (with query compression)
// or h, [batch][K] bf16.
//
// One 128-row tile of W_UQ is exactly one head's q_C, so the second product
// runs in the same CTA on the tile it just accumulated: q_C never leaves the
// SM, and the query RoPE happens in the epilogue of the W_QR product.  The
// weights are streamed once through a TMA ring (weights do not depend on the
// previous kernel, so the first stages are requested before waiting for it).
//
// Per chunk of 64 K columns the ring holds a W_UQ,i tile (128 rows), head i's
// 64 W_QR rows in the first half of a 128-row tile (the MMA runs at M = 128;
// the second half holds whatever an earlier chunk left there, and its 64
// output rows are never read) and the chunk of x.  After the K loop the same ring carries W_UK,i
// (read MN-major as W_UK,i^T, four 128-row M tiles).  D accumulates in TMEM
// with a column stride w (the padded batch rounded up to 32): q_C at columns
// [0, w), q_R at [w, 2w); then q~ tile t at [t w, (t + 1) w), written once the
// epilogue has read q_C and q_R.
//
// Warp roles: warp 0 TMA producer, warp 1 TMEM allocation + MMA issue, warps
// 2-5 epilogue.  Every wait is bounded (globaltimer); a timeout sets the error
// word and the CTA stops.
#include <cuda.h>

#include <atomic>

#include "api_checks.h"
#include "ptx.cuh"
#include "sm100.h"

namespace mla {
namespace sm100 {
namespace {

using namespace ptx;

constexpr int kThreads = 192;
constexpr int kH = 128;
constexpr int kRowLat = 576;
constexpr uint64_t kTimeoutNs = 2000000000ull;   // 2 s: every bounded wait
constexpr int kTile = 128 * 128;       // 128 rows x 64 bf16 (one A operand chunk)
constexpr int kMaxStages = 6;
constexpr int kSmemLimit = 232448;
constexpr int kRopeAhead = 16;         // q_R pairs per epilogue thread with angles ahead (batch <= 64)

struct Bars {
  uint64_t full[kMaxStages], empty[kMaxStages], acc1_full, qc_ready, acc2_full, drain;
  uint32_t tmem_base;
  volatile int abort;
};

struct AbsorbArgs {
  int n, n0, n_pad, n_cols, k_chunks, stages, tmem_cols, stage_bytes;
  int off_qc, off_qr, off_bar;
  const int32_t *positions;
  __nv_bfloat16 *q_lat;
  RopeParams rp;
  int *err;
  uint64_t timeout_ns;   // limit of every wait
  int skip_qc_arrive;    // test hook: one epilogue warp withholds its q_C-ready arrive
};

__device__ __forceinline__ bool await(Bars *bars, int *err, uint64_t *bar, uint32_t parity,
                                      uint64_t limit) {
  const uint32_t a = smem_u32(bar);
  if (mbar_try_wait(a, parity)) return true;
  const uint64_t t0 = globaltimer();
  while (true) {
    if (mbar_try_wait_sleep(a, parity, 20000)) return true;
    if (bars->abort) return false;
    if (globaltimer() - t0 > limit) {
      set_error(err, kErrTimeout);
      bars->abort = 1;
      return false;
    }
  }
}

__device__ __forceinline__ void epi_sync() { asm volatile("bar.sync 1, 128;" ::: "memory"); }

__global__ void __launch_bounds__(kThreads, 1)
    absorb_sm100_kernel(const __grid_constant__ CUtensorMap tm_uq,
                        const __grid_constant__ CUtensorMap tm_qr,
                        const __grid_constant__ CUtensorMap tm_uk,
                        const __grid_constant__ CUtensorMap tm_x, const AbsorbArgs g) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  Bars *bars = reinterpret_cast<Bars *>(smem + g.off_bar);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int head = blockIdx.x;
  const int nk1 = g.k_chunks;          // K chunks of the first products
  const int nk = nk1 + 4;              // + four W_UK,i tiles (two K chunks each)

  if (threadIdx.x == 0) {
    for (int s = 0; s < g.stages; ++s) {
      mbar_init(&bars->full[s], 1);
      mbar_init(&bars->empty[s], 1);
    }
    mbar_init(&bars->acc1_full, 1);
    mbar_init(&bars->qc_ready, 4);
    mbar_init(&bars->acc2_full, 1);
    mbar_init(&bars->drain, 1);
    bars->abort = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tmap(&tm_uq);
    prefetch_tmap(&tm_qr);
    prefetch_tmap(&tm_uk);
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
      const uint32_t tx1 = kTile + kTile / 2 + g.n_pad * 128;
      auto load_w = [&](int c, int st) {
        uint8_t *dst = smem + st * g.stage_bytes;
        if (c < nk1) {
          tma_load_2d(dst, &tm_uq, 64 * c, head * 128, &bars->full[st]);
          tma_load_2d(dst + kTile, &tm_qr, 64 * c, head * 64, &bars->full[st]);
        } else {
          // M tile t of W_UK,i^T: latent columns [128 t, 128 t + 128), both 64-row K chunks
          const int t = c - nk1;
          for (int kc = 0; kc < 2; ++kc)
            for (int half = 0; half < 2; ++half)
              tma_load_2d(dst + kc * kTile + half * (kTile / 2), &tm_uk, 128 * t + 64 * half,
                          head * 128 + 64 * kc, &bars->full[st]);
        }
      };
      auto tx_of = [&](int c) { return c < nk1 ? tx1 : (uint32_t)(2 * kTile); };
      int pre = 0;   // stages whose weights were requested before waiting for the predecessor
      for (; pre < g.stages && pre < nk; ++pre) {
        mbar_expect_tx(&bars->full[pre], tx_of(pre));
        load_w(pre, pre);
      }
      grid_dep_wait();
      grid_dep_launch();
      int c = 0;
      for (; c < nk; ++c) {
        const int st = c % g.stages;
        if (c >= g.stages && !await(bars, g.err, &bars->empty[st], ((c / g.stages) - 1) & 1, g.timeout_ns))
          break;
        if (c >= pre) {
          mbar_expect_tx(&bars->full[st], tx_of(c));
          load_w(c, st);
        }
        if (c < nk1)
          tma_load_2d(smem + st * g.stage_bytes + 2 * kTile, &tm_x, 64 * c, g.n0, &bars->full[st]);
      }
      // the CTA may not exit with loads in flight
      for (int i = max(c - g.stages, 0); i < max(c, pre); ++i) {
        const uint32_t a = smem_u32(&bars->full[i % g.stages]);
        const uint64_t t0 = globaltimer();
        while (!mbar_try_wait_sleep(a, (i / g.stages) & 1, 20000))
          if (globaltimer() - t0 > g.timeout_ns) break;
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      const uint32_t idesc1 = idesc_bf16(128, g.n_pad, 0, 0);
      const uint32_t idesc2 = idesc_bf16(128, g.n_pad, 1, 0);
      const uint32_t d_qc = tmem, d_qr = tmem + g.n_cols;
      bool ok = true;
      int c = 0;
      for (; c < nk1; ++c) {
        const int st = c % g.stages;
        if (!await(bars, g.err, &bars->full[st], (c / g.stages) & 1, g.timeout_ns)) { ok = false; break; }
        tc_fence_after();
        const uint32_t base = smem_u32(smem + st * g.stage_bytes);
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          const uint64_t bd = sdesc(base + 2 * kTile + 32 * k, 16, 1024, 2);
          const uint32_t acc = (c > 0 || k > 0) ? 1u : 0u;
          umma_bf16(d_qc, sdesc(base + 32 * k, 16, 1024, 2), bd, idesc1, acc);
          umma_bf16(d_qr, sdesc(base + kTile + 32 * k, 16, 1024, 2), bd, idesc1, acc);
        }
        umma_commit(&bars->empty[st]);
      }
      if (ok) {
        umma_commit(&bars->acc1_full);
        // q_C (bf16, K-major B operand) written and q_C / q_R read out of TMEM
        ok = await(bars, g.err, &bars->qc_ready, 0, g.timeout_ns);
        tc_fence_after();
      }
      const uint32_t qc = smem_u32(smem + g.off_qc);
      for (int t = 0; ok && t < 4; ++t, ++c) {
        const int st = c % g.stages;
        if (!await(bars, g.err, &bars->full[st], (c / g.stages) & 1, g.timeout_ns)) { ok = false; break; }
        tc_fence_after();
        const uint32_t base = smem_u32(smem + st * g.stage_bytes);
        for (int kc = 0; kc < 2; ++kc) {
#pragma unroll
          for (int k = 0; k < 4; ++k)
            umma_bf16(tmem + t * g.n_cols, sdesc(base + kc * kTile + 2048 * k, kTile / 2, 1024, 2),
                      sdesc(qc + kc * g.n_pad * 128 + 32 * k, 16, 1024, 2), idesc2,
                      (kc > 0 || k > 0) ? 1u : 0u);
        }
        umma_commit(&bars->empty[st]);
      }
      if (ok) umma_commit(&bars->acc2_full);
      umma_commit(&bars->drain);
      const uint32_t a = smem_u32(&bars->drain);
      const uint64_t t0 = globaltimer();
      while (!mbar_try_wait_sleep(a, 0, 20000))
        if (globaltimer() - t0 > g.timeout_ns) break;
    }
  } else {
    // ---------------------------------------------- epilogue: warps 2..5
    const int quad = warp & 3;             // TMEM lanes [32 quad, 32 quad + 32)
    const int row = quad * 32 + lane;
    const uint32_t lane_off = static_cast<uint32_t>(quad * 32) << 16;
    grid_dep_wait();                       // positions and q_lat follow the predecessor
    // The rotation angles of this thread's q_R pairs (w = tid + 128 k: sequence
    // w / 32, pair w % 32) depend only on the positions: their cosines and sines
    // are computed here, while the weights stream, instead of after the K loop.
    const int half = g.rp.d_rope / 2;
    const int tid = threadIdx.x - 64;
    float rc[kRopeAhead], rsn[kRopeAhead];
#pragma unroll
    for (int k = 0; k < kRopeAhead; ++k) {
      const int w = tid + 128 * k;
      rc[k] = 1.f;
      rsn[k] = 0.f;
      if (w < g.n * half) rope_cos_sin(g.positions[g.n0 + w / half], g.rp.theta[w % half], rc[k], rsn[k]);
    }
    uint8_t *qc = smem + g.off_qc;
    float *qr = reinterpret_cast<float *>(smem + g.off_qr);   // [n_pad][64]
    bool ok = await(bars, g.err, &bars->acc1_full, 0, g.timeout_ns);
    tc_fence_after();
    // q_C,i[n][a] (a = row) rounded to bf16 into the K-major operand: chunk a / 64,
    // row n, 16-byte unit (a % 64) / 8 swizzled with n & 7
    const int kc = row >> 6, u = (row & 63) >> 3, e = row & 7;
    for (int c0 = 0; c0 < g.n_pad; c0 += 32) {
      float v[32];
      tmem_ld32f(tmem + lane_off + c0, v);
      tmem_wait_ld();
#pragma unroll
      for (int j = 0; j < 32; ++j) {
        const int n = c0 + j;
        if (n < g.n_pad)
          *reinterpret_cast<__nv_bfloat16 *>(qc + kc * g.n_pad * 128 + n * 128 +
                                             ((u ^ (n & 7)) << 4) + e * 2) =
              __float2bfloat16_rn(v[j]);
      }
    }
    if (quad < 2) {
      // q_R of this head (TMEM lanes 0..63), unrotated, fp32; lanes 64..127
      // come from the unloaded half of the W_QR tile and are not read
      for (int c0 = 0; c0 < g.n_pad; c0 += 32) {
        float v[32];
        tmem_ld32f(tmem + lane_off + g.n_cols + c0, v);
        tmem_wait_ld();
#pragma unroll
        for (int j = 0; j < 32; ++j)
          if (c0 + j < g.n_pad) qr[(c0 + j) * 64 + row] = v[j];
      }
    }
    fence_proxy_async_smem();              // q_C -> the W_UK MMAs
    tc_fence_before();
    __syncwarp();
    if (lane == 0 && !(g.skip_qc_arrive && quad == 0)) mbar_arrive(&bars->qc_ready);
    epi_sync();                            // q_R staging complete
    // q_R,i rotated by the sequence's position in place in the staging tile,
    // then rounded once into q_lat (each sequence's 64 values are one 128-byte
    // line of q_lat: 16 threads store it, 8 bytes each)
    auto rotate = [&](int w, float cf, float sf) {
      const int n = w / half, t = w % half;
      int j0, j1;
      rope_idx(g.rp, t, j0, j1);
      float x0 = qr[n * 64 + j0], x1 = qr[n * 64 + j1];
      rope_rotate(cf, sf, x0, x1);
      qr[n * 64 + j0] = x0;
      qr[n * 64 + j1] = x1;
    };
#pragma unroll
    for (int k = 0; k < kRopeAhead; ++k)
      if (tid + 128 * k < g.n * half) rotate(tid + 128 * k, rc[k], rsn[k]);
    for (int w = tid + 128 * kRopeAhead; w < g.n * half; w += 128) {
      float cf, sf;
      rope_cos_sin(g.positions[g.n0 + w / half], g.rp.theta[w % half], cf, sf);
      rotate(w, cf, sf);
    }
    epi_sync();
    for (int u = tid; u < g.n * 16; u += 128) {
      const int n = u >> 4, j = (u & 15) * 4;
      const float4 v = *reinterpret_cast<const float4 *>(qr + n * 64 + j);
      const __nv_bfloat162 lo = __floats2bfloat162_rn(v.x, v.y), hi = __floats2bfloat162_rn(v.z, v.w);
      uint2 pk;
      pk.x = *reinterpret_cast<const uint32_t *>(&lo);
      pk.y = *reinterpret_cast<const uint32_t *>(&hi);
      *reinterpret_cast<uint2 *>(g.q_lat + ((long)(g.n0 + n) * kH + head) * kRowLat + 512 + j) = pk;
    }
    ok = ok && await(bars, g.err, &bars->acc2_full, 0, g.timeout_ns);
    tc_fence_after();
    if (ok) {
      // q~_i: tile t holds latent columns 128 t + row for every n
      for (int t = 0; t < 4; ++t) {
        __nv_bfloat16 *dst = g.q_lat + ((long)g.n0 * kH + head) * kRowLat + 128 * t + row;
        for (int c0 = 0; c0 < g.n_pad; c0 += 32) {
          float v[32];
          tmem_ld32f(tmem + lane_off + t * g.n_cols + c0, v);
          tmem_wait_ld();
#pragma unroll
          for (int j = 0; j < 32; ++j)
            if (c0 + j < g.n) dst[(long)(c0 + j) * kH * kRowLat] = __float2bfloat16_rn(v[j]);
        }
      }
    }
    tc_fence_before();
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

// 2-D bf16 row-major [rows][cols] map, box box_cols x box_rows, 128-byte swizzle;
// rows past the end read as zeros.
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

}  // namespace

// Test hook state (see mla_debug_absorb_timeout in include/mla.h).
static std::atomic<uint64_t> g_debug_limit_ns{0};
static std::atomic<int> g_debug_skip{0};

void absorb_debug_fault(int skip_arrive, uint64_t limit_ns) {
  g_debug_skip.store(skip_arrive);
  g_debug_limit_ns.store(limit_ns);
}

cudaError_t absorb_heads(const __nv_bfloat16 *x, int K, const __nv_bfloat16 *W_UQ,
                         const __nv_bfloat16 *W_QR, const __nv_bfloat16 *W_UK, int batch,
                         const RopeParams &rp, const int32_t *positions, __nv_bfloat16 *q_lat,
                         int *err, cudaStream_t s) {
  if (K < 64 || K % 64 || batch < 1 || rp.d_rope != 64) return cudaErrorInvalidValue;
  static api::PerDeviceOnce smem_attr;
  cudaError_t e = smem_attr.run([] {
    return cudaFuncSetAttribute(absorb_sm100_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                kSmemLimit);
  });
  if (e != cudaSuccess) return e;
  CUtensorMap tm_uq, tm_qr, tm_uk;
  if (!map2d(&tm_uq, W_UQ, (long)kH * 128, K, 64, 128) ||
      !map2d(&tm_qr, W_QR, (long)kH * 64, K, 64, 64) ||
      !map2d(&tm_uk, W_UK, (long)kH * 128, 512, 64, 64))
    return cudaErrorInvalidValue;
  // batch rows in chunks of at most 128 (four q~ tiles of n columns fill TMEM)
  for (int n0 = 0; n0 < batch; n0 += 128) {
    AbsorbArgs g{};
    g.n = batch - n0 < 128 ? batch - n0 : 128;
    g.n0 = n0;
    g.n_pad = (g.n + 15) / 16 * 16;
    g.k_chunks = K / 64;
    g.n_cols = (g.n_pad + 31) / 32 * 32;   // accumulator stride: whole 32-column loads
    g.tmem_cols = 32;
    while (g.tmem_cols < 4 * g.n_cols) g.tmem_cols *= 2;
    g.stage_bytes = 2 * kTile + g.n_pad * 128;
    const int fixed = g.n_pad * 256 + g.n_pad * 256 + 1024;   // q_C operand, q_R staging, barriers
    g.stages = (kSmemLimit - 1024 - fixed) / g.stage_bytes;
    if (g.stages > kMaxStages) g.stages = kMaxStages;
    if (g.stages < 2) return cudaErrorInvalidValue;
    g.off_qc = g.stages * g.stage_bytes;
    g.off_qr = g.off_qc + g.n_pad * 256;
    g.off_bar = g.off_qr + g.n_pad * 256;
    g.positions = positions;
    g.q_lat = q_lat;
    g.rp = rp;
    g.err = err;
    const uint64_t dbg = g_debug_limit_ns.load();
    g.timeout_ns = dbg ? dbg : kTimeoutNs;
    g.skip_qc_arrive = g_debug_skip.load();
    CUtensorMap tm_x;
    if (!map2d(&tm_x, x, batch, K, 64, g.n_pad)) return cudaErrorInvalidValue;
    const size_t smem = (size_t)g.off_bar + 1024 + 1024;
    e = launch_pdl(absorb_sm100_kernel, dim3(kH), dim3(kThreads), smem, s, tm_uq, tm_qr, tm_uk,
                   tm_x, g);
    if (e != cudaSuccess) return e;
  }
  return cudaSuccess;
}

}  // namespace sm100
}  // namespace mla
