// Latent decode attention on sm_100a tensor cores (bf16, 128 heads, 576-wide
// cache rows = 512 latent + 64 shared RoPE key, 64-row pages).
//
// The method: every head of a sequence scores the same cached rows, so the
// 128 absorbed queries q_lat form a dense [128 x 576] operand and each 64-row
// page is one [64 x 576] tile: S = q_lat . tile^T and O += P . tile[:, :512]
// are genuine tensor-core contractions ("从零理解 MLA", 解耦 RoPE absorbed_step:
// s_c + s_r against the cached [c ; k_R] rows, softmax, z = attn . c;
// "解耦 RoPE（MLA 下）" §3.3: one k_R shared by all heads, i.e. MQA-shaped).
//
// Design (one CTA pair = a 2-CTA cluster per work partition):
//  * The fp32 accumulator O = 128 x 512 would fill all 512 TMEM columns, so
//    CTA r owns latent columns [256 r, 256 r + 256) of O and loads only its
//    half of each page plus half of the k_R columns (288 of the 576 columns):
//    every cached byte crosses HBM once.
//  * Each CTA computes a partial score over its 288 columns (tcgen05.mma,
//    M = 128 heads, N = 64 rows, K = 288) and sends it to its partner through
//    distributed shared memory; both add the two halves in the same order and
//    run the identical online softmax (one TMEM lane = one head = one thread,
//    exp2 domain, lazy rescale when the running max grows by more than 2^8).
//  * P (bf16) goes to shared memory; O_half += P . V_half on tcgen05 (N = 256).
//  * Warp roles: warps 0-3 softmax + epilogue, warp 4 TMA producer, warp 5
//    TMEM allocation + MMA issue.  Tiles stream through a 2-stage TMA ring.
//  * Partitions come from the plan kernel (equal page counts); a sequence cut
//    by a partition boundary writes an unnormalised partial that the combine
//    kernel merges.
//  * Every wait is bounded (globaltimer); on expiry the kernel records
//    kErrTimeout in the error word, stops issuing work, drains what it issued
//    and exits.  No TMA multicast is used.
#include <cuda.h>

#include "ptx.cuh"
#include "sm100.h"

namespace mla {
namespace sm100 {
namespace {

using namespace ptx;

constexpr int kHeads = 128;
constexpr int kRow = 576;        // cached values per row
constexpr int kDc = 512;
constexpr int kPage = 64;
constexpr int kHalf = 256;       // latent columns per CTA
constexpr int kStages = 2;
constexpr int kThreads = 192;
constexpr uint64_t kTimeoutNs = 2000000000ull;

// Shared memory (byte offsets from a 1024-byte aligned base).
constexpr int kQChunk = 128 * 128;               // 128 heads x 64 bf16, 128B swizzle
constexpr int kQRope = 128 * 64;                 // 128 heads x 32 bf16, 64B swizzle
constexpr int kQBytes = 4 * kQChunk + kQRope;    // 72 KB
constexpr int kKChunk = kPage * 128;             // 64 rows x 64 bf16, 128B swizzle
constexpr int kKRope = kPage * 64;               // 64 rows x 32 bf16, 64B swizzle
constexpr int kStageBytes = 4 * kKChunk + kKRope;  // 36 KB
constexpr int kPBytes = 128 * 128;               // P: 128 heads x 64 bf16
constexpr int kXBytes = 128 * 64 * 4;            // partner's partial scores
constexpr int kOffQ = 0;
constexpr int kOffStage = kOffQ + kQBytes;
constexpr int kOffP = kOffStage + kStages * kStageBytes;
constexpr int kOffX = kOffP + kPBytes;
constexpr int kOffBar = kOffX + kXBytes;
constexpr int kSmemBytes = kOffBar + 256 + 1024;

// TMEM columns
constexpr uint32_t kTmemO = 0;     // O_half: 256 fp32 columns
constexpr uint32_t kTmemS = 256;   // S: 64 fp32 columns
constexpr uint32_t kTmemCols = 512;

constexpr uint32_t kIdescS = idesc_bf16(128, 64, 0, 0);    // A = Q (K-major), B = rows (K-major)
constexpr uint32_t kIdescPV = idesc_bf16(128, 256, 0, 1);  // A = P (K-major), B = V (MN-major)

struct Bars {
  uint64_t full[kStages], empty[kStages];
  uint64_t q_full, q_empty, s_full, s_free, p_full, pv_done, x_full, peer_free, drain;
  uint32_t tmem_base;
  volatile int abort;
};

struct Ctx {
  Bars *bars;
  int *err;
};

// Bounded wait; returns false (and flags the CTA) once the limit passes.
template <bool kCluster>
__device__ __forceinline__ bool wait_bar(const Ctx &c, uint64_t *bar, uint32_t parity) {
  const uint32_t a = smem_u32(bar);
  if (kCluster ? mbar_try_wait_cluster(a, parity) : mbar_try_wait(a, parity)) return true;
  const uint64_t t0 = globaltimer();
  while (true) {
    if (kCluster ? mbar_try_wait_cluster(a, parity) : mbar_try_wait(a, parity)) return true;
    if (c.bars->abort) return false;
    if (globaltimer() - t0 > kTimeoutNs) {
      set_error(c.err, kErrTimeout);
      c.bars->abort = 1;
      return false;
    }
  }
}

__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
  const __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<const uint32_t *>(&v);
}

__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kThreads, 1)
    attn_sm100_kernel(const __grid_constant__ CUtensorMap tm_kv,
                      const __grid_constant__ CUtensorMap tm_kr,
                      const __grid_constant__ CUtensorMap tm_q,
                      const __grid_constant__ CUtensorMap tm_qr, const AttnArgs a,
                      const float scale_log2) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  Bars *bars = reinterpret_cast<Bars *>(smem + kOffBar);
  const Ctx ctx{bars, a.err};
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const uint32_t peer = rank ^ 1u;
  const int part = blockIdx.x >> 1;
  const PlanHeader hdr = *a.hdr;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&bars->full[s], 1);
      mbar_init(&bars->empty[s], 1);
    }
    mbar_init(&bars->q_full, 1);
    mbar_init(&bars->q_empty, 1);
    mbar_init(&bars->s_full, 1);
    mbar_init(&bars->s_free, 4);
    mbar_init(&bars->p_full, 4);
    mbar_init(&bars->pv_done, 1);
    mbar_init(&bars->x_full, 128);
    mbar_init(&bars->peer_free, 128);
    mbar_init(&bars->drain, 1);
    bars->abort = 0;
    fence_mbar_init();
  }
  if (warp == 4 && lane == 0) {
    prefetch_tmap(&tm_kv);
    prefetch_tmap(&tm_kr);
    prefetch_tmap(&tm_q);
    prefetch_tmap(&tm_qr);
  }
  if (warp == 5) {
    tmem_alloc(&bars->tmem_base, kTmemCols);
    tc_fence_before();
  }
  __syncthreads();
  tc_fence_after();
  cluster_sync();  // the partner's barriers exist before any remote arrive
  const uint32_t tmem = bars->tmem_base;

  SegmentWalker walk;
  walk.init(a, hdr, part);
  Segment seg;

  if (warp == 4) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      int tile = 0, nseg = 0;
      uint8_t *qs = smem + kOffQ;
      while (walk.next(a, seg)) {
        if (nseg > 0 && !wait_bar<false>(ctx, &bars->q_empty, (nseg - 1) & 1)) break;
        mbar_expect_tx(&bars->q_full, kQBytes);
        const int qy = seg.b * kHeads;
        for (int i = 0; i < 4; ++i)
          tma_load_2d(qs + i * kQChunk, &tm_q, kHalf * rank + 64 * i, qy, &bars->q_full);
        tma_load_2d(qs + 4 * kQChunk, &tm_qr, kDc + 32 * rank, qy, &bars->q_full);
        bool ok = true;
        for (int lp = seg.lp0; lp < seg.lp1; ++lp, ++tile) {
          const int st = tile % kStages;
          if (tile >= kStages &&
              !wait_bar<false>(ctx, &bars->empty[st], ((tile / kStages) - 1) & 1)) {
            ok = false;
            break;
          }
          int page = a.block_table[(long)seg.b * a.max_pages + lp];
          if (page < 0 || page >= a.num_pages) {
            set_error(a.err, kErrRange);
            a.bad[seg.b] = 1;
            page = 0;
          }
          uint8_t *dst = smem + kOffStage + st * kStageBytes;
          mbar_expect_tx(&bars->full[st], kStageBytes);
          const int y = page * kPage;
          for (int i = 0; i < 4; ++i)
            tma_load_2d(dst + i * kKChunk, &tm_kv, kHalf * rank + 64 * i, y, &bars->full[st]);
          tma_load_2d(dst + 4 * kKChunk, &tm_kr, kDc + 32 * rank, y, &bars->full[st]);
        }
        ++nseg;
        if (!ok) break;
      }
      // drain: every issued load must land before the CTA may exit
      for (int t = tile - kStages; t < tile; ++t)
        if (t >= 0) wait_bar<false>(ctx, &bars->full[t % kStages], (t / kStages) & 1);
      if (nseg > 0) wait_bar<false>(ctx, &bars->q_full, (nseg - 1) & 1);
    }
  } else if (warp == 5) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      const uint32_t q_base = smem_u32(smem + kOffQ);
      const uint32_t p_base = smem_u32(smem + kOffP);
      int tile = 0, nseg = 0;
      int prev_stage = 0, prev_first = 0;
      bool ok = true;
      auto issue_pv = [&](int t, int stage, int first) -> bool {
        if (!wait_bar<false>(ctx, &bars->p_full, t & 1)) return false;
        tc_fence_after();
        const uint32_t v_base = smem_u32(smem + kOffStage + stage * kStageBytes);
        for (int k = 0; k < kPage / 16; ++k) {
          // A: P rows (heads) x 16 tokens; B: 16 tokens x 256 latent (MN-major,
          // 64-column chunks 8 KB apart, 8-token groups 1 KB apart)
          const uint64_t ad = sdesc(p_base + 32 * k, 16, 1024, 2);
          const uint64_t bd = sdesc(v_base + 2048 * k, kKChunk, 1024, 2);
          umma_bf16(tmem + kTmemO, ad, bd, kIdescPV, (first && k == 0) ? 0u : 1u);
        }
        umma_commit(&bars->pv_done);
        umma_commit(&bars->empty[stage]);
        return true;
      };
      while (ok && walk.next(a, seg)) {
        for (int lp = seg.lp0; lp < seg.lp1; ++lp, ++tile) {
          const int st = tile % kStages;
          if (!wait_bar<false>(ctx, &bars->full[st], (tile / kStages) & 1)) { ok = false; break; }
          if (lp == seg.lp0 && !wait_bar<false>(ctx, &bars->q_full, nseg & 1)) { ok = false; break; }
          if (tile > 0 && !wait_bar<false>(ctx, &bars->s_free, (tile - 1) & 1)) { ok = false; break; }
          tc_fence_after();
          const uint32_t k_base = smem_u32(smem + kOffStage + st * kStageBytes);
          int kk = 0;
          for (int i = 0; i < 4; ++i)       // latent columns: 4 chunks of 64, 128B swizzle
            for (int k = 0; k < 4; ++k, ++kk) {
              const uint64_t ad = sdesc(q_base + i * kQChunk + 32 * k, 16, 1024, 2);
              const uint64_t bd = sdesc(k_base + i * kKChunk + 32 * k, 16, 1024, 2);
              umma_bf16(tmem + kTmemS, ad, bd, kIdescS, kk ? 1u : 0u);
            }
          for (int k = 0; k < 2; ++k) {     // RoPE columns: 32 wide, 64B swizzle
            const uint64_t ad = sdesc(q_base + 4 * kQChunk + 32 * k, 16, 512, 4);
            const uint64_t bd = sdesc(k_base + 4 * kKChunk + 32 * k, 16, 512, 4);
            umma_bf16(tmem + kTmemS, ad, bd, kIdescS, 1u);
          }
          if (lp == seg.lp1 - 1) umma_commit(&bars->q_empty);
          umma_commit(&bars->s_full);
          if (tile > 0 && !issue_pv(tile - 1, prev_stage, prev_first)) { ok = false; ++tile; break; }
          prev_stage = st;
          prev_first = lp == seg.lp0;
        }
        ++nseg;
      }
      if (ok && tile > 0) issue_pv(tile - 1, prev_stage, prev_first);
      // drain: wait for every issued MMA before TMEM is released
      umma_commit(&bars->drain);
      wait_bar<false>(ctx, &bars->drain, 0);
    }
  } else {
    // ------------------------------------------------ softmax + epilogue (128 threads)
    const int t = threadIdx.x;               // head index == TMEM lane
    const uint32_t lane_off = static_cast<uint32_t>(warp * 32) << 16;
    float *xbuf = reinterpret_cast<float *>(smem + kOffX);
    const uint32_t x_row = smem_u32(xbuf) + t * 256;
    const uint32_t peer_x_row = mapa(x_row, peer);
    const uint32_t peer_x_full = mapa(smem_u32(&bars->x_full), peer);
    const uint32_t peer_free = mapa(smem_u32(&bars->peer_free), peer);
    uint8_t *pbuf = smem + kOffP;
    int tile = 0;
    bool ok = true;
    while (ok && walk.next(a, seg)) {
      float m_run = -INFINITY, l_run = 0.f;
      for (int lp = seg.lp0; lp < seg.lp1; ++lp, ++tile) {
        const int n_valid = min(kPage, seg.len - lp * kPage);
        const int st = tile % kStages;
        if (!wait_bar<false>(ctx, &bars->s_full, tile & 1)) { ok = false; break; }
        tc_fence_after();
        float s[64];
        {
          uint32_t r[32];
          tmem_ld32(tmem + lane_off + kTmemS, r);
          tmem_wait_ld();
#pragma unroll
          for (int k = 0; k < 32; ++k) s[k] = __uint_as_float(r[k]);
          tmem_ld32(tmem + lane_off + kTmemS + 32, r);
          tmem_wait_ld();
#pragma unroll
          for (int k = 0; k < 32; ++k) s[32 + k] = __uint_as_float(r[k]);
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&bars->s_free);
        // exchange partial scores with the partner CTA
        if (tile > 0 && !wait_bar<true>(ctx, &bars->peer_free, (tile - 1) & 1)) { ok = false; break; }
#pragma unroll
        for (int i = 0; i < 16; ++i)
          st_cluster_v4(peer_x_row + ((i ^ (t & 15)) << 4), s[4 * i], s[4 * i + 1], s[4 * i + 2],
                        s[4 * i + 3]);
        mbar_arrive_cluster(peer_x_full);
        if (!wait_bar<true>(ctx, &bars->x_full, tile & 1)) { ok = false; break; }
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          const float4 v = *reinterpret_cast<const float4 *>(
              reinterpret_cast<const uint8_t *>(xbuf) + t * 256 + ((i ^ (t & 15)) << 4));
          // rank 0 adds (own + partner), rank 1 (partner + own): the same sum
          if (rank == 0) {
            s[4 * i] += v.x; s[4 * i + 1] += v.y; s[4 * i + 2] += v.z; s[4 * i + 3] += v.w;
          } else {
            s[4 * i] = v.x + s[4 * i]; s[4 * i + 1] = v.y + s[4 * i + 1];
            s[4 * i + 2] = v.z + s[4 * i + 2]; s[4 * i + 3] = v.w + s[4 * i + 3];
          }
        }
        mbar_arrive_cluster(peer_free);
        // online softmax in the exp2 domain
        float mx = -INFINITY;
#pragma unroll
        for (int k = 0; k < 64; ++k) {
          s[k] = k < n_valid ? s[k] * scale_log2 : -INFINITY;
          mx = fmaxf(mx, s[k]);
        }
        const bool first = lp == seg.lp0;
        const bool grow = mx > m_run + 8.0f;
        float alpha = 1.f;
        if (grow) {
          alpha = exp2f(m_run - mx);
          m_run = mx;
        }
        float sum = 0.f;
        uint32_t pk[32];
#pragma unroll
        for (int k = 0; k < 32; ++k) {
          const float p0 = exp2f(s[2 * k] - m_run), p1 = exp2f(s[2 * k + 1] - m_run);
          sum += p0 + p1;
          pk[k] = pack_bf16(p0, p1);
        }
        l_run = l_run * alpha + sum;
        // P buffer and O are free once the previous tile's P.V has completed
        if (tile > 0 && !wait_bar<false>(ctx, &bars->pv_done, (tile - 1) & 1)) { ok = false; break; }
        tc_fence_after();
        if (!first && __any_sync(0xffffffffu, grow)) {
          for (int c = 0; c < kHalf; c += 32) {
            uint32_t r[32];
            tmem_ld32(tmem + lane_off + kTmemO + c, r);
            tmem_wait_ld();
#pragma unroll
            for (int k = 0; k < 32; ++k) r[k] = __float_as_uint(__uint_as_float(r[k]) * alpha);
            tmem_st32(tmem + lane_off + kTmemO + c, r);
          }
          tmem_wait_st();
        }
        // P row t: 8 chunks of 16 bytes, 128-byte swizzle (chunk j at j ^ (t % 8))
#pragma unroll
        for (int j = 0; j < 8; ++j)
          *reinterpret_cast<uint4 *>(pbuf + t * 128 + ((j ^ (t & 7)) << 4)) =
              make_uint4(pk[4 * j], pk[4 * j + 1], pk[4 * j + 2], pk[4 * j + 3]);
        if (n_valid < kPage) {
          // rows past the sequence end hold arbitrary bytes: zero their latent
          // part so that 0 * garbage cannot reach O
          uint8_t *stg = smem + kOffStage + st * kStageBytes;
          const int nz = (kPage - n_valid) * 32;   // 16-byte pieces over 4 chunks
          for (int i = t; i < nz; i += 128) {
            const int row = n_valid + (i >> 5), piece = i & 31;
            *reinterpret_cast<uint4 *>(stg + (piece >> 3) * kKChunk + row * 128 +
                                       (piece & 7) * 16) = make_uint4(0, 0, 0, 0);
          }
        }
        fence_proxy_async_smem();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&bars->p_full);
        if (lp == seg.lp1 - 1) {
          // ---------------------------------------------------- epilogue
          if (!wait_bar<false>(ctx, &bars->pv_done, tile & 1)) { ok = false; ++tile; break; }
          tc_fence_after();
          const int pb = a.part_base[seg.b];
          const bool whole = pb < 0;
          const long row_idx = (long)seg.b * kHeads + t;
          const int slot = whole ? 0 : pb + (part - seg.s0 / hdr.quota);
          const float inv_l = 1.f / l_run;
          for (int c = 0; c < kHalf; c += 32) {
            uint32_t r[32];
            tmem_ld32(tmem + lane_off + kTmemO + c, r);
            tmem_wait_ld();
            if (whole) {
              __nv_bfloat16 *z = reinterpret_cast<__nv_bfloat16 *>(a.z) + row_idx * kDc +
                                 kHalf * rank + c;
#pragma unroll
              for (int j = 0; j < 4; ++j) {
                uint4 v;
                v.x = pack_bf16(__uint_as_float(r[8 * j + 0]) * inv_l, __uint_as_float(r[8 * j + 1]) * inv_l);
                v.y = pack_bf16(__uint_as_float(r[8 * j + 2]) * inv_l, __uint_as_float(r[8 * j + 3]) * inv_l);
                v.z = pack_bf16(__uint_as_float(r[8 * j + 4]) * inv_l, __uint_as_float(r[8 * j + 5]) * inv_l);
                v.w = pack_bf16(__uint_as_float(r[8 * j + 6]) * inv_l, __uint_as_float(r[8 * j + 7]) * inv_l);
                *reinterpret_cast<uint4 *>(z + 8 * j) = v;
              }
            } else {
              float *o = a.part_O + ((long)slot * kHeads + t) * kDc + kHalf * rank + c;
#pragma unroll
              for (int j = 0; j < 8; ++j)
                *reinterpret_cast<uint4 *>(o + 4 * j) =
                    make_uint4(r[4 * j], r[4 * j + 1], r[4 * j + 2], r[4 * j + 3]);
            }
          }
          if (rank == 0) {
            const float ln2 = 0.6931471805599453f;
            if (whole) {
              if (a.lse) a.lse[row_idx] = (m_run + log2f(l_run)) * ln2;
            } else {
              a.part_m[(long)slot * kHeads + t] = m_run * ln2;
              a.part_l[(long)slot * kHeads + t] = l_run;
            }
          }
          tc_fence_before();
        }
      }
    }
  }

  __syncthreads();
  cluster_sync();  // the partner no longer touches this CTA's shared memory
  if (warp == 5) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

// ------------------------------------------------------------------ host side

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

// 2-D bf16 map over `rows` rows of 576 values; box = box_cols x box_rows.
bool make_map(CUtensorMap *m, const void *base, long rows, int box_cols, int box_rows,
              CUtensorMapSwizzle sw) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) return false;
  const cuuint64_t dims[2] = {(cuuint64_t)kRow, (cuuint64_t)rows};
  const cuuint64_t strides[1] = {(cuuint64_t)kRow * 2};
  const cuuint32_t box[2] = {(cuuint32_t)box_cols, (cuuint32_t)box_rows};
  const cuuint32_t estr[2] = {1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(base), dims, strides, box,
             estr, CU_TENSOR_MAP_INTERLEAVE_NONE, sw, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

cudaError_t launch_attn(const AttnArgs &a, int parts, cudaStream_t s) {
  static bool attr_set = false;
  if (!attr_set) {
    cudaError_t e = cudaFuncSetAttribute(attn_sm100_kernel,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
    if (e != cudaSuccess) return e;
    attr_set = true;
  }
  CUtensorMap tm_kv, tm_kr, tm_q, tm_qr;
  const long pool_rows = (long)a.num_pages * kPage;
  const long q_rows = (long)a.batch * kHeads;
  if (!make_map(&tm_kv, a.pool, pool_rows, 64, kPage, CU_TENSOR_MAP_SWIZZLE_128B) ||
      !make_map(&tm_kr, a.pool, pool_rows, 32, kPage, CU_TENSOR_MAP_SWIZZLE_64B) ||
      !make_map(&tm_q, a.q_lat, q_rows, 64, kHeads, CU_TENSOR_MAP_SWIZZLE_128B) ||
      !make_map(&tm_qr, a.q_lat, q_rows, 32, kHeads, CU_TENSOR_MAP_SWIZZLE_64B))
    return cudaErrorInvalidValue;
  const float scale_log2 = a.scale * 1.4426950408889634f;
  attn_sm100_kernel<<<2 * parts, kThreads, kSmemBytes, s>>>(tm_kv, tm_kr, tm_q, tm_qr, a,
                                                            scale_log2);
  return cudaGetLastError();
}

}  // namespace sm100
}  // namespace mla
