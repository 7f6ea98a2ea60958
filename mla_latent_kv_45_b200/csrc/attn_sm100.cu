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
// Design (one CTA pair = a 2-CTA cluster per work partition, pair MMAs):
//  * Scores.  One pair MMA (tcgen05 cta_group::2, M = 256, N = 64, K = 576)
//    per page: both CTAs supply the same 128 q_lat rows as A (256 columns from
//    TMEM, 320 from shared memory) and CTA r supplies page rows [32r, 32r+32)
//    as half of B, so each CTA loads half of the page yet receives the whole
//    128 x 64 score tile in its TMEM (two score buffers, so the next page's
//    scores are computed while this one's are read).  Both CTAs then run the
//    same softmax on identical scores: no score or P crosses between the CTAs.
//  * Values.  The fp32 accumulator for 128 heads x 512 latent columns would
//    fill all of TMEM, so it is held transposed and split: O^T = V^T P^T with
//    pair MMAs (M = 256 latent columns, two of them per page, N = 128 heads,
//    K = 64 rows).  CTA r owns latent columns [256b + 128r, +128) for b = 0, 1
//    (TMEM lane = latent column, TMEM column = head) and supplies heads
//    [64r, 64r+64) of P as its half of B.
//  * Once the scores of a page are complete, the stage that held the CTA's 32
//    rows (read only by the score MMA) is refilled with the page's 64 rows of
//    this CTA's latent columns (L2 hits: the pair has just streamed the page).
//  * Softmax: one thread per head (TMEM lane), two warpgroups of 32 rows each,
//    exp2 domain; the running max moves only when a tile max exceeds it by
//    more than 2^8, and only then are O^T columns rescaled in TMEM.  Row sums
//    come from the bf16 P values the MMA consumes.
//  * Warps 0-7 softmax + epilogue + q_lat TMEM staging; warp 8 loads the
//    CTA's score rows; warp 9 TMEM allocation, q_lat shared-memory loads and
//    (even CTA) the score MMAs; warp 10 (even CTA) the P.V MMAs; warp 11 the
//    latent-column loads for P.V.
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
constexpr int kOwn = 32;         // rows of a page supplied to the score MMA by each CTA
constexpr int kStages = 3;
constexpr int kSBuf = 2;   // TMEM score buffers
constexpr int kSoftmaxThreads = 256;
constexpr int kThreads = kSoftmaxThreads + 128;
constexpr int kWarpLoad = 8, kWarpS = 9, kWarpPV = 10, kWarpV = 11;
constexpr uint64_t kTimeoutNs = 2000000000ull;
constexpr uint32_t kSleepNs = 20000;   // suspend hint of a waiting thread (woken at completion)

// Shared memory (byte offsets from a 1024-byte aligned base).
constexpr int kQChunk = kHeads * 128;             // 128 heads x 64 bf16, 128-byte swizzle
constexpr int kQTmemDims = 2 * (256 - 64 * kSBuf);  // q_lat columns held in TMEM
constexpr int kQSmem = (kRow - kQTmemDims) / 64;  // the rest, in 64-column shared-memory chunks
constexpr int kChunk = kOwn * 128;                // 32 rows x 64 bf16
constexpr int kStageBytes = 9 * kChunk;           // the CTA's 32 rows, all 576 columns
constexpr int kVBox = kPage * 128;                // 64 rows x 64 latent columns
constexpr int kVBytes = 4 * kVBox;                // the CTA's 256 latent columns of a page
constexpr int kPBytes = 64 * 128;                 // P for 64 heads x 64 rows bf16
constexpr int kOffQ = 0;
constexpr int kOffStage = kOffQ + kQSmem * kQChunk;
constexpr int kOffP = kOffStage + kStages * kStageBytes;   // two P buffers
constexpr int kOffRed = kOffP + 2 * kPBytes;      // [2][128] floats: per-warpgroup scratch
constexpr int kOffAlpha = kOffRed + 1024;         // [128] rescale factors, then [128] row sums
constexpr int kOffBar = kOffAlpha + 1024;
constexpr int kSmemBytes = kOffBar + 512 + 1024;
static_assert(kVBytes <= kStageBytes, "the latent columns of a page refill its stage");

// TMEM columns
constexpr uint32_t kTmemO = 0;     // O^T: two blocks of 128 heads (lane = latent column)
constexpr uint32_t kTmemS = 256;   // S: kSBuf buffers of 64 fp32 columns
constexpr uint32_t kTmemQ = kTmemS + 64 * kSBuf;   // q_lat columns [0, kQTmemDims) as bf16 pairs
constexpr uint32_t kTmemCols = 512;

constexpr uint32_t kIdescS = idesc_bf16(256, kPage, 0, 0);   // A = q_lat (K-major), B = rows
constexpr uint32_t kIdescPV = idesc_bf16(256, 128, 1, 0);    // A = V^T (MN-major), B = P
constexpr uint16_t kBoth = 3;

struct Bars {
  uint64_t full[kStages];    // even CTA: the pair's score rows landed (tx, both CTAs)
  uint64_t empty[kStages];   // P.V of the stage's page complete (pair commit)
  uint64_t sdone[kStages];   // scores of the stage's page complete (pair commit)
  uint64_t vland[kStages];   // this CTA's latent columns landed (local tx)
  uint64_t vready[kStages];  // even CTA: both CTAs' latent columns ready (2 arrivals)
  uint64_t q_smem;           // even CTA: q_lat shared-memory part of both CTAs (tx)
  uint64_t q_tmem;           // even CTA: q_lat TMEM part staged in both CTAs (16 warps)
  uint64_t q_free;           // the segment's last score MMAs complete (pair commit)
  uint64_t s_full[kSBuf];    // scores in buffer i complete (pair commit)
  uint64_t s_free[kSBuf];    // even CTA: both CTAs read score buffer i (16 warps)
  uint64_t p_ready[2];       // even CTA: P written and O^T rescaled in both CTAs (16 warps)
  uint64_t pv_done[2];       // P.V of the tile using P buffer i complete (pair commit)
  uint64_t drain_s, drain_pv;
  uint32_t tmem_base;
  volatile int abort;
};

struct Ctx {
  Bars *bars;
  int *err;
};

// Bounded wait (acquire at cluster scope: several barriers receive remote
// arrivals or pair commits); returns false, and flags the CTA, once the limit passes.
__device__ __forceinline__ bool wait_bar(const Ctx &c, uint64_t *bar, uint32_t parity) {
  const uint32_t a = smem_u32(bar);
  if (mbar_try_wait_cluster(a, parity)) return true;
  const uint64_t t0 = globaltimer();
  while (true) {
    if (mbar_try_wait_cluster_sleep(a, parity, kSleepNs)) return true;
    if (c.bars->abort) return false;
    if (globaltimer() - t0 > kTimeoutNs) {
      set_error(c.err, kErrTimeout);
      c.bars->abort = 1;
      return false;
    }
  }
}

// Waits (bounded, ignoring the abort flag) for asynchronous work this CTA issued.
__device__ __forceinline__ void drain_bar(uint64_t *bar, uint32_t parity) {
  const uint32_t a = smem_u32(bar);
  const uint64_t t0 = globaltimer();
  while (!mbar_try_wait_cluster_sleep(a, parity, kSleepNs))
    if (globaltimer() - t0 > kTimeoutNs) return;
}

__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
  const __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<const uint32_t *>(&v);
}

__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xffff0000u); }

// Named barrier over the 256 softmax threads; the second form also returns
// whether any of them passed true.
__device__ __forceinline__ void softmax_sync() {
  asm volatile("bar.sync 1, %0;" ::"n"(kSoftmaxThreads) : "memory");
}
__device__ __forceinline__ bool softmax_any(bool p) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred a, b;\n\t"
      "setp.ne.u32 a, %1, 0;\n\t"
      "bar.red.or.pred b, 1, %2, a;\n\t"
      "selp.u32 %0, 1, 0, b;\n\t}"
      : "=r"(r)
      : "r"(static_cast<uint32_t>(p)), "n"(kSoftmaxThreads)
      : "memory");
  return r != 0;
}

// Sequential walk over the tiles (pages) of one partition.
struct TileCursor {
  SegmentWalker walk;
  Segment seg;
  int lp, nseg;
  bool valid;
  __device__ __forceinline__ void init(const AttnArgs &a, const PlanHeader &h, int part) {
    walk.init(a, h, part);
    valid = walk.next(a, seg);
    lp = seg.lp0;
    nseg = 0;
  }
  __device__ __forceinline__ void advance(const AttnArgs &a) {
    if (++lp >= seg.lp1) {
      valid = walk.next(a, seg);
      lp = seg.lp0;
      ++nseg;
    }
  }
  __device__ __forceinline__ bool first() const { return lp == seg.lp0; }
  __device__ __forceinline__ bool last() const { return lp == seg.lp1 - 1; }
  __device__ __forceinline__ int rows_valid() const { return seg.len - lp * kPage; }
  __device__ __forceinline__ int page(const AttnArgs &a) const {
    return a.block_table[(long)seg.b * a.max_pages + lp];
  }
};

// Stages q_lat[b][h][0:kQTmemDims] into TMEM lane h (bf16 pairs, blocks of 32
// columns); warpgroup g writes half of the blocks.
__device__ __forceinline__ void stage_q(const AttnArgs &a, int b, int h, int g, uint32_t taddr) {
  const uint4 *src = reinterpret_cast<const uint4 *>(
      reinterpret_cast<const __nv_bfloat16 *>(a.q_lat) + ((long)b * kHeads + h) * kRow);
  constexpr int kHalfBlocks = kQTmemDims / 128;
  for (int bb = kHalfBlocks * g; bb < kHalfBlocks * (g + 1); ++bb) {
    uint32_t v[32];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const uint4 x = src[bb * 8 + i];
      v[4 * i] = x.x; v[4 * i + 1] = x.y; v[4 * i + 2] = x.z; v[4 * i + 3] = x.w;
    }
    tmem_st32(taddr + 32 * bb, v);
  }
  tmem_wait_st();
}

__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kThreads, 1)
    attn_sm100_kernel(const __grid_constant__ CUtensorMap tm_kv,
                      const __grid_constant__ CUtensorMap tm_v,
                      const __grid_constant__ CUtensorMap tm_q, const AttnArgs a,
                      const float scale_log2) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  Bars *bars = reinterpret_cast<Bars *>(smem + kOffBar);
  const Ctx ctx{bars, a.err};
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const bool leader = rank == 0;
  const int part = blockIdx.x >> 1;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&bars->full[s], 1);
      mbar_init(&bars->empty[s], 1);
      mbar_init(&bars->sdone[s], 1);
      mbar_init(&bars->vland[s], 1);
      mbar_init(&bars->vready[s], 2);
    }
    mbar_init(&bars->q_smem, 1);
    mbar_init(&bars->q_tmem, 16);
    mbar_init(&bars->q_free, 1);
    for (int i = 0; i < kSBuf; ++i) {
      mbar_init(&bars->s_full[i], 1);
      mbar_init(&bars->s_free[i], 16);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&bars->p_ready[i], 16);
      mbar_init(&bars->pv_done[i], 1);
    }
    mbar_init(&bars->drain_s, 1);
    mbar_init(&bars->drain_pv, 1);
    bars->abort = 0;
    fence_mbar_init();
  }
  if (warp == kWarpLoad && lane == 0) {
    prefetch_tmap(&tm_kv);
    prefetch_tmap(&tm_v);
    prefetch_tmap(&tm_q);
  }
  if (warp == kWarpS) {
    tmem_alloc_pair(&bars->tmem_base, kTmemCols);
    tc_fence_before();
  }
  __syncthreads();
  tc_fence_after();
  cluster_sync();  // both CTAs' barriers exist before any remote access
  const uint32_t tmem = bars->tmem_base;
  // the set-up above overlaps the plan kernel; its results are read from here on
  grid_dep_wait();
  grid_dep_launch();
  const PlanHeader hdr = *a.hdr;
  auto lead = [&](uint64_t *bar) { return mapa(smem_u32(bar), 0); };

  TileCursor cur;
  cur.init(a, hdr, part);

  if (warp == kWarpLoad) {
    // ------------------------------- this CTA's 32 rows of each page (score B half)
    if (lane == 0) {
      int tile = 0;
      for (; cur.valid; cur.advance(a), ++tile) {
        const int st = tile % kStages;
        if (tile >= kStages && !wait_bar(ctx, &bars->empty[st], ((tile / kStages) - 1) & 1))
          break;
        int page = cur.page(a);
        if (page < 0 || page >= a.num_pages) {
          set_error(a.err, kErrRange);
          a.bad[cur.seg.b] = 1;
          page = 0;
        }
        if (leader) mbar_expect_tx(&bars->full[st], 2 * kStageBytes);
        uint8_t *dst = smem + kOffStage + st * kStageBytes;
        const uint32_t bar = lead(&bars->full[st]);
        for (int c = 0; c < 9; ++c)
          tma_load_2d_pair(dst + c * kChunk, &tm_kv, 64 * c, page * kPage + kOwn * rank, bar);
      }
    }
  } else if (warp == kWarpV) {
    // --------- after a page's scores: its 64 rows of this CTA's latent columns (P.V A)
    int tile = 0;
    for (; cur.valid; cur.advance(a), ++tile) {
      const int st = tile % kStages;
      const uint32_t par = (tile / kStages) & 1;
      if (!wait_bar(ctx, &bars->sdone[st], par)) break;
      uint8_t *dst = smem + kOffStage + st * kStageBytes;
      if (lane == 0) {
        int page = cur.page(a);
        if (page < 0 || page >= a.num_pages) page = 0;   // flagged by the row loader
        mbar_expect_tx(&bars->vland[st], kVBytes);
        // box i = (blk, sub): latent columns 256 blk + 128 r + 64 sub, all 64 rows
        for (int i = 0; i < 4; ++i)
          tma_load_2d(dst + i * kVBox, &tm_v, 256 * (i >> 1) + 128 * rank + 64 * (i & 1),
                      page * kPage, &bars->vland[st]);
      }
      if (!wait_bar(ctx, &bars->vland[st], par)) break;
      const int valid = cur.rows_valid();
      if (valid < kPage) {
        // rows past the sequence end hold arbitrary bytes: zero them so that
        // 0 * (stale bytes) cannot reach O
        for (int i = lane; i < (kPage - valid) * 32; i += 32) {
          const int row = valid + (i >> 5), box = (i >> 3) & 3, piece = i & 7;
          *reinterpret_cast<uint4 *>(dst + box * kVBox + row * 128 + piece * 16) =
              make_uint4(0, 0, 0, 0);
        }
        fence_proxy_async_smem();
      }
      __syncwarp();
      if (lane == 0) mbar_arrive_remote(lead(&bars->vready[st]));
    }
  } else if (warp == kWarpS) {
    // ------------- q_lat shared-memory part (both CTAs); the even CTA issues the scores
    if (lane == 0) {
      const uint64_t qd = sdesc(smem_u32(smem + kOffQ), 16, 1024, 2);
      int tile = 0;
      for (; cur.valid; cur.advance(a), ++tile) {
        const int st = tile % kStages;
        if (cur.first()) {
          // the previous segment's score MMAs must finish before q_lat is replaced
          if (cur.nseg > 0 && !wait_bar(ctx, &bars->q_free, (cur.nseg - 1) & 1)) break;
          if (leader) mbar_expect_tx(&bars->q_smem, 2 * kQSmem * kQChunk);
          for (int c = 0; c < kQSmem; ++c)
            tma_load_2d_pair(smem + kOffQ + c * kQChunk, &tm_q, kQTmemDims + 64 * c,
                             cur.seg.b * kHeads, lead(&bars->q_smem));
          if (leader && (!wait_bar(ctx, &bars->q_smem, cur.nseg & 1) ||
                         !wait_bar(ctx, &bars->q_tmem, cur.nseg & 1)))
            break;
        }
        if (!leader) continue;
        if (!wait_bar(ctx, &bars->full[st], (tile / kStages) & 1)) break;
        // score buffer sb was last used by tile - kSBuf
        const int sb = tile % kSBuf;
        if (tile >= kSBuf && !wait_bar(ctx, &bars->s_free[sb], ((tile / kSBuf) - 1) & 1)) break;
        const uint32_t sd = tmem + kTmemS + 64 * sb;
        tc_fence_after();
        // descriptors advance by address >> 4 in their low field (no carry: < 256 KB)
        const uint64_t kd = sdesc(smem_u32(smem + kOffStage + st * kStageBytes), 16, 1024, 2);
#pragma unroll
        for (int s = 0; s < kQTmemDims / 16; ++s)   // q_lat columns held in TMEM
          umma_pair_ts(sd, tmem + kTmemQ + 8 * s,
                       kd + (uint64_t)(((s >> 2) * kChunk + 32 * (s & 3)) >> 4), kIdescS,
                       s ? 1u : 0u);
#pragma unroll
        for (int s = 0; s < 4 * kQSmem; ++s)         // the rest from shared memory
          umma_pair_ss(sd, qd + (uint64_t)(((s >> 2) * kQChunk + 32 * (s & 3)) >> 4),
                       kd + (uint64_t)(((kQTmemDims / 64 + (s >> 2)) * kChunk + 32 * (s & 3)) >> 4),
                       kIdescS, 1u);
        if (cur.last()) umma_commit_pair(&bars->q_free, kBoth);
        umma_commit_pair(&bars->s_full[sb], kBoth);
        umma_commit_pair(&bars->sdone[st], kBoth);
      }
      if (leader) {
        umma_commit_pair(&bars->drain_s, 1);
        drain_bar(&bars->drain_s, 0);
      }
    }
  } else if (warp == kWarpPV) {
    // ------------------------------------------------- P.V pair MMAs (even CTA)
    if (lane == 0 && leader) {
      int tile = 0;
      for (; cur.valid; cur.advance(a), ++tile) {
        const int st = tile % kStages;
        const int pb = tile & 1;
        if (!wait_bar(ctx, &bars->p_ready[pb], (tile >> 1) & 1)) break;
        if (!wait_bar(ctx, &bars->vready[st], (tile / kStages) & 1)) break;
        tc_fence_after();
        const uint32_t v_base = smem_u32(smem + kOffStage + st * kStageBytes);
        const uint64_t pd = sdesc(smem_u32(smem + kOffP + pb * kPBytes), 16, 1024, 2);
        const bool first = cur.first();
#pragma unroll
        for (int blk = 0; blk < 2; ++blk) {
          // A = V^T: two 64-column boxes of 64 rows (8 KB apart), MN-major
          const uint64_t vd = sdesc(v_base + blk * 2 * kVBox, kVBox, 1024, 2);
#pragma unroll
          for (int k = 0; k < kPage / 16; ++k)
            umma_pair_ss(tmem + kTmemO + 128 * blk, vd + (uint64_t)((2048 * k) >> 4),
                         pd + (uint64_t)((32 * k) >> 4), kIdescPV, (first && k == 0) ? 0u : 1u);
        }
        umma_commit_pair(&bars->pv_done[pb], kBoth);
        umma_commit_pair(&bars->empty[st], kBoth);
      }
      umma_commit_pair(&bars->drain_pv, 1);
      drain_bar(&bars->drain_pv, 0);
    }
  } else if (warp < 8) {
    // ----------------------- softmax + epilogue + q_lat staging (warps 0-7)
    const int g = warp >> 2;                 // warpgroup: page rows [32 g, 32 g + 32)
    const int quad = warp & 3;
    const int h = threadIdx.x & 127;         // head == TMEM lane of S
    const uint32_t lane_off = static_cast<uint32_t>(quad * 32) << 16;
    float *red = reinterpret_cast<float *>(smem + kOffRed);       // [2][128]
    float *alpha_s = reinterpret_cast<float *>(smem + kOffAlpha);  // [128]
    float *lsum = alpha_s + 128;                                   // [128]
    const bool writes_p = (h >> 6) == (int)rank;   // this CTA supplies P of heads [64r, 64r+64)
    const int hl = h & 63;
    float m_run = -INFINITY;     // running max (log2 units), identical in both CTAs
    float l_part = 0.f;          // this thread's share of the row sum (its 32 rows)

    auto produce = [&](int j, const TileCursor &tc) -> bool {
      const bool first = tc.first();
      if (first) {
        // the previous segment's scores were read, so its score MMAs are complete
        stage_q(a, tc.seg.b, h, g, tmem + lane_off + kTmemQ);
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive_remote(lead(&bars->q_tmem));
      }
      const int sb = j % kSBuf;
      if (!wait_bar(ctx, &bars->s_full[sb], (j / kSBuf) & 1)) return false;
      tc_fence_after();
      float sv[32];
      tmem_ld32f(tmem + lane_off + kTmemS + 64 * sb + 32 * g, sv);
      tmem_wait_ld();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_remote(lead(&bars->s_free[sb]));
      const int mine = tc.rows_valid() - 32 * g;     // valid rows among my 32
      float mx = -INFINITY;
#pragma unroll
      for (int k = 0; k < 32; ++k) {
        sv[k] = k < mine ? sv[k] : -INFINITY;
        mx = fmaxf(mx, sv[k]);
      }
      softmax_sync();                        // previous readers of red[] are done
      red[g * 128 + h] = mx;
      softmax_sync();
      const float mx_t = fmaxf(red[h], red[128 + h]) * scale_log2;
      const float m_new = first ? mx_t : (mx_t > m_run + 8.0f ? mx_t : m_run);
      const float alpha = first ? 1.f : ex2(m_run - m_new);
      // P (bf16) for my 32 rows; the row sum is taken from the rounded values
      uint32_t w[16];
      float add = 0.f;
#pragma unroll
      for (int q = 0; q < 16; ++q) {
        const float p0 = 2 * q < mine ? ex2(fmaf(sv[2 * q], scale_log2, -m_new)) : 0.f;
        const float p1 = 2 * q + 1 < mine ? ex2(fmaf(sv[2 * q + 1], scale_log2, -m_new)) : 0.f;
        w[q] = pack_bf16(p0, p1);
        add += bf16_lo(w[q]) + bf16_hi(w[q]);
      }
      l_part = first ? add : l_part * alpha + add;
      m_run = m_new;
      const int pb = j & 1;
      if (j >= 2 && !wait_bar(ctx, &bars->pv_done[pb], ((j >> 1) - 1) & 1)) return false;
      if (writes_p) {
        // P buffer row hl: 16-byte chunk c (rows 8c..8c+7) at hl*128 + ((c ^ (hl&7)) << 4)
        uint8_t *row = smem + kOffP + pb * kPBytes + hl * 128;
#pragma unroll
        for (int c = 0; c < 4; ++c)
          *reinterpret_cast<uint4 *>(row + (((4 * g + c) ^ (hl & 7)) << 4)) =
              make_uint4(w[4 * c], w[4 * c + 1], w[4 * c + 2], w[4 * c + 3]);
      }
      // O^T holds the tiles before j: rescale its head columns when the max moved
      if (g == 0) alpha_s[h] = alpha;
      if (softmax_any(alpha != 1.f)) {
        if (!wait_bar(ctx, &bars->pv_done[(j - 1) & 1], ((j - 1) >> 1) & 1)) return false;
        tc_fence_after();
        const uint32_t ob = tmem + lane_off + kTmemO + 128 * g;   // block g, lane = column
        for (int c = 0; c < 128; c += 32) {
          uint32_t r[32];
          tmem_ld32(ob + c, r);
          tmem_wait_ld();
#pragma unroll
          for (int k = 0; k < 32; ++k)
            r[k] = __float_as_uint(__uint_as_float(r[k]) * alpha_s[c + k]);
          tmem_st32(ob + c, r);
        }
        tmem_wait_st();
      }
      fence_proxy_async_smem();              // P -> the MMA
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_remote(lead(&bars->p_ready[pb]));
      return true;
    };

    // ---- end of a segment (tile j was its last): normalise and write O^T
    auto epilogue = [&](int j, const TileCursor &tc) -> bool {
      softmax_sync();                        // previous readers of red[] / lsum[] are done
      red[g * 128 + h] = l_part;
      softmax_sync();
      if (g == 0) lsum[h] = red[h] + red[128 + h];
      if (!wait_bar(ctx, &bars->pv_done[j & 1], (j >> 1) & 1)) return false;
      softmax_sync();
      tc_fence_after();
      const int b = tc.seg.b;
      const int pbase = a.part_base[b];
      const bool whole = pbase < 0;
      const int slot_p = whole ? 0 : pbase + (part - tc.seg.s0 / hdr.quota);
      const int col = 256 * g + 128 * rank + quad * 32 + lane;   // latent column of my lane
      const uint32_t ob = tmem + lane_off + kTmemO + 128 * g;
      for (int c = 0; c < 128; c += 32) {
        float v[32];
        tmem_ld32f(ob + c, v);
        tmem_wait_ld();
        if (whole) {
          __nv_bfloat16 *z = reinterpret_cast<__nv_bfloat16 *>(a.z) + (long)b * kHeads * kDc + col;
#pragma unroll
          for (int k = 0; k < 32; ++k)
            z[(long)(c + k) * kDc] = __float2bfloat16_rn(v[k] / lsum[c + k]);
        } else {
          float *o = a.part_O + (long)slot_p * kHeads * kDc + col;
#pragma unroll
          for (int k = 0; k < 32; ++k) o[(long)(c + k) * kDc] = v[k];
        }
      }
      if (rank == 0 && g == 0) {
        const float ln2 = 0.6931471805599453f;
        const long row_idx = (long)b * kHeads + h;
        if (whole) {
          if (a.lse) a.lse[row_idx] = (m_run + __log2f(lsum[h])) * ln2;
        } else {
          a.part_m[(long)slot_p * kHeads + h] = m_run * ln2;
          a.part_l[(long)slot_p * kHeads + h] = lsum[h];
        }
      }
      tc_fence_before();
      return true;
    };

    for (int tile = 0; cur.valid; cur.advance(a), ++tile) {
      if (!produce(tile, cur)) break;
      if (cur.last() && !epilogue(tile, cur)) break;
    }
  }

  __syncthreads();
  cluster_sync();  // neither CTA touches the other's shared memory or TMEM any more
  if (warp == kWarpS) {
    tc_fence_after();
    tmem_dealloc_pair(tmem, kTmemCols);
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
  CUtensorMap tm_kv, tm_v, tm_q;
  const long pool_rows = (long)a.num_pages * kPage;
  const long q_rows = (long)a.batch * kHeads;
  if (!make_map(&tm_kv, a.pool, pool_rows, 64, kOwn, CU_TENSOR_MAP_SWIZZLE_128B) ||
      !make_map(&tm_v, a.pool, pool_rows, 64, kPage, CU_TENSOR_MAP_SWIZZLE_128B) ||
      !make_map(&tm_q, a.q_lat, q_rows, 64, kHeads, CU_TENSOR_MAP_SWIZZLE_128B))
    return cudaErrorInvalidValue;
  const float scale_log2 = a.scale * 1.4426950408889634f;
  return launch_pdl(attn_sm100_kernel, dim3(2 * parts), dim3(kThreads), kSmemBytes, s, tm_kv, tm_v,
                    tm_q, a, scale_log2);
}

}  // namespace sm100
}  // namespace mla
