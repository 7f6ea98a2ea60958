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
//  * TMEM per CTA: O half (256 columns), the CTA's 288-column slice of q_lat
//    as the A operand of the score MMA (144 columns, bf16 pairs), S (64).
//    Keeping q_lat in TMEM leaves shared memory for a 4-stage TMA ring.
//  * Each CTA computes a partial score over its 288 columns (tcgen05.mma,
//    M = 128 heads, N = 64 rows, K = 288) and writes it with asynchronous
//    remote stores (st.async) into one of two receive slots in its partner's
//    shared memory; each store completes bytes of the slot's mbarrier, so no
//    thread fences or waits for its stores.  The exchange runs one tile
//    ahead: the partial of tile j+1 is sent before tile j's softmax.  Both
//    CTAs add the halves in the same order and run the identical online
//    softmax (exp2 domain, lazy rescale when the max grows by more than 2^8).
//  * Two softmax warpgroups: TMEM lane = head, warpgroup g owns the 32 rows
//    [32 g, 32 g + 32) of each page; row maxima and sums are combined through
//    shared memory.
//  * P (bf16) goes to TMEM; O_half += P . V_half on tcgen05 with A = P read
//    from TMEM and B = the page's latent half (N = 256).
//  * Warp roles: warps 0-7 softmax + epilogue + q_lat staging, warp 8 TMA
//    producer, warp 9 TMEM allocation + score MMA issue, warp 10 P.V MMA issue
//    (two issuers, so P.V of tile j never waits for the data of tile j+1).
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
constexpr int kStages = 4;
constexpr int kSoftmaxThreads = 256;
constexpr int kThreads = kSoftmaxThreads + 96;   // + producer, score issuer, P.V issuer
constexpr int kWarpProd = 8, kWarpS = 9, kWarpPV = 10;
constexpr uint64_t kTimeoutNs = 2000000000ull;

// Shared memory (byte offsets from a 1024-byte aligned base).
constexpr int kKChunk = kPage * 128;             // 64 rows x 64 bf16, 128B swizzle
constexpr int kKRope = kPage * 64;               // 64 rows x 32 bf16, 64B swizzle
constexpr int kStageBytes = 4 * kKChunk + kKRope;  // 36 KB
constexpr int kXBytes = 128 * 64 * 4;            // one partial-score tile (fp32)
constexpr int kOffStage = 0;
constexpr int kOffX = kOffStage + kStages * kStageBytes;  // two receive slots (partner's partials)
constexpr int kOffRed = kOffX + 2 * kXBytes;     // 2 x 128 floats: per-warpgroup row max / sum
constexpr int kOffBar = kOffRed + 1024;
constexpr int kSmemBytes = kOffBar + 256 + 1024;

// TMEM columns
constexpr uint32_t kTmemO = 0;     // O_half: 256 fp32 columns
constexpr uint32_t kTmemQ = 256;   // q_lat slice: 288 bf16 = 144 columns
constexpr uint32_t kTmemP = 400;   // P: 64 bf16 = 32 columns
constexpr uint32_t kTmemS = 448;   // S: 64 fp32 columns
constexpr uint32_t kTmemCols = 512;

constexpr uint32_t kIdescS = idesc_bf16(128, 64, 0, 0);    // A = q_lat (TMEM), B = rows (K-major)
constexpr uint32_t kIdescPV = idesc_bf16(128, 256, 0, 1);  // A = P (TMEM), B = V (MN-major)

struct Bars {
  uint64_t full[kStages], empty[kStages];
  uint64_t q_full, s_full, s_free, p_full, pv_done, x_full[2], peer_free[2], drain_s, drain_pv;
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

// Named barrier over the 256 softmax threads.
__device__ __forceinline__ void softmax_sync() {
  asm volatile("bar.sync 1, %0;" ::"n"(kSoftmaxThreads) : "memory");
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
};

// Stages this warpgroup's share of the CTA's 288-column slice of q_lat[b][h]
// into TMEM (lane h): warpgroup 0 the latent columns [0, 128) of the slice,
// warpgroup 1 the latent columns [128, 256) and the 32 RoPE columns.
__device__ __forceinline__ void stage_q(const AttnArgs &a, int b, int h, int g, uint32_t rank,
                                        uint32_t taddr) {
  const uint4 *src = reinterpret_cast<const uint4 *>(
      reinterpret_cast<const __nv_bfloat16 *>(a.q_lat) + ((long)b * kHeads + h) * kRow);
  const int c0 = kHalf * rank / 8;          // 16-byte units
#pragma unroll
  for (int blk = 0; blk < 2; ++blk) {       // 2 x 32 TMEM columns (64 bf16 each)
    const int bb = 2 * g + blk;
    uint32_t v[32];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const uint4 x = src[c0 + bb * 8 + i];
      v[4 * i] = x.x; v[4 * i + 1] = x.y; v[4 * i + 2] = x.z; v[4 * i + 3] = x.w;
    }
    tmem_st32(taddr + 32 * bb, v);
  }
  if (g == 1) {                             // RoPE part: 16 TMEM columns
    const int r0 = (kDc + 32 * rank) / 8;
    uint32_t w[16];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const uint4 x = src[r0 + i];
      w[4 * i] = x.x; w[4 * i + 1] = x.y; w[4 * i + 2] = x.z; w[4 * i + 3] = x.w;
    }
    tmem_st16(taddr + 128, w);
  }
  tmem_wait_st();
}

__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kThreads, 1)
    attn_sm100_kernel(const __grid_constant__ CUtensorMap tm_kv,
                      const __grid_constant__ CUtensorMap tm_kr, const AttnArgs a,
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
    mbar_init(&bars->q_full, 8);
    mbar_init(&bars->s_full, 1);
    mbar_init(&bars->s_free, 8);
    mbar_init(&bars->p_full, 8);
    mbar_init(&bars->pv_done, 1);
    for (int i = 0; i < 2; ++i) {
      mbar_init(&bars->x_full[i], 1);
      mbar_init(&bars->peer_free[i], 1);
    }
    mbar_init(&bars->drain_s, 1);
    mbar_init(&bars->drain_pv, 1);
    bars->abort = 0;
    fence_mbar_init();
    // arm both receive slots for tiles 0 and 1 before the partner can send
    mbar_expect_tx(&bars->x_full[0], kXBytes);
    mbar_expect_tx(&bars->x_full[1], kXBytes);
  }
  if (warp == kWarpProd && lane == 0) {
    prefetch_tmap(&tm_kv);
    prefetch_tmap(&tm_kr);
  }
  if (warp == kWarpS) {
    tmem_alloc(&bars->tmem_base, kTmemCols);
    tc_fence_before();
  }
  __syncthreads();
  tc_fence_after();
  cluster_sync();  // the partner's barriers exist before any remote arrive or copy
  const uint32_t tmem = bars->tmem_base;

  TileCursor cur;
  cur.init(a, hdr, part);

  if (warp == kWarpProd) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      int tile = 0;
      for (; cur.valid; cur.advance(a), ++tile) {
        const int st = tile % kStages;
        if (tile >= kStages &&
            !wait_bar<false>(ctx, &bars->empty[st], ((tile / kStages) - 1) & 1))
          break;
        int page = a.block_table[(long)cur.seg.b * a.max_pages + cur.lp];
        if (page < 0 || page >= a.num_pages) {
          set_error(a.err, kErrRange);
          a.bad[cur.seg.b] = 1;
          page = 0;
        }
        uint8_t *dst = smem + kOffStage + st * kStageBytes;
        mbar_expect_tx(&bars->full[st], kStageBytes);
        const int y = page * kPage;
        for (int i = 0; i < 4; ++i)
          tma_load_2d(dst + i * kKChunk, &tm_kv, kHalf * rank + 64 * i, y, &bars->full[st]);
        tma_load_2d(dst + 4 * kKChunk, &tm_kr, kDc + 32 * rank, y, &bars->full[st]);
      }
      // drain: every issued load lands before the CTA may exit
      for (int t = tile - kStages; t < tile; ++t)
        if (t >= 0) wait_bar<false>(ctx, &bars->full[t % kStages], (t / kStages) & 1);
    }
  } else if (warp == kWarpS) {
    // ------------------------------------------------------------ score MMA issuer
    if (lane == 0) {
      int tile = 0;
      for (; cur.valid; cur.advance(a), ++tile) {
        const int st = tile % kStages;
        if (!wait_bar<false>(ctx, &bars->full[st], (tile / kStages) & 1)) break;
        if (cur.first() && !wait_bar<false>(ctx, &bars->q_full, cur.nseg & 1)) break;
        if (tile > 0 && !wait_bar<false>(ctx, &bars->s_free, (tile - 1) & 1)) break;
        tc_fence_after();
        const uint32_t k_base = smem_u32(smem + kOffStage + st * kStageBytes);
        int kk = 0;
        for (int i = 0; i < 4; ++i)         // latent columns: 4 chunks of 64, 128B swizzle
          for (int k = 0; k < 4; ++k, ++kk)
            umma_bf16_ts(tmem + kTmemS, tmem + kTmemQ + 32 * i + 8 * k,
                         sdesc(k_base + i * kKChunk + 32 * k, 16, 1024, 2), kIdescS,
                         kk ? 1u : 0u);
        for (int k = 0; k < 2; ++k)         // RoPE columns: 32 wide, 64B swizzle
          umma_bf16_ts(tmem + kTmemS, tmem + kTmemQ + 128 + 8 * k,
                       sdesc(k_base + 4 * kKChunk + 32 * k, 16, 512, 4), kIdescS, 1u);
        umma_commit(&bars->s_full);
      }
      umma_commit(&bars->drain_s);
      wait_bar<false>(ctx, &bars->drain_s, 0);
    }
  } else if (warp == kWarpPV) {
    // ------------------------------------------------------------ P.V MMA issuer
    if (lane == 0) {
      int tile = 0;
      for (; cur.valid; cur.advance(a), ++tile) {
        const int st = tile % kStages;
        if (!wait_bar<false>(ctx, &bars->p_full, tile & 1)) break;
        tc_fence_after();
        const uint32_t v_base = smem_u32(smem + kOffStage + st * kStageBytes);
        const bool first = cur.first();
        for (int k = 0; k < kPage / 16; ++k)
          // A: P rows (heads) x 16 tokens (TMEM, 8 columns per step); B: 16 tokens
          // x 256 latent (MN-major, 64-column chunks 8 KB apart, 8-token groups 1 KB apart)
          umma_bf16_ts(tmem + kTmemO, tmem + kTmemP + 8 * k,
                       sdesc(v_base + 2048 * k, kKChunk, 1024, 2), kIdescPV,
                       (first && k == 0) ? 0u : 1u);
        umma_commit(&bars->pv_done);
        umma_commit(&bars->empty[st]);
      }
      umma_commit(&bars->drain_pv);
      wait_bar<false>(ctx, &bars->drain_pv, 0);
    }
  } else {
    // ----------------------- softmax + epilogue + q_lat staging (warps 0-7)
    const int g = warp >> 2;                 // warpgroup: rows [32 g, 32 g + 32) of a page
    const int h = threadIdx.x & 127;         // head index == TMEM lane
    const uint32_t lane_off = static_cast<uint32_t>((warp & 3) * 32) << 16;
    float *red = reinterpret_cast<float *>(smem + kOffRed);   // [2][128]
    // partial-score tile layout (per receive slot): 16-byte chunk i (4 rows of a
    // page) of head h at (i * 128 + h) * 16; warpgroup g owns chunks [8 g, 8 g + 8)
    const uint32_t x_local = smem_u32(smem + kOffX) + h * 16;
    const uint32_t x_remote = mapa(x_local, peer);
    const uint32_t peer_x_full = mapa(smem_u32(&bars->x_full[0]), peer);
    const uint32_t peer_free = mapa(smem_u32(&bars->peer_free[0]), peer);
    TileCursor nxt = cur;
    float m_run = -INFINITY, l_part = 0.f;
    int tile = 0;
    float sa[32], sb[32];

    // S_j: this warpgroup's 32 score columns from TMEM into s, then sent to
    // the partner's receive slot j % 2 (its mbarrier counts the bytes)
    auto fetch_and_store = [&](int j, float (&s)[32]) -> bool {
      if (!wait_bar<false>(ctx, &bars->s_full, j & 1)) return false;
      tc_fence_after();
      tmem_ld32f(tmem + lane_off + kTmemS + 32 * g, s);
      tmem_wait_ld();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars->s_free);
      const int slot = j & 1;
      if (j >= 2 && !wait_bar<true>(ctx, &bars->peer_free[slot], ((j >> 1) - 1) & 1)) return false;
      const uint32_t dst = x_remote + slot * kXBytes;
      const uint32_t mb = peer_x_full + slot * 8;
#pragma unroll
      for (int i = 0; i < 8; ++i)
        st_async_v4(dst + (8 * g + i) * 2048, s[4 * i], s[4 * i + 1], s[4 * i + 2], s[4 * i + 3],
                    mb);
      return true;
    };
    auto stage_segment_q = [&](int b) {
      stage_q(a, b, h, g, rank, tmem + lane_off + kTmemQ);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars->q_full);
    };

    bool ok = cur.valid;
    if (ok) {
      stage_segment_q(cur.seg.b);
      ok = fetch_and_store(0, sa);
      nxt.advance(a);
    }
    // One tile: look ahead (stage q_lat of the next segment, fetch and store
    // S_{j+1} from `sn`), combine S_j (in `sc`) with the partner's partial,
    // softmax, P, release S_{j+1}, and the epilogue at the end of a segment.
    auto step = [&](float (&sc)[32], float (&sn)[32]) -> bool {
      const bool ahead = nxt.valid;
      if (ahead) {
        // S_j, the last score MMA that read the old q_lat, is complete
        if (nxt.first()) stage_segment_q(nxt.seg.b);
        if (!fetch_and_store(tile + 1, sn)) return false;
      }
      // ---- combine tile j with the partner's partial
      const int slot = tile & 1;
      if (!wait_bar<true>(ctx, &bars->x_full[slot], (tile >> 1) & 1)) return false;
      const bool first = cur.first();
      if (first) {
        m_run = -INFINITY;
        l_part = 0.f;
      }
      const uint8_t *xr = smem + kOffX + slot * kXBytes + h * 16;
      float mx = -INFINITY;
      const int n_valid = min(kPage, cur.seg.len - cur.lp * kPage);
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const float4 v = *reinterpret_cast<const float4 *>(xr + (8 * g + i) * 2048);
        // rank 0 adds (own + partner), rank 1 (partner + own): the same sum
        if (rank == 0) {
          sc[4 * i] += v.x; sc[4 * i + 1] += v.y; sc[4 * i + 2] += v.z; sc[4 * i + 3] += v.w;
        } else {
          sc[4 * i] = v.x + sc[4 * i]; sc[4 * i + 1] = v.y + sc[4 * i + 1];
          sc[4 * i + 2] = v.z + sc[4 * i + 2]; sc[4 * i + 3] = v.w + sc[4 * i + 3];
        }
      }
#pragma unroll
      for (int k = 0; k < 32; ++k) {
        sc[k] = 32 * g + k < n_valid ? sc[k] : -INFINITY;
        mx = fmaxf(mx, sc[k]);
      }
      red[g * 128 + h] = mx;
      softmax_sync();                        // slot read by all: the partner may refill it
      if (threadIdx.x == 0) {
        mbar_expect_tx(&bars->x_full[slot], kXBytes);   // armed for tile j + 2
        mbar_arrive_cluster_relaxed(peer_free + slot * 8);
      }
      mx = fmaxf(mx, red[(g ^ 1) * 128 + h]) * scale_log2;
      // ---- online softmax in the exp2 domain (identical in both warpgroups)
      const bool grow = mx > m_run + 8.0f;
      float alpha = 1.f;
      if (grow) {
        alpha = ex2(m_run - mx);
        m_run = mx;
      }
      // P buffer and O are free once the previous tile's P.V has completed
      if (tile > 0 && !wait_bar<false>(ctx, &bars->pv_done, (tile - 1) & 1)) return false;
      tc_fence_after();
      if (!first && __any_sync(0xffffffffu, grow)) {
        for (int c = 128 * g; c < 128 * g + 128; c += 32) {
          uint32_t r[32];
          tmem_ld32(tmem + lane_off + kTmemO + c, r);
          tmem_wait_ld();
#pragma unroll
          for (int k = 0; k < 32; ++k) r[k] = __float_as_uint(__uint_as_float(r[k]) * alpha);
          tmem_st32(tmem + lane_off + kTmemO + c, r);
        }
        tmem_wait_st();
      }
      // P row h, rows [32 g, 32 g + 32) of the page: TMEM columns
      // [16 g, 16 g + 16) of P, two bf16 per column (lower row in the low half)
      float sum = 0.f;
      {
        uint32_t w[16];
#pragma unroll
        for (int q = 0; q < 16; ++q) {
          const float p0 = ex2(fmaf(sc[2 * q], scale_log2, -m_run));
          const float p1 = ex2(fmaf(sc[2 * q + 1], scale_log2, -m_run));
          sum += p0 + p1;
          w[q] = pack_bf16(p0, p1);
        }
        tmem_st16(tmem + lane_off + kTmemP + 16 * g, w);
        tmem_wait_st();
      }
      l_part = l_part * alpha + sum;
      if (n_valid < kPage) {
        // rows past the sequence end hold arbitrary bytes: zero their latent
        // part so that 0 * garbage cannot reach O
        uint8_t *stg = smem + kOffStage + (tile % kStages) * kStageBytes;
        const int nz = (kPage - n_valid) * 32;   // 16-byte pieces over 4 chunks
        for (int i = threadIdx.x; i < nz; i += kSoftmaxThreads) {
          const int row = n_valid + (i >> 5), piece = i & 31;
          *reinterpret_cast<uint4 *>(stg + (piece >> 3) * kKChunk + row * 128 +
                                     (piece & 7) * 16) = make_uint4(0, 0, 0, 0);
        }
        fence_proxy_async_smem();
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars->p_full);
      if (cur.last()) {
        // ---------------------------------------------------- epilogue
        softmax_sync();                      // red[] reads of this tile are done
        red[g * 128 + h] = l_part;
        if (!wait_bar<false>(ctx, &bars->pv_done, tile & 1)) return false;
        softmax_sync();
        const float l_run = red[h] + red[128 + h];
        softmax_sync();                      // red[] is free for the next tile's maxima
        tc_fence_after();
        const int pb = a.part_base[cur.seg.b];
        const bool whole = pb < 0;
        const long row_idx = (long)cur.seg.b * kHeads + h;
        const int slot_p = whole ? 0 : pb + (part - cur.seg.s0 / hdr.quota);
        const float inv_l = 1.f / l_run;
        for (int c = 128 * g; c < 128 * g + 128; c += 32) {
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
            float *o = a.part_O + ((long)slot_p * kHeads + h) * kDc + kHalf * rank + c;
#pragma unroll
            for (int j = 0; j < 8; ++j)
              *reinterpret_cast<uint4 *>(o + 4 * j) =
                  make_uint4(r[4 * j], r[4 * j + 1], r[4 * j + 2], r[4 * j + 3]);
          }
        }
        if (rank == 0 && g == 0) {
          const float ln2 = 0.6931471805599453f;
          if (whole) {
            if (a.lse) a.lse[row_idx] = (m_run + __log2f(l_run)) * ln2;
          } else {
            a.part_m[(long)slot_p * kHeads + h] = m_run * ln2;
            a.part_l[(long)slot_p * kHeads + h] = l_run;
          }
        }
        tc_fence_before();
      }
      cur.advance(a);
      nxt.advance(a);
      ++tile;
      return true;
    };
    while (ok && cur.valid) {
      if (!step(sa, sb)) break;
      if (!cur.valid || !step(sb, sa)) break;
    }
  }

  __syncthreads();
  cluster_sync();  // the partner no longer touches this CTA's shared memory
  if (warp == kWarpS) {
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
  CUtensorMap tm_kv, tm_kr;
  const long pool_rows = (long)a.num_pages * kPage;
  if (!make_map(&tm_kv, a.pool, pool_rows, 64, kPage, CU_TENSOR_MAP_SWIZZLE_128B) ||
      !make_map(&tm_kr, a.pool, pool_rows, 32, kPage, CU_TENSOR_MAP_SWIZZLE_64B))
    return cudaErrorInvalidValue;
  const float scale_log2 = a.scale * 1.4426950408889634f;
  attn_sm100_kernel<<<2 * parts, kThreads, kSmemBytes, s>>>(tm_kv, tm_kr, a, scale_log2);
  return cudaGetLastError();
}

}  // namespace sm100
}  // namespace mla
