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
//    CTA r owns latent columns [256 r, 256 r + 256) of O.
//  * Rows of each 64-row page are split between the pair: CTA r scores its
//    own 32 rows [32 r, 32 r + 32) over all 576 columns (tcgen05.mma,
//    M = 128 heads, N = 32 rows, K = 576), so no partial score is exchanged.
//    q_lat is the A operand: 384 of its columns sit in TMEM, the last 192
//    (latent 384..511 and k_R) in shared memory.  S has two TMEM buffers, so
//    the scores of the next tile are computed while this tile's are read.
//  * Each CTA turns its own rows into P (bf16, exp2 domain) relative to a
//    reference max that both CTAs share, and sends its P half plus the
//    reference it used to the partner with st.async stores (8.5 KB per tile,
//    counted by the receiving mbarrier).  When a CTA's own max grew past the
//    shared reference by more than 2^8 it uses its own max instead; both CTAs
//    then see the same pair of references, take the same new shared max,
//    rescale O (TMEM) and the lagging P half (shared memory) identically.
//  * O_half += P . V_half on tcgen05 (A = the 64-row P tile in shared
//    memory, B = the page's latent half: the CTA's own rows come with its
//    full-width tile, the partner's 32 rows are loaded separately and are
//    normally L2 hits because the partner streams the same page).  The P tile
//    is written over the stage's own rows' other latent half, which only S
//    reads: once both CTAs' S of the tile is complete they say so to each
//    other and write their P halves there.
//  * Row sums are taken from the bf16 P both CTAs feed the MMA (own and
//    received halves), so no sum is exchanged; the epilogue divides O_half.
//  * Two softmax warpgroups (TMEM lane = head): warpgroup g owns 16 of the
//    CTA's 32 rows.  Warp 8: TMA producer; warp 9: TMEM allocation + score
//    MMAs + q_lat shared-memory part; warp 10: P.V MMAs.
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
constexpr int kOwn = 32;         // rows of a page scored by each CTA
constexpr int kHalf = 256;       // latent columns of O per CTA
constexpr int kStages = 3;
constexpr int kSoftmaxThreads = 256;
constexpr int kThreads = kSoftmaxThreads + 96;   // + producer, score issuer, P.V issuer
constexpr int kWarpProd = 8, kWarpS = 9, kWarpPV = 10;
constexpr uint64_t kTimeoutNs = 2000000000ull;
constexpr uint32_t kSleepNs = 20000;   // suspend hint of a waiting thread (woken at completion)

// Shared memory (byte offsets from a 1024-byte aligned base).
constexpr int kChunk = kOwn * 128;               // 32 rows x 64 bf16, 128-byte swizzle
constexpr int kQChunk = kHeads * 128;            // 128 heads x 64 bf16
constexpr int kQSmem = 3;                        // q_lat columns 384..575 in shared memory
constexpr int kOffQ = 0;
constexpr int kOffStage = kOffQ + kQSmem * kQChunk;
constexpr int kRegionB = 9 * kChunk;             // own rows: 9 chunks x 64 columns
constexpr int kStageBytes = kRegionB + 4 * kChunk;  // + partner rows, own latent half
// The P tile of a tile (128 heads x 64 rows bf16, 16 KB) is written into its
// stage's own rows' other latent half (chunks 4(1-r)..4(1-r)+3): S is the only
// reader of those chunks, so they are dead once S of the tile is complete.
constexpr int kOffRef = kOffStage + kStages * kStageBytes;  // two x 128 received reference maxima
constexpr int kOffRed = kOffRef + 1024;          // 2 x 128 floats: per-warpgroup scratch
constexpr int kOffBar = kOffRed + 1024;
constexpr int kSmemBytes = kOffBar + 512 + 1024;
constexpr uint32_t kMsgBytes = kHeads * kOwn * 2 + kHeads * 4;   // P half + references

// TMEM columns
constexpr uint32_t kTmemO = 0;     // O_half: 256 fp32 columns
constexpr uint32_t kTmemQ = 256;   // q_lat columns 0..383: 192 columns of bf16 pairs
constexpr uint32_t kTmemS = 448;   // S: two buffers of 32 fp32 columns
constexpr int kQTmemDims = 384;
constexpr uint32_t kTmemCols = 512;

constexpr uint32_t kIdescS = idesc_bf16(128, kOwn, 0, 0);  // A = q_lat, B = own rows (K-major)
constexpr uint32_t kIdescPV = idesc_bf16(128, 256, 0, 1);  // A = P (K-major), B = V (MN-major)

struct Bars {
  uint64_t full[kStages], empty[kStages];
  uint64_t q_tmem, q_smem, q_free, drain_s, drain_pv;
  uint64_t s_full[2], s_free[2];  // score buffer i written / read
  uint64_t pv_done[2];     // P.V of the tile using P tile slot i completed
  uint64_t p_ready[2];     // own P half written and partner half final (8 softmax warps)
  uint64_t p_rx[2];        // partner's P half + references landed (tx count)
  uint64_t p_slot_free[2]; // partner's S of the tile done: its P tile may be written (remote arrive)
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
    if (kCluster ? mbar_try_wait_cluster_sleep(a, parity, kSleepNs)
                 : mbar_try_wait_sleep(a, parity, kSleepNs))
      return true;
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

// Sum of the 8 bf16 values in a 16-byte chunk, each scaled by f.
__device__ __forceinline__ float sum8_bf16(uint4 v) {
  const __nv_bfloat162 *p = reinterpret_cast<const __nv_bfloat162 *>(&v);
  float s = 0.f;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float2 f = __bfloat1622float2(p[i]);
    s += f.x + f.y;
  }
  return s;
}

__device__ __forceinline__ uint4 scale8_bf16(uint4 v, float f) {
  __nv_bfloat162 *p = reinterpret_cast<__nv_bfloat162 *>(&v);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float2 x = __bfloat1622float2(p[i]);
    p[i] = __floats2bfloat162_rn(x.x * f, x.y * f);
  }
  return v;
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

// Stages q_lat[b][h][0:384] into TMEM lane h (192 columns of bf16 pairs);
// warpgroup 0 writes columns [0, 96), warpgroup 1 columns [96, 192).
__device__ __forceinline__ void stage_q(const AttnArgs &a, int b, int h, int g, uint32_t taddr) {
  const uint4 *src = reinterpret_cast<const uint4 *>(
      reinterpret_cast<const __nv_bfloat16 *>(a.q_lat) + ((long)b * kHeads + h) * kRow);
  const int b0 = g ? 3 : 0, b1 = g ? 6 : 3;       // blocks of 32 TMEM columns
  for (int bb = b0; bb < b1; ++bb) {
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
                      const __grid_constant__ CUtensorMap tm_q, const AttnArgs a,
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
    mbar_init(&bars->q_tmem, 8);
    mbar_init(&bars->q_smem, 1);
    mbar_init(&bars->q_free, 1);
    for (int i = 0; i < 2; ++i) {
      mbar_init(&bars->s_full[i], 1);
      mbar_init(&bars->s_free[i], 8);
    }
    mbar_init(&bars->drain_s, 1);
    mbar_init(&bars->drain_pv, 1);
    for (int i = 0; i < 2; ++i) {
      mbar_init(&bars->pv_done[i], 1);
      mbar_init(&bars->p_ready[i], 8);
      mbar_init(&bars->p_rx[i], 1);
      mbar_init(&bars->p_slot_free[i], 1);
    }
    bars->abort = 0;
    fence_mbar_init();
    // arm both receive slots for tiles 0 and 1 before the partner can send
    mbar_expect_tx(&bars->p_rx[0], kMsgBytes);
    mbar_expect_tx(&bars->p_rx[1], kMsgBytes);
  }
  if (warp == kWarpProd && lane == 0) {
    prefetch_tmap(&tm_kv);
    prefetch_tmap(&tm_q);
  }
  if (warp == kWarpS) {
    tmem_alloc(&bars->tmem_base, kTmemCols);
    tc_fence_before();
  }
  __syncthreads();
  tc_fence_after();
  cluster_sync();  // the partner's barriers exist (and are armed) before any remote access
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
        const int y_own = page * kPage + kOwn * rank;
        const int y_peer = page * kPage + kOwn * (1 - rank);
        for (int c = 0; c < 9; ++c)        // own rows, all 576 columns
          tma_load_2d(dst + c * kChunk, &tm_kv, 64 * c, y_own, &bars->full[st]);
        for (int c = 0; c < 4; ++c)        // partner rows, this CTA's latent half
          tma_load_2d(dst + kRegionB + c * kChunk, &tm_kv, kHalf * rank + 64 * c, y_peer,
                      &bars->full[st]);
      }
      for (int t = tile - kStages; t < tile; ++t)
        if (t >= 0) wait_bar<false>(ctx, &bars->full[t % kStages], (t / kStages) & 1);
    }
  } else if (warp == kWarpS) {
    // ---------------------------------------- score MMA issuer (+ q_lat smem part)
    if (lane == 0) {
      const uint32_t q_base = smem_u32(smem + kOffQ);
      const uint64_t qd = sdesc(q_base, 16, 1024, 2);
      int tile = 0;
      bool ok = true;
      for (; cur.valid; cur.advance(a), ++tile) {
        const int st = tile % kStages;
        if (cur.first()) {
          // the previous segment's score MMAs must finish before q_lat is replaced
          if (cur.nseg > 0 && !wait_bar<false>(ctx, &bars->q_free, (cur.nseg - 1) & 1)) { ok = false; break; }
          mbar_expect_tx(&bars->q_smem, kQSmem * kQChunk);
          for (int c = 0; c < kQSmem; ++c)
            tma_load_2d(smem + kOffQ + c * kQChunk, &tm_q, kQTmemDims + 64 * c, cur.seg.b * kHeads,
                        &bars->q_smem);
          if (!wait_bar<false>(ctx, &bars->q_smem, cur.nseg & 1)) { ok = false; break; }
          if (!wait_bar<false>(ctx, &bars->q_tmem, cur.nseg & 1)) { ok = false; break; }
        }
        if (!wait_bar<false>(ctx, &bars->full[st], (tile / kStages) & 1)) { ok = false; break; }
        // score buffer tile&1 was last used by tile-2
        const int sb = tile & 1;
        if (tile >= 2 && !wait_bar<false>(ctx, &bars->s_free[sb], ((tile >> 1) - 1) & 1)) { ok = false; break; }
        tc_fence_after();
        // descriptors advance by address >> 4 in their low field (no carry: < 256 KB)
        const uint64_t kd = sdesc(smem_u32(smem + kOffStage + st * kStageBytes), 16, 1024, 2);
        const uint32_t sd = tmem + kTmemS + 32 * sb;
#pragma unroll
        for (int s = 0; s < kQTmemDims / 16; ++s)   // q_lat columns 0..383 from TMEM
          umma_bf16_ts(sd, tmem + kTmemQ + 8 * s,
                       kd + (uint64_t)(((s >> 2) * kChunk + 32 * (s & 3)) >> 4), kIdescS,
                       s ? 1u : 0u);
#pragma unroll
        for (int s = 0; s < 4 * kQSmem; ++s)         // columns 384..575 from shared memory
          umma_bf16(sd, qd + (uint64_t)(((s >> 2) * kQChunk + 32 * (s & 3)) >> 4),
                    kd + (uint64_t)(((kQTmemDims / 64 + (s >> 2)) * kChunk + 32 * (s & 3)) >> 4),
                    kIdescS, 1u);
        if (cur.last()) umma_commit(&bars->q_free);
        umma_commit(&bars->s_full[sb]);
      }
      (void)ok;
      umma_commit(&bars->drain_s);
      wait_bar<false>(ctx, &bars->drain_s, 0);
    }
  } else if (warp == kWarpPV) {
    // ------------------------------------------------------------ P.V MMA issuer
    if (lane == 0) {
      int tile = 0;
      for (; cur.valid; cur.advance(a), ++tile) {
        const int st = tile % kStages;
        const int pb = tile & 1;
        if (!wait_bar<false>(ctx, &bars->p_ready[pb], (tile >> 1) & 1)) break;
        tc_fence_after();
        const uint32_t v_base = smem_u32(smem + kOffStage + st * kStageBytes);
        const uint32_t p_base = v_base + 4 * (1 - rank) * kChunk;
        const bool first = cur.first();
        for (int k = 0; k < kPage / 16; ++k) {
          // rows [16 k, 16 k + 16) of the page: own rows (full-width tile, latent
          // half = chunks 4r..4r+3) or partner rows (region B); chunks 4 KB apart
          const bool own = (k >> 1) == (int)rank;
          const uint32_t vb = v_base + (own ? 4 * rank * kChunk : kRegionB) + (k & 1) * 2048;
          umma_bf16(tmem + kTmemO, sdesc(p_base + 32 * k, 16, 1024, 2),
                    sdesc(vb, kChunk, 1024, 2), kIdescPV, (first && k == 0) ? 0u : 1u);
        }
        umma_commit(&bars->pv_done[pb]);
        umma_commit(&bars->empty[st]);
      }
      umma_commit(&bars->drain_pv);
      wait_bar<false>(ctx, &bars->drain_pv, 0);
    }
  } else {
    // ----------------------- softmax + epilogue + q_lat staging (warps 0-7)
    const int g = warp >> 2;                 // warpgroup: own rows [16 g, 16 g + 16)
    const int h = threadIdx.x & 127;         // head index == TMEM lane
    const uint32_t lane_off = static_cast<uint32_t>((warp & 3) * 32) << 16;
    float *red = reinterpret_cast<float *>(smem + kOffRed);   // [2][128]
    const float *refs = reinterpret_cast<const float *>(smem + kOffRef);  // [2][128]
    // P tile row h: 16-byte chunk c (rows 8c..8c+7 of the page) at h*128 + ((c ^ (h&7)) << 4);
    // the tile sits in chunks 4(1-r).. of the stage here and in chunks 4r.. at the partner
    const int c_own = 4 * rank + 2 * g;      // this thread's two own chunks: c_own, c_own + 1
    const int c_peer = 4 * (1 - rank) + 2 * g;  // and the matching partner chunks
    auto p_row = [&](int j) {
      return smem + kOffStage + (j % kStages) * kStageBytes + 4 * (1 - rank) * kChunk + h * 128;
    };
    const uint32_t p_remote0 = mapa(smem_u32(smem + kOffStage + 4 * rank * kChunk) + h * 128, peer);
    const uint32_t ref_remote = mapa(smem_u32(smem + kOffRef) + h * 4, peer);
    const uint32_t rx_remote = mapa(smem_u32(&bars->p_rx[0]), peer);
    const uint32_t slot_free_remote = mapa(smem_u32(&bars->p_slot_free[0]), peer);

    float m_run = -INFINITY;     // shared reference max (log2 units), same in both CTAs
    float l_part = 0.f;          // this thread's share of the row sum (own + partner chunks)
    float ref_own = -INFINITY;   // reference used for the latest own P half

    // ---- tile j: own rows -> P half (local + partner), reference sent along
    auto produce = [&](int j, const TileCursor &tc) -> bool {
      if (tc.first()) {
        // the previous segment's score MMAs have completed (their S was read)
        stage_q(a, tc.seg.b, h, g, tmem + lane_off + kTmemQ);
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&bars->q_tmem);
        m_run = -INFINITY;
      }
      const int sb = j & 1;
      if (!wait_bar<false>(ctx, &bars->s_full[sb], (j >> 1) & 1)) return false;
      tc_fence_after();
      float sv[16];
      tmem_ld16f(tmem + lane_off + kTmemS + 32 * sb + 16 * g, sv);
      tmem_wait_ld();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars->s_free[sb]);
      const int rows_valid = tc.seg.len - tc.lp * kPage;          // >= 1
      const int own_valid = min(max(rows_valid - kOwn * (int)rank, 0), kOwn);
      const int mine = own_valid - 16 * g;                          // valid among my 16
      float mx = -INFINITY;
#pragma unroll
      for (int k = 0; k < 16; ++k) {
        sv[k] = k < mine ? sv[k] : -INFINITY;
        mx = fmaxf(mx, sv[k]);
      }
      softmax_sync();                        // previous readers of red[] are done
      red[g * 128 + h] = mx;
      softmax_sync();
      const float mx_own = fmaxf(red[h], red[128 + h]) * scale_log2;
      ref_own = (mx_own > m_run + 8.0f) ? mx_own : m_run;
      uint32_t w[8];
#pragma unroll
      for (int q = 0; q < 8; ++q) {
        const float p0 = 2 * q < mine ? ex2(fmaf(sv[2 * q], scale_log2, -ref_own)) : 0.f;
        const float p1 = 2 * q + 1 < mine ? ex2(fmaf(sv[2 * q + 1], scale_log2, -ref_own)) : 0.f;
        w[q] = pack_bf16(p0, p1);
      }
      // rows past the sequence end hold arbitrary bytes: zero their latent
      // half in the stage so that 0 * garbage cannot reach O
      if (rows_valid < kPage) {
        uint8_t *stg = smem + kOffStage + (j % kStages) * kStageBytes;
        const int peer_valid = min(max(rows_valid - kOwn * (1 - (int)rank), 0), kOwn);
        for (int i = threadIdx.x; i < 2 * kOwn * 32; i += kSoftmaxThreads) {
          const int piece = i & 31, row = (i >> 5) % kOwn, which = i >> 10;
          const int valid = which ? peer_valid : own_valid;
          if (row >= valid) {
            uint8_t *base = which ? stg + kRegionB : stg + 4 * rank * kChunk;
            *reinterpret_cast<uint4 *>(base + (piece >> 3) * kChunk + row * 128 +
                                       (piece & 7) * 16) = make_uint4(0, 0, 0, 0);
          }
        }
      }
      const int pb = j & 1;
      // S of tile j is complete here, so the dead chunks holding this CTA's P
      // tile of tile j may be written; tell the partner, and wait for its word
      if (threadIdx.x == 0) mbar_arrive_cluster_relaxed(slot_free_remote + pb * 8);
      if (!wait_bar<true>(ctx, &bars->p_slot_free[pb], (j >> 1) & 1)) return false;
      const uint4 v0 = make_uint4(w[0], w[1], w[2], w[3]);
      const uint4 v1 = make_uint4(w[4], w[5], w[6], w[7]);
      const uint32_t o0 = (c_own ^ (h & 7)) << 4;
      const uint32_t o1 = ((c_own + 1) ^ (h & 7)) << 4;
      uint8_t *prow = p_row(j);
      *reinterpret_cast<uint4 *>(prow + o0) = v0;
      *reinterpret_cast<uint4 *>(prow + o1) = v1;
      const uint32_t mb = rx_remote + pb * 8;
      const uint32_t rrow = p_remote0 + (j % kStages) * kStageBytes;
      st_async_v4u(rrow + o0, v0, mb);
      st_async_v4u(rrow + o1, v1, mb);
      if (g == 0) st_async_f32(ref_remote + pb * 512, ref_own, mb);
      return true;
    };

    // ---- tile j: the partner's half and reference have landed: shared max,
    // rescales, row sums; hand the P tile to the P.V issuer
    auto finalize = [&](int j, const TileCursor &tc) -> bool {
      const int pb = j & 1;
      if (!wait_bar<true>(ctx, &bars->p_rx[pb], (j >> 1) & 1)) return false;
      if (threadIdx.x == 0) mbar_expect_tx(&bars->p_rx[pb], kMsgBytes);   // armed for tile j + 2
      const float ref_p = refs[pb * 128 + h];
      const float m_new = fmaxf(ref_own, ref_p);
      const bool first = tc.first();
      const float f_own = ref_own < m_new ? ex2(ref_own - m_new) : 1.f;
      const float f_peer = ref_p < m_new ? ex2(ref_p - m_new) : 1.f;
      const float alpha = (first || !(m_new > m_run)) ? 1.f : ex2(m_run - m_new);
      uint8_t *row = p_row(j);
      uint4 *q0 = reinterpret_cast<uint4 *>(row + ((c_own ^ (h & 7)) << 4));
      uint4 *q1 = reinterpret_cast<uint4 *>(row + (((c_own + 1) ^ (h & 7)) << 4));
      uint4 *q2 = reinterpret_cast<uint4 *>(row + ((c_peer ^ (h & 7)) << 4));
      uint4 *q3 = reinterpret_cast<uint4 *>(row + (((c_peer + 1) ^ (h & 7)) << 4));
      uint4 own0 = *q0, own1 = *q1, pe0 = *q2, pe1 = *q3;
      if (f_own != 1.f) {                    // rare: this CTA's reference was the lower one
        own0 = scale8_bf16(own0, f_own);
        own1 = scale8_bf16(own1, f_own);
        *q0 = own0;
        *q1 = own1;
      }
      if (f_peer != 1.f) {                   // rare: the partner's reference was the lower one
        pe0 = scale8_bf16(pe0, f_peer);
        pe1 = scale8_bf16(pe1, f_peer);
        *q2 = pe0;
        *q3 = pe1;
      }
      const float add = (sum8_bf16(own0) + sum8_bf16(own1)) + (sum8_bf16(pe0) + sum8_bf16(pe1));
      l_part = first ? add : l_part * alpha + add;
      // O holds tiles < j of this segment; rescale it when the shared max moved
      if (__any_sync(0xffffffffu, alpha != 1.f)) {
        if (!wait_bar<false>(ctx, &bars->pv_done[(j - 1) & 1], ((j - 1) >> 1) & 1)) return false;
        tc_fence_after();
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
      m_run = m_new;
      fence_proxy_async_smem();              // own P, rescaled halves, zeroed rows -> MMA
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars->p_ready[pb]);
      return true;
    };

    // ---- end of a segment (tile j was its last): normalise and write O_half
    auto epilogue = [&](int j, const TileCursor &tc) -> bool {
      softmax_sync();                        // previous readers of red[] are done
      red[g * 128 + h] = l_part;
      if (!wait_bar<false>(ctx, &bars->pv_done[j & 1], (j >> 1) & 1)) return false;
      softmax_sync();
      const float l_run = red[h] + red[128 + h];
      tc_fence_after();
      const int pbase = a.part_base[tc.seg.b];
      const bool whole = pbase < 0;
      const long row_idx = (long)tc.seg.b * kHeads + h;
      const int slot_p = whole ? 0 : pbase + (part - tc.seg.s0 / hdr.quota);
      const float inv_l = 1.f / l_run;
      for (int c = 128 * g; c < 128 * g + 128; c += 32) {
        uint32_t r[32];
        tmem_ld32(tmem + lane_off + kTmemO + c, r);
        tmem_wait_ld();
        if (whole) {
          __nv_bfloat16 *z = reinterpret_cast<__nv_bfloat16 *>(a.z) + row_idx * kDc +
                             kHalf * rank + c;
#pragma unroll
          for (int jj = 0; jj < 4; ++jj) {
            uint4 v;
            v.x = pack_bf16(__uint_as_float(r[8 * jj + 0]) * inv_l, __uint_as_float(r[8 * jj + 1]) * inv_l);
            v.y = pack_bf16(__uint_as_float(r[8 * jj + 2]) * inv_l, __uint_as_float(r[8 * jj + 3]) * inv_l);
            v.z = pack_bf16(__uint_as_float(r[8 * jj + 4]) * inv_l, __uint_as_float(r[8 * jj + 5]) * inv_l);
            v.w = pack_bf16(__uint_as_float(r[8 * jj + 6]) * inv_l, __uint_as_float(r[8 * jj + 7]) * inv_l);
            *reinterpret_cast<uint4 *>(z + 8 * jj) = v;
          }
        } else {
          float *o = a.part_O + ((long)slot_p * kHeads + h) * kDc + kHalf * rank + c;
#pragma unroll
          for (int jj = 0; jj < 8; ++jj)
            *reinterpret_cast<uint4 *>(o + 4 * jj) =
                make_uint4(r[4 * jj], r[4 * jj + 1], r[4 * jj + 2], r[4 * jj + 3]);
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
      return true;
    };

    TileCursor prev = cur;
    bool ok = true;
    for (int tile = 0; ok; ++tile) {
      if (tile > 0) {
        if (!finalize(tile - 1, prev)) break;
        if (prev.last() && !epilogue(tile - 1, prev)) break;
      }
      if (!cur.valid) break;
      if (!produce(tile, cur)) break;
      prev = cur;
      cur.advance(a);
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
  CUtensorMap tm_kv, tm_q;
  const long pool_rows = (long)a.num_pages * kPage;
  const long q_rows = (long)a.batch * kHeads;
  if (!make_map(&tm_kv, a.pool, pool_rows, 64, kOwn, CU_TENSOR_MAP_SWIZZLE_128B) ||
      !make_map(&tm_q, a.q_lat, q_rows, 64, kHeads, CU_TENSOR_MAP_SWIZZLE_128B))
    return cudaErrorInvalidValue;
  const float scale_log2 = a.scale * 1.4426950408889634f;
  attn_sm100_kernel<<<2 * parts, kThreads, kSmemBytes, s>>>(tm_kv, tm_q, a, scale_log2);
  return cudaGetLastError();
}

}  // namespace sm100
}  // namespace mla
