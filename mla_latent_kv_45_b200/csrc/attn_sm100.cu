// Latent decode attention on sm_100a tensor cores (bf16, 128 heads, 576-wide
// cache rows = 512 latent + 64 shared RoPE key, 64-row pages).
//
// The method: every head of a sequence scores the same cached rows, so the
// 128 absorbed queries q_lat form a dense [128 x 576] operand and the cached
// rows a dense [rows x 576] one: S = rows . q_lat^T and O += P^T-weighted rows
// are genuine tensor-core contractions ("从零理解 MLA", 解耦 RoPE absorbed_step:
// s_c + s_r against the cached [c ; k_R] rows, softmax, z = attn . c;
// "解耦 RoPE（MLA 下）" §3.3: one k_R shared by all heads, i.e. MQA-shaped).
//
// Design (one CTA pair = a 2-CTA cluster per work partition, pair MMAs):
//  * A step is 4 pages (256 rows): CTA r holds pages 2r and 2r+1 of the step.
//  * Scores, rows on TMEM lanes.  One pair MMA chain (tcgen05 cta_group::2,
//    M = 256 rows, N = 128 heads, K = 576) per step: CTA r supplies its 128
//    rows as A and q_lat heads [64r, 64r+64) as its half of B, and receives
//    S^T for its 128 rows x all 128 heads.  No score is computed twice.  The
//    rows stream through a ring of 64-column chunks, each released as soon as
//    its four MMAs complete.
//  * Softmax per head is a reduction over TMEM lanes: each warp reduces its
//    32 rows with a shuffle transpose (lane L ends with heads 2L, 2L+1), the
//    four warps of a column half through shared memory, and the pair by an
//    8-byte st.async exchange per lane.  Both CTAs then hold the same tile
//    maximum; the running max moves only when it grows by more than 2^8.
//  * Values.  The fp32 accumulator for 128 heads x 512 latent columns would
//    fill all of TMEM, so it is held transposed and split: O^T = V^T P with
//    pair MMAs (M = 256 latent columns, two per page, N = 128 heads, K = 64
//    rows).  CTA r owns latent columns [256b + 128r, +128) for b = 0, 1 (TMEM
//    lane = latent column, TMEM column = head) and supplies heads [64r, 64r+64)
//    of P for all 256 rows of the step as its half of B (MN-major).  It writes
//    that half for its own rows itself; the partner's rows arrive by one 16 KB
//    shared-to-shared bulk copy per step (asynchronous proxy, counted on an
//    mbarrier of the receiving CTA).
//  * The latent columns a CTA needs for P.V are loaded in their own ring
//    (mostly L2 hits: the pair has just streamed the rows for the scores; the
//    row loads carry an evict-last L2 policy and these reloads evict-first).
//  * Row sums come from the bf16 P values the MMA consumes, reduced like the
//    maxima (per warp through the shuffle transpose, across the pair at the
//    end of a sequence piece).
//  * Warps 0-7 softmax + epilogue; warp 8 loads score rows; warp 9 TMEM
//    allocation, q_lat loads and (even CTA) the score MMAs; warp 10 (even CTA)
//    the P.V MMAs; warp 11 the latent-column loads for P.V.
//  * Partitions come from the plan kernel (equal cost: each sequence counts a
//    few virtual pages for its fixed cost besides its pages); a sequence cut by
//    a partition boundary writes an unnormalised partial that the combine
//    kernel merges.
//  * Every wait is bounded (globaltimer); on expiry the kernel records
//    kErrTimeout in the error word, stops issuing work, drains what it issued
//    and exits.  No TMA multicast is used.
#include <cuda.h>

#include "api_checks.h"
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
constexpr int kStepPages = 4;    // pages per step; CTA r holds step pages 2r, 2r+1
constexpr int kKSlots = 3;       // score-row chunk ring
constexpr int kVSlots = 3;       // latent-column chunk ring
constexpr int kSoftmaxThreads = 256;
constexpr int kThreads = kSoftmaxThreads + 128;
constexpr int kWarpLoad = 8, kWarpS = 9, kWarpPV = 10, kWarpV = 11;
constexpr uint64_t kTimeoutNs = 2000000000ull;
constexpr int kI8Row = 656;      // bytes of an int8 cache row (512 codes, 64 bf16 k_R, scale, pad)
constexpr uint32_t kSleepNs = 20000;   // suspend hint of a waiting thread (woken at completion)

// Shared memory (byte offsets from a 1024-byte aligned base).  Every operand
// tile is made of 64-row x 64-column bf16 boxes with the 128-byte swizzle.
constexpr int kBox = kPage * 128;           // 8 KB
constexpr int kQBytes = 9 * kBox;           // q_lat heads [64r, 64r+64), all 576 columns
constexpr int kKChunk = 2 * kBox;           // the CTA's 128 rows x 64 columns
constexpr int kVChunk = 2 * kBox;           // one page's 64 rows x 128 latent columns
constexpr int kPBytes = kStepPages * kBox;  // P: 256 rows x this CTA's 64 heads (MN-major)
constexpr int kStgBytes = 2 * kBox;         // P of the CTA's rows for the partner's heads
constexpr int kOffQ = 0;
constexpr int kOffK = kOffQ + kQBytes;
constexpr int kOffV = kOffK + kKSlots * kKChunk;
constexpr int kOffP = kOffV + kVSlots * kVChunk;
constexpr int kOffStg = kOffP + kPBytes;
constexpr int kOffRed = kOffStg + kStgBytes;   // [2 halves][4 warps][64] floats
constexpr int kOffX = kOffRed + 2048;          // [2 parities][128] the partner's tile maxima
constexpr int kOffMb = kOffX + 1024;           // [8 warps][64] running max, per warp
constexpr int kOffAlpha = kOffMb + 2048;       // [128] rescale factors
constexpr int kOffLinv = kOffAlpha + 512;      // [128] 1 / row sum of the pair, per head
constexpr int kOffLx = kOffLinv + 512;         // [128] the partner's row sums
constexpr int kOffBar = kOffLx + 512;
constexpr int kSmemBytes = kOffBar + 512 + 1024;
static_assert(kOffK % 1024 == 0 && kOffV % 1024 == 0 && kOffP % 1024 == 0 &&
                  kOffStg % 1024 == 0,
              "swizzled tiles start on 1024-byte boundaries");
static_assert(kSmemBytes <= 232448, "shared memory per CTA");

// TMEM columns
constexpr uint32_t kTmemO = 0;     // O^T: two blocks of 128 heads (lane = latent column)
constexpr uint32_t kTmemS = 256;   // S^T: two buffers of 128 heads (lane = cache row)
constexpr uint32_t kTmemCols = 512;

constexpr uint32_t kIdescS = idesc_bf16(256, 128, 0, 0);    // A = rows, B = q_lat (K-major)
constexpr uint32_t kIdescPV = idesc_bf16(256, 128, 1, 1);   // A = V^T, B = P (MN-major)
constexpr uint16_t kBoth = 3;

struct Bars {
  uint64_t k_full[kKSlots];   // even CTA: both CTAs' row chunks landed (tx; int8 rows: 2 arrivals)
  uint64_t k_land[kKSlots];   // int8 rows: this CTA's chunk landed (local tx), before conversion
  uint64_t k_empty[kKSlots];  // the score MMAs reading the slot complete (pair commit)
  uint64_t v_land[kVSlots];   // this CTA's latent chunk landed (local tx)
  uint64_t v_full[kVSlots];   // even CTA: both CTAs' latent chunks ready (2 arrivals)
  uint64_t v_empty[kVSlots];  // the P.V MMAs reading the slot complete (pair commit)
  uint64_t q_full;            // even CTA: q_lat halves of both CTAs landed (tx)
  uint64_t q_free;            // the piece's last score MMAs complete (pair commit)
  uint64_t s_full[2];         // scores in buffer i complete (pair commit)
  uint64_t s_free[2];         // even CTA: both CTAs read score buffer i (16 warps)
  uint64_t mx[2];             // the partner's tile maxima landed (st.async tx)
  uint64_t p_rx;              // the partner's P rows landed (bulk copy tx)
  uint64_t p_ready;           // even CTA: P and rescaled O^T of both CTAs ready (16 warps)
  uint64_t pv_done;           // the step's P.V MMAs complete (pair commit)
  uint64_t lx;                // the partner's row sums landed (st.async tx)
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

// 16 int8 codes times the row's power-of-two scale s, as 16 bf16 values (two
// 16-byte units, element order kept).  q + 128 is placed in the low mantissa
// byte of 2^23, so fma(2^23 + q + 128, s, -(2^23 + 128) s) = q s exactly, and
// q s (at most 8 significant bits) is exact in bf16.
__device__ __forceinline__ void i8x16_to_bf16(const uint4 in, float s, uint4 &lo, uint4 &hi) {
  const float bias = -8388736.0f * s;
  const uint32_t w[4] = {in.x ^ 0x80808080u, in.y ^ 0x80808080u, in.z ^ 0x80808080u,
                         in.w ^ 0x80808080u};
  uint32_t o[8];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    float f[4];
#pragma unroll
    for (int k = 0; k < 4; ++k)
      f[k] = fmaf(__uint_as_float(__byte_perm(w[i], 0x4B000000u, 0x7540u + k)), s, bias);
    o[2 * i] = pack_bf16(f[0], f[1]);
    o[2 * i + 1] = pack_bf16(f[2], f[3]);
  }
  lo = make_uint4(o[0], o[1], o[2], o[3]);
  hi = make_uint4(o[4], o[5], o[6], o[7]);
}

// The fp32 scale of an int8 row (bytes 640..643 of its 656).
__device__ __forceinline__ float int8_row_scale(const AttnArgs &a, int page, int r) {
  return __ldg(reinterpret_cast<const float *>(static_cast<const uint8_t *>(a.pool) +
                                               ((long)page * kPage + r) * kI8Row + 640));
}

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
// Named barrier over the 128 threads of softmax column half g (warps 4g..4g+3).
__device__ __forceinline__ void half_sync(int g) {
  asm volatile("bar.sync %0, 128;" ::"r"(2 + g) : "memory");
}

struct MaxOp {
  __device__ __forceinline__ float operator()(float a, float b) const { return fmaxf(a, b); }
};
struct AddOp {
  __device__ __forceinline__ float operator()(float a, float b) const { return a + b; }
};

// One round of the warp transpose-reduction: n values per lane -> n / 2.  The
// lane whose bit `o` is clear keeps the lower half of its values and receives
// the partner's lower half; the other keeps and receives the upper half.
template <int n, int o, class Op>
__device__ __forceinline__ void xpose_round(float *t, int lane, Op op) {
  const bool up = lane & o;
#pragma unroll
  for (int i = 0; i < n / 2; ++i) {
    const float keep = up ? t[i + n / 2] : t[i];
    const float send = up ? t[i] : t[i + n / 2];
    t[i] = op(keep, __shfl_xor_sync(0xffffffffu, send, o));
  }
}

// Reduces 64 per-lane values across the warp's 32 lanes column-wise: on return
// t[0], t[1] of lane L hold the reductions of columns 2L and 2L+1.
template <class Op>
__device__ __forceinline__ void xpose_reduce64(const float (&v)[64], float (&t)[32], int lane,
                                               Op op) {
  const bool up = lane & 16;
#pragma unroll
  for (int i = 0; i < 32; ++i) {
    const float keep = up ? v[i + 32] : v[i];
    const float send = up ? v[i] : v[i + 32];
    t[i] = op(keep, __shfl_xor_sync(0xffffffffu, send, 16));
  }
  xpose_round<32, 8>(t, lane, op);
  xpose_round<16, 4>(t, lane, op);
  xpose_round<8, 2>(t, lane, op);
  xpose_round<4, 1>(t, lane, op);
}

// Sequential walk over the steps (4 pages) of one partition.
struct StepCursor {
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
    lp += kStepPages;
    if (lp >= seg.lp1) {
      valid = walk.next(a, seg);
      lp = seg.lp0;
      ++nseg;
    }
  }
  __device__ __forceinline__ bool first() const { return lp == seg.lp0; }
  __device__ __forceinline__ bool last() const { return lp + kStepPages >= seg.lp1; }
  // pages of this step that belong to the piece
  __device__ __forceinline__ int npages() const { return min(kStepPages, seg.lp1 - lp); }
  // rows of step page j that hold data (>= 1 for j < npages())
  __device__ __forceinline__ int rows_valid(int j) const { return seg.len - (lp + j) * kPage; }
  __device__ __forceinline__ int page(const AttnArgs &a, int j) const {
    return a.block_table[(long)seg.b * a.max_pages + lp + j];
  }
};

// kI8: the cache holds 656-byte int8 rows (MLA_CACHE_INT8).  tm_rows then maps
// the rows' bf16 k_R columns, tm_i8k 64 int8 columns x 64 rows (score chunks)
// and tm_i8v 128 int8 columns x 64 rows (latent columns for P.V); the int8
// chunks land in the upper half of their ring slot and the loading warp turns
// them in place into the same bf16 operand layout the bf16 rows arrive in.
template <bool kI8>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kThreads, 1)
    attn_sm100_kernel(const __grid_constant__ CUtensorMap tm_rows,
                      const __grid_constant__ CUtensorMap tm_q,
                      const __grid_constant__ CUtensorMap tm_i8k,
                      const __grid_constant__ CUtensorMap tm_i8v, const AttnArgs a,
                      const float scale_log2) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  Bars *bars = reinterpret_cast<Bars *>(smem + kOffBar);
  const Ctx ctx{bars, a.err};
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const uint32_t peer = rank ^ 1u;
  const bool leader = rank == 0;
  const int part = blockIdx.x >> 1;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kKSlots; ++s) {
      mbar_init(&bars->k_full[s], kI8 ? 2 : 1);
      mbar_init(&bars->k_land[s], 1);
      mbar_init(&bars->k_empty[s], 1);
    }
    for (int s = 0; s < kVSlots; ++s) {
      mbar_init(&bars->v_land[s], 1);
      mbar_init(&bars->v_full[s], 2);
      mbar_init(&bars->v_empty[s], 1);
    }
    mbar_init(&bars->q_full, 1);
    mbar_init(&bars->q_free, 1);
    for (int i = 0; i < 2; ++i) {
      mbar_init(&bars->s_full[i], 1);
      mbar_init(&bars->s_free[i], 16);
      mbar_init(&bars->mx[i], 1);
    }
    mbar_init(&bars->p_rx, 1);
    mbar_init(&bars->p_ready, 16);
    mbar_init(&bars->pv_done, 1);
    mbar_init(&bars->lx, 1);
    mbar_init(&bars->drain_s, 1);
    mbar_init(&bars->drain_pv, 1);
    bars->abort = 0;
    fence_mbar_init();
  }
  if (warp == kWarpLoad && lane == 0) {
    prefetch_tmap(&tm_rows);
    prefetch_tmap(&tm_q);
    if (kI8) {
      prefetch_tmap(&tm_i8k);
      prefetch_tmap(&tm_i8v);
    }
  }
  if (warp == kWarpS) {
    tmem_alloc_pair(&bars->tmem_base, kTmemCols);
    tc_fence_before();
  }
  __syncwarp();   // thread 0 alone set up the barriers
  __syncthreads();
  tc_fence_after();
  cluster_sync();  // both CTAs' barriers exist before any remote access
  const uint32_t tmem = bars->tmem_base;
  // the set-up above overlaps the plan kernel; its results are read from here on
  grid_dep_wait();
  grid_dep_launch();
  const PlanHeader hdr = *a.hdr;
  auto lead = [&](uint64_t *bar) { return mapa(smem_u32(bar), 0); };

  StepCursor cur;
  cur.init(a, hdr, part);

  if (kI8 && warp == kWarpLoad) {
    // ---------- int8 rows: this CTA's 128 rows of each step, 64 columns a chunk,
    // converted in place by the whole warp; the k_R chunk (bf16) is used as loaded
    int nk = 0, pend_slot = 0, pend_nk = 0, pend_c = 0;
    bool ok = true, pend = false, pend_has[2] = {false, false};
    float pend_sc[2][2] = {{0.f, 0.f}, {0.f, 0.f}};
    // chunk idx (in `slot`) landed: int8 codes of page sp at +8 KB + 4 KB sp, row r
    // at 64 r, its 16-byte unit u at (u ^ ((r >> 1) & 3)) << 4 (64-byte swizzle: the
    // lanes of a warp, one row each, read distinct banks); bf16 out at +8 KB sp,
    // row r at 128 r, 16-byte unit u at (u ^ (r & 7)) << 4.
    // Page 1's output covers page 0's input and, from row 32 on, its own: page 0
    // is converted first, and every 32-row batch is read before it is written.
    auto finish_k = [&](int slot, int idx, int c, const bool (&has)[2],
                        const float (&sc)[2][2]) -> bool {
      if (!wait_bar(ctx, &bars->k_land[slot], (idx / kKSlots) & 1)) return false;
      if (c < 8) {
        uint8_t *base = smem + kOffK + slot * kKChunk;
        for (int sp = 0; sp < 2; ++sp) {
          if (!has[sp]) continue;
          for (int hf = 0; hf < 2; ++hf) {
            const int r = 32 * hf + lane;
            const uint8_t *in = base + 8192 + 4096 * sp + 64 * r;
            uint4 v[4];
#pragma unroll
            for (int j = 0; j < 4; ++j)
              v[j] = *reinterpret_cast<const uint4 *>(in + ((j ^ ((r >> 1) & 3)) << 4));
            __syncwarp();
            uint8_t *out = base + kBox * sp + 128 * r;
#pragma unroll
            for (int j = 0; j < 4; ++j) {
              uint4 lo, hi;
              i8x16_to_bf16(v[j], sc[sp][hf], lo, hi);
              *reinterpret_cast<uint4 *>(out + (((2 * j) ^ (r & 7)) << 4)) = lo;
              *reinterpret_cast<uint4 *>(out + (((2 * j + 1) ^ (r & 7)) << 4)) = hi;
            }
            __syncwarp();
          }
        }
        fence_proxy_async_smem();
      }
      __syncwarp();
      if (lane == 0) mbar_arrive_remote(lead(&bars->k_full[slot]));
      return true;
    };
    for (; cur.valid && ok; cur.advance(a)) {
      const int np = cur.npages();
      int pages[2];
      bool has[2];
      float sc[2][2];
      for (int sp = 0; sp < 2; ++sp) {
        const int j = 2 * (int)rank + sp;
        pages[sp] = -1;
        if (j < np) {
          int page = cur.page(a, j);
          if (page < 0 || page >= a.num_pages) {
            if (lane == 0) {
              set_error(a.err, kErrRange);
              a.bad[cur.seg.b] = 1;
            }
            page = 0;
          }
          pages[sp] = page;
        }
        has[sp] = pages[sp] >= 0;
        for (int hf = 0; hf < 2; ++hf)
          sc[sp][hf] = has[sp] ? int8_row_scale(a, pages[sp], 32 * hf + lane) : 0.f;
      }
      const int nown = (int)has[0] + (int)has[1];
      for (int c = 0; c < 9; ++c, ++nk) {
        const int slot = nk % kKSlots;
        if (nk >= kKSlots && !wait_bar(ctx, &bars->k_empty[slot], ((nk / kKSlots) - 1) & 1)) {
          ok = false;
          break;
        }
        if (lane == 0) {
          uint8_t *dst = smem + kOffK + slot * kKChunk;
          if (c < 8) {
            mbar_expect_tx(&bars->k_land[slot], nown * 4096);
            for (int sp = 0; sp < 2; ++sp)
              if (has[sp])
                tma_load_2d_hint(dst + 8192 + 4096 * sp, &tm_i8k, 64 * c, pages[sp] * kPage,
                                 &bars->k_land[slot], l2_policy_evict_last());
          } else {
            mbar_expect_tx(&bars->k_land[slot], nown * kBox);
            for (int sp = 0; sp < 2; ++sp)
              if (has[sp])
                tma_load_2d_hint(dst + kBox * sp, &tm_rows, 512, pages[sp] * kPage,
                                 &bars->k_land[slot], l2_policy_evict_last());
          }
        }
        __syncwarp();
        if (pend && !finish_k(pend_slot, pend_nk, pend_c, pend_has, pend_sc)) {
          ok = false;
          break;
        }
        pend = true;
        pend_slot = slot;
        pend_nk = nk;
        pend_c = c;
        for (int sp = 0; sp < 2; ++sp) {
          pend_has[sp] = has[sp];
          pend_sc[sp][0] = sc[sp][0];
          pend_sc[sp][1] = sc[sp][1];
        }
      }
    }
    if (ok && pend) finish_k(pend_slot, pend_nk, pend_c, pend_has, pend_sc);
  } else if (warp == kWarpLoad) {
    // ------------------------- this CTA's 128 rows of each step, in 64-column chunks
    if (lane == 0) {
      int nk = 0;
      bool ok = true;
      for (; cur.valid && ok; cur.advance(a)) {
        const int np = cur.npages();
        int pages[2];
        for (int sp = 0; sp < 2; ++sp) {
          const int j = 2 * (int)rank + sp;
          pages[sp] = -1;
          if (j < np) {
            int page = cur.page(a, j);
            if (page < 0 || page >= a.num_pages) {
              set_error(a.err, kErrRange);
              a.bad[cur.seg.b] = 1;
              page = 0;
            }
            pages[sp] = page;
          }
        }
        for (int c = 0; c < 9; ++c, ++nk) {
          const int slot = nk % kKSlots;
          if (nk >= kKSlots && !wait_bar(ctx, &bars->k_empty[slot], ((nk / kKSlots) - 1) & 1)) {
            ok = false;
            break;
          }
          // one 8 KB box per page of the step, from whichever CTA holds it
          if (leader) mbar_expect_tx(&bars->k_full[slot], np * kBox);
          uint8_t *dst = smem + kOffK + slot * kKChunk;
          // evict-last: the rows are read again (latent columns) for P.V shortly after
          for (int sp = 0; sp < 2; ++sp)
            if (pages[sp] >= 0)
              tma_load_2d_pair_hint(dst + sp * kBox, &tm_rows, 64 * c, pages[sp] * kPage,
                                    lead(&bars->k_full[slot]), l2_policy_evict_last());
        }
      }
    }
  } else if (warp == kWarpV) {
    // ------------- each page's 64 rows of this CTA's 256 latent columns (P.V A operand)
    int nv = 0, prev_slot = 0, prev_valid = kPage;
    float prev_sc0 = 0.f, prev_sc1 = 0.f;
    bool ok = true, pending = false;
    // hands chunk `idx` (landed) to the P.V issuer; rows past the sequence end
    // hold arbitrary bytes and are zeroed so that 0 * (stale bytes) cannot reach O
    auto finish = [&](int slot, int idx, int valid, float sc0, float sc1) -> bool {
      if (!wait_bar(ctx, &bars->v_land[slot], (idx / kVSlots) & 1)) return false;
      if (kI8) {
        // int8 codes of row r at +8 KB + 128 r (128 latent columns, 16-byte unit j
        // at (j ^ (r & 7)) << 4: 128-byte swizzle, so the lanes read distinct banks)
        // -> bf16 boxes 0 (columns 0-63) at 128 r and 1 (64-127) at 8 KB + 128 r: box
        // 1's row r is exactly the input row r, which the lane has read before it writes
        uint8_t *dst = smem + kOffV + slot * kVChunk;
        for (int hf = 0; hf < 2; ++hf) {
          const int r = 32 * hf + lane;
          const float sc = hf ? sc1 : sc0;
          uint4 v[8];
          const uint8_t *in = dst + kBox + 128 * r;
#pragma unroll
          for (int j = 0; j < 8; ++j)
            v[j] = *reinterpret_cast<const uint4 *>(in + ((j ^ (r & 7)) << 4));
#pragma unroll
          for (int j = 0; j < 8; ++j) {
            uint4 lo = make_uint4(0, 0, 0, 0), hi = lo;
            if (r < valid) i8x16_to_bf16(v[j], sc, lo, hi);
            uint8_t *out = dst + (j >> 2) * kBox + 128 * r;
            const int u = 2 * (j & 3);
            *reinterpret_cast<uint4 *>(out + ((u ^ (r & 7)) << 4)) = lo;
            *reinterpret_cast<uint4 *>(out + (((u + 1) ^ (r & 7)) << 4)) = hi;
          }
        }
        fence_proxy_async_smem();
      } else if (valid < kPage) {
        uint8_t *dst = smem + kOffV + slot * kVChunk;
        for (int i = lane; i < (kPage - valid) * 16; i += 32) {
          const int row = valid + (i >> 4), box = (i >> 3) & 1, piece = i & 7;
          *reinterpret_cast<uint4 *>(dst + box * kBox + row * 128 + piece * 16) =
              make_uint4(0, 0, 0, 0);
        }
        fence_proxy_async_smem();
      }
      __syncwarp();
      if (lane == 0) mbar_arrive_remote(lead(&bars->v_full[slot]));
      return true;
    };
    for (; cur.valid && ok; cur.advance(a)) {
      const int np = cur.npages();
      for (int pg = 0; pg < np && ok; ++pg) {
        int page = cur.page(a, pg);
        if (page < 0 || page >= a.num_pages) page = 0;   // flagged by the row loader
        const int valid = min(cur.rows_valid(pg), kPage);
        for (int blk = 0; blk < 2; ++blk, ++nv) {
          const int slot = nv % kVSlots;
          if (nv >= kVSlots && !wait_bar(ctx, &bars->v_empty[slot], ((nv / kVSlots) - 1) & 1)) {
            ok = false;
            break;
          }
          if (lane == 0) {
            uint8_t *dst = smem + kOffV + slot * kVChunk;
            // the last read of these bytes, so evict-first
            if (kI8) {
              // int8 latent columns 256 blk + 128 r .. +128 of all 64 rows, upper half
              mbar_expect_tx(&bars->v_land[slot], kBox);
              tma_load_2d_hint(dst + kBox, &tm_i8v, 256 * blk + 128 * (int)rank, page * kPage,
                               &bars->v_land[slot], l2_policy_evict_first());
            } else {
              // box sub: latent columns 256 blk + 128 r + 64 sub, all 64 rows
              mbar_expect_tx(&bars->v_land[slot], kVChunk);
              for (int sub = 0; sub < 2; ++sub)
                tma_load_2d_hint(dst + sub * kBox, &tm_rows,
                                 256 * blk + 128 * (int)rank + 64 * sub, page * kPage,
                                 &bars->v_land[slot], l2_policy_evict_first());
            }
          }
          float sc0 = 0.f, sc1 = 0.f;
          if (kI8) {
            sc0 = int8_row_scale(a, page, lane);
            sc1 = int8_row_scale(a, page, lane + 32);
          }
          __syncwarp();
          if (pending && !finish(prev_slot, nv - 1, prev_valid, prev_sc0, prev_sc1)) {
            ok = false;
            break;
          }
          prev_slot = slot;
          prev_valid = valid;
          prev_sc0 = sc0;
          prev_sc1 = sc1;
          pending = true;
        }
      }
    }
    if (ok && pending) finish(prev_slot, nv - 1, prev_valid, prev_sc0, prev_sc1);
  } else if (warp == kWarpS) {
    // ----------------- q_lat halves (both CTAs); the even CTA issues the score MMAs
    if (lane == 0) {
      const uint64_t qd0 = sdesc(smem_u32(smem + kOffQ), 16, 1024, 2);
      const uint64_t kd0 = sdesc(smem_u32(smem + kOffK), 16, 1024, 2);
      int step = 0, nk = 0;
      bool ok = true;
      for (; cur.valid && ok; cur.advance(a), ++step) {
        if (cur.first()) {
          // the previous piece's score MMAs must finish before q_lat is replaced
          if (cur.nseg > 0 && !wait_bar(ctx, &bars->q_free, (cur.nseg - 1) & 1)) break;
          if (leader) mbar_expect_tx(&bars->q_full, 2 * kQBytes);
          for (int c = 0; c < 9; ++c)
            tma_load_2d_pair(smem + kOffQ + c * kBox, &tm_q, 64 * c,
                             cur.seg.b * kHeads + 64 * (int)rank, lead(&bars->q_full));
          if (leader && !wait_bar(ctx, &bars->q_full, cur.nseg & 1)) break;
        }
        if (!leader) continue;
        const int sb = step & 1;
        // score buffer sb was last read by the softmax of step - 2
        if (step >= 2 && !wait_bar(ctx, &bars->s_free[sb], ((step >> 1) - 1) & 1)) break;
        const uint32_t sd = tmem + kTmemS + 128 * sb;
        for (int c = 0; c < 9; ++c, ++nk) {
          const int slot = nk % kKSlots;
          if (!wait_bar(ctx, &bars->k_full[slot], (nk / kKSlots) & 1)) {
            ok = false;
            break;
          }
          tc_fence_after();
          // descriptors advance by address >> 4 in their low field (no carry: < 256 KB)
          const uint64_t kd = kd0 + (uint64_t)((slot * kKChunk) >> 4);
          const uint64_t qd = qd0 + (uint64_t)((c * kBox) >> 4);
#pragma unroll
          for (int k = 0; k < 4; ++k)
            umma_pair_ss(sd, kd + (uint64_t)((32 * k) >> 4), qd + (uint64_t)((32 * k) >> 4),
                         kIdescS, (c | k) ? 1u : 0u);
          umma_commit_pair(&bars->k_empty[slot], kBoth);
        }
        if (!ok) break;
        if (cur.last()) umma_commit_pair(&bars->q_free, kBoth);
        umma_commit_pair(&bars->s_full[sb], kBoth);
      }
      if (leader) {
        umma_commit_pair(&bars->drain_s, 1);
        drain_bar(&bars->drain_s, 0);
      }
    }
  } else if (warp == kWarpPV) {
    // ------------------------------------------------- P.V pair MMAs (even CTA)
    if (lane == 0 && leader) {
      const uint64_t vd0 = sdesc(smem_u32(smem + kOffV), kBox, 1024, 2);
      const uint64_t pd0 = sdesc(smem_u32(smem + kOffP), kBox, 1024, 2);
      int step = 0, nv = 0;
      bool ok = true;
      for (; cur.valid && ok; cur.advance(a), ++step) {
        if (!wait_bar(ctx, &bars->p_ready, step & 1)) break;
        tc_fence_after();
        const int np = cur.npages();
        const bool first = cur.first();
        for (int pg = 0; pg < np && ok; ++pg) {
          for (int blk = 0; blk < 2; ++blk, ++nv) {
            const int slot = nv % kVSlots;
            if (!wait_bar(ctx, &bars->v_full[slot], (nv / kVSlots) & 1)) {
              ok = false;
              break;
            }
            tc_fence_after();
            // A = V^T: two 64-column boxes (8 KB apart), B = P rows of page pg;
            // both MN-major, 16 rows (2 KB) per MMA
            const uint64_t vd = vd0 + (uint64_t)((slot * kVChunk) >> 4);
            const uint64_t pd = pd0 + (uint64_t)((pg * kBox) >> 4);
#pragma unroll
            for (int k = 0; k < 4; ++k)
              umma_pair_ss(tmem + kTmemO + 128 * blk, vd + (uint64_t)((2048 * k) >> 4),
                           pd + (uint64_t)((2048 * k) >> 4), kIdescPV,
                           (first && pg == 0 && k == 0) ? 0u : 1u);
            umma_commit_pair(&bars->v_empty[slot], kBoth);
          }
        }
        if (!ok) break;
        umma_commit_pair(&bars->pv_done, kBoth);
      }
      umma_commit_pair(&bars->drain_pv, 1);
      drain_bar(&bars->drain_pv, 0);
    }
  } else if (warp < 8) {
    // ------------------------------------------- softmax + epilogue (warps 0-7)
    const int g = warp >> 2;                 // column half: heads [64 g, 64 g + 64)
    const int quad = warp & 3;               // TMEM lanes [32 quad, 32 quad + 32)
    const int row = quad * 32 + lane;        // this CTA's row of the step
    const int sp = quad >> 1;                // ... on the CTA's page sp (step page 2r + sp)
    const int k = row & 63;                  // ... row k of that page
    const uint32_t lane_off = static_cast<uint32_t>(quad * 32) << 16;
    float *red = reinterpret_cast<float *>(smem + kOffRed);
    float *xmax = reinterpret_cast<float *>(smem + kOffX);
    float *mb = reinterpret_cast<float *>(smem + kOffMb) + warp * 64;
    float *alpha_s = reinterpret_cast<float *>(smem + kOffAlpha);
    float *linv = reinterpret_cast<float *>(smem + kOffLinv);
    float *lx = reinterpret_cast<float *>(smem + kOffLx);
    const bool outgoing = g != (int)rank;    // this half of P is the partner's B operand
    float m0 = -INFINITY, m1 = -INFINITY;    // running max (log2 units) of heads 64g + 2 lane, +1
    float l0 = 0.f, l1 = 0.f;                // this warp's rows' share of their row sums

    // Every softmax thread runs every barrier of a step even after a failed
    // wait (it then skips the remaining waits and computes garbage), and the
    // 256 threads agree on stopping by a vote at the end of the step, so no
    // thread is ever left alone at a named barrier.
    auto produce = [&](int i, const StepCursor &tc) -> bool {
      bool ok = true;
      const bool first = tc.first();
      const int sb = i & 1;
      if (threadIdx.x == 0) {
        mbar_expect_tx(&bars->mx[sb], 2 * 64 * 4);   // the partner's maxima of step i
        mbar_expect_tx(&bars->p_rx, kStgBytes);      // the partner's P rows of step i
      }
      ok = ok && wait_bar(ctx, &bars->s_full[sb], (i >> 1) & 1);
      tc_fence_after();
      float v[64];
      tmem_ld32f(tmem + lane_off + kTmemS + 128 * sb + 64 * g, v);
      tmem_ld32f(tmem + lane_off + kTmemS + 128 * sb + 64 * g + 32, v + 32);
      tmem_wait_ld();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_remote(lead(&bars->s_free[sb]));
      const int jp = 2 * (int)rank + sp;
      const bool valid = jp < tc.npages() && k < tc.rows_valid(jp);
#pragma unroll
      for (int h = 0; h < 64; ++h) v[h] = valid ? v[h] : -INFINITY;
      // tile max of heads 64g + 2 lane, +1: this warp, the half's four warps, the pair
      float t[32];
      xpose_reduce64(v, t, lane, MaxOp());
      reinterpret_cast<float2 *>(red + (g * 4 + quad) * 64)[lane] = make_float2(t[0], t[1]);
      half_sync(g);
      float c0 = -INFINITY, c1 = -INFINITY;
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const float2 x = reinterpret_cast<const float2 *>(red + (g * 4 + q) * 64)[lane];
        c0 = fmaxf(c0, x.x);
        c1 = fmaxf(c1, x.y);
      }
      if (quad == 0)
        st_async_v2(mapa(smem_u32(xmax + sb * 128 + 64 * g + 2 * lane), peer), c0, c1,
                    mapa(smem_u32(&bars->mx[sb]), peer));
      ok = ok && wait_bar(ctx, &bars->mx[sb], (i >> 1) & 1);
      const float2 pm = reinterpret_cast<const float2 *>(xmax + sb * 128 + 64 * g)[lane];
      const float t0 = fmaxf(c0, pm.x) * scale_log2, t1 = fmaxf(c1, pm.y) * scale_log2;
      const float n0 = first ? t0 : (t0 > m0 + 8.0f ? t0 : m0);
      const float n1 = first ? t1 : (t1 > m1 + 8.0f ? t1 : m1);
      const float a0 = first ? 1.f : ex2(m0 - n0), a1 = first ? 1.f : ex2(m1 - n1);
      m0 = n0;
      m1 = n1;
      reinterpret_cast<float2 *>(mb)[lane] = make_float2(n0, n1);
      __syncwarp();
      // P (bf16) of my row for the half's 64 heads
      uint32_t w[32];
#pragma unroll
      for (int q = 0; q < 16; ++q) {
        const float4 m4 = reinterpret_cast<const float4 *>(mb)[q];
        w[2 * q] = pack_bf16(ex2(fmaf(v[4 * q], scale_log2, -m4.x)),
                             ex2(fmaf(v[4 * q + 1], scale_log2, -m4.y)));
        w[2 * q + 1] = pack_bf16(ex2(fmaf(v[4 * q + 2], scale_log2, -m4.z)),
                                 ex2(fmaf(v[4 * q + 3], scale_log2, -m4.w)));
      }
      // row sums from the rounded values the MMA consumes
      {
        float pr[64];
#pragma unroll
        for (int q = 0; q < 32; ++q) {
          pr[2 * q] = bf16_lo(w[q]);
          pr[2 * q + 1] = bf16_hi(w[q]);
        }
        xpose_reduce64(pr, t, lane, AddOp());
      }
      l0 = first ? t[0] : fmaf(l0, a0, t[0]);
      l1 = first ? t[1] : fmaf(l1, a1, t[1]);
      // the P buffer (and the staging copy) is free once the previous step's P.V completed
      if (i > 0) ok = ok && wait_bar(ctx, &bars->pv_done, (i - 1) & 1);
      // row k of a 64-row box: 16-byte chunk c at k*128 + ((c ^ (k & 7)) << 4)
      uint8_t *prow = (outgoing ? smem + kOffStg + sp * kBox
                                : smem + kOffP + (2 * (int)rank + sp) * kBox) + k * 128;
#pragma unroll
      for (int c = 0; c < 8; ++c)
        *reinterpret_cast<uint4 *>(prow + ((c ^ (k & 7)) << 4)) =
            make_uint4(w[4 * c], w[4 * c + 1], w[4 * c + 2], w[4 * c + 3]);
      fence_proxy_async_smem();              // P -> the MMA / the bulk copy
      if (outgoing) {
        half_sync(g);
        if (quad == 0 && lane == 0)
          bulk_copy_cta_to_cluster(mapa(smem_u32(smem + kOffP + 2 * (int)rank * kBox), peer),
                                   smem_u32(smem + kOffStg), kStgBytes,
                                   mapa(smem_u32(&bars->p_rx), peer));
      }
      // O^T holds the steps before i: rescale its head columns when the max moved
      if (quad == 0) reinterpret_cast<float2 *>(alpha_s + 64 * g)[lane] = make_float2(a0, a1);
      if (softmax_any(a0 != 1.f || a1 != 1.f)) {
        tc_fence_after();
        const uint32_t ob = tmem + lane_off + kTmemO + 128 * g;   // block g, lane = column
        for (int c = 0; c < 128; c += 32) {
          uint32_t r[32];
          tmem_ld32(ob + c, r);
          tmem_wait_ld();
#pragma unroll
          for (int kk = 0; kk < 32; ++kk)
            r[kk] = __float_as_uint(__uint_as_float(r[kk]) * alpha_s[c + kk]);
          tmem_st32(ob + c, r);
        }
        tmem_wait_st();
      }
      tc_fence_before();
      // the partner's rows of this CTA's P half
      if (warp == 0) ok = ok && wait_bar(ctx, &bars->p_rx, i & 1);
      __syncwarp();
      if (lane == 0) mbar_arrive_remote(lead(&bars->p_ready));
      return !softmax_any(!ok);
    };

    // ---- end of a piece (step i was its last): row sums of the pair, normalise, write O^T
    auto epilogue = [&](int i, const StepCursor &tc) -> bool {
      bool ok = true;
      if (threadIdx.x == 0) mbar_expect_tx(&bars->lx, 2 * 64 * 4);
      reinterpret_cast<float2 *>(red + (g * 4 + quad) * 64)[lane] = make_float2(l0, l1);
      half_sync(g);
      float s0 = 0.f, s1 = 0.f;
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const float2 x = reinterpret_cast<const float2 *>(red + (g * 4 + q) * 64)[lane];
        s0 += x.x;
        s1 += x.y;
      }
      if (quad == 0)
        st_async_v2(mapa(smem_u32(lx + 64 * g + 2 * lane), peer), s0, s1,
                    mapa(smem_u32(&bars->lx), peer));
      ok = ok && wait_bar(ctx, &bars->lx, tc.nseg & 1);
      const float2 px = reinterpret_cast<const float2 *>(lx + 64 * g)[lane];
      const float f0 = s0 + px.x, f1 = s1 + px.y;   // same sum in both CTAs
      // one division per head: z is O^T times the reciprocal of its row sum
      // (a division per output value kept the softmax warps 4 us longer per call)
      if (quad == 0) reinterpret_cast<float2 *>(linv + 64 * g)[lane] = make_float2(1.f / f0, 1.f / f1);
      const int b = tc.seg.b;
      const int pbase = a.part_base[b];
      const bool whole = pbase < 0;
      const int slot_p = whole ? 0 : pbase + (part - tc.seg.s0 / hdr.quota);
      // a whole sequence writes z (normalised), or, when the caller asked for the
      // partial softmax, its unnormalised (O, m, l); a piece of a split sequence
      // writes its partial into the workspace slot the merge reads
      const bool to_z = whole && !a.pout_O;
      float *pm = whole ? a.pout_m + (long)b * kHeads : a.part_m + (long)slot_p * kHeads;
      float *pl = whole ? a.pout_l + (long)b * kHeads : a.part_l + (long)slot_p * kHeads;
      float *pO = whole ? a.pout_O + (long)b * kHeads * kDc : a.part_O + (long)slot_p * kHeads * kDc;
      if (rank == 0 && quad == 0) {
        const float ln2 = 0.6931471805599453f;
        const int h0 = 64 * g + 2 * lane;
        const long ri = (long)b * kHeads + h0;
        if (to_z) {
          if (a.lse) {
            a.lse[ri] = (m0 + __log2f(f0)) * ln2;
            a.lse[ri + 1] = (m1 + __log2f(f1)) * ln2;
          }
        } else {
          pm[h0] = m0 * ln2;
          pm[h0 + 1] = m1 * ln2;
          pl[h0] = f0;
          pl[h0 + 1] = f1;
        }
      }
      ok = ok && wait_bar(ctx, &bars->pv_done, i & 1);
      softmax_sync();                        // 1 / l complete for both halves
      tc_fence_after();
      const int col = 256 * g + 128 * (int)rank + quad * 32 + lane;   // latent column of my lane
      const uint32_t ob = tmem + lane_off + kTmemO + 128 * g;
      for (int c = 0; c < 128; c += 32) {
        float ov[32];
        tmem_ld32f(ob + c, ov);
        tmem_wait_ld();
        if (to_z) {
          __nv_bfloat16 *z = reinterpret_cast<__nv_bfloat16 *>(a.z) + (long)b * kHeads * kDc + col;
#pragma unroll
          for (int kk = 0; kk < 32; ++kk)
            z[(long)(c + kk) * kDc] = __float2bfloat16_rn(ov[kk] * linv[c + kk]);
        } else {
          float *o = pO + col;
#pragma unroll
          for (int kk = 0; kk < 32; ++kk) o[(long)(c + kk) * kDc] = ov[kk];
        }
      }
      tc_fence_before();
      return !softmax_any(!ok);
    };

    for (int step = 0; cur.valid; cur.advance(a), ++step) {
      if (!produce(step, cur)) break;
      if (cur.last() && !epilogue(step, cur)) break;
    }
  }

  // the warps whose lane 0 alone ran a loop meet again before the CTA barrier
  // (__syncthreads is warp-aligned: a warp must reach it converged)
  __syncwarp();
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

// 2-D byte map over int8 rows (656 bytes each); box = box_bytes x box_rows.
bool make_map_i8(CUtensorMap *m, const void *base, long rows, int box_bytes, int box_rows,
                 CUtensorMapSwizzle sw) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) return false;
  const cuuint64_t dims[2] = {(cuuint64_t)kI8Row, (cuuint64_t)rows};
  const cuuint64_t strides[1] = {(cuuint64_t)kI8Row};
  const cuuint32_t box[2] = {(cuuint32_t)box_bytes, (cuuint32_t)box_rows};
  const cuuint32_t estr[2] = {1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void *>(base), dims, strides, box,
             estr, CU_TENSOR_MAP_INTERLEAVE_NONE, sw, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <bool kI8>
cudaError_t launch_attn_t(const AttnArgs &a, int parts, cudaStream_t s) {
  static api::PerDeviceOnce smem_attr;
  cudaError_t e = smem_attr.run([] {
    return cudaFuncSetAttribute(attn_sm100_kernel<kI8>,
                                cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
  });
  if (e != cudaSuccess) return e;
  CUtensorMap tm_rows, tm_q, tm_i8k, tm_i8v;
  const long pool_rows = (long)a.num_pages * kPage;
  const long q_rows = (long)a.batch * kHeads;
  if (!make_map(&tm_q, a.q_lat, q_rows, 64, 64, CU_TENSOR_MAP_SWIZZLE_128B))
    return cudaErrorInvalidValue;
  if (kI8) {
    // k_R (bytes 512..639) as swizzled bf16 boxes; the codes in plain boxes that
    // the kernel converts
    if (!make_map_i8(&tm_rows, a.pool, pool_rows, 128, kPage, CU_TENSOR_MAP_SWIZZLE_128B) ||
        !make_map_i8(&tm_i8k, a.pool, pool_rows, 64, kPage, CU_TENSOR_MAP_SWIZZLE_64B) ||
        !make_map_i8(&tm_i8v, a.pool, pool_rows, 128, kPage, CU_TENSOR_MAP_SWIZZLE_128B))
      return cudaErrorInvalidValue;
  } else {
    if (!make_map(&tm_rows, a.pool, pool_rows, 64, kPage, CU_TENSOR_MAP_SWIZZLE_128B))
      return cudaErrorInvalidValue;
    tm_i8k = tm_rows;
    tm_i8v = tm_rows;
  }
  const float scale_log2 = a.scale * 1.4426950408889634f;
  return launch_pdl(attn_sm100_kernel<kI8>, dim3(2 * parts), dim3(kThreads), kSmemBytes, s,
                    tm_rows, tm_q, tm_i8k, tm_i8v, a, scale_log2);
}

}  // namespace

cudaError_t launch_attn(const AttnArgs &a, int parts, cudaStream_t s) {
  return a.int8_rows ? launch_attn_t<true>(a, parts, s) : launch_attn_t<false>(a, parts, s);
}

}  // namespace sm100
}  // namespace mla
