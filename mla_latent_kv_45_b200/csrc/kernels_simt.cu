// Generic CUDA-core kernels of the MLA decode step.
//
// These kernels accept any small head / latent sizes.  In fp32 they are the
// validation path (every step computed in fp32, one rounding per stored
// value).  The plan and combine kernels are shared with the sm_100a
// tensor-core attention kernel.
#include "common.cuh"
#include "kernels.h"

namespace mla {

// ---------------------------------------------------------------------------
// Skinny matrix products  Y[b][m] = sum_k W[m][k] X[b][k]   (per head z)
// ---------------------------------------------------------------------------

// W contiguous along k: one warp per output row m, lanes stride over k, eight
// batch rows at a time.
template <class TW, class TX, class TY>
__global__ void gemv_k_contig(GemvArgs a) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int m = blockIdx.x * (blockDim.x >> 5) + warp;
  const int head = blockIdx.z;
  if (m >= a.M) return;
  const TW *w = reinterpret_cast<const TW *>(a.W) + head * a.w_head + (long)m * a.w_m;
  const TX *x = reinterpret_cast<const TX *>(a.X) + head * a.x_head;
  TY *y = reinterpret_cast<TY *>(a.Y) + head * a.y_head;
  for (int b0 = blockIdx.y * 8; b0 < a.B; b0 += gridDim.y * 8) {
    float acc[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) acc[j] = 0.f;
    for (int k = lane; k < a.K; k += 32) {
      const float wv = ld_f(w + k);
#pragma unroll
      for (int j = 0; j < 8; ++j)
        if (b0 + j < a.B) acc[j] += wv * ld_f(x + (long)(b0 + j) * a.x_b + k);
    }
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const float v = warp_sum(acc[j]);
      if (lane == 0 && b0 + j < a.B) y[(long)(b0 + j) * a.y_b + m] = st_cast<TY>(v);
    }
  }
}

// W contiguous along m (a transposed weight, e.g. W_UK,i^T): one thread per
// output m, the batch rows' x staged in shared memory.
template <class TW, class TX, class TY>
__global__ void gemv_m_contig(GemvArgs a) {
  extern __shared__ float xs[];  // [8][K]
  const int m = blockIdx.x * blockDim.x + threadIdx.x;
  const int head = blockIdx.z;
  const TW *w = reinterpret_cast<const TW *>(a.W) + head * a.w_head;
  const TX *x = reinterpret_cast<const TX *>(a.X) + head * a.x_head;
  TY *y = reinterpret_cast<TY *>(a.Y) + head * a.y_head;
  for (int b0 = blockIdx.y * 8; b0 < a.B; b0 += gridDim.y * 8) {
    __syncthreads();
    for (int i = threadIdx.x; i < 8 * a.K; i += blockDim.x) {
      const int j = i / a.K, k = i % a.K;
      xs[i] = (b0 + j < a.B) ? ld_f(x + (long)(b0 + j) * a.x_b + k) : 0.f;
    }
    __syncthreads();
    if (m < a.M) {
      float acc[8];
#pragma unroll
      for (int j = 0; j < 8; ++j) acc[j] = 0.f;
      for (int k = 0; k < a.K; ++k) {
        const float wv = ld_f(w + (long)k * a.w_k + m);
#pragma unroll
        for (int j = 0; j < 8; ++j) acc[j] += wv * xs[j * a.K + k];
      }
#pragma unroll
      for (int j = 0; j < 8; ++j)
        if (b0 + j < a.B) y[(long)(b0 + j) * a.y_b + m] = st_cast<TY>(acc[j]);
    }
  }
}

template <class TW, class TX, class TY>
cudaError_t launch_gemv(const GemvArgs &a, int heads, cudaStream_t s) {
  const int bgrid = (a.B + 7) / 8 < 64 ? (a.B + 7) / 8 : 64;
  if (a.w_k == 1) {
    dim3 grid((a.M + 7) / 8, bgrid, heads);
    gemv_k_contig<TW, TX, TY><<<grid, 256, 0, s>>>(a);
  } else {
    dim3 grid((a.M + 127) / 128, bgrid, heads);
    gemv_m_contig<TW, TX, TY><<<grid, 128, 8 * a.K * sizeof(float), s>>>(a);
  }
  return cudaGetLastError();
}

#define MLA_INST_GEMV(TW, TX, TY) \
  template cudaError_t launch_gemv<TW, TX, TY>(const GemvArgs &, int, cudaStream_t);
MLA_INST_GEMV(float, float, float)

// ---------------------------------------------------------------------------
// Cache-append epilogue: RMSNorm on c, RoPE on k_R, one rounding, paged write
// ---------------------------------------------------------------------------

template <class T>
__global__ void append_finish(const float *xkv, int splits, int batch, int d_c, RopeParams rp,
                              const T *gamma, float eps, const int32_t *positions, T *pool,
                              int num_pages, int page_size, const int32_t *block_table,
                              int max_pages, int *err) {
  // xkv holds `splits` partial sums [splits][batch][row] of [W_DKV h ; W_KR h]
  extern __shared__ float x[];   // [row]
  grid_dep_wait();
  const int b = blockIdx.x;
  const int row = d_c + rp.d_rope;
  for (int i = threadIdx.x; i < row; i += blockDim.x) {
    float v = 0.f;
    for (int sp = 0; sp < splits; ++sp) v += xkv[((long)sp * batch + b) * row + i];
    x[i] = v;
  }
  __syncthreads();
  __shared__ float red[32];
  __shared__ float inv_rms;
  float ss = 0.f;
  for (int i = threadIdx.x; i < d_c; i += blockDim.x) ss += x[i] * x[i];
  ss = warp_sum(ss);
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = ss;
  __syncthreads();
  if (threadIdx.x < 32) {
    float v = threadIdx.x < (blockDim.x >> 5) ? red[threadIdx.x] : 0.f;
    v = warp_sum(v);
    if (threadIdx.x == 0) inv_rms = 1.0f / sqrtf(v / (float)d_c + eps);
  }
  __syncthreads();
  const int pos = positions[b];
  const long cap = (long)max_pages * page_size;
  int page = -1;
  if (pos >= 0 && pos < cap) page = block_table[(long)b * max_pages + pos / page_size];
  if (page < 0 || page >= num_pages) {
    if (threadIdx.x == 0) set_error(err, kErrRange);
    return;
  }
  T *dst = pool + ((long)page * page_size + pos % page_size) * row;
  for (int i = threadIdx.x; i < d_c; i += blockDim.x)
    dst[i] = st_cast<T>(ld_f(gamma + i) * (x[i] * inv_rms));
  for (int i = threadIdx.x; i < rp.d_rope / 2; i += blockDim.x) {
    int j0, j1;
    rope_idx(rp, i, j0, j1);
    float x0 = x[d_c + j0], x1 = x[d_c + j1];
    rope_pair(rp, i, pos, x0, x1);
    dst[d_c + j0] = st_cast<T>(x0);
    dst[d_c + j1] = st_cast<T>(x1);
  }
}

template <class T>
cudaError_t launch_append_finish(const float *xkv, int splits, int batch, int d_c,
                                 const RopeParams &rp, const T *gamma, float eps,
                                 const int32_t *positions, T *pool, int num_pages, int page_size,
                                 const int32_t *block_table, int max_pages, int *err,
                                 cudaStream_t s) {
  const size_t smem = (d_c + rp.d_rope) * sizeof(float);
  return launch_pdl(append_finish<T>, dim3(batch), dim3(256), smem, s, xkv, splits, batch, d_c, rp,
                    gamma, eps, positions, pool, num_pages, page_size, block_table, max_pages, err);
}
template cudaError_t launch_append_finish<float>(const float *, int, int, int, const RopeParams &,
                                                 const float *, float, const int32_t *, float *,
                                                 int, int, const int32_t *, int, int *,
                                                 cudaStream_t);
template cudaError_t launch_append_finish<__nv_bfloat16>(
    const float *, int, int, int, const RopeParams &, const __nv_bfloat16 *, float,
    const int32_t *, __nv_bfloat16 *, int, int, const int32_t *, int, int *, cudaStream_t);

// Cache append into an int8 row (656 bytes: 512 int8 codes, 64 bf16 k_R, the
// fp32 scale 2^e, zero padding).  c = gamma * x / rms(x) is formed in fp32 as in
// append_finish, then quantised with the row's power-of-two scale: e is the
// smallest integer with max|c| <= 127 * 2^e and q = round-half-even(c / 2^e).
__global__ void append_finish_int8(const float *xkv, int batch, int d_c, RopeParams rp,
                                   const __nv_bfloat16 *gamma, float eps,
                                   const int32_t *positions, uint8_t *pool, int num_pages,
                                   int page_size, const int32_t *block_table, int max_pages,
                                   int *err) {
  extern __shared__ float x[];   // [d_c + d_rope]
  __shared__ float red[32];
  __shared__ float inv_rms, amax_s;
  grid_dep_wait();
  const int b = blockIdx.x;
  const int row = d_c + rp.d_rope;
  for (int i = threadIdx.x; i < row; i += blockDim.x) x[i] = xkv[(long)b * row + i];
  __syncthreads();
  float ss = 0.f;
  for (int i = threadIdx.x; i < d_c; i += blockDim.x) ss += x[i] * x[i];
  ss = warp_sum(ss);
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = ss;
  __syncthreads();
  if (threadIdx.x < 32) {
    float v = threadIdx.x < (blockDim.x >> 5) ? red[threadIdx.x] : 0.f;
    v = warp_sum(v);
    if (threadIdx.x == 0) inv_rms = 1.0f / sqrtf(v / (float)d_c + eps);
  }
  __syncthreads();
  // c in fp32 (kept in place of x), then its largest magnitude
  float am = 0.f;
  for (int i = threadIdx.x; i < d_c; i += blockDim.x) {
    const float c = __bfloat162float(gamma[i]) * (x[i] * inv_rms);
    x[i] = c;
    am = fmaxf(am, fabsf(c));
  }
  am = warp_max(am);
  __syncthreads();
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = am;
  __syncthreads();
  if (threadIdx.x < 32) {
    float v = threadIdx.x < (blockDim.x >> 5) ? red[threadIdx.x] : 0.f;
    v = warp_max(v);
    if (threadIdx.x == 0) amax_s = v;
  }
  __syncthreads();
  const float amax = amax_s;
  // amax in [2^k, 2^(k+1)): 127 * 2^(k-6) = 1.98 * 2^k, so e is k - 6 or k - 5
  int e = 0;
  if (amax > 0.f) {
    e = ilogbf(amax) - 6;
    if (amax > ldexpf(127.f, e)) ++e;
  }
  const float inv_s = ldexpf(1.f, -e);
  const int pos = positions[b];
  const long cap = (long)max_pages * page_size;
  int page = -1;
  if (pos >= 0 && pos < cap) page = block_table[(long)b * max_pages + pos / page_size];
  if (page < 0 || page >= num_pages) {
    if (threadIdx.x == 0) set_error(err, kErrRange);
    return;
  }
  uint8_t *dst = pool + ((long)page * page_size + pos % page_size) * 656;
  for (int i = threadIdx.x; i < d_c; i += blockDim.x) {
    const int q = max(-127, min(127, __float2int_rn(x[i] * inv_s)));
    dst[i] = static_cast<uint8_t>(static_cast<int8_t>(q));
  }
  __nv_bfloat16 *kr = reinterpret_cast<__nv_bfloat16 *>(dst + d_c);
  for (int i = threadIdx.x; i < rp.d_rope / 2; i += blockDim.x) {
    int j0, j1;
    rope_idx(rp, i, j0, j1);
    float x0 = x[d_c + j0], x1 = x[d_c + j1];
    rope_pair(rp, i, pos, x0, x1);
    kr[j0] = __float2bfloat16_rn(x0);
    kr[j1] = __float2bfloat16_rn(x1);
  }
  if (threadIdx.x < 4) {
    uint32_t *tail = reinterpret_cast<uint32_t *>(dst + d_c + 2 * rp.d_rope);   // bytes 640..655
    tail[threadIdx.x] = threadIdx.x == 0 ? __float_as_uint(ldexpf(1.f, e)) : 0u;
  }
}

cudaError_t launch_append_finish_int8(const float *xkv, int batch, int d_c, const RopeParams &rp,
                                      const __nv_bfloat16 *gamma, float eps,
                                      const int32_t *positions, uint8_t *pool, int num_pages,
                                      int page_size, const int32_t *block_table, int max_pages,
                                      int *err, cudaStream_t s) {
  const size_t smem = (d_c + rp.d_rope) * sizeof(float);
  return launch_pdl(append_finish_int8, dim3(batch), dim3(256), smem, s, xkv, batch, d_c, rp,
                    gamma, eps, positions, pool, num_pages, page_size, block_table, max_pages, err);
}

// ---------------------------------------------------------------------------
// q_R = RoPE_pos(W_QR c_Q) written into the tail of each q_lat row
// ---------------------------------------------------------------------------

template <class T>
__global__ void rope_q(const float *qr, int n_heads, int d_c, RopeParams rp,
                       const int32_t *positions, T *q_lat) {
  // the rotation angles pos * theta_i are the same for every head of a sequence
  __shared__ float cs[64], sn[64];
  grid_dep_wait();
  const int b = blockIdx.x;
  const int half = rp.d_rope / 2;
  const int pos = positions[b];
  for (int i = threadIdx.x; i < half; i += blockDim.x) rope_cos_sin(pos, rp.theta[i], cs[i], sn[i]);
  __syncthreads();
  // 8 pairs per thread per round, loads first, so a round costs one memory latency
  constexpr int kUnroll = 8;
  const int total = n_heads * half;
  for (int base = threadIdx.x; base < total; base += blockDim.x * kUnroll) {
    float x0[kUnroll], x1[kUnroll];
#pragma unroll
    for (int k = 0; k < kUnroll; ++k) {
      const int t = base + k * blockDim.x;
      if (t < total) {
        const int h = t / half, i = t % half;
        int j0, j1;
        rope_idx(rp, i, j0, j1);
        const float *src = qr + ((long)b * n_heads + h) * rp.d_rope;
        x0[k] = __ldg(src + j0);
        x1[k] = __ldg(src + j1);
      }
    }
#pragma unroll
    for (int k = 0; k < kUnroll; ++k) {
      const int t = base + k * blockDim.x;
      if (t < total) {
        const int h = t / half, i = t % half;
        int j0, j1;
        rope_idx(rp, i, j0, j1);
        T *dst = q_lat + ((long)b * n_heads + h) * (d_c + rp.d_rope) + d_c;
        dst[j0] = st_cast<T>(x0[k] * cs[i] - x1[k] * sn[i]);
        dst[j1] = st_cast<T>(x0[k] * sn[i] + x1[k] * cs[i]);
      }
    }
  }
}

template <class T>
cudaError_t launch_rope_q(const float *qr, int batch, int n_heads, int d_c, const RopeParams &rp,
                          const int32_t *positions, T *q_lat, cudaStream_t s) {
  return launch_pdl(rope_q<T>, dim3(batch), dim3(256), 0, s, qr, n_heads, d_c, rp, positions, q_lat);
}
template cudaError_t launch_rope_q<float>(const float *, int, int, int, const RopeParams &,
                                          const int32_t *, float *, cudaStream_t);


// ---------------------------------------------------------------------------
// Plan: balanced split of the batch's pages into partitions
// ---------------------------------------------------------------------------
//
// Sequence b holds n_b = ceil(len_b / page_size) pages.  Concatenating all
// sequences' pages, each preceded by `gap` virtual pages that stand for the
// fixed cost of a sequence (its query load and its output), gives V virtual
// pages; partition p takes virtual pages [p*quota, (p+1)*quota), so every
// partition gets about the same cost, not the same number of pages.  A
// sequence cut by a partition boundary is computed in pieces whose
// unnormalised partials are merged by the combine kernel.

__global__ void plan_kernel(PlanArgs a) {
  __shared__ int warp_tot[32];
  __shared__ int carry;
  const int tid = threadIdx.x;
  // The attention kernel may launch once this kernel's predecessor is done, not
  // before: launched earlier, its CTAs (a whole SM's shared memory each) take SMs
  // that the predecessor's own pending CTAs are waiting for.  Measured on the
  // v2_batch64 step issued on one stream: 216 us with the early trigger, 203 us
  // with this order.
  grid_dep_wait();
  grid_dep_launch();
  const long cap = (long)a.max_pages * a.page_size;
  if (tid == 0) carry = 0;
  __syncthreads();
  // pass 1: page counts, validity, exclusive prefix sum -> seq_start (the
  // virtual index of each sequence's first page, after its gap)
  for (int base = 0; base < a.batch; base += blockDim.x) {
    const int b = base + tid;
    int n = 0;
    if (b < a.batch) {
      const int len = a.seq_lens[b];
      const bool ok = len > 0 && len <= cap;
      n = (ok ? (len + a.page_size - 1) / a.page_size : 0) + a.gap;
      a.bad[b] = ok ? 0 : 1;
      // an empty share of a sequence split across devices is not an error
      if (!ok && !(a.allow_empty && len == 0)) set_error(a.err, kErrRange);
    }
    // block-wide inclusive scan of n
    int v = n;
    for (int o = 1; o < 32; o <<= 1) {
      const int t = __shfl_up_sync(0xffffffffu, v, o);
      if ((tid & 31) >= o) v += t;
    }
    if ((tid & 31) == 31) warp_tot[tid >> 5] = v;
    __syncthreads();
    if (tid < 32) {
      int w = tid < (blockDim.x >> 5) ? warp_tot[tid] : 0;
      for (int o = 1; o < 32; o <<= 1) {
        const int t = __shfl_up_sync(0xffffffffu, w, o);
        if (tid >= o) w += t;
      }
      warp_tot[tid] = w;
    }
    __syncthreads();
    const int incl = v + ((tid >> 5) ? warp_tot[(tid >> 5) - 1] : 0) + carry;
    if (b < a.batch) a.seq_start[b] = incl - n + a.gap;
    __syncthreads();
    if (tid == blockDim.x - 1) carry = incl;
    __syncthreads();
  }
  __shared__ int quota;
  if (tid == 0) {
    const int V = carry;                     // virtual pages
    const int N = V - a.batch * a.gap;       // cache pages
    a.seq_start[a.batch] = V + a.gap;
    int parts = 0, q = 1;
    if (N > 0) {
      int p = a.parts_max;
      const int by_min = (N + a.min_pages - 1) / a.min_pages;
      if (p > by_min) p = by_min;
      if (p < 1) p = 1;
      q = (V + p - 1) / p;
      parts = (V + q - 1) / q;
    }
    a.hdr->total_pages = N > 0 ? V : 0;
    a.hdr->quota = q;
    a.hdr->parts = parts;
    a.hdr->gap = a.gap;
    quota = q;
    carry = 0;
  }
  __syncthreads();
  // pass 2: pieces per sequence and partial-slot bases
  for (int base = 0; base < a.batch; base += blockDim.x) {
    const int b = base + tid;
    int pieces = 0;
    if (b < a.batch) {
      const int s0 = a.seq_start[b], s1 = a.seq_start[b + 1] - a.gap;
      if (s1 > s0) pieces = (s1 - 1) / quota - s0 / quota + 1;
    }
    const int n = pieces > 1 ? pieces : 0;
    int v = n;
    for (int o = 1; o < 32; o <<= 1) {
      const int t = __shfl_up_sync(0xffffffffu, v, o);
      if ((tid & 31) >= o) v += t;
    }
    if ((tid & 31) == 31) warp_tot[tid >> 5] = v;
    __syncthreads();
    if (tid < 32) {
      int w = tid < (blockDim.x >> 5) ? warp_tot[tid] : 0;
      for (int o = 1; o < 32; o <<= 1) {
        const int t = __shfl_up_sync(0xffffffffu, w, o);
        if (tid >= o) w += t;
      }
      warp_tot[tid] = w;
    }
    __syncthreads();
    const int incl = v + ((tid >> 5) ? warp_tot[(tid >> 5) - 1] : 0) + carry;
    if (b < a.batch) a.part_base[b] = n ? incl - n : -1;
    __syncthreads();
    if (tid == blockDim.x - 1) carry = incl;
    __syncthreads();
  }
  if (tid == 0) a.hdr->num_partials = carry;
}

cudaError_t launch_plan(const PlanArgs &a, cudaStream_t s) {
  cudaError_t e = launch_pdl(plan_kernel, dim3(1), dim3(1024), 0, s, a);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

// ---------------------------------------------------------------------------
// CUDA-core latent attention (any small sizes): one block per (partition, head)
// ---------------------------------------------------------------------------

template <class T>
__global__ void attn_simt(AttnArgs a) {
  constexpr int NT = 128;
  const int p = blockIdx.x, h = blockIdx.y;
  const PlanHeader hdr = *a.hdr;
  if (p >= hdr.parts) return;
  const int row = a.d_c + a.d_rope;
  extern __shared__ float sm[];
  float *qs = sm;              // [row]
  float *ps = qs + row;        // [NT]
  int *pg = reinterpret_cast<int *>(ps + NT);  // [NT]
  __shared__ float red[NT / 32];
  const T *pool = reinterpret_cast<const T *>(a.pool);
  constexpr int MAXD = 8;  // d_c <= MAXD * NT
  const int g1 = min(hdr.total_pages, (p + 1) * hdr.quota);
  int g0 = p * hdr.quota;
  // first sequence: the last b with seq_start[b] <= g0 (or 0)
  int lo = 0, hi = a.batch;
  while (hi - lo > 1) {
    const int mid = (lo + hi) >> 1;
    if (a.seq_start[mid] <= g0) lo = mid; else hi = mid;
  }
  int b = lo;
  while (g0 < g1 && b < a.batch) {
    const int s0 = a.seq_start[b], s1 = a.seq_start[b + 1] - hdr.gap;
    const int first = max(g0, s0);
    if (first >= g1) break;                 // the range ends before sequence b's pages
    if (s1 <= first) { ++b; continue; }     // sequence b ends before (or has no pages)
    g0 = first;
    const int lp1 = min(g1, s1) - s0;
    const int len = a.seq_lens[b];
    const int r_begin = (g0 - s0) * a.page_size;
    const int r_end = min(lp1 * a.page_size, len);
    const T *q = reinterpret_cast<const T *>(a.q_lat) + ((long)b * a.n_heads + h) * row;
    __syncthreads();
    for (int j = threadIdx.x; j < row; j += NT) qs[j] = ld_f(q + j);
    __syncthreads();
    float m = -INFINITY, l = 0.f, acc[MAXD];
#pragma unroll
    for (int k = 0; k < MAXD; ++k) acc[k] = 0.f;
    for (int r0 = r_begin; r0 < r_end; r0 += NT) {
      const int s = r0 + threadIdx.x;
      float logit = -INFINITY;
      if (s < r_end) {
        int page = a.block_table[(long)b * a.max_pages + s / a.page_size];
        if (page < 0 || page >= a.num_pages) {
          set_error(a.err, kErrRange);
          a.bad[b] = 1;
          page = 0;
        }
        pg[threadIdx.x] = page;
        const T *rp = pool + ((long)page * a.page_size + s % a.page_size) * row;
        float dot = 0.f;
        for (int j = 0; j < row; ++j) dot += qs[j] * ld_f(rp + j);
        logit = dot * a.scale;
      }
      float cm = warp_max(logit);
      if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = cm;
      __syncthreads();
      cm = fmaxf(fmaxf(red[0], red[1]), fmaxf(red[2], red[3]));
      __syncthreads();
      const float m_new = fmaxf(m, cm);
      const float alpha = expf(m - m_new);
      const float pv = (s < r_end) ? expf(logit - m_new) : 0.f;
      ps[threadIdx.x] = pv;
      float cs = warp_sum(pv);
      if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = cs;
      __syncthreads();
      cs = red[0] + red[1] + red[2] + red[3];
      l = l * alpha + cs;
      m = m_new;
      const int n = min(NT, r_end - r0);
#pragma unroll
      for (int k = 0; k < MAXD; ++k) {
        const int d = threadIdx.x + k * NT;
        if (d < a.d_c) {
          float v = acc[k] * alpha;
          for (int t = 0; t < n; ++t) {
            const int st = r0 + t;
            v += ps[t] * ld_f(pool + ((long)pg[t] * a.page_size + st % a.page_size) * row + d);
          }
          acc[k] = v;
        }
      }
      __syncthreads();
    }
    const int pb = a.part_base[b];
    if (pb < 0 && a.pout_O) {
      float *O = a.pout_O + ((long)b * a.n_heads + h) * a.d_c;
#pragma unroll
      for (int k = 0; k < MAXD; ++k) {
        const int d = threadIdx.x + k * NT;
        if (d < a.d_c) O[d] = acc[k];
      }
      if (threadIdx.x == 0) {
        a.pout_m[(long)b * a.n_heads + h] = m;
        a.pout_l[(long)b * a.n_heads + h] = l;
      }
    } else if (pb < 0) {
      T *z = reinterpret_cast<T *>(a.z) + ((long)b * a.n_heads + h) * a.d_c;
      const float inv = 1.f / l;
#pragma unroll
      for (int k = 0; k < MAXD; ++k) {
        const int d = threadIdx.x + k * NT;
        if (d < a.d_c) z[d] = st_cast<T>(acc[k] * inv);
      }
      if (a.lse && threadIdx.x == 0) a.lse[(long)b * a.n_heads + h] = m + logf(l);
    } else {
      const int slot = pb + (p - s0 / hdr.quota);
      float *O = a.part_O + ((long)slot * a.n_heads + h) * a.d_c;
#pragma unroll
      for (int k = 0; k < MAXD; ++k) {
        const int d = threadIdx.x + k * NT;
        if (d < a.d_c) O[d] = acc[k];
      }
      if (threadIdx.x == 0) {
        a.part_m[(long)slot * a.n_heads + h] = m;
        a.part_l[(long)slot * a.n_heads + h] = l;
      }
    }
    g0 = s0 + lp1;
    ++b;
  }
}

template <class T>
cudaError_t launch_attn_simt(const AttnArgs &a, int parts_max, cudaStream_t s) {
  const size_t smem = (a.d_c + a.d_rope + 128) * sizeof(float) + 128 * sizeof(int);
  dim3 grid(parts_max, a.n_heads);
  attn_simt<T><<<grid, 128, smem, s>>>(a);
  return cudaGetLastError();
}
template cudaError_t launch_attn_simt<float>(const AttnArgs &, int, cudaStream_t);

// ---------------------------------------------------------------------------
// Combine split partials; zero the outputs of invalid sequences
// ---------------------------------------------------------------------------
//
// z = sum_j w_j O_j / sum_j w_j l_j with w_j = exp(m_j - max_j m_j), and
// lse = max_j m_j + log(sum_j w_j l_j): the standard merge of partial softmaxes.

constexpr int kCombineWarps = 8;   // (sequence, head) rows per 256-thread block
constexpr int kCombinePieces = 4;  // pieces whose loads are in flight together
constexpr int kCombineVecs = 4;    // float4 columns per lane per pass

template <class T> struct Vec4Out;
template <> struct Vec4Out<float> {
  static __device__ __forceinline__ void store(float *p, float4 v) {
    *reinterpret_cast<float4 *>(p) = v;
  }
};
template <> struct Vec4Out<__nv_bfloat16> {
  static __device__ __forceinline__ void store(__nv_bfloat16 *p, float4 v) {
    __nv_bfloat162 a = __floats2bfloat162_rn(v.x, v.y), b = __floats2bfloat162_rn(v.z, v.w);
    uint2 u;
    u.x = *reinterpret_cast<uint32_t *>(&a);
    u.y = *reinterpret_cast<uint32_t *>(&b);
    *reinterpret_cast<uint2 *>(p) = u;
  }
};

// One warp per (sequence, head) row: the lanes reduce the pieces' maxima and
// weighted row sums with shuffles, then merge the row's columns (4 float4 per
// lane per pass), with the loads of kCombinePieces pieces in flight together.
// Pieces are summed in increasing order.
template <class T>
__global__ void combine_kernel(AttnArgs a) {
  grid_dep_wait();
  const int row = blockIdx.x * kCombineWarps + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (row >= a.batch * a.n_heads) return;
  const int b = row / a.n_heads, h = row % a.n_heads;
  T *zr = reinterpret_cast<T *>(a.z) + (long)row * a.d_c;
  float *por = a.pout_O ? a.pout_O + (long)row * a.d_c : nullptr;
  if (a.bad[b]) {
    // no rows (an error, or an empty share): z = 0, lse = -inf; as a partial,
    // O = 0, m = -inf, l = 0 (it then carries no weight in a merge)
    if (por) {
      for (int d = lane; d < a.d_c; d += 32) por[d] = 0.f;
      if (lane == 0) {
        a.pout_m[row] = -INFINITY;
        a.pout_l[row] = 0.f;
      }
      return;
    }
    for (int d = lane; d < a.d_c; d += 32) zr[d] = st_cast<T>(0.f);
    if (a.lse && lane == 0) a.lse[row] = -INFINITY;
    return;
  }
  const int pb = a.part_base[b];
  if (pb < 0) return;
  const PlanHeader hdr = *a.hdr;
  const int s0 = a.seq_start[b], s1 = a.seq_start[b + 1] - hdr.gap;
  const int pieces = (s1 - 1) / hdr.quota - s0 / hdr.quota + 1;
  const float *pm = a.part_m + (long)pb * a.n_heads + h;   // piece j at pm[j * n_heads]
  const float *pl = a.part_l + (long)pb * a.n_heads + h;
  // w_j = exp(m_j - M) / sum_j exp(m_j - M) l_j, lse = M + log(sum)
  float M = -INFINITY;
  for (int j = lane; j < pieces; j += 32) M = fmaxf(M, __ldcg(pm + (long)j * a.n_heads));
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));
  float den = 0.f;
  for (int j = lane; j < pieces; j += 32)
    den += expf(__ldcg(pm + (long)j * a.n_heads) - M) * __ldcg(pl + (long)j * a.n_heads);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) den += __shfl_xor_sync(0xffffffffu, den, o);
  // as a partial: O = sum_j e^(m_j - M) O_j, m = M, l = den (not normalised)
  const float inv = por ? 1.f : 1.f / den;
  if (por && lane == 0) {
    a.pout_m[row] = M;
    a.pout_l[row] = den;
  }
  if (!por && a.lse && lane == 0) a.lse[row] = M + logf(den);
  const int nvec = a.d_c / 4;
  const float4 *src = reinterpret_cast<const float4 *>(a.part_O + ((long)pb * a.n_heads + h) * a.d_c);
  const long piece_stride = (long)a.n_heads * nvec;   // float4 per piece
  for (int v0 = 0; v0 < nvec; v0 += 32 * kCombineVecs) {
    float4 acc[kCombineVecs];
#pragma unroll
    for (int q = 0; q < kCombineVecs; ++q) acc[q] = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int j0 = 0; j0 < pieces; j0 += kCombinePieces) {
      float4 v[kCombinePieces][kCombineVecs];
      float w[kCombinePieces];
#pragma unroll
      for (int jj = 0; jj < kCombinePieces; ++jj) {
        const int j = j0 + jj;
        w[jj] = j < pieces ? expf(__ldcg(pm + (long)j * a.n_heads) - M) * inv : 0.f;
#pragma unroll
        for (int q = 0; q < kCombineVecs; ++q) {
          const int vi = v0 + lane + 32 * q;
          v[jj][q] = (j < pieces && vi < nvec) ? __ldcg(src + j * piece_stride + vi)
                                                : make_float4(0.f, 0.f, 0.f, 0.f);
        }
      }
#pragma unroll
      for (int jj = 0; jj < kCombinePieces; ++jj)
#pragma unroll
        for (int q = 0; q < kCombineVecs; ++q) {
          acc[q].x = fmaf(w[jj], v[jj][q].x, acc[q].x);
          acc[q].y = fmaf(w[jj], v[jj][q].y, acc[q].y);
          acc[q].z = fmaf(w[jj], v[jj][q].z, acc[q].z);
          acc[q].w = fmaf(w[jj], v[jj][q].w, acc[q].w);
        }
    }
#pragma unroll
    for (int q = 0; q < kCombineVecs; ++q) {
      const int vi = v0 + lane + 32 * q;
      if (vi >= nvec) continue;
      if (por)
        *reinterpret_cast<float4 *>(por + 4 * vi) = acc[q];
      else
        Vec4Out<T>::store(zr + 4 * vi, acc[q]);
    }
  }
}

template <class T>
cudaError_t launch_combine(const AttnArgs &a, cudaStream_t s) {
  const int rows = a.batch * a.n_heads;
  const dim3 grid((rows + kCombineWarps - 1) / kCombineWarps);
  cudaError_t e = launch_pdl(combine_kernel<T>, grid, dim3(32 * kCombineWarps), 0, s, a);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}
template cudaError_t launch_combine<float>(const AttnArgs &, cudaStream_t);
template cudaError_t launch_combine<__nv_bfloat16>(const AttnArgs &, cudaStream_t);

// Merge of n partial softmaxes [n][batch][n_heads](*d_c): one warp per
// (sequence, head) row, parts summed in increasing order.
template <class T>
__global__ void merge_partials_kernel(const float *O, const float *m, const float *l, int n_parts,
                                      int rows, int d_c, T *z, float *lse) {
  grid_dep_wait();
  grid_dep_launch();
  const int row = blockIdx.x * kCombineWarps + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (row >= rows) return;
  float M = -INFINITY;
  for (int j = lane; j < n_parts; j += 32) M = fmaxf(M, m[(long)j * rows + row]);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));
  T *zr = z + (long)row * d_c;
  if (M == -INFINITY) {   // every part empty
    for (int d = lane; d < d_c; d += 32) zr[d] = st_cast<T>(0.f);
    if (lse && lane == 0) lse[row] = -INFINITY;
    return;
  }
  float den = 0.f;
  for (int j = lane; j < n_parts; j += 32)
    den += expf(m[(long)j * rows + row] - M) * l[(long)j * rows + row];
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) den += __shfl_xor_sync(0xffffffffu, den, o);
  if (lse && lane == 0) lse[row] = M + logf(den);
  const float inv = 1.f / den;
  for (int d = lane; d < d_c; d += 32) {
    float acc = 0.f;
    for (int j = 0; j < n_parts; ++j)
      acc = fmaf(expf(m[(long)j * rows + row] - M) * inv, O[((long)j * rows + row) * d_c + d], acc);
    zr[d] = st_cast<T>(acc);
  }
}

template <class T>
cudaError_t launch_merge_partials(const float *O, const float *m, const float *l, int n_parts,
                                  int batch, int n_heads, int d_c, T *z, float *lse,
                                  cudaStream_t s) {
  const int rows = batch * n_heads;
  const dim3 grid((rows + kCombineWarps - 1) / kCombineWarps);
  cudaError_t e = launch_pdl(merge_partials_kernel<T>, grid, dim3(32 * kCombineWarps), 0, s, O, m,
                             l, n_parts, rows, d_c, z, lse);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}
template cudaError_t launch_merge_partials<float>(const float *, const float *, const float *, int,
                                                  int, int, int, float *, float *, cudaStream_t);
template cudaError_t launch_merge_partials<__nv_bfloat16>(const float *, const float *,
                                                          const float *, int, int, int, int,
                                                          __nv_bfloat16 *, float *, cudaStream_t);

}  // namespace mla
