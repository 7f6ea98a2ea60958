// bf16 DeepSeek-V2-shaped path (n_heads 128, d_c 512, d_rope 64, d_nope = d_v
// = 128, 64-row pages): projections and latent attention on sm_100a.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stddef.h>

#include "mla.h"
#include "kernels.h"

namespace mla {
namespace sm100 {

// Fewest cache pages an attention partition is given (a partition that holds
// less work than this is merged away by the plan).
constexpr int kAttnMinPages = 4;

// Virtual pages the plan charges each sequence for its fixed cost in the
// attention kernel (loading its q_lat, draining the pipeline at its end and
// writing its output).  Measured on B200 over the 74 partitions of a batch of
// 64 sequences (1024..8192 rows): a partition takes about 4.4 us per step of 4
// pages plus 5.5 us per sequence piece, so a piece costs about 5 pages.
constexpr int kAttnSeqGap = 5;

// [W_DKV h_b ; W_KR h_b] in fp32 into xkv [batch][576].
cudaError_t append_proj(const __nv_bfloat16 *h, const __nv_bfloat16 *W_DKV,
                        const __nv_bfloat16 *W_KR, int batch, int d_model, float *xkv, int *err,
                        cudaStream_t s);

// q_lat[b][i] = [W_UK,i^T q_C,i ; RoPE_pos(q_R,i)] (bf16), with c_Q = W_DQ x
// (bf16, in cq) when W_DQ is given, else c_Q = x.
cudaError_t absorb_proj(const __nv_bfloat16 *x, const __nv_bfloat16 *W_DQ,
                        const __nv_bfloat16 *W_UQ, const __nv_bfloat16 *W_QR,
                        const __nv_bfloat16 *W_UK, int batch, int d_in, int d_q,
                        const RopeParams &rp, const int32_t *positions, __nv_bfloat16 *cq,
                        __nv_bfloat16 *q_lat, int *err, cudaStream_t s);

// The per-head part of absorb_proj in one launch (one CTA per head): q_C,i =
// W_UQ,i x (rounded to bf16), q_R,i = W_QR,i x rotated by positions[b], and
// q~_i = W_UK,i^T q_C,i, written into q_lat.  x: [batch][K] bf16.
cudaError_t absorb_heads(const __nv_bfloat16 *x, int K, const __nv_bfloat16 *W_UQ,
                         const __nv_bfloat16 *W_QR, const __nv_bfloat16 *W_UK, int batch,
                         const RopeParams &rp, const int32_t *positions, __nv_bfloat16 *q_lat,
                         int *err, cudaStream_t s);

// o[b][i] = W_UV,i z[b][i] (bf16); out = W_O o when W_O is given, else out = o.
cudaError_t unabsorb_proj(const __nv_bfloat16 *z, const __nv_bfloat16 *W_UV,
                          const __nv_bfloat16 *W_O, int batch, int d_model, __nv_bfloat16 *o,
                          __nv_bfloat16 *out, int *err, cudaStream_t s);

// Test hook: when limit_ns > 0, later absorb_heads launches bound every wait
// by limit_ns instead of the default, and with skip_arrive one epilogue warp
// withholds its arrive on the q_C-ready barrier (so that wait runs out).
void absorb_debug_fault(int skip_arrive, uint64_t limit_ns);

// Latent attention over the plan's partitions (partials / z / lse).
cudaError_t launch_attn(const AttnArgs &a, int parts, cudaStream_t s);

}  // namespace sm100
}  // namespace mla
