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

// Workspace bytes the projections need beyond the fp32 intermediates.
size_t gemm_workspace_bytes(int batch, int d_model, int d_q, int n_heads, const mla_dims &d);

// [W_DKV h_b ; W_KR h_b] in fp32 as `*splits` partial sums [splits][batch][576]
// at *out (xkv itself when there is one split, else the GEMM workspace).
cudaError_t append_proj(const __nv_bfloat16 *h, const __nv_bfloat16 *W_DKV,
                        const __nv_bfloat16 *W_KR, int batch, int d_model, float *xkv,
                        void *gemm_ws, int *err, const float **out, int *splits,
                        cudaStream_t s);

// c_Q (bf16, when W_DQ), q_C (bf16), raw q_R (fp32, not yet rotated) and the
// absorbed content half q_lat[b][i][0:512] = W_UK,i^T q_C,i (bf16).
cudaError_t absorb_proj(const __nv_bfloat16 *x, const __nv_bfloat16 *W_DQ,
                        const __nv_bfloat16 *W_UQ, const __nv_bfloat16 *W_QR,
                        const __nv_bfloat16 *W_UK, int batch, int d_in, int d_q,
                        __nv_bfloat16 *cq, __nv_bfloat16 *qc, float *qr, __nv_bfloat16 *q_lat,
                        void *gemm_ws, int *err, cudaStream_t s);

// o[b][i] = W_UV,i z[b][i] (bf16); out = W_O o when W_O is given, else out = o.
cudaError_t unabsorb_proj(const __nv_bfloat16 *z, const __nv_bfloat16 *W_UV,
                          const __nv_bfloat16 *W_O, int batch, int d_model, __nv_bfloat16 *o,
                          __nv_bfloat16 *out, void *gemm_ws, int *err, cudaStream_t s);

// Latent attention over the plan's partitions (partials / z / lse).
cudaError_t launch_attn(const AttnArgs &a, int parts, cudaStream_t s);

}  // namespace sm100
}  // namespace mla
