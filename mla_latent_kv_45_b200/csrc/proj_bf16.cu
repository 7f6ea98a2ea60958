// bf16 projections of the decode step (DeepSeek-V2 sizes) on the tensor-core
// skinny GEMM and the fused per-head absorption kernel.  Intermediates (c_Q,
// q_C, o) are stored in bf16, as a bf16 model stores activations; q_R stays
// fp32 until it is rotated and rounded once into q_lat.
#include "gemm_sm100.h"
#include "sm100.h"

namespace mla {
namespace sm100 {

using bf16 = __nv_bfloat16;

namespace {

constexpr int kH = 128;

#define TRY(x)                        \
  do {                                \
    cudaError_t e_ = (x);             \
    if (e_ != cudaSuccess) return e_; \
  } while (0)

GemmOp op(const bf16 *A, int M, int heads, int a_mn) {
  GemmOp o{};
  o.A = A;
  o.M = M;
  o.heads = heads;
  o.a_mn = a_mn;
  o.splits = 1;
  return o;
}

void direct(GemmOp &o, int mode, void *out, long ldy, long y_head = 0) {
  o.out_mode = mode;
  o.out = out;
  o.ldy = ldy;
  o.y_head = y_head;
}

// the K range cut into `splits` CTAs that sum their partial tiles in-cluster
void cluster_split(GemmOp &o, int splits) { o.splits = splits; }

}  // namespace

cudaError_t append_proj(const bf16 *h, const bf16 *W_DKV, const bf16 *W_KR, int batch,
                        int d_model, float *xkv, int *err, cudaStream_t s) {
  // [W_DKV h ; W_KR h] in fp32, its K splits summed in-cluster
  const int splits = gemm_cluster_splits(5, 1, d_model / 64, batch);
  GemmOp ops[2] = {op(W_DKV, 512, 1, 0), op(W_KR, 64, 1, 0)};
  direct(ops[0], kOutF32, xkv, 576);
  direct(ops[1], kOutF32, xkv + 512, 576);
  cluster_split(ops[0], splits);
  cluster_split(ops[1], splits);
  return gemm(ops, 2, h, batch, d_model, d_model, 0, err, s);
}

cudaError_t absorb_proj(const bf16 *x, const bf16 *W_DQ, const bf16 *W_UQ, const bf16 *W_QR,
                        const bf16 *W_UK, int batch, int d_in, int d_q, const RopeParams &rp,
                        const int32_t *positions, bf16 *cq, bf16 *q_lat, int *err,
                        cudaStream_t s) {
  const bf16 *xin = x;
  if (W_DQ) {
    // c_Q = W_DQ h, its K splits summed in-cluster
    GemmOp o = op(W_DQ, d_q, 1, 0);
    direct(o, kOutBf16, cq, d_q);
    cluster_split(o, gemm_cluster_splits((d_q + 127) / 128, 1, d_in / 64, batch));
    TRY(gemm(&o, 1, x, batch, d_in, d_in, 0, err, s));
    xin = cq;
  }
  // per head: q_C,i = W_UQ,i c_Q, q_R,i = RoPE(W_QR,i c_Q), q~_i = W_UK,i^T q_C,i
  return absorb_heads(xin, W_DQ ? d_q : d_in, W_UQ, W_QR, W_UK, batch, rp, positions, q_lat, err,
                      s);
}

cudaError_t unabsorb_proj(const bf16 *z, const bf16 *W_UV, const bf16 *W_O, int batch,
                          int d_model, bf16 *o, bf16 *out, int *err, cudaStream_t s) {
  // o_i = W_UV,i z_i: per head, K = 512 (split in-cluster: one 128-row tile per
  // head leaves each CTA a short serial chain otherwise)
  GemmOp u = op(W_UV, 128, kH, 0);
  direct(u, kOutBf16, W_O ? o : out, (long)kH * 128, 128);
  cluster_split(u, gemm_cluster_splits(1, kH, 512 / 64, batch));
  TRY(gemm(&u, 1, z, batch, (long)kH * 512, 512, 512, err, s));
  if (!W_O) return cudaSuccess;
  // u = W_O o, its K splits summed in-cluster
  GemmOp w = op(W_O, d_model, 1, 0);
  direct(w, kOutBf16, out, d_model);
  cluster_split(w, gemm_cluster_splits((d_model + 127) / 128, 1, kH * 128 / 64, batch));
  return gemm(&w, 1, o, batch, kH * 128, kH * 128, 0, err, s);
}

}  // namespace sm100
}  // namespace mla
