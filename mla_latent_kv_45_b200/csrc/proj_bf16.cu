// bf16 projections of the decode step (DeepSeek-V2 sizes) on the tensor-core
// skinny GEMM.  Intermediates (c_Q, q_C, o) are stored in bf16, as a bf16
// model stores activations; q_R leaves the GEMM in fp32 for the RoPE kernel.
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
  o.part = nullptr;
}

void partial(GemmOp &o, float *part, int part_ld, int part_col, int splits) {
  o.part = part;
  o.part_ld = part_ld;
  o.part_col = part_col;
  o.splits = splits;
}

int splits_for(int m_rows_total, int k) { return gemm_splits((m_rows_total + 127) / 128, 1, k / 64); }

}  // namespace

size_t gemm_workspace_bytes(int batch, int d_model, int d_q, int n_heads, const mla_dims &d) {
  if (d.dtype != MLA_BF16) return 0;
  size_t need = 0;
  auto upd = [&](int splits, int width) {
    if (splits > 1) {
      const size_t b = sizeof(float) * (size_t)splits * batch * width;
      if (b > need) need = b;
    }
  };
  upd(gemm_splits(5, 1, d_model / 64), 576);                       // W_DKV + W_KR
  if (d_q > 0) upd(splits_for(d_q, d_model), d_q);                  // W_DQ
  const int kq = d_q > 0 ? d_q : d_model;
  upd(gemm_splits(n_heads + n_heads / 2, 1, kq / 64), n_heads * 192);  // W_UQ + W_QR
  upd(splits_for(d_model, n_heads * 128), d_model);                 // W_O
  return need;
}

cudaError_t append_proj(const bf16 *h, const bf16 *W_DKV, const bf16 *W_KR, int batch,
                        int d_model, float *xkv, void *gemm_ws, int *err, const float **out,
                        int *splits_out, cudaStream_t s) {
  const int splits = gemm_splits(5, 1, d_model / 64);
  GemmOp ops[2] = {op(W_DKV, 512, 1, 0), op(W_KR, 64, 1, 0)};
  *splits_out = splits;
  if (splits == 1) {
    direct(ops[0], kOutF32, xkv, 576);
    direct(ops[1], kOutF32, xkv + 512, 576);
    *out = xkv;
    return gemm(ops, 2, h, batch, d_model, d_model, 0, err, s);
  }
  // the partial sums are added by the append epilogue kernel
  float *part = static_cast<float *>(gemm_ws);
  partial(ops[0], part, 576, 0, splits);
  partial(ops[1], part, 576, 512, splits);
  *out = part;
  return gemm(ops, 2, h, batch, d_model, d_model, 0, err, s);
}

cudaError_t absorb_proj(const bf16 *x, const bf16 *W_DQ, const bf16 *W_UQ, const bf16 *W_QR,
                        const bf16 *W_UK, int batch, int d_in, int d_q, bf16 *cq, bf16 *qc,
                        float *qr, bf16 *q_lat, void *gemm_ws, int *err, cudaStream_t s) {
  float *part = static_cast<float *>(gemm_ws);
  const bf16 *xin = x;
  if (W_DQ) {
    // c_Q = W_DQ h
    GemmOp o = op(W_DQ, d_q, 1, 0);
    const int sp = splits_for(d_q, d_in);
    if (sp == 1) {
      direct(o, kOutBf16, cq, d_q);
      TRY(gemm(&o, 1, x, batch, d_in, d_in, 0, err, s));
    } else {
      partial(o, part, d_q, 0, sp);
      TRY(gemm(&o, 1, x, batch, d_in, d_in, 0, err, s));
      TRY(gemm_reduce(part, sp, batch, d_q, d_q, cq, d_q, true, s));
    }
    xin = cq;
  }
  // q_C = W_UQ c_Q (bf16) and raw q_R = W_QR c_Q (fp32), sharing c_Q
  {
    GemmOp ops[2] = {op(W_UQ, kH * 128, 1, 0), op(W_QR, kH * 64, 1, 0)};
    const int sp = gemm_splits(kH + kH / 2, 1, d_q / 64);
    if (sp == 1) {
      direct(ops[0], kOutBf16, qc, kH * 128);
      direct(ops[1], kOutF32, qr, kH * 64);
      TRY(gemm(ops, 2, xin, batch, d_q, d_q, 0, err, s));
    } else {
      partial(ops[0], part, kH * 192, 0, sp);
      partial(ops[1], part, kH * 192, kH * 128, sp);
      TRY(gemm(ops, 2, xin, batch, d_q, d_q, 0, err, s));
      TRY(gemm_reduce(part, sp, batch, kH * 128, kH * 192, qc, kH * 128, true, s));
      TRY(gemm_reduce(part + kH * 128, sp, batch, kH * 64, kH * 192, qr, kH * 64, false, s));
    }
  }
  // q~_i = W_UK,i^T q_C,i into q_lat[b][i][0:512]: per head, A = W_UK,i read MN-major
  GemmOp o = op(W_UK, 512, kH, 1);
  direct(o, kOutBf16, q_lat, (long)kH * 576, 576);
  return gemm(&o, 1, qc, batch, (long)kH * 128, 128, 128, err, s);
}

cudaError_t unabsorb_proj(const bf16 *z, const bf16 *W_UV, const bf16 *W_O, int batch,
                          int d_model, bf16 *o, bf16 *out, void *gemm_ws, int *err,
                          cudaStream_t s) {
  // o_i = W_UV,i z_i: per head, K = 512
  GemmOp u = op(W_UV, 128, kH, 0);
  direct(u, kOutBf16, W_O ? o : out, (long)kH * 128, 128);
  TRY(gemm(&u, 1, z, batch, (long)kH * 512, 512, 512, err, s));
  if (!W_O) return cudaSuccess;
  // u = W_O o
  GemmOp w = op(W_O, d_model, 1, 0);
  const int sp = splits_for(d_model, kH * 128);
  if (sp == 1) {
    direct(w, kOutBf16, out, d_model);
    return gemm(&w, 1, o, batch, kH * 128, kH * 128, 0, err, s);
  }
  float *part = static_cast<float *>(gemm_ws);
  partial(w, part, d_model, 0, sp);
  TRY(gemm(&w, 1, o, batch, kH * 128, kH * 128, 0, err, s));
  return gemm_reduce(part, sp, batch, d_model, d_model, out, d_model, true, s);
}

}  // namespace sm100
}  // namespace mla
