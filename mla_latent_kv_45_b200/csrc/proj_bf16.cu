// bf16 projections of the decode step (DeepSeek-V2 sizes).
#include "sm100.h"

namespace mla {
namespace sm100 {

using bf16 = __nv_bfloat16;

namespace {
template <class TW, class TX, class TY>
cudaError_t gemv(const void *W, long w_head, long w_m, long w_k, const void *X, long x_head,
                 long x_b, void *Y, long y_head, long y_b, int M, int K, int B, int heads,
                 cudaStream_t s) {
  GemvArgs a{W, w_head, w_m, w_k, X, x_head, x_b, Y, y_head, y_b, M, K, B};
  return launch_gemv<TW, TX, TY>(a, heads, s);
}
#define TRY(x)                                \
  do {                                        \
    cudaError_t e_ = (x);                     \
    if (e_ != cudaSuccess) return e_;         \
  } while (0)
}  // namespace

size_t gemm_workspace_bytes(int, int, int, int, const mla_dims &) { return 0; }

cudaError_t append_proj(const bf16 *h, const bf16 *W_DKV, const bf16 *W_KR, int batch,
                        int d_model, float *xkv, void *, cudaStream_t s) {
  TRY((gemv<bf16, bf16, float>(W_DKV, 0, d_model, 1, h, 0, d_model, xkv, 0, 576, 512, d_model,
                               batch, 1, s)));
  return gemv<bf16, bf16, float>(W_KR, 0, d_model, 1, h, 0, d_model, xkv + 512, 0, 576, 64,
                                 d_model, batch, 1, s);
}

cudaError_t absorb_proj(const bf16 *x, const bf16 *W_DQ, const bf16 *W_UQ, const bf16 *W_QR,
                        const bf16 *W_UK, int batch, int d_in, int d_q, float *cq, float *qc,
                        float *qr, bf16 *q_lat, void *, cudaStream_t s) {
  const int H = 128;
  if (W_DQ) {
    TRY((gemv<bf16, bf16, float>(W_DQ, 0, d_in, 1, x, 0, d_in, cq, 0, d_q, d_q, d_in, batch, 1,
                                 s)));
    TRY((gemv<bf16, float, float>(W_UQ, 0, d_q, 1, cq, 0, d_q, qc, 0, H * 128, H * 128, d_q,
                                  batch, 1, s)));
    TRY((gemv<bf16, float, float>(W_QR, 0, d_q, 1, cq, 0, d_q, qr, 0, H * 64, H * 64, d_q, batch,
                                  1, s)));
  } else {
    TRY((gemv<bf16, bf16, float>(W_UQ, 0, d_q, 1, x, 0, d_q, qc, 0, H * 128, H * 128, d_q, batch,
                                 1, s)));
    TRY((gemv<bf16, bf16, float>(W_QR, 0, d_q, 1, x, 0, d_q, qr, 0, H * 64, H * 64, d_q, batch,
                                 1, s)));
  }
  return gemv<bf16, float, bf16>(W_UK, 128L * 512, 1, 512, qc, 128, (long)H * 128, q_lat, 576,
                                 (long)H * 576, 512, 128, batch, H, s);
}

cudaError_t unabsorb_proj(const bf16 *z, const bf16 *W_UV, const bf16 *W_O, int batch,
                          int d_model, float *o, bf16 *out, void *, cudaStream_t s) {
  const int H = 128;
  if (!W_O)
    return gemv<bf16, bf16, bf16>(W_UV, 128L * 512, 512, 1, z, 512, (long)H * 512, out, 128,
                                  (long)H * 128, 128, 512, batch, H, s);
  TRY((gemv<bf16, bf16, float>(W_UV, 128L * 512, 512, 1, z, 512, (long)H * 512, o, 128,
                               (long)H * 128, 128, 512, batch, H, s)));
  return gemv<bf16, float, bf16>(W_O, 0, (long)H * 128, 1, o, 0, (long)H * 128, out, 0, d_model,
                                 d_model, H * 128, batch, 1, s);
}

}  // namespace sm100
}  // namespace mla
