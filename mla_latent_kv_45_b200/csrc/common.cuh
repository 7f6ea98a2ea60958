// Shared device helpers for the MLA decode kernels (sm_100a).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace mla {

// Bits of the workspace error word.
enum : int { kErrRange = 1, kErrTimeout = 2 };

// RoPE frequencies theta_i = base^(-2i/d_rope), computed on the host in fp64
// ("解耦 RoPE（MLA 下）" §七 rope; "从零理解 MLA", 解耦 RoPE precompute_cos_sin).
// The angle pos * theta_i is formed and its cos / sin evaluated in fp64 on the
// device, then rounded to fp32, so large positions keep full angle accuracy.
struct RopeParams {
  double theta[64];
  int d_rope;
  int half;  // 0: pairs (2i, 2i+1); 1: pairs (i, i + d_rope/2)
};

__device__ __forceinline__ float ld_f(const float *p) { return *p; }
__device__ __forceinline__ float ld_f(const __nv_bfloat16 *p) { return __bfloat162float(*p); }

template <class T> __device__ __forceinline__ T st_cast(float v);
template <> __device__ __forceinline__ float st_cast<float>(float v) { return v; }
template <> __device__ __forceinline__ __nv_bfloat16 st_cast<__nv_bfloat16>(float v) {
  return __float2bfloat16_rn(v);
}

__device__ __forceinline__ void set_error(int *err, int bit) { atomicOr(err, bit); }

// cos / sin of the angle pos * theta.  The angle is formed in fp64 and brought
// into [-pi, pi] by Cody-Waite reduction with 2 pi split into a double and its
// rounding remainder (exact enough for any int32 position); the reduced angle
// is then rounded to fp32 (absolute error <= 2^-24 pi) and the fp32 library
// sincosf takes it from there, so cf and sf are within a few 1e-7 of the exact
// values, far below the bf16 rounding of every value they rotate.  (An fp64
// sincos here is a long dependent chain of fp64 arithmetic on each thread.)
__device__ __forceinline__ void rope_cos_sin(int pos, double theta, float &cf, float &sf) {
  const double a = (double)pos * theta;
  const double k = rint(a * 0.15915494309189535);      // a / (2 pi), rounded
  double r = fma(-k, 6.283185307179586, a);             // 2 pi, leading double
  r = fma(-k, 2.4492935982947064e-16, r);               // 2 pi minus its leading double
  sincosf((float)r, &sf, &cf);
}

// Rotates the pair (x0, x1) by the angle whose cosine and sine are (cf, sf).
__device__ __forceinline__ void rope_rotate(float cf, float sf, float &x0, float &x1) {
  const float a = x0, b = x1;
  x0 = a * cf - b * sf;
  x1 = a * sf + b * cf;
}

// Rotates the pair (x0, x1) by pos * theta_i.
__device__ __forceinline__ void rope_pair(const RopeParams &rp, int i, int pos, float &x0,
                                          float &x1) {
  float cf, sf;
  rope_cos_sin(pos, rp.theta[i], cf, sf);
  rope_rotate(cf, sf, x0, x1);
}

// Programmatic dependent launch.  A kernel launched with launch_pdl may start
// while the previous kernel in its stream is still running: it must call
// grid_dep_wait() before it touches memory that kernel (or an earlier one)
// writes or reads, and every kernel so launched calls it, which keeps the
// stream order transitive.  grid_dep_launch() lets the next kernel start early.
__device__ __forceinline__ void grid_dep_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void grid_dep_launch() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t s,
                       Args &&...args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute at[1];
  at[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  at[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = at;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, static_cast<Args &&>(args)...);
}

// launch_pdl for a kernel launched in clusters of `cluster_x` CTAs along x
// (the grid's x extent must be a multiple of it).
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl_cluster(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem,
                               cudaStream_t s, int cluster_x, Args &&...args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute at[2];
  at[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  at[0].val.programmaticStreamSerializationAllowed = 1;
  at[1].id = cudaLaunchAttributeClusterDimension;
  at[1].val.clusterDim.x = cluster_x;
  at[1].val.clusterDim.y = 1;
  at[1].val.clusterDim.z = 1;
  cfg.attrs = at;
  cfg.numAttrs = 2;
  return cudaLaunchKernelEx(&cfg, kern, static_cast<Args &&>(args)...);
}

// Indices of the two members of RoPE pair i for width d.
__device__ __forceinline__ void rope_idx(const RopeParams &rp, int i, int &j0, int &j1) {
  if (rp.half) {
    j0 = i;
    j1 = i + rp.d_rope / 2;
  } else {
    j0 = 2 * i;
    j1 = 2 * i + 1;
  }
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}

// Per-call plan of the balanced split of a batch's cache pages into partitions.
// Written by the plan kernel into the workspace, read by the attention and
// combine kernels.
struct PlanHeader {
  int total_pages;   // sum over sequences of ceil(len / page_size) + gap (virtual pages)
  int quota;         // virtual pages per partition (last one may hold fewer)
  int parts;         // partitions with work
  int num_partials;  // partial slots used by split sequences
  int gap;           // virtual pages that stand for the fixed cost of each sequence
};

}  // namespace mla
