// Shared device helpers for the latent-attention kernels (sm_100a).
#pragma once

#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <stdint.h>

#include <cstring>
#include <utility>

#include "lla.h"

namespace lla {

// ---------------------------------------------- programmatic dependent launch --
// With LLA_PDL=1 in the environment every kernel of this library is launched
// with programmatic stream serialization: its CTAs may be scheduled, and run
// their prologue (barrier setup, TMEM allocation, tensor-map prefetch), while
// the previous kernel on the stream drains.  Each kernel executes
// griddep_wait() before its first global-memory access (it returns once the
// previous grid has completed and its writes are visible; without the
// attribute it returns at once) and griddep_launch() as the last instruction
// of its CTAs, after any TMEM is freed: dependents start only once every CTA
// of this grid has started and finished its work, so no CTA of this grid ever
// waits for resources held by a dependent.  Off by default: on the decode
// steps measured it changed the step time by less than the run-to-run spread.
__device__ __forceinline__ void griddep_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void griddep_launch() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

bool pdl_enabled();

// Launch kern<<<grid, block, smem, st>>>(args...) with programmatic stream
// serialization (when enabled) and, for cluster_x > 1, clusters of cluster_x
// CTAs along x.
template <typename... Exp, typename... Act>
cudaError_t launch_kernel(void (*kern)(Exp...), dim3 grid, dim3 block, size_t smem, cudaStream_t st, int cluster_x,
                          Act&&... args) {
  cudaLaunchConfig_t cfg;
  std::memset(&cfg, 0, sizeof(cfg));
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[2];
  std::memset(attr, 0, sizeof(attr));
  unsigned n = 0;
  if (cluster_x > 1) {
    attr[n].id = cudaLaunchAttributeClusterDimension;
    attr[n].val.clusterDim.x = cluster_x;
    attr[n].val.clusterDim.y = 1;
    attr[n].val.clusterDim.z = 1;
    ++n;
  }
  if (pdl_enabled()) {
    attr[n].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[n].val.programmaticStreamSerializationAllowed = 1;
    ++n;
  }
  cfg.attrs = attr;
  cfg.numAttrs = n;
  return cudaLaunchKernelEx(&cfg, kern, std::forward<Act>(args)...);
}

constexpr float kLog2e = 1.4426950408889634f;

__device__ __forceinline__ float load_elem(const void* base, int64_t idx, int dtype) {
  if (dtype == LLA_BF16)
    return __bfloat162float(reinterpret_cast<const __nv_bfloat16*>(base)[idx]);
  return reinterpret_cast<const float*>(base)[idx];
}

__device__ __forceinline__ void store_elem(void* base, int64_t idx, int dtype, float v) {
  if (dtype == LLA_BF16)
    reinterpret_cast<__nv_bfloat16*>(base)[idx] = __float2bfloat16_rn(v);
  else
    reinterpret_cast<float*>(base)[idx] = v;
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

// Rotary angle of pair p in a vector of even length d at position pos:
// pos * base^(-2 f / d_h) with f = floor(p * d_h / d).  fp64 throughout, so the
// angle stays accurate at positions ~16K; the cosine and sine are the CUDA
// math library's fp64 sincos, rounded once to fp32.
__device__ __forceinline__ void rope_cs(int p, int d, int d_h, double base, double pos,
                                        float* c, float* s) {
  const int f = (int)(((long long)p * d_h) / d);
  const double theta = pow(base, -2.0 * (double)f / (double)d_h);
  double sd, cd;
  sincos(pos * theta, &sd, &cd);
  *c = (float)cd;
  *s = (float)sd;
}

__host__ __device__ __forceinline__ int64_t ceil_div64(int64_t a, int64_t b) { return (a + b - 1) / b; }
__host__ __device__ __forceinline__ int ceil_div(int a, int b) { return (a + b - 1) / b; }

}  // namespace lla
