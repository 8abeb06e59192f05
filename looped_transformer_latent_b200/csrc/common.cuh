// Shared device helpers for the latent-attention kernels (sm_100a).
#pragma once

#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <stdint.h>

#include "lla.h"

namespace lla {

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
