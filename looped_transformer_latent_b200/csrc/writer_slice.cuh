// Decomposition of the latent writer into independent GEMMs ("slices"):
// out[m][n] = sum_k X(m, k) E(n, k) with m = (sequence, token) and
// k = (outer block, feature), outer = loop (HLA, PERHEAD) or (loop, head)
// (FOLDED).  Shared by the SIMT and the tensor-core writer kernels.
#pragma once

#include "kernels.cuh"

namespace lla {

struct Slice {
  const float* X;       // first feature of outer block 0 for token row 0
  int64_t x_o_t, x_o_h; // X offset per loop, per head (outer = t * o_h + h)
  int o_h;              // heads folded into the outer index (FOLDED: H, else 1)
  const float* E;       // E(n, k) at E + (k / d_in) * e_o + n * e_n + k % d_in
  int64_t e_o, e_n;
  int K_outer, d_in, N;
  void* out;
  int64_t os_b, os_n, col0;
  int rot_dim;          // leading columns rotated by R~_pos (HLA key parts)
};

__host__ __device__ __forceinline__ Slice slice_of(const WriterArgs& a, int z) {
  Slice s;
  if (a.mode == LLA_WRITE_HLA) {
    if (z == 0) {  // c_j = sum_{t=2..T} E_t h_{j,t}
      s.X = a.x + a.xs_t; s.x_o_t = a.xs_t; s.x_o_h = 0; s.o_h = 1;
      s.N = a.r_k + a.r_v;
      s.E = a.E_main; s.e_o = (int64_t)s.N * a.D; s.e_n = a.D;
      s.K_outer = a.T - 1; s.d_in = a.D;
      s.out = a.out0; s.os_b = a.os_b; s.os_n = a.os_n; s.col0 = 0;
      s.rot_dim = a.rotate ? a.r_k : 0;
    } else {       // c^(1)_j = E_1 h_{j,1}
      s.X = a.x; s.x_o_t = 0; s.x_o_h = 0; s.o_h = 1;
      s.N = 2 * a.r_1;
      s.E = a.E_1; s.e_o = 0; s.e_n = a.D;
      s.K_outer = 1; s.d_in = a.D;
      s.out = a.out1; s.os_b = a.o1s_b; s.os_n = a.o1s_n; s.col0 = 0;
      s.rot_dim = a.rotate ? a.r_1 : 0;
    }
  } else if (a.mode == LLA_WRITE_PERHEAD) {  // c_{j,h} = sum_t E_{t,h} k_{j,t,h}
    const int part = z / a.H, h = z % a.H;
    const int r = part ? a.r_v : a.r_k;
    s.X = (part ? a.xv : a.x) + (int64_t)h * a.d_h; s.x_o_t = a.xs_t; s.x_o_h = 0; s.o_h = 1;
    s.N = r;
    s.E = (part ? a.E_V : a.E_K) + (int64_t)h * r * a.d_h;
    s.e_o = (int64_t)a.H * r * a.d_h; s.e_n = a.d_h;
    s.K_outer = a.T; s.d_in = a.d_h;
    s.out = part ? a.out1 : a.out0; s.os_b = a.os_b; s.os_n = a.os_n;
    s.col0 = (int64_t)h * a.os_h;
    s.rot_dim = 0;
  } else {  // FOLDED: c_j = sum_{t,h} E_{t,h} k_{j,t,h}
    const int part = z;
    const int r = part ? a.r_v : a.r_k;
    s.X = part ? a.xv : a.x; s.x_o_t = a.xs_t; s.x_o_h = a.d_h; s.o_h = a.H;
    s.N = r;
    s.E = part ? a.E_V : a.E_K; s.e_o = (int64_t)r * a.d_h; s.e_n = a.d_h;
    s.K_outer = a.T * a.H; s.d_in = a.d_h;
    s.out = a.out0; s.os_b = a.os_b; s.os_n = a.os_n; s.col0 = part ? a.r_k : 0;
    s.rot_dim = 0;
  }
  return s;
}

// Pointer to X(m, k) for slice s (k inside one outer block).
__device__ __forceinline__ int64_t writer_xrow(const WriterArgs& a, int m) {
  const int b = m / a.n_tok, j = m % a.n_tok;
  return (int64_t)b * a.xs_b + (int64_t)j * a.xs_n;
}

}  // namespace lla
