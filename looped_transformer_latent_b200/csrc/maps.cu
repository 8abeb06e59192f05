// The per-(loop, head) linear maps of the absorbed read, as one tiled kernel:
//
//   query map  (HLA summary eq. 3):  q~[b][row] = s*log2e * R~_i A_row^T q[b][row]
//   output map (eq. 4):              o[b][row]  = (B_row^T y~[b][row] + w_win y_w[b][row]) / l
//
// Both are, for every query row (loop t, head h), a [B x K] x [K x N] product
// with that row's own codec matrix W_row = A_{t,h} (K = d_h, N = r_k) or
// B_{t,h} (K = r_v, N = d_h).  One CTA computes a 16- or 32-sequence x
// 64-column tile of one row: K is walked in chunks of 64 staged in shared memory (both the
// activations and the codec tile), the next chunk is fetched into registers
// while the current one is multiplied, and each thread owns one column pair
// (so the query map can rotate the pair in its epilogue) for four sequences.
// For the output map, the operand y~ is formed on the fly from the split
// partials: y~ = sum_s 2^(m_s - M) y~_s, with M the max over the splits and
// the window, so the split merge costs no separate pass.
#include "kernels.cuh"

namespace lla {
namespace {

constexpr int GN = 64;      // columns per tile (32 pairs)
constexpr int GT = 256;     // threads
constexpr int MAXS = 16;    // split partials the output map can combine

__device__ __forceinline__ int64_t qbf_index(int b, int row, int k, int r_k) {
  const int kb = k >> 6, e = k & 63;
  return (int64_t)b * (r_k >> 6) * 4096 + kb * 4096 + row * 64 + ((((e >> 3) ^ (row & 7)) << 3) | (e & 7));
}

template <int MODE, int GB, int GK>
__global__ void __launch_bounds__(GT) row_gemm(MapArgs g) {
  griddep_wait();
  // the query map opens the call: it clears the call's error word, which only
  // the kernels after it write
  if (MODE == 0 && g.clear_err && blockIdx.x == 0 && blockIdx.y == 0 && blockIdx.z == 0 && threadIdx.x == 0)
    *g.clear_err = 0;
  constexpr int BPW = GB / (GT / 32);   // sequences per warp
  constexpr int LX = GB * GK / GT;      // activation loads per thread
  __shared__ float Xs[2][GK][GB + 1];
  __shared__ __align__(16) float Ws[2][GK][GN];
  __shared__ float wsplit[GB][MAXS + kMaxWindowChunks];   // MODE 1: split, then window weights
  __shared__ float linv[GB];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int row = blockIdx.x;
  const int b0 = blockIdx.z * GB;
  const int nb = min(GB, g.B - b0);
  const int ntile = (g.N + GN - 1) / GN;

  if (MODE == 0) {
    if (row >= g.rows) {
      // rows of the tensor-core operand past the last query row are zero
      if (g.use_tc && (int)blockIdx.y < ntile) {
        const int n = blockIdx.y * GN + 2 * lane;
        if (n < g.N)
          for (int bb = warp; bb < nb; bb += GT / 32)
            *reinterpret_cast<__nv_bfloat162*>(g.qbf + qbf_index(b0 + bb, row, n, g.N)) =
                __floats2bfloat162_rn(0.f, 0.f);
      }
      return;
    }
  } else {
    // weights of this tile's sequences: splits, then window chunks
    const int64_t bstride = (int64_t)g.B * g.rows;
    for (int bb = tid; bb < GB; bb += GT) {
      float M = -INFINITY, L = 0.f;
      if (bb < nb) {
        const int64_t br = (int64_t)(b0 + bb) * g.rows + row;
        for (int c = 0; c < g.Sw; ++c) M = fmaxf(M, g.win_ml[(c * bstride + br) * 2]);
        for (int s = 0; s < g.S; ++s) M = fmaxf(M, g.part_ml[(s * bstride + br) * 2]);
        for (int s = 0; s < g.S; ++s) {
          const float ms = g.part_ml[(s * bstride + br) * 2];
          const float w = ms == -INFINITY ? 0.f : exp2f(ms - M);
          wsplit[bb][s] = w;
          L += w * g.part_ml[(s * bstride + br) * 2 + 1];
        }
        for (int c = 0; c < g.Sw; ++c) {
          const float mc = g.win_ml[(c * bstride + br) * 2];
          const float w = mc == -INFINITY ? 0.f : exp2f(mc - M);
          wsplit[bb][MAXS + c] = w;
          L += w * g.win_ml[(c * bstride + br) * 2 + 1];
        }
      }
      linv[bb] = bb < nb ? 1.f / L : 0.f;
    }
    __syncthreads();
  }

  const int n0 = blockIdx.y * GN;
  const int tn = lane;             // column pair within the tile
  const int tb = warp * BPW;       // first of this thread's sequences
  // several query positions share each (loop, head) codec
  const float* Wr = g.W + (int64_t)(g.ncodec > 0 ? row % g.ncodec : row) * g.K * g.N;
  // loader coordinates
  const int xb = tid / (GK / LX), xk = (tid % (GK / LX)) * LX;   // X: GB sequences x 32 k
  constexpr int LW = GK * GN / GT;                  // codec loads per thread
  const int wk = tid / (GN / LW), wn = (tid % (GN / LW)) * LW;   // W: GK k x 64 columns
  float xr[LX], wr[LW];
  auto load = [&](int k0) {
    const int b = b0 + xb;
#pragma unroll
    for (int u = 0; u < LX; ++u) {
      const int k = k0 + xk + u;
      float v = 0.f;
      if (xb < nb && k < g.K) {
        if (MODE == 0) {
          v = g.X[(int64_t)b * g.xs_b + (int64_t)row * g.xs_row + k];
        } else {
          const int64_t br = (int64_t)b * g.rows + row;
          for (int s = 0; s < g.S; ++s)
            v = fmaf(wsplit[xb][s], g.part_y[((int64_t)s * g.B * g.rows + br) * g.K + k], v);
        }
      }
      xr[u] = v;
    }
    const int k = k0 + wk;
#pragma unroll
    for (int u = 0; u < LW; ++u) {
      const int n = n0 + wn + u;
      wr[u] = (k < g.K && n < g.N) ? __ldg(Wr + (int64_t)k * g.N + n) : 0.f;
    }
  };
  auto stash = [&](int buf) {
#pragma unroll
    for (int u = 0; u < LX; ++u) Xs[buf][xk + u][xb] = xr[u];
#pragma unroll
    for (int u = 0; u < LW; u += 4)
      *reinterpret_cast<float4*>(&Ws[buf][wk][wn + u]) = make_float4(wr[u], wr[u + 1], wr[u + 2], wr[u + 3]);
  };

  float acc[BPW][2] = {};
  const int nk = (g.K + GK - 1) / GK;
  load(0);
  stash(0);
  __syncthreads();
  for (int kc = 0; kc < nk; ++kc) {
    const int buf = kc & 1;
    if (kc + 1 < nk) load((kc + 1) * GK);
#pragma unroll 16
    for (int k = 0; k < GK; ++k) {
      const float2 w = *reinterpret_cast<const float2*>(&Ws[buf][k][2 * tn]);
#pragma unroll
      for (int j = 0; j < BPW; ++j) {
        const float x = Xs[buf][k][tb + j];
        acc[j][0] = fmaf(x, w.x, acc[j][0]);
        acc[j][1] = fmaf(x, w.y, acc[j][1]);
      }
    }
    if (kc + 1 < nk) stash(buf ^ 1);
    __syncthreads();
  }

  const int n = n0 + 2 * tn;
  if (n >= g.N) return;
  if (MODE == 0) {
    float c = 1.f, s = 0.f;
    if (g.rotate)
      rope_cs(n / 2, g.N, g.d_h, g.base, (double)(g.pos + (g.rows_per_q > 0 ? row / g.rows_per_q : 0)), &c, &s);
#pragma unroll
    for (int j = 0; j < BPW; ++j) {
      const int bb = tb + j;
      if (bb >= nb) break;
      const float x = (acc[j][0] * c - acc[j][1] * s) * g.qmul;
      const float y = (acc[j][0] * s + acc[j][1] * c) * g.qmul;
      if (g.use_tc) {
        *reinterpret_cast<__nv_bfloat162*>(g.qbf + qbf_index(b0 + bb, row, n, g.N)) = __floats2bfloat162_rn(x, y);
      } else {
        float* dst = g.qlat + ((int64_t)(b0 + bb) * g.rows + row) * g.N + n;
        dst[0] = x;
        dst[1] = y;
      }
    }
  } else {
    const bool bad = g.err && *g.err;
#pragma unroll
    for (int j = 0; j < BPW; ++j) {
      const int bb = tb + j;
      if (bb >= nb) break;
      const int b = b0 + bb;
      const int64_t br = (int64_t)b * g.rows + row;
      const float li = linv[bb];
      float y0 = acc[j][0], y1 = acc[j][1];
      for (int c = 0; c < g.Sw; ++c) {
        const float* yw = g.win_y + ((int64_t)c * g.B * g.rows + br) * g.N + n;
        y0 = fmaf(wsplit[bb][MAXS + c], yw[0], y0);
        y1 = fmaf(wsplit[bb][MAXS + c], yw[1], y1);
      }
      float* dst = g.out + (int64_t)b * g.outs_b + (int64_t)row * g.N + n;
      dst[0] = bad ? NAN : y0 * li;
      dst[1] = bad ? NAN : y1 * li;
    }
  }
  griddep_launch();
}

}  // namespace

int map_max_splits() { return MAXS; }

cudaError_t launch_query_map(const MapArgs& g, cudaStream_t st) {
  const int ntile = (g.N + GN - 1) / GN;
  dim3 grid(g.use_tc ? 64 : g.rows, ntile, (g.B + 31) / 32);
  return launch_kernel(row_gemm<0, 32, 32>, grid, dim3(GT), 0, st, 1, g);
}

cudaError_t launch_output_map(const MapArgs& g, cudaStream_t st) {
  if (g.B <= 64) {
    dim3 grid(g.rows, (g.N + GN - 1) / GN, (g.B + 15) / 16);
    return launch_kernel(row_gemm<1, 16, 32>, grid, dim3(GT), 0, st, 1, g);
  }
  dim3 grid(g.rows, (g.N + GN - 1) / GN, (g.B + 31) / 32);
  return launch_kernel(row_gemm<1, 32, 32>, grid, dim3(GT), 0, st, 1, g);
}

}  // namespace lla
