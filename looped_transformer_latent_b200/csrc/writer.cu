// Latent writer: HLA eq. 2 and the LLA per-head / LLA-2D encoders.
//
// Every mode is a set of Z independent GEMMs out[m][n] = sum_k X(m,k) E(n,k)
// with m = (sequence, token) and k = (loop[, head], feature).  Phase 1 is a
// split-K SIMT fp32 GEMM writing partial sums to the workspace; phase 2 adds
// the partials in a fixed order (deterministic), rotates key pairs by
// R~_pos (HLA), rounds once to the storage type and stores the cache rows.
#include <cuda_fp8.h>

#include "writer_slice.cuh"

namespace lla {
namespace {

constexpr int BK = 32, WT = 256;

// Phase 1: C_part[z][split][m][n] = sum over this split's k-chunks.  Tile
// TM x TN (64 x 64, or 32 x 128 for decode-size batches), 32-deep k-chunks
// staged in shared memory, the next chunk prefetched into registers while the
// current one is multiplied; each thread owns a 4 x 4 block of outputs.
template <int TM, int TN>
__global__ void __launch_bounds__(WT) writer_gemm(WriterArgs a) {
  griddep_wait();
  constexpr int LA = TM * BK / WT, LB = TN * BK / WT;   // loads per thread
  constexpr int TX = TN / 4;                              // threads along n
  const int z = blockIdx.z / a.S, split = blockIdx.z % a.S;
  const Slice s = slice_of(a, z);
  const int n0 = blockIdx.x * TN, m0 = blockIdx.y * TM;
  if (n0 >= s.N) return;
  const int K = s.K_outer * s.d_in;
  const int nk = (K + BK - 1) / BK;
  const int kc0 = (int)((int64_t)nk * split / a.S), kc1 = (int)((int64_t)nk * (split + 1) / a.S);

  __shared__ float As[2][BK][TM + 4];
  __shared__ float Bs[2][BK][TN + 4];
  const int tid = threadIdx.x, tx = tid % TX, ty = tid / TX;
  float acc[4][4] = {};

  const int ar = tid / (BK / LA), ak = (tid % (BK / LA)) * LA;
  const int br = tid / (BK / LB), bk = (tid % (BK / LB)) * LB;
  const int m = m0 + ar;
  const bool mval = m < a.M;
  int64_t xrow = 0;
  if (mval) {
    const int b = m / a.n_tok, j = m % a.n_tok;
    xrow = (int64_t)b * a.xs_b + (int64_t)j * a.xs_n;
  }
  const int n = n0 + br;
  const bool nval = n < s.N;
  float ra[LA], rb[LB];
  // Each thread's run of LA (LB) consecutive k values is aligned and no longer
  // than 16, and feature blocks (d_in) are multiples of 16, so a run never
  // crosses from one (loop, head) block into the next.
  auto load = [&](int kc) {
    const int ka = kc * BK + ak, kb = kc * BK + bk;
    const bool av = mval && ka < K, bvld = nval && kb < K;
    const int oa = av ? ka / s.d_in : 0, da = av ? ka % s.d_in : 0;
    const int ob = bvld ? kb / s.d_in : 0, db = bvld ? kb % s.d_in : 0;
    const float* xp = s.X + xrow + (int64_t)(oa / s.o_h) * s.x_o_t + (int64_t)(oa % s.o_h) * s.x_o_h + da;
    const float* ep = s.E + (int64_t)ob * s.e_o + (int64_t)n * s.e_n + db;
#pragma unroll
    for (int u = 0; u < LA; ++u) ra[u] = av ? __ldg(xp + u) : 0.f;
#pragma unroll
    for (int u = 0; u < LB; ++u) rb[u] = bvld ? __ldg(ep + u) : 0.f;
  };
  auto stash = [&](int buf) {
#pragma unroll
    for (int u = 0; u < LA; ++u) As[buf][ak + u][ar] = ra[u];
#pragma unroll
    for (int u = 0; u < LB; ++u) Bs[buf][bk + u][br] = rb[u];
  };

  if (kc0 < kc1) {
    load(kc0);
    stash(0);
  }
  __syncthreads();
  for (int kc = kc0; kc < kc1; ++kc) {
    const int buf = (kc - kc0) & 1;
    if (kc + 1 < kc1) load(kc + 1);
#pragma unroll
    for (int kk = 0; kk < BK; ++kk) {
      float av[4], bv[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) av[i] = As[buf][kk][ty * 4 + i];
#pragma unroll
      for (int i = 0; i < 4; ++i) bv[i] = Bs[buf][kk][tx * 4 + i];
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int jj = 0; jj < 4; ++jj) acc[i][jj] = fmaf(av[i], bv[jj], acc[i][jj]);
    }
    if (kc + 1 < kc1) stash(buf ^ 1);
    __syncthreads();
  }
  float* P = a.part + ((int64_t)(z * a.S + split) * a.M) * a.Nmax;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int mm = m0 + ty * 4 + i;
    if (mm >= a.M) continue;
#pragma unroll
    for (int jj = 0; jj < 4; ++jj) {
      const int nn = n0 + tx * 4 + jj;
      if (nn < s.N) P[(int64_t)mm * a.Nmax + nn] = acc[i][jj];
    }
  }
  griddep_launch();
}

// Phase 2: ordered sum of the splits, rotation of key pairs, rounding, store.
__global__ void writer_epilogue(WriterArgs a) {
  griddep_wait();
  const int64_t pairs = a.Nmax / 2;
  const int64_t total = (int64_t)a.Z * a.M * pairs;
  for (int64_t idx = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; idx < total;
       idx += (int64_t)gridDim.x * blockDim.x) {
    const int p = (int)(idx % pairs);
    const int m = (int)((idx / pairs) % a.M);
    const int z = (int)(idx / (pairs * a.M));
    const Slice s = slice_of(a, z);
    const int n = 2 * p;
    if (n >= s.N) continue;
    float x = 0.f, y = 0.f;
    for (int sp = 0; sp < a.S; ++sp) {
      const float* P = a.part + ((int64_t)(z * a.S + sp) * a.M + m) * a.Nmax;
      x += P[n];
      y += P[n + 1];
    }
    if (*a.err) x = y = NAN;
    const int b = m / a.n_tok, j = m % a.n_tok;
    const int pos = a.pos0 + j;
    if (n < s.rot_dim) {
      float c, sn;
      rope_cs(p, s.rot_dim, a.d_h, a.base, (double)pos, &c, &sn);
      const float xr = x * c - y * sn, yr = x * sn + y * c;
      x = xr; y = yr;
    }
    const int64_t o = (int64_t)b * s.os_b + s.col0 + (int64_t)pos * s.os_n + n;
    store_elem(s.out, o, a.dtype, x);
    store_elem(s.out, o + 1, a.dtype, y);
  }
  griddep_launch();
}

// Phase 2 for fp8 rows (e4m3 codes with per-token, per-part scales): one warp
// per (target row, token).  HLA: target 0 is the main latent (slice 0), target
// 1 the loop-1 latent (slice 1); FOLDED: target 0 takes its key part from
// slice 0 and its value part from slice 1.  The warp sums the splits in order,
// rotates the key pairs (HLA), keeps the row in shared memory, reduces the
// largest magnitude of each part, and stores codes = e4m3(x / s) (nearest-even,
// saturating) with s = amax / 448, then s^K, s^V and 8 zero bytes.
constexpr int FP8_WARPS = 4;                 // static shared memory: 4 rows of up to 2048 floats
constexpr int FP8_ROW_MAX = 2048;

__device__ __forceinline__ float fp8_part_value(const WriterArgs& a, int tgt, int m, int n, int kw) {
  // column n of target row tgt, before rotation
  int z = tgt, nn = n;
  if (a.mode == LLA_WRITE_FOLDED && n >= kw) { z = 1; nn = n - kw; }
  float x = 0.f;
  for (int sp = 0; sp < a.S; ++sp) x += a.part[((int64_t)(z * a.S + sp) * a.M + m) * a.Nmax + nn];
  return x;
}

__global__ void __launch_bounds__(FP8_WARPS * 32) writer_epilogue_fp8(WriterArgs a) {
  griddep_wait();
  __shared__ float rowbuf[FP8_WARPS][FP8_ROW_MAX];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int ntgt = a.mode == LLA_WRITE_HLA ? 2 : 1;
  const int64_t total = (int64_t)ntgt * a.M;
  float* buf = rowbuf[warp];
  for (int64_t idx = (int64_t)blockIdx.x * FP8_WARPS + warp; idx < total; idx += (int64_t)gridDim.x * FP8_WARPS) {
    const int tgt = (int)(idx / a.M), m = (int)(idx % a.M);
    int kw, vw;
    if (a.mode == LLA_WRITE_HLA) {
      kw = tgt == 0 ? a.r_k : a.r_1;
      vw = tgt == 0 ? a.r_v : a.r_1;
    } else {
      kw = a.r_k;
      vw = a.r_v;
    }
    const bool rot = a.mode == LLA_WRITE_HLA && a.rotate;
    const int b = m / a.n_tok, j = m % a.n_tok;
    const int pos = a.pos0 + j;
    float amax_k = 0.f, amax_v = 0.f;
    for (int p = lane; p < (kw + vw) / 2; p += 32) {
      const int n = 2 * p;
      float x = fp8_part_value(a, tgt, m, n, kw), y = fp8_part_value(a, tgt, m, n + 1, kw);
      if (rot && n < kw) {
        float c, sn;
        rope_cs(p, kw, a.d_h, a.base, (double)pos, &c, &sn);
        const float xr = x * c - y * sn, yr = x * sn + y * c;
        x = xr; y = yr;
      }
      buf[n] = x;
      buf[n + 1] = y;
      const float mx = fmaxf(fabsf(x), fabsf(y));
      if (n < kw) amax_k = fmaxf(amax_k, mx); else amax_v = fmaxf(amax_v, mx);
    }
    amax_k = warp_max(amax_k);
    amax_v = warp_max(amax_v);
    __syncwarp();
    const bool bad = *a.err != 0;
    const float sk = bad ? NAN : amax_k / 448.f, sv = bad ? NAN : amax_v / 448.f;
    uint8_t* row;
    if (tgt == 0) row = reinterpret_cast<uint8_t*>(a.out0) + (int64_t)b * a.os_b + (int64_t)pos * a.os_n;
    else row = reinterpret_cast<uint8_t*>(a.out1) + (int64_t)b * a.o1s_b + (int64_t)pos * a.o1s_n;
    for (int n = lane; n < kw + vw; n += 32) {
      const float s = n < kw ? sk : sv;
      const float q = s > 0.f ? buf[n] / s : 0.f;
      const __nv_fp8_e4m3 code(q);   // nearest-even, saturating to +-448
      row[n] = *reinterpret_cast<const uint8_t*>(&code);
    }
    if (lane < 4) {
      const float sc[2] = {sk, sv};
      reinterpret_cast<float*>(row + kw + vw)[lane] = lane < 2 ? sc[lane] : 0.f;
    }
    __syncwarp();
  }
  griddep_launch();
}

}  // namespace

// Partial sums, then (16 bytes) the tensor-core error flag.
size_t writer_workspace_floats(const WriterArgs& a) {
  return (size_t)a.Z * a.S * a.M * a.Nmax + 4;
}

static bool small_batch(const WriterArgs& a) { return a.M <= 32; }

int writer_depth_splits(const WriterArgs& a) {
  int nk_max = 1;
  for (int z = 0; z < a.Z; ++z) {
    const Slice s = slice_of(a, z);
    nk_max = nk_max > ceil_div(s.K_outer * s.d_in, BK) ? nk_max : ceil_div(s.K_outer * s.d_in, BK);
  }
  const int S = ceil_div(nk_max, 16);
  return S < 1 ? 1 : S > 64 ? 64 : S;
}

int writer_pick_splits(const WriterArgs& a, int num_sms) {
  (void)num_sms;
  return writer_depth_splits(a);
}

cudaError_t launch_writer(const WriterArgs& a_in, cudaStream_t st) {
  WriterArgs a = a_in;
  if (a.M == 0) return cudaSuccess;
  a.err = reinterpret_cast<int*>(a.part + (size_t)a.Z * a.S * a.M * a.Nmax);
  cudaError_t e0 = cudaMemsetAsync(a.err, 0, sizeof(int), st);
  if (e0 != cudaSuccess) return e0;
  bool simt = !a.use_tc;
  if (a.use_tc) {
    e0 = launch_writer_tc(a, a.err, st);
    if (e0 == cudaErrorNotSupported) simt = true;   // no tensor-map view of these operands
  }
  if (simt) {
    if (small_batch(a)) {
      dim3 grid(ceil_div(a.Nmax, 128), ceil_div(a.M, 32), a.Z * a.S);
      e0 = launch_kernel(writer_gemm<32, 128>, grid, dim3(WT), 0, st, 1, a);
    } else {
      dim3 grid(ceil_div(a.Nmax, 64), ceil_div(a.M, 64), a.Z * a.S);
      e0 = launch_kernel(writer_gemm<64, 64>, grid, dim3(WT), 0, st, 1, a);
    }
  }
  if (e0 != cudaSuccess) return e0;
  if (a.dtype == LLA_FP8_E4M3) {
    const int64_t rows = (int64_t)(a.mode == LLA_WRITE_HLA ? 2 : 1) * a.M;
    int blocks = (int)((rows + FP8_WARPS - 1) / FP8_WARPS);
    if (blocks > 148 * 16) blocks = 148 * 16;
    return launch_kernel(writer_epilogue_fp8, dim3(blocks), dim3(FP8_WARPS * 32), 0, st, 1, a);
  }
  const int64_t total = (int64_t)a.Z * a.M * (a.Nmax / 2);
  int blocks = (int)((total + 255) / 256);
  if (blocks > 148 * 16) blocks = 148 * 16;
  return launch_kernel(writer_epilogue, dim3(blocks), dim3(256), 0, st, 1, a);
}

}  // namespace lla
