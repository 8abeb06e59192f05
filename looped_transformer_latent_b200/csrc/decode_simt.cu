// SIMT kernels of the decode path: query prologue (A^T q with rotation),
// split-context absorbed latent read (fp32 and bf16 latents), LLA
// reconstruct-on-read, exact-window attention, and the split merge with the
// B_t^T map back to head space.  Scores are kept in base-2 units: every query
// is pre-multiplied by scale * log2(e) so the softmax uses exp2.
#include "kernels.cuh"

namespace lla {
namespace {

// ------------------------------------------------- absorbed split, SIMT --
// One CTA per (split, sequence, block of RB query rows).  A tile of TT latent
// tokens is staged in shared memory (fp32), scores for RB x TT pairs are one
// per thread, the online softmax runs per half-warp (one row), and every
// thread accumulates y~[row][v] = sum_j p_j c^V_j for its v columns.
constexpr int RB = 16, TT = 16, VC = 4;  // r_v <= 1024

__global__ void __launch_bounds__(256) absorb_split_simt(AbsorbArgs a) {
  extern __shared__ float sm[];
  const int s = blockIdx.x, b = blockIdx.y, row0 = blockIdx.z * RB;
  const int nr = min(RB, a.rows - row0);
  const int R = a.r_k + a.r_v;
  const int LD = R + ((33 - (R % 32)) % 32);  // row stride == 1 (mod 32)
  float* qs = sm;                            // [RB][r_k]
  float* lt = qs + RB * a.r_k;               // [TT][LD]
  float* ps = lt + TT * LD;                  // [RB][TT]
  float* alpha = ps + RB * TT;               // [RB]
  float* mrun = alpha + RB;                  // [RB]
  float* lrun = mrun + RB;                   // [RB]
  const int tid = threadIdx.x;
  const int tok0 = s * a.tps, tok1 = min(a.n_lat, tok0 + a.tps);

  for (int idx = tid; idx < RB * a.r_k; idx += 256) {
    const int r = idx / a.r_k, c = idx % a.r_k;
    qs[idx] = r < nr ? a.qlat[((int64_t)b * a.rows + row0 + r) * a.r_k + c] : 0.f;
  }
  if (tid < RB) { mrun[tid] = -INFINITY; lrun[tid] = 0.f; }
  float acc[RB][VC];
#pragma unroll
  for (int r = 0; r < RB; ++r)
#pragma unroll
    for (int c = 0; c < VC; ++c) acc[r][c] = 0.f;
  __syncthreads();

  const int sr = tid / TT, si = tid % TT;  // score owner: row sr, token si
  for (int j0 = tok0; j0 < tok1; j0 += TT) {
    const int nt = min(TT, tok1 - j0);
    for (int idx = tid; idx < nt * R; idx += 256) {
      const int i = idx / R, c = idx % R;
      lt[i * LD + c] = load_elem(a.lat, (int64_t)b * a.ls_b + (int64_t)(j0 + i) * a.ls_n + c, a.lat_dtype);
    }
    __syncthreads();
    float sc = -INFINITY;
    if (sr < nr && si < nt) {
      float d = 0.f;
      const float* qr = qs + sr * a.r_k;
      const float* kr = lt + si * LD;
      for (int c = 0; c < a.r_k; ++c) d = fmaf(qr[c], kr[c], d);
      sc = d;
    }
    float tmax = sc;
#pragma unroll
    for (int o = 8; o > 0; o >>= 1) tmax = fmaxf(tmax, __shfl_xor_sync(0xffffffffu, tmax, o));
    const float mold = mrun[sr];
    const float mnew = fmaxf(mold, tmax);
    const float p = (sr < nr && si < nt) ? exp2f(sc - mnew) : 0.f;
    float psum = p;
#pragma unroll
    for (int o = 8; o > 0; o >>= 1) psum += __shfl_xor_sync(0xffffffffu, psum, o);
    ps[sr * TT + si] = p;
    __syncwarp();
    if (si == 0 && sr < nr) {
      const float al = (mold == -INFINITY) ? 0.f : exp2f(mold - mnew);
      alpha[sr] = al;
      lrun[sr] = lrun[sr] * al + psum;
      mrun[sr] = mnew;
    }
    __syncthreads();
#pragma unroll
    for (int c = 0; c < VC; ++c) {
      const int v = tid + 256 * c;
      if (v >= a.r_v) break;
      const float* cv = lt + a.r_k + v;
#pragma unroll
      for (int r = 0; r < RB; ++r) {
        if (r >= nr) break;
        float y = acc[r][c] * alpha[r];
        for (int i = 0; i < nt; ++i) y = fmaf(ps[r * TT + i], cv[i * LD], y);
        acc[r][c] = y;
      }
    }
    __syncthreads();
  }
  // partial results of this split
  if (tid < nr) {
    float* ml = a.part_ml + (((int64_t)s * a.B + b) * a.rows + row0 + tid) * 2;
    ml[0] = mrun[tid];
    ml[1] = lrun[tid];
  }
#pragma unroll
  for (int c = 0; c < VC; ++c) {
    const int v = tid + 256 * c;
    if (v >= a.r_v) break;
#pragma unroll
    for (int r = 0; r < RB; ++r) {
      if (r >= nr) break;
      a.part_y[(((int64_t)s * a.B + b) * a.rows + row0 + r) * a.r_v + v] = acc[r][c];
    }
  }
}

// --------------------------------------------------------------- window --
// Exact attention over the window ring for one (row, sequence).  Each lane
// holds 4 consecutive elements of the head dimension (one 8- or 16-byte load
// per token), each warp takes every 4th group of WU tokens and issues all of a
// group's K and V loads before using them, keeps its own online softmax, and
// the four warps are combined at the end.  Emits (max, sum, y_w) in base-2 units.
template <bool BF16>
struct WinTraits;
template <>
struct WinTraits<true> {   // 4 bf16 per lane, packed in a uint2
  typedef uint2 raw_t;
  static constexpr int WU = 16;
  __device__ __forceinline__ static raw_t load(const void* base, int64_t idx) {
    return *reinterpret_cast<const uint2*>(reinterpret_cast<const __nv_bfloat16*>(base) + idx);
  }
  __device__ __forceinline__ static void unpack(raw_t u, float* v) {
    const float2 a = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&u.x));
    const float2 b = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&u.y));
    v[0] = a.x; v[1] = a.y; v[2] = b.x; v[3] = b.y;
  }
  __device__ __forceinline__ static raw_t zero() { return make_uint2(0u, 0u); }
};
template <>
struct WinTraits<false> {  // 4 fp32 per lane
  typedef float4 raw_t;
  static constexpr int WU = 8;
  __device__ __forceinline__ static raw_t load(const void* base, int64_t idx) {
    return *reinterpret_cast<const float4*>(reinterpret_cast<const float*>(base) + idx);
  }
  __device__ __forceinline__ static void unpack(raw_t u, float* v) { v[0] = u.x; v[1] = u.y; v[2] = u.z; v[3] = u.w; }
  __device__ __forceinline__ static raw_t zero() { return make_float4(0.f, 0.f, 0.f, 0.f); }
};

template <bool BF16>
__global__ void __launch_bounds__(128) window_attn(WindowArgs w) {
  typedef WinTraits<BF16> Tr;
  constexpr int WU = Tr::WU;
  const int row = blockIdx.x, b = blockIdx.y;
  const int tt = row / w.H, h = row % w.H, t = w.t0 + tt;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int d0 = 4 * lane;
  const bool dv = d0 < w.d_h;
  float qv[4] = {0.f, 0.f, 0.f, 0.f}, acc[4] = {0.f, 0.f, 0.f, 0.f};
  if (dv) {
    const float* q = w.q + (int64_t)b * w.q_sb + (int64_t)row * w.q_srow + d0;
#pragma unroll
    for (int e = 0; e < 4; ++e) qv[e] = q[e] * w.qmul;
  }
  float m = -INFINITY, l = 0.f;
  const int64_t seq = (int64_t)b * w.wins_b;
  for (int g0 = warp * WU; g0 < w.n_win; g0 += 4 * WU) {
    typename Tr::raw_t kr[WU], vr[WU];
#pragma unroll
    for (int u = 0; u < WU; ++u) {
      const int idx = g0 + u;
      if (dv && idx < w.n_win) {
        const int slot = (w.win_start + idx) % w.Wcap;
        const int64_t base = seq + (((int64_t)t * w.Wcap + slot) * w.H + h) * w.d_h + d0;
        kr[u] = Tr::load(w.wk, base);
        vr[u] = Tr::load(w.wv, base);
      } else {
        kr[u] = Tr::zero();
        vr[u] = Tr::zero();
      }
    }
    float sc[WU];
#pragma unroll
    for (int u = 0; u < WU; ++u) {
      float kk[4];
      Tr::unpack(kr[u], kk);
      float part = 0.f;
#pragma unroll
      for (int e = 0; e < 4; ++e) part = fmaf(qv[e], kk[e], part);
      sc[u] = part;
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1)
#pragma unroll
      for (int u = 0; u < WU; ++u) sc[u] += __shfl_xor_sync(0xffffffffu, sc[u], o);
    // one max per group of tokens, then a single rescale of the running state
    float gm = -INFINITY;
#pragma unroll
    for (int u = 0; u < WU; ++u)
      if (g0 + u < w.n_win) gm = fmaxf(gm, sc[u]);
    const float mn = fmaxf(m, gm);
    const float al = (m == -INFINITY) ? 0.f : exp2f(m - mn);
    l *= al;
#pragma unroll
    for (int e = 0; e < 4; ++e) acc[e] *= al;
#pragma unroll
    for (int u = 0; u < WU; ++u) {
      if (g0 + u >= w.n_win) break;
      const float p = exp2f(sc[u] - mn);
      float vv[4];
      Tr::unpack(vr[u], vv);
      l += p;
#pragma unroll
      for (int e = 0; e < 4; ++e) acc[e] = fmaf(p, vv[e], acc[e]);
    }
    m = mn;
  }
  __shared__ float sm_m[4], sm_l[4], sm_y[4][128];
  if (lane == 0) { sm_m[warp] = m; sm_l[warp] = l; }
  if (dv) {
#pragma unroll
    for (int e = 0; e < 4; ++e) sm_y[warp][d0 + e] = acc[e];
  }
  __syncthreads();
  const float M = fmaxf(fmaxf(sm_m[0], sm_m[1]), fmaxf(sm_m[2], sm_m[3]));
  float wgt[4], L = 0.f;
#pragma unroll
  for (int u = 0; u < 4; ++u) {
    wgt[u] = (sm_m[u] == -INFINITY) ? 0.f : exp2f(sm_m[u] - M);
    L += wgt[u] * sm_l[u];
  }
  const int64_t o = (int64_t)b * w.rows + row;
  if (threadIdx.x == 0) { w.win_ml[o * 2] = M; w.win_ml[o * 2 + 1] = L; }
  for (int d = threadIdx.x; d < w.d_h; d += 128) {
    float y = 0.f;
#pragma unroll
    for (int u = 0; u < 4; ++u) y += wgt[u] * sm_y[u][d];
    w.win_y[o * w.d_h + d] = y;
  }
}

// ---------------------------------------------------------------- merge --
// Combine split partials and the window partial of each (sequence, row) for
// head-space partials (LLA reconstruct):
//   M = max_s m_s, w_s = 2^(m_s - M), l = sum_s w_s l_s + w_w l_w,
//   o = (sum_s w_s y_s + w_w y_w) / l
__global__ void __launch_bounds__(128) merge_plain(MergeArgs g) {
  const int row = blockIdx.x, b = blockIdx.y;
  const int64_t br = (int64_t)b * g.rows + row;
  float M = g.win_ml[br * 2];
  for (int s = 0; s < g.S; ++s) M = fmaxf(M, g.part_ml[((int64_t)s * g.B * g.rows + br) * 2]);
  const float ww = exp2f(g.win_ml[br * 2] - M);
  float L = ww * g.win_ml[br * 2 + 1];
  for (int s = 0; s < g.S; ++s) {
    const float ms = g.part_ml[((int64_t)s * g.B * g.rows + br) * 2];
    if (ms == -INFINITY) continue;
    L += exp2f(ms - M) * g.part_ml[((int64_t)s * g.B * g.rows + br) * 2 + 1];
  }
  const float li = 1.f / L;
  for (int d = threadIdx.x; d < g.d_h; d += blockDim.x) {
    float y = ww * g.win_y[br * g.d_h + d];
    for (int s = 0; s < g.S; ++s) {
      const float ms = g.part_ml[((int64_t)s * g.B * g.rows + br) * 2];
      if (ms == -INFINITY) continue;
      y = fmaf(exp2f(ms - M), g.part_y[((int64_t)s * g.B * g.rows + br) * g.d_h + d], y);
    }
    g.out[(int64_t)b * g.outs_b + (int64_t)row * g.d_h + d] = (g.err && *g.err) ? NAN : y * li;
  }
}

// ------------------------------------------- LLA reconstruct, SIMT --
// One CTA per (split, row = (loop, head), sequence).  For every latent tile
// the CTA rebuilds k^_j = U^K c^K_j and v^_j = U^V c^V_j in registers (8
// threads per token, each owning d = g, g+8, ...), scores them against q and
// accumulates sum_j p_j v^_j without writing rebuilt vectors anywhere.
constexpr int RT = 32;   // tokens per tile
constexpr int RKD = 16;  // d_h <= 128 -> 16 values per thread

__global__ void __launch_bounds__(256) recon_split_simt(ReconArgs a) {
  extern __shared__ float sm[];
  const int s = blockIdx.x, row = blockIdx.y, b = blockIdx.z;
  const int tt = row / a.H, h = row % a.H;
  const int r = a.r, dh = a.d_h;
  const int LDC = r + 1;
  float* UKt = sm;                 // [r][dh]  UKt[c][d] = U^K[d][c]
  float* UVt = UKt + r * dh;       // [r][dh]
  float* qsh = UVt + r * dh;       // [dh]
  float* cks = qsh + dh;           // [RT][LDC]
  float* cvs = cks + RT * LDC;     // [RT][LDC]
  float* red = cvs + RT * LDC;     // [8] per-warp scratch
  float* accs = red + 16;          // [8][dh] final reduction
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int tok = tid / 8, g = tid % 8;
  const float* UKg = a.UK + ((int64_t)(tt * a.H + h) * dh) * r;
  const float* UVg = a.UV + ((int64_t)(tt * a.H + h) * dh) * r;
  for (int idx = tid; idx < r * dh; idx += 256) {
    const int d = idx / r, c = idx % r;
    UKt[c * dh + d] = UKg[idx];
    UVt[c * dh + d] = UVg[idx];
  }
  for (int d = tid; d < dh; d += 256) qsh[d] = a.q[(int64_t)b * a.qs_b + (int64_t)row * dh + d] * a.qmul;
  const int tok0 = s * a.tps, tok1 = min(a.n_lat, tok0 + a.tps);
  float acc[RKD];
#pragma unroll
  for (int k = 0; k < RKD; ++k) acc[k] = 0.f;
  float m = -INFINITY, l = 0.f;
  const int nd = ceil_div(dh, 8);
  __syncthreads();
  for (int j0 = tok0; j0 < tok1; j0 += RT) {
    const int nt = min(RT, tok1 - j0);
    for (int idx = tid; idx < nt * r; idx += 256) {
      const int i = idx / r, c = idx % r;
      const int64_t src = (int64_t)b * a.ls_b + (int64_t)h * a.ls_h + (int64_t)(j0 + i) * r + c;
      cks[i * LDC + c] = load_elem(a.cK, src, a.lat_dtype);
      cvs[i * LDC + c] = load_elem(a.cV, src, a.lat_dtype);
    }
    __syncthreads();
    float kh[RKD], vh[RKD];
#pragma unroll
    for (int k = 0; k < RKD; ++k) kh[k] = vh[k] = 0.f;
    if (tok < nt) {
      for (int c = 0; c < r; ++c) {
        const float ck = cks[tok * LDC + c], cv = cvs[tok * LDC + c];
#pragma unroll
        for (int k = 0; k < RKD; ++k) {
          if (k >= nd) break;
          const int d = g + 8 * k;
          if (d < dh) {
            kh[k] = fmaf(UKt[c * dh + d], ck, kh[k]);
            vh[k] = fmaf(UVt[c * dh + d], cv, vh[k]);
          }
        }
      }
    }
    float sp = 0.f;
#pragma unroll
    for (int k = 0; k < RKD; ++k) {
      const int d = g + 8 * k;
      if (k < nd && d < dh) sp = fmaf(qsh[d], kh[k], sp);
    }
    sp += __shfl_xor_sync(0xffffffffu, sp, 1);
    sp += __shfl_xor_sync(0xffffffffu, sp, 2);
    sp += __shfl_xor_sync(0xffffffffu, sp, 4);
    const float sc = tok < nt ? sp : -INFINITY;
    const float wm = warp_max(sc);
    if (lane == 0) red[warp] = wm;
    __syncthreads();
    float tmax = red[0];
    for (int u = 1; u < 8; ++u) tmax = fmaxf(tmax, red[u]);
    const float mn = fmaxf(m, tmax);
    const float al = (m == -INFINITY) ? 0.f : exp2f(m - mn);
    const float p = tok < nt ? exp2f(sc - mn) : 0.f;
    const float wsum = warp_sum(g == 0 ? p : 0.f);
    __syncthreads();
    if (lane == 0) red[warp] = wsum;
    __syncthreads();
    float psum = 0.f;
    for (int u = 0; u < 8; ++u) psum += red[u];
    l = l * al + psum;
    m = mn;
#pragma unroll
    for (int k = 0; k < RKD; ++k) acc[k] = fmaf(p, vh[k], acc[k] * al);
    __syncthreads();
  }
  // sum acc over the 32 tokens: 4 per warp (lanes g, g+8, g+16, g+24) then 8 warps
#pragma unroll
  for (int k = 0; k < RKD; ++k) {
    acc[k] += __shfl_xor_sync(0xffffffffu, acc[k], 8);
    acc[k] += __shfl_xor_sync(0xffffffffu, acc[k], 16);
  }
  if (lane < 8) {
#pragma unroll
    for (int k = 0; k < RKD; ++k) {
      const int d = lane + 8 * k;
      if (k < nd && d < dh) accs[warp * dh + d] = acc[k];
    }
  }
  __syncthreads();
  const int64_t o = ((int64_t)s * a.B + b) * a.rows + row;
  if (tid == 0) { a.part_ml[o * 2] = m; a.part_ml[o * 2 + 1] = l; }
  for (int d = tid; d < dh; d += 256) {
    float y = 0.f;
    for (int u = 0; u < 8; ++u) y += accs[u * dh + d];
    a.part_y[o * dh + d] = y;
  }
}

}  // namespace

static size_t absorb_simt_smem(const AbsorbArgs& a) {
  const int R = a.r_k + a.r_v;
  const int LD = R + ((33 - (R % 32)) % 32);
  return sizeof(float) * ((size_t)RB * a.r_k + (size_t)TT * LD + RB * TT + 3 * RB);
}

cudaError_t launch_absorb_split_simt(const AbsorbArgs& a, cudaStream_t st) {
  const size_t smem = absorb_simt_smem(a);
  cudaError_t e = cudaFuncSetAttribute(absorb_split_simt, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  dim3 grid(a.S, a.B, ceil_div(a.rows, RB));
  absorb_split_simt<<<grid, 256, smem, st>>>(a);
  return cudaGetLastError();
}

cudaError_t launch_window(const WindowArgs& w, cudaStream_t st) {
  dim3 grid(w.rows, w.B);
  if (w.dtype == LLA_BF16)
    window_attn<true><<<grid, 128, 0, st>>>(w);
  else
    window_attn<false><<<grid, 128, 0, st>>>(w);
  return cudaGetLastError();
}

cudaError_t launch_merge(const MergeArgs& g, cudaStream_t st) {
  dim3 grid(g.rows, g.B);
  merge_plain<<<grid, 128, 0, st>>>(g);
  return cudaGetLastError();
}

cudaError_t launch_recon_split_simt(const ReconArgs& a, cudaStream_t st) {
  const size_t smem = sizeof(float) *
      (2 * (size_t)a.r * a.d_h + a.d_h + 2 * (size_t)RT * (a.r + 1) + 16 + 8 * (size_t)a.d_h);
  cudaError_t e = cudaFuncSetAttribute(recon_split_simt, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  dim3 grid(a.S, a.rows, a.B);
  recon_split_simt<<<grid, 256, smem, st>>>(a);
  return cudaGetLastError();
}

}  // namespace lla
