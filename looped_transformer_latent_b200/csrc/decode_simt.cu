// SIMT kernels of the decode path: query prologue (A^T q with rotation),
// split-context absorbed latent read (fp32 and bf16 latents), LLA
// reconstruct-on-read, exact-window attention, and the split merge with the
// B_t^T map back to head space.  Scores are kept in base-2 units: every query
// is pre-multiplied by scale * log2(e) so the softmax uses exp2.
#include <algorithm>
#include <cmath>

#include "kernels.cuh"
#include "tc_ptx.cuh"
#include "tmap.cuh"

namespace lla {
namespace {

// ------------------------------------------------- absorbed split, SIMT --
// One CTA per (split, sequence, block of RB query rows).  A tile of TT latent
// tokens is staged in shared memory (fp32), scores for RB x TT pairs are one
// per thread, the online softmax runs per half-warp (one row), and every
// thread accumulates y~[row][v] = sum_j p_j c^V_j for its v columns.
constexpr int RB = 16, TT = 16, VC = 4;  // r_v <= 1024

__global__ void __launch_bounds__(256) absorb_split_simt(AbsorbArgs a) {
  griddep_wait();
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
  griddep_launch();
}

// --------------------------------------------------------------- window --
// Exact attention over the window ring (eq. 4, second term) as partial
// softmax states.  One CTA per (token chunk, loop, sequence) covers every
// head: warp w takes heads w, w+8, ..., so at any moment the CTA's warps read
// neighbouring heads of the same tokens and each token's ring row [H][d_h] is
// fetched as one contiguous block.  Each lane holds 4 consecutive elements of
// the head dimension; a warp issues all K and V loads of WU tokens before
// using them.  The query is rotated here (R_i in head space, when asked) and
// scaled into base-2 units.  Emits (max, sum, y_w) per (chunk, sequence, row).
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

// WU tokens per group: the full group for long windows, 4 for windows of a
// few tokens (fewer registers, so more CTAs per SM).
template <bool BF16, int WU, int MINB>
__global__ void __launch_bounds__(256, MINB) window_part(WindowArgs w) {
  griddep_wait();
  typedef WinTraits<BF16> Tr;
  const int chunk = blockIdx.x, tt = blockIdx.y, b = blockIdx.z;
  const int t = w.t0 + tt;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int d0 = 4 * lane;
  const bool dv = d0 < w.d_h;
  const int j0 = chunk * w.cpt, j1 = min(w.n_win, j0 + w.cpt);
  // the pairs' angles are the same for every head (computed once per call)
  float c0 = 1.f, s0 = 0.f, c1 = 1.f, s1 = 0.f;
  if (w.rotate && dv) {
    c0 = w.rot[2 * lane].x; s0 = w.rot[2 * lane].y;
    c1 = w.rot[2 * lane + 1].x; s1 = w.rot[2 * lane + 1].y;
  }
  const int64_t seq = (int64_t)b * w.wins_b;
  for (int h = warp; h < w.H; h += 8) {
    const int row = w.row0 + tt * w.H + h;
    float qv[4] = {0.f, 0.f, 0.f, 0.f}, acc[4] = {0.f, 0.f, 0.f, 0.f};
    if (dv) {
      const float* q = w.q + (int64_t)b * w.q_sb + (int64_t)row * w.q_srow + d0;
      const float x0 = q[0], y0 = q[1], x1 = q[2], y1 = q[3];
      qv[0] = (x0 * c0 - y0 * s0) * w.qmul;
      qv[1] = (x0 * s0 + y0 * c0) * w.qmul;
      qv[2] = (x1 * c1 - y1 * s1) * w.qmul;
      qv[3] = (x1 * s1 + y1 * c1) * w.qmul;
    }
    float m = -INFINITY, l = 0.f;
    for (int g0 = j0; g0 < j1; g0 += WU) {
      typename Tr::raw_t kr[WU], vr[WU];
#pragma unroll
      for (int u = 0; u < WU; ++u) {
        const int idx = g0 + u;
        if (dv && idx < j1) {
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
        if (g0 + u < j1) gm = fmaxf(gm, sc[u]);
      const float mn = fmaxf(m, gm);
      const float al = (m == -INFINITY) ? 0.f : exp2f(m - mn);
      l *= al;
#pragma unroll
      for (int e = 0; e < 4; ++e) acc[e] *= al;
#pragma unroll
      for (int u = 0; u < WU; ++u) {
        if (g0 + u >= j1) break;
        const float p = exp2f(sc[u] - mn);
        float vv[4];
        Tr::unpack(vr[u], vv);
        l += p;
#pragma unroll
        for (int e = 0; e < 4; ++e) acc[e] = fmaf(p, vv[e], acc[e]);
      }
      m = mn;
    }
    const int64_t o = ((int64_t)chunk * w.B + b) * w.rows_total + row;
    if (lane == 0) {
      w.win_ml[o * 2] = m;
      w.win_ml[o * 2 + 1] = l;
    }
    if (dv) {
#pragma unroll
      for (int e = 0; e < 4; ++e) w.win_y[o * w.d_h + d0 + e] = acc[e];
    }
  }
  griddep_launch();
}

// Large windows: the same partial states, with the ring rows staged in shared
// memory by bulk copies (the TMA engine) instead of registers.  One CTA per
// (token chunk, loop x group of 8 heads, sequence), one warp per head.  A
// token's slice for the head group is contiguous in the ring (heads are
// adjacent), so each token costs one bulk copy for K and one for V; stages of
// WB_TS tokens go through a WB_NST-deep ring, so a CTA keeps up to WB_NST
// stages in flight while its warps reduce the previous one from shared memory.
constexpr int WB_HEADS = 8;
constexpr int WB_NST = 3;
constexpr long long WB_WAIT = 1ll << 32;

template <bool BF16>
struct WbTraits { static constexpr int TS = BF16 ? 8 : 4; };

// Ring tensor maps: 5-D view (feature, head, slot, loop, sequence), boxes of
// d_h x 8 heads x TS slots -- one copy lands a stage's K (or V) block in the
// [slot][head][feature] order the warps read.
struct RingMaps {
  CUtensorMap k, v;
};

template <bool BF16>
__global__ void __launch_bounds__(32 * WB_HEADS) window_bulk(const __grid_constant__ RingMaps maps, WindowArgs w) {
  griddep_wait();
  typedef WinTraits<BF16> Tr;
  constexpr int TS = WbTraits<BF16>::TS;
  constexpr int ES = BF16 ? 2 : 4;
  extern __shared__ __align__(128) uint8_t wsm[];
  const int chunk = blockIdx.x, tt = blockIdx.y / w.HG, hg = blockIdx.y % w.HG, b = blockIdx.z;
  const int t = w.t0 + tt, h0 = hg * WB_HEADS;
  const int nh = min(WB_HEADS, w.H - h0);
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const uint32_t hbytes = (uint32_t)w.d_h * ES;
  const uint32_t tok_bytes = nh * hbytes;                         // one token's head-group slice
  const uint32_t half = (uint32_t)TS * WB_HEADS * hbytes;          // K (or V) part of a stage
  uint64_t* full = reinterpret_cast<uint64_t*>(wsm + WB_NST * 2 * half);
  const int j0 = chunk * w.cpt, j1 = min(w.n_win, j0 + w.cpt);
  const int nsub = (j1 - j0 + TS - 1) / TS;
  // the copy thread (warp 1, lane 0) sets up the barriers and issues the
  // first stages before the block barrier
  const bool copier = threadIdx.x == 32;
  const char* kbase = reinterpret_cast<const char*>(w.wk) + ((int64_t)b * w.wins_b) * ES;
  const char* vbase = reinterpret_cast<const char*>(w.wv) + ((int64_t)b * w.wins_b) * ES;
  auto issue = [&](int i) {        // sub-chunk i into stage i % WB_NST (thread 0)
    const int st = i % WB_NST;
    const int jj = j0 + i * TS, nt = min(TS, j1 - jj);
    const uint32_t bar = ptx::smem_u32(&full[st]);
    const uint32_t dk = ptx::smem_u32(wsm + st * 2 * half), dv = dk + half;
    const int s0 = (w.win_start + jj) % w.Wcap;
    if (s0 + nt <= w.Wcap) {
      // the stage's slots are consecutive in the ring: one box each for K and V
      ptx::mbar_arrive_tx(bar, 2u * half);
      ptx::tma_load_5d(dk, &maps.k, bar, 0, h0, s0, t, b);
      ptx::tma_load_5d(dv, &maps.v, bar, 0, h0, s0, t, b);
    } else {
      // the stage wraps around the ring's end: one copy per token
      ptx::mbar_arrive_tx(bar, 2u * nt * tok_bytes);
      for (int u = 0; u < nt; ++u) {
        const int slot = (w.win_start + jj + u) % w.Wcap;
        const int64_t off = (((int64_t)t * w.Wcap + slot) * w.H + h0) * (int64_t)hbytes;
        ptx::bulk_load(dk + u * WB_HEADS * hbytes, kbase + off, tok_bytes, bar);
        ptx::bulk_load(dv + u * WB_HEADS * hbytes, vbase + off, tok_bytes, bar);
      }
    }
  };
  if (copier) {
    for (int i = 0; i < WB_NST; ++i) ptx::mbar_init(ptx::smem_u32(&full[i]), 1);
    ptx::fence_mbar_init();
    for (int i = 0; i < WB_NST && i < nsub; ++i) issue(i);
  }
  __syncthreads();

  const int d0 = 4 * lane;
  const bool dv = warp < nh && d0 < w.d_h;
  const int row = w.row0 + tt * w.H + h0 + warp;
  float c0 = 1.f, s0 = 0.f, c1 = 1.f, s1 = 0.f;
  if (w.rotate && dv) {
    c0 = w.rot[2 * lane].x; s0 = w.rot[2 * lane].y;
    c1 = w.rot[2 * lane + 1].x; s1 = w.rot[2 * lane + 1].y;
  }
  float qv[4] = {0.f, 0.f, 0.f, 0.f}, acc[4] = {0.f, 0.f, 0.f, 0.f};
  if (dv) {
    const float* q = w.q + (int64_t)b * w.q_sb + (int64_t)row * w.q_srow + d0;
    const float x0 = q[0], y0 = q[1], x1 = q[2], y1 = q[3];
    qv[0] = (x0 * c0 - y0 * s0) * w.qmul;
    qv[1] = (x0 * s0 + y0 * c0) * w.qmul;
    qv[2] = (x1 * c1 - y1 * s1) * w.qmul;
    qv[3] = (x1 * s1 + y1 * c1) * w.qmul;
  }
  float m = -INFINITY, l = 0.f;
  int failed_at = -1;
  for (int i = 0; i < nsub; ++i) {
    const int st = i % WB_NST;
    const uint32_t bar = ptx::smem_u32(&full[st]);
    const uint32_t par = (uint32_t)(i / WB_NST) & 1u;
    bool ok = ptx::mbar_try_wait(bar, par);
    if (!ok) {
      const long long t0c = clock64();
      while (!(ok = ptx::mbar_try_wait(bar, par)) && clock64() - t0c <= WB_WAIT) {
      }
    }
    // every thread leaves together, so no warp is left at a barrier
    if (__syncthreads_or(!ok)) {
      failed_at = i;
      break;
    }
    const int jj = j0 + i * TS, nt = min(TS, j1 - jj);
    const uint8_t* ks = wsm + st * 2 * half + (size_t)warp * hbytes + (size_t)d0 * ES;
    const uint8_t* vs = ks + half;
    float sc[TS];
    typename Tr::raw_t vr[TS];
#pragma unroll
    for (int u = 0; u < TS; ++u) {
      float kk[4];
      typename Tr::raw_t kr = Tr::zero();
      vr[u] = Tr::zero();
      if (dv && u < nt) {
        kr = *reinterpret_cast<const typename Tr::raw_t*>(ks + (size_t)u * WB_HEADS * hbytes);
        vr[u] = *reinterpret_cast<const typename Tr::raw_t*>(vs + (size_t)u * WB_HEADS * hbytes);
      }
      Tr::unpack(kr, kk);
      float part = 0.f;
#pragma unroll
      for (int e = 0; e < 4; ++e) part = fmaf(qv[e], kk[e], part);
      sc[u] = part;
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1)
#pragma unroll
      for (int u = 0; u < TS; ++u) sc[u] += __shfl_xor_sync(0xffffffffu, sc[u], o);
    float gm = -INFINITY;
#pragma unroll
    for (int u = 0; u < TS; ++u)
      if (u < nt) gm = fmaxf(gm, sc[u]);
    const float mn = fmaxf(m, gm);
    const float al = (m == -INFINITY) ? 0.f : exp2f(m - mn);
    l *= al;
#pragma unroll
    for (int e = 0; e < 4; ++e) acc[e] *= al;
#pragma unroll
    for (int u = 0; u < TS; ++u) {
      if (u >= nt) break;
      const float p = exp2f(sc[u] - mn);
      float vv[4];
      Tr::unpack(vr[u], vv);
      l += p;
#pragma unroll
      for (int e = 0; e < 4; ++e) acc[e] = fmaf(p, vv[e], acc[e]);
    }
    m = mn;
    __syncthreads();   // every warp is done with this stage
    if (copier && i + WB_NST < nsub) issue(i + WB_NST);
  }
  if (failed_at >= 0) {
    if (copier) {
      if (w.err) atomicExch(w.err, ERR_WINDOW_TIMEOUT);
      // leave no copy in flight: wait (bounded) for the stages still owed
      for (int i = failed_at; i < nsub && i < failed_at + WB_NST; ++i) {
        const uint32_t bar = ptx::smem_u32(&full[i % WB_NST]);
        const long long t0c = clock64();
        while (!ptx::mbar_try_wait(bar, (uint32_t)(i / WB_NST) & 1u) && clock64() - t0c < WB_WAIT) {
        }
      }
    }
    return;
  }
  if (warp < nh) {
    const int64_t o = ((int64_t)chunk * w.B + b) * w.rows_total + row;
    if (lane == 0) {
      w.win_ml[o * 2] = m;
      w.win_ml[o * 2 + 1] = l;
    }
    if (dv) {
#pragma unroll
      for (int e = 0; e < 4; ++e) w.win_y[o * w.d_h + d0 + e] = acc[e];
    }
  }
  griddep_launch();
}

// Windows of 16 tokens and more, in chunks of at most WC_TOK tokens: one CTA
// per (chunk, loop x group of 8 heads, sequence) lands its whole chunk with
// one pair of TMA boxes (per-token bulk copies where the chunk wraps around
// the ring's end), one warp per head.  Lanes hold 4 features each: a lane's
// partial dot products for the chunk's tokens are summed across the warp by a
// transposing butterfly (each exchange halves the values a lane holds, so the
// whole chunk takes WC_TOK shuffles instead of 5 per token), which leaves
// token u's score in lanes u * (32 / WC_TOK) ..; the values are then
// accumulated with each token's weight broadcast from its lane.  One tile, so
// the partial state is the chunk's own maximum, sum and weighted values.
template <bool BF16>
struct WcTraits { static constexpr int TOK = BF16 ? 16 : 8; };

// v[u] (u < N) summed over the warp's 32 lanes; lane l receives the total of
// v[l / (32 / N)].
template <int N>
__device__ __forceinline__ float butterfly_transpose_sum(float (&v)[N], int lane) {
  int steps = 0;
#pragma unroll
  for (int half = N / 2; half >= 1; half /= 2, ++steps) {
    const int mask = 16 >> steps;
    const bool up = (lane & mask) != 0;
#pragma unroll
    for (int i = 0; i < half; ++i) {
      const float lo = v[i], hi = v[i + half];
      v[i] = (up ? hi : lo) + __shfl_xor_sync(0xffffffffu, up ? lo : hi, mask);
    }
  }
  float s = v[0];
#pragma unroll
  for (int o = 16 / N; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
  return s;
}

template <bool BF16>
__global__ void __launch_bounds__(32 * WB_HEADS) window_chunk(const __grid_constant__ RingMaps maps, WindowArgs w) {
  griddep_wait();
  typedef WinTraits<BF16> Tr;
  constexpr int TC = WcTraits<BF16>::TOK;
  constexpr int G = 32 / TC;   // lanes holding one token's score
  constexpr int ES = BF16 ? 2 : 4;
  extern __shared__ __align__(128) uint8_t wsm[];
  const int chunk = blockIdx.x, tt = blockIdx.y / w.HG, hg = blockIdx.y % w.HG, b = blockIdx.z;
  const int t = w.t0 + tt, h0 = hg * WB_HEADS;
  const int nh = min(WB_HEADS, w.H - h0);
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const uint32_t hbytes = (uint32_t)w.d_h * ES;
  const uint32_t tok_bytes = nh * hbytes;                  // one token's head-group slice
  const uint32_t half = (uint32_t)w.cpt * WB_HEADS * hbytes;
  uint64_t* full = reinterpret_cast<uint64_t*>(wsm + 2 * half);
  const int j0 = chunk * w.cpt, nt = min(w.n_win, j0 + w.cpt) - j0;
  if (threadIdx.x == 0) {
    const uint32_t bar = ptx::smem_u32(full);
    ptx::mbar_init(bar, 1);
    ptx::fence_mbar_init();
    const uint32_t dk = ptx::smem_u32(wsm), dv = dk + half;
    const int s0 = (w.win_start + j0) % w.Wcap;
    if (s0 + nt <= w.Wcap) {
      // consecutive ring slots: one box each for K and V (slots past the
      // chunk, or past the ring's end, land too and are never read)
      ptx::mbar_arrive_tx(bar, 2u * half);
      ptx::tma_load_5d(dk, &maps.k, bar, 0, h0, s0, t, b);
      ptx::tma_load_5d(dv, &maps.v, bar, 0, h0, s0, t, b);
    } else {
      const char* kbase = reinterpret_cast<const char*>(w.wk) + ((int64_t)b * w.wins_b) * ES;
      const char* vbase = reinterpret_cast<const char*>(w.wv) + ((int64_t)b * w.wins_b) * ES;
      ptx::mbar_arrive_tx(bar, 2u * nt * tok_bytes);
      for (int u = 0; u < nt; ++u) {
        const int slot = (w.win_start + j0 + u) % w.Wcap;
        const int64_t off = (((int64_t)t * w.Wcap + slot) * w.H + h0) * (int64_t)hbytes;
        ptx::bulk_load(dk + u * WB_HEADS * hbytes, kbase + off, tok_bytes, bar);
        ptx::bulk_load(dv + u * WB_HEADS * hbytes, vbase + off, tok_bytes, bar);
      }
    }
  }
  __syncthreads();

  // the rotated, scaled query while the copies are in flight
  const int d0 = 4 * lane;
  const bool dv = warp < nh && d0 < w.d_h;
  const int row = w.row0 + tt * w.H + h0 + warp;
  float qv[4] = {0.f, 0.f, 0.f, 0.f};
  if (dv) {
    float c0 = 1.f, s0 = 0.f, c1 = 1.f, s1 = 0.f;
    if (w.rotate) {
      c0 = w.rot[2 * lane].x; s0 = w.rot[2 * lane].y;
      c1 = w.rot[2 * lane + 1].x; s1 = w.rot[2 * lane + 1].y;
    }
    const float* q = w.q + (int64_t)b * w.q_sb + (int64_t)row * w.q_srow + d0;
    const float x0 = q[0], y0 = q[1], x1 = q[2], y1 = q[3];
    qv[0] = (x0 * c0 - y0 * s0) * w.qmul;
    qv[1] = (x0 * s0 + y0 * c0) * w.qmul;
    qv[2] = (x1 * c1 - y1 * s1) * w.qmul;
    qv[3] = (x1 * s1 + y1 * c1) * w.qmul;
  }
  const uint32_t bar = ptx::smem_u32(full);
  bool ok = ptx::mbar_try_wait(bar, 0);
  if (!ok) {
    const long long t0c = clock64();
    while (!(ok = ptx::mbar_try_wait(bar, 0)) && clock64() - t0c <= WB_WAIT) {
    }
  }
  if (__syncthreads_or(!ok)) {
    if (threadIdx.x == 0) {
      if (w.err) atomicExch(w.err, ERR_WINDOW_TIMEOUT);
      // leave no copy in flight: wait (bounded) once more for the chunk
      const long long t0c = clock64();
      while (!ptx::mbar_try_wait(bar, 0) && clock64() - t0c < WB_WAIT) {
      }
    }
    return;
  }
  if (warp >= nh) return;
  const uint8_t* ks = wsm + (size_t)warp * hbytes + (size_t)d0 * ES;
  const uint8_t* vs = ks + half;
  float part[TC];
#pragma unroll
  for (int u = 0; u < TC; ++u) {
    part[u] = 0.f;
    if (dv && u < nt) {
      float kk[4];
      Tr::unpack(*reinterpret_cast<const typename Tr::raw_t*>(ks + (size_t)u * WB_HEADS * hbytes), kk);
#pragma unroll
      for (int e = 0; e < 4; ++e) part[u] = fmaf(qv[e], kk[e], part[u]);
    }
  }
  const int tok = lane / G;
  float sc = butterfly_transpose_sum<TC>(part, lane);
  if (tok >= nt) sc = -INFINITY;
  const float m = ptx::redux_max(sc);
  const float p = tok < nt ? exp2f(sc - m) : 0.f;
  float l = (lane % G) == 0 ? p : 0.f;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) l += __shfl_xor_sync(0xffffffffu, l, o);
  float acc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
  for (int u = 0; u < TC; ++u) {
    const float pu = __shfl_sync(0xffffffffu, p, u * G);
    if (dv && u < nt) {
      float vv[4];
      Tr::unpack(*reinterpret_cast<const typename Tr::raw_t*>(vs + (size_t)u * WB_HEADS * hbytes), vv);
#pragma unroll
      for (int e = 0; e < 4; ++e) acc[e] = fmaf(pu, vv[e], acc[e]);
    }
  }
  const int64_t o = ((int64_t)chunk * w.B + b) * w.rows_total + row;
  if (lane == 0) {
    w.win_ml[o * 2] = m;
    w.win_ml[o * 2 + 1] = l;
  }
  if (dv) {
#pragma unroll
    for (int e = 0; e < 4; ++e) w.win_y[o * w.d_h + d0 + e] = acc[e];
  }
  griddep_launch();
}

// ---------------------------------------------------------------- merge --
// Combine split partials and the window partial of each (sequence, row) for
// head-space partials (LLA reconstruct):
//   M = max_s m_s, w_s = 2^(m_s - M), l = sum_s w_s l_s + w_w l_w,
//   o = (sum_s w_s y_s + w_w y_w) / l
__global__ void __launch_bounds__(128) merge_plain(MergeArgs g) {
  griddep_wait();
  const int row = blockIdx.x, b = blockIdx.y;
  const int64_t br = (int64_t)b * g.rows + row;
  const int64_t bstride = (int64_t)g.B * g.rows;   // between partials of consecutive splits / chunks
  float M = -INFINITY;
  for (int c = 0; c < g.Sw; ++c) M = fmaxf(M, g.win_ml[(c * bstride + br) * 2]);
  for (int s = 0; s < g.S; ++s) M = fmaxf(M, g.part_ml[(s * bstride + br) * 2]);
  float L = 0.f;
  for (int c = 0; c < g.Sw; ++c) {
    const float mc = g.win_ml[(c * bstride + br) * 2];
    if (mc != -INFINITY) L += exp2f(mc - M) * g.win_ml[(c * bstride + br) * 2 + 1];
  }
  for (int s = 0; s < g.S; ++s) {
    const float ms = g.part_ml[(s * bstride + br) * 2];
    if (ms != -INFINITY) L += exp2f(ms - M) * g.part_ml[(s * bstride + br) * 2 + 1];
  }
  const float li = 1.f / L;
  for (int d = threadIdx.x; d < g.d_h; d += blockDim.x) {
    float y = 0.f;
    for (int c = 0; c < g.Sw; ++c) {
      const float mc = g.win_ml[(c * bstride + br) * 2];
      if (mc != -INFINITY) y = fmaf(exp2f(mc - M), g.win_y[(c * bstride + br) * g.d_h + d], y);
    }
    for (int s = 0; s < g.S; ++s) {
      const float ms = g.part_ml[(s * bstride + br) * 2];
      if (ms != -INFINITY) y = fmaf(exp2f(ms - M), g.part_y[(s * bstride + br) * g.d_h + d], y);
    }
    g.out[(int64_t)b * g.outs_b + (int64_t)row * g.d_h + d] = (g.err && *g.err) ? NAN : y * li;
  }
  griddep_launch();
}

// ------------------------------------------- LLA reconstruct, SIMT --
// One CTA per (split, row = (loop, head), sequence).  For every latent tile
// the CTA rebuilds k^_j = U^K c^K_j and v^_j = U^V c^V_j in registers (8
// threads per token, each owning d = g, g+8, ...), scores them against q and
// accumulates sum_j p_j v^_j without writing rebuilt vectors anywhere.
constexpr int RT = 32;   // tokens per tile
constexpr int RKD = 16;  // d_h <= 128 -> 16 values per thread

__global__ void __launch_bounds__(256) recon_split_simt(ReconArgs a) {
  griddep_wait();
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
  griddep_launch();
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
  return launch_kernel(absorb_split_simt, grid, dim3(256), smem, st, 1, a);
}

bool window_bulk_ok(int dtype, int d_h) {
  const int es = dtype == LLA_BF16 ? 2 : 4;
  return (d_h * es) % 16 == 0;
}

int window_chunks(int B, int nt, int H, int n_win, int dtype, int d_h, int num_sms, int* cpt, int* HG) {
  // Windows of at least 16 tokens use the bulk-copy kernels (groups of 8 heads
  // per CTA): chunks of at most WC_TOK tokens, one tile each (window_chunk),
  // when that takes at most kMaxWindowChunks chunks; longer windows stream
  // chunks of a multiple of 8 tokens through window_bulk, about four CTAs per
  // SM.  Shorter windows use the register kernel.
  const bool bulk = n_win >= 16 && window_bulk_ok(dtype, d_h);
  *HG = bulk ? (H + WB_HEADS - 1) / WB_HEADS : 0;
  if (bulk) {
    const int tc = dtype == LLA_BF16 ? WcTraits<true>::TOK : WcTraits<false>::TOK;
    const int S = (n_win + tc - 1) / tc;
    if (S <= kMaxWindowChunks) {
      *cpt = (n_win + S - 1) / S;
      return (n_win + *cpt - 1) / *cpt;
    }
  }
  const long ctas = (long)B * nt * (bulk ? *HG : 1);
  long S = ctas > 0 ? (4L * num_sms + ctas - 1) / ctas : 1;
  S = std::max(1L, std::min(S, std::min((long)kMaxWindowChunks, (long)((n_win + 7) / 8))));
  int c = (int)((n_win + S - 1) / S);
  c = (c + 7) / 8 * 8;
  *cpt = c;
  return (n_win + c - 1) / c;
}

cudaError_t launch_window(const WindowArgs& w_in, cudaStream_t st) {
  if (w_in.n_win <= 0 || w_in.B == 0) return cudaSuccess;
  WindowArgs w = w_in;
  // R_pos of the query in head space: pair p at angle pos * base^(-2p / d_h)
  for (int p = 0; p < 64; ++p) {
    w.rot[p] = make_float2(1.f, 0.f);
    if (w.rotate && p < w.d_h / 2) {
      const double ang = (double)w.pos * std::pow(w.base, -2.0 * (double)p / (double)w.d_h);
      w.rot[p] = make_float2((float)std::cos(ang), (float)std::sin(ang));
    }
  }
  const int nt = w.rows / w.H;
  if (w.HG > 0) {
    const int es = w.dtype == LLA_BF16 ? 2 : 4;
    const int tc = w.dtype == LLA_BF16 ? WcTraits<true>::TOK : WcTraits<false>::TOK;
    const bool one_tile = w.cpt <= tc;   // window_chunk: the whole chunk in one tile
    const int ts = one_tile ? w.cpt : w.dtype == LLA_BF16 ? WbTraits<true>::TS : WbTraits<false>::TS;
    const size_t smem = one_tile ? (size_t)2 * ts * WB_HEADS * w.d_h * es + 16
                                 : (size_t)WB_NST * 2 * ts * WB_HEADS * w.d_h * es + 8 * WB_NST + 16;
    dim3 grid(w.Sw, nt * w.HG, w.B);
    RingMaps maps;
    TmapEncodeFn enc = tmap_encoder();
    bool mapped = enc != nullptr;
    const cuuint64_t dims[5] = {(cuuint64_t)w.d_h, (cuuint64_t)w.H, (cuuint64_t)w.Wcap, (cuuint64_t)(w.t0 + nt),
                                (cuuint64_t)w.B};
    const cuuint64_t hb = (cuuint64_t)w.d_h * es;
    const cuuint64_t strides[4] = {hb, hb * w.H, hb * w.H * w.Wcap, (cuuint64_t)w.wins_b * es};
    const cuuint32_t box[5] = {(cuuint32_t)w.d_h, WB_HEADS, (cuuint32_t)ts, 1, 1};
    const cuuint32_t estr[5] = {1, 1, 1, 1, 1};
    const CUtensorMapDataType dt = w.dtype == LLA_BF16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT32;
    for (int m = 0; m < 2 && mapped; ++m)
      mapped = enc(m == 0 ? &maps.k : &maps.v, dt, 5, const_cast<void*>(m == 0 ? w.wk : w.wv), dims, strides, box,
                   estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
    if (!mapped) goto register_kernel;   // no tensor-map view: same chunks on the register kernel
    cudaError_t e;
    if (one_tile) {
      if (w.dtype == LLA_BF16) {
        e = cudaFuncSetAttribute(window_chunk<true>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
        e = launch_kernel(window_chunk<true>, grid, dim3(32 * WB_HEADS), smem, st, 1, maps, w);
      } else {
        e = cudaFuncSetAttribute(window_chunk<false>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
        e = launch_kernel(window_chunk<false>, grid, dim3(32 * WB_HEADS), smem, st, 1, maps, w);
      }
    } else if (w.dtype == LLA_BF16) {
      e = cudaFuncSetAttribute(window_bulk<true>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
      if (e != cudaSuccess) return e;
      e = launch_kernel(window_bulk<true>, grid, dim3(32 * WB_HEADS), smem, st, 1, maps, w);
    } else {
      e = cudaFuncSetAttribute(window_bulk<false>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
      if (e != cudaSuccess) return e;
      e = launch_kernel(window_bulk<false>, grid, dim3(32 * WB_HEADS), smem, st, 1, maps, w);
    }
    return e;
  }
register_kernel:
  dim3 grid(w.Sw, nt, w.B);
  const bool small = w.cpt <= 8;
  if (w.dtype == LLA_BF16) {
    if (small) return launch_kernel(window_part<true, 4, 4>, grid, dim3(256), 0, st, 1, w);
    return launch_kernel(window_part<true, WinTraits<true>::WU, 1>, grid, dim3(256), 0, st, 1, w);
  }
  if (small) return launch_kernel(window_part<false, 4, 4>, grid, dim3(256), 0, st, 1, w);
  return launch_kernel(window_part<false, WinTraits<false>::WU, 1>, grid, dim3(256), 0, st, 1, w);
}

cudaError_t launch_merge(const MergeArgs& g, cudaStream_t st) {
  dim3 grid(g.rows, g.B);
  return launch_kernel(merge_plain, grid, dim3(128), 0, st, 1, g);
}

cudaError_t launch_recon_split_simt(const ReconArgs& a, cudaStream_t st) {
  const size_t smem = sizeof(float) *
      (2 * (size_t)a.r * a.d_h + a.d_h + 2 * (size_t)RT * (a.r + 1) + 16 + 8 * (size_t)a.d_h);
  cudaError_t e = cudaFuncSetAttribute(recon_split_simt, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  dim3 grid(a.S, a.rows, a.B);
  return launch_kernel(recon_split_simt, grid, dim3(256), smem, st, 1, a);
}

}  // namespace lla
