// SIMT kernels of the decode path: query prologue (A^T q with rotation),
// split-context absorbed latent read (fp32 and bf16 latents), LLA
// reconstruct-on-read, exact-window attention, and the split merge with the
// B_t^T map back to head space.  Scores are kept in base-2 units: every query
// is pre-multiplied by scale * log2(e) so the softmax uses exp2.
#include "kernels.cuh"

namespace lla {
namespace {

// ------------------------------------------------------------ prologue --
// q~[b][row] = scale*log2e * R~_i A_{t,h}^T q_{t,h}   (latent space, rank r_k)
// q_w[b][row] = scale*log2e * R_i q_{t,h}             (head space, exact tokens)
// Grid: x = pair chunks of 64 (+1 block for q_w), y = row, z = 32-sequence chunk.
constexpr int PRO_B = 32;

__global__ void __launch_bounds__(64) absorb_prologue(AbsorbArgs a) {
  extern __shared__ float qsm[];  // [PRO_B][d_h]
  const int row = blockIdx.y, tt = row / a.H, h = row % a.H;
  const int b0 = blockIdx.z * PRO_B;
  const int nb = min(PRO_B, a.B - b0);
  for (int idx = threadIdx.x; idx < PRO_B * a.d_h; idx += blockDim.x) {
    const int bb = idx / a.d_h, d = idx % a.d_h;
    qsm[idx] = bb < nb ? a.q[(int64_t)(b0 + bb) * a.qs_b + (int64_t)(tt * a.H + h) * a.d_h + d] : 0.f;
  }
  __syncthreads();
  const int i = a.N - 1;
  const int nchunks = ceil_div(a.r_k / 2, 64);
  if ((int)blockIdx.x < nchunks) {
    const int p = blockIdx.x * 64 + threadIdx.x;
    if (2 * p >= a.r_k) return;
    const float* Ar = a.A + ((int64_t)(tt * a.H + h) * a.d_h) * a.r_k + 2 * p;
    float acc0[PRO_B], acc1[PRO_B];
#pragma unroll
    for (int bb = 0; bb < PRO_B; ++bb) acc0[bb] = acc1[bb] = 0.f;
    for (int d = 0; d < a.d_h; ++d) {
      const float2 av = *reinterpret_cast<const float2*>(Ar + (int64_t)d * a.r_k);
#pragma unroll
      for (int bb = 0; bb < PRO_B; ++bb) {
        const float qv = qsm[bb * a.d_h + d];
        acc0[bb] = fmaf(av.x, qv, acc0[bb]);
        acc1[bb] = fmaf(av.y, qv, acc1[bb]);
      }
    }
    float c = 1.f, s = 0.f;
    if (a.rotate) rope_cs(p, a.r_k, a.d_h, a.base, (double)i, &c, &s);
#pragma unroll
    for (int bb = 0; bb < PRO_B; ++bb) {
      if (bb >= nb) break;
      const float x = acc0[bb], y = acc1[bb];
      float* dst = a.qlat + ((int64_t)(b0 + bb) * a.rows + row) * a.r_k + 2 * p;
      dst[0] = (x * c - y * s) * a.qmul;
      dst[1] = (x * s + y * c) * a.qmul;
    }
  } else {
    const int hp = a.d_h / 2;
    for (int idx = threadIdx.x; idx < nb * hp; idx += blockDim.x) {
      const int bb = idx / hp, p = idx % hp;
      float c = 1.f, s = 0.f;
      if (a.rotate) rope_cs(p, a.d_h, a.d_h, a.base, (double)i, &c, &s);
      const float x = qsm[bb * a.d_h + 2 * p], y = qsm[bb * a.d_h + 2 * p + 1];
      float* dst = a.qwin + ((int64_t)(b0 + bb) * a.rows + row) * a.d_h + 2 * p;
      dst[0] = (x * c - y * s) * a.qmul;
      dst[1] = (x * s + y * c) * a.qmul;
    }
  }
}

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
// Exact attention over the window ring for one (row, sequence): 4 warps split
// the tokens, lanes split the head dimension, one online softmax per warp,
// combined at the end.  Emits (max, sum, y_w) in base-2 units.
__global__ void __launch_bounds__(128) window_attn(WindowArgs w) {
  const int row = blockIdx.x, b = blockIdx.y;
  const int tt = row / w.H, h = row % w.H, t = w.t0 + tt;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  constexpr int KD = 4;  // d_h <= 128
  float qv[KD], acc[KD];
#pragma unroll
  for (int k = 0; k < KD; ++k) {
    const int d = lane + 32 * k;
    qv[k] = d < w.d_h ? w.q[(int64_t)b * w.q_sb + (int64_t)row * w.q_srow + d] * w.qmul : 0.f;
    acc[k] = 0.f;
  }
  float m = -INFINITY, l = 0.f;
  for (int idx = warp; idx < w.n_win; idx += 4) {
    const int j = w.win_start + idx;
    const int slot = j % w.Wcap;
    const int64_t base = (int64_t)b * w.wins_b + (((int64_t)t * w.Wcap + slot) * w.H + h) * w.d_h;
    float part = 0.f;
    float vv[KD];
#pragma unroll
    for (int k = 0; k < KD; ++k) {
      const int d = lane + 32 * k;
      float kk = 0.f;
      vv[k] = 0.f;
      if (d < w.d_h) {
        kk = load_elem(w.wk, base + d, w.dtype);
        vv[k] = load_elem(w.wv, base + d, w.dtype);
      }
      part = fmaf(qv[k], kk, part);
    }
    const float sc = warp_sum(part);
    const float mn = fmaxf(m, sc);
    const float al = (m == -INFINITY) ? 0.f : exp2f(m - mn);
    const float p = exp2f(sc - mn);
    l = l * al + p;
#pragma unroll
    for (int k = 0; k < KD; ++k) acc[k] = fmaf(p, vv[k], acc[k] * al);
    m = mn;
  }
  __shared__ float sm_m[4], sm_l[4], sm_y[4][128];
  if (lane == 0) { sm_m[warp] = m; sm_l[warp] = l; }
#pragma unroll
  for (int k = 0; k < KD; ++k) {
    const int d = lane + 32 * k;
    if (d < 128) sm_y[warp][d] = acc[k];
  }
  __syncthreads();
  float M = fmaxf(fmaxf(sm_m[0], sm_m[1]), fmaxf(sm_m[2], sm_m[3]));
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
// Combine split partials and the window partial of each (sequence, row):
//   M = max_s m_s, w_s = 2^(m_s - M), l = sum_s w_s l_s + w_w l_w,
//   o = (B_{t,h}^T sum_s w_s y~_s + w_w y_w) / l      (mapped)
//   o = (sum_s w_s y_s + w_w y_w) / l                 (head-space partials)
// Mapped variant: one CTA per (row, chunk of MB sequences) so each B_{t,h}
// is read once per chunk.
constexpr int MB = 16;

__global__ void __launch_bounds__(256) merge_mapped(MergeArgs g) {
  extern __shared__ float sm[];
  float* ybar = sm;                 // [MB][Y]
  float* wwin = ybar + MB * g.Y;    // [MB]
  float* linv = wwin + MB;          // [MB]
  float* red = linv + MB;           // [2][MB][128] partial map results
  const int row = blockIdx.x, b0 = blockIdx.y * MB;
  const int nb = min(MB, g.B - b0);
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  for (int bb = warp; bb < nb; bb += 8) {
    const int b = b0 + bb;
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
    for (int v = lane; v < g.Y; v += 32) {
      float y = 0.f;
      for (int s = 0; s < g.S; ++s) {
        const float ms = g.part_ml[((int64_t)s * g.B * g.rows + br) * 2];
        if (ms == -INFINITY) continue;
        y = fmaf(exp2f(ms - M), g.part_y[((int64_t)s * g.B * g.rows + br) * g.Y + v], y);
      }
      ybar[bb * g.Y + v] = y;
    }
    if (lane == 0) { wwin[bb] = ww; linv[bb] = 1.f / L; }
  }
  __syncthreads();
  // o[b][d] = sum_v Bm[row][v][d] * ybar[b][v]; thread = (d, half of v range)
  const int d = threadIdx.x % 128, half = threadIdx.x / 128;
  const float* Bmr = g.Bm + (int64_t)row * g.Y * g.d_h;
  if (d < g.d_h) {
    float acc[MB];
#pragma unroll
    for (int bb = 0; bb < MB; ++bb) acc[bb] = 0.f;
    const int vh = (g.Y + 1) / 2;
    const int v0 = half * vh, v1 = min(g.Y, v0 + vh);
    for (int v = v0; v < v1; ++v) {
      const float bm = __ldg(Bmr + (int64_t)v * g.d_h + d);
#pragma unroll
      for (int bb = 0; bb < MB; ++bb) acc[bb] = fmaf(bm, ybar[bb * g.Y + v], acc[bb]);
    }
#pragma unroll
    for (int bb = 0; bb < MB; ++bb) red[(half * MB + bb) * 128 + d] = acc[bb];
  }
  __syncthreads();
  for (int idx = threadIdx.x; idx < nb * g.d_h; idx += 256) {
    const int bb = idx / g.d_h, dd = idx % g.d_h;
    const int b = b0 + bb;
    const int64_t br = (int64_t)b * g.rows + row;
    const float v = red[bb * 128 + dd] + red[(MB + bb) * 128 + dd] + wwin[bb] * g.win_y[br * g.d_h + dd];
    g.out[(int64_t)b * g.outs_b + (int64_t)row * g.d_h + dd] = v * linv[bb];
  }
}

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
    g.out[(int64_t)b * g.outs_b + (int64_t)row * g.d_h + d] = y * li;
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

cudaError_t launch_absorb_prologue(const AbsorbArgs& a, cudaStream_t st) {
  dim3 grid(ceil_div(a.r_k / 2, 64) + 1, a.rows, ceil_div(a.B, PRO_B));
  const size_t smem = (size_t)PRO_B * a.d_h * sizeof(float);
  absorb_prologue<<<grid, 64, smem, st>>>(a);
  return cudaGetLastError();
}

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
  window_attn<<<grid, 128, 0, st>>>(w);
  return cudaGetLastError();
}

cudaError_t launch_merge(const MergeArgs& g, cudaStream_t st) {
  if (g.Bm) {
    const size_t smem = sizeof(float) * ((size_t)MB * g.Y + 2 * MB + 2 * MB * 128);
    cudaError_t e = cudaFuncSetAttribute(merge_mapped, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    dim3 grid(g.rows, ceil_div(g.B, MB));
    merge_mapped<<<grid, 256, smem, st>>>(g);
  } else {
    dim3 grid(g.rows, g.B);
    merge_plain<<<grid, 128, 0, st>>>(g);
  }
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
