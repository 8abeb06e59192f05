// The dense contractions around the latent read, on the tensor cores
// (tcgen05, kind::tf32, accumulators in TMEM):
//
//   query map  (HLA eq. 3):  q~[b][row] = s*log2e * R~_i A_row^T q[b][row]        (bf16 out)
//   output map (eq. 4):      o[b][row]  = (B_row^T sum_s w_s y~_s + sum_c w_c y_c) / l
//   writer     (eq. 2, LLA encoders): fp32 partial sums of each writer slice
//
// Every one is a set of GEMMs D = A_g * X_g^T with a per-group codec matrix
// A_g (the M side, 128 rows per tile: the latent / head-dimension columns of
// the codec) and the activations X_g (the N side: sequences or tokens, BN per
// tile), so a decode batch of 32 and one of 768 both map onto the MMA's N.
//
// Operands are fp32 in HBM.  One thread of a TMA warp copies each 32-deep
// k-chunk of both operands into shared memory with tensor-map boxes that land
// directly in the MMA layouts (128-byte swizzle; for the MN-major codec of the
// maps the 128-byte swizzle with 32-byte atoms, the one layout the tensor
// cores take for MN-major tf32); out-of-range elements arrive as zeros.  Eight
// converter warps round each landed stage in place to tf32 (round to nearest,
// ties away) and, for PREC = 3, store the remainder x - tf32(x) as a second
// tf32 tile.  PREC = 3 issues hi*hi + hi*lo + lo*hi ("3xTF32"), whose error is
// that of fp32 arithmetic; PREC = 1 issues hi*hi (relative error about 2^-11
// per product).  Up to three MMA warps issue the MMAs into separate TMEM
// accumulators (one thread issuing a dependent chain is bound by its issue
// latency; see AccPlan) and release stages with tcgen05.commit; the converter
// warps then read the accumulators back (tcgen05.ld), add them, and run the
// epilogue.  Waits are bounded: on a
// timeout the CTA records an error code (outputs become NaN downstream).
#include <cuda.h>
#include <cuda_fp16.h>

#include <algorithm>
#include <cstring>

#include "tc_ptx.cuh"
#include "tmap.cuh"
#include "writer_slice.cuh"

namespace lla {
namespace {

using namespace ptx;

constexpr int GM = 128;                 // M of every MMA (codec rows per tile)
constexpr int KCH = 32;                 // k per chunk: 32 fp32 = one 128-byte row
constexpr int A_BYTES = GM * KCH * 4;   // 16 KB
constexpr int NPROD = 256;              // converter + epilogue threads (warps 0-7)
constexpr int MMA_WARP = NPROD / 32;    // warps 8..8+NISS-1: MMA issue (warp 8 also TMEM allocation)
constexpr int NISS = 3;                 // MMA issuer warps
constexpr int TMA_WARP = MMA_WARP + NISS;  // warp 11: tensor-map copies
constexpr int NTHR = NPROD + 32 * (NISS + 1);
constexpr int SMEM_MAX = 232448;
constexpr int YW_SMEM_MAX = 65536;      // output map: window term of the column slice kept in smem up to this
__host__ __device__ constexpr int align8(int x) { return (x + 7) & ~7; }
__host__ __device__ constexpr int align16(int x) { return (x + 15) & ~15; }
constexpr long long WAIT_CYCLES = 1ll << 32;

enum : int { KIND_QMAP = 0, KIND_OMAP = 1, KIND_WRITER = 2 };
enum : int { ERR_GEMM_EMPTY = 11, ERR_GEMM_FULL = 12, ERR_GEMM_DONE = 13, ERR_GEMM_LOAD = 14 };

// Tensor maps of one launch: codec operand(s) and activation operand(s).
struct TcMaps {
  CUtensorMap a[2];
  CUtensorMap x[2];
};

__host__ __device__ constexpr uint32_t idesc_tf32(int M, int N, bool a_mn_major) {
  return (1u << 4)                          // D format: fp32
         | (2u << 7)                        // A format: tf32
         | (2u << 10)                       // B format: tf32
         | ((a_mn_major ? 1u : 0u) << 15)   // B is always K-major
         | ((uint32_t)(N >> 3) << 17)
         | ((uint32_t)(M >> 4) << 24);
}

__device__ __forceinline__ void mma_tf32(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                         uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::tf32 [%0], %1, %2, %3, p;\n\t}"
      ::"r"(d_tmem), "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

__device__ __forceinline__ uint32_t to_tf32(float x) {
  uint32_t r;
  asm("cvt.rna.tf32.f32 %0, %1;" : "=r"(r) : "f"(x));
  return r;
}

__device__ __forceinline__ float4 lds4(uint32_t a) {
  float4 v;
  asm volatile("ld.shared.v4.f32 {%0, %1, %2, %3}, [%4];"
               : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w)
               : "r"(a)
               : "memory");
  return v;
}
__device__ __forceinline__ void sts4(uint32_t a, uint32_t x, uint32_t y, uint32_t z, uint32_t w) {
  asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(a), "r"(x), "r"(y), "r"(z), "r"(w) : "memory");
}

__device__ __forceinline__ bool wait_bar(uint32_t bar, uint32_t parity, volatile int* abort_flag, int* err,
                                         int code, bool honour_abort = true) {
  if (mbar_try_wait(bar, parity)) return true;
  const long long t0 = clock64();
  while (true) {
    if (honour_abort && *abort_flag) return false;
    if (mbar_try_wait(bar, parity)) return true;
    if (clock64() - t0 > WAIT_CYCLES) {
      *abort_flag = 1;
      if (err) atomicExch(err, code);
      return false;
    }
  }
}

// Shared-memory operand layouts (written by the tensor-map copies):
//   K-major tile (rows x 32 k): 128-byte rows, 8-row atoms of 1 KB, 16-byte
//   pieces swizzled by row mod 8 -- descriptor LBO 16, SBO 1024;
//   MN-major tf32 codec tile (128 rows x 32 k): four 32-row atoms 4 KB apart,
//   each 32 k-rows of 128 bytes whose 32-byte granules are swizzled by k-row
//   mod 4 -- descriptor layout type 1, LBO 4096 (atoms), SBO 512 (4 k-rows).

__device__ __forceinline__ int64_t qbf_index(int b, int row, int k, int r_k) {
  const int kb = k >> 6, e = k & 63;
  return (int64_t)b * (r_k >> 6) * 4096 + kb * 4096 + row * 64 + ((((e >> 3) ^ (row & 7)) << 3) | (e & 7));
}

// Accumulators and issuers.  One thread issuing a chain of tcgen05.mma is
// bound by its own issue latency, not the tensor pipe, so independent
// accumulator chains are spread over NISS issuer warps:
//   PREC = 3 (3xTF32):  one accumulator per product (hi*hi, lo*hi, hi*lo),
//                       issuer p issues product p of every chunk;
//   PREC = 1, nb >= 2:  one accumulator per operand block jb (output map:
//                       one per latent split), issuer jb mod NISS;
//   PREC = 1, nb = 1:   two accumulators taking alternate k-chunks, issuers
//                       0 and 1; the epilogue adds them.
// The epilogue sums the accumulators of a product in a fixed order.
struct AccPlan {
  int nacc;      // accumulators (BN columns each)
  int per_st;    // issuers that read each stage
  int active;    // issuers with work
};
__host__ __device__ inline AccPlan acc_plan(int prec, int nb) {
  if (prec == 3) return {3, 3, 3};
  if (nb >= 2) return {nb, nb < NISS ? nb : NISS, nb < NISS ? nb : NISS};
  return {2, 1, 2};
}

// Per-tile geometry, resolved from blockIdx for each kind.
struct Tile {
  int g;            // group: map row, or writer slice
  int split;        // writer k-split
  int m0, n0;       // tile origin (codec rows, activation rows)
  int Mv, Nv, K;    // valid extents of the group and its depth
  int kc0, kc1;     // chunk range
};

template <int KIND, int BN, int PREC>
__global__ void __launch_bounds__(NTHR, 1) tc_gemm(const __grid_constant__ TcMaps maps, const TcGemmArgs a) {
  const int NST = a.nst;   // stages in the ring (the host sizes it to shared memory)
  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  // the query map opens the call: it clears the call's error word, which the
  // kernels after it write (its own timeouts also turn its output into NaN)
  if (KIND == KIND_QMAP && a.clear_err && blockIdx.x == 0 && blockIdx.y == 0 && tid == 0) {
    griddep_wait();
    *a.clear_err = 0;
  }

  // ---- tile ------------------------------------------------------------
  Tile t;
  // output map: the k range of a tile is split over a cluster of ks CTAs
  const int ks = KIND == KIND_OMAP ? (int)blockIdx.x % a.ks : 0;
  const int tix = KIND == KIND_OMAP ? (int)blockIdx.x / a.ks : (int)blockIdx.x;
  const int mt = tix / a.ntiles, nti = tix % a.ntiles;
  t.m0 = mt * GM;
  t.n0 = nti * BN;
  Slice sl;
  if (KIND == KIND_WRITER) {
    t.g = (int)blockIdx.y / a.S;
    t.split = (int)blockIdx.y % a.S;
    sl = slice_of(a.w, t.g);
    t.Mv = sl.N;
    t.Nv = a.w.M;
    t.K = sl.K_outer * sl.d_in;
    const int nk = (t.K + KCH - 1) / KCH;
    t.kc0 = (int)((int64_t)nk * t.split / a.S);
    t.kc1 = (int)((int64_t)nk * (t.split + 1) / a.S);
    if (t.m0 >= t.Mv) return;   // this slice is narrower than the widest one
  } else {
    t.g = blockIdx.y;
    t.split = 0;
    t.Mv = a.Mtot;
    t.Nv = a.B;
    t.K = a.K;
    const int nk = (t.K + KCH - 1) / KCH;
    t.kc0 = KIND == KIND_OMAP ? (int)((int64_t)nk * ks / a.ks) : 0;
    t.kc1 = KIND == KIND_OMAP ? (int)((int64_t)nk * (ks + 1) / a.ks) : nk;
    if (KIND == KIND_QMAP && t.g >= a.rows) {
      // rows of the bf16 query operand past the last query row are zero
      griddep_wait();
      for (int idx = tid; idx < GM * BN; idx += NTHR) {
        const int m = t.m0 + (idx % GM), n = t.n0 + idx / GM;
        if (m < t.Mv && n < t.Nv) a.qbf[qbf_index(n, t.g, m, a.Mtot)] = __float2bfloat16_rn(0.f);
      }
      return;
    }
  }
  const int nb = KIND == KIND_OMAP ? a.NB : 1;
  const int nchunks = t.kc1 - t.kc0;

  // ---- shared memory ------------------------------------------------------
  const uint32_t b_tile = (uint32_t)BN * 128;
  const uint32_t a_part = (uint32_t)A_BYTES * (PREC == 3 ? 2 : 1);
  const uint32_t stage_bytes = a_part + b_tile * nb * (PREC == 3 ? 2 : 1);
  const uint32_t sbase = smem_u32(base);
  uint64_t* bars = reinterpret_cast<uint64_t*>(base + NST * stage_bytes);
  uint64_t* loaded = bars;            // [NST] TMA bytes landed
  uint64_t* full = bars + NST;        // [NST] converted (all converter threads)
  uint64_t* empty = bars + 2 * NST;   // [NST] MMAs reading the stage completed
  uint64_t* done = bars + 3 * NST;
  // misc region on a 16-byte boundary (the window-term tile is read as float4)
  uint8_t* misc = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(bars + 3 * NST + 1) + 15) & ~uintptr_t(15));
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(misc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(misc + 4);
  // output map: split weights, partial maxima and (for narrow column slices)
  // the window term, in dedicated shared memory (filled while the stages stream)
  const int ne = KIND == KIND_OMAP ? a.NB + a.Sw : 0;            // partials per sequence
  const int cols_per = KIND == KIND_OMAP ? (BN + a.ks - 1) / a.ks : BN;
  const int col_lo = min(BN, ks * cols_per), col_hi = min(BN, col_lo + cols_per);
  const bool yw_smem = KIND == KIND_OMAP && a.Sw > 0 && cols_per * GM * 4 <= YW_SMEM_MAX;
  float* wts = reinterpret_cast<float*>(misc + 16);                                       // [BN][ne + 1]
  float2* mls = reinterpret_cast<float2*>(misc + 16 + align8(BN * (ne + 1) * 4));         // [BN][ne]
  float* ywin_d = reinterpret_cast<float*>(misc + 16 + align8(BN * (ne + 1) * 4) + align16(BN * ne * 8));

  // The copy thread initialises the barriers and issues the first stages at
  // once, so their latency overlaps the TMEM allocation and the prologue.
  auto issue_chunk = [&](int i) {
    const int st = i % NST;
    const uint32_t s0 = sbase + st * stage_bytes;
    const uint32_t bar = smem_u32(&loaded[st]);
    mbar_arrive_tx(bar, (uint32_t)A_BYTES + nb * b_tile);
    const int k0 = (t.kc0 + i) * KCH;
    if (KIND == KIND_WRITER) {
      // chunk k0 lies in one (outer block, feature) run: outer o, feature d
      const int o = k0 / sl.d_in, d = k0 % sl.d_in;
      int ai = 0, ta = 0, ha = 0, tx = 0, hx = 0;
      if (a.w.mode == LLA_WRITE_HLA) {
        ai = t.g;                       // E_main or E_1
        ta = o;
        tx = t.g == 0 ? 1 + o : 0;      // loops 2..T, or loop 1
      } else if (a.w.mode == LLA_WRITE_PERHEAD) {
        ai = t.g / a.w.H;               // K or V
        ha = hx = t.g % a.w.H;
        ta = tx = o;
      } else {
        ai = t.g;
        ta = tx = o / a.w.H;
        ha = hx = o % a.w.H;
      }
      tma_load_4d(s0, &maps.a[ai], bar, d, t.m0, ha, ta);
      tma_load_4d(s0 + a_part, &maps.x[ai], bar, d, hx, tx, t.n0);
    } else if (KIND == KIND_QMAP) {
      tma_load_4d(s0, &maps.a[0], bar, 0, k0, t.m0 / 32, t.g % a.ncodec);
      tma_load_3d(s0 + a_part, &maps.x[0], bar, k0, t.g, t.n0);
    } else {
      tma_load_4d(s0, &maps.a[0], bar, 0, k0, t.m0 / 32, t.g % a.ncodec);
      for (int jb = 0; jb < nb; ++jb)
        tma_load_4d(s0 + a_part + jb * b_tile, &maps.x[0], bar, k0, t.g, t.n0, jb);
    }
  };
  const int first = min(NST, nchunks);
  const AccPlan ap = acc_plan(PREC, nb);
  if (warp == TMA_WARP && lane == 0) {
    for (int i = 0; i < NST; ++i) {
      mbar_init(smem_u32(&loaded[i]), 1);
      mbar_init(smem_u32(&full[i]), NPROD);
      mbar_init(smem_u32(&empty[i]), ap.per_st);
    }
    mbar_init(smem_u32(done), ap.active);
    *abort_flag = 0;
    fence_mbar_init();
    prefetch_tmap(&maps.a[0]);
    prefetch_tmap(&maps.x[0]);
    griddep_wait();
    for (int i = 0; i < first; ++i) issue_chunk(i);
  }
  uint32_t ncols = 32;
  while (ncols < (uint32_t)(ap.nacc * BN)) ncols <<= 1;
  if (warp == MMA_WARP) {
    tmem_alloc(smem_u32(tmem_slot), ncols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  griddep_wait();
  // output map with a cluster k-split: this CTA's weighted partial tile, in
  // the stage memory (free once every MMA is done)
  float* part_s = reinterpret_cast<float*>(base);                          // [BN][GM]

  if (warp < NPROD / 32) {
    // query map: the rotation of this thread's codec row (TMEM lane) for the
    // epilogue, computed while the first stage is in flight
    float cq = 1.f, sq = 0.f;
    if (KIND == KIND_QMAP && a.rotate) {
      const int mr = t.m0 + 32 * (warp & 3) + lane;
      if (mr < t.Mv) {
        const int pos = a.pos + (a.rows_per_q > 0 ? t.g / a.rows_per_q : 0);   // this row's query position
        rope_cs(mr >> 1, a.Mtot, a.d_h, a.base, (double)pos, &cq, &sq);
      }
    }
    // ---- converters: round each landed stage to tf32 in place ---------------
    // (the hi and lo tiles share one layout, so pieces are plain 16-byte slots)
    auto convert = [&](uint32_t addr, uint32_t lo_addr) {
      const float4 v = lds4(addr);
      const uint32_t hx = to_tf32(v.x), hy = to_tf32(v.y), hz = to_tf32(v.z), hw = to_tf32(v.w);
      sts4(addr, hx, hy, hz, hw);
      if (PREC == 3)
        sts4(lo_addr, to_tf32(v.x - __uint_as_float(hx)), to_tf32(v.y - __uint_as_float(hy)),
             to_tf32(v.z - __uint_as_float(hz)), to_tf32(v.w - __uint_as_float(hw)));
    };
    if constexpr (KIND == KIND_OMAP) {
      // while the first stages stream: (1) gather the (max, sum) of every split
      // and window partial of the tile's sequences; (2) one thread per sequence
      // turns them into weights 2^(m - M) and 1 / l; (3) for narrow column
      // slices, the window term sum_c w_c y_c of this CTA's columns
      const int ld = ne + 1;
      const int64_t bstride = (int64_t)a.B * a.rows;
#pragma unroll 4
      for (int idx = tid; idx < BN * ne; idx += NPROD) {
        const int bb = idx / ne, e = idx % ne;
        const int n = t.n0 + bb;
        float2 v = make_float2(-INFINITY, 0.f);
        if (n < t.Nv) {
          const int64_t br = (int64_t)n * a.rows + t.g;
          const float* src = e < a.NB ? a.part_ml + (e * bstride + br) * 2 : a.win_ml + ((e - a.NB) * bstride + br) * 2;
          v = make_float2(src[0], src[1]);
        }
        mls[idx] = v;
      }
      named_sync(1, NPROD);
      for (int bb = tid; bb < BN; bb += NPROD) {
        const float2* e = mls + bb * ne;
        float* w = wts + bb * ld;
        float M = -INFINITY;
        for (int j = 0; j < ne; ++j) M = fmaxf(M, e[j].x);
        float L = 0.f;
        for (int j = 0; j < ne; ++j) {
          const float wj = e[j].x == -INFINITY ? 0.f : exp2f(e[j].x - M);
          w[j] = wj;
          L += wj * e[j].y;
        }
        w[ne] = t.n0 + bb < t.Nv ? 1.f / L : 0.f;
      }
      named_sync(1, NPROD);
      if (yw_smem) {
        // float4 groups of 4 columns; each thread takes two groups at a time
        // and issues the loads of up to eight window chunks of both before
        // using any, so a pass costs one round trip to L2, not one per chunk
        constexpr int WCB = 8;
        const int g4_hi = (col_hi - col_lo) * (GM / 4);
        for (int base4 = 0; base4 < g4_hi; base4 += 2 * NPROD) {
          float4 acc4[2];
          int64_t off4[2];
          bool live[2];
          int bcol[2];
#pragma unroll
          for (int u = 0; u < 2; ++u) {
            const int idx4 = base4 + u * NPROD + tid;
            const int bb = col_lo + idx4 / (GM / 4), mm = 4 * (idx4 % (GM / 4));
            const int n = t.n0 + bb, m = t.m0 + mm;
            live[u] = idx4 < g4_hi && n < t.Nv && m < t.Mv;
            off4[u] = live[u] ? ((int64_t)n * a.rows + t.g) * a.Mtot + m : 0;
            bcol[u] = idx4 < g4_hi ? bb : col_lo;
            acc4[u] = make_float4(0.f, 0.f, 0.f, 0.f);
          }
          for (int c0 = 0; c0 < a.Sw; c0 += WCB) {
            float4 v4[2][WCB];
#pragma unroll
            for (int j = 0; j < WCB; ++j)
#pragma unroll
              for (int u = 0; u < 2; ++u)
                v4[u][j] = live[u] && c0 + j < a.Sw
                               ? *reinterpret_cast<const float4*>(a.win_y + (c0 + j) * bstride * a.Mtot + off4[u])
                               : make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
            for (int j = 0; j < WCB; ++j)
#pragma unroll
              for (int u = 0; u < 2; ++u) {
                const float w = live[u] && c0 + j < a.Sw ? wts[bcol[u] * ld + a.NB + c0 + j] : 0.f;
                acc4[u].x = fmaf(w, v4[u][j].x, acc4[u].x);
                acc4[u].y = fmaf(w, v4[u][j].y, acc4[u].y);
                acc4[u].z = fmaf(w, v4[u][j].z, acc4[u].z);
                acc4[u].w = fmaf(w, v4[u][j].w, acc4[u].w);
              }
          }
#pragma unroll
          for (int u = 0; u < 2; ++u) {
            const int idx4 = base4 + u * NPROD + tid;
            if (idx4 < g4_hi) reinterpret_cast<float4*>(ywin_d)[idx4] = acc4[u];
          }
        }
        named_sync(1, NPROD);
      }
    }
    const int b_pieces = nb * BN * 8;
#pragma unroll 1
    for (int i = 0; i < nchunks; ++i) {
      const int st = i % NST;
      if (!wait_bar(smem_u32(&loaded[st]), (i / NST) & 1, abort_flag, a.err, ERR_GEMM_LOAD)) break;
      const uint32_t s0 = sbase + st * stage_bytes;
#pragma unroll
      for (int u = 0; u < A_BYTES / 16 / NPROD; ++u) {
        const uint32_t off = 16u * (tid + NPROD * u);
        convert(s0 + off, s0 + A_BYTES + off);
      }
      const uint32_t bt = s0 + a_part;
      for (int p = tid; p < b_pieces; p += NPROD) convert(bt + 16u * p, bt + nb * b_tile + 16u * p);
      fence_proxy_async_smem();
      mbar_arrive(smem_u32(&full[st]));
    }

    // ---- epilogue ------------------------------------------------------------
    const bool ok = wait_bar(smem_u32(done), 0, abort_flag, a.err, ERR_GEMM_DONE, false) && !*abort_flag;
    tc_fence_after();
    // warps w and w + 4 share TMEM lanes 32 (w & 3) .. +31 and split the columns
    const int quarter = warp & 3, half = warp >> 2;
    const int m = t.m0 + 32 * quarter + lane;   // this thread's TMEM lane = codec row
    const uint32_t lane_addr = tmem + ((uint32_t)(32 * quarter) << 16);
    const bool have = nchunks > 0;
    // accumulators summed for one output column block (fixed order)
    const int nsum = PREC == 3 ? 3 : (nb == 1 && nchunks > 1 ? 2 : 1);
    auto load_sum = [&](uint32_t col, float* v) {
      tmem_ld16(lane_addr + col, v);
      tmem_wait_ld();
      for (int q = 1; q < nsum; ++q) {
        float w[16];
        tmem_ld16(lane_addr + (uint32_t)(q * BN) + col, w);
        tmem_wait_ld();
#pragma unroll
        for (int i = 0; i < 16; ++i) v[i] += w[i];
      }
    };
    const bool bad = !ok || (KIND == KIND_OMAP && a.err && *a.err);
#pragma unroll 1
    for (int c = half * (BN / 32); c < (half + 1) * (BN / 32); ++c) {
      float v[16];
      if (KIND == KIND_OMAP) {
        const int ld = ne + 1;
        float acc[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) acc[i] = 0.f;
        for (int jb = 0; jb < nb; ++jb) {
          if (have) {
            load_sum(jb * BN + 16 * c, v);
          } else {
#pragma unroll
            for (int i = 0; i < 16; ++i) v[i] = 0.f;
          }
#pragma unroll
          for (int i = 0; i < 16; ++i) acc[i] = fmaf(wts[(16 * c + i) * ld + jb], v[i], acc[i]);
        }
#pragma unroll
        for (int i = 0; i < 16; ++i) v[i] = acc[i];
      } else if (have) {
        load_sum(16 * c, v);
      } else {
#pragma unroll
        for (int i = 0; i < 16; ++i) v[i] = 0.f;
      }
      if (KIND == KIND_QMAP) {
        // rotate pair (m even, m + 1) -- neighbouring lanes -- then scale to bf16
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          const float other = __shfl_xor_sync(0xffffffffu, v[i], 1);
          // even lanes hold x of the pair, odd lanes y; the even lane stores both
          const float x = (m & 1) ? other : v[i], y = (m & 1) ? v[i] : other;
          const int n = t.n0 + 16 * c + i;
          if (!(m & 1) && m < t.Mv && n < t.Nv) {
            const float rx = bad ? NAN : (x * cq - y * sq) * a.qmul;
            const float ry = bad ? NAN : (x * sq + y * cq) * a.qmul;
            void* dst = a.qbf + qbf_index(n, t.g, m, a.Mtot);
            if (a.qf16) *reinterpret_cast<__half2*>(dst) = __floats2half2_rn(rx, ry);
            else *reinterpret_cast<__nv_bfloat162*>(dst) = __floats2bfloat162_rn(rx, ry);
          }
        }
      } else if (KIND == KIND_OMAP) {
        if (a.ks > 1) {
#pragma unroll
          for (int i = 0; i < 16; ++i) part_s[(16 * c + i) * GM + (m - t.m0)] = v[i];
        } else {
          const int ld = ne + 1;
          const int64_t bstride = (int64_t)a.B * a.rows;
          float yw[16];
          if (yw_smem) {
#pragma unroll
            for (int i = 0; i < 16; ++i) yw[i] = ywin_d[(16 * c + i) * GM + (m - t.m0)];
          } else {
            // window term from global memory: the 16 columns' loads per chunk together
#pragma unroll
            for (int i = 0; i < 16; ++i) yw[i] = 0.f;
            for (int cw = 0; cw < a.Sw; ++cw) {
              float wv[16];
#pragma unroll
              for (int i = 0; i < 16; ++i) {
                const int n = t.n0 + 16 * c + i;
                wv[i] = (m < t.Mv && n < t.Nv)
                            ? a.win_y[(cw * bstride + (int64_t)n * a.rows + t.g) * a.Mtot + m] : 0.f;
              }
#pragma unroll
              for (int i = 0; i < 16; ++i) yw[i] = fmaf(wts[(16 * c + i) * ld + a.NB + cw], wv[i], yw[i]);
            }
          }
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            const int bb = 16 * c + i, n = t.n0 + bb;
            if (m < t.Mv && n < t.Nv)
              a.out[(int64_t)n * a.outs_b + (int64_t)t.g * a.Mtot + m] = bad ? NAN : (v[i] + yw[i]) * wts[bb * ld + ne];
          }
        }
      } else {
        float* P = a.w.part + ((int64_t)(t.g * a.S + t.split) * a.w.M) * a.w.Nmax;
#pragma unroll 4
        for (int i = 0; i < 16; ++i) {
          const int n = t.n0 + 16 * c + i;
          if (m < t.Mv && n < t.Nv) P[(int64_t)n * a.w.Nmax + m] = bad ? NAN : v[i];
        }
      }
    }
    tc_fence_before();
  } else if (warp == TMA_WARP) {
    // ---- tensor-map copies ------------------------------------------------------
    if (lane == 0) {
      int issued = first;
#pragma unroll 1
      for (int i = first; i < nchunks; ++i) {
        const int st = i % NST;
        if (!wait_bar(smem_u32(&empty[st]), ((i / NST) - 1) & 1, abort_flag, a.err, ERR_GEMM_EMPTY)) break;
        issue_chunk(i);
        issued = i + 1;
      }
      if (*abort_flag) {
        // leave no copy in flight: wait (bounded) for the stages issued last
        for (int i = max(0, issued - NST); i < issued; ++i)
          wait_bar(smem_u32(&loaded[i % NST]), (i / NST) & 1, abort_flag, nullptr, 0, false);
      }
    }
  } else if (lane == 0) {
    // ---- MMA issue (warps MMA_WARP .. MMA_WARP + NISS - 1) ----------------------
    const int me = warp - MMA_WARP;
    const bool a_mn = KIND != KIND_WRITER;
    constexpr uint32_t idesc = idesc_tf32(GM, BN, KIND != KIND_WRITER);
    const uint32_t a_step = a_mn ? (1024u >> 4) : (32u >> 4);   // 8 k: two 4-row groups, or 32 bytes
    const uint32_t b_step = 32u >> 4;
    if (me < ap.active) {
#pragma unroll 1
      for (int i = 0; i < nchunks; ++i) {
        if (PREC == 1 && nb == 1 && (i & 1) != me) continue;   // alternate chunks
        const int st = i % NST;
        if (!wait_bar(smem_u32(&full[st]), (i / NST) & 1, abort_flag, a.err, ERR_GEMM_FULL)) break;
        tc_fence_after();
        const uint32_t s0 = sbase + st * stage_bytes;
        const uint64_t ahi = a_mn ? smem_desc_sw128_32b(s0, 4096, 512) : smem_desc_sw128(s0, 16, 1024);
        const uint64_t alo = a_mn ? smem_desc_sw128_32b(s0 + A_BYTES, 4096, 512) : smem_desc_sw128(s0 + A_BYTES, 16, 1024);
        if (PREC == 3) {
          // product me: 0 = hi*hi, 1 = lo*hi, 2 = hi*lo, into accumulator me
          const uint32_t bt = s0 + a_part;
          const uint64_t bhi = smem_desc_sw128(bt, 16, 1024);
          const uint64_t blo = smem_desc_sw128(bt + nb * b_tile, 16, 1024);
          const uint64_t ad = me == 1 ? alo : ahi, bd = me == 2 ? blo : bhi;
          const uint32_t d = tmem + (uint32_t)(me * BN);
#pragma unroll
          for (int j = 0; j < KCH / 8; ++j)
            mma_tf32(d, ad + j * a_step, bd + j * b_step, idesc, (i > 0 || j > 0) ? 1u : 0u);
        } else {
          for (int jb = nb == 1 ? 0 : me; jb < nb; jb += NISS) {
            const uint32_t bt = s0 + a_part + jb * b_tile;
            const uint64_t bhi = smem_desc_sw128(bt, 16, 1024);
            const uint32_t d = tmem + (uint32_t)((nb == 1 ? me : jb) * BN);
            const bool first = nb == 1 ? i < 2 : i == 0;
#pragma unroll
            for (int j = 0; j < KCH / 8; ++j)
              mma_tf32(d, ahi + j * a_step, bhi + j * b_step, idesc, (!first || j > 0) ? 1u : 0u);
          }
        }
        mma_commit(smem_u32(&empty[st]));
      }
      mma_commit(smem_u32(done));
    }
  }
  if (KIND == KIND_OMAP && a.ks > 1) {
    // every CTA's partial tile is complete: finish this CTA's columns from the
    // partials of all ks CTAs (distributed shared memory), in rank order
    __syncwarp();
    cluster_sync_all();
    if (warp < NPROD / 32) {
      const int ld = ne + 1;
      const bool bad = *abort_flag || (a.err && *a.err);
      const uint32_t ps_addr = smem_u32(part_s);
      // four elements per thread at a time, all their remote loads issued
      // before any is summed, in rank order (the launcher keeps ks <= 4)
      constexpr int EU = 4;
      for (int idx0 = col_lo * GM + tid; idx0 < col_hi * GM; idx0 += EU * NPROD) {
        float r[EU][4];
#pragma unroll
        for (int u = 0; u < EU; ++u) {
          const int idx = idx0 + u * NPROD;
#pragma unroll
          for (int rk = 0; rk < 4; ++rk)
            r[u][rk] = idx < col_hi * GM && rk < a.ks ? ld_shared_cluster(mapa_shared(ps_addr + 4u * idx, (uint32_t)rk))
                                                      : 0.f;
        }
#pragma unroll
        for (int u = 0; u < EU; ++u) {
          const int idx = idx0 + u * NPROD;
          if (idx >= col_hi * GM) break;
          const int bb = idx / GM, mm = idx % GM;
          const int n = t.n0 + bb, m = t.m0 + mm;
          float y = yw_smem ? ywin_d[idx - col_lo * GM] : 0.f;
#pragma unroll
          for (int rk = 0; rk < 4; ++rk)
            if (rk < a.ks) y += r[u][rk];
          if (m < t.Mv && n < t.Nv)
            a.out[(int64_t)n * a.outs_b + (int64_t)t.g * a.Mtot + m] = bad ? NAN : y * wts[bb * ld + ne];
        }
      }
    }
    // no CTA leaves while a neighbour may still read its partial tile
    cluster_sync_all();
  }
  __syncthreads();
  if (warp == MMA_WARP) {
    tc_fence_after();
    tmem_dealloc(tmem, ncols);
  }
  griddep_launch();
}

template <int KIND, int BN, int PREC>
cudaError_t launch_one(const TcMaps& maps, TcGemmArgs a, int grid_y, int nb, size_t smem_budget, cudaStream_t st) {
  const int stage = (A_BYTES * (PREC == 3 ? 2 : 1)) + BN * 128 * nb * (PREC == 3 ? 2 : 1);
  // output map: weights, partial maxima and the window term of the column slice
  int misc = 0;
  if (KIND == KIND_OMAP) {
    const int ne = nb + a.Sw, cols_per = (BN + a.ks - 1) / a.ks;
    misc = align8(BN * (ne + 1) * 4) + align16(BN * ne * 8) +
           (a.Sw > 0 && cols_per * GM * 4 <= YW_SMEM_MAX ? cols_per * GM * 4 : 0);
  }
  // stages: 2 to 6, as many as the budget allows (16 bytes for aligning the
  // misc region), and no more than a CTA's k-chunks of the maps: a stage that
  // is never filled only keeps other CTAs off the SM
  const size_t fixed = 1024 + 16 + 16 + misc + 8;
  const int nk = (a.K + KCH - 1) / KCH;
  const int cta_chunks = KIND == KIND_QMAP ? nk : KIND == KIND_OMAP ? (nk + a.ks - 1) / a.ks : 6;
  auto plan = [&](size_t budget) {
    auto fits = [&](int n) { return fixed + (size_t)n * (stage + 24) <= budget; };
    int n = 2;
    while (n < 6 && n < cta_chunks && fits(n + 1)) ++n;
    // a cluster k-split keeps its partial tile in the stage memory
    while (KIND == KIND_OMAP && a.ks > 1 && (size_t)BN * GM * 4 > (size_t)n * stage && n < 6 && fits(n + 1)) ++n;
    return n;
  };
  int nst = plan(smem_budget);
  // the output map runs beside the window and the other group's kernels: at
  // most half an SM's shared memory when that still leaves three stages (or
  // all its chunks); measured faster than the full budget on batch-32 calls
  const size_t half = (size_t)SMEM_MAX / 2 - 1024;
  if (KIND == KIND_OMAP && smem_budget > half) {
    const int n2 = plan(half);
    if (n2 >= std::min(3, cta_chunks) && fixed + (size_t)n2 * stage + 8 * (3 * n2 + 1) <= half &&
        !(a.ks > 1 && (size_t)BN * GM * 4 > (size_t)n2 * stage))
      nst = n2;
  }
  a.nst = nst;
  // with a cluster k-split, the partial tile reuses the stages
  if (KIND == KIND_OMAP && a.ks > 1 && (size_t)BN * GM * 4 > (size_t)nst * stage) return cudaErrorNotSupported;
  // a cluster k-split needs the window term of its slice in shared memory
  if (KIND == KIND_OMAP && a.ks > 1 && a.Sw > 0 && ((BN + a.ks - 1) / a.ks) * GM * 4 > YW_SMEM_MAX)
    return cudaErrorNotSupported;
  size_t smem = fixed + (size_t)nst * stage + 8 * (3 * nst + 1);
  // keep the CTAs an SM can hold (228 KB of shared memory, 1 KB reserved per
  // CTA) within its 512 TMEM columns, so that no allocation ever waits
  int ncols = 32;
  while (ncols < acc_plan(PREC, nb).nacc * BN) ncols <<= 1;
  const int max_ctas = 512 / ncols;
  const size_t floor_smem = (size_t)233472 / (max_ctas + 1) - 1024 + 16;
  if (smem < floor_smem) smem = floor_smem;
  if (smem > (size_t)SMEM_MAX) return cudaErrorNotSupported;
  cudaError_t e = cudaFuncSetAttribute(tc_gemm<KIND, BN, PREC>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  const int ksplit = KIND == KIND_OMAP ? a.ks : 1;
  dim3 grid(a.mtiles * a.ntiles * ksplit, grid_y);
  return launch_kernel(tc_gemm<KIND, BN, PREC>, grid, dim3(NTHR), smem, st, ksplit, maps, a);
}

int pick_bn(int n) { return n <= 32 ? 32 : n <= 64 ? 64 : n <= 128 ? 128 : 256; }

// Codec of the maps, [groups][K][Mtot] fp32, as an MN-major tf32 operand:
// 4-D view (32 rows, k, 32-row atom, group), boxes of 32 x 32 x 4 atoms.
bool map_codec_tmap(CUtensorMap* m, const float* W, int groups, int K, int Mtot) {
  if (Mtot % 32 || K % 4) return false;
  const cuuint64_t dims[4] = {32, (cuuint64_t)K, (cuuint64_t)(Mtot / 32), (cuuint64_t)groups};
  const cuuint64_t strides[3] = {(cuuint64_t)Mtot * 4, 128, (cuuint64_t)K * Mtot * 4};
  const cuuint32_t box[4] = {32, KCH, GM / 32, 1};
  return tmap_f32(m, W, 4, dims, strides, box, CU_TENSOR_MAP_SWIZZLE_128B_ATOM_32B);
}

template <int KIND, int PREC>
cudaError_t launch_bn(TcMaps& maps, TcGemmArgs a, int Nv, int grid_y, int nb, int bn_cap, size_t smem_budget,
                      bool (*x_map)(TcMaps&, const TcGemmArgs&, int), cudaStream_t st) {
  const int bn = std::min(pick_bn(Nv), bn_cap);
  a.ntiles = (Nv + bn - 1) / bn;
  if (!x_map(maps, a, bn)) return cudaErrorNotSupported;
  switch (bn) {
    case 32: return launch_one<KIND, 32, PREC>(maps, a, grid_y, nb, smem_budget, st);
    case 64: return launch_one<KIND, 64, PREC>(maps, a, grid_y, nb, smem_budget, st);
    case 128: return launch_one<KIND, 128, PREC>(maps, a, grid_y, nb, smem_budget, st);
    default: return launch_one<KIND, 256, PREC>(maps, a, grid_y, nb, smem_budget, st);
  }
}

inline bool al16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15) == 0; }

// q [B][rows][K] (batch stride xs_b): 3-D view (k, row, sequence), boxes of 32 x 1 x BN.
bool qmap_x(TcMaps& maps, const TcGemmArgs& a, int bn) {
  const cuuint64_t dims[3] = {(cuuint64_t)a.K, (cuuint64_t)a.rows, (cuuint64_t)a.B};
  const cuuint64_t strides[2] = {(cuuint64_t)a.K * 4, (cuuint64_t)a.xs_b * 4};
  const cuuint32_t box[3] = {KCH, 1, (cuuint32_t)bn};
  return tmap_f32(&maps.x[0], a.X, 3, dims, strides, box, CU_TENSOR_MAP_SWIZZLE_128B);
}

// split partials y~ [S][B][rows][K]: 4-D view (k, row, sequence, split).
bool omap_x(TcMaps& maps, const TcGemmArgs& a, int bn) {
  const cuuint64_t dims[4] = {(cuuint64_t)a.K, (cuuint64_t)a.rows, (cuuint64_t)a.B, (cuuint64_t)a.NB};
  const cuuint64_t strides[3] = {(cuuint64_t)a.K * 4, (cuuint64_t)a.rows * a.K * 4,
                                 (cuuint64_t)a.B * a.rows * a.K * 4};
  const cuuint32_t box[4] = {KCH, 1, (cuuint32_t)bn, 1};
  return tmap_f32(&maps.x[0], a.X, 4, dims, strides, box, CU_TENSOR_MAP_SWIZZLE_128B);
}

// Writer: codec E(n, k) and activations X(m, k) of both slices' operands as
// 4-D views (feature, n, head, outer) and (feature, head, loop, token).
bool writer_x(TcMaps& maps, const TcGemmArgs& a, int bn) {
  const WriterArgs& w = a.w;
  const int64_t mstride = w.n_tok == 1 ? w.xs_b : w.xs_n;
  const cuuint32_t boxa[4] = {KCH, GM, 1, 1};
  const cuuint32_t boxx[4] = {KCH, 1, 1, (cuuint32_t)bn};
  if (w.mode == LLA_WRITE_HLA) {
    const int N0 = w.r_k + w.r_v, N1 = 2 * w.r_1;
    const cuuint64_t d0[4] = {(cuuint64_t)w.D, (cuuint64_t)N0, 1, (cuuint64_t)(w.T - 1)};
    const cuuint64_t s0[3] = {(cuuint64_t)w.D * 4, (cuuint64_t)N0 * w.D * 4, (cuuint64_t)N0 * w.D * 4};
    const cuuint64_t d1[4] = {(cuuint64_t)w.D, (cuuint64_t)N1, 1, 1};
    const cuuint64_t s1[3] = {(cuuint64_t)w.D * 4, (cuuint64_t)N1 * w.D * 4, (cuuint64_t)N1 * w.D * 4};
    const cuuint64_t dx[4] = {(cuuint64_t)w.D, 1, (cuuint64_t)w.T, (cuuint64_t)w.M};
    const cuuint64_t sx[3] = {(cuuint64_t)w.xs_t * 4, (cuuint64_t)w.xs_t * 4, (cuuint64_t)mstride * 4};
    return (w.T < 2 || tmap_f32(&maps.a[0], w.E_main, 4, d0, s0, boxa, CU_TENSOR_MAP_SWIZZLE_128B)) &&
           tmap_f32(&maps.a[1], w.E_1, 4, d1, s1, boxa, CU_TENSOR_MAP_SWIZZLE_128B) &&
           tmap_f32(&maps.x[0], w.x, 4, dx, sx, boxx, CU_TENSOR_MAP_SWIZZLE_128B) &&
           tmap_f32(&maps.x[1], w.x, 4, dx, sx, boxx, CU_TENSOR_MAP_SWIZZLE_128B);
  }
  const float* E[2] = {w.E_K, w.E_V};
  const float* X[2] = {w.x, w.xv};
  const int r[2] = {w.r_k, w.r_v};
  for (int p = 0; p < 2; ++p) {
    const cuuint64_t da[4] = {(cuuint64_t)w.d_h, (cuuint64_t)r[p], (cuuint64_t)w.H, (cuuint64_t)w.T};
    const cuuint64_t sa[3] = {(cuuint64_t)w.d_h * 4, (cuuint64_t)r[p] * w.d_h * 4, (cuuint64_t)w.H * r[p] * w.d_h * 4};
    const cuuint64_t dx[4] = {(cuuint64_t)w.d_h, (cuuint64_t)w.H, (cuuint64_t)w.T, (cuuint64_t)w.M};
    const cuuint64_t sx[3] = {(cuuint64_t)w.d_h * 4, (cuuint64_t)w.xs_t * 4, (cuuint64_t)mstride * 4};
    if (!tmap_f32(&maps.a[p], E[p], 4, da, sa, boxa, CU_TENSOR_MAP_SWIZZLE_128B) ||
        !tmap_f32(&maps.x[p], X[p], 4, dx, sx, boxx, CU_TENSOR_MAP_SWIZZLE_128B))
      return false;
  }
  return true;
}

}  // namespace

// ------------------------------------------------------------- query map --
bool query_map_tc_ok(const MapArgs& g) {
  return g.use_tc && al16(g.W) && al16(g.X) && g.xs_b % 4 == 0 && g.xs_row == g.K && g.K % 4 == 0 &&
         g.N % 64 == 0 && g.N <= 1024;
}

cudaError_t launch_query_map_tc(const MapArgs& g, int* err, cudaStream_t st) {
  TcGemmArgs a;
  std::memset(&a, 0, sizeof(a));
  a.B = g.B; a.rows = g.rows; a.Mtot = g.N; a.K = g.K; a.mtiles = (g.N + GM - 1) / GM;
  a.Aw = g.W; a.X = g.X; a.xs_b = g.xs_b;
  a.rotate = g.rotate; a.pos = g.pos; a.d_h = g.d_h; a.base = g.base; a.qmul = g.qmul; a.qbf = g.qbf;
  a.qf16 = g.q_f16;
  a.clear_err = g.clear_err;
  a.ncodec = g.ncodec > 0 ? g.ncodec : g.rows;
  a.rows_per_q = g.rows_per_q;
  a.err = err; a.NB = 1; a.S = 1; a.ks = 1;
  TcMaps maps;
  std::memset(&maps, 0, sizeof(maps));
  if (!map_codec_tmap(&maps.a[0], g.W, a.ncodec, g.K, g.N)) return cudaErrorNotSupported;
  return launch_bn<KIND_QMAP, 1>(maps, a, g.B, 64, 1, 128, SMEM_MAX / 2 - 1024, qmap_x, st);
}

// ------------------------------------------------------------ output map --
bool output_map_tc_ok(const MapArgs& g) {
  // one TMEM accumulator per latent split: at most 8 splits of 32 columns
  return al16(g.W) && g.N % 32 == 0 && g.N <= GM && g.K % 4 == 0 && g.S >= 1 && g.S <= 8 &&
         g.Sw <= kMaxWindowChunks;
}

cudaError_t launch_output_map_tc(const MapArgs& g, cudaStream_t st) {
  TcGemmArgs a;
  std::memset(&a, 0, sizeof(a));
  a.B = g.B; a.rows = g.rows; a.Mtot = g.N; a.K = g.K; a.mtiles = 1;
  a.Aw = g.W; a.X = g.part_y;
  a.part_ml = g.part_ml; a.win_ml = g.win_ml; a.win_y = g.win_y; a.Sw = g.Sw;
  a.out = g.out; a.outs_b = g.outs_b; a.err = const_cast<int*>(g.err);
  a.NB = g.S; a.S = 1;
  a.ncodec = g.ncodec > 0 ? g.ncodec : g.rows;
  int bn_cap = 128;
  while (bn_cap > 32 && g.S * bn_cap > 256) bn_cap >>= 1;
  // k-splits over a cluster so that small batches still fill the SMs
  const int bn = std::min(pick_bn(g.B), bn_cap);
  const int tiles = g.rows * ((g.B + bn - 1) / bn);
  const int nk = (g.K + KCH - 1) / KCH;
  // one CTA per SM (registers), and clusters do not tile every GPC's SMs:
  // keep the whole grid to 128 CTAs so that it starts in one wave
  a.ks = std::max(1, std::min(std::min(4, nk), 128 / std::max(tiles, 1)));
  TcMaps maps;
  std::memset(&maps, 0, sizeof(maps));
  if (!map_codec_tmap(&maps.a[0], g.W, a.ncodec, g.K, g.N)) return cudaErrorNotSupported;
  return launch_bn<KIND_OMAP, 1>(maps, a, g.B, g.rows, g.S, bn_cap, SMEM_MAX, omap_x, st);
}

// ---------------------------------------------------------------- writer --
bool writer_tc_ok(const WriterArgs& w) {
  if (!al16(w.x) || (w.xv && !al16(w.xv))) return false;
  if (w.xs_b % 4 || w.xs_n % 4 || w.xs_t % 4) return false;
  if (w.n_tok > 1 && w.xs_b != (int64_t)w.n_tok * w.xs_n) return false;   // tokens must form one strided axis
  const float* es[4] = {w.E_main, w.E_1, w.E_K, w.E_V};
  for (const float* e : es)
    if (e && !al16(e)) return false;
  if (w.mode == LLA_WRITE_HLA) return w.D % KCH == 0;
  return w.d_h % KCH == 0;
}

int writer_tc_splits(const WriterArgs& w, int num_sms) {
  (void)num_sms;
  return writer_depth_splits(w);
}

cudaError_t launch_writer_tc(const WriterArgs& w, int* err, cudaStream_t st) {
  TcGemmArgs a;
  std::memset(&a, 0, sizeof(a));
  a.w = w; a.err = err; a.S = w.S; a.NB = 1; a.ks = 1;
  a.mtiles = (w.Nmax + GM - 1) / GM;
  TcMaps maps;
  std::memset(&maps, 0, sizeof(maps));
  return launch_bn<KIND_WRITER, 3>(maps, a, w.M, w.Z * w.S, 1, 128, SMEM_MAX, writer_x, st);
}

}  // namespace lla
