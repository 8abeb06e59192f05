// LLA reconstruct-on-read on the tensor cores (tcgen05 + TMEM).
//
// LLA abstract: the cache stores per-head latents c^K_{j,h}, c^V_{j,h} of rank
// r and rebuilds loop-specific keys and values only when attention reads them.
// One CTA handles one (loop t, head h, sequence b) over the whole latent
// range; CTAs of the same (h, b) are launched next to each other, so the
// latent stream of a head is read from HBM once and from L2 by its loops.
// Per 64-token tile, both reconstructions are MMAs whose results never leave
// the SM:
//   K^_t  = C^K U^K_t^T   (M = 64 tokens, N = d_h, K = r): TMEM row = token,
//   V^T_t = U^V_t C^V^T   (M = 128 >= d_h, N = 64 tokens): TMEM row = feature.
// Four softmax warps then score each token against q (one TMEM row per lane:
// a 1 x d_h dot product, no cross-lane sum), run the online softmax over the
// tile, and accumulate o[d] += sum_j p_j V^T[d][j] (one TMEM row per lane).
//
// Precision: latents are bf16 and exact as MMA operands; each codec matrix U
// (fp32) is split into U_hi = bf16(U) and U_lo = bf16(U - U_hi), and both
// products accumulate in fp32, so the rebuilt vectors carry a relative error of
// about 2^-17 (fp32 codec, bf16 cache).  The rank is padded to a multiple of 64
// with zeros (copy engine for the latents, the CTA itself for U).
//
// Waits are bounded; on a timeout the CTA records an error code (the merge then
// emits NaN), waits for its copies and MMAs, and frees TMEM.
#include <cuda.h>

#include <algorithm>
#include <cstring>

#include "kernels.cuh"
#include "tc_ptx.cuh"
#include "tmap.cuh"

namespace lla {
namespace {

using namespace ptx;

constexpr int RT_TOK = 64;            // tokens per tile
constexpr int RCH = 64;               // rank elements per 128-byte chunk
constexpr int RCT = 192;              // threads: warps 0-3 softmax, 4 TMA, 5 MMA
constexpr int R_NST = 3;              // latent stages
constexpr long long R_WAIT = 1ll << 32;

enum : int { ERR_RECON_STAGE = 31, ERR_RECON_TFREE = 32, ERR_RECON_U = 33, ERR_RECON_K = 34, ERR_RECON_V = 35,
             ERR_RECON_EMPTY = 36 };

__device__ __forceinline__ bool rwait(uint32_t bar, uint32_t parity, volatile int* abort_flag, int* err, int code,
                                      bool honour_abort = true) {
  if (mbar_try_wait(bar, parity)) return true;
  const long long t0 = clock64();
  while (true) {
    if (honour_abort && *abort_flag) return false;
    if (mbar_try_wait(bar, parity)) return true;
    if (clock64() - t0 > R_WAIT) {
      *abort_flag = 1;
      if (err) atomicExch(err, code);
      return false;
    }
  }
}

// Shared-memory plan (offsets from the 1 KB-aligned base).  Operand tiles are
// K-major, 128-byte rows, 8-row atoms of 1 KB, 16-byte pieces swizzled by row.
struct RLayout {
  int nch;          // rank chunks of 64
  int uk_rows;      // d_h rounded up to 8 (rows of the U^K operand)
  __host__ __device__ int uk_bytes() const { return nch * uk_rows * 128; }        // one of hi / lo
  __host__ __device__ int uv_bytes() const { return nch * 128 * 128; }            // 128 rows (M of V^T)
  __host__ __device__ int stage_bytes() const { return 2 * nch * RT_TOK * 128; }  // C^K then C^V
  __host__ __device__ int off_uk() const { return 0; }
  __host__ __device__ int off_uv() const { return 2 * uk_bytes(); }
  __host__ __device__ int off_stage() const { return off_uv() + 2 * uv_bytes(); }
  __host__ __device__ int off_q() const { return off_stage() + R_NST * stage_bytes(); }   // float[128]
  __host__ __device__ int off_p() const { return off_q() + 512; }                        // float[2][64]
  __host__ __device__ int off_red() const { return off_p() + 512; }                      // float[2][4]
  __host__ __device__ int off_bar() const { return off_red() + 64; }
  __host__ __device__ int nbars() const { return 2 * R_NST + 8; }
  __host__ __device__ int off_misc() const { return off_bar() + 8 * nbars(); }
  __host__ __device__ int bytes() const { return off_misc() + 64; }
};

__device__ __forceinline__ uint32_t kmaj_off(int row, int piece) {   // piece = 8 bf16 (16 bytes)
  return (uint32_t)((row >> 3) * 1024 + (row & 7) * 128 + ((piece ^ (row & 7)) << 4));
}

__global__ void __launch_bounds__(RCT, 1)
recon_split_tc(const __grid_constant__ CUtensorMap mapK, const __grid_constant__ CUtensorMap mapV,
               const ReconArgs a, int* err) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  RLayout L;
  L.nch = (a.r + RCH - 1) / RCH;
  L.uk_rows = (a.d_h + 7) / 8 * 8;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int tt = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const int row = tt * a.H + h;
  const int dh = a.d_h, r = a.r, nch = L.nch;
  const int ntiles = (a.n_lat + RT_TOK - 1) / RT_TOK;

  uint64_t* bars = reinterpret_cast<uint64_t*>(base + L.off_bar());
  uint64_t* sfull = bars;                 // [R_NST] latent tile landed
  uint64_t* sempty = bars + R_NST;        // [R_NST] both MMAs of the tile done
  uint64_t* kready = bars + 2 * R_NST;    // [2] K^ in TMEM buffer
  uint64_t* vready = kready + 2;          // [2] V^T in TMEM buffer
  uint64_t* tfree = vready + 2;           // [2] softmax done with the buffer (128 arrivals)
  uint64_t* uready = tfree + 2;           // codec operands written (128 arrivals)
  uint64_t* fin = uready + 1;             // every MMA issued has completed
  uint8_t* misc = base + L.off_misc();
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(misc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(misc + 4);
  float* q_s = reinterpret_cast<float*>(base + L.off_q());
  float* p_s = reinterpret_cast<float*>(base + L.off_p());
  float* red = reinterpret_cast<float*>(base + L.off_red());

  if (tid == 0) {
    for (int i = 0; i < R_NST; ++i) {
      mbar_init(smem_u32(&sfull[i]), 1);
      mbar_init(smem_u32(&sempty[i]), 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(smem_u32(&kready[i]), 1);
      mbar_init(smem_u32(&vready[i]), 1);
      mbar_init(smem_u32(&tfree[i]), 128);
    }
    mbar_init(smem_u32(uready), 128);
    mbar_init(smem_u32(fin), 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 5) {
    tmem_alloc(smem_u32(tmem_slot), 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint32_t bufcols = (uint32_t)(dh + 64);   // K^ (d_h columns) then V^T (64 columns)

  if (warp == 4) {
    // ---------------------------------------------------------- TMA copies --
    if (lane == 0) {
      prefetch_tmap(&mapK);
      prefetch_tmap(&mapV);
      int issued = 0;
      for (int i = 0; i < ntiles; ++i) {
        const int st = i % R_NST;
        if (i >= R_NST && !rwait(smem_u32(&sempty[st]), ((i / R_NST) - 1) & 1, abort_flag, err, ERR_RECON_EMPTY))
          break;
        const uint32_t bar = smem_u32(&sfull[st]);
        const uint32_t dst = smem_u32(base + L.off_stage() + st * L.stage_bytes());
        mbar_arrive_tx(bar, (uint32_t)L.stage_bytes());
        for (int c = 0; c < nch; ++c) {
          tma_load_4d(dst + c * RT_TOK * 128, &mapK, bar, c * RCH, i * RT_TOK, h, b);
          tma_load_4d(dst + (nch + c) * RT_TOK * 128, &mapV, bar, c * RCH, i * RT_TOK, h, b);
        }
        issued = i + 1;
      }
      if (*abort_flag) {
        // leave no copy in flight: wait (bounded) for the stages issued last
        for (int i = max(0, issued - R_NST); i < issued; ++i)
          rwait(smem_u32(&sfull[i % R_NST]), (i / R_NST) & 1, abort_flag, nullptr, 0, false);
      }
    }
  } else if (warp == 5) {
    // ---------------------------------------------------------- MMA issue --
    if (lane == 0) {
      const uint32_t idK = idesc_bf16(64, dh, false, false);     // K^ = C^K U^K^T
      const uint32_t idV = idesc_bf16(128, 64, false, false);    // V^T = U^V C^V^T
      const uint32_t uk = smem_u32(base + L.off_uk()), uv = smem_u32(base + L.off_uv());
      bool ok = rwait(smem_u32(uready), 0, abort_flag, err, ERR_RECON_U);
      for (int i = 0; i < ntiles && ok; ++i) {
        const int st = i % R_NST, buf = i & 1;
        if (!rwait(smem_u32(&sfull[st]), (i / R_NST) & 1, abort_flag, err, ERR_RECON_STAGE)) { ok = false; break; }
        if (i >= 2 && !rwait(smem_u32(&tfree[buf]), ((i >> 1) - 1) & 1, abort_flag, err, ERR_RECON_TFREE)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t sk = smem_u32(base + L.off_stage() + st * L.stage_bytes());
        const uint32_t sv = sk + nch * RT_TOK * 128;
        const uint32_t dK = tmem + buf * bufcols, dV = dK + dh;
        for (int c = 0; c < nch; ++c) {
          const uint64_t ak = smem_desc_sw128(sk + c * RT_TOK * 128, 16, 1024);
          for (int part = 0; part < 2; ++part) {
            const uint64_t bk = smem_desc_sw128(uk + part * L.uk_bytes() + c * L.uk_rows * 128, 16, 1024);
#pragma unroll
            for (int k16 = 0; k16 < 4; ++k16)
              mma_bf16(dK, ak + 2 * k16, bk + 2 * k16, idK, (c | part | k16) != 0);
          }
        }
        mma_commit(smem_u32(&kready[buf]));
        for (int c = 0; c < nch; ++c) {
          const uint64_t bv = smem_desc_sw128(sv + c * RT_TOK * 128, 16, 1024);
          for (int part = 0; part < 2; ++part) {
            const uint64_t av = smem_desc_sw128(uv + part * L.uv_bytes() + c * 128 * 128, 16, 1024);
#pragma unroll
            for (int k16 = 0; k16 < 4; ++k16)
              mma_bf16(dV, av + 2 * k16, bv + 2 * k16, idV, (c | part | k16) != 0);
          }
        }
        mma_commit(smem_u32(&vready[buf]));
        mma_commit(smem_u32(&sempty[st]));
      }
      // every MMA issued must finish before TMEM is released
      mma_commit(smem_u32(fin));
      rwait(smem_u32(fin), 0, abort_flag, nullptr, 0, false);
    }
  } else {
    // ------------------------------------------------- codec split + softmax --
    // codec operands: U^K (d_h rows) and U^V (128 rows, zero past d_h), each
    // split into bf16 hi and lo, rank zero-padded to 64 * nch
    const float* UKg = a.UK + (int64_t)row * dh * r;
    const float* UVg = a.UV + (int64_t)row * dh * r;
    uint8_t* uk = base + L.off_uk();
    uint8_t* uv = base + L.off_uv();
    const int pieces_k = L.uk_rows * nch * 8, pieces_v = 128 * nch * 8;
    const int npieces = pieces_k + pieces_v;
    // four pieces (8 rank elements each) per thread per pass, loads first
    for (int p0 = tid; p0 < npieces; p0 += 4 * 128) {
      float4 ld[4][2];
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int p = p0 + 128 * u;
        ld[u][0] = ld[u][1] = make_float4(0.f, 0.f, 0.f, 0.f);
        if (p < npieces) {
          const bool isk = p < pieces_k;
          const int pp = isk ? p : p - pieces_k;
          const int rowu = pp / (nch * 8), rest = pp % (nch * 8);
          const int k0 = (rest >> 3) * RCH + (rest & 7) * 8;
          if (rowu < dh && k0 < r) {     // r % 8 == 0: a piece is wholly in or out of range
            const float4* src = reinterpret_cast<const float4*>((isk ? UKg : UVg) + (int64_t)rowu * r + k0);
            ld[u][0] = __ldg(src);
            ld[u][1] = __ldg(src + 1);
          }
        }
      }
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int p = p0 + 128 * u;
        if (p >= npieces) break;
        const bool isk = p < pieces_k;
        const int pp = isk ? p : p - pieces_k;
        const int rowu = pp / (nch * 8), rest = pp % (nch * 8), c = rest >> 3, piece = rest & 7;
        const float v[8] = {ld[u][0].x, ld[u][0].y, ld[u][0].z, ld[u][0].w,
                            ld[u][1].x, ld[u][1].y, ld[u][1].z, ld[u][1].w};
        uint32_t hi[4], lo[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const __nv_bfloat162 hv = __floats2bfloat162_rn(v[2 * e], v[2 * e + 1]);
          const float2 hf = __bfloat1622float2(hv);
          const __nv_bfloat162 lv = __floats2bfloat162_rn(v[2 * e] - hf.x, v[2 * e + 1] - hf.y);
          hi[e] = *reinterpret_cast<const uint32_t*>(&hv);
          lo[e] = *reinterpret_cast<const uint32_t*>(&lv);
        }
        uint8_t* t0 = isk ? uk + c * L.uk_rows * 128 : uv + c * 128 * 128;
        const int part_bytes = isk ? L.uk_bytes() : L.uv_bytes();
        const uint32_t off = kmaj_off(rowu, piece);
        *reinterpret_cast<uint4*>(t0 + off) = make_uint4(hi[0], hi[1], hi[2], hi[3]);
        *reinterpret_cast<uint4*>(t0 + part_bytes + off) = make_uint4(lo[0], lo[1], lo[2], lo[3]);
      }
    }
    for (int d = tid; d < 128; d += 128)
      q_s[d] = d < dh ? a.q[(int64_t)b * a.qs_b + (int64_t)row * dh + d] * a.qmul : 0.f;
    fence_proxy_async_smem();
    mbar_arrive(smem_u32(uready));
    named_sync(1, 128);

    const bool owner = lane < 16;                  // M = 64 layout: token 16 w + (lane & 15)
    const int tok = 16 * warp + (lane & 15);
    const int d = 32 * warp + lane;                // V^T row of this lane
    const uint32_t lane_off = (uint32_t)(32 * warp) << 16;
    float m_run = -INFINITY, l_run = 0.f, acc = 0.f;
    bool ok = true;
    for (int i = 0; i < ntiles; ++i) {
      const int buf = i & 1;
      if (!rwait(smem_u32(&kready[buf]), (i >> 1) & 1, abort_flag, err, ERR_RECON_K)) { ok = false; break; }
      tc_fence_after();
      const uint32_t tK = tmem + buf * bufcols + lane_off;
      // four independent partial sums, q read as float4
      float s4[4] = {0.f, 0.f, 0.f, 0.f};
      for (int c0 = 0; c0 < dh; c0 += 16) {
        float kv[16];
        tmem_ld16(tK + c0, kv);
        tmem_wait_ld();
        const float4* q4 = reinterpret_cast<const float4*>(q_s + c0);
#pragma unroll
        for (int g = 0; g < 4; ++g) {
          const float4 qq = q4[g];
          s4[g] = fmaf(kv[4 * g], qq.x, s4[g]);
          s4[g] = fmaf(kv[4 * g + 1], qq.y, s4[g]);
          s4[g] = fmaf(kv[4 * g + 2], qq.z, s4[g]);
          s4[g] = fmaf(kv[4 * g + 3], qq.w, s4[g]);
        }
      }
      float s = (s4[0] + s4[1]) + (s4[2] + s4[3]);
      const int nvalid = min(RT_TOK, a.n_lat - i * RT_TOK);
      if (!owner || tok >= nvalid) s = -INFINITY;
      // tile max over the 64 tokens: within the warp, then across the 4 warps
      float mx = s;
#pragma unroll
      for (int o = 8; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
      if (lane == 0) red[buf * 4 + warp] = mx;
      named_sync(1, 128);
      const float tmax = fmaxf(fmaxf(red[buf * 4 + 0], red[buf * 4 + 1]), fmaxf(red[buf * 4 + 2], red[buf * 4 + 3]));
      const float m_new = fmaxf(m_run, tmax);
      const float alpha = m_run == -INFINITY ? 0.f : ex2(m_run - m_new);
      const float p = s == -INFINITY ? 0.f : ex2(s - m_new);
      if (owner) p_s[buf * 64 + tok] = p;
      m_run = m_new;
      named_sync(1, 128);                          // p_s complete
      float tsum;
      {
        // every thread sums the 64 p values (smem broadcast), so l is uniform
        const float4* p4 = reinterpret_cast<const float4*>(p_s + buf * 64);
        float t4[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int j = 0; j < 16; ++j) {
          const float4 pp = p4[j];
          t4[j & 3] += (pp.x + pp.y) + (pp.z + pp.w);
        }
        tsum = (t4[0] + t4[1]) + (t4[2] + t4[3]);
      }
      l_run = l_run * alpha + tsum;
      if (!rwait(smem_u32(&vready[buf]), (i >> 1) & 1, abort_flag, err, ERR_RECON_V)) { ok = false; break; }
      tc_fence_after();
      const uint32_t tV = tmem + buf * bufcols + dh + lane_off;
      float y4[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int c0 = 0; c0 < 64; c0 += 16) {
        float vv[16];
        tmem_ld16(tV + c0, vv);
        tmem_wait_ld();
        const float4* p4 = reinterpret_cast<const float4*>(p_s + buf * 64 + c0);
#pragma unroll
        for (int g = 0; g < 4; ++g) {
          const float4 pp = p4[g];
          y4[g] = fmaf(pp.x, vv[4 * g], y4[g]);
          y4[g] = fmaf(pp.y, vv[4 * g + 1], y4[g]);
          y4[g] = fmaf(pp.z, vv[4 * g + 2], y4[g]);
          y4[g] = fmaf(pp.w, vv[4 * g + 3], y4[g]);
        }
      }
      const float y = (y4[0] + y4[1]) + (y4[2] + y4[3]);
      acc = acc * alpha + y;
      tc_fence_before();
      mbar_arrive(smem_u32(&tfree[buf]));
    }
    if (ok && !*abort_flag) {
      const int64_t br = (int64_t)b * a.rows + row;   // split 0: this kernel covers the whole latent range
      if (tid == 0) {
        a.part_ml[br * 2] = m_run;
        a.part_ml[br * 2 + 1] = l_run;
      }
      if (d < dh) a.part_y[br * dh + d] = acc;
    }
  }
  __syncthreads();
  if (warp == 5) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

}  // namespace

bool recon_tc_supported(const ReconArgs& a) {
  return a.lat_dtype == LLA_BF16 && a.r % 8 == 0 && a.r <= 128 && a.d_h % 16 == 0 && a.d_h <= 128 &&
         (a.ls_b * 2) % 16 == 0 && (a.ls_h * 2) % 16 == 0 && a.n_lat > 0;
}

cudaError_t launch_recon_split_tc(const ReconArgs& a, int* err, cudaStream_t st) {
  // latents [B][H][tokens][r] bf16: 4-D view (rank, token, head, sequence),
  // boxes of 64 rank elements x 64 tokens (rank past r reads as zero)
  CUtensorMap mk, mv;
  const cuuint64_t dims[4] = {(cuuint64_t)a.r, (cuuint64_t)a.n_lat, (cuuint64_t)a.H, (cuuint64_t)a.B};
  const cuuint64_t strides[3] = {(cuuint64_t)a.r * 2, (cuuint64_t)a.ls_h * 2, (cuuint64_t)a.ls_b * 2};
  const cuuint32_t box[4] = {RCH, RT_TOK, 1, 1};
  TmapEncodeFn enc = tmap_encoder();
  if (!enc) return cudaErrorNotSupported;
  cuuint32_t es[4] = {1, 1, 1, 1};
  for (int w = 0; w < 2; ++w) {
    const void* ptr = w == 0 ? a.cK : a.cV;
    if (enc(w == 0 ? &mk : &mv, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(ptr), dims, strides, box, es,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return cudaErrorNotSupported;
  }
  RLayout L;
  L.nch = (a.r + RCH - 1) / RCH;
  L.uk_rows = (a.d_h + 7) / 8 * 8;
  const size_t smem = 1024 + (size_t)L.bytes();
  if (smem > 232448) return cudaErrorNotSupported;
  cudaError_t e = cudaFuncSetAttribute(recon_split_tc, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  dim3 grid(a.nt, a.H, a.B);
  recon_split_tc<<<grid, RCT, smem, st>>>(mk, mv, a, err);
  return cudaGetLastError();
}

}  // namespace lla
