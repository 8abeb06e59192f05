// LLA reconstruct-on-read on the tensor cores (tcgen05 + TMEM).
//
// LLA abstract: the cache stores per-head latents c^K_{j,h}, c^V_{j,h} of rank
// r and rebuilds loop-specific keys and values only when attention reads them.
// For one head, every loop t reads the same latent tile, so one CTA serves a
// group of G loops of one head over SB sequences:
//   * the decoders U^K_t, U^V_t of its G loops are converted to bf16 once and
//     stay in shared memory for all SB sequences;
//   * each 128-token latent tile (C^K and C^V) is landed once by TMA and then
//     rebuilt for every loop of the group, so a tile crosses L2 once per group
//     instead of once per loop.
// Per (tile, loop) unit, both reconstructions are MMAs whose results never
// leave the SM:
//   K^_t  = C^K U^K_t^T   (M = 128 tokens, N = d_h, K = r): TMEM lane = token,
//   V^T_t = U^V_t C^V^T   (M = 128 >= d_h, N = 128 tokens): TMEM lane = feature.
// Two TMEM buffers alternate between units.  Four "key" warps read a token's
// rebuilt key per lane, score it against q (a 1 x d_h dot product, no
// cross-lane sum), run the online softmax over the tile and publish the
// probabilities; four "value" warps read one rebuilt feature row per lane and
// accumulate o[d] += sum_j p_j V^T[d][j].  A producer warp streams the tiles,
// two MMA warps issue the key and the value rebuilds.
//
// Precision: latents are bf16 and exact as MMA operands; each fp32 decoder is
// rounded to bf16 for the MMA (one product, fp32 accumulation), a relative
// error of about 2^-9 per decoder entry that stays far inside the bf16-latent
// tolerance of the read.  Rank chunks past r are zero (copy engine for the
// latents, the CTA for U).
//
// Waits are bounded; on a timeout the CTA records an error code (the merge then
// emits NaN), waits for its copies and MMAs, and frees TMEM.
#include <cuda.h>

#include <algorithm>
#include <cstdlib>
#include <cstring>

#include "kernels.cuh"
#include "tc_ptx.cuh"
#include "tmap.cuh"

namespace lla {
namespace {

using namespace ptx;

constexpr int RT_TOK = 128;           // tokens per tile (M of the key rebuild, N of the value rebuild)
constexpr int RCH = 32;               // rank elements per 64-byte chunk (64-byte swizzle)
constexpr int CHUNK_BYTES = RT_TOK * 64;   // one chunk block of a latent tile: 8 KB
constexpr int RCT = 352;              // warps 0-3 keys, 4-7 values, 8 TMA, 9 and 10 MMA
constexpr int MAXG = 4;               // loops per CTA at most
constexpr int R_NST = 2;              // latent stages
constexpr int NPB = 4;                // probability buffers (unit u uses u % NPB)
constexpr int SMEM_CAP = 232448;      // 227 KB per block (opt-in)
constexpr int SMEM_MIN = 120 * 1024;  // at least this much, so one CTA (and one TMEM owner) per SM
constexpr uint32_t TMEM_COLS = 512;   // buffer u: keys at 256 u, values at 256 u + 128
constexpr long long R_WAIT = 1ll << 32;

enum : int { ERR_RECON_STAGE = 31, ERR_RECON_KFREE = 32, ERR_RECON_U = 33, ERR_RECON_K = 34, ERR_RECON_V = 35,
             ERR_RECON_EMPTY = 36, ERR_RECON_VFREE = 37, ERR_RECON_P = 38 };

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

// Shared-memory plan (offsets from the 1 KB-aligned base).  Every operand is
// K-major in the 64-byte swizzle: a chunk of 32 rank elements holds its rows
// at 64 bytes each, 8-row atoms of 512 bytes, 16-byte pieces XOR-ed with
// bits 1..2 of the row.
struct RLayout {
  int nch;      // rank chunks of 32
  int G;        // loops per CTA
  int d_h;
  __host__ __device__ int ukr() const { return G * d_h; }                 // rows of the stacked U^K
  __host__ __device__ int uvr() const { return G * d_h + 128 - d_h; }     // rows of the stacked U^V (+ pad)
  __host__ __device__ int uk_chunk() const { return ukr() * 64; }
  __host__ __device__ int uv_chunk() const { return uvr() * 64; }
  __host__ __device__ int stage_bytes() const { return 2 * nch * CHUNK_BYTES; }  // C^K chunks then C^V
  __host__ __device__ int off_uk() const { return 0; }
  __host__ __device__ int off_uv() const { return (nch * uk_chunk() + 1023) / 1024 * 1024; }
  __host__ __device__ int off_stage() const { return (off_uv() + nch * uv_chunk() + 1023) / 1024 * 1024; }
  __host__ __device__ int off_q() const { return off_stage() + R_NST * stage_bytes(); }   // float[MAXG][128]
  __host__ __device__ int off_p() const { return off_q() + MAXG * 128 * 4; }             // float[NPB][128]
  __host__ __device__ int off_red() const { return off_p() + NPB * 128 * 4; }            // float[2][4] tile max
  __host__ __device__ int off_alpha() const { return off_red() + 32; }                   // float[NPB]
  __host__ __device__ int off_lred() const { return off_alpha() + 4 * NPB; }             // float[MAXG][4]
  __host__ __device__ int off_bar() const { return off_lred() + MAXG * 4 * 4; }
  __host__ __device__ int nbars() const { return 2 * R_NST + 4 * 2 + 2 * NPB + 3; }
  __host__ __device__ int off_misc() const { return off_bar() + 8 * nbars(); }
  __host__ __device__ int bytes() const { return off_misc() + 64; }
};

// Byte offset of the 16-byte piece `piece` (0..3) of row `row` inside a chunk
// region in the 64-byte swizzle.
__device__ __forceinline__ uint32_t sw64_off(int row, int piece) {
  return (uint32_t)((row >> 3) * 512 + (row & 7) * 64 + ((piece ^ ((row >> 1) & 3)) << 4));
}

__device__ __forceinline__ uint32_t pack2_bf16(float lo, float hi) {
  const __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<const uint32_t*>(&v);
}

// KMAX: d_h rounded up to 32 (the key row a key warp holds in registers).
template <int KMAX>
__global__ void __launch_bounds__(RCT, 1)
recon_group_tc(const __grid_constant__ CUtensorMap mapK, const __grid_constant__ CUtensorMap mapV,
               const ReconArgs a, const int G, const int SB, int* err) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  RLayout L;
  L.nch = (a.r + RCH - 1) / RCH;
  L.G = G;
  L.d_h = a.d_h;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int bc = blockIdx.x, lg = blockIdx.y, h = blockIdx.z;
  const int b0 = bc * SB;
  const int nb = min(SB, a.B - b0);
  const int tt0 = lg * G;                          // first loop of the group within the call
  const int Geff = min(G, a.nt - tt0);
  const int dh = a.d_h, r = a.r, nch = L.nch;
  const int ksteps = (r + 15) / 16;                // 16-element MMA steps along the rank
  const int ntiles = (a.n_lat + RT_TOK - 1) / RT_TOK;

  uint64_t* bars = reinterpret_cast<uint64_t*>(base + L.off_bar());
  uint64_t* sfull = bars;                 // [R_NST] latent tile landed
  uint64_t* sempty = bars + R_NST;        // [R_NST] every MMA reading the tile done
  uint64_t* kready = bars + 2 * R_NST;    // [2] K^ in TMEM buffer
  uint64_t* vready = kready + 2;          // [2] V^T in TMEM buffer
  uint64_t* kfree = vready + 2;           // [2] key warps done reading K^ (128 arrivals)
  uint64_t* vfree = kfree + 2;            // [2] value warps done reading V^T (128 arrivals)
  uint64_t* pfull = vfree + 2;            // [NPB] probabilities and rescale published (128 arrivals)
  uint64_t* pfree = pfull + NPB;          // [NPB] value warps done with them (128 arrivals)
  uint64_t* uready = pfree + NPB;         // decoder operands written (256 arrivals)
  uint64_t* fin = uready + 1;             // [2] every MMA of an issuer has completed
  uint8_t* misc = base + L.off_misc();
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(misc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(misc + 4);
  float* q_s = reinterpret_cast<float*>(base + L.off_q());
  float* p_s = reinterpret_cast<float*>(base + L.off_p());
  float* red = reinterpret_cast<float*>(base + L.off_red());
  float* alpha_s = reinterpret_cast<float*>(base + L.off_alpha());
  float* lred = reinterpret_cast<float*>(base + L.off_lred());

  if (tid == 0) {
    for (int i = 0; i < R_NST; ++i) {
      mbar_init(smem_u32(&sfull[i]), 1);
      mbar_init(smem_u32(&sempty[i]), 2);   // one commit per MMA issuer
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(smem_u32(&kready[i]), 1);
      mbar_init(smem_u32(&vready[i]), 1);
      mbar_init(smem_u32(&kfree[i]), 128);
      mbar_init(smem_u32(&vfree[i]), 128);
    }
    for (int i = 0; i < NPB; ++i) {
      mbar_init(smem_u32(&pfull[i]), 128);
      mbar_init(smem_u32(&pfree[i]), 128);
    }
    mbar_init(smem_u32(uready), 256);
    mbar_init(smem_u32(fin), 1);
    mbar_init(smem_u32(fin + 1), 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 9) {
    tmem_alloc(smem_u32(tmem_slot), TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  griddep_wait();

  if (warp == 8) {
    // ---------------------------------------------------------- TMA copies --
    if (lane == 0) {
      prefetch_tmap(&mapK);
      prefetch_tmap(&mapV);
      int issued = 0;
      bool ok = true;
      for (int sb = 0; sb < nb && ok; ++sb) {
        const int b = b0 + sb;
        for (int n = 0; n < ntiles; ++n) {
          const int i = sb * ntiles + n;
          const int st = i % R_NST;
          if (i >= R_NST && !rwait(smem_u32(&sempty[st]), ((i / R_NST) - 1) & 1, abort_flag, err, ERR_RECON_EMPTY)) {
            ok = false;
            break;
          }
          const uint32_t bar = smem_u32(&sfull[st]);
          const uint32_t dst = smem_u32(base + L.off_stage() + st * L.stage_bytes());
          mbar_arrive_tx(bar, (uint32_t)L.stage_bytes());
          for (int c = 0; c < nch; ++c) {
            tma_load_4d(dst + c * CHUNK_BYTES, &mapK, bar, c * RCH, n * RT_TOK, h, b);
            tma_load_4d(dst + (nch + c) * CHUNK_BYTES, &mapV, bar, c * RCH, n * RT_TOK, h, b);
          }
          issued = i + 1;
        }
      }
      if (*abort_flag) {
        // leave no copy in flight: wait (bounded) for the stages issued last
        for (int i = max(0, issued - R_NST); i < issued; ++i)
          rwait(smem_u32(&sfull[i % R_NST]), (i / R_NST) & 1, abort_flag, nullptr, 0, false);
      }
    }
  } else if (warp == 9 || warp == 10) {
    // --------------------------------------------------------- MMA issuers --
    // Unit v = (sequence, tile, loop) in order; tile i = v / Geff.  A single
    // issuing thread is bound by its own issue latency (a few hundred cycles
    // per MMA, whatever its size), so the key rebuilds (warp 9) and the value
    // rebuilds (warp 10) each get an issuer and run side by side on the
    // tensor pipe.  A tile's stage is released when both have committed.
    if (lane == 0) {
      const bool keys = warp == 9;
      const uint32_t idK = idesc_bf16(128, dh, false, false);        // K^ = C^K U^K^T
      const uint32_t idV = idesc_bf16(128, RT_TOK, false, false);    // V^T = U^V C^V^T
      // base descriptors; an offset of k bytes adds k >> 4 (addresses < 256 KB)
      const uint64_t d_stage = smem_desc_sw64(smem_u32(base + L.off_stage()));
      const uint64_t d_uk = smem_desc_sw64(smem_u32(base + L.off_uk()));
      const uint64_t d_uv = smem_desc_sw64(smem_u32(base + L.off_uv()));
      const uint32_t stage_b = (uint32_t)L.stage_bytes(), ukc = (uint32_t)L.uk_chunk(), uvc = (uint32_t)L.uv_chunk();
      const uint32_t U = (uint32_t)(nb * ntiles * Geff);
      bool ok = rwait(smem_u32(uready), 0, abort_flag, err, ERR_RECON_U);
      for (uint32_t v = 0; v < U && ok; ++v) {
        const uint32_t i = v / Geff, g = v % Geff, st = i % R_NST, buf = v & 1;
        if (g == 0 && !rwait(smem_u32(&sfull[st]), (i / R_NST) & 1, abort_flag, err, ERR_RECON_STAGE)) {
          ok = false;
          break;
        }
        if (keys) {
          if (v >= 2 && !rwait(smem_u32(&kfree[buf]), ((v >> 1) - 1) & 1, abort_flag, err, ERR_RECON_KFREE)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint64_t a0 = d_stage + ((st * stage_b) >> 4);
          const uint64_t b0 = d_uk + ((g * (uint32_t)dh * 64) >> 4);
          for (int ks = 0; ks < ksteps; ++ks) {
            const uint32_t c = ks >> 1, half = ks & 1;
            mma_bf16(tmem + 256 * buf, a0 + ((c * CHUNK_BYTES + half * 32) >> 4), b0 + ((c * ukc + half * 32) >> 4),
                     idK, ks != 0);
          }
          mma_commit(smem_u32(&kready[buf]));
        } else {
          if (v >= 2 && !rwait(smem_u32(&vfree[buf]), ((v >> 1) - 1) & 1, abort_flag, err, ERR_RECON_VFREE)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint64_t a0 = d_uv + ((g * (uint32_t)dh * 64) >> 4);
          const uint64_t b0 = d_stage + ((st * stage_b + (uint32_t)nch * CHUNK_BYTES) >> 4);
          for (int ks = 0; ks < ksteps; ++ks) {
            const uint32_t c = ks >> 1, half = ks & 1;
            mma_bf16(tmem + 256 * buf + 128, a0 + ((c * uvc + half * 32) >> 4), b0 + ((c * CHUNK_BYTES + half * 32) >> 4),
                     idV, ks != 0);
          }
          mma_commit(smem_u32(&vready[buf]));
        }
        if (g == (uint32_t)Geff - 1) mma_commit(smem_u32(&sempty[st]));   // this issuer's last read of tile i
      }
      // every MMA this thread issued must finish before TMEM is released
      const uint32_t f = smem_u32(fin) + (keys ? 0 : 8);
      mma_commit(f);
      rwait(f, 0, abort_flag, nullptr, 0, false);
    }
  } else {
    // --------------------------------------- decoder operands (warps 0-7) --
    // U^K and U^V of the group's loops, rounded to bf16, rank zero-padded to
    // 32 nch.  The stacked U^V gets 128 - d_h zero rows after the last loop:
    // the value rebuild reads 128 rows from each loop's first row.
    {
      uint8_t* uk = base + L.off_uk();
      uint8_t* uv = base + L.off_uv();
      const int pieces_row = nch * 4;                       // 16-byte pieces (8 elements) per row
      const int rows_k = Geff * dh;
      const int rows_v = Geff * dh + 128 - dh;
      const int total = (rows_k + rows_v) * pieces_row;
      for (int p = tid; p < total; p += 256) {
        const bool isk = p < rows_k * pieces_row;
        const int pp = isk ? p : p - rows_k * pieces_row;
        const int row = pp / pieces_row, rest = pp % pieces_row;
        const int c = rest >> 2, piece = rest & 3;
        const int k0 = c * RCH + piece * 8;
        float v[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
        if (row < rows_k && k0 < r) {      // r % 8 == 0: a piece is wholly in or out of range
          const int g = row / dh, d = row % dh;
          const float* src = (isk ? a.UK : a.UV) + ((int64_t)(tt0 + g) * a.H + h) * dh * r + (int64_t)d * r + k0;
          const float4 x0 = __ldg(reinterpret_cast<const float4*>(src));
          const float4 x1 = __ldg(reinterpret_cast<const float4*>(src) + 1);
          v[0] = x0.x; v[1] = x0.y; v[2] = x0.z; v[3] = x0.w;
          v[4] = x1.x; v[5] = x1.y; v[6] = x1.z; v[7] = x1.w;
        }
        uint8_t* dst = (isk ? uk + c * L.uk_chunk() : uv + c * L.uv_chunk()) + sw64_off(row, piece);
        *reinterpret_cast<uint4*>(dst) = make_uint4(pack2_bf16(v[0], v[1]), pack2_bf16(v[2], v[3]),
                                                    pack2_bf16(v[4], v[5]), pack2_bf16(v[6], v[7]));
      }
      fence_proxy_async_smem();
      mbar_arrive(smem_u32(uready));
    }

    if (warp < 4) {
      // ------------------------------------------------------ key warps --
      const int tok = tid;                          // TMEM lane of the key rebuild
      const uint32_t lane_off = (uint32_t)(32 * warp) << 16;
      float m_run[MAXG], l_part[MAXG];
      bool ok = true;
      uint32_t u = 0;
      for (int sb = 0; sb < nb && ok; ++sb) {
        const int b = b0 + sb;
        // this sequence's queries, scaled to base-2 score units
        for (int x = tid; x < Geff * 128; x += 128) {
          const int g = x >> 7, d = x & 127;
          q_s[x] = d < dh ? a.q[(int64_t)b * a.qs_b + ((int64_t)(tt0 + g) * a.H + h) * dh + d] * a.qmul : 0.f;
        }
        named_sync(1, 128);
#pragma unroll
        for (int g = 0; g < MAXG; ++g) { m_run[g] = -INFINITY; l_part[g] = 0.f; }
        for (int n = 0; n < ntiles && ok; ++n) {
          const int nvalid = min(RT_TOK, a.n_lat - n * RT_TOK);
#pragma unroll
          for (int g = 0; g < MAXG; ++g) {
            if (g >= Geff) break;
            const uint32_t buf = u & 1, pb = u % NPB;
            // tcgen05.ld is warp-collective: the whole warp takes or skips it
            const bool okk = __all_sync(0xffffffffu, rwait(smem_u32(&kready[buf]), (u >> 1) & 1, abort_flag, err,
                                                            ERR_RECON_K));
            float s = -INFINITY;
            if (okk) {
              tc_fence_after();
              const uint32_t tK = tmem + 256 * buf + lane_off;
              // the whole key row in flight before one wait (two waits for
              // d_h > 96, which would not fit the registers); the conditions
              // are warp-uniform
              constexpr int KB = KMAX > 96 ? KMAX / 2 : KMAX;
              float s8[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
#pragma unroll
              for (int h0 = 0; h0 < KMAX; h0 += KB) {
                float kv[KB];
#pragma unroll
                for (int c0 = 0; c0 < KB; c0 += 16)
                  if (h0 + c0 < dh) tmem_ld16(tK + h0 + c0, kv + c0);
                tmem_wait_ld();
                if (h0 + KB >= KMAX) {
                  tc_fence_before();
                  mbar_arrive(smem_u32(&kfree[buf]));
                }
#pragma unroll
                for (int c0 = 0; c0 < KB; c0 += 16) {
                  if (h0 + c0 >= dh) break;
                  const float4* q4 = reinterpret_cast<const float4*>(q_s + g * 128 + h0 + c0);
#pragma unroll
                  for (int e = 0; e < 4; ++e) {
                    const float4 qq = q4[e];
                    const int k = (e & 1) * 4;
                    s8[k + 0] = fmaf(kv[c0 + 4 * e], qq.x, s8[k + 0]);
                    s8[k + 1] = fmaf(kv[c0 + 4 * e + 1], qq.y, s8[k + 1]);
                    s8[k + 2] = fmaf(kv[c0 + 4 * e + 2], qq.z, s8[k + 2]);
                    s8[k + 3] = fmaf(kv[c0 + 4 * e + 3], qq.w, s8[k + 3]);
                  }
                }
              }
              const float sd = ((s8[0] + s8[1]) + (s8[2] + s8[3])) + ((s8[4] + s8[5]) + (s8[6] + s8[7]));
              s = tok < nvalid ? sd : -INFINITY;
            }
            const float wmax = redux_max(s);
            if (lane == 0) red[buf * 4 + warp] = wmax;
            // probability buffer pb is free once the value warps finished unit u - NPB
            const bool okp = okk && (u < NPB || rwait(smem_u32(&pfree[pb]), ((u / NPB) - 1) & 1, abort_flag, err,
                                                      ERR_RECON_VFREE));
            // barrier over the key warps that also agrees on the outcome
            if (named_any(1, 128, !okp)) { ok = false; break; }
            const float tmax = fmaxf(fmaxf(red[buf * 4 + 0], red[buf * 4 + 1]), fmaxf(red[buf * 4 + 2], red[buf * 4 + 3]));
            const float m_new = fmaxf(m_run[g], tmax);
            const float alpha = m_run[g] == -INFINITY ? 0.f : ex2(m_run[g] - m_new);
            const float p = s == -INFINITY ? 0.f : ex2(s - m_new);
            p_s[pb * 128 + tok] = p;
            if (tid == 0) alpha_s[pb] = alpha;
            l_part[g] = l_part[g] * alpha + p;
            m_run[g] = m_new;
            mbar_arrive(smem_u32(&pfull[pb]));
            ++u;
          }
        }
        if (!ok) break;
        // end of the sequence: l = sum of the per-token partial sums
#pragma unroll
        for (int g = 0; g < MAXG; ++g) {
          if (g >= Geff) break;
          const float ws = warp_sum(l_part[g]);
          if (lane == 0) lred[g * 4 + warp] = ws;
        }
        named_sync(1, 128);
        if (tid < Geff) {
          const int g = tid;
          const float l = (lred[g * 4 + 0] + lred[g * 4 + 1]) + (lred[g * 4 + 2] + lred[g * 4 + 3]);
          float mg = m_run[0];
#pragma unroll
          for (int x = 1; x < MAXG; ++x)
            if (x == g) mg = m_run[x];
          const int64_t br = (int64_t)b * a.rows + (int64_t)(tt0 + g) * a.H + h;
          a.part_ml[br * 2] = mg;
          a.part_ml[br * 2 + 1] = l;
        }
        named_sync(1, 128);    // lred and q_s are rewritten for the next sequence
      }
    } else {
      // ---------------------------------------------------- value warps --
      const int vw = warp - 4;
      const int d = 32 * vw + lane;                 // TMEM lane of the value rebuild = feature
      const uint32_t lane_off = (uint32_t)(32 * vw) << 16;
      float o[MAXG];
      bool ok = true;
      uint32_t u = 0;
      for (int sb = 0; sb < nb && ok; ++sb) {
        const int b = b0 + sb;
#pragma unroll
        for (int g = 0; g < MAXG; ++g) o[g] = 0.f;
        for (int n = 0; n < ntiles && ok; ++n) {
#pragma unroll
          for (int g = 0; g < MAXG; ++g) {
            if (g >= Geff) break;
            const uint32_t buf = u & 1, pb = u % NPB;
            const bool okw = rwait(smem_u32(&vready[buf]), (u >> 1) & 1, abort_flag, err, ERR_RECON_V) &&
                             rwait(smem_u32(&pfull[pb]), (u / NPB) & 1, abort_flag, err, ERR_RECON_P);
            if (!__all_sync(0xffffffffu, okw)) {   // tcgen05.ld below is warp-collective
              ok = false;
              break;
            }
            tc_fence_after();
            const float alpha = alpha_s[pb];
            const uint32_t tV = tmem + 256 * buf + 128 + lane_off;
            // 64 columns in flight per wait
            float y8[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
#pragma unroll
            for (int h0 = 0; h0 < RT_TOK; h0 += 64) {
              float vv[64];
#pragma unroll
              for (int c0 = 0; c0 < 64; c0 += 16) tmem_ld16(tV + h0 + c0, vv + c0);
              tmem_wait_ld();
              if (h0 + 64 >= RT_TOK) {
                tc_fence_before();
                mbar_arrive(smem_u32(&vfree[buf]));
              }
#pragma unroll
              for (int c0 = 0; c0 < 64; c0 += 16) {
                const float4* p4 = reinterpret_cast<const float4*>(p_s + pb * 128 + h0 + c0);
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                  const float4 pp = p4[e];
                  const int k = (e & 1) * 4;
                  y8[k + 0] = fmaf(pp.x, vv[c0 + 4 * e], y8[k + 0]);
                  y8[k + 1] = fmaf(pp.y, vv[c0 + 4 * e + 1], y8[k + 1]);
                  y8[k + 2] = fmaf(pp.z, vv[c0 + 4 * e + 2], y8[k + 2]);
                  y8[k + 3] = fmaf(pp.w, vv[c0 + 4 * e + 3], y8[k + 3]);
                }
              }
            }
            mbar_arrive(smem_u32(&pfree[pb]));
            const float y = ((y8[0] + y8[1]) + (y8[2] + y8[3])) + ((y8[4] + y8[5]) + (y8[6] + y8[7]));
            o[g] = o[g] * alpha + y;
            ++u;
          }
        }
        if (!ok) break;
        if (d < dh) {
#pragma unroll
          for (int g = 0; g < MAXG; ++g) {
            if (g >= Geff) break;
            const int64_t br = (int64_t)b * a.rows + (int64_t)(tt0 + g) * a.H + h;
            a.part_y[br * dh + d] = o[g];
          }
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 9) {
    tc_fence_after();
    tmem_dealloc(tmem, TMEM_COLS);
  }
  griddep_launch();
}

struct ReconPlan { int G, SB, smem; };

int smem_for(int r, int d_h, int G) {
  RLayout L;
  L.nch = (r + RCH - 1) / RCH;
  L.G = G;
  L.d_h = d_h;
  return 1024 + L.bytes();
}

// Loops per CTA: as many as shared memory holds (at most MAXG and nt).
// Sequences per CTA: the count with the smallest modelled time, where a CTA
// costs its units (tiles x loops x sequences) plus a start-up of about six
// units (barriers, TMEM, decoder conversion, pipeline fill), in waves of one
// CTA per SM.  LLA_RECON_SEQ_PER_CTA overrides the sequence count (tuning and
// tests).
ReconPlan recon_plan(const ReconArgs& a, int num_sms) {
  ReconPlan p{0, 1, 0};
  for (int G = std::min(MAXG, a.nt); G >= 1; --G) {
    if (smem_for(a.r, a.d_h, G) <= SMEM_CAP) { p.G = G; break; }
  }
  if (p.G == 0) return p;
  p.smem = std::max(smem_for(a.r, a.d_h, p.G), SMEM_MIN);
  const long groups = (long)((a.nt + p.G - 1) / p.G) * a.H;
  const long tiles = (a.n_lat + RT_TOK - 1) / RT_TOK;
  double best = 1e300;
  for (int SB = 1; SB <= a.B; SB *= 2) {
    const long ctas = groups * ((a.B + SB - 1) / SB);
    const long waves = (ctas + num_sms - 1) / num_sms;
    const double t = (double)waves * ((double)SB * tiles * p.G + 6.0 * p.G);
    if (t < best * 0.98) { best = t; p.SB = SB; }
  }
  if (const char* env = std::getenv("LLA_RECON_SEQ_PER_CTA")) {
    const int v = std::atoi(env);
    if (v >= 1) p.SB = std::min(v, a.B);
  }
  return p;
}

}  // namespace

bool recon_tc_supported(const ReconArgs& a) {
  if (!(a.lat_dtype == LLA_BF16 && a.r % 8 == 0 && a.r <= 128 && a.d_h % 16 == 0 && a.d_h <= 128 &&
        (a.ls_b * 2) % 16 == 0 && (a.ls_h * 2) % 16 == 0 && a.n_lat > 0))
    return false;
  return smem_for(a.r, a.d_h, 1) <= SMEM_CAP;
}

cudaError_t launch_recon_tc(const ReconArgs& a, int* err, cudaStream_t st, int num_sms) {
  // latents [B][H][tokens][r] bf16: 4-D view (rank, token, head, sequence),
  // boxes of 32 rank elements x 128 tokens (64-byte swizzle; rank past r and
  // tokens past n_lat read as zero)
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
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_64B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return cudaErrorNotSupported;
  }
  const ReconPlan p = recon_plan(a, num_sms);
  if (p.G == 0) return cudaErrorNotSupported;
  const int kmax = (a.d_h + 31) / 32 * 32;
  auto kern = kmax <= 32 ? recon_group_tc<32> : kmax <= 64 ? recon_group_tc<64>
            : kmax <= 96 ? recon_group_tc<96> : recon_group_tc<128>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, p.smem);
  if (e != cudaSuccess) return e;
  // sequence chunks fastest: the CTAs that share a group's decoders run side
  // by side, then the loop groups of a head (which share its latent stream)
  dim3 grid((a.B + p.SB - 1) / p.SB, (a.nt + p.G - 1) / p.G, a.H);
  return launch_kernel(kern, grid, dim3(RCT), (size_t)p.smem, st, 1, mk, mv, a, p.G, p.SB, err);
}

}  // namespace lla
