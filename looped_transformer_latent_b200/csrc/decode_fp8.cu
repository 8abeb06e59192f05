// Absorbed latent read of fp8 latent rows (e4m3 codes with per-token, per-part
// scales) on the 5th-generation tensor cores.
//
// The same read as absorb_split_tc (HLA summary, "Latent Reader", eqs. 3-4;
// LLA-D) over rows stored as [codes of c^K | codes of c^V | s^K | s^V | pad]
// (HLA summary, "Conclusion / Future directions": latents combined with
// quantisation).  Since a stored element is code * s of its part and s is one
// number per token and part,
//   S[row, j]  = s^K_j * (q~[row, :] . codes^K_j)
//   O^T[v, row] += sum_j codes^V_j[v] * (P[row, j] * s^V_j)
// so the tensor cores contract the codes and the scales are applied per token
// on the softmax side.  Per 64-token tile:
//   * two producer warps land the key and the value chunks (64 tokens x 64
//     codes, 4 KB each) in fp8 landing rings, and one 1 KB box of the tile's
//     scales;
//   * two converter pairs widen the codes to f16 (exact: every e4m3 value is
//     an f16 value) into 128-byte-swizzled slots, the layout the MMAs read;
//   * two MMA warps issue S = Q~ codes^K^T (M=64 x N=64, f16 in, fp32 in
//     TMEM) and O^T += codes^V^T P'^T (M=128 x N=rows) on independent chains;
//   * four softmax warps scale the scores by s^K, run the online softmax and
//     write P' = p * s^V in f16 for the value MMA (l sums p itself).
// Every wait is bounded; on a timeout the CTA records an error code (the merge
// then emits NaN), drains its copies and frees TMEM.
#include <cuda.h>
#include <cuda_fp16.h>
#include <cuda_fp8.h>

#include "kernels.cuh"
#include "tc_ptx.cuh"
#include "tmap.cuh"

namespace lla {
namespace {

using namespace ptx;

constexpr int TOK = 64;
constexpr int BLK = 8192;             // f16 chunk block: 64 tokens x 64 elements, 128-byte rows, swizzled
constexpr int BLK8 = 4096;            // fp8 chunk block as landed: 64 tokens x 64 codes
constexpr int LSLOT = 2 * BLK8;       // landing slot: one or two chunks
constexpr int CSLOT = 2 * BLK;        // converted slot: one or two chunks
constexpr int NL = 3;                 // landing slots per ring
constexpr int NC = 2;                 // converted slots per ring
constexpr int NSB = 4;                // scale slots (one per tile)
constexpr int SBYTES = TOK * 16;      // one tile's scales: 64 x (s^K, s^V, 8 pad bytes)
constexpr int NBUF = 3;               // score buffers (TMEM) and P buffers (smem)
constexpr int NTHREADS = 384;         // 0-3 softmax, 4/6 producers, 5/7 MMA, 8-9/10-11 converters
constexpr int SMEM_LIMIT = 232448;
constexpr int MISC_BYTES = 512;
constexpr long long WAIT_CYCLES = 1ll << 32;
constexpr uint32_t TMEM_COLS = 512;
constexpr uint32_t O_COL = 64 * NBUF;

enum : int { ERR8_LEMPTY = 51, ERR8_LFULL = 52, ERR8_CEMPTY = 53, ERR8_CFULL = 54, ERR8_Q = 55, ERR8_S = 56,
             ERR8_P = 57, ERR8_O = 58, ERR8_SC = 59 };

__device__ __forceinline__ bool wait8(uint32_t bar, uint32_t parity, volatile int* abort_flag, int* err, int code,
                                      bool honour_abort = true) {
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

__device__ __forceinline__ uint32_t pack_f16(float lo, float hi) {
  const __half2 v = __floats2half2_rn(lo, hi);
  return *reinterpret_cast<const uint32_t*>(&v);
}

// four e4m3 codes (one 32-bit word, lowest byte first) -> four f16, exactly
__device__ __forceinline__ uint2 widen4(uint32_t w) {
  const __half2_raw lo = __nv_cvt_fp8x2_to_halfraw2((__nv_fp8x2_storage_t)(w & 0xFFFFu), __NV_E4M3);
  const __half2_raw hi = __nv_cvt_fp8x2_to_halfraw2((__nv_fp8x2_storage_t)(w >> 16), __NV_E4M3);
  return make_uint2((uint32_t)lo.x | ((uint32_t)lo.y << 16), (uint32_t)hi.x | ((uint32_t)hi.y << 16));
}

struct Layout8 {
  int nkb, nvb;
  __host__ __device__ int q_off() const { return 0; }
  __host__ __device__ int p_off() const { return nkb * BLK; }
  __host__ __device__ int sc_off() const { return p_off() + NBUF * BLK; }
  __host__ __device__ int lk_off() const { return sc_off() + NSB * SBYTES; }
  __host__ __device__ int lv_off() const { return lk_off() + NL * LSLOT; }
  __host__ __device__ int ck_off() const { return lv_off() + NL * LSLOT; }
  __host__ __device__ int cv_off() const { return ck_off() + NC * CSLOT; }
  __host__ __device__ int bar_off() const { return cv_off() + NC * CSLOT; }
  __host__ __device__ int nbars() const { return 4 * NL + 4 * NC + 2 * NSB + 1 + 4 * NBUF + 2; }
  __host__ __device__ int misc_off() const { return bar_off() + 8 * nbars(); }
  __host__ __device__ int bytes() const { return misc_off() + MISC_BYTES; }
};

__global__ void __launch_bounds__(NTHREADS, 1)
absorb_split_fp8(const __grid_constant__ CUtensorMap map2, const __grid_constant__ CUtensorMap map1,
                 const __grid_constant__ CUtensorMap mapsc, const AbsorbArgs a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  Layout8 L;
  L.nkb = a.r_k / 64; L.nvb = a.r_v / 64;
  uint8_t* q_s = base + L.q_off();
  uint8_t* p_s = base + L.p_off();
  uint8_t* sc_s = base + L.sc_off();
  uint64_t* bars = reinterpret_cast<uint64_t*>(base + L.bar_off());
  uint64_t* lk_full = bars;               // [NL] key codes landed
  uint64_t* lk_empty = lk_full + NL;      // [NL] key codes converted (64 arrivals)
  uint64_t* lv_full = lk_empty + NL;
  uint64_t* lv_empty = lv_full + NL;
  uint64_t* ck_full = lv_empty + NL;      // [NC] f16 key chunks written (64 arrivals)
  uint64_t* ck_empty = ck_full + NC;      // [NC] score MMAs reading them done
  uint64_t* cv_full = ck_empty + NC;
  uint64_t* cv_empty = cv_full + NC;
  uint64_t* sc_full = cv_empty + NC;      // [NSB] a tile's scales landed
  uint64_t* sc_free = sc_full + NSB;      // [NSB] softmax done with them (128 arrivals)
  uint64_t* q_full = sc_free + NSB;
  uint64_t* s_full = q_full + 1;          // [NBUF]
  uint64_t* s_free = s_full + NBUF;
  uint64_t* p_full = s_free + NBUF;
  uint64_t* o_done = p_full + NBUF;
  uint64_t* fin = o_done + NBUF;          // [2] one per MMA issuer (abort path)
  uint8_t* misc = base + L.misc_off();
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(misc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(misc + 4);
  volatile int* lead = reinterpret_cast<volatile int*>(misc + 16);   // [4]
  float* alpha_s = reinterpret_cast<float*>(misc + 64);               // [64]

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int s = blockIdx.x, b = blockIdx.y;
  const int tok0 = s * a.tps;
  const int tok1 = min(a.n_lat, tok0 + a.tps);
  const int ntiles = (tok1 - tok0 + TOK - 1) / TOK;
  const int nkb = L.nkb, nvb = L.nvb, ngrp = (nvb + 1) / 2;
  const int rows = a.rows, rows_pad = a.rows_pad;

  if (tid == 0) {
    for (int i = 0; i < NL; ++i) {
      mbar_init(smem_u32(&lk_full[i]), 1);
      mbar_init(smem_u32(&lk_empty[i]), 64);
      mbar_init(smem_u32(&lv_full[i]), 1);
      mbar_init(smem_u32(&lv_empty[i]), 64);
    }
    for (int i = 0; i < NC; ++i) {
      mbar_init(smem_u32(&ck_full[i]), 64);
      mbar_init(smem_u32(&ck_empty[i]), 1);
      mbar_init(smem_u32(&cv_full[i]), 64);
      mbar_init(smem_u32(&cv_empty[i]), 1);
    }
    for (int i = 0; i < NSB; ++i) {
      mbar_init(smem_u32(&sc_full[i]), 1);
      mbar_init(smem_u32(&sc_free[i]), 128);
    }
    mbar_init(smem_u32(q_full), 1);
    for (int i = 0; i < NBUF; ++i) {
      mbar_init(smem_u32(&s_full[i]), 1);
      mbar_init(smem_u32(&s_free[i]), 128);
      mbar_init(smem_u32(&p_full[i]), 128);
      mbar_init(smem_u32(&o_done[i]), 1);
    }
    mbar_init(smem_u32(fin), 1);
    mbar_init(smem_u32(fin + 1), 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 5) {
    tmem_alloc(smem_u32(tmem_slot), TMEM_COLS);
    tmem_relinquish();
  }
  if (warp == 4 && lane == 0) {
    prefetch_tmap(&map2);
    prefetch_tmap(&map1);
    prefetch_tmap(&mapsc);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 4 || warp == 6) {
    // ----------------------------------------------------------- producers --
    // Warp 4: Q~ (one bulk copy), then per tile the scales and the key chunks;
    // warp 6: the value chunks.  Copies carry two chunks (one for an odd last
    // chunk); copy i of a ring goes to landing slot i mod NL.
    if (lane == 0) {
      const bool kside = warp == 4;
      const int nb = kside ? nkb : nvb, c0 = kside ? 0 : nkb;
      uint8_t* ring = base + (kside ? L.lk_off() : L.lv_off());
      const uint32_t full0 = smem_u32(kside ? lk_full : lv_full), empty0 = smem_u32(kside ? lk_empty : lv_empty);
      const uint32_t qb = smem_u32(q_full);
      if (kside) {
        mbar_arrive_tx(qb, nkb * BLK);
        bulk_load(smem_u32(q_s), a.qbf + (size_t)b * nkb * (BLK / 2), nkb * BLK, qb);
      }
      uint32_t i = 0;
      int nsc = 0;
      bool ok = true;
      for (int n = 0; n < ntiles && ok; ++n) {
        const int y = tok0 + n * TOK;
        if (kside) {
          const int ss = n % NSB;
          if (!wait8(smem_u32(&sc_free[ss]), ((n / NSB) & 1) ^ 1, abort_flag, a.err, ERR8_SC)) { ok = false; break; }
          mbar_arrive_tx(smem_u32(&sc_full[ss]), SBYTES);
          tma_load_3d(smem_u32(sc_s + ss * SBYTES), &mapsc, smem_u32(&sc_full[ss]), 0, y, b);
          nsc = n + 1;
        }
        for (int c = 0; c < nb; c += 2, ++i) {
          const int cnt = nb - c >= 2 ? 2 : 1;
          const uint32_t slot = i % NL;
          if (!wait8(empty0 + 8 * slot, ((i / NL) & 1) ^ 1, abort_flag, a.err, ERR8_LEMPTY)) { ok = false; break; }
          mbar_arrive_tx(full0 + 8 * slot, cnt * BLK8);
          tma_load_4d(smem_u32(ring + slot * LSLOT), cnt == 2 ? (const void*)&map2 : (const void*)&map1,
                      full0 + 8 * slot, 0, y, c0 + c, b);
        }
      }
      if (!ok) {
        // drain: every copy this producer issued must land before the CTA exits
        if (kside) {
          wait8(qb, 0, abort_flag, nullptr, 0, false);
          for (int n = max(0, nsc - NSB); n < nsc; ++n)
            wait8(smem_u32(&sc_full[n % NSB]), (n / NSB) & 1, abort_flag, nullptr, 0, false);
        }
        for (uint32_t k = (i > (uint32_t)NL ? i - NL : 0); k < i; ++k)
          wait8(full0 + 8 * (k % NL), (k / NL) & 1, abort_flag, nullptr, 0, false);
      }
    }
  } else if (warp >= 8) {
    // ----------------------------------------------------------- converters --
    // Warps 8-9 widen the key chunks, 10-11 the value chunks, copy by copy in
    // the producers' order: 16 codes (one 16-byte piece of a landed token row)
    // per task become two 16-byte f16 pieces of the swizzled slot.
    const bool kside = warp < 10;
    const int ct = tid - (kside ? 256 : 320);      // 0..63
    const int nb = kside ? nkb : nvb;
    const uint8_t* land = base + (kside ? L.lk_off() : L.lv_off());
    uint8_t* conv = base + (kside ? L.ck_off() : L.cv_off());
    const uint32_t lfull = smem_u32(kside ? lk_full : lv_full), lempty = smem_u32(kside ? lk_empty : lv_empty);
    const uint32_t cfull = smem_u32(kside ? ck_full : cv_full), cempty = smem_u32(kside ? ck_empty : cv_empty);
    uint32_t i = 0;
    bool ok = true;
    for (int n = 0; n < ntiles && ok; ++n) {
      for (int c = 0; c < nb && ok; c += 2, ++i) {
        const int cnt = nb - c >= 2 ? 2 : 1;
        const uint32_t ls = i % NL, cs = i % NC;
        if (!wait8(lfull + 8 * ls, (i / NL) & 1, abort_flag, a.err, ERR8_LFULL) ||
            !wait8(cempty + 8 * cs, ((i / NC) & 1) ^ 1, abort_flag, a.err, ERR8_CEMPTY)) {
          ok = false;
          break;
        }
        const uint8_t* src = land + ls * LSLOT;
        uint8_t* dst = conv + cs * CSLOT;
        for (int t = ct; t < cnt * 256; t += 64) {
          const int j = t >> 8, row = (t >> 2) & 63, p = t & 3;
          const uint4 w = *reinterpret_cast<const uint4*>(src + j * BLK8 + row * 64 + p * 16);
          const uint2 h0 = widen4(w.x), h1 = widen4(w.y), h2 = widen4(w.z), h3 = widen4(w.w);
          uint8_t* drow = dst + j * BLK + row * 128;
          *reinterpret_cast<uint4*>(drow + (((2 * p) ^ (row & 7)) << 4)) = make_uint4(h0.x, h0.y, h1.x, h1.y);
          *reinterpret_cast<uint4*>(drow + (((2 * p + 1) ^ (row & 7)) << 4)) = make_uint4(h2.x, h2.y, h3.x, h3.y);
        }
        fence_proxy_async_smem();
        mbar_arrive(lempty + 8 * ls);
        mbar_arrive(cfull + 8 * cs);
      }
    }
  } else if (warp == 5 || warp == 7) {
    // --------------------------------------------------------- MMA issuers --
    if (lane == 0) {
      const bool scores = warp == 5;
      const uint32_t idS = idesc_f16(64, 64, false, false);
      const uint32_t idO = idesc_f16(128, rows_pad, true, false);
      const uint64_t q_desc = smem_desc_sw128(smem_u32(q_s), 16, 1024);
      const uint64_t k_desc = smem_desc_sw128(smem_u32(base + L.ck_off()), 16, 1024);
      const uint64_t v_desc = smem_desc_sw128(smem_u32(base + L.cv_off()), BLK, 1024);
      const uint64_t p_desc = smem_desc_sw128(smem_u32(p_s), 16, 1024);
      const uint32_t ckf = smem_u32(ck_full), cke = smem_u32(ck_empty);
      const uint32_t cvf = smem_u32(cv_full), cve = smem_u32(cv_empty);
      bool ok = !scores || wait8(smem_u32(q_full), 0, abort_flag, a.err, ERR8_Q);
      uint32_t i = 0;
      if (scores) {
        for (int n = 0; n < ntiles && ok; ++n) {
          const int buf = n % NBUF;
          if (n >= NBUF && !wait8(smem_u32(&s_free[buf]), ((n - NBUF) / NBUF) & 1, abort_flag, a.err, ERR8_S)) { ok = false; break; }
          tc_fence_after();
          const uint32_t d = tmem + buf * 64;
          for (int kb = 0; kb < nkb && ok; kb += 2, ++i) {
            const int cnt = nkb - kb >= 2 ? 2 : 1;
            const uint32_t slot = i % NC;
            if (!wait8(ckf + 8 * slot, (i / NC) & 1, abort_flag, a.err, ERR8_CFULL)) { ok = false; break; }
            tc_fence_after();
            for (int j = 0; j < cnt; ++j) {
              const uint64_t ad = q_desc + (uint64_t)(((kb + j) * BLK) >> 4);
              const uint64_t bd = k_desc + (uint64_t)((slot * CSLOT + j * BLK) >> 4);
#pragma unroll
              for (int k16 = 0; k16 < 4; ++k16)
                mma_bf16(d, ad + 2 * k16, bd + 2 * k16, idS, ((kb + j) | k16) != 0);
            }
            mma_commit(cke + 8 * slot);
          }
          if (!ok) break;
          mma_commit(smem_u32(&s_full[buf]));
        }
      } else {
        for (int m = 0; m < ntiles && ok; ++m) {
          const int buf = m % NBUF;
          if (!wait8(smem_u32(&p_full[buf]), (m / NBUF) & 1, abort_flag, a.err, ERR8_P)) { ok = false; break; }
          tc_fence_after();
          const uint64_t bd = p_desc + (uint64_t)((buf * BLK) >> 4);
          for (int vb = 0; vb < nvb && ok; vb += 2, ++i) {
            const uint32_t slot = i % NC;
            if (!wait8(cvf + 8 * slot, (i / NC) & 1, abort_flag, a.err, ERR8_CFULL)) { ok = false; break; }
            tc_fence_after();
            // one M=128 MMA covers both chunks of the slot (BLK apart); for a
            // one-chunk copy rows 64..127 are value indices >= r_v, never read
            const uint32_t dO = tmem + O_COL + (vb >> 1) * rows_pad;
            const uint64_t ad = v_desc + (uint64_t)((slot * CSLOT) >> 4);
#pragma unroll
            for (int k16 = 0; k16 < 4; ++k16)
              mma_bf16(dO, ad + 128 * k16, bd + 2 * k16, idO, (m > 0 || k16 > 0) ? 1u : 0u);
            mma_commit(cve + 8 * slot);
          }
          if (!ok) break;
          mma_commit(smem_u32(&o_done[buf]));
        }
      }
      if (!ok) {
        const uint32_t f = smem_u32(fin) + (scores ? 0 : 8);
        mma_commit(f);
        wait8(f, 0, abort_flag, nullptr, 0, false);
      }
    }
  } else {
    // -------------------------------------------------------- softmax warps --
    const int r = 16 * warp + (lane & 15);
    const bool owner = lane < 16;
    const bool active = owner && r < rows;
    // last latent token (exclusive) of this row's query position
    const int rlim = a.nq > 1 ? a.n_lat - (a.nq - 1 - r / a.rows_per_q) : a.n_lat;
    const uint32_t lane_off = (uint32_t)(32 * warp) << 16;
    float m_run = -INFINITY, l_run = 0.f;
    bool ok = true;
    for (int n = 0; n < ntiles; ++n) {
      const int buf = n % NBUF, ss = n % NSB;
      if (tid == 0)
        lead[0] = wait8(smem_u32(&s_full[buf]), (n / NBUF) & 1, abort_flag, a.err, ERR8_S) &&
                  wait8(smem_u32(&sc_full[ss]), (n / NSB) & 1, abort_flag, a.err, ERR8_SC);
      named_sync(1, 128);
      if (!lead[0]) { ok = false; break; }
      tc_fence_after();
      float sc[64];
#pragma unroll
      for (int q = 0; q < 4; ++q) tmem_ld16(tmem + buf * 64 + q * 16 + lane_off, sc + q * 16);
      tmem_wait_ld();
      tc_fence_before();
      mbar_arrive(smem_u32(&s_free[buf]));
      const float* scl = reinterpret_cast<const float*>(sc_s + ss * SBYTES);   // [64][4]: s^K, s^V, pad
      const int nvalid = min(TOK, min(tok1, rlim) - (tok0 + n * TOK));
#pragma unroll
      for (int c = 0; c < 64; ++c) sc[c] = c < nvalid ? sc[c] * scl[4 * c] : -INFINITY;
      float mx[16];
#pragma unroll
      for (int c = 0; c < 16; ++c) mx[c] = fmaxf(fmaxf(sc[c], sc[c + 16]), fmaxf(sc[c + 32], sc[c + 48]));
#pragma unroll
      for (int w = 8; w > 0; w >>= 1)
#pragma unroll
        for (int c = 0; c < w; ++c) mx[c] = fmaxf(mx[c], mx[c + w]);
      const float tmax = mx[0];
      bool need = false;
      float alpha = 1.f;
      if (active) {
        if (n == 0) {
          m_run = tmax;
        } else if (tmax > m_run + 8.f) {
          alpha = ex2(m_run - tmax);
          m_run = tmax;
          need = true;
        }
      }
      uint32_t pk[32];
      float ps[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
      // inactive rows, and rows with no token yet, give p = 0
      const float mneg = (active && m_run != -INFINITY) ? -m_run : -INFINITY;
#pragma unroll
      for (int c = 0; c < 64; c += 2) {
        const float p0 = ex2(sc[c] + mneg);
        const float p1 = ex2(sc[c + 1] + mneg);
        ps[(c >> 1) & 7] += p0 + p1;
        pk[c >> 1] = pack_f16(p0 * scl[4 * c + 1], p1 * scl[4 * c + 5]);
      }
      const float psum = ((ps[0] + ps[1]) + (ps[2] + ps[3])) + ((ps[4] + ps[5]) + (ps[6] + ps[7]));
      l_run = l_run * alpha + psum;
      mbar_arrive(smem_u32(&sc_free[ss]));   // this thread is done with the tile's scales
      if (named_any(1, 128, need)) {
        // rescale the TMEM accumulators once O(n-1) has landed
        if (owner) alpha_s[r] = alpha;
        if (tid == 0) lead[1] = wait8(smem_u32(&o_done[(n - 1) % NBUF]), ((n - 1) / NBUF) & 1, abort_flag, a.err, ERR8_O);
        named_sync(1, 128);
        if (!lead[1]) { ok = false; break; }
        tc_fence_after();
        for (int g = 0; g < ngrp; ++g) {
          for (int cc = 0; cc < rows_pad; cc += 16) {
            const uint32_t ta = tmem + O_COL + g * rows_pad + cc + lane_off;
            float v[16];
            tmem_ld16(ta, v);
            tmem_wait_ld();
#pragma unroll
            for (int j = 0; j < 16; ++j) v[j] *= alpha_s[cc + j];
            tmem_st16(ta, v);
          }
        }
        tmem_wait_st();
        tc_fence_before();
      }
      if (n >= NBUF) {
        // P buffer `buf` is free once O(n-NBUF) has completed
        if (tid == 0) lead[2] = wait8(smem_u32(&o_done[buf]), ((n - NBUF) / NBUF) & 1, abort_flag, a.err, ERR8_O);
        named_sync(1, 128);
        if (!lead[2]) { ok = false; break; }
      }
      if (owner && r < rows_pad) {
        uint8_t* prow = p_s + buf * BLK + r * 128;
#pragma unroll
        for (int ch = 0; ch < 8; ++ch)
          *reinterpret_cast<uint4*>(prow + ((ch ^ (r & 7)) << 4)) =
              make_uint4(pk[4 * ch], pk[4 * ch + 1], pk[4 * ch + 2], pk[4 * ch + 3]);
      }
      fence_proxy_async_smem();
      mbar_arrive(smem_u32(&p_full[buf]));
    }
    if (ok) {
      if (tid == 0) lead[3] = wait8(smem_u32(&o_done[(ntiles - 1) % NBUF]), ((ntiles - 1) / NBUF) & 1, abort_flag, a.err, ERR8_O);
      named_sync(1, 128);
      ok = lead[3] != 0;
    }
    if (ok) {
      tc_fence_after();
      if (active) {
        float* ml = a.part_ml + (((int64_t)s * a.B + b) * rows + r) * 2;
        ml[0] = m_run;
        ml[1] = l_run;
      }
      float* py = a.part_y + ((int64_t)s * a.B + b) * rows * (int64_t)a.r_v;
      for (int g = 0; g < ngrp; ++g) {
        const int vv = g * 128 + 32 * warp + lane;   // M=128 layout: TMEM lane = value index
        for (int cc = 0; cc < rows_pad; cc += 16) {
          float v[16];
          tmem_ld16(tmem + O_COL + g * rows_pad + cc + lane_off, v);
          tmem_wait_ld();
          if (vv < a.r_v) {
#pragma unroll
            for (int j = 0; j < 16; ++j)
              if (cc + j < rows) py[(int64_t)(cc + j) * a.r_v + vv] = v[j];
          }
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 5) {
    tc_fence_after();
    tmem_dealloc(tmem, TMEM_COLS);
  }
}

int fp8_smem(int r_k, int r_v) {
  Layout8 L;
  L.nkb = r_k / 64; L.nvb = r_v / 64;
  return L.bytes() + 1024;
}

}  // namespace

bool absorb_fp8_supported(int r_k, int r_v, int rows) {
  if (r_k % 64 || r_v % 64 || r_k < 64 || r_v < 64 || r_k > 768) return false;
  if (rows < 1 || rows > 64 || fp8_smem(r_k, r_v) > SMEM_LIMIT) return false;
  const int ngrp = (r_v / 64 + 1) / 2;
  return O_COL + (uint32_t)(ngrp * absorb_tc_rows_pad(rows)) <= TMEM_COLS;
}

cudaError_t launch_absorb_split_fp8(const AbsorbArgs& a, cudaStream_t st) {
  TmapEncodeFn enc = tmap_encoder();
  if (!enc) return cudaErrorNotSupported;
  // codes: 4-D byte view (64 codes, token, 64-code chunk, sequence); boxes of
  // one or two chunks x 64 tokens land as dense 4 KB chunk blocks
  const cuuint64_t row_bytes = (cuuint64_t)a.ls_n;
  cuuint64_t batch_bytes = (cuuint64_t)a.ls_b;
  if (a.B == 1 && batch_bytes < row_bytes * (cuuint64_t)a.n_lat) batch_bytes = row_bytes * (cuuint64_t)a.n_lat;
  const cuuint64_t dims[4] = {64, (cuuint64_t)a.n_lat, (cuuint64_t)((a.r_k + a.r_v) / 64), (cuuint64_t)a.B};
  const cuuint64_t strides[3] = {row_bytes, 64, batch_bytes};
  cuuint32_t es[4] = {1, 1, 1, 1};
  CUtensorMap map2, map1, mapsc;
  for (int w = 1; w <= 2; ++w) {
    const cuuint32_t box[4] = {64, TOK, (cuuint32_t)w, 1};
    if (enc(w == 2 ? &map2 : &map1, CU_TENSOR_MAP_DATA_TYPE_UINT8, 4, const_cast<void*>(a.lat), dims, strides, box,
            es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return cudaErrorInvalidValue;
  }
  // scales: 3-D byte view (16 bytes at offset r_k + r_v of each row, token, sequence)
  const uint8_t* sc_base = reinterpret_cast<const uint8_t*>(a.lat) + (a.r_k + a.r_v);
  const cuuint64_t sdims[3] = {16, (cuuint64_t)a.n_lat, (cuuint64_t)a.B};
  const cuuint64_t sstrides[2] = {row_bytes, batch_bytes};
  const cuuint32_t sbox[3] = {16, TOK, 1};
  if (enc(&mapsc, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<uint8_t*>(sc_base), sdims, sstrides, sbox, es,
          CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
          CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
    return cudaErrorInvalidValue;
  const int smem = fp8_smem(a.r_k, a.r_v);
  cudaError_t e = cudaFuncSetAttribute(absorb_split_fp8, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  dim3 grid(a.S, a.B);
  absorb_split_fp8<<<grid, NTHREADS, smem, st>>>(map2, map1, mapsc, a);
  return cudaGetLastError();
}

}  // namespace lla
