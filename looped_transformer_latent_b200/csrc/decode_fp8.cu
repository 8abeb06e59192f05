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
// on the softmax side.
//
// Keys: the tensor cores take the codes as they land (tcgen05.mma of
// kind::f8f6f4, e4m3 x e4m3, fp32 accumulate).  The query side is made 8-bit
// once per CTA: each row of Q~ is scaled by a power of two 2^e_row that brings
// its largest magnitude into (224, 448] and written as two e4m3 terms,
// hi = e4m3(x 2^e) and lo = e4m3(x 2^e - hi), whose sum carries about 8
// significant bits, on lines 2 row and 2 row + 1 of the operand;
// S = 2^-e_row s^K (hi + lo) . codes^K.
//
// Values: the codes become the f16 operands code * 2^-8, half of them by bit
// placement on the integer pipe (an e4m3 byte s.eeee.mmm moved to the f16
// bits s.0eeee.mmm0000000 is exactly code * 2^-8: the exponent biases are 15
// and 7, and subnormal codes m * 2^-9 become the f16 subnormals m * 2^-17),
// half by the conversion unit and a multiply by 2^-8; the value partials are
// multiplied by 2^8 when written.
//
// Four rings carry the chunks (64 tokens x 64 codes): the key chunks of the
// even and of the odd 64-token tiles (rings 0 and 1, one chunk per slot,
// landed in the 64-byte swizzle the MMA reads) and each tile's 128-wide
// value groups of the first and second half of r_V (rings 2 and 3, one group
// per slot: the codes land token-major in the slot's upper half and two
// converter warps per ring, one per half of the tokens, rewrite them in place
// into two f16 chunk blocks in the 128-byte swizzle).  A producer thread
// polls its two rings and issues whichever copy has a free slot.  Each ring
// has its own MMA issuer warp, so the four tcgen05 chains run concurrently
// (one thread's chain is bound by its own issue latency):
//   * two score chains (M = 128: the hi and lo terms of the 64 query rows on
//     interleaved lines, N = 64 tokens, K = 32), one for the even and one for
//     the odd tiles, each into its own TMEM buffer, so a chain works on its
//     next tile while the softmax reads the other's; the hi and lo partial
//     scores of a row sit in adjacent TMEM lanes, and the two softmax lanes
//     that hold them add them with one shuffle per column pair, each keeping
//     half of the row's columns;
//   * two value chains O^T += codes^V^T P'^T over their value groups
//     (M = 128 value indices, N = rows, f16 in);
//   * four softmax warps scale the scores, run the online softmax (base 2,
//     lazy rescale) and write P' = p * s^V in f16.
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
constexpr int QBLK = 8192;            // query chunk block: 128 lines (hi, lo of 64 rows) x 64 codes, 64-byte swizzle
constexpr int SLOTK = 4096;           // key ring slot: one landed code chunk (64 x 64), the MMA's operand as it is
constexpr int SLOTV = 2 * BLK;        // value ring slot: two f16 chunk blocks (one 128-wide value group)
constexpr int NRING = 4;              // key halves a/b, value halves a/b
constexpr int NSB = 4;                // scale slots (one per tile)
constexpr int SBYTES = TOK * 16;      // one tile's scales: 64 x (s^K, s^V, 8 pad bytes)
constexpr int NBP = 2;                // P buffers (smem)
constexpr int NTHREADS = 448;         // 0-3 softmax, 4/5 producers, 6/7 score MMA, 8/9 value MMA, 10-13 value converters
constexpr int SMEM_LIMIT = 232448;
constexpr int MISC_BYTES = 1024;
constexpr long long WAIT_CYCLES = 1ll << 32;
constexpr uint32_t TMEM_COLS = 512;
constexpr uint32_t O_COL = 128;       // S_a at column 0, S_b at 64, the value groups from 128
constexpr float CODE_UNIT = 256.f;    // f16 value operand = code * 2^-8

enum : int { ERR8_EMPTY = 51, ERR8_LFULL = 52, ERR8_CFULL = 54, ERR8_Q = 55, ERR8_S = 56, ERR8_P = 57,
             ERR8_O = 58, ERR8_SC = 59 };

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

// byte permute; a selector nibble with bit 3 set fills its byte with the
// sign bit of the selected byte
__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t b, uint32_t sel) {
  uint32_t d;
  asm("prmt.b32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(sel));
  return d;
}

// four e4m3 codes (one word, lowest byte first) -> four f16 equal to code * 2^-8.
// For the pair (b0, b1) the bytes [b0 & 7F, sign(b0) fill, b1 & 7F, sign(b1)
// fill] shifted left by 7 put each magnitude under the f16 exponent and
// mantissa fields and each sign on bit 15 / 31; the sign fill that spills
// into bits 16-22 (f16 mantissa bits no code sets) is cleared.
__device__ __forceinline__ uint2 code4_to_f16(uint32_t w) {
  const uint32_t m = w & 0x7F7F7F7Fu;
  const uint32_t lo = (prmt(m, w, 0xD1C0u) << 7) & 0xFF80FFFFu;
  const uint32_t hi = (prmt(m, w, 0xF3E2u) << 7) & 0xFF80FFFFu;
  return make_uint2(lo, hi);
}

// Key rings (0, 1) have nsk one-chunk slots, value rings (2, 3) nsv
// two-chunk slots; a key copy is one chunk, a value copy one value group.
// The same four values through the conversion unit: the exact f16 of each
// code (cvt.f16x2.e4m3x2), times 2^-8 (exact: a power of two, subnormal f16
// results included).  The converters alternate words between this and the
// integer form, so the two pipes share the work.
__device__ __forceinline__ uint2 code4_to_f16_cvt(uint32_t w) {
  const __half2_raw lo = __nv_cvt_fp8x2_to_halfraw2((__nv_fp8x2_storage_t)(w & 0xFFFFu), __NV_E4M3);
  const __half2_raw hi = __nv_cvt_fp8x2_to_halfraw2((__nv_fp8x2_storage_t)(w >> 16), __NV_E4M3);
  const __half2 unit = __halves2half2(__ushort_as_half((unsigned short)0x1C00u), __ushort_as_half((unsigned short)0x1C00u));
  const __half2 l = __hmul2(*reinterpret_cast<const __half2*>(&lo), unit);
  const __half2 h = __hmul2(*reinterpret_cast<const __half2*>(&hi), unit);
  return make_uint2(*reinterpret_cast<const uint32_t*>(&l), *reinterpret_cast<const uint32_t*>(&h));
}

struct Layout8 {
  int nkb, nvb, nsk, nsv;
  __host__ __device__ int q8_off() const { return 0; }
  __host__ __device__ int p_off() const { return nkb * QBLK; }
  __host__ __device__ int sc_off() const { return p_off() + NBP * BLK; }
  __host__ __device__ int ring_off(int r) const {
    const int k0 = sc_off() + NSB * SBYTES;
    return r < 2 ? k0 + r * nsk * SLOTK : k0 + 2 * nsk * SLOTK + (r - 2) * nsv * SLOTV;
  }
  __host__ __device__ int nslots(int r) const { return r < 2 ? nsk : nsv; }
  __host__ __device__ int slot_bytes(int r) const { return r < 2 ? SLOTK : SLOTV; }
  __host__ __device__ int land_off(int r) const { return r < 2 ? 0 : BLK; }      // where the codes land in a slot
  // Q~ in f16 (the query map's output) is staged in the ring memory, which is
  // free until the rings start
  __host__ __device__ int stage_off() const { return ring_off(0); }
  __host__ __device__ int ring_bytes() const { return ring_off(NRING) - ring_off(0); }
  __host__ __device__ int step(int r) const { return r < 2 ? 1 : 2; }            // chunks per copy
  __host__ __device__ int bar0(int r) const { return r < 2 ? r * nsk : 2 * nsk + (r - 2) * nsv; }
  __host__ __device__ int ring_bars() const { return 2 * nsk + 2 * nsv; }
  __host__ __device__ int bar_off() const { return ring_off(NRING); }
  __host__ __device__ int nbars() const { return 3 * ring_bars() + 2 * NSB + 1 + 4 + 2 * NBP + 4; }
  __host__ __device__ int misc_off() const { return bar_off() + 8 * nbars(); }
  __host__ __device__ int bytes() const { return misc_off() + MISC_BYTES; }
};

// Q~[t][k], Q~[t][k + 1] (k even) from the f16 staging copy: r_K/64 blocks of
// 64 rows x 64 values, 128-byte rows in the 128-byte swizzle.
__device__ __forceinline__ float2 q_pair(const uint8_t* stage, int t, int k) {
  const uint8_t* blk = stage + (k >> 6) * BLK + t * 128;
  const int kk = k & 63;
  const __half2 v = *reinterpret_cast<const __half2*>(blk + (((kk >> 3) ^ (t & 7)) << 4) + (kk & 7) * 2);
  return __half22float2(v);
}

// What ring r carries: the key rings every key chunk of the even (ring 0)
// and the odd (ring 1) tiles; the value rings every tile's chunks of the
// value groups [0, ga) and [ga, ngrp) (a group is two chunks, the last
// possibly one).
struct Rings {
  int nkb, nvb, ngrp, ga;
  __device__ int lo(int r) const { return r < 2 ? 0 : r == 2 ? 0 : 2 * ga; }
  __device__ int hi(int r) const { return r < 2 ? nkb : r == 2 ? min(nvb, 2 * ga) : nvb; }
  __device__ int tile0(int r) const { return r < 2 ? r : 0; }
  __device__ int tstep(int r) const { return r < 2 ? 2 : 1; }
};

// 14 warps: four share an SM sub-partition's 16 K registers, so at most 128 per thread
__global__ void __launch_bounds__(NTHREADS, 1)
absorb_split_fp8(const __grid_constant__ CUtensorMap mapk, const __grid_constant__ CUtensorMap map64,
                 const __grid_constant__ CUtensorMap map128, const __grid_constant__ CUtensorMap mapsc,
                 const AbsorbArgs a, const int nsk, const int nsv) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  Layout8 L;
  L.nkb = a.r_k / 64; L.nvb = a.r_v / 64; L.nsk = nsk; L.nsv = nsv;
  Rings R;
  R.nkb = L.nkb; R.nvb = L.nvb;
  R.ngrp = (L.nvb + 1) / 2;
  R.ga = (R.ngrp + 1) / 2;
  const bool two_v = R.ga < R.ngrp;     // a second value chain (r_V > 128)
  uint8_t* q8_s = base + L.q8_off();
  uint8_t* p_s = base + L.p_off();
  uint8_t* sc_s = base + L.sc_off();
  uint64_t* bars = reinterpret_cast<uint64_t*>(base + L.bar_off());
  uint64_t* lfull = bars;                       // [ring][slot] codes landed (TMA)
  uint64_t* cfull = lfull + L.ring_bars();      // [ring][slot] f16 blocks written (converter)
  uint64_t* rempty = cfull + L.ring_bars();     // [ring][slot] MMAs reading the slot done
  uint64_t* sc_full = rempty + L.ring_bars();   // [NSB] a tile's scales landed
  uint64_t* sc_free = sc_full + NSB;            // [NSB] softmax done with them (128 arrivals)
  uint64_t* q_full = sc_free + NSB;
  uint64_t* s_full = q_full + 1;                // [2] scores of the even / odd tiles in TMEM
  uint64_t* s_free = s_full + 2;                // [2] softmax has read them (128 arrivals)
  uint64_t* p_full = s_free + 2;                // [NBP]
  uint64_t* o_done = p_full + NBP;              // [NBP] the value chains are done with a tile
  uint64_t* fin = o_done + NBP;                 // [4] one per MMA issuer (abort path)
  uint8_t* misc = base + L.misc_off();
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(misc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(misc + 4);
  volatile int* lead = reinterpret_cast<volatile int*>(misc + 16);   // [4]
  float* alpha_s = reinterpret_cast<float*>(misc + 64);               // [64]
  float* qinv_s = reinterpret_cast<float*>(misc + 320);               // [64] 2^-e of each Q~ row

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int s = blockIdx.x, b = blockIdx.y;
  const int tok0 = s * a.tps;
  const int tok1 = min(a.n_lat, tok0 + a.tps);
  const int ntiles = (tok1 - tok0 + TOK - 1) / TOK;
  const int nkb = L.nkb, ngrp = R.ngrp;
  const int rows = a.rows, rows_pad = a.rows_pad;

  if (tid == 0) {
    for (int i = 0; i < L.ring_bars(); ++i) {
      mbar_init(smem_u32(&lfull[i]), 1);
      mbar_init(smem_u32(&cfull[i]), 2);   // value groups: the two converter warps (unused on key rings)
      mbar_init(smem_u32(&rempty[i]), 1);
    }
    for (int i = 0; i < NSB; ++i) {
      mbar_init(smem_u32(&sc_full[i]), 1);
      mbar_init(smem_u32(&sc_free[i]), 128);
    }
    mbar_init(smem_u32(q_full), 1);
    for (int i = 0; i < 2; ++i) {
      mbar_init(smem_u32(&s_full[i]), 1);
      mbar_init(smem_u32(&s_free[i]), 128);
    }
    for (int i = 0; i < NBP; ++i) {
      mbar_init(smem_u32(&p_full[i]), 128);
      mbar_init(smem_u32(&o_done[i]), two_v ? 2 : 1);
    }
    for (int i = 0; i < 4; ++i) mbar_init(smem_u32(&fin[i]), 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 6) {
    tmem_alloc(smem_u32(tmem_slot), TMEM_COLS);
    tmem_relinquish();
  }
  if (warp == 4 && lane == 0) {
    prefetch_tmap(&mapk);
    prefetch_tmap(&map64);
    prefetch_tmap(&map128);
    prefetch_tmap(&mapsc);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  griddep_wait();

  // ---- Q~ to e4m3 hi/lo (once per CTA) --------------------------------------
  // Q~ (f16, [r_k/64][64 rows x 64], 128-byte swizzle) lands in the ring
  // memory; warp w takes rows w, w + 14, ...: the row's largest magnitude
  // gives the power of two, then each pair of values becomes hi and lo codes,
  // stored K-major in the 64-byte swizzle (16-byte piece q of line L at
  // (L / 8) * 512 + (L % 8) * 64 + 16 (q ^ ((L / 2) % 4)); hi on line 2t, lo
  // on line 2t + 1 of row t).
  bool q_ok = true;
  {
    uint8_t* stage = base + L.stage_off();
    const uint32_t qb = smem_u32(q_full);
    if (warp == 4 && lane == 0) {
      mbar_arrive_tx(qb, nkb * BLK);
      bulk_load(smem_u32(stage), a.qbf + (size_t)b * nkb * (BLK / 2), nkb * BLK, qb);
    }
    q_ok = wait8(qb, 0, abort_flag, a.err, ERR8_Q);
    if (q_ok) {
      for (int t = warp; t < 64; t += NTHREADS / 32) {
        float amax = 0.f;
        for (int k = 2 * lane; k < a.r_k; k += 64) {
          const float2 v = q_pair(stage, t, k);
          amax = fmaxf(amax, fmaxf(fabsf(v.x), fabsf(v.y)));
        }
        amax = redux_max(amax);
        // 2^e with amax * 2^e in (224, 448] (amax = m 2^x, m in [0.5, 1):
        // e = 9 - x if m <= 0.875, else 8 - x); zero rows keep e = 0
        float sc = 1.f;
        if (amax > 0.f) {
          int x;
          const float m = frexpf(amax, &x);
          sc = ldexpf(1.f, max(-126, min(127, (m <= 0.875f ? 9 : 8) - x)));
        }
        if (lane == 0) qinv_s[t] = 1.f / sc;
        for (int k = 2 * lane; k < a.r_k; k += 64) {
          const float2 v = q_pair(stage, t, k);
          const float2 x = make_float2(v.x * sc, v.y * sc);
          const __nv_fp8x2_storage_t hi = __nv_cvt_float2_to_fp8x2(x, __NV_SATFINITE, __NV_E4M3);
          const __half2_raw hr = __nv_cvt_fp8x2_to_halfraw2(hi, __NV_E4M3);
          const float2 hv = __half22float2(*reinterpret_cast<const __half2*>(&hr));
          const __nv_fp8x2_storage_t lo =
              __nv_cvt_float2_to_fp8x2(make_float2(x.x - hv.x, x.y - hv.y), __NV_SATFINITE, __NV_E4M3);
          const int kk = k & 63;
          // hi on line 2t, lo on line 2t + 1 of the chunk's 128 lines
          const int lh = 2 * t, ll = 2 * t + 1;
          const uint32_t blk = (uint32_t)((k >> 6) * QBLK + (kk & 15));
          const uint32_t oh = blk + (lh >> 3) * 512 + (lh & 7) * 64 + ((((kk >> 4) ^ ((lh >> 1) & 3))) << 4);
          const uint32_t ol = blk + (ll >> 3) * 512 + (ll & 7) * 64 + ((((kk >> 4) ^ ((ll >> 1) & 3))) << 4);
          *reinterpret_cast<__nv_fp8x2_storage_t*>(q8_s + oh) = hi;
          *reinterpret_cast<__nv_fp8x2_storage_t*>(q8_s + ol) = lo;
        }
      }
    }
    fence_proxy_async_smem();   // the codes are read by the MMAs; the staging area is reused by TMA
    if (__syncthreads_or(!q_ok)) q_ok = false;
  }

  if (!q_ok) {
    // Q~ never landed: nothing was issued but that copy; let it land (bounded)
    if (warp == 4 && lane == 0) wait8(smem_u32(q_full), 0, abort_flag, nullptr, 0, false);
  } else if (warp == 4 || warp == 5) {
    // ----------------------------------------------------------- producers --
    // Warp 4: Q~ (one bulk copy), the tiles' scales and the key copies of
    // rings 0 and 1; warp 5: the value copies of rings 2 and 3.  A copy is two
    // chunks (one for an odd last chunk); copy i of a ring goes to slot i mod
    // ns.  The thread polls its rings without blocking, so a ring whose slots
    // are all in use never holds back the other's copies.
    if (lane == 0) {
      const bool kside = warp == 4;
      const int r0 = kside ? 0 : 2, c0 = kside ? 0 : nkb;
      uint32_t cnt[2] = {0, 0};
      int tile[2] = {R.tile0(r0), R.tile0(r0 + 1)}, chunk[2] = {R.lo(r0), R.lo(r0 + 1)};
      bool done[2] = {R.lo(r0) >= R.hi(r0) || tile[0] >= ntiles, R.lo(r0 + 1) >= R.hi(r0 + 1) || tile[1] >= ntiles};
      int nsc = kside ? 0 : ntiles;
      bool ok = true;
      long long t_last = clock64();
      while (true) {
        bool progress = false;
        if (nsc < ntiles) {
          const int ss = nsc % NSB;
          if (mbar_test_wait(smem_u32(&sc_free[ss]), ((nsc / NSB) & 1) ^ 1)) {
            mbar_arrive_tx(smem_u32(&sc_full[ss]), SBYTES);
            tma_load_3d(smem_u32(sc_s + ss * SBYTES), &mapsc, smem_u32(&sc_full[ss]), 0, tok0 + nsc * TOK, b);
            ++nsc;
            progress = true;
          }
        }
        for (int k = 0; k < 2; ++k) {
          if (done[k]) continue;
          const int r = r0 + k, ns = L.nslots(r);
          const uint32_t slot = cnt[k] % ns, ph = cnt[k] / ns;
          if (!mbar_test_wait(smem_u32(&rempty[L.bar0(r) + slot]), (ph & 1) ^ 1)) continue;
          const int c = chunk[k], w = min(L.step(r), R.hi(r) - c);
          const uint32_t fb = smem_u32(&lfull[L.bar0(r) + slot]);
          mbar_arrive_tx(fb, w * BLK8);
          // keys: one chunk in the 64-byte swizzle (the MMA's operand as it
          // lands); values: a group token-major (64 rows of 64 w codes)
          tma_load_3d(smem_u32(base + L.ring_off(r) + slot * L.slot_bytes(r) + L.land_off(r)),
                      r < 2 ? (const void*)&mapk : w == 2 ? (const void*)&map128 : (const void*)&map64, fb,
                      (c0 + c) * 64, tok0 + tile[k] * TOK, b);
          ++cnt[k];
          chunk[k] = c + w;
          if (chunk[k] >= R.hi(r)) {
            chunk[k] = R.lo(r);
            tile[k] += R.tstep(r);
            if (tile[k] >= ntiles) done[k] = true;
          }
          progress = true;
        }
        if (done[0] && done[1] && nsc == ntiles) break;
        if (progress) {
          t_last = clock64();
        } else if (*abort_flag) {
          ok = false;
          break;
        } else if (clock64() - t_last > WAIT_CYCLES) {
          *abort_flag = 1;
          atomicExch(a.err, ERR8_EMPTY);
          ok = false;
          break;
        }
      }
      if (!ok) {
        // drain: every copy this producer issued must land before the CTA exits
        if (kside) {
          for (int n = max(0, nsc - NSB); n < nsc; ++n)
            wait8(smem_u32(&sc_full[n % NSB]), (n / NSB) & 1, abort_flag, nullptr, 0, false);
        }
        for (int k = 0; k < 2; ++k) {
          const uint32_t ns = L.nslots(r0 + k);
          for (uint32_t i = (cnt[k] > ns ? cnt[k] - ns : 0); i < cnt[k]; ++i)
            wait8(smem_u32(&lfull[L.bar0(r0 + k) + i % ns]), (i / ns) & 1, abort_flag, nullptr, 0, false);
        }
      }
    }
  } else if (warp >= 10) {
    // ----------------------------------------------------- value converters --
    // Warp 10 + 2 (r - 2) + h rewrites tokens 32h .. 32h + 31 of value ring
    // r's groups into f16 chunk blocks, copy by copy in the producer's order.
    // The codes landed token-major (a token's 64 w codes in one row) in the
    // slot's upper half, so the warp's f16 rows of both chunks cover its own
    // codes and no other warp's: it loads its 2 or 4 KB, synchronises, and
    // stores into the swizzled rows.
    const int r = 2 + (warp - 10) / 2, h = (warp - 10) & 1;
    const int ns = L.nslots(r);
    uint8_t* ring = base + L.ring_off(r);
    uint32_t cnt = 0;
    bool ok = true;
    for (int n = 0; n < ntiles && ok; ++n) {
      for (int c = R.lo(r); c < R.hi(r); c += 2, ++cnt) {
        const int w = min(2, R.hi(r) - c);
        const uint32_t slot = cnt % ns, ph = cnt / ns;
        if (!wait8(smem_u32(&lfull[L.bar0(r) + slot]), ph & 1, abort_flag, a.err, ERR8_LFULL)) { ok = false; break; }
        uint8_t* sl = ring + slot * SLOTV;
        // 16-byte piece u of this warp's rows holds codes 16 (u % (4w)) .. of token 32h + u / (4w)
        const uint4* src = reinterpret_cast<const uint4*>(sl + BLK + 32 * h * 64 * w);
        const int npieces = 4 * w;   // per lane
        uint4 cw[8];
#pragma unroll
        for (int k = 0; k < 8; ++k)
          if (k < npieces) cw[k] = src[lane + 32 * k];
        __syncwarp();
#pragma unroll
        for (int k = 0; k < 8; ++k) {
          if (k >= npieces) break;
          const int u = lane + 32 * k, per = 4 * w;
          const int t = 32 * h + u / per, j = (u % per) >> 2, p = u & 3;
          uint8_t* drow = sl + j * BLK + t * 128;
          const int sw = t & 7;
          const uint2 h0 = code4_to_f16(cw[k].x), h1 = code4_to_f16_cvt(cw[k].y);
          const uint2 h2 = code4_to_f16(cw[k].z), h3 = code4_to_f16_cvt(cw[k].w);
          *reinterpret_cast<uint4*>(drow + (((2 * p) ^ sw) << 4)) = make_uint4(h0.x, h0.y, h1.x, h1.y);
          *reinterpret_cast<uint4*>(drow + (((2 * p + 1) ^ sw) << 4)) = make_uint4(h2.x, h2.y, h3.x, h3.y);
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive(smem_u32(&cfull[L.bar0(r) + slot]));
      }
    }
  } else if (warp >= 6) {
    // --------------------------------------------------------- MMA issuers --
    // Warps 6/7: the score chains of the even / odd tiles over rings 0/1, into
    // TMEM score buffers 0/1; warps 8/9: value chains a/b over rings 2/3.
    const int r = warp - 6;
    const bool scores = r < 2;
    const bool has_chain = scores ? r < ntiles : (r == 2 || two_v);
    if (lane == 0 && has_chain) {
      const uint32_t idS = idesc_e4m3(128, 64);
      const uint32_t idO = idesc_f16(128, rows_pad, true, false);
      const uint64_t q8_desc = smem_desc_sw64(smem_u32(q8_s));
      const uint64_t k_desc = smem_desc_sw64(smem_u32(base + L.ring_off(r)));
      const uint64_t v_desc = smem_desc_sw128(smem_u32(base + L.ring_off(r)), BLK, 1024);
      const uint64_t p_desc = smem_desc_sw128(smem_u32(p_s), 16, 1024);
      bool ok = true;
      uint32_t cnt = 0;
      if (scores) {
        const uint32_t d = tmem + r * 64;
        for (int n = r; n < ntiles && ok; n += 2) {
          // buffer r is free once the softmax has read tile n - 2's scores
          if (n >= 2 && !wait8(smem_u32(&s_free[r]), ((n - 2) >> 1) & 1, abort_flag, a.err, ERR8_S)) { ok = false; break; }
          tc_fence_after();
          uint32_t acc = 0;
          for (int c = R.lo(r); c < R.hi(r) && ok; ++c, ++cnt) {
            // the landed key chunk is the operand: wait for the copy itself
            const uint32_t slot = cnt % nsk, ph = cnt / nsk;
            if (!wait8(smem_u32(&lfull[L.bar0(r) + slot]), ph & 1, abort_flag, a.err, ERR8_LFULL)) { ok = false; break; }
            tc_fence_after();
            const uint64_t ad = q8_desc + (uint64_t)((c * QBLK) >> 4);
            const uint64_t bd = k_desc + (uint64_t)((slot * SLOTK) >> 4);
            // M = 128 lines (hi and lo of each row, interleaved), K = 32 codes
            // (32 bytes) per MMA: two steps per chunk
#pragma unroll
            for (int k32 = 0; k32 < 2; ++k32) {
              mma_f8f6f4(d, ad + 2 * k32, bd + 2 * k32, idS, acc);
              acc = 1;
            }
            mma_commit(smem_u32(&rempty[L.bar0(r) + slot]));
          }
          if (!ok) break;
          mma_commit(smem_u32(&s_full[r]));
        }
      } else {
        for (int m = 0; m < ntiles && ok; ++m) {
          const int buf = m % NBP;
          if (!wait8(smem_u32(&p_full[buf]), (m / NBP) & 1, abort_flag, a.err, ERR8_P)) { ok = false; break; }
          tc_fence_after();
          const uint64_t bd = p_desc + (uint64_t)((buf * BLK) >> 4);
          for (int c = R.lo(r); c < R.hi(r) && ok; c += 2, ++cnt) {
            const uint32_t slot = cnt % nsv, ph = cnt / nsv;
            if (!wait8(smem_u32(&cfull[L.bar0(r) + slot]), ph & 1, abort_flag, a.err, ERR8_CFULL)) { ok = false; break; }
            tc_fence_after();
            // one M=128 MMA covers both chunks of the slot (BLK apart); for a
            // one-chunk group rows 64..127 are value indices >= r_v, never read
            const uint32_t dO = tmem + O_COL + (c >> 1) * rows_pad;
            const uint64_t ad = v_desc + (uint64_t)((slot * SLOTV) >> 4);
#pragma unroll
            for (int k16 = 0; k16 < 4; ++k16)
              mma_bf16(dO, ad + 128 * k16, bd + 2 * k16, idO, (m > 0 || k16 > 0) ? 1u : 0u);
            mma_commit(smem_u32(&rempty[L.bar0(r) + slot]));
          }
          if (!ok) break;
          mma_commit(smem_u32(&o_done[buf]));
        }
      }
      if (!ok) {
        const uint32_t f = smem_u32(&fin[r]);
        mma_commit(f);
        wait8(f, 0, abort_flag, nullptr, 0, false);
      }
    }
  } else {
    // -------------------------------------------------------- softmax warps --
    // TMEM lane 32w + l holds the hi (l even) or lo (l odd) part of query row
    // 16w + l/2; the pair swaps halves so that the even lane owns columns
    // 0..31 of the row's scores and the odd lane columns 32..63.
    const int r = 16 * warp + (lane >> 1), part = lane & 1;
    const bool owner = part == 0;
    const bool active = r < rows;
    // last latent token (exclusive) of this row's query position
    const int rlim = a.nq > 1 ? a.n_lat - (a.nq - 1 - r / a.rows_per_q) : a.n_lat;
    const uint32_t lane_off = (uint32_t)(32 * warp) << 16;
    const float qinv = qinv_s[r];   // 2^-e of this row's 8-bit query terms
    float m_run = -INFINITY, l_run = 0.f;
    bool ok = true;
    for (int n = 0; n < ntiles; ++n) {
      const int buf = n % NBP, ss = n % NSB;
      const int sb = n & 1;   // score buffer (and chain) of tile n
      if (tid == 0)
        lead[0] = wait8(smem_u32(&s_full[sb]), (n >> 1) & 1, abort_flag, a.err, ERR8_S) &&
                  wait8(smem_u32(&sc_full[ss]), (n / NSB) & 1, abort_flag, a.err, ERR8_SC);
      named_sync(1, 128);
      if (!lead[0]) { ok = false; break; }
      tc_fence_after();
      float sc[32];
      {
        float raw[64];
#pragma unroll
        for (int q = 0; q < 4; ++q) tmem_ld16(tmem + sb * 64 + q * 16 + lane_off, raw + q * 16);
        tmem_wait_ld();
        tc_fence_before();
        mbar_arrive(smem_u32(&s_free[sb]));
        // keep this lane's half, add the partner's part of it
#pragma unroll
        for (int j = 0; j < 32; ++j) {
          const float keep = part ? raw[32 + j] : raw[j];
          const float give = part ? raw[j] : raw[32 + j];
          sc[j] = keep + __shfl_xor_sync(0xffffffffu, give, 1);
        }
      }
      const float* scl = reinterpret_cast<const float*>(sc_s + ss * SBYTES) + 4 * 32 * part;   // [32][4]: s^K, s^V, pad
      const int nvalid = min(TOK, min(tok1, rlim) - (tok0 + n * TOK)) - 32 * part;
#pragma unroll
      for (int c = 0; c < 32; ++c) sc[c] = c < nvalid ? sc[c] * (scl[4 * c] * qinv) : -INFINITY;
      float mx[4] = {sc[0], sc[1], sc[2], sc[3]};
#pragma unroll
      for (int c = 4; c < 32; ++c) mx[c & 3] = fmaxf(mx[c & 3], sc[c]);
      float tmax = fmaxf(fmaxf(mx[0], mx[1]), fmaxf(mx[2], mx[3]));
      tmax = fmaxf(tmax, __shfl_xor_sync(0xffffffffu, tmax, 1));
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
      if (n >= NBP) {
        // P buffer `buf` is free once O(n-NBP) has completed
        if (tid == 0) lead[2] = wait8(smem_u32(&o_done[buf]), ((n - NBP) / NBP) & 1, abort_flag, a.err, ERR8_O);
        named_sync(1, 128);
        if (!lead[2]) { ok = false; break; }
      }
      // inactive rows, and rows with no token yet, give p = 0
      const float mneg = (active && m_run != -INFINITY) ? -m_run : -INFINITY;
      float ps[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
      uint8_t* prow = p_s + buf * BLK + r * 128;
      const bool store = r < rows_pad;
#pragma unroll
      for (int ch = 0; ch < 4; ++ch) {
        uint32_t pk[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int c = 8 * ch + 2 * e;
          const float p0 = ex2(sc[c] + mneg);
          const float p1 = ex2(sc[c + 1] + mneg);
          ps[(c >> 1) & 7] += p0 + p1;
          pk[e] = pack_f16(p0 * scl[4 * c + 1], p1 * scl[4 * c + 5]);
        }
        const int unit = 4 * part + ch;   // 16-byte unit of the row: columns 8 unit ..
        if (store) *reinterpret_cast<uint4*>(prow + ((unit ^ (r & 7)) << 4)) = make_uint4(pk[0], pk[1], pk[2], pk[3]);
      }
      const float psum = ((ps[0] + ps[1]) + (ps[2] + ps[3])) + ((ps[4] + ps[5]) + (ps[6] + ps[7]));
      l_run = l_run * alpha + psum;   // this lane's half of the row
      if (named_any(1, 128, need)) {
        // rescale the TMEM accumulators once O(n-1) has landed (before P(n)
        // is published, after the scores are dead: fewer live registers)
        if (owner) alpha_s[r] = alpha;
        if (tid == 0) lead[1] = wait8(smem_u32(&o_done[(n - 1) % NBP]), ((n - 1) / NBP) & 1, abort_flag, a.err, ERR8_O);
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
      mbar_arrive(smem_u32(&sc_free[ss]));   // this thread is done with the tile's scales
      fence_proxy_async_smem();
      mbar_arrive(smem_u32(&p_full[buf]));
    }
    if (ok) {
      if (tid == 0)
        lead[3] = wait8(smem_u32(&o_done[(ntiles - 1) % NBP]), ((ntiles - 1) / NBP) & 1, abort_flag, a.err, ERR8_O);
      named_sync(1, 128);
      ok = lead[3] != 0;
    }
    if (ok) {
      tc_fence_after();
      const float l_row = l_run + __shfl_xor_sync(0xffffffffu, l_run, 1);
      if (active && owner) {
        float* ml = a.part_ml + (((int64_t)s * a.B + b) * rows + r) * 2;
        ml[0] = m_run;
        ml[1] = l_row;
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
              if (cc + j < rows) py[(int64_t)(cc + j) * a.r_v + vv] = v[j] * CODE_UNIT;
          }
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 6) {
    tc_fence_after();
    tmem_dealloc(tmem, TMEM_COLS);
  }
  griddep_launch();
}

int fp8_smem(int r_k, int r_v, int nsk, int nsv) {
  Layout8 L;
  L.nkb = r_k / 64; L.nvb = r_v / 64; L.nsk = nsk; L.nsv = nsv;
  return L.bytes() + 1024;
}

// ring memory must also hold the f16 staging copy of Q~ (r_K/64 blocks of 8 KB)
bool fp8_fits(int r_k, int r_v, int nsk, int nsv) {
  Layout8 L;
  L.nkb = r_k / 64; L.nvb = r_v / 64; L.nsk = nsk; L.nsv = nsv;
  return fp8_smem(r_k, r_v, nsk, nsv) <= SMEM_LIMIT && L.ring_bytes() >= L.nkb * BLK;
}

// ring depths, first that fits: value rings of three groups (a tile's worth
// for r_V up to 768, measured the better split) with key rings of four
// chunks, then shallower
bool fp8_slots(int r_k, int r_v, int* nsk, int* nsv) {
  static const int opts[7][2] = {{4, 3}, {8, 2}, {6, 2}, {4, 2}, {3, 2}, {2, 2}, {2, 1}};
  for (const auto& o : opts)
    if (fp8_fits(r_k, r_v, o[0], o[1])) { *nsk = o[0]; *nsv = o[1]; return true; }
  return false;
}

}  // namespace

bool absorb_fp8_supported(int r_k, int r_v, int rows) {
  if (r_k % 64 || r_v % 64 || r_k < 64 || r_v < 64 || r_k > 768) return false;
  int nsk, nsv;
  if (rows < 1 || rows > 64 || !fp8_slots(r_k, r_v, &nsk, &nsv)) return false;
  const int ngrp = (r_v / 64 + 1) / 2;
  return O_COL + (uint32_t)(ngrp * absorb_tc_rows_pad(rows)) <= TMEM_COLS;
}

cudaError_t launch_absorb_split_fp8(const AbsorbArgs& a, cudaStream_t st) {
  TmapEncodeFn enc = tmap_encoder();
  if (!enc) return cudaErrorNotSupported;
  // codes: 3-D byte view (code byte of the row, token, sequence).  Keys: boxes
  // of 64 codes x 64 tokens in the 64-byte swizzle (the MMA's K-major
  // operand); values: boxes of 128 or 64 codes x 64 tokens, token-major
  const cuuint64_t row_bytes = (cuuint64_t)a.ls_n;
  cuuint64_t batch_bytes = (cuuint64_t)a.ls_b;
  if (a.B == 1 && batch_bytes < row_bytes * (cuuint64_t)a.n_lat) batch_bytes = row_bytes * (cuuint64_t)a.n_lat;
  const cuuint64_t dims[3] = {(cuuint64_t)(a.r_k + a.r_v), (cuuint64_t)a.n_lat, (cuuint64_t)a.B};
  const cuuint64_t strides[2] = {row_bytes, batch_bytes};
  cuuint32_t es[3] = {1, 1, 1};
  CUtensorMap mapk, map64, map128, mapsc;
  for (int m = 0; m < 3; ++m) {
    const cuuint32_t box[3] = {m == 2 ? 128u : 64u, TOK, 1};
    CUtensorMap* dst = m == 0 ? &mapk : m == 1 ? &map64 : &map128;
    if (enc(dst, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<void*>(a.lat), dims, strides, box, es,
            CU_TENSOR_MAP_INTERLEAVE_NONE, m == 0 ? CU_TENSOR_MAP_SWIZZLE_64B : CU_TENSOR_MAP_SWIZZLE_NONE,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
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
  int nsk = 2, nsv = 1;
  if (!fp8_slots(a.r_k, a.r_v, &nsk, &nsv)) return cudaErrorNotSupported;
  const int smem = fp8_smem(a.r_k, a.r_v, nsk, nsv);
  cudaError_t e = cudaFuncSetAttribute(absorb_split_fp8, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  dim3 grid(a.S, a.B);
  return launch_kernel(absorb_split_fp8, grid, dim3(NTHREADS), smem, st, 1, mapk, map64, map128, mapsc, a, nsk,
                       nsv);
}

}  // namespace lla
