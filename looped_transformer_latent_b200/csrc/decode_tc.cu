// Absorbed latent read on the 5th-generation tensor cores (tcgen05 + TMEM).
//
// HLA summary, "Latent Reader", eqs. 3-4: every (loop, head) query row of a
// sequence reads the same latent row [R~_j c^K_j | c^V_j], so the per-token
// work is two dense contractions shared by up to 64 rows:
//   S[row, j]  = q~[row, :] . c~^K_j                (scores, base-2 units)
//   O^T[v, row] += sum_j c^V_j[v] P[row, j]          (latent-space accumulate)
// One CTA handles one (split, sequence).  Per 64-token tile:
//   * two TMA producer warps stream 64 x 64 bf16 blocks (128-byte swizzled,
//     8 KB) of the latent through shared-memory rings, one for the key
//     chunks and one for the value chunks;
//   * one MMA warp issues S = Q~ C^K^T as M=64 x N=64 tcgen05 MMAs into one of
//     three TMEM score buffers; a second issues O^T += C^V^T P^T as
//     M=128 x N=rows MMAs (two value chunks per MMA) into TMEM accumulators
//     once the softmax has written P.  A single issuing thread is bound by its
//     own issue latency (a few hundred cycles per MMA, whatever its size), so
//     the two chains need two issuers to keep the tensor pipe fed.  With three
//     score buffers the score chain -- and with it the key stream -- runs up to
//     two tiles ahead of the softmax;
//   * four softmax warps own one query row per thread (lanes 0..15 of each
//     warp, the M=64 TMEM layout), read their 64 scores with tcgen05.ld, keep
//     a running max that is only raised when it grows by more than 8 (2^8 in
//     probability, safe in fp32/bf16) so the TMEM accumulator is rarely
//     rescaled, and write P (bf16) to shared memory for the second MMA.
// Latent rows past the valid range are zero-filled by TMA and masked.  Every
// mbarrier wait is bounded; on timeout the CTA records an error code in the
// workspace (the merge then emits NaN), drains its copies and frees TMEM.
#include <cuda.h>

#include "kernels.cuh"
#include "tc_ptx.cuh"

namespace lla {
namespace {

using namespace ptx;

constexpr int TOK = 64;              // tokens per tile
constexpr int BLK = 8192;            // one chunk: 64 tokens x 64 elements (128 bytes)
constexpr int SLOT = 2 * BLK;        // ring slot: up to two chunks per TMA copy
constexpr int NTHREADS = 256;        // warps 0-3 softmax, 4 and 6 TMA, 5 and 7 MMA
constexpr int SMEM_LIMIT = 232448;   // 227 KB per block (opt-in)
constexpr int MAX_RING = 24;
constexpr int MISC_BYTES = 512;
constexpr long long WAIT_CYCLES = 1ll << 32;  // ~2 s at 2 GHz
constexpr uint32_t TMEM_COLS = 512;
constexpr int NBUF = 3;              // score buffers (TMEM) and P buffers (smem)
constexpr uint32_t O_COL = 64 * NBUF;  // score buffers use columns [0, O_COL)

enum : int { ERR_TIMEOUT_EMPTY = 1, ERR_TIMEOUT_FULL = 2, ERR_TIMEOUT_Q = 3, ERR_TIMEOUT_S = 4,
             ERR_TIMEOUT_P = 5, ERR_TIMEOUT_O = 6 };

// Bounded wait.  Gives up when the CTA's abort flag is raised (if honoured) or
// after WAIT_CYCLES, raising the flag and recording `code`.
__device__ __forceinline__ bool wait_bar(uint32_t bar, uint32_t parity, volatile int* abort_flag,
                                         int* err, int code, bool honour_abort = true) {
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

__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
  const __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<const uint32_t*>(&v);
}

struct Layout {
  int nkb, nvb, ngrp, R;
  __host__ __device__ int q_off() const { return 0; }
  __host__ __device__ int p_off() const { return nkb * BLK; }
  __host__ __device__ int ring_off() const { return p_off() + NBUF * BLK; }
  __host__ __device__ int bar_off() const { return ring_off() + R * SLOT; }
  __host__ __device__ int nbars() const { return 2 * R + 3 + 4 * NBUF; }
  __host__ __device__ int misc_off() const { return bar_off() + 8 * nbars(); }
  __host__ __device__ int bytes() const { return misc_off() + MISC_BYTES; }
};

__global__ void __launch_bounds__(NTHREADS, 1)
absorb_split_tc(const __grid_constant__ CUtensorMap tmap2, const __grid_constant__ CUtensorMap tmap1,
                const AbsorbArgs a, const int R) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  Layout L;
  L.nkb = a.r_k / 64; L.nvb = a.r_v / 64; L.ngrp = (L.nvb + 1) / 2; L.R = R;
  uint8_t* q_s = base + L.q_off();
  uint8_t* p_s = base + L.p_off();
  uint8_t* ring = base + L.ring_off();
  uint64_t* bars = reinterpret_cast<uint64_t*>(base + L.bar_off());
  uint64_t* full = bars;
  uint64_t* empty = bars + R;
  uint64_t* q_full = bars + 2 * R;
  uint64_t* s_full = q_full + 1;      // [NBUF]
  uint64_t* s_free = s_full + NBUF;   // [NBUF]
  uint64_t* p_full = s_free + NBUF;   // [NBUF]
  uint64_t* o_done = p_full + NBUF;   // [NBUF]
  uint64_t* fin = o_done + NBUF;      // [2] one per MMA issuer (abort path)
  uint8_t* misc = base + L.misc_off();
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(misc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(misc + 4);
  volatile int* lead = reinterpret_cast<volatile int*>(misc + 16);   // [4] one per wait point
  float* alpha_s = reinterpret_cast<float*>(misc + 64);               // [64]

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int s = blockIdx.x, b = blockIdx.y;
  const int tok0 = s * a.tps;
  const int tok1 = min(a.n_lat, tok0 + a.tps);
  const int ntiles = (tok1 - tok0 + TOK - 1) / TOK;
  const int nkb = L.nkb, nvb = L.nvb, ngrp = L.ngrp;
  const int rows = a.rows, rows_pad = a.rows_pad;

  if (tid == 0) {
    for (int i = 0; i < R; ++i) {
      mbar_init(smem_u32(&full[i]), 1);
      mbar_init(smem_u32(&empty[i]), 1);
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
    prefetch_tmap(&tmap2);
    prefetch_tmap(&tmap1);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  griddep_wait();

  // The ring is two rings: slots [0, RK) carry key chunks, read only by the
  // score issuer, and slots [RK, R) value chunks, read only by the value
  // issuer.  Each ring has one producer and one consumer that both walk it in
  // order, so a consumer never waits on a phase more than one use ahead (the
  // two MMA chains run at different paces; one shared ring could not keep
  // that guarantee).
  const int RK = R / 2, RV = R - RK;
  if (warp == 4 || warp == 6) {
    // ----------------------------------------------------------- producers --
    // Warp 4: Q~ (one bulk copy), then the key chunks of tiles 0, 1, ...;
    // warp 6: the value chunks of tiles 0, 1, ...  Copies carry two 64-element
    // chunks (one for an odd last chunk); copy i of a ring goes to its slot
    // i mod (ring size).
    if (lane == 0) {
      const bool kring = warp == 4;
      const int nslots = kring ? RK : RV, slot0 = kring ? 0 : RK;
      const int nb = kring ? nkb : nvb, c0 = kring ? 0 : nkb;
      const uint32_t qb = smem_u32(q_full);
      if (kring) {
        mbar_arrive_tx(qb, nkb * BLK);
        bulk_load(smem_u32(q_s), a.qbf + (size_t)b * nkb * (BLK / 2), nkb * BLK, qb);
      }
      uint32_t i = 0;
      bool ok = true;
      const uint32_t ring_addr = smem_u32(ring), full_addr = smem_u32(full), empty_addr = smem_u32(empty);
      for (int n = 0; n < ntiles && ok; ++n) {
        const int y = tok0 + n * TOK;
        for (int c = 0; c < nb; c += 2, ++i) {
          const int cnt = nb - c >= 2 ? 2 : 1;
          const uint32_t slot = slot0 + i % nslots;
          if (!wait_bar(empty_addr + 8 * slot, ((i / nslots) & 1) ^ 1, abort_flag, a.err, ERR_TIMEOUT_EMPTY)) {
            ok = false;
            break;
          }
          mbar_arrive_tx(full_addr + 8 * slot, cnt * BLK);
          tma_load_4d(ring_addr + slot * SLOT, cnt == 2 ? (const void*)&tmap2 : (const void*)&tmap1,
                      full_addr + 8 * slot, 0, y, c0 + c, b);
        }
      }
      if (!ok) {
        // drain: every copy this producer issued must land before the CTA exits
        if (kring) wait_bar(qb, 0, abort_flag, nullptr, 0, false);
        for (uint32_t k = (i > (uint32_t)nslots ? i - nslots : 0); k < i; ++k)
          wait_bar(full_addr + 8 * (slot0 + k % nslots), (k / nslots) & 1, abort_flag, nullptr, 0, false);
      }
    }
  } else if (warp == 5 || warp == 7) {
    // --------------------------------------------------------- MMA issuers --
    // One tcgen05.mma chain per issuing thread runs at the thread's issue
    // latency, not the tensor pipe's rate, so the two independent chains get
    // one issuer each: warp 5 the scores S(n) = Q~ C^K^T from the key ring,
    // warp 7 the value accumulation O(m) += C^V^T P^T from the value ring,
    // each as soon as its inputs are ready.
    if (lane == 0) {
      const bool scores = warp == 5;
      const uint32_t idS = idesc_bf16(64, 64, false, false);
      const uint32_t idO = idesc_bf16(128, rows_pad, true, false);
      const uint32_t full_addr = smem_u32(full), empty_addr = smem_u32(empty);
      // descriptors at block offset 0; advancing a descriptor by k bytes adds
      // k >> 4 to its start-address field (addresses stay below 256 KB)
      const uint64_t q_desc = smem_desc_sw128(smem_u32(q_s), 16, 1024);
      const uint64_t k_desc = smem_desc_sw128(smem_u32(ring), 16, 1024);
      const uint64_t v_desc = smem_desc_sw128(smem_u32(ring), BLK, 1024);
      const uint64_t p_desc = smem_desc_sw128(smem_u32(p_s), 16, 1024);
      bool ok = !scores || wait_bar(smem_u32(q_full), 0, abort_flag, a.err, ERR_TIMEOUT_Q);
      uint32_t i = 0;   // copy index within this issuer's ring
      if (scores) {
        for (int n = 0; n < ntiles && ok; ++n) {
          const int buf = n % NBUF;
          if (n >= NBUF && !wait_bar(smem_u32(&s_free[buf]), ((n - NBUF) / NBUF) & 1, abort_flag, a.err, ERR_TIMEOUT_S)) { ok = false; break; }
          tc_fence_after();
          const uint32_t d = tmem + buf * 64;
          for (int kb = 0; kb < nkb && ok; kb += 2, ++i) {
            const int cnt = nkb - kb >= 2 ? 2 : 1;
            const uint32_t slot = i % RK;
            if (!wait_bar(full_addr + 8 * slot, (i / RK) & 1, abort_flag, a.err, ERR_TIMEOUT_FULL)) { ok = false; break; }
            tc_fence_after();
            for (int j = 0; j < cnt; ++j) {
              const uint64_t ad = q_desc + (uint64_t)(((kb + j) * BLK) >> 4);
              const uint64_t bd = k_desc + (uint64_t)((slot * SLOT + j * BLK) >> 4);
#pragma unroll
              for (int k16 = 0; k16 < 4; ++k16)
                mma_bf16(d, ad + 2 * k16, bd + 2 * k16, idS, ((kb + j) | k16) != 0);
            }
            mma_commit(empty_addr + 8 * slot);
          }
          if (!ok) break;
          mma_commit(smem_u32(&s_full[buf]));
        }
      } else {
        for (int m = 0; m < ntiles && ok; ++m) {
          const int buf = m % NBUF;
          if (!wait_bar(smem_u32(&p_full[buf]), (m / NBUF) & 1, abort_flag, a.err, ERR_TIMEOUT_P)) { ok = false; break; }
          tc_fence_after();
          const uint64_t bd = p_desc + (uint64_t)((buf * BLK) >> 4);
          for (int vb = 0; vb < nvb && ok; vb += 2, ++i) {
            const uint32_t slot = RK + i % RV;
            if (!wait_bar(full_addr + 8 * slot, (i / RV) & 1, abort_flag, a.err, ERR_TIMEOUT_FULL)) { ok = false; break; }
            tc_fence_after();
            {
              // one M=128 MMA covers both chunks of the copy: the two 64-wide
              // value groups sit BLK apart (the descriptor's leading offset).
              // A one-chunk copy (the last, odd chunk) leaves rows 64..127 of
              // this group holding products of stale slot data; those rows
              // are value indices >= r_v and are never read.
              const uint32_t dO = tmem + O_COL + (vb >> 1) * rows_pad;
              const uint64_t ad = v_desc + (uint64_t)((slot * SLOT) >> 4);
#pragma unroll
              for (int k16 = 0; k16 < 4; ++k16)
                mma_bf16(dO, ad + 128 * k16, bd + 2 * k16, idO, (m > 0 || k16 > 0) ? 1u : 0u);
            }
            mma_commit(empty_addr + 8 * slot);
          }
          if (!ok) break;
          mma_commit(smem_u32(&o_done[buf]));
        }
      }
      if (!ok) {
        // let every MMA this thread issued finish before TMEM is released
        const uint32_t f = smem_u32(fin) + (scores ? 0 : 8);
        mma_commit(f);
        wait_bar(f, 0, abort_flag, nullptr, 0, false);
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
      const int buf = n % NBUF;
      if (tid == 0) lead[0] = wait_bar(smem_u32(&s_full[buf]), (n / NBUF) & 1, abort_flag, a.err, ERR_TIMEOUT_S);
      named_sync(1, 128);
      if (!lead[0]) { ok = false; break; }
      tc_fence_after();
      float sc[64];
#pragma unroll
      for (int q = 0; q < 4; ++q) tmem_ld16(tmem + buf * 64 + q * 16 + lane_off, sc + q * 16);
      tmem_wait_ld();
      tc_fence_before();
      mbar_arrive(smem_u32(&s_free[buf]));
      const int nvalid = min(TOK, min(tok1, rlim) - (tok0 + n * TOK));
      if (nvalid < TOK) {
#pragma unroll
        for (int c = 0; c < 64; ++c)
          if (c >= nvalid) sc[c] = -INFINITY;
      }
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
        pk[c >> 1] = pack_bf16(p0, p1);
      }
      const float psum = ((ps[0] + ps[1]) + (ps[2] + ps[3])) + ((ps[4] + ps[5]) + (ps[6] + ps[7]));
      l_run = l_run * alpha + psum;
      if (named_any(1, 128, need)) {
        // rescale the TMEM accumulators once O(n-1) has landed
        if (owner) alpha_s[r] = alpha;
        if (tid == 0) lead[1] = wait_bar(smem_u32(&o_done[(n - 1) % NBUF]), ((n - 1) / NBUF) & 1, abort_flag, a.err, ERR_TIMEOUT_O);
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
        if (tid == 0) lead[2] = wait_bar(smem_u32(&o_done[buf]), ((n - NBUF) / NBUF) & 1, abort_flag, a.err, ERR_TIMEOUT_O);
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
      if (tid == 0) lead[3] = wait_bar(smem_u32(&o_done[(ntiles - 1) % NBUF]), ((ntiles - 1) / NBUF) & 1, abort_flag, a.err, ERR_TIMEOUT_O);
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
  griddep_launch();
}

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = []() -> EncodeTiledFn {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      return nullptr;
    return reinterpret_cast<EncodeTiledFn>(p);
  }();
  return fn;
}

int ring_slots(int r_k) {
  // 1 KB alignment slack + Q~ + P buffers + fixed barriers + misc; each ring
  // slot costs two chunks plus its two mbarriers
  const int fixed = 1024 + (r_k / 64) * BLK + NBUF * BLK + 8 * (3 + 4 * NBUF) + MISC_BYTES;
  const int R = (SMEM_LIMIT - fixed) / (SLOT + 16);
  return R > MAX_RING ? MAX_RING : R;
}

}  // namespace

int absorb_tc_rows_pad(int rows) { return (rows + 15) / 16 * 16; }

bool absorb_tc_supported(int lat_dtype, int r_k, int r_v, int rows) {
  if (lat_dtype != LLA_BF16 || r_k % 64 || r_v % 64 || r_k < 64 || r_v < 64 || r_k > 768) return false;
  if (rows < 1 || rows > 64 || ring_slots(r_k) < 4) return false;   // two slots per ring at least
  // TMEM: NBUF (three) 64-column score buffers, O_COL columns in all, plus
  // ceil(r_v/128) column groups of rows_pad
  const int ngrp = (r_v / 64 + 1) / 2;
  return O_COL + (uint32_t)(ngrp * absorb_tc_rows_pad(rows)) <= TMEM_COLS;
}

int absorb_tc_splits(int B, int n_lat, int num_sms) {
  // pick the split count with the smallest modelled time: waves of one CTA per
  // SM, each CTA streaming ceil(tiles / S) tiles plus a fixed start-up cost
  const int tiles = (n_lat + TOK - 1) / TOK;
  int best = 1;
  double best_t = 1e300;
  for (int S = 1; S <= 16 && S <= tiles; ++S) {
    const long ctas = (long)B * S;
    const long waves = (ctas + num_sms - 1) / num_sms;
    const double t = (double)waves * ((tiles + S - 1) / S + 2.0) + 0.02 * S * tiles;
    if (t < best_t - 1e-9) { best_t = t; best = S; }
  }
  return best;
}

cudaError_t launch_absorb_split_tc(const AbsorbArgs& a, cudaStream_t st) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) return cudaErrorNotSupported;
  // 4D view of the latent: (64 elements, token, 64-element chunk, sequence);
  // a box of one or two chunks x 64 tokens lands as 8 KB chunk blocks.
  const cuuint64_t nch = (cuuint64_t)((a.r_k + a.r_v) / 64);
  cuuint64_t dims[4] = {64, (cuuint64_t)a.n_lat, nch, (cuuint64_t)a.B};
  const cuuint64_t row_bytes = (cuuint64_t)a.ls_n * 2;
  cuuint64_t batch_bytes = (cuuint64_t)a.ls_b * 2;
  if (a.B == 1 && batch_bytes < row_bytes * (cuuint64_t)a.n_lat) batch_bytes = row_bytes * (cuuint64_t)a.n_lat;
  cuuint64_t strides[3] = {row_bytes, 128, batch_bytes};
  cuuint32_t estr[4] = {1, 1, 1, 1};
  CUtensorMap tmap2, tmap1;
  for (int w = 1; w <= 2; ++w) {
    // one- and two-chunk copies
    cuuint32_t box[4] = {64, TOK, (cuuint32_t)w, 1};
    CUresult cr = enc(w == 2 ? &tmap2 : &tmap1, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4,
                      const_cast<void*>(a.lat), dims,
                      strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                      CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (cr != CUDA_SUCCESS) return cudaErrorInvalidValue;
  }
  const int Rslots = ring_slots(a.r_k);
  Layout L;
  L.nkb = a.r_k / 64; L.nvb = a.r_v / 64; L.ngrp = (L.nvb + 1) / 2; L.R = Rslots;
  const int smem = L.bytes() + 1024;
  cudaError_t e = cudaFuncSetAttribute(absorb_split_tc, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  dim3 grid(a.S, a.B);
  return launch_kernel(absorb_split_tc, grid, dim3(NTHREADS), smem, st, 1, tmap2, tmap1, a, Rslots);
}

}  // namespace lla
