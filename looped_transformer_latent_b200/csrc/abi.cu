// C ABI entry points: host-side validation, workspace planning and launch
// orchestration.  Nothing is launched unless every check passes.
#include <atomic>
#include <cmath>
#include <cstdlib>
#include <cstring>

#include "kernels.cuh"

namespace lla {

// Launch attribute switch for launch_kernel (LLA_PDL=1 turns programmatic
// dependent launch on); read once per process.
bool pdl_enabled() {
  static const bool on = [] {
    const char* v = std::getenv("LLA_PDL");
    return v && v[0] == '1';
  }();
  return on;
}

namespace {

constexpr int kAbiVersion = 4;   // 2: LLA_FP8_E4M3 latent rows; 3: hla_decode_params.nq; 4: win_stream
constexpr int kDefaultSms = 148;        // B200; used only when no device can be queried
constexpr int kMaxDevices = 64;
constexpr size_t kAlign = 256;

// Streaming multiprocessors of the current device, queried once per device.
// Split and wave plans (and so workspace sizes) follow it: query a workspace
// size with the same device current as the call that uses it.  Without a
// usable device (a host-only process sizing buffers) the B200's count is
// assumed; any launch then fails with LLA_ERR_CUDA anyway.
int num_sms() {
  static std::atomic<int> cache[kMaxDevices];
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
    (void)cudaGetLastError();
    return kDefaultSms;
  }
  const int known = cache[dev].load(std::memory_order_relaxed);
  if (known > 0) return known;
  int n = 0;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) {
    (void)cudaGetLastError();
    return kDefaultSms;
  }
  cache[dev].store(n, std::memory_order_relaxed);
  return n;
}

inline bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }
inline size_t elem_size(int dt) { return dt == LLA_BF16 ? 2 : dt == LLA_FP8_E4M3 ? 1 : 4; }
inline bool dtype_ok(int dt) { return dt == LLA_F32 || dt == LLA_BF16; }          // element types
inline bool lat_dtype_ok(int dt) { return dtype_ok(dt) || dt == LLA_FP8_E4M3; }   // latent row formats
constexpr int kFp8Extra = 16;   // fp8 rows: s^K, s^V (fp32) and 8 zero bytes after the codes
inline size_t round_up(size_t x) { return (x + kAlign - 1) / kAlign * kAlign; }

struct Carve {
  size_t off = 0;
  size_t take(size_t bytes) { size_t o = off; off = round_up(off + bytes); return o; }
};

inline int ring_ok(int W, int N, int Wcap) {
  const long need = (long)std::min<long>(W, (long)N - 1) + 1;
  return Wcap >= need;
}

// --------------------------------------------------------------- writer --
int check_write(const lla_write_params& p) {
  if (p.B < 0 || p.n < 0 || p.pos0 < 0 || p.Ncap < 0) return LLA_ERR_SHAPE;
  if (!lat_dtype_ok(p.out_dtype)) return LLA_ERR_DTYPE;
  const bool fp8 = p.out_dtype == LLA_FP8_E4M3;
  if (fp8 && p.mode == LLA_WRITE_PERHEAD) return LLA_ERR_UNSUPPORTED;   // fp8 rows feed the absorbed read
  if (p.mode != LLA_WRITE_HLA && p.mode != LLA_WRITE_PERHEAD && p.mode != LLA_WRITE_FOLDED)
    return LLA_ERR_UNSUPPORTED;
  if (p.T < 1 || p.H < 1 || p.d_h < 2) return LLA_ERR_SHAPE;
  if ((long)p.pos0 + p.n > p.Ncap) return LLA_ERR_SHAPE;
  const int mult = p.out_dtype == LLA_BF16 ? 8 : fp8 ? 16 : 4;
  if (p.mode == LLA_WRITE_HLA) {
    if (p.T < 2 || p.D < 16 || p.D % 16) return LLA_ERR_SHAPE;
    if (p.r_k < 2 || p.r_v < 1 || p.r_1 < 1) return LLA_ERR_SHAPE;
    if (p.r_k % 2 || p.r_1 % 2 || p.d_h % 2) return LLA_ERR_SHAPE;
    if ((p.r_k + p.r_v) % mult || (2 * p.r_1) % mult) return LLA_ERR_ALIGN;
  } else {
    if (p.d_h % 16) return LLA_ERR_SHAPE;
    if (p.r_k < 1 || p.r_v < 1) return LLA_ERR_SHAPE;
    if (p.mode == LLA_WRITE_PERHEAD && (p.r_k != p.r_v)) return LLA_ERR_SHAPE;
    if (p.mode == LLA_WRITE_PERHEAD && (p.r_k % mult)) return LLA_ERR_ALIGN;
    if (p.mode == LLA_WRITE_FOLDED && ((p.r_k + p.r_v) % mult || p.r_k % 2)) return LLA_ERR_ALIGN;
  }
  if (p.B == 0 || p.n == 0) return LLA_OK;
  if (!p.x || !p.out0) return LLA_ERR_NULL;
  if (p.mode == LLA_WRITE_HLA && (!p.E_main || !p.E_1 || !p.out1)) return LLA_ERR_NULL;
  if (p.mode != LLA_WRITE_HLA && (!p.xv || !p.E_K || !p.E_V)) return LLA_ERR_NULL;
  if (p.mode == LLA_WRITE_PERHEAD && !p.out1) return LLA_ERR_NULL;
  const size_t es = elem_size(p.out_dtype);
  if (!aligned(p.out0, 16) || (p.out1 && !aligned(p.out1, 16))) return LLA_ERR_ALIGN;
  if ((p.out_stride_b * es) % 16 || (p.out_stride_n * es) % 16) return LLA_ERR_ALIGN;
  if (p.mode == LLA_WRITE_PERHEAD && (p.out_stride_h * es) % 16) return LLA_ERR_ALIGN;
  if (p.mode == LLA_WRITE_HLA && ((p.out1_stride_b * es) % 16 || (p.out1_stride_n * es) % 16))
    return LLA_ERR_ALIGN;
  if (!aligned(p.x, 4) || (p.xv && !aligned(p.xv, 4))) return LLA_ERR_ALIGN;
  if (p.x_stride_b < 0 || p.x_stride_n < 0 || p.x_stride_t < 0) return LLA_ERR_SHAPE;
  const int64_t row = p.mode == LLA_WRITE_HLA ? (int64_t)p.D : (int64_t)p.H * p.d_h;
  if (p.x_stride_t < row) return LLA_ERR_SHAPE;
  const int extra = fp8 ? kFp8Extra : 0;
  if (fp8 && (p.r_k + p.r_v > 2048 || 2 * p.r_1 > 2048)) return LLA_ERR_UNSUPPORTED;
  if (p.mode == LLA_WRITE_HLA) {
    if (p.out_stride_n < p.r_k + p.r_v + extra || p.out1_stride_n < 2 * p.r_1 + extra) return LLA_ERR_SHAPE;
  } else if (p.mode == LLA_WRITE_PERHEAD) {
    if (p.out_stride_n < p.r_k) return LLA_ERR_SHAPE;
  } else if (p.out_stride_n < p.r_k + p.r_v + extra) {
    return LLA_ERR_SHAPE;
  }
  return LLA_OK;
}

WriterArgs writer_args(const lla_write_params& p) {
  WriterArgs a;
  std::memset(&a, 0, sizeof(a));
  a.mode = p.mode; a.B = p.B; a.n_tok = p.n; a.pos0 = p.pos0; a.T = p.T; a.H = p.H;
  a.d_h = p.d_h; a.D = p.D; a.r_k = p.r_k; a.r_v = p.r_v; a.r_1 = p.r_1;
  a.rotate = p.mode == LLA_WRITE_HLA ? (p.rotate_keys != 0) : 0;
  a.base = p.rope_base;
  a.x = p.x; a.xv = p.xv; a.xs_b = p.x_stride_b; a.xs_n = p.x_stride_n; a.xs_t = p.x_stride_t;
  a.E_main = p.E_main; a.E_1 = p.E_1; a.E_K = p.E_K; a.E_V = p.E_V;
  a.out0 = p.out0; a.out1 = p.out1; a.dtype = p.out_dtype;
  a.os_b = p.out_stride_b; a.os_h = p.out_stride_h; a.os_n = p.out_stride_n;
  a.o1s_b = p.out1_stride_b; a.o1s_n = p.out1_stride_n;
  a.M = p.B * p.n;
  if (p.mode == LLA_WRITE_HLA) {
    a.Z = 2; a.Nmax = std::max(p.r_k + p.r_v, 2 * p.r_1);
  } else if (p.mode == LLA_WRITE_PERHEAD) {
    a.Z = 2 * p.H; a.Nmax = std::max(p.r_k, p.r_v);
  } else {
    a.Z = 2; a.Nmax = std::max(p.r_k, p.r_v);
  }
  a.Nmax += a.Nmax % 2;
  // tensor cores (3xTF32, fp32-accurate) when the rows are stored as bf16 or fp8
  a.use_tc = p.out_dtype != LLA_F32 && writer_tc_ok(a);
  const int sms = num_sms();
  a.S = a.use_tc ? writer_tc_splits(a, sms) : writer_pick_splits(a, sms);
  return a;
}

// ------------------------------------------------------- decode checks --
int check_hla(const hla_decode_params& p) {
  if (p.win_stream && !p.win_events) return LLA_ERR_NULL;
  if (p.B < 0 || p.nt < 0 || p.nq < 0) return LLA_ERR_SHAPE;
  const int nq = p.nq > 1 ? p.nq : 1;
  if (!lat_dtype_ok(p.lat_dtype) || !dtype_ok(p.win_dtype)) return LLA_ERR_DTYPE;
  if (p.H < 1 || p.d_h < 4 || p.d_h % 4 || p.T < 1 || p.t0 < 0 || p.t0 + p.nt > p.T) return LLA_ERR_SHAPE;
  if (p.N < 1 || p.W < 0 || p.r_k < 2 || p.r_k % 2 || p.r_v < 1) return LLA_ERR_SHAPE;
  const bool fp8 = p.lat_dtype == LLA_FP8_E4M3;
  if (fp8 && !absorb_fp8_supported(p.r_k, p.r_v, p.nt * p.H)) return LLA_ERR_UNSUPPORTED;
  if (p.d_h > 128) return LLA_ERR_UNSUPPORTED;
  if (p.r_v > 1024 || p.r_k + p.r_v > 2048) return LLA_ERR_UNSUPPORTED;
  if ((long)nq * p.nt * p.H > 65535) return LLA_ERR_UNSUPPORTED;
  if (p.N < nq) return LLA_ERR_SHAPE;
  if (nq == 1 ? !ring_ok(p.W, p.N, p.Wcap) : (long)p.Wcap < std::min<long>(p.N, (long)p.W + nq)) return LLA_ERR_SHAPE;
  if (!std::isfinite(p.scale) || p.scale < 0.f) return LLA_ERR_SHAPE;
  if (p.B == 0 || p.nt == 0) return LLA_OK;
  const int n_lat = std::max(0, p.N - 1 - p.W);
  if (!p.A || !p.Bm || !p.q || !p.win_k || !p.win_v || !p.out) return LLA_ERR_NULL;
  if (n_lat > 0 && !p.lat) return LLA_ERR_NULL;
  // several positions share the tensor-core read (bf16 or fp8 rows, <= 64 rows)
  if (nq > 1 && n_lat > 0 &&
      !(p.lat_dtype == LLA_FP8_E4M3 ? absorb_fp8_supported(p.r_k, p.r_v, nq * p.nt * p.H)
                                    : absorb_tc_supported(p.lat_dtype, p.r_k, p.r_v, nq * p.nt * p.H)))
    return LLA_ERR_UNSUPPORTED;
  const size_t es = elem_size(p.lat_dtype);
  if (n_lat > 0) {
    if (!aligned(p.lat, 16) || (p.lat_stride_b * es) % 16 || (p.lat_stride_n * es) % 16) return LLA_ERR_ALIGN;
    if (((size_t)(p.r_k + p.r_v) * es) % 16 || ((size_t)p.r_k * es) % 16) return LLA_ERR_ALIGN;
    if (p.lat_stride_n < p.r_k + p.r_v + (fp8 ? kFp8Extra : 0) || p.lat_stride_b < 0) return LLA_ERR_SHAPE;
  }
  if (!aligned(p.A, 16) || !aligned(p.Bm, 16) || p.r_k % 4) return LLA_ERR_ALIGN;
  if (!aligned(p.q, 4) || !aligned(p.out, 4)) return LLA_ERR_ALIGN;
  if (!aligned(p.win_k, 16) || !aligned(p.win_v, 16)) return LLA_ERR_ALIGN;
  if ((p.win_stride_b * elem_size(p.win_dtype)) % 16) return LLA_ERR_ALIGN;
  const int64_t rowlen = (int64_t)nq * p.nt * p.H * p.d_h;
  if (p.q_stride_b < rowlen || p.out_stride_b < rowlen) return LLA_ERR_SHAPE;
  if (p.win_stride_b < (int64_t)p.T * p.Wcap * p.H * p.d_h) return LLA_ERR_SHAPE;
  return LLA_OK;
}

int check_lla(const lla_decode_params& p) {
  if (p.B < 0 || p.nt < 0) return LLA_ERR_SHAPE;
  if (!lat_dtype_ok(p.lat_dtype) || !dtype_ok(p.win_dtype)) return LLA_ERR_DTYPE;
  if (p.lat_dtype == LLA_FP8_E4M3) return LLA_ERR_UNSUPPORTED;   // fp8 rows are read by the absorbed read
  if (p.H < 1 || p.d_h < 4 || p.d_h % 4 || p.T < 1 || p.t0 < 0 || p.t0 + p.nt > p.T) return LLA_ERR_SHAPE;
  if (p.N < 1 || p.W < 0 || p.r < 1) return LLA_ERR_SHAPE;
  if (p.d_h > 128 || p.r > 128) return LLA_ERR_UNSUPPORTED;
  if ((long)p.nt * p.H > 65535) return LLA_ERR_UNSUPPORTED;
  if (!ring_ok(p.W, p.N, p.Wcap)) return LLA_ERR_SHAPE;
  if (!std::isfinite(p.scale) || p.scale < 0.f) return LLA_ERR_SHAPE;
  if (p.B == 0 || p.nt == 0) return LLA_OK;
  const int n_lat = std::max(0, p.N - 1 - p.W);
  if (!p.UK || !p.UV || !p.q || !p.win_k || !p.win_v || !p.out) return LLA_ERR_NULL;
  if (n_lat > 0 && (!p.cK || !p.cV)) return LLA_ERR_NULL;
  const size_t es = elem_size(p.lat_dtype);
  if (n_lat > 0) {
    if (!aligned(p.cK, 16) || !aligned(p.cV, 16)) return LLA_ERR_ALIGN;
    if ((p.lat_stride_b * es) % 16 || (p.lat_stride_h * es) % 16 || ((size_t)p.r * es) % 16) return LLA_ERR_ALIGN;
    if (p.lat_stride_h < (int64_t)n_lat * p.r || p.lat_stride_b < 0) return LLA_ERR_SHAPE;
  }
  if (!aligned(p.UK, 16) || !aligned(p.UV, 16)) return LLA_ERR_ALIGN;
  if (!aligned(p.q, 4) || !aligned(p.out, 4)) return LLA_ERR_ALIGN;
  if (!aligned(p.win_k, 16) || !aligned(p.win_v, 16)) return LLA_ERR_ALIGN;
  if ((p.win_stride_b * elem_size(p.win_dtype)) % 16) return LLA_ERR_ALIGN;
  const int64_t rowlen = (int64_t)p.nt * p.H * p.d_h;
  if (p.q_stride_b < rowlen || p.out_stride_b < rowlen) return LLA_ERR_SHAPE;
  if (p.win_stride_b < (int64_t)p.T * p.Wcap * p.H * p.d_h) return LLA_ERR_SHAPE;
  return LLA_OK;
}

// Workspace layout of the absorbed read.
struct HlaPlan {
  int rows, n_lat, win_start, n_win, S, tps, use_tc, rows_pad, Sw, cpt, HG;
  size_t o_qlat, o_pml, o_py, o_wml, o_wy, o_qbf, o_err, bytes;
};

HlaPlan plan_hla(const hla_decode_params& p) {
  HlaPlan pl;
  const int sms = num_sms();
  const long target_ctas = 4L * sms;   // SIMT split heuristic: about four CTAs per SM
  // SIMT split: one CTA per (split, sequence, 16 rows)
  pl.rows = (p.nq > 1 ? p.nq : 1) * p.nt * p.H;
  const int i = p.N - 1;
  pl.n_lat = std::max(0, i - p.W);
  pl.win_start = pl.n_lat;
  pl.n_win = i - pl.win_start + 1;
  pl.use_tc = pl.n_lat > 0 && (p.lat_dtype == LLA_FP8_E4M3 ? absorb_fp8_supported(p.r_k, p.r_v, pl.rows)
                                                             : absorb_tc_supported(p.lat_dtype, p.r_k, p.r_v, pl.rows));
  pl.rows_pad = pl.use_tc ? absorb_tc_rows_pad(pl.rows) : pl.rows;
  if (pl.use_tc) {
    // tensor-core read: one CTA per (split, sequence), 64-token tiles
    // LLA_READ_SPLITS overrides the planner's split count (tuning and tests;
    // it sizes the workspace too, so set it before the first size query)
    int S = absorb_tc_splits(p.B, pl.n_lat, sms);
    if (const char* env = std::getenv("LLA_READ_SPLITS")) {
      const int v = std::atoi(env);
      if (v >= 1) S = std::min(v, std::min((pl.n_lat + 63) / 64, 16));
    }
    pl.tps = (int)(((pl.n_lat + S - 1) / S + 63) / 64 * 64);
    pl.S = (pl.n_lat + pl.tps - 1) / pl.tps;
  } else if (pl.n_lat > 0) {
    const long ctas = (long)p.B * ((pl.rows + 15) / 16);
    long S = (target_ctas + ctas - 1) / ctas;
    const long tiles = (pl.n_lat + 15) / 16;
    S = std::max(1L, std::min(std::min(S, tiles), (long)map_max_splits()));
    pl.tps = (int)(((pl.n_lat + S - 1) / S + 15) / 16 * 16);
    pl.S = (pl.n_lat + pl.tps - 1) / pl.tps;
  } else {
    pl.S = 0; pl.tps = 0;
  }
  pl.Sw = window_chunks(p.B, p.nt, p.H, pl.n_win, p.win_dtype, p.d_h, sms, &pl.cpt, &pl.HG);
  const size_t br = (size_t)p.B * pl.rows;
  Carve c;
  pl.o_qbf = c.take(pl.use_tc ? (size_t)p.B * 64 * p.r_k * 2 : 0);
  pl.o_qlat = c.take(pl.use_tc ? 0 : br * p.r_k * 4);
  pl.o_pml = c.take((size_t)pl.S * br * 2 * 4);
  pl.o_py = c.take((size_t)pl.S * br * p.r_v * 4);
  pl.o_wml = c.take((size_t)pl.Sw * br * 2 * 4);
  pl.o_wy = c.take((size_t)pl.Sw * br * p.d_h * 4);
  pl.o_err = c.take(sizeof(int));
  pl.bytes = c.off;
  return pl;
}

HlaPlan plan_lla(const lla_decode_params& p) {
  HlaPlan pl;
  const int sms = num_sms();
  const long target_ctas = 4L * sms;
  pl.rows = p.nt * p.H;
  const int i = p.N - 1;
  pl.n_lat = std::max(0, i - p.W);
  pl.win_start = pl.n_lat;
  pl.n_win = i - pl.win_start + 1;
  // tensor-core reconstruction: bf16 latents whose rows and strides allow a
  // tensor-map view; one CTA per (loop, head, sequence) covers all tokens
  pl.use_tc = pl.n_lat > 0 && p.lat_dtype == LLA_BF16 && p.r % 8 == 0 && p.d_h % 16 == 0 &&
              (p.lat_stride_b * 2) % 16 == 0 && (p.lat_stride_h * 2) % 16 == 0;
  pl.rows_pad = pl.rows;
  if (pl.use_tc) {
    pl.S = 1;
    pl.tps = (pl.n_lat + 31) / 32 * 32;
  } else if (pl.n_lat > 0) {
    const long ctas = (long)p.B * pl.rows;
    long S = (target_ctas + ctas - 1) / ctas;
    const long tiles = (pl.n_lat + 31) / 32;
    S = std::max(1L, std::min(S, tiles));
    pl.tps = (int)(((pl.n_lat + S - 1) / S + 31) / 32 * 32);
    pl.S = (pl.n_lat + pl.tps - 1) / pl.tps;
  } else {
    pl.S = 0; pl.tps = 0;
  }
  pl.Sw = window_chunks(p.B, p.nt, p.H, pl.n_win, p.win_dtype, p.d_h, sms, &pl.cpt, &pl.HG);
  const size_t br = (size_t)p.B * pl.rows;
  Carve c;
  pl.o_qlat = 0;
  pl.o_pml = c.take((size_t)pl.S * br * 2 * 4);
  pl.o_py = c.take((size_t)pl.S * br * p.d_h * 4);
  pl.o_wml = c.take((size_t)pl.Sw * br * 2 * 4);
  pl.o_wy = c.take((size_t)pl.Sw * br * p.d_h * 4);
  pl.o_err = c.take(sizeof(int));
  pl.bytes = c.off;
  return pl;
}

int ws_ok(void* ws, size_t ws_bytes, size_t need) {
  if (need == 0) return LLA_OK;
  if (!ws || !aligned(ws, kAlign) || ws_bytes < need) return LLA_ERR_WORKSPACE;
  return LLA_OK;
}

thread_local int g_last_cuda_error = 0;   // cudaError_t behind the calling thread's last LLA_ERR_CUDA

inline int cuda_status(cudaError_t e) {
  if (e == cudaSuccess) return LLA_OK;
  g_last_cuda_error = (int)e;
  return LLA_ERR_CUDA;
}

// Optional measurement hook: record caller-owned event i (0 = before, 1 = after
// the latent-read kernel) on the stream; captured as an external event node.
inline cudaError_t mark(void* events, int i, cudaStream_t s) {
  if (!events) return cudaSuccess;
  cudaEvent_t ev = reinterpret_cast<cudaEvent_t*>(events)[i];
  cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
  cudaError_t e = cudaStreamIsCapturing(s, &cs);
  if (e != cudaSuccess) return e;
  return cs == cudaStreamCaptureStatusActive ? cudaEventRecordWithFlags(ev, s, cudaEventRecordExternal)
                                             : cudaEventRecord(ev, s);
}

}  // namespace
}  // namespace lla

using namespace lla;

extern "C" {

int lla_abi_version(void) { return kAbiVersion; }

int lla_last_cuda_error(void) { return g_last_cuda_error; }

const char* lla_cuda_error_name(int cuda_error) { return cudaGetErrorName((cudaError_t)cuda_error); }

const char* lla_status_str(int s) {
  switch (s) {
    case LLA_OK: return "ok";
    case LLA_ERR_NULL: return "a required pointer is NULL";
    case LLA_ERR_SHAPE: return "sizes are out of range or inconsistent";
    case LLA_ERR_DTYPE: return "unknown dtype code";
    case LLA_ERR_ALIGN: return "pointer or stride breaks the 16-byte alignment rule";
    case LLA_ERR_WORKSPACE: return "workspace is NULL, misaligned or too small";
    case LLA_ERR_UNSUPPORTED: return "valid arguments outside what the library supports";
    case LLA_ERR_CUDA: return "a CUDA runtime call or kernel launch failed";
    default: return "unknown status";
  }
}

size_t lla_write_workspace_bytes(const lla_write_params* p) {
  if (!p || check_write(*p) != LLA_OK) return 0;
  if (p->B == 0 || p->n == 0) return 0;
  const WriterArgs a = writer_args(*p);
  return round_up(writer_workspace_floats(a) * sizeof(float));
}

int lla_write_latents(const lla_write_params* p, void* ws, size_t ws_bytes, lla_stream stream) {
  if (!p) return LLA_ERR_NULL;
  int st = check_write(*p);
  if (st != LLA_OK) return st;
  if (p->B == 0 || p->n == 0) return LLA_OK;
  WriterArgs a = writer_args(*p);
  const size_t need = round_up(writer_workspace_floats(a) * sizeof(float));
  st = ws_ok(ws, ws_bytes, need);
  if (st != LLA_OK) return st;
  a.part = reinterpret_cast<float*>(ws);
  return cuda_status(launch_writer(a, reinterpret_cast<cudaStream_t>(stream)));
}

size_t hla_decode_workspace_bytes(const hla_decode_params* p) {
  if (!p || check_hla(*p) != LLA_OK || p->B == 0 || p->nt == 0) return 0;
  return plan_hla(*p).bytes;
}

int hla_decode_attn(const hla_decode_params* p, void* ws, size_t ws_bytes, lla_stream stream) {
  if (!p) return LLA_ERR_NULL;
  int st = check_hla(*p);
  if (st != LLA_OK) return st;
  if (p->B == 0 || p->nt == 0) return LLA_OK;
  const HlaPlan pl = plan_hla(*p);
  st = ws_ok(ws, ws_bytes, pl.bytes);
  if (st != LLA_OK) return st;
  char* w = reinterpret_cast<char*>(ws);
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);

  AbsorbArgs a;
  std::memset(&a, 0, sizeof(a));
  a.B = p->B; a.H = p->H; a.d_h = p->d_h; a.T = p->T; a.t0 = p->t0; a.nt = p->nt;
  a.N = p->N; a.W = p->W; a.r_k = p->r_k; a.r_v = p->r_v; a.rows = pl.rows;
  a.n_lat = pl.n_lat; a.win_start = pl.win_start; a.n_win = pl.n_win;
  a.lat = p->lat; a.lat_dtype = p->lat_dtype; a.ls_b = p->lat_stride_b; a.ls_n = p->lat_stride_n;
  a.A = p->A; a.Bm = p->Bm; a.q = p->q; a.qs_b = p->q_stride_b;
  a.rotate = p->rotate_query != 0; a.base = p->rope_base;
  a.wk = p->win_k; a.wv = p->win_v; a.win_dtype = p->win_dtype; a.Wcap = p->Wcap; a.wins_b = p->win_stride_b;
  a.out = p->out; a.outs_b = p->out_stride_b;
  const float scale = p->scale > 0.f ? p->scale : 1.0f / std::sqrt((float)p->d_h);
  a.qmul = scale * kLog2e;
  a.qlat = reinterpret_cast<float*>(w + pl.o_qlat);
  a.part_ml = reinterpret_cast<float*>(w + pl.o_pml);
  a.part_y = reinterpret_cast<float*>(w + pl.o_py);
  a.win_ml = reinterpret_cast<float*>(w + pl.o_wml);
  a.win_y = reinterpret_cast<float*>(w + pl.o_wy);
  a.S = pl.S; a.tps = pl.tps; a.Sw = pl.Sw; a.cpt = pl.cpt;
  a.use_tc = pl.use_tc; a.rows_pad = pl.rows_pad;
  a.qbf = reinterpret_cast<__nv_bfloat16*>(w + pl.o_qbf);
  a.err = reinterpret_cast<int*>(w + pl.o_err);
  const int nq = p->nq > 1 ? p->nq : 1;
  const int rows_q = p->nt * p->H;     // rows of one query position
  a.nq = nq; a.rows_per_q = rows_q;

  MapArgs qm;
  std::memset(&qm, 0, sizeof(qm));
  qm.B = a.B; qm.rows = a.rows; qm.K = a.d_h; qm.N = a.r_k; qm.d_h = a.d_h;
  qm.W = a.A; qm.X = a.q; qm.xs_b = a.qs_b; qm.xs_row = a.d_h;
  qm.rotate = a.rotate; qm.pos = a.N - nq; qm.use_tc = a.use_tc; qm.base = a.base; qm.qmul = a.qmul;
  if (nq > 1) { qm.ncodec = rows_q; qm.rows_per_q = rows_q; }   // position of row g: N - nq + g / rows_q
  qm.q_f16 = a.lat_dtype == LLA_FP8_E4M3 && a.use_tc;   // no latent token: the operand is unused
  qm.qlat = a.qlat; qm.qbf = a.qbf;
  cudaError_t e = cudaSuccess;
  // optional: the window on the caller's second stream, beside the map and the read
  const cudaStream_t sw = p->win_stream ? static_cast<cudaStream_t>(p->win_stream) : s;
  // the error word is cleared by the query map, the call's first kernel, unless
  // the window runs on its own stream beside it: then by a memset before both
  if (sw != s) e = cudaMemsetAsync(a.err, 0, sizeof(int), s);
  else qm.clear_err = a.err;
  cudaEvent_t* wev = reinterpret_cast<cudaEvent_t*>(p->win_events);
  if (e == cudaSuccess && sw != s) {
    e = cudaEventRecord(wev[0], s);
    if (e == cudaSuccess) e = cudaStreamWaitEvent(sw, wev[0], 0);
  }
  if (e == cudaSuccess) {
    // tensor-core map when the shapes allow a tensor-map view, else the SIMT map
    e = query_map_tc_ok(qm) ? launch_query_map_tc(qm, a.err, s) : cudaErrorNotSupported;
    // the SIMT map writes bf16 only; fp8 rows need the tensor-core map's f16 operand
    if (e == cudaErrorNotSupported && !qm.q_f16) e = launch_query_map(qm, s);
  }
  if (e == cudaSuccess) e = mark(p->timing_events, 0, s);
  if (e == cudaSuccess && a.n_lat > 0)
    e = a.lat_dtype == LLA_FP8_E4M3 ? launch_absorb_split_fp8(a, s)
        : a.use_tc ? launch_absorb_split_tc(a, s) : launch_absorb_split_simt(a, s);
  if (e == cudaSuccess) e = mark(p->timing_events, 1, s);
  // exact window: one launch per query position p (its own tokens and R_i)
  for (int qp = 0; qp < nq && e == cudaSuccess; ++qp) {
    const int ip = a.N - nq + qp;
    WindowArgs wa;
    wa.B = a.B; wa.rows = rows_q; wa.H = a.H; wa.d_h = a.d_h; wa.t0 = a.t0; wa.Wcap = a.Wcap;
    wa.win_start = std::max(0, ip - a.W); wa.n_win = ip - wa.win_start + 1;
    wa.Sw = a.Sw; wa.cpt = a.cpt; wa.HG = pl.HG;
    wa.wk = a.wk; wa.wv = a.wv; wa.dtype = a.win_dtype; wa.wins_b = a.wins_b;
    wa.q = a.q; wa.q_sb = a.qs_b; wa.q_srow = a.d_h; wa.qmul = a.qmul;
    wa.rotate = a.rotate; wa.pos = ip; wa.base = a.base;
    wa.win_ml = a.win_ml; wa.win_y = a.win_y; wa.err = a.err;
    wa.rows_total = a.rows; wa.row0 = qp * rows_q;
    e = launch_window(wa, sw);
  }
  if (e == cudaSuccess && sw != s) {
    e = cudaEventRecord(wev[1], sw);
    if (e == cudaSuccess) e = cudaStreamWaitEvent(s, wev[1], 0);
  }
  if (e == cudaSuccess) {
    MapArgs om;
    std::memset(&om, 0, sizeof(om));
    om.B = a.B; om.rows = a.rows; om.K = a.r_v; om.N = a.d_h; om.d_h = a.d_h; om.W = a.Bm;
    if (nq > 1) om.ncodec = rows_q;
    om.part_ml = a.part_ml; om.part_y = a.part_y; om.win_ml = a.win_ml; om.win_y = a.win_y; om.S = a.S;
    om.Sw = a.Sw;
    om.out = a.out; om.outs_b = a.outs_b; om.err = a.err;
    e = (a.use_tc && output_map_tc_ok(om)) ? launch_output_map_tc(om, s) : cudaErrorNotSupported;
    if (e == cudaErrorNotSupported) e = launch_output_map(om, s);
  }
  return cuda_status(e);
}

size_t lla_decode_workspace_bytes(const lla_decode_params* p) {
  if (!p || check_lla(*p) != LLA_OK || p->B == 0 || p->nt == 0) return 0;
  return plan_lla(*p).bytes;
}

int lla_decode_attn(const lla_decode_params* p, void* ws, size_t ws_bytes, lla_stream stream) {
  if (!p) return LLA_ERR_NULL;
  int st = check_lla(*p);
  if (st != LLA_OK) return st;
  if (p->B == 0 || p->nt == 0) return LLA_OK;
  const HlaPlan pl = plan_lla(*p);
  st = ws_ok(ws, ws_bytes, pl.bytes);
  if (st != LLA_OK) return st;
  char* w = reinterpret_cast<char*>(ws);
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const float scale = p->scale > 0.f ? p->scale : 1.0f / std::sqrt((float)p->d_h);

  ReconArgs a;
  std::memset(&a, 0, sizeof(a));
  a.B = p->B; a.H = p->H; a.d_h = p->d_h; a.r = p->r; a.T = p->T; a.t0 = p->t0; a.nt = p->nt;
  a.N = p->N; a.W = p->W; a.rows = pl.rows;
  a.n_lat = pl.n_lat; a.win_start = pl.win_start; a.n_win = pl.n_win;
  a.cK = p->cK; a.cV = p->cV; a.lat_dtype = p->lat_dtype; a.ls_b = p->lat_stride_b; a.ls_h = p->lat_stride_h;
  a.UK = p->UK; a.UV = p->UV; a.q = p->q; a.qs_b = p->q_stride_b;
  a.wk = p->win_k; a.wv = p->win_v; a.win_dtype = p->win_dtype; a.Wcap = p->Wcap; a.wins_b = p->win_stride_b;
  a.out = p->out; a.outs_b = p->out_stride_b;
  a.qmul = scale * kLog2e;
  a.part_ml = reinterpret_cast<float*>(w + pl.o_pml);
  a.part_y = reinterpret_cast<float*>(w + pl.o_py);
  a.win_ml = reinterpret_cast<float*>(w + pl.o_wml);
  a.win_y = reinterpret_cast<float*>(w + pl.o_wy);
  a.S = pl.S; a.tps = pl.tps; a.Sw = pl.Sw; a.cpt = pl.cpt;
  int* err = reinterpret_cast<int*>(w + pl.o_err);

  cudaError_t e = cudaMemsetAsync(err, 0, sizeof(int), s);
  if (e == cudaSuccess) e = mark(p->timing_events, 0, s);
  if (e == cudaSuccess && a.n_lat > 0) {
    e = (pl.use_tc && recon_tc_supported(a)) ? launch_recon_tc(a, err, s, num_sms()) : cudaErrorNotSupported;
    if (e == cudaErrorNotSupported) e = launch_recon_split_simt(a, s);   // S = 1 covers every token as well
  }
  if (e == cudaSuccess) e = mark(p->timing_events, 1, s);
  if (e == cudaSuccess) {
    WindowArgs wa;
    wa.B = a.B; wa.rows = a.rows; wa.H = a.H; wa.d_h = a.d_h; wa.t0 = a.t0; wa.Wcap = a.Wcap;
    wa.win_start = a.win_start; wa.n_win = a.n_win; wa.Sw = a.Sw; wa.cpt = a.cpt; wa.HG = pl.HG;
    wa.wk = a.wk; wa.wv = a.wv; wa.dtype = a.win_dtype; wa.wins_b = a.wins_b;
    wa.q = a.q; wa.q_sb = a.qs_b; wa.q_srow = a.d_h; wa.qmul = a.qmul;
    wa.rotate = 0; wa.pos = a.N - 1; wa.base = 0.0;
    wa.win_ml = a.win_ml; wa.win_y = a.win_y; wa.err = err;
    wa.rows_total = a.rows; wa.row0 = 0;
    e = launch_window(wa, s);
  }
  if (e == cudaSuccess) {
    MergeArgs g;
    g.B = a.B; g.rows = a.rows; g.H = a.H; g.d_h = a.d_h; g.S = a.S; g.Sw = a.Sw; g.Y = a.d_h;
    g.part_ml = a.part_ml; g.part_y = a.part_y; g.win_ml = a.win_ml; g.win_y = a.win_y;
    g.Bm = nullptr; g.out = a.out; g.outs_b = a.outs_b; g.err = err;
    e = launch_merge(g, s);
  }
  return cuda_status(e);
}

}  // extern "C"
