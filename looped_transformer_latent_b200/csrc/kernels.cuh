// Internal launch interface between the C ABI layer (abi.cu) and the kernels.
// Argument structs are passed by value as kernel parameters.
#pragma once

#include "common.cuh"

namespace lla {

constexpr int kMaxWindowChunks = 16;   // window partials one call can produce

// ---------------------------------------------------------------- writer --
struct WriterArgs {
  int mode, B, n_tok, pos0, T, H, d_h, D, r_k, r_v, r_1, rotate;
  double base;
  const float *x, *xv;
  int64_t xs_b, xs_n, xs_t;
  const float *E_main, *E_1, *E_K, *E_V;
  void *out0, *out1;
  int dtype;
  int64_t os_b, os_h, os_n, o1s_b, o1s_n;
  int M;       // B * n_tok
  int Z;       // independent GEMMs (HLA: 2; PERHEAD: 2H; FOLDED: 2)
  int Nmax;    // largest output width over the Z GEMMs
  int S;       // split-K factor
  int use_tc;  // phase 1 on the tensor cores (3xTF32)
  float* part; // [Z][S][M][Nmax] fp32 partial sums
  int* err;    // tensor-core phase: set on a timed-out wait; the stores are then NaN
};
size_t writer_workspace_floats(const WriterArgs& a);
// k-split count of the writer: a function of the reduction depth only (one
// split per 16 chunks of 32, at most 64), never of the number of tokens, so a
// token's stored row is bit-identical whether it is written in a prefill
// batch or alone (the streaming store of a token leaving the exact window).
int writer_depth_splits(const WriterArgs& a);
int writer_pick_splits(const WriterArgs& a, int num_sms);
cudaError_t launch_writer(const WriterArgs& a, cudaStream_t st);
// tensor-core writer phase 1 (gemm_tc.cu)
bool writer_tc_ok(const WriterArgs& w);
int writer_tc_splits(const WriterArgs& w, int num_sms);
cudaError_t launch_writer_tc(const WriterArgs& w, int* err, cudaStream_t st);

// ------------------------------------------------------ absorbed decode --
struct AbsorbArgs {
  int B, H, d_h, T, t0, nt, N, W, r_k, r_v, rows;
  int n_lat, win_start, n_win;
  const void* lat;
  int lat_dtype;
  int64_t ls_b, ls_n;
  const float *A, *Bm, *q;
  int64_t qs_b;
  int rotate;
  double base;
  const void *wk, *wv;
  int win_dtype, Wcap;
  int64_t wins_b;
  float* out;
  int64_t outs_b;
  float qmul;          // scale * log2(e): scores are kept in base-2 units
  // workspace views
  float *qlat;         // [B][rows][r_k]  (scaled, rotated)
  float *part_ml;      // [S][B][rows][2] (running max, sum) per split
  float *part_y;       // [S][B][rows][r_v]
  float *win_ml;       // [Sw][B][rows][2] per window chunk
  float *win_y;        // [Sw][B][rows][d_h]
  int S, tps;          // splits of the latent range, tokens per split
  int Sw, cpt;         // window chunks, tokens per chunk
  // tensor-core path
  int use_tc;
  int rows_pad;        // rows rounded up to 16 (N of the accumulate MMA)
  // several query positions (the last nq of the context) in one call: rows
  // are (position, loop, head); row r's latent tokens end at
  // n_lat - (nq - 1 - r / rows_per_q); nq = 1 is the plain decode read
  int nq, rows_per_q;
  __nv_bfloat16* qbf;  // [B][r_k/64][64 rows x 64] bf16 Q~, 128-byte swizzled, rows >= rows zero
  int* err;            // 0, or the code of a timed-out wait in the latent read
};

// ------------------------------------------------- reconstruct decode --
struct ReconArgs {
  int B, H, d_h, r, T, t0, nt, N, W, rows;
  int n_lat, win_start, n_win;
  const void *cK, *cV;
  int lat_dtype;
  int64_t ls_b, ls_h;
  const float *UK, *UV, *q;
  int64_t qs_b;
  const void *wk, *wv;
  int win_dtype, Wcap;
  int64_t wins_b;
  float* out;
  int64_t outs_b;
  float qmul;
  float *part_ml, *part_y, *win_ml, *win_y;
  int S, tps, Sw, cpt;
};

// Shared pieces.
// Window partials: one per (token chunk of cpt tokens, sequence, row).  The
// query is the raw q [B][rows][d_h] (strides q_sb, q_srow), rotated by R_pos
// in head space when `rotate` is set and multiplied by qmul.
struct WindowArgs {
  int B, rows, H, d_h, t0, Wcap, win_start, n_win;
  int Sw, cpt, HG;         // chunks, tokens per chunk, head groups (0: register kernel)
  const void *wk, *wv;
  int dtype;
  int64_t wins_b;
  const float* q;
  int64_t q_sb, q_srow;
  float qmul;
  int rotate, pos;
  double base;
  float2 rot[64];          // cos, sin of pair p at pos (set by launch_window when rotate)
  float *win_ml, *win_y;   // [Sw][B][rows_total][2], [Sw][B][rows_total][d_h]
  int rows_total, row0;    // this launch's rows are rows row0.. of rows_total (one query position)
  int* err;                // optional: set to ERR_WINDOW_TIMEOUT if a copy never lands
};
constexpr int ERR_WINDOW_TIMEOUT = 21;
// Kernel choice and chunking of the window for launch_window: returns the
// chunk count, sets *cpt (tokens per chunk) and *HG (head groups of the
// bulk-copy kernel, 0 for the register kernel).
int window_chunks(int B, int nt, int H, int n_win, int dtype, int d_h, int num_sms, int* cpt, int* HG);
struct MergeArgs {
  int B, rows, H, d_h, S, Sw, Y;
  const float *part_ml, *part_y, *win_ml, *win_y;
  const float* Bm;   // [rows][Y][d_h] when mapping latent space back; else null
  float* out;
  int64_t outs_b;
  const int* err;    // optional: when it holds a non-zero code the output is NaN
};

// Per-(loop, head) linear maps of the absorbed read (maps.cu).
struct MapArgs {
  int B, rows, K, N, d_h;
  const float* W;          // [rows][K][N]: A_{t,h} (query map) or B_{t,h} (output map)
  // query map: X = q [B][rows][d_h] (K = d_h, N = r_k)
  const float* X;
  int64_t xs_b, xs_row;
  int rotate, pos, use_tc;
  int q_f16;               // query operand in f16 (fp8 latent read) instead of bf16
  int ncodec;              // codec groups: row g uses codec g mod ncodec (0: rows)
  int rows_per_q;          // query map: row g is at position pos + g / rows_per_q (0: pos)
  double base;
  float qmul;
  float* qlat;
  __nv_bfloat16* qbf;
  // output map: X = sum over splits of the partials (K = r_v, N = d_h), plus
  // Sw window partials in head space
  const float *part_ml, *part_y, *win_ml, *win_y;
  int S, Sw;
  float* out;
  int64_t outs_b;
  const int* err;
  int* clear_err;          // query map: set to 0 before any later kernel of the call reads it (null: no)
};
int map_max_splits();
cudaError_t launch_query_map(const MapArgs& g, cudaStream_t st);
cudaError_t launch_output_map(const MapArgs& g, cudaStream_t st);

// Tensor-core maps (gemm_tc.cu): used with the tensor-core latent read.
struct TcGemmArgs {
  int B, rows, Mtot, K, mtiles, ntiles, S, NB, Sw;
  int nst;                 // shared-memory stages (set by the launcher)
  int ks;                  // output map: k-splits over a cluster of ks CTAs (1: none)
  const float *Aw, *X;     // codec [group][K][Mtot]; activations (per kind)
  int64_t xs_b;
  int rotate, pos, d_h;    // query map epilogue
  int qf16;                // query operand written as f16 (same layout) instead of bf16
  int ncodec;              // codec groups: group g uses codec g mod ncodec
  int rows_per_q;          // query map: group g is at position pos + g / rows_per_q (0: pos)
  double base;
  float qmul;
  __nv_bfloat16* qbf;
  const float *part_ml, *win_ml, *win_y;   // output map epilogue
  float* out;
  int64_t outs_b;
  int* err;
  int* clear_err;          // query map: the call's error word, cleared by one thread (null: no)
  WriterArgs w;            // writer slices
};
bool query_map_tc_ok(const MapArgs& g);
cudaError_t launch_query_map_tc(const MapArgs& g, int* err, cudaStream_t st);
bool output_map_tc_ok(const MapArgs& g);
cudaError_t launch_output_map_tc(const MapArgs& g, cudaStream_t st);

cudaError_t launch_absorb_split_simt(const AbsorbArgs& a, cudaStream_t st);
cudaError_t launch_window(const WindowArgs& w, cudaStream_t st);
cudaError_t launch_merge(const MergeArgs& m, cudaStream_t st);
cudaError_t launch_recon_split_simt(const ReconArgs& a, cudaStream_t st);
// tensor-core reconstruct-on-read (recon_tc.cu): one CTA per (group of loops,
// head, chunk of sequences), each sequence's whole latent range in one CTA,
// i.e. a single split
bool recon_tc_supported(const ReconArgs& a);
cudaError_t launch_recon_tc(const ReconArgs& a, int* err, cudaStream_t st, int num_sms);

bool absorb_tc_supported(int lat_dtype, int r_k, int r_v, int rows);
// fp8 latent rows (LLA_FP8_E4M3): the same read with the codes widened to f16
// on chip and the per-token scales applied on the softmax side (decode_fp8.cu)
bool absorb_fp8_supported(int r_k, int r_v, int rows);
cudaError_t launch_absorb_split_fp8(const AbsorbArgs& a, cudaStream_t st);
int absorb_tc_rows_pad(int rows);
int absorb_tc_splits(int B, int n_lat, int num_sms);
cudaError_t launch_absorb_split_tc(const AbsorbArgs& a, cudaStream_t st);

}  // namespace lla
