/*
 * lla.h -- C ABI of the decode-time latent attention library for looped
 * (weight-tied, T-recurrence) Transformers.
 *
 * The method is defined on two pages:
 *   - "Looped Latent Attention: Cross-Loop Key-Value Compression For Looped
 *     Transformers" (ICLR 2027 submission page, Abstract): per-head LLA codec
 *     that stores compact K and V latents and "reconstructs loop-specific
 *     vectors only when attention reads them", the LLA-2D variant folding
 *     heads into one latent, and the absorbed variant LLA-D that "reads latents
 *     without reconstruction".
 *   - The Hybrid Latent Attention summary page, "Methodology / Latent Writer"
 *     (eq. 2), "Methodology / Latent Reader" (eqs. 3 and 4) and "Methodology /
 *     Rotary Embedding Alignment".
 *
 * Conventions shared by every entry point
 * ----------------------------------------
 * Pointers.   Every tensor pointer is a DEVICE pointer owned by the caller.
 *             The library never allocates, frees or retains memory, with one
 *             exception: hla_decode_attn_noalloc uses a static device array
 *             held on each device that calls it (see that entry point).
 *             Scratch space is otherwise the caller's `ws` buffer of at least
 *             the size that the matching *_workspace_bytes() returns,
 *             256-byte aligned.  Its contents need not be initialised and are
 *             garbage afterwards.  Split plans, and so workspace sizes, follow
 *             the current device's multiprocessor count: query a size with the
 *             same device current as the call that uses it.
 * Layouts.    Row-major.  Sizes are in elements; strides are int64 element
 *             strides of the outermost (batch, head, token) axes only -- the
 *             inner axes named in each comment are dense.
 * Streams.    Every call only enqueues kernels on `stream` (a cudaStream_t;
 *             NULL = legacy default stream) and returns; it never synchronises.
 *             Inputs must stay valid until that work has run.  Two calls may
 *             share a workspace only if they are ordered on the GPU.  With
 *             LLA_PDL=1 in the environment (read once per process) kernels
 *             are launched with programmatic dependent launch: a kernel's
 *             set-up may overlap the end of the previous kernel on the
 *             stream, and it touches global memory only once that kernel
 *             has completed, so stream order is kept.  LLA_READ_SPLITS=S
 *             (read at each plan) fixes the number of context splits of the
 *             tensor-core latent read instead of the planner's choice; it
 *             changes the workspace size, so set it before any size query.
 *             LLA_RECON_SEQ_PER_CTA=n fixes how many sequences one CTA of
 *             the tensor-core reconstruct walks (lla_decode_attn).  Both are
 *             for tuning and tests; unset, the planners choose.
 * Threads.    Calls from several host threads are safe, each with its own
 *             workspace.  The exception is hla_decode_attn_noalloc: all of its
 *             calls share one scratch array, so calls whose work may overlap
 *             on the GPU race (see that entry point).
 * Errors.     Every function returns an lla_status.  Arguments are validated on
 *             the host before anything is launched: on a validation error
 *             (LLA_ERR_NULL, _SHAPE, _DTYPE, _ALIGN, _WORKSPACE, _UNSUPPORTED)
 *             nothing is launched and outputs are untouched.  LLA_ERR_CUDA
 *             reports a failed launch (cudaGetLastError) or device query; it
 *             can follow work the call had already enqueued, so the outputs of
 *             such a call must be ignored.  Errors raised
 *             by kernels already running surface on the caller's next CUDA
 *             synchronisation, as usual.  No call aborts or traps.  Every wait
 *             inside the kernels (copy completion, tensor-core completion) is
 *             bounded at about two seconds; a kernel that gives up records the
 *             reason in the workspace and the call's outputs are written as NaN
 *             (its status was already returned when it was enqueued).
 * Precision.  Accumulation is fp32 throughout.  bf16 latents are read on the
 *             tensor cores (query operand rounded to bf16 for the score MMA,
 *             probabilities to bf16 for the accumulate MMA, tf32 maps; fp8
 *             rows: query as two e4m3 terms, probabilities in f16); bf16
 *             writer rows use 3xTF32 products (fp32-accurate) before one
 *             round-to-nearest-even; the LLA reconstruction rounds each fp32
 *             decoder to bf16 for its tensor-core product (about 2^-9
 *             relative per entry; output error ~2e-3 relative).  fp32 latents
 *             and rows take fp32 SIMT kernels.
 * Rotary.     R_pos rotates pair p = (x[2p], x[2p+1]) of a length-d vector by
 *             +pos * base^(-2 f(p) / d_h), with f(p) = floor(p * d_h / d):
 *             textbook interleaved RoPE at d = d_h, and m = d / d_h consecutive
 *             pairs per frequency in a latent of rank d (HLA summary, "Rotary
 *             Embedding Alignment").  Angles are computed in fp64.
 * Positions.  A decode call attends from the query at position i = N - 1 to
 *             tokens j = 0..i.  Tokens j < i - W are read from the latent cache
 *             (eq. 4's first sum); tokens max(0, i-W)..i -- W+1 of them once
 *             i >= W, the current token included -- are read exact from the
 *             window ring, where token j lives in slot j mod Wcap (Wcap >= W+1).
 * Softmax.    One softmax over latent and exact scores jointly, scaled by
 *             `scale` (0 selects 1/sqrt(d_h), eq. 3's factor).
 */
#ifndef LLA_H
#define LLA_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st *lla_stream; /* identical to cudaStream_t */

typedef enum {
  LLA_OK = 0,
  LLA_ERR_NULL = 1,        /* a required pointer (or params) is NULL        */
  LLA_ERR_SHAPE = 2,       /* a size is negative, zero where it must not be,
                              inconsistent, or above a documented limit      */
  LLA_ERR_DTYPE = 3,       /* unknown dtype code                             */
  LLA_ERR_ALIGN = 4,       /* a pointer or stride breaks 16-byte alignment   */
  LLA_ERR_WORKSPACE = 5,   /* ws is NULL, misaligned or smaller than needed  */
  LLA_ERR_UNSUPPORTED = 6, /* valid, but a combination the library rejects  */
  LLA_ERR_CUDA = 7         /* a CUDA runtime call or launch failed           */
} lla_status;

/* Storage formats.  LLA_FP8_E4M3 is a latent-row format, not an element
 * type: each token's row holds the e4m3 codes (OCP FP8 E4M3: bias 7, 3
 * mantissa bits, largest finite 448) of its key part and of its value part,
 * then the two parts' fp32 scales and 8 zero bytes:
 *   [codes of c^K: r_k bytes | codes of c^V: r_v bytes | s^K | s^V | 0 x 8]
 * so a row is r_k + r_v + 16 bytes and element (byte) strides apply.  A
 * stored element's value is code * s of its part; s = (largest magnitude of
 * the part) / 448, codes rounded to nearest-even and saturated (HLA summary,
 * "Conclusion / Future directions": combining the latents with quantisation;
 * per-token, per-part scales are this library's reading).  Written by
 * lla_write_latents (HLA and FOLDED modes) and read by hla_decode_attn on the
 * tensor cores: key codes are contracted as e4m3 against the absorbed query
 * written as two e4m3 terms (hi + lo, about 8 significant bits, under a
 * per-row power of two), value codes are widened exactly to f16. */
typedef enum { LLA_F32 = 0, LLA_BF16 = 1, LLA_FP8_E4M3 = 2 } lla_dtype;

/* Version of this ABI; bumped whenever a struct below changes. */
int lla_abi_version(void);

/* Static description of a status code; never NULL. */
const char *lla_status_str(int status);

/* The cudaError_t value behind the most recent LLA_ERR_CUDA returned to the
 * calling thread by any entry point (0 if none yet), and the CUDA runtime's
 * name for it (static, never NULL).  Kept per thread; reading it clears
 * nothing. */
int lla_last_cuda_error(void);
const char *lla_cuda_error_name(int cuda_error);

/* ------------------------------------------------------------------------ */
/* (a) Latent writer                                                          */
/* ------------------------------------------------------------------------ */
typedef enum {
  /* HLA summary, "Latent Writer", eq. 2:
   *   c_j     = sum_{t=2..T} E_t h_{j,t} = [c^K_j ; c^V_j]   (r_k + r_v)
   *   c^(1)_j = E_1 h_{j,1}               = [c^K1_j; c^V1_j]  (2 r_1)
   * Stored rows are [R~_j c^K_j | c^V_j] and [R~_j c^K1_j | c^V1_j] when
   * rotate_keys = 1 (rotation at the token's position, dimension r_k or r_1;
   * eq. 3 only ever uses the rotated key latent), un-rotated otherwise. */
  LLA_WRITE_HLA = 0,
  /* LLA abstract, per-head codec: c^K_{j,h} = sum_t E^K_{t,h} k_{j,t,h},
   * c^V_{j,h} = sum_t E^V_{t,h} v_{j,t,h}, rank r = r_k = r_v.  Keys are
   * post-rotary ("full-RoPE codecs"); nothing is rotated here. */
  LLA_WRITE_PERHEAD = 1,
  /* LLA abstract, LLA-2D: heads folded into one latent,
   * c^K_j = sum_{t,h} E^K_{t,h} k_{j,t,h} (r_k), c^V_j likewise (r_v);
   * stored row [c^K_j | c^V_j]. */
  LLA_WRITE_FOLDED = 2
} lla_write_mode;

typedef struct {
  int32_t mode;            /* lla_write_mode                                   */
  int32_t B;               /* sequences                                        */
  int32_t n;               /* tokens written per sequence (n >= 0)             */
  int32_t pos0;            /* position (= cache row) of the first token        */
  int32_t T, H, d_h, D;    /* loops, heads, head dim, model dim (HLA only)     */
  int32_t r_k, r_v, r_1;   /* HLA: key/value ranks and loop-1 rank;
                              PERHEAD: r_k = r_v = r; FOLDED: r_K, r_V        */
  int32_t rotate_keys;     /* HLA: 1 stores R~_pos c^K (eq. 3's key factor)    */
  double rope_base;        /* rotary base, e.g. 10000                          */
  /* inputs, fp32:
   *   HLA:            x = h [B, n, T, D]           (D dense)
   *   PERHEAD/FOLDED: x = k, xv = v [B, n, T, H, d_h] (H, d_h dense)
   * strides in elements: x_stride_b, x_stride_n, x_stride_t               */
  const float *x;
  const float *xv;
  int64_t x_stride_b, x_stride_n, x_stride_t;
  /* codec, fp32, dense:
   *   HLA:     E_main [T-1, r_k + r_v, D] (E_2..E_T), E_1 [2 r_1, D]
   *   PERHEAD: E_K [T, H, r_k, d_h], E_V [T, H, r_v, d_h]
   *   FOLDED:  E_K [T, H, r_k, d_h], E_V [T, H, r_v, d_h]                 */
  const float *E_main, *E_1, *E_K, *E_V;
  /* outputs (rows [pos0, pos0 + n) of each sequence are overwritten):
   *   HLA:     out0 = main latent [B, Ncap, r_k + r_v], out1 = loop-1 latent
   *            [B, Ncap, 2 r_1]; strides (b, token) in out*_stride_b/_n.
   *   PERHEAD: out0 = c^K, out1 = c^V, each [B, H, Ncap, r]; strides
   *            (b, h, token) in out_stride_b, out_stride_h, out_stride_n.
   *   FOLDED:  out0 = [B, Ncap, r_k + r_v]; out1 unused.
   * Rows must start 16-byte aligned.                                       */
  void *out0, *out1;
  int32_t out_dtype;       /* lla_dtype of both outputs; LLA_FP8_E4M3 rows
                              (HLA and FOLDED only) are r_k + r_v + 16 bytes
                              (HLA loop-1: 2 r_1 + 16) and strides in bytes   */
  int32_t Ncap;            /* cache rows per sequence; pos0 + n <= Ncap        */
  int64_t out_stride_b, out_stride_h, out_stride_n;
  int64_t out1_stride_b, out1_stride_n; /* HLA loop-1 latent                   */
} lla_write_params;

/* Scratch bytes lla_write_latents needs for these params (fp32 split-K
 * partial sums).  Returns 0 for invalid params. */
size_t lla_write_workspace_bytes(const lla_write_params *p);

/* Append latents of n tokens per sequence to the caller's cache.
 * Math: fp32 products and sums; one rounding (nearest-even) to out_dtype.
 * Limits: d_h and D multiples of 16; r_k, r_v, r_1 even and multiples of 8
 * (bf16) / 4 (fp32) so that rows stay 16-byte aligned. */
int lla_write_latents(const lla_write_params *p, void *ws, size_t ws_bytes,
                      lla_stream stream);

/* ------------------------------------------------------------------------ */
/* (b) LLA reconstruct-on-read decode attention                              */
/* ------------------------------------------------------------------------ */
/* LLA abstract: the per-head codec "reconstructs loop-specific vectors only
 * when attention reads them".  For each loop t in [t0, t0+nt) and head h,
 * every latent token j < i - W is rebuilt on chip,
 *   k^_j = U^K_{t,h} c^K_{j,h},  v^_j = U^V_{t,h} c^V_{j,h},
 * and attention runs over rebuilt and exact tokens with one softmax:
 *   o_{t,h} = sum_j a_j v_j,  a = softmax(scale * q_{t,h} . k_j).
 * The rebuilt vectors never leave the chip.  q is post-rotary (the codec acts
 * on post-rotary keys), so nothing is rotated here. */
typedef struct {
  int32_t B, H, d_h, r;    /* batch, heads, head dim, latent rank              */
  int32_t T, t0, nt;       /* loops in the model; this call serves t0..t0+nt-1 */
  int32_t N, W;            /* context length (query at N-1), exact window      */
  const void *cK, *cV;     /* [B, H, >= N-1-W rows, r], lat_dtype              */
  int32_t lat_dtype;
  int64_t lat_stride_b, lat_stride_h; /* token rows are dense (stride r)       */
  const float *UK, *UV;    /* [nt, H, d_h, r] fp32: decoders of loops t0..     */
  const float *q;          /* [B, nt, H, d_h] fp32, post-rotary                */
  int64_t q_stride_b;
  const void *win_k, *win_v; /* ring [B, T, Wcap, H, d_h], win_dtype, dense per
                              sequence; post-rotary keys                       */
  int32_t win_dtype, Wcap;
  int64_t win_stride_b;
  float *out;              /* [B, nt, H, d_h] fp32                             */
  int64_t out_stride_b;
  float scale;             /* 0 -> 1/sqrt(d_h)                                 */
  /* Optional measurement hook: NULL, or the address of two cudaEvent_t
   * values (begin, end).  The call then records them on `stream` right
   * before and right after its latent-read kernel (external event nodes under
   * stream capture), so a caller can time that kernel alone.  Nothing else
   * changes; no work is skipped. */
  void *timing_events;
} lla_decode_params;

size_t lla_decode_workspace_bytes(const lla_decode_params *p);
int lla_decode_attn(const lla_decode_params *p, void *ws, size_t ws_bytes,
                    lla_stream stream);

/* ------------------------------------------------------------------------ */
/* (c) Absorbed latent read: HLA (eqs. 3-4) and LLA-D                         */
/* ------------------------------------------------------------------------ */
/* HLA summary, "Latent Reader":
 *   eq. 3: s^_{ij,t} = (R~_i A_t^T q_{i,t}) . (R~_j c^K_j) / sqrt(d_h)
 *   eq. 4: o_{i,t} = B_t^T sum_{j<i-W} a_{ij,t} c^V_j
 *                    + sum_{i-W<=j<=i} a_{ij,t} v_{j,t}
 * with one softmax a over both sums.  The stored key part is already
 * R~_j c^K_j (lla_write_latents with rotate_keys = 1).  With rotate_query = 1
 * the query is un-rotated: the call forms R~_i A_t^T q for the latent scores
 * and R_i q for the exact tokens.
 * LLA-D (LLA abstract, absorbed variant) is the same read with A = U^K,
 * Bm = (U^V)^T, rotate_query = 0 and a post-rotary q.
 * One call serves one latent (e.g. the loop-1 latent c^(1) with r_k = r_v =
 * r_1, or the main latent with loops 2..T) and the loops t0..t0+nt-1 that
 * share it: every (loop, head) pair is one query row reading the same tile. */
typedef struct {
  int32_t B, H, d_h;
  int32_t T, t0, nt;       /* loops in the model; this call serves t0..t0+nt-1 */
  int32_t N, W;            /* context length (query at N-1), exact window      */
  int32_t r_k, r_v;        /* key and value ranks of this latent               */
  const void *lat;         /* [B, >= N-1-W rows, r_k + r_v], lat_dtype; for
                              LLA_FP8_E4M3 rows of r_k + r_v + 16 bytes        */
  int32_t lat_dtype;
  int64_t lat_stride_b, lat_stride_n;
  const float *A;          /* [nt, H, d_h, r_k] fp32                           */
  const float *Bm;         /* [nt, H, r_v, d_h] fp32                           */
  const float *q;          /* [B, nt, H, d_h] fp32                             */
  int64_t q_stride_b;
  int32_t rotate_query;    /* 1: HLA (q un-rotated); 0: LLA-D (q post-rotary)  */
  double rope_base;
  const void *win_k, *win_v; /* ring [B, T, Wcap, H, d_h], dense per sequence  */
  int32_t win_dtype, Wcap;
  int64_t win_stride_b;
  float *out;              /* [B, nt, H, d_h] fp32                             */
  int64_t out_stride_b;
  float scale;             /* 0 -> 1/sqrt(d_h)                                 */
  /* Optional measurement hook: NULL, or the address of two cudaEvent_t
   * values (begin, end).  The call then records them on `stream` right
   * before and right after its latent-read kernel (external event nodes under
   * stream capture), so a caller can time that kernel alone.  Nothing else
   * changes; no work is skipped. */
  void *timing_events;
  /* Query positions served at once (0 or 1: the decode read of position
   * N - 1).  With nq > 1 the call serves the last nq positions of the context,
   * i_p = N - nq + p (a prefill chunk, or a block of the two-pass procedure's
   * parallel second pass; HLA summary, "Methodology / Fine-tuning"): q and out
   * are [B, nq, nt, H, d_h], row (p, t, h) attends to latent tokens
   * j < i_p - W and to exact tokens max(0, i_p - W) <= j <= i_p of the ring
   * (Wcap >= min(N, W + nq)), and every latent tile is shared by all
   * nq * nt * H rows on the tensor cores (at most 64 rows; bf16 or fp8 rows). */
  int32_t nq;
  /* Optional concurrency for the exact window (HLA summary eq. 4, second
   * sum), which needs neither the query map nor the latent read: NULL, or a
   * stream of the caller's on which the call runs its window kernels while
   * the query map and the latent read run on `stream`.  win_events is then
   * the address of two cudaEvent_t values of the caller's (fork, join): the
   * call records fork on `stream` after zeroing its error word, makes
   * win_stream wait on it, records join on win_stream after the window, and
   * makes `stream` wait on join before the output map; under stream capture
   * this is the usual fork and join.  Results are bit-identical to the
   * single-stream call.  win_stream without win_events: LLA_ERR_NULL. */
  lla_stream win_stream;
  void *win_events;
} hla_decode_params;

size_t hla_decode_workspace_bytes(const hla_decode_params *p);
int hla_decode_attn(const hla_decode_params *p, void *ws, size_t ws_bytes,
                    lla_stream stream);

/* ------------------------------------------------------------------------ */
/* Absorbed read without a caller-provided workspace                          */
/* ------------------------------------------------------------------------ */
/* The pages have no counterpart to this entry point; it is a convenience of
 * this library.  It computes exactly what hla_decode_attn computes, for
 * callers that cannot allocate device memory: code that is handed only input
 * and output buffers (e.g. a plugin whose host interface has no allocator), or
 * a serving engine that has reserved all device memory for its cache, where an
 * extra cudaMalloc fails or synchronises the device mid-decode.
 *
 * Scratch comes from one static device array of LLA_NOALLOC_SCRATCH_BYTES
 * inside the library, held on every device that uses it until the process
 * exits; the call allocates nothing.  The first call on a device looks up the
 * array's device address (cudaGetSymbolAddress, with that device current);
 * make that first call before any stream capture begins.
 * Errors: as hla_decode_attn; LLA_ERR_WORKSPACE when the problem needs more
 * scratch than LLA_NOALLOC_SCRATCH_BYTES (hla_decode_workspace_bytes(p) tells
 * how much).  All calls share the array: calls whose work may overlap on the
 * GPU (other streams, unordered host threads) race on it and must not be
 * issued; order them on one stream.  Nothing in the array needs to start at
 * zero -- each call writes every scratch word before it reads it. */
#define LLA_NOALLOC_SCRATCH_BYTES (32u * 1024u * 1024u)
int hla_decode_attn_noalloc(const hla_decode_params *p, lla_stream stream);

#ifdef __cplusplus
}
#endif
#endif /* LLA_H */
