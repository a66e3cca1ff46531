/*
 * spts.h -- C ABI of the SPTS prefill hot path on NVIDIA B200 (sm_100a).
 *
 * Self-Predictive Token Skipping (SPTS) is described in "Probe and Skip:
 * Self-Predictive Token Skipping for Efficient Long-Context LLM Inference"
 * (Wu, Wang, Jin, Chen, Wang, 2026).  Its prefill layer
 *   1. scores every key with a few probe queries (Partial Attention Probing,
 *      Fig. 2(a)) and keeps the informative tokens for reduced attention;
 *   2. scores every row with a low-rank proxy of the FFN (Low-rank
 *      Transformation Probing, Fig. 2(b)), fuses that with the attention
 *      score (Table D) and keeps the informative tokens for a reduced FFN;
 *   3. prunes the candidate set at stage boundaries (Multi-Stage Delayed
 *      Pruning, Fig. 2(c), Fig. A, Table B).
 * Skipped rows pass through on the residual stream.
 *
 * Conventions shared by every call
 * --------------------------------
 *  - All tensors are row-major and contiguous unless a stride is passed.
 *    Rows are tokens; pos[] holds each row's original position, strictly
 *    ascending.  Q is [rows, Hq, d]; K and V are [Nc, Hkv, d]; weights use the
 *    nn.Linear layout [out, in] (y = x W^T).  Scores are fp32, indices int32.
 *  - GQA: query head h reads KV head h / (Hq / Hkv).  Causality is by
 *    original position: key j is visible to a query at position p iff
 *    pos_j <= p.
 *  - The caller owns every buffer.  The library never allocates device
 *    memory; scratch comes from the caller's workspace `ws` of `ws_bytes`
 *    bytes, 256-byte aligned, sized by the matching *_workspace() call.  The
 *    first 256 bytes of any workspace hold the device status word; zero them
 *    once (cudaMemsetAsync) before the first use of a workspace.
 *  - Every call is asynchronous on `stream` and validates its arguments on
 *    the host first; an invalid call launches nothing.  Calls on different
 *    streams with disjoint buffers and workspaces are independent.  Calls
 *    that share a workspace must be ordered (same stream).
 *  - Device pointers must be 16-byte aligned (bf16/fp32 matrices) or 4-byte
 *    aligned (int32 vectors, fp32 score vectors).
 *  - Errors: every call returns spts_status.  Nothing is thrown across the
 *    ABI.  spts_last_error() returns a message for the calling thread's last
 *    failure.  Kernels whose pipelines wait on barriers give up after a
 *    bounded time and raise a flag in the workspace status word instead of
 *    hanging; spts_check_device_status() reads it.
 */
#ifndef SPTS_H
#define SPTS_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define SPTS_API __attribute__((visibility("default")))
#else
#define SPTS_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

/* Same type as cudaStream_t; NULL is the legacy default stream. */
typedef struct CUstream_st *spts_stream;

typedef enum {
  SPTS_OK = 0,
  SPTS_ERR_INVALID = 1,      /* null pointer, misalignment, bad enum or value  */
  SPTS_ERR_SHAPE = 2,        /* inconsistent or out-of-range sizes             */
  SPTS_ERR_UNSUPPORTED = 3,  /* valid but not implemented (e.g. bf16 with d=64)*/
  SPTS_ERR_CUDA = 4,         /* a CUDA runtime/driver call failed              */
  SPTS_ERR_TIMEOUT = 5,      /* a device-side bounded wait gave up             */
  SPTS_ERR_WORKSPACE = 6     /* ws null/misaligned or ws_bytes too small       */
} spts_status;

typedef enum { SPTS_F32 = 0, SPTS_BF16 = 1 } spts_dtype;

/* Score fusion of Table D: f = s (NONE); f = w_a*s/max(s) + w_b*c/max(c)
 * (MAXNORM_ADD, each max over all Nc entries, a term with max 0 adds 0);
 * f = s*c (MULTIPLY, the criterion C*S of Table 6);
 * f = w_a*(s - mean s)/std s + w_b*(c - mean c)/std c (STD_ADD: population
 * mean and standard deviation over all Nc entries, computed in fp64 and
 * rounded to fp32; a term with std 0 adds 0).  All in fp32 with one rounding
 * per operation.  Sequential Select is spts_select_sequential. */
typedef enum {
  SPTS_FUSE_NONE = 0,
  SPTS_FUSE_MAXNORM_ADD = 1,
  SPTS_FUSE_MULTIPLY = 2,
  SPTS_FUSE_STD_ADD = 3,
  SPTS_FUSE_SEQUENTIAL = 4 /* layer descriptor only: see spts_layer_desc.seq_pool */
} spts_fuse;

/* Attention geometry.  scale <= 0 means 1/sqrt(d).
 * Supported: F32 with d in {64, 128}; BF16 with d = 128 and Hq/Hkv in {1,2,4,8}. */
typedef struct {
  spts_dtype dtype;
  int Hq;
  int Hkv;
  int d;
  float scale;
} spts_attn_desc;

/* ---------------------------------------------------------------------- */
/* Library information and status                                         */
/* ---------------------------------------------------------------------- */

/* Version string of the library ("MAJOR.MINOR.PATCH"). */
SPTS_API const char *spts_version(void);

/* Copies the calling thread's last error message (NUL-terminated, possibly
 * truncated) into buf; returns the full message length. */
SPTS_API size_t spts_last_error(char *buf, size_t len);

/* Synchronizes `stream`, then reads and clears the device status word at the
 * start of `ws`.  Returns SPTS_OK, SPTS_ERR_TIMEOUT (a bounded wait gave up),
 * SPTS_ERR_INVALID (a kernel met an out-of-range index) or SPTS_ERR_CUDA. */
SPTS_API spts_status spts_check_device_status(void *ws, spts_stream stream);

/* Testing hook: limit (ns) of every bounded device wait launched after the
 * call (default 2 s).  0 makes any wait that is not already satisfied give up
 * at once, so tests can drive the timeout path without a real hang. */
SPTS_API void spts_debug_set_wait_limit_ns(uint64_t ns);
SPTS_API uint64_t spts_debug_get_wait_limit_ns(void);

/* Number of kernels this library has launched in the process so far (all
 * devices, all threads); a measurement aid. */
SPTS_API uint64_t spts_launch_count(void);

/* Testing hook: y[i] = the exp2 that the reduced-attention softmax kernel
 * evaluates on the FMA pipe for part of each row (range reduction to
 * 2^round(x) * 2^f, a degree-3 polynomial in f with p(0) = 1, relative error
 * <= 1.02e-4 for -126 <= x <= 0; exactly 0 for x <= -127 and -inf), on
 * device arrays x, y [n] fp32. */
SPTS_API spts_status spts_debug_exp2_poly(const float *x, int64_t n, float *y, spts_stream stream);

/* ---------------------------------------------------------------------- */
/* The six calls of the hot path                                          */
/* ---------------------------------------------------------------------- */

/* Partial Attention Probing (Fig. 2(a); probe length P as in Table C).
 * For every query head h and probe p, a causal softmax over the keys with
 * pos_j <= probe_pos[p] of scale * q[p,h] . k[j, h/(Hq/Hkv)]; the score of key
 * j is the sum of its weights over all heads and probes, so sum_j s_j = P*Hq.
 *   q_probe      [P, Hq, d] (dtype of a), the probe queries after RoPE
 *   probe_pos    [P] int32 ascending, positions of the probes
 *   k            [Nc, Hkv, d] (dtype of a), keys after RoPE
 *   key_pos      [Nc] int32 ascending
 *   scores       [Nc] fp32 out
 *   group_scores [Hkv, Nc] fp32 out, or NULL: per-KV-head partial sums
 * Limits: 1 <= P <= 128, Nc >= 1, P <= Nc.  Every probe must see >= 1 key. */
SPTS_API spts_status spts_probe_scores(const spts_attn_desc *a, const void *q_probe, const int32_t *probe_pos,
                              int P, const void *k, const int32_t *key_pos, int64_t Nc, float *scores,
                              float *group_scores, void *ws, size_t ws_bytes, spts_stream stream);
SPTS_API size_t spts_probe_scores_workspace(const spts_attn_desc *a, int P, int64_t Nc);

/* Low-rank Transformation Probing (Fig. 2(b), Table 6, Table A).
 * scores[i] = || (x_i A^T) B^T ||_2 with the rank-r intermediate kept in bf16.
 *   x [Nc, D] bf16 (the FFN input, i.e. already normalized), A [r, D] bf16,
 *   B [Dout, r] bf16, scores [Nc] fp32 out.
 * Evaluated as sqrt(t G t^T), t = bf16(x_i A^T), with the Gram matrix
 * G = B^T B built on each call in the workspace (2 * r^2 bf16 + 8 * r^2 fp32):
 * the same value up to rounding, at r x r instead of r x Dout per row.
 * Limits: dt = SPTS_BF16; D % 64 == 0; r % 64 == 0, 64 <= r <= 256;
 * Dout % 256 == 0. */
SPTS_API spts_status spts_ltp_scores(spts_dtype dt, const void *x, int64_t Nc, int D, const void *A, int r,
                            const void *B, int Dout, float *scores, void *ws, size_t ws_bytes,
                            spts_stream stream);
SPTS_API size_t spts_ltp_scores_workspace(int64_t Nc, int D, int r, int Dout);

/* Top-rho channel saliency of the same proxy (Table E with the D_low proxy
 * of Table A): scores[i] = sum of the top_m largest |y_ij| of
 * y_i = (x_i A^T) B^T over its Dout = D_low channels (top_m = ceil(rho *
 * D_low)); ties at the threshold count as often as needed to make top_m.
 * Same operands and layouts as spts_ltp_scores.
 * Limits: dt = SPTS_BF16; D % 64 == 0; r % 64 == 0, 64 <= r <= 256;
 * Dout in {256, 512}; 1 <= top_m <= Dout. */
SPTS_API spts_status spts_ltp_topm_scores(spts_dtype dt, const void *x, int64_t Nc, int D, const void *A, int r,
                                          const void *B, int Dout, int top_m, float *scores, void *ws,
                                          size_t ws_bytes, spts_stream stream);
SPTS_API size_t spts_ltp_topm_scores_workspace(int64_t Nc, int D, int r, int Dout);

/* Token selection (Fig. 2(a)/(b): the informative tokens).
 * The last force_tail candidates are always kept; the other k - force_tail
 * are the largest fused scores among the first Nc - force_tail, equal scores
 * going to the lower index (-0 counts as +0).  The fused score is computed in
 * fp32 with one rounding per operation in the order of spts_fuse.
 *   s_a [Nc] fp32, s_b [Nc] fp32 (NULL allowed when mode == NONE)
 *   idx_out       [k] int32 out, ascending
 *   fused_out     [Nc] fp32 out or NULL
 *   kth_score_out device fp32 scalar out or NULL: fused score of the last
 *                 non-forced pick (NaN when k == force_tail)
 * Limits: 0 <= force_tail <= k <= Nc < 2^31; scores must be finite. */
SPTS_API spts_status spts_select_topk(const float *s_a, const float *s_b, spts_fuse mode, float w_a, float w_b,
                             int64_t Nc, int64_t k, int64_t force_tail, int32_t *idx_out,
                             float *fused_out, float *kth_score_out, void *ws, size_t ws_bytes,
                             spts_stream stream);
SPTS_API size_t spts_select_topk_workspace(int64_t Nc);

/* Reduced attention (Fig. 2(a): the informative tokens attend).  For each
 * selected query i and head h: softmax over every candidate key j with
 * key_pos[j] <= q_pos[i] of scale * q . k_j, applied to v_j.
 *   q_sel [k, Hq, d], q_pos [k] int32 ascending, kk / v [Nc, Hkv, d],
 *   key_pos [Nc] int32 ascending, o_sel [k, Hq, d] out (dtype of a).
 * Every query must see >= 1 key (rows that see none are written as 0). */
SPTS_API spts_status spts_reduced_attention(const spts_attn_desc *a, const void *q_sel, const int32_t *q_pos,
                                   int64_t k, const void *kk, const void *v, const int32_t *key_pos,
                                   int64_t Nc, void *o_sel, void *ws, size_t ws_bytes, spts_stream stream);
SPTS_API size_t spts_reduced_attention_workspace(const spts_attn_desc *a, int64_t k, int64_t Nc);

/* Reduced FFN (Fig. 2(b): reduced feed-forward on the selected rows).
 * For i in idx: h[i] += W_down (silu(W_gate x_i) * (W_up x_i)) with
 * x_i = RMSNorm(h[i]) * norm_w (eps), x and the activation stored in bf16.
 * Rows not in idx are not touched.
 *   h [Nc, D] fp32 residual stream, in/out; idx [k] int32 ascending, unique
 *   norm_w [D] bf16; w_gate, w_up [F, D] bf16; w_down [D, F] bf16.
 * Limits: dt = SPTS_BF16; D % 256 == 0; F % 128 == 0. */
SPTS_API spts_status spts_reduced_ffn(spts_dtype dt, float *h, int64_t Nc, int D, const int32_t *idx, int64_t k,
                             const void *norm_w, float eps, const void *w_gate, const void *w_up,
                             const void *w_down, int F, void *ws, size_t ws_bytes, spts_stream stream);
SPTS_API size_t spts_reduced_ffn_workspace(int64_t k, int D, int F);

/* Multi-Stage Delayed Pruning stage boundary (Fig. 2(c), Fig. A).
 * Keeps the top k_keep candidates by `scores` (selection rule of
 * spts_select_topk with mode NONE), in ascending order, and compacts the
 * hidden rows and positions:  h_out[t] = h_in[kept[t]], pos_out[t] =
 * pos_in[kept[t]].
 *   scores [Nc] fp32; h_in [Nc, D] fp32; pos_in [Nc] int32;
 *   h_out [k_keep, D] fp32 out (must not overlap h_in); pos_out [k_keep] out;
 *   kept_idx [k_keep] int32 out or NULL. */
SPTS_API spts_status spts_stage_prune(const float *scores, int64_t Nc, int64_t k_keep, int64_t force_tail,
                             const float *h_in, const int32_t *pos_in, int D, float *h_out,
                             int32_t *pos_out, int32_t *kept_idx, void *ws, size_t ws_bytes,
                             spts_stream stream);
SPTS_API size_t spts_stage_prune_workspace(int64_t Nc);

/* Allocation-free variant of spts_stage_prune.  The paper has no
 * counterpart; this exists for callers that cannot allocate device memory
 * when they call in (a plugin inside a host framework that reserved the GPU's
 * memory up front and forbids further cudaMalloc, or a latency-critical loop
 * that cannot take cudaMalloc's implicit synchronisation).  Same arguments
 * and results as spts_stage_prune, without the workspace: when kept_idx is
 * NULL the kept indices go to a fixed device array inside the library
 * (SPTS_NOALLOC_MAX_NC int32, 1 MiB, held by every GPU that loads the library
 * until the process exits).
 *  - Nc > SPTS_NOALLOC_MAX_NC returns SPTS_ERR_SHAPE.
 *  - Calls nothing that allocates (no cudaMalloc/cudaFree).  The first call
 *    on each device looks up the array's device address
 *    (cudaGetSymbolAddress) with that device current; make that first call
 *    before any stream capture.
 *  - CUDA loads device code lazily (the default module loading mode): the
 *    first call on a device loads the code that holds the array and the
 *    kernels it launches, which does take device memory.  A call with
 *    Nc == 0 (every pointer may be NULL) is the set-up form: it only does
 *    that per-device work on the current device and returns SPTS_OK.  A
 *    caller that reserves the GPU's memory makes it once per device first;
 *    after it, calls take no device memory at all.
 *  - Every call shares the one array, which keeps the last call's contents:
 *    calls that may overlap on the GPU (different streams, or different host
 *    threads on one device) race on it and must be serialised by the caller.
 *  - Device-side checks (non-finite scores) are not reported by this variant. */
#define SPTS_NOALLOC_MAX_NC 262144
SPTS_API spts_status spts_stage_prune_noalloc(const float *scores, int64_t Nc, int64_t k_keep, int64_t force_tail,
                                              const float *h_in, const int32_t *pos_in, int D, float *h_out,
                                              int32_t *pos_out, int32_t *kept_idx, spts_stream stream);

/* ---------------------------------------------------------------------- */
/* Supporting calls used to compose the layer                             */
/* ---------------------------------------------------------------------- */

/* y[i] = bf16(x[rows[i]] / sqrt(mean(x[rows[i]]^2) + eps) * w), i < m.
 * x [*, D] fp32 (row stride D); rows [m] int32 or NULL (identity);
 * w [D] bf16 or NULL (ones); y [m, D] bf16.  D % 8 == 0. */
SPTS_API spts_status spts_rmsnorm_rows(const float *x, const int32_t *rows, int64_t m, int D, const void *w,
                              float eps, void *y, spts_stream stream);

/* In-place rotate-half RoPE of x [m, H, d] bf16 at positions pos [m] int32:
 * pair (i, i+d/2) turns by pos * theta^(-2i/d).  d % 2 == 0, d <= 256. */
SPTS_API spts_status spts_rope(void *x, int64_t m, int H, int d, const int32_t *pos, double theta,
                      spts_stream stream);

/* Row gather: dst[i] = src[rows[i]] for i < m; rows of `row_bytes` bytes
 * (a multiple of 16).  Out-of-range rows set the INVALID flag of ws (if ws is
 * not NULL) and are skipped. */
SPTS_API spts_status spts_gather_rows(const void *src, int64_t n_src, const int32_t *rows, int64_t m,
                             int64_t row_bytes, void *dst, void *ws, spts_stream stream);

/* Epilogues of spts_linear. */
typedef enum {
  SPTS_EPI_STORE = 0,       /* C[m, n] = bf16(acc)                                      */
  SPTS_EPI_ROPE = 1,        /* C = bf16(RoPE(acc)) per 128-wide head at row_pos[m]      */
  SPTS_EPI_SWIGLU = 2,      /* C[m, n] = bf16(silu(A W_gate^T) * (A W_up^T)), W2 = W_up */
  SPTS_EPI_SCATTER_ADD = 3  /* H[rows[m], n] += acc, H fp32 (rows unique)               */
} spts_epilogue;

/* bf16 tensor-core GEMM acc = A W^T on tcgen05 (fp32 accumulation) with a
 * fused epilogue.  A [M, K] bf16; W [N, K] bf16 (W2 [N, K] for SWIGLU);
 * out: bf16 [M, N] (STORE/ROPE/SWIGLU) or fp32 [*, N] (SCATTER_ADD, rows[]
 * indexing the output rows).  row_pos [M] int32 for ROPE (theta as given).
 * Limits: K % 64 == 0; N % 256 == 0 (N % 128 for SWIGLU, ROPE needs N % 128). */
SPTS_API spts_status spts_linear(const void *A, int64_t M, int K, const void *W, const void *W2, int N,
                        spts_epilogue epi, void *out, const int32_t *rows, const int32_t *row_pos,
                        double theta, void *ws, size_t ws_bytes, spts_stream stream);
SPTS_API size_t spts_linear_workspace(void);

/* Adds shift * unit(mean of the group's probe queries) to K[rows[t], g] for
 * every KV head g (K bf16 [Nc, Hkv, d], q_probe bf16 [P, Hq, d]); rows must
 * be distinct.  This is a synthetic-workload step that plants salient keys;
 * it is not part of SPTS. */
SPTS_API spts_status spts_inject_salience(void *k, int64_t Nc, const void *q_probe, int P, int Hq, int Hkv, int d,
                                 const int32_t *rows, int64_t n_rows, float shift, spts_stream stream);

/* Sequential Select of Table D (reading: the pages name it only): the pool
 * = the top-k_pool candidates by s_a (the last force_tail always kept, ties
 * to the lower index), then the top-k of the pool by s_b under the same
 * rules; idx_out [k] holds candidate indices, ascending.
 * Limits: 0 <= force_tail <= k <= k_pool <= Nc < 2^31. */
SPTS_API spts_status spts_select_sequential(const float *s_a, const float *s_b, int64_t Nc, int64_t k_pool,
                                            int64_t k, int64_t force_tail, int32_t *idx_out, void *ws,
                                            size_t ws_bytes, spts_stream stream);
SPTS_API size_t spts_select_sequential_workspace(int64_t Nc);

/* ---------------------------------------------------------------------- */
/* The composed layer (probe -> reduced MHA -> LTP -> reduced FFN)         */
/* ---------------------------------------------------------------------- */

typedef struct {
  int D, Hq, Hkv, d, F, r;  /* F == 0: attention-only layer                */
  int P;                    /* probe rows = the last P candidates           */
  int64_t k;                /* active rows of each selection                */
  spts_fuse fuse;           /* fusion of the FFN selection                  */
  float w_a, w_b;           /* fusion weights (MAXNORM_ADD)                 */
  float eps;                /* RMSNorm eps                                  */
  double theta;             /* RoPE base                                    */
  /* synthetic salient keys (not part of SPTS; n_salient = 0 to disable)    */
  const int32_t *salient_rows;
  int64_t n_salient;
  float salient_shift;
  /* LTP proxy output channels: B is [ltp_dout, r] (the channel-reduced
   * proxy D_low of Table A); 0 means D.                                    */
  int ltp_dout;
  /* 1: the reduced attention uses the keys and values of the active rows
   * only (K and V of idx_attn), the KV-cache reading behind Table 5; V is
   * then projected for the active rows only.  0: all Nc candidate keys.   */
  int kv_active_only;
  /* > 0: the LTP score is the top-rho channel saliency, the sum of the
   * ltp_top_m largest |y| (needs ltp_dout in {256, 512}); 0: ||y||_2.      */
  int ltp_top_m;
  /* fuse == SPTS_FUSE_SEQUENTIAL: the pool of the FFN selection (top
   * seq_pool rows by the probe score, then the top k of them by the LTP
   * score); 0 means min(Nc, 2k).  The layer's fused output f is then c.   */
  int64_t seq_pool;
} spts_layer_desc;

typedef struct {
  const void *w_q, *w_k, *w_v, *w_o;       /* [Hq*d,D] [Hkv*d,D] [Hkv*d,D] [D,Hq*d] */
  const void *w_gate, *w_up, *w_down;      /* [F,D] [F,D] [D,F]                    */
  const void *ltp_a, *ltp_b;               /* [r,D] [D,r]                          */
  const void *norm_attn, *norm_ffn;        /* [D] bf16 or NULL (ones)              */
} spts_layer_weights;

/* Optional outputs of one layer (any may be NULL). */
typedef struct {
  float *s;            /* [Nc] probe scores                      */
  float *c;            /* [Nc] LTP scores                        */
  float *f;            /* [Nc] fused FFN-selection scores        */
  int32_t *idx_attn;   /* [k] rows that ran reduced attention    */
  int32_t *idx_ffn;    /* [k] rows that ran the reduced FFN      */
  void *o_sel;         /* [k, Hq, d] bf16 reduced-attention out  */
  float *h_attn;       /* [Nc, D] residual after attention       */
  void *k;             /* [Nc, Hkv, d] bf16 keys after RoPE (and the synthetic salience): the probe's keys */
  void *q_probe;       /* [P, Hq, d] bf16 probe queries after RoPE */
  /* NULL, or an array of SPTS_LAYER_STAGE_EVENTS cudaEvent_t handles
   * created by the caller, any of which may be NULL (not recorded); event i
   * is recorded on the stream after stage i (see below), event 0 before the
   * first kernel.  When any of events 1..7 is given, every kernel runs on
   * the caller's stream so that stage times add up; otherwise the probe-Q
   * and V projections still run on the library's side stream (event 8
   * follows the join with it).  A measurement aid. */
  void *const *stage_events;
} spts_layer_outputs;

/* Stages of spts_layer_forward, in launch order (event i follows stage i):
 *  1 RMSNorm   2 K proj+RoPE   3 V proj   4 probe Q proj (+salience)
 *  5 PAP probe scores   6 select (MHA)   7 gathers   8 Q proj+RoPE
 *  9 reduced attention   10 O proj + scatter-add   11 RMSNorm
 * 12 LTP score   13 fuse + select (FFN) + gather   14 gate/up + SwiGLU
 * 15 down proj + scatter-add */
#define SPTS_LAYER_STAGE_EVENTS 16

/* One SPTS layer in place on h [Nc, D] fp32 with positions pos [Nc].
 * Order: RMSNorm; K/V (+RoPE) for all rows and Q for the last P rows;
 * probe scores; select; Q for the selected rows; reduced attention; O
 * projection added into the selected rows; then (F > 0) RMSNorm, LTP score,
 * fusion, select, reduced FFN.  Limits: those of the calls it makes. */
SPTS_API spts_status spts_layer_forward(const spts_layer_desc *L, const spts_layer_weights *W, float *h,
                               const int32_t *pos, int64_t Nc, const spts_layer_outputs *out, void *ws,
                               size_t ws_bytes, spts_stream stream);
SPTS_API size_t spts_layer_forward_workspace(const spts_layer_desc *L, int64_t Nc);

/* spts_layer_forward on a residual stream held in bf16 at the boundary:
 * h [Nc, D] bf16, in place.  The layer runs on an fp32 copy of h in the
 * workspace (the same kernels and results as spts_layer_forward on
 * float(h)); then the rows it changed -- its attention rows and FFN rows,
 * every row when L->k == Nc -- are rounded to bf16 (nearest even) back into
 * h, and the rows it skipped keep their input bits.  This halves what a
 * caller moves across PCIe when h lives in host memory.  `out` as for
 * spts_layer_forward (h_attn, when given, is the fp32 residual after
 * attention).  Limits: those of spts_layer_forward; D % 8 == 0. */
SPTS_API spts_status spts_layer_forward_bf16io(const spts_layer_desc *L, const spts_layer_weights *W, void *h,
                                               const int32_t *pos, int64_t Nc, const spts_layer_outputs *out,
                                               void *ws, size_t ws_bytes, spts_stream stream);
SPTS_API size_t spts_layer_forward_bf16io_workspace(const spts_layer_desc *L, int64_t Nc);

/* Multi-Stage Delayed Pruning over a stack of layers (SPTS, Fig. 2(c),
 * Fig. A, Table B).  n_stages stages of layers_per_stage layers each
 * (n_layers = n_stages * layers_per_stage).  Stage s starts with candidate
 * set C_s (C_1 = all N rows); every layer of the stage runs spts_layer_forward
 * on C_s with k = stage_k[s] active rows; at the end of the stage C_{s+1} =
 * the top stage_k[s] rows of C_s by the fused FFN-selection score of the
 * stage's last layer (last P rows kept), compacted in ascending order.
 *   L           layer geometry (L->k is ignored; stage_k gives each stage's k)
 *   W           [n_layers] weights, one entry per layer
 *   stage_k     [n_stages] host array, P <= stage_k[s] <= size of C_s
 *   h           [N, D] fp32 in/out: on return rows [0, stage_k[last]) hold
 *               the final candidates' hidden states (other rows: scratch)
 *   pos         [N] int32 in/out, likewise compacted
 *   stage_pos   nullable, [sum_s stage_k[s]] int32 out: positions of C_{s+1}
 *               for every stage, concatenated
 * Synthetic salience (L->n_salient) is not applied in this call. */
SPTS_API spts_status spts_msdp_forward(const spts_layer_desc *L, const spts_layer_weights *W, int n_layers,
                                       int layers_per_stage, const int64_t *stage_k, int n_stages, float *h,
                                       int32_t *pos, int64_t N, int32_t *stage_pos, void *ws, size_t ws_bytes,
                                       spts_stream stream);
SPTS_API size_t spts_msdp_forward_workspace(const spts_layer_desc *L, int64_t N);

/* A layer schedule of Table B (reading): layers [0, first_skip) are full
 * layers over every token; stage st covers the layers up to stage_ends[st]
 * and each of its layers selects k = min(budgets[st], |C|) active rows from
 * the stage's candidates C; at a stage end the candidates are pruned to the
 * top budgets[st] (after the last stage: the top after_last) by that
 * layer's fused score, the last P always kept; the layers after the last
 * stage are full layers over the survivors.  h [N, D] fp32 and pos [N] are
 * compacted in place: *n_out rows remain.  sel_pos (nullable, sel_cap
 * entries) receives, layer after layer, the positions of every skipping
 * layer's attention set; sel_len [n_layers] their counts (0 for full
 * layers).  W holds n_layers weight sets; F must be > 0; salience is off. */
SPTS_API spts_status spts_schedule_forward(const spts_layer_desc *L, const spts_layer_weights *W, int n_layers,
                                          int first_skip, const int *stage_ends, const int64_t *budgets,
                                          int n_stages, int64_t after_last, float *h, int32_t *pos, int64_t N,
                                          int64_t *n_out, int32_t *sel_pos, int64_t sel_cap, int64_t *sel_len,
                                          void *ws, size_t ws_bytes, spts_stream stream);
SPTS_API size_t spts_schedule_forward_workspace(const spts_layer_desc *L, int64_t N);

#ifdef __cplusplus
}
#endif
#endif /* SPTS_H */
