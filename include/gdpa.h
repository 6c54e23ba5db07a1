/*
 * gdpa.h -- C ABI of libgdpa, Generalized Dot-Product Attention on B200.
 *
 * GDPA (Kunlun paper review, §2.3 "GDPA" and Fig. 2; Kunlun Breakdown, "The
 * Core Architecture and Mechanics") recasts the personalised FFN as
 * attention: a sample's jagged behaviour sequence is the query, and weights
 * generated from the sample's context are the keys and values.  Per sample b
 * and head h it computes
 *
 *     O = phi(scale * Q K^T + beta) V
 *
 * where phi is an element-wise activation (SiLU, reproducing act(X W1) W2, or
 * GELU, the element-wise example of the Kunlun paper review, §2.3 "GDPA") or
 * a row softmax (pooling, cross-attention and sliding-window self-attention),
 * and beta is an optional per-key additive bias, or the gate log sigmoid(G)
 * of the Kunlun reproduction notes ("Core equations").  The optional band
 * (window_left, window_right) is the sliding window of the Kunlun paper
 * review, §2.5: key j is visible to query i iff
 *     (window_left < 0 || j >= i - window_left) &&
 *     (window_right < 0 || j <= i + window_right),
 * with i and j counted from the start of their own sample.
 *
 * Layouts (all tensors are DEVICE pointers, row-major, no padding):
 *   q, o, dout, dq        bf16 [total_q ][H][D]
 *   k, v, dk, dv          bf16 [total_kv][H][D]
 *   bias (or gate G), dbias  fp32 [H][total_kv]   (broadcast over queries)
 *   lse                   fp32 [H][total_q]       natural-log log-sum-exp
 *   q_offsets, kv_offsets int32 [B+1], offsets[0] = 0, non-decreasing,
 *                         offsets[B] = total.  Sample b owns rows
 *                         [offsets[b], offsets[b+1]).
 * q, k, v, o, dout, dq, dk, dv and the workspace must be 16-byte aligned.
 * D must be 32, 64 or 128.  B <= 16384.
 *
 * Ownership: the caller allocates and frees everything (inputs, outputs and
 * the workspace).  The library never allocates, frees or synchronises,
 * except gdpa_get_device_status and gdpa_forward_no_alloc_status, which
 * synchronise the stream they are given.
 * All launches are asynchronous on `stream` (a cudaStream_t; NULL = legacy
 * default stream).  Calls that share one workspace must not overlap.
 *
 * Errors: argument errors are reported at the call (GDPA_ERR_*), before
 * anything is launched.  Launch failures return GDPA_ERR_CUDA.  Errors found
 * by the device (a bounded wait that ran out, an offset beyond the declared
 * maximum length, offsets that decrease or reach past total_q / total_kv) are
 * recorded in the workspace and read back with gdpa_get_device_status; the
 * offending sample is skipped, so its output rows are not written.
 */
#ifndef GDPA_H_
#define GDPA_H_

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define GDPA_API __attribute__((visibility("default")))
#else
#define GDPA_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st* gdpa_stream_t; /* same type as cudaStream_t */

typedef enum {
  GDPA_OK = 0,
  GDPA_ERR_INVALID_ARG = 1,  /* null/unaligned pointer, bad size or offset shape */
  GDPA_ERR_UNSUPPORTED = 2,  /* D, phi, bias kind, batch size or device not supported */
  GDPA_ERR_WORKSPACE = 3,    /* workspace missing or smaller than gdpa_workspace_size */
  GDPA_ERR_CUDA = 4,         /* a CUDA runtime or driver call failed */
  GDPA_ERR_TIMEOUT = 5,      /* device: a bounded wait inside a kernel ran out */
  GDPA_ERR_DEVICE_CHECK = 6  /* device: a sample is longer than max_seqlen_q / _kv, or
                                its offsets decrease or reach past total_q / total_kv;
                                such a sample is skipped and its output rows are left
                                unwritten */
} gdpa_status_t;

enum { GDPA_PHI_SILU = 0, GDPA_PHI_SOFTMAX = 1, GDPA_PHI_IDENTITY = 2, GDPA_PHI_GELU = 3 };
enum { GDPA_BIAS_NONE = 0, GDPA_BIAS_ADD = 1, GDPA_BIAS_GATE = 2 };

typedef struct {
  int B;              /* samples */
  int H;              /* heads */
  int D;              /* head dim: 32, 64 or 128 */
  int64_t total_q;    /* q_offsets[B]  (host-known: sizes the TMA descriptors) */
  int64_t total_kv;   /* kv_offsets[B] */
  int max_seqlen_q;   /* upper bound on any sample's query length; 0 = total_q */
  int max_seqlen_kv;  /* upper bound on any sample's key length;   0 = total_kv */
  int phi;            /* GDPA_PHI_* : SiLU x*sigmoid(x), row softmax, identity, or
                         GELU x*Phi(x) (Phi the standard normal distribution) */
  float scale;        /* multiplies QK^T before beta is added (= 1/tau) */
  int window_left;    /* -1 = unbounded */
  int window_right;   /* -1 = unbounded */
  int bias_kind;      /* GDPA_BIAS_*: none, beta = bias, or beta = log sigmoid(bias) */
  int debug_flags;    /* 0 in normal use.  Bit 0 drops one producer arrival so that
                         the bounded-wait path can be tested (returns TIMEOUT);
                         bit 2 selects the in-kernel rotary turn (forward; see
                         rope_q); other bits are reserved and ignored */
  int wait_timeout_us;/* bound on any single in-kernel wait; 0 = 2000000 (2 s) */
  const int32_t* head_phi; /* optional host array of H GDPA_PHI_* values, one per
                         head (H <= 64); NULL = every head uses phi.  Read during
                         the call only.  LSE rows of non-softmax heads are not
                         written. */
  /* Rotary temporal embedding of Q and K (gdpa_rotary_table below): device
   * tables of rotations, [total_q][D/2] for the queries and [total_kv][D/2] for
   * the keys, 16-byte aligned; both NULL = no rotation.  Give both or neither
   * (self-attention passes the same table twice).  The attention then uses
   * turned Q and K (V is not turned); the backward returns dQ and dK with
   * respect to the unturned inputs.  Both calls turn Q and K in one streaming
   * pass into the workspace (which grows by (total_q + total_kv) * H * D * 2
   * bytes) and run the attention kernels on the copies; the backward turns dQ
   * and dK back in place at the end.  debug_flags bit 2 makes the forward turn
   * each Q tile and K block in shared memory inside the attention kernel
   * instead (no copies; measured slower).  The grouped forward accepts the
   * tables per problem (streamed turn only; bit 2 there is
   * GDPA_ERR_UNSUPPORTED). */
  const void* rope_q;
  const void* rope_kv;
} gdpa_params_t;

/* ---- Rotary temporal embedding (Kunlun paper review §2.2: RoPE extended from
 * positions to log-scaled time gaps, with position frequencies theta_i and time
 * frequencies phi_i; the page's formulas were lost, this is the reading used).
 *
 * Token t (0-based within its sample) of a jagged sequence has the gap
 * dt_t = time[t] - time[t-1] to the previous event of its sample (0 for the
 * first token; a negative gap counts as 0) and the scaled gap
 * tau_t = ln(1 + dt_t / time_scale).  Pair i = (2i, 2i+1) of every head vector
 * of that token turns by alpha_{t,i} = t * theta_i + tau_t * phi_i:
 *   x'_2i = x_2i cos(alpha) - x_2i+1 sin(alpha),
 *   x'_2i+1 = x_2i sin(alpha) + x_2i+1 cos(alpha). */
typedef struct {
  int D;               /* head dim: 32, 64 or 128 */
  float time_scale;    /* tau_scale, > 0, in the unit of time[] */
  const float* theta;  /* optional host [D/2] position frequencies; NULL = 10000^(-2i/D) */
  const float* phi;    /* optional host [D/2] time frequencies; NULL = theta */
} gdpa_rotary_params_t;

/* Bytes of a rotation table for `total` tokens: total * D/2 * 4
 * ((cos, sin) of each angle as two fp16 values, cos first). */
GDPA_API size_t gdpa_rotary_table_bytes(int D, int64_t total);

/* Fills table [total][D/2] (device, 16-byte aligned, the caller's) for the
 * jagged sequence given by offsets [B+1] (device int32, as elsewhere) and
 * time [total] (device int64 event times, non-decreasing within a sample for
 * the gaps to mean anything).  The position part t * theta_i is reduced
 * modulo 2 pi without rounding error (positions below 2^24; the default
 * frequencies are taken in fp64), then the cosine and sine are taken in fp32
 * and rounded to fp16.  One table serves every head, the forward and the
 * backward, and every layer that sees the same sequence.  Asynchronous on
 * stream.  Errors (before any launch): GDPA_ERR_UNSUPPORTED for another D;
 * GDPA_ERR_INVALID_ARG for a time scale that is not a positive finite number,
 * a non-finite frequency, B outside [0, 16384], total outside [0, 2^31), or a
 * null or unaligned pointer when B and total are positive; GDPA_ERR_CUDA when
 * the launch fails.  Offsets are trusted (clamped to [0, total] on the
 * device). */
GDPA_API gdpa_status_t gdpa_rotary_table(const gdpa_rotary_params_t* r, int B, int64_t total,
                                         const int32_t* offsets, const int64_t* time,
                                         void* table, gdpa_stream_t stream);

/* y = x turned by the table's angles (inverse = 0) or turned back (inverse
 * != 0: the transpose, which maps dL/dx' to dL/dx), for x, y bf16
 * [total][H][D] (device, 16-byte aligned; y may be x) and a table from
 * gdpa_rotary_table for the same tokens.  A training step can turn Q and K
 * once with this call, pass the turned copies (and no tables) to both
 * gdpa_forward and gdpa_backward, and turn dQ and dK back with inverse = 1:
 * two streaming passes instead of the three that rope_q / rope_kv imply.
 * Asynchronous on stream.  Errors:
 * GDPA_ERR_UNSUPPORTED for another D; GDPA_ERR_INVALID_ARG for H <= 0, total
 * outside [0, 2^31) or a null or unaligned pointer (total > 0);
 * GDPA_ERR_CUDA when the launch fails. */
GDPA_API gdpa_status_t gdpa_rotary_apply(int64_t total, int H, int D, const void* x,
                                         const void* table, void* y, int inverse,
                                         gdpa_stream_t stream);

/* ---- SumKronLinear (Kunlun paper review §2.4: the second stage of
 * Hierarchical Seed Pooling compresses the seed summaries X [B, S, D] to
 * Y [B, T, D] with a rank-k sum of Kronecker products, k (S T + D^2)
 * parameters; the page's formula was lost, this is the reading used):
 *   vec(Y_b) = sum_r (A_r kron W_r^T) vec(X_b),  i.e.  Y_b = sum_r A_r X_b W_r,
 * A_r [T x S], W_r [D x D], no bias.  One fused kernel: Z_b = A X_b on the
 * tensor cores, rounded to bf16 on chip, then Y_b = sum_r Z_b[r] W_r with fp32
 * accumulation; Z never reaches HBM. */
typedef struct {
  int B;               /* samples */
  int S;               /* seeds per sample: 64, 128, 192 or 256 */
  int T;               /* output tokens per sample: 32 or 64 */
  int D;               /* embedding dim: 128, 256 or 384 */
  int k;               /* Kronecker rank: k * T a multiple of 128 */
  int wait_timeout_us; /* bound on any single in-kernel wait; 0 = 2 s */
  int debug_flags;     /* 0 in normal use.  Bit 0 drops one X load in CTA 0 so that
                          the bounded-wait path can be tested (the call's status
                          becomes GDPA_ERR_TIMEOUT); other bits are ignored */
} gdpa_sumkron_params_t;

/* Workspace bytes (the device status block); 0 on invalid parameters. */
GDPA_API size_t gdpa_sumkron_workspace_size(const gdpa_sumkron_params_t* p);

/* y [B][T][D] from x [B][S][D], a [k][T][S] (A_1..A_k) and w [k][D][D]
 * (W_1..W_k), all bf16 row-major device arrays, 16-byte aligned, the
 * caller's.  The workspace's status is cleared on the stream first; read it
 * with gdpa_get_device_status (GDPA_ERR_TIMEOUT if a bounded wait ran out).
 * Asynchronous on stream.  Errors (before any launch): GDPA_ERR_UNSUPPORTED
 * for shapes outside the limits above; GDPA_ERR_INVALID_ARG for negative or
 * zero sizes, or a null or unaligned pointer; GDPA_ERR_WORKSPACE for a
 * workspace below gdpa_sumkron_workspace_size; GDPA_ERR_CUDA when a CUDA call
 * fails. */
GDPA_API gdpa_status_t gdpa_sumkron_forward(const gdpa_sumkron_params_t* p, const void* x,
                                            const void* a, const void* w, void* y,
                                            void* workspace, size_t workspace_bytes,
                                            gdpa_stream_t stream);

/* Workspace bytes of gdpa_sumkron_backward: the status block, two bf16
 * intermediates of B x k T x D elements each, and fp32 partial sums of dA
 * (min(B, 64) x k T x S) and dW (min(B, 8) x k D x D).  0 on invalid
 * parameters. */
GDPA_API size_t gdpa_sumkron_backward_workspace_size(const gdpa_sumkron_params_t* p);

/* Gradients of y = SumKronLinear(x; a, w) (Kunlun paper review §2.4; the map
 * of gdpa_sumkron_forward, Y_b = sum_r A_r X_b W_r) for the upstream gradient
 * dy [B][T][D]:
 *   dx [B][S][D] = sum_r A_r^T dY_b W_r^T
 *   da [k][T][S] = sum_b (dY_b W_r^T) X_b^T        (one T x S block per r)
 *   dw [k][D][D] = sum_b (A_r X_b)^T dY_b          (one D x D block per r)
 * All bf16 row-major device arrays, 16-byte aligned, the caller's; fp32
 * accumulation (the sums over samples are split into fp32 partials in the
 * workspace and added in fp32).  x, a, w are the forward's inputs.  Same
 * parameter limits as the forward; B = 0 gives zero da and
 * dw.  The workspace's status is cleared on the stream first (read it with
 * gdpa_get_device_status; GDPA_ERR_TIMEOUT if a bounded wait ran out).
 * Asynchronous on stream.  Errors (before any launch): as
 * gdpa_sumkron_forward, with GDPA_ERR_WORKSPACE below
 * gdpa_sumkron_backward_workspace_size. */
GDPA_API gdpa_status_t gdpa_sumkron_backward(const gdpa_sumkron_params_t* p, const void* x,
                                             const void* a, const void* w, const void* dy,
                                             void* dx, void* da, void* dw, void* workspace,
                                             size_t workspace_bytes, gdpa_stream_t stream);

/* Bytes of device workspace gdpa_forward (backward = 0) or gdpa_backward
 * (backward = 1) needs for these parameters.  0 on invalid parameters. */
GDPA_API size_t gdpa_workspace_size(const gdpa_params_t* p, int backward);

/* Forward: o (and lse when phi = softmax; lse may be NULL otherwise or when not
 * wanted) from q, k, v.  bias must be non-NULL iff bias_kind != NONE.
 * Rows with no visible key get O = 0 and LSE = -inf.
 * Defined by: Kunlun paper review §2.3 (GDPA, Fig. 2) and §2.5 (window);
 * Kunlun reproduction notes, "Core equations" (softmax with log-sigmoid gate). */
GDPA_API gdpa_status_t gdpa_forward(const gdpa_params_t* p, const void* q, const void* k,
                           const void* v, const int32_t* q_offsets,
                           const int32_t* kv_offsets, const float* bias, void* o,
                           float* lse, void* workspace, size_t workspace_bytes,
                           gdpa_stream_t stream);

/* Backward: dq, dk, dv (bf16) from the forward's inputs, its output o, the
 * upstream gradient dout, and lse (softmax only; o and lse are unused for the
 * element-wise activations and may be NULL there).  Every row of dq, dk, dv is
 * written (zeros where nothing flows).  dbias (fp32 [H][total_kv], optional,
 * only with a bias or gate, else GDPA_ERR_INVALID_ARG) receives the gradient of
 * the bias input: the library zeroes it on the stream, then every key's sum
 * over its sample's queries is added (keys no query sees stay 0).  The
 * gradient of the definition above:
 *   dV_j = sum_i p_ij dO_i,  dP_ij = dO_i . V_j,
 *   dS_ij = p_ij (dP_ij - dO_i . O_i) (softmax)  or  dP_ij * phi'(s_ij),
 *   dQ_i = scale sum_j dS_ij K_j,  dK_j = scale sum_i dS_ij Q_i,
 *   dbias_hj = sum_i dS_ij (additive bias),
 *   dG_hj = sum_i dS_ij (1 - sigma(G_hj)) (gate, beta = log sigma(G); the gate
 *   gradient Kunlun reproduction notes, "Core equations", leaves implied).
 * The pages ask that the fused backward avoid materialising large
 * intermediates (Kunlun paper review §2.3, Fig. 2 discussion). */
GDPA_API gdpa_status_t gdpa_backward(const gdpa_params_t* p, const void* q, const void* k,
                            const void* v, const void* o, const void* dout,
                            const float* lse, const int32_t* q_offsets,
                            const int32_t* kv_offsets, const float* bias, void* dq,
                            void* dk, void* dv, float* dbias, void* workspace,
                            size_t workspace_bytes, gdpa_stream_t stream);

/* Grouped forward: several independent GDPA problems in one call, each with
 * its own shapes (B, H, D), activation(s), scale, band, bias and tensors --
 * the many small problems of event-level personalisation, where each event
 * type has its own model width, head count and window (Kunlun paper review,
 * §2.5, "Event-level Personalization").  Problems that share the head dim,
 * the key-block size (64 keys when no sample has more than 64, else 128) and
 * softmax-or-not run in ONE persistent launch whose CTAs take the
 * (problem, sample, head) units of all of them, longest sample first; a call
 * makes one such launch per distinct combination.  Each problem's outputs
 * equal those of gdpa_forward on it alone.  Limits per launch group: at most
 * 256 problems and 16384 samples in total.  Every problem is validated as by
 * gdpa_forward before anything is launched; the workspace is for the whole
 * call (gdpa_forward_grouped_workspace_size) and gdpa_get_device_status
 * reads its status. */
typedef struct {
  gdpa_params_t params;
  const void* q;                /* [total_q][H][D] bf16 */
  const void* k;                /* [total_kv][H][D] bf16 */
  const void* v;                /* [total_kv][H][D] bf16 */
  const int32_t* q_offsets;     /* [B+1] */
  const int32_t* kv_offsets;    /* [B+1] */
  const float* bias;            /* [H][total_kv] fp32, or NULL (bias_kind NONE) */
  void* o;                      /* [total_q][H][D] bf16 */
  float* lse;                   /* [H][total_q] fp32 or NULL (softmax heads only) */
} gdpa_forward_problem_t;

/* One problem of a grouped backward: the arguments of gdpa_backward. */
typedef struct {
  gdpa_params_t params;
  const void* q;
  const void* k;
  const void* v;
  const void* o;
  const void* dout;
  const float* lse;
  const int32_t* q_offsets;
  const int32_t* kv_offsets;
  const float* bias;
  void* dq;
  void* dk;
  void* dv;
  float* dbias;                 /* optional, as in gdpa_backward */
} gdpa_backward_problem_t;

/* Workspace bytes of gdpa_backward_grouped: a status block, an offsets table
 * and one gdpa_backward workspace per problem; 0 when a problem is invalid or
 * n_problems is outside [1, 4096]. */
GDPA_API size_t gdpa_backward_grouped_workspace_size(const gdpa_backward_problem_t* problems,
                                                     int n_problems);

/* Grouped backward for per-event training (Kunlun paper review §2.5,
 * "Event-level Personalization"): the gradients of several independent GDPA
 * problems in one call, each problem's outputs equal to those of
 * gdpa_backward on it alone.  Every problem is validated as by gdpa_backward
 * before anything is launched.  The problems' launches go onto the stream one
 * problem after another (schedule, delta, backward kernels of each), each
 * with its own part of the workspace; a last kernel gathers their device
 * status into the status block at the workspace start, which
 * gdpa_get_device_status reads (the first error of the first problem that
 * reported one).  Asynchronous on stream. */
GDPA_API gdpa_status_t gdpa_backward_grouped(const gdpa_backward_problem_t* problems,
                                             int n_problems, void* workspace,
                                             size_t workspace_bytes, gdpa_stream_t stream);

/* Workspace bytes of gdpa_forward_grouped for these problems; 0 when they are
 * invalid or exceed the limits above. */
GDPA_API size_t gdpa_forward_grouped_workspace_size(const gdpa_forward_problem_t* problems,
                                                    int n_problems);
GDPA_API gdpa_status_t gdpa_forward_grouped(const gdpa_forward_problem_t* problems,
                                            int n_problems, void* workspace,
                                            size_t workspace_bytes, gdpa_stream_t stream);

/* Forward for callers that cannot allocate device memory.  (The Kunlun pages
 * have no counterpart to this entry point; it exists for this library's users.)
 * Some callers have no way to give the library a workspace: a plugin inside a
 * host framework that owns all device memory and exposes no allocator, or a
 * serving process that plans its memory at start-up and must not allocate on
 * the request path.  This call computes exactly what gdpa_forward computes,
 * with the forward's scratch (status, sample order, tile prefix, per-sample
 * descriptors) held in a fixed 393,728-byte array compiled into the library instead of a caller
 * workspace; every GPU that loads the library keeps its own copy until the
 * process exits.  It allocates nothing (no cudaMalloc, cudaFree or
 * allocating library routine).  The caller still passes inputs and outputs.
 * Limits: B <= 16384, the library's own batch limit; beyond it (or if the
 * scratch would not fit) it returns GDPA_ERR_WORKSPACE.  The first call on
 * each device looks up the array's device address (cudaGetSymbolAddress, with
 * that device current) and caches it, so make that first call before any
 * stream capture.  All calls on a device share the one array: calls that
 * overlap on the GPU (on different streams, or from different host threads)
 * race and must be serialised by the caller.  Each call overwrites what it
 * needs, so nothing from an earlier call leaks in.  A bounded wait that runs
 * out, or a sample that fails the device checks (see GDPA_ERR_DEVICE_CHECK),
 * leaves the affected O and LSE rows unwritten while the call still returns
 * GDPA_OK: read the call's device status with gdpa_forward_no_alloc_status.
 * With rotary
 * tables (rope_q / rope_kv) the attention kernel turns Q and K itself (as
 * debug_flags bit 2 selects for gdpa_forward): no turned copies, the same
 * results bit for bit. */
GDPA_API gdpa_status_t gdpa_forward_no_alloc(const gdpa_params_t* p, const void* q,
                                             const void* k, const void* v,
                                             const int32_t* q_offsets,
                                             const int32_t* kv_offsets, const float* bias,
                                             void* o, float* lse, gdpa_stream_t stream);

/* Device status of the last gdpa_forward_no_alloc call on the current device
 * (the status block at the start of the built-in array): GDPA_OK,
 * GDPA_ERR_TIMEOUT or GDPA_ERR_DEVICE_CHECK, as gdpa_get_device_status gives
 * for a workspace.  Synchronises `stream` (the stream of that call) first,
 * then copies the block to the host.  Every no-alloc call on a device clears
 * and rewrites the one block, so read it before the next call.  GDPA_ERR_CUDA
 * if the array's address cannot be looked up or the copy fails. */
GDPA_API gdpa_status_t gdpa_forward_no_alloc_status(gdpa_stream_t stream);

/* The jagged tile schedule the kernels use, exported so it can be checked:
 * query tiles of block_m rows, key blocks of block_n keys (both multiples of
 * 16 in [16, 256]); per sample the cost sum over its tiles of (1 + key blocks
 * the tile may touch under the window); order = samples by descending cost,
 * ties by ascending index; tile_start[p] = query tiles of order[0..p),
 * tile_start[B] = all tiles.  Outputs are device int32 arrays of B+1 and B.
 * ("tile scheduling" over "jagged sequences": Kunlun paper review §2.3.)
 * Costs are clamped to 2^32-1. */
GDPA_API gdpa_status_t gdpa_tile_schedule(const gdpa_params_t* p, int block_m, int block_n,
                                 const int32_t* q_offsets, const int32_t* kv_offsets,
                                 int32_t* tile_start, int32_t* order,
                                 gdpa_stream_t stream);

/* Tile shape (block_m, block_n) the forward kernel uses for these parameters. */
GDPA_API gdpa_status_t gdpa_forward_tile_shape(const gdpa_params_t* p, int* block_m,
                                      int* block_n);

/* Synchronises `stream`, then returns the status the last gdpa_forward /
 * gdpa_backward call on this workspace recorded on the device (GDPA_OK,
 * GDPA_ERR_TIMEOUT or GDPA_ERR_DEVICE_CHECK), or GDPA_ERR_CUDA. */
GDPA_API gdpa_status_t gdpa_get_device_status(const void* workspace, gdpa_stream_t stream);

/* Static English text for a status code. */
GDPA_API const char* gdpa_status_string(gdpa_status_t s);

/* Library version, major * 10000 + minor * 100 + patch. */
GDPA_API int gdpa_version(void);

#ifdef __cplusplus
}
#endif

#endif /* GDPA_H_ */
