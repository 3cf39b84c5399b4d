/*
 * slora.h — C ABI of the contextually sparse LoRA hot path (SparseLoRA) for
 * NVIDIA B200 (sm_100a).
 *
 * Sources of the operations (page title, section):
 *   [ART]  SparseLoRA news article (lsdiaocha.cn, ICML 2025 / arXiv 2506.16500),
 *          sections 1 "dynamic sparsity design", 2 "SVD sparsity estimator",
 *          3 "layer sensitivity" (context/output token split), 6 "compatibility"
 *          (structured sparsity that real GPUs accelerate), 7 "implementation
 *          details" (rank-8 estimator, slicing and compute order).
 *   [ABS]  "SparseLoRA: accelerating LLM fine-tuning with contextual sparsity"
 *          (xinfinite.net forum post), the paper's abstract: a training-free
 *          SVD sparsity estimator dynamically selects sparse weight subsets for
 *          the loss and gradient computation.
 *
 * Conventions shared by every call
 *   - Layout follows PyTorch nn.Linear / PEFT: a frozen weight W0 is n x k
 *     (out x in, row-major), y = x W0^T; LoRA A is r x k, B is n x r and the
 *     LoRA output is lora_scale * (x A^T) B^T.  All matrices are row-major and
 *     contiguous (leading dimension = number of columns).
 *   - Tokens: X has T = batch * seq rows; in sequence b the first ctx_len[b]
 *     rows are context tokens (sparse path), the other rows are output tokens
 *     (dense path) [ART §3].  "Compact context" matrices hold the T_C context
 *     rows in (sequence, position) order, "compact output" matrices the T_O
 *     output rows in the same order.  ctx_len is a HOST array.
 *   - Every tensor pointer is a DEVICE pointer owned by the caller and must be
 *     16-byte aligned; the library never allocates device memory.  Scratch
 *     space is the caller's workspace `ws`.  Workspace query: call with
 *     ws == NULL; the call validates its arguments, stores the bytes it needs
 *     in *ws_bytes, launches nothing and returns SLORA_OK.  Otherwise
 *     *ws_bytes is the size of `ws` and must be at least that amount.
 *   - dtype SLORA_F32 computes in fp32 throughout (CUDA-core FMA, for exact
 *     parity work); SLORA_BF16 takes bf16 activations/weights, accumulates in
 *     fp32 on the tensor cores and writes bf16 activations.  LoRA gradients
 *     (dA, dB) and estimator factors (L, U) are always fp32.
 *   - Calls are asynchronous on `stream` and return a slora_status.  A failed
 *     call launches nothing (argument errors) or reports the first CUDA error
 *     (SLORA_ERR_CUDA).  slora_last_error_string() gives a thread-local text.
 *     Calls are re-entrant when given distinct workspaces and outputs.
 *   - slora_ffn_fwd_bwd runs some small launches on a library-owned side
 *     stream of the current device (created on first use, never destroyed),
 *     forked from `stream` by an event and joined back to it before the call
 *     returns, so everything stays ordered on `stream` and the call can be
 *     captured into a CUDA graph.  While one host thread captures such a
 *     call, no other thread may run an FFN call on the same device.
 *   - Requires an sm_100 device (SLORA_ERR_UNSUPPORTED otherwise).
 */
#ifndef SLORA_H_
#define SLORA_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef void* slora_stream_t; /* a cudaStream_t; NULL = legacy default stream */

typedef enum {
  SLORA_OK = 0,
  SLORA_ERR_INVALID_ARG = 1, /* null pointer, bad enum, sparsity outside [0,1) */
  SLORA_ERR_SHAPE = 2,       /* inconsistent or unsupported sizes            */
  SLORA_ERR_ALIGN = 3,       /* a pointer is not 16-byte aligned             */
  SLORA_ERR_WORKSPACE = 4,   /* *ws_bytes smaller than required              */
  SLORA_ERR_UNSUPPORTED = 5, /* device is not sm_100                         */
  SLORA_ERR_CUDA = 6,        /* a CUDA runtime/driver call failed            */
  SLORA_ERR_TIMEOUT = 7      /* reserved: bounded device wait expired        */
} slora_status;

typedef enum { SLORA_F32 = 0, SLORA_BF16 = 1 } slora_dtype;

typedef enum {
  SLORA_CRIT_FFN_SWIGLU_L2 = 0, /* SwiGLU FFN: L2 norm of the estimated activation        */
  SLORA_CRIT_QK_NORM = 1,       /* attention q/k: QK-norm, top-k per head group            */
  SLORA_CRIT_FFN_GRAM = 2,      /* SwiGLU FFN variant: ||g_hat_j|| * ||u_hat_j||             */
  SLORA_CRIT_QK_ROPE_PAIR = 3,  /* q/k QK-norm over rotate-half pairs (c, c + head_dim/2) */
  SLORA_CRIT_L2_NORM = 4        /* one projection (v): L2 norm per channel, top-k per head */
} slora_criterion;

typedef enum {
  SLORA_SLICE_NONE = 0,     /* dense LoRA linear on every row                         */
  SLORA_SLICE_OUT_ROWS = 1, /* context rows compute only output channels idx (q,k,gate,up) */
  SLORA_SLICE_IN_COLS = 2   /* context rows read only input channels idx (down, o)    */
} slora_slice;

typedef struct {
  int32_t batch;          /* number of sequences                          */
  int32_t seq;            /* rows per sequence                            */
  const int32_t* ctx_len; /* HOST array [batch], 0 <= ctx_len[b] <= seq   */
} slora_tokens;

/* Text of the last error on this thread ("" after success). */
const char* slora_last_error_string(void);

/* Library version as MAJOR*10000 + MINOR*100 + PATCH. */
int slora_version(void);

/*
 * Errors that kernels record on the device instead of faulting (not part of
 * the method).  Waits for the current device to finish its work, then returns
 *   SLORA_ERR_INVALID_ARG  a caller-supplied channel list (idx of the linear
 *                          calls, idx_force of the FFN call) held an entry
 *                          outside its weight: the library replaced it by
 *                          channel 0 before any kernel read through it, so
 *                          that call's results are wrong but no memory
 *                          outside the caller's buffers was touched;
 *   SLORA_ERR_TIMEOUT      a pipeline wait inside a kernel gave up (its
 *                          call's outputs are undefined);
 *   SLORA_OK               neither happened since the last clear.
 * clear != 0 resets the recorded state.
 */
slora_status slora_device_error(int clear);

/*
 * Test hook for the error path above (not part of the method): the budget, in
 * SM clock cycles, of the pipeline waits of the skinny-contraction stream
 * kernel (the LoRA projections and gradients on strided inputs).  0 makes
 * every wait that does not succeed at its first poll give up, so the next
 * call raises the device flag that slora_device_error reports as
 * SLORA_ERR_TIMEOUT and leaves its outputs undefined; the device stays usable.
 * A negative value restores the default (about one second).  Synchronous;
 * affects every later call on the current device.
 */
slora_status slora_set_wait_budget(int64_t cycles);

/*
 * Launch accounting and optional per-kernel timing (not part of the method;
 * used to measure it).
 *   slora_launch_count()   kernels this library has launched in this process.
 *   slora_profile_enable() on != 0 clears the record and brackets every later
 *                          launch with CUDA events on its stream; 0 stops.
 *   slora_profile_read()   totals since enabling for one kernel class:
 *                          "gemm_tc" (tcgen05 sliced GEMMs), "gemm_simt"
 *                          (CUDA-core GEMMs), "estimate" (channel scores),
 *                          "select" (top-k), "elementwise", "aux" (row maps,
 *                          operand packing), "prepare", "skinny" (rank-r
 *                          LoRA projections and gradients), "compact"
 *                          (selected-row gather), "attention" (the causal
 *                          attention core's forward and backward), "norm"
 *                          (RMS normalisation).  It synchronizes the
 *                          recorded events.  work = algorithmic FLOPs for the
 *                          GEMM classes (2*M*N*K on the selected sizes) and
 *                          the attention kernels (2 head_dim per causal
 *                          query-key pair and product: two forward, five
 *                          backward), bytes moved for the others.  Unknown class: SLORA_ERR_INVALID_ARG.
 */
int64_t slora_launch_count(void);
void slora_profile_enable(int on);
slora_status slora_profile_read(const char* kernel_class, int64_t* launches, double* total_ms,
                                double* work);

/*
 * slora_svd_prepare — offline truncated SVD of one frozen weight, done once
 * before training [ART §2: the weights are decomposed once, ahead of training,
 * keeping the leading singular modes; §7: rank 8].
 *
 *   W      [n x k] dtype dt, the frozen weight W0.
 *   rank   r, 1 <= r <= min(n, k, 48).
 *   n_iter subspace iterations (0 = default 12).
 *   seed   seed of the counter-based Gaussian start block.
 *   L      out [k x r] fp32: V_r diag(sigma_r) (right factor times singular values).
 *   U      out [n x r] fp32: U_r (orthonormal left factor), so X W0^T ~= (X L) U^T.
 *   W_t    out [k x n] dtype dt, optional (NULL = skip): the transposed copy of W
 *          that SLORA_SLICE_IN_COLS layers and the FFN down projection take.
 * Singular-vector signs are arbitrary; only products such as L U^T are defined.
 * Method: randomized block subspace iteration with Cholesky-QR
 * re-orthonormalisation and an fp64 Jacobi eigen-solve of the small projected
 * Gram matrix, all on the device.  Ordered on `stream`; not on the hot path.
 */
slora_status slora_svd_prepare(const void* W, int64_t n, int64_t k, slora_dtype dt, int rank,
                               int n_iter, uint64_t seed, float* L, float* U, void* W_t,
                               void* ws, size_t* ws_bytes, slora_stream_t stream);

/*
 * slora_estimate_select — online low-rank estimate on the context tokens,
 * channel scores and top-k selection [ART §1 criteria (FFN: L2 norm of the
 * neuron's activity; q/k: QK-norm from the query-key product), §2 estimator,
 * §3 per-layer ratio; ABS].
 *
 *   crit     SLORA_CRIT_FFN_SWIGLU_L2 or SLORA_CRIT_QK_NORM.
 *   X        [T x d] dtype dt, layer input, full row layout (context rows used).
 *   (L0,U0)  factors of gate (FFN) or q (QK): L0 [d x rank], U0 [n0 x rank] fp32.
 *   (L1,U1)  factors of up (FFN) or k (QK):   L1 [d x rank], U1 [n1 x rank] fp32.
 *   FFN: n0 == n1 == d_ff; heads/kv_heads/head_dim ignored.  score_j is the L2
 *        norm over context tokens of silu(g_hat_j) * u_hat_j with
 *        g_hat = (X_C L0) U0^T, u_hat = (X_C L1) U1^T; k_keep = d_ff - floor(s*d_ff).
 *        idx_out [k_keep] int32 receives the kept channels in ascending order.
 *   QK:  n0 = heads*head_dim, n1 = kv_heads*head_dim, heads % kv_heads == 0.
 *        Group g (one key head, heads/kv_heads query heads) scores channel c as
 *        ||K_hat[:,g,c]|| * sum_h ||Q_hat[:,h,c]||; k_h = head_dim - floor(s*head_dim)
 *        channels are kept per group.  idx_out [(heads + kv_heads) * k_h] int32:
 *        first, for every query head h, its group's kept channels as
 *        h*head_dim + c (ascending); then for every key head g, g*head_dim + c.
 *   FFN_GRAM (estimator variant; [ART §1-§2], a cheaper stand-in for the
 *        activation norm): as FFN, but score_j = ||g_hat_j|| * ||u_hat_j||, each
 *        norm a quadratic form of the r x r Gram matrix of X_C L (no per-token
 *        nonlinearity; an upper bound of the activation-norm score).
 *   QK_ROPE_PAIR (estimator variant): as QK, but the keys of a head are the
 *        head_dim/2 rotate-half pairs (c, c + head_dim/2) that rotary position
 *        embedding turns together; a pair's norms are taken over both channels
 *        (invariant under the rotation), k_p = head_dim/2 - floor(s*head_dim/2)
 *        pairs are kept, so k_h = 2 k_p channels per head, listed as the kept
 *        first channels c ascending, then the matching c + head_dim/2.
 *   L2_NORM (projection-set variant: v sliced on its output channels and o
 *        on the matching input channels; [ART §6]): one matrix (L0, U0 of
 *        v; L1 and U1 may be NULL), n0 = kv_heads*head_dim (v's width).
 *        Channel c of value head g scores ||V_hat[:, g, c]||; k_h = head_dim -
 *        floor(s*head_dim) kept per value head.  idx_out [(heads + kv_heads)
 *        * k_h] as for QK: first, for every query head h (o's input channels),
 *        its group's set as h*head_dim + c; then for every value head g,
 *        g*head_dim + c.
 *   Ties: equal scores go to the lower index.  A selection spans at most
 *        32768 channels (d_ff for the FFN criteria, head_dim otherwise).
 *   sparsity  s in [0, 1).
 *   k_out     HOST int32*, receives k_keep (FFN criteria) or k_h (per head).
 *   scores_out optional fp32 scores: [d_ff] (FFN criteria), [kv_heads*head_dim]
 *             (QK), [kv_heads*head_dim/2] (QK_ROPE_PAIR, one per pair),
 *             [heads*head_dim] (L2_NORM).
 */
slora_status slora_estimate_select(slora_criterion crit, const void* X, slora_dtype dt,
                                   const slora_tokens* tok, int64_t d, const float* L0,
                                   const float* U0, int64_t n0, const float* L1, const float* U1,
                                   int64_t n1, int rank, int heads, int kv_heads, int head_dim,
                                   double sparsity, int32_t* idx_out, int32_t* k_out,
                                   float* scores_out, void* ws, size_t* ws_bytes,
                                   slora_stream_t stream);

/*
 * slora_estimate_select_noalloc — slora_estimate_select for callers that
 * cannot allocate device memory.  The pages have no counterpart of this call;
 * it exists for integration only.
 *
 * Some callers have no way to give the library a workspace: a plugin
 * interface of a framework that owns every device allocation through its own
 * pool and hands a kernel only its input and output buffers; a process that
 * reserved nearly all device memory at start-up, so a later cudaMalloc would
 * fail; a latency-critical loop that cannot afford cudaMalloc's implicit
 * device synchronisation.  This entry point takes the same arguments as
 * slora_estimate_select minus the workspace, and runs with a scratch buffer
 * that the library itself holds in device memory: a fixed
 * slora_noalloc_scratch_bytes() bytes (32 MiB) on every GPU that loads the
 * library, kept until the process exits.  It calls no cudaMalloc, cudaFree or
 * other allocating routine.
 *   - Problems whose scratch need exceeds the buffer are refused with
 *     SLORA_ERR_WORKSPACE (the message states both sizes); use
 *     slora_estimate_select with a workspace for those.
 *   - The first call on a device resolves the buffer's device address
 *     (cudaGetSymbolAddress, with that device current); make that first call
 *     before any stream capture.  The address is cached per device with the
 *     context it was resolved in and resolved again when a call comes from
 *     another context (a non-primary context, or the primary context
 *     recreated after cudaDeviceReset).
 *   - All calls on a device share the one buffer and it keeps the last
 *     call's contents (nothing in it needs to start at zero).  Calls that
 *     overlap on the GPU (different streams, or different host threads
 *     without ordering) race on it: serialise them.
 */
size_t slora_noalloc_scratch_bytes(void);
slora_status slora_estimate_select_noalloc(slora_criterion crit, const void* X, slora_dtype dt,
                                           const slora_tokens* tok, int64_t d, const float* L0,
                                           const float* U0, int64_t n0, const float* L1,
                                           const float* U1, int64_t n1, int rank, int heads,
                                           int kv_heads, int head_dim, double sparsity,
                                           int32_t* idx_out, int32_t* k_out, float* scores_out,
                                           slora_stream_t stream);

/*
 * slora_linear_fwd — one LoRA linear on the selected slices, output tokens
 * dense [ART §1, §3, §6, §7; ABS].
 *
 *   W       frozen weight in the layout whose ROWS are the sliced channels:
 *           NONE / OUT_ROWS: W0 [n x k];  IN_COLS: W0^T [k x n].
 *   A [r x k], B [n x r] dtype dt; lora_scale s.
 *   idx     device int32 [n_idx], ascending, distinct, within [0, n) (OUT_ROWS)
 *           or [0, k) (IN_COLS); ignored for NONE.
 *   side NONE:     X_ctx = X [T x k];                  Y_ctx = Y [T x n].
 *   side OUT_ROWS: X_ctx = X [T x k];                  Y_ctx [T_C x n_idx] compact,
 *                  Y_ctx[:, j] = X_C W0[idx_j]^T + s (X_C A^T) B[idx_j]^T;
 *                                                      Y_out [T_O x n] compact, dense.
 *   side IN_COLS:  X_ctx [T_C x n_idx] compact (column j = input channel idx_j),
 *                  X_out [T_O x k] compact;            Y_ctx = Y [T x n] full layout,
 *                  Y[C] = X_ctx W0[:, idx]^T + s (X_ctx A[:, idx]^T) B^T.
 *   XA_save [T x r] fp32 full row layout, optional: the LoRA down-projection of
 *           each row as used above (unscaled), needed by slora_linear_bwd.
 * Unused pointers may be NULL.  Channels outside idx are not computed for
 * context rows (they are not stored: outputs are compact).
 */
slora_status slora_linear_fwd(slora_dtype dt, const slora_tokens* tok, int64_t k, int64_t n,
                              const void* W, const void* A, const void* B, int r_lora,
                              float lora_scale, slora_slice side, const int32_t* idx,
                              int32_t n_idx, const void* X_ctx, const void* X_out, void* Y_ctx,
                              void* Y_out, float* XA_save, void* ws, size_t* ws_bytes,
                              slora_stream_t stream);

/*
 * slora_linear_bwd — backward of slora_linear_fwd with W0 frozen [ABS: loss
 * and gradient computed on the selected subset].
 *
 *   Same layer arguments as the forward, plus
 *   XA_save  [T x r] fp32 from the forward.
 *   dY_ctx / dY_out  shaped like Y_ctx / Y_out of the forward.
 *   dX_ctx / dX_out  shaped like X_ctx / X_out of the forward (written).
 *   dA [r x k], dB [n x r] fp32, OVERWRITTEN.  Skipped channels of context rows
 *   contribute nothing: with no output tokens, rows of dB (OUT_ROWS) or
 *   columns of dA (IN_COLS) outside idx are exactly zero.
 */
slora_status slora_linear_bwd(slora_dtype dt, const slora_tokens* tok, int64_t k, int64_t n,
                              const void* W, const void* A, const void* B, int r_lora,
                              float lora_scale, slora_slice side, const int32_t* idx,
                              int32_t n_idx, const void* X_ctx, const void* X_out,
                              const float* XA_save, const void* dY_ctx, const void* dY_out,
                              void* dX_ctx, void* dX_out, float* dA, float* dB, void* ws,
                              size_t* ws_bytes, slora_stream_t stream);

/* One SwiGLU FFN layer: out = (silu(X Wg^T) * (X Wu^T)) Wd^T, each projection
 * with its LoRA pair.  All device pointers; weights and LoRA factors in the
 * call's dtype, estimator factors fp32. */
typedef struct {
  int64_t d, d_ff;       /* model and intermediate width                       */
  int32_t r_svd;         /* estimator rank (1..48)                             */
  int32_t r_lora;        /* LoRA rank (1..32)                                  */
  float lora_scale;      /* s                                                  */
  const void* Wg;        /* [d_ff x d] gate                                    */
  const void* Wu;        /* [d_ff x d] up                                      */
  const void* Wd_t;      /* [d_ff x d] TRANSPOSED down weight (Wd is d x d_ff) */
  const void *Ag, *Bg;   /* [r x d], [d_ff x r]                                */
  const void *Au, *Bu;   /* [r x d], [d_ff x r]                                */
  const void *Ad, *Bd;   /* [r x d_ff], [d x r]                                */
  const float *Lg, *Ug;  /* gate estimator factors [d x r_svd], [d_ff x r_svd] */
  const float *Lu, *Uu;  /* up estimator factors                               */
} slora_ffn_layer;

typedef struct {
  float *dAg, *dBg, *dAu, *dBu, *dAd, *dBd; /* fp32, shapes of the factors; overwritten */
} slora_ffn_grads;

/*
 * slora_ffn_fwd_bwd — the whole hot path of one FFN layer for one step:
 * estimate + select (unless idx_force), sliced gate/up on the kept channels
 * for context rows, down projection reading only those channels, dense
 * output rows, then the matching sparse backward [ART §1-§3, §6-§7; ABS].
 *
 *   X, dOut   [T x d] dtype dt, full row layout.
 *   sparsity  s in [0, 1): k_keep = d_ff - floor(s*d_ff).
 *   out, dX   [T x d] dtype dt (written).
 *   grads     the six LoRA gradients (written).
 *   idx_out   device int32 [d_ff]: receives the k_keep channels used (ascending).
 *   k_out     HOST int32*: receives k_keep.
 *   idx_force optional device int32 [k_force] ascending channel set: skips the
 *             estimator and uses this set (same-index parity runs); then
 *             sparsity is ignored and k_keep = k_force.
 *   dOut == NULL runs the forward only (estimate, select, out, idx_out); dX
 *             and grads may then be NULL.  A layer stack runs its forwards
 *             this way and, in the backward, calls again with dOut and the
 *             forward's channel set as idx_force (the FFN forward recomputed
 *             instead of stored).
 */
slora_status slora_ffn_fwd_bwd(slora_dtype dt, const slora_ffn_layer* layer,
                               const slora_tokens* tok, double sparsity, const void* X,
                               const void* dOut, void* out, void* dX, const slora_ffn_grads* grads,
                               int32_t* idx_out, int32_t* k_out, const int32_t* idx_force,
                               int32_t k_force, void* ws, size_t* ws_bytes,
                               slora_stream_t stream);

/*
 * slora_ffn_bwd — the backward half of slora_ffn_fwd_bwd, for callers that run
 * a layer's forward earlier (a layer stack: every forward, then every
 * backward) without recomputing it.  The previous call on this workspace must
 * have been slora_ffn_fwd_bwd with dOut == NULL and the same dt, layer, tok,
 * sparsity, X, out, idx_out, idx_force and k_force, and the workspace must be
 * untouched since: it holds that forward's state (row maps, compacted weight
 * slices, g, u, h and the LoRA projections).  dOut, dX and grads as in
 * slora_ffn_fwd_bwd; out and idx_out are not written; the fp32 path returns
 * SLORA_ERR_UNSUPPORTED.
 */
slora_status slora_ffn_bwd(slora_dtype dt, const slora_ffn_layer* layer, const slora_tokens* tok,
                           double sparsity, const void* X, const void* dOut, void* out, void* dX,
                           const slora_ffn_grads* grads, int32_t* idx_out, int32_t* k_out,
                           const int32_t* idx_force, int32_t k_force, void* ws,
                           size_t* ws_bytes, slora_stream_t stream);

/*
 * slora_ffn_fwd_bwd_per_seq — slora_ffn_fwd_bwd with one channel set per
 * sequence instead of one per batch [ART §1: the channels are chosen per
 * input]: each sequence's context rows are scored and selected on their own
 * and computed on their own set S_b; output rows stay dense; the LoRA
 * gradients are the sum over sequences, added in sequence order.
 *   Arguments as slora_ffn_fwd_bwd, except:
 *   idx_out   device int32 [batch x d_ff]: sequence b's k_keep channels
 *             (ascending) at idx_out + b*d_ff.
 *   idx_force optional device int32 [batch x k_force]: sequence b's forced set
 *             at idx_force + b*k_force.
 *   The workspace holds one set of LoRA gradients per sequence and one
 *   per-sequence working area for each of up to four lanes. The sequences run
 *   in those lanes at once: lane 0 on `stream`, the others on library-owned
 *   streams that fork from `stream` and join it before the call returns in
 *   stream order. The result does not depend on the lanes. The first call on
 *   a device creates the lane streams; a call captured into a CUDA graph
 *   before that runs one lane.
 */
slora_status slora_ffn_fwd_bwd_per_seq(slora_dtype dt, const slora_ffn_layer* layer,
                                       const slora_tokens* tok, double sparsity, const void* X,
                                       const void* dOut, void* out, void* dX,
                                       const slora_ffn_grads* grads, int32_t* idx_out,
                                       int32_t* k_out, const int32_t* idx_force,
                                       int32_t k_force, void* ws, size_t* ws_bytes,
                                       slora_stream_t stream);

/* ------------------------------------------------------------------------
 * The rest of a decoder layer around the sparse linears: rotary packing of
 * the q/k rows, the causal attention core and RMS normalisation.  These make
 * the whole-layer training step (sparse q/k feeding the attention core, v/o,
 * the FFN, residuals and norms) run on this library's kernels.  The pages name
 * Llama models without restating their layer; the plainest reading is taken:
 * pre-normalised residual blocks, RMS norm with a frozen gain, rotate-half
 * rotary embedding (pair i with i + head_dim/2, angle p * base^(-2i/head_dim)
 * at position p counted from the start of the sequence), causal softmax
 * attention within each sequence with scale 1/sqrt(head_dim), and query head
 * h reading key/value head h / (heads / kv_heads).  A context row's skipped
 * q/k channels are zero before the rotation [ART §1, §3].
 *
 * Every call takes (ws, ws_bytes, stream) like the calls above (ws == NULL
 * queries the size; a call that needs none reports 0).  bf16 only
 * (SLORA_F32: SLORA_ERR_UNSUPPORTED); head_dim 64 or 128; all pointers device,
 * 16-byte aligned, rows contiguous.
 * ---------------------------------------------------------------------- */

/*
 * slora_rope_pack — full-width rotated q or k rows for the attention core.
 *   n          channels (heads * head_dim), a multiple of head_dim.
 *   idx==NULL: Y [T x n] is the projection output; Y_ctx, Y_out unused.
 *   idx!=NULL: Y_ctx [T_C x n_idx] holds the context rows' computed channels
 *              idx (any order, each in [0, n)), Y_out [T_O x n] the dense
 *              output rows; channels outside idx are zero on context rows.
 *   Y_rot      [T x n] written: every head's pairs rotated by the row's angle.
 */
slora_status slora_rope_pack(slora_dtype dt, const slora_tokens* tok, int64_t n, int head_dim,
                             double rope_base, const int32_t* idx, int32_t n_idx, const void* Y,
                             const void* Y_ctx, const void* Y_out, void* Y_rot, void* ws,
                             size_t* ws_bytes, slora_stream_t stream);

/*
 * slora_rope_unpack — transpose of slora_rope_pack for the gradient.
 *   G [T x n] fp32 gradient of Y_rot.  idx==NULL: dY [T x n] written.
 *   idx!=NULL: dY_ctx [T_C x n_idx] (kept channels) and dY_out [T_O x n]
 *   written; the skipped channels of context rows had no computed output, so
 *   their gradient is dropped.
 */
slora_status slora_rope_unpack(slora_dtype dt, const slora_tokens* tok, int64_t n, int head_dim,
                               double rope_base, const int32_t* idx, int32_t n_idx,
                               const float* G, void* dY, void* dY_ctx, void* dY_out, void* ws,
                               size_t* ws_bytes, slora_stream_t stream);

/*
 * slora_attention_fwd — O = softmax(Q K^T / sqrt(head_dim) + causal mask) V
 * per sequence and query head.
 *   Q [T x heads*head_dim], K, V [T x kv_heads*head_dim] (rotated q/k).
 *   O [T x heads*head_dim] written; lse [batch x heads x seq] fp32 written
 *   (natural log-sum-exp of each row's scaled scores, for the backward).
 */
slora_status slora_attention_fwd(slora_dtype dt, const slora_tokens* tok, int heads,
                                 int kv_heads, int head_dim, const void* Q, const void* K,
                                 const void* V, void* O, float* lse, void* ws, size_t* ws_bytes,
                                 slora_stream_t stream);

/*
 * slora_attention_bwd — gradients of slora_attention_fwd for the upstream dO.
 *   dQ [T x heads*head_dim] and dK [T x kv_heads*head_dim] fp32, dV
 *   [T x kv_heads*head_dim] in dt, all written (key/value gradients summed
 *   over their query-head group).  dQ sums per-key-tile parts with atomic
 *   adds: its rounding order is not fixed from run to run.
 */
slora_status slora_attention_bwd(slora_dtype dt, const slora_tokens* tok, int heads,
                                 int kv_heads, int head_dim, const void* Q, const void* K,
                                 const void* V, const void* O, const float* lse, const void* dO,
                                 float* dQ, float* dK, void* dV, void* ws, size_t* ws_bytes,
                                 slora_stream_t stream);

/*
 * slora_rmsnorm_fwd — H = X + A (A may be NULL: H = X and H is not written),
 * N = H / sqrt(mean(H^2) + eps) * g per row; rstd [T] fp32 = 1/sqrt(mean(H^2)+eps).
 *   X, A, H, N [T x d]; g [d]; d a multiple of 8.  N may be NULL (only the add).
 */
slora_status slora_rmsnorm_fwd(slora_dtype dt, int64_t T, int64_t d, float eps, const void* X,
                               const void* A, const void* g, void* H, void* N, float* rstd,
                               void* ws, size_t* ws_bytes, slora_stream_t stream);

/*
 * slora_rmsnorm_bwd — dX = dRes + J^T (dN0 + dN1 + dN2) for N = rmsnorm(H)
 * with g frozen: J^T dN = rstd g dN - H rstd^3 mean(H g dN).  Any of dN1, dN2,
 * dRes may be NULL (dN0 is required).  All [T x d] in dt; dX written.
 */
slora_status slora_rmsnorm_bwd(slora_dtype dt, int64_t T, int64_t d, const void* H,
                               const float* rstd, const void* g, const void* dN0,
                               const void* dN1, const void* dN2, const void* dRes, void* dX,
                               void* ws, size_t* ws_bytes, slora_stream_t stream);

#ifdef __cplusplus
}
#endif
#endif /* SLORA_H_ */
