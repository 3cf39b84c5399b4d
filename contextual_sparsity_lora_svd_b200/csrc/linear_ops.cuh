// Launch sequences of the sliced LoRA linear and the SwiGLU FFN layer.
#pragma once

#include "common.cuh"

namespace slora {

struct LinearDesc {
  int dt;
  TokenInfo ti;
  int64_t k, n;
  const void* W;  // [n x k] (NONE, OUT_ROWS) or [k x n] (IN_COLS)
  const void* A;  // [r x k]
  const void* B;  // [n x r]
  int r;
  float s;
  slora_slice side;
  const int32_t* idx;
  int32_t n_idx;
};

// With plan == true only the arena is sized (no pointer is touched).
slora_status linear_fwd_run(const LinearDesc& L, const slora_tokens* tok, const void* X_ctx,
                            const void* X_out, void* Y_ctx, void* Y_out, float* XA_save,
                            Arena& ar, bool plan, cudaStream_t st);
slora_status linear_bwd_run(const LinearDesc& L, const slora_tokens* tok, const void* X_ctx,
                            const void* X_out, const float* XA, const void* dY_ctx,
                            const void* dY_out, void* dX_ctx, void* dX_out, float* dA, float* dB,
                            Arena& ar, bool plan, cudaStream_t st);

struct FfnDesc {
  int dt;
  TokenInfo ti;
  slora_ffn_layer L;
  slora_ffn_grads G;
  int64_t kkeep;
  double sparsity;  // ratio the estimator selects at (unused with idx_force)
  cudaStream_t side = nullptr;  // side stream for the small operand layouts (null: the default one)
};

slora_status ffn_run(const FfnDesc& F, const slora_tokens* tok, const void* X, const void* dOut,
                     void* out, void* dX, int32_t* idx, const int32_t* idx_force, Arena& ar,
                     bool plan, cudaStream_t st, bool bwd_only = false);

// Estimator (estimate + select) shared by slora_estimate_select and the FFN
// call, in two steps so that a run path can take all of its workspace before
// its first launch: estimate_reserve takes the scratch buffers from the arena
// (nothing is launched), estimate_select_launch runs the kernels on them.
struct EstBufs {
  float* P = nullptr;        // X_C [L0 | L1] (when not supplied precomputed)
  float* ppart = nullptr;    // split partials of that projection (bf16 path)
  void* prs = nullptr;       // bf16 terms of [L0 | L1] for that projection (bf16 path)
  float* scores = nullptr;   // per-channel scores (the caller's scores_out when given)
  float* partial = nullptr;  // FFN score partials over token chunks
  double* gram = nullptr;    // Gram matrices of the projection
  double* gram_part = nullptr;  // their partials over token chunks
  unsigned* cnt = nullptr;   // arrival counters of the estimator kernels, zero on entry
  void* psplit = nullptr;    // split operand rows of the tensor-core score kernel
  int64_t ncnt = 0;
  int nsplit = 1;
};
// Layout of one criterion's scores and selection.
struct CritPlan {
  bool activation = false;  // SwiGLU activation norm (tensor-core score kernel)
  int mode = 0;             // Gram-form criteria: kCritModeQK or kCritModeL2
  int nmat = 2;             // projected matrices (columns of P: nmat * rank)
  int groups = 1, rep = 1, N = 0, nkeys = 0;
  bool pairs = false;
  int64_t kkeep = 0;        // keys kept per group (pairs with `pairs`)
  int64_t per_head = 0;     // channels kept per head (2 kkeep with pairs)
};
CritPlan crit_plan(slora_criterion crit, int64_t n0, int heads, int kv_heads, int head_dim,
                   double sparsity);
EstBufs estimate_reserve(slora_criterion crit, int dt, const TokenInfo& ti, int64_t d, int64_t n0,
                         int rank, int heads, int kv_heads, int head_dim, bool has_pre,
                         float* scores_out, Arena& ar);
// With has_pre the low-rank projection of the context rows is already
// available (full row layout, row t of the context set at P_pre[ctx_rows[t]]).
// sk_counters: zeroed counters of the projection stream (bf16 path without
// has_pre); eb.cnt must have been zeroed too (launch_rowmaps).
slora_status estimate_select_launch(slora_criterion crit, const void* X, int dt,
                                    const TokenInfo& ti, const int32_t* ctx_rows, int64_t d,
                                    const float* L0, const float* U0, int64_t n0, const float* L1,
                                    const float* U1, int rank, int heads, int kv_heads,
                                    int head_dim, double sparsity, int32_t* idx_out,
                                    const EstBufs& eb, cudaStream_t st, bool has_pre = false,
                                    const float* P_pre = nullptr, int64_t ldp_pre = 0,
                                    unsigned* sk_counters = nullptr);

}  // namespace slora
