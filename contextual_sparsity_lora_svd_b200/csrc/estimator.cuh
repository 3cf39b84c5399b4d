// SVD sparsity estimator, channel scores and top-k selection (device side).
#pragma once

#include "common.cuh"

namespace slora {

// FFN: sumsq partials over token chunks of (silu(P_g U_g^T) * (P_u U_u^T))^2,
// then a fixed-order reduction and sqrt into scores[n].
//   P [T_C x ldp] fp32 with P_g in columns [0, r) and P_u in [r, 2r).
// P rows are read through pmap when given (row t of the context set is P[pmap[t]]).
slora_status ffn_scores(const float* P, int64_t ldp, const int32_t* pmap, int64_t T_C,
                        const float* Ug, const float* Uu, int64_t n, int r, float* partial,
                        int nsplit, float* scores, cudaStream_t st);
int ffn_score_splits(int64_t T_C, int64_t n, int r);

// QK: Gram matrices of P_q (cols [0,r)) and P_k (cols [r,2r)) in fp64, then
// score[g, c] = ||K_hat[:, g, c]|| * sum_{h in g} ||Q_hat[:, h, c]||.
slora_status qk_scores(const float* P, int64_t ldp, const int32_t* pmap, int64_t T_C,
                       const float* Uq,
                       const float* Uk, int r, int heads, int kv_heads, int head_dim,
                       double* gram /* [2 r r] */, float* scores, cudaStream_t st);

// Top-k per group: scores [groups x N] -> for each group its k best channels
// (ties to the lower index) in ascending order.  The selected local channel
// set S_g of group g is written as
//   out_a[(g*rep + j) * k + i] = (g*rep + j) * N + S_g[i]   for j < rep,
//   out_b[g * k + i]           = g * N + S_g[i]              (if out_b != null).
slora_status topk_select(const float* scores, int groups, int N, int k, int rep,
                         int32_t* out_a, int32_t* out_b, cudaStream_t st);

}  // namespace slora
