// SVD sparsity estimator, channel scores and top-k selection (device side).
#pragma once

#include "common.cuh"

namespace slora {

// Top-k outputs of a group (one key head and its `rep` query heads, or one
// whole score vector): the kept local channels S_g, ascending, are written as
//   out_a[(g*rep + j) * k + i] = (g*rep + j) * N + S_g[i]   for j < rep,
//   out_b[g * k + i]           = g * N + S_g[i]              (if out_b != null).
// Equal scores go to the lower index.

// FFN activation-norm score (one launch), then the selection (one launch):
//   scores[j] = sqrt(sum_t (silu(P_g[t] . U_g[j]) * (P_u[t] . U_u[j]))^2),
//   P [rows x ldp] fp32 with P_g in columns [0, r), P_u in [r, 2r), context
//   token t at row pmap[t] (identity when pmap is null);
//   idx_out[0..k) = the k best channels (when idx_out != null).
// partial: [nsplit x n] floats; counters: estimator_counter_count(n, r, 1)
// unsigned ints, zero on entry; n at most topk_max_keys() when selecting.
slora_status ffn_score_select(const float* P, int64_t ldp, const int32_t* pmap, int64_t T_C,
                              const float* Ug, const float* Uu, int64_t n, int r, float* partial,
                              int nsplit, float* scores, unsigned* counters, int k,
                              int32_t* idx_out, void* psplit, cudaStream_t st);
int ffn_score_splits(int64_t T_C, int64_t n, int r);
// 64-token tiles of the split operand rows the rank <= 8 score kernel reads
// (16 KB each in the workspace argument psplit of ffn_score_select).
int64_t score_split_tiles(int64_t T_C);

// Gram-form criteria.  G_m = P_m^T P_m (fp64) for the P matrices in columns
// [m r, (m+1) r) of P; a channel's estimated norm is sqrt(u^T G_m u) for its
// factor row u.
//   mode 0 (QK-norm): group g scores channel c as
//        ||K_hat[:, g, c]|| * sum_{j < rep} ||Q_hat[:, g*rep + j, c]||
//        with Q from (P_0, U0) and K from (P_1, U1);
//   mode 1 (L2 norm): group g scores channel c as ||Y_hat[:, g, c]|| from (P_0, U0)
//        (its set still goes to the group's `rep` heads of out_a).
// With `pairs`, the keys are the N/2 rotate-half pairs (c, c + N/2), each
// norm taken over both channels of the pair; k is then the number of pairs
// kept and each head keeps 2k channels (all pair firsts, then all seconds).
// gram_part: gram_blocks(T_C) * nmat * r * r doubles; gram: nmat * r * r;
// scores: groups * nkeys floats; counters: 1, zero on entry.
constexpr int kCritModeQK = 0, kCritModeL2 = 1;
slora_status gram_scores_select(int mode, const float* P, int64_t ldp, const int32_t* pmap,
                                int64_t T_C, const float* U0, const float* U1, int r, int groups,
                                int rep, int N, bool pairs, int k, double* gram_part,
                                double* gram, float* scores, unsigned* counters, int32_t* out_a,
                                int32_t* out_b, cudaStream_t st);
int64_t gram_blocks(int64_t T_C);

// Counters (zero on entry) the estimator kernels of one call need.
int64_t estimator_counter_count(int64_t n, int r, int groups);

// Top-k per group over scores [groups x N] (see the layout above).  N at most
// topk_max_keys().
slora_status topk_select(const float* scores, int groups, int N, int k, int rep,
                         int32_t* out_a, int32_t* out_b, cudaStream_t st);
int64_t topk_max_keys();

// Device flag of the estimator kernels (see slora_device_error).
slora_status est_check_error(bool clear);

}  // namespace slora
