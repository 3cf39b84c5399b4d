// C ABI entry points: argument validation, workspace planning and the launch
// sequence of each call.  Every step of the hot path runs in this library's
// kernels; the host only validates, carves the workspace and launches.
#include <algorithm>
#include <cmath>

#include "estimator.cuh"
#include "gemm_simt.cuh"
#include "linear_ops.cuh"
#include "lora_pack.cuh"
#include "skinny.cuh"
#include "swiglu.cuh"

namespace slora {

slora_status svd_prepare_impl(const void* W, int64_t n, int64_t k, int dt, int rank, int n_iter,
                              uint64_t seed, float* L, float* U, void* W_t, Arena& ar,
                              bool plan_only, cudaStream_t st);

namespace {

#define REQ_PTR(p)                                                                      \
  do {                                                                                  \
    if (!(p)) SLORA_FAIL(SLORA_ERR_INVALID_ARG, "%s: required pointer %s is NULL", fn, #p); \
    if (!aligned16(p)) SLORA_FAIL(SLORA_ERR_ALIGN, "%s: %s is not 16-byte aligned", fn, #p); \
  } while (0)

#define OPT_PTR(p)                                                                      \
  do {                                                                                  \
    if ((p) && !aligned16(p)) SLORA_FAIL(SLORA_ERR_ALIGN, "%s: %s is not 16-byte aligned", fn, #p); \
  } while (0)

slora_status check_dtype(const char* fn, slora_dtype dt) {
  if (dt != SLORA_F32 && dt != SLORA_BF16)
    SLORA_FAIL(SLORA_ERR_INVALID_ARG, "%s: unknown dtype %d", fn, int(dt));
  return SLORA_OK;
}

slora_status check_row(const char* fn, const char* what, int64_t len, int dt) {
  const int64_t q = dt == kF32 ? 4 : 8;  // rows start on 16-byte boundaries
  if (len <= 0) SLORA_FAIL(SLORA_ERR_SHAPE, "%s: %s=%lld must be positive", fn, what, (long long)len);
  if (len % q) SLORA_FAIL(SLORA_ERR_SHAPE, "%s: %s=%lld must be a multiple of %lld", fn, what,
                          (long long)len, (long long)q);
  return SLORA_OK;
}

slora_status check_sparsity(const char* fn, double s) {
  if (!(s >= 0.0 && s < 1.0))
    SLORA_FAIL(SLORA_ERR_INVALID_ARG, "%s: sparsity %g outside [0, 1)", fn, s);
  return SLORA_OK;
}

// Channels kept at sparsity s: N - floor(s * N) (the skipped count rounds down).
int64_t keep_count(int64_t N, double s) {
  double skip = std::floor(s * double(N) + 1e-9);
  return N - int64_t(skip);
}

slora_status finish_ws(const char* fn, const Arena& ar, void* ws, size_t* ws_bytes) {
  if (!ws_bytes) SLORA_FAIL(SLORA_ERR_INVALID_ARG, "%s: ws_bytes is NULL", fn);
  if (!ws) {
    *ws_bytes = ar.used;
    return SLORA_OK;
  }
  if (*ws_bytes < ar.used)
    SLORA_FAIL(SLORA_ERR_WORKSPACE, "%s: workspace of %zu bytes, %zu needed", fn, *ws_bytes,
               ar.used);
  return SLORA_OK;
}

}  // namespace
}  // namespace slora

using namespace slora;

// --------------------------------------------------------------- prepare
extern "C" slora_status slora_svd_prepare(const void* W, int64_t n, int64_t k, slora_dtype dt,
                                          int rank, int n_iter, uint64_t seed, float* L,
                                          float* U, void* W_t, void* ws, size_t* ws_bytes,
                                          slora_stream_t stream) {
  const char* fn = "slora_svd_prepare";
  clear_error();
  SLORA_TRY(check_dtype(fn, dt));
  REQ_PTR(W); REQ_PTR(L); REQ_PTR(U); OPT_PTR(W_t); OPT_PTR(ws);
  SLORA_TRY(check_row(fn, "k", k, dt));
  SLORA_TRY(check_row(fn, "n", n, dt));
  if (rank < 1 || rank > 48 || rank > std::min(n, k))
    SLORA_FAIL(SLORA_ERR_SHAPE, "%s: rank %d outside [1, min(n, k, 48)]", fn, rank);
  if (n_iter < 0 || n_iter > 100) SLORA_FAIL(SLORA_ERR_INVALID_ARG, "%s: n_iter %d", fn, n_iter);
  Arena plan;
  SLORA_TRY(svd_prepare_impl(W, n, k, dt, rank, n_iter, seed, L, U, W_t, plan, true, nullptr));
  const bool query = ws == nullptr;
  SLORA_TRY(finish_ws(fn, plan, ws, ws_bytes));
  if (query) return SLORA_OK;
  SLORA_TRY(check_device());
  Arena ar;
  ar.base = static_cast<char*>(ws);
  ar.cap = *ws_bytes;
  return svd_prepare_impl(W, n, k, dt, rank, n_iter, seed, L, U, W_t, ar, false,
                          static_cast<cudaStream_t>(stream));
}

// --------------------------------------------------------- estimate+select
namespace slora {
CritPlan crit_plan(slora_criterion crit, int64_t n0, int heads, int kv_heads, int head_dim,
                   double sparsity) {
  CritPlan cp;
  switch (crit) {
    case SLORA_CRIT_FFN_SWIGLU_L2:
      cp.activation = true;
      cp.N = cp.nkeys = int(n0);
      break;
    case SLORA_CRIT_FFN_GRAM:  // ||g_hat_j|| * ||u_hat_j||: one group over d_ff
      cp.mode = kCritModeQK;
      cp.N = cp.nkeys = int(n0);
      break;
    case SLORA_CRIT_QK_NORM:
    case SLORA_CRIT_QK_ROPE_PAIR:
      cp.mode = kCritModeQK;
      cp.groups = kv_heads;
      cp.rep = heads / kv_heads;
      cp.N = head_dim;
      cp.pairs = crit == SLORA_CRIT_QK_ROPE_PAIR;
      cp.nkeys = cp.pairs ? head_dim / 2 : head_dim;
      break;
    case SLORA_CRIT_L2_NORM:
      cp.mode = kCritModeL2;
      cp.nmat = 1;
      cp.groups = kv_heads;
      cp.rep = heads / kv_heads;
      cp.N = cp.nkeys = head_dim;
      break;
  }
  cp.kkeep = keep_count(cp.nkeys, sparsity);
  cp.per_head = cp.pairs ? 2 * cp.kkeep : cp.kkeep;
  return cp;
}

EstBufs estimate_reserve(slora_criterion crit, int dt, const TokenInfo& ti, int64_t d, int64_t n0,
                         int rank, int heads, int kv_heads, int head_dim, bool has_pre,
                         float* scores_out, Arena& ar) {
  const CritPlan cp = crit_plan(crit, n0, heads, kv_heads, head_dim, 0.0);
  EstBufs eb;
  if (!has_pre) eb.P = ar.take<float>(size_t(std::max<int64_t>(ti.T_C, 1)) * cp.nmat * rank);
  if (!has_pre && dt == kBF16) {
    const int nc = cp.nmat * rank <= 64 ? cp.nmat * rank : rank;  // columns of one pass
    eb.ppart = ar.take<float>(size_t(rowdot_part_floats(ti.T_C, d, nc)));
    eb.prs = ar.take<__nv_bfloat16>(size_t(skinny_rsplit_elems(d)));
  }
  const int64_t nsc = int64_t(cp.groups) * cp.nkeys;
  eb.scores = scores_out ? scores_out : ar.take<float>(size_t(nsc));
  if (cp.activation) {
    eb.nsplit = ffn_score_splits(ti.T_C, n0, rank);
    eb.partial = ar.take<float>(size_t(eb.nsplit) * n0);
    if (rank <= 8) eb.psplit = ar.take<uint4>(size_t(score_split_tiles(ti.T_C)) * 1024);
  } else {
    eb.gram_part = ar.take<double>(size_t(gram_blocks(ti.T_C)) * cp.nmat * rank * rank);
    eb.gram = ar.take<double>(size_t(cp.nmat) * rank * rank);
  }
  eb.ncnt = estimator_counter_count(cp.nkeys, rank, cp.groups);
  eb.cnt = ar.take<unsigned>(size_t(eb.ncnt));
  return eb;
}

slora_status estimate_select_launch(slora_criterion crit, const void* X, int dt,
                                    const TokenInfo& ti, const int32_t* ctx_rows, int64_t d,
                                    const float* L0, const float* U0, int64_t n0, const float* L1,
                                    const float* U1, int rank, int heads, int kv_heads,
                                    int head_dim, double sparsity, int32_t* idx_out,
                                    const EstBufs& eb, cudaStream_t st, bool has_pre,
                                    const float* P_pre, int64_t ldp_pre, unsigned* sk_counters) {
  const CritPlan cp = crit_plan(crit, n0, heads, kv_heads, head_dim, sparsity);
  const float* Puse = P_pre;
  int64_t ldp = ldp_pre;
  const int32_t* pmap = has_pre ? ctx_rows : nullptr;
  const int nc = cp.nmat * rank;
  if (!has_pre) {
    // P = X_C [L0 | L1] (or X_C L0 alone)
    if (dt == kBF16) {  // tensor-core stream over X_C, fp32 factors split in 3 bf16 terms
      SkY y;
      y.ptr = X; y.ld = d; y.map = ctx_rows;
      if (!sk_counters) SLORA_FAIL(SLORA_ERR_INVALID_ARG, "estimator: counter workspace missing");
      SkWork w;
      w.part = eb.ppart;
      w.rsplit = eb.prs;
      w.counters = sk_counters;
      // one pass for both factors when their columns fit the stream kernel's 64,
      // else one pass per factor
      const bool one_pass = nc <= 64;
      for (int p = 0; p < (one_pass ? 1 : cp.nmat); ++p) {
        SkR rr;
        rr.ptr = p == 0 ? L0 : L1; rr.dt = kF32; rr.si = rank; rr.sq = 1;
        if (one_pass && cp.nmat == 2) {
          rr.qsplit = rank; rr.ptr_b = L1; rr.dt_b = kF32; rr.si_b = rank; rr.sq_b = 1;
        }
        SkRowOut o;
        o.out1 = eb.P; o.ld1 = nc; o.off1 = int64_t(p) * rank;
        SLORA_TRY(rowdot(y, ti.T_C, d, rr, one_pass ? nc : rank, o, w, st));
      }
    } else {  // fp32 activations: CUDA-core fp32 FMA
      for (int p = 0; p < cp.nmat; ++p) {
        GemmArgs g;
        g.M = ti.T_C; g.N = rank; g.nseg = 1;
        g.seg[0].a = rowmajor(X, dt, d, ctx_rows);
        g.seg[0].b = colmajor(p == 0 ? L0 : L1, kF32, rank);
        g.seg[0].K = d;
        g.c = out_rowmajor(eb.P + p * rank, kF32, nc);
        SLORA_TRY(gemm_simt(g, st));
      }
    }
    Puse = eb.P;
    ldp = nc;
  }
  if (cp.activation)
    return ffn_score_select(Puse, ldp, pmap, ti.T_C, U0, U1, n0, rank, eb.partial, eb.nsplit,
                            eb.scores, eb.cnt, int(cp.kkeep), idx_out, eb.psplit, st);
  int32_t* out_b = nullptr;
  if (crit == SLORA_CRIT_QK_NORM || crit == SLORA_CRIT_QK_ROPE_PAIR ||
      crit == SLORA_CRIT_L2_NORM)
    out_b = idx_out + int64_t(heads) * cp.per_head;
  return gram_scores_select(cp.mode, Puse, ldp, pmap, ti.T_C, U0, U1, rank, cp.groups, cp.rep,
                            cp.N, cp.pairs, int(cp.kkeep), eb.gram_part, eb.gram, eb.scores,
                            eb.cnt, idx_out, out_b, st);
}
}  // namespace slora

extern "C" slora_status slora_estimate_select(slora_criterion crit, const void* X, slora_dtype dt,
                                              const slora_tokens* tok, int64_t d, const float* L0,
                                              const float* U0, int64_t n0, const float* L1,
                                              const float* U1, int64_t n1, int rank, int heads,
                                              int kv_heads, int head_dim, double sparsity,
                                              int32_t* idx_out, int32_t* k_out, float* scores_out,
                                              void* ws, size_t* ws_bytes, slora_stream_t stream) {
  const char* fn = "slora_estimate_select";
  clear_error();
  SLORA_TRY(check_dtype(fn, dt));
  if (crit != SLORA_CRIT_FFN_SWIGLU_L2 && crit != SLORA_CRIT_QK_NORM &&
      crit != SLORA_CRIT_FFN_GRAM && crit != SLORA_CRIT_QK_ROPE_PAIR &&
      crit != SLORA_CRIT_L2_NORM)
    SLORA_FAIL(SLORA_ERR_INVALID_ARG, "%s: unknown criterion %d", fn, int(crit));
  const bool one_matrix = crit == SLORA_CRIT_L2_NORM;
  REQ_PTR(X); REQ_PTR(L0); REQ_PTR(U0); REQ_PTR(idx_out);
  if (!one_matrix) { REQ_PTR(L1); REQ_PTR(U1); }
  OPT_PTR(scores_out); OPT_PTR(ws);
  if (!k_out) SLORA_FAIL(SLORA_ERR_INVALID_ARG, "%s: k_out is NULL", fn);
  SLORA_TRY(check_sparsity(fn, sparsity));
  SLORA_TRY(check_row(fn, "d", d, dt));
  if (rank < 1 || rank > 48) SLORA_FAIL(SLORA_ERR_SHAPE, "%s: rank %d outside [1, 48]", fn, rank);
  TokenInfo ti;
  SLORA_TRY(parse_tokens(tok, &ti));
  if (crit == SLORA_CRIT_FFN_SWIGLU_L2 || crit == SLORA_CRIT_FFN_GRAM) {
    if (n0 <= 0 || n0 != n1) SLORA_FAIL(SLORA_ERR_SHAPE, "%s: FFN needs n0 == n1 > 0", fn);
    if (n0 > topk_max_keys())
      SLORA_FAIL(SLORA_ERR_SHAPE, "%s: n0=%lld beyond the %lld channels one selection supports",
                 fn, (long long)n0, (long long)topk_max_keys());
  } else if (crit == SLORA_CRIT_L2_NORM) {
    if (heads <= 0 || kv_heads <= 0 || head_dim <= 0 || heads % kv_heads ||
        n0 != int64_t(kv_heads) * head_dim)
      SLORA_FAIL(SLORA_ERR_SHAPE, "%s: L2 criterion needs n0 == kv_heads*head_dim and heads a "
                 "multiple of kv_heads (heads=%d, kv_heads=%d, head_dim=%d)", fn, heads,
                 kv_heads, head_dim);
    if (head_dim > topk_max_keys())
      SLORA_FAIL(SLORA_ERR_SHAPE, "%s: head_dim %d too large", fn, head_dim);
  } else {
    if (heads <= 0 || kv_heads <= 0 || head_dim <= 0 || heads % kv_heads)
      SLORA_FAIL(SLORA_ERR_SHAPE, "%s: heads=%d kv_heads=%d head_dim=%d", fn, heads, kv_heads,
                 head_dim);
    if (n0 != int64_t(heads) * head_dim || n1 != int64_t(kv_heads) * head_dim)
      SLORA_FAIL(SLORA_ERR_SHAPE, "%s: n0/n1 must be heads*head_dim / kv_heads*head_dim", fn);
    if (crit == SLORA_CRIT_QK_ROPE_PAIR && head_dim % 2)
      SLORA_FAIL(SLORA_ERR_SHAPE, "%s: rotate-half pairs need an even head_dim (%d)", fn,
                 head_dim);
    if (head_dim > topk_max_keys())
      SLORA_FAIL(SLORA_ERR_SHAPE, "%s: head_dim %d too large", fn, head_dim);
  }
  const CritPlan cp = crit_plan(crit, n0, heads, kv_heads, head_dim, sparsity);
  const int64_t ncnt = skinny_counter_count(ti.T_C, d);
  Arena ar;  // one pass: sizes the query and places the buffers (finish_ws checks the size)
  ar.base = static_cast<char*>(ws);
  int32_t* ctx_rows = ar.take<int32_t>(size_t(std::max<int64_t>(ti.T_C, 1)));
  unsigned* cnt = ar.take<unsigned>(size_t(ncnt));
  const EstBufs eb = estimate_reserve(crit, dt, ti, d, n0, rank, heads, kv_heads, head_dim, false,
                                      scores_out, ar);
  const bool query = ws == nullptr;
  SLORA_TRY(finish_ws(fn, ar, ws, ws_bytes));
  *k_out = int32_t(cp.per_head);
  if (query) return SLORA_OK;
  SLORA_TRY(check_device());
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  SLORA_TRY(launch_rowmaps(tok, ti, ctx_rows, nullptr, st, nullptr, nullptr, cnt, ncnt, eb.cnt,
                           eb.ncnt));
  return estimate_select_launch(crit, X, dt, ti, ctx_rows, d, L0, U0, n0, L1, U1, rank, heads,
                                kv_heads, head_dim, sparsity, idx_out, eb, st, false, nullptr, 0,
                                cnt);
}

// ------------------------------------------------------------ linear calls
namespace {
slora_status linear_common_checks(const char* fn, slora_dtype dt, const slora_tokens* tok,
                                  int64_t k, int64_t n, const void* W, const void* A,
                                  const void* B, int r_lora, slora_slice side,
                                  const int32_t* idx, int32_t n_idx, TokenInfo* ti) {
  SLORA_TRY(check_dtype(fn, dt));
  if (side != SLORA_SLICE_NONE && side != SLORA_SLICE_OUT_ROWS && side != SLORA_SLICE_IN_COLS)
    SLORA_FAIL(SLORA_ERR_INVALID_ARG, "%s: unknown slice side %d", fn, int(side));
  REQ_PTR(W); REQ_PTR(A); REQ_PTR(B);
  SLORA_TRY(check_row(fn, "k", k, dt));
  SLORA_TRY(check_row(fn, "n", n, dt));
  if (r_lora < 1 || r_lora > 64) SLORA_FAIL(SLORA_ERR_SHAPE, "%s: r_lora %d outside [1, 64]", fn, r_lora);
  SLORA_TRY(parse_tokens(tok, ti));
  if (side != SLORA_SLICE_NONE) {
    REQ_PTR(idx);
    const int64_t lim = side == SLORA_SLICE_OUT_ROWS ? n : k;
    if (n_idx < 0 || n_idx > lim)
      SLORA_FAIL(SLORA_ERR_SHAPE, "%s: n_idx=%d outside [0, %lld]", fn, n_idx, (long long)lim);
  }
  return SLORA_OK;
}
}  // namespace

extern "C" slora_status slora_linear_fwd(slora_dtype dt, const slora_tokens* tok, int64_t k,
                                         int64_t n, const void* W, const void* A, const void* B,
                                         int r_lora, float lora_scale, slora_slice side,
                                         const int32_t* idx, int32_t n_idx, const void* X_ctx,
                                         const void* X_out, void* Y_ctx, void* Y_out,
                                         float* XA_save, void* ws, size_t* ws_bytes,
                                         slora_stream_t stream) {
  const char* fn = "slora_linear_fwd";
  clear_error();
  TokenInfo ti;
  SLORA_TRY(linear_common_checks(fn, dt, tok, k, n, W, A, B, r_lora, side, idx, n_idx, &ti));
  REQ_PTR(X_ctx); REQ_PTR(Y_ctx); OPT_PTR(XA_save); OPT_PTR(ws);
  if (side == SLORA_SLICE_OUT_ROWS && ti.T_O > 0) REQ_PTR(Y_out);
  if (side == SLORA_SLICE_IN_COLS && ti.T_O > 0) REQ_PTR(X_out);
  LinearDesc L{int(dt), ti, k, n, W, A, B, r_lora, lora_scale, side, idx, n_idx};
  Arena plan;
  SLORA_TRY(linear_fwd_run(L, tok, X_ctx, X_out, Y_ctx, Y_out, XA_save, plan, true, nullptr));
  const bool query = ws == nullptr;
  SLORA_TRY(finish_ws(fn, plan, ws, ws_bytes));
  if (query) return SLORA_OK;
  SLORA_TRY(check_device());
  Arena ar;
  ar.base = static_cast<char*>(ws);
  ar.cap = *ws_bytes;
  return linear_fwd_run(L, tok, X_ctx, X_out, Y_ctx, Y_out, XA_save, ar, false,
                        static_cast<cudaStream_t>(stream));
}

extern "C" slora_status slora_linear_bwd(slora_dtype dt, const slora_tokens* tok, int64_t k,
                                         int64_t n, const void* W, const void* A, const void* B,
                                         int r_lora, float lora_scale, slora_slice side,
                                         const int32_t* idx, int32_t n_idx, const void* X_ctx,
                                         const void* X_out, const float* XA_save,
                                         const void* dY_ctx, const void* dY_out, void* dX_ctx,
                                         void* dX_out, float* dA, float* dB, void* ws,
                                         size_t* ws_bytes, slora_stream_t stream) {
  const char* fn = "slora_linear_bwd";
  clear_error();
  TokenInfo ti;
  SLORA_TRY(linear_common_checks(fn, dt, tok, k, n, W, A, B, r_lora, side, idx, n_idx, &ti));
  REQ_PTR(X_ctx); REQ_PTR(XA_save); REQ_PTR(dY_ctx); REQ_PTR(dX_ctx); REQ_PTR(dA); REQ_PTR(dB);
  OPT_PTR(ws);
  if (side == SLORA_SLICE_OUT_ROWS && ti.T_O > 0) REQ_PTR(dY_out);
  if (side == SLORA_SLICE_IN_COLS && ti.T_O > 0) { REQ_PTR(X_out); REQ_PTR(dX_out); }
  LinearDesc L{int(dt), ti, k, n, W, A, B, r_lora, lora_scale, side, idx, n_idx};
  Arena plan;
  SLORA_TRY(linear_bwd_run(L, tok, X_ctx, X_out, XA_save, dY_ctx, dY_out, dX_ctx, dX_out, dA,
                           dB, plan, true, nullptr));
  const bool query = ws == nullptr;
  SLORA_TRY(finish_ws(fn, plan, ws, ws_bytes));
  if (query) return SLORA_OK;
  SLORA_TRY(check_device());
  Arena ar;
  ar.base = static_cast<char*>(ws);
  ar.cap = *ws_bytes;
  return linear_bwd_run(L, tok, X_ctx, X_out, XA_save, dY_ctx, dY_out, dX_ctx, dX_out, dA, dB, ar,
                        false, static_cast<cudaStream_t>(stream));
}

// ------------------------------------------------------------------- FFN
namespace {
// Checks shared by the per-batch and the per-sequence FFN calls; sets kkeep.
slora_status ffn_validate(const char* fn, slora_dtype dt, const slora_ffn_layer* layer,
                          const slora_ffn_grads* grads, double sparsity, const void* X,
                          const void* dOut, void* out, void* dX, int32_t* idx_out,
                          int32_t* k_out, const int32_t* idx_force, int32_t k_force, void* ws,
                          int64_t* kkeep) {
  SLORA_TRY(check_dtype(fn, dt));
  // dOut == NULL: forward only (dX and grads unused)
  const bool fwd_only = dOut == nullptr;
  if (!layer || (!grads && !fwd_only))
    SLORA_FAIL(SLORA_ERR_INVALID_ARG, "%s: layer or grads is NULL", fn);
  const slora_ffn_layer& Ly = *layer;
  const slora_ffn_grads Gr = grads ? *grads : slora_ffn_grads{};
  REQ_PTR(Ly.Wg); REQ_PTR(Ly.Wu); REQ_PTR(Ly.Wd_t);
  REQ_PTR(Ly.Ag); REQ_PTR(Ly.Bg); REQ_PTR(Ly.Au); REQ_PTR(Ly.Bu); REQ_PTR(Ly.Ad); REQ_PTR(Ly.Bd);
  REQ_PTR(X); REQ_PTR(out); REQ_PTR(idx_out);
  if (!fwd_only) {
    REQ_PTR(dOut); REQ_PTR(dX);
    REQ_PTR(Gr.dAg); REQ_PTR(Gr.dBg); REQ_PTR(Gr.dAu); REQ_PTR(Gr.dBu); REQ_PTR(Gr.dAd);
    REQ_PTR(Gr.dBd);
  }
  OPT_PTR(ws); OPT_PTR(idx_force);
  if (!k_out) SLORA_FAIL(SLORA_ERR_INVALID_ARG, "%s: k_out is NULL", fn);
  SLORA_TRY(check_row(fn, "d", Ly.d, dt));
  SLORA_TRY(check_row(fn, "d_ff", Ly.d_ff, dt));
  if (Ly.r_lora < 1 || Ly.r_lora > 32)
    SLORA_FAIL(SLORA_ERR_SHAPE, "%s: r_lora %d outside [1, 32]", fn, Ly.r_lora);
  if (idx_force) {
    if (k_force < 0 || k_force > Ly.d_ff)
      SLORA_FAIL(SLORA_ERR_SHAPE, "%s: k_force=%d outside [0, d_ff]", fn, k_force);
    *kkeep = k_force;
  } else {
    SLORA_TRY(check_sparsity(fn, sparsity));
    REQ_PTR(Ly.Lg); REQ_PTR(Ly.Ug); REQ_PTR(Ly.Lu); REQ_PTR(Ly.Uu);
    if (Ly.r_svd < 1 || Ly.r_svd > 48)
      SLORA_FAIL(SLORA_ERR_SHAPE, "%s: r_svd %d outside [1, 48]", fn, Ly.r_svd);
    *kkeep = keep_count(Ly.d_ff, sparsity);
  }
  return SLORA_OK;
}

// One channel set per sequence: the per-batch path run on each sequence's
// rows in turn (each call estimates and selects from that sequence's context
// rows), its LoRA gradients kept per sequence in the workspace and summed in
// sequence order at the end.
slora_status ffn_per_seq_run(const FfnDesc& F, const slora_tokens* tok, const void* X,
                             const void* dOut, void* out, void* dX, int32_t* idx,
                             const int32_t* idx_force, int64_t k_force, Arena& ar, bool plan,
                             cudaStream_t st) {
  const slora_ffn_layer& L = F.L;
  const int B = tok->batch, seq = tok->seq, r = L.r_lora;
  const int64_t d = L.d, Fd = L.d_ff;
  const int64_t es = dt_size(F.dt);
  const bool fwd_only = dOut == nullptr;
  const int64_t glen[6] = {r * d, Fd * r, r * d, Fd * r, r * Fd, d * r};
  int64_t goff[6], gtot = 0;
  for (int q = 0; q < 6; ++q) {
    goff[q] = gtot;
    gtot += (glen[q] + 63) / 64 * 64;
  }
  float* gbuf = fwd_only ? nullptr : ar.take<float>(size_t(B) * gtot);
  // The sequences run in up to kSeqLanes lanes at once: lane 0 on the
  // caller's stream, lane i on side stream i of the library's pool, each
  // with its own sub-workspace (reused by its sequences in stream order) and
  // its own side stream for the operand layouts.  Every sequence writes its
  // own rows, index list and gradient slot; the gradients are summed in
  // sequence order afterwards, so the result does not depend on the lanes.
  constexpr int kSeqLanes = 4;
  const int lanes = std::min(B, kSeqLanes);
  size_t sub = 16;
  for (int b = 0; b < B; ++b) {
    slora_tokens tb{1, seq, &tok->ctx_len[b]};
    FfnDesc Fb = F;
    SLORA_TRY(parse_tokens(&tb, &Fb.ti));
    Arena p;
    SLORA_TRY(ffn_run(Fb, &tb, X, dOut, out, dX, idx, idx_force, p, true, nullptr));
    sub = std::max(sub, p.used);
  }
  char* subws[kSeqLanes] = {};
  for (int i = 0; i < lanes; ++i) subws[i] = ar.take<char>(sub);
  if (plan) return SLORA_OK;
  SLORA_TRY(arena_fits(ar, "slora_ffn_fwd_bwd_per_seq"));
  // one lane while a capture is under way and the stream pool does not exist
  // yet (streams are not created inside a capture)
  cudaStreamCaptureStatus cap = cudaStreamCaptureStatusNone;
  SLORA_CUDA(cudaStreamIsCapturing(st, &cap));
  const int nl =
      (cap == cudaStreamCaptureStatusNone || side_pool_ready(2 * kSeqLanes)) ? lanes : 1;
  cudaStream_t lane_st[kSeqLanes] = {st}, lane_side[kSeqLanes] = {};
  for (int i = 0; i < nl; ++i) {
    if (i > 0) SLORA_TRY(side_stream_at(i, &lane_st[i]));
    SLORA_TRY(side_stream_at(kSeqLanes + i, &lane_side[i]));
  }
  for (int i = 1; i < nl; ++i) SLORA_TRY(fork_side(st, lane_st[i]));
  for (int b = 0; b < B; ++b) {
    const int ln = b % nl;
    slora_tokens tb{1, seq, &tok->ctx_len[b]};
    FfnDesc Fb = F;
    Fb.side = lane_side[ln];
    SLORA_TRY(parse_tokens(&tb, &Fb.ti));
    if (!fwd_only) {
      float* g = gbuf + size_t(b) * gtot;
      Fb.G.dAg = g + goff[0]; Fb.G.dBg = g + goff[1]; Fb.G.dAu = g + goff[2];
      Fb.G.dBu = g + goff[3]; Fb.G.dAd = g + goff[4]; Fb.G.dBd = g + goff[5];
    }
    const int64_t row0 = int64_t(b) * seq;
    auto at = [&](const void* p) -> const char* {
      return p ? static_cast<const char*>(p) + row0 * d * es : nullptr;
    };
    Arena a;
    a.base = subws[ln];
    a.cap = sub;
    SLORA_TRY(ffn_run(Fb, &tb, at(X), at(dOut), const_cast<char*>(at(out)),
                      const_cast<char*>(at(dX)), idx + int64_t(b) * Fd,
                      idx_force ? idx_force + int64_t(b) * k_force : nullptr, a, false,
                      lane_st[ln]));
  }
  for (int i = 1; i < nl; ++i) SLORA_TRY(join_side(st, lane_st[i]));
  if (fwd_only) return SLORA_OK;
  float* dst[6] = {F.G.dAg, F.G.dBg, F.G.dAu, F.G.dBu, F.G.dAd, F.G.dBd};
  SumSeg segs[6];
  for (int q = 0; q < 6; ++q) {
    segs[q].dst = dst[q];
    segs[q].off = goff[q];
    segs[q].len = glen[q];
  }
  return sum_groups(gbuf, B, gtot, segs, 6, st);
}
}  // namespace

extern "C" slora_status slora_ffn_fwd_bwd(slora_dtype dt, const slora_ffn_layer* layer,
                                          const slora_tokens* tok, double sparsity, const void* X,
                                          const void* dOut, void* out, void* dX,
                                          const slora_ffn_grads* grads, int32_t* idx_out,
                                          int32_t* k_out, const int32_t* idx_force,
                                          int32_t k_force, void* ws, size_t* ws_bytes,
                                          slora_stream_t stream) {
  const char* fn = "slora_ffn_fwd_bwd";
  clear_error();
  int64_t kkeep = 0;
  SLORA_TRY(ffn_validate(fn, dt, layer, grads, sparsity, X, dOut, out, dX, idx_out, k_out,
                         idx_force, k_force, ws, &kkeep));
  const slora_ffn_grads Gr = grads ? *grads : slora_ffn_grads{};
  TokenInfo ti;
  SLORA_TRY(parse_tokens(tok, &ti));
  FfnDesc F{int(dt), ti, *layer, Gr, kkeep, sparsity};
  Arena plan;
  SLORA_TRY(ffn_run(F, tok, X, dOut, out, dX, idx_out, idx_force, plan, true, nullptr));
  const bool query = ws == nullptr;
  SLORA_TRY(finish_ws(fn, plan, ws, ws_bytes));
  *k_out = int32_t(kkeep);
  if (query) return SLORA_OK;
  SLORA_TRY(check_device());
  Arena ar;
  ar.base = static_cast<char*>(ws);
  ar.cap = *ws_bytes;
  return ffn_run(F, tok, X, dOut, out, dX, idx_out, idx_force, ar, false,
                 static_cast<cudaStream_t>(stream));
}

extern "C" slora_status slora_ffn_bwd(slora_dtype dt, const slora_ffn_layer* layer,
                                      const slora_tokens* tok, double sparsity, const void* X,
                                      const void* dOut, void* out, void* dX,
                                      const slora_ffn_grads* grads, int32_t* idx_out,
                                      int32_t* k_out, const int32_t* idx_force, int32_t k_force,
                                      void* ws, size_t* ws_bytes, slora_stream_t stream) {
  const char* fn = "slora_ffn_bwd";
  clear_error();
  if (!dOut) SLORA_FAIL(SLORA_ERR_INVALID_ARG, "%s: dOut is NULL", fn);
  int64_t kkeep = 0;
  SLORA_TRY(ffn_validate(fn, dt, layer, grads, sparsity, X, dOut, out, dX, idx_out, k_out,
                         idx_force, k_force, ws, &kkeep));
  TokenInfo ti;
  SLORA_TRY(parse_tokens(tok, &ti));
  FfnDesc F{int(dt), ti, *layer, *grads, kkeep, sparsity};
  Arena plan;
  SLORA_TRY(ffn_run(F, tok, X, dOut, out, dX, idx_out, idx_force, plan, true, nullptr, true));
  const bool query = ws == nullptr;
  SLORA_TRY(finish_ws(fn, plan, ws, ws_bytes));
  *k_out = int32_t(kkeep);
  if (query) return SLORA_OK;
  SLORA_TRY(check_device());
  Arena ar;
  ar.base = static_cast<char*>(ws);
  ar.cap = *ws_bytes;
  return ffn_run(F, tok, X, dOut, out, dX, idx_out, idx_force, ar, false,
                 static_cast<cudaStream_t>(stream), true);
}

extern "C" slora_status slora_ffn_fwd_bwd_per_seq(
    slora_dtype dt, const slora_ffn_layer* layer, const slora_tokens* tok, double sparsity,
    const void* X, const void* dOut, void* out, void* dX, const slora_ffn_grads* grads,
    int32_t* idx_out, int32_t* k_out, const int32_t* idx_force, int32_t k_force, void* ws,
    size_t* ws_bytes, slora_stream_t stream) {
  const char* fn = "slora_ffn_fwd_bwd_per_seq";
  clear_error();
  int64_t kkeep = 0;
  SLORA_TRY(ffn_validate(fn, dt, layer, grads, sparsity, X, dOut, out, dX, idx_out, k_out,
                         idx_force, k_force, ws, &kkeep));
  const slora_ffn_grads Gr = grads ? *grads : slora_ffn_grads{};
  TokenInfo ti;
  SLORA_TRY(parse_tokens(tok, &ti));
  FfnDesc F{int(dt), ti, *layer, Gr, kkeep, sparsity};
  Arena plan;
  SLORA_TRY(ffn_per_seq_run(F, tok, X, dOut, out, dX, idx_out, idx_force, k_force, plan, true,
                            nullptr));
  const bool query = ws == nullptr;
  SLORA_TRY(finish_ws(fn, plan, ws, ws_bytes));
  *k_out = int32_t(kkeep);
  if (query) return SLORA_OK;
  SLORA_TRY(check_device());
  Arena ar;
  ar.base = static_cast<char*>(ws);
  ar.cap = *ws_bytes;
  return ffn_per_seq_run(F, tok, X, dOut, out, dX, idx_out, idx_force, k_force, ar, false,
                         static_cast<cudaStream_t>(stream));
}
