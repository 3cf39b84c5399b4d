// Sliced LoRA linear and SwiGLU FFN: the sequence of gathered GEMMs.
//
// SparseLoRA article, section 1: only the selected channels are computed;
// section 3: context tokens take the sparse path, output tokens stay dense;
// sections 6-7: the sparsity is structured (whole channel slices) so the
// GPU sees smaller dense GEMMs.  Forum post with the paper's abstract: the
// loss and the gradients are computed on the selected weight subsets.
//
// Notation: W0 [n x k], A [r x k], B [n x r], s = lora_scale, C / O = context
// and output rows, S = selected channel set (idx).
#include <algorithm>

#include "estimator.cuh"
#include "gemm.cuh"
#include "gemm_tc.cuh"
#include "linear_ops.cuh"
#include "lora_pack.cuh"
#include "skinny.cuh"
#include "swiglu.cuh"

namespace slora {
namespace {

GemmArgs mk(int64_t M, int64_t N, OutRef c) {
  GemmArgs g;
  g.M = M; g.N = N; g.c = c; g.nseg = 0;
  return g;
}
void add(GemmArgs& g, MatRef a, MatRef b, int64_t K, float alpha = 1.0f) {
  Seg& s = g.seg[g.nseg++];
  s.a = a; s.b = b; s.K = K; s.alpha = alpha;
}

}  // namespace

slora_status linear_fwd_tc(const LinearDesc& L, const slora_tokens* tok, const void* X_ctx,
                           const void* X_out, void* Y_ctx, void* Y_out, float* XA_save, Arena& ar,
                           bool plan, cudaStream_t st);
slora_status linear_bwd_tc(const LinearDesc& L, const slora_tokens* tok, const void* X_ctx,
                           const void* X_out, const float* XA, const void* dY_ctx,
                           const void* dY_out, void* dX_ctx, void* dX_out, float* dA, float* dB,
                           Arena& ar, bool plan, cudaStream_t st);

// ------------------------------------------------------------------ forward
namespace {
// The caller's channel list, copied into the workspace with out-of-range
// entries replaced (sanitize_indices), so no kernel reads through a bad index.
slora_status safe_indices(const LinearDesc& L, Arena& ar, bool plan, cudaStream_t st,
                          LinearDesc* out) {
  *out = L;
  if (L.side == SLORA_SLICE_NONE || !L.idx || L.n_idx <= 0) return SLORA_OK;
  int32_t* safe = ar.take<int32_t>(size_t(L.n_idx));
  out->idx = safe;
  if (plan) return SLORA_OK;
  SLORA_TRY(arena_fits(ar, "workspace"));
  const int64_t limit = L.side == SLORA_SLICE_OUT_ROWS ? L.n : L.k;
  return sanitize_indices(L.idx, L.n_idx, limit, safe, st);
}
}  // namespace

slora_status linear_fwd_run(const LinearDesc& L0, const slora_tokens* tok, const void* X_ctx,
                            const void* X_out, void* Y_ctx, void* Y_out, float* XA_save,
                            Arena& ar, bool plan, cudaStream_t st) {
  LinearDesc L;
  SLORA_TRY(safe_indices(L0, ar, plan, st, &L));
  if (L.dt == kBF16)
    return linear_fwd_tc(L, tok, X_ctx, X_out, Y_ctx, Y_out, XA_save, ar, plan, st);
  const TokenInfo& ti = L.ti;
  const int dt = L.dt, r = L.r;
  const int64_t k = L.k, n = L.n, ni = L.n_idx;
  int32_t* ctx_rows = ar.take<int32_t>(size_t(std::max<int64_t>(ti.T_C, 1)));
  int32_t* out_rows = ar.take<int32_t>(size_t(std::max<int64_t>(ti.T_O, 1)));
  float* XA = XA_save ? XA_save : ar.take<float>(size_t(ti.T) * r);
  if (plan) return SLORA_OK;
  SLORA_TRY(arena_fits(ar, "workspace"));
  SLORA_TRY(launch_rowmaps(tok, ti, ctx_rows, out_rows, st));

  if (L.side == SLORA_SLICE_NONE) {
    GemmArgs g = mk(ti.T, r, out_rowmajor(XA, kF32, r));  // XA = X A^T
    add(g, rowmajor(X_ctx, dt, k), rowmajor(L.A, dt, k), k);
    SLORA_TRY(gemm(g, st));
    GemmArgs y = mk(ti.T, n, out_rowmajor(Y_ctx, dt, n));  // Y = X W0^T + s XA B^T
    add(y, rowmajor(X_ctx, dt, k), rowmajor(L.W, dt, k), k);
    add(y, rowmajor(XA, kF32, r), rowmajor(L.B, dt, r), r, L.s);
    return gemm(y, st);
  }
  if (L.side == SLORA_SLICE_OUT_ROWS) {
    GemmArgs g = mk(ti.T, r, out_rowmajor(XA, kF32, r));
    add(g, rowmajor(X_ctx, dt, k), rowmajor(L.A, dt, k), k);
    SLORA_TRY(gemm(g, st));
    // context rows, output channels S
    GemmArgs yc = mk(ti.T_C, ni, out_rowmajor(Y_ctx, dt, ni));
    add(yc, rowmajor(X_ctx, dt, k, ctx_rows), rowmajor(L.W, dt, k, L.idx), k);
    add(yc, rowmajor(XA, kF32, r, ctx_rows), rowmajor(L.B, dt, r, L.idx), r, L.s);
    SLORA_TRY(gemm(yc, st));
    // output rows, dense
    GemmArgs yo = mk(ti.T_O, n, out_rowmajor(Y_out, dt, n));
    add(yo, rowmajor(X_ctx, dt, k, out_rows), rowmajor(L.W, dt, k), k);
    add(yo, rowmajor(XA, kF32, r, out_rows), rowmajor(L.B, dt, r), r, L.s);
    return gemm(yo, st);
  }
  // IN_COLS: W is W0^T [k x n]; context rows read input channels S only.
  {
    GemmArgs gc = mk(ti.T_C, r, out_rowmajor(XA, kF32, r, ctx_rows));  // X_ctx A[:,S]^T
    add(gc, rowmajor(X_ctx, dt, ni), rowmajor(L.A, dt, k, nullptr, L.idx), ni);
    SLORA_TRY(gemm(gc, st));
    GemmArgs go = mk(ti.T_O, r, out_rowmajor(XA, kF32, r, out_rows));  // X_out A^T
    add(go, rowmajor(X_out, dt, k), rowmajor(L.A, dt, k), k);
    SLORA_TRY(gemm(go, st));
    GemmArgs yc = mk(ti.T_C, n, out_rowmajor(Y_ctx, dt, n, ctx_rows));
    add(yc, rowmajor(X_ctx, dt, ni), colmajor(L.W, dt, n, nullptr, L.idx), ni);
    add(yc, rowmajor(XA, kF32, r, ctx_rows), rowmajor(L.B, dt, r), r, L.s);
    SLORA_TRY(gemm(yc, st));
    GemmArgs yo = mk(ti.T_O, n, out_rowmajor(Y_ctx, dt, n, out_rows));
    add(yo, rowmajor(X_out, dt, k), colmajor(L.W, dt, n), k);
    add(yo, rowmajor(XA, kF32, r, out_rows), rowmajor(L.B, dt, r), r, L.s);
    return gemm(yo, st);
  }
}

// ----------------------------------------------------------------- backward
slora_status linear_bwd_run(const LinearDesc& L0, const slora_tokens* tok, const void* X_ctx,
                            const void* X_out, const float* XA, const void* dY_ctx,
                            const void* dY_out, void* dX_ctx, void* dX_out, float* dA, float* dB,
                            Arena& ar, bool plan, cudaStream_t st) {
  LinearDesc L;
  SLORA_TRY(safe_indices(L0, ar, plan, st, &L));
  if (L.dt == kBF16)
    return linear_bwd_tc(L, tok, X_ctx, X_out, XA, dY_ctx, dY_out, dX_ctx, dX_out, dA, dB, ar,
                         plan, st);
  const TokenInfo& ti = L.ti;
  const int dt = L.dt, r = L.r;
  const int64_t k = L.k, n = L.n, ni = L.n_idx;
  const float s = L.s;
  int32_t* ctx_rows = ar.take<int32_t>(size_t(std::max<int64_t>(ti.T_C, 1)));
  int32_t* out_rows = ar.take<int32_t>(size_t(std::max<int64_t>(ti.T_O, 1)));
  float* dYB = ar.take<float>(size_t(ti.T) * r);  // dY B per row, full row layout
  if (plan) return SLORA_OK;
  SLORA_TRY(arena_fits(ar, "workspace"));
  SLORA_TRY(launch_rowmaps(tok, ti, ctx_rows, out_rows, st));

  if (L.side == SLORA_SLICE_NONE) {
    GemmArgs g = mk(ti.T, r, out_rowmajor(dYB, kF32, r));
    add(g, rowmajor(dY_ctx, dt, n), colmajor(L.B, dt, r), n);
    SLORA_TRY(gemm(g, st));
    GemmArgs x = mk(ti.T, k, out_rowmajor(dX_ctx, dt, k));  // dX = dY W0 + s dYB A
    add(x, rowmajor(dY_ctx, dt, n), colmajor(L.W, dt, k), n);
    add(x, rowmajor(dYB, kF32, r), colmajor(L.A, dt, k), r, s);
    SLORA_TRY(gemm(x, st));
    GemmArgs a = mk(r, k, out_rowmajor(dA, kF32, k));  // dA = s dYB^T X
    add(a, colmajor(dYB, kF32, r), colmajor(X_ctx, dt, k), ti.T, s);
    SLORA_TRY(gemm(a, st));
    GemmArgs b = mk(n, r, out_rowmajor(dB, kF32, r));  // dB = s dY^T XA
    add(b, colmajor(dY_ctx, dt, n), colmajor(XA, kF32, r), ti.T, s);
    return gemm(b, st);
  }
  if (L.side == SLORA_SLICE_OUT_ROWS) {
    GemmArgs bc = mk(ti.T_C, r, out_rowmajor(dYB, kF32, r, ctx_rows));  // dY_C B[S]
    add(bc, rowmajor(dY_ctx, dt, ni), colmajor(L.B, dt, r, nullptr, L.idx), ni);
    SLORA_TRY(gemm(bc, st));
    GemmArgs bo = mk(ti.T_O, r, out_rowmajor(dYB, kF32, r, out_rows));  // dY_O B
    add(bo, rowmajor(dY_out, dt, n), colmajor(L.B, dt, r), n);
    SLORA_TRY(gemm(bo, st));
    GemmArgs xc = mk(ti.T_C, k, out_rowmajor(dX_ctx, dt, k, ctx_rows));
    add(xc, rowmajor(dY_ctx, dt, ni), colmajor(L.W, dt, k, nullptr, L.idx), ni);
    add(xc, rowmajor(dYB, kF32, r, ctx_rows), colmajor(L.A, dt, k), r, s);
    SLORA_TRY(gemm(xc, st));
    GemmArgs xo = mk(ti.T_O, k, out_rowmajor(dX_ctx, dt, k, out_rows));
    add(xo, rowmajor(dY_out, dt, n), colmajor(L.W, dt, k), n);
    add(xo, rowmajor(dYB, kF32, r, out_rows), colmajor(L.A, dt, k), r, s);
    SLORA_TRY(gemm(xo, st));
    GemmArgs a = mk(r, k, out_rowmajor(dA, kF32, k));  // all rows
    add(a, colmajor(dYB, kF32, r), colmajor(X_ctx, dt, k), ti.T, s);
    SLORA_TRY(gemm(a, st));
    GemmArgs b0 = mk(n, r, out_rowmajor(dB, kF32, r));  // output rows, every channel
    add(b0, colmajor(dY_out, dt, n), colmajor(XA, kF32, r, nullptr, out_rows), ti.T_O, s);
    SLORA_TRY(gemm(b0, st));
    GemmArgs b1 = mk(ni, r, out_rowmajor(dB, kF32, r, L.idx, nullptr, 1));  // += ctx, rows S
    add(b1, colmajor(dY_ctx, dt, ni), colmajor(XA, kF32, r, nullptr, ctx_rows), ti.T_C, s);
    return gemm(b1, st);
  }
  // IN_COLS
  {
    GemmArgs g = mk(ti.T, r, out_rowmajor(dYB, kF32, r));  // dY B, every row
    add(g, rowmajor(dY_ctx, dt, n), colmajor(L.B, dt, r), n);
    SLORA_TRY(gemm(g, st));
    GemmArgs xc = mk(ti.T_C, ni, out_rowmajor(dX_ctx, dt, ni));  // dY_C W0[:,S] + s dYB_C A[:,S]
    add(xc, rowmajor(dY_ctx, dt, n, ctx_rows), rowmajor(L.W, dt, n, L.idx), n);
    add(xc, rowmajor(dYB, kF32, r, ctx_rows), colmajor(L.A, dt, k, L.idx), r, s);
    SLORA_TRY(gemm(xc, st));
    GemmArgs xo = mk(ti.T_O, k, out_rowmajor(dX_out, dt, k));
    add(xo, rowmajor(dY_ctx, dt, n, out_rows), rowmajor(L.W, dt, n), n);
    add(xo, rowmajor(dYB, kF32, r, out_rows), colmajor(L.A, dt, k), r, s);
    SLORA_TRY(gemm(xo, st));
    GemmArgs a0 = mk(r, k, out_rowmajor(dA, kF32, k));  // output rows, every column
    add(a0, colmajor(dYB, kF32, r, nullptr, out_rows), colmajor(X_out, dt, k), ti.T_O, s);
    SLORA_TRY(gemm(a0, st));
    GemmArgs a1 = mk(r, ni, out_rowmajor(dA, kF32, k, nullptr, L.idx, 1));  // += ctx, cols S
    add(a1, colmajor(dYB, kF32, r, nullptr, ctx_rows), colmajor(X_ctx, dt, ni), ti.T_C, s);
    SLORA_TRY(gemm(a1, st));
    GemmArgs b = mk(n, r, out_rowmajor(dB, kF32, r));  // dB = s dY^T XA, every row
    add(b, colmajor(dY_ctx, dt, n), colmajor(XA, kF32, r), ti.T, s);
    return gemm(b, st);
  }
}


// ------------------------------------------------------- FFN, bf16, tcgen05
// The eight large contractions (gate|up forward, down forward, dh backward,
// dX backward; each once for the context rows on the selected channels and
// once for the dense output rows) run on the tcgen05 kernel over the selected
// slices compacted into contiguous rows; the rank-r LoRA projections and the
// LoRA gradients (HBM-bound, N or M = r) run on the skinny tensor-core
// stream kernels.
namespace {
TcMat mat(const void* p, int64_t rows, int64_t cols, int64_t ld) {
  TcMat m;
  m.ptr = p; m.rows = rows; m.cols = cols; m.ld = ld;
  return m;
}
struct TcBuilder {
  TcGemm g;
  TcBuilder(const int4* tiles, int64_t ntiles, int a_compact, int out_compact, int64_t M,
            int64_t N, int paired, int epi) {
    g.tiles = tiles; g.n_mtiles = int(ntiles); g.a_compact = a_compact;
    g.out_compact = out_compact; g.M = M; g.N = N; g.paired = paired; g.epi = epi;
  }
  TcBuilder& seg(TcMat a, TcMat b0, int bmode, int64_t K, int bpair = 0, TcMat b1 = TcMat()) {
    if (K <= 0) return *this;  // an empty slice contributes nothing
    TcSeg& s = g.seg[g.nseg++];
    s.a = a; s.b0 = b0; s.b1 = b1; s.bmode = bmode; s.bpair = bpair; s.K = K;
    return *this;
  }
  TcBuilder& out(void* o0, void* o1, void* o2, int64_t ldo) {
    g.out0 = o0; g.out1 = o1; g.out2 = o2; g.ldo = ldo;
    return *this;
  }
  // SwiGLU-backward inputs g, u and the row count of g, u, dG and dU
  TcBuilder& in(const void* i0, const void* i1, int64_t ldi, int64_t io_rows) {
    g.in0 = i0; g.in1 = i1; g.ldi = ldi; g.io_rows = io_rows;
    return *this;
  }
  // rank projection of the epilogue values (h, or dG and dU), see TcGemm
  TcBuilder& proj(const void* p0, const void* p1, int64_t ld, int pr, float* part,
                  int64_t rows) {
    g.proj0 = p0; g.proj1 = p1; g.ldproj = ld; g.proj_r = pr; g.proj_part = part;
    g.proj_rows = rows;
    return *this;
  }
};
}  // namespace

slora_status ffn_run_tc(const FfnDesc& F, const slora_tokens* tok, const void* X,
                        const void* dOut, void* out, void* dX, int32_t* idx,
                        const int32_t* idx_force, Arena& ar, bool plan, cudaStream_t st,
                        bool bwd_only) {
  const TokenInfo& ti = F.ti;
  const slora_ffn_layer& L = F.L;
  const slora_ffn_grads& G = F.G;
  const int dt = kBF16, r = L.r_lora;
  const int64_t d = L.d, Fd = L.d_ff, kk = F.kkeep, TC = ti.T_C, TO = ti.T_O, T = ti.T;
  const float s = L.lora_scale;
  const int64_t ldk = round8(std::max<int64_t>(kk, 1)), lr = round8(r), lr2 = round8(2 * r);
  const int64_t nct = count_tiles(tok, true), nott = count_tiles(tok, false);
  const int64_t nntC = (kk + 127) / 128, nntO = (Fd + 127) / 128;
  auto bf = [&](int64_t rows, int64_t cols) {
    return static_cast<void*>(
        ar.take<__nv_bfloat16>(size_t(std::max<int64_t>(rows * cols, 1))));
  };
  int32_t* ctx_rows = ar.take<int32_t>(size_t(std::max<int64_t>(TC, 1)));
  int32_t* out_rows = ar.take<int32_t>(size_t(std::max<int64_t>(TO, 1)));
  int4* ctiles = ar.take<int4>(size_t(std::max<int64_t>(nct, 1)));
  int4* otiles = ar.take<int4>(size_t(std::max<int64_t>(nott, 1)));
  float* XA = ar.take<float>(size_t(T) * 2 * r);
  void* XAb = bf(T, lr2);
  float* hA = ar.take<float>(size_t(T) * r);
  void* hAbC = bf(TC, lr);
  void* hAbO = bf(TO, lr);
  float* dOB = ar.take<float>(size_t(T) * r);
  void* dOBb = bf(T, lr);
  float* dGB = ar.take<float>(size_t(T) * 2 * r);
  void* dGBbC = bf(TC, lr2);
  void* dGBbO = bf(TO, lr2);
  void* BpC = bf(nntC * 256, lr2);
  void* BpO = bf(nntO * 256, lr2);
  void* AdtS = bf(kk, lr);
  void* Adt = bf(Fd, lr);
  void* Bdp = bf(d, lr);
  // rank-r projections done in the GEMM epilogues (h Ad^T in the gate|up GEMMs,
  // [dG Bg | dU Bu] in the dh GEMMs) instead of separate passes over h, dG, dU;
  // per-N-tile partials, summed in order by reduce_row_partials
  const bool proj = lr == 8 || lr == 16;
  const int64_t ntFc = (kk + 127) / 128, ntFo = (Fd + 127) / 128;  // paired gate|up tiles
  const int64_t ntBc = (kk + 255) / 256, ntBo = (Fd + 255) / 256;  // dh tiles
  const bool bpad = proj && (r != lr || !aligned16(L.Bg) || !aligned16(L.Bu));
  void* BgS = proj ? bf(kk, lr) : nullptr;  // rows S of B_g, B_u (padded to lr columns)
  void* BuS = proj ? bf(kk, lr) : nullptr;
  void* BgP = bpad ? bf(Fd, lr) : nullptr;  // B_g, B_u padded / realigned copies
  void* BuP = bpad ? bf(Fd, lr) : nullptr;
  float* projC = proj ? ar.take<float>(size_t(std::max({ntFc * TC * lr, ntBc * TC * 2 * lr,
                                                         int64_t(1)})))
                      : nullptr;
  float* projO = proj ? ar.take<float>(size_t(std::max({ntFo * TO * lr, ntBo * TO * 2 * lr,
                                                         int64_t(1)})))
                      : nullptr;
  void* AgAu = bf(2 * r, d);
  void* WgS = bf(kk, d);  // selected rows of the frozen weights, compacted once per step
  void* WuS = bf(kk, d);
  void* WdS = bf(kk, d);  // rows S of Wd^T
  void* gC = bf(TC, ldk);
  void* uC = bf(TC, ldk);
  void* hC = bf(TC, ldk);
  void* dGC = bf(TC, ldk);
  void* dUC = bf(TC, ldk);
  void* gO = bf(TO, Fd);
  void* uO = bf(TO, Fd);
  void* hO = bf(TO, Fd);
  void* dGO = bf(TO, Fd);
  void* dUO = bf(TO, Fd);
  // context-row parts of dAd, dBg, dBu on the channel subset (added into the
  // full-channel results after the batched contraction)
  const bool ctxg = TC > 0 && kk > 0;
  float* SAd = ar.take<float>(size_t(std::max<int64_t>(kk * r, 1)));
  float* SBg = ar.take<float>(size_t(std::max<int64_t>(kk * r, 1)));
  float* SBu = ar.take<float>(size_t(std::max<int64_t>(kk * r, 1)));
  auto Yv = [](const void* p, int64_t ld, const int32_t* map = nullptr) {
    SkY y; y.ptr = p; y.ld = ld; y.map = map; return y;
  };
  // rank-r operands of the LoRA contractions: fp32 ones rounded to one bf16
  // term (the estimator's factors keep three, set on the pass over X below)
  auto Rv = [](const void* p, int dtp, int64_t si, int64_t sq, const int32_t* map = nullptr,
               int64_t map_limit = INT64_MAX) {
    SkR rr; rr.ptr = p; rr.dt = dtp; rr.si = si; rr.sq = sq; rr.map = map;
    rr.map_limit = map_limit; rr.terms = dtp == kF32 ? 1 : 0; return rr;
  };
  // The rank-r gradients that sum over tokens, as one batched coldot:
  // dBd = s dOut^T hA, dAd = s dOB^T h, dBg = s dG^T XA_g, dBu = s dU^T XA_u,
  // each output-row part over every channel and each context-row part on S.
  auto grad_jobs = [&](SkColJob* cj, void* rHA, void* rDO, void* rDC, void* rXgO, void* rXgC,
                       void* rXuO, void* rXuC) {
    auto cjob = [&](const void* Y, int64_t ld, int64_t M, int64_t K, const SkR& Rr, void* rsp_,
                    float* o, int64_t ldo, int trans) {
      SkColJob j;
      j.Y = Yv(Y, ld); j.M = M; j.K = K; j.R = Rr; j.c = r; j.rs = rsp_;
      j.o.out = o; j.o.ldo = ldo; j.o.trans = trans; j.o.scale = s;
      return j;
    };
    int n = 0;
    cj[n++] = cjob(dOut, d, T, d, Rv(hA, kF32, r, 1), rHA, G.dBd, r, 0);
    cj[n++] = cjob(hO, Fd, TO, Fd, Rv(dOB, kF32, r, 1, out_rows), rDO, G.dAd, Fd, 1);
    cj[n++] = cjob(dGO, Fd, TO, Fd, Rv(XA, kF32, 2 * r, 1, out_rows), rXgO, G.dBg, r, 0);
    cj[n++] = cjob(dUO, Fd, TO, Fd, Rv(XA + r, kF32, 2 * r, 1, out_rows), rXuO, G.dBu, r, 0);
    if (ctxg) {
      cj[n++] = cjob(hC, ldk, TC, kk, Rv(dOB, kF32, r, 1, ctx_rows), rDC, SAd, kk, 1);
      cj[n++] = cjob(dGC, ldk, TC, kk, Rv(XA, kF32, 2 * r, 1, ctx_rows), rXgC, SBg, r, 0);
      cj[n++] = cjob(dUC, ldk, TC, kk, Rv(XA + r, kF32, 2 * r, 1, ctx_rows), rXuC, SBu, r, 0);
    }
    return n;
  };
  // partial sums of the skinny contractions (reused sequentially)
  const int rs = L.r_svd;
  const bool fused = !idx_force && 2 * r + 2 * rs <= 64;  // one pass over X for XA and P
  int64_t npart = 1;
  for (int64_t M : {T, TC, TO})
    for (int64_t K : {d, kk, Fd})
      for (int c : {r, 2 * r, fused ? 2 * r + 2 * rs : 2 * r}) {
        npart = std::max(npart, rowdot_part_floats(M, K, c));
        npart = std::max(npart, coldot_part_floats(M, K, c));
      }
  SkColJob gj[7];
  const int ngj = grad_jobs(gj, nullptr, nullptr, nullptr, nullptr, nullptr, nullptr, nullptr);
  npart = std::max(npart, coldot_batch_part_floats(gj, ngj));
  float* part = ar.take<float>(size_t(npart));
  const int64_t ncnt = std::max(skinny_counter_count(std::max({T, d, Fd}), std::max({T, d, Fd})),
                                coldot_batch_counter_count(gj, ngj));
  unsigned* rsp = ar.take<unsigned>(size_t(ncnt));
  SkWork sw;
  sw.part = part;
  sw.rsplit = ar.take<__nv_bfloat16>(size_t(skinny_rsplit_elems(std::max({T, d, Fd}))));
  sw.counters = rsp;
  // split rank-r operands of the skinny contractions, prepared in three
  // batched launches (prep_r_batch) instead of one launch per contraction
  auto rsbuf = [&](int64_t I) {
    return static_cast<void*>(ar.take<__nv_bfloat16>(size_t(skinny_rsplit_elems(I))));
  };
  void* rsX = rsbuf(d);
  void* rsBd = rsbuf(d);
  void* rsHA = rsbuf(T);
  void* rsDobO = rsbuf(TO);
  void* rsDobC = rsbuf(TC);
  void* rsXA[2][2];
  for (int p = 0; p < 2; ++p) {
    rsXA[p][0] = rsbuf(TO);
    rsXA[p][1] = rsbuf(TC);
  }
  void* rsDgb = rsbuf(T);
  auto prepared = [&](void* rs) {
    SkWork w = sw;
    w.rsplit = rs;
    w.prepared = true;
    return w;
  };
  auto job = [](const SkR& Rr, int c, int64_t I, void* rs) {
    SkPrep j;
    j.R = Rr; j.c = c; j.I = I; j.rs = rs;
    return j;
  };
  float* LgLu = fused ? ar.take<float>(size_t(d) * 2 * rs) : nullptr;
  float* Pfull = fused ? ar.take<float>(size_t(T) * 2 * rs) : nullptr;
  EstBufs eb;
  if (!idx_force)
    eb = estimate_reserve(SLORA_CRIT_FFN_SWIGLU_L2, dt, ti, d, Fd, rs, 0, 0, 0, fused, nullptr,
                          ar);
  if (plan) return SLORA_OK;
  SLORA_TRY(arena_fits(ar, "slora_ffn_fwd_bwd"));

  TcGemm first;  // the context-row half of each paired launch
  // bwd_only: the workspace still holds the forward state of a forward-only
  // call with the same arguments (same carve-up): resume at the backward
  if (!bwd_only) {
  SLORA_TRY(launch_rowmaps(tok, ti, ctx_rows, out_rows, st, ctiles, otiles, rsp, ncnt, eb.cnt,
                           eb.ncnt));
  // The small LoRA operand layouts run on the library's side stream, beside
  // the pass over X and the estimator (first those independent of the
  // selection, then, once it is known, the ones on the kept channels); the
  // main stream joins them before the first GEMM.
  cudaStream_t side = F.side;
  if (!side) SLORA_TRY(side_stream(&side));
  SLORA_TRY(fork_side(st, side));
  SLORA_TRY(pack_gate_up_b(L.Bg, L.Bu, nullptr, Fd, r, nntO, lr2, BpO, side, Fd));
  SLORA_TRY(transpose_rows(L.Ad, r, Fd, nullptr, Fd, lr, Adt, side));
  SLORA_TRY(copy_pad(L.Bd, d, r, lr, Bdp, side));
  if (bpad) {
    SLORA_TRY(gather_pad(L.Bg, r, nullptr, Fd, r, BgP, lr, side, Fd));
    SLORA_TRY(gather_pad(L.Bu, r, nullptr, Fd, r, BuP, lr, side, Fd));
  }
  SLORA_TRY(stack_rows(L.Ag, L.Au, r, r, d, AgAu, st));
  {  // one stream over X: XA = X [Ag; Au]^T (fp32 and s*XA bf16) and, for the
     // estimator, P = X [Lg | Lu] (fp32-accurate, read for the context rows)
    SkRowOut o;
    o.out1 = XA; o.ld1 = 2 * r; o.out2 = XAb; o.ld2 = lr2; o.s2 = s;
    SkR rr = Rv(AgAu, kBF16, 1, d);
    int c = 2 * r;
    if (fused) {
      SLORA_TRY(concat_cols_f32(L.Lg, L.Lu, d, rs, rs, LgLu, st));
      rr.qsplit = 2 * r; rr.ptr_b = LgLu; rr.dt_b = kF32; rr.si_b = 2 * rs; rr.sq_b = 1;
      o.qsplit = 2 * r; o.out1b = Pfull; o.ld1b = 2 * rs;
      c = 2 * r + 2 * rs;
    }
    const SkPrep jobs[2] = {job(rr, c, d, rsX), job(Rv(L.Bd, kBF16, r, 1), r, d, rsBd)};
    SLORA_TRY(prep_r_batch(jobs, 2, st));
    SLORA_TRY(rowdot(Yv(X, d), T, d, rr, c, o, prepared(rsX), st));
  }
  if (idx_force) {
    if (kk > 0)
      SLORA_TRY(sanitize_indices(idx_force, kk, Fd, idx, st));
  } else {
    SLORA_TRY(estimate_select_launch(SLORA_CRIT_FFN_SWIGLU_L2, X, dt, ti, ctx_rows, d, L.Lg,
                                     L.Ug, Fd, L.Lu, L.Uu, rs, 0, 0, 0, F.sparsity, idx, eb, st,
                                     fused, Pfull, 2 * rs, rsp));
  }
  SLORA_TRY(fork_side(st, side));  // the selection is known
  SLORA_TRY(pack_gate_up_b(L.Bg, L.Bu, idx, kk, r, nntC, lr2, BpC, side, Fd));
  SLORA_TRY(transpose_rows(L.Ad, r, Fd, idx, kk, lr, AdtS, side));
  if (proj) {
    SLORA_TRY(gather_pad(L.Bg, r, idx, kk, r, BgS, lr, side, Fd));
    SLORA_TRY(gather_pad(L.Bu, r, idx, kk, r, BuS, lr, side, Fd));
  }
  // selected slices of the frozen weights as contiguous rows (HBM-speed gather)
  {
    GatherJob gw[3];
    const void* src[3] = {L.Wg, L.Wu, L.Wd_t};
    void* dst[3] = {WgS, WuS, WdS};
    for (int k = 0; k < 3; ++k) {
      gw[k].in = src[k]; gw[k].out = dst[k];
      gw[k].ld_in16 = d / 8; gw[k].ld_out16 = d / 8; gw[k].rows_in = Fd;
    }
    SLORA_TRY(gather_rows_multi(gw, 3, idx, kk, d, st));
  }
  SLORA_TRY(join_side(st, side));

  // ---- forward (each context-row GEMM runs in one launch with its output-row twin)
  {  // gate|up, context rows, channels S: g, u, h = silu(g) u
    TcBuilder b(ctiles, nct, 0, 1, TC, kk, 1, EPI_SWIGLU_FWD);
    b.seg(mat(X, T, d, d), mat(WgS, kk, d, d), B_K, d, 1, mat(WuS, kk, d, d))
        .seg(mat(XAb, T, 2 * r, lr2), mat(BpC, nntC * 256, 2 * r, lr2), B_K, 2 * r)
        .out(gC, uC, hC, ldk);
    if (proj) b.proj(AdtS, nullptr, lr, int(lr), projC, TC);
    first = b.g;
  }
  {  // gate|up, output rows, every channel
    TcBuilder b(otiles, nott, 0, 1, TO, Fd, 1, EPI_SWIGLU_FWD);
    b.seg(mat(X, T, d, d), mat(L.Wg, Fd, d, d), B_K, d, 1, mat(L.Wu, Fd, d, d))
        .seg(mat(XAb, T, 2 * r, lr2), mat(BpO, nntO * 256, 2 * r, lr2), B_K, 2 * r)
        .out(gO, uO, hO, Fd);
    if (proj) b.proj(Adt, nullptr, lr, int(lr), projO, TO);
    SLORA_TRY(gemm_tc_pair(first, b.g, st));
  }
  {  // hA = h Ad^T on the channels used: fp32 (full rows) and s*hA bf16 (compact)
    SkRowOut oc;
    oc.out1 = hA; oc.ld1 = r; oc.map1 = ctx_rows; oc.out2 = hAbC; oc.ld2 = lr; oc.s2 = s;
    SkRowOut oo;
    oo.out1 = hA; oo.ld1 = r; oo.map1 = out_rows; oo.out2 = hAbO; oo.ld2 = lr; oo.s2 = s;
    if (proj) {
      SLORA_TRY(reduce_row_partials(projC, int(ntFc), TC, oc, projO, int(ntFo), TO, oo, int(lr),
                                    int(lr), r, st));
    } else {
      SLORA_TRY(rowdot(Yv(hC, ldk), TC, kk, Rv(L.Ad, kBF16, 1, Fd, idx, Fd), r, oc, sw, st));
      SLORA_TRY(rowdot(Yv(hO, Fd), TO, Fd, Rv(L.Ad, kBF16, 1, Fd), r, oo, sw, st));
    }
  }
  {  // down projection, context rows: reads channels S only (rows S of Wd^T)
    TcBuilder b(ctiles, nct, 1, 0, TC, d, 0, EPI_STORE);
    b.seg(mat(hC, TC, kk, ldk), mat(WdS, kk, d, d), B_MN, kk)
        .seg(mat(hAbC, TC, r, lr), mat(Bdp, d, r, lr), B_K, r)
        .out(out, nullptr, nullptr, d);
    first = b.g;
  }
  {  // down projection, output rows, dense
    TcBuilder b(otiles, nott, 1, 0, TO, d, 0, EPI_STORE);
    b.seg(mat(hO, TO, Fd, Fd), mat(L.Wd_t, Fd, d, d), B_MN, Fd)
        .seg(mat(hAbO, TO, r, lr), mat(Bdp, d, r, lr), B_K, r)
        .out(out, nullptr, nullptr, d);
    SLORA_TRY(gemm_tc_pair(first, b.g, st));
  }
  }  // forward
  if (!dOut) return SLORA_OK;  // forward only

  // ---- backward
  {  // dOB = dOut Bd: fp32 and s*dOB bf16
    SkRowOut o;
    o.out1 = dOB; o.ld1 = r; o.out2 = dOBb; o.ld2 = lr; o.s2 = s;
    SLORA_TRY(rowdot(Yv(dOut, d), T, d, Rv(L.Bd, kBF16, r, 1), r, o, prepared(rsBd), st));
    // every operand that hA, dOB and XA feed, split in one launch
    const SkPrep jobs[7] = {
        job(Rv(hA, kF32, r, 1), r, T, rsHA),
        job(Rv(dOB, kF32, r, 1, out_rows), r, TO, rsDobO),
        job(Rv(dOB, kF32, r, 1, ctx_rows), r, TC, rsDobC),
        job(Rv(XA, kF32, 2 * r, 1, out_rows), r, TO, rsXA[0][0]),
        job(Rv(XA, kF32, 2 * r, 1, ctx_rows), r, TC, rsXA[0][1]),
        job(Rv(XA + r, kF32, 2 * r, 1, out_rows), r, TO, rsXA[1][0]),
        job(Rv(XA + r, kF32, 2 * r, 1, ctx_rows), r, TC, rsXA[1][1])};
    SLORA_TRY(prep_r_batch(jobs, 7, st));
  }
  {  // dh_S = dOut_C Wd[:,S] + s dOB_C Ad[:,S]^T, SwiGLU backward in the epilogue
    TcBuilder b(ctiles, nct, 0, 1, TC, kk, 0, EPI_SWIGLU_BWD);
    b.seg(mat(dOut, T, d, d), mat(WdS, kk, d, d), B_K, d)
        .seg(mat(dOBb, T, r, lr), mat(AdtS, kk, r, lr), B_K, r)
        .out(dGC, dUC, nullptr, ldk)
        .in(gC, uC, ldk, TC);
    if (proj) b.proj(BgS, BuS, lr, int(lr), projC, TC);
    first = b.g;
  }
  {
    TcBuilder b(otiles, nott, 0, 1, TO, Fd, 0, EPI_SWIGLU_BWD);
    b.seg(mat(dOut, T, d, d), mat(L.Wd_t, Fd, d, d), B_K, d)
        .seg(mat(dOBb, T, r, lr), mat(Adt, Fd, r, lr), B_K, r)
        .out(dGO, dUO, nullptr, Fd)
        .in(gO, uO, Fd, TO);
    if (proj)
      b.proj(bpad ? BgP : L.Bg, bpad ? BuP : L.Bu, bpad ? lr : r, int(lr), projO, TO);
    SLORA_TRY(gemm_tc_pair(first, b.g, st));
  }
  if (proj) {  // dGB = [dG Bg | dU Bu] from the dh GEMMs' epilogue partials
    SkRowOut oc;
    oc.out1 = dGB; oc.ld1 = 2 * r; oc.map1 = ctx_rows; oc.out2 = dGBbC; oc.ld2 = lr2; oc.s2 = s;
    SkRowOut oo = oc;
    oo.map1 = out_rows; oo.out2 = dGBbO;
    SLORA_TRY(reduce_row_partials(projC, int(ntBc), TC, oc, projO, int(ntBo), TO, oo,
                                  int(2 * lr), int(lr), r, st));
  }
  for (int p = 0; p < 2 && !proj; ++p) {  // dGB = [dG Bg | dU Bu] (when not fused)
    const void* Bm = p ? L.Bu : L.Bg;
    SkRowOut oo;
    oo.out1 = dGB; oo.ld1 = 2 * r; oo.off1 = p * r; oo.map1 = out_rows;
    oo.out2 = dGBbO; oo.ld2 = lr2; oo.off2 = p * r; oo.s2 = s;
    SLORA_TRY(rowdot(Yv(p ? dUO : dGO, Fd), TO, Fd, Rv(Bm, kBF16, r, 1), r, oo, sw, st));
    SkRowOut oc = oo;
    oc.map1 = ctx_rows; oc.out2 = dGBbC;
    SLORA_TRY(
        rowdot(Yv(p ? dUC : dGC, ldk), TC, kk, Rv(Bm, kBF16, r, 1, idx, Fd), r, oc, sw, st));
  }
  {  // dBd, dAd, dBg, dBu in one launch; then the context rows' parts on S
    SkColJob cj[7];
    const int ncj = grad_jobs(cj, rsHA, rsDobO, rsDobC, rsXA[0][0], rsXA[0][1], rsXA[1][0],
                              rsXA[1][1]);
    SLORA_TRY(coldot_batch(cj, ncj, part, rsp, st));
    if (ctxg) {
      ScatterAddJob sj[3];
      sj[0].dst = G.dAd; sj[0].ld_dst = Fd; sj[0].src = SAd; sj[0].ld_src = kk; sj[0].trans = 1;
      sj[1].dst = G.dBg; sj[1].ld_dst = r; sj[1].src = SBg; sj[1].ld_src = r;
      sj[2].dst = G.dBu; sj[2].ld_dst = r; sj[2].src = SBu; sj[2].ld_src = r;
      SLORA_TRY(scatter_add_cols(sj, 3, idx, kk, r, Fd, st));
    }
  }
  {  // dX, context rows: dG_S Wg[S] + dU_S Wu[S] + s [dG_S Bg[S] | dU_S Bu[S]] [Ag; Au]
    TcBuilder b(ctiles, nct, 1, 0, TC, d, 0, EPI_STORE);
    b.seg(mat(dGC, TC, kk, ldk), mat(WgS, kk, d, d), B_MN, kk)
        .seg(mat(dUC, TC, kk, ldk), mat(WuS, kk, d, d), B_MN, kk)
        .seg(mat(dGBbC, TC, 2 * r, lr2), mat(AgAu, 2 * r, d, d), B_MN, 2 * r)
        .out(dX, nullptr, nullptr, d);
    first = b.g;
  }
  {  // dX, output rows, dense
    TcBuilder b(otiles, nott, 1, 0, TO, d, 0, EPI_STORE);
    b.seg(mat(dGO, TO, Fd, Fd), mat(L.Wg, Fd, d, d), B_MN, Fd)
        .seg(mat(dUO, TO, Fd, Fd), mat(L.Wu, Fd, d, d), B_MN, Fd)
        .seg(mat(dGBbO, TO, 2 * r, lr2), mat(AgAu, 2 * r, d, d), B_MN, 2 * r)
        .out(dX, nullptr, nullptr, d);
    SLORA_TRY(gemm_tc_pair(first, b.g, st));
  }
  {  // dAg | dAu = s dGB^T X over every row, one stream of X
    SkColOut c;
    c.out = G.dAg; c.out_b = G.dAu; c.qsplit = r; c.ldo = d; c.trans = 1; c.scale = s;
    const SkPrep jg = job(Rv(dGB, kF32, 2 * r, 1), 2 * r, T, rsDgb);
    SLORA_TRY(prep_r_batch(&jg, 1, st));
    SLORA_TRY(coldot(Yv(X, d), T, d, Rv(dGB, kF32, 2 * r, 1), 2 * r, c, prepared(rsDgb), st));
  }
  return SLORA_OK;
}

// ---------------------------------------------------------------------- FFN
slora_status ffn_run(const FfnDesc& F, const slora_tokens* tok, const void* X, const void* dOut,
                     void* out, void* dX, int32_t* idx, const int32_t* idx_force, Arena& ar,
                     bool plan, cudaStream_t st, bool bwd_only) {
  if (F.dt == kBF16)
    return ffn_run_tc(F, tok, X, dOut, out, dX, idx, idx_force, ar, plan, st, bwd_only);
  if (bwd_only)
    SLORA_FAIL(SLORA_ERR_UNSUPPORTED, "slora_ffn_bwd: the fp32 path has no separate backward");
  const TokenInfo& ti = F.ti;
  const slora_ffn_layer& L = F.L;
  const slora_ffn_grads& G = F.G;
  const int dt = F.dt, r = L.r_lora;
  const int64_t d = L.d, Fd = L.d_ff, kk = F.kkeep, TC = ti.T_C, TO = ti.T_O, T = ti.T;
  const float s = L.lora_scale;
  const int es = dt_size(dt);
  auto buf = [&](int64_t rows, int64_t cols) {
    return static_cast<void*>(ar.take<char>(size_t(std::max<int64_t>(rows * cols, 1)) * es));
  };
  int32_t* ctx_rows = ar.take<int32_t>(size_t(std::max<int64_t>(TC, 1)));
  int32_t* out_rows = ar.take<int32_t>(size_t(std::max<int64_t>(TO, 1)));
  float* XA = ar.take<float>(size_t(T) * 2 * r);   // [X Ag^T | X Au^T]
  float* hA = ar.take<float>(size_t(T) * r);       // h Ad^T (on the channels used)
  float* dOB = ar.take<float>(size_t(T) * r);      // dOut Bd
  float* dGB = ar.take<float>(size_t(T) * 2 * r);  // [dG Bg | dU Bu] (on the channels used)
  void* gC = buf(TC, kk);
  void* uC = buf(TC, kk);
  void* hC = buf(TC, kk);
  void* dGC = buf(TC, kk);
  void* dUC = buf(TC, kk);
  void* gO = buf(TO, Fd);
  void* uO = buf(TO, Fd);
  void* hO = buf(TO, Fd);
  void* dGO = buf(TO, Fd);
  void* dUO = buf(TO, Fd);
  EstBufs eb;
  if (!idx_force)
    eb = estimate_reserve(SLORA_CRIT_FFN_SWIGLU_L2, dt, ti, d, Fd, L.r_svd, 0, 0, 0, false,
                          nullptr, ar);
  if (plan) return SLORA_OK;
  SLORA_TRY(arena_fits(ar, "slora_ffn_fwd_bwd"));

  SLORA_TRY(launch_rowmaps(tok, ti, ctx_rows, out_rows, st, nullptr, nullptr, nullptr, 0, eb.cnt,
                           eb.ncnt));
  if (idx_force) {
    if (kk > 0)
      SLORA_TRY(sanitize_indices(idx_force, kk, Fd, idx, st));
  } else {
    SLORA_TRY(estimate_select_launch(SLORA_CRIT_FFN_SWIGLU_L2, X, dt, ti, ctx_rows, d, L.Lg,
                                     L.Ug, Fd, L.Lu, L.Uu, L.r_svd, 0, 0, 0, F.sparsity, idx, eb,
                                     st));
  }

  // ---- forward
  for (int p = 0; p < 2; ++p) {  // XA = X [Ag; Au]^T, every row
    GemmArgs g = mk(T, r, out_rowmajor(XA + p * r, kF32, 2 * r));
    add(g, rowmajor(X, dt, d), rowmajor(p ? L.Au : L.Ag, dt, d), d);
    SLORA_TRY(gemm(g, st));
  }
  for (int p = 0; p < 2; ++p) {  // gate / up on context rows, channels S
    const void* W = p ? L.Wu : L.Wg;
    const void* Bm = p ? L.Bu : L.Bg;
    GemmArgs gc = mk(TC, kk, out_rowmajor(p ? uC : gC, dt, kk));
    add(gc, rowmajor(X, dt, d, ctx_rows), rowmajor(W, dt, d, idx), d);
    add(gc, rowmajor(XA + p * r, kF32, 2 * r, ctx_rows), rowmajor(Bm, dt, r, idx), r, s);
    SLORA_TRY(gemm(gc, st));
    GemmArgs go = mk(TO, Fd, out_rowmajor(p ? uO : gO, dt, Fd));  // output rows, dense
    add(go, rowmajor(X, dt, d, out_rows), rowmajor(W, dt, d), d);
    add(go, rowmajor(XA + p * r, kF32, 2 * r, out_rows), rowmajor(Bm, dt, r), r, s);
    SLORA_TRY(gemm(go, st));
  }
  SLORA_TRY(swiglu_fwd(gC, uC, hC, TC * kk, dt, st));
  SLORA_TRY(swiglu_fwd(gO, uO, hO, TO * Fd, dt, st));
  {
    GemmArgs ac = mk(TC, r, out_rowmajor(hA, kF32, r, ctx_rows));  // h_S Ad[:,S]^T
    add(ac, rowmajor(hC, dt, kk), rowmajor(L.Ad, dt, Fd, nullptr, idx), kk);
    SLORA_TRY(gemm(ac, st));
    GemmArgs ao = mk(TO, r, out_rowmajor(hA, kF32, r, out_rows));
    add(ao, rowmajor(hO, dt, Fd), rowmajor(L.Ad, dt, Fd), Fd);
    SLORA_TRY(gemm(ao, st));
    // down projection: context rows read channels S only (rows S of Wd^T)
    GemmArgs oc = mk(TC, d, out_rowmajor(out, dt, d, ctx_rows));
    add(oc, rowmajor(hC, dt, kk), colmajor(L.Wd_t, dt, d, nullptr, idx), kk);
    add(oc, rowmajor(hA, kF32, r, ctx_rows), rowmajor(L.Bd, dt, r), r, s);
    SLORA_TRY(gemm(oc, st));
    GemmArgs oo = mk(TO, d, out_rowmajor(out, dt, d, out_rows));
    add(oo, rowmajor(hO, dt, Fd), colmajor(L.Wd_t, dt, d), Fd);
    add(oo, rowmajor(hA, kF32, r, out_rows), rowmajor(L.Bd, dt, r), r, s);
    SLORA_TRY(gemm(oo, st));
  }
  if (!dOut) return SLORA_OK;  // forward only

  // ---- backward
  {
    GemmArgs g = mk(T, r, out_rowmajor(dOB, kF32, r));  // dOut Bd
    add(g, rowmajor(dOut, dt, d), colmajor(L.Bd, dt, r), d);
    SLORA_TRY(gemm(g, st));
    // dh_S = dOut_C Wd[:,S] + s dOB_C Ad[:,S]   (into dGC, then SwiGLU bwd in place)
    GemmArgs hc = mk(TC, kk, out_rowmajor(dGC, dt, kk));
    add(hc, rowmajor(dOut, dt, d, ctx_rows), rowmajor(L.Wd_t, dt, d, idx), d);
    add(hc, rowmajor(dOB, kF32, r, ctx_rows), colmajor(L.Ad, dt, Fd, idx), r, s);
    SLORA_TRY(gemm(hc, st));
    GemmArgs ho = mk(TO, Fd, out_rowmajor(dGO, dt, Fd));
    add(ho, rowmajor(dOut, dt, d, out_rows), rowmajor(L.Wd_t, dt, d), d);
    add(ho, rowmajor(dOB, kF32, r, out_rows), colmajor(L.Ad, dt, Fd), r, s);
    SLORA_TRY(gemm(ho, st));
    // LoRA grads of the down projection
    GemmArgs a0 = mk(r, Fd, out_rowmajor(G.dAd, kF32, Fd));
    add(a0, colmajor(dOB, kF32, r, nullptr, out_rows), colmajor(hO, dt, Fd), TO, s);
    SLORA_TRY(gemm(a0, st));
    GemmArgs a1 = mk(r, kk, out_rowmajor(G.dAd, kF32, Fd, nullptr, idx, 1));
    add(a1, colmajor(dOB, kF32, r, nullptr, ctx_rows), colmajor(hC, dt, kk), TC, s);
    SLORA_TRY(gemm(a1, st));
    GemmArgs b = mk(d, r, out_rowmajor(G.dBd, kF32, r));
    add(b, colmajor(dOut, dt, d), colmajor(hA, kF32, r), T, s);
    SLORA_TRY(gemm(b, st));
  }
  SLORA_TRY(swiglu_bwd(dGC, gC, uC, dGC, dUC, TC * kk, dt, st));
  SLORA_TRY(swiglu_bwd(dGO, gO, uO, dGO, dUO, TO * Fd, dt, st));
  for (int p = 0; p < 2; ++p) {  // dGB = [dG Bg | dU Bu]
    const void* Bm = p ? L.Bu : L.Bg;
    GemmArgs bc = mk(TC, r, out_rowmajor(dGB + p * r, kF32, 2 * r, ctx_rows));
    add(bc, rowmajor(p ? dUC : dGC, dt, kk), colmajor(Bm, dt, r, nullptr, idx), kk);
    SLORA_TRY(gemm(bc, st));
    GemmArgs bo = mk(TO, r, out_rowmajor(dGB + p * r, kF32, 2 * r, out_rows));
    add(bo, rowmajor(p ? dUO : dGO, dt, Fd), colmajor(Bm, dt, r), Fd);
    SLORA_TRY(gemm(bo, st));
  }
  {
    GemmArgs xc = mk(TC, d, out_rowmajor(dX, dt, d, ctx_rows));
    add(xc, rowmajor(dGC, dt, kk), colmajor(L.Wg, dt, d, nullptr, idx), kk);
    add(xc, rowmajor(dUC, dt, kk), colmajor(L.Wu, dt, d, nullptr, idx), kk);
    add(xc, rowmajor(dGB, kF32, 2 * r, ctx_rows), colmajor(L.Ag, dt, d), r, s);
    add(xc, rowmajor(dGB + r, kF32, 2 * r, ctx_rows), colmajor(L.Au, dt, d), r, s);
    SLORA_TRY(gemm(xc, st));
    GemmArgs xo = mk(TO, d, out_rowmajor(dX, dt, d, out_rows));
    add(xo, rowmajor(dGO, dt, Fd), colmajor(L.Wg, dt, d), Fd);
    add(xo, rowmajor(dUO, dt, Fd), colmajor(L.Wu, dt, d), Fd);
    add(xo, rowmajor(dGB, kF32, 2 * r, out_rows), colmajor(L.Ag, dt, d), r, s);
    add(xo, rowmajor(dGB + r, kF32, 2 * r, out_rows), colmajor(L.Au, dt, d), r, s);
    SLORA_TRY(gemm(xo, st));
  }
  for (int p = 0; p < 2; ++p) {
    GemmArgs a = mk(r, d, out_rowmajor(p ? G.dAu : G.dAg, kF32, d));  // s dGB^T X, every row
    add(a, colmajor(dGB + p * r, kF32, 2 * r), colmajor(X, dt, d), T, s);
    SLORA_TRY(gemm(a, st));
    float* dBm = p ? G.dBu : G.dBg;
    GemmArgs b0 = mk(Fd, r, out_rowmajor(dBm, kF32, r));  // output rows, every channel
    add(b0, colmajor(p ? dUO : dGO, dt, Fd), colmajor(XA + p * r, kF32, 2 * r, nullptr, out_rows),
        TO, s);
    SLORA_TRY(gemm(b0, st));
    GemmArgs b1 = mk(kk, r, out_rowmajor(dBm, kF32, r, idx, nullptr, 1));  // += ctx, rows S
    add(b1, colmajor(p ? dUC : dGC, dt, kk), colmajor(XA + p * r, kF32, 2 * r, nullptr, ctx_rows),
        TC, s);
    SLORA_TRY(gemm(b1, st));
  }
  return SLORA_OK;
}

// ------------------------------------------------------ linear, bf16, tcgen05
// Same structure as the FFN: the selected slice of W0 is compacted into
// contiguous rows once per call, the large contractions run on tcgen05
// (context rows on the slice, output rows dense), the rank-r projections and
// the LoRA gradients on the skinny tensor-core kernels.
namespace {
SkY ykv(const void* p, int64_t ld, const int32_t* map = nullptr) {
  SkY y; y.ptr = p; y.ld = ld; y.map = map; return y;
}
// rank-r operand of a LoRA contraction; fp32 ones are rounded to one bf16 term
SkR rkv(const void* p, int dtp, int64_t si, int64_t sq, const int32_t* map = nullptr,
        int64_t map_limit = INT64_MAX) {
  SkR rr; rr.ptr = p; rr.dt = dtp; rr.si = si; rr.sq = sq; rr.map = map;
  rr.map_limit = map_limit; rr.terms = dtp == kF32 ? 1 : 0; return rr;
}
int64_t skinny_part_bound(const TokenInfo& ti, int64_t a, int64_t b, int64_t c2, int r) {
  int64_t np = 1;
  for (int64_t M : {ti.T, ti.T_C, ti.T_O})
    for (int64_t K : {a, b, c2}) {
      np = std::max(np, rowdot_part_floats(M, K, r));
      np = std::max(np, coldot_part_floats(M, K, r));
    }
  return np;
}
}  // namespace

slora_status linear_fwd_tc(const LinearDesc& L, const slora_tokens* tok, const void* X_ctx,
                           const void* X_out, void* Y_ctx, void* Y_out, float* XA_save, Arena& ar,
                           bool plan, cudaStream_t st) {
  const TokenInfo& ti = L.ti;
  const int r = L.r;
  const int64_t k = L.k, n = L.n, ni = L.n_idx, T = ti.T, TC = ti.T_C, TO = ti.T_O;
  const float s = L.s;
  const int64_t lr = round8(r), ldi = round8(std::max<int64_t>(ni, 1));
  const bool none = L.side == SLORA_SLICE_NONE, outr = L.side == SLORA_SLICE_OUT_ROWS;
  const int64_t nct = count_tiles(tok, true), nott = count_tiles(tok, false);
  auto bf = [&](int64_t rows, int64_t cols) {
    return static_cast<void*>(ar.take<__nv_bfloat16>(size_t(std::max<int64_t>(rows * cols, 1))));
  };
  int32_t* ctx_rows = ar.take<int32_t>(size_t(std::max<int64_t>(TC, 1)));
  int32_t* out_rows = ar.take<int32_t>(size_t(std::max<int64_t>(TO, 1)));
  int4* ctiles = ar.take<int4>(size_t(std::max<int64_t>(nct, 1)));
  int4* otiles = ar.take<int4>(size_t(std::max<int64_t>(nott, 1)));
  int4* ptiles = ar.take<int4>(size_t((T + 127) / 128));
  float* XA = XA_save ? XA_save : ar.take<float>(size_t(T) * r);
  void* XAb = bf(T, lr);      // s*XA, full rows (NONE, OUT_ROWS)
  void* XAbC = bf(TC, lr);    // s*XA, compact context rows (IN_COLS)
  void* XAbO = bf(TO, lr);    // s*XA, compact output rows (IN_COLS)
  void* Bp = bf(n, lr);       // B padded
  void* BS = bf(ni, lr);      // B[idx] padded (OUT_ROWS)
  void* WS = bf(ni, outr ? k : n);  // rows idx of W (W0 or W0^T)
  void* Xpad = (!none && !outr && ni % 8) ? bf(TC, ldi) : nullptr;  // X_ctx with 16-byte rows
  float* part = ar.take<float>(size_t(skinny_part_bound(ti, k, n, ni, r)));
  const int64_t ncnt = skinny_counter_count(std::max({T, k, n}), std::max({T, k, n}));
  unsigned* rsp = ar.take<unsigned>(size_t(ncnt));
  SkWork sw;
  sw.part = part;
  sw.rsplit = ar.take<__nv_bfloat16>(size_t(skinny_rsplit_elems(std::max({T, k, n}))));
  sw.counters = rsp;
  if (plan) return SLORA_OK;
  SLORA_TRY(arena_fits(ar, "workspace"));

  SLORA_TRY(launch_rowmaps(tok, ti, ctx_rows, out_rows, st, ctiles, otiles, rsp, ncnt));
  SLORA_TRY(gather_pad(L.B, r, nullptr, n, r, Bp, lr, st, n));
  if (none || outr) {
    SkRowOut o;
    o.out1 = XA; o.ld1 = r; o.out2 = XAb; o.ld2 = lr; o.s2 = s;
    SLORA_TRY(rowdot(ykv(X_ctx, k), T, k, rkv(L.A, kBF16, 1, k), r, o, sw, st));
  }
  if (none) {
    SLORA_TRY(make_plain_tiles(ptiles, T, st));
    TcBuilder b(ptiles, (T + 127) / 128, 0, 0, T, n, 0, EPI_STORE);
    b.seg(mat(X_ctx, T, k, k), mat(L.W, n, k, k), B_K, k)
        .seg(mat(XAb, T, r, lr), mat(Bp, n, r, lr), B_K, r)
        .out(Y_ctx, nullptr, nullptr, n);
    return gemm_tc(b.g, st);
  }
  if (outr) {
    SLORA_TRY(gather_rows(L.W, k, L.idx, ni, k, WS, k, st, n));
    SLORA_TRY(gather_pad(L.B, r, L.idx, ni, r, BS, lr, st, n));
    // context rows, output channels S, in one launch with the dense output rows
    TcBuilder bc(ctiles, nct, 0, 1, TC, ni, 0, EPI_STORE);
    bc.seg(mat(X_ctx, T, k, k), mat(WS, ni, k, k), B_K, k)
        .seg(mat(XAb, T, r, lr), mat(BS, ni, r, lr), B_K, r)
        .out(Y_ctx, nullptr, nullptr, ni);
    TcBuilder b(otiles, nott, 0, 1, TO, n, 0, EPI_STORE);  // output rows, dense
    b.seg(mat(X_ctx, T, k, k), mat(L.W, n, k, k), B_K, k)
        .seg(mat(XAb, T, r, lr), mat(Bp, n, r, lr), B_K, r)
        .out(Y_out, nullptr, nullptr, n);
    return gemm_tc_pair(bc.g, b.g, st);
  }
  // IN_COLS: W = W0^T [k x n]; context rows read input channels S only
  const void* Xc = X_ctx;
  int64_t ldxc = ni;
  if (Xpad) {
    SLORA_TRY(gather_pad(X_ctx, ni, nullptr, TC, ni, Xpad, ldi, st, TC));
    Xc = Xpad;
    ldxc = ldi;
  }
  {
    SkRowOut oc;
    oc.out1 = XA; oc.ld1 = r; oc.map1 = ctx_rows; oc.out2 = XAbC; oc.ld2 = lr; oc.s2 = s;
    SLORA_TRY(rowdot(ykv(Xc, ldxc), TC, ni, rkv(L.A, kBF16, 1, k, L.idx, k), r, oc, sw, st));
    SkRowOut oo;
    oo.out1 = XA; oo.ld1 = r; oo.map1 = out_rows; oo.out2 = XAbO; oo.ld2 = lr; oo.s2 = s;
    SLORA_TRY(rowdot(ykv(X_out, k), TO, k, rkv(L.A, kBF16, 1, k), r, oo, sw, st));
  }
  SLORA_TRY(gather_rows(L.W, n, L.idx, ni, n, WS, n, st, k));
  TcBuilder bc(ctiles, nct, 1, 0, TC, n, 0, EPI_STORE);  // context rows, input channels S
  bc.seg(mat(Xc, TC, ni, ldxc), mat(WS, ni, n, n), B_MN, ni)
      .seg(mat(XAbC, TC, r, lr), mat(Bp, n, r, lr), B_K, r)
      .out(Y_ctx, nullptr, nullptr, n);
  TcBuilder b(otiles, nott, 1, 0, TO, n, 0, EPI_STORE);  // output rows, dense
  b.seg(mat(X_out, TO, k, k), mat(L.W, k, n, n), B_MN, k)
      .seg(mat(XAbO, TO, r, lr), mat(Bp, n, r, lr), B_K, r)
      .out(Y_ctx, nullptr, nullptr, n);
  return gemm_tc_pair(bc.g, b.g, st);
}

slora_status linear_bwd_tc(const LinearDesc& L, const slora_tokens* tok, const void* X_ctx,
                           const void* X_out, const float* XA, const void* dY_ctx,
                           const void* dY_out, void* dX_ctx, void* dX_out, float* dA, float* dB,
                           Arena& ar, bool plan, cudaStream_t st) {
  const TokenInfo& ti = L.ti;
  const int r = L.r;
  const int64_t k = L.k, n = L.n, ni = L.n_idx, T = ti.T, TC = ti.T_C, TO = ti.T_O;
  const float s = L.s;
  const int64_t lr = round8(r), ldi = round8(std::max<int64_t>(ni, 1));
  const bool none = L.side == SLORA_SLICE_NONE, outr = L.side == SLORA_SLICE_OUT_ROWS;
  const int64_t nct = count_tiles(tok, true), nott = count_tiles(tok, false);
  auto bf = [&](int64_t rows, int64_t cols) {
    return static_cast<void*>(ar.take<__nv_bfloat16>(size_t(std::max<int64_t>(rows * cols, 1))));
  };
  int32_t* ctx_rows = ar.take<int32_t>(size_t(std::max<int64_t>(TC, 1)));
  int32_t* out_rows = ar.take<int32_t>(size_t(std::max<int64_t>(TO, 1)));
  int4* ctiles = ar.take<int4>(size_t(std::max<int64_t>(nct, 1)));
  int4* otiles = ar.take<int4>(size_t(std::max<int64_t>(nott, 1)));
  int4* ptiles = ar.take<int4>(size_t((T + 127) / 128));
  float* dYB = ar.take<float>(size_t(T) * r);
  void* dYBb = bf(T, lr);     // s*dYB, full rows (NONE, IN_COLS)
  void* dYBbC = bf(TC, lr);   // compact context rows (OUT_ROWS)
  void* dYBbO = bf(TO, lr);   // compact output rows (OUT_ROWS)
  void* WS = bf(ni, outr ? k : n);
  void* AS = bf(ni, lr);      // A[:, idx]^T padded (IN_COLS)
  void* At = bf(k, lr);       // A^T padded (IN_COLS)
  void* dYpad = (outr && ni % 8) ? bf(TC, ldi) : nullptr;
  void* Xpad = (!none && !outr && ni % 8) ? bf(TC, ldi) : nullptr;
  float* part = ar.take<float>(size_t(skinny_part_bound(ti, k, n, ni, r)));
  const int64_t ncnt = skinny_counter_count(std::max({T, k, n}), std::max({T, k, n}));
  unsigned* rsp = ar.take<unsigned>(size_t(ncnt));
  SkWork sw;
  sw.part = part;
  sw.rsplit = ar.take<__nv_bfloat16>(size_t(skinny_rsplit_elems(std::max({T, k, n}))));
  sw.counters = rsp;
  // The batched form (NONE, and OUT_ROWS with context and output rows): every
  // rank operand known up front split in one launch, and the token-summed
  // contractions (dA over X, dB over dY by row kind) in one launch; the
  // context rows' dB part lands in SB and is added onto rows idx of dB.
  const bool batched = (none && T > 0) || (outr && TC > 0 && TO > 0 && ni > 0);
  auto rsbuf = [&](int64_t I) {
    return static_cast<void*>(ar.take<__nv_bfloat16>(size_t(skinny_rsplit_elems(I))));
  };
  void* rsB0 = nullptr;  // B for the dYB rowdot(s): NONE: every row; OUT_ROWS: rows idx
  void* rsB1 = nullptr;  // OUT_ROWS: B for the output rows
  void* rsX0 = nullptr;  // XA: NONE every row; OUT_ROWS output rows
  void* rsX1 = nullptr;  // OUT_ROWS: XA of the context rows
  void* rsDY = nullptr;  // dYB (for dA)
  float* SB = nullptr;
  SkColJob bj[3];
  int nbj = 0;
  auto prepared = [&](void* rs) {
    SkWork w = sw;
    w.rsplit = rs;
    w.prepared = true;
    return w;
  };
  auto cjob = [&](const void* Y, int64_t ld, int64_t M, int64_t K, const SkR& Rr, void* rs_,
                  float* o, int64_t ldo, int trans) {
    SkColJob j;
    j.Y = ykv(Y, ld); j.M = M; j.K = K; j.R = Rr; j.c = r; j.rs = rs_;
    j.o.out = o; j.o.ldo = ldo; j.o.trans = trans; j.o.scale = s;
    return j;
  };
  if (batched) {
    rsB0 = rsbuf(none ? n : ni);
    rsX0 = rsbuf(none ? T : TO);
    rsDY = rsbuf(T);
    if (outr) {
      rsB1 = rsbuf(n);
      rsX1 = rsbuf(TC);
      SB = ar.take<float>(size_t(ni) * r);
    }
    const void* dYc0 = dYpad ? dYpad : dY_ctx;
    const int64_t lddc0 = dYpad ? ldi : ni;
    if (none) {
      bj[nbj++] = cjob(X_ctx, k, T, k, rkv(dYB, kF32, r, 1), rsDY, dA, k, 1);
      bj[nbj++] = cjob(dY_ctx, n, T, n, rkv(XA, kF32, r, 1), rsX0, dB, r, 0);
    } else {
      bj[nbj++] = cjob(X_ctx, k, T, k, rkv(dYB, kF32, r, 1), rsDY, dA, k, 1);
      bj[nbj++] = cjob(dY_out, n, TO, n, rkv(XA, kF32, r, 1, out_rows), rsX0, dB, r, 0);
      bj[nbj++] = cjob(dYc0, lddc0, TC, ni, rkv(XA, kF32, r, 1, ctx_rows), rsX1, SB, r, 0);
    }
  }
  float* bpart = nullptr;
  unsigned* bcnt = nullptr;
  if (batched) {
    bpart = ar.take<float>(size_t(coldot_batch_part_floats(bj, nbj)));
    bcnt = ar.take<unsigned>(size_t(coldot_batch_counter_count(bj, nbj)));
  }
  if (plan) return SLORA_OK;
  SLORA_TRY(arena_fits(ar, "workspace"));

  SLORA_TRY(launch_rowmaps(tok, ti, ctx_rows, out_rows, st, ctiles, otiles, rsp, ncnt, bcnt,
                           bcnt ? coldot_batch_counter_count(bj, nbj) : 0));
  if (batched && none) {
    const SkPrep jobs[2] = {{rkv(L.B, kBF16, r, 1), r, n, rsB0}, {rkv(XA, kF32, r, 1), r, T, rsX0}};
    SLORA_TRY(prep_r_batch(jobs, 2, st));
    SkRowOut o;
    o.out1 = dYB; o.ld1 = r; o.out2 = dYBb; o.ld2 = lr; o.s2 = s;
    SLORA_TRY(rowdot(ykv(dY_ctx, n), T, n, rkv(L.B, kBF16, r, 1), r, o, prepared(rsB0), st));
    SLORA_TRY(make_plain_tiles(ptiles, T, st));
    TcBuilder b(ptiles, (T + 127) / 128, 0, 0, T, k, 0, EPI_STORE);
    b.seg(mat(dY_ctx, T, n, n), mat(L.W, n, k, k), B_MN, n)
        .seg(mat(dYBb, T, r, lr), mat(L.A, r, k, k), B_MN, r)
        .out(dX_ctx, nullptr, nullptr, k);
    SLORA_TRY(gemm_tc(b.g, st));
    const SkPrep jd = {rkv(dYB, kF32, r, 1), r, T, rsDY};
    SLORA_TRY(prep_r_batch(&jd, 1, st));
    return coldot_batch(bj, nbj, bpart, bcnt, st);
  }
  if (batched && outr) {
    const void* dYc = dY_ctx;
    int64_t lddc = ni;
    if (dYpad) {
      SLORA_TRY(gather_pad(dY_ctx, ni, nullptr, TC, ni, dYpad, ldi, st, TC));
      dYc = dYpad;
      lddc = ldi;
    }
    const SkPrep jobs[4] = {{rkv(L.B, kBF16, r, 1, L.idx, n), r, ni, rsB0},
                            {rkv(L.B, kBF16, r, 1), r, n, rsB1},
                            {rkv(XA, kF32, r, 1, out_rows), r, TO, rsX0},
                            {rkv(XA, kF32, r, 1, ctx_rows), r, TC, rsX1}};
    SLORA_TRY(prep_r_batch(jobs, 4, st));
    SkRowOut oc;
    oc.out1 = dYB; oc.ld1 = r; oc.map1 = ctx_rows; oc.out2 = dYBbC; oc.ld2 = lr; oc.s2 = s;
    SLORA_TRY(rowdot(ykv(dYc, lddc), TC, ni, rkv(L.B, kBF16, r, 1, L.idx, n), r, oc,
                     prepared(rsB0), st));
    SkRowOut oo;
    oo.out1 = dYB; oo.ld1 = r; oo.map1 = out_rows; oo.out2 = dYBbO; oo.ld2 = lr; oo.s2 = s;
    SLORA_TRY(rowdot(ykv(dY_out, n), TO, n, rkv(L.B, kBF16, r, 1), r, oo, prepared(rsB1), st));
    SLORA_TRY(gather_rows(L.W, k, L.idx, ni, k, WS, k, st, n));
    {  // dX, context rows: dY_C W0[S] + s dYB_C A; output rows dense; one launch
      TcBuilder bc(ctiles, nct, 1, 0, TC, k, 0, EPI_STORE);
      bc.seg(mat(dYc, TC, ni, lddc), mat(WS, ni, k, k), B_MN, ni)
          .seg(mat(dYBbC, TC, r, lr), mat(L.A, r, k, k), B_MN, r)
          .out(dX_ctx, nullptr, nullptr, k);
      TcBuilder b(otiles, nott, 1, 0, TO, k, 0, EPI_STORE);
      b.seg(mat(dY_out, TO, n, n), mat(L.W, n, k, k), B_MN, n)
          .seg(mat(dYBbO, TO, r, lr), mat(L.A, r, k, k), B_MN, r)
          .out(dX_ctx, nullptr, nullptr, k);
      SLORA_TRY(gemm_tc_pair(bc.g, b.g, st));
    }
    const SkPrep jd = {rkv(dYB, kF32, r, 1), r, T, rsDY};
    SLORA_TRY(prep_r_batch(&jd, 1, st));
    SLORA_TRY(coldot_batch(bj, nbj, bpart, bcnt, st));
    ScatterAddJob sj;
    sj.dst = dB; sj.ld_dst = r; sj.src = SB; sj.ld_src = r; sj.trans = 0;
    return scatter_add_cols(&sj, 1, L.idx, ni, r, n, st);
  }
  if (none) {
    SkRowOut o;
    o.out1 = dYB; o.ld1 = r; o.out2 = dYBb; o.ld2 = lr; o.s2 = s;
    SLORA_TRY(rowdot(ykv(dY_ctx, n), T, n, rkv(L.B, kBF16, r, 1), r, o, sw, st));
    SLORA_TRY(make_plain_tiles(ptiles, T, st));
    TcBuilder b(ptiles, (T + 127) / 128, 0, 0, T, k, 0, EPI_STORE);
    b.seg(mat(dY_ctx, T, n, n), mat(L.W, n, k, k), B_MN, n)
        .seg(mat(dYBb, T, r, lr), mat(L.A, r, k, k), B_MN, r)
        .out(dX_ctx, nullptr, nullptr, k);
    SLORA_TRY(gemm_tc(b.g, st));
    SkColOut ca;
    ca.out = dA; ca.ldo = k; ca.trans = 1; ca.scale = s;
    SLORA_TRY(coldot(ykv(X_ctx, k), T, k, rkv(dYB, kF32, r, 1), r, ca, sw, st));
    SkColOut cb;
    cb.out = dB; cb.ldo = r; cb.scale = s;
    return coldot(ykv(dY_ctx, n), T, n, rkv(XA, kF32, r, 1), r, cb, sw, st);
  }
  if (outr) {
    const void* dYc = dY_ctx;
    int64_t lddc = ni;
    if (dYpad) {
      SLORA_TRY(gather_pad(dY_ctx, ni, nullptr, TC, ni, dYpad, ldi, st, TC));
      dYc = dYpad;
      lddc = ldi;
    }
    {  // dYB = dY B on the rows' channels; dB = s dY^T XA (output rows first, then += S rows)
      SkRowOut oc;
      oc.out1 = dYB; oc.ld1 = r; oc.map1 = ctx_rows; oc.out2 = dYBbC; oc.ld2 = lr; oc.s2 = s;
      SLORA_TRY(rowdot(ykv(dYc, lddc), TC, ni, rkv(L.B, kBF16, r, 1, L.idx, n), r, oc, sw,
                       st));
      SkRowOut oo;
      oo.out1 = dYB; oo.ld1 = r; oo.map1 = out_rows; oo.out2 = dYBbO; oo.ld2 = lr; oo.s2 = s;
      SLORA_TRY(rowdot(ykv(dY_out, n), TO, n, rkv(L.B, kBF16, r, 1), r, oo, sw, st));
      SkColOut bo;
      bo.out = dB; bo.ldo = r; bo.scale = s;
      SLORA_TRY(coldot(ykv(dY_out, n), TO, n, rkv(XA, kF32, r, 1, out_rows), r, bo, sw,
                       st));
      SkColOut bc = bo;
      bc.kmap = L.idx; bc.kmap_limit = n; bc.accumulate = 1;
      SLORA_TRY(coldot(ykv(dYc, lddc), TC, ni, rkv(XA, kF32, r, 1, ctx_rows), r, bc, sw,
                       st));
    }
    SLORA_TRY(gather_rows(L.W, k, L.idx, ni, k, WS, k, st, n));
    {  // dX, context rows: dY_C W0[S] + s dYB_C A; output rows dense; one launch
      TcBuilder bc(ctiles, nct, 1, 0, TC, k, 0, EPI_STORE);
      bc.seg(mat(dYc, TC, ni, lddc), mat(WS, ni, k, k), B_MN, ni)
          .seg(mat(dYBbC, TC, r, lr), mat(L.A, r, k, k), B_MN, r)
          .out(dX_ctx, nullptr, nullptr, k);
      TcBuilder b(otiles, nott, 1, 0, TO, k, 0, EPI_STORE);
      b.seg(mat(dY_out, TO, n, n), mat(L.W, n, k, k), B_MN, n)
          .seg(mat(dYBbO, TO, r, lr), mat(L.A, r, k, k), B_MN, r)
          .out(dX_ctx, nullptr, nullptr, k);
      SLORA_TRY(gemm_tc_pair(bc.g, b.g, st));
    }
    SkColOut ca;  // dA = s dYB^T X over every row
    ca.out = dA; ca.ldo = k; ca.trans = 1; ca.scale = s;
    return coldot(ykv(X_ctx, k), T, k, rkv(dYB, kF32, r, 1), r, ca, sw, st);
  }
  // IN_COLS: W = W0^T [k x n]; dY is the full T x n gradient
  const void* Xc = X_ctx;
  int64_t ldxc = ni;
  if (Xpad) {
    SLORA_TRY(gather_pad(X_ctx, ni, nullptr, TC, ni, Xpad, ldi, st, TC));
    Xc = Xpad;
    ldxc = ldi;
  }
  {
    SkRowOut o;
    o.out1 = dYB; o.ld1 = r; o.out2 = dYBb; o.ld2 = lr; o.s2 = s;
    SLORA_TRY(rowdot(ykv(dY_ctx, n), T, n, rkv(L.B, kBF16, r, 1), r, o, sw, st));
  }
  SLORA_TRY(gather_rows(L.W, n, L.idx, ni, n, WS, n, st, k));
  SLORA_TRY(transpose_rows(L.A, r, k, L.idx, ni, lr, AS, st));
  SLORA_TRY(transpose_rows(L.A, r, k, nullptr, k, lr, At, st));
  {  // dX_ctx = dY_C W0[:, S] + s dYB_C A[:, S]; dX_out dense; one launch
    TcBuilder bc(ctiles, nct, 0, 1, TC, ni, 0, EPI_STORE);
    bc.seg(mat(dY_ctx, T, n, n), mat(WS, ni, n, n), B_K, n)
        .seg(mat(dYBb, T, r, lr), mat(AS, ni, r, lr), B_K, r)
        .out(dX_ctx, nullptr, nullptr, ni);
    TcBuilder b(otiles, nott, 0, 1, TO, k, 0, EPI_STORE);
    b.seg(mat(dY_ctx, T, n, n), mat(L.W, k, n, n), B_K, n)
        .seg(mat(dYBb, T, r, lr), mat(At, k, r, lr), B_K, r)
        .out(dX_out, nullptr, nullptr, k);
    SLORA_TRY(gemm_tc_pair(bc.g, b.g, st));
  }
  {  // dA: output rows over every column, then += context rows on columns S
    SkColOut ao;
    ao.out = dA; ao.ldo = k; ao.trans = 1; ao.scale = s;
    SLORA_TRY(coldot(ykv(X_out, k), TO, k, rkv(dYB, kF32, r, 1, out_rows), r, ao, sw, st));
    SkColOut ac = ao;
    ac.kmap = L.idx; ac.kmap_limit = k; ac.accumulate = 1;
    SLORA_TRY(coldot(ykv(Xc, ldxc), TC, ni, rkv(dYB, kF32, r, 1, ctx_rows), r, ac, sw, st));
  }
  SkColOut cb;  // dB = s dY^T XA over every row
  cb.out = dB; cb.ldo = r; cb.scale = s;
  return coldot(ykv(dY_ctx, n), T, n, rkv(XA, kF32, r, 1), r, cb, sw, st);
}

}  // namespace slora
