// C ABI of the decoder-layer pieces around the sparse linears: rotary
// packing, the attention core and RMS normalisation.  Validation happens
// before any launch; the kernels are in attention.cu and norm.cu.
#include <cmath>

#include "attention.cuh"

using namespace slora;

namespace {

#define LREQ(p)                                                                          \
  do {                                                                                   \
    if (!(p)) SLORA_FAIL(SLORA_ERR_INVALID_ARG, "%s: required pointer %s is NULL", fn, #p); \
    if (!aligned16(p)) SLORA_FAIL(SLORA_ERR_ALIGN, "%s: %s is not 16-byte aligned", fn, #p); \
  } while (0)
#define LOPT(p)                                                                          \
  do {                                                                                   \
    if ((p) && !aligned16(p)) SLORA_FAIL(SLORA_ERR_ALIGN, "%s: %s is not 16-byte aligned", fn, #p); \
  } while (0)

slora_status check_bf16(const char* fn, slora_dtype dt) {
  if (dt == SLORA_F32)
    SLORA_FAIL(SLORA_ERR_UNSUPPORTED, "%s: the decoder-layer kernels run in bf16 only", fn);
  if (dt != SLORA_BF16) SLORA_FAIL(SLORA_ERR_INVALID_ARG, "%s: unknown dtype %d", fn, int(dt));
  return SLORA_OK;
}

slora_status check_heads(const char* fn, int heads, int kv_heads, int head_dim) {
  if (head_dim != 64 && head_dim != 128)
    SLORA_FAIL(SLORA_ERR_SHAPE, "%s: head_dim %d must be 64 or 128", fn, head_dim);
  if (heads < 1 || kv_heads < 1 || heads % kv_heads || heads > 65535)
    SLORA_FAIL(SLORA_ERR_SHAPE, "%s: heads %d must be a positive multiple of kv_heads %d", fn,
               heads, kv_heads);
  return SLORA_OK;
}

slora_status ws_none(const char* fn, void* ws, size_t* ws_bytes) {
  if (!ws_bytes) SLORA_FAIL(SLORA_ERR_INVALID_ARG, "%s: ws_bytes is NULL", fn);
  if (!ws) *ws_bytes = 0;
  return SLORA_OK;
}

slora_status ws_finish(const char* fn, const Arena& plan, void* ws, size_t* ws_bytes) {
  if (!ws_bytes) SLORA_FAIL(SLORA_ERR_INVALID_ARG, "%s: ws_bytes is NULL", fn);
  if (!ws) {
    *ws_bytes = plan.used;
    return SLORA_OK;
  }
  if (*ws_bytes < plan.used)
    SLORA_FAIL(SLORA_ERR_WORKSPACE, "%s: workspace of %zu bytes, %zu needed", fn, *ws_bytes,
               plan.used);
  return SLORA_OK;
}

slora_status rope_common(const char* fn, bool backward, slora_dtype dt, const slora_tokens* tok,
                         int64_t n, int head_dim, double base, const int32_t* idx, int32_t n_idx,
                         const void* Y, const void* Yc, const void* Yo, const float* G, void* out,
                         void* out_c, void* out_o, void* ws, size_t* ws_bytes,
                         slora_stream_t stream) {
  SLORA_TRY(check_bf16(fn, dt));
  SLORA_TRY(check_heads(fn, 1, 1, head_dim));
  if (n <= 0 || n % head_dim || n > (int64_t(1) << 30))
    SLORA_FAIL(SLORA_ERR_SHAPE, "%s: n=%lld must be a positive multiple of head_dim", fn,
               (long long)n);
  if (!(base > 1.0) || !std::isfinite(base))
    SLORA_FAIL(SLORA_ERR_INVALID_ARG, "%s: rope_base %g must be a finite value > 1", fn, base);
  TokenInfo ti;
  SLORA_TRY(parse_tokens(tok, &ti));
  if (idx) {
    if (n_idx < 0 || n_idx > n)
      SLORA_FAIL(SLORA_ERR_SHAPE, "%s: n_idx=%d outside [0, n]", fn, n_idx);
    LREQ(idx);
    if (backward) {
      if (ti.T_C > 0 && n_idx > 0) LREQ(out_c);
      if (ti.T_O > 0) LREQ(out_o);
    } else {
      if (ti.T_C > 0 && n_idx > 0) LREQ(Yc);
      if (ti.T_O > 0) LREQ(Yo);
    }
    LOPT(out_c); LOPT(out_o); LOPT(Yc); LOPT(Yo);
  } else {
    if (backward) LREQ(out); else LREQ(Y);
  }
  if (backward) LREQ(G); else LREQ(out);
  LOPT(ws);
  Arena plan;
  SLORA_TRY(rope_run(backward, Y, Yc, Yo, G, idx, n_idx, tok, ti, int(n), head_dim, base, out,
                     out_c, out_o, plan, true, nullptr));
  const bool query = ws == nullptr;
  SLORA_TRY(ws_finish(fn, plan, ws, ws_bytes));
  if (query) return SLORA_OK;
  SLORA_TRY(check_device());
  Arena ar;
  ar.base = static_cast<char*>(ws);
  ar.cap = *ws_bytes;
  return rope_run(backward, Y, Yc, Yo, G, idx, n_idx, tok, ti, int(n), head_dim, base, out, out_c,
                  out_o, ar, false, static_cast<cudaStream_t>(stream));
}

}  // namespace

extern "C" slora_status slora_rope_pack(slora_dtype dt, const slora_tokens* tok, int64_t n,
                                        int head_dim, double rope_base, const int32_t* idx,
                                        int32_t n_idx, const void* Y, const void* Y_ctx,
                                        const void* Y_out, void* Y_rot, void* ws,
                                        size_t* ws_bytes, slora_stream_t stream) {
  clear_error();
  return rope_common("slora_rope_pack", false, dt, tok, n, head_dim, rope_base, idx, n_idx, Y,
                     Y_ctx, Y_out, nullptr, Y_rot, nullptr, nullptr, ws, ws_bytes, stream);
}

extern "C" slora_status slora_rope_unpack(slora_dtype dt, const slora_tokens* tok, int64_t n,
                                          int head_dim, double rope_base, const int32_t* idx,
                                          int32_t n_idx, const float* G, void* dY, void* dY_ctx,
                                          void* dY_out, void* ws, size_t* ws_bytes,
                                          slora_stream_t stream) {
  clear_error();
  return rope_common("slora_rope_unpack", true, dt, tok, n, head_dim, rope_base, idx, n_idx,
                     nullptr, nullptr, nullptr, G, dY, dY_ctx, dY_out, ws, ws_bytes, stream);
}

extern "C" slora_status slora_attention_fwd(slora_dtype dt, const slora_tokens* tok, int heads,
                                            int kv_heads, int head_dim, const void* Q,
                                            const void* K, const void* V, void* O, float* lse,
                                            void* ws, size_t* ws_bytes, slora_stream_t stream) {
  const char* fn = "slora_attention_fwd";
  clear_error();
  SLORA_TRY(check_bf16(fn, dt));
  SLORA_TRY(check_heads(fn, heads, kv_heads, head_dim));
  LREQ(Q); LREQ(K); LREQ(V); LREQ(O); LREQ(lse);
  TokenInfo ti;
  SLORA_TRY(parse_tokens(tok, &ti));
  if (ti.batch > 65535) SLORA_FAIL(SLORA_ERR_SHAPE, "%s: batch %d above 65535", fn, ti.batch);
  const bool query = ws == nullptr;
  SLORA_TRY(ws_none(fn, ws, ws_bytes));
  if (query) return SLORA_OK;
  SLORA_TRY(check_device());
  return attention_fwd_run(Q, K, V, ti, heads, kv_heads, head_dim, O, lse,
                           static_cast<cudaStream_t>(stream));
}

extern "C" slora_status slora_attention_bwd(slora_dtype dt, const slora_tokens* tok, int heads,
                                            int kv_heads, int head_dim, const void* Q,
                                            const void* K, const void* V, const void* O,
                                            const float* lse, const void* dO, float* dQ,
                                            float* dK, void* dV, void* ws, size_t* ws_bytes,
                                            slora_stream_t stream) {
  const char* fn = "slora_attention_bwd";
  clear_error();
  SLORA_TRY(check_bf16(fn, dt));
  SLORA_TRY(check_heads(fn, heads, kv_heads, head_dim));
  LREQ(Q); LREQ(K); LREQ(V); LREQ(O); LREQ(lse); LREQ(dO); LREQ(dQ); LREQ(dK); LREQ(dV);
  LOPT(ws);
  TokenInfo ti;
  SLORA_TRY(parse_tokens(tok, &ti));
  if (ti.batch > 65535) SLORA_FAIL(SLORA_ERR_SHAPE, "%s: batch %d above 65535", fn, ti.batch);
  Arena plan;
  SLORA_TRY(attention_bwd_run(Q, K, V, O, lse, dO, ti, heads, kv_heads, head_dim, dQ, dK, dV,
                              plan, true, nullptr));
  const bool query = ws == nullptr;
  SLORA_TRY(ws_finish(fn, plan, ws, ws_bytes));
  if (query) return SLORA_OK;
  SLORA_TRY(check_device());
  Arena ar;
  ar.base = static_cast<char*>(ws);
  ar.cap = *ws_bytes;
  return attention_bwd_run(Q, K, V, O, lse, dO, ti, heads, kv_heads, head_dim, dQ, dK, dV, ar,
                           false, static_cast<cudaStream_t>(stream));
}

extern "C" slora_status slora_rmsnorm_fwd(slora_dtype dt, int64_t T, int64_t d, float eps,
                                          const void* X, const void* A, const void* g, void* H,
                                          void* N, float* rstd, void* ws, size_t* ws_bytes,
                                          slora_stream_t stream) {
  const char* fn = "slora_rmsnorm_fwd";
  clear_error();
  SLORA_TRY(check_bf16(fn, dt));
  if (T < 0 || d <= 0 || d % 8 || d > (int64_t(1) << 24))
    SLORA_FAIL(SLORA_ERR_SHAPE, "%s: T=%lld, d=%lld (d a positive multiple of 8)", fn,
               (long long)T, (long long)d);
  if (!(eps >= 0.f) || !std::isfinite(eps))
    SLORA_FAIL(SLORA_ERR_INVALID_ARG, "%s: eps %g", fn, double(eps));
  LREQ(X); LREQ(g); LOPT(A); LOPT(H); LOPT(N); LOPT(rstd);
  if (A && !H && !N)
    SLORA_FAIL(SLORA_ERR_INVALID_ARG, "%s: with A, at least one of H and N is required", fn);
  if (!A && !N) SLORA_FAIL(SLORA_ERR_INVALID_ARG, "%s: N is required when A is NULL", fn);
  const bool query = ws == nullptr;
  SLORA_TRY(ws_none(fn, ws, ws_bytes));
  if (query) return SLORA_OK;
  SLORA_TRY(check_device());
  return rmsnorm_fwd_run(X, A, g, T, d, eps, H, N, rstd, static_cast<cudaStream_t>(stream));
}

extern "C" slora_status slora_rmsnorm_bwd(slora_dtype dt, int64_t T, int64_t d, const void* H,
                                          const float* rstd, const void* g, const void* dN0,
                                          const void* dN1, const void* dN2, const void* dRes,
                                          void* dX, void* ws, size_t* ws_bytes,
                                          slora_stream_t stream) {
  const char* fn = "slora_rmsnorm_bwd";
  clear_error();
  SLORA_TRY(check_bf16(fn, dt));
  if (T < 0 || d <= 0 || d % 8 || d > (int64_t(1) << 24))
    SLORA_FAIL(SLORA_ERR_SHAPE, "%s: T=%lld, d=%lld (d a positive multiple of 8)", fn,
               (long long)T, (long long)d);
  LREQ(H); LREQ(rstd); LREQ(g); LREQ(dN0); LREQ(dX); LOPT(dN1); LOPT(dN2); LOPT(dRes);
  const bool query = ws == nullptr;
  SLORA_TRY(ws_none(fn, ws, ws_bytes));
  if (query) return SLORA_OK;
  SLORA_TRY(check_device());
  return rmsnorm_bwd_run(H, rstd, g, dN0, dN1, dN2, dRes, T, d, dX,
                         static_cast<cudaStream_t>(stream));
}
