// Attention core and rotary packing of a decoder layer (see attention.cu).
#pragma once

#include "common.cuh"

namespace slora {

// Rotary packing.  Forward (backward == false): out [T x n] bf16 = rotated
// full-width rows of Y [T x n] (idx == nullptr) or of the compact context
// rows Yc [T_C x n_idx] (channels idx, zeros elsewhere) and the dense output
// rows Yo [T_O x n].  Backward: the transpose on the fp32 gradient G [T x n],
// written to out [T x n] (idx == nullptr) or to out_c [T_C x n_idx] (kept
// channels) and out_o [T_O x n].  hd is the head width (n = heads * hd).
slora_status rope_run(bool backward, const void* Y, const void* Yc, const void* Yo,
                      const float* G, const int32_t* idx, int n_idx, const slora_tokens* tok,
                      const TokenInfo& ti, int n, int hd, double base, void* out, void* out_c,
                      void* out_o, Arena& ar, bool plan, cudaStream_t st);

// Causal attention within each sequence, grouped key/value heads, hd 64 or 128,
// bf16.  lse: [batch][H][seq] fp32 natural log-sum-exp of the scaled scores.
slora_status attention_fwd_run(const void* Q, const void* K, const void* V, const TokenInfo& ti,
                               int H, int KV, int hd, void* O, float* lse, cudaStream_t st);
// The tcgen05 forward (attention_tc.cu): head width 128, 16-byte aligned Q,
// K, V, O; attention_fwd_run takes it whenever attention_fwd_tc_ok holds.
bool attention_fwd_tc_ok(const void* Q, const void* K, const void* V, const void* O, int hd);
slora_status attention_fwd_tc_run(const void* Q, const void* K, const void* V, const TokenInfo& ti,
                                  int H, int KV, void* O, float* lse, cudaStream_t st);
// The tcgen05 backward (attention_tc.cu): a dK/dV kernel and a dQ kernel,
// each output row written once (dQ needs no zeroing); D = rowsum(dO * O)
// [batch][H][seq] computed beforehand.  attention_bwd_run takes it whenever
// attention_bwd_tc_ok holds.
bool attention_bwd_tc_ok(const void* Q, const void* K, const void* V, const void* dO,
                         const void* dQ, const void* dK, const void* dV, int hd);
slora_status attention_bwd_tc_run(const void* Q, const void* K, const void* V, const void* dO,
                                  const float* lse, const float* D, const TokenInfo& ti, int H,
                                  int KV, float* dQ, float* dK, void* dV, double flops_per_product,
                                  cudaStream_t st);
// Raised when a tcgen05 attention kernel's bounded wait ran out.
slora_status attn_check_error(bool clear);
// dQ [T x H hd] and dK [T x KV hd] fp32, dV [T x KV hd] bf16 (all written).
slora_status attention_bwd_run(const void* Q, const void* K, const void* V, const void* O,
                               const float* lse, const void* dO, const TokenInfo& ti, int H,
                               int KV, int hd, float* dQ, float* dK, void* dV, Arena& ar,
                               bool plan, cudaStream_t st);

// RMS normalisation with a frozen gain (norm.cu).  Forward: h = X + A (A may
// be null: h = X, not written when Hout is null), N = h / rms(h) * g with
// rms = sqrt(mean(h^2) + eps), rstd = 1 / rms; N may be null (only the sum).
// Backward: dX = dRes + rstd g dN - h rstd^3 mean(h g dN), dN the sum of the
// non-null dN0..dN2 (dRes may be null).
slora_status rmsnorm_fwd_run(const void* X, const void* A, const void* g, int64_t T, int64_t d,
                             float eps, void* Hout, void* N, float* rstd, cudaStream_t st);
slora_status rmsnorm_bwd_run(const void* Hin, const float* rstd, const void* g, const void* dN0,
                             const void* dN1, const void* dN2, const void* dRes, int64_t T,
                             int64_t d, void* dX, cudaStream_t st);

}  // namespace slora
