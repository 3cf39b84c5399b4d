// Generic gathered GEMM on CUDA cores (fp32 FMA):
//   C(m, n) = beta * C(m, n) + sum_s alpha_s * sum_k A_s(m, k) * B_s(n, k)
// Every operand is addressed through strides and optional int32 gathers, so
// one kernel covers the sliced shapes of the sparse LoRA linear: row slices
// (output channels), column slices (input channels), context/output row maps,
// transposed views for the LoRA gradients.  It is the exact-parity fp32 path
// and the small-shape workhorse; large bf16 contractions go to the tcgen05
// kernel instead.
#pragma once

#include "common.cuh"

namespace slora {

// element (i, k) = ptr[(gi ? gi[i] : i) * si + (gk ? gk[k] : k) * sk]
struct MatRef {
  const void* ptr = nullptr;
  int dt = kF32;
  int64_t si = 0, sk = 0;
  const int32_t* gi = nullptr;
  const int32_t* gk = nullptr;
};

struct Seg {
  MatRef a, b;
  int64_t K = 0;
  float alpha = 1.0f;
};

// C(m, n) lives at ptr[(gm ? gm[m] : m) * ldc + (gn ? gn[n] : n)]
struct OutRef {
  void* ptr = nullptr;
  int dt = kF32;
  int64_t ldc = 0;
  const int32_t* gm = nullptr;
  const int32_t* gn = nullptr;
  int accumulate = 0;  // 1: C += result (read-modify-write in fp32)
  // optional second copy: bf16(scale2 * C(m, n)) at ptr2[(gm2 ? gm2[m] : m) * ld2 + n]
  void* ptr2 = nullptr;
  int64_t ld2 = 0;
  const int32_t* gm2 = nullptr;
  float scale2 = 1.0f;
};

constexpr int kMaxSegs = 4;
struct GemmArgs {
  int64_t M = 0, N = 0;
  int nseg = 0;
  Seg seg[kMaxSegs];
  OutRef c;
};

// Helpers to describe common views.
inline MatRef rowmajor(const void* p, int dt, int64_t ld, const int32_t* gi = nullptr,
                       const int32_t* gk = nullptr) {
  MatRef r;
  r.ptr = p; r.dt = dt; r.si = ld; r.sk = 1; r.gi = gi; r.gk = gk;
  return r;
}
// (i, k) = ptr[k * ld + i]: the transpose of a row-major [K x ld] matrix.
inline MatRef colmajor(const void* p, int dt, int64_t ld, const int32_t* gi = nullptr,
                       const int32_t* gk = nullptr) {
  MatRef r;
  r.ptr = p; r.dt = dt; r.si = 1; r.sk = ld; r.gi = gi; r.gk = gk;
  return r;
}
inline OutRef out_rowmajor(void* p, int dt, int64_t ldc, const int32_t* gm = nullptr,
                           const int32_t* gn = nullptr, int acc = 0) {
  OutRef o;
  o.ptr = p; o.dt = dt; o.ldc = ldc; o.gm = gm; o.gn = gn; o.accumulate = acc;
  return o;
}

inline OutRef with_bf16_copy(OutRef o, void* p2, int64_t ld2, float scale2,
                             const int32_t* gm2 = nullptr) {
  o.ptr2 = p2; o.ld2 = ld2; o.scale2 = scale2; o.gm2 = gm2;
  return o;
}

slora_status gemm_simt(const GemmArgs& g, cudaStream_t st);

}  // namespace slora
