// Skinny contractions of the LoRA branch and of the estimator: one large
// bf16 matrix Y [M x K] (activations or gradients, M = tokens) against a
// rank-sized matrix with c <= 64 columns.  They are bound by the HBM stream of
// Y, so they run on mma.sync bf16 tensor-core fragments inside CUDA-core
// tiles (the tcgen05 tile shape would waste the machine on N = c), with fp32
// operands split into three bf16 terms (hi + mid + lo, relative residual
// 2^-24) where the result must be fp32-accurate (the estimator's projection),
// or rounded to one bf16 term (the LoRA gradients, whose forward GEMMs use the
// same rank-r operands in bf16).
//
//   rowdot:  P1[m, q] = sum_k Y[m, k] R1(k, q)      (e.g. X A^T, h A_d^T, dOut B_d)
//   coldot:  P2[k, q] = sum_m Y[m, k] R2(m, q)      (LoRA gradients, sums over tokens)
//
// The rank-sized operand is split into bf16 terms once per call (a small
// pre-pass into the rsplit workspace); the main kernel streams Y through a
// multi-stage cp.async pipeline and writes fixed-order partial sums (K or M
// split across blocks); the last block of each output block to finish (an
// atomic ticket) reduces them in order, so results are bit-reproducible.
#pragma once

#include "common.cuh"

namespace slora {

struct SkY {  // Y(m, k) = ptr[(map ? map[m] : m) * ld + k], bf16, valid k < K
  const void* ptr = nullptr;
  int64_t ld = 0;
  const int32_t* map = nullptr;
};

struct SkR {  // R(i, q) = ptr[(map ? map[i] : i) * si + q * sq], fp32 or bf16
  const void* ptr = nullptr;
  int dt = kF32;
  // bf16 terms an fp32 operand is split into: 0 = three (fp32-accurate
  // products, ~2^-24 relative), 1 = one (the operand rounded to bf16, as the
  // GEMMs' LoRA segments use it); bf16 operands always take one
  int terms = 0;
  int64_t si = 0, sq = 0;
  const int32_t* map = nullptr;
  int64_t map_limit = INT64_MAX;  // map values outside [0, map_limit) read as zero
  // columns q >= qsplit come from a second source: ptr_b[i' * si_b + (q - qsplit) * sq_b]
  int qsplit = 1 << 30;
  const void* ptr_b = nullptr;
  int dt_b = kF32;
  int64_t si_b = 0, sq_b = 0;
};

// rowdot output: out1 fp32 at [(map1 ? map1[m] : m) * ld1 + off1 + q] and,
// optionally, out2 bf16 at [(map2 ? map2[m] : m) * ld2 + off2 + q] scaled by s2.
// Columns q are split at qsplit: q < qsplit go to (off1, off2), q >= qsplit
// to (off1b + q - qsplit) of out1b / (off2b + q - qsplit) of out2b.
struct SkRowOut {
  float* out1 = nullptr;
  int64_t ld1 = 0, off1 = 0;
  const int32_t* map1 = nullptr;
  void* out2 = nullptr;
  int64_t ld2 = 0, off2 = 0;
  const int32_t* map2 = nullptr;
  float s2 = 1.0f;
  int qsplit = 64;             // columns >= qsplit go to the second destination
  float* out1b = nullptr;      // fp32 second destination (may be null)
  int64_t ld1b = 0, off1b = 0;
  const int32_t* map1b = nullptr;
};

// coldot output: v = scale * P2[k, q]; with kmap, column k is kmap[k].
// dest = trans ? out[q' * ldo + k'] : out[k' * ldo + q'] where q' = q (or
// q - qsplit into out_b); accumulate adds to the existing value.
struct SkColOut {
  float* out = nullptr;
  float* out_b = nullptr;
  int qsplit = 64;
  int64_t ldo = 0;
  int trans = 0;
  const int32_t* kmap = nullptr;
  int64_t kmap_limit = INT64_MAX;  // kmap values outside [0, kmap_limit) are not written
  float scale = 1.0f;
  int accumulate = 0;
};

// Workspace of one contraction (reusable by the next one on the same stream):
//   part     fp32, *_part_floats() elements
//   rsplit   bf16, skinny_rsplit_elems(I) elements, I = K (rowdot) or M (coldot)
//   counters skinny_counter_count(M, K) unsigned ints, zero on entry; the
//            kernels leave them zero again
struct SkWork {
  float* part = nullptr;
  void* rsplit = nullptr;
  unsigned* counters = nullptr;
  bool prepared = false;  // rsplit already holds this call's split operand (prep_r_batch)
};

// One rank-sized operand to split ahead of its contraction: R with c columns
// over I indices (I = K for a rowdot, M for a coldot) into rs (bf16,
// skinny_rsplit_elems(I) elements), exactly as the contraction would.
struct SkPrep {
  SkR R;
  int c = 0;
  int64_t I = 0;
  void* rs = nullptr;
};
// Splits up to 8 operands in one launch; the contractions then run with
// SkWork{.rsplit = rs, .prepared = true}.
slora_status prep_r_batch(const SkPrep* jobs, int n, cudaStream_t st);

// c = number of R columns (1..64).
int64_t rowdot_part_floats(int64_t M, int64_t K, int c);
int64_t coldot_part_floats(int64_t M, int64_t K, int c);
int64_t skinny_rsplit_elems(int64_t I);
int64_t skinny_counter_count(int64_t M, int64_t K);
slora_status rowdot(const SkY& Y, int64_t M, int64_t K, const SkR& R, int c,
                    const SkRowOut& o, const SkWork& w, cudaStream_t st);
slora_status coldot(const SkY& Y, int64_t M, int64_t K, const SkR& R, int c,
                    const SkColOut& o, const SkWork& w, cudaStream_t st);
// One of several independent coldots (distinct outputs) run by coldot_batch.
struct SkColJob {
  SkY Y;              // no row map
  int64_t M = 0, K = 0;
  SkR R;              // its dtype fixes the term count; read only by the fallback
  int c = 0;
  void* rs = nullptr;  // R split by prep_r_batch
  SkColOut o;
};
// Workspace of coldot_batch: part floats and counters (zero on entry, left zero).
int64_t coldot_batch_part_floats(const SkColJob* jobs, int n);
int64_t coldot_batch_counter_count(const SkColJob* jobs, int n);
// Up to 7 coldots in one TMA launch whose units come from one ticket (each job
// cut into units in proportion to its size), when every Y is a plain matrix
// with 16-byte aligned rows, every job is non-empty and all share the column
// padding and term count; otherwise one coldot per job, in order.
slora_status coldot_batch(const SkColJob* jobs, int n, float* part, unsigned* counters,
                          cudaStream_t st);
// Rows of a rank projection computed in GEMM epilogues (TcGemm::proj_*), two
// jobs per launch (typically the context-row and the output-row GEMM):
// out_k(m, g * r + q) = sum over t < nparts_k of part_k[(m * nparts_k + t) * pc + g * lr + q]
// for q < r, g < pc / lr, emitted through o_k exactly as rowdot emits column
// g * r + q.  Fixed summation order (bit-reproducible).  pc, lr multiples of 4.
slora_status reduce_row_partials(const float* part0, int nparts0, int64_t M0, const SkRowOut& o0,
                                 const float* part1, int nparts1, int64_t M1, const SkRowOut& o1,
                                 int pc, int lr, int r, cudaStream_t st);
// Device error flag of the TMA kernel (a bounded wait that expired).
slora_status skinny_check_error(bool clear);
// Budget of the TMA kernel's pipeline waits in SM clock cycles (< 0: default).
slora_status skinny_set_wait_budget(long long cycles);

}  // namespace slora
