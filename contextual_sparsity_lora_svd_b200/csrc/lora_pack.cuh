#pragma once
#include "common.cuh"

namespace slora {
// out [n_ntiles*256 x ldo]: tile nt rows 0..127 = [Bg[c] | 0], rows 128..255 =
// [0 | Bu[c]] for channels c = nt*128 + j (idx[c] if idx), zero past N.
// rows_src: rows of Bg/Bu (valid channel indices are [0, rows_src)).
slora_status pack_gate_up_b(const void* Bg, const void* Bu, const int32_t* idx, int64_t N, int r,
                            int64_t n_ntiles, int64_t ldo, void* out, cudaStream_t st,
                            int64_t rows_src);
// out [n x ldo] with out[c][q] = in[q][idx ? idx[c] : c] (in is rows x cols,
// n = number of output rows), zero columns past `rows`.
slora_status transpose_rows(const void* in, int64_t rows, int64_t cols, const int32_t* idx,
                            int64_t n, int64_t ldo, void* out, cudaStream_t st);
// Compaction of selected rows: out[j][:] = in[idx[j]][:] for j < n (bf16,
// rows of `cols` elements, cols a multiple of 8, leading dimensions ld_in/ld_out).
// rows_in: rows of `in`; an index outside [0, rows_in) yields a zero row and
// raises the flag that pack_check_error reads.
slora_status gather_rows(const void* in, int64_t ld_in, const int32_t* idx, int64_t n,
                         int64_t cols, void* out, int64_t ld_out, cudaStream_t st,
                         int64_t rows_in);
// Up to three compactions sharing one index list in one launch: job k copies
// rows idx[j] of in_k (rows_in_k rows, leading dimension ld_in16 x 16 bytes)
// to row j of out_k (leading dimension ld_out16 x 16 bytes), `cols` bf16
// (a multiple of 8) per row; same index rule as gather_rows.
struct GatherJob {
  const void* in = nullptr;
  void* out = nullptr;
  int64_t ld_in16 = 0, ld_out16 = 0, rows_in = 0;
};
struct GatherJobs {
  static constexpr int kMax = 3;
  GatherJob job[kMax];
  int njobs = 0;
};
slora_status gather_rows_multi(const GatherJob* jobs, int njobs, const int32_t* idx, int64_t n,
                               int64_t cols, cudaStream_t st);
// out [(rows_top + rows_bottom) x cols] = [top; bottom].
slora_status stack_rows(const void* top, const void* bottom, int64_t rows_top,
                        int64_t rows_bottom, int64_t cols, void* out, cudaStream_t st);
// out [rows x ldo] = in [rows x cols] with zero padding columns.
slora_status copy_pad(const void* in, int64_t rows, int64_t cols, int64_t ldo, void* out,
                      cudaStream_t st);
// out [rows x (ca + cb)] fp32 = [a | b] (a: rows x ca, b: rows x cb, both row-major).
slora_status concat_cols_f32(const float* a, const float* b, int64_t rows, int64_t ca,
                             int64_t cb, float* out, cudaStream_t st);
// out [n x ldo] bf16 = rows (idx ? idx[j] : j) of in [* x ld_in], first `cols`
// columns, zero padded to ldo.
slora_status gather_pad(const void* in, int64_t ld_in, const int32_t* idx, int64_t n,
                        int64_t cols, void* out, int64_t ldo, cudaStream_t st, int64_t rows_in);
// out[i] = in[i] for i < n when 0 <= in[i] < limit; an entry outside that
// range becomes 0 and raises the flag that pack_check_error reads.  Every
// caller-supplied channel index list goes through this before any kernel
// reads through it, so a bad list gives wrong results, never a wild access.
slora_status sanitize_indices(const int32_t* in, int64_t n, int64_t limit, int32_t* out,
                              cudaStream_t st);
// Reads (and with `clear` resets) the flag the gathers above raise when an
// index lies outside their source; SLORA_ERR_INVALID_ARG if it was raised.
// Synchronous: waits for the device.
slora_status pack_check_error(bool clear);
// Adds fp32 results computed on a channel subset into the full-channel ones:
// dst[idx[j]][q] += src[j][q] (trans: dst[q][idx[j]] += src[q][j]) for j < n,
// q < r, up to four jobs sharing idx in one launch.  An index outside
// [0, limit) is skipped and raises the flag that pack_check_error reads.
struct ScatterAddJob {
  float* dst = nullptr;
  const float* src = nullptr;
  int64_t ld_dst = 0, ld_src = 0;
  int trans = 0;
};
struct ScatterAddJobs {
  static constexpr int kMax = 4;
  ScatterAddJob job[kMax];
};
slora_status scatter_add_cols(const ScatterAddJob* jobs, int njobs, const int32_t* idx,
                              int64_t n, int r, int64_t limit, cudaStream_t st);
// Sums of per-group fp32 results in a fixed order: for each segment q,
// dst_q[i] = sum over g = 0 .. groups-1 of src[g * stride + off_q + i], i < len_q
// (up to six segments, one launch).
struct SumSeg {
  float* dst = nullptr;
  int64_t off = 0, len = 0;
};
struct SumSegs {
  static constexpr int kMax = 6;
  SumSeg seg[kMax];
};
slora_status sum_groups(const float* src, int groups, int64_t stride, const SumSeg* segs,
                        int nseg, cudaStream_t st);
// M-tile list {row0, row0, nvalid, 0} covering rows [0, M) in 128-row tiles.
slora_status make_plain_tiles(int4* tiles, int64_t M, cudaStream_t st);
}  // namespace slora
