// tcgen05 (5th-generation tensor core) GEMM for the bf16 sliced contractions.
//
//   C[M x N] = sum_seg A_seg[M x K_seg] . B_seg[N x K_seg]^T     (fp32 in TMEM)
//
// A operands are bf16 row-major (K-major) and loaded by TMA in 128 x 64
// boxes.  B operands are bf16, contiguous, in two forms:
//   B_K   K-major, rows = output channels
//   B_MN  MN-major, rows = reduction index k
// so a selected channel slice, once compacted into contiguous rows, is
// consumed as rows of W0 (output-side slice) or rows of W0^T (input-side
// slice).  Up to four segments accumulate into one tile (the LoRA branch is
// one more segment with K = rank).  Epilogues: plain bf16 store, SwiGLU
// forward on paired gate/up halves (stores g, u and h = silu(g) u), and
// SwiGLU backward (reads g, u; stores dG, dU).
//
// Rows: a list of 128-row M tiles {full_row0, compact_row0, nvalid}; a tile
// never crosses a sequence, so a tile is contiguous both in the full token
// layout and in the compact context/output layout.  Each operand picks which.
#pragma once

#include "common.cuh"

namespace slora {

enum TcBMode : int { B_K = 0, B_MN = 1 };
enum TcEpi : int { EPI_STORE = 0, EPI_SWIGLU_FWD = 1, EPI_SWIGLU_BWD = 2 };

struct TcMat {  // bf16 row-major matrix in global memory
  const void* ptr = nullptr;
  int64_t rows = 0, cols = 0, ld = 0;  // ld in elements (multiple of 8)
};

struct TcSeg {
  TcMat a;          // [rows x K]: row = tile row base + r, col = k
  TcMat b0, b1;     // b1 only with bpair (second half of the N tile)
  int bmode = B_K;
  int bpair = 0;    // K-major only: half h of the 256-row tile reads b_h rows n0p + r
  int64_t K = 0;
};

struct TcGemm {
  const int4* tiles = nullptr;  // {full_row0, compact_row0, nvalid, 0}; null: plain tiling of M
  int n_mtiles = 0;
  int a_compact = 0, out_compact = 0;
  int64_t M = 0;      // plain tiling only
  int64_t N = 0;      // valid output columns (channels)
  int paired = 0;     // N tile = 128 channels as two 128-row halves (gate | up)
  int nseg = 0;
  TcSeg seg[4];
  int epi = EPI_STORE;
  void* out0 = nullptr;  // STORE: C; SWIGLU_FWD: g; SWIGLU_BWD: dG
  void* out1 = nullptr;  // SWIGLU_FWD: u; SWIGLU_BWD: dU
  void* out2 = nullptr;  // SWIGLU_FWD: h
  int64_t ldo = 0;
  const void* in0 = nullptr;  // SWIGLU_BWD: g
  const void* in1 = nullptr;  // SWIGLU_BWD: u
  int64_t ldi = 0;
  // Optional rank-r projection of the epilogue's values, r = proj_r in {8, 16}
  // SWIGLU_FWD projects h with proj0,
  // SWIGLU_BWD projects dG with proj0 and dU with proj1.  proj0/proj1 are bf16
  // [N x ldproj] (row = output channel, ldproj a multiple of 8); each N tile
  // writes, per output row (output layout), the fp32 partial sums over its
  // channels to proj_part[(row * n_ntiles + nt) * pc + q], pc = r (FWD) or 2r
  // (BWD, dU's after dG's), proj_rows rows.  reduce_row_partials() sums them.
  const void* proj0 = nullptr;
  const void* proj1 = nullptr;
  int64_t ldproj = 0;
  int proj_r = 0;
  float* proj_part = nullptr;
  int64_t proj_rows = 0;
  // SWIGLU_BWD: rows of in0, in1, out0 and out1 (all [io_rows x N], leading
  // dimensions ldi / ldo).  When set (16-byte aligned pointers) g and u are
  // loaded and dG and dU stored by TMA through shared
  // memory, and the projection slices too; 0 keeps per-row loads and stores.
  int64_t io_rows = 0;
};

// N tiles of a GEMM (the count the projection partials are laid out over).
int64_t tc_ntiles(const TcGemm& g);

slora_status gemm_tc(const TcGemm& g, cudaStream_t st);
// Two GEMMs of the same epilogue kind (same projection rank and shared-memory
// epilogue form) in one launch: the second's tiles fill the first's last
// round.  Either may have no work.
slora_status gemm_tc_pair(const TcGemm& a, const TcGemm& b, cudaStream_t st);

// Device error flag of the tcgen05 kernels (a bounded wait that expired).
slora_status tc_check_error(bool clear);

}  // namespace slora
