#pragma once
#include "common.cuh"

namespace slora {
// out [n_ntiles*256 x ldo]: tile nt rows 0..127 = [Bg[c] | 0], rows 128..255 =
// [0 | Bu[c]] for channels c = nt*128 + j (idx[c] if idx), zero past N.
slora_status pack_gate_up_b(const void* Bg, const void* Bu, const int32_t* idx, int64_t N, int r,
                            int64_t n_ntiles, int64_t ldo, void* out, cudaStream_t st);
// out [cols x ldo] = in^T (in is rows x cols), zero columns past `rows`.
slora_status transpose_rows(const void* in, int64_t rows, int64_t cols, int64_t ldo, void* out,
                            cudaStream_t st);
// out [(rows_top + rows_bottom) x cols] = [top; bottom].
slora_status stack_rows(const void* top, const void* bottom, int64_t rows_top,
                        int64_t rows_bottom, int64_t cols, void* out, cudaStream_t st);
// out [rows x ldo] = in [rows x cols] with zero padding columns.
slora_status copy_pad(const void* in, int64_t rows, int64_t cols, int64_t ldo, void* out,
                      cudaStream_t st);
}  // namespace slora
