// Small per-step packing of the LoRA factors into the operand layouts the
// tcgen05 GEMM reads (all bf16, a few hundred KB per step):
//   pack_gate_up_b : for every 256-row N tile of the paired gate|up GEMM, rows
//                    0..127 = [B_g[c] | 0] and rows 128..255 = [0 | B_u[c]] for
//                    the tile's 128 channels c (idx[c] when sliced), so the
//                    LoRA up-projection of both halves is one K = 2r segment
//   transpose_rows : out[c][q] = in[q][c]     (A_d^T, rows = channels)
//   stack_rows     : out = [top; bottom]      ([A_g; A_u], MN-major operand)
#include <algorithm>

#include "lora_pack.cuh"

#include "gemm_tc.cuh"

namespace slora {
namespace {

// Raised by a gather that met an index outside its source (the row is read as
// zeros instead); read and cleared by pack_check_error.
__device__ int g_pack_bad_index = 0;
__device__ __forceinline__ bool index_ok(int64_t v, int64_t n) {
  if (v >= 0 && v < n) return true;
  atomicExch(&g_pack_bad_index, 1);
  return false;
}

__global__ void pack_gate_up_b_kernel(const __nv_bfloat16* __restrict__ Bg,
                                      const __nv_bfloat16* __restrict__ Bu,
                                      const int32_t* __restrict__ idx, int64_t N, int r,
                                      int64_t rows, int64_t ldo, int64_t rows_src,
                                      __nv_bfloat16* __restrict__ out) {
  const int64_t e = int64_t(blockIdx.x) * blockDim.x + threadIdx.x;
  if (e >= rows * ldo) return;
  const int64_t R = e / ldo;
  const int col = int(e % ldo);
  const int64_t nt = R / 256;
  const int h = int((R % 256) / 128);
  const int64_t c = nt * 128 + (R % 128);
  float v = 0.0f;
  if (c < N && col >= h * r && col < (h + 1) * r) {
    const int64_t src = idx ? idx[c] : c;
    if (index_ok(src, rows_src)) v = __bfloat162float((h ? Bu : Bg)[src * r + (col - h * r)]);
  }
  out[e] = __float2bfloat16_rn(v);
}

__global__ void transpose_rows_kernel(const __nv_bfloat16* __restrict__ in, int64_t rows,
                                      int64_t cols, const int32_t* __restrict__ idx, int64_t n,
                                      int64_t ldo, __nv_bfloat16* __restrict__ out) {
  const int64_t e = int64_t(blockIdx.x) * blockDim.x + threadIdx.x;
  if (e >= n * ldo) return;
  const int64_t c = e / ldo, q = e % ldo;
  const int64_t src = idx ? int64_t(idx[c]) : c;
  out[e] = (q < rows && index_ok(src, cols)) ? in[q * cols + src] : __float2bfloat16_rn(0.0f);
}

// One block per selected row and 2048-element column chunk; 16-byte copies.
__global__ void gather_rows_kernel(const uint4* __restrict__ in, int64_t ld_in16,
                                   const int32_t* __restrict__ idx, int64_t rows_in,
                                   int64_t cols16, uint4* __restrict__ out, int64_t ld_out16) {
  const int64_t j = blockIdx.x;
  const int64_t src = idx[j];
  const bool ok = index_ok(src, rows_in);
  for (int64_t c = int64_t(blockIdx.y) * blockDim.x + threadIdx.x; c < cols16;
       c += int64_t(gridDim.y) * blockDim.x)
    out[j * ld_out16 + c] = ok ? __ldg(in + src * ld_in16 + c) : make_uint4(0, 0, 0, 0);
}

// Several row compactions sharing one index list: warp w takes (job, row)
// items w, w + nwarps, ...; each lane moves 8 16-byte units per round (all
// loads of a round issued before its stores).
__global__ void __launch_bounds__(256) gather_rows_multi_kernel(const __grid_constant__ GatherJobs J,
                                                                const int32_t* __restrict__ idx,
                                                                int64_t n, int64_t cols16) {
  const int lane = threadIdx.x & 31;
  const int64_t nw = int64_t(gridDim.x) * (blockDim.x >> 5);
  const int64_t items = n * J.njobs;
  for (int64_t it = int64_t(blockIdx.x) * (blockDim.x >> 5) + (threadIdx.x >> 5); it < items;
       it += nw) {
    const int jb = int(it / n);
    const int64_t j = it % n;
    const GatherJob& g = J.job[jb];
    const int64_t src = idx[j];
    const bool ok = index_ok(src, g.rows_in);
    const uint4* in = static_cast<const uint4*>(g.in) + (ok ? src : 0) * g.ld_in16;
    uint4* out = static_cast<uint4*>(g.out) + j * g.ld_out16;
    for (int64_t c0 = lane; c0 < cols16; c0 += 32 * 8) {
      uint4 v[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        const int64_t c = c0 + 32 * u;
        v[u] = (ok && c < cols16) ? __ldg(in + c) : make_uint4(0, 0, 0, 0);
      }
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        const int64_t c = c0 + 32 * u;
        if (c < cols16) out[c] = v[u];
      }
    }
  }
}

__global__ void stack_rows_kernel(const __nv_bfloat16* __restrict__ top,
                                  const __nv_bfloat16* __restrict__ bottom, int64_t rows_top,
                                  int64_t rows_bottom, int64_t cols,
                                  __nv_bfloat16* __restrict__ out) {
  const int64_t e = int64_t(blockIdx.x) * blockDim.x + threadIdx.x;
  const int64_t total = (rows_top + rows_bottom) * cols;
  if (e >= total) return;
  const int64_t rr = e / cols, c = e % cols;
  out[e] = rr < rows_top ? top[rr * cols + c] : bottom[(rr - rows_top) * cols + c];
}

__global__ void copy_pad_kernel(const __nv_bfloat16* __restrict__ in, int64_t rows, int64_t cols,
                                int64_t ldo, __nv_bfloat16* __restrict__ out) {
  const int64_t e = int64_t(blockIdx.x) * blockDim.x + threadIdx.x;
  if (e >= rows * ldo) return;
  const int64_t rr = e / ldo, c = e % ldo;
  out[e] = c < cols ? in[rr * cols + c] : __float2bfloat16_rn(0.0f);
}

__global__ void concat_cols_kernel(const float* __restrict__ a, const float* __restrict__ b,
                                   int64_t rows, int64_t ca, int64_t cb, float* __restrict__ out) {
  const int64_t e = int64_t(blockIdx.x) * blockDim.x + threadIdx.x;
  const int64_t w = ca + cb;
  if (e >= rows * w) return;
  const int64_t rr = e / w, c = e % w;
  out[e] = c < ca ? a[rr * ca + c] : b[rr * cb + (c - ca)];
}

__global__ void gather_pad_kernel(const __nv_bfloat16* __restrict__ in, int64_t ld_in,
                                  const int32_t* __restrict__ idx, int64_t n, int64_t cols,
                                  int64_t ldo, int64_t rows_in, __nv_bfloat16* __restrict__ out) {
  const int64_t e = int64_t(blockIdx.x) * blockDim.x + threadIdx.x;
  if (e >= n * ldo) return;
  const int64_t j = e / ldo, c = e % ldo;
  const int64_t src = idx ? int64_t(idx[j]) : j;
  out[e] = (c < cols && index_ok(src, rows_in)) ? in[src * ld_in + c] : __float2bfloat16_rn(0.0f);
}

__global__ void sanitize_kernel(const int32_t* __restrict__ in, int64_t n, int64_t limit,
                                int32_t* __restrict__ out) {
  const int64_t i = int64_t(blockIdx.x) * blockDim.x + threadIdx.x;
  if (i >= n) return;
  const int32_t v = in[i];
  out[i] = index_ok(v, limit) ? v : 0;
}

// One scatter-add job per blockIdx.y: element (j, q), j < n, q < r, of src
// (row j: src[j * ld_src + q]; trans: src[q * ld_src + j]) is added to column
// idx[j] of dst in the same orientation.  With trans, consecutive threads take
// consecutive j (coalesced source rows); without, consecutive q.
__global__ void scatter_add_kernel(const __grid_constant__ ScatterAddJobs J, const int32_t* __restrict__ idx,
                                   int64_t n, int r, int64_t limit) {
  const ScatterAddJob& jb = J.job[blockIdx.y];
  const int64_t e = int64_t(blockIdx.x) * blockDim.x + threadIdx.x;
  if (e >= n * r) return;
  const int64_t j = jb.trans ? e % n : e / r;
  const int q = int(jb.trans ? e / n : e % r);
  const int64_t c = idx[j];
  if (!index_ok(c, limit)) return;
  if (jb.trans)
    jb.dst[int64_t(q) * jb.ld_dst + c] += jb.src[int64_t(q) * jb.ld_src + j];
  else
    jb.dst[c * jb.ld_dst + q] += jb.src[j * jb.ld_src + q];
}

__global__ void plain_tiles_kernel(int4* __restrict__ tiles, int64_t M, int64_t nt) {
  const int64_t t = int64_t(blockIdx.x) * blockDim.x + threadIdx.x;
  if (t >= nt) return;
  const int64_t r0 = t * 128;
  const int64_t nv = M - r0 < 128 ? M - r0 : 128;
  tiles[t] = make_int4(int(r0), int(r0), int(nv), 0);
}

unsigned blocks(int64_t n) { return unsigned((n + 255) / 256); }

__global__ void sum_groups_kernel(const float* __restrict__ src, int groups, int64_t stride,
                                  const __grid_constant__ SumSegs S) {
  const SumSeg& q = S.seg[blockIdx.y];
  const int64_t i = int64_t(blockIdx.x) * blockDim.x + threadIdx.x;
  if (i >= q.len) return;
  float acc = 0.f;
  for (int g = 0; g < groups; ++g) acc += src[g * stride + q.off + i];
  q.dst[i] = acc;
}

}  // namespace

slora_status sum_groups(const float* src, int groups, int64_t stride, const SumSeg* segs,
                        int nseg, cudaStream_t st) {
  if (nseg <= 0) return SLORA_OK;
  if (nseg > SumSegs::kMax)
    SLORA_FAIL(SLORA_ERR_SHAPE, "sum_groups: %d segments (max %d)", nseg, SumSegs::kMax);
  SumSegs S{};
  int64_t mx = 0;
  for (int k = 0; k < nseg; ++k) {
    S.seg[k] = segs[k];
    mx = std::max(mx, segs[k].len);
  }
  if (mx == 0) return SLORA_OK;
  LaunchScope ls(kAux, double(groups) * stride * 4, st);
  sum_groups_kernel<<<dim3(blocks(mx), unsigned(nseg)), 256, 0, st>>>(src, groups, stride, S);
  SLORA_CHECK_LAUNCH();
  return SLORA_OK;
}

slora_status scatter_add_cols(const ScatterAddJob* jobs, int njobs, const int32_t* idx,
                              int64_t n, int r, int64_t limit, cudaStream_t st) {
  if (njobs <= 0 || n <= 0 || r <= 0) return SLORA_OK;
  if (njobs > ScatterAddJobs::kMax)
    SLORA_FAIL(SLORA_ERR_SHAPE, "scatter_add_cols: %d jobs (max %d)", njobs, ScatterAddJobs::kMax);
  ScatterAddJobs J{};
  for (int k = 0; k < njobs; ++k) J.job[k] = jobs[k];
  LaunchScope ls(kAux, double(njobs) * double(n) * r * 12.0, st);
  scatter_add_kernel<<<dim3(blocks(n * r), unsigned(njobs)), 256, 0, st>>>(J, idx, n, r, limit);
  SLORA_CHECK_LAUNCH();
  return SLORA_OK;
}

slora_status pack_gate_up_b(const void* Bg, const void* Bu, const int32_t* idx, int64_t N, int r,
                            int64_t n_ntiles, int64_t ldo, void* out, cudaStream_t st,
                            int64_t rows_src) {
  const int64_t rows = n_ntiles * 256;
  if (rows <= 0) return SLORA_OK;
  LaunchScope ls(kAux, double(rows) * ldo * 2 + double(N) * 2 * r * 2, st);
  pack_gate_up_b_kernel<<<blocks(rows * ldo), 256, 0, st>>>(
      static_cast<const __nv_bfloat16*>(Bg), static_cast<const __nv_bfloat16*>(Bu), idx, N, r,
      rows, ldo, rows_src, static_cast<__nv_bfloat16*>(out));
  SLORA_CHECK_LAUNCH();
  return SLORA_OK;
}

slora_status transpose_rows(const void* in, int64_t rows, int64_t cols, const int32_t* idx,
                            int64_t n, int64_t ldo, void* out, cudaStream_t st) {
  if (n <= 0) return SLORA_OK;
  LaunchScope ls(kAux, double(rows) * n * 2 + double(n) * ldo * 2, st);
  transpose_rows_kernel<<<blocks(n * ldo), 256, 0, st>>>(
      static_cast<const __nv_bfloat16*>(in), rows, cols, idx, n, ldo,
      static_cast<__nv_bfloat16*>(out));
  SLORA_CHECK_LAUNCH();
  return SLORA_OK;
}

slora_status gather_rows_multi(const GatherJob* jobs, int njobs, const int32_t* idx, int64_t n,
                               int64_t cols, cudaStream_t st) {
  if (n <= 0 || njobs <= 0) return SLORA_OK;
  if (njobs > GatherJobs::kMax)
    SLORA_FAIL(SLORA_ERR_SHAPE, "gather_rows_multi: %d jobs (max %d)", njobs, GatherJobs::kMax);
  GatherJobs J{};
  J.njobs = njobs;
  for (int k = 0; k < njobs; ++k) {
    const GatherJob& g = jobs[k];
    if (cols % 8 || g.ld_in16 < 0 || g.ld_out16 < 0 ||
        (reinterpret_cast<uintptr_t>(g.in) & 15) || (reinterpret_cast<uintptr_t>(g.out) & 15))
      SLORA_FAIL(SLORA_ERR_ALIGN, "gather_rows_multi: rows must be whole 16-byte units");
    J.job[k] = g;
  }
  const int64_t items = n * njobs;
  const int64_t want = (items + 7) / 8;  // 8 warps per block
  const int64_t cap = int64_t(num_sms()) * 4;  // 32 warps per SM, 16 KB of loads in flight each
  LaunchScope ls(kCompact, 2.0 * double(njobs) * double(n) * cols * 2, st);
  gather_rows_multi_kernel<<<unsigned(std::max<int64_t>(1, std::min(want, cap))), 256, 0, st>>>(
      J, idx, n, cols / 8);
  SLORA_CHECK_LAUNCH();
  return SLORA_OK;
}

slora_status gather_rows(const void* in, int64_t ld_in, const int32_t* idx, int64_t n,
                         int64_t cols, void* out, int64_t ld_out, cudaStream_t st,
                         int64_t rows_in) {
  if (n <= 0) return SLORA_OK;
  if (cols % 8 || ld_in % 8 || ld_out % 8)
    SLORA_FAIL(SLORA_ERR_ALIGN, "gather_rows: rows must be whole 16-byte units");
  const int64_t c16 = cols / 8;
  const unsigned gy = unsigned((c16 + 255) / 256);
  if (n > 2147483647) SLORA_FAIL(SLORA_ERR_SHAPE, "gather_rows: too many rows");
  LaunchScope ls(kCompact, 2.0 * double(n) * cols * 2, st);
  gather_rows_kernel<<<dim3(unsigned(n), gy), 256, 0, st>>>(
      static_cast<const uint4*>(in), ld_in / 8, idx, rows_in, c16, static_cast<uint4*>(out),
      ld_out / 8);
  SLORA_CHECK_LAUNCH();
  return SLORA_OK;
}

slora_status stack_rows(const void* top, const void* bottom, int64_t rows_top,
                        int64_t rows_bottom, int64_t cols, void* out, cudaStream_t st) {
  LaunchScope ls(kAux, 4.0 * double(rows_top + rows_bottom) * cols, st);
  stack_rows_kernel<<<blocks((rows_top + rows_bottom) * cols), 256, 0, st>>>(
      static_cast<const __nv_bfloat16*>(top), static_cast<const __nv_bfloat16*>(bottom), rows_top,
      rows_bottom, cols, static_cast<__nv_bfloat16*>(out));
  SLORA_CHECK_LAUNCH();
  return SLORA_OK;
}

slora_status concat_cols_f32(const float* a, const float* b, int64_t rows, int64_t ca,
                             int64_t cb, float* out, cudaStream_t st) {
  LaunchScope ls(kAux, 8.0 * double(rows) * (ca + cb), st);
  concat_cols_kernel<<<blocks(rows * (ca + cb)), 256, 0, st>>>(a, b, rows, ca, cb, out);
  SLORA_CHECK_LAUNCH();
  return SLORA_OK;
}

slora_status gather_pad(const void* in, int64_t ld_in, const int32_t* idx, int64_t n,
                        int64_t cols, void* out, int64_t ldo, cudaStream_t st, int64_t rows_in) {
  if (n <= 0) return SLORA_OK;
  LaunchScope ls(kAux, double(n) * (cols + ldo) * 2, st);
  gather_pad_kernel<<<blocks(n * ldo), 256, 0, st>>>(static_cast<const __nv_bfloat16*>(in), ld_in,
                                                     idx, n, cols, ldo, rows_in,
                                                     static_cast<__nv_bfloat16*>(out));
  SLORA_CHECK_LAUNCH();
  return SLORA_OK;
}

slora_status sanitize_indices(const int32_t* in, int64_t n, int64_t limit, int32_t* out,
                              cudaStream_t st) {
  if (n <= 0) return SLORA_OK;
  LaunchScope ls(kAux, double(n) * 8, st);
  sanitize_kernel<<<blocks(n), 256, 0, st>>>(in, n, limit, out);
  SLORA_CHECK_LAUNCH();
  return SLORA_OK;
}

slora_status make_plain_tiles(int4* tiles, int64_t M, cudaStream_t st) {
  const int64_t nt = (M + 127) / 128;
  if (nt <= 0) return SLORA_OK;
  LaunchScope ls(kAux, double(nt) * 16, st);
  plain_tiles_kernel<<<blocks(nt), 256, 0, st>>>(tiles, M, nt);
  SLORA_CHECK_LAUNCH();
  return SLORA_OK;
}

slora_status copy_pad(const void* in, int64_t rows, int64_t cols, int64_t ldo, void* out,
                      cudaStream_t st) {
  LaunchScope ls(kAux, double(rows) * (cols + ldo) * 2, st);
  copy_pad_kernel<<<blocks(rows * ldo), 256, 0, st>>>(static_cast<const __nv_bfloat16*>(in), rows,
                                                      cols, ldo, static_cast<__nv_bfloat16*>(out));
  SLORA_CHECK_LAUNCH();
  return SLORA_OK;
}

slora_status pack_check_error(bool clear) {
  int v = 0;
  SLORA_CUDA(cudaMemcpyFromSymbol(&v, g_pack_bad_index, sizeof(int)));
  if (clear && v) {
    const int z = 0;
    SLORA_CUDA(cudaMemcpyToSymbol(g_pack_bad_index, &z, sizeof(int)));
  }
  if (v) SLORA_FAIL(SLORA_ERR_INVALID_ARG, "a channel index list held an entry outside its weight (replaced by channel 0)");
  return SLORA_OK;
}

}  // namespace slora
