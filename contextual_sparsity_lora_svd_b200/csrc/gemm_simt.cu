// CUDA-core gathered GEMM (see gemm_simt.cuh).  64x64 output tile per
// 256-thread block, 16-deep K slices staged in shared memory, 4x4 outputs per
// thread, fp32 accumulation.  Loads map consecutive threads along whichever
// operand index has unit stride so that plain and transposed views both
// coalesce.
#include "gemm_simt.cuh"

namespace slora {
namespace {

constexpr int BM = 64, BN = 64, BK = 16, NT = 256;

__device__ __forceinline__ float fetch(const MatRef& r, int64_t i, int64_t k, int64_t I,
                                       int64_t K) {
  if (i >= I || k >= K) return 0.0f;
  int64_t ii = r.gi ? r.gi[i] : i;
  int64_t kk = r.gk ? r.gk[k] : k;
  return ld_elem(r.ptr, ii * r.si + kk * r.sk, r.dt);
}

// Stage a [rows x BK] tile of operand r (rows starting at i0) into s[BK][64].
__device__ __forceinline__ void stage(float (*s)[BM + 4], const MatRef& r, int64_t i0,
                                      int64_t k0, int64_t I, int64_t K, int tid) {
  if (r.si == 1 && r.gi == nullptr) {
    // i is the contiguous index: lanes walk i
#pragma unroll
    for (int j = 0; j < (BM * BK) / NT; ++j) {
      int e = tid + j * NT;
      int ii = e % BM, kk = e / BM;
      s[kk][ii] = fetch(r, i0 + ii, k0 + kk, I, K);
    }
  } else {
    // k is contiguous (or both gathered): lanes walk k
#pragma unroll
    for (int j = 0; j < (BM * BK) / NT; ++j) {
      int e = tid + j * NT;
      int kk = e % BK, ii = e / BK;
      s[kk][ii] = fetch(r, i0 + ii, k0 + kk, I, K);
    }
  }
}

__global__ void __launch_bounds__(NT) gemm_simt_kernel(const __grid_constant__ GemmArgs g) {
  __shared__ float As[BK][BM + 4];
  __shared__ float Bs[BK][BN + 4];
  const int tid = threadIdx.x;
  const int tx = tid % 16, ty = tid / 16;
  const int64_t m0 = int64_t(blockIdx.y) * BM, n0 = int64_t(blockIdx.x) * BN;

  float acc[4][4];
#pragma unroll
  for (int a = 0; a < 4; ++a)
#pragma unroll
    for (int b = 0; b < 4; ++b) acc[a][b] = 0.0f;

  for (int s = 0; s < g.nseg; ++s) {
    const Seg& sg = g.seg[s];
    float part[4][4];
#pragma unroll
    for (int a = 0; a < 4; ++a)
#pragma unroll
      for (int b = 0; b < 4; ++b) part[a][b] = 0.0f;
    for (int64_t k0 = 0; k0 < sg.K; k0 += BK) {
      stage(As, sg.a, m0, k0, g.M, sg.K, tid);
      stage(Bs, sg.b, n0, k0, g.N, sg.K, tid);
      __syncthreads();
#pragma unroll
      for (int kk = 0; kk < BK; ++kk) {
        float av[4], bv[4];
#pragma unroll
        for (int a = 0; a < 4; ++a) av[a] = As[kk][ty * 4 + a];
#pragma unroll
        for (int b = 0; b < 4; ++b) bv[b] = Bs[kk][tx * 4 + b];
#pragma unroll
        for (int a = 0; a < 4; ++a)
#pragma unroll
          for (int b = 0; b < 4; ++b) part[a][b] = fmaf(av[a], bv[b], part[a][b]);
      }
      __syncthreads();
    }
#pragma unroll
    for (int a = 0; a < 4; ++a)
#pragma unroll
      for (int b = 0; b < 4; ++b) acc[a][b] = fmaf(sg.alpha, part[a][b], acc[a][b]);
  }

  const OutRef& c = g.c;
#pragma unroll
  for (int a = 0; a < 4; ++a) {
    int64_t m = m0 + ty * 4 + a;
    if (m >= g.M) continue;
    int64_t row = c.gm ? c.gm[m] : m;
#pragma unroll
    for (int b = 0; b < 4; ++b) {
      int64_t n = n0 + tx * 4 + b;
      if (n >= g.N) continue;
      int64_t col = c.gn ? c.gn[n] : n;
      int64_t off = row * c.ldc + col;
      float v = acc[a][b];
      if (c.accumulate) v += ld_elem(c.ptr, off, c.dt);
      st_elem(c.ptr, off, c.dt, v);
      if (c.ptr2) {
        const int64_t r2 = c.gm2 ? c.gm2[m] : m;
        static_cast<__nv_bfloat16*>(c.ptr2)[r2 * c.ld2 + n] = __float2bfloat16_rn(c.scale2 * v);
      }
    }
  }
}

}  // namespace

slora_status gemm_simt(const GemmArgs& g, cudaStream_t st) {
  if (g.M <= 0 || g.N <= 0) return SLORA_OK;
  dim3 grid(unsigned((g.N + BN - 1) / BN), unsigned((g.M + BM - 1) / BM));
  if (grid.y > 65535u) SLORA_FAIL(SLORA_ERR_SHAPE, "gemm_simt: M=%lld too large", (long long)g.M);
  double kk = 0.0;
  for (int s = 0; s < g.nseg; ++s) kk += double(g.seg[s].K);
  LaunchScope ls(kGemmSimt, 2.0 * double(g.M) * double(g.N) * kk, st);
  gemm_simt_kernel<<<grid, NT, 0, st>>>(g);
  SLORA_CHECK_LAUNCH();
  return SLORA_OK;
}

}  // namespace slora

namespace slora {
slora_status gemm(const GemmArgs& g, cudaStream_t st) { return gemm_simt(g, st); }
}  // namespace slora
