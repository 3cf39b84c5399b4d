// RMS normalisation with a frozen per-channel gain, fused with the residual
// add before it (forward) and with the sum of the branch gradients and the
// residual gradient (backward).  Rows of up to 16384 channels: one 128-thread
// block per row, each thread holding its 16-byte chunks in registers, so every
// input is read once and every output written once (a block-wide sum in
// between).  Longer rows: one warp per row in two passes.  Every value is
// rounded to bf16 where it is stored, and the normalisation reads the rounded
// residual sum, the value the backward sees.
#include "attention.cuh"

namespace slora {
namespace {

__device__ __forceinline__ void unpack8(const uint4& u, float (&f)[8]) {
  const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&u);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    f[2 * i] = __low2float(h[i]);
    f[2 * i + 1] = __high2float(h[i]);
  }
}
__device__ __forceinline__ uint4 pack8(const float (&f)[8]) {
  uint4 u;
  __nv_bfloat162* h = reinterpret_cast<__nv_bfloat162*>(&u);
#pragma unroll
  for (int i = 0; i < 4; ++i) h[i] = __floats2bfloat162_rn(f[2 * i], f[2 * i + 1]);
  return u;
}
__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int s = 16; s; s >>= 1) v += __shfl_xor_sync(0xffffffffu, v, s);
  return v;
}

// h = X + A (rounded), N = h rstd g
__global__ void rmsnorm_fwd_kernel(const uint4* __restrict__ X, const uint4* __restrict__ A,
                                   const uint4* __restrict__ g, int64_t T, int nch, float eps,
                                   uint4* __restrict__ Hout, uint4* __restrict__ N,
                                   float* __restrict__ rstd) {
  const int64_t row = (int64_t(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (row >= T) return;
  const int64_t o = row * nch;
  auto load_h = [&](int c, float (&h)[8]) {
    unpack8(X[o + c], h);
    if (A) {
      float a[8];
      unpack8(A[o + c], a);
#pragma unroll
      for (int i = 0; i < 8; ++i) h[i] = __bfloat162float(__float2bfloat16_rn(h[i] + a[i]));
    }
  };
  float ss = 0.f;
  for (int c = lane; c < nch; c += 32) {
    float h[8];
    load_h(c, h);
    if (A && Hout) Hout[o + c] = pack8(h);
#pragma unroll
    for (int i = 0; i < 8; ++i) ss += h[i] * h[i];
  }
  ss = warp_sum(ss);
  const float r = rsqrtf(ss / float(nch * 8) + eps);
  if (lane == 0 && rstd) rstd[row] = r;
  if (!N) return;
  for (int c = lane; c < nch; c += 32) {
    float h[8], gg[8];
    load_h(c, h);
    unpack8(g[c], gg);
#pragma unroll
    for (int i = 0; i < 8; ++i) h[i] *= r * gg[i];
    N[o + c] = pack8(h);
  }
}

// dX = dRes + r g dN - h r^3 mean(h g dN), dN = dN0 + dN1 + dN2
__global__ void rmsnorm_bwd_kernel(const uint4* __restrict__ Hin, const float* __restrict__ rstd,
                                   const uint4* __restrict__ g, const uint4* __restrict__ dN0,
                                   const uint4* __restrict__ dN1, const uint4* __restrict__ dN2,
                                   const uint4* __restrict__ dRes, int64_t T, int nch,
                                   uint4* __restrict__ dX) {
  const int64_t row = (int64_t(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (row >= T) return;
  const int64_t o = row * nch;
  auto load_dn = [&](int c, float (&dn)[8]) {
    float t[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) dn[i] = 0.f;
    const uint4* srcs[3] = {dN0, dN1, dN2};
#pragma unroll
    for (int s = 0; s < 3; ++s) {
      if (!srcs[s]) continue;
      unpack8(srcs[s][o + c], t);
#pragma unroll
      for (int i = 0; i < 8; ++i) dn[i] += t[i];
    }
  };
  float dot = 0.f;
  for (int c = lane; c < nch; c += 32) {
    float h[8], gg[8], dn[8];
    unpack8(Hin[o + c], h);
    unpack8(g[c], gg);
    load_dn(c, dn);
#pragma unroll
    for (int i = 0; i < 8; ++i) dot += h[i] * gg[i] * dn[i];
  }
  dot = warp_sum(dot);
  const float r = rstd[row];
  const float coef = r * r * r * dot / float(nch * 8);
  for (int c = lane; c < nch; c += 32) {
    float h[8], gg[8], dn[8], res[8];
    unpack8(Hin[o + c], h);
    unpack8(g[c], gg);
    load_dn(c, dn);
    if (dRes) unpack8(dRes[o + c], res);
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const float v = r * gg[i] * dn[i] - h[i] * coef;
      h[i] = dRes ? res[i] + v : v;
    }
    dX[o + c] = pack8(h);
  }
}

constexpr int kRowThreads = 128;

__device__ __forceinline__ float block_sum128(float v, float* red) {
  v = warp_sum(v);
  const int w = threadIdx.x >> 5;
  if ((threadIdx.x & 31) == 0) red[w] = v;
  __syncthreads();
  return red[0] + red[1] + red[2] + red[3];  // fixed order
}

// One block per row; thread t holds chunks t, t + 128, ... (CPT of them).
template <int CPT>
__global__ void __launch_bounds__(kRowThreads)
    rmsnorm_fwd_row_kernel(const uint4* __restrict__ X, const uint4* __restrict__ A,
                           const uint4* __restrict__ g, int nch, float eps,
                           uint4* __restrict__ Hout, uint4* __restrict__ N,
                           float* __restrict__ rstd) {
  __shared__ float red[4];
  const int64_t o = int64_t(blockIdx.x) * nch;
  float h[CPT][8];
  float ss = 0.f;
#pragma unroll
  for (int k = 0; k < CPT; ++k) {
    const int c = threadIdx.x + k * kRowThreads;
    if (c < nch) {
      unpack8(X[o + c], h[k]);
      if (A) {
        float a[8];
        unpack8(A[o + c], a);
#pragma unroll
        for (int i = 0; i < 8; ++i) h[k][i] = __bfloat162float(__float2bfloat16_rn(h[k][i] + a[i]));
        if (Hout) Hout[o + c] = pack8(h[k]);
      }
#pragma unroll
      for (int i = 0; i < 8; ++i) ss += h[k][i] * h[k][i];
    }
  }
  const float r = rsqrtf(block_sum128(ss, red) / float(nch * 8) + eps);
  if (threadIdx.x == 0 && rstd) rstd[blockIdx.x] = r;
  if (!N) return;
#pragma unroll
  for (int k = 0; k < CPT; ++k) {
    const int c = threadIdx.x + k * kRowThreads;
    if (c < nch) {
      float gg[8];
      unpack8(g[c], gg);
#pragma unroll
      for (int i = 0; i < 8; ++i) h[k][i] *= r * gg[i];
      N[o + c] = pack8(h[k]);
    }
  }
}

template <int CPT>
__global__ void __launch_bounds__(kRowThreads)
    rmsnorm_bwd_row_kernel(const uint4* __restrict__ Hin, const float* __restrict__ rstd,
                           const uint4* __restrict__ g, const uint4* __restrict__ dN0,
                           const uint4* __restrict__ dN1, const uint4* __restrict__ dN2,
                           const uint4* __restrict__ dRes, int nch, uint4* __restrict__ dX) {
  __shared__ float red[4];
  const int64_t o = int64_t(blockIdx.x) * nch;
  float h[CPT][8], gd[CPT][8];
  float dot = 0.f;
#pragma unroll
  for (int k = 0; k < CPT; ++k) {
    const int c = threadIdx.x + k * kRowThreads;
    if (c < nch) {
      float t[8], gg[8];
      unpack8(Hin[o + c], h[k]);
      unpack8(g[c], gg);
      unpack8(dN0[o + c], gd[k]);
      if (dN1) {
        unpack8(dN1[o + c], t);
#pragma unroll
        for (int i = 0; i < 8; ++i) gd[k][i] += t[i];
      }
      if (dN2) {
        unpack8(dN2[o + c], t);
#pragma unroll
        for (int i = 0; i < 8; ++i) gd[k][i] += t[i];
      }
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        gd[k][i] *= gg[i];  // g dN
        dot += h[k][i] * gd[k][i];
      }
    }
  }
  const float r = rstd[blockIdx.x];
  const float coef = r * r * r * block_sum128(dot, red) / float(nch * 8);
#pragma unroll
  for (int k = 0; k < CPT; ++k) {
    const int c = threadIdx.x + k * kRowThreads;
    if (c < nch) {
      float res[8];
      if (dRes) unpack8(dRes[o + c], res);
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const float v = r * gd[k][i] - h[k][i] * coef;
        h[k][i] = dRes ? res[i] + v : v;
      }
      dX[o + c] = pack8(h[k]);
    }
  }
}

}  // namespace

slora_status rmsnorm_fwd_run(const void* X, const void* A, const void* g, int64_t T, int64_t d,
                             float eps, void* Hout, void* N, float* rstd, cudaStream_t st) {
  if (T == 0) return SLORA_OK;
  const int nch = int(d / 8);
  LaunchScope ls(kNorm, double(T) * d * 2 * (2 + (A ? 1 : 0) + (A && Hout ? 1 : 0)), st);
  const auto* x = static_cast<const uint4*>(X);
  const auto* a = static_cast<const uint4*>(A);
  const auto* gg = static_cast<const uint4*>(g);
  auto* h = static_cast<uint4*>(Hout);
  auto* n = static_cast<uint4*>(N);
  const unsigned rows = unsigned(T);
  if (nch <= kRowThreads) {
    rmsnorm_fwd_row_kernel<1><<<rows, kRowThreads, 0, st>>>(x, a, gg, nch, eps, h, n, rstd);
  } else if (nch <= 2 * kRowThreads) {
    rmsnorm_fwd_row_kernel<2><<<rows, kRowThreads, 0, st>>>(x, a, gg, nch, eps, h, n, rstd);
  } else if (nch <= 4 * kRowThreads) {
    rmsnorm_fwd_row_kernel<4><<<rows, kRowThreads, 0, st>>>(x, a, gg, nch, eps, h, n, rstd);
  } else if (nch <= 8 * kRowThreads) {
    rmsnorm_fwd_row_kernel<8><<<rows, kRowThreads, 0, st>>>(x, a, gg, nch, eps, h, n, rstd);
  } else if (nch <= 16 * kRowThreads) {
    rmsnorm_fwd_row_kernel<16><<<rows, kRowThreads, 0, st>>>(x, a, gg, nch, eps, h, n, rstd);
  } else {
    rmsnorm_fwd_kernel<<<unsigned((T + 7) / 8), 256, 0, st>>>(x, a, gg, T, nch, eps, h, n, rstd);
  }
  SLORA_CHECK_LAUNCH();
  return SLORA_OK;
}

slora_status rmsnorm_bwd_run(const void* Hin, const float* rstd, const void* g, const void* dN0,
                             const void* dN1, const void* dN2, const void* dRes, int64_t T,
                             int64_t d, void* dX, cudaStream_t st) {
  if (T == 0) return SLORA_OK;
  const int nch = int(d / 8);
  const int nin = 2 + (dN0 ? 1 : 0) + (dN1 ? 1 : 0) + (dN2 ? 1 : 0) + (dRes ? 1 : 0);
  LaunchScope ls(kNorm, double(T) * d * 2 * nin, st);
  const auto* hin = static_cast<const uint4*>(Hin);
  const auto* gg = static_cast<const uint4*>(g);
  const auto* n0 = static_cast<const uint4*>(dN0);
  const auto* n1 = static_cast<const uint4*>(dN1);
  const auto* n2 = static_cast<const uint4*>(dN2);
  const auto* res = static_cast<const uint4*>(dRes);
  auto* dx = static_cast<uint4*>(dX);
  const unsigned rows = unsigned(T);
  if (nch <= kRowThreads) {
    rmsnorm_bwd_row_kernel<1><<<rows, kRowThreads, 0, st>>>(hin, rstd, gg, n0, n1, n2, res, nch, dx);
  } else if (nch <= 2 * kRowThreads) {
    rmsnorm_bwd_row_kernel<2><<<rows, kRowThreads, 0, st>>>(hin, rstd, gg, n0, n1, n2, res, nch, dx);
  } else if (nch <= 4 * kRowThreads) {
    rmsnorm_bwd_row_kernel<4><<<rows, kRowThreads, 0, st>>>(hin, rstd, gg, n0, n1, n2, res, nch, dx);
  } else if (nch <= 8 * kRowThreads) {
    rmsnorm_bwd_row_kernel<8><<<rows, kRowThreads, 0, st>>>(hin, rstd, gg, n0, n1, n2, res, nch, dx);
  } else if (nch <= 16 * kRowThreads) {
    rmsnorm_bwd_row_kernel<16><<<rows, kRowThreads, 0, st>>>(hin, rstd, gg, n0, n1, n2, res, nch,
                                                             dx);
  } else {
    rmsnorm_bwd_kernel<<<unsigned((T + 7) / 8), 256, 0, st>>>(hin, rstd, gg, n0, n1, n2, res, T,
                                                             nch, dx);
  }
  SLORA_CHECK_LAUNCH();
  return SLORA_OK;
}

}  // namespace slora
