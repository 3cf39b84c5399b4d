// Offline truncated SVD of a frozen weight (SparseLoRA article, section 2:
// the pretrained weights are decomposed once before training and the leading
// singular modes kept; section 7: rank 8 balances cost and accuracy).
//
// Method (all on the device, ordered on the caller's stream): randomized block
// subspace iteration in the manner of Halko, Martinsson and Tropp (2011),
// "Finding structure with randomness", Alg. 4.4, with block b = rank +
// oversampling:
//   Y = orth(W Omega);  repeat q times { Z = orth(W^T Y); Y = orth(W Z) }
//   Z = W^T Y;  M = Z^T Z = E diag(lambda) E^T;  U_r = Y E_r,  L = Z E_r.
// orth() is Cholesky-QR applied twice (CholQR2); the small Cholesky and the
// Jacobi eigen-solve of M run in fp64 in one thread block.  The Gaussian start
// block comes from SplitMix64 (Steele, Lea and Flood, 2014) counters fed to the
// Box-Muller transform.
#include "gemm_simt.cuh"

namespace slora {
namespace {

__device__ __forceinline__ uint64_t splitmix64(uint64_t x) {
  uint64_t z = x + 0x9E3779B97F4A7C15ull;
  z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
  z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
  return z ^ (z >> 31);
}

__global__ void gaussian_fill_kernel(float* out, int64_t count, uint64_t seed) {
  int64_t i = int64_t(blockIdx.x) * blockDim.x + threadIdx.x;
  if (i >= count) return;
  uint64_t a = splitmix64(seed + 0x632BE59BD9B4E019ull * uint64_t(2 * i));
  uint64_t b = splitmix64(seed + 0x632BE59BD9B4E019ull * uint64_t(2 * i + 1));
  double u1 = (double((a >> 11) + 1)) * (1.0 / 9007199254740992.0);  // (0, 1]
  double u2 = double(b >> 11) * (1.0 / 9007199254740992.0);          // [0, 1)
  out[i] = float(sqrt(-2.0 * log(u1)) * cos(6.283185307179586 * u2));
}

// Cholesky of the b x b Gram G (fp32) in fp64, then the inverse of the upper
// factor.  A pivot below 1e-10 of the largest diagonal drops that direction
// (its column of R^-1 is zero), which keeps rank-deficient blocks finite.
__global__ void chol_inv_kernel(const float* __restrict__ G, int b, float* __restrict__ Rinv) {
  extern __shared__ double sm[];
  double* R = sm;          // b*b, upper triangle used
  double* X = sm + b * b;  // b*b inverse
  __shared__ double s_tiny;
  __shared__ int s_dead[64];
  const int t = threadIdx.x;
  for (int e = t; e < b * b; e += blockDim.x) { R[e] = 0.0; X[e] = 0.0; }
  if (t == 0) {
    double mx = 0.0;
    for (int i = 0; i < b; ++i) mx = fmax(mx, double(G[i * b + i]));
    s_tiny = 1e-10 * mx + 1e-300;
  }
  __syncthreads();
  for (int j = 0; j < b; ++j) {
    if (t == 0) {
      double d = double(G[j * b + j]);
      for (int i = 0; i < j; ++i) d -= R[i * b + j] * R[i * b + j];
      s_dead[j] = !(d > s_tiny);
      R[j * b + j] = s_dead[j] ? 1.0 : sqrt(d);
    }
    __syncthreads();
    for (int c = j + 1 + t; c < b; c += blockDim.x) {
      double v = 0.0;
      if (!s_dead[j]) {
        v = double(G[j * b + c]);
        for (int i = 0; i < j; ++i) v -= R[i * b + j] * R[i * b + c];
        v /= R[j * b + j];
      }
      R[j * b + c] = v;
    }
    __syncthreads();
  }
  // column c of R^-1: back substitution, one thread per column
  for (int c = t; c < b; c += blockDim.x) {
    for (int i = c; i >= 0; --i) {
      double v = (i == c) ? 1.0 : 0.0;
      for (int q = i + 1; q <= c; ++q) v -= R[i * b + q] * X[q * b + c];
      X[i * b + c] = s_dead[i] ? 0.0 : v / R[i * b + i];
    }
  }
  __syncthreads();
  for (int e = t; e < b * b; e += blockDim.x) Rinv[e] = float(X[e]);
}

// Cyclic Jacobi eigen-solve of the symmetric b x b matrix M (fp32 in, fp64
// work, Golub & Van Loan "Matrix Computations" sec. 8.5 rotation), then the
// eigenpairs sorted by decreasing eigenvalue: E [b x b] columns, lam [b].
__global__ void jacobi_eig_kernel(const float* __restrict__ M, int b, float* __restrict__ E,
                                  float* __restrict__ lam) {
  extern __shared__ double sm[];
  double* A = sm;
  double* V = sm + b * b;
  __shared__ double s_c, s_s;
  __shared__ int s_go;
  __shared__ int order[64];
  const int t = threadIdx.x;
  for (int e = t; e < b * b; e += blockDim.x) {
    int i = e / b, j = e % b;
    A[e] = 0.5 * (double(M[i * b + j]) + double(M[j * b + i]));
    V[e] = (i == j) ? 1.0 : 0.0;
  }
  __syncthreads();
  for (int sweep = 0; sweep < 60; ++sweep) {
    if (t == 0) {
      double off = 0.0, tot = 0.0;
      for (int i = 0; i < b; ++i)
        for (int j = 0; j < b; ++j) {
          double v = A[i * b + j] * A[i * b + j];
          tot += v;
          if (i != j) off += v;
        }
      s_go = off > 1e-30 * tot;
    }
    __syncthreads();
    if (!s_go) break;
    for (int p = 0; p < b - 1; ++p) {
      for (int q = p + 1; q < b; ++q) {
        if (t == 0) {
          double apq = A[p * b + q];
          double c = 1.0, s = 0.0;
          if (apq != 0.0) {
            double tau = (A[q * b + q] - A[p * b + p]) / (2.0 * apq);
            double tt = (tau >= 0.0 ? 1.0 : -1.0) / (fabs(tau) + sqrt(1.0 + tau * tau));
            c = 1.0 / sqrt(1.0 + tt * tt);
            s = tt * c;
          }
          s_c = c;
          s_s = s;
        }
        __syncthreads();
        const double c = s_c, s = s_s;
        if (s != 0.0) {
          for (int i = t; i < b; i += blockDim.x) {  // A <- A J, V <- V J
            double aip = A[i * b + p], aiq = A[i * b + q];
            A[i * b + p] = c * aip - s * aiq;
            A[i * b + q] = s * aip + c * aiq;
            double vip = V[i * b + p], viq = V[i * b + q];
            V[i * b + p] = c * vip - s * viq;
            V[i * b + q] = s * vip + c * viq;
          }
          __syncthreads();
          for (int j = t; j < b; j += blockDim.x) {  // A <- J^T A
            double apj = A[p * b + j], aqj = A[q * b + j];
            A[p * b + j] = c * apj - s * aqj;
            A[q * b + j] = s * apj + c * aqj;
          }
        }
        __syncthreads();
      }
    }
  }
  if (t == 0) {
    for (int i = 0; i < b; ++i) order[i] = i;
    for (int i = 0; i < b; ++i) {
      int best = i;
      for (int j = i + 1; j < b; ++j)
        if (A[order[j] * b + order[j]] > A[order[best] * b + order[best]]) best = j;
      int tmp = order[i]; order[i] = order[best]; order[best] = tmp;
    }
  }
  __syncthreads();
  for (int e = t; e < b * b; e += blockDim.x) {
    int i = e / b, j = e % b;
    E[e] = float(V[i * b + order[j]]);
  }
  for (int j = t; j < b; j += blockDim.x) lam[j] = float(A[order[j] * b + order[j]]);
}

template <class T>
__global__ void transpose_kernel(const T* __restrict__ in, int64_t rows, int64_t cols,
                                 T* __restrict__ out) {
  __shared__ T tile[32][33];
  int64_t r0 = int64_t(blockIdx.y) * 32, c0 = int64_t(blockIdx.x) * 32;
  for (int i = threadIdx.y; i < 32; i += blockDim.y) {
    int64_t r = r0 + i, c = c0 + threadIdx.x;
    if (r < rows && c < cols) tile[i][threadIdx.x] = in[r * cols + c];
  }
  __syncthreads();
  for (int i = threadIdx.y; i < 32; i += blockDim.y) {
    int64_t c = c0 + i, r = r0 + threadIdx.x;
    if (r < rows && c < cols) out[c * rows + r] = tile[threadIdx.x][i];
  }
}

struct PrepBufs {
  float *Y0, *Y1, *Z0, *Z1, *G, *Rinv, *E, *lam;
};

// X (m x b) <- orth(X) by CholQR2; uses tmp (m x b) and returns the buffer
// that holds the result.
slora_status orth(float* X, float* tmp, int64_t m, int b, const PrepBufs& pb, cudaStream_t st,
                  float** result) {
  float* cur = X;
  float* nxt = tmp;
  for (int pass = 0; pass < 2; ++pass) {
    GemmArgs g;  // G = cur^T cur
    g.M = b; g.N = b; g.nseg = 1;
    g.seg[0].a = colmajor(cur, kF32, b);
    g.seg[0].b = colmajor(cur, kF32, b);
    g.seg[0].K = m;
    g.c = out_rowmajor(pb.G, kF32, b);
    SLORA_TRY(gemm_simt(g, st));
    {
      LaunchScope ls(kPrepare, double(b) * b * 8, st);
      chol_inv_kernel<<<1, 64, 2 * b * b * sizeof(double), st>>>(pb.G, b, pb.Rinv);
    }
    SLORA_CHECK_LAUNCH();
    GemmArgs h;  // nxt = cur Rinv
    h.M = m; h.N = b; h.nseg = 1;
    h.seg[0].a = rowmajor(cur, kF32, b);
    h.seg[0].b = colmajor(pb.Rinv, kF32, b);
    h.seg[0].K = b;
    h.c = out_rowmajor(nxt, kF32, b);
    SLORA_TRY(gemm_simt(h, st));
    float* t = cur; cur = nxt; nxt = t;
  }
  *result = cur;
  return SLORA_OK;
}

}  // namespace

int prepare_block(int64_t n, int64_t k, int rank) {
  int64_t mn = n < k ? n : k;
  int64_t b = rank + 24 > 32 ? rank + 24 : 32;
  if (b > 64) b = 64;
  if (b > mn) b = mn;
  return int(b);
}

slora_status svd_prepare_impl(const void* W, int64_t n, int64_t k, int dt, int rank, int n_iter,
                              uint64_t seed, float* L, float* U, void* W_t, Arena& ar,
                              bool plan_only, cudaStream_t st) {
  const int b = prepare_block(n, k, rank);
  PrepBufs pb;
  pb.Y0 = ar.take<float>(size_t(n) * b);
  pb.Y1 = ar.take<float>(size_t(n) * b);
  pb.Z0 = ar.take<float>(size_t(k) * b);
  pb.Z1 = ar.take<float>(size_t(k) * b);
  pb.G = ar.take<float>(size_t(b) * b);
  pb.Rinv = ar.take<float>(size_t(b) * b);
  pb.E = ar.take<float>(size_t(b) * b);
  pb.lam = ar.take<float>(size_t(b));
  if (plan_only) return SLORA_OK;
  SLORA_TRY(arena_fits(ar, "slora_svd_prepare"));

  static bool attr_done = false;
  if (!attr_done) {
    SLORA_CUDA(cudaFuncSetAttribute(chol_inv_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                    2 * 64 * 64 * int(sizeof(double))));
    SLORA_CUDA(cudaFuncSetAttribute(jacobi_eig_kernel,
                                    cudaFuncAttributeMaxDynamicSharedMemorySize,
                                    2 * 64 * 64 * int(sizeof(double))));
    attr_done = true;
  }
  const int q = n_iter > 0 ? n_iter : 12;

  // Omega (k x b) Gaussian, Y = W Omega
  {
  LaunchScope ls(kPrepare, double(k) * b * 4, st);
  gaussian_fill_kernel<<<unsigned((k * b + 255) / 256), 256, 0, st>>>(pb.Z0, k * b, seed);
  }
  SLORA_CHECK_LAUNCH();
  auto W_times = [&](const float* Zin, float* Yout) {  // Yout (n x b) = W Zin
    GemmArgs g;
    g.M = n; g.N = b; g.nseg = 1;
    g.seg[0].a = rowmajor(W, dt, k);
    g.seg[0].b = colmajor(Zin, kF32, b);
    g.seg[0].K = k;
    g.c = out_rowmajor(Yout, kF32, b);
    return gemm_simt(g, st);
  };
  auto Wt_times = [&](const float* Yin, float* Zout) {  // Zout (k x b) = W^T Yin
    GemmArgs g;
    g.M = k; g.N = b; g.nseg = 1;
    g.seg[0].a = colmajor(W, dt, k);
    g.seg[0].b = colmajor(Yin, kF32, b);
    g.seg[0].K = n;
    g.c = out_rowmajor(Zout, kF32, b);
    return gemm_simt(g, st);
  };
  float *Y = pb.Y0, *Yt = pb.Y1, *Z = pb.Z0, *Zt = pb.Z1;
  SLORA_TRY(W_times(Z, Y));
  float* res = nullptr;
  SLORA_TRY(orth(Y, Yt, n, b, pb, st, &res));
  if (res != Y) { Yt = Y; Y = res; }
  for (int it = 0; it < q; ++it) {
    SLORA_TRY(Wt_times(Y, Z));
    SLORA_TRY(orth(Z, Zt, k, b, pb, st, &res));
    if (res != Z) { Zt = Z; Z = res; }
    SLORA_TRY(W_times(Z, Y));
    SLORA_TRY(orth(Y, Yt, n, b, pb, st, &res));
    if (res != Y) { Yt = Y; Y = res; }
  }
  SLORA_TRY(Wt_times(Y, Z));  // Z = W^T Y = B^T
  {
    GemmArgs g;  // M = Z^T Z
    g.M = b; g.N = b; g.nseg = 1;
    g.seg[0].a = colmajor(Z, kF32, b);
    g.seg[0].b = colmajor(Z, kF32, b);
    g.seg[0].K = k;
    g.c = out_rowmajor(pb.G, kF32, b);
    SLORA_TRY(gemm_simt(g, st));
  }
  {
    LaunchScope ls(kPrepare, double(b) * b * 8, st);
    jacobi_eig_kernel<<<1, 64, 2 * b * b * sizeof(double), st>>>(pb.G, b, pb.E, pb.lam);
  }
  SLORA_CHECK_LAUNCH();
  {
    GemmArgs g;  // U = Y E[:, :rank]
    g.M = n; g.N = rank; g.nseg = 1;
    g.seg[0].a = rowmajor(Y, kF32, b);
    g.seg[0].b = colmajor(pb.E, kF32, b);
    g.seg[0].K = b;
    g.c = out_rowmajor(U, kF32, rank);
    SLORA_TRY(gemm_simt(g, st));
    g.M = k;  // L = Z E[:, :rank]
    g.seg[0].a = rowmajor(Z, kF32, b);
    g.c = out_rowmajor(L, kF32, rank);
    SLORA_TRY(gemm_simt(g, st));
  }
  if (W_t) {
    dim3 grid(unsigned((k + 31) / 32), unsigned((n + 31) / 32));
    LaunchScope ls(kPrepare, 2.0 * double(n) * k * dt_size(dt), st);
    if (dt == kF32)
      transpose_kernel<float><<<grid, dim3(32, 8), 0, st>>>(static_cast<const float*>(W), n, k,
                                                            static_cast<float*>(W_t));
    else
      transpose_kernel<__nv_bfloat16><<<grid, dim3(32, 8), 0, st>>>(
          static_cast<const __nv_bfloat16*>(W), n, k, static_cast<__nv_bfloat16*>(W_t));
    SLORA_CHECK_LAUNCH();
  }
  return SLORA_OK;
}

}  // namespace slora
