// SVD sparsity estimator scores and top-k channel selection.
//
// SparseLoRA article, section 2 (SVD sparsity estimator): the frozen weight's
// leading singular factors, computed once offline, give a cheap estimate of a
// layer's output on the current context tokens; section 1 names the channel
// criteria (FFN: L2 norm of a neuron's activity; q/k: QK-norm built from the
// query-key product) and the per-input choice of active channels.
#include "estimator.cuh"

namespace slora {
namespace {

// ---------------------------------------------------------------- FFN score
// Each thread scores CPT channels (c = first + 128 * i) over one token chunk:
// it keeps their U_g, U_u rows in registers and reads each token's projected
// row P_g | P_u from shared memory as 16-byte broadcasts, reused for its CPT
// channels (the shared-memory reads, not the math, bounded the one-channel
// version).  With an even CPT the rank-r dot products of two channels run as
// one packed fma.rn.f32x2 per rank index (the token's projection is staged
// duplicated, {v, v}); each lane's chain is the same fused multiply-adds in
// the same order as the scalar form, so the scores are unchanged.  Partial
// sums of squares per (chunk, channel), fixed token order.
constexpr int kScoreTT = 32;  // tokens staged per round
constexpr int kSMs148 = 148;  // B200 SM count (grid sizing only)
template <int RP>
constexpr int score_cpt() { return RP <= 8 ? 4 : (RP <= 16 ? 2 : 1); }

__device__ __forceinline__ unsigned long long pack_f2(float lo, float hi) {
  unsigned long long r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
  return r;
}
__device__ __forceinline__ float2 unpack_f2(unsigned long long v) {
  float2 r;
  asm("mov.b64 {%0, %1}, %2;" : "=f"(r.x), "=f"(r.y) : "l"(v));
  return r;
}
// (a.lo * b.lo + c.lo, a.hi * b.hi + c.hi), each rounded once (fused)
__device__ __forceinline__ unsigned long long ffma2(unsigned long long a, unsigned long long b,
                                                    unsigned long long c) {
  unsigned long long d;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
  return d;
}

template <int RP>
__global__ void __launch_bounds__(128) ffn_score_partial_kernel(
    const float* __restrict__ P, int64_t ldp, const int32_t* __restrict__ pmap, int64_t T_C,
    const float* __restrict__ Ug, const float* __restrict__ Uu, int64_t n, int r, int64_t chunk,
    float* __restrict__ partial) {
  constexpr int CPT = score_cpt<RP>();
  const int64_t j0 = int64_t(blockIdx.x) * 128 * CPT + threadIdx.x;
  const int64_t t0 = int64_t(blockIdx.y) * chunk;
  const int64_t t1 = min(T_C, t0 + chunk);
  float acc[CPT];
#pragma unroll
  for (int i = 0; i < CPT; ++i) acc[i] = 0.0f;
  auto uval = [&](const float* U, int i, int q) {
    const int64_t j = j0 + 128 * i;
    return (j < n && q < r) ? U[j * r + q] : 0.0f;
  };
  auto pval = [&](int64_t tb, int tt, int nt, int q) {
    const int half = q / RP, qq = q % RP;
    if (tt >= nt || qq >= r) return 0.0f;
    const int64_t row = pmap ? int64_t(pmap[tb + tt]) : tb + tt;
    return P[row * ldp + half * r + qq];
  };
  if constexpr (CPT % 2 == 0) {
    constexpr int NPR = CPT / 2;  // channel pairs per thread
    __shared__ __align__(16) unsigned long long sp2[kScoreTT][2 * RP];
    unsigned long long ug2[NPR][RP], uu2[NPR][RP];
#pragma unroll
    for (int pr = 0; pr < NPR; ++pr)
#pragma unroll
      for (int q = 0; q < RP; ++q) {
        ug2[pr][q] = pack_f2(uval(Ug, 2 * pr, q), uval(Ug, 2 * pr + 1, q));
        uu2[pr][q] = pack_f2(uval(Uu, 2 * pr, q), uval(Uu, 2 * pr + 1, q));
      }
    for (int64_t tb = t0; tb < t1; tb += kScoreTT) {
      const int nt = int((t1 - tb) < kScoreTT ? (t1 - tb) : kScoreTT);
      __syncthreads();
      for (int e = threadIdx.x; e < kScoreTT * 2 * RP; e += blockDim.x) {
        const int tt = e / (2 * RP), q = e % (2 * RP);
        const float v = pval(tb, tt, nt, q);
        sp2[tt][q] = pack_f2(v, v);
      }
      __syncthreads();
      for (int tt = 0; tt < nt; ++tt) {
        unsigned long long pg[RP], pu[RP];
#pragma unroll
        for (int q2 = 0; q2 < RP / 2; ++q2) {
          const ulonglong2 a = *reinterpret_cast<const ulonglong2*>(&sp2[tt][2 * q2]);
          const ulonglong2 b = *reinterpret_cast<const ulonglong2*>(&sp2[tt][RP + 2 * q2]);
          pg[2 * q2] = a.x; pg[2 * q2 + 1] = a.y;
          pu[2 * q2] = b.x; pu[2 * q2 + 1] = b.y;
        }
#pragma unroll
        for (int pr = 0; pr < NPR; ++pr) {
          unsigned long long g2 = 0ull, u2 = 0ull;
#pragma unroll
          for (int q = 0; q < RP; ++q) {
            g2 = ffma2(pg[q], ug2[pr][q], g2);
            u2 = ffma2(pu[q], uu2[pr][q], u2);
          }
          const float2 g = unpack_f2(g2), u = unpack_f2(u2);
          const float a0 = silu_f(g.x) * u.x, a1 = silu_f(g.y) * u.y;
          acc[2 * pr] = fmaf(a0, a0, acc[2 * pr]);
          acc[2 * pr + 1] = fmaf(a1, a1, acc[2 * pr + 1]);
        }
      }
    }
  } else {
    __shared__ __align__(16) float sp[kScoreTT][2 * RP];
    float ug[CPT][RP], uu[CPT][RP];
#pragma unroll
    for (int i = 0; i < CPT; ++i)
#pragma unroll
      for (int q = 0; q < RP; ++q) {
        ug[i][q] = uval(Ug, i, q);
        uu[i][q] = uval(Uu, i, q);
      }
    for (int64_t tb = t0; tb < t1; tb += kScoreTT) {
      const int nt = int((t1 - tb) < kScoreTT ? (t1 - tb) : kScoreTT);
      __syncthreads();
      for (int e = threadIdx.x; e < kScoreTT * 2 * RP; e += blockDim.x)
        sp[e / (2 * RP)][e % (2 * RP)] = pval(tb, e / (2 * RP), nt, e % (2 * RP));
      __syncthreads();
      for (int tt = 0; tt < nt; ++tt) {
        float pg[RP], pu[RP];
#pragma unroll
        for (int q4 = 0; q4 < RP / 4; ++q4) {
          const float4 a = *reinterpret_cast<const float4*>(&sp[tt][4 * q4]);
          const float4 b = *reinterpret_cast<const float4*>(&sp[tt][RP + 4 * q4]);
          pg[4 * q4] = a.x; pg[4 * q4 + 1] = a.y; pg[4 * q4 + 2] = a.z; pg[4 * q4 + 3] = a.w;
          pu[4 * q4] = b.x; pu[4 * q4 + 1] = b.y; pu[4 * q4 + 2] = b.z; pu[4 * q4 + 3] = b.w;
        }
#pragma unroll
        for (int i = 0; i < CPT; ++i) {
          float g = 0.0f, u = 0.0f;
#pragma unroll
          for (int q = 0; q < RP; ++q) {
            g = fmaf(pg[q], ug[i][q], g);
            u = fmaf(pu[q], uu[i][q], u);
          }
          const float a = silu_f(g) * u;
          acc[i] = fmaf(a, a, acc[i]);
        }
      }
    }
  }
#pragma unroll
  for (int i = 0; i < CPT; ++i) {
    const int64_t j = j0 + 128 * i;
    if (j < n) partial[int64_t(blockIdx.y) * n + j] = acc[i];
  }
}

__global__ void sumsq_finalize_kernel(const float* __restrict__ partial, int nsplit, int64_t n,
                                      float* __restrict__ scores) {
  int64_t j = int64_t(blockIdx.x) * blockDim.x + threadIdx.x;
  if (j >= n) return;
  double s = 0.0;
  for (int p = 0; p < nsplit; ++p) s += double(partial[int64_t(p) * n + j]);
  scores[j] = float(sqrt(s));
}

// ----------------------------------------------------------------- QK score
// Gram partials: block (p, split) sums P_p[t,a] P_p[t,b] over its token chunk.
__global__ void qk_gram_partial_kernel(const float* __restrict__ P, int64_t ldp,
                                       const int32_t* __restrict__ pmap, int64_t T_C, int r,
                                       int64_t chunk, double* __restrict__ part) {
  const int p = blockIdx.x, sp = blockIdx.y, nsp = gridDim.y;
  const int64_t t0 = int64_t(sp) * chunk, t1 = min(T_C, t0 + chunk);
  for (int e = threadIdx.x; e < r * r; e += blockDim.x) {
    int a = e / r, b = e % r;
    double s = 0.0;
    for (int64_t t = t0; t < t1; ++t) {
      const int64_t row = pmap ? int64_t(pmap[t]) : t;
      s += double(P[row * ldp + p * r + a]) * double(P[row * ldp + p * r + b]);
    }
    part[(int64_t(p) * nsp + sp) * r * r + e] = s;
  }
}

__global__ void qk_gram_finalize_kernel(const double* __restrict__ part, int nsp, int r,
                                        double* __restrict__ gram) {
  const int p = blockIdx.x;
  for (int e = threadIdx.x; e < r * r; e += blockDim.x) {
    double s = 0.0;
    for (int sp = 0; sp < nsp; ++sp) s += part[(int64_t(p) * nsp + sp) * r * r + e];
    gram[int64_t(p) * r * r + e] = s;
  }
}

__device__ double quad_form(const double* G, const float* u, int r) {
  double s = 0.0;
  for (int a = 0; a < r; ++a) {
    double ga = 0.0;
    for (int b = 0; b < r; ++b) ga += G[a * r + b] * double(u[b]);
    s += double(u[a]) * ga;
  }
  return s > 0.0 ? s : 0.0;
}

__global__ void qk_score_kernel(const double* __restrict__ gram, const float* __restrict__ Uq,
                                const float* __restrict__ Uk, int r, int heads, int kv_heads,
                                int head_dim, float* __restrict__ scores) {
  int64_t e = int64_t(blockIdx.x) * blockDim.x + threadIdx.x;
  if (e >= int64_t(kv_heads) * head_dim) return;
  const int g = int(e / head_dim), c = int(e % head_dim);
  const int rep = heads / kv_heads;
  const double* Gq = gram;
  const double* Gk = gram + r * r;
  double qs = 0.0;
  for (int j = 0; j < rep; ++j) {
    int h = g * rep + j;
    qs += sqrt(quad_form(Gq, Uq + (int64_t(h) * head_dim + c) * r, r));
  }
  double nk = sqrt(quad_form(Gk, Uk + (int64_t(g) * head_dim + c) * r, r));
  scores[e] = float(nk * qs);
}

// ----------------------------------------------------------------- select
// Radix select on the fp32 bit pattern (scores are >= 0, so unsigned order of
// the bits is numeric order), 4 passes of 8 bits, then an index-ordered
// compaction with ballot scans so the output is ascending and equal scores
// go to the lower index.
__device__ __forceinline__ uint32_t score_key(float v) {
  uint32_t b = __float_as_uint(v);
  if (b & 0x80000000u) b = 0;   // -0 (or a negative) ranks as zero
  if (b > 0x7f800000u) b = 0;   // NaN ranks lowest
  return b;
}

__global__ void __launch_bounds__(1024) topk_select_kernel(const float* __restrict__ scores,
                                                           int N, int k, int rep,
                                                           int32_t* __restrict__ out_a,
                                                           int32_t* __restrict__ out_b) {
  const int g = blockIdx.x;
  const float* sc = scores + int64_t(g) * N;
  __shared__ uint32_t hist[256];
  __shared__ uint32_t s_prefix, s_want;
  __shared__ uint32_t warp_sel[32], warp_eq[32];
  __shared__ uint32_t s_base, s_tie;
  const int tid = threadIdx.x, lane = tid & 31, wid = tid >> 5, nw = blockDim.x >> 5;
  if (k <= 0) return;
  if (tid == 0) { s_prefix = 0; s_want = uint32_t(k); }
  for (int pass = 0; pass < 4; ++pass) {
    const int shift = 24 - 8 * pass;
    const uint32_t hi_mask = pass == 0 ? 0u : (0xffffffffu << (32 - 8 * pass));
    for (int i = tid; i < 256; i += blockDim.x) hist[i] = 0;
    __syncthreads();
    const uint32_t prefix = s_prefix;
    for (int j = tid; j < N; j += blockDim.x) {
      uint32_t key = score_key(sc[j]);
      if ((key & hi_mask) == prefix) atomicAdd(&hist[(key >> shift) & 255u], 1u);
    }
    __syncthreads();
    if (wid == 0) {  // the digit holding the want-th largest key: a warp-parallel scan
      // lane l owns digits 255 - 8l down to 248 - 8l (descending key order)
      const uint32_t want = s_want;
      uint32_t own = 0;
#pragma unroll
      for (int i = 0; i < 8; ++i) own += hist[255 - 8 * lane - i];
      uint32_t incl = own;  // inclusive prefix over lanes 0..l
#pragma unroll
      for (int off = 1; off < 32; off <<= 1) {
        const uint32_t o = __shfl_up_sync(0xffffffffu, incl, off);
        if (lane >= off) incl += o;
      }
      const uint32_t hit = __ballot_sync(0xffffffffu, incl >= want);
      const int l = __ffs(hit) - 1;  // want <= count of keys with this prefix, so l exists
      if (lane == l) {
        uint32_t cum = incl - own;
        for (int i = 0; i < 8; ++i) {
          const int dg = 255 - 8 * lane - i;
          const uint32_t h = hist[dg];
          if (cum + h >= want) {
            s_prefix = prefix | (uint32_t(dg) << shift);
            s_want = want - cum;
            break;
          }
          cum += h;
        }
      }
    }
    __syncthreads();
  }
  const uint32_t tau = s_prefix, want = s_want;  // take `want` of the keys equal to tau
  if (tid == 0) { s_base = 0; s_tie = 0; }
  __syncthreads();
  for (int c0 = 0; c0 < N; c0 += blockDim.x) {
    const int j = c0 + tid;
    uint32_t key = j < N ? score_key(sc[j]) : 0u;
    const bool gt = j < N && key > tau;
    const bool eq = j < N && key == tau;
    // exclusive rank of this lane among the block's ties
    uint32_t beq = __ballot_sync(0xffffffffu, eq);
    if (lane == 0) warp_eq[wid] = __popc(beq);
    __syncthreads();
    uint32_t tie_before = s_tie;
    for (int w = 0; w < wid; ++w) tie_before += warp_eq[w];
    tie_before += __popc(beq & ((1u << lane) - 1u));
    const bool sel = gt || (eq && tie_before < want);
    uint32_t bsel = __ballot_sync(0xffffffffu, sel);
    if (lane == 0) warp_sel[wid] = __popc(bsel);
    __syncthreads();
    uint32_t pos = s_base;
    for (int w = 0; w < wid; ++w) pos += warp_sel[w];
    pos += __popc(bsel & ((1u << lane) - 1u));
    if (sel) {
      for (int q = 0; q < rep; ++q) {
        const int h = g * rep + q;
        out_a[int64_t(h) * k + pos] = h * N + j;
      }
      if (out_b) out_b[int64_t(g) * k + pos] = g * N + j;
    }
    __syncthreads();
    if (tid == 0) {
      uint32_t ts = 0, te = 0;
      for (int w = 0; w < nw; ++w) { ts += warp_sel[w]; te += warp_eq[w]; }
      s_base += ts;
      s_tie += te;
    }
    __syncthreads();
  }
}

}  // namespace

int score_cpt_for(int r) { return r <= 8 ? 4 : (r <= 16 ? 2 : 1); }

// Resident 128-thread score blocks per SM for the kernel serving rank r
// (register-limited; 4 if the query fails).
int score_blocks_per_sm(int r) {
  static int cached[4] = {0, 0, 0, 0};
  const int slot = r <= 8 ? 0 : (r <= 16 ? 1 : (r <= 32 ? 2 : 3));
  if (!cached[slot]) {
    int b = 0;
    cudaError_t e;
    switch (slot) {
      case 0: e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&b, ffn_score_partial_kernel<8>, 128, 0); break;
      case 1: e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&b, ffn_score_partial_kernel<16>, 128, 0); break;
      case 2: e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&b, ffn_score_partial_kernel<32>, 128, 0); break;
      default: e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&b, ffn_score_partial_kernel<48>, 128, 0); break;
    }
    if (e != cudaSuccess || b < 1) {
      cudaGetLastError();
      b = 4;
    }
    cached[slot] = b;
  }
  return cached[slot];
}

// Token splits: as many as keep the grid within one wave of resident blocks
// (a second, partial wave cost more than the split's extra partial sums).
int ffn_score_splits(int64_t T_C, int64_t n, int r) {
  const int64_t nb = (n + 128 * score_cpt_for(r) - 1) / (128 * score_cpt_for(r));
  const int64_t slots = int64_t(kSMs148) * score_blocks_per_sm(r);
  int64_t want = slots / std::max<int64_t>(nb, 1);
  int64_t maxs = (T_C + kScoreTT - 1) / kScoreTT;
  int64_t s = want < maxs ? want : maxs;
  if (s < 1) s = 1;
  if (s > 64) s = 64;
  return int(s);
}

slora_status ffn_scores(const float* P, int64_t ldp, const int32_t* pmap, int64_t T_C,
                        const float* Ug, const float* Uu, int64_t n, int r, float* partial,
                        int nsplit, float* scores, cudaStream_t st) {
  if (n <= 0) return SLORA_OK;
  const int64_t chunk = T_C > 0 ? (T_C + nsplit - 1) / nsplit : 1;
  dim3 grid(unsigned((n + 128 * score_cpt_for(r) - 1) / (128 * score_cpt_for(r))),
            unsigned(nsplit));
  {
  LaunchScope ls(kEstimate, double(T_C) * 2 * r * 4 + double(n) * 2 * r * 4 + double(nsplit) * n * 4, st);
  if (r <= 8)
    ffn_score_partial_kernel<8><<<grid, 128, 0, st>>>(P, ldp, pmap, T_C, Ug, Uu, n, r, chunk,
                                                         partial);
  else if (r <= 16)
    ffn_score_partial_kernel<16><<<grid, 128, 0, st>>>(P, ldp, pmap, T_C, Ug, Uu, n, r, chunk,
                                                         partial);
  else if (r <= 32)
    ffn_score_partial_kernel<32><<<grid, 128, 0, st>>>(P, ldp, pmap, T_C, Ug, Uu, n, r, chunk,
                                                         partial);
  else
    ffn_score_partial_kernel<48><<<grid, 128, 0, st>>>(P, ldp, pmap, T_C, Ug, Uu, n, r, chunk,
                                                         partial);
  }
  SLORA_CHECK_LAUNCH();
  LaunchScope ls2(kEstimate, double(nsplit) * n * 4 + double(n) * 4, st);
  sumsq_finalize_kernel<<<unsigned((n + 255) / 256), 256, 0, st>>>(partial, nsplit, n, scores);
  SLORA_CHECK_LAUNCH();
  return SLORA_OK;
}

slora_status qk_scores(const float* P, int64_t ldp, const int32_t* pmap, int64_t T_C,
                       const float* Uq,
                       const float* Uk, int r, int heads, int kv_heads, int head_dim,
                       double* gram, float* scores, cudaStream_t st) {
  constexpr int kSplits = 32;
  double* part = gram + 2 * r * r;  // caller reserves 2*r*r*(1 + kSplits) doubles
  const int64_t chunk = T_C > 0 ? (T_C + kSplits - 1) / kSplits : 1;
  {
  LaunchScope ls(kEstimate, double(T_C) * 2 * r * 4, st);
  qk_gram_partial_kernel<<<dim3(2, kSplits), 256, 0, st>>>(P, ldp, pmap, T_C, r, chunk, part);
  SLORA_CHECK_LAUNCH();
  }
  SLORA_CHECK_LAUNCH();
  {
  LaunchScope ls(kEstimate, double(kSplits) * 2 * r * r * 8, st);
  qk_gram_finalize_kernel<<<2, 256, 0, st>>>(part, kSplits, r, gram);
  }
  SLORA_CHECK_LAUNCH();
  const int64_t nsc = int64_t(kv_heads) * head_dim;
  LaunchScope ls(kEstimate, double(heads + kv_heads) * head_dim * r * 4 + double(nsc) * 4, st);
  qk_score_kernel<<<unsigned((nsc + 127) / 128), 128, 0, st>>>(gram, Uq, Uk, r, heads, kv_heads,
                                                                head_dim, scores);
  SLORA_CHECK_LAUNCH();
  return SLORA_OK;
}

slora_status topk_select(const float* scores, int groups, int N, int k, int rep,
                         int32_t* out_a, int32_t* out_b, cudaStream_t st) {
  if (k <= 0 || groups <= 0) return SLORA_OK;
  LaunchScope ls(kSelect, double(groups) * N * 4 * 5 + double(groups) * k * 4 * (rep + 1), st);
  topk_select_kernel<<<groups, 1024, 0, st>>>(scores, N, k, rep, out_a, out_b);
  SLORA_CHECK_LAUNCH();
  return SLORA_OK;
}

}  // namespace slora
