// The attention core of a decoder layer around the sparse q/k projections:
// rotary embedding of the assembled q/k rows and causal softmax attention,
// forward and backward, per sequence with grouped key/value heads.
//
// Where it sits (SparseLoRA article, section 1: q/k channels kept per head by
// the query-key product; section 3: context tokens sparse, output tokens
// dense).  A context row's skipped q/k channels are not computed, so the core
// reads them as zeros: rope_pack_kernel scatters the compact context rows
// (channels idx) and the dense output rows into full-width rows, zero
// elsewhere, and rotates each head's rotate-half pairs (i, i + hd/2) by the
// row's position angle in the same pass.  rope_unpack_kernel is its
// transpose: it rotates the core's fp32 gradient back and gathers the kept
// channels of the context rows (the skipped ones have no computed output, so
// their gradient goes nowhere) and every channel of the output rows.
//
// attn_fwd_kernel: one 128-thread block per (64 query rows, query head,
// sequence); each warp owns 16 query rows with its Q fragments in registers,
// streams 64-key K/V tiles through a two-stage cp.async pipeline in swizzled
// shared memory, and runs S = Q K^T and O += P V on mma.sync m16n8k16 (bf16 in,
// fp32 accumulate) with the online softmax in between (P reused from the S
// accumulators as the A operand).  Writes O (bf16) and the natural-log
// log-sum-exp of each row's scaled scores.
//
// attn_bwd_kernel: one block per (64 keys, key/value head, sequence); each warp
// owns 16 keys, keeps dK and dV for them in registers across every query head
// of the group and every query tile at or after the keys (causal), and per
// tile recomputes S^T = K Q^T, P^T from the saved log-sum-exp, dV += P^T dO,
// dP^T = V dO^T, dS^T = P^T (dP^T - D), dK += dS^T Q, and dQ += dS K through
// shared memory, added into an fp32 accumulator with vector reductions
// (their order across key tiles is not fixed).  D = rowsum(dO * O) comes from
// attn_rowdot_kernel.
#include <algorithm>
#include <cmath>

#include "attention.cuh"

namespace slora {
namespace {

constexpr int kBM = 64;   // query rows per block (forward) / per tile (backward)
constexpr int kBN = 64;   // keys per tile (forward) / per block (backward)
constexpr int kThreads = 128;
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;
constexpr float kNegBig = -1.0e30f;  // masked score: exp2 of it minus any row max is 0

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}
__device__ __forceinline__ void cp16(uint32_t dst, const void* src, int bytes) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(bytes)
               : "memory");
}
__device__ __forceinline__ void cp_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}
__device__ __forceinline__ void ldsm4(uint32_t addr, uint32_t (&r)[4]) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr));
}
__device__ __forceinline__ void ldsm4t(uint32_t addr, uint32_t (&r)[4]) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr));
}
__device__ __forceinline__ void mma16816(float (&c)[4], const uint32_t (&a)[4], uint32_t b0,
                                         uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
      "{%8,%9}, {%0,%1,%2,%3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}
__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}
__device__ __forceinline__ float fast_exp2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}
__device__ __forceinline__ void red_add_v2(float* p, float a, float b) {
  asm volatile("red.global.add.v2.f32 [%0], {%1, %2};" ::"l"(p), "f"(a), "f"(b) : "memory");
}

// Byte offset of 16-byte chunk c of row r in a tile whose rows hold CH
// chunks, XOR-swizzled so that the 8 rows one ldmatrix reads at a fixed
// logical chunk land on 8 different bank groups.
template <int CH>
__device__ __forceinline__ uint32_t swz(int r, int c) {
  return uint32_t(r * CH * 16 + ((c ^ (r & 7)) << 4));
}

// Copies `rows` rows of HD bf16 (row stride ld elements) starting at global
// row g0 into a swizzled [kBM x HD] tile; rows at or past `valid` are zero.
template <int HD>
__device__ __forceinline__ void load_tile(uint32_t tile, const __nv_bfloat16* base, int64_t ld,
                                          int valid) {
  constexpr int CH = HD / 8;
  for (int i = threadIdx.x; i < kBM * CH; i += kThreads) {
    const int r = i / CH, c = i % CH;
    const bool ok = r < valid;
    const __nv_bfloat16* src = ok ? base + int64_t(r) * ld + c * 8 : base;
    cp16(tile + swz<CH>(r, c), src, ok ? 16 : 0);
  }
}

// ------------------------------------------------------------------ rotary
__global__ void rope_table_kernel(float2* tab, int seq, int half, double base) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= seq * half) return;
  const int p = i / half, j = i % half;
  const double inv = pow(base, -double(2 * j) / double(2 * half));
  double s, c;
  sincos(double(p) * inv, &s, &c);
  tab[i] = make_float2(float(c), float(s));
}

// rowkind[t] = compact context row of full row t, or -1 - (its output row).
__global__ void rowkind_kernel(const int32_t* __restrict__ ctx_rows, int64_t TC,
                               const int32_t* __restrict__ out_rows, int64_t TO,
                               int32_t* __restrict__ kind) {
  const int64_t i = int64_t(blockIdx.x) * blockDim.x + threadIdx.x;
  if (i < TC) kind[ctx_rows[i]] = int32_t(i);
  else if (i < TC + TO) kind[out_rows[i - TC]] = int32_t(-1 - (i - TC));
}

// inv[ch] = position of channel ch in idx, or -1: a fill of -1, then (the
// next launch on the stream) the scatter of the positions.
__global__ void inverse_fill_kernel(int n, int32_t* __restrict__ inv) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i < n) inv[i] = -1;
}
__global__ void inverse_scatter_kernel(const int32_t* __restrict__ idx, int n_idx, int n,
                                       int32_t* __restrict__ inv) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i < n_idx) {
    const int ch = idx[i];
    if (ch >= 0 && ch < n) inv[ch] = i;
  }
}

// One thread per (row, head, two consecutive pairs).  Dense mode (kind ==
// nullptr): Y is [T x n].  Sliced mode: context rows read Yc [T_C x n_idx]
// through inv, output rows Yo [T_O x n].
__global__ void rope_pack_kernel(const __nv_bfloat16* __restrict__ Y,
                                 const __nv_bfloat16* __restrict__ Yc,
                                 const __nv_bfloat16* __restrict__ Yo,
                                 const int32_t* __restrict__ kind,
                                 const int32_t* __restrict__ inv, int n_idx, int64_t T, int n,
                                 int hd, int seq, const float2* __restrict__ tab,
                                 __nv_bfloat16* __restrict__ out) {
  const int half = hd / 2, hp = half / 2;  // pair couples per head
  const int64_t i = int64_t(blockIdx.x) * blockDim.x + threadIdx.x;
  const int64_t per_row = int64_t(n / hd) * hp;
  if (i >= T * per_row) return;
  const int64_t t = i / per_row;
  const int rem = int(i % per_row);
  const int h = rem / hp, j = (rem % hp) * 2;
  const int ch = h * hd + j;
  float a0, a1, b0, b1;
  if (!kind) {
    const __nv_bfloat16* y = Y + t * n;
    const __nv_bfloat162 va = *reinterpret_cast<const __nv_bfloat162*>(y + ch);
    const __nv_bfloat162 vb = *reinterpret_cast<const __nv_bfloat162*>(y + ch + half);
    a0 = __low2float(va); a1 = __high2float(va); b0 = __low2float(vb); b1 = __high2float(vb);
  } else {
    const int k = kind[t];
    if (k < 0) {
      const __nv_bfloat16* y = Yo + int64_t(-1 - k) * n;
      const __nv_bfloat162 va = *reinterpret_cast<const __nv_bfloat162*>(y + ch);
      const __nv_bfloat162 vb = *reinterpret_cast<const __nv_bfloat162*>(y + ch + half);
      a0 = __low2float(va); a1 = __high2float(va); b0 = __low2float(vb); b1 = __high2float(vb);
    } else {
      const __nv_bfloat16* y = Yc + int64_t(k) * n_idx;
      auto g = [&](int c) { const int q = inv[c]; return q >= 0 ? __bfloat162float(y[q]) : 0.f; };
      a0 = g(ch); a1 = g(ch + 1); b0 = g(ch + half); b1 = g(ch + half + 1);
    }
  }
  const int p = int(t % seq);
  const float2 r0 = tab[p * half + j], r1 = tab[p * half + j + 1];
  __nv_bfloat16* o = out + t * n;
  *reinterpret_cast<__nv_bfloat162*>(o + ch) =
      __floats2bfloat162_rn(a0 * r0.x - b0 * r0.y, a1 * r1.x - b1 * r1.y);
  *reinterpret_cast<__nv_bfloat162*>(o + ch + half) =
      __floats2bfloat162_rn(b0 * r0.x + a0 * r0.y, b1 * r1.x + a1 * r1.y);
}

// Transpose of rope_pack_kernel on an fp32 gradient G [T x n].
__global__ void rope_unpack_kernel(const float* __restrict__ G, const int32_t* __restrict__ kind,
                                   const int32_t* __restrict__ inv, int n_idx, int64_t T, int n,
                                   int hd, int seq, const float2* __restrict__ tab,
                                   __nv_bfloat16* __restrict__ dY,
                                   __nv_bfloat16* __restrict__ dYc,
                                   __nv_bfloat16* __restrict__ dYo) {
  const int half = hd / 2, hp = half / 2;
  const int64_t i = int64_t(blockIdx.x) * blockDim.x + threadIdx.x;
  const int64_t per_row = int64_t(n / hd) * hp;
  if (i >= T * per_row) return;
  const int64_t t = i / per_row;
  const int rem = int(i % per_row);
  const int h = rem / hp, j = (rem % hp) * 2;
  const int ch = h * hd + j;
  const float* g = G + t * n;
  const float2 ga = *reinterpret_cast<const float2*>(g + ch);
  const float2 gb = *reinterpret_cast<const float2*>(g + ch + half);
  const int p = int(t % seq);
  const float2 r0 = tab[p * half + j], r1 = tab[p * half + j + 1];
  // rotation by -angle: a' = a c + b s, b' = b c - a s
  const float a0 = ga.x * r0.x + gb.x * r0.y, a1 = ga.y * r1.x + gb.y * r1.y;
  const float b0 = gb.x * r0.x - ga.x * r0.y, b1 = gb.y * r1.x - ga.y * r1.y;
  if (!kind) {
    __nv_bfloat16* o = dY + t * n;
    *reinterpret_cast<__nv_bfloat162*>(o + ch) = __floats2bfloat162_rn(a0, a1);
    *reinterpret_cast<__nv_bfloat162*>(o + ch + half) = __floats2bfloat162_rn(b0, b1);
    return;
  }
  const int k = kind[t];
  if (k < 0) {
    __nv_bfloat16* o = dYo + int64_t(-1 - k) * n;
    *reinterpret_cast<__nv_bfloat162*>(o + ch) = __floats2bfloat162_rn(a0, a1);
    *reinterpret_cast<__nv_bfloat162*>(o + ch + half) = __floats2bfloat162_rn(b0, b1);
    return;
  }
  __nv_bfloat16* o = dYc + int64_t(k) * n_idx;
  const float v[4] = {a0, a1, b0, b1};
  const int c[4] = {ch, ch + 1, ch + half, ch + half + 1};
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    const int q = inv[c[e]];
    if (q >= 0) o[q] = __float2bfloat16_rn(v[e]);
  }
}

// ------------------------------------------------------------- forward
struct AttnFwdP {
  const __nv_bfloat16 *Q, *K, *V;
  __nv_bfloat16* O;
  float* lse;  // [batch][H][seq]
  int seq, H, KV, nqb;
  float sl2;   // softmax scale * log2(e)
};

template <int HD>
__global__ void __launch_bounds__(kThreads, 2) attn_fwd_kernel(const __grid_constant__ AttnFwdP p) {
  constexpr int CH = HD / 8, KS = HD / 16, NT = HD / 8;
  extern __shared__ __align__(128) unsigned char smem[];
  const uint32_t sQ = smem_u32(smem);
  const uint32_t sK0 = sQ + kBM * HD * 2;
  const uint32_t sV0 = sK0 + 2 * kBN * HD * 2;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int qb = p.nqb - 1 - int(blockIdx.x);  // longest causal rows first
  const int h = blockIdx.y, b = blockIdx.z, g = h / (p.H / p.KV);
  const int64_t ldq = int64_t(p.H) * HD, ldk = int64_t(p.KV) * HD;
  const int64_t row0 = int64_t(b) * p.seq;
  const int q0 = qb * kBM;
  const __nv_bfloat16* Qb = p.Q + (row0 + q0) * ldq + h * HD;
  const __nv_bfloat16* Kb = p.K + row0 * ldk + g * HD;
  const __nv_bfloat16* Vb = p.V + row0 * ldk + g * HD;
  const int nkb = min(qb + 1, (p.seq + kBN - 1) / kBN);

  load_tile<HD>(sQ, Qb, ldq, p.seq - q0);
  load_tile<HD>(sK0, Kb, ldk, p.seq);
  load_tile<HD>(sV0, Vb, ldk, p.seq);
  cp_commit();

  uint32_t qf[KS][4];
  float o[NT][4];
#pragma unroll
  for (int i = 0; i < NT; ++i) o[i][0] = o[i][1] = o[i][2] = o[i][3] = 0.f;
  float m0 = kNegBig, m1 = kNegBig, l0 = 0.f, l1 = 0.f;
  const int r_lo = warp * 16 + (lane >> 2);       // this thread's rows in the tile
  const int qi0 = q0 + r_lo, qi1 = qi0 + 8;       // their positions in the sequence

  for (int j = 0; j < nkb; ++j) {
    const int st = j & 1;
    if (j + 1 < nkb) {
      const int k1 = (j + 1) * kBN;
      load_tile<HD>(sK0 + (st ^ 1) * kBN * HD * 2, Kb + int64_t(k1) * ldk, ldk, p.seq - k1);
      load_tile<HD>(sV0 + (st ^ 1) * kBN * HD * 2, Vb + int64_t(k1) * ldk, ldk, p.seq - k1);
      cp_commit();
      cp_wait<1>();
    } else {
      cp_wait<0>();
    }
    __syncthreads();
    if (j == 0) {
#pragma unroll
      for (int kk = 0; kk < KS; ++kk)
        ldsm4(sQ + swz<CH>(warp * 16 + (lane & 15), kk * 2 + (lane >> 4)), qf[kk]);
    }
    const uint32_t sK = sK0 + st * kBN * HD * 2, sV = sV0 + st * kBN * HD * 2;
    // S = Q K^T for this warp's 16 rows x 64 keys
    float s[8][4];
#pragma unroll
    for (int i = 0; i < 8; ++i) s[i][0] = s[i][1] = s[i][2] = s[i][3] = 0.f;
#pragma unroll
    for (int kk = 0; kk < KS; ++kk) {
#pragma unroll
      for (int nt = 0; nt < 8; nt += 2) {
        uint32_t bf[4];
        ldsm4(sK + swz<CH>(nt * 8 + (lane & 7) + ((lane >> 4) << 3), kk * 2 + ((lane >> 3) & 1)),
              bf);
        mma16816(s[nt], qf[kk], bf[0], bf[1]);
        mma16816(s[nt + 1], qf[kk], bf[2], bf[3]);
      }
    }
    // scale into the log2 domain, mask, online softmax
    const int kbase = j * kBN + (lane & 3) * 2;
    const bool edge = (j == nkb - 1) || (j * kBN + kBN > p.seq);
    float mx0 = kNegBig, mx1 = kNegBig;
#pragma unroll
    for (int nt = 0; nt < 8; ++nt) {
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const int kidx = kbase + nt * 8 + e;
        float v0 = s[nt][e] * p.sl2, v1 = s[nt][2 + e] * p.sl2;
        if (edge) {
          if (kidx > qi0 || kidx >= p.seq) v0 = kNegBig;
          if (kidx > qi1 || kidx >= p.seq) v1 = kNegBig;
        }
        s[nt][e] = v0;
        s[nt][2 + e] = v1;
        mx0 = fmaxf(mx0, v0);
        mx1 = fmaxf(mx1, v1);
      }
    }
    mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 1));
    mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 2));
    mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 1));
    mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 2));
    const float mn0 = fmaxf(m0, mx0), mn1 = fmaxf(m1, mx1);
    const float c0 = fast_exp2(m0 - mn0), c1 = fast_exp2(m1 - mn1);
    m0 = mn0;
    m1 = mn1;
    float rs0 = 0.f, rs1 = 0.f;
#pragma unroll
    for (int nt = 0; nt < 8; ++nt) {
      s[nt][0] = fast_exp2(s[nt][0] - mn0);
      s[nt][1] = fast_exp2(s[nt][1] - mn0);
      s[nt][2] = fast_exp2(s[nt][2] - mn1);
      s[nt][3] = fast_exp2(s[nt][3] - mn1);
      rs0 += s[nt][0] + s[nt][1];
      rs1 += s[nt][2] + s[nt][3];
    }
    l0 = l0 * c0 + rs0;
    l1 = l1 * c1 + rs1;
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
      o[nt][0] *= c0; o[nt][1] *= c0; o[nt][2] *= c1; o[nt][3] *= c1;
    }
    // O += P V: P (bf16) straight from the S accumulators as A fragments
#pragma unroll
    for (int kk = 0; kk < 4; ++kk) {
      uint32_t pa[4];
      pa[0] = pack_bf16(s[2 * kk][0], s[2 * kk][1]);
      pa[1] = pack_bf16(s[2 * kk][2], s[2 * kk][3]);
      pa[2] = pack_bf16(s[2 * kk + 1][0], s[2 * kk + 1][1]);
      pa[3] = pack_bf16(s[2 * kk + 1][2], s[2 * kk + 1][3]);
#pragma unroll
      for (int nt = 0; nt < NT; nt += 2) {
        uint32_t bf[4];
        ldsm4t(sV + swz<CH>(kk * 16 + (lane & 7) + (((lane >> 3) & 1) << 3), nt + (lane >> 4)),
               bf);
        mma16816(o[nt], pa, bf[0], bf[1]);
        mma16816(o[nt + 1], pa, bf[2], bf[3]);
      }
    }
    __syncthreads();  // this stage is refilled by the next iteration's prefetch
  }
  // the row sums live split over the quad's four lanes
  l0 += __shfl_xor_sync(0xffffffffu, l0, 1);
  l0 += __shfl_xor_sync(0xffffffffu, l0, 2);
  l1 += __shfl_xor_sync(0xffffffffu, l1, 1);
  l1 += __shfl_xor_sync(0xffffffffu, l1, 2);
  const float inv0 = 1.f / l0, inv1 = 1.f / l1;
  const int cb = (lane & 3) * 2;
  if (qi0 < p.seq) {
    __nv_bfloat16* orow = p.O + (row0 + qi0) * ldq + h * HD;
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
      *reinterpret_cast<__nv_bfloat162*>(orow + nt * 8 + cb) =
          __floats2bfloat162_rn(o[nt][0] * inv0, o[nt][1] * inv0);
    if ((lane & 3) == 0) p.lse[(int64_t(b) * p.H + h) * p.seq + qi0] = (m0 + log2f(l0)) * kLn2;
  }
  if (qi1 < p.seq) {
    __nv_bfloat16* orow = p.O + (row0 + qi1) * ldq + h * HD;
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
      *reinterpret_cast<__nv_bfloat162*>(orow + nt * 8 + cb) =
          __floats2bfloat162_rn(o[nt][2] * inv1, o[nt][3] * inv1);
    if ((lane & 3) == 0) p.lse[(int64_t(b) * p.H + h) * p.seq + qi1] = (m1 + log2f(l1)) * kLn2;
  }
}

// ------------------------------------------------------------ backward
// D[b][h][t] = sum_c dO[t, h HD + c] O[t, h HD + c]: one warp per (row, head).
template <int HD>
__global__ void attn_rowdot_kernel(const __nv_bfloat16* __restrict__ dO,
                                   const __nv_bfloat16* __restrict__ O, int64_t T, int H, int seq,
                                   float* __restrict__ D) {
  const int64_t w = (int64_t(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (w >= T * H) return;
  const int64_t t = w / H;
  const int h = int(w % H);
  const int64_t off = t * int64_t(H) * HD + int64_t(h) * HD;
  float acc = 0.f;
#pragma unroll
  for (int c = lane * 2; c < HD; c += 64) {
    const __nv_bfloat162 a = *reinterpret_cast<const __nv_bfloat162*>(dO + off + c);
    const __nv_bfloat162 o = *reinterpret_cast<const __nv_bfloat162*>(O + off + c);
    acc += __low2float(a) * __low2float(o) + __high2float(a) * __high2float(o);
  }
#pragma unroll
  for (int s = 16; s; s >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, s);
  if (lane == 0) {
    const int64_t b = t / seq;
    D[(b * H + h) * seq + (t % seq)] = acc;
  }
}

struct AttnBwdP {
  const __nv_bfloat16 *Q, *K, *V, *dO;
  const float *lse, *D;  // [batch][H][seq]
  float* dQ;             // [T x H HD] fp32, accumulated
  float* dK;             // [T x KV HD] fp32
  __nv_bfloat16* dV;     // [T x KV HD]
  int seq, H, KV, nqb;
  float sl2, scale;
};

__device__ __forceinline__ void cp4(uint32_t dst, const void* src, int bytes) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 4, %2;" ::"r"(dst), "l"(src), "r"(bytes)
               : "memory");
}
__device__ __forceinline__ void st_shared_u32(uint32_t addr, uint32_t v) {
  asm volatile("st.shared.u32 [%0], %1;" ::"r"(addr), "r"(v) : "memory");
}

template <int HD>
__global__ void __launch_bounds__(kThreads, 2) attn_bwd_kernel(const __grid_constant__ AttnBwdP p) {
  constexpr int CH = HD / 8, KS = HD / 16, NT = HD / 8, TILE = kBM * HD * 2;
  extern __shared__ __align__(128) unsigned char smem[];
  const uint32_t sK = smem_u32(smem), sV = sK + TILE, sQ0 = sV + TILE, sO0 = sQ0 + 2 * TILE;
  const uint32_t sS = sO0 + 2 * TILE;          // dS^T [64 keys x 64 queries] bf16
  const uint32_t sL0 = sS + kBN * kBM * 2;     // lse [2][64]
  const uint32_t sD0 = sL0 + 2 * kBM * 4;      // D   [2][64]
  const float* fL = reinterpret_cast<const float*>(smem + (sL0 - sK));
  const float* fD = reinterpret_cast<const float*>(smem + (sD0 - sK));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int kb = blockIdx.x, g = blockIdx.y, b = blockIdx.z;
  const int grp = p.H / p.KV, k0 = kb * kBN;
  const int64_t ldq = int64_t(p.H) * HD, ldk = int64_t(p.KV) * HD;
  const int64_t row0 = int64_t(b) * p.seq;
  const int nq = p.nqb - kb, niter = grp * nq;

  load_tile<HD>(sK, p.K + (row0 + k0) * ldk + g * HD, ldk, p.seq - k0);
  load_tile<HD>(sV, p.V + (row0 + k0) * ldk + g * HD, ldk, p.seq - k0);
  auto issue = [&](int it, int st) {
    const int hq = g * grp + it / nq, q0 = (kb + it % nq) * kBM;
    load_tile<HD>(sQ0 + st * TILE, p.Q + (row0 + q0) * ldq + hq * HD, ldq, p.seq - q0);
    load_tile<HD>(sO0 + st * TILE, p.dO + (row0 + q0) * ldq + hq * HD, ldq, p.seq - q0);
    const int t = threadIdx.x & 63;
    const bool ok = q0 + t < p.seq;
    const int64_t li = (int64_t(b) * p.H + hq) * p.seq + (ok ? q0 + t : 0);
    if (threadIdx.x < 64) cp4(sL0 + (st * kBM + t) * 4, p.lse + li, ok ? 4 : 0);
    else cp4(sD0 + (st * kBM + t) * 4, p.D + li, ok ? 4 : 0);
  };
  issue(0, 0);
  cp_commit();

  float dk[NT][4], dv[NT][4];
#pragma unroll
  for (int i = 0; i < NT; ++i)
#pragma unroll
    for (int e = 0; e < 4; ++e) dk[i][e] = dv[i][e] = 0.f;
  const int kr0 = k0 + warp * 16 + (lane >> 2), kr1 = kr0 + 8;  // this thread's keys
  const int cq = (lane & 3) * 2;

  for (int it = 0; it < niter; ++it) {
    const int st = it & 1;
    if (it + 1 < niter) {
      issue(it + 1, st ^ 1);
      cp_commit();
      cp_wait<1>();
    } else {
      cp_wait<0>();
    }
    __syncthreads();
    const int hq = g * grp + it / nq, q0 = (kb + it % nq) * kBM;
    const uint32_t sQ = sQ0 + st * TILE, sO = sO0 + st * TILE;
    const float* L = fL + st * kBM;
    const float* Dv = fD + st * kBM;
    // S^T = K Q^T: this warp's 16 keys x 64 queries
    float s[8][4];
#pragma unroll
    for (int i = 0; i < 8; ++i) s[i][0] = s[i][1] = s[i][2] = s[i][3] = 0.f;
#pragma unroll
    for (int kk = 0; kk < KS; ++kk) {
      uint32_t ka[4];
      ldsm4(sK + swz<CH>(warp * 16 + (lane & 15), kk * 2 + (lane >> 4)), ka);
#pragma unroll
      for (int nt = 0; nt < 8; nt += 2) {
        uint32_t bf[4];
        ldsm4(sQ + swz<CH>(nt * 8 + (lane & 7) + ((lane >> 4) << 3), kk * 2 + ((lane >> 3) & 1)),
              bf);
        mma16816(s[nt], ka, bf[0], bf[1]);
        mma16816(s[nt + 1], ka, bf[2], bf[3]);
      }
    }
    // P^T from the saved log-sum-exp; causal: key <= query < seq
#pragma unroll
    for (int nt = 0; nt < 8; ++nt) {
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const int qc = nt * 8 + cq + e, qi = q0 + qc;
        const float l2 = L[qc] * kLog2e;
        const bool in = qi < p.seq;
        s[nt][e] = (in && kr0 <= qi) ? fast_exp2(s[nt][e] * p.sl2 - l2) : 0.f;
        s[nt][2 + e] = (in && kr1 <= qi) ? fast_exp2(s[nt][2 + e] * p.sl2 - l2) : 0.f;
      }
    }
    // dV += P^T dO
#pragma unroll
    for (int kk = 0; kk < 4; ++kk) {
      uint32_t pa[4];
      pa[0] = pack_bf16(s[2 * kk][0], s[2 * kk][1]);
      pa[1] = pack_bf16(s[2 * kk][2], s[2 * kk][3]);
      pa[2] = pack_bf16(s[2 * kk + 1][0], s[2 * kk + 1][1]);
      pa[3] = pack_bf16(s[2 * kk + 1][2], s[2 * kk + 1][3]);
#pragma unroll
      for (int nt = 0; nt < NT; nt += 2) {
        uint32_t bf[4];
        ldsm4t(sO + swz<CH>(kk * 16 + (lane & 7) + (((lane >> 3) & 1) << 3), nt + (lane >> 4)),
               bf);
        mma16816(dv[nt], pa, bf[0], bf[1]);
        mma16816(dv[nt + 1], pa, bf[2], bf[3]);
      }
    }
    // dP^T = V dO^T
    float dp[8][4];
#pragma unroll
    for (int i = 0; i < 8; ++i) dp[i][0] = dp[i][1] = dp[i][2] = dp[i][3] = 0.f;
#pragma unroll
    for (int kk = 0; kk < KS; ++kk) {
      uint32_t va[4];
      ldsm4(sV + swz<CH>(warp * 16 + (lane & 15), kk * 2 + (lane >> 4)), va);
#pragma unroll
      for (int nt = 0; nt < 8; nt += 2) {
        uint32_t bf[4];
        ldsm4(sO + swz<CH>(nt * 8 + (lane & 7) + ((lane >> 4) << 3), kk * 2 + ((lane >> 3) & 1)),
              bf);
        mma16816(dp[nt], va, bf[0], bf[1]);
        mma16816(dp[nt + 1], va, bf[2], bf[3]);
      }
    }
    // dS^T = P^T (dP^T - D), kept in s; staged to shared memory for dQ
#pragma unroll
    for (int nt = 0; nt < 8; ++nt) {
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const float dd = Dv[nt * 8 + cq + e];
        s[nt][e] *= dp[nt][e] - dd;
        s[nt][2 + e] *= dp[nt][2 + e] - dd;
      }
      const int r = warp * 16 + (lane >> 2);
      st_shared_u32(sS + swz<8>(r, nt) + (lane & 3) * 4, pack_bf16(s[nt][0], s[nt][1]));
      st_shared_u32(sS + swz<8>(r + 8, nt) + (lane & 3) * 4, pack_bf16(s[nt][2], s[nt][3]));
    }
    // dK += dS^T Q
#pragma unroll
    for (int kk = 0; kk < 4; ++kk) {
      uint32_t pa[4];
      pa[0] = pack_bf16(s[2 * kk][0], s[2 * kk][1]);
      pa[1] = pack_bf16(s[2 * kk][2], s[2 * kk][3]);
      pa[2] = pack_bf16(s[2 * kk + 1][0], s[2 * kk + 1][1]);
      pa[3] = pack_bf16(s[2 * kk + 1][2], s[2 * kk + 1][3]);
#pragma unroll
      for (int nt = 0; nt < NT; nt += 2) {
        uint32_t bf[4];
        ldsm4t(sQ + swz<CH>(kk * 16 + (lane & 7) + (((lane >> 3) & 1) << 3), nt + (lane >> 4)),
               bf);
        mma16816(dk[nt], pa, bf[0], bf[1]);
        mma16816(dk[nt + 1], pa, bf[2], bf[3]);
      }
    }
    __syncthreads();  // every warp's dS^T rows are in shared memory
    // dQ (64 queries x HD) += dS K, this warp's 16 queries, in two column halves
    const int qr0 = q0 + warp * 16 + (lane >> 2), qr1 = qr0 + 8;
#pragma unroll
    for (int nh = 0; nh < 2; ++nh) {
      float dq[NT / 2][4];
#pragma unroll
      for (int i = 0; i < NT / 2; ++i) dq[i][0] = dq[i][1] = dq[i][2] = dq[i][3] = 0.f;
#pragma unroll
      for (int kk = 0; kk < 4; ++kk) {
        uint32_t da[4];
        ldsm4t(sS + swz<8>(kk * 16 + (lane & 7) + ((lane >> 4) << 3), warp * 2 + ((lane >> 3) & 1)),
               da);
#pragma unroll
        for (int nt = 0; nt < NT / 2; nt += 2) {
          uint32_t bf[4];
          ldsm4t(sK + swz<CH>(kk * 16 + (lane & 7) + (((lane >> 3) & 1) << 3),
                              nh * (NT / 2) + nt + (lane >> 4)),
                 bf);
          mma16816(dq[nt], da, bf[0], bf[1]);
          mma16816(dq[nt + 1], da, bf[2], bf[3]);
        }
      }
      float* q0p = p.dQ + (row0 + qr0) * ldq + hq * HD + nh * (HD / 2) + cq;
      float* q1p = q0p + 8 * ldq;
#pragma unroll
      for (int nt = 0; nt < NT / 2; ++nt) {
        if (qr0 < p.seq) red_add_v2(q0p + nt * 8, dq[nt][0] * p.scale, dq[nt][1] * p.scale);
        if (qr1 < p.seq) red_add_v2(q1p + nt * 8, dq[nt][2] * p.scale, dq[nt][3] * p.scale);
      }
    }
    __syncthreads();  // shared tiles and dS^T are rewritten next iteration
  }
  if (kr0 < p.seq) {
    float* kp = p.dK + (row0 + kr0) * ldk + g * HD + cq;
    __nv_bfloat16* vp = p.dV + (row0 + kr0) * ldk + g * HD + cq;
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
      *reinterpret_cast<float2*>(kp + nt * 8) = make_float2(dk[nt][0] * p.scale, dk[nt][1] * p.scale);
      *reinterpret_cast<__nv_bfloat162*>(vp + nt * 8) = __floats2bfloat162_rn(dv[nt][0], dv[nt][1]);
    }
  }
  if (kr1 < p.seq) {
    float* kp = p.dK + (row0 + kr1) * ldk + g * HD + cq;
    __nv_bfloat16* vp = p.dV + (row0 + kr1) * ldk + g * HD + cq;
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
      *reinterpret_cast<float2*>(kp + nt * 8) = make_float2(dk[nt][2] * p.scale, dk[nt][3] * p.scale);
      *reinterpret_cast<__nv_bfloat162*>(vp + nt * 8) = __floats2bfloat162_rn(dv[nt][2], dv[nt][3]);
    }
  }
}

template <int HD>
constexpr int fwd_smem() { return 5 * kBM * HD * 2; }
template <int HD>
constexpr int bwd_smem() { return 6 * kBM * HD * 2 + kBN * kBM * 2 + 4 * kBM * 4; }

inline unsigned blocks_for(int64_t n, int per) { return unsigned((n + per - 1) / per); }

}  // namespace

// ------------------------------------------------------------------ host
slora_status rope_run(bool backward, const void* Y, const void* Yc, const void* Yo,
                      const float* G, const int32_t* idx, int n_idx, const slora_tokens* tok,
                      const TokenInfo& ti, int n, int hd, double base, void* out, void* out_c,
                      void* out_o, Arena& ar, bool plan, cudaStream_t st) {
  const int half = hd / 2;
  float2* tab = ar.take<float2>(size_t(ti.seq) * half);
  int32_t *ctx_rows = nullptr, *out_rows = nullptr, *kind = nullptr, *inv = nullptr;
  if (idx) {
    ctx_rows = ar.take<int32_t>(size_t(std::max<int64_t>(ti.T_C, 1)));
    out_rows = ar.take<int32_t>(size_t(std::max<int64_t>(ti.T_O, 1)));
    kind = ar.take<int32_t>(size_t(ti.T));
    inv = ar.take<int32_t>(size_t(n));
  }
  if (plan) return SLORA_OK;
  SLORA_TRY(arena_fits(ar, "rope"));
  {
    LaunchScope ls(kAux, double(ti.seq) * half * 8, st);
    rope_table_kernel<<<blocks_for(int64_t(ti.seq) * half, 256), 256, 0, st>>>(tab, ti.seq, half,
                                                                               base);
    SLORA_CHECK_LAUNCH();
  }
  if (idx) {
    SLORA_TRY(launch_rowmaps(tok, ti, ctx_rows, out_rows, st));
    {
      LaunchScope ls(kAux, double(ti.T) * 8, st);
      rowkind_kernel<<<blocks_for(ti.T, 256), 256, 0, st>>>(ctx_rows, ti.T_C, out_rows, ti.T_O,
                                                              kind);
      SLORA_CHECK_LAUNCH();
    }
    {
      LaunchScope ls(kAux, double(n) * 4, st);
      inverse_fill_kernel<<<blocks_for(n, 256), 256, 0, st>>>(n, inv);
      SLORA_CHECK_LAUNCH();
    }
    if (n_idx > 0) {
      LaunchScope ls(kAux, double(n_idx) * 8, st);
      inverse_scatter_kernel<<<blocks_for(n_idx, 256), 256, 0, st>>>(idx, n_idx, n, inv);
      SLORA_CHECK_LAUNCH();
    }
  }
  const int64_t threads = ti.T * int64_t(n / hd) * (hd / 4);
  const double bytes = backward ? double(ti.T) * n * 6 : double(ti.T) * n * 4;
  LaunchScope ls(kElementwise, bytes, st);
  if (!backward) {
    rope_pack_kernel<<<blocks_for(threads, 256), 256, 0, st>>>(
        static_cast<const __nv_bfloat16*>(Y), static_cast<const __nv_bfloat16*>(Yc),
        static_cast<const __nv_bfloat16*>(Yo), kind, inv, n_idx, ti.T, n, hd, ti.seq, tab,
        static_cast<__nv_bfloat16*>(out));
  } else {
    rope_unpack_kernel<<<blocks_for(threads, 256), 256, 0, st>>>(
        G, kind, inv, n_idx, ti.T, n, hd, ti.seq, tab, static_cast<__nv_bfloat16*>(out),
        static_cast<__nv_bfloat16*>(out_c), static_cast<__nv_bfloat16*>(out_o));
  }
  SLORA_CHECK_LAUNCH();
  return SLORA_OK;
}

// Algorithmic FLOPs of one causal product: 2 hd per (query, key <= query)
// pair, seq (seq + 1) / 2 pairs per sequence and head (the masked halves of
// the diagonal tiles the kernels also compute are not counted).
static double causal_flops(const TokenInfo& ti, int heads, int hd) {
  const double s = double(ti.seq);
  return 2.0 * hd * s * (s + 1) / 2 * heads * ti.batch;
}

slora_status attention_fwd_run(const void* Q, const void* K, const void* V, const TokenInfo& ti,
                               int H, int KV, int hd, void* O, float* lse, cudaStream_t st) {
  AttnFwdP p;
  p.Q = static_cast<const __nv_bfloat16*>(Q);
  p.K = static_cast<const __nv_bfloat16*>(K);
  p.V = static_cast<const __nv_bfloat16*>(V);
  p.O = static_cast<__nv_bfloat16*>(O);
  p.lse = lse;
  p.seq = ti.seq; p.H = H; p.KV = KV;
  p.nqb = (ti.seq + kBM - 1) / kBM;
  p.sl2 = float(1.0 / std::sqrt(double(hd)) * 1.4426950408889634);
  const dim3 grid(p.nqb, H, ti.batch);
  LaunchScope ls(kAttention, 2.0 * causal_flops(ti, H, hd), st);
  if (attention_fwd_tc_ok(Q, K, V, O, hd)) return attention_fwd_tc_run(Q, K, V, ti, H, KV, O, lse, st);
  if (hd == 128) {
    SLORA_CUDA(cudaFuncSetAttribute(attn_fwd_kernel<128>,
                                    cudaFuncAttributeMaxDynamicSharedMemorySize, fwd_smem<128>()));
    attn_fwd_kernel<128><<<grid, kThreads, fwd_smem<128>(), st>>>(p);
  } else {
    SLORA_CUDA(cudaFuncSetAttribute(attn_fwd_kernel<64>,
                                    cudaFuncAttributeMaxDynamicSharedMemorySize, fwd_smem<64>()));
    attn_fwd_kernel<64><<<grid, kThreads, fwd_smem<64>(), st>>>(p);
  }
  SLORA_CHECK_LAUNCH();
  return SLORA_OK;
}

slora_status attention_bwd_run(const void* Q, const void* K, const void* V, const void* O,
                               const float* lse, const void* dO, const TokenInfo& ti, int H,
                               int KV, int hd, float* dQ, float* dK, void* dV, Arena& ar,
                               bool plan, cudaStream_t st) {
  float* D = ar.take<float>(size_t(ti.T) * H);
  if (plan) return SLORA_OK;
  SLORA_TRY(arena_fits(ar, "attention_bwd"));
  const bool tc = attention_bwd_tc_ok(Q, K, V, dO, dQ, dK, dV, hd);
  if (!tc) SLORA_CUDA(cudaMemsetAsync(dQ, 0, size_t(ti.T) * H * hd * sizeof(float), st));
  {
    LaunchScope ls(kElementwise, double(ti.T) * H * hd * 4, st);
    const int64_t thr = ti.T * H * 32;
    if (hd == 128)
      attn_rowdot_kernel<128><<<blocks_for(thr, 256), 256, 0, st>>>(
          static_cast<const __nv_bfloat16*>(dO), static_cast<const __nv_bfloat16*>(O), ti.T, H,
          ti.seq, D);
    else
      attn_rowdot_kernel<64><<<blocks_for(thr, 256), 256, 0, st>>>(
          static_cast<const __nv_bfloat16*>(dO), static_cast<const __nv_bfloat16*>(O), ti.T, H,
          ti.seq, D);
    SLORA_CHECK_LAUNCH();
  }
  if (tc)
    return attention_bwd_tc_run(Q, K, V, dO, lse, D, ti, H, KV, dQ, dK, dV,
                                causal_flops(ti, H, hd), st);
  AttnBwdP p;
  p.Q = static_cast<const __nv_bfloat16*>(Q);
  p.K = static_cast<const __nv_bfloat16*>(K);
  p.V = static_cast<const __nv_bfloat16*>(V);
  p.dO = static_cast<const __nv_bfloat16*>(dO);
  p.lse = lse; p.D = D; p.dQ = dQ; p.dK = dK;
  p.dV = static_cast<__nv_bfloat16*>(dV);
  p.seq = ti.seq; p.H = H; p.KV = KV;
  p.nqb = (ti.seq + kBM - 1) / kBM;
  p.scale = float(1.0 / std::sqrt(double(hd)));
  p.sl2 = float(double(p.scale) * 1.4426950408889634);
  const dim3 grid(p.nqb, KV, ti.batch);
  LaunchScope ls(kAttention, 5.0 * causal_flops(ti, H, hd), st);
  if (hd == 128) {
    SLORA_CUDA(cudaFuncSetAttribute(attn_bwd_kernel<128>,
                                    cudaFuncAttributeMaxDynamicSharedMemorySize, bwd_smem<128>()));
    attn_bwd_kernel<128><<<grid, kThreads, bwd_smem<128>(), st>>>(p);
  } else {
    SLORA_CUDA(cudaFuncSetAttribute(attn_bwd_kernel<64>,
                                    cudaFuncAttributeMaxDynamicSharedMemorySize, bwd_smem<64>()));
    attn_bwd_kernel<64><<<grid, kThreads, bwd_smem<64>(), st>>>(p);
  }
  SLORA_CHECK_LAUNCH();
  return SLORA_OK;
}

}  // namespace slora
