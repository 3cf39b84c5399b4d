// Skinny (rank-sized) contractions, see skinny.cuh.
//
// 128-thread blocks over 64 x 64 tiles of Y staged in shared memory by a 3-
// or 4-stage cp.async pipeline (zero-filled past the edges, optional row
// gather).  The rank-sized operand is split into NT bf16 terms once per call
// (prep_r_kernel, laid out [term][column][index] so each stage copies it with
// 16-byte cp.async) and staged beside Y.  Each warp owns 16 rows (rowdot) or
// 16 columns (coldot) of the tile and issues mma.sync m16n8k16 (bf16 in, fp32
// accumulate).  With a split over the reduced dimension, each block writes its
// partial tile to a workspace and the last block of the output block to arrive
// (atomic ticket) sums the partials in split order and writes the outputs:
// bit-reproducible, no second launch.
//
// When Y is a plain strided matrix (no row gather) a second kernel takes the
// contraction: a persistent grid of one wave (two CTAs per SM) that takes
// fixed (output block, reduction group) units from an atomic ticket.  A
// producer warp streams each unit through a TMA ring of 128-byte-swizzled
// 64 x 64 tiles of Y (plus the matching tile of the split operand) completed
// on mbarriers; four consumer warps read fragments by ldmatrix.  A block
// covered by one unit is written directly from its accumulators; otherwise
// every unit writes its partial tile to its own slot and the last unit of the
// block to finish sums them in group order.  One launch may carry several
// independent contractions (a job table sharing the ticket).
#include <cuda.h>
#include <cudaTypedefs.h>

#include <mutex>

#include "skinny.cuh"

namespace slora {
namespace {

constexpr int TILE = 64, PAD = 72, NTH = 128;

__device__ __forceinline__ void cp_async16(void* dst, const void* src, int bytes) {
  const uint32_t d = static_cast<uint32_t>(__cvta_generic_to_shared(dst));
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(d), "l"(src), "r"(bytes)
               : "memory");
}
__device__ __forceinline__ void cp_async_commit() {
  asm volatile("cp.async.commit_group;" ::: "memory");
}
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}
__device__ __forceinline__ void mma16816(float* d, uint32_t a0, uint32_t a1, uint32_t a2,
                                         uint32_t a3, uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
      "{%8,%9}, {%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}
__device__ __forceinline__ void ldsm_x4_trans(uint32_t& r0, uint32_t& r1, uint32_t& r2,
                                              uint32_t& r3, const void* p) {
  const uint32_t a = static_cast<uint32_t>(__cvta_generic_to_shared(p));
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(a));
}
__device__ __forceinline__ uint32_t lds32(const __nv_bfloat16* p) {
  return *reinterpret_cast<const uint32_t*>(p);
}

// Split v into NT bf16 terms whose sum reproduces v to ~2^-8 (NT=1) or ~2^-24 (NT=3).
template <int NT>
__device__ __forceinline__ void split_terms(float v, __nv_bfloat16* out) {
  __nv_bfloat16 h = __float2bfloat16_rn(v);
  out[0] = h;
  if (NT > 1) {
    float r = v - __bfloat162float(h);
    __nv_bfloat16 m = __float2bfloat16_rn(r);
    out[1] = m;
    r -= __bfloat162float(m);
    out[2] = __float2bfloat16_rn(r);
  }
}

// Raised when a channel-index map holds a value outside its weight (the
// element is read as zero / not written); reported by skinny_check_error.
__device__ int g_sk_bad_index = 0;

__device__ __forceinline__ float load_r(const SkR& R, int64_t i, int q) {
  const int64_t ii = R.map ? R.map[i] : i;
  if (ii < 0 || ii >= R.map_limit) {
    atomicExch(&g_sk_bad_index, 1);
    return 0.0f;
  }
  const void* p = R.ptr;
  int dt = R.dt;
  int64_t off = ii * R.si + int64_t(q) * R.sq;
  if (q >= R.qsplit) {
    p = R.ptr_b;
    dt = R.dt_b;
    off = ii * R.si_b + int64_t(q - R.qsplit) * R.sq_b;
  }
  if (dt == kF32) return static_cast<const float*>(p)[off];
  return __bfloat162float(static_cast<const __nv_bfloat16*>(p)[off]);
}

// Pre-split of the rank-sized operand, once per call: RS[s][q][i] = term s of
// R(i, q) (zero for q >= c or i >= I), rows of I64 = roundup(I, 64) elements.
// Threads walk the source's contiguous index so the reads coalesce.
template <int NT>
__global__ void prep_r_kernel(const __grid_constant__ SkR R, int c, int CP, int64_t I, int64_t I64,
                              __nv_bfloat16* __restrict__ RS) {
  const int64_t e = int64_t(blockIdx.x) * blockDim.x + threadIdx.x;
  if (e >= int64_t(CP) * I64) return;
  const bool q_fast = R.sq == 1 && (R.ptr_b == nullptr || R.sq_b == 1);
  int q;
  int64_t i;
  if (q_fast) {
    q = int(e % CP);
    i = e / CP;
  } else {
    q = int(e / I64);
    i = e % I64;
  }
  const float v = (q < c && i < I) ? load_r(R, i, q) : 0.0f;
  __nv_bfloat16 tv[3];
  split_terms<NT>(v, tv);
#pragma unroll
  for (int s = 0; s < NT; ++s) RS[(int64_t(s) * CP + q) * I64 + i] = tv[s];
}

// Several operands at once: blockIdx.y picks the job.
struct PrepBatch {
  SkR R[8];
  int c[8], CP[8], nt[8];
  int64_t I[8], I64[8];
  __nv_bfloat16* RS[8];
};
__global__ void prep_r_batch_kernel(const __grid_constant__ PrepBatch b) {
  const int k = blockIdx.y;
  const int CP = b.CP[k];
  const int64_t I64 = b.I64[k];
  const int64_t e = int64_t(blockIdx.x) * blockDim.x + threadIdx.x;
  if (e >= int64_t(CP) * I64) return;
  const SkR& R = b.R[k];
  const bool q_fast = R.sq == 1 && (R.ptr_b == nullptr || R.sq_b == 1);
  int q;
  int64_t i;
  if (q_fast) {
    q = int(e % CP);
    i = e / CP;
  } else {
    q = int(e / I64);
    i = e % I64;
  }
  const float v = (q < b.c[k] && i < b.I[k]) ? load_r(R, i, q) : 0.0f;
  __nv_bfloat16 tv[3];
  if (b.nt[k] == 3) split_terms<3>(v, tv); else split_terms<1>(v, tv);
  for (int s = 0; s < b.nt[k]; ++s) b.RS[k][(int64_t(s) * CP + q) * I64 + i] = tv[s];
}

// Pipeline depth from the shared memory of one stage (Y tile + split R tile).
constexpr int stage_bytes(int CP, int NT) { return TILE * PAD * 2 + NT * CP * PAD * 2; }
constexpr int stages_for(int CP, int NT) { return stage_bytes(CP, NT) <= 16896 ? 4 : 3; }
constexpr int smem_for(int CP, int NT) { return stages_for(CP, NT) * stage_bytes(CP, NT); }

// Stage RS[:, :, i0 .. i0+64) into Rs[s][q][0..64) with 16-byte async copies.
template <int CP, int NT>
__device__ __forceinline__ void stage_r(__nv_bfloat16 (*Rs)[CP][PAD],
                                        const __nv_bfloat16* __restrict__ RS, int64_t I64,
                                        int64_t i0, int tid) {
#pragma unroll
  for (int e = tid; e < NT * CP * 8; e += NTH) {
    const int seg = e & 7, row = e >> 3;  // row = s * CP + q
    const int sidx = row / CP, q = row % CP;
    cp_async16(&Rs[sidx][q][seg * 8], RS + int64_t(row) * I64 + i0 + seg * 8, 16);
  }
}

// Stage the 64 x 64 tile of Y at (m0, k0) into Ys (rows m, columns k).
__device__ __forceinline__ void stage_y(__nv_bfloat16 (*Ys)[PAD], const SkY& Y, int64_t M,
                                        int64_t K, int64_t m0, int64_t k0, int tid) {
  const __nv_bfloat16* base = static_cast<const __nv_bfloat16*>(Y.ptr);
#pragma unroll
  for (int i = 0; i < (TILE * TILE / 8) / NTH; ++i) {
    const int seg = tid + NTH * i;
    const int row = seg >> 3, c8 = (seg & 7) * 8;
    const int64_t m = m0 + row, k = k0 + c8;
    int bytes = 0;
    const __nv_bfloat16* src = base;
    if (m < M && k < K) {
      const int64_t left = (K - k) * 2;
      bytes = left < 16 ? int(left) : 16;
      src = base + (Y.map ? int64_t(Y.map[m]) : m) * Y.ld + k;
    }
    cp_async16(&Ys[row][c8], src, bytes);
  }
}

// Output of one reduced element of a rowdot (row m, column q).
__device__ __forceinline__ void row_emit(const SkRowOut& o, int64_t m, int q, float v) {
  if (q < o.qsplit) {
    if (o.out1) o.out1[(o.map1 ? int64_t(o.map1[m]) : m) * o.ld1 + o.off1 + q] = v;
    if (o.out2)
      static_cast<__nv_bfloat16*>(o.out2)[(o.map2 ? int64_t(o.map2[m]) : m) * o.ld2 + o.off2 + q] =
          __float2bfloat16_rn(o.s2 * v);
  } else if (o.out1b) {
    o.out1b[(o.map1b ? int64_t(o.map1b[m]) : m) * o.ld1b + o.off1b + (q - o.qsplit)] = v;
  }
}
// Output of one reduced element of a coldot (column k, rank column q).
__device__ __forceinline__ void col_emit(const SkColOut& o, int64_t k, int q, float v) {
  v *= o.scale;
  const int64_t kk = o.kmap ? int64_t(o.kmap[k]) : k;
  if (kk < 0 || kk >= o.kmap_limit) {
    atomicExch(&g_sk_bad_index, 1);
    return;
  }
  float* base = q < o.qsplit ? o.out : o.out_b;
  const int qq = q < o.qsplit ? q : q - o.qsplit;
  float* dst = base + (o.trans ? int64_t(qq) * o.ldo + kk : kk * o.ldo + qq);
  *dst = o.accumulate ? *dst + v : v;
}

// Fixed-order sum over the splits of 4 consecutive partial columns:
// src[s * stride4] for s = 0 .. nsplit-1, eight loads in flight at a time.
__device__ __forceinline__ float4 sum_splits4(const float4* src, int64_t stride4, int nsplit) {
  float4 a = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
  int s = 0;
  for (; s + 8 <= nsplit; s += 8) {
    float4 v[8];
#pragma unroll
    for (int u = 0; u < 8; ++u) v[u] = __ldcg(src + (s + u) * stride4);
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      a.x += v[u].x; a.y += v[u].y; a.z += v[u].z; a.w += v[u].w;
    }
  }
  for (; s < nsplit; ++s) {
    const float4 v = __ldcg(src + s * stride4);
    a.x += v.x; a.y += v.y; a.z += v.z; a.w += v.w;
  }
  return a;
}

// Returns true in the one CTA (of the `n` sharing `counter`) that arrives last,
// after every CTA's partial is visible; that CTA resets the counter.
// The CTA's writes are ordered before thread 0's fence by the barrier, and
// the fence (cumulative) publishes them all before the counter increment.
__device__ __forceinline__ bool last_arrival(unsigned* counter, unsigned n, int tid) {
  __shared__ unsigned s_last;
  __syncthreads();
  if (tid == 0) {
    __threadfence();
    const unsigned prev = atomicAdd(counter, 1u);
    s_last = (prev + 1 == n) ? 1u : 0u;
    if (s_last) *counter = 0u;
  }
  __syncthreads();
  if (s_last) __threadfence();
  return s_last != 0;
}

// Partial tile of a warp's 16 x CP accumulators (rows / columns `r0`, `r0+8`
// of the output block) at part[(split * nout + r) * CP + col].
template <int NF>
__device__ __forceinline__ void store_partial(float* part, int split, int64_t nout, int64_t r0,
                                              int t, const float (*acc)[4]) {
  constexpr int CP = NF * 8;
#pragma unroll
  for (int f = 0; f < NF; ++f) {
    const int col = f * 8 + 2 * t;
    if (r0 < nout)
      *reinterpret_cast<float2*>(part + (int64_t(split) * nout + r0) * CP + col) =
          make_float2(acc[f][0], acc[f][1]);
    if (r0 + 8 < nout)
      *reinterpret_cast<float2*>(part + (int64_t(split) * nout + r0 + 8) * CP + col) =
          make_float2(acc[f][2], acc[f][3]);
  }
}

template <int NF, int NT>
__global__ void __launch_bounds__(NTH) rowdot_kernel(const __grid_constant__ SkY Y, int64_t M, int64_t K,
                                                     const __nv_bfloat16* __restrict__ RS,
                                                     int64_t I64, int c, int chunks_per_split,
                                                     float* __restrict__ part,
                                                     unsigned* __restrict__ counters,
                                                     const __grid_constant__ SkRowOut o) {
  constexpr int CP = NF * 8, S = stages_for(CP, NT);
  extern __shared__ __align__(16) unsigned char sk_smem[];
  auto Ys = reinterpret_cast<__nv_bfloat16 (*)[TILE][PAD]>(sk_smem);  // [S][TILE][PAD]
  auto Rs = reinterpret_cast<__nv_bfloat16 (*)[NT][CP][PAD]>(sk_smem + S * TILE * PAD * 2);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31, g = lane >> 2, t = lane & 3;
  const int64_t m0 = int64_t(blockIdx.x) * TILE;
  const int ks = blockIdx.y, nsplit = gridDim.y;
  const int64_t nchunks = (K + TILE - 1) / TILE;
  const int64_t kc0 = int64_t(ks) * chunks_per_split;
  const int n = int((kc0 + chunks_per_split < nchunks ? kc0 + chunks_per_split : nchunks) - kc0);
  float acc[NF][4];
#pragma unroll
  for (int f = 0; f < NF; ++f) acc[f][0] = acc[f][1] = acc[f][2] = acc[f][3] = 0.0f;
#pragma unroll
  for (int j = 0; j < S - 1; ++j) {
    if (j < n) {
      stage_y(Ys[j], Y, M, K, m0, (kc0 + j) * TILE, tid);
      stage_r<CP, NT>(Rs[j], RS, I64, (kc0 + j) * TILE, tid);
    }
    cp_async_commit();
  }
  const int r0 = warp * 16 + g;
  for (int j = 0; j < n; ++j) {
    cp_async_wait<S - 2>();
    __syncthreads();  // chunk j landed; every warp is done with chunk j-1's slot
    const int jn = j + S - 1;
    if (jn < n) {
      stage_y(Ys[jn % S], Y, M, K, m0, (kc0 + jn) * TILE, tid);
      stage_r<CP, NT>(Rs[jn % S], RS, I64, (kc0 + jn) * TILE, tid);
    }
    cp_async_commit();
    const int b = j % S;
#pragma unroll
    for (int k16 = 0; k16 < TILE / 16; ++k16) {
      const int kb = k16 * 16 + 2 * t;
      const uint32_t a0 = lds32(&Ys[b][r0][kb]), a1 = lds32(&Ys[b][r0 + 8][kb]);
      const uint32_t a2 = lds32(&Ys[b][r0][kb + 8]), a3 = lds32(&Ys[b][r0 + 8][kb + 8]);
#pragma unroll
      for (int f = 0; f < NF; ++f)
#pragma unroll
        for (int s = 0; s < NT; ++s)
          mma16816(acc[f], a0, a1, a2, a3, lds32(&Rs[b][s][f * 8 + g][kb]),
                   lds32(&Rs[b][s][f * 8 + g][kb + 8]));
    }
  }
  const int64_t row0 = m0 + r0;
  if (nsplit == 1) {  // no split: emit straight from the accumulators
#pragma unroll
    for (int f = 0; f < NF; ++f) {
      const int col = f * 8 + 2 * t;
      if (row0 < M) {
        if (col < c) row_emit(o, row0, col, acc[f][0]);
        if (col + 1 < c) row_emit(o, row0, col + 1, acc[f][1]);
      }
      if (row0 + 8 < M) {
        if (col < c) row_emit(o, row0 + 8, col, acc[f][2]);
        if (col + 1 < c) row_emit(o, row0 + 8, col + 1, acc[f][3]);
      }
    }
    return;
  }
  store_partial<NF>(part, ks, M, row0, t, acc);
  if (!last_arrival(counters + blockIdx.x, unsigned(nsplit), tid)) return;
  const int nq4 = (c + 3) / 4;
  for (int e = tid; e < TILE * nq4; e += NTH) {
    const int64_t m = m0 + e / nq4;
    const int q0 = (e % nq4) * 4;
    if (m >= M) continue;
    const float4 v = sum_splits4(reinterpret_cast<const float4*>(part + m * CP + q0),
                                 M * CP / 4, nsplit);
    row_emit(o, m, q0, v.x);
    if (q0 + 1 < c) row_emit(o, m, q0 + 1, v.y);
    if (q0 + 2 < c) row_emit(o, m, q0 + 2, v.z);
    if (q0 + 3 < c) row_emit(o, m, q0 + 3, v.w);
  }
}

template <int NF, int NT>
__global__ void __launch_bounds__(NTH) coldot_kernel(const __grid_constant__ SkY Y, int64_t M, int64_t K,
                                                     const __nv_bfloat16* __restrict__ RS,
                                                     int64_t I64, int c, int chunks_per_split,
                                                     float* __restrict__ part,
                                                     unsigned* __restrict__ counters,
                                                     const __grid_constant__ SkColOut o) {
  constexpr int CP = NF * 8, S = stages_for(CP, NT);
  extern __shared__ __align__(16) unsigned char sk_smem[];
  auto Ys = reinterpret_cast<__nv_bfloat16 (*)[TILE][PAD]>(sk_smem);  // [S][TILE][PAD]
  auto Rs = reinterpret_cast<__nv_bfloat16 (*)[NT][CP][PAD]>(sk_smem + S * TILE * PAD * 2);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31, g = lane >> 2, t = lane & 3;
  const int64_t k0 = int64_t(blockIdx.x) * TILE;
  const int ms = blockIdx.y, nsplit = gridDim.y;
  const int64_t nchunks = (M + TILE - 1) / TILE;
  const int64_t mc0 = int64_t(ms) * chunks_per_split;
  const int n = int((mc0 + chunks_per_split < nchunks ? mc0 + chunks_per_split : nchunks) - mc0);
  float acc[NF][4];
#pragma unroll
  for (int f = 0; f < NF; ++f) acc[f][0] = acc[f][1] = acc[f][2] = acc[f][3] = 0.0f;
  const int mq = lane >> 3, rr = lane & 7;  // ldmatrix: matrix index, row within it
#pragma unroll
  for (int j = 0; j < S - 1; ++j) {
    if (j < n) {
      stage_y(Ys[j], Y, M, K, (mc0 + j) * TILE, k0, tid);
      stage_r<CP, NT>(Rs[j], RS, I64, (mc0 + j) * TILE, tid);
    }
    cp_async_commit();
  }
  for (int j = 0; j < n; ++j) {
    cp_async_wait<S - 2>();
    __syncthreads();
    const int jn = j + S - 1;
    if (jn < n) {
      stage_y(Ys[jn % S], Y, M, K, (mc0 + jn) * TILE, k0, tid);
      stage_r<CP, NT>(Rs[jn % S], RS, I64, (mc0 + jn) * TILE, tid);
    }
    cp_async_commit();
    const int b = j % S;
#pragma unroll
    for (int m16 = 0; m16 < TILE / 16; ++m16) {
      // A = Y^T fragment (16 k x 16 m) for columns warp*16.. of the tile
      const int mb = m16 * 16 + (mq >> 1) * 8;
      const int kb = warp * 16 + (mq & 1) * 8;
      uint32_t a0, a1, a2, a3;
      ldsm_x4_trans(a0, a1, a2, a3, &Ys[b][mb + rr][kb]);
      const int mcol = m16 * 16 + 2 * t;
#pragma unroll
      for (int f = 0; f < NF; ++f)
#pragma unroll
        for (int s = 0; s < NT; ++s)
          mma16816(acc[f], a0, a1, a2, a3, lds32(&Rs[b][s][f * 8 + g][mcol]),
                   lds32(&Rs[b][s][f * 8 + g][mcol + 8]));
    }
  }
  const int64_t kr = k0 + warp * 16 + g;
  if (nsplit == 1) {
#pragma unroll
    for (int f = 0; f < NF; ++f) {
      const int col = f * 8 + 2 * t;
      if (kr < K) {
        if (col < c) col_emit(o, kr, col, acc[f][0]);
        if (col + 1 < c) col_emit(o, kr, col + 1, acc[f][1]);
      }
      if (kr + 8 < K) {
        if (col < c) col_emit(o, kr + 8, col, acc[f][2]);
        if (col + 1 < c) col_emit(o, kr + 8, col + 1, acc[f][3]);
      }
    }
    return;
  }
  store_partial<NF>(part, ms, K, kr, t, acc);
  if (!last_arrival(counters + blockIdx.x, unsigned(nsplit), tid)) return;
  const int nq4 = (c + 3) / 4;
  for (int e = tid; e < TILE * nq4; e += NTH) {
    const int64_t k = k0 + e / nq4;
    const int q0 = (e % nq4) * 4;
    if (k >= K) continue;
    const float4 v = sum_splits4(reinterpret_cast<const float4*>(part + k * CP + q0),
                                 K * CP / 4, nsplit);
    col_emit(o, k, q0, v.x);
    if (q0 + 1 < c) col_emit(o, k, q0 + 1, v.y);
    if (q0 + 2 < c) col_emit(o, k, q0 + 2, v.z);
    if (q0 + 3 < c) col_emit(o, k, q0 + 3, v.w);
  }
}

// One full wave of resident blocks: the shared memory of a block bounds how
// many fit on an SM (each keeps S-1 chunks of Y in flight).  The SM count is
// the device's, queried once (num_sms), so a workspace query and the run it
// sizes see the same value.
int64_t target_blocks(int CP, int NT) {
  int per_sm = (200 * 1024) / smem_for(CP, NT);
  if (per_sm > 8) per_sm = 8;
  if (per_sm < 1) per_sm = 1;
  return int64_t(num_sms()) * per_sm;
}

int64_t splits_for(int64_t nblocks, int64_t nchunks, int CP, int NT) {
  if (nblocks < 1) nblocks = 1;
  if (nchunks < 1) nchunks = 1;
  const int64_t target = target_blocks(CP, NT);
  int64_t s = (target + nblocks - 1) / nblocks;
  if (s > nchunks) s = nchunks;
  if (s < 1) s = 1;
  if (s > 64) s = 64;
  return s;
}

int padded(int c) { return ((c + 15) / 16) * 16; }  // NF even keeps the templates few
int64_t round64(int64_t x) { return (x + 63) / 64 * 64; }
bool fp32_terms(const SkR& R) {
  return R.terms != 1 && (R.dt == kF32 || (R.ptr_b && R.dt_b == kF32));
}

slora_status prep_r(const SkR& R, int c, int CP, int64_t I, int nt, __nv_bfloat16* RS,
                    cudaStream_t st) {
  const int64_t I64 = round64(std::max<int64_t>(I, 1));
  const int64_t n = int64_t(CP) * I64;
  LaunchScope ls(kSkinny, double(I) * c * (R.dt == kF32 ? 4 : 2) + double(nt) * n * 2, st);
  if (nt == 3)
    prep_r_kernel<3><<<unsigned((n + 255) / 256), 256, 0, st>>>(R, c, CP, I, I64, RS);
  else
    prep_r_kernel<1><<<unsigned((n + 255) / 256), 256, 0, st>>>(R, c, CP, I, I64, RS);
  SLORA_CHECK_LAUNCH();
  return SLORA_OK;
}

#define SLORA_SKINNY_CASE(KERNEL, NF_, NT)                                              \
  case NF_ * 8: {                                                                       \
    auto kfn = KERNEL<NF_, NT>;                                                         \
    const int sm = smem_for(NF_ * 8, NT);                                               \
    cudaFuncSetAttribute(kfn, cudaFuncAttributeMaxDynamicSharedMemorySize, sm);         \
    kfn<<<grid, NTH, sm, st>>>(Y, M, K, RS, I64, c, cps, w.part, w.counters, o);        \
  } break;
#define SLORA_SKINNY_SWITCH(KERNEL, NT)   \
  switch (CP) {                           \
    SLORA_SKINNY_CASE(KERNEL, 2, NT)      \
    SLORA_SKINNY_CASE(KERNEL, 4, NT)      \
    SLORA_SKINNY_CASE(KERNEL, 6, NT)      \
    default:                              \
    SLORA_SKINNY_CASE(KERNEL, 8, NT)      \
  }

// Split geometry shared by the launch and the workspace query.
struct Geo {
  int CP, nt, cps, nsplit;
  int64_t nblocks;
};
Geo geometry(int64_t nout, int64_t nred, int c, bool fp32) {
  Geo g;
  g.CP = padded(c);
  g.nt = fp32 ? 3 : 1;
  g.nblocks = (nout + TILE - 1) / TILE;
  const int64_t nch = std::max<int64_t>((nred + TILE - 1) / TILE, 1);
  const int64_t ns = splits_for(g.nblocks, nch, g.CP, g.nt);
  g.cps = int((nch + ns - 1) / ns);
  g.nsplit = int((nch + g.cps - 1) / g.cps);
  return g;
}


// ======================================================= TMA stream kernel
__device__ int g_sk_error = 0;
constexpr long long kSkWaitBudget = 2000000000LL;  // ~1 s of SM clocks per wait
// Budget of the pipeline waits (settable for tests of the error path); the
// drain after an abort always uses the full budget so every issued copy lands
// before the CTA exits.
__device__ long long g_sk_budget = kSkWaitBudget;

__device__ __forceinline__ uint32_t su32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}
__device__ __forceinline__ void mbar_init(uint64_t* b, uint32_t n) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(su32(b)), "r"(n) : "memory");
}
__device__ __forceinline__ void mbar_arm(uint64_t* b, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(su32(b)), "r"(bytes)
               : "memory");
}
__device__ __forceinline__ bool mbar_try(uint64_t* b, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(su32(b)), "r"(parity)
      : "memory");
  return ok != 0;
}
// Non-blocking poll (try_wait may park the thread until the phase completes).
__device__ __forceinline__ bool mbar_test(uint64_t* b, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(su32(b)), "r"(parity)
      : "memory");
  return ok != 0;
}
// Bounded wait; false (and the device error flag raised) when it expires.  The
// first poll does not block, so a budget of 0 gives up at once.
__device__ __forceinline__ bool mbar_wait_bounded(uint64_t* b, uint32_t parity,
                                                  long long budget) {
  if (mbar_test(b, parity)) return true;
  if (budget <= 0) {
    atomicExch(&g_sk_error, 1);
    return false;
  }
  const long long t0 = clock64();
  while (!mbar_try(b, parity)) {
    if (clock64() - t0 > budget) {
      atomicExch(&g_sk_error, 1);
      return false;
    }
  }
  return true;
}
__device__ __forceinline__ void tma2d(void* dst, const CUtensorMap* m, uint64_t* bar, int x,
                                      int y) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4}], [%2];" ::"r"(su32(dst)),
      "l"(reinterpret_cast<uint64_t>(m)), "r"(su32(bar)), "r"(x), "r"(y)
      : "memory");
}
__device__ __forceinline__ void ldsm4(uint32_t (&r)[4], uint32_t a) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(a));
}
__device__ __forceinline__ void ldsm4t(uint32_t (&r)[4], uint32_t a) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(a));
}

struct StreamPlan {
  int nblocks = 0, nchunks = 0, G = 1, ngroups = 1, nunits = 0;
  int ncta = 1;
};

// One contraction of a TMA launch; a launch takes up to J of them (same
// column padding and term count) and hands out their units from one ticket,
// job after job.
struct TmaJob {
  CUtensorMap ymap;  // Y [M x K], 64 x 64 boxes
  CUtensorMap rmap;  // split rank operand, 64 x (NT * CP) boxes
  StreamPlan p;
  int c = 0;
  // leading 16-column pairs whose second and third bf16 terms are zero (the
  // columns come from a bf16 operand): their MMAs for those terms are skipped
  int f1 = 0;
  int unit0 = 0;                 // first ticket of the job
  int64_t M = 0, K = 0;
  float* part = nullptr;         // p.nunits partial tiles of 64 x CP floats
  unsigned* counters = nullptr;  // p.nblocks block tickets, zero on entry, left zero
  SkRowOut ro;
  SkColOut co;
};
constexpr int kMaxTmaJobs = 7;  // keeps the launch parameters within 4 KB
template <int J>
struct TmaJobs {
  TmaJob job[J];
  int njobs = 0, nunits = 0, ncta = 1;
  // unit ticket: zero on entry (every call zeroes it with its row maps) and
  // left zero by a launch that completes; after an expired wait
  // (SLORA_ERR_TIMEOUT) it and the block counters are undefined until the
  // next call zeroes them
  unsigned* ticket = nullptr;
};
static_assert(sizeof(TmaJobs<kMaxTmaJobs>) <= 4096, "TMA job table beyond 4 KB of parameters");

// Shared memory of the TMA kernel: S stages of [Y tile 64x64 | split-R tile],
// each 1024-byte aligned (128-byte swizzle), then the stages' full and empty
// barriers (8 slots each) and work descriptors.
constexpr int kYTile = TILE * TILE * 2;
constexpr int tma_stage_bytes(int CP, int NT) { return kYTile + NT * CP * 128; }
constexpr int kTmaCtasPerSm = 2;

// Element (row, k) of a 128-byte-swizzled tile whose rows are 64 bf16: byte
// row * 128 + ((k / 8) ^ (row % 8)) * 16 + (k % 8) * 2.
__device__ __forceinline__ uint32_t swz(uint32_t base, int row, int chunk16) {
  return base + uint32_t(row) * 128u + (uint32_t((chunk16 ^ (row & 7))) << 4);
}

// Stages that fit two CTAs per SM (113 KB each with the barrier block), 2..8.
constexpr int tma_stages(int CP, int NT) {
  return (113 * 1024 - 1280) / tma_stage_bytes(CP, NT) > 8
             ? 8
             : ((113 * 1024 - 1280) / tma_stage_bytes(CP, NT) < 2
                    ? 2
                    : (113 * 1024 - 1280) / tma_stage_bytes(CP, NT));
}
constexpr int tma_smem(int CP, int NT) {
  return tma_stages(CP, NT) * tma_stage_bytes(CP, NT) + 1024 + 64 + 64 + 128;
}
// Barrier of the four consumer warps only (the producer warp never joins).
__device__ __forceinline__ void bar_consumers() { asm volatile("bar.sync 1, 128;" ::: "memory"); }
// last_arrival() among the consumer warps: true in every consumer thread of
// the CTA that brings `counter` to n (and resets it).
__device__ __forceinline__ bool last_arrival_c(unsigned* counter, unsigned n, int tid) {
  __shared__ unsigned s_last_c;
  bar_consumers();
  if (tid == 0) {
    __threadfence();  // publishes the consumer warps' partials (ordered by the barrier)
    const unsigned prev = atomicAdd(counter, 1u);
    s_last_c = (prev + 1 == n) ? 1u : 0u;
    if (s_last_c) *counter = 0u;
  }
  bar_consumers();
  if (s_last_c) __threadfence();
  return s_last_c != 0;
}
// COL = false: rowdot (output block = 64 rows of Y, reduction over K);
// COL = true: coldot (output block = 64 columns of Y, reduction over M).
// Work of one job: output blocks of 64 (rows for rowdot, columns for
// coldot), each with nchunks reduction chunks of 64 cut into ngroups fixed
// groups of up to G chunks.  A unit is one (block, group); units are handed
// out by an atomic ticket in job order and, within a job, group-major order
// (ticket u -> block u % nblocks, group u / nblocks), so SMs that stream
// faster take more units.  Each unit's partial lands in its own slot and the
// last unit of a block to finish sums the block's slots in group order: the
// result does not depend on which CTA ran which unit.
//
// Warp 4 (one lane) produces: it takes the unit tickets and keeps every stage
// of the TMA ring filled, refilling a stage as soon as the four consumer
// warps have each released it on the stage's `empty` barrier.  Warps 0-3
// consume: each owns 16 rows (rowdot) or 16 columns (coldot) of the 64 x 64
// tile and issues the mma.sync fragments; they synchronise among themselves
// (named barrier 1) only at the end of a unit whose block is shared.
template <int NF, int NT, bool COL, int J>
__global__ void __launch_bounds__(NTH + 32) skinny_tma_kernel(const __grid_constant__ TmaJobs<J> jobs) {
  constexpr int CP = NF * 8, S = tma_stages(CP, NT), SB = tma_stage_bytes(CP, NT);
  constexpr int kLast = 2, kEnd = 4, kJobShift = 4;
  extern __shared__ unsigned char sk_smem[];
  unsigned char* sm = reinterpret_cast<unsigned char*>(
      (reinterpret_cast<uintptr_t>(sk_smem) + 1023) & ~uintptr_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(sm + S * SB);
  uint64_t* empty = full + 8;
  int4* info = reinterpret_cast<int4*>(sm + S * SB + 128);  // {block, chunk, flags, group}
  __shared__ int s_abort;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31, g = lane >> 2, t = lane & 3;
  unsigned* work = jobs.ticket;
  if (tid == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 4);
    }
    s_abort = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  __syncthreads();
  if (warp == 4) {
    if (lane != 0) return;
    int pj = 0, pb = 0, pg = 0, pk = 0, pk1 = 0, issued = 0;
    bool pdone = false;
    auto next_unit = [&]() {
      const unsigned u = atomicAdd(work, 1u);
      if (u >= unsigned(jobs.nunits)) {
        if (u == unsigned(jobs.nunits + jobs.ncta - 1)) *work = 0u;
        return false;
      }
      int jb = 0;
#pragma unroll
      for (int x = 1; x < J; ++x)
        if (x < jobs.njobs && u >= unsigned(jobs.job[x].unit0)) jb = x;
      const StreamPlan& P = jobs.job[jb].p;
      const unsigned lu = u - unsigned(jobs.job[jb].unit0);
      pj = jb;
      pb = int(lu % unsigned(P.nblocks));
      pg = int(lu / unsigned(P.nblocks));
      pk = pg * P.G;
      pk1 = pk + P.G < P.nchunks ? pk + P.G : P.nchunks;
      return true;
    };
    bool ok = true;
    while (true) {
      const int st = issued % S;
      if (issued >= S && !mbar_wait_bounded(&empty[st], uint32_t(((issued / S) - 1) & 1), g_sk_budget)) {
        s_abort = 1;
        ok = false;
        break;
      }
      if (s_abort) { ok = false; break; }
      if (!pdone && pk == pk1 && !next_unit()) pdone = true;
      if (pdone) {
        info[st] = make_int4(0, 0, kEnd, 0);
        asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(su32(&full[st])) : "memory");
        ++issued;
        break;
      }
      info[st] = make_int4(pb, pk, (pk + 1 == pk1 ? kLast : 0) | (pj << kJobShift), pg);
      unsigned char* ys = sm + st * SB;
      const TmaJob& jb = jobs.job[pj];
      mbar_arm(&full[st], uint32_t(SB));
      if (COL)
        tma2d(ys, &jb.ymap, &full[st], pb * TILE, pk * TILE);
      else
        tma2d(ys, &jb.ymap, &full[st], pk * TILE, pb * TILE);
      tma2d(ys + kYTile, &jb.rmap, &full[st], pk * TILE, 0);
      ++pk;
      ++issued;
    }
    if (!ok) {  // let the copies already issued land before exiting
      for (int jj = issued > S ? issued - S : 0; jj < issued; ++jj)
        mbar_wait_bounded(&full[jj % S], uint32_t((jj / S) & 1), kSkWaitBudget);
    }
    return;
  }
  const int l7 = lane & 7, mi = lane >> 3;
  const int a_row = warp * 16 + l7 + (mi & 1) * 8, a_half = mi >> 1;
  const int at_rowoff = (mi >> 1) * 8 + l7, at_chunk = warp * 2 + (mi & 1);
  const int b_rowoff = (mi >> 1) * 8 + l7, b_half = mi & 1;
  float acc[NF][4];
#pragma unroll
  for (int f = 0; f < NF; ++f) acc[f][0] = acc[f][1] = acc[f][2] = acc[f][3] = 0.0f;
  for (int j = 0;; ++j) {
    const int st = j % S;
    if (!mbar_wait_bounded(&full[st], uint32_t((j / S) & 1), g_sk_budget)) s_abort = 1;
    const int4 inf = info[st];
    if (!s_abort && !(inf.z & kEnd)) {
      const int f1 = jobs.job[inf.z >> kJobShift].f1;  // uniform over the CTA
      const uint32_t ybase = su32(sm + st * SB), rbase = ybase + kYTile;
#pragma unroll
      for (int k16 = 0; k16 < TILE / 16; ++k16) {
        uint32_t a[4];
        if (COL)
          ldsm4t(a, swz(ybase, k16 * 16 + at_rowoff, at_chunk));
        else
          ldsm4(a, swz(ybase, a_row, k16 * 2 + a_half));
#pragma unroll
        for (int s = 0; s < NT; ++s)
#pragma unroll
          for (int fp = 0; fp < NF / 2; ++fp) {
            if (s > 0 && fp < f1) continue;  // zero terms of bf16 columns
            uint32_t bf[4];
            ldsm4(bf, swz(rbase, s * CP + fp * 16 + b_rowoff, k16 * 2 + b_half));
            mma16816(acc[2 * fp], a[0], a[1], a[2], a[3], bf[0], bf[1]);
            mma16816(acc[2 * fp + 1], a[0], a[1], a[2], a[3], bf[2], bf[3]);
          }
      }
    }
    __syncwarp();
    if (lane == 0) asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(su32(&empty[st])) : "memory");
    if (s_abort || (inf.z & kEnd)) break;
    if (!(inf.z & kLast)) continue;
    const TmaJob& jb = jobs.job[inf.z >> kJobShift];
    const int b = inf.x, c = jb.c, ngroups = jb.p.ngroups;
    const int64_t nout = COL ? jb.K : jb.M;
    const int64_t r0 = int64_t(b) * TILE + warp * 16 + g;
    if (ngroups == 1) {
#pragma unroll
      for (int f = 0; f < NF; ++f) {
        const int col = f * 8 + 2 * t;
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          const int64_t r = r0 + 8 * h;
          if (r >= nout) continue;
          if (COL) {
            if (col < c) col_emit(jb.co, r, col, acc[f][2 * h]);
            if (col + 1 < c) col_emit(jb.co, r, col + 1, acc[f][2 * h + 1]);
          } else {
            if (col < c) row_emit(jb.ro, r, col, acc[f][2 * h]);
            if (col + 1 < c) row_emit(jb.ro, r, col + 1, acc[f][2 * h + 1]);
          }
        }
      }
    } else {
      float* mine = jb.part + (int64_t(b) * ngroups + inf.w) * TILE * CP;
#pragma unroll
      for (int f = 0; f < NF; ++f) {
        const int col = f * 8 + 2 * t;
        const int lr = warp * 16 + g;
        *reinterpret_cast<float2*>(mine + lr * CP + col) = make_float2(acc[f][0], acc[f][1]);
        *reinterpret_cast<float2*>(mine + (lr + 8) * CP + col) = make_float2(acc[f][2], acc[f][3]);
      }
      if (last_arrival_c(jb.counters + b, unsigned(ngroups), tid)) {
        const int nq4 = (c + 3) / 4;
        const float* blk = jb.part + int64_t(b) * ngroups * TILE * CP;
        for (int e = tid; e < TILE * nq4; e += NTH) {
          const int lr = e / nq4, q0 = (e % nq4) * 4;
          const int64_t r = int64_t(b) * TILE + lr;
          if (r >= nout) continue;
          const float4 v = sum_splits4(reinterpret_cast<const float4*>(blk + lr * CP + q0),
                                       int64_t(TILE) * CP / 4, ngroups);
          const float vv[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            if (q0 + u >= c) break;
            if (COL)
              col_emit(jb.co, r, q0 + u, vv[u]);
            else
              row_emit(jb.ro, r, q0 + u, vv[u]);
          }
        }
      }
    }
#pragma unroll
    for (int f = 0; f < NF; ++f) acc[f][0] = acc[f][1] = acc[f][2] = acc[f][3] = 0.0f;
  }
}

// Sum of per-N-tile projection partials written by a GEMM epilogue.  Four
// consecutive lanes share one (row m, 4 columns q0..q0+3): lane s adds the
// float4s of tiles t = s, s + 4, ... in order (eight in flight), then the four
// sums combine as (l0 + l1) + (l2 + l3) through xor shuffles, which every lane
// of the four computes with the same operands (fixed order, bit-reproducible).
// Column q of row m is emitted as (q / lr) * r + q % lr when q % lr < r.  Up to
// two independent jobs per launch (blockIdx.y).
struct RowReduceJob {
  const float* part = nullptr;
  int nparts = 0;
  int64_t M = 0;
  SkRowOut o;
};
__global__ void reduce_rows_kernel(const __grid_constant__ RowReduceJob j0,
                                   const __grid_constant__ RowReduceJob j1, int pc, int lr,
                                   int r) {
  const RowReduceJob& J = blockIdx.y ? j1 : j0;
  const int nq4 = pc / 4;
  const int64_t e = int64_t(blockIdx.x) * blockDim.x + threadIdx.x;
  const int64_t item = e >> 2;
  const int sub = int(e & 3);
  const bool live = item < J.M * nq4;  // whole groups of four lanes share `live`
  const int64_t m = live ? item / nq4 : 0;
  const int q0 = live ? int(item % nq4) * 4 : 0;
  float4 v = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
  if (live) {
    const float4* src = reinterpret_cast<const float4*>(J.part + m * int64_t(J.nparts) * pc + q0);
    const int64_t stride4 = pc / 4;
    int t = sub;
    for (; t + 28 < J.nparts; t += 32) {
      float4 x[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) x[u] = __ldcg(src + int64_t(t + 4 * u) * stride4);
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        v.x += x[u].x; v.y += x[u].y; v.z += x[u].z; v.w += x[u].w;
      }
    }
    for (; t < J.nparts; t += 4) {
      const float4 x = __ldcg(src + int64_t(t) * stride4);
      v.x += x.x; v.y += x.y; v.z += x.z; v.w += x.w;
    }
  }
#pragma unroll
  for (int off = 1; off <= 2; off <<= 1) {
    v.x += __shfl_xor_sync(0xffffffffu, v.x, off);
    v.y += __shfl_xor_sync(0xffffffffu, v.y, off);
    v.z += __shfl_xor_sync(0xffffffffu, v.z, off);
    v.w += __shfl_xor_sync(0xffffffffu, v.w, off);
  }
  if (!live || sub != 0) return;
  const float vv[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
  for (int u = 0; u < 4; ++u) {
    const int q = q0 + u, gi = q / lr, qq = q % lr;
    if (qq < r) row_emit(J.o, m, gi * r + qq, vv[u]);
  }
}

PFN_cuTensorMapEncodeTiled_v12000 g_sk_encode = nullptr;
std::once_flag g_sk_encode_once;

// 2-D bf16 tensor map, 128-byte swizzle, box {box_x, box_y}, zero fill outside.
slora_status encode_bf16(CUtensorMap* m, const void* ptr, int64_t rows, int64_t cols, int64_t ld,
                         int box_x, int box_y) {
  std::call_once(g_sk_encode_once, [] {
    void* fn = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      g_sk_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
  });
  if (!g_sk_encode) SLORA_FAIL(SLORA_ERR_CUDA, "cuTensorMapEncodeTiled entry point not available");
  cuuint64_t dims[2] = {cuuint64_t(cols), cuuint64_t(rows)};
  cuuint64_t strides[1] = {cuuint64_t(ld) * 2};
  cuuint32_t box[2] = {cuuint32_t(box_x), cuuint32_t(box_y)};
  cuuint32_t es[2] = {1, 1};
  const CUresult r = g_sk_encode(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(ptr),
                                 dims, strides, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE,
                                 CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                                 CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS)
    SLORA_FAIL(SLORA_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d) for a skinny operand", int(r));
  return SLORA_OK;
}

bool tma_ok(const SkY& Y, int64_t rows, int64_t cols) {
  return !Y.map && Y.ptr && (reinterpret_cast<uintptr_t>(Y.ptr) & 15) == 0 && Y.ld % 8 == 0 &&
         rows > 0 && cols > 0 && Y.ld >= cols;
}

// Units of G chunks: about `target` units over the job's blocks (two per
// resident CTA for a job alone: dynamic balance), at most 32 groups per block
// (the last unit of a block sums that many tiles).
StreamPlan stream_plan(int64_t nout, int64_t nred,
                       int64_t target = 2 * int64_t(num_sms()) * kTmaCtasPerSm) {
  StreamPlan p;
  p.nblocks = int((nout + TILE - 1) / TILE);
  p.nchunks = int(std::max<int64_t>((nred + TILE - 1) / TILE, 1));
  const int64_t cap = int64_t(num_sms()) * kTmaCtasPerSm;
  int64_t want = (std::max<int64_t>(target, 1) + p.nblocks - 1) / std::max(p.nblocks, 1);
  if (want < 1) want = 1;
  if (want > 32) want = 32;
  if (want > p.nchunks) want = p.nchunks;
  p.G = int((p.nchunks + want - 1) / want);
  p.ngroups = (p.nchunks + p.G - 1) / p.G;
  p.nunits = p.nblocks * p.ngroups;
  p.ncta = int(std::min<int64_t>(p.nunits, cap));
  if (p.ncta < 1) p.ncta = 1;
  return p;
}

template <int NF, int NT, bool COL, int J>
slora_status launch_tma_kernel(const TmaJobs<J>& jb, cudaStream_t st) {
  auto kfn = skinny_tma_kernel<NF, NT, COL, J>;
  const int sm = tma_smem(NF * 8, NT);
  SLORA_CUDA(cudaFuncSetAttribute(kfn, cudaFuncAttributeMaxDynamicSharedMemorySize, sm));
  kfn<<<jb.ncta, NTH + 32, sm, st>>>(jb);
  SLORA_CHECK_LAUNCH();
  return SLORA_OK;
}
template <bool COL, int J>
slora_status launch_tma_jobs(const TmaJobs<J>& jb, int CP, int nt, cudaStream_t st) {
  if (nt == 3) {
    switch (CP) {
      case 16: return launch_tma_kernel<2, 3, COL, J>(jb, st);
      case 32: return launch_tma_kernel<4, 3, COL, J>(jb, st);
      case 48: return launch_tma_kernel<6, 3, COL, J>(jb, st);
      default: return launch_tma_kernel<8, 3, COL, J>(jb, st);
    }
  }
  switch (CP) {
    case 16: return launch_tma_kernel<2, 1, COL, J>(jb, st);
    case 32: return launch_tma_kernel<4, 1, COL, J>(jb, st);
    case 48: return launch_tma_kernel<6, 1, COL, J>(jb, st);
    default: return launch_tma_kernel<8, 1, COL, J>(jb, st);
  }
}

// Fills job `x` of a launch (its maps, plan, workspace slices).  The rsplit
// rows (NT * CP) are one TMA box high; the map's height is the rows that term
// count uses.
slora_status fill_tma_job(TmaJob& J, bool col, const SkY& Y, int64_t M, int64_t K, int c, int nt,
                          const void* rsplit, const StreamPlan& p, float* part,
                          unsigned* counters) {
  const int CP = padded(c);
  const int64_t I64 = round64(std::max<int64_t>(col ? M : K, 1));
  SLORA_TRY(encode_bf16(&J.ymap, Y.ptr, M, K, Y.ld, TILE, TILE));
  SLORA_TRY(encode_bf16(&J.rmap, rsplit, int64_t(nt) * CP, I64, I64, TILE, nt * CP));
  J.p = p;
  J.c = c;
  J.M = M;
  J.K = K;
  J.part = part;
  J.counters = counters;
  return SLORA_OK;
}

slora_status launch_tma(bool col, const SkY& Y, int64_t M, int64_t K, int c, int nt,
                        const SkRowOut& ro, const SkColOut& co, const SkWork& w, int64_t I64,
                        cudaStream_t st, int f1 = 0) {
  (void)I64;
  const StreamPlan p = col ? stream_plan(K, M) : stream_plan(M, K);
  TmaJobs<1> jb;
  SLORA_TRY(fill_tma_job(jb.job[0], col, Y, M, K, c, nt, w.rsplit, p, w.part, w.counters));
  jb.job[0].f1 = f1;
  jb.job[0].ro = ro;
  jb.job[0].co = co;
  jb.job[0].unit0 = 0;
  jb.njobs = 1;
  jb.nunits = p.nunits;
  jb.ncta = p.ncta;
  jb.ticket = w.counters + p.nblocks;
  LaunchScope ls(kSkinny, double(M) * K * 2, st);
  return col ? launch_tma_jobs<true, 1>(jb, padded(c), nt, st)
             : launch_tma_jobs<false, 1>(jb, padded(c), nt, st);
}

int64_t tma_part_floats(int64_t nout, int64_t nred, int c) {
  const StreamPlan p = stream_plan(nout, nred);
  return int64_t(p.nunits) * TILE * padded(c);
}
}  // namespace

// Workspace bounds hold for both term counts (the split count never exceeds
// the one of the smaller, 1-term footprint).
int64_t rowdot_part_floats(int64_t M, int64_t K, int c) {
  const Geo a = geometry(M, K, c, false), b = geometry(M, K, c, true);
  return std::max(int64_t(std::max(a.nsplit, b.nsplit)) * std::max<int64_t>(M, 1) * padded(c),
                  tma_part_floats(M, K, c));
}

int64_t coldot_part_floats(int64_t M, int64_t K, int c) {
  const Geo a = geometry(K, M, c, false), b = geometry(K, M, c, true);
  return std::max(int64_t(std::max(a.nsplit, b.nsplit)) * std::max<int64_t>(K, 1) * padded(c),
                  tma_part_floats(K, M, c));
}

namespace {
int job_terms(const SkColJob& j) { return fp32_terms(j.R) ? 3 : 1; }
// The shapes allow one launch (the workspace is sized on this alone).
bool batch_shape_ok(const SkColJob* jobs, int n) {
  if (n < 1 || n > kMaxTmaJobs) return false;
  const int CP = padded(jobs[0].c), nt = job_terms(jobs[0]);
  for (int k = 0; k < n; ++k) {
    const SkColJob& j = jobs[k];
    if (j.c <= 0 || j.c > 64 || padded(j.c) != CP || job_terms(j) != nt || j.M <= 0 ||
        j.K <= 0)
      return false;
  }
  return true;
}
// ... and the operands too.
bool batch_tma_ok(const SkColJob* jobs, int n) {
  if (!batch_shape_ok(jobs, n)) return false;
  for (int k = 0; k < n; ++k)
    if (!jobs[k].rs || !tma_ok(jobs[k].Y, jobs[k].M, jobs[k].K)) return false;
  return true;
}
// Each job's share of the two units per resident CTA, by its size.
void batch_plans(const SkColJob* jobs, int n, StreamPlan* plans) {
  double total = 0.0;
  for (int k = 0; k < n; ++k) total += double(jobs[k].M) * double(jobs[k].K);
  const double units = 2.0 * num_sms() * kTmaCtasPerSm;
  for (int k = 0; k < n; ++k) {
    const double share = total > 0 ? double(jobs[k].M) * double(jobs[k].K) / total : 1.0;
    plans[k] = stream_plan(jobs[k].K, jobs[k].M, std::max<int64_t>(1, llround(units * share)));
  }
}
}  // namespace

int64_t coldot_batch_part_floats(const SkColJob* jobs, int n) {
  int64_t most = 1;
  for (int k = 0; k < n; ++k)
    most = std::max(most, coldot_part_floats(jobs[k].M, jobs[k].K, jobs[k].c));
  if (!batch_shape_ok(jobs, n)) return most;
  StreamPlan plans[kMaxTmaJobs];
  batch_plans(jobs, n, plans);
  int64_t sum = 0;
  for (int k = 0; k < n; ++k) sum += int64_t(plans[k].nunits) * TILE * padded(jobs[k].c);
  return std::max(most, sum);
}

int64_t coldot_batch_counter_count(const SkColJob* jobs, int n) {
  int64_t most = 1;
  for (int k = 0; k < n; ++k)
    most = std::max(most, skinny_counter_count(jobs[k].M, jobs[k].K));
  if (!batch_shape_ok(jobs, n)) return most;
  StreamPlan plans[kMaxTmaJobs];
  batch_plans(jobs, n, plans);
  int64_t sum = 1;
  for (int k = 0; k < n; ++k) sum += plans[k].nblocks;
  return std::max(most, sum);
}

slora_status coldot_batch(const SkColJob* jobs, int n, float* part, unsigned* counters,
                          cudaStream_t st) {
  if (n <= 0) return SLORA_OK;
  if (!batch_tma_ok(jobs, n)) {
    for (int k = 0; k < n; ++k) {
      SkWork w;
      w.part = part;
      w.counters = counters;
      w.rsplit = jobs[k].rs;
      w.prepared = jobs[k].rs != nullptr;
      if (!w.prepared)
        SLORA_FAIL(SLORA_ERR_INVALID_ARG, "coldot_batch: job %d has no split operand", k);
      SLORA_TRY(coldot(jobs[k].Y, jobs[k].M, jobs[k].K, jobs[k].R, jobs[k].c, jobs[k].o, w, st));
    }
    return SLORA_OK;
  }
  StreamPlan plans[kMaxTmaJobs];
  batch_plans(jobs, n, plans);
  TmaJobs<kMaxTmaJobs> jb;
  const int CP = padded(jobs[0].c), nt = job_terms(jobs[0]);
  int unit = 0;
  float* pp = part;
  unsigned* cc = counters;
  double bytes = 0.0;
  for (int k = 0; k < n; ++k) {
    const SkColJob& j = jobs[k];
    SLORA_TRY(fill_tma_job(jb.job[k], true, j.Y, j.M, j.K, j.c, nt, j.rs, plans[k], pp, cc));
    jb.job[k].co = j.o;
    jb.job[k].unit0 = unit;
    unit += plans[k].nunits;
    pp += int64_t(plans[k].nunits) * TILE * CP;
    cc += plans[k].nblocks;
    bytes += double(j.M) * double(j.K) * 2.0;
  }
  jb.njobs = n;
  jb.nunits = unit;
  jb.ncta = int(std::min<int64_t>(unit, int64_t(num_sms()) * kTmaCtasPerSm));
  jb.ticket = cc;
  LaunchScope ls(kSkinny, bytes, st);
  return launch_tma_jobs<true, kMaxTmaJobs>(jb, CP, nt, st);
}

slora_status reduce_row_partials(const float* part0, int nparts0, int64_t M0, const SkRowOut& o0,
                                 const float* part1, int nparts1, int64_t M1, const SkRowOut& o1,
                                 int pc, int lr, int r, cudaStream_t st) {
  if ((M0 <= 0 && M1 <= 0) || pc <= 0) return SLORA_OK;
  if (pc % 4 || lr % 4) SLORA_FAIL(SLORA_ERR_SHAPE, "reduce_row_partials: pc, lr not multiples of 4");
  RowReduceJob j0, j1;
  j0.part = part0; j0.nparts = nparts0; j0.M = M0 > 0 ? M0 : 0; j0.o = o0;
  j1.part = part1; j1.nparts = nparts1; j1.M = M1 > 0 ? M1 : 0; j1.o = o1;
  const int64_t threads = std::max(j0.M, j1.M) * (pc / 4) * 4;
  LaunchScope ls(kSkinny,
                 (double(j0.M) * nparts0 + double(j1.M) * nparts1) * pc * 4 +
                     double(j0.M + j1.M) * r * (pc / lr) * 6, st);
  reduce_rows_kernel<<<dim3(unsigned((threads + 255) / 256), 2u), 256, 0, st>>>(j0, j1, pc, lr, r);
  SLORA_CHECK_LAUNCH();
  return SLORA_OK;
}

slora_status skinny_set_wait_budget(long long cycles) {
  const long long v = cycles < 0 ? kSkWaitBudget : cycles;
  SLORA_CUDA(cudaMemcpyToSymbol(g_sk_budget, &v, sizeof(v)));
  return SLORA_OK;
}

slora_status skinny_check_error(bool clear) {
  int v = 0, bad = 0;
  SLORA_CUDA(cudaMemcpyFromSymbol(&v, g_sk_error, sizeof(int)));
  SLORA_CUDA(cudaMemcpyFromSymbol(&bad, g_sk_bad_index, sizeof(int)));
  if (clear && (v || bad)) {
    const int z = 0;
    SLORA_CUDA(cudaMemcpyToSymbol(g_sk_error, &z, sizeof(int)));
    SLORA_CUDA(cudaMemcpyToSymbol(g_sk_bad_index, &z, sizeof(int)));
  }
  if (bad)
    SLORA_FAIL(SLORA_ERR_INVALID_ARG, "a channel index lies outside its weight (read as zero)");
  if (v) SLORA_FAIL(SLORA_ERR_TIMEOUT, "a skinny-contraction kernel's bounded wait expired");
  return SLORA_OK;
}

int64_t skinny_rsplit_elems(int64_t I) { return 3 * 64 * round64(std::max<int64_t>(I, 1)); }

int64_t skinny_counter_count(int64_t M, int64_t K) {
  return std::max<int64_t>((M + TILE - 1) / TILE, (K + TILE - 1) / TILE) + 1;
}

slora_status prep_r_batch(const SkPrep* jobs, int n, cudaStream_t st) {
  if (n <= 0) return SLORA_OK;
  if (n > 8) SLORA_FAIL(SLORA_ERR_SHAPE, "prep_r_batch: %d jobs (max 8)", n);
  PrepBatch b{};
  int64_t most = 1;
  double bytes = 0;
  for (int k = 0; k < n; ++k) {
    const SkPrep& j = jobs[k];
    if (j.c <= 0 || j.c > 64) SLORA_FAIL(SLORA_ERR_SHAPE, "prep_r_batch: %d columns", j.c);
    b.R[k] = j.R;
    b.c[k] = j.c;
    b.CP[k] = padded(j.c);
    b.nt[k] = fp32_terms(j.R) ? 3 : 1;
    b.I[k] = j.I;
    b.I64[k] = round64(std::max<int64_t>(j.I, 1));
    b.RS[k] = static_cast<__nv_bfloat16*>(j.rs);
    most = std::max(most, int64_t(b.CP[k]) * b.I64[k]);
    bytes += double(j.I) * j.c * (j.R.dt == kF32 ? 4 : 2) + double(b.nt[k]) * b.CP[k] * b.I64[k] * 2;
  }
  LaunchScope ls(kSkinny, bytes, st);
  prep_r_batch_kernel<<<dim3(unsigned((most + 255) / 256), unsigned(n)), 256, 0, st>>>(b);
  SLORA_CHECK_LAUNCH();
  return SLORA_OK;
}

slora_status rowdot(const SkY& Y, int64_t M, int64_t K, const SkR& R, int c, const SkRowOut& o,
                    const SkWork& w, cudaStream_t st) {
  if (M <= 0 || c <= 0) return SLORA_OK;
  if (c > 64) SLORA_FAIL(SLORA_ERR_SHAPE, "rowdot: %d columns (max 64)", c);
  const Geo g = geometry(M, K, c, fp32_terms(R));
  const int CP = g.CP, cps = g.cps;
  const int64_t I64 = round64(std::max<int64_t>(K, 1));
  const __nv_bfloat16* RS = static_cast<const __nv_bfloat16*>(w.rsplit);
  if (!w.prepared) SLORA_TRY(prep_r(R, c, CP, K, g.nt, static_cast<__nv_bfloat16*>(w.rsplit), st));
  if (tma_ok(Y, M, K)) {
    // columns below qsplit taken from a bf16 operand carry one nonzero term
    const int f1 = (g.nt == 3 && R.dt == kBF16 && R.ptr_b) ? std::min(R.qsplit, c) / 16 : 0;
    return launch_tma(false, Y, M, K, c, g.nt, o, SkColOut(), w, I64, st, f1);
  }
  const dim3 grid = dim3(unsigned(g.nblocks), unsigned(g.nsplit), 1u);
  LaunchScope ls(kSkinny,
                 double(M) * K * 2 + double(g.nsplit > 1 ? 2 * g.nsplit : 0) * M * CP * 4, st);
  if (g.nt == 3) {
    SLORA_SKINNY_SWITCH(rowdot_kernel, 3)
  } else {
    SLORA_SKINNY_SWITCH(rowdot_kernel, 1)
  }
  SLORA_CHECK_LAUNCH();
  return SLORA_OK;
}

slora_status coldot(const SkY& Y, int64_t M, int64_t K, const SkR& R, int c, const SkColOut& o,
                    const SkWork& w, cudaStream_t st) {
  if (K <= 0 || c <= 0) return SLORA_OK;
  if (c > 64) SLORA_FAIL(SLORA_ERR_SHAPE, "coldot: %d columns (max 64)", c);
  const Geo g = geometry(K, M, c, fp32_terms(R));
  const int CP = g.CP, cps = g.cps;
  const int64_t I64 = round64(std::max<int64_t>(M, 1));
  const __nv_bfloat16* RS = static_cast<const __nv_bfloat16*>(w.rsplit);
  if (!w.prepared) SLORA_TRY(prep_r(R, c, CP, M, g.nt, static_cast<__nv_bfloat16*>(w.rsplit), st));
  if (tma_ok(Y, M, K)) return launch_tma(true, Y, M, K, c, g.nt, SkRowOut(), o, w, I64, st);
  const dim3 grid = dim3(unsigned(g.nblocks), unsigned(g.nsplit), 1u);
  LaunchScope ls(kSkinny,
                 double(M) * K * 2 + double(g.nsplit > 1 ? 2 * g.nsplit : 0) * K * CP * 4, st);
  if (g.nt == 3) {
    SLORA_SKINNY_SWITCH(coldot_kernel, 3)
  } else {
    SLORA_SKINNY_SWITCH(coldot_kernel, 1)
  }
  SLORA_CHECK_LAUNCH();
  return SLORA_OK;
}

}  // namespace slora
