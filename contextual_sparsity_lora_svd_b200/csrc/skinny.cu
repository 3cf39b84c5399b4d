// Skinny (rank-sized) contractions, see skinny.cuh.
//
// 128-thread blocks over 64 x 64 tiles of Y staged in shared memory with
// cp.async (zero-filled past the edges, optional row gather); the rank-sized
// operand is staged transposed as 1 or 3 bf16 terms.  Each warp owns 16 rows
// (rowdot) or 16 columns (coldot) of the tile and issues mma.sync m16n8k16
// (bf16 in, fp32 accumulate).  The rank-sized operand is loaded one chunk
// ahead into registers and split on the fly.  Many small blocks per SM keep
// the HBM stream of Y busy; partial sums over the split dimension go to a
// workspace and the last block of each output block (atomic ticket) reduces
// them in a fixed order and writes the outputs: one launch per contraction,
// bit-reproducible results.
#include "skinny.cuh"

namespace slora {
namespace {

constexpr int TILE = 64, PAD = 72, NTH = 128;

__device__ __forceinline__ void cp_async16(void* dst, const void* src, int bytes) {
  const uint32_t d = static_cast<uint32_t>(__cvta_generic_to_shared(dst));
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(d), "l"(src), "r"(bytes)
               : "memory");
}
__device__ __forceinline__ void cp_async_wait_all() {
  asm volatile("cp.async.commit_group;\ncp.async.wait_group 0;" ::: "memory");
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

__device__ __forceinline__ float load_r(const SkR& R, int64_t i, int q) {
  const int64_t ii = R.map ? R.map[i] : i;
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

// The rank-sized operand for chunk rows [i0, i0 + 64): each thread holds
// CP * 64 / NTH values in registers (loaded one chunk ahead) and stores their
// NT-term split transposed into Rs[s][q][i].  Lanes walk q when q is the
// contiguous index of the source, otherwise i.
template <int CP>
struct RRegs {
  float v[CP * TILE / NTH];
};
template <int CP>
__device__ __forceinline__ void rmap(const SkR& R, int e, int& q, int& ii) {
  const bool q_fast = R.sq == 1 && (R.ptr_b == nullptr || R.sq_b == 1);
  if (q_fast) {
    q = e % CP;
    ii = e / CP;
  } else {
    q = e / TILE;
    ii = e % TILE;
  }
}
template <int CP>
__device__ __forceinline__ void load_r_regs(RRegs<CP>& rg, const SkR& R, int c, int64_t i0,
                                            int64_t I, int tid) {
#pragma unroll
  for (int j = 0; j < CP * TILE / NTH; ++j) {
    int q, ii;
    rmap<CP>(R, tid + NTH * j, q, ii);
    const int64_t i = i0 + ii;
    rg.v[j] = (q < c && i < I) ? load_r(R, i, q) : 0.0f;
  }
}
template <int CP, int NT>
__device__ __forceinline__ void store_r_regs(__nv_bfloat16 (*Rs)[CP][PAD], const RRegs<CP>& rg,
                                             const SkR& R, int tid) {
#pragma unroll
  for (int j = 0; j < CP * TILE / NTH; ++j) {
    int q, ii;
    rmap<CP>(R, tid + NTH * j, q, ii);
    __nv_bfloat16 tv[3];
    split_terms<NT>(rg.v[j], tv);
#pragma unroll
    for (int s = 0; s < NT; ++s) Rs[s][q][ii] = tv[s];
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
  float* base = q < o.qsplit ? o.out : o.out_b;
  const int qq = q < o.qsplit ? q : q - o.qsplit;
  float* dst = base + (o.trans ? int64_t(qq) * o.ldo + kk : kk * o.ldo + qq);
  *dst = o.accumulate ? *dst + v : v;
}

// cp.async double buffering: chunk j+1 is in flight while chunk j is consumed.
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
__device__ __forceinline__ void cp_async_wait_one() {
  asm volatile("cp.async.wait_group 1;" ::: "memory");
}

// Returns true in the one CTA (of the `n` sharing `counter`) that arrives last,
// after every CTA's partial is visible; that CTA resets the counter.
__device__ __forceinline__ bool last_arrival(unsigned* counter, unsigned n, int tid) {
  __shared__ unsigned s_last;
  __threadfence();
  __syncthreads();
  if (tid == 0) {
    const unsigned prev = atomicAdd(counter, 1u);
    s_last = (prev + 1 == n) ? 1u : 0u;
    if (s_last) *counter = 0u;
  }
  __syncthreads();
  if (s_last) __threadfence();
  return s_last != 0;
}

template <int NF, int NT>
__global__ void __launch_bounds__(NTH) rowdot_kernel(const SkY Y, int64_t M, int64_t K,
                                                     const SkR R, int c, int chunks_per_split,
                                                     float* __restrict__ part,
                                                     unsigned* __restrict__ counters,
                                                     const SkRowOut o) {
  constexpr int CP = NF * 8;
  extern __shared__ __align__(16) unsigned char sk_smem[];
  auto Ys = reinterpret_cast<__nv_bfloat16 (*)[TILE][PAD]>(sk_smem);  // [2][TILE][PAD]
  auto Rs = reinterpret_cast<__nv_bfloat16 (*)[NT][CP][PAD]>(sk_smem + 2 * TILE * PAD * 2);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31, g = lane >> 2, t = lane & 3;
  const int64_t m0 = int64_t(blockIdx.x) * TILE;
  const int ks = blockIdx.y, nsplit = gridDim.y;
  const int64_t nchunks = (K + TILE - 1) / TILE;
  const int64_t kc0 = int64_t(ks) * chunks_per_split;
  const int64_t kc1 = kc0 + chunks_per_split < nchunks ? kc0 + chunks_per_split : nchunks;
  float acc[NF][4];
#pragma unroll
  for (int f = 0; f < NF; ++f) acc[f][0] = acc[f][1] = acc[f][2] = acc[f][3] = 0.0f;
  RRegs<CP> rg;
  if (kc0 < kc1) {
    stage_y(Ys[0], Y, M, K, m0, kc0 * TILE, tid);
    load_r_regs<CP>(rg, R, c, kc0 * TILE, K, tid);
    store_r_regs<CP, NT>(Rs[0], rg, R, tid);
  }
  cp_async_commit();
  int buf = 0;
  for (int64_t kc = kc0; kc < kc1; ++kc, buf ^= 1) {
    const bool more = kc + 1 < kc1;
    if (more) {
      stage_y(Ys[buf ^ 1], Y, M, K, m0, (kc + 1) * TILE, tid);
      load_r_regs<CP>(rg, R, c, (kc + 1) * TILE, K, tid);
    }
    cp_async_commit();
    cp_async_wait_one();
    __syncthreads();
    const int r0 = warp * 16 + g;
#pragma unroll
    for (int k16 = 0; k16 < TILE / 16; ++k16) {
      const int kb = k16 * 16 + 2 * t;
      const uint32_t a0 = lds32(&Ys[buf][r0][kb]), a1 = lds32(&Ys[buf][r0 + 8][kb]);
      const uint32_t a2 = lds32(&Ys[buf][r0][kb + 8]), a3 = lds32(&Ys[buf][r0 + 8][kb + 8]);
#pragma unroll
      for (int f = 0; f < NF; ++f)
#pragma unroll
        for (int s = 0; s < NT; ++s)
          mma16816(acc[f], a0, a1, a2, a3, lds32(&Rs[buf][s][f * 8 + g][kb]),
                   lds32(&Rs[buf][s][f * 8 + g][kb + 8]));
    }
    __syncthreads();
    if (more) store_r_regs<CP, NT>(Rs[buf ^ 1], rg, R, tid);
  }
  const int64_t row0 = m0 + warp * 16 + g;
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
#pragma unroll
  for (int f = 0; f < NF; ++f) {
    const int col = f * 8 + 2 * t;
    if (row0 < M) {
      float* p = part + (int64_t(ks) * M + row0) * CP + col;
      p[0] = acc[f][0];
      p[1] = acc[f][1];
    }
    if (row0 + 8 < M) {
      float* p = part + (int64_t(ks) * M + row0 + 8) * CP + col;
      p[0] = acc[f][2];
      p[1] = acc[f][3];
    }
  }
  if (!last_arrival(counters + blockIdx.x, unsigned(nsplit), tid)) return;
  for (int e = tid; e < TILE * c; e += NTH) {
    const int64_t m = m0 + e / c;
    const int q = e % c;
    if (m >= M) continue;
    float v = 0.0f;
    for (int s2 = 0; s2 < nsplit; ++s2) v += __ldcg(part + (int64_t(s2) * M + m) * CP + q);
    row_emit(o, m, q, v);
  }
}

template <int NF, int NT>
__global__ void __launch_bounds__(NTH) coldot_kernel(const SkY Y, int64_t M, int64_t K,
                                                     const SkR R, int c, int chunks_per_split,
                                                     float* __restrict__ part,
                                                     unsigned* __restrict__ counters,
                                                     const SkColOut o) {
  constexpr int CP = NF * 8;
  extern __shared__ __align__(16) unsigned char sk_smem[];
  auto Ys = reinterpret_cast<__nv_bfloat16 (*)[TILE][PAD]>(sk_smem);  // [2][TILE][PAD]
  auto Rs = reinterpret_cast<__nv_bfloat16 (*)[NT][CP][PAD]>(sk_smem + 2 * TILE * PAD * 2);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31, g = lane >> 2, t = lane & 3;
  const int64_t k0 = int64_t(blockIdx.x) * TILE;
  const int ms = blockIdx.y, nsplit = gridDim.y;
  const int64_t nchunks = (M + TILE - 1) / TILE;
  const int64_t mc0 = int64_t(ms) * chunks_per_split;
  const int64_t mc1 = mc0 + chunks_per_split < nchunks ? mc0 + chunks_per_split : nchunks;
  float acc[NF][4];
#pragma unroll
  for (int f = 0; f < NF; ++f) acc[f][0] = acc[f][1] = acc[f][2] = acc[f][3] = 0.0f;
  const int mq = lane >> 3, rr = lane & 7;  // ldmatrix: matrix index, row within it
  RRegs<CP> rg;
  if (mc0 < mc1) {
    stage_y(Ys[0], Y, M, K, mc0 * TILE, k0, tid);
    load_r_regs<CP>(rg, R, c, mc0 * TILE, M, tid);
    store_r_regs<CP, NT>(Rs[0], rg, R, tid);
  }
  cp_async_commit();
  int buf = 0;
  for (int64_t mc = mc0; mc < mc1; ++mc, buf ^= 1) {
    const bool more = mc + 1 < mc1;
    if (more) {
      stage_y(Ys[buf ^ 1], Y, M, K, (mc + 1) * TILE, k0, tid);
      load_r_regs<CP>(rg, R, c, (mc + 1) * TILE, M, tid);
    }
    cp_async_commit();
    cp_async_wait_one();
    __syncthreads();
#pragma unroll
    for (int m16 = 0; m16 < TILE / 16; ++m16) {
      // A = Y^T fragment (16 k x 16 m) for columns warp*16.. of the tile
      const int mb = m16 * 16 + (mq >> 1) * 8;
      const int kb = warp * 16 + (mq & 1) * 8;
      uint32_t a0, a1, a2, a3;
      ldsm_x4_trans(a0, a1, a2, a3, &Ys[buf][mb + rr][kb]);
      const int mcol = m16 * 16 + 2 * t;
#pragma unroll
      for (int f = 0; f < NF; ++f)
#pragma unroll
        for (int s = 0; s < NT; ++s)
          mma16816(acc[f], a0, a1, a2, a3, lds32(&Rs[buf][s][f * 8 + g][mcol]),
                   lds32(&Rs[buf][s][f * 8 + g][mcol + 8]));
    }
    __syncthreads();
    if (more) store_r_regs<CP, NT>(Rs[buf ^ 1], rg, R, tid);
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
#pragma unroll
  for (int f = 0; f < NF; ++f) {
    const int col = f * 8 + 2 * t;
    if (kr < K) {
      float* p = part + (int64_t(ms) * K + kr) * CP + col;
      p[0] = acc[f][0];
      p[1] = acc[f][1];
    }
    if (kr + 8 < K) {
      float* p = part + (int64_t(ms) * K + kr + 8) * CP + col;
      p[0] = acc[f][2];
      p[1] = acc[f][3];
    }
  }
  if (!last_arrival(counters + blockIdx.x, unsigned(nsplit), tid)) return;
  for (int e = tid; e < TILE * c; e += NTH) {
    const int64_t k = k0 + e / c;
    const int q = e % c;
    if (k >= K) continue;
    float v = 0.0f;
    for (int s2 = 0; s2 < nsplit; ++s2) v += __ldcg(part + (int64_t(s2) * K + k) * CP + q);
    col_emit(o, k, q, v);
  }
}

constexpr int kTargetBlocks = 148 * 8;

int64_t splits_for(int64_t nblocks, int64_t nchunks) {
  if (nblocks < 1) nblocks = 1;
  if (nchunks < 1) nchunks = 1;
  int64_t s = (kTargetBlocks + nblocks - 1) / nblocks;
  if (s > nchunks) s = nchunks;
  if (s < 1) s = 1;
  if (s > 64) s = 64;
  return s;
}

int padded(int c) { return ((c + 15) / 16) * 16; }  // NF even keeps the templates few
bool fp32_terms(const SkR& R) { return R.dt == kF32 || (R.ptr_b && R.dt_b == kF32); }
int smem_bytes(int CP, int NT) { return 2 * TILE * PAD * 2 + 2 * NT * CP * PAD * 2; }

#define SLORA_SKINNY_CASE(KERNEL, NF_, NT)                                              \
  case NF_ * 8: {                                                                       \
    auto kfn = KERNEL<NF_, NT>;                                                         \
    const int sm = smem_bytes(NF_ * 8, NT);                                             \
    cudaFuncSetAttribute(kfn, cudaFuncAttributeMaxDynamicSharedMemorySize, sm);         \
    kfn<<<grid, NTH, sm, st>>>(Y, M, K, R, c, cps, part, counters, o);                  \
  } break;
#define SLORA_SKINNY_SWITCH(KERNEL, NT)   \
  switch (CP) {                           \
    SLORA_SKINNY_CASE(KERNEL, 2, NT)      \
    SLORA_SKINNY_CASE(KERNEL, 4, NT)      \
    SLORA_SKINNY_CASE(KERNEL, 6, NT)      \
    default:                              \
    SLORA_SKINNY_CASE(KERNEL, 8, NT)      \
  }

}  // namespace

int64_t rowdot_part_floats(int64_t M, int64_t K, int c) {
  const int64_t mb = (M + TILE - 1) / TILE, nch = (K + TILE - 1) / TILE;
  return splits_for(mb, nch) * std::max<int64_t>(M, 1) * padded(c);
}

int64_t coldot_part_floats(int64_t M, int64_t K, int c) {
  const int64_t kb = (K + TILE - 1) / TILE, nch = (M + TILE - 1) / TILE;
  return splits_for(kb, nch) * std::max<int64_t>(K, 1) * padded(c);
}

int64_t skinny_counter_count(int64_t M, int64_t K) {
  return std::max<int64_t>((M + TILE - 1) / TILE, (K + TILE - 1) / TILE) + 1;
}

slora_status rowdot(const SkY& Y, int64_t M, int64_t K, const SkR& R, int c, const SkRowOut& o,
                    float* part, unsigned* counters, cudaStream_t st) {
  if (M <= 0 || c <= 0) return SLORA_OK;
  if (c > 64) SLORA_FAIL(SLORA_ERR_SHAPE, "rowdot: %d columns (max 64)", c);
  const int CP = padded(c);
  const int nt = fp32_terms(R) ? 3 : 1;
  const int64_t mb = (M + TILE - 1) / TILE, nch = std::max<int64_t>((K + TILE - 1) / TILE, 1);
  const int64_t ns = splits_for(mb, nch);
  const int cps = int((nch + ns - 1) / ns);
  const int nsplit = int((nch + cps - 1) / cps);
  const dim3 grid = dim3(unsigned(mb), unsigned(nsplit), 1u);
  LaunchScope ls(kSkinny, double(M) * K * 2 + double(nsplit > 1 ? 2 * nsplit : 0) * M * CP * 4,
                 st);
  if (nt == 3) {
    SLORA_SKINNY_SWITCH(rowdot_kernel, 3)
  } else {
    SLORA_SKINNY_SWITCH(rowdot_kernel, 1)
  }
  SLORA_CHECK_LAUNCH();
  return SLORA_OK;
}

slora_status coldot(const SkY& Y, int64_t M, int64_t K, const SkR& R, int c, const SkColOut& o,
                    float* part, unsigned* counters, cudaStream_t st) {
  if (K <= 0 || c <= 0) return SLORA_OK;
  if (c > 64) SLORA_FAIL(SLORA_ERR_SHAPE, "coldot: %d columns (max 64)", c);
  const int CP = padded(c);
  const int nt = fp32_terms(R) ? 3 : 1;
  const int64_t kb = (K + TILE - 1) / TILE, nch = std::max<int64_t>((M + TILE - 1) / TILE, 1);
  const int64_t ns = splits_for(kb, nch);
  const int cps = int((nch + ns - 1) / ns);
  const int nsplit = int((nch + cps - 1) / cps);
  const dim3 grid = dim3(unsigned(kb), unsigned(nsplit), 1u);
  LaunchScope ls(kSkinny, double(M) * K * 2 + double(nsplit > 1 ? 2 * nsplit : 0) * K * CP * 4,
                 st);
  if (nt == 3) {
    SLORA_SKINNY_SWITCH(coldot_kernel, 3)
  } else {
    SLORA_SKINNY_SWITCH(coldot_kernel, 1)
  }
  SLORA_CHECK_LAUNCH();
  return SLORA_OK;
}

}  // namespace slora
