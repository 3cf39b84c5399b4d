// tcgen05 sliced GEMM for sm_100a (see gemm_tc.cuh for the operand forms).
//
// Persistent grid of cluster pairs (two 256-thread CTAs on two SMs) computing
// 256 x 256 tiles with tcgen05.mma.cta_group::2 (M = 256, N = 256, K = 16,
// bf16 x bf16 -> fp32 in TMEM):
//   warp 0      TMA producer: this CTA's halves of the A tile (128 x 64) and
//               of the B tile per stage
//   warp 1      MMA issuer (leader CTA): one thread issues tcgen05.mma
//   warp 2      TMEM allocator (512 columns = two 256-wide accumulators)
//   warps 4..7  epilogue: tcgen05.ld rows of the finished accumulator, apply
//               the epilogue, store bf16; the other accumulator is being
//               filled meanwhile
// Shared memory: stages of (16 KB A + 16 KB B), 128-byte swizzle (the TMA
// swizzle and the UMMA descriptor layout agree: 8-row / 1024-byte atoms).
// Every mbarrier wait is bounded (clock64 budget); on expiry the CTA raises
// an abort flag, waits (bounded) for its copies in flight, frees TMEM and
// returns, and the host reads SLORA_ERR_TIMEOUT from the device flag.
#include <cuda.h>
#include <cudaTypedefs.h>

#include <mutex>

#include "gemm_tc.cuh"

namespace slora {

__device__ int g_tc_error = 0;

namespace {

constexpr int BM = 128, BN = 256, BK = 64;
constexpr long long WAIT_BUDGET = 4000000000LL;    // ~2 s of SM clocks per wait

struct alignas(64) TcParams {
  CUtensorMap amap[4];
  CUtensorMap bmap[4][2];
  int nkb[4];
  int bmode[4];
  int bpair[4];
  int nseg;
  const int4* tiles;
  int n_mtiles, n_ntiles;
  int a_compact, out_compact;
  int paired;
  int N;
  int epi;
  int vec_out;  // output rows start on 16-byte boundaries (vector stores allowed)
  void* out0;
  void* out1;
  void* out2;
  long long ldo;
  const void* in0;
  const void* in1;
  long long ldi;
  // rank-r projection of the epilogue's values (see TcGemm::proj_*)
  const __nv_bfloat16* proj0;
  const __nv_bfloat16* proj1;
  long long ldproj;
  int proj_r;
  float* proj_part;
  long long proj_rows;
  // SwiGLU-backward epilogue through shared memory (two-CTA tiles): maps of
  // g, u (loads), dG, dU (stores), 32 x 32 boxes with 64-byte swizzle, and of
  // the projection matrices (32-channel x r boxes, unswizzled)
  CUtensorMap emap[6];
};

// One launch over the tiles of one or two GEMMs of the same epilogue kind
// (a context-row GEMM and its output-row twin): tile t < tot0 is tile t of
// p[0], the rest are p[1]'s, so the second GEMM's tiles fill the last round
// of the first's.
struct alignas(64) TcGroup {
  TcParams p[2];
  int ng;
  int tot0, tot1;
  int mpairs[2];
};

// The GEMM of combined tile t, its tile index and its M pair count.
struct TcPick {
  const TcParams* p;
  int t, n_mpairs;
};
__device__ __forceinline__ TcPick tc_pick(const TcGroup& G, int t) {
  TcPick k;
  const bool second = t >= G.tot0;
  k.p = &G.p[second ? 1 : 0];
  k.t = second ? t - G.tot0 : t;
  k.n_mpairs = G.mpairs[second ? 1 : 0];
  return k;
}

// ------------------------------------------------------------ PTX helpers
__device__ __forceinline__ uint32_t su32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}
__device__ __forceinline__ void mbar_init(uint64_t* b, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(su32(b)), "r"(count) : "memory");
}
__device__ __forceinline__ void mbar_expect_tx(uint64_t* b, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(su32(b)), "r"(bytes)
               : "memory");
}
__device__ __forceinline__ void mbar_arrive(uint64_t* b) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(su32(b)) : "memory");
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
// Bounded wait for the phase of parity `parity`; false on abort/expiry.
__device__ __forceinline__ bool mbar_wait(uint64_t* b, uint32_t parity, volatile int* abort) {
  if (mbar_try(b, parity)) return true;
  const long long t0 = clock64();
  while (true) {
    if (mbar_try(b, parity)) return true;
    if (*abort) return false;
    if (clock64() - t0 > WAIT_BUDGET) {
      *abort = 1;
      atomicExch(&g_tc_error, 1);
      return false;
    }
  }
}
__device__ __forceinline__ void fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}
// Shared-memory matrix descriptor, 128-byte swizzle, sm_100 version bits.
__device__ __forceinline__ uint64_t sdesc(uint32_t saddr, uint32_t lbo, uint32_t sbo) {
  uint64_t d = 0;
  d |= uint64_t((saddr & 0x3FFFFu) >> 4);
  d |= uint64_t((lbo >> 4) & 0x3FFFu) << 16;
  d |= uint64_t((sbo >> 4) & 0x3FFFu) << 32;
  d |= uint64_t(1) << 46;  // descriptor version (sm_100)
  d |= uint64_t(2) << 61;  // SWIZZLE_128B
  return d;
}
// Instruction descriptor: kind::f16 with bf16 A/B, fp32 D, M=128, N=256.
__host__ __device__ constexpr uint32_t idesc_bf16(int m, int n, int b_mn) {
  return (1u << 4) | (1u << 7) | (1u << 10) | (uint32_t(b_mn) << 16) |
         (uint32_t(n >> 3) << 17) | (uint32_t(m >> 4) << 24);
}
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, float* v) {
  uint32_t r[32];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
      "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, "
      "%16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
        "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]),
        "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]),
        "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr));
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
  for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
}

// Store 32 consecutive bf16 values (row-major, column c0..c0+31) with
// per-column masking at the right edge.
__device__ __forceinline__ void store_row32(__nv_bfloat16* row, int c0, int N, const float* v,
                                            bool vec = true) {
  if (vec && c0 + 32 <= N) {
    uint4* dst = reinterpret_cast<uint4*>(row + c0);
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      __nv_bfloat162 h[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) h[e] = __floats2bfloat162_rn(v[q * 8 + 2 * e], v[q * 8 + 2 * e + 1]);
      dst[q] = *reinterpret_cast<uint4*>(h);
    }
  } else {  // right edge: unrolled with predicates so v stays in registers
#pragma unroll
    for (int j = 0; j < 32; ++j)
      if (c0 + j < N) row[c0 + j] = __float2bfloat16_rn(v[j]);
  }
}
// Bulk prefetch into L2 of columns [c0, min(c0 + 256, N)) of one bf16 row
// (whole 16-byte units; rows start 16-byte aligned and c0 is a multiple of 256).
__device__ __forceinline__ void prefetch_row256(const __nv_bfloat16* row, int c0, int N) {
  const int cols = N - c0 < 256 ? N - c0 : 256;
  const uint32_t bytes = uint32_t(cols > 0 ? cols : 0) * 2u & ~15u;
  if (bytes)
    asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(row + c0), "r"(bytes)
                 : "memory");
}
__device__ __forceinline__ void load_row32(const __nv_bfloat16* row, int c0, int N, float* v) {
  if (c0 + 32 <= N) {
    const uint4* src = reinterpret_cast<const uint4*>(row + c0);
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      uint4 u = src[q];
      const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&u);
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        float2 f = __bfloat1622float2(h[e]);
        v[q * 8 + 2 * e] = f.x;
        v[q * 8 + 2 * e + 1] = f.y;
      }
    }
  } else {
#pragma unroll
    for (int j = 0; j < 32; ++j) v[j] = (c0 + j < N) ? __bfloat162float(row[c0 + j]) : 0.0f;
  }
}

// 32 consecutive bf16 of a row kept packed (4 x 16 bytes; zeros past N).
__device__ __forceinline__ void load_row32_raw(const __nv_bfloat16* row, int c0, int N,
                                               uint4 (&r)[4]) {
  if (c0 + 32 <= N) {
    const uint4* src = reinterpret_cast<const uint4*>(row + c0);
#pragma unroll
    for (int q = 0; q < 4; ++q) r[q] = src[q];
  } else {
    __nv_bfloat16* h = reinterpret_cast<__nv_bfloat16*>(r);
#pragma unroll
    for (int j = 0; j < 32; ++j) h[j] = (c0 + j < N) ? row[c0 + j] : __float2bfloat16_rn(0.0f);
  }
}
__device__ __forceinline__ float2 unpack2(const uint4 (&r)[4], int j2) {  // elements 2 j2, 2 j2 + 1
  const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(r);
  return __bfloat1622float2(h[j2]);
}

// ---- rank-r projection of epilogue rows on the tensor cores (mma.sync)
// Each epilogue warp stages its 32 rows x 32 values of a chunk as bf16 in a
// padded shared buffer (80-byte rows: the 8 row addresses of an ldmatrix fall
// in distinct bank groups), reads them back as m16n8k16 A fragments and
// multiplies by the chunk's 32 x R slice of the projection matrix P.
constexpr int PROJ_ROW = 40;                    // bf16 per staged row (32 + 8 padding)
constexpr int PROJ_BUF = 32 * PROJ_ROW;         // bf16 per warp buffer
constexpr int PROJ_SMEM = 4 * 2 * PROJ_BUF * 2;  // 4 epilogue warps x 2 buffers, bytes

__device__ __forceinline__ void mma16816_tc(float* d, const uint32_t* a, uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
      "{%8,%9}, {%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}
// Row `lane` of the warp's buffer = this lane's 32 values in bf16 (zeros if !valid).
__device__ __forceinline__ void proj_stage(__nv_bfloat16* buf, int lane, const float* v,
                                           bool valid) {
  uint4* dst = reinterpret_cast<uint4*>(buf + lane * PROJ_ROW);
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    __nv_bfloat162 h[4];
#pragma unroll
    for (int e = 0; e < 4; ++e)
      h[e] = valid ? __floats2bfloat162_rn(v[q * 8 + 2 * e], v[q * 8 + 2 * e + 1])
                   : __floats2bfloat162_rn(0.0f, 0.0f);
    dst[q] = *reinterpret_cast<const uint4*>(h);
  }
}
// acc[mb][nb] += rows mb*16.. of the staged 32 x 32 chunk times B[k][n] =
// P[(c0 + k) * ld + n] (zero for channels c0 + k >= N), n < R.
template <int R>
__device__ __forceinline__ void proj_mma(float (&acc)[2][2][4], const __nv_bfloat16* buf,
                                         const __nv_bfloat16* __restrict__ P, long long ld,
                                         int c0, int N, int lane) {
  const int g = lane >> 2, t = lane & 3;
  const unsigned short* Pu = reinterpret_cast<const unsigned short*>(P);
  auto el = [&](int k, int n) -> uint32_t {
    return (c0 + k < N) ? uint32_t(__ldg(Pu + (long long)(c0 + k) * ld + n)) : 0u;
  };
  uint32_t b[2][R / 8][2];
#pragma unroll
  for (int kb = 0; kb < 2; ++kb)
#pragma unroll
    for (int nb = 0; nb < R / 8; ++nb) {
      const int k0 = kb * 16 + 2 * t, n = nb * 8 + g;
      b[kb][nb][0] = el(k0, n) | (el(k0 + 1, n) << 16);
      b[kb][nb][1] = el(k0 + 8, n) | (el(k0 + 9, n) << 16);
    }
  const int arow = (lane & 7) + ((lane >> 3) & 1) * 8, acol = (lane >> 4) * 8;
#pragma unroll
  for (int mb = 0; mb < 2; ++mb)
#pragma unroll
    for (int kb = 0; kb < 2; ++kb) {
      uint32_t a[4];
      const uint32_t addr = su32(buf + (mb * 16 + arow) * PROJ_ROW + kb * 16 + acol);
      asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
                   : "=r"(a[0]), "=r"(a[1]), "=r"(a[2]), "=r"(a[3])
                   : "r"(addr));
#pragma unroll
      for (int nb = 0; nb < R / 8; ++nb) mma16816_tc(acc[mb][nb], a, b[kb][nb][0], b[kb][nb][1]);
    }
}
// The warp's partial of one N tile: rows rbase + mb*16 + g (+8) of the tile
// (valid ones only), columns off + nb*8 + 2t (+1), at
// part[((out_row + row) * n_ntiles + nt) * pc + col].
template <int R>
__device__ __forceinline__ void proj_store(float* part, long long out_row, int nvalid, int rbase,
                                           int nt, int n_ntiles, int pc, int off,
                                           const float (&acc)[2][2][4], int lane) {
  const int g = lane >> 2, t = lane & 3;
#pragma unroll
  for (int mb = 0; mb < 2; ++mb)
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int row = rbase + mb * 16 + g + 8 * h;
      if (row >= nvalid) continue;
      float* dst = part + ((out_row + row) * n_ntiles + nt) * pc + off;
#pragma unroll
      for (int nb = 0; nb < R / 8; ++nb)
        *reinterpret_cast<float2*>(dst + nb * 8 + 2 * t) =
            make_float2(acc[mb][nb][2 * h], acc[mb][nb][2 * h + 1]);
    }
}

// ------------------------------------------------------------------------
// 2-CTA variant: a cluster of two CTAs computes a 256 x 256 tile with
// tcgen05.mma.cta_group::2 (M = 256, N = 256, K = 16).  Each CTA loads only
// its own operand halves: its 128 rows of A and its 128 rows (or two 64-wide
// MN atoms) of B, so shared-memory traffic per SM per MMA is 8 KB instead of
// 12 KB.  The leader CTA (rank 0) arms the stage barrier for both CTAs'
// bytes; the peer's TMA loads complete on the leader's barrier
// (.cta_group::2).  The leader's single MMA thread issues the MMAs and its
// commits arrive on both CTAs' barriers (multicast commit).  Each CTA's
// epilogue drains its own 128 TMEM lanes and signals the leader.  No TMA
// multicast is used.
namespace {
constexpr int STAGES2 = 6;
constexpr int A2_BYTES = BM * BK * 2;                 // 16 KB
constexpr int B2_BYTES = (BN / 2) * BK * 2;           // 16 KB (this CTA's half)
constexpr int STAGE2_BYTES = A2_BYTES + B2_BYTES;     // 32 KB
constexpr int SMEM2_BYTES = STAGES2 * STAGE2_BYTES + 1024 + 512 + PROJ_SMEM;

// ---- TMA-staged SwiGLU-backward epilogue (two-CTA tiles)
// Each epilogue warp owns 16 KB: two load buffers of 6 KB (g and u chunks of
// 32 rows x 32 channels, 2 KB each, then the chunk's 32 x r slices of the two
// projection matrices, 1 KB each) and one 4 KB store buffer (dG and dU).
// Six main-loop stages leave too little shared memory for it, so this kernel
// variant runs five.
constexpr int STAGES2B = 5;
constexpr int EPI_WARP_BYTES = 16384;
constexpr int EPI_LOAD_BYTES = 6144;
constexpr int EPI_STORE_OFF = 2 * EPI_LOAD_BYTES;
constexpr int SMEM2B_BYTES = STAGES2B * STAGE2_BYTES + 1024 + 1024 + 4 * EPI_WARP_BYTES;
static_assert(SMEM2B_BYTES <= 232448, "shared memory of the TMA-epilogue GEMM");

// Byte offset of 16-byte unit j of row `row` in a buffer of 64-byte rows laid
// out by the TMA 64-byte swizzle (unit index XOR bits 1-2 of the row); the
// buffer starts on a 1024-byte boundary.
__device__ __forceinline__ uint32_t sw64(int row, int j) {
  return uint32_t(row * 64 + ((j ^ ((row >> 1) & 3)) << 4));
}
__device__ __forceinline__ uint4 lds128(uint32_t a) {
  uint4 v;
  asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "r"(a));
  return v;
}
__device__ __forceinline__ void sts128(uint32_t a, uint4 v) {
  asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(a), "r"(v.x), "r"(v.y),
               "r"(v.z), "r"(v.w)
               : "memory");
}
__device__ __forceinline__ void ldsm_x4(uint32_t a, uint32_t (&r)[4]) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(a));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t a, uint32_t (&r)[4]) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(a));
}
// generic-proxy shared-memory writes made visible to the TMA (async proxy)
__device__ __forceinline__ void fence_proxy_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}
__device__ __forceinline__ void tma_store(const CUtensorMap* m, uint32_t src, int x, int y) {
  asm volatile("cp.async.bulk.tensor.2d.global.shared::cta.tile.bulk_group [%0, {%2, %3}], [%1];"
               ::"l"(reinterpret_cast<uint64_t>(m)), "r"(src), "r"(x), "r"(y)
               : "memory");
}
__device__ __forceinline__ void bulk_commit() {
  asm volatile("cp.async.bulk.commit_group;" ::: "memory");
}
// the shared-memory reads of every committed bulk store are done
__device__ __forceinline__ void bulk_wait_read() {
  asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");
}
// every committed bulk store is complete
__device__ __forceinline__ void bulk_wait_all() {
  asm volatile("cp.async.bulk.wait_group 0;" ::: "memory");
}
// Pack 32 fp32 values as bf16 into row `row` of a 64-byte-swizzled buffer.
__device__ __forceinline__ void stage_row_sw64(uint32_t buf, int row, const float* v) {
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    __nv_bfloat162 h[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) h[e] = __floats2bfloat162_rn(v[8 * j + 2 * e], v[8 * j + 2 * e + 1]);
    sts128(buf + sw64(row, j), *reinterpret_cast<const uint4*>(h));
  }
}
// B fragments of a chunk's 32 x R projection slice staged densely (row k =
// channel c0 + k, R bf16 per row): b[kb][nb][h] holds rows kb*16 + h*8 + 2t,
// +1 of column nb*8 + g, the m16n8k16 B layout (ldmatrix .trans).
template <int R>
__device__ __forceinline__ void proj_bfrag(uint32_t (&b)[2][R / 8][2], uint32_t pbuf, int lane) {
  const int mi = lane >> 3, rr = lane & 7;
  if constexpr (R == 16) {
#pragma unroll
    for (int kb = 0; kb < 2; ++kb) {
      uint32_t r[4];
      ldsm_x4_t(pbuf + uint32_t((kb * 16 + (mi & 1) * 8 + rr) * 32 + (mi >> 1) * 16), r);
      b[kb][0][0] = r[0];
      b[kb][0][1] = r[1];
      b[kb][1][0] = r[2];
      b[kb][1][1] = r[3];
    }
  } else {
    uint32_t r[4];
    ldsm_x4_t(pbuf + uint32_t(((mi >> 1) * 16 + (mi & 1) * 8 + rr) * 16), r);
    b[0][0][0] = r[0];
    b[0][0][1] = r[1];
    b[1][0][0] = r[2];
    b[1][0][1] = r[3];
  }
}
// acc[mb][nb] += rows mb*16.. of the swizzle-staged 32 x 32 bf16 chunk times
// the B fragments.
template <int R>
__device__ __forceinline__ void proj_mma_sw(float (&acc)[2][2][4], uint32_t buf,
                                            const uint32_t (&b)[2][R / 8][2], int lane) {
  const int arow = (lane & 7) + ((lane >> 3) & 1) * 8, aj = lane >> 4;
#pragma unroll
  for (int mb = 0; mb < 2; ++mb)
#pragma unroll
    for (int kb = 0; kb < 2; ++kb) {
      uint32_t a[4];
      ldsm_x4(buf + sw64(mb * 16 + arow, kb * 2 + aj), a);
#pragma unroll
      for (int nb = 0; nb < R / 8; ++nb) mma16816_tc(acc[mb][nb], a, b[kb][nb][0], b[kb][nb][1]);
    }
}

__device__ __forceinline__ uint32_t cluster_rank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
__device__ __forceinline__ uint32_t map_to_rank(uint32_t saddr, uint32_t rank) {
  uint32_t out;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(out) : "r"(saddr), "r"(rank));
  return out;
}
__device__ __forceinline__ void cluster_sync_all() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;"
               ::: "memory");
}
__device__ __forceinline__ void tma_load_2sm(void* dst, const CUtensorMap* m, uint32_t bar_cluster,
                                             int x, int y) {
  asm volatile(
      "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4}], [%2];" ::"r"(su32(dst)),
      "l"(reinterpret_cast<uint64_t>(m)), "r"(bar_cluster), "r"(x), "r"(y)
      : "memory");
}
__device__ __forceinline__ void mma_bf16_2sm(uint32_t d, uint64_t a, uint64_t b, uint32_t idesc,
                                             uint32_t acc) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d),
      "l"(a), "l"(b), "r"(idesc), "r"(acc)
      : "memory");
}
// Commit the leader's MMAs; the arrival lands on the barrier at the same
// offset in both CTAs of the pair.
__device__ __forceinline__ void mma_commit_2sm(uint64_t* bar) {
  asm volatile(
      "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64"
      " [%0], %1;" ::"r"(su32(bar)), "h"(uint16_t(3))
      : "memory");
}
__device__ __forceinline__ void mbar_arrive_cluster(uint32_t bar_cluster) {
  asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(bar_cluster)
               : "memory");
}
}  // namespace

__device__ __forceinline__ void tma_load_s(uint32_t dst, const CUtensorMap* m, uint64_t* bar,
                                           int x, int y) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4}], [%2];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(m)), "r"(su32(bar)), "r"(x), "r"(y)
      : "memory");
}

// SwiGLU-backward epilogue of one epilogue warp (rows q*32 .. q*32 + 31 of
// this CTA's 128-row half), staged through shared memory:
//   * the g and u chunks (32 rows x 32 channels) and the chunk's slices of the
//     two projection matrices arrive by TMA into one of two load buffers;
//     chunks 0 and 1 of a tile are requested before the tile's accumulator is
//     ready, chunk c + 2 once chunk c has been read;
//   * dG and dU are packed to bf16 into the store buffer (64-byte swizzle,
//     conflict-free per row), written out by two TMA stores when all 32 rows
//     are valid (per-row stores otherwise), and read back by ldmatrix as the
//     A operand of the rank-R projections (mma.sync, fp32 partials).
template <int R>
__device__ __forceinline__ void tc2_bwd_epilogue(const TcGroup& G, uint8_t* wbuf, uint64_t* eb,
                                                 uint64_t* tfull, uint64_t* tempty,
                                                 volatile int* abort, uint32_t tbase,
                                                 uint32_t rank, int q, int lane, int cluster_id,
                                                 int n_clusters, int total) {
  constexpr int RB = R > 0 ? R / 8 : 1;
  const int r = q * 32 + lane;
  const uint32_t sbuf = su32(wbuf);
  const uint32_t obuf = sbuf + EPI_STORE_OFF;
  const uint32_t tempty_leader0 = map_to_rank(su32(&tempty[0]), 0);
  const uint32_t tempty_leader1 = map_to_rank(su32(&tempty[1]), 0);
  const uint32_t ebytes = 2u * 2048u + 2u * 32u * uint32_t(R) * 2u;
  uint32_t issued = 0, used = 0;
  bool ok = true;
  int it = 0;
  for (int t = cluster_id; t < total && ok; t += n_clusters, ++it) {
    const int acc = it & 1;
    const uint32_t aph = uint32_t(it >> 1) & 1u;
    const TcPick pk = tc_pick(G, t);
    const TcParams& p = *pk.p;
    const int mp = pk.t % pk.n_mpairs, nt = pk.t / pk.n_mpairs;
    const int mt = 2 * mp + int(rank);
    int out_row = 0, nvalid = 0;
    if (mt < p.n_mtiles) {
      const int4 tl = p.tiles[mt];
      out_row = p.out_compact ? tl.y : tl.x;
      nvalid = tl.z;
    }
    const int n0 = nt * BN;
    const int nch = min(8, (p.N - n0 + 31) / 32);  // n0 < N for every N tile
    const int row0 = out_row + q * 32;
    const bool valid = r < nvalid;
    const bool full_warp = q * 32 + 32 <= nvalid;
    const int64_t orow = int64_t(out_row) + r;
    auto issue = [&](int c) {  // warp-uniform; lane 0 requests chunk c
      if (lane == 0) {
        const uint32_t b = sbuf + (issued & 1u) * EPI_LOAD_BYTES;
        uint64_t* bar = eb + (issued & 1u);
        const int c0 = n0 + 32 * c;
        mbar_expect_tx(bar, ebytes);
        tma_load_s(b, &p.emap[0], bar, c0, row0);
        tma_load_s(b + 2048, &p.emap[1], bar, c0, row0);
        if (R > 0) {
          tma_load_s(b + 4096, &p.emap[4], bar, 0, c0);
          tma_load_s(b + 5120, &p.emap[5], bar, 0, c0);
        }
      }
      ++issued;
    };
    issue(0);
    if (nch > 1) issue(1);
    if (valid) {  // the rest of the tile's g and u rows on their way to L2
      prefetch_row256(static_cast<const __nv_bfloat16*>(p.in0) + orow * p.ldi, n0, p.N);
      prefetch_row256(static_cast<const __nv_bfloat16*>(p.in1) + orow * p.ldi, n0, p.N);
    }
    if (!mbar_wait(&tfull[acc], aph, abort)) { ok = false; break; }
    fence_after();
    const uint32_t tl = tbase + (uint32_t(q * 32) << 16) + uint32_t(acc * BN);
    __nv_bfloat16* dg = static_cast<__nv_bfloat16*>(p.out0) + orow * p.ldo;
    __nv_bfloat16* du = static_cast<__nv_bfloat16*>(p.out1) + orow * p.ldo;
    float pg[2][2][4] = {}, pu[2][2][4] = {};  // rank projections of dG and dU
#pragma unroll 1
    for (int c = 0; c < nch; ++c) {
      float v[32], w[32];
      tmem_ld32(tl + c * 32, v);  // dh
      const uint32_t b = sbuf + (used & 1u) * EPI_LOAD_BYTES;
      if (!mbar_wait(eb + (used & 1u), (used >> 1) & 1u, abort)) { ok = false; break; }
      ++used;
      uint4 gv[4], uv[4];
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        gv[j] = lds128(b + sw64(lane, j));
        uv[j] = lds128(b + 2048 + sw64(lane, j));
      }
      uint32_t bg[2][RB][2], bu[2][RB][2];
      if constexpr (R > 0) {
        proj_bfrag<R>(bg, b + 4096, lane);
        proj_bfrag<R>(bu, b + 5120, lane);
      }
#pragma unroll
      for (int j2 = 0; j2 < 16; ++j2) {
        const float2 g2 = unpack2(gv, j2), u2 = unpack2(uv, j2);
        const float ga[2] = {g2.x, g2.y}, ua[2] = {u2.x, u2.y};
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          const int j = 2 * j2 + e;
          const float sg = sigmoid_f(ga[e]);
          const float dh = v[j];
          v[j] = dh * ua[e] * sg * (1.0f + ga[e] * (1.0f - sg));  // dG
          w[j] = dh * ga[e] * sg;                                  // dU
        }
      }
      __syncwarp();  // every lane has read the load buffer: it may be refilled
      if (c + 2 < nch) issue(c + 2);
      if (lane == 0) bulk_wait_read();  // the previous chunk's stores have read the store buffer
      __syncwarp();
      stage_row_sw64(obuf, lane, v);
      stage_row_sw64(obuf + 2048, lane, w);
      fence_proxy_smem();
      __syncwarp();
      const int c0 = n0 + c * 32;
      if (full_warp) {
        if (lane == 0) {
          tma_store(&p.emap[2], obuf, c0, row0);
          tma_store(&p.emap[3], obuf + 2048, c0, row0);
          bulk_commit();
        }
      } else if (valid) {
        store_row32(dg, c0, p.N, v);
        store_row32(du, c0, p.N, w);
      }
      if constexpr (R > 0) {
        proj_mma_sw<R>(pg, obuf, bg, lane);
        proj_mma_sw<R>(pu, obuf + 2048, bu, lane);
      }
    }
    if (!ok) break;
    if constexpr (R > 0) {
      proj_store<R>(p.proj_part, out_row, nvalid, q * 32, nt, p.n_ntiles, 2 * R, 0, pg, lane);
      proj_store<R>(p.proj_part, out_row, nvalid, q * 32, nt, p.n_ntiles, 2 * R, R, pu, lane);
    }
    fence_before();
    __syncwarp();
    if (lane == 0) mbar_arrive_cluster(acc ? tempty_leader1 : tempty_leader0);
  }
  // before the CTA may exit: chunk loads still in flight land (bounded), and
  // the bulk stores complete
  for (uint32_t k = used; k < issued; ++k) {
    const long long t0 = clock64();
    while (!mbar_try(eb + (k & 1u), (k >> 1) & 1u) && clock64() - t0 < WAIT_BUDGET) {
    }
  }
  if (lane == 0) bulk_wait_all();
  __syncwarp();
}

template <int kStages, bool kBwdTma>
__global__ void __launch_bounds__(256, 1) tc_gemm2_kernel(const __grid_constant__ TcGroup G) {
  extern __shared__ uint8_t smem_raw2[];
  uint8_t* smem =
      reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw2) + 1023) & ~uintptr_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + kStages * STAGE2_BYTES);
  uint64_t* empty = full + kStages;
  uint64_t* tfull = empty + kStages;
  uint64_t* tempty = tfull + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(tempty + 2);
  volatile int* abort = reinterpret_cast<volatile int*>(tmem_slot + 1);
  // epilogue chunk-load barriers, two per epilogue warp (TMA-epilogue variant)
  uint64_t* ebar = reinterpret_cast<uint64_t*>(smem + kStages * STAGE2_BYTES + 256);

  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const uint32_t rank = cluster_rank();
  const bool leader = rank == 0;
  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    if (kBwdTma)
      for (int e = 0; e < 8; ++e) mbar_init(&ebar[e], 1);
    for (int a = 0; a < 2; ++a) {
      mbar_init(&tfull[a], 1);
      mbar_init(&tempty[a], 8);  // four epilogue warps in each CTA of the pair
    }
    *abort = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 2) {
    asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], 512;" ::"r"(
                     su32(tmem_slot))
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
  }
  fence_before();
  cluster_sync_all();  // barriers of both CTAs initialised before any remote signal
  fence_after();
  const uint32_t tbase = *tmem_slot;
  const int total = G.tot0 + G.tot1;
  const int cluster_id = blockIdx.x / 2, n_clusters = gridDim.x / 2;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    int stage = 0;
    uint32_t phase = 0;
    int issued = 0;
    bool ok = true;
    for (int t = cluster_id; t < total && ok; t += n_clusters) {
      const TcPick pk = tc_pick(G, t);
      const TcParams& p = *pk.p;
      const int mp = pk.t % pk.n_mpairs, nt = pk.t / pk.n_mpairs;
      const int mt = 2 * mp + int(rank);
      int a_row = 0;
      if (mt < p.n_mtiles) {
        const int4 tl = p.tiles[mt];
        a_row = p.a_compact ? tl.y : tl.x;
      }
      const int n0 = nt * (p.paired ? BN / 2 : BN);
      for (int s = 0; s < p.nseg && ok; ++s) {
        const int mode = p.bmode[s];
        const CUtensorMap* bm = &p.bmap[s][p.bpair[s] ? rank : 0];
        // this CTA's 128 B rows start at
        const int brow0 = p.bpair[s] ? n0 : nt * BN + 128 * int(rank);
        for (int kb = 0; kb < p.nkb[s]; ++kb) {
          if (!mbar_wait(&empty[stage], phase ^ 1u, abort)) { ok = false; break; }
          const uint32_t fbar = map_to_rank(su32(&full[stage]), 0);
          if (leader && lane == 0) mbar_expect_tx(&full[stage], 2 * STAGE2_BYTES);
          __syncwarp();
          uint8_t* sa = smem + stage * STAGE2_BYTES;
          uint8_t* sb = sa + A2_BYTES;
          if (lane == 0) tma_load_2sm(sa, &p.amap[s], fbar, kb * BK, a_row);
          if (mode == B_K) {
            if (lane == 1) tma_load_2sm(sb, bm, fbar, kb * BK, brow0);
          } else {  // B_MN: two 64-wide MN atoms of this CTA's half
            if (lane < 2)
              tma_load_2sm(sb + lane * 8192, bm, fbar, n0 + 64 * (2 * int(rank) + lane), kb * BK);
          }
          ++issued;
          if (++stage == kStages) { stage = 0; phase ^= 1u; }
        }
      }
    }
    if (!ok && leader && lane == 0) {
      // let the copies already armed land before the CTA can exit
      int st2 = stage;
      uint32_t ph2 = phase;
      for (int i = 0; i < kStages && i < issued; ++i) {
        if (--st2 < 0) { st2 = kStages - 1; ph2 ^= 1u; }
        const long long t0 = clock64();
        while (!mbar_try(&full[st2], ph2) && clock64() - t0 < WAIT_BUDGET) {
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------- MMA (leader CTA only)
    if (leader && lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      int it = 0;
      bool ok = true;
      for (int t = cluster_id; t < total && ok; t += n_clusters, ++it) {
        const TcParams& p = *tc_pick(G, t).p;
        const int acc = it & 1;
        const uint32_t aph = uint32_t(it >> 1) & 1u;
        if (!mbar_wait(&tempty[acc], aph ^ 1u, abort)) break;
        fence_after();
        const uint32_t d = tbase + uint32_t(acc * BN);
        bool first = true;
        for (int s = 0; s < p.nseg && ok; ++s) {
          const int bmn = p.bmode[s] == B_MN;
          const uint32_t idesc = idesc_bf16(2 * BM, BN, bmn);
          for (int kb = 0; kb < p.nkb[s]; ++kb) {
            if (!mbar_wait(&full[stage], phase, abort)) { ok = false; break; }
            fence_after();
            const uint32_t sa = su32(smem + stage * STAGE2_BYTES);
            const uint32_t sb = sa + A2_BYTES;
#pragma unroll
            for (int k = 0; k < BK / 16; ++k) {
              const uint64_t ad = sdesc(sa + k * 32, 16, 1024);
              const uint64_t bd = bmn ? sdesc(sb + k * 2048, 8192, 1024) : sdesc(sb + k * 32, 16, 1024);
              mma_bf16_2sm(d, ad, bd, idesc, (first && k == 0) ? 0u : 1u);
            }
            first = false;
            mma_commit_2sm(&empty[stage]);
            if (++stage == kStages) { stage = 0; phase ^= 1u; }
          }
        }
        mma_commit_2sm(&tfull[acc]);
      }
    }
    __syncwarp();
  } else if (kBwdTma && warp >= 4) {
    uint8_t* wb = smem + kStages * STAGE2_BYTES + 1024 + (warp - 4) * EPI_WARP_BYTES;
    uint64_t* eb = ebar + 2 * (warp - 4);
    // the group's GEMMs share proj_r (checked on the host)
    if (G.p[0].proj_r == 16)
      tc2_bwd_epilogue<16>(G, wb, eb, tfull, tempty, abort, tbase, rank, warp - 4, lane,
                           cluster_id, n_clusters, total);
    else if (G.p[0].proj_r == 8)
      tc2_bwd_epilogue<8>(G, wb, eb, tfull, tempty, abort, tbase, rank, warp - 4, lane,
                          cluster_id, n_clusters, total);
    else
      tc2_bwd_epilogue<0>(G, wb, eb, tfull, tempty, abort, tbase, rank, warp - 4, lane,
                          cluster_id, n_clusters, total);
  } else if (warp >= 4) {
    // ------------------------------------------------------------ epilogue
    const int q = warp - 4;
    const int r = q * 32 + lane;  // row within this CTA's 128-row half == TMEM lane
    __nv_bfloat16* pbuf0 = reinterpret_cast<__nv_bfloat16*>(
                               smem + kStages * STAGE2_BYTES + 512) + q * 2 * PROJ_BUF;
    __nv_bfloat16* pbuf1 = pbuf0 + PROJ_BUF;
    const uint32_t tempty_leader0 = map_to_rank(su32(&tempty[0]), 0);
    const uint32_t tempty_leader1 = map_to_rank(su32(&tempty[1]), 0);
    int it = 0;
    for (int t = cluster_id; t < total; t += n_clusters, ++it) {
      const int acc = it & 1;
      const uint32_t aph = uint32_t(it >> 1) & 1u;
      if (!mbar_wait(&tfull[acc], aph, abort)) break;
      fence_after();
      const TcPick pk = tc_pick(G, t);
      const TcParams& p = *pk.p;
      const int mp = pk.t % pk.n_mpairs, nt = pk.t / pk.n_mpairs;
      const int mt = 2 * mp + int(rank);
      int out_row = 0, nvalid = 0;
      if (mt < p.n_mtiles) {
        const int4 tl = p.tiles[mt];
        out_row = p.out_compact ? tl.y : tl.x;
        nvalid = tl.z;
      }
      const int n0 = nt * (p.paired ? BN / 2 : BN);
      const bool valid = r < nvalid;
      const int64_t orow = int64_t(out_row) + r;
      const uint32_t tl = tbase + (uint32_t(q * 32) << 16) + uint32_t(acc * BN);
      float v[32], w[32];
      if (p.epi == EPI_SWIGLU_FWD) {
        __nv_bfloat16* g = static_cast<__nv_bfloat16*>(p.out0) + orow * p.ldo;
        __nv_bfloat16* u = static_cast<__nv_bfloat16*>(p.out1) + orow * p.ldo;
        __nv_bfloat16* h = static_cast<__nv_bfloat16*>(p.out2) + orow * p.ldo;
        float pa[2][2][4] = {};  // rank projection of h over this tile's channels
#pragma unroll 1
        for (int c = 0; c < 4; ++c) {
          tmem_ld32(tl + c * 32, v);
          tmem_ld32(tl + 128 + c * 32, w);
          const int c0 = n0 + c * 32;
          if (valid) {
            store_row32(g, c0, p.N, v);
            store_row32(u, c0, p.N, w);
#pragma unroll
            for (int j = 0; j < 32; ++j) v[j] = silu_f(v[j]) * w[j];
            store_row32(h, c0, p.N, v);
          }
          if (p.proj_r && c0 < p.N) {  // warp-uniform
            proj_stage(pbuf0, lane, v, valid);
            __syncwarp();
            if (p.proj_r == 16)
              proj_mma<16>(pa, pbuf0, p.proj0, p.ldproj, c0, p.N, lane);
            else
              proj_mma<8>(pa, pbuf0, p.proj0, p.ldproj, c0, p.N, lane);
            __syncwarp();
          }
        }
        if (p.proj_r == 16)
          proj_store<16>(p.proj_part, out_row, nvalid, q * 32, nt, p.n_ntiles, 16, 0, pa, lane);
        else if (p.proj_r == 8)
          proj_store<8>(p.proj_part, out_row, nvalid, q * 32, nt, p.n_ntiles, 8, 0, pa, lane);
      } else if (p.epi == EPI_SWIGLU_BWD) {
        const __nv_bfloat16* gi = static_cast<const __nv_bfloat16*>(p.in0) + orow * p.ldi;
        const __nv_bfloat16* ui = static_cast<const __nv_bfloat16*>(p.in1) + orow * p.ldi;
        __nv_bfloat16* dg = static_cast<__nv_bfloat16*>(p.out0) + orow * p.ldo;
        __nv_bfloat16* du = static_cast<__nv_bfloat16*>(p.out1) + orow * p.ldo;
        if (valid) {  // the whole row segment of g and u on its way to L2 at once
          prefetch_row256(gi, n0, p.N);
          prefetch_row256(ui, n0, p.N);
        }
        // g and u of chunk c + 1 are loaded while chunk c is computed, so each
        // chunk's global-load latency hides behind the previous chunk's math
        uint4 gv[4], uv[4], gn[4], un[4];  // packed bf16 g and u of chunks c and c + 1
        float pg[2][2][4] = {}, pu[2][2][4] = {};  // rank projections of dG and dU
        if (valid && n0 < p.N) {
          load_row32_raw(gi, n0, p.N, gv);
          load_row32_raw(ui, n0, p.N, uv);
        }
#pragma unroll 1
        for (int c = 0; c < 8; ++c) {
          tmem_ld32(tl + c * 32, v);  // dh
          const int c0 = n0 + c * 32;
          const bool next = valid && c + 1 < 8 && c0 + 32 < p.N;
          if (next) {
            load_row32_raw(gi, c0 + 32, p.N, gn);
            load_row32_raw(ui, c0 + 32, p.N, un);
          }
          if (valid && c0 < p.N) {
#pragma unroll
            for (int j2 = 0; j2 < 16; ++j2) {
              const float2 g2 = unpack2(gv, j2), u2 = unpack2(uv, j2);
              const float ga[2] = {g2.x, g2.y}, ua[2] = {u2.x, u2.y};
#pragma unroll
              for (int e = 0; e < 2; ++e) {
                const int j = 2 * j2 + e;
                const float sg = sigmoid_f(ga[e]);
                const float dh = v[j];
                v[j] = dh * ua[e] * sg * (1.0f + ga[e] * (1.0f - sg));  // dG
                w[j] = dh * ga[e] * sg;                                  // dU
              }
            }
            store_row32(dg, c0, p.N, v);
            store_row32(du, c0, p.N, w);
          }
          if (p.proj_r && c0 < p.N) {  // warp-uniform
            const bool ok = valid;
            proj_stage(pbuf0, lane, v, ok);
            proj_stage(pbuf1, lane, w, ok);
            __syncwarp();
            if (p.proj_r == 16) {
              proj_mma<16>(pg, pbuf0, p.proj0, p.ldproj, c0, p.N, lane);
              proj_mma<16>(pu, pbuf1, p.proj1, p.ldproj, c0, p.N, lane);
            } else {
              proj_mma<8>(pg, pbuf0, p.proj0, p.ldproj, c0, p.N, lane);
              proj_mma<8>(pu, pbuf1, p.proj1, p.ldproj, c0, p.N, lane);
            }
            __syncwarp();
          }
          if (next) {
#pragma unroll
            for (int q4 = 0; q4 < 4; ++q4) {
              gv[q4] = gn[q4];
              uv[q4] = un[q4];
            }
          }
        }
        if (p.proj_r == 16) {
          proj_store<16>(p.proj_part, out_row, nvalid, q * 32, nt, p.n_ntiles, 32, 0, pg, lane);
          proj_store<16>(p.proj_part, out_row, nvalid, q * 32, nt, p.n_ntiles, 32, 16, pu, lane);
        } else if (p.proj_r == 8) {
          proj_store<8>(p.proj_part, out_row, nvalid, q * 32, nt, p.n_ntiles, 16, 0, pg, lane);
          proj_store<8>(p.proj_part, out_row, nvalid, q * 32, nt, p.n_ntiles, 16, 8, pu, lane);
        }
      } else {
        __nv_bfloat16* o = static_cast<__nv_bfloat16*>(p.out0) + orow * p.ldo;
#pragma unroll 1
        for (int c = 0; c < 8; ++c) {
          tmem_ld32(tl + c * 32, v);
          const int c0 = n0 + c * 32;
          if (valid && c0 < p.N) store_row32(o, c0, p.N, v, p.vec_out != 0);
        }
      }
      fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(acc ? tempty_leader1 : tempty_leader0);
    }
  }
  fence_before();
  __syncthreads();
  cluster_sync_all();  // the pair's MMAs, loads and remote arrivals are all finished
  if (warp == 2) {
    fence_after();
    asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, 512;" ::"r"(tbase) : "memory");
  }
}

// ----------------------------------------------------------- host helpers
PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;
std::once_flag g_encode_once;

slora_status get_encode() {
  std::call_once(g_encode_once, [] {
    void* fn = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
  });
  if (!g_encode) SLORA_FAIL(SLORA_ERR_CUDA, "cuTensorMapEncodeTiled entry point not available");
  return SLORA_OK;
}

slora_status encode(CUtensorMap* m, const TcMat& t, int box_x, int box_y,
                    CUtensorMapSwizzle swz = CU_TENSOR_MAP_SWIZZLE_128B) {
  if (!t.ptr) SLORA_FAIL(SLORA_ERR_INVALID_ARG, "tcgen05 GEMM: null operand");
  if ((reinterpret_cast<uintptr_t>(t.ptr) & 15) || (t.ld % 8) || t.rows <= 0 || t.cols <= 0)
    SLORA_FAIL(SLORA_ERR_ALIGN, "tcgen05 GEMM: operand not 16-byte aligned (ld=%lld)",
               (long long)t.ld);
  cuuint64_t dims[2] = {cuuint64_t(t.cols), cuuint64_t(t.rows)};
  cuuint64_t strides[1] = {cuuint64_t(t.ld) * 2};
  cuuint32_t box[2] = {cuuint32_t(box_x), cuuint32_t(box_y)};
  cuuint32_t es[2] = {1, 1};
  CUresult r = g_encode(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(t.ptr), dims,
                        strides, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE, swz,
                        CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS)
    SLORA_FAIL(SLORA_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d) rows=%lld cols=%lld ld=%lld",
               int(r), (long long)t.rows, (long long)t.cols, (long long)t.ld);
  return SLORA_OK;
}

bool g_attr_set = false;

}  // namespace

int64_t tc_ntiles(const TcGemm& g) {
  const int64_t ncols = g.paired ? BN / 2 : BN;
  return (g.N + ncols - 1) / ncols;
}

namespace {
// Kernel parameters of one GEMM; false in *run when it has no work.
slora_status build_params(const TcGemm& g, TcParams* pp, bool* run, bool* bwd_tma,
                          double* flops) {
  *run = false;
  if (g.proj0 && ((g.proj_r != 8 && g.proj_r != 16) || g.ldproj % 8 ||
                  !g.proj_part || (g.epi == EPI_SWIGLU_BWD && !g.proj1) || g.epi == EPI_STORE ||
                  (reinterpret_cast<uintptr_t>(g.proj0) & 15) ||
                  (reinterpret_cast<uintptr_t>(g.proj1) & 15) ||
                  (reinterpret_cast<uintptr_t>(g.proj_part) & 15)))
    SLORA_FAIL(SLORA_ERR_UNSUPPORTED, "tcgen05 GEMM: epilogue projection not available here");
  if (g.N <= 0) return SLORA_OK;
  if (g.tiles == nullptr) SLORA_FAIL(SLORA_ERR_INVALID_ARG, "tcgen05 GEMM: tile list missing");
  if (g.n_mtiles <= 0) return SLORA_OK;
  if (g.nseg < 1 || g.nseg > 4) SLORA_FAIL(SLORA_ERR_INVALID_ARG, "tcgen05 GEMM: nseg=%d", g.nseg);
  if (g.epi != EPI_STORE && (g.ldo % 8 || (g.epi == EPI_SWIGLU_BWD && g.ldi % 8)))
    SLORA_FAIL(SLORA_ERR_ALIGN, "tcgen05 GEMM: SwiGLU operands need rows of whole 16 bytes");
  if (g.N > (int64_t(1) << 30)) SLORA_FAIL(SLORA_ERR_SHAPE, "tcgen05 GEMM: N too large");
  SLORA_TRY(get_encode());
  TcParams& p = *pp;
  memset(&p, 0, sizeof(p));
  int64_t ksum = 0;
  for (int s = 0; s < g.nseg; ++s) {
    const TcSeg& sg = g.seg[s];
    if (sg.K <= 0)
      SLORA_FAIL(SLORA_ERR_SHAPE, "tcgen05 GEMM: segment %d has K=%lld", s, (long long)sg.K);
    SLORA_TRY(encode(&p.amap[s], sg.a, BK, BM));
    if (sg.bmode != B_K && sg.bmode != B_MN)
      SLORA_FAIL(SLORA_ERR_INVALID_ARG, "tcgen05 GEMM: unknown B operand form %d", sg.bmode);
    const int by = sg.bmode == B_K ? 128 : 64;
    SLORA_TRY(encode(&p.bmap[s][0], sg.b0, BK, by));
    if (sg.bpair) {
      if (sg.bmode != B_K)
        SLORA_FAIL(SLORA_ERR_INVALID_ARG, "tcgen05 GEMM: paired halves need a K-major B");
      SLORA_TRY(encode(&p.bmap[s][1], sg.b1, BK, by));
    }
    p.nkb[s] = int((sg.K + BK - 1) / BK);
    p.bmode[s] = sg.bmode;
    p.bpair[s] = sg.bpair;
    ksum += sg.K;
  }
  p.nseg = g.nseg;
  p.tiles = g.tiles;
  p.n_mtiles = g.n_mtiles;
  const int64_t ncols = g.paired ? BN / 2 : BN;
  p.n_ntiles = int((g.N + ncols - 1) / ncols);
  p.a_compact = g.a_compact;
  p.out_compact = g.out_compact;
  p.paired = g.paired;
  p.N = int(g.N);
  p.epi = g.epi;
  p.vec_out = (g.ldo % 8 == 0) && ((reinterpret_cast<uintptr_t>(g.out0) & 15) == 0);
  p.out0 = g.out0;
  p.out1 = g.out1;
  p.out2 = g.out2;
  p.ldo = g.ldo;
  p.in0 = g.in0;
  p.proj0 = static_cast<const __nv_bfloat16*>(g.proj0);
  p.proj1 = static_cast<const __nv_bfloat16*>(g.proj1);
  p.ldproj = g.ldproj;
  p.proj_r = g.proj0 ? g.proj_r : 0;
  p.proj_part = g.proj_part;
  p.proj_rows = g.proj_rows;
  p.in1 = g.in1;
  p.ldi = g.ldi;
  // SwiGLU backward through shared memory: operands addressable by TMA
  auto al16 = [](const void* q) { return (reinterpret_cast<uintptr_t>(q) & 15) == 0; };
  *bwd_tma = g.epi == EPI_SWIGLU_BWD && !g.paired && g.io_rows > 0 && al16(g.in0) &&
             al16(g.in1) && al16(g.out0) && al16(g.out1);
  if (*bwd_tma) {
    TcMat e;
    e.rows = g.io_rows;
    e.cols = g.N;
    e.ld = g.ldi;
    e.ptr = g.in0;
    SLORA_TRY(encode(&p.emap[0], e, 32, 32, CU_TENSOR_MAP_SWIZZLE_64B));
    e.ptr = g.in1;
    SLORA_TRY(encode(&p.emap[1], e, 32, 32, CU_TENSOR_MAP_SWIZZLE_64B));
    e.ld = g.ldo;
    e.ptr = g.out0;
    SLORA_TRY(encode(&p.emap[2], e, 32, 32, CU_TENSOR_MAP_SWIZZLE_64B));
    e.ptr = g.out1;
    SLORA_TRY(encode(&p.emap[3], e, 32, 32, CU_TENSOR_MAP_SWIZZLE_64B));
    if (p.proj_r) {
      e.rows = g.N;
      e.cols = p.proj_r;
      e.ld = g.ldproj;
      e.ptr = g.proj0;
      SLORA_TRY(encode(&p.emap[4], e, p.proj_r, 32, CU_TENSOR_MAP_SWIZZLE_NONE));
      e.ptr = g.proj1;
      SLORA_TRY(encode(&p.emap[5], e, p.proj_r, 32, CU_TENSOR_MAP_SWIZZLE_NONE));
    }
  }
  *flops = 2.0 * double(g.M) * double(g.paired ? 2 * g.N : g.N) * double(ksum);
  *run = true;
  return SLORA_OK;
}

// Up to two GEMMs in one launch (their tiles in one persistent schedule).
slora_status launch_group(const TcGemm* const* gs, int n, cudaStream_t st) {
  TcGroup G;  // copied into the launch's parameter buffer
  memset(&G, 0, sizeof(G));
  int ng = 0;
  bool tma[2] = {false, false};
  double flops = 0.0;
  for (int i = 0; i < n; ++i) {
    bool run = false;
    double f = 0.0;
    SLORA_TRY(build_params(*gs[i], &G.p[ng], &run, &tma[ng], &f));
    if (!run) continue;
    flops += f;
    ++ng;
  }
  if (ng == 0) return SLORA_OK;
  if (ng == 2 && (G.p[0].epi != G.p[1].epi || tma[0] != tma[1] ||
                  G.p[0].proj_r != G.p[1].proj_r)) {
    // different epilogue forms: one launch each
    const TcGemm* a[1] = {gs[0]};
    const TcGemm* b[1] = {gs[1]};
    SLORA_TRY(launch_group(a, 1, st));
    return launch_group(b, 1, st);
  }
  G.ng = ng;
  for (int i = 0; i < ng; ++i) G.mpairs[i] = (G.p[i].n_mtiles + 1) / 2;
  G.tot0 = G.mpairs[0] * G.p[0].n_ntiles;
  G.tot1 = ng > 1 ? G.mpairs[1] * G.p[1].n_ntiles : 0;
  if (!g_attr_set) {
    SLORA_CUDA(cudaFuncSetAttribute(tc_gemm2_kernel<STAGES2, false>,
                                    cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM2_BYTES));
    SLORA_CUDA(cudaFuncSetAttribute(tc_gemm2_kernel<STAGES2B, true>,
                                    cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM2B_BYTES));
    g_attr_set = true;
  }
  const int64_t ctiles = int64_t(G.tot0) + G.tot1;
  const int64_t maxc = num_sms() / 2;
  const int nclus = int(ctiles < maxc ? ctiles : maxc);
  LaunchScope ls(kGemmTC, flops, st);
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(unsigned(2 * nclus), 1, 1);
  cfg.blockDim = dim3(256, 1, 1);
  cfg.dynamicSmemBytes = tma[0] ? SMEM2B_BYTES : SMEM2_BYTES;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (tma[0])
    SLORA_CUDA(cudaLaunchKernelEx(&cfg, tc_gemm2_kernel<STAGES2B, true>, G));
  else
    SLORA_CUDA(cudaLaunchKernelEx(&cfg, tc_gemm2_kernel<STAGES2, false>, G));
  return SLORA_OK;
}
}  // namespace

slora_status gemm_tc(const TcGemm& g, cudaStream_t st) {
  const TcGemm* gs[1] = {&g};
  return launch_group(gs, 1, st);
}

slora_status gemm_tc_pair(const TcGemm& a, const TcGemm& b, cudaStream_t st) {
  const TcGemm* gs[2] = {&a, &b};
  return launch_group(gs, 2, st);
}

slora_status tc_check_error(bool clear) {
  int v = 0;
  SLORA_CUDA(cudaMemcpyFromSymbol(&v, g_tc_error, sizeof(int)));
  if (clear && v) {
    int z = 0;
    SLORA_CUDA(cudaMemcpyToSymbol(g_tc_error, &z, sizeof(int)));
  }
  if (v) SLORA_FAIL(SLORA_ERR_TIMEOUT, "a tcgen05 kernel's bounded wait expired");
  return SLORA_OK;
}

}  // namespace slora
