// Causal attention forward on the 5th-generation tensor cores (head width 128).
//
// Same result as attn_fwd_kernel (attention.cu): O = softmax(scale Q K^T,
// causal within each sequence) V per query head, with grouped key/value heads,
// and the natural-log log-sum-exp of every row's scaled scores; the P fed to
// the P V product is the bf16 rounding of the fp32 probabilities, and the row
// sums are taken before that rounding (SparseLoRA article, section 1: the
// attention core between the sparse q/k projections and the o projection).
//
// One CTA per (128 query rows, query head, sequence), 320 threads:
//   warps 0-7  softmax: query row r is tensor-memory lane r; warps w and
//              w + 4 share rows 32 (w % 4) .. + 31, w taking key / output
//              columns 0-63 and w + 4 columns 64-127.  Each reads its half row
//              of S with tcgen05.ld, masks, swaps the half maxima with its
//              partner through shared memory, exponentiates, and writes its
//              half row of P (bf16 pairs) back into tensor memory with
//              tcgen05.st; at the end it reads its half row of O, divides by
//              the row sum and stores it;
//   warp 8     TMA producer: the Q tile once, then the 128-key K and V tiles
//              through two stages (a K stage is refilled once its S is
//              computed, a V stage once its P V is done);
//   warp 9     MMA issuer (one thread): S_j = Q K_j^T into one of two S
//              buffers, and O += P_j V_j with P_j read from tensor memory as
//              the A operand and V read MN-major from shared memory.
// Tensor memory (512 columns): S at 0 and 128, O at 256, P at 384 and 448
// (128 keys as 64 columns of bf16 pairs).  S_{j+1} is computed while the
// softmax warps work on S_j; P is double-buffered, so softmax j writes P_j
// while P_{j-1} V_{j-1} may still run, and waits only for P_{j-2} V_{j-2}
// (or for P_{j-1} V_{j-1} when it has to rescale O).  Online softmax with a
// lazily moved reference: a row keeps the maximum m it started scaling with
// until a tile's maximum exceeds it by more than 8 (in log2 units); only then
// are its O row and sum rescaled by 2^(m_old - m_new).  Between rescales
// every probability is 2^(s - m) <= 2^8, so nothing overflows, and the final
// O / l and lse = (m + log2 l) ln 2 are the same quantities as with a
// reference that moves every tile.
//
// Every mbarrier wait is bounded; a wait that gives up raises g_attn_error
// (read by attn_check_error) and the CTA winds down: the producer waits (again
// bounded) for its copies in flight, the MMA thread for its MMAs, and the
// tensor memory is released.
#include <cuda.h>
#include <cudaTypedefs.h>

#include <algorithm>
#include <cmath>
#include <mutex>

#include "attention.cuh"

namespace slora {

__device__ int g_attn_error = 0;

namespace {

constexpr int kRows = 128;                 // query rows per CTA, keys per tile
constexpr int kHD = 128;                   // head width
constexpr int kPanel = 128 * 128;          // bytes: 128 rows x 64 bf16 (one 128-byte swizzle span)
constexpr int kTile = 2 * kPanel;          // 128 x 128 bf16
constexpr int kOffQ = 0;                   // 2 buffers (item parity)
constexpr int kOffK = 2 * kTile;           // 2 stages
constexpr int kOffV = 4 * kTile;           // 2 stages
constexpr int kOffBar = 6 * kTile;         // 22 mbarriers, the tensor-memory address, a flag
constexpr int kOffX = kOffBar + 256;       // row-block maxima: [tile parity][half][row] fp32
constexpr int kOffL = kOffX + 2048;        // row-sum halves: [half][row] fp32
constexpr int kOffSt = kOffL + 1024;       // per-warp store staging (8 softmax warps)
constexpr int kSmem = kOffSt + 8 * 32 * 5 * 16 + 1024; // + 1024-byte alignment slack
constexpr int kSoftWarps = 8;              // two per row block (one per 64-column half)
constexpr int kThreadsTc = (kSoftWarps + 2) * 32;
constexpr int kHalf = 64;                  // columns per softmax thread
constexpr uint32_t kTmemCols = 512;        // S buffers at 0 and 128, O at 256, P at 384 and 448
constexpr uint32_t kColP = 384;            // P: 128 keys as 64 columns of bf16 pairs, two buffers
constexpr float kLn2f = 0.6931471805599453f;
constexpr float kMasked = -1.0e30f;
constexpr float kLazy = 8.0f;              // rescale when the maximum rises by more
constexpr long long kWaitBudget = 2000000000LL;  // clock cycles

// kind::f16 instruction descriptor: fp32 D, bf16 A and B, A K-major, B K-major
// (b_mn = 0) or MN-major (1), M = 128, N = 128.
constexpr uint32_t idesc(int b_mn, int n = 128) {
  return (1u << 4) | (1u << 7) | (1u << 10) | (uint32_t(b_mn) << 16) | (uint32_t(n >> 3) << 17) |
         (uint32_t(128 >> 4) << 24);
}

__device__ __forceinline__ uint32_t su32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}
// Shared-memory matrix descriptor, 128-byte swizzle (sm_100 version bits).
__device__ __forceinline__ uint64_t sdesc(uint32_t saddr, uint32_t lbo, uint32_t sbo) {
  uint64_t d = 0;
  d |= uint64_t((saddr & 0x3FFFFu) >> 4);
  d |= uint64_t((lbo >> 4) & 0x3FFFu) << 16;
  d |= uint64_t((sbo >> 4) & 0x3FFFu) << 32;
  d |= uint64_t(1) << 46;
  d |= uint64_t(2) << 61;
  return d;
}
__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}
__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}
__device__ __forceinline__ void mbar_expect_tx(uint32_t bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes)
               : "memory");
}
// Bounded wait on the phase of parity `par`; false (and the error flag) when
// the budget runs out or another role of the CTA already gave up.
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t par, volatile int* abort) {
  const long long t0 = clock64();
  while (true) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(bar), "r"(par)
        : "memory");
    if (ok) return true;
    if (*abort) return false;
    if (clock64() - t0 > kWaitBudget) {
      *abort = 1;
      atomicExch(&g_attn_error, 1);
      return false;
    }
  }
}
__device__ __forceinline__ void tma_load(uint32_t dst, const CUtensorMap* m, uint32_t bar, int x,
                                         int y) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4}], [%2];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(m)), "r"(bar), "r"(x), "r"(y)
      : "memory");
}
__device__ __forceinline__ void mma(uint32_t d, uint64_t a, uint64_t b, uint32_t id, uint32_t acc) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d),
      "l"(a), "l"(b), "r"(id), "r"(acc)
      : "memory");
}
// A operand (M rows in lanes, two bf16 per 32-bit column) in tensor memory.
__device__ __forceinline__ void mma_ta(uint32_t d, uint32_t a_tmem, uint64_t b, uint32_t id,
                                       uint32_t acc) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d),
      "r"(a_tmem), "l"(b), "r"(id), "r"(acc)
      : "memory");
}
__device__ __forceinline__ void commit(uint32_t bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                   bar)
               : "memory");
}
__device__ __forceinline__ void fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}
// 32 consecutive fp32 columns of this thread's tensor-memory lane.
__device__ __forceinline__ void tld32(uint32_t taddr, uint32_t* r) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
      "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, "
      "%16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
        "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]),
        "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]),
        "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr)
      : "memory");
}
__device__ __forceinline__ void tst32(uint32_t taddr, const uint32_t* r) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], "
      "{%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, %16, "
      "%17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31, %32};" ::"r"(
          taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]),
      "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]),
      "r"(r[15]), "r"(r[16]), "r"(r[17]), "r"(r[18]), "r"(r[19]), "r"(r[20]), "r"(r[21]),
      "r"(r[22]), "r"(r[23]), "r"(r[24]), "r"(r[25]), "r"(r[26]), "r"(r[27]), "r"(r[28]),
      "r"(r[29]), "r"(r[30]), "r"(r[31])
      : "memory");
}
__device__ __forceinline__ void tst16(uint32_t taddr, const uint32_t* r) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], "
      "{%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, %16};" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]),
      "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]),
      "r"(r[15])
      : "memory");
}
__device__ __forceinline__ void tld_wait() {
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tst_wait() {
  asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}
__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}

// Warp-cooperative store of 32 rows (one per lane) through the warp's own
// shared staging area (32 x 5 chunks of 16 bytes): each lane hands in 4
// chunks (64 contiguous bytes) of its row; the warp writes them back 8 rows
// per instruction, each row's 64 bytes by 4 adjacent lanes, so a store
// instruction touches 8 row segments instead of 32.  `dst` is the lane's
// row address, `live` whether its row is stored.
constexpr int kStageWarp = 32 * 5 * 16;
__device__ __forceinline__ void warp_store_rows(uint32_t stage, const uint4 (&v)[4], char* dst,
                                                bool live) {
  const int lane = threadIdx.x & 31;
#pragma unroll
  for (int c = 0; c < 4; ++c)
    asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(stage + uint32_t((lane * 5 + c) * 16)),
                 "r"(v[c].x), "r"(v[c].y), "r"(v[c].z), "r"(v[c].w)
                 : "memory");
  __syncwarp();
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    const int row = k * 8 + (lane >> 2), c = lane & 3;
    char* rp = reinterpret_cast<char*>(
        __shfl_sync(0xffffffffu, reinterpret_cast<unsigned long long>(dst), row));
    const bool lv = __shfl_sync(0xffffffffu, live ? 1 : 0, row) != 0;
    uint4 x;
    asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(x.x), "=r"(x.y), "=r"(x.z), "=r"(x.w)
                 : "r"(stage + uint32_t((row * 5 + c) * 16))
                 : "memory");
    if (lv) reinterpret_cast<uint4*>(rp)[c] = x;
  }
  __syncwarp();
}
__device__ __forceinline__ uint4 f4bits(float a, float b, float c, float d) {
  return make_uint4(__float_as_uint(a), __float_as_uint(b), __float_as_uint(c), __float_as_uint(d));
}

struct TcFwdP {
  CUtensorMap mq, mk, mv;   // Q [T x H 128], K and V [T x KV 128]; boxes 64 x 128, 128-byte swizzle
  __nv_bfloat16* O;         // [T x H 128]
  float* lse;               // [batch][H][seq]
  int seq, H, KV, batch, nqb;
  int items;                // nqb * H * batch work items (query tile, head, sequence)
  float sl2;                // softmax scale * log2(e)
};

// Work item `it` (longest causal rows first): query tile qb, head h, sequence b.
// CTA c takes, in round k, item k G + c (k even) or k G + G - 1 - c (k odd):
// the alternating direction evens out the causal tile counts across CTAs.
__device__ __forceinline__ int item_at(int k, int G) {
  return k * G + ((k & 1) ? G - 1 - int(blockIdx.x) : int(blockIdx.x));
}
struct Item {
  int qb, h, b;
};
__device__ __forceinline__ Item item_of(const TcFwdP& p, int it) {
  const int hb = p.H * p.batch;
  Item x;
  x.qb = p.nqb - 1 - it / hb;
  x.h = (it % hb) % p.H;
  x.b = (it % hb) / p.H;
  return x;
}

}  // namespace

namespace {

// Waits for the phase of parity `par` with its own budget, ignoring the
// abort flag: used to let copies and MMAs already issued finish before the
// CTA releases its memory.
__device__ __forceinline__ void mbar_drain(uint32_t bar, uint32_t par) {
  volatile int never = 0;
  if (!mbar_wait(bar, par, &never)) atomicExch(&g_attn_error, 1);
}

__global__ void __launch_bounds__(kThreadsTc, 1) attn_fwd_tc_kernel(const __grid_constant__ TcFwdP p) {
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  const uint32_t raw = su32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;  // the swizzle pattern repeats every 1024 bytes
  unsigned char* gbase = smem_raw + (base - raw);
  const uint32_t sQ = base + kOffQ, sK = base + kOffK, sV = base + kOffV;
  const uint32_t bar = base + kOffBar;
  // mbarriers; those with two copies are indexed by buffer / stage (tile t uses t % 2)
  const uint32_t k_full = bar + 16, v_full = bar + 32, k_empty = bar + 48, v_empty = bar + 64,
                 s_full = bar + 80, s_free = bar + 96, p_full = bar + 112, pv_done = bar + 128,
                 o_empty = bar + 144, mma_done = bar + 152, q_full = bar + 160,
                 q_empty = bar + 176;  // Q buffer of item n: n % 2
  uint32_t* s_tmem = reinterpret_cast<uint32_t*>(gbase + kOffBar + 192);
  volatile int* abort = reinterpret_cast<volatile int*>(gbase + kOffBar + 200);
  float* xmax = reinterpret_cast<float*>(gbase + kOffX);  // [tile parity][half][row]
  float* lsum = reinterpret_cast<float*>(gbase + kOffL);  // [half][row]
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int G = int(gridDim.x);
  if (warp == 0) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     su32(s_tmem)),
                 "r"(kTmemCols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  if (tid == 32) {
    for (int s = 0; s < 2; ++s) {
      mbar_init(q_full + 8 * s, 1);
      mbar_init(q_empty + 8 * s, 1);
      mbar_init(k_full + 8 * s, 1);
      mbar_init(v_full + 8 * s, 1);
      mbar_init(k_empty + 8 * s, 1);
      mbar_init(v_empty + 8 * s, 1);
      mbar_init(s_full + 8 * s, 1);
      mbar_init(s_free + 8 * s, kSoftWarps);
      mbar_init(p_full + 8 * s, kSoftWarps);
      mbar_init(pv_done + 8 * s, 1);
    }
    mbar_init(o_empty, kSoftWarps);
    mbar_init(mma_done, 1);
    *abort = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  fence_before();
  __syncthreads();
  fence_after();
  const uint32_t tmem = *s_tmem;

  if (warp == kSoftWarps) {
    // ------------------------------------------------ TMA producer
    if (lane == 0) {
      int t = 0, nq = 0, nk = 0, nv = 0;
      bool ok = true;
      for (int n = 0; ok; ++n) {
        const int it = item_at(n, G);
        if (it >= p.items) break;
        const Item x = item_of(p, it);
        const int row0 = x.b * p.seq, g = x.h / (p.H / p.KV);
        // Q_n into buffer n % 2 once every S of item n - 2 is computed
        const int qb2 = n & 1;
        const uint32_t qf = q_full + 8 * qb2, sq = sQ + uint32_t(qb2 * kTile);
        if (n >= 2 && !mbar_wait(q_empty + 8 * qb2, uint32_t(((n - 2) >> 1) & 1), abort)) break;
        mbar_expect_tx(qf, kTile);
        tma_load(sq, &p.mq, qf, x.h * kHD, row0 + x.qb * kRows);
        tma_load(sq + kPanel, &p.mq, qf, x.h * kHD + 64, row0 + x.qb * kRows);
        nq = n + 1;
        for (int j = 0; j <= x.qb; ++j, ++t) {
          const int s = t & 1;
          const uint32_t par = uint32_t(((t - 2) >> 1) & 1);
          const int y = row0 + j * kRows;
          // K_t once S_{t-2} is computed, V_t once P_{t-2} V_{t-2} is done
          if (t >= 2 && !mbar_wait(k_empty + 8 * s, par, abort)) { ok = false; break; }
          const uint32_t kb = sK + uint32_t(s * kTile), vb = sV + uint32_t(s * kTile);
          mbar_expect_tx(k_full + 8 * s, kTile);
          tma_load(kb, &p.mk, k_full + 8 * s, g * kHD, y);
          tma_load(kb + kPanel, &p.mk, k_full + 8 * s, g * kHD + 64, y);
          nk = t + 1;
          if (t >= 2 && !mbar_wait(v_empty + 8 * s, par, abort)) { ok = false; break; }
          mbar_expect_tx(v_full + 8 * s, kTile);
          tma_load(vb, &p.mv, v_full + 8 * s, g * kHD, y);
          tma_load(vb + kPanel, &p.mv, v_full + 8 * s, g * kHD + 64, y);
          nv = t + 1;
        }
      }
      // the copies issued last into each buffer have landed before the CTA
      // can release its shared memory (on the normal path they were consumed)
      for (int u = ::max(0, nq - 2); u < nq; ++u)
        mbar_drain(q_full + 8 * (u & 1), uint32_t((u >> 1) & 1));
      for (int u = ::max(0, nk - 2); u < nk; ++u)
        mbar_drain(k_full + 8 * (u & 1), uint32_t((u >> 1) & 1));
      for (int u = ::max(0, nv - 2); u < nv; ++u)
        mbar_drain(v_full + 8 * (u & 1), uint32_t((u >> 1) & 1));
    }
    __syncwarp();
  } else if (warp == kSoftWarps + 1) {
    // ------------------------------------------------ MMA issuer
    if (lane == 0) {
      bool ok = true;
      int t = 0;
      // P V of the previous tile, issued after the next tile's S: its tile
      // index, whether it opens an item, and the item's ordinal
      int pv_t = -1, pv_n = 0;
      bool pv_first = false;
      auto issue_pv = [&]() -> bool {
        const int sp = pv_t & 1;
        if (!mbar_wait(p_full + 8 * sp, uint32_t((pv_t >> 1) & 1), abort)) return false;
        if (!mbar_wait(v_full + 8 * sp, uint32_t((pv_t >> 1) & 1), abort)) return false;
        // the first P V of an item overwrites O: the previous item's O is read
        if (pv_first && pv_n >= 1 && !mbar_wait(o_empty, uint32_t((pv_n - 1) & 1), abort))
          return false;
        fence_after();
        const uint32_t vt = sV + uint32_t(sp * kTile);
        const uint32_t pa = tmem + kColP + uint32_t(sp * 64);
#pragma unroll
        for (int kk = 0; kk < kRows / 16; ++kk)
          mma_ta(tmem + 2u * kRows, pa + uint32_t(kk * 8),
                 sdesc(vt + uint32_t(kk * 2048), kPanel, 1024), idesc(1),
                 (!pv_first || kk > 0) ? 1u : 0u);
        commit(pv_done + 8 * sp);
        commit(v_empty + 8 * sp);
        return true;
      };
      for (int n = 0; ok; ++n) {
        const int it = item_at(n, G);
        if (it >= p.items) break;
        const Item x = item_of(p, it);
        // the previous item's last P V goes first: its epilogue waits on it,
        // while this item's S waits for its Q and K to land
        if (pv_t >= 0) {
          if (!issue_pv()) { ok = false; break; }
          pv_t = -1;
        }
        const uint32_t sq = sQ + uint32_t((n & 1) * kTile);
        if (!mbar_wait(q_full + 8 * (n & 1), uint32_t((n >> 1) & 1), abort)) { ok = false; break; }
        for (int j = 0; j <= x.qb; ++j, ++t) {
          const int s = t & 1;
          // S_t = Q K_t^T into S buffer t % 2
          if (!mbar_wait(k_full + 8 * s, uint32_t((t >> 1) & 1), abort) ||
              (t >= 2 && !mbar_wait(s_free + 8 * s, uint32_t(((t - 2) >> 1) & 1), abort))) {
            ok = false;
            break;
          }
          fence_after();
          const uint32_t d = tmem + uint32_t(s * kRows);
          const uint32_t kt = sK + uint32_t(s * kTile);
#pragma unroll
          for (int kk = 0; kk < kHD / 16; ++kk) {
            const uint32_t off = uint32_t((kk >> 2) * kPanel + (kk & 3) * 32);
            mma(d, sdesc(sq + off, 16, 1024), sdesc(kt + off, 16, 1024), idesc(0),
                kk > 0 ? 1u : 0u);
          }
          commit(s_full + 8 * s);
          commit(k_empty + 8 * s);
          if (j == x.qb) commit(q_empty + 8 * (n & 1));  // every S of this item issued
          if (pv_t >= 0 && !issue_pv()) { ok = false; break; }
          pv_t = t;
          pv_n = n;
          pv_first = j == 0;
        }
      }
      if (ok && pv_t >= 0) issue_pv();
      // every MMA issued has completed before the tensor memory is released
      commit(mma_done);
      mbar_drain(mma_done, 0);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------ softmax
    // warp w: rows 32 (w % 4) .. + 31 (its tensor-memory lanes), key / output
    // columns 64 (w / 4) .. + 63; the two warps of a row block share each
    // tile's maximum through shared memory (named barrier 1 + w % 4).  A wait
    // that gives up turns this warp's `ok` off (warp-uniform, since the
    // tensor-memory accesses are warp-collective); the loops still run to
    // their end so that both warps of a row block meet at every pair barrier,
    // the waits after an abort returning at once.
    const int lq = warp & 3, hf = warp >> 2;
    const int r = lq * 32 + lane;
    const uint32_t lbase = tmem + (uint32_t(lq * 32) << 16);
    const uint32_t pair_bar = uint32_t(1 + lq);
    bool ok = true;
    int t = 0;
    for (int n = 0;; ++n) {
      const int it = item_at(n, G);
      if (it >= p.items) break;
      const Item x = item_of(p, it);
      const int row0 = x.b * p.seq;
      const int qi = x.qb * kRows + r;
      float m = kMasked, l = 0.f;
      for (int j = 0; j <= x.qb; ++j, ++t) {
        const int s = t & 1;
        ok = __all_sync(0xffffffffu, ok && mbar_wait(s_full + 8 * s, uint32_t((t >> 1) & 1), abort));
        uint32_t sv[kHalf];
        float mh = kMasked;
        if (ok) {
          fence_after();
          tld32(lbase + uint32_t(s * kRows + hf * kHalf), sv);
          tld32(lbase + uint32_t(s * kRows + hf * kHalf + 32), sv + 32);
          tld_wait();
          fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(s_free + 8 * s);
          // maximum over the raw scores (the scale is positive); the last
          // tile holds the keys past this row (causal) and past the sequence,
          // set to a huge negative raw score.  Eight partial maxima and sums
          // keep the dependency chains short.
          float mx[8];
#pragma unroll
          for (int e = 0; e < 8; ++e) mx[e] = kMasked;
          if (j == x.qb) {
            const int lim = ::min(qi, p.seq - 1) - j * kRows - hf * kHalf;  // last live column
#pragma unroll
            for (int i = 0; i < kHalf; ++i) {
              if (i > lim) sv[i] = __float_as_uint(kMasked);
              mx[i & 7] = fmaxf(mx[i & 7], __uint_as_float(sv[i]));
            }
          } else {
#pragma unroll
            for (int i = 0; i < kHalf; ++i) mx[i & 7] = fmaxf(mx[i & 7], __uint_as_float(sv[i]));
          }
          mh = fmaxf(fmaxf(fmaxf(mx[0], mx[1]), fmaxf(mx[2], mx[3])),
                     fmaxf(fmaxf(mx[4], mx[5]), fmaxf(mx[6], mx[7])));
        }
        xmax[(s * 2 + hf) * kRows + r] = mh;
        asm volatile("bar.sync %0, 64;" ::"r"(pair_bar) : "memory");
        if (!ok) continue;
        const float mt = fmaxf(mh, xmax[(s * 2 + (hf ^ 1)) * kRows + r]) * p.sl2;
        float c = 1.f;
        bool resc = false;
        if (j == 0) {
          m = mt;
        } else if (mt > m + kLazy) {
          c = ex2(m - mt);
          m = mt;
          resc = true;
        }
        const float nm = -m;
        float sm[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) sm[e] = 0.f;
        uint32_t pk[kHalf / 2];
#pragma unroll
        for (int i = 0; i < kHalf / 2; ++i) {
          const float p0 = ex2(fmaf(__uint_as_float(sv[2 * i]), p.sl2, nm));
          const float p1 = ex2(fmaf(__uint_as_float(sv[2 * i + 1]), p.sl2, nm));
          sm[(2 * i) & 7] += p0;
          sm[(2 * i + 1) & 7] += p1;
          pk[i] = pack_bf16x2(p0, p1);
        }
        const float rs = ((sm[0] + sm[1]) + (sm[2] + sm[3])) + ((sm[4] + sm[5]) + (sm[6] + sm[7]));
        l = l * c + rs;  // this half's share of the row sum
        // P_t goes to tensor-memory buffer t % 2, free once P_{t-2} V_{t-2}
        // is done; O is rescaled only after P_{t-1} V_{t-1} is done (MMAs
        // complete in order, so that covers P_{t-2} V_{t-2} too)
        if (__any_sync(0xffffffffu, resc)) {
          ok = __all_sync(0xffffffffu, mbar_wait(pv_done + 8 * ((t - 1) & 1),
                                                 uint32_t(((t - 1) >> 1) & 1), abort));
          if (!ok) continue;
          fence_after();
#pragma unroll
          for (int q = 0; q < kHalf / 32; ++q) {
            uint32_t o[32];
            const uint32_t ta = lbase + uint32_t(2 * kRows + hf * kHalf + 32 * q);
            tld32(ta, o);
            tld_wait();
#pragma unroll
            for (int e = 0; e < 32; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * c);
            tst32(ta, o);
          }
        } else if (t >= 2) {
          ok = __all_sync(0xffffffffu,
                          mbar_wait(pv_done + 8 * s, uint32_t(((t - 2) >> 1) & 1), abort));
          if (!ok) continue;
          fence_after();
        }
        // this half of row r of P: keys 64 hf .. + 63 as 32 columns of bf16 pairs
        tst32(lbase + kColP + uint32_t(s * 64 + hf * 32), pk);
        tst_wait();
        fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(p_full + 8 * s);
      }
      // both halves of the row sum, added in a fixed order
      lsum[hf * kRows + r] = l;
      asm volatile("bar.sync %0, 64;" ::"r"(pair_bar) : "memory");
      const float lt = lsum[r] + lsum[kRows + r];
      const int tl = t - 1;  // the item's last tile
      ok = __all_sync(0xffffffffu, ok && mbar_wait(pv_done + 8 * (tl & 1),
                                                   uint32_t((tl >> 1) & 1), abort));
      if (ok) {
        fence_after();
        uint32_t o[kHalf];
        tld32(lbase + uint32_t(2 * kRows + hf * kHalf), o);
        tld32(lbase + uint32_t(2 * kRows + hf * kHalf + 32), o + 32);
        tld_wait();
        fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(o_empty);  // the next item's P V may overwrite O
        {
          const float inv = 1.f / lt;
          char* dst = reinterpret_cast<char*>(p.O + (int64_t(row0) + qi) * (int64_t(p.H) * kHD) +
                                              x.h * kHD + hf * kHalf);
          const uint32_t stage = base + uint32_t(kOffSt + warp * kStageWarp);
#pragma unroll
          for (int hh = 0; hh < 2; ++hh) {  // 32 columns (64 bytes) per pass
            uint4 w[4];
#pragma unroll
            for (int v = 0; v < 4; ++v) {
              const uint32_t* oo = o + 32 * hh + 8 * v;
              w[v].x = pack_bf16x2(__uint_as_float(oo[0]) * inv, __uint_as_float(oo[1]) * inv);
              w[v].y = pack_bf16x2(__uint_as_float(oo[2]) * inv, __uint_as_float(oo[3]) * inv);
              w[v].z = pack_bf16x2(__uint_as_float(oo[4]) * inv, __uint_as_float(oo[5]) * inv);
              w[v].w = pack_bf16x2(__uint_as_float(oo[6]) * inv, __uint_as_float(oo[7]) * inv);
            }
            warp_store_rows(stage, w, dst + 64 * hh, qi < p.seq);
          }
        }
        if (qi < p.seq) {
          if (hf == 0) p.lse[(int64_t(x.b) * p.H + x.h) * p.seq + qi] = (m + log2f(lt)) * kLn2f;
        }
      }
    }
  }
  fence_before();
  __syncthreads();
  if (warp == 0) {
    fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem),
                 "r"(kTmemCols)
                 : "memory");
  }
}

// ----------------------------------------------------------------- backward
// The backward as two persistent kernels, no atomics (each output row is
// written once):
//   attn_bwd_dq_tc_kernel   per (query tile, head, sequence): for each key
//       tile j <= the query tile, S = Q K_j^T and dP = dO V_j^T into tensor
//       memory; the softmax warps form P = 2^(S scale log2e - lse log2e)
//       (causal) and dS = P (dP - D) and write dS (bf16 pairs) back into
//       tensor memory, double-buffered; dQ += dS K_j with dS as the
//       tensor-memory A operand and K_j MN-major.  dQ = scale dQ, fp32.
//   attn_bwd_dkv_tc_kernel  per (key block, key/value head, sequence): K
//       and V stay in shared memory; for every query head of the group and
//       64-query tile at or after the block, S^T = K Q^T and dP^T = V dO^T
//       into one of two tensor-memory buffers; the softmax warps (key rows)
//       form P^T and dS^T and write them (bf16 pairs) over the half rows of
//       S^T and dP^T they have read; dV += P^T dO and dK += dS^T Q (Q and
//       dO MN-major).  dK = scale dK (fp32), dV bf16.
struct TcBwdP {
  CUtensorMap mq, mk, mv, mdo;  // Q, dO [T x H 128]; K, V [T x KV 128]; boxes 64 x 128
  CUtensorMap mq64, mdo64;      // Q, dO with boxes of 64 columns x 64 rows
  const float* lse;             // [batch][H][seq], natural log
  const float* D;               // [batch][H][seq], rowsum(dO * O)
  float* dQ;                    // [T x H 128]
  float* dK;                    // [T x KV 128]
  __nv_bfloat16* dV;            // [T x KV 128]
  int seq, H, KV, batch, nqb;
  int items_q, items_k;         // nqb H batch, nqb KV batch
  float sl2, scale;
};

constexpr float kLog2ef = 1.4426950408889634f;

// dQ kernel: Q and dO at 0 and 32 KB, three K stages from 64 KB (a K tile
// stays until its dQ product is done, so its refill needs two tiles of
// lead), two V stages from 160 KB; tensor memory S 0, dP 128, dQ 256, dS at
// 384 and 448.
constexpr int kQKStages = 3;
constexpr int kQOffQ = 0, kQOffO = kTile, kQOffK = 2 * kTile, kQOffV = 5 * kTile;
constexpr int kQOffBar = 7 * kTile;
constexpr int kQSmem = kQOffBar + 256 + 1024;
constexpr uint32_t kColDP = 128, kColDQ = 256, kColDS = 384;

__global__ void __launch_bounds__(kThreadsTc, 1) attn_bwd_dq_tc_kernel(const __grid_constant__ TcBwdP p) {
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  const uint32_t raw = su32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  unsigned char* gbase = smem_raw + (base - raw);
  const uint32_t sQ = base + kQOffQ, sO = base + kQOffO, sK = base + kQOffK, sV = base + kQOffV;
  const uint32_t bar = base + kQOffBar;
  const uint32_t qo_full = bar, qo_empty = bar + 8, v_full = bar + 16, v_empty = bar + 32,
                 s_full = bar + 48, s_free = bar + 56, p_full = bar + 64, dq_done = bar + 80,
                 dq_empty = bar + 96, mma_done = bar + 104, k_full = bar + 112,
                 k_empty = bar + 136;  // K stage of tile t: t % 3
  uint32_t* s_tmem = reinterpret_cast<uint32_t*>(gbase + kQOffBar + 192);
  volatile int* abort = reinterpret_cast<volatile int*>(gbase + kQOffBar + 200);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int G = int(gridDim.x);
  TcFwdP ip;  // item decoding only
  ip.H = p.H; ip.batch = p.batch; ip.nqb = p.nqb;
  if (warp == 0) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     su32(s_tmem)),
                 "r"(kTmemCols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  if (tid == 32) {
    mbar_init(qo_full, 1);
    mbar_init(qo_empty, 1);
    for (int s = 0; s < 2; ++s) {
      mbar_init(v_full + 8 * s, 1);
      mbar_init(v_empty + 8 * s, 1);
      mbar_init(p_full + 8 * s, kSoftWarps);
      mbar_init(dq_done + 8 * s, 1);
    }
    for (int s = 0; s < kQKStages; ++s) {
      mbar_init(k_full + 8 * s, 1);
      mbar_init(k_empty + 8 * s, 1);
    }
    mbar_init(s_full, 1);
    mbar_init(s_free, kSoftWarps);
    mbar_init(dq_empty, kSoftWarps);
    mbar_init(mma_done, 1);
    *abort = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  fence_before();
  __syncthreads();
  fence_after();
  const uint32_t tmem = *s_tmem;

  if (warp == kSoftWarps) {
    // ------------------------------------------------ TMA producer
    if (lane == 0) {
      int t = 0, nq = 0, nk = 0, nv = 0;
      bool ok = true;
      for (int n = 0; ok; ++n) {
        const int it = item_at(n, G);
        if (it >= p.items_q) break;
        const Item x = item_of(ip, it);
        const int row0 = x.b * p.seq, g = x.h / (p.H / p.KV);
        const int yq = row0 + x.qb * kRows;
        if (n >= 1 && !mbar_wait(qo_empty, uint32_t((n - 1) & 1), abort)) break;
        mbar_expect_tx(qo_full, 2 * kTile);
        tma_load(sQ, &p.mq, qo_full, x.h * kHD, yq);
        tma_load(sQ + kPanel, &p.mq, qo_full, x.h * kHD + 64, yq);
        tma_load(sO, &p.mdo, qo_full, x.h * kHD, yq);
        tma_load(sO + kPanel, &p.mdo, qo_full, x.h * kHD + 64, yq);
        nq = n + 1;
        for (int j = 0; j <= x.qb; ++j, ++t) {
          const int s = t & 1, s3 = t % kQKStages;
          const int y = row0 + j * kRows;
          // V_t once dP_{t-2} is done, K_t once dQ += dS_{t-3} K_{t-3} is
          if (t >= 2 && !mbar_wait(v_empty + 8 * s, uint32_t(((t - 2) >> 1) & 1), abort)) {
            ok = false;
            break;
          }
          const uint32_t kb = sK + uint32_t(s3 * kTile), vb = sV + uint32_t(s * kTile);
          mbar_expect_tx(v_full + 8 * s, kTile);
          tma_load(vb, &p.mv, v_full + 8 * s, g * kHD, y);
          tma_load(vb + kPanel, &p.mv, v_full + 8 * s, g * kHD + 64, y);
          nv = t + 1;
          if (t >= kQKStages &&
              !mbar_wait(k_empty + 8 * s3, uint32_t(((t - kQKStages) / kQKStages) & 1), abort)) {
            ok = false;
            break;
          }
          mbar_expect_tx(k_full + 8 * s3, kTile);
          tma_load(kb, &p.mk, k_full + 8 * s3, g * kHD, y);
          tma_load(kb + kPanel, &p.mk, k_full + 8 * s3, g * kHD + 64, y);
          nk = t + 1;
        }
      }
      if (nq >= 1) mbar_drain(qo_full, uint32_t((nq - 1) & 1));
      for (int u = ::max(0, nk - kQKStages); u < nk; ++u)
        mbar_drain(k_full + 8 * (u % kQKStages), uint32_t((u / kQKStages) & 1));
      for (int u = ::max(0, nv - 2); u < nv; ++u)
        mbar_drain(v_full + 8 * (u & 1), uint32_t((u >> 1) & 1));
    }
    __syncwarp();
  } else if (warp == kSoftWarps + 1) {
    // ------------------------------------------------ MMA issuer
    if (lane == 0) {
      bool ok = true;
      int t = 0;
      int pd_t = -1, pd_n = 0;  // the pending dQ += dS K: tile, item ordinal
      bool pd_first = false;
      auto issue_dq = [&]() -> bool {
        const int sp = pd_t & 1;
        if (!mbar_wait(p_full + 8 * sp, uint32_t((pd_t >> 1) & 1), abort)) return false;
        // the first dQ product of an item overwrites the accumulator: the
        // previous item's dQ has been read
        if (pd_first && pd_n >= 1 && !mbar_wait(dq_empty, uint32_t((pd_n - 1) & 1), abort))
          return false;
        fence_after();
        const uint32_t kt = sK + uint32_t((pd_t % kQKStages) * kTile);
        const uint32_t da = tmem + kColDS + uint32_t(sp * 64);
#pragma unroll
        for (int kk = 0; kk < kRows / 16; ++kk)
          mma_ta(tmem + kColDQ, da + uint32_t(kk * 8), sdesc(kt + uint32_t(kk * 2048), kPanel, 1024),
                 idesc(1), (!pd_first || kk > 0) ? 1u : 0u);
        commit(dq_done + 8 * sp);
        commit(k_empty + 8 * (pd_t % kQKStages));
        return true;
      };
      for (int n = 0; ok; ++n) {
        const int it = item_at(n, G);
        if (it >= p.items_q) break;
        const Item x = item_of(ip, it);
        if (pd_t >= 0) {
          if (!issue_dq()) { ok = false; break; }
          pd_t = -1;
        }
        if (!mbar_wait(qo_full, uint32_t(n & 1), abort)) { ok = false; break; }
        for (int j = 0; j <= x.qb; ++j, ++t) {
          const int s = t & 1, s3 = t % kQKStages;
          if (!mbar_wait(k_full + 8 * s3, uint32_t((t / kQKStages) & 1), abort) ||
              !mbar_wait(v_full + 8 * s, uint32_t((t >> 1) & 1), abort) ||
              (t >= 1 && !mbar_wait(s_free, uint32_t((t - 1) & 1), abort))) {
            ok = false;
            break;
          }
          fence_after();
          const uint32_t kt = sK + uint32_t(s3 * kTile), vt = sV + uint32_t(s * kTile);
#pragma unroll
          for (int kk = 0; kk < kHD / 16; ++kk) {
            const uint32_t off = uint32_t((kk >> 2) * kPanel + (kk & 3) * 32);
            mma(tmem, sdesc(sQ + off, 16, 1024), sdesc(kt + off, 16, 1024), idesc(0),
                kk > 0 ? 1u : 0u);
          }
#pragma unroll
          for (int kk = 0; kk < kHD / 16; ++kk) {
            const uint32_t off = uint32_t((kk >> 2) * kPanel + (kk & 3) * 32);
            mma(tmem + kColDP, sdesc(sO + off, 16, 1024), sdesc(vt + off, 16, 1024), idesc(0),
                kk > 0 ? 1u : 0u);
          }
          commit(s_full);
          commit(v_empty + 8 * s);
          if (j == x.qb) commit(qo_empty);
          if (pd_t >= 0 && !issue_dq()) { ok = false; break; }
          pd_t = t;
          pd_n = n;
          pd_first = j == 0;
        }
      }
      if (ok && pd_t >= 0) issue_dq();
      commit(mma_done);
      mbar_drain(mma_done, 0);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------ dS (row r, key half hf)
    const int lq = warp & 3, hf = warp >> 2;
    const int r = lq * 32 + lane;
    const uint32_t lbase = tmem + (uint32_t(lq * 32) << 16);
    bool ok = true;
    int t = 0;
    for (int n = 0;; ++n) {
      const int it = item_at(n, G);
      if (it >= p.items_q) break;
      const Item x = item_of(ip, it);
      const int row0 = x.b * p.seq;
      const int qi = x.qb * kRows + r;
      const bool live = qi < p.seq;
      const int64_t li = (int64_t(x.b) * p.H + x.h) * p.seq + (live ? qi : 0);
      const float nl2 = live ? -p.lse[li] * kLog2ef : 0.f;
      const float drow = live ? p.D[li] : 0.f;
      for (int j = 0; j <= x.qb; ++j, ++t) {
        const int s = t & 1;
        ok = __all_sync(0xffffffffu, ok && mbar_wait(s_full, uint32_t(t & 1), abort));
        if (!ok) continue;
        fence_after();
        uint32_t sv[kHalf], dp[kHalf];
        tld32(lbase + uint32_t(hf * kHalf), sv);
        tld32(lbase + uint32_t(hf * kHalf + 32), sv + 32);
        tld32(lbase + kColDP + uint32_t(hf * kHalf), dp);
        tld32(lbase + kColDP + uint32_t(hf * kHalf + 32), dp + 32);
        tld_wait();
        fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(s_free);
        // keys past this row (causal) carry P = 0; a row past the sequence is all 0
        const int lim = live ? qi - j * kRows - hf * kHalf : -1;
        uint32_t pk[kHalf / 2];
#pragma unroll
        for (int i = 0; i < kHalf / 2; ++i) {
          float p0 = ex2(fmaf(__uint_as_float(sv[2 * i]), p.sl2, nl2));
          float p1 = ex2(fmaf(__uint_as_float(sv[2 * i + 1]), p.sl2, nl2));
          if (2 * i > lim) p0 = 0.f;
          if (2 * i + 1 > lim) p1 = 0.f;
          pk[i] = pack_bf16x2(p0 * (__uint_as_float(dp[2 * i]) - drow),
                              p1 * (__uint_as_float(dp[2 * i + 1]) - drow));
        }
        // dS buffer t % 2 is free once dQ += dS_{t-2} K_{t-2} is done
        if (t >= 2) {
          ok = __all_sync(0xffffffffu,
                          mbar_wait(dq_done + 8 * s, uint32_t(((t - 2) >> 1) & 1), abort));
          if (!ok) continue;
          fence_after();
        }
        tst32(lbase + kColDS + uint32_t(s * 64 + hf * 32), pk);
        tst_wait();
        fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(p_full + 8 * s);
      }
      const int tl = t - 1;
      ok = __all_sync(0xffffffffu, ok && mbar_wait(dq_done + 8 * (tl & 1),
                                                   uint32_t((tl >> 1) & 1), abort));
      if (ok) {
        fence_after();
        uint32_t o[kHalf];
        tld32(lbase + kColDQ + uint32_t(hf * kHalf), o);
        tld32(lbase + kColDQ + uint32_t(hf * kHalf + 32), o + 32);
        tld_wait();
        fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(dq_empty);
        if (live) {
          float4* dst = reinterpret_cast<float4*>(p.dQ + (int64_t(row0) + qi) * (int64_t(p.H) * kHD) +
                                                  x.h * kHD + hf * kHalf);
#pragma unroll
          for (int v = 0; v < kHalf / 4; ++v)
            dst[v] = make_float4(__uint_as_float(o[4 * v]) * p.scale, __uint_as_float(o[4 * v + 1]) * p.scale,
                                 __uint_as_float(o[4 * v + 2]) * p.scale,
                                 __uint_as_float(o[4 * v + 3]) * p.scale);
        }
      }
    }
  }
  fence_before();
  __syncthreads();
  if (warp == 0) {
    fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem),
                 "r"(kTmemCols)
                 : "memory");
  }
}

// dK/dV kernel: K and V at 0 and 32 KB, four (Q, dO) stages of 64 queries
// from 64 KB (Q 16 KB, dO 16 KB); per stage the tile's -lse log2e and D in
// shared vectors.  Tensor memory: S^T buffers at 0 and 64 (64 queries each),
// dP^T buffers at 128 and 192, dV 256, dK 384.  Within a buffer, P^T / dS^T
// of queries 0-31 overwrite columns 0-15 and those of queries 32-63 columns
// 48-63 (each inside the 32 columns its warp has read).  With two buffers the
// next tile's S^T and dP^T run while the softmax warps work on this one.
constexpr int kQT = 64;                    // queries per tile
constexpr int kKStages = 4;
constexpr int kPanel64 = 64 * 128;         // 64 rows x 64 bf16
constexpr int kKStage = 2 * 2 * kPanel64;  // Q and dO of one tile
constexpr int kKOffK = 0, kKOffV = kTile, kKOffQ = 2 * kTile;
constexpr int kKOffBar = 2 * kTile + kKStages * kKStage;
constexpr int kKOffVec = kKOffBar + 256;  // [stage][lse2 | D][64] fp32
constexpr int kKOffSt = kKOffVec + kKStages * 2 * kQT * 4;  // per-warp store staging
constexpr int kKSmem = kKOffSt + 8 * kStageWarp + 1024;
constexpr uint32_t kColDV = 256, kColDK = 384;

// Item `it` of the dK/dV kernel (longest first: key block kb ascending).
struct KItem {
  int kb, g, b;
};
__device__ __forceinline__ KItem kitem_of(const TcBwdP& p, int it) {
  const int gb = p.KV * p.batch;
  KItem x;
  x.kb = it / gb;
  x.g = (it % gb) % p.KV;
  x.b = (it % gb) / p.KV;
  return x;
}
// A-operand column of query block kk (16 queries) in the overwritten halves.
__device__ __forceinline__ uint32_t half_col(int kk) {
  return uint32_t(kk < 2 ? kk * 8 : 48 + (kk - 2) * 8);
}

__global__ void __launch_bounds__(kThreadsTc, 1) attn_bwd_dkv_tc_kernel(const __grid_constant__ TcBwdP p) {
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  const uint32_t raw = su32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  unsigned char* gbase = smem_raw + (base - raw);
  const uint32_t sK = base + kKOffK, sV = base + kKOffV, sQ0 = base + kKOffQ;
  const uint32_t bar = base + kKOffBar;
  const uint32_t kv_full = bar, kv_empty = bar + 8, qo_full = bar + 16, qo_empty = bar + 48,
                 vec_full = bar + 80, st_full = bar + 112, p_full = bar + 128,
                 pv_done = bar + 144, dkv_empty = bar + 160, mma_done = bar + 168;
  uint32_t* s_tmem = reinterpret_cast<uint32_t*>(gbase + kKOffBar + 192);
  volatile int* abort = reinterpret_cast<volatile int*>(gbase + kKOffBar + 200);
  float* vec = reinterpret_cast<float*>(gbase + kKOffVec);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int G = int(gridDim.x);
  const int rep = p.H / p.KV;
  if (warp == 0) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     su32(s_tmem)),
                 "r"(kTmemCols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  if (tid == 32) {
    mbar_init(kv_full, 1);
    mbar_init(kv_empty, 1);
    for (int s = 0; s < kKStages; ++s) {
      mbar_init(qo_full + 8 * s, 1);
      mbar_init(qo_empty + 8 * s, 1);
      mbar_init(vec_full + 8 * s, 32);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(st_full + 8 * s, 1);
      mbar_init(p_full + 8 * s, kSoftWarps);
      mbar_init(pv_done + 8 * s, 1);
    }
    mbar_init(dkv_empty, kSoftWarps);
    mbar_init(mma_done, 1);
    *abort = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  fence_before();
  __syncthreads();
  fence_after();
  const uint32_t tmem = *s_tmem;

  if (warp == kSoftWarps) {
    // ------------------------------------------------ producer warp: lane 0
    // issues the copies, every lane stages the query vectors
    int t = 0, nkv = 0, nqo = 0;
    bool ok = true;
    for (int n = 0; ok; ++n) {
      const int it = item_at(n, G);
      if (it >= p.items_k) break;
      const KItem x = kitem_of(p, it);
      const int row0 = x.b * p.seq, nq2 = 2 * (p.nqb - x.kb);
      ok = __all_sync(0xffffffffu, n == 0 || mbar_wait(kv_empty, uint32_t((n - 1) & 1), abort));
      if (!ok) break;
      if (lane == 0) {
        const int y = row0 + x.kb * kRows;
        mbar_expect_tx(kv_full, 2 * kTile);
        tma_load(sK, &p.mk, kv_full, x.g * kHD, y);
        tma_load(sK + kPanel, &p.mk, kv_full, x.g * kHD + 64, y);
        tma_load(sV, &p.mv, kv_full, x.g * kHD, y);
        tma_load(sV + kPanel, &p.mv, kv_full, x.g * kHD + 64, y);
      }
      nkv = n + 1;
      for (int jj = 0; jj < rep * nq2; ++jj, ++t) {
        const int s4 = t % kKStages;
        const int hq = x.g * rep + jj / nq2, qt = 2 * x.kb + jj % nq2;  // 64-query tile
        ok = __all_sync(0xffffffffu,
                        t < kKStages || mbar_wait(qo_empty + 8 * s4,
                                                  uint32_t(((t - kKStages) / kKStages) & 1), abort));
        if (!ok) break;
        const uint32_t sq = sQ0 + uint32_t(s4 * kKStage), so = sq + 2 * kPanel64;
        const int y = row0 + qt * kQT;
        if (lane == 0) {
          mbar_expect_tx(qo_full + 8 * s4, kKStage);
          tma_load(sq, &p.mq64, qo_full + 8 * s4, hq * kHD, y);
          tma_load(sq + kPanel64, &p.mq64, qo_full + 8 * s4, hq * kHD + 64, y);
          tma_load(so, &p.mdo64, qo_full + 8 * s4, hq * kHD, y);
          tma_load(so + kPanel64, &p.mdo64, qo_full + 8 * s4, hq * kHD + 64, y);
        }
        nqo = t + 1;
        const int64_t l0 = (int64_t(x.b) * p.H + hq) * p.seq;
        float* vl = vec + s4 * 2 * kQT;
#pragma unroll
        for (int c = lane; c < kQT; c += 32) {
          const int q = qt * kQT + c;
          vl[c] = q < p.seq ? -p.lse[l0 + q] * kLog2ef : 0.f;
          vl[kQT + c] = q < p.seq ? p.D[l0 + q] : 0.f;
        }
        mbar_arrive(vec_full + 8 * s4);
      }
    }
    if (lane == 0) {
      if (nkv >= 1) mbar_drain(kv_full, uint32_t((nkv - 1) & 1));
      for (int u = ::max(0, nqo - kKStages); u < nqo; ++u)
        mbar_drain(qo_full + 8 * (u % kKStages), uint32_t((u / kKStages) & 1));
    }
    __syncwarp();
  } else if (warp == kSoftWarps + 1) {
    // ------------------------------------------------ MMA issuer
    if (lane == 0) {
      bool ok = true;
      int t = 0;
      int pv_t = -1, pv_n = 0;  // the pending dV / dK products: tile, item ordinal
      bool pv_first = false;
      auto issue_pv = [&]() -> bool {
        const int bb = pv_t & 1, s4 = pv_t % kKStages;
        if (!mbar_wait(p_full + 8 * bb, uint32_t((pv_t >> 1) & 1), abort)) return false;
        // the first products of an item overwrite dV and dK: the previous item's are read
        if (pv_first && pv_n >= 1 && !mbar_wait(dkv_empty, uint32_t((pv_n - 1) & 1), abort))
          return false;
        fence_after();
        const uint32_t sq = sQ0 + uint32_t(s4 * kKStage), so = sq + 2 * kPanel64;
        const uint32_t ps = tmem + uint32_t(bb * kQT), pd = tmem + 128u + uint32_t(bb * kQT);
        // dV += P^T dO and dK += dS^T Q (dO and Q MN-major: two 64-column atoms)
#pragma unroll
        for (int kk = 0; kk < kQT / 16; ++kk)
          mma_ta(tmem + kColDV, ps + half_col(kk), sdesc(so + uint32_t(kk * 2048), kPanel64, 1024),
                 idesc(1), (!pv_first || kk > 0) ? 1u : 0u);
#pragma unroll
        for (int kk = 0; kk < kQT / 16; ++kk)
          mma_ta(tmem + kColDK, pd + half_col(kk), sdesc(sq + uint32_t(kk * 2048), kPanel64, 1024),
                 idesc(1), (!pv_first || kk > 0) ? 1u : 0u);
        commit(pv_done + 8 * bb);
        commit(qo_empty + 8 * s4);
        return true;
      };
      for (int n = 0; ok; ++n) {
        const int it = item_at(n, G);
        if (it >= p.items_k) break;
        const KItem x = kitem_of(p, it);
        const int ntile = rep * 2 * (p.nqb - x.kb);
        // the previous item's last products first: its epilogue waits on them
        if (pv_t >= 0) {
          if (!issue_pv()) { ok = false; break; }
          pv_t = -1;
        }
        if (!mbar_wait(kv_full, uint32_t(n & 1), abort)) { ok = false; break; }
        for (int jj = 0; jj < ntile; ++jj, ++t) {
          const int bb = t & 1, s4 = t % kKStages;
          const uint32_t sq = sQ0 + uint32_t(s4 * kKStage), so = sq + 2 * kPanel64;
          // S^T / dP^T buffer t % 2 is free once the products of tile t - 2 are done
          if (!mbar_wait(qo_full + 8 * s4, uint32_t((t / kKStages) & 1), abort) ||
              (t >= 2 && !mbar_wait(pv_done + 8 * bb, uint32_t(((t - 2) >> 1) & 1), abort))) {
            ok = false;
            break;
          }
          fence_after();
#pragma unroll
          for (int kk = 0; kk < kHD / 16; ++kk) {
            const uint32_t ok128 = uint32_t((kk >> 2) * kPanel + (kk & 3) * 32);
            const uint32_t ok64 = uint32_t((kk >> 2) * kPanel64 + (kk & 3) * 32);
            mma(tmem + uint32_t(bb * kQT), sdesc(sK + ok128, 16, 1024), sdesc(sq + ok64, 16, 1024),
                idesc(0, kQT), kk > 0 ? 1u : 0u);
          }
#pragma unroll
          for (int kk = 0; kk < kHD / 16; ++kk) {
            const uint32_t ok128 = uint32_t((kk >> 2) * kPanel + (kk & 3) * 32);
            const uint32_t ok64 = uint32_t((kk >> 2) * kPanel64 + (kk & 3) * 32);
            mma(tmem + 128u + uint32_t(bb * kQT), sdesc(sV + ok128, 16, 1024),
                sdesc(so + ok64, 16, 1024), idesc(0, kQT), kk > 0 ? 1u : 0u);
          }
          commit(st_full + 8 * bb);
          if (jj == ntile - 1) commit(kv_empty);  // K and V of this block are read
          if (pv_t >= 0 && !issue_pv()) { ok = false; break; }
          pv_t = t;
          pv_n = n;
          pv_first = jj == 0;
        }
      }
      if (ok && pv_t >= 0) issue_pv();
      commit(mma_done);
      mbar_drain(mma_done, 0);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------ P^T, dS^T (key row r, query half hf)
    const int lq = warp & 3, hf = warp >> 2;
    const int r = lq * 32 + lane;
    const uint32_t lbase = tmem + (uint32_t(lq * 32) << 16);
    const uint32_t ocol = hf ? 48u : 0u;  // where this half's bf16 pairs go
    bool ok = true;
    int t = 0;
    for (int n = 0;; ++n) {
      const int it = item_at(n, G);
      if (it >= p.items_k) break;
      const KItem x = kitem_of(p, it);
      const int nq2 = 2 * (p.nqb - x.kb), ntile = rep * nq2;
      const int key = x.kb * kRows + r;
      for (int jj = 0; jj < ntile; ++jj, ++t) {
        const int bb = t & 1, s4 = t % kKStages;
        const int qt = 2 * x.kb + jj % nq2;
        ok = __all_sync(0xffffffffu,
                        ok && mbar_wait(vec_full + 8 * s4, uint32_t((t / kKStages) & 1), abort) &&
                            mbar_wait(st_full + 8 * bb, uint32_t((t >> 1) & 1), abort));
        if (!ok) continue;
        fence_after();
        const uint32_t cs = lbase + uint32_t(bb * kQT), cd = cs + 128u;
        uint32_t sv[32], dp[32];
        tld32(cs + uint32_t(hf * 32), sv);
        tld32(cd + uint32_t(hf * 32), dp);
        tld_wait();
        // query columns c of this half with key <= query < seq
        const int q0 = qt * kQT + hf * 32;
        const int lo = key - q0, hi = p.seq - q0;  // keep lo <= c < hi
        const float4* vl = reinterpret_cast<const float4*>(vec + s4 * 2 * kQT + hf * 32);
        const float4* vd = reinterpret_cast<const float4*>(vec + s4 * 2 * kQT + kQT + hf * 32);
        uint32_t pp[16], pd[16];
#pragma unroll
        for (int v = 0; v < 8; ++v) {
          const float4 l4 = vl[v], d4 = vd[v];
          const float lv[4] = {l4.x, l4.y, l4.z, l4.w}, dv[4] = {d4.x, d4.y, d4.z, d4.w};
          float pe[4], de[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const int c = 4 * v + e;
            float pv = ex2(fmaf(__uint_as_float(sv[c]), p.sl2, lv[e]));
            if (c < lo || c >= hi) pv = 0.f;
            pe[e] = pv;
            de[e] = pv * (__uint_as_float(dp[c]) - dv[e]);
          }
          pp[2 * v] = pack_bf16x2(pe[0], pe[1]);
          pp[2 * v + 1] = pack_bf16x2(pe[2], pe[3]);
          pd[2 * v] = pack_bf16x2(de[0], de[1]);
          pd[2 * v + 1] = pack_bf16x2(de[2], de[3]);
        }
        tst16(cs + ocol, pp);
        tst16(cd + ocol, pd);
        tst_wait();
        fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(p_full + 8 * bb);
      }
      const int tl = t - 1;
      ok = __all_sync(0xffffffffu, ok && mbar_wait(pv_done + 8 * (tl & 1),
                                                   uint32_t((tl >> 1) & 1), abort));
      if (ok) {
        fence_after();
        uint32_t a[kHalf], c[kHalf];
        tld32(lbase + kColDV + uint32_t(hf * kHalf), a);
        tld32(lbase + kColDV + uint32_t(hf * kHalf + 32), a + 32);
        tld32(lbase + kColDK + uint32_t(hf * kHalf), c);
        tld32(lbase + kColDK + uint32_t(hf * kHalf + 32), c + 32);
        tld_wait();
        fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(dkv_empty);
        const int64_t row = int64_t(x.b) * p.seq + key;
        const int64_t col = int64_t(x.g) * kHD + hf * kHalf;
        char* dvp = reinterpret_cast<char*>(p.dV + row * (int64_t(p.KV) * kHD) + col);
        char* dkp = reinterpret_cast<char*>(p.dK + row * (int64_t(p.KV) * kHD) + col);
        const uint32_t stage = base + uint32_t(kKOffSt + warp * kStageWarp);
        const bool live = key < p.seq;
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {  // dV: 32 bf16 (64 bytes) per pass
          uint4 w[4];
#pragma unroll
          for (int v = 0; v < 4; ++v) {
            const uint32_t* aa = a + 32 * hh + 8 * v;
            w[v].x = pack_bf16x2(__uint_as_float(aa[0]), __uint_as_float(aa[1]));
            w[v].y = pack_bf16x2(__uint_as_float(aa[2]), __uint_as_float(aa[3]));
            w[v].z = pack_bf16x2(__uint_as_float(aa[4]), __uint_as_float(aa[5]));
            w[v].w = pack_bf16x2(__uint_as_float(aa[6]), __uint_as_float(aa[7]));
          }
          warp_store_rows(stage, w, dvp + 64 * hh, live);
        }
#pragma unroll
        for (int qq = 0; qq < 4; ++qq) {  // dK: 16 fp32 (64 bytes) per pass
          uint4 w[4];
#pragma unroll
          for (int v = 0; v < 4; ++v) {
            const uint32_t* cc = c + 16 * qq + 4 * v;
            w[v] = f4bits(__uint_as_float(cc[0]) * p.scale, __uint_as_float(cc[1]) * p.scale,
                          __uint_as_float(cc[2]) * p.scale, __uint_as_float(cc[3]) * p.scale);
          }
          warp_store_rows(stage, w, dkp + 64 * qq, live);
        }
      }
    }
  }
  fence_before();
  __syncthreads();
  if (warp == 0) {
    fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem),
                 "r"(kTmemCols)
                 : "memory");
  }
}

// ----------------------------------------------------------------- host
PFN_cuTensorMapEncodeTiled_v12000 g_enc = nullptr;
std::once_flag g_enc_once;

slora_status encode_rows(CUtensorMap* m, const void* ptr, int64_t rows, int64_t cols,
                         int box_rows = kRows) {
  std::call_once(g_enc_once, [] {
    void* fn = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      g_enc = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
  });
  if (!g_enc) SLORA_FAIL(SLORA_ERR_CUDA, "cuTensorMapEncodeTiled entry point not available");
  cuuint64_t dims[2] = {cuuint64_t(cols), cuuint64_t(rows)};
  cuuint64_t strides[1] = {cuuint64_t(cols) * 2};
  cuuint32_t box[2] = {64, cuuint32_t(box_rows)};
  cuuint32_t es[2] = {1, 1};
  const CUresult r = g_enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(ptr), dims,
                           strides, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE,
                           CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                           CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS)
    SLORA_FAIL(SLORA_ERR_CUDA, "attention: cuTensorMapEncodeTiled failed (%d) rows=%lld cols=%lld",
               int(r), (long long)rows, (long long)cols);
  return SLORA_OK;
}

}  // namespace

bool attention_fwd_tc_ok(const void* Q, const void* K, const void* V, const void* O, int hd) {
  return hd == kHD && aligned16(Q) && aligned16(K) && aligned16(V) && aligned16(O);
}

slora_status attention_fwd_tc_run(const void* Q, const void* K, const void* V, const TokenInfo& ti,
                                  int H, int KV, void* O, float* lse, cudaStream_t st) {
  if (!attention_fwd_tc_ok(Q, K, V, O, kHD))
    SLORA_FAIL(SLORA_ERR_ALIGN, "attention: Q, K, V and O must be 16-byte aligned");
  TcFwdP p;
  SLORA_TRY(encode_rows(&p.mq, Q, ti.T, int64_t(H) * kHD));
  SLORA_TRY(encode_rows(&p.mk, K, ti.T, int64_t(KV) * kHD));
  SLORA_TRY(encode_rows(&p.mv, V, ti.T, int64_t(KV) * kHD));
  p.O = static_cast<__nv_bfloat16*>(O);
  p.lse = lse;
  p.seq = ti.seq; p.H = H; p.KV = KV;
  p.nqb = (ti.seq + kRows - 1) / kRows;
  p.batch = ti.batch;
  p.items = p.nqb * H * ti.batch;
  p.sl2 = float(1.0 / std::sqrt(double(kHD)) * 1.4426950408889634);
  SLORA_CUDA(cudaFuncSetAttribute(attn_fwd_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  kSmem));
  // persistent: one CTA per SM (the shared memory admits no second one)
  const dim3 grid(unsigned(std::min(p.items, num_sms())));
  attn_fwd_tc_kernel<<<grid, kThreadsTc, kSmem, st>>>(p);
  SLORA_CHECK_LAUNCH();
  return SLORA_OK;
}

bool attention_bwd_tc_ok(const void* Q, const void* K, const void* V, const void* dO,
                         const void* dQ, const void* dK, const void* dV, int hd) {
  return hd == kHD && aligned16(Q) && aligned16(K) && aligned16(V) && aligned16(dO) &&
         aligned16(dQ) && aligned16(dK) && aligned16(dV);
}

slora_status attention_bwd_tc_run(const void* Q, const void* K, const void* V, const void* dO,
                                  const float* lse, const float* D, const TokenInfo& ti, int H,
                                  int KV, float* dQ, float* dK, void* dV, double flops_per_product,
                                  cudaStream_t st) {
  if (!attention_bwd_tc_ok(Q, K, V, dO, dQ, dK, dV, kHD))
    SLORA_FAIL(SLORA_ERR_ALIGN, "attention backward: operands must be 16-byte aligned");
  TcBwdP p;
  SLORA_TRY(encode_rows(&p.mq, Q, ti.T, int64_t(H) * kHD));
  SLORA_TRY(encode_rows(&p.mdo, dO, ti.T, int64_t(H) * kHD));
  SLORA_TRY(encode_rows(&p.mk, K, ti.T, int64_t(KV) * kHD));
  SLORA_TRY(encode_rows(&p.mv, V, ti.T, int64_t(KV) * kHD));
  SLORA_TRY(encode_rows(&p.mq64, Q, ti.T, int64_t(H) * kHD, kQT));
  SLORA_TRY(encode_rows(&p.mdo64, dO, ti.T, int64_t(H) * kHD, kQT));
  p.lse = lse; p.D = D; p.dQ = dQ; p.dK = dK;
  p.dV = static_cast<__nv_bfloat16*>(dV);
  p.seq = ti.seq; p.H = H; p.KV = KV; p.batch = ti.batch;
  p.nqb = (ti.seq + kRows - 1) / kRows;
  p.items_q = p.nqb * H * ti.batch;
  p.items_k = p.nqb * KV * ti.batch;
  p.scale = float(1.0 / std::sqrt(double(kHD)));
  p.sl2 = float(double(p.scale) * 1.4426950408889634);
  {
    // algorithmic work: S^T, dP^T, dV, dK (the dQ launch books dQ alone; its
    // S and dP are recomputed)
    LaunchScope ls(kAttention, 4.0 * flops_per_product, st);
    SLORA_CUDA(cudaFuncSetAttribute(attn_bwd_dkv_tc_kernel,
                                    cudaFuncAttributeMaxDynamicSharedMemorySize, kKSmem));
    attn_bwd_dkv_tc_kernel<<<unsigned(std::min(p.items_k, num_sms())), kThreadsTc, kKSmem, st>>>(p);
    SLORA_CHECK_LAUNCH();
  }
  {
    LaunchScope ls(kAttention, 1.0 * flops_per_product, st);
    SLORA_CUDA(cudaFuncSetAttribute(attn_bwd_dq_tc_kernel,
                                    cudaFuncAttributeMaxDynamicSharedMemorySize, kQSmem));
    attn_bwd_dq_tc_kernel<<<unsigned(std::min(p.items_q, num_sms())), kThreadsTc, kQSmem, st>>>(p);
    SLORA_CHECK_LAUNCH();
  }
  return SLORA_OK;
}

slora_status attn_check_error(bool clear) {
  int v = 0;
  SLORA_CUDA(cudaMemcpyFromSymbol(&v, g_attn_error, sizeof(int)));
  if (clear && v) {
    int z = 0;
    SLORA_CUDA(cudaMemcpyToSymbol(g_attn_error, &z, sizeof(int)));
  }
  if (v) SLORA_FAIL(SLORA_ERR_TIMEOUT, "attention: a tensor-core wait ran out of its budget");
  return SLORA_OK;
}

}  // namespace slora
