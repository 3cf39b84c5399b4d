// SVD sparsity estimator scores and top-k channel selection.
//
// SparseLoRA article, section 2 (SVD sparsity estimator): the frozen weight's
// leading singular factors, computed once offline, give a cheap estimate of a
// layer's output on the current context tokens; section 1 names the channel
// criteria (FFN: L2 norm of a neuron's activity; q/k: QK-norm built from the
// query-key product) and the per-input choice of active channels.
//
// Kernels
//   ffn_score_fma_kernel / ffn_score_mma_kernel  activation-norm score of
//       the SwiGLU channels: the rank-r dot products g_hat = P_g U_g^T,
//       u_hat = P_u U_u^T on the FMA pipe as packed f32x2 pairs (r <= 16) or
//       on the tensor cores (mma.sync, both fp32 operands split into three
//       bf16 terms, the six significant cross products packed along K; larger
//       r), the silu and the square-sum on the CUDA cores / MUFU.  Partial
//       sums per (token split, channel); the last split of a channel block to
//       arrive sums them in a fixed order (fp64).
//   gram_partial_kernel      r x r Gram matrices of P over token chunks, fp64;
//       the last chunk to arrive sums them in a fixed order.
//   norm_score_kernel        per-channel norms as Gram quadratic forms
//       ||Y_hat[:, c]||^2 = u_c^T (P^T P) u_c, combined per criterion (QK-norm
//       product with grouped query heads, plain L2 norm, rotate-half pairs).
//   topk_kernel              top-k per group, one block per group.
// Top-k (block_topk): the scores' fp32 bit patterns are the keys (scores are
// non-negative, so unsigned order is numeric order), held in registers; radix
// passes over the bits below the keys' common prefix find the k-th largest
// key; ties at it go to the lower index and the indices are written in
// ascending order (each thread owns a contiguous index range).
#include <cuda_bf16.h>

#include <algorithm>

#include "estimator.cuh"

namespace slora {

// Raised (instead of faulting) when a score kernel finds its shared staging
// buffer off its 16-byte alignment; reported by est_check_error.
__device__ int g_est_error = 0;

namespace {

// ------------------------------------------------------------------ helpers
__device__ __forceinline__ uint32_t score_key(float v) {
  uint32_t b = __float_as_uint(v);
  if (b & 0x80000000u) b = 0;  // -0 (or a negative) ranks as zero
  if (b > 0x7f800000u) b = 0;  // NaN ranks lowest
  return b;
}

__device__ __forceinline__ void mma_bf16(float* d, const uint32_t* a, uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
      "{%8,%9}, {%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// v = h + m + l with h, m, l bf16 (nearest each); the residuals are exact in
// fp32, so the three terms carry v to ~2^-24 relative.
struct Split3 {
  __nv_bfloat16 t[3];
};
__device__ __forceinline__ Split3 split3(float v) {
  Split3 s;
  s.t[0] = __float2bfloat16_rn(v);
  float r = v - __bfloat162float(s.t[0]);
  s.t[1] = __float2bfloat16_rn(r);
  r -= __bfloat162float(s.t[1]);
  s.t[2] = __float2bfloat16_rn(r);
  return s;
}
__device__ __forceinline__ uint32_t pack2(__nv_bfloat16 lo, __nv_bfloat16 hi) {
  return uint32_t(__bfloat16_as_ushort(lo)) | (uint32_t(__bfloat16_as_ushort(hi)) << 16);
}

// ------------------------------------------------------------ block reductions
// The top-k's shared memory is touched only through these scalar 32-bit
// accesses on shared-window addresses (explicit ld/st/red.shared.u32, so every
// access keeps its own 4-byte width and order).
__device__ __forceinline__ uint32_t sh_addr(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}
__device__ __forceinline__ void sh_st(uint32_t a, uint32_t v) {
  asm volatile("st.shared.u32 [%0], %1;" ::"r"(a), "r"(v) : "memory");
}
__device__ __forceinline__ uint32_t sh_ld(uint32_t a) {
  uint32_t v;
  asm volatile("ld.shared.u32 %0, [%1];" : "=r"(v) : "r"(a) : "memory");
  return v;
}
__device__ __forceinline__ void sh_add(uint32_t a, uint32_t v) {
  asm volatile("red.shared.add.u32 [%0], %1;" ::"r"(a), "r"(v) : "memory");
}

// Block-wide reductions and scan over B threads.  `s` is the shared address
// of 2 x B/32 words, double-buffered by `parity` so each call needs one
// barrier.
template <int B>
struct BlockRed {
  static constexpr int NW = B / 32;
  uint32_t s;
  int parity = 0;
  __device__ uint32_t slot(int i) const { return s + 4u * uint32_t(parity * NW + i); }
  __device__ uint32_t min(uint32_t v) {
    const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
    v = __reduce_min_sync(0xffffffffu, v);
    if (lane == 0) sh_st(slot(w), v);
    __syncthreads();
    uint32_t t = 0xffffffffu;
    for (int i = 0; i < NW; ++i) t = ::min(t, sh_ld(slot(i)));
    parity ^= 1;
    return t;
  }
  __device__ uint32_t max(uint32_t v) {
    const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
    v = __reduce_max_sync(0xffffffffu, v);
    if (lane == 0) sh_st(slot(w), v);
    __syncthreads();
    uint32_t t = 0;
    for (int i = 0; i < NW; ++i) t = ::max(t, sh_ld(slot(i)));
    parity ^= 1;
    return t;
  }
  // exclusive prefix sum in thread order
  __device__ uint32_t excl_scan(uint32_t v) {
    const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
    uint32_t inc = v;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const uint32_t up = __shfl_up_sync(0xffffffffu, inc, off);
      if (lane >= off) inc += up;
    }
    if (lane == 31) sh_st(slot(w), inc);
    __syncthreads();
    uint32_t base = 0;
    for (int i = 0; i < w; ++i) base += sh_ld(slot(i));
    parity ^= 1;
    return base + inc - v;
  }
};

// Where a group's selection goes.  The group's kept local channels S (an
// ascending list of k entries; with pairs, kp pairs p giving channels p and
// p + half, listed as all p then all p + half) are written as
//   a[(g*rep + j) * k + i] = (g*rep + j) * N + S[i]   for j < rep,
//   b[g * k + i]           = g * N + S[i]              (if b != null).
struct TopkOut {
  int32_t* a = nullptr;
  int32_t* b = nullptr;
  int rep = 1;
  int N = 0;         // channels of one head (stride of the head offsets)
  int pair_half = 0; // > 0: keys are rotate-half pairs (p, p + pair_half)
};

// The output fields travel as plain scalar arguments (registers): read
// through a struct, every index stored paid a slow reload of the fields.
// ONE: a single index list (rep 1, no b, no pairs), written directly.
template <bool ONE>
__device__ __forceinline__ void topk_emit(int32_t* __restrict__ oa, int32_t* __restrict__ ob,
                                          int rep, int hN, int ph, int g, int ktot, int kp,
                                          int pos, int c) {
  if constexpr (ONE) {
    oa[pos] = c;
  } else {
    for (int j = 0; j < rep; ++j) {
      const int h = g * rep + j;
      int32_t* row = oa + int64_t(h) * ktot;
      row[pos] = h * hN + c;
      if (ph) row[kp + pos] = h * hN + c + ph;
    }
    if (ob) {
      int32_t* row = ob + int64_t(g) * ktot;
      row[pos] = g * hN + c;
      if (ph) row[kp + pos] = g * hN + c + ph;
    }
  }
}

__device__ __forceinline__ uint32_t sh_atom_add(uint32_t a, uint32_t v) {
  uint32_t old;
  asm volatile("atom.shared.add.u32 %0, [%1], %2;" : "=r"(old) : "r"(a), "r"(v) : "memory");
  return old;
}
__device__ __forceinline__ uint32_t lanemask_lt() {
  uint32_t m;
  asm("mov.u32 %0, %%lanemask_lt;" : "=r"(m));
  return m;
}

// Radix digits of 11 bits: one shared 2048-bin histogram per pass.
constexpr int kTopkBins = 2048;
// Keys of the wanted key's bin that warp 0 finishes in registers (8 a lane).
constexpr int kCandMax = 256;

// Shared words of block_topk<B, MAXM> (see the kernel's arrays).
constexpr int topk_hist_words() { return kTopkBins; }
template <int B, int MAXM>
constexpr int topk_tab_words() { return MAXM * (B / 32); }
constexpr int topk_cand_words() { return kCandMax; }

// The k largest of n scores (ties to the lower index), written through the
// output fields for group g.  All B threads of the block call it;
// n <= B * MAXM.  Key j (the score's fp32 bits) sits in row i = j / B of
// thread j % B, so every global access of a row is one coalesced line.
//   1. the keys share their bits above hb, the highest bit where the largest
//      and the smallest key differ; a radix pass counts, in one shared
//      2048-bin histogram, the 11 bits below the prefix fixed so far, and a
//      descending block scan of the bins finds the digit holding the wanted
//      rank; the keys in higher digits are all kept (`above`) and the search
//      goes on inside the digit;
//   2. once the digit holds at most kCandMax keys they are compacted into
//      shared memory, and warp 0 takes them into registers and finds the
//      wanted key by bisection over the remaining bits;
//   3. tau is the k-th largest key: every key above it is kept, and of the
//      keys equal to it the first ones in index order.  Each (row, warp)
//      counts its keys above / equal to tau by ballot; one block scan over
//      that table, in index order, gives every kept key its output position.
// Shared memory (32-bit shared-window addresses): `red` 2 x B/32 words,
// `hist` topk_hist_words, `cand` topk_cand_words, `tab` topk_tab_words,
// `bc` 8 broadcast words.
template <int B, int MAXM, bool ONE>
__device__ void block_topk(const float* __restrict__ sc, int n, int k, int32_t* __restrict__ oa,
                           int32_t* __restrict__ ob, int rep, int hN, int ph, int g,
                           uint32_t red_smem, uint32_t hist, uint32_t cand, uint32_t tab,
                           uint32_t bc) {
  constexpr int NW = B / 32;
  constexpr int CPL = kCandMax / 32;  // candidates per lane of warp 0
  constexpr int BPT = kTopkBins / B;  // histogram bins per thread in the scan
  BlockRed<B> red{red_smem};
  const int tid = threadIdx.x, lane = tid & 31, w = tid >> 5;
  const int kp = k;
  const int ktot = ph ? 2 * k : k;
  if (k <= 0 || n <= 0) return;
  const int rows = (n + B - 1) / B;
  if (k >= n) {  // everything is kept
    for (int i = 0; i < rows; ++i)
      if (i * B + tid < n)
        topk_emit<ONE>(oa, ob, rep, hN, ph, g, ktot, kp, i * B + tid, i * B + tid);
    return;
  }
  if (tid == 0) sh_st(bc + 8u, 0u);  // candidate count (ordered by the barriers below)
  uint32_t key[MAXM];
  uint32_t kmin = 0xffffffffu, kmax = 0u;
#pragma unroll
  for (int i = 0; i < MAXM; ++i) {
    const int j = i * B + tid;
    key[i] = 0u;
    if (i < rows && j < n) {
      key[i] = score_key(__ldcg(sc + j));
      kmin = ::min(kmin, key[i]);
      kmax = ::max(kmax, key[i]);
    }
  }
  kmin = red.min(kmin);
  kmax = red.max(kmax);
  // tau: the k-th largest key; above: how many keys exceed it
  uint32_t tau = kmin, above = 0;
  if (kmin != kmax) {
    int top = 31 - __clz(int(kmin ^ kmax));  // <= 30: keys are below 2^31
    uint32_t prefix = kmin & ~((2u << top) - 1u);
    uint32_t need = uint32_t(k);  // rank of tau among the keys matching prefix
    while (true) {
      const int shift = top > 10 ? top - 10 : 0;
      const uint32_t dmask = (2u << (top - shift)) - 1u;  // digit = bits top .. shift
      const uint32_t pmask = ~((2u << top) - 1u);         // bits above top
      for (int i = tid; i < kTopkBins; i += B) sh_st(hist + 4u * uint32_t(i), 0u);
      __syncthreads();
#pragma unroll
      for (int i = 0; i < MAXM; ++i)
        if (i < rows && i * B + tid < n && (key[i] & pmask) == prefix)
          sh_add(hist + 4u * ((key[i] >> shift) & dmask), 1u);
      __syncthreads();
      // thread t owns bins [2048 - BPT (t + 1), 2048 - BPT t): thread order is
      // descending digit order, so the exclusive scan counts the higher digits
      const int b_top = kTopkBins - 1 - BPT * tid;
      uint32_t own = 0;
      for (int i = 0; i < BPT; ++i) own += sh_ld(hist + 4u * uint32_t(b_top - i));
      const uint32_t higher_t = red.excl_scan(own);
      if (higher_t < need && higher_t + own >= need) {
        uint32_t cum = higher_t;
        for (int i = 0; i < BPT; ++i) {
          const uint32_t h = sh_ld(hist + 4u * uint32_t(b_top - i));
          if (cum + h >= need) {
            sh_st(bc, uint32_t(b_top - i));
            sh_st(bc + 4u, cum);  // keys of this prefix in higher digits
            sh_st(bc + 12u, h);   // keys in the digit
            break;
          }
          cum += h;
        }
      }
      __syncthreads();
      const uint32_t dstar = sh_ld(bc), higher = sh_ld(bc + 4u), nbin = sh_ld(bc + 12u);
      above += higher;
      need -= higher;
      prefix |= dstar << shift;
      if (shift == 0) {
        tau = prefix;
        break;
      }
      top = shift - 1;
      if (nbin <= uint32_t(kCandMax)) {
        // compact the digit's keys (one shared atomic per warp for its base)
        const uint32_t pm = ~((2u << top) - 1u);
        uint32_t mine = 0;
#pragma unroll
        for (int i = 0; i < MAXM; ++i)
          if (i < rows && i * B + tid < n && (key[i] & pm) == prefix) ++mine;
        uint32_t incl = mine;
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
          const uint32_t x = __shfl_up_sync(0xffffffffu, incl, off);
          if (lane >= off) incl += x;
        }
        uint32_t base = 0;
        if (lane == 31) base = sh_atom_add(bc + 8u, incl);
        uint32_t pos = __shfl_sync(0xffffffffu, base, 31) + incl - mine;
#pragma unroll
        for (int i = 0; i < MAXM; ++i)
          if (i < rows && i * B + tid < n && (key[i] & pm) == prefix)
            sh_st(cand + 4u * pos++, key[i]);
        __syncthreads();
        if (w == 0) {
          // bisection over the remaining bits top .. 0 with the candidates in
          // registers; the padding (0) never reaches a threshold above the
          // prefix
          uint32_t ck[CPL];
#pragma unroll
          for (int q = 0; q < CPL; ++q) {
            const uint32_t idx = uint32_t(q * 32 + lane);
            ck[q] = idx < nbin ? sh_ld(cand + 4u * idx) : 0u;
          }
          uint32_t lo = prefix, hi = prefix + (2u << top);
          while (hi - lo > 1u) {
            const uint32_t mid = lo + (hi - lo) / 2u;
            uint32_t c0 = 0, c1 = 0;
#pragma unroll
            for (int q = 0; q < CPL; q += 2) {
              c0 += ck[q] >= mid ? 1u : 0u;
              c1 += ck[q + 1] >= mid ? 1u : 0u;
            }
            const uint32_t c = __reduce_add_sync(0xffffffffu, c0 + c1);
            if (c == need) {  // the wanted keys are exactly those >= mid
              uint32_t mn = 0xffffffffu;
#pragma unroll
              for (int q = 0; q < CPL; ++q)
                if (ck[q] >= mid) mn = ::min(mn, ck[q]);
              lo = __reduce_min_sync(0xffffffffu, mn);
              break;
            }
            if (c > need) lo = mid; else hi = mid;
          }
          uint32_t gt = 0;
#pragma unroll
          for (int q = 0; q < CPL; ++q) gt += ck[q] > lo ? 1u : 0u;
          gt = __reduce_add_sync(0xffffffffu, gt);
          if (lane == 0) {
            sh_st(bc + 16u, lo);
            sh_st(bc + 20u, gt);
          }
        }
        __syncthreads();
        tau = sh_ld(bc + 16u);
        above += sh_ld(bc + 20u);
        break;
      }
    }
  }
  // output positions in index order: per (row, warp) the counts of keys above
  // tau (high half) and equal to it (low half), kept by the lane whose index
  // is the row; n <= 2^15 keeps both halves apart through the scan
  static_assert(MAXM <= 64, "two table words per lane");
  const uint32_t want = uint32_t(k) - above;  // keys equal to tau that are kept
  unsigned long long fgt = 0ull, feq = 0ull;
  uint32_t row_lo = 0, row_hi = 0;  // rows lane and lane + 32
#pragma unroll
  for (int i = 0; i < MAXM; ++i) {
    if (i < rows) {
      const int j = i * B + tid;
      const bool gt = j < n && key[i] > tau, eq = j < n && key[i] == tau;
      const uint32_t bg = __ballot_sync(0xffffffffu, gt), be = __ballot_sync(0xffffffffu, eq);
      if (gt) fgt |= 1ull << i;
      if (eq) feq |= 1ull << i;
      const uint32_t cnt = (uint32_t(__popc(bg)) << 16) | uint32_t(__popc(be));
      if (i < 32) row_lo = lane == i ? cnt : row_lo;
      else row_hi = lane == i - 32 ? cnt : row_hi;
    }
  }
  if (lane < rows) sh_st(tab + 4u * uint32_t(lane * NW + w), row_lo);
  if (MAXM > 32 && lane + 32 < rows) sh_st(tab + 4u * uint32_t((lane + 32) * NW + w), row_hi);
  __syncthreads();
  {
    constexpr int EPT = (MAXM * NW + B - 1) / B;  // table entries per thread
    const int ne = rows * NW;
    uint32_t v[EPT], sum = 0;
#pragma unroll
    for (int q = 0; q < EPT; ++q) {
      const int e = tid * EPT + q;
      v[q] = e < ne ? sh_ld(tab + 4u * uint32_t(e)) : 0u;
      sum += v[q];
    }
    uint32_t run = red.excl_scan(sum);
#pragma unroll
    for (int q = 0; q < EPT; ++q) {
      const int e = tid * EPT + q;
      if (e < ne) sh_st(tab + 4u * uint32_t(e), run);
      run += v[q];
    }
  }
  __syncthreads();
  const uint32_t pre_lo = lane < rows ? sh_ld(tab + 4u * uint32_t(lane * NW + w)) : 0u;
  const uint32_t pre_hi =
      MAXM > 32 && lane + 32 < rows ? sh_ld(tab + 4u * uint32_t((lane + 32) * NW + w)) : 0u;
  const uint32_t lt = lanemask_lt();
  // a rolled loop: unrolled over every row, the general emission's code
  // outgrew the instruction cache
#pragma unroll 1
  for (int i = 0; i < rows; ++i) {
    const bool gt = (fgt >> i) & 1ull, eq = (feq >> i) & 1ull;
    const uint32_t bg = __ballot_sync(0xffffffffu, gt), be = __ballot_sync(0xffffffffu, eq);
    const uint32_t pre = __shfl_sync(0xffffffffu, i < 32 ? pre_lo : pre_hi, i & 31);
    const uint32_t gtb = (pre >> 16) + uint32_t(__popc(bg & lt));
    const uint32_t eqb = (pre & 0xffffu) + uint32_t(__popc(be & lt));
    if (gt || (eq && eqb < want))
      topk_emit<ONE>(oa, ob, rep, hN, ph, g, ktot, kp, int(gtb + ::min(eqb, want)), i * B + tid);
  }
}

// ---------------------------------------------------------------- FFN score
// Six cross products of the three-term splits P = Ph + Pm + Pl and
// U = Uh + Um + Ul carry the dot product to ~2^-23 relative: (h,h), (h,m),
// (m,h), (h,l), (l,h), (m,m).  For rank chunk ch (8 rank indices) the product
// list gives 6 "units" of K = 8; unit u = product u / C at chunk u % C, and
// K16 block kb of the mma packs units 2 kb (k 0..7) and 2 kb + 1 (k 8..15).
constexpr int pterm(int p) { return p == 2 ? 1 : (p == 4 ? 2 : (p == 5 ? 1 : 0)); }
constexpr int uterm(int p) { return p == 1 ? 1 : (p == 3 ? 2 : (p == 5 ? 1 : 0)); }

constexpr int kScoreThreads = 256;
constexpr int kScoreWarps = kScoreThreads / 32;
constexpr int kStageTokens = 128;  // tokens staged per round (multiple of 16)
// n8 tiles per warp for rank chunks C
constexpr int score_nt(int C) { return C == 1 ? 2 : 1; }
// 32-bit words per staged token: 2 matrices x 3 terms x 4C words, padded to
// a stride = 4 (mod 8) words so the fragment loads of a warp are
// bank-conflict free
constexpr int score_tw(int C) { return 24 * C + 4; }
constexpr int score_stage_bytes(int C) { return kStageTokens * score_tw(C) * 4; }

struct ScoreArgs {
  const float* P;        // [rows x ldp] fp32: P_g in columns [0, r), P_u in [r, 2r)
  int64_t ldp;
  const int32_t* pmap;   // context token t -> row of P (null: identity)
  int64_t T_C;
  const float* Ug;       // [n x r]
  const float* Uu;
  int64_t n;
  int r;
  int nsplit;
  int64_t chunk;         // tokens per split (multiple of 16)
  float* partial;        // [nsplit x n]
  float* scores;         // [n]
  unsigned* counters;    // [nblocks], zero on entry
  const uint4* psplit;   // tensor-core kernel: split P rows per 64-token tile (16 KB each)
};

// Common end of the score kernels: the last split of a channel block to
// arrive sums the block's partials in split order (fp64) and writes its
// scores.  `s_last` is one word of the kernel's shared memory.
template <int CH>
__device__ void score_tail(const ScoreArgs& a, int64_t cb, unsigned* s_last) {
  const int tid = threadIdx.x;
  __syncthreads();  // the block's partials before thread 0's (cumulative) fence
  if (tid == 0) {
    __threadfence();
    *s_last = (atomicAdd(&a.counters[cb], 1u) + 1u == unsigned(a.nsplit)) ? 1u : 0u;
  }
  __syncthreads();
  if (!*s_last) return;
  __threadfence();
  for (int c = tid; c < CH; c += kScoreThreads) {
    const int64_t j = cb * CH + c;
    if (j >= a.n) break;
    double sum = 0.0;
    for (int p = 0; p < a.nsplit; ++p) sum += double(__ldcg(a.partial + int64_t(p) * a.n + j));
    a.scores[j] = float(sqrt(sum));
  }
}

// ---- packed-FMA score kernel (rank <= 16)
// Thread t owns NPAIR pairs of adjacent channels (j, j + 1) and keeps their
// rows of U_g and U_u in registers as f32x2 pairs; each context token's
// projected row (P_g | P_u) is staged once per block in shared memory with
// every value duplicated ({v, v}), so one fma.rn.f32x2 advances the dot
// products of both channels of a pair.  The silu tail runs on the pairs too
// (exp and reciprocal stay scalar on the MUFU unit).  Legacy mma.sync issues
// at a small fraction of the FMA pipe's rate on this GPU, so at rank <= 16
// the dot products are cheaper on the FMA pipe.
__device__ __forceinline__ unsigned long long pack_f2(float lo, float hi) {
  unsigned long long v;
  asm("mov.b64 %0, {%1, %2};" : "=l"(v) : "f"(lo), "f"(hi));
  return v;
}
__device__ __forceinline__ float2 unpack_f2(unsigned long long v) {
  float2 f;
  asm("mov.b64 {%0, %1}, %2;" : "=f"(f.x), "=f"(f.y) : "l"(v));
  return f;
}
__device__ __forceinline__ unsigned long long ffma2(unsigned long long a, unsigned long long b,
                                                    unsigned long long c) {
  unsigned long long d;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
  return d;
}
__device__ __forceinline__ unsigned long long fmul2(unsigned long long a, unsigned long long b) {
  unsigned long long d;
  asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}
__device__ __forceinline__ unsigned long long fadd2(unsigned long long a, unsigned long long b) {
  unsigned long long d;
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}
__device__ __forceinline__ float ex2_approx(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}
__device__ __forceinline__ float rcp_approx(float x) {
  float y;
  asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

constexpr int kFmaTokens = 64;  // tokens staged per round
// One channel pair per thread (its U rows in registers); resident blocks per
// SM by rank (the rank-16 rows take twice the registers).
template <int RP>
constexpr int fma_npair() { return 1; }
template <int RP>
constexpr int fma_channels() { return kScoreThreads * 2 * fma_npair<RP>(); }
template <int RP>
constexpr int fma_min_blocks() { return RP <= 8 ? 3 : 2; }

// silu(g) u = g u / (1 + e^-g).  With g' = -g log2(e) and u' = -u ln(2)
// (the constants folded into the thread's U rows once), g u = g' u', and
// e^-g = 2^g', so each (token, channel) takes one ex2, one add, one
// reciprocal and two multiplies.
template <int RP>
__global__ void __launch_bounds__(kScoreThreads, fma_min_blocks<RP>())
    ffn_score_fma_kernel(const __grid_constant__ ScoreArgs a) {
  constexpr int NP = fma_npair<RP>(), CH = fma_channels<RP>();
  __shared__ __align__(16) unsigned long long sp[kFmaTokens][2 * RP];  // {v, v} pairs
  __shared__ unsigned s_last;
  const int tid = threadIdx.x;
  const int64_t cb = blockIdx.x;
  const int sp_id = blockIdx.y;
  const int r = a.r;
  if (reinterpret_cast<uintptr_t>(&sp[0][0]) & 15u) {  // the 16-byte loads below need it
    if (tid == 0) atomicExch(&g_est_error, 1);
    return;
  }
  // this thread's channel pairs: j = cb*CH + 2*(tid + kScoreThreads*p) + {0, 1}
  constexpr float kNegLog2e = -1.4426950408889634f, kNegLn2 = -0.6931471805599453f;
  unsigned long long ug[NP][RP], uu[NP][RP], acc[NP];
#pragma unroll
  for (int p = 0; p < NP; ++p) {
    const int64_t j = cb * CH + 2 * (tid + kScoreThreads * p);
#pragma unroll
    for (int q = 0; q < RP; ++q) {
      const bool ok = q < r;
      const float g0 = (ok && j < a.n) ? a.Ug[j * r + q] : 0.0f;
      const float g1 = (ok && j + 1 < a.n) ? a.Ug[(j + 1) * r + q] : 0.0f;
      const float u0 = (ok && j < a.n) ? a.Uu[j * r + q] : 0.0f;
      const float u1 = (ok && j + 1 < a.n) ? a.Uu[(j + 1) * r + q] : 0.0f;
      ug[p][q] = pack_f2(g0 * kNegLog2e, g1 * kNegLog2e);
      uu[p][q] = pack_f2(u0 * kNegLn2, u1 * kNegLn2);
    }
    acc[p] = 0ull;
  }
  const unsigned long long one2 = pack_f2(1.0f, 1.0f);
  const int64_t t0 = int64_t(sp_id) * a.chunk;
  const int64_t t1 = ::min(a.T_C, t0 + a.chunk);
  // the staging's parameters in registers, read once
  const float* __restrict__ P = a.P;
  const int32_t* __restrict__ pmap = a.pmap;
  const int64_t ldp = a.ldp;
  // staging: each thread carries EPT values of a stage's P rows; the next
  // stage's values, and the row indices of the stage after it, are loaded
  // into registers while the current one is computed (so no P load waits on
  // its row index).  Rows past the last token are zero (g' = 0 gives v = 0).
  constexpr int EPT = kFmaTokens * 2 * RP / kScoreThreads;
  const uint32_t sp0 = sh_addr(&sp[0][0]);
  float pf[EPT];
  int32_t prow[EPT];  // rows of P for the stage loaded next (-1: past the end)
  auto load_rows = [&](int64_t tb) {
#pragma unroll
    for (int e = 0; e < EPT; ++e) {
      const int tt = (tid + e * kScoreThreads) / (2 * RP);
      prow[e] = tb + tt < t1 ? (pmap ? pmap[tb + tt] : int32_t(tb + tt)) : -1;
    }
  };
  auto load_vals = [&]() {
#pragma unroll
    for (int e = 0; e < EPT; ++e) {
      const int q = (tid + e * kScoreThreads) % (2 * RP), mat = q / RP, qq = q % RP;
      pf[e] = (qq < r && prow[e] >= 0) ? P[int64_t(prow[e]) * ldp + mat * r + qq] : 0.0f;
    }
  };
  // g' and u' of one channel pair for the token row at shared address `row`
  auto dots = [&](uint32_t row, int p, unsigned long long& g2, unsigned long long& u2) {
    g2 = u2 = 0ull;
#pragma unroll
    for (int q2 = 0; q2 < RP / 2; ++q2) {
      unsigned long long px, py;
      asm volatile("ld.shared.v2.u64 {%0, %1}, [%2];" : "=l"(px), "=l"(py) : "r"(row + 16u * q2));
      g2 = ffma2(px, ug[p][2 * q2], g2);
      g2 = ffma2(py, ug[p][2 * q2 + 1], g2);
    }
#pragma unroll
    for (int q2 = 0; q2 < RP / 2; ++q2) {
      unsigned long long px, py;
      asm volatile("ld.shared.v2.u64 {%0, %1}, [%2];"
                   : "=l"(px), "=l"(py)
                   : "r"(row + 16u * (RP / 2 + q2)));
      u2 = ffma2(px, uu[p][2 * q2], u2);
      u2 = ffma2(py, uu[p][2 * q2 + 1], u2);
    }
  };
  auto tail = [&](unsigned long long g2, unsigned long long u2, unsigned long long& ac) {
    const float2 x = unpack_f2(g2);
    const unsigned long long den = fadd2(pack_f2(ex2_approx(x.x), ex2_approx(x.y)), one2);
    const float2 dn = unpack_f2(den);
    const unsigned long long inv = pack_f2(rcp_approx(dn.x), rcp_approx(dn.y));
    const unsigned long long v = fmul2(fmul2(g2, u2), inv);
    ac = ffma2(v, v, ac);
  };
  if (t0 < t1) {
    load_rows(t0);
    load_vals();
    load_rows(t0 + kFmaTokens);
  }
  for (int64_t tb = t0; tb < t1; tb += kFmaTokens) {
    const int nt = int(::min(int64_t(kFmaTokens), t1 - tb));
    __syncthreads();  // the previous stage has been consumed
#pragma unroll
    for (int e = 0; e < EPT; ++e) {
      const uint64_t v = pack_f2(pf[e], pf[e]);
      asm volatile("st.shared.u64 [%0], %1;" ::"r"(sp0 + 8u * uint32_t(tid + e * kScoreThreads)),
                   "l"(v));
    }
    __syncthreads();
    if (tb + kFmaTokens < t1) {
      load_vals();                          // stage s + 1 (its rows are known)
      load_rows(tb + 2 * kFmaTokens);       // rows of stage s + 2
    }
    // rank <= 8: two tokens per step (independent chains; a stage's rows past
    // nt are zero); rank 16: one (its U rows fill the registers)
    constexpr int TPS = RP <= 8 ? 2 : 1;
    for (int tt = 0; tt < nt; tt += TPS) {
      const uint32_t row = sp0 + uint32_t(tt) * (16u * RP);
#pragma unroll
      for (int p = 0; p < NP; ++p) {
        unsigned long long ga, ua;
        dots(row, p, ga, ua);
        if constexpr (TPS == 2) {
          unsigned long long gb, ub;
          dots(row + 16u * RP, p, gb, ub);
          tail(ga, ua, acc[p]);
          tail(gb, ub, acc[p]);
        } else {
          tail(ga, ua, acc[p]);
        }
      }
    }
  }
#pragma unroll
  for (int p = 0; p < NP; ++p) {
    const int64_t j = cb * CH + 2 * (tid + kScoreThreads * p);
    const float2 f = unpack_f2(acc[p]);
    float* dst = a.partial + int64_t(sp_id) * a.n + j;
    if (j < a.n) dst[0] = f.x;
    if (j + 1 < a.n) dst[1] = f.y;
  }
  score_tail<CH>(a, cb, &s_last);
}

template <int C>
__global__ void __launch_bounds__(kScoreThreads)
    ffn_score_mma_kernel(const __grid_constant__ ScoreArgs a) {
  constexpr int NT = score_nt(C), TW = score_tw(C), KB = 3 * C;
  constexpr int CH = kScoreWarps * NT * 8;  // channels per block
  extern __shared__ __align__(16) uint32_t s_stage[];
  __shared__ unsigned s_last;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31, g = lane >> 2, t = lane & 3;
  const int64_t cb = blockIdx.x;
  const int sp = blockIdx.y;
  const int r = a.r;

  // B fragments: channel (tile base + g), rank indices 8 ch + 2t, +1
  uint32_t bfr[NT][2][KB][2];
#pragma unroll
  for (int nt = 0; nt < NT; ++nt) {
    const int64_t j = cb * CH + (warp * NT + nt) * 8 + g;
#pragma unroll
    for (int mat = 0; mat < 2; ++mat) {
      const float* U = mat == 0 ? a.Ug : a.Uu;
      Split3 s0[C], s1[C];
#pragma unroll
      for (int ch = 0; ch < C; ++ch) {
        const int q = 8 * ch + 2 * t;
        const float v0 = (j < a.n && q < r) ? U[j * r + q] : 0.0f;
        const float v1 = (j < a.n && q + 1 < r) ? U[j * r + q + 1] : 0.0f;
        s0[ch] = split3(v0);
        s1[ch] = split3(v1);
      }
#pragma unroll
      for (int kb = 0; kb < KB; ++kb) {
#pragma unroll
        for (int half = 0; half < 2; ++half) {
          const int u = 2 * kb + half, term = uterm(u / C), ch = u % C;
          bfr[nt][mat][kb][half] = pack2(s0[ch].t[term], s1[ch].t[term]);
        }
      }
    }
  }

  float acc[NT][2];
#pragma unroll
  for (int nt = 0; nt < NT; ++nt) acc[nt][0] = acc[nt][1] = 0.0f;

  const int64_t t0 = int64_t(sp) * a.chunk;
  const int64_t t1 = ::min(a.T_C, t0 + a.chunk);
  for (int64_t tb = t0; tb < t1; tb += kStageTokens) {
    const int ntok = int(::min(int64_t(kStageTokens), t1 - tb));
    const int ntile = (ntok + 15) / 16;
    __syncthreads();
    // stage the split terms of the round's P rows: item = (token, matrix, word)
    for (int e = tid; e < ntile * 16 * 8 * C; e += kScoreThreads) {
      const int tt = e / (8 * C), rem = e % (8 * C), mat = rem / (4 * C), w = rem % (4 * C);
      float v0 = 0.0f, v1 = 0.0f;
      if (tt < ntok) {
        const int64_t row = a.pmap ? int64_t(a.pmap[tb + tt]) : tb + tt;
        const float* p = a.P + row * a.ldp + mat * r;
        if (2 * w < r) v0 = p[2 * w];
        if (2 * w + 1 < r) v1 = p[2 * w + 1];
      }
      const Split3 s0 = split3(v0), s1 = split3(v1);
      uint32_t* dst = s_stage + tt * TW + mat * 12 * C + w;
#pragma unroll
      for (int term = 0; term < 3; ++term) dst[term * 4 * C] = pack2(s0.t[term], s1.t[term]);
    }
    __syncthreads();
    for (int tile = 0; tile < ntile; ++tile) {
      const uint32_t* r0 = s_stage + (tile * 16 + g) * TW;
      const uint32_t* r1 = r0 + 8 * TW;
      // A fragment of K16 block kb of matrix mat: tokens g, g + 8; rank
      // indices 8 ch + 2t, +1 of the two units the block packs
      auto load_a = [&](int mat, int kb, uint32_t* f) {
        const int u0 = 2 * kb, u1 = 2 * kb + 1;
        const int o0 = mat * 12 * C + pterm(u0 / C) * 4 * C + 4 * (u0 % C) + t;
        const int o1 = mat * 12 * C + pterm(u1 / C) * 4 * C + 4 * (u1 % C) + t;
        f[0] = r0[o0];
        f[1] = r1[o0];
        f[2] = r0[o1];
        f[3] = r1[o1];
      };
      auto epilogue = [&](const float* cg, const float* cu, float* ac) {
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float v = silu_f(cg[e]) * cu[e];
          ac[e & 1] = fmaf(v, v, ac[e & 1]);
        }
      };
      if constexpr (C <= 2) {  // fragments loaded once per tile, reused by the NT tiles
        uint32_t afr[2][KB][4];
#pragma unroll
        for (int mat = 0; mat < 2; ++mat)
#pragma unroll
          for (int kb = 0; kb < KB; ++kb) load_a(mat, kb, afr[mat][kb]);
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
          float cg[4] = {0.0f, 0.0f, 0.0f, 0.0f}, cu[4] = {0.0f, 0.0f, 0.0f, 0.0f};
#pragma unroll
          for (int kb = 0; kb < KB; ++kb) {
            mma_bf16(cg, afr[0][kb], bfr[nt][0][kb][0], bfr[nt][0][kb][1]);
            mma_bf16(cu, afr[1][kb], bfr[nt][1][kb][0], bfr[nt][1][kb][1]);
          }
          epilogue(cg, cu, acc[nt]);
        }
      } else {  // large rank, one tile per warp: fragments loaded per K16 block
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
          float cg[4] = {0.0f, 0.0f, 0.0f, 0.0f}, cu[4] = {0.0f, 0.0f, 0.0f, 0.0f};
#pragma unroll
          for (int kb = 0; kb < KB; ++kb) {
            uint32_t fa[4], fb[4];
            load_a(0, kb, fa);
            load_a(1, kb, fb);
            mma_bf16(cg, fa, bfr[nt][0][kb][0], bfr[nt][0][kb][1]);
            mma_bf16(cu, fb, bfr[nt][1][kb][0], bfr[nt][1][kb][1]);
          }
          epilogue(cg, cu, acc[nt]);
        }
      }
    }
  }
  // sum over the 8 token rows (lanes with equal t), fixed order
#pragma unroll
  for (int nt = 0; nt < NT; ++nt)
#pragma unroll
    for (int c = 0; c < 2; ++c) {
      float v = acc[nt][c];
      v += __shfl_xor_sync(0xffffffffu, v, 4);
      v += __shfl_xor_sync(0xffffffffu, v, 8);
      v += __shfl_xor_sync(0xffffffffu, v, 16);
      acc[nt][c] = v;
    }
  if (g == 0) {
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
      const int64_t j = cb * CH + (warp * NT + nt) * 8 + 2 * t;
      float* dst = a.partial + int64_t(sp) * a.n + j;
      if (j < a.n) dst[0] = acc[nt][0];
      if (j + 1 < a.n) dst[1] = acc[nt][1];
    }
  }
  score_tail<CH>(a, cb, &s_last);
}

// ---- tensor-core score kernel (rank <= 8)
// The dot products g_hat = P_g U_g^T and u_hat = P_u U_u^T of a 128-channel
// x 64-token tile run on tcgen05 (M = 128 channels, N = 64 tokens, bf16 in,
// fp32 accumulators in tensor memory).  fp32 accuracy comes from three-term
// bf16 splits of both operands: the K dimension (64) holds six blocks of
// `rank` values pairing (U_h, P_h), (U_m, P_h), (U_h, P_m), (U_l, P_h),
// (U_h, P_l), (U_m, P_m), the rest zero.  The constants -log2(e) (gate) and
// -ln(2) (up) are folded into U before the split, so each (token, channel)
// costs one ex2, half a reciprocal (two tokens share one) and a few FMA-pipe
// operations in the epilogue, where 8 warps read the accumulators with
// tcgen05.ld (warp w: the 32 channels of lane quarter w % 4, the 32 tokens
// of half w / 4).  Operands
// are staged by the threads themselves (the split is a transformation) in the
// 128-byte-swizzled K-major layout the MMA descriptors describe.  Software
// pipeline over the block's tiles: while the epilogue of tile i reads its
// accumulators, the MMAs of tile i + 1 run into the other half of the block's
// 256 tensor-memory columns (both operand and accumulator buffers are
// doubled) and the P rows of tile i + 2 are in flight into registers.  Two
// blocks share an SM.
constexpr int kTcTok = 64;            // tokens per tile (MMA N)
constexpr int kTcCh = 128;            // channels per block (MMA M)
constexpr int kTcK = 64;              // padded K (six blocks of <= 8)
constexpr int kTcABytes = kTcCh * kTcK * 2;   // A tile: 128 rows x 64 bf16
constexpr int kTcBBytes = kTcTok * kTcK * 2;  // B tile: 64 rows x 64 bf16
// A_g, A_u, 2 x (B_g, B_u) + alignment + barriers, padded so that at most two
// blocks (2 x 256 tensor-memory columns) are resident per SM
constexpr int kTcSmem = 80 * 1024;
constexpr float kTcNegLog2e = -1.4426950408889634f, kTcNegLn2 = -0.6931471805599453f;
constexpr long long kTcWaitBudget = 2000000000LL;  // clock cycles

__device__ __forceinline__ uint32_t tc_swz(int row, int chunk) {
  return uint32_t(row * 128 + ((chunk ^ (row & 7)) << 4));
}
__device__ __forceinline__ uint64_t tc_sdesc(uint32_t saddr) {
  uint64_t d = 0;
  d |= uint64_t((saddr & 0x3FFFFu) >> 4);
  d |= uint64_t(16 >> 4) << 16;    // leading byte offset (unused with this swizzle)
  d |= uint64_t(1024 >> 4) << 32;  // 8-row group stride
  d |= uint64_t(1) << 46;          // descriptor version
  d |= uint64_t(2) << 61;          // 128-byte swizzle
  return d;
}
// kind::f16, bf16 A and B (K-major), fp32 D, M = 128, N = 64
constexpr uint32_t kTcIdesc = (1u << 4) | (1u << 7) | (1u << 10) | (uint32_t(kTcTok >> 3) << 17) |
                              (uint32_t(kTcCh >> 4) << 24);

// Three-term bf16 split of 8 fp32 values: hi, mid, lo as 16-byte chunks.
__device__ __forceinline__ void split8(const float (&x)[8], uint4& h, uint4& m, uint4& l) {
  __nv_bfloat162* ph = reinterpret_cast<__nv_bfloat162*>(&h);
  __nv_bfloat162* pm = reinterpret_cast<__nv_bfloat162*>(&m);
  __nv_bfloat162* pl = reinterpret_cast<__nv_bfloat162*>(&l);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float a = x[2 * i], b = x[2 * i + 1];
    const __nv_bfloat162 vh = __floats2bfloat162_rn(a, b);
    const float ra = a - __low2float(vh), rb = b - __high2float(vh);
    const __nv_bfloat162 vm = __floats2bfloat162_rn(ra, rb);
    ph[i] = vh;
    pm[i] = vm;
    pl[i] = __floats2bfloat162_rn(ra - __low2float(vm), rb - __high2float(vm));
  }
}
__device__ __forceinline__ void sts16(uint32_t a, uint4 v) {
  asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(a), "r"(v.x), "r"(v.y), "r"(v.z),
               "r"(v.w)
               : "memory");
}
// Row `row` of an operand tile: the six K blocks in the order of `pat` (0 =
// hi, 1 = mid, 2 = lo), then two zero chunks.
__device__ __forceinline__ void stage_split_row(uint32_t tile, int row, const float (&x)[8],
                                                const int (&pat)[6]) {
  uint4 t[3];
  split8(x, t[0], t[1], t[2]);
#pragma unroll
  for (int c = 0; c < 6; ++c) sts16(tile + tc_swz(row, c), t[pat[c]]);
  const uint4 z = make_uint4(0, 0, 0, 0);
  sts16(tile + tc_swz(row, 6), z);
  sts16(tile + tc_swz(row, 7), z);
}
__device__ __forceinline__ bool tc_mbar_wait(uint32_t bar, uint32_t parity) {
  uint32_t ok = 0;
  const long long t0 = clock64();
  while (true) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(bar), "r"(parity)
        : "memory");
    if (ok) return true;
    if (clock64() - t0 > kTcWaitBudget) {
      atomicExch(&g_est_error, 2);
      return false;
    }
  }
}
__device__ __forceinline__ void tc_ld32(uint32_t taddr, uint32_t (&r)[32]) {
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
}
__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

// The split operand rows of every 64-token tile, once for all channel blocks:
// psplit[tile][mat][row] is 128 bytes (the six K blocks of P_mat's row of
// token tile * 64 + row, then zeros) with the 128-byte swizzle applied, so a
// plain bulk copy into a 1024-byte aligned buffer gives the MMA layout.
// Rows past T_C are zero.
__global__ void score_split_p_kernel(const float* __restrict__ P, int64_t ldp,
                                     const int32_t* __restrict__ pmap, int64_t T_C, int r,
                                     int64_t ntiles, uint4* __restrict__ psplit) {
  const int64_t i = int64_t(blockIdx.x) * blockDim.x + threadIdx.x;  // (tile, mat, row)
  if (i >= ntiles * 2 * kTcTok) return;
  const int row = int(i % kTcTok), mat = int((i / kTcTok) % 2);
  const int64_t tile = i / (2 * kTcTok);
  const int64_t t = tile * kTcTok + row;
  float x[8];
  if (t < T_C) {
    const int64_t prow = pmap ? pmap[t] : t;
    const float* src = P + prow * ldp + mat * r;
#pragma unroll
    for (int q = 0; q < 8; ++q) x[q] = q < r ? src[q] : 0.f;
  } else {
#pragma unroll
    for (int q = 0; q < 8; ++q) x[q] = 0.f;
  }
  uint4 t3[3];
  split8(x, t3[0], t3[1], t3[2]);
  constexpr int patB[6] = {0, 0, 1, 0, 2, 1};  // P terms per K block
  uint4* dst = psplit + ((tile * 2 + mat) * kTcTok + row) * 8;
#pragma unroll
  for (int c = 0; c < 8; ++c) dst[c ^ (row & 7)] = c < 6 ? t3[patB[c]] : make_uint4(0, 0, 0, 0);
}

constexpr int kTcEpiWarps = 8;                       // epilogue warps
constexpr int kTcThreads = (kTcEpiWarps + 1) * 32;    // + one producer / MMA warp

__device__ __forceinline__ void tc_arrive(uint32_t bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}

// Warp-specialized: warps 0-7 read the accumulators and run the silu
// epilogue; lane 0 of warp 8 brings each tile's split P rows in by one bulk
// copy and issues the MMAs.  Handoffs through mbarriers only: loaded[b] (the
// rows of the tile in buffer b have landed), full[b] (its MMAs are done:
// tensor memory readable, its operand rows free) and empty[b] (the 8
// epilogue warps have read buffer b's accumulators).
__global__ void __launch_bounds__(kTcThreads, 2)
    ffn_score_tc_kernel(const __grid_constant__ ScoreArgs a) {
  extern __shared__ __align__(1024) unsigned char tc_smem[];
  __shared__ uint32_t s_tmem;
  __shared__ unsigned s_last;
  __shared__ float s_half[kTcCh];
  // 1024-byte aligned operand tiles (the swizzle pattern repeats every 1024 bytes)
  const uint32_t base = (sh_addr(tc_smem) + 1023u) & ~1023u;
  const uint32_t sAg = base, sAu = base + kTcABytes;
  const uint32_t sB = base + 2 * kTcABytes;   // [2 buffers][g, u] x kTcBBytes
  const uint32_t full0 = sB + 4 * kTcBBytes;  // full[2], empty[2], loaded[2]
  const uint32_t empty0 = full0 + 16, loaded0 = full0 + 32;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int64_t cb = blockIdx.x;
  const int sp = blockIdx.y;
  const int r = a.r;
  constexpr int patA[6] = {0, 1, 0, 2, 0, 1};  // U terms per K block
  constexpr int patB[6] = {0, 0, 1, 0, 2, 1};  // P terms per K block
  if (warp == 0) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], 256;" ::"r"(
                     sh_addr(&s_tmem))
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  if (tid == 0) {
    for (int b = 0; b < 2; ++b) {
      asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(full0 + 8 * b) : "memory");
      asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(empty0 + 8 * b),
                   "r"(kTcEpiWarps)
                   : "memory");
      asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(loaded0 + 8 * b) : "memory");
    }
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  // A: this block's 128 channels of U_g (x -log2 e) and U_u (x -ln 2)
  if (tid < 2 * kTcCh) {
    const int row = tid & 127, mat = tid >> 7;
    const int64_t j = cb * kTcCh + row;
    const float* U = mat ? a.Uu : a.Ug;
    const float c = mat ? kTcNegLn2 : kTcNegLog2e;
    float x[8];
#pragma unroll
    for (int q = 0; q < 8; ++q) x[q] = (j < a.n && q < r) ? U[j * r + q] * c : 0.f;
    stage_split_row(mat ? sAu : sAg, row, x, patA);
  }
  const int64_t t0 = int64_t(sp) * a.chunk;
  const int64_t t1 = ::min(a.T_C, t0 + a.chunk);
  const int ntile = t1 > t0 ? int((t1 - t0 + kTcTok - 1) / kTcTok) : 0;
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = s_tmem;
  float acc = 0.f;
  const int q4 = warp & 3, half = (warp >> 2) & 1;
  if (warp == kTcEpiWarps) {
    // ---- producer (lane 0): each tile's split P rows arrive by one bulk copy
    // (prepared once for every channel block by score_split_p_kernel), two
    // tiles ahead; the MMAs of a tile start once its rows have landed and the
    // epilogue has read the accumulator buffer they overwrite
    const int64_t tile0 = t0 / kTcTok;
    bool ok = true;
    auto copy = [&](int it) {
      const int b = it & 1;
      const uint32_t lb = loaded0 + 8 * b;
      asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(lb),
                   "r"(2 * kTcBBytes)
                   : "memory");
      asm volatile(
          "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, "
          "[%3];" ::"r"(sB + b * 2 * kTcBBytes),
          "l"(a.psplit + (tile0 + it) * (2 * kTcBBytes / 16)), "r"(2 * kTcBBytes), "r"(lb)
          : "memory");
    };
    if (lane == 0) {
      for (int it = 0; it < ::min(ntile, 2); ++it) copy(it);
      for (int it = 0; it < ntile && ok; ++it) {
        const int b = it & 1;
        const uint32_t par = uint32_t((it >> 1) & 1);
        ok = tc_mbar_wait(loaded0 + 8 * b, par);                            // rows landed
        if (ok && it >= 2) ok = tc_mbar_wait(empty0 + 8 * b, par ^ 1u);    // tile it-2 read
        if (!ok) break;
        tc_fence_after();
#pragma unroll
        for (int m = 0; m < 2; ++m) {
          const uint32_t sa = m ? sAu : sAg, sb = sB + (b * 2 + m) * kTcBBytes;
          const uint32_t d = tmem + uint32_t(b * 2 * kTcTok + m * kTcTok);
#pragma unroll
          for (int k = 0; k < kTcK / 16; ++k) {
            const uint64_t ad = tc_sdesc(sa + k * 32), bd = tc_sdesc(sb + k * 32);
            const uint32_t en = k ? 1u : 0u;
            asm volatile(
                "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
                "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d),
                "l"(ad), "l"(bd), "r"(kTcIdesc), "r"(en)
                : "memory");
          }
        }
        asm volatile(
            "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                full0 + 8 * b)
            : "memory");
        if (it + 2 < ntile) {  // its operand rows are free once these MMAs are done
          ok = tc_mbar_wait(full0 + 8 * b, par);
          if (ok) copy(it + 2);
        }
      }
      // the last MMAs complete before the block releases its tensor memory
      if (ok && ntile > 0)
        tc_mbar_wait(full0 + 8 * ((ntile - 1) & 1), uint32_t(((ntile - 1) >> 1) & 1));
    }
    __syncwarp();
  } else {
    // ---- epilogue: this warp's 32 channels x 32 tokens of each tile
    for (int it = 0; it < ntile; ++it) {
      const int b = it & 1;
      if (!tc_mbar_wait(full0 + 8 * b, uint32_t((it >> 1) & 1))) break;
      tc_fence_after();
      uint32_t g[32], u[32];
      const uint32_t ta = tmem + (uint32_t(q4 * 32) << 16) + uint32_t(b * 2 * kTcTok + half * 32);
      tc_ld32(ta, g);
      tc_ld32(ta + kTcTok, u);
      asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
      tc_fence_before();
      __syncwarp();
      if (lane == 0) tc_arrive(empty0 + 8 * b);
      // silu(g) u = g' u' / (1 + 2^g') for two tokens at a time with one
      // reciprocal (Montgomery's simultaneous inversion: 1/d1 = d2 / (d1 d2));
      // 2^g' is capped at 2^60 so the product stays finite (a capped term is
      // below 2^-60 g' u' either way)
#pragma unroll
      for (int i = 0; i < 32; i += 2) {
        const float g1 = __uint_as_float(g[i]), u1 = __uint_as_float(u[i]);
        const float g2 = __uint_as_float(g[i + 1]), u2 = __uint_as_float(u[i + 1]);
        const float d1 = 1.f + fminf(ex2_approx(g1), 0x1p60f);
        const float d2 = 1.f + fminf(ex2_approx(g2), 0x1p60f);
        const float R = rcp_approx(d1 * d2);
        const float v1 = g1 * u1 * (d2 * R), v2 = g2 * u2 * (d1 * R);
        acc = fmaf(v1, v1, acc);
        acc = fmaf(v2, v2, acc);
      }
    }
  }
  // the two token halves of each channel, added in order
  tc_fence_before();
  if (warp < kTcEpiWarps && half) s_half[q4 * 32 + lane] = acc;
  __syncthreads();
  if (warp < kTcEpiWarps && !half) {
    const int64_t j = cb * kTcCh + q4 * 32 + lane;
    if (j < a.n) a.partial[int64_t(sp) * a.n + j] = acc + s_half[q4 * 32 + lane];
  }
  if (warp == 0) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, 256;" ::"r"(tmem)
                 : "memory");
  }
  score_tail<kTcCh>(a, cb, &s_last);
}

// ------------------------------------------------------------ Gram criterion
constexpr int kGramThreads = 256;
constexpr int kGramTokens = 64;  // P rows staged per round

struct GramArgs {
  const float* P;
  int64_t ldp;
  const int32_t* pmap;
  int64_t T_C;
  int r;
  int nmat;        // 1 or 2 matrices: columns [m r, (m + 1) r)
  int64_t chunk;   // tokens per block
  double* part;    // [gridDim.x x nmat x r x r]
  double* gram;    // [nmat x r x r]
  unsigned* counter;
};

__global__ void __launch_bounds__(kGramThreads) gram_partial_kernel(const __grid_constant__ GramArgs a) {
  __shared__ float sp[kGramTokens][2 * 48 + 1];
  __shared__ unsigned s_last;
  const int tid = threadIdx.x, r = a.r, ne = a.nmat * r * r;
  const int64_t t0 = int64_t(blockIdx.x) * a.chunk, t1 = ::min(a.T_C, t0 + a.chunk);
  double acc[(2 * 48 * 48 + kGramThreads - 1) / kGramThreads];
  constexpr int NE = (2 * 48 * 48 + kGramThreads - 1) / kGramThreads;
#pragma unroll
  for (int i = 0; i < NE; ++i) acc[i] = 0.0;
  const int w = a.nmat * r;
  for (int64_t tb = t0; tb < t1; tb += kGramTokens) {
    const int nt = int(::min(int64_t(kGramTokens), t1 - tb));
    __syncthreads();
    for (int e = tid; e < nt * w; e += kGramThreads) {
      const int tt = e / w, q = e % w;
      const int64_t row = a.pmap ? int64_t(a.pmap[tb + tt]) : tb + tt;
      sp[tt][q] = a.P[row * a.ldp + q];
    }
    __syncthreads();
#pragma unroll
    for (int i = 0; i < NE; ++i) {
      const int e = tid + i * kGramThreads;
      if (e < ne) {
        const int m = e / (r * r), x = (e / r) % r, y = e % r;
        double s = acc[i];
        for (int tt = 0; tt < nt; ++tt)
          s = fma(double(sp[tt][m * r + x]), double(sp[tt][m * r + y]), s);
        acc[i] = s;
      }
    }
  }
  double* mine = a.part + int64_t(blockIdx.x) * ne;
#pragma unroll
  for (int i = 0; i < NE; ++i) {
    const int e = tid + i * kGramThreads;
    if (e < ne) mine[e] = acc[i];
  }
  __syncthreads();  // the block's partials before thread 0's (cumulative) fence
  if (tid == 0) {
    __threadfence();
    s_last = (atomicAdd(a.counter, 1u) + 1u == gridDim.x) ? 1u : 0u;
  }
  __syncthreads();
  if (!s_last) return;
  __threadfence();
  // one warp per entry: lanes load the chunks' partials (all loads in flight
  // at once) and a fixed-order shuffle tree sums them
  const int lane = tid & 31, wid = tid >> 5;
  for (int e = wid; e < ne; e += kGramThreads / 32) {
    double s = 0.0;
    for (unsigned b = lane; b < gridDim.x; b += 32) s += __ldcg(a.part + int64_t(b) * ne + e);
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) s += __shfl_down_sync(0xffffffffu, s, off);
    if (lane == 0) a.gram[e] = s;
  }
}

constexpr int kNormThreads = 256;

struct NormArgs {
  const double* gram;   // [nmat x r x r]
  const float* U0;      // QK: U_q [heads*N x r]; L2: U [groups*N x r]
  const float* U1;      // QK: U_k [kv*N x r]
  int r;
  int mode;             // kCritModeQK, kCritModeL2
  int pair_half;        // > 0: score rotate-half pairs (c, c + half), half = N / 2
  int N;                // channels per head
  int rep;              // query heads per group (QK)
  int nkeys;            // keys per group: N, or N / 2 with pairs
  float* scores;        // [groups x nkeys]
};

__device__ __forceinline__ double quad_form(const double* G, const float* u, int r) {
  double s = 0.0;
  for (int x = 0; x < r; ++x) {
    double gx = 0.0;
    for (int y = 0; y < r; ++y) gx = fma(G[x * r + y], double(u[y]), gx);
    s = fma(double(u[x]), gx, s);
  }
  return s > 0.0 ? s : 0.0;
}

__global__ void __launch_bounds__(kNormThreads) norm_score_kernel(const __grid_constant__ NormArgs a) {
  __shared__ double sg[2 * 48 * 48];
  const int tid = threadIdx.x, r = a.r;
  const int nmat = a.mode == kCritModeQK ? 2 : 1;
  for (int e = tid; e < nmat * r * r; e += kNormThreads) sg[e] = a.gram[e];
  __syncthreads();
  const int grp = blockIdx.y;
  const int key = blockIdx.x * kNormThreads + tid;
  if (key >= a.nkeys) return;
  // norm^2 of channel c of head h of matrix m
  auto nsq = [&](int m, int h, int c) {
    const float* U = m == 0 ? a.U0 : a.U1;
    return quad_form(sg + m * r * r, U + (int64_t(h) * a.N + c) * r, r);
  };
  auto nrm = [&](int m, int h) {
    double s = nsq(m, h, key);
    if (a.pair_half) s += nsq(m, h, key + a.pair_half);
    return sqrt(s);
  };
  double score;
  if (a.mode == kCritModeQK) {
    double qs = 0.0;
    for (int j = 0; j < a.rep; ++j) qs += nrm(0, grp * a.rep + j);
    score = nrm(1, grp) * qs;
  } else {
    score = nrm(0, grp);
  }
  a.scores[int64_t(grp) * a.nkeys + key] = float(score);
}

// ------------------------------------------------------------------ top-k
// One block per group; the scratch lives in the kernel's own shared arrays.
// 512 threads for long score vectors, 128 for short per-head ones.
constexpr int kTopkMaxM = 64;  // rows per thread: n <= 512 * 64

template <int B, int MAXM, bool ONE>
__global__ void __launch_bounds__(B) topk_kernel(const float* __restrict__ scores, int N, int k,
                                                 int32_t* out_a, int32_t* out_b, int rep, int hN,
                                                 int pair_half) {
  __shared__ __align__(16) uint32_t s_red[2 * (B / 32)];
  __shared__ __align__(16) uint32_t s_hist[topk_hist_words()];
  __shared__ __align__(16) uint32_t s_cand[topk_cand_words()];
  __shared__ __align__(16) uint32_t s_tab[topk_tab_words<B, MAXM>()];
  __shared__ __align__(16) uint32_t s_bc[8];
  block_topk<B, MAXM, ONE>(scores + int64_t(blockIdx.x) * N, N, k, out_a, out_b, rep, hN,
                           pair_half, blockIdx.x, sh_addr(s_red), sh_addr(s_hist),
                           sh_addr(s_cand), sh_addr(s_tab), sh_addr(s_bc));
}

int rank_chunks(int r) { return r <= 8 ? 1 : (r <= 16 ? 2 : (r <= 24 ? 3 : (r <= 32 ? 4 : 6))); }
// Score kernel by rank: packed FMA for r <= 16, tensor cores above (whose
// factor rows no longer fit the registers of the FMA form).
int channels_per_block(int r) {
  if (r <= 8) return kTcCh;
  if (r <= 16) return fma_channels<16>();
  return kScoreWarps * score_nt(rank_chunks(r)) * 8;
}

template <class K>
int blocks_per_sm_of(K kernel, int smem) {
  int b = 0;
  // the dynamic limit is raised whenever there is dynamic memory: static and
  // dynamic together may pass 48 KB even when the dynamic part alone does not
  if ((smem > 0 &&
       cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) !=
           cudaSuccess) ||
      cudaOccupancyMaxActiveBlocksPerMultiprocessor(&b, kernel, kScoreThreads, smem) !=
          cudaSuccess ||
      b < 1) {
    cudaGetLastError();
    b = 1;
  }
  return b;
}
int score_blocks_per_sm(int r) {
  if (r <= 8) return 2;  // the tensor-core kernel: two blocks of 256 TMEM columns
  static int cached[5] = {0, 0, 0, 0, 0};
  const int v = r <= 16 ? 1 : (r <= 24 ? 2 : (r <= 32 ? 3 : 4));
  if (!cached[v]) {
    switch (v) {
      case 1: cached[v] = blocks_per_sm_of(ffn_score_fma_kernel<16>, 0); break;
      case 2: cached[v] = blocks_per_sm_of(ffn_score_mma_kernel<3>, score_stage_bytes(3)); break;
      case 3: cached[v] = blocks_per_sm_of(ffn_score_mma_kernel<4>, score_stage_bytes(4)); break;
      default: cached[v] = blocks_per_sm_of(ffn_score_mma_kernel<6>, score_stage_bytes(6));
    }
  }
  return cached[v];
}

template <int C>
slora_status launch_score_mma(dim3 grid, const ScoreArgs& a, cudaStream_t st) {
  const int smem = score_stage_bytes(C);
  // static (the top-k scratch) plus dynamic staging passes 48 KB
  SLORA_CUDA(cudaFuncSetAttribute(ffn_score_mma_kernel<C>,
                                  cudaFuncAttributeMaxDynamicSharedMemorySize, smem));
  ffn_score_mma_kernel<C><<<grid, kScoreThreads, smem, st>>>(a);
  return SLORA_OK;
}

}  // namespace

int64_t ffn_score_blocks(int64_t n, int r) {
  const int ch = channels_per_block(r);
  return (n + ch - 1) / ch;
}

// Token splits: for the tensor-core kernel (rank <= 8) about one and a half
// blocks per SM, two resident per SM, each pipelining its tiles (blocks of a
// few tiles measured slower: their setup does not amortise); otherwise as
// many as keep the grid within one wave of resident blocks.
int ffn_score_splits(int64_t T_C, int64_t n, int r) {
  if (r <= 8) {
    const int64_t tiles = std::max<int64_t>((T_C + kTcTok - 1) / kTcTok, 1);
    const int64_t nb = std::max<int64_t>(ffn_score_blocks(n, r), 1);
    const int64_t want = (int64_t(num_sms()) * 3 / 2 + nb - 1) / nb;
    return int(std::min<int64_t>(std::max<int64_t>(want, 1), std::min<int64_t>(tiles, 256)));
  }
  const int64_t nb = ffn_score_blocks(n, r);
  const int64_t slots = int64_t(num_sms()) * score_blocks_per_sm(r);
  int64_t want = slots / std::max<int64_t>(nb, 1);
  const int64_t maxs = std::max<int64_t>((T_C + 15) / 16, 1);
  int64_t s = std::min(want, maxs);
  if (s < 1) s = 1;
  if (s > 256) s = 256;
  return int(s);
}

int64_t score_split_tiles(int64_t T_C) { return std::max<int64_t>((T_C + kTcTok - 1) / kTcTok, 1); }

int64_t estimator_counter_count(int64_t n, int r, int groups) {
  (void)groups;  // the score kernels count per channel block, the Gram pass in one word
  return std::max<int64_t>(ffn_score_blocks(n, r), 1) + 1;
}

// Token chunks of the Gram pass: one staging round (64 tokens) per block, at
// most 64 blocks (the last block sums every block's partial Gram matrices;
// 296 blocks of 16 tokens measured slower than 48 of 64 at 3072 tokens).
int64_t gram_blocks(int64_t T_C) {
  const int64_t want = (T_C + kGramTokens - 1) / kGramTokens;
  return std::max<int64_t>(1, std::min<int64_t>(want, 64));
}

namespace {
template <bool ONE>
void launch_topk_kernel(const float* scores, int groups, int N, int k, const TopkOut& o,
                        cudaStream_t st) {
  const unsigned gr = unsigned(groups);
  if (N <= 128 * 8)
    topk_kernel<128, 8, ONE><<<gr, 128, 0, st>>>(scores, N, k, o.a, o.b, o.rep, o.N, o.pair_half);
  else if (N <= 512 * 8)
    topk_kernel<512, 8, ONE><<<gr, 512, 0, st>>>(scores, N, k, o.a, o.b, o.rep, o.N, o.pair_half);
  else if (N <= 512 * 32)
    topk_kernel<512, 32, ONE><<<gr, 512, 0, st>>>(scores, N, k, o.a, o.b, o.rep, o.N,
                                                  o.pair_half);
  else
    topk_kernel<512, kTopkMaxM, ONE><<<gr, 512, 0, st>>>(scores, N, k, o.a, o.b, o.rep, o.N,
                                                         o.pair_half);
}

// One top-k block per group, the register array sized to the keys per thread.
slora_status launch_topk(const float* scores, int groups, int N, int k, const TopkOut& o,
                         cudaStream_t st) {
  if (k <= 0 || groups <= 0) return SLORA_OK;
  if (int64_t(N) > int64_t(512) * kTopkMaxM)
    SLORA_FAIL(SLORA_ERR_SHAPE, "top-k over %d keys per group exceeds the supported %d", N,
               512 * kTopkMaxM);
  const int per_head = o.pair_half ? 2 * k : k;
  LaunchScope ls(kSelect, double(groups) * N * 4 + double(groups) * per_head * 4 * (o.rep + 1),
                 st);
  if (o.rep == 1 && !o.b && !o.pair_half)
    launch_topk_kernel<true>(scores, groups, N, k, o, st);
  else
    launch_topk_kernel<false>(scores, groups, N, k, o, st);
  SLORA_CHECK_LAUNCH();
  return SLORA_OK;
}
}  // namespace

slora_status ffn_score_select(const float* P, int64_t ldp, const int32_t* pmap, int64_t T_C,
                              const float* Ug, const float* Uu, int64_t n, int r, float* partial,
                              int nsplit, float* scores, unsigned* counters, int k,
                              int32_t* idx_out, void* psplit, cudaStream_t st) {
  if (n <= 0) return SLORA_OK;
  ScoreArgs a;
  a.P = P; a.ldp = ldp; a.pmap = pmap; a.T_C = T_C; a.Ug = Ug; a.Uu = Uu; a.n = n; a.r = r;
  a.nsplit = nsplit;
  a.psplit = static_cast<const uint4*>(psplit);
  // tokens per split: whole 128-token tiles for the tensor-core kernel, 16 otherwise
  const int64_t q = r <= 8 ? kTcTok : 16;
  a.chunk = T_C > 0 ? ((T_C + nsplit - 1) / nsplit + q - 1) / q * q : q;
  a.partial = partial; a.scores = scores; a.counters = counters;
  const dim3 grid(unsigned(ffn_score_blocks(n, r)), unsigned(nsplit));
  {
    // bytes: P rows of the context tokens, both factors, partials and scores
    LaunchScope ls(kEstimate, double(T_C) * 2 * r * 4 + double(n) * 2 * r * 4 +
                                  double(nsplit) * n * 8 + double(n) * 4, st);
    if (r <= 8) {
      if (!psplit) SLORA_FAIL(SLORA_ERR_INVALID_ARG, "score: split-operand workspace missing");
      const int64_t ntiles = score_split_tiles(T_C);
      {
        LaunchScope lp(kAux, double(T_C) * 2 * r * 4 + double(ntiles) * 2 * kTcBBytes, st);
        score_split_p_kernel<<<unsigned((ntiles * 2 * kTcTok + 255) / 256), 256, 0, st>>>(
            P, ldp, pmap, T_C, r, ntiles, static_cast<uint4*>(psplit));
        SLORA_CHECK_LAUNCH();
      }
      SLORA_CUDA(cudaFuncSetAttribute(ffn_score_tc_kernel,
                                      cudaFuncAttributeMaxDynamicSharedMemorySize, kTcSmem));
      // the largest shared-memory carveout, or only one block fits per SM
      SLORA_CUDA(cudaFuncSetAttribute(ffn_score_tc_kernel,
                                      cudaFuncAttributePreferredSharedMemoryCarveout, 100));
      ffn_score_tc_kernel<<<grid, kTcThreads, kTcSmem, st>>>(a);
    } else if (r <= 16)
      ffn_score_fma_kernel<16><<<grid, kScoreThreads, 0, st>>>(a);
    else if (r <= 24)
      SLORA_TRY(launch_score_mma<3>(grid, a, st));
    else if (r <= 32)
      SLORA_TRY(launch_score_mma<4>(grid, a, st));
    else
      SLORA_TRY(launch_score_mma<6>(grid, a, st));
  }
  SLORA_CHECK_LAUNCH();
  if (!idx_out) return SLORA_OK;
  TopkOut o;
  o.a = idx_out;
  o.N = int(n);
  return launch_topk(scores, 1, int(n), k, o, st);
}

slora_status gram_scores_select(int mode, const float* P, int64_t ldp, const int32_t* pmap,
                                int64_t T_C, const float* U0, const float* U1, int r, int groups,
                                int rep, int N, bool pairs, int k, double* gram_part,
                                double* gram, float* scores, unsigned* counters, int32_t* out_a,
                                int32_t* out_b, cudaStream_t st) {
  const int nmat = mode == kCritModeQK ? 2 : 1;
  GramArgs ga;
  ga.P = P; ga.ldp = ldp; ga.pmap = pmap; ga.T_C = T_C; ga.r = r; ga.nmat = nmat;
  const int64_t nb = gram_blocks(T_C);
  ga.chunk = T_C > 0 ? (T_C + nb - 1) / nb : 1;
  ga.part = gram_part; ga.gram = gram; ga.counter = counters;
  {
    LaunchScope ls(kEstimate, double(T_C) * nmat * r * 4 + double(nb) * nmat * r * r * 8, st);
    gram_partial_kernel<<<unsigned(nb), kGramThreads, 0, st>>>(ga);
  }
  SLORA_CHECK_LAUNCH();
  NormArgs na;
  na.gram = gram; na.U0 = U0; na.U1 = U1; na.r = r; na.mode = mode;
  na.pair_half = pairs ? N / 2 : 0;
  na.N = N; na.rep = rep;
  na.nkeys = pairs ? N / 2 : N;
  na.scores = scores;
  const dim3 grid(unsigned((na.nkeys + kNormThreads - 1) / kNormThreads), unsigned(groups));
  {
    const int nu = mode == kCritModeQK ? (rep + 1) : 1;
    LaunchScope ls(kSelect, double(groups) * N * nu * r * 4 + double(groups) * na.nkeys * 4, st);
    norm_score_kernel<<<grid, kNormThreads, 0, st>>>(na);
  }
  SLORA_CHECK_LAUNCH();
  if (!out_a) return SLORA_OK;
  TopkOut o;
  o.a = out_a; o.b = out_b; o.rep = rep; o.N = N; o.pair_half = na.pair_half;
  return launch_topk(scores, groups, na.nkeys, k, o, st);
}

slora_status topk_select(const float* scores, int groups, int N, int k, int rep,
                         int32_t* out_a, int32_t* out_b, cudaStream_t st) {
  TopkOut o;
  o.a = out_a; o.b = out_b; o.rep = rep; o.N = N;
  return launch_topk(scores, groups, N, k, o, st);
}

int64_t topk_max_keys() { return int64_t(512) * kTopkMaxM; }

slora_status est_check_error(bool clear) {
  int v = 0;
  SLORA_CUDA(cudaMemcpyFromSymbol(&v, g_est_error, sizeof(int)));
  if (clear && v) {
    int z = 0;
    SLORA_CUDA(cudaMemcpyToSymbol(g_est_error, &z, sizeof(int)));
  }
  if (v) SLORA_FAIL(SLORA_ERR_CUDA, "estimator: a score kernel's shared staging buffer is misaligned");
  return SLORA_OK;
}

}  // namespace slora
