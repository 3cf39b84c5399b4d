// Shared internals of libslora: status reporting, workspace carving, element
// access helpers.  Nothing here is part of the C ABI.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cstdarg>
#include <cstdint>
#include <cstdio>
#include <string>

#include "../../include/slora.h"

namespace slora {

enum DT : int { kF32 = 0, kBF16 = 1 };

inline int dt_size(int dt) { return dt == kF32 ? 4 : 2; }

// ---------------------------------------------------------------- errors
void set_error(const char* fmt, ...);
void clear_error();

#define SLORA_FAIL(code, ...)      \
  do {                             \
    ::slora::set_error(__VA_ARGS__); \
    return (code);                 \
  } while (0)

#define SLORA_CUDA(call)                                                              \
  do {                                                                                \
    cudaError_t e_ = (call);                                                          \
    if (e_ != cudaSuccess)                                                            \
      SLORA_FAIL(SLORA_ERR_CUDA, "%s failed: %s (%s:%d)", #call, cudaGetErrorString(e_), \
                 __FILE__, __LINE__);                                                 \
  } while (0)

#define SLORA_CHECK_LAUNCH()                                                          \
  do {                                                                                \
    cudaError_t e_ = cudaGetLastError();                                              \
    if (e_ != cudaSuccess)                                                            \
      SLORA_FAIL(SLORA_ERR_CUDA, "kernel launch failed: %s (%s:%d)",                  \
                 cudaGetErrorString(e_), __FILE__, __LINE__);                         \
  } while (0)

#define SLORA_TRY(expr)                 \
  do {                                  \
    slora_status s_ = (expr);           \
    if (s_ != SLORA_OK) return s_;      \
  } while (0)

// ------------------------------------------------------------- workspace
// Bump allocator over the caller's workspace.  With base == nullptr it only
// counts bytes (the workspace-size query).  A run path takes every buffer it
// needs before its first launch and then calls fits(): the planning pass and
// the run pass must take the same sequence, and fits() turns any mismatch
// into an error before a kernel could touch memory past the workspace.
struct Arena {
  char* base = nullptr;
  size_t used = 0;
  size_t cap = ~size_t(0);  // bytes of the caller's workspace (run pass)
  template <class T>
  T* take(size_t count) {
    size_t off = (used + 255) & ~size_t(255);
    used = off + count * sizeof(T);
    return base ? reinterpret_cast<T*>(base + off) : nullptr;
  }
};
slora_status arena_fits(const Arena& ar, const char* where);

// ------------------------------------------------------------- devices
slora_status check_device();  // sm_100 present and current
// SMs of the current device (queried once and cached; 148 when no device
// answers, e.g. during a host-only workspace query).
int num_sms();

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// ------------------------------------------------------------- tokens
// Row maps of the context / output tokens of one call, built on the device.
constexpr int kMaxBatch = 2048;
struct TokenInfo {
  int batch = 0, seq = 0;
  int64_t T = 0, T_C = 0, T_O = 0;
};
slora_status parse_tokens(const slora_tokens* tok, TokenInfo* info);
// Writes ctx_rows[T_C] and out_rows[T_O] (int32 row indices into the full
// layout) and, when given, the 128-row M-tile lists of the context and output
// rows: int4 {full_row0, compact_row0, nvalid, 0}, one list per row kind, a
// tile never crossing a sequence.  It also zeroes the counter ranges `zero`
// [nzero] and `zero2` [nzero2] that later kernels of the call count on.
slora_status launch_rowmaps(const slora_tokens* tok, const TokenInfo& ti, int32_t* ctx_rows,
                            int32_t* out_rows, cudaStream_t st, int4* ctx_tiles = nullptr,
                            int4* out_tiles = nullptr, unsigned* zero = nullptr,
                            int64_t nzero = 0, unsigned* zero2 = nullptr, int64_t nzero2 = 0);
// A library-owned side stream of the current device (non-blocking, created on
// first use, kept until exit) with a fork and a join event, for running small
// independent launches of one call beside its main stream: fork_side() makes
// `side` wait for the work issued so far on `st`; join_side() makes `st` wait
// for what was issued on `side` since.  Both are stream-ordered (they work
// inside a CUDA-graph capture of `st`).
slora_status side_stream(cudaStream_t* side);
// Entry i of a per-device pool of kSidePool such streams (entry 0 is the one
// side_stream() gives), each with its own fork and join events; fork_side /
// join_side take any pool stream.  side_pool_ready(n): entries 1 .. n - 1
// exist (creating one is not done while a stream is being captured).
constexpr int kSidePool = 8;
slora_status side_stream_at(int i, cudaStream_t* side);
bool side_pool_ready(int n);
slora_status fork_side(cudaStream_t st, cudaStream_t side);
slora_status join_side(cudaStream_t st, cudaStream_t side);
// Number of 128-row tiles of the context rows / output rows.
int64_t count_tiles(const slora_tokens* tok, bool ctx);
inline int64_t round8(int64_t x) { return (x + 7) / 8 * 8; }

// ------------------------------------------------------------- launches
// Kernel classes for launch accounting (names in slora_profile_read).
enum KClass : int { kGemmTC = 0, kGemmSimt, kEstimate, kSelect, kElementwise, kAux, kPrepare,
                    kSkinny, kCompact, kAttention, kNorm, kNumClasses };
// Construct immediately before a kernel launch: counts it and, while
// profiling is on, records CUDA events around it on `st`.
struct LaunchScope {
  LaunchScope(int cls, double work, cudaStream_t st);
  ~LaunchScope();
  int cls_;
  cudaStream_t st_;
  int slot_;
};

// ------------------------------------------------------------- elements
__device__ __forceinline__ float ld_elem(const void* p, int64_t i, int dt) {
  if (dt == kF32) return static_cast<const float*>(p)[i];
  return __bfloat162float(static_cast<const __nv_bfloat16*>(p)[i]);
}
__device__ __forceinline__ void st_elem(void* p, int64_t i, int dt, float v) {
  if (dt == kF32)
    static_cast<float*>(p)[i] = v;
  else
    static_cast<__nv_bfloat16*>(p)[i] = __float2bfloat16_rn(v);
}

// silu(x) = x * sigmoid(x) in fp32.  __expf is the fast exp2-based intrinsic
// (relative error a few ulp); for x << 0 exp(-x) overflows to +inf and the
// reciprocal gives 0, so silu -> 0 as it should.
__device__ __forceinline__ float silu_f(float x) { return __fdividef(x, 1.0f + __expf(-x)); }
__device__ __forceinline__ float sigmoid_f(float x) { return __fdividef(1.0f, 1.0f + __expf(-x)); }

}  // namespace slora
