// slora_estimate_select_noalloc: the estimate + select call for callers that
// cannot hand the library a workspace (see include/slora.h).  Its scratch is a
// file-scope device buffer of fixed size that every GPU loading this library
// keeps until the process exits.
#include <cuda.h>

#include <mutex>

#include "common.cuh"

namespace {

constexpr size_t kNoAllocScratchBytes = size_t(32) << 20;  // 32 MiB per device
constexpr int kMaxDevices = 64;

__device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

// The resolved address is valid for the context it was resolved in: it is
// cached per device together with that context's handle and resolved again
// when the calling thread's current context differs (a non-primary context,
// or the primary context recreated after cudaDeviceReset).
struct Resolved {
  CUcontext ctx = nullptr;
  void* ptr = nullptr;
};
std::mutex g_noalloc_mu;
Resolved g_noalloc[kMaxDevices];

typedef CUresult (*CtxGetCurrentFn)(CUcontext*);

// cuCtxGetCurrent through the runtime's driver entry-point lookup (no link
// against the driver library).  *ctx is NULL when the thread has no current
// context yet.
slora_status current_context(CUcontext* ctx) {
  static CtxGetCurrentFn fn = nullptr;
  if (!fn) {
    void* f = nullptr;
    cudaDriverEntryPointQueryResult q = cudaDriverEntryPointSymbolNotFound;
    const cudaError_t e = cudaGetDriverEntryPoint("cuCtxGetCurrent", &f, cudaEnableDefault, &q);
    if (e != cudaSuccess || q != cudaDriverEntryPointSuccess || !f)
      SLORA_FAIL(SLORA_ERR_CUDA, "driver entry point cuCtxGetCurrent unavailable: %s",
                 cudaGetErrorString(e));
    fn = reinterpret_cast<CtxGetCurrentFn>(f);
  }
  *ctx = nullptr;
  if (fn(ctx) != CUDA_SUCCESS) *ctx = nullptr;
  return SLORA_OK;
}

// Device address of the scratch buffer in the current context.  In host code
// the symbol itself only names a host-side stand-in, so the address comes
// from cudaGetSymbolAddress, with the device current, once per context.
slora_status noalloc_scratch(void** out) {
  int dev = -1;
  SLORA_CUDA(cudaGetDevice(&dev));
  if (dev < 0 || dev >= kMaxDevices)
    SLORA_FAIL(SLORA_ERR_UNSUPPORTED, "device index %d beyond %d", dev, kMaxDevices);
  CUcontext ctx = nullptr;
  SLORA_TRY(current_context(&ctx));
  std::lock_guard<std::mutex> lock(g_noalloc_mu);
  Resolved& r = g_noalloc[dev];
  if (!r.ptr || !ctx || r.ctx != ctx) {
    // cudaGetSymbolAddress also makes the device's primary context current
    // when the thread has none yet; the context is read again afterwards.
    void* p = nullptr;
    const cudaError_t e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess || p == nullptr)
      SLORA_FAIL(SLORA_ERR_CUDA, "cudaGetSymbolAddress of the scratch buffer failed: %s",
                 cudaGetErrorString(e));
    SLORA_TRY(current_context(&ctx));
    r.ctx = ctx;
    r.ptr = p;
  }
  *out = r.ptr;
  return SLORA_OK;
}

}  // namespace

extern "C" size_t slora_noalloc_scratch_bytes(void) { return kNoAllocScratchBytes; }

extern "C" slora_status slora_estimate_select_noalloc(
    slora_criterion crit, const void* X, slora_dtype dt, const slora_tokens* tok, int64_t d,
    const float* L0, const float* U0, int64_t n0, const float* L1, const float* U1, int64_t n1,
    int rank, int heads, int kv_heads, int head_dim, double sparsity, int32_t* idx_out,
    int32_t* k_out, float* scores_out, slora_stream_t stream) {
  // Size the scratch with the regular entry point's workspace query (host
  // only, launches nothing) and refuse what does not fit the buffer.
  size_t need = 0;
  slora_status s = slora_estimate_select(crit, X, dt, tok, d, L0, U0, n0, L1, U1, n1, rank, heads,
                                         kv_heads, head_dim, sparsity, idx_out, k_out,
                                         scores_out, nullptr, &need, stream);
  if (s != SLORA_OK) return s;
  if (need > kNoAllocScratchBytes)
    SLORA_FAIL(SLORA_ERR_WORKSPACE,
               "slora_estimate_select_noalloc: this problem needs %zu bytes of scratch but the "
               "built-in buffer holds %zu; call slora_estimate_select with a workspace instead",
               need, kNoAllocScratchBytes);
  void* scratch = nullptr;
  s = noalloc_scratch(&scratch);
  if (s != SLORA_OK) return s;
  size_t have = kNoAllocScratchBytes;
  return slora_estimate_select(crit, X, dt, tok, d, L0, U0, n0, L1, U1, n1, rank, heads, kv_heads,
                               head_dim, sparsity, idx_out, k_out, scores_out, scratch, &have,
                               stream);
}
