// Error text, device checks and token row maps.
#include <mutex>
#include <vector>

#include "attention.cuh"
#include "common.cuh"
#include "estimator.cuh"
#include "gemm_tc.cuh"
#include "lora_pack.cuh"
#include "skinny.cuh"

namespace slora {

namespace {
thread_local std::string g_error;

// The host's ctx_len travels in the kernel parameters: a small block for the
// usual batch sizes, the full kMaxBatch block otherwise (a parameter block
// of 8 KB makes every launch slower).
template <int CAP>
struct RowmapParams {
  int batch, seq;
  int ctx_len[CAP];
};
constexpr int kSmallBatch = 64;

// One block: scan ctx_len into per-sequence offsets, then every row t of the
// full layout lands in ctx_rows or out_rows at its compact position, and every
// sequence emits its context and output M tiles.
template <int CAP>
__global__ void __launch_bounds__(1024) rowmap_kernel(const __grid_constant__ RowmapParams<CAP> p,
                                                      int32_t* __restrict__ ctx_rows,
                                                      int32_t* __restrict__ out_rows,
                                                      int4* __restrict__ ctx_tiles,
                                                      int4* __restrict__ out_tiles,
                                                      unsigned* __restrict__ zero,
                                                      int64_t nzero,
                                                      unsigned* __restrict__ zero2,
                                                      int64_t nzero2) {
  for (int64_t i = threadIdx.x; i < nzero; i += blockDim.x) zero[i] = 0u;
  for (int64_t i = threadIdx.x; i < nzero2; i += blockDim.x) zero2[i] = 0u;
  __shared__ int ctx_off[CAP], ct_off[CAP], ot_off[CAP];
  if (threadIdx.x == 0) {
    int acc = 0, ct = 0, ot = 0;
    for (int b = 0; b < p.batch; ++b) {
      ctx_off[b] = acc;
      ct_off[b] = ct;
      ot_off[b] = ot;
      const int c = p.ctx_len[b];
      acc += c;
      ct += (c + 127) / 128;
      ot += (p.seq - c + 127) / 128;
    }
  }
  __syncthreads();
  const int64_t T = int64_t(p.batch) * p.seq;
  for (int64_t t = threadIdx.x; t < T; t += blockDim.x) {
    const int b = int(t / p.seq), i = int(t % p.seq);
    const int c = p.ctx_len[b];
    if (i < c) {
      if (ctx_rows) ctx_rows[ctx_off[b] + i] = int32_t(t);
    } else {
      // output rows before sequence b: b*seq - ctx_off[b]
      if (out_rows) out_rows[int64_t(b) * p.seq - ctx_off[b] + (i - c)] = int32_t(t);
    }
  }
  for (int b = threadIdx.x; b < p.batch; b += blockDim.x) {
    const int c = p.ctx_len[b];
    const int full0 = b * p.seq;
    if (ctx_tiles)
      for (int j = 0; j * 128 < c; ++j)
        ctx_tiles[ct_off[b] + j] = make_int4(full0 + 128 * j, ctx_off[b] + 128 * j,
                                             min(128, c - 128 * j), 0);
    const int o0 = b * p.seq - ctx_off[b];
    if (out_tiles)
      for (int j = 0; j * 128 < p.seq - c; ++j)
        out_tiles[ot_off[b] + j] = make_int4(full0 + c + 128 * j, o0 + 128 * j,
                                             min(128, p.seq - c - 128 * j), 0);
  }
}
}  // namespace

void set_error(const char* fmt, ...) {
  char buf[1024];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof(buf), fmt, ap);
  va_end(ap);
  g_error = buf;
}

void clear_error() { g_error.clear(); }

slora_status arena_fits(const Arena& ar, const char* where) {
  if (ar.used > ar.cap)
    SLORA_FAIL(SLORA_ERR_WORKSPACE, "%s: internal error: the run takes %zu workspace bytes, the "
               "plan gave %zu", where, ar.used, ar.cap);
  return SLORA_OK;
}

slora_status check_device() {
  int dev = -1;
  SLORA_CUDA(cudaGetDevice(&dev));
  int major = 0, minor = 0;
  SLORA_CUDA(cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev));
  SLORA_CUDA(cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev));
  if (major != 10 || minor != 0)
    SLORA_FAIL(SLORA_ERR_UNSUPPORTED, "device %d is sm_%d%d; this library is built for sm_100a",
               dev, major, minor);
  return SLORA_OK;
}

int num_sms() {
  static int n = 0;
  if (!n) {
    int dev = 0, v = 0;
    if (cudaGetDevice(&dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || v <= 0) {
      cudaGetLastError();
      v = 148;
    }
    n = v;
  }
  return n;
}

slora_status parse_tokens(const slora_tokens* tok, TokenInfo* ti) {
  if (!tok || !tok->ctx_len) SLORA_FAIL(SLORA_ERR_INVALID_ARG, "tokens or tokens->ctx_len is NULL");
  if (tok->batch <= 0 || tok->seq <= 0)
    SLORA_FAIL(SLORA_ERR_SHAPE, "batch=%d seq=%d must be positive", tok->batch, tok->seq);
  if (tok->batch > kMaxBatch)
    SLORA_FAIL(SLORA_ERR_SHAPE, "batch=%d exceeds the supported maximum %d", tok->batch, kMaxBatch);
  int64_t T = int64_t(tok->batch) * tok->seq;
  if (T > (int64_t(1) << 30)) SLORA_FAIL(SLORA_ERR_SHAPE, "T=%lld rows too large", (long long)T);
  int64_t tc = 0;
  for (int b = 0; b < tok->batch; ++b) {
    int c = tok->ctx_len[b];
    if (c < 0 || c > tok->seq)
      SLORA_FAIL(SLORA_ERR_SHAPE, "ctx_len[%d]=%d outside [0, seq=%d]", b, c, tok->seq);
    tc += c;
  }
  ti->batch = tok->batch;
  ti->seq = tok->seq;
  ti->T = T;
  ti->T_C = tc;
  ti->T_O = T - tc;
  return SLORA_OK;
}

int64_t count_tiles(const slora_tokens* tok, bool ctx) {
  int64_t n = 0;
  for (int b = 0; b < tok->batch; ++b) {
    const int c = tok->ctx_len[b];
    n += ctx ? (c + 127) / 128 : (tok->seq - c + 127) / 128;
  }
  return n;
}

namespace {
constexpr int kSideDevices = 64;
struct Side {
  cudaStream_t s = nullptr;
  cudaEvent_t fork = nullptr, join = nullptr;
};
std::mutex g_side_mu;
// Per device: entry 0 is the side stream of a single call; the others serve
// calls that run several lanes of work at once.
Side g_side[kSideDevices][kSidePool];
slora_status side_for(int i, Side** out) {
  int dev = -1;
  SLORA_CUDA(cudaGetDevice(&dev));
  if (dev < 0 || dev >= kSideDevices)
    SLORA_FAIL(SLORA_ERR_UNSUPPORTED, "device index %d beyond %d", dev, kSideDevices);
  if (i < 0 || i >= kSidePool) SLORA_FAIL(SLORA_ERR_INVALID_ARG, "side stream %d of %d", i, kSidePool);
  std::lock_guard<std::mutex> lock(g_side_mu);
  Side& sd = g_side[dev][i];
  if (!sd.s) {
    SLORA_CUDA(cudaStreamCreateWithFlags(&sd.s, cudaStreamNonBlocking));
    SLORA_CUDA(cudaEventCreateWithFlags(&sd.fork, cudaEventDisableTiming));
    SLORA_CUDA(cudaEventCreateWithFlags(&sd.join, cudaEventDisableTiming));
  }
  *out = &sd;
  return SLORA_OK;
}
// The pool entry of stream `side` on the current device.
slora_status side_of(cudaStream_t side, Side** out) {
  int dev = -1;
  SLORA_CUDA(cudaGetDevice(&dev));
  if (dev < 0 || dev >= kSideDevices)
    SLORA_FAIL(SLORA_ERR_UNSUPPORTED, "device index %d beyond %d", dev, kSideDevices);
  std::lock_guard<std::mutex> lock(g_side_mu);
  for (int i = 0; i < kSidePool; ++i)
    if (g_side[dev][i].s == side && side) {
      *out = &g_side[dev][i];
      return SLORA_OK;
    }
  SLORA_FAIL(SLORA_ERR_INVALID_ARG, "internal error: stream is not a library side stream");
}
}  // namespace

slora_status side_stream(cudaStream_t* side) { return side_stream_at(0, side); }

slora_status side_stream_at(int i, cudaStream_t* side) {
  Side* sd = nullptr;
  SLORA_TRY(side_for(i, &sd));
  *side = sd->s;
  return SLORA_OK;
}

bool side_pool_ready(int n) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kSideDevices || n > kSidePool) {
    cudaGetLastError();
    return false;
  }
  std::lock_guard<std::mutex> lock(g_side_mu);
  for (int i = 1; i < n; ++i)
    if (!g_side[dev][i].s) return false;
  return true;
}

// The record and the wait happen under the lock, so calls from several host
// threads cannot interleave on the shared events.
slora_status fork_side(cudaStream_t st, cudaStream_t side) {
  Side* sd = nullptr;
  SLORA_TRY(side_of(side, &sd));
  std::lock_guard<std::mutex> lock(g_side_mu);
  SLORA_CUDA(cudaEventRecord(sd->fork, st));
  SLORA_CUDA(cudaStreamWaitEvent(side, sd->fork, 0));
  return SLORA_OK;
}

slora_status join_side(cudaStream_t st, cudaStream_t side) {
  Side* sd = nullptr;
  SLORA_TRY(side_of(side, &sd));
  std::lock_guard<std::mutex> lock(g_side_mu);
  SLORA_CUDA(cudaEventRecord(sd->join, side));
  SLORA_CUDA(cudaStreamWaitEvent(st, sd->join, 0));
  return SLORA_OK;
}

slora_status launch_rowmaps(const slora_tokens* tok, const TokenInfo& ti, int32_t* ctx_rows,
                            int32_t* out_rows, cudaStream_t st, int4* ctx_tiles,
                            int4* out_tiles, unsigned* zero, int64_t nzero, unsigned* zero2,
                            int64_t nzero2) {
  LaunchScope ls(kAux, double(ti.T) * 4, st);
  if (ti.batch <= kSmallBatch) {
    RowmapParams<kSmallBatch> p;
    p.batch = ti.batch;
    p.seq = ti.seq;
    for (int b = 0; b < ti.batch; ++b) p.ctx_len[b] = tok->ctx_len[b];
    rowmap_kernel<kSmallBatch><<<1, 1024, 0, st>>>(p, ctx_rows, out_rows, ctx_tiles, out_tiles,
                                                   zero, zero ? nzero : 0, zero2,
                                                   zero2 ? nzero2 : 0);
  } else {
    RowmapParams<kMaxBatch> p;
    p.batch = ti.batch;
    p.seq = ti.seq;
    for (int b = 0; b < ti.batch; ++b) p.ctx_len[b] = tok->ctx_len[b];
    rowmap_kernel<kMaxBatch><<<1, 1024, 0, st>>>(p, ctx_rows, out_rows, ctx_tiles, out_tiles,
                                                 zero, zero ? nzero : 0, zero2,
                                                 zero2 ? nzero2 : 0);
  }
  SLORA_CHECK_LAUNCH();
  return SLORA_OK;
}

}  // namespace slora

extern "C" const char* slora_last_error_string(void) { return slora::g_error.c_str(); }

extern "C" int slora_version(void) { return 100; }

extern "C" slora_status slora_device_error(int clear) {
  using namespace slora;
  clear_error();
  const slora_status a = pack_check_error(clear != 0);
  const std::string first = a != SLORA_OK ? g_error : std::string();
  const slora_status b = tc_check_error(clear != 0);
  const std::string second = b != SLORA_OK ? g_error : std::string();
  const slora_status c = skinny_check_error(clear != 0);
  const std::string third = c != SLORA_OK ? g_error : std::string();
  const slora_status d = est_check_error(clear != 0);
  const std::string fourth = d != SLORA_OK ? g_error : std::string();
  const slora_status e = attn_check_error(clear != 0);
  if (a != SLORA_OK) g_error = first;
  else if (b != SLORA_OK) g_error = second;
  else if (c != SLORA_OK) g_error = third;
  else if (d != SLORA_OK) g_error = fourth;
  return a != SLORA_OK ? a : (b != SLORA_OK ? b : (c != SLORA_OK ? c : (d != SLORA_OK ? d : e)));
}

extern "C" slora_status slora_set_wait_budget(int64_t cycles) {
  slora::clear_error();
  return slora::skinny_set_wait_budget(static_cast<long long>(cycles));
}

// ------------------------------------------------------------ launch record
namespace slora {
namespace {
const char* kClassNames[kNumClasses] = {"gemm_tc", "gemm_simt", "estimate", "select",
                                        "elementwise", "aux", "prepare", "skinny", "compact",
                                        "attention", "norm"};
struct Rec {
  int cls;
  double work;
  cudaEvent_t a, b;
};
struct Profiler {
  std::mutex mu;
  int64_t launches = 0;
  bool on = false;
  std::vector<Rec> recs;        // events of the current record
  std::vector<cudaEvent_t> pool;  // free events
  cudaEvent_t get() {
    if (!pool.empty()) {
      cudaEvent_t e = pool.back();
      pool.pop_back();
      return e;
    }
    cudaEvent_t e = nullptr;
    if (cudaEventCreate(&e) != cudaSuccess) return nullptr;
    return e;
  }
  void release_all() {
    for (auto& r : recs) {
      if (r.a) pool.push_back(r.a);
      if (r.b) pool.push_back(r.b);
    }
    recs.clear();
  }
};
Profiler& prof() {
  static Profiler* p = new Profiler();
  return *p;
}
}  // namespace

LaunchScope::LaunchScope(int cls, double work, cudaStream_t st) : cls_(cls), st_(st), slot_(-1) {
  Profiler& p = prof();
  std::lock_guard<std::mutex> g(p.mu);
  ++p.launches;
  if (!p.on) return;
  Rec r{cls, work, p.get(), p.get()};
  if (r.a) cudaEventRecord(r.a, st);
  p.recs.push_back(r);
  slot_ = int(p.recs.size()) - 1;
}

LaunchScope::~LaunchScope() {
  if (slot_ < 0) return;
  Profiler& p = prof();
  std::lock_guard<std::mutex> g(p.mu);
  if (slot_ < int(p.recs.size()) && p.recs[slot_].b) cudaEventRecord(p.recs[slot_].b, st_);
}

}  // namespace slora

extern "C" int64_t slora_launch_count(void) { return slora::prof().launches; }

extern "C" void slora_profile_enable(int on) {
  slora::Profiler& p = slora::prof();
  std::lock_guard<std::mutex> g(p.mu);
  cudaDeviceSynchronize();
  p.release_all();
  p.on = on != 0;
}

extern "C" slora_status slora_profile_read(const char* kernel_class, int64_t* launches,
                                           double* total_ms, double* work) {
  using namespace slora;
  clear_error();
  int cls = -1;
  for (int i = 0; i < kNumClasses; ++i)
    if (kernel_class && std::string(kernel_class) == kClassNames[i]) cls = i;
  if (cls < 0) SLORA_FAIL(SLORA_ERR_INVALID_ARG, "unknown kernel class '%s'",
                          kernel_class ? kernel_class : "(null)");
  Profiler& p = prof();
  std::lock_guard<std::mutex> g(p.mu);
  int64_t n = 0;
  double ms = 0.0, w = 0.0;
  for (auto& r : p.recs) {
    if (r.cls != cls || !r.a || !r.b) continue;
    SLORA_CUDA(cudaEventSynchronize(r.b));
    float e = 0.0f;
    SLORA_CUDA(cudaEventElapsedTime(&e, r.a, r.b));
    ++n;
    ms += e;
    w += r.work;
  }
  if (launches) *launches = n;
  if (total_ms) *total_ms = ms;
  if (work) *work = w;
  return SLORA_OK;
}
