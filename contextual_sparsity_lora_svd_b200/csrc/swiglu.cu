// SwiGLU elementwise forward / backward on compact [rows x cols] matrices.
//   forward : h = silu(g) * u
//   backward: dG = dh * u * sigmoid(g) * (1 + g (1 - sigmoid(g))),  dU = dh * silu(g)
// The backward may run in place on dh (dG overwrites it).
#include "swiglu.cuh"

namespace slora {
namespace {

__global__ void swiglu_fwd_kernel(const void* __restrict__ g, const void* __restrict__ u,
                                  void* __restrict__ h, int64_t count, int dt) {
  for (int64_t i = int64_t(blockIdx.x) * blockDim.x + threadIdx.x; i < count;
       i += int64_t(gridDim.x) * blockDim.x) {
    float gv = ld_elem(g, i, dt), uv = ld_elem(u, i, dt);
    st_elem(h, i, dt, silu_f(gv) * uv);
  }
}

__global__ void swiglu_bwd_kernel(const void* dh, const void* __restrict__ g,
                                  const void* __restrict__ u, void* dG, void* dU, int64_t count,
                                  int dt) {
  for (int64_t i = int64_t(blockIdx.x) * blockDim.x + threadIdx.x; i < count;
       i += int64_t(gridDim.x) * blockDim.x) {
    float dhv = ld_elem(dh, i, dt), gv = ld_elem(g, i, dt), uv = ld_elem(u, i, dt);
    float sg = sigmoid_f(gv);
    float dgv = dhv * uv * sg * (1.0f + gv * (1.0f - sg));
    float duv = dhv * gv * sg;
    st_elem(dG, i, dt, dgv);
    st_elem(dU, i, dt, duv);
  }
}

unsigned grid_for(int64_t count) {
  int64_t b = (count + 255) / 256;
  if (b > 148 * 16) b = 148 * 16;
  if (b < 1) b = 1;
  return unsigned(b);
}
}  // namespace

slora_status swiglu_fwd(const void* g, const void* u, void* h, int64_t count, int dt,
                        cudaStream_t st) {
  if (count <= 0) return SLORA_OK;
  LaunchScope ls(kElementwise, double(count) * 3 * dt_size(dt), st);
  swiglu_fwd_kernel<<<grid_for(count), 256, 0, st>>>(g, u, h, count, dt);
  SLORA_CHECK_LAUNCH();
  return SLORA_OK;
}

slora_status swiglu_bwd(const void* dh, const void* g, const void* u, void* dG, void* dU,
                        int64_t count, int dt, cudaStream_t st) {
  if (count <= 0) return SLORA_OK;
  LaunchScope ls(kElementwise, double(count) * 5 * dt_size(dt), st);
  swiglu_bwd_kernel<<<grid_for(count), 256, 0, st>>>(dh, g, u, dG, dU, count, dt);
  SLORA_CHECK_LAUNCH();
  return SLORA_OK;
}

}  // namespace slora
