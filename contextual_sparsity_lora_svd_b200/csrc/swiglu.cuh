#pragma once
#include "common.cuh"

namespace slora {
slora_status swiglu_fwd(const void* g, const void* u, void* h, int64_t count, int dt,
                        cudaStream_t st);
slora_status swiglu_bwd(const void* dh, const void* g, const void* u, void* dG, void* dU,
                        int64_t count, int dt, cudaStream_t st);
}  // namespace slora
