// GEMM entry used by the launch sequences.  fp32 problems and the small or
// skinny contractions run on the CUDA-core gathered GEMM; the large bf16
// sliced contractions run on the tcgen05 kernel.
#pragma once
#include "gemm_simt.cuh"

namespace slora {
slora_status gemm(const GemmArgs& g, cudaStream_t st);
}  // namespace slora
