// Host entry of the tensor-core GEMV path (one or two tokens).
#pragma once
#include "common.cuh"

namespace gale {

constexpr int kMmaMaxTok = 2;

bool gemv_mma_supported(int cols, int ntok);
int launch_gemv_mma(const MatView& a, const MatView& b, bool swiglu, const float* x, int ntok, float* y,
                    cudaStream_t st);

}  // namespace gale
