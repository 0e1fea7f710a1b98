#pragma once
#include <cuda_runtime.h>

namespace coli {
cudaError_t rmsnorm_launch(int H, int T, const float* x, const float* gamma, double eps, float* out,
                           cudaStream_t s);
}
