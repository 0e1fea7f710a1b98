// Grouped tensor-core GEMM path (bf16 contract): placeholder until the tcgen05 kernels land.
#include "gemm.cuh"

namespace coli {

size_t gemm_workspace_bytes(int, int, int, int, int, int64_t) { return 0; }
bool gemm_supported(const GemmArgs&) { return false; }
cudaError_t gemm_forward(const GemmArgs&, cudaStream_t) { return cudaErrorNotSupported; }

}  // namespace coli
