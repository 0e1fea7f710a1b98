// Host-visible description of the grouped tensor-core GEMM path (bf16 contract).
#pragma once
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "common.cuh"

namespace coli {

struct GemmArgs {
    int H, I, E, k, T, n_shared;
    const uint8_t* experts;
    uint64_t stride;
    const uint8_t* shared;
    const __nv_bfloat16* x;     // [T][H]
    const float* w;             // [T][k]
    const int32_t* union_ids;
    const int32_t* n_union;
    const int32_t* offsets;
    const int32_t* assign;
    const float* residual;      // [T][H] or null
    float* y;                   // [T][H]
    uint8_t* scratch;           // gemm_workspace_bytes() bytes
    WsHeader* hdr;
    int num_sms;
    size_t smem_optin;
};

size_t gemm_workspace_bytes(int H, int I, int E, int k, int n_shared, int64_t T);
bool gemm_supported(const GemmArgs& a);
cudaError_t gemm_forward(const GemmArgs& a, cudaStream_t s);

}  // namespace coli
