// Host-visible description of the router, top-k and union kernels.
#pragma once
#include <cuda_runtime.h>
#include <stdint.h>

#include "common.cuh"

namespace coli {

constexpr int kMaxExperts = 1024;   // E limit of the top-k and union kernels
constexpr int kMaxTopK = 32;        // one warp lane per selected slot
constexpr int kSmallT = 8;          // batches up to this size use the fused small router

struct RouteParams {
    int H, E, k, T;
    const void* x;            // [T][H] fp32 or bf16
    int x_bf16;
    const float* w_router;    // [E][H]
    const float* bias;        // [E] or null
    float* logits;            // [T][E]
    int32_t* idx;             // [T][k]
    float* w;                 // [T][k]
    int do_topk;              // also select top-k (otherwise logits only)
    int do_union;             // also build the batch union (implies do_topk)
    int32_t* union_ids;       // [E]
    int32_t* n_union;         // device scalar
    int32_t* offsets;         // [E+1]
    int32_t* assign;          // [T*k]
    WsHeader* hdr;
    uint32_t* status;         // == &hdr->status
    // batches up to kSmallT: launch as a programmatic dependent of the previous kernel (which
    // the router does not read); the grid waits for it before completing, so a launch that
    // waits for the router also sees everything that kernel wrote
    int pdl;
};

cudaError_t route_launch(const RouteParams& p, cudaStream_t s);
cudaError_t union_launch(const RouteParams& p, cudaStream_t s);

}  // namespace coli
