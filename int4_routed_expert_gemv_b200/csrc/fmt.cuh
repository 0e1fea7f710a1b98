// Decode forward for the other weight containers: gs64 int8, per-row int4, gs64 int2 (and
// gs64 int4 through the same code, for comparison).
#pragma once
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

namespace coli {

enum WeightFmt : int { FMT_INT4_G64 = 0, FMT_INT8_G64 = 1, FMT_INT4_ROW = 2, FMT_INT2_G64 = 3 };

constexpr int kFmtMaxT = 4;   // tokens per call

// Bytes of one expert blob in container fmt (0 for an unknown fmt).
size_t fmt_blob_bytes(int H, int I, int fmt);

struct FmtParams {
    int H, I, E, k, T, n_shared, fmt;
    const uint8_t* experts;
    uint64_t stride;
    const uint8_t* shared;
    const float* x;            // [T][H]
    const float* w;            // [T][k] routing weights
    const int32_t* union_ids;  // [E]
    const int32_t* n_union;    // device scalar
    const int32_t* offsets;    // [E+1]
    const int32_t* assign;     // [T*k]
    float* h;                  // [T*(k+n_shared)][I] workspace
    const float* residual;     // [T][H] or null
    float* y;                  // [T][H]
    uint32_t* status;
};

// Plans and enqueues the two launches (gate/up + SwiGLU, then down + combine).
cudaError_t fmt_forward_launch(const FmtParams& p, int num_sms, cudaStream_t s);

}  // namespace coli
