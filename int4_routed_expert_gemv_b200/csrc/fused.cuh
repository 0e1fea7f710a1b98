// Host-visible description of the fused decode kernel: one persistent launch runs whole
// MoE layers (RMSNorm, router, top-k, union, gate/up + SwiGLU, down + combine) for a
// decode batch of up to kFusedMaxT tokens, optionally several layers of a residual stack.
#pragma once
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "common.cuh"

namespace coli {

constexpr int kFusedMaxT = 4;          // tokens per call
constexpr int kFusedMaxLayers = 16;    // layers per launch (longer stacks: several launches)
constexpr int kFusedMaxK = 32;
constexpr int kFusedMaxSeg = 1 + kFusedMaxT * kFusedMaxK;   // shared expert + union entries
// counters: word 0 = exit ticket; then per layer kCntPerLayer words:
//   [0] unused, [1] CTAs that wrote their rows of the layer output,
//   [2 + s] gate/up stages finished of segment s
constexpr int kCntPerLayer = 2 + kFusedMaxSeg;
constexpr int kCntWords = 1 + kFusedMaxLayers * kCntPerLayer;

// Bytes of one digit row of h (I values): three planes of I digit bytes, then one
// (m / 126, epoch) word pair per 64-value group; a multiple of 16.
__host__ __device__ constexpr size_t hdg_row_bytes(int I)
{
    return ((size_t)(3 * I + 8 * (I / 64)) + 15) / 16 * 16;
}

struct FusedLayer {
    const float* w_router;   // [E][H]
    const float* bias;       // [E] or null
    const uint8_t* experts;  // E blobs at `stride`
    const uint8_t* shared;   // one blob or null
    const float* gamma;      // RMSNorm weight [H] or null (1.0)
    uint64_t stride;         // bytes from one expert blob to the next
};

struct FusedParams {
    // shape
    int H, I, E, k, T, n_shared, L;
    FusedLayer layer[kFusedMaxLayers];
    // mode
    int route;          // 1: routing computed in the launch; 0: routing given (inputs below)
    int norm;           // apply RMSNorm to every layer input (residual stack)
    double eps;
    // activations
    const float* x;          // [T][H] input of the first layer
    const float* residual;   // one-layer calls: y = residual + MoE(x) (null: 0); stacks use
                             // each layer's input as its residual
    float* y;                // [T][H] output of the last layer (may alias residual)
    float* xbuf;             // [2][T][H] outputs of intermediate layers (workspace)
    // routing of a one-layer call: outputs when route == 1, inputs when route == 0
    int32_t* idx;            // [T][k]
    float* w;                // [T][k]
    float* logits;           // [T][E] or null
    int32_t* union_ids;      // [E]
    int32_t* n_union;        // device scalar
    int32_t* offsets;        // [E+1]
    int32_t* assign;         // [T*k]
    int32_t* idx_layers;     // stacks: [L][T][k] selections of every layer, or null
    // workspace
    uint32_t* status;        // header status word (timeout site at status + 3)
    uint32_t* gen;           // header launch generation (epochs of h)
    uint32_t* cnt;           // kCntWords counters, zero between launches
    uint4* rpart;            // [T][E][RC] router partial sums: (low word, epoch, high word, epoch)
    uint2* h;                // [T*(k+n_shared)][I] SwiGLU activations as (value, epoch)
    uint8_t* hdg;            // per h row its digit row (3 planes of I bytes, then
                             // (m / 126, epoch) per 64-value group), hdg_row bytes apart
    uint32_t hdg_row;
    // plan (fused_plan)
    int grid, nslot;
    uint32_t slot_bytes;
    size_t smem;
    int NT;                  // MMA column tiles (pairs of tokens)
    int pair;                // one token: gate/up runs on pairs of 64-column groups
    int RC, RKc;             // router: column chunks per row and their width
    int KWg, RSg, GPWg, NTSg, SPS;   // gate/up: K-split warps, row slots, groups of the
                                     // widest warp, row tiles per stage, stages per segment
    int KWd, RSd, GPWd;              // down: K-split warps, row slots, groups per warp
    int rows_max, ntdm;              // down rows per CTA (at most) and their row tiles
    uint32_t gu_chunk, gu_gsc, gu_usc;   // gate/up stage: chunk stride, scale areas
    uint32_t d_chunk, d_sc_off;          // down stage: chunk stride, scale area
    uint32_t red_floats;                 // one partial-sum buffer
    uint32_t off_hdig, hdig_bytes;       // pair mode: kDigBufs copies of digit rows
    uint32_t off_hstage;                 // pair mode: the layer input row
    uint32_t off_red, off_yacc, off_scratch, off_ring;   // dynamic shared memory layout
};

// Fills the plan fields; false if the shape or batch is outside what the kernel handles.
bool fused_plan(FusedParams& p, int num_sms, size_t smem_limit);
cudaError_t fused_launch(const FusedParams& p, cudaStream_t s);

}  // namespace coli
