// Host-visible description of the streaming int4 GEMV kernels (decode path).
#pragma once
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

namespace coli {

// One launch of the gate/up (mode 0) or down+combine (mode 1) GEMV.
struct GemvParams {
    // layer shape
    int H, I, E, k, T, n_shared;
    // streamed matrices: rows x K int4 (+ fp16 scale per 64 of K)
    int K;          // input dim (H for gate/up, I for down)
    int N;          // rows per expert (I for gate/up, H for down)
    int U;          // 16-byte units per row = K / 32
    int rl;         // row lanes: active consumer threads / U (U >= 32) or consumers / U
    int SR;         // rows per pipeline stage = rl * RPT
    int NS;         // pipeline stages
    int resident;   // gate/up: the whole batch's x lives in shared memory
    int PR;         // max rows of one piece (one chunk's partials fit the buffer)
    uint32_t part_cap;  // floats in the partial-sum buffer
    uint32_t off_meta;  // chunk bookkeeping
    // shared-memory layout (bytes)
    uint32_t off_red, off_vec, off_stage;
    uint32_t vec_bytes;     // one vector buffer
    uint32_t stage_bytes;   // one stage
    uint32_t stage_sc_off;  // offset of the scale area inside a stage
    uint32_t sc_area;       // bytes of one matrix's scale area inside a stage
    // blob section offsets (bytes from the blob start) of the streamed matrices
    uint64_t q_off[2], s_off[2];
    // tensors (device)
    const uint8_t* experts;
    uint64_t stride;
    const uint8_t* shared;
    const float* x;           // gate/up: [T][H] fp32 activations
    const int32_t* union_ids; // [E]
    const int32_t* n_union;   // device scalar
    const int32_t* offsets;   // [E+1]
    const int32_t* assign;    // [T*k]
    const float* wts;         // [T][k] routing weights
    uint8_t* hd;              // SwiGLU activations h as digit records (workspace):
                              // row p (assign position, or T*k + t for the shared
                              // expert) holds I/32 records of kDigitRecBytes
    float* y;                 // [T][H] output
    const float* residual;    // [T][H] or null (down: y = residual + MoE)
    uint32_t* status;         // workspace header
    // x was complete before the preceding launch began (the layer call's router), so the
    // gate/up launch stages it and forms token 0's digits before waiting for that launch
    int x_early;
    // gate/up: x already in digit-record form ([T][H/32] records of kDigitRecBytes, written
    // by x_digits_launch before the preceding launch); read instead of x when set
    const uint8_t* xd;
};

// One 32-column unit of activations in digit form: three planes of 8 packed bytes, the
// three dp4a corrections and the scale factor (28 words).
constexpr int kDigitRecWords = 28;
constexpr int kDigitRecBytes = kDigitRecWords * 4;

struct GemvConfig {
    int maxm;         // tokens per chunk (register-resident activations)
    int consumers;    // consumer threads per CTA
    int rpt;          // rows per consumer thread per stage
    int lanes;        // butterfly width min(U, 32)
    size_t smem;      // dynamic shared memory
    int grid;
};

// Fills the layout fields of p and the launch configuration; returns false if the
// shape is not supported by the GEMV kernels.
bool gemv_plan(int mode, GemvParams& p, GemvConfig& c, int num_sms, size_t smem_limit);
cudaError_t gemv_launch(int mode, const GemvParams& p, const GemvConfig& c, cudaStream_t s);

// x [T][H] fp32 -> digit records rec [T][H/32] (one warp per 32-column unit).  The kernel
// lets the next launch start at once (programmatic dependent launch); that launch must
// wait for this grid before anything reads rec.
cudaError_t x_digits_launch(const float* x, int T, int H, uint8_t* rec, cudaStream_t s);

}  // namespace coli
