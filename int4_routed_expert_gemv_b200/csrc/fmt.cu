// Decode forward (T <= 4 tokens, fp32 activations) for the weight containers of the
// engine's other quantised kernels: gs64 int8, per-row int4 and gs64 int2, next to the
// gs64 int4 container (colibri README.zh-CN, "开始使用 / 2. 获取模型"; the technical
// article's "精度与语义" section).  Blob: Gq | Uq | Dq | Gs | Us | Ds as for gs64 int4,
// with b-bit two's-complement payload (lowest-index column in the lowest bits) and fp16
// scales per 64 input columns, or one per row for the per-row container.
//
// Two launches, CUDA-core arithmetic (the byte count of the container sets the speed):
//   gate/up: a persistent grid over (segment, block of 8 rows) tasks; a warp takes one row
//     of G and the same row of U, streams both in 16-byte loads, applies the scale once per
//     16-byte chunk and reduces with shuffles; h = silu(g) * u into the workspace;
//   down: a block owns 32 output rows; for every segment in union order (shared expert
//     first) it stages the segment's h rows in shared memory and adds the routing-weighted
//     dot products into per-row accumulators, so y has one fixed summation order.
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "common.cuh"
#include "fmt.cuh"

namespace coli {
namespace {

constexpr int kFmtWarps = 8;
constexpr int kFmtThreads = 32 * kFmtWarps;
constexpr int kDownRowsPerWarp = 4;

template <int FMT>
struct Fmt {
    static constexpr int bits = FMT == FMT_INT8_G64 ? 8 : FMT == FMT_INT2_G64 ? 2 : 4;
    static constexpr int per_word = 32 / bits;      // values in a 32-bit word
    static constexpr int per_chunk = 4 * per_word;  // values in a 16-byte chunk
    static constexpr bool per_row = FMT == FMT_INT4_ROW;
    // activations in shared memory: the per_chunk values of a chunk, then 4 floats of
    // padding, so that the lanes (one chunk each) read 16 bytes from distinct banks
    static constexpr int pad_chunk = per_chunk + 4;
};

// floats of one activation row of `n` values in the padded layout
template <int FMT>
__host__ __device__ constexpr int padded_row(int n) { return n / Fmt<FMT>::per_chunk * Fmt<FMT>::pad_chunk; }

__host__ __device__ inline int fmt_bits(int fmt) { return fmt == FMT_INT8_G64 ? 8 : fmt == FMT_INT2_G64 ? 2 : 4; }
__host__ __device__ inline int64_t scales_per_row(int fmt, int64_t in_dim) { return fmt == FMT_INT4_ROW ? 1 : in_dim / 64; }

struct FmtBlob {
    uint64_t gq, uq, dq, gs, us, ds;
};

__host__ __device__ inline FmtBlob fmt_blob(int H, int I, int fmt)
{
    const uint64_t q = (uint64_t)I * H * fmt_bits(fmt) / 8;
    FmtBlob b;
    b.gq = 0;
    b.uq = q;
    b.dq = 2 * q;
    b.gs = 3 * q;
    b.us = b.gs + (uint64_t)I * scales_per_row(fmt, H) * 2;
    b.ds = b.us + (uint64_t)I * scales_per_row(fmt, H) * 2;
    return b;
}

// value j (0 <= j < per_word) of a word as a float: the field read as an offset-binary
// code (two's complement with the sign bit flipped) inside the mantissa of 2^23, minus
// 2^23 and the offset (exact; full-rate integer and float operations only)
template <int FMT>
__device__ __forceinline__ float field_f(uint32_t w, int j)
{
    constexpr int b = Fmt<FMT>::bits;
    constexpr uint32_t mask = (1u << b) - 1u, sign = 1u << (b - 1);
    const uint32_t u = ((w >> (b * j)) & mask) ^ (sign | 0x4B000000u);
    return __uint_as_float(u) - (8388608.0f + (float)sign);
}

// sum_v q_v * act_v over one 16-byte chunk, for up to kFmtMaxT activation rows (padded
// layout in shared memory; row r of chunk ch at act + r * row_floats + ch * pad_chunk)
template <int FMT>
__device__ __forceinline__ void chunk_dot(const uint4& wv, const float* act, int row_floats, int ch, int cnt,
                                          const int (&tok)[kFmtMaxT], float (&acc)[kFmtMaxT])
{
    const uint32_t words[4] = {wv.x, wv.y, wv.z, wv.w};
#pragma unroll
    for (int wi = 0; wi < 4; wi++) {
        float v[Fmt<FMT>::per_word];
#pragma unroll
        for (int j = 0; j < Fmt<FMT>::per_word; j++) v[j] = field_f<FMT>(words[wi], j);
#pragma unroll
        for (int m = 0; m < kFmtMaxT; m++) {
            if (m < cnt) {
                const float4* xr = reinterpret_cast<const float4*>(act + (size_t)tok[m] * row_floats +
                                                                    ch * Fmt<FMT>::pad_chunk + wi * Fmt<FMT>::per_word);
                float a = acc[m];
#pragma unroll
                for (int q = 0; q < Fmt<FMT>::per_word / 4; q++) {
                    const float4 x4 = xr[q];
                    a = fmaf(v[4 * q], x4.x, a);
                    a = fmaf(v[4 * q + 1], x4.y, a);
                    a = fmaf(v[4 * q + 2], x4.z, a);
                    a = fmaf(v[4 * q + 3], x4.w, a);
                }
                acc[m] = a;
            }
        }
    }
}

// stage `rows` activation rows of n values (global, consecutive rows n apart) into the
// padded shared-memory layout
template <int FMT>
__device__ __forceinline__ void stage_padded(float* dst, const float* src, int rows, int n, bool stream)
{
    constexpr int pc = Fmt<FMT>::per_chunk;
    const int n4 = n / 4, total = rows * n4;
    for (int i = threadIdx.x; i < total; i += blockDim.x) {
        const int r = i / n4, c4 = i - r * n4, col = 4 * c4;
        const float4 v = stream ? __ldcg(reinterpret_cast<const float4*>(src) + i)
                                : __ldg(reinterpret_cast<const float4*>(src) + i);
        *reinterpret_cast<float4*>(dst + (size_t)r * padded_row<FMT>(n) + (col / pc) * Fmt<FMT>::pad_chunk + col % pc) = v;
    }
}

__device__ __forceinline__ float warp_sum(float v)
{
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

// the tokens of segment seg (shared expert first, then the union in order): their count,
// token ids, routing weights and first h row
__device__ __forceinline__ int seg_tokens(const FmtParams& p, int seg, int (&tok)[kFmtMaxT], float (&wt)[kFmtMaxT],
                                          int& hbase, const uint8_t*& blob)
{
    if (seg < p.n_shared) {
#pragma unroll
        for (int m = 0; m < kFmtMaxT; m++) {
            tok[m] = m < p.T ? m : 0;
            wt[m] = 1.0f;
        }
        hbase = p.T * p.k;
        blob = p.shared;
        return p.T;
    }
    const int u = seg - p.n_shared;
    const int o0 = __ldg(p.offsets + u), o1 = __ldg(p.offsets + u + 1);
    const int cnt = min(max(o1 - o0, 0), p.T);
#pragma unroll
    for (int m = 0; m < kFmtMaxT; m++) {
        const int a = m < cnt ? __ldg(p.assign + o0 + m) : 0;
        tok[m] = a / p.k;
        wt[m] = m < cnt ? __ldg(p.w + a) : 0.0f;
    }
    hbase = o0;
    blob = p.experts + (uint64_t)__ldg(p.union_ids + u) * p.stride;
    return cnt;
}

template <int FMT>
__global__ void __launch_bounds__(kFmtThreads) fmt_gate_up_kernel(const __grid_constant__ FmtParams p)
{
    extern __shared__ __align__(16) float xs[];   // [T] padded rows of x
    const int H = p.H, I = p.I, lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    stage_padded<FMT>(xs, p.x, p.T, H, false);
    __syncthreads();
    const int nu = *reinterpret_cast<const volatile int32_t*>(p.n_union);
    const int nseg = p.n_shared + nu;
    const int rb_n = (I + kFmtWarps - 1) / kFmtWarps;
    const FmtBlob bo = fmt_blob(H, I, FMT);
    const int row_bytes = H * Fmt<FMT>::bits / 8, nchunk = row_bytes / 16, spr = Fmt<FMT>::per_row ? 1 : H / 64;
    for (int task = blockIdx.x; task < nseg * rb_n; task += gridDim.x) {
        const int seg = task / rb_n, row = (task - seg * rb_n) * kFmtWarps + warp;
        if (row >= I) continue;
        int tok[kFmtMaxT];
        float wt[kFmtMaxT];
        int hbase;
        const uint8_t* blob;
        const int cnt = seg_tokens(p, seg, tok, wt, hbase, blob);
        const uint4* gr = reinterpret_cast<const uint4*>(blob + bo.gq + (uint64_t)row * row_bytes);
        const uint4* ur = reinterpret_cast<const uint4*>(blob + bo.uq + (uint64_t)row * row_bytes);
        const __half* gsc = reinterpret_cast<const __half*>(blob + bo.gs) + (uint64_t)row * spr;
        const __half* usc = reinterpret_cast<const __half*>(blob + bo.us) + (uint64_t)row * spr;
        float g[kFmtMaxT] = {0.f, 0.f, 0.f, 0.f}, u[kFmtMaxT] = {0.f, 0.f, 0.f, 0.f};
        for (int ch = lane; ch < nchunk; ch += 32) {
            const uint4 gw = __ldcs(gr + ch), uw = __ldcs(ur + ch);
            const int col = ch * Fmt<FMT>::per_chunk;
            const float sg = __half2float(gsc[Fmt<FMT>::per_row ? 0 : col / 64]);
            const float su = __half2float(usc[Fmt<FMT>::per_row ? 0 : col / 64]);
            float ag[kFmtMaxT] = {0.f, 0.f, 0.f, 0.f}, au[kFmtMaxT] = {0.f, 0.f, 0.f, 0.f};
            chunk_dot<FMT>(gw, xs, padded_row<FMT>(H), ch, cnt, tok, ag);
            chunk_dot<FMT>(uw, xs, padded_row<FMT>(H), ch, cnt, tok, au);
#pragma unroll
            for (int m = 0; m < kFmtMaxT; m++) {
                g[m] = fmaf(ag[m], sg, g[m]);
                u[m] = fmaf(au[m], su, u[m]);
            }
        }
#pragma unroll
        for (int m = 0; m < kFmtMaxT; m++) {
            const float gs = warp_sum(g[m]), us = warp_sum(u[m]);
            if (m < cnt && lane == 0) p.h[(size_t)(hbase + m) * I + row] = gs / (1.0f + expf(-gs)) * us;
        }
    }
}

template <int FMT>
__global__ void __launch_bounds__(kFmtThreads) fmt_down_kernel(const __grid_constant__ FmtParams p)
{
    extern __shared__ __align__(16) float hs[];   // one segment's h rows, padded
    const int H = p.H, I = p.I, lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int nu = *reinterpret_cast<const volatile int32_t*>(p.n_union);
    const int nseg = p.n_shared + nu;
    const FmtBlob bo = fmt_blob(H, I, FMT);
    const int row_bytes = I * Fmt<FMT>::bits / 8, nchunk = row_bytes / 16, spr = Fmt<FMT>::per_row ? 1 : I / 64;
    const int r0 = (blockIdx.x * kFmtWarps + warp) * kDownRowsPerWarp;
    float acc[kDownRowsPerWarp][kFmtMaxT];
#pragma unroll
    for (int rr = 0; rr < kDownRowsPerWarp; rr++)
#pragma unroll
        for (int m = 0; m < kFmtMaxT; m++) acc[rr][m] = 0.0f;
    for (int seg = 0; seg < nseg; seg++) {
        int tok[kFmtMaxT];
        float wt[kFmtMaxT];
        int hbase;
        const uint8_t* blob;
        const int cnt = seg_tokens(p, seg, tok, wt, hbase, blob);
        __syncthreads();
        stage_padded<FMT>(hs, p.h + (size_t)hbase * I, cnt, I, true);
        __syncthreads();
        int ident[kFmtMaxT];
#pragma unroll
        for (int m = 0; m < kFmtMaxT; m++) ident[m] = m;
#pragma unroll
        for (int rr = 0; rr < kDownRowsPerWarp; rr++) {
            const int row = r0 + rr;
            if (row >= H) continue;
            const uint4* dr = reinterpret_cast<const uint4*>(blob + bo.dq + (uint64_t)row * row_bytes);
            const __half* dsc = reinterpret_cast<const __half*>(blob + bo.ds) + (uint64_t)row * spr;
            float d[kFmtMaxT] = {0.f, 0.f, 0.f, 0.f};
            for (int ch = lane; ch < nchunk; ch += 32) {
                const uint4 dw = __ldcs(dr + ch);
                const int col = ch * Fmt<FMT>::per_chunk;
                const float sd = __half2float(dsc[Fmt<FMT>::per_row ? 0 : col / 64]);
                float a[kFmtMaxT] = {0.f, 0.f, 0.f, 0.f};
                chunk_dot<FMT>(dw, hs, padded_row<FMT>(I), ch, cnt, ident, a);
#pragma unroll
                for (int m = 0; m < kFmtMaxT; m++) d[m] = fmaf(a[m], sd, d[m]);
            }
#pragma unroll
            for (int m = 0; m < kFmtMaxT; m++) {
                const float v = warp_sum(d[m]);
                if (m < cnt) {
                    // the token of this h row, by a select over the (few) tokens
#pragma unroll
                    for (int t = 0; t < kFmtMaxT; t++)
                        if (t == tok[m]) acc[rr][t] = fmaf(wt[m], v, acc[rr][t]);
                }
            }
        }
    }
    if (lane == 0)
#pragma unroll
        for (int rr = 0; rr < kDownRowsPerWarp; rr++) {
            const int row = r0 + rr;
            if (row >= H) continue;
            for (int t = 0; t < p.T; t++) {
                const float base = p.residual ? p.residual[(size_t)t * H + row] : 0.0f;
                p.y[(size_t)t * H + row] = base + acc[rr][t];
            }
        }
}

template <int FMT>
cudaError_t launch_fmt(const FmtParams& p, int num_sms, cudaStream_t s)
{
    const size_t sx = (size_t)p.T * padded_row<FMT>(p.H) * 4, sh = (size_t)p.T * padded_row<FMT>(p.I) * 4;
    cudaError_t e = cudaFuncSetAttribute(fmt_gate_up_kernel<FMT>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sx);
    if (e != cudaSuccess) return e;
    e = cudaFuncSetAttribute(fmt_down_kernel<FMT>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sh);
    if (e != cudaSuccess) return e;
    fmt_gate_up_kernel<FMT><<<2 * num_sms, kFmtThreads, sx, s>>>(p);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    const int rows_per_block = kFmtWarps * kDownRowsPerWarp;
    fmt_down_kernel<FMT><<<(p.H + rows_per_block - 1) / rows_per_block, kFmtThreads, sh, s>>>(p);
    return cudaGetLastError();
}

}  // namespace

size_t fmt_blob_bytes(int H, int I, int fmt)
{
    if (fmt < FMT_INT4_G64 || fmt > FMT_INT2_G64) return 0;
    const FmtBlob b = fmt_blob(H, I, fmt);
    return (size_t)(b.ds + (uint64_t)H * scales_per_row(fmt, I) * 2);
}

cudaError_t fmt_forward_launch(const FmtParams& p, int num_sms, cudaStream_t s)
{
    switch (p.fmt) {
    case FMT_INT4_G64: return launch_fmt<FMT_INT4_G64>(p, num_sms, s);
    case FMT_INT8_G64: return launch_fmt<FMT_INT8_G64>(p, num_sms, s);
    case FMT_INT4_ROW: return launch_fmt<FMT_INT4_ROW>(p, num_sms, s);
    case FMT_INT2_G64: return launch_fmt<FMT_INT2_G64>(p, num_sms, s);
    default: return cudaErrorInvalidValue;
    }
}

}  // namespace coli
