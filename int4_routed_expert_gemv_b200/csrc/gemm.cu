// Grouped tensor-core GEMM path for large batches (bf16 contract), sm_100a tcgen05.
//
// Prefill pushes thousands of tokens through one layer; the union then holds most experts
// with very uneven token counts (a few hot experts, a long tail of experts with a handful
// of tokens).  Each expert is a dense contraction over its tokens, so this path runs on
// the 5th-generation tensor cores:
//
//   phase 0 (gate/up): for every segment (shared expert, then the union in ascending
//       expert order) and every 128-row block of G and U:
//           Dg = G_blk . X_seg^T,  Du = U_blk . X_seg^T      [128 rows x N tokens]
//           h[token][row] = bf16( silu(Dg) * Du )
//   phase 1 (down): for every segment and 128-row block of D:
//           Dd = D_blk . (h_hi + h_lo)_seg^T,  y[token][row] += w_token * Dd   (fp32 atomics)
//
// The weights sit on the MMA's M side (128 rows) and the tokens on its N side, so a tail
// expert with 11 tokens costs a 16-column tile instead of a 128-row one.  bf16 contract:
// every weight is dequantised as bf16(q * scale) (q * scale is exact in fp32, then
// round-to-nearest-even), products accumulate in fp32 in tensor memory, and h enters the
// down projection as a pair of bf16 values hi = bf16(h), lo = bf16(h - hi) (about 16
// significant bits; the two halves' MMAs accumulate into the same tensor-memory tile), so
// no result depends on where a bf16 rounding of h falls.
//
// CTA (one per SM, persistent over a static share of the task list), 14 warps:
//   warps 0-3   epilogue: tcgen05.ld of the accumulators, SwiGLU or the weighted combine
//   warps 4-11  dequantisers: threads 2r and 2r+1 turn the two halves of row r of the raw
//               int4 tile (TMA-staged) into bf16, written 128B-swizzled into the A tile
//   warp 12     TMA producer: raw nibble rows (3-D tensor map over all experts) and the
//               token tiles (2-D tensor maps, 128B swizzle)
//   warp 13     TMEM allocator and single-thread tcgen05.mma issuer
// Accumulators are double-buffered in tensor memory so a task's epilogue overlaps the
// next task's MMAs.  Every mbarrier wait is bounded (DEV_TIMEOUT, then no more waiting).
#include <cuda.h>
#include <cudaTypedefs.h>
#include <string.h>

#include "common.cuh"
#include "gemm.cuh"

namespace coli {
namespace {

constexpr int kRows = 128;        // weight rows per tile (MMA M)
constexpr int kKc = 64;           // K per pipeline stage (one scale group)
constexpr int kStages = 3;
constexpr int kThreads = 448;
constexpr int kNmax0 = 128;       // tokens per task, gate/up (G and U accumulators)
constexpr int kNmax1 = 128;       // tokens per task, down (h as a hi + lo pair)
constexpr int kNumBoxes = 5;      // token-tile heights 16, 32, 64, 128, 256
constexpr uint32_t kWaitSite = 40;

struct Task {
    int seg;      // segment index (shared first)
    int tok0;     // first token of the segment in this task
    int ntok;     // tokens in this task (<= Nmax)
    int rb;       // 128-row block of the weight matrix
    int expert;   // the segment's expert, -1 for the shared expert
};

struct GemmParams {
    CUtensorMap raw[2][3];        // [routed, shared][G, U, D] int4 rows, box {32 B, 128, 1}
    CUtensorMap tok[2][kNumBoxes];// [phase][box]: x_g (phase 0) / h hi (phase 1), bf16, SW128
    CUtensorMap tok_lo[kNumBoxes];// h lo (phase 1)
    int H, I, E, k, T, n_shared;
    const int32_t* union_ids;
    const int32_t* n_union;
    const int32_t* offsets;
    const int32_t* assign;
    const float* w;
    const uint8_t* experts;
    uint64_t stride;
    const uint8_t* shared;
    __nv_bfloat16* h;             // [T*k + T][I]  bf16(h)
    __nv_bfloat16* h_lo;          // [T*k + T][I]  bf16(h - bf16(h))
    float* y;                     // [T][H]
    const Task* tasks;
    const int32_t* ntasks;
    uint32_t* status;
    int phase;
};

// ------------------------------------------------------------------------------------
// tcgen05 / TMA wrappers
// ------------------------------------------------------------------------------------
__device__ __forceinline__ void tma_load_3d(void* dst, const CUtensorMap* map, int x, int y, int z,
                                            uint64_t* bar)
{
    asm volatile(
        "cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%2, %3, %4}], [%5];" ::"r"(smem_u32(dst)),
        "l"(map), "r"(x), "r"(y), "r"(z), "r"(smem_u32(bar))
        : "memory");
}

__device__ __forceinline__ void tma_load_2d(void* dst, const CUtensorMap* map, int x, int y,
                                            uint64_t* bar)
{
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%2, %3}], [%4];" ::"r"(smem_u32(dst)),
        "l"(map), "r"(x), "r"(y), "r"(smem_u32(bar))
        : "memory");
}

__device__ __forceinline__ void tmem_alloc(uint32_t* dst_smem, uint32_t ncols)
{
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_u32(dst_smem)),
                 "r"(ncols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}

__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols)
{
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols)
                 : "memory");
}

// K-major operand tile, rows of 128 bytes, 128B swizzle, 8-row atoms 1024 bytes apart.
__device__ __forceinline__ uint64_t sw128_desc(const void* tile)
{
    const uint32_t a = smem_u32(tile);
    uint64_t d = 0;
    d |= (uint64_t)((a >> 4) & 0x3FFFu);          // start address
    d |= (uint64_t)1u << 16;                       // leading byte offset (unused for SW128 K-major)
    d |= (uint64_t)(1024u >> 4) << 32;             // stride byte offset: 8-row atoms
    d |= (uint64_t)1u << 46;                       // descriptor version
    d |= (uint64_t)2u << 61;                       // SWIZZLE_128B
    return d;
}

// kind::f16 instruction descriptor: bf16 A and B, fp32 D, both K-major, M x N.
__device__ __forceinline__ uint32_t idesc_bf16(int M, int N)
{
    return (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(N >> 3) << 17) |
           ((uint32_t)(M >> 4) << 24);
}

__device__ __forceinline__ void umma_bf16(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc,
                                          uint32_t idesc, uint32_t accumulate)
{
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, {%5, %6, %7, %8}, p;\n\t}" ::"r"(
            d_tmem),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate), "r"(0u), "r"(0u), "r"(0u), "r"(0u)
        : "memory");
}

__device__ __forceinline__ void umma_commit(uint64_t* bar)
{
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                     smem_u32(bar))
                 : "memory");
}

__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void fence_async_smem() { asm volatile("fence.proxy.async.shared::cta;" ::: "memory"); }

__device__ __forceinline__ void tmem_ld16(uint32_t taddr, uint32_t (&r)[16])
{
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
          "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
          "=r"(r[14]), "=r"(r[15])
        : "r"(taddr));
}

__device__ __forceinline__ void tmem_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi)
{
    uint32_t d;
    asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(d) : "f"(hi), "f"(lo));
    return d;
}

// 8 int4 values of one 32-bit word (nibble j = column j) -> bf16(q * s) in 4 packed pairs.
// A nibble lands in a float mantissa whose exponent gives its lowest bit the weight 1:
// (w & 0xF<<4j) ^ (exp_j | 8<<4j) equals 2^(23-4j) + q + 8 (two's-complement nibble,
// offset binary after the xor); subtracting 2^(23-4j) + 8 leaves q exactly.  Nibbles 5..7
// come from w >> 12.  q * s is exact in fp32 (4-bit times 11-bit); the pack rounds it to
// bf16, nearest-even.
__device__ __forceinline__ void dq8_bf16(uint32_t w, uint64_t sp, uint32_t (&out)[4])
{
    const uint32_t w2 = w >> 12;
    const uint64_t q01 = fadd2(pk2(and_xor(w, 0x0000000Fu, 0x4B000008u), and_xor(w, 0x000000F0u, 0x49000080u)),
                               pk2f(-8388616.0f, -524296.0f));
    const uint64_t q23 = fadd2(pk2(and_xor(w, 0x00000F00u, 0x47000800u), and_xor(w, 0x0000F000u, 0x45008000u)),
                               pk2f(-32776.0f, -2056.0f));
    const uint64_t q45 = fadd2(pk2(and_xor(w, 0x000F0000u, 0x43080000u), and_xor(w2, 0x00000F00u, 0x47000800u)),
                               pk2f(-136.0f, -32776.0f));
    const uint64_t q67 = fadd2(pk2(and_xor(w2, 0x0000F000u, 0x45008000u), and_xor(w2, 0x000F0000u, 0x43080000u)),
                               pk2f(-2056.0f, -136.0f));
    const uint64_t qs[4] = {q01, q23, q45, q67};
#pragma unroll
    for (int j = 0; j < 4; j++) {
        const float2 v = unpk2(fmul2(qs[j], sp));
        out[j] = pack_bf16x2(v.x, v.y);
    }
}

__device__ __forceinline__ int box_of(int ntok)
{
    return ntok <= 16 ? 0 : ntok <= 32 ? 1 : ntok <= 64 ? 2 : ntok <= 128 ? 3 : 4;
}

struct SegView {
    int expert;   // -1 for the shared expert
    int base;     // first row of x_g / h
    int count;
};

__device__ __forceinline__ SegView seg_view(const GemmParams& p, int s)
{
    SegView v;
    if (p.n_shared && s == 0) {
        v.expert = -1;
        v.base = p.T * p.k;
        v.count = p.T;
    } else {
        const int u = s - p.n_shared;
        v.expert = p.union_ids[u];
        v.base = p.offsets[u];
        v.count = p.offsets[u + 1] - v.base;
    }
    return v;
}

// ------------------------------------------------------------------------------------
// the grouped GEMM kernel (one phase per launch)
// ------------------------------------------------------------------------------------
__global__ void __launch_bounds__(kThreads, 1) grouped_gemm_kernel(const __grid_constant__ GemmParams p)
{
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    // 1024-aligned carve-up
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const int phase = p.phase;
    const int nmat = phase == 0 ? 2 : 1;
    const int nmax = phase == 0 ? kNmax0 : kNmax1;
    const uint32_t a_bytes = kRows * 128;                       // bf16 weight tile, one matrix
    const int ntt = phase == 0 ? 1 : 2;                         // token tiles (x, or h hi + lo)
    const uint32_t b_bytes = (uint32_t)ntt * nmax * 128;        // token tiles
    const uint32_t raw_bytes = kRows * 32;                      // int4 tile, one matrix
    const uint32_t stage_bytes = nmat * a_bytes + b_bytes + nmat * raw_bytes;
    uint8_t* stage0 = smem;
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kStages * stage_bytes);
    uint64_t* full_in = bars;                 // [kStages] raw + token bytes landed
    uint64_t* a_full = bars + kStages;        // [kStages] dequantised A tiles written
    uint64_t* empty = bars + 2 * kStages;     // [kStages] MMAs done with the stage
    uint64_t* acc_full = bars + 3 * kStages;  // [2]
    uint64_t* acc_empty = acc_full + 2;       // [2]
    uint64_t* mma_done = acc_empty + 2;       // [1] every MMA of the CTA has completed
    uint32_t* tmem_base_smem = reinterpret_cast<uint32_t*>(mma_done + 1);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int ntasks = *p.ntasks;
    const int K = phase == 0 ? p.H : p.I;      // contraction length
    const int kchunks = K / kKc;

    if (tid == 0) {
        for (int s = 0; s < kStages; s++) {
            mbar_init(&full_in[s], 1);
            mbar_init(&a_full[s], 8);          // one arrival per dequant warp
            mbar_init(&empty[s], 1);           // MMA commit
        }
        for (int b = 0; b < 2; b++) {
            mbar_init(&acc_full[b], 1);        // MMA commit
            mbar_init(&acc_empty[b], 4);       // one arrival per epilogue warp
        }
        mbar_init(mma_done, 1);
        fence_barrier_init();
    }
    if (warp == 13) tmem_alloc(tmem_base_smem, 512);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_base_smem;

    auto stage_ptr = [&](int s) { return stage0 + (size_t)s * stage_bytes; };
    // stage layout: A tiles (nmat x 16 KB) | token tile | raw tiles (nmat x 4 KB)
    bool dead = false;

    if (warp == 12) {
        // ---------------------------------- TMA producer ------------------------------
        if (lane == 0) {
            uint32_t it = 0;
            for (int t = blockIdx.x; t < ntasks; t += gridDim.x) {
                const Task tk = p.tasks[t];
                const SegView sv = seg_view(p, tk.seg);
                const int box = box_of(tk.ntok);
                const int boxrows = 16 << box;
                const CUtensorMap* tmap = &p.tok[phase][box];
                const int shared_seg = sv.expert < 0 ? 1 : 0;
                const int z = shared_seg ? 0 : sv.expert;
                for (int kc = 0; kc < kchunks; kc++, it++) {
                    const int s = it % kStages;
                    if (!dead && !mbar_wait(&empty[s], ((it / kStages) & 1) ^ 1, p.status, kWaitSite + 1))
                        dead = true;
                    if (dead) continue;
                    uint8_t* st = stage_ptr(s);
                    mbar_arrive_expect_tx(&full_in[s], nmat * raw_bytes + (uint32_t)(ntt * boxrows) * 128);
                    for (int mt = 0; mt < nmat; mt++) {
                        const int mat = phase == 0 ? mt : 2;
                        tma_load_3d(st + nmat * a_bytes + b_bytes + mt * raw_bytes,
                                    &p.raw[shared_seg][mat], kc * 32, tk.rb * kRows, z, &full_in[s]);
                    }
                    tma_load_2d(st + nmat * a_bytes, tmap, kc * kKc, sv.base + tk.tok0, &full_in[s]);
                    if (ntt == 2)
                        tma_load_2d(st + nmat * a_bytes + (uint32_t)nmax * 128, &p.tok_lo[box], kc * kKc,
                                    sv.base + tk.tok0, &full_in[s]);
                }
            }
            // drain
            const uint32_t n_issued = it < (uint32_t)kStages ? it : (uint32_t)kStages;
            for (uint32_t q = 0; q < n_issued; q++) {
                const uint32_t last = it - 1 - q;
                mbar_wait(&full_in[last % kStages], (last / kStages) & 1, p.status, kWaitSite + 2);
            }
        }
    } else if (warp >= 4 && warp < 12) {
        // ---------------------------------- dequantisers ------------------------------
        const int r = (tid - 128) >> 1;        // weight row within the 128-row tile
        const int half = (tid - 128) & 1;      // 16-byte chunks 4*half .. 4*half+3 of the row
        const uint64_t IH = (uint64_t)p.I * p.H;
        // this thread's row of fp16 scales for a task: K / 64 consecutive values, read 8 at a
        // time (16 bytes: the scales of 8 stages) one block ahead, across task boundaries
        auto scale_row = [&](const Task& tk, int mt) {
            const uint8_t* blob = tk.expert < 0 ? p.shared : p.experts + (uint64_t)tk.expert * p.stride;
            const uint64_t soff = phase == 0 ? (3 * IH / 2 + (uint64_t)mt * (IH / 32)) : (3 * IH / 2 + 2 * (IH / 32));
            return reinterpret_cast<const uint4*>(reinterpret_cast<const uint16_t*>(blob + soff) +
                                                  (size_t)(tk.rb * kRows + r) * (K / 64));
        };
        uint32_t it = 0;
        uint4 nb[2] = {make_uint4(0, 0, 0, 0), make_uint4(0, 0, 0, 0)};
        int t = blockIdx.x;
        Task tk{};
        if (t < ntasks) {
            tk = p.tasks[t];
            for (int mt = 0; mt < nmat; mt++) nb[mt] = __ldg(scale_row(tk, mt));
        }
        for (; t < ntasks; t += gridDim.x) {
            const int tn = t + gridDim.x;
            const Task tkn = tn < ntasks ? p.tasks[tn] : tk;       // issued early, used last
            for (int kb = 0; kb < kchunks; kb += 8) {
                const uint4 cb[2] = {nb[0], nb[1]};
                for (int mt = 0; mt < nmat; mt++) {
                    if (kb + 8 < kchunks) nb[mt] = __ldg(scale_row(tk, mt) + (kb + 8) / 8);
                    else if (tn < ntasks) nb[mt] = __ldg(scale_row(tkn, mt));
                }
#pragma unroll
                for (int j = 0; j < 8; j++, it++) {
                    const int s = it % kStages;
                    if (!dead && !mbar_wait(&full_in[s], (it / kStages) & 1, p.status, kWaitSite + 3))
                        dead = true;
                    uint8_t* st = stage_ptr(s);
#pragma unroll
                    for (int mt = 0; mt < 2; mt++) {
                        if (mt >= nmat) break;
                        const uint32_t cw[4] = {cb[mt].x, cb[mt].y, cb[mt].z, cb[mt].w};
                        const uint32_t w2 = cw[j >> 1];
                        const float sc = __half2float(__ushort_as_half((unsigned short)((j & 1) ? (w2 >> 16) : (w2 & 0xFFFFu))));
                        const uint64_t sp = pk2f(sc, sc);
                        const uint4 w0 = *reinterpret_cast<const uint4*>(st + nmat * a_bytes + b_bytes +
                                                                         mt * raw_bytes + r * 32 + half * 16);
                        const uint32_t words[4] = {w0.x, w0.y, w0.z, w0.w};
                        uint8_t* arow = st + mt * a_bytes + (r >> 3) * 1024 + (r & 7) * 128;
#pragma unroll
                        for (int c4 = 0; c4 < 4; c4++) {     // 16-byte chunk c = columns 8c .. 8c+7
                            const int c = 4 * half + c4;
                            uint32_t o[4];
                            dq8_bf16(words[c4], sp, o);
                            *reinterpret_cast<uint4*>(arow + ((c ^ (r & 7)) << 4)) =
                                make_uint4(o[0], o[1], o[2], o[3]);
                        }
                    }
                    fence_async_smem();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&a_full[s]);
                }
            }
            tk = tkn;
        }
    } else if (warp == 13) {
        // ---------------------------------- MMA issuer --------------------------------
        if (lane == 0) {
            uint32_t it = 0, tcount = 0;
            for (int t = blockIdx.x; t < ntasks; t += gridDim.x, tcount++) {
                const Task tk = p.tasks[t];
                const int boxrows = 16 << box_of(tk.ntok);
                const int buf = tcount & 1;
                if (!dead && !mbar_wait(&acc_empty[buf], ((tcount >> 1) & 1) ^ 1, p.status, kWaitSite + 4))
                    dead = true;
                tc_fence_after();
                const uint32_t idesc = idesc_bf16(kRows, boxrows);
                const uint32_t dcol = tmem + (uint32_t)buf * 256u;
                for (int kc = 0; kc < kchunks; kc++, it++) {
                    const int s = it % kStages;
                    const uint32_t par = (it / kStages) & 1;
                    if (!dead && !mbar_wait(&full_in[s], par, p.status, kWaitSite + 5)) dead = true;
                    if (!dead && !mbar_wait(&a_full[s], par, p.status, kWaitSite + 6)) dead = true;
                    tc_fence_after();
                    uint8_t* st = stage_ptr(s);
                    if (!dead) {
                        for (int tt = 0; tt < ntt; tt++) {
                            const uint64_t bdesc = sw128_desc(st + nmat * a_bytes + (uint32_t)tt * nmax * 128);
                            for (int mt = 0; mt < nmat; mt++) {
                                const uint64_t adesc = sw128_desc(st + mt * a_bytes);
#pragma unroll
                                for (int kk = 0; kk < kKc / 16; kk++)   // 16 bf16 = 32 bytes per MMA
                                    umma_bf16(dcol + (uint32_t)mt * 128u, adesc + (uint64_t)(2 * kk),
                                              bdesc + (uint64_t)(2 * kk), idesc, (kc | kk | tt) != 0);
                            }
                        }
                    }
                    umma_commit(&empty[s]);
                }
                umma_commit(&acc_full[buf]);
            }
            // tensor memory is released only after every MMA of this CTA has completed
            umma_commit(mma_done);
            mbar_wait(mma_done, 0, p.status, kWaitSite + 8);
        }
    } else if (warp < 4) {
        // ---------------------------------- epilogue ----------------------------------
        const int q = warp;                    // TMEM lane quarter
        const int row = q * 32 + lane;         // weight row within the tile
        uint32_t tcount = 0;
        for (int t = blockIdx.x; t < ntasks; t += gridDim.x, tcount++) {
            const Task tk = p.tasks[t];
            const SegView sv = seg_view(p, tk.seg);
            const int buf = tcount & 1;
            if (!dead && !mbar_wait(&acc_full[buf], (tcount >> 1) & 1, p.status, kWaitSite + 7))
                dead = true;
            tc_fence_after();
            const uint32_t lane_addr = tmem + ((uint32_t)(q * 32) << 16) + (uint32_t)buf * 256u;
            const int grow = tk.rb * kRows + row;   // row of the weight matrix
            for (int c0 = 0; c0 < tk.ntok; c0 += 16) {
                uint32_t g[16], u[16];
                tmem_ld16(lane_addr + (uint32_t)c0, g);
                if (phase == 0) tmem_ld16(lane_addr + 128u + (uint32_t)c0, u);
                const int nc = min(16, tk.ntok - c0);
                // phase 1: lane j < nc fetches token c0 + j's id and routing weight once
                int my_tok = 0;
                float my_w = 0.0f;
                if (phase == 1 && lane < nc) {
                    const int tt = tk.tok0 + c0 + lane;
                    if (sv.expert < 0) {
                        my_tok = tt;
                        my_w = 1.0f;
                    } else {
                        const int a = p.assign[sv.base + tt];
                        my_tok = a / p.k;
                        my_w = p.w[a];
                    }
                }
                tmem_wait_ld();
#pragma unroll
                for (int j = 0; j < 16; j++) {            // unrolled: g, u stay in registers
                    if (j >= nc) break;
                    const int tt = tk.tok0 + c0 + j;      // token index within the segment
                    if (phase == 0) {
                        const float gv = __uint_as_float(g[j]), uv = __uint_as_float(u[j]);
                        const float hv = gv / (1.0f + expf(-gv)) * uv;
                        const __nv_bfloat16 hh = __float2bfloat16_rn(hv);
                        const size_t o = (size_t)(sv.base + tt) * p.I + grow;
                        p.h[o] = hh;
                        p.h_lo[o] = __float2bfloat16_rn(hv - __bfloat162float(hh));
                    } else {
                        const int tok = __shfl_sync(0xffffffffu, my_tok, j);
                        const float wt = __shfl_sync(0xffffffffu, my_w, j);
                        atomicAdd(p.y + (size_t)tok * p.H + grow, wt * __uint_as_float(g[j]));
                    }
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&acc_empty[buf]);
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 13) {
        tc_fence_after();
        tmem_dealloc(tmem, 512);
    }
}

// ------------------------------------------------------------------------------------
// helpers: gather x rows into union order (+ y init), task planning
// ------------------------------------------------------------------------------------
__global__ void __launch_bounds__(256) gather_kernel(const __nv_bfloat16* __restrict__ x,
                                                     __nv_bfloat16* __restrict__ xg,
                                                     const int32_t* __restrict__ assign, int k, int T,
                                                     int n_shared, int H, const float* residual,
                                                     float* y)
{
    const int rows = T * k + T * n_shared;
    const int chunks = H / 8;              // 16-byte chunks per row
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < (int64_t)rows * chunks;
         i += (int64_t)gridDim.x * blockDim.x) {
        const int r = (int)(i / chunks), c = (int)(i - (int64_t)r * chunks);
        const int tok = r < T * k ? assign[r] / k : r - T * k;
        reinterpret_cast<uint4*>(xg + (size_t)r * H)[c] = reinterpret_cast<const uint4*>(x + (size_t)tok * H)[c];
    }
    const int ych = H / 4;
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < (int64_t)T * ych;
         i += (int64_t)gridDim.x * blockDim.x) {
        reinterpret_cast<float4*>(y)[i] =
            residual ? reinterpret_cast<const float4*>(residual)[i] : make_float4(0.f, 0.f, 0.f, 0.f);
    }
}

// Both phases' task lists, segment-major, then token chunks, then row blocks, so tasks
// that share a token tile run close together.  One CTA of 1024 threads: thread s counts the
// tasks of segment s, a block-wide exclusive scan places them, thread s writes them.
__global__ void __launch_bounds__(1024) plan_kernel(const int32_t* n_union, const int32_t* offsets,
                                                    const int32_t* union_ids,
                                                    int T, int k, int n_shared, int I, int H,
                                                    Task* tasks0, int32_t* ntasks0, Task* tasks1,
                                                    int32_t* ntasks1)
{
    __shared__ int wsum[2][32];
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int nseg = n_shared + *n_union;                    // <= 1025
    const int rb0 = I / kRows, rb1 = H / kRows;
    int base0 = 0, base1 = 0;
    for (int s0 = 0; s0 < nseg; s0 += 1024) {
        const int s = s0 + tid;
        int cnt = 0;
        if (s < nseg) cnt = (n_shared && s == 0) ? T : offsets[s - n_shared + 1] - offsets[s - n_shared];
        const int c0 = (cnt + kNmax0 - 1) / kNmax0 * rb0, c1 = (cnt + kNmax1 - 1) / kNmax1 * rb1;
        int x0 = c0, x1 = c1;                                 // inclusive warp scans
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int y0 = __shfl_up_sync(0xffffffffu, x0, o), y1 = __shfl_up_sync(0xffffffffu, x1, o);
            if (lane >= o) {
                x0 += y0;
                x1 += y1;
            }
        }
        if (lane == 31) {
            wsum[0][warp] = x0;
            wsum[1][warp] = x1;
        }
        __syncthreads();
        int p0 = base0, p1 = base1, tot0 = 0, tot1 = 0;
        for (int w2 = 0; w2 < 32; w2++) {
            if (w2 < warp) {
                p0 += wsum[0][w2];
                p1 += wsum[1][w2];
            }
            tot0 += wsum[0][w2];
            tot1 += wsum[1][w2];
        }
        p0 += x0 - c0;
        p1 += x1 - c1;
        if (s < nseg) {
            const int ex = (n_shared && s == 0) ? -1 : union_ids[s - n_shared];
            for (int t0 = 0; t0 < cnt; t0 += kNmax0)
                for (int rb = 0; rb < rb0; rb++) tasks0[p0++] = Task{s, t0, min(kNmax0, cnt - t0), rb, ex};
            for (int t0 = 0; t0 < cnt; t0 += kNmax1)
                for (int rb = 0; rb < rb1; rb++) tasks1[p1++] = Task{s, t0, min(kNmax1, cnt - t0), rb, ex};
        }
        base0 += tot0;
        base1 += tot1;
        __syncthreads();
    }
    if (tid == 0) {
        *ntasks0 = base0;
        *ntasks1 = base1;
    }
}

// ------------------------------------------------------------------------------------
// host side
// ------------------------------------------------------------------------------------
PFN_cuTensorMapEncodeTiled_v12000 encode_fn()
{
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    if (!fn) {
        cudaDriverEntryPointQueryResult q;
        void* ptr = nullptr;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
    }
    return fn;
}

bool make_raw_map(CUtensorMap* m, const void* base, uint64_t row_bytes, uint64_t rows, uint64_t nexp,
                  uint64_t exp_stride)
{
    auto enc = encode_fn();
    if (!enc) return false;
    cuuint64_t dims[3] = {row_bytes, rows, nexp};
    cuuint64_t strides[2] = {row_bytes, exp_stride};
    cuuint32_t box[3] = {32, (cuuint32_t)kRows, 1};
    cuuint32_t estr[3] = {1, 1, 1};
    return enc(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<void*>(base), dims, strides, box, estr,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
               CU_TENSOR_MAP_L2_PROMOTION_L2_128B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

bool make_tok_map(CUtensorMap* m, const void* base, uint64_t cols, uint64_t rows, int boxrows)
{
    auto enc = encode_fn();
    if (!enc) return false;
    cuuint64_t dims[2] = {cols, rows};
    cuuint64_t strides[1] = {cols * 2};
    cuuint32_t box[2] = {64, (cuuint32_t)boxrows};
    cuuint32_t estr[2] = {1, 1};
    return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
               CU_TENSOR_MAP_L2_PROMOTION_L2_128B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

struct Scratch {
    size_t xg, h, h_lo, tasks0, tasks1, counts, total;
};

Scratch scratch_layout(int H, int I, int E, int k, int n_shared, int64_t T)
{
    auto up = [](size_t v) { return (v + 1023) / 1024 * 1024; };
    Scratch s;
    const int64_t rows = T * (k + n_shared);
    size_t off = 0;
    s.xg = off;
    off = up(off + (size_t)rows * H * 2);
    s.h = off;
    off = up(off + (size_t)rows * I * 2);
    s.h_lo = off;
    off = up(off + (size_t)rows * I * 2);
    const int64_t segs = (int64_t)n_shared + (E < rows ? E : rows);
    const int64_t chunks0 = rows / kNmax0 + segs + 1, chunks1 = rows / kNmax1 + segs + 1;
    s.tasks0 = off;
    off = up(off + (size_t)chunks0 * (I / kRows) * sizeof(Task));
    s.tasks1 = off;
    off = up(off + (size_t)chunks1 * (H / kRows) * sizeof(Task));
    s.counts = off;
    off = up(off + 64);
    s.total = off;
    return s;
}

size_t gemm_smem(int phase)
{
    const int nmat = phase == 0 ? 2 : 1;
    const int nmax = phase == 0 ? kNmax0 : kNmax1;
    const int ntt = phase == 0 ? 1 : 2;
    const size_t stage = (size_t)nmat * kRows * 128 + (size_t)ntt * nmax * 128 + (size_t)nmat * kRows * 32;
    return 1024 + kStages * stage + 256;
}

}  // namespace

size_t gemm_workspace_bytes(int H, int I, int E, int k, int n_shared, int64_t T)
{
    return scratch_layout(H, I, E, k, n_shared, T).total;
}

bool gemm_supported(const GemmArgs& a)
{
    if (a.H % 512 || a.I % 512) return false;           // whole 8-group scale blocks, 128-row tiles
    if (a.H / kRows > 65535 || a.T > (1 << 24)) return false;
    if (!encode_fn()) return false;
    return gemm_smem(0) <= a.smem_optin && gemm_smem(1) <= a.smem_optin;
}

cudaError_t gemm_forward(const GemmArgs& a, cudaStream_t s)
{
    const Scratch L = scratch_layout(a.H, a.I, a.E, a.k, a.n_shared, a.T);
    uint8_t* base = a.scratch;
    __nv_bfloat16* xg = reinterpret_cast<__nv_bfloat16*>(base + L.xg);
    __nv_bfloat16* h = reinterpret_cast<__nv_bfloat16*>(base + L.h);
    __nv_bfloat16* h_lo = reinterpret_cast<__nv_bfloat16*>(base + L.h_lo);
    Task* tasks0 = reinterpret_cast<Task*>(base + L.tasks0);
    Task* tasks1 = reinterpret_cast<Task*>(base + L.tasks1);
    int32_t* counts = reinterpret_cast<int32_t*>(base + L.counts);
    const int64_t rows = (int64_t)a.T * (a.k + a.n_shared);

    GemmParams p;
    memset(&p, 0, sizeof(p));
    const uint64_t IH = (uint64_t)a.I * a.H;
    const uint8_t* sh = a.n_shared ? a.shared : a.experts;
    bool ok = true;
    // [routed, shared] x [G, U, D]
    ok &= make_raw_map(&p.raw[0][0], a.experts, a.H / 2, a.I, a.E, a.stride);
    ok &= make_raw_map(&p.raw[0][1], a.experts + IH / 2, a.H / 2, a.I, a.E, a.stride);
    ok &= make_raw_map(&p.raw[0][2], a.experts + IH, a.I / 2, a.H, a.E, a.stride);
    ok &= make_raw_map(&p.raw[1][0], sh, a.H / 2, a.I, 1, a.stride);
    ok &= make_raw_map(&p.raw[1][1], sh + IH / 2, a.H / 2, a.I, 1, a.stride);
    ok &= make_raw_map(&p.raw[1][2], sh + IH, a.I / 2, a.H, 1, a.stride);
    for (int b = 0; b < kNumBoxes; b++) {
        ok &= make_tok_map(&p.tok[0][b], xg, a.H, rows, 16 << b);
        ok &= make_tok_map(&p.tok[1][b], h, a.I, rows, 16 << b);
        ok &= make_tok_map(&p.tok_lo[b], h_lo, a.I, rows, 16 << b);
    }
    if (!ok) return cudaErrorInvalidValue;
    p.H = a.H;
    p.I = a.I;
    p.E = a.E;
    p.k = a.k;
    p.T = a.T;
    p.n_shared = a.n_shared;
    p.union_ids = a.union_ids;
    p.n_union = a.n_union;
    p.offsets = a.offsets;
    p.assign = a.assign;
    p.w = a.w;
    p.experts = a.experts;
    p.stride = a.stride;
    p.shared = a.shared;
    p.h = h;
    p.h_lo = h_lo;
    p.y = a.y;
    p.status = &a.hdr->status;

    gather_kernel<<<a.num_sms * 4, 256, 0, s>>>(a.x, xg, a.assign, a.k, a.T, a.n_shared, a.H,
                                                a.residual, a.y);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    plan_kernel<<<1, 1024, 0, s>>>(a.n_union, a.offsets, a.union_ids, a.T, a.k, a.n_shared, a.I, a.H, tasks0, counts,
                                 tasks1, counts + 1);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    for (int phase = 0; phase < 2; phase++) {
        p.phase = phase;
        p.tasks = phase == 0 ? tasks0 : tasks1;
        p.ntasks = counts + phase;
        const size_t smem = gemm_smem(phase);
        e = cudaFuncSetAttribute(grouped_gemm_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 (int)gemm_smem(1) > (int)gemm_smem(0) ? (int)gemm_smem(1) : (int)gemm_smem(0));
        if (e != cudaSuccess) return e;
        grouped_gemm_kernel<<<a.num_sms, kThreads, smem, s>>>(p);
        e = cudaGetLastError();
        if (e != cudaSuccess) return e;
    }
    return cudaSuccess;
}

}  // namespace coli
