// Batch union of the selected experts, as a block-wide device routine.
//
// "Batch positions read each distinct expert once" (colibri README.zh-CN,
// "工作原理 / 绝不为同一次磁盘读取等待两遍", 批量并集).  Given idx [T][k], produce
//   union_ids [E]   distinct expert ids in ascending order, then -1
//   n_union         number of distinct ids
//   offsets [E+1]   start of each union entry's list in assign; T*k from n_union on
//   assign [T*k]    for each union entry, the flat positions t*k+slot that chose it,
//                   in ascending order
// It is a stable counting sort by expert id: counts -> exclusive scans -> ranks.  The
// rank of a position among equal ids comes from __match_any_sync inside a warp plus the
// counts of earlier warps and earlier chunks, so the output is deterministic and needs no
// ordering of atomics.
#pragma once
#include "common.cuh"

namespace coli {

// Shared memory needed by union_block for E experts and nwarps warps.
__host__ __device__ inline size_t union_smem_bytes(int E, int nwarps)
{
    return (size_t)4 * E * sizeof(int32_t) + (size_t)nwarps * E;
}

// Exclusive scan of a[0..n) in place by warp 0; returns the total to every thread of
// warp 0.
__device__ __forceinline__ int32_t warp0_exclusive_scan(int32_t* a, int n, int lane)
{
    int32_t carry = 0;
    for (int base = 0; base < n; base += 32) {
        const int i = base + lane;
        const int32_t v = i < n ? a[i] : 0;
        int32_t s = v;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int32_t t = __shfl_up_sync(0xffffffffu, s, o);
            if (lane >= o) s += t;
        }
        if (i < n) a[i] = carry + s - v;
        carry += __shfl_sync(0xffffffffu, s, 31);
    }
    return carry;
}

// Whole-block union.  Must be called by every thread of the block.  smem holds
// union_smem_bytes(E, blockDim.x / 32) bytes, 4-byte aligned.
static __device__ void union_block(int E, int k, int T, const int32_t* __restrict__ idx,
                            int32_t* __restrict__ union_ids, int32_t* __restrict__ n_union,
                            int32_t* __restrict__ offsets, int32_t* __restrict__ assign,
                            uint32_t* status, uint8_t* smem)
{
    const int tid = threadIdx.x, nt = blockDim.x;
    const int warp = tid >> 5, lane = tid & 31, nwarps = nt >> 5;
    int32_t* count = reinterpret_cast<int32_t*>(smem);
    int32_t* start = count + E;
    int32_t* upos = start + E;
    int32_t* running = upos + E;
    uint8_t* wc = reinterpret_cast<uint8_t*>(running + E);
    const int n = T * k;

    for (int e = tid; e < E; e += nt) {
        count[e] = 0;
        running[e] = 0;
    }
    for (int i = tid; i < nwarps * E; i += nt) wc[i] = 0;
    __syncthreads();
    // counts: lanes of a warp holding the same id add once (hot experts would otherwise
    // serialise on one shared-memory address)
    for (int base = 0; base < n; base += nt) {
        const int a = base + tid;
        int e = -1;
        if (a < n) {
            e = idx[a];
            if (e < 0 || e >= E) {
                set_flag(status, DEV_BAD_INDEX);
                e = -1;
            }
        }
        const unsigned peers = __match_any_sync(0xffffffffu, e);
        if (e >= 0 && (peers & ((1u << lane) - 1u)) == 0) atomicAdd(&count[e], __popc(peers));
    }
    for (int t = tid; t < T; t += nt)
        for (int s = 1; s < k; s++)
            for (int s2 = 0; s2 < s; s2++)
                if (idx[t * k + s] == idx[t * k + s2]) set_flag(status, DEV_BAD_INDEX);
    __syncthreads();
    if (warp == 0) {
        for (int e = lane; e < E; e += 32) {
            start[e] = count[e];
            upos[e] = count[e] > 0 ? 1 : 0;
        }
        __syncwarp();
        warp0_exclusive_scan(start, E, lane);
        const int32_t nu = warp0_exclusive_scan(upos, E, lane);
        __syncwarp();
        for (int e = lane; e < E; e += 32)
            if (count[e] > 0) {
                union_ids[upos[e]] = e;
                offsets[upos[e]] = start[e];
            }
        for (int u = nu + lane; u <= E; u += 32) {
            if (u < E) union_ids[u] = -1;
            offsets[u] = n;
        }
        if (lane == 0) *n_union = nu;
    }
    __syncthreads();
    const unsigned lt_mask = (1u << lane) - 1u;
    for (int base = 0; base < n; base += nt) {
        const int a = base + tid;
        int e = -1;
        if (a < n) {
            e = idx[a];
            if (e < 0 || e >= E) e = -1;
        }
        const unsigned peers = __match_any_sync(0xffffffffu, e);
        const int rank = __popc(peers & lt_mask);
        const int wcount = __popc(peers);
        if (e >= 0 && rank == 0) wc[warp * E + e] = (uint8_t)wcount;
        __syncthreads();
        if (e >= 0) {
            int pre = running[e];
            for (int w2 = 0; w2 < warp; w2++) pre += wc[w2 * E + e];
            assign[start[e] + pre + rank] = a;
        }
        __syncthreads();
        if (e >= 0 && rank == 0) {
            wc[warp * E + e] = 0;
            atomicAdd(&running[e], wcount);
        }
        __syncthreads();
    }
}

}  // namespace coli
