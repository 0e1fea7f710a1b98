// Top-k selection and the small batch union, one warp each, results in registers.
//
// Top-k: "top-8 by softmax score with index tie-break and renormalised weights" (GLM-5.2
// routing, colibri technical article "colibri 技术解读", section "MoE 的稀疏性").  The
// softmax is monotone in the logit, so selection compares logits; equal logits (+0 and -0
// included) go to the lower expert index.  The weights are exp(l_i - l_max) / sum_j
// exp(l_j - l_max) over the k selected logits, in double.
//
// Union: each distinct selected expert appears once (colibri README.zh-CN, "工作原理 /
// 绝不为同一次磁盘读取等待两遍", 批量并集): union_ids ascending, offsets into assign,
// assign = the flat positions t*k + slot grouped by expert, ascending within an expert.
//
// Both are written for latency: a selection round is two warp reductions (redux.sync) on
// 32-bit keys, and the union of up to 32 assignments is one rolled 32-step loop, so the
// code executed on the serial path of a decode step stays short.
#pragma once
#include "common.cuh"

namespace coli {

// Order-preserving 32-bit key of a float: a larger value gives a larger key, -0 == +0.  No
// finite or infinite value maps to 0, which marks a removed or absent slot.
__device__ __forceinline__ uint32_t order_key(float v)
{
    const uint32_t b = __float_as_uint(v == 0.0f ? 0.0f : v);
    return (b & 0x80000000u) ? ~b : (b | 0x80000000u);
}

__device__ __forceinline__ float key_float(uint32_t u)
{
    return __uint_as_float((u & 0x80000000u) ? (u & 0x7FFFFFFFu) : ~u);
}

// One warp selects the k (<= 32) largest of the E (<= 32 * MAXPL) logits lt[0..E).  On
// return lane s < k holds selection s (descending logit, ties to the lower index): its
// expert in e_out and its order key in key_out.
template <int MAXPL>
__device__ __forceinline__ void topk_warp_keys(const float* lt, int E, int k, int lane, int& e_out,
                                               uint32_t& key_out)
{
    uint32_t key[MAXPL];
#pragma unroll
    for (int i = 0; i < MAXPL; i++) {
        const int e = lane + 32 * i;
        key[i] = (e < E) ? order_key(__ldcg(lt + e)) : 0u;
    }
    uint32_t mine = 0u;
    int mine_e = 0;
    for (int s = 0; s < k; s++) {
        // this lane's largest key, lowest index among equals (indices grow with i)
        uint32_t b = key[0];
        int bi = 0;
#pragma unroll
        for (int i = 1; i < MAXPL; i++)
            if (key[i] > b) {
                b = key[i];
                bi = i;
            }
        const uint32_t m = __reduce_max_sync(0xffffffffu, b);
        const uint32_t cand = (b == m) ? (uint32_t)(lane + 32 * bi) : 0xFFFFFFFFu;
        const uint32_t e = __reduce_min_sync(0xffffffffu, cand);
        if ((int)(e & 31u) == lane) {
#pragma unroll
            for (int i = 0; i < MAXPL; i++)
                if (i == (int)(e >> 5)) key[i] = 0u;
        }
        if (lane == s) {
            mine = m;
            mine_e = (int)e;
        }
    }
    e_out = mine_e;
    key_out = mine;
}

// Renormalised softmax weight of selection `lane` (< k) of one token, from the order keys of
// its k selections held by lanes 0..k-1 in descending order; every lane of the warp calls.
__device__ __forceinline__ float topk_weight(uint32_t key, int k, int lane)
{
    const double lmax = (double)key_float(__shfl_sync(0xffffffffu, key, 0));
    double ex = 0.0;
    if (lane < k) ex = exp((double)key_float(key) - lmax);
    double z = ex;
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) z += __shfl_xor_sync(0xffffffffu, z, o);
    return (float)(ex / z);
}

// Selection of any E <= 1024 (keys per lane rounded up to 8, 16 or 32).
__device__ __forceinline__ void topk_warp_any(const float* lt, int E, int k, int lane, int& e_out,
                                              uint32_t& key_out)
{
    if (E <= 256) topk_warp_keys<8>(lt, E, k, lane, e_out, key_out);
    else if (E <= 512) topk_warp_keys<16>(lt, E, k, lane, e_out, key_out);
    else topk_warp_keys<32>(lt, E, k, lane, e_out, key_out);
}

// Selection and weights: lane s < k receives expert and weight of selection s.
__device__ __forceinline__ void topk_warp_any(const float* lt, int E, int k, int lane, int& e_out,
                                              float& w_out)
{
    uint32_t key;
    topk_warp_any(lt, E, k, lane, e_out, key);
    w_out = topk_weight(key, k, lane);
}

// Per-lane result of union_warp_lanes.
struct UnionLane {
    int rank;     // position of this assignment in assign (lanes < n)
    int uidx;     // union entry of its expert (valid lanes)
    int nu;       // number of distinct experts (every lane)
    bool first;   // this lane is the first assignment of its expert
};

// One warp, n = T * k <= 32 assignments: lane a < n holds e, the expert of assignment a
// (token a / k, slot a % k).  An expert outside [0, E) or repeated within one token sets
// DEV_BAD_INDEX; such an entry takes no union entry and is ranked after every valid one,
// so assign stays a permutation of 0..n-1.
__device__ __forceinline__ UnionLane union_warp_lanes(int E, int k, int n, int e, int lane,
                                                      uint32_t* status)
{
    bool valid = lane < n;
    if (valid && (e < 0 || e >= E)) {
        set_flag(status, DEV_BAD_INDEX);
        valid = false;
    }
    const int key = valid ? e : 0x7FFFFFFF;   // invalid and idle lanes sort last
    const uint32_t vmask = __ballot_sync(0xffffffffu, valid);
    const uint32_t same = __match_any_sync(0xffffffffu, key) & vmask;
    if (valid) {
        const int t = lane / k;
        const uint32_t tmask = (k >= 32) ? 0xFFFFFFFFu : (((1u << k) - 1u) << (t * k));
        if (__popc(same & tmask) > 1) set_flag(status, DEV_BAD_INDEX);
    }
    UnionLane r;
    r.first = valid && (same & ((1u << lane) - 1u)) == 0u;
    const uint32_t fmask = __ballot_sync(0xffffffffu, r.first);
    r.nu = __popc(fmask);
    int rank = 0, uidx = 0;
    for (int src = 0; src < 32; src++) {
        const int ko = __shfl_sync(0xffffffffu, key, src);
        rank += (ko < key || (ko == key && src < lane)) ? 1 : 0;
        uidx += (((fmask >> src) & 1u) && ko < key) ? 1 : 0;
    }
    r.rank = rank;
    r.uidx = uidx;
    return r;
}

// Writes the union of union_warp_lanes: assign[0..n), union_ids[0..nu) and offsets[0..nu],
// then union_ids[q] = -1 and offsets[q] = n for nu <= q < cap (offsets up to cap
// inclusive); n_union if not null.
__device__ __forceinline__ void union_store(const UnionLane& r, int e, int n, int cap, int lane,
                                            int32_t* union_ids, int32_t* n_union, int32_t* offsets,
                                            int32_t* assign)
{
    if (lane < n) assign[r.rank] = lane;
    if (r.first) {
        union_ids[r.uidx] = e;
        offsets[r.uidx] = r.rank;
    }
    for (int q = r.nu + lane; q <= cap; q += 32) {
        if (q < cap) union_ids[q] = -1;
        offsets[q] = n;
    }
    if (lane == 0 && n_union) *n_union = r.nu;
}

}  // namespace coli
