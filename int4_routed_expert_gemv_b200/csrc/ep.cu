// Expert parallelism: the part of a batch union that one rank computes.
//
// With the experts split over ranks in contiguous id ranges, each rank routes the batch
// with the full (replicated) router, takes the batch union, keeps the entries of its own
// range and runs the expert FFNs on those only; the ranks' partial outputs add up to the
// layer's y (one all-reduce of y per layer).  The pages' analogues are the all-resident
// multi-GPU host and cluster mode's one batched request per layer (colibri README.zh-CN
// "实际成果"; the technical article's "集群模式与开放问题清单").
//
// coli_moe_union_restrict does the keeping: the union's ids are ascending, so the entries
// of [e0, e1) are one contiguous run of it; their ids are renumbered to e - e0, their
// offsets rebased to 0, and their assignment positions (t * k + slot into the full idx and
// w arrays) copied in order, so the regular forward runs on the rank's experts unchanged.
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/colimoe.h"

namespace {

constexpr int kThreads = 256;

__global__ void __launch_bounds__(kThreads) union_restrict_kernel(int E, int Tk, int e0, int e1, const int32_t* union_ids,
                                                                 const int32_t* n_union, const int32_t* offsets,
                                                                 const int32_t* assign, int32_t* uid_l,
                                                                 int32_t* nu_l, int32_t* off_l, int32_t* asg_l)
{
    __shared__ int s_ua, s_ub;
    const int nu = max(0, min(*n_union, E));
    if (threadIdx.x == 0) {
        s_ua = nu;
        s_ub = nu;
    }
    __syncthreads();
    // first entries with id >= e0 and id >= e1 (ids ascending)
    for (int u = threadIdx.x; u < nu; u += kThreads) {
        const int id = union_ids[u], prev = u > 0 ? union_ids[u - 1] : INT32_MIN;
        if (id >= e0 && prev < e0) s_ua = u;
        if (id >= e1 && prev < e1) s_ub = u;
    }
    __syncthreads();
    const int ua = s_ua, ub = max(s_ub, ua), nl = ub - ua, El = e1 - e0;
    const int a0 = offsets[ua], a1 = offsets[ub], na = a1 - a0;
    for (int j = threadIdx.x; j <= El; j += kThreads) {
        if (j < El) uid_l[j] = j < nl ? union_ids[ua + j] - e0 : -1;
        off_l[j] = j <= nl ? offsets[ua + j] - a0 : na;
    }
    for (int i = threadIdx.x; i < Tk; i += kThreads) asg_l[i] = i < na ? assign[a0 + i] : 0;
    if (threadIdx.x == 0) *nu_l = nl;
}

}  // namespace

extern "C" coli_status coli_moe_union_restrict(const coli_moe_dims* dims, int32_t T, int32_t e0, int32_t e1,
                                               const int32_t* union_ids, const int32_t* n_union,
                                               const int32_t* offsets, const int32_t* assign,
                                               int32_t* union_ids_local, int32_t* n_union_local,
                                               int32_t* offsets_local, int32_t* assign_local, void* stream)
{
    if (!dims || dims->n_experts < 1 || dims->top_k < 1 || T < 0 || e0 < 0 || e1 <= e0 ||
        e1 > dims->n_experts || !union_ids || !n_union || !offsets || !union_ids_local || !n_union_local ||
        !offsets_local || (T > 0 && (!assign || !assign_local)))
        return COLI_EINVAL;
    union_restrict_kernel<<<1, kThreads, 0, (cudaStream_t)stream>>>(dims->n_experts, T * dims->top_k, e0, e1,
                                                                    union_ids, n_union, offsets, assign,
                                                                    union_ids_local, n_union_local, offsets_local,
                                                                    assign_local);
    return cudaGetLastError() == cudaSuccess ? COLI_OK : COLI_ECUDA;
}
