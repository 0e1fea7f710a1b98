// Router: logits = x . W_r^T (+ bias), top-k with index tie-break, renormalised softmax
// weights; optionally followed by the batch union in the same launch.
//
// The router is the first of the per-layer steps ("路由器选出专家", colibri technical
// article "colibri 技术解读", section "引擎结构：一个 C 文件，五步 token 路径"); GLM-5.2
// selects 8 of 256 routed experts per layer (same article, "MoE 的稀疏性").
//
// Logits are the double-precision sum of the exact float x float products, rounded once
// to float.  Any summation order gives the same float except when the exact sum lies
// within about 1e-16 (relative) of a float rounding boundary, so the selected indices
// agree bit for bit with a sequential double-precision reference.  Selection compares
// floats (ties, including +0 == -0, go to the lower expert index); the weights are
// exp(l_i - l_max) / sum_j exp(l_j - l_max) over the selected logits, in double.
#include "common.cuh"
#include "route.cuh"
#include "select.cuh"
#include "union.cuh"

namespace coli {
namespace {

template <typename XT>
__device__ __forceinline__ float4 load_x4(const XT* x, size_t i4);

template <>
__device__ __forceinline__ float4 load_x4<float>(const float* x, size_t i4)
{
    return __ldg(reinterpret_cast<const float4*>(x) + i4);
}

template <>
__device__ __forceinline__ float4 load_x4<__nv_bfloat16>(const __nv_bfloat16* x, size_t i4)
{
    const uint2 r = __ldg(reinterpret_cast<const uint2*>(x) + i4);
    return make_float4(__uint_as_float(r.x << 16), __uint_as_float(r.x & 0xFFFF0000u),
                       __uint_as_float(r.y << 16), __uint_as_float(r.y & 0xFFFF0000u));
}

__device__ __forceinline__ double dsum_warp(double v)
{
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

// Small batches: a CTA computes RB router rows for all T (<= kSmallT) tokens; threads
// split the hidden dimension.  The last CTA to finish (ticket in the workspace header)
// runs top-k for every token and, if asked, the batch union.
template <typename XT, int RB>
__global__ void __launch_bounds__(256) router_small_kernel(const __grid_constant__ RouteParams p)
{
    extern __shared__ __align__(16) uint8_t smem[];
    __shared__ double part[8][RB * kSmallT];
    __shared__ int is_last;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    pdl_launch_dependents();   // the expert kernels may be scheduled now; they wait for us
    const int e0 = blockIdx.x * RB;
    const int H4 = p.H / 4;
    const XT* x = reinterpret_cast<const XT*>(p.x);

    // token-outer: for each token every router and activation load of a pass is issued
    // before the first FMA, so a pass costs one memory round trip (the second and later
    // tokens find the CTA's router rows in L1)
    constexpr int MAXIT = 8;   // one pass covers H <= 8192
    for (int t = 0; t < p.T; t++) {
        double acc[RB];
#pragma unroll
        for (int r = 0; r < RB; r++) acc[r] = 0.0;
        for (int base = 0; base < H4; base += 256 * MAXIT) {
            float4 wv[RB][MAXIT], xv[MAXIT];
#pragma unroll
            for (int it = 0; it < MAXIT; it++) {
                const int c4 = base + it * 256 + tid;
                const bool in = c4 < H4;
#pragma unroll
                for (int r = 0; r < RB; r++)
                    wv[r][it] = (in && e0 + r < p.E)
                                    ? __ldg(reinterpret_cast<const float4*>(p.w_router) +
                                            (size_t)(e0 + r) * H4 + c4)
                                    : make_float4(0.f, 0.f, 0.f, 0.f);
                xv[it] = in ? load_x4<XT>(x, (size_t)t * H4 + c4) : make_float4(0.f, 0.f, 0.f, 0.f);
            }
#pragma unroll
            for (int it = 0; it < MAXIT; it++) {
#pragma unroll
                for (int r = 0; r < RB; r++) {
                    double a = acc[r];
                    a = fma((double)xv[it].x, (double)wv[r][it].x, a);
                    a = fma((double)xv[it].y, (double)wv[r][it].y, a);
                    a = fma((double)xv[it].z, (double)wv[r][it].z, a);
                    a = fma((double)xv[it].w, (double)wv[r][it].w, a);
                    acc[r] = a;
                }
            }
        }
#pragma unroll
        for (int r = 0; r < RB; r++) {
            const double v = dsum_warp(acc[r]);
            if (lane == 0) part[warp][r * kSmallT + t] = v;
        }
    }
    __syncthreads();
    if (tid < RB * kSmallT) {
        const int r = tid / kSmallT, t = tid % kSmallT;
        if (t < p.T && e0 + r < p.E) {
            double s = 0.0;
            for (int w = 0; w < 8; w++) s += part[w][tid];
            if (p.bias) s += (double)p.bias[e0 + r];
            const float l = (float)s;
            if (!isfinite(l)) set_flag(p.status, DEV_NONFINITE);
            p.logits[(size_t)t * p.E + e0 + r] = l;
        }
    }
    if (!p.do_topk) {
        pdl_wait();
        return;
    }
    // ---- last-CTA election: the final arrival sees every logit
    __threadfence();
    __syncthreads();
    if (tid == 0) {
        const uint32_t prev = atomicAdd(&p.hdr->route_ticket, 1u);
        is_last = (prev == gridDim.x - 1);
        if (is_last) atomicExch(&p.hdr->route_ticket, 0u);
    }
    __syncthreads();
    if (!is_last) return;
    __threadfence();
    pdl_wait();   // a programmatic launch completes only after the kernel it follows
    // one warp per token (T <= kSmallT = 8 warps of this block) selects; then warp 0 builds
    // the union of a batch of at most 32 assignments (selections passed through shared
    // memory) while the other warps compute the routing weights from the selected keys
    __shared__ int sel[32];
    __shared__ uint32_t selkey[kSmallT * kMaxTopK];
    const bool small_union = p.do_union && p.T * p.k <= 32;
    for (int t = warp; t < p.T; t += 8) {
        int e;
        uint32_t key;
        topk_warp_any(p.logits + (size_t)t * p.E, p.E, p.k, lane, e, key);
        if (lane < p.k) {
            p.idx[(size_t)t * p.k + lane] = e;
            selkey[t * p.k + lane] = key;
            if (small_union) sel[t * p.k + lane] = e;
        }
    }
    __syncthreads();
    const int wfirst = small_union ? 1 : 0;
    if (small_union && warp == 0) {
        const int n = p.T * p.k;
        const int e = lane < n ? sel[lane] : 0;
        const UnionLane r = union_warp_lanes(p.E, p.k, n, e, lane, p.status);
        union_store(r, e, n, p.E, lane, p.union_ids, p.n_union, p.offsets, p.assign);
    }
    for (int t = warp - wfirst; t >= 0 && t < p.T; t += 8 - wfirst) {
        const uint32_t key = lane < p.k ? selkey[t * p.k + lane] : 0u;
        const float wv = topk_weight(key, p.k, lane);
        if (lane < p.k) p.w[(size_t)t * p.k + lane] = wv;
    }
    if (p.do_union && !small_union) {
        __threadfence();
        __syncthreads();
        union_block(p.E, p.k, p.T, p.idx, p.union_ids, p.n_union, p.offsets, p.assign, p.status,
                    smem);
    }
}

// Large batches, few tiles (small E): 32 tokens x 32 experts per CTA, 32-column slabs converted to double once
// when staged in shared memory; each thread accumulates 2 x 2 logits in double.
template <typename XT>
__global__ void __launch_bounds__(256) router_tiled32_kernel(const __grid_constant__ RouteParams p)
{
    __shared__ __align__(16) double xs[32][34];   // [k][token]
    __shared__ __align__(16) double ws[32][34];   // [k][expert]
    const int tid = threadIdx.x;
    const int t0 = blockIdx.y * 32, e0 = blockIdx.x * 32;
    const int ty = tid / 16, tx = tid % 16;
    const XT* x = reinterpret_cast<const XT*>(p.x);
    double acc[2][2] = {{0.0, 0.0}, {0.0, 0.0}};
    const int row = tid / 8, c4 = tid % 8;        // staging: 32 rows x 8 float4
    for (int k0 = 0; k0 < p.H; k0 += 32) {
        float4 xv = make_float4(0.f, 0.f, 0.f, 0.f), wv = xv;
        if (t0 + row < p.T) xv = load_x4<XT>(x, ((size_t)(t0 + row) * p.H + k0) / 4 + c4);
        if (e0 + row < p.E)
            wv = __ldg(reinterpret_cast<const float4*>(p.w_router) + ((size_t)(e0 + row) * p.H + k0) / 4 + c4);
        __syncthreads();
        xs[c4 * 4 + 0][row] = xv.x;
        xs[c4 * 4 + 1][row] = xv.y;
        xs[c4 * 4 + 2][row] = xv.z;
        xs[c4 * 4 + 3][row] = xv.w;
        ws[c4 * 4 + 0][row] = wv.x;
        ws[c4 * 4 + 1][row] = wv.y;
        ws[c4 * 4 + 2][row] = wv.z;
        ws[c4 * 4 + 3][row] = wv.w;
        __syncthreads();
#pragma unroll 8
        for (int kk = 0; kk < 32; kk++) {
            const double2 a = *reinterpret_cast<const double2*>(&xs[kk][ty * 2]);
            const double2 b = *reinterpret_cast<const double2*>(&ws[kk][tx * 2]);
            acc[0][0] = fma(a.x, b.x, acc[0][0]);
            acc[0][1] = fma(a.x, b.y, acc[0][1]);
            acc[1][0] = fma(a.y, b.x, acc[1][0]);
            acc[1][1] = fma(a.y, b.y, acc[1][1]);
        }
    }
#pragma unroll
    for (int i = 0; i < 2; i++)
#pragma unroll
        for (int jj = 0; jj < 2; jj++) {
            const int t = t0 + ty * 2 + i, e = e0 + tx * 2 + jj;
            if (t < p.T && e < p.E) {
                double s = acc[i][jj];
                if (p.bias) s += (double)p.bias[e];
                const float l = (float)s;
                if (!isfinite(l)) set_flag(p.status, DEV_NONFINITE);
                p.logits[(size_t)t * p.E + e] = l;
            }
        }
}

// Large batches: 64 tokens x 64 experts per CTA, 16-column slabs of x and W_r converted to
// double once when staged in shared memory (two slabs in flight); each thread accumulates
// a 4 x 4 block of logits in double, reading 8 doubles per 16 FMAs.
template <typename XT>
__global__ void __launch_bounds__(256) router_tiled64_kernel(const __grid_constant__ RouteParams p)
{
    constexpr int TM = 64, KS = 16;
    __shared__ __align__(16) double xs[2][KS][TM + 2];   // [buf][k][token]
    __shared__ __align__(16) double ws[2][KS][TM + 2];   // [buf][k][expert]
    const int tid = threadIdx.x;
    const int t0 = blockIdx.y * TM, e0 = blockIdx.x * TM;
    const int ty = tid / 16, tx = tid % 16;       // 4 tokens x 4 experts per thread
    const XT* x = reinterpret_cast<const XT*>(p.x);
    double acc[4][4];
#pragma unroll
    for (int i = 0; i < 4; i++)
#pragma unroll
        for (int j = 0; j < 4; j++) acc[i][j] = 0.0;
    // staging: thread -> (row = tid / 4, four consecutive k at 4 * (tid % 4))
    const int row = tid / 4, c4 = tid % 4;
    auto load = [&](int k0, float4& xv, float4& wv) {
        xv = make_float4(0.f, 0.f, 0.f, 0.f);
        wv = xv;
        if (t0 + row < p.T) xv = load_x4<XT>(x, ((size_t)(t0 + row) * p.H + k0) / 4 + c4);
        if (e0 + row < p.E)
            wv = __ldg(reinterpret_cast<const float4*>(p.w_router) + ((size_t)(e0 + row) * p.H + k0) / 4 + c4);
    };
    auto stage = [&](int b, const float4& xv, const float4& wv) {
        xs[b][c4 * 4 + 0][row] = xv.x;
        xs[b][c4 * 4 + 1][row] = xv.y;
        xs[b][c4 * 4 + 2][row] = xv.z;
        xs[b][c4 * 4 + 3][row] = xv.w;
        ws[b][c4 * 4 + 0][row] = wv.x;
        ws[b][c4 * 4 + 1][row] = wv.y;
        ws[b][c4 * 4 + 2][row] = wv.z;
        ws[b][c4 * 4 + 3][row] = wv.w;
    };
    float4 xv, wv;
    load(0, xv, wv);
    stage(0, xv, wv);
    __syncthreads();
    const int nk = p.H / KS;
    for (int kt = 0; kt < nk; kt++) {
        const int b = kt & 1;
        if (kt + 1 < nk) load((kt + 1) * KS, xv, wv);   // next slab in flight during the FMAs
#pragma unroll
        for (int kk = 0; kk < KS; kk++) {
            const double2 a01 = *reinterpret_cast<const double2*>(&xs[b][kk][ty * 4]);
            const double2 a23 = *reinterpret_cast<const double2*>(&xs[b][kk][ty * 4 + 2]);
            const double2 b01 = *reinterpret_cast<const double2*>(&ws[b][kk][tx * 4]);
            const double2 b23 = *reinterpret_cast<const double2*>(&ws[b][kk][tx * 4 + 2]);
            const double av[4] = {a01.x, a01.y, a23.x, a23.y};
            const double bv[4] = {b01.x, b01.y, b23.x, b23.y};
#pragma unroll
            for (int i = 0; i < 4; i++)
#pragma unroll
                for (int j = 0; j < 4; j++) acc[i][j] = fma(av[i], bv[j], acc[i][j]);
        }
        if (kt + 1 < nk) stage(b ^ 1, xv, wv);
        __syncthreads();
    }
#pragma unroll
    for (int i = 0; i < 4; i++)
#pragma unroll
        for (int j = 0; j < 4; j++) {
            const int t = t0 + ty * 4 + i, e = e0 + tx * 4 + j;
            if (t < p.T && e < p.E) {
                double s = acc[i][j];
                if (p.bias) s += (double)p.bias[e];
                const float l = (float)s;
                if (!isfinite(l)) set_flag(p.status, DEV_NONFINITE);
                p.logits[(size_t)t * p.E + e] = l;
            }
        }
}

__global__ void __launch_bounds__(256) topk_kernel(const __grid_constant__ RouteParams p)
{
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int t = blockIdx.x * 8 + warp;
    if (t < p.T) {
        int e;
        float wv;
        topk_warp_any(p.logits + (size_t)t * p.E, p.E, p.k, lane, e, wv);
        if (lane < p.k) {
            p.idx[(size_t)t * p.k + lane] = e;
            p.w[(size_t)t * p.k + lane] = wv;
        }
    }
}

__global__ void __launch_bounds__(1024) union_kernel(const __grid_constant__ RouteParams p)
{
    extern __shared__ __align__(16) uint8_t smem[];
    if (p.T * p.k <= 32) {
        if (threadIdx.x < 32) {
            const int lane = threadIdx.x, n = p.T * p.k;
            const int e = lane < n ? p.idx[lane] : 0;
            const UnionLane r = union_warp_lanes(p.E, p.k, n, e, lane, p.status);
            union_store(r, e, n, p.E, lane, p.union_ids, p.n_union, p.offsets, p.assign);
        }
        return;
    }
    union_block(p.E, p.k, p.T, p.idx, p.union_ids, p.n_union, p.offsets, p.assign, p.status, smem);
}

}  // namespace

cudaError_t route_launch(const RouteParams& p, cudaStream_t s)
{
    const bool bf16 = p.x_bf16 != 0;
    if (p.T <= kSmallT) {
        constexpr int RB = 2;
        const int grid = (p.E + RB - 1) / RB;
        const size_t smem = (p.do_union && p.T * p.k > 32) ? union_smem_bytes(p.E, 8) : 0;
        auto kern = bf16 ? router_small_kernel<__nv_bfloat16, RB> : router_small_kernel<float, RB>;
        if (smem > 48 * 1024) {
            cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                                 (int)smem);
            if (e != cudaSuccess) return e;
        }
        if (!p.pdl) {
            kern<<<grid, 256, smem, s>>>(p);
            return cudaGetLastError();
        }
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3(grid);
        cfg.blockDim = dim3(256);
        cfg.dynamicSmemBytes = smem;
        cfg.stream = s;
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        attr[0].val.programmaticStreamSerializationAllowed = 1;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        return cudaLaunchKernelEx(&cfg, kern, p);
    }
    // 64 x 64 tiles (4 x 4 logits per thread, half the shared-memory reads per FMA) when
    // they still give about one CTA per SM, else 32 x 32 tiles for more CTAs
    const long tiles64 = (long)((p.E + 63) / 64) * ((p.T + 63) / 64);
    if (tiles64 >= 120) {
        dim3 grid((p.E + 63) / 64, (p.T + 63) / 64);
        if (bf16)
            router_tiled64_kernel<__nv_bfloat16><<<grid, 256, 0, s>>>(p);
        else
            router_tiled64_kernel<float><<<grid, 256, 0, s>>>(p);
    } else {
        dim3 grid((p.E + 31) / 32, (p.T + 31) / 32);
        if (bf16)
            router_tiled32_kernel<__nv_bfloat16><<<grid, 256, 0, s>>>(p);
        else
            router_tiled32_kernel<float><<<grid, 256, 0, s>>>(p);
    }
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess || !p.do_topk) return e;
    topk_kernel<<<(p.T + 7) / 8, 256, 0, s>>>(p);
    e = cudaGetLastError();
    if (e != cudaSuccess || !p.do_union) return e;
    return union_launch(p, s);
}

cudaError_t union_launch(const RouteParams& p, cudaStream_t s)
{
    const int nt = (p.T * p.k <= 32) ? 32 : 1024;
    const size_t smem = (p.T * p.k <= 32) ? 0 : union_smem_bytes(p.E, nt / 32);
    if (smem > 48 * 1024) {
        cudaError_t e = cudaFuncSetAttribute(union_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             (int)smem);
        if (e != cudaSuccess) return e;
    }
    union_kernel<<<1, nt, smem, s>>>(p);
    return cudaGetLastError();
}

}  // namespace coli
