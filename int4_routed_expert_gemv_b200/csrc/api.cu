// extern "C" entry points of the routed int4 MoE library: argument checks, workspace
// layout and kernel launches.  See include/colimoe.h for the contract of each call.
#include <cuda_runtime.h>
#include <stdint.h>
#include <string.h>

#include "../../include/colimoe.h"
#include "common.cuh"
#include "fused.cuh"
#include "fmt.cuh"
#include "gemm.cuh"
#include "gemv.cuh"
#include "rmsnorm.cuh"
#include "route.cuh"

using namespace coli;

namespace {

constexpr size_t kAlign = 256;
inline size_t up(size_t v, size_t a) { return (v + a - 1) / a * a; }

struct WsLayout {
    size_t cnt, logits, h, xd, rpart, hf, hdg, xbuf, xchunk, gemm, total;
};

constexpr size_t kCntBytes = (size_t)kCntWords * 4;

bool dims_ok(const coli_moe_dims* d)
{
    if (!d) return false;
    const int H = d->hidden, I = d->inter, E = d->n_experts, k = d->top_k;
    if (H < 64 || I < 64 || H % 64 || I % 64) return false;
    if (E < 1 || E > kMaxExperts) return false;
    if (k < 1 || k > E || k > kMaxTopK) return false;
    if (d->n_shared != 0 && d->n_shared != 1) return false;
    return true;
}

WsLayout ws_layout(const coli_moe_dims* d, int64_t T)
{
    WsLayout L;
    size_t off = sizeof(WsHeader);
    // the fused decode kernel's counters sit right after the header (cleared with it)
    L.cnt = off;
    off += kCntBytes;
    L.logits = off = up(off, kAlign);
    off += (size_t)T * d->n_experts * sizeof(float);
    L.h = off = up(off, kAlign);
    off += (size_t)T * (d->top_k + d->n_shared) * d->inter * sizeof(float);
    L.xd = off = up(off, kAlign);
    off += (size_t)T * (d->hidden / 32) * kDigitRecBytes;
    // fused decode kernel (batches up to kFusedMaxT): router partial sums, the layer
    // outputs of a stack launch, and the outputs of stack launches but the last
    const int64_t Tf = T < kFusedMaxT ? T : kFusedMaxT;
    L.rpart = off = up(off, kAlign);
    off += (size_t)Tf * d->n_experts * (d->hidden / 128 > 0 ? d->hidden / 128 : 1) * 16;
    L.hf = off = up(off, kAlign);   // SwiGLU activations as (value, epoch) pairs
    off += (size_t)Tf * (d->top_k + d->n_shared) * d->inter * 8;
    L.hdg = off = up(off, kAlign);  // digit rows of h (one per row of hf)
    off += (size_t)Tf * (d->top_k + d->n_shared) * hdg_row_bytes(d->inter);
    L.xbuf = off = up(off, kAlign);
    off += 2 * (size_t)Tf * d->hidden * sizeof(float);
    L.xchunk = off = up(off, kAlign);
    off += 2 * (size_t)Tf * d->hidden * sizeof(float);
    L.gemm = off = up(off, kAlign);
    off += gemm_workspace_bytes(d->hidden, d->inter, d->n_experts, d->top_k, d->n_shared, T);
    L.total = up(off, kAlign);
    return L;
}

inline bool aligned16(const void* p) { return ((uintptr_t)p & 15u) == 0; }

struct DevInfo {
    int sms = 0;
    size_t smem_optin = 0;
};

bool dev_info(DevInfo& di)
{
    static DevInfo cache[64];
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return false;
    if (cache[dev].sms == 0) {
        int sms = 0, optin = 0;
        if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev) !=
                cudaSuccess)
            return false;
        cache[dev].smem_optin = (size_t)optin;
        cache[dev].sms = sms;
    }
    di = cache[dev];
    return true;
}

coli_status ws_check(const coli_moe_dims* d, int32_t T, void* ws, size_t ws_bytes)
{
    if (!ws || !aligned16(ws)) return COLI_EINVAL;
    if (ws_bytes < ws_layout(d, T).total) return COLI_ENOMEM;
    return COLI_OK;
}

coli_status cuda_status(cudaError_t e) { return e == cudaSuccess ? COLI_OK : COLI_ECUDA; }

bool weights_ok(const coli_moe_dims* d, const coli_moe_weights* w, bool need_router)
{
    if (!w) return false;
    if (need_router && (!w->w_router || !aligned16(w->w_router))) return false;
    if (!w->experts || !aligned16(w->experts)) return false;
    if (d->n_shared && (!w->shared || !aligned16(w->shared))) return false;
    const size_t blob = coli_moe_blob_bytes(d->hidden, d->inter);
    if (w->expert_stride < blob || w->expert_stride % 256) return false;
    return true;
}

RouteParams route_params(const coli_moe_dims* d, const float* w_router, const float* bias,
                         const void* x, coli_dtype dtype, int32_t T, int32_t* idx, float* w,
                         float* logits, void* ws)
{
    RouteParams p;
    memset(&p, 0, sizeof(p));
    p.H = d->hidden;
    p.E = d->n_experts;
    p.k = d->top_k;
    p.T = T;
    p.x = x;
    p.x_bf16 = dtype == COLI_BF16;
    p.w_router = w_router;
    p.bias = bias;
    const WsLayout L = ws_layout(d, T);
    p.logits = logits ? logits : reinterpret_cast<float*>((uint8_t*)ws + L.logits);
    p.idx = idx;
    p.w = w;
    p.hdr = reinterpret_cast<WsHeader*>(ws);
    p.status = &p.hdr->status;
    return p;
}

GemvParams gemv_params(const coli_moe_dims* d, const coli_moe_weights* wt, const float* x,
                       int32_t T, const float* w, const int32_t* union_ids,
                       const int32_t* n_union, const int32_t* offsets, const int32_t* assign,
                       const float* residual, float* y, void* ws)
{
    GemvParams p;
    memset(&p, 0, sizeof(p));
    p.H = d->hidden;
    p.I = d->inter;
    p.E = d->n_experts;
    p.k = d->top_k;
    p.T = T;
    p.n_shared = d->n_shared;
    p.experts = wt->experts;
    p.stride = wt->expert_stride;
    p.shared = wt->shared;
    p.x = x;
    p.union_ids = union_ids;
    p.n_union = n_union;
    p.offsets = offsets;
    p.assign = assign;
    p.wts = w;
    p.hd = (uint8_t*)ws + ws_layout(d, T).h;
    p.y = y;
    p.residual = residual;
    p.status = &reinterpret_cast<WsHeader*>(ws)->status;
    return p;
}

// Fused decode kernel set-up for a batch of T tokens through L layers; false if the shape
// or batch is outside what the kernel handles (the caller then takes the separate kernels).
bool fused_setup(FusedParams& f, const coli_moe_dims* d, int32_t T, int L, void* ws)
{
    memset(&f, 0, sizeof(f));
    f.H = d->hidden;
    f.I = d->inter;
    f.E = d->n_experts;
    f.k = d->top_k;
    f.n_shared = d->n_shared;
    f.T = T;
    f.L = L;
    f.norm = L > 1;
    DevInfo di;
    if (!dev_info(di)) return false;
    if (!fused_plan(f, di.sms, di.smem_optin)) return false;
    const WsLayout W = ws_layout(d, T);
    uint8_t* base = (uint8_t*)ws;
    WsHeader* hdr = reinterpret_cast<WsHeader*>(ws);
    f.status = &hdr->status;
    f.gen = &hdr->launch_gen;
    f.cnt = reinterpret_cast<uint32_t*>(base + W.cnt);
    f.rpart = reinterpret_cast<uint4*>(base + W.rpart);
    f.h = reinterpret_cast<uint2*>(base + W.hf);
    f.hdg = base + W.hdg;
    f.hdg_row = (uint32_t)hdg_row_bytes(d->inter);
    f.xbuf = reinterpret_cast<float*>(base + W.xbuf);
    return true;
}

void fused_layer_ptrs(FusedLayer& l, const coli_moe_weights* w, const float* gamma)
{
    l.w_router = w->w_router;
    l.bias = w->router_bias;
    l.experts = w->experts;
    l.shared = w->shared;
    l.gamma = gamma;
    l.stride = w->expert_stride;
}

coli_status run_gemv(int mode, GemvParams& p, cudaStream_t s)
{
    DevInfo di;
    if (!dev_info(di)) return COLI_ECUDA;
    GemvConfig c;
    if (!gemv_plan(mode, p, c, di.sms, di.smem_optin)) return COLI_EUNSUPPORTED;
    return cuda_status(gemv_launch(mode, p, c, s));
}

bool gemv_shape_ok(const coli_moe_dims* d, int32_t T)
{
    // the current device's SM count and shared memory; without a usable device the B200's
    // (the call then fails at its first CUDA step with COLI_ECUDA)
    DevInfo di;
    if (!dev_info(di)) {
        di.sms = 148;
        di.smem_optin = 232448;
    }
    for (int mode = 0; mode < 2; mode++) {
        GemvParams p;
        memset(&p, 0, sizeof(p));
        p.H = d->hidden;
        p.I = d->inter;
        p.T = T;
        GemvConfig c;
        if (!gemv_plan(mode, p, c, di.sms, di.smem_optin)) return false;
    }
    return true;
}

}  // namespace

extern "C" {

size_t coli_moe_blob_bytes(int32_t hidden, int32_t inter)
{
    if (hidden <= 0 || inter <= 0) return 0;
    const size_t h = (size_t)hidden, i = (size_t)inter;
    return 3 * (h * i / 2) + 2 * (i * (h / 64) * 2) + h * (i / 64) * 2;
}

size_t coli_moe_workspace_bytes(const coli_moe_dims* dims, int32_t T_max)
{
    if (!dims_ok(dims) || T_max < 0) return 0;
    return ws_layout(dims, T_max).total;
}

coli_status coli_moe_workspace_init(void* ws, size_t ws_bytes, void* stream)
{
    if (!ws || !aligned16(ws) || ws_bytes < sizeof(WsHeader)) return COLI_EINVAL;
    const size_t n = ws_bytes < sizeof(WsHeader) + kCntBytes ? ws_bytes : sizeof(WsHeader) + kCntBytes;
    return cuda_status(cudaMemsetAsync(ws, 0, n, (cudaStream_t)stream));
}

coli_status coli_moe_read_status(const void* ws, uint32_t* status, void* stream)
{
    if (!ws || !status) return COLI_EINVAL;
    uint32_t v = 0;
    cudaError_t e = cudaMemcpyAsync(&v, ws, sizeof(v), cudaMemcpyDeviceToHost, (cudaStream_t)stream);
    if (e == cudaSuccess) e = cudaStreamSynchronize((cudaStream_t)stream);
    if (e != cudaSuccess) return COLI_ECUDA;
    *status = v;
    if (v & COLI_DEV_TIMEOUT) return COLI_ETIMEOUT;
    return v ? COLI_EDEVICE : COLI_OK;
}

coli_status coli_moe_route(const coli_moe_dims* dims, const float* w_router, const float* bias,
                           const void* x, coli_dtype dtype, int32_t T, int32_t* idx, float* w,
                           float* logits, void* ws, size_t ws_bytes, void* stream)
{
    if (!dims_ok(dims) || T < 0 || (dtype != COLI_F32 && dtype != COLI_BF16)) return COLI_EINVAL;
    if (T == 0) return COLI_OK;
    if (!w_router || !x || !idx || !w || !aligned16(w_router) || !aligned16(x) ||
        (logits && !aligned16(logits)))
        return COLI_EINVAL;
    coli_status st = ws_check(dims, T, ws, ws_bytes);
    if (st != COLI_OK) return st;
    RouteParams p = route_params(dims, w_router, bias, x, dtype, T, idx, w, logits, ws);
    p.do_topk = 1;
    return cuda_status(route_launch(p, (cudaStream_t)stream));
}

coli_status coli_moe_route_union(const coli_moe_dims* dims, const float* w_router,
                                 const float* bias, const void* x, coli_dtype dtype, int32_t T,
                                 int32_t* idx, float* w, float* logits, int32_t* union_ids,
                                 int32_t* n_union, int32_t* offsets, int32_t* assign, void* ws,
                                 size_t ws_bytes, void* stream)
{
    if (!dims_ok(dims) || T < 0 || (dtype != COLI_F32 && dtype != COLI_BF16)) return COLI_EINVAL;
    if (T == 0) return COLI_OK;
    if (!w_router || !x || !idx || !w || !aligned16(w_router) || !aligned16(x) ||
        (logits && !aligned16(logits)) || !union_ids || !n_union || !offsets || !assign)
        return COLI_EINVAL;
    coli_status st = ws_check(dims, T, ws, ws_bytes);
    if (st != COLI_OK) return st;
    RouteParams p = route_params(dims, w_router, bias, x, dtype, T, idx, w, logits, ws);
    p.do_topk = 1;
    p.do_union = 1;
    p.union_ids = union_ids;
    p.n_union = n_union;
    p.offsets = offsets;
    p.assign = assign;
    return cuda_status(route_launch(p, (cudaStream_t)stream));
}

coli_status coli_moe_union(const coli_moe_dims* dims, const int32_t* idx, int32_t T,
                           int32_t* union_ids, int32_t* n_union, int32_t* offsets,
                           int32_t* assign, void* ws, size_t ws_bytes, void* stream)
{
    if (!dims_ok(dims) || T < 0) return COLI_EINVAL;
    if (!idx || !union_ids || !n_union || !offsets || (T > 0 && !assign)) return COLI_EINVAL;
    coli_status st = ws_check(dims, T, ws, ws_bytes);
    if (st != COLI_OK) return st;
    RouteParams p = route_params(dims, nullptr, nullptr, nullptr, COLI_F32, T,
                                 const_cast<int32_t*>(idx), nullptr, nullptr, ws);
    p.union_ids = union_ids;
    p.n_union = n_union;
    p.offsets = offsets;
    p.assign = assign;
    return cuda_status(union_launch(p, (cudaStream_t)stream));
}

coli_status coli_moe_gate_up(const coli_moe_dims* dims, const coli_moe_weights* weights,
                             const float* x, int32_t T, const int32_t* union_ids,
                             const int32_t* n_union, const int32_t* offsets,
                             const int32_t* assign, void* ws, size_t ws_bytes, void* stream)
{
    if (!dims_ok(dims) || T < 0) return COLI_EINVAL;
    if (T == 0) return COLI_OK;
    if (!weights_ok(dims, weights, false) || !x || !aligned16(x) || !union_ids || !n_union ||
        !offsets || !assign)
        return COLI_EINVAL;
    coli_status st = ws_check(dims, T, ws, ws_bytes);
    if (st != COLI_OK) return st;
    if (!gemv_shape_ok(dims, T)) return COLI_EUNSUPPORTED;
    GemvParams p = gemv_params(dims, weights, x, T, nullptr, union_ids, n_union, offsets, assign,
                               nullptr, nullptr, ws);
    return run_gemv(0, p, (cudaStream_t)stream);
}

coli_status coli_moe_down(const coli_moe_dims* dims, const coli_moe_weights* weights,
                          int32_t T, const float* w, const int32_t* union_ids,
                          const int32_t* n_union, const int32_t* offsets, const int32_t* assign,
                          const float* residual, float* y, void* ws, size_t ws_bytes,
                          void* stream)
{
    if (!dims_ok(dims) || T < 0) return COLI_EINVAL;
    if (T == 0) return COLI_OK;
    if (!weights_ok(dims, weights, false) || !w || !union_ids || !n_union || !offsets ||
        !assign || !y || !aligned16(y) || (residual && !aligned16(residual)))
        return COLI_EINVAL;
    coli_status st = ws_check(dims, T, ws, ws_bytes);
    if (st != COLI_OK) return st;
    if (!gemv_shape_ok(dims, T)) return COLI_EUNSUPPORTED;
    GemvParams p = gemv_params(dims, weights, nullptr, T, w, union_ids, n_union, offsets, assign,
                               residual, y, ws);
    return run_gemv(1, p, (cudaStream_t)stream);
}

coli_status coli_moe_forward(const coli_moe_dims* dims, const coli_moe_weights* weights,
                             const void* x, coli_dtype dtype, int32_t T, const int32_t* idx,
                             const float* w, const int32_t* union_ids, const int32_t* n_union,
                             const int32_t* offsets, const int32_t* assign,
                             const float* residual, float* y, void* ws, size_t ws_bytes,
                             void* stream)
{
    if (!dims_ok(dims) || T < 0 || (dtype != COLI_F32 && dtype != COLI_BF16)) return COLI_EINVAL;
    if (T == 0) return COLI_OK;
    if (!weights_ok(dims, weights, false) || !x || !aligned16(x) || !idx || !w || !union_ids ||
        !n_union || !offsets || !assign || !y || !aligned16(y) ||
        (residual && !aligned16(residual)))
        return COLI_EINVAL;
    coli_status st = ws_check(dims, T, ws, ws_bytes);
    if (st != COLI_OK) return st;
    cudaStream_t s = (cudaStream_t)stream;
    WsHeader* hdr = reinterpret_cast<WsHeader*>(ws);
    if (dtype == COLI_BF16) {
        DevInfo di;
        if (!dev_info(di)) return COLI_ECUDA;
        GemmArgs a;
        memset(&a, 0, sizeof(a));
        a.H = dims->hidden;
        a.I = dims->inter;
        a.E = dims->n_experts;
        a.k = dims->top_k;
        a.T = T;
        a.n_shared = dims->n_shared;
        a.experts = weights->experts;
        a.stride = weights->expert_stride;
        a.shared = weights->shared;
        a.x = reinterpret_cast<const __nv_bfloat16*>(x);
        a.w = w;
        a.union_ids = union_ids;
        a.n_union = n_union;
        a.offsets = offsets;
        a.assign = assign;
        a.residual = residual;
        a.y = y;
        a.scratch = (uint8_t*)ws + ws_layout(dims, T).gemm;
        a.hdr = hdr;
        a.num_sms = di.sms;
        a.smem_optin = di.smem_optin;
        if (!gemm_supported(a)) return COLI_EUNSUPPORTED;
        return cuda_status(gemm_forward(a, s));
    }
    FusedParams f;
    if (fused_setup(f, dims, T, 1, ws)) {
        // decode batch: one launch for the experts and the combine
        f.route = 0;
        fused_layer_ptrs(f.layer[0], weights, nullptr);
        f.x = reinterpret_cast<const float*>(x);
        f.residual = residual;
        f.y = y;
        f.idx = const_cast<int32_t*>(idx);
        f.w = const_cast<float*>(w);
        f.union_ids = const_cast<int32_t*>(union_ids);
        f.n_union = const_cast<int32_t*>(n_union);
        f.offsets = const_cast<int32_t*>(offsets);
        f.assign = const_cast<int32_t*>(assign);
        return cuda_status(fused_launch(f, s));
    }
    if (!gemv_shape_ok(dims, T)) return COLI_EUNSUPPORTED;
    GemvParams p = gemv_params(dims, weights, reinterpret_cast<const float*>(x), T, w, union_ids,
                               n_union, offsets, assign, residual, y, ws);
    coli_status r = run_gemv(0, p, s);
    if (r != COLI_OK) return r;
    GemvParams q = gemv_params(dims, weights, nullptr, T, w, union_ids, n_union, offsets, assign,
                               residual, y, ws);
    return run_gemv(1, q, s);
}

coli_status coli_moe_layer(const coli_moe_dims* dims, const coli_moe_weights* weights,
                           const void* x, coli_dtype dtype, int32_t T, int32_t* idx, float* w,
                           float* logits, int32_t* union_ids, int32_t* n_union, int32_t* offsets,
                           int32_t* assign, const float* residual, float* y, void* ws,
                           size_t ws_bytes, void* stream)
{
    if (!dims_ok(dims) || T < 0 || (dtype != COLI_F32 && dtype != COLI_BF16)) return COLI_EINVAL;
    if (T == 0) return COLI_OK;
    if (!weights_ok(dims, weights, true) || !x || !aligned16(x) || !idx || !w || !union_ids ||
        !n_union || !offsets || !assign || !y || !aligned16(y) ||
        (residual && !aligned16(residual)) || (logits && !aligned16(logits)))
        return COLI_EINVAL;
    coli_status st = ws_check(dims, T, ws, ws_bytes);
    if (st != COLI_OK) return st;
    if (dtype == COLI_F32) {
        FusedParams f;
        if (fused_setup(f, dims, T, 1, ws)) {
            // decode batch: the whole layer in one launch
            f.route = 1;
            fused_layer_ptrs(f.layer[0], weights, nullptr);
            f.x = reinterpret_cast<const float*>(x);
            f.residual = residual;
            f.y = y;
            f.idx = idx;
            f.w = w;
            f.logits = logits;
            f.union_ids = union_ids;
            f.n_union = n_union;
            f.offsets = offsets;
            f.assign = assign;
            return cuda_status(fused_launch(f, (cudaStream_t)stream));
        }
    }
    if (dtype == COLI_F32 && !gemv_shape_ok(dims, T)) return COLI_EUNSUPPORTED;
    RouteParams p = route_params(dims, weights->w_router, weights->router_bias, x, dtype, T, idx, w,
                                 logits, ws);
    p.do_topk = 1;
    p.do_union = 1;
    p.union_ids = union_ids;
    p.n_union = n_union;
    p.offsets = offsets;
    p.assign = assign;
    cudaStream_t s = (cudaStream_t)stream;
    if (dtype == COLI_BF16) {
        if (route_launch(p, s) != cudaSuccess) return COLI_ECUDA;
        return coli_moe_forward(dims, weights, x, dtype, T, idx, w, union_ids, n_union, offsets,
                                assign, residual, y, ws, ws_bytes, stream);
    }
    GemvParams g = gemv_params(dims, weights, reinterpret_cast<const float*>(x), T, w, union_ids,
                               n_union, offsets, assign, residual, y, ws);
    if (T <= kSmallT) {
        // decode batch: x turns into digit records in a launch of its own, which the router
        // (a programmatic dependent that waits for it before completing) overlaps
        uint8_t* xd = (uint8_t*)ws + ws_layout(dims, T).xd;
        if (x_digits_launch(reinterpret_cast<const float*>(x), T, dims->hidden, xd, s) !=
            cudaSuccess)
            return COLI_ECUDA;
        p.pdl = 1;
        g.xd = xd;
    } else {
        // x was complete before the router launch began (an ordinary stream-ordered
        // launch), so the gate/up launch may stage it while the router still runs
        g.x_early = 1;
    }
    if (route_launch(p, s) != cudaSuccess) return COLI_ECUDA;
    coli_status r = run_gemv(0, g, s);
    if (r != COLI_OK) return r;
    GemvParams q = gemv_params(dims, weights, nullptr, T, w, union_ids, n_union, offsets, assign,
                               residual, y, ws);
    return run_gemv(1, q, s);
}

coli_status coli_moe_stack(const coli_moe_dims* dims, const coli_moe_weights* layers,
                           const float* const* gamma, int32_t n_layers, double eps, const float* x,
                           int32_t T, int32_t* idx, float* y, void* ws, size_t ws_bytes,
                           void* stream)
{
    if (!dims_ok(dims) || T < 0 || n_layers < 0 || !(eps >= 0.0)) return COLI_EINVAL;
    if (T == 0 || n_layers == 0) return COLI_OK;
    if (!layers || !x || !y || !aligned16(x) || !aligned16(y)) return COLI_EINVAL;
    const size_t xb = (size_t)T * dims->hidden * sizeof(float);
    if ((const uint8_t*)x < (const uint8_t*)y + xb && (const uint8_t*)y < (const uint8_t*)x + xb)
        return COLI_EINVAL;   // y may not overlap x
    for (int32_t l = 0; l < n_layers; l++) {
        if (!weights_ok(dims, &layers[l], true)) return COLI_EINVAL;
        if (gamma && gamma[l] && !aligned16(gamma[l])) return COLI_EINVAL;
    }
    coli_status st = ws_check(dims, T, ws, ws_bytes);
    if (st != COLI_OK) return st;
    const WsLayout W = ws_layout(dims, T);
    float* chunk_out = reinterpret_cast<float*>((uint8_t*)ws + W.xchunk);
    cudaStream_t s = (cudaStream_t)stream;
    const float* in = x;
    for (int32_t l0 = 0, j = 0; l0 < n_layers; l0 += kFusedMaxLayers, j++) {
        const int nl = n_layers - l0 < kFusedMaxLayers ? n_layers - l0 : kFusedMaxLayers;
        FusedParams f;
        if (!fused_setup(f, dims, T, nl, ws)) return COLI_EUNSUPPORTED;
        f.norm = 1;
        f.eps = eps;
        f.route = 1;
        for (int l = 0; l < nl; l++)
            fused_layer_ptrs(f.layer[l], &layers[l0 + l], gamma ? gamma[l0 + l] : nullptr);
        // re-plan with the normalisation on (the plan does not depend on it)
        f.x = in;
        const bool last = l0 + nl >= n_layers;
        float* out = last ? y : chunk_out + (size_t)(j & 1) * T * dims->hidden;
        f.y = out;
        f.idx_layers = idx ? idx + (size_t)l0 * T * dims->top_k : nullptr;
        if (fused_launch(f, s) != cudaSuccess) return COLI_ECUDA;
        in = out;
    }
    return COLI_OK;
}

coli_status coli_rmsnorm(int32_t hidden, int32_t T, const float* x, const float* gamma, double eps,
                         float* out, void* stream)
{
    if (hidden <= 0 || T < 0 || !(eps >= 0.0)) return COLI_EINVAL;
    if (T == 0) return COLI_OK;
    if (!x || !gamma || !out) return COLI_EINVAL;
    return cuda_status(rmsnorm_launch(hidden, T, x, gamma, eps, out, (cudaStream_t)stream));
}

const char* coli_status_string(coli_status s)
{
    switch (s) {
    case COLI_OK: return "ok";
    case COLI_EINVAL: return "invalid argument";
    case COLI_ENOMEM: return "workspace too small";
    case COLI_ECUDA: return "CUDA error";
    case COLI_ETIMEOUT: return "device wait timed out";
    case COLI_EUNSUPPORTED: return "unsupported shape or dtype";
    case COLI_EDEVICE: return "device-side error";
    }
    return "unknown status";
}

}  // extern "C"

size_t coli_moe_blob_bytes_fmt(int32_t hidden, int32_t inter, int32_t fmt)
{
    if (hidden < 64 || inter < 64 || hidden % 64 || inter % 64) return 0;
    return fmt_blob_bytes(hidden, inter, fmt);
}

coli_status coli_moe_forward_fmt(const coli_moe_dims* dims, int32_t fmt, const coli_moe_weights* weights,
                                 const float* x, int32_t T, const float* w, const int32_t* union_ids,
                                 const int32_t* n_union, const int32_t* offsets, const int32_t* assign,
                                 const float* residual, float* y, void* ws, size_t ws_bytes, void* stream)
{
    if (!dims_ok(dims) || T < 0 || fmt < 0 || fmt > 3) return COLI_EINVAL;
    if (T == 0) return COLI_OK;
    if (T > kFmtMaxT) return COLI_EUNSUPPORTED;
    const size_t blob = fmt_blob_bytes(dims->hidden, dims->inter, fmt);
    if (!weights || !weights->experts || !aligned16(weights->experts) ||
        (dims->n_shared && (!weights->shared || !aligned16(weights->shared))) ||
        weights->expert_stride < blob || weights->expert_stride % 256 || !x || !aligned16(x) || !w ||
        !union_ids || !n_union || !offsets || !assign || !y || !aligned16(y) ||
        (residual && !aligned16(residual)))
        return COLI_EINVAL;
    coli_status st = ws_check(dims, T, ws, ws_bytes);
    if (st != COLI_OK) return st;
    DevInfo di;
    if (!dev_info(di)) return COLI_ECUDA;
    // x of the batch and one segment's h in shared memory
    if ((size_t)T * dims->hidden * 5 > di.smem_optin || (size_t)T * dims->inter * 5 > di.smem_optin)
        return COLI_EUNSUPPORTED;
    const WsLayout W = ws_layout(dims, T);
    FmtParams f;
    memset(&f, 0, sizeof(f));
    f.H = dims->hidden;
    f.I = dims->inter;
    f.E = dims->n_experts;
    f.k = dims->top_k;
    f.T = T;
    f.n_shared = dims->n_shared;
    f.fmt = fmt;
    f.experts = weights->experts;
    f.stride = weights->expert_stride;
    f.shared = weights->shared;
    f.x = x;
    f.w = w;
    f.union_ids = union_ids;
    f.n_union = n_union;
    f.offsets = offsets;
    f.assign = assign;
    f.h = reinterpret_cast<float*>(static_cast<uint8_t*>(ws) + W.h);
    f.residual = residual;
    f.y = y;
    f.status = reinterpret_cast<uint32_t*>(ws);
    return cuda_status(fmt_forward_launch(f, di.sms, (cudaStream_t)stream));
}
