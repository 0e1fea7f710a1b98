// coli_moe_forward_noalloc: the fp32 decode forward (gate/up GEMV + SwiGLU, then down GEMV
// + combine) for callers that cannot allocate device memory.
//
// The regular entry points take a caller-owned workspace.  Some callers have no way to
// provide one: code that runs inside a host framework's enqueue callback, where the
// framework owns every device allocation and forbids new ones, or a latency-critical
// loop where a cudaMalloc would synchronise the device and stall other streams.  This
// entry point keeps its scratch (the workspace header and the SwiGLU activations h) in a
// fixed array in the library's own device memory instead.
//
// Facts a caller must know:
//   * the array holds kStaticScratchBytes (4 MiB) on every GPU that loads the library,
//     for as long as the process lives;
//   * a batch needs 256 + T * (top_k + n_shared) * inter * 4 bytes of it; larger batches
//     are rejected with COLI_ENOMEM before anything is enqueued;
//   * every call on a device shares the array and it keeps the last call's contents;
//     the 256-byte header (device status word) is cleared at the start of each call, h
//     is fully rewritten before it is read;
//   * two calls whose work overlaps on the GPU (e.g. on two streams) race on the array;
//     serialise them (one stream, or events);
//   * the first call on a device looks up the array's device address (set-up, once per
//     device, with that device current); make that first call before any stream capture;
//   * the device status word of a call stays in the array's header until the next call
//     clears it (coli_moe_noalloc_read_status reads it without allocating);
//   * the looked-up address is kept for the life of the process: a device reset is not
//     supported.
#include <cuda_runtime.h>
#include <mutex>
#include <stdint.h>
#include <string.h>

#include "../../include/colimoe.h"
#include "common.cuh"
#include "gemv.cuh"

namespace {

constexpr size_t kStaticScratchBytes = 4u << 20;
constexpr size_t kHeaderBytes = 256;
constexpr int kMaxDevices = 64;

// The scratch itself.  In host code the name is only a host-side stand-in for the device
// symbol: its device address comes from cudaGetSymbolAddress below.
static __device__ __align__(256) uint8_t g_scratch[kStaticScratchBytes];

struct DeviceScratch {
    void* addr = nullptr;
    int sms = 0;
    size_t smem_optin = 0;
};
DeviceScratch g_dev[kMaxDevices];
std::mutex g_mu;

// Set-up once per device, with that device current.
bool scratch_for_current_device(DeviceScratch& out)
{
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return false;
    std::lock_guard<std::mutex> lk(g_mu);
    DeviceScratch& d = g_dev[dev];
    if (!d.addr) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_scratch) != cudaSuccess || !p) return false;
        int sms = 0, optin = 0;
        if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev) !=
                cudaSuccess)
            return false;
        d.sms = sms;
        d.smem_optin = (size_t)optin;
        d.addr = p;
    }
    out = d;
    return true;
}

inline bool al16(const void* p) { return ((uintptr_t)p & 15u) == 0; }

}  // namespace

extern "C" coli_status coli_moe_forward_noalloc(const coli_moe_dims* d, const coli_moe_weights* wt,
                                                const float* x, int32_t T, const float* w,
                                                const int32_t* union_ids, const int32_t* n_union,
                                                const int32_t* offsets, const int32_t* assign,
                                                const float* residual, float* y, void* stream)
{
    if (!d || d->hidden < 64 || d->inter < 64 || d->hidden % 64 || d->inter % 64 ||
        d->n_experts < 1 || d->n_experts > 1024 || d->top_k < 1 || d->top_k > d->n_experts ||
        d->top_k > 32 || (d->n_shared != 0 && d->n_shared != 1) || T < 0)
        return COLI_EINVAL;
    if (T == 0) return COLI_OK;
    if (!wt || !wt->experts || !al16(wt->experts) || (d->n_shared && (!wt->shared || !al16(wt->shared))) ||
        wt->expert_stride % 256 ||
        wt->expert_stride < coli_moe_blob_bytes(d->hidden, d->inter) || !x || !al16(x) || !w ||
        !union_ids || !n_union || !offsets || !assign || !y || !al16(y) ||
        (residual && !al16(residual)))
        return COLI_EINVAL;
    const size_t h_bytes = (size_t)T * (d->top_k + d->n_shared) * d->inter * sizeof(float);
    if (kHeaderBytes + h_bytes > kStaticScratchBytes) return COLI_ENOMEM;

    DeviceScratch ds;
    if (!scratch_for_current_device(ds)) return COLI_ECUDA;
    cudaStream_t s = (cudaStream_t)stream;
    uint8_t* base = static_cast<uint8_t*>(ds.addr);

    coli::GemvParams ps[2];
    coli::GemvConfig cs[2];
    for (int mode = 0; mode < 2; mode++) {
        coli::GemvParams& p = ps[mode];
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
        p.x = mode == 0 ? x : nullptr;
        p.union_ids = union_ids;
        p.n_union = n_union;
        p.offsets = offsets;
        p.assign = assign;
        p.wts = w;
        p.hd = base + kHeaderBytes;
        p.y = mode == 1 ? y : nullptr;
        p.residual = mode == 1 ? residual : nullptr;
        p.status = reinterpret_cast<uint32_t*>(base);
        if (!coli::gemv_plan(mode, p, cs[mode], ds.sms, ds.smem_optin)) return COLI_EUNSUPPORTED;
    }
    if (cudaMemsetAsync(base, 0, kHeaderBytes, s) != cudaSuccess) return COLI_ECUDA;
    for (int mode = 0; mode < 2; mode++)
        if (coli::gemv_launch(mode, ps[mode], cs[mode], s) != cudaSuccess) return COLI_ECUDA;
    return COLI_OK;
}

extern "C" coli_status coli_moe_noalloc_read_status(uint32_t* status, void* stream)
{
    if (!status) return COLI_EINVAL;
    DeviceScratch ds;
    if (!scratch_for_current_device(ds)) return COLI_ECUDA;
    uint32_t v = 0;
    cudaError_t e = cudaMemcpyAsync(&v, ds.addr, sizeof(v), cudaMemcpyDeviceToHost, (cudaStream_t)stream);
    if (e == cudaSuccess) e = cudaStreamSynchronize((cudaStream_t)stream);
    if (e != cudaSuccess) return COLI_ECUDA;
    *status = v;
    if (v & COLI_DEV_TIMEOUT) return COLI_ETIMEOUT;
    return v ? COLI_EDEVICE : COLI_OK;
}
