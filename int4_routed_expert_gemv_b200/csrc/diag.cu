// Diagnostic entry: the failure path of the library's bounded device waits.
//
// Every wait of the kernels on an mbarrier, a flag or a counter gives up after a budget of
// SM clock cycles: it records COLI_DEV_TIMEOUT and the wait's site in the workspace
// header and returns, so the kernel ends and the context stays usable.  In normal runs
// nothing ever waits that long.  coli_debug_wait_timeout runs one such wait, with the
// budget the caller gives, on an mbarrier that nothing arrives at, so that a test can
// watch the budget run out and check what the host sees afterwards.
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/colimoe.h"
#include "common.cuh"

namespace {

constexpr uint32_t kDebugWaitSite = 99;

__global__ void wait_never_kernel(uint32_t* status, long long budget, int* returned)
{
    __shared__ __align__(8) uint64_t bar;
    if (threadIdx.x == 0) {
        coli::mbar_init(&bar, 1);
        coli::fence_barrier_init();
    }
    __syncwarp();
    // phase 0 never completes: nothing arrives
    const long long t0 = clock64();
    bool ok = false;
    while (!ok) {
        ok = coli::mbar_try_wait(&bar, 0u);
        if (!ok && clock64() - t0 > budget) break;
    }
    if (!ok && threadIdx.x == 0) {
        coli::set_flag(status, coli::DEV_TIMEOUT);
        atomicExch(status + 3, kDebugWaitSite);   // WsHeader::timeout_site
    }
    if (threadIdx.x == 0) *returned = ok ? 2 : 1;
}

}  // namespace

extern "C" coli_status coli_debug_wait_timeout(void* ws, size_t ws_bytes, uint64_t budget_cycles,
                                               int32_t* returned, void* stream)
{
    if (!ws || ws_bytes < sizeof(coli::WsHeader) || !returned || budget_cycles == 0 ||
        budget_cycles > (1ull << 32))
        return COLI_EINVAL;
    wait_never_kernel<<<1, 32, 0, (cudaStream_t)stream>>>(static_cast<uint32_t*>(ws), (long long)budget_cycles,
                                                           returned);
    return cudaGetLastError() == cudaSuccess ? COLI_OK : COLI_ECUDA;
}

namespace coli {
int fused_phase_stamps(unsigned long long* host, int max_ctas, int* n_stamps);
}

// Phase stamps of the last fused launch (a library built with COLI_PHASE_STAMPS; the
// regular build returns COLI_EUNSUPPORTED).
extern "C" coli_status coli_debug_phase_stamps(uint64_t* stamps, int32_t max_ctas, int32_t* n_ctas,
                                              int32_t* n_stamps)
{
    if (!stamps || !n_ctas || !n_stamps || max_ctas < 1) return COLI_EINVAL;
    int ns = 0;
    const int n = coli::fused_phase_stamps(reinterpret_cast<unsigned long long*>(stamps), max_ctas, &ns);
    if (n < 0) return COLI_ECUDA;
    *n_ctas = n;
    *n_stamps = ns;
    return ns == 0 ? COLI_EUNSUPPORTED : COLI_OK;
}

