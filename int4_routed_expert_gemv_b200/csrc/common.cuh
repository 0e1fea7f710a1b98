// Device helpers shared by the kernels of the routed int4 MoE library (sm_100a).
#pragma once
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace coli {

// Sticky error bits in the workspace header (OR-ed by kernels, cleared by workspace init).
enum DeviceFlag : uint32_t {
    DEV_NONFINITE = 1u,   // router produced a non-finite logit (NaN/Inf in x, W_r or bias)
    DEV_BAD_INDEX = 2u,   // union saw an expert id outside [0,E) or repeated within a token
    DEV_TIMEOUT = 4u,     // a bounded wait on an mbarrier gave up
    DEV_BAD_SHAPE = 8u,   // a kernel was handed a shape it cannot process
};

// First 256 bytes of every workspace.
struct WsHeader {
    uint32_t status;         // DeviceFlag bits
    uint32_t route_ticket;   // router last-block election counter (returns to 0 after use)
    int32_t path;            // last forward path: 0 fp32 GEMV, 1 bf16 grouped GEMM
    uint32_t timeout_site;   // which wait timed out (diagnostics)
    uint32_t launch_gen;     // fused decode launches completed on this workspace
    uint32_t reserved[59];
};
static_assert(sizeof(WsHeader) == 256, "header is 256 bytes");

constexpr uint64_t kWaitBudgetNs = 2000000000ull;   // 2 s: far above any legitimate wait

__device__ __forceinline__ void set_flag(uint32_t* status, uint32_t f) { atomicOr(status, f); }

__device__ __forceinline__ uint64_t globaltimer()
{
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

__device__ __forceinline__ uint32_t smem_u32(const void* p)
{
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// ---------------------------------------------------------------------------------------
// mbarrier (shared memory transaction barrier)
// ---------------------------------------------------------------------------------------
__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count)
{
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count)
                 : "memory");
}

__device__ __forceinline__ void fence_barrier_init()
{
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes)
{
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)),
                 "r"(bytes)
                 : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar)
{
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity)
{
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity)
        : "memory");
    return ok != 0;
}

// Wait until the barrier phase with the given parity has completed.  Gives up after about
// kWaitBudgetCycles SM clock cycles (about 2 s at the B200's clocks), records DEV_TIMEOUT
// and returns false.  The budget is kept with the SM-local cycle counter: reading it costs
// a cycle, where the global nanosecond timer is a slow, coarse register.
constexpr long long kWaitBudgetCycles = 4000000000LL;
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity, uint32_t* status,
                                          uint32_t site)
{
    if (mbar_try_wait(bar, parity)) return true;
    const long long t0 = clock64();
    while (true) {
        if (mbar_try_wait(bar, parity)) return true;
        if (clock64() - t0 > kWaitBudgetCycles) {
            set_flag(status, DEV_TIMEOUT);
            atomicExch(status + 3, site);   // WsHeader::timeout_site
            return false;
        }
    }
}

// ---------------------------------------------------------------------------------------
// Bulk asynchronous copy global -> shared (TMA engine, no tensor map), completing on an
// mbarrier.  Both addresses 16-byte aligned, size a multiple of 16.
// ---------------------------------------------------------------------------------------
__device__ __forceinline__ uint64_t policy_evict_first()
{
    uint64_t pol;
    asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(pol));
    return pol;
}

// Orders this thread's earlier generic-proxy accesses to global memory (and what they
// observed) before its later asynchronous-proxy (bulk copy) accesses.
__device__ __forceinline__ void fence_proxy_async_global()
{
    asm volatile("fence.proxy.async.global;" ::: "memory");
}

__device__ __forceinline__ void bulk_g2s(void* smem_dst, const void* gsrc, uint32_t bytes,
                                         uint64_t* bar)
{
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::
            "r"(smem_u32(smem_dst)),
        "l"(gsrc), "r"(bytes), "r"(smem_u32(bar))
        : "memory");
}

__device__ __forceinline__ void bulk_g2s_hint(void* smem_dst, const void* gsrc, uint32_t bytes,
                                              uint64_t* bar, uint64_t policy)
{
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint "
        "[%0], [%1], %2, [%3], %4;" ::"r"(smem_u32(smem_dst)),
        "l"(gsrc), "r"(bytes), "r"(smem_u32(bar)), "l"(policy)
        : "memory");
}

// Asynchronous 16-byte copy global -> shared through L2 (cp.async.cg); groups of them are
// committed and awaited per thread.
__device__ __forceinline__ void cp_async16(void* smem_dst, const void* gsrc)
{
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_u32(smem_dst)), "l"(gsrc) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait()
{
    asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

// Programmatic dependent launch.  launch_dependents lets the next kernel of the stream
// (launched with programmatic stream serialization) be scheduled before this one ends;
// wait blocks until the kernels this one depends on have completed and their memory is
// visible.  Both are no-ops for kernels launched without the attribute.
__device__ __forceinline__ void pdl_launch_dependents()
{
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

// Named barrier over a subset of warps (id 0 is __syncthreads).
__device__ __forceinline__ void named_bar(uint32_t id, uint32_t nthreads)
{
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}

// ---------------------------------------------------------------------------------------
// Packed fp32 pairs (Blackwell f32x2 arithmetic)
// ---------------------------------------------------------------------------------------
__device__ __forceinline__ uint64_t pk2(uint32_t lo, uint32_t hi)
{
    uint64_t r;
    asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "r"(lo), "r"(hi));
    return r;
}

__device__ __forceinline__ uint64_t pk2f(float lo, float hi)
{
    return pk2(__float_as_uint(lo), __float_as_uint(hi));
}

__device__ __forceinline__ float2 unpk2(uint64_t v)
{
    uint32_t lo, hi;
    asm("mov.b64 {%0, %1}, %2;" : "=r"(lo), "=r"(hi) : "l"(v));
    return make_float2(__uint_as_float(lo), __uint_as_float(hi));
}

__device__ __forceinline__ uint64_t ffma2(uint64_t a, uint64_t b, uint64_t c)
{
    uint64_t d;
    asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
    return d;
}

__device__ __forceinline__ uint64_t fmul2(uint64_t a, uint64_t b)
{
    uint64_t d;
    asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
    return d;
}

__device__ __forceinline__ uint64_t fadd2(uint64_t a, uint64_t b)
{
    uint64_t d;
    asm("add.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
    return d;
}

// (a & b) ^ c in one instruction
__device__ __forceinline__ uint32_t and_xor(uint32_t a, uint32_t b, uint32_t c)
{
    uint32_t d;
    asm("lop3.b32 %0, %1, %2, %3, 0x6a;" : "=r"(d) : "r"(a), "r"(b), "r"(c));
    return d;
}

}  // namespace coli
