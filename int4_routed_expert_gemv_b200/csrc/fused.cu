// Fused decode kernel: whole routed MoE layers in one persistent launch.
//
// Per layer and decode batch (T <= 4 tokens) the launch runs the pages' per-token path --
// the router picks experts, the batch union lists each distinct expert once, the experts
// run (colibri technical article "colibri 技术解读", section "引擎结构：一个 C 文件，五步
// token 路径"; README.zh-CN "工作原理 / 绝不为同一次磁盘读取等待两遍", 批量并集) -- and,
// for a residual stack, keeps the residual stream on the device from layer to layer
// (README.zh-CN, same section, COLI_CUDA_PIPE=2):
//
//   n  = RMSNorm(x)                                   (stacks only)
//   l  = n . W_r^T + b, top-k, renormalised softmax   (fp64 sums, fp32 logits)
//   h  = silu(G n) * (U n)     per union expert and the shared expert
//   y  = residual + D_s h_s + sum_slot w * D_e h_e
//
// One CTA per SM, two warp roles:
//   * a control warp streams every weight the CTA needs -- its share of the router rows,
//     gate/up row tiles (8 rows of G beside the same 8 rows of U), its rows of each down
//     matrix -- through a ring of shared-memory slots with the bulk-copy engine, in the order
//     the consumers use them; router rows and the shared expert do not depend on the
//     routing, so they stream first.  Between those and the routed experts the same warp
//     decides the routing (logits from the router partial sums, top-k, union) and
//     publishes it to the CTA in shared memory.  A block of consecutive rows arrives as
//     four contiguous chunks whose shared-memory starts are 32 bytes apart modulo 128, and
//     the four rows a half-warp reads together come from the four chunks, so the reads
//     hit distinct banks while a copy still moves kilobytes of consecutive rows;
//   * 12 consumer warps split each row tile's input columns between them and run the int4
//     dot products on the tensor cores: mma.sync m16n8k32 s8 x s8 -> s32, with the
//     weights as A (nibble q placed in the high half of a byte, i.e. 16 q, two
//     instructions per four weights) and the activations as B.  An activation value is
//     written as X = x * 126 / m = a + b/254 + c/254^2 with balanced int8 digits (m: the
//     token's largest magnitude for the layer input, the 64-column group's for h); the
//     three digit planes (and the two tokens of a pair) are the MMA's columns, so one
//     instruction forms exact integer sums for all of them.  Each group's sums are scaled
//     by the weight row's fp16 scale in fp32; the planes are combined at the end of the
//     row.  The last warp to finish a stage sums the warps' partials (SwiGLU into h, or
//     the routing-weighted combine into the CTA's output rows); nobody waits for it.
// Work is split statically: router items and gate/up stages over the CTAs, down rows as
// one contiguous range per CTA, so every CTA combines its output rows over the segments in
// a fixed order (shared expert, then the union in ascending expert order) and results are
// reproducible bit for bit.  Cross-CTA dependencies: router partials -> routing (a
// counter), gate/up -> down (each h value carries the launch and layer it belongs to, so
// readers check the data itself and writers need no fence), layer output -> next layer
// (a counter).  Every wait is bounded and marks the status word on time-out, so no launch
// can hang.
#include "common.cuh"
#include "fused.cuh"
#include "select.cuh"

namespace coli {
namespace {

constexpr int NCW = 12;               // consumer warps
constexpr int NCT = NCW * 32;         // consumer threads
constexpr int NTHR = NCT + 64;        // + the control warp + the reducer warp: 14 warps, at
                                      // most 4 per SM sub-partition -> 128 registers/thread
constexpr int kMaxSlots = 8;

// plane weights: A holds 16 q; digits a, b/254, c/254^2
constexpr float kPf0 = 1.0f / 16.0f;
constexpr float kPf1 = 1.0f / (16.0f * 254.0f);
constexpr float kPf2 = 1.0f / (16.0f * 254.0f * 254.0f);

constexpr int kDigBufs = 4;   // pair mode: digit rows of h in flight per CTA

// Phase stamps (builds with COLI_PHASE_STAMPS only; compiled out otherwise): one thread
// per CTA writes the global nanosecond timer at the phase boundaries of the launch's last
// layer, stamp i of CTA b at g_phase[b * kStamps + i].
constexpr int kStamps = 16;
constexpr int kStampCtas = 256;
enum : int {
    ST_START = 0,        // kernel entry
    ST_INPUT = 1,        // consumers: layer input loaded, scales formed
    ST_ROUTER = 2,       // consumers: router partial sums published
    ST_XOP = 3,          // consumers: input operand built
    ST_TABLE = 4,        // control warp: routing table ready
    ST_GU_ROUTED = 5,    // consumers: first routed gate/up stage begins
    ST_DOWN = 6,         // consumers: first down stage begins
    ST_DOWN_DONE = 7,    // consumers: last down stage done
    ST_REDUCED = 8,      // reducer: last reduction done
    ST_EXIT = 9,         // kernel exit
};
#ifdef COLI_PHASE_STAMPS
__device__ unsigned long long g_phase[kStampCtas * kStamps];
__device__ __forceinline__ void stamp(bool on, int i)
{
    if (on && blockIdx.x < kStampCtas) {
        if (i == ST_START)   // the CTA's row of the previous launch is cleared first
            for (int j = 1; j < kStamps; j++) g_phase[blockIdx.x * kStamps + j] = 0ull;
        unsigned long long t;
        asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
        g_phase[blockIdx.x * kStamps + i] = t;
    }
}
#else
__device__ __forceinline__ void stamp(bool, int) {}
#endif

struct Head {
    uint64_t full[kMaxSlots];
    uint64_t empty[kMaxSlots];
    uint64_t route_bar;
    int dead;
    uint32_t gen;                // launch generation (h epochs)
    uint64_t red_full[8];        // partial-sum buffer b: every consumer warp delivered
    uint64_t red_empty[8];       // partial-sum buffer b: summed, free again
    uint64_t dg_full[kDigBufs];  // pair mode: digit row buffer b filled (one bulk copy)
    uint64_t dg_empty[kDigBufs]; // pair mode: every consumer warp has read buffer b
    double rsq[NCW][kFusedMaxT];
    double rnorm[kFusedMaxT];
    float amax[NCW][kFusedMaxT];
    float xinv[kFusedMaxT];      // 126 / max|x_t| of the layer input (0 for a zero row)
    float xfac[kFusedMaxT];      // max|x_t| / 126
    int sh_tok[kFusedMaxT];      // the shared expert's segment: every token, weight 1
    float sh_wt[kFusedMaxT];
};

// Routing of one layer as the CTA uses it (shared memory, two copies by layer parity).
// Segment 0 is the shared expert when there is one, then the union in ascending order.
struct Table {
    int* hdr;    // [0] segments, [1] union size
    int* e;      // expert id (-1: shared)
    int* cnt;    // tokens of the segment
    int* base;   // first h row of the segment
    int* tok;    // [seg][kFusedMaxT] token ids, ascending
    float* wt;   // [seg][kFusedMaxT] routing weights (1 for the shared expert)
};

__host__ __device__ constexpr uint32_t table_bytes(int S)
{
    return (uint32_t)(2 + 3 * S + 2 * kFusedMaxT * S) * 4u;
}

__device__ __forceinline__ Table table_at(uint8_t* base, int S)
{
    Table t;
    int* w = reinterpret_cast<int*>(base);
    t.hdr = w;
    t.e = w + 2;
    t.cnt = t.e + S;
    t.base = t.cnt + S;
    t.tok = t.base + S;
    t.wt = reinterpret_cast<float*>(t.tok + kFusedMaxT * S);
    return t;
}

// One segment's tokens as a consumer uses them.
struct Seg {
    int c, base;
    const int* tok;     // shared memory
    const float* wt;
};

__device__ __forceinline__ Seg seg_of(const Table& tb, int s)
{
    Seg g;
    g.c = tb.cnt[s];
    g.base = tb.base[s];
    g.tok = tb.tok + s * kFusedMaxT;
    g.wt = tb.wt + s * kFusedMaxT;
    return g;
}

// ---------------------------------------------------------------------------------------
// small device helpers
// ---------------------------------------------------------------------------------------
__device__ __forceinline__ uint32_t ld_acquire(const uint32_t* p)
{
    uint32_t v;
    asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}

__device__ __forceinline__ unsigned long long ld_acquire64(const unsigned long long* p)
{
    unsigned long long v;
    asm volatile("ld.acquire.gpu.global.u64 %0, [%1];" : "=l"(v) : "l"(p) : "memory");
    return v;
}

__device__ __forceinline__ void red_release_add(uint32_t* p, uint32_t v)
{
    asm volatile("red.release.gpu.global.add.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}

__device__ __forceinline__ bool timed_out(uint32_t* status)
{
    return (*reinterpret_cast<volatile uint32_t*>(status) & DEV_TIMEOUT) != 0u;
}

__device__ __forceinline__ void give_up(uint32_t* status, uint32_t site, volatile int* dead)
{
    if (!timed_out(status)) {
        set_flag(status, DEV_TIMEOUT);
        atomicExch(status + 3, site);   // WsHeader::timeout_site
    }
    *dead = 1;
}

// The slow checks of a polling loop: whether any CTA has given up (a global read, an L2 round
// trip) and whether this wait is over its budget.  A loop calls this once per poll, and
// the checks run on every 1024th call only, so that a poll that succeeds is seen at once.
__device__ __forceinline__ bool wait_expired(uint32_t& n, long long t0, uint32_t* status)
{
    if ((++n & 1023u) != 0u) return false;
    return timed_out(status) || clock64() - t0 > kWaitBudgetCycles;
}

// Wait until *p >= target (acquire).  Bounded: after the budget, or once any CTA has timed
// out, the CTA is marked dead and the wait returns false.
__device__ __forceinline__ bool gwait(const uint32_t* p, uint32_t target, uint32_t* status, uint32_t site,
                      volatile int* dead)
{
    if (*dead) return false;
    if (ld_acquire(p) >= target) return true;
    const long long t0 = clock64();
    uint32_t npoll = 0;
    while (true) {
        __nanosleep(128);   // polls leave the issue slots to the working warps
        if (ld_acquire(p) >= target) return true;
        if (wait_expired(npoll, t0, status)) {
            give_up(status, site, dead);
            return false;
        }
    }
}

// mbarrier phase wait that suspends the thread in hardware (up to ~0.1 ms per try) instead
// of spinning, so waiting warps leave the issue slots to the working ones.
__device__ __forceinline__ bool mbar_try_wait_sleep(uint64_t* bar, uint32_t parity)
{
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity), "r"(100000u)
        : "memory");
    return ok != 0;
}

__device__ __forceinline__ bool mwait(uint64_t* bar, uint32_t parity, uint32_t* status, uint32_t site,
                      volatile int* dead)
{
    if (mbar_try_wait(bar, parity)) return true;
    if (*dead) return false;
    const long long t0 = clock64();
    uint32_t npoll = 0;
    while (true) {
        if (mbar_try_wait_sleep(bar, parity)) return true;
        if (*dead) return false;
        if (wait_expired(npoll, t0, status)) {
            give_up(status, site, dead);
            return false;
        }
    }
}

// Wait until the shared-memory word *p >= target (another warp of the CTA sets it).
__device__ __forceinline__ bool swait(const int* p, int target, uint32_t* status, uint32_t site, volatile int* dead)
{
    const volatile int* vp = p;
    if (*vp >= target) return true;
    const long long t0 = clock64();
    uint32_t npoll = 0;
    while (true) {
        __nanosleep(32);
        if (*vp >= target) return true;
        if (*dead) return false;
        if (wait_expired(npoll, t0, status)) {
            give_up(status, site, dead);
            return false;
        }
    }
}

// A[16 x 32] (s8, row) x B[32 x 8] (s8, col) + D -> D (s32)
__device__ __forceinline__ void mma_s8(int (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                       uint32_t a3, uint32_t b0, uint32_t b1)
{
    asm("mma.sync.aligned.m16n8k32.row.col.s32.s8.s8.s32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
        "{%8,%9}, {%0,%1,%2,%3};"
        : "+r"(d[0]), "+r"(d[1]), "+r"(d[2]), "+r"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// Four packed nibbles pairs -> signed bytes 16 q: even columns (low nibbles) and odd
// columns (high nibbles) of the word.
__device__ __forceinline__ uint32_t nib_lo(uint32_t w) { return (w << 4) & 0xF0F0F0F0u; }
__device__ __forceinline__ uint32_t nib_hi(uint32_t w) { return w & 0xF0F0F0F0u; }

// Round to nearest even for |v| < 2^22: the integer and its float value.
__device__ __forceinline__ int rint_small(float v, float& vf)
{
    const float t = __fadd_rn(v, 12582912.0f);
    vf = __fsub_rn(t, 12582912.0f);
    return __float_as_int(t) - 0x4B400000;
}

__device__ __forceinline__ uint32_t pack4(int a, int b, int c, int d)
{
    return __byte_perm(__byte_perm(a, b, 0x0040), __byte_perm(c, d, 0x0040), 0x5410);
}

// Lane l holds activations 4l..4l+3 of 128 consecutive columns (lanes 0-15 the first
// 64-column group, 16-31 the second).  Each value becomes three balanced int8 digits of
// X = x * 126 / m (m = the group's largest magnitude): X ~ a + b/254 + c/254^2, |error| <=
// 0.5/254^2 + rounding, a in [-126, 126], b, c in [-127, 127].  The lane's three plane
// words (4 digits each, column order) go to wd[plane]; returns m of its group.
__device__ __forceinline__ float digit_words(float4 v, uint32_t (&wd)[3])
{
    float mx = fmaxf(fmaxf(fabsf(v.x), fabsf(v.y)), fmaxf(fabsf(v.z), fabsf(v.w)));
    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 4));
    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 8));
    const float inv = mx > 0.0f ? 126.0f / mx : 0.0f;
    const float xs[4] = {v.x, v.y, v.z, v.w};
    int da[4], db[4], dc[4];
#pragma unroll
    for (int i = 0; i < 4; i++) {
        const float X = fminf(fmaxf(xs[i] * inv, -126.0f), 126.0f);
        float af, bf, cf;
        da[i] = rint_small(X, af);
        const float e1 = (X - af) * 254.0f;
        db[i] = rint_small(e1, bf);
        const float e2 = (e1 - bf) * 254.0f;
        dc[i] = rint_small(e2, cf);
    }
    wd[0] = pack4(da[0], da[1], da[2], da[3]);
    wd[1] = pack4(db[0], db[1], db[2], db[3]);
    wd[2] = pack4(dc[0], dc[1], dc[2], dc[3]);
    return mx;
}

// digit_words with the lane's three plane words stored to sc[plane * 32 + lane].
__device__ __forceinline__ float digits128(float4 v, int lane, uint32_t* sc)
{
    uint32_t wd[3];
    const float mx = digit_words(v, wd);
    sc[lane] = wd[0];
    sc[32 + lane] = wd[1];
    sc[64 + lane] = wd[2];
    return mx;
}

// As digits128 with a scale given for the whole row (inv = 126 / max|row|).
__device__ __forceinline__ void digits128_fixed(float4 v, float inv, int lane, uint32_t* sc)
{
    const float xs[4] = {v.x, v.y, v.z, v.w};
    int da[4], db[4], dc[4];
#pragma unroll
    for (int i = 0; i < 4; i++) {
        const float X = fminf(fmaxf(xs[i] * inv, -126.0f), 126.0f);
        float af, bf, cf;
        da[i] = rint_small(X, af);
        const float e1 = (X - af) * 254.0f;
        db[i] = rint_small(e1, bf);
        const float e2 = (e1 - bf) * 254.0f;
        dc[i] = rint_small(e2, cf);
    }
    sc[lane] = pack4(da[0], da[1], da[2], da[3]);
    sc[32 + lane] = pack4(db[0], db[1], db[2], db[3]);
    sc[64 + lane] = pack4(dc[0], dc[1], dc[2], dc[3]);
}

// B fragments of 64-column group gl (0/1) of the last digits128 call for the lane
// (groupID n, threadID tq): plane `plane`, columns 64 gl + 16 tq + 8 j + {0..7} split
// into even (b[2j]) and odd (b[2j+1]) columns, matching the A side's nibble expansion.
__device__ __forceinline__ void gather4(const uint32_t* sc, int plane, int gl, int tq,
                                        uint32_t (&b)[4])
{
    const uint4 w = *reinterpret_cast<const uint4*>(sc + plane * 32 + 16 * gl + 4 * tq);
    b[0] = __byte_perm(w.x, w.y, 0x6420);
    b[1] = __byte_perm(w.x, w.y, 0x7531);
    b[2] = __byte_perm(w.z, w.w, 0x6420);
    b[3] = __byte_perm(w.z, w.w, 0x7531);
}

// Activation operand of a warp's K range for MMA column tile q (token slots 0 and 1: rows
// row0 / row1, absent when !p0 / !p1): groups gbase .. gbase+gpw-1 of K columns as B
// fragments for this lane (groupID n -> slot n >> 2, plane n & 3), every element written.
// Lane l takes columns 64 (gbase + gi) + 4 l .. +3 of each pair of groups gi, gi + 1; all
// loads of the call are issued before the first digit is formed.
//   HEP false: the layer input with one scale per token (inv0 / inv1 = 126 / max|x|),
//              RMS-normalised first when NORM (n = float(x * r * gamma));
//   HEP true : SwiGLU activations h stored as (value, epoch) pairs; a pair whose epoch is
//              not `epoch` is not written yet and is read again (bounded).  Per-group
//              scales: fac receives m / 126 of the group for the lane's epilogue slot
//              (threadID >> 1).
template <int GPWM, int NTM, bool HEP>
__device__ __forceinline__ void build_tile(const void* row0, const void* row1, bool p0, bool p1,
                                           float inv0, float inv1, double rn0, double rn1,
                                           const float* gamma, uint32_t epoch, int gbase, int gpw,
                                           int q, uint32_t* sc, int lane, uint32_t (&B)[GPWM][NTM][4],
                                           float (&fac)[GPWM][NTM], uint32_t* status,
                                           volatile int* dead)
{
    constexpr int NP = (GPWM + 1) / 2;
    const int bslot = lane >> 4, plane = (lane >> 2) & 3, tq = lane & 3, fslot = tq >> 1;
    const int pl = plane < 3 ? plane : 0;
    const uint32_t keep = plane < 3 ? 0xFFFFFFFFu : 0u;
#pragma unroll
    for (int gi = 0; gi < GPWM; gi++) {
#pragma unroll
        for (int i = 0; i < 4; i++) B[gi][q][i] = 0u;
        fac[gi][q] = 0.0f;
    }
#pragma unroll 1
    for (int sl = 0; sl < 2; sl++) {
        if (!(sl ? p1 : p0)) continue;   // absent token: zeros
        const void* row = sl ? row1 : row0;
        float4 v[NP];
        bool want[NP];
#pragma unroll
        for (int pi = 0; pi < NP; pi++) {
            const int gi = 2 * pi;
            want[pi] = gi < gpw && (lane < 16 || gi + 1 < gpw);
            v[pi] = make_float4(0.f, 0.f, 0.f, 0.f);
        }
        if (HEP) {
            // (value, epoch) pairs, read until every pair carries this layer's epoch
            const long long t0 = clock64();
            uint32_t npoll = 0;
            bool ok = false;
            while (!ok) {
                ok = true;
#pragma unroll
                for (int pi = 0; pi < NP; pi++) {
                    if (want[pi]) {
                        const uint4* hp = reinterpret_cast<const uint4*>(
                            reinterpret_cast<const uint2*>(row) + 64 * (gbase + 2 * pi) + 4 * lane);
                        const uint4 a = __ldcg(hp), b = __ldcg(hp + 1);
                        ok = ok && a.y == epoch && a.w == epoch && b.y == epoch && b.w == epoch;
                        v[pi] = make_float4(__uint_as_float(a.x), __uint_as_float(a.z),
                                            __uint_as_float(b.x), __uint_as_float(b.z));
                    }
                }
                ok = __all_sync(0xffffffffu, ok);
                if (!ok && (*dead || wait_expired(npoll, t0, status))) {
                    if (lane == 0) give_up(status, 56, dead);
                    break;
                }
                if (!ok) __nanosleep(256);
            }
        } else {
#pragma unroll
            for (int pi = 0; pi < NP; pi++)
                if (want[pi])
                    v[pi] = __ldcg(reinterpret_cast<const float4*>(
                        reinterpret_cast<const float*>(row) + 64 * (gbase + 2 * pi) + 4 * lane));
            {
                const double r = sl ? rn1 : rn0;
#pragma unroll
                for (int pi = 0; pi < NP; pi++) {
                    const int c0 = 64 * (gbase + 2 * pi) + 4 * lane;
                    float4 gm = make_float4(1.f, 1.f, 1.f, 1.f);
                    if (gamma && want[pi]) gm = __ldg(reinterpret_cast<const float4*>(gamma + c0));
                    float4& x = v[pi];
                    x.x = (float)((double)x.x * r * (double)gm.x);
                    x.y = (float)((double)x.y * r * (double)gm.y);
                    x.z = (float)((double)x.z * r * (double)gm.z);
                    x.w = (float)((double)x.w * r * (double)gm.w);
                }
            }
        }
#pragma unroll
        for (int pi = 0; pi < NP; pi++) {
            const int gi = 2 * pi;
            if (gi < gpw) {
                float f0 = 0.0f, f1 = 0.0f;
                if (HEP) {
                    const float mx = digits128(v[pi], lane, sc);
                    f0 = __shfl_sync(0xffffffffu, mx, 0) * (1.0f / 126.0f);
                    f1 = __shfl_sync(0xffffffffu, mx, 16) * (1.0f / 126.0f);
                } else {
                    digits128_fixed(v[pi], sl ? inv1 : inv0, lane, sc);
                }
                __syncwarp();
                uint32_t b0[4], b1[4];
                gather4(sc, pl, 0, tq, b0);
                gather4(sc, pl, 1, tq, b1);
                __syncwarp();
                if (bslot == sl) {
#pragma unroll
                    for (int i = 0; i < 4; i++) {
                        B[gi][q][i] = b0[i] & keep;
                        if (gi + 1 < GPWM) B[gi + 1][q][i] = b1[i] & keep;
                    }
                }
                if (fslot == sl) {
                    fac[gi][q] = f0;
                    if (gi + 1 < GPWM) fac[gi + 1][q] = f1;
                }
            }
        }
    }
}

// Partial dot products of one row tile (16 MMA rows) over this warp's groups.  ra / rb: the
// lane's rows g and g + 8 (their group G starts at byte 32 G; the lane's 8 bytes at
// + 8 threadID), sa / sb: those rows' fp16 scales (one per group).  PERGROUP: multiply each
// group's sums by fac (per-group activation factors); else the activation factor is
// applied per token afterwards.
template <int GPWM, int NTM, bool PERGROUP>
__device__ __forceinline__ void tile_dot(const uint8_t* ra, const uint8_t* rb, const __half* sa,
                                         const __half* sb, int gbase, int gpw, uint32_t qmask,
                                         const uint32_t (&B)[GPWM][NTM][4],
                                         const float (&fac)[GPWM][NTM], float (&acc)[NTM][4])
{
#pragma unroll
    for (int q = 0; q < NTM; q++)
#pragma unroll
        for (int i = 0; i < 4; i++) acc[q][i] = 0.0f;
    // every warp runs GPWM groups so the groups' loads and MMAs overlap; a warp with fewer
    // (gpw) re-reads its last group against a zero operand, which adds exactly 0
#pragma unroll
    for (int gi = 0; gi < GPWM; gi++) {
        const int G = gbase + (gi < gpw ? gi : gpw - 1);
        const uint2 wa = *reinterpret_cast<const uint2*>(ra + 32 * G);
        const uint2 wb = *reinterpret_cast<const uint2*>(rb + 32 * G);
        const float s0 = __half2float(sa[G]);
        const float s1 = __half2float(sb[G]);
        const uint32_t a00 = nib_lo(wa.x), a01 = nib_lo(wb.x), a02 = nib_hi(wa.x), a03 = nib_hi(wb.x);
        const uint32_t a10 = nib_lo(wa.y), a11 = nib_lo(wb.y), a12 = nib_hi(wa.y), a13 = nib_hi(wb.y);
#pragma unroll
        for (int q = 0; q < NTM; q++) {
            if ((qmask >> q) & 1u) {
                int d0[4] = {0, 0, 0, 0}, d1[4] = {0, 0, 0, 0};
                mma_s8(d0, a00, a01, a02, a03, B[gi][q][0], B[gi][q][1]);
                mma_s8(d1, a10, a11, a12, a13, B[gi][q][2], B[gi][q][3]);
                const float f0 = PERGROUP ? s0 * fac[gi][q] : s0;
                const float f1 = PERGROUP ? s1 * fac[gi][q] : s1;
                acc[q][0] = fmaf((float)(d0[0] + d1[0]), f0, acc[q][0]);
                acc[q][1] = fmaf((float)(d0[1] + d1[1]), f0, acc[q][1]);
                acc[q][2] = fmaf((float)(d0[2] + d1[2]), f1, acc[q][2]);
                acc[q][3] = fmaf((float)(d0[3] + d1[3]), f1, acc[q][3]);
            }
        }
    }
}

// Combines the planes of the tile's accumulators and writes this warp's partial for
// (row g, token slot) and (row g + 8, token slot) into red[row][T] (stride T floats).
// xf: per-slot activation factor (max|x|/126 of the token) or null when the factors were
// applied per group.
template <int NTM>
__device__ __forceinline__ void tile_partials(const float (&acc)[NTM][4], uint32_t qmask, int lane,
                                              int nslots, float* red, int T, const float* xf)
{
    const int g = lane >> 2, t = lane & 3;
    const float pf0 = (t & 1) ? kPf2 : kPf0, pf1 = (t & 1) ? 0.0f : kPf1;
#pragma unroll
    for (int q = 0; q < NTM; q++) {
        if ((qmask >> q) & 1u) {
            float f = 1.0f;
            if (xf) {
                const int sl = 2 * q + (t >> 1);
                f = sl < T ? xf[sl] : 0.0f;
            }
            float v0 = (acc[q][0] * pf0 + acc[q][1] * pf1) * f;
            float v1 = (acc[q][2] * pf0 + acc[q][3] * pf1) * f;
            v0 += __shfl_xor_sync(0xffffffffu, v0, 1);
            v1 += __shfl_xor_sync(0xffffffffu, v1, 1);
            const int s = 2 * q + (t >> 1);
            if ((t & 1) == 0 && s < nslots) {
                red[g * T + s] = v0;
                red[(g + 8) * T + s] = v1;
            }
        }
    }
}

// ---- one-token gate/up in group pairs ------------------------------------------------
// A lane loads 16 bytes of a row (32 columns: lanes t < 2 of group 2P, t >= 2 of group
// 2P + 1) and feeds four MMAs.  The activation operand is block diagonal: columns 0-3 of
// the MMA are the digit planes of group 2P and only the k-slots of lanes t < 2 carry them,
// columns 4-7 those of group 2P + 1 from lanes t >= 2, so one accumulator holds both
// groups' sums and a lane's two columns belong to a single group (one scale per row).

// Operand of pair P of the warp's groups for the layer input (token 0): Bp[pair][8] in the
// register array B[2P + (r >> 2)][0][r & 3], r = 0..7 (MMA j uses registers 2j, 2j + 1).
template <int GPWM, int NTM>
__device__ __forceinline__ void build_x_pairs(const float* row, float inv, int gbase, int gpw, uint32_t* sc,
                                              int lane, uint32_t (&B)[GPWM][NTM][4])
{
    // row: the normalised input in shared memory
    constexpr int NP = GPWM / 2;
    const int n = lane >> 2, tq = lane & 3, plane = n & 3;
    const int pl = plane < 3 ? plane : 0;
    const bool mine = plane < 3 && (n >> 2) == (tq >> 1);
    float4 v[NP];
#pragma unroll
    for (int pi = 0; pi < NP; pi++)
        v[pi] = 2 * pi < gpw ? *reinterpret_cast<const float4*>(row + 64 * (gbase + 2 * pi) + 4 * lane)
                             : make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
    for (int pi = 0; pi < NP; pi++) {
        digits128_fixed(v[pi], inv, lane, sc);
        __syncwarp();
        // words 8 tq .. 8 tq + 7 of the plane: columns 32 tq .. 32 tq + 31 of the pair
        const uint4 w0 = *reinterpret_cast<const uint4*>(sc + pl * 32 + 8 * tq);
        const uint4 w1 = *reinterpret_cast<const uint4*>(sc + pl * 32 + 8 * tq + 4);
        __syncwarp();
        const uint32_t keep = mine ? 0xFFFFFFFFu : 0u;
        uint32_t r[8];
        r[0] = __byte_perm(w0.x, w0.y, 0x6420);
        r[1] = __byte_perm(w0.x, w0.y, 0x7531);
        r[2] = __byte_perm(w0.z, w0.w, 0x6420);
        r[3] = __byte_perm(w0.z, w0.w, 0x7531);
        r[4] = __byte_perm(w1.x, w1.y, 0x6420);
        r[5] = __byte_perm(w1.x, w1.y, 0x7531);
        r[6] = __byte_perm(w1.z, w1.w, 0x6420);
        r[7] = __byte_perm(w1.z, w1.w, 0x7531);
#pragma unroll
        for (int i = 0; i < 8; i++) B[2 * pi + (i >> 2)][0][i & 3] = r[i] & keep;
    }
}

// Operand of the warp's group pairs of h rows (one token; (value, epoch) pairs read until
// they carry `epoch`, bounded), per-group scales: the lane's factor m / 126 of its group
// (2 P + (threadID >> 1)) in fac[2 P][0].
template <int GPWM, int NTM>
__device__ __forceinline__ void build_h_pairs(const uint2* row, uint32_t epoch, int gbase, uint32_t* sc,
                                              int lane, uint32_t (&B)[GPWM][NTM][4],
                                              float (&fac)[GPWM][NTM], uint32_t* status,
                                              volatile int* dead)
{
    constexpr int NP = GPWM / 2;
    const int n = lane >> 2, tq = lane & 3, plane = n & 3;
    const int pl = plane < 3 ? plane : 0;
    const bool mine = plane < 3 && (n >> 2) == (tq >> 1);
    float4 v[NP];
    const long long t0 = clock64();
    uint32_t npoll = 0;
    bool ok = false;
    while (!ok) {
        ok = true;
#pragma unroll
        for (int pi = 0; pi < NP; pi++) {
            const uint4* hp = reinterpret_cast<const uint4*>(row + 64 * (gbase + 2 * pi) + 4 * lane);
            const uint4 a = __ldcg(hp), b = __ldcg(hp + 1);
            ok = ok && a.y == epoch && a.w == epoch && b.y == epoch && b.w == epoch;
            v[pi] = make_float4(__uint_as_float(a.x), __uint_as_float(a.z), __uint_as_float(b.x),
                                __uint_as_float(b.z));
        }
        ok = __all_sync(0xffffffffu, ok);
        if (!ok && (*dead || wait_expired(npoll, t0, status))) {
            if (lane == 0) give_up(status, 56, dead);
            break;
        }
        if (!ok) __nanosleep(256);
    }
#pragma unroll
    for (int pi = 0; pi < NP; pi++) {
        const float mx = digits128(v[pi], lane, sc);
        const float m0 = __shfl_sync(0xffffffffu, mx, 0), m1 = __shfl_sync(0xffffffffu, mx, 16);
        __syncwarp();
        const uint4 w0 = *reinterpret_cast<const uint4*>(sc + pl * 32 + 8 * tq);
        const uint4 w1 = *reinterpret_cast<const uint4*>(sc + pl * 32 + 8 * tq + 4);
        __syncwarp();
        const uint32_t keep = mine ? 0xFFFFFFFFu : 0u;
        uint32_t r[8];
        r[0] = __byte_perm(w0.x, w0.y, 0x6420);
        r[1] = __byte_perm(w0.x, w0.y, 0x7531);
        r[2] = __byte_perm(w0.z, w0.w, 0x6420);
        r[3] = __byte_perm(w0.z, w0.w, 0x7531);
        r[4] = __byte_perm(w1.x, w1.y, 0x6420);
        r[5] = __byte_perm(w1.x, w1.y, 0x7531);
        r[6] = __byte_perm(w1.z, w1.w, 0x6420);
        r[7] = __byte_perm(w1.z, w1.w, 0x7531);
#pragma unroll
        for (int i = 0; i < 8; i++) B[2 * pi + (i >> 2)][0][i & 3] = r[i] & keep;
        fac[2 * pi][0] = ((tq >> 1) ? m1 : m0) * (1.0f / 126.0f);
        fac[2 * pi + 1][0] = 0.0f;
    }
}

// Two-token column tile q of the warp's groups (as build_tile lays them out: lanes 16-31
// token slot 1, lane groups by digit plane, per-group factors by threadID >> 1) from the
// digit rows of h in global memory (drow0 / drow1 for the tile's tokens, absent when !p0 /
// !p1).  Every group's (m / 126, epoch) word is read until it carries `epoch` (bounded),
// acquiring the digits written before it; then the digit words are loaded.
template <int GPWM, int NTM>
__device__ __forceinline__ void gather_tile_digits(const uint8_t* drow0, const uint8_t* drow1, bool p0, bool p1,
                                                   int I, uint32_t epoch, int gbase, int gpw, int q, int lane,
                                                   uint32_t (&B)[GPWM][NTM][4], float (&fac)[GPWM][NTM],
                                                   uint32_t* status, volatile int* dead)
{
    const int bslot = lane >> 4, plane = (lane >> 2) & 3, tq = lane & 3, fslot = tq >> 1;
    const int pl = plane < 3 ? plane : 0;
    const uint32_t keep = plane < 3 ? 0xFFFFFFFFu : 0u;
    // lane j < 2 gpw checks the word of token slot j / gpw, group j % gpw
    {
        const int js = lane / (gpw > 0 ? gpw : 1), jg = lane - js * gpw;
        const bool mine = lane < 2 * gpw && (js ? p1 : p0);
        const unsigned long long* tag = reinterpret_cast<const unsigned long long*>(
            (js ? drow1 : drow0) + 3 * (size_t)I + 8 * (size_t)(gbase + jg));
        const long long t0 = clock64();
        uint32_t npoll = 0;
        while (true) {
            const bool ok = !mine || (uint32_t)(ld_acquire64(tag) >> 32) == epoch;
            if (__all_sync(0xffffffffu, ok)) break;
            if (*dead || wait_expired(npoll, t0, status)) {
                if (lane == 0) give_up(status, 56, dead);
                break;
            }
            __nanosleep(64);
        }
        __syncwarp();
    }
    const bool pb = bslot ? p1 : p0, pf = fslot ? p1 : p0;
    const uint8_t* rb = bslot ? drow1 : drow0;
    const uint8_t* rf = fslot ? drow1 : drow0;
#pragma unroll
    for (int gi = 0; gi < GPWM; gi++) {
        uint4 w = make_uint4(0u, 0u, 0u, 0u);
        float f = 0.0f;
        if (gi < gpw) {
            if (pb) w = __ldcg(reinterpret_cast<const uint4*>(rb + (size_t)pl * I + 64 * (gbase + gi) + 16 * tq));
            if (pf) f = __uint_as_float(__ldcg(reinterpret_cast<const unsigned int*>(rf + 3 * (size_t)I +
                                                                                      8 * (size_t)(gbase + gi))));
        }
        B[gi][q][0] = __byte_perm(w.x, w.y, 0x6420) & keep;
        B[gi][q][1] = __byte_perm(w.x, w.y, 0x7531) & keep;
        B[gi][q][2] = __byte_perm(w.z, w.w, 0x6420) & keep;
        B[gi][q][3] = __byte_perm(w.z, w.w, 0x7531) & keep;
        fac[gi][q] = f;
    }
}

// Pair-form operand of the warp's groups from a digit row (planes of I bytes, then the
// (m / 126, epoch) words of the groups).
template <int GPWM, int NTM>
__device__ __forceinline__ void gather_h_pairs(const uint32_t* dig, const uint2* tags, int I, int gbase,
                                               int lane, uint32_t (&B)[GPWM][NTM][4],
                                               float (&fac)[GPWM][NTM])
{
    constexpr int NP = GPWM / 2;
    const int n = lane >> 2, tq = lane & 3, plane = n & 3;
    const int pl = plane < 3 ? plane : 0;
    const uint32_t keep = (plane < 3 && (n >> 2) == (tq >> 1)) ? 0xFFFFFFFFu : 0u;
#pragma unroll
    for (int pi = 0; pi < NP; pi++) {
        const uint32_t* src = dig + pl * (I / 4) + 32 * (gbase / 2 + pi) + 8 * tq;
        const uint4 w0 = *reinterpret_cast<const uint4*>(src);
        const uint4 w1 = *reinterpret_cast<const uint4*>(src + 4);
        uint32_t r[8];
        r[0] = __byte_perm(w0.x, w0.y, 0x6420);
        r[1] = __byte_perm(w0.x, w0.y, 0x7531);
        r[2] = __byte_perm(w0.z, w0.w, 0x6420);
        r[3] = __byte_perm(w0.z, w0.w, 0x7531);
        r[4] = __byte_perm(w1.x, w1.y, 0x6420);
        r[5] = __byte_perm(w1.x, w1.y, 0x7531);
        r[6] = __byte_perm(w1.z, w1.w, 0x6420);
        r[7] = __byte_perm(w1.z, w1.w, 0x7531);
#pragma unroll
        for (int i = 0; i < 8; i++) B[2 * pi + (i >> 2)][0][i & 3] = r[i] & keep;
        fac[2 * pi][0] = __uint_as_float(tags[gbase + 2 * pi + (tq >> 1)].x);
        fac[2 * pi + 1][0] = 0.0f;
    }
}

// Partial sums of one row tile over the warp's group pairs: ra / rb the lane's rows g and
// g + 8 (pair P at byte 64 P, the lane's 16 bytes at + 16 threadID), sa / sb their scales.
// PG: per-group activation factors (h), the lane's in fac[2 P][0] for pair P.
template <int GPWM, int NTM, bool PG>
__device__ __forceinline__ void tile_dot_pairs(const uint8_t* ra, const uint8_t* rb, const __half* sa,
                                               const __half* sb, int gbase, int lane,
                                               const uint32_t (&B)[GPWM][NTM][4],
                                               const float (&fac)[GPWM][NTM], float (&acc)[4])
{
    constexpr int NP = GPWM / 2;
    static_assert(GPWM == 4 || GPWM == 8, "pair tiles: 4 or 8 groups per warp");
    const int half = (lane & 3) >> 1;
    // the rows' scales of the warp's groups in one read each (16 or 8 bytes, aligned: the
    // warp's first group is a multiple of GPWM)
    uint32_t swa[NP], swb[NP];
    if (GPWM == 8) {
        const uint4 a = *reinterpret_cast<const uint4*>(sa + gbase);
        const uint4 b = *reinterpret_cast<const uint4*>(sb + gbase);
        swa[0] = a.x; swa[1 % NP] = a.y; swa[2 % NP] = a.z; swa[3 % NP] = a.w;
        swb[0] = b.x; swb[1 % NP] = b.y; swb[2 % NP] = b.z; swb[3 % NP] = b.w;
    } else {
        const uint2 a = *reinterpret_cast<const uint2*>(sa + gbase);
        const uint2 b = *reinterpret_cast<const uint2*>(sb + gbase);
        swa[0] = a.x; swa[1 % NP] = a.y;
        swb[0] = b.x; swb[1 % NP] = b.y;
    }
#pragma unroll
    for (int i = 0; i < 4; i++) acc[i] = 0.0f;
#pragma unroll
    for (int pi = 0; pi < NP; pi++) {
        const int G = gbase + 2 * pi;
        const uint4 wa = *reinterpret_cast<const uint4*>(ra + 32 * G);
        const uint4 wb = *reinterpret_cast<const uint4*>(rb + 32 * G);
        float s0 = __half2float(__ushort_as_half((unsigned short)(half ? swa[pi] >> 16 : swa[pi] & 0xFFFFu)));
        float s1 = __half2float(__ushort_as_half((unsigned short)(half ? swb[pi] >> 16 : swb[pi] & 0xFFFFu)));
        if (PG) {
            s0 *= fac[2 * pi][0];
            s1 *= fac[2 * pi][0];
        }
        const uint32_t xa[4] = {wa.x, wa.y, wa.z, wa.w}, xb[4] = {wb.x, wb.y, wb.z, wb.w};
        int d0[4] = {0, 0, 0, 0}, d1[4] = {0, 0, 0, 0};
#pragma unroll
        for (int j = 0; j < 4; j++) {
            const uint32_t b0 = B[2 * pi + (j >> 1)][0][2 * (j & 1)];
            const uint32_t b1 = B[2 * pi + (j >> 1)][0][2 * (j & 1) + 1];
            if (j < 2) mma_s8(d0, nib_lo(xa[j]), nib_lo(xb[j]), nib_hi(xa[j]), nib_hi(xb[j]), b0, b1);
            else mma_s8(d1, nib_lo(xa[j]), nib_lo(xb[j]), nib_hi(xa[j]), nib_hi(xb[j]), b0, b1);
        }
        acc[0] = fmaf((float)(d0[0] + d1[0]), s0, acc[0]);
        acc[1] = fmaf((float)(d0[1] + d1[1]), s0, acc[1]);
        acc[2] = fmaf((float)(d0[2] + d1[2]), s1, acc[2]);
        acc[3] = fmaf((float)(d0[3] + d1[3]), s1, acc[3]);
    }
}

// Row sums of a pair-mode tile: every lane of a row holds two planes of one group; the
// four lanes together hold the whole row (both groups, all planes).  Writes red[g] and
// red[g + 8] (one token), scaled by the token's activation factor.
__device__ __forceinline__ void tile_partials_pairs(const float (&acc)[4], int lane, float* red, float xf)
{
    const int g = lane >> 2, t = lane & 3;
    const float pf0 = (t & 1) ? kPf2 : kPf0, pf1 = (t & 1) ? 0.0f : kPf1;
    float v0 = acc[0] * pf0 + acc[1] * pf1;
    float v1 = acc[2] * pf0 + acc[3] * pf1;
    v0 += __shfl_xor_sync(0xffffffffu, v0, 1);
    v1 += __shfl_xor_sync(0xffffffffu, v1, 1);
    v0 += __shfl_xor_sync(0xffffffffu, v0, 2);
    v1 += __shfl_xor_sync(0xffffffffu, v1, 2);
    if (t == 0) {
        red[g] = v0 * xf;
        red[g + 8] = v1 * xf;
    }
}

// Partial sums go through a ring of kRedBufs buffers: stage cs (every gate/up and down
// stage, in the consumers' order) writes buffer cs % kRedBufs; each consumer warp arrives on
// the buffer's full barrier after writing its part; the reducer warp waits for it, sums
// (SwiGLU into h, or the routing-weighted combine into the CTA's output rows, in stage
// order) and arrives on the buffer's empty barrier, which a consumer waits for before it
// writes the buffer again.  No compute warp ever waits for another one.
constexpr int kRedBufs = 6;

__device__ __forceinline__ void red_wait_free(Head& hd, uint32_t cs, uint32_t* status,
                                              volatile int* dead, int lane)
{
    if (cs >= (uint32_t)kRedBufs)
        mwait(&hd.red_empty[cs % kRedBufs], ((cs / kRedBufs) - 1u) & 1u, status, 57, dead);
}

__device__ __forceinline__ void red_deliver(Head& hd, uint32_t cs, int lane)
{
    __syncwarp();
    if (lane == 0) mbar_arrive(&hd.red_full[cs % kRedBufs]);
}

// blob section offsets (bytes)
struct BlobOff {
    uint64_t gq, uq, dq, gs, us, ds;
};
__device__ __forceinline__ BlobOff blob_off(int H, int I)
{
    const uint64_t IH = (uint64_t)I * H;
    BlobOff o;
    o.gq = 0;
    o.uq = IH / 2;
    o.dq = IH;
    o.gs = 3 * IH / 2;
    o.us = o.gs + IH / 32;
    o.ds = o.us + IH / 32;
    return o;
}

// Top-k of lt[0..E) in shared memory (E <= 1024; descending, ties to the lower index):
// lane s < k returns selection s.  Lane j owns elements j + 32 i; it keeps the best key of
// its elements not yet taken (a bitmask of taken ones) and rescans them only when its best
// is the one taken.  Absent and taken elements have key 0, which no value maps to.
__device__ __forceinline__ void topk_best(const float* lt, int E, int npl, int lane, uint32_t taken,
                                          uint32_t& bk, int& bi)
{
    bk = 0u;
    bi = 0;
#pragma unroll 8
    for (int i = 0; i < npl; i++) {
        const int e = lane + 32 * i;
        const uint32_t kk = (e < E && !((taken >> i) & 1u)) ? order_key(lt[e]) : 0u;
        if (kk > bk) {
            bk = kk;
            bi = i;
        }
    }
}

__device__ __forceinline__ void topk_smem(const float* lt, int E, int k, int lane, int& e_out,
                                          uint32_t& key_out)
{
    const int npl = (E + 31) >> 5;
    uint32_t taken = 0u, bk;
    int bi;
    topk_best(lt, E, npl, lane, taken, bk, bi);
    uint32_t mine = 0u;
    int mine_e = 0;
#pragma unroll 1
    for (int s = 0; s < k; s++) {
        const uint32_t m = __reduce_max_sync(0xffffffffu, bk);
        const uint32_t cand = (bk == m) ? (uint32_t)(lane + 32 * bi) : 0xFFFFFFFFu;
        const uint32_t e = __reduce_min_sync(0xffffffffu, cand);
        if (lane == s) {
            mine = m;
            mine_e = (int)e;
        }
        if ((int)(e & 31u) == lane) {
            taken |= 1u << (e >> 5);
            topk_best(lt, E, npl, lane, taken, bk, bi);
        }
    }
    e_out = mine_e;
    key_out = mine;
}

// Exclusive prefix sum over the warp's lanes.
__device__ __forceinline__ int warp_excl_scan(int v, int lane)
{
    int x = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, x, o);
        if (lane >= o) x += y;
    }
    return x - v;
}

// Top-k from keys held in registers (E <= 256: lane j holds elements j + 32 i, i < 8) by
// threshold and rank: the k-th largest of the 32 lane maxima is at most the k-th largest
// key, so every key of the top k is at or above it.  Those candidates (C of them, about
// k) go to shared memory and each one's rank among them is counted: larger keys, and equal
// keys of a lower index, come first; a candidate's rank among the candidates is its rank
// among all keys.  Key 0 marks an absent element.  When C is above kTopkCand (many equal
// keys), the sequential selection over lt decides instead.
constexpr int kTopkCand = 128;

__device__ __forceinline__ void topk_regs(const uint32_t (&key)[8], const float* lt, int E, int k, int lane,
                                          uint2* cand, uint2* res, int& e_out, uint32_t& key_out)
{
    uint32_t lm = key[0];
#pragma unroll
    for (int i = 1; i < 8; i++) lm = max(lm, key[i]);
    int r = 0;
#pragma unroll
    for (int j = 0; j < 32; j++) {
        const uint32_t o = __shfl_sync(0xffffffffu, lm, j);
        r += (o > lm || (o == lm && j < lane)) ? 1 : 0;
    }
    const uint32_t tau = __shfl_sync(0xffffffffu, lm, __ffs(__ballot_sync(0xffffffffu, r == k - 1)) - 1);
    int cnt = 0;
#pragma unroll
    for (int i = 0; i < 8; i++) cnt += (key[i] != 0u && key[i] >= tau) ? 1 : 0;
    const int pre = warp_excl_scan(cnt, lane);
    const int C = __shfl_sync(0xffffffffu, pre + cnt, 31);
    if (C > kTopkCand) {
        topk_smem(lt, E, k, lane, e_out, key_out);
        return;
    }
    int pos = pre;
#pragma unroll
    for (int i = 0; i < 8; i++)
        if (key[i] != 0u && key[i] >= tau) cand[pos++] = make_uint2(key[i], (uint32_t)(lane + 32 * i));
    __syncwarp();
#pragma unroll 1
    for (int ci = lane; ci < C; ci += 32) {
        const uint2 me = cand[ci];
        int rank = 0;
#pragma unroll 4
        for (int j = 0; j < C; j++) {
            const uint2 o = cand[j];
            rank += (o.x > me.x || (o.x == me.x && o.y < me.y)) ? 1 : 0;
        }
        if (rank < k) res[rank] = me;
    }
    __syncwarp();
    const uint2 mine = lane < k ? res[lane] : make_uint2(0u, 0u);
    e_out = (int)mine.y;
    key_out = mine.x;
    __syncwarp();
}

// Union of sel[t * k + s] (T * k <= 128 assignments, each token's experts distinct and in
// [0, E)) in ascending expert order: writes the routed segments of the table (after
// n_shared leading segments) and, when `out` is set, union_ids / n_union / offsets / assign.
// Scratch `bits`: per token 32 words of expert bits, then per expert word its union prefix,
// union bits and the number of assignments in lower words.
__device__ __forceinline__ void build_union(const int* sel, const float* selw, int T, int k, int E, int ns,
                            uint32_t* bits, Table tb, bool out, const FusedParams& p, int lane)
{
    const int nw = (E + 31) / 32;
    const int n = T * k;
    uint32_t* wp = bits + kFusedMaxT * 32;
#pragma unroll 1
    for (int i = lane; i < kFusedMaxT * 32; i += 32) bits[i] = 0u;
    __syncwarp();
#pragma unroll 1
    for (int a = lane; a < n; a += 32) {
        const int e = sel[a];
        atomicOr(&bits[(a / k) * 32 + (e >> 5)], 1u << (e & 31));
    }
    __syncwarp();
    uint32_t uw = 0u;
    int cw = 0;
#pragma unroll 1
    for (int t = 0; t < T; t++) {
        const uint32_t bw = lane < nw ? bits[t * 32 + lane] : 0u;
        uw |= bw;
        cw += __popc(bw);
    }
    const int upre = warp_excl_scan(__popc(uw), lane);
    const int nu = __shfl_sync(0xffffffffu, upre + __popc(uw), 31);
    wp[lane] = (uint32_t)upre;
    wp[32 + lane] = uw;
    wp[64 + lane] = (uint32_t)warp_excl_scan(cw, lane);
    __syncwarp();
#pragma unroll 1
    for (int a = lane; a < n; a += 32) {
        const int e = sel[a], t = a / k, w = e >> 5;
        const uint32_t below = (1u << (e & 31)) - 1u;
        // rank of the assignment: those of lower experts, then this expert's earlier tokens
        int off = (int)wp[64 + w], before_t = 0, count = 0;
#pragma unroll 1
        for (int tt = 0; tt < T; tt++) {
            const uint32_t bw = bits[tt * 32 + w];
            const int hit = (bw >> (e & 31)) & 1;
            off += __popc(bw & below);
            count += hit;
            before_t += tt < t ? hit : 0;
        }
        const int u = (int)wp[w] + __popc(wp[32 + w] & below);
        const int seg = ns + u;
        if (before_t == 0) {
            tb.e[seg] = e;
            tb.cnt[seg] = count;
            tb.base[seg] = off;
            if (out) {
                p.union_ids[u] = e;
                p.offsets[u] = off;
            }
        }
        tb.tok[seg * kFusedMaxT + before_t] = t;
        tb.wt[seg * kFusedMaxT + before_t] = selw[a];
        if (out) p.assign[off + before_t] = a;
    }
    if (out) {
#pragma unroll 1
        for (int q = nu + lane; q <= E; q += 32) {
            if (q < E) p.union_ids[q] = -1;
            p.offsets[q] = n;
        }
        if (lane == 0) *p.n_union = nu;
    }
    if (lane == 0) {
        tb.hdr[0] = ns + nu;
        tb.hdr[1] = nu;
    }
}

// ---------------------------------------------------------------------------------------
// the kernel
// ---------------------------------------------------------------------------------------

// Per-CTA constants shared by the roles.
struct Ctx {
    Head* hd;
    volatile int* dead;
    uint8_t* ring;
    float* red;
    float* yacc;
    uint8_t* rt_base;
    uint32_t tbytes;
    int S;
    int tid, warp, lane, b, G;
    int r0, r1, nrows, ntd;
    int ri0, ri1;          // router items of the CTA (contiguous)
    int n_ritems;
    BlobOff bo;
};

// down rows of the CTA in four chunks: chunk q = rows [dcs(q), dcs(q + 1)) of its range
__device__ __forceinline__ int dcs(const Ctx& c, int q) { return (q * c.nrows) >> 2; }

__device__ __forceinline__ Table layer_table(const Ctx& c, int l)
{
    return table_at(c.rt_base + (l & 1) * c.tbytes, c.S);
}

__device__ __forceinline__ uint32_t* layer_cnt(const FusedParams& p, int l)
{
    return p.cnt + 1 + l * kCntPerLayer;
}

__device__ __forceinline__ uint32_t h_epoch(const Ctx& c, int l)
{
    return c.hd->gen * 32u + (uint32_t)l + 1u;
}

// ----------------------------- control warp: the weight stream --------------------------
struct Stream {
    uint32_t it;
    uint64_t pol;
    uint32_t dd;   // pair mode: digit rows copied so far (every down segment)
};

__device__ __forceinline__ uint8_t* slot_begin(const FusedParams& p, const Ctx& c, Stream& st,
                                               uint32_t bytes, uint64_t*& bar)
{
    const uint32_t s = st.it % (uint32_t)p.nslot;
    mwait(&c.hd->empty[s], ((st.it / (uint32_t)p.nslot) & 1u) ^ 1u, p.status, 31, c.dead);
    bar = &c.hd->full[s];
    mbar_arrive_expect_tx(bar, bytes);
    st.it++;
    return c.ring + (size_t)s * p.slot_bytes;
}

// this CTA's router items: items [ri0, ri1) of the E x RC item list, item i = columns
// (i % RC) * RKc .. of row i / RC, i.e. floats i * RKc .. of the row-major router matrix
__device__ __forceinline__ void issue_router(const FusedParams& p, const Ctx& c, Stream& st, const FusedLayer& ly)
{
    const uint32_t bytes = (uint32_t)(c.ri1 - c.ri0) * (uint32_t)p.RKc * 4u;
    uint64_t* bar;
    uint8_t* dst = slot_begin(p, c, st, bytes, bar);
    bulk_g2s(dst, ly.w_router + (size_t)c.ri0 * p.RKc, bytes, bar);
}

// gate/up stage of `ntl` row tiles (8 intermediate rows each) from row i0: the 8 ntl rows of
// G as four chunks of 2 ntl rows (chunk q at q * gu_chunk), the same rows of U after them,
// then the G scales and the U scales of the rows
__device__ __forceinline__ void issue_gu(const FusedParams& p, const Ctx& c, Stream& st, const uint8_t* blob, int stage)
{
    const int H = p.H, i0 = stage * 8 * p.NTSg;
    const int ntl = min(p.NTSg, (p.I - i0) / 8);
    const uint32_t rowb = (uint32_t)H / 2, cr = 2u * ntl;
    const uint32_t scb = 8u * ntl * ((uint32_t)H / 32u);
    uint64_t* bar;
    uint8_t* dst = slot_begin(p, c, st, 8u * cr * rowb + 2u * scb, bar);
#pragma unroll 1
    for (int q = 0; q < 4; q++) {
        const uint64_t r = (uint64_t)i0 + q * cr;
        bulk_g2s_hint(dst + (size_t)q * p.gu_chunk, blob + c.bo.gq + r * rowb, cr * rowb, bar, st.pol);
        bulk_g2s_hint(dst + (size_t)(4 + q) * p.gu_chunk, blob + c.bo.uq + r * rowb, cr * rowb, bar, st.pol);
    }
    bulk_g2s_hint(dst + p.gu_gsc, blob + c.bo.gs + (uint64_t)i0 * (H / 32), scb, bar, st.pol);
    bulk_g2s_hint(dst + p.gu_usc, blob + c.bo.us + (uint64_t)i0 * (H / 32), scb, bar, st.pol);
}

// down stage: the CTA's rows r0..r1 of D in four chunks (chunk q at q * d_chunk), then
// their scales from the 16-byte boundary at or below row r0's first scale
__device__ __forceinline__ void issue_down(const FusedParams& p, const Ctx& c, Stream& st, const uint8_t* blob)
{
    const int I = p.I;
    const uint32_t rowb = (uint32_t)I / 2;
    const uint64_t s0 = (uint64_t)c.r0 * (I / 32), s1 = (uint64_t)c.r1 * (I / 32);
    const uint64_t a0 = s0 & ~15ull, a1 = (s1 + 15) & ~15ull;
    uint64_t* bar;
    uint8_t* dst = slot_begin(p, c, st, (uint32_t)c.nrows * rowb + (uint32_t)(a1 - a0), bar);
#pragma unroll 1
    for (int q = 0; q < 4; q++) {
        const int n = dcs(c, q + 1) - dcs(c, q);
        if (n > 0)
            bulk_g2s_hint(dst + (size_t)q * p.d_chunk,
                          blob + c.bo.dq + (uint64_t)(c.r0 + dcs(c, q)) * rowb, (uint32_t)n * rowb,
                          bar, st.pol);
    }
    bulk_g2s_hint(dst + p.d_sc_off, blob + c.bo.ds + a0, (uint32_t)(a1 - a0), bar, st.pol);
}

// One token: the digit row of h row `row` (layer l) into digit buffer dd % kDigBufs, once
// every consumer warp has released the buffer and every group of the row carries the
// layer's epoch (bounded polls), as one bulk copy completing on the buffer's barrier.
__device__ __forceinline__ void issue_digits(const FusedParams& p, const Ctx& c, Stream& st, int l, int row)
{
    const int lane = c.lane, I = p.I, ng = I / 64;
    const uint32_t b = st.dd % (uint32_t)kDigBufs;
    if (st.dd >= (uint32_t)kDigBufs)
        mwait(&c.hd->dg_empty[b], ((st.dd / (uint32_t)kDigBufs) - 1u) & 1u, p.status, 33, c.dead);
    const uint8_t* src = p.hdg + (size_t)row * p.hdg_row;
    const unsigned long long* tags = reinterpret_cast<const unsigned long long*>(src + 3 * (size_t)I);
    const uint32_t ep = __ldcg(p.gen) * 32u + (uint32_t)l + 1u;
    const long long t0 = clock64();
    uint32_t npoll = 0;
    while (true) {
        bool ok = true;
#pragma unroll 1
        for (int g = lane; g < ng; g += 32) ok = ok && (uint32_t)(ld_acquire64(tags + g) >> 32) == ep;
        if (__all_sync(0xffffffffu, ok)) break;
        if (*c.dead || wait_expired(npoll, t0, p.status)) {
            if (lane == 0) give_up(p.status, 34, c.dead);
            break;
        }
        __nanosleep(64);
    }
    // each lane's tag reads acquire the digits written before them; the warp barrier
    // orders them before lane 0's copy, which the proxy fence orders after the reads
    __syncwarp();
    fence_proxy_async_global();
    if (lane == 0) {
        uint64_t* bar = &c.hd->dg_full[b];
        mbar_arrive_expect_tx(bar, p.hdg_row);
        bulk_g2s(reinterpret_cast<uint8_t*>(c.hd) + p.off_hdig + (size_t)b * p.hdig_bytes, src, p.hdg_row, bar);
    }
    st.dd++;
    __syncwarp();
}

// ----------------------------- control warp: routing ------------------------------------
// Renormalised softmax weight of selection `lane` (< k) from the order keys held by lanes
// 0..k-1 (descending): exp(l - l_max) / sum, in fp32 (exp to a few ulp, far inside the
// 1e-6 bar on the weights).
__device__ __forceinline__ float topk_weight_f(uint32_t key, int k, int lane)
{
    const float lmax = key_float(__shfl_sync(0xffffffffu, key, 0));
    const float ex = lane < k ? expf(key_float(key) - lmax) : 0.0f;
    float z = ex;
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) z += __shfl_xor_sync(0xffffffffu, z, o);
    return ex / z;
}

// Routing of layer l: logits from the router partial sums (summed in chunk order) into
// lt [T][E], top-k and weights per token, then the union into table tb.  `dry`: the same
// code on whatever the buffers hold (run early, while the control warp would wait anyway,
// so the real pass finds its instructions cached); it writes nothing but tb and scratch.
__device__ __forceinline__ void route_compute(const FusedParams& p, const Ctx& c, int l, Table tb, bool dry)
{
    const int T = p.T, E = p.E, k = p.k, ns = p.n_shared, lane = c.lane;
    const FusedLayer& ly = p.layer[l];
    float* lt = reinterpret_cast<float*>(reinterpret_cast<uint8_t*>(c.hd) + p.off_scratch +
                                         NCW * 96 * 4);
    int* sel = reinterpret_cast<int*>(lt + T * E);
    float* selw = reinterpret_cast<float*>(sel + T * k);
    uint32_t* bits = reinterpret_cast<uint32_t*>(selw + T * k);
    // top-k candidates and results (8-byte aligned)
    uint2* cand = reinterpret_cast<uint2*>((reinterpret_cast<uintptr_t>(bits + (kFusedMaxT + 3) * 32) + 7) & ~uintptr_t(7));
    const bool out = c.b == 0 && !dry;
    // the launch generation straight from the workspace (read after the dependency wait)
    const uint32_t ep = __ldcg(p.gen) * 32u + (uint32_t)l + 1u;
    int e_sel = 0;
    float wv = 0.0f;
#pragma unroll 1
    for (int t = 0; t < T; t++) {
        uint32_t key[8];
#pragma unroll 1
        for (int e0 = 0; e0 < E; e0 += 32 * 8) {
            // the partials of eight experts per lane and their biases in one round of loads
            double v[8];
            float bv[8];
#pragma unroll
            for (int i = 0; i < 8; i++) {
                const int e = e0 + 32 * i + lane;
                v[i] = 0.0;
                bv[i] = (ly.bias && e < E) ? __ldg(ly.bias + e) : 0.0f;
            }
#pragma unroll 1
            for (int cc = 0; cc < p.RC; cc++) {
                // poll until every partial carries this layer's epoch (the dry pass takes
                // whatever is there)
                uint4 q[8];
                const long long t0 = clock64();
                uint32_t npoll = 0;
                while (true) {
#pragma unroll
                    for (int i = 0; i < 8; i++) {
                        const int e = e0 + 32 * i + lane;
                        q[i] = e < E ? __ldcg(p.rpart + ((size_t)t * E + e) * p.RC + cc) : make_uint4(0u, ep, 0u, ep);
                    }
                    bool ok = true;
#pragma unroll
                    for (int i = 0; i < 8; i++) ok = ok && q[i].y == ep && q[i].w == ep;
                    if (dry || __all_sync(0xffffffffu, ok)) break;
                    if (*c.dead || wait_expired(npoll, t0, p.status)) {
                        if (lane == 0) give_up(p.status, 41, c.dead);
                        break;
                    }
                    __nanosleep(64);
                }
#pragma unroll
                for (int i = 0; i < 8; i++) v[i] += __hiloint2double((int)q[i].z, (int)q[i].x);
            }
#pragma unroll
            for (int i = 0; i < 8; i++) {
                const int e = e0 + 32 * i + lane;
                const float lv = (float)(v[i] + (double)bv[i]);
                key[i] = e < E ? order_key(lv) : 0u;
                if (e < E) {
                    if (!dry && !isfinite(lv)) set_flag(p.status, DEV_NONFINITE);
                    lt[t * E + e] = lv;
                    if (out && p.logits) p.logits[(size_t)t * E + e] = lv;
                }
            }
        }
        __syncwarp();
        uint32_t kv;
        if (E <= 256) topk_regs(key, lt + t * E, E, k, lane, cand, cand + kTopkCand, e_sel, kv);
        else topk_smem(lt + t * E, E, k, lane, e_sel, kv);
        wv = topk_weight_f(kv, k, lane);
        if (lane < k) {
            sel[t * k + lane] = e_sel;
            selw[t * k + lane] = wv;
            if (out && p.idx) p.idx[(size_t)t * k + lane] = e_sel;
            if (out && p.w) p.w[(size_t)t * k + lane] = wv;
            if (out && p.idx_layers) p.idx_layers[((size_t)l * T + t) * k + lane] = e_sel;
        }
    }
    __syncwarp();
    if (T == 1) {
        // one token: the union is its k experts in ascending id order, one row each
        int r = 0;
#pragma unroll 8
        for (int j = 0; j < 32; j++) {
            const int ej = __shfl_sync(0xffffffffu, e_sel, j);
            r += (j < k && ej < e_sel) ? 1 : 0;
        }
        const bool uo = out && p.union_ids != nullptr;
        if (lane < k) {
            const int seg = ns + r;
            tb.e[seg] = e_sel;
            tb.cnt[seg] = 1;
            tb.base[seg] = r;
            tb.tok[seg * kFusedMaxT] = 0;
            tb.wt[seg * kFusedMaxT] = wv;
            if (uo) {
                p.union_ids[r] = e_sel;
                p.offsets[r] = r;
                p.assign[r] = lane;
            }
        }
        if (uo) {
            for (int q = k + lane; q <= E; q += 32) {
                if (q < E) p.union_ids[q] = -1;
                p.offsets[q] = k;
            }
            if (lane == 0) *p.n_union = k;
        }
        if (lane == 0) {
            tb.hdr[0] = ns + k;
            tb.hdr[1] = k;
        }
    } else {
        build_union(sel, selw, T, k, E, ns, bits, tb, out && p.union_ids != nullptr, p, lane);
    }
    __syncwarp();
}

// warm: first run the routing code once on whatever the buffers hold (into the other
// layer's table, which is rewritten before use), so that the real pass finds its code in
// the instruction caches; both passes go through one copy of the code.
__device__ __forceinline__ void route_layer(const FusedParams& p, const Ctx& c, int l, bool warm)
{
    const int T = p.T, E = p.E, k = p.k, ns = p.n_shared, lane = c.lane;
    const Table tb = layer_table(c, l);
    uint32_t* lc = layer_cnt(p, l);
    if (p.route) {
#pragma unroll 1
        for (int pass = warm ? 0 : 1; pass < 2; pass++) {
            const bool dry = pass == 0;
            route_compute(p, c, l, dry ? layer_table(c, l + 1) : tb, dry);
        }
    } else {
        // given routing (forward call): union_ids / n_union / offsets / assign / w
        int nu = __ldcg(p.n_union);
        if (nu < 0 || nu > min(E, T * k)) {
            if (lane == 0) set_flag(p.status, DEV_BAD_INDEX);
            nu = max(0, min(nu, min(E, T * k)));
        }
#pragma unroll 1
        for (int u = lane; u < nu; u += 32) {
            const int seg = ns + u;
            int e = __ldcg(p.union_ids + u);
            int o0 = __ldcg(p.offsets + u), o1 = __ldcg(p.offsets + u + 1);
            const bool bad = e < 0 || e >= E || o0 < 0 || o1 > T * k || o1 - o0 < 1 || o1 - o0 > T;
            if (bad) {
                set_flag(p.status, DEV_BAD_INDEX);
                e = min(max(e, 0), E - 1);
                o1 = o0 = 0;
            }
            tb.e[seg] = e;
            tb.cnt[seg] = o1 - o0;
            tb.base[seg] = o0;
#pragma unroll 1
            for (int m = 0; m < o1 - o0; m++) {
                int a = __ldcg(p.assign + o0 + m);
                if (a < 0 || a >= T * k) {
                    set_flag(p.status, DEV_BAD_INDEX);
                    a = 0;
                }
                tb.tok[seg * kFusedMaxT + m] = a / k;
                tb.wt[seg * kFusedMaxT + m] = __ldcg(p.w + a);
            }
        }
        if (lane == 0) {
            tb.hdr[0] = ns + nu;
            tb.hdr[1] = nu;
        }
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&c.hd->route_bar);
}

// The control warp's order of stages (the consumers and the reducer follow the same
// order): router items; the shared expert's gate/up stages of this CTA; [routing]; the
// routed gate/up stages of this CTA (one round-robin sequence over all segments' stages);
// the down rows of every segment, the shared expert's first.  Before routing it issues
// only router items and shared stages (at most the ring's depth at the first layer), then
// routes; every issue goes through one call site per kind of stage.
__device__ __forceinline__ void control_warp(const FusedParams& p, const Ctx& c)
{
    Stream st;
    st.it = 0;
    st.dd = 0;
    st.pol = policy_evict_first();
    const int ns = p.n_shared;
#pragma unroll 1
    for (int l = 0; l < p.L; l++) {
        const FusedLayer& ly = p.layer[l];
        const Table tb = layer_table(c, l);
        if (c.lane == 0 && c.ri1 > c.ri0) issue_router(p, c, st, ly);
        int nseg = ns, gi = c.b, ds = 0;
        bool routed = false;
        while (true) {
            if (gi < nseg * p.SPS) {
                const int sg = gi / p.SPS;
                if (c.lane == 0)
                    issue_gu(p, c, st, sg < ns ? ly.shared : ly.experts + (uint64_t)tb.e[sg] * ly.stride,
                             gi - sg * p.SPS);
                gi += c.G;
            } else if (!routed) {
                __syncwarp();
                if (l == 0) pdl_wait();
                route_layer(p, c, l, l == 0);
                stamp(c.lane == 0 && l == p.L - 1, ST_TABLE);
                nseg = tb.hdr[0];
                routed = true;
            } else if (c.nrows > 0 && ds < nseg) {
                if (p.pair) issue_digits(p, c, st, l, ds < ns ? p.T * p.k : tb.base[ds]);
                if (c.lane == 0)
                    issue_down(p, c, st, ds < ns ? ly.shared : ly.experts + (uint64_t)tb.e[ds] * ly.stride);
                ds++;
            } else {
                break;
            }
        }
        __syncwarp();
    }
    // drain: every issued copy has landed before the CTA may exit (bounded)
    if (c.lane == 0) {
        const uint32_t n_last = st.it < (uint32_t)p.nslot ? st.it : (uint32_t)p.nslot;
#pragma unroll 1
        for (uint32_t q = 0; q < n_last; q++) {
            const uint32_t last = st.it - 1 - q;
            const uint32_t s = last % (uint32_t)p.nslot;
            const uint32_t par = (last / (uint32_t)p.nslot) & 1u;
            if (!mbar_try_wait(&c.hd->full[s], par)) {
                const long long t0 = clock64();
                while (!mbar_try_wait(&c.hd->full[s], par) && clock64() - t0 < kWaitBudgetCycles) {
                }
            }
        }
    }
}

// ----------------------------- consumers ------------------------------------------------
struct Cons {
    uint32_t it;    // ring position (the control warp's order)
    uint32_t cs;    // reduction stages
    uint32_t ds;    // down stages (h digit buffer parity)
    uint32_t* sc;   // this warp's digit scratch (96 words)
    int g_rs, g_kw, gbase_g, gpw_g;   // gate/up: row slot, K slot, its groups
    int d_rs, d_kw, gbase_d, gpw_d;   // down
};

__device__ __forceinline__ const uint8_t* cslot_wait(const FusedParams& p, const Ctx& c, Cons& w)
{
    const uint32_t s = w.it % (uint32_t)p.nslot;
    mwait(&c.hd->full[s], (w.it / (uint32_t)p.nslot) & 1u, p.status, 51, c.dead);
    return c.ring + (size_t)s * p.slot_bytes;
}

__device__ __forceinline__ void cslot_free(const FusedParams& p, const Ctx& c, Cons& w)
{
    __syncwarp();
    if (c.lane == 0) mbar_arrive(&c.hd->empty[w.it % (uint32_t)p.nslot]);
    w.it++;
}

// Router items of this CTA, partial logits in double.  Every consumer thread takes a share
// of every item (float4 j of the item's columns goes to thread j % NCT); the warps' sums
// per (item, token) are then added in warp order by one thread, so each partial logit has
// one fixed summation order.  With one item per router row (RC = 1) the normalised input is
// loaded once per token and kept in registers across the items.
template <bool PAIR>
__device__ __forceinline__ void router_consume(const FusedParams& p, const Ctx& c, Cons& w, int l,
                                               const float* xin)
{
    const float* gamma = p.norm ? p.layer[l].gamma : nullptr;
    const int T = p.T, E = p.E, H = p.H, RKc = p.RKc, RC = p.RC, lane = c.lane, tid = c.tid;
    const int nit = c.ri1 - c.ri0, n4 = RKc / 4;
    constexpr int U = 4;   // float4 per thread per item (RKc <= 4 NCT * 4 = 6144 columns)
    double* part = reinterpret_cast<double*>(reinterpret_cast<uint8_t*>(c.hd) + p.off_scratch);
    const uint8_t* sb = cslot_wait(p, c, w);
#pragma unroll 1
    for (int t = 0; t < T; t++) {
        const double r = c.hd->rnorm[t];
        float4 nv[U];
        int cc_have = -1;
#pragma unroll 1
        for (int it = 0; it < nit; it++) {
            const int i = c.ri0 + it, e = i / RC, cc = i - e * RC;
            if constexpr (PAIR) {
              if (cc != cc_have) {
                // one token: n is in shared memory already
                const float4* xs = reinterpret_cast<const float4*>(reinterpret_cast<const uint8_t*>(c.hd) + p.off_hstage);
#pragma unroll
                for (int j = 0; j < U; j++) {
                    const int u = tid + NCT * j;
                    nv[j] = u < n4 ? xs[cc * (RKc / 4) + u] : make_float4(0.f, 0.f, 0.f, 0.f);
                }
                cc_have = cc;
              }
            } else if (cc != cc_have) {
                // n = float(x * r * gamma): exactly x for a plain input
#pragma unroll
                for (int j = 0; j < U; j++) {
                    const int u = tid + NCT * j;
                    float4 x = make_float4(0.f, 0.f, 0.f, 0.f), gm = make_float4(1.f, 1.f, 1.f, 1.f);
                    if (u < n4) {
                        x = __ldcg(reinterpret_cast<const float4*>(xin + (size_t)t * H + cc * RKc) + u);
                        if (gamma) gm = __ldg(reinterpret_cast<const float4*>(gamma + cc * RKc) + u);
                    }
                    nv[j].x = (float)((double)x.x * r * (double)gm.x);
                    nv[j].y = (float)((double)x.y * r * (double)gm.y);
                    nv[j].z = (float)((double)x.z * r * (double)gm.z);
                    nv[j].w = (float)((double)x.w * r * (double)gm.w);
                }
                cc_have = cc;
            }
            const float4* wr = reinterpret_cast<const float4*>(sb + (size_t)it * RKc * 4);
            double acc = 0.0;
#pragma unroll
            for (int j = 0; j < U; j++) {
                const int u = tid + NCT * j;
                if (u < n4) {
                    const float4 wv = wr[u];
                    acc = fma((double)nv[j].x, (double)wv.x, acc);
                    acc = fma((double)nv[j].y, (double)wv.y, acc);
                    acc = fma((double)nv[j].z, (double)wv.z, acc);
                    acc = fma((double)nv[j].w, (double)wv.w, acc);
                }
            }
#pragma unroll
            for (int o = 16; o >= 1; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
            if (lane == 0) part[(it * T + t) * NCW + c.warp] = acc;
        }
    }
    cslot_free(p, c, w);
    named_bar(5, NCT);
    // each partial as two 8-byte (half, epoch) words: a reader polls the values themselves
    const uint32_t ep = h_epoch(c, l);
    for (int q = tid; q < nit * T; q += NCT) {
        const int it = q / T, t = q - it * T, i = c.ri0 + it, e = i / RC, cc = i - e * RC;
        double sum = 0.0;
#pragma unroll 1
        for (int ww = 0; ww < NCW; ww++) sum += part[q * NCW + ww];
        p.rpart[((size_t)t * E + e) * RC + cc] =
            make_uint4((uint32_t)__double2loint(sum), ep, (uint32_t)__double2hiint(sum), ep);
    }
    named_bar(5, NCT);
}

// One token (pair mode): the layer input once per layer into shared memory as the
// normalised n = float(x * r * gamma) (exactly x for a plain input), with the RMSNorm
// factor r and the activation scale 126 / max|n| in the head.  Thread tid holds float4
// u = tid + NCT j of the row; every thread sums the warps' parts in the same order.
__device__ __forceinline__ void load_x_pair(const FusedParams& p, const Ctx& c, int l, const float* xin)
{
    const int n4 = p.H / 4, tid = c.tid, lane = c.lane, warp = c.warp;
    const float4* gamma = p.norm ? reinterpret_cast<const float4*>(p.layer[l].gamma) : nullptr;
    Head& hd = *c.hd;
    float4* xs = reinterpret_cast<float4*>(reinterpret_cast<uint8_t*>(c.hd) + p.off_hstage);
    constexpr int U = 4;   // H <= 16 NCT
    float4 v[U];
#pragma unroll
    for (int j = 0; j < U; j++) {
        const int u = tid + NCT * j;
        v[j] = u < n4 ? __ldcg(reinterpret_cast<const float4*>(xin) + u) : make_float4(0.f, 0.f, 0.f, 0.f);
    }
    if (tid == 0) hd.gen = __ldcg(p.gen);   // published by the named barriers below
    double r = 1.0;
    if (p.norm) {
        double sq = 0.0;
#pragma unroll
        for (int j = 0; j < U; j++) {
            sq = fma((double)v[j].x, (double)v[j].x, sq);
            sq = fma((double)v[j].y, (double)v[j].y, sq);
            sq = fma((double)v[j].z, (double)v[j].z, sq);
            sq = fma((double)v[j].w, (double)v[j].w, sq);
        }
#pragma unroll
        for (int o = 16; o >= 1; o >>= 1) sq += __shfl_xor_sync(0xffffffffu, sq, o);
        if (lane == 0) hd.rsq[warp][0] = sq;
        named_bar(5, NCT);
        double s2 = 0.0;
#pragma unroll 1
        for (int ww = 0; ww < NCW; ww++) s2 += hd.rsq[ww][0];
        r = 1.0 / sqrt(s2 / (double)p.H + p.eps);
    }
    float mx = 0.0f;
#pragma unroll
    for (int j = 0; j < U; j++) {
        const int u = tid + NCT * j;
        if (u < n4) {
            const float4 gm = gamma ? __ldg(gamma + u) : make_float4(1.f, 1.f, 1.f, 1.f);
            float4 n;
            n.x = (float)((double)v[j].x * r * (double)gm.x);
            n.y = (float)((double)v[j].y * r * (double)gm.y);
            n.z = (float)((double)v[j].z * r * (double)gm.z);
            n.w = (float)((double)v[j].w * r * (double)gm.w);
            xs[u] = n;
            mx = fmaxf(mx, fmaxf(fmaxf(fabsf(n.x), fabsf(n.y)), fmaxf(fabsf(n.z), fabsf(n.w))));
        }
    }
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
    if (lane == 0) hd.amax[warp][0] = mx;
    named_bar(5, NCT);
    if (tid == 0) {
        float m2 = 0.0f;
        for (int ww = 0; ww < NCW; ww++) m2 = fmaxf(m2, hd.amax[ww][0]);
        hd.rnorm[0] = r;
        hd.xinv[0] = m2 > 0.0f ? 126.0f / m2 : 0.0f;
        hd.xfac[0] = m2 * (1.0f / 126.0f);
    }
    named_bar(5, NCT);
}

// RMSNorm factors (stacks; 1 otherwise) and the per-token activation scale of the layer
// input; every CTA sums in the same order, so all CTAs agree bit for bit
__device__ __forceinline__ void input_scales(const FusedParams& p, const Ctx& c, int l, const float* xin)
{
    const int T = p.T, n4 = p.H / 4, tid = c.tid, lane = c.lane, warp = c.warp;
    const float4* gamma = p.norm ? reinterpret_cast<const float4*>(p.layer[l].gamma) : nullptr;
    Head& hd = *c.hd;
    constexpr int U = 4;   // float4 per thread per pass (H <= 6144 in one pass)
    if (p.norm) {
#pragma unroll 1
        for (int t = 0; t < T; t++) {
            const float4* xr = reinterpret_cast<const float4*>(xin + (size_t)t * p.H);
            double sq = 0.0;
#pragma unroll 1
            for (int i0 = tid; i0 < n4; i0 += NCT * U) {
                float4 v[U];
#pragma unroll
                for (int j = 0; j < U; j++)
                    v[j] = i0 + NCT * j < n4 ? __ldcg(xr + i0 + NCT * j) : make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
                for (int j = 0; j < U; j++) {
                    sq = fma((double)v[j].x, (double)v[j].x, sq);
                    sq = fma((double)v[j].y, (double)v[j].y, sq);
                    sq = fma((double)v[j].z, (double)v[j].z, sq);
                    sq = fma((double)v[j].w, (double)v[j].w, sq);
                }
            }
#pragma unroll
            for (int o = 16; o >= 1; o >>= 1) sq += __shfl_xor_sync(0xffffffffu, sq, o);
            if (lane == 0) hd.rsq[warp][t] = sq;
        }
        named_bar(5, NCT);
        if (tid < T) {
            double sq = 0.0;
#pragma unroll 1
            for (int w = 0; w < NCW; w++) sq += hd.rsq[w][tid];
            hd.rnorm[tid] = 1.0 / sqrt(sq / (double)p.H + p.eps);
        }
        named_bar(5, NCT);
    }
#pragma unroll 1
    for (int t = 0; t < T; t++) {
        const float4* xr = reinterpret_cast<const float4*>(xin + (size_t)t * p.H);
        float mx = 0.0f;
        const double r = p.norm ? hd.rnorm[t] : 1.0;
#pragma unroll 1
        for (int i0 = tid; i0 < n4; i0 += NCT * U) {
            float4 v[U];
#pragma unroll
            for (int j = 0; j < U; j++)
                v[j] = i0 + NCT * j < n4 ? __ldcg(xr + i0 + NCT * j) : make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
            for (int j = 0; j < U; j++) {
                // n = float(x * r * gamma): exactly x for a plain input
                float4 gm = make_float4(1.f, 1.f, 1.f, 1.f);
                if (gamma && i0 + NCT * j < n4) gm = __ldg(gamma + i0 + NCT * j);
                mx = fmaxf(mx, fabsf((float)((double)v[j].x * r * (double)gm.x)));
                mx = fmaxf(mx, fabsf((float)((double)v[j].y * r * (double)gm.y)));
                mx = fmaxf(mx, fabsf((float)((double)v[j].z * r * (double)gm.z)));
                mx = fmaxf(mx, fabsf((float)((double)v[j].w * r * (double)gm.w)));
            }
        }
#pragma unroll
        for (int o = 16; o >= 1; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
        if (lane == 0) hd.amax[warp][t] = mx;
    }
    named_bar(5, NCT);
    if (tid < T) {
        float mx = 0.0f;
#pragma unroll 1
        for (int w = 0; w < NCW; w++) mx = fmaxf(mx, hd.amax[w][tid]);
        hd.xinv[tid] = mx > 0.0f ? 126.0f / mx : 0.0f;
        hd.xfac[tid] = mx * (1.0f / 126.0f);
    }
    named_bar(5, NCT);
}

template <int NTM, int GPWG, bool PAIR>
__device__ __forceinline__ void build_x_operand(const FusedParams& p, const Ctx& c, Cons& w, int l,
                                                const float* xin, uint32_t (&Bx)[GPWG][NTM][4],
                                                float (&fdummy)[GPWG][NTM])
{
    const int T = p.T, H = p.H;
    const Head& hd = *c.hd;
    const float* gamma = p.norm ? p.layer[l].gamma : nullptr;
    if constexpr (PAIR) {
        build_x_pairs<GPWG, NTM>(reinterpret_cast<const float*>(reinterpret_cast<const uint8_t*>(c.hd) + p.off_hstage),
                                 hd.xinv[0], w.gbase_g, w.gpw_g, w.sc, c.lane, Bx);
    } else {
#pragma unroll
        for (int q = 0; q < NTM; q++) {
            const int t0 = 2 * q, t1 = 2 * q + 1;
            const bool p0 = t0 < T, p1 = t1 < T;
            const float* row0 = xin + (size_t)(p0 ? t0 : 0) * H;
            const float* row1 = xin + (size_t)(p1 ? t1 : 0) * H;
            build_tile<GPWG, NTM, false>(row0, row1, p0, p1, p0 ? hd.xinv[t0] : 0.0f, p1 ? hd.xinv[t1] : 0.0f,
                                         hd.rnorm[p0 ? t0 : 0], hd.rnorm[p1 ? t1 : 0], gamma, 0u,
                                         w.gbase_g, w.gpw_g, q, w.sc, c.lane, Bx, fdummy, p.status, c.dead);
        }
    }
}

// one gate/up stage (stage st of segment s, tokens sg): SwiGLU rows into h
template <int NTM, int GPWG, bool PAIR>
__device__ __forceinline__ void gu_consume(const FusedParams& p, const Ctx& c, Cons& w, int l,
                                           const Seg& sg, int st,
                                           const uint32_t (&Bx)[GPWG][NTM][4],
                                           const float (&fdummy)[GPWG][NTM])
{
    const int T = p.T, H = p.H, I = p.I, lane = c.lane;
    const uint8_t* sb = cslot_wait(p, c, w);
    const int i0 = st * 8 * p.NTSg;
    const int ntl = min(p.NTSg, (I - i0) / 8);
    const int cr = 2 * ntl;    // rows per chunk
    uint32_t qmask = 0;
#pragma unroll 1
    for (int m = 0; m < sg.c; m++) qmask |= 1u << (sg.tok[m] >> 1);
    red_wait_free(*c.hd, w.cs, p.status, c.dead, lane);
    float* rb = c.red + (size_t)(w.cs % kRedBufs) * p.red_floats;
    const int g = lane >> 2, t = lane & 3;
    const uint32_t rowb = (uint32_t)H / 2, srow = (uint32_t)H / 64;
#pragma unroll 1
    for (int tl = w.g_rs; tl < ntl; tl += p.RSg) {
        // lane row g: chunk g & 3, row 2 tl + (g >> 2) of the chunk
        const int lr = 2 * tl + (g >> 2);
        const uint8_t* ga = sb + (size_t)(g & 3) * p.gu_chunk + (size_t)lr * rowb + (PAIR ? 16 : 8) * t;
        const uint8_t* ua = ga + (size_t)4 * p.gu_chunk;
        const int sr = (g & 3) * cr + lr;
        const __half* gs = reinterpret_cast<const __half*>(sb + p.gu_gsc) + (size_t)sr * srow;
        const __half* us = reinterpret_cast<const __half*>(sb + p.gu_usc) + (size_t)sr * srow;
        float* rbt = rb + (size_t)(w.g_kw * p.NTSg + tl) * 16 * T;
        if constexpr (PAIR) {
            float acc4[4];
            tile_dot_pairs<GPWG, NTM, false>(ga, ua, gs, us, w.gbase_g, lane, Bx, fdummy, acc4);
            tile_partials_pairs(acc4, lane, rbt, c.hd->xfac[0]);
        } else {
            float acc[NTM][4];
            tile_dot<GPWG, NTM, false>(ga, ua, gs, us, w.gbase_g, w.gpw_g, qmask, Bx, fdummy, acc);
            tile_partials<NTM>(acc, qmask, lane, T, rbt, T, c.hd->xfac);
        }
    }
    cslot_free(p, c, w);
    red_deliver(*c.hd, w.cs, lane);
    w.cs++;
}

// the down stage of segment s (this CTA's output rows), combined into yacc
template <int NTM, int GPWD, bool PAIR>
__device__ __forceinline__ void down_consume(const FusedParams& p, const Ctx& c, Cons& w, int l,
                                             const Seg& sg, uint32_t (&Bh)[GPWD][NTM][4],
                                             float (&fh)[GPWD][NTM])
{
    const int T = p.T, I = p.I, lane = c.lane;
    const int cn = sg.c;
    const uint32_t ep = h_epoch(c, l);
    if constexpr (PAIR) {
        // the segment's digit row of h, copied by the control warp into buffer ds % kDigBufs
        // (the ds-th down segment of the launch); the buffer is released once read
        const uint32_t ds = w.ds, b = ds % (uint32_t)kDigBufs;
        const uint8_t* hd0 = reinterpret_cast<const uint8_t*>(c.hd) + p.off_hdig + (size_t)b * p.hdig_bytes;
        mwait(&c.hd->dg_full[b], (ds / (uint32_t)kDigBufs) & 1u, p.status, 58, c.dead);
        gather_h_pairs<GPWD, NTM>(reinterpret_cast<const uint32_t*>(hd0), reinterpret_cast<const uint2*>(hd0 + 3 * I),
                                  I, w.gbase_d, lane, Bh, fh);
        __syncwarp();
        if (lane == 0) mbar_arrive(&c.hd->dg_empty[b]);
        w.ds++;
    } else {
#pragma unroll
        for (int q = 0; q < NTM; q++) {
            const int m0 = 2 * q, m1 = 2 * q + 1;
            const bool p0 = m0 < cn, p1 = m1 < cn;
            const uint8_t* d0 = p.hdg + (size_t)(sg.base + (p0 ? m0 : 0)) * p.hdg_row;
            const uint8_t* d1 = p.hdg + (size_t)(sg.base + (p1 ? m1 : 0)) * p.hdg_row;
            gather_tile_digits<GPWD, NTM>(d0, d1, p0, p1, I, ep, w.gbase_d, w.gpw_d, q, lane, Bh, fh, p.status,
                                          c.dead);
        }
    }
    const uint32_t qmask = (1u << ((cn + 1) >> 1)) - 1u;
    const uint8_t* sb = cslot_wait(p, c, w);
    red_wait_free(*c.hd, w.cs, p.status, c.dead, lane);
    float* rb = c.red + (size_t)(w.cs % kRedBufs) * p.red_floats;
    const uint32_t delta = (uint32_t)(((uint64_t)c.r0 * (I / 32)) & 15ull);
    const int g = lane >> 2, t = lane & 3;
    const uint32_t rowb = (uint32_t)I / 2, srow = (uint32_t)I / 64;
    const __half* scb = reinterpret_cast<const __half*>(sb + p.d_sc_off + delta);
    const int ntdm = p.ntdm;
#pragma unroll 1
    for (int tl = w.d_rs; tl < c.ntd; tl += p.RSd) {
        // MMA row m: chunk m & 3, row 4 tl + (m >> 2) of the chunk (rows g and g + 8)
        const int q = g & 3, la = 4 * tl + (g >> 2), lb = la + 2;
        const uint8_t* ra = sb + (size_t)q * p.d_chunk + (size_t)la * rowb + (PAIR ? 16 : 8) * t;
        const uint8_t* rbp = sb + (size_t)q * p.d_chunk + (size_t)lb * rowb + (PAIR ? 16 : 8) * t;
        const __half* sa = scb + (size_t)(dcs(c, q) + la) * srow;
        const __half* sbh = scb + (size_t)(dcs(c, q) + lb) * srow;
        float* rbt = rb + (size_t)(w.d_kw * ntdm + tl) * 16 * T;
        if constexpr (PAIR) {
            float acc4[4];
            tile_dot_pairs<GPWD, NTM, true>(ra, rbp, sa, sbh, w.gbase_d, lane, Bh, fh, acc4);
            tile_partials_pairs(acc4, lane, rbt, 1.0f);
        } else {
            float acc[NTM][4];
            tile_dot<GPWD, NTM, true>(ra, rbp, sa, sbh, w.gbase_d, w.gpw_d, qmask, Bh, fh, acc);
            tile_partials<NTM>(acc, qmask, lane, cn, rbt, T, nullptr);
        }
    }
    cslot_free(p, c, w);
    red_deliver(*c.hd, w.cs, lane);
    w.cs++;
}

// ----------------------------- reducer warp ---------------------------------------------
// Sums of one gate/up stage (stage st of segment sg): four lanes per (row, token) over the
// K-split warps' partials, SwiGLU, h stored as (value, epoch).
// The digit rows of h (one per row of h).  Group g (64 values) of h row `row` is digitized by
// one CTA (the one that sums the group's last row) once all its values carry the layer's
// epoch; lane j (and j + 16) holds values 64 g + 4 j .. + 3 as (value, epoch) pairs.
__device__ __forceinline__ void group_load(const FusedParams& p, int row, int g, int lane, uint4& a, uint4& b)
{
    const uint4* hp = reinterpret_cast<const uint4*>(p.h + (size_t)row * p.I + 64 * g + 4 * (lane & 15));
    a = __ldcg(hp);
    b = __ldcg(hp + 1);
}

__device__ __forceinline__ bool group_ready(const uint4& a, const uint4& b, uint32_t ep)
{
    return __all_sync(0xffffffffu, a.y == ep && a.w == ep && b.y == ep && b.w == ep);
}

// The group's digits into the row's digit row, then its (m / 126, ep) word, ordered after
// the digits (a reader that sees the word sees the digits).
__device__ __forceinline__ void group_store(const FusedParams& p, int row, int g, int lane, uint32_t ep,
                                            const uint4& a, const uint4& b)
{
    const int I = p.I;
    uint32_t wd[3];
    const float m = digit_words(make_float4(__uint_as_float(a.x), __uint_as_float(a.z), __uint_as_float(b.x),
                                            __uint_as_float(b.z)), wd);
    uint8_t* dr = p.hdg + (size_t)row * p.hdg_row;
    if (lane < 16) {
#pragma unroll
        for (int pl = 0; pl < 3; pl++)
            *reinterpret_cast<uint32_t*>(dr + (size_t)pl * I + 64 * g + 4 * lane) = wd[pl];
    }
    __syncwarp();
    if (lane == 0) {
        __threadfence();
        *reinterpret_cast<unsigned long long*>(dr + 3 * (size_t)I + 8 * g) =
            ((unsigned long long)ep << 32) | __float_as_uint(m * (1.0f / 126.0f));
    }
}

// The groups this CTA still has to digitize, oldest first (lane j holds entry j:
// row << 16 | group).
struct Pending {
    uint32_t e;
    int n;
};

__device__ __forceinline__ void pending_pop(Pending& pd)
{
    pd.e = __shfl_down_sync(0xffffffffu, pd.e, 1);
    pd.n--;
}

// Every pending group, each once its values have arrived (bounded waits).
__device__ __forceinline__ void pending_drain(const FusedParams& p, const Ctx& c, Pending& pd, uint32_t ep)
{
#pragma unroll 1
    while (pd.n > 0) {
        const uint32_t e0 = __shfl_sync(0xffffffffu, pd.e, 0);
        const int row = (int)(e0 >> 16), g = (int)(e0 & 0xFFFFu);
        uint4 a, b;
        group_load(p, row, g, c.lane, a, b);
        if (!group_ready(a, b, ep)) {
            const long long t0 = clock64();
            uint32_t npoll = 0;
            while (true) {
                __nanosleep(64);
                group_load(p, row, g, c.lane, a, b);
                if (group_ready(a, b, ep)) break;
                if (*c.dead || wait_expired(npoll, t0, p.status)) {
                    if (c.lane == 0) give_up(p.status, 56, c.dead);
                    break;
                }
            }
        }
        group_store(p, row, g, c.lane, ep, a, b);
        pending_pop(pd);
    }
}

__device__ __forceinline__ void reduce_gu(const FusedParams& p, const Ctx& c, uint32_t cs, const Seg& sg,
                                          int st, uint32_t ep, Pending& pd)
{
    const int T = p.T, I = p.I, lane = c.lane;
    const float* rb = c.red + (size_t)(cs % kRedBufs) * p.red_floats;
    const int i0 = st * 8 * p.NTSg;
    const int ntl = min(p.NTSg, (I - i0) / 8);
    const int cr = 2 * ntl;
    uint2* hb = reinterpret_cast<uint2*>(p.h);
    const int ntask = ntl * 8 * sg.c, part = lane & 3;
#pragma unroll 1
    for (int t0 = 0; t0 < ntask; t0 += 8) {
        const int task = t0 + (lane >> 2);
        const bool valid = task < ntask;
        const int m = valid ? task % sg.c : 0, rr = valid ? task / sg.c : 0;
        const int tl = rr >> 3, r = rr & 7;
        const int tok = sg.tok[m];
        float gsum = 0.0f, usum = 0.0f;
        if (valid)
#pragma unroll 1
            for (int kw = part; kw < p.KWg; kw += 4) {
                const float* q = rb + (size_t)(kw * p.NTSg + tl) * 16 * T;
                gsum += q[r * T + tok];
                usum += q[(8 + r) * T + tok];
            }
        gsum += __shfl_xor_sync(0xffffffffu, gsum, 1);
        usum += __shfl_xor_sync(0xffffffffu, usum, 1);
        gsum += __shfl_xor_sync(0xffffffffu, gsum, 2);
        usum += __shfl_xor_sync(0xffffffffu, usum, 2);
        if (valid && part == 0) {
            const float hv = gsum / (1.0f + expf(-gsum)) * usum;
            const int row = i0 + (r & 3) * cr + 2 * tl + (r >> 2);
            hb[(size_t)(sg.base + m) * I + row] = make_uint2(__float_as_uint(hv), ep);
        }
    }
    {
        // this CTA digitizes, for each token of the segment, every group whose last row is
        // one of the stage's rows i0 .. i0 + 8 ntl - 1, once all its values have arrived
        const int r1 = i0 + 8 * ntl;
#pragma unroll 1
        for (int m = 0; m < sg.c; m++) {
#pragma unroll 1
            for (int g = i0 / 64; g <= (r1 - 1) / 64; g++) {
                if (64 * g + 63 < i0 || 64 * g + 63 >= r1) continue;
                if (pd.n == 32) pending_drain(p, c, pd, ep);
                if (lane == pd.n) pd.e = ((uint32_t)(sg.base + m) << 16) | (uint32_t)g;
                pd.n++;
            }
        }
    }
}

// Sums of one down stage (segment sg, the CTA's rows): routing-weighted combine into yacc.
// One lane per (row, token); the K-split partials kw are added as ((s0 + s1) + (s2 + s3)),
// s_j the sum of those with kw = j mod 4 in ascending kw.
__device__ __forceinline__ void reduce_down(const FusedParams& p, const Ctx& c, uint32_t cs, const Seg& sg)
{
    const int T = p.T, lane = c.lane, cn = sg.c, KW = p.KWd;
    const float* rb = c.red + (size_t)(cs % kRedBufs) * p.red_floats;
    const int nrs = c.ntd * 16;                        // row slots of the CTA's tiles
    const size_t kst = (size_t)p.ntdm * 16 * T;        // from one K-split warp's part to the next
#pragma unroll 1
    for (int m = 0; m < cn; m++) {
        const float wt = sg.wt[m];
        const int tok = sg.tok[m];
#pragma unroll 1
        for (int rr = lane; rr < nrs; rr += 32) {
            const int tl = rr >> 4, mm = rr & 15;
            const int q = mm & 3, lrow = 4 * tl + (mm >> 2);
            if (lrow >= dcs(c, q + 1) - dcs(c, q)) continue;
            const float* src = rb + ((size_t)tl * 16 + mm) * T + m;
            float s4[4] = {0.0f, 0.0f, 0.0f, 0.0f};
#pragma unroll 1
            for (int k0 = 0; k0 < KW; k0 += 4) {
#pragma unroll
                for (int j = 0; j < 4; j++)
                    if (k0 + j < KW) s4[j] += src[(size_t)(k0 + j) * kst];
            }
            float* ya = c.yacc + (dcs(c, q) + lrow) * T + tok;
            *ya = *ya + wt * ((s4[0] + s4[1]) + (s4[2] + s4[3]));
        }
    }
}

// The reducer follows the consumers' sequence of reduction stages: the shared gate/up
// stages of the CTA, [routing], the routed ones, then the down stages of every segment.
__device__ __forceinline__ void reducer_warp(const FusedParams& p, const Ctx& c, uint32_t gen)
{
    const int T = p.T, k = p.k, ns = p.n_shared, lane = c.lane;
    Seg sh;
    sh.c = T;
    sh.base = T * k;
    sh.tok = c.hd->sh_tok;
    sh.wt = c.hd->sh_wt;
    uint32_t cs = 0;
    Pending pd;
    pd.e = 0u;
    pd.n = 0;
#pragma unroll 1
    for (int l = 0; l < p.L; l++) {
        const uint32_t ep = gen * 32u + (uint32_t)l + 1u;
        Table tb;
        int nseg = ns, gi = c.b, ds = 0;
        bool routed = false;
        while (true) {
            int kind = 0, seg = 0;
            if (gi < nseg * p.SPS) {
                kind = 1;
                seg = gi / p.SPS;
            } else if (!routed) {
                mwait(&c.hd->route_bar, (uint32_t)l & 1u, p.status, 60, c.dead);
                tb = layer_table(c, l);
                nseg = tb.hdr[0];
                routed = true;
                continue;
            } else if (c.nrows > 0 && ds < nseg) {
                kind = 2;
                seg = ds++;
            } else {
                break;
            }
            // the groups of h left to digitize, before the first down stage (every CTA's
            // down stages need them); otherwise the oldest one's values are read while the
            // partial sums are awaited, and it is digitized after the stage if they are all in
            if (kind == 2 && pd.n > 0) pending_drain(p, c, pd, ep);
            const bool look = pd.n > 0;
            uint4 ga = make_uint4(0u, 0u, 0u, 0u), gb = ga;
            uint32_t ge = 0u;
            if (look) {
                ge = __shfl_sync(0xffffffffu, pd.e, 0);
                group_load(p, (int)(ge >> 16), (int)(ge & 0xFFFFu), lane, ga, gb);
            }
            mwait(&c.hd->red_full[cs % kRedBufs], (cs / kRedBufs) & 1u, p.status, 59, c.dead);
            const Seg sg = seg < ns ? sh : seg_of(tb, seg);
            if (kind == 1) {
                reduce_gu(p, c, cs, sg, gi - seg * p.SPS, ep, pd);
                gi += c.G;
            } else {
                reduce_down(p, c, cs, sg);
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&c.hd->red_empty[cs % kRedBufs]);
            cs++;
            if (look && group_ready(ga, gb, ep)) {
                group_store(p, (int)(ge >> 16), (int)(ge & 0xFFFFu), lane, ep, ga, gb);
                pending_pop(pd);
            }
        }
        // (a CTA without down rows still digitizes its groups)
        if (pd.n > 0) pending_drain(p, c, pd, ep);
        stamp(lane == 0 && l == p.L - 1, ST_REDUCED);
        // the layer's output rows are summed: the consumers write them, then yacc is clear
        named_bar(7, NCT + 32);
        named_bar(8, NCT + 32);
    }
}

template <int NTM, int GPWG, int GPWD, bool PAIR>
__device__ __forceinline__ void consumer_warp(const FusedParams& p, const Ctx& c)
{
    const int T = p.T, H = p.H, k = p.k, ns = p.n_shared;
    Cons w;
    w.it = 0;
    w.cs = 0;
    w.ds = 0;
    w.sc = reinterpret_cast<uint32_t*>(reinterpret_cast<uint8_t*>(c.hd) + p.off_scratch) + c.warp * 96;
    // K split: warp kw of a row slot takes groups [kw n / KW, (kw + 1) n / KW)
    const int ngg = p.H / 64, ngd = p.I / 64;
    w.g_rs = c.warp / p.KWg;
    w.g_kw = c.warp % p.KWg;
    w.gbase_g = w.g_kw * ngg / p.KWg;
    w.gpw_g = (w.g_kw + 1) * ngg / p.KWg - w.gbase_g;
    w.d_rs = c.warp / p.KWd;
    w.d_kw = c.warp % p.KWd;
    w.gbase_d = w.d_kw * ngd / p.KWd;
    w.gpw_d = (w.d_kw + 1) * ngd / p.KWd - w.gbase_d;
    uint32_t Bx[GPWG][NTM][4];
    float fdummy[GPWG][NTM];
    uint32_t Bh[GPWD][NTM][4];
    float fh[GPWD][NTM];
#pragma unroll
    for (int gi = 0; gi < GPWG; gi++)
#pragma unroll
        for (int q = 0; q < NTM; q++) fdummy[gi][q] = 0.0f;
    Seg sh;
    sh.c = T;
    sh.base = T * k;
    sh.tok = c.hd->sh_tok;
    sh.wt = c.hd->sh_wt;

#pragma unroll 1
    for (int l = 0; l < p.L; l++) {
        uint32_t* lc = layer_cnt(p, l);
        const float* xin = l == 0 ? p.x : p.xbuf + (size_t)((l - 1) & 1) * T * H;
        float* yout = l == p.L - 1 ? p.y : p.xbuf + (size_t)(l & 1) * T * H;
        const float* res = p.norm ? xin : p.residual;
        if (l > 0) {
            if (c.lane == 0) gwait(&layer_cnt(p, l - 1)[1], (uint32_t)c.G, p.status, 52, c.dead);
            __syncwarp();
        }
        // the router needs only the RMSNorm factors (1 for a plain input), so for a plain
        // input it runs first and the routing is decided while the scales are formed
        const bool w0 = c.warp == 0 && c.lane == 0 && l == p.L - 1;
        if constexpr (PAIR) {
            load_x_pair(p, c, l, xin);
            stamp(w0, ST_INPUT);
            if (c.ri1 > c.ri0) router_consume<true>(p, c, w, l, xin);
            stamp(w0, ST_ROUTER);
        } else {
#pragma unroll 1
            for (int step = 0; step < 2; step++) {
                if ((step == 0) != (p.norm != 0)) {
                    if (c.ri1 > c.ri0) router_consume<false>(p, c, w, l, xin);
                } else {
                    input_scales(p, c, l, xin);
                }
            }
            stamp(w0, ST_INPUT);
            stamp(w0, ST_ROUTER);
        }
        // stages in the control warp's order; one code path per kind of step
        //   phase 0: x operand, 1: shared gate/up, 4: routing, 5: routed gate/up,
        //   6: down rows of every segment (the shared expert's first)
        Table tb;
        int nseg = 0, phase = 0, gi = c.b, sd = 0;
        bool routed_seen = false;   // phase stamps: a routed gate/up stage has begun
        while (true) {
            int kind = -1, seg = 0, stage = 0;   // 0: x operand, 1: gate/up, 2: down
            if (phase == 0) {
                kind = 0;
                phase = 1;
            } else if (phase == 1) {
                if (ns && gi < p.SPS) {
                    kind = 1;
                    seg = 0;
                    stage = gi;
                    gi += c.G;
                } else {
                    phase = 4;
                    continue;
                }
            } else if (phase == 4) {
                mwait(&c.hd->route_bar, (uint32_t)l & 1u, p.status, 55, c.dead);
                tb = layer_table(c, l);
                nseg = tb.hdr[0];
                while (gi < ns * p.SPS) gi += c.G;
                phase = 5;
                continue;
            } else if (phase == 5) {
                if (gi < nseg * p.SPS) {
                    kind = 1;
                    seg = gi / p.SPS;
                    stage = gi - seg * p.SPS;
                    gi += c.G;
                } else {
                    phase = 6;
                    continue;
                }
            } else {
                if (c.nrows > 0 && sd < nseg) {
                    kind = 2;
                    seg = sd++;
                } else {
                    break;
                }
            }
            if (kind == 0) {
                build_x_operand<NTM, GPWG, PAIR>(p, c, w, l, xin, Bx, fdummy);
                stamp(w0, ST_XOP);
            } else {
                const Seg sg = seg < ns ? sh : seg_of(tb, seg);
                if (kind == 1) {
                    stamp(w0 && seg >= ns && !routed_seen, ST_GU_ROUTED);
                    routed_seen = routed_seen || seg >= ns;
                    gu_consume<NTM, GPWG, PAIR>(p, c, w, l, sg, stage, Bx, fdummy);
                } else {
                    stamp(w0 && seg == 0, ST_DOWN);
                    if constexpr (GPWG == GPWD) {
                        // the h operand takes the x operand's registers (the down stages
                        // follow every gate/up stage of the layer)
                        down_consume<NTM, GPWD, PAIR>(p, c, w, l, sg, Bx, fdummy);
                    } else {
                        down_consume<NTM, GPWD, PAIR>(p, c, w, l, sg, Bh, fh);
                    }
                }
            }
        }
        stamp(w0, ST_DOWN_DONE);
        // ---- this CTA's rows of the layer output (once the reducer has summed them all)
        named_bar(7, NCT + 32);
#pragma unroll 1
        for (int i = c.tid; i < c.nrows * T; i += NCT) {
            const int rr = i / T, t = i - rr * T;
            const size_t o = (size_t)t * H + c.r0 + rr;
            const float base = res ? __ldcg(res + o) : 0.0f;
            yout[o] = base + c.yacc[i];
            c.yacc[i] = 0.0f;
        }
        named_bar(8, NCT + 32);
        // the next layer's consumers wait for every CTA's rows (none wait after the last)
        if (c.tid == 0 && l < p.L - 1) {
            __threadfence();
            red_release_add(&lc[1], 1u);
        }
    }
}

template <int NTM, int GPWG, int GPWD, bool PAIR>
__global__ void __launch_bounds__(NTHR, 1) fused_moe_kernel(const __grid_constant__ FusedParams p)
{
    extern __shared__ __align__(128) uint8_t smem[];
    Ctx c;
    c.hd = reinterpret_cast<Head*>(smem);
    c.dead = &c.hd->dead;
    c.ring = smem + p.off_ring;
    c.red = reinterpret_cast<float*>(smem + p.off_red);
    c.yacc = reinterpret_cast<float*>(smem + p.off_yacc);
    c.rt_base = smem + sizeof(Head);
    c.S = 1 + p.T * p.k;
    c.tbytes = table_bytes(c.S);
    c.tid = threadIdx.x;
    c.warp = c.tid >> 5;
    c.lane = c.tid & 31;
    c.b = blockIdx.x;
    c.G = gridDim.x;
    c.r0 = (int)((int64_t)p.H * c.b / c.G);
    c.r1 = (int)((int64_t)p.H * (c.b + 1) / c.G);
    c.nrows = c.r1 - c.r0;
    c.ntd = (((c.nrows + 3) >> 2) + 3) >> 2;
    c.n_ritems = p.E * p.RC;
    c.ri0 = p.route ? (int)((int64_t)c.n_ritems * c.b / c.G) : 0;
    c.ri1 = p.route ? (int)((int64_t)c.n_ritems * (c.b + 1) / c.G) : 0;
    c.bo = blob_off(p.H, p.I);

    pdl_launch_dependents();
    stamp(c.tid == 0, ST_START);
    if (c.tid == 0) {
#pragma unroll 1
        for (int s = 0; s < p.nslot; s++) {
            mbar_init(&c.hd->full[s], 1);
            mbar_init(&c.hd->empty[s], NCW);
        }
        mbar_init(&c.hd->route_bar, 1);
        c.hd->dead = 0;
#pragma unroll 1
        for (int b2 = 0; b2 < kRedBufs; b2++) {
            mbar_init(&c.hd->red_full[b2], NCW);
            mbar_init(&c.hd->red_empty[b2], 1);
        }
#pragma unroll 1
        for (int b2 = 0; b2 < kDigBufs; b2++) {
            mbar_init(&c.hd->dg_full[b2], 1);
            mbar_init(&c.hd->dg_empty[b2], NCW);
        }
#pragma unroll 1
        for (int m = 0; m < kFusedMaxT; m++) {
            c.hd->sh_tok[m] = m;
            c.hd->sh_wt[m] = 1.0f;
            c.hd->rnorm[m] = 1.0;
        }
        fence_barrier_init();
    }
#pragma unroll 1
    for (int i = c.tid; i < p.rows_max * p.T; i += NTHR) c.yacc[i] = 0.0f;
    __syncthreads();

    if (c.warp == NCW) {
        control_warp(p, c);
    } else if (c.warp == NCW + 1) {
        pdl_wait();
        reducer_warp(p, c, __ldcg(p.gen));
    } else {
        pdl_wait();
        // the launch generation, published by the first named barrier (one token: read in
        // load_x_pair beside the layer input, so the two loads overlap)
        if (!PAIR && c.tid == 0) c.hd->gen = __ldcg(p.gen);
        consumer_warp<NTM, GPWG, GPWD, PAIR>(p, c);
    }

    // ---- exit: the last CTA returns the counters to zero and advances the generation
    __syncthreads();
    stamp(c.tid == 0, ST_EXIT);
    // (every layer's output-rows increments were seen by the waits of the layer after it,
    // so the counters the last CTA clears are no longer written by anyone)
    if (c.tid == 0) {
        const uint32_t prev = atomicAdd(&p.cnt[0], 1u);
        if (prev == (uint32_t)c.G - 1u) {
            // the only counter a layer uses is its output-rows count; the next launch, which
            // follows this one in stream order, sees these stores without a fence
#pragma unroll 1
            for (int l = 0; l < p.L; l++) layer_cnt(p, l)[1] = 0u;
            *p.gen = c.hd->gen + 1u;
            p.cnt[0] = 0u;
        }
    }
}

template <int NTM, int GPWG, int GPWD, bool PAIR>
cudaError_t launch_fused(const FusedParams& p, cudaStream_t s)
{
    auto kern = fused_moe_kernel<NTM, GPWG, GPWD, PAIR>;
    static int set_bytes[64] = {0};
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= 64 || set_bytes[dev] < (int)p.smem) {
        e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)p.smem);
        if (e != cudaSuccess) return e;
        if (dev >= 0 && dev < 64) set_bytes[dev] = (int)p.smem;
    }
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(p.grid);
    cfg.blockDim = dim3(NTHR);
    cfg.dynamicSmemBytes = p.smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kern, p);
}

inline uint32_t up128(uint32_t v) { return (v + 127u) / 128u * 128u; }

// K-split of a matrix with n 64-column groups over the consumer warps: the largest divisor
// of the warp count not above n (the remaining warps take further row tiles).
inline int kw_for(int n)
{
    const int cand[6] = {12, 6, 4, 3, 2, 1};
    for (int i = 0; i < 6; i++)
        if (cand[i] <= n) return cand[i];
    return 1;
}

// Stride of the four row chunks of a stage: at least `bytes`, and 32 bytes more than a
// multiple of 128, so the same row of the four chunks falls on four different bank groups.
inline uint32_t chunk_stride(uint32_t bytes) { return (bytes + 95u) / 128u * 128u + 32u; }
inline uint32_t chunk_stride64(uint32_t bytes) { return (bytes + 63u) / 128u * 128u + 64u; }

// Pair-mode K split: the largest divisor of the warp count giving every warp exactly 8 (or
// else 4) of the n groups; 0 if none.
inline int kw_pair(int n)
{
    const int cand[6] = {12, 6, 4, 3, 2, 1};
    for (int per : {8, 4})
        for (int i = 0; i < 6; i++)
            if (n == cand[i] * per) return cand[i];
    return 0;
}

constexpr int kGpwMax = 8;

}  // namespace

int fused_phase_stamps(unsigned long long* host, int max_ctas, int* n_stamps)
{
#ifdef COLI_PHASE_STAMPS
    *n_stamps = kStamps;
    const int n = max_ctas < kStampCtas ? max_ctas : kStampCtas;
    if (cudaMemcpyFromSymbol(host, g_phase, sizeof(unsigned long long) * (size_t)n * kStamps) != cudaSuccess)
        return -1;
    return n;
#else
    (void)host;
    (void)max_ctas;
    *n_stamps = 0;
    return 0;
#endif
}

bool fused_plan(FusedParams& p, int num_sms, size_t smem_limit)
{
    const int H = p.H, I = p.I, E = p.E, T = p.T;
    if (T < 1 || T > kFusedMaxT || p.L < 1 || p.L > kFusedMaxLayers) return false;
    if (p.k < 1 || p.k > kFusedMaxK || p.k > E || E > 1024) return false;
    if (H % 128 || I % 64 || H < 128 || I < 64) return false;
    if (p.L > 1 && !p.norm) return false;
    p.NT = (T + 1) / 2;
    const int G = num_sms;
    p.grid = G;
    // gate/up: K = H; down: K = I
    const int ngg = H / 64, ngd = I / 64;
    p.KWg = kw_for(ngg);
    p.RSg = NCW / p.KWg;
    p.GPWg = (ngg + p.KWg - 1) / p.KWg;   // groups of the widest warp
    p.KWd = kw_for(ngd);
    p.RSd = NCW / p.KWd;
    p.GPWd = (ngd + p.KWd - 1) / p.KWd;
    if (p.GPWg > kGpwMax || p.GPWd > kGpwMax) return false;
    // gate/up stage: NTSg row tiles, about 32 KB or more, dividing the I / 8 tiles of a
    // segment when that is possible
    const uint32_t tile_all = 16u * (uint32_t)H / 2u + 16u * (uint32_t)H / 32u;
    int nts = (int)(32768u / tile_all);
    if (nts < 1) nts = 1;
    while (nts > 1 && 8 * nts > I) nts--;
    for (int n = nts; n >= 1; n--)
        if ((I / 8) % n == 0) {
            if (n * 2 >= nts) nts = n;
            break;
        }
    p.NTSg = nts;
    p.SPS = (I + 8 * nts - 1) / (8 * nts);
    // one token: both matrices in group pairs when each splits into warp shares of exactly 4
    // or 8 aligned groups; the 16-byte row reads need the chunks 64 bytes (mod 128) apart
    p.pair = 0;
    if (T == 1 && H % 512 == 0 && I % 512 == 0 && H <= 16 * NCT && p.k + p.n_shared <= 65535) {
        const int kg = kw_pair(ngg), kd = kw_pair(ngd);
        if (kg && kd) {
            p.pair = 1;
            p.KWg = kg;
            p.RSg = NCW / kg;
            p.GPWg = ngg / kg;
            p.KWd = kd;
            p.RSd = NCW / kd;
            p.GPWd = ngd / kd;
            // the stage's row tiles are a multiple of the row slots
            int n2 = (int)(32768u / (16u * (uint32_t)H / 2u + 16u * (uint32_t)H / 32u));
            if (n2 < 1) n2 = 1;
            n2 = (n2 + p.RSg - 1) / p.RSg * p.RSg;
            while (n2 > p.RSg && ((I / 8) % n2 != 0 || 8 * n2 > I)) n2 -= p.RSg;
            if ((I / 8) % n2 == 0 && 8 * n2 <= I) {
                nts = n2;
                p.NTSg = nts;
                p.SPS = (I + 8 * nts - 1) / (8 * nts);
            }
        }
    }
    p.gu_chunk = p.pair ? chunk_stride64(2u * nts * (uint32_t)H / 2u)
                        : chunk_stride(2u * nts * (uint32_t)H / 2u);
    p.gu_gsc = 8u * p.gu_chunk;
    p.gu_usc = p.gu_gsc + 8u * nts * (uint32_t)H / 32u;
    const uint32_t gu_stage = p.gu_usc + 8u * nts * (uint32_t)H / 32u;
    // down stage: the CTA's rows in four chunks, tiles of four rows per chunk
    p.rows_max = (H + G - 1) / G;
    p.ntdm = (((p.rows_max + 3) / 4) + 3) / 4;
    p.d_chunk = p.pair ? chunk_stride64(4u * p.ntdm * (uint32_t)I / 2u)
                       : chunk_stride(4u * p.ntdm * (uint32_t)I / 2u);
    p.d_sc_off = 4u * p.d_chunk;
    const uint32_t d_stage = p.d_sc_off + (uint32_t)(p.rows_max + 16) * (uint32_t)I / 32u + 32u;
    // router: whole rows per item (RC = 1) when a CTA's rows fit in a weight slot, else
    // rows in RC column chunks; the consumer threads share every item (at most 16
    // columns per thread) and the per-warp partial sums of all items fit the scratch
    uint32_t slot = gu_stage > d_stage ? gu_stage : d_stage;
    p.RC = 1;
    while (true) {
        const int im = (E * p.RC + G - 1) / G;
        const bool fits = (uint32_t)im * (uint32_t)(H / p.RC) * 4u <= slot && H / p.RC <= 16 * NCT &&
                          im * T <= 48;
        if (fits || (H / (2 * p.RC)) % 128 != 0) break;
        p.RC *= 2;
    }
    if (H / p.RC > 16 * NCT || ((E * p.RC + G - 1) / G) * T > 48) return false;
    p.RKc = H / p.RC;
    const int items_max = (E * p.RC + G - 1) / G;
    const uint32_t r_stage = (uint32_t)items_max * (uint32_t)p.RKc * 4u;
    if (r_stage > slot) slot = r_stage;
    p.slot_bytes = up128(slot);
    // fixed shared memory: head, two routing tables, partial sums, y rows, scratch
    const int S = 1 + T * p.k;
    uint32_t off = up128((uint32_t)sizeof(Head) + 2u * table_bytes(S));
    p.off_red = off;
    const uint32_t red_g = (uint32_t)p.KWg * p.NTSg * 16u * T;
    const uint32_t red_d = (uint32_t)p.KWd * p.ntdm * 16u * T;
    p.red_floats = red_g > red_d ? red_g : red_d;
    off = up128(off + (uint32_t)kRedBufs * p.red_floats * 4u);
    p.off_yacc = off;
    off = up128(off + (uint32_t)p.rows_max * T * 4u);
    p.hdig_bytes = p.pair ? up128((uint32_t)hdg_row_bytes(I)) : 0u;
    p.off_hdig = off;
    off = up128(off + (uint32_t)kDigBufs * p.hdig_bytes);
    p.off_hstage = off;   // pair mode: the layer input row
    off = up128(off + (p.pair ? 4u * (uint32_t)H : 0u));
    p.off_scratch = off;
    // consumer digit scratch (96 words per warp), then the control warp's logits,
    // selections, weights and bitmaps
    off = up128(off + NCW * 96u * 4u + (uint32_t)(T * E) * 4u + 2u * (uint32_t)(T * p.k) * 4u +
                (kFusedMaxT + 3) * 32u * 4u + (kTopkCand + 32) * 8u + 8u);
    p.off_ring = off;
    if (off + 2u * p.slot_bytes > smem_limit) return false;
    int nslot = (int)((smem_limit - off) / p.slot_bytes);
    if (nslot > kMaxSlots) nslot = kMaxSlots;
    p.nslot = nslot;
    p.smem = off + (size_t)nslot * p.slot_bytes;
    return true;
}

// Kernel variants by MMA column tiles and the widest warp's group count (registers hold
// one B operand per group): gate/up up to 4 or 8 groups, down up to 3 or 8.
template <int NTM, bool PAIR>
static cudaError_t launch_nt(const FusedParams& p, cudaStream_t s)
{
    if (p.GPWg <= 4)
        return p.GPWd <= 3 ? launch_fused<NTM, 4, 3, PAIR>(p, s) : launch_fused<NTM, 4, 8, PAIR>(p, s);
    return p.GPWd <= 3 ? launch_fused<NTM, 8, 3, PAIR>(p, s) : launch_fused<NTM, 8, 8, PAIR>(p, s);
}

// Pair mode: the warps' group counts exactly (4 or 8 for each matrix).
cudaError_t launch_pair(const FusedParams& p, cudaStream_t s)
{
    if (p.GPWg == 8) return p.GPWd == 8 ? launch_fused<1, 8, 8, true>(p, s) : launch_fused<1, 8, 4, true>(p, s);
    return p.GPWd == 8 ? launch_fused<1, 4, 8, true>(p, s) : launch_fused<1, 4, 4, true>(p, s);
}

cudaError_t fused_launch(const FusedParams& p, cudaStream_t s)
{
    if (p.NT == 2) return launch_nt<2, false>(p, s);
    return p.pair ? launch_pair(p, s) : launch_nt<1, false>(p, s);
}

}  // namespace coli
