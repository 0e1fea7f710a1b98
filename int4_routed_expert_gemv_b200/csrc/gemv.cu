// Streaming int4 GEMV kernels for the decode path (fp32 arithmetic contract).
//
//   mode 0, gate/up:  for every union expert (and the shared expert) and every
//                     intermediate row i:  g = G[i].x_t, u = U[i].x_t, h = silu(g)*u
//   mode 1, down:     y_t[r] (+)= sum over segments (shared first, then the union in
//                     ascending expert order) of w_(t,e) * D_e[r].h_(e,t)
//
// The batch union makes each distinct expert's weights cross HBM once per call: a
// segment is one expert with the list of tokens that selected it (colibri README.zh-CN,
// "工作原理 / 绝不为同一次磁盘读取等待两遍", batch union; the expert's three matrices sit
// next to each other in one blob, same section).
//
// Design (one CTA per SM, persistent over a contiguous share of rows):
//   * a producer warp streams contiguous row blocks of the packed nibbles and their fp16
//     group scales into a ring of shared-memory stages with the bulk-copy (TMA) engine,
//     completing on mbarriers; activations (x, or h for the down projection) arrive the
//     same way into vector buffers;
//   * consumer thread (rho, j) owns 16-byte column unit j (32 int4 weights = half a
//     group) of every row rho, rho+rl, ... of a stage.  The unit's activations are held in
//     registers as three int8 digit planes with one scale factor (load_digits for x; the
//     gate/up launch writes h in the same form), so one unit's dot product is 24 dp4a on
//     the offset-binary nibble bytes, exact in int32, then one scaling by digit factor
//     times group scale;
//   * per stage, the partials of the 8 values a thread holds are reduced across the
//     lanes of a row with a transposing butterfly (each shuffle halves the values a lane
//     keeps), then across warps through shared memory; finalizer threads apply SwiGLU
//     (mode 0) or the routing weight and the fixed-order combine into y (mode 1).
// In the decode layer call x was complete before the router launch began, so the gate/up
// launch stages it and forms token 0's digits while the router still runs.
// Every wait on an mbarrier is bounded; a timeout marks the workspace status word and
// the CTA runs to completion without further waiting, so no launch can hang.
#include "common.cuh"
#include "gemv.cuh"

namespace coli {
namespace {

constexpr int kMaxStages = 16;
constexpr int kMaxChunks = 64;      // pending chunks per flush
constexpr int kVecBufs = 4;         // activation (x or h digit record) buffers when not resident

// dp4a: c + sum_i a_i * b_i over the four bytes, exact in 32-bit integers; a's bytes
// unsigned, b's bytes signed (dp4a_us) or unsigned (dp4a_uu, wrapping mod 2^32)
__device__ __forceinline__ int32_t dp4a_us(uint32_t a, uint32_t b, int32_t c)
{
    int32_t d;
    asm("dp4a.u32.s32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(c));
    return d;
}

__device__ __forceinline__ int32_t dp4a_uu(uint32_t a, uint32_t b, int32_t c)
{
    uint32_t d;
    asm("dp4a.u32.u32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"((uint32_t)c));
    return (int32_t)d;
}

// Integer parts without the conversion unit: for |v| < 2^22, adding 1.5 * 2^23 leaves
// the integer part of v (rounded in the requested direction) in the low mantissa bits.
constexpr float kMagic = 12582912.0f;          // 1.5 * 2^23, bits 0x4B400000
__device__ __forceinline__ int floor_small(float v, float& fv)
{
    const float t = __fadd_rd(v, kMagic);
    fv = t - kMagic;
    return __float_as_int(t) - 0x4B400000;
}
__device__ __forceinline__ int rint_small(float v)
{
    return __float_as_int(__fadd_rn(v, kMagic)) - 0x4B400000;
}

// Activations of one 32-column unit as 8-bit digits.  With m = max |x_c| over the unit,
// X_c = clamp(x_c * 126 / m, -126, 126) is written as
//     X_c = a_c + b_c / 256 + c_c / 65536 + r_c,  a_c in [-126, 126] (signed),
//     b_c, c_c in [0, 255] (unsigned),  |r_c| <= 2^-16
// (floor digits, the last one rounded; when X_c - a_c rounds to 1.0f for a tiny negative
// X_c the middle digit saturates at 255), so that
//     sum_c q_c x_c = (m / (126 * 65536)) * sum_c q_c (65536 a_c + 256 b_c + c_c)
// up to about 1.2e-7 m per column, with the integer sum exact in int32 (below 2^31 for
// |q| <= 8 over 32 columns).  Weight nibbles arrive in offset binary n' = q + 8, so each
// digit's dp4a chain starts at -8 * sum_c digit_c.  Digits are packed in the byte order
// of the nibble words: word wi holds columns 8wi + {0,2,4,6} (low nibbles, even slot) and
// 8wi + {1,3,5,7} (high nibbles, odd slot).
__device__ __forceinline__ void load_digits(const float* src, uint32_t (&dg)[3][8],
                                            int32_t (&corr)[3], float& fac)
{
    const float4* s4 = reinterpret_cast<const float4*>(src);
    float mx = 0.0f;
#pragma unroll
    for (int q4 = 0; q4 < 8; q4++) {
        const float4 v = s4[q4];
        mx = fmaxf(mx, fmaxf(fmaxf(fabsf(v.x), fabsf(v.y)), fmaxf(fabsf(v.z), fabsf(v.w))));
    }
    const float inv = mx > 0.0f ? 126.0f / mx : 0.0f;
    fac = mx * (1.0f / (126.0f * 65536.0f));
    int32_t sum[3] = {0, 0, 0};
#pragma unroll
    for (int d = 0; d < 3; d++)
#pragma unroll
        for (int q = 0; q < 8; q++) dg[d][q] = 0u;
    // byte b of every packed word per pass (a rolled loop keeps the code short): slot s
    // holds column 8 (s / 2) + 2 b + (s % 2); each pass shifts the earlier bytes down
#pragma unroll 1
    for (int b = 0; b < 4; b++) {
        float2 xv[4];
#pragma unroll
        for (int w = 0; w < 4; w++) xv[w] = *reinterpret_cast<const float2*>(src + 8 * w + 2 * b);
#pragma unroll
        for (int sl = 0; sl < 8; sl++) {
            const float xc = (sl & 1) ? xv[sl >> 1].y : xv[sl >> 1].x;
            const float X = fminf(fmaxf(xc * inv, -126.0f), 126.0f);
            float a, bq;
            const int ai = floor_small(X, a);
            // X - a can round up to exactly 1.0f when X is a tiny negative number; the
            // second digit then saturates at 255 and the third absorbs the remainder
            const float r1 = (X - a) * 256.0f;
            int bi = floor_small(r1, bq);
            if (bi > 255) {
                bi = 255;
                bq = 255.0f;
            }
            const int ci = min(rint_small((r1 - bq) * 256.0f), 255);
            dg[0][sl] = (dg[0][sl] >> 8) | ((uint32_t)ai << 24);
            dg[1][sl] = (dg[1][sl] >> 8) | ((uint32_t)bi << 24);
            dg[2][sl] = (dg[2][sl] >> 8) | ((uint32_t)ci << 24);
            sum[0] += ai;
            sum[1] += bi;
            sum[2] += ci;
        }
    }
#pragma unroll
    for (int d = 0; d < 3; d++) corr[d] = -8 * sum[d];
}

// A warp turns 32 consecutive activations (lane l holds column l) into one digit record
// with the same digits as load_digits: words 0..23 are the packed planes (plane d, slot
// 2wi + p holds columns 8wi + 2b + p at byte b), words 24..26 the corrections
// -8 * sum(digit), word 27 the factor m / (126 * 65536).
__device__ __forceinline__ void store_digit_record(float hv, int lane, uint32_t* rec)
{
    float mx = fabsf(hv);
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
    const float inv = mx > 0.0f ? 126.0f / mx : 0.0f;
    const float X = fminf(fmaxf(hv * inv, -126.0f), 126.0f);
    float a, bq;
    const int ai = floor_small(X, a);
    const float r1 = (X - a) * 256.0f;       // may be exactly 256 for tiny negative X
    int bi = floor_small(r1, bq);
    if (bi > 255) {
        bi = 255;
        bq = 255.0f;
    }
    const int ci = min(rint_small((r1 - bq) * 256.0f), 255);
    const int di[3] = {ai, bi, ci};
    // lane L < 24 assembles word L: plane d = L / 8, slot s = L % 8
    const int d_me = lane >> 3, slot = lane & 7, wi = slot >> 1, par = slot & 1;
    uint32_t word = 0;
#pragma unroll
    for (int d = 0; d < 3; d++) {
#pragma unroll
        for (int bb = 0; bb < 4; bb++) {
            const int src = 8 * wi + 2 * bb + par;
            const int v = __shfl_sync(0xffffffffu, di[d], src);
            if (d == d_me) word |= ((uint32_t)v & 0xFFu) << (8 * bb);
        }
    }
    int sums[3];
#pragma unroll
    for (int d = 0; d < 3; d++) {
        int sv = di[d];
#pragma unroll
        for (int o = 16; o >= 1; o >>= 1) sv += __shfl_xor_sync(0xffffffffu, sv, o);
        sums[d] = sv;
    }
    uint32_t out = word;
    if (lane == 24) out = (uint32_t)(-8 * sums[0]);
    if (lane == 25) out = (uint32_t)(-8 * sums[1]);
    if (lane == 26) out = (uint32_t)(-8 * sums[2]);
    if (lane == 27) out = __float_as_uint(mx * (1.0f / (126.0f * 65536.0f)));
    if (lane < kDigitRecWords) rec[lane] = out;
}

// x [T][H] into digit records, one warp per 32-column unit (same digits as load_digits).
__global__ void __launch_bounds__(256) x_digits_kernel(const float* __restrict__ x, int T, int H,
                                                       uint8_t* __restrict__ rec)
{
    pdl_launch_dependents();
    const int lane = threadIdx.x & 31;
    const int U = H / 32;
    const int u = blockIdx.x * 8 + (threadIdx.x >> 5);
    if (u >= T * U) return;
    const int t = u / U, j = u - t * U;
    store_digit_record(x[(size_t)t * H + 32 * j + lane], lane,
                       reinterpret_cast<uint32_t*>(rec + (size_t)u * kDigitRecBytes));
}

// Transposing butterfly over W*2 lanes: at each level the lane with bit W set keeps the
// upper half of its values, sends the lower half, and adds what its partner sends.
template <int CUR, int W>
struct Bfly {
    template <int V>
    static __device__ __forceinline__ void run(float (&v)[V], int lane)
    {
        if constexpr (W >= 1) {
            if constexpr (CUR > 1) {
                constexpr int HALF = CUR / 2;
                const bool up = (lane & W) != 0;
#pragma unroll
                for (int i = 0; i < HALF; i++) {
                    const float send = up ? v[i] : v[i + HALF];
                    const float keep = up ? v[i + HALF] : v[i];
                    v[i] = keep + __shfl_xor_sync(0xffffffffu, send, W);
                }
                Bfly<HALF, W / 2>::run(v, lane);
            } else {
                v[0] += __shfl_xor_sync(0xffffffffu, v[0], W);
                Bfly<1, W / 2>::run(v, lane);
            }
        }
    }
};

struct Seg {
    const uint8_t* blob;
    int count;   // tokens of the segment
    int u;       // union entry, or -1 for the shared expert
    int base;    // first assignment position (union) / first h row (shared)
};

__device__ __forceinline__ Seg seg_info(const GemvParams& p, int s)
{
    Seg g;
    if (p.n_shared && s == 0) {
        g.blob = p.shared;
        g.count = p.T;
        g.u = -1;
        g.base = p.T * p.k;
    } else {
        const int u = s - p.n_shared;
        const int e = p.union_ids[u];
        g.blob = p.experts + (uint64_t)e * p.stride;
        g.u = u;
        g.base = p.offsets[u];
        g.count = p.offsets[u + 1] - g.base;
    }
    return g;
}

// token id and routing weight of token mm of a segment (the gate/up launch has no
// routing weights: p.wts is null there and wt is 0)
__device__ __forceinline__ void seg_token(const GemvParams& p, const Seg& g, int mm, int& tok,
                                          float& wt)
{
    if (g.u < 0) {
        tok = mm;
        wt = 1.0f;
    } else {
        const int a = p.assign[g.base + mm];
        tok = a / p.k;
        wt = p.wts ? p.wts[a] : 0.0f;
    }
}

template <int MODE>
__device__ __forceinline__ void cta_rows(const GemvParams& p, int nseg, int& r0, int& r1)
{
    // 32-bit arithmetic: gemv_plan keeps (E + 1) * N * gridDim below 2^32
    const uint32_t b = blockIdx.x, G = gridDim.x;
    if (MODE == 0) {
        // whole 32-row units, so every unit of h is finished by one CTA
        const uint32_t R = (uint32_t)nseg * (uint32_t)(p.N / 32);
        r0 = (int)(32u * (R * b / G));
        r1 = (int)(32u * (R * (b + 1) / G));
    } else {
        r0 = (int)((uint32_t)p.N * b / G);
        r1 = (int)((uint32_t)p.N * (b + 1) / G);
    }
}

// Calls f(seg, row0, nrows) for the CTA's pieces in the fixed order.  A piece is a run of
// rows of one segment, at most p.PR rows long (the partial-sum buffer holds one piece).
template <int MODE, class F>
__device__ __forceinline__ void for_each_piece(const GemvParams& p, int nseg, F&& f)
{
    int r0, r1;
    cta_rows<MODE>(p, nseg, r0, r1);
    if (MODE == 0) {
        int r = r0;
        while (r < r1) {
            const int s = (int)((uint32_t)r / (uint32_t)p.N);
            const int end = min(r1, (s + 1) * p.N);
            for (int q = r; q < end; q += p.PR) f(s, q - s * p.N, min(p.PR, end - q));
            r = end;
        }
    } else {
        if (r1 > r0)
            for (int s = 0; s < nseg; s++)
                for (int q = r0; q < r1; q += p.PR) f(s, q, min(p.PR, r1 - q));
    }
}

// Bookkeeping of a chunk (piece x up to MAXM tokens) whose partial sums wait in shared
// memory for the CTA's next flush.
struct ChunkMeta {   // 60 bytes
    int base, c0, M, row0, nrows, part_off, u;
    int tok[4];
    float wt[4];
};

// Consumer threads per CTA and values per thread per stage, by tokens per chunk.
__host__ __device__ constexpr int consumers_for(int maxm) { return maxm == 4 ? 192 : 384; }
__host__ __device__ constexpr int values_for(int maxm) { return 8; }

template <int MODE, int MAXM, int L>
__global__ void __launch_bounds__(consumers_for(MAXM) + 32, 1)
    gemv_kernel(const __grid_constant__ GemvParams p)
{
    constexpr int NCONS = consumers_for(MAXM);
    constexpr int kV = values_for(MAXM);
    constexpr int NMAT = (MODE == 0) ? 2 : 1;
    constexpr int RPT = kV / (MAXM * NMAT);
    static_assert(RPT >= 1 && RPT * MAXM * NMAT == kV, "value layout");

    extern __shared__ __align__(128) uint8_t smem[];
    uint64_t* full = reinterpret_cast<uint64_t*>(smem);
    uint64_t* empty = full + kMaxStages;
    uint64_t* vfull = empty + kMaxStages;
    uint64_t* vempty = vfull + kVecBufs;
    float* red = reinterpret_cast<float*>(smem + p.off_red);
    uint8_t* vec = smem + p.off_vec;
    uint8_t* stages = smem + p.off_stage;

    const int tid = threadIdx.x;
    const int warp = tid >> 5, lane = tid & 31;
    const int K = p.K;
    pdl_launch_dependents();

    if (tid == 0) {
        for (int s = 0; s < p.NS; s++) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], NCONS / 32);
        }
        for (int b = 0; b < kVecBufs; b++) {
            mbar_init(&vfull[b], 1);
            mbar_init(&vempty[b], NCONS / 32);
        }
        fence_barrier_init();
    }
    __syncthreads();

    // consumer geometry: thread (rho, j) owns column unit j of rows rho, rho + rl, ...
    const int U = p.U;
    const int rho = tid / U;
    const int j = tid - rho * U;
    const bool active = tid < NCONS && rho < p.rl;
    bool dead = false;
    // activations of this thread's 32-column unit as three int8 digits per column,
    // packed in the byte order of the offset-binary nibble words (see load_digits)
    uint32_t dg[MAXM][3][8];
    int32_t dcorr[MAXM][3];
    float dfac[MAXM];
    // resident activations: a slot's digits stay valid while its token is unchanged
    // (every chunk of a one-token batch uses the same x)
    int dtok[MAXM];
#pragma unroll
    for (int m = 0; m < MAXM; m++) dtok[m] = -1;

    // Everything above overlaps the preceding launch.  Routing, h and (unless x_early)
    // x are read only after it has completed.  An early x is staged now and token 0's
    // digits are formed while the preceding launch still runs.
    const bool early_x = MODE == 0 && p.x_early && p.resident && !p.xd;
    if (early_x) {
        if (tid == NCONS) {
            const uint32_t bytes = (uint32_t)p.T * (uint32_t)p.H * 4u;
            mbar_arrive_expect_tx(&vfull[0], bytes);
            bulk_g2s(vec, p.x, bytes, &vfull[0]);
        }
        if (MAXM == 1 && active) {
            if (!mbar_wait(&vfull[0], 0, p.status, 20)) {
                dead = true;
            } else {
                load_digits(reinterpret_cast<const float*>(vec) + 32 * j, dg[0], dcorr[0], dfac[0]);
                dtok[0] = 0;
            }
        }
    }
    pdl_wait();
    const int nu = *p.n_union;
    const int nseg = p.n_shared + nu;

    if (warp == NCONS / 32) {
        // ------------------------------- producer ------------------------------------
        if (lane == 0) {
            const uint64_t pol = policy_evict_first();
            bool dead = false;
            uint32_t it = 0, vit = 0;
            if (p.resident && !early_x) {
                if (p.xd) {
                    const uint32_t bytes = (uint32_t)p.T * (uint32_t)(p.U * kDigitRecBytes);
                    mbar_arrive_expect_tx(&vfull[0], bytes);
                    bulk_g2s(vec, p.xd, bytes, &vfull[0]);
                } else {
                    const uint32_t bytes = (uint32_t)p.T * (uint32_t)p.H * 4u;
                    mbar_arrive_expect_tx(&vfull[0], bytes);
                    bulk_g2s(vec, p.x, bytes, &vfull[0]);
                }
            }
            for_each_piece<MODE>(p, nseg, [&](int s, int row0, int nrows) {
                const Seg g = seg_info(p, s);
                for (int c0 = 0; c0 < g.count; c0 += MAXM) {
                    const int M = min(MAXM, g.count - c0);
                    if (!p.resident) {
                        const int b = vit % kVecBufs;
                        if (!dead && !mbar_wait(&vempty[b], ((vit / kVecBufs) & 1) ^ 1, p.status, 11))
                            dead = true;
                        if (!dead) {
                            uint8_t* dst = vec + b * p.vec_bytes;
                            const uint32_t recb = (uint32_t)(p.U * kDigitRecBytes);
                            const uint32_t rowb = (MODE == 0 && !p.xd) ? (uint32_t)K * 4u : recb;
                            mbar_arrive_expect_tx(&vfull[b], rowb * M);
                            if (MODE == 0 && p.xd) {
                                for (int m = 0; m < M; m++) {
                                    int tok;
                                    float wt;
                                    seg_token(p, g, c0 + m, tok, wt);
                                    bulk_g2s(dst + m * rowb, p.xd + (size_t)tok * recb, rowb, &vfull[b]);
                                }
                            } else if (MODE == 0) {
                                for (int m = 0; m < M; m++) {
                                    int tok;
                                    float wt;
                                    seg_token(p, g, c0 + m, tok, wt);
                                    bulk_g2s(dst + m * rowb, p.x + (size_t)tok * p.H, rowb, &vfull[b]);
                                }
                            } else {
                                bulk_g2s(dst, p.hd + (size_t)(g.base + c0) * p.U * kDigitRecBytes,
                                         (uint32_t)(p.U * kDigitRecBytes) * M, &vfull[b]);
                            }
                        }
                        vit++;
                    }
                    for (int r = 0; r < nrows; r += p.SR) {
                        const int nr = min(p.SR, nrows - r);
                        const int row = row0 + r;
                        const int st = it % p.NS;
                        if (!dead && !mbar_wait(&empty[st], ((it / p.NS) & 1) ^ 1, p.status, 12))
                            dead = true;
                        if (!dead) {
                            uint8_t* sbase = stages + (size_t)st * p.stage_bytes;
                            const uint32_t qb = (uint32_t)nr * (uint32_t)(K / 2);
                            const uint64_t s0 = (uint64_t)row * (K / 32);
                            const uint64_t a0 = s0 & ~15ull;
                            const uint64_t a1 = (s0 + (uint64_t)nr * (K / 32) + 15) & ~15ull;
                            const uint32_t sb = (uint32_t)(a1 - a0);
                            mbar_arrive_expect_tx(&full[st], NMAT * (qb + sb));
    #pragma unroll
                            for (int mt = 0; mt < NMAT; mt++) {
                                bulk_g2s_hint(sbase + (size_t)mt * p.SR * (K / 2),
                                              g.blob + p.q_off[mt] + (uint64_t)row * (K / 2), qb,
                                              &full[st], pol);
                                bulk_g2s_hint(sbase + p.stage_sc_off + mt * p.sc_area,
                                              g.blob + p.s_off[mt] + a0, sb, &full[st], pol);
                            }
                        }
                        it++;
                    }
                }
            });
            // drain: every issued copy has landed before the CTA may exit
            const uint32_t n_issued = it < (uint32_t)p.NS ? it : (uint32_t)p.NS;
            for (uint32_t q = 0; q < n_issued; q++) {
                const uint32_t last = it - 1 - q;   // most recent use of slot last % NS
                mbar_wait(&full[last % p.NS], (last / p.NS) & 1, p.status, 13);
            }
            if (!p.resident) {
                for (uint32_t q = 0; q < (vit < (uint32_t)kVecBufs ? vit : (uint32_t)kVecBufs); q++) {
                    const uint32_t last = vit - 1 - q;
                    mbar_wait(&vfull[last % kVecBufs], (last / kVecBufs) & 1, p.status, 14);
                }
            } else {
                mbar_wait(&vfull[0], 0, p.status, 15);
            }
        }
        return;
    }

    // --------------------------------- consumers ---------------------------------------
    const int nwg = (U >= 32) ? (U >> 5) : 1;
    const int wg = (U >= 32) ? (j >> 5) : 0;
    const int lane_l = lane & (L - 1);
    float* part = red;                                   // partial sums of pending chunks
    ChunkMeta* meta = reinterpret_cast<ChunkMeta*>(smem + p.off_meta);
    int nch = 0;                                         // pending chunks (CTA-uniform)
    uint32_t part_used = 0;
    int r0, r1;
    cta_rows<MODE>(p, nseg, r0, r1);

    if (MODE == 1) {
        // this CTA owns rows [r0, r1) of y for every token: start from residual or zero
        const int nrw = (int)(r1 - r0);
        for (int f = tid; f < p.T * nrw; f += NCONS) {
            const int t = f / nrw, r = (int)r0 + (f - t * nrw);
            p.y[(size_t)t * p.H + r] = p.residual ? p.residual[(size_t)t * p.H + r] : 0.0f;
        }
    }
    if (p.resident) {
        if (!dead && !mbar_wait(&vfull[0], 0, p.status, 21)) dead = true;
    }

    // Sum the pending chunks' partials: SwiGLU into h (mode 0) or the fixed-order combine
    // into y (mode 1: one thread per output row walks the chunks in order).
    auto flush = [&]() {
        named_bar(1, NCONS);
        if (MODE == 0) {
            // one warp per (chunk, token, 32-row unit): lane l finishes h of row 32u + l,
            // then the warp writes the unit as a digit record for the down projection
            const int nwarps = NCONS / 32;
            for (int c = 0; c < nch; c++) {
                const ChunkMeta& cm = meta[c];
                const float* pc = part + cm.part_off;
                const int units = cm.nrows / 32;
                for (int task = warp; task < units * cm.M; task += nwarps) {
                    const int m = task / units, uu = task - m * units;
                    const int rl_ = uu * 32 + lane;
                    const float* q = pc + ((size_t)(rl_ * MAXM + m) * NMAT) * nwg;
                    float gs = 0.0f, us = 0.0f;
                    for (int w2 = 0; w2 < nwg; w2++) {
                        gs += q[w2];
                        us += q[nwg + w2];
                    }
                    const float hv = gs / (1.0f + expf(-gs)) * us;
                    const int urow = (cm.row0 >> 5) + uu;   // unit index along I
                    uint32_t* rec = reinterpret_cast<uint32_t*>(
                        p.hd + ((size_t)(cm.base + cm.c0 + m) * (p.I / 32) + urow) * kDigitRecBytes);
                    store_digit_record(hv, lane, rec);
                }
            }
        } else {
            const int nrw = (int)(r1 - r0);
            for (int rr = tid; rr < nrw; rr += NCONS) {
                const int r = (int)r0 + rr;
                if (p.T == 1) {
                    // one token: y read and written once per flush, the additions in chunk
                    // order in a register
                    for (int t = 0; t < p.T; t++) {
                        float* yp = p.y + (size_t)t * p.H + r;
                        float v = *yp;
                        for (int c = 0; c < nch; c++) {
                            const ChunkMeta& cm = meta[c];
                            const int rl_ = r - cm.row0;
                            if (rl_ < 0 || rl_ >= cm.nrows) continue;
                            const float* pc = part + cm.part_off;
                            for (int m = 0; m < cm.M; m++) {
                                if (cm.tok[m] != t) continue;
                                const float* q = pc + (size_t)(rl_ * MAXM + m) * nwg;
                                float d = 0.0f;
                                for (int w2 = 0; w2 < nwg; w2++) d += q[w2];
                                v = v + cm.wt[m] * d;
                            }
                        }
                        *yp = v;
                    }
                    continue;
                }
                for (int c = 0; c < nch; c++) {
                    const ChunkMeta& cm = meta[c];
                    const int rl_ = r - cm.row0;
                    if (rl_ < 0 || rl_ >= cm.nrows) continue;
                    const float* pc = part + cm.part_off;
                    for (int m = 0; m < cm.M; m++) {
                        const float* q = pc + (size_t)(rl_ * MAXM + m) * nwg;
                        float d = 0.0f;
                        for (int w2 = 0; w2 < nwg; w2++) d += q[w2];
                        float* yp = p.y + (size_t)cm.tok[m] * p.H + r;
                        *yp = *yp + cm.wt[m] * d;
                    }
                }
            }
        }
        named_bar(1, NCONS);
        nch = 0;
        part_used = 0;
    };

    uint32_t it = 0, vit = 0;

    for_each_piece<MODE>(p, nseg, [&](int s, int row0, int nrows) {
        const Seg g = seg_info(p, s);
        for (int c0 = 0; c0 < g.count; c0 += MAXM) {
            const int M = min(MAXM, g.count - c0);
            const uint32_t need = (uint32_t)nrows * MAXM * NMAT * nwg;
            if (nch == kMaxChunks || part_used + need > p.part_cap) flush();
            const uint32_t off = part_used;
            if (tid == 0) {
                ChunkMeta& cm = meta[nch];
                cm.base = g.base;
                cm.c0 = c0;
                cm.M = M;
                cm.row0 = row0;
                cm.nrows = nrows;
                cm.part_off = (int)off;
                cm.u = g.u;
                for (int m = 0; m < 4; m++) {
                    int tok = 0;
                    float wt = 0.0f;
                    if (m < M) seg_token(p, g, c0 + m, tok, wt);
                    cm.tok[m] = tok;
                    cm.wt[m] = wt;
                }
            }
            nch++;
            part_used += need;
            float* pc = part + off;
            // ---- activations for this chunk into registers (as int8 digits)
            const float* vsrc;
            int b = 0;
            if (!p.resident) {
                b = vit % kVecBufs;
                if (!dead && !mbar_wait(&vfull[b], (vit / kVecBufs) & 1, p.status, 22)) dead = true;
                vsrc = reinterpret_cast<const float*>(vec + b * p.vec_bytes);
            } else {
                vsrc = reinterpret_cast<const float*>(vec);
            }
#pragma unroll
            for (int m = 0; m < MAXM; m++) {
                if (m < M && active) {
                    int row_in_vec = m;
                    if (p.resident) {
                        int tok;
                        float wt;
                        seg_token(p, g, c0 + m, tok, wt);
                        row_in_vec = tok;
                    }
                    if (MODE == 0 && !p.xd) {
                        if (MAXM > 1 || !p.resident || dtok[m] != row_in_vec)   // one-token chunks only
                            load_digits(vsrc + (size_t)row_in_vec * K + 32 * j, dg[m], dcorr[m], dfac[m]);
                        dtok[m] = p.resident ? row_in_vec : -1;
                    } else {
                        // digit records: x records of the layer call, or h from the gate/up launch
                        const uint4* rec = reinterpret_cast<const uint4*>(
                            reinterpret_cast<const uint8_t*>(vsrc) +
                            ((size_t)row_in_vec * p.U + j) * kDigitRecBytes);
#pragma unroll
                        for (int d = 0; d < 3; d++) {
                            const uint4 r0v = rec[2 * d], r1v = rec[2 * d + 1];
                            dg[m][d][0] = r0v.x; dg[m][d][1] = r0v.y; dg[m][d][2] = r0v.z; dg[m][d][3] = r0v.w;
                            dg[m][d][4] = r1v.x; dg[m][d][5] = r1v.y; dg[m][d][6] = r1v.z; dg[m][d][7] = r1v.w;
                        }
                        const uint4 tail = rec[6];
                        dcorr[m][0] = (int32_t)tail.x;
                        dcorr[m][1] = (int32_t)tail.y;
                        dcorr[m][2] = (int32_t)tail.z;
                        dfac[m] = __uint_as_float(tail.w);
                    }
                } else {
#pragma unroll
                    for (int d = 0; d < 3; d++) {
                        dcorr[m][d] = 0;
#pragma unroll
                        for (int q = 0; q < 8; q++) dg[m][d][q] = 0u;
                    }
                    dfac[m] = 0.0f;
                    dtok[m] = -1;
                }
            }
            if (!p.resident) {
                __syncwarp();
                if (lane == 0) mbar_arrive(&vempty[b]);
                vit++;
            }

            // ---- stages
            for (int r = 0; r < nrows; r += p.SR) {
                const int nr = min(p.SR, nrows - r);
                const int row = row0 + r;
                const int st = it % p.NS;
                if (!dead && !mbar_wait(&full[st], (it / p.NS) & 1, p.status, 23)) dead = true;
                const uint8_t* sbase = stages + (size_t)st * p.stage_bytes;
                const int delta = (int)(((uint64_t)row * (K / 32)) & 15ull);
                float v[kV];
#pragma unroll
                for (int q = 0; q < kV; q++) v[q] = 0.0f;
                if (active) {
                    // every row slot of the stage is computed (slots past nr read stale but
                    // in-bounds shared memory and are discarded below), so the loads of all
                    // rows issue together and the dp4a chains of different rows interleave
                    uint4 wv[RPT][NMAT];
                    float scv[RPT][NMAT];
#pragma unroll
                    for (int i = 0; i < RPT; i++) {
                        const int rr = rho + p.rl * i;
#pragma unroll
                        for (int mt = 0; mt < NMAT; mt++) {
                            wv[i][mt] = *reinterpret_cast<const uint4*>(
                                sbase + (size_t)mt * p.SR * (K / 2) + (size_t)rr * (K / 2) + 16 * j);
                            scv[i][mt] = __half2float(*reinterpret_cast<const __half*>(
                                sbase + p.stage_sc_off + mt * p.sc_area + delta + rr * (K / 32) +
                                (j >> 1) * 2));
                        }
                    }
#pragma unroll
                    for (int i = 0; i < RPT; i++) {
#pragma unroll
                        for (int mt = 0; mt < NMAT; mt++) {
                            // offset-binary nibbles n' = q + 8 as bytes: even columns of word wi
                            // in lo[wi], odd columns in hi[wi]
                            const uint32_t wds[4] = {wv[i][mt].x, wv[i][mt].y, wv[i][mt].z, wv[i][mt].w};
                            uint32_t lo[4], hi[4];
#pragma unroll
                            for (int wi = 0; wi < 4; wi++) {
                                lo[wi] = and_xor(wds[wi], 0x0F0F0F0Fu, 0x08080808u);
                                hi[wi] = and_xor(wds[wi] >> 4, 0x0F0F0F0Fu, 0x08080808u);
                            }
#pragma unroll
                            for (int m = 0; m < MAXM; m++) {
                                if (m < M) {
                                    // two independent chains per digit (even / odd columns)
                                    int32_t e0 = dcorr[m][0], o0 = 0;
                                    int32_t e1 = dcorr[m][1], o1 = 0;
                                    int32_t e2 = dcorr[m][2], o2 = 0;
#pragma unroll
                                    for (int wi = 0; wi < 4; wi++) {
                                        e0 = dp4a_us(lo[wi], dg[m][0][2 * wi], e0);
                                        o0 = dp4a_us(hi[wi], dg[m][0][2 * wi + 1], o0);
                                        e1 = dp4a_uu(lo[wi], dg[m][1][2 * wi], e1);
                                        o1 = dp4a_uu(hi[wi], dg[m][1][2 * wi + 1], o1);
                                        e2 = dp4a_uu(lo[wi], dg[m][2][2 * wi], e2);
                                        o2 = dp4a_uu(hi[wi], dg[m][2][2 * wi + 1], o2);
                                    }
                                    // sum_c q_c * (65536 a_c + 256 b_c + c_c), exact in int32
                                    const int32_t S = ((e0 + o0) * 256 + (e1 + o1)) * 256 + (e2 + o2);
                                    v[(i * MAXM + m) * NMAT + mt] = (float)S * (dfac[m] * scv[i][mt]);
                                }
                            }
                        }
                    }
                }
                __syncwarp();
                if (lane == 0) mbar_arrive(&empty[st]);

                if (active) {
                    Bfly<kV, L / 2>::run(v, lane);
                    // value index vi = (i*MAXM + m)*NMAT + mt  ->  row r + rho + rl*i
                    if (kV >= L) {
#pragma unroll
                        for (int i2 = 0; i2 < kV / L; i2++) {
                            const int vi = i2 + (kV / L) * lane_l;
                            const int i = vi / (MAXM * NMAT), mm = vi % (MAXM * NMAT);
                            const int rr = rho + p.rl * i;
                            if (rr < nr)
                                pc[((size_t)(r + rr) * MAXM * NMAT + mm) * nwg + wg] = v[i2];
                        }
                    } else {
                        constexpr int REP = (kV >= L) ? 1 : L / kV;
                        if ((lane_l % REP) == 0) {
                            const int vi = lane_l / REP;
                            const int i = vi / (MAXM * NMAT), mm = vi % (MAXM * NMAT);
                            const int rr = rho + p.rl * i;
                            if (rr < nr)
                                pc[((size_t)(r + rr) * MAXM * NMAT + mm) * nwg + wg] = v[0];
                        }
                    }
                }
                it++;
            }
        }
    });
    flush();
}

template <int MODE, int MAXM, int L>
cudaError_t launch_one(const GemvParams& p, const GemvConfig& c, cudaStream_t s)
{
    auto kern = gemv_kernel<MODE, MAXM, L>;
    // the opt-in shared-memory size is set once per device and size (host-side cache)
    static int set_bytes[64] = {0};
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= 64 || set_bytes[dev] < (int)c.smem) {
        e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)c.smem);
        if (e != cudaSuccess) return e;
        if (dev >= 0 && dev < 64) set_bytes[dev] = (int)c.smem;
    }
    // programmatic stream serialization: the kernel may be scheduled while the previous
    // one finishes (it waits for it in-kernel before reading its results)
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(c.grid);
    cfg.blockDim = dim3(c.consumers + 32);
    cfg.dynamicSmemBytes = c.smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kern, p);
}

template <int MODE, int MAXM>
cudaError_t launch_l(const GemvParams& p, const GemvConfig& c, cudaStream_t s)
{
    switch (c.lanes) {
    case 32: return launch_one<MODE, MAXM, 32>(p, c, s);
    case 16: return launch_one<MODE, MAXM, 16>(p, c, s);
    case 8: return launch_one<MODE, MAXM, 8>(p, c, s);
    case 4: return launch_one<MODE, MAXM, 4>(p, c, s);
    case 2: return launch_one<MODE, MAXM, 2>(p, c, s);
    }
    return cudaErrorInvalidValue;
}

template <int MODE>
cudaError_t launch_m(const GemvParams& p, const GemvConfig& c, cudaStream_t s)
{
    switch (c.maxm) {
    case 1: return launch_l<MODE, 1>(p, c, s);
    case 2: return launch_l<MODE, 2>(p, c, s);
    case 4: return launch_l<MODE, 4>(p, c, s);
    }
    return cudaErrorInvalidValue;
}

inline uint32_t align_up(uint32_t v, uint32_t a) { return (v + a - 1) / a * a; }

}  // namespace

bool gemv_plan(int mode, GemvParams& p, GemvConfig& c, int num_sms, size_t smem_limit)
{
    const int NMAT = mode == 0 ? 2 : 1;
    p.K = mode == 0 ? p.H : p.I;
    p.N = mode == 0 ? p.I : p.H;
    p.U = p.K / 32;
    if (p.K % 64 || p.U < 2) return false;
    // the kernels split rows with 32-bit products (segments x rows x CTAs)
    if ((uint64_t)(p.E + 1) * (uint64_t)p.N * (uint64_t)num_sms >= (1ull << 32)) return false;
    // tokens per chunk: small batches spread over many experts, so most routed segments
    // hold one token; one-token chunks keep 8 rows per stage (the shared expert's rows are
    // then re-read per token, from L2).  The down projection of a short intermediate
    // dimension keeps 4-token chunks: its per-chunk h loads, not its rows, set the pace.
    if (mode == 0)
        c.maxm = p.T <= 8 ? 1 : 2;
    else
        c.maxm = p.T <= 1 ? 1 : (p.T <= 8 && p.I >= 1024 ? 1 : 4);
    c.consumers = consumers_for(c.maxm);
    const int kV = values_for(c.maxm);
    if (p.U >= 32) {
        if (p.U % 32 || p.U > c.consumers) return false;
        c.lanes = 32;
    } else {
        if (p.U & (p.U - 1)) return false;
        c.lanes = p.U;
    }
    p.rl = c.consumers / p.U;
    c.rpt = kV / (c.maxm * NMAT);
    p.SR = p.rl * c.rpt;
    const int nwg = p.U >= 32 ? p.U / 32 : 1;
    // partial sums: a decode CTA's whole share of rows fits, larger shares flush in pieces
    p.part_cap = 4096;                                    // 16 KB
    const uint32_t per_row = (uint32_t)c.maxm * NMAT * nwg;
    p.PR = (int)(p.part_cap / per_row);
    if (mode == 0) p.PR = p.PR / 32 * 32;   // pieces are whole 32-row units
    if (p.PR < 1) return false;
    p.off_meta = 512;
    p.off_red = align_up(p.off_meta + 64u * 64u, 128);    // kMaxChunks x sizeof(ChunkMeta) <= 64
    const uint32_t red_bytes = p.part_cap * 4u;
    const uint64_t xres = (uint64_t)p.T * p.H * 4ull;
    p.resident = (mode == 0 && xres <= 100u * 1024u) ? 1 : 0;
    const bool recs = mode == 1 || p.xd;   // activations arrive as digit records
    const uint32_t row_bytes = recs ? (uint32_t)p.U * kDigitRecBytes : (uint32_t)p.K * 4u;
    p.vec_bytes = p.resident ? (uint32_t)p.T * row_bytes : (uint32_t)c.maxm * row_bytes;
    const uint32_t nvec = p.resident ? 1 : kVecBufs;
    p.off_vec = align_up(p.off_red + red_bytes, 128);
    p.off_stage = align_up(p.off_vec + nvec * p.vec_bytes, 128);
    p.sc_area = align_up((uint32_t)p.SR * (p.K / 32) + 32, 16);
    p.stage_sc_off = (uint32_t)NMAT * p.SR * (p.K / 2);
    p.stage_bytes = align_up(p.stage_sc_off + NMAT * p.sc_area, 128);
    if (p.off_stage >= smem_limit) return false;
    int ns = (int)((smem_limit - p.off_stage) / p.stage_bytes);
    if (ns < 2) return false;
    p.NS = ns > 8 ? 8 : ns;
    c.smem = p.off_stage + (size_t)p.NS * p.stage_bytes;
    const uint64_t IH = (uint64_t)p.I * p.H;
    if (mode == 0) {
        p.q_off[0] = 0;
        p.q_off[1] = IH / 2;
        p.s_off[0] = 3 * IH / 2;
        p.s_off[1] = 3 * IH / 2 + IH / 32;
        c.grid = num_sms;
    } else {
        p.q_off[0] = IH;
        p.q_off[1] = 0;
        p.s_off[0] = 3 * IH / 2 + 2 * (IH / 32);
        p.s_off[1] = 0;
        c.grid = p.H < num_sms ? p.H : num_sms;
    }
    return true;
}

cudaError_t x_digits_launch(const float* x, int T, int H, uint8_t* rec, cudaStream_t s)
{
    const int units = T * (H / 32);
    if (units <= 0) return cudaSuccess;
    x_digits_kernel<<<(units + 7) / 8, 256, 0, s>>>(x, T, H, rec);
    return cudaGetLastError();
}

cudaError_t gemv_launch(int mode, const GemvParams& p, const GemvConfig& c, cudaStream_t s)
{
    return mode == 0 ? launch_m<0>(p, c, s) : launch_m<1>(p, c, s);
}

}  // namespace coli
