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
//     group) of every row rho, rho+rl, ... of a stage, keeps the matching 32 activations
//     of each token in registers, and dequantises in registers: a nibble is placed into
//     the mantissa of a float with a fixed exponent (one LOP3), the exponent's offset is
//     removed by a packed f32x2 add (exact), and f32x2 FMAs accumulate q*x; the partial
//     is scaled by the group scale, so every product and scale is exact before rounding;
//   * per stage, the partials of the 8 values a thread holds are reduced across the
//     lanes of a row with a transposing butterfly (each shuffle halves the values a lane
//     keeps), then across warps through shared memory; finalizer threads apply SwiGLU
//     (mode 0) or the routing weight and the fixed-order combine into y (mode 1).
// Every wait on an mbarrier is bounded; a timeout marks the workspace status word and
// the CTA runs to completion without further waiting, so no launch can hang.
#include "common.cuh"
#include "gemv.cuh"

namespace coli {
namespace {

constexpr int kV = 8;            // values per consumer thread and stage
constexpr int kBarFull = 0;      // mbarrier slots in shared memory
constexpr int kMaxStages = 16;

// 8 int4 values of one 32-bit word -> 4 exact float pairs (columns (0,1) (2,3) (4,5) (6,7)).
// Nibble k sits at bits 4k.  For k <= 4 the nibble lies inside a float mantissa whose
// exponent gives bit 4k the weight 1: (w & 0xF<<4k) ^ (exp_k | 8<<4k) has the value
// 2^(23-4k) + (n ^ 8), and n ^ 8 = q + 8 for the two's-complement nibble n of q.
// Nibbles 5..7 are taken from w >> 12 (positions of nibbles 2..4).  Subtracting
// 2^(23-4k) + 8 is exact, so the pairs hold q exactly.
__device__ __forceinline__ void dequant8(uint32_t w, uint64_t (&q)[4])
{
    const uint32_t w2 = w >> 12;
    const uint32_t f0 = and_xor(w, 0x0000000Fu, 0x4B000008u);   // 2^23 + q + 8
    const uint32_t f1 = and_xor(w, 0x000000F0u, 0x49000080u);   // 2^19 + q + 8
    const uint32_t f2 = and_xor(w, 0x00000F00u, 0x47000800u);   // 2^15 + q + 8
    const uint32_t f3 = and_xor(w, 0x0000F000u, 0x45008000u);   // 2^11 + q + 8
    const uint32_t f4 = and_xor(w, 0x000F0000u, 0x43080000u);   // 2^7  + q + 8
    const uint32_t f5 = and_xor(w2, 0x00000F00u, 0x47000800u);
    const uint32_t f6 = and_xor(w2, 0x0000F000u, 0x45008000u);
    const uint32_t f7 = and_xor(w2, 0x000F0000u, 0x43080000u);
    q[0] = fadd2(pk2(f0, f1), pk2f(-8388616.0f, -524296.0f));
    q[1] = fadd2(pk2(f2, f3), pk2f(-32776.0f, -2056.0f));
    q[2] = fadd2(pk2(f4, f5), pk2f(-136.0f, -32776.0f));
    q[3] = fadd2(pk2(f6, f7), pk2f(-2056.0f, -136.0f));
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

// token id and routing weight of token mm of a segment
__device__ __forceinline__ void seg_token(const GemvParams& p, const Seg& g, int mm, int& tok,
                                          float& wt)
{
    if (g.u < 0) {
        tok = mm;
        wt = 1.0f;
    } else {
        const int a = p.assign[g.base + mm];
        tok = a / p.k;
        wt = p.wts[a];
    }
}

template <int MODE>
__device__ __forceinline__ void cta_rows(const GemvParams& p, int nseg, int64_t& r0, int64_t& r1)
{
    const int64_t R = (MODE == 0) ? (int64_t)nseg * p.N : (int64_t)p.N;
    r0 = R * blockIdx.x / gridDim.x;
    r1 = R * (blockIdx.x + 1) / gridDim.x;
}

// Calls f(seg, row0, nrows) for the CTA's pieces in the fixed order.
template <int MODE, class F>
__device__ __forceinline__ void for_each_piece(const GemvParams& p, int nseg, F&& f)
{
    int64_t r0, r1;
    cta_rows<MODE>(p, nseg, r0, r1);
    if (MODE == 0) {
        int64_t r = r0;
        while (r < r1) {
            const int s = (int)(r / p.N);
            const int64_t end = min(r1, (int64_t)(s + 1) * p.N);
            f(s, (int)(r - (int64_t)s * p.N), (int)(end - r));
            r = end;
        }
    } else {
        if (r1 > r0)
            for (int s = 0; s < nseg; s++) f(s, (int)r0, (int)(r1 - r0));
    }
}

template <int MODE, int MAXM, int L>
__global__ void __launch_bounds__((MAXM == 4 ? 192 : 384) + 32, 1)
    gemv_kernel(const __grid_constant__ GemvParams p)
{
    constexpr int NCONS = (MAXM == 4) ? 192 : 384;
    constexpr int NMAT = (MODE == 0) ? 2 : 1;
    constexpr int RPT = kV / (MAXM * NMAT);
    static_assert(RPT >= 1 && RPT * MAXM * NMAT == kV, "value layout");

    extern __shared__ __align__(128) uint8_t smem[];
    uint64_t* full = reinterpret_cast<uint64_t*>(smem);
    uint64_t* empty = full + kMaxStages;
    uint64_t* vfull = empty + kMaxStages;
    uint64_t* vempty = vfull + 2;
    float* red = reinterpret_cast<float*>(smem + p.off_red);
    uint8_t* vec = smem + p.off_vec;
    uint8_t* stages = smem + p.off_stage;

    const int tid = threadIdx.x;
    const int warp = tid >> 5, lane = tid & 31;
    const int K = p.K;
    const int nu = *p.n_union;
    const int nseg = p.n_shared + nu;

    if (tid == 0) {
        for (int s = 0; s < p.NS; s++) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], NCONS / 32);
        }
        for (int b = 0; b < 2; b++) {
            mbar_init(&vfull[b], 1);
            mbar_init(&vempty[b], NCONS / 32);
        }
        fence_barrier_init();
    }
    __syncthreads();

    if (warp == NCONS / 32) {
        // ------------------------------- producer ------------------------------------
        if (lane != 0) return;
        const uint64_t pol = policy_evict_first();
        bool dead = false;
        uint32_t it = 0, vit = 0;
        if (p.resident) {
            const uint32_t bytes = (uint32_t)p.T * (uint32_t)p.H * 4u;
            mbar_arrive_expect_tx(&vfull[0], bytes);
            bulk_g2s(vec, p.x, bytes, &vfull[0]);
        }
        for_each_piece<MODE>(p, nseg, [&](int s, int row0, int nrows) {
            const Seg g = seg_info(p, s);
            for (int c0 = 0; c0 < g.count; c0 += MAXM) {
                const int M = min(MAXM, g.count - c0);
                if (!p.resident) {
                    const int b = vit & 1;
                    if (!dead && !mbar_wait(&vempty[b], ((vit >> 1) & 1) ^ 1, p.status, 11))
                        dead = true;
                    if (!dead) {
                        uint8_t* dst = vec + b * p.vec_bytes;
                        const uint32_t rowb = (uint32_t)K * 4u;
                        mbar_arrive_expect_tx(&vfull[b], rowb * M);
                        if (MODE == 0) {
                            for (int m = 0; m < M; m++) {
                                int tok;
                                float wt;
                                seg_token(p, g, c0 + m, tok, wt);
                                bulk_g2s(dst + m * rowb, p.x + (size_t)tok * p.H, rowb, &vfull[b]);
                            }
                        } else {
                            bulk_g2s(dst, p.h + (size_t)(g.base + c0) * p.I, rowb * M, &vfull[b]);
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
            for (uint32_t q = 0; q < (vit < 2u ? vit : 2u); q++) {
                const uint32_t last = vit - 1 - q;
                mbar_wait(&vfull[last & 1], (last >> 1) & 1, p.status, 14);
            }
        } else {
            mbar_wait(&vfull[0], 0, p.status, 15);
        }
        return;
    }

    // --------------------------------- consumers ---------------------------------------
    const int U = p.U;
    const int rho = tid / U;
    const int j = tid - rho * U;
    const bool active = rho < p.rl;
    const int nwg = (U >= 32) ? (U >> 5) : 1;
    const int wg = (U >= 32) ? (j >> 5) : 0;
    const int lane_l = lane & (L - 1);
    bool dead = false;

    if (MODE == 1) {
        // this CTA owns rows [r0, r1) of y for every token: start from residual or zero
        int64_t r0, r1;
        cta_rows<MODE>(p, nseg, r0, r1);
        const int nrw = (int)(r1 - r0);
        for (int f = tid; f < p.T * nrw; f += NCONS) {
            const int t = f / nrw, r = (int)r0 + (f - t * nrw);
            p.y[(size_t)t * p.H + r] = p.residual ? p.residual[(size_t)t * p.H + r] : 0.0f;
        }
    }
    if (p.resident) {
        if (!mbar_wait(&vfull[0], 0, p.status, 21)) dead = true;
    }

    uint64_t xr[MAXM][16];   // activation pairs of this thread's column unit
    uint32_t it = 0, vit = 0;

    for_each_piece<MODE>(p, nseg, [&](int s, int row0, int nrows) {
        const Seg g = seg_info(p, s);
        for (int c0 = 0; c0 < g.count; c0 += MAXM) {
            const int M = min(MAXM, g.count - c0);
            // ---- activations for this chunk into registers
            const float* vsrc;
            int b = 0;
            if (!p.resident) {
                b = vit & 1;
                if (!dead && !mbar_wait(&vfull[b], (vit >> 1) & 1, p.status, 22)) dead = true;
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
                    const float4* src =
                        reinterpret_cast<const float4*>(vsrc + (size_t)row_in_vec * K + 32 * j);
#pragma unroll
                    for (int q4 = 0; q4 < 8; q4++) {
                        const float4 v4 = src[q4];
                        xr[m][2 * q4] = pk2f(v4.x, v4.y);
                        xr[m][2 * q4 + 1] = pk2f(v4.z, v4.w);
                    }
                } else {
#pragma unroll
                    for (int q = 0; q < 16; q++) xr[m][q] = 0ull;
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
#pragma unroll
                    for (int i = 0; i < RPT; i++) {
                        const int rr = rho + p.rl * i;
                        if (rr < nr) {
#pragma unroll
                            for (int mt = 0; mt < NMAT; mt++) {
                                const uint4 wv = *reinterpret_cast<const uint4*>(
                                    sbase + (size_t)mt * p.SR * (K / 2) + (size_t)rr * (K / 2) + 16 * j);
                                const float sc = __half2float(*reinterpret_cast<const __half*>(
                                    sbase + p.stage_sc_off + mt * p.sc_area + delta + rr * (K / 32) +
                                    (j >> 1) * 2));
                                uint64_t acc[MAXM];
#pragma unroll
                                for (int m = 0; m < MAXM; m++) acc[m] = 0ull;
                                const uint32_t wds[4] = {wv.x, wv.y, wv.z, wv.w};
#pragma unroll
                                for (int wi = 0; wi < 4; wi++) {
                                    uint64_t qq[4];
                                    dequant8(wds[wi], qq);
#pragma unroll
                                    for (int m = 0; m < MAXM; m++) {
                                        if (m < M) {
#pragma unroll
                                            for (int pi = 0; pi < 4; pi++)
                                                acc[m] = ffma2(qq[pi], xr[m][wi * 4 + pi], acc[m]);
                                        }
                                    }
                                }
#pragma unroll
                                for (int m = 0; m < MAXM; m++) {
                                    const float2 a = unpk2(acc[m]);
                                    v[(i * MAXM + m) * NMAT + mt] = sc * (a.x + a.y);
                                }
                            }
                        }
                    }
                }
                __syncwarp();
                if (lane == 0) mbar_arrive(&empty[st]);

                float* rbuf = red + (size_t)(it & 1) * p.rl * nwg * kV;
                if (active) {
                    Bfly<kV, L / 2>::run(v, lane);
                    if (kV >= L) {
#pragma unroll
                        for (int i2 = 0; i2 < kV / L; i2++)
                            rbuf[((size_t)rho * nwg + wg) * kV + i2 + (kV / L) * lane_l] = v[i2];
                    } else {
                        constexpr int REP = (kV >= L) ? 1 : L / kV;
                        if ((lane_l % REP) == 0) rbuf[((size_t)rho * nwg + wg) * kV + lane_l / REP] = v[0];
                    }
                }
                named_bar(1, NCONS);
                // ---- finalize: one thread per (row, token)
                for (int f = tid; f < p.SR * M; f += NCONS) {
                    const int m = f / p.SR;
                    const int rr = f - m * p.SR;
                    if (rr >= nr) continue;
                    const int rho2 = rr % p.rl, i = rr / p.rl;
                    const float* rv = rbuf + (size_t)rho2 * nwg * kV;
                    if (MODE == 0) {
                        float gs = 0.0f, us = 0.0f;
                        for (int w2 = 0; w2 < nwg; w2++) {
                            gs += rv[w2 * kV + (i * MAXM + m) * 2 + 0];
                            us += rv[w2 * kV + (i * MAXM + m) * 2 + 1];
                        }
                        const float hv = gs / (1.0f + expf(-gs)) * us;
                        p.h[(size_t)(g.base + c0 + m) * p.I + row + rr] = hv;
                    } else {
                        float d = 0.0f;
                        for (int w2 = 0; w2 < nwg; w2++) d += rv[w2 * kV + i * MAXM + m];
                        int tok;
                        float wt;
                        seg_token(p, g, c0 + m, tok, wt);
                        float* yp = p.y + (size_t)tok * p.H + row + rr;
                        *yp = *yp + wt * d;
                    }
                }
                it++;
            }
        }
    });
}

template <int MODE, int MAXM, int L>
cudaError_t launch_one(const GemvParams& p, const GemvConfig& c, cudaStream_t s)
{
    auto kern = gemv_kernel<MODE, MAXM, L>;
    static bool attr_set = false;   // per instantiation; the attribute is per device
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)c.smem);
    if (e != cudaSuccess) return e;
    (void)attr_set;
    kern<<<c.grid, c.consumers + 32, c.smem, s>>>(p);
    return cudaGetLastError();
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
    if (mode == 0)
        c.maxm = p.T <= 1 ? 1 : (p.T <= 2 ? 2 : (p.T <= 4 ? 4 : 2));
    else
        c.maxm = p.T <= 1 ? 1 : (p.T <= 2 ? 2 : 4);
    c.consumers = c.maxm == 4 ? 192 : 384;
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
    const uint32_t red_bytes = 2u * p.rl * nwg * kV * 4u;
    p.off_red = 512;
    const uint64_t xres = (uint64_t)p.T * p.H * 4ull;
    p.resident = (mode == 0 && xres <= 100u * 1024u) ? 1 : 0;
    p.vec_bytes = p.resident ? (uint32_t)xres : (uint32_t)c.maxm * p.K * 4u;
    const uint32_t nvec = p.resident ? 1 : 2;
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

cudaError_t gemv_launch(int mode, const GemvParams& p, const GemvConfig& c, cudaStream_t s)
{
    return mode == 0 ? launch_m<0>(p, c, s) : launch_m<1>(p, c, s);
}

}  // namespace coli
