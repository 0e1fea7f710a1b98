/*
 * colimoe.h -- C ABI of the routed int4 MoE layer library for NVIDIA B200 (sm_100a).
 *
 * One call processes one MoE FFN layer for a batch of T tokens in four steps, in the
 * order the colibri pages give for every token and layer:
 *   route   the router scores every routed expert and keeps the top k
 *           (colibri technical article "colibri 技术解读", section "引擎结构：一个 C 文件，
 *           五步 token 路径"; GLM-5.2 keeps 8 of 256, section "MoE 的稀疏性");
 *   union   the distinct experts selected by the batch, each listed once, so its
 *           weights are read once per batch (colibri README.zh-CN, "工作原理 / 绝不为
 *           同一次磁盘读取等待两遍", 批量并集);
 *   experts gs64 group-scaled int4 experts (colibri README.zh-CN, "开始使用 / 2. 获取
 *           模型") with gate, up and down matrices stored next to each other (same
 *           section as the union), run as SwiGLU;
 *   combine the routing-weighted sum of the selected experts plus the always-on shared
 *           expert of the dense part (colibri README.zh-CN, "核心概念").
 * The pages give no formulas; the readings used here are:
 *   logits[t][e] = float( sum_c x[t][c] * W_r[e][c] + bias[e] )  (sum in double);
 *   top-k by (logit descending, expert index ascending);
 *   w[t][s] = exp(l_s - l_max) / sum_j exp(l_j - l_max) over the k selected logits;
 *   expert(x) = D . (silu(G x) * (U x)), silu(z) = z / (1 + exp(-z));
 *   y[t] = residual[t] + shared(x[t]) + sum_s w[t][s] * expert_{idx[t][s]}(x[t]).
 *
 * Container layout of one expert ("blob"), H = hidden, I = intermediate:
 *   Gq [I][H/2] | Uq [I][H/2] | Dq [H][I/2]  -- int4, two's complement, 2 per byte,
 *                                              the lower column in the low nibble
 *   Gs [I][H/64] | Us [I][H/64] | Ds [H][I/64] -- IEEE fp16 scale per row and per 64
 *                                              consecutive input columns
 *   weight[r][c] = q[r][c] * scale[r][c / 64].  Blob size 1.59375 * H * I bytes.
 *
 * Arithmetic contracts (selected by the activation dtype, never silently):
 *   COLI_F32  decode GEMV path: weights are applied exactly (q * scale); activations
 *             (x, and h for the down projection) enter as three 8-bit digits per value
 *             relative to the largest magnitude of each 32-column unit (about 2^-17 of
 *             that magnitude), each unit's dot product is an exact integer sum, scaled
 *             and accumulated in fp32 (routing in fp64).
 *   COLI_BF16 prefill path: x is bf16; every dequantised weight is rounded to bf16
 *             (nearest-even), products accumulate in fp32 on the tensor cores, and h
 *             enters the down projection as a pair of bf16 values (hi = bf16(h),
 *             lo = bf16(h - hi), about 16 significant bits).  Routing stays fp64/fp32.
 *
 * Conventions for every entry point:
 *   - All array pointers are DEVICE pointers owned by the caller, 16-byte aligned,
 *     row-major and contiguous.  The library allocates nothing and keeps no state
 *     between calls except what lives in the caller's workspace.
 *   - `stream` is a cudaStream_t passed as void*.  Calls only enqueue work on it and
 *     return without synchronising (except coli_moe_read_status).
 *   - Argument errors found on the host return COLI_EINVAL / COLI_EUNSUPPORTED before
 *     anything is enqueued.  Launch failures return COLI_ECUDA.  Errors found on the
 *     device (non-finite logits, invalid expert ids, a bounded wait that gave up) are
 *     OR-ed into the status word of the workspace header; read it with
 *     coli_moe_read_status.  Device errors never trap, fault or hang the GPU.
 *   - Shape limits: H and I multiples of 64 and either <= 512 powers of two or
 *     multiples of 1024 (at most 6144 for 3-4 token batches, 12288 otherwise);
 *     1 <= k <= min(E, 32); E <= 1024; n_shared 0 or 1; T >= 0 (T == 0 is a no-op).
 *   - There is no CPU fallback: without a usable CUDA device every call returns
 *     COLI_ECUDA.
 */
#ifndef COLIMOE_H
#define COLIMOE_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define COLI_API __attribute__((visibility("default")))
#else
#define COLI_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    COLI_OK = 0,
    COLI_EINVAL = 1,       /* bad argument (null/misaligned pointer, bad size) */
    COLI_ENOMEM = 2,       /* workspace smaller than coli_moe_workspace_bytes() */
    COLI_ECUDA = 3,        /* CUDA runtime or launch error */
    COLI_ETIMEOUT = 4,     /* a device-side bounded wait gave up (status word) */
    COLI_EUNSUPPORTED = 5, /* valid but unsupported shape/dtype combination */
    COLI_EDEVICE = 6       /* device-side error recorded in the status word */
} coli_status;

typedef enum { COLI_F32 = 0, COLI_BF16 = 1 } coli_dtype;

/* Device status bits (coli_moe_read_status). */
#define COLI_DEV_NONFINITE 1u /* the router produced a NaN/Inf logit */
#define COLI_DEV_BAD_INDEX 2u /* union input: id outside [0,E) or repeated in a token */
#define COLI_DEV_TIMEOUT 4u   /* a pipeline wait exceeded its time budget */
#define COLI_DEV_BAD_SHAPE 8u

typedef struct {
    int32_t hidden;    /* H */
    int32_t inter;     /* I, intermediate size of every expert */
    int32_t n_experts; /* E routed experts */
    int32_t top_k;     /* k */
    int32_t n_shared;  /* 0 or 1 shared expert of the same shape */
} coli_moe_dims;

typedef struct {
    const float* w_router;    /* [E][H] fp32 router matrix */
    const float* router_bias; /* [E] fp32 or NULL */
    const uint8_t* experts;   /* E blobs, expert e at experts + e * expert_stride */
    const uint8_t* shared;    /* one blob, or NULL when n_shared == 0 */
    size_t expert_stride;     /* bytes; >= blob size and a multiple of 256 */
} coli_moe_weights;

/* Bytes of one expert blob: 1.59375 * H * I. */
COLI_API size_t coli_moe_blob_bytes(int32_t hidden, int32_t inter);

/* Workspace bytes needed for batches of up to T_max tokens.  0 on invalid dims. */
COLI_API size_t coli_moe_workspace_bytes(const coli_moe_dims* dims, int32_t T_max);

/* Zero the workspace header (status word, counters).  Required once before the first
 * use of a workspace; also clears sticky device error bits. */
COLI_API coli_status coli_moe_workspace_init(void* ws, size_t ws_bytes, void* stream);

/* Copy the device status word into *status (synchronises `stream`).  Returns COLI_OK,
 * or COLI_EDEVICE / COLI_ETIMEOUT when bits are set. */
COLI_API coli_status coli_moe_read_status(const void* ws, uint32_t* status, void* stream);

/* Route: logits [T][E] (may be NULL: kept in the workspace), idx [T][k], w [T][k].
 * x is [T][H] in `dtype`.  bias may be NULL. */
COLI_API coli_status coli_moe_route(const coli_moe_dims* dims, const float* w_router, const float* bias,
                           const void* x, coli_dtype dtype, int32_t T, int32_t* idx, float* w,
                           float* logits, void* ws, size_t ws_bytes, void* stream);

/* Route and union in one call (for T <= 8 a single launch: the router's last block
 * selects the top-k of every token and then builds the union).  Outputs as for
 * coli_moe_route followed by coli_moe_union. */
COLI_API coli_status coli_moe_route_union(const coli_moe_dims* dims, const float* w_router,
                                 const float* bias, const void* x, coli_dtype dtype, int32_t T,
                                 int32_t* idx, float* w, float* logits, int32_t* union_ids,
                                 int32_t* n_union, int32_t* offsets, int32_t* assign, void* ws,
                                 size_t ws_bytes, void* stream);

/* Union of idx [T][k]: union_ids [E] (ascending, then -1), n_union (device int32),
 * offsets [E+1] (T*k from n_union on), assign [T*k] (positions t*k+slot grouped by
 * union entry, ascending).  Ids outside [0,E) or repeated within a token set
 * COLI_DEV_BAD_INDEX. */
COLI_API coli_status coli_moe_union(const coli_moe_dims* dims, const int32_t* idx, int32_t T,
                           int32_t* union_ids, int32_t* n_union, int32_t* offsets,
                           int32_t* assign, void* ws, size_t ws_bytes, void* stream);

/* Experts + combine from a route/union result: y [T][H] fp32 = residual + shared(x) +
 * sum_s w * expert(x).  residual may be NULL (treated as 0) and may alias y. */
COLI_API coli_status coli_moe_forward(const coli_moe_dims* dims, const coli_moe_weights* weights,
                             const void* x, coli_dtype dtype, int32_t T, const int32_t* idx,
                             const float* w, const int32_t* union_ids, const int32_t* n_union,
                             const int32_t* offsets, const int32_t* assign,
                             const float* residual, float* y, void* ws, size_t ws_bytes,
                             void* stream);

/* The two halves of coli_moe_forward for the fp32 decode path, exposed separately so a
 * caller can time or schedule them:
 *   gate_up  h [(T*k + T*n_shared)][I] fp32 (held in the workspace): row p < T*k is the
 *            SwiGLU activation of union position p (the assign order), row T*k + t the
 *            shared expert's for token t;
 *   down     y = residual + combine of D . h. */
COLI_API coli_status coli_moe_gate_up(const coli_moe_dims* dims, const coli_moe_weights* weights,
                             const float* x, int32_t T, const int32_t* union_ids,
                             const int32_t* n_union, const int32_t* offsets,
                             const int32_t* assign, void* ws, size_t ws_bytes, void* stream);
COLI_API coli_status coli_moe_down(const coli_moe_dims* dims, const coli_moe_weights* weights,
                          int32_t T, const float* w, const int32_t* union_ids,
                          const int32_t* n_union, const int32_t* offsets, const int32_t* assign,
                          const float* residual, float* y, void* ws, size_t ws_bytes,
                          void* stream);

/* Whole layer: route (+ union fused into the router's last block for T <= 8) then
 * forward.  idx, w, union_ids, n_union, offsets, assign are written as by the separate
 * calls; logits may be NULL.  fp32, T <= 8: x is also turned into activation digits in a
 * launch of its own (held in the workspace), which the router launch overlaps; larger fp32
 * batches let the gate/up launch read x before the router launch has finished (x is
 * complete by then: the first launch of the call is stream-ordered after the caller's
 * earlier work). */
COLI_API coli_status coli_moe_layer(const coli_moe_dims* dims, const coli_moe_weights* weights,
                           const void* x, coli_dtype dtype, int32_t T, int32_t* idx, float* w,
                           float* logits, int32_t* union_ids, int32_t* n_union, int32_t* offsets,
                           int32_t* assign, const float* residual, float* y, void* ws,
                           size_t ws_bytes, void* stream);

/* Allocation-free variant of coli_moe_forward for the fp32 decode path.  The colibri
 * pages have no counterpart: this exists for callers that cannot allocate device memory
 * or hand over a workspace -- e.g. code running inside a host framework's enqueue
 * callback, where the framework owns all device memory and forbids new allocations, or a
 * latency-critical loop where cudaMalloc would synchronise the device.
 * Instead of a workspace it uses a fixed 4 MiB array in the library's device memory
 * (present on every GPU that loads the library until the process exits).  A batch needs
 * 256 + T * (top_k + n_shared) * inter * 4 bytes of it; larger batches return
 * COLI_ENOMEM before anything is enqueued.  Arguments and results are those of
 * coli_moe_forward with dtype COLI_F32.  Every call on a device shares the array and it
 * keeps the previous call's contents (each call clears its 256-byte header and rewrites
 * h before reading it); calls whose GPU work overlaps (e.g. on two streams) race on it,
 * so serialise them.  The first call on a device sets up the array's device address
 * (once per device, with that device current): make that first call before any stream
 * capture.  Allocates nothing: no cudaMalloc, cudaFree or allocating library call.
 * Device errors of a call (the status bits of coli_moe_read_status) are in the array's
 * header until the next call on the device clears it: read them with
 * coli_moe_noalloc_read_status before that.  A device reset (cudaDeviceReset, or a
 * destroyed and re-created primary context) is not supported: the array's address is
 * looked up once per device for the life of the process. */
COLI_API coli_status coli_moe_forward_noalloc(const coli_moe_dims* dims,
                                              const coli_moe_weights* weights, const float* x,
                                              int32_t T, const float* w, const int32_t* union_ids,
                                              const int32_t* n_union, const int32_t* offsets,
                                              const int32_t* assign, const float* residual,
                                              float* y, void* stream);

/* Status word of the last coli_moe_forward_noalloc call on the current device (the
 * allocation-free counterpart of coli_moe_read_status; synchronises `stream`, allocates
 * nothing).  Returns COLI_OK, or COLI_EDEVICE / COLI_ETIMEOUT when bits are set; COLI_ECUDA
 * if the array's address cannot be looked up. */
COLI_API coli_status coli_moe_noalloc_read_status(uint32_t* status, void* stream);

/* Other weight containers (the engine's int8 and packed int2 kernels, and the older
 * per-row int4 container; colibri README.zh-CN "开始使用 / 2. 获取模型", the technical
 * article's "精度与语义").  The blob keeps the gs64 order Gq | Uq | Dq | Gs | Us | Ds and
 * changes the payload or the scale axis:
 *   COLI_FMT_INT4_G64  int4 nibbles, fp16 scale per 64 input columns (the gs64 blob);
 *   COLI_FMT_INT8_G64  int8 two's complement, one byte per weight, gs64 fp16 scales;
 *   COLI_FMT_INT4_ROW  int4 nibbles, one fp16 scale per row;
 *   COLI_FMT_INT2_G64  int2 two's complement in [-2, 1], four per byte, lowest-index
 *                      column in the lowest bits, gs64 fp16 scales.
 * q matrices are [rows][in * b / 8] bytes; scale blocks [rows][in / 64] (or [rows]) fp16. */
#define COLI_FMT_INT4_G64 0
#define COLI_FMT_INT8_G64 1
#define COLI_FMT_INT4_ROW 2
#define COLI_FMT_INT2_G64 3

/* Bytes of one expert blob in container fmt (0 for invalid arguments). */
COLI_API size_t coli_moe_blob_bytes_fmt(int32_t hidden, int32_t inter, int32_t fmt);

/* Decode forward (fp32 activations, 1 <= T <= 4) for blobs in container fmt: arguments and
 * result as coli_moe_forward with dtype COLI_F32 (idx is not needed: the union lists and w
 * carry the routing); expert_stride >= coli_moe_blob_bytes_fmt, a multiple of 256.  Two
 * launches (gate/up + SwiGLU, then down + combine); y's sums run in one fixed order.
 * T > 4 returns COLI_EUNSUPPORTED. */
COLI_API coli_status coli_moe_forward_fmt(const coli_moe_dims* dims, int32_t fmt,
                                          const coli_moe_weights* weights, const float* x, int32_t T,
                                          const float* w, const int32_t* union_ids,
                                          const int32_t* n_union, const int32_t* offsets,
                                          const int32_t* assign, const float* residual, float* y,
                                          void* ws, size_t ws_bytes, void* stream);

/* Expert parallelism (experts split over ranks in contiguous id ranges; README.zh-CN
 * "实际成果", the technical article's "集群模式与开放问题清单"): the entries of a batch union
 * (from coli_moe_union / coli_moe_route_union over all E experts) whose experts lie in
 * [e0, e1), renumbered to e - e0: union_ids_local [e1-e0] (ascending, then -1),
 * n_union_local (device int32), offsets_local [e1-e0+1], assign_local [T*k] (positions
 * t*k+slot into the full idx / w arrays, first offsets_local[n_union_local] of them
 * valid).  Passing these lists, the rank's experts (stride as usual, expert e0 first), the
 * full w, and dims with n_experts = e1-e0 to coli_moe_forward gives the rank's share of
 * y; the shares of all ranks (the shared expert counted on one rank only) add up to y. */
COLI_API coli_status coli_moe_union_restrict(const coli_moe_dims* dims, int32_t T, int32_t e0, int32_t e1,
                                             const int32_t* union_ids, const int32_t* n_union,
                                             const int32_t* offsets, const int32_t* assign,
                                             int32_t* union_ids_local, int32_t* n_union_local,
                                             int32_t* offsets_local, int32_t* assign_local, void* stream);

/* Diagnostic: run one bounded device wait that can only run out (an mbarrier nothing
 * arrives at), with a budget of `budget_cycles` SM clock cycles (1 .. 2^32).  When the
 * budget is spent the kernel records COLI_DEV_TIMEOUT and timeout site 99 in the workspace
 * header (as every wait of the library does), writes 1 to the device int32 *returned and
 * ends; the stream and context stay usable.  For tests of the failure path. */
COLI_API coli_status coli_debug_wait_timeout(void* ws, size_t ws_bytes, uint64_t budget_cycles,
                                             int32_t* returned, void* stream);

/* Diagnostic: the phase stamps of the last fused decode launch (coli_moe_layer /
 * coli_moe_stack for 1-4 tokens), for a library built with COLI_PHASE_STAMPS
 * (`python -m int4_routed_expert_gemv_b200.build --stamps`; the phase table of
 * `python -m int4_routed_expert_gemv_b200.phases`).  Copies, for up to max_ctas CTAs,
 * *n_stamps (16) global-timer values in ns per CTA into the host array stamps
 * [max_ctas][16]: 0 kernel entry, 1 layer input loaded, 2 router partial sums published,
 * 3 input operand built, 4 routing table ready, 5 first routed gate/up stage, 6 first down
 * stage, 7 last down stage done, 8 last reduction done, 9 exit (the last layer of the
 * launch; 0 where a CTA has no such phase, and rows of all 0 beyond the launch's
 * CTAs).  Synchronises with the device.  Returns
 * COLI_EUNSUPPORTED (and *n_stamps = 0) for the regular build. */
COLI_API coli_status coli_debug_phase_stamps(uint64_t* stamps, int32_t max_ctas, int32_t* n_ctas,
                                             int32_t* n_stamps);

/* Residual stack of decode layers, every layer resident in device memory:
 *   for l in 0 .. n_layers-1:  n = RMSNorm_l(x);  x = x + MoE_l(n);   y = x at the end,
 * with RMSNorm_l(x) = x * gamma[l] / sqrt(mean(x^2) + eps) (double, rounded once to fp32)
 * and MoE_l the layer of coli_moe_layer (its shared expert included).  The residual stream
 * stays on the device from layer to layer (colibri README.zh-CN, "工作原理 / 绝不为同一次
 * 磁盘读取等待两遍", COLI_CUDA_PIPE=2): up to 16 layers run in one launch, the weights
 * of each layer streaming while the previous layer finishes.
 *   layers  host array of n_layers weight descriptors (device pointers inside);
 *   gamma   host array of n_layers device pointers to [H] fp32 RMSNorm weights, or NULL
 *           for all-ones; an individual NULL entry also means all-ones;
 *   x, y    [T][H] fp32 device arrays; y may not overlap x;
 *   idx     [n_layers][T][k] device array receiving every layer's selected experts (the
 *           fp32 contract's routing), or NULL.
 * Decode batches only: 1 <= T <= 4; otherwise (or for a shape the fused kernel does not
 * take) COLI_EUNSUPPORTED.  fp32 activations (the COLI_F32 contract, except that the
 * activations entering each layer are quantised with one scale per token). */
COLI_API coli_status coli_moe_stack(const coli_moe_dims* dims, const coli_moe_weights* layers,
                                    const float* const* gamma, int32_t n_layers, double eps,
                                    const float* x, int32_t T, int32_t* idx, float* y, void* ws,
                                    size_t ws_bytes, void* stream);

/* RMSNorm: out [T][H] = x * gamma / sqrt(mean(x^2) + eps), computed in double and
 * rounded once to fp32.  out may alias x. */
COLI_API coli_status coli_rmsnorm(int32_t hidden, int32_t T, const float* x, const float* gamma, double eps,
                         float* out, void* stream);

/* Human-readable name of a status code (static string). */
COLI_API const char* coli_status_string(coli_status s);

#ifdef __cplusplus
}
#endif

#endif /* COLIMOE_H */
