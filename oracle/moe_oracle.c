/*
 * moe_oracle.c -- reference ("oracle") implementation of one routed int4 MoE FFN layer.
 *
 * TEST INFRASTRUCTURE ONLY.  This file is the slow, obviously-correct CPU definition that
 * the CUDA library is checked against.  Only the test suite, the package smoke check and
 * the benchmark's CPU-baseline leg may load it.  It shares no code, header, table or
 * helper with the CUDA path, and nothing in the CUDA path calls it.
 *
 * Style: plain scalar C, one loop per mathematical sum, every sum accumulated in double
 * in ascending index order, every stored result rounded once to float.  No blocking, no
 * fusion, no reordering beyond what the definitions below state.
 *
 * What the pages fix, and what is a reading (sources are the colibri pages):
 *   - Per layer and per token the engine routes, then takes the union of the selected
 *     experts over the batch, then runs the experts ("route -> union -> ..."):
 *     colibri README.zh-CN, "工作原理 / 每个 token 的处理路径" and the technical article
 *     "colibri 技术解读", section "引擎结构：一个 C 文件，五步 token 路径".
 *   - GLM-5.2 picks 8 of 256 routed experts per layer, plus a shared expert in the dense
 *     part: "colibri 技术解读", section "MoE 的稀疏性：为什么这件事在数学上成立".
 *   - Expert weights are int4 with one scale per group of 64 (the "gs64" container):
 *     colibri README.zh-CN, "开始使用 / 2. 获取模型".
 *   - An expert has three matrices stored next to each other (gate, up, down):
 *     colibri README.zh-CN, "工作原理 / 绝不为同一次磁盘读取等待两遍".
 *   - A batch reads each distinct expert once ("批量并集", batch union): same section.
 * The pages give no formula for the score function, the expert FFN or the combine.  The
 * readings taken here are the plainest ones consistent with the above:
 *   - logits = x . W_r^T (+ optional per-expert bias), top-k by (logit desc, index asc),
 *     weights = softmax over the k selected logits (= full softmax renormalised over the
 *     selected set, since the full normaliser cancels), routed scaling factor 1.0;
 *   - expert(x) = D . (silu(G x) * (U x)) (SwiGLU), silu(z) = z / (1 + exp(-z));
 *   - y = shared(x) + sum_slot w_slot * expert_slot(x);
 *   - int4 values are two's-complement nibbles in [-8, 7], packed two per byte with the
 *     lower-index column in the low nibble; the scale is an IEEE fp16 value per row and
 *     per 64 consecutive input-dimension columns; weight = q * scale.
 *
 * Expert blob layout (one contiguous blob per expert, H = hidden, I = intermediate):
 *   Gq [I][H/2] u8 | Uq [I][H/2] u8 | Dq [H][I/2] u8 |
 *   Gs [I][H/64] fp16 | Us [I][H/64] fp16 | Ds [H][I/64] fp16
 * G and U map hidden -> intermediate (groups run along H); D maps intermediate -> hidden
 * (groups run along I).
 *
 * Precision modes of the expert FFN:
 *   mode 0 (fp32 contract): weights are q*scale exactly, activations as given, all sums
 *           in double, h kept in double, y rounded once to float.
 *   mode 1 (bf16 weights and bf16 h): every dequantised weight q*scale is rounded to
 *           bfloat16 (round-to-nearest-even) before use, and h = silu(g)*u is rounded to
 *           float and then to bfloat16 before the down projection.  Sums stay in double.
 *   mode 2 (bf16 weights, exact h): weights rounded to bfloat16 as in mode 1, h kept in
 *           double.  This is the contract of the tensor-core prefill path, which carries h
 *           into the down projection as a pair of bfloat16 values (about 16 significant
 *           bits) so that no rounding decision on h has to agree between two
 *           implementations that compute g and u in different precisions.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define ORC_OK 0
#define ORC_EINVAL 1
#define ORC_ENOMEM 2

/* ------------------------------------------------------------------------------------ */
/* Encoding                                                                              */
/* ------------------------------------------------------------------------------------ */

/* Signed int4 value of column c in a packed row (two's complement, low nibble first). */
int orc_nibble(const uint8_t *row, int64_t c)
{
    uint8_t b = row[c / 2];
    int n = (c % 2 == 0) ? (b & 0x0F) : (b >> 4);
    if (n >= 8)
        n -= 16;
    return n;
}

/* Exact value of an IEEE-754 binary16 bit pattern. */
double orc_half(uint16_t h)
{
    int sign = (h >> 15) & 1;
    int e = (h >> 10) & 0x1F;
    int m = h & 0x3FF;
    double v;
    if (e == 0)
        v = ldexp((double)m, -24);               /* subnormal: m * 2^-24 */
    else if (e == 31)
        v = (m == 0) ? INFINITY : NAN;
    else
        v = ldexp((double)(1024 + m), e - 25);   /* (1 + m/1024) * 2^(e-15) */
    return sign ? -v : v;
}

/* Round a float to the nearest bfloat16 value (ties to even), returned as a float. */
float orc_bf16_round(float v)
{
    uint32_t u;
    memcpy(&u, &v, 4);
    if ((u & 0x7F800000u) == 0x7F800000u && (u & 0x007FFFFFu) != 0)
        return v;                                /* NaN passes through */
    uint32_t lsb = (u >> 16) & 1u;
    u = u + 0x7FFFu + lsb;
    u &= 0xFFFF0000u;
    float r;
    memcpy(&r, &u, 4);
    return r;
}

static int all_finite(const float *p, int64_t n)
{
    for (int64_t i = 0; i < n; i++)
        if (!isfinite(p[i]))
            return 0;
    return 1;
}

/* ------------------------------------------------------------------------------------ */
/* Blob layout                                                                           */
/* ------------------------------------------------------------------------------------ */

int64_t orc_blob_bytes(int H, int I)
{
    int64_t h = H, i = I;
    return 3 * (h * i / 2) + 2 * (i * (h / 64) * 2) + h * (i / 64) * 2;
}

typedef struct {
    const uint8_t *gq, *uq, *dq;
    const uint16_t *gs, *us, *ds;
} orc_expert_view;

static orc_expert_view view_blob(int H, int I, const uint8_t *blob)
{
    int64_t h = H, i = I;
    orc_expert_view v;
    v.gq = blob;
    v.uq = blob + i * h / 2;
    v.dq = blob + i * h;
    const uint8_t *s = blob + 3 * (i * h / 2);
    v.gs = (const uint16_t *)s;
    v.us = (const uint16_t *)(s + i * (h / 64) * 2);
    v.ds = (const uint16_t *)(s + 2 * i * (h / 64) * 2);
    return v;
}

/* Dequantised weight (r, c) of a [rows][in_dim] matrix: q * scale, optionally bf16. */
static double weight(const uint8_t *q, const uint16_t *s, int64_t in_dim, int64_t r,
                     int64_t c, int bf16)
{
    int qv = orc_nibble(q + r * (in_dim / 2), c);
    double sc = orc_half(s[r * (in_dim / 64) + c / 64]);
    double w = (double)qv * sc;                  /* exact: 4-bit times 11-bit */
    if (bf16)
        w = (double)orc_bf16_round((float)w);    /* (float)w is exact */
    return w;
}

/* Dequantised weight of a blob matrix, exposed so tests can probe the layout:
 * which = 0 (gate, [I][H]), 1 (up, [I][H]), 2 (down, [H][I]). */
double orc_blob_weight(int H, int I, const uint8_t *blob, int which, int64_t r, int64_t c,
                       int bf16)
{
    orc_expert_view v = view_blob(H, I, blob);
    if (which == 0)
        return weight(v.gq, v.gs, H, r, c, bf16);
    if (which == 1)
        return weight(v.uq, v.us, H, r, c, bf16);
    return weight(v.dq, v.ds, I, r, c, bf16);
}

/* ------------------------------------------------------------------------------------ */
/* Expert FFN (SwiGLU)                                                                   */
/* ------------------------------------------------------------------------------------ */

static double silu(double z) { return z / (1.0 + exp(-z)); }

/* One expert on one token: out[r] = sum_i D[r][i] * h[i], h = silu(G x) * (U x).
 * h_out (optional, [I]) receives h as used by the down projection. */
int orc_expert(int H, int I, const uint8_t *blob, const float *x, int bf16, double *out,
               double *h_out)
{
    if (H <= 0 || I <= 0 || H % 64 || I % 64)
        return ORC_EINVAL;
    orc_expert_view v = view_blob(H, I, blob);
    double *h = (double *)malloc(sizeof(double) * (size_t)I);
    if (!h)
        return ORC_ENOMEM;
    for (int64_t i = 0; i < I; i++) {
        double g = 0.0, u = 0.0;
        for (int64_t c = 0; c < H; c++)
            g += weight(v.gq, v.gs, H, i, c, bf16) * (double)x[c];
        for (int64_t c = 0; c < H; c++)
            u += weight(v.uq, v.us, H, i, c, bf16) * (double)x[c];
        double hi = silu(g) * u;
        if (bf16 == 1)
            hi = (double)orc_bf16_round((float)hi);
        h[i] = hi;
        if (h_out)
            h_out[i] = hi;
    }
    for (int64_t r = 0; r < H; r++) {
        double acc = 0.0;
        for (int64_t i = 0; i < I; i++)
            acc += weight(v.dq, v.ds, I, r, i, bf16) * h[i];
        out[r] = acc;
    }
    free(h);
    return ORC_OK;
}

/* ------------------------------------------------------------------------------------ */
/* Route: logits, top-k, renormalised softmax weights                                    */
/* ------------------------------------------------------------------------------------ */

/* x [T][H], Wr [E][H], bias [E] or NULL -> logits [T][E], idx [T][k], w [T][k].
 * Returns ORC_EINVAL for bad sizes or any non-finite input. */
int orc_route(int H, int E, int k, int T, const float *x, const float *Wr, const float *bias,
              int32_t *idx, float *w, float *logits)
{
    if (H <= 0 || E <= 0 || k < 1 || k > E || T < 0)
        return ORC_EINVAL;
    if (!all_finite(x, (int64_t)T * H) || !all_finite(Wr, (int64_t)E * H) ||
        (bias && !all_finite(bias, E)))
        return ORC_EINVAL;
    unsigned char *taken = (unsigned char *)malloc((size_t)E);
    if (!taken)
        return ORC_ENOMEM;
    for (int64_t t = 0; t < T; t++) {
        const float *xt = x + t * H;
        float *lt = logits + t * E;
        for (int64_t e = 0; e < E; e++) {
            double acc = 0.0;
            for (int64_t c = 0; c < H; c++)
                acc += (double)xt[c] * (double)Wr[e * H + c];   /* each product exact */
            if (bias)
                acc += (double)bias[e];
            lt[e] = (float)acc;
        }
        /* top-k: repeatedly take the largest remaining logit; a strict '>' while scanning
         * upward keeps the lowest index among equal logits. */
        memset(taken, 0, (size_t)E);
        for (int s = 0; s < k; s++) {
            int best = -1;
            for (int e = 0; e < E; e++) {
                if (taken[e])
                    continue;
                if (best < 0 || lt[e] > lt[best])
                    best = e;
            }
            taken[best] = 1;
            idx[t * k + s] = best;
        }
        /* weights: softmax over the selected logits, shifted by their maximum */
        double m = (double)lt[idx[t * k]];
        double z = 0.0;
        for (int s = 0; s < k; s++)
            z += exp((double)lt[idx[t * k + s]] - m);
        for (int s = 0; s < k; s++)
            w[t * k + s] = (float)(exp((double)lt[idx[t * k + s]] - m) / z);
    }
    free(taken);
    return ORC_OK;
}

/* ------------------------------------------------------------------------------------ */
/* Union: distinct experts of the batch, their token lists                               */
/* ------------------------------------------------------------------------------------ */

/* idx [T][k] -> union_ids [E] (ascending distinct ids, then -1), n_union,
 * offsets [E+1] (offsets[u] = start of union entry u in assign; T*k from n_union on),
 * assign [T*k] (for each union entry in order, the flat positions t*k+slot that chose
 * it, ascending).  Returns ORC_EINVAL for an id outside [0,E) or a repeated id within
 * one token. */
int orc_union(int E, int k, int T, const int32_t *idx, int32_t *union_ids, int32_t *n_union,
              int32_t *offsets, int32_t *assign)
{
    if (E <= 0 || k < 1 || k > E || T < 0)
        return ORC_EINVAL;
    int64_t n = (int64_t)T * k;
    for (int64_t t = 0; t < T; t++)
        for (int s = 0; s < k; s++) {
            int32_t e = idx[t * k + s];
            if (e < 0 || e >= E)
                return ORC_EINVAL;
            for (int s2 = 0; s2 < s; s2++)
                if (idx[t * k + s2] == e)
                    return ORC_EINVAL;
        }
    int64_t *count = (int64_t *)calloc((size_t)E, sizeof(int64_t));
    if (!count)
        return ORC_ENOMEM;
    for (int64_t a = 0; a < n; a++)
        count[idx[a]]++;
    int32_t nu = 0;
    for (int e = 0; e < E; e++)
        if (count[e] > 0)
            union_ids[nu++] = e;
    for (int u = nu; u < E; u++)
        union_ids[u] = -1;
    *n_union = nu;
    int64_t run = 0;
    for (int u = 0; u < nu; u++) {
        offsets[u] = (int32_t)run;
        run += count[union_ids[u]];
    }
    for (int u = nu; u <= E; u++)
        offsets[u] = (int32_t)n;
    int64_t p = 0;
    for (int u = 0; u < nu; u++)
        for (int64_t a = 0; a < n; a++)
            if (idx[a] == union_ids[u])
                assign[p++] = (int32_t)a;
    free(count);
    return ORC_OK;
}

/* ------------------------------------------------------------------------------------ */
/* Forward: shared expert + routing-weighted routed experts                              */
/* ------------------------------------------------------------------------------------ */

/* y[t] = shared(x[t]) + sum_slot w[t][slot] * expert_{idx[t][slot]}(x[t]), in double,
 * rounded once to float.  experts: E blobs at `stride` bytes apart; shared: NULL when
 * n_shared == 0. */
int orc_forward(int H, int I, int E, int k, int n_shared, int T, const float *x,
                const uint8_t *experts, int64_t stride, const uint8_t *shared,
                const int32_t *idx, const float *w, int bf16, float *y)
{
    if (H <= 0 || I <= 0 || H % 64 || I % 64 || E <= 0 || k < 1 || k > E || T < 0 ||
        (n_shared != 0 && n_shared != 1) || (n_shared == 1 && !shared))
        return ORC_EINVAL;
    double *acc = (double *)malloc(sizeof(double) * (size_t)H);
    double *ye = (double *)malloc(sizeof(double) * (size_t)H);
    if (!acc || !ye) {
        free(acc);
        free(ye);
        return ORC_ENOMEM;
    }
    int rc = ORC_OK;
    for (int64_t t = 0; t < T && rc == ORC_OK; t++) {
        const float *xt = x + t * H;
        for (int64_t r = 0; r < H; r++)
            acc[r] = 0.0;
        if (n_shared) {
            rc = orc_expert(H, I, shared, xt, bf16, ye, NULL);
            for (int64_t r = 0; r < H && rc == ORC_OK; r++)
                acc[r] += ye[r];
        }
        for (int s = 0; s < k && rc == ORC_OK; s++) {
            int32_t e = idx[t * k + s];
            if (e < 0 || e >= E) {
                rc = ORC_EINVAL;
                break;
            }
            rc = orc_expert(H, I, experts + (int64_t)e * stride, xt, bf16, ye, NULL);
            for (int64_t r = 0; r < H && rc == ORC_OK; r++)
                acc[r] += (double)w[t * k + s] * ye[r];
        }
        for (int64_t r = 0; r < H; r++)
            y[t * H + r] = (float)acc[r];
    }
    free(acc);
    free(ye);
    return rc;
}

/* ------------------------------------------------------------------------------------ */
/* RMSNorm (layer stack)                                                                 */
/* ------------------------------------------------------------------------------------ */

/* out[t] = x[t] * gamma / sqrt(mean(x[t]^2) + eps), in double, rounded once to float. */
int orc_rmsnorm(int H, int T, const float *x, const float *gamma, double eps, float *out)
{
    if (H <= 0 || T < 0 || !(eps >= 0.0))
        return ORC_EINVAL;
    for (int64_t t = 0; t < T; t++) {
        double ss = 0.0;
        for (int64_t c = 0; c < H; c++)
            ss += (double)x[t * H + c] * (double)x[t * H + c];
        double r = 1.0 / sqrt(ss / (double)H + eps);
        for (int64_t c = 0; c < H; c++)
            out[t * H + c] = (float)((double)x[t * H + c] * r * (double)gamma[c]);
    }
    return ORC_OK;
}

/* ------------------------------------------------------------------------------------ */
/* Other weight containers                                                               */
/* ------------------------------------------------------------------------------------ */
/* The engine's kernels also come in int8 and packed int2 forms, and the older per-row
 * int4 container predates gs64 (colibri README.zh-CN, "开始使用 / 2. 获取模型"; the
 * technical article's "精度与语义" section; the nxmr essay on the hand-written quantised
 * kernels).  The pages fix no layout for these.  The readings taken here keep the gs64
 * blob's order of matrices and change only the payload and the scale axis:
 *   fmt 0  int4, one fp16 scale per 64 input columns (the gs64 container above);
 *   fmt 1  int8 two's complement [-128, 127], one byte per weight, gs64 fp16 scales;
 *   fmt 2  int4 nibbles as in fmt 0, one fp16 scale per row ("per-row");
 *   fmt 3  int2 two's complement [-2, 1], four per byte with the lowest-index column in
 *          the lowest two bits, gs64 fp16 scales.
 * Blob: Gq [I][H*b/8] | Uq [I][H*b/8] | Dq [H][I*b/8] | Gs | Us | Ds, b the payload bits;
 * the scale blocks are [rows][in/64] fp16 (fmt 0, 1, 3) or [rows] fp16 (fmt 2).
 * Only the fp32 contract (mode 0) is defined for them. */

/* Signed 2-bit value of column c in a packed row (two's complement, lowest bits first). */
int orc_crumb(const uint8_t *row, int64_t c)
{
    int v = (row[c >> 2] >> (2 * (int)(c & 3))) & 3;
    return v >= 2 ? v - 4 : v;
}

/* Signed 8-bit value of column c. */
int orc_int8(const uint8_t *row, int64_t c)
{
    int v = row[c];
    return v >= 128 ? v - 256 : v;
}

static int fmt_bits(int fmt) { return fmt == 1 ? 8 : fmt == 3 ? 2 : 4; }
static int fmt_valid(int fmt) { return fmt >= 0 && fmt <= 3; }
/* fp16 scales per row of a matrix with `in_dim` input columns */
static int64_t fmt_scales_per_row(int fmt, int64_t in_dim) { return fmt == 2 ? 1 : in_dim / 64; }

int64_t orc_blob_bytes_fmt(int H, int I, int fmt)
{
    if (!fmt_valid(fmt))
        return -1;
    int64_t h = H, i = I, b = fmt_bits(fmt);
    int64_t payload = 3 * (h * i * b / 8);
    int64_t scales = 2 * i * fmt_scales_per_row(fmt, h) * 2 + h * fmt_scales_per_row(fmt, i) * 2;
    return payload + scales;
}

typedef struct {
    const uint8_t *gq, *uq, *dq;
    const uint16_t *gs, *us, *ds;
} orc_fmt_view;

static orc_fmt_view view_blob_fmt(int H, int I, int fmt, const uint8_t *blob)
{
    int64_t h = H, i = I, b = fmt_bits(fmt);
    orc_fmt_view v;
    v.gq = blob;
    v.uq = blob + i * h * b / 8;
    v.dq = blob + 2 * (i * h * b / 8);
    const uint8_t *s = blob + 3 * (i * h * b / 8);
    v.gs = (const uint16_t *)s;
    v.us = (const uint16_t *)(s + i * fmt_scales_per_row(fmt, h) * 2);
    v.ds = (const uint16_t *)(s + 2 * i * fmt_scales_per_row(fmt, h) * 2);
    return v;
}

/* Dequantised weight (r, c) of a [rows][in_dim] matrix in container fmt: q * scale. */
static double weight_fmt(int fmt, const uint8_t *q, const uint16_t *s, int64_t in_dim, int64_t r,
                         int64_t c)
{
    int64_t row_bytes = in_dim * fmt_bits(fmt) / 8;
    const uint8_t *row = q + r * row_bytes;
    int qv = fmt == 1 ? orc_int8(row, c) : fmt == 3 ? orc_crumb(row, c) : orc_nibble(row, c);
    double sc = fmt == 2 ? orc_half(s[r]) : orc_half(s[r * (in_dim / 64) + c / 64]);
    return (double)qv * sc;   /* exact: at most 8 bits times 11 bits */
}

double orc_blob_weight_fmt(int H, int I, int fmt, const uint8_t *blob, int which, int64_t r, int64_t c)
{
    orc_fmt_view v = view_blob_fmt(H, I, fmt, blob);
    if (which == 0)
        return weight_fmt(fmt, v.gq, v.gs, H, r, c);
    if (which == 1)
        return weight_fmt(fmt, v.uq, v.us, H, r, c);
    return weight_fmt(fmt, v.dq, v.ds, I, r, c);
}

/* One expert on one token in container fmt (fp32 contract): as orc_expert. */
int orc_expert_fmt(int H, int I, int fmt, const uint8_t *blob, const float *x, double *out)
{
    if (H <= 0 || I <= 0 || H % 64 || I % 64 || !fmt_valid(fmt))
        return ORC_EINVAL;
    orc_fmt_view v = view_blob_fmt(H, I, fmt, blob);
    double *h = (double *)malloc(sizeof(double) * (size_t)I);
    if (!h)
        return ORC_ENOMEM;
    for (int64_t i = 0; i < I; i++) {
        double g = 0.0, u = 0.0;
        for (int64_t c = 0; c < H; c++)
            g += weight_fmt(fmt, v.gq, v.gs, H, i, c) * (double)x[c];
        for (int64_t c = 0; c < H; c++)
            u += weight_fmt(fmt, v.uq, v.us, H, i, c) * (double)x[c];
        h[i] = silu(g) * u;
    }
    for (int64_t r = 0; r < H; r++) {
        double acc = 0.0;
        for (int64_t i = 0; i < I; i++)
            acc += weight_fmt(fmt, v.dq, v.ds, I, r, i) * h[i];
        out[r] = acc;
    }
    free(h);
    return ORC_OK;
}

/* The layer of orc_forward (fp32 contract) with every blob in container fmt. */
int orc_forward_fmt(int H, int I, int E, int k, int n_shared, int T, int fmt, const float *x,
                    const uint8_t *experts, int64_t stride, const uint8_t *shared,
                    const int32_t *idx, const float *w, float *y)
{
    if (H <= 0 || I <= 0 || H % 64 || I % 64 || E <= 0 || k < 1 || k > E || T < 0 ||
        (n_shared != 0 && n_shared != 1) || (n_shared == 1 && !shared) || !fmt_valid(fmt))
        return ORC_EINVAL;
    double *acc = (double *)malloc(sizeof(double) * (size_t)H);
    double *ye = (double *)malloc(sizeof(double) * (size_t)H);
    if (!acc || !ye) {
        free(acc);
        free(ye);
        return ORC_ENOMEM;
    }
    int rc = ORC_OK;
    for (int64_t t = 0; t < T && rc == ORC_OK; t++) {
        const float *xt = x + t * H;
        for (int64_t r = 0; r < H; r++)
            acc[r] = 0.0;
        if (n_shared) {
            rc = orc_expert_fmt(H, I, fmt, shared, xt, ye);
            for (int64_t r = 0; r < H && rc == ORC_OK; r++)
                acc[r] += ye[r];
        }
        for (int s = 0; s < k && rc == ORC_OK; s++) {
            int32_t e = idx[t * k + s];
            if (e < 0 || e >= E) {
                rc = ORC_EINVAL;
                break;
            }
            rc = orc_expert_fmt(H, I, fmt, experts + (int64_t)e * stride, xt, ye);
            for (int64_t r = 0; r < H && rc == ORC_OK; r++)
                acc[r] += (double)w[t * k + s] * ye[r];
        }
        for (int64_t r = 0; r < H; r++)
            y[t * H + r] = (float)acc[r];
    }
    free(acc);
    free(ye);
    return rc;
}
