// RMSNorm for the residual layer stack: out = x * gamma / sqrt(mean(x^2) + eps).
//
// The resident GPU pipeline keeps the residual stream on the device from layer to layer
// (colibri README.zh-CN, "工作原理 / 绝不为同一次磁盘读取等待两遍", COLI_CUDA_PIPE=2).
// The normalised activations feed the router, whose top-k is decided on floats, so the
// sum of squares and the scaling are done in double and rounded once to float, like the
// router's own logits.
#include "common.cuh"
#include "rmsnorm.cuh"

namespace coli {
namespace {

__global__ void __launch_bounds__(256) rmsnorm_kernel(int H, const float* __restrict__ x,
                                                      const float* __restrict__ gamma, double eps,
                                                      float* __restrict__ out)
{
    __shared__ double part[8];
    const int t = blockIdx.x;
    const float* xt = x + (size_t)t * H;
    double ss = 0.0;
    for (int c = threadIdx.x; c < H; c += 256) {
        const double v = xt[c];
        ss = fma(v, v, ss);
    }
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
    if ((threadIdx.x & 31) == 0) part[threadIdx.x >> 5] = ss;
    __syncthreads();
    double tot = 0.0;
#pragma unroll
    for (int w = 0; w < 8; w++) tot += part[w];
    const double r = 1.0 / sqrt(tot / (double)H + eps);
    for (int c = threadIdx.x; c < H; c += 256)
        out[(size_t)t * H + c] = (float)((double)xt[c] * r * (double)gamma[c]);
}

}  // namespace

cudaError_t rmsnorm_launch(int H, int T, const float* x, const float* gamma, double eps, float* out,
                           cudaStream_t s)
{
    rmsnorm_kernel<<<T, 256, 0, s>>>(H, x, gamma, eps, out);
    return cudaGetLastError();
}

}  // namespace coli
