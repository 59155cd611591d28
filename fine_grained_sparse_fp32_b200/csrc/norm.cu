// RMSNorm of the residual stream in front of the MoE sublayer.
//
// "Inside Kolibri 1" (flozi.net), section "The released stack": every block
// normalises with RMSNorm before and after the MoE and adds the residual
// after it. This kernel produces the layer input
//     x[t] = bf16( h[t] / sqrt(mean_j h[t][j]^2 + eps) * gamma_pre )
// one CTA per token row; the sum of squares is reduced in a fixed order
// (warp butterflies, then the warps in index order), so the result does not
// depend on scheduling. The post-norm and the residual addition run inside
// the combine (combine.cu), which already holds each output row in one CTA.
#include "common.cuh"

namespace kmoe {

constexpr int kNormThreads = 256;

__global__ void __launch_bounds__(kNormThreads)
rmsnorm_bf16_kernel(const __nv_bfloat16 *__restrict__ h, const __nv_bfloat16 *__restrict__ gamma, float eps, int d,
                    __nv_bfloat16 *__restrict__ x)
{
    pdl_wait();
    pdl_trigger();
    __shared__ float red[kNormThreads / 32];
    __shared__ float scale;
    const __nv_bfloat16 *row = h + (size_t)blockIdx.x * d;
    float ss = 0.f;
    for (int c = threadIdx.x * 8; c < d; c += kNormThreads * 8) {
        float v[8];
        load8(row + c, v);
#pragma unroll
        for (int q = 0; q < 8; ++q) ss = fmaf(v[q], v[q], ss);
    }
    ss = warp_sum(ss);
    if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = ss;
    __syncthreads();
    if (threadIdx.x == 0) {
        float t = 0.f;
        for (int w = 0; w < kNormThreads / 32; ++w) t += red[w];
        scale = 1.f / sqrtf(t / (float)d + eps);
    }
    __syncthreads();
    const float r = scale;
    __nv_bfloat16 *out = x + (size_t)blockIdx.x * d;
    for (int c = threadIdx.x * 8; c < d; c += kNormThreads * 8) {
        float v[8], g[8];
        load8(row + c, v);
        load8(gamma + c, g);
        uint32_t p[4];
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            const __nv_bfloat162 b = __floats2bfloat162_rn(v[2 * q] * r * g[2 * q], v[2 * q + 1] * r * g[2 * q + 1]);
            p[q] = *reinterpret_cast<const uint32_t *>(&b);
        }
        *reinterpret_cast<uint4 *>(out + c) = make_uint4(p[0], p[1], p[2], p[3]);
    }
}

kmoe_status launch_rmsnorm(const __nv_bfloat16 *h, const __nv_bfloat16 *gamma, float eps, int N, int d,
                           __nv_bfloat16 *x, cudaStream_t st)
{
    launch_pdl(rmsnorm_bf16_kernel, N, kNormThreads, 0, st, h, gamma, eps, d, x);
    return check_launch("rmsnorm");
}

}  // namespace kmoe
