// RMSNorm of the residual stream in front of the MoE sublayer.
//
// "Inside Kolibri 1" (flozi.net), section "The released stack": every block
// normalises with RMSNorm before and after the MoE and adds the residual
// after it. This kernel produces the layer input
//     x[t] = bf16( h[t] / sqrt(mean_j h[t][j]^2 + eps) * gamma_pre )
// one warp per token row; the lanes' partial sums of squares are reduced
// with a fixed butterfly, so the result does not depend on scheduling. The post-norm and the residual addition run inside
// the combine (combine.cu), which already holds each output row in one CTA.
#include "common.cuh"

namespace kmoe {

constexpr int kNormThreads = 256;
constexpr int kNormRowsPerCta = kNormThreads / 32;   // one warp per row
constexpr int kNormMaxVec = 24;                       // 16-byte pieces per lane: d <= 24 * 8 * 32 = 6144

// One warp per token row: the row is read once into registers (d / 256
// pieces of 8 values per lane), its sum of squares is reduced with warp
// shuffles in a fixed order, and the scaled row is written from registers.
template <int V>
__global__ void __launch_bounds__(kNormThreads)
rmsnorm_bf16_kernel(const __nv_bfloat16 *__restrict__ h, const __nv_bfloat16 *__restrict__ gamma, float eps, int N,
                    int d, __nv_bfloat16 *__restrict__ x)
{
    pdl_wait();
    pdl_trigger();
    const int lane = threadIdx.x & 31;
    const int row = blockIdx.x * kNormRowsPerCta + (threadIdx.x >> 5);
    if (row >= N) return;
    const __nv_bfloat16 *src = h + (size_t)row * d;
    uint4 raw[V];
#pragma unroll
    for (int v = 0; v < V; ++v) raw[v] = *reinterpret_cast<const uint4 *>(src + (v * 32 + lane) * 8);
    float ss = 0.f;
#pragma unroll
    for (int v = 0; v < V; ++v) {
        const uint32_t wd[4] = {raw[v].x, raw[v].y, raw[v].z, raw[v].w};
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            const float a = __uint_as_float(wd[q] << 16), b = __uint_as_float(wd[q] & 0xffff0000u);
            ss = fmaf(a, a, ss);
            ss = fmaf(b, b, ss);
        }
    }
    ss = warp_sum(ss);
    const float r = 1.f / sqrtf(ss / (float)d + eps);
    __nv_bfloat16 *out = x + (size_t)row * d;
#pragma unroll
    for (int v = 0; v < V; ++v) {
        const int c = (v * 32 + lane) * 8;
        const uint4 gr = *reinterpret_cast<const uint4 *>(gamma + c);
        const uint32_t wd[4] = {raw[v].x, raw[v].y, raw[v].z, raw[v].w};
        const uint32_t gd[4] = {gr.x, gr.y, gr.z, gr.w};
        uint32_t p[4];
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            const float a = __uint_as_float(wd[q] << 16), b = __uint_as_float(wd[q] & 0xffff0000u);
            const float ga = __uint_as_float(gd[q] << 16), gb = __uint_as_float(gd[q] & 0xffff0000u);
            const __nv_bfloat162 o = __floats2bfloat162_rn(a * r * ga, b * r * gb);
            p[q] = *reinterpret_cast<const uint32_t *>(&o);
        }
        *reinterpret_cast<uint4 *>(out + c) = make_uint4(p[0], p[1], p[2], p[3]);
    }
}

kmoe_status launch_rmsnorm(const __nv_bfloat16 *h, const __nv_bfloat16 *gamma, float eps, int N, int d,
                           __nv_bfloat16 *x, cudaStream_t st)
{
    // d / 256 pieces of 8 values per lane
    const int pieces = d / 256, grid = (N + kNormRowsPerCta - 1) / kNormRowsPerCta;
    if (d % 256)
        return fail(KMOE_ERR_UNSUPPORTED, "rmsnorm: d=%d must be a multiple of 256", d);
    if (pieces > kNormMaxVec)
        return fail(KMOE_ERR_UNSUPPORTED, "rmsnorm: d=%d must be at most %d", d, kNormMaxVec * 256);
#define KMOE_NORM(V) launch_pdl(rmsnorm_bf16_kernel<V>, grid, kNormThreads, 0, st, h, gamma, eps, N, d, x)
    switch (pieces) {
    case 1: KMOE_NORM(1); break;
    case 2: KMOE_NORM(2); break;
    case 3: KMOE_NORM(3); break;
    case 4: KMOE_NORM(4); break;
    case 5: KMOE_NORM(5); break;
    case 6: KMOE_NORM(6); break;
    case 7: KMOE_NORM(7); break;
    case 8: KMOE_NORM(8); break;
    case 9: KMOE_NORM(9); break;
    case 10: KMOE_NORM(10); break;
    case 11: KMOE_NORM(11); break;
    case 12: KMOE_NORM(12); break;
    case 13: KMOE_NORM(13); break;
    case 14: KMOE_NORM(14); break;
    case 15: KMOE_NORM(15); break;
    case 16: KMOE_NORM(16); break;
    case 17: KMOE_NORM(17); break;
    case 18: KMOE_NORM(18); break;
    case 19: KMOE_NORM(19); break;
    case 20: KMOE_NORM(20); break;
    case 21: KMOE_NORM(21); break;
    case 22: KMOE_NORM(22); break;
    case 23: KMOE_NORM(23); break;
    case 24: KMOE_NORM(24); break;
    default:                  // d == 0
        return fail(KMOE_ERR_UNSUPPORTED, "rmsnorm: d=%d must be positive", d);
    }
#undef KMOE_NORM
    return check_launch("rmsnorm");
}

}  // namespace kmoe
