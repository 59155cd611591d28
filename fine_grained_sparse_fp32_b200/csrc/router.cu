// Router logits and bias-corrected top-K selection.
//
// "Inside Kolibri 1" (flozi.net), section "Routing: selection bias and
// mixture weights are separate": the router maps x [N, 2560] to FP32 logits
// [N, 384]; the learned correction bias is added to the logits to pick the
// top six experts; the mixture weights are sigmoid of the unbiased logits of
// those six, not renormalised.
#include "common.cuh"

#include <cfloat>
#include <climits>

namespace kmoe {

// ------------------------------------------------------------------ logits
//
// One CTA owns EPC experts, keeps their FP32 router rows in shared memory and
// walks a strip of tokens, one warp per token: lanes stride over d in steps
// of 8 columns, every x element is read once per CTA and every router weight
// once per CTA from HBM, the dot products end in a warp reduction.
constexpr int kRouterEPC = 4;        // experts per CTA
constexpr int kRouterTPC = 64;       // tokens per CTA
constexpr int kRouterThreads = 256;

template <class XT>
__global__ void __launch_bounds__(kRouterThreads)
router_logits_kernel(const XT *__restrict__ x, const float *__restrict__ w, int N, int d, int E,
                     float *__restrict__ logits)
{
    extern __shared__ float4 smem_f4[];
    float *wsm = reinterpret_cast<float *>(smem_f4);   // [EPC][d]
    const int e0 = blockIdx.x * kRouterEPC;
    const int ne = min(kRouterEPC, E - e0);
    for (int i = threadIdx.x * 4; i < kRouterEPC * d; i += blockDim.x * 4) {
        const int e = i / d;
        float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
        if (e < ne) v = *reinterpret_cast<const float4 *>(w + (size_t)(e0 + e) * d + (i - e * d));
        *reinterpret_cast<float4 *>(wsm + i) = v;
    }
    __syncthreads();

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int t_end = min(N, (int)(blockIdx.y + 1) * kRouterTPC);
    for (int t = blockIdx.y * kRouterTPC + warp; t < t_end; t += kRouterThreads / 32) {
        float acc[kRouterEPC];
#pragma unroll
        for (int e = 0; e < kRouterEPC; ++e) acc[e] = 0.f;
        const XT *xr = x + (size_t)t * d;
        for (int j = lane * 8; j < d; j += 256) {
            float xv[8];
            load8(xr + j, xv);
#pragma unroll
            for (int e = 0; e < kRouterEPC; ++e) {
                float wv[8];
                load8(wsm + e * d + j, wv);
#pragma unroll
                for (int q = 0; q < 8; ++q) acc[e] = fmaf(xv[q], wv[q], acc[e]);
            }
        }
#pragma unroll
        for (int e = 0; e < kRouterEPC; ++e) {
            float s = warp_sum(acc[e]);
            if (lane == 0 && e < ne) logits[(size_t)t * E + e0 + e] = s;
        }
    }
}

kmoe_status launch_router_logits(const void *x, int x_dtype, const float *w_router, int N, int d,
                                 int E, float *logits, cudaStream_t st)
{
    dim3 grid((E + kRouterEPC - 1) / kRouterEPC, (N + kRouterTPC - 1) / kRouterTPC);
    size_t smem = sizeof(float) * kRouterEPC * d;
    if (x_dtype == KMOE_F32) {
        cudaFuncSetAttribute(router_logits_kernel<float>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        router_logits_kernel<float><<<grid, kRouterThreads, smem, st>>>(
            static_cast<const float *>(x), w_router, N, d, E, logits);
    } else {
        cudaFuncSetAttribute(router_logits_kernel<__nv_bfloat16>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        router_logits_kernel<__nv_bfloat16><<<grid, kRouterThreads, smem, st>>>(
            static_cast<const __nv_bfloat16 *>(x), w_router, N, d, E, logits);
    }
    return check_launch("router_logits");
}

// ------------------------------------------------------------------- top-K
//
// One warp per token. Lane l holds the biased scores s[e] = l[e] + b[e] of
// experts e = i*32 + l (NPL of them) in registers. K rounds: every lane finds
// its best remaining candidate, a butterfly reduction picks the warp's best
// by (score descending, index ascending), and its owner retires it.
template <int NPL>
__global__ void __launch_bounds__(256)
topk_kernel(const float *__restrict__ logits, const float *__restrict__ bias, int N, int E, int K,
            int32_t *__restrict__ idx, float *__restrict__ wout)
{
    const int lane = threadIdx.x & 31;
    const int t = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
    if (t >= N) return;
    const float *lr = logits + (size_t)t * E;
    float s[NPL];
#pragma unroll
    for (int i = 0; i < NPL; ++i) {
        const int e = i * 32 + lane;
        s[i] = e < E ? lr[e] + bias[e] : -FLT_MAX;
    }
    for (int k = 0; k < K; ++k) {
        float bv = -INFINITY;
        int be = INT_MAX;
#pragma unroll
        for (int i = 0; i < NPL; ++i)        // ascending e inside a lane: '>' keeps the lowest
            if (s[i] > bv) { bv = s[i]; be = i * 32 + lane; }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
            const float ov = __shfl_xor_sync(0xffffffffu, bv, o);
            const int oe = __shfl_xor_sync(0xffffffffu, be, o);
            if (ov > bv || (ov == bv && oe < be)) { bv = ov; be = oe; }
        }
#pragma unroll
        for (int i = 0; i < NPL; ++i)
            if (i * 32 + lane == be) s[i] = -INFINITY;
        if (lane == 0) {   // be < E whenever K <= E and the scores are finite
            const int e = be < E ? be : E - 1;
            idx[(size_t)t * K + k] = e;
            wout[(size_t)t * K + k] = sigmoidf_(lr[e]);
        }
    }
}

kmoe_status launch_topk(const float *logits, const float *bias, int N, int E, int K,
                        int32_t *idx, float *w, cudaStream_t st)
{
    const int warps = 8;
    dim3 grid((N + warps - 1) / warps);
    const int npl = (E + 31) / 32;
#define KMOE_TOPK(n) topk_kernel<n><<<grid, warps * 32, 0, st>>>(logits, bias, N, E, K, idx, w)
    if (npl <= 2) KMOE_TOPK(2);
    else if (npl <= 4) KMOE_TOPK(4);
    else if (npl <= 8) KMOE_TOPK(8);
    else if (npl <= 12) KMOE_TOPK(12);
    else if (npl <= 16) KMOE_TOPK(16);
    else KMOE_TOPK(32);
#undef KMOE_TOPK
    return check_launch("topk");
}

}  // namespace kmoe
