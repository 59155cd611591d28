// Weighted combine: y[t] = Y_shared[t] + sum_k g[t][k] * Y_perm[inv_pos[t][k]].
//
// "Kolibri 1 Deep Dive" (abrarakhunji.com), section 1, layer-output formula
// (its residual term lies outside this layer); "Inside Kolibri 1", routing
// section, for the always-on shared expert (weight 1 here) and the
// unnormalised sigmoid weights. A gather in fixed slot order, FP32
// accumulation, 16-byte vector loads and stores: deterministic, no atomics.
#include "common.cuh"

namespace kmoe {

template <class YT>
__device__ __forceinline__ void load_vec8(const YT *p, float *o) { load8(p, o); }

__device__ __forceinline__ void store8(float *p, const float *v)
{
    reinterpret_cast<float4 *>(p)[0] = make_float4(v[0], v[1], v[2], v[3]);
    reinterpret_cast<float4 *>(p)[1] = make_float4(v[4], v[5], v[6], v[7]);
}

__device__ __forceinline__ void store8(__nv_bfloat16 *p, const float *v)
{
    uint4 r;
    __nv_bfloat162 a = __floats2bfloat162_rn(v[0], v[1]);
    __nv_bfloat162 b = __floats2bfloat162_rn(v[2], v[3]);
    __nv_bfloat162 c = __floats2bfloat162_rn(v[4], v[5]);
    __nv_bfloat162 e = __floats2bfloat162_rn(v[6], v[7]);
    r.x = *reinterpret_cast<uint32_t *>(&a);
    r.y = *reinterpret_cast<uint32_t *>(&b);
    r.z = *reinterpret_cast<uint32_t *>(&c);
    r.w = *reinterpret_cast<uint32_t *>(&e);
    *reinterpret_cast<uint4 *>(p) = r;
}

constexpr int kCombineThreads = 128;

// grid: (N, ceil(d / 8 / threads)); thread = 8 consecutive columns of a token.
template <class YI, class YO>
__global__ void __launch_bounds__(kCombineThreads)
combine_kernel(const YI *__restrict__ y_perm, const YI *__restrict__ y_shared,
               const float *__restrict__ w, const int32_t *__restrict__ inv, int N, int K, int d,
               YO *__restrict__ y)
{
    const int t = blockIdx.x;
    const int c = (blockIdx.y * kCombineThreads + threadIdx.x) * 8;
    if (c >= d) return;
    // all K + 1 row loads are issued before the first FMA (K <= 8)
    float g[8], v[8][8];
    int p[8];
#pragma unroll
    for (int k = 0; k < 8; ++k)
        if (k < K) {
            g[k] = w[(size_t)t * K + k];
            p[k] = inv[(size_t)t * K + k];
        }
#pragma unroll
    for (int k = 0; k < 8; ++k)
        if (k < K) load_vec8(y_perm + (size_t)p[k] * d + c, v[k]);
    float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
    if (y_shared) load_vec8(y_shared + (size_t)t * d + c, acc);
#pragma unroll
    for (int k = 0; k < 8; ++k)
        if (k < K) {
#pragma unroll
            for (int q = 0; q < 8; ++q) acc[q] = fmaf(g[k], v[k][q], acc[q]);
        }
    store8(y + (size_t)t * d + c, acc);
}

kmoe_status launch_combine(const void *y_perm, const void *y_shared, int y_in_dtype,
                           const float *w, const int32_t *inv, int N, int K, int d, void *y,
                           int y_dtype, cudaStream_t st)
{
    using bf = __nv_bfloat16;
    dim3 grid(N, (d / 8 + kCombineThreads - 1) / kCombineThreads);
#define KMOE_COMB(YI, YO)                                                                            \
    combine_kernel<YI, YO><<<grid, kCombineThreads, 0, st>>>(                                        \
        static_cast<const YI *>(y_perm), static_cast<const YI *>(y_shared), w, inv, N, K, d,          \
        static_cast<YO *>(y))
    if (y_in_dtype == KMOE_F32) {
        if (y_dtype == KMOE_F32) KMOE_COMB(float, float);
        else KMOE_COMB(float, bf);
    } else {
        if (y_dtype == KMOE_F32) KMOE_COMB(bf, float);
        else KMOE_COMB(bf, bf);
    }
#undef KMOE_COMB
    return check_launch("combine");
}

}  // namespace kmoe
