// Grouped SwiGLU expert FFN, weight-streaming form (CUDA cores).
//
// "Inside Kolibri 1" (flozi.net), routing section: every routed or shared
// expert is a SwiGLU MLP, two d -> I projections combined as SiLU(gate) * up,
// then an I -> d projection, no biases. At decode a routed expert sees one or
// two tokens, so the work is a weight-bandwidth-bound GEMV: every weight is
// read from HBM exactly once and used for the few rows of its expert. The
// kernels below stream each expert's rows with 16-byte loads (FP32, BF16 or
// E4M3 + FP32 block scale) and keep the token rows in shared memory.
//
// Row space: dispatched rows 0 .. N*K-1 belong to routed experts (group e
// owns rows offsets[e] .. offsets[e+1]-1, token perm_token[row]); rows
// N*K .. N*K+N-1 belong to the shared expert (group E, token row - N*K).
// H (the SwiGLU intermediate) is [N*K + N, I] in that row space.
#include "common.cuh"

#include <algorithm>

namespace kmoe {

constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;
constexpr int kMT = 8;               // token rows per pass over the weights

__device__ __forceinline__ uint4 ld_stream(const void *p)
{
    uint4 r;
    asm volatile("ld.global.nc.L1::no_allocate.L2::256B.v4.u32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
                 : "l"(p));
    return r;
}

struct Group {
    int row0, rows;
    bool shared;
};

__device__ __forceinline__ Group group_of(int g, int N, int K, int E, const int32_t *offsets)
{
    if (g < E) return {offsets[g], offsets[g + 1] - offsets[g], false};
    return {N * K, N, true};
}

__device__ __forceinline__ int token_of(const Group &G, int row, int N, int K, const int32_t *perm)
{
    return G.shared ? row - N * K : perm[row];
}

template <class WT> struct WBytes { static constexpr int v = sizeof(WT); };

// ------------------------------------------------------------------ gate/up
template <class WT, class HT, int MT>
__device__ __forceinline__ void up_tile(const float *xs, int d, int I, const WT *wg, const WT *wu,
                                        const float *sg, const float *su, int f0, int mc,
                                        HT *H, int row0)
{
    constexpr int VEC = WVec<WT>::VEC;
    constexpr int F = 32 / VEC;                     // features per warp
    const int lane = threadIdx.x & 31;
    const int cb = d / 128;
    float ag[F][MT], au[F][MT];
#pragma unroll
    for (int f = 0; f < F; ++f)
#pragma unroll
        for (int m = 0; m < MT; ++m) ag[f][m] = au[f][m] = 0.f;

    for (int j = lane * VEC; j < d; j += 32 * VEC) {
        uint4 rg[F], ru[F];
#pragma unroll
        for (int f = 0; f < F; ++f) {
            rg[f] = ld_stream(wg + (size_t)(f0 + f) * d + j);
            ru[f] = ld_stream(wu + (size_t)(f0 + f) * d + j);
        }
#pragma unroll
        for (int f = 0; f < F; ++f) {
            float vg[VEC], vu[VEC];
            float s_g = 1.f, s_u = 1.f;
            if (sg) {
                const int sidx = ((f0 + f) / 128) * cb + j / 128;
                s_g = sg[sidx];
                s_u = su[sidx];
            }
            WVec<WT>::cvt(rg[f], vg, s_g);
            WVec<WT>::cvt(ru[f], vu, s_u);
#pragma unroll
            for (int m = 0; m < MT; ++m) {
#pragma unroll
                for (int q = 0; q < VEC; q += 4) {
                    const float4 xv = *reinterpret_cast<const float4 *>(xs + m * d + j + q);
                    ag[f][m] = fmaf(vg[q], xv.x, ag[f][m]);
                    ag[f][m] = fmaf(vg[q + 1], xv.y, ag[f][m]);
                    ag[f][m] = fmaf(vg[q + 2], xv.z, ag[f][m]);
                    ag[f][m] = fmaf(vg[q + 3], xv.w, ag[f][m]);
                    au[f][m] = fmaf(vu[q], xv.x, au[f][m]);
                    au[f][m] = fmaf(vu[q + 1], xv.y, au[f][m]);
                    au[f][m] = fmaf(vu[q + 2], xv.z, au[f][m]);
                    au[f][m] = fmaf(vu[q + 3], xv.w, au[f][m]);
                }
            }
        }
    }
#pragma unroll
    for (int f = 0; f < F; ++f)
#pragma unroll
        for (int m = 0; m < MT; ++m) {
            const float a = warp_sum(ag[f][m]);
            const float b = warp_sum(au[f][m]);
            if (lane == 0 && m < mc) store_val(H + (size_t)(row0 + m) * I + f0 + f, a * sigmoidf_(a) * b);
        }
}

template <class WT, class XT, class HT>
__global__ void __launch_bounds__(kThreads)
ffn_up_stream_kernel(const XT *__restrict__ x, int N, int d, int I, int E, int K,
                     const int32_t *__restrict__ perm, const int32_t *__restrict__ offsets,
                     ExpertPtrs routed, ExpertPtrs shared, int groups, HT *__restrict__ H)
{
    constexpr int F = 32 / WVec<WT>::VEC;
    constexpr int FS = F * kWarps;                  // features per unit
    extern __shared__ float4 smem_f4[];
    float *xs = reinterpret_cast<float *>(smem_f4); // [kMT][d]
    const int S = I / FS;
    const int warp = threadIdx.x >> 5;
    const size_t mat = (size_t)I * d;
    const int sb = (I / 128) * (d / 128);
    for (int u = blockIdx.x; u < groups * S; u += gridDim.x) {
        const int g = u / S, slice = u - (u / S) * S;
        const Group G = group_of(g, N, K, E, offsets);
        if (G.rows == 0) continue;
        const ExpertPtrs &P = G.shared ? shared : routed;
        const size_t ge = G.shared ? 0 : (size_t)g;
        const WT *wg = static_cast<const WT *>(P.wg) + ge * mat;
        const WT *wu = static_cast<const WT *>(P.wu) + ge * mat;
        const float *sg = P.sg ? P.sg + ge * sb : nullptr;
        const float *su = P.su ? P.su + ge * sb : nullptr;
        const int f0 = slice * FS + warp * F;
        for (int m0 = 0; m0 < G.rows; m0 += kMT) {
            const int mc = min(kMT, G.rows - m0);
            const int mt = mc <= 1 ? 1 : mc <= 2 ? 2 : mc <= 4 ? 4 : 8;
            __syncthreads();
            const int vpr = d / 8;
            for (int i = threadIdx.x; i < mt * vpr; i += kThreads) {
                const int m = i / vpr, c = (i - m * vpr) * 8;
                float v[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
                if (m < mc) load8(x + (size_t)token_of(G, G.row0 + m0 + m, N, K, perm) * d + c, v);
                float4 *dst = reinterpret_cast<float4 *>(xs + m * d + c);
                dst[0] = make_float4(v[0], v[1], v[2], v[3]);
                dst[1] = make_float4(v[4], v[5], v[6], v[7]);
            }
            __syncthreads();
            const int r0 = G.row0 + m0;
            switch (mt) {
            case 1: up_tile<WT, HT, 1>(xs, d, I, wg, wu, sg, su, f0, mc, H, r0); break;
            case 2: up_tile<WT, HT, 2>(xs, d, I, wg, wu, sg, su, f0, mc, H, r0); break;
            case 4: up_tile<WT, HT, 4>(xs, d, I, wg, wu, sg, su, f0, mc, H, r0); break;
            default: up_tile<WT, HT, 8>(xs, d, I, wg, wu, sg, su, f0, mc, H, r0); break;
            }
        }
    }
}

// --------------------------------------------------------------------- down
constexpr int kDownRows = 8;          // output features per warp
constexpr int kDownFS = kDownRows * kWarps;

template <class WT, class HT, int MT>
__device__ __forceinline__ void down_tile(const float *hs, int d, int I, const WT *wd, const float *sd,
                                          int j0, int mc, HT *Y)
{
    constexpr int VEC = WVec<WT>::VEC;
    const int lane = threadIdx.x & 31;
    const int ib = I / 128;
    float acc[kDownRows][MT];
#pragma unroll
    for (int r = 0; r < kDownRows; ++r)
#pragma unroll
        for (int m = 0; m < MT; ++m) acc[r][m] = 0.f;
    for (int i = lane * VEC; i < I; i += 32 * VEC) {
        uint4 raw[kDownRows];
#pragma unroll
        for (int r = 0; r < kDownRows; ++r) raw[r] = ld_stream(wd + (size_t)(j0 + r) * I + i);
#pragma unroll
        for (int r = 0; r < kDownRows; ++r) {
            float w[VEC];
            const float s = sd ? sd[((j0 + r) / 128) * ib + i / 128] : 1.f;
            WVec<WT>::cvt(raw[r], w, s);
#pragma unroll
            for (int m = 0; m < MT; ++m) {
#pragma unroll
                for (int q = 0; q < VEC; q += 4) {
                    const float4 hv = *reinterpret_cast<const float4 *>(hs + m * I + i + q);
                    acc[r][m] = fmaf(w[q], hv.x, acc[r][m]);
                    acc[r][m] = fmaf(w[q + 1], hv.y, acc[r][m]);
                    acc[r][m] = fmaf(w[q + 2], hv.z, acc[r][m]);
                    acc[r][m] = fmaf(w[q + 3], hv.w, acc[r][m]);
                }
            }
        }
    }
#pragma unroll
    for (int r = 0; r < kDownRows; ++r)
#pragma unroll
        for (int m = 0; m < MT; ++m) {
            const float v = warp_sum(acc[r][m]);
            if (lane == 0 && m < mc) store_val(Y + (size_t)m * d + j0 + r, v);
        }
}

template <class WT, class HT>
__global__ void __launch_bounds__(kThreads)
ffn_down_stream_kernel(const HT *__restrict__ H, int N, int d, int I, int E, int K,
                       const int32_t *__restrict__ offsets, ExpertPtrs routed, ExpertPtrs shared,
                       int groups, HT *__restrict__ y_perm, HT *__restrict__ y_shared)
{
    extern __shared__ float4 smem_f4[];
    float *hs = reinterpret_cast<float *>(smem_f4);  // [kMT][I]
    const int S = d / kDownFS;
    const int warp = threadIdx.x >> 5;
    const size_t mat = (size_t)I * d;
    const int sb = (I / 128) * (d / 128);
    for (int u = blockIdx.x; u < groups * S; u += gridDim.x) {
        const int g = u / S, slice = u - (u / S) * S;
        const Group G = group_of(g, N, K, E, offsets);
        if (G.rows == 0) continue;
        const ExpertPtrs &P = G.shared ? shared : routed;
        const size_t ge = G.shared ? 0 : (size_t)g;
        const WT *wd = static_cast<const WT *>(P.wd) + ge * mat;
        const float *sd = P.sd ? P.sd + ge * sb : nullptr;
        const int j0 = slice * kDownFS + warp * kDownRows;
        for (int m0 = 0; m0 < G.rows; m0 += kMT) {
            const int mc = min(kMT, G.rows - m0);
            const int mt = mc <= 1 ? 1 : mc <= 2 ? 2 : mc <= 4 ? 4 : 8;
            __syncthreads();
            for (int i = threadIdx.x; i < mt * I; i += kThreads) {
                const int m = i / I, c = i - m * I;
                hs[i] = m < mc ? to_f32(H[(size_t)(G.row0 + m0 + m) * I + c]) : 0.f;
            }
            __syncthreads();
            HT *Y = G.shared ? y_shared + (size_t)(G.row0 + m0 - N * K) * d
                             : y_perm + (size_t)(G.row0 + m0) * d;
            switch (mt) {
            case 1: down_tile<WT, HT, 1>(hs, d, I, wd, sd, j0, mc, Y); break;
            case 2: down_tile<WT, HT, 2>(hs, d, I, wd, sd, j0, mc, Y); break;
            case 4: down_tile<WT, HT, 4>(hs, d, I, wd, sd, j0, mc, Y); break;
            default: down_tile<WT, HT, 8>(hs, d, I, wd, sd, j0, mc, Y); break;
            }
        }
    }
}

// ------------------------------------------------------------------ launch
static int sm_count()
{
    static int n = 0;
    if (!n) {
        int dev = 0;
        cudaGetDevice(&dev);
        cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
        if (n <= 0) n = 148;
    }
    return n;
}

template <class WT, class XT, class HT>
static kmoe_status run_stream(const XT *x, int N, int d, int I, int E, int K, const int32_t *perm,
                              const int32_t *offsets, const ExpertPtrs &routed, const ExpertPtrs *shared,
                              HT *h, HT *y_perm, HT *y_shared, cudaStream_t st)
{
    const int groups = E + (shared ? 1 : 0);
    const ExpertPtrs sh = shared ? *shared : ExpertPtrs{};
    constexpr int FS = (32 / WVec<WT>::VEC) * kWarps;
    const int up_units = groups * (I / FS);
    const int down_units = groups * (d / kDownFS);
    const int cap = sm_count() * 4;
    const size_t up_smem = sizeof(float) * kMT * d;
    const size_t down_smem = sizeof(float) * kMT * I;
    auto upk = ffn_up_stream_kernel<WT, XT, HT>;
    auto dnk = ffn_down_stream_kernel<WT, HT>;
    cudaFuncSetAttribute(upk, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)up_smem);
    cudaFuncSetAttribute(dnk, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)down_smem);
    upk<<<std::min(up_units, cap), kThreads, up_smem, st>>>(x, N, d, I, E, K, perm, offsets, routed, sh,
                                                             groups, h);
    kmoe_status s = check_launch("ffn_up_stream");
    if (s != KMOE_OK) return s;
    dnk<<<std::min(down_units, cap), kThreads, down_smem, st>>>(h, N, d, I, E, K, offsets, routed, sh,
                                                                 groups, y_perm, y_shared);
    return check_launch("ffn_down_stream");
}

kmoe_status launch_ffn_stream(const void *x, int x_dtype, int N, int d, int I, int E, int K,
                              const int32_t *perm, const int32_t *offsets, int w_dtype,
                              const ExpertPtrs &routed, const ExpertPtrs *shared,
                              void *h, void *y_perm, void *y_shared, cudaStream_t st)
{
    using bf = __nv_bfloat16;
    if (w_dtype == KMOE_F32) {
        float *H = static_cast<float *>(h), *yp = static_cast<float *>(y_perm), *ys = static_cast<float *>(y_shared);
        if (x_dtype == KMOE_F32)
            return run_stream<float, float, float>(static_cast<const float *>(x), N, d, I, E, K, perm, offsets,
                                                   routed, shared, H, yp, ys, st);
        return run_stream<float, bf, float>(static_cast<const bf *>(x), N, d, I, E, K, perm, offsets, routed,
                                            shared, H, yp, ys, st);
    }
    bf *H = static_cast<bf *>(h), *yp = static_cast<bf *>(y_perm), *ys = static_cast<bf *>(y_shared);
    if (w_dtype == KMOE_BF16) {
        if (x_dtype == KMOE_F32)
            return run_stream<bf, float, bf>(static_cast<const float *>(x), N, d, I, E, K, perm, offsets, routed,
                                             shared, H, yp, ys, st);
        return run_stream<bf, bf, bf>(static_cast<const bf *>(x), N, d, I, E, K, perm, offsets, routed, shared,
                                      H, yp, ys, st);
    }
    using f8 = __nv_fp8_e4m3;
    if (x_dtype == KMOE_F32)
        return run_stream<f8, float, bf>(static_cast<const float *>(x), N, d, I, E, K, perm, offsets, routed,
                                         shared, H, yp, ys, st);
    return run_stream<f8, bf, bf>(static_cast<const bf *>(x), N, d, I, E, K, perm, offsets, routed, shared, H,
                                  yp, ys, st);
}

}  // namespace kmoe
