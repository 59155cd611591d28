// Weighted combine: y[t] = Y_shared[t] + sum_k g[t][k] * Y_perm[inv_pos[t][k]].
//
// "Kolibri 1 Deep Dive" (abrarakhunji.com), section 1, layer-output formula
// (its residual term lies outside this layer); "Inside Kolibri 1", routing
// section, for the always-on shared expert (weight 1 here) and the
// unnormalised sigmoid weights. A gather in fixed slot order, FP32
// accumulation, 16-byte vector loads and stores: deterministic, no atomics.
#include "common.cuh"
#include "sm100.cuh"

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
    pdl_wait();
    pdl_trigger();
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

// BF16 inputs: a persistent kernel that streams whole token rows into shared
// memory with the bulk-copy engine (K routed rows and the shared row, d * 2
// bytes each) two tokens ahead, so each SM keeps ~140 KB of reads in flight;
// the threads then form the same fixed-order FP32 sum from shared memory.
// With h_res set it finishes the sandwich block ("Inside Kolibri 1", "The
// released stack": RMSNorm after the MoE, then the residual addition):
//     y[t] = h_res[t] + m[t] / sqrt(mean_j m[t][j]^2 + eps) * g_post
// where m[t] is the combined row in FP32; its sum of squares is reduced in a
// fixed order and m is formed twice (once for the norm, once for the output)
// from the rows in shared memory.
constexpr int kBulkThreads = 320;
constexpr int kBulkStages = 2;
constexpr long long kBulkWaitLimit = 1LL << 32;

template <class YO>
__global__ void __launch_bounds__(kBulkThreads)
combine_bulk_kernel(const __nv_bfloat16 *__restrict__ y_perm, const __nv_bfloat16 *__restrict__ y_shared,
                    const float *__restrict__ w, const int32_t *__restrict__ inv, int N, int K, int d,
                    YO *y, int *err, const __nv_bfloat16 *h_res,
                    const __nv_bfloat16 *__restrict__ g_post, float eps)
{
    using namespace sm100;
    extern __shared__ __align__(128) uint8_t cb_smem[];
    __shared__ __align__(8) uint64_t full[kBulkStages];
    __shared__ int abort_flag;
    __shared__ float red[kBulkThreads / 32];
    __shared__ float post_scale;
    const int R = K + (y_shared ? 1 : 0);                 // rows per token
    const size_t row_bytes = (size_t)d * sizeof(__nv_bfloat16);
    const size_t stage_bytes = (size_t)R * row_bytes;
    if (threadIdx.x == 0) {
        for (int s = 0; s < kBulkStages; ++s) mbar_init(&full[s], 1);
        abort_flag = 0;
        fence_mbar_init();
    }
    __syncthreads();
    pdl_wait();
    pdl_trigger();
    // thread 0 issues the rows of this block's i-th token into stage i % kBulkStages
    auto issue = [&](int i) {
        const int t = blockIdx.x + i * gridDim.x;
        if (t >= N) return;
        const int s = i % kBulkStages;
        uint8_t *dst = cb_smem + (size_t)s * stage_bytes;
        mbar_arrive_expect_tx(&full[s], (uint32_t)stage_bytes);
        for (int k = 0; k < K; ++k)
            bulk_load(dst + (size_t)k * row_bytes,
                      y_perm + (size_t)checked_index(inv[(size_t)t * K + k], 0, N * K, err) * d, (uint32_t)row_bytes,
                      &full[s]);
        if (y_shared) bulk_load(dst + (size_t)K * row_bytes, y_shared + (size_t)t * d, (uint32_t)row_bytes, &full[s]);
    };
    if (threadIdx.x == 0)
        for (int i = 0; i < kBulkStages; ++i) issue(i);
    int stop = -1;                                        // the token slot at which a wait gave up
    for (int i = 0;; ++i) {
        const int t = blockIdx.x + i * gridDim.x;
        if (t >= N) break;
        const int s = i % kBulkStages;
        // every thread reaches the vote each round, so a give-up is a uniform exit
        const bool ok = mbar_wait(&full[s], (i / kBulkStages) & 1, &abort_flag, err, kBulkWaitLimit);
        if (!__syncthreads_and(ok)) {
            stop = i;
            break;
        }
        const uint8_t *rows = cb_smem + (size_t)s * stage_bytes;
        float g[8];
#pragma unroll
        for (int k = 0; k < 8; ++k) g[k] = k < K ? w[(size_t)t * K + k] : 0.f;
        auto combined = [&](int c, float (&acc)[8]) {       // m[t][c .. c+7], fixed slot order
#pragma unroll
            for (int q = 0; q < 8; ++q) acc[q] = 0.f;
            if (y_shared) load8(reinterpret_cast<const __nv_bfloat16 *>(rows + (size_t)K * row_bytes) + c, acc);
#pragma unroll
            for (int k = 0; k < 8; ++k)
                if (k < K) {
                    float v[8];
                    load8(reinterpret_cast<const __nv_bfloat16 *>(rows + (size_t)k * row_bytes) + c, v);
#pragma unroll
                    for (int q = 0; q < 8; ++q) acc[q] = fmaf(g[k], v[q], acc[q]);
                }
        };
        if (!h_res) {
            for (int c = threadIdx.x * 8; c < d; c += kBulkThreads * 8) {
                float acc[8];
                combined(c, acc);
                store8(y + (size_t)t * d + c, acc);
            }
        } else {
            float ss = 0.f;
            for (int c = threadIdx.x * 8; c < d; c += kBulkThreads * 8) {
                float acc[8];
                combined(c, acc);
#pragma unroll
                for (int q = 0; q < 8; ++q) ss = fmaf(acc[q], acc[q], ss);
            }
            ss = warp_sum(ss);
            if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = ss;
            __syncthreads();
            if (threadIdx.x == 0) {
                float tot = 0.f;
                for (int wq = 0; wq < kBulkThreads / 32; ++wq) tot += red[wq];
                post_scale = 1.f / sqrtf(tot / (float)d + eps);
            }
            __syncthreads();
            const float sc = post_scale;
            for (int c = threadIdx.x * 8; c < d; c += kBulkThreads * 8) {
                float acc[8], hv[8], gv[8];
                combined(c, acc);
                load8(h_res + (size_t)t * d + c, hv);
                load8(g_post + c, gv);
#pragma unroll
                for (int q = 0; q < 8; ++q) acc[q] = fmaf(acc[q] * sc, gv[q], hv[q]);
                store8(y + (size_t)t * d + c, acc);
            }
        }
        __syncthreads();                                  // every thread is done with stage s
        if (threadIdx.x == 0) issue(i + kBulkStages);
    }
    // A copy never landed: before the CTA exits, wait (bounded) for every
    // token slot still in flight, i.e. the ones issued as stop .. stop +
    // kBulkStages - 1, each on the phase its issue armed.
    if (stop >= 0 && threadIdx.x == 0)
        for (int j = stop; j < stop + kBulkStages; ++j)
            if (blockIdx.x + j * gridDim.x < N) mbar_wait_drain(&full[j % kBulkStages], (j / kBulkStages) & 1, kBulkWaitLimit);
}

static size_t bulk_smem(int K, int d, bool shared) { return (size_t)kBulkStages * (K + (shared ? 1 : 0)) * d * 2; }

kmoe_status launch_combine(const void *y_perm, const void *y_shared, int y_in_dtype,
                           const float *w, const int32_t *inv, int N, int K, int d, void *y,
                           int y_dtype, int *err, cudaStream_t st, const void *h_res, const void *g_post, float eps)
{
    using bf = __nv_bfloat16;
    const size_t bsm = bulk_smem(K, d, y_shared != nullptr);
    const bf *hr = static_cast<const bf *>(h_res), *gp = static_cast<const bf *>(g_post);
    if (h_res && !(y_in_dtype == KMOE_BF16 && y_dtype == KMOE_BF16 && bsm <= 100 * 1024))
        return fail(KMOE_ERR_UNSUPPORTED, "post-norm combine: BF16 rows with K + 1 rows of d in 100 KB");
    if (y_in_dtype == KMOE_BF16 && bsm <= 100 * 1024) {
        int dev = 0, sms = 148;
        cudaGetDevice(&dev);
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
        const int per_sm = (int)((220 * 1024) / bsm) < 3 ? (int)((220 * 1024) / bsm) : 3;
        const int grid = N < sms * per_sm ? N : sms * per_sm;
        const bf *yp = static_cast<const bf *>(y_perm), *ys = static_cast<const bf *>(y_shared);
        if (y_dtype == KMOE_F32) {
            cudaFuncSetAttribute(combine_bulk_kernel<float>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bsm);
            launch_pdl(combine_bulk_kernel<float>, grid, kBulkThreads, bsm, st, yp, ys, w, inv, N, K, d,
                       static_cast<float *>(y), err, hr, gp, eps);
        } else {
            cudaFuncSetAttribute(combine_bulk_kernel<bf>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bsm);
            launch_pdl(combine_bulk_kernel<bf>, grid, kBulkThreads, bsm, st, yp, ys, w, inv, N, K, d,
                       static_cast<bf *>(y), err, hr, gp, eps);
        }
        return check_launch("combine");
    }
    dim3 grid(N, (d / 8 + kCombineThreads - 1) / kCombineThreads);
#define KMOE_COMB(YI, YO)                                                                            \
    launch_pdl(combine_kernel<YI, YO>, grid, kCombineThreads, 0, st,                                 \
               static_cast<const YI *>(y_perm), static_cast<const YI *>(y_shared), w, inv, N, K, d,  \
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
