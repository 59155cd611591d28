// Router logits and bias-corrected top-K selection.
//
// "Inside Kolibri 1" (flozi.net), section "Routing: selection bias and
// mixture weights are separate": the router maps x [N, 2560] to FP32 logits
// [N, 384]; the learned correction bias is added to the logits to pick the
// top six experts; the mixture weights are sigmoid of the unbiased logits of
// those six, not renormalised.
#include "common.cuh"
#include "permute_dev.cuh"
#include "sm100.cuh"

#include <algorithm>
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
    pdl_wait();
    pdl_trigger();
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
        launch_pdl(router_logits_kernel<float>, grid, kRouterThreads, smem, st,
            static_cast<const float *>(x), w_router, N, d, E, logits);
    } else {
        cudaFuncSetAttribute(router_logits_kernel<__nv_bfloat16>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        launch_pdl(router_logits_kernel<__nv_bfloat16>, grid, kRouterThreads, smem, st,
            static_cast<const __nv_bfloat16 *>(x), w_router, N, d, E, logits);
    }
    return check_launch("router_logits");
}

// Order-preserving integer key of a finite score (-0 and +0 map to the same
// key, so they tie like equal floats do).
__device__ __forceinline__ int score_key(float s)
{
    const int b = __float_as_int(s + 0.f);
    return b < 0 ? b ^ 0x7fffffff : b;
}

// ------------------------------------------------------------------- top-K
//
// One warp per token. Lane l holds the biased scores s[e] = l[e] + b[e] of
// experts e = i*32 + l (NPL of them) in registers, as order-preserving
// integer keys. K rounds: every lane finds its best remaining candidate, the
// warp's largest key and then the lowest expert index holding it are found
// with one reduce instruction each (score descending, index ascending), and
// the owner retires it. Logits are read through L2 (they may come from other
// CTAs of the same kernel).
// Mixture weights from the unbiased logits of the K chosen experts: sigmoid
// of each ("Inside Kolibri 1", routing section) or, with KMOE_SCORE_SOFTMAX,
// a softmax over the K ("Kolibri 1 Deep Dive", routing formulation).
template <int NPL>
__device__ __forceinline__ void topk_warp(const float *lr, const float *__restrict__ bias, int E, int K, int score,
                                          int32_t *idx_row, float *w_row, int32_t *hist_row = nullptr)
{
    // Unbiased logits of the chosen experts (K <= 8). Up to 512 experts they
    // travel with their scores through the selection; beyond that lane 0
    // reads them back (registers would spill).
    constexpr bool kCarry = NPL <= 16;
    float lsel[8];
    const int lane = threadIdx.x & 31;
    int key[NPL];
    float l[kCarry ? NPL : 1];
#pragma unroll
    for (int i = 0; i < NPL; ++i) {
        const int e = i * 32 + lane;
        const float li = e < E ? __ldcg(lr + e) : 0.f;
        if (kCarry) l[i] = li;
        key[i] = e < E ? score_key(li + bias[e]) : INT_MIN;
    }
#pragma unroll
    for (int k = 0; k < 8; ++k) {
        if (k >= K) break;
        // best of this lane (ascending e: '>' keeps the lowest index on ties),
        // then the warp's largest key and the lowest expert holding it
        int bk = INT_MIN, be = INT_MAX;
        float bl = 0.f;
#pragma unroll
        for (int i = 0; i < NPL; ++i)
            if (key[i] > bk) { bk = key[i]; be = i * 32 + lane; if (kCarry) bl = l[i]; }
        const int mk = __reduce_max_sync(0xffffffffu, bk);
        const int me = __reduce_min_sync(0xffffffffu, bk == mk ? be : INT_MAX);
        const int e = me < E ? me : E - 1;     // me < E whenever K <= E and the scores are finite
        const float wl = kCarry ? __shfl_sync(0xffffffffu, bl, me & 31) : 0.f;
#pragma unroll
        for (int i = 0; i < NPL; ++i)
            if (i * 32 + lane == me) key[i] = INT_MIN;
        lsel[k] = kCarry ? wl : (lane == 0 ? __ldcg(lr + e) : 0.f);
        if (lane == 0) {
            idx_row[k] = e;
            if (hist_row) atomicAdd(hist_row + e, 1);   // integer counts: exact in any order
        }
    }
    if (lane == 0) {
        if (score == KMOE_SCORE_SOFTMAX) {
            float mx = -INFINITY, sum = 0.f;
#pragma unroll
            for (int k = 0; k < 8; ++k)
                if (k < K) mx = fmaxf(mx, lsel[k]);
#pragma unroll
            for (int k = 0; k < 8; ++k)
                if (k < K) {
                    lsel[k] = expf(lsel[k] - mx);
                    sum += lsel[k];
                }
#pragma unroll
            for (int k = 0; k < 8; ++k)
                if (k < K) w_row[k] = lsel[k] / sum;
        } else {
#pragma unroll
            for (int k = 0; k < 8; ++k)
                if (k < K) w_row[k] = sigmoidf_(lsel[k]);
        }
    }
}

template <int NPL>
__global__ void __launch_bounds__(256)
topk_kernel(const float *__restrict__ logits, const float *__restrict__ bias, int N, int E, int K, int score,
            int32_t *__restrict__ idx, float *__restrict__ wout, int32_t *__restrict__ hist)
{
    pdl_wait();
    pdl_trigger();
    const int t = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
    if (t >= N) return;
    topk_warp<NPL>(logits + (size_t)t * E, bias, E, K, score, idx + (size_t)t * K, wout + (size_t)t * K,
                   hist ? hist + (size_t)(t / kChunk) * E : nullptr);
}

kmoe_status launch_topk(const float *logits, const float *bias, int N, int E, int K, int score,
                        int32_t *idx, float *w, cudaStream_t st, int32_t *hist)
{
    const int warps = 8;
    dim3 grid((N + warps - 1) / warps);
    const int npl = (E + 31) / 32;
#define KMOE_TOPK(n) launch_pdl(topk_kernel<n>, grid, warps * 32, 0, st, logits, bias, N, E, K, score, idx, w, hist)
    if (npl <= 2) KMOE_TOPK(2);
    else if (npl <= 4) KMOE_TOPK(4);
    else if (npl <= 8) KMOE_TOPK(8);
    else if (npl <= 12) KMOE_TOPK(12);
    else if (npl <= 16) KMOE_TOPK(16);
    else KMOE_TOPK(32);
#undef KMOE_TOPK
    return check_launch("topk");
}

// ------------------------------------------------- small-batch router logits
//
// For N <= 256 tokens (decode) the logits come from 128 CTAs of 32 warps.
// Each CTA owns kRouteEPC experts: the bulk-copy engine brings their FP32
// router rows and a chunk of up to 32 token rows into shared memory. Warp w
// handles tokens 8*(w%4) .. 8*(w%4)+7 of the chunk over column part w/4 (one
// eighth of d), four columns per lane and step, so every router weight read
// from shared memory feeds eight tokens and no load has a bank conflict; the
// eight part sums of a logit are added in a fixed order. Top-K and the
// dispatch permutation follow as separate dependent launches (one warp per
// token, then one CTA), which keeps the selection off a single SM.
// The router rows are layer weights that no earlier kernel writes, so their
// copy is issued before the wait for the previous kernel; with zero_ints > 0
// CTA 0 also zeroes the call's status block (status word and the FFN's
// counters) once that kernel has finished, in place of a separate memset.
constexpr int kRouteEPC = 3;
constexpr int kRouteThreads = 1024;
constexpr int kRouteWarps = kRouteThreads / 32;
constexpr int kRouteTPW = 8;                          // tokens per warp
constexpr int kRouteTG = 4;                           // token groups per chunk
constexpr int kRouteCQ = kRouteWarps / kRouteTG;      // column parts (8)
constexpr int kRouteChunkMax = kRouteTPW * kRouteTG;  // 32 tokens per chunk
constexpr int kRouteSmemMax = 200 * 1024;
constexpr long long kRouteWaitLimit = 1LL << 32;

__device__ __forceinline__ void load4(const float *p, float (&o)[4])
{
    const float4 v = *reinterpret_cast<const float4 *>(p);
    o[0] = v.x; o[1] = v.y; o[2] = v.z; o[3] = v.w;
}
__device__ __forceinline__ void load4(const __nv_bfloat16 *p, float (&o)[4])
{
    const uint2 v = *reinterpret_cast<const uint2 *>(p);
    o[0] = __uint_as_float(v.x << 16); o[1] = __uint_as_float(v.x & 0xffff0000u);
    o[2] = __uint_as_float(v.y << 16); o[3] = __uint_as_float(v.y & 0xffff0000u);
}

template <class XT>
__global__ void __launch_bounds__(kRouteThreads, 1)
router_small_kernel(const XT *__restrict__ x, const float *__restrict__ w, int N, int d, int E, int chunk, int x_off,
                    float *__restrict__ logits, int *status, int zero_ints)
{
    using namespace sm100;
    extern __shared__ __align__(128) uint8_t sm_raw[];
    __shared__ __align__(8) uint64_t bar, wbar;
    __shared__ int abort_flag;
    __shared__ float red[kRouteCQ][kRouteChunkMax][kRouteEPC];
    float *wsm = reinterpret_cast<float *>(sm_raw);
    XT *xsm = reinterpret_cast<XT *>(sm_raw + x_off);
    const int e0 = blockIdx.x * kRouteEPC;
    const int ne = min(kRouteEPC, E - e0);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int tg = warp % kRouteTG, cq = warp / kRouteTG;
    const int qd = d / kRouteCQ;                     // columns per part (d % 128 == 0)
    if (threadIdx.x == 0) {
        mbar_init(&bar, 1);
        mbar_init(&wbar, 1);
        abort_flag = 0;
        fence_mbar_init();
        // the router rows do not come from the previous kernel: fetch them now
        const uint32_t wbytes = (uint32_t)ne * d * 4;
        mbar_arrive_expect_tx(&wbar, wbytes);
        bulk_load(wsm, w + (size_t)e0 * d, wbytes, &wbar);
    }
    __syncthreads();
    pdl_wait();
    pdl_trigger();
    if (blockIdx.x == 0)
        for (int i = threadIdx.x; i < zero_ints; i += blockDim.x) status[i] = 0;
    uint32_t phase = 0;
    bool w_ok = true;
    for (int c0 = 0; c0 < N; c0 += chunk) {
        const int nt = min(chunk, N - c0);
        if (threadIdx.x == 0) {
            fence_proxy_async();      // earlier generic reads of xsm before the async overwrite
            const uint32_t xbytes = (uint32_t)nt * d * sizeof(XT);
            mbar_arrive_expect_tx(&bar, xbytes);
            bulk_load(xsm, x + (size_t)c0 * d, xbytes, &bar);
        }
        if (c0 == 0) w_ok = mbar_wait(&wbar, 0, &abort_flag, status, kRouteWaitLimit);
        if (w_ok) mbar_wait(&bar, phase, &abort_flag, status, kRouteWaitLimit);
        phase ^= 1;
        __syncthreads();
        if (abort_flag) break;
        const int t0 = tg * kRouteTPW;
        float acc[kRouteTPW][kRouteEPC];
#pragma unroll
        for (int a = 0; a < kRouteTPW; ++a)
#pragma unroll
            for (int e = 0; e < kRouteEPC; ++e) acc[a][e] = 0.f;
        if (t0 < nt) {
            for (int j = cq * qd + lane * 4; j < (cq + 1) * qd; j += 128) {
                float wv[kRouteEPC][4];
#pragma unroll
                for (int e = 0; e < kRouteEPC; ++e) {
                    const float4 v = e < ne ? *reinterpret_cast<const float4 *>(wsm + e * d + j)
                                            : make_float4(0.f, 0.f, 0.f, 0.f);
                    wv[e][0] = v.x; wv[e][1] = v.y; wv[e][2] = v.z; wv[e][3] = v.w;
                }
#pragma unroll
                for (int a = 0; a < kRouteTPW; ++a) {
                    if (t0 + a < nt) {
                        float xv[4];
                        load4(xsm + (size_t)(t0 + a) * d + j, xv);
#pragma unroll
                        for (int e = 0; e < kRouteEPC; ++e)
#pragma unroll
                            for (int q = 0; q < 4; ++q) acc[a][e] = fmaf(xv[q], wv[e][q], acc[a][e]);
                    }
                }
            }
        }
        // Reduce the 24 partial sums across the warp in one transposing
        // butterfly (31 shuffles instead of 24 x 5): at the level with offset
        // o every lane keeps one half of its values and sends the other, so
        // lane i ends up holding the warp total of value i.
        static_assert(kRouteTPW * kRouteEPC <= 32, "one value per lane");
        float v[32];
#pragma unroll
        for (int i = 0; i < 32; ++i) v[i] = i < kRouteTPW * kRouteEPC ? acc[i / kRouteEPC][i % kRouteEPC] : 0.f;
#pragma unroll
        for (int o = 16; o >= 1; o >>= 1) {
            const bool upper = (lane & o) != 0;
#pragma unroll
            for (int j = 0; j < o; ++j) {
                const float send = upper ? v[j] : v[j + o];
                const float keep = upper ? v[j + o] : v[j];
                v[j] = keep + __shfl_xor_sync(0xffffffffu, send, o);
            }
        }
        if (lane < kRouteTPW * kRouteEPC) red[cq][t0 + lane / kRouteEPC][lane % kRouteEPC] = v[0];
        __syncthreads();
        if (threadIdx.x < nt * ne) {
            const int t = threadIdx.x / ne, e = threadIdx.x - t * ne;
            float v = red[0][t][e];
#pragma unroll
            for (int q = 1; q < kRouteCQ; ++q) v += red[q][t][e];
            logits[(size_t)(c0 + t) * E + e0 + e] = v;
        }
        __syncthreads();
    }
    if (abort_flag && threadIdx.x == 0) {   // a copy never landed: let it finish (bounded) and leave
        mbar_wait_drain(&wbar, 0, kRouteWaitLimit);
        mbar_wait_drain(&bar, phase ^ 1, kRouteWaitLimit);
    }
}


kmoe_status launch_router_small(const void *x, int x_dtype, const float *w_router, int N, int d, int E,
                                float *logits, int *status, cudaStream_t st, int zero_ints)
{
    if (N > kChunk) return fail(KMOE_ERR_UNSUPPORTED, "small-batch router: N=%d > %d", N, kChunk);
    const int xb = x_dtype == KMOE_F32 ? 4 : 2;
    const int w_bytes = ((kRouteEPC * d * 4) + 127) / 128 * 128;
    const int chunk = std::min(std::min(N, kRouteChunkMax), std::max(1, (kRouteSmemMax - w_bytes) / (d * xb)));
    const size_t smem = (size_t)w_bytes + (size_t)chunk * d * xb;
    const int grid = (E + kRouteEPC - 1) / kRouteEPC;
    if (x_dtype == KMOE_F32) {
        cudaFuncSetAttribute(router_small_kernel<float>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        launch_pdl(router_small_kernel<float>, grid, kRouteThreads, smem, st, static_cast<const float *>(x), w_router,
                   N, d, E, chunk, w_bytes, logits, status, zero_ints);
    } else {
        cudaFuncSetAttribute(router_small_kernel<__nv_bfloat16>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)smem);
        launch_pdl(router_small_kernel<__nv_bfloat16>, grid, kRouteThreads, smem, st,
                   static_cast<const __nv_bfloat16 *>(x), w_router, N, d, E, chunk, w_bytes, logits, status, zero_ints);
    }
    return check_launch("router_small");
}

}  // namespace kmoe
