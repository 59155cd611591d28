// Grouped SwiGLU expert FFN, weight-streaming form (CUDA cores).
//
// "Inside Kolibri 1" (flozi.net), routing section: every routed or shared
// expert is a SwiGLU MLP, two d -> I projections combined as SiLU(gate) * up,
// then an I -> d projection, no biases. At decode a routed expert sees one or
// two tokens, so the work is a weight-bandwidth-bound GEMV: every weight is
// read from HBM once and used for the few rows of its expert. Tensor cores
// would not help here; what matters is keeping enough bytes in flight.
//
// Row space: dispatched rows 0 .. N*K-1 belong to routed experts (group e
// owns rows offsets[e] .. offsets[e+1]-1, token perm_token[row]); rows
// N*K .. N*K+N-1 belong to the shared expert (group E, token row - N*K).
// H (the SwiGLU intermediate) is [N*K + N, I] in that row space.
//
// Work decomposition: a unit is (expert, chunk of up to MT rows, slice of
// output features). Every CTA builds the same prefix over the non-empty
// experts in shared memory and takes units round-robin from that compacted
// list, so active work is spread evenly over the grid whatever the routing.
// Units of one (expert, slice) with several row chunks are adjacent, so
// their repeated weight reads are served by L2. Each lane streams 16-byte
// vectors (FP32, BF16, or E4M3 with its FP32 block scale) with two column
// blocks in flight, token rows sit in shared memory as FP32, and dot
// products end in warp reductions.
#include "common.cuh"

#include <algorithm>

namespace kmoe {

constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;
constexpr int kMaxGroupsS = 1025;

__device__ __forceinline__ uint4 ld_stream(const void *p)
{
    uint4 r;
    asm volatile("ld.global.nc.L1::no_allocate.L2::256B.v4.u32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
                 : "l"(p));
    return r;
}

// Groups are visited in the order [shared, 0, 1, ..., E-1].
struct GroupView {
    int g, row0, rows;
    bool shared;
};

__device__ __forceinline__ GroupView group_at(int ord, int N, int K, int E, bool has_shared,
                                              const int32_t *offsets)
{
    if (has_shared && ord == 0) return {E, N * K, N, true};
    const int g = ord - (has_shared ? 1 : 0);
    return {g, offsets[g], offsets[g + 1] - offsets[g], false};
}

// unit prefix over groups: pre[o] = sum over earlier groups of chunks * S.
template <int MT>
__device__ void build_unit_prefix(int *pre, int n_ord, int S, int N, int K, int E, bool has_shared,
                                  const int32_t *offsets)
{
    if (threadIdx.x >= 32) return;
    const int lane = threadIdx.x;
    const int per = (n_ord + 31) / 32;
    const int o0 = lane * per;
    int sum = 0;
    for (int i = 0; i < per; ++i) {
        const int o = o0 + i;
        if (o < n_ord) sum += (group_at(o, N, K, E, has_shared, offsets).rows + MT - 1) / MT * S;
    }
    int incl = sum;
#pragma unroll
    for (int s = 1; s < 32; s <<= 1) {
        const int v = __shfl_up_sync(0xffffffffu, incl, s);
        if (lane >= s) incl += v;
    }
    int run = incl - sum;
    for (int i = 0; i < per; ++i) {
        const int o = o0 + i;
        if (o < n_ord) {
            pre[o] = run;
            run += (group_at(o, N, K, E, has_shared, offsets).rows + MT - 1) / MT * S;
        }
    }
    if (lane == 31) pre[n_ord] = incl;
}

struct Unit {
    GroupView G;
    int m0, mc, slice;
};

template <int MT>
__device__ __forceinline__ Unit decode_unit(int u, const int *pre, int n_ord, int S, int N, int K, int E,
                                            bool has_shared, const int32_t *offsets)
{
    int lo = 1, hi = n_ord;      // smallest j with pre[j] > u
    while (lo < hi) {
        const int mid = (lo + hi) >> 1;
        if (pre[mid] > u) hi = mid;
        else lo = mid + 1;
    }
    Unit U;
    U.G = group_at(lo - 1, N, K, E, has_shared, offsets);
    const int chunks = (U.G.rows + MT - 1) / MT;
    const int local = u - pre[lo - 1];
    U.slice = local / chunks;
    const int c = local - U.slice * chunks;
    U.m0 = c * MT;
    U.mc = min(MT, U.G.rows - U.m0);
    return U;
}

__device__ __forceinline__ int token_of(const GroupView &G, int row, int N, int K, const int32_t *perm)
{
    return G.shared ? row - N * K : perm[row];
}

// ------------------------------------------------------------------ gate/up
// Features per warp: two 16-byte loads per lane and matrix per column block
// for the 2-byte and 1-byte weights (so that as many bytes are in flight
// for E4M3 as for BF16), four for FP32.
template <class WT> struct UpF { static constexpr int v = WVec<WT>::VEC == 4 ? 4 : 2; };

template <class WT, class XT, class HT, int MT>
__global__ void __launch_bounds__(kThreads, MT <= 2 ? 3 : 1)
ffn_up_stream_kernel(const XT *__restrict__ x, int N, int d, int I, int E, int K,
                     const int32_t *__restrict__ perm, const int32_t *__restrict__ offsets,
                     ExpertPtrs routed, ExpertPtrs shared, int has_shared, HT *__restrict__ H)
{
    constexpr int VEC = WVec<WT>::VEC;
    constexpr int EPW = WVec<WT>::EPW;
    constexpr int CH = VEC == 16 ? 4 : VEC;         // weights converted at a time
    constexpr int F = UpF<WT>::v;                   // features per warp
    constexpr int FS = F * kWarps;                  // features per unit
    __shared__ int pre[kMaxGroupsS + 1];
    extern __shared__ float4 smem_f4[];
    float *xs = reinterpret_cast<float *>(smem_f4); // [MT][d]
    const int S = I / FS;
    const int n_ord = E + (has_shared ? 1 : 0);
    build_unit_prefix<MT>(pre, n_ord, S, N, K, E, has_shared, offsets);
    __syncthreads();
    const int total = pre[n_ord];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const size_t mat = (size_t)I * d;
    const int sb = (I / 128) * (d / 128);
    const int cb = d / 128;

    for (int u = blockIdx.x; u < total; u += gridDim.x) {
        const Unit U = decode_unit<MT>(u, pre, n_ord, S, N, K, E, has_shared, offsets);
        const ExpertPtrs &P = U.G.shared ? shared : routed;
        const size_t ge = U.G.shared ? 0 : (size_t)U.G.g;
        const int f0 = U.slice * FS + warp * F;
        const WT *wg = static_cast<const WT *>(P.wg) + ge * mat + (size_t)f0 * d;
        const WT *wu = static_cast<const WT *>(P.wu) + ge * mat + (size_t)f0 * d;
        const float *sg = P.sg ? P.sg + ge * sb : nullptr;
        const float *su = P.su ? P.su + ge * sb : nullptr;

        __syncthreads();                            // previous unit done with xs
        const int vpr = d / 8;
        for (int i = threadIdx.x; i < MT * vpr; i += kThreads) {
            const int m = i / vpr, c = (i - m * vpr) * 8;
            float v[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
            if (m < U.mc) load8(x + (size_t)token_of(U.G, U.G.row0 + U.m0 + m, N, K, perm) * d + c, v);
            float4 *dst = reinterpret_cast<float4 *>(xs + m * d + c);
            dst[0] = make_float4(v[0], v[1], v[2], v[3]);
            dst[1] = make_float4(v[4], v[5], v[6], v[7]);
        }
        __syncthreads();

        float ag[F][MT], au[F][MT];
#pragma unroll
        for (int f = 0; f < F; ++f)
#pragma unroll
            for (int m = 0; m < MT; ++m) ag[f][m] = au[f][m] = 0.f;

        for (int j0 = lane * VEC; j0 < d; j0 += 64 * VEC) {
            uint4 rg[2][F], ru[2][F];
            const bool two = j0 + 32 * VEC < d;
#pragma unroll
            for (int b = 0; b < 2; ++b)
#pragma unroll
                for (int f = 0; f < F; ++f) {
                    if (b == 0 || two) {
                        rg[b][f] = ld_stream(wg + (size_t)f * d + j0 + b * 32 * VEC);
                        ru[b][f] = ld_stream(wu + (size_t)f * d + j0 + b * 32 * VEC);
                    }
                }
#pragma unroll
            for (int b = 0; b < 2; ++b) {
                if (b == 1 && !two) break;
                const int j = j0 + b * 32 * VEC;
#pragma unroll
                for (int f = 0; f < F; ++f) {
                    float s_g = 1.f, s_u = 1.f;
                    if (sg) {
                        const int sidx = ((f0 + f) / 128) * cb + j / 128;
                        s_g = sg[sidx];
                        s_u = su[sidx];
                    }
                    // CH weights at a time (all 8 for BF16, one 32-bit word of 4 for
                    // E4M3): few values live, x read with 16-byte shared loads
#pragma unroll
                    for (int c = 0; c < VEC / CH; ++c) {
                        float vg[CH], vu[CH];
#pragma unroll
                        for (int w = 0; w < CH / EPW; ++w) {
                            WVec<WT>::cvt_word(word_of(rg[b][f], c * (CH / EPW) + w), vg + w * EPW, s_g);
                            WVec<WT>::cvt_word(word_of(ru[b][f], c * (CH / EPW) + w), vu + w * EPW, s_u);
                        }
#pragma unroll
                        for (int m = 0; m < MT; ++m) {
#pragma unroll
                            for (int q = 0; q < CH; q += 4) {
                                const float4 xv = *reinterpret_cast<const float4 *>(xs + m * d + j + c * CH + q);
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
            }
        }
        const int r0 = U.G.row0 + U.m0;
#pragma unroll
        for (int f = 0; f < F; ++f)
#pragma unroll
            for (int m = 0; m < MT; ++m) {
                const float a = warp_sum(ag[f][m]);
                const float b = warp_sum(au[f][m]);
                if (lane == 0 && m < U.mc) store_val(H + (size_t)(r0 + m) * I + f0 + f, a * sigmoidf_(a) * b);
            }
    }
}

// --------------------------------------------------------------------- down
constexpr int kDownRows = 4;          // output features per warp and pass
constexpr int kDownPasses = 4;        // passes per unit
constexpr int kDownFS = kDownRows * kWarps * kDownPasses;   // 128 output features per unit

template <class WT, class HT, int MT>
__global__ void __launch_bounds__(kThreads, MT <= 2 ? 3 : 1)
ffn_down_stream_kernel(const HT *__restrict__ H, int N, int d, int I, int E, int K,
                       const int32_t *__restrict__ offsets, ExpertPtrs routed, ExpertPtrs shared,
                       int has_shared, HT *__restrict__ y_perm, HT *__restrict__ y_shared)
{
    constexpr int VEC = WVec<WT>::VEC;
    constexpr int EPW = WVec<WT>::EPW;
    constexpr int CH = VEC == 16 ? 4 : VEC;
    __shared__ int pre[kMaxGroupsS + 1];
    extern __shared__ float4 smem_f4[];
    float *hs = reinterpret_cast<float *>(smem_f4);  // [MT][I]
    const int S = d / kDownFS;
    const int n_ord = E + (has_shared ? 1 : 0);
    build_unit_prefix<MT>(pre, n_ord, S, N, K, E, has_shared, offsets);
    __syncthreads();
    const int total = pre[n_ord];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const size_t mat = (size_t)I * d;
    const int sb = (I / 128) * (d / 128);
    const int ib = I / 128;

    for (int u = blockIdx.x; u < total; u += gridDim.x) {
        const Unit U = decode_unit<MT>(u, pre, n_ord, S, N, K, E, has_shared, offsets);
        const ExpertPtrs &P = U.G.shared ? shared : routed;
        const size_t ge = U.G.shared ? 0 : (size_t)U.G.g;
        const float *sd = P.sd ? P.sd + ge * sb : nullptr;
        const int r0 = U.G.row0 + U.m0;

        __syncthreads();
        for (int i = threadIdx.x; i < MT * I; i += kThreads) {
            const int m = i / I, c = i - m * I;
            hs[i] = m < U.mc ? to_f32(H[(size_t)(r0 + m) * I + c]) : 0.f;
        }
        __syncthreads();
        HT *Y = U.G.shared ? y_shared + (size_t)(r0 - N * K) * d : y_perm + (size_t)r0 * d;

        for (int pass = 0; pass < kDownPasses; ++pass) {
        const int j0 = U.slice * kDownFS + (pass * kWarps + warp) * kDownRows;
        const WT *wd = static_cast<const WT *>(P.wd) + ge * mat + (size_t)j0 * I;
        float acc[kDownRows][MT];
#pragma unroll
        for (int r = 0; r < kDownRows; ++r)
#pragma unroll
            for (int m = 0; m < MT; ++m) acc[r][m] = 0.f;
        for (int i0 = lane * VEC; i0 < I; i0 += 64 * VEC) {
            uint4 raw[2][kDownRows];
            const bool two = i0 + 32 * VEC < I;
#pragma unroll
            for (int b = 0; b < 2; ++b)
#pragma unroll
                for (int r = 0; r < kDownRows; ++r)
                    if (b == 0 || two) raw[b][r] = ld_stream(wd + (size_t)r * I + i0 + b * 32 * VEC);
#pragma unroll
            for (int b = 0; b < 2; ++b) {
                if (b == 1 && !two) break;
                const int i = i0 + b * 32 * VEC;
#pragma unroll
                for (int r = 0; r < kDownRows; ++r) {
                    const float s = sd ? sd[((j0 + r) / 128) * ib + i / 128] : 1.f;
#pragma unroll
                    for (int c = 0; c < VEC / CH; ++c) {
                        float w[CH];
#pragma unroll
                        for (int wi = 0; wi < CH / EPW; ++wi)
                            WVec<WT>::cvt_word(word_of(raw[b][r], c * (CH / EPW) + wi), w + wi * EPW, s);
#pragma unroll
                        for (int m = 0; m < MT; ++m) {
#pragma unroll
                            for (int q = 0; q < CH; q += 4) {
                                const float4 hv = *reinterpret_cast<const float4 *>(hs + m * I + i + c * CH + q);
                                acc[r][m] = fmaf(w[q], hv.x, acc[r][m]);
                                acc[r][m] = fmaf(w[q + 1], hv.y, acc[r][m]);
                                acc[r][m] = fmaf(w[q + 2], hv.z, acc[r][m]);
                                acc[r][m] = fmaf(w[q + 3], hv.w, acc[r][m]);
                            }
                        }
                    }
                }
            }
        }
#pragma unroll
        for (int r = 0; r < kDownRows; ++r)
#pragma unroll
            for (int m = 0; m < MT; ++m) {
                const float v = warp_sum(acc[r][m]);
                if (lane == 0 && m < U.mc) store_val(Y + (size_t)m * d + j0 + r, v);
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

template <class Kern>
static int resident_grid(Kern k, size_t smem)
{
    int per_sm = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, k, kThreads, smem) != cudaSuccess || per_sm < 1)
        per_sm = 1;
    return sm_count() * per_sm;
}

template <class WT, class XT, class HT, int MT>
static kmoe_status run_stream_mt(const XT *x, int N, int d, int I, int E, int K, const int32_t *perm,
                                 const int32_t *offsets, const ExpertPtrs &routed, const ExpertPtrs *shared,
                                 HT *h, HT *y_perm, HT *y_shared, cudaStream_t st)
{
    const int has_shared = shared ? 1 : 0;
    const ExpertPtrs sh = shared ? *shared : ExpertPtrs{};
    const size_t up_smem = sizeof(float) * MT * d;
    const size_t down_smem = sizeof(float) * MT * I;
    auto upk = ffn_up_stream_kernel<WT, XT, HT, MT>;
    auto dnk = ffn_down_stream_kernel<WT, HT, MT>;
    cudaFuncSetAttribute(upk, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)up_smem);
    cudaFuncSetAttribute(dnk, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)down_smem);
    upk<<<resident_grid(upk, up_smem), kThreads, up_smem, st>>>(x, N, d, I, E, K, perm, offsets, routed, sh,
                                                                 has_shared, h);
    kmoe_status s = check_launch("ffn_up_stream");
    if (s != KMOE_OK) return s;
    dnk<<<resident_grid(dnk, down_smem), kThreads, down_smem, st>>>(h, N, d, I, E, K, offsets, routed, sh,
                                                                     has_shared, y_perm, y_shared);
    return check_launch("ffn_down_stream");
}

// Decode batches (a routed expert sees one or two tokens) use 2-row chunks,
// which keeps registers low enough for three CTAs per SM; larger batches use
// 8-row chunks so that the weights are re-read from L2 fewer times.
constexpr int kSmallBatch = 256;

template <class WT, class XT, class HT>
static kmoe_status run_stream(const XT *x, int N, int d, int I, int E, int K, const int32_t *perm,
                              const int32_t *offsets, const ExpertPtrs &routed, const ExpertPtrs *shared,
                              HT *h, HT *y_perm, HT *y_shared, cudaStream_t st)
{
    if (N < kSmallBatch)
        return run_stream_mt<WT, XT, HT, 2>(x, N, d, I, E, K, perm, offsets, routed, shared, h, y_perm, y_shared, st);
    return run_stream_mt<WT, XT, HT, 8>(x, N, d, I, E, K, perm, offsets, routed, shared, h, y_perm, y_shared, st);
}

kmoe_status launch_ffn_stream(const void *x, int x_dtype, int N, int d, int I, int E, int K,
                              const int32_t *perm, const int32_t *offsets, int w_dtype,
                              const ExpertPtrs &routed, const ExpertPtrs *shared,
                              void *h, void *y_perm, void *y_shared, cudaStream_t st)
{
    using bf = __nv_bfloat16;
    if (E + 1 > kMaxGroupsS) return fail(KMOE_ERR_UNSUPPORTED, "streaming FFN: too many experts");
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
