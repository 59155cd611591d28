// FP32 router logits on the tensor cores, for large batches (prefill).
//
// "Inside Kolibri 1" (flozi.net), routing section: the router produces FP32
// logits [N, 384] from x [N, 2560]; the FP8 section adds that the serving
// path keeps router output logits in FP32. With x in BF16 and the router
// weight stored in FP32, the logits are computed without giving up FP32
// weight precision: W_r is split into three BF16 terms
//     W_r = W1 + W2 + W3,  W1 = bf16(W_r), W2 = bf16(W_r - W1), W3 = bf16(W_r - W1 - W2)
// (together they carry the 24-bit FP32 significand), every product x * Wi is
// exact in FP32, and the three GEMMs accumulate into one FP32 accumulator in
// tensor memory: l = x W1^T + x W2^T + x W3^T. On CUDA cores the same
// 2*N*d*E FLOPs (16 GFLOP at N = 8192) would cost ~0.2 ms at the FP32 peak.
//
// The tensor cores' FP32 accumulation does not round like a scalar FP32 add:
// summing all 2560 columns in one accumulator drifted by up to 5e-5 from the
// double-precision logits, too much for a top-6 decided at 1e-5. So every
// 128 columns of K start a fresh accumulator (double-buffered in tensor
// memory, 2 x 192 columns), and the epilogue warps add the 20 partial sums in
// FP32 registers on the CUDA cores, which brings the error back to ~1e-7.
//
// One CTA computes a 128-token x 192-expert tile: warp 9 loads x and the
// weight-term tiles by TMA (128-byte swizzle) into a 5-stage ring, one
// thread of warp 8 issues tcgen05.mma (per 128-column round: 2 blocks of 64
// x 3 terms), warps 0-7 read each round's partial sums out of tensor memory
// (warps w and w+4 share lane quadrant w%4 and split the 192 columns) and
// finally store the logits. The top-K selection then runs on the stored
// logits.
#include "common.cuh"
#include "sm100.cuh"

#include <cudaTypedefs.h>

namespace kmoe {
using namespace sm100;

constexpr int kRBM = 128, kRBN = 192, kRBK = 64;
constexpr int kRStages = 5;
constexpr int kRA = kRBM * kRBK * 2;        // 16 KB
constexpr int kRB = kRBN * kRBK * 2;        // 24 KB
constexpr int kRStage = kRA + kRB;          // 40 KB (multiple of 1024)
constexpr int kRThreads = 10 * 32;
constexpr int kRMmaWarp = 8, kRProdWarp = 9;
constexpr int kRRoundBlocks = 2;            // 64-column blocks per fresh accumulator
constexpr int kRColsPerThread = kRBN / 2;   // 96
constexpr long long kRWaitLimit = 1LL << 32;

struct RouterMaps {
    CUtensorMap x;     // [N, d] BF16, box 128 rows x 64 columns
    CUtensorMap w;     // [3E, d] BF16 (the three weight terms stacked), box 192 rows x 64 columns
};

struct RouterTail {
    uint64_t full[kRStages], empty[kRStages], tfull[2], tempty[2], drain;
    uint32_t tmem_base;
    int abort;
};

constexpr size_t kRSmem = 1024 + (size_t)kRStages * kRStage + sizeof(RouterTail);

__global__ void __launch_bounds__(256)
router_split_kernel(const float *__restrict__ w, int n, __nv_bfloat16 *__restrict__ out)
{
    pdl_wait();
    pdl_trigger();
    for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < n; i += gridDim.x * blockDim.x) {
        const float v = w[i];
        const __nv_bfloat16 a = __float2bfloat16_rn(v);
        const float r1 = v - __bfloat162float(a);
        const __nv_bfloat16 b = __float2bfloat16_rn(r1);
        const float r2 = r1 - __bfloat162float(b);
        out[i] = a;
        out[n + i] = b;
        out[2 * n + i] = __float2bfloat16_rn(r2);
    }
}

__global__ void __launch_bounds__(kRThreads, 1)
router_tc_kernel(const __grid_constant__ RouterMaps maps, int N, int d, int E, float *__restrict__ logits,
                 int *err)
{
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    RouterTail *tail = reinterpret_cast<RouterTail *>(smem + (size_t)kRStages * kRStage);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    volatile int *abort = &tail->abort;
    const int m0 = blockIdx.x * kRBM, n0 = blockIdx.y * kRBN;
    const int iters = (d / kRBK) * 3;

    if (threadIdx.x == 0) {
        for (int s = 0; s < kRStages; ++s) {
            mbar_init(&tail->full[s], 1);
            mbar_init(&tail->empty[s], 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&tail->tfull[b], 1);
            mbar_init(&tail->tempty[b], 256);
        }
        mbar_init(&tail->drain, 1);
        tail->abort = 0;
        fence_mbar_init();
    }
    if (warp == 0) {
        tmem_alloc(&tail->tmem_base, 512);
        tmem_relinquish();
    }
    if (warp == kRProdWarp && lane == 0) {
        prefetch_map(&maps.x);
        prefetch_map(&maps.w);
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    pdl_wait();
    pdl_trigger();

    const uint32_t tmem = tail->tmem_base;

    if (warp == kRProdWarp) {
        if (lane == 0) {
            const uint64_t pol = policy_evict_last();   // x and the weight terms are read by several CTAs
            int i = 0;
            for (; i < iters; ++i) {
                const int s = i % kRStages;
                if (!mbar_wait(&tail->empty[s], ((i / kRStages) & 1) ^ 1, abort, err, kRWaitLimit)) break;
                const int kb = i / 3, term = i - kb * 3;
                uint8_t *As = smem + (size_t)s * kRStage;
                mbar_arrive_expect_tx(&tail->full[s], kRStage);
                tma_load_2d_hint(As, &maps.x, &tail->full[s], kb * kRBK, m0, pol);
                tma_load_2d_hint(As + kRA, &maps.w, &tail->full[s], kb * kRBK, term * E + n0, pol);
            }
            if (i < iters)     // aborted: let the loads already issued land
                for (int j = i > kRStages ? i - kRStages : 0; j < i; ++j)
                    mbar_wait_drain(&tail->full[j % kRStages], (j / kRStages) & 1, kRWaitLimit);
        }
    } else if (warp == kRMmaWarp) {
        if (lane == 0) {
            constexpr uint32_t idesc = idesc_bf16_f32(kRBM, kRBN);
            constexpr int per_round = kRRoundBlocks * 3;
            bool ok = true;
            for (int i = 0; i < iters && ok; ++i) {
                const int round = i / per_round, b = round & 1;
                const bool first = i % per_round == 0;
                if (first) {
                    if (!mbar_wait(&tail->tempty[b], ((round >> 1) & 1) ^ 1, abort, err, kRWaitLimit)) { ok = false; break; }
                    tc_fence_after();
                }
                const int s = i % kRStages;
                if (!mbar_wait(&tail->full[s], (i / kRStages) & 1, abort, err, kRWaitLimit)) { ok = false; break; }
                tc_fence_after();
                const uint64_t ad = sw128_kmajor_desc(smem_u32(smem + (size_t)s * kRStage));
                const uint64_t bd = sw128_kmajor_desc(smem_u32(smem + (size_t)s * kRStage + kRA));
#pragma unroll
                for (int k = 0; k < kRBK / 16; ++k)
                    umma_bf16(tmem + b * kRBN, ad + (uint64_t)(k * 2), bd + (uint64_t)(k * 2), idesc,
                              !(first && k == 0));
                umma_commit(&tail->empty[s]);
                if (i % per_round == per_round - 1 || i == iters - 1) umma_commit(&tail->tfull[b]);
            }
            umma_commit(&tail->drain);
            mbar_wait_drain(&tail->drain, 0, kRWaitLimit);
        }
        __syncwarp();
    } else {
        // epilogue: warp w reads lane quadrant w % 4, columns [half * 96, half * 96 + 96)
        const int q = warp & 3, half = warp >> 2;
        const int row = q * 32 + lane;
        const int rounds = (iters + kRRoundBlocks * 3 - 1) / (kRRoundBlocks * 3);
        float acc[kRColsPerThread];
#pragma unroll
        for (int c = 0; c < kRColsPerThread; ++c) acc[c] = 0.f;
        bool ok = true;
        for (int r = 0; r < rounds; ++r) {
            const int b = r & 1;
            if (!mbar_wait(&tail->tfull[b], (r >> 1) & 1, abort, err, kRWaitLimit)) { ok = false; break; }
            tc_fence_after();
            const uint32_t tbase = tmem + ((uint32_t)(q * 32) << 16) + b * kRBN + half * kRColsPerThread;
#pragma unroll
            for (int c = 0; c < kRColsPerThread; c += 16) {
                uint32_t v[16];
                tmem_ld16(tbase + c, v);
                tmem_ld_wait();
#pragma unroll
                for (int j = 0; j < 16; ++j) acc[c + j] += __uint_as_float(v[j]);
            }
            tc_fence_before();
            mbar_arrive(&tail->tempty[b]);
        }
        if (ok && m0 + row < N) {
            const int cbase = n0 + half * kRColsPerThread;
            float *dst = logits + (size_t)(m0 + row) * E + cbase;
            if (cbase + kRColsPerThread <= E && (E & 3) == 0) {
#pragma unroll
                for (int c = 0; c < kRColsPerThread; c += 4)
                    *reinterpret_cast<float4 *>(dst + c) = make_float4(acc[c], acc[c + 1], acc[c + 2], acc[c + 3]);
            } else {
#pragma unroll
                for (int c = 0; c < kRColsPerThread; ++c)
                    if (cbase + c < E) dst[c] = acc[c];
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, 512);
    }
}

static PFN_cuTensorMapEncodeTiled_v12000 encode_fn_r()
{
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    if (!fn) {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    }
    return fn;
}

static bool make_map_r(CUtensorMap *m, const void *base, uint64_t rows, uint64_t cols, uint32_t box_rows)
{
    auto fn = encode_fn_r();
    if (!fn) return false;
    cuuint64_t dims[2] = {cols, rows};
    cuuint64_t strides[1] = {cols * 2};
    cuuint32_t box[2] = {kRBK, box_rows};
    cuuint32_t estr[2] = {1, 1};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(base), dims, strides, box, estr,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

size_t router_tc_ws_bytes(int d, int E) { return (size_t)3 * E * d * sizeof(__nv_bfloat16); }

kmoe_status launch_router_tc(const __nv_bfloat16 *x, const float *w_router, int N, int d, int E,
                             __nv_bfloat16 *w_split, float *logits, int *err, cudaStream_t st)
{
    const int n = E * d;
    launch_pdl(router_split_kernel, (n + 255) / 256 < 1184 ? (n + 255) / 256 : 1184, 256, 0, st, w_router, n, w_split);
    kmoe_status s = check_launch("router_split");
    if (s != KMOE_OK) return s;
    RouterMaps maps{};
    if (!make_map_r(&maps.x, x, N, d, kRBM) || !make_map_r(&maps.w, w_split, (uint64_t)3 * E, d, kRBN))
        return fail(KMOE_ERR_CUDA, "cuTensorMapEncodeTiled failed (router)");
    cudaFuncSetAttribute(router_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kRSmem);
    dim3 grid((N + kRBM - 1) / kRBM, (E + kRBN - 1) / kRBN);
    launch_pdl(router_tc_kernel, grid, kRThreads, kRSmem, st, maps, N, d, E, logits, err);
    return check_launch("router_tc");
}

}  // namespace kmoe
