// Shared device helpers and host-side plumbing of the kmoe library.
#pragma once

#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <cuda_fp8.h>
#include <cstdint>
#include <cstddef>

#include "kmoe.h"

namespace kmoe {

// Index checks of the KMOE_DEBUG build (nvcc -DKMOE_DEBUG): a kernel that
// reads a dispatch index outside its range (a token or dispatched row past the
// batch, expert offsets that are not a monotone partition of the N*K rows)
// records kErrIndex in the device status word and uses a safe index (or skips
// the work) instead, so that no access leaves its buffer. Compiled out of the
// release library.
#ifdef KMOE_DEBUG
constexpr bool kDebugChecks = true;
#else
constexpr bool kDebugChecks = false;
#endif
enum : int { kErrIndex = 3 };

// Debug build: v if lo <= v < hi, else records kErrIndex in *err and returns lo.
__device__ __forceinline__ int checked_index(int v, int lo, int hi, int *err)
{
    if constexpr (kDebugChecks) {
        if (v < lo || v >= hi) {
            if (err) atomicCAS(err, 0, kErrIndex);
            return lo;
        }
    }
    return v;
}

// Debug build: whether off[0..E] is 0, monotone and ends at rows (one warp;
// records kErrIndex in *err otherwise). Always true in the release build.
__device__ __forceinline__ bool offsets_ok(const int *off, int E, int rows, int *err)
{
    if constexpr (kDebugChecks) {
        const int lane = threadIdx.x & 31;
        bool bad = false;
        for (int i = lane; i < E; i += 32) bad |= off[i] > off[i + 1];
        if (lane == 0) bad |= off[0] != 0 || off[E] != rows;
        bad = __any_sync(0xffffffffu, bad);
        if (bad && lane == 0 && err) atomicCAS(err, 0, kErrIndex);
        return !bad;
    }
    return true;
}

// Default give-up limit of a pipeline wait, in SM clock cycles (about 2 s at
// 1.9 GHz): far beyond any wait of a healthy launch. Waits that drain
// in-flight copies after another wait gave up always use this limit.
constexpr long long kDefaultWaitLimit = 1LL << 32;

// ---------------------------------------------------------------- host side

// Records a printf-style message as the calling thread's last error and
// returns `code`, so that call sites can write `return fail(...)`.
kmoe_status fail(kmoe_status code, const char *fmt, ...);
void clear_error();

// Checks the last launch; on failure records the CUDA error string.
kmoe_status check_launch(const char *what);

// Programmatic dependent launch. The kernels of a layer call are launched
// with launch_pdl, so each may start (its prologue: barriers, tensor memory,
// descriptor prefetch) while the previous kernel on the stream is still
// finishing. Every such kernel calls pdl_wait() before it reads anything an
// earlier kernel wrote (the wait returns once that kernel has completed and
// its writes are visible), then pdl_trigger() so that the next kernel can
// be scheduled. Without a programmatic predecessor both are no-ops.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_trigger() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

template <typename... KArgs, typename... Args>
inline void launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st, Args... args)
{
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr{};
    attr.id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr.val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = &attr;
    cfg.numAttrs = 1;
    cudaLaunchKernelEx(&cfg, kernel, static_cast<KArgs>(args)...);   // errors surface in check_launch
}

inline bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Carves 256-byte aligned pieces out of a caller-provided workspace.
struct Carver {
    char *base;
    size_t used = 0;
    explicit Carver(void *b) : base(static_cast<char *>(b)) {}
    template <class T>
    T *take(size_t count) {
        used = (used + 255) & ~size_t(255);
        T *p = base ? reinterpret_cast<T *>(base + used) : nullptr;
        used += count * sizeof(T);
        return p;
    }
};

// Weight pointers of one expert stack, as seen by the kernels.
struct ExpertPtrs {
    const void *wg, *wu, *wd;
    const float *sg, *su, *sd;
};

// ----------------------------------------------------------- device helpers

__device__ __forceinline__ float bf16_lo(uint32_t v) { return __uint_as_float(v << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t v) { return __uint_as_float(v & 0xffff0000u); }

// 16 bytes of weights -> VEC floats, for the three storage types.
template <class WT> struct WVec;

// cvt_word: one 32-bit word of the vector -> EPW = VEC/4 floats.
template <> struct WVec<float> {
    static constexpr int VEC = 4;
    static constexpr int EPW = 1;
    __device__ __forceinline__ static void cvt_word(uint32_t v, float *o, float) { o[0] = __uint_as_float(v); }
    __device__ __forceinline__ static void cvt(uint4 r, float *o, float) {
        o[0] = __uint_as_float(r.x); o[1] = __uint_as_float(r.y);
        o[2] = __uint_as_float(r.z); o[3] = __uint_as_float(r.w);
    }
};

template <> struct WVec<__nv_bfloat16> {
    static constexpr int VEC = 8;
    static constexpr int EPW = 2;
    __device__ __forceinline__ static void cvt_word(uint32_t v, float *o, float) { o[0] = bf16_lo(v); o[1] = bf16_hi(v); }
    __device__ __forceinline__ static void cvt(uint4 r, float *o, float) {
        o[0] = bf16_lo(r.x); o[1] = bf16_hi(r.x); o[2] = bf16_lo(r.y); o[3] = bf16_hi(r.y);
        o[4] = bf16_lo(r.z); o[5] = bf16_hi(r.z); o[6] = bf16_lo(r.w); o[7] = bf16_hi(r.w);
    }
};

template <> struct WVec<__nv_fp8_e4m3> {
    static constexpr int VEC = 16;
    static constexpr int EPW = 4;
    __device__ __forceinline__ static void cvt2(uint32_t v, float *o, float s) {
        __half2_raw lo = __nv_cvt_fp8x2_to_halfraw2(static_cast<__nv_fp8x2_storage_t>(v & 0xffffu), __NV_E4M3);
        __half2_raw hi = __nv_cvt_fp8x2_to_halfraw2(static_cast<__nv_fp8x2_storage_t>(v >> 16), __NV_E4M3);
        float2 a = __half22float2(*reinterpret_cast<__half2 *>(&lo));
        float2 b = __half22float2(*reinterpret_cast<__half2 *>(&hi));
        o[0] = a.x * s; o[1] = a.y * s; o[2] = b.x * s; o[3] = b.y * s;
    }
    __device__ __forceinline__ static void cvt(uint4 r, float *o, float s) {
        cvt2(r.x, o, s); cvt2(r.y, o + 4, s); cvt2(r.z, o + 8, s); cvt2(r.w, o + 12, s);
    }
    __device__ __forceinline__ static void cvt_word(uint32_t v, float *o, float s) { cvt2(v, o, s); }
};

// Activations: 8 consecutive values -> floats.
__device__ __forceinline__ void load8(const float *p, float *o) {
    float4 a = *reinterpret_cast<const float4 *>(p);
    float4 b = *reinterpret_cast<const float4 *>(p + 4);
    o[0] = a.x; o[1] = a.y; o[2] = a.z; o[3] = a.w; o[4] = b.x; o[5] = b.y; o[6] = b.z; o[7] = b.w;
}
__device__ __forceinline__ void load8(const __nv_bfloat16 *p, float *o) {
    uint4 r = *reinterpret_cast<const uint4 *>(p);
    WVec<__nv_bfloat16>::cvt(r, o, 1.f);
}

__device__ __forceinline__ void store_val(float *p, float v) { *p = v; }
__device__ __forceinline__ void store_val(__nv_bfloat16 *p, float v) { *p = __float2bfloat16_rn(v); }

__device__ __forceinline__ uint32_t word_of(const uint4 &r, int w) { return w == 0 ? r.x : w == 1 ? r.y : w == 2 ? r.z : r.w; }

__device__ __forceinline__ float to_f32(float v) { return v; }
__device__ __forceinline__ float to_f32(__nv_bfloat16 v) { return __bfloat162float(v); }

__device__ __forceinline__ float sigmoidf_(float z) { return 1.f / (1.f + expf(-z)); }

// SiLU(z) * u for the tensor-core FFN epilogues: z / (1 + e^-z) with the
// hardware exponential and reciprocal (__expf, __fdividef; a few ulp of
// FP32, far below the BF16 rounding of the result). z -> -inf gives 0
// (e^-z overflows to inf and __fdividef returns 0). The router's mixture
// weights use the IEEE sigmoidf_ above.
__device__ __forceinline__ float silu_mul(float z, float u) { return __fdividef(z, 1.f + __expf(-z)) * u; }

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

}  // namespace kmoe

// ------------------------------------------------ launchers between units

namespace kmoe {

kmoe_status launch_router_logits(const void *x, int x_dtype, const float *w_router, int N, int d,
                                 int E, float *logits, cudaStream_t st);
// hist (may be NULL): per-chunk expert histogram [ceil(N / 256), E], zero on
// entry, counted by the top-K kernel for the dispatch that follows.
kmoe_status launch_topk(const float *logits, const float *bias, int N, int E, int K, int score,
                        int32_t *idx, float *w, cudaStream_t st, int32_t *hist = nullptr);

// Router logits for N <= 256 (128 CTAs, three experts each); status is the
// device status word for a bounded wait that gives up. With zero_ints > 0 the
// kernel zeroes status[0 .. zero_ints) once the previous kernel on the stream
// has finished (the layer call's status block, in place of a memset).
kmoe_status launch_router_small(const void *x, int x_dtype, const float *w_router, int N, int d, int E,
                                float *logits, int *status, cudaStream_t st, int zero_ints = 0);

// Tensor-core FP32 router (x in BF16): W_r split into three BF16 terms in
// `w_split` (router_tc_ws_bytes), logits [N, E] written out.
size_t router_tc_ws_bytes(int d, int E);
kmoe_status launch_router_tc(const __nv_bfloat16 *x, const float *w_router, int N, int d, int E,
                             __nv_bfloat16 *w_split, float *logits, int *err, cudaStream_t st);
constexpr int kTcRouterTokens = 512;

size_t permute_ws_bytes(int N, int E);
// hist_ready: hist already holds the chunk histograms (counted by the top-K
// kernel), so the histogram pass is skipped.
kmoe_status launch_permute(const int32_t *idx, int N, int K, int E, int32_t *counts,
                           int32_t *offsets, int32_t *perm, int32_t *inv, int32_t *hist,
                           cudaStream_t st, bool hist_ready = false);

kmoe_status launch_ffn_stream(const void *x, int x_dtype, int N, int d, int I, int E, int K,
                              const int32_t *perm, const int32_t *offsets, int w_dtype,
                              const ExpertPtrs &routed, const ExpertPtrs *shared,
                              void *h, void *y_perm, void *y_shared, cudaStream_t st);

// Tensor-core grouped FFN (BF16 activations; BF16 or E4M3 + FP32 block-scale
// weights; d % 256 == 0). `sync` holds two tile counters and one finished-up-
// tiles counter per group (E + 3 ints), zero at launch.
kmoe_status launch_ffn_tc(const __nv_bfloat16 *x, int N, int d, int I, int E, int K, const int32_t *perm,
                          const int32_t *offsets, int w_dtype, const ExpertPtrs &routed, const ExpertPtrs *shared,
                          __nv_bfloat16 *h, __nv_bfloat16 *y_perm, __nv_bfloat16 *y_shared, int *err, int *sync,
                          long long wait_limit, cudaStream_t st);

// Batches of at least this many tokens take the tensor-core FFN.
constexpr int kTcMinTokens = 256;

// Swap-AB tensor-core FFN for small batches (BF16 activations and weights;
// d % 256 == 0). `sync` holds kSyncInts
// counters that must be zero at launch (a unit counter and one per expert).
// wait_limit (both tensor-core FFNs): SM cycles before a pipeline wait gives
// up and the kernel writes status 1 and returns.
constexpr int kSyncInts = 1088;
kmoe_status launch_ffn_swap(const __nv_bfloat16 *x, int N, int d, int I, int E, int K, const int32_t *perm,
                            const int32_t *offsets, const ExpertPtrs &routed, const ExpertPtrs *shared,
                            __nv_bfloat16 *h, __nv_bfloat16 *y_perm, __nv_bfloat16 *y_shared, int *status,
                            int *sync, long long wait_limit, cudaStream_t st);

// Grouped FFN with FP8 activations (E4M3 weights + FP32 128 x 128 block
// scales; x given as E4M3 codes xq [N, d] with FP32 scales xs [N, d / 128];
// H kept as codes hq [N*K + N, I] with scales hs [N*K + N, I / 128]; d % 256
// == 0). `sync` as for launch_ffn_swap. wait_limit: SM cycles before a
// pipeline wait gives up.
// With xl / hl set (two-term mode, 16-row chunks): x and H are each held as
// high and low E4M3 codes, x = s * (hi + lo / 16), which carries BF16
// precision (E4M3 weights with BF16 activations on the FP8 tensor cores).
kmoe_status launch_ffn_a8(const uint8_t *xq, const float *xs, int N, int d, int I, int E, int K, const int32_t *perm,
                          const int32_t *offsets, const ExpertPtrs &routed, const ExpertPtrs *shared, uint8_t *hq,
                          float *hs, __nv_bfloat16 *y_perm, __nv_bfloat16 *y_shared, int *status, int *sync,
                          long long wait_limit, cudaStream_t st, const uint8_t *xl = nullptr,
                          uint8_t *hl = nullptr);

// err: device status word for a bounded wait that gives up (may be NULL).
// h_res / g_post (BF16, NULL for the plain combine): y = h_res + RMSNorm(m) * g_post.
kmoe_status launch_combine(const void *y_perm, const void *y_shared, int y_in_dtype,
                           const float *w, const int32_t *inv, int N, int K, int d, void *y,
                           int y_dtype, int *err, cudaStream_t st, const void *h_res = nullptr,
                           const void *g_post = nullptr, float eps = 0.f);

// Dynamic FP8 quantisation of BF16 rows in groups of 128 columns: codes
// [rows, cols] (E4M3), scales [rows, cols / 128] (FP32).
kmoe_status launch_quant_1x128(const __nv_bfloat16 *x, int rows, int cols, uint8_t *codes, float *scales,
                               cudaStream_t st);

// Two E4M3 terms per value with the same group scale: x = s * (hi + lo / 16)
// up to about 2^-8 of |x| (BF16-precision activations for the FP8 MMA).
kmoe_status launch_quant_1x128_split(const __nv_bfloat16 *x, int rows, int cols, uint8_t *hi, uint8_t *lo,
                                     float *scales, cudaStream_t st);

// x = bf16(h / sqrt(mean(h^2) + eps) * gamma), row by row.
kmoe_status launch_rmsnorm(const __nv_bfloat16 *h, const __nv_bfloat16 *gamma, float eps, int N, int d,
                           __nv_bfloat16 *x, cudaStream_t st);

}  // namespace kmoe
