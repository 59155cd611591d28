// moe_permute_noalloc: the dispatch permutation for callers that cannot
// allocate device memory.
//
// moe_permute needs a scratch buffer for its per-chunk expert histograms when
// N > 256, and asks the caller for it as a workspace. Some callers cannot
// provide one: an engine that has already handed nearly all of the GPU's
// memory to a fixed pool (a KV cache, a weight arena) and must not make
// new cudaMalloc calls on the serving path, or a host application that loads
// this library as a plugin and gives it no allocator at all. For them this
// entry point keeps the scratch in a fixed array that the library itself
// owns in device global memory, so the call allocates nothing.
//
// The array lives for as long as the library is loaded, on every GPU that
// loads it (kScratchInts int32 = 1 MiB per GPU), and is shared by all calls
// on that GPU: two calls whose kernels overlap on the GPU (different
// streams, no ordering between them) race on it and give wrong results.
// Its contents are whatever the last call left there; every cell that a call
// reads was first written by the same call (the per-chunk histogram pass
// writes all of its chunks x E entries), so nothing needs clearing.
#include "common.cuh"

#include <mutex>

namespace kmoe {

// 256 chunks of 256 tokens (N <= 65536) times E <= 1024 experts.
constexpr size_t kScratchInts = 256 * 1024;

static __device__ __align__(256) int32_t g_permute_scratch[kScratchInts];

constexpr int kMaxDevices = 64;
static std::mutex g_scratch_mu;
static int32_t *g_scratch_ptr[kMaxDevices] = {};

// Device address of g_permute_scratch on the current device. In host code
// the symbol's name is only a host-side stand-in, so the address is looked
// up once per device (with that device current) and cached for the life of
// the process; the cache assumes the primary context of the device is not
// torn down (cudaDeviceReset) while the library is in use.
static kmoe_status scratch_on_current_device(int32_t **out)
{
    int dev = -1;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return fail(KMOE_ERR_CUDA, "cudaGetDevice: %s", cudaGetErrorString(e));
    if (dev < 0 || dev >= kMaxDevices) return fail(KMOE_ERR_UNSUPPORTED, "device ordinal %d >= %d", dev, kMaxDevices);
    std::lock_guard<std::mutex> lock(g_scratch_mu);
    if (!g_scratch_ptr[dev]) {
        void *p = nullptr;
        e = cudaGetSymbolAddress(&p, g_permute_scratch);
        if (e != cudaSuccess || !p)
            return fail(KMOE_ERR_CUDA, "cudaGetSymbolAddress(permute scratch): %s", cudaGetErrorString(e));
        g_scratch_ptr[dev] = static_cast<int32_t *>(p);
    }
    *out = g_scratch_ptr[dev];
    return KMOE_OK;
}

}  // namespace kmoe

using namespace kmoe;

extern "C" kmoe_status moe_permute_noalloc(const int32_t *topk_idx, int N, int K, int E, int32_t *counts,
                                           int32_t *offsets, int32_t *perm_token, int32_t *inv_pos,
                                           void *stream)
{
    clear_error();
    if (N < 0) return fail(KMOE_ERR_INVALID_ARG, "N=%d must be >= 0", N);
    if (K < 1 || K > 8) return fail(KMOE_ERR_UNSUPPORTED, "K=%d: supported 1 <= K <= 8", K);
    if (E < K) return fail(KMOE_ERR_INVALID_ARG, "E=%d must be >= K=%d", E, K);
    if (E > 1024) return fail(KMOE_ERR_UNSUPPORTED, "E=%d: supported E <= 1024", E);
    const size_t need = permute_ws_bytes(N, E) / sizeof(int32_t);
    if (need > kScratchInts)
        return fail(KMOE_ERR_UNSUPPORTED,
                    "moe_permute_noalloc: N=%d, E=%d need %zu scratch ints, the fixed array holds %zu "
                    "(ceil(N/256) * E <= 262144, e.g. N <= 65536 at E = 1024); use moe_permute with a workspace",
                    N, E, need, kScratchInts);
    if (!counts || !offsets) return fail(KMOE_ERR_INVALID_ARG, "counts/offsets is NULL");
    if (!aligned16(counts) || !aligned16(offsets)) return fail(KMOE_ERR_INVALID_ARG, "counts/offsets not 16-byte aligned");
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (N == 0) {
        if (cudaMemsetAsync(counts, 0, sizeof(int32_t) * E, st) != cudaSuccess ||
            cudaMemsetAsync(offsets, 0, sizeof(int32_t) * (E + 1), st) != cudaSuccess)
            return check_launch("permute_noalloc memset");
        return KMOE_OK;
    }
    if (!topk_idx || !perm_token || !inv_pos) return fail(KMOE_ERR_INVALID_ARG, "topk_idx/perm_token/inv_pos is NULL");
    if (!aligned16(topk_idx) || !aligned16(perm_token) || !aligned16(inv_pos))
        return fail(KMOE_ERR_INVALID_ARG, "topk_idx/perm_token/inv_pos not 16-byte aligned");
    int32_t *scratch = nullptr;
    kmoe_status s = scratch_on_current_device(&scratch);
    if (s != KMOE_OK) return s;
    return launch_permute(topk_idx, N, K, E, counts, offsets, perm_token, inv_pos, scratch, st);
}
