// Dispatch: histogram, exclusive scan and the stable (expert, token)
// permutation of the N*K routed (token, slot) pairs.
//
// The pages say only that routing is token-choice top-k and that tokens are
// sent to the experts they selected ("Inside Kolibri 1", routing section).
// The order chosen here (expert ascending, token ascending inside an expert)
// is a pure function of the indices, so every output is bit-exact and
// independent of scheduling: no atomics decide a position. Per-chunk
// ballot masks (permute_dev.cuh) give chunk histograms and in-chunk ranks;
// chunk histograms are scanned per expert in chunk order. Inside a layer
// call the top-K kernel counts the chunk histograms instead (integer
// atomics, exact in any order), and up to 64 chunks the scatter kernel
// forms the scan itself.
#include "permute_dev.cuh"

namespace kmoe {

// Pass 1: per-chunk histogram hist[c][e].
__global__ void __launch_bounds__(kChunk)
chunk_hist_kernel(const int32_t *__restrict__ idx, int N, int K, int E, int32_t *__restrict__ hist)
{
    pdl_wait();
    pdl_trigger();
    extern __shared__ uint32_t mask[];
    build_masks(idx, N, K, E, blockIdx.x, mask);
    for (int e = threadIdx.x; e < E; e += blockDim.x) {
        int c = 0;
#pragma unroll
        for (int w = 0; w < kChunkWarps; ++w) c += __popc(mask[w * E + e]);
        hist[(size_t)blockIdx.x * E + e] = c;
    }
}

// Pass 2 (one CTA, thread e): counts, offsets, and hist[c][e] replaced by
// the first dispatched row of chunk c for expert e.
__global__ void __launch_bounds__(1024)
scan_kernel(int32_t *__restrict__ hist, int chunks, int E, int32_t *__restrict__ counts,
            int32_t *__restrict__ offsets)
{
    pdl_wait();
    pdl_trigger();
    __shared__ int tmp[32];
    const int e = threadIdx.x;
    int total = 0;
    if (e < E)
        for (int c = 0; c < chunks; ++c) total += hist[(size_t)c * E + e];
    const int excl = block_exclusive_scan(e < E ? total : 0, tmp);
    if (e < E) {
        counts[e] = total;
        offsets[e] = excl;
        if (e == E - 1) offsets[E] = excl + total;
        int run = excl;
        for (int c = 0; c < chunks; ++c) {
            const int v = hist[(size_t)c * E + e];
            hist[(size_t)c * E + e] = run;
            run += v;
        }
    }
}

// Pass 3: scatter perm_token and inv_pos.
__global__ void __launch_bounds__(kChunk)
scatter_kernel(const int32_t *__restrict__ idx, int N, int K, int E,
               const int32_t *__restrict__ base, int32_t *__restrict__ perm, int32_t *__restrict__ inv)
{
    pdl_wait();
    pdl_trigger();
    extern __shared__ uint32_t mask[];
    build_masks(idx, N, K, E, blockIdx.x, mask);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int t = blockIdx.x * kChunk + threadIdx.x;
    if (t >= N) return;
    for (int k = 0; k < K; ++k) {
        const int e = idx[(size_t)t * K + k];
        if ((unsigned)e >= (unsigned)E) continue;
        const int pos = base[(size_t)blockIdx.x * E + e] + rank_in_chunk(mask, E, e, warp, lane);
        perm[pos] = t;
        inv[(size_t)t * K + k] = pos;
    }
}

// Pass 3 with the scan folded in, for up to kScanChunks chunks: every CTA
// sums the chunk histograms itself, in chunk order (the same sums the scan
// pass forms), so no separate scan launch is needed; CTA 0 also writes
// counts and offsets.
constexpr int kScanChunks = 64;

__global__ void __launch_bounds__(kChunk)
scatter_scan_kernel(const int32_t *__restrict__ idx, int N, int K, int E, int chunks,
                    const int32_t *__restrict__ hist, int32_t *__restrict__ counts, int32_t *__restrict__ offsets,
                    int32_t *__restrict__ perm, int32_t *__restrict__ inv)
{
    pdl_wait();
    pdl_trigger();
    extern __shared__ uint32_t mask[];               // kChunkWarps * E ballot words, then E row bases
    int *base = reinterpret_cast<int *>(mask + kChunkWarps * E);
    __shared__ int tmp[32];
    __shared__ int round_total;
    const int c = blockIdx.x;
    int carry = 0;
    for (int e0 = 0; e0 < E; e0 += blockDim.x) {
        const int e = e0 + threadIdx.x;
        int total = 0, before = 0;
        if (e < E)
            for (int q = 0; q < chunks; ++q) {
                const int v = hist[(size_t)q * E + e];
                before += q < c ? v : 0;
                total += v;
            }
        const int excl = block_exclusive_scan(e < E ? total : 0, tmp);
        if (e < E) {
            base[e] = carry + excl + before;
            if (c == 0) {
                counts[e] = total;
                offsets[e] = carry + excl;
            }
        }
        if (threadIdx.x == blockDim.x - 1) round_total = excl + total;
        __syncthreads();
        carry += round_total;
        __syncthreads();
    }
    if (c == 0 && threadIdx.x == 0) offsets[E] = carry;
    build_masks(idx, N, K, E, c, mask);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int t = c * kChunk + threadIdx.x;
    if (t >= N) return;
    for (int k = 0; k < K; ++k) {
        const int e = idx[(size_t)t * K + k];
        if ((unsigned)e >= (unsigned)E) continue;
        const int pos = base[e] + rank_in_chunk(mask, E, e, warp, lane);
        perm[pos] = t;
        inv[(size_t)t * K + k] = pos;
    }
}

// N <= 256: everything in one CTA (decode batches); W ballot-mask words per expert.
template <int W>
__global__ void __launch_bounds__(kChunk)
permute_single_kernel(const int32_t *__restrict__ idx, int N, int K, int E,
                      int32_t *__restrict__ counts, int32_t *__restrict__ offsets,
                      int32_t *__restrict__ perm, int32_t *__restrict__ inv)
{
    pdl_wait();
    pdl_trigger();
    extern __shared__ uint32_t mask[];
    permute_small_block<W>(idx, N, K, E, counts, offsets, perm, inv, mask);
}

size_t permute_ws_bytes(int N, int E)
{
    const size_t chunks = (size_t)(N + kChunk - 1) / kChunk;
    return chunks * E * sizeof(int32_t);
}

kmoe_status launch_permute(const int32_t *idx, int N, int K, int E, int32_t *counts,
                           int32_t *offsets, int32_t *perm, int32_t *inv, int32_t *hist,
                           cudaStream_t st, bool hist_ready)
{
    const size_t mask_bytes = sizeof(uint32_t) * kChunkWarps * E;
    if (N <= kChunk) {
        const size_t smem = mask_bytes + sizeof(int) * E;
        if (N <= 32) {
            launch_pdl(permute_single_kernel<1>, 1, kChunk, sizeof(uint32_t) * 2 * E, st, idx, N, K, E, counts,
                       offsets, perm, inv);
        } else {
            cudaFuncSetAttribute(permute_single_kernel<kChunkWarps>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 (int)smem);
            launch_pdl(permute_single_kernel<kChunkWarps>, 1, kChunk, smem, st, idx, N, K, E, counts, offsets, perm,
                       inv);
        }
        return check_launch("permute_single");
    }
    const int chunks = (N + kChunk - 1) / kChunk;
    if (hist_ready && chunks <= kScanChunks) {
        const size_t smem = mask_bytes + sizeof(int) * E;
        cudaFuncSetAttribute(scatter_scan_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        launch_pdl(scatter_scan_kernel, chunks, kChunk, smem, st, idx, N, K, E, chunks,
                   static_cast<const int32_t *>(hist), counts, offsets, perm, inv);
        return check_launch("permute_scatter_scan");
    }
    cudaFuncSetAttribute(chunk_hist_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)mask_bytes);
    cudaFuncSetAttribute(scatter_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)mask_bytes);
    kmoe_status s;
    if (!hist_ready) {
        launch_pdl(chunk_hist_kernel, chunks, kChunk, mask_bytes, st, idx, N, K, E, hist);
        s = check_launch("permute_hist");
        if (s != KMOE_OK) return s;
    }
    launch_pdl(scan_kernel, 1, 1024, 0, st, hist, chunks, E, counts, offsets);
    s = check_launch("permute_scan");
    if (s != KMOE_OK) return s;
    launch_pdl(scatter_kernel, chunks, kChunk, mask_bytes, st, idx, N, K, E,
               static_cast<const int32_t *>(hist), perm, inv);
    return check_launch("permute_scatter");
}

}  // namespace kmoe
