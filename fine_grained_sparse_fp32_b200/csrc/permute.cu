// Dispatch: histogram, exclusive scan and the stable (expert, token)
// permutation of the N*K routed (token, slot) pairs.
//
// The pages say only that routing is token-choice top-k and that tokens are
// sent to the experts they selected ("Inside Kolibri 1", routing section).
// The order chosen here (expert ascending, token ascending inside an expert)
// is a pure function of the indices, so every output is bit-exact and
// independent of scheduling: no atomics decide a position.
//
// Tokens are cut into chunks of 256 (one CTA, 8 warps of 32 tokens). Inside
// a CTA, bit `lane` of mask[w][e] says "token 32*w + lane of this chunk chose
// expert e"; popcounts of those masks give the per-chunk histogram and the
// rank of a token among the earlier tokens of its chunk that chose the same
// expert. Chunk histograms are scanned per expert in chunk order.
#include "common.cuh"

namespace kmoe {

constexpr int kChunk = 256;
constexpr int kChunkWarps = kChunk / 32;

// Builds the 8 x E ballot masks of one chunk in shared memory.
__device__ __forceinline__ void build_masks(const int32_t *__restrict__ idx, int N, int K, int E,
                                            int chunk, uint32_t *mask)
{
    for (int i = threadIdx.x; i < kChunkWarps * E; i += blockDim.x) mask[i] = 0u;
    __syncthreads();
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int t = chunk * kChunk + threadIdx.x;
    if (t < N) {
        for (int k = 0; k < K; ++k) {
            const int e = idx[(size_t)t * K + k];
            if ((unsigned)e < (unsigned)E) atomicOr(&mask[warp * E + e], 1u << lane);
        }
    }
    __syncthreads();
}

// Pass 1: per-chunk histogram hist[c][e].
__global__ void __launch_bounds__(kChunk)
chunk_hist_kernel(const int32_t *__restrict__ idx, int N, int K, int E, int32_t *__restrict__ hist)
{
    extern __shared__ uint32_t mask[];
    build_masks(idx, N, K, E, blockIdx.x, mask);
    for (int e = threadIdx.x; e < E; e += blockDim.x) {
        int c = 0;
#pragma unroll
        for (int w = 0; w < kChunkWarps; ++w) c += __popc(mask[w * E + e]);
        hist[(size_t)blockIdx.x * E + e] = c;
    }
}

// Block-wide exclusive scan over threadIdx.x (blockDim.x a multiple of 32).
__device__ __forceinline__ int block_exclusive_scan(int v, int *tmp)
{
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    int incl = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int n = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += n;
    }
    if (lane == 31) tmp[warp] = incl;
    __syncthreads();
    if (warp == 0) {
        const int nw = blockDim.x >> 5;
        int s = lane < nw ? tmp[lane] : 0;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int n = __shfl_up_sync(0xffffffffu, s, o);
            if (lane >= o) s += n;
        }
        if (lane < nw) tmp[lane] = s;   // inclusive warp totals
    }
    __syncthreads();
    const int before = warp ? tmp[warp - 1] : 0;
    __syncthreads();
    return before + incl - v;
}

// Pass 2 (one CTA, thread e): counts, offsets, and hist[c][e] replaced by
// the first dispatched row of chunk c for expert e.
__global__ void __launch_bounds__(1024)
scan_kernel(int32_t *__restrict__ hist, int chunks, int E, int32_t *__restrict__ counts,
            int32_t *__restrict__ offsets)
{
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

// Rank of token (warp, lane) among the earlier tokens of its chunk that chose e.
__device__ __forceinline__ int rank_in_chunk(const uint32_t *mask, int E, int e, int warp, int lane)
{
    int r = __popc(mask[warp * E + e] & ((1u << lane) - 1u));
    for (int w = 0; w < warp; ++w) r += __popc(mask[w * E + e]);
    return r;
}

// Pass 3: scatter perm_token and inv_pos.
__global__ void __launch_bounds__(kChunk)
scatter_kernel(const int32_t *__restrict__ idx, int N, int K, int E,
               const int32_t *__restrict__ base, int32_t *__restrict__ perm, int32_t *__restrict__ inv)
{
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

// N <= 256: everything in one CTA (decode batches).
__global__ void __launch_bounds__(kChunk)
permute_single_kernel(const int32_t *__restrict__ idx, int N, int K, int E,
                      int32_t *__restrict__ counts, int32_t *__restrict__ offsets,
                      int32_t *__restrict__ perm, int32_t *__restrict__ inv)
{
    extern __shared__ uint32_t mask[];
    __shared__ int tmp[32];
    int *start = reinterpret_cast<int *>(mask + kChunkWarps * E);   // [E]
    build_masks(idx, N, K, E, 0, mask);
    // E may exceed the CTA: scan in rounds of blockDim.x experts.
    int carry = 0;
    for (int e0 = 0; e0 < E; e0 += blockDim.x) {
        const int e = e0 + threadIdx.x;
        int c = 0;
        if (e < E) {
#pragma unroll
            for (int w = 0; w < kChunkWarps; ++w) c += __popc(mask[w * E + e]);
        }
        const int excl = block_exclusive_scan(c, tmp);
        if (e < E) {
            counts[e] = c;
            offsets[e] = carry + excl;
            start[e] = carry + excl;
        }
        // total of this round = last thread's exclusive + its count
        __shared__ int round_total;
        if (threadIdx.x == blockDim.x - 1) round_total = excl + c;
        __syncthreads();
        carry += round_total;
        __syncthreads();
    }
    if (threadIdx.x == 0) offsets[E] = carry;
    __syncthreads();
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int t = threadIdx.x;
    if (t >= N) return;
    for (int k = 0; k < K; ++k) {
        const int e = idx[(size_t)t * K + k];
        if ((unsigned)e >= (unsigned)E) continue;
        const int pos = start[e] + rank_in_chunk(mask, E, e, warp, lane);
        perm[pos] = t;
        inv[(size_t)t * K + k] = pos;
    }
}

size_t permute_ws_bytes(int N, int E)
{
    const size_t chunks = (size_t)(N + kChunk - 1) / kChunk;
    return chunks * E * sizeof(int32_t);
}

kmoe_status launch_permute(const int32_t *idx, int N, int K, int E, int32_t *counts,
                           int32_t *offsets, int32_t *perm, int32_t *inv, int32_t *hist,
                           cudaStream_t st)
{
    const size_t mask_bytes = sizeof(uint32_t) * kChunkWarps * E;
    if (N <= kChunk) {
        const size_t smem = mask_bytes + sizeof(int) * E;
        cudaFuncSetAttribute(permute_single_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        permute_single_kernel<<<1, kChunk, smem, st>>>(idx, N, K, E, counts, offsets, perm, inv);
        return check_launch("permute_single");
    }
    const int chunks = (N + kChunk - 1) / kChunk;
    cudaFuncSetAttribute(chunk_hist_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)mask_bytes);
    cudaFuncSetAttribute(scatter_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)mask_bytes);
    chunk_hist_kernel<<<chunks, kChunk, mask_bytes, st>>>(idx, N, K, E, hist);
    kmoe_status s = check_launch("permute_hist");
    if (s != KMOE_OK) return s;
    scan_kernel<<<1, 1024, 0, st>>>(hist, chunks, E, counts, offsets);
    s = check_launch("permute_scan");
    if (s != KMOE_OK) return s;
    scatter_kernel<<<chunks, kChunk, mask_bytes, st>>>(idx, N, K, E, hist, perm, inv);
    return check_launch("permute_scatter");
}

}  // namespace kmoe
