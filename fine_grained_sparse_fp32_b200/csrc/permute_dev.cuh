// Device helpers of the dispatch permutation, shared by the permute kernels
// and by the fused small-batch router (which permutes in its last CTA).
//
// Tokens are cut into chunks of 256 (one CTA, 8 warps of 32 tokens). Inside
// a CTA, bit `lane` of mask[w][e] says "token 32*w + lane of this chunk chose
// expert e"; popcounts of those masks give the per-chunk histogram and the
// rank of a token among the earlier tokens of its chunk that chose the same
// expert, so every position is a pure function of the indices.
#pragma once

#include "common.cuh"

namespace kmoe {

constexpr int kChunk = 256;
constexpr int kChunkWarps = kChunk / 32;

// Builds the W x E ballot masks of one chunk of W*32 tokens in shared memory
// (a CTA of W warps, thread i <-> token chunk * W*32 + i).
template <int W = kChunkWarps>
__device__ __forceinline__ void build_masks(const int32_t *__restrict__ idx, int N, int K, int E,
                                            int chunk, uint32_t *mask)
{
    for (int i = threadIdx.x; i < W * E; i += blockDim.x) mask[i] = 0u;
    __syncthreads();
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int t = chunk * W * 32 + threadIdx.x;
    if (t < N) {
        for (int k = 0; k < K; ++k) {
            const int e = idx[(size_t)t * K + k];
            if ((unsigned)e < (unsigned)E) atomicOr(&mask[warp * E + e], 1u << lane);
        }
    }
    __syncthreads();
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

// Rank of token (warp, lane) among the earlier tokens of its chunk that chose e.
__device__ __forceinline__ int rank_in_chunk(const uint32_t *mask, int E, int e, int warp, int lane)
{
    int r = __popc(mask[warp * E + e] & ((1u << lane) - 1u));
    for (int w = 0; w < warp; ++w) r += __popc(mask[w * E + e]);
    return r;
}

// Whole permutation of N <= W*32 tokens by one CTA of W warps.
// `mask` is shared memory of W * E + E 32-bit words.
template <int W = kChunkWarps>
__device__ __forceinline__ void permute_small_block(const int32_t *__restrict__ idx, int N, int K, int E,
                                                    int32_t *__restrict__ counts, int32_t *__restrict__ offsets,
                                                    int32_t *__restrict__ perm, int32_t *__restrict__ inv,
                                                    uint32_t *mask)
{
    __shared__ int tmp[32];
    __shared__ int round_total;
    int *start = reinterpret_cast<int *>(mask + W * E);   // [E]
    build_masks<W>(idx, N, K, E, 0, mask);
    // E may exceed the CTA: scan in rounds of blockDim.x experts.
    int carry = 0;
    for (int e0 = 0; e0 < E; e0 += blockDim.x) {
        const int e = e0 + threadIdx.x;
        int c = 0;
        if (e < E) {
#pragma unroll 8
            for (int w = 0; w < W; ++w) c += __popc(mask[w * E + e]);
        }
        const int excl = block_exclusive_scan(c, tmp);
        if (e < E) {
            counts[e] = c;
            offsets[e] = carry + excl;
            start[e] = carry + excl;
        }
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

}  // namespace kmoe
