// Grouped SwiGLU expert FFN on the 5th-generation tensor cores (tcgen05),
// for batches where experts see many tokens (prefill).
//
// "Inside Kolibri 1" (flozi.net), routing section: each routed or shared
// expert is a SwiGLU MLP (two d -> I projections, SiLU(gate) * up, one
// I -> d projection, no biases). Per expert e with rows X_e (the tokens
// dispatched to it, gathered through perm_token):
//   up kernel   : H_e = SiLU(X_e W_g,e^T) * (X_e W_u,e^T)     [rows, I]
//   down kernel : Y_e = H_e W_d,e^T                           [rows, d]
// Both are persistent, warp-specialised grouped GEMMs (BF16 operands, FP32
// accumulation in tensor memory). A CTA tile is up to 256 rows of one
// expert (two M = 128 m-tiles) by 256 accumulator columns: every 64-column
// weight tile (N = 256 rows) that lands in shared memory feeds both
// m-tiles, into the two 256-column halves of tensor memory, so a weight tile
// crosses HBM and L2 once per expert and n-tile even when the expert's rows
// spill past 128 (at prefill an expert sees ~128 +- 11 tokens).
//   warps 0-3  epilogue: tcgen05.ld of each half, SwiGLU (up) or the BF16
//              cast (down), stores to global memory; a half is handed back
//              to the MMA as soon as it is drained, so the next tile's first
//              MMAs overlap the epilogue of the second half;
//   warp  4    one thread issues tcgen05.mma and tcgen05.commit;
//   warps 5-8  producers: weight tiles by TMA (128-byte swizzle); the
//              activation rows of the up kernel are gathered with cp.async
//              straight into the swizzled layout (no permuted copy of x is
//              ever written) and complete on the stage barrier without the
//              producer waiting; the down kernel loads H tiles by TMA.
// The up tile pairs 128 gate features with the same 128 up features (one
// N = 256 MMA), so SiLU(g) * u is computed in registers. Tiles are
// enumerated per expert as (n-tile, row pair), so CTAs running at the same
// time share the expert's token rows in L2.
//
// E4M3 weights ("Inside Kolibri 1", FP8 section: 128 x 128 blocks, one FP32
// scale per block) take the same kernels with four more warps: the weight
// tile arrives by TMA as E4M3 bytes in a staging buffer, and converter warps
// 9-12 decode it (hardware e4m3x2 -> f16x2), multiply by the FP32 scale of
// its block, round to BF16 and write it in the swizzled layout the MMA reads.
// Activations stay BF16, so the tensor cores see BF16 x BF16 with FP32
// accumulation, and the weights cross HBM at one byte each.
#include "common.cuh"
#include "sm100.cuh"

#include <cudaTypedefs.h>

namespace kmoe {
using namespace sm100;

constexpr int kBM = 128, kBN = 256, kBK = 64;
constexpr int kPairRows = 2 * kBM;           // rows of one CTA tile
constexpr int kATile = kBM * kBK * 2;        // 16 KB per m-tile
constexpr int kBTile = kBN * kBK * 2;        // 32 KB
constexpr int kB8Tile = kBN * kBK;           // 16 KB of E4M3 staging
constexpr int kMaxStages = 3;
__host__ __device__ constexpr int stages_of(bool fp8) { return fp8 ? 2 : 3; }
__host__ __device__ constexpr int stage_bytes(bool fp8) { return 2 * kATile + kBTile + (fp8 ? kB8Tile : 0); }
constexpr int kMmaWarp = 4;
constexpr int kProdWarp = 5;
constexpr int kConvWarp = 9;                 // E4M3 only: warps 9-12
__host__ __device__ constexpr int threads_of(bool fp8) { return (fp8 ? 13 : 9) * 32; }
constexpr int kMaxGroups = 1025;
constexpr long long kWaitLimit = 1LL << 32;  // SM cycles (about 2 s)

struct TcMaps {
    CUtensorMap b0_routed, b1_routed, b0_shared, b1_shared;   // up: gate, up; down: W_d (b0 only)
    CUtensorMap a;                                            // down: H [R, I]
};

struct TcArgs {
    const int32_t *offsets;
    const int32_t *perm;
    const __nv_bfloat16 *x;
    int N, K, E, groups;
    int d, I, kblocks, n_tiles;
    __nv_bfloat16 *out0;      // up: H [R, I]; down: y_perm [N*K, d]
    __nv_bfloat16 *out1;      // down: y_shared [N, d]
    // E4M3 block scales (up: s0 = gate, s1 = up; down: s0 = W_d), routed and shared
    const float *s0_routed, *s1_routed, *s0_shared, *s1_shared;
    int *err;
};

struct SmemTail {
    uint64_t full[kMaxStages], empty[kMaxStages], b8full[kMaxStages], tfull, tempty[2], drain;
    uint32_t tmem_base;
    int abort;
    int pre[kMaxGroups + 1];
};

__host__ __device__ constexpr size_t tc_smem(bool fp8)
{
    return 1024 /*align slack*/ + (size_t)stages_of(fp8) * stage_bytes(fp8) + sizeof(SmemTail);
}

struct Tile {
    int g, row0, rows, n0;
    bool shared, two;     // two: rows > 128 (second m-tile present)
};

__device__ __forceinline__ Tile decode_tile(int t, const int *pre, const TcArgs &a, int bn)
{
    int lo = 1, hi = a.groups;            // smallest j with pre[j] * n_tiles > t
    while (lo < hi) {
        const int mid = (lo + hi) >> 1;
        if (pre[mid] * a.n_tiles > t) hi = mid;
        else lo = mid + 1;
    }
    Tile T;
    T.g = lo - 1;
    T.shared = T.g >= a.E;
    const int pcount = pre[T.g + 1] - pre[T.g];
    const int local = t - pre[T.g] * a.n_tiles;
    const int nt = local / pcount, mp = local - nt * pcount;
    int start, cnt;
    if (T.shared) { start = a.N * a.K; cnt = a.N; }
    else { start = a.offsets[T.g]; cnt = a.offsets[T.g + 1] - start; }
    T.row0 = start + mp * kPairRows;
    T.rows = min(kPairRows, cnt - mp * kPairRows);
    T.two = T.rows > kBM;
    T.n0 = nt * bn;
    return T;
}

// row-pair prefix over groups, computed by one warp.
__device__ __forceinline__ void build_prefix(int *pre, const TcArgs &a)
{
    const int lane = threadIdx.x & 31;
    const int per = (a.groups + 31) / 32;
    const int g0 = lane * per;
    int sum = 0;
    for (int i = 0; i < per; ++i) {
        const int g = g0 + i;
        if (g < a.groups) {
            const int cnt = g < a.E ? a.offsets[g + 1] - a.offsets[g] : a.N;
            sum += (cnt + kPairRows - 1) / kPairRows;
        }
    }
    int incl = sum;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int v = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += v;
    }
    int run = incl - sum;
    for (int i = 0; i < per; ++i) {
        const int g = g0 + i;
        if (g < a.groups) {
            pre[g] = run;
            const int cnt = g < a.E ? a.offsets[g + 1] - a.offsets[g] : a.N;
            run += (cnt + kPairRows - 1) / kPairRows;
        }
    }
    if (lane == 31) pre[a.groups] = incl;
}

// Decodes one 64-element E4M3 row of the staging tile, scales it and writes
// it as BF16 into row r of the 128-byte-swizzled B tile.
__device__ __forceinline__ void convert_row(const uint8_t *src, uint8_t *dst, int r, float scale)
{
#pragma unroll
    for (int c4 = 0; c4 < 4; ++c4) {
        const int c = (c4 + r) & 3;                  // rotate 16-byte reads across banks
        const uint4 q = *reinterpret_cast<const uint4 *>(src + c * 16);
        const uint32_t wds[4] = {q.x, q.y, q.z, q.w};
        uint32_t out[8];
#pragma unroll
        for (int h = 0; h < 4; ++h) {
            __half2_raw lo = __nv_cvt_fp8x2_to_halfraw2(static_cast<__nv_fp8x2_storage_t>(wds[h] & 0xffffu), __NV_E4M3);
            __half2_raw hi = __nv_cvt_fp8x2_to_halfraw2(static_cast<__nv_fp8x2_storage_t>(wds[h] >> 16), __NV_E4M3);
            const float2 a = __half22float2(*reinterpret_cast<__half2 *>(&lo));
            const float2 b = __half22float2(*reinterpret_cast<__half2 *>(&hi));
            out[2 * h] = pack_bf16x2(a.x * scale, a.y * scale);
            out[2 * h + 1] = pack_bf16x2(b.x * scale, b.y * scale);
        }
        // elements c*16 .. c*16+15 = 16-byte chunks 2c and 2c+1 of the BF16 row
        uint8_t *row = dst + r * 128;
        *reinterpret_cast<uint4 *>(row + (((2 * c) ^ (r & 7)) << 4)) = make_uint4(out[0], out[1], out[2], out[3]);
        *reinterpret_cast<uint4 *>(row + (((2 * c + 1) ^ (r & 7)) << 4)) = make_uint4(out[4], out[5], out[6], out[7]);
    }
}

// Epilogue of one 128-row half of the accumulator (rows r_base .. r_base+127
// of the tile). tbase addresses this warp's 32 lanes in that half.
template <bool kUp>
__device__ __forceinline__ void epilogue_half(uint32_t tbase, const Tile &T, const TcArgs &a, int row)
{
    const bool valid = row < T.rows;
    const int grow = T.row0 + row;
    if (kUp) {
        __nv_bfloat16 *dst = a.out0 + (size_t)grow * a.I + T.n0;
#pragma unroll 1
        for (int c = 0; c < kBN / 2; c += 16) {
            uint32_t g[16], u[16];
            tmem_ld16(tbase + c, g);
            tmem_ld16(tbase + kBN / 2 + c, u);
            tmem_ld_wait();
            uint32_t packed[8];
#pragma unroll
            for (int q = 0; q < 8; ++q) {
                const float g0 = __uint_as_float(g[2 * q]), g1 = __uint_as_float(g[2 * q + 1]);
                const float u0 = __uint_as_float(u[2 * q]), u1 = __uint_as_float(u[2 * q + 1]);
                packed[q] = pack_bf16x2(silu_mul(g0, u0), silu_mul(g1, u1));
            }
            if (valid) {
                uint4 *o = reinterpret_cast<uint4 *>(dst + c);
                o[0] = make_uint4(packed[0], packed[1], packed[2], packed[3]);
                o[1] = make_uint4(packed[4], packed[5], packed[6], packed[7]);
            }
        }
    } else {
        __nv_bfloat16 *dst = T.shared ? a.out1 + (size_t)(grow - a.N * a.K) * a.d + T.n0
                                      : a.out0 + (size_t)grow * a.d + T.n0;
#pragma unroll 1
        for (int c = 0; c < kBN; c += 16) {
            uint32_t v[16];
            tmem_ld16(tbase + c, v);
            tmem_ld_wait();
            uint32_t packed[8];
#pragma unroll
            for (int q = 0; q < 8; ++q)
                packed[q] = pack_bf16x2(__uint_as_float(v[2 * q]), __uint_as_float(v[2 * q + 1]));
            if (valid) {
                uint4 *o = reinterpret_cast<uint4 *>(dst + c);
                o[0] = make_uint4(packed[0], packed[1], packed[2], packed[3]);
                o[1] = make_uint4(packed[4], packed[5], packed[6], packed[7]);
            }
        }
    }
}

template <bool kUp, bool kFp8>
__global__ void __launch_bounds__(threads_of(kFp8), 1)
ffn_tc_kernel(const __grid_constant__ TcMaps maps, const TcArgs a)
{
    constexpr int kStages = stages_of(kFp8);
    constexpr int kStage = stage_bytes(kFp8);
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    SmemTail *tail = reinterpret_cast<SmemTail *>(smem + (size_t)kStages * kStage);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    volatile int *abort = &tail->abort;

    if (threadIdx.x == 0) {
        for (int s = 0; s < kStages; ++s) {
            // arrivals: up = 128 cp.async producers + (TMA expect_tx | 128 converters);
            //           down = TMA expect_tx (+ 128 converters)
            mbar_init(&tail->full[s], (kUp ? 128 : 1) + (kFp8 ? 128 : (kUp ? 1 : 0)));
            mbar_init(&tail->empty[s], 1);
            mbar_init(&tail->b8full[s], 1);
        }
        mbar_init(&tail->tfull, 1);
        mbar_init(&tail->tempty[0], 128);
        mbar_init(&tail->tempty[1], 128);
        mbar_init(&tail->drain, 1);
        tail->abort = 0;
        fence_mbar_init();
    }
    if (warp == kMmaWarp) build_prefix(tail->pre, a);
    if (warp == 0) {
        tmem_alloc(&tail->tmem_base, 512);
        tmem_relinquish();
    }
    if (warp == kProdWarp && lane == 0) {
        prefetch_map(&maps.b0_routed);
        prefetch_map(&maps.b0_shared);
        if (kUp) { prefetch_map(&maps.b1_routed); prefetch_map(&maps.b1_shared); }
        else prefetch_map(&maps.a);
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();

    const int bn = kUp ? kBN / 2 : kBN;     // output columns per tile
    const int total = tail->pre[a.groups] * a.n_tiles;
    const uint32_t tmem = tail->tmem_base;

    if (kFp8 && warp >= kConvWarp) {
        // ------------------------------------------- E4M3 -> BF16 converters
        const int q = threadIdx.x - kConvWarp * 32;          // rows q and q + 128 of the B tile
        uint32_t it = 0;
        bool ok = true;
        for (int t = blockIdx.x; t < total && ok; t += gridDim.x) {
            const Tile T = decode_tile(t, tail->pre, a, bn);
            const size_t ge = T.shared ? 0 : (size_t)T.g;
            const float *s0 = T.shared ? a.s0_shared : a.s0_routed;
            const float *s1 = T.shared ? a.s1_shared : a.s1_routed;
            for (int kb = 0; kb < a.kblocks; ++kb, ++it) {
                const int s = it % kStages;
                if (!mbar_wait(&tail->b8full[s], (it / kStages) & 1, abort, a.err, kWaitLimit)) { ok = false; break; }
                uint8_t *Bs = smem + (size_t)s * kStage + 2 * kATile;
                const uint8_t *B8 = Bs + kBTile;
                float sc0, sc1;
                if (kUp) {     // gate rows n0.., up rows n0..; blocks [G, I/128, d/128]
                    const size_t si = (ge * (a.I / 128) + T.n0 / 128) * (a.d / 128) + (kb * kBK) / 128;
                    sc0 = s0[si];
                    sc1 = s1[si];
                } else {       // W_d rows n0.. and n0+128..; blocks [G, d/128, I/128]
                    const size_t si = (ge * (a.d / 128) + T.n0 / 128) * (a.I / 128) + (kb * kBK) / 128;
                    sc0 = s0[si];
                    sc1 = s0[si + a.I / 128];
                }
                convert_row(B8 + q * kBK, Bs, q, sc0);
                convert_row(B8 + (q + 128) * kBK, Bs, q + 128, sc1);
                fence_proxy_async();
                mbar_arrive(&tail->full[s]);
            }
        }
    } else if (warp >= kProdWarp) {
        // ------------------------------------------------------- producers
        const int p = threadIdx.x - kProdWarp * 32;
        const bool leader = p == 0;
        const uint64_t pol_w = policy_evict_first();   // weight tiles: streamed
        const uint64_t pol_a = policy_evict_last();    // token rows / H rows: reused across n-tiles
        uint32_t it = 0;
        bool ok = true;
        for (int t = blockIdx.x; t < total && ok; t += gridDim.x) {
            const Tile T = decode_tile(t, tail->pre, a, bn);
            const CUtensorMap *m0 = T.shared ? &maps.b0_shared : &maps.b0_routed;
            const CUtensorMap *m1 = T.shared ? &maps.b1_shared : &maps.b1_routed;
            const int gi = T.shared ? 0 : T.g;
            int tok0 = -1, tok1 = -1;
            if (kUp) {
                if (p < T.rows) tok0 = T.shared ? T.row0 + p - a.N * a.K : a.perm[T.row0 + p];
                if (p + kBM < T.rows) tok1 = T.shared ? T.row0 + kBM + p - a.N * a.K : a.perm[T.row0 + kBM + p];
            }
            const __nv_bfloat16 *src0 = a.x + (size_t)(tok0 < 0 ? 0 : tok0) * a.d;
            const __nv_bfloat16 *src1 = a.x + (size_t)(tok1 < 0 ? 0 : tok1) * a.d;
            for (int kb = 0; kb < a.kblocks; ++kb, ++it) {
                const int s = it % kStages;
                const uint32_t ph = (it / kStages) & 1;
                if (!mbar_wait(&tail->empty[s], ph ^ 1, abort, a.err, kWaitLimit)) { ok = false; break; }
                uint8_t *As = smem + (size_t)s * kStage;           // A0 | A1 | B | (B8)
                uint8_t *Bs = As + 2 * kATile;
                if (kFp8 && leader) {       // E4M3 weight rows into the staging buffer
                    uint8_t *B8 = Bs + kBTile;
                    const int r0 = kUp ? gi * a.I + T.n0 : gi * a.d + T.n0;
                    mbar_arrive_expect_tx(&tail->b8full[s], kB8Tile);
                    tma_load_2d_hint(B8, m0, &tail->b8full[s], kb * kBK, r0, pol_w);
                    tma_load_2d_hint(B8 + kB8Tile / 2, kUp ? m1 : m0, &tail->b8full[s], kb * kBK,
                                     kUp ? r0 : r0 + kBN / 2, pol_w);
                }
                if (kUp) {
                    if (leader && !kFp8) {
                        mbar_arrive_expect_tx(&tail->full[s], kBTile);
                        tma_load_2d_hint(Bs, m0, &tail->full[s], kb * kBK, gi * a.I + T.n0, pol_w);
                        tma_load_2d_hint(Bs + kBTile / 2, m1, &tail->full[s], kb * kBK, gi * a.I + T.n0, pol_w);
                    }
                    const uint32_t dst0 = smem_u32(As) + p * 128;
#pragma unroll
                    for (int c = 0; c < 8; ++c)
                        cp_async16_hint(dst0 + ((c ^ (p & 7)) << 4), src0 + kb * kBK + c * 8, tok0 >= 0 ? 16u : 0u,
                                        pol_a);
                    if (T.two) {
                        const uint32_t dst1 = smem_u32(As + kATile) + p * 128;
#pragma unroll
                        for (int c = 0; c < 8; ++c)
                            cp_async16_hint(dst1 + ((c ^ (p & 7)) << 4), src1 + kb * kBK + c * 8,
                                            tok1 >= 0 ? 16u : 0u, pol_a);
                    }
                    cp_async_arrive_noinc(&tail->full[s]);   // the stage completes when these rows land
                } else if (leader) {
                    mbar_arrive_expect_tx(&tail->full[s], kATile * (T.two ? 2 : 1) + (kFp8 ? 0 : kBTile));
                    tma_load_2d_hint(As, &maps.a, &tail->full[s], kb * kBK, T.row0, pol_a);
                    if (T.two) tma_load_2d_hint(As + kATile, &maps.a, &tail->full[s], kb * kBK, T.row0 + kBM, pol_a);
                    if (!kFp8) {
                        tma_load_2d_hint(Bs, m0, &tail->full[s], kb * kBK, gi * a.d + T.n0, pol_w);
                        tma_load_2d_hint(Bs + kBTile / 2, m0, &tail->full[s], kb * kBK, gi * a.d + T.n0 + kBN / 2,
                                         pol_w);
                    }
                }
            }
        }
        if (kUp) cp_async_wait_all();   // this thread's row copies have landed before it leaves
        if (!ok && leader) {   // let in-flight TMA loads land before the CTA exits
            for (uint32_t j = it > (uint32_t)kStages ? it - kStages : 0; j < it; ++j) {
                if (kFp8) mbar_wait_drain(&tail->b8full[j % kStages], (j / kStages) & 1, kWaitLimit);
                if (!kFp8 || !kUp) mbar_wait_drain(&tail->full[j % kStages], (j / kStages) & 1, kWaitLimit);
            }
        }
    } else if (warp == kMmaWarp) {
        // ------------------------------------------------------------ MMA
        if (lane == 0) {
            constexpr uint32_t idesc = idesc_bf16_f32(kBM, kBN);
            // Tensor memory holds two 256-column halves. A tile with one
            // m-tile takes the half that the previous single tile did not,
            // so its MMAs overlap that tile's epilogue; a tile with two
            // m-tiles takes both (starting with the half drained first).
            uint32_t it = 0, use0 = 0, use1 = 0;     // uses of half 0 / half 1 so far
            int hn = 0;
            bool ok = true;
            for (int t = blockIdx.x; t < total && ok; t += gridDim.x) {
                const Tile T = decode_tile(t, tail->pre, a, bn);
                const int h0 = hn, h1 = hn ^ 1;
                const uint32_t c0 = h0 ? use1 : use0, c1 = h0 ? use0 : use1;
                for (int kb = 0; kb < a.kblocks; ++kb, ++it) {
                    const int s = it % kStages;
                    if (!mbar_wait(&tail->full[s], (it / kStages) & 1, abort, a.err, kWaitLimit)) { ok = false; break; }
                    if (kb == 0 &&   // half h0 drained by the epilogue of its last use
                        !mbar_wait(&tail->tempty[h0], (c0 & 1) ^ 1, abort, a.err, kWaitLimit)) { ok = false; break; }
                    tc_fence_after();
                    const uint32_t sa = smem_u32(smem + (size_t)s * kStage);
                    const uint64_t a0 = sw128_kmajor_desc(sa);
                    const uint64_t bd = sw128_kmajor_desc(sa + 2 * kATile);
#pragma unroll
                    for (int k = 0; k < kBK / 16; ++k)
                        umma_bf16(tmem + h0 * kBN, a0 + (uint64_t)(k * 2), bd + (uint64_t)(k * 2), idesc, (kb | k) != 0);
                    if (T.two) {
                        if (kb == 0 &&
                            !mbar_wait(&tail->tempty[h1], (c1 & 1) ^ 1, abort, a.err, kWaitLimit)) { ok = false; break; }
                        tc_fence_after();
                        const uint64_t a1 = sw128_kmajor_desc(sa + kATile);
#pragma unroll
                        for (int k = 0; k < kBK / 16; ++k)
                            umma_bf16(tmem + h1 * kBN, a1 + (uint64_t)(k * 2), bd + (uint64_t)(k * 2), idesc,
                                      (kb | k) != 0);
                    }
                    umma_commit(&tail->empty[s]);
                }
                if (!ok) break;
                umma_commit(&tail->tfull);
                const uint32_t inc1 = T.two ? 1u : 0u;    // half h0 always, h1 for two m-tiles
                if (h0) { ++use1; use0 += inc1; } else { ++use0; use1 += inc1; }
                hn = T.two ? h0 : h1;
            }
            umma_commit(&tail->drain);     // every MMA done before tensor memory is released
            mbar_wait_drain(&tail->drain, 0, kWaitLimit);
        }
        __syncwarp();
    } else {
        // ------------------------------------------------------- epilogue
        uint32_t at = 0;
        int hn = 0;                       // the half rotation of the MMA thread, replayed
        const int row = warp * 32 + lane;
        for (int t = blockIdx.x; t < total; t += gridDim.x, ++at) {
            const Tile T = decode_tile(t, tail->pre, a, bn);
            const int h0 = hn, h1 = hn ^ 1;
            if (!mbar_wait(&tail->tfull, at & 1, abort, a.err, kWaitLimit)) break;
            tc_fence_after();
            const uint32_t tlane = tmem + ((uint32_t)(warp * 32) << 16);
            epilogue_half<kUp>(tlane + h0 * kBN, T, a, row);
            tc_fence_before();
            mbar_arrive(&tail->tempty[h0]);
            if (T.two) {
                epilogue_half<kUp>(tlane + h1 * kBN, T, a, row + kBM);
                tc_fence_before();
                mbar_arrive(&tail->tempty[h1]);
            }
            hn = T.two ? h0 : h1;
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, 512);
    }
}

// ------------------------------------------------------------------- host
static PFN_cuTensorMapEncodeTiled_v12000 encode_fn()
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

// 2D BF16 map over a row-major [rows, cols] matrix, box 128 rows x 64 columns
// (128 bytes), 128-byte swizzle; reads outside the matrix return zeros.
static bool make_map(CUtensorMap *m, const void *base, uint64_t rows, uint64_t cols)
{
    auto fn = encode_fn();
    if (!fn) return false;
    cuuint64_t dims[2] = {cols, rows};
    cuuint64_t strides[1] = {cols * 2};
    cuuint32_t box[2] = {kBK, 128};
    cuuint32_t estr[2] = {1, 1};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(base), dims, strides, box, estr,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// 2D byte map (E4M3 weights) over [rows, cols], box 128 rows x 64 bytes, no
// swizzle (the converter warps read it with plain shared-memory loads).
static bool make_map_u8(CUtensorMap *m, const void *base, uint64_t rows, uint64_t cols)
{
    auto fn = encode_fn();
    if (!fn) return false;
    cuuint64_t dims[2] = {cols, rows};
    cuuint64_t strides[1] = {cols};
    cuuint32_t box[2] = {kBK, 128};
    cuuint32_t estr[2] = {1, 1};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void *>(base), dims, strides, box, estr,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

static int sm_count_tc()
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

template <bool kFp8>
static kmoe_status run_tc(const TcMaps &up, const TcMaps &dn, TcArgs a, int d, int I, __nv_bfloat16 *h,
                          __nv_bfloat16 *y_perm, __nv_bfloat16 *y_shared, const ExpertPtrs &routed,
                          const ExpertPtrs &sh, cudaStream_t st)
{
    const int grid = sm_count_tc();
    constexpr size_t smem = tc_smem(kFp8);
    cudaFuncSetAttribute(ffn_tc_kernel<true, kFp8>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    cudaFuncSetAttribute(ffn_tc_kernel<false, kFp8>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    a.kblocks = d / kBK;
    a.n_tiles = I / (kBN / 2);
    a.out0 = h;
    a.s0_routed = routed.sg;
    a.s1_routed = routed.su;
    a.s0_shared = sh.sg;
    a.s1_shared = sh.su;
    ffn_tc_kernel<true, kFp8><<<grid, threads_of(kFp8), smem, st>>>(up, a);
    kmoe_status s = check_launch("ffn_up_tc");
    if (s != KMOE_OK) return s;
    a.kblocks = I / kBK;
    a.n_tiles = d / kBN;
    a.out0 = y_perm;
    a.out1 = y_shared;
    a.s0_routed = routed.sd;
    a.s1_routed = nullptr;
    a.s0_shared = sh.sd;
    a.s1_shared = nullptr;
    ffn_tc_kernel<false, kFp8><<<grid, threads_of(kFp8), smem, st>>>(dn, a);
    return check_launch("ffn_down_tc");
}

kmoe_status launch_ffn_tc(const __nv_bfloat16 *x, int N, int d, int I, int E, int K, const int32_t *perm,
                          const int32_t *offsets, int w_dtype, const ExpertPtrs &routed, const ExpertPtrs *shared,
                          __nv_bfloat16 *h, __nv_bfloat16 *y_perm, __nv_bfloat16 *y_shared, int *err,
                          cudaStream_t st)
{
    if (E + 1 > kMaxGroups) return fail(KMOE_ERR_UNSUPPORTED, "tensor-core FFN: too many experts");
    const bool fp8 = w_dtype == KMOE_E4M3_B128;
    const ExpertPtrs sh = shared ? *shared : routed;    // unused maps still need a valid base
    const long long R = (long long)N * K + N;
    auto wmap = [&](CUtensorMap *m, const void *base, uint64_t rows, uint64_t cols) {
        return fp8 ? make_map_u8(m, base, rows, cols) : make_map(m, base, rows, cols);
    };
    TcMaps up{}, dn{};
    bool ok = wmap(&up.b0_routed, routed.wg, (uint64_t)E * I, d) && wmap(&up.b1_routed, routed.wu, (uint64_t)E * I, d) &&
              wmap(&up.b0_shared, sh.wg, I, d) && wmap(&up.b1_shared, sh.wu, I, d) && make_map(&up.a, h, R, I) &&
              wmap(&dn.b0_routed, routed.wd, (uint64_t)E * d, I) && wmap(&dn.b0_shared, sh.wd, d, I) &&
              wmap(&dn.b1_routed, routed.wd, (uint64_t)E * d, I) && wmap(&dn.b1_shared, sh.wd, d, I) &&
              make_map(&dn.a, h, R, I);
    if (!ok) return fail(KMOE_ERR_CUDA, "cuTensorMapEncodeTiled failed");
    TcArgs a{};
    a.offsets = offsets;
    a.perm = perm;
    a.x = x;
    a.N = N;
    a.K = K;
    a.E = E;
    a.groups = E + (shared ? 1 : 0);
    a.d = d;
    a.I = I;
    a.err = err;
    if (fp8) return run_tc<true>(up, dn, a, d, I, h, y_perm, y_shared, routed, sh, st);
    return run_tc<false>(up, dn, a, d, I, h, y_perm, y_shared, routed, sh, st);
}

}  // namespace kmoe
