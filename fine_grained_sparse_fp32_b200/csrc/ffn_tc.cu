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
//   warps 5-8  token producers: the activation rows of the up kernel are
//              gathered with cp.async straight into the swizzled layout (no
//              permuted copy of x is ever written) and complete on the slot
//              barrier without the producer waiting; the down kernel loads H
//              tiles by TMA;
//   warp  9    weight producer: claims the CTA's next tile from a global
//              counter, publishes it to the other roles through a small
//              shared-memory queue, and streams its weight tiles by TMA
//              (128-byte swizzle).
// Token tiles (16 KB per m-tile and k-block) and weight tiles (32 KB per
// k-block) sit in two separate rings (six and three deep), so the weight
// stream runs ahead of the MMA whatever the token gather is doing. Token rows
// are gathered with 8 lanes per 128-byte row segment, and the epilogue goes
// through a per-warp staging area so that its stores also cover whole
// 128-byte segments.
// The up tile pairs 128 gate features with the same 128 up features (one
// N = 256 MMA), so SiLU(g) * u is computed in registers. Tiles are
// enumerated per expert as (row pair, n-tile), so CTAs running at the same
// time share a row pair's token rows in L2, and the weights of an expert with
// several row pairs are kept in L2 (evict-last) for its next row pair.
//
// E4M3 weights ("Inside Kolibri 1", FP8 section: 128 x 128 blocks, one FP32
// scale per block) take the same kernels with eight more warps: warp 9
// brings the E4M3 bytes by TMA into a four-deep staging ring (16 KB per
// k-block), and converter warps 10-17 (one thread per weight row) decode
// them (hardware e4m3x2 -> f16x2), multiply by the FP32 scale of the block,
// round to BF16 and write the swizzled tile the MMA reads. Activations stay BF16, so the tensor cores see BF16 x BF16
// with FP32 accumulation, and the weights cross HBM at one byte each.
#include "common.cuh"
#include "sm100.cuh"
#include "swap_units.cuh"

#include <cudaTypedefs.h>

namespace kmoe {
using namespace sm100;

constexpr int kBM = 128, kBN = 256, kBK = 64;
constexpr int kPairRows = 2 * kBM;           // rows of one CTA tile
constexpr int kATile = kBM * kBK * 2;        // 16 KB: one m-tile of one k-block
constexpr int kBTile = kBN * kBK * 2;        // 32 KB
constexpr int kB8Tile = kBN * kBK;           // 16 KB of E4M3 staging
constexpr int kMaxRing = 6;
constexpr int kSStages = 4;                  // E4M3 staging ring
constexpr int kEpiStage = 4 * 32 * 128;      // epilogue: 32 rows x 128 bytes per warp
__host__ __device__ constexpr int a_stages(bool fp8) { return fp8 ? 4 : 6; }
__host__ __device__ constexpr int b_stages(bool fp8) { return fp8 ? 2 : 3; }
__host__ __device__ constexpr int ring_bytes(bool fp8)
{
    return a_stages(fp8) * kATile + b_stages(fp8) * kBTile + (fp8 ? kSStages * kB8Tile : 0);
}
constexpr int kMmaWarp = 4;
constexpr int kProdWarp = 5;                 // token producers: warps 5-8
constexpr int kWProdWarp = 9;                // weight producer
constexpr int kConvWarp = 10;                // E4M3 only: warps 10-17
constexpr int kConvThreads = 256;            // one converter thread per weight row of a tile
__host__ __device__ constexpr int threads_of(bool fp8) { return (fp8 ? 18 : 10) * 32; }
constexpr int kMaxGroups = 1025;
constexpr int kTQ = 4;                       // tile queue depth
constexpr long long kWaitLimit = kDefaultWaitLimit;   // SM cycles (about 2 s): waits that drain after a give-up

__device__ __forceinline__ void st_shared_v4(uint32_t addr, uint32_t x, uint32_t y, uint32_t z, uint32_t w)
{
    asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(x), "r"(y), "r"(z), "r"(w) : "memory");
}
__device__ __forceinline__ uint4 ld_shared_v4(uint32_t addr)
{
    uint4 v;
    asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(addr)
                 : "memory");
    return v;
}

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
    int *tile_ctr;            // tiles claimed so far by all CTAs (zero at launch)
    int *up_done;             // [groups] up tiles finished per group (zero before the up launch)
    long long wait_limit;     // SM cycles before a pipeline wait gives up
};

struct SmemTail {
    uint64_t afull[kMaxRing], aempty[kMaxRing], bfull[kMaxRing], bempty[kMaxRing];
    uint64_t sfull[kSStages], sempty[kSStages], tfull, tempty[2], drain;
    uint64_t tqfull[kTQ], tqempty[kTQ];
    int tq[kTQ];
    uint32_t tmem_base;
    int abort;
    int pre[kMaxGroups + 1];
};

__host__ __device__ constexpr size_t tc_smem(bool fp8)
{
    return 1024 /*align slack*/ + (size_t)ring_bytes(fp8) + kEpiStage + sizeof(SmemTail);
}
static_assert(tc_smem(false) <= 227 * 1024 && tc_smem(true) <= 227 * 1024, "shared memory budget");

struct Tile {
    int g, row0, rows, n0;
    bool shared, two;     // two: rows > 128 (second m-tile present)
    bool reused;          // the group has several row pairs: its weight tiles are read again
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
    // row pair major, n-tile minor: the n-tiles of one row pair are claimed
    // side by side, so the CTAs running them share its token (or H) rows in L2
    const int mp = local / a.n_tiles, nt = local - mp * a.n_tiles;
    int start, cnt;
    if (T.shared) { start = a.N * a.K; cnt = a.N; }
    else { start = a.offsets[T.g]; cnt = a.offsets[T.g + 1] - start; }
    T.row0 = start + mp * kPairRows;
    T.rows = min(kPairRows, cnt - mp * kPairRows);
    T.two = T.rows > kBM;
    T.reused = pcount > 1;
    T.n0 = nt * bn;
    return T;
}

// Claim order -> tile index. Tiles are claimed dynamically from a global
// counter; the shared expert's tiles (indices routed .. total - 1) are spread
// evenly among the routed ones, so the CTAs running at any time mix
// weight-streaming routed tiles with the shared expert's compute-heavy ones.
__device__ __forceinline__ int claim_to_tile(int c, int routed, int total)
{
    const int S = total - routed;
    const int before = (int)((long long)c * S / total);       // shared tiles among claims 0 .. c-1
    const int upto = (int)((long long)(c + 1) * S / total);
    return upto > before ? routed + before : c - before;
}

// The next tile of this CTA (or -1: no more, -2: a wait gave up), published
// by the weight producer in the tile queue.
__device__ __forceinline__ int tq_take(SmemTail *tail, uint32_t q, volatile int *abort, int *err, long long limit)
{
    const int s = q % kTQ;
    if (!mbar_wait(&tail->tqfull[s], (q / kTQ) & 1, abort, err, limit)) return -2;
    const int t = reinterpret_cast<volatile int *>(tail->tq)[s];
    mbar_arrive(&tail->tqempty[s]);
    return t;
}

// row-pair prefix over groups, computed by one warp.
__device__ __forceinline__ void build_prefix(int *pre, const TcArgs &a)
{
    const int lane = threadIdx.x & 31;
    if (!offsets_ok(a.offsets, a.E, a.N * a.K, a.err)) {   // debug build: no tiles at all
        for (int i = lane; i <= a.groups; i += 32) pre[i] = 0;
        __syncwarp();
        return;
    }
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

// Epilogue of one 128-row half of the accumulator (tile rows rbase ..
// rbase + 127); warp w owns rows rbase + 32w .. + 31, its lane quarter of
// tensor memory, and tbase addresses that quarter in the half. Every 64
// output columns are first written row by row into the warp's 4 KB staging
// area (16-byte pieces XOR-swizzled by row, so neither side has bank
// conflicts) and then stored with 8 lanes per row: each store instruction
// writes four whole 128-byte row segments.
template <bool kUp>
__device__ __forceinline__ void epilogue_half(uint32_t tbase, const Tile &T, const TcArgs &a, int rbase,
                                              uint32_t stage)
{
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int wrow0 = rbase + warp * 32;
    constexpr int kCols = kUp ? kBN / 2 : kBN;       // output columns of the tile
    const uint32_t mine = stage + lane * 128;        // this thread's staging row
    for (int c0 = 0; c0 < kCols; c0 += 64) {
#pragma unroll 1
        for (int q = 0; q < 4; ++q) {                // columns c0 + 16q .. + 15: pieces 2q, 2q + 1
            uint32_t packed[8];
            if (kUp) {
                uint32_t g[16], u[16];
                tmem_ld16(tbase + c0 + 16 * q, g);
                tmem_ld16(tbase + kBN / 2 + c0 + 16 * q, u);
                tmem_ld_wait();
#pragma unroll
                for (int e = 0; e < 8; ++e)
                    packed[e] = pack_bf16x2(silu_mul(__uint_as_float(g[2 * e]), __uint_as_float(u[2 * e])),
                                            silu_mul(__uint_as_float(g[2 * e + 1]), __uint_as_float(u[2 * e + 1])));
            } else {
                uint32_t v[16];
                tmem_ld16(tbase + c0 + 16 * q, v);
                tmem_ld_wait();
#pragma unroll
                for (int e = 0; e < 8; ++e)
                    packed[e] = pack_bf16x2(__uint_as_float(v[2 * e]), __uint_as_float(v[2 * e + 1]));
            }
            st_shared_v4(mine + (((2 * q) ^ (lane & 7)) << 4), packed[0], packed[1], packed[2], packed[3]);
            st_shared_v4(mine + (((2 * q + 1) ^ (lane & 7)) << 4), packed[4], packed[5], packed[6], packed[7]);
        }
        __syncwarp();
#pragma unroll
        for (int j = 0; j < 8; ++j) {                // rows 4j .. 4j + 3 of the warp, 8 lanes each
            const int r = 4 * j + (lane >> 3), pc = lane & 7;
            const uint4 v = ld_shared_v4(stage + r * 128 + ((pc ^ (r & 7)) << 4));
            const int trow = wrow0 + r;
            if (trow < T.rows) {
                const size_t grow = (size_t)T.row0 + trow;
                __nv_bfloat16 *dst = kUp      ? a.out0 + grow * a.I
                                     : T.shared ? a.out1 + (grow - (size_t)a.N * a.K) * a.d
                                                : a.out0 + grow * a.d;
                *reinterpret_cast<uint4 *>(dst + T.n0 + c0 + pc * 8) = v;
            }
        }
        __syncwarp();                                // staging free for the next 64 columns
    }
}

template <bool kUp, bool kFp8>
__global__ void __launch_bounds__(threads_of(kFp8), 1)
ffn_tc_kernel(const __grid_constant__ TcMaps maps, const TcArgs a)
{
    constexpr int kAS = a_stages(kFp8), kBS = b_stages(kFp8);
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t *ring_a = smem;                                   // kAS x 16 KB token tiles
    uint8_t *ring_b = ring_a + (size_t)kAS * kATile;          // kBS x 32 KB BF16 weight tiles
    uint8_t *ring_s = ring_b + (size_t)kBS * kBTile;          // E4M3: kSStages x 16 KB staging
    uint8_t *epi = smem + ring_bytes(kFp8);                   // epilogue staging, 4 KB per warp
    SmemTail *tail = reinterpret_cast<SmemTail *>(epi + kEpiStage);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    volatile int *abort = &tail->abort;

    if (threadIdx.x == 0) {
        for (int s = 0; s < kAS; ++s) {
            mbar_init(&tail->afull[s], kUp ? 128 : 1);    // up: 128 cp.async arrivals; down: TMA expect_tx
            mbar_init(&tail->aempty[s], 1);
        }
        for (int s = 0; s < kBS; ++s) {
            mbar_init(&tail->bfull[s], kFp8 ? kConvThreads : 1);   // E4M3: the converter threads
            mbar_init(&tail->bempty[s], 1);
        }
        for (int s = 0; s < kSStages; ++s) {
            mbar_init(&tail->sfull[s], 1);
            mbar_init(&tail->sempty[s], kConvThreads);
        }
        mbar_init(&tail->tfull, 1);
        mbar_init(&tail->tempty[0], 128);
        mbar_init(&tail->tempty[1], 128);
        mbar_init(&tail->drain, 1);
        for (int s = 0; s < kTQ; ++s) {
            mbar_init(&tail->tqfull[s], 1);
            // readers: token producers (up: 128, down: 1), the MMA thread, 128 epilogue threads, converters
            mbar_init(&tail->tqempty[s], (kUp ? 128 : 1) + 1 + 128 + (kFp8 ? kConvThreads : 0));
        }
        tail->abort = 0;
        fence_mbar_init();
    }
    if (warp == 0) {
        tmem_alloc(&tail->tmem_base, 512);
        tmem_relinquish();
    }
    if (warp == kWProdWarp && lane == 0) {
        prefetch_map(&maps.b0_routed);
        prefetch_map(&maps.b0_shared);
        if (kUp) { prefetch_map(&maps.b1_routed); prefetch_map(&maps.b1_shared); }
        else prefetch_map(&maps.a);
    }
    // The up kernel waits for routing and x. The down kernel does not wait for
    // the whole up grid: its CTAs start on SMs as up CTAs retire, stream W_d
    // at once, and load a row pair's H only after every up tile of that
    // expert has been counted in up_done (release / acquire at GPU scope).
    // Routing itself finished before the up kernel passed its own wait.
    if (kUp) pdl_wait();
    pdl_trigger();
    if (warp == kMmaWarp) build_prefix(tail->pre, a);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();

    const int bn = kUp ? kBN / 2 : kBN;     // output columns per tile
    const int total = tail->pre[a.groups] * a.n_tiles;
    const uint32_t tmem = tail->tmem_base;

    if (kFp8 && warp >= kConvWarp) {
        // ------------------------------------------- E4M3 -> BF16 converters
        const int q = threadIdx.x - kConvWarp * 32;          // row q of the B tile
        uint32_t it = 0;
        bool ok = true;
        for (uint32_t tq = 0; ok; ++tq) {
            const int t = tq_take(tail, tq, abort, a.err, a.wait_limit);
            if (t < 0) break;
            const Tile T = decode_tile(t, tail->pre, a, bn);
            const size_t ge = T.shared ? 0 : (size_t)T.g;
            const float *s0 = T.shared ? a.s0_shared : a.s0_routed;
            const float *s1 = T.shared ? a.s1_shared : a.s1_routed;
            for (int kb = 0; kb < a.kblocks; ++kb, ++it) {
                const int ss = it % kSStages, sb = it % kBS;
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
                if (!mbar_wait(&tail->sfull[ss], (it / kSStages) & 1, abort, a.err, a.wait_limit) ||
                    !mbar_wait(&tail->bempty[sb], ((it / kBS) & 1) ^ 1, abort, a.err, a.wait_limit)) {
                    ok = false;
                    break;
                }
                const uint8_t *B8 = ring_s + (size_t)ss * kB8Tile;
                uint8_t *Bs = ring_b + (size_t)sb * kBTile;
                convert_row(B8 + q * kBK, Bs, q, q < 128 ? sc0 : sc1);
                mbar_arrive(&tail->sempty[ss]);      // staging slot read
                fence_proxy_async();                 // converted rows visible to the tensor cores
                mbar_arrive(&tail->bfull[sb]);
            }
        }
    } else if (warp == kWProdWarp) {
        // ------------------------------------------------- weight producer
        if (lane == 0) {
            const uint64_t pol_w = policy_evict_first();   // routed weight tiles: streamed once
            const uint64_t pol_s = policy_evict_last();    // shared expert: reused by every row pair
            const int routed_tiles = tail->pre[a.E] * a.n_tiles;
            constexpr int S = kFp8 ? kSStages : kBS;
            uint64_t *full = kFp8 ? tail->sfull : tail->bfull;
            uint64_t *empty = kFp8 ? tail->sempty : tail->bempty;
            uint8_t *ring = kFp8 ? ring_s : ring_b;
            constexpr uint32_t bytes = kFp8 ? kB8Tile : kBTile;
            uint32_t it = 0;
            bool ok = true;
            // The next tile is claimed while this tile's last k-blocks are issued
            // (kClaimLead before its end), so the atomic's round trip overlaps
            // the loads instead of sitting between two tiles.
            constexpr int kClaimLead = 2;
            int c_next = atomicAdd(a.tile_ctr, 1);
            for (uint32_t tq = 0; ok; ++tq) {
                const int c = c_next;
                const int t = c < total ? claim_to_tile(c, routed_tiles, total) : -1;
                const int qs = tq % kTQ;
                if (!mbar_wait(&tail->tqempty[qs], ((tq / kTQ) & 1) ^ 1, abort, a.err, a.wait_limit)) {
                    ok = false;
                    break;
                }
                reinterpret_cast<volatile int *>(tail->tq)[qs] = t;
                mbar_arrive(&tail->tqfull[qs]);
                if (t < 0) break;
                const Tile T = decode_tile(t, tail->pre, a, bn);
                // weights read by one row pair are streamed once; an expert with
                // several row pairs (and the shared expert) reads them again
                const uint64_t pol = T.shared || T.reused ? pol_s : pol_w;
                const CUtensorMap *m0 = T.shared ? &maps.b0_shared : &maps.b0_routed;
                const CUtensorMap *m1 = T.shared ? &maps.b1_shared : &maps.b1_routed;
                const int gi = T.shared ? 0 : T.g;
                const int r0 = kUp ? gi * a.I + T.n0 : gi * a.d + T.n0;
                const int claim_at = a.kblocks > kClaimLead ? a.kblocks - 1 - kClaimLead : 0;
                for (int kb = 0; kb < a.kblocks; ++kb, ++it) {
                    if (kb == claim_at) c_next = atomicAdd(a.tile_ctr, 1);
                    const int s = it % S;
                    if (!mbar_wait(&empty[s], ((it / S) & 1) ^ 1, abort, a.err, a.wait_limit)) { ok = false; break; }
                    uint8_t *dst = ring + (size_t)s * bytes;
                    mbar_arrive_expect_tx(&full[s], bytes);
                    // rows 0-127: gate (up) or W_d rows n0..; rows 128-255: up rows n0.. or W_d rows n0+128..
                    tma_load_2d_hint(dst, m0, &full[s], kb * kBK, r0, pol);
                    tma_load_2d_hint(dst + bytes / 2, kUp ? m1 : m0, &full[s], kb * kBK, kUp ? r0 : r0 + kBN / 2,
                                     pol);
                }
            }
            if (!ok)   // let in-flight loads land before the CTA exits
                for (uint32_t j = it > (uint32_t)S ? it - S : 0; j < it; ++j)
                    mbar_wait_drain(&full[j % S], (j / S) & 1, kWaitLimit);
        }
    } else if (warp >= kProdWarp) {
        // -------------------------------------------------- token producers
        const int p = threadIdx.x - kProdWarp * 32;
        const uint64_t pol_a = policy_evict_last();    // token rows / H rows: reused across n-tiles
        uint32_t ia = 0;
        bool ok = true;
        if (kUp) {
            // 8 lanes per row: thread p copies 16-byte piece pc of rows
            // 32 * (p / 32) + 4j + (p % 32) / 8, j = 0..7, so every cp.async
            // instruction of a warp reads four whole 128-byte row segments.
            const int pw = p >> 5, pl = p & 31, pc = pl & 7;
            for (uint32_t tq = 0; ok; ++tq) {
                const int t = tq_take(tail, tq, abort, a.err, a.wait_limit);
                if (t < 0) break;
                const Tile T = decode_tile(t, tail->pre, a, bn);
                int tok0[8], tok1[8];
#pragma unroll
                for (int j = 0; j < 8; ++j) {
                    const int r = pw * 32 + 4 * j + (pl >> 3);
                    tok0[j] = r >= T.rows ? -1
                              : T.shared  ? T.row0 + r - a.N * a.K
                                          : checked_index(a.perm[T.row0 + r], 0, a.N, a.err);
                    tok1[j] = r + kBM >= T.rows ? -1
                              : T.shared        ? T.row0 + kBM + r - a.N * a.K
                                                : checked_index(a.perm[T.row0 + kBM + r], 0, a.N, a.err);
                }
                const int mt = T.two ? 2 : 1;
                for (int kb = 0; kb < a.kblocks && ok; ++kb) {
                    for (int m = 0; m < mt; ++m, ++ia) {
                        const int sa = ia % kAS;
                        if (!mbar_wait(&tail->aempty[sa], ((ia / kAS) & 1) ^ 1, abort, a.err, a.wait_limit)) {
                            ok = false;
                            break;
                        }
                        const uint32_t dst = smem_u32(ring_a + (size_t)sa * kATile);
#pragma unroll
                        for (int j = 0; j < 8; ++j) {
                            const int r = pw * 32 + 4 * j + (pl >> 3);
                            const int tk = m ? tok1[j] : tok0[j];
                            const __nv_bfloat16 *src = a.x + (size_t)(tk < 0 ? 0 : tk) * a.d + kb * kBK + pc * 8;
                            cp_async16_hint(dst + r * 128 + ((pc ^ (r & 7)) << 4), src, tk >= 0 ? 16u : 0u, pol_a);
                        }
                        cp_async_arrive_noinc(&tail->afull[sa]);   // the slot completes when these rows land
                    }
                }
            }
            cp_async_wait_all();   // this thread's row copies have landed before it leaves
        } else if (p == 0) {
            const int up_tiles_per_pair = a.I / (kBN / 2);
            for (uint32_t tq = 0; ok; ++tq) {
                const int t = tq_take(tail, tq, abort, a.err, a.wait_limit);
                if (t < 0) break;
                const Tile T = decode_tile(t, tail->pre, a, bn);
                const int mt = T.two ? 2 : 1;
                // H of this expert is complete once all its up tiles are counted
                const int need = (tail->pre[T.g + 1] - tail->pre[T.g]) * up_tiles_per_pair;
                if (swp::ld_acquire(a.up_done + T.g) < need) {
                    const long long t0 = clock64();
                    while (swp::ld_acquire(a.up_done + T.g) < need) {
                        if (*abort) { ok = false; break; }
                        if (clock64() - t0 > a.wait_limit) {
                            *abort = 1;
                            atomicCAS(a.err, kErrNone, kErrWaitTimeout);
                            ok = false;
                            break;
                        }
                        __nanosleep(128);
                    }
                    if (!ok) break;
                }
                swp::fence_proxy_async_global();   // H written by other CTAs, read by TMA
                for (int kb = 0; kb < a.kblocks && ok; ++kb) {
                    for (int m = 0; m < mt; ++m, ++ia) {
                        const int sa = ia % kAS;
                        if (!mbar_wait(&tail->aempty[sa], ((ia / kAS) & 1) ^ 1, abort, a.err, a.wait_limit)) {
                            ok = false;
                            break;
                        }
                        mbar_arrive_expect_tx(&tail->afull[sa], kATile);
                        tma_load_2d_hint(ring_a + (size_t)sa * kATile, &maps.a, &tail->afull[sa], kb * kBK,
                                         T.row0 + m * kBM, pol_a);
                    }
                }
            }
            if (!ok)
                for (uint32_t j = ia > (uint32_t)kAS ? ia - kAS : 0; j < ia; ++j)
                    mbar_wait_drain(&tail->afull[j % kAS], (j / kAS) & 1, kWaitLimit);
        }
    } else if (warp == kMmaWarp) {
        // ------------------------------------------------------------ MMA
        if (lane == 0) {
            constexpr uint32_t idesc = idesc_bf16_f32(kBM, kBN);
            // Tensor memory holds two 256-column halves. A tile with one
            // m-tile takes the half that the previous single tile did not,
            // so its MMAs overlap that tile's epilogue; a tile with two
            // m-tiles takes both (starting with the half drained first).
            uint32_t ia = 0, ib = 0, use0 = 0, use1 = 0;     // uses of half 0 / half 1 so far
            int hn = 0;
            bool ok = true;
            for (uint32_t tq = 0; ok; ++tq) {
                const int t = tq_take(tail, tq, abort, a.err, a.wait_limit);
                if (t < 0) break;
                const Tile T = decode_tile(t, tail->pre, a, bn);
                const int h0 = hn, h1 = hn ^ 1;
                const uint32_t c0 = h0 ? use1 : use0, c1 = h0 ? use0 : use1;
                const int mt = T.two ? 2 : 1;
                for (int kb = 0; kb < a.kblocks && ok; ++kb, ++ib) {
                    const int sb = ib % kBS;
                    if (!mbar_wait(&tail->bfull[sb], (ib / kBS) & 1, abort, a.err, a.wait_limit)) { ok = false; break; }
                    const uint64_t bd = sw128_kmajor_desc(smem_u32(ring_b + (size_t)sb * kBTile));
                    for (int m = 0; m < mt; ++m, ++ia) {
                        const int sa = ia % kAS, h = m ? h1 : h0;
                        if (!mbar_wait(&tail->afull[sa], (ia / kAS) & 1, abort, a.err, a.wait_limit) ||
                            (kb == 0 &&   // half h drained by the epilogue of its last use
                             !mbar_wait(&tail->tempty[h], ((m ? c1 : c0) & 1) ^ 1, abort, a.err, a.wait_limit))) {
                            ok = false;
                            break;
                        }
                        tc_fence_after();
                        const uint64_t ad = sw128_kmajor_desc(smem_u32(ring_a + (size_t)sa * kATile));
#pragma unroll
                        for (int k = 0; k < kBK / 16; ++k)
                            umma_bf16(tmem + h * kBN, ad + (uint64_t)(k * 2), bd + (uint64_t)(k * 2), idesc,
                                      (kb | k) != 0);
                        umma_commit(&tail->aempty[sa]);
                    }
                    if (ok) umma_commit(&tail->bempty[sb]);
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
        const uint32_t stage = smem_u32(epi) + warp * 4096;
        for (;; ++at) {
            // give-up decisions are votes of the four warps (they meet at a barrier per tile)
            const int tt = tq_take(tail, at, abort, a.err, a.wait_limit);
            const int t = bar_and(1, 128, tt != -2) ? tt : -2;
            if (t < 0) break;
            const Tile T = decode_tile(t, tail->pre, a, bn);
            const int h0 = hn, h1 = hn ^ 1;
            if (!bar_and(1, 128, mbar_wait(&tail->tfull, at & 1, abort, a.err, a.wait_limit))) break;
            tc_fence_after();
            const uint32_t tlane = tmem + ((uint32_t)(warp * 32) << 16);
            epilogue_half<kUp>(tlane + h0 * kBN, T, a, 0, stage);
            tc_fence_before();
            mbar_arrive(&tail->tempty[h0]);
            if (T.two) {
                epilogue_half<kUp>(tlane + h1 * kBN, T, a, kBM, stage);
                tc_fence_before();
                mbar_arrive(&tail->tempty[h1]);
            }
            hn = T.two ? h0 : h1;
            if (kUp) {   // this tile's H rows are stored: count it for its expert
                // the barrier orders the group's stores before thread 0's
                // fence, which publishes them before the count rises
                swp::epi_sync<128>();
                if (threadIdx.x == 0) {
                    __threadfence();
                    swp::red_release_add(a.up_done + T.g, 1);
                }
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
static kmoe_status run_tc(const TcMaps &up, const TcMaps &dn, TcArgs a, int d, int I, int *sync, __nv_bfloat16 *h,
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
    a.tile_ctr = sync;
    a.up_done = sync + 2;
    launch_pdl(ffn_tc_kernel<true, kFp8>, grid, threads_of(kFp8), smem, st, up, a);
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
    a.tile_ctr = sync + 1;
    a.up_done = sync + 2;
    launch_pdl(ffn_tc_kernel<false, kFp8>, grid, threads_of(kFp8), smem, st, dn, a);
    return check_launch("ffn_down_tc");
}

kmoe_status launch_ffn_tc(const __nv_bfloat16 *x, int N, int d, int I, int E, int K, const int32_t *perm,
                          const int32_t *offsets, int w_dtype, const ExpertPtrs &routed, const ExpertPtrs *shared,
                          __nv_bfloat16 *h, __nv_bfloat16 *y_perm, __nv_bfloat16 *y_shared, int *err, int *sync,
                          long long wait_limit, cudaStream_t st)
{
    if (E + 1 > kMaxGroups || E + 3 > kSyncInts) return fail(KMOE_ERR_UNSUPPORTED, "tensor-core FFN: too many experts");
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
    a.wait_limit = wait_limit;
    if (fp8) return run_tc<true>(up, dn, a, d, I, sync, h, y_perm, y_shared, routed, sh, st);
    return run_tc<false>(up, dn, a, d, I, sync, h, y_perm, y_shared, routed, sh, st);
}

}  // namespace kmoe
