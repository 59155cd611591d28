// Grouped SwiGLU expert FFN on the tcgen05 tensor cores with the weights as
// the M operand ("swap-AB").
//
// "Inside Kolibri 1" (flozi.net), routing section: every routed or shared
// expert is a SwiGLU MLP (two d -> I projections, SiLU(gate) * up, one
// I -> d projection, no biases). Each selected expert's 3*d*I weights cross
// HBM once and meet the expert's token rows; at decode one or two rows, so
// the layer is a weight stream. This kernel serves batches below 256 tokens
// (prefill batches take the tokens-as-M kernel in ffn_tc.cu).
//
// A 128-row weight tile is the MMA's A operand (M = 128, streamed by TMA in
// 128-byte column stages) and a chunk of the expert's token rows is its B
// operand, with N = the chunk's rows rounded up to 16 (chunks of at most
// kNT = 16 rows are compiled). Work units:
//   up unit   (expert, 128 intermediate features, token chunk): the gate rows
//             and the up rows of those features are two A tiles multiplied
//             by the same B; gate and up accumulate side by side in tensor
//             memory, so the thread holding a feature's accumulator lane
//             has both and writes H = SiLU(gate) * up;
//   down unit (expert, 256 output features, token chunk): two A tiles of
//             128 W_d rows each against the chunk's H rows (B), so a stage
//             carries as many weight bytes as an up unit's.
// One persistent launch runs every up unit, then every down unit. A
// scheduler warp claims units from a global counter, resolves each one into
// a shared-memory slot (rows, weight rows, scales) and, before a down unit,
// waits (bounded) until all up units of that expert have published H.
//
// Warp roles (one CTA per SM):
//   warps 0-3  epilogue: tcgen05.ld of the accumulators, SwiGLU or the BF16
//              cast, global stores; hands the accumulator back to the MMA
//              (with chunks above 32 rows, warps 7-10 form a second group);
//   warp  4    one thread issues tcgen05.mma / tcgen05.commit;
//   warp  5    producer: TMA loads of the weight tiles (lane 0), cp.async
//              gathers of the token (or H) rows (all lanes);
//   warp  6    scheduler.
// BF16 weights only: small batches with E4M3 weights run on the FP8 tensor
// cores (ffn_a8.cu, two-term activations).
#include "common.cuh"
#include "sm100.cuh"
#include "swap_units.cuh"

#include <cudaTypedefs.h>

namespace kmoe {
using namespace sm100;

namespace swp {

constexpr int kM = 128;                 // weight rows per tile (MMA M)
constexpr int kATile = kM * 128;        // 16 KB: 128 rows x 128 bytes
constexpr int kNU = 8;                  // unit-info slots
constexpr long long kWaitLimit = kDefaultWaitLimit;   // SM cycles, about 2 s: waits that drain after a give-up
constexpr int kSmemLimit = 232448;            // 227 KB per CTA

// Per configuration: kNT = token rows per unit at most (16 are compiled).
template <int kNT>
struct Cfg {
    static constexpr int BK = 64;                        // k per stage
    static constexpr int Panel = kNT * 128;              // one 64-column panel of a B tile
    static constexpr int BTile = kNT * BK * 2;           // token rows of a stage (16-bit)
    static constexpr int Stage = 2 * kATile + BTile;     // gate | up (or W_d) | tokens
    static constexpr int AccW = 2 * kNT;                 // accumulator slot: gate | up
    static constexpr int NAcc = 256 / kNT < 4 ? 256 / kNT : 4;
    static constexpr int AccCols = NAcc * AccW;
    static constexpr int TmemCols = AccCols <= 128 ? 128 : AccCols <= 256 ? 256 : 512;
    static constexpr int Stages = kNT <= 16 ? 6 : 4;
    static constexpr int Ring = Stages * Stage;
    static constexpr int EpiGroups = kNT > 32 ? 2 : 1;   // groups of four epilogue warps
    static constexpr int Warps = EpiGroups == 2 ? 11 : 7;
    static constexpr int EpiThreads = 128 * EpiGroups;
    static constexpr int W = kNT < 32 ? kNT : 32;        // accumulator columns an epilogue warp loads at once
    static_assert(kNT % 16 == 0 && kNT >= 16 && kNT <= 128, "token chunk");
    static_assert(AccCols <= TmemCols && TmemCols <= 512, "tensor memory columns");
};

// Warps 0-3 (and 7-10 when EpiGroups == 2) run the epilogue.
constexpr int kMmaWarp = 4, kProdWarp = 5, kSchedWarp = 6, kEpi2Warp = 7;

// A unit as the scheduler warp resolved it: everything the other roles need,
// so that none of them touches global memory to set a unit up.
template <int kNT>
struct Slot {
    int u;                   // unit index, -1 = no more work
    int up, shared, o;       // kind, shared expert, position in the group order
    int f0, mc, nmma, kb;    // first feature, token rows, MMA N, stages
    int row0;                // first dispatched row of the chunk
    int wrow;                // first weight row in the stacked weight matrix
    int src[kNT];            // B row n: token (up) or dispatched row (down), n < mc
};

template <int kNT>
struct Tail {
    uint64_t full[6], empty[6];          // weight + token ring (Stages <= 6)
    uint64_t ufull[kNU], uempty[kNU];
    uint64_t tfull[4], tempty[4];
    uint64_t drain, pstart;              // pstart: the producer has started a unit
    uint32_t tmem_base;
    int abort;
    Slot<kNT> slot[kNU];
    alignas(16) uint16_t stage[8][16][32];   // epilogue transposes (16-byte reads): 16 tokens x 32 features per warp
    int pre[kMaxOrd + 1];        // token-chunk prefix over the group order
    int off[kMaxOrd + 1];        // copy of the routed groups' row offsets
};

static_assert(offsetof(Tail<16>, stage) % 16 == 0 && offsetof(Tail<128>, stage) % 16 == 0, "16-byte staging");
static_assert(sizeof(Tail<16>) % 16 == 0 && sizeof(Tail<128>) % 16 == 0, "tail size");

template <int kNT>
__host__ __device__ constexpr size_t smem_bytes()
{
    return 1024 + (size_t)Cfg<kNT>::Ring + sizeof(Tail<kNT>);
}

struct Maps {
    CUtensorMap g_r, u_r, g_s, u_s;   // up: gate / up rows
    CUtensorMap d_r, d_s;             // down: W_d rows (boxes of 128 rows x 128 bytes)
    CUtensorMap xg;                   // x [N, d]: boxes of 1 row x 64 columns (gathered four at a time)
    CUtensorMap hb;                   // H [N*K + N, I]: boxes of kNT rows x 64 columns
};

struct Args {
    const __nv_bfloat16 *x;           // [N, d]
    const int32_t *perm, *offsets;
    __nv_bfloat16 *h;                 // [N*K + N, I]
    __nv_bfloat16 *y_perm, *y_shared;
    int *err;                         // device status word
    int *claim;                       // unit counter (zero at launch)
    int *up_done;                     // [groups] finished up units (zero at launch)
    long long wait_limit;             // SM cycles before a pipeline wait gives up
    int N, K, E, d, I, has_shared, n_ord;
    int sk;                           // k per stage
    int nt;                           // token rows per unit at most
};

// Instruction descriptor of tcgen05.mma kind::f16: A and B both BF16
// (K-major), FP32 accumulator, M x N.
__host__ __device__ constexpr uint32_t idesc_bf16(int M, int N)
{
    return (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}

}  // namespace swp

using namespace swp;

template <int kNT>
__global__ void __launch_bounds__(Cfg<kNT>::Warps * 32, 1)
ffn_swap_kernel(const __grid_constant__ Maps maps, const Args a)
{
    using C = Cfg<kNT>;
    constexpr int SA = C::Stages;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    Tail<kNT> *T = reinterpret_cast<Tail<kNT> *>(smem + C::Ring);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    volatile int *abort = &T->abort;

    if (threadIdx.x == 0) {
        for (int s = 0; s < SA; ++s) {
            mbar_init(&T->full[s], 1);                   // TMA expect_tx (weights and token rows)
            mbar_init(&T->empty[s], 1);                  // tcgen05.commit
        }
        for (int j = 0; j < kNU; ++j) {
            mbar_init(&T->ufull[j], 1);
            mbar_init(&T->uempty[j], 1);
        }
        for (int c = 0; c < C::NAcc; ++c) {
            mbar_init(&T->tfull[c], 1);
            mbar_init(&T->tempty[c], C::EpiThreads);
        }
        mbar_init(&T->drain, 1);
        mbar_init(&T->pstart, 1);
        T->abort = 0;
        fence_mbar_init();
    }
    if (warp == 0) {
        tmem_alloc(&T->tmem_base, C::TmemCols);
        tmem_relinquish();
    }
    if (warp == kProdWarp && lane == 0) {
        prefetch_map(&maps.g_r); prefetch_map(&maps.u_r); prefetch_map(&maps.d_r);
        if (a.has_shared) { prefetch_map(&maps.g_s); prefetch_map(&maps.u_s); prefetch_map(&maps.d_s); }
        prefetch_map(&maps.xg); prefetch_map(&maps.hb);
    }
    pdl_wait();               // routing (offsets, permutation) and x come from earlier kernels
    pdl_trigger();
    if (warp == kSchedWarp) build_prefix(T->pre, T->off, a);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = T->tmem_base;

    if (warp == kSchedWarp) {
        // ----------------------------------------------------------- scheduler
        // Claims units one ahead, resolves each into a slot and, for a down
        // unit, waits until the expert's up units have published H. Runs up
        // to kNU units ahead of the epilogue, so its global-memory round trips
        // overlap the weight stream.
        // A unit is claimed only once the producer has started the previous
        // one, so a CTA never holds work that it will reach much later (a
        // down unit claimed by anyone waits on the up units the others hold).
        const int total = total_units(T->pre, a);
        for (int us = 0;; ++us) {
            const int j = us % kNU;
            if (!mbar_wait(&T->uempty[j], ((us / kNU) & 1) ^ 1, abort, a.err, a.wait_limit)) break;
            if (us > 0 && !mbar_wait(&T->pstart, (us - 1) & 1, abort, a.err, a.wait_limit)) break;
            int u = 0;
            if (lane == 0) u = atomicAdd(a.claim, 1);
            u = __shfl_sync(0xffffffffu, u, 0);
            if (u >= total) u = -1;
            Slot<kNT> &sl = T->slot[j];
            if (u < 0) {
                if (lane == 0) {
                    sl.u = -1;
                    mbar_arrive(&T->ufull[j]);
                }
                break;
            }
            const Unit U = decode(u, T->pre, T->off, a);
            const int row0 = U.G.row0 + U.m0;
            // every global load of the unit is issued before any is used: one round trip
            constexpr int RPL = (kNT + 31) / 32;         // rows per lane
            int srcv[RPL];
#pragma unroll
            for (int i = 0; i < RPL; ++i) {
                const int n = lane + 32 * i;
                srcv[i] = 0;
                if (n < U.mc)
                    srcv[i] = U.up ? (U.G.shared ? row0 + n - a.N * a.K : checked_index(a.perm[row0 + n], 0, a.N, a.err))
                                   : row0 + n;
            }
            const int need = (a.I / kF) * chunks_of(U.G.rows, a.nt);
            int done = need;
            if (!U.up && lane == 0) done = ld_acquire(a.up_done + U.o);
#pragma unroll
            for (int i = 0; i < RPL; ++i)
                if (lane + 32 * i < U.mc) sl.src[lane + 32 * i] = srcv[i];
            bool good = true;
            if (lane == 0 && done < need) {       // the expert's H rows come from up units of any CTA
                const long long t0 = clock64();
                while (ld_acquire(a.up_done + U.o) < need) {
                    if (*abort) { good = false; break; }
                    if (clock64() - t0 > a.wait_limit) {
                        *abort = 1;
                        atomicCAS(a.err, kErrNone, kErrWaitTimeout);
                        good = false;
                        break;
                    }
                    __nanosleep(64);
                }
            }
            if (!__shfl_sync(0xffffffffu, good ? 1 : 0, 0)) break;
            if (lane == 0) {
                sl.u = u;
                sl.up = U.up;
                sl.shared = U.G.shared;
                sl.o = U.o;
                sl.f0 = U.f0;
                sl.mc = U.mc;
                sl.nmma = U.nmma;
                sl.kb = U.kb;
                sl.row0 = row0;
                const int gi = U.G.shared ? 0 : U.G.g;
                sl.wrow = U.up ? gi * a.I + U.f0 : gi * a.d + U.f0;
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&T->ufull[j]);
        }
    } else if (warp == kProdWarp) {
        // ------------------------------------------------------------ producer
        // Weight tiles (lane 0) and token tiles all by TMA: a down unit's H
        // rows are contiguous (one box of kNT rows per 64-column panel); an
        // up unit's token rows are gathered four at a time (lane i: rows
        // 4i .. 4i+3), rows past the chunk repeating its first row.
        const uint64_t pol_w = policy_evict_first();    // weights: streamed once
        const uint64_t pol_a = policy_evict_last();     // token / H rows: reused by many units
        constexpr int NP = C::BK / 64;                  // 64-column panels per stage
        uint32_t it = 0;
        bool ok = true;
        for (int us = 0;; ++us) {
            const int j = us % kNU;
            if (!mbar_wait(&T->ufull[j], (us / kNU) & 1, abort, a.err, a.wait_limit)) { ok = false; break; }
            const Slot<kNT> &sl = T->slot[j];
            if (sl.u < 0) break;
            const bool up = sl.up, shared = sl.shared;
            const int kb_n = sl.kb, wrow = sl.wrow, mc = sl.mc, nmma = sl.nmma, r0 = sl.row0;
            const bool gl = up && 4 * lane < nmma;       // this lane gathers four token rows
            int gr[4];
#pragma unroll
            for (int q = 0; q < 4; ++q) gr[q] = 4 * lane + q < mc ? sl.src[4 * lane + q] : sl.src[0];
            __syncwarp();
            if (lane == 0) mbar_arrive(&T->pstart);
            if (!up) fence_proxy_async_global();        // H written by other CTAs, seen through the scheduler
            const CUtensorMap *m0 = up ? (shared ? &maps.g_s : &maps.g_r) : (shared ? &maps.d_s : &maps.d_r);
            const CUtensorMap *m1 = shared ? &maps.u_s : &maps.u_r;
            const uint32_t bbytes = (uint32_t)(up ? nmma : kNT) * 128 * NP;
            for (int kb = 0; kb < kb_n; ++kb, ++it) {
                const int s = it % SA;
                if (!mbar_wait(&T->empty[s], ((it / SA) & 1) ^ 1, abort, a.err, a.wait_limit)) { ok = false; break; }
                uint8_t *A = smem + (size_t)s * C::Stage;
                uint8_t *B = A + 2 * kATile;
                if (lane == 0) {
                    mbar_arrive_expect_tx(&T->full[s], 2 * kATile + bbytes);
                    tma_load_2d_hint(A, m0, &T->full[s], kb * C::BK, wrow, pol_w);
                    // second tile: the up rows of the same features, or the next 128 W_d rows
                    tma_load_2d_hint(A + kATile, up ? m1 : m0, &T->full[s], kb * C::BK, up ? wrow : wrow + kM, pol_w);
                    if (!up)
#pragma unroll
                        for (int p = 0; p < NP; ++p)
                            tma_load_2d_hint(B + p * C::Panel, &maps.hb, &T->full[s], kb * C::BK + p * 64, r0, pol_a);
                }
                __syncwarp();
                if (gl)
#pragma unroll
                    for (int p = 0; p < NP; ++p)
                        tma_gather4_hint(B + p * C::Panel + lane * 512, &maps.xg, &T->full[s], kb * C::BK + p * 64,
                                         gr[0], gr[1], gr[2], gr[3], pol_a);
            }
            if (!ok) break;
        }
        if (!ok && lane == 0)    // let in-flight TMA loads land before the CTA exits
            for (uint32_t j = it > (uint32_t)SA ? it - SA : 0; j < it; ++j)
                mbar_wait_drain(&T->full[j % SA], (j / SA) & 1, kWaitLimit);
    } else if (warp == kMmaWarp) {
        // ----------------------------------------------------------------- MMA
        if (lane == 0) {
            uint32_t it = 0;
            for (int us = 0;; ++us) {
                const int j = us % kNU;
                if (!mbar_wait(&T->ufull[j], (us / kNU) & 1, abort, a.err, a.wait_limit)) break;
                const Slot<kNT> &sl = T->slot[j];
                if (sl.u < 0) break;
                const bool up = sl.up;
                const int kb_n = sl.kb;
                const int acc = us % C::NAcc;
                if (!mbar_wait(&T->tempty[acc], ((us / C::NAcc) & 1) ^ 1, abort, a.err, a.wait_limit)) break;
                tc_fence_after();
                const uint32_t dg = tmem + acc * C::AccW;          // gate (or W_d) accumulator
                const uint32_t du = dg + kNT;                      // up accumulator
                const uint32_t id = idesc_bf16(kM, sl.nmma);
                bool ok = true;
                for (int kb = 0; kb < kb_n; ++kb, ++it) {
                    const int s = it % SA;
                    if (!mbar_wait(&T->full[s], (it / SA) & 1, abort, a.err, a.wait_limit)) { ok = false; break; }
                    tc_fence_after();
                    const uint32_t sa = smem_u32(smem + (size_t)s * C::Stage);
                    const uint64_t a0 = sw128_kmajor_desc(sa), a1 = sw128_kmajor_desc(sa + kATile);
                    const uint64_t bd = sw128_kmajor_desc(sa + 2 * kATile);
                    // all k-steps of one accumulator before the other: an MMA
                    // that switches accumulators costs nearly twice as much
#pragma unroll
                    for (int k = 0; k < C::BK / 16; ++k)
                        umma_bf16(dg, a0 + (uint64_t)(k * 2), bd + (uint64_t)(k * 2), id, (kb | k) != 0);
#pragma unroll
                    for (int k = 0; k < C::BK / 16; ++k)
                        umma_bf16(du, a1 + (uint64_t)(k * 2), bd + (uint64_t)(k * 2), id, (kb | k) != 0);
                    umma_commit(&T->empty[s]);
                }
                if (!ok) break;
                umma_commit(&T->tfull[acc]);
            }
            umma_commit(&T->drain);     // every MMA done before tensor memory is released
            mbar_wait_drain(&T->drain, 0, kWaitLimit);
        }
        __syncwarp();
    } else if (warp < 4 || (C::EpiGroups == 2 && warp >= kEpi2Warp)) {
        // ------------------------------------------------------------ epilogue
        // A warp reads its quadrant of accumulator lanes (32 features of the
        // unit), W token columns at a time; group eg takes every EpiGroups-th
        // block. Results go through a 16 x 32 shared-memory transpose so that
        // each global store writes 16 bytes (8 features of one token).
        constexpr int W = C::W;
        const int quad = warp & 3, eg = warp < 4 ? 0 : 1;
        uint16_t *stg = &T->stage[eg * 4 + quad][0][0];
        for (int us = 0;; ++us) {
            const int j = us % kNU;
            // the group's give-up decisions are votes (it meets at epi_sync later)
            if (!bar_and(1, C::EpiThreads, mbar_wait(&T->ufull[j], (us / kNU) & 1, abort, a.err, a.wait_limit))) break;
            const Slot<kNT> &sl = T->slot[j];
            if (sl.u < 0) break;
            const bool up = sl.up, shared = sl.shared;
            const int mc = sl.mc, nmma = sl.nmma, f0 = sl.f0, r0 = sl.row0, o = sl.o;
            const int acc = us % C::NAcc;
            if (!bar_and(1, C::EpiThreads, mbar_wait(&T->tfull[acc], (us / C::NAcc) & 1, abort, a.err, a.wait_limit)))
                break;
            tc_fence_after();
            const uint32_t tg = tmem + ((uint32_t)(quad * 32) << 16) + acc * C::AccW;
            const int ld = up ? a.I : a.d;               // row stride of the output
            __nv_bfloat16 *dst = up ? a.h + (size_t)r0 * a.I
                                    : (shared ? a.y_shared + (size_t)(r0 - a.N * a.K) * a.d : a.y_perm + (size_t)r0 * a.d);
            dst += f0 + quad * 32;
            // up: one pass, gate and up accumulators combined; down: the two
            // W_d tiles (features f0 .. f0+127 and f0+128 .. f0+255) in turn
#pragma unroll 1
            for (int t = 0; t < (up ? 1 : 2); ++t)
#pragma unroll 1
            for (int c = eg * W; c < nmma; c += W * C::EpiGroups) {
                uint32_t g[W], u[W];
                const uint32_t ta = tg + t * kNT + c;
                if (W == 32) {
                    tmem_ld32(ta, *reinterpret_cast<uint32_t(*)[32]>(g));
                    if (up) tmem_ld32(tg + kNT + c, *reinterpret_cast<uint32_t(*)[32]>(u));
                } else {
                    tmem_ld16(ta, *reinterpret_cast<uint32_t(*)[16]>(g));
                    if (up) tmem_ld16(tg + kNT + c, *reinterpret_cast<uint32_t(*)[16]>(u));
                }
                tmem_ld_wait();
                __nv_bfloat16 *dt = dst + t * kM;
#pragma unroll
                for (int half = 0; half < W / 16; ++half) {
#pragma unroll
                    for (int n = 0; n < 16; ++n) {
                        const float gv = __uint_as_float(g[half * 16 + n]);
                        const float val = up ? silu_mul(gv, __uint_as_float(u[half * 16 + n])) : gv;
                        stg[n * 32 + lane] = __bfloat16_as_ushort(__float2bfloat16_rn(val));
                    }
                    __syncwarp();
#pragma unroll
                    for (int hh = 0; hh < 2; ++hh) {
                        const int idx = lane + 32 * hh, n = idx >> 2, p = idx & 3;
                        const int tok = c + half * 16 + n;
                        if (tok < mc)
                            *reinterpret_cast<uint4 *>(dt + (size_t)tok * ld + p * 8) =
                                *reinterpret_cast<const uint4 *>(stg + n * 32 + p * 8);
                    }
                    __syncwarp();
                }
            }
            tc_fence_before();
            mbar_arrive(&T->tempty[acc]);
            epi_sync<C::EpiThreads>();
            if (threadIdx.x == 0) {
                // H visible before the expert's count is raised: the group's
                // stores are ordered before this fence by the barrier
                if (up) {
                    __threadfence();
                    red_release_add(a.up_done + o, 1);
                }
                mbar_arrive(&T->uempty[j]);
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, C::TmemCols);
    }
}

// ------------------------------------------------------------------- host
static PFN_cuTensorMapEncodeTiled_v12000 swap_encode_fn()
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

// BF16 weight map over a row-major [rows, cols] matrix, box of 128 rows x 64
// columns, 128-byte swizzle: the layout the MMA reads.
static bool weight_map(CUtensorMap *m, const void *base, uint64_t rows, uint64_t cols)
{
    auto fn = swap_encode_fn();
    if (!fn) return false;
    cuuint64_t dims[2] = {cols, rows};
    cuuint64_t strides[1] = {cols * 2};
    cuuint32_t box[2] = {64, (cuuint32_t)kM};
    cuuint32_t estr[2] = {1, 1};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(base),
              dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
              CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// BF16 activation map over [rows, cols], box of box_rows x 64 columns,
// 128-byte swizzle (the layout of a B tile panel).
static bool act_map(CUtensorMap *m, const void *base, uint64_t rows, uint64_t cols, int box_rows)
{
    auto fn = swap_encode_fn();
    if (!fn) return false;
    cuuint64_t dims[2] = {cols, rows};
    cuuint64_t strides[1] = {cols * 2};
    cuuint32_t box[2] = {64, (cuuint32_t)box_rows};
    cuuint32_t estr[2] = {1, 1};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(base), dims, strides, box, estr,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_128B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

static int swap_sm_count()
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

template <int kNT>
static void launch_cfg(const Maps &m, const Args &a, cudaStream_t st)
{
    using C = Cfg<kNT>;
    constexpr size_t smem = smem_bytes<kNT>();
    static_assert(smem <= (size_t)kSmemLimit, "shared memory per CTA");
    auto k = ffn_swap_kernel<kNT>;
    cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    launch_pdl(k, swap_sm_count(), C::Warps * 32, smem, st, m, a);
}

kmoe_status launch_ffn_swap(const __nv_bfloat16 *x, int N, int d, int I, int E, int K, const int32_t *perm,
                            const int32_t *offsets, const ExpertPtrs &routed, const ExpertPtrs *shared,
                            __nv_bfloat16 *h, __nv_bfloat16 *y_perm, __nv_bfloat16 *y_shared, int *status,
                            int *sync, long long wait_limit, cudaStream_t st)
{
    constexpr int token_chunk = 16;
    if (E + 1 > kMaxOrd || E + 2 > kSyncInts) return fail(KMOE_ERR_UNSUPPORTED, "swap-AB FFN: too many experts");
    if (d % kFD || I % kF) return fail(KMOE_ERR_UNSUPPORTED, "swap-AB FFN: d %% 256, I %% 128 must be 0");
    const ExpertPtrs sh = shared ? *shared : routed;     // unused maps still need a valid base
    Maps m{};
    const bool ok = weight_map(&m.g_r, routed.wg, (uint64_t)E * I, d) &&
                    weight_map(&m.u_r, routed.wu, (uint64_t)E * I, d) &&
                    weight_map(&m.g_s, sh.wg, I, d) && weight_map(&m.u_s, sh.wu, I, d) &&
                    weight_map(&m.d_r, routed.wd, (uint64_t)E * d, I) && weight_map(&m.d_s, sh.wd, d, I) &&
                    act_map(&m.xg, x, N, d, 1) && act_map(&m.hb, h, (uint64_t)N * K + N, I, token_chunk);
    if (!ok) return fail(KMOE_ERR_CUDA, "cuTensorMapEncodeTiled failed");
    Args a{};
    a.x = x;
    a.perm = perm;
    a.offsets = offsets;
    a.h = h;
    a.y_perm = y_perm;
    a.y_shared = y_shared;
    a.err = status;
    a.claim = sync;
    a.up_done = sync + 1;
    a.wait_limit = wait_limit;
    a.N = N; a.K = K; a.E = E; a.d = d; a.I = I;
    a.has_shared = shared ? 1 : 0;
    a.n_ord = E + a.has_shared;
    a.sk = Cfg<token_chunk>::BK;
    a.nt = token_chunk;
    launch_cfg<token_chunk>(m, a, st);
    return check_launch("ffn_swap");
}

}  // namespace kmoe
