// Grouped SwiGLU expert FFN on the FP8 tensor cores: E4M3 x E4M3 tcgen05
// MMAs (kind::f8f6f4), weights as the M operand, for E4M3 weights with FP8
// activations, or with BF16 activations held as two E4M3 terms (below).
//
// "Inside Kolibri 1" (flozi.net), section "The FP8 path is explicitly mixed
// precision": the weights are E4M3 in 128 x 128 blocks with one FP32 scale
// per block, and the activations are quantised dynamically in groups of
// 1 x 128 (an FP32 scale per row and 128 columns). Both scales are used as
// stored, never rounded to powers of two, so the tensor cores cannot apply
// them: every 128-column K block is one scale block of both operands, its
// partial sums are accumulated by the tensor cores into a fresh tensor-
// memory slot, and CUDA-core warps fold each slot into FP32 registers:
//     acc[f][t] += P_kb[f][t] * s_w[f / 128][kb] * s_x[t][kb].
// The routing section gives the expert: H = SiLU(x W_g^T) * (x W_u^T),
// y = H W_d^T. Activations here are x's E4M3 codes for gate/up and H's for
// down; H is rounded to BF16 and quantised in groups of 1 x 128 in the up
// epilogue (an up unit's 128 features are exactly one group of each of its
// token rows).
//
// Units and their order are those of the swap-AB kernel (swap_units.cuh):
// an up unit is 128 gate rows + the same 128 up rows against a chunk of kNT
// token rows, a down unit two tiles of 128 W_d rows against a chunk of H
// rows. One 128 x 128 E4M3 weight tile (16 KB) is one MMA A operand per
// K block, the chunk's codes (kNT rows x 128 bytes) the B operand; four
// K = 32 MMAs per tile and block.
//
// Chunks hold kNT = 16, 32 or 64 token rows (the host picks one from the
// expected rows per expert): a weight tile crosses shared memory once per
// chunk, so larger batches take larger chunks.
//
// Two-term mode (kTwo): the same kernel serves E4M3 weights with BF16
// activations. Every activation group is held as two E4M3 codes
// with one scale, x = s * (hi + lo / 16) up to about 2^-8 of |x| (the size of
// a BF16 rounding); the hi rows of a chunk are B rows 0 .. kNT-1 and the lo
// rows B rows kNT .. 2 kNT-1 of one N = 2 kNT operand, so a K block still
// takes four MMAs per weight tile, and the promotion adds
// (P_hi + P_lo / 16) * s_w * s_x. H is kept in the same two-term form
// between up and down.
//
// Warp roles (one CTA per SM, persistent), P = 4 promotion warps for chunks
// of up to 32 rows and 8 for 64:
//   warps 0..P-1  promotion: tcgen05.ld of each partial slot, scale and add
//                 into registers (thread = weight row of its quadrant, warp
//                 w & 3; with 8 warps, warp w >> 2 takes token columns
//                 32 (w >> 2) ..), then the unit's epilogue (SwiGLU + H
//                 quantisation, or the BF16 output);
//   warp  P       one thread issues tcgen05.mma / tcgen05.commit;
//   warp  P+1     producer: TMA of the weight tiles and of the H codes (one
//                 box of H rows, lane 0); an up unit's x-code rows are
//                 gathered with cp.async, 8 lanes per 128-byte row, straight
//                 into the swizzled layout, and complete on the stage barrier;
//   warp  P+2     scheduler: claims units, resolves them into shared-memory
//                 slots, and before a down unit waits (bounded) for the up
//                 units of its expert.
#include "common.cuh"
#include "sm100.cuh"
#include "swap_units.cuh"

#include <cudaTypedefs.h>

namespace kmoe {
using namespace sm100;

namespace a8 {

using swp::kF;
using swp::kFD;
using swp::kMaxOrd;

constexpr int kM = 128;                 // weight rows per tile (MMA M)
constexpr int kBK = 128;                // K columns per stage: one scale block of both operands
constexpr int kATile = kM * kBK;        // 16 KB of E4M3 weights
constexpr int kNU = 8;                  // unit slots
constexpr int kSmemLimit = 232448;      // 227 KB per CTA

template <int kNT, bool kTwo = false>
struct Cfg {
    static constexpr int TPW = kNT < 32 ? kNT : 32;      // token columns of one promotion warp
    static constexpr int PWarps = 4 * (kNT / TPW);       // promotion warps: 4 lane quadrants x column groups
    static constexpr int PThreads = 32 * PWarps;
    static constexpr int MmaWarp = PWarps, ProdWarp = PWarps + 1, SchedWarp = PWarps + 2, Warps = PWarps + 3;
    static constexpr int BRows = kTwo ? 2 * kNT : kNT;   // B operand rows: the chunk's codes (hi | lo)
    static constexpr int BTile = BRows * kBK;            // token codes of one stage
    static constexpr int Stage = 2 * kATile + BTile;     // weight tile 0 | weight tile 1 | token codes
    static constexpr int Stages = kTwo ? (kNT == 64 ? 3 : 5) : kNT == 16 ? 6 : kNT == 32 ? 5 : 4;
    static constexpr int PW = 2 * BRows;                 // one partial slot: tile 0 | tile 1
    static constexpr int NP = 512 / PW < 8 ? 512 / PW : 8;   // partial slots in tensor memory
    static constexpr int TmemCols = NP * PW <= 256 ? 256 : 512;
    static constexpr int RPL = (kNT + 31) / 32;          // chunk rows per scheduler lane
    static_assert(kNT == 16 || kNT == 32 || kNT == 64, "token chunk of 16, 32 or 64 rows");
    static_assert(Stage % 1024 == 0, "tiles on 1024-byte boundaries (128-byte swizzle atoms)");
    static_assert(NP * PW <= TmemCols, "tensor memory columns");
};

template <int kNT>
struct Slot {
    int u;                   // unit index, -1 = no more work
    int up, shared, o;       // kind, shared expert, position in the group order
    int f0, mc, nmma, kb;    // first feature, token rows, MMA N, K blocks
    int row0;                // first dispatched row of the chunk
    int wrow;                // first weight row in the stacked weight matrix
    float s[2][48];          // weight block scales of the two tiles along K (K / 128 <= 48)
    int src[kNT];            // B row n: token (up) or dispatched row (down), n < mc
};

template <int kNT, bool kTwo>
struct Tail {
    uint64_t full[6], empty[6];
    uint64_t pfull[8], pempty[8];
    uint64_t ufull[kNU], uempty[kNU];
    uint64_t drain, pstart;
    uint32_t tmem_base;
    int abort;
    Slot<kNT> slot[kNU];
    alignas(16) uint32_t amax[4][kNT];                        // up epilogue: |H| maximum per quadrant and token (float bits)
    alignas(16) uint8_t codes[kTwo ? 2 : 1][kNT][128];        // up epilogue: the unit's H codes (hi, lo), token-major
    alignas(16) uint16_t stage[Cfg<kNT>::PWarps][16][32];     // down epilogue: 16 tokens x 32 features per warp
    int pre[kMaxOrd + 1];
    int off[kMaxOrd + 1];
};

template <int kNT, bool kTwo>
__host__ __device__ constexpr size_t smem_bytes()
{
    return 1024 + (size_t)Cfg<kNT, kTwo>::Stages * Cfg<kNT, kTwo>::Stage + sizeof(Tail<kNT, kTwo>);
}

struct Maps {
    CUtensorMap g_r, u_r, g_s, u_s;   // gate / up rows, routed and shared (128 rows x 128 bytes)
    CUtensorMap d_r, d_s;             // W_d rows
    CUtensorMap hq;                   // H codes [N*K + N, I]: boxes of kNT rows x 128 bytes
    CUtensorMap hl;                   // two-term mode: H low codes, same shape
};

struct Args {
    const uint8_t *xq;                // x codes [N, d] (two-term mode: the high codes)
    const uint8_t *xl;                // two-term mode: x low codes [N, d]
    const float *xs;                  // x scales [N, d / 128]
    const int32_t *perm, *offsets;
    uint8_t *hq;                      // H codes [N*K + N, I] (two-term mode: the high codes)
    uint8_t *hl;                      // two-term mode: H low codes [N*K + N, I]
    float *hs;                        // H scales [N*K + N, I / 128]
    __nv_bfloat16 *y_perm, *y_shared;
    const float *sg_r, *su_r, *sd_r, *sg_s, *su_s, *sd_s;   // weight block scales
    int *err;                         // device status word
    int *claim;                       // unit counter (zero at launch)
    int *up_done;                     // [groups] finished up units (zero at launch)
    long long wait_limit;             // SM cycles before a pipeline wait gives up
    int N, K, E, d, I, has_shared, n_ord;
    int sk;                           // K columns per stage (128)
    int nt;                           // token rows per chunk (kNT)
};

// A scale written by another CTA during this launch: a strong load at GPU
// scope, so that no stale L1 line is read.
__device__ __forceinline__ float ld_relaxed_f32(const float *p)
{
    float v;
    asm volatile("ld.relaxed.gpu.global.f32 %0, [%1];" : "=f"(v) : "l"(p) : "memory");
    return v;
}

template <int kN>
__device__ __forceinline__ void tmem_load(uint32_t taddr, uint32_t (&r)[kN])
{
    if constexpr (kN == 16) tmem_ld16(taddr, r);
    else tmem_ld32(taddr, r);
}

__device__ __forceinline__ uint8_t e4m3_code(float v)
{
    return (uint8_t)__nv_cvt_float_to_fp8(v, __NV_SATFINITE, __NV_E4M3);
}

}  // namespace a8

using namespace a8;

template <int kNT, bool kTwo>
__global__ void __launch_bounds__(Cfg<kNT, kTwo>::Warps * 32, 1)
ffn_a8_kernel(const __grid_constant__ Maps maps, const Args a)
{
    using C = Cfg<kNT, kTwo>;
    constexpr int SA = C::Stages, NP = C::NP, TPW = C::TPW;
    constexpr int kMmaWarp = C::MmaWarp, kProdWarp = C::ProdWarp, kSchedWarp = C::SchedWarp;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    Tail<kNT, kTwo> *T = reinterpret_cast<Tail<kNT, kTwo> *>(smem + (size_t)SA * C::Stage);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    volatile int *abort = &T->abort;
    const long long lim = a.wait_limit;

    if (threadIdx.x == 0) {
        for (int s = 0; s < SA; ++s) {
            mbar_init(&T->full[s], 1 + 32);              // TMA expect_tx (lane 0) + every producer lane's cp.async
            mbar_init(&T->empty[s], 1);                  // tcgen05.commit
        }
        for (int p = 0; p < NP; ++p) {
            mbar_init(&T->pfull[p], 1);                  // tcgen05.commit
            mbar_init(&T->pempty[p], C::PThreads);       // every promotion thread has read the slot
        }
        for (int j = 0; j < kNU; ++j) {
            mbar_init(&T->ufull[j], 1);
            mbar_init(&T->uempty[j], 1);
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
        prefetch_map(&maps.hq);
        if (kTwo) prefetch_map(&maps.hl);
    }
    pdl_wait();               // routing, x codes and scales come from earlier kernels
    pdl_trigger();
    if (warp == kSchedWarp) swp::build_prefix(T->pre, T->off, a);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = T->tmem_base;

    if (warp == kSchedWarp) {
        // ----------------------------------------------------------- scheduler
        // As in the swap-AB kernel: a unit is claimed only once the producer
        // has started the previous one, every global load of a unit is issued
        // before any is used, and a down unit waits (bounded) until all up
        // units of its expert have published their H rows.
        const int total = swp::total_units(T->pre, a);
        for (int us = 0;; ++us) {
            const int j = us % kNU;
            if (!mbar_wait(&T->uempty[j], ((us / kNU) & 1) ^ 1, abort, a.err, lim)) break;
            if (us > 0 && !mbar_wait(&T->pstart, (us - 1) & 1, abort, a.err, lim)) break;
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
            const swp::Unit U = swp::decode(u, T->pre, T->off, a);
            const int row0 = U.G.row0 + U.m0;
            const size_t ge = U.G.shared ? 0 : (size_t)U.G.g;
            int srcv[C::RPL];                              // chunk rows lane, lane + 32
#pragma unroll
            for (int i = 0; i < C::RPL; ++i) {
                const int n = lane + 32 * i;
                srcv[i] = 0;
                if (n < U.mc)
                    srcv[i] = U.up ? (U.G.shared ? row0 + n - a.N * a.K : checked_index(a.perm[row0 + n], 0, a.N, a.err))
                                   : row0 + n;
            }
            swp::WarpScales w0, w1;
            if (U.up) {
                const int nkb = a.d / kBK;
                const size_t off = (ge * (a.I / 128) + U.f0 / 128) * nkb;
                w0.load((U.G.shared ? a.sg_s : a.sg_r) + off, nkb);
                w1.load((U.G.shared ? a.su_s : a.su_r) + off, nkb);
            } else {                                       // the two row blocks of W_d
                const int nkb = a.I / kBK;
                const float *sd = (U.G.shared ? a.sd_s : a.sd_r) + (ge * (a.d / 128) + U.f0 / 128) * nkb;
                w0.load(sd, nkb);
                w1.load(sd + nkb, nkb);
            }
            const int need = (a.I / kF) * swp::chunks_of(U.G.rows, a.nt);
            bool good = true;
            if (!U.up && lane == 0 && swp::ld_acquire(a.up_done + U.o) < need) {
                const long long t0 = clock64();
                while (swp::ld_acquire(a.up_done + U.o) < need) {
                    if (*abort) { good = false; break; }
                    if (clock64() - t0 > lim) {
                        *abort = 1;
                        atomicCAS(a.err, kErrNone, kErrWaitTimeout);
                        good = false;
                        break;
                    }
                    __nanosleep(64);
                }
            }
            if (!__shfl_sync(0xffffffffu, good ? 1 : 0, 0)) break;
#pragma unroll
            for (int i = 0; i < C::RPL; ++i)
                if (lane + 32 * i < U.mc) sl.src[lane + 32 * i] = srcv[i];
            sl.s[0][lane] = w0.lo;
            sl.s[1][lane] = w1.lo;
            if (lane < 16) { sl.s[0][lane + 32] = w0.hi; sl.s[1][lane + 32] = w1.hi; }
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
        // Lane l copies the 16-byte piece l % 8 of chunk rows 4j + l / 8, so
        // that every cp.async instruction of the warp reads four whole
        // 128-byte row segments; rows past the chunk are zero-filled.
        const uint64_t pol_w = policy_evict_first();    // routed weights: streamed once
        const uint64_t pol_k = policy_evict_last();     // token / H codes and the shared expert: reused
        const int pc = lane & 7, rl = lane >> 3;
        uint32_t it = 0;
        bool ok = true;
        for (int us = 0;; ++us) {
            const int j = us % kNU;
            if (!mbar_wait(&T->ufull[j], (us / kNU) & 1, abort, a.err, lim)) { ok = false; break; }
            const Slot<kNT> &sl = T->slot[j];
            if (sl.u < 0) break;
            const bool up = sl.up, shared = sl.shared;
            const int kb_n = sl.kb, wrow = sl.wrow, mc = sl.mc, nmma = sl.nmma, r0 = sl.row0;
            int tokr[kNT / 4];                           // token of chunk row 4j + rl, -1 past the chunk
#pragma unroll
            for (int q = 0; q < kNT / 4; ++q) tokr[q] = up && 4 * q + rl < mc ? sl.src[4 * q + rl] : -1;
            __syncwarp();
            if (lane == 0) mbar_arrive(&T->pstart);
            if (!up) swp::fence_proxy_async_global();   // H codes written by other CTAs, seen through the scheduler
            const CUtensorMap *m0 = up ? (shared ? &maps.g_s : &maps.g_r) : (shared ? &maps.d_s : &maps.d_r);
            const CUtensorMap *m1 = shared ? &maps.u_s : &maps.u_r;
            const uint64_t pw = shared ? pol_k : pol_w;
            for (int kb = 0; kb < kb_n; ++kb, ++it) {
                const int s = it % SA;
                if (!mbar_wait(&T->empty[s], ((it / SA) & 1) ^ 1, abort, a.err, lim)) { ok = false; break; }
                uint8_t *A = smem + (size_t)s * C::Stage;
                uint8_t *B = A + 2 * kATile;
                if (lane == 0) {
                    mbar_arrive_expect_tx(&T->full[s], 2 * kATile + (up ? 0u : (uint32_t)C::BRows * kBK));
                    tma_load_2d_hint(A, m0, &T->full[s], kb * kBK, wrow, pw);
                    // second tile: the up rows of the same features, or the next 128 W_d rows
                    tma_load_2d_hint(A + kATile, up ? m1 : m0, &T->full[s], kb * kBK, up ? wrow : wrow + kM, pw);
                    if (!up) {
                        tma_load_2d_hint(B, &maps.hq, &T->full[s], kb * kBK, r0, pol_k);
                        if (kTwo) tma_load_2d_hint(B + kNT * kBK, &maps.hl, &T->full[s], kb * kBK, r0, pol_k);
                    }
                }
                if (up) {
                    const uint32_t bdst = smem_u32(B);
#pragma unroll
                    for (int q = 0; q < kNT / 4; ++q)
                        if (4 * q < nmma) {
                            const int r = 4 * q + rl, tk = tokr[q];
                            const size_t off = (size_t)(tk < 0 ? 0 : tk) * a.d + kb * kBK + pc * 16;
                            cp_async16_hint(bdst + r * 128 + ((pc ^ (r & 7)) << 4), a.xq + off, tk >= 0 ? 16u : 0u, pol_k);
                            if (kTwo) {       // low codes: row kNT + r (kNT is a multiple of 8: same swizzle phase)
                                const int r2 = kNT + r;
                                cp_async16_hint(bdst + r2 * 128 + ((pc ^ (r2 & 7)) << 4), a.xl + off, tk >= 0 ? 16u : 0u,
                                                pol_k);
                            }
                        }
                }
                cp_async_arrive_noinc(&T->full[s]);       // the stage completes when these rows land
            }
            if (!ok) break;
        }
        cp_async_wait_all();     // this lane's row copies have landed before it leaves
        if (!ok && lane == 0)    // let in-flight TMA loads land before the CTA exits
            for (uint32_t j = it > (uint32_t)SA ? it - SA : 0; j < it; ++j)
                mbar_wait_drain(&T->full[j % SA], (j / SA) & 1, kDefaultWaitLimit);
    } else if (warp == kMmaWarp) {
        // ----------------------------------------------------------------- MMA
        if (lane == 0) {
            uint32_t it = 0;
            for (int us = 0;; ++us) {
                const int j = us % kNU;
                if (!mbar_wait(&T->ufull[j], (us / kNU) & 1, abort, a.err, lim)) break;
                const Slot<kNT> &sl = T->slot[j];
                if (sl.u < 0) break;
                const int kb_n = sl.kb;
                // two-term: N covers the hi rows 0 .. kNT-1 and the lo rows kNT .. 2 kNT-1
                const uint32_t id = idesc_e4m3_f32(kM, kTwo ? C::BRows : sl.nmma);
                bool ok = true;
                for (int kb = 0; kb < kb_n; ++kb, ++it) {
                    const int s = it % SA, p = it % NP;
                    if (!mbar_wait(&T->full[s], (it / SA) & 1, abort, a.err, lim) ||
                        !mbar_wait(&T->pempty[p], ((it / NP) & 1) ^ 1, abort, a.err, lim)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t sa = smem_u32(smem + (size_t)s * C::Stage);
                    const uint64_t a0 = sw128_kmajor_desc(sa), a1 = sw128_kmajor_desc(sa + kATile);
                    const uint64_t bd = sw128_kmajor_desc(sa + 2 * kATile);
                    const uint32_t d0 = tmem + p * C::PW, d1 = d0 + C::BRows;
                    // a fresh partial per K block; one accumulator's k-steps back to back
#pragma unroll
                    for (int k = 0; k < kBK / 32; ++k) umma_f8(d0, a0 + (uint64_t)(k * 2), bd + (uint64_t)(k * 2), id, k);
#pragma unroll
                    for (int k = 0; k < kBK / 32; ++k) umma_f8(d1, a1 + (uint64_t)(k * 2), bd + (uint64_t)(k * 2), id, k);
                    umma_commit(&T->empty[s]);
                    umma_commit(&T->pfull[p]);
                }
                if (!ok) break;
            }
            umma_commit(&T->drain);     // every MMA done before tensor memory is released
            mbar_wait_drain(&T->drain, 0, kDefaultWaitLimit);
        }
        __syncwarp();
    } else if (warp < C::PWarps) {
        // ------------------------------------------------- promotion, epilogue
        // Thread = weight row quad * 32 + lane of the unit's tiles, for the
        // token columns c0 .. c0 + TPW - 1 of the chunk; lane n also carries
        // token c0 + n's activation scale of the current K block (loaded two
        // blocks ahead) and hands it out by shuffle.
        const int quad = warp & 3, c0 = (warp >> 2) * TPW;
        uint32_t it = 0;
        for (int us = 0;; ++us) {
            const int j = us % kNU;
            // the group's give-up decisions are votes (it meets at epi_sync later)
            if (!bar_and(1, C::PThreads, mbar_wait(&T->ufull[j], (us / kNU) & 1, abort, a.err, lim))) break;
            const Slot<kNT> &sl = T->slot[j];
            if (sl.u < 0) break;
            const bool up = sl.up, shared = sl.shared;
            const int mc = sl.mc, f0 = sl.f0, r0 = sl.row0, o = sl.o, kb_n = sl.kb;
            const int tok = c0 + lane;                     // this lane's token column (scales, epilogue)
            const bool mine = lane < TPW && tok < mc;
            const int nkb = up ? a.d / kBK : a.I / kBK;
            const float *sp = up ? a.xs + (size_t)(mine ? sl.src[tok] : 0) * nkb
                                 : a.hs + (size_t)(r0 + (mine ? tok : 0)) * nkb;
            float sx0 = mine ? ld_relaxed_f32(sp) : 0.f;
            float sx1 = mine && kb_n > 1 ? ld_relaxed_f32(sp + 1) : 0.f;
            float acc0[TPW], acc1[TPW];
#pragma unroll
            for (int n = 0; n < TPW; ++n) acc0[n] = acc1[n] = 0.f;
            bool ok = true;
            for (int kb = 0; kb < kb_n; ++kb, ++it) {
                const float sx2 = mine && kb + 2 < kb_n ? ld_relaxed_f32(sp + kb + 2) : 0.f;
                const int p = it % NP;
                if (!bar_and(1, C::PThreads, mbar_wait(&T->pfull[p], (it / NP) & 1, abort, a.err, lim))) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint32_t ta = tmem + ((uint32_t)(quad * 32) << 16) + p * C::PW + c0;
                const float w0 = sl.s[0][kb], w1 = sl.s[1][kb];
                if constexpr (kTwo && TPW == 32) {
                    // 32 columns per warp: hi and lo in turn through one register block
                    const float w0l = 0.0625f * w0, w1l = 0.0625f * w1;
                    uint32_t v[TPW];
                    tmem_load<TPW>(ta, v);                 // tile 0, hi
                    tmem_ld_wait();
#pragma unroll
                    for (int n = 0; n < TPW; ++n)
                        acc0[n] = fmaf(__uint_as_float(v[n]), w0 * __shfl_sync(0xffffffffu, sx0, n), acc0[n]);
                    tmem_load<TPW>(ta + kNT, v);           // tile 0, lo
                    tmem_ld_wait();
#pragma unroll
                    for (int n = 0; n < TPW; ++n)
                        acc0[n] = fmaf(__uint_as_float(v[n]), w0l * __shfl_sync(0xffffffffu, sx0, n), acc0[n]);
                    tmem_load<TPW>(ta + C::BRows, v);      // tile 1, hi
                    tmem_ld_wait();
#pragma unroll
                    for (int n = 0; n < TPW; ++n)
                        acc1[n] = fmaf(__uint_as_float(v[n]), w1 * __shfl_sync(0xffffffffu, sx0, n), acc1[n]);
                    tmem_load<TPW>(ta + C::BRows + kNT, v);   // tile 1, lo
                    tmem_ld_wait();
                    tc_fence_before();
                    mbar_arrive(&T->pempty[p]);
#pragma unroll
                    for (int n = 0; n < TPW; ++n)
                        acc1[n] = fmaf(__uint_as_float(v[n]), w1l * __shfl_sync(0xffffffffu, sx0, n), acc1[n]);
                } else if constexpr (kTwo) {
                    // 16 columns per warp: the K block's four products (hi and lo
                    // of both tiles) in one tensor-memory round trip
                    uint32_t vh0[TPW], vl0[TPW], vh1[TPW], vl1[TPW];
                    tmem_load<TPW>(ta, vh0);
                    tmem_load<TPW>(ta + kNT, vl0);
                    tmem_load<TPW>(ta + C::BRows, vh1);
                    tmem_load<TPW>(ta + C::BRows + kNT, vl1);
                    tmem_ld_wait();
                    tc_fence_before();
                    mbar_arrive(&T->pempty[p]);
#pragma unroll
                    for (int n = 0; n < TPW; ++n) {
                        const float sn = __shfl_sync(0xffffffffu, sx0, n);
                        acc0[n] = fmaf(fmaf(__uint_as_float(vl0[n]), 0.0625f, __uint_as_float(vh0[n])), w0 * sn, acc0[n]);
                        acc1[n] = fmaf(fmaf(__uint_as_float(vl1[n]), 0.0625f, __uint_as_float(vh1[n])), w1 * sn, acc1[n]);
                    }
                } else {
                    {
                        uint32_t v[TPW];                   // tile 0 (gate or the first W_d rows)
                        tmem_load<TPW>(ta, v);
                        tmem_ld_wait();
#pragma unroll
                        for (int n = 0; n < TPW; ++n)
                            acc0[n] = fmaf(__uint_as_float(v[n]), w0 * __shfl_sync(0xffffffffu, sx0, n), acc0[n]);
                    }
                    {
                        uint32_t v[TPW];                   // tile 1 (up or the next W_d rows)
                        tmem_load<TPW>(ta + kNT, v);
                        tmem_ld_wait();
                        tc_fence_before();
                        mbar_arrive(&T->pempty[p]);
#pragma unroll
                        for (int n = 0; n < TPW; ++n)
                            acc1[n] = fmaf(__uint_as_float(v[n]), w1 * __shfl_sync(0xffffffffu, sx0, n), acc1[n]);
                    }
                }
                sx0 = sx1;
                sx1 = sx2;
            }
            if (!ok) break;
            if (up) {
                // H = bf16(SiLU(gate) * up); each token's 128 features (this
                // unit's rows, spread over the four lane quadrants) form one
                // 1 x 128 group: scale = amax / 448, code = E4M3(h * (1 / scale))
                // with the reciprocal and the product in FP32 (within 2^-23 of
                // h / scale, so at most one code step away from E4M3(h / scale)
                // when that quotient lies next to a rounding boundary).
                float hv[TPW];
#pragma unroll
                for (int n = 0; n < TPW; ++n) {
                    hv[n] = __bfloat162float(__float2bfloat16_rn(silu_mul(acc0[n], acc1[n])));
                    const uint32_t m = __reduce_max_sync(0xffffffffu, __float_as_uint(fabsf(hv[n])));
                    if (lane == n) T->amax[quad][c0 + n] = m;
                }
                swp::epi_sync<C::PThreads>();
                float s_l = 1.f;                           // lane n: scale of token c0 + n
                if (lane < TPW) {
                    const float am = fmaxf(fmaxf(__uint_as_float(T->amax[0][tok]), __uint_as_float(T->amax[1][tok])),
                                           fmaxf(__uint_as_float(T->amax[2][tok]), __uint_as_float(T->amax[3][tok])));
                    s_l = am > 0.f ? __fdiv_rn(am, 448.f) : 1.f;
                }
                const float r_l = __frcp_rn(s_l);
#pragma unroll
                for (int n = 0; n < TPW; ++n) {
                    const float y = hv[n] * __shfl_sync(0xffffffffu, r_l, n);
                    const uint8_t hc = e4m3_code(y);
                    T->codes[0][c0 + n][quad * 32 + lane] = hc;
                    if (kTwo) {       // lo = E4M3((y - hi) * 16)
                        const float hd = __half2float(__half(__nv_cvt_fp8_to_halfraw(hc, __NV_E4M3)));
                        T->codes[kTwo ? 1 : 0][c0 + n][quad * 32 + lane] = e4m3_code((y - hd) * 16.f);
                    }
                }
                swp::epi_sync<C::PThreads>();
                // 16-byte pieces: token n = i / 8, piece i % 8 of its 128 codes (per plane)
                for (int i = threadIdx.x; i < kNT * 8; i += C::PThreads) {
                    const int n = i >> 3, pc = i & 7;
                    if (n < mc) {
                        const size_t at = (size_t)(r0 + n) * a.I + f0 + pc * 16;
                        *reinterpret_cast<uint4 *>(a.hq + at) = *reinterpret_cast<const uint4 *>(&T->codes[0][n][pc * 16]);
                        if (kTwo)
                            *reinterpret_cast<uint4 *>(a.hl + at) =
                                *reinterpret_cast<const uint4 *>(&T->codes[kTwo ? 1 : 0][n][pc * 16]);
                    }
                }
                if (quad == 0 && mine) a.hs[(size_t)(r0 + tok) * (a.I / kBK) + f0 / kBK] = s_l;
            } else {
                // Y = BF16 of the two tiles (features f0 .. f0+127, f0+128 ..
                // f0+255) through a per-warp 16 x 32 transpose, so that every
                // global store writes 16 bytes (8 features of one token).
                __nv_bfloat16 *dst = shared ? a.y_shared + (size_t)(r0 - a.N * a.K) * a.d
                                            : a.y_perm + (size_t)r0 * a.d;
                dst += f0 + quad * 32;
                uint16_t *stg = &T->stage[warp][0][0];
#pragma unroll
                for (int t = 0; t < 2; ++t)
#pragma unroll
                    for (int half = 0; half < TPW / 16; ++half) {
#pragma unroll
                        for (int n = 0; n < 16; ++n) {
                            const float v = t ? acc1[half * 16 + n] : acc0[half * 16 + n];
                            stg[n * 32 + lane] = __bfloat16_as_ushort(__float2bfloat16_rn(v));
                        }
                        __syncwarp();
#pragma unroll
                        for (int hh = 0; hh < 2; ++hh) {
                            const int idx = lane + 32 * hh, n = idx >> 2, pc = idx & 3;
                            const int tk = c0 + half * 16 + n;
                            if (tk < mc)
                                *reinterpret_cast<uint4 *>(dst + t * kM + (size_t)tk * a.d + pc * 8) =
                                    *reinterpret_cast<const uint4 *>(stg + n * 32 + pc * 8);
                        }
                        __syncwarp();
                    }
            }
            swp::epi_sync<C::PThreads>();                  // the slot and the staging areas are free
            if (threadIdx.x == 0) {
                // the group's H codes and scales are ordered before this
                // thread's fence by the barrier: one fence publishes them all
                if (up) {
                    __threadfence();
                    swp::red_release_add(a.up_done + o, 1);
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
static PFN_cuTensorMapEncodeTiled_v12000 a8_encode_fn()
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

// Byte map over a row-major [rows, cols] matrix of E4M3 codes, box of
// box_rows x 128 bytes, 128-byte swizzle (the K-major layout the MMA reads).
static bool code_map(CUtensorMap *m, const void *base, uint64_t rows, uint64_t cols, int box_rows)
{
    auto fn = a8_encode_fn();
    if (!fn) return false;
    cuuint64_t dims[2] = {cols, rows};
    cuuint64_t strides[1] = {cols};
    cuuint32_t box[2] = {(cuuint32_t)kBK, (cuuint32_t)box_rows};
    cuuint32_t estr[2] = {1, 1};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void *>(base), dims, strides, box, estr,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

static int a8_sm_count()
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

template <int kNT, bool kTwo = false>
static kmoe_status launch_a8_cfg(const ExpertPtrs &routed, const ExpertPtrs &sh, Args a, cudaStream_t st)
{
    const uint64_t R = (uint64_t)a.N * a.K + a.N;
    Maps m{};
    const bool ok = code_map(&m.g_r, routed.wg, (uint64_t)a.E * a.I, a.d, kM) &&
                    code_map(&m.u_r, routed.wu, (uint64_t)a.E * a.I, a.d, kM) &&
                    code_map(&m.g_s, sh.wg, a.I, a.d, kM) && code_map(&m.u_s, sh.wu, a.I, a.d, kM) &&
                    code_map(&m.d_r, routed.wd, (uint64_t)a.E * a.d, a.I, kM) &&
                    code_map(&m.d_s, sh.wd, a.d, a.I, kM) && code_map(&m.hq, a.hq, R, a.I, kNT) &&
                    code_map(&m.hl, kTwo ? a.hl : a.hq, R, a.I, kNT);
    if (!ok) return fail(KMOE_ERR_CUDA, "cuTensorMapEncodeTiled failed");
    a.nt = kNT;
    constexpr size_t smem = smem_bytes<kNT, kTwo>();
    static_assert(smem <= (size_t)kSmemLimit, "shared memory per CTA");
    auto k = ffn_a8_kernel<kNT, kTwo>;
    cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    launch_pdl(k, a8_sm_count(), Cfg<kNT, kTwo>::Warps * 32, smem, st, m, a);
    return check_launch("ffn_a8");
}

kmoe_status launch_ffn_a8(const uint8_t *xq, const float *xs, int N, int d, int I, int E, int K, const int32_t *perm,
                          const int32_t *offsets, const ExpertPtrs &routed, const ExpertPtrs *shared, uint8_t *hq,
                          float *hs, __nv_bfloat16 *y_perm, __nv_bfloat16 *y_shared, int *status, int *sync,
                          long long wait_limit, cudaStream_t st, const uint8_t *xl, uint8_t *hl)
{
    if (E + 1 > kMaxOrd || E + 2 > kSyncInts) return fail(KMOE_ERR_UNSUPPORTED, "FP8 FFN: too many experts");
    if (d % kFD || I % kF || d / kBK > 48 || I / kBK > 48)
        return fail(KMOE_ERR_UNSUPPORTED, "FP8 FFN: d %% 256 and I %% 128 must be 0, d and I <= 6144");
    const ExpertPtrs sh = shared ? *shared : routed;     // unused maps still need a valid base
    Args a{};
    a.xq = xq;
    a.xl = xl;
    a.xs = xs;
    a.perm = perm;
    a.offsets = offsets;
    a.hq = hq;
    a.hl = hl;
    a.hs = hs;
    a.y_perm = y_perm;
    a.y_shared = y_shared;
    a.sg_r = routed.sg; a.su_r = routed.su; a.sd_r = routed.sd;
    a.sg_s = sh.sg; a.su_s = sh.su; a.sd_s = sh.sd;
    a.err = status;
    a.claim = sync;
    a.up_done = sync + 1;
    a.wait_limit = wait_limit;
    a.N = N; a.K = K; a.E = E; a.d = d; a.I = I;
    a.has_shared = shared ? 1 : 0;
    a.n_ord = E + a.has_shared;
    a.sk = kBK;
    // Chunk rows from the expected rows per routed expert, N * K / E: 16 while
    // experts see a dozen tokens or fewer, then 32, then 64 (a weight tile
    // crosses shared memory once per chunk).
    const long long avg = (long long)N * K / E;
    if (xl) {                 // two-term operands (BF16-precision activations)
        if (!hl) return fail(KMOE_ERR_INVALID_ARG, "FP8 FFN: two-term mode needs both low-code planes");
        if (avg <= 12) return launch_a8_cfg<16, true>(routed, sh, a, st);
        if (avg <= 32) return launch_a8_cfg<32, true>(routed, sh, a, st);
        return launch_a8_cfg<64, true>(routed, sh, a, st);
    }
    if (avg <= 12) return launch_a8_cfg<16>(routed, sh, a, st);
    if (avg <= 32) return launch_a8_cfg<32>(routed, sh, a, st);
    return launch_a8_cfg<64>(routed, sh, a, st);
}

}  // namespace kmoe
