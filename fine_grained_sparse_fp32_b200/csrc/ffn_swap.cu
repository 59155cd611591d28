// Grouped SwiGLU expert FFN for small batches (decode) on the tcgen05 tensor
// cores, weights as the M operand ("swap-AB").
//
// "Inside Kolibri 1" (flozi.net), routing section: every routed or shared
// expert is a SwiGLU MLP (two d -> I projections, SiLU(gate) * up, one
// I -> d projection, no biases). At decode a routed expert sees one or two
// tokens, so the layer is a weight stream: each selected expert's 3*d*I
// weights cross HBM once and meet a handful of token rows.
//
// Here a 128-row weight tile is the MMA's A operand (M = 128, streamed by
// TMA in 64-column stages) and the expert's tokens are its B operand
// (N = 16 rows), so the tensor cores do the dot products and the SM's
// issue slots stay free: the kernel only moves bytes. Work units:
//   up unit   (expert, 64 intermediate features, chunk of <= 16 tokens):
//             A = [64 gate rows ; 64 up rows] x d, one M = 128 MMA per k16
//             gives gate in accumulator lanes 0-63 and up in lanes 64-127;
//             the epilogue pairs them through shared memory and writes
//             H = SiLU(gate) * up;
//   down unit (expert, 128 output features, same token chunk):
//             A = W_d rows x I, B = the chunk's H rows.
// One persistent launch runs every up unit, then every down unit: a CTA
// claims units from a global counter, and the producer of a down unit waits
// (bounded) until all up units of that expert have published their H rows.
// Units are small (655 KB / 131 KB of BF16 weights), so the grid finishes
// within one down unit of the mean.
//
// Warp roles (one CTA per SM):
//   warps 0-3  epilogue: tcgen05.ld of the accumulator, SwiGLU or the BF16
//              cast, global stores; hands the accumulator back to the MMA;
//   warp  4    one thread issues tcgen05.mma / tcgen05.commit;
//   warp  5    producer: claims units, TMA loads of the weight tiles,
//              cp.async gathers of the token (or H) rows;
//   warps 6-9  E4M3 weights only: converters.
// E4M3 weights ("Inside Kolibri 1", FP8 section: 128 x 128 blocks with one
// FP32 scale each) arrive by TMA as bytes. Converter warps decode them
// exactly to F16 (hardware e4m3x2 -> f16x2), multiply each row by
// s_kb / s_ref (its block's scale over the largest scale of the row block,
// so the factor is at most 1 and nothing overflows), and write the tile
// straight into tensor memory with tcgen05.st: the MMA takes A from tensor
// memory, so the decoded weights never cross shared memory. The token rows
// are converted to F16 for the B operand, the MMA is F16 x F16 with FP32
// accumulation, and the epilogue multiplies by s_ref. |x| must stay inside
// the F16 range (65504); a value outside it sets device status 2.
#include "common.cuh"
#include "sm100.cuh"

#include <cudaTypedefs.h>

namespace kmoe {
using namespace sm100;

namespace swp {

constexpr int kM = 128;                 // weight rows per unit (MMA M)
constexpr int kBK = 64;                 // k per BF16 stage: 128 bytes of BF16
constexpr int kBK8 = 128;               // k per E4M3 stage: one scale block, 128 bytes of E4M3
__host__ __device__ constexpr int stage_k(bool fp8) { return fp8 ? kBK8 : kBK; }
constexpr int kNT = 16;                 // tokens per unit at most (the MMA's N)
constexpr int kPanel = kNT * 128;       // one 64-element column panel of a B tile (2 KB)
constexpr int kUpF = 64;                // intermediate features per up unit
constexpr int kDnF = 128;               // output features per down unit
constexpr int kATile = kM * kBK * 2;    // 16 KB
constexpr int kBTile = kNT * kBK * 2;   // 2 KB
constexpr int kA8Tile = kM * kBK8;      // 16 KB of E4M3
constexpr int kB8Tile = kNT * kBK8 * 2;  // 4 KB: two column panels
constexpr int kNU = 8;                  // unit-info slots
constexpr int kNAcc = 4;                // accumulators of 32 TMEM columns (N <= 32)
static_assert(kNT % 16 == 0 && kNT <= 32, "token chunk: a multiple of 16, at most 32");
constexpr int kAccCols = kNAcc * 32;    // E4M3: A stages follow at this column
constexpr int kMaxOrd = 1025;
constexpr long long kWaitLimit = 1LL << 32;   // SM cycles, about 2 s

// BF16 weights: one ring of (A | B) stages.
constexpr int kStagesBf = 11;
constexpr int kStageBf = kATile + kBTile;                       // 18 KB
// E4M3 weights: a raw ring (E4M3 A | BF16 B rows) in shared memory and a
// converted ring: F16 A in tensor memory (64 columns a stage), F16 B in
// shared memory. Two groups of four converter warps take alternate stages.
constexpr int kRawStages = 10;
constexpr int kRawStage = kA8Tile + kB8Tile;                    // 20 KB
constexpr int kConvStages = 3;
constexpr int kConvStage = kB8Tile;                             // 4 KB
constexpr int kConvGroups = 2;
__host__ __device__ constexpr int tmem_cols(bool fp8) { return fp8 ? 512 : 128; }
static_assert(kAccCols + kConvStages * 64 <= 512, "tensor memory columns");

constexpr int kEpiWarps = 4, kMmaWarp = 4, kProdWarp = 5, kSchedWarp = 6, kConvWarp = 7;
__host__ __device__ constexpr int threads_of(bool fp8) { return (fp8 ? kConvWarp + 4 * kConvGroups : kConvWarp) * 32; }

// A unit as the scheduler warp resolved it: everything the other roles need,
// so that none of them touches global memory to set a unit up.
struct Slot {
    int u;                   // unit index, -1 = no more work
    int up, shared, o;       // kind, shared expert, position in the group order
    int g;                   // expert (E = shared)
    int f0, mc, nmma, kb;    // first feature, token rows, MMA N, stages
    int row0;                // first dispatched row of the chunk
    int wrow;                // first weight row in the stacked weight matrix
    int src[kNT];            // B row n: token (up) or dispatched row (down), n < mc
    float ref[2];            // E4M3: largest block scale of the rows (gate or W_d, up)
    float s[2][48];          // E4M3: block scales of the rows along K (d / 128 <= 48)
};

struct Tail {
    uint64_t full[kRawStages > kStagesBf ? kRawStages : kStagesBf];
    uint64_t empty[kRawStages > kStagesBf ? kRawStages : kStagesBf];
    uint64_t cfull[kConvStages], cempty[kConvStages];
    uint64_t ufull[kNU], uempty[kNU];
    uint64_t tfull[kNAcc], tempty[kNAcc];
    uint64_t drain;
    uint32_t tmem_base;
    int abort;
    Slot slot[kNU];
    uint16_t pre[kMaxOrd + 1];   // token-chunk prefix over the group order
    uint16_t off[kMaxOrd + 1];   // copy of the routed groups' row offsets
    float xch[kUpF][kNT + 1];    // up-unit epilogue: up values handed to the gate warps
};

__host__ __device__ constexpr size_t ring_bytes(bool fp8)
{
    return fp8 ? (size_t)kRawStages * kRawStage + (size_t)kConvStages * kConvStage
               : (size_t)kStagesBf * kStageBf;
}
__host__ __device__ constexpr size_t smem_bytes(bool fp8) { return 1024 + ring_bytes(fp8) + sizeof(Tail); }
static_assert(smem_bytes(false) <= 232448 && smem_bytes(true) <= 232448, "227 KB of shared memory per CTA");

struct Maps {
    CUtensorMap g_r, u_r, g_s, u_s;   // up: gate / up rows, box 64 columns x 64 rows
    CUtensorMap d_r, d_s;             // down: W_d rows, box 64 columns x 128 rows
};

struct Args {
    const __nv_bfloat16 *x;           // [N, d]
    const int32_t *perm, *offsets;
    __nv_bfloat16 *h;                 // [N*K + N, I]
    __nv_bfloat16 *y_perm, *y_shared;
    const float *sg_r, *su_r, *sd_r, *sg_s, *su_s, *sd_s;   // E4M3 block scales
    int *err;                         // device status word
    int *claim;                       // unit counter (zero at launch)
    int *up_done;                     // [groups] finished up units (zero at launch)
    int N, K, E, d, I, has_shared, n_ord;
    int sk;                           // k per stage (stage_k)
};

// Group order: [shared (if any), routed 0 .. E-1].
struct Group {
    int g, row0, rows;
    bool shared;
};

// Batches on this path have N * (K + 1) < 65536, so row offsets and chunk
// counts fit 16 bits; `off` is the shared-memory copy of `offsets`.
__device__ __forceinline__ Group group_at(int o, const uint16_t *off, const Args &a)
{
    if (a.has_shared && o == 0) return {a.E, a.N * a.K, a.N, true};
    const int g = o - a.has_shared;
    return {g, off[g], off[g + 1] - off[g], false};
}

__device__ __forceinline__ int chunks_of(int rows) { return (rows + kNT - 1) / kNT; }

struct Unit {
    bool up;
    Group G;
    int o;          // position in the group order
    int f0;         // first feature (up: intermediate, down: output)
    int m0, mc;     // first row of the chunk inside the group, rows in it
    int nmma;       // MMA N: 16 or 32
    int kb;         // k stages
};

// off = offsets; pre[o] = token chunks of the groups before o (one warp).
__device__ void build_prefix(uint16_t *pre, uint16_t *off, const Args &a)
{
    const int lane = threadIdx.x & 31;
    for (int i = lane; i <= a.E; i += 32) off[i] = static_cast<uint16_t>(a.offsets[i]);
    __syncwarp();
    const int per = (a.n_ord + 31) / 32;
    const int o0 = lane * per;
    int sum = 0;
    for (int i = 0; i < per; ++i)
        if (o0 + i < a.n_ord) sum += chunks_of(group_at(o0 + i, off, a).rows);
    int incl = sum;
#pragma unroll
    for (int s = 1; s < 32; s <<= 1) {
        const int v = __shfl_up_sync(0xffffffffu, incl, s);
        if (lane >= s) incl += v;
    }
    int run = incl - sum;
    for (int i = 0; i < per; ++i)
        if (o0 + i < a.n_ord) {
            pre[o0 + i] = static_cast<uint16_t>(run);
            run += chunks_of(group_at(o0 + i, off, a).rows);
        }
    if (lane == 31) pre[a.n_ord] = static_cast<uint16_t>(incl);
}

// Unit u: up units first (per group: feature tile major, chunk minor), then
// down units in the same order.
__device__ __forceinline__ Unit decode(int u, const uint16_t *pre, const uint16_t *off, const Args &a)
{
    const int up_tiles = a.I / kUpF, dn_tiles = a.d / kDnF;
    const int total_ch = pre[a.n_ord];
    Unit U;
    U.up = u < up_tiles * total_ch;
    const int tiles = U.up ? up_tiles : dn_tiles;
    const int v = U.up ? u : u - up_tiles * total_ch;
    int lo = 1, hi = a.n_ord;       // smallest j with pre[j] * tiles > v
    while (lo < hi) {
        const int mid = (lo + hi) >> 1;
        if (pre[mid] * tiles > v) hi = mid;
        else lo = mid + 1;
    }
    U.o = lo - 1;
    U.G = group_at(U.o, off, a);
    const int ch = chunks_of(U.G.rows);
    const int local = v - pre[U.o] * tiles;
    const int tile = local / ch, c = local - tile * ch;
    U.f0 = tile * (U.up ? kUpF : kDnF);
    U.m0 = c * kNT;
    U.mc = min(kNT, U.G.rows - U.m0);
    U.nmma = U.mc > 16 ? 32 : 16;          // <= kNT
    U.kb = (U.up ? a.d : a.I) / a.sk;
    return U;
}

__device__ __forceinline__ int total_units(const uint16_t *pre, const Args &a)
{
    return pre[a.n_ord] * (a.I / kUpF + a.d / kDnF);
}

__device__ __forceinline__ int ld_acquire(const int *p)
{
    int v;
    asm volatile("ld.acquire.gpu.global.b32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}

__device__ __forceinline__ void red_release_add(int *p, int v)
{
    asm volatile("red.release.gpu.global.add.s32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}

__device__ __forceinline__ void fence_proxy_async_global()
{
    asm volatile("fence.proxy.async.global;" ::: "memory");
}

__device__ __forceinline__ void epi_sync() { asm volatile("bar.sync 1, 128;" ::: "memory"); }

// Instruction descriptor of tcgen05.mma kind::f16: A and B both BF16 or both
// F16 (K-major), FP32 accumulator, M x N.
__host__ __device__ constexpr uint32_t idesc(int M, int N, bool bf16)
{
    return (1u << 4) | ((bf16 ? 1u : 0u) << 7) | ((bf16 ? 1u : 0u) << 10) | ((uint32_t)(N >> 3) << 17) |
           ((uint32_t)(M >> 4) << 24);
}

// The block scales of one row block, s[0 .. nkb-1] (nkb <= 48), loaded by a
// whole warp at once: lane l holds s[l] in lo and s[l + 32] in hi (0 past
// the end). ref() is their maximum (the F16 path's normaliser), at(i) is s[i].
struct WarpScales {
    float lo, hi;
    __device__ __forceinline__ void load(const float *s, int nkb)
    {
        const int l = threadIdx.x & 31;
        lo = l < nkb ? s[l] : 0.f;
        hi = l + 32 < nkb ? s[l + 32] : 0.f;
    }
    __device__ __forceinline__ float ref() const
    {
        float m = fmaxf(lo, hi);
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
        return m;
    }
    __device__ __forceinline__ float at(int i) const
    {
        return __shfl_sync(0xffffffffu, i < 32 ? lo : hi, i & 31);
    }
};

// Four E4M3 values (one 32-bit word, element 0 in the low byte) -> two F16x2
// words, exactly (every E4M3 value is an F16 value).
__device__ __forceinline__ void e4m3x4_to_f16(uint32_t w, uint32_t &a, uint32_t &b)
{
    asm("{\n\t.reg .b16 l, h;\n\t"
        "mov.b32 {l, h}, %2;\n\t"
        "cvt.rn.f16x2.e4m3x2 %0, l;\n\t"
        "cvt.rn.f16x2.e4m3x2 %1, h;\n\t}"
        : "=r"(a), "=r"(b)
        : "r"(w));
}

__device__ __forceinline__ uint32_t pack_f16x2(float lo, float hi)
{
    uint32_t r;
    asm("cvt.rn.f16x2.f32 %0, %2, %1;" : "=r"(r) : "f"(lo), "f"(hi));
    return r;
}

__device__ __forceinline__ uint32_t hmul2(uint32_t a, uint32_t b)
{
    uint32_t r;
    asm("mul.rn.f16x2 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(b));
    return r;
}

}  // namespace swp

using namespace swp;

enum : int { kErrF16Range = 2 };

template <bool kFp8>
__global__ void __launch_bounds__(threads_of(kFp8), 1)
ffn_swap_kernel(const __grid_constant__ Maps maps, const Args a)
{
    constexpr int S = kFp8 ? kRawStages : kStagesBf;     // producer ring
    constexpr int SB = kFp8 ? kRawStage : kStageBf;
    constexpr int ABytes = kFp8 ? kA8Tile : kATile;      // A bytes a stage receives by TMA
    constexpr int BK = stage_k(kFp8);
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t *conv = smem + (size_t)kRawStages * kRawStage;   // E4M3 only
    Tail *T = reinterpret_cast<Tail *>(smem + ring_bytes(kFp8));
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    volatile int *abort = &T->abort;

    if (threadIdx.x == 0) {
        for (int s = 0; s < S; ++s) {
            mbar_init(&T->full[s], 1 + 32);              // TMA expect_tx + 32 cp.async arrivals
            mbar_init(&T->empty[s], kFp8 ? 128 : 1);     // converters | tcgen05.commit
        }
        for (int s = 0; s < kConvStages; ++s) {
            mbar_init(&T->cfull[s], 128);
            mbar_init(&T->cempty[s], 1);
        }
        for (int j = 0; j < kNU; ++j) {
            mbar_init(&T->ufull[j], 1);
            mbar_init(&T->uempty[j], 1);
        }
        for (int c = 0; c < kNAcc; ++c) {
            mbar_init(&T->tfull[c], 1);
            mbar_init(&T->tempty[c], 128);
        }
        mbar_init(&T->drain, 1);
        T->abort = 0;
        fence_mbar_init();
    }
    if (warp == kSchedWarp) build_prefix(T->pre, T->off, a);
    if (warp == 0) {
        tmem_alloc(&T->tmem_base, tmem_cols(kFp8));
        tmem_relinquish();
    }
    if (warp == kProdWarp && lane == 0) {
        prefetch_map(&maps.g_r); prefetch_map(&maps.u_r); prefetch_map(&maps.d_r);
        if (a.has_shared) { prefetch_map(&maps.g_s); prefetch_map(&maps.u_s); prefetch_map(&maps.d_s); }
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = T->tmem_base;

    if (warp == kSchedWarp) {
        // ----------------------------------------------------------- scheduler
        // Claims units one ahead, resolves each into a slot (rows, weight
        // rows, E4M3 scales) and, for a down unit, waits until the expert's
        // up units have published H. Runs up to kNU units ahead of the
        // epilogue, so these global-memory round trips overlap the stream.
        const int total = total_units(T->pre, a);
        int ahead = lane == 0 ? atomicAdd(a.claim, 1) : 0;
        for (int us = 0;; ++us) {
            const int j = us % kNU;
            if (!mbar_wait(&T->uempty[j], ((us / kNU) & 1) ^ 1, abort, a.err, kWaitLimit)) break;
            int u = __shfl_sync(0xffffffffu, ahead, 0);
            if (u >= total) u = -1;
            if (lane == 0 && u >= 0) ahead = atomicAdd(a.claim, 1);
            Slot &sl = T->slot[j];
            if (u < 0) {
                if (lane == 0) {
                    sl.u = -1;
                    mbar_arrive(&T->ufull[j]);
                }
                break;
            }
            const Unit U = decode(u, T->pre, T->off, a);
            const int row0 = U.G.row0 + U.m0;
            const size_t ge = U.G.shared ? 0 : (size_t)U.G.g;
            // every global load of the unit is issued before any is used: one round trip
            int srcv = 0;
            if (lane < U.mc)
                srcv = U.up ? (U.G.shared ? row0 + lane - a.N * a.K : a.perm[row0 + lane]) : row0 + lane;
            WarpScales w0, w1;
            w0.lo = w0.hi = w1.lo = w1.hi = 0.f;
            if (kFp8) {
                if (U.up) {
                    const int nkb = a.d / 128;
                    const size_t off = (ge * (a.I / 128) + U.f0 / 128) * nkb;
                    w0.load((U.G.shared ? a.sg_s : a.sg_r) + off, nkb);
                    w1.load((U.G.shared ? a.su_s : a.su_r) + off, nkb);
                } else {
                    const int nkb = a.I / 128;
                    w0.load((U.G.shared ? a.sd_s : a.sd_r) + (ge * (a.d / 128) + U.f0 / 128) * nkb, nkb);
                }
            }
            const int need = (a.I / kUpF) * chunks_of(U.G.rows);
            int done = need;
            if (!U.up && lane == 0) done = ld_acquire(a.up_done + U.o);
            if (lane < U.mc) sl.src[lane] = srcv;
            if (kFp8) {
                sl.s[0][lane] = w0.lo;
                sl.s[1][lane] = w1.lo;
                if (lane < 16) { sl.s[0][lane + 32] = w0.hi; sl.s[1][lane + 32] = w1.hi; }
                const float r0 = w0.ref(), r1 = w1.ref();
                if (lane == 0) { sl.ref[0] = r0; sl.ref[1] = r1; }
            }
            bool good = true;
            if (lane == 0 && done < need) {       // the expert's H rows come from up units of any CTA
                const long long t0 = clock64();
                while (ld_acquire(a.up_done + U.o) < need) {
                    if (*abort) { good = false; break; }
                    if (clock64() - t0 > kWaitLimit) {
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
                sl.g = U.G.g;
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
        const uint64_t pol_w = policy_evict_first();    // weights: streamed once
        const uint64_t pol_a = policy_evict_last();     // token / H rows: reused by many units
        uint32_t it = 0;
        bool ok = true;
        for (int us = 0;; ++us) {
            const int j = us % kNU;
            if (!mbar_wait(&T->ufull[j], (us / kNU) & 1, abort, a.err, kWaitLimit)) { ok = false; break; }
            const Slot &sl = T->slot[j];
            if (sl.u < 0) break;
            const bool up = sl.up, shared = sl.shared;
            const int kb_n = sl.kb, wrow = sl.wrow, mc = sl.mc, nmma = sl.nmma;
            const int n = lane;                         // B row of this lane
            const bool live = n < nmma, valid = n < mc;
            const int srow = valid ? sl.src[n] : 0;
            if (!up) fence_proxy_async_global();        // H written by other CTAs, seen through the scheduler
            const __nv_bfloat16 *src = up ? a.x + (size_t)srow * a.d : a.h + (size_t)srow * a.I;
            const CUtensorMap *m0 = up ? (shared ? &maps.g_s : &maps.g_r) : (shared ? &maps.d_s : &maps.d_r);
            const CUtensorMap *m1 = shared ? &maps.u_s : &maps.u_r;
            for (int kb = 0; kb < kb_n; ++kb, ++it) {
                const int s = it % S;
                if (!mbar_wait(&T->empty[s], ((it / S) & 1) ^ 1, abort, a.err, kWaitLimit)) { ok = false; break; }
                uint8_t *A = smem + (size_t)s * SB;
                uint8_t *B = A + ABytes;
                if (lane == 0) {
                    mbar_arrive_expect_tx(&T->full[s], ABytes);
                    if (up) {
                        tma_load_2d_hint(A, m0, &T->full[s], kb * BK, wrow, pol_w);
                        tma_load_2d_hint(A + ABytes / 2, m1, &T->full[s], kb * BK, wrow, pol_w);
                    } else {
                        tma_load_2d_hint(A, m0, &T->full[s], kb * BK, wrow, pol_w);
                    }
                }
                if (live) {     // 64-element column panels of 128-byte swizzled rows
                    const uint32_t dst = smem_u32(B) + n * 128;
                    const __nv_bfloat16 *sp = src + kb * BK;
#pragma unroll
                    for (int c = 0; c < BK / 8; ++c)
                        cp_async16_hint(dst + (c >> 3) * kPanel + (((c & 7) ^ (n & 7)) << 4), sp + c * 8,
                                        valid ? 16u : 0u, pol_a);
                }
                cp_async_arrive_noinc(&T->full[s]);
            }
            if (!ok) break;
        }
        cp_async_wait_all();
        if (!ok && lane == 0)    // let in-flight TMA loads land before the CTA exits
            for (uint32_t j = it > (uint32_t)S ? it - S : 0; j < it; ++j)
                mbar_wait_drain(&T->full[j % S], (j / S) & 1, kWaitLimit);
    } else if (warp == kMmaWarp) {
        // ----------------------------------------------------------------- MMA
        if (lane == 0) {
            constexpr int CS = kFp8 ? kConvStages : kStagesBf;
            uint32_t it = 0;
            for (int us = 0;; ++us) {
                const int j = us % kNU;
                if (!mbar_wait(&T->ufull[j], (us / kNU) & 1, abort, a.err, kWaitLimit)) break;
                const Slot &sl = T->slot[j];
                if (sl.u < 0) break;
                const int kb_n = sl.kb;
                const int acc = us % kNAcc;
                if (!mbar_wait(&T->tempty[acc], ((us / kNAcc) & 1) ^ 1, abort, a.err, kWaitLimit)) break;
                tc_fence_after();
                const uint32_t dcol = tmem + acc * 32;
                const uint32_t id = idesc(kM, sl.nmma, !kFp8);
                bool ok = true;
                for (int kb = 0; kb < kb_n; ++kb, ++it) {
                    const int s = it % CS;
                    uint64_t *fullb = kFp8 ? &T->cfull[s] : &T->full[s];
                    if (!mbar_wait(fullb, (it / CS) & 1, abort, a.err, kWaitLimit)) { ok = false; break; }
                    tc_fence_after();
                    if (kFp8) {       // A: F16 in tensor memory (8 columns per k16); B: F16 panels in shared memory
                        const uint32_t at = tmem + kAccCols + s * 64;
                        const uint64_t bd = sw128_kmajor_desc(smem_u32(conv + (size_t)s * kConvStage));
#pragma unroll
                        for (int k = 0; k < kBK8 / 16; ++k)
                            umma_f16_tmem_a(dcol, at + k * 8, bd + (uint64_t)(((k >> 2) * kPanel + (k & 3) * 32) >> 4), id,
                                            (kb | k) != 0);
                        umma_commit(&T->cempty[s]);
                    } else {
                        const uint32_t sa = smem_u32(smem + (size_t)s * kStageBf);
                        const uint64_t ad = sw128_kmajor_desc(sa);
                        const uint64_t bd = sw128_kmajor_desc(sa + kATile);
#pragma unroll
                        for (int k = 0; k < kBK / 16; ++k)
                            umma_bf16(dcol, ad + (uint64_t)(k * 2), bd + (uint64_t)(k * 2), id, (kb | k) != 0);
                        umma_commit(&T->empty[s]);
                    }
                }
                if (!ok) break;
                umma_commit(&T->tfull[acc]);
            }
            umma_commit(&T->drain);     // every MMA done before tensor memory is released
            mbar_wait_drain(&T->drain, 0, kWaitLimit);
        }
        __syncwarp();
    } else if (warp < kEpiWarps) {
        // ------------------------------------------------------------ epilogue
        const int row = warp * 32 + lane;              // accumulator lane = weight row of the unit
        for (int us = 0;; ++us) {
            const int j = us % kNU;
            if (!mbar_wait(&T->ufull[j], (us / kNU) & 1, abort, a.err, kWaitLimit)) break;
            const Slot &sl = T->slot[j];
            if (sl.u < 0) break;
            const bool up = sl.up, shared = sl.shared;
            const int mc = sl.mc, f0 = sl.f0, r0 = sl.row0, o = sl.o;
            // E4M3: rows 0-63 of an up unit are gate rows, 64-127 up rows
            const float sref = kFp8 ? sl.ref[(up && warp >= 2) ? 1 : 0] : 1.f;
            const int acc = us % kNAcc;
            if (!mbar_wait(&T->tfull[acc], (us / kNAcc) & 1, abort, a.err, kWaitLimit)) break;
            tc_fence_after();
            const uint32_t taddr = tmem + ((uint32_t)(warp * 32) << 16) + acc * 32;
            uint32_t v[kNT];
#pragma unroll
            for (int c = 0; c < kNT; c += 16)
                if (c < sl.nmma) tmem_ld16(taddr + c, *reinterpret_cast<uint32_t(*)[16]>(v + c));
            tmem_ld_wait();
            tc_fence_before();
            mbar_arrive(&T->tempty[acc]);
            if (up) {
                if (warp >= 2) {
#pragma unroll
                    for (int n = 0; n < kNT; ++n)
                        if (n < mc) T->xch[row - kUpF][n] = __uint_as_float(v[n]) * sref;
                }
                epi_sync();
                if (warp < 2) {
                    __nv_bfloat16 *dst = a.h + (size_t)r0 * a.I + f0 + row;
#pragma unroll
                    for (int n = 0; n < kNT; ++n)
                        if (n < mc) {
                            const float g = __uint_as_float(v[n]) * sref;
                            dst[(size_t)n * a.I] = __float2bfloat16_rn(g * sigmoidf_(g) * T->xch[row][n]);
                        }
                    __threadfence();
                }
                epi_sync();
                if (threadIdx.x == 0) red_release_add(a.up_done + o, 1);
            } else {
                __nv_bfloat16 *dst = shared ? a.y_shared + (size_t)(r0 - a.N * a.K) * a.d : a.y_perm + (size_t)r0 * a.d;
                dst += f0 + row;
#pragma unroll
                for (int n = 0; n < kNT; ++n)
                    if (n < mc) dst[(size_t)n * a.d] = __float2bfloat16_rn(__uint_as_float(v[n]) * sref);
                epi_sync();
            }
            if (threadIdx.x == 0) mbar_arrive(&T->uempty[j]);
        }
    } else if (kFp8 && warp >= kConvWarp) {
        // ---------------------------------------------------------- converters
        // A warp reaches only its own quadrant of tensor-memory lanes, so the
        // A row a thread converts is its lane in that quadrant. Group `grp`
        // takes the stages it with it % kConvGroups == grp.
        const int quad = warp & 3, grp = (warp - kConvWarp) / 4;
        const int q = quad * 32 + lane;                 // A row; B chunks q + 128 i
        uint32_t it = 0;
        bool ok = true;
        for (int us = 0; ok; ++us) {
            const int j = us % kNU;
            if (!mbar_wait(&T->ufull[j], (us / kNU) & 1, abort, a.err, kWaitLimit)) break;
            const Slot &sl = T->slot[j];
            if (sl.u < 0) break;
            const int kb_n = sl.kb, nmma = sl.nmma;
            // this row's scales: up units = gate (rows 0-63) or up (64-127); down = W_d
            const int which = (sl.up && quad >= 2) ? 1 : 0;
            const float ref = sl.ref[which];
            const float inv = ref > 0.f ? 1.f / ref : 0.f;
            const float *srow = sl.s[which];
            bool range_ok = true;
            for (int kb = 0; kb < kb_n; ++kb, ++it) {
                if ((int)(it % kConvGroups) != grp) continue;
                const int rs = it % kRawStages, cs = it % kConvStages;
                const float r = srow[kb] * inv;                      // in [0, 1]
                if (!mbar_wait(&T->full[rs], (it / kRawStages) & 1, abort, a.err, kWaitLimit) ||
                    !mbar_wait(&T->cempty[cs], ((it / kConvStages) & 1) ^ 1, abort, a.err, kWaitLimit)) {
                    ok = false;
                    break;
                }
                const uint8_t *A8 = smem + (size_t)rs * kRawStage;
                const uint8_t *Braw = A8 + kA8Tile;
                uint8_t *B = conv + (size_t)cs * kConvStage;
                // A row q: 128 E4M3 bytes (128-byte swizzle) -> 128 F16 * r -> 64 columns of tensor memory
                const uint32_t r2 = pack_f16x2(r, r);
                const uint32_t tq = tmem + ((uint32_t)(quad * 32) << 16) + kAccCols + cs * 64;
#pragma unroll
                for (int half = 0; half < 2; ++half) {
                    uint32_t o[32];
#pragma unroll
                    for (int c4 = 0; c4 < 4; ++c4) {
                        const int c = half * 4 + c4;
                        const uint4 w = *reinterpret_cast<const uint4 *>(A8 + q * 128 + ((c ^ (q & 7)) << 4));
                        const uint32_t wd[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
                        for (int h = 0; h < 4; ++h) {
                            uint32_t lo, hi;
                            e4m3x4_to_f16(wd[h], lo, hi);
                            o[c4 * 8 + 2 * h] = hmul2(lo, r2);
                            o[c4 * 8 + 2 * h + 1] = hmul2(hi, r2);
                        }
                    }
                    tmem_st32(tq + half * 32, o);
                }
                // B: BF16 token (or H) rows -> F16 at the same swizzled positions;
                // a panel holds kNT rows of eight 16-byte chunks
#pragma unroll
                for (int i4 = 0; i4 < kB8Tile / 16 / 128; ++i4) {
                    const int c16 = q + i4 * 128;
                    if (((c16 % (kNT * 8)) >> 3) < nmma) {
                        const uint4 w = *reinterpret_cast<const uint4 *>(Braw + c16 * 16);
                        const uint32_t wd[4] = {w.x, w.y, w.z, w.w};
                        uint32_t p[4];
                        float mx = 0.f;
#pragma unroll
                        for (int i = 0; i < 4; ++i) {
                            const float f0 = bf16_lo(wd[i]), f1 = bf16_hi(wd[i]);
                            p[i] = pack_f16x2(f0, f1);
                            mx = fmaxf(mx, fmaxf(fabsf(f0), fabsf(f1)));
                        }
                        if (!(mx <= 65504.f)) range_ok = false;
                        *reinterpret_cast<uint4 *>(B + c16 * 16) = make_uint4(p[0], p[1], p[2], p[3]);
                    }
                }
                tmem_st_wait();
                fence_proxy_async();
                tc_fence_before();
                mbar_arrive(&T->cfull[cs]);
                mbar_arrive(&T->empty[rs]);
            }
            if (!range_ok) atomicCAS(a.err, kErrNone, kErrF16Range);
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, tmem_cols(kFp8));
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

// Weight map over a row-major [rows, cols] matrix, box of 128-byte rows
// (64 BF16 or 128 E4M3 columns) x box_rows, 128-byte swizzle: the layout
// the MMA reads (BF16), and one the converters read without bank conflicts
// (E4M3).
static bool weight_map(CUtensorMap *m, const void *base, uint64_t rows, uint64_t cols, int box_rows, bool fp8)
{
    auto fn = swap_encode_fn();
    if (!fn) return false;
    const uint64_t es = fp8 ? 1 : 2;
    cuuint64_t dims[2] = {cols, rows};
    cuuint64_t strides[1] = {cols * es};
    cuuint32_t box[2] = {(cuuint32_t)(fp8 ? kBK8 : kBK), (cuuint32_t)box_rows};
    cuuint32_t estr[2] = {1, 1};
    return fn(m, fp8 ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(base),
              dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
              CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
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

kmoe_status launch_ffn_swap(const __nv_bfloat16 *x, int N, int d, int I, int E, int K, const int32_t *perm,
                            const int32_t *offsets, int w_dtype, const ExpertPtrs &routed, const ExpertPtrs *shared,
                            __nv_bfloat16 *h, __nv_bfloat16 *y_perm, __nv_bfloat16 *y_shared, int *status,
                            int *sync, cudaStream_t st)
{
    if (E + 1 > kMaxOrd || E + 2 > kSyncInts) return fail(KMOE_ERR_UNSUPPORTED, "swap-AB FFN: too many experts");
    if (d % kDnF || I % 128) return fail(KMOE_ERR_UNSUPPORTED, "swap-AB FFN: d, I must be multiples of 128");
    if ((long long)N * (K + 1) >= 65536) return fail(KMOE_ERR_UNSUPPORTED, "swap-AB FFN: batch too large");
    const bool fp8 = w_dtype == KMOE_E4M3_B128;
    const ExpertPtrs sh = shared ? *shared : routed;     // unused maps still need a valid base
    Maps m{};
    const bool ok = weight_map(&m.g_r, routed.wg, (uint64_t)E * I, d, kUpF, fp8) &&
                    weight_map(&m.u_r, routed.wu, (uint64_t)E * I, d, kUpF, fp8) &&
                    weight_map(&m.g_s, sh.wg, I, d, kUpF, fp8) && weight_map(&m.u_s, sh.wu, I, d, kUpF, fp8) &&
                    weight_map(&m.d_r, routed.wd, (uint64_t)E * d, I, kDnF, fp8) &&
                    weight_map(&m.d_s, sh.wd, d, I, kDnF, fp8);
    if (!ok) return fail(KMOE_ERR_CUDA, "cuTensorMapEncodeTiled failed");
    Args a{};
    a.x = x;
    a.perm = perm;
    a.offsets = offsets;
    a.h = h;
    a.y_perm = y_perm;
    a.y_shared = y_shared;
    a.sg_r = routed.sg; a.su_r = routed.su; a.sd_r = routed.sd;
    a.sg_s = sh.sg; a.su_s = sh.su; a.sd_s = sh.sd;
    a.err = status;
    a.claim = sync;
    a.up_done = sync + 1;
    a.N = N; a.K = K; a.E = E; a.d = d; a.I = I;
    a.has_shared = shared ? 1 : 0;
    a.n_ord = E + a.has_shared;
    a.sk = stage_k(fp8);
    const int grid = swap_sm_count();
    if (fp8) {
        constexpr size_t smem = smem_bytes(true);
        cudaFuncSetAttribute(ffn_swap_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        ffn_swap_kernel<true><<<grid, threads_of(true), smem, st>>>(m, a);
    } else {
        constexpr size_t smem = smem_bytes(false);
        cudaFuncSetAttribute(ffn_swap_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        ffn_swap_kernel<false><<<grid, threads_of(false), smem, st>>>(m, a);
    }
    return check_launch("ffn_swap");
}

}  // namespace kmoe
