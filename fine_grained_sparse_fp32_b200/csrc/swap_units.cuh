// Work units of the swap-AB grouped expert FFNs (weights as the MMA's M
// operand, token rows as N): the group order, token chunks, and the claim
// order of up and down units, shared by the BF16 / E4M3-weight kernel
// (ffn_swap.cu) and the FP8-activation kernel (ffn_a8.cu).
//
// "Inside Kolibri 1" (flozi.net), routing section: every routed or shared
// expert is a SwiGLU MLP, so each unit is one weight tile of one expert
// against one chunk of that expert's token rows:
//   up unit   (expert, 128 intermediate features, token chunk): gate and up
//             rows of the same features, H = SiLU(gate) * up;
//   down unit (expert, 256 output features, token chunk): two tiles of 128
//             W_d rows against the chunk's H rows.
// Every kernel argument struct A used with these helpers has the fields
// offsets, N, K, E, d, I, has_shared, n_ord (groups), nt (rows per chunk)
// and sk (K columns per pipeline stage), and err (the device status word).
#pragma once

#include <cstdint>

namespace kmoe {
namespace swp {

constexpr int kF = 128;                 // intermediate features per up unit (gate and up rows)
constexpr int kFD = 256;                // output features per down unit (two tiles of W_d rows)
constexpr int kMaxOrd = 1025;           // groups: E <= 1024 routed experts + the shared one

// Group order: [shared (if any), routed 0 .. E-1]; `off` is the
// shared-memory copy of `offsets`.
struct Group {
    int g, row0, rows;
    bool shared;
};

template <class A>
__device__ __forceinline__ Group group_at(int o, const int *off, const A &a)
{
    if (a.has_shared && o == 0) return {a.E, a.N * a.K, a.N, true};
    const int g = o - a.has_shared;
    return {g, off[g], off[g + 1] - off[g], false};
}

__device__ __forceinline__ int chunks_of(int rows, int nt) { return (rows + nt - 1) / nt; }

struct Unit {
    bool up;
    Group G;
    int o;          // position in the group order
    int f0;         // first feature (up: intermediate, down: output)
    int m0, mc;     // first row of the chunk inside the group, rows in it
    int nmma;       // MMA N: mc rounded up to 16
    int kb;         // k stages
};

// off = offsets; pre[o] = token chunks of the groups before o (one warp).
template <class A>
__device__ void build_prefix(int *pre, int *off, const A &a)
{
    const int lane = threadIdx.x & 31;
    for (int i = lane; i <= a.E; i += 32) off[i] = a.offsets[i];
    __syncwarp();
    if (!offsets_ok(off, a.E, a.N * a.K, a.err)) {     // debug build: no units at all
        for (int i = lane; i <= a.n_ord; i += 32) pre[i] = 0;
        __syncwarp();
        return;
    }
    const int per = (a.n_ord + 31) / 32;
    const int o0 = lane * per;
    int sum = 0;
    for (int i = 0; i < per; ++i)
        if (o0 + i < a.n_ord) sum += chunks_of(group_at(o0 + i, off, a).rows, a.nt);
    int incl = sum;
#pragma unroll
    for (int s = 1; s < 32; s <<= 1) {
        const int v = __shfl_up_sync(0xffffffffu, incl, s);
        if (lane >= s) incl += v;
    }
    int run = incl - sum;
    for (int i = 0; i < per; ++i)
        if (o0 + i < a.n_ord) {
            pre[o0 + i] = run;
            run += chunks_of(group_at(o0 + i, off, a).rows, a.nt);
        }
    if (lane == 31) pre[a.n_ord] = incl;
}

// Unit u: up units first (per group: feature tile major, chunk minor, so the
// chunks of one weight tile run back to back and share it in L2), then the
// down units in the same order.
template <class A>
__device__ __forceinline__ Unit decode(int u, const int *pre, const int *off, const A &a)
{
    const int up_tiles = a.I / kF, dn_tiles = a.d / kFD;
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
    const int ch = chunks_of(U.G.rows, a.nt);
    const int local = v - pre[U.o] * tiles;
    const int tile = local / ch, c = local - tile * ch;
    U.f0 = tile * (U.up ? kF : kFD);
    U.m0 = c * a.nt;
    U.mc = min(a.nt, U.G.rows - U.m0);
    U.nmma = (U.mc + 15) & ~15;
    U.kb = (U.up ? a.d : a.I) / a.sk;
    return U;
}

template <class A>
__device__ __forceinline__ int total_units(const int *pre, const A &a)
{
    return pre[a.n_ord] * (a.I / kF + a.d / kFD);
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

template <int kThreads>
__device__ __forceinline__ void epi_sync() { asm volatile("bar.sync 1, %0;" ::"n"(kThreads) : "memory"); }

// The block scales of one row block, s[0 .. nkb-1] (nkb <= 48), loaded by a
// whole warp at once: lane l holds s[l] in lo and s[l + 32] in hi (0 past
// the end).
struct WarpScales {
    float lo, hi;
    __device__ __forceinline__ void load(const float *s, int nkb)
    {
        const int l = threadIdx.x & 31;
        lo = l < nkb ? s[l] : 0.f;
        hi = l + 32 < nkb ? s[l + 32] : 0.f;
    }
};

}  // namespace swp
}  // namespace kmoe
