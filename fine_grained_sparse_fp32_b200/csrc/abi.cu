// C ABI of the kmoe library: argument checks, workspace layout, dispatch to
// the kernels, and the whole-layer forward.
#include "common.cuh"

#include <cstdarg>
#include <cstdio>
#include <cstring>

namespace kmoe {

static thread_local char g_err[512] = "";

// Workspace status block: the status word and tickets (ints 0..63), then the
// grouped FFN's counters (kSyncInts ints). Router-only calls use 256 bytes.
constexpr int kSyncOffset = 64;                         // ints
constexpr int kStatusInts = kSyncOffset + kSyncInts;    // status word, tickets, FFN counters
constexpr size_t kStatusBytes = 256;                    // router-only calls
constexpr size_t kFfnStatusBytes = kStatusInts * sizeof(int);


kmoe_status fail(kmoe_status code, const char *fmt, ...)
{
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(g_err, sizeof g_err, fmt, ap);
    va_end(ap);
    return code;
}

void clear_error() { g_err[0] = '\0'; }

kmoe_status check_launch(const char *what)
{
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return fail(KMOE_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
    return KMOE_OK;
}

// ------------------------------------------------------------ validation

static kmoe_status check_sizes(int N, int d, int E, int K, int I)
{
    if (N < 0) return fail(KMOE_ERR_INVALID_ARG, "N=%d must be >= 0", N);
    if (K < 1 || K > 8) return fail(KMOE_ERR_UNSUPPORTED, "K=%d: supported 1 <= K <= 8", K);
    if (E < K) return fail(KMOE_ERR_INVALID_ARG, "E=%d must be >= K=%d", E, K);
    if (E > 1024) return fail(KMOE_ERR_UNSUPPORTED, "E=%d: supported E <= 1024", E);
    if (d < 128 || d % 128 || d > 6144)
        return fail(KMOE_ERR_UNSUPPORTED, "d=%d: must be a multiple of 128 in [128, 6144]", d);
    if (I >= 0 && (I < 128 || I % 128 || I > 4096))
        return fail(KMOE_ERR_UNSUPPORTED, "I=%d: must be a multiple of 128 in [128, 4096]", I);
    if ((long long)N * K > (1LL << 30)) return fail(KMOE_ERR_UNSUPPORTED, "N*K too large");
    return KMOE_OK;
}

static kmoe_status check_ptr(const void *p, const char *name, bool nullable = false)
{
    if (!p) return nullable ? KMOE_OK : fail(KMOE_ERR_INVALID_ARG, "%s is NULL", name);
    if (!aligned16(p)) return fail(KMOE_ERR_INVALID_ARG, "%s is not 16-byte aligned", name);
    return KMOE_OK;
}

#define KMOE_TRY(expr)                          \
    do {                                        \
        kmoe_status s_ = (expr);                \
        if (s_ != KMOE_OK) return s_;           \
    } while (0)

static kmoe_status check_act_dtype(int t, const char *name)
{
    if (t != KMOE_F32 && t != KMOE_BF16) return fail(KMOE_ERR_UNSUPPORTED, "%s dtype %d: F32 or BF16 only", name, t);
    return KMOE_OK;
}

// E4M3 weights with FP32 128 x 128 block scales (BF16 or FP8 activations).
static bool fp8_weights(int w_dtype) { return w_dtype == KMOE_E4M3_B128 || w_dtype == KMOE_E4M3_B128_A8; }

static bool known_w_dtype(int w_dtype) { return w_dtype == KMOE_F32 || w_dtype == KMOE_BF16 || fp8_weights(w_dtype); }

// FP8 activations need BF16 x and d % 256 == 0 (the FP8 FFN's down units);
// checked on the host before anything is enqueued.
static kmoe_status check_a8(int x_dtype, int d, int w_dtype)
{
    if (w_dtype == KMOE_E4M3_B128_A8 && (x_dtype != KMOE_BF16 || d % 256))
        return fail(KMOE_ERR_UNSUPPORTED, "FP8 activations: x must be BF16 and d (%d) a multiple of 256", d);
    return KMOE_OK;
}

static kmoe_status check_experts(const kmoe_experts *x, const char *name)
{
    if (!x) return fail(KMOE_ERR_INVALID_ARG, "%s is NULL", name);
    if (x->dtype != KMOE_F32 && x->dtype != KMOE_BF16 && !fp8_weights(x->dtype))
        return fail(KMOE_ERR_UNSUPPORTED, "%s dtype %d unknown", name, x->dtype);
    KMOE_TRY(check_ptr(x->w_gate, "w_gate"));
    KMOE_TRY(check_ptr(x->w_up, "w_up"));
    KMOE_TRY(check_ptr(x->w_down, "w_down"));
    if (fp8_weights(x->dtype)) {
        KMOE_TRY(check_ptr(x->s_gate, "s_gate"));
        KMOE_TRY(check_ptr(x->s_up, "s_up"));
        KMOE_TRY(check_ptr(x->s_down, "s_down"));
    }
    return KMOE_OK;
}

static ExpertPtrs ptrs(const kmoe_experts *x)
{
    ExpertPtrs p{x->w_gate, x->w_up, x->w_down, nullptr, nullptr, nullptr};
    if (fp8_weights(x->dtype)) {
        p.sg = x->s_gate;
        p.su = x->s_up;
        p.sd = x->s_down;
    }
    return p;
}

static size_t act_bytes(int w_dtype) { return w_dtype == KMOE_F32 ? 4 : 2; }

// Bytes of one H element: the output dtype, or an E4M3 code with FP8 activations.
static size_t h_bytes(int w_dtype) { return w_dtype == KMOE_E4M3_B128_A8 ? 1 : act_bytes(w_dtype); }

// Batches that run E4M3 weights on the FP8 tensor cores with two-term
// (BF16-precision) activations: below kTcMinTokens tokens.
static bool two_term(int w_dtype, int N) { return w_dtype == KMOE_E4M3_B128 && N < kTcMinTokens; }

// The grouped FFN's scratch after the status block: H [N*K + N, I] and, with
// FP8 activations, H's scales [N*K + N, I / 128], x's codes [N, d] and x's
// scales [N, d / 128]. In two-term mode H's two bytes per element are its
// high and low code planes (each [N*K + N, I]) and x has low codes as well.
struct FfnScratch {
    void *h;
    float *hs;
    uint8_t *xq, *xl;
    float *xs;
};

static FfnScratch take_ffn_scratch(Carver &c, int N, int d, int K, int I, int w_dtype)
{
    const size_t R = (size_t)N * K + N;
    FfnScratch f{};
    f.h = c.take<char>(R * I * h_bytes(w_dtype));
    if (w_dtype == KMOE_E4M3_B128_A8 || two_term(w_dtype, N)) {
        f.hs = c.take<float>(R * (I / 128));
        f.xq = c.take<uint8_t>((size_t)N * d);
        if (two_term(w_dtype, N)) f.xl = c.take<uint8_t>((size_t)N * d);
        f.xs = c.take<float>((size_t)N * (d / 128));
    }
    return f;
}

// Bytes of a moe_grouped_ffn workspace: the status block, then the scratch.
static size_t ffn_ws_bytes(int N, int d, int K, int I, int w_dtype)
{
    Carver c(nullptr);
    c.take<int>(kStatusInts);
    take_ffn_scratch(c, N, d, K, I, w_dtype);
    return c.used;
}

// Give-up limit of the pipeline waits of the FFN kernels this thread
// launches (moe_set_wait_limit; 0 = the default).
static thread_local long long g_wait_limit = 0;
static long long wait_limit() { return g_wait_limit > 0 ? g_wait_limit : kDefaultWaitLimit; }

// Workspace of the whole forward; every entry point uses a prefix-compatible
// subset (router: logits; permute: chunk histograms; grouped FFN: H).
struct Layout {
    int *status;
    float *logits;
    int32_t *idx;
    float *w;
    int32_t *counts, *offsets, *perm, *inv, *hist;
    __nv_bfloat16 *w_split;
    FfnScratch ffn;
    void *y_perm, *y_shared;
    __nv_bfloat16 *x_norm;   // sandwich block only: the normalised layer input
    size_t bytes;
};

static Layout layout(void *ws, int N, int d, int E, int K, int I, int w_dtype, bool block = false)
{
    Carver c(ws);
    Layout L;
    const size_t ab = act_bytes(w_dtype);
    L.status = c.take<int>(kStatusInts);
    L.logits = c.take<float>((size_t)N * E);
    L.idx = c.take<int32_t>((size_t)N * K);
    L.w = c.take<float>((size_t)N * K);
    L.counts = c.take<int32_t>(E);
    L.offsets = c.take<int32_t>(E + 1);
    L.perm = c.take<int32_t>((size_t)N * K);
    L.inv = c.take<int32_t>((size_t)N * K);
    L.hist = reinterpret_cast<int32_t *>(c.take<char>(permute_ws_bytes(N, E)));
    L.w_split = c.take<__nv_bfloat16>(router_tc_ws_bytes(d, E) / sizeof(__nv_bfloat16));
    L.ffn = take_ffn_scratch(c, N, d, K, I, w_dtype);
    L.y_perm = c.take<char>((size_t)N * K * d * ab);
    L.y_shared = c.take<char>((size_t)N * d * ab);
    L.x_norm = block ? c.take<__nv_bfloat16>((size_t)N * d) : nullptr;
    L.bytes = c.used + 256;
    return L;
}

// Grouped FFN kernel for a batch (BF16 activations, BF16 or E4M3 weights,
// d % 256 == 0): below kTcMinTokens tokens the swap-AB tcgen05 kernel
// (weights as M, 16-token chunks as N) for BF16 weights and the FP8
// tensor-core kernel in two-term mode for E4M3 weights, from there the
// tokens-as-M tcgen05 kernel; FP32 activations or weights take the CUDA-core
// streaming kernel. FP8 activations (KMOE_E4M3_B128_A8) take the FP8
// tensor-core kernel at every batch size.
enum FfnPath { kPathStream, kPathSwap, kPathTc, kPathA8, kPathTwo };

static FfnPath ffn_path(int x_dtype, int w_dtype, int N, int d)
{
    if (w_dtype == KMOE_E4M3_B128_A8) return kPathA8;
    if (x_dtype != KMOE_BF16 || (w_dtype != KMOE_BF16 && w_dtype != KMOE_E4M3_B128) || d % 256) return kPathStream;
    if (two_term(w_dtype, N)) return kPathTwo;
    return N < kTcMinTokens ? kPathSwap : kPathTc;
}

// `status` is the workspace status block: the status word, tickets, then
// kSyncInts counters at kSyncOffset (all zeroed by clear_status).
static kmoe_status run_ffn(const void *x, int x_dtype, int N, int d, int I, int E, int K, const int32_t *perm,
                           const int32_t *offsets, int w_dtype, const ExpertPtrs &r, const ExpertPtrs *s,
                           const FfnScratch &f, void *y_perm, void *y_shared, int *status, cudaStream_t st)
{
    const FfnPath path = ffn_path(x_dtype, w_dtype, N, d);
    void *h = f.h;
    if (path == kPathA8) {
        if (x_dtype != KMOE_BF16 || d % 256)
            return fail(KMOE_ERR_UNSUPPORTED, "FP8 activations: x must be BF16 and d a multiple of 256");
        KMOE_TRY(launch_quant_1x128(static_cast<const __nv_bfloat16 *>(x), N, d, f.xq, f.xs, st));
        return launch_ffn_a8(f.xq, f.xs, N, d, I, E, K, perm, offsets, r, s, static_cast<uint8_t *>(h), f.hs,
                             static_cast<__nv_bfloat16 *>(y_perm), static_cast<__nv_bfloat16 *>(y_shared), status,
                             status + kSyncOffset, wait_limit(), st);
    }
    if (path == kPathTwo) {
        const size_t R = (size_t)N * K + N;
        uint8_t *hq = static_cast<uint8_t *>(h), *hl = hq + R * I;
        KMOE_TRY(launch_quant_1x128_split(static_cast<const __nv_bfloat16 *>(x), N, d, f.xq, f.xl, f.xs, st));
        return launch_ffn_a8(f.xq, f.xs, N, d, I, E, K, perm, offsets, r, s, hq, f.hs,
                             static_cast<__nv_bfloat16 *>(y_perm), static_cast<__nv_bfloat16 *>(y_shared), status,
                             status + kSyncOffset, wait_limit(), st, f.xl, hl);
    }
    if (path == kPathSwap)
        return launch_ffn_swap(static_cast<const __nv_bfloat16 *>(x), N, d, I, E, K, perm, offsets, r, s,
                               static_cast<__nv_bfloat16 *>(h), static_cast<__nv_bfloat16 *>(y_perm),
                               static_cast<__nv_bfloat16 *>(y_shared), status, status + kSyncOffset, wait_limit(), st);
    if (path == kPathTc)
        return launch_ffn_tc(static_cast<const __nv_bfloat16 *>(x), N, d, I, E, K, perm, offsets, w_dtype, r, s,
                             static_cast<__nv_bfloat16 *>(h), static_cast<__nv_bfloat16 *>(y_perm),
                             static_cast<__nv_bfloat16 *>(y_shared), status, status + kSyncOffset, wait_limit(), st);
    return launch_ffn_stream(x, x_dtype, N, d, I, E, K, perm, offsets, w_dtype, r, s, h, y_perm, y_shared, st);
}

static kmoe_status clear_status(int *status, cudaStream_t st, size_t bytes = kStatusBytes)
{
    // status word, tickets and counters of this call's kernels
    if (cudaMemsetAsync(status, 0, bytes, st) != cudaSuccess) return check_launch("status memset");
    return KMOE_OK;
}

constexpr int kSmallRouteTokens = 256;   // small-batch router (bulk-copied token rows) up to here
constexpr int kChunkTokens = 256;        // the dispatch works in chunks of this many tokens

static kmoe_status check_score(int score)
{
    if (score != KMOE_SCORE_SIGMOID && score != KMOE_SCORE_SOFTMAX)
        return fail(KMOE_ERR_INVALID_ARG, "score %d: KMOE_SCORE_SIGMOID or KMOE_SCORE_SOFTMAX", score);
    return KMOE_OK;
}

// Validation shared by moe_forward and moe_block_forward.
static kmoe_status check_forward(int N, int d, int E, int K, int I, int score, const kmoe_experts *routed,
                                 const kmoe_experts *shared, const float *w_router, const float *bias,
                                 int32_t *topk_idx_out, float *topk_w_out, int32_t *counts_out, void *ws)
{
    KMOE_TRY(check_sizes(N, d, E, K, I));
    KMOE_TRY(check_score(score));
    KMOE_TRY(check_experts(routed, "routed"));
    if (shared) {
        KMOE_TRY(check_experts(shared, "shared"));
        if (shared->dtype != routed->dtype) return fail(KMOE_ERR_UNSUPPORTED, "shared and routed dtypes differ");
    }
    if (N == 0) return KMOE_OK;
    KMOE_TRY(check_ptr(w_router, "w_router"));
    KMOE_TRY(check_ptr(bias, "bias"));
    KMOE_TRY(check_ptr(topk_idx_out, "topk_idx_out", true));
    KMOE_TRY(check_ptr(topk_w_out, "topk_w_out", true));
    KMOE_TRY(check_ptr(counts_out, "counts_out", true));
    return check_ptr(ws, "ws");
}

// Routing, dispatch, expert FFNs and combine of one layer call on laid-out
// workspace L; with h_res set the combine also applies the post-norm and the
// residual addition of the sandwich block. The status block must be zero
// before the first kernel that uses it: the caller clears it, except for
// batches of the small-batch router (N <= kSmallRouteTokens), whose kernel
// zeroes it itself (no memset between this call's kernels and the previous
// call's, so the programmatic launch chain carries over).
static bool router_zeroes_status(int N) { return N <= kSmallRouteTokens; }

static kmoe_status forward_path(const void *x, int x_dtype, int N, int d, int E, int K, int I, int score,
                                const float *w_router, const float *bias, const kmoe_experts *routed,
                                const kmoe_experts *shared, void *y, int y_dtype, int32_t *topk_idx_out,
                                float *topk_w_out, int32_t *counts_out, const Layout &L, const void *h_res,
                                const void *g_post, float eps, cudaStream_t st)
{
    int32_t *idx = topk_idx_out ? topk_idx_out : L.idx;
    float *w = topk_w_out ? topk_w_out : L.w;
    int32_t *counts = counts_out ? counts_out : L.counts;
    // logits, then top-K (one warp per token), then the dispatch permutation;
    // above one chunk the top-K kernel also counts the chunk histograms
    const bool chunked = N > kChunkTokens;
    if (chunked && cudaMemsetAsync(L.hist, 0, permute_ws_bytes(N, E), st) != cudaSuccess)
        return check_launch("histogram memset");
    if (N <= kSmallRouteTokens)
        KMOE_TRY(launch_router_small(x, x_dtype, w_router, N, d, E, L.logits, L.status, st, kStatusInts));
    else if (x_dtype == KMOE_BF16 && N >= kTcRouterTokens)
        KMOE_TRY(launch_router_tc(static_cast<const __nv_bfloat16 *>(x), w_router, N, d, E, L.w_split, L.logits,
                                  L.status, st));
    else
        KMOE_TRY(launch_router_logits(x, x_dtype, w_router, N, d, E, L.logits, st));
    KMOE_TRY(launch_topk(L.logits, bias, N, E, K, score, idx, w, st, chunked ? L.hist : nullptr));
    KMOE_TRY(launch_permute(idx, N, K, E, counts, L.offsets, L.perm, L.inv, L.hist, st, chunked));
    const ExpertPtrs r = ptrs(routed);
    ExpertPtrs s{};
    if (shared) s = ptrs(shared);
    KMOE_TRY(run_ffn(x, x_dtype, N, d, I, E, K, L.perm, L.offsets, routed->dtype, r, shared ? &s : nullptr,
                     L.ffn, L.y_perm, L.y_shared, L.status, st));
    const int yin = routed->dtype == KMOE_F32 ? KMOE_F32 : KMOE_BF16;
    return launch_combine(L.y_perm, shared ? L.y_shared : nullptr, yin, w, L.inv, N, K, d, y, y_dtype, L.status, st,
                          h_res, g_post, eps);
}

}  // namespace kmoe

using namespace kmoe;

extern "C" {

int moe_abi_version(void) { return KMOE_ABI_VERSION; }

const char *moe_last_error(void) { return g_err; }

size_t moe_workspace_size(int N, int d, int E, int K, int I, int x_dtype, int w_dtype)
{
    if (check_sizes(N, d, E, K, I) != KMOE_OK) return 0;
    if (check_act_dtype(x_dtype, "x") != KMOE_OK) return 0;
    if (!known_w_dtype(w_dtype)) return 0;
    clear_error();
    return layout(nullptr, N, d, E, K, I, w_dtype).bytes;
}


kmoe_status moe_router_topk(const void *x, int x_dtype, const float *w_router, const float *bias,
                            int N, int d, int E, int K, int score, float *logits, int32_t *topk_idx,
                            float *topk_w, void *ws, size_t ws_bytes, void *stream)
{
    clear_error();
    KMOE_TRY(check_sizes(N, d, E, K, -1));
    KMOE_TRY(check_score(score));
    KMOE_TRY(check_act_dtype(x_dtype, "x"));
    if (N == 0) return KMOE_OK;
    KMOE_TRY(check_ptr(x, "x"));
    KMOE_TRY(check_ptr(w_router, "w_router"));
    KMOE_TRY(check_ptr(bias, "bias"));
    KMOE_TRY(check_ptr(topk_idx, "topk_idx"));
    KMOE_TRY(check_ptr(topk_w, "topk_w"));
    KMOE_TRY(check_ptr(logits, "logits", true));
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    KMOE_TRY(check_ptr(ws, "ws", logits != nullptr));
    // workspace: [logits if not supplied][status 256 B][three BF16 weight terms]
    size_t used = 0;
    if (!logits) {
        if (ws_bytes < (size_t)N * E * sizeof(float))
            return fail(KMOE_ERR_WORKSPACE, "workspace %zu < %zu bytes", ws_bytes, (size_t)N * E * sizeof(float));
        logits = static_cast<float *>(ws);
        used = ((size_t)N * E * sizeof(float) + 255) & ~size_t(255);
    }
    const size_t tc_need = used + kStatusBytes + router_tc_ws_bytes(d, E);
    if (x_dtype == KMOE_BF16 && N >= kTcRouterTokens && ws && ws_bytes >= tc_need) {
        int *status = reinterpret_cast<int *>(static_cast<char *>(ws) + used);
        KMOE_TRY(clear_status(status, st));
        KMOE_TRY(launch_router_tc(static_cast<const __nv_bfloat16 *>(x), w_router, N, d, E,
                                  reinterpret_cast<__nv_bfloat16 *>(reinterpret_cast<char *>(status) + kStatusBytes),
                                  logits, status, st));
    } else {
        KMOE_TRY(launch_router_logits(x, x_dtype, w_router, N, d, E, logits, st));
    }
    return launch_topk(logits, bias, N, E, K, score, topk_idx, topk_w, st);
}

kmoe_status moe_permute(const int32_t *topk_idx, int N, int K, int E, int32_t *counts,
                        int32_t *offsets, int32_t *perm_token, int32_t *inv_pos, void *ws,
                        size_t ws_bytes, void *stream)
{
    clear_error();
    KMOE_TRY(check_sizes(N, 128, E, K, -1));
    KMOE_TRY(check_ptr(counts, "counts"));
    KMOE_TRY(check_ptr(offsets, "offsets"));
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (N == 0) {
        if (cudaMemsetAsync(counts, 0, sizeof(int32_t) * E, st) != cudaSuccess ||
            cudaMemsetAsync(offsets, 0, sizeof(int32_t) * (E + 1), st) != cudaSuccess)
            return check_launch("permute memset");
        return KMOE_OK;
    }
    KMOE_TRY(check_ptr(topk_idx, "topk_idx"));
    KMOE_TRY(check_ptr(perm_token, "perm_token"));
    KMOE_TRY(check_ptr(inv_pos, "inv_pos"));
    const size_t need = permute_ws_bytes(N, E);
    if (N > 256) {
        KMOE_TRY(check_ptr(ws, "ws"));
        if (ws_bytes < need) return fail(KMOE_ERR_WORKSPACE, "workspace %zu < %zu bytes", ws_bytes, need);
    }
    return launch_permute(topk_idx, N, K, E, counts, offsets, perm_token, inv_pos,
                          static_cast<int32_t *>(ws), st);
}

kmoe_status moe_grouped_ffn(const void *x, int x_dtype, int N, int d, int I, int E, int K,
                            const int32_t *perm_token, const int32_t *offsets,
                            const kmoe_experts *routed, const kmoe_experts *shared, void *y_perm,
                            void *y_shared, void *ws, size_t ws_bytes, void *stream)
{
    clear_error();
    KMOE_TRY(check_sizes(N, d, E, K, I));
    KMOE_TRY(check_act_dtype(x_dtype, "x"));
    KMOE_TRY(check_experts(routed, "routed"));
    if (shared) {
        KMOE_TRY(check_experts(shared, "shared"));
        if (shared->dtype != routed->dtype) return fail(KMOE_ERR_UNSUPPORTED, "shared and routed dtypes differ");
    }
    KMOE_TRY(check_a8(x_dtype, d, routed->dtype));
    if (N == 0) return KMOE_OK;
    KMOE_TRY(check_ptr(x, "x"));
    KMOE_TRY(check_ptr(perm_token, "perm_token"));
    KMOE_TRY(check_ptr(offsets, "offsets"));
    KMOE_TRY(check_ptr(y_perm, "y_perm"));
    if (shared) KMOE_TRY(check_ptr(y_shared, "y_shared"));
    KMOE_TRY(check_ptr(ws, "ws"));
    const size_t need = ffn_ws_bytes(N, d, K, I, routed->dtype);
    if (ws_bytes < need) return fail(KMOE_ERR_WORKSPACE, "workspace %zu < %zu bytes", ws_bytes, need);
    const ExpertPtrs r = ptrs(routed);
    ExpertPtrs s{};
    if (shared) s = ptrs(shared);
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    Carver c(ws);
    int *status = c.take<int>(kStatusInts);
    const FfnScratch f = take_ffn_scratch(c, N, d, K, I, routed->dtype);
    KMOE_TRY(clear_status(status, st, kFfnStatusBytes));
    return run_ffn(x, x_dtype, N, d, I, E, K, perm_token, offsets, routed->dtype, r, shared ? &s : nullptr, f,
                   y_perm, y_shared, status, st);
}

kmoe_status moe_combine(const void *y_perm, const void *y_shared, int y_in_dtype, const float *topk_w,
                        const int32_t *inv_pos, int N, int K, int d, void *y, int y_dtype, void *stream)
{
    clear_error();
    KMOE_TRY(check_sizes(N, d, K, K, -1));
    KMOE_TRY(check_act_dtype(y_in_dtype, "y_in"));
    KMOE_TRY(check_act_dtype(y_dtype, "y"));
    if (N == 0) return KMOE_OK;
    KMOE_TRY(check_ptr(y_perm, "y_perm"));
    KMOE_TRY(check_ptr(y_shared, "y_shared", true));
    KMOE_TRY(check_ptr(topk_w, "topk_w"));
    KMOE_TRY(check_ptr(inv_pos, "inv_pos"));
    KMOE_TRY(check_ptr(y, "y"));
    return launch_combine(y_perm, y_shared, y_in_dtype, topk_w, inv_pos, N, K, d, y, y_dtype, nullptr,
                          static_cast<cudaStream_t>(stream));
}

kmoe_status moe_forward(const void *x, int x_dtype, int N, int d, int E, int K, int I, int score,
                        const float *w_router, const float *bias, const kmoe_experts *routed,
                        const kmoe_experts *shared, void *y, int y_dtype, int32_t *topk_idx_out,
                        float *topk_w_out, int32_t *counts_out, void *ws, size_t ws_bytes, void *stream)
{
    clear_error();
    KMOE_TRY(check_act_dtype(x_dtype, "x"));
    KMOE_TRY(check_act_dtype(y_dtype, "y"));
    KMOE_TRY(check_forward(N, d, E, K, I, score, routed, shared, w_router, bias, topk_idx_out, topk_w_out, counts_out,
                           ws));
    KMOE_TRY(check_a8(x_dtype, d, routed->dtype));
    if (N == 0) return KMOE_OK;
    KMOE_TRY(check_ptr(x, "x"));
    KMOE_TRY(check_ptr(y, "y"));
    const Layout need = layout(nullptr, N, d, E, K, I, routed->dtype);
    if (ws_bytes < need.bytes) return fail(KMOE_ERR_WORKSPACE, "workspace %zu < %zu bytes", ws_bytes, need.bytes);
    // the base the Carver sees is 256-aligned by construction of the pieces
    const Layout L = layout(ws, N, d, E, K, I, routed->dtype);
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (!router_zeroes_status(N)) KMOE_TRY(clear_status(L.status, st, kFfnStatusBytes));
    return forward_path(x, x_dtype, N, d, E, K, I, score, w_router, bias, routed, shared, y, y_dtype, topk_idx_out,
                        topk_w_out, counts_out, L, nullptr, nullptr, 0.f, st);
}

size_t moe_block_workspace_size(int N, int d, int E, int K, int I, int w_dtype)
{
    if (check_sizes(N, d, E, K, I) != KMOE_OK) return 0;
    if (w_dtype != KMOE_BF16 && !fp8_weights(w_dtype)) return 0;
    clear_error();
    return layout(nullptr, N, d, E, K, I, w_dtype, true).bytes;
}

kmoe_status moe_block_forward(const void *h, int N, int d, int E, int K, int I, int score, const void *gamma_pre,
                              const void *gamma_post, float eps, const float *w_router, const float *bias,
                              const kmoe_experts *routed, const kmoe_experts *shared, void *h_out,
                              void *x_out, int32_t *topk_idx_out, float *topk_w_out, int32_t *counts_out, void *ws,
                              size_t ws_bytes, void *stream)
{
    clear_error();
    KMOE_TRY(check_forward(N, d, E, K, I, score, routed, shared, w_router, bias, topk_idx_out, topk_w_out, counts_out,
                           ws));
    if (routed->dtype != KMOE_BF16 && !fp8_weights(routed->dtype))
        return fail(KMOE_ERR_UNSUPPORTED, "block: routed weights must be BF16 or E4M3 with 128x128 scales");
    if (!(eps >= 0.f) || eps > 1.f) return fail(KMOE_ERR_INVALID_ARG, "eps=%g: must be in [0, 1]", (double)eps);
    if (d % 256) return fail(KMOE_ERR_UNSUPPORTED, "block: d=%d must be a multiple of 256", d);
    const size_t row_smem = (size_t)(K + (shared ? 1 : 0)) * d * 2;
    if (2 * row_smem > 100 * 1024)
        return fail(KMOE_ERR_UNSUPPORTED, "block: (K + 1) * d = %zu BF16 values per token exceed the combine's "
                    "staging buffer", row_smem / 2);
    if (N == 0) return KMOE_OK;
    KMOE_TRY(check_ptr(h, "h"));
    KMOE_TRY(check_ptr(gamma_pre, "gamma_pre"));
    KMOE_TRY(check_ptr(gamma_post, "gamma_post"));
    KMOE_TRY(check_ptr(h_out, "h_out"));
    KMOE_TRY(check_ptr(x_out, "x_out", true));
    const Layout need = layout(nullptr, N, d, E, K, I, routed->dtype, true);
    if (ws_bytes < need.bytes) return fail(KMOE_ERR_WORKSPACE, "workspace %zu < %zu bytes", ws_bytes, need.bytes);
    const Layout L = layout(ws, N, d, E, K, I, routed->dtype, true);
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (!router_zeroes_status(N)) KMOE_TRY(clear_status(L.status, st, kFfnStatusBytes));
    __nv_bfloat16 *x = x_out ? static_cast<__nv_bfloat16 *>(x_out) : L.x_norm;
    KMOE_TRY(launch_rmsnorm(static_cast<const __nv_bfloat16 *>(h), static_cast<const __nv_bfloat16 *>(gamma_pre), eps,
                            N, d, x, st));
    return forward_path(x, KMOE_BF16, N, d, E, K, I, score, w_router, bias, routed, shared, h_out, KMOE_BF16,
                        topk_idx_out, topk_w_out, counts_out, L, h, gamma_post, eps, st);
}

kmoe_status moe_quant_1x128(const void *x, int rows, int cols, uint8_t *codes, float *scales, void *stream)
{
    clear_error();
    if (rows < 0) return fail(KMOE_ERR_INVALID_ARG, "rows=%d must be >= 0", rows);
    if (cols < 128 || cols % 128) return fail(KMOE_ERR_UNSUPPORTED, "cols=%d: must be a positive multiple of 128", cols);
    if (rows == 0) return KMOE_OK;
    KMOE_TRY(check_ptr(x, "x"));
    KMOE_TRY(check_ptr(codes, "codes"));
    KMOE_TRY(check_ptr(scales, "scales"));
    return launch_quant_1x128(static_cast<const __nv_bfloat16 *>(x), rows, cols, codes, scales,
                              static_cast<cudaStream_t>(stream));
}

kmoe_status moe_set_wait_limit(long long cycles)
{
    clear_error();
    if (cycles < 0) return fail(KMOE_ERR_INVALID_ARG, "wait limit %lld cycles must be >= 0", cycles);
    g_wait_limit = cycles;
    return KMOE_OK;
}

kmoe_status moe_device_status(const void *ws, int *status, void *stream)
{
    clear_error();
    KMOE_TRY(check_ptr(ws, "ws"));
    if (!status) return fail(KMOE_ERR_INVALID_ARG, "status is NULL");
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (cudaMemcpyAsync(status, ws, sizeof(int), cudaMemcpyDeviceToHost, st) != cudaSuccess ||
        cudaStreamSynchronize(st) != cudaSuccess)
        return check_launch("device status read");
    if (*status != 0) return fail(KMOE_ERR_DEVICE, "device status %d: a pipeline wait gave up", *status);
    return KMOE_OK;
}

}  // extern "C"
