/*
 * kmoe — C ABI of the fine-grained sparse MoE feed-forward layer for NVIDIA
 * B200 (sm_100a).
 *
 * The layer (page "Inside Kolibri 1: Hybrid RNoPE Attention, Sparse MoE, and
 * FP8 Serving", flozi.net, section "Routing: selection bias and mixture
 * weights are separate"):
 *   l      = x W_r^T                        FP32 logits [N, E]
 *   idx    = top-K of (l + b) per token     b: learned expert-correction bias
 *   g      = sigmoid(l[idx])                unbiased logits, not renormalised
 *   F_e(x) = W_d,e (SiLU(W_g,e x) * (W_u,e x))   SwiGLU expert, no biases
 *   y      = F_shared(x) + sum_k g_k F_{idx_k}(x)
 * With the Kolibri-1 shape: d = 2560, E = 384 routed experts, K = 6, one
 * shared expert, I = 512. FP8 weights (same page, section "The FP8 path is
 * explicitly mixed precision") are E4M3 in 128 x 128 blocks with one FP32
 * scale per block; scales are used as stored (never rounded to 2^k).
 *
 * Conventions shared by every entry point:
 *   - Pointers marked "device" point to GPU global memory owned by the
 *     caller; the library never allocates or frees device memory and keeps
 *     no state between calls other than a per-thread error message and
 *     give-up limit (moe_set_wait_limit); moe_permute_noalloc works in the
 *     library's own static device array (see there).
 *   - `stream` is a cudaStream_t (NULL = legacy default stream). Work is
 *     enqueued asynchronously; no entry point synchronises the device.
 *   - Matrices are dense row-major. Every device pointer must be 16-byte
 *     aligned.
 *   - Sizes: 1 <= K <= 8, K <= E <= 1024, d and I multiples of 128 (needed by
 *     the 128 x 128 FP8 blocks and the tensor-core tiles) with d <= 6144 and
 *     I <= 4096, N >= 0. N == 0 is a successful no-op.
 *   - Return value: KMOE_OK, or an error code with a message available from
 *     moe_last_error(). Argument errors are detected on the host before any
 *     work is enqueued. KMOE_ERR_CUDA reports a failed launch.
 *   - Inputs are assumed finite.
 */
#ifndef KMOE_H
#define KMOE_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    KMOE_OK = 0,
    KMOE_ERR_INVALID_ARG = 1,   /* null / misaligned pointer, bad size */
    KMOE_ERR_UNSUPPORTED = 2,   /* size or dtype combination not compiled */
    KMOE_ERR_CUDA = 3,          /* a CUDA launch or runtime call failed */
    KMOE_ERR_WORKSPACE = 4,     /* workspace smaller than moe_workspace_size() */
    KMOE_ERR_DEVICE = 5         /* a kernel reported a failure in the device status word */
} kmoe_status;

/*
 * Mixture weights of the K chosen experts, from their unbiased logits l:
 *   KMOE_SCORE_SIGMOID  g_k = 1 / (1 + exp(-l_k)), not renormalised
 *                       ("Inside Kolibri 1", routing section; the default);
 *   KMOE_SCORE_SOFTMAX  g_k = exp(l_k) / sum_j exp(l_j) over the K chosen
 *                       ("Kolibri 1 Deep Dive", section "Mathematical Routing
 *                       & Load Balancing Formulation"). The selection itself
 *                       (top-K of l + bias) is the same for both.
 */
typedef enum {
    KMOE_SCORE_SIGMOID = 0,
    KMOE_SCORE_SOFTMAX = 1
} kmoe_score;

typedef enum {
    KMOE_F32 = 0,           /* IEEE binary32 */
    KMOE_BF16 = 1,          /* bfloat16 */
    KMOE_E4M3_B128 = 2,     /* OCP E4M3 bytes + one FP32 scale per 128x128 block */
    KMOE_E4M3_B128_A8 = 3   /* expert weights only: stored exactly as KMOE_E4M3_B128, and
                               the expert GEMMs run on FP8 activations ("Inside Kolibri 1",
                               FP8 section: activations quantised dynamically in groups of
                               1 x 128). x (BF16) is quantised per row and 128 columns:
                               scale = amax / 448 in FP32 (1 for an all-zero group), code =
                               E4M3(x / scale) with the quotient in FP32, round to nearest
                               even, saturated; H is rounded to BF16 and quantised with the
                               same scale rule before the down projection, its codes taken
                               from h * (1 / scale) in FP32 (at most one code step from
                               E4M3(h / scale), where that quotient lies within 2^-23 of a
                               rounding boundary). Each 128-column K block's
                               E4M3 x E4M3 partial sums (FP32) are scaled by both FP32
                               block scales and added in FP32. Routing sees x as given. */
} kmoe_dtype;

/*
 * One stack of G SwiGLU experts (routed: G = E; shared: G = 1).
 *   w_gate, w_up : device [G, I, d]  row i = weights of intermediate feature i
 *   w_down       : device [G, d, I]  row j = weights of output feature j
 *   s_gate, s_up : device [G, I/128, d/128] FP32 block scales (E4M3 only,
 *   s_down       : device [G, d/128, I/128]  else ignored and may be NULL)
 * The weight value of an E4M3 element is decode(q) * scale of its block.
 */
typedef struct {
    const void *w_gate;
    const void *w_up;
    const void *w_down;
    const float *s_gate;
    const float *s_up;
    const float *s_down;
    int dtype;           /* kmoe_dtype of the weights */
} kmoe_experts;

/*
 * Bytes of device workspace that any entry point below needs for these
 * sizes (x_dtype: activations; w_dtype: expert weights). Pass a buffer of at
 * least this size as `ws` (contents need not be initialised; the library
 * overwrites what it uses). Returns 0 for unsupported arguments.
 */
size_t moe_workspace_size(int N, int d, int E, int K, int I, int x_dtype, int w_dtype);

/*
 * Router and selection ("Inside Kolibri 1", routing section, steps 1-2):
 *   logits[t][e] = sum_j x[t][j] * w_router[e][j]        (FP32 accumulate)
 *   topk_idx[t]  = the K experts with the largest logits[t][e] + bias[e],
 *                  ordered by that biased score, highest first; on equal
 *                  scores the lower expert index wins
 *   topk_w[t][k] = 1 / (1 + exp(-logits[t][topk_idx[t][k]]))   (score KMOE_SCORE_SIGMOID),
 *                  or the softmax of the K chosen logits      (score KMOE_SCORE_SOFTMAX)
 * x        device [N, d], x_dtype KMOE_F32 or KMOE_BF16
 * w_router device [E, d] FP32;   bias device [E] FP32
 * logits   device [N, E] FP32 output, or NULL to keep it in the workspace
 * topk_idx device [N, K] int32 output;  topk_w device [N, K] FP32 output
 * ws       device workspace (may be NULL when logits is given). With BF16 x,
 *          N >= 512 and a workspace of at least moe_workspace_size() bytes,
 *          the logits run on the tensor cores: W_r is split into three BF16
 *          terms (W1 = bf16(W), W2 = bf16(W - W1), W3 = bf16(W - W1 - W2))
 *          whose exact products accumulate in FP32, otherwise on CUDA cores
 *          in FP32. Its status word is read by moe_device_status on
 *          (ws + the logits bytes rounded up to 256 when logits is NULL).
 */
kmoe_status moe_router_topk(const void *x, int x_dtype, const float *w_router,
                            const float *bias, int N, int d, int E, int K, int score,
                            float *logits, int32_t *topk_idx, float *topk_w,
                            void *ws, size_t ws_bytes, void *stream);

/*
 * Dispatch: histogram, exclusive scan and a stable permutation of the N*K
 * (token, slot) pairs by expert. The pages state only that tokens are sent
 * to their selected experts (routing section); the order here is grouped by
 * expert ascending and, inside one expert, by token ascending, which makes
 * every output a deterministic function of topk_idx (bit-exact).
 *   counts[e]      = #{(t,k) : topk_idx[t][k] == e}
 *   offsets[e]     = sum_{e' < e} counts[e'],  offsets[E] = N*K
 *   perm_token[p]  = token of dispatched row p
 *   inv_pos[t][k]  = dispatched row of (t, k)
 * topk_idx device [N, K] int32, each row holding K distinct values in
 * [0, E); out-of-range values are skipped (outputs then unspecified).
 * counts device [E], offsets device [E+1], perm_token device [N*K],
 * inv_pos device [N, K]: int32 outputs.
 */
kmoe_status moe_permute(const int32_t *topk_idx, int N, int K, int E,
                        int32_t *counts, int32_t *offsets, int32_t *perm_token,
                        int32_t *inv_pos, void *ws, size_t ws_bytes, void *stream);

/*
 * moe_permute without a workspace, for callers that cannot allocate device
 * memory: for example an engine that has already given almost all of the
 * GPU's memory to a fixed pool and makes no cudaMalloc calls while serving,
 * or a host program that loads this library as a plugin and offers it no
 * allocator. The pages have no counterpart of this call; it exists only for
 * such callers. Outputs, layout and results are those of moe_permute
 * (bit-identical). The per-chunk histograms live in a fixed array owned by
 * the library in device memory: 1 MiB (262144 int32) on every GPU that loads
 * the library, held until the process exits. Sizes needing more than that,
 * ceil(N / 256) * E > 262144 (e.g. N > 65536 at E = 1024), are rejected with
 * KMOE_ERR_UNSUPPORTED. The first call on a device looks up the array's
 * device address (once per device, with that device current); make that
 * first call before any stream capture. The address is then kept for the
 * life of the process: it assumes the device's primary context lives as
 * long, so do not call this entry point after a cudaDeviceReset (or another
 * teardown of the primary context) in the same process. All calls on a GPU share the array:
 * calls whose kernels may overlap on the GPU (different streams without
 * ordering) race and give wrong results, so order them on one stream. The
 * array keeps the last call's contents; each call overwrites every entry it
 * reads, so no clearing is needed. No allocation is made by this call.
 */
kmoe_status moe_permute_noalloc(const int32_t *topk_idx, int N, int K, int E,
                                int32_t *counts, int32_t *offsets, int32_t *perm_token,
                                int32_t *inv_pos, void *stream);

/*
 * Grouped expert FFN (routing section, last paragraph: each routed or
 * shared expert is a SwiGLU MLP):
 *   y_perm[p]   = F_e(x[perm_token[p]])  for offsets[e] <= p < offsets[e+1]
 *   y_shared[t] = F_shared(x[t])         (skipped when shared == NULL)
 * with F(x) = W_d (SiLU(W_g x) * (W_u x)), FP32 accumulation, and the
 * intermediate SiLU(.)*up rounded to the output dtype.
 * With KMOE_E4M3_B128 weights, BF16 x, d a multiple of 256 and N < 256 the
 * GEMMs run on the FP8 tensor cores: each 128-column group of a GEMM input
 * row (x, and H before the down projection) is held as two E4M3 terms with
 * one FP32 scale, v = s * (hi + lo / 16), within about 2^-8 of |v| (BF16's
 * own rounding is 2^-9), over the whole BF16 range.
 * x device [N, d] (x_dtype F32 or BF16). perm_token, offsets as produced by
 * moe_permute. Output dtype: FP32 when the weights are FP32, else BF16.
 * y_perm device [N*K, d]; y_shared device [N, d]. With KMOE_E4M3_B128_A8
 * weights the activations are FP8 (see kmoe_dtype): x must be BF16 and d a
 * multiple of 256 (KMOE_ERR_UNSUPPORTED otherwise). ws: at least
 * moe_workspace_size() bytes for these sizes and dtypes; its first 4 bytes
 * are the status word read by moe_device_status.
 */
kmoe_status moe_grouped_ffn(const void *x, int x_dtype, int N, int d, int I, int E, int K,
                            const int32_t *perm_token, const int32_t *offsets,
                            const kmoe_experts *routed, const kmoe_experts *shared,
                            void *y_perm, void *y_shared,
                            void *ws, size_t ws_bytes, void *stream);

/*
 * Weighted combine ("Kolibri 1 Deep Dive", section 1, the layer-output
 * formula without its residual term; the shared expert has weight 1):
 *   y[t] = y_shared[t] + sum_{k<K} topk_w[t][k] * y_perm[inv_pos[t][k]]
 * summed in slot order k = 0..K-1 in FP32 (deterministic, no atomics).
 * y_perm device [N*K, d], y_shared device [N, d] (both y_in_dtype: F32 or
 * BF16; y_shared may be NULL for no shared expert); topk_w device [N, K];
 * inv_pos device [N, K]; y device [N, d] of y_dtype (F32 or BF16).
 */
kmoe_status moe_combine(const void *y_perm, const void *y_shared, int y_in_dtype,
                        const float *topk_w, const int32_t *inv_pos,
                        int N, int K, int d, void *y, int y_dtype, void *stream);

/*
 * The whole layer: moe_router_topk -> moe_permute -> moe_grouped_ffn ->
 * moe_combine on one stream, with every intermediate in `ws`; `score`
 * (kmoe_score) picks the mixture weights.
 * y device [N, d] output of y_dtype (F32 or BF16). topk_idx_out [N, K],
 * topk_w_out [N, K] and counts_out [E] are optional device outputs (NULL to
 * skip). `shared` may be NULL (no shared expert). Routed and shared weights
 * have the same dtype; KMOE_E4M3_B128_A8 runs the expert GEMMs on FP8
 * activations (BF16 x, d a multiple of 256), with routing on x as given.
 */
kmoe_status moe_forward(const void *x, int x_dtype, int N, int d, int E, int K, int I, int score,
                        const float *w_router, const float *bias,
                        const kmoe_experts *routed, const kmoe_experts *shared,
                        void *y, int y_dtype,
                        int32_t *topk_idx_out, float *topk_w_out, int32_t *counts_out,
                        void *ws, size_t ws_bytes, void *stream);

/*
 * The sandwich block around the layer ("Inside Kolibri 1", section "The
 * released stack": RMSNorm before and after the MoE sublayer, residual added
 * after the second norm):
 *   x[t]     = bf16( h[t] / sqrt(mean_j h[t][j]^2 + eps) * gamma_pre )
 *   m        = the layer of moe_forward applied to x (FP32 combine)
 *   h_out[t] = bf16( h[t] + m[t] / sqrt(mean_j m[t][j]^2 + eps) * gamma_post )
 * Both sums of squares are FP32 in a fixed order (deterministic). The pages
 * give neither eps nor the dtype of the residual stream; this call takes eps
 * (0 <= eps <= 1) and keeps the residual stream in BF16.
 * h device [N, d] BF16; gamma_pre, gamma_post device [d] BF16; h_out device
 * [N, d] BF16, which may be the same buffer as h (each element of h is read
 * before its h_out element is written, by the same thread) but must not
 * overlap it otherwise. x_out: optional device [N, d] BF16 output of the
 * normalised layer input x (NULL keeps it in the workspace). Routed (and shared) weights must be BF16 or E4M3
 * with 128 x 128 scales (KMOE_E4M3_B128 or KMOE_E4M3_B128_A8) and d a multiple of 256
 * (KMOE_ERR_UNSUPPORTED otherwise), and
 * (K + 1) * d <= 25600 BF16 values must fit the combine's staging buffer
 * (K + 1 counts the shared expert). Other arguments and outputs as in
 * moe_forward. ws: at least moe_block_workspace_size() bytes; its first 4
 * bytes are the status word read by moe_device_status.
 */
size_t moe_block_workspace_size(int N, int d, int E, int K, int I, int w_dtype);
kmoe_status moe_block_forward(const void *h, int N, int d, int E, int K, int I, int score,
                              const void *gamma_pre, const void *gamma_post, float eps,
                              const float *w_router, const float *bias,
                              const kmoe_experts *routed, const kmoe_experts *shared,
                              void *h_out, void *x_out,
                              int32_t *topk_idx_out, float *topk_w_out, int32_t *counts_out,
                              void *ws, size_t ws_bytes, void *stream);

/*
 * Dynamic FP8 quantisation of activations ("Inside Kolibri 1", FP8 section:
 * activations are quantised dynamically in groups of 1 x 128). For each row
 * and each group of 128 consecutive columns:
 *   scales[r][g] = amax / 448 in FP32 (1 for an all-zero group)
 *   codes[r][c]  = E4M3(x[r][c] / scales[r][c / 128]), the quotient in FP32,
 *                  rounded to nearest even and saturated to +-448
 * x device [rows, cols] BF16; codes device [rows, cols] bytes (E4M3, sign
 * bit 7, exponent bias 7); scales device [rows, cols / 128] FP32. cols must
 * be a multiple of 128. rows == 0 is a no-op. Every x must be finite: a
 * group holding an Inf or a NaN gets an unspecified scale and codes.
 */
kmoe_status moe_quant_1x128(const void *x, int rows, int cols, uint8_t *codes, float *scales,
                            void *stream);

/*
 * Device status word. moe_forward, moe_block_forward and moe_grouped_ffn clear the first 4
 * bytes of `ws` when they are enqueued; a tensor-core kernel whose pipeline
 * wait gives up (after about two seconds, which only a fault elsewhere can
 * cause) writes a non-zero code there and returns early, leaving its outputs
 * invalid. This call copies the word to *status and synchronises `stream`
 * (the one exception to the no-synchronisation rule). Returns KMOE_OK when
 * the word is 0, KMOE_ERR_DEVICE otherwise (1 = a wait timed out).
 */
kmoe_status moe_device_status(const void *ws, int *status, void *stream);

/*
 * Give-up limit of the pipeline waits in the tensor-core expert FFN kernels
 * that later calls of the calling host thread launch (moe_grouped_ffn,
 * moe_forward, moe_block_forward), in SM clock cycles; 0 restores the
 * default of 2^32 cycles (about 2 s). This exists to test the failure path
 * without faulting a GPU: with a limit far below what a wait normally takes,
 * a kernel gives up, writes 1 to the workspace status word, lets its
 * in-flight copies and MMAs finish (those waits always use the default
 * limit), frees its tensor memory and returns; that call's outputs are then
 * invalid, moe_device_status reports KMOE_ERR_DEVICE with status 1, and the
 * next call with the default limit runs normally. cycles < 0 ->
 * KMOE_ERR_INVALID_ARG. The setting is per host thread.
 */
kmoe_status moe_set_wait_limit(long long cycles);

/* Message of the last error on the calling thread ("" after success). */
const char *moe_last_error(void);

/* ABI version of this header (bumped on incompatible change). */
int moe_abi_version(void);
#define KMOE_ABI_VERSION 3

#ifdef __cplusplus
}
#endif

#endif /* KMOE_H */
