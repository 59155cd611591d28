// Dynamic FP8 quantisation of activations in groups of 1 x 128.
//
// "Inside Kolibri 1" (flozi.net), section "The FP8 path is explicitly mixed
// precision": activations are quantised dynamically in groups of 1 x 128
// (weights are E4M3 in 128 x 128 blocks with FP32 scales). For each row and
// each group of 128 consecutive columns:
//     s = amax / 448 (FP32; 1 for an all-zero group)
//     q = E4M3(x / s), the quotient in FP32, rounded to nearest even and
//         saturated to +-448
// One warp per group: each lane holds four BF16 values (8 bytes), the group
// maximum comes from a warp reduction, and the codes are written four per
// lane (one 4-byte store).
#include "common.cuh"

namespace kmoe {

constexpr int kQuantGroup = 128;
constexpr int kQuantThreads = 256;                    // 8 groups per CTA

__global__ void __launch_bounds__(kQuantThreads)
quant_1x128_kernel(const __nv_bfloat16 *__restrict__ x, int rows, int cols, uint8_t *__restrict__ codes,
                   float *__restrict__ scales)
{
    pdl_wait();
    pdl_trigger();
    const int lane = threadIdx.x & 31;
    const int groups = cols / kQuantGroup;
    const long long grp = (long long)blockIdx.x * (kQuantThreads / 32) + (threadIdx.x >> 5);
    if (grp >= (long long)rows * groups) return;
    const long long base = grp * kQuantGroup + lane * 4;   // row-major: group g of row r starts at (r*groups+g)*128
    const uint2 raw = *reinterpret_cast<const uint2 *>(x + base);
    float v[4] = {__uint_as_float(raw.x << 16), __uint_as_float(raw.x & 0xffff0000u),
                  __uint_as_float(raw.y << 16), __uint_as_float(raw.y & 0xffff0000u)};
    float amax = fmaxf(fmaxf(fabsf(v[0]), fabsf(v[1])), fmaxf(fabsf(v[2]), fabsf(v[3])));
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
    const float s = amax > 0.f ? __fdiv_rn(amax, 448.f) : 1.f;
    uint32_t packed = 0;
#pragma unroll
    for (int q = 0; q < 4; ++q) {
        const __nv_fp8_storage_t c = __nv_cvt_float_to_fp8(__fdiv_rn(v[q], s), __NV_SATFINITE, __NV_E4M3);
        packed |= (uint32_t)c << (8 * q);
    }
    *reinterpret_cast<uint32_t *>(codes + base) = packed;
    if (lane == 0) scales[grp] = s;
}

// Two-term variant: the same group scale s, and two E4M3 codes per value,
//     hi = E4M3(x / s),   lo = E4M3((x / s - hi) * 16)
// (each quotient and difference in FP32), so that x = s * (hi + lo / 16) up
// to the rounding of lo: about 2^-8 of |x|, the size of a BF16 rounding. The
// tensor cores then take BF16-precision activations as E4M3 operands (the
// two terms as separate rows of one MMA operand).
__global__ void __launch_bounds__(kQuantThreads)
quant_1x128_split_kernel(const __nv_bfloat16 *__restrict__ x, int rows, int cols, uint8_t *__restrict__ hi,
                         uint8_t *__restrict__ lo, float *__restrict__ scales)
{
    pdl_wait();
    pdl_trigger();
    const int lane = threadIdx.x & 31;
    const int groups = cols / kQuantGroup;
    const long long grp = (long long)blockIdx.x * (kQuantThreads / 32) + (threadIdx.x >> 5);
    if (grp >= (long long)rows * groups) return;
    const long long base = grp * kQuantGroup + lane * 4;
    const uint2 raw = *reinterpret_cast<const uint2 *>(x + base);
    float v[4] = {__uint_as_float(raw.x << 16), __uint_as_float(raw.x & 0xffff0000u),
                  __uint_as_float(raw.y << 16), __uint_as_float(raw.y & 0xffff0000u)};
    float amax = fmaxf(fmaxf(fabsf(v[0]), fabsf(v[1])), fmaxf(fabsf(v[2]), fabsf(v[3])));
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
    const float s = amax > 0.f ? __fdiv_rn(amax, 448.f) : 1.f;
    uint32_t ph = 0, pl = 0;
#pragma unroll
    for (int q = 0; q < 4; ++q) {
        const float y = __fdiv_rn(v[q], s);
        const __nv_fp8_storage_t h = __nv_cvt_float_to_fp8(y, __NV_SATFINITE, __NV_E4M3);
        const float hv = __half2float(__half(__nv_cvt_fp8_to_halfraw(h, __NV_E4M3)));
        const __nv_fp8_storage_t l = __nv_cvt_float_to_fp8((y - hv) * 16.f, __NV_SATFINITE, __NV_E4M3);
        ph |= (uint32_t)h << (8 * q);
        pl |= (uint32_t)l << (8 * q);
    }
    *reinterpret_cast<uint32_t *>(hi + base) = ph;
    *reinterpret_cast<uint32_t *>(lo + base) = pl;
    if (lane == 0) scales[grp] = s;
}

kmoe_status launch_quant_1x128_split(const __nv_bfloat16 *x, int rows, int cols, uint8_t *hi, uint8_t *lo,
                                     float *scales, cudaStream_t st)
{
    const long long groups = (long long)rows * (cols / kQuantGroup);
    const long long grid = (groups + kQuantThreads / 32 - 1) / (kQuantThreads / 32);
    if (grid > 0x7fffffffLL) return fail(KMOE_ERR_UNSUPPORTED, "quant_1x128_split: %lld groups", groups);
    launch_pdl(quant_1x128_split_kernel, (unsigned)grid, kQuantThreads, 0, st, x, rows, cols, hi, lo, scales);
    return check_launch("quant_1x128_split");
}

kmoe_status launch_quant_1x128(const __nv_bfloat16 *x, int rows, int cols, uint8_t *codes, float *scales,
                               cudaStream_t st)
{
    const long long groups = (long long)rows * (cols / kQuantGroup);
    const long long grid = (groups + kQuantThreads / 32 - 1) / (kQuantThreads / 32);
    if (grid > 0x7fffffffLL) return fail(KMOE_ERR_UNSUPPORTED, "quant_1x128: %lld groups", groups);
    launch_pdl(quant_1x128_kernel, (unsigned)grid, kQuantThreads, 0, st, x, rows, cols, codes, scales);
    return check_launch("quant_1x128");
}

}  // namespace kmoe
