// mx.cu -- MXFP8 / MXFP4 quantization, one UE8M0 scale per 32 values
// (sm_100a).
//
// Method (azampatti/Qwen3.8-Flash-Next-FP4-Local-AZ, "The shared expert":
// e4m3 values, one power-of-two scale per 32 weights,
// e = ceil(log2(amax / 448)); MJPansa/Qwen3.8-Flash-Next-MXFP4-FP8-R12,
// "Quantization format": E2M1 weights with UE8M0 microscales, qmax 6):
//   e = smallest integer with amax <= qmax * 2^e, clamped to [-127, 127];
//   scale byte = e + 127; code_i = FMT(x_i * 2^-e), round to nearest even.
//
// The exponent is read off the bf16 bits of amax, exactly: with
// amax = m * 2^E (1 <= m < 2) and qmax = c * 2^k (448 = 1.75 * 2^8,
// 6 = 1.5 * 2^2), amax <= qmax * 2^e  <=>  e >= E - k + (m > c).  A
// subnormal or zero amax always lands on the lower clamp.
#include "mxq_device.cuh"
#include "mxq_internal.h"
#include "mxq.h"

namespace mxq {

template <int FMT>
__device__ __forceinline__ int mx_exponent(uint32_t amax_bits)
{
    constexpr int k = (FMT == MXQ_FMT_MXFP8) ? 8 : 2;
    constexpr uint32_t c_mant = (FMT == MXQ_FMT_MXFP8) ? 0x60u : 0x40u;  // .75 / .5 in 7 bits
    const uint32_t E = amax_bits >> 7;
    if (E == 0)
        return -127;
    int e = (int)E - 127 - k + ((amax_bits & 0x7Fu) > c_mant ? 1 : 0);
    return e < -127 ? -127 : (e > 127 ? 127 : e);
}

// One thread per block of 32: 64 bytes in, 32 (MXFP8) or 16 (MXFP4) out.
template <int FMT>
__global__ void __launch_bounds__(256)
mx_quant_kernel(const uint4 *__restrict__ x, int64_t nblk, uint8_t *__restrict__ codes,
                uint8_t *__restrict__ scales, const ScaleLayout sl, uint32_t *__restrict__ status)
{
    for (int64_t b = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; b < nblk;
         b += (int64_t)gridDim.x * blockDim.x) {
        uint4 v[4];
#pragma unroll
        for (int k = 0; k < 4; ++k)
            v[k] = __ldg(x + b * 4 + k);
        const uint32_t w[16] = {v[0].x, v[0].y, v[0].z, v[0].w, v[1].x, v[1].y, v[1].z, v[1].w,
                                v[2].x, v[2].y, v[2].z, v[2].w, v[3].x, v[3].y, v[3].z, v[3].w};
        uint32_t m = 0;
#pragma unroll
        for (int j = 0; j < 16; ++j)
            m = absmax_bf16x2(m, w[j]);
        const uint32_t a = fold_halves(m);
        if (a >= 0x7F80u && status)
            atomicOr(status, MXQ_DEV_NONFINITE_INPUT);
        const int e = mx_exponent<FMT>(a);
        const float sc = __uint_as_float((uint32_t)(127 - e) << 23);   // 2^-e, normal
        const float2 sc2 = make_float2(sc, sc);
        float2 y[16];
#pragma unroll
        for (int j = 0; j < 16; ++j)
            y[j] = __fmul2_rn(make_float2(bf16_lo(w[j]), bf16_hi(w[j])), sc2);
        scales[sl.swz ? tiled_scale_offset(sl, 0, (uint32_t)b) : (uint64_t)b] = (uint8_t)(e + 127);
        if (FMT == MXQ_FMT_MXFP8) {
            uint32_t o[8];
#pragma unroll
            for (int j = 0; j < 8; ++j)
                o[j] = e4m3x2(y[2 * j].x, y[2 * j].y) | (e4m3x2(y[2 * j + 1].x, y[2 * j + 1].y) << 16);
            uint4 *dst = reinterpret_cast<uint4 *>(codes) + b * 2;
            dst[0] = make_uint4(o[0], o[1], o[2], o[3]);
            dst[1] = make_uint4(o[4], o[5], o[6], o[7]);
        } else {
            uint4 o;
            o.x = e2m1x8(y[0], y[1], y[2], y[3]);
            o.y = e2m1x8(y[4], y[5], y[6], y[7]);
            o.z = e2m1x8(y[8], y[9], y[10], y[11]);
            o.w = e2m1x8(y[12], y[13], y[14], y[15]);
            reinterpret_cast<uint4 *>(codes)[b] = o;
        }
    }
}

// ---------------------------------------------------------------------------
// FP8 -> MX requantization of a block-FP8 source
// (MJPansa/Qwen3.8-Flash-Next-MXFP4-FP8-R12, "Quantization and layer
// selection": the conversion starts from the released FP8 weights;
// "Quantization format": retained layers stay in the source block-FP8
// format).  Each value is dequantized once to fp32, w = RN32(E4M3 * scale)
// with the fp32 scale of its brows x bcols source block, and each run of 32
// w is MX-quantized as above, the exponent read off the fp32 amax bits:
// amax = m * 2^E, qmax = c * 2^k  =>  e = E - k + (m > c), clamped.
// ---------------------------------------------------------------------------
template <int FMT>
__device__ __forceinline__ int mx_exponent_f32(uint32_t amax_bits)
{
    constexpr int k = (FMT == MXQ_FMT_MXFP8) ? 8 : 2;
    constexpr uint32_t c_mant = (FMT == MXQ_FMT_MXFP8) ? 0x600000u : 0x400000u;  // .75 / .5
    const uint32_t E = amax_bits >> 23;
    if (E == 0)
        return -127;
    int e = (int)E - 127 - k + ((amax_bits & 0x7FFFFFu) > c_mant ? 1 : 0);
    return e < -127 ? -127 : (e > 127 ? 127 : e);
}

struct RequantArgs {
    const uint4 *fp8;        // 32 E4M3 bytes per MX block (2 x uint4)
    const float *bscale;     // [ceil(rows / brows), nbc]
    int64_t nblk;            // MX blocks (rows * cols / 32), < 2^32
    uint32_t cb, nbc;        // MX blocks per row; source blocks per row
    FastDiv cbdiv, browsdiv, bcdiv;   // / cb, / brows, / (bcols / 32)
    uint8_t *codes, *scales;
    ScaleLayout sl;
    uint32_t *status;
};

// Running max of |v| over f16x2 words, per half (max.NaN.xorsign.abs; the
// sign bits are dropped by the fold below, NaN propagates).
__device__ __forceinline__ uint32_t absmax_f16x2(uint32_t acc, uint32_t v)
{
    uint32_t r;
    asm("max.NaN.xorsign.abs.f16x2 %0, %1, %2;" : "=r"(r) : "r"(acc), "r"(v));
    return r;
}

// Per MX block of 32: w_i = RN32(q_i * sc) (q_i the E4M3 source value, sc
// its block scale) is MX-quantized.  Two exact shortcuts:
//  - max |w_i| = RN32(max |q_i| * |sc|), RN being monotone, so the block
//    amax comes from the decoded source (one f16x2 max per pair);
//  - with |sc| in [2^-117, 2^100] every non-zero product q_i sc is a normal
//    fp32, and with |e| < 127 the scale sc 2^-e is normal, so
//    RN32(RN32(q_i sc) 2^-e) = RN32(q_i (sc 2^-e)): one multiply per value.
//    Outside that range the two roundings are kept.
template <int FMT>
__global__ void __launch_bounds__(256) requant_fp8_mx_kernel(const RequantArgs a)
{
    for (int64_t bb = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; bb < a.nblk;
         bb += (int64_t)gridDim.x * blockDim.x) {
        const uint32_t b = (uint32_t)bb;
        const uint4 v0 = __ldg(a.fp8 + 2 * bb), v1 = __ldg(a.fp8 + 2 * bb + 1);
        const uint32_t r = fastdiv(b, a.cbdiv), j = b - r * a.cb;
        const float sc = __ldg(a.bscale + (uint64_t)fastdiv(r, a.browsdiv) * a.nbc + fastdiv(j, a.bcdiv));
        const uint32_t w8[8] = {v0.x, v0.y, v0.z, v0.w, v1.x, v1.y, v1.z, v1.w};
        uint32_t qh[16];                                // the E4M3 values as f16x2 pairs (exact)
        uint32_t m16 = 0;
#pragma unroll
        for (int t = 0; t < 8; ++t) {
            qh[2 * t] = e4m3x2_to_f16x2(w8[t]);
            qh[2 * t + 1] = e4m3x2_to_f16x2(w8[t] >> 16);
            m16 = absmax_f16x2(absmax_f16x2(m16, qh[2 * t]), qh[2 * t + 1]);
        }
        const uint32_t mq = max(m16 & 0x7FFFu, (m16 >> 16) & 0x7FFFu);
        const float asc = fabsf(sc);
        const uint32_t m = __float_as_uint(__fmul_rn(__half2float(__ushort_as_half((unsigned short)mq)), asc));
        if (m >= 0x7F800000u && a.status)               // Inf / NaN source value or scale
            atomicOr(a.status, MXQ_DEV_NONFINITE_INPUT);
        const int e = mx_exponent_f32<FMT>(m);
        float2 w[16];
        if (asc >= 0x1p-117f && asc <= 0x1p100f && e > -127 && e < 127) {
            const float sce = __fmul_rn(sc, __uint_as_float((uint32_t)(127 - e) << 23));   // exact
            const float2 s2 = make_float2(sce, sce);
#pragma unroll
            for (int t = 0; t < 16; ++t)
                w[t] = __fmul2_rn(f16x2_to_float2(qh[t]), s2);
        } else {
            const float2 sc2 = make_float2(sc, sc);
            const float s = e == 127 ? 0x1p-127f : __uint_as_float((uint32_t)(127 - e) << 23);   // 2^-e
            const float2 s2 = make_float2(s, s);
#pragma unroll
            for (int t = 0; t < 16; ++t)
                w[t] = __fmul2_rn(__fmul2_rn(f16x2_to_float2(qh[t]), sc2), s2);
        }
        a.scales[a.sl.swz ? tiled_scale_offset(a.sl, 0, b) : (uint64_t)b] = (uint8_t)(e + 127);
        if (FMT == MXQ_FMT_MXFP8) {
            uint32_t o[8];
#pragma unroll
            for (int t = 0; t < 8; ++t)
                o[t] = e4m3x2(w[2 * t].x, w[2 * t].y) | (e4m3x2(w[2 * t + 1].x, w[2 * t + 1].y) << 16);
            uint4 *dst = reinterpret_cast<uint4 *>(a.codes) + 2 * bb;
            dst[0] = make_uint4(o[0], o[1], o[2], o[3]);
            dst[1] = make_uint4(o[4], o[5], o[6], o[7]);
        } else {
            uint4 o;
            o.x = e2m1x8(w[0], w[1], w[2], w[3]);
            o.y = e2m1x8(w[4], w[5], w[6], w[7]);
            o.z = e2m1x8(w[8], w[9], w[10], w[11]);
            o.w = e2m1x8(w[12], w[13], w[14], w[15]);
            reinterpret_cast<uint4 *>(a.codes)[bb] = o;
        }
    }
}

cudaError_t launch_requant_fp8_mx(const uint8_t *fp8, const float *bscale, int64_t rows, int64_t cols,
                                  int64_t brows, int64_t bcols, int fmt, uint8_t *codes,
                                  uint8_t *scales, const ScaleLayout &sl, uint32_t *status,
                                  cudaStream_t s)
{
    RequantArgs a;
    a.fp8 = reinterpret_cast<const uint4 *>(fp8);
    a.bscale = bscale;
    a.nblk = rows * cols / 32;
    a.cb = (uint32_t)(cols / 32);
    a.nbc = (uint32_t)((cols + bcols - 1) / bcols);
    a.cbdiv = make_fastdiv(a.cb);
    a.browsdiv = make_fastdiv((uint32_t)brows);
    a.bcdiv = make_fastdiv((uint32_t)(bcols / 32));
    a.codes = codes;
    a.scales = scales;
    a.sl = sl;
    a.status = status;
    if (a.nblk == 0)
        return cudaSuccess;
    int64_t ctas = (a.nblk + 255) / 256;
    if (ctas > 148 * 64)
        ctas = 148 * 64;
    if (fmt == MXQ_FMT_MXFP8)
        requant_fp8_mx_kernel<MXQ_FMT_MXFP8><<<(unsigned)ctas, 256, 0, s>>>(a);
    else
        requant_fp8_mx_kernel<MXQ_FMT_MXFP4><<<(unsigned)ctas, 256, 0, s>>>(a);
    return cudaGetLastError();
}

cudaError_t launch_mx_quant(const uint16_t *x, int64_t nblk32, int fmt, uint8_t *codes,
                            uint8_t *scales, const ScaleLayout &sl, uint32_t *status, cudaStream_t s)
{
    if (nblk32 == 0)
        return cudaSuccess;
    int64_t ctas = (nblk32 + 255) / 256;
    if (ctas > 0x7FFFFFFF)
        ctas = 0x7FFFFFFF;
    const uint4 *xv = reinterpret_cast<const uint4 *>(x);
    if (fmt == MXQ_FMT_MXFP8)
        mx_quant_kernel<MXQ_FMT_MXFP8><<<(unsigned)ctas, 256, 0, s>>>(xv, nblk32, codes, scales, sl, status);
    else
        mx_quant_kernel<MXQ_FMT_MXFP4><<<(unsigned)ctas, 256, 0, s>>>(xv, nblk32, codes, scales, sl, status);
    return cudaGetLastError();
}

} // namespace mxq
