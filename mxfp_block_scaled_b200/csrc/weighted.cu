// weighted.cu -- NVFP4 with a weighted-SSE block-scale search (sm_100a).
//
// Method (josch15366/Qwen3.8-Flash-Next-NVFP4-LocalHessian-Experts, "What is
// different about it": block scales chosen by a Hessian-weighted search
// instead of the plain amax / MSE sweep; no formula is given).  Readings:
// per-input-channel weights h >= 0 supplied by the caller (a diagonal
// Hessian estimate); per block, every E4M3 scale code from the amax/6
// plan's code to the four-over-six plan's code is a candidate; each
// candidate's codes follow from its scale as in the 4/6 plans; the
// objective sum h (x - q D s2)^2 is the binary64 sum in element order, the
// lowest value wins and ties go to the smaller code.  The kernel scores
// candidates in fp32 with a certified error bound and runs the binary64
// procedure only where the bound cannot separate the best two, so its
// choice is the binary64 argmin.
#include "nvfp4_block.cuh"

namespace mxq {

// ---------------------------------------------------------------------------
// Weighted-SSE block scale search (josch15366/Qwen3.8-Flash-Next-NVFP4-
// LocalHessian-Experts, "What is different about it": per-group weight
// scales chosen by a Hessian-weighted search instead of the plain amax / MSE
// sweep).  Readings: per-input-channel weights h >= 0 (a diagonal Hessian
// estimate); candidates are the E4M3 scale codes from the amax/6 plan's code
// to the four-over-six plan's code of the block; the objective
// sum h_i (x_i - q_i D s2)^2 is formed in binary64 in element order with
// explicit roundings (deq = (q D) s2 exact, e = x - deq, acc += h (e e));
// the lowest value wins, ties to the smaller code.  Second pass after
// group_amax_kernel; one thread per block.
// ---------------------------------------------------------------------------
__device__ __forceinline__ double block_wsse(const double (&xd)[16], const double (&hd)[16], uint2 c,
                                             float D, double ds2)
{
    uint32_t q[8];
    e2m1x8_to_f16x2(c.x, *reinterpret_cast<uint32_t(*)[4]>(&q[0]));
    e2m1x8_to_f16x2(c.y, *reinterpret_cast<uint32_t(*)[4]>(&q[4]));
    const float2 D2 = make_float2(D, D);
    double acc = 0.0;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
        // q * D is exact in fp32 (2 + 4 significant bits); (q D) s2 exact in fp64
        const float2 qd = __fmul2_rn(f16x2_to_float2(q[j]), D2);
        const double e0 = __dsub_rn(xd[2 * j], __dmul_rn((double)qd.x, ds2));
        acc = __dadd_rn(acc, __dmul_rn(hd[2 * j], __dmul_rn(e0, e0)));
        const double e1 = __dsub_rn(xd[2 * j + 1], __dmul_rn((double)qd.y, ds2));
        acc = __dadd_rn(acc, __dmul_rn(hd[2 * j + 1], __dmul_rn(e1, e1)));
    }
    return acc;
}

// The same objective in fp32 pairs, for the filter below:
// W32 = sum h RN32(x - q d)^2 with d = RN32(D s2), the candidate's divisor:
// each error term is one FMA (the product q d exact inside it, one
// rounding), then one rounding per product and sum.  Against the exact
// error x - q D s2 the divisor's rounding moves a term by at most
// 2^-24 |q D s2|, the same size as rounding the dequantized value before
// the subtraction, which the bound below covers.  q: the candidate's
// decoded values as f16x2 pairs.
__device__ __forceinline__ float block_wsse32(const float2 (&xf)[8], const float2 (&h2)[8], const uint32_t (&q)[8],
                                              float d)
{
    const float2 ND = make_float2(-d, -d);
    float2 acc = make_float2(0.0f, 0.0f);
#pragma unroll
    for (int j = 0; j < 8; ++j) {
        const float2 e = __ffma2_rn(f16x2_to_float2(q[j]), ND, xf[j]);      // RN32(x - q d)
        acc = __ffma2_rn(h2[j], __fmul2_rn(e, e), acc);
    }
    return __fadd_rn(acc.x, acc.y);
}

// Codes of one candidate scale (divisor d in [2^-60, 2^60], r = RN32(1/d))
// and their decoded values as f16x2 pairs, taken from the same bytes.
__device__ __forceinline__ uint2 candidate_codes(const float2 (&x)[8], float d, float r, uint32_t (&q)[8])
{
    const float2 d2 = make_float2(d, d), nr2 = make_float2(-r, -r);
    float2 y[8];
#pragma unroll
    for (int j = 0; j < 8; ++j)
        y[j] = div2_bf16(x[j], d2, nr2);
    uint2 c;
    c.x = e2m1x8_enc_dec(y[0], y[1], y[2], y[3], *reinterpret_cast<uint32_t(*)[4]>(&q[0]));
    c.y = e2m1x8_enc_dec(y[4], y[5], y[6], y[7], *reinterpret_cast<uint32_t(*)[4]>(&q[4]));
    return c;
}

// Error bound of W32 against the exact weighted error W, and against the
// binary64 value the definition forms.  With u = 2^-24 and A = sum h x^2:
// each error term is (e + eta)(1 + delta) with |eta| <= u |q D s2| <=
// u (|x| + |e|) (the divisor's rounding) and |delta| <= u, so by
// Cauchy-Schwarz on sum h |x| |e| the terms cost at most
// 2.1u sqrt(A W32) + 4.2u W32 + 4.2u^2 A, and the products and the
// eight-step pair sums at most 10.5u W32: |W32 - W| <= 2.1u sqrt(A W32) +
// 14.7u W32 + 4.2u^2 A.  The constants below take about twice that, which
// also covers the binary64 procedure's own error (below 2^-48 W) and the
// error of forming the bound in fp32.
// The last term covers terms that underflow, with every weight <= 2^40 and
// s2 in [2^-50, 2^50] (every non-zero dequantized value normal).
__device__ __forceinline__ float wsse_bound(float W, float sqrtA_scaled, float c_block)
{
    float r;
    asm("sqrt.approx.f32 %0, %1;" : "=f"(r) : "f"(W));
    return __fmaf_rn(sqrtA_scaled, r, __fmaf_rn(0x1p-19f, W, c_block));
}

// The binary64 search of the definition, for blocks the fp32 filter leaves
// undecided (kept out of line: its doubles stay off the common path).
__device__ __noinline__ void weighted_search_exact(const uint32_t (&w)[8], const float (&hh)[16], uint32_t lo,
                                                   uint32_t hi, const GroupConst gc, uint32_t &best_sc,
                                                   uint2 &best_c)
{
    float2 xf[8];
    unpack_x(w, xf);
    double xd[16], hd[16];                              // converted once, used by every candidate
#pragma unroll
    for (int k = 0; k < 8; ++k) {
        xd[2 * k] = (double)xf[k].x;
        xd[2 * k + 1] = (double)xf[k].y;
    }
#pragma unroll
    for (int k = 0; k < 16; ++k)
        hd[k] = (double)hh[k];
    double best_w = 0.0;
    for (uint32_t sc = lo; sc <= hi; ++sc) {
        const float D = f16x2_to_float2(e4m3x2_to_f16x2(sc)).x;
        const Plan p = make_plan_any(xf, __fmul_rn(D, gc.s2));
        const double wv = block_wsse(xd, hd, p.codes, D, (double)gc.s2);
        if (sc == lo || wv < best_w) {
            best_w = wv;
            best_sc = sc;
            best_c = p.codes;
        }
    }
}

// Four CTAs per SM (64 registers, some values spilled to an L1 that shared
// memory does not crowd): the occupancy pays more than the spills cost
// (7.76 against 8.16 ms per full-size layer at three CTAs and 80 registers,
// 9.41 ms at two CTAs and 128 registers).
__global__ void __launch_bounds__(kNvThreads, 4)
nvfp4_weighted_kernel(const uint4 *__restrict__ x, int64_t n_groups, int64_t nb,
                      const uint32_t *__restrict__ amax_bits, const float *__restrict__ h,
                      int64_t h_stride, uint32_t cb, uint2 *__restrict__ codes,
                      uint8_t *__restrict__ scales, const ScaleLayout sl, float *__restrict__ s2_out,
                      uint32_t *__restrict__ status)
{
    __shared__ GroupConst s_gc;
    for (int64_t g = blockIdx.y; g < n_groups; g += gridDim.y) {
        if (threadIdx.x == 0) {
            s_gc = make_group_const(amax_bits[g]);
            if (blockIdx.x == 0)
                s2_out[g] = s_gc.s2;
        }
        __syncthreads();
        const GroupConst gc = s_gc;
        const float *hg = h + g * h_stride;
        for (int64_t b = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; b < nb;
             b += (int64_t)gridDim.x * blockDim.x) {
            const uint4 v0 = __ldg(x + (g * nb + b) * 2), v1 = __ldg(x + (g * nb + b) * 2 + 1);
            const uint32_t w[8] = {v0.x, v0.y, v0.z, v0.w, v1.x, v1.y, v1.z, v1.w};
            uint32_t m = 0;
#pragma unroll
            for (int j = 0; j < 8; ++j)
                m = absmax_bf16x2(m, w[j]);
            const float amax_b = __uint_as_float(fold_halves(m) << 16);
            const float4 *hp = reinterpret_cast<const float4 *>(hg + (b % cb) * 16);
            float hh[16];
            bool bad_h = false;
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                const float4 t = __ldg(hp + k);
                hh[4 * k] = t.x; hh[4 * k + 1] = t.y; hh[4 * k + 2] = t.z; hh[4 * k + 3] = t.w;
            }
#pragma unroll
            for (int k = 0; k < 16; ++k)
                bad_h = bad_h || !(hh[k] >= 0.0f && hh[k] <= 3.402823466e38f);
            if (bad_h)
                atomicOr(status, MXQ_DEV_NONFINITE_INPUT);
            float2 xf[8], h2[8];
            unpack_x(w, xf);
            float2 a2 = make_float2(0.0f, 0.0f);
            float hmax = 0.0f;
#pragma unroll
            for (int k = 0; k < 8; ++k) {
                h2[k] = make_float2(hh[2 * k], hh[2 * k + 1]);
                a2 = __ffma2_rn(h2[k], __fmul2_rn(xf[k], xf[k]), a2);
                hmax = fmaxf(hmax, fmaxf(h2[k].x, h2[k].y));
            }
            const float A = __fadd_rn(a2.x, a2.y);
            uint32_t lo = 0, hi = 0;
            if (gc.s2 > 0.0f) {
                float t6, t4;
                if (gc.tfast) {
                    t6 = div_bf16(amax_b, gc.den.x, -gc.nr.x);
                    t4 = div_bf16(amax_b, gc.den.y, -gc.nr.y);
                } else {
                    t6 = __fdiv_rn(amax_b, gc.den.x);
                    t4 = __fdiv_rn(amax_b, gc.den.y);
                }
                const uint32_t sb = e4m3x2(t6, t4);
                lo = sb & 0xFFu;
                hi = sb >> 8;
            }
            // fp32 filter: the fp32 argmin is the binary64 argmin when it beats
            // every other candidate by more than both error bounds
            uint32_t best_sc = lo;
            uint2 best_c = make_uint2(0u, 0u);
            bool decided = gc.qfast && !bad_h && hmax <= 0x1p40f && A >= 0x1p-60f && A <= 0x1p100f;
            if (decided) {
                float sa;
                asm("sqrt.approx.f32 %0, %1;" : "=f"(sa) : "f"(A));
                const float sqrtA_scaled = 0x1p-22f * sa;
                const float c_block = __fmaf_rn(0x1p-45f, A, 0x1p-100f);
                float bw = 0.0f, be = 0.0f, lb = __int_as_float(0x7F800000);   // lb: min (W - eps) of the others
                auto consider = [&](uint32_t sc, float wv, uint2 c) {
                    const float ev = wsse_bound(wv, sqrtA_scaled, c_block);
                    if (sc == lo || wv < bw) {
                        if (sc != lo)
                            lb = fminf(lb, __fsub_rn(bw, be));
                        bw = wv;
                        be = ev;
                        best_sc = sc;
                        best_c = c;
                    } else {
                        lb = fminf(lb, __fsub_rn(wv, ev));
                    }
                };
                uint32_t sc = lo;
                if (sc == 0) {                          // scale 0: every code 0, W = A
                    consider(0, A, make_uint2(0u, 0u));
                    ++sc;
                }
                // one candidate per step (the warp runs as many steps as its widest block); with
                // s2 in [2^-50, 2^50] and D >= 2^-9 every divisor lies in [2^-59, 2^59]
                for (; sc <= hi; ++sc) {
                    const float D = f16x2_to_float2(e4m3x2_to_f16x2(sc)).x;
                    const float d = __fmul_rn(D, gc.s2);
                    uint32_t q[8];
                    const uint2 c = candidate_codes(xf, d, rcp_rn_mid(d), q);
                    consider(sc, block_wsse32(xf, h2, q, d), c);
                }
                decided = lb > __fadd_rn(bw, be);
            }
            if (!decided)
                weighted_search_exact(w, hh, lo, hi, gc, best_sc, best_c);
            codes[g * nb + b] = best_c;
            scales[sl.swz ? tiled_scale_offset(sl, (uint64_t)g, (uint32_t)b) : (uint64_t)(g * nb + b)] =
                (uint8_t)best_sc;
        }
        __syncthreads();
    }
}

cudaError_t launch_nvfp4_weighted(const uint16_t *x, int64_t n_groups, int64_t nb, int64_t cols,
                                  const uint32_t *amax_bits, const float *h, int64_t h_stride,
                                  uint8_t *codes, uint8_t *scales, const ScaleLayout &sl, float *s2,
                                  uint32_t *status, cudaStream_t s)
{
    if (n_groups == 0)
        return cudaSuccess;
    const int64_t tiles = nb > 0 ? (nb + kNvThreads - 1) / kNvThreads : 1;
    dim3 grid((unsigned)(tiles < 4096 ? tiles : 4096), (unsigned)(n_groups < 65535 ? n_groups : 65535));
    nvfp4_weighted_kernel<<<grid, kNvThreads, 0, s>>>(reinterpret_cast<const uint4 *>(x), n_groups, nb,
                                                      amax_bits, h, h_stride, (uint32_t)(cols / 16),
                                                      reinterpret_cast<uint2 *>(codes), scales, sl, s2,
                                                      status);
    return cudaGetLastError();
}

} // namespace mxq
