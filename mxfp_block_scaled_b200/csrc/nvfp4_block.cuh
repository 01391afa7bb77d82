// nvfp4_block.cuh -- the NVFP4 block quantizer with 4/6-optimal block scales
// (sm_100a), shared by the schedules in nvfp4.cu and the weighted search in
// weighted.cu.
//
// Method (dabsLabs/Qwen3.8-Flash-Next-NVFP4, "What makes this build
// different"; josch15366/Qwen3.8-Flash-Next-NVFP4-LocalHessian-Experts,
// introduction):
//   s2 = RN32(amax_g / 2688) per group (one expert's fused gate_up slab, so
//   gate and up share weight_scale_2; or one down slab; or one token tile);
//   per block of 16 and plan M in {6, 4}:
//     t_M = RN32(amax_b / RN32(M * s2)),  S_M = E4M3(t_M),  D_M = value(S_M)
//     d_M = RN32(D_M * s2),  code_i = E2M1(RN32(x_i / d_M))
//   and the M=4 plan is kept only when its exact squared error
//   sum (x_i - q_i D_M s2)^2 is strictly lower than the M=6 plan's.
//
// Exact decision.  sum x_i^2 is common to both plans, so
//   SSE_M - sum x^2 = s2 * D_M * (D_M s2 B_M - 2 A_M),
//   A_M = sum x_i q_i,  B_M = sum q_i^2,
// and since s2 > 0 the comparison SSE_4 < SSE_6 is G_4 < G_6 with
// G_M = D_M * (D_M s2 B_M - 2 A_M).  Every term is exact in the precision
// it is formed in: x_i q_i has at most 8 + 2 significant bits and every
// non-zero term lies within 2^21 of the smallest one (a non-zero code needs
// |x| > d/4 and |x| <= 9 d), so A_M is exact in fp32 in any order; B_M is a
// sum of quarter-integers <= 576, exact in f16 half-sums of 8 and in fp32;
// D_M s2 (4 + 24 bits), D_M s2 B_M - 2 A_M (< 2^40 span) and D_M * P (4 + 40
// bits) are exact in fp64.  So the decision has no rounding at all.
//
#pragma once

#include "mxq_device.cuh"
#include "mxq_internal.h"
#include "mxq.h"

namespace mxq {

// ---------------------------------------------------------------------------
// The block quantizer.
// ---------------------------------------------------------------------------
struct GroupConst {
    float s2;        // global scale
    float2 den;      // (RN32(6 s2), 4 s2): the divisors of the two plans' block scales
    float2 nr;       // (-RN32(1 / den.x), -RN32(1 / den.y)) when `tfast`
    double s2h;      // s2 / 2 (exact), for the exact decision
    float s2hf;      // s2 / 2 in fp32 (exact when `qfast`), for the filtered decision
    int tfast;       // den in the range where the reciprocal quotient is exact
    int qfast;       // s2 in [2^-50, 2^50]: every non-zero block scale gives a
                     // divisor d = RN32(D s2) in [2^-59, 2^59], where the
                     // reciprocal quotient of the block values is exact
};

// Constants of a group from its global scale s2 (finite, >= 0).
__device__ __forceinline__ GroupConst make_group_const_from_s2(float s2)
{
    GroupConst c;
    c.s2 = s2;
    c.den = make_float2(__fmul_rn(6.0f, c.s2), __fmul_rn(4.0f, c.s2));
    c.tfast = (c.s2 >= 0x1p-100f && c.s2 <= 0x1p100f) ? 1 : 0;
    c.qfast = (c.s2 >= 0x1p-50f && c.s2 <= 0x1p50f) ? 1 : 0;
    c.nr = c.tfast ? make_float2(-__frcp_rn(c.den.x), -__frcp_rn(c.den.y)) : make_float2(0.0f, 0.0f);
    c.s2h = 0.5 * (double)c.s2;
    c.s2hf = 0.5f * c.s2;
    return c;
}

// Constants of a group from its amax (bf16 magnitude bits): s2 = RN32(amax / 2688).
__device__ __forceinline__ GroupConst make_group_const(uint32_t amax_bits)
{
    const float amax = __uint_as_float(amax_bits << 16);
    return make_group_const_from_s2(__fdiv_rn(amax, kGlobalDivisor));
}

struct Plan {
    uint2 codes;   // 16 E2M1 nibbles
    float a;       // sum x_i q_i (exact)
    float b;       // sum q_i^2 (exact)
};

// One plan's codes and the exact sums A and B from the quotients y.  The
// decoded pair q comes from the same byte register the code was written to.
// B is accumulated in f16 (<= 8 quarter-integers <= 36 per half: exact), A
// in fp32 pairs (exact).
__device__ __forceinline__ Plan plan_from_quotients(const float2 (&x)[8], const float2 (&y)[8])
{
    Plan p;
    uint32_t q[8];
    p.codes.x = e2m1x8_enc_dec(y[0], y[1], y[2], y[3], *reinterpret_cast<uint32_t(*)[4]>(&q[0]));
    p.codes.y = e2m1x8_enc_dec(y[4], y[5], y[6], y[7], *reinterpret_cast<uint32_t(*)[4]>(&q[4]));
    // Two independent partial sums each (pairs 0-3 and 4-7): the sums are
    // exact in any order, so splitting them only shortens the dependency
    // chains.
    float2 acc0 = make_float2(0.0f, 0.0f), acc1 = make_float2(0.0f, 0.0f);
    uint32_t bh0 = 0u, bh1 = 0u;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        bh0 = hfma2_bits(q[j], q[j], bh0);
        bh1 = hfma2_bits(q[j + 4], q[j + 4], bh1);
        acc0 = __ffma2_rn(x[j], f16x2_to_float2(q[j]), acc0);
        acc1 = __ffma2_rn(x[j + 4], f16x2_to_float2(q[j + 4]), acc1);
    }
    const float2 acc = __fadd2_rn(acc0, acc1);
    p.a = __fadd_rn(acc.x, acc.y);
    const uint32_t bh = hadd2_bits(bh0, bh1);         // <= 288 per half: exact in f16
    const float2 bf = f16x2_to_float2(bh);
    p.b = __fadd_rn(bf.x, bf.y);
    return p;
}

// y = RN32(x / d) from r = RN32(1 / d) with the reciprocal + FMA quotient,
// exact for d in [2^-60, 2^60] (see div_bf16).
__device__ __forceinline__ Plan make_plan_fast(const float2 (&x)[8], float d, float r)
{
    const float2 d2 = make_float2(d, d), nr2 = make_float2(-r, -r);
    float2 y[8];
#pragma unroll
    for (int j = 0; j < 8; ++j)
        y[j] = div2_bf16(x[j], d2, nr2);
    return plan_from_quotients(x, y);
}

__device__ __forceinline__ bool fast_scale(float d) { return d >= 0x1p-60f && d <= 0x1p60f; }

// Any d: all codes 0 when d is 0 (D == 0, or D * s2 underflowed), IEEE
// division outside the fast range.
__device__ __forceinline__ Plan make_plan_any(const float2 (&x)[8], float d)
{
    if (!(d > 0.0f)) {
        Plan p;
        p.codes = make_uint2(0u, 0u);
        p.a = 0.0f;
        p.b = 0.0f;
        return p;
    }
    if (fast_scale(d))
        return make_plan_fast(x, d, __frcp_rn(d));
    float2 y[8];
#pragma unroll
    for (int j = 0; j < 8; ++j)
        y[j] = make_float2(__fdiv_rn(x[j].x, d), __fdiv_rn(x[j].y, d));
    return plan_from_quotients(x, y);
}

// G_M / 2 = D (D (s2/2) B - A) in fp64, exact (see the file comment); the
// factor 1/2 is common to both plans.
__device__ __forceinline__ double plan_g(float D, double s2h, const Plan &p)
{
    const double dD = (double)D;
    return dD * fma(dD * s2h, (double)p.b, -(double)p.a);
}

// The same decision, settled in fp32 for all but near-ties (fast path only:
// s2 in [2^-50, 2^50], both scale codes non-zero).  With D_M = m 2^e (m a
// 4-bit integer) the two scales satisfy 1 <= D4 / D6 <= 2, so e4 - e6 is 0
// or 1; B_M = k/4 with k <= 2304.  Hence D_M B_M (<= 16 bits) and D_M^2 B_M
// (<= 20 bits) are exact, and P = D6^2 B6 - D4^2 B4 is an integer multiple of
// 2^(2 e6 - 2) below 2^(2 e6 + 20): exact as well.  What remains rounds
// three times (v4 = D4 A4, Q = D6 A6 - v4, dl = s2/2 P - Q, each RN32 of an
// exact product or FMA), so dl differs from G6/2 - G4/2 by at most
// 2^-24 (|v4| + |Q| + |dl|) (1 + 2^-23).  When |dl| > 2^-20 (|v4| + |Q|)
// that error is below |dl| / 15: the sign of dl is the sign of the exact
// difference and it is not zero.  Otherwise it is a tie or a near-tie: equal
// scales (both saturated at 448, as in every block whose amax is within a
// few percent of the group amax) make the two plans identical, a tie kept at
// M=6; the rest goes to the fp64 decision above.
__device__ __forceinline__ bool prefer_four(float2 D, const GroupConst &gc, const Plan &p6, const Plan &p4)
{
    const float2 u = __fmul2_rn(D, make_float2(p6.b, p4.b));              // D B, exact
    const float P = __fmaf_rn(D.x, u.x, -__fmul_rn(D.y, u.y));            // exact
    const float v4 = __fmul_rn(D.y, p4.a);
    const float Q = __fmaf_rn(D.x, p6.a, -v4);
    const float dl = __fmaf_rn(gc.s2hf, P, -Q);
    if (fabsf(dl) > 0x1p-20f * (fabsf(v4) + fabsf(Q)))
        return dl > 0.0f;
    if (D.x == D.y)
        return false;
    return plan_g(D.y, gc.s2h, p4) < plan_g(D.x, gc.s2h, p6);
}

struct BlockOut {
    uint2 codes;
    uint32_t scale;
    bool m4;
    float amax;   // the block amax (Inf or NaN when an element is not finite)
};

__device__ __forceinline__ void unpack_x(const uint32_t (&w)[8], float2 (&x)[8])
{
#pragma unroll
    for (int j = 0; j < 8; ++j)
        x[j] = make_float2(bf16_lo(w[j]), bf16_hi(w[j]));
}

// The general block quantizer: any s2, any block scale (zero, or a divisor
// outside the fast range).  Taken for whole groups whose s2 is outside
// [2^-50, 2^50] and for blocks whose scale code is 0 in a plan.
template <bool FOUR_SIX>
__device__ __noinline__ BlockOut quantize_block_general(uint4 v0, uint4 v1, float amax_b, const GroupConst gc)
{
    BlockOut o;
    o.amax = amax_b;
    if (!(gc.s2 > 0.0f)) {  // all-zero group
        o.codes = make_uint2(0u, 0u);
        o.scale = 0u;
        o.m4 = false;
        return o;
    }
    const uint32_t w[8] = {v0.x, v0.y, v0.z, v0.w, v1.x, v1.y, v1.z, v1.w};
    float2 x[8];
    unpack_x(w, x);
    float t6, t4;
    if (gc.tfast) {
        t6 = div_bf16(amax_b, gc.den.x, -gc.nr.x);
        t4 = div_bf16(amax_b, gc.den.y, -gc.nr.y);
    } else {
        t6 = __fdiv_rn(amax_b, gc.den.x);
        t4 = __fdiv_rn(amax_b, gc.den.y);
    }
    const uint32_t sb = e4m3x2(t6, FOUR_SIX ? t4 : 0.0f);   // S6 low byte, S4 high
    const float2 D = f16x2_to_float2(e4m3x2_to_f16x2(sb));
    const float d6 = __fmul_rn(D.x, gc.s2), d4 = __fmul_rn(D.y, gc.s2);
    const Plan p6 = make_plan_any(x, d6);
    if (!FOUR_SIX) {
        o.codes = p6.codes;
        o.scale = sb & 0xFFu;
        o.m4 = false;
        return o;
    }
    const Plan p4 = make_plan_any(x, d4);
    const bool use4 = plan_g(D.y, gc.s2h, p4) < plan_g(D.x, gc.s2h, p6);
    o.codes = use4 ? p4.codes : p6.codes;
    o.scale = use4 ? (sb >> 8) : (sb & 0xFFu);
    o.m4 = use4;
    return o;
}

// One block of 16.  With s2 in [2^-50, 2^50] (`qfast`, uniform over a group)
// and both scale codes non-zero, every divisor lies in the exact range of
// the reciprocal quotient, so the two plans run straight-line with no range
// tests; the block amax quotients of both plans share packed operations, the
// two reciprocals come from one refined approximation pair (rcp2_rn_mid) and
// the M choice is settled in fp32 except at near-ties (prefer_four).
template <bool FOUR_SIX>
__device__ __forceinline__ BlockOut quantize_block(uint4 v0, uint4 v1, const GroupConst &gc)
{
    const uint32_t w[8] = {v0.x, v0.y, v0.z, v0.w, v1.x, v1.y, v1.z, v1.w};
    const uint32_t m = absmax_bf16x2(absmax_bf16x2(absmax_bf16x2(w[0], w[1]), absmax_bf16x2(w[2], w[3])),
                                     absmax_bf16x2(absmax_bf16x2(w[4], w[5]), absmax_bf16x2(w[6], w[7])));
    const float amax_b = __uint_as_float(fold_halves(m) << 16);
    if (!gc.qfast)
        return quantize_block_general<FOUR_SIX>(v0, v1, amax_b, gc);
    const float2 t = div2_bf16(make_float2(amax_b, amax_b), gc.den, gc.nr);
    const uint32_t sb = e4m3x2(t.x, FOUR_SIX ? t.y : 1.0f);   // S6 low byte, S4 high
    if ((sb & 0xFFu) == 0u || (sb & 0xFF00u) == 0u)
        return quantize_block_general<FOUR_SIX>(v0, v1, amax_b, gc);
    const float2 D = f16x2_to_float2(e4m3x2_to_f16x2(sb));
    const float2 d = __fmul2_rn(D, make_float2(gc.s2, gc.s2));
    float2 x[8];
    unpack_x(w, x);
    BlockOut o;
    o.amax = amax_b;
    if (!FOUR_SIX) {
        const Plan p6 = make_plan_fast(x, d.x, __frcp_rn(d.x));
        o.codes = p6.codes;
        o.scale = sb & 0xFFu;
        o.m4 = false;
        return o;
    }
    const float2 r = rcp2_rn_mid(d);                    // d in [2^-59, 2^59]
    const Plan p6 = make_plan_fast(x, d.x, r.x);
    const Plan p4 = make_plan_fast(x, d.y, r.y);
    const bool use4 = prefer_four(D, gc, p6, p4);
    o.codes = use4 ? p4.codes : p6.codes;
    o.scale = use4 ? (sb >> 8) : (sb & 0xFFu);
    o.m4 = use4;
    return o;
}

} // namespace mxq
