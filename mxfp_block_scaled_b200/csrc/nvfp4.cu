// nvfp4.cu -- NVFP4 quantization with 4/6-optimal block scales (sm_100a).
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
// Pipeline: group_amax_kernel (pass 1) -> nvfp4_quant_kernel (pass 2).
#include <atomic>

#include <cooperative_groups.h>

#include "mxq_device.cuh"
#include "mxq_internal.h"
#include "mxq.h"
#include "mxq_test.h"

namespace mxq {

// ---------------------------------------------------------------------------
// Pass 1: per-group amax as bf16 magnitude bits (atomicMax is order-free).
// grid = (tiles of 512 blocks, groups); each thread reads 4 x 16 bytes.
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(kNvThreads)
group_amax_kernel(const uint4 *__restrict__ x, int64_t n_groups, int64_t nb,
                  uint32_t *__restrict__ amax_bits, uint32_t *__restrict__ status)
{
    __shared__ uint32_t warp_max[kNvThreads / 32];
    const int64_t vec_per_group = nb * 2;  // 16-byte vectors per group
    for (int64_t g = blockIdx.y; g < n_groups; g += gridDim.y) {
        const uint4 *xg = x + g * vec_per_group;
        uint32_t m = 0;
        for (int64_t base = (int64_t)blockIdx.x * (kNvTileBlocks * 2); base < vec_per_group;
             base += (int64_t)gridDim.x * (kNvTileBlocks * 2)) {
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                int64_t i = base + threadIdx.x + k * kNvThreads;
                if (i < vec_per_group) {
                    uint4 v = __ldg(xg + i);
                    m = absmax_bf16x2(m, v.x);
                    m = absmax_bf16x2(m, v.y);
                    m = absmax_bf16x2(m, v.z);
                    m = absmax_bf16x2(m, v.w);
                }
            }
        }
        uint32_t a = __reduce_max_sync(0xFFFFFFFFu, fold_halves(m));
        if ((threadIdx.x & 31) == 0)
            warp_max[threadIdx.x >> 5] = a;
        __syncthreads();
        if (threadIdx.x == 0) {
            uint32_t r = 0;
            for (int w = 0; w < kNvThreads / 32; ++w)
                r = max(r, warp_max[w]);
            if (r != 0)
                atomicMax(amax_bits + g, r);
            if (r >= 0x7F80u)
                atomicOr(status, MXQ_DEV_NONFINITE_INPUT);
        }
        __syncthreads();
    }
}

// ---------------------------------------------------------------------------
// Pass 2: the block quantizer.
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

__device__ __forceinline__ GroupConst make_group_const(uint32_t amax_bits)
{
    GroupConst c;
    const float amax = __uint_as_float(amax_bits << 16);
    c.s2 = __fdiv_rn(amax, kGlobalDivisor);
    c.den = make_float2(__fmul_rn(6.0f, c.s2), __fmul_rn(4.0f, c.s2));
    c.tfast = (c.s2 >= 0x1p-100f && c.s2 <= 0x1p100f) ? 1 : 0;
    c.qfast = (c.s2 >= 0x1p-50f && c.s2 <= 0x1p50f) ? 1 : 0;
    c.nr = c.tfast ? make_float2(-__frcp_rn(c.den.x), -__frcp_rn(c.den.y)) : make_float2(0.0f, 0.0f);
    c.s2h = 0.5 * (double)c.s2;
    c.s2hf = 0.5f * c.s2;
    return c;
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

// grid = (tiles of 512 blocks, groups).  Thread t of a tile handles blocks
// t and t + 256, so each warp covers 32 consecutive blocks per step and its
// M bits form one 32-bit word.
template <bool FOUR_SIX>
__global__ void __launch_bounds__(kNvThreads)
nvfp4_quant_kernel(const uint4 *__restrict__ x, int64_t n_groups, int64_t nb,
                   const uint32_t *__restrict__ amax_bits, uint2 *__restrict__ codes,
                   uint8_t *__restrict__ scales, const ScaleLayout sl, float *__restrict__ s2_out,
                   uint32_t *__restrict__ mbits, int mbits_atomic, uint32_t *__restrict__ m4_count)
{
    __shared__ GroupConst s_gc;
    __shared__ uint32_t s_m4;
    const int lane = threadIdx.x & 31;
    for (int64_t g = blockIdx.y; g < n_groups; g += gridDim.y) {
        if (threadIdx.x == 0) {
            s_gc = make_group_const(amax_bits[g]);
            if (blockIdx.x == 0)
                s2_out[g] = s_gc.s2;
            s_m4 = 0;
        }
        __syncthreads();
        const GroupConst gc = s_gc;
        uint32_t my_m4 = 0;
        for (int64_t tile = blockIdx.x; tile * kNvTileBlocks < nb; tile += gridDim.x) {
            const int64_t b0 = tile * kNvTileBlocks + threadIdx.x;
            uint4 v[2][2];
#pragma unroll
            for (int k = 0; k < 2; ++k) {
                const int64_t b = b0 + k * kNvThreads;
                if (b < nb) {
                    const uint4 *src = x + (g * nb + b) * 2;
                    v[k][0] = __ldg(src);
                    v[k][1] = __ldg(src + 1);
                }
            }
#pragma unroll
            for (int k = 0; k < 2; ++k) {
                const int64_t b = b0 + k * kNvThreads;
                const bool live = b < nb;
                BlockOut o;
                o.m4 = false;
                if (live) {
                    o = quantize_block<FOUR_SIX>(v[k][0], v[k][1], gc);
                    const int64_t gb = g * nb + b;
                    codes[gb] = o.codes;
                    scales[sl.swz ? tiled_scale_offset(sl, (uint64_t)g, (uint32_t)b) : (uint64_t)gb] =
                        (uint8_t)o.scale;
                }
                if (mbits) {
                    const uint32_t word = __ballot_sync(0xFFFFFFFFu, o.m4);
                    const int64_t warp_first = g * nb + (b - lane);
                    if (!mbits_atomic) {
                        if (lane == 0 && (b - lane) < nb)
                            mbits[warp_first >> 5] = word;
                    } else if (live && o.m4) {
                        const int64_t gb = g * nb + b;
                        atomicOr(mbits + (gb >> 5), 1u << (gb & 31));
                    }
                }
                my_m4 += o.m4 ? 1u : 0u;
            }
        }
        if (FOUR_SIX && m4_count) {
            const uint32_t wsum = __reduce_add_sync(0xFFFFFFFFu, my_m4);
            if (lane == 0 && wsum)
                atomicAdd(&s_m4, wsum);
            __syncthreads();
            if (threadIdx.x == 0 && s_m4)
                atomicAdd(m4_count + g, s_m4);
        }
        __syncthreads();
    }
}

// ---------------------------------------------------------------------------
// Single-pass schedule: nvfp4_fused_kernel.
//
// A cooperative persistent grid of one CTA per SM.  Every group's blocks are
// cut into one contiguous slice per CTA (a multiple of 32 blocks, so a warp's
// M bits fill one word).  Each CTA walks the groups in order; its slice of
// a group is brought into shared memory twice by bulk copies:
//   scout copy     (ring of `sstages`): two scout warps reduce the slice
//                  amax, publish it as one tagged 64-bit slot per group
//                  and CTA (tag and value land together: no fence needed)
//                  and then count the group's arrivals up by one;
//   quantize copy  (ring of `qstages`), issued only after the scouts are
//                  done with that group, `distance` groups behind them, so
//                  it normally hits the L2 copy the scout read left behind:
//                  20 compute warps quantize it once a publisher warp has
//                  seen every CTA's slot for the group.  The publisher polls
//                  only the one arrival word of a group; it reads the slots
//                  (and checks their tags) once the count is complete, so
//                  the polling of every CTA stays off the slots' L2 lines.
// The grid-wide amax of a group is therefore resolved while the compute
// warps work on earlier groups; its latency is off the critical path.
// Roles hand over through mbarriers (sfull / sfreed: scout ring, qfull /
// qfreed: quantize ring, ready: group amax known) and one shared counter
// (groups scouted).  Every wait is bounded: on time-out the CTA sets
// MXQ_DEV_WAIT_TIMEOUT, lets its copies in flight land (bounded) and
// returns.
// ---------------------------------------------------------------------------
struct FusedArgs {
    const uint16_t *x;
    int64_t n_groups, nb, slice;   // blocks per group, blocks per CTA slice
    int teams, team_size;          // the grid is `teams` teams of `team_size` CTAs
    int sstages, qstages, distance;
    uint32_t *status;
    unsigned long long *slots;     // [n_groups][kMaxFusedCtas] (tag << 32 | slice amax bits)
    uint32_t *arrived;             // [n_groups] slots stored so far (starts at 0)
    uint2 *codes;
    uint8_t *scales;
    ScaleLayout sl;
    float *s2_out;
    uint32_t *mbits, *m4_count;
    int test_stall;                // test hook: the publisher releases no group
};

constexpr uint32_t kSpinLimit = 1u << 22;   // polls of a flag / barrier before giving up
constexpr int kMaxStages = 8;
constexpr int kReadyRing = 16;   // > distance + qstages: ready phases never run a lap ahead
constexpr int kPollGroups = 4;   // groups whose readiness one publisher poll tests

// Bounded wait on an mbarrier phase that also gives up once another role of
// the CTA has aborted.  With `sleep_ns` the phase is tested without blocking
// and the warp sleeps about that long between tests: a blocking try_wait
// with a suspend-time hint keeps polling inside the instruction and takes
// issue slots from the compute warps of the same SM.
__device__ __forceinline__ bool wait_phase(uint64_t *bar, uint32_t parity, volatile int *abort_flag,
                                           uint32_t sleep_ns = 0)
{
    for (uint32_t i = 0; i < kSpinLimit; ++i) {
        if (sleep_ns ? mbar_test_wait(bar, parity) : mbar_try_wait(bar, parity))
            return true;
        if (*abort_flag)
            return false;
        if (sleep_ns)
            __nanosleep(sleep_ns);
    }
    *abort_flag = 1;
    return false;
}

template <bool FOUR_SIX, bool SWZ>
__global__ void __launch_bounds__(kFusedThreads, 1)
nvfp4_fused_kernel(const FusedArgs a)
{
    extern __shared__ __align__(128) uint8_t smem[];
    uint64_t *sfull = reinterpret_cast<uint64_t *>(smem);
    uint64_t *sfreed = sfull + kMaxStages;
    uint64_t *qfull = sfreed + kMaxStages;
    uint64_t *qfreed = qfull + kMaxStages;
    uint64_t *ready = qfreed + kMaxStages;              // kReadyRing barriers
    uint8_t *buf = smem + 512;
    __shared__ GroupConst s_gc[kReadyRing];             // group constants, set before ready
    __shared__ uint32_t s_scout_part[kFusedScoutWarps];
    __shared__ int s_scout_stop;
    __shared__ int s_scouted;                           // groups whose slot this CTA published
    __shared__ int s_abort;
    volatile int *abort_flag = &s_abort;
    volatile int *scouted = &s_scouted;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    // Team `team` takes groups team, team + teams, ...; rank is this CTA's
    // place in the team and picks its slice of each of those groups.
    const int team = (int)blockIdx.x / a.team_size, rank = (int)blockIdx.x % a.team_size;
    if (team >= a.teams)
        return;                                         // spare CTA (whole CTA: no barrier missed)
    const uint32_t P = (uint32_t)a.team_size;
    const int64_t my_lo = (int64_t)rank * a.slice;
    const int64_t my_n = max((int64_t)0, min(a.slice, a.nb - my_lo));   // multiple of 32
    const uint32_t bytes = (uint32_t)(my_n * 32);
    const int64_t stage_bytes = a.slice * 32;
    const int LS = a.sstages, LQ = a.qstages, D = a.distance;
    // groups of this team (the launch keeps n_groups below 2^31)
    const int G = a.n_groups > team ? (int)((a.n_groups - team + a.teams - 1) / a.teams) : 0;
    auto group_of = [&](int64_t i) -> int64_t { return team + i * a.teams; };
    uint8_t *sbuf = buf;                                // scout ring
    uint8_t *qbuf = buf + LS * stage_bytes;             // quantize ring

    if (threadIdx.x == 0) {
        for (int k = 0; k < kMaxStages; ++k) {
            mbar_init(sfull + k, 1);
            mbar_init(sfreed + k, kFusedScoutWarps);    // every scout warp
            mbar_init(qfull + k, 1);
            mbar_init(qfreed + k, kFusedComputeWarps);
        }
        for (int k = 0; k < kReadyRing; ++k)
            mbar_init(ready + k, 1);
        s_scouted = 0;
        s_abort = 0;
        fence_mbar_init();
    }
    __syncthreads();

    if (warp == 0) {
        // -------------------------------------------------------- publisher
        // Releases group j to the compute warps once all P CTAs have counted
        // their arrival for j and all P slots of j carry j's tag; the group
        // amax is the max over the slots.
        if (bytes == 0)
            return;                                     // no compute here to release
        int next_ready = 0;
        uint32_t idle = 0;
        while (next_ready < G) {
            bool progress = false;
            const int npoll = a.test_stall ? 0 : min(kPollGroups, *scouted - next_ready);
            if (npoll > 0) {
                uint32_t cnt = 0;
                if (lane < npoll)
                    cnt = ld_relaxed_u32(a.arrived + group_of(next_ready + lane));
                const uint32_t full = __ballot_sync(0xFFFFFFFFu, lane < npoll && cnt >= P);
                const int nfull = __ffs(~full) - 1;     // complete groups, in order
                for (int q = 0; q < nfull; ++q) {
                    const int64_t gq = group_of(next_ready);
                    const unsigned long long *sl = a.slots + gq * kMaxFusedCtas;
                    const uint32_t tag = (uint32_t)(gq + 1);
                    bool all = true;
                    uint32_t mx = 0;
                    for (uint32_t c = lane; c < P; c += 32) {
                        const unsigned long long v = ld_relaxed_u64(sl + c);
                        all = all && ((uint32_t)(v >> 32) == tag);
                        mx = max(mx, (uint32_t)v);
                    }
                    if (!__all_sync(0xFFFFFFFFu, all))
                        break;                          // a slot not visible yet: poll again
                    const uint32_t m = __reduce_max_sync(0xFFFFFFFFu, mx);
                    if (lane == 0) {
                        const int rs = next_ready & (kReadyRing - 1);
                        s_gc[rs] = make_group_const(m);
                        if (rank == 0)
                            a.s2_out[gq] = s_gc[rs].s2;
                        mbar_arrive(ready + rs);
                    }
                    ++next_ready;
                    progress = true;
                }
            }
            if (progress) {
                idle = 0;
            } else {
                if (__any_sync(0xFFFFFFFFu, ++idle > (kSpinLimit >> 4) || *abort_flag)) {
                    if (lane == 0) {
                        *abort_flag = 1;
                        atomicOr(a.status, MXQ_DEV_WAIT_TIMEOUT);
                    }
                    break;
                }
                __nanosleep(256);
            }
        }
        return;
    }
    if (warp == 1) {
        // ----------------------------------------------------------- loader
        // Scout copies run up to `distance` groups ahead of quantize copies;
        // a group's quantize copy waits until the scouts are done with it.
        if (lane != 0 || bytes == 0)
            return;
        // Stages and phase parities advance incrementally (no division).
        int s_next = 0, q_next = 0, s_st = 0, q_st = 0;
        uint32_t s_par = 0, q_par = 0;                  // parity of (next / ring size)
        int s_last[kMaxStages], q_last[kMaxStages];     // phase parity of the copy in flight, or -1
        for (int k = 0; k < kMaxStages; ++k)
            s_last[k] = q_last[k] = -1;
        uint32_t idle = 0;
        while (q_next < G) {
            bool progress = false;
            if (s_next < G && s_next < q_next + D) {
                if (s_next < LS || mbar_test_wait(sfreed + s_st, s_par ^ 1u)) {
                    fence_proxy_async_smem();
                    mbar_arrive_expect_tx(sfull + s_st, bytes);
                    bulk_g2s(sbuf + s_st * stage_bytes, a.x + (group_of(s_next) * a.nb + my_lo) * 16, bytes,
                             sfull + s_st);
                    s_last[s_st] = (int)s_par;
                    ++s_next;
                    if (++s_st == LS) {
                        s_st = 0;
                        s_par ^= 1u;
                    }
                    progress = true;
                }
            }
            if (q_next < *scouted) {
                if (q_next < LQ || mbar_test_wait(qfreed + q_st, q_par ^ 1u)) {
                    fence_proxy_async_smem();
                    mbar_arrive_expect_tx(qfull + q_st, bytes);
                    bulk_g2s(qbuf + q_st * stage_bytes, a.x + (group_of(q_next) * a.nb + my_lo) * 16, bytes,
                             qfull + q_st);
                    q_last[q_st] = (int)q_par;
                    ++q_next;
                    if (++q_st == LQ) {
                        q_st = 0;
                        q_par ^= 1u;
                    }
                    progress = true;
                }
            }
            if (progress) {
                idle = 0;
            } else if (++idle > kSpinLimit || *abort_flag) {
                *abort_flag = 1;
                atomicOr(a.status, MXQ_DEV_WAIT_TIMEOUT);
                break;
            } else {
                __nanosleep(200);
            }
        }
        if (*abort_flag) {
            // let this CTA's copies in flight land before its smem is released
            for (int k = 0; k < kMaxStages; ++k) {
                if (s_last[k] >= 0)
                    for (uint32_t n = 0; n < kSpinLimit; ++n)
                        if (mbar_try_wait(sfull + k, (uint32_t)s_last[k]))
                            break;
                if (q_last[k] >= 0)
                    for (uint32_t n = 0; n < kSpinLimit; ++n)
                        if (mbar_try_wait(qfull + k, (uint32_t)q_last[k]))
                            break;
            }
        }
        return;
    }
    if (warp < 2 + kFusedScoutWarps) {
        // ----------------------------------------------------------- scouts
        // The scout warps meet at a named barrier twice per group; the
        // decision to stop is taken from a flag snapshot written before the
        // first meeting, so every scout warp makes the same choice.
        const int sw = warp - 2;
        const int nvec = (int)(my_n * 2);               // 16-byte vectors of the slice
        int st = 0;
        uint32_t par = 0;
        for (int g = 0; g < G; ++g) {
            bool ok = true;
            if (bytes)
                ok = __all_sync(0xFFFFFFFFu, wait_phase(sfull + st, par, abort_flag, 500u));
            uint32_t m = 0;
            if (ok && bytes) {
                const uint4 *v = reinterpret_cast<const uint4 *>(sbuf + st * stage_bytes);
#pragma unroll 2
                for (int u = lane + 32 * sw; u < nvec; u += 32 * kFusedScoutWarps) {
                    const uint4 q = v[u];
                    m = absmax_bf16x2(m, q.x);
                    m = absmax_bf16x2(m, q.y);
                    m = absmax_bf16x2(m, q.z);
                    m = absmax_bf16x2(m, q.w);
                }
            }
            const uint32_t r = __reduce_max_sync(0xFFFFFFFFu, fold_halves(m));
            if (lane == 0) {
                s_scout_part[sw] = r;
                if (!ok)
                    *abort_flag = 1;
            }
            if (sw == 0 && lane == 0)
                s_scout_stop = *abort_flag;
            named_barrier_sync(1, 32 * kFusedScoutWarps);   // parts written, stop decided
            const int stop = s_scout_stop;
            if (!stop && sw == 0 && lane == 0) {
                uint32_t mx = 0;
                for (int k = 0; k < kFusedScoutWarps; ++k)
                    mx = max(mx, s_scout_part[k]);
                if (mx >= 0x7F80u)
                    atomicOr(a.status, MXQ_DEV_NONFINITE_INPUT);
                const int64_t gg = group_of(g);
                st_relaxed_u64(a.slots + gg * kMaxFusedCtas + rank,
                               ((unsigned long long)(gg + 1) << 32) | mx);
                red_relaxed_add_u32(a.arrived + gg, 1u);
                *scouted = (int)(g + 1);
            }
            named_barrier_sync(1, 32 * kFusedScoutWarps);   // parts and snapshot may be rewritten
            if (stop)
                break;
            if (lane == 0 && bytes)
                mbar_arrive(sfreed + st);
            if (++st == LS) {
                st = 0;
                par ^= 1u;
            }
        }
        return;
    }

    // -------------------------------------------------------- compute warps
    if (bytes == 0)
        return;
    // Chunks of 32 blocks are dealt per SM sub-partition (warp index mod 4):
    // the n32 chunks of a group are cut into four runs, the longer runs going
    // to sub-partitions 0 and 1, which host the light publisher and loader
    // warps, and the shorter ones to 2 and 3, which host the scout warps (with
    // the 42 chunks of the full-size slices: 11, 11, 10, 10).  Inside a
    // sub-partition the chunks go round-robin over its compute warps along
    // the whole group sequence, so a run whose length is not a multiple of
    // the warp count stays balanced; a warp with no chunk in a group still
    // frees the group's buffer.
    static_assert(kFusedComputeWarps % 4 == 0 && (2 + kFusedScoutWarps) % 4 == 0,
                  "compute warps must fill the four sub-partitions evenly");
    constexpr int kWarpsPerPart = kFusedComputeWarps / 4;
    const int cw = warp - 2 - kFusedScoutWarps;
    const int part = warp & 3, li = cw >> 2;            // sub-partition, index inside it
    const int n32 = (int)(my_n / 32);
    const int run = (n32 >> 2) + (part < (n32 & 3) ? 1 : 0);
    const int run0 = part * (n32 >> 2) + min(part, n32 & 3);
    const int step = run % kWarpsPerPart;               // offset gained per group
    int first = li;                                     // this warp's first chunk of the run
    int st = 0, rs = 0;                                 // quantize stage and ready slot of group j
    uint32_t qpar = 0, rpar = 0;                        // their phase parities
    for (int j = 0; j < G; ++j) {
        bool ok = wait_phase(ready + rs, rpar, abort_flag, 200u);
        ok = ok && wait_phase(qfull + st, qpar, abort_flag, 200u);
        if (!__all_sync(0xFFFFFFFFu, ok))
            break;
        const GroupConst gc = s_gc[rs];
        const uint4 *v = reinterpret_cast<const uint4 *>(qbuf + st * stage_bytes);
        const int64_t gj = group_of(j);
        const int64_t gb0 = gj * a.nb + my_lo;            // first block of the slice
        uint2 *codes = a.codes + gb0;
        uint8_t *scales = a.scales + gb0;
        uint32_t *mbits = a.mbits ? a.mbits + (gb0 >> 5) : nullptr;
        uint32_t cnt = 0;
        for (int c = first; c < run; c += kWarpsPerPart) {
            const int k32 = run0 + c;
            const int k = k32 * 32 + lane;
            const BlockOut o = quantize_block<FOUR_SIX>(v[2 * k], v[2 * k + 1], gc);
            codes[k] = o.codes;
            if (SWZ)
                a.scales[tiled_scale_offset(a.sl, (uint64_t)gj, (uint32_t)(my_lo + k))] = (uint8_t)o.scale;
            else
                scales[k] = (uint8_t)o.scale;
            const uint32_t word = __ballot_sync(0xFFFFFFFFu, o.m4);
            if (lane == 0) {
                if (mbits)
                    mbits[k32] = word;
                cnt += __popc(word);
            }
        }
        __syncwarp();
        if (lane == 0) {
            if (a.m4_count && cnt)
                atomicAdd(a.m4_count + gj, cnt);
            mbar_arrive(qfreed + st);
        }
        if (++st == LQ) {
            st = 0;
            qpar ^= 1u;
        }
        if (++rs == kReadyRing) {
            rs = 0;
            rpar ^= 1u;
        }
        first -= step;                                  // (li - run * (j + 1)) mod warps
        if (first < 0)
            first += kWarpsPerPart;
    }
}

cudaError_t launch_group_amax(const uint16_t *x, int64_t n_groups, int64_t nb,
                              uint32_t *amax_bits, uint32_t *status, cudaStream_t s)
{
    if (n_groups == 0 || nb == 0)
        return cudaSuccess;
    const int64_t tiles = (nb + kNvTileBlocks - 1) / kNvTileBlocks;
    dim3 grid((unsigned)(tiles < 0x7FFFFFFF ? tiles : 0x7FFFFFFF),
              (unsigned)(n_groups < 65535 ? n_groups : 65535));
    group_amax_kernel<<<grid, kNvThreads, 0, s>>>(reinterpret_cast<const uint4 *>(x), n_groups, nb,
                                                  amax_bits, status);
    return cudaGetLastError();
}

// Test hook (include/mxq_test.h): the next single-pass launch stalls on
// purpose and must end with MXQ_DEV_WAIT_TIMEOUT.
static std::atomic<int> g_test_stall{0};

static int sm_count()
{
    int dev = 0, n = 0;
    if (cudaGetDevice(&dev) != cudaSuccess)
        return 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
        return 0;
    return n;
}

// Returns cudaErrorNotSupported (and launches nothing) when the shape or the
// device does not suit the single-pass schedule; the caller then takes the
// two-pass path.
cudaError_t launch_nvfp4_fused(const uint16_t *x, int64_t n_groups, int64_t nb, int four_six,
                               unsigned long long *slots, uint32_t *arrived, uint8_t *codes, uint8_t *scales,
                               const ScaleLayout &sl, float *s2, uint32_t *mbits, uint32_t *m4_count,
                               uint32_t *status, cudaStream_t s)
{
    if (n_groups <= 0 || n_groups > 0x7FFFFFFF || nb <= 0 || nb % 32 != 0)
        return cudaErrorNotSupported;
    int dev = 0, coop = 0, max_optin = 0;
    if (cudaGetDevice(&dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&coop, cudaDevAttrCooperativeLaunch, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&max_optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev) != cudaSuccess)
        return cudaErrorNotSupported;
    const int sms = sm_count();
    if (!coop || sms <= 0 || !slots || !arrived)
        return cudaErrorNotSupported;
    // Teams: the largest number of teams whose slices (one per CTA of a
    // team) still fit four stage buffers; small groups then get larger
    // slices and fewer, cheaper hand-overs.
    const int64_t avail = (int64_t)max_optin - 512 - 2048;   // barriers + static smem margin
    const int64_t target = avail / 4;
    int teams = 1, team_size = sms;
    int64_t slice = 0;
    for (int h = (int)min((int64_t)sms, n_groups); h >= 1; --h) {
        const int ts = sms / h;
        if (ts > kMaxFusedCtas)
            continue;
        int64_t sl = (nb + ts - 1) / ts;
        sl = (sl + 31) / 32 * 32;
        if (sl * 32 <= target || h == 1) {
            teams = h;
            team_size = ts;
            slice = sl;
            break;
        }
    }
    if (team_size > kMaxFusedCtas)
        return cudaErrorNotSupported;
    const int64_t slice_bytes = slice * 32;
    const int64_t stages = avail / slice_bytes;               // scout + quantize buffers
    if (stages < 2)
        return cudaErrorNotSupported;
    // Split the buffers between the two rings; the scouts run `distance`
    // groups ahead of the compute warps.
    int LS = (int)(stages / 2), LQ = (int)(stages - stages / 2);
    if (LS > kMaxStages)
        LS = kMaxStages;
    if (LQ > kMaxStages)
        LQ = kMaxStages;
    const int D = LQ + 2 <= kReadyRing - 1 - LQ ? LQ + 2 : kReadyRing - 1 - LQ;
    const size_t dyn = 512 + (size_t)(LS + LQ) * (size_t)slice_bytes;
    const void *fn = four_six ? (sl.swz ? (const void *)nvfp4_fused_kernel<true, true>
                                        : (const void *)nvfp4_fused_kernel<true, false>)
                              : (sl.swz ? (const void *)nvfp4_fused_kernel<false, true>
                                        : (const void *)nvfp4_fused_kernel<false, false>);
    cudaError_t e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)dyn);
    if (e != cudaSuccess)
        return e;
    int per_sm = 0;
    e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, fn, kFusedThreads, dyn);
    if (e != cudaSuccess)
        return e;
    if (per_sm < 1)
        return cudaErrorNotSupported;
    FusedArgs args;
    args.x = x;
    args.n_groups = n_groups;
    args.nb = nb;
    args.slice = slice;
    args.teams = teams;
    args.team_size = team_size;
    args.sstages = LS;
    args.qstages = LQ;
    args.distance = D;
    args.slots = slots;
    args.arrived = arrived;
    args.status = status;
    args.codes = reinterpret_cast<uint2 *>(codes);
    args.scales = scales;
    args.sl = sl;
    args.s2_out = s2;
    args.mbits = mbits;
    args.m4_count = four_six ? m4_count : nullptr;
    args.test_stall = g_test_stall.exchange(0) ? 1 : 0;
    void *params[] = {&args};
    return cudaLaunchCooperativeKernel(fn, dim3((unsigned)sms), dim3(kFusedThreads), params, dyn, s);
}

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
// W32 = sum h (x - RN32(qD s2))^2 with one rounding per operation.
__device__ __forceinline__ float block_wsse32(const float2 (&xf)[8], const float2 (&h2)[8], uint2 c, float D,
                                              float s2)
{
    uint32_t q[8];
    e2m1x8_to_f16x2(c.x, *reinterpret_cast<uint32_t(*)[4]>(&q[0]));
    e2m1x8_to_f16x2(c.y, *reinterpret_cast<uint32_t(*)[4]>(&q[4]));
    const float2 D2 = make_float2(D, D), S2 = make_float2(s2, s2);
    float2 acc = make_float2(0.0f, 0.0f);
#pragma unroll
    for (int j = 0; j < 8; ++j) {
        const float2 deq = __fmul2_rn(__fmul2_rn(f16x2_to_float2(q[j]), D2), S2);
        const float2 e = __fadd2_rn(xf[j], make_float2(-deq.x, -deq.y));
        acc = __ffma2_rn(h2[j], __fmul2_rn(e, e), acc);
    }
    return __fadd_rn(acc.x, acc.y);
}

// Error bound of W32 against the exact weighted error W, and against the
// binary64 value the definition forms.  With u = 2^-24, A = sum h x^2 and
// Cauchy-Schwarz on sum h |x| |e|, the rounding of deq and e costs at most
// 2u (sqrt(A W) + 2 W) + O(u^2 A), the products and the eight-step pair
// sums at most 10u W32; bounding W by W32 the same way gives
// |W32 - W| <= 2.1u sqrt(A W32) + 14.7u W32 + 4.2u^2 A.  The constants
// below take about twice that, which also covers the binary64 procedure's
// own error (below 2^-48 W) and the error of forming the bound in fp32.
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

__global__ void __launch_bounds__(kNvThreads)
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
                for (uint32_t sc = lo; sc <= hi; ++sc) {
                    const float D = f16x2_to_float2(e4m3x2_to_f16x2(sc)).x;
                    const Plan p = make_plan_any(xf, __fmul_rn(D, gc.s2));
                    const float wv = block_wsse32(xf, h2, p.codes, D, gc.s2);
                    const float ev = wsse_bound(wv, sqrtA_scaled, c_block);
                    if (sc == lo || wv < bw) {
                        if (sc != lo)
                            lb = fminf(lb, __fsub_rn(bw, be));
                        bw = wv;
                        be = ev;
                        best_sc = sc;
                        best_c = p.codes;
                    } else {
                        lb = fminf(lb, __fsub_rn(wv, ev));
                    }
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

cudaError_t launch_nvfp4_quant(const uint16_t *x, int64_t n_groups, int64_t nb, int four_six,
                               const uint32_t *amax_bits, uint8_t *codes, uint8_t *scales,
                               const ScaleLayout &sl, float *s2, uint32_t *mbits, int mbits_atomic,
                               uint32_t *m4_count, cudaStream_t s)
{
    if (n_groups == 0)
        return cudaSuccess;
    const int64_t tiles = nb > 0 ? (nb + kNvTileBlocks - 1) / kNvTileBlocks : 1;
    dim3 grid((unsigned)(tiles < 0x7FFFFFFF ? tiles : 0x7FFFFFFF),
              (unsigned)(n_groups < 65535 ? n_groups : 65535));
    const uint4 *xv = reinterpret_cast<const uint4 *>(x);
    uint2 *cv = reinterpret_cast<uint2 *>(codes);
    if (four_six)
        nvfp4_quant_kernel<true><<<grid, kNvThreads, 0, s>>>(xv, n_groups, nb, amax_bits, cv, scales,
                                                             sl, s2, mbits, mbits_atomic, m4_count);
    else
        nvfp4_quant_kernel<false><<<grid, kNvThreads, 0, s>>>(xv, n_groups, nb, amax_bits, cv, scales,
                                                              sl, s2, mbits, mbits_atomic, m4_count);
    return cudaGetLastError();
}

// ---------------------------------------------------------------------------
// One small group (an activation tile of up to a few hundred tokens) by one
// thread-block cluster of P CTAs: each CTA copies its share of the blocks
// into shared memory while reducing its amax, the cluster combines the P
// maxima through distributed shared memory, and each CTA quantizes its share
// from shared memory.  One launch, no grid-wide hand-over and no workspace.
// Shares are multiples of 32 blocks, so each warp's M bits fill one word.
// ---------------------------------------------------------------------------
constexpr int kSmallThreads = 512;
constexpr int kSmallMaxCtas = 16;

template <bool FOUR_SIX, bool SWZ>
__global__ void __launch_bounds__(kSmallThreads)
nvfp4_small_kernel(const uint4 *__restrict__ x, int64_t nb, int64_t share, uint2 *__restrict__ codes,
                   uint8_t *__restrict__ scales, const ScaleLayout sl, float *__restrict__ s2_out,
                   uint32_t *__restrict__ mbits, uint32_t *__restrict__ m4_count, uint32_t *__restrict__ status)
{
    namespace cg = cooperative_groups;
    extern __shared__ uint4 tile[];                     // 2 vectors per block of this CTA's share
    __shared__ uint32_t s_warp[kSmallThreads / 32];
    __shared__ uint32_t s_amax;                         // this CTA's amax, read by the whole cluster
    __shared__ GroupConst s_gc;
    __shared__ uint32_t s_m4;
    cg::cluster_group cluster = cg::this_cluster();
    const unsigned rank = cluster.block_rank(), P = cluster.num_blocks();
    const int64_t b0 = min(nb, (int64_t)rank * share);
    const int n = (int)(min(nb, b0 + share) - b0);
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;

    // eight loads in flight per thread before any is used: a 64 KB share
    // arrives in one memory round trip
    uint32_t m = 0;
    for (int base = 0; base < 2 * n; base += 8 * kSmallThreads) {
        uint4 v[8];
#pragma unroll
        for (int u = 0; u < 8; ++u) {
            const int i = base + u * kSmallThreads + threadIdx.x;
            if (i < 2 * n)
                v[u] = __ldg(x + 2 * b0 + i);
        }
#pragma unroll
        for (int u = 0; u < 8; ++u) {
            const int i = base + u * kSmallThreads + threadIdx.x;
            if (i < 2 * n) {
                tile[i] = v[u];
                m = absmax_bf16x2(absmax_bf16x2(m, v[u].x), absmax_bf16x2(v[u].y, v[u].z));
                m = absmax_bf16x2(m, v[u].w);
            }
        }
    }
    m = __reduce_max_sync(0xFFFFFFFFu, fold_halves(m));
    if (lane == 0)
        s_warp[warp] = m;
    if (threadIdx.x == 0)
        s_m4 = 0;
    __syncthreads();
    if (threadIdx.x == 0) {
        uint32_t a = 0;
        for (int w = 0; w < kSmallThreads / 32; ++w)
            a = max(a, s_warp[w]);
        s_amax = a;
    }
    cluster.sync();                                     // every CTA's s_amax is written
    if (threadIdx.x == 0) {
        uint32_t g = 0;
        for (unsigned r = 0; r < P; ++r)
            g = max(g, *cluster.map_shared_rank(&s_amax, r));
        s_gc = make_group_const(g);
        if (rank == 0) {
            s2_out[0] = s_gc.s2;
            if (g >= 0x7F80u)
                atomicOr(status, MXQ_DEV_NONFINITE_INPUT);
        }
    }
    cluster.sync();                                     // remote reads done; s_gc set
    const GroupConst gc = s_gc;
    uint32_t my_m4 = 0;
    for (int base = 0; base < n; base += kSmallThreads) {
        const int j = base + threadIdx.x;
        const bool live = j < n;
        BlockOut o;
        o.m4 = false;
        if (live) {
            o = quantize_block<FOUR_SIX>(tile[2 * j], tile[2 * j + 1], gc);
            const int64_t b = b0 + j;
            codes[b] = o.codes;
            scales[SWZ ? tiled_scale_offset(sl, 0, (uint32_t)b) : (uint64_t)b] = (uint8_t)o.scale;
        }
        if (mbits) {
            const uint32_t word = __ballot_sync(0xFFFFFFFFu, o.m4);
            const int64_t first = b0 + base + 32 * warp;   // first block of this warp's word
            if (lane == 0 && first < b0 + n)
                mbits[first >> 5] = word;
        }
        my_m4 += o.m4 ? 1u : 0u;
    }
    if (FOUR_SIX && m4_count) {
        const uint32_t wsum = __reduce_add_sync(0xFFFFFFFFu, my_m4);
        if (lane == 0 && wsum)
            atomicAdd(&s_m4, wsum);
        __syncthreads();
        if (threadIdx.x == 0 && s_m4)
            atomicAdd(m4_count, s_m4);
    }
}

cudaError_t launch_nvfp4_small(const uint16_t *x, int64_t nb, int four_six, uint8_t *codes, uint8_t *scales,
                               const ScaleLayout &sl, float *s2, uint32_t *mbits, uint32_t *m4_count,
                               uint32_t *status, cudaStream_t s)
{
    if (nb <= 0 || nb > kSmallMaxBlocks)
        return cudaErrorNotSupported;
    int dev = 0, cluster_ok = 0, max_optin = 0;
    if (cudaGetDevice(&dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&cluster_ok, cudaDevAttrClusterLaunch, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&max_optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev) != cudaSuccess ||
        !cluster_ok)
        return cudaErrorNotSupported;
    // about 16 KB of the tile per CTA (up to 16 CTAs), shares a multiple of
    // 32 blocks
    int P = (int)((nb * 32 + 16383) / 16384);
    P = P < 1 ? 1 : (P > kSmallMaxCtas ? kSmallMaxCtas : P);
    int64_t share = (nb + P - 1) / P;
    share = (share + 31) / 32 * 32;
    P = (int)((nb + share - 1) / share);
    const size_t dyn = (size_t)share * 32;
    if (dyn + 4096 > (size_t)max_optin)
        return cudaErrorNotSupported;
    const void *fn = four_six ? (sl.swz ? (const void *)nvfp4_small_kernel<true, true>
                                        : (const void *)nvfp4_small_kernel<true, false>)
                              : (sl.swz ? (const void *)nvfp4_small_kernel<false, true>
                                        : (const void *)nvfp4_small_kernel<false, false>);
    cudaError_t e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)dyn);
    if (e == cudaSuccess && P > 8)
        e = cudaFuncSetAttribute(fn, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
    if (e != cudaSuccess) {
        (void)cudaGetLastError();
        return cudaErrorNotSupported;
    }
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)P);
    cfg.blockDim = dim3(kSmallThreads);
    cfg.dynamicSmemBytes = dyn;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = (unsigned)P;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    int clusters = 0;
    e = cudaOccupancyMaxActiveClusters(&clusters, fn, &cfg);
    if (e != cudaSuccess || clusters < 1) {
        (void)cudaGetLastError();
        return cudaErrorNotSupported;
    }
    const uint4 *xv = reinterpret_cast<const uint4 *>(x);
    uint2 *cv = reinterpret_cast<uint2 *>(codes);
    if (four_six) {
        if (sl.swz)
            e = cudaLaunchKernelEx(&cfg, nvfp4_small_kernel<true, true>, xv, nb, share, cv, scales, sl, s2, mbits,
                                   m4_count, status);
        else
            e = cudaLaunchKernelEx(&cfg, nvfp4_small_kernel<true, false>, xv, nb, share, cv, scales, sl, s2, mbits,
                                   m4_count, status);
    } else {
        if (sl.swz)
            e = cudaLaunchKernelEx(&cfg, nvfp4_small_kernel<false, true>, xv, nb, share, cv, scales, sl, s2,
                                   mbits, m4_count, status);
        else
            e = cudaLaunchKernelEx(&cfg, nvfp4_small_kernel<false, false>, xv, nb, share, cv, scales, sl, s2,
                                   mbits, m4_count, status);
    }
    return e;
}

} // namespace mxq

extern "C" MXQ_API void mxq_test_stall_next_single_pass(int on)
{
    mxq::g_test_stall.store(on ? 1 : 0);
}
