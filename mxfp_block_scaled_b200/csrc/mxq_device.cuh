// mxq_device.cuh -- device helpers shared by the quantizer and verifier
// kernels (sm_100a).  Number-format conversions use the PTX cvt
// instructions of the public PTX ISA (e2m1x2 / e4m3x2 packing and
// unpacking); everything else is plain IEEE fp32 / fp64 arithmetic with
// explicit rounding intrinsics, so no FMA contraction changes a result.
#pragma once

#include <cuda_runtime.h>
#include <cuda_fp16.h>
#include <cuda_bf16.h>
#include <stdint.h>

namespace mxq {

// ---- bf16 <-> fp32 ------------------------------------------------------
__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

// Running max of |x| over bf16x2 words, per half, in one instruction
// (max.NaN.xorsign.abs): the magnitude bits hold max(|acc|, |w|), the sign
// bit is garbage (the xor of the operands' signs) and is dropped by
// fold_halves.  NaN propagates as the canonical NaN, so a non-finite element
// leaves magnitude bits >= 0x7F80 (Inf or NaN) in its half.
__device__ __forceinline__ uint32_t absmax_bf16x2(uint32_t acc, uint32_t w)
{
    uint32_t r;
    asm("max.NaN.xorsign.abs.bf16x2 %0, %1, %2;" : "=r"(r) : "r"(acc), "r"(w));
    return r;
}
// Larger magnitude of the two halves of an absmax_bf16x2 result, as bf16
// bits (bit patterns of non-negative bf16 values order like the values).
__device__ __forceinline__ uint32_t fold_halves(uint32_t m) { return max(m & 0x7FFFu, (m >> 16) & 0x7FFFu); }

// ---- packed conversions (PTX ISA: cvt with .e2m1x2 / .e4m3x2) ------------
// Two fp32 values -> one byte of two E2M1 codes (lo in the low nibble),
// round to nearest even, saturating at +-6, sign kept; zero-extended.
// Bytes move between .b8 and 32-bit registers only with cvt.u8.u32 /
// cvt.u32.u8: vector moves of .b8 registers ({b0, b1, ...}) corrupted
// bytes when a packed word was unpacked again in the same kernel.
__device__ __forceinline__ uint32_t e2m1x2(float lo, float hi)
{
    uint32_t out;
    asm("{\n\t.reg .b8 t;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 t, %2, %1;\n\t"
        "cvt.u32.u8 %0, t;\n\t}"
        : "=r"(out) : "f"(lo), "f"(hi));
    return out;
}

// Eight fp32 values (four pairs) -> one word of eight E2M1 codes (pair j in
// byte j, element 2j in its low nibble) and the four decoded pairs as f16x2,
// decoded from the same byte registers.  The bytes are only ever packed into
// the word here, never unpacked from it.
__device__ __forceinline__ uint32_t e2m1x8_enc_dec(float2 p0, float2 p1, float2 p2, float2 p3,
                                                   uint32_t (&q)[4])
{
    uint32_t out;
    asm("{\n\t.reg .b8 b0, b1, b2, b3;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b0, %6, %5;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b1, %8, %7;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b2, %10, %9;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b3, %12, %11;\n\t"
        "cvt.rn.f16x2.e2m1x2 %1, b0;\n\t"
        "cvt.rn.f16x2.e2m1x2 %2, b1;\n\t"
        "cvt.rn.f16x2.e2m1x2 %3, b2;\n\t"
        "cvt.rn.f16x2.e2m1x2 %4, b3;\n\t"
        "mov.b32 %0, {b0, b1, b2, b3};\n\t}"
        : "=r"(out), "=r"(q[0]), "=r"(q[1]), "=r"(q[2]), "=r"(q[3])
        : "f"(p0.x), "f"(p0.y), "f"(p1.x), "f"(p1.y), "f"(p2.x), "f"(p2.y), "f"(p3.x), "f"(p3.y));
    return out;
}

// Four zero-extended bytes -> one word, b0 lowest.
__device__ __forceinline__ uint32_t pack4(uint32_t b0, uint32_t b1, uint32_t b2, uint32_t b3)
{
    return __byte_perm(__byte_perm(b0, b1, 0x0040), __byte_perm(b2, b3, 0x0040), 0x5410);
}

// Eight fp32 values -> eight E2M1 codes in one word, element 2j in the low
// nibble of byte j.
__device__ __forceinline__ uint32_t e2m1x8(float2 p0, float2 p1, float2 p2, float2 p3)
{
    return pack4(e2m1x2(p0.x, p0.y), e2m1x2(p1.x, p1.y), e2m1x2(p2.x, p2.y), e2m1x2(p3.x, p3.y));
}

// Low byte of `v` (two E2M1 codes) -> f16x2, low nibble in the low half.
__device__ __forceinline__ uint32_t e2m1x2_to_f16x2(uint32_t v)
{
    uint32_t out;
    asm("{\n\t.reg .b8 t;\n\t"
        "cvt.u8.u32 t, %1;\n\t"
        "cvt.rn.f16x2.e2m1x2 %0, t;\n\t}"
        : "=r"(out) : "r"(v));
    return out;
}

// The four bytes of `w` (eight E2M1 codes) -> four f16x2 values; pair j
// holds the codes of byte j.  Exact.
__device__ __forceinline__ void e2m1x8_to_f16x2(uint32_t w, uint32_t (&h)[4])
{
    h[0] = e2m1x2_to_f16x2(w);
    h[1] = e2m1x2_to_f16x2(w >> 8);
    h[2] = e2m1x2_to_f16x2(w >> 16);
    h[3] = e2m1x2_to_f16x2(w >> 24);
}

// Two fp32 -> two E4M3 bytes (lo from `lo`, hi from `hi`), round to nearest
// even, saturating at +-448 (never the NaN code).
__device__ __forceinline__ uint32_t e4m3x2(float lo, float hi)
{
    uint16_t out;
    asm("cvt.rn.satfinite.e4m3x2.f32 %0, %2, %1;" : "=h"(out) : "f"(lo), "f"(hi));
    return out;
}

// Two E4M3 bytes (low 16 bits of `v`) -> f16x2 values, exact.
__device__ __forceinline__ uint32_t e4m3x2_to_f16x2(uint32_t v)
{
    uint32_t out;
    uint16_t h = (uint16_t)v;
    asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(out) : "h"(h));
    return out;
}

__device__ __forceinline__ float2 f16x2_to_float2(uint32_t h)
{
    return __half22float2(*reinterpret_cast<const __half2 *>(&h));
}

__device__ __forceinline__ uint32_t hmul2_bits(uint32_t a, uint32_t b)
{
    __half2 r = __hmul2(*reinterpret_cast<const __half2 *>(&a), *reinterpret_cast<const __half2 *>(&b));
    return *reinterpret_cast<uint32_t *>(&r);
}

__device__ __forceinline__ uint32_t hadd2_bits(uint32_t a, uint32_t b)
{
    __half2 r = __hadd2(*reinterpret_cast<const __half2 *>(&a), *reinterpret_cast<const __half2 *>(&b));
    return *reinterpret_cast<uint32_t *>(&r);
}

__device__ __forceinline__ uint32_t hfma2_bits(uint32_t a, uint32_t b, uint32_t c)
{
    __half2 r = __hfma2(*reinterpret_cast<const __half2 *>(&a), *reinterpret_cast<const __half2 *>(&b),
                        *reinterpret_cast<const __half2 *>(&c));
    return *reinterpret_cast<uint32_t *>(&r);
}

// ---- correctly rounded quotient of a bf16 numerator ---------------------
// y = RN32(x / d) from r = RN32(1 / d) with one FMA correction (Markstein,
// IBM J. Res. Dev. 34(1), 1990).  Proven exact by exhaustion over every
// pair of significands (8-bit x, 24-bit d) for normal operands and results
// (tests/csrc/division_check.c); callers take __fdiv_rn outside that range.
// The residual is formed as q0*d - x and subtracted, which keeps -0 / d = -0.
__device__ __forceinline__ float div_bf16(float x, float d, float r)
{
    float q0 = __fmul_rn(x, r);
    float e = __fmaf_rn(q0, d, -x);
    return __fmaf_rn(-e, r, q0);
}

// Pairwise form of div_bf16 with nr = -r: the same IEEE operations, the
// negations moved onto operands, so each lane is bit-identical to it.
__device__ __forceinline__ float2 div2_bf16(float2 x, float2 d, float2 nr)
{
    const float2 q0 = __fmul2_rn(x, make_float2(-nr.x, -nr.y));        // x * r
    const float2 e = __ffma2_rn(q0, d, make_float2(-x.x, -x.y));        // q0 * d - x
    return __ffma2_rn(e, nr, q0);                                       // q0 - e * r
}

// ---- correctly rounded reciprocal of a pair -----------------------------
// RN32(1/d) for |d| in [2^-60, 2^60]: the hardware approximation
// (rcp.approx.ftz.f32 of the PTX ISA) refined by one Newton-Raphson step
// whose residual 1 - d*y0 is formed by an FMA (Markstein, IBM J. Res. Dev.
// 34(1), 1990).  In that range no operand or result is subnormal, so the
// result depends on the significand of d alone; it equals the correctly
// rounded reciprocal for every significand at every exponent of the range
// (exhaustive check on the device: tests/test_gpu_reciprocal.py).  Outside
// the range callers use __frcp_rn.
__device__ __forceinline__ float2 rcp2_rn_mid(float2 d)
{
    float2 y0;
    asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(y0.x) : "f"(d.x));
    asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(y0.y) : "f"(d.y));
    const float2 e = __ffma2_rn(make_float2(-d.x, -d.y), y0, make_float2(1.0f, 1.0f));
    return __ffma2_rn(y0, e, y0);
}

// One lane of rcp2_rn_mid: the same operations on a single value.
__device__ __forceinline__ float rcp_rn_mid(float d)
{
    float y0;
    asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(y0) : "f"(d));
    const float e = __fmaf_rn(-d, y0, 1.0f);
    return __fmaf_rn(y0, e, y0);
}

// ---- division by a run-time invariant divisor ---------------------------
// q = n / d for unsigned 32-bit n and 1 <= d < 2^31 with one high multiply
// (Granlund and Montgomery, "Division by invariant integers using
// multiplication", PLDI 1994, section 4): with l = ceil(log2 d) and
// m = floor(2^32 (2^l - d) / d) + 1, q = (t + ((n - t) >> 1)) >> (l - 1)
// where t = mulhi(m, n); d = 1 uses shift 0 and m = 0 (then q = n).
struct FastDiv {
    uint32_t d, m, s1, s2;
};

__host__ __device__ inline FastDiv make_fastdiv(uint32_t d)
{
    FastDiv f;
    f.d = d;
    uint32_t l = 0;
    while (l < 32 && (1ull << l) < d)
        ++l;
    f.m = (uint32_t)((((1ull << l) - d) << 32) / d + 1);
    f.s1 = l ? 1u : 0u;
    f.s2 = l ? l - 1 : 0u;
    if (d == 1)
        f.m = 0;
    return f;
}

__device__ __forceinline__ uint32_t fastdiv(uint32_t n, const FastDiv &f)
{
    const uint32_t t = __umulhi(f.m, n);
    return (t + ((n - t) >> f.s1)) >> f.s2;
}

// ---- 128x4 tiled scale layout ---------------------------------------------
// Byte offset of the scale of (row r, column c) of one scale matrix whose
// column count rounds up to `ntc` groups of 4: the matrix is cut into tiles
// of 128 rows x 4 columns (512 bytes each), stored row-tile-major
// (tile (r / 128, c / 4) at ((r / 128) * ntc + c / 4) * 512); inside a tile
// the byte of (r, c) sits at (r % 32) * 16 + ((r / 32) % 4) * 4 + c % 4.
// This is the scale-factor layout that block-scaled tensor-core GEMMs read
// (four 32-row slabs interleaved so that one 16-byte row holds the scales of
// rows r, r + 32, r + 64, r + 96 for four consecutive blocks).
__host__ __device__ __forceinline__ uint32_t swz128x4(uint32_t r, uint32_t c, uint32_t ntc)
{
    return (((r >> 7) * ntc + (c >> 2)) << 9) + ((r & 31u) << 4) + (((r >> 5) & 3u) << 2) + (c & 3u);
}

// Bytes of one scale matrix of `rows` x `cols` scales in the tiled layout
// (rows padded to 128, columns to 4).
__host__ __device__ __forceinline__ uint64_t swz128x4_bytes(uint64_t rows, uint64_t cols)
{
    return ((rows + 127) / 128) * 128 * (((cols + 3) / 4) * 4);
}

// Barrier `id` (1..15) among `count` threads (a multiple of 32).
__device__ __forceinline__ void named_barrier_sync(int id, int count)
{
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(count) : "memory");
}

__device__ __forceinline__ uint32_t ld_relaxed_u32(const uint32_t *p)
{
    uint32_t v;
    asm volatile("ld.relaxed.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}

__device__ __forceinline__ void red_relaxed_add_u32(uint32_t *p, uint32_t v)
{
    asm volatile("red.relaxed.gpu.global.add.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}

__device__ __forceinline__ unsigned long long ld_relaxed_u64(const unsigned long long *p)
{
    unsigned long long v;
    asm volatile("ld.relaxed.gpu.global.u64 %0, [%1];" : "=l"(v) : "l"(p) : "memory");
    return v;
}

__device__ __forceinline__ void st_relaxed_u64(unsigned long long *p, unsigned long long v)
{
    asm volatile("st.relaxed.gpu.global.u64 [%0], %1;" ::"l"(p), "l"(v) : "memory");
}

// ---- shared-memory barriers and bulk copies (PTX ISA, sm_90+) -----------
__device__ __forceinline__ uint32_t smem_addr(const void *p)
{
    return (uint32_t)__cvta_generic_to_shared(p);
}

__device__ __forceinline__ void mbar_init(uint64_t *bar, uint32_t count)
{
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_addr(bar)), "r"(count) : "memory");
}

__device__ __forceinline__ void fence_mbar_init()
{
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void fence_proxy_async_smem()
{
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t *bar)
{
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_addr(bar)) : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t *bar, uint32_t bytes)
{
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;"
                 ::"r"(smem_addr(bar)), "r"(bytes) : "memory");
}

// One bulk copy global -> shared (16-byte aligned, size a multiple of 16),
// completing `bytes` transactions on `bar`.
__device__ __forceinline__ void bulk_g2s(void *dst, const void *src, uint32_t bytes, uint64_t *bar)
{
    asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
                 ::"r"(smem_addr(dst)), "l"(src), "r"(bytes), "r"(smem_addr(bar)) : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t *bar, uint32_t parity)
{
    uint32_t ok;
    asm volatile("{\n\t.reg .pred p;\n\t"
                 "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
                 "selp.u32 %0, 1, 0, p;\n\t}"
                 : "=r"(ok) : "r"(smem_addr(bar)), "r"(parity) : "memory");
    return ok != 0;
}

// Non-blocking test of phase `parity` of `bar` (never suspends the thread).
__device__ __forceinline__ bool mbar_test_wait(uint64_t *bar, uint32_t parity)
{
    uint32_t ok;
    asm volatile("{\n\t.reg .pred p;\n\t"
                 "mbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
                 "selp.u32 %0, 1, 0, p;\n\t}"
                 : "=r"(ok) : "r"(smem_addr(bar)), "r"(parity) : "memory");
    return ok != 0;
}

} // namespace mxq
