// verify.cu -- fused dequantize + relative-error reduction (sm_100a).
//
// Method (dabsLabs/Qwen3.8-Flash-Next-NVFP4, metric table: relative error
// of the quantized experts against the bf16 source, per tensor, mean and
// max over the census; azampatti/Qwen3.8-Flash-Next-FP4-Local-AZ, "The
// shared expert": error of the MXFP8 tensors against the bf16 master):
//   deq_i = (q_i * D) * s2         NVFP4 (q_i * D is exact in f16)
//   deq_i = q_i * 2^e              MXFP4 / MXFP8 (exact in fp32)
//   err_t = sum (x_i - deq_i)^2, ref_t = sum x_i^2 per tensor t,
// with e_i = RN32(x_i - deq_i) rounded once (for NVFP4 one FMA of the exact
// q_i * D with -s2), so each e_i^2 is within 2^-23 of its exact value.
// Squares are added by fp32 FMAs into pairs of partial sums of 8 terms
// (one pair per NVFP4 block, two per MX block), each pair added once in
// fp32 and then in fp64: err_t is within 11 * 2^-24 (6.6e-7) of the exact
// sum and ref_t within 9 * 2^-24, whatever the data.
//
// Fixed summation order: every tensor is cut into chunks of kVerifyChunk
// elements; one CTA reduces one chunk with a fixed thread -> element map,
// fp32 partials per block of 16 / 32, fp64 across blocks, a fixed shuffle
// tree and a fixed warp order.  The finalize kernel adds the chunk
// partials of each tensor in chunk order.  Results do not depend on
// scheduling, so repeated runs are bit-identical.
#include "mxq_device.cuh"
#include "mxq_internal.h"
#include "mxq.h"

namespace mxq {

__device__ __forceinline__ void accum_sq(float2 x, float2 deq, float2 &err, float2 &ref)
{
    const float2 e = __fadd2_rn(x, make_float2(-deq.x, -deq.y));
    err = __ffma2_rn(e, e, err);
    ref = __ffma2_rn(x, x, ref);
}

// One NVFP4 block of 16: x (2 x uint4), codes (uint2), scale byte, s2.
__device__ __forceinline__ void nvfp4_block_sq(uint4 v0, uint4 v1, uint2 c, uint32_t sbyte, float s2,
                                               double &err, double &ref)
{
    const uint32_t w[8] = {v0.x, v0.y, v0.z, v0.w, v1.x, v1.y, v1.z, v1.w};
    const uint32_t dh = e4m3x2_to_f16x2(sbyte);          // D in the low half
    const uint32_t dd = __byte_perm(dh, 0, 0x1010);      // D in both halves
    const float2 s22 = make_float2(-s2, -s2);
    float2 e2 = make_float2(0.f, 0.f), r2 = make_float2(0.f, 0.f);
    uint32_t q[8];
    e2m1x8_to_f16x2(c.x, *reinterpret_cast<uint32_t(*)[4]>(&q[0]));
    e2m1x8_to_f16x2(c.y, *reinterpret_cast<uint32_t(*)[4]>(&q[4]));
#pragma unroll
    for (int j = 0; j < 8; ++j) {
        const float2 qd = f16x2_to_float2(hmul2_bits(q[j], dd));   // q * D, exact
        const float2 x = make_float2(bf16_lo(w[j]), bf16_hi(w[j]));
        const float2 e = __ffma2_rn(qd, s22, x);                    // RN32(x - q D s2)
        e2 = __ffma2_rn(e, e, e2);
        r2 = __ffma2_rn(x, x, r2);
    }
    err += (double)__fadd_rn(e2.x, e2.y);
    ref += (double)__fadd_rn(r2.x, r2.y);
}

// One MX block of 32: x (4 x uint4), codes, scale byte.
template <int FMT>
__device__ __forceinline__ void mx_block_sq(const uint4 (&v)[4], const uint32_t *cw, uint32_t sbyte,
                                            double &err, double &ref)
{
    // 2^(sbyte - 127); sbyte = 0 is the subnormal 2^-127
    const float sc = sbyte ? __uint_as_float(sbyte << 23) : 0x1p-127f;
    const float2 sc2 = make_float2(sc, sc);
    const uint32_t w[16] = {v[0].x, v[0].y, v[0].z, v[0].w, v[1].x, v[1].y, v[1].z, v[1].w,
                            v[2].x, v[2].y, v[2].z, v[2].w, v[3].x, v[3].y, v[3].z, v[3].w};
    float2 e2 = make_float2(0.f, 0.f), r2 = make_float2(0.f, 0.f);
    uint32_t q4[16];
    if (FMT == MXQ_FMT_MXFP4) {
#pragma unroll
        for (int k = 0; k < 4; ++k)
            e2m1x8_to_f16x2(cw[k], *reinterpret_cast<uint32_t(*)[4]>(&q4[4 * k]));
    }
#pragma unroll
    for (int j = 0; j < 16; ++j) {
        const uint32_t qh = (FMT == MXQ_FMT_MXFP8)
                                ? e4m3x2_to_f16x2(j & 1 ? (cw[j >> 1] >> 16) : cw[j >> 1])
                                : q4[j];
        const float2 deq = __fmul2_rn(f16x2_to_float2(qh), sc2);   // exact
        accum_sq(make_float2(bf16_lo(w[j]), bf16_hi(w[j])), deq, e2, r2);
        if (j == 7) {   // each fp32 partial sums at most 8 squares, as for NVFP4
            err += (double)__fadd_rn(e2.x, e2.y);
            ref += (double)__fadd_rn(r2.x, r2.y);
            e2 = make_float2(0.f, 0.f);
            r2 = make_float2(0.f, 0.f);
        }
    }
    err += (double)__fadd_rn(e2.x, e2.y);
    ref += (double)__fadd_rn(r2.x, r2.y);
}

__device__ __forceinline__ void cta_reduce_store(double err, double ref, double *out2)
{
    __shared__ double s_err[kVerifyThreads / 32], s_ref[kVerifyThreads / 32];
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) {
        err += __shfl_down_sync(0xFFFFFFFFu, err, off);
        ref += __shfl_down_sync(0xFFFFFFFFu, ref, off);
    }
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    if (lane == 0) {
        s_err[warp] = err;
        s_ref[warp] = ref;
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        double a = 0.0, b = 0.0;
        for (int w = 0; w < kVerifyThreads / 32; ++w) {
            a += s_err[w];
            b += s_ref[w];
        }
        out2[0] = a;
        out2[1] = b;
    }
    __syncthreads();
}

// Four CTAs per SM (at most 64 registers): the loads a thread issues
// before its arithmetic are what keeps HBM busy, so occupancy sets the
// bytes in flight.
template <int FMT, bool SWZ>
__global__ void __launch_bounds__(kVerifyThreads, 4)
verify_chunk_kernel(const uint16_t *__restrict__ x, const uint8_t *__restrict__ codes,
                    const uint8_t *__restrict__ scales, const float *__restrict__ s2,
                    const ScaleLayout sl, int64_t n_tensors, int64_t rows, int64_t tsize,
                    int64_t chunks_per_tensor, int64_t tensors_per_scale, const FastDiv cptdiv,
                    const FastDiv tpsdiv, double *__restrict__ partials)
{
    constexpr int BLK = (FMT == MXQ_FMT_NVFP4) ? 16 : 32;
    // blocks per thread per chunk; all of a thread's loads are issued before
    // any of its arithmetic, so each thread keeps PER blocks in flight
    constexpr int PER = (int)(kVerifyChunk / BLK / kVerifyThreads);
    constexpr int XV = BLK / 8;                                   // uint4 of x per block
    constexpr int CV = (FMT == MXQ_FMT_MXFP8) ? 2 : 1;            // uint4 of codes (MX)
    const int64_t n_chunks = n_tensors * chunks_per_tensor;
    for (int64_t c = blockIdx.x; c < n_chunks; c += gridDim.x) {
        // chunk -> (tensor, chunk of the tensor) with one multiply-shift
        // division (chunk counts stay below 2^32: checked at launch)
        const int64_t t = fastdiv((uint32_t)c, cptdiv);
        const int64_t k = c - t * chunks_per_tensor;
        const int64_t ts = fastdiv((uint32_t)t, tpsdiv);      // scale matrix / s2 of tensor t
        const int64_t lo = k * kVerifyChunk;
        const int64_t hi = min(lo + kVerifyChunk, tsize);
        const int64_t nblk = (hi - lo) / BLK;
        const int64_t first = (t * tsize + lo) / BLK;   // global block index
        const float sv = (FMT == MXQ_FMT_NVFP4) ? __ldg(s2 + ts) : 0.0f;
        // tiled scales: tensor t is rows [(t % tps) * rows, ...) of matrix t / tps
        const uint64_t smat = SWZ ? (uint64_t)ts : 0;
        const uint32_t sb0 = SWZ ? (uint32_t)((t - ts * tensors_per_scale) * rows) * sl.cb + (uint32_t)(lo / BLK) : 0;
        uint4 xv[PER][XV];
        uint4 cv[PER][CV];
        uint2 c2[PER];
        uint32_t sb[PER];
#pragma unroll
        for (int u = 0; u < PER; ++u) {
            const int64_t i = threadIdx.x + (int64_t)u * kVerifyThreads;
            if (i < nblk) {
                const int64_t gb = first + i;
                const uint4 *src = reinterpret_cast<const uint4 *>(x) + gb * XV;
#pragma unroll
                for (int q = 0; q < XV; ++q)
                    xv[u][q] = __ldg(src + q);
                if (FMT == MXQ_FMT_NVFP4) {
                    c2[u] = __ldg(reinterpret_cast<const uint2 *>(codes) + gb);
                } else {
#pragma unroll
                    for (int q = 0; q < CV; ++q)
                        cv[u][q] = __ldg(reinterpret_cast<const uint4 *>(codes) + gb * CV + q);
                }
                sb[u] = __ldg(scales + (SWZ ? tiled_scale_offset(sl, smat, sb0 + (uint32_t)i) : (uint64_t)gb));
            }
        }
        double err = 0.0, ref = 0.0;
#pragma unroll
        for (int u = 0; u < PER; ++u) {
            const int64_t i = threadIdx.x + (int64_t)u * kVerifyThreads;
            if (i < nblk) {
                if (FMT == MXQ_FMT_NVFP4) {
                    nvfp4_block_sq(xv[u][0], xv[u][1], c2[u], sb[u], sv, err, ref);
                } else {
                    uint32_t cw[8];
                    cw[0] = cv[u][0].x; cw[1] = cv[u][0].y; cw[2] = cv[u][0].z; cw[3] = cv[u][0].w;
                    if (CV == 2) {
                        cw[4] = cv[u][CV - 1].x; cw[5] = cv[u][CV - 1].y;
                        cw[6] = cv[u][CV - 1].z; cw[7] = cv[u][CV - 1].w;
                    }
                    const uint4 v4[4] = {xv[u][0], xv[u][XV > 1 ? 1 : 0], xv[u][XV > 2 ? 2 : 0],
                                         xv[u][XV > 3 ? 3 : 0]};
                    mx_block_sq<FMT>(v4, cw, sb[u], err, ref);
                }
            }
        }
        cta_reduce_store(err, ref, partials + 2 * c);
    }
}

// One warp per tensor.  Lane l adds the chunk partials l, l + 32, ... in
// chunk order (coalesced 16-byte loads), then the 32 lane sums are combined
// by the same butterfly every time: a fixed summation order, so repeated
// runs give identical sums.
__global__ void verify_finalize_kernel(const double *__restrict__ partials, int64_t n_tensors,
                                       int64_t chunks_per_tensor, double *__restrict__ sum_sq_err,
                                       double *__restrict__ sum_sq_ref, double *__restrict__ relerr)
{
    const int64_t t = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const int lane = threadIdx.x & 31;
    if (t >= n_tensors)
        return;                                         // whole warp (n_tensors is warp-uniform)
    const double2 *p = reinterpret_cast<const double2 *>(partials) + t * chunks_per_tensor;
    double a = 0.0, b = 0.0;
    for (int64_t k = lane; k < chunks_per_tensor; k += 32) {
        const double2 v = p[k];
        a += v.x;
        b += v.y;
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        a += __shfl_xor_sync(0xFFFFFFFFu, a, o);
        b += __shfl_xor_sync(0xFFFFFFFFu, b, o);
    }
    if (lane == 0) {
        sum_sq_err[t] = a;
        sum_sq_ref[t] = b;
        if (relerr)
            relerr[t] = (b > 0.0) ? sqrt(a) / sqrt(b)
                                  : (a > 0.0 ? __longlong_as_double(0x7FF0000000000000LL) : 0.0);
    }
}

// ---------------------------------------------------------------------------
// Census of a conversion: the verifier's per-tensor figures reduced to the
// pages' summary figures (dabsLabs/Qwen3.8-Flash-Next-NVFP4, metric table:
// mean and max relative error over the expert tensors; "What makes this
// build different": total squared error of the 4/6 choice against plain
// RTN block scales, share of 16-blocks that chose M=4).  One CTA: thread t
// adds elements t, t + 256, ... in order, then a fixed tree, then the call's
// totals are added to the census; so a sequence of calls gives the same
// bits every time.
// ---------------------------------------------------------------------------
constexpr int kCensusThreads = 256;

__global__ void __launch_bounds__(kCensusThreads)
census_add_kernel(mxq_census *__restrict__ c, int64_t n_tensors, const double *__restrict__ err,
                  const double *__restrict__ ref, const double *__restrict__ rel,
                  const double *__restrict__ err_rtn, int64_t n_groups, const uint32_t *__restrict__ m4,
                  int64_t blocks_per_group)
{
    __shared__ double s_sum[4][kCensusThreads];
    __shared__ double s_max[kCensusThreads];
    __shared__ unsigned long long s_m4[kCensusThreads];
    const int t = threadIdx.x;
    double a = 0.0, b = 0.0, r = 0.0, q = 0.0, mx = 0.0;
    for (int64_t i = t; i < n_tensors; i += kCensusThreads) {
        r += rel[i];
        a += err[i];
        b += ref[i];
        if (err_rtn)
            q += err_rtn[i];
        mx = fmax(mx, rel[i]);
    }
    unsigned long long k = 0;
    for (int64_t g = t; g < n_groups; g += kCensusThreads)
        k += m4[g];
    s_sum[0][t] = r;
    s_sum[1][t] = a;
    s_sum[2][t] = b;
    s_sum[3][t] = q;
    s_max[t] = mx;
    s_m4[t] = k;
    __syncthreads();
    for (int off = kCensusThreads / 2; off > 0; off >>= 1) {
        if (t < off) {
#pragma unroll
            for (int j = 0; j < 4; ++j)
                s_sum[j][t] += s_sum[j][t + off];
            s_max[t] = fmax(s_max[t], s_max[t + off]);
            s_m4[t] += s_m4[t + off];
        }
        __syncthreads();
    }
    if (t == 0) {
        c->sum_relerr += s_sum[0][0];
        c->sum_sq_err += s_sum[1][0];
        c->sum_sq_ref += s_sum[2][0];
        if (n_tensors > 0)
            c->max_relerr = fmax(c->max_relerr, s_max[0]);
        c->n_tensors += (uint64_t)n_tensors;
        if (err_rtn) {
            c->sum_sq_err_rtn += s_sum[3][0];
            c->n_tensors_rtn += (uint64_t)n_tensors;
        }
        c->blocks += (uint64_t)(n_groups * blocks_per_group);
        c->blocks_m4 += s_m4[0];
        c->mean_relerr = c->n_tensors ? c->sum_relerr / (double)c->n_tensors : 0.0;
        c->sse_vs_rtn = (c->n_tensors > 0 && c->n_tensors_rtn == c->n_tensors && c->sum_sq_err_rtn > 0.0)
                            ? c->sum_sq_err / c->sum_sq_err_rtn - 1.0
                            : __longlong_as_double(0x7FF8000000000000LL);
        c->m4_fraction = c->blocks ? (double)c->blocks_m4 / (double)c->blocks : 0.0;
    }
}

cudaError_t launch_census_add(mxq_census *c, int64_t n_tensors, const double *err, const double *ref,
                              const double *rel, const double *err_rtn, int64_t n_groups, const uint32_t *m4,
                              int64_t blocks_per_group, cudaStream_t s)
{
    census_add_kernel<<<1, kCensusThreads, 0, s>>>(c, n_tensors, err, ref, rel, err_rtn, n_groups, m4,
                                                   blocks_per_group);
    return cudaGetLastError();
}

cudaError_t launch_verify(const uint16_t *x, const uint8_t *codes, const uint8_t *scales,
                          const float *s2, int fmt, const ScaleLayout &sl, int64_t n_tensors,
                          int64_t rows, int64_t tsize, int64_t tensors_per_scale, double *partials,
                          double *sum_sq_err, double *sum_sq_ref, double *relerr, cudaStream_t s)
{
    if (n_tensors == 0)
        return cudaSuccess;
    const int64_t cpt = tsize > 0 ? (tsize + kVerifyChunk - 1) / kVerifyChunk : 1;
    int64_t n_chunks = n_tensors * cpt;
    const unsigned grid = (unsigned)(n_chunks < 0x7FFFFFFF ? n_chunks : 0x7FFFFFFF);
    if (n_chunks > 0x7FFFFFFF || cpt > 0x7FFFFFFF || tensors_per_scale > 0x7FFFFFFF)
        return cudaErrorInvalidValue;                         // indices below are 32-bit
    const FastDiv cptdiv = make_fastdiv((uint32_t)cpt);
    const FastDiv tpsdiv = make_fastdiv((uint32_t)tensors_per_scale);
#define MXQ_VERIFY(F, W)                                                                      \
    verify_chunk_kernel<F, W><<<grid, kVerifyThreads, 0, s>>>(x, codes, scales, s2, sl, n_tensors, \
                                                              rows, tsize, cpt, tensors_per_scale, \
                                                              cptdiv, tpsdiv, partials)
    if (fmt == MXQ_FMT_NVFP4) {
        if (sl.swz) MXQ_VERIFY(MXQ_FMT_NVFP4, true); else MXQ_VERIFY(MXQ_FMT_NVFP4, false);
    } else if (fmt == MXQ_FMT_MXFP8) {
        if (sl.swz) MXQ_VERIFY(MXQ_FMT_MXFP8, true); else MXQ_VERIFY(MXQ_FMT_MXFP8, false);
    } else {
        if (sl.swz) MXQ_VERIFY(MXQ_FMT_MXFP4, true); else MXQ_VERIFY(MXQ_FMT_MXFP4, false);
    }
#undef MXQ_VERIFY
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess)
        return e;
    const unsigned fgrid = (unsigned)((n_tensors + 3) / 4);             // four warps (tensors) per CTA
    verify_finalize_kernel<<<fgrid, 128, 0, s>>>(partials, n_tensors, cpt, sum_sq_err, sum_sq_ref, relerr);
    return cudaGetLastError();
}

} // namespace mxq
