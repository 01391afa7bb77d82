// nvfp4.cu -- NVFP4 quantization schedules (sm_100a): the single-pass
// kernel for stacks of groups, one thread-block cluster for a small lone
// group, and the two-pass fallback (group_amax_kernel, then
// nvfp4_quant_kernel); the block arithmetic itself is in nvfp4_block.cuh.
#include <atomic>

#include <cooperative_groups.h>

#include "nvfp4_block.cuh"
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

// s2 = RN32(amax / 2688) in place: word g holds the group's amax as bf16
// magnitude bits (group_amax_kernel) and becomes its fp32 global scale.
__global__ void global_scale_kernel(uint32_t *__restrict__ s2_bits, int64_t n_groups)
{
    const int64_t g = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (g < n_groups)
        s2_bits[g] = __float_as_uint(__fdiv_rn(__uint_as_float(s2_bits[g] << 16), kGlobalDivisor));
}

cudaError_t launch_global_scale(const uint16_t *x, int64_t n_groups, int64_t nb, float *s2, uint32_t *status,
                                cudaStream_t s)
{
    uint32_t *bits = reinterpret_cast<uint32_t *>(s2);
    cudaError_t e = cudaMemsetAsync(bits, 0, (size_t)n_groups * sizeof(uint32_t), s);
    if (e == cudaSuccess)
        e = launch_group_amax(x, n_groups, nb, bits, status, s);
    if (e != cudaSuccess)
        return e;
    global_scale_kernel<<<(unsigned)((n_groups + 255) / 256), 256, 0, s>>>(bits, n_groups);
    return cudaGetLastError();
}

// grid = (tiles of 512 blocks, groups).  Thread t of a tile handles blocks
// t and t + 256, so each warp covers 32 consecutive blocks per step and its
// M bits form one 32-bit word.  The group's global scale is either formed
// from its amax (amax_bits, from group_amax_kernel; written to s2_out) or,
// with S2IN, given by the caller (s2_in): then a scale that is negative or
// not finite sets MXQ_DEV_INVALID_SCALE, and a non-finite element, found
// through its block amax, sets MXQ_DEV_NONFINITE_INPUT.
// Four CTAs per SM (64 registers, a few values spilled): 6 % faster on the
// full-size gate_up stack with given scales than two CTAs at 96 registers.
template <bool FOUR_SIX, bool S2IN>
__global__ void __launch_bounds__(kNvThreads, 4)
nvfp4_quant_kernel(const uint4 *__restrict__ x, int64_t n_groups, int64_t nb,
                   const uint32_t *__restrict__ amax_bits, const float *__restrict__ s2_in,
                   uint2 *__restrict__ codes,
                   uint8_t *__restrict__ scales, const ScaleLayout sl, float *__restrict__ s2_out,
                   uint32_t *__restrict__ mbits, int mbits_atomic, uint32_t *__restrict__ m4_count,
                   uint32_t *__restrict__ status)
{
    __shared__ GroupConst s_gc;
    __shared__ uint32_t s_m4;
    const int lane = threadIdx.x & 31;
    for (int64_t g = blockIdx.y; g < n_groups; g += gridDim.y) {
        if (threadIdx.x == 0) {
            if (S2IN) {
                const float v = s2_in[g];
                const bool valid = v >= 0.0f && v <= 0x1.fffffep127f;   // false for NaN
                s_gc = make_group_const_from_s2(valid ? v : 0.0f);
                if (!valid && blockIdx.x == 0)
                    atomicOr(status, MXQ_DEV_INVALID_SCALE);
            } else {
                s_gc = make_group_const(amax_bits[g]);
                if (blockIdx.x == 0)
                    s2_out[g] = s_gc.s2;
            }
            s_m4 = 0;
        }
        __syncthreads();
        const GroupConst gc = s_gc;
        uint32_t my_m4 = 0;
        // Tiles in reverse order: pass 1 read the group front to back, so
        // its last part is the part still in L2 (a group larger than L2, an
        // activation tile of many tokens, then reads that part from L2).
        const int64_t ntiles = (nb + kNvTileBlocks - 1) / kNvTileBlocks;
        for (int64_t t = blockIdx.x; t < ntiles; t += gridDim.x) {
            const int64_t tile = ntiles - 1 - t;
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
                    if (S2IN && !(o.amax <= 0x1.fep127f))       // Inf or NaN element
                        atomicOr(status, MXQ_DEV_NONFINITE_INPUT);
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
//   quantize copy  (ring of `qstages`), issued only after a publisher warp
//                  has seen every CTA's slot for the group and released it
//                  (group constants set), `distance` groups behind the
//                  scouts, so it normally hits the L2 copy the scout read
//                  left behind: 20 compute warps quantize it as soon as it
//                  lands, one barrier per hand-over.  The publisher polls
//                  only the one arrival word of a group; it reads the slots
//                  (and checks their tags) once the count is complete, so
//                  the polling of every CTA stays off the slots' L2 lines.
// The grid-wide amax of a group is therefore resolved while the compute
// warps work on earlier groups; its latency is off the critical path.
// Roles hand over through mbarriers (sfull / sfreed: scout ring, qfull /
// qfreed: quantize ring, ready: group released, which the loader waits for)
// and one shared counter (groups scouted).  Every wait is bounded: on time-out the CTA sets
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
        // a group's quantize copy is issued once the publisher has released
        // the group (its constants are set), so a compute warp that sees the
        // copy land may use the group at once: one barrier per hand-over.
        if (lane != 0 || bytes == 0)
            return;
        // Stages and phase parities advance incrementally (no division).
        int s_next = 0, q_next = 0, s_st = 0, q_st = 0, q_rs = 0;
        uint32_t s_par = 0, q_par = 0, q_rpar = 0;      // parity of (next / ring size)
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
            if (q_next < *scouted && mbar_test_wait(ready + q_rs, q_rpar)) {
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
                    if (++q_rs == kReadyRing) {
                        q_rs = 0;
                        q_rpar ^= 1u;
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
    uint32_t qpar = 0;                                  // the stage's phase parity
    for (int j = 0; j < G; ++j) {
        // the stage's copy is issued only after the group's release, so its
        // completion also orders the publisher's constants before their use
        const bool ok = wait_phase(qfull + st, qpar, abort_flag, 200u);
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
        if (++rs == kReadyRing)
            rs = 0;
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

cudaError_t launch_nvfp4_quant(const uint16_t *x, int64_t n_groups, int64_t nb, int four_six,
                               const uint32_t *amax_bits, const float *s2_in, uint8_t *codes,
                               uint8_t *scales, const ScaleLayout &sl, float *s2, uint32_t *mbits,
                               int mbits_atomic, uint32_t *m4_count, uint32_t *status, cudaStream_t s)
{
    if (n_groups == 0)
        return cudaSuccess;
    const int64_t tiles = nb > 0 ? (nb + kNvTileBlocks - 1) / kNvTileBlocks : 1;
    dim3 grid((unsigned)(tiles < 0x7FFFFFFF ? tiles : 0x7FFFFFFF),
              (unsigned)(n_groups < 65535 ? n_groups : 65535));
    const uint4 *xv = reinterpret_cast<const uint4 *>(x);
    uint2 *cv = reinterpret_cast<uint2 *>(codes);
#define MXQ_QUANT(F, S)                                                                                  \
    nvfp4_quant_kernel<F, S><<<grid, kNvThreads, 0, s>>>(xv, n_groups, nb, amax_bits, s2_in, cv, scales, sl, \
                                                         s2, mbits, mbits_atomic, m4_count, status)
    if (s2_in) {
        if (four_six) MXQ_QUANT(true, true); else MXQ_QUANT(false, true);
    } else {
        if (four_six) MXQ_QUANT(true, false); else MXQ_QUANT(false, false);
    }
#undef MXQ_QUANT
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

// ---------------------------------------------------------------------------
// One group too large for a cluster whose blocks still fit the SMs' shared
// memory (an activation tile of about 800 to 8000 tokens of 2048 values):
// a cooperative grid of one CTA per SM (all resident at once).  Each CTA
// brings its share into shared memory with bulk copies issued together (the
// whole share in flight), reduces its amax piece by piece as the pieces
// land, publishes it as a tagged 64-bit slot (tag and value in one store)
// and counts its arrival; once every CTA has arrived and every slot shows
// its tag (bounded waits), each CTA takes the group amax from the slots and
// quantizes its share from shared memory.  One HBM read of the group, one
// launch.  Shares are multiples of 32 blocks, so each warp's M bits fill one
// word.  On a time-out the CTA sets MXQ_DEV_WAIT_TIMEOUT and returns.
// ---------------------------------------------------------------------------
constexpr int kGridThreads = 512;
constexpr int kGridPieces = 4;

template <bool FOUR_SIX, bool SWZ>
__global__ void __launch_bounds__(kGridThreads, 1)
nvfp4_grid_kernel(const uint4 *__restrict__ x, int64_t nb, int64_t share, uint2 *__restrict__ codes,
                  uint8_t *__restrict__ scales, const ScaleLayout sl, float *__restrict__ s2_out,
                  uint32_t *__restrict__ mbits, uint32_t *__restrict__ m4_count, uint32_t *__restrict__ status,
                  uint32_t *arrived, unsigned long long *slots, int test_stall)
{
    extern __shared__ __align__(128) uint8_t gsmem[];
    uint64_t *bar = reinterpret_cast<uint64_t *>(gsmem);            // kGridPieces barriers
    uint4 *tile = reinterpret_cast<uint4 *>(gsmem + 128);           // 2 vectors per block of the share
    __shared__ uint32_t s_warp[kGridThreads / 32];
    __shared__ GroupConst s_gc;
    __shared__ uint32_t s_m4;
    __shared__ int s_arrived;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const uint32_t P = gridDim.x;
    const int64_t b0 = min(nb, (int64_t)blockIdx.x * share);
    const int n = (int)(min(nb, b0 + share) - b0);
    const int piece = ((n + kGridPieces - 1) / kGridPieces + 31) / 32 * 32;   // blocks, a multiple of 32

    if (threadIdx.x == 0) {
        for (int k = 0; k < kGridPieces; ++k)
            mbar_init(bar + k, 1);
        s_m4 = 0;
        fence_mbar_init();
        for (int k = 0; k < kGridPieces; ++k) {
            const int lo = k * piece, cnt = min(n, lo + piece) - lo;
            if (cnt > 0) {
                mbar_arrive_expect_tx(bar + k, (uint32_t)cnt * 32u);
                bulk_g2s(reinterpret_cast<uint8_t *>(tile) + (size_t)lo * 32, x + 2 * (b0 + lo),
                         (uint32_t)cnt * 32u, bar + k);
            }
        }
    }
    __syncthreads();                                    // barriers initialised before anyone waits
    // the CTA's amax, each piece as it lands
    uint32_t m = 0;
    bool landed = true;
    for (int k = 0; k < kGridPieces && landed; ++k) {
        const int lo = k * piece, cnt = min(n, lo + piece) - lo;
        if (cnt <= 0)
            break;
        landed = false;
        for (uint32_t i = 0; i < kSpinLimit && !landed; ++i)
            landed = mbar_try_wait(bar + k, 0u);
        if (landed)
            for (int i = 2 * lo + (int)threadIdx.x; i < 2 * (lo + cnt); i += kGridThreads) {
                const uint4 v = tile[i];
                m = absmax_bf16x2(absmax_bf16x2(m, v.x), absmax_bf16x2(v.y, v.z));
                m = absmax_bf16x2(m, v.w);
            }
    }
    m = __reduce_max_sync(0xFFFFFFFFu, fold_halves(m));
    if (lane == 0)
        s_warp[warp] = m;
    if (!__syncthreads_and(landed ? 1 : 0)) {
        if (threadIdx.x == 0) {
            atomicOr(status, MXQ_DEV_WAIT_TIMEOUT);
            // let the copies still in flight land (bounded) before the CTA's
            // shared memory is released
            for (int k = 0; k < kGridPieces; ++k)
                if (min(n, k * piece + piece) - k * piece > 0)
                    for (uint32_t i = 0; i < kSpinLimit; ++i)
                        if (mbar_try_wait(bar + k, 0u))
                            break;
        }
        return;                                         // the other CTAs time out at the barrier below
    }
    if (threadIdx.x == 0) {
        uint32_t a = 0;
        for (int w = 0; w < kGridThreads / 32; ++w)
            a = max(a, s_warp[w]);
        if (!test_stall || blockIdx.x != 0) {             // test hook: CTA 0 never arrives
            st_relaxed_u64(slots + blockIdx.x, (1ull << 32) | a);
            red_relaxed_add_u32(arrived, 1u);
        }
        // all CTAs are resident (cooperative launch) and arrive within
        // microseconds; the limit is tens of milliseconds
        bool all = false;
        for (uint32_t i = 0; i < (kSpinLimit >> 4) && !all; ++i) {
            all = ld_relaxed_u32(arrived) >= P;
            if (!all)
                __nanosleep(64);
        }
        s_arrived = all ? 1 : 0;
    }
    __syncthreads();
    // every slot, one per thread (a slot whose store is not visible yet still
    // reads tag 0: poll it again, bounded)
    bool seen = s_arrived != 0;
    uint32_t g = 0;
    if (seen && threadIdx.x < P) {
        unsigned long long v = ld_relaxed_u64(slots + threadIdx.x);
        for (uint32_t i = 0; i < (kSpinLimit >> 4) && (v >> 32) != 1ull; ++i) {
            __nanosleep(64);
            v = ld_relaxed_u64(slots + threadIdx.x);
        }
        seen = (v >> 32) == 1ull;
        g = (uint32_t)v;
    }
    g = __reduce_max_sync(0xFFFFFFFFu, g);
    __syncthreads();                                    // s_warp is reused
    if (lane == 0)
        s_warp[warp] = g;
    if (!__syncthreads_and(seen ? 1 : 0)) {
        if (threadIdx.x == 0)
            atomicOr(status, MXQ_DEV_WAIT_TIMEOUT);
        return;
    }
    if (threadIdx.x == 0) {
        uint32_t a = 0;
        for (int w = 0; w < kGridThreads / 32; ++w)
            a = max(a, s_warp[w]);
        s_gc = make_group_const(a);
        if (blockIdx.x == 0) {
            s2_out[0] = s_gc.s2;
            if (a >= 0x7F80u)
                atomicOr(status, MXQ_DEV_NONFINITE_INPUT);
        }
    }
    __syncthreads();
    const GroupConst gc = s_gc;
    uint32_t my_m4 = 0;
    for (int base = 0; base < n; base += kGridThreads) {
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

cudaError_t launch_nvfp4_grid(const uint16_t *x, int64_t nb, int four_six, uint8_t *codes, uint8_t *scales,
                              const ScaleLayout &sl, float *s2, uint32_t *mbits, uint32_t *m4_count,
                              uint32_t *status, uint32_t *arrived, unsigned long long *slots, cudaStream_t s)
{
    if (nb <= 0 || !arrived || !slots)
        return cudaErrorNotSupported;
    int dev = 0, coop = 0, max_optin = 0;
    if (cudaGetDevice(&dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&coop, cudaDevAttrCooperativeLaunch, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&max_optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev) != cudaSuccess)
        return cudaErrorNotSupported;
    const int sms = sm_count();
    if (!coop || sms <= 0 || sms > kMaxFusedCtas)
        return cudaErrorNotSupported;
    int64_t share = (nb + sms - 1) / sms;
    share = (share + 31) / 32 * 32;
    const int P = (int)((nb + share - 1) / share);
    const size_t dyn = 128 + (size_t)share * 32;
    if (dyn + 2048 > (size_t)max_optin)                 // + static shared memory
        return cudaErrorNotSupported;
    const void *fn = four_six ? (sl.swz ? (const void *)nvfp4_grid_kernel<true, true>
                                        : (const void *)nvfp4_grid_kernel<true, false>)
                              : (sl.swz ? (const void *)nvfp4_grid_kernel<false, true>
                                        : (const void *)nvfp4_grid_kernel<false, false>);
    cudaError_t e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)dyn);
    if (e != cudaSuccess) {
        (void)cudaGetLastError();
        return cudaErrorNotSupported;
    }
    int per_sm = 0;
    e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, fn, kGridThreads, dyn);
    if (e != cudaSuccess || per_sm < 1) {
        (void)cudaGetLastError();
        return cudaErrorNotSupported;
    }
    const uint4 *xv = reinterpret_cast<const uint4 *>(x);
    uint2 *cv = reinterpret_cast<uint2 *>(codes);
    int test_stall = g_test_stall.exchange(0) ? 1 : 0;
    void *params[] = {(void *)&xv, (void *)&nb, (void *)&share, (void *)&cv, (void *)&scales,
                      (void *)&sl, (void *)&s2, (void *)&mbits, (void *)&m4_count, (void *)&status,
                      (void *)&arrived, (void *)&slots, (void *)&test_stall};
    return cudaLaunchCooperativeKernel(fn, dim3((unsigned)P), dim3(kGridThreads), params, dyn, s);
}

} // namespace mxq

extern "C" MXQ_API void mxq_test_stall_next_single_pass(int on)
{
    mxq::g_test_stall.store(on ? 1 : 0);
}
