// mxq_internal.h -- launch interface between the C-ABI layer (api.cu) and
// the kernel translation units.  Not part of the public ABI.
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "mxq_device.cuh"
#include "mxq.h"

namespace mxq {

constexpr float kGlobalDivisor = 2688.0f;  // 6 * 448: weight_scale_2 / input_scale

// NVFP4 streaming kernels: CTA tile of 512 blocks of 16 (256 threads x 2).
constexpr int kNvThreads = 256;
constexpr int kNvTileBlocks = 512;

// Single-pass NVFP4 schedule: one cooperative CTA per SM.
// 20 compute warps, a publisher warp, a loader warp and two scout warps.
// Warps map to the SM's four sub-partitions by warp index mod 4: warps 0-3
// (the four other roles) take one slot of each, and 20 compute warps give
// every sub-partition the same five, so no sub-partition holds more of the
// statically dealt chunks than the others (21 compute warps left one
// sub-partition with six and made it the slowest; measured 1.67 against
// 1.54 ms for the full-size gate_up stack).
constexpr int kFusedComputeWarps = 20;
constexpr int kFusedScoutWarps = 2;
constexpr int kFusedThreads = 32 * (kFusedComputeWarps + 2 + kFusedScoutWarps);

// Verifier: one CTA reduces one chunk of a tensor.
constexpr int kVerifyThreads = 256;
constexpr int64_t kVerifyChunk = 16384;  // elements per chunk (multiple of 32)

size_t align_up(size_t v, size_t a);

// Where block scales go (mxq_layout).  Linear: the scale of block b of a
// matrix is byte b of it.  Tiled: byte swz128x4(b / cb, b % cb, ntc) of the
// matrix, each matrix msz bytes.
struct ScaleLayout {
    int swz;          // 0 linear, 1 tiled 128 x 4
    uint32_t cb;      // blocks per row (cols / block size)
    uint32_t ntc;     // column tiles per matrix, ceil(cb / 4)
    uint64_t msz;     // bytes of one tiled matrix
    FastDiv cbdiv;    // division by cb
};

inline ScaleLayout make_scale_layout(int swz, int64_t rows_per_matrix, int64_t cb)
{
    ScaleLayout l;
    l.swz = swz;
    l.cb = (uint32_t)cb;
    l.ntc = (uint32_t)((cb + 3) / 4);
    l.msz = swz128x4_bytes((uint64_t)rows_per_matrix, (uint64_t)cb);
    l.cbdiv = make_fastdiv(cb > 0 ? (uint32_t)cb : 1u);
    return l;
}

// Byte offset of the scale of block bg (row-major block index inside its
// matrix) of matrix m.
__device__ __forceinline__ uint64_t tiled_scale_offset(const ScaleLayout &l, uint64_t m, uint32_t bg)
{
    const uint32_t r = fastdiv(bg, l.cbdiv), c = bg - r * l.cb;
    return m * l.msz + swz128x4(r, c, l.ntc);
}

// Largest grid of the single-pass NVFP4 schedule (one CTA per SM).
constexpr int kMaxFusedCtas = 256;

// Workspace of the NVFP4 quantizer: one word per group (the amax bits of the
// two-pass schedule, or the arrival count of the single-pass schedule) and
// per-group, per-CTA amax slots (single-pass schedule), each region padded
// to 256 bytes.
size_t nvfp4_workspace_bytes(int64_t n_groups);
size_t nvfp4_slots_offset(int64_t n_groups);

cudaError_t launch_group_amax(const uint16_t *x, int64_t n_groups, int64_t nb,
                              uint32_t *amax_bits, uint32_t *status, cudaStream_t s);
// s2 = RN32(amax_g / 2688) per group, written to s2 (which holds the running
// amax bits in between).
cudaError_t launch_global_scale(const uint16_t *x, int64_t n_groups, int64_t nb, float *s2, uint32_t *status,
                                cudaStream_t s);
// Block quantizer of the two-pass schedule; the group scale comes from
// amax_bits (s2_in NULL; s2 written) or from the caller's s2_in.
cudaError_t launch_nvfp4_quant(const uint16_t *x, int64_t n_groups, int64_t nb, int four_six,
                               const uint32_t *amax_bits, const float *s2_in, uint8_t *codes,
                               uint8_t *scales, const ScaleLayout &sl, float *s2, uint32_t *mbits,
                               int mbits_atomic, uint32_t *m4_count, uint32_t *status, cudaStream_t s);
cudaError_t launch_nvfp4_fused(const uint16_t *x, int64_t n_groups, int64_t nb, int four_six,
                               unsigned long long *slots, uint32_t *arrived, uint8_t *codes, uint8_t *scales,
                               const ScaleLayout &sl,
                               float *s2, uint32_t *mbits, uint32_t *m4_count, uint32_t *status,
                               cudaStream_t s);
// One group of at most kSmallMaxBlocks blocks by one thread-block cluster
// (cudaErrorNotSupported where the device or the size does not allow it).
constexpr int64_t kSmallMaxBlocks = 96 * 1024;    // 3 MiB of bf16
cudaError_t launch_nvfp4_small(const uint16_t *x, int64_t nb, int four_six, uint8_t *codes, uint8_t *scales,
                               const ScaleLayout &sl, float *s2, uint32_t *mbits, uint32_t *m4_count,
                               uint32_t *status, cudaStream_t s);
// One group too large for a cluster whose blocks still fit the SMs' shared
// memory (an activation tile of up to several thousand tokens): a
// cooperative grid of one CTA per SM, one HBM read of the group
// (cudaErrorNotSupported where the device or the size does not allow it).
// `arrived` and `slots` (kMaxFusedCtas words) must start at zero.
cudaError_t launch_nvfp4_grid(const uint16_t *x, int64_t nb, int four_six, uint8_t *codes, uint8_t *scales,
                              const ScaleLayout &sl, float *s2, uint32_t *mbits, uint32_t *m4_count,
                              uint32_t *status, uint32_t *arrived, unsigned long long *slots, cudaStream_t s);
cudaError_t launch_nvfp4_weighted(const uint16_t *x, int64_t n_groups, int64_t nb, int64_t cols,
                                  const uint32_t *amax_bits, const float *h, int64_t h_stride,
                                  uint8_t *codes, uint8_t *scales, const ScaleLayout &sl, float *s2,
                                  uint32_t *status, cudaStream_t s);
cudaError_t launch_mx_quant(const uint16_t *x, int64_t nblk32, int fmt, uint8_t *codes,
                            uint8_t *scales, const ScaleLayout &sl, uint32_t *status, cudaStream_t s);
cudaError_t launch_requant_fp8_mx(const uint8_t *fp8, const float *bscale, int64_t rows, int64_t cols,
                                  int64_t brows, int64_t bcols, int fmt, uint8_t *codes,
                                  uint8_t *scales, const ScaleLayout &sl, uint32_t *status,
                                  cudaStream_t s);
cudaError_t launch_census_add(mxq_census *c, int64_t n_tensors, const double *err, const double *ref,
                              const double *rel, const double *err_rtn, int64_t n_groups, const uint32_t *m4,
                              int64_t blocks_per_group, cudaStream_t s);
cudaError_t launch_verify(const uint16_t *x, const uint8_t *codes, const uint8_t *scales,
                          const float *s2, int fmt, const ScaleLayout &sl, int64_t n_tensors,
                          int64_t rows, int64_t tsize, int64_t tensors_per_scale, double *partials, double *sum_sq_err,
                          double *sum_sq_ref, double *relerr, cudaStream_t s);

} // namespace mxq
