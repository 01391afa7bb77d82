// api.cu -- the C ABI declared in include/mxq.h: argument checks,
// workspace carving and kernel launches.  No allocation, no host-device
// synchronisation; no state (the no-alloc verifier keeps its own, in noalloc.cu).
#include "mxq.h"
#include "mxq_internal.h"

#include <limits.h>
#include <nvtx3/nvToolsExt.h>

namespace mxq {

size_t align_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

size_t nvfp4_slots_offset(int64_t n_groups)
{
    return align_up((size_t)n_groups * sizeof(uint32_t), 256);
}

size_t nvfp4_workspace_bytes(int64_t n_groups)
{
    return nvfp4_slots_offset(n_groups) +
           align_up((size_t)n_groups * kMaxFusedCtas * sizeof(unsigned long long), 256);
}

static size_t verify_workspace_bytes(int64_t n_tensors, int64_t rows, int64_t cols)
{
    const int64_t tsize = rows * cols;
    const int64_t cpt = tsize > 0 ? (tsize + kVerifyChunk - 1) / kVerifyChunk : 1;
    return align_up((size_t)(n_tensors * cpt) * 2 * sizeof(double), 256);
}

static bool aligned(const void *p, size_t a) { return ((uintptr_t)p % a) == 0; }

static bool layout_ok(mxq_layout l) { return l == MXQ_LAYOUT_LINEAR || l == MXQ_LAYOUT_SWIZZLED_128X4; }

// Tiled scales of `n` matrices of rows x cb scales: zero the whole buffer
// first when a matrix has padding (rows % 128 or cb % 4), so that the
// padding bytes are 0; the kernels write every real scale.
static cudaError_t zero_tiled_padding(uint8_t *scales, int64_t n, int64_t rows, int64_t cb,
                                      cudaStream_t stream)
{
    if (rows % 128 == 0 && cb % 4 == 0)
        return cudaSuccess;
    return cudaMemsetAsync(scales, 0, (size_t)n * swz128x4_bytes((uint64_t)rows, (uint64_t)cb), stream);
}

// rows * cols * n without overflow, all non-negative.
static bool mul_ok(int64_t a, int64_t b, int64_t *out)
{
    if (a < 0 || b < 0)
        return false;
    if (a != 0 && b > INT64_MAX / a)
        return false;
    *out = a * b;
    return true;
}

// NVTX range around one API call (visible in Nsight timelines; a no-op
// without a tool attached).
struct ApiRange {
    explicit ApiRange(const char *name) { nvtxRangePushA(name); }
    ~ApiRange() { nvtxRangePop(); }
    ApiRange(const ApiRange &) = delete;
    ApiRange &operator=(const ApiRange &) = delete;
};

} // namespace mxq

using namespace mxq;

extern "C" {

int mxq_version(void) { return 10200; }

const char *mxq_status_string(mxq_status s)
{
    switch (s) {
    case MXQ_OK: return "ok";
    case MXQ_ERR_INVALID_ARG: return "invalid argument";
    case MXQ_ERR_SHAPE: return "unsupported shape (cols must be a multiple of the block size)";
    case MXQ_ERR_ALIGN: return "misaligned pointer";
    case MXQ_ERR_WORKSPACE: return "workspace missing or too small";
    case MXQ_ERR_CUDA: return "CUDA runtime error";
    case MXQ_ERR_UNSUPPORTED: return "unsupported request";
    }
    return "unknown status";
}

size_t mxq_scale_bytes(mxq_fmt fmt, mxq_layout layout, int64_t n_matrices, int64_t rows,
                       int64_t cols)
{
    int64_t tmp;
    if (n_matrices < 0 || rows < 0 || cols < 0 || !layout_ok(layout))
        return 0;
    const int64_t blk = fmt == MXQ_FMT_NVFP4 ? 16 : (fmt == MXQ_FMT_MXFP4 || fmt == MXQ_FMT_MXFP8 ? 32 : 0);
    if (blk == 0 || cols % blk != 0 || !mul_ok(rows, cols, &tmp) || !mul_ok(tmp, n_matrices, &tmp))
        return 0;
    const int64_t cb = cols / blk;
    if (layout == MXQ_LAYOUT_LINEAR)
        return (size_t)(n_matrices * rows * cb);
    return (size_t)n_matrices * (size_t)swz128x4_bytes((uint64_t)rows, (uint64_t)cb);
}

size_t mxq_workspace_bytes(mxq_op op, int64_t n, int64_t rows, int64_t cols)
{
    int64_t tmp;
    if (n < 0 || rows < 0 || (op != MXQ_OP_QUANTIZE_ACT && cols < 0))
        return 0;
    switch (op) {
    case MXQ_OP_QUANTIZE_NVFP4:
        if (!mul_ok(rows, cols, &tmp) || !mul_ok(tmp, n, &tmp))
            return 0;
        return nvfp4_workspace_bytes(n);
    case MXQ_OP_QUANTIZE_ACT:
        if (!mul_ok(n, rows, &tmp))
            return 0;
        return nvfp4_workspace_bytes(1);
    case MXQ_OP_DEQUANT_RELERR:
        if (!mul_ok(rows, cols, &tmp) || !mul_ok(tmp, n, &tmp))
            return 0;
        return verify_workspace_bytes(n, rows, cols);
    }
    return 0;
}

// Groups with no elements: their amax is 0, so s2 = RN32(0 / 2688) = 0 and
// no block exists; x, codes, scales and the workspace are not needed.
static mxq_status empty_groups(int64_t n_groups, float *s2, uint32_t *m4_count, uint32_t *status,
                               cudaStream_t stream)
{
    if (!s2 || !status)
        return MXQ_ERR_INVALID_ARG;
    if (!aligned(s2, 4) || !aligned(status, 4) || (m4_count && !aligned(m4_count, 4)))
        return MXQ_ERR_ALIGN;
    cudaError_t e = cudaMemsetAsync(s2, 0, (size_t)n_groups * sizeof(float), stream);
    if (e == cudaSuccess && m4_count)
        e = cudaMemsetAsync(m4_count, 0, (size_t)n_groups * sizeof(uint32_t), stream);
    return e == cudaSuccess ? MXQ_OK : MXQ_ERR_CUDA;
}

mxq_status mxq_quantize_nvfp4(const uint16_t *x, int64_t n_groups, int64_t rows, int64_t cols,
                              mxq_scale_mode mode, mxq_layout layout, uint8_t *codes,
                              uint8_t *scales, float *s2,
                              uint32_t *mbits, uint32_t *m4_count, uint32_t *status,
                              void *workspace, size_t workspace_bytes, cudaStream_t stream)
{
    const ApiRange range_("mxq_quantize_nvfp4");
    if (n_groups < 0 || rows < 0 || cols < 0)
        return MXQ_ERR_INVALID_ARG;
    if (mode != MXQ_SCALE_RTN && mode != MXQ_SCALE_FOUR_SIX)
        return MXQ_ERR_INVALID_ARG;
    if (!layout_ok(layout))
        return MXQ_ERR_INVALID_ARG;
    if (cols % 16 != 0)
        return MXQ_ERR_SHAPE;
    int64_t gsize, total;
    if (!mul_ok(rows, cols, &gsize) || !mul_ok(gsize, n_groups, &total) || total > (INT64_MAX / 4))
        return MXQ_ERR_SHAPE;
    const bool swz = layout == MXQ_LAYOUT_SWIZZLED_128X4;
    if (swz && gsize / 16 > 0x7FFFFFFF)
        return MXQ_ERR_SHAPE;   // tiled offsets index the blocks of a group in 32 bits
    if (n_groups == 0)
        return MXQ_OK;
    if (total == 0)   // groups without elements: amax 0, so s2 = 0 and M=4 count 0
        return empty_groups(n_groups, s2, m4_count, status, stream);
    if (!x || !codes || !scales || !s2 || !status)
        return MXQ_ERR_INVALID_ARG;
    if (!aligned(x, 16) || !aligned(codes, 16) || !aligned(scales, 16) || !aligned(s2, 4) ||
        !aligned(status, 4) || (mbits && !aligned(mbits, 4)) || (m4_count && !aligned(m4_count, 4)))
        return MXQ_ERR_ALIGN;
    const size_t need = nvfp4_workspace_bytes(n_groups);
    if (!workspace || workspace_bytes < need)
        return MXQ_ERR_WORKSPACE;
    if (!aligned(workspace, 256))
        return MXQ_ERR_ALIGN;
    const int64_t nb = gsize / 16;
    const int64_t total_blocks = total / 16;
    const ScaleLayout sl = make_scale_layout(swz ? 1 : 0, rows, cols / 16);
    uint32_t *amax_bits = static_cast<uint32_t *>(workspace);
    unsigned long long *slots = reinterpret_cast<unsigned long long *>(
        static_cast<uint8_t *>(workspace) + nvfp4_slots_offset(n_groups));
    cudaError_t e = cudaSuccess;
    // one small group (an activation tile): one thread-block cluster, no
    // workspace traffic
    if (n_groups == 1 && nb <= kSmallMaxBlocks) {
        if (swz)
            e = zero_tiled_padding(scales, n_groups, rows, cols / 16, stream);
        if (e == cudaSuccess && m4_count)
            e = cudaMemsetAsync(m4_count, 0, sizeof(uint32_t), stream);
        if (e != cudaSuccess)
            return MXQ_ERR_CUDA;
        e = launch_nvfp4_small(x, nb, mode == MXQ_SCALE_FOUR_SIX, codes, scales, sl, s2, mbits, m4_count,
                               status, stream);
        if (e == cudaSuccess)
            return MXQ_OK;
        if (e != cudaErrorNotSupported)
            return MXQ_ERR_CUDA;
        (void)cudaGetLastError();
    }
    // amax bits / arrival counts and amax slots start at zero (a slot's tag
    // is its group + 1)
    e = cudaMemsetAsync(workspace, 0, need, stream);
    if (e == cudaSuccess && swz)
        e = zero_tiled_padding(scales, n_groups, rows, cols / 16, stream);
    if (e == cudaSuccess && m4_count)
        e = cudaMemsetAsync(m4_count, 0, (size_t)n_groups * sizeof(uint32_t), stream);
    if (e != cudaSuccess)
        return MXQ_ERR_CUDA;
    // single pass (one HBM read of x) when the shape allows it: several
    // groups overlap each group's grid-wide amax with the quantization of
    // earlier ones; a lone group whose blocks fit the SMs' shared memory is
    // read once into it by one grid
    if (n_groups > 1)
        e = launch_nvfp4_fused(x, n_groups, nb, mode == MXQ_SCALE_FOUR_SIX, slots, amax_bits, codes, scales, sl,
                               s2, mbits, m4_count, status, stream);
    else    // one group that fits the SMs' shared memory: one grid, one read
        e = launch_nvfp4_grid(x, nb, mode == MXQ_SCALE_FOUR_SIX, codes, scales, sl, s2, mbits, m4_count, status,
                              amax_bits, slots, stream);
    // a context that may use fewer SMs than the device has (a shared or
    // partitioned GPU) cannot hold the one-CTA-per-SM grid: two passes instead
    if (e == cudaErrorCooperativeLaunchTooLarge)
        e = cudaErrorNotSupported;
    if (e == cudaSuccess)
        return MXQ_OK;
    if (e != cudaErrorNotSupported)
        return MXQ_ERR_CUDA;
    (void)cudaGetLastError();
    // two passes: group amax, then the block quantizer
    const int mbits_atomic = (nb % 32) != 0;
    if (mbits && mbits_atomic)
        e = cudaMemsetAsync(mbits, 0, (size_t)((total_blocks + 31) / 32) * sizeof(uint32_t), stream);
    else
        e = cudaSuccess;
    if (e == cudaSuccess)
        e = launch_group_amax(x, n_groups, nb, amax_bits, status, stream);
    if (e == cudaSuccess)
        e = launch_nvfp4_quant(x, n_groups, nb, mode == MXQ_SCALE_FOUR_SIX, amax_bits, nullptr, codes, scales,
                               sl, s2, mbits, mbits_atomic, mode == MXQ_SCALE_FOUR_SIX ? m4_count : nullptr,
                               status, stream);
    return e == cudaSuccess ? MXQ_OK : MXQ_ERR_CUDA;
}

mxq_status mxq_global_scale_nvfp4(const uint16_t *x, int64_t n_groups, int64_t rows, int64_t cols, float *s2,
                                  uint32_t *status, cudaStream_t stream)
{
    const ApiRange range_("mxq_global_scale_nvfp4");
    if (n_groups < 0 || rows < 0 || cols < 0)
        return MXQ_ERR_INVALID_ARG;
    if (cols % 16 != 0)
        return MXQ_ERR_SHAPE;
    int64_t gsize, total;
    if (!mul_ok(rows, cols, &gsize) || !mul_ok(gsize, n_groups, &total) || total > (INT64_MAX / 4))
        return MXQ_ERR_SHAPE;
    if (n_groups == 0)
        return MXQ_OK;
    if (total == 0)
        return empty_groups(n_groups, s2, nullptr, status, stream);
    if (!x || !s2 || !status)
        return MXQ_ERR_INVALID_ARG;
    if (!aligned(x, 16) || !aligned(s2, 4) || !aligned(status, 4))
        return MXQ_ERR_ALIGN;
    return launch_global_scale(x, n_groups, gsize / 16, s2, status, stream) == cudaSuccess ? MXQ_OK
                                                                                          : MXQ_ERR_CUDA;
}

mxq_status mxq_quantize_nvfp4_s2(const uint16_t *x, int64_t n_groups, int64_t rows, int64_t cols,
                                 const float *s2_in, mxq_scale_mode mode, mxq_layout layout,
                                 uint8_t *codes, uint8_t *scales, uint32_t *mbits, uint32_t *m4_count,
                                 uint32_t *status, cudaStream_t stream)
{
    const ApiRange range_("mxq_quantize_nvfp4_s2");
    if (n_groups < 0 || rows < 0 || cols < 0)
        return MXQ_ERR_INVALID_ARG;
    if (mode != MXQ_SCALE_RTN && mode != MXQ_SCALE_FOUR_SIX)
        return MXQ_ERR_INVALID_ARG;
    if (!layout_ok(layout))
        return MXQ_ERR_INVALID_ARG;
    if (cols % 16 != 0)
        return MXQ_ERR_SHAPE;
    int64_t gsize, total;
    if (!mul_ok(rows, cols, &gsize) || !mul_ok(gsize, n_groups, &total) || total > (INT64_MAX / 4))
        return MXQ_ERR_SHAPE;
    const bool swz = layout == MXQ_LAYOUT_SWIZZLED_128X4;
    if (swz && gsize / 16 > 0x7FFFFFFF)
        return MXQ_ERR_SHAPE;
    if (n_groups == 0)
        return MXQ_OK;
    // without elements x, codes and scales are not read or written (the
    // kernel still checks the given scales)
    if ((total > 0 && (!x || !codes || !scales)) || !s2_in || !status)
        return MXQ_ERR_INVALID_ARG;
    if (!aligned(x, 16) || !aligned(codes, 16) || !aligned(scales, 16) || !aligned(s2_in, 4) ||
        !aligned(status, 4) || (mbits && !aligned(mbits, 4)) || (m4_count && !aligned(m4_count, 4)))
        return MXQ_ERR_ALIGN;
    const int64_t nb = gsize / 16;
    const int64_t total_blocks = total / 16;
    const ScaleLayout sl = make_scale_layout(swz ? 1 : 0, rows, cols / 16);
    const int mbits_atomic = (nb % 32) != 0;
    cudaError_t e = cudaSuccess;
    if (swz)
        e = zero_tiled_padding(scales, n_groups, rows, cols / 16, stream);
    if (e == cudaSuccess && m4_count)
        e = cudaMemsetAsync(m4_count, 0, (size_t)n_groups * sizeof(uint32_t), stream);
    if (e == cudaSuccess && mbits && mbits_atomic)
        e = cudaMemsetAsync(mbits, 0, (size_t)((total_blocks + 31) / 32) * sizeof(uint32_t), stream);
    if (e == cudaSuccess)
        e = launch_nvfp4_quant(x, n_groups, nb, mode == MXQ_SCALE_FOUR_SIX, nullptr, s2_in, codes, scales, sl,
                               nullptr, mbits, mbits_atomic, mode == MXQ_SCALE_FOUR_SIX ? m4_count : nullptr,
                               status, stream);
    return e == cudaSuccess ? MXQ_OK : MXQ_ERR_CUDA;
}

mxq_status mxq_quantize_nvfp4_weighted(const uint16_t *x, int64_t n_groups, int64_t rows,
                                       int64_t cols, const float *h, int64_t h_groups,
                                       mxq_layout layout, uint8_t *codes, uint8_t *scales, float *s2,
                                       uint32_t *status, void *workspace, size_t workspace_bytes,
                                       cudaStream_t stream)
{
    const ApiRange range_("mxq_quantize_nvfp4_weighted");
    if (n_groups < 0 || rows < 0 || cols < 0)
        return MXQ_ERR_INVALID_ARG;
    if (!layout_ok(layout) || (h_groups != 1 && h_groups != n_groups))
        return MXQ_ERR_INVALID_ARG;
    if (cols % 16 != 0)
        return MXQ_ERR_SHAPE;
    int64_t gsize, total;
    if (!mul_ok(rows, cols, &gsize) || !mul_ok(gsize, n_groups, &total) || total > (INT64_MAX / 4))
        return MXQ_ERR_SHAPE;
    const bool swz = layout == MXQ_LAYOUT_SWIZZLED_128X4;
    if (swz && gsize / 16 > 0x7FFFFFFF)
        return MXQ_ERR_SHAPE;
    if (n_groups == 0)
        return MXQ_OK;
    if (total == 0)
        return empty_groups(n_groups, s2, nullptr, status, stream);
    if (!x || !h || !codes || !scales || !s2 || !status)
        return MXQ_ERR_INVALID_ARG;
    if (!aligned(x, 16) || !aligned(h, 16) || !aligned(codes, 16) || !aligned(scales, 16) ||
        !aligned(s2, 4) || !aligned(status, 4))
        return MXQ_ERR_ALIGN;
    const size_t need = nvfp4_workspace_bytes(n_groups);
    if (!workspace || workspace_bytes < need)
        return MXQ_ERR_WORKSPACE;
    if (!aligned(workspace, 256))
        return MXQ_ERR_ALIGN;
    const int64_t nb = gsize / 16;
    const ScaleLayout sl = make_scale_layout(swz ? 1 : 0, rows, cols / 16);
    uint32_t *amax_bits = static_cast<uint32_t *>(workspace);
    cudaError_t e = cudaMemsetAsync(amax_bits, 0, (size_t)n_groups * sizeof(uint32_t), stream);
    if (e == cudaSuccess && swz)
        e = zero_tiled_padding(scales, n_groups, rows, cols / 16, stream);
    if (e == cudaSuccess)
        e = launch_group_amax(x, n_groups, nb, amax_bits, status, stream);
    if (e == cudaSuccess)
        e = launch_nvfp4_weighted(x, n_groups, nb, cols, amax_bits, h, h_groups == 1 ? 0 : cols, codes,
                                  scales, sl, s2, status, stream);
    return e == cudaSuccess ? MXQ_OK : MXQ_ERR_CUDA;
}

mxq_status mxq_quantize_mx(const uint16_t *x, int64_t rows, int64_t cols, mxq_fmt fmt, int block,
                           mxq_layout layout, uint8_t *codes, uint8_t *scales, uint32_t *status,
                           cudaStream_t stream)
{
    const ApiRange range_("mxq_quantize_mx");
    if (rows < 0 || cols < 0)
        return MXQ_ERR_INVALID_ARG;
    if (fmt != MXQ_FMT_MXFP4 && fmt != MXQ_FMT_MXFP8)
        return MXQ_ERR_INVALID_ARG;
    if (!layout_ok(layout))
        return MXQ_ERR_INVALID_ARG;
    if (block != 32)
        return MXQ_ERR_UNSUPPORTED;
    if (cols % 32 != 0)
        return MXQ_ERR_SHAPE;
    int64_t total;
    if (!mul_ok(rows, cols, &total) || total > (INT64_MAX / 4))
        return MXQ_ERR_SHAPE;
    if (total == 0)
        return MXQ_OK;
    if (!x || !codes || !scales)
        return MXQ_ERR_INVALID_ARG;
    if (!aligned(x, 16) || !aligned(codes, 16) || !aligned(scales, 16) || (status && !aligned(status, 4)))
        return MXQ_ERR_ALIGN;
    const bool swz = layout == MXQ_LAYOUT_SWIZZLED_128X4;
    if (swz && total / 32 > 0x7FFFFFFF)
        return MXQ_ERR_SHAPE;   // tiled offsets index the blocks in 32 bits
    const ScaleLayout sl = make_scale_layout(swz ? 1 : 0, rows, cols / 32);
    cudaError_t e = swz ? zero_tiled_padding(scales, 1, rows, cols / 32, stream) : cudaSuccess;
    if (e == cudaSuccess)
        e = launch_mx_quant(x, total / 32, (int)fmt, codes, scales, sl, status, stream);
    return e == cudaSuccess ? MXQ_OK : MXQ_ERR_CUDA;
}

mxq_status mxq_requant_fp8_mx(const uint8_t *fp8, const float *bscale, int64_t rows, int64_t cols,
                              int64_t brows, int64_t bcols, mxq_fmt fmt, mxq_layout layout,
                              uint8_t *codes, uint8_t *scales, uint32_t *status, cudaStream_t stream)
{
    const ApiRange range_("mxq_requant_fp8_mx");
    if (rows < 0 || cols < 0 || brows < 1 || bcols < 1)
        return MXQ_ERR_INVALID_ARG;
    if (fmt != MXQ_FMT_MXFP4 && fmt != MXQ_FMT_MXFP8)
        return MXQ_ERR_INVALID_ARG;
    if (!layout_ok(layout))
        return MXQ_ERR_INVALID_ARG;
    if (cols % 32 != 0 || bcols % 32 != 0 || brows > 0x7FFFFFFF || bcols > 0x7FFFFFFF)
        return MXQ_ERR_SHAPE;
    int64_t total;
    if (!mul_ok(rows, cols, &total) || total / 32 > 0xFFFFFFFFll)
        return MXQ_ERR_SHAPE;
    if (total == 0)
        return MXQ_OK;
    if (!fp8 || !bscale || !codes || !scales)
        return MXQ_ERR_INVALID_ARG;
    if (!aligned(fp8, 16) || !aligned(bscale, 4) || !aligned(codes, 16) || !aligned(scales, 16) ||
        (status && !aligned(status, 4)))
        return MXQ_ERR_ALIGN;
    const bool swz = layout == MXQ_LAYOUT_SWIZZLED_128X4;
    const ScaleLayout sl = make_scale_layout(swz ? 1 : 0, rows, cols / 32);
    cudaError_t e = swz ? zero_tiled_padding(scales, 1, rows, cols / 32, stream) : cudaSuccess;
    if (e == cudaSuccess)
        e = launch_requant_fp8_mx(fp8, bscale, rows, cols, brows, bcols, (int)fmt, codes, scales, sl,
                                  status, stream);
    return e == cudaSuccess ? MXQ_OK : MXQ_ERR_CUDA;
}

mxq_status mxq_quantize_act(const uint16_t *tokens, int64_t T, int64_t hidden, mxq_fmt fmt,
                            mxq_scale_mode mode, mxq_layout layout, uint8_t *codes,
                            uint8_t *scales, float *input_scale, uint32_t *status,
                            void *workspace, size_t workspace_bytes, cudaStream_t stream)
{
    const ApiRange range_("mxq_quantize_act");
    if (T < 0 || hidden < 0)
        return MXQ_ERR_INVALID_ARG;
    if (mode != MXQ_SCALE_RTN && mode != MXQ_SCALE_FOUR_SIX)
        return MXQ_ERR_INVALID_ARG;
    if (!layout_ok(layout))
        return MXQ_ERR_INVALID_ARG;
    if (!status)
        return MXQ_ERR_INVALID_ARG;
    if (fmt == MXQ_FMT_NVFP4) {
        if (!input_scale)
            return MXQ_ERR_INVALID_ARG;
        if (T == 0 || hidden == 0) {
            if (hidden % 16 != 0)
                return MXQ_ERR_SHAPE;
            return cudaMemsetAsync(input_scale, 0, sizeof(float), stream) == cudaSuccess ? MXQ_OK
                                                                                          : MXQ_ERR_CUDA;
        }
        return mxq_quantize_nvfp4(tokens, 1, T, hidden, mode, layout, codes, scales, input_scale,
                                  nullptr, nullptr, status, workspace, workspace_bytes, stream);
    }
    if (fmt == MXQ_FMT_MXFP4 || fmt == MXQ_FMT_MXFP8) {
        if (mode != MXQ_SCALE_RTN)
            return MXQ_ERR_UNSUPPORTED;
        return mxq_quantize_mx(tokens, T, hidden, fmt, 32, layout, codes, scales, status, stream);
    }
    return MXQ_ERR_INVALID_ARG;
}

mxq_status mxq_dequant_relerr(const uint16_t *x, const uint8_t *codes, const uint8_t *scales,
                              const float *s2, mxq_fmt fmt, mxq_layout layout, int64_t n_tensors,
                              int64_t rows,
                              int64_t cols, int64_t tensors_per_scale, double *sum_sq_err,
                              double *sum_sq_ref, double *relerr, void *workspace,
                              size_t workspace_bytes, cudaStream_t stream)
{
    const ApiRange range_("mxq_dequant_relerr");
    if (n_tensors < 0 || rows < 0 || cols < 0)
        return MXQ_ERR_INVALID_ARG;
    if (fmt != MXQ_FMT_NVFP4 && fmt != MXQ_FMT_MXFP4 && fmt != MXQ_FMT_MXFP8)
        return MXQ_ERR_INVALID_ARG;
    if (!layout_ok(layout))
        return MXQ_ERR_INVALID_ARG;
    const bool swz = layout == MXQ_LAYOUT_SWIZZLED_128X4;
    if ((fmt == MXQ_FMT_NVFP4 || swz) && tensors_per_scale < 1)
        return MXQ_ERR_INVALID_ARG;
    const int blk = (fmt == MXQ_FMT_NVFP4) ? 16 : 32;
    if (cols % blk != 0)
        return MXQ_ERR_SHAPE;
    int64_t tsize, total;
    if (!mul_ok(rows, cols, &tsize) || !mul_ok(tsize, n_tensors, &total) || total > (INT64_MAX / 4))
        return MXQ_ERR_SHAPE;
    int64_t msize = 0;
    if (swz && (!mul_ok(tsize, tensors_per_scale, &msize) || msize / blk > 0x7FFFFFFF))
        return MXQ_ERR_SHAPE;   // tiled offsets index the blocks of a matrix in 32 bits
    const int64_t cpt = tsize > 0 ? (tsize + kVerifyChunk - 1) / kVerifyChunk : 1;
    if (n_tensors > 0x7FFFFFFF / cpt || tensors_per_scale > 0x7FFFFFFF)
        return MXQ_ERR_SHAPE;   // the verifier indexes its chunks in 32 bits
    if (n_tensors == 0)
        return MXQ_OK;
    if (!sum_sq_err || !sum_sq_ref)
        return MXQ_ERR_INVALID_ARG;
    if (total > 0 && (!x || !codes || !scales || (fmt == MXQ_FMT_NVFP4 && !s2)))
        return MXQ_ERR_INVALID_ARG;
    if (!aligned(x, 16) || !aligned(codes, 16) || !aligned(scales, 16) || (s2 && !aligned(s2, 4)) ||
        !aligned(sum_sq_err, 8) || !aligned(sum_sq_ref, 8) || (relerr && !aligned(relerr, 8)))
        return MXQ_ERR_ALIGN;
    if (total == 0) {
        // tensors without elements: both sums 0 and a relative error of 0
        // (the convention for a tensor reproduced exactly); nothing is read
        cudaError_t e = cudaMemsetAsync(sum_sq_err, 0, (size_t)n_tensors * sizeof(double), stream);
        if (e == cudaSuccess)
            e = cudaMemsetAsync(sum_sq_ref, 0, (size_t)n_tensors * sizeof(double), stream);
        if (e == cudaSuccess && relerr)
            e = cudaMemsetAsync(relerr, 0, (size_t)n_tensors * sizeof(double), stream);
        return e == cudaSuccess ? MXQ_OK : MXQ_ERR_CUDA;
    }
    const size_t need = verify_workspace_bytes(n_tensors, rows, cols);
    if (!workspace || workspace_bytes < need)
        return MXQ_ERR_WORKSPACE;
    if (!aligned(workspace, 256))
        return MXQ_ERR_ALIGN;
    const ScaleLayout sl = make_scale_layout(swz ? 1 : 0, rows * (swz ? tensors_per_scale : 1), cols / blk);
    cudaError_t e = launch_verify(x, codes, scales, s2, (int)fmt, sl, n_tensors, rows, tsize,
                                  tensors_per_scale < 1 ? 1 : tensors_per_scale,
                                  static_cast<double *>(workspace), sum_sq_err, sum_sq_ref, relerr, stream);
    return e == cudaSuccess ? MXQ_OK : MXQ_ERR_CUDA;
}

mxq_status mxq_census_reset(mxq_census *census, cudaStream_t stream)
{
    const ApiRange range_("mxq_census_reset");
    if (!census)
        return MXQ_ERR_INVALID_ARG;
    if (!aligned(census, 8))
        return MXQ_ERR_ALIGN;
    return cudaMemsetAsync(census, 0, sizeof(mxq_census), stream) == cudaSuccess ? MXQ_OK : MXQ_ERR_CUDA;
}

mxq_status mxq_census_add(mxq_census *census, int64_t n_tensors, const double *sum_sq_err,
                          const double *sum_sq_ref, const double *relerr, const double *sum_sq_err_rtn,
                          int64_t n_groups, const uint32_t *m4_count, int64_t blocks_per_group,
                          cudaStream_t stream)
{
    const ApiRange range_("mxq_census_add");
    if (!census || n_tensors < 0 || n_groups < 0 || blocks_per_group < 0)
        return MXQ_ERR_INVALID_ARG;
    if (n_tensors > 0 && (!sum_sq_err || !sum_sq_ref || !relerr))
        return MXQ_ERR_INVALID_ARG;
    if (n_groups > 0 && !m4_count)
        return MXQ_ERR_INVALID_ARG;
    int64_t blocks;
    if (!mul_ok(n_groups, blocks_per_group, &blocks))
        return MXQ_ERR_SHAPE;
    if (!aligned(census, 8) || (n_tensors > 0 && (!aligned(sum_sq_err, 8) || !aligned(sum_sq_ref, 8) ||
                                                  !aligned(relerr, 8) ||
                                                  (sum_sq_err_rtn && !aligned(sum_sq_err_rtn, 8)))) ||
        (n_groups > 0 && !aligned(m4_count, 4)))
        return MXQ_ERR_ALIGN;
    if (n_tensors == 0 && n_groups == 0)
        return MXQ_OK;
    const cudaError_t e = launch_census_add(census, n_tensors, sum_sq_err, sum_sq_ref, relerr,
                                            n_tensors > 0 ? sum_sq_err_rtn : nullptr, n_groups, m4_count,
                                            blocks_per_group, stream);
    return e == cudaSuccess ? MXQ_OK : MXQ_ERR_CUDA;
}

} // extern "C"
