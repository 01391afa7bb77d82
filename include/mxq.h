/*
 * mxq.h -- C ABI of the B200 (sm_100a) block-scaled microscaling quantizer.
 *
 * One library, libmxq.so, converts bf16 tensors into three block-scaled
 * formats and verifies the result:
 *   NVFP4  E2M1 values, one E4M3 scale per 16 values, one fp32 global
 *          scale per group (weight_scale_2 / input_scale = amax / 2688);
 *          block scales chosen by plain amax/6 (RTN) or by the 4/6-optimal
 *          rule;
 *   MXFP4  E2M1 values, one UE8M0 power-of-two scale per 32 values;
 *   MXFP8  E4M3 values, one UE8M0 power-of-two scale per 32 values;
 * and measures ||W - deq(Q(W))|| / ||W|| per tensor.
 *
 * Sources (model-card pages, section in quotes):
 *   dabsLabs/Qwen3.8-Flash-Next-NVFP4, "What makes this build different":
 *     4/6-optimal block scales; stacked [512, out, in] experts with fused
 *     gate_up, unstacked per expert; relative-error metrics.
 *   josch15366/Qwen3.8-Flash-Next-NVFP4-LocalHessian-Experts, introduction:
 *     input_scale = amax/2688 (not amax/6); gate and up share one
 *     weight_scale_2; "What is different about it": one weight_scale_2 per
 *     expert.
 *   azampatti/Qwen3.8-Flash-Next-FP4-Local-AZ, "The shared expert":
 *     MXFP8 = e4m3 values, one power-of-two scale per 32 weights,
 *     e = ceil(log2(amax/448)).
 *   MJPansa/Qwen3.8-Flash-Next-MXFP4-FP8-R12, "Quantization format":
 *     MXFP4 E2M1 weights with UE8M0 microscales; activations dynamically
 *     quantized to MXFP8 at run time.
 *
 * Conventions for every entry point
 *   - All pointers are DEVICE pointers unless stated; the caller owns every
 *     buffer.  The library allocates nothing.  State kept between calls:
 *     the device address of the fixed scratch array of
 *     mxq_dequant_relerr_noalloc (per device and context, see there) and the
 *     one-shot request flag of the test hook in mxq_test.h; nothing else.
 *   - All work is enqueued asynchronously on `stream` (0 = legacy default
 *     stream).  The call returns after enqueueing; results are valid once
 *     the stream has reached that point.
 *   - Errors found on the host (bad arguments) are returned before anything
 *     is enqueued, and no output is touched.  MXQ_ERR_CUDA means a CUDA
 *     runtime call failed while enqueueing; outputs are then undefined.
 *   - Conditions found on the device are OR-ed into *status (a uint32 the
 *     caller zeroes and reads after synchronising): MXQ_DEV_NONFINITE_INPUT
 *     when an input element is Inf or NaN (outputs are then undefined),
 *     MXQ_DEV_WAIT_TIMEOUT when a bounded inter-CTA wait gave up (outputs
 *     are then undefined), MXQ_DEV_INVALID_SCALE when a caller-given global
 *     scale is negative or not finite (that group's outputs are undefined).  `status` may be NULL on the MX entry point
 *     only (the check is then skipped); elsewhere it is required.
 *   - Input bf16 data must be 16-byte aligned; code and scale outputs
 *     must be 16-byte aligned; fp32 / fp64 arrays naturally aligned.
 *     Otherwise MXQ_ERR_ALIGN.
 *   - Inputs without elements are valid.  A group with no elements has
 *     amax 0, so its s2 is 0 and its M=4 count 0; an empty activation tile
 *     has input_scale 0; a tensor with no elements has both verifier sums
 *     0 and a relative error of 0.  Pointers to data of zero bytes (x,
 *     codes, scales, M bits, the workspace) may then be NULL; the global
 *     scales, status and per-group or per-tensor outputs are still required.
 *   - Tensors are row-major and contiguous; blocks run along the last
 *     dimension (`cols`), which must be a multiple of the block size
 *     (16 for NVFP4, 32 for MX), otherwise MXQ_ERR_SHAPE.
 *   - Value codes: two 4-bit codes per byte, element 2j in the low nibble
 *     and element 2j+1 in the high nibble (NVFP4, MXFP4); one byte per
 *     element for MXFP8.  Scales: one byte per block, in one of two layouts
 *     (mxq_layout): MXQ_LAYOUT_LINEAR, row-major [rows, cols / block] per
 *     scale matrix (the checkpoint layout), or MXQ_LAYOUT_SWIZZLED_128X4,
 *     the tiled layout block-scaled tensor-core GEMMs read: the matrix is
 *     padded to a multiple of 128 rows and 4 columns and cut into tiles of
 *     128 x 4 scales (512 bytes) stored row-tile-major; inside a tile the
 *     scale of (row r, column c) sits at byte
 *     (r % 32) * 16 + ((r / 32) % 4) * 4 + (c % 4).  Padding bytes are 0.
 *     The pages only say that a loader may repack or interleave quantized
 *     weights for the kernel (josch15366/Qwen3.8-Flash-Next-NVFP4-
 *     LocalHessian-Experts, "Verifying the merge"); the tile layout is the
 *     public block-scaling convention of the tensor-core GEMMs, not
 *     something the pages define.
 */
#ifndef MXQ_H
#define MXQ_H

#include <stddef.h>
#include <stdint.h>
#include <cuda_runtime_api.h>

#if defined(__GNUC__)
#define MXQ_API __attribute__((visibility("default")))
#else
#define MXQ_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum mxq_status {
    MXQ_OK = 0,
    MXQ_ERR_INVALID_ARG = 1,  /* null pointer, negative size, unknown enum */
    MXQ_ERR_SHAPE = 2,        /* cols not a multiple of the block, overflow */
    MXQ_ERR_ALIGN = 3,        /* a pointer is not aligned as required */
    MXQ_ERR_WORKSPACE = 4,    /* workspace NULL or smaller than required */
    MXQ_ERR_CUDA = 5,         /* a CUDA runtime call failed */
    MXQ_ERR_UNSUPPORTED = 6   /* valid but unsupported request (MX block != 32) */
} mxq_status;

/* Bits of the device status word. */
#define MXQ_DEV_NONFINITE_INPUT 0x1u
#define MXQ_DEV_WAIT_TIMEOUT 0x2u
#define MXQ_DEV_INVALID_SCALE 0x4u

typedef enum mxq_fmt {
    MXQ_FMT_NVFP4 = 0,
    MXQ_FMT_MXFP4 = 1,
    MXQ_FMT_MXFP8 = 2
} mxq_fmt;

typedef enum mxq_scale_mode {
    MXQ_SCALE_RTN = 0,       /* plain amax/6 block scales */
    MXQ_SCALE_FOUR_SIX = 1   /* 4/6-optimal block scales */
} mxq_scale_mode;

typedef enum mxq_layout {
    MXQ_LAYOUT_LINEAR = 0,          /* row-major [rows, cols / block] */
    MXQ_LAYOUT_SWIZZLED_128X4 = 1   /* 128 x 4 tiles, see the conventions */
} mxq_layout;

typedef enum mxq_op {
    MXQ_OP_QUANTIZE_NVFP4 = 0,
    MXQ_OP_QUANTIZE_ACT = 1,
    MXQ_OP_DEQUANT_RELERR = 2
} mxq_op;

/* Census of a conversion, accumulated on the device by mxq_census_add
 * (device memory, caller-owned, 8-byte aligned; 13 fields of 8 bytes).
 * Source: dabsLabs/Qwen3.8-Flash-Next-NVFP4, metric table (mean and max
 * relative error of the quantized expert tensors against the bf16 source,
 * over the census of 48 x 512 x 3 tensors) and "What makes this build
 * different" (total squared error of the 4/6 choice against plain RTN block
 * scales; share of 16-blocks that chose the four-over-six plan). */
typedef struct mxq_census {
    double sum_relerr;       /* sum of the tensors' relative errors */
    double max_relerr;       /* largest relative error (0 before any tensor) */
    double sum_sq_err;       /* sum over the tensors of sum (x - deq)^2 */
    double sum_sq_ref;       /* sum over the tensors of sum x^2 */
    double sum_sq_err_rtn;   /* the same error total of the RTN comparison tensors */
    uint64_t n_tensors;      /* tensors added */
    uint64_t n_tensors_rtn;  /* of which added with an RTN counterpart */
    uint64_t blocks;         /* NVFP4 blocks of the groups added */
    uint64_t blocks_m4;      /* of which took the M=4 plan */
    double mean_relerr;      /* sum_relerr / n_tensors (0 when none) */
    double sse_vs_rtn;       /* sum_sq_err / sum_sq_err_rtn - 1: NaN unless
                                every tensor came with its RTN counterpart and
                                that total is > 0 */
    double m4_fraction;      /* blocks_m4 / blocks (0 when none) */
    double reserved;         /* 0 */
} mxq_census;

/* Version of this ABI (major * 10000 + minor * 100 + patch). */
MXQ_API int mxq_version(void);

/* Human-readable name of a status code (static string, never NULL). */
MXQ_API const char *mxq_status_string(mxq_status s);

/* Bytes of the scale output of `n_matrices` scale matrices, each holding the
 * block scales of a [rows, cols] tensor (block 16 for NVFP4, 32 for MX), in
 * `layout`: n * rows * (cols / block) when linear, n * pad128(rows) *
 * pad4(cols / block) when swizzled.  Returns 0 for invalid arguments. */
MXQ_API size_t mxq_scale_bytes(mxq_fmt fmt, mxq_layout layout, int64_t n_matrices, int64_t rows,
                               int64_t cols);

/* Bytes of device workspace an entry point needs (0 if none).
 *   MXQ_OP_QUANTIZE_NVFP4: n = n_groups, rows, cols as passed to it;
 *   MXQ_OP_QUANTIZE_ACT:   n = T, rows = hidden, cols ignored;
 *   MXQ_OP_DEQUANT_RELERR: n = n_tensors, rows, cols as passed to it.
 * Returns 0 for invalid arguments. */
MXQ_API size_t mxq_workspace_bytes(mxq_op op, int64_t n, int64_t rows, int64_t cols);

/* NVFP4 quantization of a stack of groups.
 * Source: dabsLabs/Qwen3.8-Flash-Next-NVFP4, "What makes this build
 * different"; josch15366/Qwen3.8-Flash-Next-NVFP4-LocalHessian-Experts,
 * introduction.
 *   x        bf16 [n_groups, rows, cols].  A group shares one global scale:
 *            pass one expert's fused gate_up slab [2I, H] per group so that
 *            gate and up share weight_scale_2; down slabs [H, I] form their
 *            own groups.  cols % 16 == 0.
 *   mode     MXQ_SCALE_RTN or MXQ_SCALE_FOUR_SIX.
 *   layout   scale layout; each group is one scale matrix [rows, cols/16].
 *   codes    out, uint8 [n_groups, rows, cols/2] E2M1 nibbles.
 *   scales   out, E4M3 block scales, mxq_scale_bytes(MXQ_FMT_NVFP4, layout,
 *            n_groups, rows, cols) bytes: [n_groups, rows, cols/16] when
 *            linear.
 *   s2       out, fp32 [n_groups]: s2 = RN32(amax_g / 2688).
 *   mbits    out, nullable, uint32 [ceil(n_groups*rows*cols/16 / 32)]:
 *            bit (b % 32) of word (b / 32) is 1 when block b (row-major
 *            block index over the whole stack) took the M=4 plan.  Unused
 *            high bits of the last word are written 0.
 *   m4_count out, nullable, uint32 [n_groups]: number of M=4 blocks per
 *            group (4/6 mode; zeros in RTN mode).
 *   status   required, see conventions.
 *   workspace / workspace_bytes: at least
 *            mxq_workspace_bytes(MXQ_OP_QUANTIZE_NVFP4, n_groups, rows, cols).
 * Per block of 16 (M in {6, 4}): t = RN32(amax_b / RN32(M*s2)), scale byte
 * S = E4M3(t) (round to nearest even, saturating at 448), D its value,
 * d = RN32(D*s2), code_i = E2M1(RN32(x_i / d)) (round to nearest even,
 * saturating at 6, sign kept; all codes 0 when D or d is 0).  In 4/6 mode
 * the M=4 plan is kept only when its exact squared error
 * sum (x_i - q_i*D*s2)^2 is strictly lower than the M=6 plan's. */
MXQ_API mxq_status mxq_quantize_nvfp4(const uint16_t *x, int64_t n_groups, int64_t rows,
                              int64_t cols, mxq_scale_mode mode, mxq_layout layout, uint8_t *codes,
                              uint8_t *scales, float *s2, uint32_t *mbits,
                              uint32_t *m4_count, uint32_t *status, void *workspace,
                              size_t workspace_bytes, cudaStream_t stream);

/* The global scale of each NVFP4 group alone: s2 = RN32(amax_g / 2688).
 * Source: josch15366/Qwen3.8-Flash-Next-NVFP4-LocalHessian-Experts,
 * introduction (weight_scale_2 and input_scale are amax / 2688).
 *   x       bf16 [n_groups, rows, cols], cols % 16 == 0 (as mxq_quantize_nvfp4).
 *   s2      out, fp32 [n_groups]; the bits of s2 equal what mxq_quantize_nvfp4
 *           writes for the same groups.  Rounding is monotone, so the scale of
 *           a group split over two calls (gate and up held apart) is the
 *           larger of its two parts' scales.
 *   status  required: MXQ_DEV_NONFINITE_INPUT when an element is Inf or NaN.
 * No workspace: s2 holds the running amax until the last kernel of the call
 * turns it into the scale.  With mxq_quantize_nvfp4_s2 this is the two-pass
 * form of mxq_quantize_nvfp4 (x is read twice). */
MXQ_API mxq_status mxq_global_scale_nvfp4(const uint16_t *x, int64_t n_groups, int64_t rows,
                                          int64_t cols, float *s2, uint32_t *status,
                                          cudaStream_t stream);

/* NVFP4 quantization with a caller-given global scale per group.
 * Source: josch15366/Qwen3.8-Flash-Next-NVFP4-LocalHessian-Experts,
 * introduction: gate and up share one weight_scale_2, and an activation's
 * input_scale is amax / 2688.  This entry point serves callers that hold the
 * two halves of a shared group apart (gate and up as separate tensors, which
 * must both use RN32(max(amax_gate, amax_up) / 2688)), or that reduced a
 * tile's amax elsewhere (a token-sharded activation tile).
 *   x, n_groups, rows, cols, mode, layout, codes, scales, mbits, m4_count,
 *            status: as mxq_quantize_nvfp4.
 *   s2_in    fp32 [n_groups], the global scale of each group, finite and
 *            >= 0 (a negative or non-finite scale sets
 *            MXQ_DEV_INVALID_SCALE; s2 = 0 gives all-zero codes and scales).
 * No workspace: the block quantizer of mxq_quantize_nvfp4 runs with s2 taken
 * from s2_in instead of RN32(amax_g / 2688), in one read of x.  With s2_in
 * equal to what mxq_quantize_nvfp4 writes, the outputs are byte-identical to
 * its outputs. */
MXQ_API mxq_status mxq_quantize_nvfp4_s2(const uint16_t *x, int64_t n_groups, int64_t rows,
                                         int64_t cols, const float *s2_in, mxq_scale_mode mode,
                                         mxq_layout layout, uint8_t *codes, uint8_t *scales,
                                         uint32_t *mbits, uint32_t *m4_count, uint32_t *status,
                                         cudaStream_t stream);

/* NVFP4 quantization with a weighted-SSE block-scale search.
 * Source: josch15366/Qwen3.8-Flash-Next-NVFP4-LocalHessian-Experts, "What is
 * different about it": the per-group weight scales are chosen by a
 * Hessian-weighted search (ModelOpt local_hessian) instead of the plain
 * amax / MSE sweep.  The pages give no formula; the readings are stated here.
 *   x, n_groups, rows, cols, layout, codes, scales, s2, status, workspace:
 *            as mxq_quantize_nvfp4 (same groups, same s2 = RN32(amax_g / 2688),
 *            workspace of MXQ_OP_QUANTIZE_NVFP4).
 *   h        fp32 weights >= 0 per input channel (a diagonal Hessian estimate,
 *            e.g. the mean squared activation of that channel), 16-byte
 *            aligned: [cols] shared by every group (h_groups == 1) or
 *            [n_groups, cols] (h_groups == n_groups).
 * Per block of 16: the candidates are every E4M3 scale code from the amax/6
 * plan's code to the four-over-six plan's code (both plans as in
 * mxq_quantize_nvfp4); each candidate's value codes follow as in that entry
 * point, and its weighted error sum_i h_i (x_i - q_i D s2)^2 is formed in
 * binary64 in element order (deq = (q D) s2, e = x - deq, acc += h (e e),
 * each operation rounded to nearest).  The lowest error wins; ties go to the
 * smaller code.  A negative or non-finite weight, like a non-finite input,
 * sets MXQ_DEV_NONFINITE_INPUT. */
MXQ_API mxq_status mxq_quantize_nvfp4_weighted(const uint16_t *x, int64_t n_groups, int64_t rows,
                                               int64_t cols, const float *h, int64_t h_groups,
                                               mxq_layout layout, uint8_t *codes, uint8_t *scales,
                                               float *s2, uint32_t *status, void *workspace,
                                               size_t workspace_bytes, cudaStream_t stream);

/* MX quantization (MXFP4 or MXFP8), one UE8M0 scale per 32 values.
 * Source: azampatti/Qwen3.8-Flash-Next-FP4-Local-AZ, "The shared expert";
 * MJPansa/Qwen3.8-Flash-Next-MXFP4-FP8-R12, "Quantization format".
 *   x       bf16 [rows, cols], cols % 32 == 0 (stacked tensors: pass
 *           rows = product of the leading dimensions).
 *   fmt     MXQ_FMT_MXFP4 (E2M1, qmax 6) or MXQ_FMT_MXFP8 (E4M3, qmax 448).
 *   block   must be 32 (MXQ_ERR_UNSUPPORTED otherwise).
 *   layout  scale layout; the whole [rows, cols/32] is one scale matrix
 *           (stack tensors whose row count is a multiple of 128, or call
 *           once per tensor, to get one tiled matrix per tensor).
 *   codes   out, uint8 [rows, cols/2] (MXFP4) or [rows, cols] (MXFP8).
 *   scales  out, mxq_scale_bytes(fmt, layout, 1, rows, cols) bytes
 *           ([rows, cols/32] when linear), byte = e + 127 with e the smallest
 *           integer such that amax <= qmax * 2^e (= ceil(log2(amax/qmax))),
 *           clamped to [-127, 127]; an all-zero block gives byte 0.
 *   status  nullable.
 * code_i = FMT(x_i * 2^-e), round to nearest even, sign kept. */
MXQ_API mxq_status mxq_quantize_mx(const uint16_t *x, int64_t rows, int64_t cols, mxq_fmt fmt,
                           int block, mxq_layout layout, uint8_t *codes, uint8_t *scales,
                           uint32_t *status, cudaStream_t stream);

/* FP8 -> MX requantization of a block-FP8 source tensor.
 * Source: MJPansa/Qwen3.8-Flash-Next-MXFP4-FP8-R12, "Quantization and layer
 * selection" (the conversion started from the released FP8 weights, without
 * a BF16 copy) and "Quantization format" (converted routed experts are MXFP4
 * E2M1 with UE8M0 scales; retained layers keep the source block-FP8 format).
 * The pages do not give the source block shape or the arithmetic of the
 * conversion; the readings are stated here.
 *   fp8     E4M3 codes [rows, cols], one byte per value, 16-byte aligned.
 *   bscale  fp32 [ceil(rows / brows), ceil(cols / bcols)]: value (r, c) of
 *           the source is E4M3(code) * bscale[r / brows][c / bcols].
 *   brows, bcols  source block shape (128 x 128 in the usual block-FP8
 *           checkpoints); bcols must be a multiple of 32 (MXQ_ERR_SHAPE).
 *   fmt, layout, codes, scales, status  as mxq_quantize_mx (block 32; the
 *           whole [rows, cols/32] is one scale matrix); rows * cols / 32 must
 *           stay below 2^32 (MXQ_ERR_SHAPE).
 * Each value is dequantized once to fp32, w = RN32(E4M3(code) * scale), and
 * every run of 32 w is MX-quantized as mxq_quantize_mx does with bf16 input:
 * e = smallest integer with amax <= qmax * 2^e (clamped to [-127, 127]),
 * code = FMT(w * 2^-e).  A NaN source code (S.1111.111) or a non-finite
 * scale sets MXQ_DEV_NONFINITE_INPUT. */
MXQ_API mxq_status mxq_requant_fp8_mx(const uint8_t *fp8, const float *bscale, int64_t rows,
                                      int64_t cols, int64_t brows, int64_t bcols, mxq_fmt fmt,
                                      mxq_layout layout, uint8_t *codes, uint8_t *scales,
                                      uint32_t *status, cudaStream_t stream);

/* Dynamic activation quantization of a token tile [T, hidden].
 * Source: josch15366/Qwen3.8-Flash-Next-NVFP4-LocalHessian-Experts,
 * introduction (input_scale = amax/2688); MJPansa/Qwen3.8-Flash-Next-MXFP4-FP8-R12,
 * "Quantization format" (activations dynamically quantized to MXFP8).
 *   fmt = MXQ_FMT_NVFP4: the whole tile is one group, input_scale =
 *         RN32(amax / 2688) written to *input_scale (device fp32); block
 *         scales by `mode`: MXQ_SCALE_RTN (plain amax/6, the pages'
 *         activation recipe) or MXQ_SCALE_FOUR_SIX (the weights' 4/6-optimal
 *         rule applied to the tile); codes [T, hidden/2], scales as
 *         mxq_quantize_nvfp4 with one group; workspace required.
 *   fmt = MXQ_FMT_MXFP8 or MXQ_FMT_MXFP4: as mxq_quantize_mx with block 32;
 *         mode must be MXQ_SCALE_RTN (MXQ_ERR_UNSUPPORTED otherwise);
 *         input_scale, workspace may be NULL.
 *   layout scale layout, as for the quantizers above.
 *   status required. */
MXQ_API mxq_status mxq_quantize_act(const uint16_t *tokens, int64_t T, int64_t hidden,
                            mxq_fmt fmt, mxq_scale_mode mode, mxq_layout layout,
                            uint8_t *codes, uint8_t *scales,
                            float *input_scale, uint32_t *status, void *workspace,
                            size_t workspace_bytes, cudaStream_t stream);

/* Dequantize and measure per-tensor squared errors (the verifier).
 * Source: dabsLabs/Qwen3.8-Flash-Next-NVFP4 (relative error of the
 * quantized experts against the bf16 source, per tensor, mean and max);
 * azampatti/Qwen3.8-Flash-Next-FP4-Local-AZ, "The shared expert" (error
 * against the bf16 master).
 *   x, codes, scales  as written by the quantizers, viewed as n_tensors
 *            tensors of [rows, cols] stored back to back (unstacking a
 *            fused gate_up [E, 2I, H] gives 2E tensors of [I, H]).
 *   s2       NVFP4 only: fp32 [n_tensors / tensors_per_scale]; tensor t
 *            reads s2[t / tensors_per_scale] (2 for fused gate_up, so that
 *            gate_e and up_e read the shared weight_scale_2).  NULL for MX.
 *   layout   layout of `scales`.  For the tiled layout, tensors_per_scale
 *            consecutive tensors form one scale matrix (one NVFP4 group;
 *            for MX pass n_tensors when the stack was quantized as one
 *            matrix, 1 when each tensor was).
 *   sum_sq_err, sum_sq_ref   out, fp64 [n_tensors]: sum (x - deq)^2 and
 *            sum x^2 with deq = q * D * s2 (NVFP4) or q * 2^e (MX); each
 *            x - deq is rounded once to fp32 and the squares are summed in
 *            fp32 runs of 8 and fp64 across blocks, so both sums lie within
 *            11 * 2^-24 (6.6e-7) relative of the exact ones.
 *   relerr   out, nullable, fp64 [n_tensors]: sqrt(err) / sqrt(ref)
 *            (0 when both are 0).
 *   workspace: mxq_workspace_bytes(MXQ_OP_DEQUANT_RELERR, n_tensors, rows, cols).
 * The sums are formed in a fixed order that does not depend on scheduling,
 * so repeated calls give bit-identical results. */
MXQ_API mxq_status mxq_dequant_relerr(const uint16_t *x, const uint8_t *codes,
                              const uint8_t *scales, const float *s2, mxq_fmt fmt,
                              mxq_layout layout, int64_t n_tensors, int64_t rows, int64_t cols,
                              int64_t tensors_per_scale, double *sum_sq_err,
                              double *sum_sq_ref, double *relerr, void *workspace,
                              size_t workspace_bytes, cudaStream_t stream);

/* The verifier above, for callers that cannot allocate device memory.
 * The pages have no counterpart to this entry point; it exists for callers
 * that reserve their whole device-memory budget up front (and so cannot
 * cudaMalloc a workspace) or must not risk the synchronisation a cudaMalloc
 * can cause.  It takes no workspace: the per-chunk partial sums live in a
 * fixed 2 MiB array inside the library's device image, which every GPU that
 * loads the library holds until the process exits.  Arguments, outputs and
 * results are those of mxq_dequant_relerr with linear scales.
 *   Limit: n_tensors * ceil(rows * cols / 16384) <= 131072 chunks (for
 *   example 1024 tensors of 768 x 2048, or 512 of 2048 x 768); larger
 *   requests return MXQ_ERR_WORKSPACE before anything is enqueued.
 *   The first call on a device looks up the array's device address on that
 *   device (cudaGetSymbolAddress) and caches it with the id of the device's
 *   current context; a later call made in another context (after a
 *   cudaDeviceReset, say) looks it up again.  Make the first call on a
 *   device, and the first after such a reset, before any stream capture.
 *   It allocates nothing: no cudaMalloc, no cudaFree.
 *   Every call on a device uses the same array and leaves its last contents
 *   there (each call writes every partial it reads, so nothing needs to
 *   start at zero); calls whose GPU work overlaps in time, on any streams,
 *   race on it and give undefined results. */
MXQ_API mxq_status mxq_dequant_relerr_noalloc(const uint16_t *x, const uint8_t *codes,
                                              const uint8_t *scales, const float *s2,
                                              mxq_fmt fmt, int64_t n_tensors, int64_t rows,
                                              int64_t cols, int64_t tensors_per_scale,
                                              double *sum_sq_err, double *sum_sq_ref,
                                              double *relerr, cudaStream_t stream);

/* Zero a census (enqueued on `stream`).  census: device mxq_census. */
MXQ_API mxq_status mxq_census_reset(mxq_census *census, cudaStream_t stream);

/* Add one verifier call's per-tensor figures, and one quantizer call's M=4
 * counts, to a census (see mxq_census for the source passages).
 *   census          device mxq_census, 8-byte aligned.
 *   n_tensors       tensors to add (0: none); then sum_sq_err, sum_sq_ref and
 *                   relerr (fp64 [n_tensors], as mxq_dequant_relerr writes
 *                   them) are required.
 *   sum_sq_err_rtn  nullable, fp64 [n_tensors]: the verifier's sum_sq_err of
 *                   the same tensors quantized with MXQ_SCALE_RTN, for
 *                   sse_vs_rtn.
 *   n_groups        groups whose M=4 counts to add (0: none); then m4_count
 *                   (uint32 [n_groups], as mxq_quantize_nvfp4 writes it) is
 *                   required and blocks_per_group >= 0 gives their blocks.
 * One CTA adds the arrays in a fixed order (element i to partial i % 256,
 * in order, then a fixed tree) and then adds the totals to the census and
 * recomputes its derived fields, so the same sequence of calls gives the
 * same bits.  Calls on one census must be ordered (one stream). */
MXQ_API mxq_status mxq_census_add(mxq_census *census, int64_t n_tensors, const double *sum_sq_err,
                                  const double *sum_sq_ref, const double *relerr,
                                  const double *sum_sq_err_rtn, int64_t n_groups,
                                  const uint32_t *m4_count, int64_t blocks_per_group,
                                  cudaStream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* MXQ_H */
