/*
 * mxq_oracle.c -- plain, slow, scalar CPU oracle of the block-scaled
 * microscaling quantizer (NVFP4 4/6-optimal, MXFP4, MXFP8) and its
 * dequantize + relative-error verifier.
 *
 * TEST INFRASTRUCTURE ONLY.  This file is the checker, not the product:
 * only the test suite, the package smoke check and the benchmark's CPU
 * baseline leg load it.  It shares no code, header, table or helper with
 * the CUDA library, and the CUDA library never calls it.
 *
 * Build: gcc -O2 -std=c11 -ffp-contract=off -fno-fast-math -fPIC -shared
 * (no FMA contraction, no flush-to-zero: every float operation below is
 * one IEEE-754 binary32 or binary64 operation, rounded to nearest even).
 *
 * Sources (model-card pages; section in quotes):
 *  [P1] josch15366/Qwen3.8-Flash-Next-NVFP4-LocalHessian-Experts,
 *       introduction (input_scale = amax/2688; gate and up share one
 *       weight_scale_2) and "What is different about it" (one
 *       weight_scale_2 per expert).
 *  [P2] azampatti/Qwen3.8-Flash-Next-FP4-Local-AZ, "The shared expert"
 *       (MXFP8: e4m3 values, one power-of-two scale per 32 weights,
 *       e = ceil(log2(amax / 448))) and the zero-padded 640 -> 1280
 *       shared expert (silu(0) * 0 = 0).
 *  [P3] dabsLabs/Qwen3.8-Flash-Next-NVFP4, "What makes this build
 *       different" (per 16-element block, choose between the amax/6 plan
 *       and the four-over-six plan by exact post-rounding squared error;
 *       never worse than plain RTN) and the metric table (relative error
 *       of quantized experts against the bf16 source).
 *  [P4] MJPansa/Qwen3.8-Flash-Next-MXFP4-FP8-R12, "Quantization format"
 *       (MXFP4 E2M1 weights with UE8M0 microscales; activations
 *       dynamically quantized to MXFP8).
 *
 * Readings taken where the pages are silent are stated at each function.
 * Every function here is pinned by tests that do not use this file's
 * arithmetic (see tests/test_oracle_*.py).
 */
#include <math.h>
#include <stdint.h>
#include <string.h>

/* ------------------------------------------------------------------ */
/* Number formats.  The pages name E2M1, E4M3 and UE8M0 without giving  */
/* bit layouts; the reading is the OCP microscaling / OCP FP8 "fn"       */
/* definitions: E2M1 = sign, 2 exponent bits (bias 1), 1 mantissa bit;   */
/* E4M3 = sign, 4 exponent bits (bias 7), 3 mantissa bits, no infinity,  */
/* S.1111.111 is NaN, largest finite 448; UE8M0 byte b = 2^(b-127),      */
/* 0xFF is NaN.                                                          */
/* ------------------------------------------------------------------ */

double oracle_e2m1_value(unsigned code)
{
    unsigned s = (code >> 3) & 1u, e = (code >> 1) & 3u, m = code & 1u;
    double mag;
    if (e == 0)
        mag = 0.5 * (double)m;                      /* subnormal: m * 2^-1 */
    else
        mag = ldexp(1.0 + 0.5 * (double)m, (int)e - 1);
    return s ? -mag : mag;
}

double oracle_e4m3_value(unsigned code)
{
    unsigned s = (code >> 7) & 1u, e = (code >> 3) & 15u, m = code & 7u;
    double mag;
    if (e == 15 && m == 7)
        return NAN;
    if (e == 0)
        mag = ldexp((double)m / 8.0, -6);           /* subnormal: m/8 * 2^-6 */
    else
        mag = ldexp(1.0 + (double)m / 8.0, (int)e - 7);
    return s ? -mag : mag;
}

double oracle_ue8m0_value(unsigned code)
{
    if ((code & 0xFFu) == 0xFFu)
        return NAN;
    return ldexp(1.0, (int)(code & 0xFFu) - 127);
}

/* Round a finite real value to the nearest representable magnitude of a
 * format, ties to the even code (the code whose last mantissa bit is 0),
 * magnitudes beyond the largest finite one saturate to it ("satfinite"),
 * and the sign bit is copied from the input, so a negative value that
 * rounds to zero gives negative zero.  This is round-to-nearest-even
 * stated as a search over the format's codes: it needs no bit tricks. */
static unsigned nearest_code(double v, unsigned n_mag_codes,
                             double (*value_of)(unsigned), unsigned sign_bit,
                             double max_finite, unsigned max_code)
{
    double a = fabs(v);
    unsigned best = 0;
    if (a >= max_finite) {
        best = max_code;
    } else {
        double best_dist = INFINITY;
        for (unsigned c = 0; c < n_mag_codes; ++c) {
            double dist = fabs(a - value_of(c));   /* exact: both are short dyadics */
            if (dist < best_dist || (dist == best_dist && (c & 1u) == 0u)) {
                best = c;
                best_dist = dist;
            }
        }
    }
    return signbit(v) ? (best | sign_bit) : best;
}

/* E2M1 encode of a real value (round to nearest even code, satfinite).
 * Non-finite input returns 0xFF, which is not a valid code. */
unsigned oracle_e2m1_encode(double v)
{
    if (!isfinite(v))
        return 0xFFu;
    return nearest_code(v, 8u, oracle_e2m1_value, 0x8u, 6.0, 0x7u);
}

/* E4M3 encode of a real value (round to nearest even code, satfinite to
 * +-448: the NaN code is never produced).  Non-finite input -> 0xFFFF. */
unsigned oracle_e4m3_encode(double v)
{
    if (!isfinite(v))
        return 0xFFFFu;
    return nearest_code(v, 127u, oracle_e4m3_value, 0x80u, 448.0, 0x7Eu);
}

/* MX shared exponent [P2 "The shared expert"; P4 "Quantization format"]:
 * e = ceil(log2(amax / qmax)), read as the smallest integer e with
 * amax <= qmax * 2^e, so no element of the block needs saturation.
 * Clamped to the UE8M0 range [-127, 127]; amax = 0 gives -127 (byte 0). */
int oracle_mx_exponent(double amax, double qmax)
{
    int e = -127;
    if (!(amax > 0.0))
        return -127;
    while (e < 127 && amax > ldexp(qmax, e))
        ++e;
    return e;
}

static float bf16_to_float(uint16_t b)
{
    uint32_t u = (uint32_t)b << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return f;
}

/* ------------------------------------------------------------------ */
/* Exactness guards.  The 4/6 decision below is evaluated with binary64 */
/* operations that are exact for every block the method can produce;    */
/* each step is checked and a violated premise is reported, never       */
/* silently rounded.                                                     */
/* ------------------------------------------------------------------ */
static double exact_mul(double a, double b, int *ok)
{
    double p = a * b;
    if (fma(a, b, -p) != 0.0)
        *ok = 0;
    return p;
}

static double exact_add(double a, double b, int *ok)
{
    double s = a + b;
    double bb = s - a;
    double err = (a - (s - bb)) + (b - bb);        /* Knuth two-sum */
    if (err != 0.0)
        *ok = 0;
    return s;
}

/* One NVFP4 plan for one 16-element block [P3 "What makes this build
 * different"; P1 introduction].
 *   t   = RN32(amax_b / RN32(M * s2))             block scale in s2 units
 *   S   = E4M3(t), D its value                    stored weight_scale byte
 *   d   = RN32(D * s2)                            fp32 effective block scale
 *   c_i = E2M1(RN32(x_i / d))                     stored value codes
 * Readings: the pages name the plan "amax/6" (in units of weight_scale_2)
 * without an operation order; the divisor M * s2 is rounded once to fp32
 * and the block amax divided by it once.  D = 0, s2 = 0 or d = 0
 * (underflow) give all-zero codes 0x0.
 * Returns, through G, the exact value of (SSE_M - sum x_i^2) / s2 where
 * SSE_M = sum_i (x_i - q_i * D * s2)^2 is the exact squared error of the
 * stored reconstruction q_i * D * s2 (q_i = value of c_i).  Expanding the
 * square, SSE_M - sum x^2 = s2 * D * (D * s2 * B - 2 * A) with
 * A = sum x_i q_i and B = sum q_i^2, so G = D * (D*s2*B - 2A).
 * Return 0 on success, -2 if an exactness premise failed. */
static int nvfp4_plan(const float x[16], float amax_b, float s2, float M,
                      unsigned *scale_code, uint8_t codes[16], double *G)
{
    int ok = 1;
    unsigned sc = 0;
    double D = 0.0;
    float d = 0.0f;

    if (s2 > 0.0f) {
        float den = M * s2;                          /* RN32(M * s2) */
        float t = amax_b / den;
        sc = oracle_e4m3_encode((double)t);
        D = oracle_e4m3_value(sc);
        d = (float)D * s2;
    }
    *scale_code = sc;
    if (D == 0.0 || d == 0.0f) {
        for (int i = 0; i < 16; ++i)
            codes[i] = 0;
        *G = 0.0;
        return 0;
    }
    double A = 0.0, B = 0.0;
    for (int i = 0; i < 16; ++i) {
        float y = x[i] / d;
        unsigned c = oracle_e2m1_encode((double)y);
        codes[i] = (uint8_t)c;
        double q = oracle_e2m1_value(c);
        A = exact_add(A, exact_mul((double)x[i], q, &ok), &ok);
        B = exact_add(B, exact_mul(q, q, &ok), &ok);
    }
    double dS = exact_mul(D, (double)s2, &ok);
    double P = exact_add(exact_mul(dS, B, &ok), -2.0 * A, &ok);
    *G = exact_mul(D, P, &ok);
    return ok ? 0 : -2;
}

/* The blocks of one NVFP4 group with global scale s2 [P3 "What makes this
 * build different"]: per block of 16 the amax/6 plan and, in 4/6 mode
 * (mode 1), the four-over-six plan; the M=4 plan wins only when its exact
 * squared error is strictly lower, so ties keep the amax/6 plan and the
 * result equals plain RTN unless it is strictly better.  xg holds the
 * group's nblk * 16 bf16 values, g is the group's index in the stack (the
 * outputs are written at its blocks).  Returns 0 or -2. */
static int nvfp4_group(const uint16_t *xg, int64_t nblk, int64_t g, float s2, int mode,
                       uint8_t *codes, uint8_t *scales, uint8_t *m4)
{
    int rc = 0;
    for (int64_t b = 0; b < nblk; ++b) {
        float xb[16];
        float amax_b = 0.0f;
        for (int i = 0; i < 16; ++i) {
            xb[i] = bf16_to_float(xg[b * 16 + i]);
            if (fabsf(xb[i]) > amax_b)
                amax_b = fabsf(xb[i]);
        }
        unsigned sc6, sc4 = 0;
        uint8_t c6[16], c4[16];
        double G6, G4 = 0.0;
        int r = nvfp4_plan(xb, amax_b, s2, 6.0f, &sc6, c6, &G6);
        if (r)
            rc = r;
        int use4 = 0;
        if (mode == 1) {
            r = nvfp4_plan(xb, amax_b, s2, 4.0f, &sc4, c4, &G4);
            if (r)
                rc = r;
            use4 = (G4 < G6);
        }
        const uint8_t *c = use4 ? c4 : c6;
        int64_t gb = g * nblk + b;
        for (int j = 0; j < 8; ++j)
            codes[gb * 8 + j] = (uint8_t)((c[2 * j] & 0xF) | ((c[2 * j + 1] & 0xF) << 4));
        scales[gb] = (uint8_t)(use4 ? sc4 : sc6);
        if (m4)
            m4[gb] = (uint8_t)use4;
    }
    return rc;
}

/* NVFP4 quantization of a stack of groups [P1 introduction; P3 "What
 * makes this build different"].
 *   x            bf16 bits, [n_groups, rows, cols] row-major
 *   global_div   2688 = 6 * 448 (weight_scale_2 and input_scale); tests
 *                pass other values only to plant the historical bug
 *   mode         0 = plain amax/6 (RTN), 1 = 4/6-optimal
 *   codes        [n_groups, rows, cols/2]: element 2j in the low nibble,
 *                element 2j+1 in the high nibble
 *   scales       [n_groups, rows, cols/16] E4M3 bytes
 *   s2_out       [n_groups] fp32 global scale RN32(amax_g / global_div)
 *   m4           nullable, one byte per block: 1 if the M=4 plan won
 * Group = one expert's fused gate_up slab (gate and up share one
 * weight_scale_2), or one down slab, or one activation tile.  Returns 0,
 * -1 on bad shape, -2 on a failed exactness premise, -3 on non-finite
 * input. */
int oracle_quantize_nvfp4(const uint16_t *x, int64_t n_groups, int64_t rows,
                          int64_t cols, int mode, double global_div,
                          uint8_t *codes, uint8_t *scales, float *s2_out,
                          uint8_t *m4)
{
    if (n_groups < 0 || rows < 0 || cols < 0 || cols % 16 != 0)
        return -1;
    const int64_t gsize = rows * cols;
    const int64_t nblk = gsize / 16;
    int rc = 0;
    for (int64_t g = 0; g < n_groups; ++g) {
        const uint16_t *xg = x + g * gsize;
        float amax_g = 0.0f;
        for (int64_t i = 0; i < gsize; ++i) {
            float v = fabsf(bf16_to_float(xg[i]));
            if (!isfinite(v))
                return -3;
            if (v > amax_g)
                amax_g = v;
        }
        float s2 = amax_g / (float)global_div;
        s2_out[g] = s2;
        int r = nvfp4_group(xg, nblk, g, s2, mode, codes, scales, m4);
        if (r)
            rc = r;
    }
    return rc;
}

/* NVFP4 quantization with a caller-given global scale per group [P1
 * introduction: gate and up share one weight_scale_2, so a caller that holds
 * them apart passes the scale they share; an activation's input_scale may be
 * reduced elsewhere].  As oracle_quantize_nvfp4 with s2 = s2_in[g] instead
 * of RN32(amax_g / 2688).  s2_in must be finite and >= 0.  Returns 0, -1 on
 * bad shape or scale, -2 on a failed exactness premise, -3 on non-finite
 * input. */
int oracle_quantize_nvfp4_s2(const uint16_t *x, int64_t n_groups, int64_t rows,
                             int64_t cols, int mode, const float *s2_in,
                             uint8_t *codes, uint8_t *scales, uint8_t *m4)
{
    if (n_groups < 0 || rows < 0 || cols < 0 || cols % 16 != 0)
        return -1;
    const int64_t gsize = rows * cols;
    const int64_t nblk = gsize / 16;
    int rc = 0;
    for (int64_t g = 0; g < n_groups; ++g) {
        if (!(s2_in[g] >= 0.0f) || !isfinite(s2_in[g]))
            return -1;
        for (int64_t i = 0; i < gsize; ++i)
            if (!isfinite(bf16_to_float(x[g * gsize + i])))
                return -3;
        int r = nvfp4_group(x + g * gsize, nblk, g, s2_in[g], mode, codes, scales, m4);
        if (r)
            rc = r;
    }
    return rc;
}

/* MX quantization, one UE8M0 scale per 32 consecutive elements of a row
 * [P2 "The shared expert"; P4 "Quantization format"].
 *   fmt 1 = MXFP4 (E2M1 values, qmax 6, codes [rows, cols/2] nibbles,
 *           element 2j low), fmt 2 = MXFP8 (E4M3 values, qmax 448, codes
 *           [rows, cols]).  scales [rows, cols/32] = e + 127.
 * Value code = FMT(x * 2^-e), rounded to nearest even, satfinite (no
 * element exceeds qmax by the choice of e).  Returns 0, -1 bad shape,
 * -3 non-finite input. */
int oracle_quantize_mx(const uint16_t *x, int64_t rows, int64_t cols, int fmt,
                       uint8_t *codes, uint8_t *scales)
{
    if (rows < 0 || cols < 0 || cols % 32 != 0 || (fmt != 1 && fmt != 2))
        return -1;
    const double qmax = (fmt == 1) ? 6.0 : 448.0;
    const int64_t nblk = rows * cols / 32;
    for (int64_t b = 0; b < nblk; ++b) {
        double v[32];
        double amax = 0.0;
        for (int i = 0; i < 32; ++i) {
            v[i] = (double)bf16_to_float(x[b * 32 + i]);
            if (!isfinite(v[i]))
                return -3;
            if (fabs(v[i]) > amax)
                amax = fabs(v[i]);
        }
        int e = oracle_mx_exponent(amax, qmax);
        scales[b] = (uint8_t)(e + 127);
        for (int i = 0; i < 32; ++i) {
            double y = ldexp(v[i], -e);                 /* exact */
            if (fmt == 1) {
                unsigned c = oracle_e2m1_encode(y) & 0xFu;
                if (i & 1)
                    codes[b * 16 + i / 2] |= (uint8_t)(c << 4);
                else
                    codes[b * 16 + i / 2] = (uint8_t)c;
            } else {
                codes[b * 32 + i] = (uint8_t)oracle_e4m3_encode(y);
            }
        }
    }
    return 0;
}

/* Codes of one NVFP4 block for a given E4M3 scale code (the value half of
 * nvfp4_plan): d = RN32(D * s2), code_i = E2M1(RN32(x_i / d)); all codes 0
 * when D or d is 0. */
static void nvfp4_codes_for_scale(const float x[16], float s2, unsigned sc, uint8_t codes[16])
{
    const double D = oracle_e4m3_value(sc);
    const float d = (float)D * s2;
    for (int i = 0; i < 16; ++i)
        codes[i] = (D == 0.0 || d == 0.0f) ? 0 : (uint8_t)oracle_e2m1_encode((double)(x[i] / d));
}

/* Weighted squared error of one block in binary64, in this exact order
 * (the GPU forms the same operations in the same order):
 *   deq_i = (q_i * D) * s2            exact (2 + 4 + 24 significant bits)
 *   e_i   = x_i - deq_i               rounded to nearest
 *   acc  += h_i * (e_i * e_i)         two roundings, i = 0 .. 15 */
static double nvfp4_wsse(const float x[16], const float h[16], float s2, unsigned sc,
                         const uint8_t codes[16])
{
    const double D = oracle_e4m3_value(sc);
    double acc = 0.0;
    for (int i = 0; i < 16; ++i) {
        const double deq = (oracle_e2m1_value(codes[i]) * D) * (double)s2;
        const double e = (double)x[i] - deq;
        acc = acc + (double)h[i] * (e * e);
    }
    return acc;
}

/* NVFP4 with a weighted-SSE scale search [P1 "What is different about it":
 * per-group weight scales chosen by a Hessian-weighted search (ModelOpt
 * local_hessian) instead of the plain amax / MSE sweep].  The pages give
 * the idea, not the search; readings:
 *   - weights h >= 0 per input channel (a diagonal Hessian estimate such
 *     as the mean squared activation of that channel), one row of `cols`
 *     per group (h_groups == n_groups) or one shared row (h_groups == 1);
 *   - candidates: every E4M3 scale code from the amax/6 plan's code to the
 *     four-over-six plan's code of the same block (the codes between the
 *     two plans of the 4/6 rule, both included);
 *   - objective: sum h_c (x - q D s2)^2 over the block, formed in binary64
 *     as nvfp4_wsse states; the lowest value wins, ties to the smaller
 *     code (the amax/6 side).
 * s2, the plans' codes and the value codes follow oracle_quantize_nvfp4.
 * Returns 0, -1 on bad arguments, -3 on non-finite input or weight. */
int oracle_quantize_nvfp4_weighted(const uint16_t *x, int64_t n_groups, int64_t rows,
                                   int64_t cols, const float *h, int64_t h_groups,
                                   uint8_t *codes, uint8_t *scales, float *s2_out)
{
    if (n_groups < 0 || rows < 0 || cols < 0 || cols % 16 != 0 ||
        (h_groups != 1 && h_groups != n_groups))
        return -1;
    const int64_t gsize = rows * cols;
    const int64_t nblk = gsize / 16;
    for (int64_t i = 0; i < h_groups * cols; ++i)
        if (!isfinite(h[i]) || h[i] < 0.0f)
            return -3;
    for (int64_t g = 0; g < n_groups; ++g) {
        const uint16_t *xg = x + g * gsize;
        const float *hg = h + (h_groups == 1 ? 0 : g * cols);
        float amax_g = 0.0f;
        for (int64_t i = 0; i < gsize; ++i) {
            float v = fabsf(bf16_to_float(xg[i]));
            if (!isfinite(v))
                return -3;
            if (v > amax_g)
                amax_g = v;
        }
        const float s2 = amax_g / 2688.0f;
        s2_out[g] = s2;
        for (int64_t b = 0; b < nblk; ++b) {
            float xb[16];
            float amax_b = 0.0f;
            for (int i = 0; i < 16; ++i) {
                xb[i] = bf16_to_float(xg[b * 16 + i]);
                if (fabsf(xb[i]) > amax_b)
                    amax_b = fabsf(xb[i]);
            }
            const float *hb = hg + (b * 16) % cols;
            unsigned lo = 0, hi = 0;
            if (s2 > 0.0f) {
                lo = oracle_e4m3_encode((double)(amax_b / (6.0f * s2)));
                hi = oracle_e4m3_encode((double)(amax_b / (4.0f * s2)));
            }
            unsigned best_sc = lo;
            uint8_t best[16], c[16];
            nvfp4_codes_for_scale(xb, s2, lo, best);
            double best_w = nvfp4_wsse(xb, hb, s2, lo, best);
            for (unsigned sc = lo + 1; sc <= hi; ++sc) {
                nvfp4_codes_for_scale(xb, s2, sc, c);
                const double w = nvfp4_wsse(xb, hb, s2, sc, c);
                if (w < best_w) {
                    best_w = w;
                    best_sc = sc;
                    memcpy(best, c, 16);
                }
            }
            const int64_t gb = g * nblk + b;
            for (int j = 0; j < 8; ++j)
                codes[gb * 8 + j] = (uint8_t)((best[2 * j] & 0xF) | ((best[2 * j + 1] & 0xF) << 4));
            scales[gb] = (uint8_t)best_sc;
        }
    }
    return 0;
}

/* FP8 -> MX requantization [P4 "Quantization and layer selection": the
 * conversion started from the released FP8 weights, without a BF16 copy;
 * "Quantization format": the retained layers stay in the source block-FP8
 * format, the converted ones are MXFP4 E2M1 with UE8M0 scales].
 * Readings (the pages give neither): the source stores one E4M3 byte per
 * value and one fp32 scale per brows x bcols block, value = E4M3 * scale;
 * the conversion dequantizes each value to fp32 with one rounding,
 * w = RN32(E4M3(code) * scale), then quantizes the fp32 w exactly as the
 * bf16 MX path does (same exponent rule on the block amax, same encoding of
 * w * 2^-e).  fp8 [rows, cols]; bscale [ceil(rows/brows), ceil(cols/bcols)].
 * Returns -3 for a NaN source code or a non-finite scale. */
int oracle_requant_fp8_mx(const uint8_t *fp8, const float *bscale, int64_t rows,
                          int64_t cols, int64_t brows, int64_t bcols, int fmt,
                          uint8_t *codes, uint8_t *scales)
{
    if (rows < 0 || cols < 0 || cols % 32 != 0 || brows < 1 || bcols < 1 ||
        (fmt != 1 && fmt != 2))
        return -1;
    const double qmax = (fmt == 1) ? 6.0 : 448.0;
    const int64_t nbc = (cols + bcols - 1) / bcols;
    for (int64_t r = 0; r < rows; ++r) {
        for (int64_t j = 0; j < cols / 32; ++j) {
            float w[32];
            double amax = 0.0;
            for (int i = 0; i < 32; ++i) {
                const int64_t c = j * 32 + i;
                const uint8_t q = fp8[r * cols + c];
                const float sc = bscale[(r / brows) * nbc + c / bcols];
                if ((q & 0x7F) == 0x7F || !isfinite(sc))
                    return -3;
                /* E4M3 value (4 significant bits) times the fp32 scale is
                   exact in binary64; the cast rounds it once to binary32 */
                w[i] = (float)(oracle_e4m3_value(q) * (double)sc);
                if (!isfinite(w[i]))
                    return -3;
                if (fabs((double)w[i]) > amax)
                    amax = fabs((double)w[i]);
            }
            const int e = oracle_mx_exponent(amax, qmax);
            const int64_t b = r * (cols / 32) + j;
            scales[b] = (uint8_t)(e + 127);
            for (int i = 0; i < 32; ++i) {
                const double y = ldexp((double)w[i], -e);      /* exact */
                if (fmt == 1) {
                    const unsigned cc = oracle_e2m1_encode(y) & 0xFu;
                    if (i & 1)
                        codes[b * 16 + i / 2] |= (uint8_t)(cc << 4);
                    else
                        codes[b * 16 + i / 2] = (uint8_t)cc;
                } else {
                    codes[b * 32 + i] = (uint8_t)oracle_e4m3_encode(y);
                }
            }
        }
    }
    return 0;
}

/* Dequantize and measure the relative error of every unstacked tensor
 * [P3 metric table: relative error of quantized experts vs the bf16
 * source; P2 "The shared expert": error against the bf16 master].
 *   tensors t = 0..n_tensors-1, each [rows, cols], stored back to back;
 *   NVFP4 (fmt 0): deq = q * D * s2[t / tensors_per_scale] (so the gate
 *   and up halves of a fused slab read the same weight_scale_2);
 *   MXFP4 / MXFP8: deq = q * 2^(b - 127).
 * sum_sq_err[t] = sum (x - deq)^2, sum_sq_ref[t] = sum x^2, both as
 * binary64 sums in element order.  Returns 0 or -1. */
int oracle_dequant_relerr(const uint16_t *x, const uint8_t *codes,
                          const uint8_t *scales, const float *s2, int fmt,
                          int64_t n_tensors, int64_t rows, int64_t cols,
                          int64_t tensors_per_scale, double *sum_sq_err,
                          double *sum_sq_ref)
{
    const int blk = (fmt == 0) ? 16 : 32;
    if (n_tensors < 0 || rows < 0 || cols < 0 || cols % blk != 0 ||
        fmt < 0 || fmt > 2 || (fmt == 0 && tensors_per_scale < 1))
        return -1;
    const int64_t tsize = rows * cols;
    for (int64_t t = 0; t < n_tensors; ++t) {
        double err = 0.0, ref = 0.0;
        for (int64_t i = 0; i < tsize; ++i) {
            int64_t gi = t * tsize + i;
            double xv = (double)bf16_to_float(x[gi]);
            double deq;
            if (fmt == 2) {
                deq = oracle_e4m3_value(codes[gi]) *
                      oracle_ue8m0_value(scales[gi / 32]);
            } else {
                uint8_t byte = codes[gi / 2];
                unsigned c = (gi & 1) ? (byte >> 4) : (byte & 0xFu);
                double q = oracle_e2m1_value(c);
                if (fmt == 1)
                    deq = q * oracle_ue8m0_value(scales[gi / 32]);
                else
                    deq = q * oracle_e4m3_value(scales[gi / 16]) *
                          (double)s2[t / tensors_per_scale];
            }
            double e = xv - deq;
            err += e * e;
            ref += xv * xv;
        }
        sum_sq_err[t] = err;
        sum_sq_ref[t] = ref;
    }
    return 0;
}
