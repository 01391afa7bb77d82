/* Exhaustive check of the quotient method the NVFP4 kernel uses for
 * y = RN32(x / d) with x a bf16 value and d any fp32 value:
 *     r  = RN32(1 / d)                  (correctly rounded reciprocal)
 *     q0 = RN32(x * r)
 *     e  = RN32(q0 * d - x)             (one FMA; exact)
 *     y  = RN32(q0 - e * r)             (one FMA)
 * which is the quotient-correction step of Markstein (IBM J. Res. Dev.
 * 34(1), 1990), written with the residual negated so that x = -0 keeps
 * its sign.  It is compared with the correctly rounded IEEE quotient over
 * every pair of significands: x in [1, 2) with 8 significant bits (all 128
 * bf16 significands) and d in [1, 2) with all 2^23 fp32 significands,
 * for both signs of x.  Every step scales exactly by powers of two while
 * its operands and results stay normal, so this covers every exponent
 * combination with normal intermediates.
 * Prints the number of mismatches (0 expected) and exits 1 on any. */
#include <math.h>
#include <stdint.h>
#include <stdio.h>
#include <string.h>

static float from_bits(uint32_t u) { float f; memcpy(&f, &u, 4); return f; }
static uint32_t to_bits(float f) { uint32_t u; memcpy(&u, &f, 4); return u; }

int main(void)
{
    long long bad = 0;
    #pragma omp parallel for reduction(+:bad) schedule(static)
    for (int k = 0; k < 128; ++k) {
        for (int s = 0; s < 2; ++s) {
            float x = from_bits(0x3F800000u | ((uint32_t)k << 16) | ((uint32_t)s << 31));
            for (uint32_t m = 0; m < (1u << 23); ++m) {
                float d = from_bits(0x3F800000u | m);
                float r = 1.0f / d;
                float q0 = x * r;
                float e = fmaf(q0, d, -x);
                float y = fmaf(-e, r, q0);
                float ref = x / d;
                if (to_bits(y) != to_bits(ref))
                    ++bad;
            }
        }
    }
    /* signed zeros keep their sign */
    float dz = 1.375f, rz = 1.0f / dz;
    for (int s = 0; s < 2; ++s) {
        float x = s ? -0.0f : 0.0f;
        float q0 = x * rz;
        float y = fmaf(-fmaf(q0, dz, -x), rz, q0);
        if (to_bits(y) != to_bits(x / dz))
            ++bad;
    }
    printf("mismatches %lld\n", bad);
    return bad ? 1 : 0;
}
