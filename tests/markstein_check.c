/*
 * Exhaustive check of the division shortcut used by the GPU quantizer.
 *
 * The quantizer needs X^scaled = RN(x / d) (binary32, nearest-even) for every
 * element of a 16-element block that shares one divisor d.  The GPU computes
 * y = RN(1/d) once per block and then, per element,
 *     q  = RN(x * y)
 *     r  = fma(-q, d, x)          (exact remainder)
 *     q' = fma(r, y, q)
 * (Markstein, "Computation of elementary functions on the IBM RISC
 * System/6000 processor", IBM J. Res. Dev. 34(1), 1990).  This program checks
 * q' == RN(x / d) for EVERY x significand of an fp16 input (which includes
 * every bfloat16 significand) and EVERY binary32 significand of d, with both
 * in [1, 2).  Scaling x or d by a power of two scales every intermediate by
 * the same power of two, so the check covers all inputs whose intermediates
 * stay in the normal range; the quantizer takes the plain IEEE divide for the
 * rare blocks whose d lies outside [2^-90, 2^90].
 *
 * Build: gcc -O2 -ffp-contract=off -fopenmp -o markstein_check markstein_check.c -lm
 * Usage: markstein_check [stride]   (stride > 1 checks every stride-th d)
 * Prints the number of pairs checked and of mismatches; exit code 1 on any.
 */
#include <math.h>
#include <stdint.h>
#include <stdio.h>
#include <stdlib.h>
#include <string.h>

static float from_bits(uint32_t u)
{
    float f;
    memcpy(&f, &u, 4);
    return f;
}

int main(int argc, char **argv)
{
    long stride = argc > 1 ? atol(argv[1]) : 1;
    long long checked = 0, bad = 0;
#pragma omp parallel for schedule(dynamic, 4096) reduction(+ : checked, bad)
    for (long dm = 0; dm < (1L << 23); dm += stride) {
        float d = from_bits(0x3f800000u | (uint32_t)dm);
        volatile float one = 1.0f;
        float y = one / d;
        for (uint32_t xm = 0; xm < (1u << 10); xm++) {
            float x = from_bits(0x3f800000u | (xm << 13));
            float q = x * y;
            float r = fmaf(-q, d, x);
            float q2 = fmaf(r, y, q);
            float ref = x / d;
            checked++;
            if (q2 != ref) {
                bad++;
                if (bad < 10)
                    printf("mismatch x=%a d=%a got=%a want=%a\n", x, d, q2, ref);
            }
        }
    }
    printf("checked %lld pairs, %lld mismatches\n", checked, bad);
    return bad != 0;
}
