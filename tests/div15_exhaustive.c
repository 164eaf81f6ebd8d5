/* Exhaustive check of the quantizer's division by 15 for a known divisor
 * (Markstein's correction step: q0 = w * RN(1/15), rem = fma(-q0, 15, w),
 * q = fma(rem, RN(1/15), q0)) against IEEE division, over every positive normal
 * binary32 w. Prints the number of mismatches. */
#include <math.h>
#include <stdint.h>
#include <stdio.h>
#include <string.h>

int main(void)
{
    const float inv15 = 1.0f / 15.0f;
    long bad = 0;
#pragma omp parallel for reduction(+ : bad) schedule(static)
    for (int64_t u = 0x00800000; u < 0x7f800000; ++u) {
        uint32_t b = (uint32_t)u;
        float w;
        memcpy(&w, &b, 4);
        volatile float want = w / 15.0f;
        float q0 = w * inv15;
        float rem = fmaf(-q0, 15.0f, w);
        float q = fmaf(rem, inv15, q0);
        if (q != want)
            bad++;
    }
    printf("%ld\n", bad);
    return 0;
}
