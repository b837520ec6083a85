/* Exhaustive check of the quantize kernels' bf16 quotient (test only).
 *
 * For a tile with bf16 maximum amax, the kernels compute s = RN32(amax/448)
 * and r = RN32(1/s), and encode a bf16 element x, through n = -x, as
 *     q0 = RN32(n (-r)),  t = RN32(q0 s + n)  (FMA),  q1 = RN32(t (-r) + q0)  (FMA)
 * instead of the IEEE quotient RN32(x/s).  The method fixes the code as
 * E4M3_RNE_satfinite(RN32(x/s)) (codingmall.com "Kan du förklara rollen för
 * FP8 precision i träningsprocessen för DeepSeek-V3", "Online-kvantisering").
 * This program walks every positive finite bf16 amax whose s lies in
 * [2^-100, 2^125] and every bf16 x with |x| <= amax, both signs and both
 * zeros, and counts the elements whose two codes differ; codes are taken
 * from the oracle's encoder.  It prints "pairs N mismatches M" and exits
 * non-zero if M > 0.  With --uncorrected the code is taken from q0 alone.
 * Built with -ffp-contract=off so that each line below is one IEEE
 * operation. */
#include <math.h>
#include <stdint.h>
#include <stdio.h>
#include <string.h>

#include "fp8_oracle.h"

static float bf16_to_float(uint32_t h) {
    const uint32_t u = h << 16;
    float f;
    memcpy(&f, &u, 4);
    return f;
}

static uint32_t float_bits(float f) {
    uint32_t u;
    memcpy(&u, &f, 4);
    return u;
}

int main(int argc, char** argv) {
    const int only_q0 = argc > 1 && strcmp(argv[1], "--uncorrected") == 0;
    long long pairs = 0, mismatches = 0;
#pragma omp parallel for schedule(dynamic, 64) reduction(+ : pairs, mismatches)
    for (int ha = 1; ha < 0x7F80; ++ha) {
        const float amax = bf16_to_float((uint32_t)ha);
        float s = amax / 448.0f;
        if (s == 0.0f) s = 1.0f;
        if (!(s >= 0x1p-100f && s <= 0x1p125f)) continue;
        const float r = 1.0f / s;
        for (int sign = 0; sign < 2; ++sign) {
            for (int hx = 0; hx <= ha; ++hx) {
                const float x = bf16_to_float((uint32_t)hx | (sign ? 0x8000u : 0u));
                const float n = -x;
                const float q0 = n * -r;
                const float t = fmaf(q0, s, n);
                const float q1 = only_q0 ? q0 : fmaf(t, -r, q0);
                const float ref = x / s;
                ++pairs;
                if (float_bits(q1) != float_bits(ref) &&
                    orc_e4m3_encode(q1) != orc_e4m3_encode(ref))
                    ++mismatches;
            }
        }
    }
    printf("pairs %lld mismatches %lld\n", pairs, mismatches);
    return mismatches != 0;
}
