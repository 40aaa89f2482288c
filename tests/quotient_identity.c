/* Exhaustive check of the division-free quotient used by the quantize kernel
 * (quantize_stream_kernel in w4a16_bit_gemm_b200/csrc/quantize.cu):
 *
 *   rcp = rn(1/s); q0 = rn(x * rcp); r = fma(-q0, s, x); q1 = fma(r, rcp, q0)
 *   t = rn(q1 + 1.5*2^23)                      (round half to even)
 *
 * For every finite bf16 x and every positive finite fp16 s with |x/s| <= 40
 * (the codes' range, with margin), t - 1.5*2^23 must equal rint(fl(x/s)), the
 * round-half-to-even of the IEEE fp32 quotient.  Plain C99 on the host: IEEE
 * binary32 arithmetic, fmaf correctly rounded, no contraction.  Prints the
 * number of pairs checked and of mismatches; exits 1 on any mismatch. */
#include <math.h>
#include <stdint.h>
#include <stdio.h>
#include <string.h>

static float bits_to_float(uint32_t u) {
    float f;
    memcpy(&f, &u, 4);
    return f;
}

static float fp16_value(uint32_t h) { /* positive fp16 bits -> float */
    const int e = (int)((h >> 10) & 31), m = (int)(h & 1023);
    return e == 0 ? ldexpf((float)m, -24) : ldexpf((float)(m | 1024), e - 25);
}

int main(void) {
    const float magic = 12582912.0f; /* 1.5 * 2^23 */
    long long pairs = 0, bad = 0;
#pragma omp parallel for schedule(dynamic, 64) reduction(+ : pairs, bad)
    for (int h = 1; h < 0x7c00; ++h) {
        const float s = fp16_value((uint32_t)h);
        const float rcp = 1.0f / s;
        for (uint32_t b = 0; b < 0x10000u; ++b) {
            const float x = bits_to_float(b << 16);
            if (!isfinite(x)) continue;
            const float q = x / s;
            if (!(fabsf(q) <= 40.0f)) continue;
            const float q0 = x * rcp;
            const float r = fmaf(-q0, s, x);
            const float q1 = fmaf(r, rcp, q0);
            const float t = q1 + magic;
            ++pairs;
            if (t - magic != rintf(q)) {
                ++bad;
            }
        }
    }
    printf("pairs %lld mismatches %lld\n", pairs, bad);
    return bad != 0;
}
