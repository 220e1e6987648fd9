/* Exhaustive check of the division by 6 that the NVFP4 encoder uses for its block scale:
 * for every finite fp32 a >= 2^-125, q0 = a * RN(1/6) corrected by one fused residual step,
 * q = fma(fma(-q0, 6, a), RN(1/6), q0), must equal the IEEE quotient a / 6 (round to nearest
 * even). Prints the number of inputs checked and of mismatches. Build with -ffp-contract=off. */
#include <math.h>
#include <stdint.h>
#include <stdio.h>
#include <string.h>

static float from_bits(uint32_t u) { float x; memcpy(&x, &u, 4); return x; }
static uint32_t to_bits(float x) { uint32_t u; memcpy(&u, &x, 4); return u; }

int main(void) {
    const float c = 1.0f / 6.0f;
    const uint32_t lo = to_bits(0x1p-125f), hi = 0x7F7FFFFFu;   /* largest finite float */
    unsigned long long checked = 0, bad = 0;
    for (uint32_t u = lo;; ++u) {
        const float a = from_bits(u);
        volatile float ref = a / 6.0f;
        const float q0 = a * c;
        const float q = fmaf(fmaf(-q0, 6.0f, a), c, q0);
        if (to_bits(q) != to_bits(ref)) ++bad;
        ++checked;
        if (u == hi) break;
    }
    printf("%llu %llu\n", checked, bad);
    return 0;
}
