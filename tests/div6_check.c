/* Host check of div6 (bit_quantized_attention_sa3_b200/csrc/quant.cuh), run
 * by tests/test_div6.py.  The quantizer forms each block's E4M3 scale from
 * fp32(amax / 6) with div6 instead of a division.  For every non-negative
 * fp32 x (inf included): either div6(x) is bit-identical to the IEEE
 * quotient x / 6, or both are below 2^-10 (E4M3 code 0 after
 * round-to-nearest), or x is inf and both are at least 448 (the saturated
 * code).  The formula is restated here because quant.cuh is device code;
 * test_div6.py checks that the two texts agree. */
#include <math.h>
#include <stdint.h>
#include <stdio.h>
#include <string.h>

static float f_of(uint32_t u) { float f; memcpy(&f, &u, 4); return f; }
static uint32_t u_of(float f) { uint32_t u; memcpy(&u, &f, 4); return u; }

static float div6(float x) {
    x = fminf(x, 0x1.fffffep127f);
    return fmaf(x, 0x1.555556p-3f, x * -0x1.555556p-28f);
}

int main(void) {
    uint64_t exact = 0, tiny = 0;
    for (uint64_t i = 0; i <= 0x7f800000u; ++i) {
        const float x = f_of((uint32_t)i);
        const float want = x / 6.0f, got = div6(x);
        if (u_of(got) == u_of(want)) { ++exact; continue; }
        if (want < 0x1p-10f && got >= 0.0f && got < 0x1p-10f) { ++tiny; continue; }
        if (isinf(x) && got >= 448.0f && want >= 448.0f) continue;
        printf("x = %a: div6 %a, x / 6 %a\n", x, got, want);
        return 1;
    }
    printf("ok exact %llu tiny %llu\n", (unsigned long long)exact, (unsigned long long)tiny);
    return 0;
}
