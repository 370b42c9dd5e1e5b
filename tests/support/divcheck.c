/* Checks, on a sample of non-negative finite fp32 values and on boundary
 * values, that dividing by the grid size d as
 *     q0 = fl(a * fl(1/d)),  rem = fma(-q0, d, a),  q = fma(rem, fl(1/d), q0)
 * gives the correctly rounded a / d (the library's refit uses this form).
 * Prints the number of mismatches; exit status 0 when there are none. */
#include <math.h>
#include <stdint.h>
#include <stdio.h>
#include <string.h>

static uint64_t s = 0x9E3779B97F4A7C15ull;
static uint32_t next(void) { s ^= s << 13; s ^= s >> 7; s ^= s << 17; return (uint32_t)s; }

static int check(float d, uint32_t u)
{
    float a, r = 1.0f / d;
    memcpy(&a, &u, 4);
    float q0 = a * r;
    float rem = fmaf(-q0, d, a);
    float q = fmaf(rem, r, q0);
    return q != a / d;
}

int main(void)
{
    const float ds[] = {255.f, 15.f, 127.f, 7.f};
    unsigned long long bad = 0;
    for (int k = 0; k < 4; ++k) {
        for (uint32_t u = 0; u < (1u << 24); ++u) bad += check(ds[k], u);          /* zero and subnormals */
        for (uint32_t e = 0; e < 255; ++e)                                         /* every binade's edges */
            for (uint32_t m = 0; m < 4096; ++m) {
                bad += check(ds[k], (e << 23) | m);
                bad += check(ds[k], (e << 23) | (0x7fffffu - m));
            }
        for (int i = 0; i < 20000000; ++i) bad += check(ds[k], next() & 0x7f7fffffu);
    }
    printf("%llu\n", bad);
    return bad != 0;
}
