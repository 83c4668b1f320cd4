/*
 * Host-side checks of two exact-arithmetic identities the quantizer kernels rely on.  This is
 * test code: it restates, operation by operation, the FP32 sequences of the device functions
 * div6_rn and e2m1_sr_code (nvfp4_device.cuh), so that their claims can be checked over far
 * more inputs than the GPU parity tests sample.  Built by the test with gcc -O2
 * -ffp-contract=off -frounding-math; every FP32 operation below is one IEEE-754 operation in
 * the rounding mode the device instruction uses.
 */
#include <fenv.h>
#include <math.h>
#include <stdint.h>
#include <string.h>

#pragma STDC FENV_ACCESS ON

static float f_of(uint32_t u) { float f; memcpy(&f, &u, 4); return f; }
static uint32_t u_of(float f) { uint32_t u; memcpy(&u, &f, 4); return u; }

/* div6_rn: correctly rounded b / 6 without a division.  Below 2^-125 the quotient's bit
 * pattern is the integer m / 6 rounded to nearest even (m the pattern of b, floor(m / 6) as
 * (m * 0xAAAAAAAB) >> 34); above it q0 = RN(b z), z = RN(1/6), the exact remainder
 * r = b - 6 q0 by one FMA, and RN(q0 + r z) by one FMA. */
static float div6_emul(float b)
{
    if (b < 0x1p-125f) {
        uint32_t m = u_of(b);
        uint32_t n = (uint32_t)(((uint64_t)m * 0xAAAAAAABull) >> 34);
        uint32_t rem = m - 6u * n;
        return f_of(n + ((rem > 3u || (rem == 3u && (n & 1u))) ? 1u : 0u));
    }
    const float z = 0x1.555556p-3f;
    float q0 = b * z;
    return fmaf(fmaf(-q0, 6.0f, b), z, q0);
}

/* Count of finite non-negative FP32 patterns in [lo, hi) where div6_emul(b) and the FPU's
 * b / 6 (round to nearest even) differ; the first such pattern goes to *first_bad. */
int64_t kid_div6_mismatches(uint32_t lo, uint32_t hi, uint32_t* first_bad)
{
    fesetround(FE_TONEAREST);
    int64_t bad = 0;
    for (uint32_t u = lo; u < hi; ++u) {
        float b = f_of(u);
        if (u_of(div6_emul(b)) != u_of(b / 6.0f)) {
            if (bad == 0) *first_bad = u;
            ++bad;
        }
    }
    return bad;
}

/* e2m1_sr_code: the magnitude code of a >= 0 stochastically rounded with the 16-bit random
 * integer r16, on the FMA pipe: the lines 2^17 a, 2^16 a + 2^17 and 2^15 a + 2^18, each plus
 * 2^23 and rounded upward by one FMA, and the constant 2^23 + 7 * 2^16; their minimum P;
 * Q = P - (2^23 + r16) (exact); k = RU(Q 2^-16 + 1.5 * 2^23); the code is the low byte of k's
 * pattern. */
static uint32_t sr_code_emul(float a, uint32_t r16)
{
    const float rbits = f_of(0x4B000000u | (r16 & 0xFFFFu)); /* 2^23 + r16 */
    fesetround(FE_UPWARD);
    float l0 = fmaf(a, 131072.0f, 8388608.0f);
    float l1 = fmaf(a, 65536.0f, 8519680.0f);
    float l2 = fmaf(a, 32768.0f, 8650752.0f);
    float P = fminf(fminf(fminf(l0, l1), l2), 8847360.0f);
    fesetround(FE_TONEAREST);
    float Q = P - rbits;
    fesetround(FE_UPWARD);
    float k = fmaf(Q, 0x1p-16f, 12582912.0f);
    fesetround(FE_TONEAREST);
    return u_of(k) & 0xFFu;
}

void kid_sr_codes(const float* a, const uint32_t* r16, int64_t n, uint8_t* out)
{
    for (int64_t i = 0; i < n; ++i) out[i] = (uint8_t)sr_code_emul(a[i], r16[i]);
    fesetround(FE_TONEAREST);
}
