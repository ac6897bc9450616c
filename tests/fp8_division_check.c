/* Exhaustive host check of the FP8 quantiser's division.
 *
 * The quantiser divides every element x of a 128-channel block by the
 * block's scale s = amax / 448 (binary32, round to nearest even) and
 * converts the quotient to E4M3.  The device computes the quotient as
 * Markstein's corrected reciprocal product (P. Markstein, "Computation of
 * elementary functions on the IBM RISC System/6000 processor", IBM J. Res.
 * Dev. 34(1), 1990):
 *     r = RN(1 / s),  q0 = RN(x r),  e = RN(x - q0 s) (one FMA, exact),
 *     q = RN(q0 + e r) (one FMA), with the sign of x,
 * for scales s >= 2^-100 (finite), and IEEE division otherwise.
 *
 * This program restates those steps in C (binary32 arithmetic, fmaf) and
 * compares q with IEEE division x / s for EVERY pair of 16-bit values
 * (amax, x) of one input format with amax > 0 finite and |x| <= amax, both
 * signs of x.  A pair passes when the binary32 quotients are identical, or
 * when both have magnitude <= 2^-10 and the sign of x (every such value
 * converts to the E4M3 zero of that sign: 2^-10 is half the smallest E4M3
 * subnormal and ties go to the even code, zero).
 *
 * usage: fp8_division_check bf16|fp16 [nocorr]
 *   nocorr: drop the correction (q = q0) -- the check must then fail.
 * Prints one line: "<fmt> pairs P fast F zero_equiv Z ieee I bad B". */
#include <float.h>
#include <math.h>
#include <stdint.h>
#include <stdio.h>
#include <string.h>

#if !defined(FLT_EVAL_METHOD) || FLT_EVAL_METHOD != 0
#error "binary32 expressions must be evaluated in binary32"
#endif

static float from_bits(uint32_t b)
{
    float f;
    memcpy(&f, &b, sizeof f);
    return f;
}

static uint32_t to_bits(float f)
{
    uint32_t b;
    memcpy(&b, &f, sizeof b);
    return b;
}

/* bfloat16: the upper half of a binary32. */
static float bf16_value(uint32_t h) { return from_bits(h << 16); }

/* binary16: 1 sign, 5 exponent (bias 15), 10 fraction bits; finite only. */
static float fp16_value(uint32_t h)
{
    const int e = (int)((h >> 10) & 31u), m = (int)(h & 1023u);
    const float v = e == 0 ? ldexpf((float)m, -24) : ldexpf((float)(1024 + m), e - 25);
    return (h & 0x8000u) ? -v : v;
}

int main(int argc, char** argv)
{
    if (argc < 2 || (strcmp(argv[1], "bf16") && strcmp(argv[1], "fp16"))) {
        fprintf(stderr, "usage: %s bf16|fp16 [nocorr]\n", argv[0]);
        return 2;
    }
    const int half = strcmp(argv[1], "fp16") == 0;
    const int nocorr = argc > 2 && strcmp(argv[2], "nocorr") == 0;
    /* largest positive finite encoding: bf16 0x7f7f, fp16 0x7bff */
    const int top = half ? 0x7bff : 0x7f7f;
    long long pairs = 0, fast = 0, zero_equiv = 0, ieee = 0, bad = 0;
    int shown = 0;

#pragma omp parallel for schedule(dynamic, 64) reduction(+ : pairs, fast, zero_equiv, ieee, bad)
    for (int a = 1; a <= top; ++a) {
        const float amax = half ? fp16_value((uint32_t)a) : bf16_value((uint32_t)a);
        const float s = amax / 448.0f;
        const long long n = 2LL * (a + 1); /* x in [-amax, amax]: encodings 0..a, both signs */
        pairs += n;
        if (!(s >= 0x1p-100f && s <= FLT_MAX)) {
            ieee += n;
            continue;
        }
        fast += n;
        const float r = 1.0f / s;
        long long bad_here = 0;
        float first_x = 0.0f, first_exact = 0.0f, first_q = 0.0f;
        for (int b = 0; b <= a; ++b) {
            for (int neg = 0; neg < 2; ++neg) {
                const uint32_t hb = (uint32_t)b | (neg ? 0x8000u : 0u);
                const float x = half ? fp16_value(hb) : bf16_value(hb);
                const float exact = x / s;
                const float q0 = x * r;
                const float e = fmaf(-q0, s, x);
                const float q = copysignf(nocorr ? q0 : fmaf(e, r, q0), x);
                if (to_bits(q) == to_bits(exact))
                    continue;
                if (fabsf(q) <= 0x1p-10f && fabsf(exact) <= 0x1p-10f &&
                    (signbit(q) != 0) == (neg != 0) && (signbit(exact) != 0) == (neg != 0)) {
                    ++zero_equiv;
                    continue;
                }
                if (bad_here++ == 0) {
                    first_x = x;
                    first_exact = exact;
                    first_q = q;
                }
            }
        }
        if (bad_here) {
            bad += bad_here;
#pragma omp critical
            if (shown < 5) {
                ++shown;
                fprintf(stderr, "mismatch: amax %a x %a s %a: ieee %a, corrected %a\n",
                        (double)amax, (double)first_x, (double)s, (double)first_exact,
                        (double)first_q);
            }
        }
    }
    printf("%s pairs %lld fast %lld zero_equiv %lld ieee %lld bad %lld\n", argv[1], pairs, fast,
           zero_equiv, ieee, bad);
    return bad == 0 ? 0 : 1;
}
