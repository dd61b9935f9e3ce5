/*
 * CPU checks of the arithmetic shortcuts the CUDA kernels take (test
 * infrastructure).  Each mode restates one shortcut in plain C, compares it
 * with the definition it replaces, and prints the number of cases and of
 * mismatches.  The shortcuts, as the kernels' own comments state them:
 *
 *   ue8m0  <fmax>        UE8M0 byte without a division: for FMAX = 448 the
 *                        byte is E(amax) - 8 + [mantissa(amax) > 0x600000],
 *                        for FMAX = 6 it is E(amax) - 2 + [mantissa > 0x400000];
 *                        the definition is the biased exponent of
 *                        fp32(amax / FMAX), plus one for a nonzero mantissa.
 *   cdiv   <c>           RN(a / c) for c in {448, 127, 6} by q = a * RN(1/c)
 *                        and two Markstein corrections with exact FMA residuals.
 *   hard   <bits> <kind> the same comparison on the cases where it can fail:
 *                        for every significand of x and every rounding
 *                        midpoint M of the code (between two E4M3 values, or
 *                        k + 1/2 for INT8), the 65 fp32 values of s nearest to
 *                        x / M, so that x / s lies within a few ulps of M.
 *   steps  <bits> <kind> the codes of x / s after ONE Markstein correction
 *                        (q = x*y, r = x - q*s, q += r*y with y = RN(1/s))
 *                        against the codes of the correctly rounded x / s, for
 *                        x with a <bits>-bit significand (8 bf16, 11 fp16),
 *                        every fp32 significand of s, and every binade of x/s
 *                        that can give a nonzero code; kind 0 = E4M3 (the
 *                        quotient carried negated, as the kernel does), 1 = INT8.
 *
 *   divsegs [<stride> <dmin> <dmax>]
 *                        s / segs by umulhi(s, magic) >> shift with l =
 *                        ceil(log2 segs), magic = ceil(2^(31+l) / segs), shift =
 *                        l - 1 (segs == 1: s itself), against the division, for
 *                        every segs in [dmin, dmax] (default 1 .. 2^20) and, per
 *                        segs, the s < 2^31 next to every quotient boundary at
 *                        both ends of the range plus pseudo-random s.
 *
 * A <stride> > 1 checks every stride-th case only.  Build:
 * gcc -O2 -mfma -fopenmp -ffp-contract=off kernel_arith.c -lm
 * (fmaf must be a true fused multiply-add; -ffp-contract=off keeps every
 * other operation rounded on its own).
 *
 * References: P. Markstein, "Computation of elementary functions on the IBM
 * RISC System/6000 processor", IBM J. Res. Dev. 34(1), 1990 (the correction
 * step); the OCP 8-bit floating point specification (E4M3).
 */
#include <math.h>
#include <stdint.h>
#include <stdio.h>
#include <stdlib.h>
#include <string.h>

static uint32_t bits_of(float f) { uint32_t b; memcpy(&b, &f, 4); return b; }
static float float_of(uint32_t b) { float f; memcpy(&f, &b, 4); return f; }

/* ---- ue8m0 ---------------------------------------------------------- */
static int ue8m0_rule(float a, float fmax) {
    uint32_t b = bits_of(a / fmax);
    return (int)((b >> 23) & 0xFF) + ((b & 0x7FFFFF) != 0);
}
static int ue8m0_fast(float a, float fmax) {
    uint32_t b = bits_of(a);
    if (fmax == 448.0f) return (int)((b >> 23) & 0xFF) - 8 + ((b & 0x7FFFFF) > 0x600000u);
    return (int)((b >> 23) & 0xFF) - 2 + ((b & 0x7FFFFF) > 0x400000u);
}

/* ---- cdiv ----------------------------------------------------------- */
static float cdiv(float a, float c, float rc) {
    float q = a * rc;
    float r = fmaf(-q, c, a);
    q = fmaf(r, rc, q);
    r = fmaf(-q, c, a);
    return fmaf(r, rc, q);
}

/* ---- steps ---------------------------------------------------------- */
/* E4M3 code of a >= 0: nearest value, ties to the even mantissa, saturating
 * at 448 (written from the OCP definition). */
static int e4m3_code(double a) {
    if (a > 448.0) a = 448.0;
    int E = (a >= ldexp(1.0, -6)) ? ilogb(a) : -6;
    double quantum = ldexp(1.0, E - 3);
    double r = nearbyint(a / quantum) * quantum;
    if (r == 0.0) return 0;
    int Er = ilogb(r);
    if (Er < -6) return (int)(r / ldexp(1.0, -9));
    return ((Er + 7) << 3) | ((int)(r / ldexp(1.0, Er - 3)) - 8);
}

/* Codes of RN(x/s) and of the one-step quotient; 1 when they agree. */
static int same_code(float x, float s, int kind) {
    volatile float one = 1.0f;
    const float y = one / s, ny = -y;
    const float t = x / s;
    float q1;
    if (kind == 0) {
        float q = x * ny;
        float r = fmaf(q, s, x);
        q1 = -fmaf(r, ny, q);
        return e4m3_code(t) == e4m3_code(q1);
    }
    float q = x * y;
    float r = fmaf(q, -s, x);
    q1 = fmaf(r, y, q);
    return nearbyint(fmin(t, 127.0)) == nearbyint(fmin(q1, 127.0));
}

int main(int argc, char **argv) {
    if (argc < 2) { fprintf(stderr, "usage: ue8m0|cdiv|steps ...\n"); return 2; }
    long long bad = 0, n = 0;
    if (!strcmp(argv[1], "ue8m0") || !strcmp(argv[1], "cdiv")) {
        const float c = (float)atof(argv[2]);
        const long long stride = argc > 3 ? atoll(argv[3]) : 1;
        volatile float one = 1.0f;
        const float rc = one / c;
        const int is_ue8m0 = !strcmp(argv[1], "ue8m0");
        const uint32_t lo = bits_of(1e-10f), hi = 0x7F7FFFFFu;
#pragma omp parallel for schedule(static) reduction(+ : bad, n)
        for (long long u = lo; u <= (long long)hi; u += stride) {
            const float a = float_of((uint32_t)u);
            int same = is_ue8m0 ? ue8m0_rule(a, c) == ue8m0_fast(a, c)
                                : bits_of(cdiv(a, c, rc)) == bits_of(a / c);
            ++n;
            bad += !same;
        }
    } else if (!strcmp(argv[1], "hard")) {
        const int bits = atoi(argv[2]), kind = atoi(argv[3]);
        double mids[256];
        int nm = 0;
        if (kind == 0) {
            double prev = 0.0;
            for (int c = 1; c <= 0x7E; ++c) {          /* consecutive E4M3 values */
                const int e = c >> 3, m = c & 7;
                const double v = e ? ldexp(1.0 + m / 8.0, e - 7) : ldexp(m / 8.0, -6);
                mids[nm++] = (prev + v) / 2.0;
                prev = v;
            }
        } else {
            for (int k = 0; k < 127; ++k) mids[nm++] = k + 0.5;
        }
        const uint32_t X0 = 1u << (bits - 1), X1 = 1u << bits;
#pragma omp parallel for schedule(dynamic) reduction(+ : bad, n)
        for (int i = 0; i < nm; ++i) {
            for (uint32_t X = X0; X < X1; ++X) {
                /* s0 = x / M brought into [1, 2) by scaling x and s together */
                const double x0 = ldexp((double)X, -(bits - 1));
                const double s0 = x0 / mids[i];
                const int m = -ilogb(s0);
                const float x = (float)ldexp(x0, m);
                float s = (float)ldexp(s0, m);
                for (int j = 0; j < 32; ++j) s = nextafterf(s, 0.0f);
                for (int j = 0; j <= 64; ++j, s = nextafterf(s, 4.0f)) {
                    ++n;
                    bad += !same_code(x, s, kind);
                }
            }
        }
    } else if (!strcmp(argv[1], "steps")) {
        const int bits = atoi(argv[2]), kind = atoi(argv[3]);
        const long long stride = argc > 4 ? atoll(argv[4]) : 1;
        const int lo_k = kind == 0 ? -12 : -3, hi_k = kind == 0 ? 9 : 7;
        const uint32_t X0 = 1u << (bits - 1), X1 = 1u << bits;
#pragma omp parallel for schedule(dynamic, 64) reduction(+ : bad, n)
        for (long long S = 1ll << 23; S < (1ll << 24); S += stride) {
            const float s = ldexpf((float)S, -23);
            volatile float one = 1.0f;
            const float y = one / s, ny = -y;
            for (int k = lo_k; k <= hi_k; ++k) {
                for (uint32_t X = X0; X < X1; ++X) {
                    const float x = ldexpf((float)X, k - (bits - 1));
                    const float t = x / s;
                    float q1;
                    if (kind == 0) {
                        float q = x * ny;
                        float r = fmaf(q, s, x);
                        q1 = -fmaf(r, ny, q);
                    } else {
                        float q = x * y;
                        float r = fmaf(q, -s, x);
                        q1 = fmaf(r, y, q);
                    }
                    int same = kind == 0
                                   ? e4m3_code(t) == e4m3_code(q1)
                                   : nearbyint(fmin(t, 127.0)) == nearbyint(fmin(q1, 127.0));
                    ++n;
                    bad += !same;
                }
            }
        }
    } else if (!strcmp(argv[1], "divsegs")) {
        const long long stride = argc > 2 ? atoll(argv[2]) : 1;
        const long long dmin = argc > 3 ? atoll(argv[3]) : 1;
        const long long dmax = argc > 4 ? atoll(argv[4]) : (1ll << 20);
#pragma omp parallel for schedule(dynamic, 256) reduction(+ : bad, n)
        for (long long d = dmin; d <= dmax; d += stride) {
            uint32_t magic = 0, shift = 0;
            if (d > 1) {
                uint32_t l = 0;
                while ((1ull << l) < (unsigned long long)d) ++l;
                magic = (uint32_t)(((1ull << (31u + l)) + (unsigned long long)d - 1u) / (unsigned long long)d);
                shift = l - 1u;
            }
            const uint32_t top = 0x7FFFFFFFu;
            uint64_t x = 0x9E3779B97F4A7C15ull ^ (uint64_t)d;
            for (int i = 0; i < 200; ++i) {
                uint32_t s;
                if (i < 64) {                        /* around the lowest boundaries */
                    s = (uint32_t)((i / 2) * d + (i % 2 ? d - 1 : 0));
                } else if (i < 128) {                /* around the highest ones */
                    const uint64_t k = top / (uint64_t)d - (uint64_t)((i - 64) / 2);
                    const uint64_t v = k * (uint64_t)d + ((i % 2) ? (uint64_t)d - 1 : 0);
                    s = (uint32_t)(v > top ? top : v);
                } else {                             /* pseudo-random */
                    x ^= x << 13; x ^= x >> 7; x ^= x << 17;
                    s = (uint32_t)(x & top);
                }
                const uint32_t q = magic == 0u ? s
                                   : (uint32_t)(((uint64_t)s * magic) >> 32) >> shift;
                ++n;
                bad += q != s / (uint32_t)d;
            }
        }
    } else {
        return 2;
    }
    printf("%lld %lld\n", n, bad);
    return 0;
}
