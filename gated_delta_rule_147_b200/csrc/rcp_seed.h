/*
 * Reciprocal of a positive normal float by Newton-Raphson from a bit-pattern
 * seed, in plain C so the same routine builds for the device (it runs on the
 * FMA pipe instead of the special-function unit) and for a host-side check.
 *
 * Seed. For a = 2^e (1 + m), 0 <= m < 1, the float's bit pattern read as an
 * integer is I(a) = 2^23 (127 + e + m). The seed y0 = float(K - I(a)) with
 * K = 2^23 (254 - d) is, for m <= 1 - d, y0 = 2^(-e-1) (2 - d - m), so
 * a y0 = (1 + m)(2 - d - m) / 2. Over m this product is smallest at m = 0,
 * (2 - d) / 2, and largest at m = (1 - d) / 2, (3 - d)^2 / 8 (for m > 1 - d the
 * borrow into the exponent keeps it between those values). The two extremes
 * sit symmetrically around 1 when d^2 - 10 d + 1 = 0, d = 5 - 2 sqrt(6) =
 * 0.1010205, and the seed's relative error is then at most d / 2 = 5.06%.
 * K = round(2^23 (254 - d)) = 0x7EF311C3.
 *
 * Steps. x <- x (2 - a x) maps a relative error r to r^2: 2.6e-3, 6.5e-6, then
 * below fp32 rounding after the third step.
 */
#ifndef GDR_RCP_SEED_H
#define GDR_RCP_SEED_H

#include <stdint.h>
#include <string.h>

#ifdef __CUDACC__
#define GDR_RCP_FN __host__ __device__ __forceinline__
#else
#include <math.h>
#define GDR_RCP_FN static inline
#endif

#define GDR_RCP_SEED_K 0x7EF311C3u

GDR_RCP_FN float gdr_rcp_seed(float a) {
    uint32_t u;
    memcpy(&u, &a, sizeof(u));
    u = GDR_RCP_SEED_K - u;
    float x;
    memcpy(&x, &u, sizeof(x));
    return x;
}

GDR_RCP_FN float gdr_rcp_newton3(float a) {
    float x = gdr_rcp_seed(a);
    x = x * fmaf(-a, x, 2.f);
    x = x * fmaf(-a, x, 2.f);
    x = x * fmaf(-a, x, 2.f);
    return x;
}

#endif
