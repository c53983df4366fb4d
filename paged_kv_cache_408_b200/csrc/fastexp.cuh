// fastexp.cuh -- base-2 exponential on the FMA pipe, for softmax kernels
// that would otherwise be bound by the MUFU unit (16 ex2 per clock per SM on
// sm_100, the same rate a 128-wide tcgen05 tile consumes scores at when
// head_dim is 128).
//
// Method: x = n + f with n = round-to-nearest(x), so f lies in [-1/2, 1/2]
// (an exact split for base 2); 2^f from the degree-3 minimax polynomial of
// exp2_poly.h (Remez fit of the relative error, 7.5e-5, coefficients written
// by exp2_poly_fit.py); 2^n applied by adding n to the exponent field.
// n is obtained by adding 1.5 * 2^23: the fp32 sum rounds x to an integer
// and holds n in its low mantissa bits, so (bits << 23) is n << 23 in two's
// complement.  x is clamped to >= -120 first, which keeps the exponent
// arithmetic in the normal range: arguments below give 2^-120 instead of 0
// (masked scores are -inf), a weight 120 binades below the row maximum.
// The caller keeps x below 2^22 (a softmax argument is at most a few units
// above 0).  Two lanes at a time with packed fp32x2 adds and FMAs.
#pragma once

#include "common.cuh"
#include "exp2_poly.h"

namespace pa {

PA_DEVICE float2 exp2_fma2(float2 x) {
    constexpr float kRound = 12582912.0f;  // 1.5 * 2^23
    x = make_float2(fmaxf(x.x, -120.f), fmaxf(x.y, -120.f));
    const float2 t = fadd2(x, make_float2(kRound, kRound));       // 1.5*2^23 + n
    const float2 n = fadd2(t, make_float2(-kRound, -kRound));     // n, exactly
    const float2 f = fadd2(x, make_float2(-n.x, -n.y));           // in [-1/2, 1/2], exactly
    float2 p = ffma2(make_float2(kExp2Poly3, kExp2Poly3), f, make_float2(kExp2Poly2, kExp2Poly2));
    p = ffma2(p, f, make_float2(kExp2Poly1, kExp2Poly1));
    p = ffma2(p, f, make_float2(kExp2Poly0, kExp2Poly0));
    return make_float2(__uint_as_float(__float_as_uint(p.x) + (__float_as_uint(t.x) << 23)),
                       __uint_as_float(__float_as_uint(p.y) + (__float_as_uint(t.y) << 23)));
}

}  // namespace pa
