// exp2_poly.h -- written by exp2_poly_fit.py (do not edit): the degree-3
// polynomial p(f) ~ 2^f on [-1/2, 1/2] with minimax relative error (Remez
// exchange), coefficients rounded to fp32.  Levelled relative error of the
// exact polynomial 7.478e-05; of the fp32 Horner evaluation 7.484e-05.
#pragma once

namespace pa {

constexpr float kExp2Poly0 = 0.9999280571937561f;  // 0x1.fff6920000000p-1
constexpr float kExp2Poly1 = 0.6932609677314758f;  // 0x1.62f31a0000000p-1
constexpr float kExp2Poly2 = 0.2426111251115799f;  // 0x1.f0de1a0000000p-3
constexpr float kExp2Poly3 = 0.0551716685295105f;  // 0x1.c3f7600000000p-5

}  // namespace pa
