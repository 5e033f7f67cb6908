// exp2_poly.cuh -- written by exp2_poly_fit.py; do not edit by hand.
// 2^r on [-1/2, 1/2], degree-3 minimax in relative error (Remez exchange),
// coefficients rounded to fp32.  Levelled relative error of the fit: 7.478e-05;
// max relative error of the full fp32 sequence over x in [-125, 8]: 7.484e-05.
#pragma once

namespace fa {
constexpr float kExp2C0 = 0.9999280571937561f;
constexpr float kExp2C1 = 0.6932609677314758f;
constexpr float kExp2C2 = 0.2426111251115799f;
constexpr float kExp2C3 = 0.0551716685295105f;
constexpr float kExp2MaxRelErr = 7.484e-05f;
}  // namespace fa
