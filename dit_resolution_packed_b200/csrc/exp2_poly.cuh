// exp2_poly.cuh -- written by fit_exp2_poly.py; do not edit by hand.
//
// 2^f ~ C0 + f*(C1 + f*(C2 + f*C3)) on |f| <= 1/2: degree-3 minimax fit of the
// relative error (Remez exchange), coefficients rounded to fp32.
// Max relative error of the fp32 evaluation (fused multiply-adds): 7.483e-05.
#pragma once

namespace pa {
constexpr float kExp2C0 = 0.9999280571937561f;
constexpr float kExp2C1 = 0.6932609677314758f;
constexpr float kExp2C2 = 0.2426111251115799f;
constexpr float kExp2C3 = 0.0551716685295105f;
constexpr float kExp2PolyMaxRelErr = 7.482753e-05f;
}  // namespace pa
