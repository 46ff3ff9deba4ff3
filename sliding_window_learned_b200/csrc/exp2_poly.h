// exp2_poly.h -- written by gen_exp2_poly.py; do not edit.
// 2^f ~ c0 + c1 f + c2 f^2 + c3 f^3 on f in [-1/2, 1/2]: weighted least-squares
// fit on Chebyshev nodes (relative error), after Cody-Waite reduction x = n + f.
// measured max relative error (float32 Horner): 7.738e-05
#pragma once
namespace attnsink {
constexpr float kExp2C0 = 0.9999289512634277f;
constexpr float kExp2C1 = 0.6932762265205383f;
constexpr float kExp2C2 = 0.24260404706001282f;
constexpr float kExp2C3 = 0.05508868396282196f;
constexpr float kExp2PolyMaxRelErr = 7.738e-05f;
}  // namespace attnsink
