// exp2_poly.h -- written by gen_exp2_poly.py; do not edit by hand.
// 2^f on [-1/2, 1/2] by a degree-3 polynomial, minimax in relative error
// (Remez exchange), coefficients rounded to float32.
// Max relative error on [-1/2, 1/2] with float32 coefficients: 7.480e-05
#pragma once
namespace wf {
constexpr int kExp2PolyDegree = 3;
constexpr float kExp2PolyRelErr = 7.479879442e-05f;
constexpr float kExp2C0 = 0.9999280571937561f;
constexpr float kExp2C1 = 0.6932609677314758f;
constexpr float kExp2C2 = 0.2426111251115799f;
constexpr float kExp2C3 = 0.0551716685295105f;
}  // namespace wf
