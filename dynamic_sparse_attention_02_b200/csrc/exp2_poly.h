// exp2_poly.h -- 2^x on the FMA pipe, for part of the softmax exponentials.
//
// Method: Cody-Waite style range reduction x = n + f with n = round-to-nearest
// (adding 1.5 * 2^23 in fp32 puts n in the low mantissa bits, and f = x - n is
// exact, |f| <= 1/2), then 2^f by a degree-3 polynomial whose coefficients
// minimise the maximum relative error on [-1/2, 1/2] (Remez exchange, fitted
// for this library by fit_exp2.py beside this header, which prints these
// constants: max relative error 7.5e-5, well below the 3.9e-3
// rounding of the bf16 probabilities it feeds), and 2^n by adding n to the
// exponent field.  Arguments are clamped at -126.5 so that n >= -126 and the
// exponent never wraps; a clamped argument yields at most a denormal, which
// the flush-to-zero row sum treats as 0.
#pragma once

namespace minfer {

constexpr float kExp2C0 = 0x1.fff692p-1f;
constexpr float kExp2C1 = 0x1.62f31ap-1f;
constexpr float kExp2C2 = 0x1.f0de1ap-3f;
constexpr float kExp2C3 = 0x1.c3f76p-5f;
constexpr float kExp2Clamp = -126.5f;
constexpr float kExp2Round = 12582912.0f;  // 1.5 * 2^23

}  // namespace minfer
