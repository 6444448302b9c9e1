// A software 2^x, kept with its self-test entry point (pv_selftest_exp2_poly).
// Computing a share of the softmax exponentials with it instead of the XU
// pipe measured slower at every share tried, so the attention kernel does not
// use it; it stays tested against exp2f for when the balance of the pipes
// changes.
#pragma once

#include <stdint.h>

namespace pv {

// 2^x on the FMA and ALU pipes, to take part of the exponentials off the
// XU (ex2) pipe.  Range reduction in the manner of Cody and Waite: n =
// round(x) by the 1.5 * 2^23 addition trick, f = x - n in [-1/2, 1/2]; 2^f
// by the minimax cubic that exp2_poly_fit.py fits (max relative error
// 7.5e-5, far below the 2^-9 of the bf16 rounding that follows); 2^n by
// adding n to the exponent field.  Valid for x in [-125, 128); smaller x is
// clamped (the result is then below 2^-124 of the row sum, and the
// exponent field never reaches the denormal range).
__device__ __forceinline__ float exp2_poly(float x) {
    constexpr float kC0 = 9.999280572e-01f;
    constexpr float kC1 = 6.932609677e-01f;
    constexpr float kC2 = 2.426111251e-01f;
    constexpr float kC3 = 5.517166853e-02f;
    constexpr float kRound = 12582912.0f;  // 1.5 * 2^23
    x = fmaxf(x, -125.0f);
    const float t = x + kRound;
    const float f = x - (t - kRound);
    const float p = fmaf(fmaf(fmaf(kC3, f, kC2), f, kC1), f, kC0);
    return __int_as_float(__float_as_int(p) + (__float_as_int(t) << 23));
}

}  // namespace pv
