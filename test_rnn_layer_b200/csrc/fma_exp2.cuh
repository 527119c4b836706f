// 2^x on the FMA pipe (for kernels whose exponential unit, 16 results per
// cycle per SM, is the scarce resource).
//
// x = n + f with n = rint(x), read from the low mantissa bits of x + 1.5 * 2^23
// (valid for |x| < 2^22), and f = x - n in [-1/2, 1/2]; 2^f from a polynomial
// whose coefficients are a least-squares fit of 2^f on [-1/2, 1/2] weighted for
// equal relative error (Lawson's iteration); then 2^n is added to the exponent
// field: the bits of x + 1.5 * 2^23 shifted left by 23 are n << 23 (the shift
// drops the bits of 1.5 * 2^23).  Inputs below -125 give 2^-125 (times the
// polynomial's value at 0); NaN stays NaN.  Maximum relative error in fp32
// over [-125, 8]: cubic 7.6e-5, quartic 2.7e-6 (tests/test_attention_exp2_poly.py).
#pragma once

#include <stdint.h>

namespace ttt {
namespace fexp {

constexpr float kShift = 12582912.0f;   // 1.5 * 2^23
// cubic coefficients of f^0 .. f^3, quartic coefficients of f^0 .. f^4
constexpr float kC3_0 = 0.9999281764030457f, kC3_1 = 0.6932609677314758f, kC3_2 = 0.24260970950126648f,
                kC3_3 = 0.05517097935080528f;
constexpr float kC4_0 = 0.9999992847442627f, kC4_1 = 0.6931218504905701f, kC4_2 = 0.240247443318367f,
                kC4_3 = 0.05591771379113197f, kC4_4 = 0.009570036083459854f;

__device__ __forceinline__ float clamp_low(float x) { return x < -125.0f ? -125.0f : x; }   // NaN stays NaN

__device__ __forceinline__ float scale_by_rint(float p, float t) {
    return __int_as_float(__float_as_int(p) + (__float_as_int(t) << 23));
}

// cubic: relative error 7.6e-5
__device__ __forceinline__ float ex2_fma3(float x) {
    x = clamp_low(x);
    const float t = x + kShift;
    const float f = x - (t - kShift);
    float p = fmaf(kC3_3, f, kC3_2);
    p = fmaf(p, f, kC3_1);
    p = fmaf(p, f, kC3_0);
    return scale_by_rint(p, t);
}

// quartic: relative error 2.7e-6
__device__ __forceinline__ float ex2_fma4(float x) {
    x = clamp_low(x);
    const float t = x + kShift;
    const float f = x - (t - kShift);
    float p = fmaf(kC4_4, f, kC4_3);
    p = fmaf(p, f, kC4_2);
    p = fmaf(p, f, kC4_1);
    p = fmaf(p, f, kC4_0);
    return scale_by_rint(p, t);
}

}  // namespace fexp
}  // namespace ttt
