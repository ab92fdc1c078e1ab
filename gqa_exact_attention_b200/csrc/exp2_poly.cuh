// 2^x on the FMA and integer pipes (no special-function unit), for a share of the softmax
// exponentials so that they do not all queue on the MUFU.
//
// Method: Cody-Waite argument reduction x = j + f with j = rint(x), f in [-1/2, 1/2]
// (adding 1.5 * 2^23 rounds x to an integer held in the low mantissa bits of t), then a
// polynomial 2^f ~ 1 + f (c1 + f (c2 + f c3)) whose coefficients minimise the maximum
// relative error on [-1/2, 1/2] with the constant term held at exactly 1 (a minimax fit,
// computed by exp2_poly_fit.py in this directory as a linear program).  Max relative error
// 1.02e-4, against 2^-9 = 1.95e-3 for the bf16 rounding that P receives next.  2^j is then
// added to the exponent field.  Properties: 2^0 = 1 exactly, and 2^j is exact for every
// integer j in [-126, 8].  x is clamped at -126, so the exponent field cannot underflow (the
// result there is 2^-126, not a smaller number); the softmax never passes more than 8 (its
// deferred-rescale bound), far below overflow.  For finite x only: masked keys keep the
// exact zero of ex2.approx(-inf).
#pragma once

#include "ptx_sm100.cuh"

namespace gqa {

struct Exp2Poly {
    static constexpr float kRound = 12582912.f;  // 1.5 * 2^23
    static constexpr float kLow = -126.f;
    static constexpr float c1 = 0.6932829022407532f;
    static constexpr float c2 = 0.24221095442771912f;
    static constexpr float c3 = 0.055008936673402786f;
};

// two lanes at once with the packed fp32 instructions
__device__ __forceinline__ void exp2_poly2(float x0, float x1, float& y0, float& y1) {
    using P = Exp2Poly;
    x0 = fmaxf(x0, P::kLow);
    x1 = fmaxf(x1, P::kLow);
    float t0, t1, r0, r1, f0, f1, q0, q1;
    ptx::add2(x0, x1, P::kRound, P::kRound, t0, t1);    // t = x + 1.5 * 2^23 (j in the low bits)
    ptx::add2(t0, t1, -P::kRound, -P::kRound, r0, r1);  // r = j as a float
    ptx::add2(x0, x1, -r0, -r1, f0, f1);                // f = x - j
    ptx::fma2(f0, f1, P::c3, P::c3, P::c2, P::c2, q0, q1);
    ptx::fma2(q0, q1, f0, f1, P::c1, P::c1, q0, q1);
    ptx::fma2(q0, q1, f0, f1, 1.f, 1.f, q0, q1);
    y0 = __int_as_float(__float_as_int(q0) + (__float_as_int(t0) << 23));
    y1 = __int_as_float(__float_as_int(q1) + (__float_as_int(t1) << 23));
}

}  // namespace gqa
