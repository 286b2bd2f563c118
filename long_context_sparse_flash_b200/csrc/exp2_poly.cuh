// exp2_poly.cuh -- 2^x on the FMA and integer pipes, to share the work of the
// special-function unit (whose ex2 throughput is the limit of attention's
// softmax on this GPU).
//
// Method: range reduction 2^x = 2^n * 2^f with n = rint(x), f = x - n in
// [-1/2, 1/2]; n is obtained by adding 1.5 * 2^23 (the sum's low mantissa
// bits then hold n in two's complement) and is added to the exponent field of
// P(f) as an integer.  P is a least-squares fit of the relative error of 2^f
// on Chebyshev nodes of [-1/2, 1/2] with P(0) = 1 (gen_exp2_poly.py in this
// directory recomputes the coefficients and their error).  Inputs below -127
// give 0 (also -inf); inputs must stay below 127.
#pragma once

#include "hs2_common.cuh"

namespace hs2 {

// degree 3: max relative error 1.136e-04 (float64 eval), 1.136e-04 (float32 Horner)
// coefficients of f^0 .. f^3: 1, 6.933686137e-01, 2.422178388e-01, 5.459282547e-02
// degree 5: max relative error 1.044e-07 (float64 eval), 1.773e-07 (float32 Horner)
// coefficients of f^0 .. f^5: 1, 6.931468844e-01, 2.402223796e-01, 5.550893024e-02,
//                             9.671698324e-03, 1.321867225e-03

template <int DEG>
__device__ __forceinline__ float exp2_poly(float x) {
    static_assert(DEG == 3 || DEG == 5, "fitted degrees: 3 and 5");
    constexpr float kRound = 12582912.0f;  // 1.5 * 2^23
    x = fmaxf(x, -127.0f);
    const float t = x + kRound;
    const float f = x - (t - kRound);
    float p;
    if constexpr (DEG == 3) {
        p = fmaf(fmaf(fmaf(5.459282547e-02f, f, 2.422178388e-01f), f, 6.933686137e-01f), f, 1.0f);
    } else {
        p = fmaf(fmaf(fmaf(fmaf(fmaf(1.321867225e-03f, f, 9.671698324e-03f), f, 5.550893024e-02f), f,
                            2.402223796e-01f), f, 6.931468844e-01f), f, 1.0f);
    }
    return __int_as_float(__float_as_int(p) + (__float_as_int(t) << 23));
}

// Two lanes at once: the same steps with packed fp32x2 adds and FMAs (the
// clamp and the exponent insertion stay per lane).
__device__ __forceinline__ float2 exp2_poly5_x2(float2 x) {
    constexpr float kRound = 12582912.0f;  // 1.5 * 2^23
    x.x = fmaxf(x.x, -127.0f);
    x.y = fmaxf(x.y, -127.0f);
    const float2 rnd = make_float2(kRound, kRound), nrnd = make_float2(-kRound, -kRound);
    const float2 t = fadd2(x, rnd);
    const float2 n = fadd2(t, nrnd);
    const float2 f = fsub2(x, n);
    float2 p = ffma2(make_float2(1.321867225e-03f, 1.321867225e-03f), f, make_float2(9.671698324e-03f, 9.671698324e-03f));
    p = ffma2(p, f, make_float2(5.550893024e-02f, 5.550893024e-02f));
    p = ffma2(p, f, make_float2(2.402223796e-01f, 2.402223796e-01f));
    p = ffma2(p, f, make_float2(6.931468844e-01f, 6.931468844e-01f));
    p = ffma2(p, f, make_float2(1.0f, 1.0f));
    return make_float2(__int_as_float(__float_as_int(p.x) + (__float_as_int(t.x) << 23)),
                       __int_as_float(__float_as_int(p.y) + (__float_as_int(t.y) << 23)));
}

}  // namespace hs2
