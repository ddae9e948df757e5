// lard_exp2.cuh -- 2^x on the FMA pipe, to share the exponential load of the
// softmax warps between the MUFU unit (ex2.approx) and the FP32 pipe.
//
// Range reduction: n = rint(x) by the round-to-nearest of an fp32 add of
// 1.5 * 2^23 (the integer lands in the low mantissa bits), f = x - n in
// [-1/2, 1/2]; then 2^x = p(f) * 2^n, with 2^n applied by adding n to the
// exponent field of p(f).  p is the degree-5 minimax polynomial (relative
// error) of 2^f on [-1/2, 1/2], produced by gen_exp2_poly.py (Remez
// exchange); its approximation error is below the fp32 rounding of the
// evaluation.  Inputs below -125 are clamped so that the result stays a
// normal number (2^-125 ~ 2.4e-38 stands for "zero" in the sums it feeds).
#pragma once

namespace lard {

// degree 5 minimax (relative) fit of 2^f on [-1/2, 1/2]; max rel. error 7.494e-08
#define LARD_EXP2_POLY {1.000000072e+00f, 6.931469671e-01f, 2.402211972e-01f, 5.550713273e-02f, 9.675541334e-03f, 1.327647199e-03f}

__device__ __forceinline__ float exp2_fma(float x) {
    x = fmaxf(x, -125.0f);
    const float t = __fadd_rn(x, 12582912.0f);  // 1.5 * 2^23
    const float n = __fadd_rn(t, -12582912.0f);
    const float f = __fadd_rn(x, -n);
    constexpr float c[6] = LARD_EXP2_POLY;
    float p = c[5];
    p = fmaf(p, f, c[4]);
    p = fmaf(p, f, c[3]);
    p = fmaf(p, f, c[2]);
    p = fmaf(p, f, c[1]);
    p = fmaf(p, f, c[0]);
    return __int_as_float(__float_as_int(p) + (__float_as_int(t) << 23));
}

// Packed-pair arithmetic of sm_100 (two fp32 lanes per instruction).
__device__ __forceinline__ float2 fma2(float2 a, float2 b, float2 c) { return __ffma2_rn(a, b, c); }
__device__ __forceinline__ float2 add2(float2 a, float2 b) { return __fadd2_rn(a, b); }
__device__ __forceinline__ float2 mul2(float2 a, float2 b) { return __fmul2_rn(a, b); }
// a - b, exactly as an fp32 subtraction: b * -1 is exact, then one rounding.
__device__ __forceinline__ float2 sub2(float2 a, float2 b) { return __ffma2_rn(b, make_float2(-1.f, -1.f), a); }
__device__ __forceinline__ float2 splat2(float v) { return make_float2(v, v); }

// exp2_fma on a pair, with the reduction and the polynomial in packed form.
__device__ __forceinline__ float2 exp2_fma2(float2 x) {
    x.x = fmaxf(x.x, -125.0f);
    x.y = fmaxf(x.y, -125.0f);
    const float2 t = add2(x, splat2(12582912.0f));
    const float2 n = add2(t, splat2(-12582912.0f));
    const float2 f = sub2(x, n);
    constexpr float c[6] = LARD_EXP2_POLY;
    float2 p = splat2(c[5]);
    p = fma2(p, f, splat2(c[4]));
    p = fma2(p, f, splat2(c[3]));
    p = fma2(p, f, splat2(c[2]));
    p = fma2(p, f, splat2(c[1]));
    p = fma2(p, f, splat2(c[0]));
    return make_float2(__int_as_float(__float_as_int(p.x) + (__float_as_int(t.x) << 23)),
                       __int_as_float(__float_as_int(p.y) + (__float_as_int(t.y) << 23)));
}

}  // namespace lard
