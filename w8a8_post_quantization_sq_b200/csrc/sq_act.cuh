// The MLP activations of the path, each a fixed sequence of correctly rounded
// fp32 operations, so that any IEEE machine evaluating the same sequence gets
// the same bits (the int8 codes they decide must agree exactly).
//
// exp(x): Cody-Waite reduction x = n ln2 + r (ln 2 in two parts, the high
// part 2839/4096 so that n * LN2_HI is exact), the Taylor polynomial of exp(r)
// to degree 7 by Horner's rule with fma, then the exact scaling by 2^n;
// +inf above 88 and 0 below -87. Within 4 ulp of exp.
// silu(g) = g / (1 + exp(-g)).
// gelu(x), the tanh form 0.5 x (1 + tanh(u)), u = sqrt(2/pi) (x + 0.044715 x^3),
// evaluated as x / (1 + exp(-2u)) (the same function: 1 + tanh(u) =
// 2 / (1 + exp(-2u))), which has no cancellation for negative x.
#pragma once

namespace sq {

__device__ __forceinline__ float exp_fixed(float x) {
    if (x > 88.0f) return __int_as_float(0x7f800000);
    if (x < -87.0f) return 0.0f;
    // n = x * log2(e) rounded to the nearest integer (ties to even): adding
    // 1.5 * 2^23 rounds it into the low bits of the sum, which also hold n as
    // an integer; this is rint() with two adds instead of conversions
    const float sh = __fadd_rn(__fmul_rn(x, 0x1.715476p+0f), 12582912.0f);  // log2(e) in fp32
    const float n = __fsub_rn(sh, 12582912.0f);                            // exact; in [-126, 127]
    const int ni = __float_as_int(sh) - 0x4B400000;
    float r = __fmaf_rn(-n, 0x1.62e000p-1f, x);            // ln 2, high part (12 bits)
    r = __fmaf_rn(-n, 0x1.0bfbe8p-15f, r);                 // ln 2, low part
    float p = 0x1.a01a02p-13f;                             // 1/7!
    p = __fmaf_rn(p, r, 0x1.6c16c2p-10f);                  // 1/6!
    p = __fmaf_rn(p, r, 0x1.111112p-7f);                   // 1/5!
    p = __fmaf_rn(p, r, 0x1.555556p-5f);                   // 1/4!
    p = __fmaf_rn(p, r, 0x1.555556p-3f);                   // 1/3!
    p = __fmaf_rn(p, r, 0.5f);
    p = __fmaf_rn(p, r, 1.0f);
    p = __fmaf_rn(p, r, 1.0f);
    return __fmul_rn(p, __int_as_float((ni + 127) << 23));
}

__device__ __forceinline__ float silu_fixed(float g) { return __fdiv_rn(g, __fadd_rn(1.0f, exp_fixed(-g))); }

__device__ __forceinline__ float gelu_fixed(float x) {
    const float x3 = __fmul_rn(__fmul_rn(x, x), x);
    const float u = __fmul_rn(0x1.988454p-1f, __fmaf_rn(0x1.6e4e26p-5f, x3, x));  // sqrt(2/pi), 0.044715
    return __fdiv_rn(x, __fadd_rn(1.0f, exp_fixed(__fmul_rn(-2.0f, u))));
}

}  // namespace sq
