// Scalar pieces of the quantizers: the IEEE fp32 quotient x / S without a
// division instruction, and the constant of the integer rounding.
#pragma once

#include <cuda_runtime.h>

#include <cstdint>

namespace q8 {
namespace qm {

constexpr float kEps = 1e-8f;
constexpr float kMagic = 12582912.0f;   // 1.5 * 2^23: RN(q + kMagic) is q rounded to an integer

// The quotient below is exact when |x / S| < 2^99 and S >= 2^-90 (no overflow,
// and the residuals of quotients large enough to matter for a code do not
// underflow); callers divide outside that domain.
constexpr float kQuotientMax = 0x1p99f;
constexpr float kScaleMin = 0x1p-90f;

// RN(x / S), the correctly rounded fp32 quotient, from R = RN(1/S) with four
// fused multiply-adds, after Markstein ("Computation of elementary functions on
// the IBM RISC System/6000 processor", IBM J. Res. Dev. 34(1), 1990; also
// Muller et al., Handbook of Floating-Point Arithmetic, the chapter on
// division with an FMA).
//   q0 = RN(x R) is within about 1.5 ulp of x / S (R and the product each
//   round once).
//   One correction q1 = RN(q0 + RN(x - q0 S) R): the corrected value is
//   within about 2^-46 relative of x / S, so q1 is a faithful rounding (one
//   of the two floats around x / S).
//   Markstein's theorem: with R within half an ulp of 1/S and q1 faithful,
//   the residual x - q1 S is a float (the FMA computes it exactly) and
//   RN(q1 + (x - q1 S) R) = RN(x / S).
// The residuals are kept negated (q S - x) and subtracted, so that x = -0
// keeps its sign through the corrections (-0 / S = -0).
__device__ __forceinline__ float quotient(float x, float S, float R) {
    const float q0 = __fmul_rn(x, R);
    const float e0 = __fmaf_rn(q0, S, -x);
    const float q1 = __fmaf_rn(-e0, R, q0);
    const float e1 = __fmaf_rn(q1, S, -x);
    return __fmaf_rn(-e1, R, q1);
}

// The same for two elements with paired fp32 instructions and one correction
// instead of two: with 1/S carried as R + Rlo (Rlo = RN(RN(1 - S R) R), the
// next 24 bits of the reciprocal), q0 = RN(x R + RN(x Rlo)) is within 2^-47
// relative of x / S before its rounding, so q0 is faithful and Markstein's
// step gives RN(x / S) directly.  The residual is formed as x - q0 S
// (nS = -S), which returns +0 for x = -0; every other quotient has x's sign,
// and callers whose codes keep the sign of zero restore it.
__device__ __forceinline__ float2 quotient2(float2 x, float2 nS, float2 R, float2 Rlo) {
    const float2 q0 = __ffma2_rn(x, R, __fmul2_rn(x, Rlo));
    const float2 e0 = __ffma2_rn(q0, nS, x);
    return __ffma2_rn(e0, R, q0);
}

// The low part of 1/S for quotient2: 1 - S R is exact in an FMA (R = RN(1/S)),
// and (1 - S R) / S = 1/S - R.
__device__ __forceinline__ float reciprocal_low(float S, float R) {
    return __fmul_rn(__fmaf_rn(-S, R, 1.0f), R);
}

}  // namespace qm
}  // namespace q8
