// Scalar pieces of the quantizers: constants of the division-free rounding and
// the directed reciprocals that bracket the IEEE quotient x / S.
#pragma once

#include <cstdint>

namespace q8 {
namespace qm {

constexpr float kEps = 1e-8f;
constexpr float kMagic = 12582912.0f;     // 1.5 * 2^23: x + kMagic rounds x to an integer
constexpr float kFastLimit = 2097152.0f;  // 2^21: bound on |x * r| for the integer fast path

// 1/S rounded down and up, from R = RN(1/S) and the sign of the residual
// 1 - S R, which one FMA gives exactly (|1 - S R| <= 2^-24 fits in a float).
// Equal when S is a power of two (1/S exact).  S is a positive normal float.
__device__ __forceinline__ void reciprocal_bounds(float S, float& rd, float& ru) {
    const float R = __frcp_rn(S);
    const float res = __fmaf_rn(-S, R, 1.0f);
    const uint32_t rb = __float_as_uint(R);
    rd = res < 0.f ? __uint_as_float(rb - 1u) : R;   // R > 1/S: one ulp down
    ru = res > 0.f ? __uint_as_float(rb + 1u) : R;   // R < 1/S: one ulp up
}

}  // namespace qm
}  // namespace q8
