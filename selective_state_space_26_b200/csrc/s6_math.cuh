// s6_math.cuh -- fp32 element functions of the S6 layer.
//
//   softplus(v) = log(1 + e^v)      (the step size Delta)
//   silu(z)     = z / (1 + e^-z)    (the output gate)
//
// Both are built from the MUFU ex2 / rcp approximations plus a short series,
// accurate to a few fp32 ulp over the whole range (the MUFU lg2 is not used:
// its error is absolute, which would be a large relative error of Delta for
// the small steps the layer mostly takes).
#pragma once

#include "device_utils.cuh"

namespace jssm {

constexpr float kLog2e = 1.4426950408889634f;  // 1 / ln 2

// softplus(v) = max(v, 0) + log1p(w) with w = e^{-|v|} in (0, 1].
// log1p(w) = 2 atanh(s) with s = w / (2 + w) in (0, 1/3], and
// 2 atanh(s) = 2 s (1 + s^2/3 + s^4/5 + ...).  With s^2 <= 1/9 the series
// truncated after s^12/13 is within 1.5e-8 relative of log1p(w).
__device__ __forceinline__ float softplus_f32(float v) {
    const float w = ex2_mufu(-fabsf(v) * kLog2e);
    const float s = w * rcp_mufu(2.0f + w);
    const float u = s * s;
    float p = 2.0f / 13.0f;
    p = fmaf(p, u, 2.0f / 11.0f);
    p = fmaf(p, u, 2.0f / 9.0f);
    p = fmaf(p, u, 2.0f / 7.0f);
    p = fmaf(p, u, 2.0f / 5.0f);
    p = fmaf(p, u, 2.0f / 3.0f);
    p = fmaf(p, u, 2.0f);
    return fmaf(s, p, fmaxf(v, 0.0f));
}

// silu(z) = z * sigmoid(z).  For z -> -inf, e^-z overflows to +inf and the
// reciprocal gives 0, which is the correctly rounded limit.
__device__ __forceinline__ float silu_f32(float z) {
    const float e = ex2_mufu(-z * kLog2e);
    return z * rcp_mufu(1.0f + e);
}

// Delta for one (t, d): raw step input plus bias, through softplus if asked.
__device__ __forceinline__ float delta_f32(float raw, float bias, bool use_softplus) {
    const float v = raw + bias;
    return use_softplus ? softplus_f32(v) : v;
}

}  // namespace jssm
