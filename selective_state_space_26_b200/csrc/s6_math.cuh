// s6_math.cuh -- fp32 element functions of the S6 layer.
//
//   softplus(v) = log(1 + e^v)      (the step size Delta)
//   silu(z)     = z / (1 + e^-z)    (the output gate)
//
// Both are built from the MUFU ex2 / rcp approximations plus a polynomial,
// accurate to a few fp32 ulp over the whole range (the MUFU lg2 is not used:
// its error is absolute, which would be a large relative error of Delta for
// the small steps the layer mostly takes).
#pragma once

#include "device_utils.cuh"

namespace jssm {

constexpr float kLog2e = 1.4426950408889634f;  // 1 / ln 2

// softplus(v) = max(v, 0) + log1p(w) with w = e^{-|v|} in (0, 1], and
// log1p(w) = w q(w) with q a degree-8 polynomial: the least-squares fit of
// log1p(w) / w at 4000 Chebyshev nodes of [0, 1] (q(0) = 1 exactly).  The fit is
// within 3e-8 relative of log1p on (0, 1]; evaluated by Horner in fp32 the
// result is within 2e-7.  One MUFU op (the ex2) instead of ex2 + rcp of the
// w / (2 + w) series form, which matters because the scan is bound by the
// MUFU pipe.
__device__ __forceinline__ float softplus_f32(float v) {
    const float w = ex2_mufu(-fabsf(v) * kLog2e);
    float p = 5.253457930e-03f;
    p = fmaf(p, w, -2.958850749e-02f);
    p = fmaf(p, w, 7.836166769e-02f);
    p = fmaf(p, w, -1.367477030e-01f);
    p = fmaf(p, w, 1.911143064e-01f);
    p = fmaf(p, w, -2.484436929e-01f);
    p = fmaf(p, w, 3.331927061e-01f);
    p = fmaf(p, w, -4.999950230e-01f);
    p = fmaf(p, w, 1.0f);
    return fmaf(w, p, fmaxf(v, 0.0f));
}

// The same form with a degree-6 q (the least-squares fit at the same nodes):
// within 1.6e-6 relative of log1p in fp32, three orders of magnitude below
// half a bf16 ulp (2^-9 relative), two FMAs shorter.  Used where the layer's
// inputs and outputs are bf16; fp32 I/O keeps the degree-8 form above.
__device__ __forceinline__ float softplus6_f32(float v) {
    const float w = ex2_mufu(-fabsf(v) * kLog2e);
    float p = 1.459241658e-02f;
    p = fmaf(p, w, -6.785421818e-02f);
    p = fmaf(p, w, 1.510172933e-01f);
    p = fmaf(p, w, -2.360982597e-01f);
    p = fmaf(p, w, 3.313975036e-01f);
    p = fmaf(p, w, -4.999065399e-01f);
    p = fmaf(p, w, 1.0f);
    return fmaf(w, p, fmaxf(v, 0.0f));
}

// softplus at the accuracy that the I/O type shows.
template <typename IoT>
__device__ __forceinline__ float softplus_io(float v) {
    return softplus_f32(v);
}
template <>
__device__ __forceinline__ float softplus_io<__nv_bfloat16>(float v) {
    return softplus6_f32(v);
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
template <typename IoT>
__device__ __forceinline__ float delta_io(float raw, float bias, bool use_softplus) {
    const float v = raw + bias;
    return use_softplus ? softplus_io<IoT>(v) : v;
}

}  // namespace jssm
