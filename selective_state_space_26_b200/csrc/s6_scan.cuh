// s6_scan.cuh -- pieces shared by the S6 prefill kernel (s6_scan_fused.cuh):
// the device status word, the kernel arguments, B/C widening, and one step of
// a lane's selective-scan recurrence.
//
// The recurrence (the "Mamba 레이어" section of the Jamba notes, with the
// discretisation read as exp(Delta A) and Delta B x):
//     h[n] = exp(Delta A[d,n]) h[n] + Delta B[b,t,n] x[b,t,d],   y = sum_n C[b,t,n] h[n].
#pragma once

#include <type_traits>

#include "device_utils.cuh"
#include "s6_math.cuh"

namespace jssm {


struct ScanArgs {
    int64_t batch, seqlen, d_inner;
    const float *A, *D, *delta_bias, *h0;
    float *h_final;
    int delta_softplus;
    uint32_t debug_flags;
    uint64_t timeout_cycles;
};

// Widen 16 bytes of B or C to floats.
__device__ __forceinline__ void widen16(const uint4 v, const __nv_bfloat16 *, float (&f)[8]) {
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        f[2 * i] = __uint_as_float(w[i] << 16);
        f[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
    }
}
__device__ __forceinline__ void widen16(const uint4 v, const float *, float (&f)[4]) {
    f[0] = __uint_as_float(v.x);
    f[1] = __uint_as_float(v.y);
    f[2] = __uint_as_float(v.z);
    f[3] = __uint_as_float(v.w);
}

// Sum of v over the G lanes of a channel.  Partners are taken in the order
// reduce_transpose uses (lane ^ G/2 first), so both give bit-identical sums.
template <int G>
__device__ __forceinline__ float lane_group_sum(float v) {
#pragma unroll
    for (int off = G / 2; off >= 1; off >>= 1) v += __shfl_xor_sync(0xffffffffu, v, off);
    return v;
}

// For G consecutive steps held by each of the G lanes of a channel (v[j] is
// this lane's partial sum of step j), returns the full sum of step `sub` on
// lane `sub`: a butterfly where each round keeps the half of the values the
// lane's own index selects and trades the other half with the partner lane.
template <int G>
__device__ __forceinline__ float reduce_transpose(const float *v, int sub) {
    if constexpr (G == 1) {
        return v[0];
    } else {
        constexpr int H = G / 2;
        const bool upper = (sub & H) != 0;
        float w[H];
#pragma unroll
        for (int i = 0; i < H; ++i) {
            const float keep = upper ? v[i + H] : v[i];
            const float send = upper ? v[i] : v[i + H];
            w[i] = keep + __shfl_xor_sync(0xffffffffu, send, H);
        }
        return reduce_transpose<H>(w, sub & (H - 1));
    }
}

// One step of a lane's recurrence: its NS states advance by one token and its
// partial sum of C.h is returned.  States are processed in pairs with packed
// fp32x2 multiplies / FMAs (one issue slot per two states); Abar comes from the
// MUFU ex2.
template <int N, int NS>
__device__ __forceinline__ float recurrence_step(float2 (&h)[NS / 2], const float2 (&a2)[NS / 2],
                                                 float2 dlx, const float *bcrow, int sub) {
    const float4 *row = reinterpret_cast<const float4 *>(bcrow);
    const float2 dl = make_float2(dlx.x, dlx.x), dx = make_float2(dlx.y, dlx.y);
    float2 y0 = make_float2(0.0f, 0.0f), y1 = make_float2(0.0f, 0.0f);
#pragma unroll
    for (int q = 0; q < NS / 4; ++q) {
        const float4 bq = row[(sub * NS) / 4 + q];
        const float4 cq = row[(N + sub * NS) / 4 + q];
        const float2 bv[2] = {make_float2(bq.x, bq.y), make_float2(bq.z, bq.w)};
        const float2 cv[2] = {make_float2(cq.x, cq.y), make_float2(cq.z, cq.w)};
#pragma unroll
        for (int e = 0; e < 2; ++e) {
            const int i = 2 * q + e;
            const float2 arg = mul2(dl, a2[i]);
            const float2 abar = make_float2(ex2_mufu(arg.x), ex2_mufu(arg.y));
            h[i] = fma2(abar, h[i], mul2(dx, bv[e]));
            if (e) y1 = fma2(cv[e], h[i], y1);
            else y0 = fma2(cv[e], h[i], y0);
        }
    }
    const float2 y = add2(y0, y1);
    return y.x + y.y;
}

}  // namespace jssm
