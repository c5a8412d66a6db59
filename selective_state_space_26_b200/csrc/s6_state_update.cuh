// s6_state_update.cuh -- one-token decode step of the S6 layer (sm_100a).
//
// The O(1)-per-token update of "한 페이지로 보는 SSM" (Jamba -- Hybrid
// SSM-Transformer lesson): y_t needs only h_{t-1} and x_t.  For request b and
// channel d:
//     Delta = softplus(delta[b,d] + delta_bias[d])
//     h[n]  = exp(Delta A[d,n]) h[n] + Delta B[b,n] x[b,d]     (in place)
//     out   = (sum_n C[b,n] h[n] + D[d] x[b,d]) * silu(z[b,d])
//
// The fp32 state dominates the bytes (it is read and written once per step),
// so the kernel is a streaming, HBM-bound pass: Q = N/4 consecutive lanes own
// one (b, d) and each moves one float4 of its state with a 128-bit load and
// store (a warp touches 512 contiguous bytes).  The partial sums of C.h are
// combined with Q-1 xor-shuffles; the per-(b, d) scalars (softplus, gate) are
// recomputed by each of the Q lanes, which costs MUFU issue slots that this
// memory-bound kernel has to spare.
#pragma once

#include "device_utils.cuh"
#include "s6_math.cuh"

namespace jssm {

struct UpdateArgs {
    int64_t batch, d_inner;
    float *state;
    const void *x, *delta, *z, *B, *C;
    const float *A, *D, *delta_bias;
    void *out;
    int delta_softplus;
};

template <typename IoT>
__device__ __forceinline__ void load4(const IoT *p, float (&v)[4]);
template <>
__device__ __forceinline__ void load4<float>(const float *p, float (&v)[4]) {
    const float4 q = *reinterpret_cast<const float4 *>(p);
    v[0] = q.x; v[1] = q.y; v[2] = q.z; v[3] = q.w;
}
template <>
__device__ __forceinline__ void load4<__nv_bfloat16>(const __nv_bfloat16 *p, float (&v)[4]) {
    const uint2 q = *reinterpret_cast<const uint2 *>(p);
    v[0] = __uint_as_float(q.x << 16);
    v[1] = __uint_as_float(q.x & 0xffff0000u);
    v[2] = __uint_as_float(q.y << 16);
    v[3] = __uint_as_float(q.y & 0xffff0000u);
}

template <typename IoT, int N>
__global__ void __launch_bounds__(256) s6_state_update_kernel(const UpdateArgs a) {
    constexpr int Q = N / 4;
    static_assert(N % 4 == 0 && (Q & (Q - 1)) == 0, "N/4 lanes per channel, power of two");
    const int64_t gid = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
    const int64_t total = a.batch * a.d_inner;
    const int64_t bd_raw = gid / Q;
    const bool valid = bd_raw < total;
    const int64_t bd = valid ? bd_raw : total - 1;  // invalid lanes still join the shuffles
    const int q = static_cast<int>(gid % Q);
    const int64_t b = bd / a.d_inner, d = bd % a.d_inner;

    const IoT *x = static_cast<const IoT *>(a.x);
    const IoT *dt = static_cast<const IoT *>(a.delta);
    const IoT *z = static_cast<const IoT *>(a.z);
    float4 *st = reinterpret_cast<float4 *>(a.state) + bd * Q + q;

    const float4 h4 = *st;
    float Av[4], Bv[4], Cv[4];
    load4<float>(a.A + d * N + 4 * q, Av);
    load4<IoT>(static_cast<const IoT *>(a.B) + b * N + 4 * q, Bv);
    load4<IoT>(static_cast<const IoT *>(a.C) + b * N + 4 * q, Cv);
    const float xv = to_f32(x[bd]);
    const float bias = a.delta_bias ? __ldg(a.delta_bias + d) : 0.0f;
    const float dl = delta_f32(to_f32(dt[bd]), bias, a.delta_softplus != 0);
    const float dx = dl * xv;

    float h[4] = {h4.x, h4.y, h4.z, h4.w};
    float y = 0.0f;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const float abar = ex2_mufu(dl * (Av[i] * kLog2e));
        h[i] = fmaf(abar, h[i], dx * Bv[i]);
        y = fmaf(Cv[i], h[i], y);
    }
#pragma unroll
    for (int off = 1; off < Q; off <<= 1) y += __shfl_xor_sync(0xffffffffu, y, off);

    if (valid) {
        *st = make_float4(h[0], h[1], h[2], h[3]);
        if (q == 0) {
            const float dskip = a.D ? __ldg(a.D + d) : 0.0f;
            const float o = (y + dskip * xv) * silu_f32(to_f32(z[bd]));
            static_cast<IoT *>(a.out)[bd] = from_f32<IoT>(o);
        }
    }
}

}  // namespace jssm
