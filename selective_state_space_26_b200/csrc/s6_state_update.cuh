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
// so both kernels are streaming, HBM-bound passes in which Q = N/4 lanes own
// one (request, channel), 4 states each, moved as one 16-byte load and store:
//  * s6_state_update_stream_kernel (rows of whole 16-byte chunks, the usual
//    case): a producer warp streams each request's state slab and activations
//    into a ring of shared-memory stages with 1-D bulk copies; the lanes of a
//    channel take requests Q at a time, lane q computing request q's softplus
//    and gate once and handing Delta, Delta x over by shuffles.
//  * s6_state_update_kernel (any other row size): plain vector loads, two
//    requests in flight per thread, each of the Q lanes computing the scalars.
// The partial sums of C.h are combined across the Q lanes with shuffles.
#pragma once

#include "device_utils.cuh"
#include "s6_math.cuh"
#include "s6_scan.cuh"  // reduce_transpose

namespace jssm {

struct UpdateArgs {
    int64_t batch, d_inner;
    float *state;
    const void *x, *delta, *z, *B, *C;
    const float *A, *D, *delta_bias;
    void *out;
    int delta_softplus;
    const int *state_indices;  // state-cache row of each request, or null (row b)
    int64_t num_slots;         // rows of the state cache
    uint32_t debug_flags;      // bit 0: withhold each CTA's first load (tests the bounded waits)
    int *status;               // the call's status word (caller workspace), or null
};

// State-cache row of request b, or -1 when the request is skipped (a negative
// index: padding; or one past the cache, recorded as an invalid argument).
__device__ __forceinline__ int64_t state_row(const UpdateArgs &a, int64_t b, bool record) {
    if (!a.state_indices) return b;
    const int64_t r = __ldg(a.state_indices + b);
    if (r >= a.num_slots) {
        if (record) record_status(a.status, kStInvalidArg);
        return -1;
    }
    return r < 0 ? -1 : r;
}

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

// A block of 256 threads owns 256/Q consecutive channels d and walks BPC
// requests b: the per-channel parameters (A[d, 4q..4q+3], delta_bias, D) are
// loaded once into registers and reused for every request, so A is not re-read
// per request; for each request the Q lanes of a channel move its N fp32
// states as Q float4s (a warp touches 512 contiguous bytes).  Requests are
// processed two at a time with every load issued before the math.
template <typename IoT, int N, int BPC>
__global__ void __launch_bounds__(256) s6_state_update_kernel(const UpdateArgs a) {
    constexpr int Q = N / 4;
    constexpr int CPB = 256 / Q;  // channels per block
    static_assert(N % 4 == 0 && (Q & (Q - 1)) == 0, "N/4 lanes per channel, power of two");
    static_assert(BPC % 2 == 0, "requests are processed in pairs");
    const int q = threadIdx.x % Q;
    const int64_t d = static_cast<int64_t>(blockIdx.x) * CPB + threadIdx.x / Q;
    const bool dvalid = d < a.d_inner;
    const int64_t dc = dvalid ? d : a.d_inner - 1;  // invalid lanes still join the shuffles
    float Av[4];
    load4<float>(a.A + dc * N + 4 * q, Av);
#pragma unroll
    for (int i = 0; i < 4; ++i) Av[i] *= kLog2e;
    const float bias = a.delta_bias ? __ldg(a.delta_bias + dc) : 0.0f;
    const float dskip = a.D ? __ldg(a.D + dc) : 0.0f;
    const bool use_softplus = a.delta_softplus != 0;
    const IoT *x = static_cast<const IoT *>(a.x);
    const IoT *dt = static_cast<const IoT *>(a.delta);
    const IoT *z = static_cast<const IoT *>(a.z);
    float4 *st = reinterpret_cast<float4 *>(a.state);
    const int64_t b0 = static_cast<int64_t>(blockIdx.y) * BPC;

#pragma unroll 1
    for (int j = 0; j < BPC; j += 2) {
        float4 h4[2];
        float Bv[2][4], Cv[2][4], xv[2], dtv[2], zv[2];
        bool valid[2];
        int64_t bd[2], sd[2];  // activation row, state row
#pragma unroll
        for (int u = 0; u < 2; ++u) {
            const int64_t b = b0 + j + u;
            const int64_t bc = b < a.batch ? b : a.batch - 1;
            const int64_t srow = state_row(a, bc, threadIdx.x == 0 && b < a.batch);
            valid[u] = dvalid && b < a.batch && srow >= 0;
            bd[u] = bc * a.d_inner + dc;
            sd[u] = (srow >= 0 ? srow : 0) * a.d_inner + dc;
            h4[u] = st[sd[u] * Q + q];
            load4<IoT>(static_cast<const IoT *>(a.B) + bc * N + 4 * q, Bv[u]);
            load4<IoT>(static_cast<const IoT *>(a.C) + bc * N + 4 * q, Cv[u]);
            xv[u] = to_f32(x[bd[u]]);
            dtv[u] = to_f32(dt[bd[u]]);
            zv[u] = to_f32(z[bd[u]]);
        }
#pragma unroll
        for (int u = 0; u < 2; ++u) {
            const float dl = delta_io<IoT>(dtv[u], bias, use_softplus);
            const float dx = dl * xv[u];
            float h[4] = {h4[u].x, h4[u].y, h4[u].z, h4[u].w};
            float y = 0.0f;
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const float abar = ex2_mufu(dl * Av[i]);
                h[i] = fmaf(abar, h[i], dx * Bv[u][i]);
                y = fmaf(Cv[u][i], h[i], y);
            }
#pragma unroll
            for (int off = 1; off < Q; off <<= 1) y += __shfl_xor_sync(0xffffffffu, y, off);
            if (valid[u]) {
                st[sd[u] * Q + q] = make_float4(h[0], h[1], h[2], h[3]);
                if (q == 0) {
                    const float o = (y + dskip * xv[u]) * silu_f32(zv[u]);
                    static_cast<IoT *>(a.out)[bd[u]] = from_f32<IoT>(o);
                }
            }
        }
    }
}

// Streaming form for the usual shapes (rows of whole 16-byte chunks).  A CTA
// owns one block of CPB channels and walks BPC requests.  One producer warp
// keeps a STAGES-deep ring of 1-D bulk copies (no multicast) in flight -- per
// request the CPB x N fp32 state slab (contiguous) and the x / delta / z
// slices and B / C rows -- so the bytes in flight per SM are set by shared
// memory, not registers; full / empty mbarriers per stage let it refill a
// stage as soon as the compute warps have read it (no CTA-wide barrier).
// Q = N/4 lanes own a channel, 4 states each.  Requests are taken in groups of
// Q: lane q computes the per-(request, channel) scalars of request q of the
// group (softplus, Delta x, gate, skip) and hands Delta, Delta x to the other
// lanes by shuffles, so no lane repeats another's transcendental work; the Q
// partial sums of C.h of the group's requests are reduced with the
// transposing butterfly, which leaves request q's sum on lane q, who writes
// its output.  The new state goes straight back to HBM (128-bit stores).
// Every wait is bounded; on a timeout the CTA records JAMBA_SSM_ERR_TIMEOUT
// and leaves, the producer first waiting (bounded) for its copies in flight.
template <typename IoT, int N, int CPB, int STAGES>
struct UpdateCfg {
    static constexpr int Q = N / 4;
    static constexpr int kComputeThreads = CPB * Q;
    static constexpr int kComputeWarps = kComputeThreads / 32;
    static constexpr int kThreads = kComputeThreads + 32;
    static constexpr int kStateBytes = CPB * N * 4;
    static constexpr int kActBytes = CPB * (int)sizeof(IoT);
    static constexpr int kBCBytes = N * (int)sizeof(IoT);
    static constexpr int kStage = kStateBytes + 3 * kActBytes + 2 * kBCBytes;
    static_assert(kComputeThreads % 32 == 0, "whole compute warps");
    static_assert(STAGES % Q == 0 && STAGES >= 2 * Q, "two request groups in flight");
    static_assert(kActBytes % 16 == 0 && kBCBytes % 16 == 0 && kStage % 16 == 0, "bulk sizes");
    static constexpr int kOffBar = STAGES * kStage;  // full[STAGES], empty[STAGES]
    static constexpr int kSmemBytes = kOffBar + 2 * STAGES * 8 + 16;
};

// SLOTS: the state is a cache addressed by state_indices (a template parameter
// so that the plain kernel carries no per-request lookups).
template <typename IoT, int N, int CPB, int BPC, int STAGES, bool SLOTS>
__global__ void __launch_bounds__(UpdateCfg<IoT, N, CPB, STAGES>::kThreads, 4)
    s6_state_update_stream_kernel(const UpdateArgs a, uint64_t limit) {
    using Cfg = UpdateCfg<IoT, N, CPB, STAGES>;
    constexpr int Q = Cfg::Q, NW = Cfg::kComputeWarps;
    extern __shared__ __align__(1024) uint8_t smem[];
    uint64_t *full = reinterpret_cast<uint64_t *>(smem + Cfg::kOffBar);
    uint64_t *empty = full + STAGES;
    volatile int *abort_flag = reinterpret_cast<volatile int *>(empty + STAGES);
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    // This CTA: channels [blockIdx.x * CPB, +nd), requests [blockIdx.y * BPC, +nu).
    const int64_t d0 = static_cast<int64_t>(blockIdx.x) * CPB;
    const int nd = static_cast<int>(a.d_inner - d0 < CPB ? a.d_inner - d0 : CPB);
    const int64_t breq0 = static_cast<int64_t>(blockIdx.y) * BPC;
    const int nu = static_cast<int>(a.batch - breq0 < BPC ? a.batch - breq0 : BPC);

    if (tid == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], NW);
        }
        *abort_flag = 0;
        fence_mbarrier_init();
    }
    __syncthreads();

    if (warp == NW) {
        // ================= producer warp: the bulk-copy ring =================
        if (lane == 0) {
            const IoT *xg = static_cast<const IoT *>(a.x);
            const IoT *dtg = static_cast<const IoT *>(a.delta);
            const IoT *zg = static_cast<const IoT *>(a.z);
            const IoT *Bg = static_cast<const IoT *>(a.B);
            const IoT *Cg = static_cast<const IoT *>(a.C);
            const uint32_t state_bytes = static_cast<uint32_t>(nd) * N * 4;
            const uint32_t act_bytes = static_cast<uint32_t>(nd) * sizeof(IoT);
            int issued = 0;
            bool ok = true, withheld0 = false;
            for (int u = 0; u < nu; ++u) {
                const int s = u % STAGES;
                if (u >= STAGES &&
                    !mbar_wait_or_abort(&empty[s], static_cast<uint32_t>(u / STAGES - 1) & 1u, limit,
                                        abort_flag)) {
                    ok = false;
                    break;
                }
                if ((a.debug_flags & 1u) && u == 0) {  // test hook: this load never comes
                    withheld0 = true;
                    issued = 1;
                    continue;
                }
                uint8_t *st = smem + s * Cfg::kStage;
                const int64_t b = breq0 + u, row = b * a.d_inner + d0;
                const int64_t srow = SLOTS ? state_row(a, b, false) : b;  // skipped: loads row 0
                mbar_arrive_expect_tx(&full[s], state_bytes + 3 * act_bytes + 2 * Cfg::kBCBytes);
                bulk_load_1d(st, a.state + ((srow >= 0 ? srow : 0) * a.d_inner + d0) * N, state_bytes,
                             &full[s]);
                bulk_load_1d(st + Cfg::kStateBytes, xg + row, act_bytes, &full[s]);
                bulk_load_1d(st + Cfg::kStateBytes + Cfg::kActBytes, dtg + row, act_bytes, &full[s]);
                bulk_load_1d(st + Cfg::kStateBytes + 2 * Cfg::kActBytes, zg + row, act_bytes, &full[s]);
                bulk_load_1d(st + Cfg::kStateBytes + 3 * Cfg::kActBytes, Bg + b * N, Cfg::kBCBytes,
                             &full[s]);
                bulk_load_1d(st + Cfg::kStateBytes + 3 * Cfg::kActBytes + Cfg::kBCBytes, Cg + b * N,
                             Cfg::kBCBytes, &full[s]);
                issued = u + 1;
            }
            if (!ok) {
                *abort_flag = 1;
                record_status(a.status, kStTimeout);
            }
            // copies still in flight when the compute warps may have left:
            // wait (bounded) for each stage's last fill before the CTA exits
            for (int u = issued - STAGES > 0 ? issued - STAGES : 0; u < issued; ++u)
                if (!(withheld0 && u == 0))
                    mbar_wait_bounded(&full[u % STAGES], static_cast<uint32_t>(u / STAGES) & 1u, limit);
        }
        return;
    }

    // =========================== compute warps ===========================
    const int q = tid % Q, cl = tid / Q;
    const int gbase = lane & ~(Q - 1);
    const bool dvalid = cl < nd;
    const int c = dvalid ? cl : nd - 1;  // idle lanes shadow a valid channel
    const int64_t d = d0 + c;
    float2 a2[2];
    {
        float Av[4];
        load4<float>(a.A + d * N + 4 * q, Av);
        a2[0] = make_float2(Av[0] * kLog2e, Av[1] * kLog2e);
        a2[1] = make_float2(Av[2] * kLog2e, Av[3] * kLog2e);
    }
    const float bias = a.delta_bias ? __ldg(a.delta_bias + d) : 0.0f;
    const float dskip = a.D ? __ldg(a.D + d) : 0.0f;
    const bool use_softplus = a.delta_softplus != 0;
    float4 *stg = reinterpret_cast<float4 *>(a.state);
    IoT *outg = static_cast<IoT *>(a.out);

    for (int r0 = 0; r0 < nu; r0 += Q) {
        const int nr = nu - r0 < Q ? nu - r0 : Q;
        bool ok = true;
        for (int r = 0; r < nr && ok; ++r)
            ok = mbar_wait_or_abort(&full[(r0 + r) % STAGES], static_cast<uint32_t>((r0 + r) / STAGES) & 1u,
                                    limit, abort_flag);
        ok = warp_agree(ok);
        if (!ok) {
            *abort_flag = 1;
            record_status(a.status, kStTimeout);
            break;
        }
        // this lane's owned request r0 + q (a copy of request r0 when q >= nr)
        const uint8_t *so = smem + ((r0 + (q < nr ? q : 0)) % STAGES) * Cfg::kStage;
        const IoT *xs = reinterpret_cast<const IoT *>(so + Cfg::kStateBytes);
        const float xv = to_f32(xs[c]);
        const float dl = delta_io<IoT>(to_f32(xs[CPB + c]), bias, use_softplus);
        const float gate = silu_f32(to_f32(xs[2 * CPB + c]));
        const float dxo = dl * xv, skg = dskip * xv * gate;
        float yp[Q];
#pragma unroll
        for (int r = 0; r < Q; ++r) {
            const float dlr = Q == 1 ? dl : __shfl_sync(0xffffffffu, dl, gbase | r);
            const float dxr = Q == 1 ? dxo : __shfl_sync(0xffffffffu, dxo, gbase | r);
            yp[r] = 0.0f;
            if (r < nr) {
                const uint8_t *st = smem + ((r0 + r) % STAGES) * Cfg::kStage;
                const float4 h4 = reinterpret_cast<const float4 *>(st)[c * Q + q];
                const IoT *Bs = reinterpret_cast<const IoT *>(st + Cfg::kStateBytes + 3 * Cfg::kActBytes);
                float Bv[4], Cv[4];
                load4<IoT>(Bs + 4 * q, Bv);
                load4<IoT>(Bs + N + 4 * q, Cv);
                const float2 dlp = make_float2(dlr, dlr), dxp = make_float2(dxr, dxr);
                const float2 arg0 = mul2(dlp, a2[0]), arg1 = mul2(dlp, a2[1]);
                float2 h0 = fma2(make_float2(ex2_mufu(arg0.x), ex2_mufu(arg0.y)), make_float2(h4.x, h4.y),
                                 mul2(dxp, make_float2(Bv[0], Bv[1])));
                float2 h1 = fma2(make_float2(ex2_mufu(arg1.x), ex2_mufu(arg1.y)), make_float2(h4.z, h4.w),
                                 mul2(dxp, make_float2(Bv[2], Bv[3])));
                float2 y2 = mul2(make_float2(Cv[0], Cv[1]), h0);
                y2 = fma2(make_float2(Cv[2], Cv[3]), h1, y2);
                yp[r] = y2.x + y2.y;
                const int64_t srow = SLOTS ? state_row(a, breq0 + r0 + r, tid == 0) : breq0 + r0 + r;
                if (dvalid && srow >= 0)
                    stg[(srow * a.d_inner + d) * Q + q] = make_float4(h0.x, h0.y, h1.x, h1.y);
            }
        }
        // every lane of the warp has read the group's stages
        __syncwarp();
        if (lane == 0)
            for (int r = 0; r < nr; ++r) mbar_arrive(&empty[(r0 + r) % STAGES]);
        const float y = reduce_transpose<Q>(yp, q);
        if (dvalid && q < nr && (!SLOTS || state_row(a, breq0 + r0 + q, false) >= 0))
            outg[(breq0 + r0 + q) * a.d_inner + d] = from_f32<IoT>(fmaf(y, gate, skg));
        if (*abort_flag) break;
    }
}

}  // namespace jssm
