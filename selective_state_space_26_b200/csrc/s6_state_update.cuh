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
// store (a warp touches 512 contiguous bytes); each thread does UNITS such
// float4s so enough loads are in flight to cover the HBM latency.  The partial
// sums of C.h are combined with Q-1 xor-shuffles; the per-(b, d) scalars (softplus, gate) are
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
        int64_t bd[2];
#pragma unroll
        for (int u = 0; u < 2; ++u) {
            const int64_t b = b0 + j + u;
            valid[u] = dvalid && b < a.batch;
            const int64_t bc = b < a.batch ? b : a.batch - 1;
            bd[u] = bc * a.d_inner + dc;
            h4[u] = st[bd[u] * Q + q];
            load4<IoT>(static_cast<const IoT *>(a.B) + bc * N + 4 * q, Bv[u]);
            load4<IoT>(static_cast<const IoT *>(a.C) + bc * N + 4 * q, Cv[u]);
            xv[u] = to_f32(x[bd[u]]);
            dtv[u] = to_f32(dt[bd[u]]);
            zv[u] = to_f32(z[bd[u]]);
        }
#pragma unroll
        for (int u = 0; u < 2; ++u) {
            const float dl = delta_f32(dtv[u], bias, use_softplus);
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
                st[bd[u] * Q + q] = make_float4(h[0], h[1], h[2], h[3]);
                if (q == 0) {
                    const float o = (y + dskip * xv[u]) * silu_f32(zv[u]);
                    static_cast<IoT *>(a.out)[bd[u]] = from_f32<IoT>(o);
                }
            }
        }
    }
}

// Streaming form for the usual shapes (d_inner a multiple of 16 bytes of I/O):
// a CTA owns one block of CPB channels and walks BPC requests; thread 0 keeps a
// STAGES-deep
// ring of 1-D bulk copies (no multicast) in flight -- the request's CPB x N fp32
// state slab (contiguous), its x / delta / z slices and its B / C rows -- so
// the bytes in flight per SM are set by shared memory, not by registers.  The
// threads read their float4 of state from shared memory, update it and write
// it back to HBM with coalesced 128-bit stores.  Waits are bounded; on a
// timeout the CTA records JAMBA_SSM_ERR_TIMEOUT and stops after the barrier.
template <typename IoT, int N, int CPB, int STAGES>
struct UpdateCfg {
    static constexpr int Q = N / 4;
    static constexpr int kThreads = CPB * Q;
    static constexpr int kStateBytes = CPB * N * 4;
    static constexpr int kActBytes = CPB * (int)sizeof(IoT);
    static constexpr int kBCBytes = N * (int)sizeof(IoT);
    static constexpr int kStage = kStateBytes + 3 * kActBytes + 2 * kBCBytes;
    static_assert(kActBytes % 16 == 0 && kBCBytes % 16 == 0 && kStage % 16 == 0, "bulk sizes");
    static constexpr int kOffBar = STAGES * kStage;
    static constexpr int kSmemBytes = kOffBar + STAGES * 8 + 16;
};

template <typename IoT, int N, int CPB, int BPC, int STAGES>
__global__ void __launch_bounds__(CPB *(N / 4), 6) s6_state_update_stream_kernel(const UpdateArgs a,
                                                                            uint64_t limit) {
    using Cfg = UpdateCfg<IoT, N, CPB, STAGES>;
    constexpr int Q = Cfg::Q;
    extern __shared__ __align__(1024) uint8_t smem[];
    uint64_t *full = reinterpret_cast<uint64_t *>(smem + Cfg::kOffBar);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + Cfg::kOffBar + STAGES * 8);
    const int tid = threadIdx.x, q = tid % Q, cl = tid / Q;
    // This CTA: channel block blockIdx.x, requests [blockIdx.y * BPC, +BPC).
    const int64_t breq0 = static_cast<int64_t>(blockIdx.y) * BPC;
    const int nu = static_cast<int>(a.batch - breq0 < BPC ? a.batch - breq0 : BPC);
    const IoT *xg = static_cast<const IoT *>(a.x);
    const IoT *dtg = static_cast<const IoT *>(a.delta);
    const IoT *zg = static_cast<const IoT *>(a.z);
    const IoT *Bg = static_cast<const IoT *>(a.B);
    const IoT *Cg = static_cast<const IoT *>(a.C);

    if (tid == 0) {
        for (int s = 0; s < STAGES; ++s) mbar_init(&full[s], 1);
        *abort_flag = 0;
        fence_mbarrier_init();
    }
    __syncthreads();
    // (channel block, request) cursors advance by one unit without divisions
    struct Unit {
        int64_t blk, b;
        __device__ void next(int64_t batch) {
            if (++b == batch) {
                b = 0;
                ++blk;
            }
        }
    };
    const Unit first{static_cast<int64_t>(blockIdx.x), breq0};
    Unit icur = first;  // thread 0: next unit to load
    auto issue = [&](int j) {  // thread 0, called for j = 0, 1, 2, ... in order
        const int64_t blk = icur.blk, b = icur.b;
        icur.next(a.batch);
        const int64_t d0 = blk * CPB;
        const int nd = static_cast<int>(a.d_inner - d0 < CPB ? a.d_inner - d0 : CPB);
        const uint32_t state_bytes = static_cast<uint32_t>(nd) * N * 4;
        const uint32_t act_bytes = static_cast<uint32_t>(nd) * sizeof(IoT);
        const int s = j % STAGES;
        uint8_t *st = smem + s * Cfg::kStage;
        const int64_t row = b * a.d_inner + d0;
        mbar_arrive_expect_tx(&full[s], state_bytes + 3 * act_bytes + 2 * Cfg::kBCBytes);
        bulk_load_1d(st, a.state + row * N, state_bytes, &full[s]);
        bulk_load_1d(st + Cfg::kStateBytes, xg + row, act_bytes, &full[s]);
        bulk_load_1d(st + Cfg::kStateBytes + Cfg::kActBytes, dtg + row, act_bytes, &full[s]);
        bulk_load_1d(st + Cfg::kStateBytes + 2 * Cfg::kActBytes, zg + row, act_bytes, &full[s]);
        bulk_load_1d(st + Cfg::kStateBytes + 3 * Cfg::kActBytes, Bg + b * N, Cfg::kBCBytes, &full[s]);
        bulk_load_1d(st + Cfg::kStateBytes + 3 * Cfg::kActBytes + Cfg::kBCBytes, Cg + b * N,
                     Cfg::kBCBytes, &full[s]);
    };
    int issued = nu < STAGES ? nu : STAGES;
    if (tid == 0)
        for (int j = 0; j < issued; ++j) issue(j);

    const bool use_softplus = a.delta_softplus != 0;
    int64_t cur_blk = -1;
    float Av[4] = {0.0f, 0.0f, 0.0f, 0.0f};
    float bias = 0.0f, dskip = 0.0f;
    Unit cur = first;
    for (int j = 0; j < nu; ++j, cur.next(a.batch)) {
        const int64_t blk = cur.blk, b = cur.b;
        const int64_t d0 = blk * CPB;
        const int nd = static_cast<int>(a.d_inner - d0 < CPB ? a.d_inner - d0 : CPB);
        const bool dvalid = cl < nd;
        const int c = dvalid ? cl : nd - 1;
        const int64_t d = d0 + c;
        if (blk != cur_blk) {  // parameters of this channel block
            cur_blk = blk;
            load4<float>(a.A + d * N + 4 * q, Av);
#pragma unroll
            for (int i = 0; i < 4; ++i) Av[i] *= kLog2e;
            bias = a.delta_bias ? __ldg(a.delta_bias + d) : 0.0f;
            dskip = a.D ? __ldg(a.D + d) : 0.0f;
        }
        const int s = j % STAGES;
        const uint8_t *st = smem + s * Cfg::kStage;
        if (mbar_wait_bounded(&full[s], static_cast<uint32_t>(j / STAGES) & 1u, limit)) {
            const float4 h4 = reinterpret_cast<const float4 *>(st)[c * Q + q];
            const IoT *xs = reinterpret_cast<const IoT *>(st + Cfg::kStateBytes);
            const IoT *dts = xs + CPB, *zs = dts + CPB;
            const IoT *Bs = zs + CPB, *Cs = Bs + N;
            float Bv[4], Cv[4];
            load4<IoT>(Bs + 4 * q, Bv);
            load4<IoT>(Cs + 4 * q, Cv);
            const float xv = to_f32(xs[c]);
            const float dl = delta_f32(to_f32(dts[c]), bias, use_softplus);
            const float dx = dl * xv;
            float h[4] = {h4.x, h4.y, h4.z, h4.w};
            float y = 0.0f;
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const float abar = ex2_mufu(dl * Av[i]);
                h[i] = fmaf(abar, h[i], dx * Bv[i]);
                y = fmaf(Cv[i], h[i], y);
            }
#pragma unroll
            for (int off = 1; off < Q; off <<= 1) y += __shfl_xor_sync(0xffffffffu, y, off);
            if (dvalid) {
                const int64_t bd = b * a.d_inner + d;
                reinterpret_cast<float4 *>(a.state)[bd * Q + q] = make_float4(h[0], h[1], h[2], h[3]);
                if (q == 0)
                    static_cast<IoT *>(a.out)[bd] =
                        from_f32<IoT>((y + dskip * xv) * silu_f32(to_f32(zs[c])));
            }
        } else {
            *abort_flag = 1;
            atomicCAS(&g_status_word, 0, 5 /* JAMBA_SSM_ERR_TIMEOUT */);
        }
        __syncthreads();  // stage s has been read by every thread
        if (*abort_flag) break;
        if (tid == 0 && issued < nu) {
            fence_proxy_async_smem();
            issue(issued);
            ++issued;
        }
    }
    if (tid == 0 && *abort_flag) {
        // loads still in flight on the ring: wait (bounded) before the CTA exits
        for (int j = 0; j < issued; ++j)
            mbar_wait_bounded(&full[j % STAGES], static_cast<uint32_t>(j / STAGES) & 1u, limit);
    }
}

}  // namespace jssm
