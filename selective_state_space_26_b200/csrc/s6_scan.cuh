// s6_scan.cuh -- prefill selective scan (S6) kernel for sm_100a.
//
// Computes, for every sequence b, channel d and step t (the recurrence of the
// "Mamba 레이어" section of the Jamba notes, with the discretisation and the
// output gate read as exp(Delta A), Delta B x and (C.h + D x) silu(z)):
//     Delta  = softplus(delta[b,t,d] + delta_bias[d])
//     h[n]   = exp(Delta A[d,n]) h[n] + Delta B[b,t,n] x[b,t,d]      n < N
//     out    = (sum_n C[b,t,n] h[n] + D[d] x[b,t,d]) * silu(z[b,t,d])
// and finally h_final[b,d,:] = h.
//
// Design (B200-first; details and the roofline in the design doc):
//  * Time-serial per lane, exps computed exactly once.  A channel's N fp32
//    states live in registers of G lanes of one warp (N/G states per lane) and
//    are carried across the whole sequence, so there is no cross-chunk carry,
//    no second pass and no recomputation of exp(Delta A) -- the transcendental
//    pipe (MUFU) is the roof of this kernel, not HBM.
//  * Work per step that does not depend on n (softplus, Delta x, the gate) is
//    computed once per (t, d): in each group of G consecutive steps lane `sub`
//    owns step sub, and Delta / Delta x are exchanged with warp shuffles; the
//    G partial sums of C.h are combined with a transposing butterfly so the
//    owning lane ends up with the full sum of its step.
//  * Persistent CTAs: a task is (sequence, group of CC channels); CTAs loop
//    over tasks with a grid-stride so the grid can be sized to the SM count.
//  * Per time tile of TT steps one thread issues TMA (cp.async.bulk.tensor,
//    no multicast) loads of the x, delta, z tiles [TT x CC] and of the B, C
//    tiles [TT x N] into a STAGES-deep shared-memory ring signalled by
//    mbarriers; B/C are widened to fp32 once per tile and read back as
//    broadcast 128-bit loads by all channels of the CTA; the output tile is
//    written to shared memory and stored with one TMA store (double-buffered).
//  * Every mbarrier wait is bounded; a wait that runs out records
//    JAMBA_SSM_ERR_TIMEOUT in the device status word, waits (bounded) for the
//    copies this CTA still has in flight, and the CTA returns.
#pragma once

#include "device_utils.cuh"
#include "s6_math.cuh"

namespace jssm {

__device__ int g_status_word;  // sticky device-side status (0 = ok)

struct ScanArgs {
    int64_t batch, seqlen, d_inner;
    const float *A, *D, *delta_bias, *h0;
    float *h_final;
    int delta_softplus;
    uint32_t debug_flags;
    uint64_t timeout_cycles;
};

template <typename IoT, int N_, int G_, int NW_, int TT_, int STAGES_>
struct ScanCfg {
    static constexpr int N = N_, G = G_, NW = NW_, TT = TT_, STAGES = STAGES_;
    static constexpr int NS = N / G;        // states per lane
    static constexpr int CW = 32 / G;       // channels per warp
    static constexpr int CC = NW * CW;      // channels per CTA tile
    static constexpr int kThreads = NW * 32;
    static_assert(NS % 4 == 0, "each lane reads its B/C slice as float4");
    static_assert(32 % G == 0 && G >= 1, "lanes per channel must divide the warp");
    static constexpr int kActTile = TT * CC * (int)sizeof(IoT);  // x / delta / z / out tile
    static constexpr int kBCTile = TT * N * (int)sizeof(IoT);
    static constexpr int kStageBytes = 3 * kActTile + 2 * kBCTile;
    static_assert(kActTile % 128 == 0 && kBCTile % 128 == 0, "TMA destinations 128B aligned");
    static constexpr int kOffBCf = STAGES * kStageBytes;            // float [TT][2N]
    static constexpr int kOffOut = kOffBCf + TT * 2 * N * 4;        // IoT [2][TT][CC]
    static constexpr int kOffBar = kOffOut + 2 * kActTile;          // uint64 [STAGES]
    static constexpr int kOffFlag = kOffBar + STAGES * 8;
    static constexpr int kSmemBytes = kOffFlag + 16;
    static constexpr uint32_t kTxBytes = kStageBytes;
};

// Sum over the G lanes of a channel of v[j], delivered to lane sub == j:
// a butterfly where each round every lane keeps the half of its values its
// own index selects and sends the other half to the partner lane.
template <int G>
__device__ __forceinline__ float reduce_transpose(const float (&v)[G], int sub) {
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

template <typename IoT, int N, int G, int NW, int TT, int STAGES>
__global__ void __launch_bounds__(NW * 32, 1)
    s6_scan_fwd_kernel(const __grid_constant__ CUtensorMap tm_x,
                       const __grid_constant__ CUtensorMap tm_dt,
                       const __grid_constant__ CUtensorMap tm_z,
                       const __grid_constant__ CUtensorMap tm_B,
                       const __grid_constant__ CUtensorMap tm_C,
                       const __grid_constant__ CUtensorMap tm_out, const ScanArgs args) {
    using Cfg = ScanCfg<IoT, N, G, NW, TT, STAGES>;
    constexpr int NS = Cfg::NS, CW = Cfg::CW, CC = Cfg::CC;
    extern __shared__ __align__(1024) uint8_t smem[];
    uint64_t *full = reinterpret_cast<uint64_t *>(smem + Cfg::kOffBar);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + Cfg::kOffFlag);
    float *bcf = reinterpret_cast<float *>(smem + Cfg::kOffBCf);

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int c_local = warp * CW + lane / G;  // channel inside the CTA tile
    const int sub = lane % G;                  // which N/G-slice of the states
    const int64_t d_inner = args.d_inner, seqlen = args.seqlen;
    const int64_t ngroups = (d_inner + CC - 1) / CC;
    const int64_t ntasks = args.batch * ngroups;
    const int ntiles = static_cast<int>((seqlen + TT - 1) / TT);
    const uint64_t limit = args.timeout_cycles;
    const bool use_softplus = args.delta_softplus != 0;

    auto stage_base = [&](int s) { return smem + s * Cfg::kStageBytes; };

    if (tid == 0) {
        for (int s = 0; s < STAGES; ++s) mbar_init(&full[s], 1);
        *abort_flag = 0;
        fence_mbarrier_init();
        prefetch_tensormap(&tm_x);
        prefetch_tensormap(&tm_dt);
        prefetch_tensormap(&tm_z);
        prefetch_tensormap(&tm_B);
        prefetch_tensormap(&tm_C);
        prefetch_tensormap(&tm_out);
    }
    __syncthreads();

    // Producer side (thread 0 only): stages holding an issued, unconsumed load.
    uint32_t armed = 0;
    auto issue = [&](uint32_t g, int64_t b, int c0, int tile) {
        const int s = static_cast<int>(g % STAGES);
        if ((args.debug_flags & 1u) && tile == 0) return;  // test hook: withhold tile 0
        uint8_t *base = stage_base(s);
        mbar_arrive_expect_tx(&full[s], Cfg::kTxBytes);
        const int t0 = tile * TT, bb = static_cast<int>(b);
        tma_load_3d(base, &tm_x, c0, t0, bb, &full[s]);
        tma_load_3d(base + Cfg::kActTile, &tm_dt, c0, t0, bb, &full[s]);
        tma_load_3d(base + 2 * Cfg::kActTile, &tm_z, c0, t0, bb, &full[s]);
        tma_load_3d(base + 3 * Cfg::kActTile, &tm_B, 0, t0, bb, &full[s]);
        tma_load_3d(base + 3 * Cfg::kActTile + Cfg::kBCTile, &tm_C, 0, t0, bb, &full[s]);
        armed |= 1u << s;
    };

    uint32_t it = 0;  // tiles consumed by this CTA so far (stage / phase counter)
    bool aborted = false;
    for (int64_t task = blockIdx.x; task < ntasks && !aborted; task += gridDim.x) {
        const int64_t b = task / ngroups;
        const int c0 = static_cast<int>((task % ngroups) * CC);
        const int64_t d = c0 + c_local;
        const bool dvalid = d < d_inner;

        float a2[NS], h[NS];
#pragma unroll
        for (int i = 0; i < NS; ++i) {
            const int n = sub * NS + i;
            a2[i] = dvalid ? __ldg(args.A + d * N + n) * kLog2e : 0.0f;
            h[i] = (dvalid && args.h0) ? __ldg(args.h0 + (b * d_inner + d) * N + n) : 0.0f;
        }
        const float dskip = (dvalid && args.D) ? __ldg(args.D + d) : 0.0f;
        const float bias = (dvalid && args.delta_bias) ? __ldg(args.delta_bias + d) : 0.0f;

        if (tid == 0) {
            const int pre = ntiles < STAGES ? ntiles : STAGES;
            for (int k = 0; k < pre; ++k) issue(it + k, b, c0, k);
        }

        for (int k = 0; k < ntiles; ++k, ++it) {
            const int s = static_cast<int>(it % STAGES);
            const uint32_t phase = (it / STAGES) & 1u;
            const bool ok = mbar_wait_bounded(&full[s], phase, limit);
            const uint8_t *base = stage_base(s);
            if (ok) {
                // widen this tile's B and C to fp32, interleaved per step: [B(0..N) C(0..N)]
                const IoT *Bs = reinterpret_cast<const IoT *>(base + 3 * Cfg::kActTile);
                const IoT *Cs = reinterpret_cast<const IoT *>(base + 3 * Cfg::kActTile +
                                                              Cfg::kBCTile);
                for (int i = tid; i < TT * N; i += Cfg::kThreads) {
                    const int t = i / N, n = i % N;
                    bcf[t * 2 * N + n] = to_f32(Bs[i]);
                    bcf[t * 2 * N + N + n] = to_f32(Cs[i]);
                }
            } else {
                *abort_flag = 1;
                atomicCAS(&g_status_word, 0, 5 /* JAMBA_SSM_ERR_TIMEOUT */);
            }
            __syncthreads();  // (A) tile + fp32 B/C visible to all; abort decision uniform
            if (*abort_flag) {
                aborted = true;
                break;
            }
            if (tid == 0) armed &= ~(1u << s);

            const IoT *xs = reinterpret_cast<const IoT *>(base);
            const IoT *dts = reinterpret_cast<const IoT *>(base + Cfg::kActTile);
            const IoT *zs = reinterpret_cast<const IoT *>(base + 2 * Cfg::kActTile);
            IoT *outs = reinterpret_cast<IoT *>(smem + Cfg::kOffOut + (it & 1u) * Cfg::kActTile);
            const int nsteps =
                static_cast<int>((seqlen - int64_t(k) * TT) < TT ? (seqlen - int64_t(k) * TT) : TT);

            for (int tg = 0; tg * G < nsteps; ++tg) {
                const int t_own = tg * G + sub;
                const int idx = t_own * CC + c_local;
                const float xo = to_f32(xs[idx]);
                const float zo = to_f32(zs[idx]);
                const float dl = delta_f32(to_f32(dts[idx]), bias, use_softplus);
                const float dx = dl * xo;
                float dls[G], dxs[G], ys[G];
                if constexpr (G == 1) {
                    dls[0] = dl;
                    dxs[0] = dx;
                } else {
#pragma unroll
                    for (int j = 0; j < G; ++j) {
                        const int src = (lane & ~(G - 1)) | j;
                        dls[j] = __shfl_sync(0xffffffffu, dl, src);
                        dxs[j] = __shfl_sync(0xffffffffu, dx, src);
                    }
                }
#pragma unroll
                for (int j = 0; j < G; ++j) {
                    ys[j] = 0.0f;
                    if (tg * G + j < nsteps) {  // warp-uniform
                        const float4 *row =
                            reinterpret_cast<const float4 *>(bcf + (tg * G + j) * 2 * N);
                        float bv[NS], cv[NS];
#pragma unroll
                        for (int q = 0; q < NS / 4; ++q) {
                            const float4 bq = row[(sub * NS) / 4 + q];
                            const float4 cq = row[(N + sub * NS) / 4 + q];
                            bv[4 * q] = bq.x; bv[4 * q + 1] = bq.y;
                            bv[4 * q + 2] = bq.z; bv[4 * q + 3] = bq.w;
                            cv[4 * q] = cq.x; cv[4 * q + 1] = cq.y;
                            cv[4 * q + 2] = cq.z; cv[4 * q + 3] = cq.w;
                        }
                        float y0 = 0.0f, y1 = 0.0f;
#pragma unroll
                        for (int i = 0; i < NS; ++i) {
                            const float abar = ex2_mufu(dls[j] * a2[i]);
                            h[i] = fmaf(abar, h[i], dxs[j] * bv[i]);
                            if (i & 1) y1 = fmaf(cv[i], h[i], y1);
                            else y0 = fmaf(cv[i], h[i], y0);
                        }
                        ys[j] = y0 + y1;
                    }
                }
                const float y = reduce_transpose<G>(ys, sub);
                if (t_own < nsteps)
                    outs[idx] = from_f32<IoT>((y + dskip * xo) * silu_f32(zo));
            }

            fence_proxy_async_smem();  // make the output tile visible to the TMA store
            __syncthreads();           // (B) stage s and the fp32 B/C are free again
            if (tid == 0) {
                tma_store_3d(&tm_out, outs, c0, k * TT, static_cast<int>(b));
                bulk_commit();
                if (k + STAGES < ntiles) {
                    fence_proxy_async_smem();
                    issue(it + STAGES, b, c0, k + STAGES);
                }
                bulk_wait_read<1>();  // the other output buffer may be rewritten next tile
            }
        }

        if (!aborted && dvalid && args.h_final) {
#pragma unroll
            for (int i = 0; i < NS; ++i) args.h_final[(b * d_inner + d) * N + sub * NS + i] = h[i];
        }
    }

    if (tid == 0) {
        // Drain: loads still armed after an abort, then every store.
        for (int s = 0; s < STAGES; ++s) {
            if (armed & (1u << s)) {
                // phase of the pending load on stage s is that of the next tile using it
                uint32_t g = it;
                while (g % STAGES != static_cast<uint32_t>(s)) ++g;
                mbar_wait_bounded(&full[s], (g / STAGES) & 1u, limit);
            }
        }
        bulk_wait<0>();
    }
}

}  // namespace jssm
