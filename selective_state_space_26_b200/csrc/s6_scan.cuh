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
// Design (B200-first; the roofline is in the design doc):
//  * Time-serial per lane, exps computed exactly once.  A channel's N fp32
//    states live in registers of G lanes of one warp (N/G states per lane) and
//    are carried across the whole sequence, so there is no cross-chunk carry,
//    no second pass and no recomputation of exp(Delta A): the transcendental
//    pipe (MUFU, 16 ops/clk/SM) is the roof of this kernel, not HBM.
//  * Warp-specialised pipeline over time tiles of TT steps.  A CTA owns CC
//    channels of one sequence (a task) and walks its tiles in order:
//      - a producer warp issues TMA loads (cp.async.bulk.tensor, no multicast)
//        of the x, delta, z tiles [TT x CC] and the B, C tiles [TT x N] into a
//        STAGES-deep ring (mbarrier `full`) and the TMA stores of the output
//        tiles (mbarriers `out_full` / `out_free`);
//      - the NWS scalar warps run phase A of tile g+1 -- Delta =
//        softplus(delta + bias) and Delta x for every (t, d), B and C widened to
//        fp32 -- into double-buffered shared memory (mbarrier `a_done`), then
//        phase C of tile g -- out = (y + D x) silu(z) with y = C.h -- into a
//        double-buffered output tile;
//      - the NWB recurrence warps run phase B of tile g: lane (d, sub) carries
//        its N/G states through the TT steps (Abar = 2^(Delta A log2 e) on the
//        MUFU, h = Abar h + Delta x B, partial C.h to shared memory; mbarrier
//        `b_done`).
//    Phase B is MUFU-bound; A and C (one softplus and one gate per (t, d))
//    overlap it on the other warps instead of stalling the recurrence.
//  * Persistent CTAs: tasks are (sequence, group of CC channels) and CTAs walk
//    them with a grid stride, so the grid is sized to the SM count; the tiles of
//    a CTA's tasks form one stream so the pipeline never drains between tasks.
//  * Every wait is a bounded mbarrier wait that also watches a CTA abort flag;
//    there is no unbounded barrier in the loop.  A wait that runs out records
//    JAMBA_SSM_ERR_TIMEOUT in the device status word and sets the flag; every
//    warp then leaves its loop, and the producer waits (bounded) for its loads
//    and stores still in flight before the CTA exits.
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

template <typename IoT, int N_, int G_, int NWB_, int NWS_, int TT_, int STAGES_>
struct ScanCfg {
    static constexpr int N = N_, G = G_, NWB = NWB_, NWS = NWS_, TT = TT_, STAGES = STAGES_;
    static constexpr int NS = N / G;          // states per recurrence lane
    static constexpr int CW = 32 / G;         // channels per recurrence warp
    static constexpr int CC = NWB * CW;       // channels per CTA tile
    static constexpr int kThreads = (NWB + NWS + 1) * 32;  // + one TMA producer warp
    static constexpr int kScalarThreads = NWS * 32;
    static constexpr int PAIRS = CC / 2;      // scalar threads own channel pairs
    static constexpr int ROWSTEP = kScalarThreads / PAIRS;
    static constexpr int ROWS = TT / ROWSTEP; // rows of a tile per scalar thread
    static constexpr int VEC = 16 / (int)sizeof(IoT);  // B/C elements per 16-byte load
    static_assert(NS % 4 == 0, "each lane reads its B/C slice as float4");
    static_assert(32 % G == 0 && G >= 1, "lanes per channel must divide the warp");
    static_assert(kScalarThreads % PAIRS == 0 && TT % ROWSTEP == 0, "scalar row mapping");
    static_assert(N % VEC == 0, "B/C rows are widened 16 bytes at a time");
    static_assert(STAGES >= 2 && STAGES <= 8, "TMA ring depth");
    static constexpr int kActTile = TT * CC * (int)sizeof(IoT);  // x / delta / z / out tile
    static constexpr int kBCTile = TT * N * (int)sizeof(IoT);
    static constexpr int kStageBytes = 3 * kActTile + 2 * kBCTile;
    static_assert(kActTile % 128 == 0 && kBCTile % 128 == 0, "TMA destinations 128B aligned");
    static constexpr int kBCRow = 2 * N + 4;    // fp32 B/C row [B(N) C(N) pad]: the pad
                                                // spreads consecutive rows over banks
    static constexpr int kBCf = TT * kBCRow;    // floats per fp32 B/C slot
    static constexpr int kDD = TT * CC;         // float2 per Delta slot
    static constexpr int kYP = TT * CC;         // floats per C.h slot
    static constexpr int kOffBCf = STAGES * kStageBytes;
    static constexpr int kOffDD = kOffBCf + 2 * kBCf * 4;
    static constexpr int kOffYP = kOffDD + 2 * kDD * 8;
    static constexpr int kOffOut = kOffYP + 2 * kYP * 4;
    // full[S], a_done[2], b_done[2], out_full[2], out_free[2]
    static constexpr int kOffBar = kOffOut + 2 * kActTile;
    static constexpr int kNumBars = STAGES + 8;
    static constexpr int kOffFlag = kOffBar + kNumBars * 8;
    static constexpr int kSmemBytes = kOffFlag + 16;
    static constexpr uint32_t kTxBytes = kStageBytes;
};

// Two consecutive I/O elements as floats / back.
__device__ __forceinline__ float2 unpack2(uint32_t v) {
    return make_float2(__uint_as_float(v << 16), __uint_as_float(v & 0xffff0000u));
}
__device__ __forceinline__ float2 unpack2(uint2 v) {
    return make_float2(__uint_as_float(v.x), __uint_as_float(v.y));
}
template <typename IoT> struct Pair;
template <> struct Pair<__nv_bfloat16> { using T = uint32_t; };
template <> struct Pair<float> { using T = uint2; };

__device__ __forceinline__ void store2(__nv_bfloat16 *p, float a, float b) {
    *reinterpret_cast<__nv_bfloat162 *>(p) = __floats2bfloat162_rn(a, b);
}
__device__ __forceinline__ void store2(float *p, float a, float b) {
    *reinterpret_cast<float2 *>(p) = make_float2(a, b);
}

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

// Sum of v over the G lanes of a channel (lanes lane^1, lane^2, ...).
template <int G>
__device__ __forceinline__ float lane_group_sum(float v) {
#pragma unroll
    for (int off = 1; off < G; off <<= 1) v += __shfl_xor_sync(0xffffffffu, v, off);
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
// partial sum of C.h is returned.
template <int N, int NS>
__device__ __forceinline__ float recurrence_step(float (&h)[NS], const float (&a2)[NS],
                                                 float2 dlx, const float *bcrow, int sub) {
    const float4 *row = reinterpret_cast<const float4 *>(bcrow);
    float y0 = 0.0f, y1 = 0.0f;
#pragma unroll
    for (int q = 0; q < NS / 4; ++q) {
        const float4 bq = row[(sub * NS) / 4 + q];
        const float4 cq = row[(N + sub * NS) / 4 + q];
        const float bv[4] = {bq.x, bq.y, bq.z, bq.w};
        const float cv[4] = {cq.x, cq.y, cq.z, cq.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const int i = 4 * q + e;
            const float abar = ex2_mufu(dlx.x * a2[i]);
            h[i] = fmaf(abar, h[i], dlx.y * bv[e]);
            if (e & 1) y1 = fmaf(cv[e], h[i], y1);
            else y0 = fmaf(cv[e], h[i], y0);
        }
    }
    return y0 + y1;
}

template <typename IoT, int N, int G, int NWB, int NWS, int TT, int STAGES>
__global__ void __launch_bounds__((NWB + NWS + 1) * 32, 1)
    s6_scan_fwd_kernel(const __grid_constant__ CUtensorMap tm_x,
                       const __grid_constant__ CUtensorMap tm_dt,
                       const __grid_constant__ CUtensorMap tm_z,
                       const __grid_constant__ CUtensorMap tm_B,
                       const __grid_constant__ CUtensorMap tm_C,
                       const __grid_constant__ CUtensorMap tm_out, const ScanArgs args) {
    using Cfg = ScanCfg<IoT, N, G, NWB, NWS, TT, STAGES>;
    constexpr int NS = Cfg::NS, CW = Cfg::CW, CC = Cfg::CC, PAIRS = Cfg::PAIRS;
    constexpr int ROWSTEP = Cfg::ROWSTEP, ROWS = Cfg::ROWS, VEC = Cfg::VEC;
    using PairT = typename Pair<IoT>::T;
    extern __shared__ __align__(1024) uint8_t smem[];
    uint64_t *full = reinterpret_cast<uint64_t *>(smem + Cfg::kOffBar);
    uint64_t *a_done = full + STAGES;
    uint64_t *b_done = a_done + 2;
    uint64_t *out_full = b_done + 2;
    uint64_t *out_free = out_full + 2;
    volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + Cfg::kOffFlag);
    float *bcf_all = reinterpret_cast<float *>(smem + Cfg::kOffBCf);
    float2 *dd_all = reinterpret_cast<float2 *>(smem + Cfg::kOffDD);
    float *yp_all = reinterpret_cast<float *>(smem + Cfg::kOffYP);

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int64_t d_inner = args.d_inner, seqlen = args.seqlen;
    const int64_t ngroups = (d_inner + CC - 1) / CC;
    const int64_t ntasks = args.batch * ngroups;
    const int ntiles = static_cast<int>((seqlen + TT - 1) / TT);
    const int64_t my_tasks =
        static_cast<int64_t>(blockIdx.x) < ntasks ? (ntasks - 1 - blockIdx.x) / gridDim.x + 1 : 0;
    const int64_t total = my_tasks * ntiles;  // tiles this CTA walks
    const uint64_t limit = args.timeout_cycles;

    if (tid == 0) {
        for (int s = 0; s < STAGES; ++s) mbar_init(&full[s], 1);
        mbar_init(&a_done[0], Cfg::kScalarThreads);
        mbar_init(&a_done[1], Cfg::kScalarThreads);
        mbar_init(&b_done[0], NWB * 32);
        mbar_init(&b_done[1], NWB * 32);
        mbar_init(&out_full[0], Cfg::kScalarThreads);
        mbar_init(&out_full[1], Cfg::kScalarThreads);
        mbar_init(&out_free[0], 1);
        mbar_init(&out_free[1], 1);
        *abort_flag = 0;
        fence_mbarrier_init();
    }
    __syncthreads();

    auto fail = [&]() {
        *abort_flag = 1;
        atomicCAS(&g_status_word, 0, 5 /* JAMBA_SSM_ERR_TIMEOUT */);
    };
    // (sequence, first channel, tile index) of the CTA's g-th tile
    auto tile_of = [&](int64_t g, int64_t &b, int &c0, int &k) {
        const int64_t j = g / ntiles;
        k = static_cast<int>(g - j * ntiles);
        const int64_t task = blockIdx.x + j * gridDim.x;
        b = task / ngroups;
        c0 = static_cast<int>((task % ngroups) * CC);
    };
    auto steps_in = [&](int k) {
        const int64_t rem = seqlen - int64_t(k) * TT;
        return static_cast<int>(rem < TT ? rem : TT);
    };

    if (warp < NWB) {
        // =================== recurrence warps: phase B ===================
        const int c_local = warp * CW + lane / G;
        const int sub = lane % G;
        float a2[NS], h[NS];
        int64_t d = 0;
        bool dvalid = false;
        for (int64_t g = 0; g < total; ++g) {
            int64_t b;
            int c0, k;
            tile_of(g, b, c0, k);
            if (k == 0) {
                d = c0 + c_local;
                dvalid = d < d_inner;
#pragma unroll
                for (int i = 0; i < NS; ++i) {
                    const int n = sub * NS + i;
                    a2[i] = dvalid ? __ldg(args.A + d * N + n) * kLog2e : 0.0f;
                    h[i] = (dvalid && args.h0) ? __ldg(args.h0 + (b * d_inner + d) * N + n) : 0.0f;
                }
            }
            const int slot = static_cast<int>(g & 1);
            if (!mbar_wait_or_abort(&a_done[slot], static_cast<uint32_t>(g >> 1) & 1u, limit,
                                    abort_flag)) {
                fail();
                return;
            }
            const int nsteps = steps_in(k);
            const float2 *dd = dd_all + slot * Cfg::kDD;
            const float *bcf = bcf_all + slot * Cfg::kBCf;
            float *yp = yp_all + slot * Cfg::kYP;

            if (nsteps == TT) {
                // Full tile: straight-line code over the TT steps with the partial
                // sums kept in registers, so no shared-memory store sits between
                // one step's loads and the next step's (issue stays in order).
                float y[TT];
#pragma unroll
                for (int t = 0; t < TT; ++t)
                    y[t] = recurrence_step<N, NS>(h, a2, dd[t * CC + c_local],
                                                  bcf + t * Cfg::kBCRow, sub);
#pragma unroll
                for (int t0 = 0; t0 < TT; t0 += G)
                    yp[(t0 + sub) * CC + c_local] = reduce_transpose<G>(y + t0, sub);
            } else {
                // Tail tile of a sequence.
                for (int t = 0; t < nsteps; ++t) {
                    const float y = lane_group_sum<G>(recurrence_step<N, NS>(
                        h, a2, dd[t * CC + c_local], bcf + t * Cfg::kBCRow, sub));
                    if (sub == 0) yp[t * CC + c_local] = y;
                }
            }
            mbar_arrive(&b_done[slot]);
            if (k == ntiles - 1 && dvalid && args.h_final) {
#pragma unroll
                for (int i = 0; i < NS; ++i) args.h_final[(b * d_inner + d) * N + sub * NS + i] = h[i];
            }
        }
        return;
    }

    if (warp == NWB + NWS) {
        // ======================= TMA producer warp (lane 0) =======================
        if (lane != 0) return;
        uint32_t armed = 0;       // stages holding an issued, unconsumed load
        int64_t issued = 0;       // loads issued: tiles [0, issued)
        auto issue = [&](int64_t g) {
            if (g >= total) return;
            issued = g + 1;
            int64_t b;
            int c0, k;
            tile_of(g, b, c0, k);
            const int s = static_cast<int>(g % STAGES);
            if ((args.debug_flags & 1u) && k == 0) return;  // test hook: withhold a task's first tile
            uint8_t *base = smem + s * Cfg::kStageBytes;
            mbar_arrive_expect_tx(&full[s], Cfg::kTxBytes);
            const int t0 = k * TT, bb = static_cast<int>(b);
            tma_load_3d(base, &tm_x, c0, t0, bb, &full[s]);
            tma_load_3d(base + Cfg::kActTile, &tm_dt, c0, t0, bb, &full[s]);
            tma_load_3d(base + 2 * Cfg::kActTile, &tm_z, c0, t0, bb, &full[s]);
            tma_load_3d(base + 3 * Cfg::kActTile, &tm_B, 0, t0, bb, &full[s]);
            tma_load_3d(base + 3 * Cfg::kActTile + Cfg::kBCTile, &tm_C, 0, t0, bb, &full[s]);
            armed |= 1u << s;
        };
        prefetch_tensormap(&tm_x);
        prefetch_tensormap(&tm_dt);
        prefetch_tensormap(&tm_z);
        prefetch_tensormap(&tm_B);
        prefetch_tensormap(&tm_C);
        prefetch_tensormap(&tm_out);
        for (int64_t g = 0; g < STAGES; ++g) issue(g);
        int64_t consumed = 0;  // tiles whose output has been handed over (stage free again)
        bool ok = true;
        for (int64_t g = 0; g < total; ++g) {
            const int slot = static_cast<int>(g & 1);
            if (!mbar_wait_or_abort(&out_full[slot], static_cast<uint32_t>(g >> 1) & 1u, limit,
                                    abort_flag)) {
                ok = false;
                break;
            }
            consumed = g + 1;
            armed &= ~(1u << static_cast<int>(g % STAGES));
            int64_t b;
            int c0, k;
            tile_of(g, b, c0, k);
            tma_store_3d(&tm_out, smem + Cfg::kOffOut + slot * Cfg::kActTile, c0, k * TT,
                         static_cast<int>(b));
            bulk_commit();
            issue(g + STAGES);  // the scalar warps are done with stage g % STAGES
            if (g > 0) {
                bulk_wait_read<1>();               // the store of tile g-1 has read its buffer
                mbar_arrive(&out_free[slot ^ 1]);
            }
        }
        if (!ok) fail();
        // Drain: loads still armed after an abort (tiles [consumed, issued)), then
        // every store.
        for (int64_t g = consumed; g < issued; ++g) {
            const int s = static_cast<int>(g % STAGES);
            if (armed & (1u << s)) {
                mbar_wait_bounded(&full[s], static_cast<uint32_t>(g / STAGES) & 1u, limit);
                armed &= ~(1u << s);
            }
        }
        bulk_wait<0>();
        return;
    }

    // ======================= scalar warps: phases A and C =======================
    const int stid = tid - NWB * 32;
    const int pair = stid % PAIRS;
    const int row0 = stid / PAIRS;
    const bool use_softplus = args.delta_softplus != 0;

    // Per-channel parameters of this thread's channel pair.  Phase A reloads
    // them when a new task starts; the skip weights travel with the tile's
    // slot (A runs one tile ahead of C, so C may still be on the previous task).
    float bias0 = 0.0f, bias1 = 0.0f, dskT0 = 0.0f, dskT1 = 0.0f;
    float dskS0[2] = {0.0f, 0.0f}, dskS1[2] = {0.0f, 0.0f};
    auto load_pair_params = [&](int c0) {
        const int64_t dp = c0 + 2 * pair;
        const bool v0 = dp < d_inner, v1 = dp + 1 < d_inner;
        bias0 = (v0 && args.delta_bias) ? __ldg(args.delta_bias + dp) : 0.0f;
        bias1 = (v1 && args.delta_bias) ? __ldg(args.delta_bias + dp + 1) : 0.0f;
        dskT0 = (v0 && args.D) ? __ldg(args.D + dp) : 0.0f;
        dskT1 = (v1 && args.D) ? __ldg(args.D + dp + 1) : 0.0f;
    };

    // Phase A of tile g: fp32 B/C and (Delta, Delta x) into slot g & 1.
    auto phase_a = [&](int64_t g) -> bool {
        int64_t b;
        int c0, k;
        tile_of(g, b, c0, k);
        const int s = static_cast<int>(g % STAGES);
        if (!mbar_wait_or_abort(&full[s], static_cast<uint32_t>(g / STAGES) & 1u, limit,
                                abort_flag))
            return false;
        const int nsteps = steps_in(k);
        const uint8_t *base = smem + s * Cfg::kStageBytes;
        const IoT *xs = reinterpret_cast<const IoT *>(base);
        const IoT *dts = reinterpret_cast<const IoT *>(base + Cfg::kActTile);
        const IoT *Bs = reinterpret_cast<const IoT *>(base + 3 * Cfg::kActTile);
        const IoT *Cs = reinterpret_cast<const IoT *>(base + 3 * Cfg::kActTile + Cfg::kBCTile);
        const int slot = static_cast<int>(g & 1);
        float *bcf = bcf_all + slot * Cfg::kBCf;
        float2 *dd = dd_all + slot * Cfg::kDD;
        if (k == 0) load_pair_params(c0);
        if (slot == 0) {
            dskS0[0] = dskT0;
            dskS1[0] = dskT1;
        } else {
            dskS0[1] = dskT0;
            dskS1[1] = dskT1;
        }
        // B and C, 16 bytes per thread-iteration
        for (int v = stid; v < nsteps * N / VEC; v += Cfg::kScalarThreads) {
            const int t = (v * VEC) / N, n = (v * VEC) % N;
            float fb[VEC], fc[VEC];
            widen16(*reinterpret_cast<const uint4 *>(Bs + v * VEC), Bs, fb);
            widen16(*reinterpret_cast<const uint4 *>(Cs + v * VEC), Cs, fc);
#pragma unroll
            for (int q = 0; q < VEC / 4; ++q) {
                *reinterpret_cast<float4 *>(bcf + t * Cfg::kBCRow + n + 4 * q) =
                    make_float4(fb[4 * q], fb[4 * q + 1], fb[4 * q + 2], fb[4 * q + 3]);
                *reinterpret_cast<float4 *>(bcf + t * Cfg::kBCRow + N + n + 4 * q) =
                    make_float4(fc[4 * q], fc[4 * q + 1], fc[4 * q + 2], fc[4 * q + 3]);
            }
        }
        // all rows' inputs first (independent loads), then the math and stores
        PairT xr[ROWS], dr[ROWS];
#pragma unroll
        for (int j = 0; j < ROWS; ++j) {
            const int t = row0 + j * ROWSTEP;
            if (t < nsteps) {
                xr[j] = *reinterpret_cast<const PairT *>(xs + t * CC + 2 * pair);
                dr[j] = *reinterpret_cast<const PairT *>(dts + t * CC + 2 * pair);
            }
        }
#pragma unroll
        for (int j = 0; j < ROWS; ++j) {
            const int t = row0 + j * ROWSTEP;
            if (t < nsteps) {
                const float2 xv = unpack2(xr[j]), dv = unpack2(dr[j]);
                const float dl0 = delta_f32(dv.x, bias0, use_softplus);
                const float dl1 = delta_f32(dv.y, bias1, use_softplus);
                *reinterpret_cast<float4 *>(dd + t * CC + 2 * pair) =
                    make_float4(dl0, dl0 * xv.x, dl1, dl1 * xv.y);
            }
        }
        mbar_arrive(&a_done[slot]);
        return true;
    };

    // Phase C of tile g: the output tile from the sums of C.h, handed to the
    // producer warp for its TMA store (and with it, stage g % STAGES).
    auto phase_c = [&](int64_t g) -> bool {
        int64_t b;
        int c0, k;
        tile_of(g, b, c0, k);
        const int slot = static_cast<int>(g & 1);
        if (!mbar_wait_or_abort(&b_done[slot], static_cast<uint32_t>(g >> 1) & 1u, limit,
                                abort_flag))
            return false;
        const int nsteps = steps_in(k);
        const int s = static_cast<int>(g % STAGES);
        const uint8_t *base = smem + s * Cfg::kStageBytes;
        const IoT *xs = reinterpret_cast<const IoT *>(base);
        const IoT *zs = reinterpret_cast<const IoT *>(base + 2 * Cfg::kActTile);
        const float *yp = yp_all + slot * Cfg::kYP;
        const float dsk0 = slot == 0 ? dskS0[0] : dskS0[1];
        const float dsk1 = slot == 0 ? dskS1[0] : dskS1[1];
        IoT *outs = reinterpret_cast<IoT *>(smem + Cfg::kOffOut + slot * Cfg::kActTile);
        PairT xr[ROWS], zr[ROWS];
        float2 yr[ROWS];
#pragma unroll
        for (int j = 0; j < ROWS; ++j) {
            const int t = row0 + j * ROWSTEP;
            if (t < nsteps) {
                xr[j] = *reinterpret_cast<const PairT *>(xs + t * CC + 2 * pair);
                zr[j] = *reinterpret_cast<const PairT *>(zs + t * CC + 2 * pair);
                yr[j] = *reinterpret_cast<const float2 *>(yp + t * CC + 2 * pair);
            }
        }
        // the store of tile g-2 must have read this output buffer
        if (g >= 2 && !mbar_wait_or_abort(&out_free[slot], static_cast<uint32_t>((g >> 1) - 1) & 1u,
                                          limit, abort_flag))
            return false;
#pragma unroll
        for (int j = 0; j < ROWS; ++j) {
            const int t = row0 + j * ROWSTEP;
            if (t < nsteps) {
                const float2 xv = unpack2(xr[j]), zv = unpack2(zr[j]);
                const float o0 = (yr[j].x + dsk0 * xv.x) * silu_f32(zv.x);
                const float o1 = (yr[j].y + dsk1 * xv.y) * silu_f32(zv.y);
                store2(outs + t * CC + 2 * pair, o0, o1);
            }
        }
        fence_proxy_async_smem();  // output tile (and the stage reads) before the TMA store
        mbar_arrive(&out_full[slot]);
        return true;
    };

    bool ok = total == 0 || phase_a(0);
    for (int64_t g = 0; ok && g < total; ++g) {
        if (g + 1 < total) ok = phase_a(g + 1);
        if (ok) ok = phase_c(g);
    }
    if (!ok) fail();
}

}  // namespace jssm
