// s6_ssd.cuh -- the scalar-identity variant of the selective scan (Mamba-2's
// state matrix) on sm_100a.
//
// Source: "Jamba -- Hybrid SSM-Transformer" (factory.pai-world.com lesson),
// section "Mamba-3: 2026년의 순수 SSM 기준선", items 1 and 2: the state matrix
// is a scaled identity and the discretisation is Euler's.  Reading (the pages
// print no equations of this variant): d_inner = nheads * headdim channels,
// channel d = head * headdim + p; per head and token one step size
// Delta = softplus(delta[t, head] + bias[head]) and one decay
// exp(Delta A[head]), shared by all of the head's channels and states:
//     h[n] = exp(Delta A) h[n] + Delta B[t, n] x[t, d],
//     out  = (sum_n C[t, n] h[n] + D[d] x[t, d]) silu(z[t, d]).
//
// With a scalar decay the exp-class work is 4 operations per (token, channel)
// -- the gate's exp and reciprocal, plus softplus and the decay once per head
// and token -- against d_state + 4 for the diagonal scan, so this layer is not
// bound by the MUFU pipe but by issue: a lane-step is a dozen instructions
// (its table entry, x, its B and C slices, the packed update and readout).
//
// Layout: one CTA per (sequence, slice of CC channels of one head); CC divides
// headdim.  NW compute warps with G lanes per channel, NS = N / G states per
// lane on fp32 pairs; one producer warp.
//  * The producer's lane 0 feeds TT-step tiles by TMA into a STAGES ring (x, z
//    [TT x CC], the delta columns of a 16-byte box of heads [TT x 16 B], B, C
//    [TT x N]) and stores the output tiles by TMA.
//  * All producer lanes then prepare each landed tile for the compute warps:
//    the [TT] table of (Delta, decay) of the CTA's head, and B and C widened to
//    fp32 in per-lane slots (load_bc's layout), so that a compute lane-step
//    reads one broadcast table entry, one x value and two 16-byte vectors.
//  * The compute warps walk a whole tile with its loop unrolled: the G steps of
//    a group advance the states and give G partial readouts, which the
//    transposing butterfly turns into the owner lane's sum; the owners' skip,
//    gate and output stores come after the tile's last group, so nothing in the
//    walk waits on them.  NOUT output buffers let the store of tile k-1 and the
//    walk of tile k+1 proceed while the producer retires tile k.
// Every wait is bounded and watches the CTA's abort flag.
#pragma once

#include "device_utils.cuh"
#include "s6_math.cuh"
#include "s6_scan.cuh"

namespace jssm {

struct SsdArgs {
    int64_t batch, seqlen, nheads, headdim;
    const float *A, *D, *delta_bias, *h0;
    float *h_final;
    int delta_softplus;
    int *status;
    uint32_t debug_flags;
    uint64_t timeout_cycles;
};

template <typename IoT, int N, int G, int NW, int TT, int STAGES_>
struct SsdCfg {
    static constexpr int NS = N / G, NP = NS / 2, CW = 32 / G, CC = NW * CW, STAGES = STAGES_;
    static_assert(NS == 2 || NS == 4 || NS == 8, "2, 4 or 8 states per lane");
    static constexpr int kHeadsBox = 16 / (int)sizeof(IoT);  // delta columns per 16-byte row
    static constexpr int kAct = TT * CC * (int)sizeof(IoT);
    static constexpr int kDt = TT * kHeadsBox * (int)sizeof(IoT);
    static constexpr int kBC = TT * N * (int)sizeof(IoT);
    static constexpr int kStage = 2 * kAct + kDt + 2 * kBC;  // x, z, delta, B, C
    static_assert(kAct % 128 == 0 && kDt % 128 == 0 && kBC % 128 == 0, "128-byte TMA boxes");
    static constexpr int kBCRow = 2 * N;                     // widened floats per step
    static constexpr int kOffWide = STAGES * kStage;         // [STAGES][TT][2N] fp32
    static constexpr int kWide = TT * kBCRow * 4;
    static constexpr int kOffTab = kOffWide + STAGES * kWide;  // [STAGES][TT] (Delta, decay)
    static constexpr int NOUT = 3;
    static constexpr int kOffOut = kOffTab + STAGES * TT * 8;
    static_assert(kOffOut % 128 == 0, "TMA store sources 128-byte aligned");
    static constexpr int kOffBar = kOffOut + NOUT * kAct;
    static constexpr int kNumBars = 2 * STAGES + 2 * NOUT;  // full, ready, out_full, out_free
    static constexpr int kOffFlag = kOffBar + kNumBars * 8;
    static constexpr int kSmemBytes = kOffFlag + 16;
    static_assert(TT % G == 0, "whole step groups");
};

// One tile of a compute lane: TT steps if FULL, else the first `nsteps`
// (the states do not move past them; the rows past them are written to the
// output buffer but clipped by the TMA store).
template <bool FULL, typename IoT, int N, int G, int TT, int CC>
__device__ __forceinline__ void ssd_tile(float2 (&h)[N / G / 2], const float2 *tab,
                                         const float *wide, const IoT *xs, const IoT *zs,
                                         IoT *outs, float dskip, int c_local, int sub,
                                         int nsteps) {
    constexpr int NS = N / G, NP = NS / 2, NQ = TT / G;
    float yown[NQ];  // C.h of the owned steps q * G + sub
#pragma unroll
    for (int q = 0; q < NQ; ++q) {
        float yp[G];
#pragma unroll
        for (int j = 0; j < G; ++j) {
            const int t = q * G + j;
            yp[j] = 0.0f;
            if (FULL || t < nsteps) {
                const float2 dd = tab[t];
                const float dx = dd.x * to_f32(xs[t * CC + c_local]);
                const BCPairs<NS> bc = load_bc<NS>(wide + t * 2 * N, sub);
                const float2 dec2 = make_float2(dd.y, dd.y), dx2 = make_float2(dx, dx);
                float2 y2;
#pragma unroll
                for (int i = 0; i < NP; ++i) {
                    h[i] = fma2(dec2, h[i], mul2(dx2, bc.b[i]));
                    y2 = i == 0 ? mul2(bc.c[i], h[i]) : fma2(bc.c[i], h[i], y2);
                }
                yp[j] = y2.x + y2.y;
            }
        }
        yown[q] = reduce_transpose<G>(yp, sub);
    }
#pragma unroll
    for (int q = 0; q < NQ; ++q) {
        const int idx = (q * G + sub) * CC + c_local;
        const float xo = to_f32(xs[idx]);
        outs[idx] = from_f32<IoT>(fmaf(dskip, xo, yown[q]) * silu_f32(to_f32(zs[idx])));
    }
}

struct SsdMaps {
    CUtensorMap x, z, dt, B, C, out;
};

// grid (d_inner / CC, batch), (NW + 1) * 32 threads; SP: softplus on.
template <typename IoT, int N, int G, int NW, int TT, int STAGES, bool SP>
__global__ void __launch_bounds__((NW + 1) * 32, 1)
    s6_ssd_kernel(const __grid_constant__ SsdMaps maps, const SsdArgs a) {
    using Cfg = SsdCfg<IoT, N, G, NW, TT, STAGES>;
    constexpr int NS = Cfg::NS, NP = Cfg::NP, CW = Cfg::CW, CC = Cfg::CC, NOUT = Cfg::NOUT;
    extern __shared__ __align__(1024) uint8_t smem[];
    uint64_t *full = reinterpret_cast<uint64_t *>(smem + Cfg::kOffBar);
    uint64_t *ready = full + STAGES;
    uint64_t *out_full = ready + STAGES;
    uint64_t *out_free = out_full + NOUT;
    volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + Cfg::kOffFlag);

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int64_t b = blockIdx.y;
    const int c0 = blockIdx.x * CC;
    const int64_t D = a.nheads * a.headdim, L = a.seqlen;
    const int head = static_cast<int>(c0 / a.headdim);
    const int hbox = head - head % Cfg::kHeadsBox;  // first head column of the delta box
    const int ntiles = static_cast<int>((L + TT - 1) / TT);
    const uint64_t limit = a.timeout_cycles;

    if (tid == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&ready[s], 32);
        }
        for (int o = 0; o < NOUT; ++o) {
            mbar_init(&out_full[o], NW * 32);
            mbar_init(&out_free[o], 1);
        }
        *abort_flag = 0;
        fence_mbarrier_init();
    }
    __syncthreads();
    auto fail = [&]() {
        if (!*abort_flag) record_status(a.status, kStTimeout);
        *abort_flag = 1;
    };

    if (warp == NW) {
        // ============== producer: TMA, the tables, B / C widening ==============
        const int bb = static_cast<int>(b);
        const float a2 = __ldg(a.A + head) * kLog2e;
        const float bias = a.delta_bias ? __ldg(a.delta_bias + head) : 0.0f;
        int last_k[STAGES];  // lane 0: the tile whose load is in flight in each stage, or -1
        for (int s = 0; s < STAGES; ++s) last_k[s] = -1;
        auto issue = [&](int k) {  // lane 0 only; stage k % STAGES is free
            if (k >= ntiles) return;
            if ((a.debug_flags & 1u) && k == 0) return;  // test hook: withhold tile 0
            const int s = k % STAGES;
            uint8_t *st = smem + s * Cfg::kStage;
            const int t0 = k * TT;
            mbar_arrive_expect_tx(&full[s], Cfg::kStage);
            tma_load_3d(st, &maps.x, c0, t0, bb, &full[s]);
            tma_load_3d(st + Cfg::kAct, &maps.z, c0, t0, bb, &full[s]);
            tma_load_3d(st + 2 * Cfg::kAct, &maps.dt, hbox, t0, bb, &full[s]);
            tma_load_3d(st + 2 * Cfg::kAct + Cfg::kDt, &maps.B, 0, t0, bb, &full[s]);
            tma_load_3d(st + 2 * Cfg::kAct + Cfg::kDt + Cfg::kBC, &maps.C, 0, t0, bb, &full[s]);
            last_k[s] = k;
        };
        // tile k landed: its (Delta, decay) table and widened B / C
        auto prepare = [&](int k) -> bool {
            const int s = k % STAGES;
            if (!warp_agree(mbar_wait_or_abort(&full[s], (k / STAGES) & 1, limit, abort_flag)))
                return false;
            if (lane == 0) last_k[s] = -1;
            const uint8_t *st = smem + s * Cfg::kStage;
            const IoT *dts = reinterpret_cast<const IoT *>(st + 2 * Cfg::kAct);
            const IoT *Bs = reinterpret_cast<const IoT *>(st + 2 * Cfg::kAct + Cfg::kDt);
            const IoT *Cs = reinterpret_cast<const IoT *>(st + 2 * Cfg::kAct + Cfg::kDt + Cfg::kBC);
            float2 *tab = reinterpret_cast<float2 *>(smem + Cfg::kOffTab) + s * TT;
            float *wide = reinterpret_cast<float *>(smem + Cfg::kOffWide + s * Cfg::kWide);
            for (int t = lane; t < TT; t += 32) {
                const float v = to_f32(dts[t * Cfg::kHeadsBox + (head - hbox)]) + bias;
                const float dl = SP ? softplus_io<IoT>(v) : v;
                tab[t] = make_float2(dl, ex2_mufu(dl * a2));
            }
            // unit u = (step t, slot j, half: 0 = B, 1 = C): one slice of NS values
            for (int u = lane; u < TT * 2 * G; u += 32) {
                const int t = u / (2 * G), j = (u / 2) % G, half = u & 1;
                stage_slice<NS>(wide + t * Cfg::kBCRow + (2 * j + half) * NS,
                                (half ? Cs : Bs) + t * N + j * NS);
            }
            mbar_arrive(&ready[s]);
            return true;
        };
        // the compute warps are done with tile k: store it, refill its stage
        auto retire = [&](int k) -> bool {
            const int slot = k % NOUT;
            if (!warp_agree(mbar_wait_or_abort(&out_full[slot], (k / NOUT) & 1, limit, abort_flag)))
                return false;
            if (lane == 0) {
                tma_store_3d(&maps.out, smem + Cfg::kOffOut + slot * Cfg::kAct, c0, k * TT, bb);
                bulk_commit();
                issue(k + STAGES);
                if (k > 0) {
                    bulk_wait_read<1>();  // the store of tile k-1 has read its buffer
                    mbar_arrive(&out_free[(k - 1) % NOUT]);
                }
            }
            __syncwarp();
            return true;
        };
        if (lane == 0) {
            prefetch_tensormap(&maps.x);
            prefetch_tensormap(&maps.z);
            prefetch_tensormap(&maps.dt);
            prefetch_tensormap(&maps.B);
            prefetch_tensormap(&maps.C);
            prefetch_tensormap(&maps.out);
            for (int k = 0; k < STAGES; ++k) issue(k);
        }
        __syncwarp();
        bool ok = ntiles == 0 || prepare(0);
        for (int k = 0; ok && k < ntiles; ++k) {
            if (k + 1 < ntiles) ok = prepare(k + 1);
            if (ok) ok = retire(k);
        }
        if (!ok) fail();
        if (lane == 0) {
            for (int s = 0; s < STAGES; ++s)
                if (last_k[s] >= 0 && !mbar_wait_bounded(&full[s], (last_k[s] / STAGES) & 1, limit))
                    fail();
            bulk_wait<0>();
        }
        __syncwarp();
        return;
    }

    // ============================ compute warps ============================
    const int c_local = warp * CW + lane / G;
    const int sub = lane % G;
    const int64_t d = c0 + c_local;  // < D: CC divides headdim
    const float dskip = a.D ? __ldg(a.D + d) : 0.0f;
    float2 h[NP];
#pragma unroll
    for (int i = 0; i < NP; ++i)
        h[i] = a.h0 ? make_float2(__ldg(a.h0 + (b * D + d) * N + sub * NS + 2 * i),
                                  __ldg(a.h0 + (b * D + d) * N + sub * NS + 2 * i + 1))
                    : make_float2(0.0f, 0.0f);

    bool ok = true;
    for (int k = 0; k < ntiles; ++k) {
        const int s = k % STAGES, slot = k % NOUT;
        const bool got =
            mbar_wait_or_abort(&ready[s], (k / STAGES) & 1, limit, abort_flag) &&
            mbar_wait_or_abort(&full[s], (k / STAGES) & 1, limit, abort_flag) &&
            (k < NOUT || mbar_wait_or_abort(&out_free[slot], ((k / NOUT) - 1) & 1, limit, abort_flag));
        if (!warp_agree(got)) {
            ok = false;
            fail();
            break;
        }
        const uint8_t *st = smem + s * Cfg::kStage;
        const IoT *xs = reinterpret_cast<const IoT *>(st);
        const IoT *zs = reinterpret_cast<const IoT *>(st + Cfg::kAct);
        const float2 *tab = reinterpret_cast<const float2 *>(smem + Cfg::kOffTab) + s * TT;
        const float *wide = reinterpret_cast<const float *>(smem + Cfg::kOffWide + s * Cfg::kWide);
        IoT *outs = reinterpret_cast<IoT *>(smem + Cfg::kOffOut + slot * Cfg::kAct);
        const int nsteps = static_cast<int>(L - int64_t(k) * TT < TT ? L - int64_t(k) * TT : TT);
        if (nsteps == TT)
            ssd_tile<true, IoT, N, G, TT, CC>(h, tab, wide, xs, zs, outs, dskip, c_local, sub, TT);
        else
            ssd_tile<false, IoT, N, G, TT, CC>(h, tab, wide, xs, zs, outs, dskip, c_local, sub,
                                               nsteps);
        fence_proxy_async_smem();  // the output tile before the TMA store reads it
        mbar_arrive(&out_full[slot]);
    }
    if (ok && a.h_final) {
#pragma unroll
        for (int i = 0; i < NP; ++i) {
            a.h_final[(b * D + d) * N + sub * NS + 2 * i] = h[i].x;
            a.h_final[(b * D + d) * N + sub * NS + 2 * i + 1] = h[i].y;
        }
    }
}

}  // namespace jssm
