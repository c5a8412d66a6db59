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
// and token -- against d_state + 4 for the diagonal scan, so this layer is
// bound by memory traffic and by delivering B and C to the lanes that hold the
// states, not by the MUFU pipe.
//
// Layout: one CTA per (sequence, slice of CC channels of one head); CC divides
// headdim.  One producer warp feeds TT-step tiles by TMA (x, z [TT x CC], the
// delta columns of 8 heads [TT x 8], B, C [TT x N]) into a STAGES ring and
// stores the output tiles by TMA; NW compute warps with G lanes per channel,
// NS = N / G states per lane on fp32 pairs.  At the start of each tile the
// compute threads write a [TT] table of (Delta, decay) for the CTA's head;
// then each lane walks the tile: a broadcast read of (Delta, decay) and x,
// vector reads of its B and C slices, the state update and its share of C.h;
// the transposing butterfly hands step j's sum to lane j of the channel, which
// applies the skip and the gate.  Bounded waits and the abort flag as in the
// other kernels.
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
    static constexpr int NOUT = 2;
    static constexpr int kOffOut = STAGES * kStage;
    static constexpr int kOffTab = kOffOut + NOUT * kAct;      // [TT] float2 (Delta, decay)
    static constexpr int kOffBar = kOffTab + TT * 8;
    static constexpr int kNumBars = 2 * STAGES + 2 * NOUT;
    static constexpr int kOffFlag = kOffBar + kNumBars * 8;
    static constexpr int kSmemBytes = kOffFlag + 16;
    static_assert(TT <= NW * 32, "one compute thread per step writes the tile's table");
};

// NS values of one lane's B or C slice as fp32 pairs (one vector load).
template <int NS>
__device__ __forceinline__ void ssd_pairs(const __nv_bfloat16 *p, float2 (&v)[NS / 2]) {
    if constexpr (NS == 8) {
        const uint4 w = *reinterpret_cast<const uint4 *>(p);
        v[0] = bf16x2_to_f2(w.x);
        v[1] = bf16x2_to_f2(w.y);
        v[2] = bf16x2_to_f2(w.z);
        v[3] = bf16x2_to_f2(w.w);
    } else if constexpr (NS == 4) {
        const uint2 w = *reinterpret_cast<const uint2 *>(p);
        v[0] = bf16x2_to_f2(w.x);
        v[1] = bf16x2_to_f2(w.y);
    } else {
        v[0] = bf16x2_to_f2(*reinterpret_cast<const uint32_t *>(p));
    }
}
template <int NS>
__device__ __forceinline__ void ssd_pairs(const float *p, float2 (&v)[NS / 2]) {
#pragma unroll
    for (int i = 0; i < NS / 2; ++i) v[i] = reinterpret_cast<const float2 *>(p)[i];
}

struct SsdMaps {
    CUtensorMap x, z, dt, B, C, out;
};

// grid (ceil(d_inner / CC), batch), (NW + 1) * 32 threads; SP: softplus on.
template <typename IoT, int N, int G, int NW, int TT, int STAGES, bool SP>
__global__ void __launch_bounds__((NW + 1) * 32, 1)
    s6_ssd_kernel(const __grid_constant__ SsdMaps maps, const SsdArgs a) {
    using Cfg = SsdCfg<IoT, N, G, NW, TT, STAGES>;
    constexpr int NS = Cfg::NS, NP = Cfg::NP, CW = Cfg::CW, CC = Cfg::CC, NOUT = Cfg::NOUT;
    extern __shared__ __align__(1024) uint8_t smem[];
    uint64_t *full = reinterpret_cast<uint64_t *>(smem + Cfg::kOffBar);
    uint64_t *empty = full + STAGES;
    uint64_t *out_full = empty + STAGES;
    uint64_t *out_free = out_full + NOUT;
    volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + Cfg::kOffFlag);
    float2 *tab = reinterpret_cast<float2 *>(smem + Cfg::kOffTab);

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
            mbar_init(&empty[s], NW * 32);
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
        // ===================== producer: TMA loads and stores =====================
        if (lane == 0) {
            prefetch_tensormap(&maps.x);
            prefetch_tensormap(&maps.z);
            prefetch_tensormap(&maps.dt);
            prefetch_tensormap(&maps.B);
            prefetch_tensormap(&maps.C);
            prefetch_tensormap(&maps.out);
            const int bb = static_cast<int>(b);
            int last_k[STAGES];
            for (int s = 0; s < STAGES; ++s) last_k[s] = -1;
            auto issue = [&](int k) -> bool {
                const int s = k % STAGES;
                if (k >= STAGES &&
                    !mbar_wait_or_abort(&empty[s], ((k / STAGES) & 1) ^ 1, limit, abort_flag))
                    return false;
                if ((a.debug_flags & 1u) && k == 0) return true;  // test hook: withhold tile 0
                uint8_t *st = smem + s * Cfg::kStage;
                const int t0 = k * TT;
                mbar_arrive_expect_tx(&full[s], Cfg::kStage);
                tma_load_3d(st, &maps.x, c0, t0, bb, &full[s]);
                tma_load_3d(st + Cfg::kAct, &maps.z, c0, t0, bb, &full[s]);
                tma_load_3d(st + 2 * Cfg::kAct, &maps.dt, hbox, t0, bb, &full[s]);
                tma_load_3d(st + 2 * Cfg::kAct + Cfg::kDt, &maps.B, 0, t0, bb, &full[s]);
                tma_load_3d(st + 2 * Cfg::kAct + Cfg::kDt + Cfg::kBC, &maps.C, 0, t0, bb, &full[s]);
                last_k[s] = k;
                return true;
            };
            bool ok = true;
            int next = 0;
            for (; next < STAGES && next < ntiles && ok; ++next) ok = issue(next);
            for (int k = 0; k < ntiles && ok; ++k) {
                const int slot = k % NOUT;
                if (!mbar_wait_or_abort(&out_full[slot], (k / NOUT) & 1, limit, abort_flag)) {
                    ok = false;
                    break;
                }
                tma_store_3d(&maps.out, smem + Cfg::kOffOut + slot * Cfg::kAct, c0, k * TT, bb);
                bulk_commit();
                if (next < ntiles) ok = issue(next++);
                if (k > 0) {
                    bulk_wait_read<1>();
                    mbar_arrive(&out_free[(k - 1) % NOUT]);
                }
            }
            if (!ok) fail();
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
    const int64_t d = c0 + c_local;
    const bool dvalid = d < D;
    const int64_t dc = dvalid ? d : D - 1;
    const float a2 = __ldg(a.A + head) * kLog2e;
    const float bias = a.delta_bias ? __ldg(a.delta_bias + head) : 0.0f;
    const float dskip = a.D ? __ldg(a.D + dc) : 0.0f;
    float2 h[NP];
#pragma unroll
    for (int i = 0; i < NP; ++i)
        h[i] = a.h0 ? make_float2(__ldg(a.h0 + (b * D + dc) * N + sub * NS + 2 * i),
                                  __ldg(a.h0 + (b * D + dc) * N + sub * NS + 2 * i + 1))
                    : make_float2(0.0f, 0.0f);

    bool ok = true;
    for (int k = 0; k < ntiles; ++k) {
        const int s = k % STAGES, slot = k % NOUT;
        if (ok && (!mbar_wait_or_abort(&full[s], (k / STAGES) & 1, limit, abort_flag) ||
                   (k >= NOUT &&
                    !mbar_wait_or_abort(&out_free[slot], ((k / NOUT) - 1) & 1, limit, abort_flag)))) {
            ok = false;
            fail();
        }
        const int nsteps = static_cast<int>(L - int64_t(k) * TT < TT ? L - int64_t(k) * TT : TT);
        const uint8_t *st = smem + s * Cfg::kStage;
        const IoT *xs = reinterpret_cast<const IoT *>(st);
        const IoT *zs = reinterpret_cast<const IoT *>(st + Cfg::kAct);
        const IoT *dts = reinterpret_cast<const IoT *>(st + 2 * Cfg::kAct);
        const IoT *Bs = reinterpret_cast<const IoT *>(st + 2 * Cfg::kAct + Cfg::kDt);
        const IoT *Cs = reinterpret_cast<const IoT *>(st + 2 * Cfg::kAct + Cfg::kDt + Cfg::kBC);
        IoT *outs = reinterpret_cast<IoT *>(smem + Cfg::kOffOut + slot * Cfg::kAct);
        // the head's (Delta, decay) of every step of the tile
        if (ok && tid < TT) {
            const float v = to_f32(dts[tid * Cfg::kHeadsBox + (head - hbox)]) + bias;
            const float dl = SP ? softplus_f32(v) : v;
            tab[tid] = make_float2(dl, ex2_mufu(dl * a2));
        }
        asm volatile("bar.sync 1, %0;" ::"r"(NW * 32) : "memory");
        if (ok) {
#pragma unroll 1
            for (int t0 = 0; t0 < nsteps; t0 += G) {
                float yp[G];
#pragma unroll
                for (int j = 0; j < G; ++j) {
                    const int t = t0 + j;
                    yp[j] = 0.0f;
                    if (t < nsteps) {
                        const float2 dd = tab[t];
                        const float dx = dd.x * to_f32(xs[t * CC + c_local]);
                        float2 bv[NP], cv[NP];
                        ssd_pairs<NS>(Bs + t * N + sub * NS, bv);
                        ssd_pairs<NS>(Cs + t * N + sub * NS, cv);
                        const float2 dec2 = make_float2(dd.y, dd.y), dx2 = make_float2(dx, dx);
                        float2 y2 = make_float2(0.0f, 0.0f);
#pragma unroll
                        for (int i = 0; i < NP; ++i) {
                            h[i] = fma2(dec2, h[i], mul2(dx2, bv[i]));
                            y2 = fma2(cv[i], h[i], y2);
                        }
                        yp[j] = y2.x + y2.y;
                    }
                }
                const float y = reduce_transpose<G>(yp, sub);
                const int t = t0 + sub;
                if (t < nsteps) {
                    const float xo = to_f32(xs[t * CC + c_local]);
                    outs[t * CC + c_local] =
                        from_f32<IoT>(fmaf(dskip, xo, y) * silu_f32(to_f32(zs[t * CC + c_local])));
                }
            }
            mbar_arrive(&empty[s]);
            fence_proxy_async_smem();
            mbar_arrive(&out_full[slot]);
        }
        // the table is rewritten at the next tile: every lane is done with it
        asm volatile("bar.sync 1, %0;" ::"r"(NW * 32) : "memory");
    }
    if (ok && dvalid && a.h_final) {
#pragma unroll
        for (int i = 0; i < NP; ++i) {
            a.h_final[(b * D + d) * N + sub * NS + 2 * i] = h[i].x;
            a.h_final[(b * D + d) * N + sub * NS + 2 * i + 1] = h[i].y;
        }
    }
}

}  // namespace jssm
