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
// bound by the MUFU pipe.  What bounds it is the shared-memory pipe: a 16-byte
// vector read costs four wavefronts whatever the broadcast, and every lane
// reads its B and C slices at every step.  So the tile is prepared once per
// CTA into the forms that cost a lane-step the fewest wavefronts: the decay
// (one broadcast word), Delta x (one word per channel) and the lane's B and C
// slices side by side in the I/O type (one 16-byte vector in bf16).
//
// Layout: one CTA per (sequence, slice of CC channels of one head); CC divides
// headdim.  NW compute warps with G lanes per channel, NS = N / G states per
// lane on fp32 pairs; one producer warp.
//  * The producer's lane 0 feeds TT-step tiles by TMA into a STAGES ring (x, z
//    [TT x CC], the delta columns of a 16-byte box of heads [TT x 16 B], B, C
//    [TT x N]) and stores the output tiles by TMA.
//  * All producer lanes then prepare each landed tile: the [TT] table of
//    (Delta, decay) of the CTA's head, Delta x in fp32 [TT x CC], and the
//    per-lane slots [TT][G][B slice | C slice].
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
    // prepared per stage: Delta x [TT][CC] fp32, slots [TT][G][2 NS] IoT, (Delta, decay) [TT]
    static constexpr int kOffDx = STAGES * kStage;
    static constexpr int kDx = TT * CC * 4;
    static constexpr int kOffSlot = kOffDx + STAGES * kDx;
    static constexpr int kSlot = TT * 2 * N * (int)sizeof(IoT);
    static constexpr int kOffTab = kOffSlot + STAGES * kSlot;
    static constexpr int NOUT = 3;
    static constexpr int kOffOut = kOffTab + STAGES * TT * 8;
    static_assert(kOffOut % 128 == 0, "TMA store sources 128-byte aligned");
    static constexpr int kOffBar = kOffOut + NOUT * kAct;
    static constexpr int kNumBars = 2 * STAGES + 2 * NOUT;  // full, ready, out_full, out_free
    static constexpr int kOffFlag = kOffBar + kNumBars * 8;
    static constexpr int kSmemBytes = kOffFlag + 16;
    static_assert(TT % G == 0 && CC % (16 / (int)sizeof(IoT)) == 0, "whole groups and vectors");
};

// A lane's slot (its NS values of B, then its NS values of C) as fp32 pairs:
// one 16-byte read for bf16 with NS = 4.
template <int NS>
__device__ __forceinline__ void load_slot(const __nv_bfloat16 *p, float2 (&b)[NS / 2],
                                          float2 (&c)[NS / 2]) {
    if constexpr (NS == 2) {  // B0 B1 | C0 C1: 8 bytes
        const uint2 w = *reinterpret_cast<const uint2 *>(p);
        b[0] = bf16x2_to_f2(w.x);
        c[0] = bf16x2_to_f2(w.y);
    } else if constexpr (NS == 4) {  // B0..3 | C0..3: 16 bytes
        const uint4 w = *reinterpret_cast<const uint4 *>(p);
        b[0] = bf16x2_to_f2(w.x);
        b[1] = bf16x2_to_f2(w.y);
        c[0] = bf16x2_to_f2(w.z);
        c[1] = bf16x2_to_f2(w.w);
    } else {  // B0..7 | C0..7: two 16-byte vectors
        const uint4 wb = reinterpret_cast<const uint4 *>(p)[0];
        const uint4 wc = reinterpret_cast<const uint4 *>(p)[1];
        b[0] = bf16x2_to_f2(wb.x);
        b[1] = bf16x2_to_f2(wb.y);
        b[2] = bf16x2_to_f2(wb.z);
        b[3] = bf16x2_to_f2(wb.w);
        c[0] = bf16x2_to_f2(wc.x);
        c[1] = bf16x2_to_f2(wc.y);
        c[2] = bf16x2_to_f2(wc.z);
        c[3] = bf16x2_to_f2(wc.w);
    }
}
template <int NS>
__device__ __forceinline__ void load_slot(const float *p, float2 (&b)[NS / 2], float2 (&c)[NS / 2]) {
#pragma unroll
    for (int i = 0; i < NS / 2; ++i) {
        b[i] = reinterpret_cast<const float2 *>(p)[i];
        c[i] = reinterpret_cast<const float2 *>(p + NS)[i];
    }
}

// One tile of a compute lane: TT steps if FULL, else the first `nsteps`
// (the states do not move past them; the rows past them are written to the
// output buffer but clipped by the TMA store).
template <bool FULL, typename IoT, int N, int G, int TT, int CC>
__device__ __forceinline__ void ssd_tile(float2 (&h)[N / G / 2], const float2 *tab,
                                         const float *dxs, const IoT *slots, const IoT *xs,
                                         const IoT *zs, IoT *outs, float dskip, int c_local,
                                         int sub, int nsteps) {
    constexpr int NS = N / G, NP = NS / 2, NQ = TT / G;
    const float *decay = reinterpret_cast<const float *>(tab) + 1;  // .y of each entry
    float yown[NQ];  // C.h of the owned steps q * G + sub
#pragma unroll
    for (int q = 0; q < NQ; ++q) {
        float yp[G];
#pragma unroll
        for (int j = 0; j < G; ++j) {
            const int t = q * G + j;
            yp[j] = 0.0f;
            if (FULL || t < nsteps) {
                const float dec = decay[2 * t];
                const float dx = dxs[t * CC + c_local];
                float2 bv[NP], cv[NP];
                load_slot<NS>(slots + (t * G + sub) * 2 * NS, bv, cv);
                const float2 dec2 = make_float2(dec, dec), dx2 = make_float2(dx, dx);
                float2 y2;
#pragma unroll
                for (int i = 0; i < NP; ++i) {
                    h[i] = fma2(dec2, h[i], mul2(dx2, bv[i]));
                    y2 = i == 0 ? mul2(cv[i], h[i]) : fma2(cv[i], h[i], y2);
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

// One 16-byte vector of an I/O tile as floats (8 bf16 or 4 fp32).
__device__ __forceinline__ void load_vec16(const __nv_bfloat16 *p, float (&v)[8]) {
    const uint4 w = *reinterpret_cast<const uint4 *>(p);
    const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const float2 f = bf16x2_to_f2(ws[i]);
        v[2 * i] = f.x;
        v[2 * i + 1] = f.y;
    }
}
__device__ __forceinline__ void load_vec16(const float *p, float (&v)[4]) {
    const float4 w = *reinterpret_cast<const float4 *>(p);
    v[0] = w.x;
    v[1] = w.y;
    v[2] = w.z;
    v[3] = w.w;
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
        // tile k landed: (Delta, decay), Delta x and the lanes' B | C slots
        auto prepare = [&](int k) -> bool {
            const int s = k % STAGES;
            if (!warp_agree(mbar_wait_or_abort(&full[s], (k / STAGES) & 1, limit, abort_flag)))
                return false;
            if (lane == 0) last_k[s] = -1;
            const uint8_t *st = smem + s * Cfg::kStage;
            const IoT *xs = reinterpret_cast<const IoT *>(st);
            const IoT *dts = reinterpret_cast<const IoT *>(st + 2 * Cfg::kAct);
            const IoT *Bs = reinterpret_cast<const IoT *>(st + 2 * Cfg::kAct + Cfg::kDt);
            const IoT *Cs = reinterpret_cast<const IoT *>(st + 2 * Cfg::kAct + Cfg::kDt + Cfg::kBC);
            float2 *tab = reinterpret_cast<float2 *>(smem + Cfg::kOffTab) + s * TT;
            float *dxs = reinterpret_cast<float *>(smem + Cfg::kOffDx + s * Cfg::kDx);
            IoT *slots = reinterpret_cast<IoT *>(smem + Cfg::kOffSlot + s * Cfg::kSlot);
            for (int t = lane; t < TT; t += 32) {
                const float v = to_f32(dts[t * Cfg::kHeadsBox + (head - hbox)]) + bias;
                const float dl = SP ? softplus_io<IoT>(v) : v;
                tab[t] = make_float2(dl, ex2_mufu(dl * a2));
            }
            __syncwarp();  // each step's Delta is read by other lanes below
            // Delta x, one 16-byte vector of x (VEC channels of one step) per unit
            constexpr int VEC = 16 / (int)sizeof(IoT), VPR = CC / VEC;
            for (int u = lane; u < TT * VPR; u += 32) {
                const int t = u / VPR, cv = (u % VPR) * VEC;
                const float dl = tab[t].x;
                float xv[VEC];
                load_vec16(xs + t * CC + cv, xv);
#pragma unroll
                for (int q = 0; q < VEC / 4; ++q)
                    reinterpret_cast<float4 *>(dxs + t * CC + cv)[q] =
                        make_float4(dl * xv[4 * q], dl * xv[4 * q + 1], dl * xv[4 * q + 2],
                                    dl * xv[4 * q + 3]);
            }
            // slot (t, j): B[t, j NS ..] then C[t, j NS ..]
            constexpr int W = NS * (int)sizeof(IoT) / 4;
            for (int u = lane; u < TT * G; u += 32) {
                const int t = u / G, j = u % G;
                IoT *dst = slots + (t * G + j) * 2 * NS;
                copy_words<W>(reinterpret_cast<uint32_t *>(dst),
                              reinterpret_cast<const uint32_t *>(Bs + t * N + j * NS));
                copy_words<W>(reinterpret_cast<uint32_t *>(dst + NS),
                              reinterpret_cast<const uint32_t *>(Cs + t * N + j * NS));
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
        const float *dxs = reinterpret_cast<const float *>(smem + Cfg::kOffDx + s * Cfg::kDx);
        const IoT *slots = reinterpret_cast<const IoT *>(smem + Cfg::kOffSlot + s * Cfg::kSlot);
        IoT *outs = reinterpret_cast<IoT *>(smem + Cfg::kOffOut + slot * Cfg::kAct);
        const int nsteps = static_cast<int>(L - int64_t(k) * TT < TT ? L - int64_t(k) * TT : TT);
        if (nsteps == TT)
            ssd_tile<true, IoT, N, G, TT, CC>(h, tab, dxs, slots, xs, zs, outs, dskip, c_local,
                                              sub, TT);
        else
            ssd_tile<false, IoT, N, G, TT, CC>(h, tab, dxs, slots, xs, zs, outs, dskip, c_local,
                                               sub, nsteps);
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
