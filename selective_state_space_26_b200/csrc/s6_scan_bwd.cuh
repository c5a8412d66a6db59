// s6_scan_bwd.cuh -- backward pass (reverse-mode gradient) of the S6 prefill
// scan on sm_100a, for training.
//
// The forward recurrence is the one of the "Mamba 레이어" section of the
// Jamba notes, read as h_t = exp(Delta_t A) h_{t-1} + Delta_t B_t x_t,
// y_t = C_t . h_t + D x_t, out_t = y_t silu(z_t), Delta = softplus(delta +
// bias).  Given dout = dL/dout (and dL/dh_final), the chain rule in reverse
// time with the carry g = dL/dh_t gives, per channel d and step t (g first
// takes the readout's share, g += dy C_t, with dy = dout silu(z)):
//   dz       = dout y sigma(z) (1 + z (1 - sigma(z)))
//   dC_t[n] += dy h_t[n]               dB_t[n] += g_n Delta x      (summed over d)
//   dDelta   = sum_n g_n h_{t-1}[n] Abar_n A_n + x sum_n g_n B_n
//   dx       = dy D + Delta sum_n g_n B_n
//   dA[n]   += g_n h_{t-1}[n] Abar_n Delta,  dD += dy x,  ddelta = dDelta sigma(v)
//   g_n     <- Abar_n g_n                  (and dh0 = g after step 0)
// where sigma(v) = d softplus / dv for v = delta + bias.  (This is the
// derivative the fp64 oracle's scan_bwd takes, step for step.)
//
// Three kernels, all deterministic (no atomics, fixed summation orders):
//  1. the checkpoint pass: the forward kernel (s6_scan_fused_kernel) in its
//     checkpoint mode runs the recurrence once more, TMA-fed, storing the
//     state before every kCk-th step in the workspace (no readout, no output).
//  2. s6_bwd_kernel: per (sequence, channel group), 64-step tiles from the last
//     to the first, fed by TMA (x, delta, z, dout, B, C) like the forward.  In
//     each tile, segments of kCk steps from the last to the first: the lanes
//     recompute the segment's states from its checkpoint into registers, then
//     walk it backwards with g in registers.  The lane layout is the forward's:
//     G lanes per channel, NS = N / G states per lane, lane `sub` owning the
//     per-(t, d) scalars of steps sub, sub + G, ...; sums over a channel's
//     states go through the transposing butterfly; the state math runs on
//     fp32 pairs.  dB and dC, sums over channels, are summed over a warp's
//     channels through a small per-warp shared-memory scratch (each lane
//     stores its slices, then lane k adds slot k), then over the CTA's warps,
//     and written as one partial per CTA.  dx, ddelta and dz leave through
//     shared memory and TMA stores.
//  3. s6_bwd_reduce_kernel: dB and dC = the sum of the CTA partials, and dA,
//     dD, dbias = the sum over sequences, in a fixed order in fp64.
// Every mbarrier wait is bounded; a wait that runs out records
// JAMBA_SSM_ERR_TIMEOUT, sets the CTA's abort flag, and every warp winds down
// after the producer has waited (bounded) for the copies it issued.
#pragma once

#include "device_utils.cuh"
#include "s6_math.cuh"
#include "s6_scan.cuh"

namespace jssm {

struct BwdArgs {
    int64_t batch, seqlen, d_inner;
    const float *A, *D, *delta_bias, *h0, *dh_final;
    int delta_softplus;
    const float *ckpt;          // [batch, nck, d_inner, N] fp32, from the checkpoint pass
    float *part_bc;             // [batch, ngroups, seqlen, 2N] fp32: CTA partials of dB | dC
    float *part_par;            // [batch, d_inner, N + 2] fp32: dA[N], dD, dbias per sequence
    float *dh0;                 // [batch, d_inner, N] or null
    int *status;
    uint32_t debug_flags;
    uint64_t timeout_cycles;
};

template <typename IoT, int N, int G, int NW, int TT>
struct BwdCfg {
    static constexpr int NS = N / G, CW = 32 / G, CC = NW * CW;
    static_assert(NS == 2 || NS == 4, "two or four states per lane");
    static_assert(TT % kCk == 0 && kCk % G == 0, "segments of whole step groups");
    static constexpr int kAct = TT * CC * (int)sizeof(IoT);   // one [TT x CC] tile
    static constexpr int kBC = TT * N * (int)sizeof(IoT);     // one [TT x N] tile
    static constexpr int kStage = 4 * kAct + 2 * kBC;         // x, delta, z, dout, B, C
    static constexpr int STAGES = 2;
    static constexpr int NOUT = 2;                            // output tile sets in flight
    static constexpr int kOffOut = STAGES * kStage;           // dx, ddelta, dz per set
    static constexpr int kOffPart = kOffOut + NOUT * 3 * kAct;  // [NW][TT][2N] fp32
    static constexpr int kPart = NW * TT * 2 * N * 4;
    // per warp, two steps' [slot][channel][dB | dC] scratch (see BcScratch)
    static constexpr int kOffScr = kOffPart + kPart;
    static constexpr int kScrWords = 2 * CW * (N == 16 ? 48 : (N == 8 ? 24 : 12));
    // per stage, B and C widened to fp32 in per-lane slots ([TT][G][2][NS], load_bc's layout)
    static constexpr int kOffWide = kOffScr + NW * kScrWords * 4;
    static constexpr int kWide = TT * 2 * N * 4;
    static constexpr int kOffBar = kOffWide + STAGES * kWide;
    static_assert(kOffWide % 16 == 0, "16-byte slot reads");
    // full, ready, empty, out_full, out_free
    static constexpr int kNumBars = 3 * STAGES + 2 * NOUT;
    static constexpr int kOffFlag = kOffBar + kNumBars * 8;
    static constexpr int kSmemBytes = kOffFlag + 16;
    static_assert(kAct % 128 == 0 && kBC % 128 == 0, "TMA boxes 128-byte aligned");
};

// NS consecutive values (one lane's B or C slice of one step) as NS / 2 fp32
// pairs, read with one vector load: 4 or 8 bytes of bf16, 8 or 16 of fp32.
template <int NS>
__device__ __forceinline__ void load_pairs(const __nv_bfloat16 *p, float2 (&v)[NS / 2]) {
    if constexpr (NS == 4) {
        const uint2 w = *reinterpret_cast<const uint2 *>(p);
        v[0] = bf16x2_to_f2(w.x);
        v[1] = bf16x2_to_f2(w.y);
    } else {
        static_assert(NS == 2, "two or four values");
        v[0] = bf16x2_to_f2(*reinterpret_cast<const uint32_t *>(p));
    }
}
template <int NS>
__device__ __forceinline__ void load_pairs(const float *p, float2 (&v)[NS / 2]) {
    if constexpr (NS == 4) {
        const float4 w = *reinterpret_cast<const float4 *>(p);
        v[0] = make_float2(w.x, w.y);
        v[1] = make_float2(w.z, w.w);
    } else {
        static_assert(NS == 2, "two or four values");
        v[0] = *reinterpret_cast<const float2 *>(p);
    }
}

// --------------------------------------------------------------- backward
// A warp's scratch for summing dB | dC over its channels, two steps at a time:
// slot k (the step of the pair, k = step & 1) holds one row per channel of 2N
// values.  Row stride RS (in words): 2N plus padding chosen so that the lanes
// of one vector-store wavefront (the slices of 2, 4 or 8 channels) land in
// distinct banks.
template <int N, int G>
struct BcScratch {
    static constexpr int CW = 32 / G;
    static constexpr int RS = N == 16 ? 48 : (N == 8 ? 24 : 12);
    static constexpr int kSlot = CW * RS;
    static constexpr int kWords = 2 * kSlot;
};

// One segment of kCk steps (starting at tile step s0, `nst` of them valid),
// recomputed from h_in and walked backwards.  Owner scalars come from the
// stage's x / delta / z / dout tiles; B / C slices from the stage's widened
// fp32 slots (`wide`, [TT][G][2][NS]), 16-byte loads without conversions;
// the state math is on fp32 pairs.  `part` is
// the warp's [TT][2N] slab of the CTA's dB | dC partial sums and `bcs` its
// [2][CW][RS] scratch for summing two steps over the warp's channels.
template <bool FULL, bool SP, typename IoT, int N, int G, int CC>
__device__ __forceinline__ void bwd_segment(
    const float2 (&h_in)[N / G / 2], float2 (&g)[N / G / 2], float2 (&dA)[N / G / 2],
    float &dD_acc, float &dbias_acc, const float2 (&a2)[N / G / 2], const float2 (&Araw)[N / G / 2],
    float bias, float dskip, const IoT *xs, const IoT *dts, const IoT *zs, const IoT *dos,
    const float *wide, IoT *dxs, IoT *dds, IoT *dzs, float *part, float *bcs, int s0,
    int nst, int c_local, int sub, int gbase, int lane) {
    constexpr int NS = N / G, NP = NS / 2, NQ = kCk / G;
    using SC = BcScratch<N, G>;
    // ---- recompute: the state after every step of the segment, and the
    // steps' Delta and Delta x on every lane of the channel
    float2 hs[kCk][NP];
    float dl[kCk], dxv[kCk];
    float dl_own[NQ], w_own[NQ], v_own[NQ];  // owned steps: Delta, e^{-|v|}, v
    float2 h[NP];
#pragma unroll
    for (int i = 0; i < NP; ++i) h[i] = h_in[i];
#pragma unroll
    for (int q = 0; q < NQ; ++q) {
        const int idx = (s0 + q * G + sub) * CC + c_local;
        const float xo = to_f32(xs[idx]);
        const float v = to_f32(dts[idx]) + bias;
        const float dlo = SP ? softplus_f32(v) : v;
        dl_own[q] = dlo;
        v_own[q] = v;
        w_own[q] = SP ? ex2_mufu(-fabsf(v) * kLog2e) : 0.0f;
        const float dxo = dlo * xo;
#pragma unroll
        for (int jj = 0; jj < G; ++jj) {
            const int j = q * G + jj;
            dl[j] = __shfl_sync(0xffffffffu, dlo, gbase | jj);
            dxv[j] = __shfl_sync(0xffffffffu, dxo, gbase | jj);
            if (FULL || j < nst) {
                float2 bv[NP];
                load_pairs<NS>(wide + (s0 + j) * 2 * N + sub * 2 * NS, bv);
#pragma unroll
                for (int i = 0; i < NP; ++i) {
                    const float2 arg = mul2(make_float2(dl[j], dl[j]), a2[i]);
                    const float2 ab = make_float2(ex2_mufu(arg.x), ex2_mufu(arg.y));
                    h[i] = fma2(ab, h[i], mul2(make_float2(dxv[j], dxv[j]), bv[i]));
                }
            }
#pragma unroll
            for (int i = 0; i < NP; ++i) hs[j][i] = h[i];
        }
    }
    // ---- backward walk, groups of G steps from the last
    const int c_in_warp = lane / G;
    float *my_row = bcs + c_in_warp * SC::RS + sub * NS;  // + (step & 1) * SC::kSlot
    static_assert(G % 2 == 0, "steps pair up inside a group");
#pragma unroll
    for (int q = NQ - 1; q >= 0; --q) {
        const int jo = q * G + sub;
        const int idx = (s0 + jo) * CC + c_local;
        const bool own_ok = FULL || jo < nst;
        const float zo = to_f32(zs[idx]);
        const float doo = own_ok ? to_f32(dos[idx]) : 0.0f;
        const float xo = to_f32(xs[idx]);
        const float sz = rcp_mufu(1.0f + ex2_mufu(-zo * kLog2e));  // sigma(z)
        const float dy_o = doo * zo * sz;
        float yp[G], pa[G], gb[G];
#pragma unroll
        for (int jj = G - 1; jj >= 0; --jj) {
            const int j = q * G + jj;
            const float dy = __shfl_sync(0xffffffffu, dy_o, gbase | jj);
            float2 dBp[NP], dCp[NP];
            float2 y2 = make_float2(0.0f, 0.0f), pa2 = y2, gb2 = y2;
#pragma unroll
            for (int i = 0; i < NP; ++i) dBp[i] = dCp[i] = make_float2(0.0f, 0.0f);
            if (FULL || j < nst) {
                const BCPairs<NS> bc = load_bc<NS>(wide + (s0 + j) * 2 * N, sub);
                const float2(&bv)[NP] = bc.b;
                const float2(&cv)[NP] = bc.c;
                const float2 dy2 = make_float2(dy, dy), dl2 = make_float2(dl[j], dl[j]);
                const float2 dx2 = make_float2(dxv[j], dxv[j]);
#pragma unroll
                for (int i = 0; i < NP; ++i) {
                    const float2 hprev = j > 0 ? hs[j - 1][i] : h_in[i];
                    y2 = fma2(cv[i], hs[j][i], y2);
                    g[i] = fma2(dy2, cv[i], g[i]);           // dL/dh_t: the readout's share
                    dCp[i] = mul2(dy2, hs[j][i]);            // dC_t[n], this channel
                    const float2 arg = mul2(dl2, a2[i]);
                    const float2 ab = make_float2(ex2_mufu(arg.x), ex2_mufu(arg.y));
                    const float2 P = mul2(mul2(g[i], hprev), ab);  // dL/dAbar * Abar
                    pa2 = fma2(P, Araw[i], pa2);
                    dA[i] = fma2(P, dl2, dA[i]);
                    gb2 = fma2(g[i], bv[i], gb2);
                    dBp[i] = mul2(g[i], dx2);                // dB_t[n], this channel
                    g[i] = mul2(g[i], ab);                   // dL/dh_{t-1}
                }
            }
            yp[jj] = y2.x + y2.y;
            pa[jj] = pa2.x + pa2.y;
            gb[jj] = gb2.x + gb2.y;
            // dB / dC of this step summed over the warp's channels, through the
            // warp's scratch, two steps at a time: each lane stores its slices
            // (zeros for a step past the segment) in the step's slot; after the
            // pair's second step (jj even: the walk goes down), lane l adds
            // values 2 (l % N) and 2 (l % N) + 1 of slot l / N over the channels
            // in order, on one fp32 pair.
            {
                float *row = my_row + (jj & 1) * SC::kSlot;
#pragma unroll
                for (int i = 0; i < NP; ++i) {
                    reinterpret_cast<float2 *>(row)[i] = dBp[i];
                    reinterpret_cast<float2 *>(row + N)[i] = dCp[i];
                }
            }
            if ((jj & 1) == 0) {
                __syncwarp();
                const int sl = lane / N, v = 2 * (lane % N);
                const int js = q * G + jj + sl;  // the step whose values this lane sums
                if (lane < 2 * N && (FULL || js < nst)) {
                    const float *src = bcs + sl * SC::kSlot + v;
                    float2 acc = *reinterpret_cast<const float2 *>(src);
                    const float2 one = make_float2(1.0f, 1.0f);
#pragma unroll
                    for (int c = 1; c < SC::CW; ++c)
                        acc = fma2(*reinterpret_cast<const float2 *>(src + c * SC::RS), one, acc);
                    *reinterpret_cast<float2 *>(part + (s0 + js) * 2 * N + v) = acc;
                }
                __syncwarp();
            }
        }
        // the owner's totals for its step: y (pre-gate), sum P A, sum g B
        const float ys = reduce_transpose<G>(yp, sub);
        const float pas = reduce_transpose<G>(pa, sub);
        const float gbs = reduce_transpose<G>(gb, sub);
        if (own_ok) {
            const float y = fmaf(dskip, xo, ys);
            const float dz = doo * y * sz * (1.0f + zo * (1.0f - sz));
            const float dDelta = fmaf(xo, gbs, pas);
            float ddr = dDelta;
            if (SP) {  // d softplus / dv = sigma(v), from w = e^{-|v|}
                const float r = rcp_mufu(1.0f + w_own[q]);
                ddr = dDelta * (v_own[q] >= 0.0f ? r : w_own[q] * r);
            }
            dbias_acc += ddr;
            dD_acc = fmaf(dy_o, xo, dD_acc);
            dxs[idx] = from_f32<IoT>(fmaf(dy_o, dskip, dl_own[q] * gbs));
            dds[idx] = from_f32<IoT>(ddr);
            dzs[idx] = from_f32<IoT>(dz);
        }
    }
}

struct BwdMaps {
    CUtensorMap x, dt, z, dout, B, C, dx, ddt, dz;
};

// grid (ceil(d_inner / CC), batch); NW compute warps + 1 producer warp.  SP:
// Delta = softplus(delta + bias) (else delta + bias).
template <typename IoT, int N, int G, int NW, int TT, bool SP>
__global__ void __launch_bounds__((NW + 1) * 32, 1)
    s6_bwd_kernel(const __grid_constant__ BwdMaps maps, const BwdArgs a) {
    using Cfg = BwdCfg<IoT, N, G, NW, TT>;
    constexpr int NS = Cfg::NS, CW = Cfg::CW, CC = Cfg::CC, STAGES = Cfg::STAGES,
                  NOUT = Cfg::NOUT;
    extern __shared__ __align__(1024) uint8_t smem[];
    uint64_t *full = reinterpret_cast<uint64_t *>(smem + Cfg::kOffBar);
    uint64_t *ready = full + STAGES;
    uint64_t *empty = ready + STAGES;
    uint64_t *out_full = empty + STAGES;
    uint64_t *out_free = out_full + NOUT;
    volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + Cfg::kOffFlag);
    float *part_all = reinterpret_cast<float *>(smem + Cfg::kOffPart);
    static_assert(Cfg::kScrWords == BcScratch<N, G>::kWords, "scratch layout");

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int64_t b = blockIdx.y;
    const int c0 = blockIdx.x * CC;
    const int64_t D = a.d_inner, L = a.seqlen;
    const int ntiles = static_cast<int>((L + TT - 1) / TT);
    const int64_t nck = (L + kCk - 1) / kCk;
    const uint64_t limit = a.timeout_cycles;

    if (tid == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&ready[s], 32);
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
        // ========== producer: TMA loads and stores, B / C widening ==========
        const int bb = static_cast<int>(b);
        int last_i[STAGES];  // lane 0: the walked tile whose load is in flight per stage, or -1
        for (int s = 0; s < STAGES; ++s) last_i[s] = -1;
        // the i-th tile walked is tile ntiles - 1 - i (lane 0 only)
        auto issue = [&](int i) -> bool {
            const int s = i % STAGES;
            if (i >= STAGES &&
                !mbar_wait_or_abort(&empty[s], ((i / STAGES) & 1) ^ 1, limit, abort_flag))
                return false;
            if ((a.debug_flags & 1u) && i == 0) return true;  // test hook: withhold tile 0
            uint8_t *st = smem + s * Cfg::kStage;
            const int t0 = (ntiles - 1 - i) * TT;
            mbar_arrive_expect_tx(&full[s], Cfg::kStage);
            tma_load_3d(st, &maps.x, c0, t0, bb, &full[s]);
            tma_load_3d(st + Cfg::kAct, &maps.dt, c0, t0, bb, &full[s]);
            tma_load_3d(st + 2 * Cfg::kAct, &maps.z, c0, t0, bb, &full[s]);
            tma_load_3d(st + 3 * Cfg::kAct, &maps.dout, c0, t0, bb, &full[s]);
            tma_load_3d(st + 4 * Cfg::kAct, &maps.B, 0, t0, bb, &full[s]);
            tma_load_3d(st + 4 * Cfg::kAct + Cfg::kBC, &maps.C, 0, t0, bb, &full[s]);
            last_i[s] = i;
            return true;
        };
        // walked tile i landed: B and C into the stage's fp32 slots (all lanes)
        auto prepare = [&](int i) -> bool {
            const int s = i % STAGES;
            if (!warp_agree(mbar_wait_or_abort(&full[s], (i / STAGES) & 1, limit, abort_flag)))
                return false;
            if (lane == 0) last_i[s] = -1;
            const uint8_t *st = smem + s * Cfg::kStage;
            const IoT *Bs = reinterpret_cast<const IoT *>(st + 4 * Cfg::kAct);
            const IoT *Cs = reinterpret_cast<const IoT *>(st + 4 * Cfg::kAct + Cfg::kBC);
            float *wide = reinterpret_cast<float *>(smem + Cfg::kOffWide + s * Cfg::kWide);
            // unit u = (step t, slot j, half: 0 = B, 1 = C): one slice of NS values
            for (int u = lane; u < TT * 2 * G; u += 32) {
                const int t = u / (2 * G), j = (u / 2) % G, half = u & 1;
                stage_slice<NS>(wide + t * 2 * N + (2 * j + half) * NS,
                                (half ? Cs : Bs) + t * N + j * NS);
            }
            mbar_arrive(&ready[s]);
            return true;
        };
        // outputs of walked tile i are complete: store them, then refill its stage
        auto retire = [&](int i, int &next) -> bool {
            const int slot = i % NOUT;
            if (!warp_agree(mbar_wait_or_abort(&out_full[slot], (i / NOUT) & 1, limit, abort_flag)))
                return false;
            bool ok = true;
            if (lane == 0) {
                uint8_t *ob = smem + Cfg::kOffOut + slot * 3 * Cfg::kAct;
                const int t0 = (ntiles - 1 - i) * TT;
                tma_store_3d(&maps.dx, ob, c0, t0, bb);
                tma_store_3d(&maps.ddt, ob + Cfg::kAct, c0, t0, bb);
                tma_store_3d(&maps.dz, ob + 2 * Cfg::kAct, c0, t0, bb);
                bulk_commit();
                if (next < ntiles) ok = issue(next);
                if (i > 0) {
                    bulk_wait_read<1>();  // the stores of tile i-1 have read their buffers
                    mbar_arrive(&out_free[(i - 1) % NOUT]);
                }
            }
            ++next;
            return warp_agree(ok);
        };
        bool ok = true;
        if (lane == 0) {
            prefetch_tensormap(&maps.x);
            prefetch_tensormap(&maps.dt);
            prefetch_tensormap(&maps.z);
            prefetch_tensormap(&maps.dout);
            prefetch_tensormap(&maps.B);
            prefetch_tensormap(&maps.C);
            prefetch_tensormap(&maps.dx);
            prefetch_tensormap(&maps.ddt);
            prefetch_tensormap(&maps.dz);
            for (int i = 0; i < STAGES && i < ntiles && ok; ++i) ok = issue(i);
        }
        ok = warp_agree(ok);
        int next = STAGES;
        if (ok && ntiles > 0) ok = prepare(0);
        for (int i = 0; i < ntiles && ok; ++i) {
            if (i + 1 < ntiles) ok = prepare(i + 1);
            if (ok) ok = retire(i, next);
        }
        if (!ok) fail();
        if (lane == 0) {
            // nothing in flight may outlive the CTA
            for (int s = 0; s < STAGES; ++s)
                if (last_i[s] >= 0 && !mbar_wait_bounded(&full[s], (last_i[s] / STAGES) & 1, limit))
                    fail();
            bulk_wait<0>();
        }
        __syncwarp();
        return;
    }

    // ============================ compute warps ============================
    const int c_local = warp * CW + lane / G;
    const int sub = lane % G;
    const int gbase = lane & ~(G - 1);
    const int64_t d = c0 + c_local;
    const bool dvalid = d < D;
    const int64_t dc = dvalid ? d : D - 1;
    constexpr int NP = NS / 2;
    float2 a2[NP], Araw[NP], g[NP], dA[NP];
#pragma unroll
    for (int i = 0; i < NP; ++i) {
        const int n = sub * NS + 2 * i;
        Araw[i] = make_float2(__ldg(a.A + dc * N + n), __ldg(a.A + dc * N + n + 1));
        a2[i] = make_float2(Araw[i].x * kLog2e, Araw[i].y * kLog2e);
        g[i] = a.dh_final ? make_float2(__ldg(a.dh_final + (b * D + dc) * N + n),
                                        __ldg(a.dh_final + (b * D + dc) * N + n + 1))
                          : make_float2(0.0f, 0.0f);
        dA[i] = make_float2(0.0f, 0.0f);
    }
    const float bias = a.delta_bias ? __ldg(a.delta_bias + dc) : 0.0f;
    const float dskip = a.D ? __ldg(a.D + dc) : 0.0f;
    float dD_acc = 0.0f, dbias_acc = 0.0f;
    float *part = part_all + warp * TT * 2 * N;
    float *bcs = reinterpret_cast<float *>(smem + Cfg::kOffScr) + warp * Cfg::kScrWords;
    // checkpoints are consumed from the last to the first; the next one is
    // loaded one segment ahead
    const float *ck = a.ckpt + (b * nck * D + dc) * N + sub * NS;  // + c * D * N
    int64_t c_next = nck - 1;
    float2 hnext[NP];
#pragma unroll
    for (int i = 0; i < NP; ++i) hnext[i] = *reinterpret_cast<const float2 *>(ck + c_next * D * N + 2 * i);

    // Every compute warp makes every iteration and reaches both named
    // barriers of each, doing the work only while nothing has aborted.
    bool ok = true;
    for (int it = 0; it < ntiles; ++it) {
        const int k = ntiles - 1 - it;
        const int s = it % STAGES, slot = it % NOUT;
        if (ok) {
            const bool got =
                mbar_wait_or_abort(&ready[s], (it / STAGES) & 1, limit, abort_flag) &&
                mbar_wait_or_abort(&full[s], (it / STAGES) & 1, limit, abort_flag) &&
                (it < NOUT ||
                 mbar_wait_or_abort(&out_free[slot], ((it / NOUT) - 1) & 1, limit, abort_flag));
            ok = warp_agree(got);
            if (!ok) fail();
        }
        const int64_t t_tile = int64_t(k) * TT;
        const int nsteps = static_cast<int>(L - t_tile < TT ? L - t_tile : TT);
        if (ok) {
            const uint8_t *st = smem + s * Cfg::kStage;
            const IoT *xs = reinterpret_cast<const IoT *>(st);
            const IoT *dts = reinterpret_cast<const IoT *>(st + Cfg::kAct);
            const IoT *zs = reinterpret_cast<const IoT *>(st + 2 * Cfg::kAct);
            const IoT *dos = reinterpret_cast<const IoT *>(st + 3 * Cfg::kAct);
            const float *wide = reinterpret_cast<const float *>(smem + Cfg::kOffWide + s * Cfg::kWide);
            uint8_t *ob = smem + Cfg::kOffOut + slot * 3 * Cfg::kAct;
            IoT *dxs = reinterpret_cast<IoT *>(ob);
            IoT *dds = reinterpret_cast<IoT *>(ob + Cfg::kAct);
            IoT *dzs = reinterpret_cast<IoT *>(ob + 2 * Cfg::kAct);
            const int nseg = (nsteps + kCk - 1) / kCk;
#pragma unroll 1
            for (int sg = nseg - 1; sg >= 0; --sg) {
                float2 hcur[NP];
#pragma unroll
                for (int i = 0; i < NP; ++i) hcur[i] = hnext[i];
                if (c_next > 0) {
                    --c_next;
#pragma unroll
                    for (int i = 0; i < NP; ++i)
                        hnext[i] = *reinterpret_cast<const float2 *>(ck + c_next * D * N + 2 * i);
                }
                const int rem = nsteps - sg * kCk;
                if (rem >= kCk)
                    bwd_segment<true, SP, IoT, N, G, CC>(hcur, g, dA, dD_acc, dbias_acc, a2, Araw,
                                                         bias, dskip, xs, dts, zs, dos, wide, dxs,
                                                         dds, dzs, part, bcs, sg * kCk, kCk, c_local,
                                                         sub, gbase, lane);
                else
                    bwd_segment<false, SP, IoT, N, G, CC>(hcur, g, dA, dD_acc, dbias_acc, a2, Araw,
                                                          bias, dskip, xs, dts, zs, dos, wide,
                                                          dxs, dds, dzs, part, bcs, sg * kCk, rem,
                                                          c_local, sub, gbase, lane);
            }
            mbar_arrive(&empty[s]);    // the input stage may be refilled
            fence_proxy_async_smem();  // output tiles, before the TMA engine reads them
            mbar_arrive(&out_full[slot]);
        }
        // this tile's dB | dC partials: the sum over the CTA's warps, to global
        asm volatile("bar.sync 1, %0;" ::"r"(NW * 32) : "memory");
        if (ok) {
            float *dst = a.part_bc + ((b * gridDim.x + blockIdx.x) * L + t_tile) * 2 * N;
            for (int e = tid; e < nsteps * 2 * N; e += NW * 32) {
                float acc = 0.0f;
#pragma unroll
                for (int w = 0; w < NW; ++w) acc += part_all[w * TT * 2 * N + e];
                dst[e] = acc;
            }
        }
        asm volatile("bar.sync 1, %0;" ::"r"(NW * 32) : "memory");
    }
    if (!ok) return;
    // per-sequence parameter partials, and dL/dh0
    float dD_sum = dD_acc, db_sum = dbias_acc;
#pragma unroll
    for (int m = 1; m < G; m <<= 1) {
        dD_sum += __shfl_xor_sync(0xffffffffu, dD_sum, m);
        db_sum += __shfl_xor_sync(0xffffffffu, db_sum, m);
    }
    if (dvalid) {
        float *pp = a.part_par + (b * D + d) * (N + 2);
#pragma unroll
        for (int i = 0; i < NP; ++i) {
            pp[sub * NS + 2 * i] = dA[i].x;
            pp[sub * NS + 2 * i + 1] = dA[i].y;
        }
        if (sub == 0) {
            pp[N] = dD_sum;
            pp[N + 1] = db_sum;
        }
        if (a.dh0) {
#pragma unroll
            for (int i = 0; i < NP; ++i) {
                a.dh0[(b * D + d) * N + sub * NS + 2 * i] = g[i].x;
                a.dh0[(b * D + d) * N + sub * NS + 2 * i + 1] = g[i].y;
            }
        }
    }
}

// --------------------------------------------------------------- reduction
// dB, dC [batch, seqlen, N] = the sum of the ngroups CTA partials; dA [D, N],
// dD, dbias [D] = the sums over the batch; fp64 accumulation in a fixed order.
// grid-stride over (batch * seqlen * 2N) + (D * (N + 2)) elements.
template <typename IoT, int N>
__global__ void __launch_bounds__(256)
    s6_bwd_reduce_kernel(const float *__restrict__ part_bc, const float *__restrict__ part_par,
                         int64_t batch, int64_t seqlen, int64_t d_inner, int64_t ngroups, IoT *dB,
                         IoT *dC, float *dA, float *dD, float *dbias) {
    const int64_t n_bc = batch * seqlen * 2 * N;
    const int64_t n_par = d_inner * (N + 2);
    for (int64_t e = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; e < n_bc + n_par;
         e += static_cast<int64_t>(gridDim.x) * blockDim.x) {
        if (e < n_bc) {
            const int64_t slot = e % (2 * N), bt = e / (2 * N);
            const int64_t b = bt / seqlen, t = bt % seqlen;
            double acc = 0.0;
            for (int64_t gi = 0; gi < ngroups; ++gi)
                acc += part_bc[((b * ngroups + gi) * seqlen + t) * 2 * N + slot];
            IoT *o = slot < N ? dB : dC;
            o[bt * N + (slot % N)] = from_f32<IoT>(static_cast<float>(acc));
        } else {
            const int64_t f = e - n_bc;
            const int64_t dd = f / (N + 2), j = f % (N + 2);
            double acc = 0.0;
            for (int64_t b = 0; b < batch; ++b) acc += part_par[(b * d_inner + dd) * (N + 2) + j];
            if (j < N) {
                if (dA) dA[dd * N + j] = static_cast<float>(acc);
            }
            else if (j == N) {
                if (dD) dD[dd] = static_cast<float>(acc);
            } else if (dbias) {
                dbias[dd] = static_cast<float>(acc);
            }
        }
    }
}

}  // namespace jssm
