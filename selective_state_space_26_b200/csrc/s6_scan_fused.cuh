// s6_scan_fused.cuh -- prefill selective scan (S6), fused-warp form (sm_100a).
//
// The recurrence of the "Mamba 레이어" section of the Jamba notes, read as
// h = exp(Delta A) h + Delta B x, out = (C.h + D x) silu(z),
// Delta = softplus(delta + bias) (per-step pieces in s6_scan.cuh), organised so
// that every warp that carries states also does the per-(t, d) scalar work of
// its own channels -- no hand-off of Delta or of C.h through shared memory:
//
//  * NW compute warps; lane (d, sub) of a warp holds N/G states of channel d
//    in registers for the whole sequence.  In each group of G consecutive
//    steps lane `sub` owns step sub: it loads x, delta, z of that (t, d),
//    computes Delta (softplus) and Delta x, and broadcasts them to the other
//    G-1 lanes of the channel with shuffles; each lane advances its states
//    through the G steps (packed fp32x2 math, Abar = 2^(Delta A log2 e) on the
//    MUFU); a transposing butterfly sums the G partial C.h of each step onto
//    the owner, which applies the skip and the gate and writes the output tile.
//  * One producer warp: lane 0 issues the TMA loads (no multicast) of the x,
//    delta, z tiles [TT x CC] and of B, C [TT x N] into a STAGES-deep ring and
//    the TMA stores of the output tiles; all 32 lanes regroup each tile's B
//    and C into per-lane slots (load_bc) once for every channel of the CTA.
//  * Persistent CTAs over (sequence, channel-group) tasks; the tiles of a CTA's
//    tasks form one stream.
//  * Every wait is a bounded mbarrier wait that also watches a CTA abort flag;
//    a wait that runs out records JAMBA_SSM_ERR_TIMEOUT, every warp leaves its
//    loop, and the producer waits (bounded) for copies still in flight.
#pragma once

#include <type_traits>

#include "device_utils.cuh"
#include "s6_math.cuh"
#include "s6_scan.cuh"

namespace jssm {

// IoT: I/O element type; N: d_state; G: lanes per channel; NW: compute warps;
// TT: time tile; STAGES: TMA ring depth.
template <typename IoT, int N_, int G_, int NW_, int TT_, int STAGES_>
struct FusedCfg {
    static constexpr int N = N_, G = G_, NW = NW_, TT = TT_, STAGES = STAGES_;
    static constexpr int NS = N / G;    // states per lane
    static constexpr int CW = 32 / G;   // channels per warp
    static constexpr int CC = NW * CW;  // channels per CTA tile
    static_assert((CC * (int)sizeof(IoT)) % 16 == 0, "TMA boxes and offsets of 16-byte multiples");
    static constexpr int kThreads = (NW + 1) * 32;
    static constexpr int VEC = 16 / (int)sizeof(IoT);
    static_assert(NS == 2 || (NS % 4 == 0 && NS >= 4), "a lane reads its B/C slice as float2/float4");
    static_assert(32 % G == 0 && TT % G == 0, "step groups of G");
    static_assert(N % VEC == 0, "B / C rows are whole 16-byte TMA units");
    static constexpr int kActTile = TT * CC * (int)sizeof(IoT);
    static constexpr int kBCTile = TT * N * (int)sizeof(IoT);
    static constexpr int kStageBytes = 3 * kActTile + 2 * kBCTile;
    static_assert(kActTile % 128 == 0 && kBCTile % 128 == 0, "TMA destinations 128B aligned");
    // staged fp32 B / C rows ([G][2][NS] floats per step, see load_bc)
    static constexpr int kBCRow = 2 * N;
    static constexpr int kBCe = TT * kBCRow;  // floats per stage
    static constexpr int kOffBCs = STAGES * kStageBytes;
    static constexpr int NOUT = 3;  // output tiles in flight (compute, TMA store, spare)
    static constexpr int kOffOut = kOffBCs + STAGES * kBCe * 4;
    static_assert(kOffOut % 128 == 0, "TMA store source 128B aligned");
    // full[S], bc_ready[S], out_full[NOUT], out_free[NOUT]
    static constexpr int kOffBar = kOffOut + NOUT * kActTile;
    static constexpr int kNumBars = 2 * STAGES + 2 * NOUT;
    static constexpr int kOffFlag = kOffBar + kNumBars * 8;
    static constexpr int kSmemBytes = kOffFlag + 16;
    static constexpr uint32_t kTxBytes = kStageBytes;
};

// Per-lane scalars of the step a lane owns: Delta, Delta x, and the skip and
// gate folded as out = y * gate + skg (skg = D x gate).
struct OwnedStep {
    float dl, dx, gate, skg;
};

template <bool SOFTPLUS, bool LDS, bool NO_OUT, typename IoT>
__device__ __forceinline__ OwnedStep owned_step(const IoT *xs, const IoT *dts, const IoT *zs, int idx,
                                                float bias, float dskip) {
    const float xo = LDS ? lds_f32(xs + idx) : to_f32(xs[idx]);
    const float v = (LDS ? lds_f32(dts + idx) : to_f32(dts[idx])) + bias;
    const float dl = SOFTPLUS ? softplus_io<IoT>(v) : v;
    if (NO_OUT) return OwnedStep{dl, dl * xo, 0.0f, 0.0f};  // no output, no gate
    const float gate = silu_f32(LDS ? lds_f32(zs + idx) : to_f32(zs[idx]));
    return OwnedStep{dl, dl * xo, gate, dskip * xo * gate};
}

// Delta and Delta x of the G steps owned in `o` gathered from the channel's
// lanes, and the group's Abar = exp(Delta A) (NS / 2 packed multiplies and NS
// MUFU ex2 per step).
template <int G, int NS>
__device__ __forceinline__ void group_exps(const OwnedStep &o, const float2 (&a2)[NS / 2], int gbase,
                                           float2 (&dxp)[G], float2 (&ab)[G][NS / 2]) {
#pragma unroll
    for (int j = 0; j < G; ++j) {
        const float dl = G == 1 ? o.dl : __shfl_sync(0xffffffffu, o.dl, gbase | j);
        const float dx = G == 1 ? o.dx : __shfl_sync(0xffffffffu, o.dx, gbase | j);
        dxp[j] = make_float2(dx, dx);
#pragma unroll
        for (int i = 0; i < NS / 2; ++i) {
            const float2 arg = mul2(make_float2(dl, dl), a2[i]);
            ab[j][i] = make_float2(ex2_mufu(arg.x), ex2_mufu(arg.y));
        }
    }
}

// One full tile (TT steps) of a compute lane.  Lane `sub` of each channel
// owns steps sub, sub + G, ... of the tile: it computes their Delta, Delta x,
// gate and skip (owned_step) and hands Delta and Delta x to the channel's
// other lanes by shuffles.  The loop is software-pipelined over groups of G
// steps because a sub-partition holds only a few of these warps and issue is
// in order (a warp whose next instruction waits on a dependency issues
// nothing): while the states of group g advance, the exps of group g+2 are
// issued and the owners' softplus / gate of group g+3 are computed, so an
// exp's result is consumed about 2G steps after issue even when the MUFU
// queue is long.  SOFTPLUS is a template parameter: a runtime test inside the
// unrolled body would split it into basic blocks that the scheduler cannot
// interleave.
//
// MODE 0: the forward.  MODE 1 (the backward's checkpoint pass): only the
// states advance; before every kCk-th step of the tile the lane stores its NS
// states at ck + (step / kCk) * ck_stride (ck null: nothing stored), and the
// readout, gate and output tile are skipped.  MODE 2: the forward, storing the
// same checkpoints as it goes (for a backward that follows).
template <bool SOFTPLUS, typename IoT, int N, int G, int NS, int TT, int CC, int BCROW,
          int MODE = 0>
__device__ __forceinline__ void fused_tile_full(float2 (&h)[NS / 2], const float2 (&a2)[NS / 2],
                                                float bias, float dskip,
                                                const IoT *xs, const IoT *dts, const IoT *zs,
                                                const float *bcs, IoT *outs, int c_local, int sub,
                                                int gbase, float *ck = nullptr,
                                                int64_t ck_stride = 0) {
    constexpr int NG = TT / G;
    static_assert(NG >= 3, "a tile holds at least three groups");
    constexpr bool LDS = G == 2;  // explicit shared-space accesses (see load_bc_shared)
    constexpr bool kStoreCk = MODE != 0, kNoOut = MODE == 1;
    static_assert(!kStoreCk || (TT % kCk == 0 && kCk % G == 0), "checkpoints at group starts");
    OwnedStep o0 = owned_step<SOFTPLUS, LDS, kNoOut>(xs, dts, zs, sub * CC + c_local, bias, dskip);
    OwnedStep o1 = owned_step<SOFTPLUS, LDS, kNoOut>(xs, dts, zs, (G + sub) * CC + c_local, bias, dskip);
    OwnedStep o2 = owned_step<SOFTPLUS, LDS, kNoOut>(xs, dts, zs, (2 * G + sub) * CC + c_local, bias, dskip);
    float2 dxa[G], aba[G][NS / 2], dxb[G], abb[G][NS / 2];
    group_exps<G, NS>(o0, a2, gbase, dxa, aba);
    group_exps<G, NS>(o1, a2, gbase, dxb, abb);
#pragma unroll
    for (int g = 0; g < NG; ++g) {
        const int t0 = g * G;
        OwnedStep o3 = o2;
        if (g + 3 < NG)
            o3 = owned_step<SOFTPLUS, LDS, kNoOut>(xs, dts, zs, (t0 + 3 * G + sub) * CC + c_local, bias, dskip);
        float2 dxc[G], abc[G][NS / 2];
        float yp[G];
        if (kStoreCk && (t0 % kCk) == 0 && ck) store_states<NS>(ck + (t0 / kCk) * ck_stride, h);
#pragma unroll
        for (int j = 0; j < G; ++j) {
            if (g + 2 < NG) {
                const float dl = G == 1 ? o2.dl : __shfl_sync(0xffffffffu, o2.dl, gbase | j);
                const float dx = G == 1 ? o2.dx : __shfl_sync(0xffffffffu, o2.dx, gbase | j);
                dxc[j] = make_float2(dx, dx);
#pragma unroll
                for (int i = 0; i < NS / 2; ++i) {
                    const float2 arg = mul2(make_float2(dl, dl), a2[i]);
                    abc[j][i] = make_float2(ex2_mufu(arg.x), ex2_mufu(arg.y));
                }
            }
            const BCPairs<NS> bc = LDS ? load_bc_shared<NS>(bcs + (t0 + j) * BCROW, sub)
                                       : load_bc<NS>(bcs + (t0 + j) * BCROW, sub);
            float2 y2;
#pragma unroll
            for (int i = 0; i < NS / 2; ++i) {
                h[i] = fma2(aba[j][i], h[i], mul2(dxa[j], bc.b[i]));
                if (!kNoOut) y2 = i == 0 ? mul2(bc.c[i], h[i]) : fma2(bc.c[i], h[i], y2);
            }
            yp[j] = kNoOut ? 0.0f : y2.x + y2.y;
        }
        if (!kNoOut) {
            const float y = reduce_transpose<G>(yp, sub);
            const IoT ov = from_f32<IoT>(fmaf(y, o0.gate, o0.skg));
            if (LDS)
                sts_io(outs + (t0 + sub) * CC + c_local, ov);
            else
                outs[(t0 + sub) * CC + c_local] = ov;
        }
#pragma unroll
        for (int j = 0; j < G; ++j) {
            dxa[j] = dxb[j];
            if (g + 2 < NG) dxb[j] = dxc[j];
#pragma unroll
            for (int i = 0; i < NS / 2; ++i) {
                aba[j][i] = abb[j][i];
                if (g + 2 < NG) abb[j][i] = abc[j][i];
            }
        }
        o0 = o1;
        o1 = o2;
        o2 = o3;
    }
}

// MODE (see fused_tile_full): 0 the forward; 1 the backward's checkpoint pass
// (no z or C loads, no output stores); 2 the forward storing checkpoints.  In
// modes 1 and 2 args.ckpt receives the states before every kCk-th step.
template <typename IoT, int N, int G, int NW, int TT, int STAGES, int MODE = 0>
__global__ void __launch_bounds__((NW + 1) * 32, 1)
    s6_scan_fused_kernel(const __grid_constant__ CUtensorMap tm_x,
                         const __grid_constant__ CUtensorMap tm_dt,
                         const __grid_constant__ CUtensorMap tm_z,
                         const __grid_constant__ CUtensorMap tm_B,
                         const __grid_constant__ CUtensorMap tm_C,
                         const __grid_constant__ CUtensorMap tm_out, const ScanArgs args) {
    using Cfg = FusedCfg<IoT, N, G, NW, TT, STAGES>;
    constexpr int NS = Cfg::NS, CW = Cfg::CW, CC = Cfg::CC, NOUT = Cfg::NOUT;
    extern __shared__ __align__(1024) uint8_t smem[];
    uint64_t *full = reinterpret_cast<uint64_t *>(smem + Cfg::kOffBar);
    uint64_t *bc_ready = full + STAGES;
    uint64_t *out_full = bc_ready + STAGES;
    uint64_t *out_free = out_full + NOUT;
    volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + Cfg::kOffFlag);
    float *bcs_all = reinterpret_cast<float *>(smem + Cfg::kOffBCs);

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int64_t d_inner = args.d_inner, seqlen = args.seqlen;
    const int64_t ngroups = (d_inner + CC - 1) / CC;
    const int64_t ntasks = args.batch * ngroups;
    const int ntiles = static_cast<int>((seqlen + TT - 1) / TT);
    constexpr bool kStoreCk = MODE != 0, kNoOut = MODE == 1;
    const int64_t nck = (seqlen + kCk - 1) / kCk;  // checkpoints per sequence (modes 1, 2)
    const int64_t my_tasks =
        static_cast<int64_t>(blockIdx.x) < ntasks ? (ntasks - 1 - blockIdx.x) / gridDim.x + 1 : 0;
    const int64_t total = my_tasks * ntiles;
    const uint64_t limit = args.timeout_cycles;

    if (tid == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&bc_ready[s], 32);
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
        *abort_flag = 1;
        record_status(args.status, kStTimeout);
    };
    // (sequence, first channel, tile index) of the CTA's g-th tile.  Callers
    // walk g upward, so the cursor advances without 64-bit divisions except
    // when it has to jump.
    struct Cursor {
        int64_t g = -1, b = 0;
        int c0 = 0, k = 0;
    };
    auto seek = [&](Cursor &cu, int64_t g) {
        if (g == cu.g + 1 && cu.g >= 0 && cu.k + 1 < ntiles) {
            ++cu.k;
        } else if (g == cu.g + 1 && cu.g >= 0) {
            cu.k = 0;
            int64_t task = cu.b * ngroups + cu.c0 / CC + gridDim.x;
            cu.b = task / ngroups;
            cu.c0 = static_cast<int>((task % ngroups) * CC);
        } else if (g != cu.g) {
            const int64_t j = g / ntiles;
            cu.k = static_cast<int>(g - j * ntiles);
            const int64_t task = blockIdx.x + j * gridDim.x;
            cu.b = task / ngroups;
            cu.c0 = static_cast<int>((task % ngroups) * CC);
        }
        cu.g = g;
    };
    auto tile_of = [&](Cursor &cu, int64_t g, int64_t &b, int &c0, int &k) {
        seek(cu, g);
        b = cu.b;
        c0 = cu.c0;
        k = cu.k;
    };
    auto steps_in = [&](int k) {
        const int64_t rem = seqlen - int64_t(k) * TT;
        return static_cast<int>(rem < TT ? rem : TT);
    };

    if (warp == NW) {
        // ============ producer warp: TMA loads / stores, B and C widening ============
        uint32_t armed = 0;
        int64_t issued = 0;
        Cursor cur_issue, cur_main, cur_store;
        auto issue = [&](int64_t g) {  // lane 0 only
            if (g >= total) return;
            issued = g + 1;
            int64_t b;
            int c0, k;
            tile_of(cur_issue, g, b, c0, k);
            const int s = static_cast<int>(g % STAGES);
            if ((args.debug_flags & 1u) && k == 0) return;  // test hook: withhold a first tile
            uint8_t *base = smem + s * Cfg::kStageBytes;
            mbar_arrive_expect_tx(&full[s], kNoOut ? Cfg::kTxBytes - Cfg::kActTile - Cfg::kBCTile
                                                 : Cfg::kTxBytes);
            const int t0 = k * TT, bb = static_cast<int>(b);
            tma_load_3d(base, &tm_x, c0, t0, bb, &full[s]);
            tma_load_3d(base + Cfg::kActTile, &tm_dt, c0, t0, bb, &full[s]);
            if (!kNoOut) tma_load_3d(base + 2 * Cfg::kActTile, &tm_z, c0, t0, bb, &full[s]);
            tma_load_3d(base + 3 * Cfg::kActTile, &tm_B, 0, t0, bb, &full[s]);
            if (!kNoOut)
                tma_load_3d(base + 3 * Cfg::kActTile + Cfg::kBCTile, &tm_C, 0, t0, bb, &full[s]);
            armed |= 1u << s;
        };
        // store of tile g (its output buffer is complete), then release stage g
        auto retire = [&](int64_t g) -> bool {
            const int slot = static_cast<int>(g % NOUT);
            if (!warp_agree(mbar_wait_or_abort(&out_full[slot], static_cast<uint32_t>(g / NOUT) & 1u,
                                               limit, abort_flag)))
                return false;
            if (lane == 0) {
                if (!kNoOut) {
                    int64_t b;
                    int c0, k;
                    tile_of(cur_store, g, b, c0, k);
                    tma_store_3d(&tm_out, smem + Cfg::kOffOut + slot * Cfg::kActTile, c0, k * TT,
                                 static_cast<int>(b));
                    bulk_commit();
                }
                issue(g + STAGES);  // the compute warps are done with stage g % STAGES
                if (g > 0) {
                    if (!kNoOut) bulk_wait_read<1>();  // the store of tile g-1 has read its buffer
                    mbar_arrive(&out_free[static_cast<int>((g - 1) % NOUT)]);
                }
            }
            __syncwarp();
            return true;
        };
        if (lane == 0) {
            prefetch_tensormap(&tm_x);
            prefetch_tensormap(&tm_dt);
            prefetch_tensormap(&tm_z);
            prefetch_tensormap(&tm_B);
            prefetch_tensormap(&tm_C);
            prefetch_tensormap(&tm_out);
            for (int64_t g = 0; g < STAGES; ++g) issue(g);
        }
        __syncwarp();
        int64_t consumed = 0;
        // tile g's B and C regrouped into per-lane slots (after its TMA load landed)
        auto widen = [&](int64_t g) -> bool {
            int64_t b;
            int c0, k;
            tile_of(cur_main, g, b, c0, k);
            const int s = static_cast<int>(g % STAGES);
            if (!warp_agree(mbar_wait_or_abort(&full[s], static_cast<uint32_t>(g / STAGES) & 1u,
                                               limit, abort_flag)))
                return false;
            consumed = g + 1;
            if (lane == 0) armed &= ~(1u << s);
            const int nsteps = steps_in(k);
            const uint8_t *base = smem + s * Cfg::kStageBytes;
            const IoT *Bs = reinterpret_cast<const IoT *>(base + 3 * Cfg::kActTile);
            const IoT *Cs = reinterpret_cast<const IoT *>(base + 3 * Cfg::kActTile + Cfg::kBCTile);
            float *dst = bcs_all + s * Cfg::kBCe;
            // unit u = (step t, slot j, half: 0 = B, 1 = C): one slice of NS values
            // (B only for checkpoints)
            constexpr int kHalves = kNoOut ? 1 : 2;
            for (int u = lane; u < nsteps * kHalves * G; u += 32) {
                const int t = u / (kHalves * G), j = (u / kHalves) % G;
                const int half = kNoOut ? 0 : (u & 1);
                stage_slice<NS>(dst + t * Cfg::kBCRow + (2 * j + half) * NS,
                                (half ? Cs : Bs) + t * N + j * NS);
            }
            mbar_arrive(&bc_ready[s]);
            return true;
        };
        // tile g+1 is widened before tile g is waited for, so the compute warps
        // find the next tile ready when they finish the current one
        bool ok = total == 0 || widen(0);
        for (int64_t g = 0; ok && g < total; ++g) {
            if (g + 1 < total) ok = widen(g + 1);
            if (ok) ok = retire(g);
        }
        if (!ok) fail();
        if (lane == 0) {
            for (int64_t g = consumed; g < issued; ++g) {
                const int s = static_cast<int>(g % STAGES);
                if (armed & (1u << s)) {
                    mbar_wait_bounded(&full[s], static_cast<uint32_t>(g / STAGES) & 1u, limit);
                    armed &= ~(1u << s);
                }
            }
            bulk_wait<0>();
        }
        return;
    }

    // =========================== compute warps ===========================
    const int c_local = warp * CW + lane / G;
    const int sub = lane % G;
    const int gbase = lane & ~(G - 1);  // first lane of this channel's group
    const bool use_softplus = args.delta_softplus != 0;
    float2 a2[NS / 2], h[NS / 2];
    int64_t d = 0;
    bool dvalid = false;
    float bias = 0.0f, dskip = 0.0f;
    bool ok = true;
    Cursor cur;
    for (int64_t g = 0; ok && g < total; ++g) {
        int64_t b;
        int c0, k;
        tile_of(cur, g, b, c0, k);
        if (k == 0) {
            d = c0 + c_local;
            dvalid = d < d_inner;
#pragma unroll
            for (int i = 0; i < NS / 2; ++i) {
                const int n = sub * NS + 2 * i;
                a2[i] = dvalid ? make_float2(__ldg(args.A + d * N + n) * kLog2e,
                                             __ldg(args.A + d * N + n + 1) * kLog2e)
                               : make_float2(0.0f, 0.0f);
                h[i] = (dvalid && args.h0)
                           ? make_float2(__ldg(args.h0 + (b * d_inner + d) * N + n),
                                         __ldg(args.h0 + (b * d_inner + d) * N + n + 1))
                           : make_float2(0.0f, 0.0f);
            }
            bias = (dvalid && args.delta_bias) ? __ldg(args.delta_bias + d) : 0.0f;
            dskip = (dvalid && args.D) ? __ldg(args.D + d) : 0.0f;
        }
        const int s = static_cast<int>(g % STAGES);
        const int slot = static_cast<int>(g % NOUT);
        // the output buffer was last used by tile g - NOUT, whose store must
        // have read it (the (g / NOUT - 1)-th release of this buffer)
        const bool got =
            mbar_wait_or_abort(&bc_ready[s], static_cast<uint32_t>(g / STAGES) & 1u, limit,
                               abort_flag) &&
            mbar_wait_or_abort(&full[s], static_cast<uint32_t>(g / STAGES) & 1u, limit, abort_flag) &&
            (g < NOUT ||
             mbar_wait_or_abort(&out_free[slot], static_cast<uint32_t>(g / NOUT - 1) & 1u, limit,
                                abort_flag));
        if (!warp_agree(got)) {
            ok = false;
            break;
        }
        const int nsteps = steps_in(k);
        const uint8_t *base = smem + s * Cfg::kStageBytes;
        const IoT *xs = reinterpret_cast<const IoT *>(base);
        const IoT *dts = reinterpret_cast<const IoT *>(base + Cfg::kActTile);
        const IoT *zs = reinterpret_cast<const IoT *>(base + 2 * Cfg::kActTile);
        const float *bcs = bcs_all + s * Cfg::kBCe;
        IoT *outs = reinterpret_cast<IoT *>(smem + Cfg::kOffOut + slot * Cfg::kActTile);
        // checkpoint pass: this lane's slice of the tile's first checkpoint
        float *ck = nullptr;
        const int64_t ck_stride = d_inner * N;
        if (kStoreCk && dvalid)
            ck = args.ckpt + ((b * nck + int64_t(k) * (TT / kCk)) * d_inner + d) * N + sub * NS;

        // One group of G steps starting at t0: the owner lane's scalars, the
        // exchange, G recurrence steps, the butterfly, the owner's output.
        auto group = [&](int t0, int valid) {
            const int t_own = t0 + sub;
            const int idx = t_own * CC + c_local;
            const float xo = to_f32(xs[idx]);
            const float dl = delta_io<IoT>(to_f32(dts[idx]), bias, use_softplus);
            const float dx = dl * xo;
            if (kStoreCk && (t0 % kCk) == 0 && ck) store_states<NS>(ck + (t0 / kCk) * ck_stride, h);
            float yp[G];
#pragma unroll
            for (int j = 0; j < G; ++j) {
                const float dlj = G == 1 ? dl : __shfl_sync(0xffffffffu, dl, gbase | j);
                const float dxj = G == 1 ? dx : __shfl_sync(0xffffffffu, dx, gbase | j);
                yp[j] = 0.0f;
                if (j < valid)
                    yp[j] = recurrence_step<NS>(h, a2, make_float2(dlj, dxj),
                                                bcs + (t0 + j) * Cfg::kBCRow, sub);
            }
            if (!kNoOut) {
                const float y = reduce_transpose<G>(yp, sub);
                const float gate = silu_f32(to_f32(zs[idx]));
                if (sub < valid) outs[idx] = from_f32<IoT>((y + dskip * xo) * gate);
            }
        };
        if (nsteps == TT && use_softplus) {
            fused_tile_full<true, IoT, N, G, NS, TT, CC, Cfg::kBCRow, MODE>(
                h, a2, bias, dskip, xs, dts, zs, bcs, outs, c_local, sub, gbase, ck, ck_stride);
        } else if (nsteps == TT) {
            fused_tile_full<false, IoT, N, G, NS, TT, CC, Cfg::kBCRow, MODE>(
                h, a2, bias, dskip, xs, dts, zs, bcs, outs, c_local, sub, gbase, ck, ck_stride);
        } else {
            for (int t0 = 0; t0 < nsteps; t0 += G) group(t0, nsteps - t0 < G ? nsteps - t0 : G);
        }
        fence_proxy_async_smem();  // output tile (and this tile's stage reads) before TMA
        mbar_arrive(&out_full[slot]);
        if (k == ntiles - 1 && dvalid && args.h_final) {
#pragma unroll
            for (int i = 0; i < NS / 2; ++i) {
                float *o = args.h_final + (b * d_inner + d) * N + sub * NS + 2 * i;
                o[0] = h[i].x;
                o[1] = h[i].y;
            }
        }
    }
    if (!ok) fail();
}

}  // namespace jssm
