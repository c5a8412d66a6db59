// s6_scan_serving.cuh -- the prefill scan for serving layouts (sm_100a):
// packed variable-length sequences (cu_seqlens) and per-sequence state-cache
// slots (state_indices).  Same warp roles, tile body and pipeline as the
// batched kernel in s6_scan_fused.cuh (whose per-step code it reuses); it
// differs in the tile schedule -- each sequence has its own number of tiles,
// which the producer warp publishes per stage in a small descriptor -- in the
// addressing of the initial / final states, and in storing the last, short
// tile of a packed sequence row by row.  It is a separate kernel because code
// around the unrolled tile body changes how the whole kernel is scheduled:
// folding this bookkeeping into the batched kernel cost it 15 % at batch 1.
#pragma once

#include "s6_scan_fused.cuh"

namespace jssm {

template <typename IoT, int N, int G, int NW, int TT, int STAGES>
struct ServingCfg : FusedCfg<IoT, N, G, NW, TT, STAGES> {
    using Base = FusedCfg<IoT, N, G, NW, TT, STAGES>;
    // per stage, the descriptor of the tile it holds (TileHdr, written by the
    // producer before it arms the stage)
    static constexpr int kOffHdr = Base::kOffBar + Base::kNumBars * 8;
    static constexpr int kOffFlag = kOffHdr + STAGES * 16;
    static constexpr int kSmemBytes = kOffFlag + 16;
};

// What the compute warps need of a tile, published by the producer with the
// stage so that they carry no tile cursor of their own (its registers would be
// live across the unrolled tile body).
struct TileHdr {
    int32_t b;       // sequence
    int32_t c0;      // first channel
    int32_t nsteps;  // valid steps (0 for an empty sequence)
    int32_t flags;   // bit 0: first tile of its task, bit 1: last
};

template <typename IoT, int N, int G, int NW, int TT, int STAGES>
__global__ void __launch_bounds__((NW + 1) * 32, 1)
    s6_scan_serving_kernel(const __grid_constant__ CUtensorMap tm_x,
                           const __grid_constant__ CUtensorMap tm_dt,
                           const __grid_constant__ CUtensorMap tm_z,
                           const __grid_constant__ CUtensorMap tm_B,
                           const __grid_constant__ CUtensorMap tm_C,
                           const __grid_constant__ CUtensorMap tm_out, const ScanArgs args) {
    using Cfg = ServingCfg<IoT, N, G, NW, TT, STAGES>;
    constexpr int NS = Cfg::NS, CW = Cfg::CW, CC = Cfg::CC, NOUT = Cfg::NOUT;
    extern __shared__ __align__(1024) uint8_t smem[];
    uint64_t *full = reinterpret_cast<uint64_t *>(smem + Cfg::kOffBar);
    uint64_t *bc_ready = full + STAGES;
    uint64_t *out_full = bc_ready + STAGES;
    uint64_t *out_free = out_full + NOUT;
    volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + Cfg::kOffFlag);
    TileHdr *hdr = reinterpret_cast<TileHdr *>(smem + Cfg::kOffHdr);
    float *bcs_all = reinterpret_cast<float *>(smem + Cfg::kOffBCs);

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int64_t d_inner = args.d_inner;
    const int64_t ngroups = (d_inner + CC - 1) / CC;
    const int64_t ntasks = args.batch * ngroups;
    const bool packed = args.cu_seqlens != nullptr;  // else the batched layout
    const uint64_t limit = args.timeout_cycles;

    // Token rows [start, start + len) of sequence b: the whole batch row, or
    // its slice of the packed layout (offsets clamped to [0, total_tokens]).
    auto seq_range = [&](int64_t b, int64_t &start, int64_t &len) {
        if (packed) {
            const int64_t tot = args.total_tokens;
            int64_t s0 = __ldg(args.cu_seqlens + b), s1 = __ldg(args.cu_seqlens + b + 1);
            s0 = s0 < 0 ? 0 : (s0 > tot ? tot : s0);
            s1 = s1 < s0 ? s0 : (s1 > tot ? tot : s1);
            start = s0;
            len = s1 - s0;
        } else {
            start = 0;
            len = args.seqlen;
        }
    };
    // an empty sequence still takes one (zero-step) tile: it hands its initial
    // state on as its final state
    auto tiles_for = [](int64_t len) { return len > 0 ? (len + TT - 1) / TT : int64_t(1); };
    int64_t total = 0;  // tiles of this CTA's tasks
    if (!packed) {
        const int64_t my_tasks =
            static_cast<int64_t>(blockIdx.x) < ntasks ? (ntasks - 1 - blockIdx.x) / gridDim.x + 1 : 0;
        total = my_tasks * tiles_for(args.seqlen);
    } else {
        for (int64_t task = blockIdx.x; task < ntasks; task += gridDim.x) {
            int64_t st, ln;
            seq_range(task / ngroups, st, ln);
            total += tiles_for(ln);
        }
    }

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
    // The CTA's g-th tile: task (sequence b, channels from c0), tile k of the
    // task.  Every caller walks g upward one at a time, so the cursor only
    // steps (a 64-bit division per task change).
    struct Cursor {
        int64_t g = -1, task = 0, b = 0, start = 0, len = 0, nt = 0;
        int c0 = 0, k = 0;
    };
    struct Tile {
        int64_t b, row;  // sequence, first token row of the tile
        int c0, k, nsteps;
        bool last;       // last tile of its task
    };
    auto load_task = [&](Cursor &cu, int64_t task) {
        cu.task = task;
        cu.b = task / ngroups;
        cu.c0 = static_cast<int>((task % ngroups) * CC);
        cu.k = 0;
        seq_range(cu.b, cu.start, cu.len);
        cu.nt = tiles_for(cu.len);
    };
    auto tile_of = [&](Cursor &cu, int64_t g) -> Tile {
        if (cu.g < 0 || g < cu.g) {
            load_task(cu, blockIdx.x);
            cu.g = 0;
        }
        while (cu.g < g) {
            if (cu.k + 1 < cu.nt) ++cu.k;
            else load_task(cu, cu.task + gridDim.x);
            ++cu.g;
        }
        const int64_t rem = cu.len - static_cast<int64_t>(cu.k) * TT;
        Tile t;
        t.b = cu.b;
        t.row = cu.start + static_cast<int64_t>(cu.k) * TT;
        t.c0 = cu.c0;
        t.k = cu.k;
        t.nsteps = static_cast<int>(rem <= 0 ? 0 : (rem < TT ? rem : TT));
        t.last = cu.k + 1 == cu.nt;
        return t;
    };

    if (warp == NW) {
        // ============ producer warp: TMA loads / stores, B and C widening ============
        uint32_t armed = 0;
        int64_t issued = 0;
        Cursor cur_issue, cur_main, cur_store;
        auto issue = [&](int64_t g) {  // lane 0 only
            if (g >= total) return;
            issued = g + 1;
            const Tile t = tile_of(cur_issue, g);
            const int s = static_cast<int>(g % STAGES);
            if ((args.debug_flags & 1u) && t.k == 0) return;  // test hook: withhold a first tile
            uint8_t *base = smem + s * Cfg::kStageBytes;
            hdr[s] = TileHdr{static_cast<int32_t>(t.b), t.c0, t.nsteps,
                             (t.k == 0 ? 1 : 0) | (t.last ? 2 : 0)};
            mbar_arrive_expect_tx(&full[s], Cfg::kTxBytes);  // releases the header too
            // rows past the tile's sequence are loaded too (the next sequence,
            // or zero fill past the tensor) and never used
            const int r = static_cast<int>(t.row), bb = packed ? 0 : static_cast<int>(t.b);
            tma_load_3d(base, &tm_x, t.c0, r, bb, &full[s]);
            tma_load_3d(base + Cfg::kActTile, &tm_dt, t.c0, r, bb, &full[s]);
            tma_load_3d(base + 2 * Cfg::kActTile, &tm_z, t.c0, r, bb, &full[s]);
            tma_load_3d(base + 3 * Cfg::kActTile, &tm_B, 0, r, bb, &full[s]);
            tma_load_3d(base + 3 * Cfg::kActTile + Cfg::kBCTile, &tm_C, 0, r, bb, &full[s]);
            armed |= 1u << s;
        };
        // store of tile g (its output buffer is complete), then release stage g
        auto retire = [&](int64_t g) -> bool {
            const int slot = static_cast<int>(g % NOUT);
            if (!warp_agree(mbar_wait_or_abort(&out_full[slot], static_cast<uint32_t>(g / NOUT) & 1u,
                                               limit, abort_flag)))
                return false;
            const Tile t = tile_of(cur_store, g);
            const uint8_t *ob = smem + Cfg::kOffOut + slot * Cfg::kActTile;
            // In the packed layout the rows after a sequence's last step belong
            // to the next sequence, so a short tile is stored row by row with
            // 16-byte stores of its valid channels (a whole-box TMA store is
            // only clipped at the tensor's end).
            const bool rowwise = packed && t.nsteps < TT;
            if (rowwise) {
                constexpr int EV = 16 / (int)sizeof(IoT), CPR = CC / EV;  // 16-byte chunks per row
                IoT *outg = static_cast<IoT *>(args.out);
                for (int u = lane; u < t.nsteps * CPR; u += 32) {
                    const int tr = u / CPR, qc = u % CPR;
                    const int64_t c = t.c0 + qc * EV;
                    if (c < d_inner)
                        *reinterpret_cast<uint4 *>(outg + (t.row + tr) * d_inner + c) =
                            *reinterpret_cast<const uint4 *>(ob + (tr * CC + qc * EV) * sizeof(IoT));
                }
                __syncwarp();
            }
            if (lane == 0) {
                if (!rowwise)
                    tma_store_3d(&tm_out, ob, t.c0, static_cast<int>(t.row),
                                 packed ? 0 : static_cast<int>(t.b));
                bulk_commit();  // one bulk group per tile, empty for a row-wise tile
                issue(g + STAGES);  // the compute warps are done with stage g % STAGES
                if (g > 0) {
                    bulk_wait_read<1>();  // the store of tile g-1 has read its buffer
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
            const Tile t = tile_of(cur_main, g);
            const int s = static_cast<int>(g % STAGES);
            if (!warp_agree(mbar_wait_or_abort(&full[s], static_cast<uint32_t>(g / STAGES) & 1u,
                                               limit, abort_flag)))
                return false;
            consumed = g + 1;
            if (lane == 0) armed &= ~(1u << s);
            const int nsteps = t.nsteps;
            const uint8_t *base = smem + s * Cfg::kStageBytes;
            const IoT *Bs = reinterpret_cast<const IoT *>(base + 3 * Cfg::kActTile);
            const IoT *Cs = reinterpret_cast<const IoT *>(base + 3 * Cfg::kActTile + Cfg::kBCTile);
            float *dst = bcs_all + s * Cfg::kBCe;
            // unit u = (step t, slot j, half: 0 = B, 1 = C): one slice of NS values
            for (int u = lane; u < nsteps * 2 * G; u += 32) {
                const int t = u / (2 * G), j = (u / 2) % G, half = u & 1;
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
    int64_t d = 0, srow = 0;
    bool dvalid = false, svalid = false;
    float bias = 0.0f, dskip = 0.0f;
    bool ok = true;
    // first tile of a task: its channel, parameters and initial state
    auto setup_task = [&](int64_t b, int c0) {
        d = c0 + c_local;
        dvalid = d < d_inner;
        // row of this sequence's initial / final state (a cache slot, or b)
        srow = b;
        svalid = true;
        if (args.state_indices) {
            srow = __ldg(args.state_indices + b);
            svalid = srow >= 0 && srow < args.num_slots;
            if (srow >= args.num_slots && tid == 0)
                record_status(args.status, kStInvalidArg);
        }
#pragma unroll
        for (int i = 0; i < NS / 2; ++i) {
            const int n = sub * NS + 2 * i;
            a2[i] = dvalid ? make_float2(__ldg(args.A + d * N + n) * kLog2e,
                                         __ldg(args.A + d * N + n + 1) * kLog2e)
                           : make_float2(0.0f, 0.0f);
            h[i] = (dvalid && svalid && args.h0)
                       ? make_float2(__ldg(args.h0 + (srow * d_inner + d) * N + n),
                                     __ldg(args.h0 + (srow * d_inner + d) * N + n + 1))
                       : make_float2(0.0f, 0.0f);
        }
        bias = (dvalid && args.delta_bias) ? __ldg(args.delta_bias + d) : 0.0f;
        dskip = (dvalid && args.D) ? __ldg(args.D + d) : 0.0f;
    };
    for (int64_t g = 0; ok && g < total; ++g) {
        int nsteps = 0;
        bool last_tile = false;
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
        {  // the producer's descriptor of this tile
            const TileHdr t = hdr[s];
            if (t.flags & 1) setup_task(t.b, t.c0);
            nsteps = t.nsteps;
            last_tile = (t.flags & 2) != 0;
        }
        const uint8_t *base = smem + s * Cfg::kStageBytes;
        const IoT *xs = reinterpret_cast<const IoT *>(base);
        const IoT *dts = reinterpret_cast<const IoT *>(base + Cfg::kActTile);
        const IoT *zs = reinterpret_cast<const IoT *>(base + 2 * Cfg::kActTile);
        const float *bcs = bcs_all + s * Cfg::kBCe;
        IoT *outs = reinterpret_cast<IoT *>(smem + Cfg::kOffOut + slot * Cfg::kActTile);

        // One group of G steps starting at t0: the owner lane's scalars, the
        // exchange, G recurrence steps, the butterfly, the owner's output.
        auto group = [&](int t0, int valid) {
            const int t_own = t0 + sub;
            const int idx = t_own * CC + c_local;
            const float xo = to_f32(xs[idx]);
            const float zo = to_f32(zs[idx]);
            const float dl = delta_io<IoT>(to_f32(dts[idx]), bias, use_softplus);
            const float gate = silu_f32(zo);
            const float dx = dl * xo;
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
            const float y = reduce_transpose<G>(yp, sub);
            if (sub < valid) outs[idx] = from_f32<IoT>((y + dskip * xo) * gate);
        };
        if (nsteps == TT && use_softplus) {
            fused_tile_full<true, IoT, N, G, NS, TT, CC, Cfg::kBCRow>(h, a2, bias, dskip, xs, dts, zs,
                                                                     bcs, outs, c_local, sub, gbase);
        } else if (nsteps == TT) {
            fused_tile_full<false, IoT, N, G, NS, TT, CC, Cfg::kBCRow>(h, a2, bias, dskip, xs, dts,
                                                                      zs, bcs, outs, c_local, sub,
                                                                      gbase);
        } else {
            for (int t0 = 0; t0 < nsteps; t0 += G) group(t0, nsteps - t0 < G ? nsteps - t0 : G);
        }
        fence_proxy_async_smem();  // output tile (and this tile's stage reads) before TMA
        mbar_arrive(&out_full[slot]);
        if (last_tile && dvalid && svalid && args.h_final) {
#pragma unroll
            for (int i = 0; i < NS / 2; ++i) {
                float *o = args.h_final + (srow * d_inner + d) * N + sub * NS + 2 * i;
                o[0] = h[i].x;
                o[1] = h[i].y;
            }
        }
    }
    if (!ok) fail();
}

}  // namespace jssm
