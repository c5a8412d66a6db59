// s6_x_proj.cuh -- the first product of the step that feeds the S6 scan:
//     xdbl_t = W_x u_t,  [dt_low_t | B_t | C_t] = xdbl_t   (R, N, N entries)
// with each part RMS-normalised (v <- w * v / sqrt(mean(v^2) + eps)), on the
// sm_100a tensor cores.
//
// Source: "Jamba: A Hybrid Transformer-Mamba Language Model" (obsidian-dorae222
// notes), section "Mamba 레이어": Bbar_t, C_t and Delta_t are functions of x_t,
// and the layer carries an RMSNorm.  The reading taken (Mamba-1's x_proj, with
// an RMSNorm on each of its three outputs) is the one the oracle's `project`
// states.
//
// Outputs: B and C in bf16 in the scan's [token, d_state] layout, and dt_low as
// two bf16 planes hi = bf16(v), lo = bf16(v - hi) for the dt_proj kernel, so
// that no bf16 rounding of dt_low reaches Delta.
//
// Shape handled: R = 256, N = 16 (Jamba), so one CTA's accumulator is 128 tokens
// x 288 fp32 columns of TMEM, filled by two MMAs per K step (N = 256 for dt_low
// and N = 32 for B and C) on one u tile.
//
// Split K.  With 128 tokens per CTA a 4096-token batch has only 32 row tiles, so
// K = d_inner is split across the KS CTAs of a thread-block cluster (KS in
// {1, 2, 4, 8}).  After its MMAs each CTA streams its partial accumulator, row
// by row from TMEM, into the shared memory of the CTA that owns that row's
// reduction (rank = row / (128 / KS)), through distributed shared memory; the
// ring the MMAs used is free by then and holds the receive buffer.  Two cluster
// barriers order this: one after every CTA's MMAs have completed (so no ring is
// still being read), one after every partial has been written.  The owners then
// add the KS partials, normalise, round and store.  No workspace is needed.
//
// Roles (192 threads): warp 0 (one lane) TMA loads, warp 1 TMEM allocation and
// (one lane) the MMAs, warps 2-5 the TMEM read-out and the owners' epilogue.
// Every mbarrier wait is bounded; a wait that runs out records
// JAMBA_SSM_ERR_TIMEOUT and sets the CTA's abort flag.  Before cluster barrier
// 1 the producer waits (bounded) for every load it issued to land and the MMA
// thread for every MMA to complete, so the ring holds no copy in flight when it
// becomes the receive buffer.  An aborted CTA sends no partials, every CTA
// tells every other CTA of the cluster whether it aborted (before barrier 2),
// and owners write no output row when any CTA of their cluster aborted.  Every
// thread reaches both cluster barriers on every path.  Bit 0 of debug_flags
// withholds each CTA's first k-block (a test of the timeout path).
#pragma once

#include "s6_dt_proj.cuh"  // tcgen05 / TMA 2-D helpers and umma_desc_sw128

namespace jssm {

struct XProjCfg {
    static constexpr int kBM = 128;               // tokens per CTA (the MMA's M)
    static constexpr int kR = 256;                // dt_rank
    static constexpr int kN = 16;                 // d_state
    static constexpr int kCols = kR + 2 * kN;     // 288 accumulator columns
    static constexpr int kBK = 64;                // d_inner per stage (128-byte rows)
    static constexpr int kUK = 16;
    static constexpr int kStages = 4;
    static constexpr uint32_t kTileA = kBM * kBK * 2;        // 16 KB of u
    static constexpr uint32_t kTileW1 = kR * kBK * 2;        // 32 KB: W_x rows 0..255
    static constexpr uint32_t kTileW2 = 2 * kN * kBK * 2;    //  4 KB: W_x rows 256..287
    static constexpr uint32_t kStage = kTileA + kTileW1 + kTileW2;  // 52 KB, 1 KB multiple
    static constexpr uint32_t kOffBar = kStages * kStage;
    // full[4], empty[4], acc_full (72 bytes), the TMEM slot (4), the CTA's abort
    // flag (at +80) and the cluster's abort flags (8 words at +96)
    static constexpr uint32_t kOffAbort = kOffBar + 80, kOffAbortAll = kOffBar + 96;
    static constexpr uint32_t kSmemBytes = kOffBar + 128 + 1024;
    // receive buffer (reuses the ring): [KS][128 / KS rows][kRowWords] fp32;
    // 288 columns padded to 292 words so that a warp's 16-byte stores to 8
    // consecutive rows fall in distinct bank groups
    static constexpr int kRowWords = kCols + 4;
    static constexpr uint32_t kRecvBytes = kBM * kRowWords * 4;  // 149.5 KB for every KS
    static constexpr int kThreads = 192;
    static constexpr uint32_t kTmemCols = 512;  // power of two >= 288
    static constexpr uint32_t kIdescDt = (1u << 4) | (1u << 7) | (1u << 10) |
                                         (uint32_t(kR >> 3) << 17) | (uint32_t(kBM >> 4) << 24);
    static constexpr uint32_t kIdescBC = (1u << 4) | (1u << 7) | (1u << 10) |
                                         (uint32_t((2 * kN) >> 3) << 17) |
                                         (uint32_t(kBM >> 4) << 24);
    static_assert(kRecvBytes <= kOffBar, "the receive buffer must fit in the ring");
    static_assert(kStage % 1024 == 0, "stages must keep the 1 KB swizzle alignment");
    static_assert(kCols % 32 == 0, "the read-out takes 32 columns at a time");
};

struct XProjArgs {
    __nv_bfloat16 *dt_hi, *dt_lo, *B, *C;  // outputs
    const float *w_dt, *w_B, *w_C;          // RMSNorm weights or nullptr
    float eps;
    int ntok, d_inner, ks;
    uint64_t limit;
    uint32_t debug_flags;  // bit 0: withhold each CTA's first k-block (tests the timeout path)
};

__device__ __forceinline__ uint32_t cluster_ctarank() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
    return r;
}
__device__ __forceinline__ void cluster_sync_all() {
    asm volatile("barrier.cluster.arrive.release.aligned;\n\t"
                 "barrier.cluster.wait.acquire.aligned;" ::: "memory");
}
// Address in CTA `rank`'s shared memory of the location `saddr` names in ours.
__device__ __forceinline__ uint32_t map_to_rank(uint32_t saddr, uint32_t rank) {
    uint32_t r;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(saddr), "r"(rank));
    return r;
}
__device__ __forceinline__ void st_cluster_u32(uint32_t addr, uint32_t v) {
    asm volatile("st.shared::cluster.u32 [%0], %1;" ::"r"(addr), "r"(v) : "memory");
}
__device__ __forceinline__ void st_cluster_v4(uint32_t addr, float a, float b, float c, float d) {
    asm volatile("st.shared::cluster.v4.f32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "f"(a), "f"(b),
                 "f"(c), "f"(d)
                 : "memory");
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

// Grid: x = KS * token tiles (cluster dims {KS, 1, 1}: one cluster per 128
// tokens, rank = which K slice).
__global__ void __launch_bounds__(XProjCfg::kThreads, 1)
    s6_x_proj_kernel(const __grid_constant__ CUtensorMap map_u,
                     const __grid_constant__ CUtensorMap map_w1,
                     const __grid_constant__ CUtensorMap map_w2, const XProjArgs args) {
    using C = XProjCfg;
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw = smem_u32(smem_raw);
    uint8_t *smem = smem_raw + (((raw + 1023u) & ~1023u) - raw);
    uint64_t *full = reinterpret_cast<uint64_t *>(smem + C::kOffBar);
    uint64_t *empty = full + C::kStages;
    uint64_t *acc_full = empty + C::kStages;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(acc_full + 1);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + C::kOffAbort);
    volatile int *abort_all = reinterpret_cast<volatile int *>(smem + C::kOffAbortAll);
    float *recv = reinterpret_cast<float *>(smem);  // valid after cluster barrier 1

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int ks = args.ks;
    const uint32_t rank = ks > 1 ? cluster_ctarank() : 0u;
    const int m0 = (blockIdx.x / ks) * C::kBM;
    const int kb_total = (args.d_inner + C::kBK - 1) / C::kBK;
    const int per = (kb_total + ks - 1) / ks;
    const int kb0 = min(kb_total, static_cast<int>(rank) * per);
    const int kb1 = min(kb_total, kb0 + per);
    const int nkb = kb1 - kb0;
    auto fail = [&]() {
        if (!*abort_flag) record_status(nullptr, kStTimeout);
        *abort_flag = 1;
    };

    if (threadIdx.x == 0) {
        for (int s = 0; s < C::kStages; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        mbar_init(acc_full, 1);
        *abort_flag = 0;
        fence_mbarrier_init();
        prefetch_tensormap(&map_u);
        prefetch_tensormap(&map_w1);
        prefetch_tensormap(&map_w2);
    }
    if (warp == 1) {
        tmem_alloc(tmem_slot, C::kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *reinterpret_cast<volatile uint32_t *>(tmem_slot);

    if (warp == 0) {
        if (lane == 0) {
            int last_i[C::kStages];  // the last k-block whose loads each stage was armed for
            for (int s = 0; s < C::kStages; ++s) last_i[s] = -1;
            for (int i = 0; i < nkb; ++i) {
                const int s = i % C::kStages;
                if (i >= C::kStages &&
                    !mbar_wait_or_abort(&empty[s], ((i / C::kStages) & 1) ^ 1, args.limit,
                                        abort_flag)) {
                    fail();
                    break;
                }
                if ((args.debug_flags & 1u) && i == 0) continue;  // test hook: withhold k-block 0
                uint8_t *st = smem + s * C::kStage;
                const int k = (kb0 + i) * C::kBK;
                mbar_arrive_expect_tx(&full[s], C::kStage);
                tma_load_2d(st, &map_u, k, m0, &full[s]);
                tma_load_2d(st + C::kTileA, &map_w1, k, 0, &full[s]);
                tma_load_2d(st + C::kTileA + C::kTileW1, &map_w2, k, C::kR, &full[s]);
                last_i[s] = i;
            }
            // The ring becomes the receive buffer after barrier 1: no load may
            // still be landing in it.
            for (int s = 0; s < C::kStages; ++s)
                if (last_i[s] >= 0 &&
                    !mbar_wait_bounded(&full[s], (last_i[s] / C::kStages) & 1, args.limit))
                    fail();
        }
        __syncwarp();
    } else if (warp == 1) {
        if (lane == 0) {
            for (int i = 0; i < nkb; ++i) {
                const int s = i % C::kStages;
                if (!mbar_wait_or_abort(&full[s], (i / C::kStages) & 1, args.limit, abort_flag)) {
                    fail();
                    break;
                }
                tc_fence_after();
                const uint32_t a = smem_u32(smem + s * C::kStage);
#pragma unroll
                for (int k = 0; k < C::kBK / C::kUK; ++k) {
                    const uint32_t koff = k * C::kUK * 2;
                    const uint64_t adesc = umma_desc_sw128(a + koff);
                    const uint32_t acc = (i | k) != 0 ? 1u : 0u;
                    umma_bf16(tmem, adesc, umma_desc_sw128(a + C::kTileA + koff), C::kIdescDt,
                              acc);
                    umma_bf16(tmem + C::kR, adesc,
                              umma_desc_sw128(a + C::kTileA + C::kTileW1 + koff), C::kIdescBC,
                              acc);
                }
                tc_commit(&empty[s]);
            }
            tc_commit(acc_full);
            if (!mbar_wait_bounded(acc_full, 0, args.limit)) fail();
        }
        __syncwarp();
    } else {
        if (!mbar_wait_bounded(acc_full, 0, args.limit)) fail();
        tc_fence_after();
    }

    // Barrier 1: every CTA of the cluster has finished its MMAs and its loads,
    // so every ring may now be overwritten by partial sums.
    tc_fence_before();
    if (ks > 1) cluster_sync_all(); else __syncthreads();
    tc_fence_after();

    const int rows_per_owner = C::kBM / ks;
    const bool aborted = *abort_flag != 0;
    if (threadIdx.x == 0) {  // tell every CTA of the cluster (self included)
        if (ks > 1) {
            const uint32_t slot = smem_u32(const_cast<int *>(abort_all)) + 4u * rank;
            for (int r = 0; r < ks; ++r)
                st_cluster_u32(map_to_rank(slot, static_cast<uint32_t>(r)), aborted ? 1u : 0u);
        } else {
            abort_all[0] = aborted ? 1 : 0;
        }
    }
    if (warp >= 2 && !aborted) {
        // Each thread sends its token row's 288 partial sums to the row's owner.
        const int q = warp & 3;
        const int row = q * 32 + lane;
        const uint32_t owner = static_cast<uint32_t>(row / rows_per_owner);
        const uint32_t local = smem_u32(recv) +
                               4u * static_cast<uint32_t>((rank * rows_per_owner +
                                                           row % rows_per_owner) * C::kRowWords);
        const uint32_t dst = ks > 1 ? map_to_rank(local, owner) : local;
        // 16 columns at a time; the next group's TMEM load is in flight while
        // this group is sent
        const uint32_t trow = tmem + ((uint32_t)(q * 32) << 16);
        uint32_t va[16], vb[16];
        auto send = [&](int c, const uint32_t (&v)[16]) {
#pragma unroll
            for (int j = 0; j < 16; j += 4) {
                float f[4];
#pragma unroll
                for (int e = 0; e < 4; ++e)  // an empty K slice never wrote the accumulator
                    f[e] = nkb == 0 ? 0.0f : __uint_as_float(v[j + e]);
                st_cluster_v4(dst + 4u * (c + j), f[0], f[1], f[2], f[3]);
            }
        };
        tmem_ld16_async(trow, va);
        tmem_wait_ld();
        tmem_regs_ready(va);
        static_assert(C::kCols % 32 == 0, "pairs of 16-column groups");
#pragma unroll 1
        for (int c = 0; c < C::kCols; c += 32) {
            tmem_ld16_async(trow + (uint32_t)(c + 16), vb);
            send(c, va);
            tmem_wait_ld();
            tmem_regs_ready(vb);
            if (c + 32 < C::kCols) tmem_ld16_async(trow + (uint32_t)(c + 32), va);
            send(c + 16, vb);
            tmem_wait_ld();
            tmem_regs_ready(va);
        }
    }
    tc_fence_before();
    // Barrier 2: every partial (and every CTA's abort flag) has landed.
    if (ks > 1) cluster_sync_all(); else __syncthreads();
    bool cluster_aborted = false;
    for (int r = 0; r < ks; ++r) cluster_aborted |= abort_all[r] != 0;

    if (!cluster_aborted) {
        // Owner epilogue, all six warps: warp w takes rows w, w + 6, ... of this
        // CTA's share; lane j holds columns j + 32 k (k = 0..7: dt_low; k = 8:
        // B for j < 16, C for j >= 16).
        const bool is_b = lane < 16;
        const float *w8 = is_b ? args.w_B : args.w_C;
        for (int r = warp; r < rows_per_owner; r += C::kThreads / 32) {
            const int m = m0 + static_cast<int>(rank) * rows_per_owner + r;
            float v[9];
#pragma unroll
            for (int k = 0; k < 9; ++k) v[k] = 0.0f;
            for (int src = 0; src < ks; ++src) {
                const float *p = recv + (src * rows_per_owner + r) * C::kRowWords;
#pragma unroll
                for (int k = 0; k < 9; ++k) v[k] += p[lane + 32 * k];
            }
            if (args.w_dt) {
                float ss = 0.0f;
#pragma unroll
                for (int k = 0; k < 8; ++k) ss += v[k] * v[k];
                const float inv = rsqrtf(warp_sum(ss) * (1.0f / C::kR) + args.eps);
#pragma unroll
                for (int k = 0; k < 8; ++k) v[k] = args.w_dt[lane + 32 * k] * (v[k] * inv);
            }
            const float sq = v[8] * v[8];
            const float ss_b = warp_sum(is_b ? sq : 0.0f), ss_c = warp_sum(is_b ? 0.0f : sq);
            if (w8) {
                const float inv = rsqrtf((is_b ? ss_b : ss_c) * (1.0f / C::kN) + args.eps);
                v[8] = w8[lane & 15] * (v[8] * inv);
            }
            if (m < args.ntok) {
                __nv_bfloat16 *hi = args.dt_hi + static_cast<size_t>(m) * C::kR;
                __nv_bfloat16 *lo = args.dt_lo + static_cast<size_t>(m) * C::kR;
#pragma unroll
                for (int k = 0; k < 8; ++k) {
                    const __nv_bfloat16 h = __float2bfloat16_rn(v[k]);
                    hi[lane + 32 * k] = h;
                    lo[lane + 32 * k] = __float2bfloat16_rn(v[k] - __bfloat162float(h));
                }
                __nv_bfloat16 *bc = (is_b ? args.B : args.C) + static_cast<size_t>(m) * C::kN;
                bc[lane & 15] = __float2bfloat16_rn(v[8]);
            }
        }
    }
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, C::kTmemCols);
    }
}

}  // namespace jssm
