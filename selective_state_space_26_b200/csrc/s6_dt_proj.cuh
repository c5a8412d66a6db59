// s6_dt_proj.cuh -- the low-rank step that produces the scan's raw Delta:
//     delta[t, d] = sum_r W_dt[d, r] * dt_low[t, r]
// on the sm_100a tensor cores (tcgen05.mma, accumulator in TMEM).
//
// Source: "Jamba: A Hybrid Transformer-Mamba Language Model" (obsidian-dorae222
// notes), section "Mamba 레이어": Bbar_t, C_t and Delta_t are functions of x_t.
// The pages do not spell the function out; the reading taken is Mamba-1's,
// where Delta comes from a rank-R vector dt_low_t (R = dt_rank) through one
// linear map W_dt [d_inner, R].  The per-channel bias and the softplus are the
// scan's own first step and are not applied here.
//
// Precision.  dt_low is an fp32 quantity (it leaves an RMSNorm).  Rounding it
// to bf16 before this product would add ~1.6e-3 relative error to Delta, more
// than the layer's bf16 tolerance leaves room for, so it arrives as two bf16
// planes, hi = bf16(v) and lo = bf16(v - hi), and every k-step issues two MMAs
// (hi and lo against the same W_dt tile) into one fp32 accumulator.  With lo
// absent (NULL) only the hi plane is used.
//
// Work unit and roles.  One CTA computes a 128-token x 128-channel tile of
// delta; K = dt_rank runs in 64-wide blocks through a 2-stage ring.  A CTA
// takes 97 KB of shared memory and 128 TMEM columns, so two run on each SM and
// one's loads and epilogue overlap the other's MMAs.
//   warp 0 (one lane): TMA loads of the hi / lo / W_dt tiles (128-byte swizzle);
//   warp 1: allocates 128 TMEM columns; one lane issues the MMAs
//           (M = 128, N = 128, K = 16, bf16 x bf16 -> fp32) and commits each
//           stage back to the producer, then the finished accumulator;
//   warps 2-5: epilogue -- each thread owns one token row (TMEM lane), reads
//           its 128 fp32 columns with tcgen05.ld, rounds them to bf16 into a
//           staged copy of the output tile in shared memory (the operand ring,
//           free once every MMA has completed), laid out as two 64-column
//           slabs with the 128-byte swizzle so that the 32 rows a warp writes
//           at once fall in distinct banks; one thread then writes the tile
//           with two TMA stores, which clip it to [ntok, d_inner].
// Every wait is bounded; a wait that runs out records JAMBA_SSM_ERR_TIMEOUT in
// the module's status word and sets a CTA abort flag.  The CTA then winds down
// in order: the producer waits (bounded) for every TMA load it issued to land,
// the MMA thread for every MMA it issued to complete, and only then -- past a
// CTA barrier, and only if nothing aborted -- is the accumulator read out; the
// TMEM is freed last.  Bit 0 of debug_flags withholds the first k-block's
// loads so that the MMA thread's wait runs out (a test of this path).
#pragma once

#include "device_utils.cuh"
#include "tcgen05_utils.cuh"

namespace jssm {

struct DtProjCfg {
    static constexpr int kBM = 128;  // tokens per tile: the MMA's M (one TMEM lane each)
    static constexpr int kBN = 128;  // channels per tile: the MMA's N (one TMEM column each)
    static constexpr int kBK = 64;   // dt_rank per stage: one 128-byte swizzled bf16 row
    static constexpr int kUK = 16;   // K of one kind::f16 MMA
    static constexpr int kStages = 2;
    static constexpr uint32_t kTileA = kBM * kBK * 2;        // 16 KB per plane
    static constexpr uint32_t kTileW = kBN * kBK * 2;        // 16 KB
    static constexpr uint32_t kStage = 2 * kTileA + kTileW;  // 48 KB
    static constexpr uint32_t kOffBar = kStages * kStage;    // barriers after the tiles
    // full[2], empty[2], acc_full (40 bytes), the TMEM slot, the abort flag
    static constexpr uint32_t kSmemBytes = kOffBar + 64 + 1024;  // + room to align to 1 KB
    static constexpr int kThreads = 192;
    static constexpr uint32_t kTmemCols = kBN;
    static_assert(kStage % 1024 == 0, "stages keep the 1 KB swizzle alignment");
    static_assert(kBM * kBN * 2 <= kStage, "the staged output tile fits in ring stage 0");
    // Instruction descriptor of kind::f16: fp32 accumulator (bits 4-5 = 1),
    // A and B bf16 (bits 7-9 and 10-12 = 1), both K-major (bits 15, 16 = 0),
    // N >> 3 in bits 17-22, M >> 4 in bits 24-28.
    static constexpr uint32_t kIdesc = (1u << 4) | (1u << 7) | (1u << 10) |
                                       (uint32_t(kBN >> 3) << 17) | (uint32_t(kBM >> 4) << 24);
};

// ------------------------------------------------------------------- kernel
// Grid: x = token tiles of 128, y = channel tiles of 128.  delta is written
// only inside [ntok, d_inner] (the TMA stores clip the tile); TMA fills
// out-of-range operand rows and K columns with zeros, so ragged edges need no
// special case in the MMAs.
__global__ void __launch_bounds__(DtProjCfg::kThreads, 2)
    s6_dt_proj_kernel(const __grid_constant__ CUtensorMap map_hi,
                      const __grid_constant__ CUtensorMap map_lo,
                      const __grid_constant__ CUtensorMap map_w,
                      const __grid_constant__ CUtensorMap map_out, int dt_rank, int two_planes,
                      uint64_t limit, uint32_t debug_flags) {
    using C = DtProjCfg;
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw = smem_u32(smem_raw);
    uint8_t *smem = smem_raw + (((raw + 1023u) & ~1023u) - raw);
    uint64_t *full = reinterpret_cast<uint64_t *>(smem + C::kOffBar);
    uint64_t *empty = full + C::kStages;
    uint64_t *acc_full = empty + C::kStages;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(acc_full + 1);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int m0 = blockIdx.x * C::kBM, n0 = blockIdx.y * C::kBN;
    const int kblocks = (dt_rank + C::kBK - 1) / C::kBK;
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
        prefetch_tensormap(&map_hi);
        prefetch_tensormap(&map_lo);
        prefetch_tensormap(&map_w);
        prefetch_tensormap(&map_out);
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
            const uint32_t bytes = (two_planes ? 2u : 1u) * C::kTileA + C::kTileW;
            int last_kb[C::kStages];  // the last k-block whose loads each stage was armed for
            for (int s = 0; s < C::kStages; ++s) last_kb[s] = -1;
            for (int kb = 0; kb < kblocks; ++kb) {
                const int s = kb % C::kStages;
                if (kb >= C::kStages &&
                    !mbar_wait_or_abort(&empty[s], ((kb / C::kStages) & 1) ^ 1, limit, abort_flag)) {
                    fail();
                    break;
                }
                if ((debug_flags & 1u) && kb == 0) continue;  // test hook: withhold k-block 0
                uint8_t *st = smem + s * C::kStage;
                mbar_arrive_expect_tx(&full[s], bytes);
                tma_load_2d(st, &map_hi, kb * C::kBK, m0, &full[s]);
                if (two_planes) tma_load_2d(st + C::kTileA, &map_lo, kb * C::kBK, m0, &full[s]);
                tma_load_2d(st + 2 * C::kTileA, &map_w, kb * C::kBK, n0, &full[s]);
                last_kb[s] = kb;
            }
            // No load may still be landing in the ring when the CTA moves on.
            for (int s = 0; s < C::kStages; ++s)
                if (last_kb[s] >= 0 &&
                    !mbar_wait_bounded(&full[s], (last_kb[s] / C::kStages) & 1, limit))
                    fail();
        }
        __syncwarp();
    } else if (warp == 1) {
        if (lane == 0) {
            for (int kb = 0; kb < kblocks; ++kb) {
                const int s = kb % C::kStages;
                if (!mbar_wait_or_abort(&full[s], (kb / C::kStages) & 1, limit, abort_flag)) {
                    fail();
                    break;
                }
                tc_fence_after();
                const uint32_t a = smem_u32(smem + s * C::kStage);
#pragma unroll
                for (int k = 0; k < C::kBK / C::kUK; ++k) {
                    const uint32_t koff = k * C::kUK * 2;  // bytes along the 128-byte row
                    const uint64_t bdesc = umma_desc_sw128(a + 2 * C::kTileA + koff);
                    umma_bf16(tmem, umma_desc_sw128(a + koff), bdesc, C::kIdesc,
                              (kb | k) != 0 ? 1u : 0u);
                    if (two_planes)
                        umma_bf16(tmem, umma_desc_sw128(a + C::kTileA + koff), bdesc, C::kIdesc,
                                  1u);
                }
                tc_commit(&empty[s]);  // the stage is free once these MMAs have read it
            }
            tc_commit(acc_full);  // every MMA issued above has completed
            // Do not leave (and let the accumulator be freed) while MMAs run.
            if (!mbar_wait_bounded(acc_full, 0, limit)) fail();
        }
        __syncwarp();
    }
    // Every load has landed and every MMA has completed (or the CTA aborted).
    tc_fence_before();
    __syncthreads();
    if (warp >= 2) {
        // Epilogue: warp w may read TMEM lanes 32*(w%4) .. 32*(w%4)+31.
        const int q = warp & 3;
        const int r = q * 32 + lane;  // this thread's token row of the tile
        const bool ok = !*abort_flag && mbar_wait_bounded(acc_full, 0, limit);
        tc_fence_after();
        if (ok) {
            // The bf16 tile as 4 slabs of [128 rows][64 columns] (16 KB each)
            // in ring stage 0: 16-byte chunk j of row r at r * 128 + ((j ^ (r
            // % 8)) * 16), the TMA 128-byte swizzle.
            const uint32_t stage = smem_u32(smem);
#pragma unroll 1
            for (int c = 0; c < C::kBN; c += 32) {
                float v[32];
                tmem_ld32(tmem + ((uint32_t)(q * 32) << 16) + (uint32_t)c, v);
                const uint32_t slab = stage + (uint32_t)(c / 64) * (C::kBM * 128u) + r * 128u;
#pragma unroll
                for (int g = 0; g < 4; ++g) {
                    const uint32_t j = (uint32_t)((c % 64) / 8 + g);
                    uint4 o;
                    o.x = pack_bf16x2(v[8 * g + 0], v[8 * g + 1]);
                    o.y = pack_bf16x2(v[8 * g + 2], v[8 * g + 3]);
                    o.z = pack_bf16x2(v[8 * g + 4], v[8 * g + 5]);
                    o.w = pack_bf16x2(v[8 * g + 6], v[8 * g + 7]);
                    st_shared_v4(slab + ((j ^ (uint32_t)(r & 7)) * 16u), o);
                }
            }
            fence_proxy_async_smem();  // the staged tile, before the TMA engine reads it
        }
        epilogue_sync(128);
        if (ok && warp == 2 && lane == 0) {
#pragma unroll
            for (int s = 0; s < C::kBN / 64; ++s)
                tma_store_2d(&map_out, smem + s * (C::kBM * 128), n0 + 64 * s, m0);
            bulk_commit();
            bulk_wait<0>();  // the stores are done before the CTA (and its smem) goes
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, C::kTmemCols);
    }
}

// ===================================================== persistent form
// For dt_rank <= 256 (Jamba's 256 included): one CTA per SM walks a
// contiguous range of (token block, 256-channel tile) items.  An MMA of
// 128 x 256 x 16 reads 12 KB of operands from shared memory per 136 tensor
// cycles, against 8 KB per 68 cycles for N = 128, which is the SM's whole
// shared-memory bandwidth; so this form takes N = 256.  Per k-block a stage of
// the 3-stage ring holds the hi and lo planes (16 KB each) and 256 rows of W_dt
// (32 KB).  Two TMEM accumulators of 256 columns alternate between items, so
// the epilogue of item j (TMEM read-out, bf16 rounding, TMA store of two
// 128-column halves through a 32 KB staging buffer) overlaps the MMAs of item
// j + 1.
//   warp 0 (one lane): TMA loads;
//   warp 1: allocates 512 TMEM columns; one lane issues the MMAs of item j
//           into accumulator j % 2 once the epilogue has drained it, commits
//           each ring stage back to the producer and the finished
//           accumulator to the epilogue;
//   warps 2-5: the epilogue, each thread one token row (TMEM lane).
// Every wait is bounded.  The epilogue warps decide together whether to go on
// (a barrier reduction of their wait outcomes), so an abort cannot split them
// at a named barrier; the producer waits (bounded) for every load it issued
// and the MMA thread for its last MMAs before the CTA frees TMEM.  Bit 0 of
// debug_flags withholds the first k-block (a test of the timeout path).
struct DtProjPCfg {
    static constexpr int kBM = 128, kBN = 256, kBK = 64, kUK = 16;
    static constexpr int kMaxKB = 4;  // dt_rank <= 256 (the persistent kernel's range)
    static constexpr int kStages = 3;
    static constexpr uint32_t kTileA = kBM * kBK * 2;       // 16 KB per plane
    static constexpr uint32_t kTileW = kBN * kBK * 2;       // 32 KB: two boxes of 128 rows
    static constexpr uint32_t kStage = 2 * kTileA + kTileW;  // 64 KB
    static constexpr uint32_t kOffOut = kStages * kStage;
    static constexpr uint32_t kHalf = kBM * 128 * 2;        // 32 KB: 128 columns, two slabs
    static constexpr uint32_t kOffBar = kOffOut + kHalf;
    // full[3], empty[3], acc_full[2], acc_empty[2], drain, TMEM slot, abort flag
    static constexpr uint32_t kSmemBytes = kOffBar + 128 + 1024;  // + room to align to 1 KB
    static constexpr int kThreads = 192;
    static constexpr uint32_t kTmemCols = 2 * kBN;  // 512: two accumulators
    static_assert(kStage % 1024 == 0, "stages keep the 1 KB swizzle alignment");
    // kind::f16: fp32 accumulator, A and B bf16, both K-major, N >> 3, M >> 4.
    static constexpr uint32_t kIdesc = (1u << 4) | (1u << 7) | (1u << 10) |
                                       (uint32_t(kBN >> 3) << 17) | (uint32_t(kBM >> 4) << 24);
};

__global__ void __launch_bounds__(DtProjPCfg::kThreads, 1)
    s6_dt_proj_persistent_kernel(const __grid_constant__ CUtensorMap map_hi,
                                 const __grid_constant__ CUtensorMap map_lo,
                                 const __grid_constant__ CUtensorMap map_w,
                                 const __grid_constant__ CUtensorMap map_out, int ntok,
                                 int d_inner, int dt_rank, int two_planes, uint64_t limit,
                                 uint32_t debug_flags) {
    using C = DtProjPCfg;
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw = smem_u32(smem_raw);
    uint8_t *smem = smem_raw + (((raw + 1023u) & ~1023u) - raw);
    uint64_t *full = reinterpret_cast<uint64_t *>(smem + C::kOffBar);
    uint64_t *empty = full + C::kStages;
    uint64_t *acc_full = empty + C::kStages;
    uint64_t *acc_empty = acc_full + 2;
    uint64_t *drain = acc_empty + 2;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(drain + 1);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int kblocks = (dt_rank + C::kBK - 1) / C::kBK;  // <= kMaxKB (checked by the host)
    const int ntn = (d_inner + C::kBN - 1) / C::kBN;
    const int64_t items = int64_t((ntok + C::kBM - 1) / C::kBM) * ntn;
    const int64_t lo_item = items * blockIdx.x / gridDim.x;
    const int cnt = static_cast<int>(items * (blockIdx.x + 1) / gridDim.x - lo_item);
    auto fail = [&]() {
        if (!*abort_flag) record_status(nullptr, kStTimeout);
        *abort_flag = 1;
    };

    if (threadIdx.x == 0) {
        for (int s = 0; s < C::kStages; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&acc_full[b], 1);
            mbar_init(&acc_empty[b], 128);
        }
        mbar_init(drain, 1);
        *abort_flag = 0;
        fence_mbarrier_init();
        prefetch_tensormap(&map_hi);
        prefetch_tensormap(&map_lo);
        prefetch_tensormap(&map_w);
        prefetch_tensormap(&map_out);
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
            const uint32_t bytes = (two_planes ? 2u : 1u) * C::kTileA + C::kTileW;
            int last[C::kStages];  // the last load issued into each stage, or -1
            for (int s = 0; s < C::kStages; ++s) last[s] = -1;
            int wi = 0;
            bool ok = true;
            for (int j = 0; j < cnt && ok; ++j) {
                const int64_t it = lo_item + j;
                const int m0 = static_cast<int>(it / ntn) * C::kBM;
                const int n0 = static_cast<int>(it % ntn) * C::kBN;
                for (int kb = 0; kb < kblocks; ++kb, ++wi) {
                    const int s = wi % C::kStages;
                    if (wi >= C::kStages &&
                        !mbar_wait_or_abort(&empty[s], ((wi / C::kStages) & 1) ^ 1, limit,
                                            abort_flag)) {
                        ok = false;
                        break;
                    }
                    if ((debug_flags & 1u) && wi == 0) continue;  // test hook: withhold k-block 0
                    uint8_t *st = smem + s * C::kStage;
                    mbar_arrive_expect_tx(&full[s], bytes);
                    tma_load_2d(st, &map_hi, kb * C::kBK, m0, &full[s]);
                    if (two_planes) tma_load_2d(st + C::kTileA, &map_lo, kb * C::kBK, m0, &full[s]);
                    tma_load_2d(st + 2 * C::kTileA, &map_w, kb * C::kBK, n0, &full[s]);
                    tma_load_2d(st + 2 * C::kTileA + C::kTileW / 2, &map_w, kb * C::kBK, n0 + 128,
                                &full[s]);
                    last[s] = wi;
                }
            }
            if (!ok) fail();
            // No load may still be landing when the CTA moves on.
            for (int s = 0; s < C::kStages; ++s)
                if (last[s] >= 0 && !mbar_wait_bounded(&full[s], (last[s] / C::kStages) & 1, limit))
                    fail();
        }
        __syncwarp();
    } else if (warp == 1) {
        if (lane == 0) {
            int wi = 0;
            bool ok = true;
            for (int j = 0; j < cnt && ok; ++j) {
                const int buf = j & 1;
                // accumulator `buf` was last drained by the epilogue of item j - 2
                if (j >= 2 &&
                    !mbar_wait_or_abort(&acc_empty[buf], ((j / 2) - 1) & 1, limit, abort_flag)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint32_t d = tmem + uint32_t(buf) * C::kBN;
                for (int kb = 0; kb < kblocks; ++kb, ++wi) {
                    const int s = wi % C::kStages;
                    if (!mbar_wait_or_abort(&full[s], (wi / C::kStages) & 1, limit, abort_flag)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t a = smem_u32(smem + s * C::kStage);
#pragma unroll
                    for (int k = 0; k < C::kBK / C::kUK; ++k) {
                        const uint32_t koff = k * C::kUK * 2;  // bytes along the 128-byte row
                        const uint64_t bdesc = umma_desc_sw128(a + 2 * C::kTileA + koff);
                        umma_bf16(d, umma_desc_sw128(a + koff), bdesc, C::kIdesc,
                                  (kb | k) != 0 ? 1u : 0u);
                        if (two_planes)
                            umma_bf16(d, umma_desc_sw128(a + C::kTileA + koff), bdesc, C::kIdesc,
                                      1u);
                    }
                    tc_commit(&empty[s]);  // the stage is free once these MMAs have read it
                }
                if (!ok) break;
                tc_commit(&acc_full[buf]);  // item j's accumulator is complete
            }
            if (!ok) fail();
            // Do not let TMEM be freed while MMAs run: this commit arrives once
            // every MMA issued above (an aborted item's included) has completed.
            tc_commit(drain);
            if (!mbar_wait_bounded(drain, 0, limit)) fail();
        }
        __syncwarp();
    } else {
        // Epilogue: warp w may read TMEM lanes 32*(w%4) .. 32*(w%4)+31.
        const int q = warp & 3;
        const int r = q * 32 + lane;  // this thread's token row of the tile
        const bool storer = warp == 2 && lane == 0;
        const uint32_t stage = smem_u32(smem + C::kOffOut);
        for (int j = 0; j < cnt; ++j) {
            const int64_t it = lo_item + j;
            const int m0 = static_cast<int>(it / ntn) * C::kBM;
            const int n0 = static_cast<int>(it % ntn) * C::kBN;
            const int buf = j & 1;
            const bool got = mbar_wait_or_abort(&acc_full[buf], (j / 2) & 1, limit, abort_flag);
            if (!got) fail();
            if (storer) bulk_wait_read<0>();  // the previous store has read the staging buffer
            if (!epilogue_all(got, 128)) break;
            tc_fence_after();
#pragma unroll 1
            for (int h = 0; h < 2; ++h) {  // two halves of 128 columns through one buffer
                if (h == 1) {
                    if (storer) bulk_wait_read<0>();
                    epilogue_sync(128);
                }
                // The bf16 half as 2 slabs of [128 rows][64 columns]: 16-byte
                // chunk c of row r at r * 128 + ((c ^ (r % 8)) * 16), the TMA
                // 128-byte swizzle, so the 32 rows a warp writes at once fall in
                // distinct banks.
#pragma unroll 1
                for (int c = 0; c < 128; c += 32) {
                    float v[32];
                    tmem_ld32(tmem + (uint32_t(q * 32) << 16) + uint32_t(buf) * C::kBN +
                                  uint32_t(h * 128 + c),
                              v);
                    const uint32_t slab = stage + uint32_t(c / 64) * (C::kBM * 128u) + r * 128u;
#pragma unroll
                    for (int g = 0; g < 4; ++g) {
                        const uint32_t ch = uint32_t((c % 64) / 8 + g);
                        uint4 o;
                        o.x = pack_bf16x2(v[8 * g + 0], v[8 * g + 1]);
                        o.y = pack_bf16x2(v[8 * g + 2], v[8 * g + 3]);
                        o.z = pack_bf16x2(v[8 * g + 4], v[8 * g + 5]);
                        o.w = pack_bf16x2(v[8 * g + 6], v[8 * g + 7]);
                        st_shared_v4(slab + ((ch ^ uint32_t(r & 7)) * 16u), o);
                    }
                }
                if (h == 1) {
                    tc_fence_before();
                    mbar_arrive(&acc_empty[buf]);  // the accumulator may take item j + 2
                }
                fence_proxy_async_smem();  // the staged half, before the TMA engine reads it
                epilogue_sync(128);
                if (storer) {
                    tma_store_2d(&map_out, smem + C::kOffOut, n0 + h * 128, m0);
                    tma_store_2d(&map_out, smem + C::kOffOut + C::kBM * 128, n0 + h * 128 + 64, m0);
                    bulk_commit();
                }
            }
        }
        if (storer) bulk_wait<0>();  // the stores are done before the CTA (and its smem) goes
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, C::kTmemCols);
    }
}

}  // namespace jssm
