// s6_ssd_chunk.cuh -- the scalar-identity scan (Mamba-2's state matrix) in its
// chunked matrix form, on the sm_100a tensor cores.
//
// Source: "Jamba -- Hybrid SSM-Transformer" (factory.pai-world.com lesson),
// section "Mamba-3: 2026년의 순수 SSM 기준선", items 1 and 2 (the state matrix is
// a scaled identity, Euler-discretised); the per-step map is the one s6_ssd.cuh
// computes: per head one step size Delta_t and one decay e^{Delta_t A}.
//
// Chunked form.  Take a chunk of Q = 128 tokens of one head (local index t)
// and, inside it, the inclusive sums s_t = A * sum_{tau <= t} Delta_tau.  The
// product of the decays from token j + 1 to t is e^{s_t - s_j}, so unrolling
// the recurrence from the chunk's incoming state h_in gives
//     h_t = e^{s_t} h_in + sum_{j <= t} e^{s_t - s_j} Delta_j B_j x_j^T
// and therefore
//     y_t     = sum_j M[t, j] x_j + e^{s_t} (C_t . h_in) + D x_t,
//     M[t, j] = (C_t . B_j) e^{s_t - s_j} Delta_j      (j <= t; 0 above),
//     h_out   = e^{s_127} h_in + sum_j W[:, j] x_j^T,   W[n, j] = e^{s_127 - s_j} Delta_j B_j[n],
//     out_t   = y_t silu(z_t).
// This is the per-step map with its products of exponentials gathered (they
// are exponentials of sums); only the fp32 rounding order differs.
//
// Contractions and their tensor-core form (kind::f16, bf16 operands, fp32
// accumulators in TMEM; M = 128 rows):
//   CB  = C . B^T        [128 x 128], K = d_state 16: C and B straight from TMA
//                        (rows of 32 bytes, 32-byte swizzle, K-major).
//   Y   = M . X          [128 x 64],  K = 128 tokens: M is built by the math
//                        warps from CB; X is the TMA tile [tokens][64 channels]
//                        as an MN-major operand.
//   DS  = W . X          [16 x 64],   K = 128: W has 16 rows; the MMA runs with
//                        M = 128 and the 112 rows past them are don't-care
//                        (their descriptor reads run on into the M buffer).
//   YI  = C . h_in       [128 x 64],  K = 16: h_in (fp32, kept by the state
//                        warp) as an MN-major operand.
// sigma_t = s_t log2(e) is kept as an unevaluated pair hi + lo (a compensated
// prefix sum): within a chunk |sigma| reaches thousands when the decay is
// strong, and the exponents sigma_t - sigma_j of nearby tokens, which carry the
// weight, would otherwise lose ~ulp(|sigma|) to cancellation; as
// (hi_t - hi_j) + (lo_t - lo_j) they keep fp32 accuracy of the difference.
//
// M, W and h_in are fp32 quantities; each is passed as two bf16 planes,
// hi = bf16(v) and lo = bf16(v - hi), and each product is issued once per plane
// into the same accumulator, which keeps them to ~2^-17 relative (a single bf16
// rounding, 2^-9, would exceed the layer's bf16 parity bound).
//
// One CTA per (sequence, 64-channel slice of a head) walks the sequence's chunks
// in order; a head wider than 64 channels takes several CTAs, each repeating the
// head's per-token work (Delta, sigma, M, W).  Warps:
//   0     the state warp: lanes n < 16 keep h[n][0..63] in fp32 registers; per
//         chunk h = e^{s_127} h + DS (DS read from TMEM lanes 0-15), then h as
//         hi / lo planes into the buffer the next chunk's YI reads; h_final.
//   1     producer: lane 0 feeds a 3-stage ring by TMA (x, z [128 x 64], C, B
//         [128 x 16]); all lanes then compute the chunk's Delta_t (from plain
//         loads of delta, one chunk ahead; softplus, bias; zero past the
//         sequence's end) and sigma_t = s_t log2(e) (a compensated warp prefix
//         sum), as soon as the chunk lands.
//   2     allocates TMEM (CB 128 columns, Y and YI two buffers of 64 each, DS
//         64) and one lane issues the MMAs, in the order
//         [Y_c] -> [CB_{c+1}] -> [DS_c] -> [YI_c, once h_{c-1} is there], so
//         that the M buffer and CB are handed back to the math warps early.
//   3-10  math warps, two groups of four (one per TMEM lane quarter), each
//         thread one token row: build M_c (the group's half of the 16-column
//         blocks, blocks above the diagonal are zeros; the exponent as
//         (sigma_t - sigma_ref) + delta_j, the first term once per block and
//         delta_j = sigma_ref - sigma_j from the producer's table, ref the
//         block's first token, or with softplus its last, j1; with softplus a
//         block below the diagonal for all the warp's rows takes one exp,
//         e^{s_t - s_j1}, times the table's e^{s_j1 - s_j} Delta_j, both at
//         most 1 or Delta_j); the warps of lane quarters 0 and 1, whose share of
//         M is the smallest, also write W_c into the stage (one token each);
//         then the epilogue of chunk c - 1: Y + e^{s_t} YI + D x, times silu(z),
//         rounded to bf16 and stored to global memory (64 bytes per thread and
//         chunk half).
// Every wait is bounded and watches the CTA's abort flag; a wait that runs out
// records JAMBA_SSM_ERR_TIMEOUT.  Before the CTA frees TMEM the producer waits
// (bounded) for the loads it issued and the MMA lane for the MMAs it issued.
// Bit 0 of debug_flags withholds the first chunk's loads (a test of that path).
#pragma once

#include "device_utils.cuh"
#include "s6_math.cuh"
#include "s6_scan.cuh"
#include "tcgen05_utils.cuh"

namespace jssm {

struct SsdChunkCfg {
    static constexpr int Q = 128;  // tokens per chunk: the MMAs' M, one TMEM lane each
    static constexpr int P = 64;   // channels per head: the MMAs' N
    static constexpr int N = 16;   // d_state
    static constexpr int STAGES = 3;
    // one ring stage
    static constexpr uint32_t kX = 0;              // x [128][64] bf16, 128-byte swizzle
    static constexpr uint32_t kZ = 16384;          // z, the same
    static constexpr uint32_t kC = 32768;          // C [128][16] bf16, 32-byte swizzle
    static constexpr uint32_t kB = 36864;          // B, the same
    static constexpr uint32_t kDel = 40960;        // Delta_t (softplus: e^{s_j1 - s_t} Delta_t) fp32 [128]
    static constexpr uint32_t kSig = kDel + 512;   // sigma_t as hi [128] and lo [128] fp32
    // delta_t = sigma_ref - sigma_t, ref the first token of t's 16-token block
    // (with softplus: its last, + log2 Delta_t) fp32 [128]
    static constexpr uint32_t kDlt = kSig + 1024;
    // W: per plane two K atoms (tokens 0-63, 64-127) of 16 rows x 128 bytes
    static constexpr uint32_t kW = 43008;
    static constexpr uint32_t kWPlane = 4096;
    static constexpr uint32_t kStage = kW + 2 * kWPlane;  // 50 KB
    static constexpr uint32_t kLoadBytes = 2 * 16384 + 2 * 4096;
    // M: per plane two K atoms of 128 rows x 128 bytes
    static constexpr uint32_t kOffM = STAGES * kStage;
    static constexpr uint32_t kMPlane = 32768;
    // h_in operand: two buffers x (hi, lo) of 16 rows x 128 bytes
    static constexpr uint32_t kOffH = kOffM + 2 * kMPlane;
    static constexpr uint32_t kHPlane = 2048;
    static constexpr uint32_t kOffD = kOffH + 4 * kHPlane;  // D of the head's channels, fp32 [64]
    static constexpr uint32_t kOffBar = kOffD + 256;
    static constexpr int kNumBars = 3 * STAGES + 12;
    static constexpr uint32_t kOffSlot = kOffBar + kNumBars * 8;
    static constexpr uint32_t kSmemBytes = kOffSlot + 16 + 1024;  // + room to align to 1 KB
    static constexpr int kThreads = 352;
    static constexpr uint32_t kTmemCols = 512;
    static constexpr uint32_t kColCB = 0, kColY = 128, kColYI = 256, kColDS = 384;
    static_assert(kStage % 1024 == 0 && kW % 1024 == 0 && kOffM % 1024 == 0 &&
                      kOffH % 1024 == 0,
                  "swizzled operands keep their 1 KB alignment");
    static_assert(kDlt + 512 <= kW, "the stage holds its tables");
    // W's descriptor reads 128 rows (16 KB) from each K atom's start: they must
    // stay inside the buffers that follow it (the next stage, or M).
    static_assert((STAGES - 1) * kStage + kW + kWPlane + kWPlane / 2 + 16384 + 128 <= kOffH,
                  "W's don't-care rows");
    static_assert(kSmemBytes <= 232448, "fits the opt-in shared memory of one CTA");
    // kind::f16, fp32 accumulator, A and B bf16, M = 128: N = 128 with both
    // operands K-major (C . B^T); N = 64 with B MN-major (bit 16) for the rest.
    static constexpr uint32_t kIdescCB =
        (1u << 4) | (1u << 7) | (1u << 10) | (uint32_t(128 >> 3) << 17) | (uint32_t(128 >> 4) << 24);
    static constexpr uint32_t kIdescX = (1u << 4) | (1u << 7) | (1u << 10) | (1u << 16) |
                                        (uint32_t(64 >> 3) << 17) | (uint32_t(128 >> 4) << 24);
};

struct SsdChunkMaps {
    CUtensorMap x, z, B, C;
};

struct SsdChunkArgs {
    int64_t seqlen, nheads, headdim;  // headdim a multiple of 64
    const __nv_bfloat16 *delta;  // [batch, seqlen, nheads]
    const float *A, *D, *delta_bias, *h0;
    float *h_final;
    __nv_bfloat16 *out;
    int *status;
    uint32_t debug_flags;
    uint64_t timeout_cycles;
};

// log2(x) on the special-function unit (flush-to-zero; log2(0) = -inf).
__device__ __forceinline__ float lg2_mufu(float x) {
    float y;
    asm("lg2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// s + e = a + b exactly, s = fl(a + b) (Knuth's TwoSum, six additions).
__device__ __forceinline__ void two_sum(float a, float b, float &s, float &e) {
    s = __fadd_rn(a, b);
    const float bb = __fsub_rn(s, a);
    e = __fadd_rn(__fsub_rn(a, __fsub_rn(s, bb)), __fsub_rn(b, bb));
}

// grid (nheads * headdim / 64, batch), 352 threads; SP: softplus on.  headdim a
// multiple of 64, d_state 16, bf16 I/O, nheads a multiple of 8.
template <bool SP>
__global__ void __launch_bounds__(SsdChunkCfg::kThreads, 1)
    s6_ssd_chunk_kernel(const __grid_constant__ SsdChunkMaps maps, const SsdChunkArgs a) {
    using C = SsdChunkCfg;
    constexpr int S = C::STAGES;
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw = smem_u32(smem_raw);
    uint8_t *smem = smem_raw + (((raw + 1023u) & ~1023u) - raw);
    const uint32_t sbase = smem_u32(smem);
    uint64_t *loaded = reinterpret_cast<uint64_t *>(smem + C::kOffBar);
    uint64_t *full = loaded + S;      // the chunk's tables are written
    uint64_t *empty = full + S;       // the math warps and the state warp are done with it
    uint64_t *cb_full = empty + S;    // CB_c is in TMEM
    uint64_t *m_full = cb_full + 1;   // M_c and W_c are in shared memory
    uint64_t *m_free = m_full + 1;    // the MMAs have read M_c and W_c
    uint64_t *ds_full = m_free + 1;   // DS_c is in TMEM
    uint64_t *ds_empty = ds_full + 1; // the state warp has read DS_c
    // [2] h_{c-1} planes are in h buffer c % 2 for YI_c.  One barrier per
    // buffer: a buffer is refilled only after the MMA that read it completed,
    // so neither barrier can run a phase ahead of the MMA lane's wait.
    uint64_t *h_ready = ds_empty + 1;
    uint64_t *y_full = h_ready + 2;   // [2] Y_c and YI_c are complete
    uint64_t *y_empty = y_full + 2;   // [2] the epilogue has read them
    uint64_t *drain = y_empty + 2;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + C::kOffSlot);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);
    float *dsk = reinterpret_cast<float *>(smem + C::kOffD);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    // this CTA's 64 channels: slice blockIdx.x % (headdim / 64) of head
    // blockIdx.x / (headdim / 64); channel d = head * headdim + p, so the slice
    // starts at channel blockIdx.x * 64
    const int head = static_cast<int>(blockIdx.x / (a.headdim / C::P));
    const int64_t c0 = int64_t(blockIdx.x) * C::P;
    const int64_t b = blockIdx.y;
    const int64_t L = a.seqlen, Dm = a.nheads * a.headdim;
    const int nc = static_cast<int>((L + C::Q - 1) / C::Q);
    const uint64_t limit = a.timeout_cycles;
    auto fail = [&]() {
        if (!*abort_flag) record_status(a.status, kStTimeout);
        *abort_flag = 1;
    };
    auto stage_u32 = [&](int s) { return sbase + uint32_t(s) * C::kStage; };

    if (threadIdx.x == 0) {
        for (int s = 0; s < S; ++s) {
            mbar_init(&loaded[s], 1);
            mbar_init(&full[s], 32);
            mbar_init(&empty[s], 256 + 1);
        }
        mbar_init(cb_full, 1);
        mbar_init(m_full, 256);
        mbar_init(m_free, 1);
        mbar_init(ds_full, 1);
        mbar_init(ds_empty, 32);
        for (int i = 0; i < 2; ++i) {
            mbar_init(&h_ready[i], 32);
            mbar_init(&y_full[i], 1);
            mbar_init(&y_empty[i], 256);
        }
        mbar_init(drain, 1);
        *abort_flag = 0;
        fence_mbarrier_init();
        prefetch_tensormap(&maps.x);
        prefetch_tensormap(&maps.z);
        prefetch_tensormap(&maps.B);
        prefetch_tensormap(&maps.C);
    }
    if (threadIdx.x < C::P)
        dsk[threadIdx.x] = a.D ? __ldg(a.D + c0 + threadIdx.x) : 0.0f;
    if (warp == 2) {
        tmem_alloc(tmem_slot, C::kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *reinterpret_cast<volatile uint32_t *>(tmem_slot);

    if (warp == 1) {
        // ================= producer: TMA ring and the chunk tables =================
        const int bb = static_cast<int>(b);
        const float a2 = __ldg(a.A + head) * kLog2e;
        const float bias = a.delta_bias ? __ldg(a.delta_bias + head) : 0.0f;
        int last[S];  // lane 0: the chunk whose loads are in flight in each stage, or -1
        for (int s = 0; s < S; ++s) last[s] = -1;
        auto issue = [&](int k) {  // lane 0; stage k % S is free
            if (k >= nc) return;
            if ((a.debug_flags & 1u) && k == 0) return;  // test hook: withhold chunk 0
            const int s = k % S;
            uint8_t *st = smem + s * C::kStage;
            const int t0 = k * C::Q;
            mbar_arrive_expect_tx(&loaded[s], C::kLoadBytes);
            tma_load_3d(st + C::kX, &maps.x, static_cast<int>(c0), t0, bb, &loaded[s]);
            tma_load_3d(st + C::kZ, &maps.z, static_cast<int>(c0), t0, bb, &loaded[s]);
            tma_load_3d(st + C::kC, &maps.C, 0, t0, bb, &loaded[s]);
            tma_load_3d(st + C::kB, &maps.B, 0, t0, bb, &loaded[s]);
            last[s] = k;
        };
        // chunk k landed: Delta_t and sigma_t = log2(e) A sum_{tau <= t} Delta_tau
        const __nv_bfloat16 *dseq = a.delta + b * L * a.nheads + head;  // + t * nheads
        // this lane's 4 tokens of delta for chunk k (plain loads, one chunk ahead)
        auto fetch = [&](int k, __nv_bfloat16 (&raw)[4]) {
            const int64_t rem = L - int64_t(k) * C::Q;
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const int t = lane * 4 + i;
                raw[i] = k < nc && t < rem ? dseq[(int64_t(k) * C::Q + t) * a.nheads]
                                           : __float2bfloat16_rn(0.0f);
            }
        };
        __nv_bfloat16 raw[4];
        auto prepare = [&](int k) -> bool {
            const int s = k % S;
            const int64_t rem = L - int64_t(k) * C::Q;  // tokens left in the sequence
            float rv[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) rv[i] = to_f32(raw[i]);
            fetch(k + 1, raw);
            if (!warp_agree(mbar_wait_or_abort(&loaded[s], (k / S) & 1, limit, abort_flag)))
                return false;
            if (lane == 0) last[s] = -1;
            uint8_t *st = smem + s * C::kStage;
            // Delta_t, and the prefix sums of Delta as hi + lo pairs (TwoSum at
            // every addition: within the lane, then a warp scan of the lanes'
            // totals)
            float dl[4], ch[4], cl[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const int t = lane * 4 + i;
                const float v = rv[i] + bias;
                dl[i] = t < rem ? (SP ? softplus_io<__nv_bfloat16>(v) : v) : 0.0f;
                if (i == 0) {
                    ch[0] = dl[0];
                    cl[0] = 0.0f;
                } else {
                    two_sum(ch[i - 1], dl[i], ch[i], cl[i]);
                    cl[i] += cl[i - 1];
                }
            }
            float ih = ch[3], il = cl[3];  // inclusive prefix over the lanes' totals
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const float uh = __shfl_up_sync(0xffffffffu, ih, o);
                const float ul = __shfl_up_sync(0xffffffffu, il, o);
                if (lane >= o) {
                    float e;
                    two_sum(uh, ih, ih, e);
                    il += ul + e;
                }
            }
            float eh = __shfl_up_sync(0xffffffffu, ih, 1);  // exclusive prefix
            float el = __shfl_up_sync(0xffffffffu, il, 1);
            if (lane == 0) eh = el = 0.0f;
            float sh[4], sl[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                float h, e;
                two_sum(eh, ch[i], h, e);
                const float l = e + el + cl[i];
                // sigma = a2 (h + l) as hi + lo: the product's rounding error by fma
                sh[i] = a2 * h;
                sl[i] = fmaf(a2, h, -sh[i]) + a2 * l;
            }
            // within each 16-token block, sigma relative to a reference token of
            // the block: its first (lane 4 (lane / 4), component 0) without
            // softplus; its last (lane 4 (lane / 4) + 3, component 3) with it
            const int ref_lane = SP ? (lane | 3) : (lane & ~3);
            const float bh = __shfl_sync(0xffffffffu, SP ? sh[3] : sh[0], ref_lane);
            const float bl = __shfl_sync(0xffffffffu, SP ? sl[3] : sl[0], ref_lane);
            float dt4[4], tab[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                dt4[i] = (bh - sh[i]) + (bl - sl[i]);
                tab[i] = dl[i];
                if (SP) {
                    // with softplus, Delta >= 0: log2(Delta) joins the exponent, so
                    // that M's Delta factor costs no multiply (Delta = 0 gives
                    // -inf, e^-inf = 0); and the Delta table holds
                    // e^{s_j1 - s_j} Delta_j instead (j1 the block's last token:
                    // at most Delta_j, so it never overflows)
                    dt4[i] += lg2_mufu(dl[i]);
                    tab[i] = ex2_mufu(dt4[i]);
                }
            }
            reinterpret_cast<float4 *>(st + C::kDel)[lane] = make_float4(tab[0], tab[1], tab[2], tab[3]);
            reinterpret_cast<float4 *>(st + C::kSig)[lane] = make_float4(sh[0], sh[1], sh[2], sh[3]);
            reinterpret_cast<float4 *>(st + C::kSig + 512)[lane] = make_float4(sl[0], sl[1], sl[2], sl[3]);
            reinterpret_cast<float4 *>(st + C::kDlt)[lane] = make_float4(dt4[0], dt4[1], dt4[2], dt4[3]);
            mbar_arrive(&full[s]);
            return true;
        };
        // the chunk's readers are done with it: refill its stage
        auto retire = [&](int k) -> bool {
            const int s = k % S;
            if (!warp_agree(mbar_wait_or_abort(&empty[s], (k / S) & 1, limit, abort_flag)))
                return false;
            if (lane == 0) issue(k + S);
            __syncwarp();
            return true;
        };
        // Each chunk's tables are prepared as soon as its loads land, so that
        // they are never what the MMA lane waits for.
        if (lane == 0)
            for (int k = 0; k < S; ++k) issue(k);
        __syncwarp();
        fetch(0, raw);
        bool ok = true;
        for (int k = 0; ok && k < S && k < nc; ++k) ok = prepare(k);
        for (int k = 0; ok && k < nc; ++k) {
            ok = retire(k);  // the stage of chunk k takes chunk k + S
            if (ok && k + S < nc) ok = prepare(k + S);
        }
        if (!ok) fail();
        if (lane == 0)
            for (int s = 0; s < S; ++s)  // no load may still be landing when the CTA ends
                if (last[s] >= 0 && !mbar_wait_bounded(&loaded[s], (last[s] / S) & 1, limit))
                    fail();
        __syncwarp();
    } else if (warp == 2) {
        // ============================ MMA issue ============================
        if (lane == 0) {
            bool ok = true;
            auto wait = [&](uint64_t *bar, uint32_t par) {
                if (!mbar_wait_or_abort(bar, par, limit, abort_flag)) ok = false;
                return ok;
            };
            auto mma_cb = [&](int k) {  // CB = C_k . B_k^T
                const uint32_t st = stage_u32(k % S);
                umma_bf16(tmem + C::kColCB, umma_desc_sw32_k(st + C::kC),
                          umma_desc_sw32_k(st + C::kB), C::kIdescCB, 0u);
                tc_commit(cb_full);
            };
            if (nc > 0 && wait(&loaded[0], 0) && wait(&full[0], 0)) {
                tc_fence_after();
                mma_cb(0);
            }
            for (int c = 0; ok && c < nc; ++c) {
                const int s = c % S, yb = c & 1;
                if (!wait(m_full, c & 1)) break;
                if (c >= 2 && !wait(&y_empty[yb], ((c >> 1) - 1) & 1)) break;
                tc_fence_after();
                const uint32_t xs = stage_u32(s) + C::kX;
                const uint32_t mh = sbase + C::kOffM, ml = mh + C::kMPlane;
                const uint32_t wh = stage_u32(s) + C::kW, wl = wh + C::kWPlane;
                // Y_c = M_c X_c; the M buffer is released as soon as these complete
#pragma unroll
                for (int kk = 0; kk < 8; ++kk) {  // K = 128 tokens in steps of 16
                    const uint64_t bx = umma_desc_sw128_mn(xs + kk * 2048u);
                    const uint32_t ka = (kk >> 2) * C::kMPlane / 2 + (kk & 3) * 32u;
                    umma_bf16(tmem + C::kColY + 64u * yb, umma_desc_sw128(mh + ka), bx, C::kIdescX,
                              kk > 0 ? 1u : 0u);
                    umma_bf16(tmem + C::kColY + 64u * yb, umma_desc_sw128(ml + ka), bx, C::kIdescX,
                              1u);
                }
                tc_commit(m_free);
                // CB_{c+1}, so that the math warps can build M_{c+1} meanwhile
                if (c + 1 < nc) {
                    const int s1 = (c + 1) % S;
                    if (!wait(&loaded[s1], ((c + 1) / S) & 1) || !wait(&full[s1], ((c + 1) / S) & 1))
                        break;
                    tc_fence_after();
                    mma_cb(c + 1);
                }
                // DS_c = W_c X_c, once the state warp has read DS_{c-1}
                if (c >= 1 && !wait(ds_empty, (c - 1) & 1)) break;
                tc_fence_after();
#pragma unroll
                for (int kk = 0; kk < 8; ++kk) {
                    const uint64_t bx = umma_desc_sw128_mn(xs + kk * 2048u);
                    const uint32_t kw = (kk >> 2) * C::kWPlane / 2 + (kk & 3) * 32u;
                    umma_bf16(tmem + C::kColDS, umma_desc_sw128(wh + kw), bx, C::kIdescX,
                              kk > 0 ? 1u : 0u);
                    umma_bf16(tmem + C::kColDS, umma_desc_sw128(wl + kw), bx, C::kIdescX, 1u);
                }
                tc_commit(ds_full);
                if (!wait(&h_ready[yb], (c >> 1) & 1)) break;  // h_{c-1} in buffer c % 2
                tc_fence_after();
                const uint32_t hb = sbase + C::kOffH + uint32_t(yb) * 2 * C::kHPlane;
                const uint64_t ca = umma_desc_sw32_k(stage_u32(s) + C::kC);
                umma_bf16(tmem + C::kColYI + 64u * yb, ca, umma_desc_sw128_mn(hb), C::kIdescX, 0u);
                umma_bf16(tmem + C::kColYI + 64u * yb, ca, umma_desc_sw128_mn(hb + C::kHPlane),
                          C::kIdescX, 1u);
                tc_commit(&y_full[yb]);
            }
            if (!ok) fail();
            // TMEM is not freed while MMAs run: this arrives once every MMA
            // issued above has completed.
            tc_commit(drain);
            if (!mbar_wait_bounded(drain, 0, limit)) fail();
        }
        __syncwarp();
    } else if (warp == 0) {
        // ============================ state warp ============================
        // lane n < 16 keeps h[n][p], p = 0..63; lanes 16-31 follow the warp-wide
        // TMEM loads and arrivals.
        const int n = lane & 15;
        const bool own = lane < 16;
        const int64_t hrow = (b * Dm + c0) * C::N + n;  // + p * N
        float h[64];
#pragma unroll
        for (int p = 0; p < 64; ++p) h[p] = own && a.h0 ? __ldg(a.h0 + hrow + p * C::N) : 0.0f;
        // h as the hi / lo planes of an MN-major [16 K rows][64] operand
        auto put_h = [&](int buf) {
            const uint32_t base = sbase + C::kOffH + uint32_t(buf) * 2 * C::kHPlane +
                                  uint32_t(n >> 3) * 1024u + uint32_t(n & 7) * 128u;
            if (own) {
#pragma unroll
                for (int g = 0; g < 8; ++g) {
                    uint4 hi, lo;
                    split_bf16x2(h[8 * g + 0], h[8 * g + 1], hi.x, lo.x);
                    split_bf16x2(h[8 * g + 2], h[8 * g + 3], hi.y, lo.y);
                    split_bf16x2(h[8 * g + 4], h[8 * g + 5], hi.z, lo.z);
                    split_bf16x2(h[8 * g + 6], h[8 * g + 7], hi.w, lo.w);
                    const uint32_t off = uint32_t(g ^ (n & 7)) * 16u;
                    st_shared_v4(base + off, hi);
                    st_shared_v4(base + C::kHPlane + off, lo);
                }
            }
            fence_proxy_async_smem();
            mbar_arrive(&h_ready[buf]);
        };
        put_h(0);
        bool ok = true;
        for (int c = 0; ok && c < nc; ++c) {
            const int s = c % S;
            const bool got = mbar_wait_or_abort(ds_full, c & 1, limit, abort_flag) &&
                             mbar_wait_or_abort(&full[s], (c / S) & 1, limit, abort_flag);
            if (!warp_agree(got)) {
                ok = false;
                break;
            }
            tc_fence_after();
            uint32_t r[64];
#pragma unroll
            for (int i = 0; i < 4; ++i)
                tmem_ld16_async(tmem + C::kColDS + 16u * i,
                                *reinterpret_cast<uint32_t(*)[16]>(r + 16 * i));
            tmem_wait_ld();
#pragma unroll
            for (int i = 0; i < 4; ++i) tmem_regs_ready(*reinterpret_cast<uint32_t(*)[16]>(r + 16 * i));
            tc_fence_before();
            mbar_arrive(ds_empty);
            const float *sgs = reinterpret_cast<const float *>(smem + s * C::kStage + C::kSig);
            const float sig_end = sgs[C::Q - 1] + sgs[2 * C::Q - 1];
            __syncwarp();
            if (lane == 0) mbar_arrive(&empty[s]);
            const float dec = ex2_mufu(sig_end);
#pragma unroll
            for (int p = 0; p < 64; ++p) h[p] = fmaf(dec, h[p], __uint_as_float(r[p]));
            if (c + 1 < nc) {
                // buffer (c + 1) % 2 was last read by YI_{c-1}
                if (c >= 1 &&
                    !warp_agree(mbar_wait_or_abort(&y_full[(c - 1) & 1], ((c - 1) >> 1) & 1, limit,
                                                   abort_flag))) {
                    ok = false;
                    break;
                }
                put_h((c + 1) & 1);
            }
        }
        if (!ok) fail();
        if (ok && own && a.h_final) {
#pragma unroll
            for (int p = 0; p < 64; ++p) a.h_final[hrow + p * C::N] = h[p];
        }
    } else {
        // ============================ math warps ============================
        const int wg = (warp - 3) >> 2;  // column group
        const int q = warp & 3;          // TMEM lane quarter
        const int r = q * 32 + lane;     // this thread's token row of the chunk
        const uint32_t lane_off = uint32_t(q * 32) << 16;
        const uint32_t mh = sbase + C::kOffM, ml = mh + C::kMPlane;
        bool ok = true;
        for (int it = 0; it <= nc; ++it) {
            if (it < nc) {
                // ------------------------------- build M_c and W_c
                const int c = it, s = c % S;
                bool got = c == 0 || mbar_wait_or_abort(m_free, (c - 1) & 1, limit, abort_flag);
                got = got && mbar_wait_or_abort(cb_full, c & 1, limit, abort_flag) &&
                      mbar_wait_or_abort(&loaded[s], (c / S) & 1, limit, abort_flag) &&
                      mbar_wait_or_abort(&full[s], (c / S) & 1, limit, abort_flag);
                if (!warp_agree(got)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const float *del = reinterpret_cast<const float *>(smem + s * C::kStage + C::kDel);
                const float *sgh = reinterpret_cast<const float *>(smem + s * C::kStage + C::kSig);
                const float *sgl = sgh + C::Q;
                const float *dlt = reinterpret_cast<const float *>(smem + s * C::kStage + C::kDlt);
                const float shr = sgh[r], slr = sgl[r];
                const uint32_t rowm = uint32_t(r) * 128u;
                // this group's 16-column blocks, one at a time (a rolled loop keeps
                // the warps' code small)
#pragma unroll 1
                for (int i = 0; i < 4; ++i) {
                    const int jb = wg + 2 * i;
                    const int j0 = 16 * jb;
                    uint32_t hi[8], lo[8];
                    if (j0 > q * 32 + 31) {  // above the diagonal for every row of the warp
#pragma unroll
                        for (int u = 0; u < 8; ++u) hi[u] = lo[u] = 0u;
                    } else {
                        uint32_t v[16];
                        tmem_ld16_async(tmem + lane_off + C::kColCB + uint32_t(j0), v);
                        // sigma_r - sigma_j = (sigma_r - sigma_ref) + delta_j: the first
                        // term once per block (from the hi + lo pairs; ref the block's
                        // first token, or with softplus its last), the second from
                        // the table
                        const int jr = SP ? j0 + 15 : j0;
                        const float base = (shr - sgh[jr]) + (slr - sgl[jr]);
                        const float2 base2 = make_float2(base, base), one2 = make_float2(1.0f, 1.0f);
                        tmem_wait_ld();
                        tmem_regs_ready(v);
                        if (SP && j0 + 15 <= q * 32) {
                            // the block is below the diagonal for every row of the
                            // warp: e^{s_r - s_j} Delta_j = e^{s_r - s_j1} (e^{s_j1 - s_j}
                            // Delta_j), one exp for the block and the table's factor,
                            // both at most 1 (resp. Delta_j)
                            const float ub = ex2_mufu(base);
                            const float2 u2 = make_float2(ub, ub);
#pragma unroll
                            for (int u = 0; u < 8; u += 2) {
                                const float4 w4 = *reinterpret_cast<const float4 *>(del + j0 + 2 * u);
#pragma unroll
                                for (int hh = 0; hh < 2; ++hh) {
                                    const int uu = u + hh;
                                    const float2 wj = hh ? make_float2(w4.z, w4.w) : make_float2(w4.x, w4.y);
                                    const float2 cb = make_float2(__uint_as_float(v[2 * uu]),
                                                                  __uint_as_float(v[2 * uu + 1]));
                                    const float2 m = mul2(mul2(cb, wj), u2);
                                    split_bf16x2(m.x, m.y, hi[uu], lo[uu]);
                                }
                            }
                        } else
#pragma unroll
                        for (int u = 0; u < 8; u += 2) {
                            const int j = j0 + 2 * u;
                            const float4 d4 = SP ? make_float4(1.0f, 1.0f, 1.0f, 1.0f)
                                                 : *reinterpret_cast<const float4 *>(del + j);
                            const float4 t4 = *reinterpret_cast<const float4 *>(dlt + j);
#pragma unroll
                            for (int hh = 0; hh < 2; ++hh) {
                                const float2 dj = hh ? make_float2(d4.z, d4.w) : make_float2(d4.x, d4.y);
                                const float2 tj = hh ? make_float2(t4.z, t4.w) : make_float2(t4.x, t4.y);
                                const float2 arg = fma2(base2, one2, tj);
                                const float2 e2 = make_float2(ex2_mufu(arg.x), ex2_mufu(arg.y));
                                const int uu = u + hh, jj = j + 2 * hh;
                                const float2 cb = make_float2(__uint_as_float(v[2 * uu]),
                                                              __uint_as_float(v[2 * uu + 1]));
                                float2 m = mul2(SP ? cb : mul2(cb, dj), e2);
                                if (jj > r) m.x = 0.0f;
                                if (jj + 1 > r) m.y = 0.0f;
                                split_bf16x2(m.x, m.y, hi[uu], lo[uu]);
                            }
                        }
                    }
                    // row r of the K-major 128-byte-swizzled M planes: K atom j0 / 64,
                    // 16-byte chunks (j0 % 64) / 8 and the next
                    const uint32_t atom = uint32_t(j0 >> 6) * (C::kMPlane / 2) + rowm;
                    const uint32_t ch = uint32_t((j0 & 63) >> 3);
                    const uint32_t o0 = ((ch ^ uint32_t(r & 7)) << 4), o1 = (((ch + 1) ^ uint32_t(r & 7)) << 4);
                    st_shared_v4(mh + atom + o0, make_uint4(hi[0], hi[1], hi[2], hi[3]));
                    st_shared_v4(mh + atom + o1, make_uint4(hi[4], hi[5], hi[6], hi[7]));
                    st_shared_v4(ml + atom + o0, make_uint4(lo[0], lo[1], lo[2], lo[3]));
                    st_shared_v4(ml + atom + o1, make_uint4(lo[4], lo[5], lo[6], lo[7]));
                }
                if (q < 2) {
                    // W of the chunk into the stage, by the warps of the first two
                    // lane quarters (their share of M is the smallest): token
                    // j = 32 (2 q + wg) + lane, w_j = Delta_j e^{s_127 - s_j},
                    // W[n][j] = w_j B_j[n]
                    const int j = 32 * (2 * q + wg) + lane;
                    // SP: del holds e^{s_j1 - s_j} Delta_j, j1 = j | 15
                    const int jw = SP ? (j | 15) : j;
                    const float w = del[j] * ex2_mufu((sgh[C::Q - 1] - sgh[jw]) + (sgl[C::Q - 1] - sgl[jw]));
                    const uint32_t brow = stage_u32(s) + C::kB + uint32_t(j) * 32u;
                    const uint32_t sw = uint32_t((j >> 2) & 1);
                    const uint4 b0 = ld_shared_v4(brow + (sw << 4));         // n 0-7
                    const uint4 b1 = ld_shared_v4(brow + ((sw ^ 1u) << 4));  // n 8-15
                    const uint32_t bwd[8] = {b0.x, b0.y, b0.z, b0.w, b1.x, b1.y, b1.z, b1.w};
                    const uint32_t wh = stage_u32(s) + C::kW, wl = wh + C::kWPlane;
                    const uint32_t col = uint32_t(j >> 6) * (C::kWPlane / 2) + uint32_t(j & 7) * 2u;
                    const uint32_t chk = uint32_t((j & 63) >> 3);
#pragma unroll
                    for (int u = 0; u < 8; ++u) {
                        const float2 bf = bf16x2_to_f2(bwd[u]);
                        uint32_t h2, l2;
                        split_bf16x2(w * bf.x, w * bf.y, h2, l2);
#pragma unroll
                        for (int e = 0; e < 2; ++e) {
                            const int nn = 2 * u + e;  // row of W
                            const uint32_t off = col + uint32_t(nn >> 3) * 1024u + uint32_t(nn & 7) * 128u +
                                                 ((chk ^ uint32_t(nn & 7)) << 4);
                            st_shared_u16(wh + off, uint16_t(e ? h2 >> 16 : h2 & 0xFFFFu));
                            st_shared_u16(wl + off, uint16_t(e ? l2 >> 16 : l2 & 0xFFFFu));
                        }
                    }
                }
                fence_proxy_async_smem();  // M and W, before the tensor cores read them
                tc_fence_before();         // the CB reads, before MMA CB_{c+1} may overwrite it
                mbar_arrive(m_full);
            }
            if (it >= 1) {
                // ------------------------------- epilogue of chunk e = it - 1
                const int e = it - 1, s = e % S, yb = e & 1;
                if (!warp_agree(mbar_wait_or_abort(&y_full[yb], (e >> 1) & 1, limit, abort_flag))) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const float *sgh = reinterpret_cast<const float *>(smem + s * C::kStage + C::kSig);
                const float coef = ex2_mufu(sgh[r] + sgh[C::Q + r]);  // e^{s_t}
                const int64_t t = int64_t(e) * C::Q + r;
                const uint32_t xrow = stage_u32(s) + C::kX + uint32_t(r) * 128u;
                const uint32_t zrow = stage_u32(s) + C::kZ + uint32_t(r) * 128u;
                const float2 coef2 = make_float2(coef, coef), one2 = make_float2(1.0f, 1.0f);
                const float2 nl2 = make_float2(-kLog2e, -kLog2e);
                uint4 *dst = reinterpret_cast<uint4 *>(a.out + (b * L + t) * Dm + c0 +
                                                       32 * wg);
                // this group's 32 columns in two rolled halves of 16 (small code):
                // Y and YI from TMEM, x and z from shared memory, the 32 bytes of
                // output straight to global memory
#pragma unroll 1
                for (int hh = 0; hh < 2; ++hh) {
                    const int p0 = 32 * wg + 16 * hh;
                    uint32_t yv[16], yi[16];
                    tmem_ld16_async(tmem + lane_off + C::kColY + 64u * yb + uint32_t(p0), yv);
                    tmem_ld16_async(tmem + lane_off + C::kColYI + 64u * yb + uint32_t(p0), yi);
                    uint4 xv[2], zv[2];
#pragma unroll
                    for (int g = 0; g < 2; ++g) {
                        const uint32_t off = ((uint32_t(p0 / 8 + g) ^ uint32_t(r & 7)) << 4);
                        xv[g] = ld_shared_v4(xrow + off);
                        zv[g] = ld_shared_v4(zrow + off);
                    }
                    tmem_wait_ld();
                    tmem_regs_ready(yv);
                    tmem_regs_ready(yi);
                    uint4 o[2];
#pragma unroll
                    for (int g = 0; g < 2; ++g) {
                        const uint32_t xw[4] = {xv[g].x, xv[g].y, xv[g].z, xv[g].w};
                        const uint32_t zw[4] = {zv[g].x, zv[g].y, zv[g].z, zv[g].w};
                        uint32_t ow[4];
#pragma unroll
                        for (int u = 0; u < 4; ++u) {
                            const int k = 8 * g + 2 * u;  // column p0 + k
                            const float2 xf = bf16x2_to_f2(xw[u]);
                            const float2 zf = bf16x2_to_f2(zw[u]);
                            const float2 dd = *reinterpret_cast<const float2 *>(dsk + p0 + k);
                            // y = Y + e^{s_t} YI + D x;  out = y z / (1 + e^{-z})
                            float2 y = fma2(coef2,
                                            make_float2(__uint_as_float(yi[k]), __uint_as_float(yi[k + 1])),
                                            make_float2(__uint_as_float(yv[k]), __uint_as_float(yv[k + 1])));
                            y = fma2(dd, xf, y);
                            const float2 nz = mul2(zf, nl2);
                            const float2 den =
                                fma2(make_float2(ex2_mufu(nz.x), ex2_mufu(nz.y)), one2, one2);
                            const float2 g2 = mul2(zf, make_float2(rcp_mufu(den.x), rcp_mufu(den.y)));
                            const float2 ov = mul2(y, g2);
                            ow[u] = pack_bf16x2(ov.x, ov.y);
                        }
                        o[g] = make_uint4(ow[0], ow[1], ow[2], ow[3]);
                    }
                    if (t < L) {
                        dst[2 * hh] = o[0];
                        dst[2 * hh + 1] = o[1];
                    }
                }
                tc_fence_before();
                mbar_arrive(&y_empty[yb]);  // Y and YI of this buffer may be overwritten
                mbar_arrive(&empty[s]);     // and the stage refilled
            }
        }
        if (!ok) fail();
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 2) {
        tc_fence_after();
        tmem_dealloc(tmem, C::kTmemCols);
    }
}

}  // namespace jssm
