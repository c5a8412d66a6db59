// jamba_ssm.cu -- host side of the C ABI declared in include/jamba_ssm.h:
// argument validation, variant selection, TMA tensor-map encoding and the
// launches of the S6 kernels.  Nothing here allocates device memory.
#include <cuda.h>
#include <cuda_runtime.h>

#include <cstddef>
#include <cstdlib>
#include <cstring>
#include <mutex>

#include "jamba_ssm.h"
#include "s6_scan.cuh"
#include "s6_scan_bwd.cuh"
#include "s6_scan_fused.cuh"
#include "s6_scan_serving.cuh"
#include "s6_scan_small.cuh"
#include "s6_ssd.cuh"
#include "s6_ssd_chunk.cuh"
#include "s6_state_update.cuh"

using jssm::ScanArgs;
using jssm::UpdateArgs;

namespace {

thread_local int t_last_cuda_error = 0;

jamba_ssm_status cuda_fail(cudaError_t e) {
    t_last_cuda_error = static_cast<int>(e);
    return JAMBA_SSM_ERR_CUDA;
}

// ------------------------------------------------------------------ devices
constexpr int kMaxDevices = 64;
struct DeviceInfo {
    bool ready = false;
    bool usable = false;
    int sms = 0;
};
DeviceInfo g_devices[kMaxDevices];
std::mutex g_mutex;

// Returns the current device's info, or sets *st on failure.
const DeviceInfo *current_device(jamba_ssm_status *st) {
    int dev = -1;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
        *st = e == cudaSuccess ? JAMBA_SSM_ERR_NO_DEVICE : cuda_fail(e);
        if (e != cudaSuccess && (e == cudaErrorNoDevice || e == cudaErrorInsufficientDriver))
            *st = JAMBA_SSM_ERR_NO_DEVICE;
        return nullptr;
    }
    std::lock_guard<std::mutex> lock(g_mutex);
    DeviceInfo &info = g_devices[dev];
    if (!info.ready) {
        int major = 0, minor = 0, sms = 0;
        if ((e = cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev)) != cudaSuccess ||
            (e = cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev)) != cudaSuccess ||
            (e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess) {
            *st = cuda_fail(e);
            return nullptr;
        }
        info.usable = (major == 10 && minor == 0);  // built for sm_100a only
        info.sms = sms;
        info.ready = true;
    }
    if (!info.usable) {
        *st = JAMBA_SSM_ERR_NO_DEVICE;
        return nullptr;
    }
    return &info;
}

// ---------------------------------------------------------- tensor maps (TMA)
using EncodeTiledFn = CUresult (*)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *,
                                   const cuuint64_t *, const cuuint64_t *, const cuuint32_t *,
                                   const cuuint32_t *, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn(jamba_ssm_status *st) {
    static EncodeTiledFn fn = nullptr;
    static std::once_flag once;
    static cudaError_t err = cudaSuccess;
    std::call_once(once, [] {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        err = cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q);
        if (err == cudaSuccess && q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
        else if (err == cudaSuccess)
            err = cudaErrorSymbolNotFound;
    });
    if (!fn) *st = cuda_fail(err);
    return fn;
}

// 3-D map over [dim2][dim1][dim0] (dim0 innermost), box {box0, box1, 1}.
bool encode_3d(EncodeTiledFn fn, CUtensorMap *map, const void *ptr, CUtensorMapDataType dt,
               int elem_bytes, int64_t dim0, int64_t dim1, int64_t dim2, int box0, int box1,
               CUtensorMapSwizzle swizzle = CU_TENSOR_MAP_SWIZZLE_NONE) {
    cuuint64_t dims[3] = {(cuuint64_t)dim0, (cuuint64_t)dim1, (cuuint64_t)dim2};
    cuuint64_t strides[2] = {(cuuint64_t)(dim0 * elem_bytes), (cuuint64_t)(dim0 * dim1 * elem_bytes)};
    cuuint32_t box[3] = {(cuuint32_t)box0, (cuuint32_t)box1, 1};
    cuuint32_t estr[3] = {1, 1, 1};
    CUresult r = fn(map, dt, 3, const_cast<void *>(ptr), dims, strides, box, estr,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                    CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

// ----------------------------------------------------------- scan variants
struct ScanVariant {
    int io_dtype, n, g, nw, tt, cw;
    int threads;
    double step_cost;  // measured time per channel-step, relative (multi-task steady state)
    int smem, smem_serving;
    const void *kernel;          // batched layout
    const void *kernel_serving;  // packed layout and / or state-cache slots
    const void *kernel_ckpt;      // the backward's checkpoint pass, or null
    const void *kernel_fwd_ckpt;  // the forward storing the same checkpoints, or null
    bool attr_set_ckpt[kMaxDevices], attr_set_fwd_ckpt[kMaxDevices];
    bool attr_set[kMaxDevices], attr_set_serving[kMaxDevices];
};

// NW compute warps (each does its channels' recurrence, softplus and gate) and
// one producer warp (TMA, B/C widening).
template <typename IoT, int N, int G, int NW, int TT, int S, bool CKPT = false>
ScanVariant make_fused(double step_cost) {
    using Cfg = jssm::FusedCfg<IoT, N, G, NW, TT, S>;
    ScanVariant v{};
    v.io_dtype = std::is_same<IoT, float>::value ? JAMBA_SSM_F32 : JAMBA_SSM_BF16;
    v.n = N;
    v.g = G;
    v.nw = NW;
    v.tt = TT;
    v.cw = Cfg::CW;
    v.threads = (NW + 1) * 32;
    v.step_cost = step_cost;
    v.smem = Cfg::kSmemBytes;
    v.smem_serving = jssm::ServingCfg<IoT, N, G, NW, TT, S>::kSmemBytes;
    v.kernel = reinterpret_cast<const void *>(&jssm::s6_scan_fused_kernel<IoT, N, G, NW, TT, S>);
    v.kernel_serving =
        reinterpret_cast<const void *>(&jssm::s6_scan_serving_kernel<IoT, N, G, NW, TT, S>);
    if constexpr (CKPT) {
        v.kernel_ckpt =
            reinterpret_cast<const void *>(&jssm::s6_scan_fused_kernel<IoT, N, G, NW, TT, S, 1>);
        v.kernel_fwd_ckpt =
            reinterpret_cast<const void *>(&jssm::s6_scan_fused_kernel<IoT, N, G, NW, TT, S, 2>);
    }
    return v;
}

// <io type, d_state, lanes per channel, compute warps, time tile, TMA stages>
// with the relative time per channel-step each variant sustains when every SM
// is busy (measured on B200 at Jamba's sizes, bf16 I/O; the fp32 ones serve
// small and test shapes).  Fewer lanes per channel cost less per step; more
// lanes give narrower CTAs, so a single sequence's 8192 channels still cover
// the 148 SMs (56 channels per CTA -> 147 CTAs).  The variants marked `true`
// also serve the backward's checkpoint pass (the states alone, stored every
// kCk steps) and the forward that stores those checkpoints, chosen by the same
// cost model.
ScanVariant g_variants[] = {
    make_fused<__nv_bfloat16, 16, 2, 8, 64, 2, true>(1.00),  // 1: 128 channels / CTA
    make_fused<__nv_bfloat16, 16, 4, 7, 64, 3, true>(1.33),  // 2:  56 channels / CTA
    make_fused<__nv_bfloat16, 16, 4, 8, 64, 3>(1.35),        // 3:  64 channels / CTA
    make_fused<__nv_bfloat16, 16, 4, 7, 32, 4>(1.47),        // 4:  56 channels / CTA
    make_fused<__nv_bfloat16, 8, 2, 8, 32, 4, true>(1.00),   // 5: 128 channels / CTA
    make_fused<__nv_bfloat16, 8, 1, 4, 32, 4>(1.70),         // 6: 128 channels / CTA
    make_fused<__nv_bfloat16, 8, 4, 7, 64, 3, true>(1.29),   // 7:  56 channels / CTA
    make_fused<float, 16, 1, 2, 32, 3, true>(1.00),          // 8:  64 channels / CTA
    make_fused<float, 8, 1, 2, 32, 3, true>(1.00),           // 9:  64 channels / CTA
    make_fused<float, 4, 1, 2, 32, 3, true>(1.00),           // 10: 64 channels / CTA
};
constexpr int kNumVariants = sizeof(g_variants) / sizeof(g_variants[0]);

int channels_per_cta(const ScanVariant &v) { return v.nw * v.cw; }

bool variant_applies(const ScanVariant &v, const jamba_ssm_scan_params *p) {
    return v.io_dtype == p->io_dtype && v.n == p->d_state;
}

// State sizes whose B / C rows are shorter than a 16-byte TMA row (bf16 with
// d_state < 8, fp32 with d_state < 4) take the small-state kernel.
bool small_state(const jamba_ssm_scan_params *p) {
    return p->d_state * (p->io_dtype == JAMBA_SSM_BF16 ? 2 : 4) < 16;
}
constexpr int kSmallThreads = 128;

// Estimated relative time of a variant on `sms` SMs.  One CTA runs per SM and
// walks its share of the (sequence, channel-group) tasks one after another;
// the busiest SM decides: tasks per CTA x channels per task x the variant's
// measured cost per channel-step.
double variant_cost(const ScanVariant &v, const jamba_ssm_scan_params *p, int sms) {
    const int cc = channels_per_cta(v);
    const int64_t tasks = p->batch * ((p->d_inner + cc - 1) / cc);
    const int64_t per_cta = (tasks + sms - 1) / sms;
    return double(per_cta) * cc * v.step_cost;
}

int choose_variant(const jamba_ssm_scan_params *p, int sms, bool ckpt = false) {
    int best = -1;
    double best_cost = 0;
    for (int i = 0; i < kNumVariants; ++i) {
        if (!variant_applies(g_variants[i], p)) continue;
        if (ckpt && !g_variants[i].kernel_ckpt) continue;
        const double c = variant_cost(g_variants[i], p, sms);
        if (best < 0 || c < best_cost) {
            best = i;
            best_cost = c;
        }
    }
    return best;
}

bool aligned(const void *p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

bool overlaps(const void *a, size_t an, const void *b, size_t bn) {
    if (!a || !b || !an || !bn) return false;
    const uintptr_t a0 = reinterpret_cast<uintptr_t>(a), b0 = reinterpret_cast<uintptr_t>(b);
    return a0 < b0 + bn && b0 < a0 + an;
}

constexpr int64_t kMaxElems = int64_t(1) << 40;
constexpr int64_t kMaxI32 = (int64_t(1) << 31) - 1;

// The caller's parameters as this library version reads them: copied over a
// zeroed struct, so the fields past a smaller (ABI version 1) struct_size read
// as zero / NULL.
constexpr size_t kScanParamsV1 = offsetof(jamba_ssm_scan_params, cu_seqlens);
constexpr size_t kUpdateParamsV1 = offsetof(jamba_ssm_state_update_params, state_indices);
constexpr size_t kBwdParamsV3 = offsetof(jamba_ssm_scan_bwd_params, ckpt);

// A workspace, when given, holds the call's status word in its first bytes.
jamba_ssm_status check_workspace(const void *ws, size_t bytes) {
    if (!ws) return JAMBA_SSM_OK;
    if (!aligned(ws, 16)) return JAMBA_SSM_ERR_MISALIGNED;
    return bytes < JAMBA_SSM_STATUS_BYTES ? JAMBA_SSM_ERR_WORKSPACE : JAMBA_SSM_OK;
}

template <typename P>
bool read_params(const P *p, size_t v1_size, P *q) {
    if (!p || p->struct_size < v1_size) return false;
    std::memset(q, 0, sizeof(P));
    std::memcpy(q, p, p->struct_size < sizeof(P) ? p->struct_size : sizeof(P));
    return true;
}

// Token rows of the activations: batch * seqlen, or the packed total.
int64_t token_rows(const jamba_ssm_scan_params *p) {
    return p->cu_seqlens ? p->total_tokens : p->batch * p->seqlen;
}

jamba_ssm_status validate_scan(const jamba_ssm_scan_params *p) {
    if (p->batch < 0 || p->seqlen < 0 || p->d_inner < 1 || p->d_state < 1)
        return JAMBA_SSM_ERR_INVALID_ARG;
    if (p->io_dtype != JAMBA_SSM_BF16 && p->io_dtype != JAMBA_SSM_F32)
        return JAMBA_SSM_ERR_INVALID_ARG;
    if (p->cu_seqlens && p->total_tokens < 0) return JAMBA_SSM_ERR_INVALID_ARG;
    if (p->state_indices && p->num_slots < 1) return JAMBA_SSM_ERR_INVALID_ARG;
    if (!aligned(p->cu_seqlens, 4) || !aligned(p->state_indices, 4)) return JAMBA_SSM_ERR_MISALIGNED;
    // token rows are int32 TMA coordinates, and a tile may start up to one
    // time tile past the last row
    const int64_t kMaxRows = kMaxI32 - 256;
    if (p->batch > kMaxI32 || p->seqlen > kMaxRows || p->d_inner > (int64_t(1) << 30) ||
        p->total_tokens > kMaxRows || p->num_slots > kMaxI32)
        return JAMBA_SSM_ERR_UNSUPPORTED;
    if (!p->cu_seqlens && p->batch && p->seqlen && p->batch > kMaxElems / p->seqlen)
        return JAMBA_SSM_ERR_UNSUPPORTED;
    if (token_rows(p) > kMaxElems / p->d_inner) return JAMBA_SSM_ERR_UNSUPPORTED;
    const int es = p->io_dtype == JAMBA_SSM_BF16 ? 2 : 4;
    const bool n_ok = p->d_state == 1 || p->d_state == 2 || p->d_state == 4 || p->d_state == 8 ||
                      p->d_state == 16;
    if (!n_ok || (p->d_inner * es) % 16 != 0) return JAMBA_SSM_ERR_UNSUPPORTED;
    if (p->kernel_variant < 0 || p->kernel_variant > kNumVariants) return JAMBA_SSM_ERR_UNSUPPORTED;
    if (p->kernel_variant > 0 && !variant_applies(g_variants[p->kernel_variant - 1], p))
        return JAMBA_SSM_ERR_UNSUPPORTED;
    if (small_state(p) && (p->batch > 65535 || p->d_inner > int64_t(kSmallThreads) * 0x7fffffff))
        return JAMBA_SSM_ERR_UNSUPPORTED;  // grid (channel blocks, sequences)
    jamba_ssm_status ws = check_workspace(p->workspace, p->workspace_bytes);
    if (ws != JAMBA_SSM_OK) return ws;
    if (p->ckpt) {  // the backward's checkpoints: its layouts and state sizes only
        const bool bf = p->io_dtype == JAMBA_SSM_BF16;
        const bool n_ck = p->d_state == 16 || p->d_state == 8 || (!bf && p->d_state == 4);
        if (p->cu_seqlens || p->state_indices || !n_ck) return JAMBA_SSM_ERR_UNSUPPORTED;
        if (p->kernel_variant > 0 && !g_variants[p->kernel_variant - 1].kernel_fwd_ckpt)
            return JAMBA_SSM_ERR_UNSUPPORTED;
        if (!aligned(p->ckpt, 16)) return JAMBA_SSM_ERR_MISALIGNED;
    }
    const int64_t tok = token_rows(p);
    const int64_t state_rows = p->state_indices ? p->num_slots : p->batch;
    const size_t state_bytes = size_t(state_rows) * p->d_inner * p->d_state * 4;
    if (tok > 0) {
        if (!p->x || !p->delta || !p->z || !p->B || !p->C || !p->A || !p->out)
            return JAMBA_SSM_ERR_INVALID_ARG;
        if (!aligned(p->x, 16) || !aligned(p->delta, 16) || !aligned(p->z, 16) ||
            !aligned(p->B, 16) || !aligned(p->C, 16) || !aligned(p->out, 16) ||
            !aligned(p->A, 16) || !aligned(p->D, 4) || !aligned(p->delta_bias, 4) ||
            !aligned(p->h0, 16) || !aligned(p->h_final, 16))
            return JAMBA_SSM_ERR_MISALIGNED;
        const size_t act = size_t(tok) * p->d_inner * es, bc = size_t(tok) * p->d_state * es;
        const void *ins[] = {p->x, p->delta, p->z, p->B, p->C};
        const size_t insz[] = {act, act, act, bc, bc};
        for (int i = 0; i < 5; ++i)
            if (overlaps(p->out, act, ins[i], insz[i])) return JAMBA_SSM_ERR_INVALID_ARG;
        if (overlaps(p->h_final, state_bytes, p->out, act)) return JAMBA_SSM_ERR_INVALID_ARG;
        if (p->ckpt) {
            const size_t ckb = size_t(p->batch) * size_t((p->seqlen + jssm::kCk - 1) / jssm::kCk) *
                               p->d_inner * p->d_state * 4;
            const void *all[] = {p->x, p->delta, p->z, p->B, p->C, p->out, p->h0, p->h_final};
            const size_t allsz[] = {act, act, act, bc, bc, act, state_bytes, state_bytes};
            for (int i = 0; i < 8; ++i)
                if (overlaps(p->ckpt, ckb, all[i], allsz[i])) return JAMBA_SSM_ERR_INVALID_ARG;
        }
    } else if (p->batch > 0) {
        if (!aligned(p->h0, 16) || !aligned(p->h_final, 16)) return JAMBA_SSM_ERR_MISALIGNED;
    }
    if (p->h0 && p->h_final && p->h0 != p->h_final &&
        overlaps(p->h0, state_bytes, p->h_final, state_bytes))
        return JAMBA_SSM_ERR_INVALID_ARG;
    return JAMBA_SSM_OK;
}

struct ScanPlan {
    int variant;  // index into g_variants
    int grid;
    int64_t tasks;
};

jamba_ssm_status plan_scan(const jamba_ssm_scan_params *p, const DeviceInfo *dev, ScanPlan *plan) {
    if (small_state(p)) {  // one thread per (sequence, channel), no variant table
        const int64_t blocks = (p->d_inner + kSmallThreads - 1) / kSmallThreads;
        plan->variant = -1;
        plan->tasks = p->batch * blocks;
        plan->grid = static_cast<int>(plan->tasks < 1 ? 1 : (plan->tasks > 0x7fffffff ? 0x7fffffff
                                                                                    : plan->tasks));
        return JAMBA_SSM_OK;
    }
    const int vi = p->kernel_variant > 0 ? p->kernel_variant - 1
                                         : choose_variant(p, dev->sms, p->ckpt != nullptr);
    if (vi < 0) return JAMBA_SSM_ERR_UNSUPPORTED;
    const ScanVariant &v = g_variants[vi];
    const int cc = channels_per_cta(v);
    plan->variant = vi;
    plan->tasks = p->batch * ((p->d_inner + cc - 1) / cc);
    const int64_t g = plan->tasks < dev->sms ? plan->tasks : dev->sms;
    plan->grid = static_cast<int>(g < 1 ? 1 : g);
    return JAMBA_SSM_OK;
}

// ------------------------------------------------------------ backward pass
// Launch shape of the backward per (io dtype, d_state): G lanes per channel,
// NW compute warps, TT-step tiles (fp32 tiles are half as long so that the
// stage ring, the output tiles and the dB / dC partials fit in shared memory).
struct BwdShape {
    int g, nw, tt, cc;
};
bool bwd_shape(int io_dtype, int64_t n, BwdShape *s) {
    const bool bf = io_dtype == JAMBA_SSM_BF16;
    if (n == 16 || n == 8) *s = {4, 7, bf ? 64 : 32, 7 * 8};
    else if (n == 4 && !bf) *s = {2, 4, 32, 4 * 16};
    else return false;
    return true;
}

// Workspace of the backward: the status block, then the checkpoints, the
// per-CTA dB | dC partials and the per-sequence parameter partials.
struct BwdLayout {
    int64_t nck, ngroups;
    size_t off_ckpt, off_bc, off_par, total;
};
size_t round256(size_t v) { return (v + 255) & ~size_t(255); }
BwdLayout bwd_layout(int64_t batch, int64_t seqlen, int64_t d_inner, int64_t d_state, int cc) {
    BwdLayout l;
    l.nck = (seqlen + jssm::kCk - 1) / jssm::kCk;
    l.ngroups = (d_inner + cc - 1) / cc;
    l.off_ckpt = 256;
    l.off_bc = l.off_ckpt + round256(size_t(batch) * l.nck * d_inner * d_state * 4);
    l.off_par = l.off_bc + round256(size_t(batch) * l.ngroups * seqlen * 2 * d_state * 4);
    l.total = l.off_par + round256(size_t(batch) * d_inner * (d_state + 2) * 4);
    return l;
}

struct BwdKernels {
    const void *bwd, *reduce;
    int smem;
    bool attr[kMaxDevices];
};

template <typename IoT, int N, int G, int NW, int TT, bool SP>
BwdKernels make_bwd() {
    BwdKernels k{};
    k.bwd = reinterpret_cast<const void *>(&jssm::s6_bwd_kernel<IoT, N, G, NW, TT, SP>);
    k.reduce = reinterpret_cast<const void *>(&jssm::s6_bwd_reduce_kernel<IoT, N>);
    k.smem = jssm::BwdCfg<IoT, N, G, NW, TT>::kSmemBytes;
    return k;
}

// [dtype][d_state 16, 8, 4][softplus off, on]
BwdKernels g_bwd[2][3][2] = {
    {{make_bwd<__nv_bfloat16, 16, 4, 7, 64, false>(), make_bwd<__nv_bfloat16, 16, 4, 7, 64, true>()},
     {make_bwd<__nv_bfloat16, 8, 4, 7, 64, false>(), make_bwd<__nv_bfloat16, 8, 4, 7, 64, true>()},
     {BwdKernels{}, BwdKernels{}}},
    {{make_bwd<float, 16, 4, 7, 32, false>(), make_bwd<float, 16, 4, 7, 32, true>()},
     {make_bwd<float, 8, 4, 7, 32, false>(), make_bwd<float, 8, 4, 7, 32, true>()},
     {make_bwd<float, 4, 2, 4, 32, false>(), make_bwd<float, 4, 2, 4, 32, true>()}},
};

// ------------------------------------------------------- scalar-identity scan
// 4 lanes per channel and 4 compute warps: 32 channels of one head per CTA.
// (8 lanes and 8 warps, two states per lane, measured 264 against 215 us at
// batch 1 x 4096 tokens x 128 heads of 64: the butterfly's extra level costs
// more than the extra warps hide.)
constexpr int kSsdTT = 64, kSsdStages = 3, kSsdCC = 32;
struct SsdKernel {
    const void *k;
    int smem, threads;
    bool attr[kMaxDevices];
};
template <typename IoT, int N, bool SP>
SsdKernel make_ssd() {
    constexpr int G = 4, NW = 4;
    using Cfg = jssm::SsdCfg<IoT, N, G, NW, kSsdTT, kSsdStages>;
    static_assert(Cfg::CC == kSsdCC, "32 channels per CTA");
    SsdKernel k{};
    k.k = reinterpret_cast<const void *>(&jssm::s6_ssd_kernel<IoT, N, G, NW, kSsdTT, kSsdStages, SP>);
    k.smem = Cfg::kSmemBytes;
    k.threads = (NW + 1) * 32;
    return k;
}
// [dtype][d_state 16, 8][softplus off, on]
SsdKernel g_ssd[2][2][2] = {
    {{make_ssd<__nv_bfloat16, 16, false>(), make_ssd<__nv_bfloat16, 16, true>()},
     {make_ssd<__nv_bfloat16, 8, false>(), make_ssd<__nv_bfloat16, 8, true>()}},
    {{make_ssd<float, 16, false>(), make_ssd<float, 16, true>()},
     {make_ssd<float, 8, false>(), make_ssd<float, 8, true>()}},
};

// The chunked tensor-core form (bf16, d_state 16, headdim 64), softplus off / on.
struct SsdChunkKernel {
    const void *k;
    bool attr[kMaxDevices];
};
SsdChunkKernel g_ssd_chunk[2] = {
    {reinterpret_cast<const void *>(&jssm::s6_ssd_chunk_kernel<false>), {}},
    {reinterpret_cast<const void *>(&jssm::s6_ssd_chunk_kernel<true>), {}},
};

}  // namespace

extern "C" jamba_ssm_status jamba_ssm_get_status(void *workspace, void *stream);

namespace {

// After an enqueue: with JAMBA_SSM_SYNC_CHECK set (and not "0") in the
// environment -- a debugging aid, read once per process -- wait for the work
// and return any device-side condition it recorded (a timeout, a bad state
// slot) or launch error as this call's own status.
jamba_ssm_status finish_launch(cudaStream_t s, void *workspace) {
    static const bool sync_check = [] {
        const char *v = std::getenv("JAMBA_SSM_SYNC_CHECK");
        return v != nullptr && *v != '\0' && *v != '0';
    }();
    return sync_check ? jamba_ssm_get_status(workspace, s) : JAMBA_SSM_OK;
}

}  // namespace

extern "C" {

const char *jamba_ssm_status_string(jamba_ssm_status s) {
    switch (s) {
        case JAMBA_SSM_OK: return "ok";
        case JAMBA_SSM_ERR_INVALID_ARG: return "invalid argument";
        case JAMBA_SSM_ERR_UNSUPPORTED: return "unsupported size, dtype or variant";
        case JAMBA_SSM_ERR_MISALIGNED: return "misaligned pointer";
        case JAMBA_SSM_ERR_WORKSPACE: return "workspace too small";
        case JAMBA_SSM_ERR_CUDA: return "CUDA call failed";
        case JAMBA_SSM_ERR_TIMEOUT: return "device-side bounded wait ran out";
        case JAMBA_SSM_ERR_NO_DEVICE: return "no usable sm_100 device";
    }
    return "unknown status";
}

int jamba_ssm_last_cuda_error(void) { return t_last_cuda_error; }

int jamba_ssm_abi_version(void) { return JAMBA_SSM_ABI_VERSION; }

jamba_ssm_status jamba_ssm_scan_variant_info(int32_t k, int32_t *io_dtype, int32_t *d_state,
                                             int32_t *lanes_per_channel, int32_t *warps_per_cta,
                                             int32_t *time_tile) {
    if (k < 1 || k > kNumVariants) return JAMBA_SSM_ERR_UNSUPPORTED;
    const ScanVariant &v = g_variants[k - 1];
    if (io_dtype) *io_dtype = v.io_dtype;
    if (d_state) *d_state = v.n;
    if (lanes_per_channel) *lanes_per_channel = v.g;
    if (warps_per_cta) *warps_per_cta = v.threads / 32;
    if (time_tile) *time_tile = v.tt;
    return JAMBA_SSM_OK;
}

jamba_ssm_status jamba_ssm_scan_plan(const jamba_ssm_scan_params *pin, int32_t *variant,
                                     int32_t *lanes_per_channel, int32_t *channels_per_cta_out,
                                     int32_t *grid, int64_t *tasks) {
    jamba_ssm_scan_params prm;
    if (!read_params(pin, kScanParamsV1, &prm)) return JAMBA_SSM_ERR_INVALID_ARG;
    const jamba_ssm_scan_params *p = &prm;
    jamba_ssm_status st = validate_scan(p);
    if (st != JAMBA_SSM_OK) return st;
    const DeviceInfo *dev = current_device(&st);
    if (!dev) return st;
    ScanPlan plan;
    if ((st = plan_scan(p, dev, &plan)) != JAMBA_SSM_OK) return st;
    const bool small = plan.variant < 0;
    if (variant) *variant = plan.variant + 1;
    if (lanes_per_channel) *lanes_per_channel = small ? 1 : g_variants[plan.variant].g;
    if (channels_per_cta_out)
        *channels_per_cta_out = small ? kSmallThreads : channels_per_cta(g_variants[plan.variant]);
    if (grid) *grid = plan.grid;
    if (tasks) *tasks = plan.tasks;
    return JAMBA_SSM_OK;
}

jamba_ssm_status jamba_ssm_scan(const jamba_ssm_scan_params *pin, void *stream) {
    jamba_ssm_scan_params prm;
    if (!read_params(pin, kScanParamsV1, &prm)) return JAMBA_SSM_ERR_INVALID_ARG;
    const jamba_ssm_scan_params *p = &prm;
    jamba_ssm_status st = validate_scan(p);
    if (st != JAMBA_SSM_OK) return st;
    const DeviceInfo *dev = current_device(&st);
    if (!dev) return st;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const size_t state_bytes = size_t(p->batch) * p->d_inner * p->d_state * 4;
    if (p->batch == 0) return JAMBA_SSM_OK;
    const int64_t rows = token_rows(p);
    if (rows == 0) {  // no steps anywhere: every final state is its initial state
        if (!p->h_final) return JAMBA_SSM_OK;
        if (!p->state_indices) {
            cudaError_t e = p->h0 ? (p->h0 == p->h_final
                                         ? cudaSuccess
                                         : cudaMemcpyAsync(p->h_final, p->h0, state_bytes,
                                                           cudaMemcpyDeviceToDevice, s))
                                  : cudaMemsetAsync(p->h_final, 0, state_bytes, s);
            return e == cudaSuccess ? JAMBA_SSM_OK : cuda_fail(e);
        }
        const int64_t per = p->d_inner * p->d_state;
        const int64_t n = p->batch * per;
        const int threads = 256;
        const int64_t blocks = (n + threads - 1) / threads;
        if (blocks > 0x7fffffff) return JAMBA_SSM_ERR_UNSUPPORTED;
        jssm::s6_copy_states_kernel<<<static_cast<unsigned>(blocks), threads, 0, s>>>(
            p->batch, per, p->h0, p->h_final, p->state_indices, p->num_slots,
            static_cast<int *>(p->workspace));
        cudaError_t e = cudaGetLastError();
        return e == cudaSuccess ? finish_launch(s, p->workspace) : cuda_fail(e);
    }

    ScanArgs args{};
    args.batch = p->batch;
    args.seqlen = p->seqlen;
    args.d_inner = p->d_inner;
    args.A = p->A;
    args.D = p->D;
    args.delta_bias = p->delta_bias;
    args.h0 = p->h0;
    args.h_final = p->h_final;
    args.delta_softplus = p->delta_softplus != 0;
    args.debug_flags = p->debug_flags;
    args.timeout_cycles = p->timeout_cycles ? p->timeout_cycles : (uint64_t(1) << 31);
    args.cu_seqlens = p->cu_seqlens;
    args.total_tokens = p->total_tokens;
    args.state_indices = p->state_indices;
    args.num_slots = p->num_slots;
    args.out = p->out;
    args.status = static_cast<int *>(p->workspace);

    ScanPlan plan;
    if ((st = plan_scan(p, dev, &plan)) != JAMBA_SSM_OK) return st;
    if (plan.variant < 0) {  // small state: one thread per (sequence, channel)
        const dim3 grid(static_cast<unsigned>((p->d_inner + kSmallThreads - 1) / kSmallThreads),
                        static_cast<unsigned>(p->batch));
        constexpr int U = 8;  // steps per register block
        const void *k = nullptr;
        const bool bf = p->io_dtype == JAMBA_SSM_BF16;
        switch (p->d_state) {
            case 1: k = bf ? (const void *)&jssm::s6_scan_small_kernel<__nv_bfloat16, 1, U>
                           : (const void *)&jssm::s6_scan_small_kernel<float, 1, U>; break;
            case 2: k = bf ? (const void *)&jssm::s6_scan_small_kernel<__nv_bfloat16, 2, U>
                           : (const void *)&jssm::s6_scan_small_kernel<float, 2, U>; break;
            default: k = (const void *)&jssm::s6_scan_small_kernel<__nv_bfloat16, 4, U>; break;
        }
        const void *x = p->x, *dtp = p->delta, *z = p->z, *B = p->B, *C = p->C;
        void *kargs[] = {&args, &x, &dtp, &z, &B, &C};
        cudaError_t e = cudaLaunchKernel(k, grid, dim3(kSmallThreads), kargs, 0, s);
        return e == cudaSuccess ? finish_launch(s, p->workspace) : cuda_fail(e);
    }
    ScanVariant &v = g_variants[plan.variant];
    EncodeTiledFn fn = encode_fn(&st);
    if (!fn) return st;

    const int cc = channels_per_cta(v);
    const int es = p->io_dtype == JAMBA_SSM_BF16 ? 2 : 4;
    const CUtensorMapDataType dt =
        p->io_dtype == JAMBA_SSM_BF16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT32;
    // [batch][seqlen][channels], or the packed [1][total_tokens][channels]
    const int64_t dim_t = p->cu_seqlens ? p->total_tokens : p->seqlen;
    const int64_t dim_b = p->cu_seqlens ? 1 : p->batch;
    CUtensorMap maps[6];
    const void *act_ptrs[4] = {p->x, p->delta, p->z, p->out};
    const int act_idx[4] = {0, 1, 2, 5};
    for (int i = 0; i < 4; ++i)
        if (!encode_3d(fn, &maps[act_idx[i]], act_ptrs[i], dt, es, p->d_inner, dim_t, dim_b, cc, v.tt))
            return JAMBA_SSM_ERR_UNSUPPORTED;
    if (!encode_3d(fn, &maps[3], p->B, dt, es, p->d_state, dim_t, dim_b, (int)p->d_state, v.tt) ||
        !encode_3d(fn, &maps[4], p->C, dt, es, p->d_state, dim_t, dim_b, (int)p->d_state, v.tt))
        return JAMBA_SSM_ERR_UNSUPPORTED;

    // the serving kernel for packed sequences or cache slots, the batched one
    // storing checkpoints when asked, else the batched one
    const bool serving = p->cu_seqlens != nullptr || p->state_indices != nullptr;
    const bool with_ckpt = p->ckpt != nullptr;
    const void *kernel = serving ? v.kernel_serving : (with_ckpt ? v.kernel_fwd_ckpt : v.kernel);
    const int smem = serving ? v.smem_serving : v.smem;
    args.ckpt = p->ckpt;
    int devid = 0;
    cudaGetDevice(&devid);
    {
        std::lock_guard<std::mutex> lock(g_mutex);
        bool &set = serving ? v.attr_set_serving[devid]
                            : (with_ckpt ? v.attr_set_fwd_ckpt[devid] : v.attr_set[devid]);
        if (!set) {
            cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                                 smem);
            if (e != cudaSuccess) return cuda_fail(e);
            set = true;
        }
    }

    void *kargs[] = {&maps[0], &maps[1], &maps[2], &maps[3], &maps[4], &maps[5], &args};
    cudaError_t e = cudaLaunchKernel(kernel, dim3(plan.grid), dim3(v.threads), kargs,
                                     static_cast<size_t>(smem), s);
    if (e != cudaSuccess) return cuda_fail(e);
    return finish_launch(s, p->workspace);
}

jamba_ssm_status jamba_ssm_state_update(const jamba_ssm_state_update_params *pin, void *stream) {
    jamba_ssm_state_update_params prm;
    if (!read_params(pin, kUpdateParamsV1, &prm)) return JAMBA_SSM_ERR_INVALID_ARG;
    const jamba_ssm_state_update_params *p = &prm;
    if (p->batch < 0 || p->d_inner < 1 || p->d_state < 1) return JAMBA_SSM_ERR_INVALID_ARG;
    if (p->state_indices && p->num_slots < 1) return JAMBA_SSM_ERR_INVALID_ARG;
    if (p->num_slots > kMaxI32) return JAMBA_SSM_ERR_UNSUPPORTED;
    if (!aligned(p->state_indices, 4)) return JAMBA_SSM_ERR_MISALIGNED;
    if (p->io_dtype != JAMBA_SSM_BF16 && p->io_dtype != JAMBA_SSM_F32) return JAMBA_SSM_ERR_INVALID_ARG;
    if (p->d_state != 1 && p->d_state != 2 && p->d_state != 4 && p->d_state != 8 &&
        p->d_state != 16)
        return JAMBA_SSM_ERR_UNSUPPORTED;
    {
        const jamba_ssm_status ws = check_workspace(p->workspace, p->workspace_bytes);
        if (ws != JAMBA_SSM_OK) return ws;
    }
    if (p->batch > (int64_t(1) << 31) || p->d_inner > (int64_t(1) << 30)) return JAMBA_SSM_ERR_UNSUPPORTED;
    if (p->d_state < 4 && p->batch > 65535) return JAMBA_SSM_ERR_UNSUPPORTED;  // grid.y = requests
    if (p->batch == 0) return JAMBA_SSM_OK;
    if (!p->state || !p->x || !p->delta || !p->z || !p->B || !p->C || !p->A || !p->out)
        return JAMBA_SSM_ERR_INVALID_ARG;
    const int es = p->io_dtype == JAMBA_SSM_BF16 ? 2 : 4;
    const uintptr_t vec = p->d_state < 4 ? 4 : 16;  // the state / A / B / C vector width
    if (!aligned(p->state, vec) || !aligned(p->A, vec) || !aligned(p->B, p->d_state < 4 ? es : 16) ||
        !aligned(p->C, p->d_state < 4 ? es : 16) ||
        !aligned(p->x, es) || !aligned(p->delta, es) || !aligned(p->z, es) || !aligned(p->out, es) ||
        !aligned(p->D, 4) || !aligned(p->delta_bias, 4))
        return JAMBA_SSM_ERR_MISALIGNED;
    const size_t act = size_t(p->batch) * p->d_inner * es, bc = size_t(p->batch) * p->d_state * es;
    const size_t sb = size_t(p->state_indices ? p->num_slots : p->batch) * p->d_inner * p->d_state * 4;
    const void *ins[] = {p->x, p->delta, p->z, p->B, p->C, p->state};
    const size_t insz[] = {act, act, act, bc, bc, sb};
    for (int i = 0; i < 6; ++i)
        if (overlaps(p->out, act, ins[i], insz[i])) return JAMBA_SSM_ERR_INVALID_ARG;
    for (int i = 0; i < 5; ++i)
        if (overlaps(p->state, sb, ins[i], insz[i])) return JAMBA_SSM_ERR_INVALID_ARG;

    jamba_ssm_status st;
    const DeviceInfo *dev = current_device(&st);
    if (!dev) return st;

    UpdateArgs a{};
    a.batch = p->batch;
    a.d_inner = p->d_inner;
    a.state = p->state;
    a.x = p->x;
    a.delta = p->delta;
    a.z = p->z;
    a.B = p->B;
    a.C = p->C;
    a.A = p->A;
    a.D = p->D;
    a.delta_bias = p->delta_bias;
    a.out = p->out;
    a.delta_softplus = p->delta_softplus != 0;
    a.state_indices = p->state_indices;
    a.num_slots = p->num_slots;
    a.debug_flags = p->debug_flags;
    a.status = static_cast<int *>(p->workspace);
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const bool bf = p->io_dtype == JAMBA_SSM_BF16;
    if (p->d_state < 4) {  // one thread per (request, channel)
        const int64_t gx = (p->d_inner + kSmallThreads - 1) / kSmallThreads;
        const void *k = p->d_state == 1
                            ? (bf ? (const void *)&jssm::s6_state_update_small_kernel<__nv_bfloat16, 1>
                                  : (const void *)&jssm::s6_state_update_small_kernel<float, 1>)
                            : (bf ? (const void *)&jssm::s6_state_update_small_kernel<__nv_bfloat16, 2>
                                  : (const void *)&jssm::s6_state_update_small_kernel<float, 2>);
        void *kargs[] = {&a};
        cudaError_t e = cudaLaunchKernel(k, dim3(static_cast<unsigned>(gx), static_cast<unsigned>(p->batch)),
                                         dim3(kSmallThreads), kargs, 0, s);
        if (e != cudaSuccess) return cuda_fail(e);
        return finish_launch(s, p->workspace);
    }
    // Streaming kernel when every slice is a whole number of 16-byte chunks.
    const bool stream_ok = (p->d_inner * es) % 16 == 0 && (p->d_state * es) % 16 == 0 &&
                           aligned(p->x, 16) && aligned(p->delta, 16) && aligned(p->z, 16);
    if (stream_ok) {
        constexpr int kCPB = 32, kBPC = 16, kS = 8;
        const int64_t gx = (p->d_inner + kCPB - 1) / kCPB, gy = (p->batch + kBPC - 1) / kBPC;
        if (gx > 0x7fffffff || gy > 65535) return JAMBA_SSM_ERR_UNSUPPORTED;
        const void *k = nullptr;
        int threads = 0, smem = 0;
#define JSSM_STREAM(T, NN)                                                                    \
    do {                                                                                      \
        k = p->state_indices                                                                  \
                ? (const void *)&jssm::s6_state_update_stream_kernel<T, NN, kCPB, kBPC, kS, true> \
                : (const void *)&jssm::s6_state_update_stream_kernel<T, NN, kCPB, kBPC, kS, false>; \
        threads = jssm::UpdateCfg<T, NN, kCPB, kS>::kThreads;                                 \
        smem = jssm::UpdateCfg<T, NN, kCPB, kS>::kSmemBytes;                                  \
    } while (0)
        switch (p->d_state) {
            case 4: JSSM_STREAM(float, 4); break;  // bf16 rows of 4 states are not 16 bytes
            case 8: if (bf) JSSM_STREAM(__nv_bfloat16, 8); else JSSM_STREAM(float, 8); break;
            default: if (bf) JSSM_STREAM(__nv_bfloat16, 16); else JSSM_STREAM(float, 16); break;
        }
#undef JSSM_STREAM
        uint64_t limit = p->timeout_cycles ? p->timeout_cycles : (uint64_t(1) << 31);
        void *kargs[] = {&a, &limit};
        cudaError_t e = cudaLaunchKernel(k, dim3(static_cast<unsigned>(gx), static_cast<unsigned>(gy)),
                                         dim3(threads), kargs, static_cast<size_t>(smem), s);
        if (e != cudaSuccess) return cuda_fail(e);
        return finish_launch(s, p->workspace);
    }
    constexpr int kBPC = 2;  // requests per block (parameters reused across them)
    const int64_t cpb = 256 / (p->d_state / 4);
    const int64_t gx = (p->d_inner + cpb - 1) / cpb, gy = (p->batch + kBPC - 1) / kBPC;
    if (gx > 0x7fffffff || gy > 65535) return JAMBA_SSM_ERR_UNSUPPORTED;
    const void *k = nullptr;
    switch (p->d_state) {
        case 4: k = bf ? (const void *)&jssm::s6_state_update_kernel<__nv_bfloat16, 4, kBPC>
                       : (const void *)&jssm::s6_state_update_kernel<float, 4, kBPC>; break;
        case 8: k = bf ? (const void *)&jssm::s6_state_update_kernel<__nv_bfloat16, 8, kBPC>
                       : (const void *)&jssm::s6_state_update_kernel<float, 8, kBPC>; break;
        default: k = bf ? (const void *)&jssm::s6_state_update_kernel<__nv_bfloat16, 16, kBPC>
                        : (const void *)&jssm::s6_state_update_kernel<float, 16, kBPC>; break;
    }
    void *kargs[] = {&a};
    cudaError_t e = cudaLaunchKernel(k, dim3(static_cast<unsigned>(gx), static_cast<unsigned>(gy)),
                                     dim3(256), kargs, 0, s);
    if (e != cudaSuccess) return cuda_fail(e);
    return finish_launch(s, p->workspace);
}

jamba_ssm_status jamba_ssm_get_status(void *workspace, void *stream) {
    jamba_ssm_status st;
    if (!current_device(&st)) return st;
    if (!aligned(workspace, 16)) return JAMBA_SSM_ERR_MISALIGNED;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    cudaError_t e = cudaStreamSynchronize(s);
    if (e != cudaSuccess) return cuda_fail(e);
    int word = 0;
    e = workspace ? cudaMemcpy(&word, workspace, sizeof(int), cudaMemcpyDeviceToHost)
                  : cudaMemcpyFromSymbol(&word, jssm::g_status_word, sizeof(int));
    if (e != cudaSuccess) return cuda_fail(e);
    if (word != 0) {
        const int zero = 0;
        e = workspace ? cudaMemcpy(workspace, &zero, sizeof(int), cudaMemcpyHostToDevice)
                      : cudaMemcpyToSymbol(jssm::g_status_word, &zero, sizeof(int));
        if (e != cudaSuccess) return cuda_fail(e);
    }
    return static_cast<jamba_ssm_status>(word);
}

size_t jamba_ssm_scan_bwd_workspace_size(int64_t batch, int64_t seqlen, int64_t d_inner,
                                         int64_t d_state) {
    BwdShape sh;
    if (batch < 0 || seqlen < 0 || d_inner < 1 || !bwd_shape(JAMBA_SSM_F32, d_state, &sh))
        return 0;
    // the layout depends on the channel-group width, which is the same for
    // both dtypes at a given d_state
    return bwd_layout(batch, seqlen, d_inner, d_state, sh.cc).total;
}

size_t jamba_ssm_scan_ckpt_size(int64_t batch, int64_t seqlen, int64_t d_inner, int64_t d_state) {
    if (batch < 0 || seqlen < 0 || d_inner < 0 || d_state < 0) return 0;
    return size_t(batch) * size_t((seqlen + jssm::kCk - 1) / jssm::kCk) * size_t(d_inner) *
           size_t(d_state) * 4;
}

jamba_ssm_status jamba_ssm_scan_bwd(const jamba_ssm_scan_bwd_params *pin, void *stream) {
    jamba_ssm_scan_bwd_params prm;
    if (!read_params(pin, kBwdParamsV3, &prm)) return JAMBA_SSM_ERR_INVALID_ARG;
    const jamba_ssm_scan_bwd_params *p = &prm;
    if (p->batch < 0 || p->seqlen < 0 || p->d_inner < 1 || p->d_state < 1)
        return JAMBA_SSM_ERR_INVALID_ARG;
    if (p->io_dtype != JAMBA_SSM_BF16 && p->io_dtype != JAMBA_SSM_F32) return JAMBA_SSM_ERR_INVALID_ARG;
    BwdShape sh;
    const int es = p->io_dtype == JAMBA_SSM_BF16 ? 2 : 4;
    if (!bwd_shape(p->io_dtype, p->d_state, &sh) || (p->d_inner * es) % 16 != 0)
        return JAMBA_SSM_ERR_UNSUPPORTED;
    const int64_t kMaxRows = kMaxI32 - 256;
    if (p->batch > 65535 || p->seqlen > kMaxRows || p->d_inner > (int64_t(1) << 30) ||
        (p->batch && p->seqlen && p->batch > kMaxElems / p->seqlen) ||
        p->batch * p->seqlen > kMaxElems / p->d_inner)
        return JAMBA_SSM_ERR_UNSUPPORTED;
    if (!p->workspace) return JAMBA_SSM_ERR_INVALID_ARG;
    if (!aligned(p->workspace, 16)) return JAMBA_SSM_ERR_MISALIGNED;
    const BwdLayout lay = bwd_layout(p->batch, p->seqlen, p->d_inner, p->d_state, sh.cc);
    if (p->workspace_bytes < lay.total) return JAMBA_SSM_ERR_WORKSPACE;
    const int64_t tok = p->batch * p->seqlen;
    const size_t act = size_t(tok) * p->d_inner * es, bc = size_t(tok) * p->d_state * es;
    const size_t st = size_t(p->batch) * p->d_inner * p->d_state * 4;
    const size_t pn = size_t(p->d_inner) * 4, an = size_t(p->d_inner) * p->d_state * 4;
    if (tok > 0) {
        if (!p->x || !p->delta || !p->z || !p->B || !p->C || !p->A || !p->dout || !p->dx ||
            !p->ddelta || !p->dz || !p->dB || !p->dC)
            return JAMBA_SSM_ERR_INVALID_ARG;
        const void *a16[] = {p->x, p->delta, p->z, p->B, p->C, p->A, p->dout, p->dx, p->ddelta,
                             p->dz, p->dB, p->dC, p->h0, p->dh_final, p->dh0};
        for (const void *q : a16)
            if (!aligned(q, 16)) return JAMBA_SSM_ERR_MISALIGNED;
    }
    if (!aligned(p->D, 4) || !aligned(p->delta_bias, 4) || !aligned(p->dA, 4) ||
        !aligned(p->dD, 4) || !aligned(p->ddelta_bias, 4) || !aligned(p->h0, 4) ||
        !aligned(p->dh_final, 4) || !aligned(p->dh0, 4) || !aligned(p->ckpt, 16))
        return JAMBA_SSM_ERR_MISALIGNED;
    // no output may overlap an input, another output or the workspace
    const void *outs[] = {p->dx, p->ddelta, p->dz, p->dB, p->dC, p->dA, p->dD, p->ddelta_bias,
                          p->dh0};
    const size_t outsz[] = {act, act, act, bc, bc, an, pn, pn, st};
    const size_t ckb = size_t(p->batch) * size_t(lay.nck) * p->d_inner * p->d_state * 4;
    const void *ins[] = {p->x,  p->delta, p->z,        p->B,         p->C,
                         p->A,  p->D,     p->delta_bias, p->h0,      p->dout,
                         p->dh_final, p->workspace, p->ckpt};
    const size_t insz[] = {act, act, act, bc, bc, an, pn, pn, st, act, st, lay.total, ckb};
    for (int i = 0; i < 9; ++i) {
        for (int j = 0; j < 13; ++j)
            if (overlaps(outs[i], outsz[i], ins[j], insz[j])) return JAMBA_SSM_ERR_INVALID_ARG;
        for (int j = i + 1; j < 9; ++j)
            if (overlaps(outs[i], outsz[i], outs[j], outsz[j])) return JAMBA_SSM_ERR_INVALID_ARG;
    }
    jamba_ssm_status stt;
    const DeviceInfo *dev = current_device(&stt);
    if (!dev) return stt;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    int *status = static_cast<int *>(p->workspace);
    uint8_t *ws = static_cast<uint8_t *>(p->workspace);
    cudaError_t e;
    if (tok == 0) {  // no steps: the parameter gradients are zero and dh0 = dh_final
        if (p->dA && (e = cudaMemsetAsync(p->dA, 0, an, s)) != cudaSuccess) return cuda_fail(e);
        if (p->dD && (e = cudaMemsetAsync(p->dD, 0, pn, s)) != cudaSuccess) return cuda_fail(e);
        if (p->ddelta_bias && (e = cudaMemsetAsync(p->ddelta_bias, 0, pn, s)) != cudaSuccess)
            return cuda_fail(e);
        if (p->dh0 && st) {
            e = p->dh_final ? cudaMemcpyAsync(p->dh0, p->dh_final, st, cudaMemcpyDeviceToDevice, s)
                            : cudaMemsetAsync(p->dh0, 0, st, s);
            if (e != cudaSuccess) return cuda_fail(e);
        }
        return finish_launch(s, p->workspace);
    }
    const int di = p->io_dtype == JAMBA_SSM_BF16 ? 0 : 1;
    const int ni = p->d_state == 16 ? 0 : (p->d_state == 8 ? 1 : 2);
    BwdKernels &K = g_bwd[di][ni][p->delta_softplus ? 1 : 0];
    EncodeTiledFn fn = encode_fn(&stt);
    if (!fn) return stt;
    int devid = 0;
    cudaGetDevice(&devid);
    {
        std::lock_guard<std::mutex> lock(g_mutex);
        if (!K.attr[devid]) {
            e = cudaFuncSetAttribute(K.bwd, cudaFuncAttributeMaxDynamicSharedMemorySize, K.smem);
            if (e != cudaSuccess) return cuda_fail(e);
            K.attr[devid] = true;
        }
    }
    jssm::BwdArgs a{};
    a.batch = p->batch;
    a.seqlen = p->seqlen;
    a.d_inner = p->d_inner;
    a.A = p->A;
    a.D = p->D;
    a.delta_bias = p->delta_bias;
    a.h0 = p->h0;
    a.dh_final = p->dh_final;
    a.delta_softplus = p->delta_softplus != 0;
    // the forward's checkpoints when the caller has them, else this call's own
    float *ckpt = reinterpret_cast<float *>(ws + lay.off_ckpt);
    a.ckpt = p->ckpt ? p->ckpt : ckpt;
    a.part_bc = reinterpret_cast<float *>(ws + lay.off_bc);
    a.part_par = reinterpret_cast<float *>(ws + lay.off_par);
    a.dh0 = p->dh0;
    a.status = status;
    a.debug_flags = p->debug_flags;
    a.timeout_cycles = p->timeout_cycles ? p->timeout_cycles : (uint64_t(1) << 31);

    const CUtensorMapDataType dt = p->io_dtype == JAMBA_SSM_BF16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16
                                                                 : CU_TENSOR_MAP_DATA_TYPE_FLOAT32;
    // 1. checkpoints (unless the caller passed the forward's): the forward
    //    kernel in its checkpoint mode, the variant the forward's cost model
    //    picks for this shape
    if (!p->ckpt) {
        jamba_ssm_scan_params fp{};
        fp.struct_size = sizeof(fp);
        fp.batch = p->batch;
        fp.seqlen = p->seqlen;
        fp.d_inner = p->d_inner;
        fp.d_state = p->d_state;
        fp.io_dtype = p->io_dtype;
        const int vi = choose_variant(&fp, dev->sms, true);
        if (vi < 0) return JAMBA_SSM_ERR_UNSUPPORTED;
        ScanVariant &v = g_variants[vi];
        const int cc = channels_per_cta(v);
        CUtensorMap maps[6];
        if (!encode_3d(fn, &maps[0], p->x, dt, es, p->d_inner, p->seqlen, p->batch, cc, v.tt) ||
            !encode_3d(fn, &maps[1], p->delta, dt, es, p->d_inner, p->seqlen, p->batch, cc, v.tt) ||
            !encode_3d(fn, &maps[3], p->B, dt, es, p->d_state, p->seqlen, p->batch, (int)p->d_state,
                       v.tt))
            return JAMBA_SSM_ERR_UNSUPPORTED;
        maps[2] = maps[0];  // z, C and the output are not read or written in this mode
        maps[4] = maps[3];
        maps[5] = maps[0];
        {
            std::lock_guard<std::mutex> lock(g_mutex);
            if (!v.attr_set_ckpt[devid]) {
                e = cudaFuncSetAttribute(v.kernel_ckpt, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         v.smem);
                if (e != cudaSuccess) return cuda_fail(e);
                v.attr_set_ckpt[devid] = true;
            }
        }
        jssm::ScanArgs fa{};
        fa.batch = p->batch;
        fa.seqlen = p->seqlen;
        fa.d_inner = p->d_inner;
        fa.A = p->A;
        fa.delta_bias = p->delta_bias;
        fa.h0 = p->h0;
        fa.delta_softplus = p->delta_softplus != 0;
        fa.debug_flags = p->debug_flags;
        fa.timeout_cycles = a.timeout_cycles;
        fa.status = status;
        fa.ckpt = ckpt;
        const int64_t tasks = p->batch * ((p->d_inner + cc - 1) / cc);
        const int grid = static_cast<int>(tasks < dev->sms ? tasks : dev->sms);
        void *kargs[] = {&maps[0], &maps[1], &maps[2], &maps[3], &maps[4], &maps[5], &fa};
        e = cudaLaunchKernel(v.kernel_ckpt, dim3(grid < 1 ? 1 : grid), dim3(v.threads), kargs,
                             static_cast<size_t>(v.smem), s);
        if (e != cudaSuccess) return cuda_fail(e);
    }
    // 2. the reverse walk
    {
        jssm::BwdMaps m;
        CUtensorMap *acts[] = {&m.x, &m.dt, &m.z, &m.dout, &m.dx, &m.ddt, &m.dz};
        const void *aptr[] = {p->x, p->delta, p->z, p->dout, p->dx, p->ddelta, p->dz};
        for (int i = 0; i < 7; ++i)
            if (!encode_3d(fn, acts[i], aptr[i], dt, es, p->d_inner, p->seqlen, p->batch, sh.cc, sh.tt))
                return JAMBA_SSM_ERR_UNSUPPORTED;
        if (!encode_3d(fn, &m.B, p->B, dt, es, p->d_state, p->seqlen, p->batch, (int)p->d_state, sh.tt) ||
            !encode_3d(fn, &m.C, p->C, dt, es, p->d_state, p->seqlen, p->batch, (int)p->d_state, sh.tt))
            return JAMBA_SSM_ERR_UNSUPPORTED;
        const dim3 grid(static_cast<unsigned>(lay.ngroups), static_cast<unsigned>(p->batch));
        void *kargs[] = {&m, &a};
        e = cudaLaunchKernel(K.bwd, grid, dim3((sh.nw + 1) * 32), kargs, static_cast<size_t>(K.smem), s);
        if (e != cudaSuccess) return cuda_fail(e);
    }
    // 3. sums over CTAs and sequences
    {
        const int64_t total = tok * 2 * p->d_state + p->d_inner * (p->d_state + 2);
        int64_t blocks = (total + 255) / 256;
        if (blocks > int64_t(dev->sms) * 16) blocks = int64_t(dev->sms) * 16;
        const float *pbc = a.part_bc, *ppar = a.part_par;
        int64_t batch = p->batch, seqlen = p->seqlen, d_inner = p->d_inner, ng = lay.ngroups;
        void *dB = p->dB, *dC = p->dC;
        float *dA = p->dA, *dD = p->dD, *db = p->ddelta_bias;
        void *kargs[] = {&pbc, &ppar, &batch, &seqlen, &d_inner, &ng, &dB, &dC, &dA, &dD, &db};
        e = cudaLaunchKernel(K.reduce, dim3(static_cast<unsigned>(blocks)), dim3(256), kargs, 0, s);
        if (e != cudaSuccess) return cuda_fail(e);
    }
    return finish_launch(s, p->workspace);
}

jamba_ssm_status jamba_ssm_ssd_scan(const jamba_ssm_ssd_params *p, void *stream) {
    if (!p || p->struct_size < sizeof(jamba_ssm_ssd_params)) return JAMBA_SSM_ERR_INVALID_ARG;
    if (p->batch < 0 || p->seqlen < 0 || p->nheads < 1 || p->headdim < 1 || p->d_state < 1)
        return JAMBA_SSM_ERR_INVALID_ARG;
    if (p->io_dtype != JAMBA_SSM_BF16 && p->io_dtype != JAMBA_SSM_F32) return JAMBA_SSM_ERR_INVALID_ARG;
    const int es = p->io_dtype == JAMBA_SSM_BF16 ? 2 : 4;
    if ((p->d_state != 8 && p->d_state != 16) || p->headdim % kSsdCC != 0 ||
        (p->nheads * es) % 16 != 0)
        return JAMBA_SSM_ERR_UNSUPPORTED;
    const int64_t D = p->nheads * p->headdim;
    const int64_t kMaxRows = kMaxI32 - 256;
    if (p->batch > 65535 || p->seqlen > kMaxRows || D > (int64_t(1) << 30) ||
        (p->batch && p->seqlen && p->batch > kMaxElems / p->seqlen) ||
        p->batch * p->seqlen > kMaxElems / D)
        return JAMBA_SSM_ERR_UNSUPPORTED;
    {
        const jamba_ssm_status ws = check_workspace(p->workspace, p->workspace_bytes);
        if (ws != JAMBA_SSM_OK) return ws;
    }
    const int64_t tok = p->batch * p->seqlen;
    const size_t act = size_t(tok) * D * es, dts = size_t(tok) * p->nheads * es;
    const size_t bc = size_t(tok) * p->d_state * es, st = size_t(p->batch) * D * p->d_state * 4;
    if (tok > 0) {
        if (!p->x || !p->delta || !p->z || !p->B || !p->C || !p->A || !p->out)
            return JAMBA_SSM_ERR_INVALID_ARG;
        const void *a16[] = {p->x, p->delta, p->z, p->B, p->C, p->out, p->h0, p->h_final};
        for (const void *q : a16)
            if (!aligned(q, 16)) return JAMBA_SSM_ERR_MISALIGNED;
        const void *ins[] = {p->x, p->delta, p->z, p->B, p->C};
        const size_t insz[] = {act, dts, act, bc, bc};
        for (int i = 0; i < 5; ++i)
            if (overlaps(p->out, act, ins[i], insz[i])) return JAMBA_SSM_ERR_INVALID_ARG;
        if (overlaps(p->h_final, st, p->out, act)) return JAMBA_SSM_ERR_INVALID_ARG;
    }
    if (!aligned(p->A, 4) || !aligned(p->D, 4) || !aligned(p->delta_bias, 4) ||
        !aligned(p->h0, 16) || !aligned(p->h_final, 16))
        return JAMBA_SSM_ERR_MISALIGNED;
    if (p->h0 && p->h_final && p->h0 != p->h_final && overlaps(p->h0, st, p->h_final, st))
        return JAMBA_SSM_ERR_INVALID_ARG;
    jamba_ssm_status stt;
    const DeviceInfo *dev = current_device(&stt);
    if (!dev) return stt;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (p->batch == 0) return JAMBA_SSM_OK;
    if (tok == 0) {  // no steps: the final state is the initial state
        if (!p->h_final || p->h0 == p->h_final) return JAMBA_SSM_OK;
        cudaError_t e = p->h0 ? cudaMemcpyAsync(p->h_final, p->h0, st, cudaMemcpyDeviceToDevice, s)
                              : cudaMemsetAsync(p->h_final, 0, st, s);
        return e == cudaSuccess ? finish_launch(s, p->workspace) : cuda_fail(e);
    }
    EncodeTiledFn fn = encode_fn(&stt);
    if (!fn) return stt;
    int devid = 0;
    cudaGetDevice(&devid);
    const uint64_t timeout = p->timeout_cycles ? p->timeout_cycles : (uint64_t(1) << 31);
    if (p->io_dtype == JAMBA_SSM_BF16 && p->d_state == 16 && p->headdim % jssm::SsdChunkCfg::P == 0 &&
        !(p->debug_flags & 2u)) {
        // chunked form on the tensor cores: one CTA per (sequence, 64-channel
        // slice of a head)
        using CC = jssm::SsdChunkCfg;
        const CUtensorMapDataType bf = CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
        jssm::SsdChunkMaps m;
        if (!encode_3d(fn, &m.x, p->x, bf, 2, D, p->seqlen, p->batch, CC::P, CC::Q,
                       CU_TENSOR_MAP_SWIZZLE_128B) ||
            !encode_3d(fn, &m.z, p->z, bf, 2, D, p->seqlen, p->batch, CC::P, CC::Q,
                       CU_TENSOR_MAP_SWIZZLE_128B) ||
            !encode_3d(fn, &m.B, p->B, bf, 2, CC::N, p->seqlen, p->batch, CC::N, CC::Q,
                       CU_TENSOR_MAP_SWIZZLE_32B) ||
            !encode_3d(fn, &m.C, p->C, bf, 2, CC::N, p->seqlen, p->batch, CC::N, CC::Q,
                       CU_TENSOR_MAP_SWIZZLE_32B))
            return JAMBA_SSM_ERR_UNSUPPORTED;
        SsdChunkKernel &K = g_ssd_chunk[p->delta_softplus ? 1 : 0];
        {
            std::lock_guard<std::mutex> lock(g_mutex);
            if (!K.attr[devid]) {
                cudaError_t e = cudaFuncSetAttribute(K.k, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                                     static_cast<int>(CC::kSmemBytes));
                if (e != cudaSuccess) return cuda_fail(e);
                K.attr[devid] = true;
            }
        }
        jssm::SsdChunkArgs a{};
        a.seqlen = p->seqlen;
        a.nheads = p->nheads;
        a.headdim = p->headdim;
        a.delta = static_cast<const __nv_bfloat16 *>(p->delta);
        a.A = p->A;
        a.D = p->D;
        a.delta_bias = p->delta_bias;
        a.h0 = p->h0;
        a.h_final = p->h_final;
        a.out = static_cast<__nv_bfloat16 *>(p->out);
        a.status = static_cast<int *>(p->workspace);
        a.debug_flags = p->debug_flags;
        a.timeout_cycles = timeout;
        const dim3 grid(static_cast<unsigned>(D / CC::P), static_cast<unsigned>(p->batch));
        void *kargs[] = {&m, &a};
        cudaError_t e = cudaLaunchKernel(K.k, grid, dim3(CC::kThreads), kargs,
                                         static_cast<size_t>(CC::kSmemBytes), s);
        if (e != cudaSuccess) return cuda_fail(e);
        return finish_launch(s, p->workspace);
    }
    SsdKernel &K = g_ssd[p->io_dtype == JAMBA_SSM_BF16 ? 0 : 1][p->d_state == 16 ? 0 : 1]
                        [p->delta_softplus ? 1 : 0];
    const CUtensorMapDataType dt =
        p->io_dtype == JAMBA_SSM_BF16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT32;
    jssm::SsdMaps m;
    if (!encode_3d(fn, &m.x, p->x, dt, es, D, p->seqlen, p->batch, kSsdCC, kSsdTT) ||
        !encode_3d(fn, &m.z, p->z, dt, es, D, p->seqlen, p->batch, kSsdCC, kSsdTT) ||
        !encode_3d(fn, &m.out, p->out, dt, es, D, p->seqlen, p->batch, kSsdCC, kSsdTT) ||
        !encode_3d(fn, &m.dt, p->delta, dt, es, p->nheads, p->seqlen, p->batch, 16 / es, kSsdTT) ||
        !encode_3d(fn, &m.B, p->B, dt, es, p->d_state, p->seqlen, p->batch, (int)p->d_state, kSsdTT) ||
        !encode_3d(fn, &m.C, p->C, dt, es, p->d_state, p->seqlen, p->batch, (int)p->d_state, kSsdTT))
        return JAMBA_SSM_ERR_UNSUPPORTED;
    {
        std::lock_guard<std::mutex> lock(g_mutex);
        if (!K.attr[devid]) {
            cudaError_t e = cudaFuncSetAttribute(K.k, cudaFuncAttributeMaxDynamicSharedMemorySize, K.smem);
            if (e != cudaSuccess) return cuda_fail(e);
            K.attr[devid] = true;
        }
    }
    jssm::SsdArgs a{};
    a.batch = p->batch;
    a.seqlen = p->seqlen;
    a.nheads = p->nheads;
    a.headdim = p->headdim;
    a.A = p->A;
    a.D = p->D;
    a.delta_bias = p->delta_bias;
    a.h0 = p->h0;
    a.h_final = p->h_final;
    a.delta_softplus = p->delta_softplus != 0;
    a.status = static_cast<int *>(p->workspace);
    a.debug_flags = p->debug_flags;
    a.timeout_cycles = timeout;
    const dim3 grid(static_cast<unsigned>(D / kSsdCC), static_cast<unsigned>(p->batch));
    void *kargs[] = {&m, &a};
    cudaError_t e = cudaLaunchKernel(K.k, grid, dim3(K.threads), kargs,
                                     static_cast<size_t>(K.smem), s);
    if (e != cudaSuccess) return cuda_fail(e);
    return finish_launch(s, p->workspace);
}

size_t jamba_ssm_scan_workspace_size(int64_t batch, int64_t seqlen, int64_t d_inner,
                                     int64_t d_state) {
    // Only the status word: every lane carries its channel's states through the
    // whole sequence in registers, so no carry between chunks of the sequence
    // is ever stored, whatever the sizes.
    (void)batch;
    (void)seqlen;
    (void)d_inner;
    (void)d_state;
    return JAMBA_SSM_STATUS_BYTES;
}

}  // extern "C"

// ------------------------------------------- backward without a caller workspace
// Some callers cannot allocate device memory where they run the backward pass:
// a plug-in whose host framework owns every device allocation and fixes its
// memory plan before the run, or code on a path where cudaMalloc's implicit
// device synchronisation is not acceptable.  jamba_ssm_scan_bwd_noalloc serves
// them with scratch the library owns: this array, reserved in every device's
// memory when the library's module is loaded and kept until the process exits.
static __device__ __align__(256) uint8_t g_bwd_noalloc_scratch[JAMBA_SSM_BWD_NOALLOC_SCRATCH_BYTES];

namespace {

// Device address of the array above on each device.  In host code the
// array's name only stands in for the symbol (it is not a device address), so
// the address is looked up once per device, with that device current.
void *g_noalloc_ptr[kMaxDevices];

// Moves a condition the backward recorded in the scratch's status word into
// the library's per-device word, where jamba_ssm_get_status(NULL, ...) reads it.
__global__ void s6_noalloc_status_kernel(const int *word) {
    const int w = *word;
    if (w != 0) atomicCAS(&jssm::g_status_word, 0, w);
}

}  // namespace

extern "C" jamba_ssm_status jamba_ssm_scan_bwd_noalloc(const jamba_ssm_scan_bwd_params *pin,
                                                       void *stream) {
    jamba_ssm_scan_bwd_params q;  // an ABI version 3 caller's struct reads with ckpt NULL
    if (!read_params(pin, kBwdParamsV3, &q)) return JAMBA_SSM_ERR_INVALID_ARG;
    if (q.workspace || q.workspace_bytes) return JAMBA_SSM_ERR_INVALID_ARG;
    const size_t need = jamba_ssm_scan_bwd_workspace_size(q.batch, q.seqlen, q.d_inner, q.d_state);
    if (need == 0)  // sizes the backward does not take
        return (q.batch < 0 || q.seqlen < 0 || q.d_inner < 1 || q.d_state < 1)
                   ? JAMBA_SSM_ERR_INVALID_ARG
                   : JAMBA_SSM_ERR_UNSUPPORTED;
    if (need > JAMBA_SSM_BWD_NOALLOC_SCRATCH_BYTES) return JAMBA_SSM_ERR_WORKSPACE;
    jamba_ssm_status st;
    if (!current_device(&st)) return st;
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return cuda_fail(e);
    void *scratch = nullptr;
    {
        std::lock_guard<std::mutex> lock(g_mutex);
        if (!g_noalloc_ptr[dev]) {  // set-up, once per device, on this call
            void *ptr = nullptr;
            e = cudaGetSymbolAddress(&ptr, g_bwd_noalloc_scratch);
            if (e != cudaSuccess || !ptr) return cuda_fail(e != cudaSuccess ? e : cudaErrorInvalidSymbol);
            g_noalloc_ptr[dev] = ptr;
        }
        scratch = g_noalloc_ptr[dev];
    }
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    // the array keeps the previous call's contents; only its status word has to
    // start at zero (every other part is written before it is read)
    e = cudaMemsetAsync(scratch, 0, JAMBA_SSM_STATUS_BYTES, s);
    if (e != cudaSuccess) return cuda_fail(e);
    q.struct_size = sizeof(q);
    q.workspace = scratch;
    q.workspace_bytes = JAMBA_SSM_BWD_NOALLOC_SCRATCH_BYTES;
    st = jamba_ssm_scan_bwd(&q, stream);
    if (st != JAMBA_SSM_OK) return st;
    s6_noalloc_status_kernel<<<1, 1, 0, s>>>(static_cast<const int *>(scratch));
    e = cudaGetLastError();
    return e == cudaSuccess ? JAMBA_SSM_OK : cuda_fail(e);
}
