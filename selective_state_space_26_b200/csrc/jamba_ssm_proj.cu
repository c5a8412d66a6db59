// jamba_ssm_proj.cu -- host side of the C ABI declared in
// include/jamba_ssm_proj.h: argument validation, TMA tensor-map encoding and
// the launches of the x_proj and dt_proj kernels.  Nothing here allocates device memory.
// Built as its own library, so its kernels and status word form a module of
// their own.
#include <cuda.h>
#include <cuda_runtime.h>

#include <cstddef>
#include <cstdlib>
#include <cstring>
#include <mutex>

#include "jamba_ssm_proj.h"
#include "s6_dt_proj.cuh"
#include "s6_x_proj.cuh"

#define JSSM_PROJ_API extern "C" __attribute__((visibility("default")))

namespace {

thread_local int t_last_cuda_error = 0;

jamba_ssm_status cuda_fail(cudaError_t e) {
    t_last_cuda_error = static_cast<int>(e);
    return JAMBA_SSM_ERR_CUDA;
}

constexpr int kMaxDevices = 64;
struct DeviceState {
    bool ready = false;
    bool usable = false;
    bool dt_attr = false;   // s6_dt_proj_kernel's shared-memory limit is set
    bool dtp_attr = false;  // s6_dt_proj_persistent_kernel's
    bool x_attr = false;   // s6_x_proj_kernel's
    int sms = 0;
};
DeviceState g_devices[kMaxDevices];
std::mutex g_mutex;

// Checks that the current device is an sm_100 part and, once per device and
// kernel, raises `kernel`'s dynamic shared-memory limit to `smem` bytes (the
// flag `attr_done` selects which kernel's record).  *sms receives the SM count.
jamba_ssm_status prepare_device(const void *kernel, int smem, bool DeviceState::*attr_done,
                                int *sms = nullptr) {
    int dev = -1;
    cudaError_t e = cudaGetDevice(&dev);
    if (e == cudaErrorNoDevice || e == cudaErrorInsufficientDriver) return JAMBA_SSM_ERR_NO_DEVICE;
    if (e != cudaSuccess) return cuda_fail(e);
    if (dev < 0 || dev >= kMaxDevices) return JAMBA_SSM_ERR_NO_DEVICE;
    std::lock_guard<std::mutex> lock(g_mutex);
    DeviceState &d = g_devices[dev];
    if (!d.ready) {
        int major = 0, minor = 0;
        if ((e = cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev)) != cudaSuccess ||
            (e = cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev)) != cudaSuccess ||
            (e = cudaDeviceGetAttribute(&d.sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess)
            return cuda_fail(e);
        d.usable = (major == 10 && minor == 0);
        d.ready = true;
    }
    if (!d.usable) return JAMBA_SSM_ERR_NO_DEVICE;
    if (kernel && !(d.*attr_done)) {
        e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
        if (e != cudaSuccess) return cuda_fail(e);
        d.*attr_done = true;
    }
    if (sms) *sms = d.sms;
    return JAMBA_SSM_OK;
}

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

// 2-D bf16 map over [rows][cols] (cols innermost), box {64 cols, box_rows},
// 128-byte swizzle, zero fill outside the tensor.  Both kernels take 64-wide
// K blocks, and dt_proj stores its output tile as 64-column slabs.
bool encode_kmajor(EncodeTiledFn fn, CUtensorMap *map, const void *ptr, int64_t cols,
                   int64_t rows, int box_rows) {
    cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
    cuuint64_t strides[1] = {(cuuint64_t)(cols * 2)};
    cuuint32_t box[2] = {(cuuint32_t)jssm::DtProjCfg::kBK, (cuuint32_t)box_rows};
    cuuint32_t estr[2] = {1, 1};
    CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(ptr), dims,
                    strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                    CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                    CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
bool aligned4(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 3u) == 0; }

bool overlaps(const void *a, size_t an, const void *b, size_t bn) {
    if (!a || !b || an == 0 || bn == 0) return false;
    const uintptr_t x = reinterpret_cast<uintptr_t>(a), y = reinterpret_cast<uintptr_t>(b);
    return x < y + bn && y < x + an;
}

// Version 1 structs end before debug_flags; a caller's shorter struct is copied
// over a zeroed one, so its missing fields read as zero.
constexpr size_t kDtProjParamsV1 = offsetof(jamba_ssm_dt_proj_params, debug_flags);
constexpr size_t kXProjParamsV1 = offsetof(jamba_ssm_x_proj_params, debug_flags);
template <typename P>
bool read_params(const P *pin, size_t v1_size, P *p) {
    if (!pin || pin->struct_size < v1_size) return false;
    std::memset(p, 0, sizeof(P));
    std::memcpy(p, pin, pin->struct_size < sizeof(P) ? pin->struct_size : sizeof(P));
    return true;
}
static_assert(jssm::DtProjCfg::kBK == jssm::XProjCfg::kBK, "one tensor-map box width");

// Cluster size of the x_proj split over d_inner: the largest power of two up
// to 8 that keeps (token tiles x split) within one wave of the SMs and gives
// every CTA at least one 64-wide K block.
int choose_k_split(int64_t m_tiles, int64_t k_blocks, int sms) {
    int ks = 8;
    while (ks > 1 && (m_tiles * ks > sms || ks > k_blocks)) ks >>= 1;
    return ks;
}
constexpr uint64_t kDefaultTimeoutCycles = 4000000000ull;  // ~2 s at the boost clock

}  // namespace

JSSM_PROJ_API jamba_ssm_status jamba_ssm_proj_get_status(void *stream);

namespace {
// After an enqueue: with JAMBA_SSM_SYNC_CHECK set (and not "0") in the
// environment -- a debugging aid, read once per process -- wait for the work
// and return any device-side condition it recorded as this call's own status.
jamba_ssm_status finish_launch(void *stream) {
    static const bool sync_check = [] {
        const char *v = std::getenv("JAMBA_SSM_SYNC_CHECK");
        return v != nullptr && *v != '\0' && *v != '0';
    }();
    return sync_check ? jamba_ssm_proj_get_status(stream) : JAMBA_SSM_OK;
}

}  // namespace

JSSM_PROJ_API jamba_ssm_status jamba_ssm_dt_proj(const jamba_ssm_dt_proj_params *pin,
                                                 void *stream) {
    jamba_ssm_dt_proj_params p;
    if (!read_params(pin, kDtProjParamsV1, &p)) return JAMBA_SSM_ERR_INVALID_ARG;
    if (p.ntok < 0 || p.d_inner < 1 || p.dt_rank < 1) return JAMBA_SSM_ERR_INVALID_ARG;
    // d_inner / 256 channel tiles must fit the grid's y dimension
    if (p.d_inner % 8 != 0 || p.dt_rank % 8 != 0 || p.d_inner > int64_t(65535) * jssm::DtProjCfg::kBN ||
        p.dt_rank > (int64_t(1) << 16) || p.ntok > int64_t(0x7fffffff) - jssm::DtProjCfg::kBM)
        return JAMBA_SSM_ERR_UNSUPPORTED;
    if (p.ntok == 0) return JAMBA_SSM_OK;  // no work; the pointers are not used
    if (!p.dt_low_hi || !p.W_dt || !p.delta) return JAMBA_SSM_ERR_INVALID_ARG;
    if (!aligned16(p.dt_low_hi) || !aligned16(p.dt_low_lo) || !aligned16(p.W_dt) ||
        !aligned16(p.delta))
        return JAMBA_SSM_ERR_MISALIGNED;
    const size_t a_bytes = size_t(p.ntok) * size_t(p.dt_rank) * 2;
    const size_t w_bytes = size_t(p.d_inner) * size_t(p.dt_rank) * 2;
    const size_t out_bytes = size_t(p.ntok) * size_t(p.d_inner) * 2;
    if (overlaps(p.delta, out_bytes, p.dt_low_hi, a_bytes) ||
        overlaps(p.delta, out_bytes, p.dt_low_lo, a_bytes) ||
        overlaps(p.delta, out_bytes, p.W_dt, w_bytes))
        return JAMBA_SSM_ERR_INVALID_ARG;
    // dt_rank <= 256 (Jamba's included): the persistent kernel, whose CTAs keep
    // a token block's planes resident; larger ranks: one tile per CTA.
    const bool persistent = p.dt_rank <= int64_t(jssm::DtProjPCfg::kMaxKB) * jssm::DtProjPCfg::kBK;
    int sms = 0;
    jamba_ssm_status st =
        persistent
            ? prepare_device(reinterpret_cast<const void *>(&jssm::s6_dt_proj_persistent_kernel),
                             static_cast<int>(jssm::DtProjPCfg::kSmemBytes), &DeviceState::dtp_attr,
                             &sms)
            : prepare_device(reinterpret_cast<const void *>(&jssm::s6_dt_proj_kernel),
                             static_cast<int>(jssm::DtProjCfg::kSmemBytes), &DeviceState::dt_attr);
    if (st != JAMBA_SSM_OK) return st;

    EncodeTiledFn fn = encode_fn(&st);
    if (!fn) return st;
    CUtensorMap map_hi, map_lo, map_w, map_out;
    const void *lo = p.dt_low_lo ? p.dt_low_lo : p.dt_low_hi;
    if (!encode_kmajor(fn, &map_hi, p.dt_low_hi, p.dt_rank, p.ntok, jssm::DtProjCfg::kBM) ||
        !encode_kmajor(fn, &map_lo, lo, p.dt_rank, p.ntok, jssm::DtProjCfg::kBM) ||
        !encode_kmajor(fn, &map_w, p.W_dt, p.dt_rank, p.d_inner, jssm::DtProjCfg::kBN) ||
        !encode_kmajor(fn, &map_out, p.delta, p.d_inner, p.ntok, jssm::DtProjCfg::kBM))
        return cuda_fail(cudaErrorInvalidValue);
    int dt_rank = static_cast<int>(p.dt_rank), two = p.dt_low_lo ? 1 : 0;
    uint64_t limit = p.timeout_cycles ? p.timeout_cycles : kDefaultTimeoutCycles;
    uint32_t debug_flags = p.debug_flags;
    if (persistent) {
        int ntok = static_cast<int>(p.ntok), d_inner = static_cast<int>(p.d_inner);
        const int64_t items = ((p.ntok + jssm::DtProjPCfg::kBM - 1) / jssm::DtProjPCfg::kBM) *
                              ((p.d_inner + jssm::DtProjPCfg::kBN - 1) / jssm::DtProjPCfg::kBN);
        const int grid = static_cast<int>(items < sms ? items : sms);
        void *pargs[] = {&map_hi, &map_lo,  &map_w, &map_out, &ntok,
                         &d_inner, &dt_rank, &two,  &limit,   &debug_flags};
        cudaError_t e = cudaLaunchKernel(
            reinterpret_cast<const void *>(&jssm::s6_dt_proj_persistent_kernel), dim3(grid),
            dim3(jssm::DtProjPCfg::kThreads), pargs, jssm::DtProjPCfg::kSmemBytes,
            static_cast<cudaStream_t>(stream));
        if (e != cudaSuccess) return cuda_fail(e);
        return finish_launch(stream);
    }
    void *args[] = {&map_hi, &map_lo, &map_w, &map_out, &dt_rank, &two, &limit, &debug_flags};
    const dim3 grid(static_cast<unsigned>((p.ntok + jssm::DtProjCfg::kBM - 1) / jssm::DtProjCfg::kBM),
                    static_cast<unsigned>((p.d_inner + jssm::DtProjCfg::kBN - 1) / jssm::DtProjCfg::kBN));
    cudaError_t e = cudaLaunchKernel(reinterpret_cast<const void *>(&jssm::s6_dt_proj_kernel), grid,
                                     dim3(jssm::DtProjCfg::kThreads), args,
                                     jssm::DtProjCfg::kSmemBytes, static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return cuda_fail(e);
    return finish_launch(stream);
}

JSSM_PROJ_API jamba_ssm_status jamba_ssm_proj_get_status(void *stream) {
    jamba_ssm_status st = prepare_device(nullptr, 0, nullptr);
    if (st != JAMBA_SSM_OK) return st;
    cudaError_t e = cudaStreamSynchronize(static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return cuda_fail(e);
    int word = 0;
    e = cudaMemcpyFromSymbol(&word, jssm::g_status_word, sizeof(int));
    if (e != cudaSuccess) return cuda_fail(e);
    if (word != 0) {
        const int zero = 0;
        e = cudaMemcpyToSymbol(jssm::g_status_word, &zero, sizeof(int));
        if (e != cudaSuccess) return cuda_fail(e);
    }
    return static_cast<jamba_ssm_status>(word);
}

JSSM_PROJ_API int jamba_ssm_proj_last_cuda_error(void) { return t_last_cuda_error; }

JSSM_PROJ_API int jamba_ssm_proj_abi_version(void) { return JAMBA_SSM_PROJ_ABI_VERSION; }

JSSM_PROJ_API jamba_ssm_status jamba_ssm_x_proj(const jamba_ssm_x_proj_params *pin,
                                                void *stream) {
    using XC = jssm::XProjCfg;
    jamba_ssm_x_proj_params p;
    if (!read_params(pin, kXProjParamsV1, &p)) return JAMBA_SSM_ERR_INVALID_ARG;
    if (p.ntok < 0 || p.d_inner < 1 || p.dt_rank < 1 || p.d_state < 1 || !(p.eps >= 0.0f))
        return JAMBA_SSM_ERR_INVALID_ARG;
    if (p.k_split != 0 && p.k_split != 1 && p.k_split != 2 && p.k_split != 4 && p.k_split != 8)
        return JAMBA_SSM_ERR_INVALID_ARG;
    if (p.dt_rank != XC::kR || p.d_state != XC::kN || p.d_inner % 8 != 0 ||
        p.d_inner > (int64_t(1) << 30) || p.ntok > int64_t(0x7fffffff) - XC::kBM)
        return JAMBA_SSM_ERR_UNSUPPORTED;
    if (p.ntok == 0) return JAMBA_SSM_OK;  // no work; the pointers are not used
    if (!p.u || !p.W_x || !p.dt_low_hi || !p.dt_low_lo || !p.B || !p.C)
        return JAMBA_SSM_ERR_INVALID_ARG;
    if (!aligned16(p.u) || !aligned16(p.W_x) || !aligned16(p.dt_low_hi) ||
        !aligned16(p.dt_low_lo) || !aligned16(p.B) || !aligned16(p.C) || !aligned4(p.w_dt) ||
        !aligned4(p.w_B) || !aligned4(p.w_C))
        return JAMBA_SSM_ERR_MISALIGNED;
    const size_t u_bytes = size_t(p.ntok) * size_t(p.d_inner) * 2;
    const size_t w_bytes = size_t(XC::kCols) * size_t(p.d_inner) * 2;
    const size_t dt_bytes = size_t(p.ntok) * XC::kR * 2, bc_bytes = size_t(p.ntok) * XC::kN * 2;
    const void *outs[] = {p.dt_low_hi, p.dt_low_lo, p.B, p.C};
    const size_t outsz[] = {dt_bytes, dt_bytes, bc_bytes, bc_bytes};
    const void *ins[] = {p.u, p.W_x, p.w_dt, p.w_B, p.w_C};
    const size_t insz[] = {u_bytes, w_bytes, XC::kR * 4, XC::kN * 4, XC::kN * 4};
    for (int i = 0; i < 4; ++i) {
        for (int j = 0; j < 5; ++j)
            if (overlaps(outs[i], outsz[i], ins[j], insz[j])) return JAMBA_SSM_ERR_INVALID_ARG;
        for (int j = i + 1; j < 4; ++j)
            if (overlaps(outs[i], outsz[i], outs[j], outsz[j])) return JAMBA_SSM_ERR_INVALID_ARG;
    }
    int sms = 0;
    jamba_ssm_status st =
        prepare_device(reinterpret_cast<const void *>(&jssm::s6_x_proj_kernel),
                       static_cast<int>(XC::kSmemBytes), &DeviceState::x_attr, &sms);
    if (st != JAMBA_SSM_OK) return st;
    EncodeTiledFn fn = encode_fn(&st);
    if (!fn) return st;
    CUtensorMap map_u, map_w1, map_w2;
    if (!encode_kmajor(fn, &map_u, p.u, p.d_inner, p.ntok, XC::kBM) ||
        !encode_kmajor(fn, &map_w1, p.W_x, p.d_inner, XC::kCols, XC::kR) ||
        !encode_kmajor(fn, &map_w2, p.W_x, p.d_inner, XC::kCols, 2 * XC::kN))
        return cuda_fail(cudaErrorInvalidValue);

    const int64_t m_tiles = (p.ntok + XC::kBM - 1) / XC::kBM;
    const int64_t k_blocks = (p.d_inner + XC::kBK - 1) / XC::kBK;
    int ks = p.k_split ? p.k_split : choose_k_split(m_tiles, k_blocks, sms);
    if (m_tiles * ks > int64_t(0x7fffffff)) return JAMBA_SSM_ERR_UNSUPPORTED;
    jssm::XProjArgs a;
    a.dt_hi = static_cast<__nv_bfloat16 *>(p.dt_low_hi);
    a.dt_lo = static_cast<__nv_bfloat16 *>(p.dt_low_lo);
    a.B = static_cast<__nv_bfloat16 *>(p.B);
    a.C = static_cast<__nv_bfloat16 *>(p.C);
    a.w_dt = p.w_dt;
    a.w_B = p.w_B;
    a.w_C = p.w_C;
    a.eps = p.eps;
    a.ntok = static_cast<int>(p.ntok);
    a.d_inner = static_cast<int>(p.d_inner);
    a.limit = p.timeout_cycles ? p.timeout_cycles : kDefaultTimeoutCycles;
    a.debug_flags = p.debug_flags;

    cudaLaunchConfig_t cfg = {};
    cfg.blockDim = dim3(XC::kThreads);
    cfg.dynamicSmemBytes = XC::kSmemBytes;
    cfg.stream = static_cast<cudaStream_t>(stream);
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    // The library's own choice falls back to smaller clusters if the device
    // cannot co-schedule this many CTAs of this size; an explicit k_split is
    // launched as asked (and fails as a launch error if it cannot run).
    for (;;) {
        a.ks = ks;
        cfg.gridDim = dim3(static_cast<unsigned>(m_tiles * ks));
        attr[0].val.clusterDim.x = static_cast<unsigned>(ks);
        cfg.numAttrs = ks > 1 ? 1 : 0;
        if (ks == 1 || p.k_split != 0) break;
        int clusters = 0;
        if (cudaOccupancyMaxActiveClusters(&clusters, jssm::s6_x_proj_kernel, &cfg) ==
                cudaSuccess &&
            clusters > 0)
            break;
        (void)cudaGetLastError();  // clear a failed query before trying a smaller cluster
        ks >>= 1;
    }
    cudaError_t e = cudaLaunchKernelEx(&cfg, jssm::s6_x_proj_kernel, map_u, map_w1, map_w2, a);
    if (e != cudaSuccess) return cuda_fail(e);
    return finish_launch(stream);
}
