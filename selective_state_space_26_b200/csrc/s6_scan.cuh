// s6_scan.cuh -- pieces shared by the S6 prefill kernels (s6_scan_fused.cuh,
// s6_scan_serving.cuh) and the decode kernels: the scan arguments, the state
// copy for calls without steps, the staging of B / C into per-lane slots, the
// transposing butterfly over a channel's lanes, and one step of a lane's
// selective-scan recurrence.
//
// The recurrence (the "Mamba 레이어" section of the Jamba notes, with the
// discretisation read as exp(Delta A) and Delta B x):
//     h[n] = exp(Delta A[d,n]) h[n] + Delta B[b,t,n] x[b,t,d],   y = sum_n C[b,t,n] h[n].
#pragma once

#include <type_traits>

#include "device_utils.cuh"
#include "s6_math.cuh"

namespace jssm {

// Steps between the backward's checkpoints (and the length of its segments).
constexpr int kCk = 16;

struct ScanArgs {
    int64_t batch, seqlen, d_inner;
    const float *A, *D, *delta_bias, *h0;
    float *h_final;
    int delta_softplus;
    uint32_t debug_flags;
    uint64_t timeout_cycles;
    const int *cu_seqlens;     // packed layout: sequence offsets [batch + 1], or null
    int64_t total_tokens;      // rows of the packed layout
    const int *state_indices;  // state-cache row of each sequence, or null
    int64_t num_slots;         // rows of the state cache
    void *out;                 // output base (row-wise stores of short packed tiles)
    int *status;               // the call's status word (caller workspace), or null
    float *ckpt;               // checkpoint pass: [batch, ceil(seqlen / kCk), d_inner, N]
};

// A lane's NS states (fp32 pairs) to global memory.
template <int NS>
__device__ __forceinline__ void store_states(float *dst, const float2 (&h)[NS / 2]) {
#pragma unroll
    for (int i = 0; i < NS / 2; ++i) reinterpret_cast<float2 *>(dst)[i] = h[i];
}

// No steps at all (every sequence empty) with a state cache: final state =
// initial state (or zeros) for each sequence's slot; one thread per float.
// An index past num_slots is recorded as JAMBA_SSM_ERR_INVALID_ARG.
__global__ void s6_copy_states_kernel(int64_t batch, int64_t per_seq, const float *h0, float *h_final,
                                      const int *state_indices, int64_t num_slots, int *status) {
    const int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
    if (i >= batch * per_seq) return;
    const int64_t b = i / per_seq, e = i - b * per_seq;
    const int64_t row = state_indices[b];
    if (row >= num_slots && e == 0) record_status(status, kStInvalidArg);
    if (row < 0 || row >= num_slots) return;
    h_final[row * per_seq + e] = h0 ? h0[row * per_seq + e] : 0.0f;
}

// Staged B / C of one step.  The producer lays each step out in fp32 as G
// slots, one per lane of a channel: slot s holds the NS values of B and then
// the NS values of C that lane s's states use ([G][2][NS] floats), so a lane
// reads its slot with NS / 2 16-byte loads and gets B and C already paired
// for the packed fp32x2 math.
template <int NS>
struct BCPairs {
    float2 b[NS / 2], c[NS / 2];
};

__device__ __forceinline__ float2 bf16x2_to_f2(uint32_t w) {
    return make_float2(__uint_as_float(w << 16), __uint_as_float(w & 0xffff0000u));
}

template <int NS>
__device__ __forceinline__ BCPairs<NS> load_bc(const float *row, int sub) {
    const float4 *p = reinterpret_cast<const float4 *>(row + sub * 2 * NS);
    float f[2 * NS];
#pragma unroll
    for (int q = 0; q < NS / 2; ++q) {
        const float4 v = p[q];
        f[4 * q] = v.x;
        f[4 * q + 1] = v.y;
        f[4 * q + 2] = v.z;
        f[4 * q + 3] = v.w;
    }
    BCPairs<NS> r;
#pragma unroll
    for (int i = 0; i < NS / 2; ++i) {
        r.b[i] = make_float2(f[2 * i], f[2 * i + 1]);
        r.c[i] = make_float2(f[NS + 2 * i], f[NS + 2 * i + 1]);
    }
    return r;
}

// The same slot read with explicit shared-space loads, and explicit
// shared-space accesses of the bf16 / fp32 activation tiles.  Kept in program
// order (volatile) and named as shared memory rather than left to generic
// addressing; with 2 lanes per channel the tile loop ran 2-4% faster this way
// on B200, with 4 lanes 2% slower, so only the 2-lane form uses them.
template <int NS>
__device__ __forceinline__ BCPairs<NS> load_bc_shared(const float *row, int sub) {
    const uint32_t a = smem_u32(row + sub * 2 * NS);
    float f[2 * NS];
#pragma unroll
    for (int q = 0; q < NS / 2; ++q) {
        float4 v;
        asm volatile("ld.shared.v4.f32 {%0, %1, %2, %3}, [%4];"
                     : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w)
                     : "r"(a + 16 * q));
        f[4 * q] = v.x;
        f[4 * q + 1] = v.y;
        f[4 * q + 2] = v.z;
        f[4 * q + 3] = v.w;
    }
    BCPairs<NS> r;
#pragma unroll
    for (int i = 0; i < NS / 2; ++i) {
        r.b[i] = make_float2(f[2 * i], f[2 * i + 1]);
        r.c[i] = make_float2(f[NS + 2 * i], f[NS + 2 * i + 1]);
    }
    return r;
}
__device__ __forceinline__ float lds_f32(const __nv_bfloat16 *p) {
    unsigned short v;
    asm volatile("ld.shared.u16 %0, [%1];" : "=h"(v) : "r"(smem_u32(p)));
    return __uint_as_float(uint32_t(v) << 16);
}
__device__ __forceinline__ float lds_f32(const float *p) {
    float v;
    asm volatile("ld.shared.f32 %0, [%1];" : "=f"(v) : "r"(smem_u32(p)));
    return v;
}
__device__ __forceinline__ void sts_io(__nv_bfloat16 *p, __nv_bfloat16 v) {
    asm volatile("st.shared.b16 [%0], %1;" ::"r"(smem_u32(p)), "h"(__bfloat16_as_ushort(v)));
}
__device__ __forceinline__ void sts_io(float *p, float v) {
    asm volatile("st.shared.f32 [%0], %1;" ::"r"(smem_u32(p)), "f"(v));
}

// One B or C slice of NS values from the TMA tile into its staged slot: a
// copy when both have the same type, else bf16 widened to fp32.
template <int NS>
__device__ __forceinline__ void stage_slice(float *dst, const __nv_bfloat16 *src) {
    const uint32_t *w = reinterpret_cast<const uint32_t *>(src);
    float f[NS];
#pragma unroll
    for (int i = 0; i < NS / 2; ++i) {
        const float2 v = bf16x2_to_f2(w[i]);
        f[2 * i] = v.x;
        f[2 * i + 1] = v.y;
    }
    if constexpr (NS % 4 == 0) {
#pragma unroll
        for (int q = 0; q < NS / 4; ++q)
            reinterpret_cast<float4 *>(dst)[q] =
                make_float4(f[4 * q], f[4 * q + 1], f[4 * q + 2], f[4 * q + 3]);
    } else {
        static_assert(NS == 2, "slices of 2 or 4k values");
        *reinterpret_cast<float2 *>(dst) = make_float2(f[0], f[1]);
    }
}

// Copy of W 32-bit words with the widest aligned vector accesses.
template <int W>
__device__ __forceinline__ void copy_words(uint32_t *dst, const uint32_t *src) {
    if constexpr (W % 4 == 0) {
#pragma unroll
        for (int q = 0; q < W / 4; ++q)
            reinterpret_cast<uint4 *>(dst)[q] = reinterpret_cast<const uint4 *>(src)[q];
    } else if constexpr (W == 2) {
        *reinterpret_cast<uint2 *>(dst) = *reinterpret_cast<const uint2 *>(src);
    } else {
        static_assert(W == 1, "slice of 1, 2 or 4k words");
        *dst = *src;
    }
}

template <int NS, typename T>
__device__ __forceinline__ void stage_slice(T *dst, const T *src) {
    copy_words<NS * (int)sizeof(T) / 4>(reinterpret_cast<uint32_t *>(dst),
                                        reinterpret_cast<const uint32_t *>(src));
}

// For G consecutive steps held by each of the G lanes of a channel (v[j] is
// this lane's partial sum of step j), returns the full sum of step `sub` on
// lane `sub`: a butterfly where each round keeps the half of the values the
// lane's own index selects and trades the other half with the partner lane.
template <int G>
__device__ __forceinline__ float reduce_transpose(const float *v, int sub) {
    if constexpr (G == 1) {
        return v[0];
    } else {
        constexpr int H = G / 2;
        const bool upper = (sub & H) != 0;
        float w[H];
#pragma unroll
        for (int i = 0; i < H; ++i) {
            const float keep = upper ? v[i + H] : v[i];
            const float send = upper ? v[i] : v[i + H];
            w[i] = keep + __shfl_xor_sync(0xffffffffu, send, H);
        }
        return reduce_transpose<H>(w, sub & (H - 1));
    }
}

// One step of a lane's recurrence: its NS states advance by one token and its
// partial sum of C.h is returned.  States are processed in pairs with packed
// fp32x2 multiplies / FMAs (one issue slot per two states); Abar comes from the
// MUFU ex2.  dl = (Delta, Delta) and dx = (Delta x, Delta x) are duplicated
// into both halves of a register pair for the packed math.
template <int NS>
__device__ __forceinline__ float recurrence_step2(float2 (&h)[NS / 2], const float2 (&a2)[NS / 2],
                                                  const float2 dl, const float2 dx,
                                                  const BCPairs<NS> &bc) {
    static_assert(NS == 2 || NS % 4 == 0, "states per lane: 2 or a multiple of 4");
    float2 y2;
#pragma unroll
    for (int i = 0; i < NS / 2; ++i) {
        const float2 arg = mul2(dl, a2[i]);
        const float2 abar = make_float2(ex2_mufu(arg.x), ex2_mufu(arg.y));
        h[i] = fma2(abar, h[i], mul2(dx, bc.b[i]));
        y2 = i == 0 ? mul2(bc.c[i], h[i]) : fma2(bc.c[i], h[i], y2);
    }
    return y2.x + y2.y;
}

template <int NS, typename T>
__device__ __forceinline__ float recurrence_step(float2 (&h)[NS / 2], const float2 (&a2)[NS / 2],
                                                 float2 dlx, const T *row, int sub) {
    return recurrence_step2<NS>(h, a2, make_float2(dlx.x, dlx.x), make_float2(dlx.y, dlx.y),
                                load_bc<NS>(row, sub));
}

}  // namespace jssm
