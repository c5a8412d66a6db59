// s6_scan_small.cuh -- the S6 prefill scan and decode update for small state
// sizes (d_state of 1, 2, or 4 with bf16 I/O), where a B / C row is shorter
// than the 16 bytes a TMA tile row needs.
//
// The recurrence of the "Mamba 레이어" section of the Jamba notes, with the
// discretisation read as exp(Delta A) and Delta B x:
//     h[n] = exp(Delta A[d,n]) h[n] + Delta B[t,n] x[t,d],
//     out  = (sum_n C[t,n] h[n] + D[d] x[t,d]) * silu(z[t,d]).
// One thread carries one (sequence, channel) and all of its N states in
// registers.  Consecutive threads take consecutive channels, so the loads of
// x, delta, z and the stores of out are coalesced; the B and C of a step are
// the same address for the whole warp (a broadcast).  Steps are loaded U at a
// time into registers, one block of U ahead of the block being computed, so
// the loads of the next block are in flight while the current one runs.
// Both kernels take every serving layout of the boundary (packed sequences,
// state-cache slots).
#pragma once

#include "device_utils.cuh"
#include "s6_math.cuh"
#include "s6_scan.cuh"
#include "s6_state_update.cuh"

namespace jssm {

// The steps of one block: U (x, delta, z, B[N], C[N]) in registers.
template <int N, int U>
struct SmallBlock {
    float x[U], dt[U], z[U], B[U][N], C[U][N];
};

template <typename IoT, int N, int U>
__device__ __forceinline__ void small_load(SmallBlock<N, U> &s, const IoT *x, const IoT *dt,
                                           const IoT *z, const IoT *B, const IoT *C, int64_t row0,
                                           int64_t nrows, int64_t d, int64_t d_inner) {
#pragma unroll
    for (int u = 0; u < U; ++u) {
        const bool ok = u < nrows;
        const int64_t r = row0 + (ok ? u : 0);
        s.x[u] = ok ? to_f32(x[r * d_inner + d]) : 0.0f;
        s.dt[u] = ok ? to_f32(dt[r * d_inner + d]) : 0.0f;
        s.z[u] = ok ? to_f32(z[r * d_inner + d]) : 0.0f;
#pragma unroll
        for (int n = 0; n < N; ++n) {
            s.B[u][n] = ok ? to_f32(__ldg(B + r * N + n)) : 0.0f;
            s.C[u][n] = ok ? to_f32(__ldg(C + r * N + n)) : 0.0f;
        }
    }
}

template <typename IoT, int N, int U>
__device__ __forceinline__ void small_steps(const SmallBlock<N, U> &s, float (&h)[N],
                                            const float (&a2)[N], float bias, float dskip,
                                            bool use_softplus, IoT *out, int64_t row0,
                                            int64_t nrows, int64_t d, int64_t d_inner) {
#pragma unroll
    for (int u = 0; u < U; ++u) {
        if (u < nrows) {
            const float dl = delta_io<IoT>(s.dt[u], bias, use_softplus);
            const float dx = dl * s.x[u];
            float y = 0.0f;
#pragma unroll
            for (int n = 0; n < N; ++n) {
                h[n] = fmaf(ex2_mufu(dl * a2[n]), h[n], dx * s.B[u][n]);
                y = fmaf(s.C[u][n], h[n], y);
            }
            out[(row0 + u) * d_inner + d] = from_f32<IoT>((y + dskip * s.x[u]) * silu_f32(s.z[u]));
        }
    }
}

// grid (ceil(d_inner / 128), batch), 128 threads: thread (blockIdx.y, d).
template <typename IoT, int N, int U>
__global__ void __launch_bounds__(128) s6_scan_small_kernel(const ScanArgs a, const IoT *x,
                                                            const IoT *dt, const IoT *z,
                                                            const IoT *B, const IoT *C) {
    const int64_t d = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
    const int64_t b = blockIdx.y;
    if (d >= a.d_inner) return;
    const int64_t D = a.d_inner;
    // token rows of sequence b: its batch row, or its slice of the packed layout
    int64_t start = b * a.seqlen, len = a.seqlen;
    if (a.cu_seqlens) {
        const int64_t tot = a.total_tokens;
        int64_t s0 = __ldg(a.cu_seqlens + b), s1 = __ldg(a.cu_seqlens + b + 1);
        s0 = s0 < 0 ? 0 : (s0 > tot ? tot : s0);
        s1 = s1 < s0 ? s0 : (s1 > tot ? tot : s1);
        start = s0;
        len = s1 - s0;
    }
    // state row: the sequence itself, or its cache slot (negative: none)
    int64_t srow = b;
    if (a.state_indices) {
        srow = __ldg(a.state_indices + b);
        if (srow >= a.num_slots) {
            if (d == 0) record_status(a.status, kStInvalidArg);
            srow = -1;
        }
    }
    float h[N], a2[N];
#pragma unroll
    for (int n = 0; n < N; ++n) {
        a2[n] = __ldg(a.A + d * N + n) * kLog2e;
        h[n] = (a.h0 && srow >= 0) ? __ldg(a.h0 + (srow * D + d) * N + n) : 0.0f;
    }
    const float bias = a.delta_bias ? __ldg(a.delta_bias + d) : 0.0f;
    const float dskip = a.D ? __ldg(a.D + d) : 0.0f;
    const bool sp = a.delta_softplus != 0;
    IoT *out = static_cast<IoT *>(a.out);

    SmallBlock<N, U> s0, s1;
    small_load<IoT, N, U>(s0, x, dt, z, B, C, start, len, d, D);
    for (int64_t t = 0; t < len; t += 2 * U) {
        small_load<IoT, N, U>(s1, x, dt, z, B, C, start + t + U, len - t - U, d, D);
        small_steps<IoT, N, U>(s0, h, a2, bias, dskip, sp, out, start + t, len - t, d, D);
        small_load<IoT, N, U>(s0, x, dt, z, B, C, start + t + 2 * U, len - t - 2 * U, d, D);
        small_steps<IoT, N, U>(s1, h, a2, bias, dskip, sp, out, start + t + U, len - t - U, d, D);
    }
    if (a.h_final && srow >= 0) {
#pragma unroll
        for (int n = 0; n < N; ++n) a.h_final[(srow * D + d) * N + n] = h[n];
    }
}

// One decode step, one thread per (request, channel): grid (ceil(d_inner /
// 128), batch), 128 threads.  The state row is read and written in place.
template <typename IoT, int N>
__global__ void __launch_bounds__(128) s6_state_update_small_kernel(const UpdateArgs a) {
    const int64_t d = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
    const int64_t b = blockIdx.y;
    if (d >= a.d_inner) return;
    const int64_t srow = state_row(a, b, d == 0);
    if (srow < 0) return;
    const int64_t D = a.d_inner;
    const int64_t i = b * D + d;
    const float xv = to_f32(static_cast<const IoT *>(a.x)[i]);
    const float dl = delta_io<IoT>(to_f32(static_cast<const IoT *>(a.delta)[i]),
                                   a.delta_bias ? __ldg(a.delta_bias + d) : 0.0f, a.delta_softplus != 0);
    const float dx = dl * xv;
    const IoT *Bp = static_cast<const IoT *>(a.B) + b * N;
    const IoT *Cp = static_cast<const IoT *>(a.C) + b * N;
    float *st = a.state + (srow * D + d) * N;
    float y = 0.0f;
#pragma unroll
    for (int n = 0; n < N; ++n) {
        const float hn = fmaf(ex2_mufu(dl * (__ldg(a.A + d * N + n) * kLog2e)), st[n],
                              dx * to_f32(Bp[n]));
        st[n] = hn;
        y = fmaf(to_f32(Cp[n]), hn, y);
    }
    const float dskip = a.D ? __ldg(a.D + d) : 0.0f;
    const float zv = to_f32(static_cast<const IoT *>(a.z)[i]);
    static_cast<IoT *>(a.out)[i] = from_f32<IoT>((y + dskip * xv) * silu_f32(zv));
}

}  // namespace jssm
