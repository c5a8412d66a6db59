/*
 * jamba_ssm.h -- C ABI of the B200 (sm_100a) Mamba-1 selective-scan (S6)
 * library: the prefill scan and the one-token decode state update of the S6
 * mixer that makes up seven of every eight Jamba layers.
 *
 * The operation (sources):
 *   - "Jamba: A Hybrid Transformer-Mamba Language Model" (obsidian-dorae222
 *     notes), section "Mamba 레이어" (Mamba layer): the selective SSM
 *         h_t = Abar_t h_{t-1} + Bbar_t x_t,   y_t = C_t h_t,
 *     with Bbar_t, C_t, Delta_t functions of the input; d_state = 16 and
 *     expansion factor 2 (d_model 4096 -> d_inner 8192).
 *   - the same notes, section "KV 캐시 효율 분석": the Mamba state is a fixed
 *     D x N array per layer and sequence, independent of the length L.
 *   - "Jamba -- Hybrid SSM-Transformer" (factory.pai-world.com), section
 *     "한 페이지로 보는 SSM": y_t needs only h_{t-1} and x_t (O(1) decode);
 *     item 2 of its Mamba-3 list: Mamba's state matrix A is real diagonal.
 *   Readings where the pages are silent: Abar = exp(Delta * A[d,n]),
 *   Bbar x = Delta * B[t,n] * x, Delta = softplus(delta + delta_bias[d]) (or
 *   delta + delta_bias[d] without softplus), and the layer output
 *   out = (sum_n C[t,n] h[n] + D[d] x) * silu(z), silu(z) = z / (1 + e^-z).
 *
 * Conventions shared by every entry point:
 *   - All array pointers are DEVICE pointers owned by the caller.  The library
 *     allocates nothing, frees nothing and keeps no per-call state (it caches
 *     only per-device attributes).
 *   - `stream` is a cudaStream_t passed as void* (NULL = legacy default
 *     stream).  Work is enqueued asynchronously on it.
 *   - Activations are row-major with the channel index innermost:
 *     x/delta/z/out [batch, seqlen, d_inner], B/C [batch, seqlen, d_state];
 *     the state is fp32 [batch, d_inner, d_state]; A is fp32
 *     [d_inner, d_state]; D and delta_bias are fp32 [d_inner].
 *   - Argument errors are detected on the host before anything is enqueued and
 *     returned as a status; nothing is launched then.  A failed launch returns
 *     JAMBA_SSM_ERR_CUDA (the CUDA error code is kept per host thread, see
 *     jamba_ssm_last_cuda_error).  A device-side condition (a bounded wait that
 *     ran out, a state slot past the cache) is recorded in a status word: the
 *     first word of the caller's workspace when the call was given one, else
 *     a per-device word of the library; jamba_ssm_get_status reads it.  No C++
 *     exception crosses this interface.
 *   - Workspace: the calls take an optional caller-owned device buffer of at
 *     least jamba_ssm_scan_workspace_size() bytes (16-byte aligned).  The
 *     scan needs no scratch of its own -- every lane carries its channel's
 *     states through the whole sequence in registers, so no carry between
 *     chunks of a sequence is ever stored -- and the workspace holds only the
 *     call's status word.  A caller that gives each stream its own workspace
 *     keeps the streams' device-side conditions apart.  The caller zero-fills
 *     a workspace once before its first use; jamba_ssm_get_status clears it
 *     again after reading a condition.
 *   - Debugging aid: with the environment variable JAMBA_SSM_SYNC_CHECK set
 *     (and not "0") when the library is first called, every call waits for
 *     its work and returns jamba_ssm_get_status()'s result itself.
 */
#ifndef JAMBA_SSM_H
#define JAMBA_SSM_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Version 3: the workspace fields, jamba_ssm_scan_workspace_size, the
 * (workspace, stream) form of jamba_ssm_get_status, d_state 1 and 2 (and 4 in
 * bf16), and the status codes renumbered so that ERR_WORKSPACE is 4: a caller
 * built against an earlier version of this header must be rebuilt. */
#define JAMBA_SSM_ABI_VERSION 4

/* Bytes of the status block at the start of a workspace. */
#define JAMBA_SSM_STATUS_BYTES 16

typedef enum {
    JAMBA_SSM_OK = 0,
    JAMBA_SSM_ERR_INVALID_ARG = 1,  /* NULL pointer, negative size, aliasing, bad struct_size */
    JAMBA_SSM_ERR_UNSUPPORTED = 2,  /* d_state / dtype / d_inner combination not built        */
    JAMBA_SSM_ERR_MISALIGNED = 3,   /* a pointer is not aligned as documented below            */
    JAMBA_SSM_ERR_WORKSPACE = 4,    /* workspace given but smaller than required               */
    JAMBA_SSM_ERR_CUDA = 5,         /* a CUDA runtime/driver call or the launch failed         */
    JAMBA_SSM_ERR_TIMEOUT = 6,      /* device side: a bounded wait ran out (get_status only)   */
    JAMBA_SSM_ERR_NO_DEVICE = 7     /* no usable sm_100 device is current                      */
} jamba_ssm_status;

typedef enum {
    JAMBA_SSM_BF16 = 0,  /* x, delta, z, B, C, out are bfloat16 */
    JAMBA_SSM_F32 = 1    /* x, delta, z, B, C, out are float32  */
} jamba_ssm_dtype;

/*
 * Prefill scan over whole sequences (the S6 recurrence of "Mamba 레이어",
 * evaluated for t = 0 .. seqlen-1 from the initial state h0).
 *
 * Sizes: batch >= 0, seqlen >= 0, d_inner >= 1, d_state in {1, 2, 4, 8, 16},
 * and d_inner % 8 == 0 for bf16 I/O, d_inner % 4 == 0 for f32 I/O (each
 * activation row is a multiple of 16 bytes).  Jamba's layer is d_inner = 8192,
 * d_state = 16.  State sizes whose B / C rows are shorter than 16 bytes (bf16
 * d_state 1, 2, 4; f32 d_state 1, 2) take a one-thread-per-channel kernel
 * with plain loads, at most 65535 sequences per call; the others take the
 * TMA-fed kernels.
 * Pointers (device):
 *   x, delta, z   [batch, seqlen, d_inner] io_dtype, 16-byte aligned, required.
 *                 delta is the raw step input; Delta is formed in the kernel.
 *   B, C          [batch, seqlen, d_state] io_dtype, 16-byte aligned, required.
 *   A             [d_inner, d_state] fp32, 16-byte aligned, required (A < 0
 *                 in a trained layer; any finite value is accepted).
 *   D             [d_inner] fp32 or NULL (no skip term).
 *   delta_bias    [d_inner] fp32 or NULL (zero bias).
 *   h0            [batch, d_inner, d_state] fp32, 16-byte aligned, or NULL
 *                 (zero initial state).  Resuming a sequence = passing the
 *                 h_final of the previous chunk here (chunked prefill).
 *   out           [batch, seqlen, d_inner] io_dtype, 16-byte aligned, required;
 *                 must not overlap any input.
 *   h_final       [batch, d_inner, d_state] fp32, 16-byte aligned, or NULL.
 *                 The state after the last step: the decode cache entry.
 *                 h_final == h0 (resume in place) is allowed.
 * delta_softplus: nonzero -> Delta = softplus(delta + delta_bias), else
 *                 Delta = delta + delta_bias.
 * kernel_variant: 0 = let the library choose the launch shape; k > 0 forces
 *                 built variant k (see jamba_ssm_scan_variant_info); an
 *                 unknown or inapplicable k returns JAMBA_SSM_ERR_UNSUPPORTED.
 * debug_flags / timeout_cycles: 0 in production.  Bit 0 of debug_flags
 *                 withholds the first input tile of every CTA so its bounded
 *                 wait runs out (test of the timeout path); timeout_cycles
 *                 overrides the wait limit (SM clock cycles, 0 = ~1 s).
 * Empty input: batch == 0 does nothing; seqlen == 0 copies h0 (or zeros)
 * into h_final.
 *
 * Serving layouts (ABI version 2; a caller whose struct_size ends before
 * these fields gets both off):
 *   cu_seqlens    device int32 [batch + 1] or NULL.  Non-NULL selects the
 *                 packed variable-length layout: x, delta, z, out are
 *                 [total_tokens, d_inner] and B, C [total_tokens, d_state];
 *                 sequence b is rows cu_seqlens[b] .. cu_seqlens[b+1] - 1
 *                 (0 = cu_seqlens[0] <= ... <= cu_seqlens[batch] =
 *                 total_tokens; the kernel clamps every offset to
 *                 [0, total_tokens]).  `seqlen` is ignored.  An empty
 *                 sequence copies its initial state to its final state.
 *   total_tokens  rows of the packed layout (cu_seqlens != NULL), >= 0.
 *   state_indices device int32 [batch] or NULL.  Non-NULL: h0 and h_final
 *                 are [num_slots, d_inner, d_state] state caches and
 *                 sequence b reads / writes row state_indices[b].  A negative
 *                 index means "no cached state": zero initial state and no
 *                 final state written (outputs are still computed).  An
 *                 index >= num_slots is treated the same way and recorded as
 *                 JAMBA_SSM_ERR_INVALID_ARG in the status word.  Indices of
 *                 one call must be distinct.
 *   num_slots     rows of the state caches (state_indices != NULL).
 *
 * Workspace (ABI version 3; absent -- NULL -- for a shorter struct_size):
 *   workspace     device buffer of workspace_bytes >= the size
 *                 jamba_ssm_scan_workspace_size returns, 16-byte aligned, or
 *                 NULL (the status goes to the library's per-device word).
 *                 Too small: JAMBA_SSM_ERR_WORKSPACE.
 *
 * Checkpoints for the backward (ABI version 4; absent -- NULL -- for a
 * shorter struct_size).  The source pages say nothing of training kernels;
 * this is a convenience for a training step that runs the forward and then
 * jamba_ssm_scan_bwd on the same inputs:
 *   ckpt          device fp32 [batch, ceil(seqlen / 16), d_inner, d_state]
 *                 (jamba_ssm_scan_ckpt_size bytes), 16-byte aligned, or NULL.
 *                 Non-NULL: entry [b, k] receives sequence b's state before
 *                 step 16 k (entry [b, 0] is the initial state), and `out`
 *                 and `h_final` are the same bits as without it.  Batched
 *                 layout only (cu_seqlens and state_indices NULL), and the
 *                 backward's state sizes (d_state 8 or 16 with bf16 I/O, 4, 8
 *                 or 16 with fp32); otherwise JAMBA_SSM_ERR_UNSUPPORTED.  Must
 *                 not overlap any input or output.
 */
typedef struct jamba_ssm_scan_params {
    size_t struct_size;          /* = sizeof(jamba_ssm_scan_params); callers of
                                    ABI version 1 pass the size ending at
                                    timeout_cycles                             */
    int64_t batch, seqlen, d_inner, d_state;
    int32_t io_dtype;            /* jamba_ssm_dtype                            */
    int32_t delta_softplus;
    const void *x, *delta, *z;
    const void *B, *C;
    const float *A;
    const float *D;
    const float *delta_bias;
    const float *h0;
    void *out;
    float *h_final;
    int32_t kernel_variant;
    uint32_t debug_flags;
    uint64_t timeout_cycles;
    /* ABI version 2 */
    const int32_t *cu_seqlens;
    int64_t total_tokens;
    const int32_t *state_indices;
    int64_t num_slots;
    /* ABI version 3 */
    void *workspace;
    size_t workspace_bytes;
    /* ABI version 4 */
    float *ckpt;
} jamba_ssm_scan_params;

/* Bytes of workspace a scan of these sizes may use: the status block
 * (JAMBA_SSM_STATUS_BYTES) at any size, since nothing else is stored. */
size_t jamba_ssm_scan_workspace_size(int64_t batch, int64_t seqlen, int64_t d_inner,
                                     int64_t d_state);

jamba_ssm_status jamba_ssm_scan(const jamba_ssm_scan_params *p, void *stream);

/*
 * One decode step for `batch` requests (the O(1) update of "한 페이지로 보는
 * SSM"): for every request b and channel d,
 *   h'[n] = exp(Delta A[d,n]) h[n] + Delta B[b,n] x,
 *   out   = (sum_n C[b,n] h'[n] + D[d] x) * silu(z),
 * and the state is overwritten with h' IN PLACE.
 * Sizes: as jamba_ssm_scan with seqlen = 1, except d_inner only needs
 * d_inner >= 1; d_state in {1, 2, 4, 8, 16} for both dtypes (1 and 2: at most
 * 65535 requests per call).
 * Pointers (device):
 *   state      [batch, d_inner, d_state] fp32, 16-byte aligned (4-byte for
 *              d_state 1 and 2), read + written.
 *   x, delta, z, out [batch, d_inner] io_dtype, aligned to the element size;
 *              out must not overlap an input.  (When x, delta and z are
 *              16-byte aligned and the rows are multiples of 16 bytes, a
 *              bulk-copy kernel is used; otherwise a plain-load kernel.)
 *   B, C       [batch, d_state] io_dtype, 16-byte aligned (element-aligned
 *              for d_state 1 and 2).
 *   A          [d_inner, d_state] fp32, 16-byte aligned (4-byte for d_state 1
 *              and 2); D, delta_bias as above (4-byte aligned or NULL).
 * Serving layout (ABI version 2; absent when struct_size ends before it):
 *   state_indices device int32 [batch] or NULL.  Non-NULL: `state` is a
 *              [num_slots, d_inner, d_state] cache and request b updates row
 *              state_indices[b].  A negative index skips request b (its state
 *              row and its out row are left untouched: padding in a
 *              continuous batch); an index >= num_slots is skipped too and
 *              recorded as JAMBA_SSM_ERR_INVALID_ARG in the status word.
 *              Indices of one call must be distinct.
 *   num_slots  rows of the state cache (state_indices != NULL), >= 1.
 *   debug_flags / timeout_cycles: 0 in production.  Bit 0 of debug_flags
 *              withholds the first state load of every CTA of the bulk-copy
 *              kernel so its bounded wait runs out (test of the timeout path;
 *              rows of 16-byte multiples take that kernel); timeout_cycles
 *              overrides the wait limit (SM clock cycles, 0 = ~1 s).
 * Workspace (ABI version 3): as jamba_ssm_scan (status word only), or NULL.
 */
typedef struct jamba_ssm_state_update_params {
    size_t struct_size;          /* = sizeof(jamba_ssm_state_update_params);
                                    ABI version 1 callers: size ending at out  */
    int64_t batch, d_inner, d_state;
    int32_t io_dtype;
    int32_t delta_softplus;
    float *state;
    const void *x, *delta, *z;
    const void *B, *C;
    const float *A;
    const float *D;
    const float *delta_bias;
    void *out;
    /* ABI version 2 */
    const int32_t *state_indices;
    int64_t num_slots;
    uint32_t debug_flags;
    uint64_t timeout_cycles;
    /* ABI version 3 */
    void *workspace;
    size_t workspace_bytes;
} jamba_ssm_state_update_params;

jamba_ssm_status jamba_ssm_state_update(const jamba_ssm_state_update_params *p, void *stream);

/*
 * Backward pass of jamba_ssm_scan (training): the gradients of a loss L with
 * respect to every input of the scan, given dout = dL/dout and, optionally,
 * dL/dh_final.  The chain rule through the recurrence of "Mamba 레이어" in
 * reverse time, with g = dL/dh_t:  g += dy C_t (dy = dout silu(z)); then per
 * state dC_t += dy h_t, dB_t += g Delta x, dDelta += g h_{t-1} Abar A + g B x,
 * dx += g Delta B, dA += g h_{t-1} Abar Delta, g <- Abar g; dz and dD from the
 * gate and the skip; ddelta = dDelta * d softplus(v)/dv; dh0 = the final g.
 *
 * Sizes: as jamba_ssm_scan (batched layout only; no cu_seqlens or state
 * slots), with d_state in {8, 16} for bf16 I/O and {4, 8, 16} for f32 I/O.
 * Pointers (device; the forward's inputs as given to jamba_ssm_scan):
 *   x, delta, z, B, C, A, D, delta_bias, h0, delta_softplus: as the forward.
 *   dout       [batch, seqlen, d_inner] io_dtype, 16-byte aligned, required.
 *   dh_final   [batch, d_inner, d_state] fp32 or NULL (zero).
 *   dx, ddelta, dz  [batch, seqlen, d_inner] io_dtype, 16-byte aligned,
 *              written (ddelta is the gradient of the raw step input delta).
 *   dB, dC     [batch, seqlen, d_state] io_dtype, 16-byte aligned, written.
 *   dA         [d_inner, d_state] fp32 (summed over the batch), or NULL.
 *   dD, ddelta_bias [d_inner] fp32 (summed over the batch), or NULL.
 *   dh0        [batch, d_inner, d_state] fp32, or NULL.
 *   Outputs must not overlap one another or an input.
 *   workspace  REQUIRED: device buffer of at least
 *              jamba_ssm_scan_bwd_workspace_size() bytes, 16-byte aligned, its
 *              first JAMBA_SSM_STATUS_BYTES zero-filled before first use (the
 *              status word, read with jamba_ssm_get_status(workspace, ...)).
 *              The rest is scratch: the states every 16 steps (recomputed from
 *              the inputs), per-CTA partial sums of dB and dC, and per-sequence
 *              partials of dA, dD, ddelta_bias.
 * The result does not depend on the launch shape or on timing: every sum is
 * taken in a fixed order (no atomics).  Calls sharing one workspace must not
 * overlap on the GPU.
 * debug_flags / timeout_cycles: as jamba_ssm_scan (bit 0 withholds each
 * CTA's first tile of the backward kernel).
 * ckpt (ABI version 4; absent -- NULL -- for a shorter struct_size): the
 *   checkpoints a forward call with the same inputs stored (see
 *   jamba_ssm_scan_params.ckpt), or NULL.  Non-NULL: the backward uses them
 *   and skips its own checkpoint pass; the results are the same bits either
 *   way.  Must not overlap any output.  The workspace size is unchanged.
 */
typedef struct jamba_ssm_scan_bwd_params {
    size_t struct_size;          /* = sizeof(jamba_ssm_scan_bwd_params)       */
    int64_t batch, seqlen, d_inner, d_state;
    int32_t io_dtype;
    int32_t delta_softplus;
    const void *x, *delta, *z;
    const void *B, *C;
    const float *A;
    const float *D;
    const float *delta_bias;
    const float *h0;
    const void *dout;
    const float *dh_final;
    void *dx, *ddelta, *dz;
    void *dB, *dC;
    float *dA;
    float *dD;
    float *ddelta_bias;
    float *dh0;
    void *workspace;
    size_t workspace_bytes;
    uint32_t debug_flags;
    uint64_t timeout_cycles;
    /* ABI version 4 */
    const float *ckpt;
} jamba_ssm_scan_bwd_params;

/* Bytes of the forward's checkpoints for these sizes (jamba_ssm_scan_params.
 * ckpt): batch * ceil(seqlen / 16) * d_inner * d_state * 4; 0 for negative
 * sizes. */
size_t jamba_ssm_scan_ckpt_size(int64_t batch, int64_t seqlen, int64_t d_inner, int64_t d_state);

/* Bytes of workspace jamba_ssm_scan_bwd needs for these sizes (0 for an
 * unsupported d_state). */
size_t jamba_ssm_scan_bwd_workspace_size(int64_t batch, int64_t seqlen, int64_t d_inner,
                                         int64_t d_state);

jamba_ssm_status jamba_ssm_scan_bwd(const jamba_ssm_scan_bwd_params *p, void *stream);

/*
 * jamba_ssm_scan_bwd for callers that cannot allocate device memory where
 * they run it -- for instance a plug-in whose host framework owns every device
 * allocation and fixes its memory plan before the run, or code on a path where
 * cudaMalloc's implicit device synchronisation is not acceptable.  The source
 * pages have no counterpart of this call; it is a deployment convenience.
 *
 * Same parameters and results as jamba_ssm_scan_bwd, except that `workspace`
 * must be NULL and `workspace_bytes` 0: the scratch is a fixed array of
 * JAMBA_SSM_BWD_NOALLOC_SCRATCH_BYTES that the library reserves in the memory
 * of every device it is loaded on and keeps until the process exits.  Nothing
 * is allocated or freed by this call.
 *   - Sizes whose jamba_ssm_scan_bwd_workspace_size exceeds that array return
 *     JAMBA_SSM_ERR_WORKSPACE before anything is enqueued (at Jamba's width,
 *     d_inner 8192 and d_state 16, about 1300 tokens fit).
 *   - Every call shares the one array of its device: calls that overlap on the
 *     GPU (other streams, other host threads) race on it and must be ordered
 *     by the caller.  The array keeps the last call's contents; each call
 *     clears the part that must start at zero (its status word) itself.
 *   - A device-side condition (a bounded wait that ran out) is moved into the
 *     library's per-device status word: read it with
 *     jamba_ssm_get_status(NULL, stream).
 *   - The first call on each device looks the array's device address up
 *     (cudaGetSymbolAddress), once; make that first call before any stream
 *     capture on that device.
 */
#define JAMBA_SSM_BWD_NOALLOC_SCRATCH_BYTES (64u * 1024u * 1024u)
jamba_ssm_status jamba_ssm_scan_bwd_noalloc(const jamba_ssm_scan_bwd_params *p, void *stream);

/*
 * The scalar-identity variant of the selective scan (Mamba-2's state matrix).
 * Sources: "Jamba -- Hybrid SSM-Transformer" (factory.pai-world.com), section
 * "Mamba-3: 2026년의 순수 SSM 기준선", items 1-2: the state matrix is a scaled
 * identity, discretised by Euler's method.  Reading: d_inner = nheads *
 * headdim channels, channel d = head * headdim + p; per head and token
 *     Delta = softplus(delta[t, head] + delta_bias[head]) (or without softplus),
 *     h[n]  = exp(Delta A[head]) h[n] + Delta B[t, n] x[t, d],
 *     out   = (sum_n C[t, n] h[n] + D[d] x[t, d]) silu(z[t, d]).
 *
 * Sizes: batch in [0, 65535], seqlen >= 0, headdim a multiple of 32, nheads a
 * multiple of 8 (bf16) or 4 (f32), d_state in {8, 16}.
 * Pointers (device, 16-byte aligned unless noted):
 *   x, z, out   [batch, seqlen, nheads * headdim] io_dtype (out written; it must
 *               not overlap an input).
 *   delta       [batch, seqlen, nheads] io_dtype: one raw step size per head.
 *   B, C        [batch, seqlen, d_state] io_dtype.
 *   A           [nheads] fp32 (4-byte aligned); delta_bias [nheads] fp32 or NULL;
 *               D [nheads * headdim] fp32 or NULL.
 *   h0, h_final [batch, nheads * headdim, d_state] fp32 or NULL (the same
 *               state layout as jamba_ssm_scan's).
 *   workspace   optional status block, as for jamba_ssm_scan.
 * debug_flags / timeout_cycles: as jamba_ssm_scan; bit 1 of debug_flags runs
 *               the per-step kernel where the chunked one would be used.
 * Kernels: bf16 I/O with d_state 16 and headdim a multiple of 64 runs the
 * chunked form on the tensor cores (128-token chunks: per chunk and 64-channel
 * slice of a head the products C B^T, M x and W x of the unrolled recurrence,
 * the state passed from chunk to chunk in fp32); every other shape runs the
 * per-step recurrence.
 */
typedef struct jamba_ssm_ssd_params {
    size_t struct_size;          /* = sizeof(jamba_ssm_ssd_params)            */
    int64_t batch, seqlen, nheads, headdim, d_state;
    int32_t io_dtype;
    int32_t delta_softplus;
    const void *x, *delta, *z;
    const void *B, *C;
    const float *A;
    const float *D;
    const float *delta_bias;
    const float *h0;
    void *out;
    float *h_final;
    void *workspace;
    size_t workspace_bytes;
    uint32_t debug_flags;
    uint64_t timeout_cycles;
} jamba_ssm_ssd_params;

jamba_ssm_status jamba_ssm_ssd_scan(const jamba_ssm_ssd_params *p, void *stream);

/* Launch shape the scan would use for these parameters (no launch).  Any of
 * the out pointers may be NULL.  variant: the built variant chosen (0 for the
 * one-thread-per-channel kernel of the small state sizes);
 * lanes_per_channel: lanes sharing one channel's states; channels_per_cta;
 * grid: CTAs launched; tasks: (sequence, channel-group) units. */
jamba_ssm_status jamba_ssm_scan_plan(const jamba_ssm_scan_params *p, int32_t *variant,
                                     int32_t *lanes_per_channel, int32_t *channels_per_cta,
                                     int32_t *grid, int64_t *tasks);

/* Description of built scan variant k (1-based); returns
 * JAMBA_SSM_ERR_UNSUPPORTED past the last one.  Out pointers may be NULL. */
jamba_ssm_status jamba_ssm_scan_variant_info(int32_t k, int32_t *io_dtype, int32_t *d_state,
                                             int32_t *lanes_per_channel, int32_t *warps_per_cta,
                                             int32_t *time_tile);

/* Synchronizes `stream`, then reads and clears a sticky status word: the
 * first word of `workspace` (the calls that were given this workspace), or,
 * for workspace == NULL, the current device's word of the library (the calls
 * given none).  Returns JAMBA_SSM_OK, or the first device-side error recorded
 * there since the last read (JAMBA_SSM_ERR_TIMEOUT, or
 * JAMBA_SSM_ERR_INVALID_ARG for a state index past num_slots).  Returns
 * JAMBA_SSM_ERR_CUDA if the synchronization or the read itself failed, and
 * JAMBA_SSM_ERR_MISALIGNED for a workspace that is not 16-byte aligned. */
jamba_ssm_status jamba_ssm_get_status(void *workspace, void *stream);

/* CUDA error code (cudaError_t as int) behind the last JAMBA_SSM_ERR_CUDA
 * returned on this host thread, 0 if none. */
int jamba_ssm_last_cuda_error(void);

/* Static, NUL-terminated description of a status code. */
const char *jamba_ssm_status_string(jamba_ssm_status s);

/* JAMBA_SSM_ABI_VERSION the library was built with. */
int jamba_ssm_abi_version(void);

#ifdef __cplusplus
}
#endif

#endif /* JAMBA_SSM_H */
