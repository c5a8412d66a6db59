/*
 * jamba_ssm_proj.h -- C ABI of the projection step that feeds the S6 scan
 * (libjamba_ssm_proj.so, sm_100a).
 *
 * The operation (source): "Jamba: A Hybrid Transformer-Mamba Language Model"
 * (obsidian-dorae222 notes), section "Mamba 레이어": Bbar_t, C_t and Delta_t
 * are functions of the token x_t, and Jamba's Mamba layer carries an RMSNorm.
 * The pages do not spell the function out.  The reading taken is Mamba-1's:
 *     xdbl_t = W_x u_t,   [dt_low_t | B_t | C_t] = xdbl_t  (R, N, N entries),
 *     each part RMS-normalised with its own weight,
 *     delta_t = W_dt dt_low_t                            (rank R = dt_rank),
 * where u_t is the scan's input x_t, and delta_t is the scan's raw step input
 * (its per-channel bias and softplus stay the scan's first step).
 *
 * This library provides both products on the tensor cores: jamba_ssm_x_proj
 * (W_x u with the three RMSNorms) and jamba_ssm_dt_proj (delta = dt_low W_dt^T).
 * dt_low is fp32 (it leaves the RMSNorm); a bf16 rounding of it between the two
 * would add ~1.6e-3 relative error to delta, so it travels as two bf16 planes
 * hi = bf16(v), lo = bf16(v - hi) whose sum is v to ~2^-16 relative.
 *
 * Conventions are those of jamba_ssm.h: device pointers owned by the caller,
 * nothing allocated, `stream` a cudaStream_t passed as void*, argument errors
 * returned before anything is enqueued, no C++ exception across the interface.
 * Device-side conditions of this library are read with
 * jamba_ssm_proj_get_status (this library keeps its own status word): a call
 * returns as soon as its kernel is enqueued, so a caller that must know the
 * outputs are valid checks that status after the stream's work.  With
 * JAMBA_SSM_SYNC_CHECK set (and not "0") every call waits and returns it.
 */
#ifndef JAMBA_SSM_PROJ_H
#define JAMBA_SSM_PROJ_H

#include <stddef.h>
#include <stdint.h>

#include "jamba_ssm.h"

#ifdef __cplusplus
extern "C" {
#endif

/* Version 2 appends debug_flags to both parameter structs. */
#define JAMBA_SSM_PROJ_ABI_VERSION 2

/*
 * delta[t, d] = sum_r W_dt[d, r] * (dt_low_hi[t, r] + dt_low_lo[t, r]),
 * accumulated in fp32 and rounded once (RNE) to bf16.
 *
 * Sizes: ntok >= 0 (0: nothing is launched, the pointers are not checked and
 * may be NULL, and JAMBA_SSM_OK is returned), ntok <= 2^31 - 129;
 * 1 <= d_inner <= 65535 * 128 with d_inner % 8 == 0; 1 <= dt_rank <= 2^16
 * with dt_rank % 8 == 0 (Jamba: d_inner 8192, dt_rank 256).
 * Pointers (device, 16-byte aligned):
 *   dt_low_hi  [ntok, dt_rank]   bf16, required.
 *   dt_low_lo  [ntok, dt_rank]   bf16, or NULL (only the hi plane is used).
 *   W_dt       [d_inner, dt_rank] bf16, required.
 *   delta      [ntok, d_inner]   bf16, written; must not overlap an input.
 * timeout_cycles: SM clock cycles a bounded wait may spin before the kernel
 *   gives up and records JAMBA_SSM_ERR_TIMEOUT (0 = the default, ~2 s).
 * debug_flags (version 2; 0 in production): bit 0 withholds every CTA's first
 *   k-block of operands so that its bounded wait runs out (a test of the
 *   timeout path); the tiles of such a call are not written.
 * Errors: INVALID_ARG (NULL, bad size or struct_size, overlap), UNSUPPORTED
 * (sizes out of range or not multiples of 8), MISALIGNED, NO_DEVICE, CUDA.
 */
typedef struct {
    size_t struct_size; /* sizeof(jamba_ssm_dt_proj_params) */
    int64_t ntok;
    int64_t d_inner;
    int64_t dt_rank;
    const void *dt_low_hi;
    const void *dt_low_lo;
    const void *W_dt;
    void *delta;
    uint64_t timeout_cycles;
    uint32_t debug_flags; /* version 2 */
} jamba_ssm_dt_proj_params;

jamba_ssm_status jamba_ssm_dt_proj(const jamba_ssm_dt_proj_params *p, void *stream);

/*
 * [dt_low | B | C] = W_x u for every token, each part then RMS-normalised:
 * v_i <- w_i * v_i / sqrt(mean_j v_j^2 + eps) (a part whose weight pointer is
 * NULL is not normalised).  Products accumulate in fp32; B and C are rounded
 * once to bf16, dt_low is written as its hi / lo planes.
 *
 * Sizes: ntok >= 0 (0: nothing is launched, the pointers are not checked and
 * JAMBA_SSM_OK is returned), ntok <= 2^31 - 129; 8 <= d_inner <= 2^30 with
 * d_inner % 8 == 0; dt_rank == 256 and d_state == 16 (Jamba's layer; other
 * values return JAMBA_SSM_ERR_UNSUPPORTED).
 * Pointers (device, 16-byte aligned unless noted):
 *   u          [ntok, d_inner] bf16, the scan's input x; required.
 *   W_x        [dt_rank + 2 d_state, d_inner] bf16 (rows: dt_low, B, C); required.
 *   w_dt [dt_rank], w_B [d_state], w_C [d_state]: fp32 RMSNorm weights, 4-byte
 *              aligned, or NULL.
 *   dt_low_hi, dt_low_lo  [ntok, dt_rank] bf16, written.
 *   B, C       [ntok, d_state] bf16, written (the scan's B and C layout).
 * Outputs must not overlap one another or an input.
 * k_split: CTAs that share one 128-token tile's reduction over d_inner, as a
 *   thread-block cluster: 1, 2, 4 or 8, or 0 for the library's choice (the
 *   largest that keeps the grid within one wave of the SMs).
 * timeout_cycles, debug_flags: as for jamba_ssm_dt_proj (a withheld k-block
 *   of one CTA leaves its whole cluster's rows unwritten).
 */
typedef struct {
    size_t struct_size; /* sizeof(jamba_ssm_x_proj_params) */
    int64_t ntok;
    int64_t d_inner;
    int64_t dt_rank;
    int64_t d_state;
    const void *u;
    const void *W_x;
    const float *w_dt;
    const float *w_B;
    const float *w_C;
    float eps;
    int32_t k_split;
    void *dt_low_hi;
    void *dt_low_lo;
    void *B;
    void *C;
    uint64_t timeout_cycles;
    uint32_t debug_flags; /* version 2 */
} jamba_ssm_x_proj_params;

jamba_ssm_status jamba_ssm_x_proj(const jamba_ssm_x_proj_params *p, void *stream);

/* Waits for `stream`, then returns and clears this library's device-side
 * status word (JAMBA_SSM_OK, or JAMBA_SSM_ERR_TIMEOUT). */
jamba_ssm_status jamba_ssm_proj_get_status(void *stream);

/* CUDA error code of the last call on this host thread that returned
 * JAMBA_SSM_ERR_CUDA. */
int jamba_ssm_proj_last_cuda_error(void);

int jamba_ssm_proj_abi_version(void);

#ifdef __cplusplus
}
#endif

#endif /* JAMBA_SSM_PROJ_H */
