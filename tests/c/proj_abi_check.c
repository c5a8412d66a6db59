/*
 * proj_abi_check.c -- a plain C client of libjamba_ssm_proj.so (no Python, no
 * torch, no GPU needed): calls the projection entry points with arguments the
 * library must reject or accept before touching a device, and checks each
 * returned status.  Pointer values are never dereferenced on these paths.
 * Exit status 0 when every check holds; otherwise the failing check is printed.
 */
#include <stdint.h>
#include <stdio.h>
#include <string.h>

#include "jamba_ssm_proj.h"

static int failures = 0;

static void expect(jamba_ssm_status got, jamba_ssm_status want, const char *what) {
    if (got != want) {
        fprintf(stderr, "%s: got status %d, want %d\n", what, (int)got, (int)want);
        ++failures;
    }
}

int main(void) {
    if (jamba_ssm_proj_abi_version() != JAMBA_SSM_PROJ_ABI_VERSION) {
        fprintf(stderr, "ABI version mismatch\n");
        return 1;
    }
    char *base = (char *)(uintptr_t)0x7f0000000000ull; /* aligned, never dereferenced */

    jamba_ssm_dt_proj_params d;
    memset(&d, 0, sizeof(d));
    d.struct_size = sizeof(d);
    d.ntok = 0;
    d.d_inner = 8192;
    d.dt_rank = 256;
    expect(jamba_ssm_dt_proj(&d, NULL), JAMBA_SSM_OK, "dt_proj: zero tokens");
    expect(jamba_ssm_dt_proj(NULL, NULL), JAMBA_SSM_ERR_INVALID_ARG, "dt_proj: NULL params");
    d.ntok = 4;
    expect(jamba_ssm_dt_proj(&d, NULL), JAMBA_SSM_ERR_INVALID_ARG, "dt_proj: NULL pointers");
    d.dt_low_hi = base;
    d.W_dt = base + (1 << 20);
    d.delta = base + (2 << 20) + 2;
    expect(jamba_ssm_dt_proj(&d, NULL), JAMBA_SSM_ERR_MISALIGNED, "dt_proj: misaligned delta");
    d.delta = base + (2 << 20);
    d.dt_rank = 12;
    expect(jamba_ssm_dt_proj(&d, NULL), JAMBA_SSM_ERR_UNSUPPORTED, "dt_proj: dt_rank % 8");
    d.dt_rank = 256;
    d.struct_size = 8;
    expect(jamba_ssm_dt_proj(&d, NULL), JAMBA_SSM_ERR_INVALID_ARG, "dt_proj: struct_size");

    jamba_ssm_x_proj_params x;
    memset(&x, 0, sizeof(x));
    x.struct_size = sizeof(x);
    x.ntok = 0;
    x.d_inner = 8192;
    x.dt_rank = 256;
    x.d_state = 16;
    x.eps = 1e-6f;
    expect(jamba_ssm_x_proj(&x, NULL), JAMBA_SSM_OK, "x_proj: zero tokens");
    x.d_state = 8;
    expect(jamba_ssm_x_proj(&x, NULL), JAMBA_SSM_ERR_UNSUPPORTED, "x_proj: d_state 8");
    x.d_state = 16;
    x.k_split = 3;
    expect(jamba_ssm_x_proj(&x, NULL), JAMBA_SSM_ERR_INVALID_ARG, "x_proj: k_split 3");
    x.k_split = 0;
    x.ntok = 4;
    x.u = base;
    x.W_x = base + (1 << 20);
    x.dt_low_hi = base + (8 << 20);
    x.dt_low_lo = base + (9 << 20);
    x.B = base + (10 << 20);
    x.C = base + (10 << 20); /* overlaps B */
    expect(jamba_ssm_x_proj(&x, NULL), JAMBA_SSM_ERR_INVALID_ARG, "x_proj: B overlaps C");
    if (failures == 0) printf("proj ABI checks passed\n");
    return failures ? 1 : 0;
}
