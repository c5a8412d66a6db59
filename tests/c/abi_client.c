/*
 * abi_client.c -- a plain C client of libjamba_ssm.so (no Python, no torch):
 * reads a scan problem from a binary file, moves it to the device with the
 * CUDA runtime, calls jamba_ssm_scan and jamba_ssm_state_update through the C
 * ABI, and writes the results back for the test to compare with the oracle.
 *
 * Input file (little endian): int64 batch, seqlen, d_inner, d_state; then
 * fp32 x, delta, z [batch, seqlen, d_inner], B, C [batch, seqlen, d_state],
 * A [d_inner, d_state], D [d_inner], delta_bias [d_inner]; then one decode
 * token: fp32 x1, delta1, z1 [batch, d_inner], B1, C1 [batch, d_state].
 * Output file: fp32 out [batch, seqlen, d_inner], h_final [batch, d_inner,
 * d_state], out1 [batch, d_inner], state after the decode step.
 * Exit status 0 on success; a nonzero status prints the library's message.
 */
#include <cuda_runtime.h>
#include <stdio.h>
#include <stdlib.h>

#include "jamba_ssm.h"

static void *dev_copy(const float *h, size_t n) {
    void *d = NULL;
    if (cudaMalloc(&d, n * sizeof(float) + 16) != cudaSuccess) return NULL;
    if (h && cudaMemcpy(d, h, n * sizeof(float), cudaMemcpyHostToDevice) != cudaSuccess) return NULL;
    return d;
}

static float *read_block(FILE *f, size_t n) {
    float *p = (float *)malloc(n * sizeof(float));
    if (!p || fread(p, sizeof(float), n, f) != n) return NULL;
    return p;
}

static int check(jamba_ssm_status s, const char *what) {
    if (s != JAMBA_SSM_OK) {
        fprintf(stderr, "%s: %s (cuda %d)\n", what, jamba_ssm_status_string(s), jamba_ssm_last_cuda_error());
        return 1;
    }
    return 0;
}

int main(int argc, char **argv) {
    if (argc != 3) return 2;
    FILE *f = fopen(argv[1], "rb");
    if (!f) return 2;
    int64_t dims[4];
    if (fread(dims, sizeof(int64_t), 4, f) != 4) return 2;
    const int64_t b = dims[0], l = dims[1], d = dims[2], n = dims[3];
    const size_t act = (size_t)(b * l * d), bc = (size_t)(b * l * n), st = (size_t)(b * d * n);
    float *x = read_block(f, act), *dt = read_block(f, act), *z = read_block(f, act);
    float *B = read_block(f, bc), *C = read_block(f, bc);
    float *A = read_block(f, (size_t)(d * n)), *D = read_block(f, (size_t)d), *bias = read_block(f, (size_t)d);
    float *x1 = read_block(f, (size_t)(b * d)), *dt1 = read_block(f, (size_t)(b * d));
    float *z1 = read_block(f, (size_t)(b * d)), *B1 = read_block(f, (size_t)(b * n));
    float *C1 = read_block(f, (size_t)(b * n));
    fclose(f);
    if (!x || !dt || !z || !B || !C || !A || !D || !bias || !x1 || !dt1 || !z1 || !B1 || !C1) return 2;

    if (jamba_ssm_abi_version() != JAMBA_SSM_ABI_VERSION) return 3;
    void *dx = dev_copy(x, act), *ddt = dev_copy(dt, act), *dz = dev_copy(z, act);
    void *dB = dev_copy(B, bc), *dC = dev_copy(C, bc);
    void *dA = dev_copy(A, (size_t)(d * n)), *dD = dev_copy(D, (size_t)d), *dbias = dev_copy(bias, (size_t)d);
    void *dout = dev_copy(NULL, act), *dhf = dev_copy(NULL, st);
    void *dx1 = dev_copy(x1, (size_t)(b * d)), *ddt1 = dev_copy(dt1, (size_t)(b * d));
    void *dz1 = dev_copy(z1, (size_t)(b * d)), *dB1 = dev_copy(B1, (size_t)(b * n));
    void *dC1 = dev_copy(C1, (size_t)(b * n)), *dout1 = dev_copy(NULL, (size_t)(b * d));
    if (!dx || !ddt || !dz || !dB || !dC || !dA || !dD || !dbias || !dout || !dhf || !dx1 || !ddt1 ||
        !dz1 || !dB1 || !dC1 || !dout1)
        return 4;

    jamba_ssm_scan_params p = {0};
    p.struct_size = sizeof(p);
    p.batch = b; p.seqlen = l; p.d_inner = d; p.d_state = n;
    p.io_dtype = JAMBA_SSM_F32;
    p.delta_softplus = 1;
    p.x = dx; p.delta = ddt; p.z = dz; p.B = dB; p.C = dC;
    p.A = (const float *)dA; p.D = (const float *)dD; p.delta_bias = (const float *)dbias;
    p.out = dout; p.h_final = (float *)dhf;
    /* the optional workspace: the call's status word, zero-filled once */
    const size_t ws_bytes = jamba_ssm_scan_workspace_size(b, l, d, n);
    void *ws = NULL;
    if (ws_bytes < JAMBA_SSM_STATUS_BYTES || cudaMalloc(&ws, ws_bytes) != cudaSuccess ||
        cudaMemset(ws, 0, ws_bytes) != cudaSuccess)
        return 4;
    p.workspace = ws; p.workspace_bytes = ws_bytes;
    if (check(jamba_ssm_scan(&p, NULL), "jamba_ssm_scan")) return 5;
    if (check(jamba_ssm_get_status(ws, NULL), "jamba_ssm_get_status (workspace)")) return 5;

    jamba_ssm_state_update_params u = {0};
    u.struct_size = sizeof(u);
    u.batch = b; u.d_inner = d; u.d_state = n;
    u.io_dtype = JAMBA_SSM_F32;
    u.delta_softplus = 1;
    u.state = (float *)dhf;
    u.x = dx1; u.delta = ddt1; u.z = dz1; u.B = dB1; u.C = dC1;
    u.A = (const float *)dA; u.D = (const float *)dD; u.delta_bias = (const float *)dbias;
    u.out = dout1;
    /* the state is copied first so that both the scan's final state and the
       state after the decode step can be written out */
    float *hf = (float *)malloc(st * sizeof(float));
    if (!hf || cudaMemcpy(hf, dhf, st * sizeof(float), cudaMemcpyDeviceToHost) != cudaSuccess) return 6;
    if (check(jamba_ssm_state_update(&u, NULL), "jamba_ssm_state_update")) return 5;
    if (check(jamba_ssm_get_status(NULL, NULL), "jamba_ssm_get_status")) return 5;

    float *out = (float *)malloc(act * sizeof(float)), *out1 = (float *)malloc((size_t)(b * d) * sizeof(float));
    float *st1 = (float *)malloc(st * sizeof(float));
    if (!out || !out1 || !st1) return 6;
    if (cudaMemcpy(out, dout, act * sizeof(float), cudaMemcpyDeviceToHost) != cudaSuccess ||
        cudaMemcpy(out1, dout1, (size_t)(b * d) * sizeof(float), cudaMemcpyDeviceToHost) != cudaSuccess ||
        cudaMemcpy(st1, dhf, st * sizeof(float), cudaMemcpyDeviceToHost) != cudaSuccess)
        return 6;
    FILE *o = fopen(argv[2], "wb");
    if (!o) return 7;
    fwrite(out, sizeof(float), act, o);
    fwrite(hf, sizeof(float), st, o);
    fwrite(out1, sizeof(float), (size_t)(b * d), o);
    fwrite(st1, sizeof(float), st, o);
    fclose(o);
    return 0;
}
