/*
 * ssd_client.c -- a plain C client of libjamba_ssm.so for the scalar-identity
 * variant (no Python, no torch): reads a problem from a binary file, moves it
 * to the device with the CUDA runtime, calls jamba_ssm_ssd_scan on bf16 data
 * through the C ABI, and writes the results back for the test to compare with
 * the oracle.
 *
 * Input file (little endian): int64 batch, seqlen, nheads, headdim, d_state;
 * then the raw bf16 bits of x, z [batch, seqlen, nheads * headdim], delta
 * [batch, seqlen, nheads], B, C [batch, seqlen, d_state]; then fp32 A
 * [nheads], D [nheads * headdim], delta_bias [nheads], h0 [batch, nheads *
 * headdim, d_state].
 * Output file: the raw bf16 bits of out [batch, seqlen, nheads * headdim],
 * then fp32 h_final [batch, nheads * headdim, d_state].
 * Exit status 0 on success; a nonzero status prints the library's message.
 */
#include <cuda_runtime.h>
#include <stdint.h>
#include <stdio.h>
#include <stdlib.h>

#include "jamba_ssm.h"

static void *read_dev(FILE *f, size_t bytes) {
    void *h = malloc(bytes ? bytes : 1), *d = NULL;
    if (!h || fread(h, 1, bytes, f) != bytes) return NULL;
    if (cudaMalloc(&d, bytes + 16) != cudaSuccess ||
        cudaMemcpy(d, h, bytes, cudaMemcpyHostToDevice) != cudaSuccess)
        return NULL;
    free(h);
    return d;
}

int main(int argc, char **argv) {
    if (argc != 3) return 2;
    FILE *f = fopen(argv[1], "rb");
    if (!f) return 2;
    int64_t dims[5];
    if (fread(dims, sizeof(int64_t), 5, f) != 5) return 2;
    const int64_t b = dims[0], l = dims[1], h = dims[2], p = dims[3], n = dims[4];
    const size_t act = (size_t)(b * l * h * p), dts = (size_t)(b * l * h), bc = (size_t)(b * l * n);
    const size_t st = (size_t)(b * h * p * n);
    void *dx = read_dev(f, act * 2), *dz = read_dev(f, act * 2), *ddt = read_dev(f, dts * 2);
    void *dB = read_dev(f, bc * 2), *dC = read_dev(f, bc * 2);
    void *dA = read_dev(f, (size_t)h * 4), *dD = read_dev(f, (size_t)(h * p) * 4);
    void *dbias = read_dev(f, (size_t)h * 4), *dh0 = read_dev(f, st * 4);
    fclose(f);
    void *dout = NULL, *dhf = NULL;
    if (!dx || !dz || !ddt || !dB || !dC || !dA || !dD || !dbias || !dh0 ||
        cudaMalloc(&dout, act * 2 + 16) != cudaSuccess || cudaMalloc(&dhf, st * 4 + 16) != cudaSuccess)
        return 4;

    if (jamba_ssm_abi_version() != JAMBA_SSM_ABI_VERSION) return 3;
    jamba_ssm_ssd_params q = {0};
    q.struct_size = sizeof(q);
    q.batch = b; q.seqlen = l; q.nheads = h; q.headdim = p; q.d_state = n;
    q.io_dtype = JAMBA_SSM_BF16;
    q.delta_softplus = 1;
    q.x = dx; q.delta = ddt; q.z = dz; q.B = dB; q.C = dC;
    q.A = (const float *)dA; q.D = (const float *)dD; q.delta_bias = (const float *)dbias;
    q.h0 = (const float *)dh0;
    q.out = dout; q.h_final = (float *)dhf;
    jamba_ssm_status s = jamba_ssm_ssd_scan(&q, NULL);
    if (s == JAMBA_SSM_OK) s = jamba_ssm_get_status(NULL, NULL);
    if (s != JAMBA_SSM_OK) {
        fprintf(stderr, "jamba_ssm_ssd_scan: %s (cuda %d)\n", jamba_ssm_status_string(s),
                jamba_ssm_last_cuda_error());
        return 5;
    }
    void *out = malloc(act * 2), *hf = malloc(st * 4);
    if (!out || !hf || cudaMemcpy(out, dout, act * 2, cudaMemcpyDeviceToHost) != cudaSuccess ||
        cudaMemcpy(hf, dhf, st * 4, cudaMemcpyDeviceToHost) != cudaSuccess)
        return 6;
    FILE *o = fopen(argv[2], "wb");
    if (!o) return 7;
    fwrite(out, 1, act * 2, o);
    fwrite(hf, 1, st * 4, o);
    fclose(o);
    return 0;
}
