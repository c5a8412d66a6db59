// mufu_rate.cu -- throughput of the special-function unit (MUFU) on sm_100a:
// ex2.approx.ftz.f32 and rcp.approx.ftz.f32 operations per SM per clock.
//
// One CTA of 1024 threads per SM; every thread runs 8 independent chains of
// `iters` MUFU operations (each followed by one FADD that keeps the value in
// range and makes the next operation depend on it), so the MUFU pipe, not the
// chain latency, sets the rate.  Each CTA times itself with the SM cycle
// counter; the program prints the median over CTAs of
//     (threads x chains x iters) / (end cycle - start cycle)
// and the SM clock that the same interval implies against globaltimer.
// Usage: mufu_rate [iters]  ->  "ex2 <ops/clk/SM> rcp <ops/clk/SM> mhz <MHz> sms <n>"
#include <cuda_runtime.h>

#include <algorithm>
#include <cstdio>
#include <cstdlib>
#include <vector>

constexpr int kThreads = 1024, kChains = 8;

template <int OP>
__device__ __forceinline__ float mufu(float x) {
    float y;
    if (OP == 0)
        asm volatile("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    else
        asm volatile("rcp.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

__device__ __forceinline__ unsigned long long global_ns() {
    unsigned long long t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

template <int OP>
__global__ void __launch_bounds__(kThreads, 1)
    mufu_kernel(int iters, float seed, float *sink, long long *cycles, unsigned long long *ns) {
    float v[kChains];
#pragma unroll
    for (int c = 0; c < kChains; ++c) v[c] = seed * (c + 1) * 1e-3f - 0.25f;
    __syncthreads();
    const long long c0 = clock64();
    const unsigned long long t0 = global_ns();
    for (int i = 0; i < iters; ++i) {
#pragma unroll
        for (int c = 0; c < kChains; ++c) v[c] = mufu<OP>(v[c]) - (OP == 0 ? 1.5f : 0.75f);
    }
    __syncthreads();
    const long long c1 = clock64();
    const unsigned long long t1 = global_ns();
    float s = 0.0f;
#pragma unroll
    for (int c = 0; c < kChains; ++c) s += v[c];
    if (s == 12345.0f) sink[threadIdx.x] = s;  // keeps the chains live
    if (threadIdx.x == 0) {
        cycles[blockIdx.x] = c1 - c0;
        ns[blockIdx.x] = t1 - t0;
    }
}

template <int OP>
static double rate(int sms, int iters, double *mhz) {
    float *sink;
    long long *cyc;
    unsigned long long *ns;
    cudaMalloc(&sink, kThreads * sizeof(float));
    cudaMalloc(&cyc, sms * sizeof(long long));
    cudaMalloc(&ns, sms * sizeof(unsigned long long));
    mufu_kernel<OP><<<sms, kThreads>>>(iters / 10, 1.0f, sink, cyc, ns);  // warm-up
    mufu_kernel<OP><<<sms, kThreads>>>(iters, 1.0f, sink, cyc, ns);
    if (cudaDeviceSynchronize() != cudaSuccess) {
        std::fprintf(stderr, "kernel failed\n");
        std::exit(2);
    }
    std::vector<long long> c(sms);
    std::vector<unsigned long long> t(sms);
    cudaMemcpy(c.data(), cyc, sms * sizeof(long long), cudaMemcpyDeviceToHost);
    cudaMemcpy(t.data(), ns, sms * sizeof(unsigned long long), cudaMemcpyDeviceToHost);
    std::vector<double> r(sms), f(sms);
    const double ops = double(kThreads) * kChains * iters;
    for (int i = 0; i < sms; ++i) {
        r[i] = ops / double(c[i]);
        f[i] = double(c[i]) / double(t[i]) * 1e3;  // cycles per ns * 1000 = MHz
    }
    std::sort(r.begin(), r.end());
    std::sort(f.begin(), f.end());
    *mhz = f[sms / 2];
    cudaFree(sink);
    cudaFree(cyc);
    cudaFree(ns);
    return r[sms / 2];
}

int main(int argc, char **argv) {
    const int iters = argc > 1 ? std::atoi(argv[1]) : 4096;
    int sms = 0;
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, 0);
    double mhz_e = 0, mhz_r = 0;
    const double e = rate<0>(sms, iters, &mhz_e);
    const double r = rate<1>(sms, iters, &mhz_r);
    std::printf("ex2 %.3f rcp %.3f mhz %.0f sms %d\n", e, r, 0.5 * (mhz_e + mhz_r), sms);
    return 0;
}
