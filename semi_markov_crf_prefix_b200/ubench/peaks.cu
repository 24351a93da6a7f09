// peaks.cu -- throughput of the arithmetic units the semi-CRF chains are bound by,
// measured on the GPU the program runs on: FP64 FMA, FP32 FMA and the MUFU
// (special-function unit) ex2.  Each thread runs NCH independent dependency
// chains so that latency is hidden; the grid fills every SM several times over.
// Prints one JSON object: operations per second for each unit and the launch
// shape.  Per-SM-per-clock figures need the SM clock during the run, which the
// Python driver (peaks.py) samples with nvidia-smi.
#include <cuda_runtime.h>
#include <stdio.h>
#include <stdlib.h>

namespace {

constexpr int NCH = 8;       // independent chains per thread

__global__ void __launch_bounds__(256) k_fp64(double *out, double b, double c, int iters)
{
    double a[NCH];
#pragma unroll
    for (int i = 0; i < NCH; ++i) a[i] = threadIdx.x * 1e-3 + i;
    for (int it = 0; it < iters; ++it) {
#pragma unroll
        for (int i = 0; i < NCH; ++i) a[i] = fma(a[i], b, c);
    }
    double s = 0.0;
#pragma unroll
    for (int i = 0; i < NCH; ++i) s += a[i];
    if (s == 12345.678) out[0] = s;   // keeps the chains live; never true for these inputs
}

__global__ void __launch_bounds__(256) k_fp32(float *out, float b, float c, int iters)
{
    float a[NCH];
#pragma unroll
    for (int i = 0; i < NCH; ++i) a[i] = threadIdx.x * 1e-3f + i;
    for (int it = 0; it < iters; ++it) {
#pragma unroll
        for (int i = 0; i < NCH; ++i) a[i] = fmaf(a[i], b, c);
    }
    float s = 0.f;
#pragma unroll
    for (int i = 0; i < NCH; ++i) s += a[i];
    if (s == 12345.678f) out[0] = s;
}

// x <- 2^(-x): stays in (0.5, 1] for x in [0, 1], so no chain over- or underflows.
__global__ void __launch_bounds__(256) k_ex2(float *out, int iters)
{
    float a[NCH];
#pragma unroll
    for (int i = 0; i < NCH; ++i) a[i] = (threadIdx.x & 7) * 0.1f + i * 0.01f;
    for (int it = 0; it < iters; ++it) {
#pragma unroll
        for (int i = 0; i < NCH; ++i) {
            float y;
            asm volatile("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(-a[i]));
            a[i] = y;
        }
    }
    float s = 0.f;
#pragma unroll
    for (int i = 0; i < NCH; ++i) s += a[i];
    if (s == 12345.678f) out[0] = s;
}

#define CK(x)                                                                        \
    do {                                                                             \
        cudaError_t e_ = (x);                                                        \
        if (e_ != cudaSuccess) {                                                     \
            fprintf(stderr, "%s: %s\n", #x, cudaGetErrorString(e_));                 \
            return 1;                                                                \
        }                                                                            \
    } while (0)

template <typename F>
int time_it(F launch, int reps, double *ms_best)
{
    cudaEvent_t e0, e1;
    CK(cudaEventCreate(&e0));
    CK(cudaEventCreate(&e1));
    for (int i = 0; i < 3; ++i) launch();   // warm-up
    CK(cudaDeviceSynchronize());
    *ms_best = 1e30;
    for (int r = 0; r < reps; ++r) {
        CK(cudaEventRecord(e0));
        launch();
        CK(cudaEventRecord(e1));
        CK(cudaEventSynchronize(e1));
        float ms = 0.f;
        CK(cudaEventElapsedTime(&ms, e0, e1));
        if (ms < *ms_best) *ms_best = ms;
    }
    CK(cudaGetLastError());
    CK(cudaEventDestroy(e0));
    CK(cudaEventDestroy(e1));
    return 0;
}

}  // namespace

int main(int argc, char **argv)
{
    int reps = 10, waves = 8;
    if (argc > 1) reps = atoi(argv[1]);
    cudaDeviceProp p;
    CK(cudaGetDeviceProperties(&p, 0));
    const int nsm = p.multiProcessorCount;
    const int threads = 256;
    const int blocks = nsm * waves;   // 8 CTAs of 256 threads per SM: 64 warps resident
    double *d64;
    float *d32;
    CK(cudaMalloc(&d64, sizeof(double)));
    CK(cudaMalloc(&d32, sizeof(float)));
    // about 5 ms per launch at the nominal rates (64, 128 and 16 per SM per clock),
    // long against launch and ramp-up costs
    const int it64 = 32768, it32 = 131072, itx = 8192;
    const double per = (double)blocks * threads * NCH;
    double ms64, ms32, msx;
    if (time_it([&] { k_fp64<<<blocks, threads>>>(d64, 0.999999, 1e-7, it64); }, reps, &ms64)) return 1;
    if (time_it([&] { k_fp32<<<blocks, threads>>>(d32, 0.999999f, 1e-7f, it32); }, reps, &ms32)) return 1;
    if (time_it([&] { k_ex2<<<blocks, threads>>>(d32, itx); }, reps, &msx)) return 1;
    printf("{\"sms\": %d, \"blocks\": %d, \"threads\": %d, \"chains_per_thread\": %d, \"iters\": [%d, %d, %d], "
           "\"reps\": %d, \"fp64_fma_per_s\": %.6e, \"fp32_fma_per_s\": %.6e, \"mufu_ex2_per_s\": %.6e, "
           "\"ms_fp64\": %.4f, \"ms_fp32\": %.4f, \"ms_ex2\": %.4f}\n",
           nsm, blocks, threads, NCH, it64, it32, itx, reps, per * it64 / (ms64 * 1e-3), per * it32 / (ms32 * 1e-3),
           per * itx / (msx * 1e-3),
           ms64, ms32, msx);
    cudaFree(d64);
    cudaFree(d32);
    return 0;
}
