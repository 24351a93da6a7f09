// device_util.cuh -- small sm_100a device helpers: cluster barrier, distributed
// shared-memory stores, exact power-of-two scaling, error flag.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

namespace semicrf {

__device__ __forceinline__ uint32_t cluster_rank()
{
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
    return r;
}

// All threads of all CTAs in the cluster: release our shared-memory writes
// (local and remote), then wait for everyone and acquire theirs.
__device__ __forceinline__ void cluster_barrier()
{
    asm volatile("barrier.cluster.arrive.release.aligned;\n\t"
                 "barrier.cluster.wait.acquire.aligned;" ::: "memory");
}

// Store a double into the shared memory of CTA `rank` of this cluster, at the
// same offset as `local` has in ours.
__device__ __forceinline__ void st_cluster_f64(const double *local, uint32_t rank, double v)
{
    uint32_t laddr = static_cast<uint32_t>(__cvta_generic_to_shared(local));
    uint32_t raddr;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(raddr) : "r"(laddr), "r"(rank));
    asm volatile("st.shared::cluster.f64 [%0], %1;" ::"r"(raddr), "d"(v) : "memory");
}

// Unbiased binary exponent of a positive normal double (floor(log2 v)), read
// from its bit pattern.  Zero, subnormals and non-finite values give 0.
__device__ __forceinline__ int exponent_of(double v)
{
    long long bits = __double_as_longlong(v);
    int e = static_cast<int>((bits >> 52) & 0x7ff);
    if (e == 0 || e == 0x7ff) return 0;
    return e - 1023;
}

// 2^h as a double for |h| <= 1022, built from its bit pattern (exact).
__device__ __forceinline__ double pow2(int h)
{
    return __longlong_as_double(static_cast<long long>(h + 1023) << 52);
}

// Record the first device-side error in the workspace status word.
__device__ __forceinline__ void set_status(int32_t *status, int code)
{
    atomicCAS(reinterpret_cast<int *>(status), 0, code);
}

// 2^h with h clamped to the normal range [-1022, 1023] (branch free).
__device__ __forceinline__ double pow2c(int h)
{
    h = max(-1022, min(1023, h));
    return __longlong_as_double(static_cast<long long>(h + 1023) << 52);
}

// x * 2^h, exact unless the result over/underflows; |h| up to ~3000.
__device__ __forceinline__ double scale2(double x, int h)
{
    while (h > 1000) {
        x *= pow2(1000);
        h -= 1000;
    }
    while (h < -1000) {
        x *= pow2(-1000);
        h += 1000;
    }
    return x * pow2(h);
}

// x * 2^h for |h| <= 2044 without branches (two exact power-of-two factors).
__device__ __forceinline__ double scale2c(double x, int h)
{
    const int h1 = h / 2;
    return (x * pow2c(h1)) * pow2c(h - h1);
}

// Asynchronous global -> shared copies (Ampere-and-later cp.async), grouped.
__device__ __forceinline__ void cp_async8(void *smem, const void *gmem)
{
    const uint32_t s = static_cast<uint32_t>(__cvta_generic_to_shared(smem));
    asm volatile("cp.async.ca.shared.global [%0], [%1], 8;" ::"r"(s), "l"(gmem) : "memory");
}

__device__ __forceinline__ void cp_async4(void *smem, const void *gmem)
{
    const uint32_t s = static_cast<uint32_t>(__cvta_generic_to_shared(smem));
    asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(s), "l"(gmem) : "memory");
}

__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }

template <int N>
__device__ __forceinline__ void cp_async_wait()
{
    asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

// v mod K in [0, K) for any sign of v
__device__ __forceinline__ int mod_pos(int v, int K)
{
    v %= K;
    return v < 0 ? v + K : v;
}

constexpr double kLn2 = 0.69314718055994530941723212145818;

}  // namespace semicrf
