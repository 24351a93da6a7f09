// prefix_scan.cu -- centring baseline and prefix sums of centred emissions.
//
// Streaming Structured Inference with Flash-SemiCRF, technical summary 2.A
// (segment content as a difference of two cumulative scores) and 2.C (a
// per-sequence, per-label emission baseline nu[b,c] is subtracted before the
// prefix sums, keeping |S| at O(sqrt(T)) instead of O(T)):
//   nu[b,c]  = (1/L_b) sum_{t<L_b} x[b,t,c]
//   S[b,0,c] = 0,  S[b,t+1,c] = S[b,t,c] + (x[b,t,c] - nu[b,c])   (t < L_b)
//   S[b,t,c] = S[b,L_b,c]                                          (t > L_b)
//
// Three HBM-bound passes over a chunked t axis (chunks of R rows, NCH per
// sequence): (1) per-chunk label sums, (2) nu and chunk start values, (3) the
// in-chunk running sums, written as float64.  Pass 3 re-reads the chunk pass 1
// read; with R*C*4 bytes per chunk and chunks launched in order the re-read is
// mostly served from L2.  Rows t >= L_b of x are never read.  All sums are
// float64.
//
// Short sequences with C <= 32 (T <= 1024) take one launch instead: one CTA per
// sequence, label c on lane c of each warp, the 16 warps on 16 consecutive row
// ranges; the range totals meet in shared memory, give nu and each range's
// starting value, and every warp sweeps its range again (its first 32 rows kept
// in registers, the rest re-read from L1/L2) to write S.
#include "device_util.cuh"
#include "semicrf_internal.h"

namespace semicrf {
namespace {

constexpr int kScanThreads = 256;

__device__ __forceinline__ int chunk_rows(int T, int NCH) { return (T + NCH - 1) / NCH; }

// Pass 1: part[b][ch][c] = sum of x[b,t,c] over the chunk's valid rows.
__global__ void __launch_bounds__(kScanThreads) scan_partials(ScanArgs a)
{
    const int ch = blockIdx.x, b = blockIdx.y;
    const int L = a.lengths[b];
    if (L < 1 || L > a.T) {
        if (ch == 0 && threadIdx.x == 0) set_status(a.status, SEMICRF_ERR_INVALID_LENGTH);
        return;
    }
    const int R = chunk_rows(a.T, a.NCH);
    const int t0 = ch * R;
    const int t1 = min(t0 + R, L);
    const float *xb = a.x + (size_t)b * a.T * a.C;
    for (int c = threadIdx.x; c < a.C; c += blockDim.x) {
        double s0 = 0.0, s1 = 0.0, s2 = 0.0, s3 = 0.0;
        int t = t0;
        for (; t + 4 <= t1; t += 4) {
            float v0 = __ldg(xb + (size_t)(t + 0) * a.C + c);
            float v1 = __ldg(xb + (size_t)(t + 1) * a.C + c);
            float v2 = __ldg(xb + (size_t)(t + 2) * a.C + c);
            float v3 = __ldg(xb + (size_t)(t + 3) * a.C + c);
            s0 += v0; s1 += v1; s2 += v2; s3 += v3;
        }
        for (; t < t1; ++t) s0 += __ldg(xb + (size_t)t * a.C + c);
        a.part[((size_t)b * a.NCH + ch) * a.C + c] = (s0 + s1) + (s2 + s3);
    }
}

// Pass 2: nu and the value of S at each chunk's first row (stored over part).
__global__ void __launch_bounds__(kScanThreads) scan_offsets(ScanArgs a)
{
    const int b = blockIdx.x;
    const int L = a.lengths[b];
    if (L < 1 || L > a.T) return;
    const int R = chunk_rows(a.T, a.NCH);
    for (int c = threadIdx.x; c < a.C; c += blockDim.x) {
        double tot = 0.0;
        for (int ch = 0; ch < a.NCH; ++ch) tot += a.part[((size_t)b * a.NCH + ch) * a.C + c];
        const double nu = tot / (double)L;
        a.nu[(size_t)b * a.C + c] = nu;
        double run = 0.0;
        for (int ch = 0; ch < a.NCH; ++ch) {
            double p = a.part[((size_t)b * a.NCH + ch) * a.C + c];
            int t0 = ch * R;
            int nrows = max(0, min(t0 + R, L) - t0);
            a.part[((size_t)b * a.NCH + ch) * a.C + c] = run;   // S[t0] = sum_{u<t0} (x - nu)
            run += p - (double)nrows * nu;
        }
    }
}

// Pass 3: running sums inside each chunk; the chunk holding row L_b-1 also fills
// the rows past L_b with S[L_b].
__global__ void __launch_bounds__(kScanThreads) scan_apply(ScanArgs a)
{
    const int ch = blockIdx.x, b = blockIdx.y;
    const int L = a.lengths[b];
    if (L < 1 || L > a.T) return;
    const int R = chunk_rows(a.T, a.NCH);
    const int t0 = ch * R;
    if (t0 >= L) return;
    const int t1 = min(t0 + R, L);
    const float *xb = a.x + (size_t)b * a.T * a.C;
    double *Sb = a.S + (size_t)b * (a.T + 1) * a.C;
    for (int c = threadIdx.x; c < a.C; c += blockDim.x) {
        const double nu = a.nu[(size_t)b * a.C + c];
        double s = a.part[((size_t)b * a.NCH + ch) * a.C + c];
        if (ch == 0) Sb[c] = 0.0;
        int t = t0;
        for (; t + 4 <= t1; t += 4) {
            float v0 = __ldg(xb + (size_t)(t + 0) * a.C + c);
            float v1 = __ldg(xb + (size_t)(t + 1) * a.C + c);
            float v2 = __ldg(xb + (size_t)(t + 2) * a.C + c);
            float v3 = __ldg(xb + (size_t)(t + 3) * a.C + c);
            s += ((double)v0 - nu); Sb[(size_t)(t + 1) * a.C + c] = s;
            s += ((double)v1 - nu); Sb[(size_t)(t + 2) * a.C + c] = s;
            s += ((double)v2 - nu); Sb[(size_t)(t + 3) * a.C + c] = s;
            s += ((double)v3 - nu); Sb[(size_t)(t + 4) * a.C + c] = s;
        }
        for (; t < t1; ++t) {
            s += ((double)__ldg(xb + (size_t)t * a.C + c) - nu);
            Sb[(size_t)(t + 1) * a.C + c] = s;
        }
        if (t1 == L)
            for (int u = L + 1; u <= a.T; ++u) Sb[(size_t)u * a.C + c] = s;
    }
}

constexpr int kSingleMaxT = 1024;
constexpr int kSingleGroups = 16;   // warps per CTA, one row range each

__global__ void __launch_bounds__(32 * kSingleGroups) scan_single(ScanArgs a)
{
    __shared__ double part[kSingleGroups][32];
    __shared__ double nu_s[32];
    __shared__ double last[32];
    const int b = blockIdx.x, lane = threadIdx.x & 31, grp = threadIdx.x >> 5;
    const int L = a.lengths[b];
    if (L < 1 || L > a.T) {
        if (threadIdx.x == 0) set_status(a.status, SEMICRF_ERR_INVALID_LENGTH);
        return;
    }
    const int C = a.C;
    const bool act = lane < C;
    const int R = (L + kSingleGroups - 1) / kSingleGroups;
    const int t0 = min(grp * R, L), t1 = min(t0 + R, L);
    const float *xb = a.x + (size_t)b * a.T * C + min(lane, C - 1);
    // the range's first kCache rows stay in registers for the second sweep
    constexpr int kCache = 32;
    float v[kCache];
    double s0 = 0.0, s1 = 0.0, s2 = 0.0, s3 = 0.0;
#pragma unroll
    for (int k = 0; k < kCache; ++k) v[k] = __ldg(xb + (size_t)min(t0 + k, L - 1) * C);   // clamped: no branch
#pragma unroll
    for (int k = 0; k < kCache; ++k) v[k] = (act && t0 + k < t1) ? v[k] : 0.0f;
#pragma unroll
    for (int k = 0; k < kCache; k += 4) {
        s0 += (double)v[k];
        s1 += (double)v[k + 1];
        s2 += (double)v[k + 2];
        s3 += (double)v[k + 3];
    }
    if (act) {
        int t = t0 + kCache;
        for (; t + 8 <= t1; t += 8) {
            float u[8];
#pragma unroll
            for (int k = 0; k < 8; ++k) u[k] = __ldg(xb + (size_t)(t + k) * C);
            s0 += (double)u[0] + (double)u[4];
            s1 += (double)u[1] + (double)u[5];
            s2 += (double)u[2] + (double)u[6];
            s3 += (double)u[3] + (double)u[7];
        }
        for (; t < t1; ++t) s0 += __ldg(xb + (size_t)t * C);
    }
    part[grp][lane] = (s0 + s1) + (s2 + s3);
    __syncthreads();
    if (grp == 0) {
        double tot = 0.0;
        for (int g = 0; g < kSingleGroups; ++g) tot += part[g][lane];
        nu_s[lane] = tot / (double)L;
    }
    __syncthreads();
    const double nu = nu_s[lane];
    double run = 0.0;   // S at row t0: the earlier ranges, centred
    for (int g = 0; g < grp; ++g) {
        const int g0 = min(g * R, L), g1 = min(g0 + R, L);
        run += part[g][lane] - (double)(g1 - g0) * nu;
    }
    double *Sb = a.S + (size_t)b * (a.T + 1) * C + lane;
    if (act) {
        if (grp == 0) {
            Sb[0] = 0.0;
            a.nu[(size_t)b * C + lane] = nu;
        }
#pragma unroll
        for (int k = 0; k < kCache; ++k) {
            if (t0 + k < t1) {
                run += (double)v[k] - nu;
                Sb[(size_t)(t0 + k + 1) * C] = run;
            }
        }
        int t = t0 + kCache;
        for (; t + 4 <= t1; t += 4) {
            float u[4];
#pragma unroll
            for (int k = 0; k < 4; ++k) u[k] = __ldg(xb + (size_t)(t + k) * C);
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                run += (double)u[k] - nu;
                Sb[(size_t)(t + k + 1) * C] = run;
            }
        }
        for (; t < t1; ++t) {
            run += (double)__ldg(xb + (size_t)t * C) - nu;
            Sb[(size_t)(t + 1) * C] = run;
        }
        if (t0 < t1 && t1 == L) last[lane] = run;   // the range holding row L-1
    }
    __syncthreads();
    if (act)
        for (int u = L + 1 + grp; u <= a.T; u += kSingleGroups) Sb[(size_t)u * C] = last[lane];
}

}  // namespace

cudaError_t launch_prefix_scan(const ScanArgs &a, cudaStream_t st, int *launches)
{
    if (a.C <= 32 && a.T <= kSingleMaxT) {
        prof_before(st);
        scan_single<<<a.B, 32 * kSingleGroups, 0, st>>>(a);
        prof_after(st);
        *launches += 1;
        return cudaGetLastError();
    }
    dim3 g1(a.NCH, a.B);
    prof_before(st);
    scan_partials<<<g1, kScanThreads, 0, st>>>(a);
    prof_after(st);
    prof_before(st);
    scan_offsets<<<a.B, kScanThreads, 0, st>>>(a);
    prof_after(st);
    prof_before(st);
    scan_apply<<<g1, kScanThreads, 0, st>>>(a);
    prof_after(st);
    *launches += 3;
    return cudaGetLastError();
}

}  // namespace semicrf
