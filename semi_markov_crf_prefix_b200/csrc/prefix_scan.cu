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

}  // namespace

cudaError_t launch_prefix_scan(const ScanArgs &a, cudaStream_t st, int *launches)
{
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
