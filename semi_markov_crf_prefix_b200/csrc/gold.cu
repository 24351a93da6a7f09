// gold.cu -- score of given segmentations and its gradient (the term of the
// negative log-likelihood log Z - score(y*) that does not come from log Z;
// Streaming Structured Inference with Flash-SemiCRF, technical summary section 3:
// training by negative log-likelihood; section 2.A: segment content as a
// prefix-sum difference).
//
// One CTA per sequence.  Every thread takes the segment starts among its
// positions, finds the segment's end (the next start, at most K ahead, or L),
// checks that every position of the segment carries the segment's label, and
// adds S[e,c] - S[s,c] + D[e-s-1,c] (+ A[previous label, c] when s > 0).  The
// per-thread sums are added in a fixed tree order, so the score does not depend
// on scheduling.  The gradient counts transitions, durations and positions per
// label with integer atomics (exact), then applies the weights in sequence order.
#include "device_util.cuh"
#include "semicrf_internal.h"

namespace semicrf {
namespace {

constexpr int kGoldThreads = 256;

// Weight of sequence b in the gradient: wsign * g_b (g_b = 1 without weights).
__device__ __forceinline__ double gold_weight(const GoldArgs &a, int b)
{
    return a.wsign * (a.grad ? a.grad[b] : 1.0);
}

// End of the segment starting at s, or -1 if the segmentation is malformed there.
__device__ __forceinline__ int gold_segment_end(const GoldArgs &a, size_t pb, int s, int L, int c)
{
    if (c < 0 || c >= a.C) return -1;
    const int lim = min(L, s + a.K);
    int e = L;
    for (int t = s + 1; t < L; ++t) {
        if (a.seg_start[pb + t]) {
            e = t;
            break;
        }
        if (a.labels[pb + t] != c) return -1;
        if (t >= lim) return -1;   // longer than K
    }
    if (e - s > a.K) return -1;
    return e;
}

__global__ void __launch_bounds__(kGoldThreads) gold_score_kernel(GoldArgs a)
{
    __shared__ double part[kGoldThreads];
    const int b = blockIdx.x, tid = threadIdx.x;
    const int L = a.lengths[b];
    const bool ok_len = L >= 1 && L <= a.T;
    const size_t pb = (size_t)b * a.T;
    const size_t rowbase = (size_t)b * (a.T + 1);
    const int C = a.C;
    double acc = 0.0;
    bool bad = ok_len && a.seg_start[pb] == 0;
    if (ok_len) {
        for (int s = tid; s < L; s += kGoldThreads) {
            if (!a.seg_start[pb + s]) continue;
            const int c = a.labels[pb + s];
            const int e = gold_segment_end(a, pb, s, L, c);
            if (e < 0) {
                bad = true;
                continue;
            }
            acc += (a.S[(rowbase + e) * C + c] - a.S[(rowbase + s) * C + c]) + (double)a.D[(size_t)(e - s - 1) * C + c];
            if (s > 0) {
                const int cp = a.labels[pb + s - 1];
                if (cp >= 0 && cp < C) acc += (double)a.A[(size_t)cp * C + c];
            }
        }
    }
    part[tid] = acc;
    __syncthreads();
    for (int w = kGoldThreads / 2; w > 0; w >>= 1) {
        if (tid < w) part[tid] += part[tid + w];
        __syncthreads();
    }
    if (tid == 0) {
        if (!ok_len) set_status(a.status, SEMICRF_ERR_INVALID_LENGTH);
        a.score[b] = part[0];
        if (a.nll) a.nll[b] = a.logZ[b] - part[0];
    }
    if (bad) set_status(a.status, SEMICRF_ERR_INVALID_SEGMENTATION);
}

__global__ void __launch_bounds__(kGoldThreads) gold_count_kernel(GoldArgs a)
{
    const int b = blockIdx.x, tid = threadIdx.x;
    const int C = a.C, K = a.K;
    int32_t *cA = a.cntA + (size_t)b * C * C;
    int32_t *cD = a.cntD + (size_t)b * K * C;
    int32_t *cN = a.cntN + (size_t)b * C;
    for (int i = tid; i < C * C; i += kGoldThreads) cA[i] = 0;
    for (int i = tid; i < K * C; i += kGoldThreads) cD[i] = 0;
    for (int i = tid; i < C; i += kGoldThreads) cN[i] = 0;
    __syncthreads();
    const int L = a.lengths[b];
    if (L < 1 || L > a.T) {
        if (tid == 0) set_status(a.status, SEMICRF_ERR_INVALID_LENGTH);
        return;
    }
    const size_t pb = (size_t)b * a.T;
    bool bad = a.seg_start[pb] == 0;
    for (int s = tid; s < L; s += kGoldThreads) {
        if (!a.seg_start[pb + s]) continue;
        const int c = a.labels[pb + s];
        const int e = gold_segment_end(a, pb, s, L, c);
        if (e < 0) {
            bad = true;
            continue;
        }
        atomicAdd(&cD[(size_t)(e - s - 1) * C + c], 1);
        atomicAdd(&cN[c], e - s);
        if (s > 0) {
            const int cp = a.labels[pb + s - 1];
            if (cp >= 0 && cp < C) atomicAdd(&cA[(size_t)cp * C + c], 1);
        }
    }
    if (bad) set_status(a.status, SEMICRF_ERR_INVALID_SEGMENTATION);
}

// dA += sum_b g_b cntA[b],  dD += sum_b g_b cntD[b]   (sequence order)
__global__ void gold_param_kernel(GoldArgs a)
{
    const int nA = a.C * a.C, nD = a.K * a.C;
    for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < nA + nD; i += gridDim.x * blockDim.x) {
        double s = 0.0;
        if (i < nA) {
            for (int b = 0; b < a.B; ++b) s += gold_weight(a, b) * (double)a.cntA[(size_t)b * nA + i];
            a.dA[i] += s;
        } else {
            const int k = i - nA;
            for (int b = 0; b < a.B; ++b) s += gold_weight(a, b) * (double)a.cntD[(size_t)b * nD + k];
            a.dD[k] += s;
        }
    }
}

// dX[b,u,c] += g_b (1[labels[b,u] == c] - n_{b,c} / L_b)  for u < L_b
__global__ void gold_dx_kernel(GoldArgs a)
{
    const size_t n = (size_t)a.B * a.T * a.C;
    for (size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += (size_t)gridDim.x * blockDim.x) {
        const int c = (int)(i % a.C);
        const size_t bt = i / a.C;
        const int u = (int)(bt % a.T);
        const int b = (int)(bt / a.T);
        const int L = a.lengths[b];
        if (L < 1 || L > a.T || u >= L) continue;
        const double g = gold_weight(a, b);
        const double ind = a.labels[bt] == c ? 1.0 : 0.0;
        const double mean = (double)a.cntN[(size_t)b * a.C + c] / (double)L;
        a.dX[i] = (float)((double)a.dX[i] + g * (ind - mean));
    }
}

}  // namespace

cudaError_t launch_gold_score(const GoldArgs &a, cudaStream_t st, int *launches)
{
    prof_before(st);
    gold_score_kernel<<<a.B, kGoldThreads, 0, st>>>(a);
    prof_after(st);
    *launches += 1;
    return cudaGetLastError();
}

cudaError_t launch_gold_backward(const GoldArgs &a, cudaStream_t st, int *launches)
{
    prof_before(st);
    gold_count_kernel<<<a.B, kGoldThreads, 0, st>>>(a);
    prof_after(st);
    const int np = a.C * a.C + a.K * a.C;
    prof_before(st);
    gold_param_kernel<<<(np + 255) / 256, 256, 0, st>>>(a);
    prof_after(st);
    const size_t n = (size_t)a.B * a.T * a.C;
    int blocks = (int)((n + 255) / 256);
    if (blocks > device_sm_count() * 16) blocks = device_sm_count() * 16;
    prof_before(st);
    gold_dx_kernel<<<blocks, 256, 0, st>>>(a);
    prof_after(st);
    *launches += 3;
    return cudaGetLastError();
}

}  // namespace semicrf
