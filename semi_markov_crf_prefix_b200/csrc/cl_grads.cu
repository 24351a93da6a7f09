// cl_grads.cu -- gradients of the duration bias and the transitions as dense
// contractions over all positions, from the rows the cluster backward chain
// stores (Streaming Structured Inference with Flash-SemiCRF, abstract: exact
// gradients; technical summary 2.C: marginals from forward and backward scores).
//
//   dD[d-1,c] = exp(D[d-1,c]) sum_b g_b sum_s  X[b,s,c] Y[b,s+d,c] 2^(rb[b,s+d,c] - rb[b,s+1,c])
//   dA[c,c2]  = exp(A[c,c2])  sum_b g_b sum_{s=1..L_b-1} a2[b,s,c] bp[b,s,c2]
// where, with at/al the forward scores, S the prefix sums and log Z = ln2 kZ + logn:
//   X[s,c]  = exp(at[s,c] - S[s,c] - log Z + ln2 rb[s+1,c])    (from cU, eU; s = 0: U = 1)
//   Y[t,c]  = V[t,c], stored by the backward at its reference rb[t,c]
//   a2[s,c] = exp(al[s,c] - log Z + ln2 kb[s])                  (from cA, eA)
//   bp[s,c2]= the normalised backward score of a segment of label c2 starting at s
// so X Y 2^(...) is the marginal of one segment (without exp D) and a2 bp the
// marginal of one transition (without exp A).  The power-of-two factor is 1
// unless the label's column was rebased between s+1 and s+d; a chunk checks that
// once per label and takes the plain FMA path when it holds.
//
// Layout: each CTA owns a 32 x 32 tile of outputs ((d, c) or (c, c2)) and a
// split z of the (sequence, 32-position chunk) list, which it walks chunk by
// chunk, staging the chunk's rows in shared memory; it writes its tile of
// partial sums to part*[z].  A last kernel adds the splits in order (the
// result does not depend on scheduling) and applies exp(D), exp(A).
#include <math.h>

#include "device_util.cuh"
#include "semicrf_internal.h"

namespace semicrf {
namespace {

constexpr int kCh = 32;    // start positions per chunk
constexpr int kTile = 32;  // output tile edge

__global__ void __launch_bounds__(256) dur_grad_kernel(FbArgs a)
{
    __shared__ double xs[kCh][kTile];
    __shared__ int rs[kCh][kTile];
    __shared__ double ys[kCh + kTile][kTile];
    __shared__ int ry[kCh + kTile][kTile];
    __shared__ int uni[kTile];
    const int K = a.K, C = a.C, T = a.T;
    const int z = blockIdx.x, c0 = blockIdx.y * kTile, d0 = 1 + blockIdx.z * kTile;   // d is 1-based
    const int tid = threadIdx.x, lc = tid & 31, dq = tid >> 5;
    const int c = c0 + lc;
    const bool c_ok = c < C;
    const int nch = (T + kCh - 1) / kCh;
    const long long Q = (long long)a.B * nch;
    double acc[4] = {0.0, 0.0, 0.0, 0.0};
    for (long long q = z; q < Q; q += a.nsD) {
        const int b = (int)(q / nch), s0 = (int)(q % nch) * kCh;
        const int L = a.lengths[b];
        if (L < 1 || L > T || s0 >= L) continue;   // uniform over the CTA
        const size_t rowbase = (size_t)b * (T + 1);
        const double g = a.grad ? a.grad[b] : 1.0;
        const int kZ = a.lz[b].k;
        const double cz = exp(-a.lz[b].logn);
        __syncthreads();   // previous chunk's reads are done
        // start factors X for s in [s0, s0 + kCh), zero beyond L - 1
        for (int i = tid; i < kCh * kTile; i += 256) {
            const int si = i / kTile, l2 = i % kTile, s = s0 + si, cc = c0 + l2;
            double x = 0.0;
            int r = INT_MIN;
            if (s <= L - 1 && cc < C) {
                r = a.rbst[(rowbase + s + 1) * C + cc];
                x = (s == 0) ? scale2c(cz, r - kZ)
                             : scale2c(a.cU[(rowbase + s) * C + cc], a.eU[(rowbase + s) * C + cc] + r);
                x *= g;
            }
            xs[si][l2] = x;
            rs[si][l2] = r;
        }
        // end rows V for t in [s0 + d0, s0 + d0 + kCh + kTile), zero beyond L
        for (int i = tid; i < (kCh + kTile) * kTile; i += 256) {
            const int ti = i / kTile, l2 = i % kTile, t = s0 + d0 + ti, cc = c0 + l2;
            double y = 0.0;
            int r = INT_MIN;
            if (t <= L && cc < C) {
                y = a.Vst[(rowbase + t) * C + cc];
                r = a.rbst[(rowbase + t) * C + cc];
            }
            ys[ti][l2] = y;
            ry[ti][l2] = r;
        }
        __syncthreads();
        if (tid < kTile) {
            // one reference for the whole chunk of this label?
            int lo = INT_MAX, hi = INT_MIN;
            for (int si = 0; si < kCh; ++si) {
                const int r = rs[si][tid];
                if (r != INT_MIN) {
                    lo = min(lo, r);
                    hi = max(hi, r);
                }
            }
            for (int ti = 0; ti < kCh + kTile; ++ti) {
                const int r = ry[ti][tid];
                if (r != INT_MIN) {
                    lo = min(lo, r);
                    hi = max(hi, r);
                }
            }
            uni[tid] = lo >= hi;
        }
        __syncthreads();
        if (uni[lc]) {
#pragma unroll 4
            for (int si = 0; si < kCh; ++si) {
                const double x = xs[si][lc];
#pragma unroll
                for (int k = 0; k < 4; ++k) acc[k] = fma(x, ys[si + dq + 8 * k][lc], acc[k]);
            }
        } else {
            for (int si = 0; si < kCh; ++si) {
                const double x = xs[si][lc];
                const int r = rs[si][lc];
                if (r == INT_MIN) continue;
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                    const int ti = si + dq + 8 * k;
                    const double y = ys[ti][lc];
                    if (y != 0.0) acc[k] += scale2c(x * y, ry[ti][lc] - r);
                }
            }
        }
    }
#pragma unroll
    for (int k = 0; k < 4; ++k) {
        const int d = d0 + dq + 8 * k;
        if (d <= K && c_ok) a.partD[((size_t)z * K + (d - 1)) * C + c] = acc[k];
    }
}

__global__ void __launch_bounds__(256) trans_grad_kernel(FbArgs a)
{
    __shared__ double as[kCh][kTile];
    __shared__ double bs[kCh][kTile];
    const int C = a.C, T = a.T;
    const int z = blockIdx.x, c0 = blockIdx.y * kTile, e0 = blockIdx.z * kTile;
    const int tid = threadIdx.x, ci = tid >> 3, cj = tid & 7;
    const int nch = (T + kCh - 1) / kCh;
    const long long Q = (long long)a.B * nch;
    double acc[4] = {0.0, 0.0, 0.0, 0.0};
    for (long long q = z; q < Q; q += a.nsA) {
        const int b = (int)(q / nch), s0 = (int)(q % nch) * kCh;
        const int L = a.lengths[b];
        if (L < 2 || L > T || s0 >= L - 1 + 1) continue;   // transitions at s in [1, L-1]
        const size_t rowbase = (size_t)b * (T + 1);
        const double g = a.grad ? a.grad[b] : 1.0;
        __syncthreads();
        for (int i = tid; i < kCh * kTile; i += 256) {
            const int si = i / kTile, l2 = i % kTile, s = s0 + si;
            const bool ok = s >= 1 && s <= L - 1;
            double x = 0.0, y = 0.0;
            if (ok && c0 + l2 < C) {
                const size_t ix = (rowbase + s) * C + c0 + l2;
                x = g * scale2c(a.cA[ix], a.eA[rowbase + s] + a.kbst[rowbase + s]);
            }
            if (ok && e0 + l2 < C) y = a.bpst[(rowbase + s) * C + e0 + l2];
            as[si][l2] = x;
            bs[si][l2] = y;
        }
        __syncthreads();
#pragma unroll 4
        for (int si = 0; si < kCh; ++si) {
            const double x = as[si][ci];
#pragma unroll
            for (int k = 0; k < 4; ++k) acc[k] = fma(x, bs[si][cj + 8 * k], acc[k]);
        }
    }
    const int c = c0 + ci;
#pragma unroll
    for (int k = 0; k < 4; ++k) {
        const int e = e0 + cj + 8 * k;
        if (c < C && e < C) a.partA[((size_t)z * C + c) * C + e] = acc[k];
    }
}

// dD = exp(D) * sum_z partD[z],  dA = exp(A) * sum_z partA[z]   (splits in order)
__global__ void cl_finalise_params(FbArgs a)
{
    const int nA = a.C * a.C, nD = a.K * a.C;
    for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < nA + nD; i += gridDim.x * blockDim.x) {
        if (i < nA) {
            double s = 0.0;
            for (int z = 0; z < a.nsA; ++z) s += a.partA[(size_t)z * nA + i];
            a.dA[i] = exp((double)a.A[i]) * s;
        } else {
            const int k = i - nA;
            double s = 0.0;
            for (int z = 0; z < a.nsD; ++z) s += a.partD[(size_t)z * nD + k];
            a.dD[k] = exp((double)a.D[k]) * s;
        }
    }
}

int ceil_div(long long a, long long b) { return (int)((a + b - 1) / b); }

}  // namespace

// Splits so that each contraction launches about four CTAs per SM.
void cl_grad_splits(int B, int T, int K, int C, int *nsD, int *nsA)
{
    const long long Q = (long long)B * ceil_div(T, kCh);
    const int tilesD = ceil_div(K, kTile) * ceil_div(C, kTile);
    const int tilesA = ceil_div(C, kTile) * ceil_div(C, kTile);
    long long d = ceil_div(4 * 148, tilesD), e = ceil_div(4 * 148, tilesA);
    *nsD = (int)(d < Q ? d : Q);
    *nsA = (int)(e < Q ? e : Q);
    if (*nsD < 1) *nsD = 1;
    if (*nsA < 1) *nsA = 1;
}

cudaError_t launch_cl_param_grads(const FbArgs &a, cudaStream_t st)
{
    prof_before(st);
    dur_grad_kernel<<<dim3(a.nsD, ceil_div(a.C, kTile), ceil_div(a.K, kTile)), 256, 0, st>>>(a);
    prof_after(st);
    prof_before(st);
    trans_grad_kernel<<<dim3(a.nsA, ceil_div(a.C, kTile), ceil_div(a.C, kTile)), 256, 0, st>>>(a);
    prof_after(st);
    const int n = a.C * a.C + a.K * a.C;
    prof_before(st);
    cl_finalise_params<<<(n + 255) / 256, 256, 0, st>>>(a);
    prof_after(st);
    return cudaGetLastError();
}

}  // namespace semicrf
