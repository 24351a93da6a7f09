// forward_backward.cu -- the recursions the forward / recompute / backward
// kernels implement, the gradient finalisation kernels and the dispatch between
// the two kernel families (fb_small.cu for C, K <= 32; fb_cluster.cu otherwise).
//
// Streaming Structured Inference with Flash-SemiCRF:
//   abstract             edge potentials evaluated on the fly from a prefix-sum
//                        array; streaming forward-backward with checkpoint-
//                        boundary normalisation; exact gradients
//   technical summary    2.A  segment content = S[s+d,c] - S[s,c]
//                        2.B  forward and backward messages in fixed O(K*C) rings
//                        2.C  checkpoints, local recompute of the forward
//                             messages per checkpoint segment, normalisation
//
// Recursions (log space; the kernels run them in scaled exp space):
//   at[0,c] = 0
//   al[t,c] = lse_d ( at[t-d,c] + S[t,c] - S[t-d,c] + D[d-1,c] ),   1 <= d <= min(K,t)
//   at[t,c] = lse_c' ( al[t,c'] + A[c',c] ),                         1 <= t < L
//   logZ    = lse_c al[L,c]
//   be[L,c] = 0
//   ga[s,c] = lse_d ( S[s+d,c] - S[s,c] + D[d-1,c] + be[s+d,c] ),    1 <= d <= min(K,L-s)
//   be[s,c']= lse_c ( A[c',c] + ga[s,c] ),                           1 <= s < L
// Marginals: Pseg(s,d,c) = exp(at[s,c] + S[s+d,c] - S[s,c] + D[d-1,c] + be[s+d,c] - logZ),
//            Ptr(s,c',c) = exp(al[s,c'] + A[c',c] + ga[s,c] - logZ).
// dD = sum Pseg, dA = sum Ptr, dX[u,c] = mu[u,c] - mean_u' mu[u',c] where the
// coverage mu[u,c] = sum_{s'>u} (end[s',c] - start[s',c]),
// end[t,c] = exp(al[t,c] + be[t,c] - logZ), start[s,c] = exp(at[s,c] + ga[s,c] - logZ).
//
// Scaled exp space (float64).  The forward ring holds, for each row s and label
// c, U[s,c] = exp(at[s,c] - S[s,c] - ln2 * r_c): a per-label power-of-two
// reference r_c absorbs the O(sqrt T) spread of S across labels, and is moved
// by an exact power-of-two rescale of the column whenever the weighted column
// sum p[c] = sum_d U[t-d,c] exp(D[d-1,c]) leaves [2^-256, 2^256].  Then
//   al[t,c]        = S[t,c] + ln2 r_c + log p[c]
//   a'[t,c]        = exp(al[t,c] - ln2 k_t) = p[c] * exp(S[t,c] + ln2 (r_c - k_t))
//   q[c]           = sum_c' a'[t,c'] exp(A[c',c])    (= exp(at[t,c] - ln2 k_t))
//   U[t,c]         = q[c] * exp(ln2 (k_t - r_c) - S[t,c])
//   k_{t+1}        = k_t + floor(log2 sum_c a'[t,c])  (the running normaliser;
//                    log Z = ln2 k_L + log sum_c a'[L,c])
// so the K*C duration sum and the C*C transition sum are plain FMAs; the only
// exponentials are two per label per step.  All exponents are integers, so
// every rescale is exact.
//
// Parallel layout: see fb_small.cu (one CTA per sequence, warp-specialised) and
// fb_cluster.cu (one thread-block cluster per sequence, labels split across its
// CTAs, a'[t,:] all-gathered through distributed shared memory every position).
#include <math.h>
#include <stdlib.h>
#include <string.h>

#include "device_util.cuh"
#include "semicrf_internal.h"

namespace semicrf {
namespace {

// dD = sum_b g_b exp(D) accD_b,  dA = sum_b g_b exp(A) accA_b  (sequence order)
__global__ void finalise_params(FbArgs a)
{
    const int nA = a.C * a.C, nD = a.K * a.C;
    for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < nA + nD; i += gridDim.x * blockDim.x) {
        double s = 0.0;
        if (i < nA) {
            for (int b = 0; b < a.B; ++b) {
                const double g = a.grad ? a.grad[b] : 1.0;
                s = fma(g, a.accA[(size_t)b * nA + i], s);
            }
            a.dA[i] = s * exp((double)a.A[i]);
        } else {
            const int k = i - nA;
            for (int b = 0; b < a.B; ++b) {
                const double g = a.grad ? a.grad[b] : 1.0;
                s = fma(g, a.accD[(size_t)b * nD + k], s);
            }
            a.dD[k] = s * exp((double)a.D[k]);
        }
    }
}

// dX[b,u,c] = g_b (mu[b,u,c] - musum[b,c] / L_b) for u < L_b, else 0 (in place)
__global__ void finalise_dx(FbArgs a)
{
    const size_t n = (size_t)a.B * a.T * a.C;
    for (size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += (size_t)gridDim.x * blockDim.x) {
        const int c = (int)(i % a.C);
        const size_t bt = i / a.C;
        const int u = (int)(bt % a.T);
        const int b = (int)(bt / a.T);
        const int L = a.lengths[b];
        float out = 0.0f;
        if (L >= 1 && L <= a.T && u < L) {
            const double g = a.grad ? a.grad[b] : 1.0;
            const double mean = a.musum[(size_t)b * a.C + c] / (double)L;
            out = (float)(g * ((double)a.dX[i] - mean));
        }
        a.dX[i] = out;
    }
}

// Posterior outputs: zero mu beyond L_b; pstart[b,t] = sum_c P(start at t, label c).
__global__ void posterior_finalise(FbArgs a, float *mu, float *pstart)
{
    const size_t nmu = mu ? (size_t)a.B * a.T * a.C : 0;
    const size_t nps = pstart ? (size_t)a.B * a.T : 0;
    for (size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x; i < nmu + nps;
         i += (size_t)gridDim.x * blockDim.x) {
        if (i < nmu) {
            const size_t bt = i / a.C;
            const int u = (int)(bt % a.T), b = (int)(bt / a.T);
            const int L = a.lengths[b];
            if (L < 1 || L > a.T || u >= L) mu[i] = 0.0f;
        } else {
            const size_t bt = i - nmu;
            const int t = (int)(bt % a.T), b = (int)(bt / a.T);
            const int L = a.lengths[b];
            double p = 0.0;
            if (L >= 1 && L <= a.T && t < L) {
                const double *row = a.stst + ((size_t)b * (a.T + 1) + t) * a.C;
                for (int c = 0; c < a.C; ++c) p += row[c];
            }
            pstart[bt] = (float)p;
        }
    }
}

}  // namespace

// Which kernel family runs: the warp-per-sequence kernels when the shape allows,
// else the cluster kernels.  SEMICRF_KERNEL_PATH=general forces the cluster
// kernels (used by the tests to keep both families under parity checks).
bool use_small(int K, int C)
{
    const char *env = getenv("SEMICRF_KERNEL_PATH");
    if (env && strcmp(env, "general") == 0) return false;
    return small_path_ok(K, C);
}

cudaError_t launch_forward(const Plan &p, const FbArgs &a, cudaStream_t st, int *launches)
{
    (void)p;
    cudaError_t e = launch_exp_tables(a, st);
    if (e != cudaSuccess) return e;
    *launches += 1;
    e = use_small(a.K, a.C) ? launch_small(a, st, 0) : launch_cl_forward(a, st, false);
    if (e == cudaSuccess) *launches += 1;
    return e;
}

cudaError_t launch_backward(const Plan &p, const FbArgs &a, cudaStream_t st, int *launches)
{
    (void)p;
    const bool small = use_small(a.K, a.C);
    // recompute every checkpoint segment, then the backward pass with marginals
    cudaError_t e = small ? launch_small(a, st, 1) : launch_cl_forward(a, st, true);
    if (e != cudaSuccess) return e;
    e = small ? launch_small(a, st, 2) : launch_cl_backward(a, st);
    if (e != cudaSuccess) return e;
    if (small) {
        // the warp-per-sequence backward accumulated dA, dD per sequence
        const int nparam = a.C * a.C + a.K * a.C;
        prof_before(st);
        finalise_params<<<(nparam + 255) / 256, 256, 0, st>>>(a);
        prof_after(st);
    } else {
        // the cluster backward stored its rows; dD and dA are contractions over them
        e = launch_cl_param_grads(a, st);
        if (e != cudaSuccess) return e;
    }
    const size_t n = (size_t)a.B * a.T * a.C;
    int blocks = (int)((n + 255) / 256);
    if (blocks > device_sm_count() * 16) blocks = device_sm_count() * 16;
    prof_before(st);
    finalise_dx<<<blocks, 256, 0, st>>>(a);
    prof_after(st);
    *launches += small ? 4 : 6;
    return cudaGetLastError();
}

cudaError_t launch_posteriors(const FbArgs &a0, float *mu, float *pstart, cudaStream_t st, int *launches)
{
    FbArgs a = a0;
    a.dX = mu;   // raw coverage; the parameter gradients are not formed
    const bool small = use_small(a.K, a.C);
    cudaError_t e = small ? launch_small(a, st, 1) : launch_cl_forward(a, st, true);
    if (e != cudaSuccess) return e;
    e = small ? launch_small(a, st, 2) : launch_cl_backward(a, st);
    if (e != cudaSuccess) return e;
    const size_t n = (mu ? (size_t)a.B * a.T * a.C : 0) + (pstart ? (size_t)a.B * a.T : 0);
    int blocks = (int)((n + 255) / 256);
    if (blocks > device_sm_count() * 16) blocks = device_sm_count() * 16;
    if (blocks < 1) blocks = 1;
    prof_before(st);
    posterior_finalise<<<blocks, 256, 0, st>>>(a, mu, pstart);
    prof_after(st);
    *launches += 3;
    return cudaGetLastError();
}

// Forward and backward at once: the forward chain (storing its rows unscaled, no
// checkpoints) and the beta chain run side by side in one launch -- the beta
// chain needs only S, A, D and the lengths -- then the marginals, coverage and
// parameter gradients are parallel passes over the stored rows: two launches
// for C, K <= 32 (4 in all), else the rows get the log Z scaling and nine
// launches follow (11 in all).
cudaError_t launch_forward_backward(const FbArgs &a, cudaStream_t st, int *launches)
{
    cudaError_t e = launch_exp_tables(a, st);
    if (e != cudaSuccess) return e;
    const bool small = use_small(a.K, a.C);
    e = small ? launch_small(a, st, 3) : launch_cl_fused(a, st);
    if (e != cudaSuccess) return e;
    if (small && a.npost > 0) {
        e = launch_team_post(a, st);
        if (e == cudaSuccess) *launches += 4;
        return e;
    }
    e = launch_rows_rescale(a, st);
    if (e != cudaSuccess) return e;
    e = launch_coverage(a, st);
    if (e != cudaSuccess) return e;
    e = launch_cl_param_grads(a, st);
    if (e != cudaSuccess) return e;
    const size_t n = (size_t)a.B * a.T * a.C;
    int blocks = (int)((n + 255) / 256);
    if (blocks > device_sm_count() * 16) blocks = device_sm_count() * 16;
    prof_before(st);
    finalise_dx<<<blocks, 256, 0, st>>>(a);
    prof_after(st);
    *launches += 11;
    return cudaGetLastError();
}

}  // namespace semicrf
