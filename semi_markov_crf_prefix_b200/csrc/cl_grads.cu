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
// unless the label's column was rebased between s+1 and s+d; a chunk stages both
// factors at one base reference per label (exact powers of two) so that every
// term is one FMA, and falls back to exact per-term scaling for the whole CTA
// only when a pre-scaled row would leave the safe range.
//
// Layout: each CTA owns a tile of outputs (128 or 32 durations x 32 labels for dD,
// 32 x 32 (c, c2) for dA) and a
// split z of the (sequence, 32-position chunk) list, which it walks chunk by
// chunk, staging the chunk's rows in shared memory; it writes its tile of
// partial sums to part*[z].  A last kernel adds the splits in order (the
// result does not depend on scheduling) and applies exp(D), exp(A).
#include <limits.h>
#include <math.h>

#include "device_util.cuh"
#include "semicrf_internal.h"

namespace semicrf {
namespace {

constexpr int kCh = 32;    // start positions per chunk
constexpr int kTile = 32;  // output tile edge

// Rows pre-scaled to a chunk's base reference are usable when none exceeds
// 2^900: a product of two normal doubles is then exact to rounding, and where one
// factor underflowed the product is below 2^-122 (negligible).
__device__ __forceinline__ bool too_large(double v) { return !(fabs(v) <= 0x1p900); }

// Shared memory of dur_grad_kernel<TD>: X [kCh][kTile] f64 and its references
// (int), Y [kCh + TD][kTile] f64 and its references.
template <int TD>
constexpr size_t dur_smem_bytes()
{
    return (size_t)kCh * kTile * 12 + (size_t)(kCh + TD) * kTile * 12;
}

// TD durations per CTA tile (32 or 128): every staged chunk of rows serves TD
// durations, so the wider tile stages a quarter as many rows per product.  Warp
// dq owns the NA = TD/8 consecutive durations d0 + dq NA + k; for start s its
// lanes need the end rows s + d0 + dq NA + k, a window that slides by one row
// per start, so each start costs two shared loads (X and the window's new row)
// for NA FMAs.
template <int TD>
__global__ void __launch_bounds__(256) dur_grad_kernel(FbArgs a)
{
    constexpr int NA = TD / 8;   // durations per thread
    extern __shared__ __align__(16) unsigned char dsm[];
    double(*xs)[kTile] = reinterpret_cast<double(*)[kTile]>(dsm);
    double(*ys)[kTile] = reinterpret_cast<double(*)[kTile]>(dsm + (size_t)kCh * kTile * 8);
    int(*rs)[kTile] = reinterpret_cast<int(*)[kTile]>(dsm + (size_t)(2 * kCh + TD) * kTile * 8);
    int(*ry)[kTile] = reinterpret_cast<int(*)[kTile]>(dsm + (size_t)(2 * kCh + TD) * kTile * 8 + (size_t)kCh * kTile * 4);
    const int K = a.K, C = a.C, T = a.T;
    const int z = blockIdx.x, c0 = blockIdx.y * kTile, d0 = 1 + blockIdx.z * TD;   // d is 1-based
    const int tid = threadIdx.x, lc = tid & 31, dq = tid >> 5;
    const int c = c0 + lc;
    const bool c_ok = c < C;
    const int nch = (T + kCh - 1) / kCh;
    const long long Q = (long long)a.B * nch;
    double acc[NA];
#pragma unroll
    for (int k = 0; k < NA; ++k) acc[k] = 0.0;
    for (long long q = z; q < Q; q += a.nsD) {
        const int b = (int)(q / nch), s0 = (int)(q % nch) * kCh;
        const int L = a.lengths[b];
        if (L < 1 || L > T || s0 >= L) continue;   // uniform over the CTA
        const size_t rowbase = (size_t)b * (T + 1);
        const double g = a.grad ? a.grad[b] : 1.0;
        const int kZ = a.lz[b].k;
        const double cz = exp(-a.lz[b].logn);
        const int tb = min(max(s0 + d0, 1), L);   // the chunk's base reference: rb at row tb
        // Stage the chunk's start factors X (s in [s0, s0 + kCh), zero beyond L - 1)
        // and end rows Y (t in [s0 + d0, s0 + d0 + kCh + kTile), zero beyond L).
        // scaled: both at the label's base reference R0 (X 2^(R0 - rX), Y 2^(rY - R0)),
        // so a segment marginal is one product; else at their own references.
        auto stage = [&](bool scaled) {
            bool bad = false;
            for (int i = tid; i < kCh * kTile; i += 256) {
                const int si = i / kTile, l2 = i % kTile, s = s0 + si, cc = c0 + l2;
                double x = 0.0;
                int r = INT_MIN;
                if (s <= L - 1 && cc < C) {
                    r = a.rbst[(rowbase + s + 1) * C + cc];
                    x = (s == 0) ? scale2c(cz, r - kZ)
                                 : scale2c(a.cU[(rowbase + s) * C + cc], a.eU[(rowbase + s) * C + cc] + r);
                    x *= g;
                    if (scaled) {
                        x = scale2c(x, a.rbst[(rowbase + tb) * C + cc] - r);
                        bad |= too_large(x);
                    }
                }
                xs[si][l2] = x;
                rs[si][l2] = r;
            }
            for (int i = tid; i < (kCh + TD) * kTile; i += 256) {
                const int ti = i / kTile, l2 = i % kTile, t = s0 + d0 + ti, cc = c0 + l2;
                double y = 0.0;
                int r = INT_MIN;
                if (t <= L && cc < C) {
                    y = a.Vst[(rowbase + t) * C + cc];
                    r = a.rbst[(rowbase + t) * C + cc];
                    if (scaled) {
                        y = scale2c(y, r - a.rbst[(rowbase + tb) * C + cc]);
                        bad |= too_large(y);
                    }
                }
                ys[ti][l2] = y;
                ry[ti][l2] = r;
            }
            return bad;
        };
        __syncthreads();   // previous chunk's reads are done
        // Extreme growth (a label's references over ~900 bits apart inside the
        // chunk): the whole CTA restages at the own references and scales every term.
        const bool exact = __syncthreads_or(stage(true));
        if (exact) {
            stage(false);
            __syncthreads();
        }
        if (!exact) {
            // w[(si + k) % NA] holds end row si + dq NA + k (relative to s0 + d0)
            double w[NA];
#pragma unroll
            for (int k = 0; k < NA; ++k) w[k] = ys[dq * NA + k][lc];
#pragma unroll
            for (int si = 0; si < kCh; ++si) {
                const double x = xs[si][lc];
                const double nxt = ys[si + dq * NA + NA][lc];   // row <= kCh - 1 + TD: staged
#pragma unroll
                for (int k = 0; k < NA; ++k) acc[k] = fma(x, w[(si + k) % NA], acc[k]);
                w[si % NA] = nxt;
            }
        } else {
            for (int si = 0; si < kCh; ++si) {
                const double x = xs[si][lc];
                const int r = rs[si][lc];
                if (r == INT_MIN) continue;
#pragma unroll
                for (int k = 0; k < NA; ++k) {
                    const int ti = si + dq * NA + k;
                    const double y = ys[ti][lc];
                    if (y != 0.0) acc[k] += scale2c(x * y, ry[ti][lc] - r);
                }
            }
        }
    }
#pragma unroll
    for (int k = 0; k < NA; ++k) {
        const int d = d0 + dq * NA + k;
        if (d <= K && c_ok) a.partD[((size_t)z * K + (d - 1)) * C + c] = acc[k];
    }
}

// TA x TA outputs (c, c2) per CTA (32 or 64): thread (ti, tj) = (tid / 16,
// tid % 16) owns the RA x RA outputs c = c0 + RA ti + r, c2 = e0 + tj + 16 k,
// so a start row costs 2 RA shared loads (the c values as one or two 16-byte
// loads, the c2 values conflict-free) for RA^2 FMAs.
template <int TA>
__global__ void __launch_bounds__(256) trans_grad_kernel(FbArgs a)
{
    constexpr int RA = TA / 16;
    __shared__ __align__(16) double as[kCh][TA];
    __shared__ double bs[kCh][TA];
    const int C = a.C, T = a.T;
    const int z = blockIdx.x, c0 = blockIdx.y * TA, e0 = blockIdx.z * TA;
    const int tid = threadIdx.x, ti = tid >> 4, tj = tid & 15;
    const int nch = (T + kCh - 1) / kCh;
    const long long Q = (long long)a.B * nch;
    double acc[RA][RA];
#pragma unroll
    for (int r = 0; r < RA; ++r)
#pragma unroll
        for (int k = 0; k < RA; ++k) acc[r][k] = 0.0;
    for (long long q = z; q < Q; q += a.nsA) {
        const int b = (int)(q / nch), s0 = (int)(q % nch) * kCh;
        const int L = a.lengths[b];
        if (L < 2 || L > T || s0 >= L - 1 + 1) continue;   // transitions at s in [1, L-1]
        const size_t rowbase = (size_t)b * (T + 1);
        const double g = a.grad ? a.grad[b] : 1.0;
        __syncthreads();
        for (int i = tid; i < kCh * TA; i += 256) {
            const int si = i / TA, l2 = i % TA, s = s0 + si;
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
            double x[RA], y[RA];
#pragma unroll
            for (int r = 0; r < RA; r += 2) {
                const double2 v = *reinterpret_cast<const double2 *>(&as[si][RA * ti + r]);
                x[r] = v.x;
                x[r + 1] = v.y;
            }
#pragma unroll
            for (int k = 0; k < RA; ++k) y[k] = bs[si][tj + 16 * k];
#pragma unroll
            for (int r = 0; r < RA; ++r)
#pragma unroll
                for (int k = 0; k < RA; ++k) acc[r][k] = fma(x[r], y[k], acc[r][k]);
        }
    }
#pragma unroll
    for (int r = 0; r < RA; ++r) {
        const int c = c0 + RA * ti + r;
#pragma unroll
        for (int k = 0; k < RA; ++k) {
            const int e = e0 + tj + 16 * k;
            if (c < C && e < C) a.partA[((size_t)z * C + c) * C + e] = acc[r][k];
        }
    }
}

// dD = exp(D) * sum_z partD[z],  dA = exp(A) * sum_z partA[z]: one warp per
// output, lane l adds the splits z = l, l+32, ... in order, then a fixed xor tree
// (the result does not depend on scheduling).
__global__ void cl_finalise_params(FbArgs a)
{
    const int nA = a.C * a.C, nD = a.K * a.C;
    const int lane = threadIdx.x & 31;
    const int w0 = (blockIdx.x * blockDim.x + threadIdx.x) >> 5, nw = (gridDim.x * blockDim.x) >> 5;
    for (int i = w0; i < nA + nD; i += nw) {
        double s = 0.0;
        if (i < nA) {
            for (int z = lane; z < a.nsA; z += 32) s += a.partA[(size_t)z * nA + i];
        } else {
            for (int z = lane; z < a.nsD; z += 32) s += a.partD[(size_t)z * nD + (i - nA)];
        }
        for (int off = 16; off > 0; off >>= 1) s += __shfl_xor_sync(0xffffffffu, s, off);
        if (lane == 0) {
            if (i < nA) a.dA[i] = exp((double)a.A[i]) * s;
            else a.dD[i - nA] = exp((double)a.D[i - nA]) * s;
        }
    }
}

int ceil_div(long long a, long long b) { return (int)((a + b - 1) / b); }

// Rows the forward stored unscaled (cU = U, eU = r, cA = a', eA = k) become the
// recompute's convention once log Z = ln2 kZ + logn is known:
//   cU *= exp(-logn), eU -= kZ, cA *= exp(-logn), eA -= kZ     (t in [1, L])
__global__ void rows_rescale(FbArgs a)
{
    const size_t n = (size_t)a.B * (a.T + 1) * a.C;
    for (size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += (size_t)gridDim.x * blockDim.x) {
        const size_t bt = i / a.C;
        const int t = (int)(bt % (a.T + 1)), b = (int)(bt / (a.T + 1));
        const int L = a.lengths[b];
        if (L < 1 || L > a.T || t < 1 || t > L) continue;
        const int kZ = a.lz[b].k;
        const double cz = exp(-a.lz[b].logn);
        if (t < L) {
            a.cU[i] *= cz;
            a.eU[i] -= kZ;
        }
        a.cA[i] *= cz;
        if ((int)(i % a.C) == 0) a.eA[bt] -= kZ;
    }
}

// Segment start and end marginals of label c at position u from the stored rows:
//   start(u) = exp(at[u] - S[u] - log Z) exp(be[u]) exp(S[u])   (a segment begins at u)
//   end(u)   = exp(al[u] - log Z) exp(ga[u])                     (a segment ends at u, u >= 1)
// with every factor a mantissa and a power of two, so the product is exact up to
// rounding whatever the references.
__device__ __forceinline__ double seg_start_marg(const FbArgs &a, size_t rowbase, int b, int u, int c)
{
    const size_t ix = (rowbase + u) * a.C + c;
    const double bp = a.bpst[ix], es = a.tES[ix];
    const int kb = a.kbst[rowbase + u], m = a.tM[ix];
    if (u == 0) return scale2c(exp(-a.lz[b].logn) * bp * es, kb + m - a.lz[b].k);
    return scale2c(a.cU[ix] * bp * es, a.eU[ix] + kb + m);
}

__device__ __forceinline__ double seg_end_marg(const FbArgs &a, size_t rowbase, int u, int c)
{
    const size_t ix = (rowbase + u) * a.C + c;
    return scale2c(a.cA[ix] * a.Vst[ix] * a.tIES[ix], a.eA[rowbase + u] + a.rbst[ix] - a.tM[ix]);
}

// Coverage mu[u,c] = sum_{s<=u} start(s,c) - sum_{1<=t<=u} end(t,c), a prefix scan
// per (sequence, label) in chunks of covch positions (cov_chunk: about T/1024,
// at least 32): chunk totals; their
// exclusive prefix per (sequence, label), in order; the scan within each chunk
// from that offset (writing raw mu into dX and the chunk's sum of mu); the
// per-label sum over positions for the path through nu.
__device__ __forceinline__ int cov_end(const FbArgs &a, int b, int u0)
{
    const int L = a.lengths[b];
    return min(u0 + a.covch, (L >= 1 && L <= a.T) ? L : 0);
}

__global__ void cov_delta_kernel(FbArgs a)
{
    const int b = blockIdx.y, ch = blockIdx.x, c = threadIdx.x;
    if (c >= a.C) return;
    const int nch = (a.T + a.covch - 1) / a.covch;
    const int u0 = ch * a.covch, u1 = cov_end(a, b, u0);
    const size_t rowbase = (size_t)b * (a.T + 1);
    double d0 = 0.0, d1 = 0.0;
    int u = u0;
    for (; u + 1 < u1; u += 2) {   // two independent positions per round
        d0 += seg_start_marg(a, rowbase, b, u, c) - (u >= 1 ? seg_end_marg(a, rowbase, u, c) : 0.0);
        d1 += seg_start_marg(a, rowbase, b, u + 1, c) - seg_end_marg(a, rowbase, u + 1, c);
    }
    if (u < u1) d0 += seg_start_marg(a, rowbase, b, u, c) - (u >= 1 ? seg_end_marg(a, rowbase, u, c) : 0.0);
    a.covd[((size_t)b * nch + ch) * a.C + c] = d0 + d1;
}

// exclusive prefix of the chunk totals, in place, one thread per (sequence, label)
__global__ void cov_offsets_kernel(FbArgs a)
{
    const int i = blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= a.B * a.C) return;
    const int b = i / a.C, c = i % a.C;
    const int nch = (a.T + a.covch - 1) / a.covch;
    double run = 0.0;
    for (int k = 0; k < nch; ++k) {
        double *p = &a.covd[((size_t)b * nch + k) * a.C + c];
        const double d = *p;
        *p = run;
        run += d;
    }
}

__global__ void cov_scan_kernel(FbArgs a)
{
    const int b = blockIdx.y, ch = blockIdx.x, c = threadIdx.x;
    if (c >= a.C) return;
    const int nch = (a.T + a.covch - 1) / a.covch;
    const int u0 = ch * a.covch, u1 = cov_end(a, b, u0);
    const size_t rowbase = (size_t)b * (a.T + 1);
    double mu = a.covd[((size_t)b * nch + ch) * a.C + c];
    double msum = 0.0;
    for (int u = u0; u < u1; ++u) {
        mu += seg_start_marg(a, rowbase, b, u, c) - (u >= 1 ? seg_end_marg(a, rowbase, u, c) : 0.0);
        a.dX[((size_t)b * a.T + u) * a.C + c] = (float)mu;
        msum += mu;
    }
    a.covm[((size_t)b * nch + ch) * a.C + c] = msum;
}

__global__ void cov_musum_kernel(FbArgs a)
{
    const int i = blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= a.B * a.C) return;
    const int b = i / a.C, c = i % a.C;
    const int nch = (a.T + a.covch - 1) / a.covch;
    double s = 0.0;
    for (int k = 0; k < nch; ++k) s += a.covm[((size_t)b * nch + k) * a.C + c];
    a.musum[(size_t)b * a.C + c] = s;
}

}  // namespace

// Duration tile of the dD contraction: 128 durations per CTA when K reaches it.
inline int dur_tile(int K) { return K >= 128 ? 128 : kTile; }

// Resident CTAs per SM of the dD contraction (the runtime's figure; without a
// device, the one its register and shared-memory use gives on sm_100a).
int dur_grad_occupancy(int TD)
{
    int n = 0;
    cudaError_t e;
    if (TD == 128) {
        e = cudaFuncSetAttribute(dur_grad_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 (int)dur_smem_bytes<128>());
        if (e == cudaSuccess)
            e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, dur_grad_kernel<128>, 256, dur_smem_bytes<128>());
    } else {
        e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, dur_grad_kernel<kTile>, 256, dur_smem_bytes<kTile>());
    }
    if (e != cudaSuccess || n < 1) {
        cudaGetLastError();
        n = TD == 128 ? 3 : 5;
    }
    return n;
}

// Output tile of the dA contraction: 64 x 64 when C exceeds 32.
inline int trans_tile(int C) { return C > kTile ? 64 : kTile; }

int trans_grad_occupancy(int TA)
{
    int n = 0;
    const cudaError_t e = TA == 64 ? cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, trans_grad_kernel<64>, 256, 0)
                                   : cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, trans_grad_kernel<kTile>, 256, 0);
    if (e != cudaSuccess || n < 1) {
        cudaGetLastError();
        n = TA == 64 ? 3 : 4;
    }
    return n;
}

// Splits: each contraction fills two waves of resident CTAs (every CTA walks the
// same number of chunks, so a partial last wave would idle the rest).
void cl_grad_splits(int B, int T, int K, int C, int *nsD, int *nsA)
{
    const long long Q = (long long)B * ceil_div(T, kCh);
    const int tilesD = ceil_div(K, dur_tile(K)) * ceil_div(C, kTile);
    const int tilesA = ceil_div(C, trans_tile(C)) * ceil_div(C, trans_tile(C));
    const int nsm = device_sm_count();
    const long long slotsD = 2LL * nsm * dur_grad_occupancy(dur_tile(K));
    const long long slotsA = 2LL * nsm * trans_grad_occupancy(trans_tile(C));
    long long d = slotsD / tilesD, e = slotsA / tilesA;
    if (d < 1) d = 1;
    if (e < 1) e = 1;
    if (d > 1024) d = 1024;
    if (e > 1024) e = 1024;
    *nsD = (int)(d < Q ? d : Q);
    *nsA = (int)(e < Q ? e : Q);
    if (*nsD < 1) *nsD = 1;
    if (*nsA < 1) *nsA = 1;
}

cudaError_t launch_rows_rescale(const FbArgs &a, cudaStream_t st)
{
    const size_t n = (size_t)a.B * (a.T + 1) * a.C;
    int blocks = (int)((n + 255) / 256);
    if (blocks > device_sm_count() * 16) blocks = device_sm_count() * 16;
    prof_before(st);
    rows_rescale<<<blocks, 256, 0, st>>>(a);
    prof_after(st);
    return cudaGetLastError();
}

cudaError_t launch_coverage(const FbArgs &a, cudaStream_t st)
{
    const int nch = ceil_div(a.T, a.covch);
    const int threads = ceil_div(a.C, 32) * 32;
    const int nbc = ceil_div((long long)a.B * a.C, 128);
    prof_before(st);
    cov_delta_kernel<<<dim3(nch, a.B), threads, 0, st>>>(a);
    prof_after(st);
    prof_before(st);
    cov_offsets_kernel<<<nbc, 128, 0, st>>>(a);
    prof_after(st);
    prof_before(st);
    cov_scan_kernel<<<dim3(nch, a.B), threads, 0, st>>>(a);
    prof_after(st);
    prof_before(st);
    cov_musum_kernel<<<nbc, 128, 0, st>>>(a);
    prof_after(st);
    return cudaGetLastError();
}

cudaError_t launch_cl_param_grads(const FbArgs &a, cudaStream_t st)
{
    if (dur_tile(a.K) == 128) {
        const size_t smem = dur_smem_bytes<128>();
        cudaError_t e = cudaFuncSetAttribute(dur_grad_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             (int)smem);
        if (e != cudaSuccess) return e;
        prof_before(st);
        dur_grad_kernel<128><<<dim3(a.nsD, ceil_div(a.C, kTile), ceil_div(a.K, 128)), 256, smem, st>>>(a);
        prof_after(st);
    } else {
        prof_before(st);
        dur_grad_kernel<kTile><<<dim3(a.nsD, ceil_div(a.C, kTile), ceil_div(a.K, kTile)), 256, dur_smem_bytes<kTile>(),
                                 st>>>(a);
        prof_after(st);
    }
    prof_before(st);
    const int TA = trans_tile(a.C);
    if (TA == 64)
        trans_grad_kernel<64><<<dim3(a.nsA, ceil_div(a.C, 64), ceil_div(a.C, 64)), 256, 0, st>>>(a);
    else
        trans_grad_kernel<kTile><<<dim3(a.nsA, ceil_div(a.C, kTile), ceil_div(a.C, kTile)), 256, 0, st>>>(a);
    prof_after(st);
    const int n = a.C * a.C + a.K * a.C;   // one warp per output
    int blocks = ceil_div((long long)n * 32, 256);
    if (blocks > device_sm_count() * 16) blocks = device_sm_count() * 16;
    prof_before(st);
    cl_finalise_params<<<blocks, 256, 0, st>>>(a);
    prof_after(st);
    return cudaGetLastError();
}

}  // namespace semicrf
