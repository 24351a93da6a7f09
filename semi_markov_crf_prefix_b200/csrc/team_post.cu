// team_post.cu -- the passes after the two chains of semicrf_forward_backward
// for the shapes the warp-per-sequence kernels take (C <= 32, K <= 32): two
// launches over the stored rows, where the general shapes take nine.
//
// Streaming Structured Inference with Flash-SemiCRF, abstract (exact gradients
// of log Z) and technical summary 2.C (marginals from the forward and backward
// scores).  The forward chain stored its rows unscaled (U with exponent eU, a'
// with exponent eA), the beta chain V at its reference rb, the normalised beta
// bp and its exponent kb.  With log Z = ln2 kZ + logn:
//   X[s,c]  = exp(at[s,c] - S[s,c] - log Z + ln2 rb[s+1,c])     0 <= s <= L-1
//   Y[t,c]  = V[t,c] = exp(be[t,c] + S[t,c] - ln2 rb[t,c])       1 <= t <= L
//   Pseg(s,d,c) = X[s,c] exp(D[d-1,c]) Y[s+d,c] 2^(rb[s+d,c] - rb[s+1,c])
//   a2[s,c] = exp(al[s,c] - log Z + ln2 kb[s]),   Ptr(s,c,e) = a2[s,c] exp(A[c,e]) bp[s,e]
//
// Pass 1 (team_post_kernel), one item per (sequence, 32 start positions):
//   * partial sums of dD (without exp D) and dA (without exp A) over the item;
//   * the coverage mu[u,c] (the probability that a segment of label c covers u)
//     at the item's first position u0 as a window sum -- the segments covering
//     u0 start at most K-1 positions earlier -- and then
//     mu[u] = mu[u-1] + start(u) - end(u), start and end the sums of Pseg over the
//     segments that start / end at u; raw mu goes into dX, its sum over the
//     item's positions into covm.  No item waits for another.
// Pass 2 (team_finalise_kernel): dX = g (mu - mean_u mu), zero past L; dD and dA
// as the pass-1 partials added in a fixed order, times exp(D), exp(A).  The
// results do not depend on scheduling.
#include <limits.h>
#include <math.h>

#include "device_util.cuh"
#include "semicrf_internal.h"

namespace semicrf {
namespace {

constexpr int kPC = 32;             // start positions per item
constexpr int kPT = 256;            // threads per CTA: 32 label lanes x 8 groups
constexpr int kRows = kPC + 32;     // staged X and Y rows (K <= 32)
constexpr int kDxPer = 1024;        // dX elements per finalise CTA, at least

struct PostSmem {
    double X[kRows][32];     // row i: s = u0 - (K-1) + i
    double Y[kRows][32];     // row i: t = u0 + i
    double w[32][32];        // exp(D[d-1,c])
    double a2[kPC][32];      // row i: s = u0 + i
    double bp[kPC][32];
    double delta[kPC][32];   // start(u) - end(u), row u - u0
    double win[8][32];       // window partial sums
    double red[8][4][32];    // dD partial sums of the row parts, at the end
    int rX[kRows][32];       // rb[s+1,c]
    int rY[kRows][32];       // rb[t,c]
};

// x * w * y at references rx (of x) and ry (of y): exact scaling, zero terms skipped
__device__ __forceinline__ double scaled_term(double x, double wy, int rx, int ry)
{
    return (x != 0.0 && wy != 0.0) ? scale2c(x * wy, ry - rx) : 0.0;
}

// Pre-scaled rows are usable when none exceeds 2^900: a product X^ w Y^ of two
// normal doubles is then exact to rounding, and where one factor underflowed the
// product is below 2^-122 (negligible).
__device__ __forceinline__ bool too_large(double v) { return !(fabs(v) <= 0x1p900); }

__global__ void __launch_bounds__(kPT, 2) team_post_kernel(FbArgs a)
{
    extern __shared__ __align__(16) unsigned char post_raw[];
    PostSmem &sm = *reinterpret_cast<PostSmem *>(post_raw);
    const int K = a.K, C = a.C, T = a.T;
    const int tid = threadIdx.x, lane = tid & 31, grp = tid >> 5;
    const int nch = (T + kPC - 1) / kPC;
    const long long Q = (long long)a.B * nch;
    const long long q0 = Q * blockIdx.x / gridDim.x, q1 = Q * (blockIdx.x + 1) / gridDim.x;
    for (int i = tid; i < 32 * 32; i += kPT) {
        const int d = i >> 5, c = i & 31;
        sm.w[d][c] = (d < K && c < C) ? exp((double)a.D[d * C + c]) : 0.0;
    }
    // dD: durations in blocks of four, d0 = 1 + 4 db; nDB blocks (a power of two),
    // the 8 / nDB groups of one block split the item's start positions
    const int nDB = K <= 4 ? 1 : K <= 8 ? 2 : K <= 16 ? 4 : 8;
    const int db = grp & (nDB - 1), dpart = grp / nDB, nparts = 8 / nDB;
    const int d0 = 1 + 4 * db;
    const int si0 = dpart * (kPC / nparts), si1 = si0 + kPC / nparts;
    // start / end: rows j0 .. j0+3 of the item; dA: rows 2 ci2 .. +1, columns 2 cj2 .. +1
    const int j0 = 4 * grp;
    const int ci2 = tid >> 4, cj2 = tid & 15;
    double accD[4] = {0.0, 0.0, 0.0, 0.0}, accA[4] = {0.0, 0.0, 0.0, 0.0};
    const int c = lane;
    for (long long q = q0; q < q1; ++q) {
        const int b = (int)(q / nch), ch = (int)(q % nch), u0 = ch * kPC;
        // the item's scalars in one round trip
        const int L = a.lengths[b];
        const double g = a.grad ? a.grad[b] : 1.0;
        const LogZState lzb = a.lz[b];
        if (L < 1 || L > T || u0 >= L) continue;   // uniform over the CTA
        const size_t rb0 = (size_t)b * (T + 1);
        const int kZ = lzb.k;
        const double cz = exp(-lzb.logn);
        __syncthreads();   // the previous item's reads are done
        // Stage the item's rows (up to 8 X rows, 8 Y rows, 4 transition rows of
        // column `lane`).  Every load goes out first, from an index clamped into
        // the written rows so that no load waits on a branch; the out-of-range
        // entries are zeroed afterwards.
        const int lc = min(lane, C - 1);
        const bool cok = lane < C;
        const int R0 = a.rbst[(rb0 + min(max(u0, 1), L)) * C + lc];   // the label's base reference
        double xu[8], yv[8], ca[4], bv[4];
        int xr[8], xeu[8], ye[8], ea[4], kb[4];
#pragma unroll
        for (int it = 0; it < 8; ++it) {
            const int r = grp + 8 * it;
            const int sc = min(max(u0 - (K - 1) + r, 0), L - 1);
            const size_t ix = (rb0 + sc) * C + lc;
            xr[it] = a.rbst[ix + C];   // rb[s+1]
            xu[it] = a.cU[ix];
            xeu[it] = a.eU[ix];
            const int tc = min(max(u0 + r, 1), L);
            const size_t iy = (rb0 + tc) * C + lc;
            yv[it] = a.Vst[iy];
            ye[it] = a.rbst[iy];
        }
#pragma unroll
        for (int it = 0; it < 4; ++it) {
            const int sc = min(max(u0 + grp + 8 * it, 1), max(L - 1, 1));
            const size_t ix = (rb0 + sc) * C + lc;
            ca[it] = a.cA[ix];
            ea[it] = a.eA[rb0 + sc];
            kb[it] = a.kbst[rb0 + sc];
            bv[it] = a.bpst[ix];
        }
        // X^ = X 2^(R0 - rX), Y^ = Y 2^(rY - R0): both at the base reference, so a
        // segment marginal is X^ w Y^ with no per-term scaling
        double xv[8];
        int xe[8];
        bool bad = false;
#pragma unroll
        for (int it = 0; it < 8; ++it) {
            const int r = grp + 8 * it;
            const int s = u0 - (K - 1) + r;
            const bool okx = cok && r < kPC + K - 1 && s >= 0 && s <= L - 1;
            xv[it] = !okx ? 0.0 : (s == 0) ? scale2c(cz, xr[it] - kZ) : scale2c(xu[it] * cz, xeu[it] - kZ + xr[it]);
            xe[it] = okx ? xr[it] : INT_MIN;
            const int t = u0 + r;
            const bool oky = cok && r < kPC + K && t >= 1 && t <= L;
            yv[it] = oky ? yv[it] : 0.0;
            ye[it] = oky ? ye[it] : INT_MIN;
            const double xs = okx ? scale2c(xv[it], okx ? R0 - xe[it] : 0) : 0.0;
            const double ys = oky ? scale2c(yv[it], oky ? ye[it] - R0 : 0) : 0.0;
            bad |= too_large(xs) || too_large(ys);
            if (r < kPC + K - 1) {
                sm.X[r][lane] = xs;
                sm.rX[r][lane] = xe[it];
            }
            if (r < kPC + K) {
                sm.Y[r][lane] = ys;
                sm.rY[r][lane] = ye[it];
            }
        }
#pragma unroll
        for (int it = 0; it < 4; ++it) {
            const int s = u0 + grp + 8 * it;
            const bool ok = cok && s >= 1 && s <= L - 1;
            sm.a2[grp + 8 * it][lane] = ok ? scale2c(ca[it] * cz, ea[it] - kZ + kb[it]) : 0.0;
            sm.bp[grp + 8 * it][lane] = ok ? bv[it] : 0.0;
        }
        // Extreme growth (a label's references more than ~900 bits apart inside the
        // item): the unscaled rows and exact scaling of every term instead.
        const bool exact = __syncthreads_or(bad);
        if (exact) {
#pragma unroll
            for (int it = 0; it < 8; ++it) {
                const int r = grp + 8 * it;
                if (r < kPC + K - 1) sm.X[r][lane] = xv[it];
                if (r < kPC + K) sm.Y[r][lane] = yv[it];
            }
            __syncthreads();
        }
        // ---- dD over the item's start positions [si0, si1), durations d0 .. d0+3
        {
            double acc[4] = {0.0, 0.0, 0.0, 0.0};
            if (!exact) {
                double y0 = sm.Y[si0 + d0][c], y1 = sm.Y[si0 + d0 + 1][c], y2 = sm.Y[si0 + d0 + 2][c];
                for (int si = si0; si < si1; ++si) {
                    const double x = sm.X[si + K - 1][c];
                    const double y3 = sm.Y[si + d0 + 3][c];
                    acc[0] = fma(x, y0, acc[0]);
                    acc[1] = fma(x, y1, acc[1]);
                    acc[2] = fma(x, y2, acc[2]);
                    acc[3] = fma(x, y3, acc[3]);
                    y0 = y1;
                    y1 = y2;
                    y2 = y3;
                }
            } else {
                for (int si = si0; si < si1; ++si)
#pragma unroll
                    for (int k = 0; k < 4; ++k)
                        if (d0 + k <= K)
                            acc[k] += scaled_term(sm.X[si + K - 1][c], sm.Y[si + d0 + k][c], sm.rX[si + K - 1][c],
                                                  sm.rY[si + d0 + k][c]);
            }
#pragma unroll
            for (int k = 0; k < 4; ++k) accD[k] = fma(g, acc[k], accD[k]);
        }
        // ---- start(u) - end(u), u = u0 + j for j = j0 .. j0+3:
        //   start = X^[u] sum_d w[d] Y^[u+d],   end = Y^[u] sum_d w[d] X^[u-d]
        {
            double st[4] = {0.0, 0.0, 0.0, 0.0}, en[4] = {0.0, 0.0, 0.0, 0.0};
            const int rx = j0 + K - 1;   // X row of s = u0 + j0
            if (!exact) {
                double y0 = sm.Y[j0 + 1][c], y1 = sm.Y[j0 + 2][c], y2 = sm.Y[j0 + 3][c];
                double x1 = sm.X[rx][c], x2 = sm.X[rx + 1][c], x3 = sm.X[rx + 2][c];   // X rows rx+m-d at d = 1
                for (int d = 1; d <= K; ++d) {
                    const double wd = sm.w[d - 1][c];
                    const double y3 = sm.Y[j0 + d + 3][c];
                    const double x0 = sm.X[max(rx - d, 0)][c];   // row -1 only feeds j = 0, unused
                    st[0] = fma(wd, y0, st[0]);
                    st[1] = fma(wd, y1, st[1]);
                    st[2] = fma(wd, y2, st[2]);
                    st[3] = fma(wd, y3, st[3]);
                    en[0] = fma(wd, x0, en[0]);
                    en[1] = fma(wd, x1, en[1]);
                    en[2] = fma(wd, x2, en[2]);
                    en[3] = fma(wd, x3, en[3]);
                    y0 = y1;
                    y1 = y2;
                    y2 = y3;
                    x3 = x2;
                    x2 = x1;
                    x1 = x0;
                }
#pragma unroll
                for (int m = 0; m < 4; ++m) sm.delta[j0 + m][c] = sm.X[rx + m][c] * st[m] - sm.Y[j0 + m][c] * en[m];
            } else {
#pragma unroll
                for (int m = 0; m < 4; ++m) {
                    const int j = j0 + m, rxs = rx + m;
                    if (j == 0) continue;
                    const double xs = sm.X[rxs][c], yu = sm.Y[j][c];
                    const int rxu = sm.rX[rxs][c], ryu = sm.rY[j][c];
                    for (int d = 1; d <= K; ++d) {
                        const double wd = sm.w[d - 1][c];
                        st[m] += scaled_term(xs, wd * sm.Y[j + d][c], rxu, sm.rY[j + d][c]);
                        en[m] += scaled_term(sm.X[rxs - d][c], wd * yu, sm.rX[rxs - d][c], ryu);
                    }
                    sm.delta[j][c] = st[m] - en[m];
                }
            }
            if (j0 == 0) sm.delta[0][c] = 0.0;   // mu[u0] comes from the window sum
        }
        // ---- window: segments starting at s = u0 - jj (jj < K) with d > jj cover u0
        {
            double part = 0.0;
#pragma unroll
            for (int m = 0; m < 4; ++m) {
                const int jj = grp + 8 * m;
                if (jj >= K) break;
                const int rxw = K - 1 - jj;
                const double x = sm.X[rxw][c];
                if (!exact) {
                    double sum = 0.0;
                    for (int d = jj + 1; d <= K; ++d) sum = fma(sm.w[d - 1][c], sm.Y[d - jj][c], sum);
                    part = fma(x, sum, part);
                } else {
                    const int rxv = sm.rX[rxw][c];
                    for (int d = jj + 1; d <= K; ++d)
                        part += scaled_term(x, sm.w[d - 1][c] * sm.Y[d - jj][c], rxv, sm.rY[d - jj][c]);
                }
            }
            sm.win[grp][c] = part;
        }
        __syncthreads();
        if (grp == 0 && c < C) {
            double mu = 0.0;
#pragma unroll
            for (int gg = 0; gg < 8; ++gg) mu += sm.win[gg][c];
            const int u1 = min(u0 + kPC, L);
            float *dx = a.dX + ((size_t)b * T + u0) * C + c;
            double msum = mu;
            dx[0] = (float)mu;
            for (int u = u0 + 1; u < u1; ++u) {
                mu += sm.delta[u - u0][c];
                dx[(size_t)(u - u0) * C] = (float)mu;
                msum += mu;
            }
            a.covm[((size_t)b * nch + ch) * C + c] = msum;
        }
        // ---- dA over the item's transition positions, a 2 x 2 block per thread
        {
            double t4[4] = {0.0, 0.0, 0.0, 0.0};
#pragma unroll 4
            for (int si = 0; si < kPC; ++si) {
                const double2 x = *reinterpret_cast<const double2 *>(&sm.a2[si][2 * ci2]);
                const double2 y = *reinterpret_cast<const double2 *>(&sm.bp[si][2 * cj2]);
                t4[0] = fma(x.x, y.x, t4[0]);
                t4[1] = fma(x.x, y.y, t4[1]);
                t4[2] = fma(x.y, y.x, t4[2]);
                t4[3] = fma(x.y, y.y, t4[3]);
            }
#pragma unroll
            for (int k = 0; k < 4; ++k) accA[k] = fma(g, t4[k], accA[k]);
        }
    }
    const size_t z = blockIdx.x;
    // dD: the row parts of each duration block added in order
    __syncthreads();
#pragma unroll
    for (int k = 0; k < 4; ++k) sm.red[grp][k][lane] = accD[k];
    __syncthreads();
    if (grp < nDB && lane < C) {
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            const int d = d0 + k;
            if (d > K) break;
            double sD = 0.0;
            for (int p2 = 0; p2 < nparts; ++p2) sD += sm.red[p2 * nDB + grp][k][lane];
            a.partD[(z * K + (d - 1)) * C + lane] = sD;
        }
    }
#pragma unroll
    for (int k = 0; k < 4; ++k) {
        const int cc = 2 * ci2 + (k >> 1), e = 2 * cj2 + (k & 1);
        if (cc < C && e < C) a.partA[(z * C + cc) * C + e] = accA[k];
    }
}

// CTAs [0, B*ppb): dX of part p of sequence b.  CTAs past them: one warp per
// parameter-gradient output.
__global__ void __launch_bounds__(256) team_finalise_kernel(FbArgs a, int ppb)
{
    __shared__ double red[8][32];
    __shared__ double mean[32];
    const int C = a.C, T = a.T, K = a.K;
    const int nch = (T + kPC - 1) / kPC;
    const int nX = a.B * ppb;
    if ((int)blockIdx.x < nX) {
        const int b = blockIdx.x / ppb, p = blockIdx.x % ppb;
        const int L = a.lengths[b];
        const bool okL = L >= 1 && L <= T;
        const int lane = threadIdx.x & 31, grp = threadIdx.x >> 5;
        if (okL) {
            double s = 0.0;
            const int nchL = (L + kPC - 1) / kPC;
            const double *cm = a.covm + (size_t)b * nch * C + min(lane, C - 1);
            for (int ch0 = grp; ch0 < nchL; ch0 += 32) {   // four chunks per round, loads first
                double v[4];
#pragma unroll
                for (int k = 0; k < 4; ++k) v[k] = cm[(size_t)min(ch0 + 8 * k, nchL - 1) * C];
#pragma unroll
                for (int k = 0; k < 4; ++k)
                    if (ch0 + 8 * k < nchL) s += v[k];
            }
            if (lane >= C) s = 0.0;
            red[grp][lane] = s;
            __syncthreads();
            if (grp == 0) {
                double m = 0.0;
#pragma unroll
                for (int gg = 0; gg < 8; ++gg) m += red[gg][lane];
                mean[lane] = m / (double)L;
            }
            __syncthreads();
        }
        const double g = a.grad ? a.grad[b] : 1.0;
        const int rows = (T + ppb - 1) / ppb;
        const int r0 = p * rows, r1 = min(T, r0 + rows);
        float *dx = a.dX + (size_t)b * T * C;
        const size_t e0 = (size_t)r0 * C, e1 = (size_t)r1 * C;
        for (size_t i0 = e0 + threadIdx.x; i0 < e1; i0 += 4 * blockDim.x) {
            float v[4];
#pragma unroll
            for (int k = 0; k < 4; ++k) v[k] = dx[min(i0 + (size_t)k * blockDim.x, e1 - 1)];
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                const size_t i = i0 + (size_t)k * blockDim.x;
                if (i >= e1) break;
                const int u = (int)(i / C), c = (int)(i % C);
                dx[i] = (okL && u < L) ? (float)(g * ((double)v[k] - mean[c])) : 0.0f;
            }
        }
        return;
    }
    const int nA = C * C, nD = K * C;
    const int lane = threadIdx.x & 31;
    const int w0 = ((blockIdx.x - nX) * blockDim.x + threadIdx.x) >> 5;
    const int nw = ((gridDim.x - nX) * blockDim.x) >> 5;
    for (int i = w0; i < nA + nD; i += nw) {
        const double *src = i < nA ? a.partA + i : a.partD + (i - nA);
        const size_t stride = i < nA ? (size_t)nA : (size_t)nD;
        double s = 0.0;
        for (int z0 = lane; z0 < a.npost; z0 += 8 * 32) {   // eight splits per round, loads first
            double v[8];
#pragma unroll
            for (int k = 0; k < 8; ++k) v[k] = src[(size_t)min(z0 + 32 * k, a.npost - 1) * stride];
#pragma unroll
            for (int k = 0; k < 8; ++k)
                if (z0 + 32 * k < a.npost) s += v[k];
        }
        for (int off = 16; off > 0; off >>= 1) s += __shfl_xor_sync(0xffffffffu, s, off);
        if (lane == 0) {
            if (i < nA) a.dA[i] = exp((double)a.A[i]) * s;
            else a.dD[i - nA] = exp((double)a.D[i - nA]) * s;
        }
    }
}

}  // namespace

// Pass-1 CTAs: one item each up to two CTAs per SM (the shared-memory footprint
// allows two), then items are shared out in contiguous runs.
int team_post_splits(int B, int T)
{
    const long long Q = (long long)B * ((T + kPC - 1) / kPC);
    const int cap = 2 * device_sm_count();
    return (int)(Q < cap ? Q : cap);
}

int team_post_chunks(int T) { return (T + kPC - 1) / kPC; }

cudaError_t launch_team_post(const FbArgs &a, cudaStream_t st)
{
    const size_t smem = sizeof(PostSmem);
    cudaError_t e = cudaFuncSetAttribute(team_post_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    prof_before(st);
    team_post_kernel<<<a.npost, kPT, smem, st>>>(a);
    prof_after(st);
    long long ppb = ((long long)a.T * a.C + kDxPer - 1) / kDxPer;
    if (ppb > kPC) ppb = kPC;
    if (ppb < 1) ppb = 1;
    const int nP = (int)(((long long)(a.C * a.C + a.K * a.C) * 32 + 255) / 256);
    prof_before(st);
    const int nsm = device_sm_count();
    team_finalise_kernel<<<(unsigned)(a.B * ppb + (nP < nsm ? nP : nsm)), 256, 0, st>>>(a, (int)ppb);
    prof_after(st);
    return cudaGetLastError();
}

}  // namespace semicrf
