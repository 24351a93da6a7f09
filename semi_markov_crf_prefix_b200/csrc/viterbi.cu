// viterbi.cu -- best segmentation of the semi-CRF, (max, +) in float64.
//
// The segment score is the one of Streaming Structured Inference with
// Flash-SemiCRF (abstract; technical summary 2.A): S[t,c] - S[s,c] + D[t-s-1,c],
// plus A[c',c] between consecutive segments.  The pages do not describe
// decoding; this is the forward recursion with (max, +) in place of (lse, +):
//   vt[0,c] = 0
//   v[t,c]  = max_d ( (vt[t-d,c] + (S[t,c] - S[t-d,c])) + D[d-1,c] ),  1 <= d <= min(K,t)
//   vt[t,c] = max_c' ( v[t,c'] + A[c',c] ),                            1 <= t < L
// evaluated in exactly this operand order, with ties broken towards the smallest
// d, then the smallest c', and the final label the smallest c reaching
// max_c v[L,c].  Backpointers: bd[t,c] (best d), bc[t,c] (best c').
//
// Same cluster layout as the forward kernel: labels split across the CTAs of a
// cluster, each CTA keeps rings of vt and S for its labels in shared memory,
// v[t,:] is all-gathered through distributed shared memory every step.  A
// second kernel walks the backpointers (one thread per sequence).
#include <math.h>

#include "device_util.cuh"
#include "semicrf_internal.h"

namespace semicrf {
namespace {

struct VGeom {
    int G, NT, Cg, JL;
};

template <bool CLUSTER>
__device__ __forceinline__ void vbarrier()
{
    if constexpr (CLUSTER)
        cluster_barrier();
    else
        __syncthreads();
}

// better (value, index): larger value; on equal values the smaller index
__device__ __forceinline__ bool better(double v, int i, double bv, int bi)
{
    return v > bv || (v == bv && i < bi);
}

template <int DPT, int CPT, bool CLUSTER>
__global__ void __launch_bounds__(kMaxThreads, 1) viterbi_kernel(VitArgs a, VGeom geo)
{
    extern __shared__ __align__(16) unsigned char smem_raw[];
    const int K = a.K, C = a.C, Cg = geo.Cg, NT = geo.NT, JL = geo.JL;
    double *vring = reinterpret_cast<double *>(smem_raw);   // [K][Cg] vt rows
    double *sring = vring + (size_t)K * Cg;                    // [K][Cg] S rows
    double *gath = sring + (size_t)K * Cg;                     // [2][C]
    double *pv = gath + 2 * C;                                 // [NT]
    int *pi = reinterpret_cast<int *>(pv + NT);                // [NT]

    const int rank = CLUSTER ? (int)cluster_rank() : 0;
    const int b = blockIdx.x / geo.G;
    const int L = a.lengths[b];
    if (L < 1 || L > a.T) {
        if (rank == 0 && threadIdx.x == 0) set_status(a.status, SEMICRF_ERR_INVALID_LENGTH);
        return;
    }
    const int tid = threadIdx.x, lc = tid % Cg, j = tid / Cg;
    const bool active = j < JL;
    const int c0 = rank * Cg, cg_own = min(Cg, C - c0), c = c0 + lc;
    const bool valid_lc = lc < cg_own, is_label = tid < cg_own;
    const double *Sb = a.S + (size_t)b * (a.T + 1) * C;
    const size_t rowbase = (size_t)b * (a.T + 1);

    double Dv[DPT], Av[CPT];
#pragma unroll
    for (int m = 0; m < DPT; ++m) {
        int d = 1 + j + m * JL;
        Dv[m] = (active && valid_lc && d <= K) ? (double)a.D[(size_t)(d - 1) * C + c] : 0.0;
    }
#pragma unroll
    for (int m = 0; m < CPT; ++m) {
        int cp = j + m * JL;
        Av[m] = (active && valid_lc && cp < C) ? (double)a.A[(size_t)cp * C + c] : 0.0;
    }
    for (int i = tid; i < K * Cg; i += NT) {
        vring[i] = 0.0;
        sring[i] = 0.0;
    }
    if constexpr (CLUSTER) cluster_barrier();
    else __syncthreads();

    const bool in_use = active && valid_lc;
    double St = in_use ? Sb[(size_t)1 * C + c] : 0.0;
    for (int t = 1; t <= L; ++t) {
        const int par = t & 1;
        const double St_next = (in_use && t < L) ? Sb[(size_t)(t + 1) * C + c] : 0.0;
        // (A) best duration over this thread's share, smallest d on ties
        double best = -INFINITY;
        int arg = 0;
        if (in_use) {
            int slot = mod_pos(t - 1 - j, K);
#pragma unroll
            for (int m = 0; m < DPT; ++m) {
                const int d = 1 + j + m * JL;
                if (d <= K && d <= t) {
                    const double cand = (vring[slot * Cg + lc] + (St - sring[slot * Cg + lc])) + Dv[m];
                    if (cand > best) {
                        best = cand;
                        arg = d;
                    }
                }
                slot -= JL;
                if (slot < 0) slot += K;
            }
        }
        pv[tid] = best;
        pi[tid] = arg;
        __syncthreads();
        // (B) per label: v[t,c] and bd[t,c]; all-gather v
        if (is_label) {
            double bv = -INFINITY;
            int bi = 0;
            for (int jj = 0; jj < JL; ++jj) {
                const int idx = lc + Cg * jj;
                if (pi[idx] > 0 && (bi == 0 || better(pv[idx], pi[idx], bv, bi))) {
                    bv = pv[idx];
                    bi = pi[idx];
                }
            }
            a.bd[(rowbase + t) * C + c] = (uint16_t)bi;
            if constexpr (CLUSTER) {
                for (int g2 = 0; g2 < geo.G; ++g2) st_cluster_f64(&gath[par * C + c], g2, bv);
            } else {
                gath[par * C + c] = bv;
            }
        }
        vbarrier<CLUSTER>();
        if (t == L) {
            if (rank == 0 && tid < 32) {
                double bv = -INFINITY;
                int bi = C;
                for (int cc = tid; cc < C; cc += 32) {
                    const double v = gath[par * C + cc];
                    if (v > bv) {
                        bv = v;
                        bi = cc;
                    }
                }
#pragma unroll
                for (int off = 16; off > 0; off >>= 1) {
                    const double ov = __shfl_xor_sync(0xffffffffu, bv, off);
                    const int oi = __shfl_xor_sync(0xffffffffu, bi, off);
                    if (better(ov, oi, bv, bi)) {
                        bv = ov;
                        bi = oi;
                    }
                }
                if (tid == 0) {
                    a.score[b] = bv;
                    a.vfin[b] = bi;
                }
            }
            break;
        }
        // (C) best previous label over this thread's share, smallest c' on ties
        best = -INFINITY;
        arg = -1;
        if (in_use) {
#pragma unroll
            for (int m = 0; m < CPT; ++m) {
                const int cp = j + m * JL;
                if (cp < C) {
                    const double cand = gath[par * C + cp] + Av[m];
                    if (cand > best) {
                        best = cand;
                        arg = cp;
                    }
                }
            }
        }
        pv[tid] = best;
        pi[tid] = arg;
        __syncthreads();
        // (D) per label: vt[t,c], bc[t,c]; ring rows
        if (is_label) {
            double bv = -INFINITY;
            int bi = -1;
            for (int jj = 0; jj < JL; ++jj) {
                const int idx = lc + Cg * jj;
                if (pi[idx] >= 0 && (bi < 0 || better(pv[idx], pi[idx], bv, bi))) {
                    bv = pv[idx];
                    bi = pi[idx];
                }
            }
            a.bc[(rowbase + t) * C + c] = (uint16_t)bi;
            vring[(t % K) * Cg + lc] = bv;
            sring[(t % K) * Cg + lc] = St;
        }
        St = St_next;
        __syncthreads();
    }
    if constexpr (CLUSTER) cluster_barrier();
}

// Walk the backpointers from (L, final label): labels and segment starts.
__global__ void viterbi_backtrack(VitArgs a)
{
    const int b = blockIdx.x * blockDim.x + threadIdx.x;
    if (b >= a.B) return;
    const int L = a.lengths[b];
    int32_t *lab = a.labels + (size_t)b * a.T;
    uint8_t *ss = a.seg_start + (size_t)b * a.T;
    if (L < 1 || L > a.T) return;
    for (int u = L; u < a.T; ++u) {
        lab[u] = -1;
        ss[u] = 0;
    }
    const size_t rowbase = (size_t)b * (a.T + 1);
    int t = L, c = a.vfin[b];
    while (t > 0) {
        int d = a.bd[(rowbase + t) * a.C + c];
        if (d < 1 || d > t) {   // cannot happen for finite scores; stop rather than loop
            set_status(a.status, SEMICRF_ERR_DEVICE_RANGE);
            return;
        }
        const int s = t - d;
        for (int u = s; u < t; ++u) {
            lab[u] = c;
            ss[u] = (u == s) ? 1 : 0;
        }
        if (s > 0) c = a.bc[(rowbase + s) * a.C + c];
        t = s;
    }
}

template <int DPT, int CPT>
cudaError_t launch_vit_tpl(const Plan &p, const VitArgs &a, cudaStream_t st)
{
    VGeom geo{p.G, p.NT, p.Cg, p.JL};
    const bool cl = p.G > 1;
    void *fn = cl ? (void *)viterbi_kernel<DPT, CPT, true> : (void *)viterbi_kernel<DPT, CPT, false>;
    cudaError_t e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)p.smem_vit);
    if (e != cudaSuccess) return e;
    if (p.G > 8) {
        e = cudaFuncSetAttribute(fn, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
        if (e != cudaSuccess) return e;
    }
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)a.B * p.G);
    cfg.blockDim = dim3(p.NT);
    cfg.dynamicSmemBytes = p.smem_vit;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    if (cl) {
        attr[0].id = cudaLaunchAttributeClusterDimension;
        attr[0].val.clusterDim.x = p.G;
        attr[0].val.clusterDim.y = 1;
        attr[0].val.clusterDim.z = 1;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
    }
    VitArgs aa = a;
    void *args[] = {&aa, &geo};
    prof_before(st);
    e = cudaLaunchKernelExC(&cfg, fn, args);
    prof_after(st);
    return e;
}

using VitLauncher = cudaError_t (*)(const Plan &, const VitArgs &, cudaStream_t);
#define SEMICRF_VROW(D) \
    { launch_vit_tpl<D, 2>, launch_vit_tpl<D, 4>, launch_vit_tpl<D, 8>, launch_vit_tpl<D, 16> }
const VitLauncher kVitTable[5][4] = {SEMICRF_VROW(2), SEMICRF_VROW(4), SEMICRF_VROW(8),
                                     SEMICRF_VROW(16), SEMICRF_VROW(32)};
#undef SEMICRF_VROW

int vlog2_index(int v, int lo)
{
    int i = 0;
    for (int x = lo; x < v; x <<= 1) ++i;
    return i;
}

}  // namespace

cudaError_t launch_viterbi(const Plan &p, const VitArgs &a, cudaStream_t st, int *launches)
{
    int di = vlog2_index(p.DPT, 2), ci = vlog2_index(p.CPT, 2);
    if (di > 4 || ci > 3) return cudaErrorInvalidConfiguration;
    cudaError_t e = kVitTable[di][ci](p, a, st);
    if (e != cudaSuccess) return e;
    prof_before(st);
    viterbi_backtrack<<<(a.B + 63) / 64, 64, 0, st>>>(a);
    prof_after(st);
    *launches += 2;
    return cudaGetLastError();
}

}  // namespace semicrf
