// forward_backward.cu -- streaming semi-CRF forward, checkpoint recompute,
// backward with marginals, and gradient finalisation.
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
// Parallel layout: one thread-block cluster per sequence (per checkpoint
// segment when recomputing), labels split across its CTAs; each CTA keeps its
// ring slice in shared memory, exp(D) and exp(A) for its (d, c) and (c', c)
// items in registers, and all-gathers the C values a'[t,:] through distributed
// shared memory once per step.
#include <math.h>
#include <stdlib.h>
#include <string.h>

#include "device_util.cuh"
#include "semicrf_internal.h"

namespace semicrf {
namespace {

struct KernelGeom {
    int G, NT, Cg, JL;
};

struct Roles {
    int tid, lc, j, c0, cg_own, c;
    bool active, is_label, valid_lc;
};

__device__ __forceinline__ Roles make_roles(const KernelGeom &g, int C, int rank)
{
    Roles r;
    r.tid = threadIdx.x;
    r.lc = r.tid % g.Cg;
    r.j = r.tid / g.Cg;
    r.active = r.j < g.JL;
    r.c0 = rank * g.Cg;
    r.cg_own = min(g.Cg, C - r.c0);
    r.c = r.c0 + r.lc;
    r.valid_lc = r.lc < r.cg_own;
    r.is_label = (r.tid < r.cg_own);
    return r;
}

template <bool CLUSTER>
__device__ __forceinline__ void step_barrier()
{
    if constexpr (CLUSTER)
        cluster_barrier();
    else
        __syncthreads();
}

// Deterministic sum of v[0..n) by one warp (identical on every CTA that calls it).
__device__ __forceinline__ double warp_sum(const double *v, int n)
{
    const int lane = threadIdx.x & 31;
    double s = 0.0;
    for (int i = lane; i < n; i += 32) s += v[i];
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) s += __shfl_xor_sync(0xffffffffu, s, off);
    return s;
}

// ---------------------------------------------------------------------------
// Forward (RECOMPUTE = false): one cluster per sequence, t = 1..L, writes a
// checkpoint (ring, r, k_{t+1}) after every delta-th step and log Z at t = L.
// Recompute (RECOMPUTE = true): one cluster per (sequence, checkpoint segment j),
// restores checkpoint j and replays t = j*delta+1 .. min((j+1)*delta, L),
// storing U[t,:], r, a'[t,:] and k_t per position for the backward.
// ---------------------------------------------------------------------------
template <int DPT, int CPT, bool CLUSTER, bool RECOMPUTE>
__global__ void __launch_bounds__(kMaxThreads, 1) fwd_kernel(FbArgs a, KernelGeom geo)
{
    extern __shared__ __align__(16) unsigned char smem_raw[];
    const int K = a.K, C = a.C, Cg = geo.Cg, NT = geo.NT, JL = geo.JL;
    double *ring = reinterpret_cast<double *>(smem_raw);   // [K][Cg]
    double *gath = ring + (size_t)K * Cg;                     // [2][C]
    double *part = gath + 2 * C;                              // [NT]
    int *shift = reinterpret_cast<int *>(part + NT);          // [Cg]
    int *flags = shift + Cg;                                  // [0]=any rebase, [1]=k_next

    const int rank = CLUSTER ? (int)cluster_rank() : 0;
    const int cluster_id = blockIdx.x / geo.G;
    int b, seg;
    if constexpr (RECOMPUTE) {
        b = cluster_id / a.J;
        seg = cluster_id % a.J;
    } else {
        b = cluster_id;
        seg = 0;
    }
    const int L = a.lengths[b];
    if (L < 1 || L > a.T) {
        if (rank == 0 && threadIdx.x == 0 && seg == 0) set_status(a.status, SEMICRF_ERR_INVALID_LENGTH);
        return;
    }
    const int t_begin = seg * a.delta;
    if (RECOMPUTE && t_begin >= L) return;
    const int t_end = RECOMPUTE ? min(t_begin + a.delta, L) : L;

    const Roles ro = make_roles(geo, C, rank);
    const double *Sb = a.S + (size_t)b * (a.T + 1) * C;

    // exp(D) for this thread's durations, exp(A[c', c]) for its previous labels
    double W[DPT], E[CPT];
#pragma unroll
    for (int m = 0; m < DPT; ++m) {
        int d = 1 + ro.j + m * JL;
        W[m] = (ro.active && ro.valid_lc && d <= K) ? exp((double)a.D[(size_t)(d - 1) * C + ro.c]) : 0.0;
    }
#pragma unroll
    for (int m = 0; m < CPT; ++m) {
        int cp = ro.j + m * JL;
        E[m] = (ro.active && ro.valid_lc && cp < C) ? exp((double)a.A[(size_t)cp * C + ro.c]) : 0.0;
    }

    unsigned char *ck_base = a.ckpt + ((size_t)b * a.J) * a.ckpt_stride;
    int r = 0;   // label thread: ring exponent of its column
    int k = 0;   // all threads: alpha exponent k_t for the current step
    if constexpr (RECOMPUTE) {
        const unsigned char *ck = ck_base + (size_t)seg * a.ckpt_stride;
        const double *ck_ring = reinterpret_cast<const double *>(ck);
        const int32_t *ck_r = reinterpret_cast<const int32_t *>(ck_ring + (size_t)K * C);
        for (int i = ro.tid; i < K * Cg; i += NT) {
            int slot = i / Cg, l2 = i % Cg;
            ring[i] = (l2 < ro.cg_own) ? ck_ring[(size_t)slot * C + ro.c0 + l2] : 0.0;
        }
        if (ro.is_label) r = ck_r[ro.c];
        k = ck_r[C];
    } else {
        for (int i = ro.tid; i < K * Cg; i += NT) ring[i] = 0.0;
        __syncthreads();
        if (ro.is_label) ring[ro.lc] = 1.0;   // row 0: U[0,c] = exp(0)
        // checkpoint 0: the initial state
        __syncthreads();
        double *ck_ring = reinterpret_cast<double *>(ck_base);
        int32_t *ck_r = reinterpret_cast<int32_t *>(ck_ring + (size_t)K * C);
        for (int i = ro.tid; i < K * Cg; i += NT) {
            int slot = i / Cg, l2 = i % Cg;
            if (l2 < ro.cg_own) ck_ring[(size_t)slot * C + ro.c0 + l2] = ring[i];
        }
        if (ro.is_label) ck_r[ro.c] = 0;
        if (rank == 0 && ro.tid == 0) ck_r[C] = 0;
    }
    if (ro.tid == 0) flags[0] = 0;
    if (ro.tid < Cg) shift[ro.tid] = 0;
    if constexpr (CLUSTER) cluster_barrier();
    else __syncthreads();

    double ap = 0.0;
    double St = ro.is_label ? Sb[(size_t)(t_begin + 1) * C + ro.c] : 0.0;
    // recompute output is relative to Z: c0 = exp(-log sum a'_L), exponents minus k_L
    int kZ = 0;
    double c0 = 0.0;
    if constexpr (RECOMPUTE) {
        kZ = a.lz[b].k;
        c0 = exp(-a.lz[b].logn);
    }
    for (int t = t_begin + 1; t <= t_end; ++t) {
        const int par = t & 1;
        // next step's S row, fetched a step ahead
        const double St_next = (ro.is_label && t < t_end) ? Sb[(size_t)(t + 1) * C + ro.c] : 0.0;
        // (A) duration sum, this thread's share: sum_m U[t-d_m, c] exp(D[d_m-1, c])
        double pacc = 0.0;
        if (ro.active) {
            int slot = mod_pos(t - 1 - ro.j, K);
#pragma unroll
            for (int m = 0; m < DPT; ++m) {
                pacc = fma(ring[slot * Cg + ro.lc], W[m], pacc);
                slot -= JL;
                if (slot < 0) slot += K;
            }
        }
        part[ro.tid] = pacc;
        __syncthreads();
        // (B) per label: p, a'[t,c], rebase decision, all-gather of a'
        if (ro.is_label) {
            double p = 0.0;
            for (int jj = 0; jj < JL; ++jj) p += part[ro.lc + Cg * jj];
            ap = p * exp(St + kLn2 * (double)(r - k));
            int ex = exponent_of(p);
            int h = (ex > kRebaseBits || ex < -kRebaseBits) ? -ex : 0;
            shift[ro.lc] = h;
            if (h) {
                r -= h;
                flags[0] = 1;
            }
            if constexpr (CLUSTER) {
                for (int g2 = 0; g2 < geo.G; ++g2) st_cluster_f64(&gath[par * C + ro.c], g2, ap);
            } else {
                gath[par * C + ro.c] = ap;
            }
        }
        step_barrier<CLUSTER>();
        if (t == L) {
            // log Z = ln2 k_L + log sum_c a'[L,c]
            if (ro.tid < 32) {
                double n = warp_sum(gath + par * C, C);
                if (!RECOMPUTE && rank == 0 && ro.tid == 0) {
                    double lz = kLn2 * (double)k + log(n);
                    a.logZ[b] = lz;
                    a.lz[b].logn = log(n);
                    a.lz[b].k = k;
                    if (!isfinite(lz)) set_status(a.status, SEMICRF_ERR_DEVICE_RANGE);
                }
            }
            if (RECOMPUTE) {
                size_t row = ((size_t)b * (a.T + 1) + t) * C;
                if (ro.is_label) a.cA[row + ro.c] = ap * c0;
                if (rank == 0 && ro.tid == 0) a.eA[(size_t)b * (a.T + 1) + t] = k - kZ;
            }
            break;
        }
        // (C) transition sum, next normaliser, pending column rescales
        double qacc = 0.0;
        if (ro.active) {
#pragma unroll
            for (int m = 0; m < CPT; ++m) {
                int cp = ro.j + m * JL;
                if (cp < C) qacc = fma(gath[par * C + cp], E[m], qacc);
            }
        }
        part[ro.tid] = qacc;
        if (ro.tid < 32) {
            double n = warp_sum(gath + par * C, C);
            if (ro.tid == 0) flags[1] = k + exponent_of(n);
        }
        if (flags[0]) {
            for (int i = ro.tid; i < K * Cg; i += NT) {
                int h = shift[i % Cg];
                if (h) ring[i] *= pow2(h);
            }
        }
        __syncthreads();
        // (D) per label: new ring row U[t,c]
        const int knext = flags[1];
        if (ro.is_label) {
            double q = 0.0;
            for (int jj = 0; jj < JL; ++jj) q += part[ro.lc + Cg * jj];
            double U = q * exp(kLn2 * (double)(k - r) - St);
            ring[(t % K) * Cg + ro.lc] = U;
            if constexpr (RECOMPUTE) {
                size_t row = ((size_t)b * (a.T + 1) + t) * C + ro.c;
                a.cU[row] = U * c0;
                a.cA[row] = ap * c0;
                a.eU[row] = r - kZ;
            }
        }
        if (RECOMPUTE && rank == 0 && ro.tid == 0) a.eA[(size_t)b * (a.T + 1) + t] = k - kZ;
        if (!RECOMPUTE && (t % a.delta) == 0) {
            // checkpoint t / delta: ring after step t, r, k_{t+1}
            __syncthreads();
            unsigned char *ck = ck_base + (size_t)(t / a.delta) * a.ckpt_stride;
            double *ck_ring = reinterpret_cast<double *>(ck);
            int32_t *ck_r = reinterpret_cast<int32_t *>(ck_ring + (size_t)K * C);
            for (int i = ro.tid; i < K * Cg; i += NT) {
                int slot = i / Cg, l2 = i % Cg;
                if (l2 < ro.cg_own) ck_ring[(size_t)slot * C + ro.c0 + l2] = ring[i];
            }
            if (ro.is_label) ck_r[ro.c] = r;
            if (rank == 0 && ro.tid == 0) ck_r[C] = knext;
        }
        k = knext;
        St = St_next;
        __syncthreads();
        if (ro.tid == 0) flags[0] = 0;
    }
    if constexpr (CLUSTER) cluster_barrier();   // no CTA leaves while peers may still store to it
}

// ---------------------------------------------------------------------------
// Backward: one cluster per sequence, s = L-1 .. 0.  The ring holds
// V[s,c] = exp(be[s,c] + S[s,c] - ln2 rb_c) for rows s+1..s+K; the backward
// normaliser kb_s scales b'[s,c] = exp(ga[s,c] - ln2 kb_s).
// Per step: pb[c] = sum_d V[s+d,c] exp(D[d-1,c]) (and the dD accumulation
// coef_s[c] * V[s+d,c]), start/end marginals, all-gather of b', the transposed
// transition q[c'] = sum_c exp(A[c',c]) b'[c] (and the dA accumulation
// a2_s[c'] * b'[c]), new ring row, coverage mu written into dX.
// ---------------------------------------------------------------------------
template <int DPT, int CPT, bool CLUSTER>
__global__ void __launch_bounds__(kMaxThreads, 1) bwd_kernel(FbArgs a, KernelGeom geo)
{
    extern __shared__ __align__(16) unsigned char smem_raw[];
    const int K = a.K, C = a.C, Cg = geo.Cg, NT = geo.NT, JL = geo.JL;
    double *ring = reinterpret_cast<double *>(smem_raw);   // [K][Cg]
    double *accD = ring + (size_t)K * Cg;                     // [K][Cg]
    double *gath = accD + (size_t)K * Cg;                     // [2][C]
    double *part = gath + 2 * C;                              // [NT]
    double *coef = part + NT;                                 // [Cg]
    double *a2 = coef + Cg;                                   // [Cg]
    int *shift = reinterpret_cast<int *>(a2 + Cg);            // [Cg]
    int *flags = shift + Cg;

    const int rank = CLUSTER ? (int)cluster_rank() : 0;
    const int b = blockIdx.x / geo.G;
    const int L = a.lengths[b];
    if (L < 1 || L > a.T) {
        if (rank == 0 && threadIdx.x == 0) set_status(a.status, SEMICRF_ERR_INVALID_LENGTH);
        return;
    }
    const Roles ro = make_roles(geo, C, rank);
    const double *Sb = a.S + (size_t)b * (a.T + 1) * C;
    const size_t rowbase = (size_t)b * (a.T + 1);
    const int kZ = a.lz[b].k;
    const double c0 = exp(-a.lz[b].logn);   // 1/sum_c a'[L,c]

    double W[DPT], E[CPT], accA[CPT];
#pragma unroll
    for (int m = 0; m < DPT; ++m) {
        int d = 1 + ro.j + m * JL;
        W[m] = (ro.active && ro.valid_lc && d <= K) ? exp((double)a.D[(size_t)(d - 1) * C + ro.c]) : 0.0;
    }
#pragma unroll
    for (int m = 0; m < CPT; ++m) {
        int cc = ro.j + m * JL;   // next label; this thread's own label is the previous one
        E[m] = (ro.active && ro.valid_lc && cc < C) ? exp((double)a.A[(size_t)ro.c * C + cc]) : 0.0;
        accA[m] = 0.0;
    }
    for (int i = ro.tid; i < K * Cg; i += NT) {
        ring[i] = 0.0;
        accD[i] = 0.0;
    }
    if (ro.tid == 0) flags[0] = 0;
    if (ro.tid < Cg) {
        shift[ro.tid] = 0;
        coef[ro.tid] = 0.0;
        a2[ro.tid] = 0.0;
    }
    __syncthreads();

    int rb = 0, kb = 0;
    double mu_acc = 0.0, musum = 0.0;
    if (ro.is_label) {
        // row L: be[L,c] = 0, so V[L,c] = exp(S[L,c] - ln2 rb) with rb = round(S[L,c]/ln2)
        const double SL = Sb[(size_t)L * C + ro.c];
        rb = (int)rint(SL / kLn2);
        ring[(L % K) * Cg + ro.lc] = exp(SL - kLn2 * (double)rb);
        // coverage of position L-1: P(the last segment has label c) = a'[L,c] / sum a'[L,:]
        mu_acc = scale2(a.cA[(rowbase + L) * C + ro.c], a.eA[rowbase + L]);
        const int s = L - 1;
        if (s == 0) {
            coef[ro.lc] = scale2(c0, rb - kZ);
        } else {
            const size_t row = (rowbase + s) * C + ro.c;
            coef[ro.lc] = scale2(a.cU[row], a.eU[row] + rb);
            a2[ro.lc] = scale2(a.cA[row], a.eA[rowbase + s] + kb);
        }
    }
    if constexpr (CLUSTER) cluster_barrier();
    else __syncthreads();

    double start = 0.0, bp = 0.0;
    double St = ro.is_label ? Sb[(size_t)(L - 1) * C + ro.c] : 0.0;
    for (int s = L - 1; s >= 0; --s) {
        const int par = s & 1;
        // fetched a step ahead: S[s-1] and the forward quantities at s-1
        double St_next = 0.0, nU = 0.0, nA = 0.0;
        int nR = 0, nK = 0;
        if (ro.is_label && s >= 1) {
            St_next = Sb[(size_t)(s - 1) * C + ro.c];
            if (s - 1 >= 1) {
                const size_t row = (rowbase + s - 1) * C + ro.c;
                nU = a.cU[row];
                nA = a.cA[row];
                nR = a.eU[row];
                nK = a.eA[rowbase + s - 1];
            }
        }
        // (A) pb share and dD accumulation over this thread's durations
        double pacc = 0.0;
        if (ro.active) {
            const double cf = coef[ro.lc];
            int slot = mod_pos(s + 1 + ro.j, K);
#pragma unroll
            for (int m = 0; m < DPT; ++m) {
                const int d = 1 + ro.j + m * JL;
                const double v = ring[slot * Cg + ro.lc];
                pacc = fma(v, W[m], pacc);
                if (d <= K) accD[(d - 1) * Cg + ro.lc] = fma(cf, v, accD[(d - 1) * Cg + ro.lc]);
                slot += JL;
                if (slot >= K) slot -= K;
            }
        }
        part[ro.tid] = pacc;
        __syncthreads();
        // (B) per label: pb, start marginal, b', rebase decision, all-gather of b'
        if (ro.is_label) {
            double pb = 0.0;
            for (int jj = 0; jj < JL; ++jj) pb += part[ro.lc + Cg * jj];
            start = coef[ro.lc] * pb;
            bp = pb * exp(kLn2 * (double)(rb - kb) - St);
            int ex = exponent_of(pb);
            int h = (ex > kRebaseBits || ex < -kRebaseBits) ? -ex : 0;
            shift[ro.lc] = h;
            if (h) {
                rb -= h;
                flags[0] = 1;
            }
            if constexpr (CLUSTER) {
                for (int g2 = 0; g2 < geo.G; ++g2) st_cluster_f64(&gath[par * C + ro.c], g2, bp);
            } else {
                gath[par * C + ro.c] = bp;
            }
        }
        step_barrier<CLUSTER>();
        if (s == 0) {
            if (ro.tid < 32) {
                double n = warp_sum(gath + par * C, C);
                if (rank == 0 && ro.tid == 0) a.logzb[b] = kLn2 * (double)kb + log(n);
            }
            if (ro.is_label) {
                a.dX[((size_t)b * a.T + 0) * C + ro.c] = (float)mu_acc;
                musum += mu_acc;
                mu_acc -= start;
            }
            break;
        }
        // (C) transposed transition share and dA accumulation; next normaliser; rescales
        double qacc = 0.0;
        if (ro.active) {
            const double a2v = a2[ro.lc];
#pragma unroll
            for (int m = 0; m < CPT; ++m) {
                const int cc = ro.j + m * JL;
                if (cc < C) {
                    const double g = gath[par * C + cc];
                    qacc = fma(E[m], g, qacc);
                    accA[m] = fma(a2v, g, accA[m]);
                }
            }
        }
        part[ro.tid] = qacc;
        if (ro.tid < 32) {
            double n = warp_sum(gath + par * C, C);
            if (ro.tid == 0) flags[1] = kb + exponent_of(n);
        }
        if (flags[0]) {
            for (int i = ro.tid; i < K * Cg; i += NT) {
                int h = shift[i % Cg];
                if (h) ring[i] *= pow2(h);
            }
        }
        __syncthreads();
        // (D) per label: new ring row, end marginal, coverage; next step's coefficients
        const int kbn = flags[1];
        if (ro.is_label) {
            double q = 0.0;
            for (int jj = 0; jj < JL; ++jj) q += part[ro.lc + Cg * jj];
            ring[(s % K) * Cg + ro.lc] = q * exp(kLn2 * (double)(kb - rb) + St);
            const double end = a2[ro.lc] * q;
            a.dX[((size_t)b * a.T + s) * C + ro.c] = (float)mu_acc;
            musum += mu_acc;
            mu_acc += end - start;
            if (s - 1 == 0) {
                coef[ro.lc] = scale2(c0, rb - kZ);
                a2[ro.lc] = 0.0;
            } else {
                coef[ro.lc] = scale2(nU, nR + rb);
                a2[ro.lc] = scale2(nA, nK + kbn);
            }
        }
        kb = kbn;
        St = St_next;
        __syncthreads();
        if (ro.tid == 0) flags[0] = 0;
    }
    __syncthreads();
    // per-sequence partial gradients
    double *accD_g = a.accD + (size_t)b * K * C;
    for (int i = ro.tid; i < K * Cg; i += NT) {
        int d0 = i / Cg, l2 = i % Cg;
        if (l2 < ro.cg_own) accD_g[(size_t)d0 * C + ro.c0 + l2] = accD[i];
    }
    if (ro.active && ro.valid_lc) {
        double *accA_g = a.accA + (size_t)b * C * C + (size_t)ro.c * C;
#pragma unroll
        for (int m = 0; m < CPT; ++m) {
            const int cc = ro.j + m * JL;
            if (cc < C) accA_g[cc] = accA[m];
        }
    }
    if (ro.is_label) {
        a.musum[(size_t)b * C + ro.c] = musum;
        a.mures[(size_t)b * C + ro.c] = mu_acc;
    }
    if constexpr (CLUSTER) cluster_barrier();
}

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

// ---------------------------------------------------------------------------
// Template dispatch over (DPT, CPT, cluster or not)
// ---------------------------------------------------------------------------
template <int DPT, int CPT>
cudaError_t launch_fb_tpl(const Plan &p, const FbArgs &a, cudaStream_t st, int kind)
{
    KernelGeom geo{p.G, p.NT, p.Cg, p.JL};
    const bool cl = p.G > 1;
    void *fn;
    size_t smem;
    unsigned nclusters;
    if (kind == 0) {
        fn = cl ? (void *)fwd_kernel<DPT, CPT, true, false> : (void *)fwd_kernel<DPT, CPT, false, false>;
        smem = p.smem_fwd;
        nclusters = a.B;
    } else if (kind == 1) {
        fn = cl ? (void *)fwd_kernel<DPT, CPT, true, true> : (void *)fwd_kernel<DPT, CPT, false, true>;
        smem = p.smem_fwd;
        nclusters = (unsigned)a.B * (unsigned)a.J;
    } else {
        fn = cl ? (void *)bwd_kernel<DPT, CPT, true> : (void *)bwd_kernel<DPT, CPT, false>;
        smem = p.smem_bwd;
        nclusters = a.B;
    }
    cudaError_t e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    if (p.G > 8) {
        e = cudaFuncSetAttribute(fn, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
        if (e != cudaSuccess) return e;
    }
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(nclusters * p.G);
    cfg.blockDim = dim3(p.NT);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    cfg.numAttrs = 0;
    if (cl) {
        attr[0].id = cudaLaunchAttributeClusterDimension;
        attr[0].val.clusterDim.x = p.G;
        attr[0].val.clusterDim.y = 1;
        attr[0].val.clusterDim.z = 1;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
    }
    FbArgs aa = a;
    void *args[] = {&aa, &geo};
    prof_before(st);
    e = cudaLaunchKernelExC(&cfg, fn, args);
    prof_after(st);
    return e;
}

using FbLauncher = cudaError_t (*)(const Plan &, const FbArgs &, cudaStream_t, int);

#define SEMICRF_CPT_ROW(D)                                                                     \
    { launch_fb_tpl<D, 2>, launch_fb_tpl<D, 4>, launch_fb_tpl<D, 8>, launch_fb_tpl<D, 16> }
const FbLauncher kFbTable[5][4] = {SEMICRF_CPT_ROW(2), SEMICRF_CPT_ROW(4), SEMICRF_CPT_ROW(8),
                                   SEMICRF_CPT_ROW(16), SEMICRF_CPT_ROW(32)};
#undef SEMICRF_CPT_ROW

int log2_index(int v, int lo)
{
    int i = 0;
    for (int x = lo; x < v; x <<= 1) ++i;
    return i;
}

FbLauncher pick(const Plan &p)
{
    int di = log2_index(p.DPT, 2), ci = log2_index(p.CPT, 2);
    if (di > 4 || ci > 3) return nullptr;
    return kFbTable[di][ci];
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
    cudaError_t e = launch_exp_tables(a, st);
    if (e != cudaSuccess) return e;
    *launches += 1;
    if (use_small(a.K, a.C)) {
        e = launch_small(a, st, 0);
    } else {
        FbLauncher f = pick(p);
        if (!f) return cudaErrorInvalidConfiguration;
        e = f(p, a, st, 0);
    }
    if (e == cudaSuccess) *launches += 1;
    return e;
}

cudaError_t launch_backward(const Plan &p, const FbArgs &a, cudaStream_t st, int *launches)
{
    cudaError_t e;
    if (use_small(a.K, a.C)) {
        e = launch_small(a, st, 1);   // recompute every checkpoint segment
        if (e != cudaSuccess) return e;
        e = launch_small(a, st, 2);   // backward with marginals
        if (e != cudaSuccess) return e;
    } else {
        FbLauncher f = pick(p);
        if (!f) return cudaErrorInvalidConfiguration;
        e = f(p, a, st, 1);   // recompute every checkpoint segment
        if (e != cudaSuccess) return e;
        e = f(p, a, st, 2);   // backward with marginals
        if (e != cudaSuccess) return e;
    }
    const int nparam = a.C * a.C + a.K * a.C;
    prof_before(st);
    finalise_params<<<(nparam + 255) / 256, 256, 0, st>>>(a);
    prof_after(st);
    const size_t n = (size_t)a.B * a.T * a.C;
    int blocks = (int)((n + 255) / 256);
    if (blocks > 148 * 16) blocks = 148 * 16;
    prof_before(st);
    finalise_dx<<<blocks, 256, 0, st>>>(a);
    prof_after(st);
    *launches += 4;
    return cudaGetLastError();
}

}  // namespace semicrf
