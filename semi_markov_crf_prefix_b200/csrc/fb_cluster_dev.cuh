// fb_cluster_dev.cuh -- device side of the latency-first forward, recompute and
// backward chains for any K and C within the compiled limits: one thread-block
// cluster per sequence (per checkpoint segment when recomputing), labels split
// across its G CTAs.  Included by fb_cluster.cu (planner, launches, the kernels
// whose owners send) and fb_cluster_ts.cu (the kernels whose transition lanes
// send), two sources compiled side by side.
//
// Same recursions and scaled exp-space representation as forward_backward.cu
// (Streaming Structured Inference with Flash-SemiCRF, abstract; technical
// summary 2.A-2.C).  A CTA has three kinds of warps.  Owner warps run the chain
// of one label per lane; transition warps form the C x C product; window warps
// form the duration sums.  The sequential chain of one position is
//   send:        a'[t,c] = U[t-1] (W0 e) + pre e to every CTA of the cluster,
//                completing its bytes on that CTA's mbarrier for the position.
//                TS = 0: the owners form it into a stage buffer and up to four
//                warps issue one bulk copy of the CTA's block per destination
//                (cp.async.bulk, shared::cta to shared::cluster, no multicast).
//                TS = 1: the transition lanes of the label form it right after
//                their sum of the previous position, from values the owners
//                published, and lane j stores it into CTAs j, j + LPL, ... with
//                st.async (no stage, fence or barrier before the send).
//                G = 1: a plain store + bar.arrive;
//   transition:  wait on the mbarrier, q[c] = sum_c' a'[t,c'] exp(A[c',c])
//                (LPL lanes per label, CPL terms each, shuffle reduction);
//                bar.arrive to the owners; the lanes of the first label also
//                sum n_t = sum_c' a'[t,c'] for the normaliser
//   owners:      bar.sync, U[t,c] = q f, the new ring row.
// Work off the chain:
//  * window warps form the duration sum over d >= 3 two positions ahead,
//      pre3_{t+2} = sum_{d=3..K} U[t+2-d] exp(D[d-1]),
//    with their weights exp(D) in registers when their rows fit (8, 16 or 32
//    per lane; zero rows around the ring stand in for the rows past the window).
//    They are paced by their own pair of alternating named barriers with the
//    owners (the owners' new row; the window sums), so a window pass may lag by
//    about a position and a half.  They read the rows at the reference of
//    position t-1 and bring them there themselves (a rebase of a column at t-1
//    rescales every stored row of it by the same power of two, exactly); the
//    owner scales pre3 by the rebases of the two positions in between.
//  * the ring holds every row twice (slots r mod K and r mod K + K), so the
//    K - 2 rows of a window are contiguous and need no wrap arithmetic.
//  * the normaliser is pipelined: k_{t+2} = k_t + floor(log2 n_t) is formed in
//    every CTA from the same sum in the same order and used two positions
//    later; log Z = ln2 k_L + log n_L stays exact.
//  * exp(S) comes from the exp tables, prefetched with cp.async by the owners.
// The backward chain computes beta only and stores, per position, the rows the
// parameter gradients need (V, its reference, the normalised beta and the
// backward normaliser); dA and dD are then dense contractions over all
// positions done by cl_grads.cu on the whole GPU.  The coverage marginal and
// dX stay on the chain (one running sum per label).
// The exchange wait is bounded: a wait that runs out sets
// SEMICRF_ERR_DEVICE_TIMEOUT and that warp skips its later waits; no other wait
// crosses CTAs, so every CTA finishes its loop and all meet at the final
// cluster barrier.  Buffers of a position are indexed by the step count u (0 for
// the first position the kernel runs), so mbarrier phases start at 0.
#pragma once
#include <math.h>
#include <stdint.h>

#include "device_util.cuh"
#include "semicrf_internal.h"

namespace semicrf {
namespace {

constexpr int kPF = 8;                        // exp-table prefetch ring depth (positions)
// Named barriers between the owner and the window warps, two each so that
// consecutive steps alternate: kBarRow + (u & 1) the owners' new row of step u
// (owners arrive, window warps wait), kBarWin + (u & 1) the window sums of step u
// (window warps arrive, owners wait).  Ids 1-5 and 7 serve the other roles.
constexpr int kBarRow = 8;
constexpr int kBarWin = 10;
// Cluster kernels: the owners' values for the next exchange are published
// (owners arrive, transition warps wait), once per step.
constexpr int kBarPub = 6;
// The window warps among themselves: rows of rebased labels rescaled (step u).
constexpr int kBarResc = 12;
constexpr long long kWaitCycles = 1ll << 31;  // ~1 s at 2 GHz

__device__ __forceinline__ void cta_barrier(int id, int nthreads)
{
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}

__device__ __forceinline__ void cta_arrive(int id, int nthreads)
{
    asm volatile("bar.arrive %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}

__device__ __forceinline__ uint32_t smem_addr(const void *p)
{
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint64_t *bar, int count)
{
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_addr(bar)), "r"(count) : "memory");
}

__device__ __forceinline__ void mbar_expect_tx(uint64_t *bar, int bytes)
{
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_addr(bar)), "r"(bytes)
                 : "memory");
}

// One potentially blocking test of the phase: the warp is suspended (not
// spinning, so it takes no issue slots from the warps doing the work) until the
// phase completes or about 0.5 ms pass.
__device__ __forceinline__ bool mbar_try(uint32_t bar, uint32_t parity)
{
    uint32_t done;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2, %3;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(done)
        : "r"(bar), "r"(parity), "r"(500000u)
        : "memory");
    return done != 0;
}

// Wait (bounded) for the completion of the mbarrier phase of the given parity.
// One warp of the CTA polls; the others block on a named barrier it arrives at.
__device__ __forceinline__ bool mbar_wait(uint64_t *bar, uint32_t parity)
{
    const uint32_t a = smem_addr(bar);
    if (mbar_try(a, parity)) return true;
    const long long t0 = clock64();
    for (unsigned i = 1;; ++i) {
        if (mbar_try(a, parity)) return true;
        if ((i & 63) == 0 && clock64() - t0 > kWaitCycles) return false;
    }
}

// group_sum of two values at once (the same order for each as group_sum)
__device__ __forceinline__ void group_sum2(double &v, double &w, int width)
{
#pragma unroll
    for (int off = 16; off > 0; off >>= 1)
        if (off < width) {
            v += __shfl_xor_sync(0xffffffffu, v, off);
            w += __shfl_xor_sync(0xffffffffu, w, off);
        }
}

// The label whose value sits at position i of the exchange buffer (CTA r's Cg
// labels at r*CgE ..., CgE = Cg rounded up to even; with one CTA the labels in
// order), or -1 for a padding position.
__host__ __device__ __forceinline__ int exch_label(int i, int C, int Cg, int G)
{
    if (G <= 1) return i < C ? i : -1;
    const int CgE = (Cg + 1) & ~1;
    const int r = i / CgE, o = i - r * CgE;
    const int lab = r * Cg + o;
    return (o < Cg && r < G && lab < C) ? lab : -1;
}

// Bulk copy of `bytes` (a multiple of 16) from this CTA's shared memory at src to
// the shared::cluster address dst, completing the bytes on the mbarrier at the
// shared::cluster address bar (both 16-byte aligned; no multicast).
__device__ __forceinline__ void bulk_to_peer(uint32_t dst, uint32_t src, uint32_t bytes, uint32_t bar)
{
    asm volatile("cp.async.bulk.shared::cluster.shared::cta.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(dst),
                 "r"(src), "r"(bytes), "r"(bar)
                 : "memory");
}

// st.async of v to the shared::cluster address ra, completing 8 bytes on the
// mbarrier at the shared::cluster address rb.
__device__ __forceinline__ void st_async_at(uint32_t ra, uint32_t rb, double v)
{
    asm volatile("st.async.shared::cluster.mbarrier::complete_tx::bytes.b64 [%0], %1, [%2];" ::"r"(ra),
                 "l"(__double_as_longlong(v)), "r"(rb)
                 : "memory");
}

__device__ __forceinline__ uint32_t mapa_rank(uint32_t local, uint32_t rank)
{
    uint32_t r;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(local), "r"(rank));
    return r;
}

// xor-shuffle sum over groups of `width` consecutive lanes (width a power of two
// <= 32): offsets width/2, ..., 1 in that order, unrolled
__device__ __forceinline__ double group_sum(double v, int width)
{
#pragma unroll
    for (int off = 16; off > 0; off >>= 1)
        if (off < width) v += __shfl_xor_sync(0xffffffffu, v, off);
    return v;
}

// x * 2^h, with the common h = 0 free
__device__ __forceinline__ double rescale(double x, int h) { return h == 0 ? x : scale2c(x, h); }

// Shared memory of both chains (the backward uses the pf_cu/pf_ca/pf_eu/pf_ea rings).
struct ClSmem {
    double *ring;    // [2K][RS] every row twice, with LPW zero rows before and after
    double *Wd;      // [K][RS]  exp(D), when the window lanes do not hold it in registers
    double *gath;    // [2][GP]  a' (forward) or bp (backward) of the position: CTA r's labels at
                     //          positions r*CgE .. r*CgE + Cg - 1 (CgE = Cg rounded up to even), zeros elsewhere
    double *stage;   // [2][CgE] this CTA's values of the position, the source of the bulk copies
    double *qbuf;    // [2][CgE] transition result of each label, for its owner (by step parity)
    double *pub;     // [3][CgE] owner values the transition lanes form the next value from
    double *pre3;    // [4][Cg][PW] window sums two positions ahead
    double *pf_es, *pf_ies, *pf_cu, *pf_ca;   // [kPF][Cg] prefetch rings
    uint64_t *full;  // [2] exchange mbarriers
    int *pf_m, *pf_eu, *pf_ea;                // [kPF][Cg] each
    int *hbuf;       // [4][Cg] rebase exponent of each label at the last four positions
    int *kbuf;       // [4]     normaliser exponents
};

__host__ __device__ __forceinline__ size_t even_up(size_t n) { return (n + 1) & ~(size_t)1; }

// Doubles before the exchange buffers (rounded up to an even count, so that the
// exchange buffers start on a 16-byte boundary, as bulk copies require).
__host__ __device__ __forceinline__ size_t cl_head_doubles(int K, const ClGeom &g)
{
    return even_up(((g.NRB > 0 ? 2 : 3) * (size_t)K + 2 * (size_t)g.PAD) * g.RS);
}

__host__ __device__ __forceinline__ size_t cl_smem_bytes_impl(int K, int C, const ClGeom &g, bool bwd)
{
    const size_t npf = bwd ? 4 : 2;
    const size_t nd = cl_head_doubles(K, g) + 2 * (size_t)g.GP + 2 * even_up(g.Cg) + 5 * even_up(g.Cg) +
                      4 * (size_t)g.Cg * g.PW + npf * kPF * g.Cg;
    const size_t ni = (bwd ? 3 : 1) * (size_t)kPF * g.Cg + 4 * (size_t)g.Cg + 4;
    return nd * sizeof(double) + 2 * sizeof(uint64_t) + ni * sizeof(int);
}

__device__ __forceinline__ ClSmem cl_smem(double *base, int K, int C, const ClGeom &g, bool bwd)
{
    ClSmem s;
    s.ring = base + (size_t)g.PAD * g.RS;
    s.Wd = s.ring + (2 * (size_t)K + g.PAD) * g.RS;
    s.gath = base + cl_head_doubles(K, g);
    s.stage = s.gath + 2 * (size_t)g.GP;
    s.qbuf = s.stage + 2 * even_up(g.Cg);
    s.pub = s.qbuf + 2 * even_up(g.Cg);
    s.pre3 = s.pub + 3 * even_up(g.Cg);
    s.pf_es = s.pre3 + 4 * g.Cg * g.PW;
    s.pf_ies = s.pf_es + kPF * g.Cg;
    s.pf_cu = s.pf_ies + kPF * g.Cg;
    s.pf_ca = bwd ? s.pf_cu + kPF * g.Cg : s.pf_cu;
    double *dend = bwd ? s.pf_ca + kPF * g.Cg : s.pf_cu;
    s.full = reinterpret_cast<uint64_t *>(dend);
    s.pf_m = reinterpret_cast<int *>(s.full + 2);
    s.pf_eu = s.pf_m + kPF * g.Cg;
    s.pf_ea = bwd ? s.pf_eu + kPF * g.Cg : s.pf_eu;
    s.hbuf = bwd ? s.pf_ea + kPF * g.Cg : s.pf_eu;
    s.kbuf = s.hbuf + 4 * g.Cg;
    return s;
}

// sum_i a[i] b[i] as a pairwise tree (products in parallel, log2 N levels of adds):
// with FP64 latency in the tens of cycles, depth matters more than op count.
template <int N>
__device__ __forceinline__ double tree_dot(const double (&x)[N], const double (&y)[N])
{
    static_assert(N >= 2 && (N & (N - 1)) == 0, "N must be a power of two");
    double p[N / 2];
#pragma unroll
    for (int i = 0; i < N / 2; ++i) p[i] = fma(x[2 * i], y[2 * i], x[2 * i + 1] * y[2 * i + 1]);
#pragma unroll
    for (int w = N / 2; w > 1; w >>= 1) {
#pragma unroll
        for (int i = 0; i < w / 2; ++i) p[i] = p[2 * i] + p[2 * i + 1];
    }
    return p[0];
}

// Sum of n rows spaced `step` doubles apart from u (downwards when dir < 0)
// times weights spaced `step` apart from w (upwards), eight rows per chunk: all
// sixteen loads of a chunk issue together, then a product tree.
__device__ __forceinline__ double strided_dot(const double *u, int ustep, const double *w, int wstep, int n)
{
    double acc = 0.0;
#pragma unroll 2
    for (int m0 = 0; m0 < n; m0 += 8) {
        double v[8], x[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const bool ok = m0 + i < n;
            v[i] = ok ? u[(m0 + i) * ustep] : 0.0;
            x[i] = ok ? w[(m0 + i) * wstep] : 0.0;
        }
        acc += tree_dot<8>(v, x);
    }
    return acc;
}

// The lane's window rows m in [m0, n), at ring slots sl0 + m*dsl (dsl = -LPW in
// the forward, +LPW in the backward), times the power of two 2^h in both copies:
// one multiplication when 2^h is a normal double, else scale2c's two factors
// (either way exact unless the result leaves the normal range).  This runs on
// the rebase positions that set the chain's pace, and each row's store waits on
// its multiply: dropping the second multiply cut the large-label step by 4 %.
// Row by row and not unrolled (the loads and stores alias, so unrolling
// overlaps nothing and costs registers the rest of the kernel needs); staging
// rows ahead, a software-pipelined loop and an exponent-field add all measured
// slower on the large-label chains.
__device__ __forceinline__ void rescale_rows(double *ring, int K, int RS, int lc, int sl0, int dsl, int m0, int n,
                                             int h)
{
    if (h >= -1022 && h <= 1023) {   // 2^h is a normal double
        const double s = pow2c(h);
#pragma unroll 1
        for (int m = m0; m < n; ++m) {
            const int sl = sl0 + m * dsl;
            const int other = sl >= K ? sl - K : sl + K;
            const double w = ring[sl * RS + lc] * s;
            ring[sl * RS + lc] = w;
            ring[other * RS + lc] = w;
        }
        return;
    }
    const int h1 = h / 2;
    const double s2a = pow2c(h1), s2b = pow2c(h - h1);
#pragma unroll 1
    for (int m = m0; m < n; ++m) {
        const int sl = sl0 + m * dsl;
        const int other = sl >= K ? sl - K : sl + K;
        const double w = (ring[sl * RS + lc] * s2a) * s2b;
        ring[sl * RS + lc] = w;
        ring[other * RS + lc] = w;
    }
}

// The stored rows of every label that rebased one position earlier, brought to
// its new reference by all the window lanes together (wl of nw): n rows per
// label at ring slots sl0 + i*dsl, both copies, times 2^h as rescale_rows does.
// A rebase is a few positions' burst over all labels of a chain, and on those
// positions the slowest CTA sets the cluster's pace: spread over every window
// lane a label's rows take about two rounds instead of a 32-row loop in its
// own lanes.  Returns whether any label rebased, the same answer in every
// window warp (they read the same exponents), so the barrier after it is
// uniform.
__device__ __forceinline__ bool coop_rescale(double *ring, const int *hrow, int K, int RS, int cg_own, int sl0,
                                             int dsl, int n, int wl, int nw, int lane)
{
    unsigned any = 0;
    for (int l0 = 0; l0 < cg_own; l0 += 32) {
        const int hl = l0 + lane < cg_own ? hrow[l0 + lane] : 0;
        unsigned mask = __ballot_sync(0xffffffffu, hl != 0);
        any |= mask;
        while (mask) {
            const int bit = __ffs(mask) - 1;
            mask &= mask - 1;
            const int h = __shfl_sync(0xffffffffu, hl, bit), l = l0 + bit;
            const bool one = h >= -1022 && h <= 1023;   // 2^h is a normal double
            const int h1 = h / 2;
            const double s = pow2c(h), s2a = pow2c(h1), s2b = pow2c(h - h1);
            for (int i = wl; i < n; i += nw) {
                const int sl = sl0 + i * dsl;
                const int other = sl >= K ? sl - K : sl + K;
                const double v = ring[sl * RS + l];
                const double w = one ? v * s : (v * s2a) * s2b;
                ring[sl * RS + l] = w;
                ring[other * RS + l] = w;
            }
        }
    }
    return any != 0;
}

// Forward window: sum over d = d0 + m*LPW <= K (d0 = 3 + j) of ring row (tau - d)
// times exp(D[d-1]) for label lc, with tau mod K = tauK.  Rows with d >= 4 are
// first brought to the reference of position tau - 3 (multiplied by 2^hp, both
// copies); row tau - 3 (d = 3) was written at that reference.
__device__ __forceinline__ double window_fwd(double *ring, const double *Wd, int K, int RS, int lc, int LPW, int j,
                                             int tauK, int hp)
{
    const int d0 = 3 + j;
    if (d0 > K) return 0.0;
    const int n = (K - d0) / LPW + 1;
    const int step = LPW * RS;
    if (hp != 0) rescale_rows(ring, K, RS, lc, tauK + K - d0, -LPW, d0 < 4 ? 1 : 0, n, hp);   // rows d >= 4
    // the copy whose slots fall in [0, 2K): rows tau - d at slot tauK + K - d
    return strided_dot(ring + (size_t)(tauK + K - d0) * RS + lc, -step, Wd + (size_t)(d0 - 1) * RS + lc, step, n);
}

// Backward window: sum over i = i0 + m*LPW <= K-2 (i0 = 1 + j) of ring row (s + i)
// times exp(D[i+1]) (position s-2, duration i+2), s mod K = sK.  Rows with i >= 2
// are first brought to the reference of position s+1 (multiplied by 2^hp).
__device__ __forceinline__ double window_bwd(double *ring, const double *Wd, int K, int RS, int lc, int LPW, int j,
                                             int sK, int hp)
{
    const int i0 = 1 + j;
    if (i0 > K - 2) return 0.0;
    const int n = (K - 2 - i0) / LPW + 1;
    const int step = LPW * RS;
    if (hp != 0) rescale_rows(ring, K, RS, lc, sK + i0, LPW, i0 < 2 ? 1 : 0, n, hp);   // rows i >= 2
    return strided_dot(ring + (size_t)(sK + i0) * RS + lc, step, Wd + (size_t)(i0 + 1) * RS + lc, step, n);
}

// A zero the compiler cannot see through, computed from v: adding it to an
// address makes the loads from that address wait for v.
__device__ __forceinline__ int opaque_zero(double v)
{
    int z;
    asm("and.b32 %0, %1, 0;" : "=r"(z) : "r"((int)__double_as_longlong(v)));
    return z;
}

// The same window sums with the lane's weights in registers (W[m] for row m of
// the lane, 0 past the last duration) and no per-row bounds: NR rows per lane
// (a bucket >= the rows the lane has), the rows beyond the window read the
// ring's zero padding or older finite rows, times weight 0.  Four interleaved
// partial sums.
template <int NR, int NU>
__device__ __forceinline__ double window_fwd_reg(double *ring, int K, int RS, int lc, int LPW, int j, int tauK,
                                                 int hp, const double (&W)[NU])
{
    static_assert(NR <= NU, "window rows exceed the register array");
    const int d0 = 3 + j;
    // a rebase at tau - 3 (every label rebases about every 500 bits of growth of
    // its column, and the labels of a chain within a few positions of each
    // other): the lane's rows d >= 4 of the window
    if (hp != 0 && d0 <= K) rescale_rows(ring, K, RS, lc, tauK + K - d0, -LPW, d0 < 4 ? 1 : 0, (K - d0) / LPW + 1, hp);
    const double *p = ring + (tauK + K - d0) * RS + lc;
    const int step = LPW * RS;
    double acc[8] = {0.0, 0.0, 0.0, 0.0, 0.0, 0.0, 0.0, 0.0};
    // eight rows at a time, each chunk's loads after the previous chunk's products:
    // at most eight loads of a lane in the shared-memory queue, so the chain's own
    // loads (the owners' q) do not wait behind a whole window pass
#pragma unroll
    for (int m0 = 0; m0 < NR; m0 += 8) {
        double v[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) v[i] = p[-(m0 + i) * step];
#pragma unroll
        for (int i = 0; i < 8; ++i) acc[i] = fma(v[i], W[m0 + i], acc[i]);
        if (m0 + 8 < NR) p += opaque_zero(acc[7]);
    }
    return ((acc[0] + acc[1]) + (acc[2] + acc[3])) + ((acc[4] + acc[5]) + (acc[6] + acc[7]));
}

template <int NR, int NU>
__device__ __forceinline__ double window_bwd_reg(double *ring, int K, int RS, int lc, int LPW, int j, int sK, int hp,
                                                 const double (&W)[NU])
{
    static_assert(NR <= NU, "window rows exceed the register array");
    const int i0 = 1 + j;
    if (hp != 0 && i0 <= K - 2)   // as in the forward: rows i >= 2
        rescale_rows(ring, K, RS, lc, sK + i0, LPW, i0 < 2 ? 1 : 0, (K - 2 - i0) / LPW + 1, hp);
    const double *p = ring + (sK + i0) * RS + lc;
    const int step = LPW * RS;
    double acc[8] = {0.0, 0.0, 0.0, 0.0, 0.0, 0.0, 0.0, 0.0};
#pragma unroll
    for (int m0 = 0; m0 < NR; m0 += 8) {   // eight rows at a time (as forward)
        double v[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) v[i] = p[(m0 + i) * step];
#pragma unroll
        for (int i = 0; i < 8; ++i) acc[i] = fma(v[i], W[m0 + i], acc[i]);
        if (m0 + 8 < NR) p += opaque_zero(acc[7]);
    }
    return ((acc[0] + acc[1]) + (acc[2] + acc[3])) + ((acc[4] + acc[5]) + (acc[6] + acc[7]));
}

// Window sum with the row count of the plan's bucket (8, 16 or 32 rows per lane).
template <int NU>
__device__ __forceinline__ double window_fwd_nr(int NRB, double *ring, int K, int RS, int lc, int LPW, int j,
                                                int tauK, int hp, const double (&W)[NU])
{
    if constexpr (NU >= 32)
        if (NRB == 32) return window_fwd_reg<32, NU>(ring, K, RS, lc, LPW, j, tauK, hp, W);
    if (NRB == 16) return window_fwd_reg<16, NU>(ring, K, RS, lc, LPW, j, tauK, hp, W);
    return window_fwd_reg<8, NU>(ring, K, RS, lc, LPW, j, tauK, hp, W);
}

template <int NU>
__device__ __forceinline__ double window_bwd_nr(int NRB, double *ring, int K, int RS, int lc, int LPW, int j, int sK,
                                                int hp, const double (&W)[NU])
{
    if constexpr (NU >= 32)
        if (NRB == 32) return window_bwd_reg<32, NU>(ring, K, RS, lc, LPW, j, sK, hp, W);
    if (NRB == 16) return window_bwd_reg<16, NU>(ring, K, RS, lc, LPW, j, sK, hp, W);
    return window_bwd_reg<8, NU>(ring, K, RS, lc, LPW, j, sK, hp, W);
}

// Pairwise sum of N values (N a power of two).
template <int N>
__device__ __forceinline__ double tree_sum(const double (&x)[N])
{
    double p[N];
#pragma unroll
    for (int i = 0; i < N; ++i) p[i] = x[i];
#pragma unroll
    for (int w = N; w > 1; w >>= 1) {
#pragma unroll
        for (int i = 0; i < w / 2; ++i) p[i] = p[2 * i] + p[2 * i + 1];
    }
    return p[0];
}

// sum_m v[m] E[m] with v[m] = gp[m * stride], and the plain sum of the v[m]
// into *vsum: chunks of eight (loads, a product tree, a sum tree) combined
// pairwise, so that at most a chunk of loaded values is live.
template <int N>
__device__ __forceinline__ double chunked_dot(const double *gp, int stride, const double (&E)[N], double *vsum)
{
    if constexpr (N <= 8) {
        double v[N];
#pragma unroll
        for (int m = 0; m < N; ++m) v[m] = gp[m * stride];
        *vsum = tree_sum<N>(v);
        return tree_dot<N>(v, E);
    } else {
        double part[N / 8], sums[N / 8];
#pragma unroll
        for (int c8 = 0; c8 < N / 8; ++c8) {
            double v[8];
            const double(&e8)[8] = *reinterpret_cast<const double(*)[8]>(&E[c8 * 8]);
#pragma unroll
            for (int i = 0; i < 8; ++i) v[i] = gp[(c8 * 8 + i) * stride];
            part[c8] = tree_dot<8>(v, e8);
            sums[c8] = tree_sum<8>(v);
        }
        *vsum = tree_sum<N / 8>(sums);
        return tree_sum<N / 8>(part);
    }
}

// Roles of a thread: owner warps (label lc = lane of the warp's 32), then
// transition warps (LPL lanes per label), then window warps (LPW lanes per label).
struct Roles {
    bool is_own, is_tr, is_win, lab_ok;
    int lc, j, c;
};

__device__ __forceinline__ Roles cl_roles(const ClGeom &g, int warp, int lane, int c0l, int cg_own)
{
    Roles r;
    r.is_own = warp < g.NWO;
    r.is_tr = !r.is_own && warp < g.NWO + g.NWT;
    r.is_win = !r.is_own && !r.is_tr && warp < g.NWO + g.NWT + g.NWW;
    r.lc = 0;
    r.j = 0;
    if (r.is_own) {
        r.lc = warp * 32 + lane;
    } else if (r.is_tr) {
        const int tl = (warp - g.NWO) * 32 + lane;
        r.lc = tl / g.LPL;
        r.j = tl % g.LPL;
    } else if (r.is_win) {
        const int wl = (warp - g.NWO - g.NWT) * 32 + lane;
        r.lc = wl / g.LPW;
        r.j = wl % g.LPW;
    }
    r.lab_ok = (r.is_own || r.is_tr || r.is_win) && r.lc < cg_own;
    r.c = c0l + (r.lab_ok ? r.lc : 0);
    return r;
}

// Wait of owner warp 0 for the C values of a position: the mbarrier of the
// cluster exchange (with one CTA the owners' plain stores are already ordered by
// the barriers around this call).  Warp 0 then releases the transition warps
// through named barrier 5, so only one warp polls.
template <bool CLUSTER>
__device__ __forceinline__ bool wait_values(ClSmem &sm, int par, int u, bool skip)
{
    if constexpr (CLUSTER) {
        if (skip) return true;
        return mbar_wait(&sm.full[par], (u >> 1) & 1);
    } else {
        return true;
    }
}

// MODE 0: forward with checkpoints and log Z.  MODE 1: recompute one checkpoint
// segment, writing the per-position rows relative to Z.  MODE 2: the whole
// sequence once, log Z and the rows unscaled (scaled later by exp(-log Z)),
// no checkpoints.  cid: the cluster's index among those running this body.
template <int CPL, int MAXT, bool CLUSTER, int MODE, bool TS>
__device__ __forceinline__ void cl_fwd_body(const FbArgs &a, const ClGeom &g, int cid)
{
    constexpr bool RECOMPUTE = MODE == 1;
    constexpr bool ROWS = MODE != 0;
    constexpr bool CKPT = MODE == 0;
    extern __shared__ __align__(16) double smc[];
    const int K = a.K, C = a.C, Cg = g.Cg, NT = g.NT, RS = g.RS, PW = g.PW;
    const int NOT = 32 * (g.NWO + g.NWT);   // owner + transition threads
    const int NOW = 32 * (g.NWO + g.NWW);   // owner + window threads
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int rank = CLUSTER ? (int)cluster_rank() : 0;
    int b, seg;
    if constexpr (RECOMPUTE) {
        b = cid / a.J;
        seg = cid % a.J;
    } else {
        b = cid;
        seg = 0;
    }
    const int L = a.lengths[b];
    if (L < 1 || L > a.T) {
        if (rank == 0 && tid == 0 && seg == 0) set_status(a.status, SEMICRF_ERR_INVALID_LENGTH);
        return;
    }
    const int t0 = seg * a.delta;
    if (RECOMPUTE && t0 >= L) return;
    const int t_end = RECOMPUTE ? min(t0 + a.delta, L) : L;
    const int c0l = rank * Cg, cg_own = min(Cg, C - c0l);
    ClSmem sm = cl_smem(smc, K, C, g, false);
    const size_t rowbase = (size_t)b * (a.T + 1);
    unsigned char *ck_base = a.ckpt + ((size_t)b * a.J) * a.ckpt_stride;
    int kZ = 0;
    double cz = MODE == 2 ? 1.0 : 0.0;
    if constexpr (RECOMPUTE) {
        kZ = a.lz[b].k;
        cz = exp(-a.lz[b].logn);
    }
    const Roles ro = cl_roles(g, warp, lane, c0l, cg_own);
    const int lc = ro.lc, j = ro.j, c = ro.c;
    const bool own = ro.is_own && ro.lab_ok;

    // ------------------------------------------------------------------ init
    {
        const unsigned char *ck = ck_base + (size_t)seg * a.ckpt_stride;
        const double *ck_ring = reinterpret_cast<const double *>(ck);
        double *ck_ring_w = reinterpret_cast<double *>(ck_base);
        for (int i = tid; i < K * Cg; i += NT) {
            const int sl = i / Cg, l2 = i % Cg;
            const bool ok = l2 < cg_own;
            if (g.NRB == 0) sm.Wd[sl * RS + l2] = ok ? exp((double)a.D[(size_t)sl * C + c0l + l2]) : 0.0;
            double v;
            if constexpr (RECOMPUTE) {
                v = ok ? ck_ring[(size_t)sl * C + c0l + l2] : 0.0;
            } else {
                v = (ok && sl == 0) ? 1.0 : 0.0;   // row 0 = exp(0), rows < 0 empty
                if (ok) ck_ring_w[(size_t)sl * C + c0l + l2] = v;   // checkpoint 0
            }
            sm.ring[sl * RS + l2] = v;
            sm.ring[(sl + K) * RS + l2] = v;
        }
        for (int i = tid; i < g.PAD * RS; i += NT) {   // the zero rows around the ring
            sm.ring[i - g.PAD * RS] = 0.0;
            sm.ring[2 * K * RS + i] = 0.0;
        }
        for (int i = tid; i < 2 * g.GP; i += NT) sm.gath[i] = 0.0;
        for (int i = tid; i < 2 * (int)even_up(Cg); i += NT) sm.stage[i] = 0.0;
        for (int i = tid; i < 4 * Cg * PW; i += NT) sm.pre3[i] = 0.0;
        for (int i = tid; i < 4 * Cg; i += NT) sm.hbuf[i] = 0;
        if (tid == 0) {
            if constexpr (RECOMPUTE) {
                const int32_t *ck_r = reinterpret_cast<const int32_t *>(ck_ring + (size_t)K * C);
                sm.kbuf[0] = ck_r[C];       // k_{t0+1}
                sm.kbuf[1] = ck_r[C + 1];   // k_{t0+2}
            } else {
                sm.kbuf[0] = 0;
                sm.kbuf[1] = 0;
                int32_t *ck_r = reinterpret_cast<int32_t *>(ck_ring_w + (size_t)K * C);
                if (rank == 0) {
                    ck_r[C] = 0;
                    ck_r[C + 1] = 0;
                }
            }
            if constexpr (CLUSTER) {
                mbar_init(&sm.full[0], 1);
                mbar_init(&sm.full[1], 1);
                asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
            }
        }
        if (!RECOMPUTE && tid < cg_own) {
            int32_t *ck_r = reinterpret_cast<int32_t *>(ck_ring_w + (size_t)K * C);
            ck_r[c0l + tid] = 0;
        }
    }
    __syncthreads();
    // One register array holds the transition weights E (transition lanes), the
    // window weights exp(D) of the lane's rows (window lanes, when they fit) or
    // the chain state (owner lanes): a thread has one role, and sharing keeps
    // the register count of the kernel that of the largest of the three.
    // Chain state at the start of step t: U1 = U[t-1], U2 = U[t-2] (reference of
    // t-1) and the values prepared for t from everything but U[t-1]:
    //   pre = U[t-2] W1 + pre3_t,  e = exp(S_t + ln2 (r - k_t)),  f = exp(ln2 (k_t - r) - S_t),
    //   pe = pre e,  w0e = W0 e,  so a'[t] = U[t-1] w0e + pe is one FMA after U[t-1].
    constexpr int NU = CPL > 16 ? CPL : 16;
    const int nrw = K > 2 ? (K - 2 + g.LPW - 1) / g.LPW : 0;   // window rows per lane
    const bool wreg = g.NRB > 0;
    double R[NU];
#pragma unroll
    for (int m = 0; m < NU; ++m) {
        const int cp = j + m * g.LPL;
        double v = 0.0;
        const int lp = exch_label(cp, C, Cg, g.G);   // the label at exchange position cp, or -1
        if (m < CPL && ro.is_tr && ro.lab_ok && lp >= 0) v = exp((double)a.A[(size_t)lp * C + c]);
        const int d = 3 + j + m * g.LPW;   // window lanes: duration of row m
        if (ro.is_win && wreg && ro.lab_ok && m < nrw && d <= K) v = exp((double)a.D[(size_t)(d - 1) * C + c]);
        R[m] = v;
    }
    // window sums for the first two positions, from the restored ring (one reference)
    if (ro.is_win) {
        for (int q = 1; q <= 2; ++q) {
            const int tau = t0 + q;
            double v = 0.0;
            if (ro.lab_ok)
                v = wreg ? window_fwd_nr<NU>(g.NRB, sm.ring, K, RS, lc, g.LPW, j, tau % K, 0, R)
                         : window_fwd(sm.ring, sm.Wd, K, RS, lc, g.LPW, j, tau % K, 0);
            const double s = group_sum(v, g.LPW < 32 ? g.LPW : 32);
            if (ro.lab_ok && (j & 31) == 0) sm.pre3[(q - 1) * Cg * PW + lc * PW + (j >> 5)] = s;
        }
    }
    // The exchange: each CTA's block of values (its labels, padded with zeros to an
    // even count CgE, so 16-byte units) goes to every CTA of the cluster by one bulk
    // copy per destination, into position rank*CgE of the destination's exchange
    // buffer, completing on its mbarrier.
    const int CgE = (int)even_up(Cg);
    // The copies are issued from up to four warps, one per scheduler: issuing to
    // many CTAs from one warp serialises (~70 cycles per destination, measured).
    // With TS the first four transition warps, else the owner warps first, then
    // transition warps; issuing warp w lane l sends to CTA w + nwi*l.
    constexpr bool ts = CLUSTER && TS;
    const int iw0 = ts ? g.NWO : 0;
    const int nwi = ts ? (g.NWT < 4 ? g.NWT : 4) : (g.NWO + g.NWT < 4 ? g.NWO + g.NWT : 4);
    const int dst_rank = (warp - iw0) + nwi * lane;
    const bool issuer = CLUSTER && warp >= iw0 && warp < iw0 + nwi && dst_rank < g.G;
    const uint32_t bdst = issuer ? mapa_rank(smem_addr(&sm.gath[rank * CgE]), (uint32_t)dst_rank) : 0u;
    const uint32_t bbar = issuer ? mapa_rank(smem_addr(&sm.full[0]), (uint32_t)dst_rank) : 0u;
    // TS: a label's value goes from its own lanes to every CTA by st.async
    const uint32_t xg = smem_addr(&sm.gath[rank * CgE + (ro.lab_ok ? lc : 0)]), xb = smem_addr(&sm.full[0]);
    double(&E)[CPL] = *reinterpret_cast<double(*)[CPL]>(&R[0]);
    double &W0 = R[0], &W1 = R[1], &U1 = R[2], &U2 = R[3], &pre = R[4], &f = R[5], &pe = R[6], &w0e = R[7],
           &ap = R[8];
    double f_n = 0.0;
    int r = 0, h1 = 0, h2 = 0, kt = 0, kt_n = 0;
    auto prefetch = [&](int tp) {
        if (tp <= t_end) {
            const size_t ix = (rowbase + tp) * C + c;
            const int sl = tp & (kPF - 1);
            cp_async8(&sm.pf_es[sl * Cg + lc], a.tES + ix);
            cp_async8(&sm.pf_ies[sl * Cg + lc], a.tIES + ix);
            cp_async4(&sm.pf_m[sl * Cg + lc], a.tM + ix);
        }
        cp_async_commit();
    };
    // values for position tn (step un) from row d2 = U[tn-2] at the current reference
    auto prepare = [&](int tn, int un, double d2, double &pre_o, double &f_o, double &pe_o, double &w0e_o,
                       int &kt_o) {
        const int sl = tn & (kPF - 1);
        const double es = sm.pf_es[sl * Cg + lc], ies = sm.pf_ies[sl * Cg + lc];
        const int m = sm.pf_m[sl * Cg + lc];
        kt_o = sm.kbuf[un & 3];
        double p3 = 0.0;
        for (int q = 0; q < PW; ++q) p3 += sm.pre3[(un & 3) * Cg * PW + lc * PW + q];
        pre_o = fma(d2, W1, rescale(p3, h1 + h2));
        const double e = es * pow2c(m + r - kt_o);   // exp(S + ln2 (r - k))
        f_o = ies * pow2c(kt_o - r - m);             // exp(ln2 (k - r) - S)
        pe_o = pre_o * e;
        w0e_o = W0 * e;
    };
    if (own) {
        W0 = exp((double)a.D[c]);
        W1 = K >= 2 ? exp((double)a.D[C + c]) : 0.0;
        U1 = sm.ring[(t0 % K) * RS + lc];
        U2 = K >= 2 ? sm.ring[(((t0 - 1) % K + K) % K) * RS + lc] : 0.0;
        if constexpr (RECOMPUTE) {
            const int32_t *ck_r = reinterpret_cast<const int32_t *>(
                reinterpret_cast<const double *>(ck_base + (size_t)seg * a.ckpt_stride) + (size_t)K * C);
            r = ck_r[c];
        }
        for (int i = 1; i < kPF; ++i) prefetch(t0 + i);
    }
    __syncthreads();   // look-ahead sums written
    if (own) {
        cp_async_wait<kPF - 2>();   // position t0+1 has landed
        prepare(t0 + 1, 0, U2, pre, f, pe, w0e, kt);
    }
    if constexpr (CLUSTER) cluster_barrier();   // mbarriers of every CTA initialised
    else __syncthreads();
    if (ts) {
        // a'[t0+1] from the owners; from then on the transition lanes form each
        // position's value from the previous q and send it
        if (own) {
            const double a0 = fma(U1, w0e, pe);
            for (int dr = 0; dr < g.G; ++dr) st_async_at(mapa_rank(xg, dr), mapa_rank(xb, dr), a0);
        }
    }

    int tK = (t0 + 1) % K;
    int td = (t0 + 1) % a.delta;
    bool timed_out = false;
    for (int t = t0 + 1; t <= t_end; ++t) {
        const int u = t - t0 - 1;   // step count
        const int par = u & 1;
        if (ro.is_own) {
            // ------------------------------------------------ owners: chain
            // a'[t] (with TS the transition lanes formed and sent the same value)
            if (own) ap = fma(U1, w0e, pe);
            if constexpr (CLUSTER) {
                if (!ts) {
                    // the owners' values into the stage, visible to the copy engine, then
                    // one bulk copy per destination CTA
                    if (own) sm.stage[par * CgE + lc] = ap;
                    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
                    cta_barrier(5, NOT);   // the stage is written, for the issuing warps
                    if (issuer)
                        bulk_to_peer(bdst + par * g.GP * 8, smem_addr(sm.stage + par * CgE), (uint32_t)(CgE * 8),
                                     bbar + par * 8);
                }
            } else if (own) {
                sm.gath[par * g.GP + c] = ap;
            }
            if (own) {
                // rebase when p = a' / e leaves [2^-512, 2^512]
                const double p = fma(U1, W0, pre);
                const int ex = exponent_of(p);
                const int h = (ex > kRebaseBits || ex < -kRebaseBits) ? -ex : 0;
                if (h != 0) {
                    const double s2 = pow2(h);
                    r -= h;
                    f *= s2;
                    U1 *= s2;
                }
                sm.hbuf[(u & 3) * Cg + lc] = h;
                h2 = h1;
                h1 = h;
            }
            if (u >= 1 && t < t_end) cta_barrier(kBarWin + ((u - 1) & 1), NOW);   // window sums of step u-1
            if (own) {
                // prepare position t+1 (row t-1 = U1 is its d = 2 row); this step's
                // prefetch is issued after the new row, off the owners' path to it
                cp_async_wait<kPF - 3>();  // position t+1 has landed
                if (t < t_end) prepare(t + 1, u + 1, U1, pre, f_n, pe, w0e, kt_n);
            }
            if (ts) {
                // f_t (after this step's rebase) and W0 e, pre e of t+1: a'[t+1] =
                // (q_t f_t) (W0 e) + pre e is then formed where q_t is summed
                if (own && t < t_end) {
                    sm.pub[lc] = f;
                    sm.pub[CgE + lc] = w0e;
                    sm.pub[2 * CgE + lc] = pe;
                }
                cta_arrive(kBarPub, NOT);
            } else if constexpr (!CLUSTER) {
                cta_arrive(1, NOT);   // a'[t] stored (for the transition warps)
                if (g.NWO > 1) cta_barrier(7, 32 * g.NWO);
                else __syncwarp();
            }
            cta_barrier(4, NOT);   // q[t] ready
            // ------------------------------------------------ owners: new row
            if (own) {
                const size_t row = (rowbase + t) * C + c;
                if (t < L) {
                    const double U = sm.qbuf[par * CgE + lc] * f;
                    sm.ring[tK * RS + lc] = U;
                    sm.ring[(tK + K) * RS + lc] = U;
                    U2 = U1;
                    U1 = U;
                    if constexpr (ROWS) {
                        a.cU[row] = U * cz;
                        a.cA[row] = ap * cz;
                        a.eU[row] = r - kZ;
                    }
                } else if constexpr (ROWS) {
                    a.cA[row] = ap * cz;
                }
                if (ROWS && c == 0) a.eA[rowbase + t] = kt - kZ;
                f = f_n;
                kt = kt_n;
                prefetch(t + kPF - 1);   // into the slot position t-1 used
            }
            if (t < t_end) cta_arrive(kBarRow + (u & 1), NOW);   // row t and h_t stored, for the window
        } else if (ro.is_tr) {
            // -------------------------------------------------------- transition
            if constexpr (CLUSTER) {
                // this position's exchange: every CTA's block, G*CgE doubles (the
                // barrier's phase for position t-2 completed at this warp's last wait)
                if (tid == 32 * g.NWO) mbar_expect_tx(&sm.full[par], ts ? C * 8 : g.G * (int)even_up(Cg) * 8);
                if (!ts) {
                    cta_barrier(5, NOT);   // the owners' stage is written
                    if (issuer)
                        bulk_to_peer(bdst + par * g.GP * 8, smem_addr(sm.stage + par * CgE), (uint32_t)(CgE * 8),
                                     bbar + par * 8);
                }
                if (!wait_values<CLUSTER>(sm, par, u, timed_out)) {
                    timed_out = true;
                    set_status(a.status, SEMICRF_ERR_DEVICE_TIMEOUT);
                }
            } else {
                cta_barrier(1, NOT);
            }
            const double *gp = sm.gath + par * g.GP + j;   // zeros past C
            // q, and the normaliser n_t = sum_c a'[t,c] from the values the lanes loaded
            // (the same order in every CTA); n is needed two positions later
            double n;
            double q = chunked_dot<CPL>(gp, g.LPL, E, &n);
            group_sum2(q, n, g.LPL);
            if (ts) {
                cta_barrier(kBarPub, NOT);   // the owners' values of this step
                if (t < t_end && ro.lab_ok) {
                    // a'[t+1], the owners' own FMA one step early, from every lane of the
                    // label; lane j stores it into CTAs j, j + LPL, ... (st.async, completing
                    // 8 bytes on that CTA's mbarrier for the position)
                    const double an = fma(q * sm.pub[lc], sm.pub[CgE + lc], sm.pub[2 * CgE + lc]);
                    const uint32_t og = xg + (uint32_t)((par ^ 1) * g.GP * 8), ob = xb + (uint32_t)((par ^ 1) * 8);
                    for (int dr = j; dr < g.G; dr += g.LPL) st_async_at(mapa_rank(og, dr), mapa_rank(ob, dr), an);
                }
            }
            if (ro.lab_ok && j == 0) sm.qbuf[par * CgE + lc] = q;
            // k_{t+2} must reach the owners before they prepare t+2: a cluster without
            // TS orders it by the next step's bar 5, otherwise it is stored before
            // this arrival (the owners only arrive at bar 1)
            const bool k_late = CLUSTER && !ts;
            if (k_late) cta_arrive(4, NOT);
            if (lc == 0 && j == 0) {
                const int kk = sm.kbuf[u & 3];
                if (t == L) {
                    if (!RECOMPUTE && rank == 0) {
                        const double lz = kLn2 * (double)kk + log(n);
                        a.logZ[b] = lz;
                        a.lz[b].logn = log(n);
                        a.lz[b].k = kk;
                        if (!isfinite(lz)) set_status(a.status, SEMICRF_ERR_DEVICE_RANGE);
                    }
                } else {
                    sm.kbuf[(u + 2) & 3] = kk + exponent_of(n);
                }
            }
            if (!k_late) cta_arrive(4, NOT);   // q_t and k_{t+2} stored, for the owners
        } else if (ro.is_win) {
            // ------------------------------------- window sums two positions ahead
            // They run a position ahead of the owners at most: row t-1 and h_{t-1}
            // come from the owners' step u-1, the sums go to their step u+1.
            if (u >= 1) cta_barrier(kBarRow + ((u - 1) & 1), NOW);
            const int tau2K = tK + 2 >= K ? tK + 2 - K : tK + 2;   // K >= 3 whenever a row is read
            // rebases at t-1: rows d = 4..K of those labels (row d = 3 was written after
            // it), by all window lanes together on TS plans (many labels per CTA, few
            // lanes each), else by each label's own lanes inside its window sum
            int hp = ro.lab_ok ? sm.hbuf[((u - 1) & 3) * Cg + lc] : 0;
            if constexpr (ts) {
                const int wl = tid - 32 * (g.NWO + g.NWT), nw = 32 * g.NWW;   // window lane index
                if (coop_rescale(sm.ring, sm.hbuf + ((u - 1) & 3) * Cg, K, RS, cg_own, tau2K + K - 4, -1, K - 3, wl,
                                 nw, lane))
                    cta_barrier(kBarResc, nw);
                hp = 0;   // the rows are at the new reference
            }
            double v = 0.0;
            if (ro.lab_ok)
                v = wreg ? window_fwd_nr<NU>(g.NRB, sm.ring, K, RS, lc, g.LPW, j, tau2K, hp, R)
                         : window_fwd(sm.ring, sm.Wd, K, RS, lc, g.LPW, j, tau2K, hp);
            const double s = group_sum(v, g.LPW < 32 ? g.LPW : 32);
            if (ro.lab_ok && (j & 31) == 0) sm.pre3[((u + 2) & 3) * Cg * PW + lc * PW + (j >> 5)] = s;
            if (t + 1 < t_end) cta_arrive(kBarWin + (u & 1), NOW);
        }
        if (CKPT && td == 0 && t < L) {
            cta_barrier(2, NT);   // every role is through step u
            // checkpoint t / delta: the ring at the reference of position t, r, k_{t+1}, k_{t+2}.
            // Row age 0 (row t) is there; ages 1..K-2 are at the reference of t-1; the
            // oldest row (age K-1, K >= 3) at that of t-2.
            unsigned char *ck = ck_base + (size_t)(t / a.delta) * a.ckpt_stride;
            double *ck_ring = reinterpret_cast<double *>(ck);
            int32_t *ck_r = reinterpret_cast<int32_t *>(ck_ring + (size_t)K * C);
            for (int i = tid; i < K * Cg; i += NT) {
                const int sl = i / Cg, l2 = i % Cg;
                if (l2 < cg_own) {
                    int age = tK - sl;
                    if (age < 0) age += K;
                    int hh = 0;
                    if (age >= 1) hh = sm.hbuf[(u & 3) * Cg + l2];
                    if (age == K - 1 && K >= 3) hh += sm.hbuf[((u - 1) & 3) * Cg + l2];
                    ck_ring[(size_t)sl * C + c0l + l2] = rescale(sm.ring[sl * RS + l2], hh);
                }
            }
            if (own) ck_r[c] = r;
            if (rank == 0 && tid == 0) {
                ck_r[C] = sm.kbuf[(u + 1) & 3];
                ck_r[C + 1] = sm.kbuf[(u + 2) & 3];
            }
            cta_barrier(3, NT);
        }
        tK = (tK + 1 == K) ? 0 : tK + 1;
        td = (td + 1 == a.delta) ? 0 : td + 1;
    }
    if constexpr (CLUSTER) cluster_barrier();   // no CTA leaves while peers may still store to it
}

template <int CPL, int MAXT, bool CLUSTER, bool RECOMPUTE, bool TS>
__global__ void __launch_bounds__(MAXT, 1) cl_fwd_kernel(FbArgs a, ClGeom g)
{
    cl_fwd_body<CPL, MAXT, CLUSTER, RECOMPUTE ? 1 : 0, TS>(a, g, blockIdx.x / g.G);
}

// CHAIN = false: beta chain with the coverage marginal and dX on the chain, from
// the recomputed forward rows.  CHAIN = true: the beta chain alone (it needs
// nothing from the forward, so it can run beside it); the coverage is formed
// later from the stored rows.  b: the sequence.
template <int CPL, int MAXT, bool CLUSTER, bool CHAIN, bool TS>
__device__ __forceinline__ void cl_bwd_body(const FbArgs &a, const ClGeom &g, int b)
{
    extern __shared__ __align__(16) double smc[];
    const int K = a.K, C = a.C, Cg = g.Cg, NT = g.NT, RS = g.RS, PW = g.PW;
    const int NOT = 32 * (g.NWO + g.NWT);
    const int NOW = 32 * (g.NWO + g.NWW);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int rank = CLUSTER ? (int)cluster_rank() : 0;
    const int L = a.lengths[b];
    if (L < 1 || L > a.T) {
        if (rank == 0 && tid == 0) set_status(a.status, SEMICRF_ERR_INVALID_LENGTH);
        return;
    }
    const int c0l = rank * Cg, cg_own = min(Cg, C - c0l);
    ClSmem sm = cl_smem(smc, K, C, g, true);
    const size_t rowbase = (size_t)b * (a.T + 1);
    const int kZ = CHAIN ? 0 : a.lz[b].k;   // the chain-only variant runs beside the forward
    const double cz = CHAIN ? 0.0 : exp(-a.lz[b].logn);
    const Roles ro = cl_roles(g, warp, lane, c0l, cg_own);
    const int lc = ro.lc, j = ro.j, c = ro.c;
    const bool own = ro.is_own && ro.lab_ok;

    // ------------------------------------------------------------------ init
    // row L: be = 0, so V[L,c] = exp(S[L,c] - ln2 rb) = es with rb = m; rows > L empty
    for (int i = tid; i < K * Cg; i += NT) {
        const int sl = i / Cg, l2 = i % Cg;
        const bool ok = l2 < cg_own;
        if (g.NRB == 0) sm.Wd[sl * RS + l2] = ok ? exp((double)a.D[(size_t)sl * C + c0l + l2]) : 0.0;
        const size_t ixL = (rowbase + L) * C + c0l + l2;
        const double v = (ok && sl == L % K) ? a.tES[ixL] : 0.0;
        sm.ring[sl * RS + l2] = v;
        sm.ring[(sl + K) * RS + l2] = v;
    }
    for (int i = tid; i < g.PAD * RS; i += NT) {   // the zero rows around the ring
        sm.ring[i - g.PAD * RS] = 0.0;
        sm.ring[2 * K * RS + i] = 0.0;
    }
    for (int i = tid; i < 2 * g.GP; i += NT) sm.gath[i] = 0.0;
    for (int i = tid; i < 2 * (int)even_up(Cg); i += NT) sm.stage[i] = 0.0;
    for (int i = tid; i < 4 * Cg * PW; i += NT) sm.pre3[i] = 0.0;   // positions L-1, L-2: no rows beyond L
    for (int i = tid; i < 4 * Cg; i += NT) sm.hbuf[i] = 0;
    if (tid == 0) {
        sm.kbuf[0] = 0;
        sm.kbuf[1] = 0;
        if constexpr (CLUSTER) {
            mbar_init(&sm.full[0], 1);
            mbar_init(&sm.full[1], 1);
            asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        }
    }
    // One register array holds the transposed transition weights Er (transition
    // lanes), the window weights exp(D) of the lane's rows (window lanes, when
    // they fit) or the chain state (owner lanes).
    // Chain state at the start of step s: V1 = V[s+1], V2 = V[s+2] (reference of
    // s+1) and, prepared from everything but V[s+1]:
    //   pre = V[s+2] W1 + pre3_s, eb = exp(ln2 (rb - kb) - S_s), gg = exp(S_s + ln2 (kb - rb)),
    //   pbe = pre eb, w0e = W0 eb, so bp[s] = V[s+1] w0e + pbe is one FMA after V[s+1];
    //   coef = X[s] (start factor at the reference rb), a2 (transition factor).
    constexpr int NU = CPL > 16 ? CPL : 16;
    const int nrw = K > 2 ? (K - 2 + g.LPW - 1) / g.LPW : 0;   // window rows per lane
    const bool wreg = g.NRB > 0;
    double R[NU];
#pragma unroll
    for (int m = 0; m < NU; ++m) {
        const int cc = j + m * g.LPL;
        double v = 0.0;
        const int lp = exch_label(cc, C, Cg, g.G);
        if (m < CPL && ro.is_tr && ro.lab_ok && lp >= 0) v = exp((double)a.A[(size_t)c * C + lp]);
        const int i = 1 + j + m * g.LPW;   // window lanes: row s + i, duration i + 2
        if (ro.is_win && wreg && ro.lab_ok && m < nrw && i <= K - 2) v = exp((double)a.D[(size_t)(i + 1) * C + c]);
        R[m] = v;
    }
    // The exchange: each CTA's block of values (its labels, padded with zeros to an
    // even count CgE, so 16-byte units) goes to every CTA of the cluster by one bulk
    // copy per destination, into position rank*CgE of the destination's exchange
    // buffer, completing on its mbarrier.
    const int CgE = (int)even_up(Cg);
    // The copies are issued from up to four warps, one per scheduler: issuing to
    // many CTAs from one warp serialises (~70 cycles per destination, measured).
    // With TS the first four transition warps, else the owner warps first, then
    // transition warps; issuing warp w lane l sends to CTA w + nwi*l.
    constexpr bool ts = CLUSTER && TS;
    const int iw0 = ts ? g.NWO : 0;
    const int nwi = ts ? (g.NWT < 4 ? g.NWT : 4) : (g.NWO + g.NWT < 4 ? g.NWO + g.NWT : 4);
    const int dst_rank = (warp - iw0) + nwi * lane;
    const bool issuer = CLUSTER && warp >= iw0 && warp < iw0 + nwi && dst_rank < g.G;
    const uint32_t bdst = issuer ? mapa_rank(smem_addr(&sm.gath[rank * CgE]), (uint32_t)dst_rank) : 0u;
    const uint32_t bbar = issuer ? mapa_rank(smem_addr(&sm.full[0]), (uint32_t)dst_rank) : 0u;
    // TS: a label's value goes from its own lanes to every CTA by st.async
    const uint32_t xg = smem_addr(&sm.gath[rank * CgE + (ro.lab_ok ? lc : 0)]), xb = smem_addr(&sm.full[0]);
    double(&Er)[CPL] = *reinterpret_cast<double(*)[CPL]>(&R[0]);
    double &W0 = R[0], &W1 = R[1], &V1 = R[2], &V2 = R[3], &pre = R[4], &gg = R[5], &pbe = R[6], &w0e = R[7],
           &coef = R[8], &a2 = R[9], &mu_acc = R[10], &musum = R[11], &bp = R[12], &start = R[13];
    double gg_n = 0.0, coef_n = 0.0, a2_n = 0.0;
    int rb = 0, h1 = 0, h2 = 0, kb = 0, kb_n = 0;
    auto prefetch = [&](int sp) {   // owners: position sp's tables and recomputed rows
        if (sp >= 0) {
            const size_t ix = (rowbase + sp) * C + c;
            const int sl = sp & (kPF - 1);
            cp_async8(&sm.pf_es[sl * Cg + lc], a.tES + ix);
            cp_async8(&sm.pf_ies[sl * Cg + lc], a.tIES + ix);
            cp_async4(&sm.pf_m[sl * Cg + lc], a.tM + ix);
            if (!CHAIN && sp >= 1) {
                cp_async8(&sm.pf_cu[sl * Cg + lc], a.cU + ix);
                cp_async8(&sm.pf_ca[sl * Cg + lc], a.cA + ix);
                cp_async4(&sm.pf_eu[sl * Cg + lc], a.eU + ix);
                cp_async4(&sm.pf_ea[sl * Cg + lc], a.eA + rowbase + sp);
            }
        }
        cp_async_commit();
    };
    auto prepare = [&](int sn, int un, double d2, double &pre_o, double &gg_o, double &pbe_o, double &w0e_o,
                       double &coef_o, double &a2_o, int &kb_o) {
        const int sl = sn & (kPF - 1);
        kb_o = sm.kbuf[un & 3];
        double p3 = 0.0;
        for (int q = 0; q < PW; ++q) p3 += sm.pre3[(un & 3) * Cg * PW + lc * PW + q];
        pre_o = fma(d2, W1, rescale(p3, h1 + h2));
        const int m = sm.pf_m[sl * Cg + lc];
        gg_o = sm.pf_es[sl * Cg + lc] * pow2c(m + kb_o - rb);               // exp(S + ln2 (kb - rb))
        const double eb = sm.pf_ies[sl * Cg + lc] * pow2c(rb - kb_o - m);   // exp(ln2 (rb - kb) - S)
        pbe_o = pre_o * eb;
        w0e_o = W0 * eb;
        if constexpr (!CHAIN) {
            coef_o = (sn == 0) ? scale2c(cz, rb - kZ)
                               : scale2c(sm.pf_cu[sl * Cg + lc], sm.pf_eu[sl * Cg + lc] + rb);
            a2_o = (sn >= 1) ? scale2c(sm.pf_ca[sl * Cg + lc], sm.pf_ea[sl * Cg + lc] + kb_o) : 0.0;
        } else {
            coef_o = 0.0;
            a2_o = 0.0;
        }
    };
    if (own) {
        W0 = exp((double)a.D[c]);
        W1 = K >= 2 ? exp((double)a.D[C + c]) : 0.0;
        V2 = 0.0;
        musum = 0.0;
        rb = a.tM[(rowbase + L) * C + c];
        V1 = a.tES[(rowbase + L) * C + c];
        a.Vst[(rowbase + L) * C + c] = V1;
        a.rbst[(rowbase + L) * C + c] = rb;
        mu_acc = CHAIN ? 0.0 : scale2(a.cA[(rowbase + L) * C + c], a.eA[rowbase + L]);
        for (int i = 1; i < kPF; ++i) prefetch(L - i);
        cp_async_wait<kPF - 2>();   // position L-1 has landed
        prepare(L - 1, 0, V2, pre, gg, pbe, w0e, coef, a2, kb);
    }
    if constexpr (CLUSTER) cluster_barrier();
    else __syncthreads();
    if (ts) {   // bp[L-1] from the owners, later ones from the transition lanes (as forward)
        if (own) {
            const double b0 = fma(V1, w0e, pbe);
            for (int dr = 0; dr < g.G; ++dr) st_async_at(mapa_rank(xg, dr), mapa_rank(xb, dr), b0);
        }
    }

    int sK = (L - 1) % K;   // s mod K
    bool timed_out = false;
    for (int s = L - 1; s >= 0; --s) {
        const int u = L - 1 - s;   // step count: buffers by u
        const int par = u & 1;
        if (ro.is_own) {
            // ------------------------------------------------ owners: chain
            if (own) bp = fma(V1, w0e, pbe);   // as in the forward
            if constexpr (CLUSTER) {
                if (!ts) {
                    if (own) sm.stage[par * CgE + lc] = bp;
                    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
                    cta_barrier(5, NOT);
                    if (issuer)
                        bulk_to_peer(bdst + par * g.GP * 8, smem_addr(sm.stage + par * CgE), (uint32_t)(CgE * 8),
                                     bbar + par * 8);
                }
            } else if (own) {
                sm.gath[par * g.GP + c] = bp;
            }
            if (own) {
                const double pb = fma(V1, W0, pre);
                start = coef * pb;   // marginal of a segment of label c starting at s
                const int ex = exponent_of(pb);
                const int h = (ex > kRebaseBits || ex < -kRebaseBits) ? -ex : 0;
                if (h != 0) {
                    const double s2 = pow2(h);
                    rb -= h;
                    gg *= s2;
                    V1 *= s2;
                }
                sm.hbuf[(u & 3) * Cg + lc] = h;
                h2 = h1;
                h1 = h;
            }
            if (u >= 1 && s >= 1) cta_barrier(kBarWin + ((u - 1) & 1), NOW);   // window sums of step u-1
            if (own) {
                cp_async_wait<kPF - 3>();   // position s-1 has landed (the prefetch follows the new row)
                if (s >= 1) prepare(s - 1, u + 1, V1, pre, gg_n, pbe, w0e, coef_n, a2_n, kb_n);
            }
            if (ts) {   // gg_s, W0 eb and pre eb of s-1 (as forward)
                if (own && s >= 1) {
                    sm.pub[lc] = gg;
                    sm.pub[CgE + lc] = w0e;
                    sm.pub[2 * CgE + lc] = pbe;
                }
                cta_arrive(kBarPub, NOT);
            } else if constexpr (!CLUSTER) {
                cta_arrive(1, NOT);
                if (g.NWO > 1) cta_barrier(7, 32 * g.NWO);
                else __syncwarp();
            }
            cta_barrier(4, NOT);
            // ------------------------------------------------ owners: new row
            if (own) {
                // mu_acc holds the coverage of x[s] by label c; moving to x[s-1] adds the
                // segments ending at s and removes those starting at s
                const size_t row = (rowbase + s) * C + c;
                if constexpr (!CHAIN) {
                    if (a.dX) a.dX[((size_t)b * a.T + s) * C + c] = (float)mu_acc;
                    if (a.stst) a.stst[row] = start;
                }
                musum += mu_acc;
                a.bpst[row] = bp;
                if (c == 0) a.kbst[rowbase + s] = kb;
                if (s >= 1) {
                    const double q = sm.qbuf[par * CgE + lc];
                    const double V = q * gg;
                    sm.ring[sK * RS + lc] = V;
                    sm.ring[(sK + K) * RS + lc] = V;
                    V2 = V1;
                    V1 = V;
                    mu_acc += a2 * q - start;
                    a.Vst[row] = V;
                    a.rbst[row] = rb;
                } else {
                    mu_acc -= start;
                }
                gg = gg_n;
                coef = coef_n;
                a2 = a2_n;
                kb = kb_n;
                prefetch(s - (kPF - 1));   // into the slot position s+1 used
            }
            if (s >= 1) cta_arrive(kBarRow + (u & 1), NOW);   // row s and h_s stored, for the window
        } else if (ro.is_tr) {
            // ------------------------------------------- transposed transition
            if constexpr (CLUSTER) {
                if (tid == 32 * g.NWO) mbar_expect_tx(&sm.full[par], ts ? C * 8 : g.G * (int)even_up(Cg) * 8);   // as forward
                if (!ts) {
                    cta_barrier(5, NOT);   // the owners' stage is written
                    if (issuer)
                        bulk_to_peer(bdst + par * g.GP * 8, smem_addr(sm.stage + par * CgE), (uint32_t)(CgE * 8),
                                     bbar + par * 8);
                }
                if (!wait_values<CLUSTER>(sm, par, u, timed_out)) {
                    timed_out = true;
                    set_status(a.status, SEMICRF_ERR_DEVICE_TIMEOUT);
                }
            } else {
                cta_barrier(1, NOT);
            }
            const double *gp = sm.gath + par * g.GP + j;   // zeros past C
            // q and the backward normaliser, formed as in the forward
            double n;
            double q = chunked_dot<CPL>(gp, g.LPL, Er, &n);
            group_sum2(q, n, g.LPL);
            if (ts) {
                cta_barrier(kBarPub, NOT);
                if (s >= 1 && ro.lab_ok) {   // bp[s-1] = (q_s gg_s) (W0 eb) + pre eb, sent (as forward)
                    const double bn = fma(q * sm.pub[lc], sm.pub[CgE + lc], sm.pub[2 * CgE + lc]);
                    const uint32_t og = xg + (uint32_t)((par ^ 1) * g.GP * 8), ob = xb + (uint32_t)((par ^ 1) * 8);
                    for (int dr = j; dr < g.G; dr += g.LPL) st_async_at(mapa_rank(og, dr), mapa_rank(ob, dr), bn);
                }
            }
            if (ro.lab_ok && j == 0) sm.qbuf[par * CgE + lc] = q;
            const bool k_late = CLUSTER && !ts;   // as forward
            if (k_late) cta_arrive(4, NOT);
            if (lc == 0 && j == 0) {
                const int kk = sm.kbuf[u & 3];
                if (s == 0) {
                    if (rank == 0) a.logzb[b] = kLn2 * (double)kk + log(n);
                } else if (s >= 2) {
                    sm.kbuf[(u + 2) & 3] = kk + exponent_of(n);
                }
            }
            if (!k_late) cta_arrive(4, NOT);
        } else if (ro.is_win) {
            // ----------------------- window sums two positions ahead (position s-2)
            if (u >= 1) cta_barrier(kBarRow + ((u - 1) & 1), NOW);   // row s+1, h_{s+1} (as forward)
            // rebases at s+1: rows i = 2..K-2 of those labels (as forward)
            int hp = ro.lab_ok ? sm.hbuf[((u - 1) & 3) * Cg + lc] : 0;
            if constexpr (ts) {
                const int wl = tid - 32 * (g.NWO + g.NWT), nw = 32 * g.NWW;   // window lane index
                if (coop_rescale(sm.ring, sm.hbuf + ((u - 1) & 3) * Cg, K, RS, cg_own, sK + 2, 1, K - 3, wl, nw,
                                 lane))
                    cta_barrier(kBarResc, nw);
                hp = 0;
            }
            double v = 0.0;
            if (ro.lab_ok)
                v = wreg ? window_bwd_nr<NU>(g.NRB, sm.ring, K, RS, lc, g.LPW, j, sK, hp, R)
                         : window_bwd(sm.ring, sm.Wd, K, RS, lc, g.LPW, j, sK, hp);
            const double sum = group_sum(v, g.LPW < 32 ? g.LPW : 32);
            if (ro.lab_ok && (j & 31) == 0 && s >= 2) sm.pre3[((u + 2) & 3) * Cg * PW + lc * PW + (j >> 5)] = sum;
            if (s >= 2) cta_arrive(kBarWin + (u & 1), NOW);
        }
        sK = (sK == 0) ? K - 1 : sK - 1;
    }
    if (own) {
        if constexpr (!CHAIN) {
            a.musum[(size_t)b * C + c] = musum;
            a.mures[(size_t)b * C + c] = mu_acc;
        }
    }
    if constexpr (CLUSTER) cluster_barrier();
}

template <int CPL, int MAXT, bool CLUSTER, bool TS>
__global__ void __launch_bounds__(MAXT, 1) cl_bwd_kernel(FbArgs a, ClGeom g)
{
    cl_bwd_body<CPL, MAXT, CLUSTER, false, TS>(a, g, blockIdx.x / g.G);
}

// Forward (storing its rows) and the beta chain side by side: clusters [0, B)
// run the forward of sequence b, clusters [B, 2B) the beta chain of b - B.
template <int CPL, int MAXT, bool CLUSTER, bool TS>
__global__ void __launch_bounds__(MAXT, 1) cl_fused_kernel(FbArgs a, ClGeom g)
{
    const int cid = blockIdx.x / g.G;
    if (cid < a.B) cl_fwd_body<CPL, MAXT, CLUSTER, 2, TS>(a, g, cid);
    else cl_bwd_body<CPL, MAXT, CLUSTER, true, TS>(a, g, cid - a.B);
}

// The kernel of one (CPL, MAXT) class for a launch kind.  TS = true: the cluster
// kernels whose transition lanes send (instantiated in their own source file).
enum ClKind { kClFwd = 0, kClFwdRecompute = 1, kClBwd = 2, kClFused = 3 };
template <int CPL, int MAXT, bool TS>
void *cl_kernel_tpl(bool cl, int kind)
{
    if constexpr (TS) {
        switch (kind) {
        case kClFwd: return (void *)cl_fwd_kernel<CPL, MAXT, true, false, true>;
        case kClFwdRecompute: return (void *)cl_fwd_kernel<CPL, MAXT, true, true, true>;
        case kClBwd: return (void *)cl_bwd_kernel<CPL, MAXT, true, true>;
        default: return (void *)cl_fused_kernel<CPL, MAXT, true, true>;
        }
    } else {
        switch (kind) {
        case kClFwd: return cl ? (void *)cl_fwd_kernel<CPL, MAXT, true, false, false>
                               : (void *)cl_fwd_kernel<CPL, MAXT, false, false, false>;
        case kClFwdRecompute: return cl ? (void *)cl_fwd_kernel<CPL, MAXT, true, true, false>
                                        : (void *)cl_fwd_kernel<CPL, MAXT, false, true, false>;
        case kClBwd: return cl ? (void *)cl_bwd_kernel<CPL, MAXT, true, false>
                               : (void *)cl_bwd_kernel<CPL, MAXT, false, false>;
        default: return cl ? (void *)cl_fused_kernel<CPL, MAXT, true, false>
                           : (void *)cl_fused_kernel<CPL, MAXT, false, false>;
        }
    }
}
template <int CPL, int MAXT>
void *cl_kernel_ts0(bool cl, int kind) { return cl_kernel_tpl<CPL, MAXT, false>(cl, kind); }
template <int CPL, int MAXT>
void *cl_kernel_ts1(bool cl, int kind) { return cl_kernel_tpl<CPL, MAXT, true>(cl, kind); }

int cl_cpl_bucket(int cpl) { return cpl <= 4 ? 4 : cpl <= 8 ? 8 : cpl <= 16 ? 16 : 32; }
// Launch-bounds classes: the kernel's register budget is 65536 / class per thread
// (256, 152, 128, 80, 64), so a plan takes the smallest class that holds it.
int cl_max_threads(int nt) { return nt <= 256 ? 256 : nt <= 416 ? 416 : nt <= 512 ? 512 : nt <= 768 ? 768 : 1024; }

#define SEMICRF_CL_CASE(CPL, MAXT, CALL) \
    if (cpl == CPL && maxt == MAXT) return CALL<CPL, MAXT>
#define SEMICRF_CL_TABLE(CALL, ...)                                                                        \
    SEMICRF_CL_CASE(4, 256, CALL)(__VA_ARGS__); SEMICRF_CL_CASE(4, 416, CALL)(__VA_ARGS__);                \
    SEMICRF_CL_CASE(4, 512, CALL)(__VA_ARGS__);                                                            \
    SEMICRF_CL_CASE(4, 768, CALL)(__VA_ARGS__); SEMICRF_CL_CASE(4, 1024, CALL)(__VA_ARGS__);               \
    SEMICRF_CL_CASE(8, 256, CALL)(__VA_ARGS__); SEMICRF_CL_CASE(8, 416, CALL)(__VA_ARGS__);                \
    SEMICRF_CL_CASE(8, 512, CALL)(__VA_ARGS__);                                                            \
    SEMICRF_CL_CASE(8, 768, CALL)(__VA_ARGS__); SEMICRF_CL_CASE(8, 1024, CALL)(__VA_ARGS__);               \
    SEMICRF_CL_CASE(16, 256, CALL)(__VA_ARGS__); SEMICRF_CL_CASE(16, 416, CALL)(__VA_ARGS__);              \
    SEMICRF_CL_CASE(16, 512, CALL)(__VA_ARGS__);                                                           \
    SEMICRF_CL_CASE(16, 768, CALL)(__VA_ARGS__); SEMICRF_CL_CASE(32, 256, CALL)(__VA_ARGS__);              \
    SEMICRF_CL_CASE(32, 416, CALL)(__VA_ARGS__); SEMICRF_CL_CASE(32, 512, CALL)(__VA_ARGS__);

}  // namespace

// fb_cluster_ts.cu: the kernel of a plan with TS = 1 for a launch kind.
void *cl_kernel_ts(const ClGeom &g, int kind);

}  // namespace semicrf
