// fb_small.cu -- latency-first forward, recompute and backward for few labels and
// short durations (C <= 32, K <= 32): one CTA per sequence, warp-specialised.
//
// Same recursions and scaled exp-space representation as forward_backward.cu
// (Streaming Structured Inference with Flash-SemiCRF, abstract; technical
// summary 2.A-2.C), laid out for the shortest dependent chain per position.
// The sequential chain of one step is: the d = 1 duration term, the exchange of
// the C values a'[t,:] (b'[s,:] backward), the C-term transition dot product and
// the new ring row.  Everything else is split off onto other warps so that it
// runs on other SM sub-partitions, one step ahead or behind:
//
//   forward / recompute (3 warps)        backward (4 warps)
//   warp 0  chain (lane = label)          warp 0  chain (lane = label)
//   warp 1  window: sum of durations      warp 1  window: durations 2..K of the
//           2..K for the next step,               next step, and the dD terms
//           checkpoints                   warp 2  dA terms (one step behind)
//   warp 2  io: cp.async prefetch of the  warp 3  io: cp.async prefetch of the
//           exp tables, recompute output          tables and recomputed rows
//
// One named barrier per step orders the roles.  A ring-column rescale (rare) is
// a synchronous event: the chain decides it, the window warp applies it after
// the step barrier, and a second barrier follows only on such steps.
//
// Other choices:
//  * No exponential or division in the loops: exp(S + ln2 (r - k)) is an exp
//    table entry (exp_tables.cu) times an exactly built power of two, so a
//    recompute started from a checkpoint reproduces the forward pass bit for bit.
//  * Each ring column stores every row twice, so the K-row window is a run of
//    compile-time offsets from one base address; durations beyond K read finite
//    values that meet a zero weight.
//  * The idle lane C (when C < 32) has a row of ones for exp(A) and so computes
//    the normaliser sum_c a'[t,c] inside the transition dot product.
#include <math.h>

#include "device_util.cuh"
#include "semicrf_internal.h"

namespace semicrf {
namespace {

constexpr int kP = 8;   // exp-table prefetch ring depth (steps); prefetch distance kP-1

__host__ __device__ __forceinline__ int col_len(int KM) { return 2 * KM + 1; }

// ring columns, padded to an even count so what follows stays 16-byte aligned
__host__ __device__ __forceinline__ size_t ring_doubles(int KM, int C)
{
    return ((size_t)C * col_len(KM) + 1) & ~(size_t)1;
}

__device__ __forceinline__ void team_barrier(int nthreads)
{
    asm volatile("bar.sync 1, %0;" ::"r"(nthreads) : "memory");
}

// Shared-memory carve-up, forward (in doubles, then ints)
struct FwdSmem {
    double *ring, *xsh, *prebuf, *Ubuf, *apbuf, *tES, *tIES;
    int *tM, *hbuf, *rbuf, *kbuf;
};

__host__ __device__ __forceinline__ size_t fwd_smem_bytes(int KM, int C)
{
    return (ring_doubles(KM, C) + 4 * 64 + 2 * kP * 32) * sizeof(double) +
           (kP * 32 + 64 + 64 + 4) * sizeof(int);
}

__device__ __forceinline__ FwdSmem fwd_smem(double *base, int KM, int C)
{
    FwdSmem s;
    s.ring = base;
    s.xsh = s.ring + ring_doubles(KM, C);
    s.prebuf = s.xsh + 64;
    s.Ubuf = s.prebuf + 64;
    s.apbuf = s.Ubuf + 64;
    s.tES = s.apbuf + 64;
    s.tIES = s.tES + kP * 32;
    s.tM = reinterpret_cast<int *>(s.tIES + kP * 32);
    s.hbuf = s.tM + kP * 32;
    s.rbuf = s.hbuf + 64;
    s.kbuf = s.rbuf + 64;
    return s;
}

struct BwdSmem {
    double *ring, *xsh, *prebuf, *a2buf, *tES, *tIES, *tCU, *tCA;
    int *tM, *tEU, *tEA, *hbuf;
};

__host__ __device__ __forceinline__ size_t bwd_smem_bytes(int KM, int C)
{
    return (ring_doubles(KM, C) + 3 * 64 + 4 * kP * 32) * sizeof(double) +
           (2 * kP * 32 + kP + 64) * sizeof(int);
}

__device__ __forceinline__ BwdSmem bwd_smem(double *base, int KM, int C)
{
    BwdSmem s;
    s.ring = base;
    s.xsh = s.ring + ring_doubles(KM, C);
    s.prebuf = s.xsh + 64;
    s.a2buf = s.prebuf + 64;
    s.tES = s.a2buf + 64;
    s.tIES = s.tES + kP * 32;
    s.tCU = s.tIES + kP * 32;
    s.tCA = s.tCU + kP * 32;
    s.tM = reinterpret_cast<int *>(s.tCA + kP * 32);
    s.tEU = s.tM + kP * 32;
    s.tEA = s.tEU + kP * 32;
    s.hbuf = s.tEA + kP;
    return s;
}

// ===========================================================================
// Forward, MODE 0: one CTA per sequence, t = 1..L; checkpoint after every
// delta-th step, log Z at t = L.  MODE 1 (recompute): one CTA per (sequence,
// checkpoint segment), replaying t = j*delta+1 .. min((j+1)*delta, L) and
// writing the per-position forward quantities relative to Z.  MODE 2: the
// whole sequence once, log Z, and the per-position quantities unscaled (the
// caller applies exp(-log Z) once log Z is known); no checkpoints.
// ===========================================================================
template <int KM, int CM, int MODE>
__device__ __forceinline__ void team_fwd_body(const FbArgs &a, int blk)
{
    constexpr bool RECOMPUTE = MODE == 1;
    constexpr bool ROWS = MODE != 0;   // writes the per-position rows
    constexpr bool CKPT = MODE == 0;   // writes checkpoints
    constexpr int NT = 96;
    extern __shared__ __align__(16) double smt[];
    const int K = a.K, C = a.C;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (warp >= 3) return;   // launched with a fourth warp alongside the backward
    int b, seg;
    if constexpr (RECOMPUTE) {
        b = blk / a.J;
        seg = blk % a.J;
    } else {
        b = blk;
        seg = 0;
    }
    const int L = a.lengths[b];
    if (L < 1 || L > a.T) {
        if (threadIdx.x == 0 && seg == 0) set_status(a.status, SEMICRF_ERR_INVALID_LENGTH);
        return;
    }
    const int t_begin = seg * a.delta;
    if (RECOMPUTE && t_begin >= L) return;
    const int t_end = RECOMPUTE ? min(t_begin + a.delta, L) : L;

    const bool act = lane < C;
    const int c = act ? lane : 0;
    FwdSmem sm = fwd_smem(smt, KM, C);
    double *col = sm.ring + (size_t)c * col_len(KM);   // row rho at (rho%K)+KM and (rho%K)+KM-K
    const size_t rowbase = (size_t)b * (a.T + 1);
    unsigned char *ck_base = a.ckpt + ((size_t)b * a.J) * a.ckpt_stride;
    int kZ = 0;
    double c0 = MODE == 2 ? 1.0 : 0.0;
    if constexpr (RECOMPUTE) {
        kZ = a.lz[b].k;
        c0 = exp(-a.lz[b].logn);
    }

    for (int i = threadIdx.x; i < 64; i += NT) {
        sm.xsh[i] = 0.0;
        sm.prebuf[i] = 0.0;
        sm.hbuf[i] = 0;
    }

    if (warp == 0) {
        // ------------------------------------------------------------------ chain
        const bool nlane = lane == C;
        double E[CM];
#pragma unroll
        for (int cp = 0; cp < CM; ++cp)
            E[cp] = (cp < C) ? (act ? exp((double)a.A[(size_t)cp * C + c]) : (nlane ? 1.0 : 0.0)) : 0.0;
        const double W0 = act ? exp((double)a.D[c]) : 0.0;
        int r = 0, k = 0;
        if constexpr (RECOMPUTE) {
            const int32_t *ck_r = reinterpret_cast<const int32_t *>(
                reinterpret_cast<const double *>(ck_base + (size_t)seg * a.ckpt_stride) + (size_t)K * C);
            r = act ? ck_r[c] : 0;
            k = ck_r[C];
        }
        team_barrier(NT);   // ring initialised
        team_barrier(NT);   // initial look-ahead and first tables in place
        double Uprev = act ? col[(t_begin % K) + KM] : 0.0;
        int tk = (t_begin + 1) % K;          // t % K, kept incrementally
        int td = (t_begin + 1) % a.delta;    // t % delta
        for (int t = t_begin + 1; t <= t_end; ++t) {
            const int par = t & 1;
            const int slot = t & (kP - 1);
            const int m = sm.tM[slot * 32 + lane];
            const double e = sm.tES[slot * 32 + lane] * pow2c(m + r - k);   // exp(S_t + ln2 (r - k))
            double f = sm.tIES[slot * 32 + lane] * pow2c(k - r - m);        // exp(ln2 (k - r) - S_t)
            const double p = fma(Uprev, W0, sm.prebuf[par * 32 + lane]);
            const double ap = p * e;
            const int ex = exponent_of(p);
            const int h = (act && (ex > kRebaseBits || ex < -kRebaseBits)) ? -ex : 0;
            if (h != 0) {
                f *= pow2(h);
                r -= h;
            }
            sm.hbuf[par * 32 + lane] = h;
            if (act) sm.xsh[par * 32 + lane] = ap;
            __syncwarp();
            double q0 = 0.0, q1 = 0.0, q2 = 0.0, q3 = 0.0;
#pragma unroll
            for (int cp = 0; cp < CM; cp += 4) {
                const double2 v01 = *reinterpret_cast<const double2 *>(&sm.xsh[par * 32 + cp]);
                const double2 v23 = *reinterpret_cast<const double2 *>(&sm.xsh[par * 32 + cp + 2]);
                q0 = fma(v01.x, E[cp], q0);
                q1 = fma(v01.y, E[cp + 1], q1);
                q2 = fma(v23.x, E[cp + 2], q2);
                q3 = fma(v23.y, E[cp + 3], q3);
            }
            const double q = (q0 + q1) + (q2 + q3);
            double n;
            if (C < 32) {
                n = __shfl_sync(0xffffffffu, q, C);
            } else {
                n = 0.0;
                for (int cc = 0; cc < C; ++cc) n += sm.xsh[par * 32 + cc];
            }
            if (t == L) {
                if constexpr (!RECOMPUTE) {
                    if (lane == 0) {
                        const double lz = kLn2 * (double)k + log(n);
                        a.logZ[b] = lz;
                        a.lz[b].logn = log(n);
                        a.lz[b].k = k;
                        if (!isfinite(lz)) set_status(a.status, SEMICRF_ERR_DEVICE_RANGE);
                    }
                }
                if constexpr (ROWS) {
                    if (act) a.cA[(rowbase + t) * C + c] = ap * c0;
                    if (lane == 0) a.eA[rowbase + t] = k - kZ;
                }
            } else {
                const int knext = k + exponent_of(n);
                const double U = q * f;
                if (act) {
                    col[tk + KM] = U;
                    col[tk + KM - K] = U;
                }
                Uprev = U;
                sm.Ubuf[par * 32 + lane] = U;
                sm.apbuf[par * 32 + lane] = ap;
                sm.rbuf[par * 32 + lane] = r;
                if (lane == 0) {
                    sm.kbuf[par * 2] = k;
                    sm.kbuf[par * 2 + 1] = knext;
                }
                k = knext;
            }
            team_barrier(NT);
            if (__any_sync(0xffffffffu, sm.hbuf[par * 32 + lane] != 0)) team_barrier(NT);
            if (CKPT && td == 0 && t < L) team_barrier(NT);
            tk = (tk + 1 == K) ? 0 : tk + 1;
            td = (td + 1 == a.delta) ? 0 : td + 1;
        }
    } else if (warp == 1) {
        // ----------------------------------------------------------------- window
        double W[KM];
#pragma unroll
        for (int d = 0; d < KM; ++d) W[d] = (act && d < K) ? exp((double)a.D[(size_t)d * C + c]) : 0.0;
        if (act)
            for (int j = 0; j < 2 * KM + 1; ++j) col[j] = 0.0;
        if constexpr (RECOMPUTE) {
            const double *ck_ring = reinterpret_cast<const double *>(ck_base + (size_t)seg * a.ckpt_stride);
            if (act)
                for (int sl = 0; sl < K; ++sl) {
                    const double v = ck_ring[(size_t)sl * C + c];
                    col[sl + KM] = v;
                    col[sl + KM - K] = v;
                }
        } else {
            if (act) {
                col[KM] = 1.0;   // row 0
                col[KM - K] = 1.0;
            }
            double *ck_ring = reinterpret_cast<double *>(ck_base);
            int32_t *ck_r = reinterpret_cast<int32_t *>(ck_ring + (size_t)K * C);
            if (act) {
                for (int sl = 0; sl < K; ++sl) ck_ring[(size_t)sl * C + c] = col[sl + KM];
                ck_r[c] = 0;
            }
            if (lane == 0) ck_r[C] = 0;
        }
        team_barrier(NT);   // ring initialised
        {
            const double *base = col + (t_begin % K) + KM;   // row t_begin; base[-j] is row t_begin-j
            double s0 = 0.0, s1 = 0.0;
#pragma unroll
            for (int d = 2; d <= KM; ++d) {
                if (d <= K) {
                    if (d & 1) s1 = fma(base[-(d - 1)], W[d - 1], s1);
                    else s0 = fma(base[-(d - 1)], W[d - 1], s0);
                }
            }
            sm.prebuf[((t_begin + 1) & 1) * 32 + lane] = s0 + s1;
        }
        team_barrier(NT);
        int tk = (t_begin + 1) % K;          // t % K, kept incrementally
        int td = (t_begin + 1) % a.delta;    // t % delta
        for (int t = t_begin + 1; t <= t_end; ++t) {
            const int par = t & 1;
            if (t < t_end) {   // durations 2..K of step t+1: rows t-1 .. t+1-K
                // (never the two places of row t, which the chain writes concurrently)
                const double *base = col + tk + KM;
                double s0 = 0.0, s1 = 0.0;
#pragma unroll
                for (int d = 2; d <= KM; ++d) {
                    if (d <= K) {
                        if (d & 1) s1 = fma(base[-(d - 1)], W[d - 1], s1);
                        else s0 = fma(base[-(d - 1)], W[d - 1], s0);
                    }
                }
                sm.prebuf[((t + 1) & 1) * 32 + lane] = s0 + s1;
            }
            team_barrier(NT);
            const int h = sm.hbuf[par * 32 + lane];
            if (__any_sync(0xffffffffu, h != 0)) {
                if (act && h != 0) {   // rescale every row but row t (already at the new reference)
                    const double s2 = pow2(h);
                    const int p1 = tk + KM;
                    const double keep = col[p1];
#pragma unroll
                    for (int j = 0; j < 2 * KM + 1; ++j) col[j] *= s2;
                    col[p1] = keep;
                    col[p1 - K] = keep;
                    sm.prebuf[((t + 1) & 1) * 32 + lane] *= s2;
                }
                team_barrier(NT);
            }
            if (CKPT && td == 0 && t < L) {
                // checkpoint t / delta: ring after step t, r, k_{t+1}
                unsigned char *ck = ck_base + (size_t)(t / a.delta) * a.ckpt_stride;
                double *ck_ring = reinterpret_cast<double *>(ck);
                int32_t *ck_r = reinterpret_cast<int32_t *>(ck_ring + (size_t)K * C);
                if (act) {
                    for (int sl = 0; sl < K; ++sl) ck_ring[(size_t)sl * C + c] = col[sl + KM];
                    ck_r[c] = sm.rbuf[par * 32 + lane];
                }
                if (lane == 0) ck_r[C] = sm.kbuf[par * 2 + 1];
                team_barrier(NT);
            }
            tk = (tk + 1 == K) ? 0 : tk + 1;
            td = (td + 1 == a.delta) ? 0 : td + 1;
        }
    } else {
        // --------------------------------------------------------------------- io
        auto prefetch = [&](int tp) {
            if (tp <= t_end && act) {
                const size_t ix = (rowbase + tp) * C + c;
                const int sl = tp & (kP - 1);
                cp_async8(&sm.tES[sl * 32 + lane], a.tES + ix);
                cp_async8(&sm.tIES[sl * 32 + lane], a.tIES + ix);
                cp_async4(&sm.tM[sl * 32 + lane], a.tM + ix);
            }
            cp_async_commit();
        };
        for (int i = 1; i < kP; ++i) prefetch(t_begin + i);
        cp_async_wait<kP - 2>();   // step t_begin+1 has landed
        team_barrier(NT);
        team_barrier(NT);
        auto write_out = [&](int t) {   // recomputed quantities of step t < L
            const int pp = t & 1;
            const size_t row = (rowbase + t) * C + c;
            if (act) {
                a.cU[row] = sm.Ubuf[pp * 32 + lane] * c0;
                a.cA[row] = sm.apbuf[pp * 32 + lane] * c0;
                a.eU[row] = sm.rbuf[pp * 32 + lane] - kZ;
            }
            if (lane == 0) a.eA[rowbase + t] = sm.kbuf[pp * 2] - kZ;
        };
        int td = (t_begin + 1) % a.delta;    // t % delta
        for (int t = t_begin + 1; t <= t_end; ++t) {
            const int par = t & 1;
            prefetch(t + kP - 1);   // into the slot step t-1 used
            if (ROWS && t - 1 > t_begin) write_out(t - 1);
            cp_async_wait<kP - 2>();   // step t+1 has landed
            team_barrier(NT);
            if (__any_sync(0xffffffffu, sm.hbuf[par * 32 + lane] != 0)) team_barrier(NT);
            if (CKPT && td == 0 && t < L) team_barrier(NT);
            td = (td + 1 == a.delta) ? 0 : td + 1;
        }
        if (ROWS && t_end < L) write_out(t_end);
    }
}

template <int KM, int CM, bool RECOMPUTE>
__global__ void __launch_bounds__(96) team_fwd_kernel(FbArgs a)
{
    team_fwd_body<KM, CM, RECOMPUTE ? 1 : 0>(a, blockIdx.x);
}

// ===========================================================================
// Backward: one CTA per sequence, s = L-1 .. 0.  CHAIN = false: the marginals,
// coverage and per-sequence dA, dD on the chain, from the recomputed forward
// rows.  CHAIN = true: the beta chain only (it needs nothing from the forward,
// so it can run beside it), storing per position V and its reference, the
// normalised beta and the backward normaliser for the parallel passes.
// ===========================================================================
template <int KM, int CM, bool CHAIN>
__device__ __forceinline__ void team_bwd_body(const FbArgs &a, int b)
{
    constexpr int NT = 128;
    extern __shared__ __align__(16) double smt[];
    const int K = a.K, C = a.C;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int L = a.lengths[b];
    if (L < 1 || L > a.T) {
        if (threadIdx.x == 0) set_status(a.status, SEMICRF_ERR_INVALID_LENGTH);
        return;
    }
    const bool act = lane < C;
    const int c = act ? lane : 0;
    BwdSmem sm = bwd_smem(smt, KM, C);
    double *col = sm.ring + (size_t)c * col_len(KM);   // row rho at (rho%K) and (rho%K)+K
    const size_t rowbase = (size_t)b * (a.T + 1);
    const int kZ = CHAIN ? 0 : a.lz[b].k;
    const double c0 = CHAIN ? 0.0 : exp(-a.lz[b].logn);

    for (int i = threadIdx.x; i < 64; i += NT) {
        sm.xsh[i] = 0.0;
        sm.prebuf[i] = 0.0;
        sm.a2buf[i] = 0.0;
        sm.hbuf[i] = 0;
    }
    // row L: be = 0, so V[L,c] = exp(S[L,c] - ln2 rb) = es with rb = m
    const size_t ixL = (rowbase + L) * C + c;
    const int rb0 = act ? a.tM[ixL] : 0;

    if (warp == 0) {
        // ------------------------------------------------------------------ chain
        const bool nlane = lane == C;
        double Er[CM];
#pragma unroll
        for (int cc = 0; cc < CM; ++cc)
            Er[cc] = (cc < C) ? (act ? exp((double)a.A[(size_t)c * C + cc]) : (nlane ? 1.0 : 0.0)) : 0.0;
        const double W0 = act ? exp((double)a.D[c]) : 0.0;
        int rb = rb0, kb = 0;
        double Vprev = act ? a.tES[ixL] : 0.0;
        double mu_acc = (act && !CHAIN) ? scale2(a.cA[ixL], a.eA[rowbase + L]) : 0.0;
        double musum = 0.0;
        if (CHAIN && act) {
            a.Vst[ixL] = Vprev;
            a.rbst[ixL] = rb;
        }
        team_barrier(NT);
        team_barrier(NT);
        int sk = (L - 1) % K;   // s % K, kept incrementally
        for (int s = L - 1; s >= 0; --s) {
            const int par = s & 1;
            const int slot = s & (kP - 1);
            const int m = sm.tM[slot * 32 + lane];
            double g = sm.tES[slot * 32 + lane] * pow2c(m + kb - rb);          // exp(S_s + ln2 (kb - rb))
            const double eb = sm.tIES[slot * 32 + lane] * pow2c(rb - kb - m);  // exp(ln2 (rb - kb) - S_s)
            double coef = 0.0, a2 = 0.0;
            if constexpr (!CHAIN) {
                coef = (s == 0) ? scale2c(c0, rb - kZ)
                                : scale2c(sm.tCU[slot * 32 + lane], sm.tEU[slot * 32 + lane] + rb);
                a2 = (s >= 1 && act) ? scale2c(sm.tCA[slot * 32 + lane], sm.tEA[slot] + kb) : 0.0;
            }
            const double pb = fma(Vprev, W0, sm.prebuf[par * 32 + lane]);
            const double start = coef * pb;
            const double bp = pb * eb;
            if (CHAIN && act) {
                a.bpst[(rowbase + s) * C + c] = bp;
                if (lane == 0) a.kbst[rowbase + s] = kb;
            }
            const int ex = exponent_of(pb);
            const int h = (act && (ex > kRebaseBits || ex < -kRebaseBits)) ? -ex : 0;
            if (h != 0) {
                g *= pow2(h);
                rb -= h;
            }
            sm.hbuf[par * 32 + lane] = h;
            if (act) {
                sm.xsh[par * 32 + lane] = bp;
                sm.a2buf[par * 32 + lane] = a2;
            }
            __syncwarp();
            double q0 = 0.0, q1 = 0.0, q2 = 0.0, q3 = 0.0;
#pragma unroll
            for (int cc = 0; cc < CM; cc += 4) {
                const double2 v01 = *reinterpret_cast<const double2 *>(&sm.xsh[par * 32 + cc]);
                const double2 v23 = *reinterpret_cast<const double2 *>(&sm.xsh[par * 32 + cc + 2]);
                q0 = fma(Er[cc], v01.x, q0);
                q1 = fma(Er[cc + 1], v01.y, q1);
                q2 = fma(Er[cc + 2], v23.x, q2);
                q3 = fma(Er[cc + 3], v23.y, q3);
            }
            const double q = (q0 + q1) + (q2 + q3);
            double n;
            if (C < 32) {
                n = __shfl_sync(0xffffffffu, q, C);
            } else {
                n = 0.0;
                for (int cc = 0; cc < C; ++cc) n += sm.xsh[par * 32 + cc];
            }
            if constexpr (!CHAIN) {
                if (act && a.dX) a.dX[((size_t)b * a.T + s) * C + c] = (float)mu_acc;
                if (act && a.stst) a.stst[(rowbase + s) * C + c] = start;
            }
            musum += mu_acc;
            if (s == 0) {
                if (lane == 0) a.logzb[b] = kLn2 * (double)kb + log(n);
                mu_acc -= start;
            } else {
                const int kbn = kb + exponent_of(n);
                const double V = q * g;
                if (act) {
                    col[sk] = V;
                    col[sk + K] = V;
                    if constexpr (CHAIN) {
                        a.Vst[(rowbase + s) * C + c] = V;
                        a.rbst[(rowbase + s) * C + c] = rb;
                    }
                }
                mu_acc += a2 * q - start;
                Vprev = V;
                kb = kbn;
            }
            team_barrier(NT);
            if (__any_sync(0xffffffffu, sm.hbuf[par * 32 + lane] != 0)) team_barrier(NT);
            sk = (sk == 0) ? K - 1 : sk - 1;
        }
        if (act && !CHAIN) {
            a.musum[(size_t)b * C + c] = musum;
            a.mures[(size_t)b * C + c] = mu_acc;
        }
    } else if (warp == 1) {
        // ----------------------------------------------------------------- window
        double W[KM], accD[KM];
#pragma unroll
        for (int d = 0; d < KM; ++d) {
            W[d] = (act && d < K) ? exp((double)a.D[(size_t)d * C + c]) : 0.0;
            accD[d] = 0.0;
        }
        int rb = rb0;
        if (act) {
            for (int j = 0; j < 2 * KM + 1; ++j) col[j] = 0.0;
            const double VL = a.tES[ixL];
            col[L % K] = VL;
            col[(L % K) + K] = VL;
        }
        team_barrier(NT);
        team_barrier(NT);
        int sk1 = L % K;   // (s + 1) % K, kept incrementally
        for (int s = L - 1; s >= 0; --s) {
            const int par = s & 1;
            const int slot = s & (kP - 1);
            // Rows s+1 .. s+K-1 only: the chain overwrites row s+K's slot with row s
            // during this step.  They give the d = 1 dD term of position s and the
            // d = 2..K dD terms and duration sum of position s-1.
            double coef = 0.0, coef_n = 0.0;
            if constexpr (!CHAIN) {
                coef = (s == 0) ? scale2c(c0, rb - kZ)
                                : scale2c(sm.tCU[slot * 32 + lane], sm.tEU[slot * 32 + lane] + rb);
                if (s >= 1) {
                    const int sn = (s - 1) & (kP - 1);
                    coef_n = (s - 1 == 0) ? scale2c(c0, rb - kZ)
                                          : scale2c(sm.tCU[sn * 32 + lane], sm.tEU[sn * 32 + lane] + rb);
                }
            }
            const double *base = col + sk1;   // base[j-1] is row s+j
            if constexpr (!CHAIN) accD[0] = fma(coef, base[0], accD[0]);
            double s0 = 0.0, s1 = 0.0;
#pragma unroll
            for (int j = 1; j < KM; ++j) {
                if (j < K) {
                    const double v = base[j - 1];
                    if constexpr (!CHAIN) accD[j] = fma(coef_n, v, accD[j]);
                    if (j & 1) s1 = fma(v, W[j], s1);
                    else s0 = fma(v, W[j], s0);
                }
            }
            if (s >= 1) sm.prebuf[((s - 1) & 1) * 32 + lane] = s0 + s1;
            team_barrier(NT);
            const int h = sm.hbuf[par * 32 + lane];
            if (__any_sync(0xffffffffu, h != 0)) {
                if (act && h != 0) {   // rescale every row but row s (already at the new reference)
                    const double s2 = pow2(h);
                    const int p1 = (sk1 == 0) ? K - 1 : sk1 - 1;   // s % K
                    const double keep = col[p1];
#pragma unroll
                    for (int j = 0; j < 2 * KM + 1; ++j) col[j] *= s2;
                    col[p1] = keep;
                    col[p1 + K] = keep;
                    if (s >= 1) sm.prebuf[((s - 1) & 1) * 32 + lane] *= s2;
                    rb -= h;
                }
                team_barrier(NT);
            }
            sk1 = (sk1 == 0) ? K - 1 : sk1 - 1;
        }
        if (act && !CHAIN) {
            double *accD_g = a.accD + (size_t)b * K * C;
#pragma unroll
            for (int d = 0; d < KM; ++d)
                if (d < K) accD_g[(size_t)d * C + c] = accD[d];
        }
    } else if (warp == 2) {
        // ------------------------------------------------------------- dA terms
        double accA[CM];
#pragma unroll
        for (int cc = 0; cc < CM; ++cc) accA[cc] = 0.0;
        team_barrier(NT);
        team_barrier(NT);
        for (int s = L - 1; s >= 0; --s) {
            const int par = s & 1;
            if (!CHAIN && s + 1 <= L - 1) {   // transition of position s+1: a2[s+1] outer b'[s+1]
                const int pp = (s + 1) & 1;
                const double a2v = sm.a2buf[pp * 32 + lane];
#pragma unroll
                for (int cc = 0; cc < CM; cc += 4) {
                    const double2 v01 = *reinterpret_cast<const double2 *>(&sm.xsh[pp * 32 + cc]);
                    const double2 v23 = *reinterpret_cast<const double2 *>(&sm.xsh[pp * 32 + cc + 2]);
                    accA[cc] = fma(a2v, v01.x, accA[cc]);
                    accA[cc + 1] = fma(a2v, v01.y, accA[cc + 1]);
                    accA[cc + 2] = fma(a2v, v23.x, accA[cc + 2]);
                    accA[cc + 3] = fma(a2v, v23.y, accA[cc + 3]);
                }
            }
            team_barrier(NT);
            if (__any_sync(0xffffffffu, sm.hbuf[par * 32 + lane] != 0)) team_barrier(NT);
        }
        if (act && !CHAIN) {
            double *accA_g = a.accA + (size_t)b * C * C + (size_t)c * C;
#pragma unroll
            for (int cc = 0; cc < CM; ++cc)
                if (cc < C) accA_g[cc] = accA[cc];
        }
    } else {
        // --------------------------------------------------------------------- io
        auto prefetch = [&](int sp) {
            if (sp >= 0 && act) {
                const size_t ix = (rowbase + sp) * C + c;
                const int sl = sp & (kP - 1);
                cp_async8(&sm.tES[sl * 32 + lane], a.tES + ix);
                cp_async8(&sm.tIES[sl * 32 + lane], a.tIES + ix);
                cp_async4(&sm.tM[sl * 32 + lane], a.tM + ix);
                if (!CHAIN && sp >= 1) {
                    cp_async8(&sm.tCU[sl * 32 + lane], a.cU + ix);
                    cp_async8(&sm.tCA[sl * 32 + lane], a.cA + ix);
                    cp_async4(&sm.tEU[sl * 32 + lane], a.eU + ix);
                    if (lane == 0) cp_async4(&sm.tEA[sl], a.eA + rowbase + sp);
                }
            }
            cp_async_commit();
        };
        // positions s and s-1 are read during step s (chain and window), so keep two
        // positions landed ahead of the step being entered
        for (int i = 1; i < kP; ++i) prefetch(L - i);
        cp_async_wait<kP - 3>();   // positions L-1 and L-2 have landed
        team_barrier(NT);
        team_barrier(NT);
        for (int s = L - 1; s >= 0; --s) {
            const int par = s & 1;
            prefetch(s - kP + 1);   // into the slot position s+1 used (last read in step s+1)
            cp_async_wait<kP - 3>();   // position s-2 has landed
            team_barrier(NT);
            if (__any_sync(0xffffffffu, sm.hbuf[par * 32 + lane] != 0)) team_barrier(NT);
        }
    }
}

template <int KM, int CM>
__global__ void __launch_bounds__(128) team_bwd_kernel(FbArgs a)
{
    team_bwd_body<KM, CM, false>(a, blockIdx.x);
}

// Forward (storing its rows) and the beta chain side by side: blocks [0, B)
// run the forward of sequence b, blocks [B, 2B) the beta chain of sequence b - B.
template <int KM, int CM>
__global__ void __launch_bounds__(128) team_fused_kernel(FbArgs a)
{
    if ((int)blockIdx.x < a.B) team_fwd_body<KM, CM, 2>(a, blockIdx.x);
    else team_bwd_body<KM, CM, true>(a, blockIdx.x - a.B);
}

template <int KM, int CM>
cudaError_t launch_team_tpl(const FbArgs &a, cudaStream_t st, int kind)
{
    const size_t sf = fwd_smem_bytes(KM, a.C), sb = bwd_smem_bytes(KM, a.C);
    const size_t smem = kind == 2 ? sb : kind == 3 ? (sf > sb ? sf : sb) : sf;
    const unsigned grid = kind == 1 ? (unsigned)a.B * (unsigned)a.J : kind == 3 ? 2u * (unsigned)a.B : (unsigned)a.B;
    const unsigned block = kind >= 2 ? 128 : 96;
    void *fn = kind == 0 ? (void *)team_fwd_kernel<KM, CM, false>
               : kind == 1 ? (void *)team_fwd_kernel<KM, CM, true>
               : kind == 2 ? (void *)team_bwd_kernel<KM, CM>
                           : (void *)team_fused_kernel<KM, CM>;
    cudaError_t e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    FbArgs aa = a;
    void *args[] = {&aa};
    prof_before(st);
    e = cudaLaunchKernel(fn, dim3(grid), dim3(block), args, smem, st);
    prof_after(st);
    return e;
}

}  // namespace

bool small_path_ok(int K, int C) { return K <= 32 && C <= 32; }

cudaError_t launch_small(const FbArgs &a, cudaStream_t st, int kind)
{
    const int km = (a.K + 7) / 8 * 8;
    const int cm = (a.C + 3) / 4 * 4;
#define SEMICRF_SMALL_CASE(KK, CC) \
    if (km == KK && cm == CC) return launch_team_tpl<KK, CC>(a, st, kind);
#define SEMICRF_SMALL_ROW(KK)                                                                   \
    SEMICRF_SMALL_CASE(KK, 4) SEMICRF_SMALL_CASE(KK, 8) SEMICRF_SMALL_CASE(KK, 12)             \
    SEMICRF_SMALL_CASE(KK, 16) SEMICRF_SMALL_CASE(KK, 20) SEMICRF_SMALL_CASE(KK, 24)           \
    SEMICRF_SMALL_CASE(KK, 28) SEMICRF_SMALL_CASE(KK, 32)
    SEMICRF_SMALL_ROW(8)
    SEMICRF_SMALL_ROW(16)
    SEMICRF_SMALL_ROW(24)
    SEMICRF_SMALL_ROW(32)
#undef SEMICRF_SMALL_ROW
#undef SEMICRF_SMALL_CASE
    return cudaErrorInvalidConfiguration;
}

}  // namespace semicrf
