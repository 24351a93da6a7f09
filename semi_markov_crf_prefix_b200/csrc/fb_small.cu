// fb_small.cu -- latency-first forward, recompute and backward for few labels and
// short durations (C <= 32, K <= 32): one warp per sequence, lane = label.
//
// Same recursions and scaled exp-space representation as forward_backward.cu
// (Streaming Structured Inference with Flash-SemiCRF, abstract; technical
// summary 2.A-2.C), laid out for the shortest dependent chain per position:
//
//  * Lane c owns ring column c in shared memory, exp(D[., c]) and one row or
//    column of exp(A) in registers, so the only cross-lane traffic per step is
//    the C values a'[t,:] (or b'[s,:]) through shared memory and one __syncwarp.
//  * Look-ahead: the d >= 2 part of the next step's duration sum only needs
//    ring rows that already exist, so it is formed during the current step; the
//    chain per step is one FMA (the d = 1 term), one multiply, the exchange, the
//    C-term transition dot product and one multiply.
//  * No exponential or division in the loop: exp(S + ln2 (r - k)) is read from
//    the exp tables (exp_tables.cu) times an exactly built power of two, so a
//    recompute started from a checkpoint reproduces the forward pass bit for bit.
//  * Each ring column stores every row twice, so the K-row window is a run of
//    compile-time offsets from one base address (no wrap-around arithmetic);
//    durations beyond K read finite values that meet a zero weight.
//  * The idle lane C (when C < 32) has a row of ones for exp(A) and so computes
//    the normaliser sum_c a'[t,c] inside the transition dot product.
#include <math.h>

#include "device_util.cuh"
#include "semicrf_internal.h"

namespace semicrf {
namespace {

constexpr int kWarpsPerBlock = 4;   // four sequences per CTA, one per SM sub-partition
constexpr int kXsh = 64;            // per-warp exchange buffer: [2][32] doubles

__host__ __device__ __forceinline__ int col_len(int KM) { return 2 * KM + 1; }

// ring columns, padded to an even count so the exchange buffer that follows is
// 16-byte aligned for its double2 loads
__host__ __device__ __forceinline__ size_t ring_doubles(int KM, int C)
{
    return ((size_t)C * col_len(KM) + 1) & ~(size_t)1;
}

__host__ __device__ __forceinline__ size_t warp_smem_doubles(int KM, int C)
{
    return ring_doubles(KM, C) + kXsh;
}

template <int KM, int CM, bool RECOMPUTE>
__global__ void __launch_bounds__(kWarpsPerBlock * 32) small_fwd_kernel(FbArgs a)
{
    extern __shared__ __align__(16) double sm_small[];
    const int K = a.K, C = a.C;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int item = blockIdx.x * kWarpsPerBlock + warp;
    int b, seg;
    if constexpr (RECOMPUTE) {
        b = item / a.J;
        seg = item % a.J;
    } else {
        b = item;
        seg = 0;
    }
    if (b >= a.B) return;
    const int L = a.lengths[b];
    if (L < 1 || L > a.T) {
        if (lane == 0 && seg == 0) set_status(a.status, SEMICRF_ERR_INVALID_LENGTH);
        return;
    }
    const int t_begin = seg * a.delta;
    if (RECOMPUTE && t_begin >= L) return;
    const int t_end = RECOMPUTE ? min(t_begin + a.delta, L) : L;

    const bool act = lane < C;
    const bool nlane = lane == C;   // computes sum_c a'[t,c] (exists when C < 32)
    const int c = act ? lane : 0;
    double *wsm = sm_small + (size_t)warp * warp_smem_doubles(KM, C);
    double *col = wsm + (size_t)c * col_len(KM);   // row rho at (rho % K) + KM and (rho % K) + KM - K
    double *xsh = wsm + ring_doubles(KM, C);       // [2][32]
    const size_t rowbase = (size_t)b * (a.T + 1);

    double W[KM], E[CM];
#pragma unroll
    for (int d = 0; d < KM; ++d) W[d] = (act && d < K) ? exp((double)a.D[(size_t)d * C + c]) : 0.0;
#pragma unroll
    for (int cp = 0; cp < CM; ++cp)
        E[cp] = (cp < C) ? (act ? exp((double)a.A[(size_t)cp * C + c]) : (nlane ? 1.0 : 0.0)) : 0.0;

    xsh[lane] = 0.0;
    xsh[32 + lane] = 0.0;
    if (act)
        for (int j = 0; j < 2 * KM + 1; ++j) col[j] = 0.0;
    unsigned char *ck_base = a.ckpt + ((size_t)b * a.J) * a.ckpt_stride;
    int r = 0, k = 0;
    if constexpr (RECOMPUTE) {
        const unsigned char *ck = ck_base + (size_t)seg * a.ckpt_stride;
        const double *ck_ring = reinterpret_cast<const double *>(ck);
        const int32_t *ck_r = reinterpret_cast<const int32_t *>(ck_ring + (size_t)K * C);
        if (act)
            for (int sl = 0; sl < K; ++sl) {
                const double v = ck_ring[(size_t)sl * C + c];
                col[sl + KM] = v;
                col[sl + KM - K] = v;
            }
        r = act ? ck_r[c] : 0;
        k = ck_r[C];
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
    int kZ = 0;
    double c0 = 0.0;
    if constexpr (RECOMPUTE) {
        kZ = a.lz[b].k;
        c0 = exp(-a.lz[b].logn);
    }
    __syncwarp();

    // state entering step t = t_begin + 1
    int t = t_begin + 1;
    double Uprev = act ? col[(t_begin % K) + KM] : 0.0;
    double pre = 0.0;
    {
        const double *base = col + (t_begin % K) + KM;   // row t-1; base[-j] is row t-1-j
        double s0 = 0.0, s1 = 0.0;
#pragma unroll
        for (int d = 2; d <= KM; ++d) {
            if (d & 1) s1 = fma(base[-(d - 1)], W[d - 1], s1);
            else s0 = fma(base[-(d - 1)], W[d - 1], s0);
        }
        pre = s0 + s1;
    }
    size_t ix = (rowbase + t) * C + c;
    double e = scale2(a.tES[ix], a.tM[ix] + r - k);   // exp(S_t + ln2 (r - k))
    double f = scale2(a.tIES[ix], k - r - a.tM[ix]);  // exp(ln2 (k - r) - S_t)
    // tables for t+1, fetched a step ahead
    double es_n = 0.0, ies_n = 0.0;
    int m_n = 0;
    if (t < t_end) {
        ix += C;
        es_n = a.tES[ix];
        ies_n = a.tIES[ix];
        m_n = a.tM[ix];
    }

    for (; t <= t_end; ++t) {
        const int par = t & 1;
        // --- look-ahead for step t+1: rows t-1 .. t+1-K against durations 2..K
        double pn;
        {
            const double *base = col + (t % K) + KM;   // row t's place; base[-j] is row t-j
            double s0 = 0.0, s1 = 0.0;
#pragma unroll
            for (int d = 2; d <= KM; ++d) {
                if (d & 1) s1 = fma(base[-(d - 1)], W[d - 1], s1);
                else s0 = fma(base[-(d - 1)], W[d - 1], s0);
            }
            pn = s0 + s1;
        }
        double es_n2 = 0.0, ies_n2 = 0.0;
        int m_n2 = 0;
        if (t + 1 < t_end) {
            const size_t ix2 = (rowbase + t + 2) * C + c;
            es_n2 = a.tES[ix2];
            ies_n2 = a.tIES[ix2];
            m_n2 = a.tM[ix2];
        }
        // --- chain
        const double p = fma(Uprev, W[0], pre);
        const double ap = p * e;
        const int ex = exponent_of(p);
        const int h = (act && (ex > kRebaseBits || ex < -kRebaseBits)) ? -ex : 0;
        if (h != 0) {   // rescale this lane's column by 2^h (exact); r moves by -h
            const double s2 = pow2(h);
            for (int j = 0; j < 2 * KM + 1; ++j) col[j] *= s2;
            pn *= s2;
            f *= s2;
            r -= h;
        }
        if (act) xsh[par * 32 + lane] = ap;
        __syncwarp();
        double q0 = 0.0, q1 = 0.0, q2 = 0.0, q3 = 0.0;
#pragma unroll
        for (int cp = 0; cp < CM; cp += 4) {
            const double2 v01 = *reinterpret_cast<const double2 *>(&xsh[par * 32 + cp]);
            const double2 v23 = *reinterpret_cast<const double2 *>(&xsh[par * 32 + cp + 2]);
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
            for (int cc = 0; cc < C; ++cc) n += xsh[par * 32 + cc];
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
            } else {
                if (act) a.cA[(rowbase + t) * C + c] = ap * c0;
                if (lane == 0) a.eA[rowbase + t] = k - kZ;
            }
            break;
        }
        const int knext = k + exponent_of(n);
        const double U = q * f;
        if (act) {
            col[(t % K) + KM] = U;
            col[(t % K) + KM - K] = U;
        }
        if constexpr (RECOMPUTE) {
            const size_t row = (rowbase + t) * C + c;
            if (act) {
                a.cU[row] = U * c0;
                a.cA[row] = ap * c0;
                a.eU[row] = r - kZ;
            }
            if (lane == 0) a.eA[rowbase + t] = k - kZ;
        } else if ((t % a.delta) == 0) {
            unsigned char *ck = ck_base + (size_t)(t / a.delta) * a.ckpt_stride;
            double *ck_ring = reinterpret_cast<double *>(ck);
            int32_t *ck_r = reinterpret_cast<int32_t *>(ck_ring + (size_t)K * C);
            if (act) {
                for (int sl = 0; sl < K; ++sl) ck_ring[(size_t)sl * C + c] = col[sl + KM];
                ck_r[c] = r;
            }
            if (lane == 0) ck_r[C] = knext;
        }
        // --- advance to t+1
        Uprev = U;
        pre = pn;
        e = es_n * pow2c(m_n + r - knext);
        f = ies_n * pow2c(knext - r - m_n);
        k = knext;
        es_n = es_n2;
        ies_n = ies_n2;
        m_n = m_n2;
    }
}

template <int KM, int CM>
__global__ void __launch_bounds__(kWarpsPerBlock * 32) small_bwd_kernel(FbArgs a)
{
    extern __shared__ __align__(16) double sm_small[];
    const int K = a.K, C = a.C;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int b = blockIdx.x * kWarpsPerBlock + warp;
    if (b >= a.B) return;
    const int L = a.lengths[b];
    if (L < 1 || L > a.T) {
        if (lane == 0) set_status(a.status, SEMICRF_ERR_INVALID_LENGTH);
        return;
    }
    const bool act = lane < C;
    const bool nlane = lane == C;
    const int c = act ? lane : 0;
    double *wsm = sm_small + (size_t)warp * warp_smem_doubles(KM, C);
    double *col = wsm + (size_t)c * col_len(KM);   // row rho at (rho % K) and (rho % K) + K
    double *xsh = wsm + ring_doubles(KM, C);
    const size_t rowbase = (size_t)b * (a.T + 1);
    const int kZ = a.lz[b].k;
    const double c0 = exp(-a.lz[b].logn);

    double W[KM], Er[CM], accD[KM], accA[CM];
#pragma unroll
    for (int d = 0; d < KM; ++d) {
        W[d] = (act && d < K) ? exp((double)a.D[(size_t)d * C + c]) : 0.0;
        accD[d] = 0.0;
    }
#pragma unroll
    for (int cc = 0; cc < CM; ++cc) {
        Er[cc] = (cc < C) ? (act ? exp((double)a.A[(size_t)c * C + cc]) : (nlane ? 1.0 : 0.0)) : 0.0;
        accA[cc] = 0.0;
    }
    xsh[lane] = 0.0;
    xsh[32 + lane] = 0.0;
    if (act)
        for (int j = 0; j < 2 * KM + 1; ++j) col[j] = 0.0;

    // row L: be = 0, so V[L,c] = exp(S[L,c] - ln2 rb) = es with rb = m
    size_t ix = (rowbase + L) * C + c;
    int rb = act ? a.tM[ix] : 0, kb = 0;
    double Vprev = act ? a.tES[ix] : 0.0;
    if (act) {
        col[L % K] = Vprev;
        col[(L % K) + K] = Vprev;
    }
    __syncwarp();
    double pre = 0.0;
    double mu_acc = act ? scale2(a.cA[(rowbase + L) * C + c], a.eA[rowbase + L]) : 0.0;
    double musum = 0.0;
    int s = L - 1;
    double coef, a2 = 0.0;
    if (s == 0) {
        coef = scale2(c0, rb - kZ);
    } else {
        const size_t row = (rowbase + s) * C + c;
        coef = act ? scale2(a.cU[row], a.eU[row] + rb) : 0.0;
        a2 = act ? scale2(a.cA[row], a.eA[rowbase + s] + kb) : 0.0;
    }
    ix = (rowbase + s) * C + c;
    double g = scale2(a.tES[ix], a.tM[ix] + kb - rb);    // exp(S_s + ln2 (kb - rb))
    double eb = scale2(a.tIES[ix], rb - kb - a.tM[ix]);  // exp(ln2 (rb - kb) - S_s)
    // position s-1, fetched a step ahead
    double nU = 0.0, nA = 0.0, es_n = 0.0, ies_n = 0.0;
    int nR = 0, nK = 0, m_n = 0;
    if (s >= 1) {
        const size_t row = (rowbase + s - 1) * C + c;
        es_n = a.tES[row];
        ies_n = a.tIES[row];
        m_n = a.tM[row];
        if (s - 1 >= 1 && act) {
            nU = a.cU[row];
            nA = a.cA[row];
            nR = a.eU[row];
            nK = a.eA[rowbase + s - 1];
        }
    }

    for (; s >= 0; --s) {
        const int par = s & 1;
        // --- look-ahead for step s-1: rows s+1 .. s+K-1 are its durations 2..K
        double coef_n = (s - 1 == 0) ? scale2(c0, rb - kZ) : (act ? scale2(nU, nR + rb) : 0.0);
        double pn = 0.0;
        {
            const double *base = col + (s % K);   // row s (written this step) belongs at base[0]
            double s0 = 0.0, s1 = 0.0;
#pragma unroll
            for (int d = 2; d <= KM; ++d) {
                const double v = base[d - 1];
                if (d & 1) s1 = fma(v, W[d - 1], s1);
                else s0 = fma(v, W[d - 1], s0);
                accD[d - 1] = fma(coef_n, v, accD[d - 1]);
            }
            pn = s0 + s1;
        }
        double nU2 = 0.0, nA2 = 0.0, es_n2 = 0.0, ies_n2 = 0.0;
        int nR2 = 0, nK2 = 0, m_n2 = 0;
        if (s >= 2) {
            const size_t row = (rowbase + s - 2) * C + c;
            es_n2 = a.tES[row];
            ies_n2 = a.tIES[row];
            m_n2 = a.tM[row];
            if (s - 2 >= 1 && act) {
                nU2 = a.cU[row];
                nA2 = a.cA[row];
                nR2 = a.eU[row];
                nK2 = a.eA[rowbase + s - 2];
            }
        }
        // --- chain
        const double pb = fma(Vprev, W[0], pre);
        accD[0] = fma(coef, Vprev, accD[0]);
        const double start = coef * pb;
        const double bp = pb * eb;
        const int ex = exponent_of(pb);
        const int h = (act && (ex > kRebaseBits || ex < -kRebaseBits)) ? -ex : 0;
        if (h != 0) {   // rescale this lane's column by 2^h; rb moves by -h
            const double s2 = pow2(h);
            for (int j = 0; j < 2 * KM + 1; ++j) col[j] *= s2;
            pn *= s2;
            g *= s2;
            coef_n *= pow2(-h);
            rb -= h;
        }
        if (act) xsh[par * 32 + lane] = bp;
        __syncwarp();
        double q0 = 0.0, q1 = 0.0, q2 = 0.0, q3 = 0.0;
#pragma unroll
        for (int cc = 0; cc < CM; cc += 4) {
            const double2 v01 = *reinterpret_cast<const double2 *>(&xsh[par * 32 + cc]);
            const double2 v23 = *reinterpret_cast<const double2 *>(&xsh[par * 32 + cc + 2]);
            q0 = fma(Er[cc], v01.x, q0);
            q1 = fma(Er[cc + 1], v01.y, q1);
            q2 = fma(Er[cc + 2], v23.x, q2);
            q3 = fma(Er[cc + 3], v23.y, q3);
            accA[cc] = fma(a2, v01.x, accA[cc]);
            accA[cc + 1] = fma(a2, v01.y, accA[cc + 1]);
            accA[cc + 2] = fma(a2, v23.x, accA[cc + 2]);
            accA[cc + 3] = fma(a2, v23.y, accA[cc + 3]);
        }
        const double q = (q0 + q1) + (q2 + q3);
        double n;
        if (C < 32) {
            n = __shfl_sync(0xffffffffu, q, C);
        } else {
            n = 0.0;
            for (int cc = 0; cc < C; ++cc) n += xsh[par * 32 + cc];
        }
        if (s == 0) {
            if (lane == 0) a.logzb[b] = kLn2 * (double)kb + log(n);
            if (act) {
                a.dX[((size_t)b * a.T + 0) * C + c] = (float)mu_acc;
                musum += mu_acc;
                mu_acc -= start;
            }
            break;
        }
        const int kbn = kb + exponent_of(n);
        const double V = q * g;
        if (act) {
            col[s % K] = V;
            col[(s % K) + K] = V;
            a.dX[((size_t)b * a.T + s) * C + c] = (float)mu_acc;
        }
        const double end = a2 * q;
        musum += mu_acc;
        mu_acc += end - start;
        // --- advance to s-1
        Vprev = V;
        pre = pn;
        coef = coef_n;
        a2 = (s - 1 >= 1 && act) ? scale2(nA, nK + kbn) : 0.0;
        g = es_n * pow2c(m_n + kbn - rb);
        eb = ies_n * pow2c(rb - kbn - m_n);
        kb = kbn;
        nU = nU2;
        nA = nA2;
        nR = nR2;
        nK = nK2;
        es_n = es_n2;
        ies_n = ies_n2;
        m_n = m_n2;
    }
    // per-sequence partial gradients (this lane's column of dD, row of dA)
    if (act) {
        double *accD_g = a.accD + (size_t)b * K * C;
#pragma unroll
        for (int d = 0; d < KM; ++d)
            if (d < K) accD_g[(size_t)d * C + c] = accD[d];
        double *accA_g = a.accA + (size_t)b * C * C + (size_t)c * C;
#pragma unroll
        for (int cc = 0; cc < CM; ++cc)
            if (cc < C) accA_g[cc] = accA[cc];
        a.musum[(size_t)b * C + c] = musum;
        a.mures[(size_t)b * C + c] = mu_acc;
    }
}

template <int KM, int CM>
cudaError_t launch_small_tpl(const FbArgs &a, cudaStream_t st, int kind)
{
    const size_t smem = (size_t)kWarpsPerBlock * warp_smem_doubles(KM, a.C) * sizeof(double);
    unsigned items = kind == 1 ? (unsigned)a.B * (unsigned)a.J : (unsigned)a.B;
    dim3 grid((items + kWarpsPerBlock - 1) / kWarpsPerBlock), block(kWarpsPerBlock * 32);
    void *fn = kind == 0 ? (void *)small_fwd_kernel<KM, CM, false>
               : kind == 1 ? (void *)small_fwd_kernel<KM, CM, true>
                           : (void *)small_bwd_kernel<KM, CM>;
    cudaError_t e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    FbArgs aa = a;
    void *args[] = {&aa};
    prof_before(st);
    e = cudaLaunchKernel(fn, grid, block, args, smem, st);
    prof_after(st);
    return e;
}

}  // namespace

bool small_path_ok(int K, int C) { return K <= 32 && C <= 32; }

cudaError_t launch_small(const FbArgs &a, cudaStream_t st, int kind)
{
    const int km = (a.K + 7) / 8 * 8;
    const int cm = (a.C + 7) / 8 * 8;
#define SEMICRF_SMALL_CASE(KK, CC) \
    if (km == KK && cm == CC) return launch_small_tpl<KK, CC>(a, st, kind);
#define SEMICRF_SMALL_ROW(KK) \
    SEMICRF_SMALL_CASE(KK, 8) SEMICRF_SMALL_CASE(KK, 16) SEMICRF_SMALL_CASE(KK, 24) SEMICRF_SMALL_CASE(KK, 32)
    SEMICRF_SMALL_ROW(8)
    SEMICRF_SMALL_ROW(16)
    SEMICRF_SMALL_ROW(24)
    SEMICRF_SMALL_ROW(32)
#undef SEMICRF_SMALL_ROW
#undef SEMICRF_SMALL_CASE
    return cudaErrorInvalidConfiguration;
}

}  // namespace semicrf
