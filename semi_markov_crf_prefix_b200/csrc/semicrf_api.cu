// semicrf_api.cu -- the extern "C" boundary of libsemicrf.so: argument checks,
// launch planning, workspace layout and kernel launches on the caller's stream.
// No allocation, no synchronisation (except semicrf_get_device_status).
#include <math.h>
#include <string.h>

#include <atomic>

#include "semicrf_internal.h"

namespace semicrf {

namespace {
thread_local int g_last_launches = 0;
thread_local void *const *g_prof_events = nullptr;
thread_local int g_prof_n = 0;
thread_local int g_prof_i = 0;

size_t align_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

int round_up_pow2(int v, int lo)
{
    int x = lo;
    while (x < v) x <<= 1;
    return x;
}
}  // namespace

int device_sm_count()
{
    static std::atomic<int> cache[64];
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) {
        cudaGetLastError();
        return 148;
    }
    int v = cache[dev].load(std::memory_order_relaxed);
    if (v > 0) return v;
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) {
        cudaGetLastError();
        return 148;
    }
    cache[dev].store(n, std::memory_order_relaxed);
    return n;
}

void prof_reset() { g_prof_i = 0; }

void record_launches(int n) { g_last_launches = n; }

void prof_before(cudaStream_t st)
{
    if (g_prof_events && 2 * g_prof_i + 1 < g_prof_n)
        cudaEventRecord(static_cast<cudaEvent_t>(g_prof_events[2 * g_prof_i]), st);
}

void prof_after(cudaStream_t st)
{
    if (g_prof_events && 2 * g_prof_i + 1 < g_prof_n)
        cudaEventRecord(static_cast<cudaEvent_t>(g_prof_events[2 * g_prof_i + 1]), st);
    ++g_prof_i;
}

int default_delta(int T)
{
    int d = (int)ceil(sqrt((double)T));
    return d < 1 ? 1 : d;
}

// Smallest cluster (G CTAs, labels split evenly) whose per-CTA shared memory and
// per-thread register tiles fit, preferring <= 12288 duration+transition terms
// per CTA per step so that a step stays short.
Plan make_plan(int K, int C)
{
    Plan best;
    const int Gs[] = {1, 2, 4, 8, 16};
    for (int gi = 0; gi < 5; ++gi) {
        const int G = Gs[gi];
        if (G > C) break;
        Plan p;
        p.G = G;
        p.Cg = (C + G - 1) / G;
        if ((G - 1) * p.Cg >= C) continue;   // every CTA must own at least one label
        const long work = (long)(K + C) * p.Cg;
        int nt = (int)align_up((size_t)((work + 15) / 16), 32);
        if (nt < 32) nt = 32;
        if (nt > kMaxThreads) nt = kMaxThreads;
        if (nt < p.Cg) nt = (int)align_up((size_t)p.Cg, 32);
        if (nt > kMaxThreads) continue;
        p.NT = nt;
        p.JL = nt / p.Cg;
        p.DPT = round_up_pow2((K + p.JL - 1) / p.JL, 2);
        p.CPT = round_up_pow2((C + p.JL - 1) / p.JL, 2);
        if (p.DPT > 32 || p.CPT > 16) continue;
        const size_t ring = (size_t)K * p.Cg * 8;
        const size_t common = 2 * (size_t)C * 8 + (size_t)nt * 8 + 64;
        p.smem_fwd = ring + common + (size_t)p.Cg * 4 + 16;
        p.smem_bwd = 2 * ring + common + (size_t)p.Cg * 20 + 16;
        p.smem_vit = 2 * ring + common + (size_t)nt * 4;
        if (p.smem_bwd > kSmemBudget || p.smem_vit > kSmemBudget) continue;
        best = p;
        if (work <= 12288) break;
    }
    return best;
}

bool make_layout(const semicrf_dims &d, int what, const Plan &p, Layout *out)
{
    (void)p;
    Layout L;
    const size_t B = d.B, T = d.T, K = d.K, C = d.C;
    L.delta = d.ckpt_interval > 0 ? d.ckpt_interval : default_delta(d.T);
    if (L.delta > d.T) L.delta = d.T;
    L.J = (d.T + L.delta - 1) / L.delta;
    // prefix-scan chunks: eight CTAs per SM over the batch, so that the two
    // HBM-bound passes keep enough loads in flight (two per SM left them at
    // about half the copy bandwidth)
    int nch = (8 * device_sm_count() + d.B - 1) / d.B;
    int maxch = (d.T + 63) / 64;
    if (nch > maxch) nch = maxch;
    if (nch < 1) nch = 1;
    L.NCH = nch;
    size_t off = 0;
    auto take = [&](size_t bytes) {
        size_t o = off;
        off = align_up(off + bytes, 256);
        return o;
    };
    L.status = take(16);
    L.scan = take(B * L.NCH * C * 8);
    if (what == SEMICRF_WS_TRAIN) {
        L.logz = take(B * sizeof(LogZState));
        L.ckpt_stride = align_up(K * C * 8 + (C + 2) * 4, 256);
        L.ckpt = take(B * (size_t)L.J * L.ckpt_stride);
        L.tES = take(B * (T + 1) * C * 8);
        L.tIES = take(B * (T + 1) * C * 8);
        L.tM = take(B * (T + 1) * C * 4);
        L.cU = take(B * (T + 1) * C * 8);
        L.cA = take(B * (T + 1) * C * 8);
        L.eU = take(B * (T + 1) * C * 4);
        L.eA = take(B * (T + 1) * 4);
        L.accD = take(B * K * C * 8);
        L.accA = take(B * C * C * 8);
        L.Vst = take(B * (T + 1) * C * 8);
        L.rbst = take(B * (T + 1) * C * 4);
        L.bpst = take(B * (T + 1) * C * 8);
        L.kbst = take(B * (T + 1) * 4);
        cl_grad_splits(d.B, d.T, d.K, d.C, &L.nsD, &L.nsA);
        L.npost = small_path_ok(d.K, d.C) ? team_post_splits(d.B, d.T) : 0;
        L.partD = take((size_t)(L.nsD > L.npost ? L.nsD : L.npost) * K * C * 8);
        L.partA = take((size_t)(L.nsA > L.npost ? L.nsA : L.npost) * C * C * 8);
        L.stst = take(B * (T + 1) * C * 8);
        L.gcA = take(B * C * C * 4);
        L.gcD = take(B * K * C * 4);
        L.gcN = take(B * C * 4);
        const size_t nch = (T + cov_chunk(d.T) - 1) / cov_chunk(d.T);
        L.covd = take(B * nch * C * 8);
        L.covm = take(B * (size_t)team_post_chunks(d.T) * C * 8);   // cov_chunk >= 32: the larger count
        L.musum = take(B * C * 8);
        L.mures = take(B * C * 8);
        L.logzb = take(B * 8);
    } else if (what == SEMICRF_WS_VITERBI) {
        L.bd = take(B * (T + 1) * C * 2);
        L.bc = take(B * (T + 1) * C * 2);
        L.vfin = take(B * 4);
    } else if (what != SEMICRF_WS_SCAN) {
        return false;
    }
    L.total = off;
    *out = L;
    return true;
}

}  // namespace semicrf

using namespace semicrf;

namespace {

// chains = false: the prefix scan alone, which runs no chain kernel (its dims
// carry K = 1), so no chain geometry is required.
semicrf_status check_dims_impl(const semicrf_dims *d, bool chains = true)
{
    if (!d) return SEMICRF_ERR_INVALID_ARG;
    if (d->B < 1 || d->T < 1 || d->K < 1 || d->C < 1 || d->ckpt_interval < 0)
        return SEMICRF_ERR_INVALID_ARG;
    if (d->C > SEMICRF_MAX_C || d->K > SEMICRF_MAX_K) return SEMICRF_ERR_UNSUPPORTED_SHAPE;
    if ((long long)d->B * (d->T + 1) * d->C > (1LL << 40)) return SEMICRF_ERR_UNSUPPORTED_SHAPE;
    if (!chains) return SEMICRF_OK;
    if (!make_plan(d->K, d->C).ok()) return SEMICRF_ERR_UNSUPPORTED_SHAPE;   // Viterbi layout
    if (!small_path_ok(d->K, d->C)) {
        ClGeom g;
        if (!cl_plan(d->K, d->C, false, &g) || !cl_plan(d->K, d->C, true, &g))
            return SEMICRF_ERR_UNSUPPORTED_SHAPE;
    }
    return SEMICRF_OK;
}

semicrf_status prepare(const semicrf_dims *d, int what, void *ws, size_t ws_bytes, Plan *p,
                       Layout *lay)
{
    prof_reset();
    semicrf_status s = check_dims_impl(d, what != SEMICRF_WS_SCAN);
    if (s != SEMICRF_OK) return s;
    if (!ws) return SEMICRF_ERR_INVALID_ARG;
    if (reinterpret_cast<uintptr_t>(ws) % 256 != 0) return SEMICRF_ERR_INVALID_ARG;
    *p = make_plan(d->K, d->C);
    if (!make_layout(*d, what, *p, lay)) return SEMICRF_ERR_INVALID_ARG;
    if (ws_bytes < lay->total) return SEMICRF_ERR_WORKSPACE_TOO_SMALL;
    return SEMICRF_OK;
}

template <typename T>
T *at(void *ws, size_t off)
{
    return reinterpret_cast<T *>(static_cast<unsigned char *>(ws) + off);
}

semicrf_status finish(cudaError_t e, int launches)
{
    if (e != cudaSuccess) return SEMICRF_ERR_CUDA;
    g_last_launches = launches;
    return SEMICRF_OK;
}

FbArgs fb_args(const semicrf_dims *d, const Layout &lay, void *ws)
{
    FbArgs a;
    memset(&a, 0, sizeof(a));
    a.B = d->B;
    a.T = d->T;
    a.K = d->K;
    a.C = d->C;
    a.delta = lay.delta;
    a.J = lay.J;
    a.lz = at<LogZState>(ws, lay.logz);
    a.ckpt = at<unsigned char>(ws, lay.ckpt);
    a.ckpt_stride = lay.ckpt_stride;
    a.tES = at<double>(ws, lay.tES);
    a.tIES = at<double>(ws, lay.tIES);
    a.tM = at<int32_t>(ws, lay.tM);
    a.cU = at<double>(ws, lay.cU);
    a.cA = at<double>(ws, lay.cA);
    a.eU = at<int32_t>(ws, lay.eU);
    a.eA = at<int32_t>(ws, lay.eA);
    a.accD = at<double>(ws, lay.accD);
    a.accA = at<double>(ws, lay.accA);
    a.musum = at<double>(ws, lay.musum);
    a.mures = at<double>(ws, lay.mures);
    a.logzb = at<double>(ws, lay.logzb);
    a.Vst = at<double>(ws, lay.Vst);
    a.rbst = at<int32_t>(ws, lay.rbst);
    a.bpst = at<double>(ws, lay.bpst);
    a.kbst = at<int32_t>(ws, lay.kbst);
    a.nsD = lay.nsD;
    a.nsA = lay.nsA;
    a.npost = lay.npost;
    a.partD = at<double>(ws, lay.partD);
    a.partA = at<double>(ws, lay.partA);
    a.covd = at<double>(ws, lay.covd);
    a.covm = at<double>(ws, lay.covm);
    a.covch = cov_chunk(d->T);
    a.status = at<int32_t>(ws, lay.status);
    return a;
}

}  // namespace

extern "C" {

semicrf_status semicrf_check_dims(const semicrf_dims *dims) { return check_dims_impl(dims); }

size_t semicrf_workspace_bytes(const semicrf_dims *dims, int32_t what)
{
    if (check_dims_impl(dims, what != SEMICRF_WS_SCAN) != SEMICRF_OK) return 0;
    Plan p = make_plan(dims->K, dims->C);
    Layout lay;
    if (!make_layout(*dims, what, p, &lay)) return 0;
    return lay.total;
}

semicrf_status semicrf_prefix_scan(const semicrf_dims *dims, const float *x, const int32_t *lengths,
                                   double *S, double *nu, void *ws, size_t ws_bytes, void *stream)
{
    Plan p;
    Layout lay;
    // status and scan regions sit at the same offsets in every workspace kind
    semicrf_status s = prepare(dims, SEMICRF_WS_SCAN, ws, ws_bytes, &p, &lay);
    if (s != SEMICRF_OK) return s;
    if (!x || !lengths || !S || !nu) return SEMICRF_ERR_INVALID_ARG;
    ScanArgs a;
    a.B = dims->B;
    a.T = dims->T;
    a.C = dims->C;
    a.NCH = lay.NCH;
    a.x = x;
    a.lengths = lengths;
    a.S = S;
    a.nu = nu;
    a.part = at<double>(ws, lay.scan);
    a.status = at<int32_t>(ws, lay.status);
    int n = 0;
    cudaError_t e = launch_prefix_scan(a, static_cast<cudaStream_t>(stream), &n);
    return finish(e, n);
}

semicrf_status semicrf_forward(const semicrf_dims *dims, const double *S, const float *A, const float *D,
                               const int32_t *lengths, double *logZ, void *ws, size_t ws_bytes,
                               void *stream)
{
    Plan p;
    Layout lay;
    semicrf_status s = prepare(dims, SEMICRF_WS_TRAIN, ws, ws_bytes, &p, &lay);
    if (s != SEMICRF_OK) return s;
    if (!S || !A || !D || !lengths || !logZ) return SEMICRF_ERR_INVALID_ARG;
    FbArgs a = fb_args(dims, lay, ws);
    a.S = S;
    a.A = A;
    a.D = D;
    a.lengths = lengths;
    a.logZ = logZ;
    int n = 0;
    cudaError_t e = launch_forward(p, a, static_cast<cudaStream_t>(stream), &n);
    return finish(e, n);
}

semicrf_status semicrf_backward(const semicrf_dims *dims, const double *S, const float *A, const float *D,
                                const int32_t *lengths, const double *grad_logZ, void *ws,
                                size_t ws_bytes, float *dX, double *dA, double *dD, void *stream)
{
    Plan p;
    Layout lay;
    semicrf_status s = prepare(dims, SEMICRF_WS_TRAIN, ws, ws_bytes, &p, &lay);
    if (s != SEMICRF_OK) return s;
    if (!S || !A || !D || !lengths || !dX || !dA || !dD) return SEMICRF_ERR_INVALID_ARG;
    FbArgs a = fb_args(dims, lay, ws);
    a.S = S;
    a.A = A;
    a.D = D;
    a.lengths = lengths;
    a.grad = grad_logZ;
    a.dX = dX;
    a.dA = dA;
    a.dD = dD;
    int n = 0;
    cudaError_t e = launch_backward(p, a, static_cast<cudaStream_t>(stream), &n);
    return finish(e, n);
}

semicrf_status semicrf_forward_backward(const semicrf_dims *dims, const double *S, const float *A,
                                       const float *D, const int32_t *lengths, const double *grad_logZ,
                                       void *ws, size_t ws_bytes, double *logZ, float *dX, double *dA,
                                       double *dD, void *stream)
{
    Plan p;
    Layout lay;
    semicrf_status s = prepare(dims, SEMICRF_WS_TRAIN, ws, ws_bytes, &p, &lay);
    if (s != SEMICRF_OK) return s;
    if (!S || !A || !D || !lengths || !logZ || !dX || !dA || !dD) return SEMICRF_ERR_INVALID_ARG;
    FbArgs a = fb_args(dims, lay, ws);
    a.S = S;
    a.A = A;
    a.D = D;
    a.lengths = lengths;
    a.grad = grad_logZ;
    a.logZ = logZ;
    a.dX = dX;
    a.dA = dA;
    a.dD = dD;
    int n = 0;
    cudaError_t e = launch_forward_backward(a, static_cast<cudaStream_t>(stream), &n);
    return finish(e, n);
}

namespace {

// Device staging of semicrf_forward_backward_host, in this order, each region
// 256-byte aligned: x, A, D, lengths, grad, S, nu, logZ, dX, dA, dD.
struct HostStage {
    size_t x, A, D, len, grad, S, nu, logZ, dX, dA, dD, total;
};

HostStage host_stage_layout(const semicrf_dims &d)
{
    const size_t B = d.B, T = d.T, K = d.K, C = d.C;
    HostStage h;
    size_t off = 0;
    auto take = [&](size_t bytes) {
        const size_t o = off;
        off = align_up(off + bytes, 256);
        return o;
    };
    h.x = take(B * T * C * 4);
    h.A = take(C * C * 4);
    h.D = take(K * C * 4);
    h.len = take(B * 4);
    h.grad = take(B * 8);
    h.S = take(B * (T + 1) * C * 8);
    h.nu = take(B * C * 8);
    h.logZ = take(B * 8);
    h.dX = take(B * T * C * 4);
    h.dA = take(C * C * 8);
    h.dD = take(K * C * 8);
    h.total = off;
    return h;
}

}  // namespace

size_t semicrf_host_stage_bytes(const semicrf_dims *dims)
{
    if (check_dims_impl(dims) != SEMICRF_OK) return 0;
    return host_stage_layout(*dims).total;
}

semicrf_status semicrf_forward_backward_host(const semicrf_dims *dims, const float *x, const float *A,
                                            const float *D, const int32_t *lengths, const double *grad_logZ,
                                            double *logZ, float *dX, double *dA, double *dD, void *stage,
                                            size_t stage_bytes, void *ws, size_t ws_bytes, void *stream)
{
    semicrf_status s = check_dims_impl(dims);
    if (s != SEMICRF_OK) return s;
    if (!x || !A || !D || !lengths || !logZ || !dA || !dD || !stage) return SEMICRF_ERR_INVALID_ARG;
    if (reinterpret_cast<uintptr_t>(stage) % 256 != 0) return SEMICRF_ERR_INVALID_ARG;
    const HostStage h = host_stage_layout(*dims);
    if (stage_bytes < h.total) return SEMICRF_ERR_WORKSPACE_TOO_SMALL;
    const size_t B = dims->B, T = dims->T, K = dims->K, C = dims->C;
    char *st = static_cast<char *>(stage);
    cudaStream_t cs = static_cast<cudaStream_t>(stream);
    auto h2d = [&](size_t off, const void *src, size_t bytes) {
        return cudaMemcpyAsync(st + off, src, bytes, cudaMemcpyHostToDevice, cs);
    };
    cudaError_t e = h2d(h.x, x, B * T * C * 4);
    if (e == cudaSuccess) e = h2d(h.A, A, C * C * 4);
    if (e == cudaSuccess) e = h2d(h.D, D, K * C * 4);
    if (e == cudaSuccess) e = h2d(h.len, lengths, B * 4);
    if (e == cudaSuccess && grad_logZ) e = h2d(h.grad, grad_logZ, B * 8);
    if (e != cudaSuccess) return SEMICRF_ERR_CUDA;
    s = semicrf_prefix_scan(dims, reinterpret_cast<const float *>(st + h.x),
                            reinterpret_cast<const int32_t *>(st + h.len), reinterpret_cast<double *>(st + h.S),
                            reinterpret_cast<double *>(st + h.nu), ws, ws_bytes, stream);
    if (s != SEMICRF_OK) return s;
    const int n_scan = g_last_launches;
    s = semicrf_forward_backward(dims, reinterpret_cast<const double *>(st + h.S),
                                 reinterpret_cast<const float *>(st + h.A), reinterpret_cast<const float *>(st + h.D),
                                 reinterpret_cast<const int32_t *>(st + h.len),
                                 grad_logZ ? reinterpret_cast<const double *>(st + h.grad) : nullptr, ws, ws_bytes,
                                 reinterpret_cast<double *>(st + h.logZ), reinterpret_cast<float *>(st + h.dX),
                                 reinterpret_cast<double *>(st + h.dA), reinterpret_cast<double *>(st + h.dD), stream);
    if (s != SEMICRF_OK) return s;
    const int n_fb = g_last_launches;
    auto d2h = [&](void *dst, size_t off, size_t bytes) {
        return cudaMemcpyAsync(dst, st + off, bytes, cudaMemcpyDeviceToHost, cs);
    };
    e = d2h(logZ, h.logZ, B * 8);
    if (e == cudaSuccess) e = d2h(dA, h.dA, C * C * 8);
    if (e == cudaSuccess) e = d2h(dD, h.dD, K * C * 8);
    if (e == cudaSuccess && dX) e = d2h(dX, h.dX, B * T * C * 4);
    if (e != cudaSuccess) return SEMICRF_ERR_CUDA;
    g_last_launches = n_scan + n_fb;
    return SEMICRF_OK;
}

semicrf_status semicrf_posteriors(const semicrf_dims *dims, const double *S, const float *A, const float *D,
                                  const int32_t *lengths, void *ws, size_t ws_bytes, float *mu, float *pstart,
                                  void *stream)
{
    Plan p;
    Layout lay;
    semicrf_status s = prepare(dims, SEMICRF_WS_TRAIN, ws, ws_bytes, &p, &lay);
    if (s != SEMICRF_OK) return s;
    if (!S || !A || !D || !lengths) return SEMICRF_ERR_INVALID_ARG;
    FbArgs a = fb_args(dims, lay, ws);
    a.S = S;
    a.A = A;
    a.D = D;
    a.lengths = lengths;
    a.stst = at<double>(ws, lay.stst);
    int n = 0;
    cudaError_t e = launch_posteriors(a, mu, pstart, static_cast<cudaStream_t>(stream), &n);
    return finish(e, n);
}

namespace {
GoldArgs gold_args(const semicrf_dims *dims, const Layout &lay, void *ws, const int32_t *lengths,
                   const int32_t *labels, const uint8_t *seg_start)
{
    GoldArgs g;
    memset(&g, 0, sizeof(g));
    g.B = dims->B;
    g.T = dims->T;
    g.K = dims->K;
    g.C = dims->C;
    g.lengths = lengths;
    g.labels = labels;
    g.seg_start = seg_start;
    g.cntA = at<int32_t>(ws, lay.gcA);
    g.cntD = at<int32_t>(ws, lay.gcD);
    g.cntN = at<int32_t>(ws, lay.gcN);
    g.status = at<int32_t>(ws, lay.status);
    g.wsign = 1.0;
    return g;
}
}  // namespace

semicrf_status semicrf_gold_score(const semicrf_dims *dims, const double *S, const float *A, const float *D,
                                  const int32_t *lengths, const int32_t *labels, const uint8_t *seg_start,
                                  double *score, void *ws, size_t ws_bytes, void *stream)
{
    Plan p;
    Layout lay;
    semicrf_status s = prepare(dims, SEMICRF_WS_TRAIN, ws, ws_bytes, &p, &lay);
    if (s != SEMICRF_OK) return s;
    if (!S || !A || !D || !lengths || !labels || !seg_start || !score) return SEMICRF_ERR_INVALID_ARG;
    GoldArgs g = gold_args(dims, lay, ws, lengths, labels, seg_start);
    g.S = S;
    g.A = A;
    g.D = D;
    g.score = score;
    int n = 0;
    cudaError_t e = launch_gold_score(g, static_cast<cudaStream_t>(stream), &n);
    return finish(e, n);
}

semicrf_status semicrf_gold_backward(const semicrf_dims *dims, const int32_t *lengths, const int32_t *labels,
                                     const uint8_t *seg_start, const double *grad_score, float *dX, double *dA,
                                     double *dD, void *ws, size_t ws_bytes, void *stream)
{
    Plan p;
    Layout lay;
    semicrf_status s = prepare(dims, SEMICRF_WS_TRAIN, ws, ws_bytes, &p, &lay);
    if (s != SEMICRF_OK) return s;
    if (!lengths || !labels || !seg_start || !dX || !dA || !dD) return SEMICRF_ERR_INVALID_ARG;
    GoldArgs g = gold_args(dims, lay, ws, lengths, labels, seg_start);
    g.grad = grad_score;
    g.dX = dX;
    g.dA = dA;
    g.dD = dD;
    int n = 0;
    cudaError_t e = launch_gold_backward(g, static_cast<cudaStream_t>(stream), &n);
    return finish(e, n);
}

semicrf_status semicrf_nll(const semicrf_dims *dims, const double *S, const float *A, const float *D,
                           const int32_t *lengths, const int32_t *labels, const uint8_t *seg_start, double *logZ,
                           double *score, double *nll, void *ws, size_t ws_bytes, void *stream)
{
    if (!nll || !score || !logZ) return SEMICRF_ERR_INVALID_ARG;
    semicrf_status s = semicrf_forward(dims, S, A, D, lengths, logZ, ws, ws_bytes, stream);
    if (s != SEMICRF_OK) return s;
    const int nf = g_last_launches;
    Plan p;
    Layout lay;
    s = prepare(dims, SEMICRF_WS_TRAIN, ws, ws_bytes, &p, &lay);
    if (s != SEMICRF_OK) return s;
    if (!labels || !seg_start) return SEMICRF_ERR_INVALID_ARG;
    GoldArgs g = gold_args(dims, lay, ws, lengths, labels, seg_start);
    g.S = S;
    g.A = A;
    g.D = D;
    g.score = score;
    g.logZ = logZ;
    g.nll = nll;
    int n = 0;
    cudaError_t e = launch_gold_score(g, static_cast<cudaStream_t>(stream), &n);
    return finish(e, nf + n);
}

semicrf_status semicrf_nll_backward(const semicrf_dims *dims, const double *S, const float *A, const float *D,
                                    const int32_t *lengths, const int32_t *labels, const uint8_t *seg_start,
                                    const double *grad_nll, void *ws, size_t ws_bytes, float *dX, double *dA,
                                    double *dD, void *stream)
{
    if (!labels || !seg_start) return SEMICRF_ERR_INVALID_ARG;
    semicrf_status s = semicrf_backward(dims, S, A, D, lengths, grad_nll, ws, ws_bytes, dX, dA, dD, stream);
    if (s != SEMICRF_OK) return s;
    const int nb = g_last_launches;
    Plan p;
    Layout lay;
    s = prepare(dims, SEMICRF_WS_TRAIN, ws, ws_bytes, &p, &lay);
    if (s != SEMICRF_OK) return s;
    GoldArgs g = gold_args(dims, lay, ws, lengths, labels, seg_start);
    g.grad = grad_nll;
    g.wsign = -1.0;   // the NLL subtracts the gold score
    g.dX = dX;
    g.dA = dA;
    g.dD = dD;
    int n = 0;
    cudaError_t e = launch_gold_backward(g, static_cast<cudaStream_t>(stream), &n);
    return finish(e, nb + n);
}

semicrf_status semicrf_viterbi(const semicrf_dims *dims, const double *S, const float *A, const float *D,
                               const int32_t *lengths, double *score, int32_t *labels,
                               uint8_t *seg_start, void *ws, size_t ws_bytes, void *stream)
{
    Plan p;
    Layout lay;
    semicrf_status s = prepare(dims, SEMICRF_WS_VITERBI, ws, ws_bytes, &p, &lay);
    if (s != SEMICRF_OK) return s;
    if (!S || !A || !D || !lengths || !score || !labels || !seg_start) return SEMICRF_ERR_INVALID_ARG;
    VitArgs a;
    a.B = dims->B;
    a.T = dims->T;
    a.K = dims->K;
    a.C = dims->C;
    a.S = S;
    a.A = A;
    a.D = D;
    a.lengths = lengths;
    a.score = score;
    a.labels = labels;
    a.seg_start = seg_start;
    a.bd = at<uint16_t>(ws, lay.bd);
    a.bc = at<uint16_t>(ws, lay.bc);
    a.vfin = at<int32_t>(ws, lay.vfin);
    a.status = at<int32_t>(ws, lay.status);
    int n = 0;
    cudaError_t e = launch_viterbi(p, a, static_cast<cudaStream_t>(stream), &n);
    return finish(e, n);
}

semicrf_status semicrf_clear_device_status(void *ws, void *stream)
{
    if (!ws) return SEMICRF_ERR_INVALID_ARG;
    cudaError_t e = cudaMemsetAsync(ws, 0, 16, static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? SEMICRF_OK : SEMICRF_ERR_CUDA;
}

semicrf_status semicrf_get_device_status(const void *ws, void *stream)
{
    if (!ws) return SEMICRF_ERR_INVALID_ARG;
    if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess) return SEMICRF_ERR_CUDA;
    int32_t h = 0;
    if (cudaMemcpy(&h, ws, sizeof(h), cudaMemcpyDeviceToHost) != cudaSuccess) return SEMICRF_ERR_CUDA;
    return static_cast<semicrf_status>(h);
}

const char *semicrf_status_string(semicrf_status s)
{
    switch (s) {
    case SEMICRF_OK: return "ok";
    case SEMICRF_ERR_INVALID_ARG: return "invalid argument";
    case SEMICRF_ERR_UNSUPPORTED_SHAPE: return "unsupported shape";
    case SEMICRF_ERR_WORKSPACE_TOO_SMALL: return "workspace too small";
    case SEMICRF_ERR_CUDA: return "CUDA error";
    case SEMICRF_ERR_DEVICE_TIMEOUT: return "device wait timed out";
    case SEMICRF_ERR_DEVICE_RANGE: return "non-finite value on device";
    case SEMICRF_ERR_INVALID_LENGTH: return "sequence length outside [1, T]";
    case SEMICRF_ERR_INVALID_SEGMENTATION: return "malformed gold segmentation";
    }
    return "unknown status";
}

semicrf_status semicrf_chain_plan(const semicrf_dims *dims, int32_t path, int32_t *info, int32_t n)
{
    semicrf_status s = check_dims_impl(dims);
    if (s != SEMICRF_OK) return s;
    if (!info || n < 9 || path < 0 || path > 2) return SEMICRF_ERR_INVALID_ARG;
    for (int i = 0; i < n; ++i) info[i] = 0;
    if (small_path_ok(dims->K, dims->C)) {
        info[0] = 0;   // one CTA per sequence (warp-specialised team kernels)
        info[1] = 1;
        info[8] = path == 0 ? 2 * dims->B : dims->B;
        info[7] = -1;
        return SEMICRF_OK;
    }
    info[0] = 1;
    if (!cl_plan_info(dims->K, dims->C, dims->B, path, info + 1)) return SEMICRF_ERR_UNSUPPORTED_SHAPE;
    info[8] = path == 0 ? 2 * dims->B : dims->B;
    return SEMICRF_OK;
}

int32_t semicrf_last_launch_count(void) { return g_last_launches; }

semicrf_status semicrf_set_profile_events(void *const *events, int32_t n)
{
    if (n < 0 || (n > 0 && !events)) return SEMICRF_ERR_INVALID_ARG;
    g_prof_events = n > 0 ? events : nullptr;
    g_prof_n = n;
    g_prof_i = 0;
    return SEMICRF_OK;
}

}  // extern "C"
