// fb_cluster.cu -- planning and launching the cluster chains (fb_cluster_dev.cuh
// holds the device code): the latency model over candidate geometries, the
// residency query that picks a plan whose clusters all run at once, and the
// launches of the forward, recompute, backward and fused kernels.
#include <stdio.h>
#include <stdlib.h>
#include <string.h>

#include <algorithm>
#include <map>
#include <mutex>
#include <tuple>
#include <utility>
#include <vector>

#include "fb_cluster_dev.cuh"

namespace semicrf {
namespace {

// The kernel of a plan for a launch kind (TS = 1 cluster plans: fb_cluster_ts.cu).
void *cl_kernel(const ClGeom &g, int kind)
{
    if (g.G > 1 && g.TS) return cl_kernel_ts(g, kind);
    const int cpl = cl_cpl_bucket(g.CPL), maxt = cl_max_threads(g.NT);
    SEMICRF_CL_TABLE(cl_kernel_ts0, g.G > 1, kind)
    return nullptr;
}

// Shared memory and (G > 8) non-portable cluster size allowed for a kernel.
cudaError_t cl_prepare(void *fn, const ClGeom &g, size_t smem)
{
    cudaError_t e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e == cudaSuccess && g.G > 8) e = cudaFuncSetAttribute(fn, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
    return e;
}

// nclusters clusters of G CTAs (G = 1: plain CTAs) of the plan's kernel for `kind`.
cudaError_t cl_launch(const ClGeom &g, const FbArgs &a, cudaStream_t st, int kind, unsigned nclusters, bool bwd_layout)
{
    void *fn = cl_kernel(g, kind);
    if (!fn) return cudaErrorInvalidConfiguration;
    const size_t smem = cl_smem_bytes_impl(a.K, a.C, g, bwd_layout);
    cudaError_t e = cl_prepare(fn, g, smem);
    if (e != cudaSuccess) return e;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(nclusters * (unsigned)g.G);
    cfg.blockDim = dim3(g.NT);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    if (g.G > 1) {
        attr[0].id = cudaLaunchAttributeClusterDimension;
        attr[0].val.clusterDim.x = g.G;
        attr[0].val.clusterDim.y = 1;
        attr[0].val.clusterDim.z = 1;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
    }
    FbArgs aa = a;
    ClGeom gg = g;
    void *args[] = {&aa, &gg};
    prof_before(st);
    e = cudaLaunchKernelExC(&cfg, fn, args);
    prof_after(st);
    return e;
}

// How many clusters of the plan the GPU holds at once (G = 1: CTAs).
cudaError_t cl_occupancy(void *fn, const ClGeom &g, size_t smem, int *nclusters)
{
    cudaError_t e = cl_prepare(fn, g, smem);
    if (e != cudaSuccess) return e;
    if (g.G <= 1) {
        int nb = 0;
        e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&nb, fn, g.NT, smem);
        *nclusters = nb * device_sm_count();
        return e;
    }
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)g.G);
    cfg.blockDim = dim3(g.NT);
    cfg.dynamicSmemBytes = smem;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = g.G;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaOccupancyMaxActiveClusters(nclusters, fn, &cfg);
}

}  // namespace


// One candidate geometry: G CTAs, LPL transition lanes per label, LPW window
// lanes per label.  Returns false when it does not fit 1024 threads or shared
// memory.  *cost estimates the cycles of one position, calibrated on this part:
// the owner-transition chain is about 2.5x the sum of its dependent latencies
// (FP64 operation ~33 cycles, shared load ~55, shuffle level ~58, exchange
// ~230 + C*G/2, at most 830: it grows with the values sent and the CTAs they
// go to) plus
// ~12 cycles of issue per transition
// term; a window chunk of eight rows costs ~1000 cycles in context; every
// resident warp adds ~25 cycles of contention; register classes that spill pay
// extra (more above 512 threads).  The chain and the window warps run in
// parallel, the slower one sets the pace.
static bool cl_try(int K, int C, bool bwd, int G, int LPL, int LPW, ClGeom *out, double *cost)
{
    ClGeom g;
    g.G = G;
    if (G > C) return false;
    g.Cg = (C + G - 1) / G;
    if ((G - 1) * g.Cg >= C) return false;   // every CTA owns at least one label
    if (G > 16) return false;
    g.LPL = LPL;
    if (LPL < 1 || LPL > 32 || (LPL & (LPL - 1))) return false;
    const int npos = G > 1 ? G * (int)even_up(g.Cg) : C;   // exchange positions (labels plus padding)
    g.CPL = (npos + LPL - 1) / LPL;
    if (g.CPL > 32) return false;
    g.GP = (int)even_up((size_t)(npos > cl_cpl_bucket(g.CPL) * LPL ? npos : cl_cpl_bucket(g.CPL) * LPL));

    g.NWO = (g.Cg + 31) / 32;
    g.NWT = (g.Cg * LPL + 31) / 32;
    g.TS = G > 1 && g.NWT >= 4 ? 1 : 0;
    const int rows = K > 2 ? K - 2 : 1;   // window rows d = 3..K (forward), i = 1..K-2 (backward)
    g.LPW = LPW;
    if (LPW < 1 || LPW > 256 || (LPW & (LPW - 1)) || LPW > rows) return false;
    g.PW = g.LPW > 32 ? g.LPW / 32 : 1;
    // Row stride of the ring (doubles).  A half-warp's 64-bit window loads cover
    // 16/LPW labels x LPW consecutive rows when LPW < 16: a stride = 16/LPW
    // (mod 16) puts them in 16 distinct bank pairs.  With LPW >= 16 the 16 lanes
    // are rows of one label, and an odd stride does it.
    if (LPW >= 16) {
        g.RS = g.Cg | 1;
    } else {
        const int want = 16 / LPW;
        g.RS = g.Cg + (((want - g.Cg) % 16) + 16) % 16;
    }
    g.NWW = (g.Cg * g.LPW + 31) / 32;
    if (g.NWW < 1) g.NWW = 1;
    // window weights in registers when a lane's rows fit the kernel's register
    // array (max(CPL bucket, 16) doubles), read in buckets of 8, 16 or 32 rows;
    // the ring then carries zero rows on both sides for the rows past the window
    {
        const int nrw = K > 2 ? (K - 2 + LPW - 1) / LPW : 0;
        const int nu = cl_cpl_bucket(g.CPL) > 16 ? cl_cpl_bucket(g.CPL) : 16;
        g.NRB = (nrw > 0 && nrw <= nu) ? (nrw <= 8 ? 8 : nrw <= 16 ? 16 : 32) : 0;
        g.PAD = g.NRB > 0 && g.NRB * LPW + 2 > K ? g.NRB * LPW + 2 - K : 0;
    }
    g.NT = 32 * (g.NWO + g.NWT + g.NWW);
    if (g.NT > 1024) return false;
    const int maxt = cl_max_threads(g.NT);
    const int cpl = cl_cpl_bucket(g.CPL);
    if (cpl == 32 && maxt > 512) return false;
    if (cpl == 16 && maxt > 768) return false;
    const size_t smem = cl_smem_bytes_impl(K, C, g, bwd);
    if (smem > kSmemBudget) return false;
    auto lg2 = [](int v) {
        int l = 0;
        while ((1 << l) < v) ++l;
        return l;
    };
    const int R = (rows + LPW - 1) / LPW;
    const double chain =
        2.5 * (33 + (G > 1 ? 230 + (C * G < 1200 ? 0.5 * C * G : 600.0) : 40) + 55 + 33 * (1 + lg2(cpl)) +
               58 * lg2(LPL) + 150 + 12 * cpl);
    const double window = 1000.0 * ((R + 7) / 8) + 60 * lg2(LPW < 32 ? LPW : 32);
    double c = (chain > window ? chain : window) + 25.0 * (g.NT / 32);
    if (maxt > 512) c += 2000;                     // register classes that spill
    else if (cpl == 32 && maxt > 256) c += 600;
    *out = g;
    *cost = c;
    return true;
}

// Every feasible geometry with its cost, cheapest first (ties: the smaller
// cluster).  Cluster sizes are powers of two; extra = true adds 12 and 14 (the
// fallbacks when no power of two keeps enough clusters resident at once).
// SEMICRF_CL_PLAN="G,LPL,LPW" (0 = free choice for that field) restricts the
// search.
static bool cl_candidates(int K, int C, bool bwd, bool extra, std::vector<std::pair<double, ClGeom>> &out)
{
    int fG = 0, fL = 0, fW = 0;
    const char *env = getenv("SEMICRF_CL_PLAN");
    if (env && *env && sscanf(env, "%d,%d,%d", &fG, &fL, &fW) < 1) return false;
    const int pow2[] = {1, 2, 4, 8, 16}, more[] = {12, 14};
    const int *Gs = extra ? more : pow2;
    int nG = extra ? 2 : 5;
    if (fG > 0) {   // a forced cluster size is taken as given (any of 1..16)
        if (extra) return true;
        Gs = &fG;
        nG = 1;
    }
    for (int gi = 0; gi < nG; ++gi) {
        const int G = Gs[gi];
        for (int LPL = 1; LPL <= 32; LPL *= 2) {
            if (fL > 0 && LPL != fL) continue;
            for (int LPW = 1; LPW <= 256; LPW *= 2) {
                if (fW > 0 && LPW != fW) continue;
                ClGeom g;
                double cost;
                if (cl_try(K, C, bwd, G, LPL, LPW, &g, &cost)) out.push_back({cost, g});
            }
        }
    }
    std::stable_sort(out.begin(), out.end(),
                     [](const std::pair<double, ClGeom> &x, const std::pair<double, ClGeom> &y) {
                         return x.first < y.first;
                     });
    return true;
}

// The cheapest geometry by the cost model; the shape is unsupported if nothing fits.
bool cl_plan(int K, int C, bool bwd, ClGeom *out)
{
    std::vector<std::pair<double, ClGeom>> c;
    if (!cl_candidates(K, C, bwd, false, c) || c.empty()) return false;
    *out = c.front().second;
    return true;
}

// Clusters of this geometry the current device holds at once (path 0: fused
// launch, 1: forward, 2: backward), -1 when the query fails.
static int cl_resident(const ClGeom &g, int K, int C, int path)
{
    int n = -1;
    void *fn = cl_kernel(g, path == 0 ? kClFused : path == 1 ? kClFwd : kClBwd);
    const cudaError_t e = fn ? cl_occupancy(fn, g, cl_smem_bytes_impl(K, C, g, path != 1), &n)
                             : cudaErrorInvalidConfiguration;
    if (e != cudaSuccess) {
        cudaGetLastError();   // clear a failed query
        return -1;
    }
    return n;
}

// The geometry a launch of `need` concurrent clusters uses: the cheapest one of
// which the device holds `need` clusters at once (all chains of the launch then
// run side by side), trying the power-of-two cluster sizes first and 12 and 14
// after; if none does, the cheapest.  Cached per device and shape.
static bool cl_plan_resident(int K, int C, int path, int need, ClGeom *out)
{
    static std::mutex mu;
    static std::map<std::tuple<int, int, int, int, int>, ClGeom> cache;
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess) {
        cudaGetLastError();
        dev = -1;
    }
    const char *env = getenv("SEMICRF_CL_PLAN");
    const bool forced = env && *env;
    const auto key = std::make_tuple(K, C, path, need, dev);
    if (!forced) {
        std::lock_guard<std::mutex> lock(mu);
        auto it = cache.find(key);
        if (it != cache.end()) {
            *out = it->second;
            return true;
        }
    }
    const bool bwd = path != 1;
    std::vector<std::pair<double, ClGeom>> c;
    if (!cl_candidates(K, C, bwd, false, c) || c.empty()) return false;
    ClGeom pick = c.front().second;
    bool ok = forced || dev < 0 || need <= 1 || cl_resident(pick, K, C, path) >= need;
    for (size_t i = 1; !ok && i < c.size(); ++i)
        if (cl_resident(c[i].second, K, C, path) >= need) {
            pick = c[i].second;
            ok = true;
        }
    if (!ok) {
        std::vector<std::pair<double, ClGeom>> x;
        cl_candidates(K, C, bwd, true, x);
        for (size_t i = 0; !ok && i < x.size(); ++i)
            if (cl_resident(x[i].second, K, C, path) >= need) {
                pick = x[i].second;
                ok = true;
            }
    }
    *out = pick;
    if (!forced) {
        std::lock_guard<std::mutex> lock(mu);
        cache[key] = pick;
    }
    return true;
}

cudaError_t launch_cl_forward(const FbArgs &a, cudaStream_t st, bool recompute)
{
    ClGeom g;
    // the checkpoint recompute launches B*J clusters that queue by design
    if (!(recompute ? cl_plan(a.K, a.C, false, &g) : cl_plan_resident(a.K, a.C, 1, a.B, &g)))
        return cudaErrorInvalidConfiguration;
    return cl_launch(g, a, st, recompute ? kClFwdRecompute : kClFwd,
                     recompute ? (unsigned)a.B * (unsigned)a.J : (unsigned)a.B, false);
}

// One geometry for both chains (the backward layout is the larger of the two and
// fits both), chosen so that all 2B chains are resident at once when possible.
cudaError_t launch_cl_fused(const FbArgs &a, cudaStream_t st)
{
    ClGeom g;
    if (!cl_plan_resident(a.K, a.C, 0, 2 * a.B, &g)) return cudaErrorInvalidConfiguration;
    return cl_launch(g, a, st, kClFused, 2u * (unsigned)a.B, true);   // the larger (backward) layout
}

cudaError_t launch_cl_backward(const FbArgs &a, cudaStream_t st)
{
    ClGeom g;
    if (!cl_plan_resident(a.K, a.C, 2, a.B, &g)) return cudaErrorInvalidConfiguration;
    return cl_launch(g, a, st, kClBwd, (unsigned)a.B, true);
}

// The geometry a launch of B sequences uses for a path and how many such
// clusters fit at once: info = {G, NT, Cg, LPL, LPW, shared bytes, resident
// clusters (-1 when the CUDA query fails, e.g. without a GPU)}.
bool cl_plan_info(int K, int C, int B, int path, int32_t *info)
{
    ClGeom g;
    if (!cl_plan_resident(K, C, path, path == 0 ? 2 * B : B, &g)) return false;
    info[0] = g.G;
    info[1] = g.NT;
    info[2] = g.Cg;
    info[3] = g.LPL;
    info[4] = g.LPW;
    info[5] = (int32_t)cl_smem_bytes_impl(K, C, g, path != 1);
    info[6] = cl_resident(g, K, C, path);
    return true;
}

}  // namespace semicrf
