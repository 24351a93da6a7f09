// fb_cluster_ts.cu -- the cluster kernels whose transition lanes form and send
// each position's value (plans with ClGeom::TS = 1), compiled apart from
// fb_cluster.cu so that the two sets of kernels build side by side.
#include "fb_cluster_dev.cuh"

namespace semicrf {

void *cl_kernel_ts(const ClGeom &g, int kind)
{
    const int cpl = cl_cpl_bucket(g.CPL), maxt = cl_max_threads(g.NT);
    SEMICRF_CL_TABLE(cl_kernel_ts1, true, kind)
    return nullptr;
}

}  // namespace semicrf
