// exp_tables.cu -- exp(S) for every position and label, split into an exact power
// of two and a bounded mantissa:  S = ln2 * m + s,  |s| <= ln2/2,
//   tES = exp(s),  tIES = exp(-s),  tM = m.
// The recursions then form exp(S + ln2 * (r - k)) = tES * 2^(m + r - k) and its
// inverse with one multiply by an exactly constructed power of two, so no
// exponential or division sits inside the sequential loops, and every pass that
// reads the tables (forward, recompute, backward) sees identical bits.
// One fully parallel, HBM-bound pass (8 bytes read, 20 bytes written per entry).
#include <math.h>

#include "device_util.cuh"
#include "semicrf_internal.h"

namespace semicrf {
namespace {

__global__ void exp_tables_kernel(FbArgs a)
{
    const size_t n = (size_t)a.B * (a.T + 1) * a.C;
    for (size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += (size_t)gridDim.x * blockDim.x) {
        const double S = a.S[i];
        const double mr = rint(S * (1.0 / kLn2));
        const double s = fma(-mr, kLn2, S);
        a.tES[i] = exp(s);
        a.tIES[i] = exp(-s);
        a.tM[i] = (int32_t)mr;
    }
}

}  // namespace

cudaError_t launch_exp_tables(const FbArgs &a, cudaStream_t st)
{
    const size_t n = (size_t)a.B * (a.T + 1) * a.C;
    int blocks = (int)((n + 255) / 256);
    if (blocks > device_sm_count() * 8) blocks = device_sm_count() * 8;
    prof_before(st);
    exp_tables_kernel<<<blocks, 256, 0, st>>>(a);
    prof_after(st);
    return cudaGetLastError();
}

}  // namespace semicrf
