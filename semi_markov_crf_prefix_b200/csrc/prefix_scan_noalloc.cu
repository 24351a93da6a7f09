// prefix_scan_noalloc.cu -- semicrf_prefix_scan_noalloc: the centring and prefix
// scan for callers that cannot hand the library any device memory beyond their
// inputs and outputs.
//
// Who needs it: code that is given only its input and output buffers (a plugin
// or custom-op interface with no workspace hook), or that runs under a fixed
// device-memory budget where a cudaMalloc could block on the device or fail at
// the wrong moment.  Such callers cannot size and pass the workspace that
// semicrf_prefix_scan asks for.
//
// How: the scan's scratch (one float64 partial sum per sequence, chunk and label,
// plus a status word) lives in the file-scope array g_noalloc_scratch below,
// 1 MiB + 256 bytes, which every GPU that loads the library keeps until the
// process exits.  Host code cannot use the array's name as a device address, so
// the first call on each device (with that device current) looks the address up
// with cudaGetSymbolAddress and caches it; that first call should come before any
// stream capture.  The address is kept for the life of the process: after a
// cudaDeviceReset on a device the entry point must not be used there again.  All
// calls share the one array and it keeps the last call's contents, so calls
// issued in order on one stream are safe, while calls that can overlap on the
// GPU (on different streams, or from different host threads) race on it and
// must be serialised by the caller.  The
// status word is cleared at the start of every call; the chunk sums are fully
// written before they are read.
#include <mutex>

#include "device_util.cuh"
#include "semicrf_internal.h"

namespace semicrf {

// Largest scratch the no-allocation scan may use: B * C float64 chunk sums must
// fit at least once (B * C <= 131072).
constexpr size_t kNoAllocScratchBytes = size_t(1) << 20;

namespace {

static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes + 256];

constexpr int kMaxDevices = 64;
void *g_scratch_addr[kMaxDevices] = {};
std::mutex g_scratch_mu;

// Device address of g_noalloc_scratch on the current device (looked up once).
cudaError_t scratch_address(void **out)
{
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> lock(g_scratch_mu);
    if (!g_scratch_addr[dev]) {
        void *p = nullptr;
        e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
        if (e != cudaSuccess) return e;
        g_scratch_addr[dev] = p;
    }
    *out = g_scratch_addr[dev];
    return cudaSuccess;
}

}  // namespace
}  // namespace semicrf

using namespace semicrf;

extern "C" semicrf_status semicrf_prefix_scan_noalloc(const semicrf_dims *dims, const float *x,
                                                      const int32_t *lengths, double *S, double *nu,
                                                      void *stream)
{
    prof_reset();
    if (!dims) return SEMICRF_ERR_INVALID_ARG;
    if (dims->B < 1 || dims->T < 1 || dims->C < 1) return SEMICRF_ERR_INVALID_ARG;
    if (dims->C > SEMICRF_MAX_C) return SEMICRF_ERR_UNSUPPORTED_SHAPE;
    const size_t per_chunk = (size_t)dims->B * dims->C * sizeof(double);
    if (per_chunk > kNoAllocScratchBytes) return SEMICRF_ERR_UNSUPPORTED_SHAPE;
    if (!x || !lengths || !S || !nu) return SEMICRF_ERR_INVALID_ARG;

    // same chunking as the workspace version, capped by the fixed scratch
    semicrf_dims sd = *dims;
    sd.K = 1;
    sd.ckpt_interval = 0;
    Layout lay;
    if (!make_layout(sd, SEMICRF_WS_SCAN, Plan(), &lay)) return SEMICRF_ERR_INVALID_ARG;
    int nch = lay.NCH;
    const int cap = (int)(kNoAllocScratchBytes / per_chunk);
    if (nch > cap) nch = cap;

    void *base = nullptr;
    if (scratch_address(&base) != cudaSuccess) return SEMICRF_ERR_CUDA;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (cudaMemsetAsync(base, 0, 256, st) != cudaSuccess) return SEMICRF_ERR_CUDA;

    ScanArgs a;
    a.B = dims->B;
    a.T = dims->T;
    a.C = dims->C;
    a.NCH = nch;
    a.x = x;
    a.lengths = lengths;
    a.S = S;
    a.nu = nu;
    a.status = static_cast<int32_t *>(base);
    a.part = reinterpret_cast<double *>(static_cast<unsigned char *>(base) + 256);
    int n = 0;
    if (launch_prefix_scan(a, st, &n) != cudaSuccess) return SEMICRF_ERR_CUDA;
    record_launches(n);
    return SEMICRF_OK;
}
