// noalloc.cu -- nvfp4_gemm_decode_noalloc: the decode GEMM for callers that
// must not allocate device memory (an engine whose device-memory plan is
// fixed at load, a plugin whose host owns all device memory, a path that
// cannot take cudaMalloc's implicit synchronisation).  The split-K scratch
// that nvfp4_gemm_decode allocates on first use lives here instead, in a
// file-scope static device array that every GPU loading the library holds
// until exit.  The kernel and its launch are those of nvfp4_gemm_decode.
#include <cuda_runtime.h>
#include <stdint.h>

#include <mutex>

#include "internal.h"

namespace nvfp4 {
namespace {

// Capacity in warps: 160 SMs x 16 warps.  Each warp owns two partial-sum
// slots of 512 floats (4 KiB) and one arrival counter.
constexpr long long kNoAllocMaxWarps = 2560;
constexpr size_t kNoAllocPartialFloats = (size_t)kNoAllocMaxWarps * 1024;  // 10 MiB

static __device__ __align__(256) float g_noalloc_partials[kNoAllocPartialFloats];
static __device__ __align__(256) unsigned g_noalloc_counters[kNoAllocMaxWarps];

struct NoAllocDevice {
    int ready = 0;
    int sm_count = 0;
    float* partials = nullptr;     // device address of g_noalloc_partials
    unsigned* counters = nullptr;  // device address of g_noalloc_counters
};

std::mutex g_noalloc_mu;
NoAllocDevice g_noalloc_dev[64];

// Once per device, with that device current: the arrays' device addresses
// (in host code the array names are host-side stand-ins, not addresses).
// Resolving a symbol may load the module, which a stream capture does not
// allow, so the first call on a device is refused while `stream` is captured.
int noalloc_setup(int dev, cudaStream_t stream, NoAllocDevice** out)
{
    std::lock_guard<std::mutex> lock(g_noalloc_mu);
    NoAllocDevice& d = g_noalloc_dev[dev];
    if (!d.ready) {
        cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
        NVFP4_CUDA_TRY(cudaStreamIsCapturing(stream, &cs));
        if (cs != cudaStreamCaptureStatusNone) return NVFP4_ERR_CAPTURE;
        if (gemm_workspace_floats_per_warp() * kNoAllocMaxWarps > kNoAllocPartialFloats)
            return NVFP4_ERR_SCRATCH;
        void* p = nullptr;
        NVFP4_CUDA_TRY(cudaGetSymbolAddress(&p, g_noalloc_partials));
        d.partials = static_cast<float*>(p);
        p = nullptr;
        NVFP4_CUDA_TRY(cudaGetSymbolAddress(&p, g_noalloc_counters));
        d.counters = static_cast<unsigned*>(p);
        NVFP4_CUDA_TRY(cudaDeviceGetAttribute(&d.sm_count, cudaDevAttrMultiProcessorCount, dev));
        d.ready = 1;
    }
    *out = &d;
    return NVFP4_OK;
}

}  // namespace

// After a bounded wait gave up, slots may be left unconsumed: zero the
// array on every device whose address was resolved (current device restored).
cudaError_t noalloc_clear_scratch()
{
    std::lock_guard<std::mutex> lock(g_noalloc_mu);
    int cur = 0;
    cudaError_t e = cudaGetDevice(&cur);
    if (e != cudaSuccess) return e;
    for (int dev = 0; dev < 64; ++dev) {
        if (!g_noalloc_dev[dev].ready) continue;
        e = cudaSetDevice(dev);
        if (e == cudaSuccess) e = cudaMemset(g_noalloc_dev[dev].partials, 0, kNoAllocPartialFloats * sizeof(float));
        if (e != cudaSuccess) break;
    }
    const cudaError_t e2 = cudaSetDevice(cur);
    return e != cudaSuccess ? e : e2;
}

}  // namespace nvfp4

using namespace nvfp4;

extern "C" int nvfp4_gemm_decode_noalloc(const void* X, int M, const uint8_t* wq_dev, const uint8_t* ws_dev,
                                         float gscale, float* Y, int64_t N, int64_t K, nvfp4_stream_t stream)
{
    GemmArgs a = {};
    a.kind = 0;
    a.X = X;
    a.M = M;
    a.wq[0] = wq_dev;
    a.ws[0] = ws_dev;
    a.gscale[0] = gscale;
    a.out = Y;
    a.N = N;
    a.K = K;
    if (M > kMaxM) return NVFP4_ERR_M;  // decode lanes only
    int st = validate_gemm(a);
    if (st != NVFP4_OK) return st;
    int dev = 0;
    NVFP4_CUDA_TRY(cudaGetDevice(&dev));
    if (dev < 0 || dev >= 64) return NVFP4_ERR_ARG;
    NoAllocDevice* d = nullptr;
    st = noalloc_setup(dev, (cudaStream_t)stream, &d);
    if (st != NVFP4_OK) return st;
    DeviceState ds;
    ds.device = dev;
    ds.sm_count = d->sm_count;
    ds.max_warps = (int)kNoAllocMaxWarps;
    ds.partials = d->partials;
    ds.counters = d->counters;
    long long warps = 0;
    st = gemm_launch_warps(a, &ds, &warps);
    if (st != NVFP4_OK) return st;
    // A launch that would use more warps than the array holds runs with fewer
    // (launch_gemm clamps the grid to ds.max_warps; the split-K partition stays
    // correct for any warp count), so no shape is refused for its size.
    if (warps > kNoAllocMaxWarps) warps = kNoAllocMaxWarps;
    // The array keeps the last call's contents: the arrival counters must start at zero.
    NVFP4_CUDA_TRY(cudaMemsetAsync(d->counters, 0, (size_t)warps * sizeof(unsigned), (cudaStream_t)stream));
    return launch_gemm(a, (cudaStream_t)stream, false, &ds);
}
