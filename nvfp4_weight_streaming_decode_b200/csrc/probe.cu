// probe.cu -- nvfp4_stream_read: a read-only stream of device memory, the
// bandwidth the decode GEMM's weight stream is measured against beside the
// copy (read + write) figure.  The round is meant to run at the card's read
// bandwidth (ignis README, section "The decode round"), so its own read-only
// ceiling is the natural second denominator.
//
// Each thread reads 16-byte words with the cache-streaming hint, four strided
// words in flight per step, and folds them into one 32-bit XOR; a CTA writes
// the XOR of its threads' values.  The XOR over all CTAs' words equals the XOR
// of every 32-bit word of the buffer, so the host can check that every byte
// was read and the compiler cannot drop a load.
#include <cuda_runtime.h>
#include <stdint.h>

#include "internal.h"

namespace nvfp4 {
namespace {

constexpr int kProbeThreads = 512;
constexpr int kProbeMaxCtas = 1 << 20;

__global__ void __launch_bounds__(kProbeThreads) stream_read_kernel(const uint4* __restrict__ buf, long long n16,
                                                                    uint32_t* __restrict__ out)
{
    const long long stride = (long long)gridDim.x * kProbeThreads;
    long long i = (long long)blockIdx.x * kProbeThreads + threadIdx.x;
    uint32_t acc = 0u;
    for (; i + 3 * stride < n16; i += 4 * stride) {
        const uint4 a = __ldcs(buf + i);
        const uint4 b = __ldcs(buf + i + stride);
        const uint4 c = __ldcs(buf + i + 2 * stride);
        const uint4 d = __ldcs(buf + i + 3 * stride);
        acc ^= a.x ^ a.y ^ a.z ^ a.w ^ b.x ^ b.y ^ b.z ^ b.w ^ c.x ^ c.y ^ c.z ^ c.w ^ d.x ^ d.y ^ d.z ^ d.w;
    }
    for (; i < n16; i += stride) {
        const uint4 a = __ldcs(buf + i);
        acc ^= a.x ^ a.y ^ a.z ^ a.w;
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) acc ^= __shfl_xor_sync(0xffffffffu, acc, o);
    __shared__ uint32_t warp_acc[kProbeThreads / 32];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (lane == 0) warp_acc[warp] = acc;
    __syncthreads();
    if (warp == 0) {
        acc = lane < kProbeThreads / 32 ? warp_acc[lane] : 0u;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) acc ^= __shfl_xor_sync(0xffffffffu, acc, o);
        if (lane == 0) out[blockIdx.x] = acc;
    }
}

}  // namespace
}  // namespace nvfp4

extern "C" int nvfp4_stream_read(const void* buf, size_t bytes, uint32_t* out, int ctas, nvfp4_stream_t stream)
{
    using namespace nvfp4;
    if (!buf || !out) return NVFP4_ERR_ARG;
    if (ctas < 1 || ctas > kProbeMaxCtas) return NVFP4_ERR_ARG;
    if (bytes == 0 || bytes % 16 != 0 || bytes > ((size_t)1 << 50)) return NVFP4_ERR_SHAPE;
    if (!aligned16(buf) || ((uintptr_t)out & 3u) != 0) return NVFP4_ERR_ALIGN;
    stream_read_kernel<<<ctas, kProbeThreads, 0, (cudaStream_t)stream>>>(static_cast<const uint4*>(buf),
                                                                        (long long)(bytes / 16), out);
    NVFP4_CUDA_TRY(cudaGetLastError());
    return NVFP4_OK;
}
