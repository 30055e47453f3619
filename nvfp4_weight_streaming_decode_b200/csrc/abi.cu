// abi.cu -- status codes, argument checks and small queries of the C ABI.
#include <cuda_runtime.h>
#include <stdint.h>

#include "internal.h"
#include "layout.cuh"

namespace nvfp4 {

static thread_local int t_last_cuda_error = 0;

int fail_cuda(cudaError_t e)
{
    t_last_cuda_error = (int)e;
    cudaGetLastError();  // clear a sticky-free error so the next call starts clean
    return NVFP4_ERR_CUDA;
}

int check_m(int M) { return (M >= 1 && M <= kMaxM) ? NVFP4_OK : NVFP4_ERR_M; }

int check_shape(int64_t N, int64_t K)
{
    if (N < 1 || K < 16 || (K % 16) != 0) return NVFP4_ERR_SHAPE;
    // keep every byte offset and element index well inside int64
    if (N > ((int64_t)1 << 31) || K > ((int64_t)1 << 31) || (N / kTileN + 1) * (K / kChunkK + 1) > ((int64_t)1 << 40))
        return NVFP4_ERR_SHAPE;
    return NVFP4_OK;
}

Geometry geometry(int64_t N, int64_t K)
{
    Geometry g;
    g.n_tiles = (N + kTileN - 1) / kTileN;
    g.k_chunks = (K + kChunkK - 1) / kChunkK;
    g.units = g.n_tiles * g.k_chunks;
    return g;
}

}  // namespace nvfp4

extern "C" const char* nvfp4_status_string(int status)
{
    switch (status) {
    case NVFP4_OK: return "ok";
    case NVFP4_ERR_ARG: return "invalid argument (NULL pointer, bad kind or count)";
    case NVFP4_ERR_M: return "M out of range for this entry point (1..8; nvfp4_gemm_decode also takes 9..64)";
    case NVFP4_ERR_SHAPE: return "bad shape: need N >= 1, K >= 16, K % 16 == 0";
    case NVFP4_ERR_ALIGN: return "device pointer not 16-byte aligned";
    case NVFP4_ERR_BAD_SCALE: return "scale plane holds an E4M3 NaN code (0x7F or 0xFF)";
    case NVFP4_ERR_CUDA: return "CUDA runtime error (see nvfp4_last_cuda_error)";
    case NVFP4_ERR_CAPTURE: return "first use of the device inside a stream capture";
    case NVFP4_ERR_DEVICE: return "a kernel's bounded wait gave up (see nvfp4_device_status)";
    case NVFP4_ERR_SCRATCH: return "needs more scratch than the no-alloc entry point's static array holds";
    default: return "unknown status";
    }
}

extern "C" int nvfp4_last_cuda_error(void) { return nvfp4::t_last_cuda_error; }

extern "C" int nvfp4_device_status(void)
{
    int v = 0;
    int st = nvfp4::read_and_clear_device_status(&v);
    if (st != NVFP4_OK) return st;
    unsigned vv = 0;
    st = nvfp4::read_and_clear_verify_status(&vv);
    if (st != NVFP4_OK) return st;
    unsigned vg = 0;
    st = nvfp4::read_and_clear_grouped_status(&vg);
    if (st != NVFP4_OK) return st;
    // verify kernel: 8 = a streaming warp gave up, 16 = its MMA thread did;
    // grouped kernel: 32 = an invalid route, 64 = a bounded wait gave up
    return v | (int)(vv << 3) | (int)(vg << 5);
}

extern "C" int nvfp4_version(void) { return 100; }
