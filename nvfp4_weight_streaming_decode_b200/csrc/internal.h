// internal.h -- host-side plumbing shared by the library's translation units:
// status handling, argument checks, per-device state and the launch hooks
// the round builder uses.  Not part of the C ABI.
#pragma once
#include <cuda_runtime.h>
#include <stdint.h>

#include "nvfp4decode.h"
#include "layout.cuh"

namespace nvfp4 {

// Remember a failed CUDA call for nvfp4_last_cuda_error() and map it to a status.
int fail_cuda(cudaError_t e);
#define NVFP4_CUDA_TRY(expr)                          \
    do {                                              \
        cudaError_t e_ = (expr);                      \
        if (e_ != cudaSuccess) return ::nvfp4::fail_cuda(e_); \
    } while (0)

inline bool aligned16(const void* p) { return ((uintptr_t)p & 15u) == 0; }

int check_shape(int64_t N, int64_t K);
int check_m(int M);

struct Geometry {
    int64_t n_tiles, k_chunks, units;
};
Geometry geometry(int64_t N, int64_t K);

// Per-device state: SM count, split-K workspace and counters.  Created by
// the first call on a device, which must not be inside a stream capture.
struct DeviceState {
    int device = -1;
    int sm_count = 0;
    int max_warps = 0;        // capacity of the workspace, in warps
    float* partials = nullptr;        // the decode kernels' workspace slots (zeroed between launches)
    float* round_partials = nullptr;  // the persistent round kernel's
    unsigned* counters = nullptr;
};
int device_state(cudaStream_t stream, DeviceState** out);

// Launch one decode GEMM (kind 0) or fused gate/up (kind 1).  `pdl` marks the
// launch as a programmatic dependent of the previous work on the stream.
struct GemmArgs {
    int kind;
    const void* X;
    int M;
    const uint8_t* wq[2];
    const uint8_t* ws[2];
    float gscale[2];
    void* out;
    int64_t N, K;
};
int launch_gemm(const GemmArgs& a, cudaStream_t stream, bool pdl, DeviceState* ds);
int validate_gemm(const GemmArgs& a);
// Resolve a kernel variant (attributes, occupancy) ahead of a stream capture.
int prepare_kernel(DeviceState* ds, int kind, int M);

// Warps the launch of `a` would use on this device (before any clamping to the
// workspace), and the workspace floats each warp needs.
int gemm_launch_warps(const GemmArgs& a, DeviceState* ds, long long* warps);
size_t gemm_workspace_floats_per_warp();

// The persistent round: per-width preparation and the cooperative launch.
// The node table travels as the kernel's parameter block (host buffer of
// round_persistent_params_size() bytes, at most 360 nodes per launch).
int round_persistent_params_size();
int round_persistent_max_nodes();
size_t round_persistent_temp_floats(const GemmArgs* nodes, int n);
int round_persistent_build(const GemmArgs* nodes, int n, DeviceState* ds, float* temp, void* params_host,
                           int* count);
int round_persistent_prepare(DeviceState* ds, int M, int* grid);
int round_persistent_launch(void* params_host, unsigned* d_arrive, int M, int grid, cudaStream_t stream);

// Device-side status word (nonzero after a bounded wait gave up).  When it is
// nonzero the workspaces are cleared, the no-allocation entry point's included
// (noalloc_clear_scratch, a cudaError_t).
int read_and_clear_device_status(int* status);
cudaError_t noalloc_clear_scratch();

// The decode GEMM at verify widths (M = kVerifyMinM..kVerifyMaxM) on the
// tensor-memory path: geometry of a call, its launch, and its status word.
constexpr int kVerifyMinM = 9, kVerifyMaxM = 64;
struct VerifyGeometry {
    long long n_tiles32, n_groups, k_chunks, k_pairs, units, ctas;
    int nl, tmem_cols;
};
int verify_geometry(int M, int64_t N, int64_t K, int sm_count, VerifyGeometry* g);
int launch_verify(const void* X, int M, const uint8_t* wq, const uint8_t* ws, float gscale, float* Y, int64_t N,
                  int64_t K, cudaStream_t stream);
int read_and_clear_verify_status(unsigned* status);

// Status word of the grouped expert kernel (1 = an invalid route, 2 = a bounded wait gave up).
int read_and_clear_grouped_status(unsigned* status);

}  // namespace nvfp4
