// round.cu -- the batch-wide decode round: a chain of decode GEMMs captured
// once per batch width M = 1..8 into CUDA graphs and replayed with one graph
// launch per round (ignis README, "The decode round": one round for all
// lanes, replayed from per-width CUDA graphs, widths 1..8).  Consecutive
// nodes are programmatic dependent launches, so each GEMM streams its
// weights while its predecessor drains (the "PDL decode chain" the README's
// credits name).
#include <cuda_runtime.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#include "internal.h"

struct nvfp4_round {
    int device;
    int n;
    nvfp4_gemm_desc* descs;
    cudaStream_t stream;
    cudaGraph_t graphs[nvfp4::kMaxM];
    cudaGraphExec_t execs[nvfp4::kMaxM];
    int nodes;
};

namespace {

nvfp4::GemmArgs args_of(const nvfp4_gemm_desc& d, int M)
{
    nvfp4::GemmArgs a = {};
    a.kind = d.kind == NVFP4_DESC_GATEUP_SILU ? 1 : (d.kind == NVFP4_DESC_GEMM ? 0 : -1);
    a.X = d.X;
    a.M = M;
    a.wq[0] = d.wq;
    a.ws[0] = d.ws;
    a.gscale[0] = d.gscale;
    a.wq[1] = d.wq2;
    a.ws[1] = d.ws2;
    a.gscale[1] = d.gscale2;
    a.out = d.out;
    a.N = d.N;
    a.K = d.K;
    return a;
}

void release(nvfp4_round* r)
{
    if (!r) return;
    for (int i = 0; i < nvfp4::kMaxM; ++i) {
        if (r->execs[i]) cudaGraphExecDestroy(r->execs[i]);
        if (r->graphs[i]) cudaGraphDestroy(r->graphs[i]);
    }
    if (r->stream) cudaStreamDestroy(r->stream);
    free(r->descs);
    free(r);
}

}  // namespace

extern "C" int nvfp4_round_create(const nvfp4_gemm_desc* descs, int n, nvfp4_round** out)
{
    using namespace nvfp4;
    if (!descs || !out || n < 1) return NVFP4_ERR_ARG;
    *out = nullptr;
    for (int i = 0; i < n; ++i) {
        const GemmArgs a = args_of(descs[i], kMaxM);
        const int st = validate_gemm(a);
        if (st != NVFP4_OK) return st;
    }
    nvfp4_round* r = (nvfp4_round*)calloc(1, sizeof(nvfp4_round));
    if (!r) return NVFP4_ERR_ARG;
    r->descs = (nvfp4_gemm_desc*)malloc(sizeof(nvfp4_gemm_desc) * (size_t)n);
    if (!r->descs) {
        free(r);
        return NVFP4_ERR_ARG;
    }
    memcpy(r->descs, descs, sizeof(nvfp4_gemm_desc) * (size_t)n);
    r->n = n;
    cudaError_t e = cudaGetDevice(&r->device);
    if (e == cudaSuccess) e = cudaStreamCreateWithFlags(&r->stream, cudaStreamNonBlocking);
    if (e != cudaSuccess) {
        release(r);
        return fail_cuda(e);
    }
    DeviceState* ds = nullptr;
    int st = device_state(r->stream, &ds);
    // Resolve every kernel (attributes, occupancy) outside the capture.
    for (int M = 1; st == NVFP4_OK && M <= kMaxM; ++M)
        for (int k = 0; st == NVFP4_OK && k < 2; ++k) st = prepare_kernel(ds, k, M);
    for (int M = 1; st == NVFP4_OK && M <= kMaxM; ++M) {
        e = cudaStreamBeginCapture(r->stream, cudaStreamCaptureModeThreadLocal);
        if (e != cudaSuccess) {
            st = fail_cuda(e);
            break;
        }
        int lst = NVFP4_OK;
        for (int i = 0; i < n && lst == NVFP4_OK; ++i)
            lst = launch_gemm(args_of(r->descs[i], M), r->stream, i > 0, ds);
        cudaGraph_t graph = nullptr;
        e = cudaStreamEndCapture(r->stream, &graph);
        r->graphs[M - 1] = graph;
        if (lst != NVFP4_OK) {
            st = lst;
            break;
        }
        if (e != cudaSuccess) {
            st = fail_cuda(e);
            break;
        }
        e = cudaGraphInstantiate(&r->execs[M - 1], graph, 0);
        if (e != cudaSuccess) {
            st = fail_cuda(e);
            break;
        }
        if (M == 1) {
            size_t count = 0;
            e = cudaGraphGetNodes(graph, nullptr, &count);
            if (e != cudaSuccess) {
                st = fail_cuda(e);
                break;
            }
            r->nodes = (int)count;
        }
    }
    if (st == NVFP4_OK) {
        e = cudaStreamSynchronize(r->stream);
        if (e != cudaSuccess) st = fail_cuda(e);
    }
    if (st != NVFP4_OK) {
        release(r);
        return st;
    }
    *out = r;
    return NVFP4_OK;
}

extern "C" int nvfp4_round_nodes(const nvfp4_round* r, int* nodes)
{
    if (!r || !nodes) return NVFP4_ERR_ARG;
    *nodes = r->nodes;
    return NVFP4_OK;
}

extern "C" int nvfp4_round_replay(nvfp4_round* r, int M, nvfp4_stream_t stream)
{
    if (!r) return NVFP4_ERR_ARG;
    int st = nvfp4::check_m(M);
    if (st != NVFP4_OK) return st;
    NVFP4_CUDA_TRY(cudaGraphLaunch(r->execs[M - 1], (cudaStream_t)stream));
    return NVFP4_OK;
}

extern "C" int nvfp4_round_replay_host(nvfp4_round* r, int M, const void* x_host, void* x_dev, size_t x_bytes,
                                       const void* y_dev, void* y_host, size_t y_bytes, nvfp4_stream_t stream)
{
    if (!r) return NVFP4_ERR_ARG;
    if ((x_bytes && (!x_host || !x_dev)) || (y_bytes && (!y_host || !y_dev))) return NVFP4_ERR_ARG;
    int st = nvfp4::check_m(M);
    if (st != NVFP4_OK) return st;
    cudaStream_t s = (cudaStream_t)stream;
    if (x_bytes) NVFP4_CUDA_TRY(cudaMemcpyAsync(x_dev, x_host, x_bytes, cudaMemcpyHostToDevice, s));
    NVFP4_CUDA_TRY(cudaGraphLaunch(r->execs[M - 1], s));
    if (y_bytes) NVFP4_CUDA_TRY(cudaMemcpyAsync(y_host, y_dev, y_bytes, cudaMemcpyDeviceToHost, s));
    return NVFP4_OK;
}

extern "C" int nvfp4_round_destroy(nvfp4_round* r)
{
    release(r);
    return NVFP4_OK;
}
