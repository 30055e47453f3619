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
    int mode;                 // NVFP4_ROUND_PERSISTENT or NVFP4_ROUND_CHAIN
    int n_chunks;             // persistent mode: launches per round (node tables of at most 360 nodes)
    void** params;            // persistent mode: host copies of the kernel parameter blocks, per chunk
    unsigned** d_arrive;      // persistent mode: per-chunk arrival counters (nodes + 1)
    float* d_temp;            // persistent mode: FP32 gate/up results of a fused node
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
    for (int c = 0; c < r->n_chunks; ++c) {
        if (r->params) free(r->params[c]);
        if (r->d_arrive && r->d_arrive[c]) cudaFree(r->d_arrive[c]);
    }
    free(r->params);
    free(r->d_arrive);
    if (r->d_temp) cudaFree(r->d_temp);
    free(r->descs);
    free(r);
}

}  // namespace

extern "C" int nvfp4_round_create(const nvfp4_gemm_desc* descs, int n, nvfp4_round** out)
{
    return nvfp4_round_create_ex(descs, n, NVFP4_ROUND_CHAIN, out);
}

extern "C" int nvfp4_round_create_ex(const nvfp4_gemm_desc* descs, int n, int mode, nvfp4_round** out)
{
    using namespace nvfp4;
    if (!descs || !out || n < 1) return NVFP4_ERR_ARG;
    if (mode != NVFP4_ROUND_PERSISTENT && mode != NVFP4_ROUND_CHAIN) return NVFP4_ERR_ARG;
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
    r->mode = mode;
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
    int grid = 0;
    if (st == NVFP4_OK && mode == NVFP4_ROUND_PERSISTENT) {
        for (int M = 1; st == NVFP4_OK && M <= kMaxM; ++M) st = round_persistent_prepare(ds, M, &grid);
        GemmArgs* args = (GemmArgs*)malloc(sizeof(GemmArgs) * (size_t)n);
        if (!args) st = NVFP4_ERR_ARG;
        for (int i = 0; st == NVFP4_OK && i < n; ++i) args[i] = args_of(r->descs[i], kMaxM);
        const size_t temp_floats = st == NVFP4_OK ? round_persistent_temp_floats(args, n) : 0;
        if (st == NVFP4_OK && temp_floats) {
            e = cudaMalloc(&r->d_temp, temp_floats * sizeof(float));
            if (e != cudaSuccess) st = fail_cuda(e);
        }
        // Chunks of descriptors whose expanded node tables fit one launch's parameter block.
        const int cap = round_persistent_max_nodes();
        r->params = (void**)calloc((size_t)n, sizeof(void*));
        r->d_arrive = (unsigned**)calloc((size_t)n, sizeof(unsigned*));
        if (!r->params || !r->d_arrive) st = NVFP4_ERR_ARG;
        for (int i0 = 0; st == NVFP4_OK && i0 < n;) {
            int i1 = i0, nodes = 0;
            while (i1 < n && nodes + 1 + (args[i1].kind == 1) <= cap) nodes += 1 + (args[i1++].kind == 1);
            const int c = r->n_chunks++;
            r->params[c] = malloc((size_t)round_persistent_params_size());
            if (!r->params[c]) {
                st = NVFP4_ERR_ARG;
                break;
            }
            int count = 0;
            st = round_persistent_build(args + i0, i1 - i0, ds, r->d_temp, r->params[c], &count);
            if (st != NVFP4_OK) break;
            e = cudaMalloc(&r->d_arrive[c], sizeof(unsigned) * (size_t)(count + 1));
            if (e == cudaSuccess) e = cudaMemset(r->d_arrive[c], 0, sizeof(unsigned) * (size_t)(count + 1));
            if (e != cudaSuccess) st = fail_cuda(e);
            i0 = i1;
        }
        if (st == NVFP4_OK) {
            e = cudaDeviceSynchronize();
            if (e != cudaSuccess) st = fail_cuda(e);
        }
        free(args);
    }
    for (int M = 1; st == NVFP4_OK && M <= kMaxM; ++M) {
        e = cudaStreamBeginCapture(r->stream, cudaStreamCaptureModeThreadLocal);
        if (e != cudaSuccess) {
            st = fail_cuda(e);
            break;
        }
        int lst = NVFP4_OK;
        if (mode == NVFP4_ROUND_PERSISTENT)
            for (int c = 0; c < r->n_chunks && lst == NVFP4_OK; ++c)
                lst = round_persistent_launch(r->params[c], r->d_arrive[c], M, grid, r->stream);
        else
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
