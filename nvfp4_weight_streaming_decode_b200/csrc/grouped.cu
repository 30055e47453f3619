// grouped.cu -- grouped NVFP4 expert decode: one launch over a route list.
//
// ignis, "Models and artifacts" (the model table): Flash-Next is a mixture of
// experts, 512 routed experts per layer and ten chosen per token.  Decoding M
// lanes therefore multiplies each lane's activation by the ten expert
// matrices its router picked.  This kernel does one projection of that step
// for all lanes in one launch:
//     Y[m][t][n] = gscale_e * sum_k x[k] * e2m1(q_e[n][k]) * e4m3(s_e[n][k/16]),
//     e = route[m][t],  x = X[m] (shared input) or X[m*T + t] (one per route),
// with every expert matrix in the NVFP4 device layout of the decode GEMM.
//
// Weight streaming as in the decode GEMM: an expert picked by several lanes
// is read once for all of them.  Each CTA groups the route list the same
// deterministic way -- valid routes sorted by (expert, route position), runs
// of one expert cut into groups of at most 8 rows (the MMA's lane side) --
// and the selected groups' units are concatenated into one virtual matrix
// that the warps split evenly (stream-K, at least one 4-unit stage per warp),
// each block of rows coming from its own expert's planes and its own X rows.  Split-K partial sums are combined
// by the last contributor in warp order, as in the decode GEMM.  Routes whose
// expert id is outside 0..E-1, or whose planes are not 16-byte aligned, give
// zero rows and set a device status bit.  Every wait is bounded; no CTA waits
// for another.
#include <cuda_runtime.h>
#include <stdint.h>

#include <mutex>

#include "async.cuh"
#include "dequant.cuh"
#include "internal.h"
#include "layout.cuh"

namespace nvfp4 {

__device__ unsigned int g_grouped_status;

namespace {

constexpr int kGWarps = 16;     // one CTA of 16 warps per SM
static_assert(kGWarps * 32 >= 4 * NVFP4_GROUPED_MAX_ROUTES, "grouping counts each route with four threads");
constexpr int kGStages = 3;     // per-warp ring depth
constexpr int kGUPS = 4;        // units per stage (a stage crossing to the next expert takes one copy per part)
constexpr int kGStage = kGUPS * kUnitBytes;
constexpr int kGSlot = 256;     // a partial: 32 lanes x 8 floats
// Units per warp at least: a small call (M = 1: ten experts) runs on fewer
// warps, each with one full stage in flight and fewer split-K partials per
// tile (measured at M = 1, T = 10 on 768 x 2,048 experts: 1 unit 11.0 us,
// 2-3 units 10.8-10.9, 4 units 9.4, 5-6 units 11.0-11.3, 8 units 11.3).
constexpr int kGMinUnits = kGUPS;
constexpr int kGMaxTiles = 4096;  // 32-row tiles per expert (N <= 131,072)

struct GParams {
    const uint16_t* X;
    int x_per_route;
    const int32_t* route;  // [M][T]
    int M, T;
    const nvfp4_expert* experts;  // [E]
    int E;
    float* Y;  // [M][T][N]
    long long N, K;
    int KC, tiles;
    long long UE;  // units per expert
    float* partials;
    unsigned* counters;
};

__device__ __forceinline__ long long g_range_begin(long long u, long long tw, long long w) { return u * w / tw; }
__device__ __forceinline__ long long g_range_owner(long long u, long long tw, long long x)
{
    return ((x + 1) * tw - 1) / u;
}

// 32 bytes of X (two 16-byte loads) when `pred`, zeros otherwise.
__device__ __forceinline__ void g_ld_x32(const void* p, bool pred, uint32_t (&x)[8])
{
    asm volatile(
        "{\n .reg .pred q;\n setp.ne.u32 q, %9, 0;\n"
        " mov.b32 %0, 0; mov.b32 %1, 0; mov.b32 %2, 0; mov.b32 %3, 0;\n"
        " mov.b32 %4, 0; mov.b32 %5, 0; mov.b32 %6, 0; mov.b32 %7, 0;\n"
        " @q ld.global.nc.v4.u32 {%0,%1,%2,%3}, [%8];\n"
        " @q ld.global.nc.v4.u32 {%4,%5,%6,%7}, [%8+16];\n}"
        : "=r"(x[0]), "=r"(x[1]), "=r"(x[2]), "=r"(x[3]), "=r"(x[4]), "=r"(x[5]), "=r"(x[6]), "=r"(x[7])
        : "l"(p), "r"((uint32_t)pred));
}

// The same without `volatile`, so the fast path's four loads can be issued
// together (X is never written while the kernel runs).
__device__ __forceinline__ void g_ld_x32_nv(const void* p, bool pred, uint32_t (&x)[8])
{
    asm("{\n .reg .pred q;\n setp.ne.u32 q, %9, 0;\n"
        " mov.b32 %0, 0; mov.b32 %1, 0; mov.b32 %2, 0; mov.b32 %3, 0;\n"
        " mov.b32 %4, 0; mov.b32 %5, 0; mov.b32 %6, 0; mov.b32 %7, 0;\n"
        " @q ld.global.nc.v4.u32 {%0,%1,%2,%3}, [%8];\n"
        " @q ld.global.nc.v4.u32 {%4,%5,%6,%7}, [%8+16];\n}"
        : "=r"(x[0]), "=r"(x[1]), "=r"(x[2]), "=r"(x[3]), "=r"(x[4]), "=r"(x[5]), "=r"(x[6]), "=r"(x[7])
        : "l"(p), "r"((uint32_t)pred));
}

// The grouping every CTA computes (shared memory).
struct GroupTable {
    int n_groups;
    int sorted[NVFP4_GROUPED_MAX_ROUTES];    // valid route positions (m*T + t), sorted by (expert, position)
    int g_expert[NVFP4_GROUPED_MAX_ROUTES];  // per group: expert id
    int g_first[NVFP4_GROUPED_MAX_ROUTES];   // per group: its first index into `sorted`
    int g_rows[NVFP4_GROUPED_MAX_ROUTES];    // per group: rows, 1..8
    int start[NVFP4_GROUPED_MAX_ROUTES];     // per sorted position: 1 if it starts a group
    int exp[NVFP4_GROUPED_MAX_ROUTES];       // per route: its expert, or -1 (no expert / invalid)
    // per route: its expert's planes and scale, read once while grouping, so that
    // the copies and the epilogue need no further read of the expert table
    const uint8_t* r_wq[NVFP4_GROUPED_MAX_ROUTES];
    const uint8_t* r_ws[NVFP4_GROUPED_MAX_ROUTES];
    float r_gs[NVFP4_GROUPED_MAX_ROUTES];
};

__device__ __forceinline__ bool expert_ok(const nvfp4_expert& ex)
{
    return ex.wq && ex.ws && (((uintptr_t)ex.wq | (uintptr_t)ex.ws) & 15u) == 0;
}

// Group the routes: valid ones sorted by (expert, position), each expert's run
// cut every 8 rows.  All threads of the CTA call it; the result is the same in
// every CTA.
__device__ void build_groups(const GParams& p, GroupTable& gt)
{
    const int R = p.M * p.T;
    const int tid = threadIdx.x;
    if (tid < R) {
        const int e = p.route[tid];
        bool ok = e >= 0 && e < p.E;
        if (ok) {
            const nvfp4_expert ex = p.experts[e];
            ok = expert_ok(ex);
            gt.r_wq[tid] = ex.wq;
            gt.r_ws[tid] = ex.ws;
            gt.r_gs[tid] = ex.gscale;
        }
        gt.exp[tid] = ok ? e : -1;
    }
    // every thread sees the count of valid routes
    const int nv = __syncthreads_count(tid < R && gt.exp[tid] >= 0);
    // Route r's rank among the valid routes (by expert, then position) and where its
    // expert's run starts, counted by the four threads 4r..4r+3 over every fourth route
    // and summed across the quad.
    {
        const int r = tid >> 2, part = tid & 3;
        const int e = r < R ? gt.exp[r] : -1;
        int rank = 0, run = 0;
        if (e >= 0) {
            for (int q = part; q < R; q += 4) {
                const int eq = gt.exp[q];
                if (eq < 0) continue;
                if (eq < e || (eq == e && q < r)) ++rank;
                if (eq < e) ++run;
            }
        }
        rank += __shfl_xor_sync(0xffffffffu, rank, 1);
        run += __shfl_xor_sync(0xffffffffu, run, 1);
        rank += __shfl_xor_sync(0xffffffffu, rank, 2);
        run += __shfl_xor_sync(0xffffffffu, run, 2);
        if (e >= 0 && part == 0) {
            gt.sorted[rank] = r;
            gt.start[rank] = (rank - run) % 8 == 0 ? 1 : 0;
        }
    }
    __syncthreads();
    // Group index of each sorted position: the count of group starts up to it
    // (a ballot prefix within each warp, then across the first four warps).
    __shared__ int warp_starts[NVFP4_GROUPED_MAX_ROUTES / 32];
    const bool st = tid < nv && gt.start[tid] != 0;
    const unsigned ballot = __ballot_sync(0xffffffffu, st);
    const int lane = tid & 31, w = tid >> 5;
    if (w < NVFP4_GROUPED_MAX_ROUTES / 32 && lane == 0) warp_starts[w] = __popc(ballot);
    __syncthreads();
    if (st) {
        int g = __popc(ballot & ((1u << lane) - 1u));
        for (int k = 0; k < w; ++k) g += warp_starts[k];
        gt.g_expert[g] = gt.exp[gt.sorted[tid]];
        gt.g_first[g] = tid;
    }
    if (tid == 0) {
        int ng = 0;
        for (int k = 0; k < NVFP4_GROUPED_MAX_ROUTES / 32; ++k) ng += warp_starts[k];
        gt.n_groups = ng;
    }
    __syncthreads();
    // a group runs to the next group's first position (or to the end)
    if (tid < gt.n_groups) gt.g_rows[tid] = (tid + 1 < gt.n_groups ? gt.g_first[tid + 1] : nv) - gt.g_first[tid];
    __syncthreads();
}

__global__ void __launch_bounds__(kGWarps * 32, 1) grouped_kernel(const GParams p)
{
    extern __shared__ __align__(128) uint8_t gsm[];
    __shared__ GroupTable gt;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const long long gw = (long long)blockIdx.x * kGWarps + warp;
    const uint8_t* ring = gsm + warp * (kGStages * kGStage);
    const uint32_t ring_s = smem_addr(gsm) + warp * (kGStages * kGStage);
    const uint32_t bar_s = smem_addr(gsm + kGWarps * kGStages * kGStage) + warp * kGStages * 8;
    if (lane == 0) {
        for (int s = 0; s < kGStages; ++s) mbar_init(bar_s + 8 * s);
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    __syncwarp();
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    // the route list and X come from earlier kernels
    asm volatile("griddepcontrol.wait;" ::: "memory");
    build_groups(p, gt);

    // rows of routes without a valid expert are zero (CTA 0); a bad id or misaligned planes is flagged
    if (blockIdx.x == 0) {
        for (int q = 0; q < p.M * p.T; ++q) {
            if (gt.exp[q] >= 0) continue;
            if (threadIdx.x == 0 && p.route[q] >= 0) atomicOr(&g_grouped_status, 1u);
            for (long long nn = threadIdx.x; nn < p.N; nn += blockDim.x) p.Y[q * p.N + nn] = 0.f;
        }
    }

    const long long U = gt.n_groups * p.UE;
    // at least kGMinUnits units per warp: for small calls fewer warps, each with
    // more copies in flight, and fewer split-K partials per tile
    const long long TWmax = (long long)gridDim.x * kGWarps;
    const long long TWu = (U + kGMinUnits - 1) / kGMinUnits;
    const long long TW = TWmax < TWu ? TWmax : TWu;
    if (gw >= TW) return;  // (no CTA-wide barrier follows)
    const long long KC = p.KC, UE = p.UE;
    const long long u0 = g_range_begin(U, TW, gw), u1 = g_range_begin(U, TW, gw + 1);
    const int n = (int)(u1 - u0);
    const int n_stages = (n + kGUPS - 1) / kGUPS;
    const uint64_t pol = evict_first_policy();

    // issue cursor (lane 0): group and unit within the expert of the next stage
    int ig = (int)(u0 / UE);
    long long iul = u0 - ig * UE;
    auto issue = [&](int j) {  // stage j: units [u0 + 4j, ...), in stage order
        const int slot = j % kGStages;
        const uint32_t bar = bar_s + 8 * slot;
        const int rem = n - j * kGUPS;
        const int cnt = rem < kGUPS ? rem : kGUPS;
        mbar_expect_tx(bar, (uint32_t)(cnt * kUnitBytes));
        const uint32_t dst = ring_s + slot * kGStage;
        for (int v = 0; v < cnt;) {
            // the longest run of this stage's units within one expert
            const long long left = UE - iul;
            const int part = (long long)(cnt - v) < left ? cnt - v : (int)left;
            const int r0 = gt.sorted[gt.g_first[ig]];  // a route of this group: its expert's planes
            bulk_load(dst + v * kUnitQ, gt.r_wq[r0] + iul * kUnitQ, part * kUnitQ, bar, pol);
            bulk_load(dst + kGUPS * kUnitQ + v * kUnitS, gt.r_ws[r0] + iul * kUnitS, part * kUnitS, bar, pol);
            v += part;
            iul += part;
            if (iul == UE) {
                iul = 0;
                ++ig;
            }
        }
    };
    if (lane == 0) {
        const int npre = n_stages < kGStages ? n_stages : kGStages;
        for (int j = 0; j < npre; ++j) issue(j);
    }

    const int g8 = lane >> 2, t = lane & 3;
    int grp = (int)(u0 / UE);
    long long ul = u0 - grp * UE;
    int tile = (int)(ul / KC);
    int chunk = (int)(ul - (long long)tile * KC);
    // per-group state: this lane's X row, the group's rows and scale
    int rows = 0, first = 0;
    float gscale = 0.f;
    const uint16_t* xrow = p.X;
    auto set_group = [&]() {
        rows = gt.g_rows[grp];
        first = gt.g_first[grp];
        gscale = gt.r_gs[gt.sorted[first]];
        // past the group's rows a lane loads its first row, which feeds only dropped output columns
        const int pos = gt.sorted[first + (g8 < rows ? g8 : 0)];
        xrow = p.X + (long long)(p.x_per_route ? pos : pos / p.T) * p.K;
    };
    set_group();

    float acc[2][4];
#pragma unroll
    for (int r = 0; r < 2; ++r)
#pragma unroll
        for (int i = 0; i < 4; ++i) acc[r][i] = 0.f;
    const long long first_tg = grp * (long long)p.tiles + tile;
    int i = 0;  // units consumed
    for (int js = 0; js < n_stages; ++js) {
        const int slot = js % kGStages;
        if (!warp_wait(bar_s + 8 * slot, (uint32_t)((js / kGStages) & 1))) {
            // give up: flag it, then wait (bounded) for the copies still in flight
            if (lane == 0) atomicOr(&g_grouped_status, 2u);
            for (int j2 = js; j2 < n_stages && j2 < js + kGStages; ++j2)
                warp_wait(bar_s + 8 * (j2 % kGStages), (uint32_t)((j2 / kGStages) & 1));
            return;
        }
        const uint8_t* st = ring + slot * kGStage;
        if (n - i > kGUPS && (int)KC - 1 - chunk >= kGUPS) {
            // Fast path: four units inside one tile (so one group), none ending the
            // tile or the range, and none in the last (possibly partial) chunk.
            uint32_t xa[kGUPS][8];
#pragma unroll
            for (int v = 0; v < kGUPS; ++v) g_ld_x32_nv(xrow + (chunk + v) * kChunkK + 16 * t, true, xa[v]);
#pragma unroll
            for (int v = 0; v < kGUPS; ++v)
                mma_unit(st + v * kUnitQ + 16 * lane, st + kGUPS * kUnitQ + v * kUnitS + 4 * lane, xa[v], acc);
            i += kGUPS;
            chunk += kGUPS;
        } else {
#pragma unroll 1
            for (int v = 0; v < kGUPS && i < n; ++v) {
                const int col = chunk * kChunkK + 16 * t;
                uint32_t xw[8];
                g_ld_x32(xrow + col, col < p.K, xw);
                mma_unit(st + v * kUnitQ + 16 * lane, st + kGUPS * kUnitQ + v * kUnitS + 4 * lane, xw, acc);
                ++i;
                const bool tile_end = chunk == (int)KC - 1;
                if (tile_end || i == n) {
                const long long tg = grp * (long long)p.tiles + tile;  // tile of the virtual matrix
                const long long ts = tg * KC;
                const long long glo = g_range_owner(U, TW, ts), ghi = g_range_owner(U, TW, ts + KC - 1);
                bool write = true;
                if (glo != ghi) {
                    const int slot_id = (tg == first_tg) ? 0 : 1;
                    float* dst = p.partials + ((size_t)gw * 2 + slot_id) * kGSlot + lane * 8;
                    reinterpret_cast<float4*>(dst)[0] = make_float4(acc[0][0], acc[0][1], acc[0][2], acc[0][3]);
                    reinterpret_cast<float4*>(dst)[1] = make_float4(acc[1][0], acc[1][1], acc[1][2], acc[1][3]);
                    // the lanes' stores are ordered before lane 0's release by the warp barrier
                    __syncwarp();
                    unsigned last = 0;
                    if (lane == 0) {
                        unsigned old;
                        asm volatile("atom.acq_rel.gpu.global.add.u32 %0, [%1], 1;" : "=r"(old) : "l"(p.counters + tg) : "memory");
                        last = (old == (unsigned)(ghi - glo)) ? 1u : 0u;
                    }
                    last = __shfl_sync(0xffffffffu, last, 0);
                    write = last != 0;
                    if (write) {
                        // every contributor's partial, in warp order
                        const int glo_slot = g_range_begin(U, TW, glo) >= ts ? 0 : 1;
    #pragma unroll
                        for (int r = 0; r < 2; ++r)
    #pragma unroll
                            for (int k = 0; k < 4; ++k) acc[r][k] = 0.f;
                        // four contributors' loads in flight at a time, added in warp order
                        for (long long w0 = glo; w0 <= ghi; w0 += 4) {
                            float4 pa[4], pb[4];
#pragma unroll
                            for (int b = 0; b < 4; ++b) {
                                const long long w = w0 + b;
                                if (w <= ghi) {
                                    const int ws = (w == glo) ? glo_slot : 0;
                                    const float4* src = reinterpret_cast<const float4*>(
                                        p.partials + ((size_t)w * 2 + ws) * kGSlot + lane * 8);
                                    pa[b] = __ldcg(src);
                                    pb[b] = __ldcg(src + 1);
                                }
                            }
#pragma unroll
                            for (int b = 0; b < 4; ++b) {
                                if (w0 + b <= ghi) {
                                    acc[0][0] += pa[b].x; acc[0][1] += pa[b].y; acc[0][2] += pa[b].z; acc[0][3] += pa[b].w;
                                    acc[1][0] += pb[b].x; acc[1][1] += pb[b].y; acc[1][2] += pb[b].z; acc[1][3] += pb[b].w;
                                }
                            }
                        }
                        if (lane == 0) p.counters[tg] = 0u;  // every contributor is in
                    }
                }
                if (write) {
    #pragma unroll
                    for (int r = 0; r < 2; ++r)
    #pragma unroll
                        for (int k = 0; k < 4; ++k) {
                            const int m = 2 * t + (k & 1);
                            const long long nrow = (long long)tile * kTileN + 16 * r + g8 + ((k & 2) ? 8 : 0);
                            if (m < rows && nrow < p.N) {
                                const int pos = gt.sorted[first + m];
                                p.Y[pos * p.N + nrow] = (acc[r][k] * kEpilogueScale) * gscale;
                            }
                        }
                }
#pragma unroll
                    for (int r = 0; r < 2; ++r)
#pragma unroll
                        for (int k = 0; k < 4; ++k) acc[r][k] = 0.f;
                }
                if (tile_end) {
                    chunk = 0;
                    if (++tile == p.tiles) {
                        tile = 0;
                        if (++grp < gt.n_groups) set_group();
                    }
                } else {
                    ++chunk;
                }
            }
        }
        // the MMAs above consumed every word read from the stage: refill it
        __syncwarp();
        if (lane == 0 && js + kGStages < n_stages) issue(js + kGStages);
    }
}

struct GroupedState {
    int device = -1;
    int sm_count = 0;
    float* partials = nullptr;
    unsigned* counters = nullptr;
};
std::mutex g_gmu;
GroupedState g_gstate[64];

int grouped_state(cudaStream_t stream, GroupedState** out)
{
    int dev = 0;
    NVFP4_CUDA_TRY(cudaGetDevice(&dev));
    if (dev < 0 || dev >= 64) return NVFP4_ERR_ARG;
    std::lock_guard<std::mutex> lock(g_gmu);
    GroupedState& s = g_gstate[dev];
    if (s.device == dev) {
        *out = &s;
        return NVFP4_OK;
    }
    cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
    NVFP4_CUDA_TRY(cudaStreamIsCapturing(stream, &cs));
    if (cs != cudaStreamCaptureStatusNone) return NVFP4_ERR_CAPTURE;
    int sms = 0;
    NVFP4_CUDA_TRY(cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev));
    float* partials = nullptr;
    unsigned* counters = nullptr;
    const size_t n_counters = (size_t)NVFP4_GROUPED_MAX_ROUTES * kGMaxTiles;
    NVFP4_CUDA_TRY(cudaMalloc(&partials, (size_t)sms * kGWarps * 2 * kGSlot * sizeof(float)));
    cudaError_t e = cudaMalloc(&counters, n_counters * sizeof(unsigned));
    if (e == cudaSuccess) e = cudaMemset(counters, 0, n_counters * sizeof(unsigned));
    if (e == cudaSuccess)
        e = cudaFuncSetAttribute(grouped_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 kGWarps * kGStages * (kGStage + 8));
    if (e == cudaSuccess) e = cudaDeviceSynchronize();
    if (e != cudaSuccess) {
        cudaFree(partials);
        if (counters) cudaFree(counters);
        return fail_cuda(e);
    }
    s.sm_count = sms;
    s.partials = partials;
    s.counters = counters;
    s.device = dev;
    *out = &s;
    return NVFP4_OK;
}

}  // namespace

int read_and_clear_grouped_status(unsigned* status)
{
    unsigned v = 0;
    NVFP4_CUDA_TRY(cudaDeviceSynchronize());
    NVFP4_CUDA_TRY(cudaMemcpyFromSymbol(&v, g_grouped_status, sizeof v));
    if (v != 0) {
        const unsigned zero = 0;
        NVFP4_CUDA_TRY(cudaMemcpyToSymbol(g_grouped_status, &zero, sizeof zero));
        int dev = 0;
        NVFP4_CUDA_TRY(cudaGetDevice(&dev));
        std::lock_guard<std::mutex> lock(g_gmu);
        if (dev >= 0 && dev < 64 && g_gstate[dev].device == dev)
            NVFP4_CUDA_TRY(cudaMemset(g_gstate[dev].counters, 0,
                                      (size_t)NVFP4_GROUPED_MAX_ROUTES * kGMaxTiles * sizeof(unsigned)));
        NVFP4_CUDA_TRY(cudaDeviceSynchronize());
    }
    *status = v;
    return NVFP4_OK;
}

}  // namespace nvfp4

using namespace nvfp4;

extern "C" int nvfp4_gemm_grouped(const void* X, int x_per_route, const int32_t* route, int M, int T,
                                  const nvfp4_expert* experts, int E, float* Y, int64_t N, int64_t K,
                                  nvfp4_stream_t stream)
{
    if (!X || !route || !experts || !Y || E < 1) return NVFP4_ERR_ARG;
    if (M < 1 || M > 8) return NVFP4_ERR_M;
    if (T < 1 || M * T > NVFP4_GROUPED_MAX_ROUTES) return NVFP4_ERR_ARG;
    int st = check_shape(N, K);
    if (st != NVFP4_OK) return st;
    if ((N + kTileN - 1) / kTileN > kGMaxTiles) return NVFP4_ERR_SHAPE;
    if (!aligned16(X) || ((uintptr_t)Y & 3) != 0 || ((uintptr_t)route & 3) != 0 || ((uintptr_t)experts & 7) != 0)
        return NVFP4_ERR_ALIGN;
    GroupedState* gs = nullptr;
    st = grouped_state((cudaStream_t)stream, &gs);
    if (st != NVFP4_OK) return st;
    GParams p;
    p.X = static_cast<const uint16_t*>(X);
    p.x_per_route = x_per_route ? 1 : 0;
    p.route = route;
    p.M = M;
    p.T = T;
    p.experts = experts;
    p.E = E;
    p.Y = Y;
    p.N = N;
    p.K = K;
    p.KC = (int)((K + kChunkK - 1) / kChunkK);
    p.tiles = (int)((N + kTileN - 1) / kTileN);
    p.UE = (long long)p.KC * p.tiles;
    p.partials = gs->partials;
    p.counters = gs->counters;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)gs->sm_count);
    cfg.blockDim = dim3(kGWarps * 32);
    cfg.dynamicSmemBytes = (size_t)kGWarps * kGStages * (kGStage + 8);
    cfg.stream = (cudaStream_t)stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    NVFP4_CUDA_TRY(cudaLaunchKernelEx(&cfg, grouped_kernel, p));
    return NVFP4_OK;
}
