// gemm.cu -- the NVFP4 decode GEMM kernels for sm_100a and their launch.
//
// Y[M][N] = gscale * X[M][K] . dequant(W)^T for M = 1..8 lanes (ignis
// README, "The decode round": all lanes share one pass over the weights,
// which streams at the card's memory bandwidth), and the fused gate/up
// variant H = bf16(silu(Xg) * Xu) that reads both projections in the same
// pass.  The same kernel takes verify widths M = 9..32 (README, "What sets
// it apart", "Speculative decoding (DFlash2)") as two to four blocks of 8
// lanes, each dequantised word feeding one MMA per block.
//
// Work split ("stream-K"): the matrix is a sequence of 32 x 64 units stored
// contiguously in tile-major order.  Every warp of the grid takes one
// contiguous range of units -- one contiguous run of bytes in each weight
// plane -- so all warps stream nearly the same number of bytes whatever N
// and K are.  A warp pulls its range through a private ring of shared-memory
// stages with 1-D bulk copies (the TMA engine, no tensor map, no multicast),
// one mbarrier per stage, dequantises in registers and feeds bf16 m16n8k16
// tensor-core MMAs with the lanes of X as the 8-wide N side.  A tile
// (32 rows) that straddles warp ranges is combined in two levels: inside a
// CTA, each contributing warp leaves its partial sums in shared memory and
// raises a flag; across CTAs, each later CTA's designated warp writes its
// CTA's sum into a workspace slot as 64-bit words carrying a ready bit.  One
// warp -- the last range-end contributor of the CTA that holds the tile's
// first unit -- waits (bounded) on those flags and words and adds them in warp
// order, then CTA order (finish_tile).  A later CTA's designated warp waits
// only on its own CTA's contributors, and those publish without waiting, so
// the waits form no cycle.  The fused gate/up kernel keeps a one-level last-arriver
// combine through a global counter (tile_done_global) and never waits.  Both
// orders are fixed, so results are bit-identical run to run.  The persistent
// round kernel at the end of the file also meets the whole grid at a bounded
// barrier between nodes.
//
// PDL: every kernel signals its dependents at entry, issues its weight
// copies (which depend on nothing), and only then waits for the preceding
// grid before it reads X or touches outputs and workspace.
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>
#include <string.h>

#include <mutex>

#include "async.cuh"
#include "dequant.cuh"
#include "internal.h"
#include "layout.cuh"

namespace nvfp4 {

__device__ unsigned int g_device_status;

constexpr int kWarps = 16;                 // warps per CTA at M <= 8 (one CTA per SM, every warp at equal priority);
                                           // the lane-block kernels run 12 or 8 (wide_warps below)
constexpr int kMinBlocks = 1;              // CTAs per SM the register budget is sized for
constexpr int kSlotFloats = 512;           // partial-sum slot: 2 matrices x 32 rows x 8 lanes


struct KParams {
    const uint8_t* wq[2];
    const uint8_t* ws[2];
    float gs[2];
    const uint16_t* X;
    void* out;
    long long N, K, k_chunks, units;
    long long total_warps;
    float* partials;
    unsigned* counters;
    long long rb_q;  // units / total_warps
    unsigned rb_r;   // units % total_warps
    float* legacy_partials;  // the fused kernel's one-level combine (plain floats, its own region)
};

// range_begin(units, total_warps, w) of the decode kernels without a 64-bit
// division: q*w + (r*w)/TW, with r*w < 2^32 (total_warps < 2^16).
__device__ __forceinline__ long long kp_begin(const KParams& p, long long w)
{
    return p.rb_q * w + (long long)((unsigned)p.rb_r * (unsigned)w / (unsigned)p.total_warps);
}

// range_owner(units, total_warps, x) for x < units: a double-precision
// estimate of ((x+1)*TW - 1) / units (numerator < 2^53, so off by at most one)
// corrected to the exact quotient.
__device__ __forceinline__ long long kp_owner(const KParams& p, long long x)
{
    const long long n = (x + 1) * p.total_warps - 1;
    long long w = (long long)((double)n / (double)p.units);
    if ((w + 1) * p.units <= n)
        ++w;
    else if (w * p.units > n)
        --w;
    return w;
}

// 32 bytes of X into x when `pred`; x keeps its contents otherwise.
__device__ __forceinline__ void ld_x32_keep(const void* p, bool pred, uint32_t (&x)[8])
{
    asm(
        "{\n .reg .pred q;\n setp.ne.u32 q, %9, 0;\n"
        " @q ld.global.nc.v4.u32 {%0,%1,%2,%3}, [%8];\n"
        " @q ld.global.nc.v4.u32 {%4,%5,%6,%7}, [%8+16];\n}"
        : "+r"(x[0]), "+r"(x[1]), "+r"(x[2]), "+r"(x[3]), "+r"(x[4]), "+r"(x[5]), "+r"(x[6]), "+r"(x[7])
        : "l"(p), "r"((uint32_t)pred));
}

// 32 bytes of X (two 16-byte loads) when `pred`, zeros otherwise; no branch.
__device__ __forceinline__ void ld_x32(const void* p, bool pred, uint32_t (&x)[8])
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

__device__ __forceinline__ float4 ld_cg_f4(const float* p)
{
    float4 v;
    asm volatile("ld.global.cg.v4.f32 {%0,%1,%2,%3}, [%4];"
                 : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w)
                 : "l"(p));
    return v;
}

__device__ __forceinline__ long long range_begin(long long units, long long tw, long long w)
{
    return units * w / tw;
}

// Warp whose range holds unit x.
__device__ __forceinline__ long long range_owner(long long units, long long tw, long long x)
{
    return ((x + 1) * tw - 1) / units;
}

// Output side of a kernel, passed by value to the out-of-line tile finisher.
struct OutArgs {
    void* out;
    float* partials;
    unsigned* counters;
    long long N, units, total_warps, k_chunks;
    float gs0, gs1;
};

// Accumulator sets per warp: one per matrix and block of 8 decode lanes.
template <int M, int NW>
constexpr int kAccSets = NW * ((M + 7) / 8);

template <int M, int NW>
__device__ __forceinline__ void epilogue(const OutArgs& o, long long tile, const float (&acc)[kAccSets<M, NW>][2][4],
                                         int g, int t)
{
    constexpr int NB = (M + 7) / 8;  // blocks of 8 decode lanes (plain GEMM only when more than one)
    static_assert(NW == 1 || NB == 1, "the fused gate/up variant takes at most 8 lanes");
#pragma unroll
    for (int b = 0; b < NB; ++b)
#pragma unroll
    for (int r = 0; r < 2; ++r)
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const int m = 8 * b + 2 * t + (i & 1);
            const long long n = tile * kTileN + 16 * r + g + ((i & 2) ? 8 : 0);
            if (m < M && n < o.N) {
                if (NW == 1) {
                    static_cast<float*>(o.out)[m * o.N + n] = (acc[b][r][i] * kEpilogueScale) * o.gs0;
                } else {
                    const float gv = (acc[0][r][i] * kEpilogueScale) * o.gs0;
                    const float uv = (acc[NW - 1][r][i] * kEpilogueScale) * o.gs1;
                    const float h = gv / (1.0f + expf(-gv)) * uv;
                    static_cast<__nv_bfloat16*>(o.out)[m * o.N + n] = __float2bfloat16_rn(h);
                }
            }
        }
}

// Load one contributor's partial sums (this lane's NW*8 floats).
template <int NW>
__device__ __forceinline__ void load_partial(const float* src, float4 (&v)[NW * 2])
{
#pragma unroll
    for (int k = 0; k < NW * 2; ++k) v[k] = ld_cg_f4(src + 4 * k);
}

// The persistent round kernel's combine, through the workspace only: end of a
// tile for this warp, after it stored its sums in its partial slot.  A tile
// the warp covered alone goes straight to the epilogue.  Otherwise the warp
// counts itself in, and the last contributor adds the partials in the order
// the decode kernel's two-level combine uses -- each CTA's contributors in
// warp order, then those CTA sums in CTA order -- so a GEMM node of the
// persistent round equals a direct call bit for bit.  Out of line, so the
// streaming loop does not carry its registers.
template <int M>
__device__ __noinline__ void tile_done_round(const OutArgs o, long long tile, int lane)
{
    const long long U = o.units, TW = o.total_warps, KC = o.k_chunks;
    const long long ts = tile * KC, te = ts + KC;
    const long long glo = range_owner(U, TW, ts), ghi = range_owner(U, TW, te - 1);
    if (glo != ghi) {
        // The lanes' partial stores are ordered before lane 0's release by the
        // warp barrier; the acquire side orders the last contributor's reads
        // of the other partials after theirs.
        __syncwarp();
        unsigned last = 0;
        if (lane == 0) {
            unsigned old;
            asm volatile("atom.acq_rel.gpu.global.add.u32 %0, [%1], 1;" : "=r"(old) : "l"(o.counters + glo) : "memory");
            last = (old == (unsigned)(ghi - glo)) ? 1u : 0u;
        }
        last = __shfl_sync(0xffffffffu, last, 0);
        if (!last) return;
    }
    const int glo_slot = (range_begin(U, TW, glo) >= ts) ? 0 : 1;
    float total[1][2][4], local[1][2][4];
#pragma unroll
    for (int r = 0; r < 2; ++r)
#pragma unroll
        for (int i = 0; i < 4; ++i) total[0][r][i] = local[0][r][i] = 0.f;
    long long cta = glo / kWarps;
    constexpr int kBatch = 4;  // contributors whose loads are in flight together
    for (long long w0 = glo; w0 <= ghi; w0 += kBatch) {
        float4 v[kBatch][2];
#pragma unroll
        for (int b = 0; b < kBatch; ++b) {
            const long long w = w0 + b;
            if (w <= ghi) {
                const int ws = (w == glo) ? glo_slot : 0;
                load_partial<1>(o.partials + ((size_t)w * 2 + ws) * kSlotFloats + lane * 8, v[b]);
            }
        }
#pragma unroll
        for (int b = 0; b < kBatch; ++b) {
            const long long w = w0 + b;
            if (w <= ghi) {
                if (w / kWarps != cta) {
#pragma unroll
                    for (int r = 0; r < 2; ++r)
#pragma unroll
                        for (int i = 0; i < 4; ++i) {
                            total[0][r][i] += local[0][r][i];
                            local[0][r][i] = 0.f;
                        }
                    cta = w / kWarps;
                }
#pragma unroll
                for (int r = 0; r < 2; ++r) {
                    local[0][r][0] += v[b][r].x;
                    local[0][r][1] += v[b][r].y;
                    local[0][r][2] += v[b][r].z;
                    local[0][r][3] += v[b][r].w;
                }
            }
        }
    }
#pragma unroll
    for (int r = 0; r < 2; ++r)
#pragma unroll
        for (int i = 0; i < 4; ++i) total[0][r][i] += local[0][r][i];
    epilogue<M, 1>(o, tile, total, lane >> 2, lane & 3);
    if (glo != ghi && lane == 0) atomicExch(&o.counters[glo], 0u);
}

// Slot stride of the one-level combine for NA accumulator sets per lane.
template <int NA>
constexpr int kLegacyStride = NA <= 2 ? kSlotFloats : 2 * kSlotFloats;

// The fused gate/up kernel's combine, one level through the workspace (its
// streaming loop sits at the register limit, with no room for the two-level
// combine's bookkeeping): end of a tile for this warp, after it stored its
// sums in its partial slot of the legacy region.
// A tile the warp covered alone goes straight to the epilogue.  Otherwise the
// warp counts itself in, and the last contributor adds every partial in warp
// order (glo..ghi, a fixed order, so the result does not depend on who arrives
// last) and runs the epilogue.  A warp that finds every other contributor
// already counted in is the last one without counting itself in, which saves
// the release and the atomic's round trip on the path that ends the kernel.
// When the finishing warp's bulk-copy ring is idle (its range is done;
// gather_smem != 0), the first contributors' partials are gathered into it
// with one bulk copy each, all in flight at once, and the rest are loaded
// into registers a few at a time, the first few while the copies are in
// flight.  Out of line, so the streaming loop does not carry its registers.
template <int M, int NW>
__device__ __noinline__ void tile_done_global(const OutArgs o, long long tile, int lane, uint32_t gather_smem,
                                       uint32_t gather_bytes, uint32_t gather_bar)
{
    constexpr int NA = kAccSets<M, NW>;  // accumulator sets per lane in a partial
    const long long U = o.units, TW = o.total_warps, KC = o.k_chunks;
    const long long ts = tile * KC, te = ts + KC;
    const long long glo = range_owner(U, TW, ts), ghi = range_owner(U, TW, te - 1);
    if (glo != ghi) {
        // The lanes' partial stores are ordered before lane 0's release by the
        // warp barrier; the acquire side (of the load or of the atomic) orders
        // the last contributor's reads of the other partials after theirs.
        __syncwarp();
        // Every warp below total_warps has a non-empty range, so the
        // contributors are exactly the warps glo..ghi.
        unsigned last = 0;
        if (lane == 0) {
            const unsigned others = (unsigned)(ghi - glo);
            // Leaving a tile in mid-range (no idle ring: gather_smem == 0), the
            // warp is almost never the last contributor, so it counts in at once.
            unsigned seen = ~0u;
            if (gather_smem != 0)
                asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(seen) : "l"(o.counters + glo) : "memory");
            if (seen == others) {
                last = 1u;
            } else {
                unsigned old;
                asm volatile("atom.acq_rel.gpu.global.add.u32 %0, [%1], 1;" : "=r"(old) : "l"(o.counters + glo) : "memory");
                last = (old == others) ? 1u : 0u;
            }
        }
        last = __shfl_sync(0xffffffffu, last, 0);
        if (!last) return;
    }
    const int glo_slot = (range_begin(U, TW, glo) >= ts) ? 0 : 1;
    float sum[NA][2][4];
#pragma unroll
    for (int a = 0; a < NA; ++a)
#pragma unroll
        for (int r = 0; r < 2; ++r)
#pragma unroll
            for (int i = 0; i < 4; ++i) sum[a][r][i] = 0.f;
    const int C = (int)(ghi - glo + 1);
    constexpr uint32_t kPartBytes = NA * 1024;  // the used part of a slot: 32 lanes x NA x 8 floats
    // contributors 0..nb-1 through the ring, nb..C-1 through registers
    int nb = gather_smem != 0 ? (int)(gather_bytes / kPartBytes) : 0;
    if (nb > C) nb = C;
    if (nb > 0) {
        // order this warp's earlier reads of the ring, and the partials it
        // acquired, before the bulk copies (async proxy)
        asm volatile("fence.proxy.async;" ::: "memory");
        if (lane == 0) mbar_expect_tx(gather_bar, (uint32_t)nb * kPartBytes);
        __syncwarp();
        for (int c = lane; c < nb; c += 32) {
            const long long w = glo + c;
            const int ws = (w == glo) ? glo_slot : 0;
            const uint64_t pol = evict_first_policy();
            bulk_load(gather_smem + c * kPartBytes, o.partials + ((size_t)w * 2 + ws) * kLegacyStride<NA>, kPartBytes,
                      gather_bar, pol);
        }
    }
    constexpr int kBatch = NA == 1 ? 4 : NA == 2 ? 2 : 1;  // contributors whose loads are in flight together (more costs the callers spills)
    float4 v[kBatch][NA * 2];
    long long w0 = glo + nb;
#pragma unroll
    for (int b = 0; b < kBatch; ++b) {
        const long long w = w0 + b;
        if (w <= ghi) {
            const int ws = (w == glo) ? glo_slot : 0;
            load_partial<NA>(o.partials + ((size_t)w * 2 + ws) * kLegacyStride<NA> + lane * (NA * 8), v[b]);
        }
    }
    if (nb > 0) {
        // used once per warp and kernel, so the phase is always 0
        const bool gathered = warp_wait(gather_bar, 0u);
        if (!gathered) {
            // flag it, wait once more (bounded) for the copies, and read these partials from global memory
            if (lane == 0) atomicOr(&g_device_status, 4u);
            warp_wait(gather_bar, 0u);
        }
        // with one accumulator set, two contributors' loads in flight at a time (more
        // registers here would make the callers save theirs); added in warp order
        constexpr int kPair = NA == 1 ? 2 : 1;
        for (int c = 0; c < nb; c += kPair) {
            float4 x[kPair][NA * 2];
            const int cnt = nb - c < kPair ? nb - c : kPair;
#pragma unroll
            for (int e = 0; e < kPair; ++e) {
                if (e < cnt) {
                    if (gathered) {
                        const uint32_t src = gather_smem + (c + e) * kPartBytes + lane * (NA * 32);
#pragma unroll
                        for (int k = 0; k < NA * 2; ++k)
                            asm volatile("ld.shared.v4.f32 {%0,%1,%2,%3}, [%4];"
                                         : "=f"(x[e][k].x), "=f"(x[e][k].y), "=f"(x[e][k].z), "=f"(x[e][k].w)
                                         : "r"(src + 16 * k));
                    } else {
                        const long long w = glo + c + e;
                        const int ws = (w == glo) ? glo_slot : 0;
                        load_partial<NA>(o.partials + ((size_t)w * 2 + ws) * kLegacyStride<NA> + lane * (NA * 8), x[e]);
                    }
                }
            }
#pragma unroll
            for (int e = 0; e < kPair; ++e) {
                if (e < cnt) {
#pragma unroll
                    for (int k = 0; k < NA * 2; ++k) {
                        sum[k >> 1][k & 1][0] += x[e][k].x;
                        sum[k >> 1][k & 1][1] += x[e][k].y;
                        sum[k >> 1][k & 1][2] += x[e][k].z;
                        sum[k >> 1][k & 1][3] += x[e][k].w;
                    }
                }
            }
        }
    }
    for (;;) {
#pragma unroll
        for (int b = 0; b < kBatch; ++b) {
            if (w0 + b <= ghi) {
#pragma unroll
                for (int k = 0; k < NA * 2; ++k) {
                    sum[k >> 1][k & 1][0] += v[b][k].x;
                    sum[k >> 1][k & 1][1] += v[b][k].y;
                    sum[k >> 1][k & 1][2] += v[b][k].z;
                    sum[k >> 1][k & 1][3] += v[b][k].w;
                }
            }
        }
        w0 += kBatch;
        if (w0 > ghi) break;
#pragma unroll
        for (int b = 0; b < kBatch; ++b) {
            const long long w = w0 + b;
            if (w <= ghi) {
                const int ws = (w == glo) ? glo_slot : 0;
                load_partial<NA>(o.partials + ((size_t)w * 2 + ws) * kLegacyStride<NA> + lane * (NA * 8), v[b]);
            }
        }
    }
    epilogue<M, NW>(o, tile, sum, lane >> 2, lane & 3);
    if (glo != ghi && lane == 0) atomicExch(&o.counters[glo], 0u);
}


// ------------------------------------------------------------------ the combine of the decode kernels
//
// Warp gw owns units [kp_begin(gw), kp_begin(gw + 1)); CTA c owns the union of
// its warps' ranges, [uc, uc1).  A tile with several contributors is summed by
// a designated finisher, first inside each CTA, then across CTAs:
//   - inside a CTA, the finisher is the last contributor whose range ends in
//     the tile.  A contributor whose range ends in the tile leaves its partial
//     sums in its own ring (idle from then on) and raises its shared-memory
//     flag; the one contributor that may leave the tile in mid-range (the
//     tile's last in the CTA) writes them to a slot of the CTA's shared-memory
//     pool (slot = the tile's index among the CTA's tiles) and raises its
//     other flag, or, when the CTA spans more tiles than the pool has slots,
//     to its workspace slot 0;
//   - across CTAs, the finisher is the one of the CTA that holds the tile's
//     first unit; every other CTA's sum goes to one of that CTA's two CTA
//     slots.
// Workspace slots hold LL words: 64 bits, a float's bits below a ready flag, so
// a 64-bit store publishes data and flag together and the reader polls the
// data itself -- no fence, no atomic, no release on the writer's side, which at
// GPU scope would cost a round trip to L2 under load.  The reader clears each
// slot it consumed, so every slot is zero when the next launch starts.  A
// finisher waits only for warps of higher index, and those never wait for it,
// so the waits form no cycle; all CTAs of the grid are resident (one per SM,
// at most as many as SMs), and every wait is bounded.  Sums run in warp order
// inside a CTA and in CTA order across, so results are bit-identical run to run.

// Workspace slot s of warp w: [lane][NA * 8] LL words.
template <int NA>
__device__ __forceinline__ uint64_t* ll_slot(const KParams& p, long long w, int s)
{
    return reinterpret_cast<uint64_t*>(p.partials) + ((size_t)w * 2 + s) * (NA * 256);
}

// Slot of CTA c's sum of `tile`: slot 1 of the CTA's first warp for the last
// tile of its range, of its second warp for the first (slot 1 of a warp is
// used for nothing else).
template <int W, int NA>
__device__ __forceinline__ uint64_t* cta_slot(const KParams& p, long long c, long long tile)
{
    const long long w1 = (c + 1) * W < p.total_warps ? (c + 1) * W : p.total_warps;
    const long long last_tile = (kp_begin(p, w1) - 1) / p.k_chunks;
    return ll_slot<NA>(p, c * W + (tile == last_tile ? 0 : 1), 1);
}

constexpr unsigned long long kLLReady = 1ull << 32;

template <int NA>
__device__ __forceinline__ void ll_write(uint64_t* slot, int lane, const float (&acc)[NA][2][4])
{
    uint64_t* d = slot + lane * (NA * 8);
#pragma unroll
    for (int a = 0; a < NA; ++a)
#pragma unroll
        for (int r = 0; r < 2; ++r)
#pragma unroll
            for (int i = 0; i < 4; i += 2)
                asm volatile("st.relaxed.gpu.global.v2.b64 [%0], {%1, %2};" ::"l"(d + (a * 2 + r) * 4 + i),
                             "l"(kLLReady | __float_as_uint(acc[a][r][i])),
                             "l"(kLLReady | __float_as_uint(acc[a][r][i + 1]))
                             : "memory");
}

// Poll slot (bounded) until every word carries the ready flag, add its
// floats into sum, and clear the slot for the next launch.  Returns false if
// the wait gave up.
template <int NA>
__device__ __forceinline__ bool ll_read_add(uint64_t* slot, int lane, float (&sum)[NA][2][4])
{
    uint64_t* d = slot + lane * (NA * 8);
    unsigned long long v[NA * 8];
    bool ok = false;
    for (uint32_t it = 0; it < kWaitLimit; ++it) {
        bool ready = true;
#pragma unroll
        for (int k = 0; k < NA * 8; k += 2) {
            asm volatile("ld.relaxed.gpu.global.v2.b64 {%0, %1}, [%2];" : "=l"(v[k]), "=l"(v[k + 1]) : "l"(d + k) : "memory");
            ready = ready && (v[k] >> 32) == 1u && (v[k + 1] >> 32) == 1u;
        }
        if (__all_sync(0xffffffffu, ready)) {
            ok = true;
            break;
        }
        __nanosleep(64);
    }
#pragma unroll
    for (int k = 0; k < NA * 8; ++k) sum[k >> 3][(k >> 2) & 1][k & 3] += __uint_as_float((unsigned)v[k]);
#pragma unroll
    for (int k = 0; k < NA * 8; k += 2)
        asm volatile("st.relaxed.gpu.global.v2.b64 [%0], {%1, %2};" ::"l"(d + k), "l"(0ull), "l"(0ull) : "memory");
    return ok;
}

template <int NA>
__device__ __forceinline__ void store_ring_partial(uint32_t ring, int lane, const float (&acc)[NA][2][4])
{
#pragma unroll
    for (int a = 0; a < NA; ++a)
#pragma unroll
        for (int r = 0; r < 2; ++r)
            asm volatile("st.shared.v4.f32 [%0], {%1,%2,%3,%4};" ::"r"(ring + (uint32_t)(((a * 2 + r) * 32 + lane) * 16)),
                         "f"(acc[a][r][0]), "f"(acc[a][r][1]), "f"(acc[a][r][2]), "f"(acc[a][r][3])
                         : "memory");
}

template <int NA>
__device__ __forceinline__ void add_ring_partial(uint32_t ring, int lane, float (&sum)[NA][2][4])
{
#pragma unroll
    for (int k = 0; k < NA * 2; ++k) {
        float4 x;
        asm volatile("ld.shared.v4.f32 {%0,%1,%2,%3}, [%4];"
                     : "=f"(x.x), "=f"(x.y), "=f"(x.z), "=f"(x.w)
                     : "r"(ring + (uint32_t)((k * 32 + lane) * 16))
                     : "memory");
        sum[k >> 1][k & 1][0] += x.x;
        sum[k >> 1][k & 1][1] += x.y;
        sum[k >> 1][k & 1][2] += x.z;
        sum[k >> 1][k & 1][3] += x.w;
    }
}

template <int NA>
__device__ __forceinline__ void add_into(float (&sum)[NA][2][4], const float4 (&x)[NA * 2])
{
#pragma unroll
    for (int k = 0; k < NA * 2; ++k) {
        sum[k >> 1][k & 1][0] += x[k].x;
        sum[k >> 1][k & 1][1] += x[k].y;
        sum[k >> 1][k & 1][2] += x[k].z;
        sum[k >> 1][k & 1][3] += x[k].w;
    }
}

template <int M, int NW>
__device__ __forceinline__ void epilogue_p(const KParams& p, long long tile, const float (&acc)[kAccSets<M, NW>][2][4],
                                           int g, int t)
{
    OutArgs o;
    o.out = p.out;
    o.N = p.N;
    o.gs0 = p.gs[0];
    o.gs1 = p.gs[1];
    epilogue<M, NW>(o, tile, acc, g, t);
}

// Dynamic shared memory of a decode kernel: the warps' rings, their stage
// barriers, the pool of mid-range partial sums, the flags (ring partial ready
// [0, W), pool partial ready [W, 2W)) and the warps' unit boundaries.
template <int NA>
struct AccPack {
    float v[NA][2][4];
};

constexpr int kSmemPerBlock = 227 * 1024;

template <int M, int NW, int STAGES, int UPS, int W>
struct SmemLayout {
    static constexpr int kStage = NW * UPS * kUnitBytes;
    static constexpr int kRings = W * STAGES * kStage;
    static constexpr int kBars = kRings;                       // W * STAGES mbarriers
    static constexpr int kPool = kBars + W * STAGES * 8;
    static constexpr int kSlot = kAccSets<M, NW> * 1024;        // one partial: NA x 32 lanes x 8 floats
    static constexpr int kTail = 2 * W * 4 + (W + 1) * 8 + 64;  // flags, boundaries, alignment slack
    static constexpr int kFit = (kSmemPerBlock - kPool - kTail) / kSlot;
    static constexpr int kPoolSlots = NW == 2 ? 0 : kFit < 0 ? 0 : kFit > 8 ? 8 : kFit;  // at most 8
    static constexpr int kGather = kPool + kPoolSlots * kSlot;   // NW == 2: one gather mbarrier per warp
    static constexpr int kFlags = kGather + (NW == 2 ? W * 8 : 0);
    static constexpr int kWb = kFlags + 2 * W * 4;              // 8-byte aligned: kFlags is a multiple of 8
    static constexpr int kBytes = kWb + (W + 1) * 8;
    static_assert(kBytes <= kSmemPerBlock, "shared memory over budget");
};

// The warp of this CTA whose range holds unit x (uc <= x < uc1): wb[w] is the
// first unit of local warp w, wb[W] = uc1 (a binary search over W + 1 entries).
template <int W>
__device__ __forceinline__ int local_owner(const long long* wb, long long x)
{
    int lo = 0, hi = W;
#pragma unroll
    for (int s = 0; s < 5; ++s)
        if (hi - lo > 1) {
            const int mid = (lo + hi) >> 1;
            if (wb[mid] <= x)
                lo = mid;
            else
                hi = mid;
        }
    return lo;
}

// The designated finisher of `tile` in this CTA (its own partial is already
// in its ring): add the CTA's partials in warp order, then either run the
// epilogue (the tile lies in this CTA), publish the CTA's sum (another CTA
// finishes the tile), or add the other CTAs' sums in CTA order and run the
// epilogue.
template <int M, int NW, int STAGES, int UPS, int W>
__device__ __noinline__ void finish_tile(const KParams& p, long long tile, int self, int lane)
{
    using L = SmemLayout<M, NW, STAGES, UPS, W>;
    extern __shared__ __align__(128) uint8_t smem[];
    constexpr int NA = kAccSets<M, NW>;
    constexpr int POOL = L::kPoolSlots;
    const uint32_t base = smem_addr(smem);
    const uint32_t flags_s = base + L::kFlags, pool_s = base + L::kPool;
    const long long* wb = reinterpret_cast<const long long*>(smem + L::kWb);
    const long long cta = blockIdx.x, uc = wb[0], uc1 = wb[W];
    const long long KC = p.k_chunks;
    const long long ts = tile * KC, te = ts + KC;
    const long long a = ts > uc ? ts : uc, b = te < uc1 ? te : uc1;
    const int wlo = local_owner<W>(wb, a), whi = local_owner<W>(wb, b - 1);
    const bool whi_crosses = wb[whi + 1] > b;
    const long long ps = tile - uc / KC;  // the crossing contributor's pool slot
    const bool cross_ll = whi_crosses && ps >= POOL;
    // 1. every flag at once: lane i watches contributor wlo + i
    bool ok;
    {
        const int v = wlo + lane;
        bool done = true;
        uint32_t f = 0;
        if (v <= whi && v != self && !(v == whi && cross_ll)) {
            done = false;
            f = flags_s + 4u * (uint32_t)((v == whi && whi_crosses) ? W + v : v);
        }
        for (uint32_t it = 0; it < kWaitLimit; ++it) {
            if (!done) {
                uint32_t up;
                asm volatile("ld.acquire.cta.shared::cta.u32 %0, [%1];" : "=r"(up) : "r"(f) : "memory");
                done = up != 0;
            }
            if (__all_sync(0xffffffffu, done)) break;
            __nanosleep(32);
        }
        ok = __all_sync(0xffffffffu, done);
        // the lanes' acquires order every lane's reads below after the contributors' writes
        __syncwarp();
    }
    // 2. the partials in warp order, 4 / NA contributors' loads in flight at a time
    float sum[NA][2][4];
#pragma unroll
    for (int x = 0; x < NA; ++x)
#pragma unroll
        for (int r = 0; r < 2; ++r)
#pragma unroll
            for (int i = 0; i < 4; ++i) sum[x][r][i] = 0.f;
    constexpr int kB = NA >= 4 ? 1 : 4 / NA;
    const int last_smem = cross_ll ? whi - 1 : whi;
    for (int v0 = wlo; v0 <= last_smem; v0 += kB) {
        float4 x[kB][NA * 2];
#pragma unroll
        for (int bb = 0; bb < kB; ++bb) {
            const int v = v0 + bb;
            if (v <= last_smem) {
                const uint32_t src = (v == whi && whi_crosses) ? pool_s + (uint32_t)ps * L::kSlot
                                                               : base + (uint32_t)v * (STAGES * L::kStage);
#pragma unroll
                for (int k = 0; k < NA * 2; ++k)
                    asm volatile("ld.shared.v4.f32 {%0,%1,%2,%3}, [%4];"
                                 : "=f"(x[bb][k].x), "=f"(x[bb][k].y), "=f"(x[bb][k].z), "=f"(x[bb][k].w)
                                 : "r"(src + (uint32_t)((k * 32 + lane) * 16))
                                 : "memory");
            }
        }
#pragma unroll
        for (int bb = 0; bb < kB; ++bb)
            if (v0 + bb <= last_smem) add_into<NA>(sum, x[bb]);
    }
    if (cross_ll) ok = ll_read_add<NA>(ll_slot<NA>(p, cta * W + whi, 0), lane, sum) && ok;
    const long long clo = kp_owner(p, ts) / W, chi = kp_owner(p, te - 1) / W;
    if (clo != chi) {
        if (cta != clo) {
            ll_write<NA>(cta_slot<W, NA>(p, cta, tile), lane, sum);
            if (!ok && lane == 0) atomicOr(&g_device_status, 4u);
            return;
        }
        for (long long c = clo + 1; c <= chi; ++c) ok = ll_read_add<NA>(cta_slot<W, NA>(p, c, tile), lane, sum) && ok;
    }
    if (!__all_sync(0xffffffffu, ok) && lane == 0) atomicOr(&g_device_status, 4u);
    epilogue_p<M, NW>(p, tile, sum, lane >> 2, lane & 3);
}

// This warp is done with its part of `tile` (at the tile's last chunk or the
// end of its range), its sums in acc.  Out of line, so the streaming loop
// carries none of its registers.
template <int M, int NW, int STAGES, int UPS, int W>
__device__ __noinline__ void flush_tile(const KParams& p, long long tile, const AccPack<kAccSets<M, NW>> acc, int lane,
                                        int warp)
{
    using L = SmemLayout<M, NW, STAGES, UPS, W>;
    extern __shared__ __align__(128) uint8_t smem[];
    constexpr int NA = kAccSets<M, NW>;
    const long long* wb = reinterpret_cast<const long long*>(smem + L::kWb);
    const uint32_t base = smem_addr(smem);
    const long long cta = blockIdx.x, KC = p.k_chunks;
    const long long uc = wb[0], uc1 = wb[W], w0 = wb[warp], w1 = wb[warp + 1];
    const long long ts = tile * KC, te = ts + KC;
    const long long a = ts > uc ? ts : uc, b = te < uc1 ? te : uc1;  // the tile's units in this CTA
    const bool alone = a >= w0 && b <= w1;  // this warp is the tile's only contributor in the CTA
    if (alone && ts >= uc && te <= uc1) {
        epilogue_p<M, NW>(p, tile, acc.v, lane >> 2, lane & 3);  // and the only one at all
    } else if (w1 > b) {
        // Leaves the tile in mid-range: publish the partial and go on (no wait, no
        // fence): to the CTA's pool when it has the slot, else to the workspace.
        const long long ps = tile - uc / KC;
        if (!alone && ps < L::kPoolSlots) {
            store_ring_partial<NA>(base + L::kPool + (uint32_t)ps * L::kSlot, lane, acc.v);
            __syncwarp();
            if (lane == 0)
                asm volatile("st.release.cta.shared::cta.u32 [%0], 1;" ::"r"(base + L::kFlags + 4u * (W + warp))
                             : "memory");
        } else {
            ll_write<NA>(alone ? cta_slot<W, NA>(p, cta, tile) : ll_slot<NA>(p, cta * W + warp, 0), lane, acc.v);
        }
    } else {
        // Its range ends in the tile: every stage is consumed and the ring is idle.
        store_ring_partial<NA>(base + (uint32_t)warp * (STAGES * L::kStage), lane, acc.v);
        // the designated finisher: the last contributor in the CTA whose range ends here
        const int whi = local_owner<W>(wb, b - 1);
        const int fin = wb[whi + 1] > b ? whi - 1 : whi;
        if (warp == fin) {
            finish_tile<M, NW, STAGES, UPS, W>(p, tile, warp, lane);
        } else {
            __syncwarp();
            if (lane == 0)
                asm volatile("st.release.cta.shared::cta.u32 [%0], 1;" ::"r"(base + L::kFlags + 4u * warp) : "memory");
        }
    }
}

// STAGES shared-memory stages per warp, each holding UPS consecutive units of
// each of the NW matrices (one bulk copy per plane and matrix per stage).
// W warps per CTA (one CTA per SM).  M up to 32: lanes 8b..8b+7 form block b
// of the MMA's 8-wide side, and every dequantised word feeds each block.
template <int M, int NW, int STAGES, int UPS, int W>
__global__ void __launch_bounds__(W * 32, kMinBlocks)
decode_gemm_kernel(const __grid_constant__ KParams p)
{
    extern __shared__ __align__(128) uint8_t smem[];
    using L = SmemLayout<M, NW, STAGES, UPS, W>;
    constexpr int kMatStage = UPS * kUnitBytes;
    constexpr int kStage = NW * kMatStage;
    constexpr int NB = (M + 7) / 8;        // blocks of 8 decode lanes
    constexpr int NA = kAccSets<M, NW>;    // accumulator sets
    unsigned* s_flag = reinterpret_cast<unsigned*>(smem + L::kFlags);
    long long* s_wb = reinterpret_cast<long long*>(smem + L::kWb);  // warp w owns units [s_wb[w], s_wb[w + 1])

    const int lane = threadIdx.x & 31;
    const int warp = threadIdx.x >> 5;
    const int g = lane >> 2, t = lane & 3;
    const long long cta = blockIdx.x;
    const long long gw = cta * W + warp;

    // Dependents may begin launching; they wait for this grid before using its results.
    asm volatile("griddepcontrol.launch_dependents;");

    if (threadIdx.x < 2 * W) s_flag[threadIdx.x] = 0u;
    if (threadIdx.x <= W) {
        const long long w = cta * W + threadIdx.x;
        s_wb[threadIdx.x] = kp_begin(p, w < p.total_warps ? w : p.total_warps);
    }
    __syncthreads();
    const long long TW = p.total_warps, KC = p.k_chunks;
    if (gw >= TW) return;
    // this warp's units [s_wb[warp], s_wb[warp + 1]), the CTA's [s_wb[0], s_wb[W]): read from
    // shared memory where needed, so the streaming loop keeps none of them in registers
    const long long u0 = s_wb[warp];
    const int n_units = (int)(s_wb[warp + 1] - u0);
    const int n_stages = (n_units + UPS - 1) / UPS;

    uint8_t* ring = smem + warp * (STAGES * kStage);
    const uint32_t ring_s = smem_addr(ring);
    const uint32_t bar_s = smem_addr(smem + W * STAGES * kStage) + warp * STAGES * 8;

    const uint32_t gather_bar = smem_addr(smem + L::kGather) + warp * 8;  // NW == 2 only
    if (lane == 0) {
#pragma unroll
        for (int s = 0; s < STAGES; ++s) mbar_init(bar_s + 8 * s);
        if constexpr (NW == 2) mbar_init(gather_bar);
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    __syncwarp();

    auto issue = [&](int j, int slot) {
        const uint64_t pol = evict_first_policy();  // made here: one register pair less across the loop
        const long long ub = u0 + (long long)j * UPS;
        const int rem = n_units - j * UPS;
        const int cnt = rem < UPS ? rem : UPS;
        const uint32_t dst = ring_s + slot * kStage;
        const uint32_t bar = bar_s + 8 * slot;
        mbar_expect_tx(bar, (uint32_t)(NW * cnt * kUnitBytes));
#pragma unroll
        for (int mat = 0; mat < NW; ++mat) {
            bulk_load(dst + mat * kMatStage, p.wq[mat] + ub * kUnitQ, cnt * kUnitQ, bar, pol);
            bulk_load(dst + mat * kMatStage + UPS * kUnitQ, p.ws[mat] + ub * kUnitS, cnt * kUnitS, bar, pol);
        }
    };

    if (lane == 0) {
        const int npre = n_stages < STAGES ? n_stages : STAGES;
        for (int j = 0; j < npre; ++j) issue(j, j);
    }

    // Everything below reads X or writes outputs / workspace: wait for the producer grid.
    asm volatile("griddepcontrol.wait;" ::: "memory");

    float acc[NA][2][4];
#pragma unroll
    for (int a = 0; a < NA; ++a)
#pragma unroll
        for (int r = 0; r < 2; ++r)
#pragma unroll
            for (int i = 0; i < 4; ++i) acc[a][r][i] = 0.f;

    long long tile = u0 / KC;
    const long long first_tile = tile;  // NW == 2: the partial slot of a tile left in mid-range
    int chunk = (int)(u0 - tile * KC);
    const int kc_last = (int)KC - 1;
    const int K32 = (int)p.K;
    // X row of this lane.  Past M a lane loads row g % M instead: it feeds only
    // MMA output columns m >= M, which depend on nothing else and which the
    // epilogue drops, and every lane then runs the same unpredicated loads.
    const uint16_t* xp = p.X + (long long)(g % M) * p.K + chunk * kChunkK + 16 * t;
    // block b's row, (8b + g) % M (a valid row: only the last block reaches past
    // M, and by less than M), as an offset from block 0's
    long long x_off[NB];
#pragma unroll
    for (int b = 0; b < NB; ++b) x_off[b] = (long long)((8 * b + g) % M - g % M) * p.K;
    int col = chunk * kChunkK + 16 * t;                 // this lane's first column in the unit
    const uint32_t q_off = 16 * lane, s_off = 4 * lane;
    int slot = 0;
    uint32_t parity = 0;
    int i = 0;                                          // units consumed
    uint32_t xf[NB][8];                                 // fast-path X
#pragma unroll
    for (int b = 0; b < NB; ++b)
#pragma unroll
        for (int k = 0; k < 8; ++k) xf[b][k] = 0u;
    for (int j = 0; j < n_stages; ++j) {
        if (!warp_wait(bar_s + 8 * slot, parity)) {
            // Give up: flag it, then wait (bounded) for the copies still in flight.
            if (lane == 0) atomicOr(&g_device_status, 1u);
            int s2 = slot;
            uint32_t p2 = parity;
            for (int j2 = j; j2 < n_stages && j2 < j + STAGES; ++j2) {
                warp_wait(bar_s + 8 * s2, p2);
                if (++s2 == STAGES) {
                    s2 = 0;
                    p2 ^= 1u;
                }
            }
            return;
        }
        const uint8_t* stage = ring + slot * kStage;
        if (n_units - i > UPS && kc_last - chunk >= UPS) {
            // Fast path: a full stage inside one tile that reaches neither the
            // tile's last chunk nor the end of the warp's range, so no unit
            // needs a bounds, tile-end or range-end check.
#pragma unroll
            for (int v = 0; v < UPS; ++v) {
#pragma unroll
                for (int b = 0; b < NB; ++b) ld_x32_keep(xp + x_off[b] + v * kChunkK, true, xf[b]);
                const uint8_t* sq = stage + v * kUnitQ + q_off;
                const uint8_t* ss = stage + UPS * kUnitQ + v * kUnitS + s_off;
#pragma unroll
                for (int mat = 0; mat < NW; ++mat)
                    mma_unit_nb<NB>(sq + mat * kMatStage, ss + mat * kMatStage, xf,
                                    *reinterpret_cast<float(*)[NB][2][4]>(acc + mat * NB));
            }
            i += UPS;
            chunk += UPS;
            col += UPS * kChunkK;
            xp += UPS * kChunkK;
        } else {
#pragma unroll 1
        for (int v = 0; v < UPS; ++v) {
            if (i < n_units) {
                // This lane's 16 columns of X (zeros past K).
                uint32_t xw[NB][8];
#pragma unroll
                for (int b = 0; b < NB; ++b) ld_x32(xp + x_off[b], col < K32, xw[b]);
                const uint8_t* sq = stage + v * kUnitQ + q_off;
                const uint8_t* ss = stage + UPS * kUnitQ + v * kUnitS + s_off;
#pragma unroll
                for (int mat = 0; mat < NW; ++mat)
                    mma_unit_nb<NB>(sq + mat * kMatStage, ss + mat * kMatStage, xw,
                                    *reinterpret_cast<float(*)[NB][2][4]>(acc + mat * NB));
                ++i;
                const bool tile_end = chunk == kc_last;
                if (tile_end || i == n_units) {
                    if constexpr (NW == 2) {
                        // Partial slot: 0 for the tile this warp's range starts in, 1 for a later one.
                        const int slot_id = (tile == first_tile) ? 0 : 1;
                        float* dst = p.legacy_partials + ((size_t)gw * 2 + slot_id) * kLegacyStride<NA> + lane * (NA * 8);
#pragma unroll
                        for (int a = 0; a < NA; ++a)
#pragma unroll
                            for (int r = 0; r < 2; ++r)
                                reinterpret_cast<float4*>(dst)[a * 2 + r] =
                                    make_float4(acc[a][r][0], acc[a][r][1], acc[a][r][2], acc[a][r][3]);
                        OutArgs o;
                        o.out = p.out;
                        o.partials = p.legacy_partials;
                        o.counters = p.counters;
                        o.N = p.N;
                        o.units = p.units;
                        o.total_warps = p.total_warps;
                        o.k_chunks = p.k_chunks;
                        o.gs0 = p.gs[0];
                        o.gs1 = p.gs[1];
                        // At the end of the range every stage has been consumed and no copy is
                        // in flight, so the ring can take the partial sums of a combine.
                        tile_done_global<M, NW>(o, tile, lane, i == n_units ? ring_s : 0u, STAGES * kStage, gather_bar);
                    } else {
                        AccPack<NA> pk;
#pragma unroll
                        for (int x = 0; x < NA; ++x)
#pragma unroll
                            for (int r = 0; r < 2; ++r)
#pragma unroll
                                for (int k = 0; k < 4; ++k) pk.v[x][r][k] = acc[x][r][k];
                        flush_tile<M, NW, STAGES, UPS, W>(p, tile, pk, lane, warp);
                    }
#pragma unroll
                    for (int a = 0; a < NA; ++a)
#pragma unroll
                        for (int r = 0; r < 2; ++r)
#pragma unroll
                            for (int k = 0; k < 4; ++k) acc[a][r][k] = 0.f;
                }
                if (tile_end) {
                    ++tile;
                    chunk = 0;
                    col = 16 * t;
                    xp -= kc_last * kChunkK;                 // back to column 16t of the same row
                } else {
                    ++chunk;
                    col += kChunkK;
                    xp += kChunkK;
                }
            }
        }
        }
        // The MMAs above consumed every word read from this stage, so the
        // stage can be refilled.
        __syncwarp();
        if (lane == 0 && j + STAGES < n_stages) issue(j + STAGES, slot);
        if (++slot == STAGES) {
            slot = 0;
            parity ^= 1u;
        }
    }
}

// ------------------------------------------------------------------ persistent round
//
// The whole decode round as one cooperative launch: every warp walks the
// nodes in order.  A GEMM node is done as a standalone launch would do it
// (same stream-K partition); the fused gate/up node becomes one GEMM node
// over both matrices stacked (gate rows, then up rows, into an FP32 buffer)
// followed by an elementwise node H = bf16(silu(g) * u).  Each warp's
// bulk-copy ring runs across node boundaries, so the next node's weights
// (which depend on nothing) stream in while the current node drains.  Between
// nodes the grid synchronises hierarchically: the warps of a CTA meet at a CTA
// barrier, one thread per CTA counts the CTA in at the node's counter and
// polls (bounded) until every CTA has, and a second CTA barrier releases the
// warps.  All CTAs are co-resident (cooperative launch), so no wait depends on
// a CTA that cannot run.

enum { kNodeGemm = 0, kNodeSiluMul = 1 };

struct RoundNode {
    const uint8_t* wq[2];  // GEMM: planes A (units below split_units) and B
    const uint8_t* ws[2];
    const void* X;         // GEMM: bf16 [M][K];  SiLU-mul: FP32 [M][2*K] (g rows, then u rows)
    void* out;             // GEMM: FP32 [M][N];  SiLU-mul: bf16 [M][N]
    float gs[2];           // GEMM: global scale (gs[0]);  SiLU-mul: gate and up scales
    int N, K, k_chunks, units, total_warps, split_units;
    int kind;
};

// Passed whole as the kernel's parameter block (constant bank), so node
// fields cost no registers; up to kMaxRoundNodes nodes per launch.
constexpr int kMaxRoundNodes = 360;

struct RoundParams {
    float* partials;
    unsigned* counters;
    unsigned* arrive;  // per node: CTAs of the grid that finished it
    int n_nodes;
    int grid_ctas;
    RoundNode nodes[kMaxRoundNodes];
};

constexpr int kRoundStages = 3;
constexpr int kRoundUPS = 4;                        // GEMM units per stage
constexpr int kRoundStageBytes = kRoundUPS * kUnitBytes;

// Coherent 32-byte X load (X may have been written earlier in this launch).
__device__ __forceinline__ void ld_x32_coherent(const void* p, bool pred, uint32_t (&x)[8])
{
    asm volatile(
        "{\n .reg .pred q;\n setp.ne.u32 q, %9, 0;\n"
        " @q ld.global.v4.u32 {%0,%1,%2,%3}, [%8];\n"
        " @q ld.global.v4.u32 {%4,%5,%6,%7}, [%8+16];\n}"
        : "+r"(x[0]), "+r"(x[1]), "+r"(x[2]), "+r"(x[3]), "+r"(x[4]), "+r"(x[5]), "+r"(x[6]), "+r"(x[7])
        : "l"(p), "r"((uint32_t)pred)
        : "memory");
}

// The bulk-copy side of a warp: which GEMM node and stage it issues next.
// Lives in shared memory and is read and written by lane 0 only, so the
// streaming loop carries none of it in registers.
struct RoundIssuer {
    int node, stage, n_stages, n_units;
    int issued;  // stages issued so far (for the drain on the error path)
    int u0;
};

// Move the issuer to the first GEMM node >= n where this warp has work (lane 0).
__device__ __forceinline__ void issuer_seek(const RoundParams& rp, int gw, int n, RoundIssuer* is)
{
    for (; n < rp.n_nodes; ++n) {
        const RoundNode& nd = rp.nodes[n];
        if (nd.kind != kNodeGemm || gw >= nd.total_warps) continue;
        const long long u0 = range_begin(nd.units, nd.total_warps, gw);
        const long long u1 = range_begin(nd.units, nd.total_warps, gw + 1);
        is->node = n;
        is->stage = 0;
        is->u0 = (int)u0;
        is->n_units = (int)(u1 - u0);
        is->n_stages = (is->n_units + kRoundUPS - 1) / kRoundUPS;
        return;
    }
    is->node = rp.n_nodes;
}

// Issue the issuer's next stage into `slot` (lane 0 only).  A stage that
// crosses from plane A to plane B is fetched with one copy from each.
__device__ __forceinline__ void issuer_issue(const RoundParams& rp, int gw, uint32_t ring_s, uint32_t bar_s,
                                             int slot, RoundIssuer* is)
{
    if (is->node >= rp.n_nodes) return;
    const RoundNode& nd = rp.nodes[is->node];
    const int ub = is->u0 + is->stage * kRoundUPS;
    const int rem = is->n_units - is->stage * kRoundUPS;
    const int cnt = rem < kRoundUPS ? rem : kRoundUPS;
    const uint32_t dst = ring_s + slot * kRoundStageBytes;
    const uint32_t bar = bar_s + 8 * slot;
    const uint64_t pol = evict_first_policy();
    mbar_expect_tx(bar, (uint32_t)(cnt * kUnitBytes));
    const int split = nd.split_units;
    const int na = ub >= split ? 0 : (split - ub < cnt ? split - ub : cnt);  // units from plane A
    if (na > 0) {
        bulk_load(dst, nd.wq[0] + (long long)ub * kUnitQ, na * kUnitQ, bar, pol);
        bulk_load(dst + kRoundUPS * kUnitQ, nd.ws[0] + (long long)ub * kUnitS, na * kUnitS, bar, pol);
    }
    if (cnt > na) {
        const long long b0 = (long long)(ub + na - split);
        bulk_load(dst + na * kUnitQ, nd.wq[1] + b0 * kUnitQ, (cnt - na) * kUnitQ, bar, pol);
        bulk_load(dst + kRoundUPS * kUnitQ + na * kUnitS, nd.ws[1] + b0 * kUnitS, (cnt - na) * kUnitS, bar, pol);
    }
    ++is->issued;
    if (++is->stage == is->n_stages) issuer_seek(rp, gw, is->node + 1, is);
}

// This warp's stream-K range of one GEMM node.  Mirrors the standalone
// kernel's loop; the ring (slot, parity) and the issuer carry over between
// nodes.
template <int M>
__device__ __forceinline__ bool round_gemm(const RoundParams& rp, const RoundNode* cur, int gw, int lane,
                                           uint8_t* ring, uint32_t ring_s, uint32_t bar_s, int& slot,
                                           uint32_t& parity, RoundIssuer* is, int& consumed)
{
    const RoundNode& nd = *cur;
    constexpr int UPS = kRoundUPS;
    const int g = lane >> 2, t = lane & 3;
    const long long TW = nd.total_warps, KC = nd.k_chunks;
    const long long u0 = range_begin(nd.units, TW, gw), u1 = range_begin(nd.units, TW, gw + 1);
    const int n_units = (int)(u1 - u0);
    const int n_stages = (n_units + UPS - 1) / UPS;
    float acc[1][2][4];
#pragma unroll
    for (int r = 0; r < 2; ++r)
#pragma unroll
        for (int i = 0; i < 4; ++i) acc[0][r][i] = 0.f;
    long long tile = u0 / KC;
    const long long first_tile = tile;
    int chunk = (int)(u0 - tile * KC);
    const int kc_last = (int)KC - 1;
    const int K32 = nd.K;
    // past M a lane loads row g % M, which feeds only dropped output columns
    const uint16_t* xp = static_cast<const uint16_t*>(nd.X) + (long long)(g % M) * nd.K + chunk * kChunkK + 16 * t;
    int col = chunk * kChunkK + 16 * t;
    const uint32_t q_off = 16 * lane, s_off = 4 * lane;
    uint32_t xf[8] = {0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u};
    int i = 0;
    for (int j = 0; j < n_stages; ++j) {
        if (!warp_wait(bar_s + 8 * slot, parity)) return false;
        ++consumed;
        const uint8_t* stage = ring + slot * kRoundStageBytes;
        if (n_units - i > UPS && kc_last - chunk >= UPS) {
#pragma unroll
            for (int v = 0; v < UPS; ++v) {
                ld_x32_coherent(xp + v * kChunkK, true, xf);
                mma_unit(stage + v * kUnitQ + q_off, stage + UPS * kUnitQ + v * kUnitS + s_off, xf, acc[0]);
            }
            i += UPS;
            chunk += UPS;
            col += UPS * kChunkK;
            xp += UPS * kChunkK;
        } else {
#pragma unroll 1
            for (int v = 0; v < UPS; ++v) {
                if (i < n_units) {
                    uint32_t xw[8] = {0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u};
                    ld_x32_coherent(xp, col < K32, xw);
                    mma_unit(stage + v * kUnitQ + q_off, stage + UPS * kUnitQ + v * kUnitS + s_off, xw, acc[0]);
                    ++i;
                    const bool tile_end = chunk == kc_last;
                    if (tile_end || i == n_units) {
                        const int slot_id = (tile == first_tile) ? 0 : 1;
                        float* dst = rp.partials + ((size_t)gw * 2 + slot_id) * kSlotFloats + lane * 8;
#pragma unroll
                        for (int r = 0; r < 2; ++r)
                            reinterpret_cast<float4*>(dst)[r] =
                                make_float4(acc[0][r][0], acc[0][r][1], acc[0][r][2], acc[0][r][3]);
                        // Node fields for the epilogue come from shared memory here, so the
                        // streaming loop does not keep them in registers.
                        volatile const RoundNode* vn = cur;
                        OutArgs o;
                        o.out = vn->out;
                        o.partials = rp.partials;
                        o.counters = rp.counters;
                        o.N = vn->N;
                        o.units = vn->units;
                        o.total_warps = vn->total_warps;
                        o.k_chunks = vn->k_chunks;
                        o.gs0 = vn->gs[0];
                        o.gs1 = vn->gs[1];
                        tile_done_round<M>(o, tile, lane);
#pragma unroll
                        for (int r = 0; r < 2; ++r)
#pragma unroll
                            for (int k = 0; k < 4; ++k) acc[0][r][k] = 0.f;
                    }
                    if (tile_end) {
                        ++tile;
                        chunk = 0;
                        col = 16 * t;
                        xp -= kc_last * kChunkK;
                    } else {
                        ++chunk;
                        col += kChunkK;
                        xp += kChunkK;
                    }
                }
            }
        }
        __syncwarp();
        if (lane == 0) issuer_issue(rp, gw, ring_s, bar_s, slot, is);
        if (++slot == kRoundStages) {
            slot = 0;
            parity ^= 1u;
        }
    }
    return true;
}

// H[m][n] = bf16(silu(g) * u) with g = X[m][n] * gs[0], u = X[m][P + n] * gs[1]
// (P = nd.K; X holds the stacked GEMM's acc * 2^8, so each product is the
// single rounding the fused kernel's epilogue makes).
template <int M>
__device__ __forceinline__ void round_silu_mul(const RoundNode& nd, int gtid, int nthreads)
{
    const float* gu = static_cast<const float*>(nd.X);
    __nv_bfloat16* H = static_cast<__nv_bfloat16*>(nd.out);
    const int N = nd.N, P = nd.K;
    for (int e = gtid; e < M * N; e += nthreads) {
        const int m = e / N, n = e - m * N;
        float gv, uv;
        asm volatile("ld.global.f32 %0, [%1];" : "=f"(gv) : "l"(gu + (long long)m * 2 * P + n) : "memory");
        asm volatile("ld.global.f32 %0, [%1];" : "=f"(uv) : "l"(gu + (long long)m * 2 * P + P + n) : "memory");
        gv *= nd.gs[0];
        uv *= nd.gs[1];
        H[(long long)m * N + n] = __float2bfloat16_rn(gv / (1.0f + expf(-gv)) * uv);
    }
}

// Bounded wait until `*ctr >= target` (one thread, acquire semantics).
__device__ __forceinline__ bool wait_count_thread(const unsigned* ctr, unsigned target)
{
    for (uint32_t it = 0; it < kWaitLimit; ++it) {
        unsigned v;
        asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(ctr) : "memory");
        if (v >= target) return true;
        __nanosleep(32);
    }
    return false;
}

template <int M>
__global__ void __launch_bounds__(kWarps * 32, 1) round_kernel(const RoundParams rp)
{
    extern __shared__ __align__(128) uint8_t smem[];
    __shared__ RoundIssuer issuers[kWarps];
    __shared__ RoundNode cur_node;  // the node being worked on (copied by thread 0 at each node start)
    __shared__ int cta_ok;
    const int lane = threadIdx.x & 31;
    const int warp = threadIdx.x >> 5;
    const int gw = blockIdx.x * kWarps + warp;

    uint8_t* ring = smem + warp * (kRoundStages * kRoundStageBytes);
    const uint32_t ring_s = smem_addr(ring);
    const uint32_t bar_s = smem_addr(smem + kWarps * kRoundStages * kRoundStageBytes) + warp * kRoundStages * 8;
    RoundIssuer* is = issuers + warp;
    if (lane == 0) {
#pragma unroll
        for (int s = 0; s < kRoundStages; ++s) mbar_init(bar_s + 8 * s);
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        is->issued = 0;
        issuer_seek(rp, gw, 0, is);
        for (int s = 0; s < kRoundStages; ++s) issuer_issue(rp, gw, ring_s, bar_s, s, is);
    }
    if (threadIdx.x == 0) {
        cta_ok = 1;
        cur_node = rp.nodes[0];
    }
    __syncthreads();

    int slot = 0, consumed = 0;
    uint32_t parity = 0;
    bool ok = true;
    for (int c = 0; c < rp.n_nodes; ++c) {
        if (cur_node.kind == kNodeGemm) {
            if (gw < cur_node.total_warps)
                ok = round_gemm<M>(rp, &cur_node, gw, lane, ring, ring_s, bar_s, slot, parity, is, consumed);
        } else {
            round_silu_mul<M>(cur_node, blockIdx.x * blockDim.x + threadIdx.x, gridDim.x * blockDim.x);
        }
        if (!ok && lane == 0) atomicAnd(&cta_ok, 0);
        // Grid barrier: this CTA's warps meet, one thread counts the CTA in and
        // waits for all CTAs, then releases the CTA.  Every thread first makes
        // its own output stores visible at GPU scope.
        __threadfence();
        __syncthreads();
        if (threadIdx.x == 0) {
            __threadfence();
            atomicAdd(rp.arrive + c, 1u);
            if (cta_ok && !wait_count_thread(rp.arrive + c, (unsigned)rp.grid_ctas)) cta_ok = 0;
            __threadfence();
            if (c + 1 < rp.n_nodes) cur_node = rp.nodes[c + 1];
        }
        __syncthreads();
        if (!cta_ok) break;
    }
    if (threadIdx.x == 0 && cta_ok) {
        // The last CTA to get here resets the counters for the next launch.
        const unsigned done = atomicAdd(rp.arrive + rp.n_nodes, 1u);
        if (done == (unsigned)rp.grid_ctas - 1) {
            for (int k = 0; k <= rp.n_nodes; ++k) rp.arrive[k] = 0u;
        }
    }
    if (!cta_ok) {
        // Give up: flag it, then wait (bounded) for this warp's copies still in flight.
        if (threadIdx.x == 0) atomicOr(&g_device_status, 2u);
        __syncwarp();
        const int issued = is->issued;
        for (int s = consumed; s < issued; ++s) {
            warp_wait(bar_s + 8 * slot, parity);
            if (++slot == kRoundStages) {
                slot = 0;
                parity ^= 1u;
            }
        }
    }
}

// ------------------------------------------------------------------ host side

namespace {

// Two deep stages: the same bytes in flight per warp as three shallower ones,
// in fewer, larger bulk copies (measured faster on the round at every width).
constexpr int kStagesPlain = 2, kUnitsPerStagePlain = 6;
// Plain GEMMs at M = 5..8 with few units per warp (a layer's projections, not
// the head): three stages of 4 units, the same bytes in flight in smaller
// copies, so a warp starts on its first units sooner.
constexpr int kStagesPlainShort = 3, kUnitsPerStagePlainShort = 4;
constexpr int kShortMinM = 5, kShortMaxUnitsPerWarp = 32;
constexpr int kStagesFused = 2, kUnitsPerStageFused = 3;

// M = 9..32 (plain GEMM): NB = 2..4 blocks of 8 lanes.  Each block's X
// fragments and accumulators take registers, so the CTA runs fewer warps
// (12 for two or three blocks, 8 for four), each with a deeper ring for the
// same bytes in flight.
constexpr int kStagesWide = 2;
constexpr int wide_warps(int nb) { return nb <= 3 ? 12 : 8; }
constexpr int wide_units_per_stage(int nb) { return nb <= 3 ? 8 : 12; }

template <int M, int NW, bool SHORT = false>
struct KernelOf {
    static constexpr bool wide = M > kMaxM;
    static constexpr int nb = (M + 7) / 8;
    static constexpr int warps = wide ? wide_warps(nb) : kWarps;
    static constexpr int stages = wide ? kStagesWide : NW == 2 ? kStagesFused : SHORT ? kStagesPlainShort : kStagesPlain;
    static constexpr int ups = wide ? wide_units_per_stage(nb)
                               : NW == 2 ? kUnitsPerStageFused : SHORT ? kUnitsPerStagePlainShort : kUnitsPerStagePlain;
    static constexpr int acc_sets = kAccSets<M, NW>;
    static void* fn() { return (void*)decode_gemm_kernel<M, NW, stages, ups, warps>; }
    static size_t smem() { return SmemLayout<M, NW, stages, ups, warps>::kBytes; }
};

struct KernelInfo {
    void* fn = nullptr;
    size_t smem = 0;
    int warps = 0;
    int acc_sets = 0;       // accumulator sets per lane: a workspace slot holds acc_sets * 512 floats
    int blocks_per_sm = 0;  // filled on first use
};

template <int NW>
KernelInfo kernel_info_for(int M, bool short_stages)
{
    KernelInfo k;
    if constexpr (NW == 1) {
        if (short_stages) {
            switch (M) {
#define NVFP4_SHORT(m)                                     \
    case m:                                                \
        k.fn = KernelOf<m, 1, true>::fn();                 \
        k.smem = KernelOf<m, 1, true>::smem();             \
        k.warps = KernelOf<m, 1, true>::warps;             \
        k.acc_sets = KernelOf<m, 1, true>::acc_sets;       \
        return k;
                NVFP4_SHORT(5) NVFP4_SHORT(6) NVFP4_SHORT(7) NVFP4_SHORT(8)
#undef NVFP4_SHORT
            }
            return k;
        }
    }
    switch (M) {
#define NVFP4_CASE(m)                        \
    case m:                                  \
        k.fn = KernelOf<m, NW>::fn();        \
        k.smem = KernelOf<m, NW>::smem();    \
        k.warps = KernelOf<m, NW>::warps;    \
        k.acc_sets = KernelOf<m, NW>::acc_sets; \
        break;
        NVFP4_CASE(1) NVFP4_CASE(2) NVFP4_CASE(3) NVFP4_CASE(4)
        NVFP4_CASE(5) NVFP4_CASE(6) NVFP4_CASE(7) NVFP4_CASE(8)
    }
    if constexpr (NW == 1) {
        switch (M) {
            NVFP4_CASE(9) NVFP4_CASE(10) NVFP4_CASE(11) NVFP4_CASE(12)
            NVFP4_CASE(13) NVFP4_CASE(14) NVFP4_CASE(15) NVFP4_CASE(16)
            NVFP4_CASE(17) NVFP4_CASE(18) NVFP4_CASE(19) NVFP4_CASE(20)
            NVFP4_CASE(21) NVFP4_CASE(22) NVFP4_CASE(23) NVFP4_CASE(24)
            NVFP4_CASE(25) NVFP4_CASE(26) NVFP4_CASE(27) NVFP4_CASE(28)
            NVFP4_CASE(29) NVFP4_CASE(30) NVFP4_CASE(31) NVFP4_CASE(32)
        }
    }
#undef NVFP4_CASE
    return k;
}

std::mutex g_mu;
DeviceState g_states[64];
KernelInfo g_kernels[64][2][kWideMaxM][2];  // [device][kind][M-1][short stages]

}  // namespace

int device_state(cudaStream_t stream, DeviceState** out)
{
    int dev = 0;
    NVFP4_CUDA_TRY(cudaGetDevice(&dev));
    if (dev < 0 || dev >= 64) return NVFP4_ERR_ARG;
    std::lock_guard<std::mutex> lock(g_mu);
    DeviceState& s = g_states[dev];
    if (s.device == dev) {
        *out = &s;
        return NVFP4_OK;
    }
    cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
    NVFP4_CUDA_TRY(cudaStreamIsCapturing(stream, &cs));
    if (cs != cudaStreamCaptureStatusNone) return NVFP4_ERR_CAPTURE;
    int sms = 0;
    NVFP4_CUDA_TRY(cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev));
    int max_threads = 0;
    NVFP4_CUDA_TRY(cudaDeviceGetAttribute(&max_threads, cudaDevAttrMaxThreadsPerMultiProcessor, dev));
    const int max_warps = sms * (max_threads / 32);
    float* partials = nullptr;
    unsigned* counters = nullptr;
    // two regions: the decode kernels' slots (which must start zeroed: their
    // ready flags), then the persistent round kernel's
    const size_t region = (size_t)max_warps * 2 * kSlotFloats;
    NVFP4_CUDA_TRY(cudaMalloc(&partials, 2 * region * sizeof(float)));
    cudaError_t e = cudaMalloc(&counters, (size_t)max_warps * sizeof(unsigned));
    if (e != cudaSuccess) {
        cudaFree(partials);
        return fail_cuda(e);
    }
    e = cudaMemset(counters, 0, (size_t)max_warps * sizeof(unsigned));
    if (e == cudaSuccess) e = cudaMemset(partials, 0, region * sizeof(float));
    if (e == cudaSuccess) e = cudaDeviceSynchronize();
    if (e != cudaSuccess) {
        cudaFree(partials);
        cudaFree(counters);
        return fail_cuda(e);
    }
    s.sm_count = sms;
    s.max_warps = max_warps;
    s.partials = partials;
    s.round_partials = partials + region;
    s.counters = counters;
    s.device = dev;
    *out = &s;
    return NVFP4_OK;
}

// Whether a plain GEMM of this width and shape takes the short-stage kernel.
static bool short_stages(int kind, int M, long long units, const DeviceState* ds)
{
    return kind == 0 && M >= kShortMinM && M <= kMaxM &&
           units < (long long)kShortMaxUnitsPerWarp * ds->sm_count * kWarps;
}

static int kernel_for(int dev, int kind, int M, bool shrt, KernelInfo** out)
{
    if (M < 1 || M > (kind == 0 ? kWideMaxM : kMaxM)) return NVFP4_ERR_M;
    std::lock_guard<std::mutex> lock(g_mu);
    KernelInfo& k = g_kernels[dev][kind][M - 1][shrt ? 1 : 0];
    if (k.blocks_per_sm == 0) {
        KernelInfo fresh = kind == 0 ? kernel_info_for<1>(M, shrt) : kernel_info_for<2>(M, false);
        if (!fresh.fn) return NVFP4_ERR_M;
        NVFP4_CUDA_TRY(cudaFuncSetAttribute(fresh.fn, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                            (int)fresh.smem));
        int nb = 0;
        NVFP4_CUDA_TRY(cudaOccupancyMaxActiveBlocksPerMultiprocessor(&nb, fresh.fn, fresh.warps * 32,
                                                                     fresh.smem));
        if (nb < 1) return NVFP4_ERR_CUDA;
        fresh.blocks_per_sm = nb;
        k = fresh;
    }
    *out = &k;
    return NVFP4_OK;
}

int prepare_kernel(DeviceState* ds, int kind, int M)
{
    KernelInfo* k = nullptr;
    int st = kernel_for(ds->device, kind, M, false, &k);
    if (st == NVFP4_OK && kind == 0 && M >= kShortMinM && M <= kMaxM) st = kernel_for(ds->device, kind, M, true, &k);
    return st;
}

int validate_gemm(const GemmArgs& a)
{
    if (a.kind != 0 && a.kind != 1) return NVFP4_ERR_ARG;
    const int nw = a.kind == 0 ? 1 : 2;
    if (!a.X || !a.out) return NVFP4_ERR_ARG;
    for (int i = 0; i < nw; ++i)
        if (!a.wq[i] || !a.ws[i]) return NVFP4_ERR_ARG;
    // the plain GEMM also takes M = 9..32 (two to four blocks of 8 lanes)
    int st = a.kind == 0 ? ((a.M >= 1 && a.M <= kWideMaxM) ? NVFP4_OK : NVFP4_ERR_M) : check_m(a.M);
    if (st != NVFP4_OK) return st;
    st = check_shape(a.N, a.K);
    if (st != NVFP4_OK) return st;
    if (!aligned16(a.X) || !aligned16(a.out)) return NVFP4_ERR_ALIGN;
    for (int i = 0; i < nw; ++i)
        if (!aligned16(a.wq[i]) || !aligned16(a.ws[i])) return NVFP4_ERR_ALIGN;
    return NVFP4_OK;
}

int launch_gemm(const GemmArgs& a, cudaStream_t stream, bool pdl, DeviceState* ds)
{
    const Geometry geo = geometry(a.N, a.K);
    KernelInfo* k = nullptr;
    int st = kernel_for(ds->device, a.kind, a.M, short_stages(a.kind, a.M, geo.units, ds), &k);
    if (st != NVFP4_OK) return st;
    const int W = k->warps;
    long long ctas = (long long)ds->sm_count * k->blocks_per_sm;
    const long long need = (geo.units + W - 1) / W;
    if (need < ctas) ctas = need;
    // The workspace holds max_warps warps of two 512-float slots; a warp of this
    // kernel takes acc_sets times that.
    const long long per_cta = (long long)W * k->acc_sets;
    if (ctas * per_cta > ds->max_warps) ctas = ds->max_warps / per_cta;
    if (ctas < 1) return NVFP4_ERR_SCRATCH;
    // Never more warps than units: every warp below total_warps gets a
    // non-empty range (the split-K combine relies on it).
    const long long total_warps = ctas * W < geo.units ? ctas * W : geo.units;

    KParams p;
    const int nw = a.kind == 0 ? 1 : 2;
    for (int i = 0; i < 2; ++i) {
        p.wq[i] = a.wq[i < nw ? i : 0];
        p.ws[i] = a.ws[i < nw ? i : 0];
        p.gs[i] = a.gscale[i < nw ? i : 0];
    }
    p.X = static_cast<const uint16_t*>(a.X);
    p.out = a.out;
    p.N = a.N;
    p.K = a.K;
    p.k_chunks = geo.k_chunks;
    p.units = geo.units;
    p.total_warps = total_warps;
    p.partials = ds->partials;
    p.counters = ds->counters;
    if (total_warps >= (1 << 16)) return NVFP4_ERR_SHAPE;  // kp_begin keeps r * w below 2^32
    p.legacy_partials = ds->round_partials;
    p.rb_q = geo.units / total_warps;
    p.rb_r = (unsigned)(geo.units % total_warps);

    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)ctas);
    cfg.blockDim = dim3(W * 32);
    cfg.dynamicSmemBytes = k->smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = pdl ? 1 : 0;
    void* args[] = {&p};
    NVFP4_CUDA_TRY(cudaLaunchKernelExC(&cfg, k->fn, args));
    return NVFP4_OK;
}

namespace {

template <int M>
void* round_kernel_fn()
{
    return (void*)round_kernel<M>;
}

void* round_kernel_for(int M)
{
    switch (M) {
    case 1: return round_kernel_fn<1>();
    case 2: return round_kernel_fn<2>();
    case 3: return round_kernel_fn<3>();
    case 4: return round_kernel_fn<4>();
    case 5: return round_kernel_fn<5>();
    case 6: return round_kernel_fn<6>();
    case 7: return round_kernel_fn<7>();
    default: return round_kernel_fn<8>();
    }
}

constexpr size_t kRoundSmem = (size_t)kWarps * kRoundStages * (kRoundStageBytes + 8);

}  // namespace

int round_persistent_params_size() { return (int)sizeof(RoundParams); }
int round_persistent_max_nodes() { return kMaxRoundNodes; }

size_t round_persistent_temp_floats(const GemmArgs* nodes, int n)
{
    size_t need = 0;
    for (int i = 0; i < n; ++i)
        if (nodes[i].kind == 1) {
            const size_t p = (size_t)geometry(nodes[i].N, nodes[i].K).n_tiles * kTileN;
            if (2 * p * kMaxM > need) need = 2 * p * kMaxM;
        }
    return need;
}

// Expands descriptors into round nodes; a fused gate/up descriptor becomes a
// stacked GEMM node (into `temp`) plus a SiLU-multiply node.  Returns the
// node count in *count, or NVFP4_ERR_ARG if more than kMaxRoundNodes result.
int round_persistent_build(const GemmArgs* nodes, int n, DeviceState* ds, float* temp, void* params_host,
                           int* count)
{
    RoundParams* rp = static_cast<RoundParams*>(params_host);
    memset(rp, 0, sizeof(RoundParams));
    int k = 0;
    for (int i = 0; i < n; ++i) {
        const GemmArgs& a = nodes[i];
        const Geometry geo = geometry(a.N, a.K);
        const int fused = a.kind == 1;
        if (k + 1 + fused > kMaxRoundNodes) return NVFP4_ERR_ARG;
        GemmArgs g = a;
        g.kind = 0;
        long long rows = a.N;
        if (fused) rows = 2 * geo.n_tiles * (long long)kTileN;  // gate rows, then up rows (tile-padded)
        g.N = rows;
        long long warps = 0;
        int st = gemm_launch_warps(g, ds, &warps);
        if (st != NVFP4_OK) return st;
        const long long units = fused ? 2 * geo.units : geo.units;
        if (units > 0x7fffffffLL || rows > 0x7fffffffLL || a.K > 0x7fffffffLL) return NVFP4_ERR_SHAPE;
        RoundNode& r = rp->nodes[k++];
        r.kind = kNodeGemm;
        r.wq[0] = a.wq[0];
        r.ws[0] = a.ws[0];
        r.wq[1] = fused ? a.wq[1] : a.wq[0];
        r.ws[1] = fused ? a.ws[1] : a.ws[0];
        r.gs[0] = fused ? 1.0f : a.gscale[0];  // a stacked gate/up node leaves the scales to its SiLU node
        r.gs[1] = r.gs[0];
        r.X = a.X;
        r.out = fused ? (void*)temp : a.out;
        r.N = (int)rows;
        r.K = (int)a.K;
        r.k_chunks = (int)geo.k_chunks;
        r.units = (int)units;
        r.total_warps = (int)(warps < units ? warps : units);  // a standalone launch's partition
        r.split_units = (int)geo.units;
        if (fused) {
            RoundNode& h = rp->nodes[k++];
            memset(&h, 0, sizeof h);
            h.kind = kNodeSiluMul;
            h.X = temp;
            h.out = a.out;
            h.N = (int)a.N;
            h.K = (int)(geo.n_tiles * kTileN);
            h.gs[0] = a.gscale[0];
            h.gs[1] = a.gscale[1];
        }
    }
    rp->n_nodes = k;
    rp->partials = ds->round_partials;
    rp->counters = ds->counters;
    *count = k;
    return NVFP4_OK;
}

int round_persistent_prepare(DeviceState* ds, int M, int* grid)
{
    void* fn = round_kernel_for(M);
    NVFP4_CUDA_TRY(cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kRoundSmem));
    int nb = 0;
    NVFP4_CUDA_TRY(cudaOccupancyMaxActiveBlocksPerMultiprocessor(&nb, fn, kWarps * 32, kRoundSmem));
    if (nb < 1) return NVFP4_ERR_CUDA;
    *grid = ds->sm_count;  // one CTA per SM, all co-resident
    return NVFP4_OK;
}

int round_persistent_launch(void* params_host, unsigned* d_arrive, int M, int grid, cudaStream_t stream)
{
    RoundParams* rp = static_cast<RoundParams*>(params_host);
    rp->arrive = d_arrive;
    rp->grid_ctas = grid;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)grid);
    cfg.blockDim = dim3(kWarps * 32);
    cfg.dynamicSmemBytes = kRoundSmem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeCooperative;
    attr[0].val.cooperative = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    void* args[] = {rp};
    NVFP4_CUDA_TRY(cudaLaunchKernelExC(&cfg, round_kernel_for(M), args));
    return NVFP4_OK;
}

int gemm_launch_warps(const GemmArgs& a, DeviceState* ds, long long* warps)
{
    const Geometry geo = geometry(a.N, a.K);
    KernelInfo* k = nullptr;
    int st = kernel_for(ds->device, a.kind, a.M, short_stages(a.kind, a.M, geo.units, ds), &k);
    if (st != NVFP4_OK) return st;
    const int W = k->warps;
    long long ctas = (long long)ds->sm_count * k->blocks_per_sm;
    const long long need = (geo.units + W - 1) / W;
    if (need < ctas) ctas = need;
    *warps = ctas * W;
    return NVFP4_OK;
}

size_t gemm_workspace_floats_per_warp() { return 2 * (size_t)kSlotFloats; }

int read_and_clear_device_status(int* status)
{
    unsigned v = 0;
    NVFP4_CUDA_TRY(cudaDeviceSynchronize());
    NVFP4_CUDA_TRY(cudaMemcpyFromSymbol(&v, g_device_status, sizeof v));
    if (v != 0) {
        const unsigned zero = 0;
        NVFP4_CUDA_TRY(cudaMemcpyToSymbol(g_device_status, &zero, sizeof zero));
        int dev = 0;
        NVFP4_CUDA_TRY(cudaGetDevice(&dev));
        std::lock_guard<std::mutex> lock(g_mu);
        if (dev >= 0 && dev < 64 && g_states[dev].device == dev) {
            // a wait that gave up may have left counters raised and slots unconsumed
            NVFP4_CUDA_TRY(cudaMemset(g_states[dev].counters, 0,
                                      (size_t)g_states[dev].max_warps * sizeof(unsigned)));
            NVFP4_CUDA_TRY(cudaMemset(g_states[dev].partials, 0,
                                      (size_t)g_states[dev].max_warps * 2 * kSlotFloats * sizeof(float)));
        }
        NVFP4_CUDA_TRY(noalloc_clear_scratch());
        NVFP4_CUDA_TRY(cudaDeviceSynchronize());
    }
    *status = (int)v;
    return NVFP4_OK;
}

}  // namespace nvfp4

using namespace nvfp4;

extern "C" int nvfp4_gemm_decode(const void* X, int M, const uint8_t* wq_dev, const uint8_t* ws_dev,
                                 float gscale, float* Y, int64_t N, int64_t K, nvfp4_stream_t stream)
{
    // M = 33..64 run on the tensor-memory kernel; up to 32 on the register-MMA kernel (lane blocks past 8)
    if (M > kWideMaxM && M <= kVerifyMaxM) return launch_verify(X, M, wq_dev, ws_dev, gscale, Y, N, K, (cudaStream_t)stream);
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
    int st = validate_gemm(a);
    if (st != NVFP4_OK) return st;
    DeviceState* ds = nullptr;
    st = device_state((cudaStream_t)stream, &ds);
    if (st != NVFP4_OK) return st;
    return launch_gemm(a, (cudaStream_t)stream, false, ds);
}

extern "C" int nvfp4_gemm_gateup_silu(const void* X, int M, const uint8_t* wq_gate,
                                      const uint8_t* ws_gate, float gscale_gate, const uint8_t* wq_up,
                                      const uint8_t* ws_up, float gscale_up, void* H, int64_t Nff,
                                      int64_t K, nvfp4_stream_t stream)
{
    GemmArgs a = {};
    a.kind = 1;
    a.X = X;
    a.M = M;
    a.wq[0] = wq_gate;
    a.ws[0] = ws_gate;
    a.gscale[0] = gscale_gate;
    a.wq[1] = wq_up;
    a.ws[1] = ws_up;
    a.gscale[1] = gscale_up;
    a.out = H;
    a.N = Nff;
    a.K = K;
    int st = validate_gemm(a);
    if (st != NVFP4_OK) return st;
    DeviceState* ds = nullptr;
    st = device_state((cudaStream_t)stream, &ds);
    if (st != NVFP4_OK) return st;
    return launch_gemm(a, (cudaStream_t)stream, false, ds);
}
