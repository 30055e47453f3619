// verify.cu -- the decode GEMM at verify widths, M = 33..64 rows of X (up to
// 32 run on the decode kernel with several lane blocks).
//
// ignis README, "What sets it apart", "Speculative decoding (DFlash2)": each
// lane's drafts are verified in the same pass over the weights, so the GEMM
// takes lanes x (1 + drafts) rows of X -- up to 8 x 8 = 64.  The format and
// the result are those of the decode kernel (ignis, "Models and artifacts",
// "The artifact": 4-bit floating point with one scale per 16 values):
//     Y[m][n] = gscale * sum_k x[m][k] * e2m1(q[n][k]) * e4m3(s[n][k/16]).
//
// At these widths the product no longer fits the register MMA path, so the
// multiply runs on the fifth-generation tensor cores (tcgen05) with both the
// accumulators and the A operand in tensor memory:
//   * A CTA (one per SM) owns a contiguous range of (512-row tile group,
//     64-column chunk) units -- stream-K at CTA granularity -- so every SM
//     gets the same number of weight bytes, whatever the shape.
//   * Sixteen dequantisation warps each stream one 32-row tile of the group
//     through their own ring of 1-D bulk copies, dequantise it exactly (the
//     same bit placement and bf16 scale multiply as the decode kernel) and
//     store it as bf16 into tensor memory with one tcgen05.st per row group:
//     the 16x256b store shape takes the m16n8k16 A fragment as it stands,
//     so the MMA's k order is the fragment's (per step s, k = 4t + j is the
//     chunk's column 16t + 4s + j).  They also stage the chunk of X (the
//     MMA's N side, M rows padded to a multiple of 16) in shared memory in
//     that k order.  A and X are double-buffered; keeping A out of shared
//     memory leaves its bandwidth to the weight ring and X.
//   * One thread of a seventeenth warp issues tcgen05.mma (M = 128, N =
//     16..64, K = 16; four per tile and chunk) into four accumulators in
//     tensor memory and commits each chunk to an mbarrier that frees its
//     buffers.  (The commit latency is paid once per chunk, so the more rows
//     a chunk carries, the less of it shows.)
//   * At the end of a tile group's K range the dequantisation warps read the
//     accumulators back (tcgen05.ld) and write Y, or, for a group split
//     between CTAs, a partial sum; the last CTA to finish a split group adds
//     the partials in CTA order (deterministic) and writes Y.
// Every wait is bounded; a wait that runs out flags the device status,
// stops the CTA's work, waits (bounded) for its copies and MMAs in flight,
// frees its tensor memory and returns.
#include <cuda_runtime.h>
#include <stdint.h>

#include <mutex>

#include "async.cuh"
#include "dequant.cuh"
#include "internal.h"
#include "layout.cuh"

namespace nvfp4 {

__device__ unsigned int g_verify_status;

namespace {

constexpr int kVTiles = 4;                     // 128-row tiles per CTA group (512 rows)
constexpr int kVWarps = 4 * kVTiles;           // dequantisation warps: one per 32-row tile
constexpr int kVCtasPerSM = 1;                 // one CTA per SM: shared memory holds its operands
constexpr int kVBufs = 2;                      // operand (A, X) buffers: chunks in flight to the tensor cores
constexpr int kVThreads = (kVWarps + 1) * 32;  // + the MMA / tensor-memory warp
constexpr int kVStages = 6;                    // per-warp ring depth, one unit per stage
constexpr int kVTileRows = 128;                // MMA M
constexpr int kVMaxNL = 64;                    // MMA N at most (M rows of X, padded to 16)
constexpr int kXBytes = kVMaxNL * kChunkK * 2;     // one chunk of X: 8 KB
static_assert(kVMaxNL * 8 <= kVWarps * 32, "each dequantisation thread stages at most one 16-byte piece of X");
// Tensor memory (512 columns): accumulators in columns [0, 4 * nl) (nl <= 64),
// the bf16 A operand from column 256: per buffer and tile, 128 lanes x 32
// columns (a chunk's 64 values per row, two per column).
constexpr int kVTmemCols = 512;
constexpr int kATmemCol = kVTiles * kVMaxNL;       // 256
constexpr int kATmemTileCols = kChunkK / 2;        // 32
constexpr int kVGroupRows = kVTiles * kVTileRows;  // 512
constexpr int kVSlotFloats = kVMaxNL * kVGroupRows;  // a partial: [512 rows][64 m] floats
constexpr int kVMaxGroups = 1 << 16;                // tile groups a call may have
constexpr int kVMaxSplit = 4;                      // CTAs per tile group at most, on average

// shared-memory map (bytes)
constexpr int kOffX = 0;                                   // [kVBufs buffers][8 KB]
constexpr int kOffRing = kOffX + kVBufs * kXBytes;         // [kVWarps warps][kVStages stages][1152 B]
constexpr int kOffBar = kOffRing + kVWarps * kVStages * kUnitBytes;
// barriers: ring[8][3], full[2], empty[2], acc, acc_free, part_done, last_ready, fin
constexpr int kBarRing = 0, kBarFull = kVWarps * kVStages, kBarEmpty = kBarFull + kVBufs, kBarAcc = kBarEmpty + kVBufs,
              kBarAccFree = kBarAcc + 1, kBarPart = kBarAccFree + 1, kBarLast = kBarPart + 1,
              kBarFin = kBarLast + 1, kNumBars = kBarFin + 1;
constexpr int kOffMisc = kOffBar + kNumBars * 8;            // tmem base, abort, last, pad
constexpr int kVSmemBytes = kOffMisc + 16;

struct VParams {
    const uint8_t* wq;
    const uint8_t* ws;
    const uint16_t* X;
    float* Y;
    float* part;         // [ctas][2 slots][64][256]
    unsigned* counters;  // [groups]
    float gscale;
    int M, NL, tmem_cols;
    long long N, K;
    int KC, n_tiles32, n_groups;
    long long units, ctas;  // stream-K over units = n_groups * KC
    uint32_t idesc;
};

__device__ __forceinline__ long long vrange_begin(long long units, long long t, long long i)
{
    return units * i / t;
}
__device__ __forceinline__ long long vrange_owner(long long units, long long t, long long x)
{
    return ((x + 1) * t - 1) / units;
}

// K-major operand in shared memory without swizzle: 8-row core matrices of
// 16-byte rows; the two k-octets of one K = 16 step are 128 bytes apart
// (leading byte offset) and consecutive 8-row groups 1024 bytes apart
// (stride byte offset), i.e. [row/8][k/8][row%8][16 B] over a 64-column chunk.
__device__ __forceinline__ uint64_t kmajor_desc(uint32_t saddr)
{
    return (uint64_t)((saddr >> 4) & 0x3FFFu) | ((uint64_t)(128u >> 4) << 16) | ((uint64_t)(1024u >> 4) << 32) |
           ((uint64_t)1 << 46);  // descriptor version for this architecture; no swizzle, base offset 0
}
__device__ __forceinline__ uint32_t kmajor_off(int row, int octet)
{
    return (uint32_t)((row >> 3) * 1024 + octet * 128 + (row & 7) * 16);
}

__device__ __forceinline__ void st_shared_v2(uint32_t a, uint32_t x, uint32_t y)
{
    asm volatile("st.shared.v2.b32 [%0], {%1,%2};" ::"r"(a), "r"(x), "r"(y) : "memory");
}

// 16 lanes x 4 x 256 bits of this warp's lane quarter from registers: register
// 4i + j goes to lane (taddr's lane) + (t / 4) + 8 * (j / 2), column (taddr's
// column) + 8i + 2 * (t % 4) + (j % 2), for thread t -- the layout of the
// m16n8k16 A fragment, so a lane's dequantised words go out as they are.
__device__ __forceinline__ void tc_st_16x256b_x4(uint32_t taddr, const uint32_t (&v)[16])
{
    asm volatile(
        "tcgen05.st.sync.aligned.16x256b.x4.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};" ::"r"(
            taddr),
        "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7]), "r"(v[8]), "r"(v[9]),
        "r"(v[10]), "r"(v[11]), "r"(v[12]), "r"(v[13]), "r"(v[14]), "r"(v[15])
        : "memory");
}

__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }

// D[tmem] (+)= A[tmem] . B[smem]^T, bf16 x bf16 -> f32, no output lane disabled.
__device__ __forceinline__ void tc_mma_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t bdesc, uint32_t idesc,
                                          uint32_t accumulate)
{
    asm volatile(
        "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n"
        " tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, {%5, %6, %7, %8}, p;\n}" ::"r"(d_tmem),
        "r"(a_tmem), "l"(bdesc), "r"(idesc), "r"(accumulate), "r"(0u), "r"(0u), "r"(0u), "r"(0u)
        : "memory");
}

// Arrive on `bar` once every tcgen05 operation this thread issued so far is done.
__device__ __forceinline__ void tc_commit(uint32_t bar)
{
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar)
                 : "memory");
}

// 16 consecutive 32-bit columns of this warp's 32 lanes.
__device__ __forceinline__ void tc_ld16(uint32_t taddr, uint32_t (&v)[16])
{
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
        : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]), "=r"(v[7]),
          "=r"(v[8]), "=r"(v[9]), "=r"(v[10]), "=r"(v[11]), "=r"(v[12]), "=r"(v[13]), "=r"(v[14]), "=r"(v[15])
        : "r"(taddr)
        : "memory");
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

// Waits here are often long (operands, tensor-core commits), so the polls
// sleep (up to kVSleepNs each) rather than spin and take issue slots from the
// dequantisation warps; at most kVWaitLimit polls (about a second).
constexpr uint32_t kVSleepNs = 1000;
constexpr uint32_t kVWaitLimit = 1u << 20;

// Bounded wait of a whole warp that also gives up once the CTA aborted.
__device__ __forceinline__ bool vwait(uint32_t bar, uint32_t parity, const volatile int* abort)
{
    for (uint32_t it = 0; it < kVWaitLimit; ++it) {
        if (__all_sync(0xffffffffu, mbar_try_wait_sleep(bar, parity, kVSleepNs))) return true;
        if (*abort) return false;
    }
    return false;
}

// The same for one thread.
__device__ __forceinline__ bool vwait1(uint32_t bar, uint32_t parity, const volatile int* abort)
{
    for (uint32_t it = 0; it < kVWaitLimit; ++it) {
        if (mbar_try_wait_sleep(bar, parity, kVSleepNs)) return true;
        if (*abort) return false;
    }
    return false;
}

__device__ __forceinline__ void vabort(volatile int* abort, unsigned bit)
{
    *abort = 1;
    atomicOr(&g_verify_status, bit);
}

__global__ void __launch_bounds__(kVThreads, kVCtasPerSM) verify_kernel(const VParams p)
{
    extern __shared__ __align__(1024) uint8_t vsm[];
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const uint32_t base = smem_addr(vsm);
    const uint32_t bars = base + kOffBar;
    volatile int* misc = reinterpret_cast<volatile int*>(vsm + kOffMisc);  // [0] tmem base [1] abort [2] last
    volatile int* abort = misc + 1;
    const long long U = p.units, T = p.ctas, KC = p.KC;
    const long long cta = blockIdx.x;
    const long long u0 = vrange_begin(U, T, cta), u1 = vrange_begin(U, T, cta + 1);
    const int n = (int)(u1 - u0);  // this CTA's (group, chunk) units; >= 1 as ctas <= units

    if (tid == 0) {
        for (int i = 0; i < kNumBars; ++i) {
            const bool per_warp = (i >= kBarFull && i < kBarFull + kVBufs) || i == kBarAccFree || i == kBarPart;
            mbar_init(bars + 8 * i, per_warp ? (uint32_t)kVWarps : 1u);
        }
        misc[1] = 0;
        misc[2] = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    if (warp == kVWarps) {
        // tensor memory for the accumulators and the A operand (all 512 columns)
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(base + kOffMisc),
                     "r"(p.tmem_cols)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
        tc_fence_before();
    }
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = (uint32_t)misc[0];
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");

    if (warp < kVWarps) {
        const int w = warp;
        const uint8_t* ring = vsm + kOffRing + w * (kVStages * kUnitBytes);
        const uint32_t ring_s = base + kOffRing + w * (kVStages * kUnitBytes);
        const uint32_t rbar = bars + 8 * (kBarRing + w * kVStages);
        const uint64_t pol = evict_first_policy();
        // stage j <-> unit x = u0 + j: this warp's 32-row tile of that unit's group, one chunk
        auto tile_ok = [&](int j) { return ((u0 + j) / KC) * kVWarps + w < p.n_tiles32; };
        // (group, chunk) of unit u0 once; every later position advances incrementally
        const long long group0 = u0 / KC;
        const int c0 = (int)(u0 - group0 * KC);
        long long igroup = group0;  // the next stage to issue (lane 0), in stage order
        int ic = c0;
        auto issue = [&](int j) {  // lane 0; called for j = 0, 1, 2, ... in order
            const long long t32 = igroup * kVWarps + w;
            const long long unit = t32 * KC + ic;
            if (++ic == (int)KC) {
                ic = 0;
                ++igroup;
            }
            if (t32 >= p.n_tiles32) return;  // rows past N: no data, zeros below
            const int slot = j % kVStages;
            const uint32_t bar = rbar + 8 * slot;
            mbar_expect_tx(bar, (uint32_t)kUnitBytes);
            bulk_load(ring_s + slot * kUnitBytes, p.wq + unit * kUnitQ, kUnitQ, bar, pol);
            bulk_load(ring_s + slot * kUnitBytes + kUnitQ, p.ws + unit * kUnitS, kUnitS, bar, pol);
        };
        if (lane == 0) {
            const int npre = n < kVStages ? n : kVStages;
            for (int j = 0; j < npre; ++j) issue(j);
        }
        // X and the outputs come from / go to the previous kernel's buffers
        asm volatile("griddepcontrol.wait;" ::: "memory");

        // X pieces of this thread: piece pc = 16 bytes of row pc / 8, columns 8 (pc % 8)
        // .. +7 of a chunk (nl <= 64 rows: at most one piece per thread, 512 threads).
        // In the MMA's k order step s takes, as k = 4u + j (u = 0..3, j = 0..3), the
        // chunk's columns 16u + 4s + j -- the order in which the dequantised words go
        // to tensor memory -- so each 8-byte half of a piece (four columns) lands in
        // step s's octet u / 2, at byte 8 * (u % 2).  Everything but the chunk's column
        // and the buffer is fixed per thread, so it is worked out once here.
        const int pc = w * 32 + lane;
        const bool x_piece = pc < p.NL * 8;                  // this thread stages a piece
        const int x_row = pc >> 3, x_o = pc & 7;
        const bool x_row_ok = x_piece && x_row < p.M;        // rows past M stay zero
        const uint16_t* x_src = p.X + (long long)(x_row_ok ? x_row : 0) * p.K + 8 * x_o;
        uint32_t x_dst[2];
#pragma unroll
        for (int half = 0; half < 2; ++half) {
            const int c4 = 8 * x_o + 4 * half;  // first of the four columns
            const int u = c4 >> 4, st = (c4 >> 2) & 3;
            x_dst[half] = kmajor_off(x_piece ? x_row : 0, 2 * st + (u >> 1)) + 8 * (u & 1);
        }
        auto load_x = [&](int cc, uint4& xr) {
            xr = make_uint4(0u, 0u, 0u, 0u);
            if (x_row_ok && (long long)cc * kChunkK + 8 * x_o < p.K)
                xr = *reinterpret_cast<const uint4*>(x_src + (long long)cc * kChunkK);
        };
        auto store_x = [&](int bb, const uint4& xr) {
            if (x_piece) {
                const uint32_t xb = base + kOffX + bb * kXBytes;
                st_shared_v2(xb + x_dst[0], xr.x, xr.y);
                st_shared_v2(xb + x_dst[1], xr.z, xr.w);
            }
        };
        // X of the first chunk goes straight into buffer 0; every later chunk's X is
        // loaded at the top of the iteration before it and stored at that iteration's
        // end, once its buffer is free (the loads have landed by then).
        uint4 xr;
        load_x(c0, xr);
        store_x(0, xr);
        const int trow = 32 * (w & 3);  // first row of this warp in its 128-row tile
        const int tt = w >> 2;          // which tile of the group
        int seg = 0, split = 0;
        int pend_lo = n, pend_hi = n;   // ring stages issued but not consumed, for the abort drain
        long long group = group0;
        int c = c0;
        for (int j = 0; j < n; ++j) {
            const long long t32 = group * kVWarps + w;
            const bool valid = t32 < p.n_tiles32;
            const int slot = j % kVStages;
            if (j + 1 < n) load_x(c + 1 == (int)KC ? 0 : c + 1, xr);  // stored into the next buffer at this iteration's end
            uint32_t q[8] = {0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u};
            uint32_t sw = 0u;
            if (valid) {
                if (!vwait(rbar + 8 * slot, (uint32_t)((j / kVStages) & 1), abort)) {
                    if (lane == 0 && !*abort) vabort(abort, 1u);
                    pend_lo = j;
                    pend_hi = (j + kVStages < n) ? j + kVStages : n;
                    break;
                }
                const uint8_t* st = ring + slot * kUnitBytes;
                const uint4 q0 = *reinterpret_cast<const uint4*>(st + 16 * lane);
                const uint4 q1 = *reinterpret_cast<const uint4*>(st + 512 + 16 * lane);
                sw = *reinterpret_cast<const uint32_t*>(st + kUnitQ + 4 * lane);
                q[0] = q0.x; q[1] = q0.y; q[2] = q0.z; q[3] = q0.w;
                q[4] = q1.x; q[5] = q1.y; q[6] = q1.z; q[7] = q1.w;
            }
            const int b = j % kVBufs;  // buffer b is free: the previous iteration's end waited for it
            // A: this warp's 32 rows of its tile for this chunk, bf16, into tensor memory
            // (lanes = rows, two values per column).  Word s of row group r holds rows
            // 16r+g (a[s][0], a[s][2]) and 16r+g+8 (a[s][1], a[s][3]) at columns
            // 16t+4s+{0,1} and {2,3}: MMA step s, k = 4t + {0,1} and {2,3}, i.e. the
            // step's columns 2t and 2t + 1.
            const uint32_t acol = tmem + (uint32_t)(kATmemCol + (b * kVTiles + tt) * kATmemTileCols);
            uint32_t S[2][2] = {{0u, 0u}, {0u, 0u}};
            if (valid) scale_pairs(sw, S);
#pragma unroll
            for (int r = 0; r < 2; ++r) {
                uint32_t a[4][4];
#pragma unroll
                for (int s = 0; s < 4; ++s) {
                    if (valid) {
                        dequant_word(q[4 * r + s], S, r, a[s]);
                    } else {
                        a[s][0] = a[s][1] = a[s][2] = a[s][3] = 0u;
                    }
                }
                const uint32_t v[16] = {a[0][0], a[0][2], a[0][1], a[0][3], a[1][0], a[1][2], a[1][1], a[1][3],
                                        a[2][0], a[2][2], a[2][1], a[2][3], a[3][0], a[3][2], a[3][1], a[3][3]};
                tc_st_16x256b_x4(acol + ((uint32_t)(trow + 16 * r) << 16), v);
            }
            // the A stores are complete before the MMA thread is told
            asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
            tc_fence_before();
            // The tensor cores read A and X, and the next bulk copy writes this ring
            // slot, through the async proxy: order this warp's shared-memory accesses
            // first.  The slot is refilled only now, after the dequantisation above
            // consumed every word read from it.
            asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
            __syncwarp();
            if (lane == 0) {
                if (j + kVStages < n) issue(j + kVStages);
                mbar_arrive(bars + 8 * (kBarFull + b));
            }

            if (c == (int)KC - 1 || j == n - 1) {
                // end of this group's K range in this CTA: read the accumulators back
                if (!vwait(bars + 8 * kBarAcc, (uint32_t)(seg & 1), abort)) {
                    if (lane == 0 && !*abort) vabort(abort, 1u);
                    pend_lo = j + 1;
                    pend_hi = (j + 1 + kVStages < n) ? j + 1 + kVStages : n;
                    break;
                }
                tc_fence_after();
                const long long ps = group * KC;  // the group's first unit
                const bool whole = ps >= u0 && ps + KC <= u1;
                const long long row_g = t32 * 32 + lane;  // output row of this thread
                const uint32_t taddr = tmem + ((uint32_t)(32 * (w & 3)) << 16) + (uint32_t)(tt * p.NL);
                const int pslot = ps <= u0 ? 0 : 1;  // this CTA's first or last segment
                // a partial: this row's nl sums, contiguous ([512 rows][64] per slot)
                float* pdst = p.part + (cta * 2 + pslot) * (long long)kVSlotFloats + (w * 32 + lane) * kVMaxNL;
                for (int m0 = 0; m0 < p.NL; m0 += 16) {
                    uint32_t v[16];
                    tc_ld16(taddr + (uint32_t)m0, v);
                    if (!whole) {
#pragma unroll
                        for (int i = 0; i < 16; i += 4)
                            *reinterpret_cast<uint4*>(pdst + m0 + i) = make_uint4(v[i], v[i + 1], v[i + 2], v[i + 3]);
                    } else if (row_g < p.N) {
#pragma unroll
                        for (int i = 0; i < 16; ++i)
                            if (m0 + i < p.M) p.Y[(m0 + i) * p.N + row_g] = (__uint_as_float(v[i]) * kEpilogueScale) * p.gscale;
                    }
                }
                tc_fence_before();
                // Partials go to another CTA: each lane makes its own stores visible at GPU
                // scope before its warp signals (one thread's release does not cover the
                // other warps' stores still in flight).
                if (!whole) __threadfence();
                __syncwarp();
                if (lane == 0) mbar_arrive(bars + 8 * kBarAccFree);
                ++seg;
                if (!whole) {
                    // count the CTA in on the group; its last contributor adds every partial
                    const long long glo = vrange_owner(U, T, ps), ghi = vrange_owner(U, T, ps + KC - 1);
                    if (lane == 0) mbar_arrive(bars + 8 * kBarPart);
                    if (w == 0) {
                        if (!vwait(bars + 8 * kBarPart, (uint32_t)(split & 1), abort)) {
                            if (lane == 0 && !*abort) vabort(abort, 1u);
                        } else if (lane == 0) {
                            unsigned old;
                            asm volatile("atom.acq_rel.gpu.global.add.u32 %0, [%1], 1;"
                                         : "=r"(old)
                                         : "l"(p.counters + group)
                                         : "memory");
                            misc[2] = (old == (unsigned)(ghi - glo)) ? 1 : 0;
                            mbar_arrive(bars + 8 * kBarLast);
                        }
                    }
                    if (!vwait(bars + 8 * kBarLast, (uint32_t)(split & 1), abort)) {
                        if (lane == 0 && !*abort) vabort(abort, 1u);
                        pend_lo = j + 1;
                        pend_hi = (j + 1 + kVStages < n) ? j + 1 + kVStages : n;
                        break;
                    }
                    const int last = misc[2];
                    ++split;
                    if (last) {
                        // every contributor's partial of this row, in CTA order, 16 sums at a time
                        const int glo_slot = vrange_begin(U, T, glo) >= ps ? 0 : 1;
                        for (int m0 = 0; m0 < p.NL; m0 += 16) {
                            float sum[16];
#pragma unroll
                            for (int i = 0; i < 16; ++i) sum[i] = 0.f;
                            for (long long ci = glo; ci <= ghi; ++ci) {
                                const int sl = ci == glo ? glo_slot : 0;
                                const float4* src = reinterpret_cast<const float4*>(
                                    p.part + (ci * 2 + sl) * (long long)kVSlotFloats + (w * 32 + lane) * kVMaxNL + m0);
                                float4 v4[4];
#pragma unroll
                                for (int i = 0; i < 4; ++i) v4[i] = __ldcg(src + i);
#pragma unroll
                                for (int i = 0; i < 4; ++i) {
                                    sum[4 * i] += v4[i].x;
                                    sum[4 * i + 1] += v4[i].y;
                                    sum[4 * i + 2] += v4[i].z;
                                    sum[4 * i + 3] += v4[i].w;
                                }
                            }
                            if (row_g < p.N) {
#pragma unroll
                                for (int i = 0; i < 16; ++i)
                                    if (m0 + i < p.M) p.Y[(m0 + i) * p.N + row_g] = (sum[i] * kEpilogueScale) * p.gscale;
                            }
                        }
                        if (w == 0 && lane == 0) p.counters[group] = 0u;  // every contributor is in
                    }
                }
            }
            // the next chunk's buffers: wait until the MMAs that last read them are done,
            // then store its X (rows past M, columns past K: zero)
            if (j + 1 < n) {
                const int b1 = (j + 1) % kVBufs;  // last used by chunk j + 1 - kVBufs
                if (j + 1 >= kVBufs &&
                    !vwait(bars + 8 * (kBarEmpty + b1), (uint32_t)((((j + 1) / kVBufs) - 1) & 1), abort)) {
                    if (lane == 0 && !*abort) vabort(abort, 1u);
                    pend_lo = j + 1;
                    pend_hi = (j + 1 + kVStages < n) ? j + 1 + kVStages : n;
                    break;
                }
                // the MMAs that read this buffer's A (tensor memory) are done: later stores follow them
                tc_fence_after();
                store_x(b1, xr);
            }
            if (++c == (int)KC) {
                c = 0;
                ++group;
            }
        }
        // after an abort: wait (bounded) for this warp's copies still in flight
        for (int s = pend_lo; s < pend_hi; ++s)
            if (tile_ok(s)) warp_wait(rbar + 8 * (s % kVStages), (uint32_t)((s / kVStages) & 1));
    } else {
        if (lane == 0) {
            int seg = 0;
            bool any = false;
            int c = (int)(u0 % KC) - 1;
            for (int j = 0; j < n; ++j) {
                if (++c == (int)KC) c = 0;
                const int b = j % kVBufs;
                const bool first = j == 0 || c == 0;
                if (!vwait1(bars + 8 * (kBarFull + b), (uint32_t)((j / kVBufs) & 1), abort)) {
                    if (!*abort) vabort(abort, 2u);
                    break;
                }
                // the previous group's accumulators have been read back before they are overwritten
                if (first && seg > 0 && !vwait1(bars + 8 * kBarAccFree, (uint32_t)((seg - 1) & 1), abort)) {
                    if (!*abort) vabort(abort, 2u);
                    break;
                }
                tc_fence_after();
                const uint32_t xs = base + kOffX + b * kXBytes;
#pragma unroll
                for (int tt = 0; tt < kVTiles; ++tt) {
                    const uint32_t at = tmem + (uint32_t)(kATmemCol + (b * kVTiles + tt) * kATmemTileCols);
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk)
                        tc_mma_ts(tmem + (uint32_t)(tt * p.NL), at + (uint32_t)(8 * kk), kmajor_desc(xs + 256 * kk),
                                  p.idesc, (first && kk == 0) ? 0u : 1u);
                }
                any = true;
                tc_commit(bars + 8 * (kBarEmpty + b));
                if (c == (int)KC - 1 || j == n - 1) {
                    tc_commit(bars + 8 * kBarAcc);
                    ++seg;
                }
            }
            // every MMA finished before the tensor memory is released
            if (any) {
                tc_commit(bars + 8 * kBarFin);
                for (uint32_t it = 0; it < kWaitLimit && !mbar_try_wait(bars + 8 * kBarFin, 0u); ++it) {
                }
            }
        }
        __syncwarp();
    }
    tc_fence_before();
    __syncthreads();
    if (warp == kVWarps) {
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(p.tmem_cols)
                     : "memory");
    }
}

}  // namespace

namespace {

struct VerifyState {
    int device = -1;
    int sm_count = 0;
    int max_ctas = 0;
    float* part = nullptr;
    unsigned* counters = nullptr;
};
std::mutex g_vmu;
VerifyState g_vstate[64];

int verify_state(cudaStream_t stream, VerifyState** out)
{
    int dev = 0;
    NVFP4_CUDA_TRY(cudaGetDevice(&dev));
    if (dev < 0 || dev >= 64) return NVFP4_ERR_ARG;
    std::lock_guard<std::mutex> lock(g_vmu);
    VerifyState& s = g_vstate[dev];
    if (s.device == dev) {
        *out = &s;
        return NVFP4_OK;
    }
    cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
    NVFP4_CUDA_TRY(cudaStreamIsCapturing(stream, &cs));
    if (cs != cudaStreamCaptureStatusNone) return NVFP4_ERR_CAPTURE;
    int sms = 0;
    NVFP4_CUDA_TRY(cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev));
    const int max_ctas = kVCtasPerSM * sms;
    float* part = nullptr;
    unsigned* counters = nullptr;
    NVFP4_CUDA_TRY(cudaMalloc(&part, (size_t)max_ctas * 2 * kVSlotFloats * sizeof(float)));
    cudaError_t e = cudaMalloc(&counters, (size_t)kVMaxGroups * sizeof(unsigned));
    if (e == cudaSuccess) e = cudaMemset(counters, 0, (size_t)kVMaxGroups * sizeof(unsigned));
    if (e == cudaSuccess)
        e = cudaFuncSetAttribute(verify_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kVSmemBytes);
    if (e == cudaSuccess) e = cudaDeviceSynchronize();
    if (e != cudaSuccess) {
        cudaFree(part);
        if (counters) cudaFree(counters);
        return fail_cuda(e);
    }
    s.sm_count = sms;
    s.max_ctas = max_ctas;
    s.part = part;
    s.counters = counters;
    s.device = dev;
    *out = &s;
    return NVFP4_OK;
}

}  // namespace

int verify_geometry(int M, int64_t N, int64_t K, int sm_count, VerifyGeometry* g)
{
    if (M < kVerifyMinM || M > kVerifyMaxM) return NVFP4_ERR_M;
    int st = check_shape(N, K);
    if (st != NVFP4_OK) return st;
    g->n_tiles32 = (N + kTileN - 1) / kTileN;
    g->n_groups = (g->n_tiles32 + kVWarps - 1) / kVWarps;  // groups of kVWarps 32-row tiles
    if (g->n_groups > kVMaxGroups) return NVFP4_ERR_SHAPE;
    g->k_chunks = (K + kChunkK - 1) / kChunkK;
    g->units = g->n_groups * g->k_chunks;
    // one CTA per SM, but no more than kVMaxSplit CTAs per tile group on average: a group
    // split between more CTAs costs more in partial sums than the extra SMs stream
    long long ctas = (long long)kVCtasPerSM * sm_count;
    if (ctas > g->n_groups * kVMaxSplit) ctas = g->n_groups * kVMaxSplit;
    if (ctas > g->units) ctas = g->units;
    g->ctas = ctas;
    g->nl = (M + 15) / 16 * 16;
    g->tmem_cols = kVTmemCols;  // accumulators (4 x nl <= 256 columns) and the double-buffered A operand
    return NVFP4_OK;
}

int launch_verify(const void* X, int M, const uint8_t* wq, const uint8_t* ws, float gscale, float* Y, int64_t N,
                  int64_t K, cudaStream_t stream)
{
    if (!X || !wq || !ws || !Y) return NVFP4_ERR_ARG;
    if (M < kVerifyMinM || M > kVerifyMaxM) return NVFP4_ERR_M;
    int st = check_shape(N, K);
    if (st != NVFP4_OK) return st;
    if (!aligned16(X) || !aligned16(wq) || !aligned16(ws) || ((uintptr_t)Y & 3) != 0) return NVFP4_ERR_ALIGN;
    VerifyState* vs = nullptr;
    st = verify_state(stream, &vs);
    if (st != NVFP4_OK) return st;
    VerifyGeometry geo;
    st = verify_geometry(M, N, K, vs->sm_count, &geo);
    if (st != NVFP4_OK) return st;
    VParams p;
    p.wq = wq;
    p.ws = ws;
    p.X = static_cast<const uint16_t*>(X);
    p.Y = Y;
    p.part = vs->part;
    p.counters = vs->counters;
    p.gscale = gscale;
    p.M = M;
    p.NL = geo.nl;
    p.tmem_cols = geo.tmem_cols;
    p.N = N;
    p.K = K;
    p.KC = (int)geo.k_chunks;
    p.n_tiles32 = (int)geo.n_tiles32;
    p.n_groups = (int)geo.n_groups;
    p.units = geo.units;
    p.ctas = geo.ctas;
    // kind::f16 instruction: F32 accumulator, BF16 A and B, both K-major, N = nl, M = 128
    p.idesc = (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(geo.nl >> 3) << 17) | ((uint32_t)(kVTileRows >> 4) << 24);
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)geo.ctas);
    cfg.blockDim = dim3(kVThreads);
    cfg.dynamicSmemBytes = kVSmemBytes;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    NVFP4_CUDA_TRY(cudaLaunchKernelEx(&cfg, verify_kernel, p));
    return NVFP4_OK;
}

int read_and_clear_verify_status(unsigned* status)
{
    unsigned v = 0;
    NVFP4_CUDA_TRY(cudaDeviceSynchronize());
    NVFP4_CUDA_TRY(cudaMemcpyFromSymbol(&v, g_verify_status, sizeof v));
    if (v != 0) {
        const unsigned zero = 0;
        NVFP4_CUDA_TRY(cudaMemcpyToSymbol(g_verify_status, &zero, sizeof zero));
        int dev = 0;
        NVFP4_CUDA_TRY(cudaGetDevice(&dev));
        std::lock_guard<std::mutex> lock(g_vmu);
        if (dev >= 0 && dev < 64 && g_vstate[dev].device == dev)
            NVFP4_CUDA_TRY(cudaMemset(g_vstate[dev].counters, 0, (size_t)kVMaxGroups * sizeof(unsigned)));
        NVFP4_CUDA_TRY(cudaDeviceSynchronize());
    }
    *status = v;
    return NVFP4_OK;
}

}  // namespace nvfp4

extern "C" int nvfp4_verify_geometry(int M, int64_t N, int64_t K, int sm_count, int64_t* ctas, int64_t* units,
                                     int* nl)
{
    if (!ctas || !units || !nl || sm_count < 1) return NVFP4_ERR_ARG;
    nvfp4::VerifyGeometry g;
    const int st = nvfp4::verify_geometry(M, N, K, sm_count, &g);
    if (st != NVFP4_OK) return st;
    *ctas = g.ctas;
    *units = g.units;
    *nl = g.nl;
    return NVFP4_OK;
}
