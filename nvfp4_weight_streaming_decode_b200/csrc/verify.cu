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
//   * A first kernel (verify_xprep_kernel) writes X once per call in the
//     MMA's operand order (K-major 8 x 16-byte core matrices, the columns of
//     each 64-column chunk permuted to the order in which the dequantised
//     words reach tensor memory), so a CTA stages a hand-off's X with one
//     1-D bulk copy.
//   * A CTA (one per SM) owns a contiguous range of (256-row group, pair of
//     64-column chunks) units -- stream-K at CTA granularity -- so every SM
//     gets the same number of weight bytes, whatever the shape.  A unit is
//     one hand-off to the tensor cores.
//   * Eight dequantisation warps each stream one 32-row slice of the group
//     through their own ring of 1-D bulk copies (both units of a hand-off per
//     stage), read the next hand-off's codes while they dequantise this one
//     exactly (the same bit placement and bf16 scale multiply as the decode
//     kernel), and store it as bf16 into tensor memory with one tcgen05.st
//     per unit and row group: the 16x256b store shape takes the m16n8k16 A
//     fragment as it stands.
//   * Hand-offs rotate through three buffers: A in tensor memory, X in shared
//     memory.  Buffer b's full barrier takes the eight warps' arrivals and
//     X's bytes (one thread of an eleventh warp copies X); its free barrier
//     takes the commits of the MMAs that read it.
//   * Two issuing threads, one per 128-row tile and on two sub-partitions
//     (the issue competes with the dequantisation there), each wait for a
//     full buffer and issue tcgen05.mma (M = 128, N = 16..64, K = 16; eight
//     per tile and hand-off) into the tile's accumulator in tensor memory,
//     then commit to the buffer's free barrier.
//   * At the end of a group's K range the dequantisation warps read the
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

// 128-row MMA tiles per group.  (One tile with two CTAs per SM, each with half
// the tensor memory, measured faster on the head at M = 64 -- 203 against
// 210 us -- but slower where groups are few: down at M = 40 62 against 51 us.)
constexpr int kVTiles = 2;
constexpr int kVSlices = 4 * kVTiles;            // 32-row slices per group
constexpr int kVPair = 2;                        // 64-column chunks per hand-off
#ifndef NVFP4_VSPLIT
#define NVFP4_VSPLIT 1
#endif
constexpr int kVSplit = NVFP4_VSPLIT;            // dequantisation warps per slice, each on its share of the chunks
constexpr int kVWarps = kVSlices * kVSplit;
constexpr int kVUPW = kVPair / kVSplit;          // units per warp and hand-off
static_assert(kVPair % kVSplit == 0, "the chunks of a hand-off divide among a slice's warps");
constexpr int kVBufs = 3;                        // hand-offs in flight: A buffers (tensor memory), X buffers (shared)
constexpr int kVStages = kVTiles == 1 ? 6 : 7;   // per-warp ring depth, one hand-off per stage
constexpr int kVMmaWarp = kVWarps;               // one thread per tile issues its MMAs (warps kVWarps..)
constexpr int kVXWarp = kVWarps + kVTiles;       // one thread stages X
constexpr int kVThreads = (kVXWarp + 1) * 32;
constexpr int kVCtasPerSM = kVTiles == 1 ? 2 : 1;  // CTAs per SM, sharing the 512 tensor-memory columns
constexpr int kVTileRows = 128;                  // MMA M
constexpr int kVMaxNL = 64;                      // MMA N at most (M rows of X, padded to 16)
constexpr int kVGroupRows = kVTiles * kVTileRows;        // 256
constexpr int kVStageBytes = kVUPW * kUnitBytes;         // codes of the warp's units, then their scales
constexpr int kXChunkBytes = kVMaxNL * kChunkK * 2;      // one chunk of X at NL = 64: 8 KB
constexpr int kXBufBytes = kVPair * kXChunkBytes;        // 16 KB
// Tensor memory (512 columns): accumulators in columns [0, kVTiles * nl)
// (nl <= 64); the bf16 A operand from column 128: per buffer and tile, 128
// lanes x 64 columns (a hand-off's 128 values per row, two per column).
constexpr int kVTmemCols = 512 / kVCtasPerSM;
constexpr int kATmemCol = kVTiles * kVMaxNL;             // 128
constexpr int kATmemTileCols = kVPair * kChunkK / 2;     // 64
static_assert(kATmemCol + kVBufs * kVTiles * kATmemTileCols <= kVTmemCols, "tensor memory holds A and D");
static_assert(kVSlices * 32 == kVGroupRows, "one dequantisation thread per row of a group and warp share");
constexpr int kVSlotFloats = kVMaxNL * kVGroupRows;      // a partial: [256 rows][64 m] floats
constexpr int kVMaxGroups = 1 << 16;                     // groups a call may have
constexpr int kVMaxSplit = 8;                            // CTAs per group at most, on average
constexpr int kFinBatch = kVSplit == 1 ? 4 : 2;          // contributors' partials in flight in the final sum

// shared-memory map (bytes)
constexpr int kOffX = 0;                                          // [kVBufs][16 KB]
constexpr int kOffRing = kOffX + kVBufs * kXBufBytes;             // [kVWarps][kVStages][kVStageBytes]
constexpr int kOffBar = kOffRing + kVWarps * kVStages * kVStageBytes;
// full[b]: the dequantisation warps' arrivals and X's bytes for the hand-off in buffer b;
// free[b]: the MMAs that read buffer b are done (one commit)
constexpr int kBarRing = 0, kBarFull = kVWarps * kVStages, kBarFree = kBarFull + kVBufs, kBarAcc = kBarFree + kVBufs,
              kBarPart = kBarAcc + 1, kBarLast = kBarPart + 1, kBarFin = kBarLast + 1, kNumBars = kBarFin + 1;
constexpr int kOffMisc = kOffBar + kNumBars * 8;                  // tmem base, abort, last, pad
constexpr int kVSmemBytes = kOffMisc + 16;
static_assert(kVSmemBytes * kVCtasPerSM <= 226 * 1024, "shared memory per SM");

struct VParams {
    const uint8_t* wq;
    const uint8_t* ws;
    const uint8_t* Xp;   // X in the MMA's order: [chunk][nl / 8][8 octets][8 rows][16 B]
    float* Y;
    float* part;         // [ctas][2 slots][256 rows][64]
    unsigned* counters;  // [groups]
    float gscale;
    int M, NL, tmem_cols;
    long long N;
    int KC, KP, n_tiles32, n_groups;  // chunks, chunk pairs, 32-row tiles, groups
    long long units, ctas;            // stream-K over units = n_groups * KP
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

__device__ __forceinline__ uint64_t evict_last_policy()
{
    uint64_t pol;
    asm volatile("createpolicy.fractional.L2::evict_last.b64 %0, 1.0;" : "=l"(pol));
    return pol;
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

// Non-blocking test of a phase (cheaper than try_wait when it has completed,
// the common case for the ring and buffer waits).
__device__ __forceinline__ bool mbar_test(uint32_t bar, uint32_t parity)
{
    uint32_t ok;
    asm volatile(
        "{\n .reg .pred p;\n mbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n"
        " selp.u32 %0, 1, 0, p;\n}"
        : "=r"(ok)
        : "r"(bar), "r"(parity)
        : "memory");
    return ok != 0;
}

// Bounded wait of a whole warp that also gives up once the CTA aborted.
__device__ __forceinline__ bool vwait(uint32_t bar, uint32_t parity, const volatile int* abort)
{
    if (__all_sync(0xffffffffu, mbar_test(bar, parity))) return true;
    for (uint32_t it = 0; it < kVWaitLimit; ++it) {
        if (__all_sync(0xffffffffu, mbar_try_wait_sleep(bar, parity, kVSleepNs))) return true;
        if (*abort) return false;
    }
    return false;
}

// The same for one thread.
__device__ __forceinline__ bool vwait1(uint32_t bar, uint32_t parity, const volatile int* abort)
{
    if (mbar_test(bar, parity)) return true;
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

// X in the MMA's operand order, once per call: Xp[c] is chunk c (columns
// 64c..64c+63) as nl / 8 groups of 8 rows, each group 8 k-octets of 8 rows x
// 16 bytes (the K-major core matrices of kmajor_desc).  MMA step s of a chunk
// takes as its k = 4t + j (t, j = 0..3) the chunk's column 16t + 4s + j --
// the order in which the dequantised words reach tensor memory -- so octet
// 2s + h holds columns 32h + 4s + (0..3) and 32h + 16 + 4s + (0..3).  Rows
// past M and columns past K are zero.  One thread per 16-byte piece.
__global__ void __launch_bounds__(256) verify_xprep_kernel(const uint16_t* __restrict__ X, uint8_t* __restrict__ Xp,
                                                           int M, int NL, long long K, long long pieces)
{
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    // X comes from the preceding kernel, and the preceding verify kernel may still read Xp
    asm volatile("griddepcontrol.wait;" ::: "memory");
    const long long i = (long long)blockIdx.x * 256 + threadIdx.x;
    if (i >= pieces) return;
    const int r8 = (int)(i & 7), o = (int)((i >> 3) & 7);
    const long long rest = i >> 6;
    const int groups8 = NL >> 3;
    const int row = (int)(rest % groups8) * 8 + r8;
    const long long c = rest / groups8;
    uint2 lo = make_uint2(0u, 0u), hi = make_uint2(0u, 0u);
    if (row < M) {
        const long long col = c * kChunkK + 32 * (o & 1) + 4 * (o >> 1);
        const uint16_t* src = X + (long long)row * K + col;
        if (col < K) lo = *reinterpret_cast<const uint2*>(src);  // K % 16 == 0: all four columns exist
        if (col + 16 < K) hi = *reinterpret_cast<const uint2*>(src + 16);
    }
    *reinterpret_cast<uint4*>(Xp + i * 16) = make_uint4(lo.x, lo.y, hi.x, hi.y);
}

__global__ void __launch_bounds__(kVThreads, kVCtasPerSM) verify_kernel(const VParams p)
{
    extern __shared__ __align__(1024) uint8_t vsm[];
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const uint32_t base = smem_addr(vsm);
    const uint32_t bars = base + kOffBar;
    volatile int* misc = reinterpret_cast<volatile int*>(vsm + kOffMisc);  // [0] tmem base [1] abort [2] last
    volatile int* abort = misc + 1;
    const long long U = p.units, T = p.ctas;
    const int KC = p.KC, KP = p.KP;
    const long long cta = blockIdx.x;
    const long long u0 = vrange_begin(U, T, cta), u1 = vrange_begin(U, T, cta + 1);
    const int n = (int)(u1 - u0);  // this CTA's (group, chunk pair) units; >= 1 as ctas <= units
    const long long group0 = u0 / KP;
    const int pr0 = (int)(u0 - group0 * KP);

    if (tid == 0) {
        for (int i = 0; i < kNumBars; ++i) {
            const bool full = i >= kBarFull && i < kBarFull + kVBufs;
            const bool per_issuer = (i >= kBarFree && i < kBarFree + kVBufs) || i == kBarAcc || i == kBarFin;
            mbar_init(bars + 8 * i, full ? (uint32_t)(kVWarps + 1)
                                    : i == kBarPart ? (uint32_t)kVWarps
                                    : per_issuer    ? (uint32_t)kVTiles
                                                    : 1u);
        }
        misc[1] = 0;
        misc[2] = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    if (warp == kVMmaWarp) {
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
        const int slice = w % kVSlices;        // this warp's 32 rows of the group
        const int h0 = (w / kVSlices) * kVUPW;  // and its first chunk of each pair
        const uint8_t* ring = vsm + kOffRing + w * (kVStages * kVStageBytes);
        const uint32_t ring_s = base + kOffRing + w * (kVStages * kVStageBytes);
        const uint32_t rbar = bars + 8 * (kBarRing + w * kVStages);
        const uint64_t pol = evict_first_policy();
        // Stage j <-> unit u0 + j: this warp's slice of that unit's group, chunks
        // 2 pr + h0 .. + kVUPW - 1 of its pair pr that exist; the units it copies.
        auto stage_units = [&](long long x) {
            const long long g = x / KP;
            const int c0 = 2 * (int)(x - g * KP) + h0;
            const int nw = KC - c0 < kVUPW ? KC - c0 : kVUPW;
            return (g * kVSlices + slice < p.n_tiles32 && nw > 0) ? nw : 0;
        };
        long long igroup = group0;  // the next stage to issue (lane 0), in stage order
        int ipr = pr0;
        auto issue = [&](int j) {  // lane 0; called for j = 0, 1, 2, ... in order
            const long long t32 = igroup * kVSlices + slice;
            const int c0 = 2 * ipr + h0;
            if (++ipr == KP) {
                ipr = 0;
                ++igroup;
            }
            const int nw = KC - c0 < kVUPW ? KC - c0 : kVUPW;
            if (t32 >= p.n_tiles32 || nw <= 0) return;  // rows past N, chunks past K: no data
            const long long unit = t32 * KC + c0;  // a slice's units of one pair are consecutive
            const int slot = j % kVStages;
            const uint32_t bar = rbar + 8 * slot;
            mbar_expect_tx(bar, (uint32_t)(nw * kUnitBytes));
            bulk_load(ring_s + slot * kVStageBytes, p.wq + unit * kUnitQ, (uint32_t)(nw * kUnitQ), bar, pol);
            bulk_load(ring_s + slot * kVStageBytes + kVUPW * kUnitQ, p.ws + unit * kUnitS, (uint32_t)(nw * kUnitS),
                      bar, pol);
        };
        if (lane == 0) {
            const int npre = n < kVStages ? n : kVStages;
            for (int j = 0; j < npre; ++j) issue(j);
        }
        // the outputs and the workspace are the previous kernels' until they are done
        asm volatile("griddepcontrol.wait;" ::: "memory");

        const int trow = 32 * (slice & 3);  // first row of this warp in its 128-row tile
        const int tt = slice >> 2;          // which tile of the group
        int seg = 0, split = 0;
        // Ring bookkeeping for the abort drain: stages [0, issued) have been issued and
        // [0, waited) waited for, so the copies of [waited, issued) may be in flight.
        int issued = n < kVStages ? n : kVStages, waited = 0;
        // units this warp dequantises at (group, pair): none past N or past K
        auto units_at = [&](long long g, int prr) {
            const int nw0 = KC - (2 * prr + h0);
            return g * kVSlices + slice >= p.n_tiles32 ? 0 : nw0 < kVUPW ? (nw0 > 0 ? nw0 : 0) : kVUPW;
        };
        // the codes and scales of stage j (ring slot rslot, phase parity rpar) into
        // registers, after its ring wait; stages are loaded in order
        int rslot = 0;
        uint32_t rpar = 0;
        auto load_stage = [&](int j, int nwj, uint32_t (&qq)[kVUPW][8], uint32_t (&ss)[kVUPW]) {
            const int slot = rslot;
            const uint32_t par = rpar;
            if (++rslot == kVStages) {
                rslot = 0;
                rpar ^= 1u;
            }
            if (nwj > 0) {
                if (!__all_sync(0xffffffffu, mbar_test(rbar + 8 * slot, par)) && !warp_wait(rbar + 8 * slot, par))
                    return false;
                const uint8_t* st = ring + slot * kVStageBytes;
#pragma unroll
                for (int h = 0; h < kVUPW; ++h) {
                    if (h < nwj) {
                        const uint4 q0 = *reinterpret_cast<const uint4*>(st + h * kUnitQ + 16 * lane);
                        const uint4 q1 = *reinterpret_cast<const uint4*>(st + h * kUnitQ + 512 + 16 * lane);
                        ss[h] = *reinterpret_cast<const uint32_t*>(st + kVUPW * kUnitQ + h * kUnitS + 4 * lane);
                        qq[h][0] = q0.x; qq[h][1] = q0.y; qq[h][2] = q0.z; qq[h][3] = q0.w;
                        qq[h][4] = q1.x; qq[h][5] = q1.y; qq[h][6] = q1.z; qq[h][7] = q1.w;
                    }
                }
            }
            waited = j + 1;
            return true;
        };
        long long group = group0;
        int pr = pr0;
        int nw = units_at(group, pr);
        // The next hand-off's codes are read one iteration ahead: its ring wait and
        // loads overlap this hand-off's dequantisation.
        uint32_t q[kVUPW][8], sw[kVUPW];
        bool ok = load_stage(0, nw, q, sw);
        int ab = 0;         // A buffer of hand-off j: j % kVBufs
        uint32_t apar = 0;  // (j / kVBufs) & 1: the buffer's use j - kVBufs completed phase apar ^ 1
        for (int j = 0; ok && j < n; ++j) {
            const long long t32 = group * kVSlices + slice;
            long long group1 = group;
            int pr1 = pr + 1;
            if (pr1 == KP) {
                pr1 = 0;
                ++group1;
            }
            int nw1 = 0;
            uint32_t q1[kVUPW][8], sw1[kVUPW];
            if (j + 1 < n) {
                nw1 = units_at(group1, pr1);
                if (!load_stage(j + 1, nw1, q1, sw1)) {
                    ok = false;
                    break;
                }
            }
            // A buffer b was last read by the MMAs of hand-off j - kVBufs
            const int b = ab;
            if (j >= kVBufs && !vwait(bars + 8 * (kBarFree + b), apar ^ 1u, abort)) {
                ok = false;
                break;
            }
            if (++ab == kVBufs) {
                ab = 0;
                apar ^= 1u;
            }
            tc_fence_after();
            if (nw > 0) {
                // A: this warp's 32 rows of its tile for its chunks, bf16, into tensor memory
                // (lanes = rows, two values per column).  Word s of row group r of unit h
                // holds rows 16r+g (a[s][0], a[s][2]) and 16r+g+8 (a[s][1], a[s][3]) at
                // columns 16t+4s+{0,1} and {2,3} of chunk h: MMA step 4h + s, k = 4t +
                // {0,1} and {2,3}, i.e. the step's columns 2t and 2t + 1.
                const uint32_t acol = tmem + (uint32_t)(kATmemCol + (b * kVTiles + tt) * kATmemTileCols);
#pragma unroll
                for (int h = 0; h < kVUPW; ++h) {
                    if (h < nw) {
                        uint32_t S[2][2];
                        scale_pairs(sw[h], S);
#pragma unroll
                        for (int r = 0; r < 2; ++r) {
                            uint32_t a[4][4];
#pragma unroll
                            for (int s = 0; s < 4; ++s) dequant_word(q[h][4 * r + s], S, r, a[s]);
                            const uint32_t v[16] = {a[0][0], a[0][2], a[0][1], a[0][3], a[1][0], a[1][2],
                                                    a[1][1], a[1][3], a[2][0], a[2][2], a[2][1], a[2][3],
                                                    a[3][0], a[3][2], a[3][1], a[3][3]};
                            tc_st_16x256b_x4(acol + (uint32_t)(32 * (h0 + h)) + ((uint32_t)(trow + 16 * r) << 16), v);
                        }
                    }
                }
            }
            // the A stores are complete before the MMA threads are told
            asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
            tc_fence_before();
            // Slot j is refilled only now: every word read from it has been dequantised
            // and stored, so the copy cannot overtake the reads.
            __syncwarp();
            if (lane == 0) {
                if (j + kVStages < n) issue(j + kVStages);
                mbar_arrive(bars + 8 * (kBarFull + b));
            }
            if (j + kVStages < n) issued = j + kVStages + 1;

            if (pr == KP - 1 || j == n - 1) {
                // end of this group's K range in this CTA: read the accumulators back
                if (!vwait(bars + 8 * kBarAcc, (uint32_t)(seg & 1), abort)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const long long ps = group * KP;  // the group's first unit
                const bool whole = ps >= u0 && ps + KP <= u1;
                const long long row_g = t32 * 32 + lane;  // output row of this thread
                const uint32_t taddr = tmem + ((uint32_t)trow << 16) + (uint32_t)(tt * p.NL);
                const int pslot = ps <= u0 ? 0 : 1;  // this CTA's first or last segment
                // a partial: this row's nl sums, contiguous ([256 rows][64] per slot)
                float* pdst = p.part + (cta * 2 + pslot) * (long long)kVSlotFloats + (slice * 32 + lane) * kVMaxNL;
                // the slice's warps share the columns: blocks of 16, dealt round robin
                for (int m0 = 16 * (w / kVSlices); m0 < p.NL; m0 += 16 * kVSplit) {
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
                // The next group's first MMA overwrites the accumulators only after every
                // warp's next arrival on a full barrier, which follows these loads.
                tc_fence_before();
                ++seg;
                if (!whole) {
                    // Partials go to another CTA: each lane makes its own stores visible at GPU
                    // scope before its warp signals (one thread's release does not cover the
                    // other warps' stores still in flight).
                    __threadfence();
                    __syncwarp();
                    // count the CTA in on the group; its last contributor adds every partial
                    const long long glo = vrange_owner(U, T, ps), ghi = vrange_owner(U, T, ps + KP - 1);
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
                        ok = false;
                        break;
                    }
                    const int last = misc[2];
                    ++split;
                    if (last) {
                        // every contributor's partial of this row, in CTA order, 16 sums at a
                        // time, four contributors' loads in flight at once
                        const int glo_slot = vrange_begin(U, T, glo) >= ps ? 0 : 1;
                        const float* rowp = p.part + (slice * 32 + lane) * kVMaxNL;
                        for (int m0 = 16 * (w / kVSlices); m0 < p.NL; m0 += 16 * kVSplit) {
                            float sum[16];
#pragma unroll
                            for (int i = 0; i < 16; ++i) sum[i] = 0.f;
                            for (long long c0 = glo; c0 <= ghi; c0 += kFinBatch) {
                                float4 v4[kFinBatch][4];
#pragma unroll
                                for (int cc = 0; cc < kFinBatch; ++cc) {
                                    const long long ci = c0 + cc;
                                    if (ci <= ghi) {
                                        const int sl = ci == glo ? glo_slot : 0;
                                        const float4* src = reinterpret_cast<const float4*>(
                                            rowp + (ci * 2 + sl) * (long long)kVSlotFloats + m0);
#pragma unroll
                                        for (int i = 0; i < 4; ++i) v4[cc][i] = __ldcg(src + i);
                                    }
                                }
#pragma unroll
                                for (int cc = 0; cc < kFinBatch; ++cc) {
                                    if (c0 + cc <= ghi) {
#pragma unroll
                                        for (int i = 0; i < 4; ++i) {
                                            sum[4 * i] += v4[cc][i].x;
                                            sum[4 * i + 1] += v4[cc][i].y;
                                            sum[4 * i + 2] += v4[cc][i].z;
                                            sum[4 * i + 3] += v4[cc][i].w;
                                        }
                                    }
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
            group = group1;
            pr = pr1;
            nw = nw1;
#pragma unroll
            for (int h = 0; h < kVUPW; ++h) {
                sw[h] = sw1[h];
#pragma unroll
                for (int i = 0; i < 8; ++i) q[h][i] = q1[h][i];
            }
        }
        if (!ok) {
            if (lane == 0 && !*abort) vabort(abort, 1u);
            // wait (bounded) for this warp's copies still in flight
            for (int s = waited; s < issued; ++s)
                if (stage_units(u0 + s) > 0) warp_wait(rbar + 8 * (s % kVStages), (uint32_t)((s / kVStages) & 1));
        }
    } else if (warp < kVXWarp) {
        // The MMAs of tile tt = warp - kVMmaWarp, issued by one thread: two issuers on
        // two sub-partitions halve the issue work that competes with the dequantisation
        // warps there.  Each tile has its own accumulator, so the two streams of MMAs
        // need no order between them.
        if (lane == 0) {
            const int tt = warp - kVMmaWarp;
            const uint32_t d = tmem + (uint32_t)(tt * p.NL);
            const uint32_t xoff = (uint32_t)(p.NL * 128) >> 4;  // second chunk of a buffer, in 16-byte steps
            bool any = false;
            int pr = pr0;
            for (int j = 0; j < n; ++j) {
                const int b = j % kVBufs;
                const int nch = 2 * pr + 1 < KC ? 2 : 1;
                const bool first = j == 0 || pr == 0;
                if (!vwait1(bars + 8 * (kBarFull + b), (uint32_t)((j / kVBufs) & 1), abort)) {
                    if (!*abort) vabort(abort, 2u);
                    break;
                }
                tc_fence_after();
                // X chunk h of buffer b, MMA step s at 256 s bytes (16 s in the
                // descriptor's address field); A of this tile at column 32 h + 8 s
                const uint64_t xd = kmajor_desc(base + kOffX + b * kXBufBytes);
                const uint32_t a0 = tmem + (uint32_t)(kATmemCol + (b * kVTiles + tt) * kATmemTileCols);
                tc_mma_ts(d, a0, xd, p.idesc, first ? 0u : 1u);
#pragma unroll
                for (int kk = 1; kk < 4; ++kk) tc_mma_ts(d, a0 + (uint32_t)(8 * kk), xd + (uint64_t)(16 * kk), p.idesc, 1u);
                if (nch == 2) {
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk)
                        tc_mma_ts(d, a0 + (uint32_t)(32 + 8 * kk), xd + (uint64_t)(xoff + 16 * kk), p.idesc, 1u);
                }
                any = true;
                tc_commit(bars + 8 * (kBarFree + b));
                if (pr == KP - 1 || j == n - 1) tc_commit(bars + 8 * kBarAcc);
                if (++pr == KP) pr = 0;
            }
            // every MMA finished before the tensor memory is released
            if (any) {
                tc_commit(bars + 8 * kBarFin);
                for (uint32_t it = 0; it < kWaitLimit && !mbar_try_wait(bars + 8 * kBarFin, 0u); ++it) {
                }
            }
        }
        __syncwarp();
    } else if (warp == kVXWarp) {
        if (lane == 0) {
            // Xp is written by the preceding kernel
            asm volatile("griddepcontrol.wait;" ::: "memory");
            const uint64_t pol = evict_last_policy();
            int pr = pr0, issued = 0;
            for (int j = 0; j < n; ++j) {
                const int b = j % kVBufs;
                // buffer b was last read by the MMAs of hand-off j - kVBufs
                if (j >= kVBufs && !vwait1(bars + 8 * (kBarFree + b), (uint32_t)(((j / kVBufs) - 1) & 1), abort)) {
                    if (!*abort) vabort(abort, 2u);
                    break;
                }
                const int nch = 2 * pr + 1 < KC ? 2 : 1;
                const uint32_t bytes = (uint32_t)(nch * p.NL * 128);
                const uint32_t bar = bars + 8 * (kBarFull + b);
                mbar_expect_tx(bar, bytes);  // also this thread's arrival on full[b]
                bulk_load(base + kOffX + b * kXBufBytes, p.Xp + (long long)(2 * pr) * p.NL * 128, bytes, bar, pol);
                issued = j + 1;
                if (++pr == KP) pr = 0;
            }
            // After an abort the last copies may still be in flight: wait (bounded) for
            // their phases, which complete once they land unless a warp's arrival is
            // missing too, in which case the wait runs out well after they landed.
            if (*abort)
                for (int j = issued > kVBufs ? issued - kVBufs : 0; j < issued; ++j)
                    for (uint32_t it = 0; it < kWaitLimit; ++it)
                        if (mbar_try_wait(bars + 8 * (kBarFull + j % kVBufs), (uint32_t)((j / kVBufs) & 1))) break;
        }
        __syncwarp();
    }
    tc_fence_before();
    __syncthreads();
    if (warp == kVMmaWarp) {
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
    uint8_t* xp = nullptr;  // X in the MMA's order, rewritten by every call
    size_t xp_bytes = 0;
};
std::mutex g_vmu;
VerifyState g_vstate[64];

constexpr size_t kXpInitialBytes = (size_t)kVMaxNL * 128 * 1024;  // K up to 65,536 at nl = 64: 8 MB

int verify_state(cudaStream_t stream, size_t xp_need, VerifyState** out)
{
    int dev = 0;
    NVFP4_CUDA_TRY(cudaGetDevice(&dev));
    if (dev < 0 || dev >= 64) return NVFP4_ERR_ARG;
    std::lock_guard<std::mutex> lock(g_vmu);
    VerifyState& s = g_vstate[dev];
    if (s.device == dev && s.xp_bytes >= xp_need) {
        *out = &s;
        return NVFP4_OK;
    }
    cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
    NVFP4_CUDA_TRY(cudaStreamIsCapturing(stream, &cs));
    if (cs != cudaStreamCaptureStatusNone) return NVFP4_ERR_CAPTURE;
    if (s.device == dev) {
        // a longer K than before: a larger X buffer, once nothing uses the old one
        NVFP4_CUDA_TRY(cudaDeviceSynchronize());
        NVFP4_CUDA_TRY(cudaFree(s.xp));
        s.xp = nullptr;
        s.xp_bytes = 0;
        NVFP4_CUDA_TRY(cudaMalloc(&s.xp, xp_need));
        s.xp_bytes = xp_need;
        *out = &s;
        return NVFP4_OK;
    }
    int sms = 0;
    NVFP4_CUDA_TRY(cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev));
    const int max_ctas = kVCtasPerSM * sms;
    const size_t xp_bytes = xp_need > kXpInitialBytes ? xp_need : kXpInitialBytes;
    float* part = nullptr;
    unsigned* counters = nullptr;
    uint8_t* xp = nullptr;
    NVFP4_CUDA_TRY(cudaMalloc(&part, (size_t)max_ctas * 2 * kVSlotFloats * sizeof(float)));
    cudaError_t e = cudaMalloc(&counters, (size_t)kVMaxGroups * sizeof(unsigned));
    if (e == cudaSuccess) e = cudaMalloc(&xp, xp_bytes);
    if (e == cudaSuccess) e = cudaMemset(counters, 0, (size_t)kVMaxGroups * sizeof(unsigned));
    if (e == cudaSuccess)
        e = cudaFuncSetAttribute(verify_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kVSmemBytes);
    if (e == cudaSuccess) e = cudaDeviceSynchronize();
    if (e != cudaSuccess) {
        cudaFree(part);
        if (counters) cudaFree(counters);
        if (xp) cudaFree(xp);
        return fail_cuda(e);
    }
    s.sm_count = sms;
    s.max_ctas = max_ctas;
    s.part = part;
    s.counters = counters;
    s.xp = xp;
    s.xp_bytes = xp_bytes;
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
    g->n_groups = (g->n_tiles32 + kVSlices - 1) / kVSlices;  // groups of kVSlices 32-row tiles
    if (g->n_groups > kVMaxGroups) return NVFP4_ERR_SHAPE;
    g->k_chunks = (K + kChunkK - 1) / kChunkK;
    g->k_pairs = (g->k_chunks + kVPair - 1) / kVPair;
    g->units = g->n_groups * g->k_pairs;
    // one CTA per SM, but no more than kVMaxSplit CTAs per group on average: a group
    // split between more CTAs costs more in partial sums than the extra SMs stream
    long long ctas = (long long)kVCtasPerSM * sm_count;
    if (ctas > g->n_groups * kVMaxSplit) ctas = g->n_groups * kVMaxSplit;
    if (ctas > g->units) ctas = g->units;
    g->ctas = ctas;
    g->nl = (M + 15) / 16 * 16;
    g->tmem_cols = kVTmemCols;  // accumulators (2 x nl <= 128 columns) and the triple-buffered A operand
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
    const long long pieces = (K + kChunkK - 1) / kChunkK * ((M + 15) / 16 * 16) * 8;  // 16-byte pieces of X
    VerifyState* vs = nullptr;
    st = verify_state(stream, (size_t)pieces * 16, &vs);
    if (st != NVFP4_OK) return st;
    VerifyGeometry geo;
    st = verify_geometry(M, N, K, vs->sm_count, &geo);
    if (st != NVFP4_OK) return st;
    VParams p;
    p.wq = wq;
    p.ws = ws;
    p.Xp = vs->xp;
    p.Y = Y;
    p.part = vs->part;
    p.counters = vs->counters;
    p.gscale = gscale;
    p.M = M;
    p.NL = geo.nl;
    p.tmem_cols = geo.tmem_cols;
    p.N = N;
    p.KC = (int)geo.k_chunks;
    p.KP = (int)geo.k_pairs;
    p.n_tiles32 = (int)geo.n_tiles32;
    p.n_groups = (int)geo.n_groups;
    p.units = geo.units;
    p.ctas = geo.ctas;
    // kind::f16 instruction: F32 accumulator, BF16 A and B, both K-major, N = nl, M = 128
    p.idesc = (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(geo.nl >> 3) << 17) | ((uint32_t)(kVTileRows >> 4) << 24);
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)((pieces + 255) / 256));
    cfg.blockDim = dim3(256);
    cfg.dynamicSmemBytes = 0;
    cfg.stream = stream;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    NVFP4_CUDA_TRY(cudaLaunchKernelEx(&cfg, verify_xprep_kernel, static_cast<const uint16_t*>(X), vs->xp, M,
                                      geo.nl, (long long)K, pieces));
    cfg.gridDim = dim3((unsigned)geo.ctas);
    cfg.blockDim = dim3(kVThreads);
    cfg.dynamicSmemBytes = kVSmemBytes;
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
