/*
 * nvfp4decode.h -- C ABI of libnvfp4decode.so, the NVFP4 weight-streaming
 * decode round for NVIDIA B200 (sm_100a).
 *
 * The operation (ignis README, section "The decode round"; "Why ignis", tile
 * "One round for every lane"): up to eight decode lanes share one pass over
 * the weights,
 *
 *     Y[M][N] = X[M][K] . dequant(W)^T,        M = 1..8,
 *     dequant(W)[n][k] = gscale * e2m1(q[n][k]) * e4m3(s[n][k/16]),
 *
 * with W stored as NVFP4: 4-bit E2M1 elements and one E4M3 scale per 16
 * consecutive K values ("Models and artifacts", section "The artifact"),
 * plus one FP32 global scale.  X is BF16, accumulation is FP32.  The whole
 * round is replayed from one CUDA graph per batch width (README, "The decode
 * round"); the step-level boundary is flat and device-resident (README,
 * introduction: "flat, device-resident step-level C ABI").
 *
 * Conventions shared by every call:
 *  - Pointers are DEVICE pointers unless a parameter says "host".  The caller
 *    owns every buffer; the library never frees caller memory.
 *  - Device pointers must be 16-byte aligned (else NVFP4_ERR_ALIGN).
 *  - M in 1..8 (else NVFP4_ERR_M), except nvfp4_gemm_decode, which also
 *    takes verify widths 9..64; N >= 1; K >= 16 and K % 16 == 0 (else
 *    NVFP4_ERR_SHAPE).
 *  - X, Y and H are dense row-major with leading dimension K, N and N.
 *  - Calls never throw, abort or trap.  Asynchronous calls return once the
 *    work is enqueued on `stream`; a device fault surfaces at the caller's
 *    next synchronisation, or as NVFP4_ERR_CUDA here with the CUDA error code
 *    kept for nvfp4_last_cuda_error().
 *  - `stream` may be NULL (the legacy default stream).
 */
#ifndef NVFP4DECODE_H
#define NVFP4DECODE_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define NVFP4_API __attribute__((visibility("default")))
#else
#define NVFP4_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st* nvfp4_stream_t; /* the same handle as cudaStream_t */
typedef struct nvfp4_round nvfp4_round;     /* opaque graph-replay handle */

enum {
    NVFP4_OK = 0,
    NVFP4_ERR_ARG = -1,       /* NULL pointer, bad kind, bad count */
    NVFP4_ERR_M = -2,         /* M outside 1..8 (1..64 for nvfp4_gemm_decode) */
    NVFP4_ERR_SHAPE = -3,     /* N < 1, K < 16 or K % 16 != 0, size overflow */
    NVFP4_ERR_ALIGN = -4,     /* a device pointer is not 16-byte aligned */
    NVFP4_ERR_BAD_SCALE = -5, /* a scale byte is an E4M3 NaN code (0x7F / 0xFF) */
    NVFP4_ERR_CUDA = -6,      /* a CUDA runtime call failed; see nvfp4_last_cuda_error() */
    NVFP4_ERR_CAPTURE = -7,   /* first use of a device while its stream is being captured */
    NVFP4_ERR_DEVICE = -8,    /* a kernel's bounded wait gave up; see nvfp4_device_status() */
    NVFP4_ERR_SCRATCH = -9    /* the call needs more scratch than nvfp4_gemm_decode_noalloc's array holds */
};

/*
 * Sizes of the device-layout planes of an N x K NVFP4 matrix.
 *
 * The device layout ("Models and artifacts", "The artifact": the kernels read
 * the weight planes directly) keeps the canonical byte counts per element --
 * half a byte per weight and one scale byte per 16 -- but permutes them into
 * 32-row x 64-column units (1024 nibble bytes + 128 scale bytes each) so that
 * every warp streams one contiguous run of bytes.  N is padded to a multiple
 * of 32 and K to a multiple of 64 with zero codes and zero scales.
 * Writes *wq_bytes and *ws_bytes (host pointers).  Pure host call.
 */
NVFP4_API int nvfp4_packed_bytes(int64_t N, int64_t K, size_t* wq_bytes, size_t* ws_bytes);

/*
 * Load-time pack: canonical planes -> device layout, plus a scan for NaN
 * scale codes.  Canonical planes ("Models and artifacts", "The artifact"):
 *   wq_canon  u8[N][K/2]: element k of row n in byte k/2, the even element
 *             in the low nibble and the odd element in the high nibble;
 *   ws_canon  u8[N][K/16]: E4M3 scale of k in [16b, 16b+15] of row n.
 * wq_dev / ws_dev receive nvfp4_packed_bytes() bytes each.  The call
 * synchronises `stream` and returns NVFP4_ERR_BAD_SCALE if any scale byte is
 * 0x7F or 0xFF (the planes are still written).  Not reentrant across host
 * threads on one device (serialised internally).
 */
NVFP4_API int nvfp4_pack_check(const uint8_t* wq_canon, const uint8_t* ws_canon, int64_t N, int64_t K,
                     uint8_t* wq_dev, uint8_t* ws_dev, nvfp4_stream_t stream);

/*
 * The decode GEMM, asynchronous:  Y[m][n] = gscale * sum_k X[m][k] w[n][k].
 *   X   bf16 [M][K];  Y float [M][N];  wq_dev / ws_dev from nvfp4_pack_check.
 * The weights are read once per call for all M lanes (README, "The decode
 * round").  Split-K partial sums are combined in a fixed order, so results
 * are bit-identical from call to call.  Uses a per-device workspace that the
 * first call on a device allocates; that first call must not be made while
 * `stream` is being captured (NVFP4_ERR_CAPTURE).  Calls on one device that
 * overlap in time share that workspace and must not run concurrently.
 *
 * M: 1..8 decode lanes, or 9..64 rows at verify widths (README, "What sets
 * it apart", "Speculative decoding (DFlash2)": lanes x (1 + drafts) rows
 * verified in the same pass).  Widths 9..32 run on the decode kernel with
 * two to four blocks of 8 lanes sharing each dequantised word; widths 33..64
 * run on the tensor-memory kernel (its own per-device workspace, allocated by
 * its first call under the same capture rule, and a buffer for X in the
 * MMA's order sized for K up to 65,536 at first; a call with a longer K than
 * any before grows it, synchronising the device, under the same rule;
 * nvfp4_verify_geometry describes its work split).  Those widths launch two
 * kernels: X's reordering, then the GEMM.  Other M: NVFP4_ERR_M.
 */
NVFP4_API int nvfp4_gemm_decode(const void* X, int M, const uint8_t* wq_dev, const uint8_t* ws_dev,
                      float gscale, float* Y, int64_t N, int64_t K, nvfp4_stream_t stream);

/*
 * The decode GEMM of nvfp4_gemm_decode, for callers that must not allocate
 * device memory.  (No counterpart in the pages; it exists for callers.)
 *
 * nvfp4_gemm_decode allocates its split-K workspace with cudaMalloc on the
 * first call on each device.  Some callers cannot allow that: an engine that
 * reserves its whole device-memory plan at load time and forbids any later
 * allocation, a plugin whose host application owns all device memory, or a
 * latency-critical path that cannot take cudaMalloc's implicit device
 * synchronisation.  This entry point calls no cudaMalloc, cudaFree or other
 * allocating routine: its scratch (the split-K partial sums and arrival
 * counters) is a file-scope static device array of this library, 10 MiB of
 * partial sums plus 10 KiB of counters, enough for 2,560 warps; every GPU
 * that loads the library holds it until the process exits.
 *
 * Arguments, layout and result are those of nvfp4_gemm_decode at M = 1..8
 * (the same kernel runs); verify widths are not taken here (NVFP4_ERR_M).
 * The first call on a device resolves the array's device address
 * (cudaGetSymbolAddress) with that device current, so make that first call
 * before any stream capture (a first call made while `stream` is captured
 * returns NVFP4_ERR_CAPTURE).  Each call clears the arrival counters on
 * `stream` before the kernel.  All calls share the one array, which keeps the
 * previous call's contents: calls that overlap on the GPU (other streams,
 * other host threads) race on it and must be serialised by the caller.
 * A launch that would use more warps than the array holds (a device with more
 * than 160 SMs) runs with 2,560 warps instead; the result is the same GEMM
 * within the bound, though not bit-identical to nvfp4_gemm_decode on such a
 * device, whose work split differs.
 */
NVFP4_API int nvfp4_gemm_decode_noalloc(const void* X, int M, const uint8_t* wq_dev, const uint8_t* ws_dev,
                                        float gscale, float* Y, int64_t N, int64_t K, nvfp4_stream_t stream);

/*
 * Fused MLP front half, asynchronous, one launch for both projections:
 *   g = gscale_gate * X . Wg^T,  u = gscale_up * X . Wu^T,
 *   H[m][n] = bf16( silu(g) * u ),  silu(g) = g / (1 + exp(-g)).
 * X bf16 [M][K]; H bf16 [M][Nff]; the gate and up matrices are separate
 * Nff x K matrices in device layout.  Same workspace rules as
 * nvfp4_gemm_decode.  The pages describe no such fused projection: the 27B
 * body has an MLP in every layer ("Models and artifacts", model table), and
 * fusing its gate and up projections with the SiLU-multiply into one pass over
 * both weight matrices is this library's design.
 */
NVFP4_API int nvfp4_gemm_gateup_silu(const void* X, int M,
                           const uint8_t* wq_gate, const uint8_t* ws_gate, float gscale_gate,
                           const uint8_t* wq_up, const uint8_t* ws_up, float gscale_up,
                           void* H, int64_t Nff, int64_t K, nvfp4_stream_t stream);

/* One node of a decode round. */
enum { NVFP4_DESC_GEMM = 0, NVFP4_DESC_GATEUP_SILU = 1 };
typedef struct {
    int kind;              /* NVFP4_DESC_GEMM or NVFP4_DESC_GATEUP_SILU */
    const void* X;         /* bf16 [M][K], rows for M = 8 must be allocated */
    const uint8_t* wq;     /* device-layout planes (gate for GATEUP_SILU) */
    const uint8_t* ws;
    float gscale;
    const uint8_t* wq2;    /* up projection planes (GATEUP_SILU only, else NULL) */
    const uint8_t* ws2;
    float gscale2;
    void* out;             /* float [M][N] (GEMM) or bf16 [M][N] (GATEUP_SILU) */
    int64_t N, K;
} nvfp4_gemm_desc;

/*
 * Build a decode round: the n descriptors are launched in order, each as a
 * programmatic-dependent launch of the previous one (a PDL chain: every node
 * prefetches its weights before waiting on its predecessor), and captured
 * once per batch width M = 1..8 into eight CUDA graphs (README, "The decode
 * round": per-width CUDA graphs, widths 1..8).  The descriptor array is
 * copied; the buffers it names must outlive the round.  Allocates the graphs
 * and the per-device workspace.  Synchronous; *out is a host pointer.
 */
NVFP4_API int nvfp4_round_create(const nvfp4_gemm_desc* descs, int n, nvfp4_round** out);

/*
 * nvfp4_round_create with a choice of how the round runs:
 *   NVFP4_ROUND_CHAIN (what nvfp4_round_create uses): each width's graph holds
 *     one kernel per node, linked by programmatic dependent launch (the chain
 *     described above).  Results are bit-identical to direct calls.
 *   NVFP4_ROUND_PERSISTENT: each width's graph holds one cooperative kernel
 *     that runs every node in order on all SMs.  Each warp's weight stream
 *     runs on from one node into the next, and a node's X is read only after
 *     every CTA has finished the node before it (a counter per node, bounded
 *     waits).  A fused gate/up node runs as one GEMM over both matrices
 *     stacked into an FP32 buffer the round owns, then an elementwise
 *     SiLU-multiply node; plain GEMM nodes keep the work split of a direct
 *     call (bit-identical), fused ones agree with it within the GEMM bound.
 *     At most 360 nodes per launch; longer rounds take several launches.
 */
enum { NVFP4_ROUND_PERSISTENT = 0, NVFP4_ROUND_CHAIN = 1 };
NVFP4_API int nvfp4_round_create_ex(const nvfp4_gemm_desc* descs, int n, int mode, nvfp4_round** out);

/* Number of kernel nodes in each of the round's graphs (host call). */
NVFP4_API int nvfp4_round_nodes(const nvfp4_round* r, int* nodes);

/*
 * Replay the width-M graph on `stream` (one graph launch, asynchronous).
 * The graph reads whatever the descriptor buffers hold when it runs.
 * A round handle is not thread-safe.
 */
NVFP4_API int nvfp4_round_replay(nvfp4_round* r, int M, nvfp4_stream_t stream);

/*
 * The same replay with host buffers at both ends, all on `stream`:
 * copy x_bytes from x_host (host) to x_dev, replay the width-M graph, copy
 * y_bytes from y_dev to y_host (host).  Asynchronous; pinned host memory
 * makes the copies asynchronous too.
 */
NVFP4_API int nvfp4_round_replay_host(nvfp4_round* r, int M, const void* x_host, void* x_dev,
                            size_t x_bytes, const void* y_dev, void* y_host, size_t y_bytes,
                            nvfp4_stream_t stream);

/* Release the graphs of a round (synchronises nothing; NULL is accepted). */
NVFP4_API int nvfp4_round_destroy(nvfp4_round* r);

/*
 * Top-k over rows of FP32 logits: the step after the output head (ignis
 * README, "What sets it apart", "Speculative decoding (DFlash2)": the
 * drafter's top-k over the vocabulary, replaced by a row-split kernel with
 * a bit-identical answer).
 *
 * For each row m < rows, the k largest of logits[m*ldv + 0 .. m*ldv + V),
 * best first, into values[m*k + j] and indices[m*k + j] (j < k).  Ranking:
 * IEEE 754 totalOrder, except that -0 and +0 are equal, and equal values
 * rank by lower index.  So numbers (and infinities) rank by value; a NaN
 * with sign 0 ranks above +inf and one with sign 1 below -inf.  The answer
 * is unique, and values are the input's own bits.
 *
 * Arguments: device pointers; logits 16-byte aligned with ldv % 4 == 0 and
 * ldv >= V; values float[rows][k], indices int32[rows][k], 4-byte aligned.
 * Limits: 1 <= rows <= NVFP4_TOPK_MAX_ROWS, 1 <= k <= NVFP4_TOPK_MAX_K,
 * k <= V <= NVFP4_TOPK_MAX_V, and the row split must fit (S*k <= 16384,
 * see nvfp4_topk_splits), else NVFP4_ERR_SHAPE.  Bad rows: NVFP4_ERR_M.
 * Alignment: NVFP4_ERR_ALIGN.  NULL: NVFP4_ERR_ARG.
 *
 * One asynchronous launch on `stream`.  The library owns a per-device
 * candidate workspace, allocated by the first call on a device (which must
 * not be inside a stream capture: NVFP4_ERR_CAPTURE); later calls, captured
 * or not, allocate nothing.  Calls on one device share that workspace and
 * must be ordered (one stream, or synchronised).
 */
#define NVFP4_TOPK_MAX_ROWS 64
#define NVFP4_TOPK_MAX_K 64
#define NVFP4_TOPK_MAX_V (1 << 24)
NVFP4_API int nvfp4_topk(const float* logits, int rows, int64_t V, int64_t ldv, int k, float* values,
                         int32_t* indices, nvfp4_stream_t stream);

/*
 * Host helper (no GPU needed): the row split nvfp4_topk uses on a device
 * with `sm_count` SMs -- `splits` slices per row of `slice` elements (a
 * multiple of 4; the last slice may be shorter).  Returns the status the
 * call itself would return for these sizes.
 */
NVFP4_API int nvfp4_topk_splits(int rows, int64_t V, int k, int sm_count, int* splits, int* slice);

/*
 * Test aid: the dequantised weights exactly as the GEMM kernels form them,
 * W[n][k] = fp32(e2m1 * e4m3 * gscale), float [N][K] (unpadded).  Asynchronous.
 */
NVFP4_API int nvfp4_dequant_debug(const uint8_t* wq_dev, const uint8_t* ws_dev, float gscale, float* W,
                        int64_t N, int64_t K, nvfp4_stream_t stream);

/*
 * Test aid: device layout -> canonical planes (the inverse of the pack).
 * wq_canon u8[N][K/2], ws_canon u8[N][K/16].  Asynchronous.
 */
NVFP4_API int nvfp4_unpack_debug(const uint8_t* wq_dev, const uint8_t* ws_dev, int64_t N, int64_t K,
                       uint8_t* wq_canon, uint8_t* ws_canon, nvfp4_stream_t stream);

/*
 * Host-side model of the device layout, for CPU tests (no GPU needed):
 * dequantise one packed 32 x 64 unit with the same bit placement and the
 * same bf16 arithmetic the kernels use.  q_unit: 1024 host bytes, s_unit:
 * 128 host bytes; W: float [32][64] host output (gscale applied).
 */
NVFP4_API int nvfp4_host_dequant_unit(const uint8_t* q_unit, const uint8_t* s_unit, float gscale,
                            float* W);

/* Host-side pack of one unit: canonical host planes -> one 1024 + 128 byte unit. */
NVFP4_API int nvfp4_host_pack_unit(const uint8_t* wq_canon, const uint8_t* ws_canon, int64_t N, int64_t K,
                         int64_t tile, int64_t chunk, uint8_t* q_unit, uint8_t* s_unit);

/*
 * Grouped expert decode, one asynchronous launch (ignis, "Models and
 * artifacts", the model table: Flash-Next has 512 routed experts per layer
 * and ten chosen per token).  For every route (m, t), m < M lanes, t < T picks:
 *   Y[(m*T + t)*N + n] = gscale_e * sum_k x[k] * w_e[n][k],  e = route[m*T + t],
 *   x = X + m*K (x_per_route == 0: one input per lane, as for gate / up)
 *     or X + (m*T + t)*K (x_per_route != 0: one input per route, as for down).
 * experts[e] holds expert e's device-layout planes (nvfp4_pack_check) and
 * global scale; every expert matrix is N x K.  An expert picked by several
 * lanes is streamed once for all of them.  X bf16, Y float, route int32 and
 * experts are device memory; route and experts may change between calls (and
 * between graph replays).  Routes with a negative id give zero rows; ids >= E
 * or experts whose planes are not 16-byte aligned also give zero rows and set
 * bit 32 of nvfp4_device_status().  Results are deterministic.
 * Limits: 1 <= M <= 8 (NVFP4_ERR_M), T >= 1 and M*T <= NVFP4_GROUPED_MAX_ROUTES
 * (NVFP4_ERR_ARG), N <= 131,072 (NVFP4_ERR_SHAPE).  X 16-byte aligned, route
 * and Y 4-byte, experts 8-byte (NVFP4_ERR_ALIGN).  Per-device workspace as for
 * nvfp4_gemm_decode (first call outside any capture).
 */
typedef struct {
    const uint8_t* wq; /* device-layout nibble plane */
    const uint8_t* ws; /* device-layout scale plane */
    float gscale;
    int32_t reserved;
} nvfp4_expert;
#define NVFP4_GROUPED_MAX_ROUTES 128
NVFP4_API int nvfp4_gemm_grouped(const void* X, int x_per_route, const int32_t* route, int M, int T,
                                 const nvfp4_expert* experts, int E, float* Y, int64_t N, int64_t K,
                                 nvfp4_stream_t stream);

/*
 * Host helper (no GPU needed): the work split nvfp4_gemm_decode uses at a
 * verify width M (9..64) on a device with `sm_count` SMs -- `ctas` CTAs,
 * each owning a contiguous range of the `units` (256-row group, pair of
 * 64-column chunks) units -- and `nl`, the MMA's N (M padded to a multiple
 * of 16).
 * Returns NVFP4_ERR_M / NVFP4_ERR_SHAPE exactly when the call would.
 */
NVFP4_API int nvfp4_verify_geometry(int M, int64_t N, int64_t K, int sm_count, int64_t* ctas, int64_t* units,
                                    int* nl);

/*
 * Measurement aid: read `bytes` of device memory once, as the decode round's
 * weight stream does (README, "The decode round": the round is weight
 * streaming at the card's bandwidth), to measure the read-only HBM bandwidth
 * that the round's GB/s is compared with beside the copy figure.
 *
 * buf: device, 16-byte aligned, `bytes` a positive multiple of 16; it is only
 * read.  out: device u32[ctas], 4-byte aligned; CTA c writes out[c], the XOR
 * of the 32-bit words it read, so the XOR over all of `out` equals the XOR of
 * every 32-bit word of `buf`.  ctas: grid size, 1..2^20 (four per SM keeps
 * enough loads in flight for the full bandwidth).  One asynchronous launch.
 * Returns NVFP4_ERR_ARG (NULL pointer, ctas out of range), NVFP4_ERR_SHAPE,
 * NVFP4_ERR_ALIGN or NVFP4_ERR_CUDA (launch failed).
 */
NVFP4_API int nvfp4_stream_read(const void* buf, size_t bytes, uint32_t* out, int ctas, nvfp4_stream_t stream);

/* Text for a status code (static storage). */
NVFP4_API const char* nvfp4_status_string(int status);

/* CUDA error code of the last NVFP4_ERR_CUDA on this host thread (0 if none). */
NVFP4_API int nvfp4_last_cuda_error(void);

/*
 * Device-side status of the current device: 0 when every kernel finished its
 * bounded waits, else an OR of these flags:
 *    1  decode GEMM: a warp's bulk-copy ring wait gave up
 *    2  persistent round: the grid barrier between nodes gave up
 *    4  decode GEMM: a split-K combine wait gave up -- a gather copy (sums
 *       then read from global memory) or a finisher's wait on a partial
 *       (that tile's Y is wrong)
 *    8  verify widths (33..64): a dequantisation warp's wait gave up
 *   16  verify widths (33..64): the MMA or X-staging thread's wait gave up
 *   32  grouped experts: a route named an expert outside 0..E-1 or with
 *       misaligned planes (its rows are zero)
 *   64  grouped experts: a bounded wait gave up
 * Reading it synchronises the device; a nonzero status also clears the flags
 * and re-zeroes the split-K counters.
 */
NVFP4_API int nvfp4_device_status(void);

/* Library version, e.g. 100 for 1.0. */
NVFP4_API int nvfp4_version(void);

#ifdef __cplusplus
}
#endif

#endif /* NVFP4DECODE_H */
