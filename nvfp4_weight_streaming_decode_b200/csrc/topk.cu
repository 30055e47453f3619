// topk.cu -- top-k over rows of FP32 logits, the step after the output head.
//
// ignis README, "What sets it apart", "Speculative decoding (DFlash2)": the
// drafter's top-k over the vocabulary, replaced by a row-split kernel that
// gives a bit-identical answer.  Here: for each row, the k largest logits
// (values and indices, best first) under IEEE totalOrder with -0 == +0 and
// equal values ranked by lower index.  That order is strict on (value,
// index), so the answer is unique and does not depend on scheduling.
//
// One launch, row-split: blockIdx.y is the row, blockIdx.x one of S slices of
// it.  Each CTA
//   1. loads its slice as 32-bit order keys into shared memory,
//   2. finds the k-th largest key by radix select (four 8-bit digit passes,
//      histograms in shared memory with warp-aggregated atomics),
//   3. if more elements tie at that key than are needed, finds the needed
//      ones by a second radix select on the index (smallest first),
//   4. sorts the k winners (bitonic, one warp) and publishes them,
// and the last CTA of a row to finish (counter, acquire/release) merges the
// S*k candidates with the same routine and writes the row's answer.  No CTA
// ever waits for another.
#include <cuda_runtime.h>
#include <stdint.h>

#include <mutex>

#include "internal.h"

namespace nvfp4 {

namespace {

constexpr int kTopkThreads = 256;
constexpr int kSliceCap = 12288;   // slice elements a CTA holds (48 KB of keys)
constexpr int kMergeCap = 16384;   // candidates the merging CTA holds (S * k; 128 KB keys + indices)
constexpr int kSortSlots = 64;     // >= k
constexpr uint32_t kPadIdx = 0x7FFFFFFFu;

// Order key: a larger key ranks first.  Sign-0 patterns (positive numbers,
// +inf, sign-0 NaNs) map above sign-1 ones; within a sign the bit pattern's
// order is kept (sign 0) or reversed (sign 1), which is IEEE totalOrder.  The
// pattern of -0 is taken as +0 first, so the two tie.
__device__ __forceinline__ uint32_t order_key(uint32_t bits)
{
    if (bits == 0x80000000u) bits = 0u;
    return (bits & 0x80000000u) ? ~bits : (bits | 0x80000000u);
}

struct TopkParams {
    const float* logits;
    long long ldv;
    int V, k, S, slice;
    float* values;
    int32_t* indices;
    uint32_t* cand_key;   // [rows][kMergeCap]
    uint32_t* cand_idx;
    unsigned* counters;   // [rows]
};

struct SelectShared {
    unsigned hist[2][256];  // double-buffered: one pass fills one while the other is cleared
    uint32_t sel_key[kSortSlots], sel_idx[kSortSlots];  // the winners, in arrival order
    uint32_t out_key[kSortSlots], out_idx[kSortSlots];  // the winners, best first
    uint64_t wc[8 * 16];                                // small-k path: each warp's best, as composites
    int digit, above, ties, count;
    int last;
};

// Radix select over the elements for which `part(i, &v)` is true: the
// largest T with count(v >= T) >= want, digit by digit from the top byte.
// It stops early once the elements sharing the current prefix are exactly
// the ones still wanted; T then has zero low bits, and `count(v >= T)` is
// exactly `want` (r.all).  Otherwise T is a full value, r.need elements equal
// to it are wanted and r.ties of them exist.  All threads of the block call it.
struct Select {
    uint32_t T;
    int need, ties;
    bool all;  // take every v >= T (exactly `want` elements)
};

template <class Part>
__device__ Select radix_select(int n, int want, Part part, SelectShared& sh)
{
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    uint32_t prefix = 0u, mask = 0u;
    Select r{0u, want, 0, false};
    sh.hist[0][tid] = 0u;  // kTopkThreads == 256 bins
    __syncthreads();
    int b = 0;
    for (int shift = 24; shift >= 0; shift -= 8, b ^= 1) {
        for (int base = 0; base < n; base += kTopkThreads) {
            const int i = base + tid;
            uint32_t v = 0u;
            bool ok = false;
            if (i < n) ok = part(i, &v) && ((v & mask) == prefix);
            const unsigned d = ok ? ((v >> shift) & 255u) : 256u;
            const unsigned peers = __match_any_sync(0xffffffffu, d);
            if (ok && lane == __ffs(peers) - 1) atomicAdd(&sh.hist[b][d], (unsigned)__popc(peers));
        }
        __syncthreads();
        if (warp == 0) {
            // lane l covers bins 255-8l down to 248-8l; counts run from the top bin down
            unsigned c[8], local = 0u;
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                c[j] = sh.hist[b][255 - 8 * lane - j];
                local += c[j];
            }
            unsigned incl = local;
#pragma unroll
            for (int off = 1; off < 32; off <<= 1) {
                const unsigned o = __shfl_up_sync(0xffffffffu, incl, off);
                if (lane >= off) incl += o;
            }
            const unsigned excl = incl - local;
            if (lane == 0) {
                sh.digit = 0;
                sh.above = 0;
                sh.ties = 0;
            }
            __syncwarp();
            if (excl < (unsigned)want && (unsigned)want <= incl) {
                unsigned run = excl;
#pragma unroll
                for (int j = 0; j < 8; ++j) {
                    if (run < (unsigned)want && (unsigned)want <= run + c[j]) {
                        sh.digit = 255 - 8 * lane - j;
                        sh.above = (int)run;
                        sh.ties = (int)c[j];
                    }
                    run += c[j];
                }
            }
        } else {
            for (int j = tid - 32; j < 256; j += kTopkThreads - 32) sh.hist[b ^ 1][j] = 0u;  // for the next pass
        }
        __syncthreads();
        const int digit = sh.digit, above = sh.above, ties = sh.ties;
        prefix |= (uint32_t)digit << shift;
        mask |= 0xFFu << shift;
        want -= above;
        r.T = prefix;
        r.need = want;
        r.ties = ties;
        if (ties == want) {
            r.all = true;
            break;
        }
    }
    __syncthreads();  // every thread has read sh before anyone writes it again
    return r;
}

// Select the top `kk` (kk <= n, kk <= kSortSlots) of n elements given by
// key(i) and idx(i), and leave them best first in sh.out_key/out_idx.
template <class KeyF, class IdxF>
__device__ void block_topk(int n, int kk, KeyF key, IdxF idx, SelectShared& sh)
{
    const int tid = threadIdx.x;
    const Select s1 = radix_select(n, kk, [&](int i, uint32_t* v) { *v = key(i); return true; }, sh);
    // Among the elements tied at T, the `need` with the smallest indices: the
    // largest ~idx, found the same way.
    uint32_t t2 = 0u;
    const bool all = s1.all;
    if (!all) {
        const Select s2 = radix_select(
            n, s1.need,
            [&](int i, uint32_t* v) {
                if (key(i) != s1.T) return false;
                *v = ~idx(i);
                return true;
            },
            sh);
        t2 = s2.T;  // ~idx >= t2 picks exactly s1.need of the tied elements
    }
    if (tid == 0) sh.count = 0;
    if (tid < kSortSlots) {
        sh.out_key[tid] = 0u;
        sh.out_idx[tid] = kPadIdx;
    }
    __syncthreads();
    for (int i = tid; i < n; i += kTopkThreads) {
        const uint32_t v = key(i);
        if (all ? v >= s1.T : (v > s1.T || (v == s1.T && ~idx(i) >= t2))) {
            const int pos = atomicAdd(&sh.count, 1);
            if (pos < kSortSlots) {
                sh.sel_key[pos] = v;
                sh.sel_idx[pos] = idx(i);
            }
        }
    }
    __syncthreads();
    // Order the winners: each one's place is the number of winners that rank
    // before it on (key, lower index); all of them are distinct.
    const int cnt = sh.count < kSortSlots ? sh.count : kSortSlots;
    if (tid < cnt) {
        const uint32_t mk = sh.sel_key[tid], mi = sh.sel_idx[tid];
        int rank = 0;
        for (int j = 0; j < cnt; ++j) {
            const uint32_t ok = sh.sel_key[j], oi = sh.sel_idx[j];
            rank += (ok > mk || (ok == mk && oi < mi)) ? 1 : 0;
        }
        sh.out_key[rank] = mk;
        sh.out_idx[rank] = mi;
    }
    __syncthreads();
}

// Small k (k <= KL <= 16): the same selection without histograms.  An
// element's composite (key << 32 | ~index) orders it exactly as the ranking
// does (larger is better) and is never 0, so 0 marks an empty slot.  Each
// thread keeps its best KL composites sorted in registers; each warp then
// takes its best kk in kk rounds of an arg-max across the lanes' list heads
// (the winning lane shifts its list); warp 0 merges the eight warps' results
// the same way.  Result: sh.out_key / out_idx, best first.
template <int KL, class KeyF, class IdxF>
__device__ void small_topk(int n, int kk, KeyF key, IdxF idx, SelectShared& sh)
{
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    uint64_t L[KL];
#pragma unroll
    for (int j = 0; j < KL; ++j) L[j] = 0ull;
    for (int i = tid; i < n; i += kTopkThreads) {
        const uint64_t c = ((uint64_t)key(i) << 32) | (uint32_t)~idx(i);
        if (c > L[KL - 1]) {
#pragma unroll
            for (int j = KL - 1; j > 0; --j) L[j] = c > L[j - 1] ? L[j - 1] : (c > L[j] ? c : L[j]);
            L[0] = c > L[0] ? c : L[0];
        }
    }
    if (tid < 8 * 16) sh.wc[tid] = 0ull;
    __syncthreads();
    uint64_t mine = 0ull;  // lane r keeps the warp's r-th best
    for (int r = 0; r < kk; ++r) {
        uint64_t best = L[0];
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) {
            const uint64_t o = __shfl_xor_sync(0xffffffffu, best, off);
            best = o > best ? o : best;
        }
        if (best != 0ull && L[0] == best) {
#pragma unroll
            for (int j = 0; j < KL - 1; ++j) L[j] = L[j + 1];
            L[KL - 1] = 0ull;
        }
        if (lane == r) mine = best;
    }
    if (lane < kk) sh.wc[warp * KL + lane] = mine;
    __syncthreads();
    if (warp == 0) {
        constexpr int kPer = KL * (kTopkThreads / 32) / 32;  // candidates per lane
        uint64_t C[kPer];
#pragma unroll
        for (int q = 0; q < kPer; ++q) C[q] = sh.wc[lane + 32 * q];
        for (int r = 0; r < kk; ++r) {
            uint64_t best = C[0];
#pragma unroll
            for (int q = 1; q < kPer; ++q) best = C[q] > best ? C[q] : best;
#pragma unroll
            for (int off = 16; off > 0; off >>= 1) {
                const uint64_t o = __shfl_xor_sync(0xffffffffu, best, off);
                best = o > best ? o : best;
            }
#pragma unroll
            for (int q = 0; q < kPer; ++q)
                if (best != 0ull && C[q] == best) C[q] = 0ull;
            if (lane == 0) {
                sh.out_key[r] = (uint32_t)(best >> 32);
                sh.out_idx[r] = ~(uint32_t)best;
            }
        }
    }
    __syncthreads();
}

// The selection for kk winners, best first, in sh.out_key / out_idx.
template <class KeyF, class IdxF>
__device__ void select_topk(int n, int kk, KeyF key, IdxF idx, SelectShared& sh)
{
    if (kk <= 8)
        small_topk<8>(n, kk, key, idx, sh);
    else if (kk <= 16)
        small_topk<16>(n, kk, key, idx, sh);
    else
        block_topk(n, kk, key, idx, sh);
}

__global__ void __launch_bounds__(kTopkThreads) topk_kernel(const TopkParams p)
{
    extern __shared__ __align__(16) uint32_t tk_smem[];
    __shared__ SelectShared sh;
    const int tid = threadIdx.x;
    const int m = blockIdx.y, s = blockIdx.x;
    const int lo = s * p.slice;
    const int n = (p.V - lo < p.slice) ? p.V - lo : p.slice;  // >= 1: every slice is non-empty
    const float* row = p.logits + (long long)m * p.ldv;
    // Programmatic launch: let the next kernel start early, and read the
    // logits only once the kernel that produced them has finished.
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    asm volatile("griddepcontrol.wait;" ::: "memory");

    // 1. the slice as order keys (16-byte loads; lo and the row start are 16-byte aligned)
    uint32_t* keys = tk_smem;
    for (int i = 4 * tid; i < n; i += 4 * kTopkThreads) {
        if (i + 4 <= n) {
            const uint4 b = __ldg(reinterpret_cast<const uint4*>(row + lo + i));
            keys[i] = order_key(b.x);
            keys[i + 1] = order_key(b.y);
            keys[i + 2] = order_key(b.z);
            keys[i + 3] = order_key(b.w);
        } else {
            for (int j = i; j < n; ++j) keys[j] = order_key(__float_as_uint(__ldg(row + lo + j)));
        }
    }
    __syncthreads();
    const int kl = p.k < n ? p.k : n;
    select_topk(
        n, kl, [&](int i) { return keys[i]; }, [&](int i) { return (uint32_t)(lo + i); }, sh);

    // 2. publish this slice's candidates (padding past kl ranks below every real element)
    uint32_t* ck = p.cand_key + (long long)m * kMergeCap + (long long)s * p.k;
    uint32_t* ci = p.cand_idx + (long long)m * kMergeCap + (long long)s * p.k;
    if (tid < p.k) {
        ck[tid] = tid < kl ? sh.out_key[tid] : 0u;
        ci[tid] = tid < kl ? sh.out_idx[tid] : kPadIdx - (uint32_t)(s * p.k + tid);
    }
    // The CTA barrier orders every writer's stores before thread 0's count-in,
    // whose release side publishes them at GPU scope (cumulatively) and whose
    // acquire side orders the merge's loads after the other CTAs' stores.
    __syncthreads();
    if (tid == 0) {
        unsigned old;
        asm volatile("atom.acq_rel.gpu.global.add.u32 %0, [%1], 1;" : "=r"(old) : "l"(p.counters + m) : "memory");
        sh.last = (old == (unsigned)(p.S - 1)) ? 1 : 0;
    }
    __syncthreads();
    if (!sh.last) return;

    // 3. the row's last CTA merges every slice's candidates
    const int n2 = p.S * p.k;
    uint32_t* mk = tk_smem;
    uint32_t* mi = tk_smem + n2;
    const uint32_t* gk = p.cand_key + (long long)m * kMergeCap;
    const uint32_t* gi = p.cand_idx + (long long)m * kMergeCap;
    for (int i = tid; i < n2; i += kTopkThreads) {
        mk[i] = __ldcg(gk + i);
        mi[i] = __ldcg(gi + i);
    }
    __syncthreads();
    select_topk(
        n2, p.k, [&](int i) { return mk[i]; }, [&](int i) { return mi[i]; }, sh);
    if (tid < p.k) {
        const uint32_t id = sh.out_idx[tid];
        // the input's own bits (-0 stays -0); an index past V cannot occur, but is never read
        p.indices[(long long)m * p.k + tid] = id < (uint32_t)p.V ? (int32_t)id : -1;
        p.values[(long long)m * p.k + tid] = id < (uint32_t)p.V ? row[id] : __int_as_float(0x7fffffff);
    }
    if (tid == 0) p.counters[m] = 0u;  // ready for the next call
}

struct TopkState {
    int device = -1;
    int sm_count = 0;
    uint32_t* cand = nullptr;  // keys then indices
    unsigned* counters = nullptr;
    bool attr_set = false;
};
std::mutex g_topk_mu;
TopkState g_topk[64];

int topk_state(cudaStream_t stream, TopkState** out)
{
    int dev = 0;
    NVFP4_CUDA_TRY(cudaGetDevice(&dev));
    if (dev < 0 || dev >= 64) return NVFP4_ERR_ARG;
    std::lock_guard<std::mutex> lock(g_topk_mu);
    TopkState& s = g_topk[dev];
    if (s.device == dev) {
        *out = &s;
        return NVFP4_OK;
    }
    cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
    NVFP4_CUDA_TRY(cudaStreamIsCapturing(stream, &cs));
    if (cs != cudaStreamCaptureStatusNone) return NVFP4_ERR_CAPTURE;
    int sms = 0;
    NVFP4_CUDA_TRY(cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev));
    const size_t entries = (size_t)NVFP4_TOPK_MAX_ROWS * kMergeCap;
    uint32_t* cand = nullptr;
    unsigned* counters = nullptr;
    NVFP4_CUDA_TRY(cudaMalloc(&cand, 2 * entries * sizeof(uint32_t)));
    cudaError_t e = cudaMalloc(&counters, NVFP4_TOPK_MAX_ROWS * sizeof(unsigned));
    if (e == cudaSuccess) e = cudaMemset(counters, 0, NVFP4_TOPK_MAX_ROWS * sizeof(unsigned));
    if (e == cudaSuccess) e = cudaFuncSetAttribute(topk_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                                   2 * kMergeCap * (int)sizeof(uint32_t));
    if (e == cudaSuccess) e = cudaDeviceSynchronize();
    if (e != cudaSuccess) {
        cudaFree(cand);
        if (counters) cudaFree(counters);
        return fail_cuda(e);
    }
    s.sm_count = sms;
    s.cand = cand;
    s.counters = counters;
    s.device = dev;
    *out = &s;
    return NVFP4_OK;
}

}  // namespace

// Split count for a call: slices of at most kSliceCap elements; otherwise
// about sqrt(V / k) slices (balancing slice length against the merge), about
// two CTAs per SM over all rows, at least 256 elements per slice.
int topk_geometry(int rows, int64_t V, int k, int sm_count, int* S_out, int* slice_out)
{
    if (rows < 1 || rows > NVFP4_TOPK_MAX_ROWS) return NVFP4_ERR_M;
    if (k < 1 || k > NVFP4_TOPK_MAX_K || V < k || V > NVFP4_TOPK_MAX_V) return NVFP4_ERR_SHAPE;
    const long long s_min = (V + kSliceCap - 1) / kSliceCap;
    long long s = (2LL * sm_count + rows - 1) / rows;
    long long s_bal = 1;
    while (s_bal * s_bal * k < V) ++s_bal;
    if (s_bal < s) s = s_bal;
    const long long s_len = (V + 255) / 256;
    if (s_len < s) s = s_len;
    if (s < s_min) s = s_min;
    if (s < 1) s = 1;
    long long slice = (V + s - 1) / s;
    slice = (slice + 3) / 4 * 4;
    s = (V + slice - 1) / slice;  // no empty slice
    if (slice > kSliceCap || s * k > kMergeCap) return NVFP4_ERR_SHAPE;
    *S_out = (int)s;
    *slice_out = (int)slice;
    return NVFP4_OK;
}

}  // namespace nvfp4

using namespace nvfp4;

extern "C" int nvfp4_topk(const float* logits, int rows, int64_t V, int64_t ldv, int k, float* values,
                          int32_t* indices, cudaStream_t stream)
{
    if (!logits || !values || !indices) return NVFP4_ERR_ARG;
    if (rows < 1 || rows > NVFP4_TOPK_MAX_ROWS) return NVFP4_ERR_M;
    if (k < 1 || k > NVFP4_TOPK_MAX_K || V < k || V > NVFP4_TOPK_MAX_V || ldv < V) return NVFP4_ERR_SHAPE;
    if (!aligned16(logits) || (ldv & 3) != 0 || ((uintptr_t)values & 3) != 0 || ((uintptr_t)indices & 3) != 0)
        return NVFP4_ERR_ALIGN;
    TopkState* ts = nullptr;
    int st = topk_state(stream, &ts);
    if (st != NVFP4_OK) return st;
    int S = 0, slice = 0;
    st = topk_geometry(rows, V, k, ts->sm_count, &S, &slice);
    if (st != NVFP4_OK) return st;
    TopkParams p;
    p.logits = logits;
    p.ldv = ldv;
    p.V = (int)V;
    p.k = k;
    p.S = S;
    p.slice = slice;
    p.values = values;
    p.indices = indices;
    p.cand_key = ts->cand;
    p.cand_idx = ts->cand + (size_t)NVFP4_TOPK_MAX_ROWS * kMergeCap;
    p.counters = ts->counters;
    // shared memory: the slice's keys, or the merge's keys and indices, whichever is larger
    const size_t merge_bytes = (size_t)2 * S * k * sizeof(uint32_t);
    const size_t slice_bytes = (size_t)slice * sizeof(uint32_t);
    const size_t dyn = merge_bytes > slice_bytes ? merge_bytes : slice_bytes;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)S, (unsigned)rows);
    cfg.blockDim = dim3(kTopkThreads);
    cfg.dynamicSmemBytes = dyn;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    NVFP4_CUDA_TRY(cudaLaunchKernelEx(&cfg, topk_kernel, p));
    return NVFP4_OK;
}

extern "C" int nvfp4_topk_splits(int rows, int64_t V, int k, int sm_count, int* splits, int* slice)
{
    if (!splits || !slice || sm_count < 1) return NVFP4_ERR_ARG;
    return topk_geometry(rows, V, k, sm_count, splits, slice);
}
