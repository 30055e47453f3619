// pack.cu -- load-time pack of canonical NVFP4 planes into the device layout
// (layout.cuh), the NaN-scale scan, the two debug exports, and the host-side
// model of the layout used by CPU tests.
//
// "Models and artifacts", section "The artifact": the kernels read the weight
// planes directly, with no conversion on the host at load.  Here the one
// conversion is a byte permutation done on the device, once per matrix.
#include <cuda_runtime.h>
#include <stdint.h>
#include <string.h>

#include <mutex>

#include "dequant.cuh"
#include "internal.h"
#include "layout.cuh"

namespace nvfp4 {

__device__ unsigned long long g_bad_scales;

// Code (low nibble) of canonical element (n, k); zero outside the matrix.
__host__ __device__ __forceinline__ uint8_t canon_code(const uint8_t* q, int64_t N, int64_t K, int64_t n,
                                                       int64_t k)
{
    if (n >= N || k >= K) return 0;
    const uint8_t b = q[n * (K / 2) + (k >> 1)];
    return (k & 1) ? (uint8_t)(b >> 4) : (uint8_t)(b & 15u);
}

// One lane's share of unit (tile, chunk): 8 code words and its scale word.
__host__ __device__ __forceinline__ void pack_lane(const uint8_t* q, const uint8_t* s, int64_t N, int64_t K,
                                                   int64_t tile, int64_t chunk, int lane, uint32_t (&words)[8],
                                                   uint32_t& sword, unsigned& bad)
{
    const int g = lane >> 2, t = lane & 3;
    const int64_t row0 = tile * kTileN + g;
    const int64_t col0 = chunk * kChunkK + 16 * t;
    for (int r = 0; r < 2; ++r)
        for (int st = 0; st < 4; ++st) {
            uint8_t codes[8];
            for (int p = 0; p < 4; ++p)
                for (int h = 0; h < 2; ++h) {
                    const int64_t n = row0 + 16 * r + 8 * (p & 1);
                    const int64_t k = col0 + 4 * st + 2 * (p >> 1) + h;
                    codes[2 * p + h] = canon_code(q, N, K, n, k);
                }
            words[4 * r + st] = pack_code_word(codes);
        }
    sword = 0;
    bad = 0;
    const int64_t blk = col0 / 16;
    for (int r = 0; r < 2; ++r)
        for (int h = 0; h < 2; ++h) {
            const int64_t n = row0 + 16 * r + 8 * h;
            uint8_t b = 0;
            if (n < N && col0 < K) {
                b = s[n * (K / 16) + blk];
                if ((b & 0x7Fu) == 0x7Fu) ++bad;
            }
            sword |= (uint32_t)scale_store(b) << (8 * (2 * r + h));
        }
}

__global__ void pack_kernel(const uint8_t* __restrict__ q, const uint8_t* __restrict__ s, int64_t N, int64_t K,
                            int64_t k_chunks, int64_t units, uint8_t* __restrict__ wq_dev,
                            uint8_t* __restrict__ ws_dev)
{
    const int64_t tid = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    const int64_t u = tid >> 5;
    const int lane = (int)(tid & 31);
    if (u >= units) return;
    uint32_t words[8], sword;
    unsigned bad;
    pack_lane(q, s, N, K, u / k_chunks, u % k_chunks, lane, words, sword, bad);
    uint8_t* qu = wq_dev + u * kUnitQ;
    reinterpret_cast<uint4*>(qu)[lane] = make_uint4(words[0], words[1], words[2], words[3]);
    reinterpret_cast<uint4*>(qu + 512)[lane] = make_uint4(words[4], words[5], words[6], words[7]);
    reinterpret_cast<uint32_t*>(ws_dev + u * kUnitS)[lane] = sword;
    if (bad) atomicAdd(&g_bad_scales, (unsigned long long)bad);
}

__global__ void unpack_kernel(const uint8_t* __restrict__ wq_dev, const uint8_t* __restrict__ ws_dev, int64_t N,
                              int64_t K, int64_t k_chunks, int64_t units, uint8_t* __restrict__ q,
                              uint8_t* __restrict__ s)
{
    const int64_t tid = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    const int64_t u = tid >> 5;
    const int lane = (int)(tid & 31);
    if (u >= units) return;
    const int g = lane >> 2, t = lane & 3;
    const int64_t tile = u / k_chunks, chunk = u % k_chunks;
    const int64_t row0 = tile * kTileN + g, col0 = chunk * kChunkK + 16 * t;
    const uint4 a = reinterpret_cast<const uint4*>(wq_dev + u * kUnitQ)[lane];
    const uint4 b = reinterpret_cast<const uint4*>(wq_dev + u * kUnitQ + 512)[lane];
    const uint32_t words[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
    const uint32_t sword = reinterpret_cast<const uint32_t*>(ws_dev + u * kUnitS)[lane];
    if (col0 >= K) return;
    // codes of rows {g, g+8, 16+g, 24+g} at columns col0 .. col0+15
    uint8_t rowcodes[4][16];
    for (int r = 0; r < 2; ++r)
        for (int st = 0; st < 4; ++st) {
            uint8_t codes[8];
            unpack_code_word_codes(words[4 * r + st], codes);
            for (int p = 0; p < 4; ++p)
                for (int h = 0; h < 2; ++h)
                    rowcodes[2 * r + (p & 1)][4 * st + 2 * (p >> 1) + h] = codes[2 * p + h];
        }
    for (int r = 0; r < 2; ++r)
        for (int h = 0; h < 2; ++h) {
            const int64_t n = row0 + 16 * r + 8 * h;
            if (n >= N) continue;
            const uint8_t* rc = rowcodes[2 * r + h];
            for (int j = 0; j < 8; ++j)
                q[n * (K / 2) + col0 / 2 + j] = (uint8_t)(rc[2 * j] | (rc[2 * j + 1] << 4));
            s[n * (K / 16) + col0 / 16] = scale_load((uint8_t)(sword >> (8 * (2 * r + h))));
        }
}

__global__ void dequant_kernel(const uint8_t* __restrict__ wq_dev, const uint8_t* __restrict__ ws_dev,
                               float gscale, int64_t N, int64_t K, int64_t k_chunks, int64_t units,
                               float* __restrict__ W)
{
    const int64_t tid = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    const int64_t u = tid >> 5;
    const int lane = (int)(tid & 31);
    if (u >= units) return;
    const int g = lane >> 2, t = lane & 3;
    const int64_t tile = u / k_chunks, chunk = u % k_chunks;
    const int64_t row0 = tile * kTileN + g, col0 = chunk * kChunkK + 16 * t;
    const uint4 a = reinterpret_cast<const uint4*>(wq_dev + u * kUnitQ)[lane];
    const uint4 b = reinterpret_cast<const uint4*>(wq_dev + u * kUnitQ + 512)[lane];
    const uint32_t words[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
    const uint32_t sword = reinterpret_cast<const uint32_t*>(ws_dev + u * kUnitS)[lane];
    uint32_t S[2][2];
    scale_pairs(sword, S);
    for (int r = 0; r < 2; ++r)
        for (int st = 0; st < 4; ++st) {
            uint32_t frag[4];
            dequant_word(words[4 * r + st], S, r, frag);
            for (int p = 0; p < 4; ++p)
                for (int h = 0; h < 2; ++h) {
                    const int64_t n = row0 + 16 * r + 8 * (p & 1);
                    const int64_t k = col0 + 4 * st + 2 * (p >> 1) + h;
                    if (n < N && k < K) {
                        const uint32_t bits = (frag[p] >> (16 * h)) << 16;
                        W[n * K + k] = (__uint_as_float(bits) * kEpilogueScale) * gscale;
                    }
                }
        }
}

static std::mutex g_pack_mu;

static unsigned grid_for(int64_t units, int threads)
{
    return (unsigned)((units * 32 + threads - 1) / threads);
}

// ---------------------------------------------------------------- host model

// bf16 bits -> float (exact; subnormals included).
static float bf16_bits_to_float(uint32_t h16)
{
    uint32_t u = h16 << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return f;
}

// float -> bf16 bits, round to nearest even (no NaN inputs here).
static uint32_t float_to_bf16_bits(float f)
{
    uint32_t u;
    memcpy(&u, &f, sizeof u);
    return (u + 0x7FFFu + ((u >> 16) & 1u)) >> 16;
}

// bf16 multiply of each half, computed exactly and rounded to bf16.
static uint32_t host_hmul2(uint32_t a, uint32_t b)
{
    uint32_t r = 0;
    for (int h = 0; h < 2; ++h) {
        const float x = bf16_bits_to_float((a >> (16 * h)) & 0xFFFFu);
        const float y = bf16_bits_to_float((b >> (16 * h)) & 0xFFFFu);
        r |= float_to_bf16_bits((float)((double)x * (double)y)) << (16 * h);
    }
    return r;
}

}  // namespace nvfp4

using namespace nvfp4;

extern "C" int nvfp4_packed_bytes(int64_t N, int64_t K, size_t* wq_bytes, size_t* ws_bytes)
{
    if (!wq_bytes || !ws_bytes) return NVFP4_ERR_ARG;
    int st = check_shape(N, K);
    if (st != NVFP4_OK) return st;
    const Geometry geo = geometry(N, K);
    *wq_bytes = (size_t)geo.units * kUnitQ;
    *ws_bytes = (size_t)geo.units * kUnitS;
    return NVFP4_OK;
}

extern "C" int nvfp4_pack_check(const uint8_t* wq_canon, const uint8_t* ws_canon, int64_t N, int64_t K,
                                uint8_t* wq_dev, uint8_t* ws_dev, nvfp4_stream_t stream)
{
    if (!wq_canon || !ws_canon || !wq_dev || !ws_dev) return NVFP4_ERR_ARG;
    int st = check_shape(N, K);
    if (st != NVFP4_OK) return st;
    if (!aligned16(wq_dev) || !aligned16(ws_dev)) return NVFP4_ERR_ALIGN;
    const Geometry geo = geometry(N, K);
    cudaStream_t s = (cudaStream_t)stream;
    std::lock_guard<std::mutex> lock(g_pack_mu);
    const unsigned long long zero = 0;
    NVFP4_CUDA_TRY(cudaMemcpyToSymbolAsync(g_bad_scales, &zero, sizeof zero, 0, cudaMemcpyHostToDevice, s));
    pack_kernel<<<grid_for(geo.units, 256), 256, 0, s>>>(wq_canon, ws_canon, N, K, geo.k_chunks, geo.units,
                                                         wq_dev, ws_dev);
    NVFP4_CUDA_TRY(cudaGetLastError());
    unsigned long long bad = 0;
    NVFP4_CUDA_TRY(cudaMemcpyFromSymbolAsync(&bad, g_bad_scales, sizeof bad, 0, cudaMemcpyDeviceToHost, s));
    NVFP4_CUDA_TRY(cudaStreamSynchronize(s));
    return bad ? NVFP4_ERR_BAD_SCALE : NVFP4_OK;
}

extern "C" int nvfp4_unpack_debug(const uint8_t* wq_dev, const uint8_t* ws_dev, int64_t N, int64_t K,
                                  uint8_t* wq_canon, uint8_t* ws_canon, nvfp4_stream_t stream)
{
    if (!wq_dev || !ws_dev || !wq_canon || !ws_canon) return NVFP4_ERR_ARG;
    int st = check_shape(N, K);
    if (st != NVFP4_OK) return st;
    if (!aligned16(wq_dev) || !aligned16(ws_dev)) return NVFP4_ERR_ALIGN;
    const Geometry geo = geometry(N, K);
    unpack_kernel<<<grid_for(geo.units, 256), 256, 0, (cudaStream_t)stream>>>(
        wq_dev, ws_dev, N, K, geo.k_chunks, geo.units, wq_canon, ws_canon);
    NVFP4_CUDA_TRY(cudaGetLastError());
    return NVFP4_OK;
}

extern "C" int nvfp4_dequant_debug(const uint8_t* wq_dev, const uint8_t* ws_dev, float gscale, float* W,
                                   int64_t N, int64_t K, nvfp4_stream_t stream)
{
    if (!wq_dev || !ws_dev || !W) return NVFP4_ERR_ARG;
    int st = check_shape(N, K);
    if (st != NVFP4_OK) return st;
    if (!aligned16(wq_dev) || !aligned16(ws_dev) || !aligned16(W)) return NVFP4_ERR_ALIGN;
    const Geometry geo = geometry(N, K);
    dequant_kernel<<<grid_for(geo.units, 256), 256, 0, (cudaStream_t)stream>>>(
        wq_dev, ws_dev, gscale, N, K, geo.k_chunks, geo.units, W);
    NVFP4_CUDA_TRY(cudaGetLastError());
    return NVFP4_OK;
}

extern "C" int nvfp4_host_pack_unit(const uint8_t* wq_canon, const uint8_t* ws_canon, int64_t N, int64_t K,
                                    int64_t tile, int64_t chunk, uint8_t* q_unit, uint8_t* s_unit)
{
    if (!wq_canon || !ws_canon || !q_unit || !s_unit) return NVFP4_ERR_ARG;
    int st = check_shape(N, K);
    if (st != NVFP4_OK) return st;
    const Geometry geo = geometry(N, K);
    if (tile < 0 || tile >= geo.n_tiles || chunk < 0 || chunk >= geo.k_chunks) return NVFP4_ERR_ARG;
    for (int lane = 0; lane < 32; ++lane) {
        uint32_t words[8], sword;
        unsigned bad;
        pack_lane(wq_canon, ws_canon, N, K, tile, chunk, lane, words, sword, bad);
        memcpy(q_unit + 16 * lane, words, 16);
        memcpy(q_unit + 512 + 16 * lane, words + 4, 16);
        memcpy(s_unit + 4 * lane, &sword, 4);
    }
    return NVFP4_OK;
}

extern "C" int nvfp4_host_dequant_unit(const uint8_t* q_unit, const uint8_t* s_unit, float gscale, float* W)
{
    if (!q_unit || !s_unit || !W) return NVFP4_ERR_ARG;
    for (int lane = 0; lane < 32; ++lane) {
        const int g = lane >> 2, t = lane & 3;
        uint32_t words[8], sword;
        memcpy(words, q_unit + 16 * lane, 16);
        memcpy(words + 4, q_unit + 512 + 16 * lane, 16);
        memcpy(&sword, s_unit + 4 * lane, 4);
        // scale pairs, as the kernels form them
        const uint32_t rows_hi = sword & 0xFF00FF00u;
        const uint32_t rows_lo = (sword << 8) & 0xFF00FF00u;
        const uint32_t p_lo = host_hmul2(host_hmul2(scale_raw_pair(rows_lo), kBf16Pow2_119x2), kBf16Pow2_119x2);
        const uint32_t p_hi = host_hmul2(host_hmul2(scale_raw_pair(rows_hi), kBf16Pow2_119x2), kBf16Pow2_119x2);
        for (int r = 0; r < 2; ++r)
            for (int st = 0; st < 4; ++st) {
                uint32_t c[4];
                code_pairs(words[4 * r + st], c);
                for (int p = 0; p < 4; ++p) {
                    const uint32_t sc16 = ((p & 1) ? p_hi : p_lo) >> (16 * r) & 0xFFFFu;
                    const uint32_t sc = sc16 | (sc16 << 16);
                    const uint32_t v = host_hmul2(c[p], sc);
                    for (int h = 0; h < 2; ++h) {
                        const int n = g + 16 * r + 8 * (p & 1);
                        const int k = 16 * t + 4 * st + 2 * (p >> 1) + h;
                        W[n * kChunkK + k] = (bf16_bits_to_float((v >> (16 * h)) & 0xFFFFu) * kEpilogueScale) * gscale;
                    }
                }
            }
    }
    return NVFP4_OK;
}
