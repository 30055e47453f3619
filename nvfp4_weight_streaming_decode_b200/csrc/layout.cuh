// layout.cuh -- the device layout of an NVFP4 matrix and the register-level
// dequantisation that reads it.  Shared by the pack, debug and GEMM kernels
// and by the host-side model of the layout.
//
// Format ("Models and artifacts", section "The artifact"): 4-bit E2M1
// elements, one E4M3 scale per 16 consecutive K values, plus an FP32 global
// scale; the kernels read these planes directly.
//
// Work unit.  A matrix is cut into units of 32 rows x 64 columns.  A unit is
// 1024 nibble bytes plus 128 scale bytes, and is what one warp consumes per
// step; units are stored tile-major (all K-chunks of rows 0..31, then rows
// 32..63, ...), so any run of consecutive units is one contiguous run of
// bytes in each plane.
//
// Inside a unit, lane l = 4g + t of a warp owns rows {g, g+8, 16+g, 24+g}
// and columns [16t, 16t+16) -- exactly one scale block per row.  It holds
// 8 code words (32 bytes: bytes [16l, 16l+16) and [512+16l, 512+16l+16) of
// the nibble block) and one scale word (bytes [4l, 4l+4) of the scale block).
//
// Code words.  Word j = 4r + s (row group r = 0/1, MMA step s = 0..3) holds
// the 8 codes that lane feeds to one m16n8k16 MMA as its A fragment:
//   pair 0 -> a0,a1 : row 16r+g,   columns 16t+4s+{0,1}
//   pair 1 -> a2,a3 : row 16r+g+8, columns 16t+4s+{0,1}
//   pair 2 -> a4,a5 : row 16r+g,   columns 16t+4s+{2,3}
//   pair 3 -> a6,a7 : row 16r+g+8, columns 16t+4s+{2,3}
// (The MMA's k index runs over a permutation of the actual columns; the
// activation fragments use the same permutation, so the dot product is the
// same.)  The bits of the 8 codes are placed so that each pair comes out of
// the word as a bf16x2 register with one rotate and one AND (pair 3: two of
// each).  A code c = (sign, e1, e0, m) lands at bf16 bits 15, 8, 7, 6 of its
// half: as a bf16 number that is exactly e2m1(c) * 2^-126, subnormal case
// included, because E2M1 and bf16 share the subnormal rule with biases 1
// and 127.
//
// Scale word.  Bytes [row 16r+g, row 16r+g+8] for r = 0, 1, each stored as a
// bit permutation of its E4M3 code chosen so that one shift and one 3-input
// logic op yield the bf16 pattern sign<<15 | exponent<<7 | mantissa<<4,
// which is exactly e4m3(b) * 2^-120 (subnormal codes included).  Two exact
// bf16 multiplies by 2^119 bring it to scale * 2^118; the product with a
// code is then e2m1 * e4m3 * 2^-8, exact in bf16 (at most 6 significant
// bits, magnitude within [2^-18, 10.5]).  The GEMM epilogue multiplies the
// FP32 accumulator by 2^8 and the global scale.
#pragma once
#include <stdint.h>

#if defined(__CUDACC__)
#define NVFP4_HD __host__ __device__ __forceinline__
#else
#define NVFP4_HD inline
#endif

namespace nvfp4 {

constexpr int kTileN = 32;          // rows per unit
constexpr int kChunkK = 64;         // columns per unit
constexpr int kUnitQ = 1024;        // nibble bytes per unit
constexpr int kUnitS = 128;         // scale bytes per unit
constexpr int kUnitBytes = kUnitQ + kUnitS;
constexpr int kMaxM = 8;            // decode lanes
constexpr int kWideMaxM = 32;       // plain-GEMM rows on the register-MMA path (up to four blocks of 8)

// bf16x2 bit positions of the two codes of a pair: sign, e1, e0, m.
constexpr uint32_t kPairMask = 0x81C081C0u;
// Rotations (right) that bring pairs 0..3 to kPairMask; pair 3 takes its
// mantissa bits (6 and 22) from rotation kRot3b and the rest from kRot3a.
constexpr int kRot1 = 22, kRot2 = 28, kRot3a = 2, kRot3b = 10;
constexpr uint32_t kPair3MaskB = 0x00400040u;
constexpr uint32_t kPair3MaskA = kPairMask & ~kPair3MaskB;

NVFP4_HD uint32_t rotr32(uint32_t x, int r)
{
#if defined(__CUDA_ARCH__)
    return __funnelshift_r(x, x, r);
#else
    return r == 0 ? x : ((x >> r) | (x << (32 - r)));
#endif
}

// Rotation that feeds output bit `bit` of pair p.
NVFP4_HD int pair_rotation(int p, int bit)
{
    return p == 0 ? 0 : p == 1 ? kRot1 : p == 2 ? kRot2 : ((bit == 6 || bit == 22) ? kRot3b : kRot3a);
}

// Output bit of code bit cb (0 = m, 1 = e0, 2 = e1, 3 = sign) in half h.
NVFP4_HD int code_bit_target(int h, int cb)
{
    return 16 * h + (cb == 0 ? 6 : cb == 1 ? 7 : cb == 2 ? 8 : 15);
}

// Word bit that holds code bit cb of the half-h element of pair p.
NVFP4_HD int code_bit_source(int p, int h, int cb)
{
    int t = code_bit_target(h, cb);
    return (t + pair_rotation(p, t)) & 31;
}

// Place 8 codes (pair p, half h -> codes[2p + h], low nibble used) in a word.
NVFP4_HD uint32_t pack_code_word(const uint8_t codes[8])
{
    uint32_t w = 0;
    for (int p = 0; p < 4; ++p)
        for (int h = 0; h < 2; ++h)
            for (int cb = 0; cb < 4; ++cb)
                w |= (uint32_t)((codes[2 * p + h] >> cb) & 1u) << code_bit_source(p, h, cb);
    return w;
}

NVFP4_HD void unpack_code_word_codes(uint32_t w, uint8_t codes[8])
{
    for (int p = 0; p < 4; ++p)
        for (int h = 0; h < 2; ++h) {
            uint32_t c = 0;
            for (int cb = 0; cb < 4; ++cb) c |= ((w >> code_bit_source(p, h, cb)) & 1u) << cb;
            codes[2 * p + h] = (uint8_t)c;
        }
}

// The four bf16x2 code pairs of a word (each value = e2m1 * 2^-126).
NVFP4_HD void code_pairs(uint32_t w, uint32_t out[4])
{
    out[0] = w & kPairMask;
    out[1] = rotr32(w, kRot1) & kPairMask;
    out[2] = rotr32(w, kRot2) & kPairMask;
    out[3] = (rotr32(w, kRot3a) & kPair3MaskA) | (rotr32(w, kRot3b) & kPair3MaskB);
}

// Stored form of an E4M3 scale byte b = s eeee mmm (bit 7 .. bit 0):
// stored bits 0..7 = E1 E2 E3 m0 m1 m2 E0 s.
NVFP4_HD uint8_t scale_store(uint8_t b)
{
    uint32_t E = (b >> 3) & 15u, m = b & 7u, s = b >> 7;
    return (uint8_t)(((E >> 1) & 7u) | (m << 3) | ((E & 1u) << 6) | (s << 7));
}

NVFP4_HD uint8_t scale_load(uint8_t B)
{
    uint32_t E = ((B & 7u) << 1) | ((B >> 6) & 1u), m = (B >> 3) & 7u, s = B >> 7;
    return (uint8_t)((s << 7) | (E << 3) | m);
}

// x holds stored scale bytes in bytes 1 and 3 (bytes 0 and 2 zero); returns
// the bf16x2 patterns sign<<15 | E<<7 | m<<4 of both (= e4m3 * 2^-120).
// Per bit: where the constant is 1 take (x >> 7) & ~x, elsewhere take x.
NVFP4_HD uint32_t scale_raw_pair(uint32_t x)
{
    uint32_t y = x >> 7;
    const uint32_t c = 0x78F078F0u;
#if defined(__CUDA_ARCH__)
    uint32_t r;
    // lop3 truth table for f(a=x, b=y, c) = c ? (b & ~a) : a
    //   a=0xF0, b=0xCC, c=0xAA: (0xAA & 0xCC & 0x0F) | (0x55 & 0xF0) = 0x08 | 0x50 = 0x58
    asm("lop3.b32 %0, %1, %2, %3, 0x58;" : "=r"(r) : "r"(x), "r"(y), "r"(c));
    return r;
#else
    return (c & y & ~x) | (~c & x);
#endif
}

constexpr uint32_t kBf16Pow2_119x2 = 0x7B007B00u;  // bf16x2 {2^119, 2^119}
constexpr float kEpilogueScale = 256.0f;           // undoes the 2^-8 of the products

}  // namespace nvfp4
