// dequant.cuh -- device-side register dequantisation of one lane's share of
// a 32 x 64 unit (see layout.cuh for the layout), and the bf16 tensor-core
// step that consumes it.  Used by the GEMM kernels and by the dequant debug
// export, so the exported weights are exactly the ones the GEMMs multiply.
#pragma once
#include <stdint.h>

#include "layout.cuh"

namespace nvfp4 {

__device__ __forceinline__ uint32_t hmul2_bf16(uint32_t a, uint32_t b)
{
    uint32_t r;
    asm("mul.rn.bf16x2 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(b));
    return r;
}

__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t b, uint32_t sel)
{
    uint32_t r;
    asm("prmt.b32 %0, %1, %2, %3;" : "=r"(r) : "r"(a), "r"(b), "r"(sel));
    return r;
}

// {lo, lo} and {hi, hi} of a bf16x2 (the multiply can take these as operand
// swizzles).
__device__ __forceinline__ uint32_t bcast_lo(uint32_t p)
{
    uint32_t r;
    asm("{\n .reg .b16 l, h;\n mov.b32 {l, h}, %1;\n mov.b32 %0, {l, l};\n}" : "=r"(r) : "r"(p));
    return r;
}
__device__ __forceinline__ uint32_t bcast_hi(uint32_t p)
{
    uint32_t r;
    asm("{\n .reg .b16 l, h;\n mov.b32 {l, h}, %1;\n mov.b32 %0, {h, h};\n}" : "=r"(r) : "r"(p));
    return r;
}

// The lane's four scales as broadcast bf16x2 pairs, each = e4m3 * 2^118:
// S[r][0] for row 16r+g, S[r][1] for row 16r+g+8.
__device__ __forceinline__ void scale_pairs(uint32_t sw, uint32_t (&S)[2][2])
{
    const uint32_t rows_hi = sw & 0xFF00FF00u;          // rows g+8 of groups 0, 1
    const uint32_t rows_lo = (sw << 8) & 0xFF00FF00u;   // rows g of groups 0, 1
    uint32_t p_lo = hmul2_bf16(hmul2_bf16(scale_raw_pair(rows_lo), kBf16Pow2_119x2), kBf16Pow2_119x2);
    uint32_t p_hi = hmul2_bf16(hmul2_bf16(scale_raw_pair(rows_hi), kBf16Pow2_119x2), kBf16Pow2_119x2);
    S[0][0] = bcast_lo(p_lo);
    S[0][1] = bcast_lo(p_hi);
    S[1][0] = bcast_hi(p_lo);
    S[1][1] = bcast_hi(p_hi);
}

// A fragment (a0a1, a2a3, a4a5, a6a7) of code word w of row group r:
// bf16x2 values e2m1 * e4m3 * 2^-8, exact.
__device__ __forceinline__ void dequant_word(uint32_t w, const uint32_t (&S)[2][2], int r,
                                             uint32_t (&a)[4])
{
    uint32_t c[4];
    code_pairs(w, c);
    a[0] = hmul2_bf16(c[0], S[r][0]);
    a[1] = hmul2_bf16(c[1], S[r][1]);
    a[2] = hmul2_bf16(c[2], S[r][0]);
    a[3] = hmul2_bf16(c[3], S[r][1]);
}

// d += A(16x16, bf16) . B(16x8, bf16), FP32 accumulation.
__device__ __forceinline__ void mma_bf16_16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0,
                                               uint32_t b1)
{
    asm("mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 "
        "{%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// One lane's share of one unit: dequantise its 8 code words (rows g, g+8,
// 16+g, 24+g; columns 16t..16t+15 of the unit, read from the stage in shared
// memory) and multiply them into acc with the lane's X fragment xw.
__device__ __forceinline__ void mma_unit(const uint8_t* sq, const uint8_t* ss, const uint32_t (&xw)[8],
                                         float (&acc)[2][4])
{
    const uint4 q0 = *reinterpret_cast<const uint4*>(sq);
    const uint4 q1 = *reinterpret_cast<const uint4*>(sq + 512);
    const uint32_t sw = *reinterpret_cast<const uint32_t*>(ss);
    const uint32_t q[8] = {q0.x, q0.y, q0.z, q0.w, q1.x, q1.y, q1.z, q1.w};
    uint32_t S[2][2];
    scale_pairs(sw, S);
#pragma unroll
    for (int r = 0; r < 2; ++r)
#pragma unroll
        for (int s = 0; s < 4; ++s) {
            uint32_t a[4];
            dequant_word(q[4 * r + s], S, r, a);
            mma_bf16_16816(acc[r], a, xw[2 * s], xw[2 * s + 1]);
        }
}

// The same for NB blocks of 8 decode lanes (M up to 8 * NB): each word is
// dequantised once and feeds one MMA per block; xw[b] and acc[b] belong to
// lanes 8b..8b+7.
template <int NB>
__device__ __forceinline__ void mma_unit_nb(const uint8_t* sq, const uint8_t* ss, const uint32_t (&xw)[NB][8],
                                            float (&acc)[NB][2][4])
{
    if constexpr (NB == 1) {
        mma_unit(sq, ss, xw[0], acc[0]);
    } else {
        const uint4 q0 = *reinterpret_cast<const uint4*>(sq);
        const uint4 q1 = *reinterpret_cast<const uint4*>(sq + 512);
        const uint32_t sw = *reinterpret_cast<const uint32_t*>(ss);
        const uint32_t q[8] = {q0.x, q0.y, q0.z, q0.w, q1.x, q1.y, q1.z, q1.w};
        uint32_t S[2][2];
        scale_pairs(sw, S);
#pragma unroll
        for (int r = 0; r < 2; ++r)
#pragma unroll
            for (int s = 0; s < 4; ++s) {
                uint32_t a[4];
                dequant_word(q[4 * r + s], S, r, a);
#pragma unroll
                for (int b = 0; b < NB; ++b) mma_bf16_16816(acc[b][r], a, xw[b][2 * s], xw[b][2 * s + 1]);
            }
    }
}

}  // namespace nvfp4
