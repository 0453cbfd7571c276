// Warp-level W4A16 fragment arithmetic shared by the small-M streaming kernels.
//
// A 16 x 128 block of packed weights (16 rows, 16 words a row) meets up to 8 tokens in
// mma.m16n8k16 (weights in the 16-row slot). One LOP3 with the fp16 pattern of 1024 turns a
// word's nibbles into fp16 pairs x = 1024 + q (even nibble positions) or 1024 + 16 q (odd
// ones); the odd-position activations are pre-scaled by 1/16, so that the MMA returns
//     D = sum_k a_k q_k + sum_k c_k a_k,        c_k = 1024 (even) or 64 (odd),
// and one MMA against a constant operand returns corr = sum_k c_k a_k (rows 0..7) and
// sum_k a_k (rows 8..15). Per group, in fp32:
//     sum_k a_k (q_k - z) s = s * (D - corr - z * sum_k a_k).
// Lane (g, t) of the warp holds weight rows g and g + 8 and the 32 K values 32 t .. 32 t + 31
// of the block (its 16-byte piece of each row), and token g's activations at the same K.
// The K order inside an MMA is a permutation shared by both operands (the result is a sum).
#pragma once

#include "common.cuh"

namespace qg {

// fp16 bit patterns of the constant operand: rows 0..7 give sum c_k a_k, rows 8..15 sum a_k
__device__ __forceinline__ void w4_corr_operand(uint32_t (&k)[4])
{
    k[0] = 0x64006400u;   // row g,     K pair (2t, 2t+1):    1024, 1024 (meets unscaled a)
    k[1] = 0x3C003C00u;   // row g + 8, K pair (2t, 2t+1):    1, 1
    k[2] = 0x64006400u;   // row g,     K pair (2t+8, 2t+9):  1024 (meets a / 16: 64 a)
    k[3] = 0x4C004C00u;   // row g + 8, K pair (2t+8, 2t+9):  16 (meets a / 16: a)
}

// Activations of one lane (8 consecutive K values in v) paired like the codes the LOP3 upcast
// yields (natural packing: (a0,a4) (a1,a5) (a2,a6) (a3,a7); interleaved packing: (a0,a1)
// (a2,a3) (a4,a5) (a6,a7)), the pairs that meet 16 q scaled by 1/16.
template <bool ILV>
__device__ __forceinline__ void w4_act_pairs(const uint4 &v, uint32_t (&b)[4])
{
    constexpr uint32_t kInv16 = 0x2C002C00u;   // fp16 1/16 in both halves
    if constexpr (ILV) {
        b[0] = v.x;
        b[1] = hmul2_u32(v.y, kInv16);
        b[2] = v.z;
        b[3] = hmul2_u32(v.w, kInv16);
    } else {
        b[0] = prmt(v.x, v.z, 0x5410);
        b[1] = hmul2_u32(prmt(v.x, v.z, 0x7632), kInv16);
        b[2] = prmt(v.y, v.w, 0x5410);
        b[3] = hmul2_u32(prmt(v.y, v.w, 0x7632), kInv16);
    }
}

// One packed word of row g (xa) and of row g + 8 (xb) against the paired activations of the
// same 8 K values: two MMAs into two independent accumulation chains.
__device__ __forceinline__ void w4_word_mma(uint32_t xa, uint32_t xb, const uint32_t (&b)[4],
                                            float (&d)[4], float (&d2)[4])
{
    constexpr uint32_t kMagic = 0x64006400u, kLo = 0x000F000Fu, kHi = 0x00F000F0u;
    const uint32_t xa8 = xa >> 8, xb8 = xb >> 8;
    const uint32_t a0[4] = {lop3_and_or(xa, kLo, kMagic), lop3_and_or(xb, kLo, kMagic),
                            lop3_and_or(xa, kHi, kMagic), lop3_and_or(xb, kHi, kMagic)};
    const uint32_t a1[4] = {lop3_and_or(xa8, kLo, kMagic), lop3_and_or(xb8, kLo, kMagic),
                            lop3_and_or(xa8, kHi, kMagic), lop3_and_or(xb8, kHi, kMagic)};
    mma_16816_f16(d, a0, b[0], b[1], d);
    mma_16816_f16(d2, a1, b[2], b[3], d2);
}

} // namespace qg
