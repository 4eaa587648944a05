// dequant_magic.cuh -- code -> exact fp16 (q - z) pairs with the magic-number
// trick, used by the tensor-core kernel (k_prefill.cuh) to write dequantized
// operand tiles.  OR-ing a code into the mantissa of 1024.0 (0x6400) gives the
// fp16 value 1024 + q*m exactly (m = 2^bit position); one HADD2/HFMA2 then
// removes the 1024 and the zero point.  The results are small integers, exact
// in fp16.  Pair layout: for one row, one 8-code group i of the lane's 32
// columns and j = 0..3, out[j] = (q[8i+j] - z, q[8i+j+4] - z).
#pragma once
#include "common.cuh"

namespace mpq {

constexpr uint32_t DEC_MAGIC = 0x64006400u;   // fp16 1024.0 in both halves

__device__ __forceinline__ uint32_t h2c(float lo, float hi) {
    return h2_bits(__halves2half2(__float2half_rn(lo), __float2half_rn(hi)));
}


// p = 4: word i holds codes 8i..8i+7 as nibbles.  c1 = -(1024 + z), c16 = -(64 + z).
__device__ __forceinline__ void ext4(uint32_t w, uint32_t c1, uint32_t c16, uint32_t (&o)[4]) {
    const uint32_t k116 = 0x2C002C00u;  // 1/16
    const uint32_t w8 = w >> 8;
    o[0] = h2_bits(__hadd2(bits_h2(lop_and_or(w, 0x000F000Fu, DEC_MAGIC)), bits_h2(c1)));
    o[1] = hfma2_bits(lop_and_or(w, 0x00F000F0u, DEC_MAGIC), k116, c16);
    o[2] = h2_bits(__hadd2(bits_h2(lop_and_or(w8, 0x000F000Fu, DEC_MAGIC)), bits_h2(c1)));
    o[3] = hfma2_bits(lop_and_or(w8, 0x00F000F0u, DEC_MAGIC), k116, c16);
}

// p = 2: bytes 2i, 2i+1 of the lane's 8 bytes hold codes 8i..8i+7.
// c[j] = -(1024/4^j + z) in both halves.
__device__ __forceinline__ void ext2(uint32_t v, int sel, const uint32_t (&c)[4], uint32_t (&o)[4]) {
    const uint32_t P = __byte_perm(v, 0u, sel);
    o[0] = h2_bits(__hadd2(bits_h2(lop_and_or(P, 0x00030003u, DEC_MAGIC)), bits_h2(c[0])));
    o[1] = hfma2_bits(lop_and_or(P, 0x000C000Cu, DEC_MAGIC), 0x34003400u, c[1]);  // 1/4
    o[2] = hfma2_bits(lop_and_or(P, 0x00300030u, DEC_MAGIC), 0x2C002C00u, c[2]);  // 1/16
    o[3] = hfma2_bits(lop_and_or(P, 0x00C000C0u, DEC_MAGIC), 0x24002400u, c[3]);  // 1/64
}

// p = 1: byte i of the lane's word holds codes 8i..8i+7 (bit k = code 8i+k).
// c[j] = (-(1024/2^j + z), -(1024/2^(j+4) + z)).
__device__ __forceinline__ void ext1(uint32_t u, int sel, const uint32_t (&c)[4], uint32_t (&o)[4]) {
    const uint32_t P = __byte_perm(u, 0u, sel);
    // low half scaled by 2^-j, high half by 2^-(j+4)
    o[0] = hfma2_bits(lop_and_or(P, 0x00100001u, DEC_MAGIC), 0x2C003C00u, c[0]);
    o[1] = hfma2_bits(lop_and_or(P, 0x00200002u, DEC_MAGIC), 0x28003800u, c[1]);
    o[2] = hfma2_bits(lop_and_or(P, 0x00400004u, DEC_MAGIC), 0x24003400u, c[2]);
    o[3] = hfma2_bits(lop_and_or(P, 0x00800008u, DEC_MAGIC), 0x20003000u, c[3]);
}

// p = 8: words 2i and 2i+1 hold codes 8i..8i+3 and 8i+4..8i+7 as bytes.
// c1 = -(1024 + z).
__device__ __forceinline__ void ext8(uint32_t xa, uint32_t xb, uint32_t c1, uint32_t (&o)[4]) {
    const uint32_t T0 = __byte_perm(xa, xb, 0x5140);
    const uint32_t T1 = __byte_perm(xa, xb, 0x7362);
    o[0] = h2_bits(__hadd2(bits_h2(__byte_perm(T0, 0x64646464u, 0x4140)), bits_h2(c1)));
    o[1] = h2_bits(__hadd2(bits_h2(__byte_perm(T0, 0x64646464u, 0x4342)), bits_h2(c1)));
    o[2] = h2_bits(__hadd2(bits_h2(__byte_perm(T1, 0x64646464u, 0x4140)), bits_h2(c1)));
    o[3] = h2_bits(__hadd2(bits_h2(__byte_perm(T1, 0x64646464u, 0x4342)), bits_h2(c1)));
}

// High piece of a split code, already multiplied by 2^w (w = low width):
// the exact values 2^w * hi, no zero point.  Magic-number pairs carry
// multipliers m (low half) / m' (high half); an HFMA2 with scale 2^w/m and
// offset -1024*2^w/m removes the magic.  The constants are fp16 bit patterns
// (low half in bits 0-15).
// p = 1: m = 2^j, m' = 2^(j+4).
template <int W>
__device__ __forceinline__ void ext1_hi(uint32_t u, int sel, uint32_t (&o)[4]) {
    const uint32_t P = __byte_perm(u, 0u, sel);
    // W = 2: scale (4/2^j, 4/2^(j+4)); W = 4: scale (16/2^j, 16/2^(j+4))
    constexpr uint32_t sc2[4] = {0x34004400u, 0x30004000u, 0x2C003C00u, 0x28003800u};
    constexpr uint32_t of2[4] = {0xDC00EC00u, 0xD800E800u, 0xD400E400u, 0xD000E000u};
    constexpr uint32_t sc4[4] = {0x3C004C00u, 0x38004800u, 0x34004400u, 0x30004000u};
    constexpr uint32_t of4[4] = {0xE400F400u, 0xE000F000u, 0xDC00EC00u, 0xD800E800u};
    const uint32_t msk[4] = {0x00100001u, 0x00200002u, 0x00400004u, 0x00800008u};
#pragma unroll
    for (int j = 0; j < 4; ++j)
        o[j] = hfma2_bits(lop_and_or(P, msk[j], DEC_MAGIC), W == 2 ? sc2[j] : sc4[j],
                          W == 2 ? of2[j] : of4[j]);
}
// p = 2 (w = 4): m = m' = 4^j: scale 16/4^j, offset -16384/4^j.
__device__ __forceinline__ void ext2_hi(uint32_t v, int sel, uint32_t (&o)[4]) {
    const uint32_t P = __byte_perm(v, 0u, sel);
    constexpr uint32_t sc[4] = {0x4C004C00u, 0x44004400u, 0x3C003C00u, 0x34003400u};
    constexpr uint32_t of[4] = {0xF400F400u, 0xEC00EC00u, 0xE400E400u, 0xDC00DC00u};
    const uint32_t msk[4] = {0x00030003u, 0x000C000Cu, 0x00300030u, 0x00C000C0u};
#pragma unroll
    for (int j = 0; j < 4; ++j) o[j] = hfma2_bits(lop_and_or(P, msk[j], DEC_MAGIC), sc[j], of[j]);
}

// Zero-point constants for a row with zero point z (an fp16 integer).
__device__ __forceinline__ uint32_t zc(float base, float z) { return h2c(-(base + z), -(base + z)); }

// The same constants from z as (z, z) fp16 pair bits: -(base + z) = z*(-1) - base,
// exact in fp16 (base + z <= 1279).
__device__ __forceinline__ uint32_t zc2(uint32_t z2, uint32_t neg_base2) {
    return hfma2_bits(z2, 0xBC00BC00u, neg_base2);
}

// Low-piece zero-point constants for a row (see the ext* functions).
template <int P0>
__device__ __forceinline__ void zero_consts(uint32_t z2, uint32_t (&k)[4]) {
    if (P0 == 4) {
        k[0] = zc2(z2, 0xE400E400u);        // -(1024 + z)
        k[1] = zc2(z2, 0xD400D400u);        // -(64 + z)
    } else if (P0 == 8) {
        k[0] = zc2(z2, 0xE400E400u);
    } else if (P0 == 2) {
        k[0] = zc2(z2, 0xE400E400u);        // -(1024 + z)
        k[1] = zc2(z2, 0xDC00DC00u);        // -(256 + z)
        k[2] = zc2(z2, 0xD400D400u);        // -(64 + z)
        k[3] = zc2(z2, 0xCC00CC00u);        // -(16 + z)
    } else {
        k[0] = zc2(z2, 0xD400E400u);        // (-(1024 + z), -(64 + z))
        k[1] = zc2(z2, 0xD000E000u);        // (-(512 + z),  -(32 + z))
        k[2] = zc2(z2, 0xCC00DC00u);        // (-(256 + z),  -(16 + z))
        k[3] = zc2(z2, 0xC800D800u);        // (-(128 + z),  -(8 + z))
    }
}


}  // namespace mpq
