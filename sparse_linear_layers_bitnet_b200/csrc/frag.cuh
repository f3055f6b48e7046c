// Warp-level pieces shared by the decode kernels: the int8 code of one
// activation, the expansion of 2-bit ternary codes to int8 A-fragment
// registers, and the m16n8k64 sparse MMA with ordered metadata.
#pragma once

#include <cstdint>

namespace bitnet {

// int8 code of one activation: clamp(rint(fp32(x * s)), -127, 127)
__device__ __forceinline__ int8_t quant_code(float x, float s) {
    int q = __float2int_rn(__fmul_rn(x, s));
    q = q > 127 ? 127 : (q < -127 ? -127 : q);
    return static_cast<int8_t>(q);
}

__device__ __forceinline__ uint32_t expand_codes(uint32_t codes, int r) {
    // bytes of t hold 2-bit codes {0: 0, 1: +1, 3: -1}; int8 = t + (t & 2) * 0x7e
    // (3 -> 3 + 252 = 0xff, 1 -> 1, 0 -> 0; no byte carries into the next)
    const uint32_t t = (codes >> (2 * r)) & 0x03030303u;
    return (t & 0x02020202u) * 0x7eu + t;
}

// Codes of register r as int8 values 64 c (c in {-1, 0, 1}): the two code bits
// moved to bits 6-7 of each byte, the rest cleared (00 -> 0, 01 -> 64,
// 11 -> -64).  Two instructions instead of four; a product accumulated from
// these is 64 times the ternary one, exactly (int32 holds 64 * 127 * k / 2
// for k < 2^18), and an arithmetic shift by 6 recovers it.
__device__ __forceinline__ uint32_t expand_codes_x64(uint32_t codes, int r) {
    return (codes << (6 - 2 * r)) & 0xC0C0C0C0u;
}

__device__ __forceinline__ void mma_sp_m16n8k64(int (&d)[4], const uint32_t (&a)[4], const uint32_t (&b)[4],
                                                uint32_t e) {
    asm volatile(
        "mma.sp::ordered_metadata.sync.aligned.m16n8k64.row.col.s32.s8.s8.s32 "
        "{%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9, %10, %11}, {%0, %1, %2, %3}, %12, 0x0;"
        : "+r"(d[0]), "+r"(d[1]), "+r"(d[2]), "+r"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b[0]), "r"(b[1]), "r"(b[2]), "r"(b[3]), "r"(e));
}

}  // namespace bitnet
