// convert.cuh -- FP4 (E2M1) and FP8 (E4M3) conversions through the sm_100a cvt instructions.
#pragma once

#include <stdint.h>

namespace csa {

// Eight floats -> eight E2M1 codes (round-to-nearest-even, saturating), x[0] in the low nibble.
__device__ __forceinline__ uint32_t f32x8_to_e2m1x8(const float *x)
{
    uint32_t out;
    asm("{\n"
        ".reg .b8 b0, b1, b2, b3;\n"
        "cvt.rn.satfinite.e2m1x2.f32 b0, %2, %1;\n"
        "cvt.rn.satfinite.e2m1x2.f32 b1, %4, %3;\n"
        "cvt.rn.satfinite.e2m1x2.f32 b2, %6, %5;\n"
        "cvt.rn.satfinite.e2m1x2.f32 b3, %8, %7;\n"
        "mov.b32 %0, {b0, b1, b2, b3};\n"
        "}"
        : "=r"(out)
        : "f"(x[0]), "f"(x[1]), "f"(x[2]), "f"(x[3]), "f"(x[4]), "f"(x[5]), "f"(x[6]), "f"(x[7]));
    return out;
}

// Two floats -> two E4M3 codes (round-to-nearest-even, saturating), lo in the low byte.
__device__ __forceinline__ uint16_t f32x2_to_e4m3x2(float lo, float hi)
{
    uint16_t out;
    asm("cvt.rn.satfinite.e4m3x2.f32 %0, %2, %1;" : "=h"(out) : "f"(lo), "f"(hi));
    return out;
}

// Two E4M3 codes (low byte first) -> two halves packed in a 32-bit word (exact).
__device__ __forceinline__ uint32_t e4m3x2_to_f16x2(uint16_t v)
{
    uint32_t out;
    asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(out) : "h"(v));
    return out;
}

// Two E2M1 codes (one byte, low nibble first) -> two halves packed in a 32-bit word (exact).
__device__ __forceinline__ uint32_t e2m1x2_to_f16x2(uint8_t v)
{
    uint32_t out;
    asm("{\n"
        ".reg .b8 b;\n"
        "cvt.u8.u16 b, %1;\n"
        "cvt.rn.f16x2.e2m1x2 %0, b;\n"
        "}"
        : "=r"(out)
        : "h"((uint16_t)v));
    return out;
}

// Four E2M1 byte pairs of a word (byte 0 first) -> four f16x2 words (exact).  The word is split into
// byte registers with one vector move, which the conversions read directly; narrowing one byte at a
// time (as e2m1x2_to_f16x2 does) costs a second conversion instruction per byte, which halves the
// throughput of a dequantisation loop.
__device__ __forceinline__ void e2m1x8_to_f16x2x4(uint32_t w, uint32_t *out)
{
    asm("{\n"
        ".reg .b8 b0, b1, b2, b3;\n"
        "mov.b32 {b0, b1, b2, b3}, %4;\n"
        "cvt.rn.f16x2.e2m1x2 %0, b0;\n"
        "cvt.rn.f16x2.e2m1x2 %1, b1;\n"
        "cvt.rn.f16x2.e2m1x2 %2, b2;\n"
        "cvt.rn.f16x2.e2m1x2 %3, b3;\n"
        "}"
        : "=r"(out[0]), "=r"(out[1]), "=r"(out[2]), "=r"(out[3])
        : "r"(w));
}

// Four E4M3 codes of a word (byte 0 first) -> two f16x2 words, (byte 0, byte 1) and (byte 2, byte 3),
// through one vector move into 16-bit registers (exact).
__device__ __forceinline__ void e4m3x4_to_f16x2x2(uint32_t w, uint32_t *out)
{
    asm("{\n"
        ".reg .b16 h0, h1;\n"
        "mov.b32 {h0, h1}, %2;\n"
        "cvt.rn.f16x2.e4m3x2 %0, h0;\n"
        "cvt.rn.f16x2.e4m3x2 %1, h1;\n"
        "}"
        : "=r"(out[0]), "=r"(out[1])
        : "r"(w));
}

__device__ __forceinline__ float h_lo(uint32_t w) { return __half2float(__ushort_as_half((unsigned short)(w & 0xFFFF))); }
__device__ __forceinline__ float h_hi(uint32_t w) { return __half2float(__ushort_as_half((unsigned short)(w >> 16))); }

__device__ __forceinline__ float e4m3_to_f32(uint8_t v) { return h_lo(e4m3x2_to_f16x2(v)); }

}  // namespace csa
