// Exact conversions of the NVFP4 weight format's narrow types (sm_100a PTX).
//   e2m1: 1 sign, 2 exponent (bias 1), 1 mantissa bit: 0, 0.5, 1, 1.5, 2, 3, 4, 6.
//   e4m3: 1 sign, 4 exponent (bias 7), 3 mantissa bits, max 448.
// Both convert exactly to f16, and an e2m1 * e4m3 product (at most six
// significant bits, magnitude in [2^-10, 2688]) is exact in f16 and in bf16.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <stdint.h>

#include "common.cuh"

namespace moe {

// Four bytes of e2m1 codes (two per byte, the low nibble the lower k) -> four
// f16 pairs: (k0 k1), (k2 k3), (k4 k5), (k6 k7).
MOE_DEV void e2m1x8_to_f16(uint32_t w, uint32_t (&p)[4]) {
    asm("{\n\t.reg .b8 b0, b1, b2, b3;\n\t"
        "mov.b32 {b0, b1, b2, b3}, %4;\n\t"
        "cvt.rn.f16x2.e2m1x2 %0, b0;\n\t"
        "cvt.rn.f16x2.e2m1x2 %1, b1;\n\t"
        "cvt.rn.f16x2.e2m1x2 %2, b2;\n\t"
        "cvt.rn.f16x2.e2m1x2 %3, b3;\n\t}"
        : "=r"(p[0]), "=r"(p[1]), "=r"(p[2]), "=r"(p[3])
        : "r"(w));
}

// Two e4m3 bytes (bits 0-7 and 8-15 of v) -> an f16 pair.
MOE_DEV uint32_t e4m3x2_to_f16x2(uint32_t v) {
    uint32_t r;
    asm("{\n\t.reg .b16 t;\n\tcvt.u16.u32 t, %1;\n\tcvt.rn.f16x2.e4m3x2 %0, t;\n\t}" : "=r"(r) : "r"(v));
    return r;
}

MOE_DEV uint32_t hmul2_u32(uint32_t a, uint32_t b) {
    const __half2 r = __hmul2(*reinterpret_cast<const __half2*>(&a), *reinterpret_cast<const __half2*>(&b));
    return *reinterpret_cast<const uint32_t*>(&r);
}

// An f16 pair holding values exact in bf16 -> the same values as a bf16 pair.
MOE_DEV uint32_t f16x2_to_bf16x2(uint32_t a) {
    const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&a));
    const __nv_bfloat162 b = __floats2bfloat162_rn(f.x, f.y);
    return *reinterpret_cast<const uint32_t*>(&b);
}

}  // namespace moe
