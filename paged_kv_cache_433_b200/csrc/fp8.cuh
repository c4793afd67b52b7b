// E4M3 (8-bit float: 1 sign, 4 exponent bits with bias 7, 3 mantissa bits,
// largest finite 448) helpers for the FP8 K/V cache: hardware conversions
// between E4M3 pairs and f16 / fp32 pairs, byte permutes, 64-bit shared loads.
#pragma once

#include <cstdint>

namespace kvp {

// Four E4M3 codes (bytes 0-3 of w) -> two f16x2 (lo: bytes 0-1, hi: bytes
// 2-3; the lower code of a pair in the lower half). Exact: every E4M3 value
// is an f16 value. The 32-bit register is split into halves without an
// instruction.
__device__ __forceinline__ void e4m3x4_to_f16x2x2(uint32_t w, uint32_t& lo, uint32_t& hi) {
    asm("{\n\t.reg .b16 a, b;\n\tmov.b32 {a, b}, %2;\n\tcvt.rn.f16x2.e4m3x2 %0, a;\n\tcvt.rn.f16x2.e4m3x2 %1, b;\n\t}"
        : "=r"(lo), "=r"(hi)
        : "r"(w));
}

// Two fp32 values -> two E4M3 codes (lo in bits 0-7, hi in bits 8-15):
// round to nearest even, saturating at +-448; NaN stays NaN.
__device__ __forceinline__ uint32_t f32x2_to_e4m3x2(float lo, float hi) {
    uint32_t r;
    asm("{\n\t.reg .b16 t;\n\tcvt.rn.satfinite.e4m3x2.f32 t, %1, %2;\n\tcvt.u32.u16 %0, t;\n\t}"
        : "=r"(r)
        : "f"(hi), "f"(lo));
    return r;
}

// Bytes of {b, a} (a = bytes 0-3, b = bytes 4-7) picked by the selector's nibbles.
__device__ __forceinline__ uint32_t byte_perm(uint32_t a, uint32_t b, uint32_t sel) {
    uint32_t r;
    asm("prmt.b32 %0, %1, %2, %3;" : "=r"(r) : "r"(a), "r"(b), "r"(sel));
    return r;
}

// Two fp32 values -> f16x2 (lo in the low half), round to nearest even,
// saturating at +-65504 instead of overflowing to infinity.
__device__ __forceinline__ uint32_t pack2_satfinite_f16(float lo, float hi) {
    uint32_t r;
    asm("cvt.rn.satfinite.f16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
    return r;
}

__device__ __forceinline__ uint2 lds64(uint32_t addr) {
    uint2 v;
    asm volatile("ld.shared.v2.u32 {%0, %1}, [%2];" : "=r"(v.x), "=r"(v.y) : "r"(addr));
    return v;
}

}  // namespace kvp
