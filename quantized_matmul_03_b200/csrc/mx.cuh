// mx.cuh -- device helpers for the microscaled modes (Emily.QuantizedWeight,
// section Microscaled modes): mxfp4 (group 32, E2M1 elements, E8M0 scale),
// mxfp8 (group 32, E4M3 elements, E8M0 scale), nvfp4 (group 16, E2M1
// elements, E4M3 scale); scales are one byte per group, there are no biases.
// Element and scale encodings are those of the OCP Microscaling Formats (MX)
// v1.0 definitions; conversions use the hardware's nearest-even, saturating
// cvt instructions.
#pragma once

#include <cuda_fp16.h>
#include <stdint.h>

#include "qmm_internal.cuh"

namespace qmm {
namespace mxf {

// 8 floats -> 8 E2M1 codes, v[0] in the lowest nibble.
__device__ __forceinline__ uint32_t e2m1x8(const float *v) {
    uint32_t r;
    asm("{\n\t.reg .b8 b0, b1, b2, b3;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b0, %2, %1;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b1, %4, %3;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b2, %6, %5;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b3, %8, %7;\n\t"
        "mov.b32 %0, {b0, b1, b2, b3};\n\t}"
        : "=r"(r)
        : "f"(v[0]), "f"(v[1]), "f"(v[2]), "f"(v[3]), "f"(v[4]), "f"(v[5]), "f"(v[6]), "f"(v[7]));
    return r;
}

// 4 floats -> 4 E4M3 codes, v[0] in the lowest byte.
__device__ __forceinline__ uint32_t e4m3x4(const float *v) {
    uint32_t r;
    asm("{\n\t.reg .b16 h0, h1;\n\t"
        "cvt.rn.satfinite.e4m3x2.f32 h0, %2, %1;\n\t"
        "cvt.rn.satfinite.e4m3x2.f32 h1, %4, %3;\n\t"
        "mov.b32 %0, {h0, h1};\n\t}"
        : "=r"(r)
        : "f"(v[0]), "f"(v[1]), "f"(v[2]), "f"(v[3]));
    return r;
}

// Two E2M1 codes (byte i of w: low nibble first) -> f16x2 (exact).
__device__ __forceinline__ uint32_t e2m1x2_to_h2(uint32_t w, int i) {
    uint32_t r;
    const uint16_t b = (uint16_t)((w >> (8 * i)) & 0xFFu);
    asm("{\n\t.reg .b8 lo, hi;\n\tmov.b16 {lo, hi}, %1;\n\tcvt.rn.f16x2.e2m1x2 %0, lo;\n\t}"
        : "=r"(r)
        : "h"(b));
    return r;
}

// Two E4M3 codes (bytes 2i, 2i+1 of w) -> f16x2 (exact).
__device__ __forceinline__ uint32_t e4m3x2_to_h2(uint32_t w, int i) {
    uint32_t r;
    const uint16_t h = (uint16_t)((w >> (16 * i)) & 0xFFFFu);
    asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(r) : "h"(h));
    return r;
}

// Value of a scale byte: E8M0 (2^(s - 127); 0xFF is NaN) or E4M3 (nvfp4).
template <int MODE>
__device__ __forceinline__ float scale_value(uint32_t s) {
    if constexpr (MODE == QMM_MODE_NVFP4) {
        const uint32_t h = e4m3x2_to_h2(s & 0xFFu, 0);
        return __half2float(__ushort_as_half((unsigned short)(h & 0xFFFFu)));
    } else {
        if (s == 0xFFu) return __uint_as_float(0x7FC00000u);
        return s == 0 ? __uint_as_float(0x00400000u) : __uint_as_float(s << 23);
    }
}

// The 32/bits element values of one packed word (mxfp4/nvfp4: 8, mxfp8: 4)
// as floats, exact.
template <int MODE>
__device__ __forceinline__ void elements(uint32_t w, float *out) {
    if constexpr (MODE == QMM_MODE_MXFP8) {
#pragma unroll
        for (int i = 0; i < 2; ++i) {
            const uint32_t h = e4m3x2_to_h2(w, i);
            const float2 f = __half22float2(*reinterpret_cast<const __half2 *>(&h));
            out[2 * i] = f.x;
            out[2 * i + 1] = f.y;
        }
    } else {
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const uint32_t h = e2m1x2_to_h2(w, i);
            const float2 f = __half22float2(*reinterpret_cast<const __half2 *>(&h));
            out[2 * i] = f.x;
            out[2 * i + 1] = f.y;
        }
    }
}

}  // namespace mxf
}  // namespace qmm
