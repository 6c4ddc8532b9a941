// The OCP Microscaling (MX) v1.0 MXFP4 element and scale formats, for the
// kernels that read MXFP4 expert weights ("Mixture of Experts (MoEs) in
// Transformers", section From Dense to Sparse: gpt-oss ships its experts in
// mxfp4).  An element is FP4 E2M1 (sign, two exponent bits with bias 1, one
// mantissa bit: 0, 0.5, 1, 1.5, 2, 3, 4, 6); 32 consecutive elements along the
// reduction dimension share one E8M0 scale byte s standing for 2^(s - 127),
// s = 255 meaning NaN.  Storage: two codes per byte, the element with the
// lower index in the low nibble; a row's 16-byte blocks are contiguous.
#pragma once
#include <cstdint>

namespace moe {

// Four bytes of E2M1 pairs -> four f16x2 values (byte j -> elements 2j in
// the low half, 2j+1 in the high half); every E2M1 value is exact in f16.
__device__ __forceinline__ void e2m1x8_to_f16x2(uint32_t w, uint32_t (&o)[4]) {
    asm("{\n\t.reg .b8 b0, b1, b2, b3;\n\t"
        "mov.b32 {b0, b1, b2, b3}, %4;\n\t"
        "cvt.rn.f16x2.e2m1x2 %0, b0;\n\t"
        "cvt.rn.f16x2.e2m1x2 %1, b1;\n\t"
        "cvt.rn.f16x2.e2m1x2 %2, b2;\n\t"
        "cvt.rn.f16x2.e2m1x2 %3, b3;\n\t}"
        : "=r"(o[0]), "=r"(o[1]), "=r"(o[2]), "=r"(o[3])
        : "r"(w));
}

// 2^(s - 127) for an E8M0 byte: s = 0 is the subnormal 2^-127, s = 255 NaN.
__device__ __forceinline__ float e8m0_value(uint32_t s) {
    if (s == 255u) return __int_as_float(0x7fc00000);
    return s == 0u ? __int_as_float(0x00400000) : __int_as_float((int)(s << 23));
}

}  // namespace moe
