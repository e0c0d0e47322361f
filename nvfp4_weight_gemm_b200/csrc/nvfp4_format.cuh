// nvfp4_format.cuh -- device-side element decoders and encoders of the NVFP4 weight format.
//
// Format (TandemLLM docs v0.12.0, "What TandemLLM is", section 1.2: four bits a weight,
// one scale per 16 weights): E2M1 codes two per byte (low nibble = even k), one E4M3 scale
// per 16-element K block, one FP32 tensor scale that multiplies.
#pragma once
#include <cstdint>
#include <cuda_fp16.h>

namespace tl {

// Two E2M1 codes (one byte: low nibble first) -> half2 {low, high}, exact (hardware convert).
__device__ __forceinline__ __half2 e2m1x2_to_half2(uint32_t byte) {
    uint32_t out;
    asm("{\n\t.reg .b8 b;\n\tcvt.u8.u32 b, %1;\n\tcvt.rn.f16x2.e2m1x2 %0, b;\n\t}" : "=r"(out) : "r"(byte));
    return *reinterpret_cast<__half2*>(&out);
}

// Two E4M3 bytes (low byte first) -> half2, exact (every finite E4M3 value is an f16 normal).
__device__ __forceinline__ __half2 e4m3x2_to_half2(uint32_t two_bytes) {
    uint32_t out;
    asm("{\n\t.reg .b16 h;\n\tcvt.u16.u32 h, %1;\n\tcvt.rn.f16x2.e4m3x2 %0, h;\n\t}" : "=r"(out) : "r"(two_bytes));
    return *reinterpret_cast<__half2*>(&out);
}

__device__ __forceinline__ float e4m3_to_float(uint32_t byte) {
    return __low2float(e4m3x2_to_half2(byte & 0xFFu));
}

// Round t >= 0 to E4M3 (nearest, ties to even mantissa), saturating at 448 (0x7E).
// Computed from the binary exponent of t: subnormal step 2^-9 below 2^-6, else 3 mantissa bits.
__device__ __forceinline__ uint32_t e4m3_encode_rne_sat(double t) {
    if (!(t < 448.0)) return 0x7Eu;
    if (t < 0.015625) {                          // below 2^-6: multiples of 2^-9
        return (uint32_t)__double2int_rn(t * 512.0);  // 8 -> 0x08 = 2^-6, the first normal
    }
    int ex;
    double f = frexp(t, &ex);                    // t = f * 2^ex, f in [0.5, 1)
    int e = ex - 1 + 7;                          // biased exponent of t in [1, 15]
    int m = __double2int_rn((2.0 * f - 1.0) * 8.0);
    if (m == 8) { m = 0; e += 1; }
    if (e > 15 || (e == 15 && m == 7)) return 0x7Eu;
    return (uint32_t)((e << 3) | m);
}

// Round q to the E2M1 grid (nearest, ties to even mantissa; |q| clamped to 6; 0 -> +0).
__device__ __forceinline__ uint32_t e2m1_encode_rne(double q) {
    double a = fabs(q);
    uint32_t c;
    if (a <= 0.25) c = 0;
    else if (a < 0.75) c = 1;
    else if (a <= 1.25) c = 2;
    else if (a < 1.75) c = 3;
    else if (a <= 2.5) c = 4;
    else if (a < 3.5) c = 5;
    else if (a <= 5.0) c = 6;
    else c = 7;
    if (c != 0 && q < 0.0) c |= 8u;
    return c;
}

}  // namespace tl
