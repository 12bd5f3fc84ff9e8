// mxfp8.cuh -- device helpers for MXFP8 (OCP Microscaling v1.0): E8M0 block
// scale from the block's largest magnitude, E4M3 conversion with
// round-to-nearest-even and saturation to +-448.
#pragma once

#include <cstdint>

namespace moe {

// Scale of a 32-element block: s = floor(log2(amax)) - 8 clamped to
// [-127, 127] (-127 for an all-zero block).  floor(log2(amax)) is read from
// the fp32 exponent field (a subnormal amax gives an s below -127, which
// clamps).  Returns the biased byte s + 127 and sets *inv = 2^-s exactly.
__device__ __forceinline__ uint8_t mxfp8_block_scale(float amax, float* inv) {
    int s;
    if (amax == 0.0f) {
        s = -127;
    } else {
        const int e = (int)((__float_as_uint(amax) >> 23) & 0xFFu) - 127;
        s = e - 8;
        s = s < -127 ? -127 : (s > 127 ? 127 : s);
    }
    // finite inputs give s <= 120, so 127 - s >= 7 is a normal exponent field
    *inv = __uint_as_float((uint32_t)(127 - s) << 23);
    return (uint8_t)(s + 127);
}

// Two fp32 values to two E4M3 codes: `lo` in the low byte, `hi` in the high
// byte (round to nearest even, out-of-range magnitudes saturate to 448).
__device__ __forceinline__ uint32_t e4m3x2(float hi, float lo) {
    uint16_t r;
    asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(hi), "f"(lo));
    return (uint32_t)r;
}

__device__ __forceinline__ float bf16lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

// Quantise 8 bf16 values held by one lane; a 32-element block is spread
// over 4 neighbouring lanes (lane & ~3 .. lane | 3), which must all call
// this together.  Returns the 8 codes (byte i = element i).
__device__ __forceinline__ uint2 mxfp8_quantize_8(uint4 v, uint8_t* sbyte) {
    float f[8] = {bf16lo(v.x), bf16hi(v.x), bf16lo(v.y), bf16hi(v.y),
                  bf16lo(v.z), bf16hi(v.z), bf16lo(v.w), bf16hi(v.w)};
    float a = 0.0f;
#pragma unroll
    for (int i = 0; i < 8; ++i) a = fmaxf(a, fabsf(f[i]));
    a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, 1));
    a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, 2));
    float inv;
    *sbyte = mxfp8_block_scale(a, &inv);
    const uint32_t c01 = e4m3x2(f[1] * inv, f[0] * inv);
    const uint32_t c23 = e4m3x2(f[3] * inv, f[2] * inv);
    const uint32_t c45 = e4m3x2(f[5] * inv, f[4] * inv);
    const uint32_t c67 = e4m3x2(f[7] * inv, f[6] * inv);
    return make_uint2(c01 | (c23 << 16), c45 | (c67 << 16));
}

}  // namespace moe
