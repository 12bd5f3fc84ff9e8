// nvfp4.cuh -- device helpers for NVFP4 as the per-token recipe uses it
// (Megatron-LM PR #7798, "Per-token NVFP4": TE's NVFP4BlockScaling with
// row-scaled activations, 1-D blocks, no Hadamard transform, no stochastic
// rounding).  E2M1 elements, one E4M3 scale per 16 elements along K, and an
// fp32 second-level scale g per activation row (per matrix for weights):
//   g = amax / (6 * 448)            (1 when that is 0)
//   s = E4M3((amax_16 / g) / 6)     round to nearest even, saturating at 448
//   d = value(s) * g;  code = E2M1(v / d)   (signed zero when d is 0)
// every step an fp32 operation in that order; codes two per byte, element 2i
// in the low nibble.
#pragma once

#include <cstdint>

#include "mxfp8.cuh"

namespace moe {

__device__ __forceinline__ float nvfp4_global(float amax) {
    const float g = __fdiv_rn(amax, 2688.0f);
    return (amax > 0.0f && g > 0.0f) ? g : 1.0f;
}

// Value of a non-negative E4M3 code (the format definition: bias 7, subnormal
// step 2^-9; the codes here come from a saturating conversion, never NaN).
__device__ __forceinline__ float e4m3_value(uint32_t c) {
    const uint32_t e = (c >> 3) & 15u, m = c & 7u;
    return e == 0 ? (float)m * 0.001953125f : __uint_as_float(((e + 120u) << 23) | (m << 20));
}

// Block scale byte of a 16-element block with largest magnitude amax under
// the second-level scale g; *d = value(s) * g, the block's divisor.
__device__ __forceinline__ uint8_t nvfp4_block_scale(float amax, float g, float* d) {
    const float sf = __fdiv_rn(__fdiv_rn(amax, g), 6.0f);
    const uint8_t sb = (uint8_t)(e4m3x2(0.0f, sf) & 0xFFu);
    *d = __fmul_rn(e4m3_value(sb), g);
    return sb;
}

// Two fp32 values to one byte of E2M1 codes, `lo` in bits 0-3 and `hi` in
// bits 4-7 (round to nearest even, magnitudes past 6 saturate).
__device__ __forceinline__ uint32_t e2m1x2(float hi, float lo) {
    uint32_t r;
    asm("{\n\t.reg .b8 t;\n\tcvt.rn.satfinite.e2m1x2.f32 t, %1, %2;\n\tcvt.u32.u8 %0, t;\n\t}" : "=r"(r)
        : "f"(hi), "f"(lo));
    return r;
}

// E2M1 code pair of two values under divisor d (the signed zero codes when d is 0).
__device__ __forceinline__ uint32_t nvfp4_pair(float v0, float v1, float d) {
    if (d == 0.0f) return (signbit(v0) ? 8u : 0u) | (signbit(v1) ? 0x80u : 0u);
    return e2m1x2(__fdiv_rn(v1, d), __fdiv_rn(v0, d));
}

// Codes of 8 consecutive values of one block (4 bytes, element 0 in the low nibble of byte 0).
__device__ __forceinline__ uint32_t nvfp4_codes_8(const float (&v)[8], float d) {
    return nvfp4_pair(v[0], v[1], d) | (nvfp4_pair(v[2], v[3], d) << 8) | (nvfp4_pair(v[4], v[5], d) << 16) |
           (nvfp4_pair(v[6], v[7], d) << 24);
}

// Byte offset of the block scale of (row within a 128-row tile, 16-element
// block within a 64-element MMA step) inside one 512-byte scale block: the
// layout of MXFP8's scale blocks with the MMA step's 4 blocks in place of
// 4 k-groups (one tcgen05.cp moves it to 4 TMEM columns for one MMA).
__host__ __device__ __forceinline__ uint32_t nvfp4_sf_offset(int row, int blk) {
    return (uint32_t)((row & 31) * 16 + ((row >> 5) & 3) * 4 + blk);
}

}  // namespace moe
