// quant.cu -- MXFP8 quantisation of bf16 rows (E4M3 elements, one E8M0
// scale per 32 elements along the row).
//
// Megatron-LM PR #7830, "1. Mega backend for generation" (mxfp8 weights
// quantised per block of 32); cudnn-frontend PR #448 review (MXFP8 uses a
// 32-element block).  Scale rule of the OCP Microscaling spec v1.0:
// X = 2^(floor(log2(amax)) - 8), 8 being the largest exponent of E4M3;
// elements are value / X rounded to nearest-even on the E4M3 grid,
// saturating at +-448 (the hardware conversion's satfinite mode).
#include "moe_internal.cuh"
#include "mxfp8.cuh"

namespace moe {
namespace {

// One warp walks a row in chunks of 256 elements: lane l holds elements
// [8l, 8l+8) of the chunk, so a 32-element block spans 4 neighbouring lanes.
__global__ void __launch_bounds__(256) quantize_rows_kernel(const uint4* __restrict__ in, long long rows, int cols,
                                                            long long ld_in_chunks, const int* __restrict__ live,
                                                            uint2* __restrict__ q, uint8_t* __restrict__ scales) {
    long long n = rows;
    if (live != nullptr) {
        const long long l = (long long)__ldg(live);
        n = l < 0 ? 0 : (l < rows ? l : rows);
    }
    const int lane = threadIdx.x & 31;
    const int wpb = blockDim.x >> 5;
    const int chunks = cols / 8;
    for (long long r = (long long)blockIdx.x * wpb + (threadIdx.x >> 5); r < n; r += (long long)gridDim.x * wpb) {
        const uint4* src = in + r * ld_in_chunks;
        for (int c = lane; c < ((chunks + 31) & ~31); c += 32) {
            const bool active = c < chunks;  // cols % 32 == 0: whole 4-lane groups are active together
            uint4 v = active ? __ldg(src + c) : make_uint4(0, 0, 0, 0);
            uint8_t sbyte;
            const uint2 codes = mxfp8_quantize_8(v, &sbyte);
            if (active) {
                q[r * chunks + c] = codes;
                if ((lane & 3) == 0) scales[r * (cols / 32) + c / 4] = sbyte;
            }
        }
    }
}

}  // namespace

cudaError_t launch_quantize_rows(const __nv_bfloat16* in, long long rows, int cols, long long ld_in, uint8_t* q,
                                 uint8_t* scales, const int* live_rows, cudaStream_t s) {
    long long blocks = (rows + 7) / 8;
    const long long cap = (long long)num_sms() * 8;
    if (blocks > cap) blocks = cap;
    if (blocks < 1) blocks = 1;
    quantize_rows_kernel<<<(unsigned)blocks, 256, 0, s>>>(reinterpret_cast<const uint4*>(in), rows, cols, ld_in / 8,
                                                          live_rows, reinterpret_cast<uint2*>(q), scales);
    return cudaGetLastError();
}

}  // namespace moe
