// prepare.cu -- rebuild the kernel-layout weight buffer in place (Megatron-LM
// PR #7830, "1. Mega backend for generation": the refit calls
// refresh_mega_weights(), which rewrites the kernel's own copy of the
// weights; no allocation, no teardown).
//
// bf16 layout:  W1 [E][fp/64][4][2][16][hp]  (per block of 64 f, per group of
//                                           16 f: the 16 gate rows, then the
//                                           16 up rows of the same f),
//               W2 [E][H][fp]               (down projection),
// with the K pitches hp, fp = H, F rounded up to 128 and the padding zero
// (rows of f >= F too).  A gate/up weight tile is two consecutive blocks, one
// per CTA of a pair; a group of 32 rows is one 32-lane TMEM quarter, so gate
// and up of one f land in the same warp's reach.
#include "moe_internal.cuh"
#include "mxfp8.cuh"

namespace moe {
namespace {

__global__ void __launch_bounds__(256) prepare_bf16_kernel(const uint4* __restrict__ wg, const uint4* __restrict__ wu,
                                                           const uint4* __restrict__ wd, uint4* __restrict__ w1,
                                                           uint4* __restrict__ w2, int E, int F, int H, int hp, int fp) {
    // 16-byte chunks of the destination; rows are padded with zeros to hp / fp
    const long long c1 = hp / 8, c2 = fp / 8;
    const long long rows1 = 2ll * fp;  // W1 rows per expert
    const long long n1 = (long long)E * rows1 * c1;
    const long long n2 = (long long)E * H * c2;
    const long long stride = (long long)gridDim.x * blockDim.x;
    for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < n1 + n2; i += stride) {
        if (i < n1) {
            const long long row = i / c1;  // e * 2fp + block * 128 + group * 32 + g * 16 + f % 16
            const int c = (int)(i - row * c1);
            const long long e = row / rows1;
            const int rem = (int)(row - e * rows1);
            const int g = (rem >> 4) & 1;
            const int f = (rem >> 7) * 64 + ((rem >> 5) & 3) * 16 + (rem & 15);
            uint4 v = make_uint4(0u, 0u, 0u, 0u);
            if (f < F && c * 8 < H) v = __ldg((g ? wu : wg) + (e * F + f) * (H / 8) + c);
            w1[i] = v;
        } else {
            const long long j = i - n1;
            const long long row = j / c2;  // e * H + h
            const int c = (int)(j - row * c2);
            w2[j] = c * 8 < F ? __ldg(wd + row * (F / 8) + c) : make_uint4(0u, 0u, 0u, 0u);
        }
    }
}

}  // namespace

cudaError_t launch_prepare_bf16(const moe_plan* p, const __nv_bfloat16* wg, const __nv_bfloat16* wu,
                                const __nv_bfloat16* wd, void* buf, cudaStream_t s) {
    const long long H = p->d.hidden, F = p->d.ffn, E = p->d.num_experts;
    uint8_t* base = static_cast<uint8_t*>(buf);
    prepare_bf16_kernel<<<num_sms() * 8, 256, 0, s>>>(
        reinterpret_cast<const uint4*>(wg), reinterpret_cast<const uint4*>(wu), reinterpret_cast<const uint4*>(wd),
        reinterpret_cast<uint4*>(base + p->wb.w1), reinterpret_cast<uint4*>(base + p->wb.w2), (int)E, (int)F, (int)H,
        (int)p->hp, (int)p->fp);
    return cudaGetLastError();
}

}  // namespace moe

namespace moe {
namespace {

// MXFP8 weights: one 128-thread block per weight row (grid-stride), blocks of
// 32 along the row (the GEMM's K).  Codes, K pitches hp, fp = H, F rounded up
// to 128 with zero padding:
//   W1 [E][fp/64][4][2][16][hp]  (as the bf16 W1: per 16 f the gate rows,
//                                 then the up rows; 64 f per weight tile;
//                                 rows of f >= F zero)
//   W2 [E][H][fp]
// and scale bytes in the GEMMs' weight scale blocks ([tile][K stage][512 B]):
//   gate/up row (e, g/u, f): tile f / 64, tile row (f % 64 / 16) * 32 + g/u * 16 + f % 16
//   down row (e, c):         tile c / 128, tile row c % 128
__global__ void __launch_bounds__(128) prepare_mxfp8_kernel(const uint4* __restrict__ wg, const uint4* __restrict__ wu,
                                                            const uint4* __restrict__ wd, uint2* __restrict__ w1q,
                                                            uint8_t* __restrict__ w1s, uint2* __restrict__ w2q,
                                                            uint8_t* __restrict__ w2s, int E, int F, int H, int hp,
                                                            int fp, int nt1, int ks1, int nt2, int ks2) {
    const long long rows1 = (long long)E * 2 * F;
    const long long rows2 = (long long)E * H;
    for (long long row = blockIdx.x; row < rows1 + rows2; row += gridDim.x) {
        const uint4* src;
        uint2* dst;
        uint8_t* sf_tile;  // the K-stage-0 scale block of this row's N tile
        int len, trow;
        if (row < rows1) {
            const long long e = row / (2 * F);
            const int rem = (int)(row - e * 2 * F);
            const int gu = rem / F, f = rem - gu * F;
            src = (gu ? wu : wg) + ((size_t)e * F + f) * (H / 8);
            trow = ((f % kG1BN8) >> 4) * 32 + gu * 16 + (f & 15);
            dst = w1q + ((size_t)(e * nt1 + f / kG1BN8) * 128 + trow) * (hp / 8);
            len = H;
            sf_tile = w1s + ((size_t)e * nt1 + f / kG1BN8) * ks1 * kSfBlock;
        } else {
            const long long r2 = row - rows1;
            const long long e = r2 / H;
            const int c = (int)(r2 - e * H);
            src = wd + (size_t)r2 * (F / 8);
            dst = w2q + (size_t)r2 * (fp / 8);
            len = F;
            trow = c % kG2BN8;
            sf_tile = w2s + ((size_t)e * nt2 + c / kG2BN8) * ks2 * kSfBlock;
        }
        const int chunks = len / 8;
        for (int c0 = 0; c0 < chunks; c0 += blockDim.x) {
            const int c = c0 + threadIdx.x;
            const bool active = c < chunks;
            const uint4 v = active ? __ldg(src + c) : make_uint4(0u, 0u, 0u, 0u);
            uint8_t sb;
            const uint2 codes = mxfp8_quantize_8(v, &sb);
            if (active) {
                dst[c] = codes;
                const int g = c >> 2;
                if ((c & 3) == 0) sf_tile[(size_t)(g / 4) * kSfBlock + sf_block_offset(trow, g % 4)] = sb;
            }
        }
    }
}

}  // namespace

cudaError_t launch_prepare_mxfp8(const moe_plan* p, const __nv_bfloat16* wg, const __nv_bfloat16* wu,
                                 const __nv_bfloat16* wd, void* buf, cudaStream_t s) {
    uint8_t* base = static_cast<uint8_t*>(buf);
    const int E = p->d.num_experts, F = p->d.ffn, H = p->d.hidden;
    // padding rows and k-groups of the scale blocks hold byte 0 (scale 2^-127); the K padding
    // of the code rows and the W1 rows of f >= F hold code 0
    cudaError_t err = cudaMemsetAsync(base + p->wb.w1s, 0, p->wb.w2 - p->wb.w1s, s);
    if (err != cudaSuccess) return err;
    if (H != p->hp || F != p->fp) err = cudaMemsetAsync(base + p->wb.w1, 0, p->wb.w1s - p->wb.w1, s);
    if (err != cudaSuccess) return err;
    if (F != p->fp) err = cudaMemsetAsync(base + p->wb.w2, 0, p->wb.w2s - p->wb.w2, s);
    if (err != cudaSuccess) return err;
    err = cudaMemsetAsync(base + p->wb.w2s, 0, p->wb.total - p->wb.w2s, s);
    if (err != cudaSuccess) return err;
    prepare_mxfp8_kernel<<<num_sms() * 16, 128, 0, s>>>(
        reinterpret_cast<const uint4*>(wg), reinterpret_cast<const uint4*>(wu), reinterpret_cast<const uint4*>(wd),
        reinterpret_cast<uint2*>(base + p->wb.w1), base + p->wb.w1s, reinterpret_cast<uint2*>(base + p->wb.w2),
        base + p->wb.w2s, E, F, H, (int)p->hp, (int)p->fp, p->nt1, p->ks1, p->nt2, p->ks2);
    return cudaGetLastError();
}

}  // namespace moe
