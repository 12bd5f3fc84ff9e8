// prepare.cu -- rebuild the kernel-layout weight buffer in place (Megatron-LM
// PR #7830, "1. Mega backend for generation": the refit calls
// refresh_mega_weights(), which rewrites the kernel's own copy of the
// weights; no allocation, no teardown).
//
// bf16 layout: every weight matrix is stored as blocks of 32 KB, one per
// (expert, block of 128 weight rows, K stage of 128 elements), each block
// [2 atoms][128 rows][64 elements] -- exactly the GEMM's shared-memory image
// of one operand stage before swizzling, so one TMA box reads 32 KB of
// contiguous memory:
//   W1  rows of an expert: 2fp, in the order (per block of 64 f, per group
//       of 16 f) the 16 gate rows, then the 16 up rows of the same f; K = hp
//       (squared-ReLU experts: the one projection's rows in f order, padded
//       to a multiple of 256)
//   W2  rows of an expert: hr (H padded to 128); K = fp
// with hp, fp = H, F rounded up to 128.  Padding (K past H or F, rows of
// f >= F, rows c >= H) is zero.  A gate/up weight tile is two consecutive
// row blocks, one per CTA of a pair; a group of 32 rows is one 32-lane TMEM
// quarter, so gate and up of one f land in the same warp's reach.
#include "moe_internal.cuh"
#include "mxfp8.cuh"

namespace moe {
namespace {

__global__ void __launch_bounds__(256) prepare_bf16_kernel(const uint4* __restrict__ wg, const uint4* __restrict__ wu,
                                                           const uint4* __restrict__ wd, uint4* __restrict__ w1,
                                                           uint4* __restrict__ w2, int E, int F, int H, int hp, int fp,
                                                           int hr, int w1r, int relu2) {
    // one thread per 16-byte chunk of the destination: block, atom, row, 8-element chunk
    constexpr long long kBlockChunks = 2 * 128 * 8;  // 32 KB
    const int kb1 = hp / 128, kb2 = fp / 128;
    const int rb1 = w1r / 128, rb2 = hr / 128;  // row blocks per expert
    const long long n1 = (long long)E * rb1 * kb1 * kBlockChunks;
    const long long n2 = (long long)E * rb2 * kb2 * kBlockChunks;
    const long long stride = (long long)gridDim.x * blockDim.x;
    for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < n1 + n2; i += stride) {
        const bool first = i < n1;
        const long long j = first ? i : i - n1;
        const long long blk = j / kBlockChunks;
        const int w = (int)(j - blk * kBlockChunks);
        const int atom = w >> 10, r = (w >> 3) & 127, c8 = w & 7;
        const int kbs = first ? kb1 : kb2, rbs = first ? rb1 : rb2;
        const int kb = (int)(blk % kbs);
        const long long erb = blk / kbs;
        const int rb = (int)(erb % rbs);
        const long long e = erb / rbs;
        const int k = kb * 128 + atom * 64 + c8 * 8;  // first K element of the chunk
        const int rem = rb * 128 + r;                 // weight row within the expert
        uint4 v = make_uint4(0u, 0u, 0u, 0u);
        if (first) {
            // squared-ReLU experts: row = f; SwiGLU: the 16-row gate / up interleave
            const int g = relu2 ? 0 : (rem >> 4) & 1;
            const int f = relu2 ? rem : (rem >> 7) * 64 + ((rem >> 5) & 3) * 16 + (rem & 15);
            if (f < F && k < H) v = __ldg((g ? wu : wg) + ((e * F + f) * H + k) / 8);
            w1[i] = v;
        } else {
            if (rem < H && k < F) v = __ldg(wd + ((e * H + rem) * F + k) / 8);
            w2[j] = v;
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
        (int)p->hp, (int)p->fp, (int)p->hr, (int)p->w1r, (p->d.flags & MOE_FLAG_SQUARED_RELU) ? 1 : 0);
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
                                                            int fp, int nt1, int ks1, int nt2, int ks2, int relu2) {
    const long long rows1 = (long long)E * (relu2 ? 1 : 2) * F;
    const long long rows2 = (long long)E * H;
    for (long long row = blockIdx.x; row < rows1 + rows2; row += gridDim.x) {
        const uint4* src;
        uint2* dst;
        uint8_t* sf_tile;  // the K-stage-0 scale block of this row's N tile
        int len, trow;
        if (row < rows1) {
            const int per_e = relu2 ? F : 2 * F;
            const long long e = row / per_e;
            const int rem = (int)(row - e * per_e);
            const int gu = rem / F, f = rem - gu * F;
            src = (gu ? wu : wg) + ((size_t)e * F + f) * (H / 8);
            // SwiGLU: 64 f per 128-row tile, gate / up interleaved in groups of 16;
            // squared-ReLU experts: 128 f per tile in f order
            const int tile = relu2 ? f / 128 : f / kG1BN8;
            trow = relu2 ? f % 128 : ((f % kG1BN8) >> 4) * 32 + gu * 16 + (f & 15);
            dst = w1q + ((size_t)(e * nt1 + tile) * 128 + trow) * (hp / 8);
            len = H;
            sf_tile = w1s + ((size_t)e * nt1 + tile) * ks1 * kSfBlock;
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
        base + p->wb.w2s, E, F, H, (int)p->hp, (int)p->fp, p->nt1, p->ks1, p->nt2, p->ks2,
        (p->d.flags & MOE_FLAG_SQUARED_RELU) ? 1 : 0);
    return cudaGetLastError();
}

}  // namespace moe
