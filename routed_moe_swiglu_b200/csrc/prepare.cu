// prepare.cu -- rebuild the kernel-layout weight buffer in place (Megatron-LM
// PR #7830, "1. Mega backend for generation": the refit calls
// refresh_mega_weights(), which rewrites the kernel's own copy of the
// weights; no allocation, no teardown).
//
// bf16 layout:  W1 [E][2][F][H]  (gate rows, then up rows of each expert),
//               W2 [E][H][F]     (down projection).
// A gate/up tile loads the same 128 f rows from W1[e][0] and W1[e][1] into
// one 256-row B operand, so gate and up of one f meet in one accumulator row.
#include "moe_internal.cuh"

namespace moe {
namespace {

__global__ void __launch_bounds__(256) prepare_bf16_kernel(const uint4* __restrict__ wg, const uint4* __restrict__ wu,
                                                           const uint4* __restrict__ wd, uint4* __restrict__ w1,
                                                           uint4* __restrict__ w2, long long fh_chunks,
                                                           long long hf_chunks, int E) {
    const long long n1 = (long long)E * 2 * fh_chunks;
    const long long n2 = (long long)E * hf_chunks;
    const long long stride = (long long)gridDim.x * blockDim.x;
    for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < n1 + n2; i += stride) {
        if (i < n1) {
            const long long e = i / (2 * fh_chunks);
            const long long r = i - e * 2 * fh_chunks;
            w1[i] = r < fh_chunks ? __ldg(wg + e * fh_chunks + r) : __ldg(wu + e * fh_chunks + (r - fh_chunks));
        } else {
            w2[i - n1] = __ldg(wd + (i - n1));
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
        reinterpret_cast<uint4*>(base + p->wb.w1), reinterpret_cast<uint4*>(base + p->wb.w2), F * H / 8, H * F / 8,
        (int)E);
    return cudaGetLastError();
}

}  // namespace moe

namespace moe {
// MXFP8 weight preparation is built with the MXFP8 GEMMs; until then plans
// reject MXFP8 and this is never reached.
cudaError_t launch_prepare_mxfp8(const moe_plan*, const __nv_bfloat16*, const __nv_bfloat16*, const __nv_bfloat16*,
                                 void*, cudaStream_t) {
    return cudaErrorNotSupported;
}
}  // namespace moe
