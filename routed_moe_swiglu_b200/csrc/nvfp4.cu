// nvfp4.cu -- NVFP4 quantisation for the per-token recipe (Megatron-LM PR
// #7798, "Per-token NVFP4"; the arithmetic is in nvfp4.cuh): rows of bf16
// through the public entry point, token rows of x into their padded route
// rows, the fp32 h rows of the gate/up GEMM, and the expert weights into the
// GEMMs' layout.
//
// Layout of the GEMM operands (K pitches padded to 256 elements = 128 bytes
// with zero codes and zero scale bytes):
//   codes     rows of K/2 bytes;
//   scales    per 128-row tile and 128-byte K block, four 512-byte blocks,
//             one per 64-element MMA step, each [row%32][row/32][4 blocks of
//             16] (nvfp4_sf_offset) -- the image one tcgen05.cp moves;
//   g         fp32 per padded route row (x, h) or per expert matrix (W1, W2).
#include "moe_internal.cuh"
#include "nvfp4.cuh"

namespace moe {
namespace {

constexpr int kQThreads = 128;

__device__ __forceinline__ void bf16x8(uint4 v, float (&f)[8]) {
    f[0] = bf16lo(v.x); f[1] = bf16hi(v.x); f[2] = bf16lo(v.y); f[3] = bf16hi(v.y);
    f[4] = bf16lo(v.z); f[5] = bf16hi(v.z); f[6] = bf16lo(v.w); f[7] = bf16hi(v.w);
}
__device__ __forceinline__ float amax8(const float (&f)[8]) {
    float a = 0.0f;
#pragma unroll
    for (int i = 0; i < 8; ++i) a = fmaxf(a, fabsf(f[i]));
    return a;
}
__device__ __forceinline__ float block_max(float a, float* s_red) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, o));
    __syncthreads();
    if ((threadIdx.x & 31) == 0) s_red[threadIdx.x >> 5] = a;
    __syncthreads();
    float m = 0.0f;
    for (int w = 0; w < (int)(blockDim.x >> 5); ++w) m = fmaxf(m, s_red[w]);
    return m;
}
// Scale-block byte index of element `e0` (a multiple of 16) of padded row `row`
// in an operand whose 128-row tiles hold `ks` K blocks of 256 elements.
__device__ __forceinline__ size_t sf_index(long long row, int e0, int ks) {
    return ((((size_t)(row / 128) * ks + e0 / 256) * 4 + (e0 % 256) / 64) * kSfBlock) +
           nvfp4_sf_offset((int)(row % 128), (e0 % 64) / 16);
}

// Public quantiser: one warp per row; pass 1 the row's amax, pass 2 the codes.
// Lane l holds 8 elements per chunk, so a block of 16 is two neighbouring lanes.
__global__ void __launch_bounds__(256) nvfp4_quantize_rows_kernel(const uint4* __restrict__ in, long long rows,
                                                                  int cols, long long ld_in_chunks,
                                                                  const int* __restrict__ live,
                                                                  uint32_t* __restrict__ q, uint8_t* __restrict__ scales,
                                                                  float* __restrict__ gout) {
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
        float a = 0.0f;
        for (int c = lane; c < chunks; c += 32) {
            float f[8];
            bf16x8(__ldg(src + c), f);
            a = fmaxf(a, amax8(f));
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, o));
        const float g = nvfp4_global(a);
        if (lane == 0) gout[r] = g;
        for (int c = lane; c < ((chunks + 31) & ~31); c += 32) {  // uniform trip count: shuffles inside
            const bool active = c < chunks;  // cols % 16 == 0: lane pairs are in or out together
            float f[8];
            bf16x8(active ? __ldg(src + c) : make_uint4(0u, 0u, 0u, 0u), f);
            const float ab = fmaxf(amax8(f), __shfl_xor_sync(0xffffffffu, amax8(f), 1));
            float d;
            const uint8_t sb = nvfp4_block_scale(ab, g, &d);
            if (active) {
                q[r * chunks + c] = nvfp4_codes_8(f, d);
                if ((lane & 1) == 0) scales[r * (cols / 16) + c / 2] = sb;
            }
        }
    }
}

// x rows: one block per token (grid-stride) quantises the token's row with its
// own scale and writes the codes, block scales and g to each of its k padded
// route rows (zero codes and scales from H to the pitch hp).
__global__ void __launch_bounds__(kQThreads) gather_rows_nvfp4_kernel(const uint4* __restrict__ x,
                                                                      const int* __restrict__ live, int max_live,
                                                                      int H, int hp, int k, int ks1,
                                                                      const int* __restrict__ inv,
                                                                      uint32_t* __restrict__ xq,
                                                                      uint8_t* __restrict__ xs,
                                                                      float* __restrict__ xg,
                                                                      const unsigned* status) {
    __shared__ int s_prow[kMaxTopK];
    __shared__ float s_red[kQThreads / 32];
    pdl_trigger();
    pdl_wait();
    const int n = live_rows(live, max_live, status);
    const int chunks = H / 8, chunks_out = hp / 8;
    for (int t = blockIdx.x; t < n; t += gridDim.x) {
        __syncthreads();
        if (threadIdx.x < k) s_prow[threadIdx.x] = __ldg(inv + (size_t)t * k + threadIdx.x);
        const uint4* src = x + (size_t)t * chunks;
        float a = 0.0f;
        for (int c = threadIdx.x; c < chunks; c += kQThreads) {
            float f[8];
            bf16x8(__ldg(src + c), f);
            a = fmaxf(a, amax8(f));
        }
        const float g = nvfp4_global(block_max(a, s_red));
        if (threadIdx.x < k && s_prow[threadIdx.x] >= 0) xg[s_prow[threadIdx.x]] = g;
        for (int c0 = 0; c0 < chunks_out; c0 += kQThreads) {  // uniform trip count: shuffles inside
            const int c = c0 + threadIdx.x;
            float f[8];
            bf16x8(c < chunks ? __ldg(src + c) : make_uint4(0u, 0u, 0u, 0u), f);
            const float ab = fmaxf(amax8(f), __shfl_xor_sync(0xffffffffu, amax8(f), 1));
            float d;
            const uint8_t sb = nvfp4_block_scale(ab, g, &d);
            const uint32_t codes = nvfp4_codes_8(f, d);
            if (c < chunks_out) {
                for (int j = 0; j < k; ++j) {
                    const int pr = s_prow[j];
                    if (pr < 0) continue;
                    xq[(size_t)pr * (chunks_out) + c] = codes;
                    if ((c & 1) == 0) xs[sf_index(pr, c * 8, ks1)] = sb;
                }
            }
        }
    }
}

// h rows: one block per live route (grid-stride over n * k) quantises its fp32
// row of the gate/up GEMM (pitch fp, zeros past F) with the row's own scale.
__global__ void __launch_bounds__(kQThreads) quantize_h_nvfp4_kernel(const float4* __restrict__ hf,
                                                                     const int* __restrict__ live, int max_live,
                                                                     int k, int fp, int ks2,
                                                                     const int* __restrict__ inv,
                                                                     uint32_t* __restrict__ hq,
                                                                     uint8_t* __restrict__ hs,
                                                                     float* __restrict__ hg,
                                                                     const unsigned* status) {
    __shared__ float s_red[kQThreads / 32];
    pdl_trigger();
    pdl_wait();
    const int n = live_rows(live, max_live, status);
    const int chunks = fp / 8;
    for (long long i = blockIdx.x; i < (long long)n * k; i += gridDim.x) {
        const int pr = __ldg(inv + i);  // uniform over the block
        if (pr < 0) continue;
        const float4* src = hf + (size_t)pr * (fp / 4);
        float a = 0.0f;
        for (int c = threadIdx.x; c < chunks; c += kQThreads) {
            const float4 u = __ldg(src + 2 * c), w = __ldg(src + 2 * c + 1);
            a = fmaxf(a, fmaxf(fmaxf(fabsf(u.x), fabsf(u.y)), fmaxf(fabsf(u.z), fabsf(u.w))));
            a = fmaxf(a, fmaxf(fmaxf(fabsf(w.x), fabsf(w.y)), fmaxf(fabsf(w.z), fabsf(w.w))));
        }
        const float g = nvfp4_global(block_max(a, s_red));
        if (threadIdx.x == 0) hg[pr] = g;
        for (int c0 = 0; c0 < chunks; c0 += kQThreads) {
            const int c = c0 + threadIdx.x;
            float f[8] = {0.0f, 0.0f, 0.0f, 0.0f, 0.0f, 0.0f, 0.0f, 0.0f};
            if (c < chunks) {
                const float4 u = __ldg(src + 2 * c), w = __ldg(src + 2 * c + 1);
                f[0] = u.x; f[1] = u.y; f[2] = u.z; f[3] = u.w; f[4] = w.x; f[5] = w.y; f[6] = w.z; f[7] = w.w;
            }
            const float ab = fmaxf(amax8(f), __shfl_xor_sync(0xffffffffu, amax8(f), 1));
            float d;
            const uint8_t sb = nvfp4_block_scale(ab, g, &d);
            if (c < chunks) {
                hq[(size_t)pr * chunks + c] = nvfp4_codes_8(f, d);
                if ((c & 1) == 0) hs[sf_index(pr, c * 8, ks2)] = sb;
            }
        }
    }
}

// Weights, pass 1: the largest magnitude of each expert matrix (W1 = gate and
// up together, W2), as the bit pattern of a non-negative float (whose integer
// order is its value order) in gbits[2e] and gbits[2e + 1], zeroed beforehand.
__global__ void __launch_bounds__(256) weights_amax_kernel(const uint4* __restrict__ wg, const uint4* __restrict__ wu,
                                                           const uint4* __restrict__ wd, long long fh_chunks,
                                                           unsigned* __restrict__ gbits) {
    __shared__ float s_red[8];
    const int e = blockIdx.y, m = blockIdx.z;
    float a = 0.0f;
    const long long per = (m == 0 && wu != nullptr) ? 2 * fh_chunks : fh_chunks;
    for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < per; i += (long long)gridDim.x * blockDim.x) {
        const uint4* src = m == 1 ? wd : (i < fh_chunks ? wg : wu);
        float f[8];
        bf16x8(__ldg(src + (long long)e * fh_chunks + (i < fh_chunks ? i : i - fh_chunks)), f);
        a = fmaxf(a, amax8(f));
    }
    a = block_max(a, s_red);
    if (threadIdx.x == 0) atomicMax(gbits + 2 * e + m, __float_as_uint(a));
}

// Weights, pass 2: amax bits -> the second-level scale, in place.
__global__ void weights_global_kernel(unsigned* gbits, int n) {
    const int i = blockIdx.x * blockDim.x + threadIdx.x;
    if (i < n) gbits[i] = __float_as_uint(nvfp4_global(__uint_as_float(gbits[i])));
}

// Weights, pass 3: one block per weight row (grid-stride), codes and block scales
// in the GEMMs' layout (as the MXFP8 weights: W1 tiles of 64 f with gate / up
// interleaved in groups of 16, squared-ReLU experts 128 f per tile; W2 rows in
// order, 128 per tile).
__global__ void __launch_bounds__(kQThreads) prepare_nvfp4_kernel(
    const uint4* __restrict__ wg, const uint4* __restrict__ wu, const uint4* __restrict__ wd,
    const float* __restrict__ gw, uint32_t* __restrict__ w1q, uint8_t* __restrict__ w1s, uint32_t* __restrict__ w2q,
    uint8_t* __restrict__ w2s, int E, int F, int H, int hp, int fp, int nt1, int ks1, int nt2, int ks2, int relu2) {
    const long long rows1 = (long long)E * (relu2 ? 1 : 2) * F;
    const long long rows2 = (long long)E * H;
    for (long long row = blockIdx.x; row < rows1 + rows2; row += gridDim.x) {
        const uint4* src;
        uint32_t* dst;
        uint8_t* sf;
        long long srow;  // row index within the scale layout (tile * 128 + tile row)
        int len, ks;
        float g;
        if (row < rows1) {
            const int per_e = relu2 ? F : 2 * F;
            const long long e = row / per_e;
            const int rem = (int)(row - e * per_e);
            const int gu = rem / F, f = rem - gu * F;
            src = (gu ? wu : wg) + ((size_t)e * F + f) * (H / 8);
            const int tile = relu2 ? f / 128 : f / kG1BN8;
            const int trow = relu2 ? f % 128 : ((f % kG1BN8) >> 4) * 32 + gu * 16 + (f & 15);
            srow = (e * nt1 + tile) * 128 + trow;
            dst = w1q + (size_t)srow * (hp / 8);
            len = H;
            ks = ks1;
            sf = w1s;
            g = __ldg(gw + 2 * e);
        } else {
            const long long r2 = row - rows1;
            const long long e = r2 / H;
            const int c = (int)(r2 - e * H);
            src = wd + (size_t)r2 * (F / 8);
            dst = w2q + (size_t)r2 * (fp / 8);
            srow = (e * nt2 + c / kG2BN8) * 128 + c % kG2BN8;
            len = F;
            ks = ks2;
            sf = w2s;
            g = __ldg(gw + 2 * e + 1);
        }
        const int chunks = len / 8;
        for (int c0 = 0; c0 < chunks; c0 += kQThreads) {  // len % 32 == 0: lane pairs in or out together
            const int c = c0 + threadIdx.x;
            const bool active = c < chunks;
            float f[8];
            bf16x8(active ? __ldg(src + c) : make_uint4(0u, 0u, 0u, 0u), f);
            const float ab = fmaxf(amax8(f), __shfl_xor_sync(0xffffffffu, amax8(f), 1));
            float d;
            const uint8_t sb = nvfp4_block_scale(ab, g, &d);
            if (active) {
                dst[c] = nvfp4_codes_8(f, d);
                if ((c & 1) == 0) sf[sf_index(srow, c * 8, ks)] = sb;
            }
        }
    }
}

}  // namespace

cudaError_t launch_nvfp4_quantize_rows(const __nv_bfloat16* in, long long rows, int cols, long long ld_in,
                                       uint8_t* q, uint8_t* scales, float* g, const int* live_rows, cudaStream_t s) {
    long long blocks = (rows + 7) / 8;
    const long long cap = (long long)num_sms() * 8;
    if (blocks > cap) blocks = cap;
    if (blocks < 1) blocks = 1;
    nvfp4_quantize_rows_kernel<<<(unsigned)blocks, 256, 0, s>>>(reinterpret_cast<const uint4*>(in), rows, cols,
                                                                ld_in / 8, live_rows, reinterpret_cast<uint32_t*>(q),
                                                                scales, g);
    return cudaGetLastError();
}

cudaError_t launch_gather_nvfp4(const __nv_bfloat16* x, const int* live, int max_live, int H, int hp, int k,
                                const int* inv, uint8_t* xq, uint8_t* xs, float* xg, const unsigned* status,
                                cudaStream_t s) {
    long long grid = max_live;
    const long long cap = (long long)num_sms() * 16;
    if (grid > cap) grid = cap;
    if (grid < 1) grid = 1;
    return launch_dependent(gather_rows_nvfp4_kernel, dim3((unsigned)grid), dim3(kQThreads), 0, s,
                            reinterpret_cast<const uint4*>(x), live, max_live, H, hp, k, hp / 256, inv,
                            reinterpret_cast<uint32_t*>(xq), xs, xg, status);
}

cudaError_t launch_quantize_h_nvfp4(const float* hf, const int* live, int max_live, int k, int fp, const int* inv,
                                    uint8_t* hq, uint8_t* hs, float* hg, const unsigned* status, cudaStream_t s) {
    long long grid = (long long)max_live * k;
    const long long cap = (long long)num_sms() * 16;
    if (grid > cap) grid = cap;
    if (grid < 1) grid = 1;
    return launch_dependent(quantize_h_nvfp4_kernel, dim3((unsigned)grid), dim3(kQThreads), 0, s,
                            reinterpret_cast<const float4*>(hf), live, max_live, k, fp, fp / 256, inv,
                            reinterpret_cast<uint32_t*>(hq), hs, hg, status);
}

cudaError_t launch_prepare_nvfp4(const moe_plan* p, const __nv_bfloat16* wg, const __nv_bfloat16* wu,
                                 const __nv_bfloat16* wd, void* buf, cudaStream_t s) {
    uint8_t* base = static_cast<uint8_t*>(buf);
    const int E = p->d.num_experts, F = p->d.ffn, H = p->d.hidden;
    const bool relu2 = (p->d.flags & MOE_FLAG_SQUARED_RELU) != 0;
    // padding codes and scale bytes are zero; so are the W1 rows of f >= F
    cudaError_t err = cudaMemsetAsync(base, 0, p->wb.total, s);
    if (err != cudaSuccess) return err;
    unsigned* gbits = reinterpret_cast<unsigned*>(base + p->wb.wg);
    const long long fh_chunks = (long long)F * H / 8;
    weights_amax_kernel<<<dim3(16, (unsigned)E, 2), 256, 0, s>>>(
        reinterpret_cast<const uint4*>(wg), relu2 ? nullptr : reinterpret_cast<const uint4*>(wu),
        reinterpret_cast<const uint4*>(wd), fh_chunks, gbits);
    err = cudaGetLastError();
    if (err != cudaSuccess) return err;
    weights_global_kernel<<<(2 * E + 255) / 256, 256, 0, s>>>(gbits, 2 * E);
    err = cudaGetLastError();
    if (err != cudaSuccess) return err;
    prepare_nvfp4_kernel<<<num_sms() * 16, kQThreads, 0, s>>>(
        reinterpret_cast<const uint4*>(wg), reinterpret_cast<const uint4*>(wu), reinterpret_cast<const uint4*>(wd),
        reinterpret_cast<const float*>(gbits), reinterpret_cast<uint32_t*>(base + p->wb.w1), base + p->wb.w1s,
        reinterpret_cast<uint32_t*>(base + p->wb.w2), base + p->wb.w2s, E, F, H, (int)p->hp, (int)p->fp, p->nt1,
        p->ks1, p->nt2, p->ks2, relu2 ? 1 : 0);
    return cudaGetLastError();
}

}  // namespace moe
