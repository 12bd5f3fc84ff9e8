// permute.cu -- dispatch as a local permute: every (token, expert) route
// becomes one row, rows grouped by expert and stable by token inside an
// expert ("core.transformer.moe.training_matches_inference" API doc,
// `expert_value_pass`: "each row is one route, sorted by local expert";
// Megatron-LM PR #7830: with one rank the dispatch stages are a pass-through).
//
// Three deterministic passes, no atomics on positions:
//   hist     per 256-token block, per-expert route counts (shared-memory
//            counters: a count does not depend on the order of increments)
//   scan     one CTA: per-expert prefix over blocks, exclusive scan over
//            experts -> offsets[E+1]; the same over ceil(count/128) -> the
//            padded row space the GEMM tiles live in, and the M-tile list
//   scatter  per block: one 32-bit lane mask per (warp, expert) gives every
//            route its rank among earlier tokens of the block routed to the
//            same expert (popcount of the lower lanes plus the earlier warps)
// and a gather that copies x rows into their padded route rows.
#include "moe_internal.cuh"

namespace moe {
namespace {

__global__ void __launch_bounds__(kTokPerBlk) route_hist_kernel(const int* __restrict__ ids,
                                                                const int* __restrict__ live, int max_live,
                                                                int E, int k, int* __restrict__ blkcnt) {
    extern __shared__ int s_hist[];
    const int n = clamp_live(live, max_live);
    const int t0 = blockIdx.x * kTokPerBlk;
    if (t0 >= n) return;
    for (int e = threadIdx.x; e < E; e += blockDim.x) s_hist[e] = 0;
    __syncthreads();
    const int t = t0 + threadIdx.x;
    if (t < n) {
        for (int j = 0; j < k; ++j) {
            const int e = __ldg(ids + (size_t)t * k + j);
            if (e >= 0) atomicAdd(&s_hist[e], 1);
        }
    }
    __syncthreads();
    for (int e = threadIdx.x; e < E; e += blockDim.x) blkcnt[(size_t)blockIdx.x * E + e] = s_hist[e];
}

// Exclusive scan of one int per thread over a 1024-thread block; returns the
// exclusive prefix and writes the total to *total (all threads see it).
__device__ __forceinline__ int block_exclusive_scan_1024(int v, int* s_warp, int* total) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    int x = v;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, x, off);
        if (lane >= off) x += y;
    }
    if (lane == 31) s_warp[warp] = x;
    __syncthreads();
    if (warp == 0) {
        int w = s_warp[lane];
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
            const int y = __shfl_up_sync(0xffffffffu, w, off);
            if (lane >= off) w += y;
        }
        s_warp[lane] = w;  // inclusive over warps
    }
    __syncthreads();
    const int warp_prefix = warp > 0 ? s_warp[warp - 1] : 0;
    *total = s_warp[31];
    __syncthreads();
    return warp_prefix + x - v;
}

__global__ void __launch_bounds__(1024) route_scan_kernel(const int* __restrict__ live, int max_live, int E,
                                                          int* __restrict__ blkcnt, int* __restrict__ offsets,
                                                          int* __restrict__ padoff, int4* __restrict__ tiles,
                                                          unsigned* __restrict__ status_words) {
    __shared__ int s_warp[32];
    const int n = clamp_live(live, max_live);
    const int nb = (n + kTokPerBlk - 1) / kTokPerBlk;
    const int e = threadIdx.x;
    int tot = 0;
    if (e < E) {
        for (int b = 0; b < nb; ++b) {
            const int c = blkcnt[(size_t)b * E + e];
            blkcnt[(size_t)b * E + e] = tot;  // becomes the exclusive prefix over earlier blocks
            tot += c;
        }
    }
    const int mt = (tot + kBM - 1) / kBM;
    int sum_tot, sum_mt;
    const int ex_tot = block_exclusive_scan_1024(tot, s_warp, &sum_tot);
    const int ex_mt = block_exclusive_scan_1024(mt, s_warp, &sum_mt);
    if (e < E) {
        offsets[e] = ex_tot;
        padoff[e] = ex_mt * kBM;
        for (int i = 0; i < mt; ++i) {
            const int rows = tot - i * kBM;
            tiles[ex_mt + i] = make_int4(e, (ex_mt + i) * kBM, rows < kBM ? rows : kBM, 0);
        }
    }
    if (e == 0) {
        offsets[E] = sum_tot;
        padoff[E] = sum_mt * kBM;
        status_words[kStNumMTiles] = (unsigned)sum_mt;
        status_words[kStTotalRoutes] = (unsigned)sum_tot;
    }
}

__global__ void __launch_bounds__(kTokPerBlk) route_scatter_kernel(
    const int* __restrict__ ids, const int* __restrict__ live, int max_live, int E, int k,
    const int* __restrict__ blkprefix, const int* __restrict__ offsets, const int* __restrict__ padoff,
    int* __restrict__ perm, int* __restrict__ inv) {
    extern __shared__ uint32_t s_mem[];
    const int n = clamp_live(live, max_live);
    const int t0 = blockIdx.x * kTokPerBlk;
    if (t0 >= n) return;
    constexpr int kWarps = kTokPerBlk / 32;
    uint32_t* masks = s_mem;                                // [kWarps][E]
    int* wbase = reinterpret_cast<int*>(s_mem + kWarps * E);  // [kWarps][E]
    for (int i = threadIdx.x; i < kWarps * E; i += blockDim.x) masks[i] = 0u;
    __syncthreads();
    const int t = t0 + threadIdx.x;
    const int w = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const bool is_live = t < n;
    int my_e[kMaxTopK];
#pragma unroll
    for (int j = 0; j < kMaxTopK; ++j) {
        my_e[j] = -1;
        if (j < k && is_live) {
            my_e[j] = __ldg(ids + (size_t)t * k + j);
            if (my_e[j] >= 0) atomicOr(&masks[w * E + my_e[j]], 1u << lane);
        }
    }
    __syncthreads();
    for (int e = threadIdx.x; e < E; e += blockDim.x) {
        int base = offsets[e] + blkprefix[(size_t)blockIdx.x * E + e];
#pragma unroll
        for (int w2 = 0; w2 < kWarps; ++w2) {
            wbase[w2 * E + e] = base;
            base += __popc(masks[w2 * E + e]);
        }
    }
    __syncthreads();
    if (!is_live) return;
    const uint32_t lower = (1u << lane) - 1u;
#pragma unroll
    for (int j = 0; j < kMaxTopK; ++j) {
        if (j < k) {
            const int e = my_e[j];
            if (e < 0) {
                inv[(size_t)t * k + j] = -1;
            } else {
                const int row = wbase[w * E + e] + __popc(masks[w * E + e] & lower);
                perm[row] = t * k + j;
                inv[(size_t)t * k + j] = padoff[e] + (row - offsets[e]);
            }
        }
    }
}

// One warp per token: read the token's x row once, write it to each of its
// k padded route rows (16-byte chunks, coalesced).
__global__ void __launch_bounds__(256) gather_rows_bf16_kernel(const uint4* __restrict__ x,
                                                               const int* __restrict__ live, int max_live,
                                                               int H, int k, const int* __restrict__ inv,
                                                               uint4* __restrict__ xp) {
    const int n = clamp_live(live, max_live);
    const int lane = threadIdx.x & 31;
    const int wpb = blockDim.x >> 5;
    const int chunks = H / 8;  // 8 bf16 per 16 bytes
    for (int t = blockIdx.x * wpb + (threadIdx.x >> 5); t < n; t += gridDim.x * wpb) {
        const int mine = lane < k ? __ldg(inv + (size_t)t * k + lane) : -1;
        int prow[kMaxTopK];
#pragma unroll
        for (int j = 0; j < kMaxTopK; ++j) prow[j] = __shfl_sync(0xffffffffu, mine, j);
        const uint4* src = x + (size_t)t * chunks;
        for (int c = lane; c < chunks; c += 32) {
            const uint4 v = __ldg(src + c);
#pragma unroll
            for (int j = 0; j < kMaxTopK; ++j)
                if (j < k && prow[j] >= 0) xp[(size_t)prow[j] * chunks + c] = v;
        }
    }
}

// One warp per token: out[t] = sum_j p_j * y[inv[t,j]] as fp32 FMAs from
// zero, j in ascending expert id (Megatron-LM PR #7798, "What is changed":
// the unpermute adds a token's routes as fp32 fused multiply-adds of
// probability and row, from zero, in a fixed order; PR #8367: fp32 result).
__global__ void __launch_bounds__(256) combine_kernel(const float4* __restrict__ y, const int* __restrict__ inv,
                                                      const float* __restrict__ probs,
                                                      const int* __restrict__ live, int max_live, int H, int k,
                                                      float4* __restrict__ out) {
    const int n = clamp_live(live, max_live);
    const int lane = threadIdx.x & 31;
    const int wpb = blockDim.x >> 5;
    const int chunks = H / 4;
    for (int t = blockIdx.x * wpb + (threadIdx.x >> 5); t < n; t += gridDim.x * wpb) {
        const int mine = lane < k ? __ldg(inv + (size_t)t * k + lane) : -1;
        const float pmine = lane < k ? __ldg(probs + (size_t)t * k + lane) : 0.0f;
        int prow[kMaxTopK];
        float pj[kMaxTopK];
#pragma unroll
        for (int j = 0; j < kMaxTopK; ++j) {
            prow[j] = __shfl_sync(0xffffffffu, mine, j);
            pj[j] = __shfl_sync(0xffffffffu, pmine, j);
        }
        for (int c = lane; c < chunks; c += 32) {
            float4 acc = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
#pragma unroll
            for (int j = 0; j < kMaxTopK; ++j) {
                if (j < k && prow[j] >= 0) {
                    const float4 v = __ldg(y + (size_t)prow[j] * chunks + c);
                    acc.x = __fmaf_rn(pj[j], v.x, acc.x);
                    acc.y = __fmaf_rn(pj[j], v.y, acc.y);
                    acc.z = __fmaf_rn(pj[j], v.z, acc.z);
                    acc.w = __fmaf_rn(pj[j], v.w, acc.w);
                }
            }
            out[(size_t)t * chunks + c] = acc;
        }
    }
}

int grid_for_warps(long long items, int warps_per_block, int per_sm) {
    long long blocks = (items + warps_per_block - 1) / warps_per_block;
    const long long cap = (long long)num_sms() * per_sm;
    if (blocks > cap) blocks = cap;
    if (blocks < 1) blocks = 1;
    return (int)blocks;
}

}  // namespace

cudaError_t launch_permute(const moe_plan* p, const int* live, int* r_ids, int* blkcnt, int* offsets,
                           int* padoff, int4* tiles, int* perm, int* inv, unsigned* status_words,
                           cudaStream_t s) {
    const int E = p->d.num_experts, k = p->d.top_k;
    const int max_live = (int)p->max_live;
    const int nblk = p->nblk;
    route_hist_kernel<<<nblk, kTokPerBlk, E * sizeof(int), s>>>(r_ids, live, max_live, E, k, blkcnt);
    cudaError_t err = cudaGetLastError();
    if (err != cudaSuccess) return err;
    route_scan_kernel<<<1, 1024, 0, s>>>(live, max_live, E, blkcnt, offsets, padoff, tiles, status_words);
    err = cudaGetLastError();
    if (err != cudaSuccess) return err;
    const size_t smem = (size_t)(kTokPerBlk / 32) * E * 8;
    if (smem > 48 * 1024) {
        // once per device, at the largest size any plan can ask for
        static int configured_device = -1;
        int dev = 0;
        err = cudaGetDevice(&dev);
        if (err != cudaSuccess) return err;
        if (configured_device != dev) {
            err = cudaFuncSetAttribute(route_scatter_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)((kTokPerBlk / 32) * kMaxExperts * 8));
            if (err != cudaSuccess) return err;
            configured_device = dev;
        }
    }
    route_scatter_kernel<<<nblk, kTokPerBlk, smem, s>>>(r_ids, live, max_live, E, k, blkcnt, offsets, padoff,
                                                        perm, inv);
    return cudaGetLastError();
}

cudaError_t launch_gather_bf16(const __nv_bfloat16* x, const int* live, int max_live, int H, int k,
                               const int* inv, __nv_bfloat16* xp, cudaStream_t s) {
    const int grid = grid_for_warps(max_live, 8, 8);
    gather_rows_bf16_kernel<<<grid, 256, 0, s>>>(reinterpret_cast<const uint4*>(x), live, max_live, H, k, inv,
                                                 reinterpret_cast<uint4*>(xp));
    return cudaGetLastError();
}

cudaError_t launch_combine(const float* y, const int* inv, const float* probs, const int* live, int max_live,
                           int H, int k, float* out, cudaStream_t s) {
    const int grid = grid_for_warps(max_live, 8, 8);
    combine_kernel<<<grid, 256, 0, s>>>(reinterpret_cast<const float4*>(y), inv, probs, live, max_live, H, k,
                                        reinterpret_cast<float4*>(out));
    return cudaGetLastError();
}

}  // namespace moe
