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
//            experts -> offsets[E+1]; the same over the counts rounded up to
//            row_align -> the padded row space the GEMMs read, and over
//            ceil(count / tile_rows) -> the list of route tiles
//   scatter  per block: one 32-bit lane mask per (warp, expert) gives every
//            route its rank among earlier tokens of the block routed to the
//            same expert (popcount of the lower lanes plus the earlier warps)
//            The scan also zeroes the per-tile counters and the chunk counter
//            through which the bf16 gate/up GEMM copies x rows itself.
// and, for MXFP8, a gather that quantises each token's x row once and writes
// it to its padded route rows.
#include "moe_internal.cuh"
#include "mxfp8.cuh"

namespace moe {
namespace {

__global__ void __launch_bounds__(kTokPerBlk) route_hist_kernel(const int* __restrict__ ids,
                                                                const int* __restrict__ live, int max_live,
                                                                int E, int k, int* __restrict__ blkcnt) {
    extern __shared__ int s_hist[];
    pdl_trigger();
    pdl_wait();
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

// Exclusive scan of one int per thread over a block of kWarps warps; returns
// the exclusive prefix and writes the total to *total (all threads see it).
template <int kWarps>
__device__ __forceinline__ int block_exclusive_scan(int v, int* s_warp, int* total) {
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
        int w = lane < kWarps ? s_warp[lane] : 0;
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
            const int y = __shfl_up_sync(0xffffffffu, w, off);
            if (lane >= off) w += y;
        }
        if (lane < kWarps) s_warp[lane] = w;  // inclusive over warps
    }
    __syncthreads();
    const int warp_prefix = warp > 0 ? s_warp[warp - 1] : 0;
    *total = s_warp[kWarps - 1];
    __syncthreads();
    return warp_prefix + x - v;
}
__device__ __forceinline__ int block_exclusive_scan_1024(int v, int* s_warp, int* total) {
    return block_exclusive_scan<32>(v, s_warp, total);
}

__global__ void __launch_bounds__(1024) route_scan_kernel(const int* __restrict__ live, int max_live, int E,
                                                          int tile_rows, int row_align, int* __restrict__ blkcnt,
                                                          int* __restrict__ offsets,
                                                          int* __restrict__ padoff, int4* __restrict__ tiles,
                                                          int* __restrict__ ready,
                                                          unsigned* __restrict__ status_words) {
    __shared__ int s_warp[32];
    pdl_trigger();
    pdl_wait();
    const int n = clamp_live(live, max_live);
    const int nb = (n + kTokPerBlk - 1) / kTokPerBlk;
    const int e = threadIdx.x;
    int tot = 0;
    if (e < E) {
        // each block's count becomes the exclusive prefix over earlier blocks; the counts
        // of 16 blocks are loaded before any is rewritten, so the loads overlap
        constexpr int kBatch = 16;
        for (int b0 = 0; b0 < nb; b0 += kBatch) {
            int c[kBatch];
#pragma unroll
            for (int i = 0; i < kBatch; ++i) c[i] = b0 + i < nb ? blkcnt[(size_t)(b0 + i) * E + e] : 0;
#pragma unroll
            for (int i = 0; i < kBatch; ++i) {
                if (b0 + i < nb) blkcnt[(size_t)(b0 + i) * E + e] = tot;
                tot += c[i];
            }
        }
    }
    const int mt = (tot + tile_rows - 1) / tile_rows;
    const int padded = (tot + row_align - 1) / row_align * row_align;
    int sum_tot, sum_mt, sum_pad;
    const int ex_tot = block_exclusive_scan_1024(tot, s_warp, &sum_tot);
    const int ex_mt = block_exclusive_scan_1024(mt, s_warp, &sum_mt);
    const int ex_pad = block_exclusive_scan_1024(padded, s_warp, &sum_pad);
    if (e < E) {
        offsets[e] = ex_tot;
        padoff[e] = ex_pad;
        for (int i = 0; i < mt; ++i) {
            const int rows = tot - i * tile_rows;
            tiles[ex_mt + i] =
                make_int4(e, ex_pad + i * tile_rows, rows < tile_rows ? rows : tile_rows, ex_tot + i * tile_rows);
            if (ready != nullptr) ready[ex_mt + i] = 0;
        }
    }
    if (e == 0) {
        offsets[E] = sum_tot;
        padoff[E] = sum_pad;
        status_words[kStNumMTiles] = (unsigned)sum_mt;
        status_words[kStTotalRoutes] = (unsigned)sum_tot;
        status_words[kStCopyNext] = 0u;
    }
}

__global__ void __launch_bounds__(kTokPerBlk) route_scatter_kernel(
    const int* __restrict__ ids, const int* __restrict__ live, int max_live, int E, int k,
    const int* __restrict__ blkprefix, const int* __restrict__ offsets, const int* __restrict__ padoff,
    int* __restrict__ perm, int* __restrict__ inv) {
    extern __shared__ uint32_t s_mem[];
    pdl_trigger();
    pdl_wait();
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
                inv[(size_t)t * k + j] = padoff[e] + row - offsets[e];
            }
        }
    }
}

// Plans of at most kSmallPermuteTokens live rows: the three passes above in
// one 256-thread block, one launch instead of three (each dependent launch
// waits for its predecessor to finish, which at decode sizes costs more than
// the work).  Tokens are taken in chunks of 256 with a running per-expert
// base, so every route gets the same row as in the three-pass form.
constexpr int kSmallPermuteTokens = 4 * kTokPerBlk;

__global__ void __launch_bounds__(kTokPerBlk) route_permute_small_kernel(
    const int* __restrict__ ids, const int* __restrict__ live, int max_live, int E, int k, int tile_rows,
    int row_align, int* __restrict__ offsets, int* __restrict__ padoff, int4* __restrict__ tiles,
    int* __restrict__ perm, int* __restrict__ inv, int* __restrict__ ready, unsigned* __restrict__ status_words) {
    constexpr int kWarps = kTokPerBlk / 32;
    extern __shared__ int s_small[];
    int* s_base = s_small;                                         // [E] count, then next free row
    int* s_off = s_small + E;                                      // [E] offsets[e]
    int* s_pad = s_small + 2 * E;                                  // [E] padoff[e]
    uint32_t* masks = reinterpret_cast<uint32_t*>(s_small + 3 * E);  // [kWarps][E]
    int* wbase = s_small + (3 + kWarps) * E;                       // [kWarps][E]
    __shared__ int s_warp[32];
    pdl_trigger();
    pdl_wait();
    const int n = clamp_live(live, max_live);
    const int tid = threadIdx.x, lane = tid & 31, w = tid >> 5;

    // histogram
    for (int e = tid; e < E; e += kTokPerBlk) s_base[e] = 0;
    __syncthreads();
    for (int i = tid; i < n * k; i += kTokPerBlk) {
        const int e = __ldg(ids + i);
        if (e >= 0) atomicAdd(&s_base[e], 1);
    }
    __syncthreads();

    // scan: thread tid owns the experts [tid * q, tid * q + q)
    const int q = (E + kTokPerBlk - 1) / kTokPerBlk;
    const int e0 = tid * q, e1 = min(E, e0 + q);
    int tot = 0, nmt = 0, npad = 0;
    for (int e = e0; e < e1; ++e) {
        const int c = s_base[e];
        tot += c;
        nmt += (c + tile_rows - 1) / tile_rows;
        npad += (c + row_align - 1) / row_align * row_align;
    }
    int sum_tot, sum_mt, sum_pad;
    int ex_tot = block_exclusive_scan<kWarps>(tot, s_warp, &sum_tot);
    int ex_mt = block_exclusive_scan<kWarps>(nmt, s_warp, &sum_mt);
    int ex_pad = block_exclusive_scan<kWarps>(npad, s_warp, &sum_pad);
    for (int e = e0; e < e1; ++e) {
        const int c = s_base[e];
        const int mt = (c + tile_rows - 1) / tile_rows;
        offsets[e] = ex_tot;
        padoff[e] = ex_pad;
        s_off[e] = ex_tot;
        s_pad[e] = ex_pad;
        for (int i = 0; i < mt; ++i) {
            const int rows = c - i * tile_rows;
            tiles[ex_mt + i] =
                make_int4(e, ex_pad + i * tile_rows, rows < tile_rows ? rows : tile_rows, ex_tot + i * tile_rows);
            if (ready != nullptr) ready[ex_mt + i] = 0;
        }
        s_base[e] = ex_tot;  // the scatter's next free row of expert e
        ex_tot += c;
        ex_mt += mt;
        ex_pad += (c + row_align - 1) / row_align * row_align;
    }
    if (tid == 0) {
        offsets[E] = sum_tot;
        padoff[E] = sum_pad;
        status_words[kStNumMTiles] = (unsigned)sum_mt;
        status_words[kStTotalRoutes] = (unsigned)sum_tot;
        status_words[kStCopyNext] = 0u;
    }

    // stable scatter, 256 tokens at a time (as route_scatter_kernel per block)
    const uint32_t lower = (1u << lane) - 1u;
    for (int t0 = 0; t0 < n; t0 += kTokPerBlk) {
        for (int i = tid; i < kWarps * E; i += kTokPerBlk) masks[i] = 0u;
        __syncthreads();
        const int t = t0 + tid;
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
        for (int e = tid; e < E; e += kTokPerBlk) {
            int base = s_base[e];
#pragma unroll
            for (int w2 = 0; w2 < kWarps; ++w2) {
                wbase[w2 * E + e] = base;
                base += __popc(masks[w2 * E + e]);
            }
            s_base[e] = base;
        }
        __syncthreads();
        if (is_live) {
#pragma unroll
            for (int j = 0; j < kMaxTopK; ++j) {
                if (j < k) {
                    const int e = my_e[j];
                    if (e < 0) {
                        inv[(size_t)t * k + j] = -1;
                    } else {
                        const int row = wbase[w * E + e] + __popc(masks[w * E + e] & lower);
                        perm[row] = t * k + j;
                        inv[(size_t)t * k + j] = s_pad[e] + row - s_off[e];
                    }
                }
            }
        }
        __syncthreads();  // masks and wbase are rewritten by the next chunk
    }
}

constexpr int kRowThreads = 128;

// MXFP8 gather: one 128-thread block per token quantises the token's x row
// once (blocks of 32 along H, 4 threads per block) and writes the E4M3 codes
// to each of its k padded route rows (pitch hp, zero codes past H) and the
// E8M0 bytes into the scale blocks of those rows' 128-row tiles
// ([tile][K block of 128][512 B]).
__global__ void __launch_bounds__(kRowThreads) gather_rows_mxfp8_kernel(const uint4* __restrict__ x,
                                                                        const int* __restrict__ live, int max_live,
                                                                        int H, int hp, int k, int ks1,
                                                                        const int* __restrict__ inv,
                                                                        uint2* __restrict__ xq,
                                                                        uint8_t* __restrict__ xs) {
    __shared__ int s_prow[kMaxTopK];
    pdl_trigger();
    pdl_wait();
    const int n = clamp_live(live, max_live);
    const int chunks = H / 8;       // 8 elements per thread and chunk
    const int chunks_out = hp / 8;  // destination pitch
    for (int t = blockIdx.x; t < n; t += gridDim.x) {
        __syncthreads();
        if (threadIdx.x < k) s_prow[threadIdx.x] = __ldg(inv + (size_t)t * k + threadIdx.x);
        __syncthreads();
        const uint4* src = x + (size_t)t * chunks;
        for (int c0 = 0; c0 < chunks_out; c0 += kRowThreads) {  // uniform trip count: shuffles inside
            const int c = c0 + threadIdx.x;
            const bool active = c < chunks;  // H % 32 == 0: 4-thread groups are all in or all out
            const uint4 v = active ? __ldg(src + c) : make_uint4(0u, 0u, 0u, 0u);
            uint8_t sb;
            const uint2 codes = mxfp8_quantize_8(v, &sb);  // zero codes past H
            if (c < chunks_out) {
                const int g = c >> 2;  // 32-element block index along H
                for (int j = 0; j < k; ++j) {
                    const int pr = s_prow[j];
                    if (pr < 0) continue;
                    xq[(size_t)pr * chunks_out + c] = codes;
                    if (active && (c & 3) == 0)
                        xs[((size_t)(pr / kBM) * ks1 + g / 4) * kSfBlock + sf_block_offset(pr % kBM, g % 4)] = sb;
                }
            }
        }
        // k-group slots past H/32 in the last K stage: scale byte 0 (their codes are TMA zero fill)
        if (threadIdx.x < k) {
            const int pr = s_prow[threadIdx.x];
            if (pr >= 0)
                for (int g = H / 32; g < 4 * ks1; ++g)
                    xs[((size_t)(pr / kBM) * ks1 + g / 4) * kSfBlock + sf_block_offset(pr % kBM, g % 4)] = 0;
        }
    }
}

// Blocks of 128 threads stride over (token, part of its row) items.  With
// fewer live tokens than blocks a row is split over up to one chunk per
// thread, so that a decode-sized launch waits for one round of loads rather
// than several; with many tokens a block takes whole rows (one setup per
// row).  out[t] = sum_j p_j * y[inv[t,j]] as fp32
// FMAs from zero, j in ascending expert id (Megatron-LM PR #7798, "What is
// changed": the unpermute adds a token's routes as fp32 fused multiply-adds
// of probability and row, from zero, in a fixed order; PR #8367: fp32
// result).  The k rows' loads of a chunk are all issued before the FMA chain.
// probs == nullptr: the probabilities were applied in the gate/up epilogue
// and every weight is 1 (fma(1, y, acc) is the plain fp32 sum).  kBf16Out:
// the sum is rounded to bf16, nearest even (the pages' BF16 finalize).
template <bool kBf16Out>
__global__ void __launch_bounds__(kRowThreads) combine_kernel(const float4* __restrict__ y,
                                                              const int* __restrict__ inv,
                                                              const float* __restrict__ probs,
                                                              const int* __restrict__ live, int max_live, int H,
                                                              int k, void* __restrict__ out) {
    __shared__ int s_prow[kMaxTopK];
    __shared__ float s_p[kMaxTopK];
    pdl_trigger();
    pdl_wait();
    const int n = clamp_live(live, max_live);
    const int chunks = H / 4;
    const int max_parts = (chunks + kRowThreads - 1) / kRowThreads;
    int parts = n > 0 ? (int)(gridDim.x / (unsigned)n) : 1;
    parts = parts < 1 ? 1 : (parts > max_parts ? max_parts : parts);
    const int span = (chunks + parts - 1) / parts;  // chunks per item
    const long long items = (long long)n * parts;
    for (long long it = blockIdx.x; it < items; it += gridDim.x) {
        const int t = (int)(it / parts);
        const int c_end = min(chunks, ((int)(it % parts) + 1) * span);
        __syncthreads();
        if (threadIdx.x < k) {
            s_prow[threadIdx.x] = __ldg(inv + (size_t)t * k + threadIdx.x);
            s_p[threadIdx.x] = probs != nullptr ? __ldg(probs + (size_t)t * k + threadIdx.x) : 1.0f;
        }
        __syncthreads();
        for (int c = (int)(it % parts) * span + threadIdx.x; c < c_end; c += kRowThreads) {
            // loads of up to 8 routes in flight at once, then their FMAs in order
            float4 acc = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
            for (int j0 = 0; j0 < k; j0 += 8) {
                float4 v[8];
#pragma unroll
                for (int jj = 0; jj < 8; ++jj) {
                    const int pr = j0 + jj < k ? s_prow[j0 + jj] : -1;
                    v[jj] = pr >= 0 ? __ldg(y + (size_t)pr * chunks + c) : make_float4(0.f, 0.f, 0.f, 0.f);
                }
#pragma unroll
                for (int jj = 0; jj < 8; ++jj) {
                    if (j0 + jj < k && s_prow[j0 + jj] >= 0) {
                        const float p = s_p[j0 + jj];
                        acc.x = __fmaf_rn(p, v[jj].x, acc.x);
                        acc.y = __fmaf_rn(p, v[jj].y, acc.y);
                        acc.z = __fmaf_rn(p, v[jj].z, acc.z);
                        acc.w = __fmaf_rn(p, v[jj].w, acc.w);
                    }
                }
            }
            if (kBf16Out) {
                const __nv_bfloat162 lo = __floats2bfloat162_rn(acc.x, acc.y);
                const __nv_bfloat162 hi = __floats2bfloat162_rn(acc.z, acc.w);
                uint2 w;
                w.x = *reinterpret_cast<const uint32_t*>(&lo);
                w.y = *reinterpret_cast<const uint32_t*>(&hi);
                reinterpret_cast<uint2*>(out)[(size_t)t * chunks + c] = w;
            } else {
                reinterpret_cast<float4*>(out)[(size_t)t * chunks + c] = acc;
            }
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
                           int* padoff, int4* tiles, int* perm, int* inv, int* ready, unsigned* status_words,
                           cudaStream_t s) {
    const int E = p->d.num_experts, k = p->d.top_k;
    const int max_live = (int)p->max_live;
    const int nblk = p->nblk;
    cudaError_t err;
    if (max_live <= kSmallPermuteTokens) {
        const size_t smem = (size_t)(3 + 2 * (kTokPerBlk / 32)) * E * sizeof(int);
        if (smem > 48 * 1024) {
            static int configured_device = -1;  // once per device, at the largest size any plan can ask for
            int dev = 0;
            err = cudaGetDevice(&dev);
            if (err != cudaSuccess) return err;
            if (configured_device != dev) {
                err = cudaFuncSetAttribute(route_permute_small_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                           (int)((3 + 2 * (kTokPerBlk / 32)) * kMaxExperts * sizeof(int)));
                if (err != cudaSuccess) return err;
                configured_device = dev;
            }
        }
        return launch_dependent(route_permute_small_kernel, dim3(1), dim3(kTokPerBlk), smem, s, r_ids, live,
                                max_live, E, k, p->tile_rows, p->row_align, offsets, padoff, tiles, perm, inv, ready,
                                status_words);
    }
    err = launch_dependent(route_hist_kernel, dim3(nblk), dim3(kTokPerBlk), E * sizeof(int), s, r_ids,
                                       live, max_live, E, k, blkcnt);
    if (err != cudaSuccess) return err;
    err = launch_dependent(route_scan_kernel, dim3(1), dim3(1024), 0, s, live, max_live, E, p->tile_rows,
                           p->row_align, blkcnt, offsets, padoff, tiles, ready, status_words);
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
    return launch_dependent(route_scatter_kernel, dim3(nblk), dim3(kTokPerBlk), smem, s, r_ids, live, max_live, E, k,
                            blkcnt, offsets, padoff, perm, inv);
}

cudaError_t launch_gather_mxfp8(const __nv_bfloat16* x, const int* live, int max_live, int H, int hp, int k,
                                const int* inv, uint8_t* xq, uint8_t* xs, cudaStream_t s) {
    const int grid = grid_for_warps(max_live, 1, 16);
    return launch_dependent(gather_rows_mxfp8_kernel, dim3(grid), dim3(kRowThreads), 0, s,
                            reinterpret_cast<const uint4*>(x), live, max_live, H, hp, k, hp / 128, inv,
                            reinterpret_cast<uint2*>(xq), xs);
}

cudaError_t launch_combine(const float* y, const int* inv, const float* probs, const int* live, int max_live,
                           int H, int k, void* out, bool out_bf16, cudaStream_t s) {
    const dim3 grid((unsigned)grid_for_warps((long long)max_live * ((H / 4 + kRowThreads - 1) / kRowThreads), 1, 16));
    if (out_bf16)
        return launch_dependent(combine_kernel<true>, grid, dim3(kRowThreads), 0, s,
                                reinterpret_cast<const float4*>(y), inv, probs, live, max_live, H, k, out);
    return launch_dependent(combine_kernel<false>, grid, dim3(kRowThreads), 0, s,
                            reinterpret_cast<const float4*>(y), inv, probs, live, max_live, H, k, out);
}

}  // namespace moe
