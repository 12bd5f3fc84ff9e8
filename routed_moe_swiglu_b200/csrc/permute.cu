// permute.cu -- dispatch as a local permute: every (token, expert) route
// becomes one row, rows grouped by expert and stable by token inside an
// expert ("core.transformer.moe.training_matches_inference" API doc,
// `expert_value_pass`: "each row is one route, sorted by local expert";
// Megatron-LM PR #7830: with one rank the dispatch stages are a pass-through).
//
// One launch, deterministic, no atomics on positions:
//   hist     per 256-token chunk, per-expert route counts (shared-memory
//            counters: a count does not depend on the order of increments)
//   scan     a warp per expert: the counts of the chunks become exclusive
//            prefixes over earlier chunks, and the expert's total; then every
//            block scans the totals over experts -> offsets[E+1], the same
//            over the counts rounded up to row_align -> the padded row space
//            the GEMMs read, and over ceil(count / tile_rows) -> the list of
//            route tiles
//   scatter  per chunk: one 32-bit lane mask per (warp, expert) gives every
//            route its rank among earlier tokens of the chunk routed to the
//            same expert (popcount of the lower lanes plus the earlier warps)
// The three phases meet in two grid-wide barriers (a counter in the
// workspace's status words, zeroed by the router kernel of the same forward;
// every wait bounded).  With at most 1,024 live rows one block does all three
// phases and no barrier is needed.  The scan also zeroes the per-tile
// counters, the chunk counter and the started-tile mark through which the
// bf16 gate/up GEMM copies x rows itself.  For MXFP8, a gather then quantises each token's x row once
// and writes it to its padded route rows.
#include "moe_internal.cuh"
#include "mxfp8.cuh"
#include "ptx.cuh"

namespace moe {
namespace {

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

constexpr int kPermWarps = kTokPerBlk / 32;
// Plans with at most this many live rows permute in one block, without barriers.
constexpr int kSmallPermuteTokens = 4 * kTokPerBlk;

struct PermuteArgs {
    const int* ids;       // canonical routes [max_live, k] (-1: dropped)
    const int* live;
    int max_live, E, k, tile_rows, row_align;
    int* blkcnt;          // [chunks][E]: counts, then exclusive prefixes over chunks
    int* tot;             // [E]: routes per expert
    int* offsets;         // [E + 1]
    int* padoff;          // [E + 1]
    int4* tiles;
    int* perm;
    int* inv;
    int* ready;           // bf16: per-tile copy counters (zeroed here), else null
    unsigned* status;     // status words
    unsigned long long wait_limit_ns;
};

// Shared memory of the permute block: s_count[E] (count, then the chunk's next
// free row), s_off[E], s_pad[E], masks[kPermWarps][E], wbase[kPermWarps][E].
__host__ __device__ constexpr size_t permute_smem_bytes(int E) {
    return (size_t)(3 + 2 * kPermWarps) * (size_t)E * sizeof(int);
}

// The scan over experts of per-expert counts c[e] (read through count(e)):
// offsets, padded offsets and the tile list; thread tid owns experts
// [tid * q, tid * q + q).  Every thread of the block calls it; s_off / s_pad
// receive offsets[e] / padoff[e]; when `write`, the globals are written too.
template <class CountFn>
__device__ __forceinline__ void scan_experts(const PermuteArgs& a, CountFn count, int* s_off, int* s_pad,
                                             int* s_warp, bool write) {
    const int tid = threadIdx.x, E = a.E;
    const int q = (E + kTokPerBlk - 1) / kTokPerBlk;
    const int e0 = tid * q, e1 = min(E, e0 + q);
    int tot = 0, nmt = 0, npad = 0, widest = 0;
    for (int e = e0; e < e1; ++e) {
        const int c = count(e);
        tot += c;
        nmt += (c + a.tile_rows - 1) / a.tile_rows;
        npad += (c + a.row_align - 1) / a.row_align * a.row_align;
        widest = max(widest, min(c, a.tile_rows));
    }
    // the widest route tile (a block-wide max, through the scan's scratch)
    widest = __reduce_max_sync(0xffffffffu, widest);
    if ((tid & 31) == 0) s_warp[tid >> 5] = widest;
    __syncthreads();
    widest = 0;
    for (int w = 0; w < kPermWarps; ++w) widest = max(widest, s_warp[w]);
    __syncthreads();
    int sum_tot, sum_mt, sum_pad;
    int ex_tot = block_exclusive_scan<kPermWarps>(tot, s_warp, &sum_tot);
    int ex_mt = block_exclusive_scan<kPermWarps>(nmt, s_warp, &sum_mt);
    int ex_pad = block_exclusive_scan<kPermWarps>(npad, s_warp, &sum_pad);
    for (int e = e0; e < e1; ++e) {
        const int c = count(e);
        const int mt = (c + a.tile_rows - 1) / a.tile_rows;
        s_off[e] = ex_tot;
        s_pad[e] = ex_pad;
        if (write) {
            a.offsets[e] = ex_tot;
            a.padoff[e] = ex_pad;
            for (int i = 0; i < mt; ++i) {
                const int rows = c - i * a.tile_rows;
                a.tiles[ex_mt + i] = make_int4(e, ex_pad + i * a.tile_rows, rows < a.tile_rows ? rows : a.tile_rows,
                                               ex_tot + i * a.tile_rows);
                if (a.ready != nullptr) a.ready[ex_mt + i] = 0;
            }
        }
        ex_tot += c;
        ex_mt += mt;
        ex_pad += (c + a.row_align - 1) / a.row_align * a.row_align;
    }
    if (write && tid == 0) {
        a.offsets[E] = sum_tot;
        a.padoff[E] = sum_pad;
        a.status[kStTotalRoutes] = (unsigned)sum_tot;
        a.status[kStCopyNext] = 0u;
        a.status[kStTileStarted] = 0u;
        a.status[kStMaxTileRows] = (unsigned)widest;
        __threadfence();
        a.status[kStNumMTiles] = (unsigned)sum_mt;
    }
}

// Stable scatter of the 256 tokens from t0: each route's row is s_base[e]
// (the chunk's first free row of expert e) plus its rank in the chunk;
// s_base[e] is advanced past the chunk.  s_off / s_pad map a row to its
// padded row.
// The k canonical expert ids of token t (all -1 past the live count), loaded together.
__device__ __forceinline__ void load_token_ids(const PermuteArgs& a, int t, int n, int (&ids)[kMaxTopK]) {
#pragma unroll
    for (int j = 0; j < kMaxTopK; ++j) ids[j] = (j < a.k && t < n) ? __ldg(a.ids + (size_t)t * a.k + j) : -1;
}

// my_e: the ids of this thread's token t0 + threadIdx.x (load_token_ids).
__device__ __forceinline__ void scatter_chunk(const PermuteArgs& a, int n, int t0, const int (&my_e)[kMaxTopK],
                                              int* s_base, const int* s_off, const int* s_pad, uint32_t* masks,
                                              int* wbase) {
    const int tid = threadIdx.x, lane = tid & 31, w = tid >> 5, E = a.E, k = a.k;
    for (int i = tid; i < kPermWarps * E; i += kTokPerBlk) masks[i] = 0u;
    __syncthreads();
    const int t = t0 + tid;
    const bool is_live = t < n;
#pragma unroll
    for (int j = 0; j < kMaxTopK; ++j)
        if (j < k && my_e[j] >= 0) atomicOr(&masks[w * E + my_e[j]], 1u << lane);
    __syncthreads();
    for (int e = tid; e < E; e += kTokPerBlk) {
        int base = s_base[e];
#pragma unroll
        for (int w2 = 0; w2 < kPermWarps; ++w2) {
            wbase[w2 * E + e] = base;
            base += __popc(masks[w2 * E + e]);
        }
        s_base[e] = base;
    }
    __syncthreads();
    if (is_live) {
        const uint32_t lower = (1u << lane) - 1u;
#pragma unroll
        for (int j = 0; j < kMaxTopK; ++j) {
            if (j < k) {
                const int e = my_e[j];
                if (e < 0) {
                    a.inv[(size_t)t * k + j] = -1;
                } else {
                    const int row = wbase[w * E + e] + __popc(masks[w * E + e] & lower);
                    a.perm[row] = t * k + j;
                    a.inv[(size_t)t * k + j] = s_pad[e] + row - s_off[e];
                }
            }
        }
    }
    __syncthreads();  // masks and wbase are rewritten by the next chunk
}

// Grid-wide barrier of the `parts` participating blocks (all resident: the
// grid is at most one block per SM and the next kernel is released only after
// the barriers).  Returns false when the wait ran out (MOE_DEV_TIMEOUT set).
__device__ __forceinline__ bool permute_grid_barrier(const PermuteArgs& a, int target, int* s_flag) {
    __syncthreads();  // the block's writes precede the arrival (bar.sync is cumulative)
    if (threadIdx.x == 0) {
        int* bar = reinterpret_cast<int*>(a.status + kStPermBar);
        __threadfence();
        red_release_gpu_add(bar, 1);
        volatile int never = 0;
        const bool ok = wait_count_bounded(bar, target, &never, a.wait_limit_ns);
        if (!ok) atomicOr(a.status + kStFlags, MOE_DEV_TIMEOUT);
        __threadfence();
        *s_flag = ok ? 1 : 0;
    }
    __syncthreads();
    return *s_flag != 0;
}

__global__ void __launch_bounds__(kTokPerBlk) route_permute_kernel(const PermuteArgs a) {
    extern __shared__ int s_perm[];
    __shared__ int s_warp[32];
    __shared__ int s_flag;
    const int E = a.E;
    int* s_count = s_perm;
    int* s_off = s_perm + E;
    int* s_pad = s_perm + 2 * E;
    uint32_t* masks = reinterpret_cast<uint32_t*>(s_perm + 3 * E);
    int* wbase = s_perm + (3 + kPermWarps) * E;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    // No early launch of the next kernel: it is released once every block of
    // this grid has passed the barriers (see permute_grid_barrier).
    pdl_wait();
    const int n = clamp_live(a.live, a.max_live);

    if (n <= kSmallPermuteTokens) {
        // one block: histogram, scan, scatter in chunks of 256 with a running base
        if (blockIdx.x == 0) {
            for (int e = tid; e < E; e += kTokPerBlk) s_count[e] = 0;
            // thread tid takes token tid of each chunk; the first chunk's ids stay in
            // registers for its scatter (decode: the only chunk)
            int first[kMaxTopK];
            load_token_ids(a, tid, n, first);
            __syncthreads();
            for (int t0 = 0; t0 < n; t0 += kTokPerBlk) {
                int ids[kMaxTopK];
                if (t0 == 0) {
#pragma unroll
                    for (int j = 0; j < kMaxTopK; ++j) ids[j] = first[j];
                } else {
                    load_token_ids(a, t0 + tid, n, ids);
                }
#pragma unroll
                for (int j = 0; j < kMaxTopK; ++j)
                    if (ids[j] >= 0) atomicAdd(&s_count[ids[j]], 1);
            }
            __syncthreads();
            scan_experts(a, [&](int e) { return s_count[e]; }, s_off, s_pad, s_warp, true);
            __syncthreads();
            for (int e = tid; e < E; e += kTokPerBlk) s_count[e] = s_off[e];  // next free row of expert e
            __syncthreads();
            for (int t0 = 0; t0 < n; t0 += kTokPerBlk) {
                int ids[kMaxTopK];
                if (t0 == 0) {
#pragma unroll
                    for (int j = 0; j < kMaxTopK; ++j) ids[j] = first[j];
                } else {
                    load_token_ids(a, t0 + tid, n, ids);
                }
                scatter_chunk(a, n, t0, ids, s_count, s_off, s_pad, masks, wbase);
            }
        }
        pdl_trigger();
        return;
    }

    const int nb = (n + kTokPerBlk - 1) / kTokPerBlk;  // chunks of 256 tokens
    const int parts = (int)gridDim.x < nb ? (int)gridDim.x : nb;
    if ((int)blockIdx.x >= parts) {
        pdl_trigger();
        return;
    }
    // phase 1: the histogram of each chunk this block owns
    for (int c = blockIdx.x; c < nb; c += parts) {
        int ids[kMaxTopK];
        load_token_ids(a, c * kTokPerBlk + tid, n, ids);
        for (int e = tid; e < E; e += kTokPerBlk) s_count[e] = 0;
        __syncthreads();
#pragma unroll
        for (int j = 0; j < kMaxTopK; ++j)
            if (ids[j] >= 0) atomicAdd(&s_count[ids[j]], 1);
        __syncthreads();
        for (int e = tid; e < E; e += kTokPerBlk) a.blkcnt[(size_t)c * E + e] = s_count[e];
        __syncthreads();
    }
    bool ok = permute_grid_barrier(a, parts, &s_flag);
    // phase 2: a warp per expert turns its column of chunk counts into exclusive
    // prefixes over earlier chunks (32 chunks per step, in place) and its total
    if (ok) {
        for (int e = blockIdx.x * kPermWarps + warp; e < E; e += parts * kPermWarps) {
            int carry = 0;
            for (int c0 = 0; c0 < nb; c0 += 32) {
                const int c = c0 + lane;
                const int v = c < nb ? __ldcg(a.blkcnt + (size_t)c * E + e) : 0;
                int x = v;
#pragma unroll
                for (int off = 1; off < 32; off <<= 1) {
                    const int y = __shfl_up_sync(0xffffffffu, x, off);
                    if (lane >= off) x += y;
                }
                if (c < nb) a.blkcnt[(size_t)c * E + e] = carry + x - v;
                carry += __shfl_sync(0xffffffffu, x, 31);
            }
            if (lane == 0) a.tot[e] = carry;
        }
        ok = permute_grid_barrier(a, 2 * parts, &s_flag);
    }
    if (!ok) {
        // a barrier ran out: the GEMMs get an empty tile list instead of a partial one
        if (blockIdx.x == 0 && tid == 0) a.status[kStNumMTiles] = 0u;
        pdl_trigger();
        return;
    }
    // phase 3: every block scans the totals (block 0 writes the results), then
    // scatters its chunks from their first free rows
    scan_experts(a, [&](int e) { return __ldcg(a.tot + e); }, s_off, s_pad, s_warp, blockIdx.x == 0);
    __syncthreads();
    for (int c = blockIdx.x; c < nb; c += parts) {
        int ids[kMaxTopK];
        load_token_ids(a, c * kTokPerBlk + tid, n, ids);
        for (int e = tid; e < E; e += kTokPerBlk) s_count[e] = s_off[e] + __ldcg(a.blkcnt + (size_t)c * E + e);
        __syncthreads();
        scatter_chunk(a, n, c * kTokPerBlk, ids, s_count, s_off, s_pad, masks, wbase);
    }
    pdl_trigger();
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
                                                                        uint8_t* __restrict__ xs,
                                                                        const unsigned* status) {
    __shared__ int s_prow[kMaxTopK];
    pdl_trigger();
    pdl_wait();
    const int n = live_rows(live, max_live, status);
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
                                                              int k, void* __restrict__ out, const unsigned* status) {
    __shared__ int s_prow[kMaxTopK];
    __shared__ float s_p[kMaxTopK];
    pdl_trigger();
    pdl_wait();
    const int n = live_rows(live, max_live, status);
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
    const int E = p->d.num_experts;
    PermuteArgs a;
    a.ids = r_ids;
    a.live = live;
    a.max_live = (int)p->max_live;
    a.E = E;
    a.k = p->d.top_k;
    a.tile_rows = p->tile_rows;
    a.row_align = p->row_align;
    a.blkcnt = blkcnt;
    a.tot = blkcnt + (size_t)p->nblk * E;  // the workspace's count area has E ints past the chunks'
    a.offsets = offsets;
    a.padoff = padoff;
    a.tiles = tiles;
    a.perm = perm;
    a.inv = inv;
    a.ready = ready;
    a.status = status_words;
    a.wait_limit_ns = kWaitLimitNs;
    const size_t smem = permute_smem_bytes(E);
    if (smem > 48 * 1024) {
        static int configured_device = -1;  // once per device, at the largest size any plan can ask for
        int dev = 0;
        cudaError_t err = cudaGetDevice(&dev);
        if (err != cudaSuccess) return err;
        if (configured_device != dev) {
            err = cudaFuncSetAttribute(route_permute_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)permute_smem_bytes(kMaxExperts));
            if (err != cudaSuccess) return err;
            configured_device = dev;
        }
    }
    // at most one block per SM: the blocks meet in grid-wide barriers
    int grid = p->nblk < num_sms() ? p->nblk : num_sms();
    if (grid < 1) grid = 1;
    return launch_dependent(route_permute_kernel, dim3((unsigned)grid), dim3(kTokPerBlk), smem, s, a);
}

cudaError_t launch_gather_mxfp8(const __nv_bfloat16* x, const int* live, int max_live, int H, int hp, int k,
                                const int* inv, uint8_t* xq, uint8_t* xs, const unsigned* status, cudaStream_t s) {
    const int grid = grid_for_warps(max_live, 1, 16);
    return launch_dependent(gather_rows_mxfp8_kernel, dim3(grid), dim3(kRowThreads), 0, s,
                            reinterpret_cast<const uint4*>(x), live, max_live, H, hp, k, hp / 128, inv,
                            reinterpret_cast<uint2*>(xq), xs, status);
}

cudaError_t launch_combine(const float* y, const int* inv, const float* probs, const int* live, int max_live,
                           int H, int k, void* out, bool out_bf16, const unsigned* status, cudaStream_t s) {
    const dim3 grid((unsigned)grid_for_warps((long long)max_live * ((H / 4 + kRowThreads - 1) / kRowThreads), 1, 16));
    if (out_bf16)
        return launch_dependent(combine_kernel<true>, grid, dim3(kRowThreads), 0, s,
                                reinterpret_cast<const float4*>(y), inv, probs, live, max_live, H, k, out, status);
    return launch_dependent(combine_kernel<false>, grid, dim3(kRowThreads), 0, s,
                            reinterpret_cast<const float4*>(y), inv, probs, live, max_live, H, k, out, status);
}

}  // namespace moe
