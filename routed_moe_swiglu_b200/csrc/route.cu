// route.cu -- router top-k and canonical route order.
//
// Router: "core.transformer.moe.training_matches_inference" API doc, `_route`
// ([tokens, topk] probabilities and expert ids); Megatron-LM PR #7830,
// "1. Mega backend for generation" (a token's expert ids are put in a
// canonical sorted order before the combine).  Per token: softmax over the
// E experts, the k largest (ties to the lower id), probabilities
// renormalised over the k, emitted in ascending expert id.
#include <cfloat>
#include <cmath>

#include "moe_internal.cuh"

namespace moe {
namespace {

// Order-preserving map of a logit to an unsigned key: a larger logit gives a
// larger key; -0 is taken as +0 and NaN as -infinity (a NaN never wins over a
// number).  Key 0 is below every logit and marks an absent or taken slot.
__device__ __forceinline__ uint32_t logit_key(float x) {
    if (x != x) x = -INFINITY;
    if (x == 0.0f) x = 0.0f;
    const uint32_t b = __float_as_uint(x);
    return (b & 0x80000000u) ? ~b : (b | 0x80000000u);
}
__device__ __forceinline__ float key_logit(uint32_t key) {
    return __uint_as_float((key & 0x80000000u) ? (key ^ 0x80000000u) : ~key);
}

// One warp per token.  Logit `id` lives in lane id % 32, slot id / 32;
// kSlots = ceil(E / 32) is a template parameter so the per-lane scans are
// fully unrolled over registers.  Each of the k rounds takes every lane's
// best untaken slot (the lower slot, i.e. the lower id, on equal keys), a
// warp max of the keys and a warp min of the ids holding that key: the
// largest logit, ties to the lower expert id.
template <int kSlots>
__global__ void __launch_bounds__(256) route_topk_kernel(const float* __restrict__ logits,
                                                         const int* __restrict__ live, int max_live, int E,
                                                         int k, int* __restrict__ ids,
                                                         float* __restrict__ probs, unsigned* status) {
    pdl_trigger();
    pdl_wait();
    int n = __ldg(live);
    if (status != nullptr && blockIdx.x == 0 && threadIdx.x == 0) {
        if (n < 0 || n > max_live) atomicOr(status, MOE_DEV_LIVE_CLAMPED);
        status[kStPermBar] = 0u;  // the permute that follows meets in barriers on this count
    }
    n = n < 0 ? 0 : (n > max_live ? max_live : n);

    const int lane = threadIdx.x & 31;
    const int warps_per_block = blockDim.x >> 5;
    for (int t = blockIdx.x * warps_per_block + (threadIdx.x >> 5); t < n; t += gridDim.x * warps_per_block) {
        const float* row = logits + (size_t)t * E;
        uint32_t key[kSlots];
#pragma unroll
        for (int s = 0; s < kSlots; ++s) {
            const int id = lane + 32 * s;
            key[s] = id < E ? logit_key(__ldg(row + id)) : 0u;
        }
        float first_v = 0.0f, my_v = 0.0f;
        int my_id = 0x7fffffff;
        for (int j = 0; j < k; ++j) {
            uint32_t best = 0u;
            int bs = 0;
#pragma unroll
            for (int s = 0; s < kSlots; ++s)
                if (key[s] > best) {
                    best = key[s];
                    bs = s;
                }
            const uint32_t wkey = __reduce_max_sync(0xffffffffu, best);
            const uint32_t wid = __reduce_min_sync(0xffffffffu, best == wkey ? (uint32_t)(lane + 32 * bs) : 0xffffffffu);
            if ((int)(wid & 31u) == lane) {
#pragma unroll
                for (int s = 0; s < kSlots; ++s)
                    if (s == (int)(wid >> 5)) key[s] = 0u;
            }
            const float bv = key_logit(wkey);
            if (j == 0) first_v = bv;
            if (j == lane) {
                my_v = bv;
                my_id = (int)wid;
            }
        }
        // Renormalised softmax over the chosen k: exp(l_j - max) / sum, in
        // double, summed in selection order (the same order in every lane).
        const double w = lane < k ? exp((double)my_v - (double)first_v) : 0.0;
        double z = 0.0;
        for (int j = 0; j < k; ++j) z += __shfl_sync(0xffffffffu, w, j);
        // rank of route j among the k in ascending expert id
        int rank = 0;
        for (int j = 0; j < k; ++j) {
            const int other = __shfl_sync(0xffffffffu, my_id, j);
            rank += other < my_id ? 1 : 0;
        }
        if (lane < k) {
            ids[(size_t)t * k + rank] = my_id;
            probs[(size_t)t * k + rank] = (float)(w / z);
        }
    }
}

// Caller-provided routes: sort each token's k (id, prob) pairs by id; a
// token with an id outside [0, E) or a repeated id is dropped (ids -1, its
// output row stays zero) and flagged.
__global__ void __launch_bounds__(256) canon_routes_kernel(const int* __restrict__ ids_in,
                                                           const float* __restrict__ probs_in,
                                                           const int* __restrict__ live, int max_live, int E,
                                                           int k, int* __restrict__ ids_out,
                                                           float* __restrict__ probs_out, unsigned* status) {
    pdl_trigger();
    pdl_wait();
    int n = __ldg(live);
    if (status != nullptr && blockIdx.x == 0 && threadIdx.x == 0) {
        if (n < 0 || n > max_live) atomicOr(status, MOE_DEV_LIVE_CLAMPED);
        status[kStPermBar] = 0u;  // the permute that follows meets in barriers on this count
    }
    n = n < 0 ? 0 : (n > max_live ? max_live : n);
    for (int t = blockIdx.x * blockDim.x + threadIdx.x; t < n; t += gridDim.x * blockDim.x) {
        int id[kMaxTopK];
        float p[kMaxTopK];
        bool bad = false;
        for (int j = 0; j < k; ++j) {
            id[j] = __ldg(ids_in + (size_t)t * k + j);
            p[j] = __ldg(probs_in + (size_t)t * k + j);
            if (id[j] < 0 || id[j] >= E) bad = true;
        }
        for (int a = 1; a < k; ++a) {
            const int ia = id[a];
            const float pa = p[a];
            int b = a - 1;
            while (b >= 0 && id[b] > ia) {
                id[b + 1] = id[b];
                p[b + 1] = p[b];
                --b;
            }
            id[b + 1] = ia;
            p[b + 1] = pa;
        }
        for (int j = 1; j < k; ++j)
            if (id[j] == id[j - 1]) bad = true;
        if (bad && status != nullptr) atomicOr(status, MOE_DEV_BAD_ROUTE);
        for (int j = 0; j < k; ++j) {
            ids_out[(size_t)t * k + j] = bad ? -1 : id[j];
            probs_out[(size_t)t * k + j] = bad ? 0.0f : p[j];
        }
    }
}

}  // namespace

cudaError_t launch_route_topk(const float* logits, const int* live, int max_live, int E, int k, int* ids,
                              float* probs, unsigned* status, cudaStream_t s) {
    const int warps = 8;
    long long blocks = ((long long)max_live + warps - 1) / warps;
    const long long cap = (long long)num_sms() * 16;
    if (blocks > cap) blocks = cap;
    if (blocks < 1) blocks = 1;
    const int slots = (E + 31) / 32;
    if (slots <= 4)
        return launch_dependent(route_topk_kernel<4>, dim3((unsigned)blocks), dim3(warps * 32), 0, s, logits, live,
                                max_live, E, k, ids, probs, status);
    else if (slots <= 8)
        return launch_dependent(route_topk_kernel<8>, dim3((unsigned)blocks), dim3(warps * 32), 0, s, logits, live,
                                max_live, E, k, ids, probs, status);
    else if (slots <= 16)
        return launch_dependent(route_topk_kernel<16>, dim3((unsigned)blocks), dim3(warps * 32), 0, s, logits, live,
                                max_live, E, k, ids, probs, status);
    else
        return launch_dependent(route_topk_kernel<32>, dim3((unsigned)blocks), dim3(warps * 32), 0, s, logits, live,
                                max_live, E, k, ids, probs, status);
}

cudaError_t launch_canon_routes(const int* ids_in, const float* probs_in, const int* live, int max_live, int E,
                                int k, int* ids_out, float* probs_out, unsigned* status, cudaStream_t s) {
    long long blocks = ((long long)max_live + 255) / 256;
    const long long cap = (long long)num_sms() * 8;
    if (blocks > cap) blocks = cap;
    if (blocks < 1) blocks = 1;
    return launch_dependent(canon_routes_kernel, dim3((unsigned)blocks), dim3(256), 0, s, ids_in, probs_in, live,
                            max_live, E, k, ids_out, probs_out, status);
}

}  // namespace moe
