// ep.cu -- expert-parallel dispatch: the send side of an all-to-all of route rows.
//
// Experts are split into ep_size equal contiguous ranges, range g owned by EP
// rank g.  A rank routes its own tokens and orders its routes by expert with
// the forward's permute (stable: by token within an expert), so the routes
// bound for rank g are one contiguous run of that order.  This kernel packs
// each route's x row into a send buffer at its place in that run, with the
// route's expert id local to the owning rank, and counts the rows per
// destination.  The owning rank computes each received row as a top-1 token
// with probability 1.0 (or the route's probability when it is applied in
// FC1), so it returns the route's expert output as is (Megatron-LM PR #7798,
// "What is changed": expert compute over all dispatched rows, each a top-1
// token with probability 1.0).  Back on the source rank the combine adds a
// token's routes in ascending expert id as fp32 FMAs from zero, the same
// chain as the one-GPU forward, so the output does not depend on the EP size
// (the same PR's "Limitations" names generation's combine, which adds rank
// partials, as not EP-invariant).
#include "ep.cuh"
#include "moe_internal.cuh"

namespace moe {
namespace {

constexpr int kPackThreads = 128;  // also the largest EP size (one count per thread of block 0)

// One block per live token (strided): the block loads the token's x row once
// in 16-byte chunks and stores it to the send row of each of its routes.
__global__ void __launch_bounds__(kPackThreads) ep_pack_kernel(
    const uint4* __restrict__ x, const int* __restrict__ live, int max_live, int chunks, int k,
    const int* __restrict__ r_ids, const float* __restrict__ r_probs, const int* __restrict__ inv,
    const int* __restrict__ offsets, const int* __restrict__ padoff, int E, int ep_size, int probs_in_fc1,
    uint4* __restrict__ send_x, int* __restrict__ send_ids, float* __restrict__ send_probs,
    int* __restrict__ send_counts, int* __restrict__ route_rows, float* __restrict__ route_probs,
    const unsigned* status) {
    __shared__ int s_row[kMaxTopK];
    pdl_trigger();
    pdl_wait();
    const bool poisoned = forward_poisoned(status);  // a partial permutation sends nothing
    const int n = poisoned ? 0 : clamp_live(live, max_live);
    const int el = E / ep_size;  // experts per EP rank
    if (blockIdx.x == 0 && (int)threadIdx.x < ep_size)
        send_counts[threadIdx.x] = poisoned ? 0 : offsets[(threadIdx.x + 1) * el] - offsets[threadIdx.x * el];
    for (int t = blockIdx.x; t < n; t += gridDim.x) {
        __syncthreads();
        if ((int)threadIdx.x < k) {
            const size_t idx = (size_t)t * k + threadIdx.x;
            const int e = r_ids[idx];
            int row = -1;
            float p_combine = 0.0f;
            if (e >= 0) {
                // the route's padded row in the forward's layout, less its expert's padding
                row = inv[idx] - padoff[e] + offsets[e];
                const float p = r_probs[idx];
                send_ids[row] = e - (e / el) * el;
                send_probs[row] = probs_in_fc1 ? p : 1.0f;
                p_combine = probs_in_fc1 ? 1.0f : p;
            }
            route_rows[idx] = row;
            route_probs[idx] = p_combine;
            s_row[threadIdx.x] = row;
        }
        __syncthreads();
        for (int c = threadIdx.x; c < chunks; c += blockDim.x) {
            const uint4 v = __ldg(x + (size_t)t * chunks + c);
            for (int j = 0; j < k; ++j) {
                const int row = s_row[j];
                if (row >= 0) send_x[(size_t)row * chunks + c] = v;
            }
        }
    }
}

}  // namespace

int ep_max_size() { return kPackThreads; }

cudaError_t launch_ep_pack(const void* x, const int* live, int max_live, int H, int k, const int* r_ids,
                           const float* r_probs, const int* inv, const int* offsets, const int* padoff, int E,
                           int ep_size, bool probs_in_fc1, void* send_x, int* send_ids, float* send_probs,
                           int* send_counts, int* route_rows, float* route_probs, const unsigned* status,
                           cudaStream_t s) {
    long long blocks = max_live;
    const long long cap = (long long)num_sms() * 16;
    if (blocks > cap) blocks = cap;
    if (blocks < 1) blocks = 1;
    return launch_dependent(ep_pack_kernel, dim3((unsigned)blocks), dim3(kPackThreads), 0, s,
                            static_cast<const uint4*>(x), live, max_live, H * 2 / 16, k, r_ids, r_probs, inv, offsets,
                            padoff, E, ep_size, probs_in_fc1 ? 1 : 0, static_cast<uint4*>(send_x), send_ids,
                            send_probs, send_counts, route_rows, route_probs, status);
}

}  // namespace moe
