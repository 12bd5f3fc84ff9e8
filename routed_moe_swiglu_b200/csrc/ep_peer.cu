// ep_peer.cu -- the expert-parallel exchange through peer memory: rows are
// stored straight into the owning rank's receive region (over NVLink between
// GPUs), with no host read of split sizes, so one CUDA graph can capture a
// whole EP step.
//
// Megatron-LM PR #7830 puts the EP transport inside the expert kernels;
// Megatron-LM PR #7798, "Performance", prices the NCCL all-to-all path and
// its host sync for split sizes.  Here every rank owns one region (laid out
// by ep_region_layout) that every peer maps:
//   - a receive slot per source rank (x rows, local expert ids, FC1 weights),
//     filled by that source's pack kernel with plain 16-byte stores, with a
//     row count, the source's first send row and an epoch flag per source;
//   - the y rows of the rank's own routes as the owners return them, with a
//     return flag per owner;
//   - local state: the step's epoch, arrival counters, the status word, and
//     the compacted received rows the expert forward reads.
// A flag is stored (release, system scope) by the last block of the kernel
// that wrote the rows, after every block fenced its stores at system scope;
// the reader waits (acquire, system scope, bounded) until each flag equals
// the step's epoch.  No TMA touches peer memory.
//
// Reuse across steps needs no more flags: a source's next dispatch follows,
// in its stream, its combine, which saw every owner's return flag; an owner
// returns rows only after its forward has read its receive slots.
#include "ep.cuh"
#include "moe_internal.cuh"
#include "ptx.cuh"

namespace moe {
namespace {

constexpr int kPeerThreads = 128;

__device__ __forceinline__ unsigned ld_acquire_sys_u32(const unsigned* p) {
    unsigned v;
    asm volatile("ld.acquire.sys.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}
__device__ __forceinline__ void st_release_sys_u32(unsigned* p, unsigned v) {
    asm volatile("st.release.sys.global.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}

__device__ __forceinline__ unsigned* hdr(void* region) { return static_cast<unsigned*>(region); }

// The last block of a grid to arrive on `counter` (a local word, left at 0)
// returns true, after every block's earlier stores were fenced at system scope.
__device__ __forceinline__ bool last_block_arrives(unsigned* counter, int* s_last) {
    __syncthreads();
    if (threadIdx.x == 0) {
        __threadfence_system();
        const unsigned old = atomicAdd(counter, 1u);
        const bool last = old == gridDim.x - 1;
        if (last) {
            *counter = 0u;
            __threadfence_system();
        }
        *s_last = last ? 1 : 0;
    }
    __syncthreads();
    return *s_last != 0;
}

// Step 1 (source side), after the forward's route and permute: every live
// route's x row, local expert id and FC1 weight into its owner's slot for
// this source, at the route's place in the owner's run; the route's send row
// and combine weight for the combine; then the counts and, from the last
// block, the epoch flags.
__global__ void __launch_bounds__(kPeerThreads) ep_peer_pack_kernel(
    const uint4* __restrict__ x, const int* __restrict__ live, int max_live, int chunks, int k,
    const int* __restrict__ r_ids, const float* __restrict__ r_probs, const int* __restrict__ inv,
    const int* __restrict__ offsets, const int* __restrict__ padoff, int E, int ep_size, int rank,
    int probs_in_fc1, void* const* __restrict__ regions, EpRegionLayout lay, int* __restrict__ route_rows,
    float* __restrict__ route_probs, const unsigned* ws_status) {
    __shared__ int s_row[kMaxTopK];
    __shared__ int s_dst[kMaxTopK];
    __shared__ int s_last;
    pdl_trigger();
    pdl_wait();
    unsigned* own = hdr(regions[rank]);
    const unsigned epoch = own[kEpEpoch] + 1u;
    const bool poisoned = forward_poisoned(ws_status);  // a partial permutation sends nothing
    const int n = poisoned ? 0 : clamp_live(live, max_live);
    const int el = E / ep_size;
    if (blockIdx.x == 0 && (int)threadIdx.x < ep_size) {
        const int g = threadIdx.x;
        unsigned* dst = hdr(regions[g]);
        dst[kEpInCount + rank] = poisoned ? 0u : (unsigned)(offsets[(g + 1) * el] - offsets[g * el]);
        dst[kEpInBase + rank] = poisoned ? 0u : (unsigned)offsets[g * el];
    }
    for (int t = blockIdx.x; t < n; t += gridDim.x) {
        __syncthreads();
        if ((int)threadIdx.x < k) {
            const size_t idx = (size_t)t * k + threadIdx.x;
            const int e = r_ids[idx];
            int send_row = -1, g = -1, r = -1;
            float p_combine = 0.0f;
            if (e >= 0) {
                send_row = inv[idx] - padoff[e] + offsets[e];  // in this rank's expert order
                g = e / el;
                r = send_row - offsets[g * el];  // its place in owner g's run
                uint8_t* slot = static_cast<uint8_t*>(regions[g]) + lay.slots + (size_t)rank * lay.slot_bytes;
                const float p = r_probs[idx];
                reinterpret_cast<int*>(slot + lay.slot_ids)[r] = e - g * el;
                reinterpret_cast<float*>(slot + lay.slot_probs)[r] = probs_in_fc1 ? p : 1.0f;
                p_combine = probs_in_fc1 ? 1.0f : p;
            }
            route_rows[idx] = send_row;
            route_probs[idx] = p_combine;
            s_row[threadIdx.x] = r;
            s_dst[threadIdx.x] = g;
        }
        __syncthreads();
        for (int c = threadIdx.x; c < chunks; c += blockDim.x) {
            const uint4 v = __ldg(x + (size_t)t * chunks + c);
            for (int j = 0; j < k; ++j) {
                if (s_row[j] < 0) continue;
                uint8_t* slot =
                    static_cast<uint8_t*>(regions[s_dst[j]]) + lay.slots + (size_t)rank * lay.slot_bytes;
                reinterpret_cast<uint4*>(slot + lay.slot_x)[(size_t)s_row[j] * chunks + c] = v;
            }
        }
    }
    if (last_block_arrives(own + kEpPackDone, &s_last)) {
        if (threadIdx.x == 0) own[kEpEpoch] = epoch;
        for (int g = threadIdx.x; g < ep_size; g += blockDim.x)
            st_release_sys_u32(hdr(regions[g]) + kEpInFlag + rank, epoch);
    }
}

// Wait (bounded) until flags[0 .. n) all equal the step's epoch; on expiry
// set MOE_DEV_TIMEOUT in the region's status word (the kernels after it then
// do no work).
__global__ void __launch_bounds__(32) ep_peer_wait_kernel(void* region, int flag_word, int n,
                                                          unsigned long long limit_ns) {
    pdl_trigger();
    pdl_wait();
    if (threadIdx.x != 0) return;
    unsigned* h = hdr(region);
    const unsigned epoch = h[kEpEpoch];
    const unsigned long long t0 = global_timer_ns();
    for (int s = 0; s < n; ++s) {
        while (ld_acquire_sys_u32(h + flag_word + s) != epoch) {
            if (global_timer_ns() - t0 > limit_ns) {
                atomicOr(h + kEpStatus, MOE_DEV_TIMEOUT);
                return;
            }
            __nanosleep(64);
        }
    }
    __threadfence_system();
}

// Step 2 (owner side), after the wait: the rows of every source's slot, in
// source order, into the contiguous rows the expert forward reads; each
// row's (source, send row) for the return; the live row count.
__global__ void __launch_bounds__(kPeerThreads) ep_peer_compact_kernel(void* region, int ep_size, int chunks,
                                                                     EpRegionLayout lay) {
    __shared__ int s_pre[kEpMaxRanks + 1];
    pdl_trigger();
    pdl_wait();
    uint8_t* base = static_cast<uint8_t*>(region);
    unsigned* h = hdr(region);
    const bool poisoned = forward_poisoned(h + kEpStatus);
    if (threadIdx.x == 0) {
        int acc = 0;
        for (int s = 0; s < ep_size; ++s) {
            s_pre[s] = acc;
            acc += poisoned ? 0 : (int)h[kEpInCount + s];
        }
        s_pre[ep_size] = acc;
    }
    __syncthreads();
    const int total = s_pre[ep_size];
    if (blockIdx.x == 0 && threadIdx.x == 0) reinterpret_cast<int*>(h)[kEpRecvLive] = total;
    uint4* rx = reinterpret_cast<uint4*>(base + lay.recv_x);
    int* rid = reinterpret_cast<int*>(base + lay.recv_ids);
    float* rp = reinterpret_cast<float*>(base + lay.recv_probs);
    int2* map = reinterpret_cast<int2*>(base + lay.src_map);
    for (int i = blockIdx.x; i < total; i += gridDim.x) {
        int s = 0;
        while (s + 1 < ep_size && s_pre[s + 1] <= i) ++s;
        const int r = i - s_pre[s];
        const uint8_t* slot = base + lay.slots + (size_t)s * lay.slot_bytes;
        const uint4* src = reinterpret_cast<const uint4*>(slot + lay.slot_x) + (size_t)r * chunks;
        for (int c = threadIdx.x; c < chunks; c += blockDim.x) rx[(size_t)i * chunks + c] = __ldcg(src + c);
        if (threadIdx.x == 0) {
            rid[i] = __ldcg(reinterpret_cast<const int*>(slot + lay.slot_ids) + r);
            rp[i] = __ldcg(reinterpret_cast<const float*>(slot + lay.slot_probs) + r);
            map[i] = make_int2(s, (int)h[kEpInBase + s] + r);
        }
    }
}

// Step 4 (owner side), after the expert forward: each received row's y into
// its source's y_back at the route's send row; then, from the last block,
// the return flags of every source.
__global__ void __launch_bounds__(kPeerThreads) ep_peer_return_kernel(void* const* __restrict__ regions, int rank,
                                                                    int ep_size, int ychunks, EpRegionLayout lay) {
    __shared__ int s_last;
    pdl_trigger();
    pdl_wait();
    uint8_t* base = static_cast<uint8_t*>(regions[rank]);
    unsigned* h = hdr(regions[rank]);
    const unsigned epoch = h[kEpEpoch];
    const bool poisoned = forward_poisoned(h + kEpStatus);
    const int total = poisoned ? 0 : reinterpret_cast<const int*>(h)[kEpRecvLive];
    const int2* map = reinterpret_cast<const int2*>(base + lay.src_map);
    const uint4* ry = reinterpret_cast<const uint4*>(base + lay.recv_y);
    for (int i = blockIdx.x; i < total; i += gridDim.x) {
        const int2 m = map[i];
        uint4* dst = reinterpret_cast<uint4*>(static_cast<uint8_t*>(regions[m.x]) + lay.y_back) +
                     (size_t)m.y * ychunks;
        for (int c = threadIdx.x; c < ychunks; c += blockDim.x) dst[c] = ry[(size_t)i * ychunks + c];
    }
    // a rank whose wait ran out returns nothing and raises no flag: its sources' waits run
    // out too, so every rank of the step reports MOE_DEV_TIMEOUT instead of a partial result
    if (last_block_arrives(h + kEpReturnDone, &s_last) && !poisoned)
        for (int g = threadIdx.x; g < ep_size; g += blockDim.x)
            st_release_sys_u32(hdr(regions[g]) + kEpRetFlag + rank, epoch);
}

long long peer_grid(long long items) {
    const long long cap = (long long)num_sms() * 8;
    if (items > cap) items = cap;
    return items < 1 ? 1 : items;
}

}  // namespace

EpRegionLayout ep_region_layout(int H, int max_live, int k, int ep_size) {
    auto al = [](size_t v) { return (v + 255) & ~size_t(255); };
    EpRegionLayout l{};
    const size_t max_send = (size_t)max_live * (size_t)k;  // routes one source can send one owner
    const size_t recv = max_send * (size_t)ep_size;
    size_t off = 0;
    l.hdr = off;
    off += al(kEpHeaderWords * 4);
    l.slot_x = 0;
    l.slot_ids = al(max_send * (size_t)H * 2);
    l.slot_probs = l.slot_ids + al(max_send * 4);
    l.slot_bytes = l.slot_probs + al(max_send * 4);
    l.slots = off;
    off += l.slot_bytes * (size_t)ep_size;
    l.y_back = off;
    off += al(max_send * (size_t)H * 4);
    l.recv_x = off;
    off += al(recv * (size_t)H * 2);
    l.recv_ids = off;
    off += al(recv * 4);
    l.recv_probs = off;
    off += al(recv * 4);
    l.recv_y = off;
    off += al(recv * (size_t)H * 4);
    l.src_map = off;
    off += al(recv * 8);
    l.total = off;
    l.max_send = (long long)max_send;
    return l;
}

cudaError_t launch_ep_peer_pack(const void* x, const int* live, int max_live, int H, int k, const int* r_ids,
                                const float* r_probs, const int* inv, const int* offsets, const int* padoff, int E,
                                int ep_size, int rank, bool probs_in_fc1, void* const* regions,
                                const EpRegionLayout& lay, int* route_rows, float* route_probs,
                                const unsigned* ws_status, cudaStream_t s) {
    return launch_dependent(ep_peer_pack_kernel, dim3((unsigned)peer_grid(max_live)), dim3(kPeerThreads), 0, s,
                            static_cast<const uint4*>(x), live, max_live, H * 2 / 16, k, r_ids, r_probs, inv,
                            offsets, padoff, E, ep_size, rank, probs_in_fc1 ? 1 : 0, regions, lay, route_rows,
                            route_probs, ws_status);
}

cudaError_t launch_ep_peer_receive(void* region, int ep_size, int H, const EpRegionLayout& lay,
                                   unsigned long long wait_limit_ns, cudaStream_t s) {
    cudaError_t e = launch_dependent(ep_peer_wait_kernel, dim3(1), dim3(32), 0, s, region, (int)kEpInFlag, ep_size,
                                     wait_limit_ns);
    if (e != cudaSuccess) return e;
    return launch_dependent(ep_peer_compact_kernel, dim3((unsigned)peer_grid(lay.max_send * ep_size)),
                            dim3(kPeerThreads), 0, s, region, ep_size, H * 2 / 16, lay);
}

cudaError_t launch_ep_peer_return(void* const* regions, void* own_region, int rank, int ep_size, int H,
                                  const EpRegionLayout& lay, cudaStream_t s) {
    (void)own_region;  // read on the device as regions[rank]
    return launch_dependent(ep_peer_return_kernel, dim3((unsigned)peer_grid(lay.max_send * ep_size)),
                            dim3(kPeerThreads), 0, s, regions, rank, ep_size, H * 4 / 16, lay);
}

cudaError_t launch_ep_peer_wait_returns(void* region, int ep_size, unsigned long long wait_limit_ns,
                                        cudaStream_t s) {
    return launch_dependent(ep_peer_wait_kernel, dim3(1), dim3(32), 0, s, region, (int)kEpRetFlag, ep_size,
                            wait_limit_ns);
}

}  // namespace moe
