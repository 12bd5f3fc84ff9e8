// ep.cuh -- host launchers of the expert-parallel send side (ep.cu).
#pragma once
#include <cuda_runtime.h>

#include <cstddef>

namespace moe {

// Largest EP size the pack kernel supports (one count per thread of its first block).
int ep_max_size();

// After the forward's route and permute: the x row of every live route into
// send_x in expert order, the local expert id and FC1 weight of each row, the
// rows per destination rank, and each route's send row and combine weight.
cudaError_t launch_ep_pack(const void* x, const int* live, int max_live, int H, int k, const int* r_ids,
                           const float* r_probs, const int* inv, const int* offsets, const int* padoff, int E,
                           int ep_size, bool probs_in_fc1, void* send_x, int* send_ids, float* send_probs,
                           int* send_counts, int* route_rows, float* route_probs, const unsigned* status,
                           cudaStream_t s);

// ---------------------------------------------------------------- peer-memory exchange (ep_peer.cu)

// Words of the header at the start of every rank's EP region (uint32).
// Local to the owner: kEpStatus (MOE_DEV_* bits), kEpEpoch (the step the
// rank last dispatched), kEpPackDone / kEpReturnDone (arrival counters, left
// at 0), kEpRecvLive (int: rows received this step).  Written by peers:
// kEpInFlag + s, kEpInCount + s, kEpInBase + s (from source s's dispatch:
// epoch, rows, first send row) and kEpRetFlag + g (from owner g's return).
constexpr int kEpMaxRanks = 128;
enum : int {
    kEpStatus = 0,
    kEpEpoch = 1,
    kEpPackDone = 2,
    kEpReturnDone = 3,
    kEpRecvLive = 4,
    kEpInFlag = 64,
    kEpInCount = kEpInFlag + kEpMaxRanks,
    kEpInBase = kEpInCount + kEpMaxRanks,
    kEpRetFlag = kEpInBase + kEpMaxRanks,
    kEpHeaderWords = kEpRetFlag + kEpMaxRanks
};

// Byte offsets of one rank's EP region (the same on every rank of a step).
struct EpRegionLayout {
    size_t hdr;
    size_t slots;        // ep_size receive slots, one per source rank
    size_t slot_bytes;   // bytes of one slot: x [max_send][H] bf16, ids [max_send], FC1 weights [max_send]
    size_t slot_x, slot_ids, slot_probs;  // offsets inside a slot
    size_t y_back;       // fp32 [max_send][H]: this rank's routes' y rows, at their send rows
    size_t recv_x, recv_ids, recv_probs, recv_y, src_map;  // local: rows received this step, compacted
    size_t total;
    long long max_send;  // max_live * k: the most routes one source sends one owner
};
EpRegionLayout ep_region_layout(int H, int max_live, int k, int ep_size);

cudaError_t launch_ep_peer_pack(const void* x, const int* live, int max_live, int H, int k, const int* r_ids,
                                const float* r_probs, const int* inv, const int* offsets, const int* padoff, int E,
                                int ep_size, int rank, bool probs_in_fc1, void* const* regions,
                                const EpRegionLayout& lay, int* route_rows, float* route_probs,
                                const unsigned* ws_status, cudaStream_t s);
cudaError_t launch_ep_peer_receive(void* region, int ep_size, int H, const EpRegionLayout& lay,
                                   unsigned long long wait_limit_ns, cudaStream_t s);
cudaError_t launch_ep_peer_return(void* const* regions, void* own_region, int rank, int ep_size, int H,
                                  const EpRegionLayout& lay, cudaStream_t s);
cudaError_t launch_ep_peer_wait_returns(void* region, int ep_size, unsigned long long wait_limit_ns,
                                        cudaStream_t s);

}  // namespace moe
