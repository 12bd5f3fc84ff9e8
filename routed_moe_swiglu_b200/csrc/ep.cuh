// ep.cuh -- host launchers of the expert-parallel send side (ep.cu).
#pragma once
#include <cuda_runtime.h>

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

}  // namespace moe
