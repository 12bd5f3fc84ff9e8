// noalloc.cu -- moe_forward_noalloc: the forward for callers that cannot
// allocate device memory.
//
// Some callers are handed only their input and output pointers and have no
// allocator to call: a plug-in running inside another engine's memory
// budget, code that must not call cudaMalloc because it would synchronise
// the device or fail under a pool-less stream capture, or firmware-like
// hosts with a fixed memory map.  For them the forward's scratch (routes,
// permutation, tile list, intermediate rows, status word) lives in one
// file-scope device array of fixed size that the CUDA runtime places when it
// loads this module; this entry point calls no cudaMalloc, cudaFree or any
// other allocating routine.
#include <mutex>

#include "moe_internal.cuh"

namespace {

// The scratch every call of moe_forward_noalloc uses (MOE_NOALLOC_SCRATCH_BYTES).
static_assert(MOE_NOALLOC_SCRATCH_BYTES % 256 == 0, "scratch size");
__device__ __align__(256) unsigned char g_noalloc_scratch[MOE_NOALLOC_SCRATCH_BYTES];

// Device address of g_noalloc_scratch per device, looked up with that device
// current (in host code the array's name is only a host-side handle).  Outside
// stream capture every call looks it up again, so the address stays right
// after a cudaDeviceReset reloads the module; under capture (where a lookup
// that loads the module is not allowed) the address the last call outside
// capture found is used.
void* g_scratch_addr[64];
std::mutex g_scratch_mu;

moe_status scratch_address(cudaStream_t s, void** out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return MOE_ERR_CUDA;
    cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
    const bool capturing = cudaStreamIsCapturing(s, &cs) != cudaSuccess || cs != cudaStreamCaptureStatusNone;
    std::lock_guard<std::mutex> lock(g_scratch_mu);
    if (!capturing || g_scratch_addr[dev] == nullptr) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr) return MOE_ERR_CUDA;
        g_scratch_addr[dev] = p;
    }
    *out = g_scratch_addr[dev];
    return MOE_OK;
}

}  // namespace

extern "C" moe_status moe_forward_noalloc(const moe_plan* plan, const void* x, const float* logits, const int* ids,
                                          const float* probs, const void* kernel_buf, const int* live_count_dev,
                                          void* out, void* stream) {
    if (plan == nullptr) return MOE_ERR_INVALID_ARG;
    if (plan->ws.total > (size_t)MOE_NOALLOC_SCRATCH_BYTES) return MOE_ERR_WORKSPACE_TOO_SMALL;
    void* scratch = nullptr;
    const moe_status st = scratch_address(static_cast<cudaStream_t>(stream), &scratch);
    if (st != MOE_OK) return st;
    // the sticky status word is the only scratch that must start at zero
    if (cudaMemsetAsync(scratch, 0, sizeof(unsigned), static_cast<cudaStream_t>(stream)) != cudaSuccess)
        return MOE_ERR_CUDA;
    return moe_forward(plan, x, logits, ids, probs, kernel_buf, live_count_dev, out, scratch,
                       (size_t)MOE_NOALLOC_SCRATCH_BYTES, stream);
}
