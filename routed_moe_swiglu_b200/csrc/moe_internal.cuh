// moe_internal.cuh -- shared definitions of the routed-MoE library: tile
// constants, the plan, the workspace / weight-buffer layouts and the
// launchers each .cu file provides.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cstddef>
#include <cstdint>
#include <utility>

#include "moe.h"

namespace moe {

// ---------------------------------------------------------------- tiling
constexpr int kBM = 128;           // MXFP8: routes per M tile (and the row alignment of its scale blocks)
constexpr int kBK = 64;            // bf16 K elements per pipeline stage (128-byte rows)
constexpr int kBK8 = 128;          // E4M3 K elements per pipeline stage (128-byte rows)
constexpr int kG1BN = 128;         // bf16: f values per gate/up weight tile (256 weight rows, gate and up)
constexpr int kG2BN = 256;         // bf16: output columns per down weight tile
constexpr int kRouteTile = 256;    // bf16: most routes per tile (N of a pair MMA)
constexpr int kRouteAlign = 32;    // bf16: route rows of an expert start on a multiple of this
constexpr int kGatherInGemmMax = 32;  // bf16: route tiles of at most this many routes read x rows by token
constexpr int kCopyChunk = 8;         // bf16: routes per chunk the gate/up GEMM's copy warps claim
constexpr int kChunksPerTile = kRouteTile / kCopyChunk;
constexpr int kG1BN8 = 64;         // MXFP8: f values per gate/up tile (64 gate + 64 up MMA columns)
constexpr int kG2BN8 = 128;        // MXFP8: output columns per down tile
constexpr int kSfBlock = 512;      // MXFP8 scales of 128 rows x 4 k-groups, [row%32][row/32][k-group]
constexpr int kTokPerBlk = 256;    // tokens per histogram / scatter block
constexpr int kMaxTopK = 16;
constexpr int kMaxExperts = 1024;

// Status word layout (uint32 words at the start of the workspace).
// kStPermBar: arrivals at the permute's grid-wide barriers, zeroed by the router kernel
// (route or canonicalise) that precedes the permute in every forward.  kStMaxTileRows:
// the most routes in one route tile of this forward (the GEMMs size their pipelines by it).
// kStTileStarted: the highest route tile a bf16 gate/up producer has started (zeroed with
// the tile list); the copy warps stay a bounded distance ahead of it.
enum : int {
    kStFlags = 0,
    kStNumMTiles = 1,
    kStTotalRoutes = 2,
    kStCopyNext = 3,
    kStPermBar = 4,
    kStMaxTileRows = 5,
    kStTileStarted = 6,
    kStWords = 64
};

// Default bound of any on-device wait before the kernel gives up (ns).
constexpr unsigned long long kWaitLimitNs = 4000000000ull;

struct WsLayout {
    size_t status, r_ids, r_probs, blkcnt, offsets, padoff, tiles, perm, inv, ready;
    size_t xq, xs, h, hs, y;
    size_t xg, hf, hg;  // NVFP4: per-row scales of x and h; the fp32 h rows (NVFP4, or MXFP8 keeping them)
    size_t total;
};

struct WbufLayout {
    size_t w1, w1s, w2, w2s;
    size_t wg;  // NVFP4: second-level scales [E][2] (W1, W2)
    size_t total;
};

}  // namespace moe

struct moe_plan {
    moe_desc d;
    long long max_live;
    long long max_routes;   // max_live * k
    long long max_m_tiles;  // upper bound on route tiles: ceil(routes / tile_rows) + E
    long long rows_pad;     // rows of the padded intermediates (an upper bound on the padded route space)
    int nblk;               // ceil(max_live / kTokPerBlk)
    int tile_rows;          // most routes per tile: 256 (bf16, N of a pair MMA) or 128 (MXFP8, M of the MMA)
    int row_align;          // each expert's route rows start on a multiple of this: 32 (bf16) or 128 (MXFP8)
    long long hp, fp;       // K row pitch (elements) of x / gate-up rows and of h / down rows:
                            // H and F padded to multiples of 128 with zeros
    long long hr;           // bf16: rows of an expert's down weights, H padded to 128 with zero rows
    long long w1r;          // bf16: rows of an expert's FC1 weights: 2 * fp (gate and up interleaved),
                            // or fp rounded up to 256 (squared-ReLU experts), zero rows past F
    int ks1, ks2;           // K blocks of 128 elements of the gate/up and down GEMMs
    int nt1, nt2;           // weight (bf16) / N (MXFP8) tiles of the gate/up and down GEMMs
    moe::WsLayout ws;
    moe::WbufLayout wb;
};

namespace moe {

// Tensor maps of one route-row operand with several box heights, so that a
// tile of N routes loads its rows with one TMA instruction: bf16 (CTA pairs)
// entry i has 16 * (i + 1) rows (N/2 per CTA), MXFP8 entry i < 4 has
// 32 * (i + 1) rows.
struct BoxMaps8 {
    CUtensorMap m[8];
};

struct GemmParams {
    const int4* tiles;              // {expert, first padded row, valid rows, first permuted row} per route tile
    const unsigned* status_words;   // [kStNumMTiles] = number of M tiles
    unsigned* status_flags;         // sticky MOE_DEV_* bits
    void* out;                      // h (bf16 / E4M3) or y (fp32)
    uint8_t* out_scales;            // E8M0 scales of h (MXFP8), else null
    long long out_ld;               // row stride of out, elements
    int out_cols;                   // valid output columns (F or H)
    int n_tiles;                    // weight tiles per route tile
    int k_blocks;                   // pipeline stages per tile
    long long a_rows;               // bf16: weight rows of one expert (a multiple of 128)
    unsigned long long wait_limit_ns;
    // MXFP8 only: scale blocks of A, the weights ([expert][weight tile][K stage][512 B]),
    // and of B, the route rows ([128-row tile][K stage][512 B]); K stages of the down
    // GEMM (the gate/up epilogue writes h's scales for it).
    const uint8_t* sfa;
    const uint8_t* sfb;
    int sf_ks_out;
    // bf16 gate/up: the B rows are gathered from x by token, route r of the
    // permuted order being token perm[r] / top_k
    const int* perm;
    int top_k;
    // gate/up epilogue variants: route_probs (canonical [max_live, k], or null)
    // scales each route's SwiGLU row by its probability; clamp > 0 clamps the
    // gate and up pre-activations to [-clamp, clamp]
    const float* route_probs;
    float clamp;
    int relu2;                      // bf16 gate/up GEMM: squared-ReLU experts (A = one FC1 projection)
    // bf16 gate/up: the copy warps write the x rows of tiles of more than
    // kGatherInGemmMax routes into their padded route rows xg (pitch xg_pitch
    // bytes, zeros from x_bytes to the pitch), counting each 32-route chunk in
    // ready[tile]; copy_next (zeroed with the tile list) hands out the chunks
    const uint8_t* x;
    long long x_pitch;              // bytes between x rows
    int x_bytes;                    // bytes of one x row (H * 2)
    uint8_t* xg;
    long long xg_pitch;
    int* ready;
    unsigned* copy_next;
    int* tile_started;              // highest route tile whose loads a producer has started
    // NVFP4: second-level scales of the B rows (fp32 per padded route row: x for the
    // gate/up GEMM, h for the down GEMM) and of the weights ([E][2]: W1, W2)
    const float* row_scale;
    const float* w_scale;
    // MXFP8 gate/up, plans with MOE_FLAG_KEEP_H_FP32 (else null): the fp32 h values the
    // epilogue quantises, stored at the codes' positions (pitch out_ld)
    float* h_fp32;
};

// ---------------------------------------------------------------- launchers
int num_sms();
bool get_tensor_map_encoder();
bool make_tensor_map(CUtensorMap* map, CUtensorMapDataType dtype, int rank, const void* base,
                     const unsigned long long* dims, const unsigned long long* strides_bytes,
                     const unsigned* box, CUtensorMapSwizzle swizzle);

cudaError_t launch_route_topk(const float* logits, const int* live, int max_live, int E, int k, int* ids,
                              float* probs, unsigned* status, cudaStream_t s);
cudaError_t launch_canon_routes(const int* ids_in, const float* probs_in, const int* live, int max_live, int E,
                                int k, int* ids_out, float* probs_out, unsigned* status, cudaStream_t s);
// ready (bf16 only, else null): one counter per route tile, zeroed with the
// tile list; the gate/up GEMM's copy warps count the tile's copied chunks in it
cudaError_t launch_permute(const moe_plan* p, const int* live, int* r_ids, int* blkcnt, int* offsets,
                           int* padoff, int4* tiles, int* perm, int* inv, int* ready, unsigned* status_words,
                           cudaStream_t s);
// status (the workspace's status words, or null) on the launchers below: see forward_poisoned()
cudaError_t launch_gather_mxfp8(const __nv_bfloat16* x, const int* live, int max_live, int H, int hp, int k,
                                const int* inv, uint8_t* xq, uint8_t* xs, const unsigned* status, cudaStream_t s);
// probs null: every route's weight is 1 (the probabilities were applied in FC1);
// out_bf16: out is bf16 (the fp32 sum rounded to nearest even), else fp32
cudaError_t launch_combine(const float* y, const int* inv, const float* probs, const int* live, int max_live,
                           int H, int k, void* out, bool out_bf16, const unsigned* status, cudaStream_t s);
cudaError_t launch_gemm1_bf16_pair(const CUtensorMap& a, const CUtensorMap& x_rows, const BoxMaps8& b,
                                   const GemmParams& gp, long long max_tiles, cudaStream_t s);
cudaError_t launch_gemm2_bf16_pair(const CUtensorMap& a, const BoxMaps8& b, const GemmParams& gp, long long max_tiles,
                                   cudaStream_t s);
cudaError_t launch_gemm1_mxfp8(const CUtensorMap& a, const BoxMaps8& b, const GemmParams& gp, long long max_tiles,
                               cudaStream_t s);
cudaError_t launch_gemm2_mxfp8(const CUtensorMap& a, const BoxMaps8& b, const GemmParams& gp, long long max_tiles,
                               cudaStream_t s);
cudaError_t launch_gemm1_nvfp4(const CUtensorMap& a, const BoxMaps8& b, const GemmParams& gp, long long max_tiles,
                               cudaStream_t s);
cudaError_t launch_gemm2_nvfp4(const CUtensorMap& a, const BoxMaps8& b, const GemmParams& gp, long long max_tiles,
                               cudaStream_t s);
cudaError_t launch_nvfp4_quantize_rows(const __nv_bfloat16* in, long long rows, int cols, long long ld_in,
                                       uint8_t* q, uint8_t* scales, float* g, const int* live_rows, cudaStream_t s);
cudaError_t launch_gather_nvfp4(const __nv_bfloat16* x, const int* live, int max_live, int H, int hp, int k,
                                const int* inv, uint8_t* xq, uint8_t* xs, float* xg, const unsigned* status,
                                cudaStream_t s);
cudaError_t launch_quantize_h_nvfp4(const float* hf, const int* live, int max_live, int k, int fp, const int* inv,
                                    uint8_t* hq, uint8_t* hs, float* hg, const unsigned* status, cudaStream_t s);
cudaError_t launch_prepare_nvfp4(const moe_plan* p, const __nv_bfloat16* wg, const __nv_bfloat16* wu,
                                 const __nv_bfloat16* wd, void* buf, cudaStream_t s);
cudaError_t launch_prepare_bf16(const moe_plan* p, const __nv_bfloat16* wg, const __nv_bfloat16* wu,
                                const __nv_bfloat16* wd, void* buf, cudaStream_t s);
cudaError_t launch_prepare_mxfp8(const moe_plan* p, const __nv_bfloat16* wg, const __nv_bfloat16* wu,
                                 const __nv_bfloat16* wd, void* buf, cudaStream_t s);
cudaError_t launch_quantize_rows(const __nv_bfloat16* in, long long rows, int cols, long long ld_in, uint8_t* q,
                                 uint8_t* scales, const int* live_rows, cudaStream_t s);

// ---------------------------------------------------------------- dependent launches
// Every kernel of the forward is launched with programmatic stream
// serialisation: it may be scheduled while its predecessor in the stream is
// still running, does its set-up (barriers, TMEM, descriptor prefetch), and
// waits in pdl_wait() until the predecessor has completed and its writes are
// visible before reading anything another kernel (or the caller) produced.
// pdl_trigger() lets the next kernel be scheduled; it changes no ordering
// of memory, so each kernel issues it first thing.
__device__ __forceinline__ void pdl_trigger() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

template <class... KArgs, class... Args>
cudaError_t launch_dependent(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t s,
                             Args&&... args) {
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    const cudaError_t err = cudaLaunchKernelEx(&cfg, kern, std::forward<Args>(args)...);
    return err != cudaSuccess ? err : cudaGetLastError();
}

// Byte offset of (row within a 128-row tile, k-group within a 4-group K
// stage) inside one 512-byte MXFP8 scale block.
__host__ __device__ __forceinline__ uint32_t sf_block_offset(int row, int kg) {
    return (uint32_t)((row & 31) * 16 + ((row >> 5) & 3) * 4 + kg);
}

__device__ __forceinline__ int clamp_live(const int* live, int max_live) {
    int n = __ldg(live);
    return n < 0 ? 0 : (n > max_live ? max_live : n);
}

// Whether a bounded wait of this forward (or of an earlier one on the same
// workspace, until the word is cleared) gave up: the permutation may then be
// partial, so the kernels after it do no work rather than index memory
// through it.  status: the workspace's status words (null: not checked).
__device__ __forceinline__ bool forward_poisoned(const unsigned* status) {
    return status != nullptr && (*status & MOE_DEV_TIMEOUT) != 0u;
}
__device__ __forceinline__ int live_rows(const int* live, int max_live, const unsigned* status) {
    return forward_poisoned(status) ? 0 : clamp_live(live, max_live);
}

}  // namespace moe
