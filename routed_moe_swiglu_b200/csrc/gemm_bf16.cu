// gemm_bf16.cu -- the two grouped expert GEMMs in bf16 on the 5th-generation
// tensor cores (tcgen05, accumulators in TMEM, operands staged by TMA).
//
//   gate/up:  for an M tile of 128 route rows of expert e (rows of the
//             permuted x) and an N tile of 128 f values, one MMA of
//             M=128 x N=256 x K=16 per 16 K elements: B rows 0..127 are
//             W_gate[e, f0:f0+128, :], rows 128..255 W_up[e, f0:f0+128, :].
//             The epilogue reads gate and up of the same f from TMEM columns
//             c and 128+c, forms h = silu(g) * u and stores it as bf16
//             (Megatron-LM PR #7798, "Background": the activation is fused
//             into the FC1 epilogue).
//   down:     A = h rows, B = W_down[e, c0:c0+256, :], fp32 y rows out
//             (probabilities are applied later, in the combine).
//
// One persistent CTA per SM, 6 warps: warp 0 issues TMA loads, warp 1 owns
// TMEM and issues the MMAs (one thread), warps 2-5 drain the accumulators.
// Tiles are walked in a static round-robin order; every tile does the same
// amount of MMA work, so the walk is balanced whatever the expert loads.
// Two accumulator buffers of 256 fp32 columns (512 TMEM columns) let the
// epilogue of tile i overlap the MMAs of tile i+1.
//
// Every row's result depends only on that row of A and on the weights, with
// one instruction shape and one K order for every tile, so a route's output
// does not depend on which tile, how many rows or which live count it came
// with.
#include "moe_internal.cuh"
#include "ptx.cuh"

namespace moe {
namespace {

constexpr int kStages = 4;
constexpr int kThreads = 192;
constexpr int kABoxRows = 32;                           // A is loaded in 32-row boxes, only as many as needed
constexpr uint32_t kABytes = kBM * kBK * 2;             // 16 KB per stage
constexpr uint32_t kABoxBytes = kABoxRows * kBK * 2;    // 4 KB
constexpr uint32_t kBBytes = 256 * kBK * 2;             // 32 KB per stage
constexpr uint32_t kAccCols = 256;                      // fp32 columns per accumulator buffer
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kStageOutBytes = 32 * 128;           // one 32-row x 128-byte output box
constexpr uint32_t kOutBytes = 4 * 2 * kStageOutBytes;  // 4 epilogue warps x 2 buffers
constexpr size_t kSmemBytes = 1024 /*alignment slack*/ + kStages * (kABytes + kBBytes) + kOutBytes + 256 /*barriers*/;

struct __align__(8) Barriers {
    uint64_t full[kStages];
    uint64_t empty[kStages];
    uint64_t acc_full[2];
    uint64_t acc_empty[2];
    uint64_t done;
    uint32_t tmem_base;
    int abort_flag;
};

__device__ __forceinline__ float silu_f(float g) {
    // silu(g) = g / (1 + e^-g); for very negative g, e^-g overflows to inf and
    // the reciprocal gives 0, so silu -> -0.
    return g * __frcp_rn(1.0f + __expf(-g));
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
    const __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<const uint32_t*>(&v);
}

template <int kMode>  // 0: gate/up + SwiGLU -> bf16 h;  1: down -> fp32 y
__device__ __forceinline__ void grouped_gemm_body(const CUtensorMap& tmA, const CUtensorMap& tmB,
                                                  const CUtensorMap& tmOut, const GemmParams& p) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t* sA = smem;
    uint8_t* sB = smem + kStages * kABytes;
    uint8_t* sOut = sB + kStages * kBBytes;  // 1024-aligned
    Barriers* bars = reinterpret_cast<Barriers*>(sOut + kOutBytes);
    volatile int* abort_flag = &bars->abort_flag;

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;

    if (threadIdx.x == 0) {
        for (int s = 0; s < kStages; ++s) {
            mbar_init(&bars->full[s], 1);
            mbar_init(&bars->empty[s], 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&bars->acc_full[b], 1);
            mbar_init(&bars->acc_empty[b], 4);  // one arrival per epilogue warp
        }
        mbar_init(&bars->done, 1);
        bars->abort_flag = 0;
        fence_barrier_init();
    }
    if (warp == 1) {
        tmem_alloc(&bars->tmem_base, kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before_sync();
    __syncthreads();
    tc_fence_after_sync();
    const uint32_t tmem_base = bars->tmem_base;

    const int num_m = (int)p.status_words[kStNumMTiles];
    const int total_tiles = num_m * p.n_tiles;
    const int kb_count = p.k_blocks;

    if (warp == 0) {
        if (lane == 0) {
            // ---------------- TMA producer
            tma_prefetch_desc(&tmA);
            tma_prefetch_desc(&tmB);
            int stage = 0;
            uint32_t phase = 0;
            bool ok = true;
            int last_phase[kStages];
            for (int s = 0; s < kStages; ++s) last_phase[s] = -1;
            for (int t = blockIdx.x; t < total_tiles && ok; t += gridDim.x) {
                const int mt = t / p.n_tiles, nt = t - mt * p.n_tiles;
                const int4 ti = __ldg(p.tiles + mt);
                const int n_abox = (ti.z + kABoxRows - 1) / kABoxRows;
                const uint32_t tx = (uint32_t)n_abox * kABoxBytes + kBBytes;
                for (int kb = 0; kb < kb_count; ++kb) {
                    if (!mbar_wait_bounded(&bars->empty[stage], phase ^ 1u, abort_flag, p.wait_limit_ns)) {
                        ok = false;
                        break;
                    }
                    mbar_arrive_expect_tx(&bars->full[stage], tx);
                    last_phase[stage] = (int)phase;
                    uint8_t* a_dst = sA + stage * kABytes;
                    for (int i = 0; i < n_abox; ++i)
                        tma_load_2d(a_dst + i * kABoxBytes, &tmA, &bars->full[stage], kb * kBK, ti.y + i * kABoxRows);
                    uint8_t* b_dst = sB + stage * kBBytes;
                    if (kMode == 0) {
                        // B rows 0..127: gate, 128..255: up, same f range
                        tma_load_4d(b_dst, &tmB, &bars->full[stage], kb * kBK, nt * kG1BN, 0, ti.x);
                        tma_load_4d(b_dst + kBBytes / 2, &tmB, &bars->full[stage], kb * kBK, nt * kG1BN, 1, ti.x);
                    } else {
                        tma_load_3d(b_dst, &tmB, &bars->full[stage], kb * kBK, nt * kG2BN, ti.x);
                    }
                    if (++stage == kStages) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
            }
            if (!ok) {
                *abort_flag = 1;
                atomicOr(p.status_flags, MOE_DEV_TIMEOUT);
                // let copies already issued land before the CTA's shared memory goes away
                for (int s = 0; s < kStages; ++s)
                    if (last_phase[s] >= 0) {
                        volatile int never = 0;
                        (void)mbar_wait_bounded(&bars->full[s], (uint32_t)last_phase[s], &never, 100000000ull);
                    }
            }
        }
        __syncwarp();
    } else if (warp == 1) {
        if (lane == 0) {
            // ---------------- MMA issuer
            constexpr uint32_t idesc = idesc_bf16_f32(128, 256);
            int stage = 0;
            uint32_t phase = 0;
            bool ok = true;
            int it = 0;
            for (int t = blockIdx.x; t < total_tiles && ok; t += gridDim.x, ++it) {
                const int buf = it & 1;
                const uint32_t acc_phase = (uint32_t)(it >> 1) & 1u;
                if (!mbar_wait_bounded(&bars->acc_empty[buf], acc_phase ^ 1u, abort_flag, p.wait_limit_ns)) {
                    ok = false;
                    break;
                }
                tc_fence_after_sync();
                const uint32_t d_tmem = tmem_base + (uint32_t)buf * kAccCols;
                for (int kb = 0; kb < kb_count; ++kb) {
                    if (!mbar_wait_bounded(&bars->full[stage], phase, abort_flag, p.wait_limit_ns)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after_sync();
                    const uint32_t a_addr = smem_u32(sA + stage * kABytes);
                    const uint32_t b_addr = smem_u32(sB + stage * kBBytes);
#pragma unroll
                    for (int kk = 0; kk < kBK / 16; ++kk) {
                        mma_bf16_ss(d_tmem, sdesc_kmajor_sw128(a_addr + kk * 32), sdesc_kmajor_sw128(b_addr + kk * 32),
                                    idesc, (kb | kk) != 0 ? 1u : 0u);
                    }
                    mma_commit(&bars->empty[stage]);  // frees the stage once these MMAs have read it
                    if (++stage == kStages) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
                if (!ok) break;
                mma_commit(&bars->acc_full[buf]);
            }
            if (!ok) {
                *abort_flag = 1;
                atomicOr(p.status_flags, MOE_DEV_TIMEOUT);
            }
            // all MMAs issued by this thread complete before TMEM is released
            mma_commit(&bars->done);
            volatile int never = 0;
            (void)mbar_wait_bounded(&bars->done, 0, &never, 100000000ull);
        }
        __syncwarp();
    } else {
        // ---------------- epilogue: warps 2..5, TMEM lane quadrant = warp % 4
        const int quad = warp & 3;
        const int r = quad * 32 + lane;  // row inside the tile
        int it = 0;
        uint32_t out_chunk = 0;  // output boxes this warp has staged (mode 1)
        for (int t = blockIdx.x; t < total_tiles; t += gridDim.x, ++it) {
            const int buf = it & 1;
            const uint32_t acc_phase = (uint32_t)(it >> 1) & 1u;
            const int mt = t / p.n_tiles, nt = t - mt * p.n_tiles;
            const int4 ti = __ldg(p.tiles + mt);
            // the decision to go on must be warp-uniform: tcgen05.ld is a warp-wide instruction
            const bool got = __all_sync(0xffffffffu,
                                        mbar_wait_bounded(&bars->acc_full[buf], acc_phase, abort_flag, p.wait_limit_ns));
            if (!got) {
                if (lane == 0) {
                    *abort_flag = 1;
                    atomicOr(p.status_flags, MOE_DEV_TIMEOUT);
                }
                break;
            }
            tc_fence_after_sync();
            const bool valid = r < ti.z;
            const uint32_t taddr = tmem_base + ((uint32_t)(quad * 32) << 16) + (uint32_t)buf * kAccCols;
            if (kMode == 0) {
                __nv_bfloat16* out_row =
                    reinterpret_cast<__nv_bfloat16*>(p.out) + (size_t)(ti.y + r) * (size_t)p.out_ld;
#pragma unroll 1
                for (int c = 0; c < kG1BN / 32; ++c) {
                    uint32_t g[32], u[32];
                    tmem_ld_32x32b_x32(taddr + c * 32, g);
                    tmem_ld_32x32b_x32(taddr + kG1BN + c * 32, u);
                    tmem_ld_wait();
                    const int f0 = nt * kG1BN + c * 32;
                    if (valid) {
#pragma unroll
                        for (int q = 0; q < 4; ++q) {
                            if (f0 + q * 8 < p.out_cols) {
                                uint32_t w[4];
#pragma unroll
                                for (int i = 0; i < 4; ++i) {
                                    const int a = q * 8 + 2 * i;
                                    const float h0 = silu_f(__uint_as_float(g[a])) * __uint_as_float(u[a]);
                                    const float h1 = silu_f(__uint_as_float(g[a + 1])) * __uint_as_float(u[a + 1]);
                                    w[i] = pack_bf16x2(h0, h1);
                                }
                                *reinterpret_cast<uint4*>(out_row + f0 + q * 8) = make_uint4(w[0], w[1], w[2], w[3]);
                            }
                        }
                    }
                }
            } else {
                // fp32 rows leave through shared memory: each warp stages its 32 rows x 32
                // columns in the 128-byte-swizzled box layout and one lane issues a TMA
                // store.  Only warps whose 32-row slice holds valid rows store; rows past
                // the expert's count inside a slice land in its own padding rows.
                const bool slice_live = quad * 32 < ti.z;
                uint8_t* my_out = sOut + (size_t)quad * 2 * kStageOutBytes;
#pragma unroll 1
                for (int c = 0; c < kG2BN / 32; ++c) {
                    uint32_t v[32];
                    tmem_ld_32x32b_x32(taddr + c * 32, v);
                    tmem_ld_wait();
                    const int c0 = nt * kG2BN + c * 32;
                    if (slice_live && c0 < p.out_cols) {
                        uint8_t* box = my_out + (out_chunk & 1) * kStageOutBytes;
                        if (lane == 0) bulk_wait_group_read<1>();  // the store that used this buffer has read it
                        __syncwarp();
#pragma unroll
                        for (int q = 0; q < 8; ++q) {
                            const uint32_t off = (uint32_t)lane * 128u + (uint32_t)((q ^ (lane & 7)) * 16);
                            *reinterpret_cast<uint4*>(box + off) = make_uint4(v[q * 4], v[q * 4 + 1], v[q * 4 + 2], v[q * 4 + 3]);
                        }
                        fence_proxy_async_smem();
                        __syncwarp();
                        if (lane == 0) {
                            tma_store_2d(&tmOut, box, c0, ti.y + quad * 32);
                            bulk_commit_group();
                        }
                        ++out_chunk;
                    }
                }
            }
            tc_fence_before_sync();
            __syncwarp();
            if (lane == 0) mbar_arrive(&bars->acc_empty[buf]);
        }
        if (kMode == 1 && lane == 0) bulk_wait_group<0>();  // stores complete before the CTA exits
        __syncwarp();
    }

    // ---------------- teardown: every role is done (or gave up); free TMEM
    tc_fence_before_sync();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after_sync();
        tmem_dealloc(tmem_base, kTmemCols);
    }
}

// Distinct names so profilers can tell the two GEMMs apart.
__global__ void __launch_bounds__(kThreads, 1)
    moe_gemm_gate_up_swiglu_bf16(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                                 const __grid_constant__ CUtensorMap tmOut, const GemmParams p) {
    grouped_gemm_body<0>(tmA, tmB, tmOut, p);
}

__global__ void __launch_bounds__(kThreads, 1)
    moe_gemm_down_bf16(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                       const __grid_constant__ CUtensorMap tmOut, const GemmParams p) {
    grouped_gemm_body<1>(tmA, tmB, tmOut, p);
}

using GemmKernel = void (*)(CUtensorMap, CUtensorMap, CUtensorMap, GemmParams);

cudaError_t launch_impl(GemmKernel kern, int* configured_device, const CUtensorMap& a, const CUtensorMap& b,
                        const CUtensorMap& o, const GemmParams& gp, int grid, cudaStream_t s) {
    int dev = 0;
    cudaError_t err = cudaGetDevice(&dev);
    if (err != cudaSuccess) return err;
    if (*configured_device != dev) {
        err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kSmemBytes);
        if (err != cudaSuccess) return err;
        *configured_device = dev;
    }
    kern<<<grid, kThreads, kSmemBytes, s>>>(a, b, o, gp);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_gemm1_bf16(const CUtensorMap& a, const CUtensorMap& b, const CUtensorMap& o, const GemmParams& gp,
                              int grid, cudaStream_t s) {
    static int configured = -1;
    return launch_impl(moe_gemm_gate_up_swiglu_bf16, &configured, a, b, o, gp, grid, s);
}

cudaError_t launch_gemm2_bf16(const CUtensorMap& a, const CUtensorMap& b, const CUtensorMap& o, const GemmParams& gp,
                              int grid, cudaStream_t s) {
    static int configured = -1;
    return launch_impl(moe_gemm_down_bf16, &configured, a, b, o, gp, grid, s);
}

}  // namespace moe
