// gemm_mxfp8.cu -- the two grouped expert GEMMs in MXFP8 (E4M3 operands with
// one E8M0 scale per 32 K elements per row), block-scaled tcgen05 MMAs with
// the scale factors in TMEM.
//
// Megatron-LM PR #7798, "Background": the FC1 epilogue fuses the activation
// and the FC2-input quantisation; probabilities are applied after FC2.
// Megatron-LM PR #7830 / cudnn-frontend PR #448: MXFP8 blocks are 32
// elements along K.
//
//   gate/up:  M tile = 128 route rows, N tile = 64 f values (B rows 0..63
//             W_gate[e, f0:f0+64], rows 64..127 W_up[e, f0:f0+64]), K stage
//             = 128 E4M3 elements = 4 MMAs of K=32.  The epilogue forms
//             h = silu(g) * u in fp32 and re-quantises it to MXFP8 (blocks of
//             32 along F): E4M3 codes to h, E8M0 bytes straight into the
//             scale layout the down GEMM reads.
//   down:     A = h codes + scales, B = W_down[e, c0:c0+128], fp32 y out.
//
// Scale factors: for each 128-row operand tile and K stage, 512 bytes laid
// out as [row % 32][row / 32][k-group] (16 bytes per 32-row lane group),
// which one tcgen05.cp (32x128b, replicated to the 4 lane quarters) moves to
// 4 TMEM columns; MMA k-group kk selects byte kk of each 32-bit cell.  Both
// the weights (at prepare time) and the activations (gather, epilogue) are
// written in that layout, so a stage's scales arrive with one bulk copy.
//
// Pipeline as in the bf16 kernel: persistent CTA per SM, warp 0 TMA,
// warp 1 MMA + TMEM owner, warps 2-5 epilogue; 5 stages; two 128-column
// accumulators; one scale-factor TMEM slot per stage (a slot is rewritten
// only after the MMAs that read it have completed, which the producer's wait
// on that stage's "empty" barrier already implies).
#include "moe_internal.cuh"
#include "mxfp8.cuh"
#include "ptx.cuh"

namespace moe {
namespace {

constexpr int kStages = 5;
constexpr int kThreads = 192;
constexpr int kBN = 128;                               // MMA N (both GEMMs)
constexpr int kABoxRows = 32;
constexpr uint32_t kABytes = kBM * kBK8;               // 16 KB
constexpr uint32_t kABoxBytes = kABoxRows * kBK8;      // 4 KB
constexpr uint32_t kBBytes = kBN * kBK8;               // 16 KB
constexpr uint32_t kSfBytes = kSfBlock;
constexpr uint32_t kStageBytes = kABytes + kBBytes + 2 * kSfBytes;
constexpr uint32_t kAccCols = kBN;
constexpr uint32_t kSfCol0 = 2 * kAccCols;             // first scale-factor column
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kStageOutBytes = 32 * 128;
constexpr uint32_t kOutBytes = 4 * 2 * kStageOutBytes;
constexpr size_t kSmemBytes = 1024 + kStages * kStageBytes + kOutBytes + 256;
static_assert(kSfCol0 + 16 * kStages <= kTmemCols, "TMEM budget");

struct __align__(8) Barriers {
    uint64_t full[kStages];
    uint64_t empty[kStages];
    uint64_t acc_full[2];
    uint64_t acc_empty[2];
    uint64_t done;
    uint32_t tmem_base;
    int abort_flag;
};

__host__ __device__ constexpr uint32_t idesc_mxf8(int M, int N, uint32_t sfa_id, uint32_t sfb_id) {
    return (sfb_id << 4)                   // B scale-factor byte
           | (0u << 7) | (0u << 10)        // A, B: E4M3
           | ((uint32_t)(N >> 3) << 17)    // N / 8
           | (1u << 23)                    // scale type: E8M0
           | ((uint32_t)(M >> 4) << 24)    // M / 16
           | (sfa_id << 29);               // A scale-factor byte
}

// Descriptor of a 32-row x 16-byte scale block in shared memory (no
// swizzle; 8-row groups 128 bytes apart) as the source of tcgen05.cp.
__device__ __forceinline__ uint64_t sdesc_sf(uint32_t saddr) {
    uint64_t d = 0;
    d |= (uint64_t)((saddr & 0x3FFFFu) >> 4);
    d |= (uint64_t)(128u >> 4) << 32;  // stride byte offset
    d |= (uint64_t)1u << 46;           // descriptor version
    return d;                          // layout type 0: no swizzle
}

__device__ __forceinline__ void bulk_load(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
    asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
                     smem_u32(dst)),
                 "l"(src), "r"(bytes), "r"(smem_u32(bar))
                 : "memory");
}

__device__ __forceinline__ float silu_f(float g) { return g * __frcp_rn(1.0f + __expf(-g)); }


template <int kMode>  // 0: gate/up + SwiGLU -> MXFP8 h;  1: down -> fp32 y
__device__ __forceinline__ void gemm_mxfp8_body(const CUtensorMap& tmA, const CUtensorMap& tmB,
                                                const CUtensorMap& tmOut, const GemmParams& p) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t* sOut = smem + kStages * kStageBytes;  // 1024-aligned (kStageBytes is a multiple of 1024)
    Barriers* bars = reinterpret_cast<Barriers*>(sOut + kOutBytes);
    volatile int* abort_flag = &bars->abort_flag;
    auto stage_a = [&](int s) { return smem + s * kStageBytes; };
    auto stage_b = [&](int s) { return smem + s * kStageBytes + kABytes; };
    auto stage_sfa = [&](int s) { return smem + s * kStageBytes + kABytes + kBBytes; };
    auto stage_sfb = [&](int s) { return smem + s * kStageBytes + kABytes + kBBytes + kSfBytes; };

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;

    if (threadIdx.x == 0) {
        for (int s = 0; s < kStages; ++s) {
            mbar_init(&bars->full[s], 1);
            mbar_init(&bars->empty[s], 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&bars->acc_full[b], 1);
            mbar_init(&bars->acc_empty[b], 4);
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
                const uint32_t tx = (uint32_t)n_abox * kABoxBytes + kBBytes + 2 * kSfBytes;
                const uint8_t* sfa_src = p.sfa + ((size_t)(ti.y / kBM) * kb_count) * kSfBytes;
                const uint8_t* sfb_src = p.sfb + ((size_t)ti.x * p.n_tiles + nt) * kb_count * kSfBytes;
                for (int kb = 0; kb < kb_count; ++kb) {
                    if (!mbar_wait_bounded(&bars->empty[stage], phase ^ 1u, abort_flag, p.wait_limit_ns)) {
                        ok = false;
                        break;
                    }
                    mbar_arrive_expect_tx(&bars->full[stage], tx);
                    last_phase[stage] = (int)phase;
                    for (int i = 0; i < n_abox; ++i)
                        tma_load_2d(stage_a(stage) + i * kABoxBytes, &tmA, &bars->full[stage], kb * kBK8,
                                    ti.y + i * kABoxRows);
                    if (kMode == 0) {
                        tma_load_4d(stage_b(stage), &tmB, &bars->full[stage], kb * kBK8, nt * (kBN / 2), 0, ti.x);
                        tma_load_4d(stage_b(stage) + kBBytes / 2, &tmB, &bars->full[stage], kb * kBK8, nt * (kBN / 2),
                                    1, ti.x);
                    } else {
                        tma_load_3d(stage_b(stage), &tmB, &bars->full[stage], kb * kBK8, nt * kBN, ti.x);
                    }
                    bulk_load(stage_sfa(stage), sfa_src + (size_t)kb * kSfBytes, kSfBytes, &bars->full[stage]);
                    bulk_load(stage_sfb(stage), sfb_src + (size_t)kb * kSfBytes, kSfBytes, &bars->full[stage]);
                    if (++stage == kStages) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
            }
            if (!ok) {
                *abort_flag = 1;
                atomicOr(p.status_flags, MOE_DEV_TIMEOUT);
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
                    const uint32_t sfa_t = tmem_base + kSfCol0 + (uint32_t)stage * 16u;
                    const uint32_t sfb_t = sfa_t + 8u;
                    tmem_cp_32x128b_warpx4(sfa_t, sdesc_sf(smem_u32(stage_sfa(stage))));
                    tmem_cp_32x128b_warpx4(sfb_t, sdesc_sf(smem_u32(stage_sfb(stage))));
                    const uint32_t a_addr = smem_u32(stage_a(stage));
                    const uint32_t b_addr = smem_u32(stage_b(stage));
#pragma unroll
                    for (int kk = 0; kk < kBK8 / 32; ++kk) {
                        mma_mxf8_ss(d_tmem, sdesc_kmajor_sw128(a_addr + kk * 32), sdesc_kmajor_sw128(b_addr + kk * 32),
                                    idesc_mxf8(128, kBN, (uint32_t)kk, (uint32_t)kk), sfa_t, sfb_t,
                                    (kb | kk) != 0 ? 1u : 0u);
                    }
                    mma_commit(&bars->empty[stage]);
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
            mma_commit(&bars->done);
            volatile int never = 0;
            (void)mbar_wait_bounded(&bars->done, 0, &never, 100000000ull);
        }
        __syncwarp();
    } else {
        // ---------------- epilogue: warps 2..5, TMEM lane quadrant = warp % 4
        const int quad = warp & 3;
        const int r = quad * 32 + lane;
        int it = 0;
        uint32_t out_chunk = 0;
        for (int t = blockIdx.x; t < total_tiles; t += gridDim.x, ++it) {
            const int buf = it & 1;
            const uint32_t acc_phase = (uint32_t)(it >> 1) & 1u;
            const int mt = t / p.n_tiles, nt = t - mt * p.n_tiles;
            const int4 ti = __ldg(p.tiles + mt);
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
                uint8_t* h_row = reinterpret_cast<uint8_t*>(p.out) + (size_t)(ti.y + r) * (size_t)p.out_ld;
                uint8_t* hs_tile = p.out_scales + (size_t)(ti.y / kBM) * p.sf_ks_out * kSfBytes;
#pragma unroll 1
                for (int c = 0; c < 2; ++c) {
                    uint32_t g[32], u[32];
                    tmem_ld_32x32b_x32(taddr + c * 32, g);
                    tmem_ld_32x32b_x32(taddr + kBN / 2 + c * 32, u);
                    tmem_ld_wait();
                    const int f0 = nt * (kBN / 2) + c * 32;  // one MXFP8 block of h
                    float h[32];
                    float amax = 0.0f;
#pragma unroll
                    for (int i = 0; i < 32; ++i) {
                        h[i] = silu_f(__uint_as_float(g[i])) * __uint_as_float(u[i]);
                        amax = fmaxf(amax, fabsf(h[i]));
                    }
                    float inv;
                    const uint8_t sbyte = mxfp8_block_scale(amax, &inv);
                    if (valid) {
                        if (f0 < p.out_cols) {
                            uint32_t w[8];
#pragma unroll
                            for (int i = 0; i < 8; ++i)
                                w[i] = e4m3x2(h[4 * i + 1] * inv, h[4 * i] * inv) |
                                       (e4m3x2(h[4 * i + 3] * inv, h[4 * i + 2] * inv) << 16);
                            *reinterpret_cast<uint4*>(h_row + f0) = make_uint4(w[0], w[1], w[2], w[3]);
                            *reinterpret_cast<uint4*>(h_row + f0 + 16) = make_uint4(w[4], w[5], w[6], w[7]);
                        }
                        hs_tile[(size_t)(f0 / 128) * kSfBytes + sf_block_offset(r, (f0 % 128) / 32)] = sbyte;
                    }
                }
                // k-group slots of the down GEMM's last K stage that no gate/up tile covers hold scale 0
                if (valid && nt == p.n_tiles - 1) {
                    for (int g = 2 * p.n_tiles; g < 4 * p.sf_ks_out; ++g)
                        hs_tile[(size_t)(g / 4) * kSfBytes + sf_block_offset(r, g % 4)] = 0;
                }
            } else {
                const bool slice_live = quad * 32 < ti.z;
                uint8_t* my_out = sOut + (size_t)quad * 2 * kStageOutBytes;
#pragma unroll 1
                for (int c = 0; c < kBN / 32; ++c) {
                    uint32_t v[32];
                    tmem_ld_32x32b_x32(taddr + c * 32, v);
                    tmem_ld_wait();
                    const int c0 = nt * kBN + c * 32;
                    if (slice_live && c0 < p.out_cols) {
                        uint8_t* box = my_out + (out_chunk & 1) * kStageOutBytes;
                        if (lane == 0) bulk_wait_group_read<1>();
                        __syncwarp();
#pragma unroll
                        for (int q = 0; q < 8; ++q) {
                            const uint32_t off = (uint32_t)lane * 128u + (uint32_t)((q ^ (lane & 7)) * 16);
                            *reinterpret_cast<uint4*>(box + off) =
                                make_uint4(v[q * 4], v[q * 4 + 1], v[q * 4 + 2], v[q * 4 + 3]);
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
        if (kMode == 1 && lane == 0) bulk_wait_group<0>();
        __syncwarp();
    }

    tc_fence_before_sync();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after_sync();
        tmem_dealloc(tmem_base, kTmemCols);
    }
}

__global__ void __launch_bounds__(kThreads, 1)
    moe_gemm_gate_up_swiglu_mxfp8(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                                  const __grid_constant__ CUtensorMap tmOut, const GemmParams p) {
    gemm_mxfp8_body<0>(tmA, tmB, tmOut, p);
}

__global__ void __launch_bounds__(kThreads, 1)
    moe_gemm_down_mxfp8(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                        const __grid_constant__ CUtensorMap tmOut, const GemmParams p) {
    gemm_mxfp8_body<1>(tmA, tmB, tmOut, p);
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

cudaError_t launch_gemm1_mxfp8(const CUtensorMap& a, const CUtensorMap& b, const CUtensorMap& o,
                               const GemmParams& gp, int grid, cudaStream_t s) {
    static int configured = -1;
    return launch_impl(moe_gemm_gate_up_swiglu_mxfp8, &configured, a, b, o, gp, grid, s);
}

cudaError_t launch_gemm2_mxfp8(const CUtensorMap& a, const CUtensorMap& b, const CUtensorMap& o,
                               const GemmParams& gp, int grid, cudaStream_t s) {
    static int configured = -1;
    return launch_impl(moe_gemm_down_mxfp8, &configured, a, b, o, gp, grid, s);
}

}  // namespace moe
