// gemm_bf16_pair.cu -- the two grouped expert GEMMs in bf16, each tile
// computed by a pair of CTAs on two SMs with one tcgen05 MMA (cta_group::2).
//
//   gate/up:  M tile = 256 route rows of expert e (CTA r holds rows
//             128r..128r+127), N = 256: B rows 0..127 = W_gate[e, f0:f0+128]
//             in CTA 0's shared memory, rows 128..255 = W_up[e, f0:f0+128] in
//             CTA 1's.  Each CTA's TMEM receives its 128 rows x 256 columns,
//             so gate and up of one f sit in columns c and 128+c of the same
//             row; the epilogue forms h = silu(g) * u and stores bf16
//             (Megatron-LM PR #7798, "Background": the activation is fused
//             into the FC1 epilogue).
//   down:     A = h rows, B rows = W_down[e, c0:c0+256] (128 per CTA), fp32 y
//             rows out through a shared-memory transpose and coalesced stores.
//
// Each CTA loads half of B (the other half feeds the same MMA from the peer),
// so per SM and MMA FLOP the operand traffic is 2/3 of a one-CTA 128x256
// tile.  Issuing a TMA copy costs the producer thread on the order of a
// hundred cycles at these rates, so a K stage is 128 elements (two 128-byte
// swizzle atoms, 8 MMAs) and each operand of a stage is one 32 KB box: a
// 3-D (A) or 4-/5-D (B) tensor map whose third dimension walks the atoms of
// a row (the K row pitch of every bf16 operand buffer is padded to 128 with
// zeros).  A CTA with fewer than 128 valid rows (decode: a few routes per
// expert) loads only the 32-row boxes that hold valid rows.
//
// Roles (10 warps per CTA): warp 0 issues TMA loads in both CTAs (the
// completion of both halves is counted on CTA 0's "full" barrier); warp 1
// owns TMEM in both CTAs and, in CTA 0 only, issues the pair MMAs, whose
// completion is signalled to both CTAs' barriers (commit with a CTA mask);
// warps 2-9 drain the accumulators (lane quarter warp % 4, column half
// (warp - 2) / 4) and release each accumulator on CTA 0's barrier.
// Two accumulators of 256 fp32 columns (512 TMEM columns) per CTA.
//
// Every wait is bounded; the pair meets in cluster barriers only at start-up
// and before TMEM is released.  Each output row depends only on its own A row
// with one instruction shape and K order, so results do not depend on the
// tile a row lands in or on the live count.
#include "moe_internal.cuh"
#include "ptx.cuh"

namespace moe {
namespace {

// Pipeline depth per mode: the gate/up epilogue stores h straight from
// registers, so its shared memory all goes to stages; the down epilogue keeps
// one 4 KB transpose box per epilogue warp.
constexpr int kStagesGateUp = 3;
constexpr int kStagesDown = 3;
constexpr int kThreads = 320;
constexpr int kEpiWarps = 8;
constexpr int kPairRows = 256;                          // M of the pair tile
constexpr int kAtoms = 2;                               // 64-element (128-byte) swizzle atoms per K stage
constexpr int kStageK = kAtoms * kBK;                   // 128 K elements per stage
constexpr uint32_t kAtomBytes = 128 * kBK * 2;          // 16 KB: 128 rows x 128 bytes
constexpr int kABoxRows = 32;
constexpr uint32_t kABytes = kAtoms * kAtomBytes;       // 32 KB: this CTA's 128 rows
constexpr uint32_t kABoxBytes = kABoxRows * kBK * 2;    // 4 KB: 32 rows of one atom
constexpr uint32_t kBBytes = kAtoms * kAtomBytes;       // 32 KB: this CTA's half of N = 256
constexpr uint32_t kAccCols = 256;
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kStageOutBytes = 32 * 128;
template <int kMode>
struct PairCfg {
    static constexpr int kStages = kMode == 0 ? kStagesGateUp : kStagesDown;
    static constexpr uint32_t kOutBytes = kMode == 0 ? 0u : kEpiWarps * kStageOutBytes;
    static constexpr size_t kSmemBytes = 1024 + kStages * (kABytes + kBBytes) + kOutBytes + 256;
    static_assert(kSmemBytes <= 232448, "shared memory budget");
};

template <int kStages>
struct __align__(8) Barriers {
    uint64_t full[kStages];   // CTA 0's counts both CTAs' loads of a stage
    uint64_t empty[kStages];  // each CTA's: its stage may be refilled
    uint64_t acc_full[2];     // each CTA's: its accumulator rows are ready
    uint64_t acc_empty[2];    // CTA 0's: both CTAs drained the accumulator
    uint64_t done;
    uint32_t tmem_base;
    int abort_flag;
};

__device__ __forceinline__ float silu_f(float g) { return g * __frcp_rn(1.0f + __expf(-g)); }

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
    const __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<const uint32_t*>(&v);
}

__device__ __forceinline__ int rows_of(int nvalid, uint32_t rank) {
    const int r = nvalid - 128 * (int)rank;
    return r < 0 ? 0 : (r > 128 ? 128 : r);
}

template <int kMode>  // 0: gate/up + SwiGLU -> bf16 h;  1: down -> fp32 y
__device__ __forceinline__ void pair_gemm_body(const CUtensorMap& tmA, const CUtensorMap& tmA128,
                                               const CUtensorMap& tmB, const CUtensorMap& tmOut,
                                               const GemmParams& p) {
    constexpr int kStages = PairCfg<kMode>::kStages;
    constexpr uint32_t kOutBytes = PairCfg<kMode>::kOutBytes;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t* sA = smem;
    uint8_t* sB = smem + kStages * kABytes;
    uint8_t* sOut = sB + kStages * kBBytes;
    Barriers<kStages>* bars = reinterpret_cast<Barriers<kStages>*>(sOut + kOutBytes);
    volatile int* abort_flag = &bars->abort_flag;

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const uint32_t rank = cluster_ctarank();
    const bool leader = rank == 0;
    const int pair = (int)cluster_id_x();
    const int npairs = (int)cluster_count_x();

    if (threadIdx.x == 0) {
        for (int s = 0; s < kStages; ++s) {
            mbar_init(&bars->full[s], 1);
            mbar_init(&bars->empty[s], 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&bars->acc_full[b], 1);
            mbar_init(&bars->acc_empty[b], 2 * kEpiWarps);
        }
        mbar_init(&bars->done, 1);
        bars->abort_flag = 0;
        fence_barrier_init();
    }
    if (warp == 1) {
        tmem_alloc_pair(&bars->tmem_base, kTmemCols);
        tmem_relinquish_pair();
    }
    tc_fence_before_sync();
    __syncthreads();
    cluster_sync();  // both CTAs' barriers and TMEM exist before any cross-CTA traffic
    tc_fence_after_sync();
    const uint32_t tmem_base = bars->tmem_base;

    const int num_m = (int)p.status_words[kStNumMTiles];
    const int total_tiles = num_m * p.n_tiles;
    const int kb_count = p.k_blocks;

    if (warp == 0) {
        if (lane == 0) {
            // ---------------- TMA producer (both CTAs)
            tma_prefetch_desc(&tmA);
            tma_prefetch_desc(&tmA128);
            tma_prefetch_desc(&tmB);
            int stage = 0;
            uint32_t phase = 0;
            bool ok = true;
            int last_phase[kStages];
            for (int s = 0; s < kStages; ++s) last_phase[s] = -1;
            for (int t = pair; t < total_tiles && ok; t += npairs) {
                const int mt = t / p.n_tiles, nt = t - mt * p.n_tiles;
                const int4 ti = __ldg(p.tiles + mt);
                const int box0 = (rows_of(ti.z, 0) + kABoxRows - 1) / kABoxRows;
                const int box1 = (rows_of(ti.z, 1) + kABoxRows - 1) / kABoxRows;
                const int my_boxes = leader ? box0 : box1;
                const uint32_t tx = (uint32_t)(box0 + box1) * kAtoms * kABoxBytes + 2 * kBBytes;
                const int my_row0 = ti.y + 128 * (int)rank;
                for (int kb = 0; kb < kb_count; ++kb) {
                    if (!mbar_wait_bounded(&bars->empty[stage], phase ^ 1u, abort_flag, p.wait_limit_ns)) {
                        ok = false;
                        break;
                    }
                    if (leader) {
                        mbar_arrive_expect_tx(&bars->full[stage], tx);
                        last_phase[stage] = (int)phase;
                    }
                    const uint32_t full0 = map_to_cta(smem_u32(&bars->full[stage]), 0);
                    // operands as [atom][row][64 elements]; a box spans both atoms of the stage
                    uint8_t* a_dst = sA + stage * kABytes;
                    if (my_boxes == 128 / kABoxRows)  // full tile: one TMA instruction, 32 KB
                        tma_load_3d_pair(a_dst, &tmA128, full0, 0, my_row0, kb * kAtoms);
                    else
                        for (int a = 0; a < kAtoms; ++a)
                            for (int i = 0; i < my_boxes; ++i)
                                tma_load_3d_pair(a_dst + a * kAtomBytes + i * kABoxBytes, &tmA, full0, 0,
                                                 my_row0 + i * kABoxRows, kb * kAtoms + a);
                    uint8_t* b_dst = sB + stage * kBBytes;
                    if (kMode == 0)  // CTA 0: gate rows, CTA 1: up rows of the same 128 f
                        tma_load_5d_pair(b_dst, &tmB, full0, 0, nt * kG1BN, kb * kAtoms, (int)rank, ti.x);
                    else
                        tma_load_4d_pair(b_dst, &tmB, full0, 0, nt * kG2BN + 128 * (int)rank, kb * kAtoms, ti.x);
                    if (++stage == kStages) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
            }
            if (!ok) {
                *abort_flag = 1;
                atomicOr(p.status_flags, MOE_DEV_TIMEOUT);
                if (leader) {  // copies already issued land before shared memory goes away
                    for (int s = 0; s < kStages; ++s)
                        if (last_phase[s] >= 0) {
                            volatile int never = 0;
                            (void)mbar_wait_bounded(&bars->full[s], (uint32_t)last_phase[s], &never, 100000000ull);
                        }
                }
            }
        }
        __syncwarp();
    } else if (warp == 1) {
        if (lane == 0 && leader) {
            // ---------------- pair MMA issuer (CTA 0)
            constexpr uint32_t idesc = idesc_bf16_f32(kPairRows, 256);
            int stage = 0;
            uint32_t phase = 0;
            bool ok = true;
            int it = 0;
            for (int t = pair; t < total_tiles && ok; t += npairs, ++it) {
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
                    for (int kk = 0; kk < kStageK / 16; ++kk) {
                        const uint32_t off = (uint32_t)(kk >> 2) * kAtomBytes + (uint32_t)(kk & 3) * 32;
                        mma_bf16_pair(d_tmem, sdesc_kmajor_sw128(a_addr + off), sdesc_kmajor_sw128(b_addr + off), idesc,
                                      (kb | kk) != 0 ? 1u : 0u);
                    }
                    mma_commit_pair_multicast(&bars->empty[stage], 0x3);  // both CTAs may refill the stage
                    if (++stage == kStages) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
                if (!ok) break;
                mma_commit_pair_multicast(&bars->acc_full[buf], 0x3);
            }
            if (!ok) {
                *abort_flag = 1;
                atomicOr(p.status_flags, MOE_DEV_TIMEOUT);
            }
            mma_commit_pair(&bars->done);
            volatile int never = 0;
            (void)mbar_wait_bounded(&bars->done, 0, &never, 100000000ull);
        }
        __syncwarp();
    } else {
        // ---------------- epilogue: warps 2..9
        const int ew = warp - 2;
        const int quad = warp & 3;   // TMEM lane quarter this warp may read
        const int half = ew >> 2;    // column half
        const int r = quad * 32 + lane;
        const uint32_t acc_empty0[2] = {map_to_cta(smem_u32(&bars->acc_empty[0]), 0),
                                        map_to_cta(smem_u32(&bars->acc_empty[1]), 0)};
        uint8_t* my_out = sOut + (size_t)ew * kStageOutBytes;
        int it = 0;
        for (int t = pair; t < total_tiles; t += npairs, ++it) {
            const int buf = it & 1;
            const uint32_t acc_phase = (uint32_t)(it >> 1) & 1u;
            const int mt = t / p.n_tiles, nt = t - mt * p.n_tiles;
            const int4 ti = __ldg(p.tiles + mt);
            const int my_rows = rows_of(ti.z, rank);
            const int my_row0 = ti.y + 128 * (int)rank;
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
            const bool valid = r < my_rows;
            const uint32_t taddr = tmem_base + ((uint32_t)(quad * 32) << 16) + (uint32_t)buf * kAccCols;
            if (kMode == 0) {
                __nv_bfloat16* out_row =
                    reinterpret_cast<__nv_bfloat16*>(p.out) + (size_t)(my_row0 + r) * (size_t)p.out_ld;
#pragma unroll 1
                for (int cc = 0; cc < 2; ++cc) {
                    const int c = half * 2 + cc;
                    uint32_t g[32], u[32];
                    tmem_ld_32x32b_x32(taddr + c * 32, g);
                    tmem_ld_32x32b_x32(taddr + kG1BN + c * 32, u);
                    tmem_ld_wait();
                    const int f0 = nt * kG1BN + c * 32;
                    if (valid) {
#pragma unroll
                        for (int q = 0; q < 4; ++q) {
                            {  // f >= F are zero-weight rows: h = 0, which pads h's K pitch to 128
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
                // fp32 rows leave through the LSU, not the TMA engine (which the
                // operand loads saturate): the warp stages its 32 rows x 32
                // columns in a swizzled 4 KB box, reads it back transposed and
                // writes 4 rows x 128 bytes per instruction, valid rows only.
                const bool slice_live = quad * 32 < my_rows;
                float* y = reinterpret_cast<float*>(p.out);
#pragma unroll 1
                for (int cc = 0; cc < 4; ++cc) {
                    const int c = half * 4 + cc;
                    uint32_t v[32];
                    tmem_ld_32x32b_x32(taddr + c * 32, v);
                    tmem_ld_wait();
                    const int c0 = nt * kG2BN + c * 32;
                    if (slice_live && c0 < p.out_cols) {
#pragma unroll
                        for (int q = 0; q < 8; ++q) {
                            const uint32_t off = (uint32_t)lane * 128u + (uint32_t)((q ^ (lane & 7)) * 16);
                            *reinterpret_cast<uint4*>(my_out + off) =
                                make_uint4(v[q * 4], v[q * 4 + 1], v[q * 4 + 2], v[q * 4 + 3]);
                        }
                        __syncwarp();
                        const int q = lane & 7;
                        const bool col_ok = c0 + q * 4 < p.out_cols;
#pragma unroll
                        for (int i = 0; i < 8; ++i) {
                            const int row = i * 4 + (lane >> 3);
                            const uint4 w = *reinterpret_cast<const uint4*>(my_out + row * 128 + ((q ^ (row & 7)) * 16));
                            if (col_ok && quad * 32 + row < my_rows)
                                *reinterpret_cast<uint4*>(y + (size_t)(my_row0 + quad * 32 + row) * (size_t)p.out_ld + c0 +
                                                          q * 4) = w;
                        }
                        __syncwarp();
                    }
                }
            }
            tc_fence_before_sync();
            __syncwarp();
            if (lane == 0) mbar_arrive_cluster(acc_empty0[buf]);  // release on CTA 0's barrier
        }
    }

    // ---------------- teardown: no pair MMA is in flight once CTA 0 has seen "done"
    tc_fence_before_sync();
    __syncthreads();
    cluster_sync();
    if (warp == 1) {
        tc_fence_after_sync();
        tmem_dealloc_pair(tmem_base, kTmemCols);
    }
}

__global__ void __launch_bounds__(kThreads, 1)
    moe_gemm_gate_up_swiglu_bf16_pair(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmA128,
                                      const __grid_constant__ CUtensorMap tmB,
                                      const __grid_constant__ CUtensorMap tmOut, const GemmParams p) {
    pair_gemm_body<0>(tmA, tmA128, tmB, tmOut, p);
}

__global__ void __launch_bounds__(kThreads, 1)
    moe_gemm_down_bf16_pair(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmA128,
                            const __grid_constant__ CUtensorMap tmB, const __grid_constant__ CUtensorMap tmOut,
                            const GemmParams p) {
    pair_gemm_body<1>(tmA, tmA128, tmB, tmOut, p);
}

using GemmKernel = void (*)(CUtensorMap, CUtensorMap, CUtensorMap, CUtensorMap, GemmParams);

struct PairLaunchCache {
    size_t smem = 0;
    int device = -1;
    int pairs = 0;
};

cudaError_t launch_pair(GemmKernel kern, PairLaunchCache* cache, const CUtensorMap& a, const CUtensorMap& a128,
                        const CUtensorMap& b, const CUtensorMap& o, const GemmParams& gp, long long max_tiles,
                        cudaStream_t s) {
    int dev = 0;
    cudaError_t err = cudaGetDevice(&dev);
    if (err != cudaSuccess) return err;
    cudaLaunchConfig_t cfg = {};
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = cache->smem;
    cfg.stream = s;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (cache->device != dev) {
        err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)cache->smem);
        if (err != cudaSuccess) return err;
        // persistent grid: as many CTA pairs as can be resident at once
        int clusters = 0;
        cfg.gridDim = dim3(2 * (num_sms() / 2));
        err = cudaOccupancyMaxActiveClusters(&clusters, kern, &cfg);
        if (err != cudaSuccess) return err;
        if (clusters < 1) return cudaErrorInvalidConfiguration;
        cache->pairs = clusters < num_sms() / 2 ? clusters : num_sms() / 2;
        cache->device = dev;
    }
    long long pairs = cache->pairs;
    if (pairs > max_tiles) pairs = max_tiles;
    if (pairs < 1) pairs = 1;
    cfg.gridDim = dim3((unsigned)(2 * pairs));
    err = cudaLaunchKernelEx(&cfg, kern, a, a128, b, o, gp);
    if (err != cudaSuccess) return err;
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_gemm1_bf16_pair(const CUtensorMap& a, const CUtensorMap& a128, const CUtensorMap& b,
                                   const CUtensorMap& o, const GemmParams& gp, long long max_tiles, cudaStream_t s) {
    static PairLaunchCache cache{PairCfg<0>::kSmemBytes};
    return launch_pair(moe_gemm_gate_up_swiglu_bf16_pair, &cache, a, a128, b, o, gp, max_tiles, s);
}

cudaError_t launch_gemm2_bf16_pair(const CUtensorMap& a, const CUtensorMap& a128, const CUtensorMap& b,
                                   const CUtensorMap& o, const GemmParams& gp, long long max_tiles, cudaStream_t s) {
    static PairLaunchCache cache{PairCfg<1>::kSmemBytes};
    return launch_pair(moe_gemm_down_bf16_pair, &cache, a, a128, b, o, gp, max_tiles, s);
}

}  // namespace moe
