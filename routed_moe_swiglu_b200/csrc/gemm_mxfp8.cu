// gemm_mxfp8.cu -- the two grouped expert GEMMs in MXFP8 (E4M3 operands with
// one E8M0 scale per 32 K elements per row), block-scaled tcgen05 MMAs with
// the scale factors in TMEM, expert weights as the MMA's M operand and routes
// as its N operand (as in the bf16 kernels: the last tile of an expert costs
// its route count rounded up to 32, not a full tile).
//
// Megatron-LM PR #7798, "Background": the FC1 epilogue fuses the activation
// and the FC2-input quantisation; probabilities are applied after FC2.
// Megatron-LM PR #7830 / cudnn-frontend PR #448: MXFP8 blocks are 32
// elements along K.
//
//   gate/up:  A = 128 rows of W1 = 64 f values: TMEM lane quarter q holds
//             the gate rows of f = f0 + 16q + i in lanes 32q+i and the up
//             rows of the same f in lanes 32q+16+i (the prepared W1 is
//             interleaved so); B = N <= 128 route rows of x codes.  The
//             epilogue forms h = silu(g) * u in fp32 (half-warps swap gate
//             and up with shfl.xor 16), stages 32 routes x 64 f in shared
//             memory, and two threads per (route, 32-f block) re-quantise it
//             to MXFP8: E4M3 codes to h, E8M0 bytes into the scale layout the
//             down GEMM reads.
//   down:     A = 128 rows of W_down[e] (output columns), B = N route rows of
//             h codes; fp32 y rows leave through a shared-memory transpose.
//
// A K stage is 256 elements: two 128-byte swizzle atoms, 8 MMAs, and each
// operand of a stage one TMA instruction (a 3-D map whose third dimension
// walks the atoms of a row; the K pitches are padded to 128 with zeros).
// Fewer, larger stages matter here: the per-stage fixed cost (barrier
// hand-offs, commits, TMA issue) dominated with 128-element stages.
//
// Scale factors: for each 128-row operand tile (a weight tile, or the 128
// padded route rows a route tile lies in) and K block of 128 elements, 512
// bytes laid out as [row % 32][row / 32][k-group], which one tcgen05.cp
// (32x128b, replicated to the 4 lane quarters) moves to 4 TMEM columns; MMA
// k-group kk selects byte kk of each 32-bit cell.  The blocks of 8
// consecutive K blocks (4 stages) of a tile are contiguous, so they arrive
// with one bulk copy per operand into a double-buffered shared-memory area,
// and the MMA thread moves each stage's blocks to TMEM just before its MMAs.
//
// Pipeline: persistent CTA per SM, warp 0 TMA, warp 1 MMA + TMEM owner,
// warps 2-5 epilogue; two 128-column accumulators; one scale-factor TMEM
// slot per stage (rewritten only after the MMAs that read it have completed,
// which the producer's wait on that stage's "empty" barrier already
// implies).  Every wait is bounded.
#include "moe_internal.cuh"
#include "mxfp8.cuh"
#include "nvfp4.cuh"
#include "ptx.cuh"

namespace moe {
namespace {

constexpr int kStagesMax = 4;  // pipeline stages per launch: 3 or 4, by the widest route tile
constexpr int kThreads = 192;
constexpr int kTileM = 128;                            // weight rows per tile
constexpr int kMaxN = 128;                             // routes per tile
constexpr int kAtoms = 2;                              // 128-element K blocks (swizzle atoms) per stage
constexpr uint32_t kAtomBytesA = kTileM * kBK8;        // 16 KB
constexpr uint32_t kABytes = kAtoms * kAtomBytesA;     // 32 KB
constexpr uint32_t kBBytes = kAtoms * kMaxN * kBK8;    // up to 32 KB
// the stages: 4 x (32 + 16) KB when every route tile holds at most 64 routes, else 3 x (32 + 32) KB
constexpr uint32_t kStageRegion = 3 * (kABytes + kBBytes);
static_assert(kStageRegion == 4 * (kABytes + kBBytes / 2), "both pipelines fill the stage region");
// Scale blocks: MXFP8 (kFmt 0) has one 512-byte block per operand and 128-byte K block
// (4 MMAs, a byte each); NVFP4 (kFmt 1) has one per 64-element MMA step, four per K block.
template <int kFmt>
struct SfCfg {
    static constexpr int kPerKb = kFmt == 0 ? 1 : 4;               // scale blocks per K block
    static constexpr int kGroup = kFmt == 0 ? 8 : 2;               // K blocks per bulk copy (4 stages / 1)
    static constexpr int kStagesPerGroup = kGroup / kAtoms;
    static constexpr uint32_t kGroupBytes = (uint32_t)(kGroup * kPerKb) * kSfBlock;  // 4 KB either way
    static constexpr uint32_t kColsPerStage = (uint32_t)(kAtoms * kPerKb) * 8u;     // A 4 + B 4 per block
};
constexpr uint32_t kSfGroupBytes = SfCfg<0>::kGroupBytes;
static_assert(SfCfg<1>::kGroupBytes == kSfGroupBytes, "one scale staging size for both formats");
constexpr uint32_t kSfBytes = 2 * 2 * kSfGroupBytes;   // [buffer][A/B][group][512 B blocks]
constexpr uint32_t kAccCols = kMaxN;
constexpr uint32_t kSfCol0 = 2 * kAccCols;             // first scale-factor TMEM column
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kStageHBytes = 32 * 64 * 4;         // gate/up: fp32 h of 32 routes x 64 f
constexpr uint32_t kYTBytes = 32 * 32 * 4;             // down: fp32 y of 32 routes x 32 columns, per warp
constexpr uint32_t kEpiBytes = 2 * kStageHBytes > 4 * kYTBytes ? 2 * kStageHBytes : 4 * kYTBytes;
constexpr size_t kSmemBytes = 1024 + kStageRegion + kSfBytes + kEpiBytes + 256;
static_assert(kSmemBytes <= 232448, "shared memory budget");
static_assert(kSfCol0 + SfCfg<1>::kColsPerStage * kStagesMax <= kTmemCols, "TMEM budget");
static_assert(kEpiBytes >= 4 * 32 * 32 * 4, "squared-ReLU epilogue boxes");
constexpr uint32_t kEpiBar = 1;                        // named barrier of the 4 epilogue warps

struct __align__(8) Barriers {
    uint64_t full[kStagesMax];
    uint64_t empty[kStagesMax];
    uint64_t acc_full[2];
    uint64_t acc_empty[2];
    uint64_t sf_empty[2];
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

// NVFP4: E2M1 x E2M1 (kind::mxf4nvf4), E4M3 scales, one per 16 K elements
// (scale_vec::4X: an MMA of K = 64 reads a whole 32-bit scale cell per row).
__host__ __device__ constexpr uint32_t idesc_nvf4(int M, int N) {
    return (1u << 7) | (1u << 10)          // A, B: E2M1
           | ((uint32_t)(N >> 3) << 17)    // N / 8
           | (0u << 23)                    // scale type: E4M3
           | ((uint32_t)(M >> 4) << 24);   // M / 16
}

__device__ __forceinline__ void mma_nvf4_ss(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                            uint32_t sfa_tmem, uint32_t sfb_tmem, uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::mxf4nvf4.block_scale.scale_vec::4X [%0], %1, %2, %3, [%5], [%6], p;\n\t}\n" ::"r"(
            d_tmem),
        "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate), "r"(sfa_tmem), "r"(sfb_tmem)
        : "memory");
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

__device__ __forceinline__ float silu_f(float g) { return __fdividef(g, 1.0f + __expf(-g)); }

// silu(g) * u, the two pre-activations first clamped to [-clamp, clamp] when clamp > 0
// (the MoeEp `gate_up_clamp` option of cudnn-frontend PR #448)
__device__ __forceinline__ float swiglu_value(float g, float u, float clamp) {
    if (clamp > 0.0f) {
        g = fminf(fmaxf(g, -clamp), clamp);
        u = fminf(fmaxf(u, -clamp), clamp);
    }
    return silu_f(g) * u;
}

// Routes of a tile rounded up to the MMA's N granularity.
__device__ __forceinline__ int tile_n(int nvalid) { return (nvalid + 31) & ~31; }

// kMode 0: gate/up + SwiGLU -> h (MXFP8 codes, or NVFP4's fp32 rows for a second pass);
// kMode 1: down -> fp32 y.  kFmt 0: MXFP8; 1: NVFP4.
template <int kMode, int kFmt>
__device__ __forceinline__ void gemm_mxfp8_body(const CUtensorMap& tmA, const BoxMaps8& tmB, const GemmParams& p) {
    using Sf = SfCfg<kFmt>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t* sSf = smem + kStageRegion;  // [buffer][A/B][8][512]
    uint8_t* sEpi = sSf + kSfBytes;
    Barriers* bars = reinterpret_cast<Barriers*>(sEpi + kEpiBytes);
    volatile int* abort_flag = &bars->abort_flag;
    auto sf_buf = [&](int b, int ab) { return sSf + (size_t)(b * 2 + ab) * kSfGroupBytes; };

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    pdl_trigger();

    if (threadIdx.x == 0) {
        for (int s = 0; s < kStagesMax; ++s) {
            mbar_init(&bars->full[s], 1);
            mbar_init(&bars->empty[s], 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&bars->acc_full[b], 1);
            mbar_init(&bars->acc_empty[b], 4);
            mbar_init(&bars->sf_empty[b], 1);
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
    pdl_wait();  // the tile list, route rows, scales and status words come from earlier kernels

    const int num_m = forward_poisoned(p.status_words) ? 0 : (int)p.status_words[kStNumMTiles];
    // the pipeline of this launch, from the widest route tile of the forward (every role
    // derives the same): weight slots first, at multiples of 32 KB, then the route-row slots
    const int kStages = tile_n((int)p.status_words[kStMaxTileRows]) <= 64 ? 4 : 3;
    const uint32_t b_slot = kStages == 4 ? kBBytes / 2 : kBBytes;
    auto stage_a = [&](int s) { return smem + s * kABytes; };
    auto stage_b = [&](int s) { return smem + kStages * kABytes + s * b_slot; };
    const int total_tiles = num_m * p.n_tiles;
    const int nblk = p.k_blocks;               // K blocks of 128
    const int kb_count = (nblk + 1) / kAtoms;  // stages of 256 (the last may hold one block)

    if (warp == 0) {
        if (lane == 0) {
            // ---------------- TMA producer
            tma_prefetch_desc(&tmA);
            // no expert with more than one route tile (decode): each weight tile is read by
            // one CTA only, and its lines go first out of L2 (the h and y rows stay)
            const bool weights_once = (int)p.status_words[kStMaxTileRows] < kBM;
            const uint64_t pol_once = l2_policy_evict_first();
            int stage = 0;
            uint32_t phase = 0;
            uint32_t groups = 0;  // scale-factor groups issued so far
            bool ok = true;
            int last_phase[kStagesMax];
            for (int s = 0; s < kStagesMax; ++s) last_phase[s] = -1;
            for (int t = blockIdx.x; t < total_tiles && ok; t += gridDim.x) {
                const int mt = t / p.n_tiles, nt = t - mt * p.n_tiles;
                const int4 ti = __ldg(p.tiles + mt);
                const int n = tile_n(ti.z);
                const CUtensorMap* mapB = &tmB.m[(n >> 5) - 1];
                const int a_row = (int)((long long)ti.x * p.a_rows) + nt * kTileM;
                const uint8_t* sfa_src = p.sfa + ((size_t)ti.x * p.n_tiles + nt) * nblk * Sf::kPerKb * kSfBlock;
                const uint8_t* sfb_src = p.sfb + (size_t)(ti.y / kBM) * nblk * Sf::kPerKb * kSfBlock;
                for (int kb = 0; kb < kb_count; ++kb) {
                    if (!mbar_wait_bounded(&bars->empty[stage], phase ^ 1u, abort_flag, p.wait_limit_ns)) {
                        ok = false;
                        break;
                    }
                    // both atoms' bytes count even where the second lies past K (zero fill)
                    uint32_t tx = kABytes + (uint32_t)n * (kAtoms * kBK8);
                    int gs = 0;
                    const int blk0 = kb * kAtoms;
                    if (kb % Sf::kStagesPerGroup == 0) {
                        // the scale blocks of this stage and the next gs-1 stages, once the MMAs
                        // that read this buffer two groups ago are done
                        const int sb = (int)(groups & 1u);
                        if (!mbar_wait_bounded(&bars->sf_empty[sb], ((groups >> 1) & 1u) ^ 1u, abort_flag,
                                               p.wait_limit_ns)) {
                            ok = false;
                            break;
                        }
                        gs = nblk - blk0 < Sf::kGroup ? nblk - blk0 : Sf::kGroup;
                        tx += 2u * (uint32_t)(gs * Sf::kPerKb) * kSfBlock;
                    }
                    mbar_arrive_expect_tx(&bars->full[stage], tx);
                    last_phase[stage] = (int)phase;
                    if (weights_once)
                        tma_load_3d_hint(stage_a(stage), &tmA, &bars->full[stage], 0, a_row, blk0, pol_once);
                    else
                        tma_load_3d(stage_a(stage), &tmA, &bars->full[stage], 0, a_row, blk0);
                    tma_load_3d(stage_b(stage), mapB, &bars->full[stage], 0, ti.y, blk0);
                    if (gs > 0) {
                        const int sb = (int)(groups & 1u);
                        const uint32_t sf_bytes = (uint32_t)(gs * Sf::kPerKb) * kSfBlock;
                        bulk_load(sf_buf(sb, 0), sfa_src + (size_t)blk0 * Sf::kPerKb * kSfBlock, sf_bytes,
                                  &bars->full[stage]);
                        bulk_load(sf_buf(sb, 1), sfb_src + (size_t)blk0 * Sf::kPerKb * kSfBlock, sf_bytes,
                                  &bars->full[stage]);
                        ++groups;
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
            uint32_t groups = 0;
            bool ok = true;
            int it = 0;
            for (int t = blockIdx.x; t < total_tiles && ok; t += gridDim.x, ++it) {
                const int buf = it & 1;
                const uint32_t acc_phase = (uint32_t)(it >> 1) & 1u;
                const int mt = t / p.n_tiles;
                const int n = tile_n(__ldg(&p.tiles[mt].z));
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
                    const int sb = (int)(groups & 1u);
                    const int blk0 = kb * kAtoms;
                    const int nb = nblk - blk0 < kAtoms ? nblk - blk0 : kAtoms;  // K blocks in this stage
                    const uint32_t a_addr = smem_u32(stage_a(stage));
                    const uint32_t b_addr = smem_u32(stage_b(stage));
                    const uint32_t b_atom = (uint32_t)n * kBK8;  // bytes of one atom of the B box
                    for (int h = 0; h < nb; ++h) {
                        const int gi = (blk0 + h) % Sf::kGroup;
                        const uint32_t a_h = a_addr + (uint32_t)h * kAtomBytesA;
                        const uint32_t b_h = b_addr + (uint32_t)h * b_atom;
                        const uint32_t sf_t0 = tmem_base + kSfCol0 + (uint32_t)stage * Sf::kColsPerStage +
                                               (uint32_t)(h * Sf::kPerKb) * 8u;
                        if constexpr (kFmt == 0) {
                            // one scale block per operand: MMA kk reads byte kk of each cell
                            tmem_cp_32x128b_warpx4(sf_t0, sdesc_sf(smem_u32(sf_buf(sb, 0) + gi * kSfBlock)));
                            tmem_cp_32x128b_warpx4(sf_t0 + 4u, sdesc_sf(smem_u32(sf_buf(sb, 1) + gi * kSfBlock)));
#pragma unroll
                            for (int kk = 0; kk < kBK8 / 32; ++kk) {
                                mma_mxf8_ss(d_tmem, sdesc_kmajor_sw128(a_h + kk * 32),
                                            sdesc_kmajor_sw128(b_h + kk * 32),
                                            idesc_mxf8(kTileM, n, (uint32_t)kk, (uint32_t)kk), sf_t0, sf_t0 + 4u,
                                            (kb | h | kk) != 0 ? 1u : 0u);
                            }
                        } else {
                            // one scale block per operand and 64-element MMA step (32 bytes of K)
#pragma unroll
                            for (int kk = 0; kk < kBK8 / 32; ++kk) {
                                const uint32_t sfa_t = sf_t0 + (uint32_t)kk * 8u;
                                const uint32_t src = (uint32_t)(gi * Sf::kPerKb + kk) * kSfBlock;
                                tmem_cp_32x128b_warpx4(sfa_t, sdesc_sf(smem_u32(sf_buf(sb, 0) + src)));
                                tmem_cp_32x128b_warpx4(sfa_t + 4u, sdesc_sf(smem_u32(sf_buf(sb, 1) + src)));
                                mma_nvf4_ss(d_tmem, sdesc_kmajor_sw128(a_h + kk * 32),
                                            sdesc_kmajor_sw128(b_h + kk * 32), idesc_nvf4(kTileM, n), sfa_t,
                                            sfa_t + 4u, (kb | h | kk) != 0 ? 1u : 0u);
                            }
                        }
                    }
                    mma_commit(&bars->empty[stage]);
                    if (kb % Sf::kStagesPerGroup == Sf::kStagesPerGroup - 1 || kb == kb_count - 1) {  // group consumed
                        mma_commit(&bars->sf_empty[sb]);
                        ++groups;
                    }
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
        // ---------------- epilogue: warps 2..5, TMEM lane quarter = warp % 4
        const int quad = warp & 3;
        const int et = threadIdx.x - 64;  // 0..127
        int it = 0;
        uint32_t chunk_count = 0;  // chunks staged so far (the staging buffer alternates)
        for (int t = blockIdx.x; t < total_tiles; t += gridDim.x, ++it) {
            const int buf = it & 1;
            const uint32_t acc_phase = (uint32_t)(it >> 1) & 1u;
            const int mt = t / p.n_tiles, nt = t - mt * p.n_tiles;
            const int4 ti = __ldg(p.tiles + mt);
            const int nch = tile_n(ti.z) >> 5;
            bool got = __all_sync(0xffffffffu,
                                  mbar_wait_bounded(&bars->acc_full[buf], acc_phase, abort_flag, p.wait_limit_ns));
            // the four warps decide together: the gate/up epilogue meets in a named barrier per chunk
            if (kMode == 0) got = named_bar_and(kEpiBar, 128, got);
            if (!got) {
                if (lane == 0) {
                    *abort_flag = 1;
                    atomicOr(p.status_flags, MOE_DEV_TIMEOUT);
                }
                break;
            }
            tc_fence_after_sync();
            const uint32_t taddr = tmem_base + ((uint32_t)(quad * 32) << 16) + (uint32_t)buf * kAccCols;
            if constexpr (kMode == 0 && kFmt == 1) {
                // NVFP4: the accumulator times g_x(route) * g_w1(expert) is the pre-activation;
                // h leaves as fp32 rows (pitch out_ld) for the per-row quantisation pass.
                float* hf = reinterpret_cast<float*>(p.out);
                const float gw = __ldg(p.w_scale + 2 * ti.x);
                if (p.relu2) {
                    // squared-ReLU experts: lane = f (32 f from f0), register j = route 32c + j
                    const int f0 = nt * kTileM + 32 * quad;
#pragma unroll 1
                    for (int c = 0; c < nch; ++c) {
                        uint32_t v[32];
                        tmem_ld_32x32b_x32(taddr + c * 32, v);
                        float pv = 1.0f, sc = 0.0f;
                        if (c * 32 + lane < ti.z) {
                            sc = __ldg(p.row_scale + ti.y + c * 32 + lane) * gw;
                            if (p.route_probs != nullptr) pv = __ldg(p.route_probs + __ldg(p.perm + ti.w + c * 32 + lane));
                        }
                        tmem_ld_wait();
#pragma unroll
                        for (int j = 0; j < 32; ++j) {
                            float g = __uint_as_float(v[j]) * __shfl_sync(0xffffffffu, sc, j);
                            if (p.clamp > 0.0f) g = fminf(fmaxf(g, -p.clamp), p.clamp);
                            const float r = fmaxf(g, 0.0f);
                            float hv = r * r;
                            if (p.route_probs != nullptr) hv *= __shfl_sync(0xffffffffu, pv, j);
                            if (c * 32 + j < ti.z && f0 < p.out_cols)
                                hf[(size_t)(ti.y + c * 32 + j) * (size_t)p.out_ld + f0 + lane] = hv;
                        }
                    }
                } else {
                    const bool lo = lane < 16;
                    const int fl = 16 * quad + (lane & 15);  // this lane's f within the tile's 64
                    const int qr = et >> 2, qf = (et & 3) * 16;  // store role: route qr, f qf..qf+15
#pragma unroll 1
                    for (int c = 0; c < nch; ++c, ++chunk_count) {
                        float* st = reinterpret_cast<float*>(sEpi + (chunk_count & 1u) * kStageHBytes);
                        uint32_t v[32];
                        tmem_ld_32x32b_x32(taddr + c * 32, v);
                        float pv = 1.0f, sc = 0.0f;
                        if (c * 32 + lane < ti.z) {
                            sc = __ldg(p.row_scale + ti.y + c * 32 + lane) * gw;
                            if (p.route_probs != nullptr) pv = __ldg(p.route_probs + __ldg(p.perm + ti.w + c * 32 + lane));
                        }
                        tmem_ld_wait();
#pragma unroll
                        for (int j = 0; j < 16; ++j) {
                            const uint32_t mine = lo ? v[j] : v[16 + j];
                            const uint32_t other = __shfl_xor_sync(0xffffffffu, lo ? v[16 + j] : v[j], 16);
                            const int route = lo ? j : 16 + j;
                            const float rs = __shfl_sync(0xffffffffu, sc, route);
                            const float g = __uint_as_float(lo ? mine : other) * rs;
                            const float u = __uint_as_float(lo ? other : mine) * rs;
                            float hv = swiglu_value(g, u, p.clamp);
                            if (p.route_probs != nullptr) hv *= __shfl_sync(0xffffffffu, pv, route);
                            st[route * 64 + (fl ^ (lo ? 0 : 16))] = hv;
                        }
                        named_bar_sync(kEpiBar, 128);
                        const int route = c * 32 + qr;
                        const int fb = nt * 64 + qf;
                        if (route < ti.z && fb < p.out_cols) {
                            const float4* src = reinterpret_cast<const float4*>(st + qr * 64 + (qf ^ (qr >= 16 ? 16 : 0)));
                            float4* dst = reinterpret_cast<float4*>(hf + (size_t)(ti.y + route) * (size_t)p.out_ld + fb);
#pragma unroll
                            for (int i = 0; i < 4; ++i) dst[i] = src[i];
                        }
                    }
                }
            } else if (kMode == 0 && p.relu2) {
                // squared-ReLU experts: lane = f (this warp's 32 f from f0, one 32-f block),
                // register j = route 32c + j.  h = relu(g)^2 goes through a per-warp box
                // [route][32 f] fp32 (column rotated by the route against bank conflicts); then
                // lane l quantises route 32c + l's block: amax, E8M0 scale, 32 E4M3 codes.
                const int f0 = nt * kTileM + 32 * quad;
                uint8_t* hq = reinterpret_cast<uint8_t*>(p.out);
                uint8_t* hs_tile = p.out_scales + (size_t)(ti.y / kBM) * p.sf_ks_out * kSfBlock;
                float* box = reinterpret_cast<float*>(sEpi + (size_t)quad * 32 * 32 * 4);
                if (f0 < p.out_cols) {
#pragma unroll 1
                    for (int c = 0; c < nch; ++c) {
                        uint32_t v[32];
                        tmem_ld_32x32b_x32(taddr + c * 32, v);
                        float pv = 1.0f;
                        if (p.route_probs != nullptr && c * 32 + lane < ti.z)
                            pv = __ldg(p.route_probs + __ldg(p.perm + ti.w + c * 32 + lane));
                        tmem_ld_wait();
#pragma unroll
                        for (int j = 0; j < 32; ++j) {
                            float g = __uint_as_float(v[j]);
                            if (p.clamp > 0.0f) g = fminf(fmaxf(g, -p.clamp), p.clamp);
                            const float r = fmaxf(g, 0.0f);
                            float hv = r * r;
                            if (p.route_probs != nullptr) hv *= __shfl_sync(0xffffffffu, pv, j);
                            box[j * 32 + ((lane + j) & 31)] = hv;
                        }
                        __syncwarp();
                        float hv[32];
                        float amax = 0.0f;
#pragma unroll
                        for (int i = 0; i < 32; ++i) {
                            hv[i] = box[lane * 32 + ((i + lane) & 31)];
                            amax = fmaxf(amax, fabsf(hv[i]));
                        }
                        __syncwarp();
                        float inv;
                        const uint8_t sbyte = mxfp8_block_scale(amax, &inv);
                        const int route = c * 32 + lane;
                        if (p.h_fp32 != nullptr && route < ti.z) {
                            float4* hd = reinterpret_cast<float4*>(p.h_fp32 + (size_t)(ti.y + route) * (size_t)p.out_ld + f0);
#pragma unroll
                            for (int i = 0; i < 8; ++i) hd[i] = make_float4(hv[4 * i], hv[4 * i + 1], hv[4 * i + 2], hv[4 * i + 3]);
                        }
                        if (route < ti.z) {
                            uint32_t w[8];
#pragma unroll
                            for (int i = 0; i < 8; ++i)
                                w[i] = e4m3x2(hv[4 * i + 1] * inv, hv[4 * i] * inv) |
                                       (e4m3x2(hv[4 * i + 3] * inv, hv[4 * i + 2] * inv) << 16);
                            uint4* dst = reinterpret_cast<uint4*>(hq + (size_t)(ti.y + route) * (size_t)p.out_ld + f0);
                            dst[0] = make_uint4(w[0], w[1], w[2], w[3]);
                            dst[1] = make_uint4(w[4], w[5], w[6], w[7]);
                            hs_tile[(size_t)(f0 / 128) * kSfBlock + sf_block_offset(route, (f0 % 128) / 32)] = sbyte;
                        }
                    }
                }
            } else if (kMode == 0) {
                const bool lo = lane < 16;
                const int fl = 16 * quad + (lane & 15);  // this lane's f within the tile's 64
                uint8_t* hq = reinterpret_cast<uint8_t*>(p.out);
                uint8_t* hs_tile = p.out_scales + (size_t)(ti.y / kBM) * p.sf_ks_out * kSfBlock;
                // quantisation role: route qr of the chunk, 32-f block qb, half qh (16 f)
                const int qr = et >> 2, qb = (et >> 1) & 1, qh = et & 1;
                const int f_blk = nt * 64 + qb * 32;  // first f of the 32-f block
#pragma unroll 1
                for (int c = 0; c < nch; ++c, ++chunk_count) {
                    float* st = reinterpret_cast<float*>(sEpi + (chunk_count & 1u) * kStageHBytes);
                    uint32_t v[32];
                    tmem_ld_32x32b_x32(taddr + c * 32, v);
                    // apply_topk_in_fc1: lane l fetches the probability of route 32c + l
                    float pv = 1.0f;
                    if (p.route_probs != nullptr && c * 32 + lane < ti.z)
                        pv = __ldg(p.route_probs + __ldg(p.perm + ti.w + c * 32 + lane));
                    tmem_ld_wait();
                    // h of (route (lo ? j : 16 + j), f = fl) into st[route][64 f]; the f index of
                    // routes 16..31 is xor-ed with 16 so that the two half-warps hit different banks
#pragma unroll
                    for (int j = 0; j < 16; ++j) {
                        const uint32_t mine = lo ? v[j] : v[16 + j];
                        const uint32_t other = __shfl_xor_sync(0xffffffffu, lo ? v[16 + j] : v[j], 16);
                        const float g = __uint_as_float(lo ? mine : other);
                        const float u = __uint_as_float(lo ? other : mine);
                        const int route = lo ? j : 16 + j;
                        float hv = swiglu_value(g, u, p.clamp);
                        if (p.route_probs != nullptr) hv *= __shfl_sync(0xffffffffu, pv, route);
                        st[route * 64 + (fl ^ (lo ? 0 : 16))] = hv;
                    }
                    named_bar_sync(kEpiBar, 128);
                    // quantise: 16 values of (route qr, block qb); the block's other half is lane ^ 1
                    const float4* src =
                        reinterpret_cast<const float4*>(st + qr * 64 + ((qb * 32 + qh * 16) ^ (qr >= 16 ? 16 : 0)));
                    float h[16];
                    float amax = 0.0f;
#pragma unroll
                    for (int i = 0; i < 4; ++i) {
                        const float4 w = src[i];
                        h[4 * i] = w.x;
                        h[4 * i + 1] = w.y;
                        h[4 * i + 2] = w.z;
                        h[4 * i + 3] = w.w;
                        amax = fmaxf(amax, fmaxf(fmaxf(fabsf(w.x), fabsf(w.y)), fmaxf(fabsf(w.z), fabsf(w.w))));
                    }
                    amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 1));
                    float inv;
                    const uint8_t sbyte = mxfp8_block_scale(amax, &inv);
                    const int route = c * 32 + qr;
                    if (p.h_fp32 != nullptr && route < ti.z && f_blk < p.out_cols) {
                        float4* hd = reinterpret_cast<float4*>(p.h_fp32 + (size_t)(ti.y + route) * (size_t)p.out_ld +
                                                               f_blk + qh * 16);
#pragma unroll
                        for (int i = 0; i < 4; ++i) hd[i] = make_float4(h[4 * i], h[4 * i + 1], h[4 * i + 2], h[4 * i + 3]);
                    }
                    if (route < ti.z && f_blk < p.out_cols) {
                        uint32_t w[4];
#pragma unroll
                        for (int i = 0; i < 4; ++i)
                            w[i] = e4m3x2(h[4 * i + 1] * inv, h[4 * i] * inv) |
                                   (e4m3x2(h[4 * i + 3] * inv, h[4 * i + 2] * inv) << 16);
                        *reinterpret_cast<uint4*>(hq + (size_t)(ti.y + route) * (size_t)p.out_ld + f_blk + qh * 16) =
                            make_uint4(w[0], w[1], w[2], w[3]);
                        if (qh == 0)
                            hs_tile[(size_t)(f_blk / 128) * kSfBlock + sf_block_offset(route, (f_blk % 128) / 32)] =
                                sbyte;
                    }
                }
            } else {
                // output columns of this warp: nt*128 + 32*quad + lane
                const int c_base = nt * kTileM + 32 * quad;
                float* y = reinterpret_cast<float*>(p.out);
                uint8_t* tbuf = sEpi + (size_t)quad * kYTBytes;
                if (c_base < p.out_cols) {
                    const bool col_ok = c_base + (lane & 7) * 4 < p.out_cols;
#pragma unroll 1
                    for (int c = 0; c < nch; ++c) {
                        uint32_t v[32];
                        tmem_ld_32x32b_x32(taddr + c * 32, v);
                        float sc = 0.0f;  // NVFP4: g_h(route 32c + lane) * g_w2(expert)
                        if (kFmt == 1 && c * 32 + lane < ti.z)
                            sc = __ldg(p.row_scale + ti.y + c * 32 + lane) * __ldg(p.w_scale + 2 * ti.x + 1);
                        tmem_ld_wait();
                        if constexpr (kFmt == 1) {
#pragma unroll
                            for (int r = 0; r < 32; ++r)
                                v[r] = __float_as_uint(__uint_as_float(v[r]) * __shfl_sync(0xffffffffu, sc, r));
                        }
#pragma unroll
                        for (int r = 0; r < 32; ++r) *reinterpret_cast<uint32_t*>(tbuf + r * 128 + lane * 4) = v[r];
                        __syncwarp();
#pragma unroll
                        for (int i = 0; i < 8; ++i) {
                            const int r = i * 4 + (lane >> 3);
                            const int route = c * 32 + r;
                            const uint4 w = *reinterpret_cast<const uint4*>(tbuf + r * 128 + (lane & 7) * 16);
                            if (col_ok && route < ti.z)
                                *reinterpret_cast<uint4*>(y + (size_t)(ti.y + route) * (size_t)p.out_ld + c_base +
                                                          (lane & 7) * 4) = w;
                        }
                        __syncwarp();
                    }
                }
            }
            tc_fence_before_sync();
            __syncwarp();
            if (lane == 0) mbar_arrive(&bars->acc_empty[buf]);
        }
    }

    tc_fence_before_sync();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after_sync();
        tmem_dealloc(tmem_base, kTmemCols);
    }
}

__global__ void __launch_bounds__(kThreads, 1)
    moe_gemm_gate_up_swiglu_mxfp8(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ BoxMaps8 tmB,
                                  const GemmParams p) {
    gemm_mxfp8_body<0, 0>(tmA, tmB, p);
}

__global__ void __launch_bounds__(kThreads, 1)
    moe_gemm_down_mxfp8(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ BoxMaps8 tmB,
                        const GemmParams p) {
    gemm_mxfp8_body<1, 0>(tmA, tmB, p);
}

__global__ void __launch_bounds__(kThreads, 1)
    moe_gemm_gate_up_swiglu_nvfp4(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ BoxMaps8 tmB,
                                  const GemmParams p) {
    gemm_mxfp8_body<0, 1>(tmA, tmB, p);
}

__global__ void __launch_bounds__(kThreads, 1)
    moe_gemm_down_nvfp4(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ BoxMaps8 tmB,
                        const GemmParams p) {
    gemm_mxfp8_body<1, 1>(tmA, tmB, p);
}

using GemmKernel = void (*)(CUtensorMap, BoxMaps8, GemmParams);

cudaError_t launch_impl(GemmKernel kern, int* configured_device, const CUtensorMap& a, const BoxMaps8& b,
                        const GemmParams& gp, long long max_tiles, cudaStream_t s) {
    int dev = 0;
    cudaError_t err = cudaGetDevice(&dev);
    if (err != cudaSuccess) return err;
    if (*configured_device != dev) {
        err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kSmemBytes);
        if (err != cudaSuccess) return err;
        *configured_device = dev;
    }
    long long grid = num_sms();  // persistent: one CTA per SM
    if (grid > max_tiles) grid = max_tiles;
    if (grid < 1) grid = 1;
    return launch_dependent(kern, dim3((unsigned)grid), dim3(kThreads), kSmemBytes, s, a, b, gp);
}

}  // namespace

cudaError_t launch_gemm1_mxfp8(const CUtensorMap& a, const BoxMaps8& b, const GemmParams& gp, long long max_tiles,
                               cudaStream_t s) {
    static int configured = -1;
    return launch_impl(moe_gemm_gate_up_swiglu_mxfp8, &configured, a, b, gp, max_tiles, s);
}

cudaError_t launch_gemm2_mxfp8(const CUtensorMap& a, const BoxMaps8& b, const GemmParams& gp, long long max_tiles,
                               cudaStream_t s) {
    static int configured = -1;
    return launch_impl(moe_gemm_down_mxfp8, &configured, a, b, gp, max_tiles, s);
}

cudaError_t launch_gemm1_nvfp4(const CUtensorMap& a, const BoxMaps8& b, const GemmParams& gp, long long max_tiles,
                               cudaStream_t s) {
    static int configured = -1;
    return launch_impl(moe_gemm_gate_up_swiglu_nvfp4, &configured, a, b, gp, max_tiles, s);
}

cudaError_t launch_gemm2_nvfp4(const CUtensorMap& a, const BoxMaps8& b, const GemmParams& gp, long long max_tiles,
                               cudaStream_t s) {
    static int configured = -1;
    return launch_impl(moe_gemm_down_nvfp4, &configured, a, b, gp, max_tiles, s);
}

}  // namespace moe
