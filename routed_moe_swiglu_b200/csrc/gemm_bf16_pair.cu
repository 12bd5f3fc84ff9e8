// gemm_bf16_pair.cu -- the two grouped expert GEMMs in bf16, each tile
// computed by a pair of CTAs on two SMs with one tcgen05 MMA (cta_group::2),
// expert weights as the MMA's M operand and routes as its N operand.
//
// Why weights are M: a tile holds the routes of one expert, and experts get
// very different numbers of routes (a Zipf-skewed router sends a few rows to
// most experts).  M of a pair MMA is fixed at 256, N may be any multiple of
// 16 up to 256; with routes along N the last tile of an expert costs its
// route count rounded up to 32, not a full 256-row tile.
//
//   gate/up:  A = 128 f values of expert e as 256 weight rows, 64 f per CTA,
//             B = N route rows of x.  The prepared W1 interleaves gate and up
//             so that each 32-lane TMEM quarter q of CTA r holds 16 f: lane
//             32q+i the gate value of f = f0 + 64r + 16q + i, lane 32q+16+i
//             the up value of the same f.  The warp reading a quarter swaps
//             half of its columns across the half-warps (shfl.xor 16), so
//             every lane forms h = silu(g) * u for 16 routes of one f, bf16
//             (Megatron-LM PR #7798, "Background": the activation is fused
//             into the FC1 epilogue).
//   down:     A = 256 rows of W_down[e] (output columns c0..c0+255, 128 per
//             CTA), B = N route rows of h; fp32 y out.
//
// Both epilogues transpose through shared memory so that y and h rows leave
// as coalesced 16-byte stores (one route row per store group).
//
// A K stage is 128 elements (two 128-byte swizzle atoms, 8 MMAs).  A is one
// TMA box of 32 KB that is contiguous in memory: the prepared weights are
// stored as blocks of [2 atoms][128 rows][64 elements], one per (expert,
// 128-row block, K stage), so the weight stream reads whole 32 KB runs.  B
// is an (N/2)-row x 2-atom box of padded route rows (one tensor map per N/2
// in {16, 32, ..., 128}; K pitches padded to 128 with zeros), except for
// gate/up tiles of at most 32 routes, which gather their x rows by token
// with tile::gather4 (four one-atom rows per instruction) instead.
//
// Roles (10 warps per CTA): warp 0 issues TMA loads in both CTAs (the
// completion of both halves is counted on CTA 0's "full" barrier); warp 1
// owns TMEM in both CTAs and, in CTA 0 only, issues the pair MMAs, whose
// completion is signalled to both CTAs' barriers (commit with a CTA mask);
// warps 2-9 drain the accumulators and release each accumulator on CTA 0's
// barrier.  Two accumulators of 256 fp32 columns (512 TMEM columns) per CTA.
// The gate/up kernel has two more warps that copy the x rows of tiles of
// more than 32 routes into their padded route rows while the MMAs run (the
// dispatch fused into the GEMM: no separate gather pass over HBM).  They
// claim 8-route chunks in tile order from a global counter and count each
// finished chunk in its tile's ready counter; a producer acquires that count
// before the tile's first route-row load.  The copy runs at most 16 tiles
// ahead of the highest tile a producer has started (rows copied further ahead
// leave L2 before their loads); a producer marks its tile before it waits for
// the tile's rows, chunks are claimed in tile order, and every CTA of the
// persistent grid is resident, so every one of these waits ends.
//
// Every mbarrier wait is bounded; the pair meets in cluster barriers only at
// start-up and before TMEM is released.  Each output element is one route's
// dot product over K in a fixed order with one instruction shape, so results
// do not depend on the tile or column a route lands in or on the live count.
#include "moe_internal.cuh"
#include "ptx.cuh"

namespace moe {
namespace {

constexpr int kStagesMax = 5;  // pipeline stages per launch: 3..5, by the widest route tile (see StageCfg)
constexpr int kEpiWarps = 8;
constexpr int kCopyWarps = 2;                           // gate/up: x rows of large tiles into their route rows
constexpr int kCopyAhead = 16;                          // route tiles the copy may run ahead of the producers
constexpr int kPairM = 256;                             // M of the pair MMA (weight rows)
constexpr int kAtoms = 2;                               // 64-element (128-byte) swizzle atoms per K stage
constexpr int kStageK = kAtoms * kBK;                   // 128 K elements per stage
constexpr uint32_t kAtomBytes = 128 * kBK * 2;          // 16 KB: 128 rows x 128 bytes
constexpr uint32_t kABytes = kAtoms * kAtomBytes;       // 32 KB: this CTA's 128 weight rows
constexpr uint32_t kBBytesMax = kAtoms * kAtomBytes;    // up to 32 KB: this CTA's N/2 <= 128 route rows
constexpr uint32_t kAccCols = 256;
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kHTBytes = 32 * 16 * 2 + 64;         // gate/up: h of 32 routes x 16 f, bf16 (+ bank offset)
constexpr uint32_t kRTBytes = 32 * 32 * 2;              // squared ReLU: h of 32 routes x 32 f, bf16
constexpr uint32_t kH0Bytes = kHTBytes > kRTBytes ? kHTBytes : kRTBytes;  // gate/up epilogue box per warp
constexpr uint32_t kYTBytes = 32 * 32 * 4;              // down: y of 32 routes x 32 c, fp32

template <int kMode>
struct PairCfg {
    static constexpr int kThreads = (2 + kEpiWarps + (kMode == 0 ? kCopyWarps : 0)) * 32;
    // one transpose box per epilogue warp
    static constexpr uint32_t kEpiBytes = kEpiWarps * (kMode == 0 ? kH0Bytes : kYTBytes);
    // the stages: gate/up up to 5 x (32 + 8) KB, down up to 4 x (32 + 16) KB; 3 x (32 + 32) KB at most width
    static constexpr uint32_t kStageRegion = kMode == 0 ? 5 * (kABytes + 8192) : 4 * (kABytes + 16384);
    static constexpr size_t kSmemBytes = 1024 + kStageRegion + kEpiBytes + 256;
    static_assert(kSmemBytes <= 232448, "shared memory budget");
    static_assert(kStageRegion >= 3 * (kABytes + kBBytesMax), "three full-width stages");
};

struct __align__(8) Barriers {
    uint64_t full[kStagesMax];   // CTA 0's counts both CTAs' loads of a stage
    uint64_t empty[kStagesMax];  // each CTA's: its stage may be refilled
    uint64_t acc_full[2];     // each CTA's: its accumulator rows are ready
    uint64_t acc_empty[2];    // CTA 0's: both CTAs drained the accumulator
    uint64_t done;
    uint32_t tmem_base;
    int abort_flag;
};

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

// Routes of a tile rounded up to the MMA's N granularity (both CTAs hold N/2 rows of B).
__device__ __forceinline__ int tile_n(int nvalid) { return (nvalid + 31) & ~31; }

// The pipeline of one launch, from the widest route tile of the forward
// (known after the permute): narrow tiles (decode) leave room for more stages
// in flight.  Weight slots (kABytes each) come first, at multiples of 32 KB,
// then the route-row slots.  Every CTA and role of the launch derives the same
// configuration.
struct StageCfg {
    int n;          // stages
    uint32_t b;     // route-row slot bytes
};
template <int kMode>
__device__ __forceinline__ StageCfg stage_cfg(int widest_tile) {
    const int hb = tile_n(widest_tile) >> 1;  // route rows per CTA
    if (kMode == 0 && hb <= 32) return {5, 8192u};
    if (hb <= 64) return {4, 16384u};
    return {3, kBBytesMax};
}

template <int kMode>  // 0: gate/up + SwiGLU -> bf16 h;  1: down -> fp32 y
__device__ __forceinline__ void pair_gemm_body(const CUtensorMap& tmA, const CUtensorMap* tmX, const BoxMaps8* tmB,
                                               const GemmParams& p) {
    constexpr uint32_t kEpiBytes = PairCfg<kMode>::kEpiBytes;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t* sA = smem;
    uint8_t* sEpi = smem + PairCfg<kMode>::kStageRegion;
    Barriers* bars = reinterpret_cast<Barriers*>(sEpi + kEpiBytes);
    volatile int* abort_flag = &bars->abort_flag;

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const uint32_t rank = cluster_ctarank();
    const bool leader = rank == 0;
    const int pair = (int)cluster_id_x();
    const int npairs = (int)cluster_count_x();
    pdl_trigger();

    if (threadIdx.x == 0) {
        for (int s = 0; s < kStagesMax; ++s) {
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
    pdl_wait();  // the tile list, x / h rows and status words come from earlier kernels

    const int num_m = forward_poisoned(p.status_words) ? 0 : (int)p.status_words[kStNumMTiles];
    const int total_tiles = num_m * p.n_tiles;
    const int kb_count = p.k_blocks;
    const StageCfg sc = stage_cfg<kMode>((int)p.status_words[kStMaxTileRows]);
    const int kStages = sc.n;
    const uint32_t kBBytes = sc.b;
    uint8_t* sB = smem + kStages * kABytes;

    if (warp == 0) {
        // ---------------- TMA producer (both CTAs; lane 0 waits and loads A, and B of the down GEMM)
        if (lane == 0) {
            tma_prefetch_desc(&tmA);
            if (kMode == 0) tma_prefetch_desc(tmX);
        }
        // When no expert has more than one route tile (decode), every weight tile is read by
        // one unit only: its lines go first out of L2, which keeps the h and y rows that the
        // next kernels read resident there instead of written back and read from HBM.
        const bool weights_once = (int)p.status_words[kStMaxTileRows] < kRouteTile;
        const uint64_t pol_once = l2_policy_evict_first();
        int stage = 0;
        uint32_t phase = 0;
        bool ok = true;
        int last_phase[kStagesMax];
        for (int s = 0; s < kStagesMax; ++s) last_phase[s] = -1;
        for (int t = pair; t < total_tiles && ok; t += npairs) {
            const int mt = t / p.n_tiles, nt = t - mt * p.n_tiles;
            const int4 ti = __ldg(p.tiles + mt);
            const int hb = tile_n(ti.z) >> 1;  // route rows of B in each CTA
            const uint32_t tx = 2u * (kABytes + (uint32_t)hb * (kAtoms * 128u));
            // this CTA's 128 weight rows: row block a_rb of the blocked weight buffer, whose
            // K stage kb is atoms 2 * (a_rb * kb_count + kb) and + 1
            const long long a_rb = ((long long)ti.x * p.a_rows + nt * kPairM + 128 * (int)rank) / 128;
            const int a_atom0 = (int)(a_rb * kb_count) * kAtoms;
            const int b_row = ti.y + hb * (int)rank;
            // gate/up tiles of at most kGatherInGemmMax routes: lane L gathers this CTA's B
            // rows 4L..4L+3 from x, the rows of the tokens of routes hb * rank + 4L + q
            // (rows past the tile's routes repeat its first token: in bounds, and their
            // output columns are never stored).  Larger tiles load their rows, written by
            // the copy warps, as one box: a gather moves 512 bytes per TMA instruction, too
            // few to feed a full tile.
            int tok[4] = {0, 0, 0, 0};
            const bool from_x = kMode == 0 && ti.z <= kGatherInGemmMax;
            const bool gathers = from_x && 4 * lane < hb;
            // mark this tile as started: the copy warps may now run up to kCopyAhead tiles past it
            if (kMode == 0 && leader && lane == 0) atomicMax(p.tile_started, mt);
            if (kMode == 0 && !from_x) {
                // the copy warps (of any CTA) have written all of this tile's route rows:
                // acquire their counts, then order them before this thread's TMA reads
                bool rdy = true;
                if (lane == 0) {
                    rdy = wait_count_bounded(p.ready + mt, (ti.z + kCopyChunk - 1) / kCopyChunk, abort_flag,
                                             p.wait_limit_ns);
                    fence_proxy_async_global();
                }
                if (!__shfl_sync(0xffffffffu, rdy, 0)) {
                    ok = false;
                    break;
                }
            }
            if (from_x) {
                const int first = __ldg(p.perm + ti.w) / p.top_k;
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    const int i = hb * (int)rank + 4 * lane + q;
                    tok[q] = i < ti.z ? __ldg(p.perm + ti.w + i) / p.top_k : first;
                }
            }
            for (int kb = 0; kb < kb_count; ++kb) {
                bool got = true;
                if (lane == 0) got = mbar_wait_bounded(&bars->empty[stage], phase ^ 1u, abort_flag, p.wait_limit_ns);
                if (!__shfl_sync(0xffffffffu, got, 0)) {
                    ok = false;
                    break;
                }
                const uint32_t full0 = map_to_cta(smem_u32(&bars->full[stage]), 0);
                if (lane == 0) {
                    if (leader) {
                        mbar_arrive_expect_tx(&bars->full[stage], tx);
                        last_phase[stage] = (int)phase;
                    }
                    // boxes land as [atom][row][64 elements]
                    if (weights_once)
                        tma_load_3d_pair_hint(sA + stage * kABytes, &tmA, full0, 0, 0, a_atom0 + kb * kAtoms, pol_once);
                    else
                        tma_load_3d_pair(sA + stage * kABytes, &tmA, full0, 0, 0, a_atom0 + kb * kAtoms);
                    if (!from_x)
                        tma_load_3d_pair(sB + stage * kBBytes, &tmB->m[(hb >> 4) - 1], full0, 0, b_row,
                                         kb * kAtoms);
                }
                if (gathers) {
#pragma unroll
                    for (int at = 0; at < kAtoms; ++at)
                        tma_gather4_pair(sB + stage * kBBytes + (uint32_t)at * (uint32_t)hb * 128u + lane * 512u,
                                         tmX, full0, kb * kStageK + at * kBK, tok[0], tok[1], tok[2], tok[3]);
                }
                if (++stage == kStages) {
                    stage = 0;
                    phase ^= 1u;
                }
            }
        }
        if (!ok && lane == 0) {
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
        __syncwarp();
    } else if (warp == 1) {
        if (lane == 0 && leader) {
            // ---------------- pair MMA issuer (CTA 0)
            int stage = 0;
            uint32_t phase = 0;
            bool ok = true;
            int it = 0;
            for (int t = pair; t < total_tiles && ok; t += npairs, ++it) {
                const int buf = it & 1;
                const uint32_t acc_phase = (uint32_t)(it >> 1) & 1u;
                const int mt = t / p.n_tiles;
                const int n = tile_n(__ldg(&p.tiles[mt].z));
                const uint32_t idesc = idesc_bf16_f32(kPairM, n);
                const uint32_t b_atom = (uint32_t)(n >> 1) * 128u;  // bytes of one atom of this CTA's B rows
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
                        const uint32_t koff = (uint32_t)(kk & 3) * 32;
                        mma_bf16_pair(d_tmem, sdesc_kmajor_sw128(a_addr + (uint32_t)(kk >> 2) * kAtomBytes + koff),
                                      sdesc_kmajor_sw128(b_addr + (uint32_t)(kk >> 2) * b_atom + koff), idesc,
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
    } else if (warp < 2 + kEpiWarps) {
        // ---------------- epilogue: warps 2..9
        const int ew = warp - 2;
        const int quad = warp & 3;   // TMEM lane quarter this warp may read
        const int half = ew >> 2;    // this warp takes the 32-route chunks c with c % 2 == half
        const uint32_t acc_empty0[2] = {map_to_cta(smem_u32(&bars->acc_empty[0]), 0),
                                        map_to_cta(smem_u32(&bars->acc_empty[1]), 0)};
        uint8_t* tbuf = sEpi + (size_t)ew * (kMode == 0 ? kH0Bytes : kYTBytes);
        // Experts with several route tiles (prefill): the weights and route rows are read
        // again by other units while h / y (larger than L2) stream out; the output lines go
        // first out of L2 so that they do not push the operands out.  With one tile per
        // expert (decode) the outputs stay, for the next kernel to read from L2.
        const bool out_first = (int)p.status_words[kStMaxTileRows] >= kRouteTile;
        const uint64_t pol_out = l2_policy_evict_first();
        auto store_out = [&](void* dst, uint4 w) {
            if (out_first)
                st_global_v4_hint(dst, w, pol_out);
            else
                *reinterpret_cast<uint4*>(dst) = w;
        };
        int it = 0;
        for (int t = pair; t < total_tiles; t += npairs, ++it) {
            const int buf = it & 1;
            const uint32_t acc_phase = (uint32_t)(it >> 1) & 1u;
            const int mt = t / p.n_tiles, nt = t - mt * p.n_tiles;
            const int4 ti = __ldg(p.tiles + mt);
            const int nch = tile_n(ti.z) >> 5;
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
            const uint32_t taddr = tmem_base + ((uint32_t)(quad * 32) << 16) + (uint32_t)buf * kAccCols;
            if (kMode == 0 && p.relu2) {
                // squared-ReLU experts: lane = f (this warp's 32 f from f0), register j = route
                // 32c + j; h = relu(g)^2 goes through a [route][32 f] bf16 box to 64-byte rows
                const int f0 = nt * kPairM + 128 * (int)rank + 32 * quad;
                __nv_bfloat16* h = reinterpret_cast<__nv_bfloat16*>(p.out);
                if (f0 < p.out_cols) {
#pragma unroll 1
                    for (int c = half; c < nch; c += 2) {
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
                            *reinterpret_cast<__nv_bfloat16*>(tbuf + j * 64 + lane * 2) = __float2bfloat16_rn(hv);
                        }
                        __syncwarp();
#pragma unroll
                        for (int i = 0; i < 4; ++i) {
                            const int r = i * 8 + (lane >> 2);
                            const int route = c * 32 + r;
                            const uint4 w = *reinterpret_cast<const uint4*>(tbuf + r * 64 + (lane & 3) * 16);
                            if (route < ti.z)
                                store_out(h + (size_t)(ti.y + route) * (size_t)p.out_ld + f0 + (lane & 3) * 8, w);
                        }
                        __syncwarp();
                    }
                }
            } else if (kMode == 0) {
                // f of this lane: f_base + (lane & 15); lanes < 16 hold gate, the others up
                const int f_base = nt * 128 + 64 * (int)rank + 16 * quad;
                const bool lo = lane < 16;
                // transpose box: route r at r * 32 bytes, routes 16..31 shifted by 64 bytes so that
                // the two half-warps' rows fall in different banks
                __nv_bfloat16* h = reinterpret_cast<__nv_bfloat16*>(p.out);
#pragma unroll 1
                for (int c = half; c < nch; c += 2) {
                    uint32_t v[32];
                    tmem_ld_32x32b_x32(taddr + c * 32, v);
                    // apply_topk_in_fc1: lane l fetches the probability of route 32c + l
                    float pv = 1.0f;
                    if (p.route_probs != nullptr && c * 32 + lane < ti.z)
                        pv = __ldg(p.route_probs + __ldg(p.perm + ti.w + c * 32 + lane));
                    tmem_ld_wait();
                    // lanes < 16 keep their gate values of routes 0..15 and receive the up values;
                    // lanes >= 16 keep their up values of routes 16..31 and receive the gate values
                    uint8_t* row0 = tbuf + (lo ? 0 : 16 * 32 + 64) + (lane & 15) * 2;
#pragma unroll
                    for (int j = 0; j < 16; ++j) {
                        const uint32_t mine = lo ? v[j] : v[16 + j];
                        const uint32_t other = __shfl_xor_sync(0xffffffffu, lo ? v[16 + j] : v[j], 16);
                        const float g = __uint_as_float(lo ? mine : other);
                        const float u = __uint_as_float(lo ? other : mine);
                        float hv = swiglu_value(g, u, p.clamp);
                        if (p.route_probs != nullptr) hv *= __shfl_sync(0xffffffffu, pv, lo ? j : 16 + j);
                        *reinterpret_cast<__nv_bfloat16*>(row0 + j * 32) = __float2bfloat16_rn(hv);
                    }
                    __syncwarp();
#pragma unroll
                    for (int i = 0; i < 2; ++i) {
                        const int r = i * 16 + (lane >> 1);
                        const int route = c * 32 + r;
                        const uint4 w = *reinterpret_cast<const uint4*>(tbuf + r * 32 + (r >= 16 ? 64 : 0) +
                                                                        (lane & 1) * 16);
                        if (route < ti.z)
                            store_out(h + (size_t)(ti.y + route) * (size_t)p.out_ld + f_base + (lane & 1) * 8, w);
                    }
                    __syncwarp();
                }
            } else {
                // output columns of this warp: nt*256 + 128*rank + 32*quad + lane
                const int c_base = nt * kPairM + 128 * (int)rank + 32 * quad;
                float* y = reinterpret_cast<float*>(p.out);
                if (c_base < p.out_cols) {
                    const bool col_ok = c_base + (lane & 7) * 4 < p.out_cols;
#pragma unroll 1
                    for (int c = half; c < nch; c += 2) {
                        uint32_t v[32];
                        tmem_ld_32x32b_x32(taddr + c * 32, v);
                        tmem_ld_wait();
                        // transpose: [route][32 c] fp32, 128 bytes per route
#pragma unroll
                        for (int r = 0; r < 32; ++r) *reinterpret_cast<uint32_t*>(tbuf + r * 128 + lane * 4) = v[r];
                        __syncwarp();
#pragma unroll
                        for (int i = 0; i < 8; ++i) {
                            const int r = i * 4 + (lane >> 3);
                            const int route = c * 32 + r;
                            const uint4 w = *reinterpret_cast<const uint4*>(tbuf + r * 128 + (lane & 7) * 16);
                            if (col_ok && route < ti.z)
                                store_out(y + (size_t)(ti.y + route) * (size_t)p.out_ld + c_base + (lane & 7) * 4, w);
                        }
                        __syncwarp();
                    }
                }
            }
            tc_fence_before_sync();
            __syncwarp();
            if (lane == 0) mbar_arrive_cluster(acc_empty0[buf]);  // release on CTA 0's barrier
        }
    } else if constexpr (kMode == 0) {
        // ---------------- copy warps (gate/up): the x rows of tiles of more than
        // kGatherInGemmMax routes into their padded route rows, one 8-route chunk at a
        // time, claimed in tile order so that the first tiles the producers load are
        // the first complete.  A chunk's rows are made visible (and ordered before TMA
        // reads) before it is counted in ready[tile].
        const unsigned units = (unsigned)num_m * kChunksPerTile;
        const int chunks_in = p.x_bytes >> 4;  // 16-byte chunks of an x row
        const int chunks_out = (int)(p.xg_pitch >> 4);
        while (true) {
            unsigned u = 0;
            if (lane == 0) u = atomicAdd(p.copy_next, 1u);
            u = __shfl_sync(0xffffffffu, u, 0);
            if (u >= units || *abort_flag != 0) break;
            const int mt = (int)(u / kChunksPerTile);
            const int r0 = (int)(u % kChunksPerTile) * kCopyChunk;
            const int4 ti = __ldg(p.tiles + mt);
            if (ti.z <= kGatherInGemmMax || r0 >= ti.z) continue;
            // stay at most kCopyAhead tiles ahead of the highest tile a producer has started:
            // rows copied further ahead would leave L2 before their loads and come back from
            // HBM.  A producer marks its tile before it waits for the tile's rows, so this
            // wait ends whenever a producer waits on this chunk.
            bool go = true;
            if (lane == 0 && mt > kCopyAhead)
                go = wait_count_bounded(p.tile_started, mt - kCopyAhead, abort_flag, p.wait_limit_ns);
            if (!__shfl_sync(0xffffffffu, go, 0)) {
                if (lane == 0) {
                    *abort_flag = 1;
                    atomicOr(p.status_flags, MOE_DEV_TIMEOUT);
                }
                break;
            }
            const int nrows = min(kCopyChunk, ti.z - r0);
            const int my_tok = lane < nrows ? __ldg(p.perm + ti.w + r0 + lane) / p.top_k : 0;
            // two rows at a time: 16 loads of 16 bytes in flight per lane
#pragma unroll 1
            for (int i = 0; i < nrows; i += 2) {
                const bool two = i + 1 < nrows;
                const int tok0 = __shfl_sync(0xffffffffu, my_tok, i);
                const int tok1 = __shfl_sync(0xffffffffu, my_tok, two ? i + 1 : i);
                const uint4* src0 = reinterpret_cast<const uint4*>(p.x + (size_t)tok0 * (size_t)p.x_pitch);
                const uint4* src1 = reinterpret_cast<const uint4*>(p.x + (size_t)tok1 * (size_t)p.x_pitch);
                uint4* dst0 = reinterpret_cast<uint4*>(p.xg + (size_t)(ti.y + r0 + i) * (size_t)p.xg_pitch);
                uint4* dst1 = reinterpret_cast<uint4*>(reinterpret_cast<uint8_t*>(dst0) + p.xg_pitch);
                for (int c0 = 0; c0 < chunks_out; c0 += 8 * 32) {
                    uint4 v0[8], v1[8];
#pragma unroll
                    for (int j = 0; j < 8; ++j) {
                        const int ch = c0 + j * 32 + lane;
                        const bool in = ch < chunks_in;
                        v0[j] = in ? __ldg(src0 + ch) : make_uint4(0u, 0u, 0u, 0u);
                        v1[j] = in && two ? __ldg(src1 + ch) : make_uint4(0u, 0u, 0u, 0u);
                    }
#pragma unroll
                    for (int j = 0; j < 8; ++j) {
                        const int ch = c0 + j * 32 + lane;
                        if (ch < chunks_out) {
                            dst0[ch] = v0[j];
                            if (two) dst1[ch] = v1[j];
                        }
                    }
                }
            }
            fence_proxy_async_global();
            __threadfence();
            __syncwarp();
            if (lane == 0) red_release_gpu_add(p.ready + mt, 1);
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

__global__ void __launch_bounds__(PairCfg<0>::kThreads, 1)
    moe_gemm_gate_up_swiglu_bf16_pair(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmX,
                                      const __grid_constant__ BoxMaps8 tmB, const GemmParams p) {
    pair_gemm_body<0>(tmA, &tmX, &tmB, p);
}

__global__ void __launch_bounds__(PairCfg<1>::kThreads, 1)
    moe_gemm_down_bf16_pair(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ BoxMaps8 tmB,
                            const GemmParams p) {
    pair_gemm_body<1>(tmA, nullptr, &tmB, p);
}


struct PairLaunchCache {
    size_t smem = 0;
    int threads = 0;
    int device = -1;
    int pairs = 0;
};

template <class... Operands>
cudaError_t launch_pair(void (*kern)(CUtensorMap, Operands..., GemmParams), PairLaunchCache* cache,
                        const CUtensorMap& a, const Operands&... b, const GemmParams& gp, long long max_tiles,
                        cudaStream_t s) {
    int dev = 0;
    cudaError_t err = cudaGetDevice(&dev);
    if (err != cudaSuccess) return err;
    cudaLaunchConfig_t cfg = {};
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;  // see pdl_wait()
    attr[1].val.programmaticStreamSerializationAllowed = 1;
    cfg.blockDim = dim3(cache->threads);
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
    cfg.numAttrs = 2;
    err = cudaLaunchKernelEx(&cfg, kern, a, b..., gp);
    if (err != cudaSuccess) return err;
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_gemm1_bf16_pair(const CUtensorMap& a, const CUtensorMap& x_rows, const BoxMaps8& b,
                                   const GemmParams& gp, long long max_tiles, cudaStream_t s) {
    static PairLaunchCache cache{PairCfg<0>::kSmemBytes, PairCfg<0>::kThreads};
    return launch_pair<CUtensorMap, BoxMaps8>(moe_gemm_gate_up_swiglu_bf16_pair, &cache, a, x_rows, b, gp, max_tiles,
                                              s);
}

cudaError_t launch_gemm2_bf16_pair(const CUtensorMap& a, const BoxMaps8& b, const GemmParams& gp, long long max_tiles,
                                   cudaStream_t s) {
    static PairLaunchCache cache{PairCfg<1>::kSmemBytes, PairCfg<1>::kThreads};
    return launch_pair<BoxMaps8>(moe_gemm_down_bf16_pair, &cache, a, b, gp, max_tiles, s);
}

}  // namespace moe
