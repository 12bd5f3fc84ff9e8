// api.cu -- the C ABI declared in include/moe.h: plan validation, buffer
// layouts, TMA descriptors and the launch sequence of the forward.
#include <cudaTypedefs.h>

#include <cstdlib>
#include <cstring>
#include <new>

#include "ep.cuh"
#include "moe_internal.cuh"

namespace moe {

// ---------------------------------------------------------------- device info

int num_sms() {
    static int cached[64];
    static bool have[64];
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 148;
    if (!have[dev]) {
        int n = 0;
        if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) n = 148;
        cached[dev] = n;
        have[dev] = true;
    }
    return cached[dev];
}

// ---------------------------------------------------------------- TMA descriptors

static PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;

bool get_tensor_map_encoder() {
    if (g_encode != nullptr) return true;
    void* fn = nullptr;
    cudaDriverEntryPointQueryResult q{};
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &fn, 12000, cudaEnableDefault, &q) !=
            cudaSuccess ||
        q != cudaDriverEntryPointSuccess || fn == nullptr)
        return false;
    g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
    return true;
}

bool make_tensor_map(CUtensorMap* map, CUtensorMapDataType dtype, int rank, const void* base,
                     const unsigned long long* dims, const unsigned long long* strides_bytes, const unsigned* box,
                     CUtensorMapSwizzle swizzle) {
    if (!get_tensor_map_encoder()) return false;
    cuuint64_t gdim[5];
    cuuint64_t gstride[4];
    cuuint32_t bdim[5];
    cuuint32_t estride[5];
    for (int i = 0; i < rank; ++i) {
        gdim[i] = dims[i];
        bdim[i] = box[i];
        estride[i] = 1;
        if (i + 1 < rank) gstride[i] = strides_bytes[i];
    }
    const CUresult r = g_encode(map, dtype, (cuuint32_t)rank, const_cast<void*>(base), gdim, gstride, bdim, estride,
                                CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                                CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

static size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

static void compute_layouts(moe_plan* p) {
    const size_t H = (size_t)p->d.hidden, E = (size_t)p->d.num_experts;
    const size_t k = (size_t)p->d.top_k;
    const size_t L = (size_t)p->max_live;
    const size_t R = (size_t)p->rows_pad;
    const bool fp8 = p->d.precision == MOE_MXFP8;
    WsLayout& w = p->ws;
    size_t off = 0;
    auto take = [&off](size_t bytes) {
        const size_t at = off;
        off += align256(bytes);
        return at;
    };
    w.status = take(kStWords * 4);
    w.r_ids = take(L * k * 4);
    w.r_probs = take(L * k * 4);
    w.blkcnt = take(((size_t)p->nblk + 1) * E * 4);  // per-chunk counts, then the per-expert totals
    w.offsets = take((E + 1) * 4);
    w.padoff = take((E + 1) * 4);
    w.tiles = take((size_t)p->max_m_tiles * 16);
    w.perm = take(L * k * 4);
    w.inv = take(L * k * 4);
    const size_t mtiles = (size_t)p->max_m_tiles;
    const bool fp4 = p->d.precision == MOE_NVFP4;
    w.ready = fp8 || fp4 ? 0 : take(mtiles * 4);
    w.xg = w.hf = w.hg = 0;
    if (fp4) {
        // codes two per byte; four 512-byte scale blocks per 128-row tile and K block of 256
        w.xq = take(R * (size_t)p->hp / 2);
        w.xs = take(mtiles * p->ks1 * 4 * kSfBlock);
        w.xg = take(R * 4);
        w.hf = take(R * (size_t)p->fp * 4);
        w.h = take(R * (size_t)p->fp / 2);
        w.hs = take(mtiles * p->ks2 * 4 * kSfBlock);
        w.hg = take(R * 4);
    } else if (fp8) {
        w.xq = take(R * (size_t)p->hp);
        w.xs = take(mtiles * p->ks1 * kSfBlock);
        w.h = take(R * (size_t)p->fp);
        w.hs = take(mtiles * p->ks2 * kSfBlock);
        if ((p->d.flags & MOE_FLAG_KEEP_H_FP32) != 0) w.hf = take(R * (size_t)p->fp * 4);
    } else {
        w.xq = take(R * (size_t)p->hp * 2);  // x rows of tiles of more than kGatherInGemmMax routes
        w.xs = 0;
        w.h = take(R * (size_t)p->fp * 2);
        w.hs = 0;
    }
    w.y = take(R * H * 4);
    w.total = off;

    WbufLayout& b = p->wb;
    off = 0;
    b.wg = 0;
    if (fp4) {
        b.w1 = take(E * (size_t)p->w1r * (size_t)p->hp / 2);
        b.w1s = take(E * p->nt1 * p->ks1 * 4 * kSfBlock);
        b.w2 = take(E * H * (size_t)p->fp / 2);
        b.w2s = take(E * p->nt2 * p->ks2 * 4 * kSfBlock);
        b.wg = take(E * 2 * 4);
    } else if (fp8) {
        b.w1 = take(E * (size_t)p->w1r * (size_t)p->hp);
        b.w1s = take(E * p->nt1 * p->ks1 * kSfBlock);
        b.w2 = take(E * H * (size_t)p->fp);
        b.w2s = take(E * p->nt2 * p->ks2 * kSfBlock);
    } else {
        b.w1 = take(E * (size_t)p->w1r * (size_t)p->hp * 2);
        b.w1s = 0;
        b.w2 = take(E * (size_t)p->hr * (size_t)p->fp * 2);
        b.w2s = 0;
    }
    b.total = off;
}

static bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; }

}  // namespace moe

using namespace moe;

extern "C" {

const char* moe_version(void) { return "0.1.0"; }

const char* moe_status_string(moe_status s) {
    switch (s) {
        case MOE_OK: return "ok";
        case MOE_ERR_INVALID_ARG: return "invalid argument";
        case MOE_ERR_UNSUPPORTED: return "unsupported configuration";
        case MOE_ERR_ALIGNMENT: return "pointer or stride not aligned";
        case MOE_ERR_WORKSPACE_TOO_SMALL: return "workspace or weight buffer too small";
        case MOE_ERR_CUDA: return "CUDA runtime error";
        case MOE_ERR_NOT_PREPARED: return "weight buffer not prepared";
    }
    return "unknown status";
}

moe_status moe_plan_create(const moe_desc* desc, moe_plan** plan_out) {
    if (desc == nullptr || plan_out == nullptr) return MOE_ERR_INVALID_ARG;
    *plan_out = nullptr;
    const moe_desc& d = *desc;
    if (d.precision != MOE_BF16 && d.precision != MOE_MXFP8 && d.precision != MOE_NVFP4) return MOE_ERR_INVALID_ARG;
    const bool blockscaled = d.precision != MOE_BF16;  // MXFP8 or NVFP4: one CTA, 128-row tiles
    if (d.hidden <= 0 || d.ffn <= 0 || d.num_experts <= 0 || d.top_k <= 0 || d.capacity <= 0)
        return MOE_ERR_UNSUPPORTED;
    const int mult = blockscaled ? 32 : 8;
    if (d.hidden % mult != 0 || d.ffn % mult != 0) return MOE_ERR_UNSUPPORTED;
    if (d.hidden > 16384 || d.ffn > 16384) return MOE_ERR_UNSUPPORTED;
    if (d.num_experts > kMaxExperts || d.top_k > kMaxTopK || d.top_k > d.num_experts) return MOE_ERR_UNSUPPORTED;
    if (d.capacity > (1ll << 24)) return MOE_ERR_UNSUPPORTED;
    if (d.max_live_rows < 0 || d.max_live_rows > d.capacity) return MOE_ERR_UNSUPPORTED;
    if ((d.flags & ~(MOE_FLAG_PROBS_IN_FC1 | MOE_FLAG_OUT_BF16 | MOE_FLAG_SQUARED_RELU | MOE_FLAG_KEEP_H_FP32)) != 0)
        return MOE_ERR_INVALID_ARG;
    if ((d.flags & MOE_FLAG_KEEP_H_FP32) != 0 && d.precision == MOE_BF16) return MOE_ERR_INVALID_ARG;
    if (!(d.gate_up_clamp >= 0.0f) || d.gate_up_clamp > 3.0e38f) return MOE_ERR_INVALID_ARG;
    moe_plan* p = new (std::nothrow) moe_plan();
    if (p == nullptr) return MOE_ERR_INVALID_ARG;
    p->d = d;
    p->max_live = d.max_live_rows > 0 ? d.max_live_rows : d.capacity;
    p->d.max_live_rows = p->max_live;
    p->max_routes = p->max_live * d.top_k;
    p->tile_rows = blockscaled ? kBM : kRouteTile;
    p->row_align = blockscaled ? kBM : kRouteAlign;
    p->max_m_tiles = (p->max_routes + p->tile_rows - 1) / p->tile_rows + d.num_experts;
    // every expert's rows are padded to row_align: at most routes + E * row_align rows
    p->rows_pad = blockscaled ? p->max_m_tiles * p->tile_rows
                                           : p->max_routes + (long long)d.num_experts * p->row_align;
    p->nblk = (int)((p->max_live + kTokPerBlk - 1) / kTokPerBlk);
    // K in blocks of 128 elements (bf16: the GEMMs' K stage; MXFP8: the unit of the scale
    // blocks, two per K stage); K pitches padded to whole blocks with zeros
    // (NVFP4: K blocks of 256 elements, which are 128 bytes of codes as in MXFP8)
    const int kblk = d.precision == MOE_NVFP4 ? 256 : 128;
    p->ks1 = (d.hidden + kblk - 1) / kblk;
    p->ks2 = (d.ffn + kblk - 1) / kblk;
    p->hp = (long long)p->ks1 * kblk;
    p->fp = (long long)p->ks2 * kblk;
    p->hr = p->hp;
    // FC1 rows per expert: gate and up interleaved (2 fp), or one projection (squared-ReLU
    // experts), padded to whole weight tiles (bf16: pair tiles of 256 rows; MXFP8: 128)
    const bool relu2 = (d.flags & MOE_FLAG_SQUARED_RELU) != 0;
    p->w1r = !relu2 ? 2 * p->fp : (blockscaled ? p->fp : (p->fp + 255) / 256 * 256);
    if (blockscaled) {
        p->nt1 = (int)(p->w1r / 128);  // weight tiles of 128 rows; h's padding columns come out zero
        p->nt2 = (d.hidden + kG2BN8 - 1) / kG2BN8;
    } else {
        p->nt1 = (int)(p->w1r / 256);  // pair tiles of 256 FC1 rows (SwiGLU: 128 f of gate and up)
        p->nt2 = (d.hidden + kG2BN - 1) / kG2BN;
    }
    compute_layouts(p);
    *plan_out = p;
    return MOE_OK;
}

void moe_plan_destroy(moe_plan* plan) { delete plan; }

moe_status moe_plan_get_desc(const moe_plan* plan, moe_desc* desc_out) {
    if (plan == nullptr || desc_out == nullptr) return MOE_ERR_INVALID_ARG;
    *desc_out = plan->d;
    return MOE_OK;
}

size_t moe_weight_buffer_bytes(const moe_plan* plan) { return plan ? plan->wb.total : 0; }
size_t moe_workspace_bytes(const moe_plan* plan) { return plan ? plan->ws.total : 0; }

moe_status moe_prepare_weights(const moe_plan* plan, const void* w_gate, const void* w_up, const void* w_down,
                               void* kernel_buf, size_t buf_bytes, void* stream) {
    const bool relu2 = plan != nullptr && (plan->d.flags & MOE_FLAG_SQUARED_RELU) != 0;
    if (plan == nullptr || w_gate == nullptr || (w_up == nullptr && !relu2) || w_down == nullptr ||
        kernel_buf == nullptr)
        return MOE_ERR_INVALID_ARG;
    if (buf_bytes < plan->wb.total) return MOE_ERR_WORKSPACE_TOO_SMALL;
    if (!aligned(w_gate, 16) || !aligned(relu2 ? w_gate : w_up, 16) || !aligned(w_down, 16) ||
        !aligned(kernel_buf, 256))
        return MOE_ERR_ALIGNMENT;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const auto* g = static_cast<const __nv_bfloat16*>(w_gate);
    const auto* u = static_cast<const __nv_bfloat16*>(w_up);
    const auto* dn = static_cast<const __nv_bfloat16*>(w_down);
    const cudaError_t e = plan->d.precision == MOE_MXFP8   ? launch_prepare_mxfp8(plan, g, u, dn, kernel_buf, s)
                          : plan->d.precision == MOE_NVFP4 ? launch_prepare_nvfp4(plan, g, u, dn, kernel_buf, s)
                                                           : launch_prepare_bf16(plan, g, u, dn, kernel_buf, s);
    return e == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

moe_status mxfp8_quantize_block32(const void* in, long long rows, int cols, long long ld_in, uint8_t* q,
                                  uint8_t* scales, const int* live_rows_dev, void* stream) {
    if (in == nullptr || q == nullptr || scales == nullptr) return MOE_ERR_INVALID_ARG;
    if (rows < 0 || cols <= 0 || ld_in < cols) return MOE_ERR_INVALID_ARG;
    if (cols % 32 != 0) return MOE_ERR_UNSUPPORTED;
    if (ld_in % 8 != 0 || !aligned(in, 16) || !aligned(q, 8)) return MOE_ERR_ALIGNMENT;
    if (rows == 0) return MOE_OK;
    const cudaError_t e = launch_quantize_rows(static_cast<const __nv_bfloat16*>(in), rows, cols, ld_in, q, scales,
                                               live_rows_dev, static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

moe_status nvfp4_quantize_block16(const void* in, long long rows, int cols, long long ld_in, uint8_t* q,
                                  uint8_t* scales, float* row_scales, const int* live_rows_dev, void* stream) {
    if (in == nullptr || q == nullptr || scales == nullptr || row_scales == nullptr) return MOE_ERR_INVALID_ARG;
    if (rows < 0 || cols <= 0 || ld_in < cols) return MOE_ERR_INVALID_ARG;
    if (cols % 32 != 0) return MOE_ERR_UNSUPPORTED;
    if (ld_in % 8 != 0 || !aligned(in, 16) || !aligned(q, 4) || !aligned(row_scales, 4)) return MOE_ERR_ALIGNMENT;
    if (rows == 0) return MOE_OK;
    const cudaError_t e = launch_nvfp4_quantize_rows(static_cast<const __nv_bfloat16*>(in), rows, cols, ld_in, q,
                                                     scales, row_scales, live_rows_dev,
                                                     static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

moe_status moe_route_topk(const moe_plan* plan, const float* logits, const int* live_count_dev, int* ids,
                          float* probs, void* stream) {
    if (plan == nullptr || logits == nullptr || live_count_dev == nullptr || ids == nullptr || probs == nullptr)
        return MOE_ERR_INVALID_ARG;
    const cudaError_t e = launch_route_topk(logits, live_count_dev, (int)plan->max_live, plan->d.num_experts,
                                            plan->d.top_k, ids, probs, nullptr, static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

}  // extern "C"

namespace {

static moe_status forward_impl(const moe_plan* plan, const void* x, const float* logits, const int* ids,
                               const float* probs, const void* kernel_buf, const int* live_count_dev, void* out,
                               void* workspace, size_t ws_bytes, void* stream, void* const* stage_events) {
    if (plan == nullptr || x == nullptr || kernel_buf == nullptr || live_count_dev == nullptr || out == nullptr ||
        workspace == nullptr)
        return MOE_ERR_INVALID_ARG;
    const bool have_logits = logits != nullptr;
    const bool have_routes = ids != nullptr && probs != nullptr;
    if (have_logits == have_routes || ((ids == nullptr) != (probs == nullptr))) return MOE_ERR_INVALID_ARG;
    if (ws_bytes < plan->ws.total) return MOE_ERR_WORKSPACE_TOO_SMALL;
    if (!aligned(x, 16) || !aligned(out, 16) || !aligned(workspace, 256) || !aligned(kernel_buf, 256))
        return MOE_ERR_ALIGNMENT;

    cudaStream_t s = static_cast<cudaStream_t>(stream);
    // Under stream capture the events are recorded as "external" so that the
    // graph gets real event-record nodes; outside capture a plain record.
    cudaStreamCaptureStatus capturing = cudaStreamCaptureStatusNone;
    if (stage_events != nullptr && cudaStreamIsCapturing(s, &capturing) != cudaSuccess) return MOE_ERR_CUDA;
    const unsigned record_flags =
        capturing == cudaStreamCaptureStatusActive ? cudaEventRecordExternal : cudaEventRecordDefault;
    auto mark = [&](int i) -> bool {
        return stage_events == nullptr ||
               cudaEventRecordWithFlags(static_cast<cudaEvent_t>(stage_events[i]), s, record_flags) == cudaSuccess;
    };
    const int H = plan->d.hidden, E = plan->d.num_experts, k = plan->d.top_k;
    const int max_live = (int)plan->max_live;
    uint8_t* ws = static_cast<uint8_t*>(workspace);
    const uint8_t* wb = static_cast<const uint8_t*>(kernel_buf);
    const WsLayout& L = plan->ws;
    unsigned* status = reinterpret_cast<unsigned*>(ws + L.status);
    int* r_ids = reinterpret_cast<int*>(ws + L.r_ids);
    float* r_probs = reinterpret_cast<float*>(ws + L.r_probs);

    // TMA descriptors for this call's buffers (host-side encoding only)
    const bool fp8 = plan->d.precision == MOE_MXFP8;
    const bool fp4 = plan->d.precision == MOE_NVFP4;
    const unsigned long long R = (unsigned long long)plan->rows_pad;
    const unsigned long long uH = (unsigned long long)H, uE = (unsigned long long)E;
    const CUtensorMapDataType dt = fp8 || fp4 ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
    CUtensorMap tA1, tA2;  // weight operands
    BoxMaps8 rB1, rB2;     // route-row operands (x rows, h rows)
    CUtensorMap tX;        // bf16: x rows, gathered by token
    if (fp8 || fp4) {
        // MXFP8 / NVFP4 (one CTA per tile): K stage = 256 bytes of codes (256 E4M3 or 512
        // E2M1 elements) = two 128-byte swizzle atoms; the maps address byte b of a row as
        // (b % 128, row, b / 128), so a box lands as [atom][row][128 bytes].  Weights (A) load
        // 128 rows, route rows (B) N <= 128 rows, one map per N in {32, 64, 96, 128}; the
        // K pitches (hp, fp elements) are whole 128-byte blocks padded with zero codes.
        const unsigned long long hp = (unsigned long long)(fp4 ? plan->hp / 2 : plan->hp);
        const unsigned long long fpp = (unsigned long long)(fp4 ? plan->fp / 2 : plan->fp);
        const unsigned box128[3] = {128, 128, 2};
        const unsigned long long dW1[3] = {128ull, uE * (unsigned long long)plan->w1r, hp / 128};
        const unsigned long long sW1[2] = {hp, 128ull};
        const unsigned long long dW2[3] = {128ull, uE * uH, fpp / 128};
        const unsigned long long sW2[2] = {fpp, 128ull};
        const unsigned long long dX[3] = {128ull, R, hp / 128};
        const unsigned long long dH[3] = {128ull, R, fpp / 128};
        if (!make_tensor_map(&tA1, dt, 3, wb + plan->wb.w1, dW1, sW1, box128, CU_TENSOR_MAP_SWIZZLE_128B) ||
            !make_tensor_map(&tA2, dt, 3, wb + plan->wb.w2, dW2, sW2, box128, CU_TENSOR_MAP_SWIZZLE_128B))
            return MOE_ERR_CUDA;
        for (int i = 0; i < 4; ++i) {
            const unsigned box[3] = {128, 32u * (unsigned)(i + 1), 2};
            if (!make_tensor_map(&rB1.m[i], dt, 3, ws + L.xq, dX, sW1, box, CU_TENSOR_MAP_SWIZZLE_128B) ||
                !make_tensor_map(&rB2.m[i], dt, 3, ws + L.h, dH, sW2, box, CU_TENSOR_MAP_SWIZZLE_128B))
                return MOE_ERR_CUDA;
        }
    } else {
        // bf16 (CTA pairs): K stage = 128 elements = two 64-element swizzle atoms, and
        // every operand box lands as [atom][row][64 elements].  The permuted x rows and h
        // have their K pitch padded to 128 (hp, fp) with zeros; their maps address element
        // k of a row as (k % 64, row, k / 64), the box's third dimension walking the two
        // atoms.  Weights (A) load 128 rows per CTA; route rows (B) N/2 rows, one map per N/2 in
        // {16, ..., 128}.  Gate/up tiles of at most kGatherInGemmMax routes instead gather
        // their B rows straight from x (one-row boxes of one atom, four rows per
        // instruction; columns past H read as zeros); the gate/up GEMM's copy warps write
        // the permuted x rows of the larger tiles ahead of their loads.
        const unsigned long long hp = (unsigned long long)plan->hp, fpp = (unsigned long long)plan->fp;
        // weights: blocks of [2 atoms][128 rows][64 elements], 32 KB contiguous, one per
        // (expert, 128-row block, K stage); atom a of block b is index 2b + a of the map's
        // third dimension
        const unsigned box128[3] = {64, 128, 2};
        const unsigned long long dW1[3] = {64ull, 128ull,
                                           2ull * (uE * (unsigned long long)plan->w1r / 128) * (hp / 128)};
        const unsigned long long dW2[3] = {64ull, 128ull, 2ull * (uE * (unsigned long long)plan->hr / 128) * (fpp / 128)};
        const unsigned long long sWb[2] = {128ull, 128ull * 128ull};
        const unsigned long long sW1[2] = {hp * 2, 128ull};
        const unsigned long long sW2[2] = {fpp * 2, 128ull};
        const unsigned long long dXP[3] = {64ull, R, hp / 64};
        const unsigned long long dH[3] = {64ull, R, fpp / 64};
        const unsigned long long dX[2] = {uH, (unsigned long long)plan->d.capacity};
        const unsigned long long sX[1] = {uH * 2};
        const unsigned boxX[2] = {64, 1};
        if (!make_tensor_map(&tA1, dt, 3, wb + plan->wb.w1, dW1, sWb, box128, CU_TENSOR_MAP_SWIZZLE_128B) ||
            !make_tensor_map(&tA2, dt, 3, wb + plan->wb.w2, dW2, sWb, box128, CU_TENSOR_MAP_SWIZZLE_128B) ||
            !make_tensor_map(&tX, dt, 2, x, dX, sX, boxX, CU_TENSOR_MAP_SWIZZLE_128B))
            return MOE_ERR_CUDA;
        for (int i = 0; i < 8; ++i) {
            const unsigned box[3] = {64, 16u * (unsigned)(i + 1), 2};
            if (!make_tensor_map(&rB1.m[i], dt, 3, ws + L.xq, dXP, sW1, box, CU_TENSOR_MAP_SWIZZLE_128B) ||
                !make_tensor_map(&rB2.m[i], dt, 3, ws + L.h, dH, sW2, box, CU_TENSOR_MAP_SWIZZLE_128B))
                return MOE_ERR_CUDA;
        }
    }

    cudaError_t e;
    if (!mark(0)) return MOE_ERR_CUDA;
    if (have_logits)
        e = launch_route_topk(logits, live_count_dev, max_live, E, k, r_ids, r_probs, status, s);
    else
        e = launch_canon_routes(ids, probs, live_count_dev, max_live, E, k, r_ids, r_probs, status, s);
    if (e != cudaSuccess) return MOE_ERR_CUDA;

    if (!mark(1)) return MOE_ERR_CUDA;
    int* perm = reinterpret_cast<int*>(ws + L.perm);
    int* inv = reinterpret_cast<int*>(ws + L.inv);
    int4* tiles = reinterpret_cast<int4*>(ws + L.tiles);
    int* ready = fp8 || fp4 ? nullptr : reinterpret_cast<int*>(ws + L.ready);  // bf16 only
    e = launch_permute(plan, live_count_dev, r_ids, reinterpret_cast<int*>(ws + L.blkcnt),
                       reinterpret_cast<int*>(ws + L.offsets), reinterpret_cast<int*>(ws + L.padoff), tiles, perm, inv,
                       ready, status, s);
    if (e != cudaSuccess) return MOE_ERR_CUDA;

    if (!mark(2)) return MOE_ERR_CUDA;
    if (fp8) {  // bf16: the gate/up GEMM copies the x rows itself
        e = launch_gather_mxfp8(static_cast<const __nv_bfloat16*>(x), live_count_dev, max_live, H, (int)plan->hp, k,
                                inv, ws + L.xq, ws + L.xs, status, s);
        if (e != cudaSuccess) return MOE_ERR_CUDA;
    } else if (fp4) {
        e = launch_gather_nvfp4(static_cast<const __nv_bfloat16*>(x), live_count_dev, max_live, H, (int)plan->hp, k,
                                inv, ws + L.xq, ws + L.xs, reinterpret_cast<float*>(ws + L.xg), status, s);
        if (e != cudaSuccess) return MOE_ERR_CUDA;
    }

    const long long m_tiles = plan->max_m_tiles;
    GemmParams g1{};
    g1.tiles = tiles;
    g1.status_words = status;
    g1.status_flags = status + kStFlags;
    g1.out = fp4 ? ws + L.hf : ws + L.h;  // NVFP4: fp32 h rows for the per-row quantisation pass
    g1.out_scales = nullptr;
    g1.out_ld = plan->fp;  // h rows: F values + zero padding to the down GEMM's K pitch
    g1.out_cols = (int)plan->fp;  // every padded column: f >= F are zero-weight rows, h = 0
    g1.a_rows = plan->w1r;  // FC1 weight rows of an expert
    g1.n_tiles = plan->nt1;
    g1.k_blocks = plan->ks1;
    g1.wait_limit_ns = kWaitLimitNs;
    g1.sfa = wb + plan->wb.w1s;  // MXFP8: A = weights, B = route rows
    g1.sfb = ws + L.xs;
    g1.out_scales = fp8 ? ws + L.hs : nullptr;
    g1.sf_ks_out = plan->ks2;
    g1.perm = perm;
    g1.top_k = k;
    const bool probs_in_fc1 = (plan->d.flags & MOE_FLAG_PROBS_IN_FC1) != 0;
    g1.route_probs = probs_in_fc1 ? r_probs : nullptr;
    g1.clamp = plan->d.gate_up_clamp;
    g1.relu2 = (plan->d.flags & MOE_FLAG_SQUARED_RELU) != 0;
    g1.x = static_cast<const uint8_t*>(x);
    g1.x_pitch = (long long)H * 2;
    g1.x_bytes = H * 2;
    g1.xg = ws + L.xq;
    g1.xg_pitch = plan->hp * 2;
    g1.ready = ready;
    g1.copy_next = status + kStCopyNext;
    g1.tile_started = reinterpret_cast<int*>(status + kStTileStarted);
    g1.row_scale = fp4 ? reinterpret_cast<const float*>(ws + L.xg) : nullptr;
    g1.w_scale = fp4 ? reinterpret_cast<const float*>(wb + plan->wb.wg) : nullptr;
    g1.h_fp32 = fp8 && L.hf != 0 ? reinterpret_cast<float*>(ws + L.hf) : nullptr;
    if (!mark(3)) return MOE_ERR_CUDA;
    e = fp8   ? launch_gemm1_mxfp8(tA1, rB1, g1, m_tiles * g1.n_tiles, s)
        : fp4 ? launch_gemm1_nvfp4(tA1, rB1, g1, m_tiles * g1.n_tiles, s)
              : launch_gemm1_bf16_pair(tA1, tX, rB1, g1, m_tiles * g1.n_tiles, s);
    if (e != cudaSuccess) return MOE_ERR_CUDA;
    if (fp4) {  // h rows -> NVFP4 with a scale per row (timed with the gate/up stage)
        e = launch_quantize_h_nvfp4(reinterpret_cast<const float*>(ws + L.hf), live_count_dev, max_live, k,
                                    (int)plan->fp, inv, ws + L.h, ws + L.hs, reinterpret_cast<float*>(ws + L.hg),
                                    status, s);
        if (e != cudaSuccess) return MOE_ERR_CUDA;
    }

    GemmParams g2 = g1;
    g2.out = ws + L.y;
    g2.out_ld = H;
    g2.out_cols = H;
    g2.n_tiles = plan->nt2;
    g2.k_blocks = plan->ks2;
    g2.a_rows = fp8 || fp4 ? H : plan->hr;
    g2.sfa = wb + plan->wb.w2s;
    g2.sfb = ws + L.hs;
    g2.out_scales = nullptr;
    g2.row_scale = fp4 ? reinterpret_cast<const float*>(ws + L.hg) : nullptr;
    g2.h_fp32 = nullptr;
    if (!mark(4)) return MOE_ERR_CUDA;
    e = fp8   ? launch_gemm2_mxfp8(tA2, rB2, g2, m_tiles * g2.n_tiles, s)
        : fp4 ? launch_gemm2_nvfp4(tA2, rB2, g2, m_tiles * g2.n_tiles, s)
              : launch_gemm2_bf16_pair(tA2, rB2, g2, m_tiles * g2.n_tiles, s);
    if (e != cudaSuccess) return MOE_ERR_CUDA;
    if (!mark(5)) return MOE_ERR_CUDA;

    // the probabilities were applied in the gate/up epilogue: the combine adds the rows
    e = launch_combine(reinterpret_cast<const float*>(ws + L.y), inv, probs_in_fc1 ? nullptr : r_probs,
                       live_count_dev, max_live, H, k, out, (plan->d.flags & MOE_FLAG_OUT_BF16) != 0, status, s);
    if (e != cudaSuccess) return MOE_ERR_CUDA;
    return mark(6) ? MOE_OK : MOE_ERR_CUDA;
}

}  // namespace

extern "C" {

moe_status moe_forward(const moe_plan* plan, const void* x, const float* logits, const int* ids, const float* probs,
                       const void* kernel_buf, const int* live_count_dev, void* out, void* workspace,
                       size_t ws_bytes, void* stream) {
    return forward_impl(plan, x, logits, ids, probs, kernel_buf, live_count_dev, out, workspace, ws_bytes, stream,
                        nullptr);
}

moe_status moe_forward_with_events(const moe_plan* plan, const void* x, const float* logits, const int* ids,
                                   const float* probs, const void* kernel_buf, const int* live_count_dev, void* out,
                                   void* workspace, size_t ws_bytes, void* stream, void* const* stage_events) {
    if (stage_events == nullptr) return MOE_ERR_INVALID_ARG;
    for (int i = 0; i <= MOE_NUM_STAGES; ++i)
        if (stage_events[i] == nullptr) return MOE_ERR_INVALID_ARG;
    return forward_impl(plan, x, logits, ids, probs, kernel_buf, live_count_dev, out, workspace, ws_bytes, stream,
                        stage_events);
}

// Expert-parallel send side: the forward's route (or canonicalisation) and
// permute stages into the workspace, then the pack kernel.
moe_status moe_ep_dispatch(const moe_plan* plan, int ep_size, const void* x, const float* logits, const int* ids,
                           const float* probs, const int* live_count_dev, void* send_x, int* send_ids,
                           float* send_probs, int* send_counts, int* route_rows, float* route_probs,
                           void* workspace, size_t ws_bytes, void* stream) {
    if (plan == nullptr || x == nullptr || live_count_dev == nullptr || send_x == nullptr || send_ids == nullptr ||
        send_probs == nullptr || send_counts == nullptr || route_rows == nullptr || route_probs == nullptr ||
        workspace == nullptr)
        return MOE_ERR_INVALID_ARG;
    const bool have_logits = logits != nullptr;
    const bool have_routes = ids != nullptr && probs != nullptr;
    if (have_logits == have_routes || ((ids == nullptr) != (probs == nullptr))) return MOE_ERR_INVALID_ARG;
    const int H = plan->d.hidden, E = plan->d.num_experts, k = plan->d.top_k;
    if (ep_size < 1 || ep_size > ep_max_size() || E % ep_size != 0) return MOE_ERR_UNSUPPORTED;
    if (ws_bytes < plan->ws.total) return MOE_ERR_WORKSPACE_TOO_SMALL;
    if (!aligned(x, 16) || !aligned(send_x, 16) || !aligned(workspace, 256)) return MOE_ERR_ALIGNMENT;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const int max_live = (int)plan->max_live;
    uint8_t* ws = static_cast<uint8_t*>(workspace);
    const WsLayout& L = plan->ws;
    unsigned* status = reinterpret_cast<unsigned*>(ws + L.status);
    int* r_ids = reinterpret_cast<int*>(ws + L.r_ids);
    float* r_probs = reinterpret_cast<float*>(ws + L.r_probs);
    const bool blockscaled = plan->d.precision != MOE_BF16;
    cudaError_t e = have_logits ? launch_route_topk(logits, live_count_dev, max_live, E, k, r_ids, r_probs, status, s)
                                : launch_canon_routes(ids, probs, live_count_dev, max_live, E, k, r_ids, r_probs,
                                                      status, s);
    if (e != cudaSuccess) return MOE_ERR_CUDA;
    int* inv = reinterpret_cast<int*>(ws + L.inv);
    int* offsets = reinterpret_cast<int*>(ws + L.offsets);
    int* padoff = reinterpret_cast<int*>(ws + L.padoff);
    e = launch_permute(plan, live_count_dev, r_ids, reinterpret_cast<int*>(ws + L.blkcnt), offsets, padoff,
                       reinterpret_cast<int4*>(ws + L.tiles), reinterpret_cast<int*>(ws + L.perm), inv,
                       blockscaled ? nullptr : reinterpret_cast<int*>(ws + L.ready), status, s);
    if (e != cudaSuccess) return MOE_ERR_CUDA;
    e = launch_ep_pack(x, live_count_dev, max_live, H, k, r_ids, r_probs, inv, offsets, padoff, E, ep_size,
                       (plan->d.flags & MOE_FLAG_PROBS_IN_FC1) != 0, send_x, send_ids, send_probs, send_counts,
                       route_rows, route_probs, status, s);
    return e == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

moe_status moe_ep_combine(const moe_plan* plan, const float* y_rows, const int* route_rows,
                          const float* route_probs, const int* live_count_dev, void* out, void* stream) {
    if (plan == nullptr || y_rows == nullptr || route_rows == nullptr || route_probs == nullptr ||
        live_count_dev == nullptr || out == nullptr)
        return MOE_ERR_INVALID_ARG;
    if (!aligned(y_rows, 16) || !aligned(out, 16)) return MOE_ERR_ALIGNMENT;
    const cudaError_t e = launch_combine(y_rows, route_rows, route_probs, live_count_dev, (int)plan->max_live,
                                         plan->d.hidden, plan->d.top_k, out,
                                         (plan->d.flags & MOE_FLAG_OUT_BF16) != 0, nullptr,
                                         static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

// ---------------------------------------------------------------- peer-memory EP exchange

size_t moe_ep_region_bytes(const moe_plan* plan, int ep_size) {
    if (plan == nullptr || ep_size < 1 || ep_size > kEpMaxRanks) return 0;
    return ep_region_layout(plan->d.hidden, (int)plan->max_live, plan->d.top_k, ep_size).total;
}

moe_status moe_ep_region_views_get(const moe_plan* plan, int ep_size, void* region, moe_ep_region_views* v) {
    if (plan == nullptr || region == nullptr || v == nullptr) return MOE_ERR_INVALID_ARG;
    if (ep_size < 1 || ep_size > kEpMaxRanks) return MOE_ERR_UNSUPPORTED;
    const EpRegionLayout l = ep_region_layout(plan->d.hidden, (int)plan->max_live, plan->d.top_k, ep_size);
    uint8_t* b = static_cast<uint8_t*>(region);
    std::memset(v, 0, sizeof(*v));
    v->status = reinterpret_cast<unsigned*>(b) + kEpStatus;
    v->recv_live = reinterpret_cast<int*>(b) + kEpRecvLive;
    v->recv_x = b + l.recv_x;
    v->recv_ids = reinterpret_cast<int*>(b + l.recv_ids);
    v->recv_probs = reinterpret_cast<float*>(b + l.recv_probs);
    v->recv_y = reinterpret_cast<float*>(b + l.recv_y);
    v->y_back = reinterpret_cast<float*>(b + l.y_back);
    v->recv_rows = l.max_send * ep_size;
    return MOE_OK;
}

moe_status moe_ep_peer_dispatch(const moe_plan* plan, int ep_size, int rank, const void* x, const float* logits,
                                const int* ids, const float* probs, const int* live_count_dev,
                                void* const* regions_dev, int* route_rows, float* route_probs, void* workspace,
                                size_t ws_bytes, void* stream) {
    if (plan == nullptr || x == nullptr || live_count_dev == nullptr || regions_dev == nullptr ||
        route_rows == nullptr || route_probs == nullptr || workspace == nullptr)
        return MOE_ERR_INVALID_ARG;
    const bool have_logits = logits != nullptr;
    const bool have_routes = ids != nullptr && probs != nullptr;
    if (have_logits == have_routes || ((ids == nullptr) != (probs == nullptr))) return MOE_ERR_INVALID_ARG;
    const int H = plan->d.hidden, E = plan->d.num_experts, k = plan->d.top_k;
    if (ep_size < 1 || ep_size > kEpMaxRanks || E % ep_size != 0) return MOE_ERR_UNSUPPORTED;
    if (rank < 0 || rank >= ep_size) return MOE_ERR_INVALID_ARG;
    if (ws_bytes < plan->ws.total) return MOE_ERR_WORKSPACE_TOO_SMALL;
    if (!aligned(x, 16) || !aligned(workspace, 256) || !aligned(regions_dev, 8)) return MOE_ERR_ALIGNMENT;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const int max_live = (int)plan->max_live;
    uint8_t* ws = static_cast<uint8_t*>(workspace);
    const WsLayout& L = plan->ws;
    unsigned* status = reinterpret_cast<unsigned*>(ws + L.status);
    int* r_ids = reinterpret_cast<int*>(ws + L.r_ids);
    float* r_probs = reinterpret_cast<float*>(ws + L.r_probs);
    const bool blockscaled = plan->d.precision != MOE_BF16;
    cudaError_t e = have_logits ? launch_route_topk(logits, live_count_dev, max_live, E, k, r_ids, r_probs, status, s)
                                : launch_canon_routes(ids, probs, live_count_dev, max_live, E, k, r_ids, r_probs,
                                                      status, s);
    if (e != cudaSuccess) return MOE_ERR_CUDA;
    int* inv = reinterpret_cast<int*>(ws + L.inv);
    int* offsets = reinterpret_cast<int*>(ws + L.offsets);
    int* padoff = reinterpret_cast<int*>(ws + L.padoff);
    e = launch_permute(plan, live_count_dev, r_ids, reinterpret_cast<int*>(ws + L.blkcnt), offsets, padoff,
                       reinterpret_cast<int4*>(ws + L.tiles), reinterpret_cast<int*>(ws + L.perm), inv,
                       blockscaled ? nullptr : reinterpret_cast<int*>(ws + L.ready), status, s);
    if (e != cudaSuccess) return MOE_ERR_CUDA;
    const EpRegionLayout lay = ep_region_layout(H, max_live, k, ep_size);
    e = launch_ep_peer_pack(x, live_count_dev, max_live, H, k, r_ids, r_probs, inv, offsets, padoff, E, ep_size, rank,
                            (plan->d.flags & MOE_FLAG_PROBS_IN_FC1) != 0, regions_dev, lay, route_rows, route_probs,
                            status, s);
    return e == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

moe_status moe_ep_peer_receive(const moe_plan* plan, int ep_size, void* region, unsigned long long wait_limit_ns,
                               void* stream) {
    if (plan == nullptr || region == nullptr) return MOE_ERR_INVALID_ARG;
    if (ep_size < 1 || ep_size > kEpMaxRanks || plan->d.num_experts % ep_size != 0) return MOE_ERR_UNSUPPORTED;
    if (wait_limit_ns == 0 || !aligned(region, 256)) return wait_limit_ns == 0 ? MOE_ERR_INVALID_ARG : MOE_ERR_ALIGNMENT;
    const EpRegionLayout lay = ep_region_layout(plan->d.hidden, (int)plan->max_live, plan->d.top_k, ep_size);
    const cudaError_t e = launch_ep_peer_receive(region, ep_size, plan->d.hidden, lay, wait_limit_ns,
                                                 static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

moe_status moe_ep_peer_return(const moe_plan* plan, int ep_size, int rank, void* const* regions_dev, void* stream) {
    if (plan == nullptr || regions_dev == nullptr) return MOE_ERR_INVALID_ARG;
    if (ep_size < 1 || ep_size > kEpMaxRanks || plan->d.num_experts % ep_size != 0) return MOE_ERR_UNSUPPORTED;
    if (rank < 0 || rank >= ep_size) return MOE_ERR_INVALID_ARG;
    const EpRegionLayout lay = ep_region_layout(plan->d.hidden, (int)plan->max_live, plan->d.top_k, ep_size);
    const cudaError_t e = launch_ep_peer_return(regions_dev, nullptr, rank, ep_size, plan->d.hidden, lay,
                                                static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

moe_status moe_ep_peer_combine(const moe_plan* plan, int ep_size, void* region, const int* route_rows,
                               const float* route_probs, const int* live_count_dev, void* out,
                               unsigned long long wait_limit_ns, void* stream) {
    if (plan == nullptr || region == nullptr || route_rows == nullptr || route_probs == nullptr ||
        live_count_dev == nullptr || out == nullptr || wait_limit_ns == 0)
        return MOE_ERR_INVALID_ARG;
    if (ep_size < 1 || ep_size > kEpMaxRanks || plan->d.num_experts % ep_size != 0) return MOE_ERR_UNSUPPORTED;
    if (!aligned(out, 16) || !aligned(region, 256)) return MOE_ERR_ALIGNMENT;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const EpRegionLayout lay = ep_region_layout(plan->d.hidden, (int)plan->max_live, plan->d.top_k, ep_size);
    cudaError_t e = launch_ep_peer_wait_returns(region, ep_size, wait_limit_ns, s);
    if (e != cudaSuccess) return MOE_ERR_CUDA;
    uint8_t* b = static_cast<uint8_t*>(region);
    e = launch_combine(reinterpret_cast<const float*>(b + lay.y_back), route_rows, route_probs, live_count_dev,
                       (int)plan->max_live, plan->d.hidden, plan->d.top_k, out,
                       (plan->d.flags & MOE_FLAG_OUT_BF16) != 0, reinterpret_cast<const unsigned*>(b) + kEpStatus, s);
    return e == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

moe_status moe_ep_ipc_handle(void* dev_ptr, void* handle_out) {
    if (dev_ptr == nullptr || handle_out == nullptr) return MOE_ERR_INVALID_ARG;
    static_assert(sizeof(cudaIpcMemHandle_t) == MOE_EP_IPC_HANDLE_BYTES, "IPC handle size");
    cudaIpcMemHandle_t h;
    if (cudaIpcGetMemHandle(&h, dev_ptr) != cudaSuccess) return MOE_ERR_CUDA;
    std::memcpy(handle_out, &h, sizeof(h));
    return MOE_OK;
}

moe_status moe_ep_ipc_open(const void* handle, void** dev_ptr_out) {
    if (handle == nullptr || dev_ptr_out == nullptr) return MOE_ERR_INVALID_ARG;
    cudaIpcMemHandle_t h;
    std::memcpy(&h, handle, sizeof(h));
    return cudaIpcOpenMemHandle(dev_ptr_out, h, cudaIpcMemLazyEnablePeerAccess) == cudaSuccess ? MOE_OK
                                                                                                : MOE_ERR_CUDA;
}

moe_status moe_ep_ipc_close(void* dev_ptr) {
    if (dev_ptr == nullptr) return MOE_ERR_INVALID_ARG;
    return cudaIpcCloseMemHandle(dev_ptr) == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

moe_status moe_get_workspace_views(const moe_plan* plan, const void* workspace, moe_workspace_views* v) {
    if (plan == nullptr || workspace == nullptr || v == nullptr) return MOE_ERR_INVALID_ARG;
    const uint8_t* ws = static_cast<const uint8_t*>(workspace);
    const WsLayout& L = plan->ws;
    std::memset(v, 0, sizeof(*v));
    v->route_ids = reinterpret_cast<const int*>(ws + L.r_ids);
    v->route_probs = reinterpret_cast<const float*>(ws + L.r_probs);
    v->offsets = reinterpret_cast<const int*>(ws + L.offsets);
    v->perm = reinterpret_cast<const int*>(ws + L.perm);
    v->inv = reinterpret_cast<const int*>(ws + L.inv);
    v->pad_offsets = reinterpret_cast<const int*>(ws + L.padoff);
    v->h = ws + L.h;
    const bool scaled = plan->d.precision != MOE_BF16;
    const bool fp4 = plan->d.precision == MOE_NVFP4;
    v->h_scales = scaled ? ws + L.hs : nullptr;
    v->xq = ws + L.xq;
    v->xq_scales = scaled ? ws + L.xs : nullptr;
    v->xq_row_scales = fp4 ? reinterpret_cast<const float*>(ws + L.xg) : nullptr;
    v->h_row_scales = fp4 ? reinterpret_cast<const float*>(ws + L.hg) : nullptr;
    v->h_fp32 = L.hf != 0 ? reinterpret_cast<const float*>(ws + L.hf) : nullptr;
    v->rows_padded = plan->rows_pad;
    v->status = reinterpret_cast<const unsigned*>(ws + L.status);
    return MOE_OK;
}

moe_status moe_get_device_status(const void* workspace, unsigned* flags_host, void* stream) {
    if (workspace == nullptr || flags_host == nullptr) return MOE_ERR_INVALID_ARG;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (cudaMemcpyAsync(flags_host, workspace, sizeof(unsigned), cudaMemcpyDeviceToHost, s) != cudaSuccess)
        return MOE_ERR_CUDA;
    return cudaStreamSynchronize(s) == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

moe_status moe_clear_device_status(void* workspace, void* stream) {
    if (workspace == nullptr) return MOE_ERR_INVALID_ARG;
    return cudaMemsetAsync(workspace, 0, sizeof(unsigned), static_cast<cudaStream_t>(stream)) == cudaSuccess
               ? MOE_OK
               : MOE_ERR_CUDA;
}

}  // extern "C"
