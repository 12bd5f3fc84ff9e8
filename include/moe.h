/*
 * moe.h -- C ABI of the B200 (sm_100a) routed-MoE SwiGLU expert forward.
 *
 * The path: router softmax/top-k -> permute of every (token, expert) route
 * into expert-contiguous rows -> gate/up grouped GEMM with SwiGLU fused into
 * its epilogue -> down-projection grouped GEMM -> probability-weighted
 * combine accumulated in fp32 in ascending expert-id order.  All work is
 * bounded by a live-row count that lives in device memory, so one CUDA-graph
 * capture serves every step.
 *
 * Sources (page title, section):
 *   [P1] Megatron-LM PR #7830 ("flashinfer_mega" backend): "1. Mega backend
 *        for generation" -- kernel weight layout rebuilt into a caller-owned
 *        buffer on refit (refresh_mega_weights), canonical expert-id order
 *        before the combine, MXFP8 quantisation per block of 32.
 *   [P2] Megatron-LM PR #7798 (moe_training_matches_inference): "Background"
 *        (activation fused into FC1's epilogue, probabilities applied after
 *        FC2) and "What is changed" (a token's routes summed as fp32 fused
 *        multiply-adds of probability and row, from zero, in a fixed order);
 *        "Per-token NVFP4" (TE's NVFP4BlockScaling recipe with row-scaled
 *        activations, 1-D blocks, no Hadamard transform, no stochastic
 *        rounding).  "What is changed" also runs every row an all-to-all
 *        dispatcher delivers as a top-1 token with probability 1.0;
 *        "Limitations": generation's combine is not EP-invariant.
 *   [P3] Megatron-LM PR #8367 ("bound the FlashInfer MoE expert kernels by
 *        token count"): "Problem" -- the live token count is known only on
 *        the device; results are returned in fp32.
 *   [P4] core.transformer.moe.training_matches_inference API doc: `_route`
 *        ([tokens, topk] probs and ids) and `expert_value_pass` (rows sorted
 *        by local expert).
 *   [P5] cudnn-frontend PR #448 (MoeEp API): MXFP8 uses 32-element blocks;
 *        the parts of an EP layer: a variable-size all-to-all dispatch of
 *        routes, local experts, a top-k combine.
 *
 * Conventions for every entry point:
 *   - Every pointer named *_dev or described as "device" is a device pointer
 *     the caller allocated; the library never allocates or frees device
 *     memory and never synchronises the stream, except where stated
 *     (moe_get_device_status).
 *   - `stream` is a cudaStream_t (CUstream) passed as void*; NULL is the
 *     legacy default stream.
 *   - bf16 tensors are passed as void* to 16-bit bfloat16 elements.
 *   - Row-major layouts, dense, no padding between rows unless an ld_* stride
 *     is given.
 *   - Host-detectable errors (null pointers, bad sizes, misalignment, a too
 *     small buffer) return a status before anything is launched.  Conditions
 *     found on the device set bits in a status word inside the workspace
 *     (MOE_DEV_*) and never trap, fault or hang.
 *   - moe_forward, moe_route_topk and mxfp8_quantize_block32 enqueue work
 *     only, so they may be captured into a CUDA graph.
 *   - A plan is immutable after creation and may be shared by threads; use
 *     one workspace per concurrently running stream.
 */
#ifndef ROUTED_MOE_SWIGLU_B200_MOE_H
#define ROUTED_MOE_SWIGLU_B200_MOE_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    MOE_OK = 0,
    MOE_ERR_INVALID_ARG = 1,          /* null pointer, negative size, bad enum   */
    MOE_ERR_UNSUPPORTED = 2,          /* shape outside the supported envelope    */
    MOE_ERR_ALIGNMENT = 3,            /* pointer or stride not 16-byte aligned   */
    MOE_ERR_WORKSPACE_TOO_SMALL = 4,  /* workspace / weight buffer too small     */
    MOE_ERR_CUDA = 5,                 /* a CUDA runtime call failed              */
    MOE_ERR_NOT_PREPARED = 6          /* reserved: weight buffer not prepared    */
} moe_status;

typedef enum { MOE_BF16 = 0, MOE_MXFP8 = 1, MOE_NVFP4 = 2 } moe_precision;

/* Device status bits (sticky until moe_clear_device_status). */
#define MOE_DEV_LIVE_CLAMPED 0x1u  /* live count < 0 or > max live rows: clamped    */
#define MOE_DEV_BAD_ROUTE 0x2u     /* caller ids out of [0,E) or repeated in a token:
                                      that token's output row is all zeros          */
#define MOE_DEV_TIMEOUT 0x4u       /* a bounded on-device wait gave up; outputs of
                                      that call are not valid, and while the bit is
                                      set, forwards on this workspace write no
                                      output rows (clear it to run again)           */

typedef struct {
    int hidden;              /* H: model width (K of the gate/up GEMM)            */
    int ffn;                 /* F: expert intermediate width (K of the down GEMM) */
    int num_experts;         /* E                                                 */
    int top_k;               /* k: routes per token                               */
    long long capacity;      /* rows of the caller's preallocated token buffers   */
    long long max_live_rows; /* largest live count a call will pass (<= capacity);
                                0 means capacity.  The workspace is sized for it;
                                larger live counts are clamped and flagged.       */
    moe_precision precision; /* MOE_BF16, MOE_MXFP8 or MOE_NVFP4                  */
    unsigned flags;          /* MOE_FLAG_* variants; 0 for the plain forward      */
    float gate_up_clamp;     /* > 0: gate and up pre-activations clamped to
                                [-gate_up_clamp, gate_up_clamp] before SwiGLU
                                (cudnn-frontend PR #448, MoeEp `gate_up_clamp`);
                                0: no clamp                                       */
} moe_desc;

/* Variants of the forward the pages' kernels offer (cudnn-frontend PR #448,
 * the MoeEp constructor; Megatron-LM PR #8367 for the output type):
 *   MOE_FLAG_PROBS_IN_FC1  `apply_topk_in_fc1`: each route's probability
 *       multiplies its SwiGLU row before that row is rounded for the down
 *       GEMM, h = round(p * silu(g) * u); the combine then adds the routes'
 *       rows as fp32 additions from 0.0f in ascending expert id.
 *   MOE_FLAG_OUT_BF16      bf16 finalize: out is bf16 [capacity, H], the
 *       fp32 sum rounded to nearest even (the plain output is fp32). */
#define MOE_FLAG_PROBS_IN_FC1 0x1u
#define MOE_FLAG_OUT_BF16 0x2u
/*   MOE_FLAG_SQUARED_RELU  squared-ReLU experts (the Nano-v3 shapes of
 *       Megatron-LM PR #8367's measurements): one FC1 projection,
 *       h = relu(W_gate[e] . x)^2; W_up is not used.  The clamp and the
 *       probability in FC1 act on the one pre-activation and on the row. */
#define MOE_FLAG_SQUARED_RELU 0x4u
/*   MOE_FLAG_KEEP_H_FP32   MXFP8 only, for checking the fused quantiser: the
 *       gate/up epilogue also stores the fp32 SwiGLU values it quantises,
 *       [rows_padded, ceil(F/128)*128], into the workspace (the h_fp32
 *       view).  The workspace grows by that buffer and every h element costs
 *       one more 4-byte store; results are unchanged.  NVFP4 plans keep
 *       these rows always (its quantisation pass reads them); bf16 plans
 *       reject the flag. */
#define MOE_FLAG_KEEP_H_FP32 0x8u

typedef struct moe_plan moe_plan; /* opaque, host memory only */

/* Validate `desc` and build a host-side plan (no device work, no device
 * allocation).  Rejected (MOE_ERR_UNSUPPORTED): H or F not a multiple of 8
 * (bf16) or of 32 (MXFP8, NVFP4); k < 1, k > 16 or k > E; E < 1 or E > 1024;
 * capacity < 1 or > 2^24 rows; max_live_rows < 0 or > capacity;
 * H > 16384 or F > 16384.  Rejected (MOE_ERR_INVALID_ARG): unknown flag
 * bits, a negative or non-finite gate_up_clamp. */
moe_status moe_plan_create(const moe_desc* desc, moe_plan** plan_out);
void moe_plan_destroy(moe_plan* plan);
/* Copy of the descriptor the plan was made from (max_live_rows resolved). */
moe_status moe_plan_get_desc(const moe_plan* plan, moe_desc* desc_out);

/* Bytes of the caller-owned kernel-layout weight buffer and of the
 * per-stream workspace (routes, permutation, tile list, intermediate rows,
 * status word).  Both buffers must be 256-byte aligned. */
size_t moe_weight_buffer_bytes(const moe_plan* plan);
size_t moe_workspace_bytes(const moe_plan* plan);

/* Rebuild the kernel-layout weight buffer in place from the experts' bf16
 * weights ([P1] "refresh_mega_weights": a refit rewrites the same buffer; no
 * allocation, no teardown).  Inputs (device, bf16, row-major):
 *   w_gate [E, F, H], w_up [E, F, H]  (gate and up projections; for
 *                                      MOE_FLAG_SQUARED_RELU plans w_gate is
 *                                      the one FC1 projection and w_up is not
 *                                      read and may be NULL)
 *   w_down [E, H, F]                  (down projection)
 * In MXFP8 the weights are quantised here (blocks of 32 along each GEMM's K:
 * H for gate/up, F for down); in NVFP4 likewise (blocks of 16) with one
 * second-level scale per expert matrix (W1 = gate and up together, W2), as
 * nvfp4_quantize_block16 describes.  Enqueued on `stream`; forwards enqueued later
 * on the same stream see the new weights, forwards enqueued earlier finish
 * with the old ones.  Returns MOE_ERR_WORKSPACE_TOO_SMALL if buf_bytes <
 * moe_weight_buffer_bytes. */
moe_status moe_prepare_weights(const moe_plan* plan, const void* w_gate, const void* w_up,
                               const void* w_down, void* kernel_buf, size_t buf_bytes,
                               void* stream);

/* MXFP8 quantisation ([P1], [P5]; OCP MX v1.0): each row of `in` (bf16,
 * [rows, cols], row stride ld_in elements) is cut into blocks of 32; each
 * block gets the E8M0 scale byte floor(log2(amax)) - 8 + 127 (clamped to
 * [0, 254]; 0 for an all-zero block) and E4M3 codes of value/scale rounded
 * to nearest-even, saturating to +-448, sign kept.
 *   q      [rows, cols] uint8 codes (row stride cols)
 *   scales [rows, cols/32] uint8 E8M0 bytes (row stride cols/32)
 * live_rows_dev: nullable device int32; when given, only rows
 * [0, min(max(*live_rows_dev,0), rows)) are written.
 * cols must be a positive multiple of 32, ld_in >= cols and a multiple of 8,
 * `in` 16-byte aligned. */
moe_status mxfp8_quantize_block32(const void* in, long long rows, int cols, long long ld_in,
                                  uint8_t* q, uint8_t* scales, const int* live_rows_dev,
                                  void* stream);

/* NVFP4 quantisation of bf16 rows as the per-token recipe does it ([P2]
 * "Per-token NVFP4": TE's NVFP4BlockScaling with row-scaled activations,
 * 1-D blocks, no Hadamard transform, no stochastic rounding).  Per row:
 *   g = amax(row) / 2688 in fp32 (1 for an all-zero row), row_scales[r];
 *   per 16 elements: s = E4M3((amax_16 / g) / 6) (fp32 divisions, round to
 *   nearest even, saturating at 448), scales[r, c/16];
 *   each element: E2M1(v / (value(s) * g)) (fp32, round to nearest even,
 *   saturating at 6; signed zero when the divisor is 0), packed two per
 *   byte with element 2i in the low nibble, q[r, c/2].
 * The value of an element is E2M1 * value(s) * g.  in bf16 [rows, ld_in];
 * q uint8 [rows, cols/2], scales uint8 [rows, cols/16], row_scales fp32
 * [rows], all row-major, device pointers.  live_rows_dev as for
 * mxfp8_quantize_block32.  cols a positive multiple of 32, ld_in >= cols and
 * a multiple of 8, `in` 16-byte aligned, q and row_scales 4-byte aligned. */
moe_status nvfp4_quantize_block16(const void* in, long long rows, int cols, long long ld_in,
                                  uint8_t* q, uint8_t* scales, float* row_scales,
                                  const int* live_rows_dev, void* stream);

/* Router ([P4] `_route`): for each live row t of logits (fp32 [capacity, E]),
 * softmax over the E experts, the k largest (ties: lower expert id), the k
 * probabilities renormalised to sum to 1; written in ascending expert id
 * ([P1] canonical order).  ids int32 [capacity, k], probs fp32 [capacity, k];
 * rows >= the live count are not read or written.  live_count_dev: device
 * int32, clamped to [0, max_live_rows] (no status word here: no workspace). */
moe_status moe_route_topk(const moe_plan* plan, const float* logits, const int* live_count_dev,
                          int* ids, float* probs, void* stream);

/* The routed SwiGLU expert forward.
 *   x        bf16 [capacity, H]: token rows; only rows < live count are read.
 *   logits   fp32 [capacity, E] or NULL: routed here as moe_route_topk does;
 *   ids      int32 [capacity, k] and probs fp32 [capacity, k], or both NULL:
 *            an outside router's routes in any order; they are put in
 *            ascending id order with their probabilities, not renormalised.
 *            Exactly one of `logits` or (`ids`, `probs`) must be given.
 *   kernel_buf  the buffer moe_prepare_weights filled.
 *   live_count_dev  device int32 live row count (clamped, flagged).
 *   out      fp32 [capacity, H]: row t < live count gets
 *            sum over its routes j in ascending expert id of
 *            p_j * y_j as fp32 FMAs from 0.0f, where
 *            y_j = W_down[e_j] . (silu(W_gate[e_j] . x_t) * (W_up[e_j] . x_t))
 *            with the SwiGLU row rounded to bf16 (or re-quantised to MXFP8,
 *            or to NVFP4 with the row's own scale) and y_j kept in fp32; in
 *            MXFP8 and NVFP4, x_t and the weights are quantised as their
 *            quantisation entry points describe.  Rows >= live count are not
 *            written.
 *            The plan's flags change this as MOE_FLAG_* states (bf16 out,
 *            probabilities applied in FC1), and gate_up_clamp clamps the
 *            two pre-activations before silu and the product.
 *   workspace  moe_workspace_bytes(plan) bytes, 256-byte aligned.
 * Each token's output is bitwise independent of the live count and of the
 * other tokens in the launch. */
moe_status moe_forward(const moe_plan* plan, const void* x, const float* logits, const int* ids,
                       const float* probs, const void* kernel_buf, const int* live_count_dev,
                       void* out, void* workspace, size_t ws_bytes, void* stream);

/* moe_forward for callers that cannot allocate device memory (no
 * counterpart in the pages: an addition of this library).  Some callers get
 * only their input and output pointers and have no allocator to call -- a
 * plug-in living inside another engine's memory budget, or code that must not
 * call cudaMalloc because it would synchronise the device or is not allowed
 * under the caller's stream capture.  This entry point takes no workspace:
 * its scratch is one fixed array of MOE_NOALLOC_SCRATCH_BYTES (64 MiB) in
 * the library's device memory, which every GPU that loads this part of the
 * library holds until the process exits.  It calls no cudaMalloc, cudaFree
 * or other allocating routine.
 *   - Arguments as moe_forward, minus the workspace.
 *   - Plans whose moe_workspace_bytes exceeds MOE_NOALLOC_SCRATCH_BYTES are
 *     rejected with MOE_ERR_WORKSPACE_TOO_SMALL before anything runs (use a
 *     smaller max_live_rows, or moe_forward with your own workspace).
 *   - Each call outside stream capture looks up the array's device address
 *     on the current device (so a cudaDeviceReset between calls is safe);
 *     a call under capture uses the address that the last call outside
 *     capture found.  Make one call on each device before any stream capture,
 *     and again after a device reset.
 *   - Every call, on every stream, shares the one array, which keeps the
 *     last call's contents: calls that overlap on the GPU race with each
 *     other.  Serialise them (one stream, or events).
 *   - The device status word lives in the shared array and is cleared at the
 *     start of each call; it cannot be read back through this entry point.
 *   - Same results as moe_forward on the same inputs. */
#define MOE_NOALLOC_SCRATCH_BYTES (64ull << 20)
moe_status moe_forward_noalloc(const moe_plan* plan, const void* x, const float* logits, const int* ids,
                               const float* probs, const void* kernel_buf, const int* live_count_dev,
                               void* out, void* stream);

/* Stages of moe_forward, in launch order: route (or canonicalise the
 * caller's routes), permute (histogram, scan, scatter), gather of x rows
 * (and their MXFP8 quantisation; bf16 gathers only the rows of route tiles
 * of more than 32 routes, the gate/up GEMM reads the others from x itself),
 * gate/up GEMM with SwiGLU, down GEMM, combine. */
#define MOE_NUM_STAGES 6

/* moe_forward that also records stage_events[i] (cudaEvent_t passed as void*,
 * MOE_NUM_STAGES + 1 of them, created by the caller with timing enabled) on
 * `stream` before stage i, and stage_events[MOE_NUM_STAGES] after the last
 * stage; for measuring each stage's device time.  Same results as
 * moe_forward. */
moe_status moe_forward_with_events(const moe_plan* plan, const void* x, const float* logits, const int* ids,
                                   const float* probs, const void* kernel_buf, const int* live_count_dev,
                                   void* out, void* workspace, size_t ws_bytes, void* stream,
                                   void* const* stage_events);

/* Expert parallelism ([P2] "What is changed" and "Limitations"; [P5]: a
 * variable-size all-to-all of route rows, local experts, a top-k combine).
 * The E experts are split into ep_size equal contiguous ranges; EP rank g
 * owns experts [g*E/ep_size, (g+1)*E/ep_size).  One step on each rank:
 *   1. moe_ep_dispatch with the rank's own tokens and its full-E plan: route,
 *      order the routes by expert, pack one send row per route;
 *   2. exchange send_counts, then the first sum(send_counts) send rows
 *      (x, ids, probs) with an all-to-all: the rows for rank g are the g-th
 *      run of send_counts[g] rows (the caller's collective, e.g. NCCL);
 *   3. on the receiving rank, moe_forward of a plan with the E/ep_size local
 *      experts, top_k 1, fp32 output and the same precision, flags (but
 *      MOE_FLAG_OUT_BF16) and clamp, over the received rows as tokens with
 *      ids = received ids and probs = received probs: its output rows are
 *      the routes' expert outputs y (each row a top-1 token whose weight
 *      multiplies y exactly: 1.0, or its probability under
 *      MOE_FLAG_PROBS_IN_FC1, which the FC1 epilogue then applies);
 *   4. return those rows with the reverse all-to-all, so that send row r
 *      gets back its route's y row at row r;
 *   5. moe_ep_combine with the full-E plan.
 * The output of step 5 is bitwise the one-GPU moe_forward's for the same
 * tokens, whatever ep_size: each y row is one route's arithmetic whatever
 * launch computes it, and the combine is the same ascending-id fp32 FMA chain
 * (the pages' generation combine adds per-rank partials and is not
 * EP-invariant). */

/* Send side (step 1).  plan: the source rank's plan (all E experts).
 *   ep_size  1 .. 128, dividing E; MOE_ERR_UNSUPPORTED otherwise.
 *   x, logits / ids + probs, live_count_dev, workspace: as moe_forward.
 *   send_x       bf16 [max_live_rows * k, H], 16-byte aligned: row r is the
 *                x row of the r-th live route in expert order (stable by
 *                token within an expert); rows >= the route count are not
 *                written.
 *   send_ids     int32 [max_live_rows * k]: row r's expert id local to its
 *                owning rank (e mod E/ep_size).
 *   send_probs   fp32 [max_live_rows * k]: row r's weight in the receiving
 *                forward: 1.0, or the route's probability under
 *                MOE_FLAG_PROBS_IN_FC1.
 *   send_counts  int32 [ep_size]: rows for each destination rank, in rank
 *                order (they sum to the live route count).
 *   route_rows   int32 [max_live_rows, k]: the send row of route (t, j) of
 *                live token t in canonical (ascending id) order; -1 for the
 *                routes of a dropped token (a caller id out of range or
 *                repeated, flagged MOE_DEV_BAD_ROUTE).
 *   route_probs  fp32 [max_live_rows, k]: the route's combine weight (its
 *                probability, or 1.0 under MOE_FLAG_PROBS_IN_FC1).
 * All outputs are device memory the caller owns; rows of tokens >= the live
 * count are not written.  The workspace holds the routes and the permutation
 * as in moe_forward: one workspace serves one stream, and a moe_forward on the
 * same workspace before step 5 would not disturb this step (step 5 reads only
 * route_rows, route_probs and the returned rows). */
moe_status moe_ep_dispatch(const moe_plan* plan, int ep_size, const void* x, const float* logits, const int* ids,
                           const float* probs, const int* live_count_dev, void* send_x, int* send_ids,
                           float* send_probs, int* send_counts, int* route_rows, float* route_probs,
                           void* workspace, size_t ws_bytes, void* stream);

/* Combine (step 5).  plan: the source rank's plan.  y_rows fp32 [rows, H],
 * 16-byte aligned, row r = the returned y of send row r.  out (fp32, or bf16
 * under MOE_FLAG_OUT_BF16) [capacity, H]: row t < live count gets the sum
 * over j in ascending expert id of route_probs[t,j] * y_rows[route_rows[t,j]]
 * as fp32 FMAs from 0.0f (routes with row -1 skipped), as moe_forward's
 * combine; rows >= the live count are not written. */
moe_status moe_ep_combine(const moe_plan* plan, const float* y_rows, const int* route_rows,
                          const float* route_probs, const int* live_count_dev, void* out, void* stream);

/* Expert-parallel exchange through peer memory (no counterpart to call in
 * the pages, which put the EP transport inside their expert kernels:
 * Megatron-LM PR #7830; the NCCL all-to-all of steps 2 and 4 above reads the
 * split sizes on the host, Megatron-LM PR #7798, "Performance").  The same
 * step with the exchange done by the library's kernels over NVLink peer
 * memory, so that no host read of sizes is needed and one CUDA graph can
 * capture the whole step.  Every rank owns one region of
 * moe_ep_region_bytes(plan, ep_size) bytes (device memory, 256-byte aligned,
 * zero-filled once before the first step) that every other rank maps (e.g.
 * through moe_ep_ipc_handle / moe_ep_ipc_open); regions_dev is a device array
 * of ep_size pointers, entry g = rank g's region as this rank addresses it
 * (entry `rank` its own).  All ranks use plans of the same shape.  One step:
 *   1. moe_ep_peer_dispatch: route, permute, and store every route's x row,
 *      local expert id and FC1 weight into its owner's region (slot of this
 *      source); then raise this source's flag in every owner's region;
 *   2. moe_ep_peer_receive: wait until every source's flag is raised, then
 *      compact the received rows into the region's recv_x / recv_ids /
 *      recv_probs and set *recv_live (views below);
 *   3. moe_forward of the rank's expert plan (as in step 3 above) with
 *      x = recv_x, ids = recv_ids, probs = recv_probs, live = recv_live,
 *      out = recv_y;
 *   4. moe_ep_peer_return: store each received row's y into its source's
 *      region at the route's send row; then raise this owner's return flag
 *      in every source's region;
 *   5. moe_ep_peer_combine: wait until every owner's return flag is raised,
 *      then combine as moe_ep_combine.
 * Every step of every rank runs in stream order; every wait is bounded by
 * wait_limit_ns (> 0) and on expiry sets MOE_DEV_TIMEOUT in the region's
 * status word, after which the rank's later kernels of the step do no work
 * and its return flags stay down, so its sources time out too.  Flags carry
 * the step number (kept in the region), so no flag needs clearing between
 * steps.  The output is bitwise the one-GPU moe_forward's.  Not run across
 * several GPUs in this library's tests (one GPU per test machine): the tests
 * run every rank's steps in turn on one GPU, all regions in its memory. */
#define MOE_EP_IPC_HANDLE_BYTES 64
size_t moe_ep_region_bytes(const moe_plan* plan, int ep_size);
typedef struct {
    unsigned* status;  /* MOE_DEV_* bits of this rank's exchange (device word) */
    int* recv_live;    /* device int: rows received this step (step 2)         */
    void* recv_x;      /* bf16 [recv_rows, H]                                   */
    int* recv_ids;     /* int32 [recv_rows]: expert id local to this rank       */
    float* recv_probs; /* fp32 [recv_rows]: FC1 weight of the row               */
    float* recv_y;     /* fp32 [recv_rows, H]: the expert forward's output       */
    float* y_back;     /* fp32 [max_live_rows * k, H]: this rank's routes' y     */
    long long recv_rows; /* ep_size * max_live_rows * k: the expert plan's capacity */
} moe_ep_region_views;
moe_status moe_ep_region_views_get(const moe_plan* plan, int ep_size, void* region, moe_ep_region_views* views);
/* Step 1.  plan, ep_size, x, logits / ids + probs, live_count_dev,
 * route_rows, route_probs, workspace: as moe_ep_dispatch; rank: this rank. */
moe_status moe_ep_peer_dispatch(const moe_plan* plan, int ep_size, int rank, const void* x, const float* logits,
                                const int* ids, const float* probs, const int* live_count_dev,
                                void* const* regions_dev, int* route_rows, float* route_probs, void* workspace,
                                size_t ws_bytes, void* stream);
/* Step 2.  region: this rank's region. */
moe_status moe_ep_peer_receive(const moe_plan* plan, int ep_size, void* region, unsigned long long wait_limit_ns,
                               void* stream);
/* Step 4. */
moe_status moe_ep_peer_return(const moe_plan* plan, int ep_size, int rank, void* const* regions_dev, void* stream);
/* Step 5.  out, route_rows, route_probs, live_count_dev: as moe_ep_combine. */
moe_status moe_ep_peer_combine(const moe_plan* plan, int ep_size, void* region, const int* route_rows,
                               const float* route_probs, const int* live_count_dev, void* out,
                               unsigned long long wait_limit_ns, void* stream);
/* CUDA IPC of a region between the ranks' processes (host calls, thin
 * wrappers of the runtime's IPC handles; handle: MOE_EP_IPC_HANDLE_BYTES). */
moe_status moe_ep_ipc_handle(void* dev_ptr, void* handle_out);
moe_status moe_ep_ipc_open(const void* handle, void** dev_ptr_out);
moe_status moe_ep_ipc_close(void* dev_ptr);

/* Views into a workspace after a forward (device pointers into it), for
 * tests and diagnostics:
 *   route_ids/route_probs [max_live, k]: canonical routes of the last forward
 *   offsets int32 [E+1]: first row of each expert in the permuted order
 *   perm    int32 [routes]: permuted row r holds route t*k + j
 *   inv     int32 [max_live, k]: padded intermediate row of route (t, j)
 *   pad_offsets int32 [E+1]: first padded intermediate row of each expert,
 *           a multiple of 32 (bf16) or 128 (MXFP8, NVFP4)
 *   h       intermediate rows [rows_padded, ceil(F/128)*128], bf16 or
 *           E4M3 codes, the columns past F zero
 *   xq      permuted x rows [rows_padded, ceil(H/128)*128], bf16 or E4M3
 *           codes, the columns past H zero; bf16 writes only the rows of
 *           route tiles of more than 32 routes (the gate/up GEMM reads the
 *           x rows of smaller tiles in place)
 *   h_scales, xq_scales  MXFP8 and NVFP4 (else NULL).  MXFP8: E8M0 bytes
 *           in blocks of 512 bytes, one per (128-row tile, K stage of 128
 *           elements), block index tile * ceil(K/128) + stage; inside a block
 *           the byte of (row r of the tile, 32-element group g of the stage)
 *           is at (r % 32) * 16 + (r / 32) * 4 + g.  K = F for h, H for x.
 *           NVFP4: E4M3 bytes, four 512-byte blocks per (128-row tile, K
 *           block of 256 elements), block index (tile * ceil(K/256) + K
 *           block) * 4 + (64-element step within it); inside a block the
 *           byte of (row r, 16-element block b of the step) is at
 *           (r % 32) * 16 + (r / 32) * 4 + b.  NVFP4 h and xq are codes two
 *           per byte ([rows_padded, ceil(K/256)*128] bytes).
 *   xq_row_scales, h_row_scales  NVFP4 only: fp32 second-level scale per
 *           padded row;  h_fp32  the gate/up GEMM's fp32 h rows before
 *           quantisation: NVFP4 [rows_padded, ceil(F/256)*256]; MXFP8 plans
 *           made with MOE_FLAG_KEEP_H_FP32 [rows_padded, ceil(F/128)*128];
 *           else NULL. */
typedef struct {
    const int* route_ids;
    const float* route_probs;
    const int* offsets;
    const int* perm;
    const int* inv;
    const int* pad_offsets;
    const void* h;
    const uint8_t* h_scales;
    const void* xq;
    const uint8_t* xq_scales;
    long long rows_padded; /* rows of the padded intermediate buffers */
    const unsigned* status; /* device status word */
    const float* xq_row_scales;
    const float* h_row_scales;
    const float* h_fp32;
} moe_workspace_views;
moe_status moe_get_workspace_views(const moe_plan* plan, const void* workspace,
                                   moe_workspace_views* views);

/* Copy the workspace's device status word to *flags_host.  Synchronises
 * `stream` (the only call that does). */
moe_status moe_get_device_status(const void* workspace, unsigned* flags_host, void* stream);
/* Zero the status word (enqueued on `stream`).  A newly allocated workspace
 * holds an undefined status word: clear it once before the first read. */
moe_status moe_clear_device_status(void* workspace, void* stream);

/* Diagnostic of the device-side failure detection (no counterpart in the
 * pages).  Every pipeline wait inside the forward's kernels is bounded: a
 * wait that runs out sets MOE_DEV_TIMEOUT in the status word, tells the
 * other roles of its CTA to stop, and the kernel exits without trapping.
 * This call runs that mechanism on the device without a forward: one CTA
 * waits on mbarriers that nothing arrives on; the first wait gives up after
 * `limit_ns` (1 ns .. 10 s) and sets MOE_DEV_TIMEOUT in *status_dev (a
 * device word the caller owns; bits are OR-ed in), the second wait ends
 * through the CTA's abort flag.  elapsed_ns_dev (nullable) receives the two
 * waits' durations in ns, [0] the one that ran out, [1] the one that was
 * told to stop.  Enqueued on `stream`; returns MOE_ERR_INVALID_ARG for a
 * null status pointer or a limit outside the range. */
moe_status moe_check_bounded_wait(unsigned long long limit_ns, unsigned* status_dev,
                                  unsigned long long* elapsed_ns_dev, void* stream);

/* Static string for a status code. */
const char* moe_status_string(moe_status s);

/* Library version, e.g. "0.1.0". */
const char* moe_version(void);

#ifdef __cplusplus
}
#endif
#endif /* ROUTED_MOE_SWIGLU_B200_MOE_H */
