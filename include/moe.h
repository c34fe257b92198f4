/*
 * moe.h -- C ABI of the B200 (sm_100a) routed mixture-of-experts block.
 *
 * The block, as the pages define it:
 *   route    sigmoid router with a selection-only expert bias and normalised
 *            top-k: s = sigmoid(x . W_router^T); the k experts with the
 *            largest s + bias are picked; w_j = s_j / (sum_j s_j + eps) * scale.
 *            (TileGym PR #187 "[E2E Model Support] Add TileGym kernel
 *            integration for LFM2 MoE", section "Weight layout and routing";
 *            TensorFold pull #1492, sections "What" and "Verification".)
 *   plan     the grouped expert plan: per-expert counts, offsets and the
 *            permutation of routed pairs (TensorFold issue #548, "Zig CUDA
 *            ports: shared layers below lanes.Backend ...", the shared
 *            grouped-MoE layer and its routing plan).
 *   experts  grouped expert GEMMs: gate_up (E, 2I, H) gate-first with a SwiGLU
 *            epilogue, or the non-gated up (E, I, H) -> relu^2; then down
 *            (E, H, I) whose output is weighted by w and summed into the
 *            token's row (TileGym PR #187 "Weight layout and routing";
 *            vllm.cpp PR #684 "W2 (MODEL-NEMOTRON-H): the non-gated relu^2 MoE
 *            expert", section "The seam decision").
 *   combine  y = out_scale * sum_j w_j * expert_j(x): the output scale
 *            multiplies the finished sum once (vllm.cpp PR #684, "The finding
 *            that justifies the row").
 *
 * Variants, each declared below with its passage: softmax router scores and
 * norm_topk off (moe_router_cfg, moe_route_ex / moe_forward_ex), the SwiGLU
 * input clamp (moe_experts_w.swiglu_limit), a shared expert added after the
 * routed scale (moe_shared_expert, moe_forward_ex's y_shared), a skipped
 * plan expert (moe_experts_ex's skip_expert: the 9-slot plan with the shared
 * expert's id), and a slot-ordered, batch-invariant combine (moe_exec_cfg /
 * moe_set_combine).
 *
 * Conventions for every entry point
 *   - Pointers named x, logits, w_router, expert_bias, topk_*, plan arrays,
 *     weights, y and ws are DEVICE pointers (the caller owns the memory; the
 *     library allocates nothing on these paths).  moe_forward_host is the one
 *     exception and says so.
 *   - Layouts are dense row-major.  bf16 tensors are IEEE bfloat16 bit
 *     patterns (uint16).  Indices are int32.
 *   - All work is enqueued on `stream` (a cudaStream_t; NULL = the legacy
 *     default stream).  No entry point synchronises the host, except
 *     moe_device_error and moe_forward_host.
 *   - A non-OK status comes from host-side validation before anything is
 *     launched (MOE_ERR_NULL/SHAPE/ALIGN/UNSUPPORTED/WORKSPACE) or from a
 *     failed launch (MOE_ERR_CUDA).  moe_last_error() then returns a message
 *     for the calling thread.  Validation failures enqueue nothing.
 *   - Kernels never trap.  A device-side check that fails (an expert id out
 *     of range, a bounded wait that expired) writes a code to the library's
 *     device error word and the kernel returns; moe_device_error() reads it.
 */
#ifndef MOE_B200_H
#define MOE_B200_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define MOE_API __attribute__((visibility("default")))
#else
#define MOE_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st* moe_stream_t; /* same type as cudaStream_t */

typedef enum {
    MOE_OK = 0,
    MOE_ERR_NULL = 1,        /* a required pointer is NULL */
    MOE_ERR_SHAPE = 2,       /* a size is out of range (see each call) */
    MOE_ERR_ALIGN = 3,       /* a pointer is not 16-byte aligned */
    MOE_ERR_UNSUPPORTED = 4, /* an enum value or combination this build does not run */
    MOE_ERR_WORKSPACE = 5,   /* ws is NULL or smaller than moe_workspace_bytes() */
    MOE_ERR_CUDA = 6,        /* a CUDA runtime call or launch failed */
    MOE_ERR_DEVICE = 7       /* moe_device_error found a device-side error code */
} moe_status;

typedef enum { MOE_ACT_SWIGLU = 0, MOE_ACT_RELU2 = 1 } moe_act;
typedef enum { MOE_W_BF16 = 0, MOE_W_AFFINE4_G64 = 1, MOE_W_NVFP4 = 2 } moe_wfmt;

/* Which expert kernels run (per call through moe_exec_cfg, or the process-wide
 * default of moe_set_dispatch). */
typedef enum {
    MOE_DISPATCH_AUTO = 0, /* the library's choice: the tcgen05 grouped GEMM, except 4-bit
                              (affine or NVFP4) experts at <= 8 routed pairs per expert on
                              average (T*k <= 8*E, H and I <= 8192), which take the 4-bit GEMV */
    MOE_DISPATCH_GEMV = 1, /* the weight-streaming grouped GEMV (bf16: CUDA cores; 4-bit: codes
                              streamed by TMA or into registers and dequantised there,
                              m16n8k16 dot products) */
    MOE_DISPATCH_GEMM = 2  /* the tcgen05 grouped GEMM */
} moe_dispatch;

/* Problem sizes.  T tokens, H hidden, E experts, k picks per token, I expert
 * intermediate width.  P = T * k routed pairs.
 * Limits: 0 <= T, T * k < 2^31; H % 64 == 0 and 64 <= H <= 16384;
 *         I % 64 == 0 and 64 <= I <= 16384; 1 <= E <= 256; 1 <= k <= min(E, 32). */
typedef struct {
    int32_t T, H, E, k, I;
} moe_dims;

/* Expert weights (device pointers).
 *   fmt = MOE_W_BF16:
 *     act SWIGLU: w1 = gate_up (E, 2I, H) bf16, rows [0, I) gate, [I, 2I) up;
 *     act RELU2:  w1 = up (E, I, H) bf16;
 *     w2 = down (E, H, I) bf16.  *_scale and *_bias are unused (may be NULL).
 *   fmt = MOE_W_AFFINE4_G64 (MLX-style affine 4-bit, group 64 along K):
 *     w1 = codes (E, N1, H/8) uint32 with N1 = 2I (SWIGLU) or I (RELU2),
 *     w1_scale, w1_bias = (E, N1, H/64) bf16;
 *     w2 = codes (E, H, I/8) uint32, w2_scale, w2_bias = (E, H, I/64) bf16.
 *     A uint32 holds 8 consecutive k, the low nibble first; the weight is
 *     scale * q + bias (TensorFold pull #1492, "What": Affine4 experts).
 *   fmt = MOE_W_NVFP4 (ModelOpt NVFP4, read as stored, W4A16: TensorFold
 *     issue #548, "weight uint8 [N, K/2], weight_scale e4m3 [N, K/16],
 *     weight_scale_2 as the global scale", and the down projection's own
 *     global scale):
 *     w1 = codes (E, N1, H/2) uint8, two e2m1 codes per byte, the low nibble
 *     the lower k; w1_scale = (E, N1, H/16) e4m3 bytes; w1_global = (E) fp32;
 *     w2 = codes (E, H, I/2), w2_scale = (E, H, I/16), w2_global = (E) fp32;
 *     the weight is e2m1(q) * e4m3(scale) * global.  *_bias are unused.
 *     Kernels dequantise e2m1 * e4m3 exactly (into bf16 for the tcgen05
 *     GEMM, into f16 for the decode GEMV, whose token rows are staged in f16
 *     after an exact per-token power-of-two scale) and apply the global scale
 *     to the fp32 sum.
 *   swiglu_limit (SWIGLU only; 0 = off, must be >= 0 and finite): before the
 *     activation the gate is clamped from above, g = min(g, limit), and the
 *     up value on both sides, u = clamp(u, -limit, limit); NaN stays NaN
 *     (TensorFold issue #548, "Paths your experts test does not reach":
 *     swiglu_limit 10, gate and up pre-activations clamp). */
typedef struct {
    int32_t fmt; /* moe_wfmt */
    int32_t act; /* moe_act */
    const void* w1;
    const void* w1_scale;
    const void* w1_bias;
    const void* w2;
    const void* w2_scale;
    const void* w2_bias;
    float swiglu_limit;
    const float* w1_global; /* MOE_W_NVFP4 only (else unused, may be NULL) */
    const float* w2_global;
} moe_experts_w;

/* Router variants (TensorFold issue #548: the pieces each model family
 * builds include "routers (softmax, sigmoid + bias)").
 *   score = MOE_SCORE_SIGMOID (default): s = 1 / (1 + exp(-L));
 *           MOE_SCORE_SOFTMAX: s = exp(L - max L) / sum exp(L - max L) over
 *           the token's E logits (a NaN logit makes the row's scores NaN).
 *   The expert bias is added to s for selection only, either way.
 *   norm_topk = 1 (default): w_j = s_j / (sum of the k picked s + eps) * scale;
 *             = 0:           w_j = s_j * scale. */
typedef enum { MOE_SCORE_SIGMOID = 0, MOE_SCORE_SOFTMAX = 1 } moe_score;
typedef struct {
    int32_t score;     /* moe_score */
    int32_t norm_topk; /* 0 or 1 */
} moe_router_cfg;

/* The routing plan (device arrays the caller allocates).
 *   counts  [E]    pairs routed to each expert
 *   offsets [E+1]  exclusive scan of counts
 *   perm    [P]    pair ids p = t*k + j sorted stably by (expert, p)
 *   inv     [P]    inv[p] = position of pair p in perm
 *   tiles   [E+1]  exclusive scan of ceil(counts / MOE_TILE_M): the grouped
 *                  GEMM's M-tile table (tiles[E] = number of M-tiles) */
typedef struct {
    int32_t* counts;
    int32_t* offsets;
    int32_t* perm;
    int32_t* inv;
    int32_t* tiles;
} moe_plan_t;

#define MOE_TILE_M 128

/* Per-call execution choices.  Every entry point that takes a
 * `const moe_exec_cfg*` reads it once per call; NULL means the process-wide
 * defaults set by moe_set_dispatch / moe_set_combine.  Two callers in one
 * process that pass their own cfg never affect each other's kernels or
 * workspace sizes.  MOE_ERR_UNSUPPORTED for a value outside the enums.
 *   dispatch: moe_dispatch (which expert kernels run)
 *   combine:  moe_combine  (atomic or slot-ordered combine; see moe_set_combine) */
typedef struct {
    int32_t dispatch;
    int32_t combine;
} moe_exec_cfg;

/* Byte offsets of the regions inside the workspace (for inspection/tests). */
typedef struct {
    size_t y_acc;   /* fp32 (T, H): the unscaled routed sum; (P, H) weighted slot outputs
                       under MOE_COMBINE_ORDERED */
    size_t h;       /* bf16 (P, I): activations in plan order */
    size_t xs;      /* bf16 (P, H): token rows gathered in plan order (tcgen05 GEMM path) */
    size_t scratch; /* plan and scheduler scratch */
    size_t total;   /* == moe_workspace_bytes() */
} moe_ws_layout;

/* Bytes of device workspace moe_plan / moe_experts / moe_forward need for
 * these sizes and weight format (0 on invalid sizes).  256-byte aligned
 * regions; ws itself must be 256-byte aligned. */
MOE_API size_t moe_workspace_bytes(const moe_dims* d, int32_t fmt);
MOE_API moe_status moe_workspace_layout(const moe_dims* d, int32_t fmt, moe_ws_layout* out);
/* The same for the combine mode of `exec` (NULL = the process-wide default);
 * 0 / MOE_ERR_UNSUPPORTED for an invalid exec. */
MOE_API size_t moe_workspace_bytes_ex(const moe_dims* d, int32_t fmt, const moe_exec_cfg* exec);
MOE_API moe_status moe_workspace_layout_ex(const moe_dims* d, int32_t fmt, const moe_exec_cfg* exec,
                                           moe_ws_layout* out);

/* Router.  Exactly one of x (bf16 (T, H)) or logits (fp32 (T, E)) is given;
 * with x, w_router (fp32 (E, H)) is required and the logits are computed in
 * fp32 with a fixed summation order (a token's result never depends on T).
 * expert_bias (fp32 (E)) may be NULL (no bias).  Writes topk_idx (T, k) int32
 * in rank order (descending s + bias, ties to the lower id, NaN last; an
 * all-NaN row picks 0..k-1) and topk_w (T, k) fp32 = s / (sum s + eps) * scale.
 * A row whose logits are all NaN gets NaN weights. */
MOE_API moe_status moe_route(const void* x, const float* logits, const float* w_router,
                     const float* expert_bias, const moe_dims* d, float eps, float scale,
                     int32_t* topk_idx, float* topk_w, moe_stream_t stream);

/* Plan of topk_idx (T, k) int32 (values must lie in [0, E); a value outside
 * sets device error code 1 and is counted nowhere).  Fills every array of
 * *plan.  Uses the scratch region of ws. */
MOE_API moe_status moe_plan(const int32_t* topk_idx, const moe_dims* d, const moe_plan_t* plan, void* ws,
                    size_t ws_bytes, moe_stream_t stream);

/* Grouped experts + combine: y (T, H) bf16 = bf16_rn(out_scale * y_acc) where
 * y_acc[t] = sum_j topk_w[t, j] * down_e(act(up_e(x[t]))) in fp32, e = the
 * pair's expert.  The activation is rounded once to bf16 (stored in ws.h);
 * y_acc is kept in ws.y_acc.  Rows of y for tokens with no pairs are 0. */
MOE_API moe_status moe_experts(const void* x, const moe_plan_t* plan, const float* topk_w,
                       const moe_dims* d, const moe_experts_w* W, float out_scale, void* y,
                       void* ws, size_t ws_bytes, moe_stream_t stream);

/* moe_experts with a per-call exec cfg, a skipped plan expert and a shared
 * expert's output.
 *   skip_expert = -1: as moe_experts.
 *   skip_expert = s in [0, E): the pairs the plan routes to plan expert s are
 *     computed nowhere and left out of the combine, and the rows they own
 *     (their h rows, and their slot rows under the ordered combine) are not
 *     written.  This is the 9-slot plan of TensorFold issue #548 ("Paths your
 *     experts test does not reach", the skip-a-slot row): top-8 plus the
 *     shared expert's id E over E + 1 plan experts, with id E skipped, gives
 *     the bytes of the 8-slot block.  Here d->E counts the plan experts; W
 *     holds d->E - 1 experts when s == d->E - 1 (the shared id has no routed
 *     weights), else d->E.  MOE_ERR_SHAPE for s outside [-1, E) or s >= 0 with E == 1.
 *   y_shared: fp32 (T, H) or NULL, added after the routed scale as in
 *     moe_forward_ex. */
MOE_API moe_status moe_experts_ex(const void* x, const moe_plan_t* plan, const float* topk_w,
                                  const moe_dims* d, const moe_experts_w* W, const moe_exec_cfg* exec,
                                  int32_t skip_expert, const float* y_shared, float out_scale, void* y,
                                  void* ws, size_t ws_bytes, moe_stream_t stream);

/* route -> plan -> experts -> combine in one call (same arguments as the three
 * calls; logits may be NULL to route from x). */
MOE_API moe_status moe_forward(const void* x, const float* logits, const float* w_router,
                       const float* expert_bias, const moe_dims* d, float eps, float router_scale,
                       float out_scale, const moe_experts_w* W, int32_t* topk_idx, float* topk_w,
                       const moe_plan_t* plan, void* y, void* ws, size_t ws_bytes,
                       moe_stream_t stream);

/* moe_route and moe_forward with a router configuration (NULL = the
 * defaults above: sigmoid scores, normalised top-k).  Everything else as
 * moe_route / moe_forward; MOE_ERR_UNSUPPORTED for an unknown score or a
 * norm_topk other than 0 or 1.  moe_forward_ex also takes y_shared, an fp32
 * (T, H) shared-expert output (from moe_shared_expert) or NULL: the output is
 * then y = bf16_rn(out_scale * routed sum + y_shared) -- the routed scale
 * multiplies the routed sum before the shared term is added, which itself is
 * not scaled (vllm.cpp PR #684, "The finding that justifies the row").
 * moe_forward_ex's exec (NULL = the process-wide defaults) picks its expert
 * kernels and combine mode for this call. */
MOE_API moe_status moe_route_ex(const void* x, const float* logits, const float* w_router,
                                const float* expert_bias, const moe_dims* d, float eps, float scale,
                                const moe_router_cfg* cfg, int32_t* topk_idx, float* topk_w,
                                moe_stream_t stream);
MOE_API moe_status moe_forward_ex(const void* x, const float* logits, const float* w_router,
                                  const float* expert_bias, const moe_dims* d, float eps,
                                  float router_scale, float out_scale, const moe_router_cfg* cfg,
                                  const moe_exec_cfg* exec,
                                  const float* y_shared, const moe_experts_w* W, int32_t* topk_idx,
                                  float* topk_w,
                                  const moe_plan_t* plan, void* y, void* ws, size_t ws_bytes,
                                  moe_stream_t stream);

/* The shared expert: one expert applied to every token with weight 1,
 *   y_shared[t] = down_s(act(up_s(x[t])))   (fp32 (T, H), overwritten),
 * for moe_forward_ex's y_shared.  d = {T, H, E = 1, k = 1, I = the shared
 * expert's width}; Ws has the same layout as one expert of moe_experts_w
 * (E = 1; act, fmt and swiglu_limit as for the routed experts).  The
 * workspace is moe_workspace_bytes(d, Ws->fmt) for that d.  Runs the same
 * kernels as the routed experts (tcgen05 GEMM or GEMV, per moe_set_dispatch)
 * over a one-expert identity plan.  MOE_ERR_SHAPE unless E == 1 and k == 1. */
MOE_API moe_status moe_shared_expert(const void* x, const moe_experts_w* Ws, const moe_dims* d,
                                     float* y_shared, void* ws, size_t ws_bytes, moe_stream_t stream);
/* moe_shared_expert with a per-call exec cfg (NULL = the process-wide defaults). */
MOE_API moe_status moe_shared_expert_ex(const void* x, const moe_experts_w* Ws, const moe_dims* d,
                                        const moe_exec_cfg* exec, float* y_shared, void* ws,
                                        size_t ws_bytes, moe_stream_t stream);

/* moe_forward with HOST buffers for the token rows: x_host (T, H) bf16 is
 * copied to x_dev, the block runs, and y_dev is copied back to y_host (T, H)
 * bf16, all on `stream`; the call then synchronises `stream`.  x_host/y_host
 * should be pinned for the copies to be asynchronous.  Everything else is as
 * moe_forward (device pointers). */
MOE_API moe_status moe_forward_host(const void* x_host, void* x_dev, const float* w_router,
                            const float* expert_bias, const moe_dims* d, float eps,
                            float router_scale, float out_scale, const moe_experts_w* W,
                            int32_t* topk_idx, float* topk_w, const moe_plan_t* plan, void* y_dev,
                            void* y_host, void* ws, size_t ws_bytes, moe_stream_t stream);

/* Stages of the block, for moe_profile_hook. */
typedef enum {
    MOE_STAGE_ROUTE = 0,   /* the router kernel(s): logits + selection (+ plan for T <= 32) */
    MOE_STAGE_PLAN = 1,    /* the plan kernel (fused into the router for T <= 32) */
    MOE_STAGE_UP = 2,      /* the expert up-projection + activation kernel */
    MOE_STAGE_DOWN = 3,    /* the expert down-projection + weighted scatter kernel */
    MOE_STAGE_FINAL = 4,   /* the output scale + bf16 rounding kernel */
    MOE_STAGE_GATHER = 5   /* the copy of token rows into plan order (tcgen05 GEMM path) */
} moe_stage;

/* One-shot timing hook for the calling thread: the next moe_forward /
 * moe_experts call on this thread records ev_begin (a cudaEvent_t) on its
 * stream just before launching `stage`'s kernel and ev_end just after, then
 * forgets the hook.  Pass NULL events to clear it.  Works under stream
 * capture (the records become event nodes). */
MOE_API moe_status moe_profile_hook(void* ev_begin, void* ev_end, int32_t stage);

/* Number of kernels the calling thread's last successful moe_* call launched. */
MOE_API int32_t moe_last_launch_count(void);

/* moe_forward for callers that cannot allocate device memory.  (The pages
 * have no counterpart: this is an interface choice of this library.)
 * Some callers have no workspace to give: a plugin host that hands a custom
 * op only its input and output tensors, or a latency-bound serving loop that
 * must never wait on an allocator.  This call takes the same arguments as moe_forward
 * minus ws/ws_bytes: its scratch (fp32 accumulator, bf16 activations, router
 * logits) is one fixed 16 MiB device array inside the library, which every GPU
 * that loads the library holds until the process exits.  It allocates
 * nothing: no cudaMalloc, cudaFree or allocating library call.
 *   - Sizes whose scratch exceeds 16 MiB (T*H*4 + T*k*I*2 + 32*E*4 + 4 KiB,
 *     each rounded up to 256 bytes) are refused with MOE_ERR_WORKSPACE and a
 *     message giving the bytes needed.  Runs bf16 weights only, always on the
 *     weight-streaming grouped GEMV (MOE_ERR_UNSUPPORTED for affine 4-bit).
 *   - The first call on a device looks up the array's device address on that
 *     device (cudaGetSymbolAddress, once per device, with the device current).
 *   - Every call shares the array and it keeps the last call's contents (the
 *     accumulator is cleared at the start of each call).  Calls whose work
 *     overlaps on the GPU (other streams, other threads) race on it: run them
 *     one after another on one stream. */
MOE_API moe_status moe_forward_static(const void* x, const float* logits, const float* w_router,
                                      const float* expert_bias, const moe_dims* d, float eps,
                                      float router_scale, float out_scale, const moe_experts_w* W,
                                      int32_t* topk_idx, float* topk_w, const moe_plan_t* plan,
                                      void* y, moe_stream_t stream);

/* Process-wide default choice of expert kernels (moe_dispatch), used by calls
 * given no moe_exec_cfg; returns the old one. */
MOE_API int32_t moe_set_dispatch(int32_t mode);

/* How the weighted expert outputs of a token are combined: the process-wide
 * default, used by calls given no moe_exec_cfg.
 *   MOE_COMBINE_ATOMIC  (default): the down projection adds w_j * o_j into the
 *     fp32 accumulator y_acc (T, H) with atomic reductions; the order of the
 *     k additions, and so the last bits of y, can vary from run to run.
 *   MOE_COMBINE_ORDERED: the down projection stores w_j * o_j per plan slot
 *     (fp32 (P, H), in the workspace's y_acc region) and the finalize sums a
 *     token's k slots in slot order j = 0..k-1, then scales once.  y is then
 *     bitwise reproducible, and for bf16 experts a token's y does not depend
 *     on the other tokens of the batch (the router already has a fixed
 *     summation order).  The workspace is larger (P * H * 4 bytes for that
 *     region): query moe_workspace_bytes after setting the mode, or pass the mode
 *     per call through moe_exec_cfg and moe_workspace_bytes_ex.  Not used by
 *     moe_forward_static. */
typedef enum { MOE_COMBINE_ATOMIC = 0, MOE_COMBINE_ORDERED = 1 } moe_combine;
MOE_API int32_t moe_set_combine(int32_t mode);

/* Failure-detection check (the pages have no counterpart; this exercises the
 * library's own stall detection).  Every mbarrier wait of the tcgen05
 * pipelines is bounded: when its poll limit runs out the kernel writes device
 * error code 2, drains what it issued, frees its TMEM and returns.  This call
 * launches one single-warp kernel that runs that same bounded wait, with a
 * limit of `polls` polls (1 <= polls <= 2^20), on an mbarrier nothing arrives
 * on -- no TMA, no TMEM, no other work -- so the wait expires, code 2 is
 * written and the kernel returns.  moe_device_error then reports code 2 and
 * the context stays usable.  MOE_ERR_SHAPE for polls out of range. */
MOE_API moe_status moe_wait_bound_check(uint32_t polls, moe_stream_t stream);

/* Synchronises `stream`, then reads and clears the device error word of the
 * current device.  *code = 0 when no kernel reported an error.  Codes:
 * 1 expert id out of range in moe_plan; 2 a bounded pipeline wait expired in
 * a grouped GEMM kernel.  Returns MOE_ERR_DEVICE when *code != 0. */
MOE_API moe_status moe_device_error(int32_t* code, moe_stream_t stream);

/* Message for the calling thread's last non-OK status ("" if none). */
MOE_API const char* moe_last_error(void);

/* Library version string. */
MOE_API const char* moe_version(void);

#ifdef __cplusplus
}
#endif

#endif /* MOE_B200_H */
