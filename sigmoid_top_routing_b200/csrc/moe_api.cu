// C-ABI host layer: argument validation, workspace layout, launch sequencing.
// Every stage is enqueued on the caller's stream with programmatic dependent
// launch, so a kernel's launch overlaps the tail of the one before it; each
// kernel waits (griddepcontrol.wait) before it reads anything.
#include <cstdarg>
#include <cstdio>
#include <map>
#include <mutex>
#include <string>

#include "../../include/moe.h"
#include "internal.h"

namespace moe {

__device__ int g_err_word;   // the library's device error word (one per device)

const DeviceInfo& device_info() {
    static std::mutex mu;
    static std::map<int, DeviceInfo> cache;
    int dev = 0;
    cudaGetDevice(&dev);
    std::lock_guard<std::mutex> lock(mu);
    auto it = cache.find(dev);
    if (it != cache.end()) return it->second;
    DeviceInfo di{};
    cudaDeviceGetAttribute(&di.sm_count, cudaDevAttrMultiProcessorCount, dev);
    cudaDeviceGetAttribute(&di.max_smem_optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev);
    cudaDeviceGetAttribute(&di.smem_per_sm, cudaDevAttrMaxSharedMemoryPerMultiprocessor, dev);
    if (cudaGetSymbolAddress(reinterpret_cast<void**>(&di.err_word), g_err_word) != cudaSuccess)
        di.err_word = nullptr;
    if (di.sm_count <= 0) di.sm_count = 1;
    return cache.emplace(dev, di).first->second;
}

}  // namespace moe

using namespace moe;

namespace {

thread_local std::string g_last_error;
thread_local int g_launches = 0;      // kernels launched by the thread's last successful call
struct Hook {
    cudaEvent_t begin = nullptr, end = nullptr;
    int stage = -1;
};
thread_local Hook g_hook;
std::mutex g_dispatch_mu;
int g_dispatch = MOE_DISPATCH_AUTO;
int g_combine = MOE_COMBINE_ATOMIC;   // guarded by g_dispatch_mu

moe_status fail(moe_status st, const char* fmt, ...) {
    char buf[512];
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(buf, sizeof buf, fmt, ap);
    va_end(ap);
    g_last_error = buf;
    return st;
}

moe_status cuda_fail(cudaError_t e, const char* what) {
    return fail(MOE_ERR_CUDA, "%s: %s (%s)", what, cudaGetErrorName(e), cudaGetErrorString(e));
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
size_t align256(size_t v) { return (v + 255) & ~size_t(255); }

moe_status check_dims(const moe_dims* d) {
    if (!d) return fail(MOE_ERR_NULL, "dims is NULL");
    if (d->T < 0) return fail(MOE_ERR_SHAPE, "T = %d < 0", d->T);
    if (d->H < 64 || d->H > 16384 || d->H % 64)
        return fail(MOE_ERR_SHAPE, "H = %d: need 64 <= H <= 16384 and H %% 64 == 0", d->H);
    if (d->I < 64 || d->I > 16384 || d->I % 64)
        return fail(MOE_ERR_SHAPE, "I = %d: need 64 <= I <= 16384 and I %% 64 == 0", d->I);
    if (d->E < 1 || d->E > 256) return fail(MOE_ERR_SHAPE, "E = %d: need 1 <= E <= 256", d->E);
    if (d->k < 1 || d->k > d->E || d->k > 32)
        return fail(MOE_ERR_SHAPE, "k = %d: need 1 <= k <= min(E, 32)", d->k);
    if ((long long)d->T * d->k >= (1ll << 31)) return fail(MOE_ERR_SHAPE, "T * k >= 2^31");
    return MOE_OK;
}

moe_status check_fmt(int32_t fmt) {
    if (fmt != MOE_W_BF16 && fmt != MOE_W_AFFINE4_G64 && fmt != MOE_W_NVFP4)
        return fail(MOE_ERR_UNSUPPORTED, "weight format %d", fmt);
    return MOE_OK;
}

// A call's execution choices, read once per call.
struct Exec {
    int dispatch;            // moe_dispatch
    bool ordered;            // slot-ordered combine
};

// The call's cfg, or the process-wide defaults when it passes none.
moe_status resolve_exec(const moe_exec_cfg* cfg, Exec* x) {
    if (!cfg) {
        std::lock_guard<std::mutex> lock(g_dispatch_mu);
        x->dispatch = g_dispatch;
        x->ordered = g_combine == MOE_COMBINE_ORDERED;
        return MOE_OK;
    }
    if (cfg->dispatch != MOE_DISPATCH_AUTO && cfg->dispatch != MOE_DISPATCH_GEMV && cfg->dispatch != MOE_DISPATCH_GEMM)
        return fail(MOE_ERR_UNSUPPORTED, "exec dispatch %d", cfg->dispatch);
    if (cfg->combine != MOE_COMBINE_ATOMIC && cfg->combine != MOE_COMBINE_ORDERED)
        return fail(MOE_ERR_UNSUPPORTED, "exec combine %d", cfg->combine);
    x->dispatch = cfg->dispatch;
    x->ordered = cfg->combine == MOE_COMBINE_ORDERED;
    return MOE_OK;
}

// ordered: the combine mode the call runs with (read once per call)
void layout(const moe_dims* d, moe_ws_layout* L, bool ordered) {
    const size_t T = d->T, H = d->H, E = d->E, P = (size_t)d->T * d->k, I = d->I;
    size_t off = 0;
    L->y_acc = off;       // (T, H) sums, or (P, H) slot outputs for the ordered combine
    off = align256(off + (ordered ? P : T) * H * 4);
    L->h = off;
    off = align256(off + P * I * 2);
    L->xs = off;          // token rows gathered in plan order (the up GEMM reads them by TMA)
    off = align256(off + P * H * 2);
    // scratch: router logits (T <= 32) | plan histograms and bases | per-segment partial logits
    L->scratch = off;
    off = align256(off + (size_t)kSmallT * E * 4 + 4096 + plan_scratch_ints((int)P, (int)E) * 4);
    off = align256(off + (size_t)8 * T * E * 4);
    L->total = off;
}

struct WsView {
    float* y_acc;
    uint16_t* h;
    uint16_t* xs;
    float* l_scratch;
    int32_t* plan_scratch;
    float* part;
    bool ordered;            // the combine mode of this call (read once)
};

moe_status check_ws(const moe_dims* d, void* ws, size_t ws_bytes, bool ordered, WsView* v) {
    moe_ws_layout L;
    v->ordered = ordered;
    layout(d, &L, ordered);
    if (!ws) return fail(MOE_ERR_WORKSPACE, "workspace is NULL");
    if (reinterpret_cast<uintptr_t>(ws) & 255u) return fail(MOE_ERR_ALIGN, "workspace not 256-byte aligned");
    if (ws_bytes < L.total)
        return fail(MOE_ERR_WORKSPACE, "workspace %zu bytes < %zu needed", ws_bytes, L.total);
    char* b = static_cast<char*>(ws);
    v->y_acc = reinterpret_cast<float*>(b + L.y_acc);
    v->h = reinterpret_cast<uint16_t*>(b + L.h);
    v->xs = reinterpret_cast<uint16_t*>(b + L.xs);
    v->l_scratch = reinterpret_cast<float*>(b + L.scratch);
    const size_t off_plan = L.scratch + (size_t)kSmallT * d->E * 4 + 4096;
    v->plan_scratch = reinterpret_cast<int32_t*>(b + off_plan);
    v->part = reinterpret_cast<float*>(
        b + align256(off_plan + plan_scratch_ints(d->T * d->k, d->E) * 4));
    return MOE_OK;
}

moe_status check_plan(const moe_plan_t* plan) {
    if (!plan) return fail(MOE_ERR_NULL, "plan is NULL");
    if (!plan->counts || !plan->offsets || !plan->perm || !plan->inv || !plan->tiles)
        return fail(MOE_ERR_NULL, "a plan array is NULL");
    return MOE_OK;
}

moe_status check_weights(const moe_experts_w* W) {
    if (!W) return fail(MOE_ERR_NULL, "weights struct is NULL");
    if (W->act != MOE_ACT_SWIGLU && W->act != MOE_ACT_RELU2)
        return fail(MOE_ERR_UNSUPPORTED, "activation %d", W->act);
    moe_status st = check_fmt(W->fmt);
    if (st != MOE_OK) return st;
    if (!W->w1 || !W->w2) return fail(MOE_ERR_NULL, "w1 or w2 is NULL");
    if (!aligned16(W->w1) || !aligned16(W->w2)) return fail(MOE_ERR_ALIGN, "w1/w2 not 16-byte aligned");
    if (W->fmt == MOE_W_AFFINE4_G64) {
        if (!W->w1_scale || !W->w1_bias || !W->w2_scale || !W->w2_bias)
            return fail(MOE_ERR_NULL, "affine-4 scale/bias pointer is NULL");
        if (!aligned16(W->w1_scale) || !aligned16(W->w1_bias) || !aligned16(W->w2_scale) ||
            !aligned16(W->w2_bias))
            return fail(MOE_ERR_ALIGN, "affine-4 scale/bias not 16-byte aligned");
    }
    if (W->fmt == MOE_W_NVFP4) {
        if (!W->w1_scale || !W->w2_scale || !W->w1_global || !W->w2_global)
            return fail(MOE_ERR_NULL, "NVFP4 block-scale or global-scale pointer is NULL");
        if (!aligned16(W->w1_scale) || !aligned16(W->w2_scale))
            return fail(MOE_ERR_ALIGN, "NVFP4 block scales not 16-byte aligned");
        if ((reinterpret_cast<uintptr_t>(W->w1_global) | reinterpret_cast<uintptr_t>(W->w2_global)) & 3u)
            return fail(MOE_ERR_ALIGN, "NVFP4 global scales not 4-byte aligned");
    }
    if (!(W->swiglu_limit >= 0.0f) || W->swiglu_limit > 3.0e38f)
        return fail(MOE_ERR_SHAPE, "swiglu_limit must be finite and >= 0 (0 = off)");
    return MOE_OK;
}

// The router configuration (NULL: sigmoid scores, normalised top-k).
moe_status check_router_cfg(const moe_router_cfg* cfg, RouteArgs* r) {
    if (!cfg) return MOE_OK;
    if (cfg->score != MOE_SCORE_SIGMOID && cfg->score != MOE_SCORE_SOFTMAX)
        return fail(MOE_ERR_UNSUPPORTED, "router score %d", cfg->score);
    if (cfg->norm_topk != 0 && cfg->norm_topk != 1) return fail(MOE_ERR_UNSUPPORTED, "norm_topk %d", cfg->norm_topk);
    r->softmax = cfg->score == MOE_SCORE_SOFTMAX;
    r->no_norm = cfg->norm_topk == 0;
    return MOE_OK;
}

moe_status check_route_args(const void* x, const float* logits, const float* w_router,
                            const moe_dims* d, int32_t* idx, float* w) {
    if ((x == nullptr) == (logits == nullptr))
        return fail(MOE_ERR_NULL, "give exactly one of x or logits");
    if (x && !w_router) return fail(MOE_ERR_NULL, "w_router is NULL (routing from x)");
    if (!idx || !w) return fail(MOE_ERR_NULL, "topk_idx or topk_w is NULL");
    if (x && (!aligned16(x) || !aligned16(w_router)))
        return fail(MOE_ERR_ALIGN, "x / w_router not 16-byte aligned");
    (void)d;
    return MOE_OK;
}

// bf16: the tcgen05 grouped GEMM serves every token count (its token tiles
// shrink to 32 for decode batches); the CUDA-core GEMV stays selectable.
// 4-bit (affine, NVFP4): up to a few pairs per expert the GEMVs stream the
// codes faster than the GEMM's shared-memory dequant pipeline.
bool use_gemv(const moe_dims* d, int32_t fmt, int mode) {
    if (mode != MOE_DISPATCH_AUTO) return mode == MOE_DISPATCH_GEMV;
    if (fmt == MOE_W_NVFP4 && !kNvfp4Gemm) return true;   // no tcgen05 NVFP4 path in this build
    return (fmt == MOE_W_AFFINE4_G64 || fmt == MOE_W_NVFP4) && d->H <= 8192 && d->I <= 8192 &&
           (size_t)d->T * d->k <= (size_t)kAffineGemvMaxPairsPerExpert * d->E;
}

ExpertArgs make_expert_args(const void* x, const moe_plan_t* plan, const float* topk_w,
                            const moe_dims* d, const moe_experts_w* W, float out_scale, void* y,
                            const WsView& v) {
    ExpertArgs a{};
    a.x = static_cast<const uint16_t*>(x);
    a.topk_w = topk_w;
    a.counts = plan->counts;
    a.offsets = plan->offsets;
    a.perm = plan->perm;
    a.inv = plan->inv;
    a.tiles = plan->tiles;
    a.T = d->T;
    a.H = d->H;
    a.E = d->E;
    a.k = d->k;
    a.I = d->I;
    a.E_w = d->E;
    a.skip = -1;
    a.act = W->act;
    a.fmt = W->fmt;
    a.swiglu_limit = W->swiglu_limit;
    a.w1 = W->w1;
    a.w1_scale = static_cast<const uint16_t*>(W->w1_scale);
    a.w1_bias = static_cast<const uint16_t*>(W->w1_bias);
    a.w2 = W->w2;
    a.w2_scale = static_cast<const uint16_t*>(W->w2_scale);
    a.w2_bias = static_cast<const uint16_t*>(W->w2_bias);
    a.w1_global = W->fmt == MOE_W_NVFP4 ? W->w1_global : nullptr;
    a.w2_global = W->fmt == MOE_W_NVFP4 ? W->w2_global : nullptr;
    a.h = v.h;
    a.xs = v.xs;
    a.y_acc = v.y_acc;
    a.ordered = v.ordered ? 1 : 0;
    a.y = static_cast<uint16_t*>(y);
    a.out_scale = out_scale;
    a.err = device_info().err_word;
    return a;
}

// Event record that also works under stream capture (an event node there).
cudaError_t record_event(cudaEvent_t ev, cudaStream_t s) {
    cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
    cudaError_t e = cudaStreamIsCapturing(s, &cs);
    if (e != cudaSuccess) return e;
    if (cs == cudaStreamCaptureStatusActive) return cudaEventRecordWithFlags(ev, s, cudaEventRecordExternal);
    return cudaEventRecord(ev, s);
}

// Enqueues stages on one stream; records the one-shot hook's events around
// the hooked stage and counts kernels.
struct Seq {
    cudaStream_t s;
    int n = 0;
    template <class F>
    cudaError_t stage(int id, F&& f) {   // f(int* launched) -> cudaError_t
        const bool hooked = g_hook.stage == id && g_hook.begin && g_hook.end;
        cudaError_t e;
        if (hooked && (e = record_event(g_hook.begin, s)) != cudaSuccess) return e;
        int launched = 1;
        if ((e = f(&launched)) != cudaSuccess) return e;
        n += launched;
        if (hooked) {
            e = record_event(g_hook.end, s);
            g_hook = Hook{};
            if (e != cudaSuccess) return e;
        }
        return cudaSuccess;
    }
};

moe_status run_experts(Seq& q, const ExpertArgs& a, const moe_dims* d, int dispatch) {
    const bool gemv = use_gemv(d, a.fmt, dispatch);
    cudaError_t e;
    if (!gemv && !gemm_up_reads_x(a)) {
        // token rows in plan order for the up GEMM's TMA (part of the plan's data movement)
        e = q.stage(MOE_STAGE_GATHER, [&](int*) { return launch_gather_x(a, true, q.s); });
        if (e != cudaSuccess) return cuda_fail(e, "gather token rows");
    }
    e = q.stage(MOE_STAGE_UP, [&](int*) {
        return gemv ? launch_gemv_up(a, true, q.s) : launch_gemm_up(a, true, q.s);
    });
    if (e == cudaErrorNotSupported)
        return fail(MOE_ERR_UNSUPPORTED, "no expert kernel for this format/path in this build");
    if (e != cudaSuccess) return cuda_fail(e, "expert up kernel");
    e = q.stage(MOE_STAGE_DOWN, [&](int*) {
        return gemv ? launch_gemv_down(a, true, q.s) : launch_gemm_down(a, true, q.s);
    });
    if (e == cudaErrorNotSupported)
        return fail(MOE_ERR_UNSUPPORTED, "no expert kernel for this format/path in this build");
    if (e != cudaSuccess) return cuda_fail(e, "expert down kernel");
    e = q.stage(MOE_STAGE_FINAL, [&](int*) { return launch_finalize(a, true, q.s); });
    if (e != cudaSuccess) return cuda_fail(e, "finalize");
    return MOE_OK;
}

PlanArgs make_plan_args(const int32_t* idx, const moe_dims* d, const moe_plan_t* plan, int32_t* scratch) {
    PlanArgs p{};
    p.scratch = scratch;
    p.idx = idx;
    p.P = d->T * d->k;
    p.E = d->E;
    p.k = d->k;
    p.counts = plan->counts;
    p.offsets = plan->offsets;
    p.perm = plan->perm;
    p.inv = plan->inv;
    p.tiles = plan->tiles;
    p.err = device_info().err_word;
    return p;
}

}  // namespace

namespace moe {
// For entry points defined in other files of the library.
void set_last_error(const char* msg) { g_last_error = msg; }
void set_last_launch_count(int n) { g_launches = n; }
moe_status validate_dims(const moe_dims* d) { return check_dims(d); }
moe_status validate_plan(const moe_plan_t* plan) { return check_plan(plan); }
moe_status validate_weights(const moe_experts_w* W) { return check_weights(W); }
}  // namespace moe

extern "C" {

size_t moe_workspace_bytes(const moe_dims* d, int32_t fmt) { return moe_workspace_bytes_ex(d, fmt, nullptr); }

size_t moe_workspace_bytes_ex(const moe_dims* d, int32_t fmt, const moe_exec_cfg* exec) {
    Exec x;
    if (check_dims(d) != MOE_OK || check_fmt(fmt) != MOE_OK || resolve_exec(exec, &x) != MOE_OK) return 0;
    moe_ws_layout L;
    layout(d, &L, x.ordered);
    return L.total;
}

moe_status moe_workspace_layout(const moe_dims* d, int32_t fmt, moe_ws_layout* out) {
    return moe_workspace_layout_ex(d, fmt, nullptr, out);
}

moe_status moe_workspace_layout_ex(const moe_dims* d, int32_t fmt, const moe_exec_cfg* exec, moe_ws_layout* out) {
    moe_status st = check_dims(d);
    if (st != MOE_OK) return st;
    if ((st = check_fmt(fmt)) != MOE_OK) return st;
    Exec x;
    if ((st = resolve_exec(exec, &x)) != MOE_OK) return st;
    if (!out) return fail(MOE_ERR_NULL, "out is NULL");
    layout(d, out, x.ordered);
    return MOE_OK;
}

moe_status moe_route(const void* x, const float* logits, const float* w_router,
                     const float* expert_bias, const moe_dims* d, float eps, float scale,
                     int32_t* topk_idx, float* topk_w, moe_stream_t stream) {
    return moe_route_ex(x, logits, w_router, expert_bias, d, eps, scale, nullptr, topk_idx, topk_w, stream);
}

moe_status moe_route_ex(const void* x, const float* logits, const float* w_router,
                        const float* expert_bias, const moe_dims* d, float eps, float scale,
                        const moe_router_cfg* cfg, int32_t* topk_idx, float* topk_w, moe_stream_t stream) {
    moe_status st = check_dims(d);
    if (st != MOE_OK) return st;
    RouteArgs a{};
    if ((st = check_router_cfg(cfg, &a)) != MOE_OK) return st;
    if (d->T == 0) return g_launches = 0, MOE_OK;   // empty batch: nothing to do
    if ((st = check_route_args(x, logits, w_router, d, topk_idx, topk_w)) != MOE_OK) return st;
    a.x = static_cast<const uint16_t*>(x);
    a.logits = logits;
    a.w_router = w_router;
    a.bias = expert_bias;
    a.T = d->T;
    a.H = d->H;
    a.E = d->E;
    a.k = d->k;
    a.eps = eps;
    a.scale = scale;
    a.idx = topk_idx;
    a.w = topk_w;
    a.err = device_info().err_word;
    Seq q{reinterpret_cast<cudaStream_t>(stream)};
    cudaError_t e = q.stage(MOE_STAGE_ROUTE, [&](int* n) { return launch_route(a, false, true, q.s, n); });
    if (e != cudaSuccess) return cuda_fail(e, "route");
    g_launches = q.n;
    return MOE_OK;
}

moe_status moe_plan(const int32_t* topk_idx, const moe_dims* d, const moe_plan_t* plan, void* ws,
                    size_t ws_bytes, moe_stream_t stream) {
    moe_status st = check_dims(d);
    if (st != MOE_OK) return st;
    if (d->T == 0) return g_launches = 0, MOE_OK;   // empty batch: nothing to do
    if (!topk_idx) return fail(MOE_ERR_NULL, "topk_idx is NULL");
    if ((st = check_plan(plan)) != MOE_OK) return st;
    WsView v;   // the plan uses only the scratch region, placed as in the (smaller) atomic layout
    if ((st = check_ws(d, ws, ws_bytes, false, &v)) != MOE_OK) return st;
    const PlanArgs p = make_plan_args(topk_idx, d, plan, v.plan_scratch);
    Seq q{reinterpret_cast<cudaStream_t>(stream)};
    cudaError_t e = q.stage(MOE_STAGE_PLAN, [&](int* n) { return launch_plan(p, true, q.s, n); });
    if (e != cudaSuccess) return cuda_fail(e, "plan");
    g_launches = q.n;
    return MOE_OK;
}

moe_status moe_experts(const void* x, const moe_plan_t* plan, const float* topk_w,
                       const moe_dims* d, const moe_experts_w* W, float out_scale, void* y,
                       void* ws, size_t ws_bytes, moe_stream_t stream) {
    return moe_experts_ex(x, plan, topk_w, d, W, nullptr, -1, nullptr, out_scale, y, ws, ws_bytes, stream);
}

moe_status moe_experts_ex(const void* x, const moe_plan_t* plan, const float* topk_w, const moe_dims* d,
                          const moe_experts_w* W, const moe_exec_cfg* exec, int32_t skip_expert,
                          const float* y_shared, float out_scale, void* y, void* ws, size_t ws_bytes,
                          moe_stream_t stream) {
    moe_status st = check_dims(d);
    if (st != MOE_OK) return st;
    if (skip_expert < -1 || skip_expert >= d->E)
        return fail(MOE_ERR_SHAPE, "skip_expert = %d: need -1 <= skip_expert < E = %d", skip_expert, d->E);
    if (skip_expert >= 0 && d->E < 2) return fail(MOE_ERR_SHAPE, "skip_expert needs E >= 2 plan experts");
    Exec xc;
    if ((st = resolve_exec(exec, &xc)) != MOE_OK) return st;
    if (d->T == 0) return g_launches = 0, MOE_OK;   // empty batch: nothing to do
    if (!x || !topk_w || !y) return fail(MOE_ERR_NULL, "x, topk_w or y is NULL");
    if (!aligned16(x) || !aligned16(y)) return fail(MOE_ERR_ALIGN, "x or y not 16-byte aligned");
    if (y_shared && !aligned16(y_shared)) return fail(MOE_ERR_ALIGN, "y_shared not 16-byte aligned");
    if ((st = check_plan(plan)) != MOE_OK) return st;
    if ((st = check_weights(W)) != MOE_OK) return st;
    WsView v;
    if ((st = check_ws(d, ws, ws_bytes, xc.ordered, &v)) != MOE_OK) return st;
    Seq q{reinterpret_cast<cudaStream_t>(stream)};
    ExpertArgs a = make_expert_args(x, plan, topk_w, d, W, out_scale, y, v);
    a.skip = skip_expert;
    a.E_w = skip_expert == d->E - 1 ? d->E - 1 : d->E;   // the last plan expert skipped: no weights for it
    a.y_shared = y_shared;
    if (!a.ordered) {   // the ordered combine writes every slot row it sums: nothing to clear
        cudaError_t e = launch_zero(v.y_acc, (size_t)d->T * d->H, true, q.s);
        if (e != cudaSuccess) return cuda_fail(e, "zero y_acc");
        q.n = 1;
    }
    if ((st = run_experts(q, a, d, xc.dispatch)) != MOE_OK) return st;
    g_launches = q.n;
    return MOE_OK;
}

moe_status moe_forward(const void* x, const float* logits, const float* w_router,
                       const float* expert_bias, const moe_dims* d, float eps, float router_scale,
                       float out_scale, const moe_experts_w* W, int32_t* topk_idx, float* topk_w,
                       const moe_plan_t* plan, void* y, void* ws, size_t ws_bytes,
                       moe_stream_t stream) {
    return moe_forward_ex(x, logits, w_router, expert_bias, d, eps, router_scale, out_scale, nullptr, nullptr,
                          nullptr, W, topk_idx, topk_w, plan, y, ws, ws_bytes, stream);
}

moe_status moe_forward_ex(const void* x, const float* logits, const float* w_router,
                          const float* expert_bias, const moe_dims* d, float eps, float router_scale,
                          float out_scale, const moe_router_cfg* cfg, const moe_exec_cfg* exec,
                          const float* y_shared, const moe_experts_w* W, int32_t* topk_idx, float* topk_w,
                          const moe_plan_t* plan, void* y, void* ws, size_t ws_bytes, moe_stream_t stream) {
    moe_status st = check_dims(d);
    if (st != MOE_OK) return st;
    Exec xc;
    if ((st = resolve_exec(exec, &xc)) != MOE_OK) return st;
    if (y_shared && !aligned16(y_shared)) return fail(MOE_ERR_ALIGN, "y_shared not 16-byte aligned");
    RouteArgs r0{};
    if ((st = check_router_cfg(cfg, &r0)) != MOE_OK) return st;
    if (d->T == 0) return g_launches = 0, MOE_OK;   // empty batch: nothing to do
    if (!x || !y) return fail(MOE_ERR_NULL, "x or y is NULL (both are needed by the experts)");
    if (!aligned16(x) || !aligned16(y)) return fail(MOE_ERR_ALIGN, "x or y not 16-byte aligned");
    if (!logits && !w_router) return fail(MOE_ERR_NULL, "w_router is NULL (routing from x)");
    if (!topk_idx || !topk_w) return fail(MOE_ERR_NULL, "topk_idx or topk_w is NULL");
    if (!logits && !aligned16(w_router)) return fail(MOE_ERR_ALIGN, "w_router not 16-byte aligned");
    if ((st = check_plan(plan)) != MOE_OK) return st;
    if ((st = check_weights(W)) != MOE_OK) return st;
    WsView v;
    if ((st = check_ws(d, ws, ws_bytes, xc.ordered, &v)) != MOE_OK) return st;

    RouteArgs r{};
    r.x = logits ? nullptr : static_cast<const uint16_t*>(x);
    r.logits = logits;
    r.w_router = w_router;
    r.bias = expert_bias;
    r.l_scratch = v.l_scratch;
    r.part = v.part;
    r.T = d->T;
    r.H = d->H;
    r.E = d->E;
    r.k = d->k;
    r.eps = eps;
    r.scale = router_scale;
    r.softmax = r0.softmax;
    r.no_norm = r0.no_norm;
    r.idx = topk_idx;
    r.w = topk_w;
    r.counts = plan->counts;
    r.offsets = plan->offsets;
    r.perm = plan->perm;
    r.inv = plan->inv;
    r.tiles = plan->tiles;
    r.zero_ptr = v.ordered ? nullptr : v.y_acc;   // the router also clears the accumulator
    r.zero_count = (size_t)d->T * d->H;
    r.err = device_info().err_word;
    const bool fuse = d->T <= kSmallT;  // one CTA routes and plans all pairs
    Seq q{reinterpret_cast<cudaStream_t>(stream)};
    cudaError_t e = q.stage(MOE_STAGE_ROUTE, [&](int* n) { return launch_route(r, fuse, true, q.s, n); });
    if (e != cudaSuccess) return cuda_fail(e, "route");
    if (!fuse) {
        const PlanArgs p = make_plan_args(topk_idx, d, plan, v.plan_scratch);
        e = q.stage(MOE_STAGE_PLAN, [&](int* n) { return launch_plan(p, true, q.s, n); });
        if (e != cudaSuccess) return cuda_fail(e, "plan");
    }
    ExpertArgs a = make_expert_args(x, plan, topk_w, d, W, out_scale, y, v);
    a.y_shared = y_shared;
    if ((st = run_experts(q, a, d, xc.dispatch)) != MOE_OK) return st;
    g_launches = q.n;
    return MOE_OK;
}

moe_status moe_shared_expert(const void* x, const moe_experts_w* Ws, const moe_dims* d, float* y_shared,
                             void* ws, size_t ws_bytes, moe_stream_t stream) {
    return moe_shared_expert_ex(x, Ws, d, nullptr, y_shared, ws, ws_bytes, stream);
}

moe_status moe_shared_expert_ex(const void* x, const moe_experts_w* Ws, const moe_dims* d, const moe_exec_cfg* exec,
                                float* y_shared, void* ws, size_t ws_bytes, moe_stream_t stream) {
    moe_status st = check_dims(d);
    if (st != MOE_OK) return st;
    Exec xc;
    if ((st = resolve_exec(exec, &xc)) != MOE_OK) return st;
    if (d->E != 1 || d->k != 1) return fail(MOE_ERR_SHAPE, "the shared expert needs E == 1 and k == 1");
    if (d->T == 0) return g_launches = 0, MOE_OK;   // empty batch: nothing to do
    if (!x || !y_shared) return fail(MOE_ERR_NULL, "x or y_shared is NULL");
    if (!aligned16(x) || !aligned16(y_shared)) return fail(MOE_ERR_ALIGN, "x or y_shared not 16-byte aligned");
    if ((st = check_weights(Ws)) != MOE_OK) return st;
    WsView v;
    if ((st = check_ws(d, ws, ws_bytes, xc.ordered, &v)) != MOE_OK) return st;
    // the identity plan and the weights of 1 live in the scratch region (at
    // E = 1 it holds >= 4224 + 32 T bytes, more than the 3 align256(4 T) + 48
    // used here); x is already in plan order, so nothing is gathered
    const size_t T = d->T;
    char* b = reinterpret_cast<char*>(v.l_scratch);
    float* ones = reinterpret_cast<float*>(b);
    int32_t* perm = reinterpret_cast<int32_t*>(b + align256(T * 4));
    int32_t* inv = reinterpret_cast<int32_t*>(b + 2 * align256(T * 4));
    int32_t* misc = reinterpret_cast<int32_t*>(b + 3 * align256(T * 4));   // counts[1] | offsets[2] | tiles[2]
    moe_plan_t plan{misc, misc + 4, perm, inv, misc + 8};
    Seq q{reinterpret_cast<cudaStream_t>(stream)};
    cudaError_t e = launch_shared_prep(d->T, ones, plan.counts, plan.offsets, perm, inv, plan.tiles, true, q.s);
    if (e != cudaSuccess) return cuda_fail(e, "shared-expert plan");
    q.n = 1;
    ExpertArgs a = make_expert_args(x, &plan, ones, d, Ws, 1.0f, nullptr, v);
    a.xs = static_cast<uint16_t*>(const_cast<void*>(x));
    a.y_acc = y_shared;
    if (!a.ordered) {
        if ((e = launch_zero(y_shared, T * d->H, true, q.s)) != cudaSuccess) return cuda_fail(e, "zero y_shared");
        ++q.n;
    }
    const bool gemv = use_gemv(d, a.fmt, xc.dispatch);
    e = q.stage(MOE_STAGE_UP, [&](int*) { return gemv ? launch_gemv_up(a, true, q.s) : launch_gemm_up(a, true, q.s); });
    if (e == cudaErrorNotSupported) return fail(MOE_ERR_UNSUPPORTED, "no expert kernel for this format/path");
    if (e != cudaSuccess) return cuda_fail(e, "shared expert up kernel");
    e = q.stage(MOE_STAGE_DOWN, [&](int*) { return gemv ? launch_gemv_down(a, true, q.s) : launch_gemm_down(a, true, q.s); });
    if (e != cudaSuccess) return cuda_fail(e, "shared expert down kernel");
    g_launches = q.n;
    return MOE_OK;
}

moe_status moe_forward_host(const void* x_host, void* x_dev, const float* w_router,
                            const float* expert_bias, const moe_dims* d, float eps,
                            float router_scale, float out_scale, const moe_experts_w* W,
                            int32_t* topk_idx, float* topk_w, const moe_plan_t* plan, void* y_dev,
                            void* y_host, void* ws, size_t ws_bytes, moe_stream_t stream) {
    moe_status st = check_dims(d);
    if (st != MOE_OK) return st;
    if (d->T == 0) return MOE_OK;   // empty batch: nothing to do
    if (!x_host || !y_host || !x_dev) return fail(MOE_ERR_NULL, "x_host, x_dev or y_host is NULL");
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    const size_t bytes = (size_t)d->T * d->H * 2;
    cudaError_t e = cudaMemcpyAsync(x_dev, x_host, bytes, cudaMemcpyHostToDevice, s);
    if (e != cudaSuccess) return cuda_fail(e, "copy x to device");
    st = moe_forward(x_dev, nullptr, w_router, expert_bias, d, eps, router_scale, out_scale, W,
                     topk_idx, topk_w, plan, y_dev, ws, ws_bytes, stream);
    if (st != MOE_OK) return st;
    e = cudaMemcpyAsync(y_host, y_dev, bytes, cudaMemcpyDeviceToHost, s);
    if (e != cudaSuccess) return cuda_fail(e, "copy y to host");
    e = cudaStreamSynchronize(s);
    if (e != cudaSuccess) return cuda_fail(e, "stream synchronize");
    return MOE_OK;
}

int32_t moe_set_combine(int32_t mode) {
    std::lock_guard<std::mutex> lock(g_dispatch_mu);
    const int old = g_combine;
    if (mode == MOE_COMBINE_ATOMIC || mode == MOE_COMBINE_ORDERED) g_combine = mode;
    return old;
}

int32_t moe_set_dispatch(int32_t mode) {
    std::lock_guard<std::mutex> lock(g_dispatch_mu);
    const int old = g_dispatch;
    if (mode == MOE_DISPATCH_AUTO || mode == MOE_DISPATCH_GEMV || mode == MOE_DISPATCH_GEMM)
        g_dispatch = mode;
    return old;
}

moe_status moe_device_error(int32_t* code, moe_stream_t stream) {
    if (!code) return fail(MOE_ERR_NULL, "code is NULL");
    cudaError_t e = cudaStreamSynchronize(reinterpret_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return cuda_fail(e, "stream synchronize");
    int v = 0;
    e = cudaMemcpyFromSymbol(&v, moe::g_err_word, sizeof(int));
    if (e != cudaSuccess) return cuda_fail(e, "read device error word");
    const int zero = 0;
    e = cudaMemcpyToSymbol(moe::g_err_word, &zero, sizeof(int));
    if (e != cudaSuccess) return cuda_fail(e, "clear device error word");
    *code = v;
    if (v != 0) return fail(MOE_ERR_DEVICE, "device error code %d", v);
    return MOE_OK;
}

moe_status moe_profile_hook(void* ev_begin, void* ev_end, int32_t stage) {
    if (!ev_begin || !ev_end) {
        g_hook = Hook{};
        return MOE_OK;
    }
    if (stage < MOE_STAGE_ROUTE || stage > MOE_STAGE_GATHER) return fail(MOE_ERR_UNSUPPORTED, "stage %d", stage);
    g_hook.begin = static_cast<cudaEvent_t>(ev_begin);
    g_hook.end = static_cast<cudaEvent_t>(ev_end);
    g_hook.stage = stage;
    return MOE_OK;
}

int32_t moe_last_launch_count(void) { return g_launches; }

const char* moe_last_error(void) { return g_last_error.c_str(); }

const char* moe_version(void) { return "moe-b200 0.1 (sm_100a)"; }

}  // extern "C"
