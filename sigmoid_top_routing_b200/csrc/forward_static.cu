// moe_forward_static: the block's forward pass for callers that cannot
// allocate device memory.
//
// Some callers have no way to hand the library a workspace: a plugin host
// that gives a custom op only its input and output tensors, or a
// latency-bound serving loop that must never wait on an allocator.  For them
// the scratch the forward needs (the fp32 accumulator, the bf16 activations
// and the router-logit scratch) lives in one fixed device array defined in
// this file.  The caller still passes the inputs, the weights, the plan arrays
// and the outputs; this entry point calls no cudaMalloc, cudaFree or any
// allocating library routine.
#include <cstdio>
#include <map>
#include <mutex>

#include "../../include/moe.h"
#include "internal.h"

namespace moe {
namespace {

// The fixed scratch: every GPU that loads the library holds it until exit.
constexpr size_t kStaticScratchBytes = size_t(16) << 20;   // 16 MiB
static __device__ __align__(256) unsigned char g_static_scratch[kStaticScratchBytes];

size_t align256(size_t v) { return (v + 255) & ~size_t(255); }

// Device address of g_static_scratch on the current device, looked up once
// per device (the symbol's name in host code is not a device address).
cudaError_t scratch_address(unsigned char** out) {
    static std::mutex mu;
    static std::map<int, unsigned char*> addr;
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    std::lock_guard<std::mutex> lock(mu);
    auto it = addr.find(dev);
    if (it != addr.end()) {
        *out = it->second;
        return cudaSuccess;
    }
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_static_scratch);
    if (e != cudaSuccess) return e;
    addr[dev] = static_cast<unsigned char*>(p);
    *out = static_cast<unsigned char*>(p);
    return cudaSuccess;
}

moe_status fail(moe_status st, const char* msg) {
    set_last_error(msg);
    return st;
}

moe_status cuda_fail(cudaError_t e, const char* what) {
    char buf[256];
    snprintf(buf, sizeof buf, "%s: %s (%s)", what, cudaGetErrorName(e), cudaGetErrorString(e));
    set_last_error(buf);
    return MOE_ERR_CUDA;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

}  // namespace
}  // namespace moe

using namespace moe;

extern "C" moe_status moe_forward_static(const void* x, const float* logits, const float* w_router,
                                         const float* expert_bias, const moe_dims* d, float eps,
                                         float router_scale, float out_scale, const moe_experts_w* W,
                                         int32_t* topk_idx, float* topk_w, const moe_plan_t* plan,
                                         void* y, moe_stream_t stream) {
    moe_status st = validate_dims(d);
    if (st != MOE_OK) return st;
    if (d->T == 0) {
        set_last_launch_count(0);
        return MOE_OK;
    }
    if (!x || !y || !topk_idx || !topk_w) return fail(MOE_ERR_NULL, "x, y, topk_idx or topk_w is NULL");
    if (!logits && !w_router) return fail(MOE_ERR_NULL, "w_router is NULL (routing from x)");
    if (!aligned16(x) || !aligned16(y) || (!logits && !aligned16(w_router)))
        return fail(MOE_ERR_ALIGN, "x, y or w_router not 16-byte aligned");
    if ((st = validate_plan(plan)) != MOE_OK) return st;
    if ((st = validate_weights(W)) != MOE_OK) return st;
    if (W->fmt != MOE_W_BF16) return fail(MOE_ERR_UNSUPPORTED, "moe_forward_static runs bf16 weights only");

    // scratch layout: y_acc fp32 (T, H) | h bf16 (P, I) | router-logit scratch
    const size_t T = d->T, H = d->H, I = d->I, E = d->E, P = T * d->k;
    const size_t off_h = align256(T * H * 4);
    const size_t off_l = align256(off_h + P * I * 2);
    const size_t need = align256(off_l + (size_t)kSmallT * E * 4 + 4096);
    if (need > kStaticScratchBytes) {
        char buf[200];
        snprintf(buf, sizeof buf,
                 "moe_forward_static needs %zu bytes of scratch for these sizes, more than its fixed "
                 "%zu; use moe_forward with a workspace",
                 need, kStaticScratchBytes);
        return fail(MOE_ERR_WORKSPACE, buf);
    }
    unsigned char* base = nullptr;
    cudaError_t e = scratch_address(&base);
    if (e != cudaSuccess) return cuda_fail(e, "cudaGetSymbolAddress(static scratch)");
    float* y_acc = reinterpret_cast<float*>(base);
    uint16_t* h = reinterpret_cast<uint16_t*>(base + off_h);
    float* l_scratch = reinterpret_cast<float*>(base + off_l);
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    int* err = device_info().err_word;

    RouteArgs r{};
    r.x = logits ? nullptr : static_cast<const uint16_t*>(x);
    r.logits = logits;
    r.w_router = w_router;
    r.bias = expert_bias;
    r.l_scratch = l_scratch;
    r.T = d->T;
    r.H = d->H;
    r.E = d->E;
    r.k = d->k;
    r.eps = eps;
    r.scale = router_scale;
    r.idx = topk_idx;
    r.w = topk_w;
    r.counts = plan->counts;
    r.offsets = plan->offsets;
    r.perm = plan->perm;
    r.inv = plan->inv;
    r.tiles = plan->tiles;
    r.zero_ptr = y_acc;             // the accumulator keeps the last call's sums: clear it
    r.zero_count = T * H;
    r.err = err;
    const bool fuse = d->T <= kSmallT;
    int n = 0, launched = 0;
    if ((e = launch_route(r, fuse, true, s, &n)) != cudaSuccess) return cuda_fail(e, "route");
    launched += n;
    if (!fuse) {
        PlanArgs p{};
        p.idx = topk_idx;
        p.P = (int)P;
        p.E = d->E;
        p.k = d->k;
        p.counts = plan->counts;
        p.offsets = plan->offsets;
        p.perm = plan->perm;
        p.inv = plan->inv;
        p.tiles = plan->tiles;
        p.err = err;
        int np = 0;   // no scratch given: the single-CTA plan
        if ((e = launch_plan(p, true, s, &np)) != cudaSuccess) return cuda_fail(e, "plan");
        launched += np;
    }
    ExpertArgs a{};
    a.x = static_cast<const uint16_t*>(x);
    a.topk_w = topk_w;
    a.counts = plan->counts;
    a.offsets = plan->offsets;
    a.perm = plan->perm;
    a.tiles = plan->tiles;
    a.T = d->T;
    a.H = d->H;
    a.E = d->E;
    a.E_w = d->E;
    a.skip = -1;              // every plan expert has weights and is computed
    a.k = d->k;
    a.I = d->I;
    a.act = W->act;
    a.fmt = W->fmt;
    a.swiglu_limit = W->swiglu_limit;
    a.w1 = W->w1;
    a.w2 = W->w2;
    a.h = h;
    a.xs = nullptr;
    a.y_acc = y_acc;
    a.y = static_cast<uint16_t*>(y);
    a.out_scale = out_scale;
    a.err = err;
    if ((e = launch_gemv_up(a, true, s)) != cudaSuccess) return cuda_fail(e, "expert up kernel");
    if ((e = launch_gemv_down(a, true, s)) != cudaSuccess) return cuda_fail(e, "expert down kernel");
    if ((e = launch_finalize(a, true, s)) != cudaSuccess) return cuda_fail(e, "finalize");
    set_last_launch_count(launched + 3);
    return MOE_OK;
}
