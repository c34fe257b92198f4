// Host-side interfaces between the C-ABI layer (moe_api.cu) and the kernel
// files.  Plain structs of device pointers and sizes; nothing here allocates.
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "../../include/moe.h"

namespace moe {

struct RouteArgs {
    const uint16_t* x;       // (T, H) bf16, or null when logits are given
    const float* logits;     // (T, E) fp32, or null
    const float* w_router;   // (E, H) fp32
    const float* bias;       // (E) fp32 or null
    float* l_scratch;        // (T, E) fp32 scratch for the small-T logits pass
    float* part;             // (8, T, E) fp32 per-segment partial logits, or null
    int T, H, E, k;
    float eps, scale;
    int softmax;             // 1: softmax scores over the E logits; 0: sigmoid
    int no_norm;             // 1: w = s * scale (no division by the picked sum)
    int32_t* idx;            // (T, k)
    float* w;                // (T, k)
    // optional fused plan (single-CTA select path only)
    int32_t *counts, *offsets, *perm, *inv, *tiles;
    // optional zeroing of the fp32 accumulator (forward path)
    float* zero_ptr;
    size_t zero_count;       // floats
    int* err;
};

struct PlanArgs {
    const int32_t* idx;
    int P, E, k;
    int32_t *counts, *offsets, *perm, *inv, *tiles;
    int32_t* scratch;        // plan_scratch_ints(P, E) ints for the multi-CTA plan, or null
    int* err;
};

struct ExpertArgs {
    const uint16_t* x;       // (T, H) bf16
    const float* topk_w;     // (T, k)
    const int32_t* counts;
    const int32_t* offsets;
    const int32_t* perm;
    const int32_t* inv;      // pair t * k + j -> plan slot (ordered combine)
    const int32_t* tiles;
    int T, H, E, k, I;       // E: plan experts
    int E_w;                 // experts the weight tensors hold (E, or E - 1 when the last is skipped)
    int skip;                // plan expert whose pairs are computed nowhere and left out, or -1
    int act;                 // 0 swiglu, 1 relu2
    int fmt;                 // 0 bf16, 1 affine4, 2 nvfp4
    float swiglu_limit;      // > 0: g = min(g, L), u = clamp(u, -L, L) before silu(g) * u
    const void* w1;
    const uint16_t* w1_scale;
    const uint16_t* w1_bias;
    const void* w2;
    const uint16_t* w2_scale;
    const uint16_t* w2_bias;
    const float* w1_global;  // NVFP4: (E) fp32 global scales of W1 and W2
    const float* w2_global;
    uint16_t* h;             // (P, I) bf16 in plan order
    uint16_t* xs;            // (P, H) bf16 gathered rows (GEMM path)
    float* y_acc;            // (T, H) fp32, or (P, H) weighted slot outputs when ordered
    int ordered;             // 1: down stores w * o per plan slot; finalize sums slots in order
    uint16_t* y;             // (T, H) bf16
    const float* y_shared;   // (T, H) fp32 shared-expert output added after the routed scale, or null
    float out_scale;
    int* err;
};

struct DeviceInfo {
    int sm_count;
    int max_smem_optin;      // dynamic shared memory one CTA may opt into
    int smem_per_sm;         // shared memory of one SM (all resident CTAs together)
    int* err_word;           // device address of this device's error word
};

const DeviceInfo& device_info();   // of the current device (cached)

// Launchers: return the first CUDA error, cudaSuccess otherwise.
// launch_route sets *n_launched to the number of kernels it enqueued.
cudaError_t launch_route(const RouteArgs& a, bool fuse_plan, bool pdl, cudaStream_t s, int* n_launched);
// launch_plan sets *n_launched to the number of kernels it enqueued (1 or 3).
cudaError_t launch_plan(const PlanArgs& a, bool pdl, cudaStream_t s, int* n_launched);
size_t plan_scratch_ints(int P, int E);
cudaError_t launch_gemv_up(const ExpertArgs& a, bool pdl, cudaStream_t s);
cudaError_t launch_gemv_down(const ExpertArgs& a, bool pdl, cudaStream_t s);
// 4-bit GEMV (affine or NVFP4 codes dequantised in registers, K <= 8192);
// launch_gemv_up/down route fmt 1 and 2 here.
cudaError_t launch_gemv_q4_up(const ExpertArgs& a, bool pdl, cudaStream_t s);
cudaError_t launch_gemv_q4_down(const ExpertArgs& a, bool pdl, cudaStream_t s);
// The TMA-fed 4-bit GEMV (gemv_q4t.cu), which launch_gemv_q4_up/down use
// when gemv_q4t_fits: whole 128-row units and stage-aligned scale rows; the
// register GEMV takes the other shapes.
bool gemv_q4t_fits(const ExpertArgs& a, bool down);
cudaError_t launch_gemv_q4t_up(const ExpertArgs& a, bool pdl, cudaStream_t s);
cudaError_t launch_gemv_q4t_down(const ExpertArgs& a, bool pdl, cudaStream_t s);
// MOE_DISPATCH_AUTO's choice: the GEMV for 4-bit experts with at most this
// many routed pairs per expert on average, the tcgen05 GEMM otherwise.
constexpr int kAffineGemvMaxPairsPerExpert = 8;
// Whether the tcgen05 GEMM runs NVFP4 experts in this build.
constexpr bool kNvfp4Gemm = true;
// The tcgen05 grouped GEMMs (cudaErrorNotSupported where a format has none).
cudaError_t launch_gemm_up(const ExpertArgs& a, bool pdl, cudaStream_t s);
cudaError_t launch_gemm_down(const ExpertArgs& a, bool pdl, cudaStream_t s);
// The up GEMM takes its token rows by TMA from xs, the rows of x in plan
// order, filled by launch_gather_x before it -- except when
// gemm_up_reads_x(a) (bf16 experts, T <= 16), where it reads x itself.
cudaError_t launch_gather_x(const ExpertArgs& a, bool pdl, cudaStream_t s);
bool gemm_up_reads_x(const ExpertArgs& a);
cudaError_t launch_finalize(const ExpertArgs& a, bool pdl, cudaStream_t s);
// The one-expert identity plan of the shared expert: counts = {T},
// offsets = {0, T}, perm = inv = 0..T-1, tiles = {0, ceil(T / 128)}, and
// routing weights of 1.
cudaError_t launch_shared_prep(int T, float* ones, int32_t* counts, int32_t* offsets, int32_t* perm,
                               int32_t* inv, int32_t* tiles, bool pdl, cudaStream_t s);
cudaError_t launch_zero(float* p, size_t n, bool pdl, cudaStream_t s);

// Largest T for which the route kernels run the fused single-CTA select+plan.
constexpr int kSmallT = 32;

// Thread-local status text and launch count of the C-ABI layer (moe_api.cu).
void set_last_error(const char* msg);
void set_last_launch_count(int n);
// The C-ABI layer's argument checks, shared by every entry point: on failure
// they set the thread's status text and return the status.
moe_status validate_dims(const moe_dims* d);          // sizes within moe_dims' limits
moe_status validate_plan(const moe_plan_t* plan);     // plan struct and its arrays non-NULL
moe_status validate_weights(const moe_experts_w* W);  // pointers, alignment, enums, swiglu_limit

}  // namespace moe
