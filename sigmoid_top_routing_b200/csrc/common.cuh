// Device helpers shared by the routed-MoE kernels (sm_100a).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#define MOE_DEV __device__ __forceinline__

namespace moe {

constexpr int kWarp = 32;
constexpr int kTileM = 128;   // rows of a grouped-GEMM M-tile (MOE_TILE_M)

// Device error codes (written to the library's error word, never trapped).
constexpr int kErrBadExpert = 1;
constexpr int kErrWaitExpired = 2;

MOE_DEV void report_error(int* err, int code) {
    if (err) atomicCAS(err, 0, code);
}

// ---- programmatic dependent launch -----------------------------------------
// Wait until the preceding kernel in the stream has completed and its writes
// are visible (no-op when the launch had no programmatic dependency).
MOE_DEV void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
// Let the next kernel in the stream start launching its CTAs.
MOE_DEV void pdl_trigger() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

// ---- bf16 ------------------------------------------------------------------
MOE_DEV float bf16lo(uint32_t v) { return __uint_as_float(v << 16); }
MOE_DEV float bf16hi(uint32_t v) { return __uint_as_float(v & 0xFFFF0000u); }
MOE_DEV float bf16f(uint16_t v) { return __uint_as_float(uint32_t(v) << 16); }
MOE_DEV uint16_t f2bf16(float f) {
    __nv_bfloat16 b = __float2bfloat16_rn(f);
    return *reinterpret_cast<uint16_t*>(&b);
}
MOE_DEV uint32_t pack_bf16x2(float lo, float hi) {
    return uint32_t(f2bf16(lo)) | (uint32_t(f2bf16(hi)) << 16);
}

// ---- loads -----------------------------------------------------------------
// Streaming 16-byte load for weights read once: no L1 allocation, L2 evict-first.
MOE_DEV uint4 ld_stream(const void* p, uint64_t policy) {
    uint4 v;
    asm volatile(
        "ld.global.nc.L1::no_allocate.L2::cache_hint.v4.u32 {%0,%1,%2,%3}, [%4], %5;"
        : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
        : "l"(p), "l"(policy));
    return v;
}
MOE_DEV uint64_t policy_evict_first() {
    uint64_t p;
    asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(p));
    return p;
}
MOE_DEV uint64_t policy_evict_last() {
    uint64_t p;
    asm volatile("createpolicy.fractional.L2::evict_last.b64 %0, 1.0;" : "=l"(p));
    return p;
}
// 16-byte store with an L2 eviction policy (a buffer the next kernel re-reads)
MOE_DEV void st_hint(void* p, uint4 v, uint64_t policy) {
    asm volatile("st.global.L2::cache_hint.v4.u32 [%0], {%1,%2,%3,%4}, %5;" ::"l"(p), "r"(v.x), "r"(v.y), "r"(v.z),
                 "r"(v.w), "l"(policy)
                 : "memory");
}
// Read-only 16-byte load that may stay in L1 (activations reused across rows).
MOE_DEV uint4 ld_nc(const void* p) { return __ldg(reinterpret_cast<const uint4*>(p)); }

// dot of 8 bf16 weights with 8 bf16 activations, accumulated in fp32
MOE_DEV float dot8(uint4 w, uint4 x, float acc) {
    acc = fmaf(bf16lo(w.x), bf16lo(x.x), acc);
    acc = fmaf(bf16hi(w.x), bf16hi(x.x), acc);
    acc = fmaf(bf16lo(w.y), bf16lo(x.y), acc);
    acc = fmaf(bf16hi(w.y), bf16hi(x.y), acc);
    acc = fmaf(bf16lo(w.z), bf16lo(x.z), acc);
    acc = fmaf(bf16hi(w.z), bf16hi(x.z), acc);
    acc = fmaf(bf16lo(w.w), bf16lo(x.w), acc);
    acc = fmaf(bf16hi(w.w), bf16hi(x.w), acc);
    return acc;
}

MOE_DEV float warp_sum(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

// SwiGLU and relu^2 activations in fp32.
// silu(g) * u with the logistic computed as 1 / (1 + exp(-g)).
MOE_DEV float act_swiglu(float g, float u) { return g / (1.0f + expf(-g)) * u; }

// The SwiGLU input clamp (limit > 0): gate from above, up on both sides;
// comparisons keep NaN (NaN > L is false).
MOE_DEV void clamp_swiglu(float& g, float& u, float limit) {
    if (limit > 0.0f) {
        g = g > limit ? limit : g;
        u = u > limit ? limit : (u < -limit ? -limit : u);
    }
}
// relu(u)^2 that keeps NaN: a NaN input is squared (stays NaN), never clamped.
MOE_DEV float act_relu2(float u) {
    float r = (u > 0.0f || u != u) ? u : 0.0f;
    return r * r;
}

}  // namespace moe
