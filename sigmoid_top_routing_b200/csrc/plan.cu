// The grouped expert plan (TensorFold issue #548, "Zig CUDA ports: shared
// layers below lanes.Backend ...": the routing plan shared by the grouped
// expert kernels).  One CTA of 1024 threads: histogram of the picks, two
// exclusive scans (pair offsets and M-tile offsets), then a stable scatter
// that keeps pairs of one expert in increasing pair order, so the plan is
// deterministic and equal to sorting pairs by (expert, pair id).
#include "common.cuh"
#include "internal.h"
#include "launch.h"
#include "plan_dev.cuh"

namespace moe {
namespace {

constexpr int kPlanWarps = 32;
constexpr int kPlanChunk = 32768;   // pair ids staged in shared memory at a time

__global__ void __launch_bounds__(kPlanWarps * 32) k_plan(PlanArgs a) {
    extern __shared__ int s_idx[];   // up to kPlanChunk ids
    __shared__ int s_cnt[256], s_off[257], s_til[257], s_cur[256];
    __shared__ int s_wcnt[kPlanWarps * 256];
    pdl_wait();
    const int tid = threadIdx.x, nthr = blockDim.x;
    const int P = a.P, E = a.E;
    for (int i = tid; i < 256; i += nthr) s_cnt[i] = 0;
    for (int i = tid; i < kPlanWarps * 256; i += nthr) s_wcnt[i] = 0;
    __syncthreads();
    for (int p = tid; p < P; p += nthr) {
        const int e = a.idx[p];
        if (e >= 0 && e < E) atomicAdd(&s_cnt[e], 1);
        else report_error(a.err, kErrBadExpert);
    }
    __syncthreads();
    const int warp = tid >> 5;
    if (warp == 0) warp_exclusive_scan(s_cnt, s_off, E, 0);
    if (warp == 1) warp_exclusive_scan(s_cnt, s_til, E, kTileM);
    __syncthreads();
    for (int e = tid; e <= E; e += nthr) {
        a.offsets[e] = s_off[e];
        a.tiles[e] = s_til[e];
        if (e < E) {
            a.counts[e] = s_cnt[e];
            s_cur[e] = s_off[e];
        }
    }
    __syncthreads();
    for (int base = 0; base < P; base += kPlanChunk) {
        const int n = min(kPlanChunk, P - base);
        for (int i = tid; i < n; i += nthr) s_idx[i] = a.idx[base + i];
        __syncthreads();
        stable_scatter<kPlanWarps>(s_idx, n, E, s_cur, s_wcnt, a.perm, a.inv, base);
    }
    pdl_trigger();
}

}  // namespace

cudaError_t launch_plan(const PlanArgs& a, bool pdl, cudaStream_t s) {
    const size_t smem = (size_t)(a.P < kPlanChunk ? (a.P > 0 ? a.P : 1) : kPlanChunk) * sizeof(int);
    cudaError_t e = ensure_smem(k_plan, smem);
    if (e != cudaSuccess) return e;
    return launch_k(k_plan, dim3(1), dim3(kPlanWarps * 32), smem, s, pdl, a);
}

}  // namespace moe
