// The grouped expert plan (TensorFold issue #548, "Zig CUDA ports: shared
// layers below lanes.Backend ...": the routing plan shared by the grouped
// expert kernels): histogram of the picks, two exclusive scans (pair offsets
// and M-tile offsets), then a stable scatter that keeps pairs of one expert in
// increasing pair order, so the plan is deterministic and equal to sorting
// pairs by (expert, pair id).  Small P: one CTA of 1024 threads.  Large P
// (with scratch): per-CTA histograms, one scan CTA, per-CTA scatters.
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

// ---- multi-CTA plan: the same result, in three short passes ----------------
// pass 1: each CTA's histogram of its kCtaPairs pairs -> hist[b][e]
constexpr int kCtaPairs = 1024;
constexpr int kScatterWarps = 16;

__global__ void __launch_bounds__(512) k_plan_hist(PlanArgs a) {
    __shared__ int s_cnt[256];
    pdl_wait();
    const int b = blockIdx.x, E = a.E;
    for (int i = threadIdx.x; i < E; i += blockDim.x) s_cnt[i] = 0;
    __syncthreads();
    const int p0 = b * kCtaPairs, p1 = min(a.P, p0 + kCtaPairs);
    for (int p = p0 + threadIdx.x; p < p1; p += blockDim.x) {
        const int e = a.idx[p];
        if (e >= 0 && e < E) atomicAdd(&s_cnt[e], 1);
        else report_error(a.err, kErrBadExpert);
    }
    __syncthreads();
    for (int i = threadIdx.x; i < E; i += blockDim.x) a.scratch[(size_t)b * E + i] = s_cnt[i];
    pdl_trigger();
}

// pass 2 (one CTA): counts, offsets, tiles, and base[b][e] = the first plan
// position of CTA b's pairs of expert e
__global__ void __launch_bounds__(256) k_plan_scan(PlanArgs a, int nb) {
    __shared__ int s_cnt[256], s_off[257], s_til[257];
    pdl_wait();
    const int E = a.E;
    const int32_t* hist = a.scratch;
    int32_t* base = a.scratch + (size_t)nb * E;
    for (int e = threadIdx.x; e < E; e += blockDim.x) {
        int c = 0;
        for (int b = 0; b < nb; ++b) c += hist[(size_t)b * E + e];
        s_cnt[e] = c;
    }
    __syncthreads();
    const int warp = threadIdx.x >> 5;
    if (warp == 0) warp_exclusive_scan(s_cnt, s_off, E, 0);
    if (warp == 1) warp_exclusive_scan(s_cnt, s_til, E, kTileM);
    __syncthreads();
    for (int e = threadIdx.x; e <= E; e += blockDim.x) {
        a.offsets[e] = s_off[e];
        a.tiles[e] = s_til[e];
        if (e < E) {
            a.counts[e] = s_cnt[e];
            int run = s_off[e];
            for (int b = 0; b < nb; ++b) {
                base[(size_t)b * E + e] = run;
                run += hist[(size_t)b * E + e];
            }
        }
    }
    pdl_trigger();
}

// pass 3: each CTA scatters its pairs stably from its bases
__global__ void __launch_bounds__(kScatterWarps * 32) k_plan_scatter(PlanArgs a, int nb) {
    __shared__ int s_idx[kCtaPairs], s_cur[256], s_wcnt[kScatterWarps * 256];
    pdl_wait();
    const int b = blockIdx.x, E = a.E;
    const int p0 = b * kCtaPairs, n = min(kCtaPairs, a.P - p0);
    const int32_t* base = a.scratch + (size_t)nb * E;
    for (int i = threadIdx.x; i < n; i += blockDim.x) s_idx[i] = a.idx[p0 + i];
    for (int i = threadIdx.x; i < kScatterWarps * E; i += blockDim.x) s_wcnt[i] = 0;
    for (int e = threadIdx.x; e < E; e += blockDim.x) s_cur[e] = base[(size_t)b * E + e];
    __syncthreads();
    stable_scatter<kScatterWarps>(s_idx, n, E, s_cur, s_wcnt, a.perm, a.inv, p0);
    pdl_trigger();
}

}  // namespace

size_t plan_scratch_ints(int P, int E) {
    const size_t nb = ((size_t)P + kCtaPairs - 1) / kCtaPairs;
    return 2 * nb * (size_t)E;
}

cudaError_t launch_plan(const PlanArgs& a, bool pdl, cudaStream_t s, int* n_launched) {
    *n_launched = 1;
    if (a.scratch && a.P > 4 * kCtaPairs) {
        const int nb = (a.P + kCtaPairs - 1) / kCtaPairs;
        cudaError_t e = launch_k(k_plan_hist, dim3(nb), dim3(512), 0, s, pdl, a);
        if (e != cudaSuccess) return e;
        if ((e = launch_k(k_plan_scan, dim3(1), dim3(256), 0, s, pdl, a, nb)) != cudaSuccess) return e;
        *n_launched = 3;
        return launch_k(k_plan_scatter, dim3(nb), dim3(kScatterWarps * 32), 0, s, pdl, a, nb);
    }
    const size_t smem = (size_t)(a.P < kPlanChunk ? (a.P > 0 ? a.P : 1) : kPlanChunk) * sizeof(int);
    cudaError_t e = ensure_smem(k_plan, smem);
    if (e != cudaSuccess) return e;
    return launch_k(k_plan, dim3(1), dim3(kPlanWarps * 32), smem, s, pdl, a);
}

}  // namespace moe
