// Block-level pieces of the grouped expert plan, shared by the fused
// select+plan kernel (small T) and the standalone plan kernel.
#pragma once

#include "common.cuh"

namespace moe {

// Exclusive scan of n <= 256 ints by one warp: out[0..n] (n + 1 entries).
// `tile_div` > 0 scans ceil(in / tile_div) instead of in.
MOE_DEV void warp_exclusive_scan(const int* in, int* out, int n, int tile_div) {
    const int lane = threadIdx.x & 31;
    const int per = (n + 31) / 32;
    int local = 0;
    for (int j = 0; j < per; ++j) {
        int i = lane * per + j;
        if (i < n) {
            int v = in[i];
            local += tile_div > 0 ? (v + tile_div - 1) / tile_div : v;
        }
    }
    int incl = local;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        int t = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += t;
    }
    int run = incl - local;
    for (int j = 0; j < per; ++j) {
        int i = lane * per + j;
        if (i < n) {
            out[i] = run;
            int v = in[i];
            run += tile_div > 0 ? (v + tile_div - 1) / tile_div : v;
        }
    }
    if (lane == 31) out[n] = incl;
}

// Stable scatter of pairs p_base + [0, P) with expert ids in s_idx (shared memory) to
// their plan positions: pairs of one expert keep increasing pair order.
// `cursor` (shared, E ints) holds each expert's first position on entry and
// is advanced; `wcnt` (shared, NW * E ints) must be zero on entry and is zero
// on exit.  Invalid ids (outside [0, E)) are skipped: inv = -1.
template <int NW>
MOE_DEV void stable_scatter(const int* s_idx, int P, int E, int* cursor, int* wcnt, int32_t* perm,
                            int32_t* inv, int p_base = 0) {
    const int tid = threadIdx.x;
    const int warp = tid >> 5, lane = tid & 31;
    const unsigned lt_mask = (1u << lane) - 1u;
    for (int base = 0; base < P; base += NW * 32) {
        const int p = base + tid;
        int e = p < P ? s_idx[p] : -1;
        const bool valid = e >= 0 && e < E;
        const int key = valid ? e : -1;
        const unsigned peers = __match_any_sync(0xffffffffu, key);
        const int rank = __popc(peers & lt_mask);
        if (valid && rank == 0) wcnt[warp * E + e] = __popc(peers);
        __syncthreads();
        if (valid) {
            int pre = 0;
            for (int w = 0; w < warp; ++w) pre += wcnt[w * E + e];
            const int pos = cursor[e] + pre + rank;
            perm[pos] = p_base + p;
            inv[p_base + p] = pos;
        } else if (p < P) {
            inv[p_base + p] = -1;
        }
        __syncthreads();
        for (int ee = tid; ee < E; ee += NW * 32) {
            int s = 0;
            for (int w = 0; w < NW; ++w) {
                s += wcnt[w * E + ee];
                wcnt[w * E + ee] = 0;
            }
            cursor[ee] += s;
        }
        __syncthreads();
    }
}

}  // namespace moe
