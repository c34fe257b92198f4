// Decode-sized grouped expert GEMV (bf16 weights).
//
// Prior art: TensorFold issue #548, "Prompt rows of the grouped experts: two
// forms" -- the decode form works on small items of pairs and streams each
// expert's weights; TileGym PR #187 notes that at one token the stock path
// only touches the picked experts.  Here every active expert's weight rows
// are streamed once from HBM with 16-byte non-allocating loads (L2
// evict-first), a warp per output row, and reused from registers for all of
// the expert's tokens (read through L1).
//
//   up:   h[pos, i] = bf16_rn(act(W1[e] rows . x[t]))   SwiGLU: rows i and I+i
//                                                       (gate first), relu^2: row i
//   down: y_acc[t, n] += w[p] * (W2[e][n] . h[pos])      (fp32 atomics)
//
// Work is spread as units of (active expert, 8 rows) over a persistent grid;
// each CTA takes a contiguous range of units, so most CTAs see one expert.
#include <algorithm>

#include "common.cuh"
#include "internal.h"
#include "launch.h"

namespace moe {
namespace {

constexpr int kWarps = 8;
constexpr int kTokGroup = 8;          // tokens whose partial sums a warp keeps at once
constexpr int kChunksPerLane = 8;     // 16-byte chunks of a row a lane holds per pass

// Active experts (count > 0, not the skipped one) compacted in id order into
// s_act; returns how many.
MOE_DEV int build_active(const int32_t* counts, int E, int skip, int* s_act, int* s_n) {
    if (threadIdx.x < 32) {
        const int lane = threadIdx.x;
        int base = 0;
        for (int e0 = 0; e0 < E; e0 += 32) {
            const int e = e0 + lane;
            const bool on = e < E && e != skip && counts[e] > 0;
            const unsigned m = __ballot_sync(0xffffffffu, on);
            if (on) s_act[base + __popc(m & ((1u << lane) - 1u))] = e;
            base += __popc(m);
        }
        if (lane == 0) *s_n = base;
    }
    __syncthreads();
    return *s_n;
}

// One warp: dot products of one or two weight rows (length K, bf16) with the
// rows of up to kTokGroup tokens.  Returns warp-reduced sums in every lane.
template <bool TWO>
MOE_DEV void rows_dot_tokens(const uint16_t* __restrict__ r0, const uint16_t* __restrict__ r1, int K,
                             const uint16_t* const* xrow, int mt, float* s0, float* s1,
                             uint64_t pol) {
    const int lane = threadIdx.x & 31;
    const int nc = K / 8;
    float a0[kTokGroup], a1[kTokGroup];
#pragma unroll
    for (int m = 0; m < kTokGroup; ++m) { a0[m] = 0.f; a1[m] = 0.f; }
    for (int seg = 0; seg < nc; seg += 32 * kChunksPerLane) {
        uint4 w0[kChunksPerLane], w1[kChunksPerLane];
#pragma unroll
        for (int j = 0; j < kChunksPerLane; ++j) {
            const int c = seg + lane + 32 * j;
            if (c < nc) {
                w0[j] = ld_stream(r0 + 8 * c, pol);
                if (TWO) w1[j] = ld_stream(r1 + 8 * c, pol);
            }
        }
#pragma unroll
        for (int m = 0; m < kTokGroup; ++m) {
            if (m < mt) {
                const uint16_t* xr = xrow[m];
#pragma unroll
                for (int j = 0; j < kChunksPerLane; ++j) {
                    const int c = seg + lane + 32 * j;
                    if (c < nc) {
                        const uint4 xv = ld_nc(xr + 8 * c);
                        a0[m] = dot8(w0[j], xv, a0[m]);
                        if (TWO) a1[m] = dot8(w1[j], xv, a1[m]);
                    }
                }
            }
        }
    }
#pragma unroll
    for (int m = 0; m < kTokGroup; ++m) {
        if (m < mt) {
            s0[m] = warp_sum(a0[m]);
            if (TWO) s1[m] = warp_sum(a1[m]);
        }
    }
}

template <int ACT>
__global__ void __launch_bounds__(kWarps * 32, 2) k_gemv_up(ExpertArgs a) {
    __shared__ int s_act[256];
    __shared__ int s_n;
    pdl_wait();
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int n_act = build_active(a.counts, a.E, a.skip, s_act, &s_n);
    const int I = a.I, H = a.H;
    const int n1 = ACT == 0 ? 2 * I : I;
    const int upe = (I + kWarps - 1) / kWarps;
    const long long total = (long long)n_act * upe;
    const long long u0 = total * blockIdx.x / gridDim.x;
    const long long u1 = total * (blockIdx.x + 1) / gridDim.x;
    const uint64_t pol = policy_evict_first();
    const uint16_t* W1 = reinterpret_cast<const uint16_t*>(a.w1);
    for (long long u = u0; u < u1; ++u) {
        const int e = s_act[u / upe];
        const int r = (int)(u % upe) * kWarps + warp;
        if (r >= I) continue;
        const int cnt = a.counts[e], off = a.offsets[e];
        const uint16_t* rg = W1 + ((size_t)e * n1 + r) * H;
        const uint16_t* ru = ACT == 0 ? W1 + ((size_t)e * n1 + I + r) * H : rg;
        for (int m0 = 0; m0 < cnt; m0 += kTokGroup) {
            const int mt = min(kTokGroup, cnt - m0);
            const uint16_t* xrow[kTokGroup];
#pragma unroll
            for (int m = 0; m < kTokGroup; ++m) {
                const int pm = m < mt ? a.perm[off + m0 + m] : 0;
                xrow[m] = a.x + (size_t)(pm / a.k) * H;
            }
            float sg[kTokGroup], su[kTokGroup];
            rows_dot_tokens<ACT == 0>(rg, ru, H, xrow, mt, sg, su, pol);
#pragma unroll
            for (int m = 0; m < kTokGroup; ++m) {
                if (m < mt && lane == m) {
                    float gv = sg[m], uv = su[m];
                    if (ACT == 0) clamp_swiglu(gv, uv, a.swiglu_limit);
                    const float v = ACT == 0 ? act_swiglu(gv, uv) : act_relu2(gv);
                    a.h[(size_t)(off + m0 + m) * I + r] = f2bf16(v);
                }
            }
        }
    }
    pdl_trigger();
}

__global__ void __launch_bounds__(kWarps * 32, 2) k_gemv_down(ExpertArgs a) {
    __shared__ int s_act[256];
    __shared__ int s_n;
    pdl_wait();
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int n_act = build_active(a.counts, a.E, a.skip, s_act, &s_n);
    const int I = a.I, H = a.H;
    const int upe = (H + kWarps - 1) / kWarps;
    const long long total = (long long)n_act * upe;
    const long long u0 = total * blockIdx.x / gridDim.x;
    const long long u1 = total * (blockIdx.x + 1) / gridDim.x;
    const uint64_t pol = policy_evict_first();
    const uint16_t* W2 = reinterpret_cast<const uint16_t*>(a.w2);
    for (long long u = u0; u < u1; ++u) {
        const int e = s_act[u / upe];
        const int n = (int)(u % upe) * kWarps + warp;
        if (n >= H) continue;
        const int cnt = a.counts[e], off = a.offsets[e];
        const uint16_t* rw = W2 + ((size_t)e * H + n) * I;
        for (int m0 = 0; m0 < cnt; m0 += kTokGroup) {
            const int mt = min(kTokGroup, cnt - m0);
            const uint16_t* hrow[kTokGroup];
            int pm[kTokGroup];
#pragma unroll
            for (int m = 0; m < kTokGroup; ++m) {
                pm[m] = m < mt ? a.perm[off + m0 + m] : 0;
                hrow[m] = a.h + (size_t)(off + m0 + (m < mt ? m : 0)) * I;
            }
            float so[kTokGroup], unused[kTokGroup];
            rows_dot_tokens<false>(rw, rw, I, hrow, mt, so, unused, pol);
#pragma unroll
            for (int m = 0; m < kTokGroup; ++m) {
                if (m < mt && lane == m) {
                    const float wv = a.topk_w[pm[m]];
                    if (a.ordered)
                        a.y_acc[(size_t)(off + m0 + m) * H + n] = wv * so[m];
                    else
                        atomicAdd(a.y_acc + (size_t)(pm[m] / a.k) * H + n, wv * so[m]);
                }
            }
        }
    }
    pdl_trigger();
}

// y = bf16_rn(out_scale * y_acc): one multiply on the finished sum
// (vllm.cpp PR #684, "The finding that justifies the row").
__global__ void __launch_bounds__(256) k_finalize(ExpertArgs a) {
    pdl_wait();
    const size_t n8 = (size_t)a.T * a.H / 8;
    const float4* src = reinterpret_cast<const float4*>(a.y_acc);
    uint4* dst = reinterpret_cast<uint4*>(a.y);
    const float sc = a.out_scale;
    for (size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x; i < n8; i += (size_t)gridDim.x * blockDim.x) {
        float4 v0 = src[2 * i], v1 = src[2 * i + 1];
        v0 = make_float4(__fmul_rn(sc, v0.x), __fmul_rn(sc, v0.y), __fmul_rn(sc, v0.z), __fmul_rn(sc, v0.w));
        v1 = make_float4(__fmul_rn(sc, v1.x), __fmul_rn(sc, v1.y), __fmul_rn(sc, v1.z), __fmul_rn(sc, v1.w));
        if (a.y_shared) {   // the shared expert's output, after the routed scale (vllm.cpp PR #684)
            const float4 s0 = reinterpret_cast<const float4*>(a.y_shared)[2 * i];
            const float4 s1 = reinterpret_cast<const float4*>(a.y_shared)[2 * i + 1];
            v0 = make_float4(v0.x + s0.x, v0.y + s0.y, v0.z + s0.z, v0.w + s0.w);
            v1 = make_float4(v1.x + s1.x, v1.y + s1.y, v1.z + s1.z, v1.w + s1.w);
        }
        uint4 o;
        o.x = pack_bf16x2(v0.x, v0.y);
        o.y = pack_bf16x2(v0.z, v0.w);
        o.z = pack_bf16x2(v1.x, v1.y);
        o.w = pack_bf16x2(v1.z, v1.w);
        dst[i] = o;
    }
    pdl_trigger();
}

// Ordered combine: y[t] = bf16_rn(out_scale * (sum over j = 0..k-1, in that
// order, of the slot row inv[t * k + j])); the rows already carry w_j.  Slots
// of the skipped plan expert (positions offsets[skip] .. offsets[skip + 1])
// hold nothing and are left out.
__global__ void __launch_bounds__(256) k_finalize_ordered(ExpertArgs a) {
    pdl_wait();
    const size_t n4 = (size_t)a.T * a.H / 4;
    const int h4 = a.H / 4;
    const float sc = a.out_scale;
    const int skip_lo = a.skip >= 0 ? a.offsets[a.skip] : 0;
    const int skip_hi = a.skip >= 0 ? a.offsets[a.skip + 1] : 0;
    for (size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x; i < n4; i += (size_t)gridDim.x * blockDim.x) {
        const int t = (int)(i / h4), c = (int)(i - (size_t)t * h4);
        float4 s = make_float4(0.f, 0.f, 0.f, 0.f);
        for (int j = 0; j < a.k; ++j) {
            const int slot = a.inv[(size_t)t * a.k + j];
            if (slot >= skip_lo && slot < skip_hi) continue;
            const float4 v = __ldcg(reinterpret_cast<const float4*>(a.y_acc + (size_t)slot * a.H) + c);
            s.x += v.x;
            s.y += v.y;
            s.z += v.z;
            s.w += v.w;
        }
        s = make_float4(__fmul_rn(sc, s.x), __fmul_rn(sc, s.y), __fmul_rn(sc, s.z), __fmul_rn(sc, s.w));
        if (a.y_shared) {
            const float4 sh = reinterpret_cast<const float4*>(a.y_shared)[i];
            s = make_float4(s.x + sh.x, s.y + sh.y, s.z + sh.z, s.w + sh.w);
        }
        uint2 o;
        o.x = pack_bf16x2(s.x, s.y);
        o.y = pack_bf16x2(s.z, s.w);
        reinterpret_cast<uint2*>(a.y)[i] = o;
    }
    pdl_trigger();
}

__global__ void __launch_bounds__(256) k_shared_prep(int T, float* ones, int32_t* counts, int32_t* offsets,
                                                     int32_t* perm, int32_t* inv, int32_t* tiles) {
    pdl_wait();
    for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < T; i += gridDim.x * blockDim.x) {
        ones[i] = 1.0f;
        perm[i] = i;
        inv[i] = i;
    }
    if (blockIdx.x == 0 && threadIdx.x == 0) {
        counts[0] = T;
        offsets[0] = 0;
        offsets[1] = T;
        tiles[0] = 0;
        tiles[1] = (T + kTileM - 1) / kTileM;
    }
    pdl_trigger();
}

__global__ void __launch_bounds__(256) k_zero(float* p, size_t n4) {
    pdl_wait();
    for (size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x; i < n4; i += (size_t)gridDim.x * blockDim.x)
        reinterpret_cast<float4*>(p)[i] = make_float4(0.f, 0.f, 0.f, 0.f);
    pdl_trigger();
}

}  // namespace

// Persistent grids: two CTAs of 8 warps per SM.
cudaError_t launch_gemv_up(const ExpertArgs& a, bool pdl, cudaStream_t s) {
    if (a.fmt == 1 || a.fmt == 2) return launch_gemv_q4_up(a, pdl, s);
    if (a.fmt != 0) return cudaErrorNotSupported;
    const int grid = device_info().sm_count * 2;
    if (a.act == 0) return launch_k(k_gemv_up<0>, dim3(grid), dim3(kWarps * 32), 0, s, pdl, a);
    return launch_k(k_gemv_up<1>, dim3(grid), dim3(kWarps * 32), 0, s, pdl, a);
}

cudaError_t launch_gemv_down(const ExpertArgs& a, bool pdl, cudaStream_t s) {
    if (a.fmt == 1 || a.fmt == 2) return launch_gemv_q4_down(a, pdl, s);
    if (a.fmt != 0) return cudaErrorNotSupported;
    const int grid = device_info().sm_count * 2;
    return launch_k(k_gemv_down, dim3(grid), dim3(kWarps * 32), 0, s, pdl, a);
}

cudaError_t launch_finalize(const ExpertArgs& a, bool pdl, cudaStream_t s) {
    const size_t n8 = (size_t)a.T * a.H / 8;
    if (n8 == 0) return cudaSuccess;
    const DeviceInfo& di = device_info();
    if (a.ordered) {
        const size_t n4 = n8 * 2;
        size_t blocks = (n4 + 255) / 256, cap = (size_t)di.sm_count * 8;
        return launch_k(k_finalize_ordered, dim3((unsigned)(blocks < cap ? blocks : cap)), dim3(256), 0, s, pdl, a);
    }
    size_t blocks = (n8 + 255) / 256;
    size_t cap = (size_t)di.sm_count * 8;
    return launch_k(k_finalize, dim3((unsigned)(blocks < cap ? blocks : cap)), dim3(256), 0, s, pdl, a);
}

cudaError_t launch_shared_prep(int T, float* ones, int32_t* counts, int32_t* offsets, int32_t* perm,
                               int32_t* inv, int32_t* tiles, bool pdl, cudaStream_t s) {
    const int blocks = std::max(1, std::min((T + 255) / 256, device_info().sm_count * 4));
    return launch_k(k_shared_prep, dim3(blocks), dim3(256), 0, s, pdl, T, ones, counts, offsets, perm, inv, tiles);
}

cudaError_t launch_zero(float* p, size_t n, bool pdl, cudaStream_t s) {
    const size_t n4 = n / 4;
    if (n4 == 0) return cudaSuccess;
    const DeviceInfo& di = device_info();
    size_t blocks = (n4 + 255) / 256;
    size_t cap = (size_t)di.sm_count * 8;
    return launch_k(k_zero, dim3((unsigned)(blocks < cap ? blocks : cap)), dim3(256), 0, s, pdl, p, n4);
}

}  // namespace moe
