// Sigmoid router with a selection-only expert bias and normalised top-k.
//
// TileGym PR #187 ("[E2E Model Support] Add TileGym kernel integration for
// LFM2 MoE"), section "Weight layout and routing": sigmoid scores, the bias
// only chooses the experts, the gathered weights stay unbiased, norm_topk
// divides by sum + 1e-6 and then routed_scaling_factor multiplies.
// TensorFold pull #1492, "What": fp32 router weights; "Verification": an
// all-NaN router row must never pick the same expert twice.
//
// Logits are fp32 FMA chains in one fixed order, the same in every kernel
// here, so a token's logits (and so its picks and weights) do not depend on
// how many tokens share the launch:
//   H is cut into chunks of 32 consecutive h; segment w (0..7) holds chunks
//   c with c % 8 == w; p_w is an fmaf chain over segment w in increasing h,
//   starting at 0; L = p_0 + p_1 + ... + p_7, left to right.
//
// Selection: a warp per token; each lane holds experts lane, lane+32, ...;
// k rounds of a warp-wide max over 64-bit keys (score key, ~expert id).  The
// score key orders c = s + bias with NaN below every number and -0 == +0;
// a picked expert's key drops below every NaN key, so picks stay distinct
// even when every score is NaN (the row then picks 0, 1, ..., k-1).
#include "common.cuh"
#include "internal.h"
#include "launch.h"
#include "plan_dev.cuh"

namespace moe {
namespace {

constexpr int kSegs = 8;      // segments of the canonical logit order (= warps per CTA)
constexpr int kChunk = 32;    // h per chunk

MOE_DEV uint32_t score_key(float c) {
    if (c != c) return 0u;                      // NaN: below every number
    if (c == 0.0f) c = 0.0f;                    // -0 -> +0
    uint32_t u = __float_as_uint(c);
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

MOE_DEV float sigmoid_f32(float L) { return 1.0f / (1.0f + expf(-L)); }

// Picks and weights of one token.  Lv[i] is the logit of expert lane + 32 i.
// Lane j (< k) returns slot j's expert in *e_out (and writes idx/w rows).
template <int NE>
MOE_DEV int select_token(const float (&Lv)[NE], const float* __restrict__ bias, int E, int k,
                         float eps, float scale, bool softmax, bool no_norm, int32_t* idx_row,
                         float* w_row) {
    const int lane = threadIdx.x & 31;
    float s[NE];
    uint32_t khi[NE], klo[NE];
    // softmax: exp(L - max) / sum over the row (warp reductions); a NaN logit
    // makes every score of the row NaN
    float smax = 0.0f, sinv = 0.0f;
    bool row_nan = false;
    if (softmax) {
        float m = -INFINITY;
        bool nan_here = false;
#pragma unroll
        for (int i = 0; i < NE; ++i) {
            if (lane + 32 * i < E) {
                if (Lv[i] != Lv[i]) nan_here = true;
                else m = fmaxf(m, Lv[i]);
            }
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
        row_nan = __any_sync(0xffffffffu, nan_here);
        float z = 0.0f;
#pragma unroll
        for (int i = 0; i < NE; ++i)
            if (lane + 32 * i < E) z += expf(Lv[i] - m);
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) z += __shfl_xor_sync(0xffffffffu, z, o);
        smax = m;
        sinv = z;
    }
#pragma unroll
    for (int i = 0; i < NE; ++i) {
        const int e = lane + 32 * i;
        if (e < E) {
            s[i] = softmax ? (row_nan ? __int_as_float(0x7fc00000) : expf(Lv[i] - smax) / sinv)
                           : sigmoid_f32(Lv[i]);
            const float c = s[i] + (bias ? __ldg(bias + e) : 0.0f);
            khi[i] = score_key(c);
            klo[i] = 0xFFFFFFFFu - (uint32_t)e;
        } else {
            s[i] = 0.0f;
            khi[i] = 0u;
            klo[i] = 0u;
        }
    }
    int my_e = 0;
    float my_s = 0.0f, sum = 0.0f;
    for (int j = 0; j < k; ++j) {
        uint32_t bh = khi[0], bl = klo[0];
#pragma unroll
        for (int i = 1; i < NE; ++i)
            if (khi[i] > bh || (khi[i] == bh && klo[i] > bl)) { bh = khi[i]; bl = klo[i]; }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
            const uint32_t oh = __shfl_xor_sync(0xffffffffu, bh, o);
            const uint32_t ol = __shfl_xor_sync(0xffffffffu, bl, o);
            if (oh > bh || (oh == bh && ol > bl)) { bh = oh; bl = ol; }
        }
        const int ej = (int)(0xFFFFFFFFu - bl);
        const int owner = ej & 31, ii = ej >> 5;
        float mine = 0.0f;
#pragma unroll
        for (int i = 0; i < NE; ++i)
            if (i == ii) mine = s[i];
        if (lane == owner) {
#pragma unroll
            for (int i = 0; i < NE; ++i)
                if (i == ii) { khi[i] = 0u; klo[i] = 0u; }
        }
        const float sj = __shfl_sync(0xffffffffu, mine, owner);
        if (lane == j) { my_e = ej; my_s = sj; }
        sum += sj;                                 // slot order
    }
    const float denom = sum + eps;
    if (lane < k) {
        idx_row[lane] = my_e;
        w_row[lane] = no_norm ? my_s * scale : my_s / denom * scale;
    }
    return my_e;
}

MOE_DEV void zero_slice(const RouteArgs& a) {
    if (!a.zero_ptr) return;
    const size_t n4 = a.zero_count / 4;
    float4* p = reinterpret_cast<float4*>(a.zero_ptr);
    const size_t blocks = (size_t)gridDim.x * gridDim.y;
    const size_t block = (size_t)blockIdx.y * gridDim.x + blockIdx.x;
    const size_t stride = blocks * blockDim.x;
    for (size_t i = block * blockDim.x + threadIdx.x; i < n4; i += stride)
        p[i] = make_float4(0.f, 0.f, 0.f, 0.f);
}

// ---------------------------------------------------------------------------
// Small T (<= 32): one CTA per expert.  Warp w computes segment w's chain for
// every token (lane = token); the 8 partials are summed in order.
__global__ void __launch_bounds__(256) k_logits_small(RouteArgs a) {
    extern __shared__ float sm[];
    float* wr = sm;                       // H floats: this expert's router row
    float* part = sm + a.H;               // 8 x 32
    pdl_wait();
    zero_slice(a);
    const int e = blockIdx.x;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const float4* src = reinterpret_cast<const float4*>(a.w_router + (size_t)e * a.H);
    for (int i = threadIdx.x; i < a.H / 4; i += blockDim.x) reinterpret_cast<float4*>(wr)[i] = __ldg(src + i);
    __syncthreads();
    float acc = 0.0f;
    if (lane < a.T) {
        const uint16_t* xr = a.x + (size_t)lane * a.H;
        for (int c = warp; c < a.H / kChunk; c += kSegs) {
#pragma unroll
            for (int q = 0; q < kChunk / 8; ++q) {
                const int h = c * kChunk + q * 8;
                const uint4 xv = ld_nc(xr + h);
                acc = fmaf(bf16lo(xv.x), wr[h + 0], acc);
                acc = fmaf(bf16hi(xv.x), wr[h + 1], acc);
                acc = fmaf(bf16lo(xv.y), wr[h + 2], acc);
                acc = fmaf(bf16hi(xv.y), wr[h + 3], acc);
                acc = fmaf(bf16lo(xv.z), wr[h + 4], acc);
                acc = fmaf(bf16hi(xv.z), wr[h + 5], acc);
                acc = fmaf(bf16lo(xv.w), wr[h + 6], acc);
                acc = fmaf(bf16hi(xv.w), wr[h + 7], acc);
            }
        }
    }
    part[warp * 32 + lane] = acc;
    __syncthreads();
    if (warp == 0 && lane < a.T) {
        float L = part[lane];
#pragma unroll
        for (int w = 1; w < kSegs; ++w) L += part[w * 32 + lane];
        a.l_scratch[(size_t)lane * a.E + e] = L;
    }
    pdl_trigger();
}

// ---------------------------------------------------------------------------
// Selection from fp32 logits in memory; FUSE also builds the plan (one CTA,
// T <= 32 so P <= 1024).
template <int NE, bool FUSE, bool PART>
__global__ void __launch_bounds__(256) k_select(RouteArgs a) {
    __shared__ int s_idx[FUSE ? 1024 : 1];
    __shared__ int s_cnt[FUSE ? 256 : 1], s_off[FUSE ? 257 : 1], s_til[FUSE ? 257 : 1];
    __shared__ int s_cur[FUSE ? 256 : 1], s_wcnt[FUSE ? 8 * 256 : 1];
    pdl_wait();
    zero_slice(a);
    const float* L = a.logits ? a.logits : a.l_scratch;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    for (int t = blockIdx.x * 8 + warp; t < a.T; t += gridDim.x * 8) {
        float Lv[NE];
#pragma unroll
        for (int i = 0; i < NE; ++i) {
            const int e = lane + 32 * i;
            if (PART) {       // L = p_0 + p_1 + ... + p_7, left to right
                float L = 0.0f;
                if (e < a.E) {
                    L = a.part[(size_t)t * a.E + e];
#pragma unroll
                    for (int w = 1; w < kSegs; ++w) L += a.part[((size_t)w * a.T + t) * a.E + e];
                }
                Lv[i] = L;
            } else {
                Lv[i] = e < a.E ? L[(size_t)t * a.E + e] : 0.0f;
            }
        }
        const int e = select_token<NE>(Lv, a.bias, a.E, a.k, a.eps, a.scale, a.softmax != 0, a.no_norm != 0,
                                       a.idx + (size_t)t * a.k, a.w + (size_t)t * a.k);
        if (FUSE && lane < a.k) s_idx[t * a.k + lane] = e;
    }
    if (FUSE) {
        const int P = a.T * a.k, E = a.E;
        for (int i = threadIdx.x; i < 256; i += blockDim.x) s_cnt[i] = 0;
        for (int i = threadIdx.x; i < 8 * 256; i += blockDim.x) s_wcnt[i] = 0;
        __syncthreads();
        for (int p = threadIdx.x; p < P; p += blockDim.x) atomicAdd(&s_cnt[s_idx[p]], 1);
        __syncthreads();
        if (warp == 0) warp_exclusive_scan(s_cnt, s_off, E, 0);
        if (warp == 1) warp_exclusive_scan(s_cnt, s_til, E, kTileM);
        __syncthreads();
        for (int e = threadIdx.x; e <= E; e += blockDim.x) {
            a.offsets[e] = s_off[e];
            a.tiles[e] = s_til[e];
            if (e < E) {
                a.counts[e] = s_cnt[e];
                s_cur[e] = s_off[e];
            }
        }
        __syncthreads();
        stable_scatter<8>(s_idx, P, E, s_cur, s_wcnt, a.perm, a.inv);
    }
    pdl_trigger();
}

// ---------------------------------------------------------------------------
// Large T: TT tokens per CTA.  Warp w computes segment w (the canonical order)
// for all TT tokens and all EP = 32 NE experts as a register-blocked
// micro-GEMM: lane (tg = lane % 8, eg = lane / 8) owns tokens tg TPT .. and
// experts eg EPT .. (TPT = TT / 8, EPT = EP / 4), so each h costs 1-2 shared
// loads of token values and EPT / 4 of router values for TPT x EPT FMAs.
// Every (token, expert) logit is still one fmaf chain over the segment in
// increasing h, so the bits equal the small-T kernel's.  For E <= 64 the next
// chunk's router and token values are loaded into registers while the
// current chunk is computed.
template <int NE, int TT, int HCH>
__global__ void __launch_bounds__(256) k_route_large(RouteArgs a) {
    extern __shared__ float sm[];
    constexpr int EP = 32 * NE, TPT = TT / 8, EPT = EP / 4;
    constexpr int WARP_FLOATS = HCH * EP + HCH * TT;
    constexpr bool PF = NE <= 2;                  // register prefetch of the next chunk
    constexpr int WV = HCH / 4;                   // float4 of router values per expert per chunk
    constexpr int XV = HCH / 8;                   // uint4 of token values per token per chunk
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int tg = lane & 7, eg = lane >> 3;
    float* wt = sm + warp * WARP_FLOATS;          // [HCH][EP]
    float* xs = wt + HCH * EP;                    // [HCH][TT]
    pdl_wait();
    zero_slice(a);
    const int t0 = blockIdx.x * TT;
    const int E = a.E, H = a.H;
    const int nsub = H / HCH;                     // staging pieces along h
    constexpr int kPer = kChunk / HCH;            // pieces per canonical chunk

    float acc[TPT][EPT];
#pragma unroll
    for (int i = 0; i < TPT; ++i)
#pragma unroll
        for (int j = 0; j < EPT; ++j) acc[i][j] = 0.0f;

    float4 rw[NE][WV];
    uint4 rx[XV];
    // piece q of this warp's segment: canonical chunk warp + 8 (q / kPer), part q % kPer
    auto piece_h0 = [&](int q) { return (warp + kSegs * (q / kPer)) * kChunk + (q % kPer) * HCH; };
    const int npieces = ((H / kChunk - warp + kSegs - 1) / kSegs) * kPer;
    auto load = [&](int q) {
        const int h0 = piece_h0(q);
#pragma unroll
        for (int i = 0; i < NE; ++i) {
            const int e = lane + 32 * i;
            const float4* src = reinterpret_cast<const float4*>(a.w_router + (size_t)(e < E ? e : 0) * H + h0);
#pragma unroll
            for (int v = 0; v < WV; ++v) rw[i][v] = e < E ? __ldg(src + v) : make_float4(0.f, 0.f, 0.f, 0.f);
        }
        const int t = t0 + lane;
        const bool tv = lane < TT && t < a.T;
        const uint4* xsrc = reinterpret_cast<const uint4*>(a.x + (size_t)(tv ? t : 0) * H + h0);
#pragma unroll
        for (int v = 0; v < XV; ++v) rx[v] = tv ? ld_nc(xsrc + v) : make_uint4(0u, 0u, 0u, 0u);
    };
    auto stage = [&]() {
#pragma unroll
        for (int i = 0; i < NE; ++i) {
            const int e = lane + 32 * i;
#pragma unroll
            for (int v = 0; v < WV; ++v) {
                wt[(4 * v + 0) * EP + e] = rw[i][v].x;
                wt[(4 * v + 1) * EP + e] = rw[i][v].y;
                wt[(4 * v + 2) * EP + e] = rw[i][v].z;
                wt[(4 * v + 3) * EP + e] = rw[i][v].w;
            }
        }
        if (lane < TT) {
#pragma unroll
            for (int v = 0; v < XV; ++v) {
                xs[(8 * v + 0) * TT + lane] = bf16lo(rx[v].x);
                xs[(8 * v + 1) * TT + lane] = bf16hi(rx[v].x);
                xs[(8 * v + 2) * TT + lane] = bf16lo(rx[v].y);
                xs[(8 * v + 3) * TT + lane] = bf16hi(rx[v].y);
                xs[(8 * v + 4) * TT + lane] = bf16lo(rx[v].z);
                xs[(8 * v + 5) * TT + lane] = bf16hi(rx[v].z);
                xs[(8 * v + 6) * TT + lane] = bf16lo(rx[v].w);
                xs[(8 * v + 7) * TT + lane] = bf16hi(rx[v].w);
            }
        }
    };
    (void)nsub;
    if (PF && npieces > 0) load(0);
    for (int q = 0; q < npieces; ++q) {
        if (!PF) load(q);
        stage();
        __syncwarp();
        if (PF && q + 1 < npieces) load(q + 1);
#pragma unroll 4
        for (int hh = 0; hh < HCH; ++hh) {
            float xv[TPT];
            const float* xr = xs + hh * TT + tg * TPT;
            if (TPT == 4) {
                const float4 t4 = *reinterpret_cast<const float4*>(xr);
                xv[0] = t4.x; xv[TPT > 1 ? 1 : 0] = t4.y; xv[TPT > 2 ? 2 : 0] = t4.z; xv[TPT > 3 ? 3 : 0] = t4.w;
            } else if (TPT == 2) {
                const float2 t2 = *reinterpret_cast<const float2*>(xr);
                xv[0] = t2.x; xv[TPT > 1 ? 1 : 0] = t2.y;
            } else {
                xv[0] = xr[0];
            }
            const float4* wr = reinterpret_cast<const float4*>(wt + hh * EP + eg * EPT);
#pragma unroll
            for (int v = 0; v < EPT / 4; ++v) {
                const float4 w4 = wr[v];
#pragma unroll
                for (int i = 0; i < TPT; ++i) {
                    acc[i][4 * v + 0] = fmaf(xv[i], w4.x, acc[i][4 * v + 0]);
                    acc[i][4 * v + 1] = fmaf(xv[i], w4.y, acc[i][4 * v + 1]);
                    acc[i][4 * v + 2] = fmaf(xv[i], w4.z, acc[i][4 * v + 2]);
                    acc[i][4 * v + 3] = fmaf(xv[i], w4.w, acc[i][4 * v + 3]);
                }
            }
        }
        __syncwarp();
    }
    __syncthreads();
    float* part = sm;                              // [8][TT][EP]
#pragma unroll
    for (int i = 0; i < TPT; ++i)
#pragma unroll
        for (int j = 0; j < EPT; ++j) part[(warp * TT + tg * TPT + i) * EP + eg * EPT + j] = acc[i][j];
    __syncthreads();
    for (int m = warp; m < TT; m += kSegs) {
        const int t = t0 + m;
        if (t >= a.T) break;
        float Lv[NE];
#pragma unroll
        for (int i = 0; i < NE; ++i) {
            const int e = lane + 32 * i;
            float L = part[(0 * TT + m) * EP + e];
#pragma unroll
            for (int w = 1; w < kSegs; ++w) L += part[(w * TT + m) * EP + e];
            Lv[i] = L;
        }
        select_token<NE>(Lv, a.bias, E, a.k, a.eps, a.scale, a.softmax != 0, a.no_norm != 0,
                         a.idx + (size_t)t * a.k, a.w + (size_t)t * a.k);
    }
    pdl_trigger();
}

template <int NE, int TT, int HCH>
cudaError_t run_large(const RouteArgs& a, bool pdl, cudaStream_t s) {
    constexpr int EP = 32 * NE;
    size_t stage = (size_t)8 * (HCH * EP + HCH * TT) * sizeof(float);
    size_t part = (size_t)8 * TT * EP * sizeof(float);
    size_t smem = stage > part ? stage : part;
    auto kern = k_route_large<NE, TT, HCH>;
    cudaError_t e = ensure_smem(kern, smem);
    if (e != cudaSuccess) return e;
    return launch_k(kern, dim3((a.T + TT - 1) / TT), dim3(256), smem, s, pdl, a);
}

template <int NE, bool PART>
cudaError_t run_select(const RouteArgs& a, bool fuse, bool pdl, cudaStream_t s) {
    if (fuse) return launch_k(k_select<NE, true, PART>, dim3(1), dim3(256), 0, s, pdl, a);
    return launch_k(k_select<NE, false, PART>, dim3((a.T + 7) / 8), dim3(256), 0, s, pdl, a);
}

template <bool PART>
cudaError_t dispatch_select(const RouteArgs& a, bool fuse, bool pdl, cudaStream_t s) {
    if (a.E <= 32) return run_select<1, PART>(a, fuse, pdl, s);
    if (a.E <= 64) return run_select<2, PART>(a, fuse, pdl, s);
    if (a.E <= 128) return run_select<4, PART>(a, fuse, pdl, s);
    return run_select<8, PART>(a, fuse, pdl, s);
}

// ---------------------------------------------------------------------------
// Segment partials: each CTA computes one segment's fmaf chains (the
// canonical order above) for a block of tokens and all experts and writes
// p_w[t][e]; k_select<.., PART> then forms L = p_0 + ... + p_7 in order, so
// these logits are bit-identical to the one-CTA kernels', with 8x the CTAs.

// T <= 32: CTA (expert e, segment w), one warp, lane = token.  The
// segment's router values and token rows (up to kSmallPass chunks at a time)
// are requested by 16-byte cp.async all at once, so the loads pay one memory
// latency rather than one per chunk; then each lane runs its chain from
// shared memory.
constexpr int kSmallPass = 8;                         // chunks staged per pass
constexpr int kSmallRow = kSmallPass * kChunk + 8;    // bf16 per staged token row (+16 B: LDS.128 phases
                                                      // of 8 lanes fall on distinct bank groups)

MOE_DEV void cp_async16(void* dst, const void* src) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(static_cast<uint32_t>(__cvta_generic_to_shared(dst))),
                 "l"(src)
                 : "memory");
}

__global__ void __launch_bounds__(32) k_logits_seg_small(RouteArgs a) {
    __shared__ __align__(16) float s_w[kSmallPass * kChunk];
    __shared__ __align__(16) uint16_t s_x[32 * kSmallRow];
    pdl_wait();
    zero_slice(a);
    const int e = blockIdx.x, w = blockIdx.y, lane = threadIdx.x;
    const int H = a.H, T = a.T;
    const int nch = (H / kChunk - w + kSegs - 1) / kSegs;
    const float* wr = a.w_router + (size_t)e * H;
    float acc = 0.0f;
    for (int j0 = 0; j0 < nch; j0 += kSmallPass) {
        const int np = min(kSmallPass, nch - j0);
        // router: np chunks x 8 pieces of 16 B; tokens: T rows x np chunks x 4 pieces
        for (int i = lane; i < np * 8; i += 32) {
            const int j = i >> 3, q = i & 7;
            cp_async16(s_w + j * kChunk + 4 * q, wr + (w + kSegs * (j0 + j)) * kChunk + 4 * q);
        }
        for (int i = lane; i < T * np * 4; i += 32) {
            const int t = i / (np * 4), r = i - t * np * 4, j = r >> 2, q = r & 3;
            cp_async16(s_x + t * kSmallRow + j * kChunk + 8 * q,
                       a.x + (size_t)t * H + (w + kSegs * (j0 + j)) * kChunk + 8 * q);
        }
        asm volatile("cp.async.wait_all;" ::: "memory");
        __syncwarp();
        if (lane < T) {
            const uint4* xr = reinterpret_cast<const uint4*>(s_x + lane * kSmallRow);
            const float4* wv = reinterpret_cast<const float4*>(s_w);
            for (int j = 0; j < np; ++j) {
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    const uint4 xv = xr[j * 4 + q];
                    const float4 w0 = wv[j * 8 + 2 * q], w1 = wv[j * 8 + 2 * q + 1];
                    acc = fmaf(bf16lo(xv.x), w0.x, acc);
                    acc = fmaf(bf16hi(xv.x), w0.y, acc);
                    acc = fmaf(bf16lo(xv.y), w0.z, acc);
                    acc = fmaf(bf16hi(xv.y), w0.w, acc);
                    acc = fmaf(bf16lo(xv.z), w1.x, acc);
                    acc = fmaf(bf16hi(xv.z), w1.y, acc);
                    acc = fmaf(bf16lo(xv.w), w1.z, acc);
                    acc = fmaf(bf16hi(xv.w), w1.w, acc);
                }
            }
        }
        __syncwarp();      // the next pass overwrites the staged values
    }
    if (lane < T) a.part[((size_t)w * T + lane) * a.E + e] = acc;
    pdl_trigger();
}

// Large T: CTA (token block, segment w), 64 threads; thread (tg, eg) owns
// TPT tokens x EPT experts of the TT x EP block (register-blocked FMAs, the
// router chunk staged transposed, the token chunk staged as fp32).
template <int NE, int TT, int TPT, int EPT>
__global__ void __launch_bounds__(64) k_logits_seg(RouteArgs a) {
    constexpr int EP = 32 * NE;
    static_assert(TT == 8 * TPT && EP == 8 * EPT, "thread tiling");
    constexpr int WF4 = EP * 8 / 64;      // float4 of router values per thread per chunk
    constexpr int XV4 = TT * 4 / 64;      // uint4 of token values per thread per chunk
    constexpr bool PF = NE <= 4;          // register prefetch of the next chunk
    __shared__ __align__(16) float wt[kChunk * EP];
    __shared__ __align__(16) float xs[kChunk * TT];
    pdl_wait();
    zero_slice(a);
    const int w = blockIdx.y, t0 = blockIdx.x * TT, tid = threadIdx.x;
    const int tg = tid & 7, eg = tid >> 3;
    const int E = a.E, H = a.H;
    const int nch = (H / kChunk - w + kSegs - 1) / kSegs;
    float acc[TPT][EPT];
#pragma unroll
    for (int i = 0; i < TPT; ++i)
#pragma unroll
        for (int j = 0; j < EPT; ++j) acc[i][j] = 0.0f;
    float4 rw[WF4];
    uint4 rx[XV4 > 0 ? XV4 : 1];
    auto load = [&](int j) {
        const int h0 = (w + kSegs * j) * kChunk;
#pragma unroll
        for (int i = 0; i < WF4; ++i) {
            const int f = tid + 64 * i;
            const int e = f % EP, v = f / EP;              // consecutive threads: consecutive experts
            rw[i] = e < E ? __ldg(reinterpret_cast<const float4*>(a.w_router + (size_t)e * H + h0) + v)
                          : make_float4(0.f, 0.f, 0.f, 0.f);
        }
#pragma unroll
        for (int i = 0; i < XV4; ++i) {
            const int f = tid + 64 * i;
            const int t = f % TT, v = f / TT;
            const bool ok = t0 + t < a.T;
            rx[i] = ok ? ld_nc(reinterpret_cast<const uint4*>(a.x + (size_t)(t0 + t) * H + h0) + v)
                       : make_uint4(0u, 0u, 0u, 0u);
        }
    };
    auto stage = [&]() {
#pragma unroll
        for (int i = 0; i < WF4; ++i) {
            const int f = tid + 64 * i;
            const int e = f % EP, v = f / EP;
            wt[(4 * v + 0) * EP + e] = rw[i].x;
            wt[(4 * v + 1) * EP + e] = rw[i].y;
            wt[(4 * v + 2) * EP + e] = rw[i].z;
            wt[(4 * v + 3) * EP + e] = rw[i].w;
        }
#pragma unroll
        for (int i = 0; i < XV4; ++i) {
            const int f = tid + 64 * i;
            const int t = f % TT, v = f / TT;
            xs[(8 * v + 0) * TT + t] = bf16lo(rx[i].x);
            xs[(8 * v + 1) * TT + t] = bf16hi(rx[i].x);
            xs[(8 * v + 2) * TT + t] = bf16lo(rx[i].y);
            xs[(8 * v + 3) * TT + t] = bf16hi(rx[i].y);
            xs[(8 * v + 4) * TT + t] = bf16lo(rx[i].z);
            xs[(8 * v + 5) * TT + t] = bf16hi(rx[i].z);
            xs[(8 * v + 6) * TT + t] = bf16lo(rx[i].w);
            xs[(8 * v + 7) * TT + t] = bf16hi(rx[i].w);
        }
    };
    if (PF && nch > 0) load(0);
    for (int j = 0; j < nch; ++j) {
        if (!PF) load(j);
        __syncthreads();            // the previous chunk's compute is done with the buffers
        stage();
        __syncthreads();
        if (PF && j + 1 < nch) load(j + 1);
#pragma unroll 4
        for (int hh = 0; hh < kChunk; ++hh) {
            float xv[TPT];
            if (TPT == 4) {
                const float4 t4 = *reinterpret_cast<const float4*>(xs + hh * TT + tg * TPT);
                xv[0] = t4.x; xv[TPT > 1 ? 1 : 0] = t4.y; xv[TPT > 2 ? 2 : 0] = t4.z; xv[TPT > 3 ? 3 : 0] = t4.w;
            } else {
                const float2 t2 = *reinterpret_cast<const float2*>(xs + hh * TT + tg * TPT);
                xv[0] = t2.x; xv[TPT > 1 ? 1 : 0] = t2.y;
            }
            const float4* wp = reinterpret_cast<const float4*>(wt + hh * EP + eg * EPT);
#pragma unroll
            for (int q = 0; q < EPT / 4; ++q) {
                const float4 w4 = wp[q];
#pragma unroll
                for (int i = 0; i < TPT; ++i) {
                    acc[i][4 * q + 0] = fmaf(xv[i], w4.x, acc[i][4 * q + 0]);
                    acc[i][4 * q + 1] = fmaf(xv[i], w4.y, acc[i][4 * q + 1]);
                    acc[i][4 * q + 2] = fmaf(xv[i], w4.z, acc[i][4 * q + 2]);
                    acc[i][4 * q + 3] = fmaf(xv[i], w4.w, acc[i][4 * q + 3]);
                }
            }
        }
    }
#pragma unroll
    for (int i = 0; i < TPT; ++i) {
        const int t = t0 + tg * TPT + i;
        if (t >= a.T) continue;
#pragma unroll
        for (int j = 0; j < EPT; ++j) {
            const int e = eg * EPT + j;
            if (e < E) a.part[((size_t)w * a.T + t) * E + e] = acc[i][j];
        }
    }
    pdl_trigger();
}

}  // namespace

cudaError_t launch_route(const RouteArgs& a, bool fuse_plan, bool pdl, cudaStream_t s, int* n_launched) {
    *n_launched = 0;
    if (a.T == 0) return cudaSuccess;
    *n_launched = 1;
    const bool small = a.T <= kSmallT;
    if (a.logits) return dispatch_select<false>(a, fuse_plan && small, pdl, s);
    if (a.part) {
        // per-segment partials (8x the CTAs), then select from their ordered sum
        cudaError_t e;
        if (small) {
            e = launch_k(k_logits_seg_small, dim3(a.E, kSegs), dim3(32), 0, s, pdl, a);
        } else if (a.E <= 32) {
            e = launch_k(k_logits_seg<1, 32, 4, 4>, dim3((a.T + 31) / 32, kSegs), dim3(64), 0, s, pdl, a);
        } else if (a.E <= 64) {
            e = launch_k(k_logits_seg<2, 32, 4, 8>, dim3((a.T + 31) / 32, kSegs), dim3(64), 0, s, pdl, a);
        } else if (a.E <= 128) {
            e = launch_k(k_logits_seg<4, 32, 4, 16>, dim3((a.T + 31) / 32, kSegs), dim3(64), 0, s, pdl, a);
        } else {
            e = launch_k(k_logits_seg<8, 16, 2, 32>, dim3((a.T + 15) / 16, kSegs), dim3(64), 0, s, pdl, a);
        }
        if (e != cudaSuccess) return e;
        *n_launched = 2;
        RouteArgs b = a;
        b.zero_ptr = nullptr;
        return dispatch_select<true>(b, fuse_plan && small, pdl, s);
    }
    if (small && a.l_scratch) {
        // two launches: per-expert logits into scratch (this one also zeroes
        // the accumulator), then select (+ plan)
        size_t smem = (size_t)a.H * sizeof(float) + 8 * 32 * sizeof(float);
        cudaError_t e = ensure_smem(k_logits_small, smem);
        if (e != cudaSuccess) return e;
        e = launch_k(k_logits_small, dim3(a.E), dim3(256), smem, s, pdl, a);
        if (e != cudaSuccess) return e;
        *n_launched = 2;
        RouteArgs b = a;
        b.zero_ptr = nullptr;
        return dispatch_select<false>(b, fuse_plan, pdl, s);
    }
    if (a.E <= 32) return run_large<1, 32, 32>(a, pdl, s);
    if (a.E <= 64) return run_large<2, 32, 32>(a, pdl, s);
    if (a.E <= 128) return run_large<4, 16, 32>(a, pdl, s);
    return run_large<8, 8, 16>(a, pdl, s);
}

}  // namespace moe
