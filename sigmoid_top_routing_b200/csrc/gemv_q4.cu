// Decode-sized grouped GEMV over 4-bit experts, dequantised in registers:
// MLX-style affine 4-bit (group 64) and NVFP4 (ModelOpt layout).
//
// Weight formats (the pages name both):
//   affine (TensorFold pull #1492, "What"): codes (E, N, K/8) uint32, 8 nibbles
//     per word with the low nibble the lowest k; scale and bias (E, N, K/64)
//     bf16; w = scale * q + bias.
//   NVFP4 (TensorFold issue #548: "weight uint8 [N, K/2], weight_scale e4m3
//     [N, K/16], weight_scale_2 as the global scale"): codes (E, N, K/2) uint8,
//     two e2m1 codes per byte with the low nibble the lower k; one e4m3 scale
//     per 16 k; one fp32 global scale per expert and projection;
//     w = e2m1(q) * e4m3(s) * g.
//
// At a few tokens per expert the step is a stream of codes from HBM, so the
// kernel is built around issuing as few instructions per weight as it can
// while keeping many loads in flight.  The legacy m16n8k16 tensor-core MMA is
// the dot-product engine (A = 16 weight rows x 16 k, B = 16 k x 8 tokens).
//
// Work.  A CTA of 8 warps takes a unit (active expert, chunk of <= 8 of its
// tokens, block of weight rows).  Warp w owns 16 MMA rows and one of KS
// slices of K (KS = 1, 2, 4 or 8: more slices when there are few units, as
// at one token); the slices' partial sums meet in shared memory in a fixed
// order.  A lane streams 8 bytes (16 k) of each of its two MMA rows per step,
// an 8-deep ring of steps in flight; the chunk's token rows are staged in
// shared memory once per unit while the first codes are already in flight.
//
// Affine (bf16 MMA): a nibble pair (q_j, q_j+4) of a code word becomes the
// exact bf16 pair (128 + q) with one mask-and-or; the token rows are staged
// with each 8-k group reordered (x0 x4 x1 x5 x2 x6 x3 x7) to match, so the B
// fragments load straight from shared memory.  Per group of 64 k and row,
//     sum_k w x = s * sum_k (128 + q) x + (b - 128 s) * sum_k x,
// with sum_k x precomputed per token and group at staging; the group's scale
// and bias ride in the code ring (lane tq of a quad fetches one of the four
// values its quad needs, and shuffles share them).
//
// NVFP4 (f16 MMA): cvt.rn.f16x2.e2m1x2 turns a code byte into an f16 pair and
// one f16 multiply by the block scale gives e2m1 * e4m3 exactly (at most six
// significant bits, within f16's normal range).  The token rows are staged in
// f16 after a per-token power-of-two scale 2^-e that puts the row's largest
// magnitude in [2^14, 2^15): exact, and no finite bf16 activation can
// overflow.  The accumulator is multiplied back by 2^e and by the global
// scale in the epilogue.
//
//   up   (SwiGLU): h[slot, i] = bf16_rn(silu(g) * u); MMA rows 0..7 hold gate
//                  rows i0..i0+7 and rows 8..15 the matching up rows, so a lane
//                  holds gate and up of the same (feature, token)
//   up   (relu^2): h[slot, i] = bf16_rn(relu(u)^2), 16 consecutive rows
//   down:          y_acc[t, n] += w[pair] * (W2[e][n] . h[slot])   (fp32 atomics;
//                  a plain store per plan slot under the ordered combine)
#include <cuda_fp16.h>

#include "common.cuh"
#include "internal.h"
#include "launch.h"
#include "quant.cuh"

namespace moe {
namespace {

constexpr int kQWarps = 8;                // warps per CTA
constexpr int kQTok = 8;                  // tokens per unit (the MMA's N)
constexpr int kQRing = 8;                 // steps of codes in flight per warp
constexpr int kQStepK = 64;               // k per warp step: 4 lanes x 16
constexpr int kQMaxK = 8192;              // the token tile of 8 rows must fit in shared memory

enum { kQUpSwiglu = 0, kQUpRelu2 = 1, kQDown = 2 };
enum { kQAffine = 1, kQNvfp4 = 2 };       // the library's weight format codes

MOE_DEV void mma_bf16_16816(float* c, uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3, uint32_t b0,
                            uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};\n"
        : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

MOE_DEV void mma_f16_16816(float* c, uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3, uint32_t b0,
                           uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};\n"
        : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// Nibbles j and j + 4 of v as the bf16 pair (128 + q_j, 128 + q_{j+4}): exact.
MOE_DEV uint32_t nib_pair(uint32_t v, int j) { return ((v >> (4 * j)) & 0x000F000Fu) | 0x43004300u; }

MOE_DEV uint32_t prmt(uint32_t a, uint32_t b, uint32_t sel) {
    uint32_t r;
    asm("prmt.b32 %0, %1, %2, %3;" : "=r"(r) : "r"(a), "r"(b), "r"(sel));
    return r;
}

MOE_DEV uint2 ld_codes(const void* p, uint64_t pol) {
    uint2 r;
    asm volatile("ld.global.nc.L1::no_allocate.L2::cache_hint.v2.u32 {%0,%1}, [%2], %3;"
                 : "=r"(r.x), "=r"(r.y)
                 : "l"(p), "l"(pol));
    return r;
}

MOE_DEV uint32_t ld_u8(const uint8_t* p) {
    unsigned short v;
    asm volatile("ld.global.nc.u8 %0, [%1];" : "=h"(v) : "l"(p));
    return v;
}

// Shared-memory row stride of the token tile, in 16-bit elements: K + 8 puts
// the rows of one LDS.128 phase on distinct bank groups.
MOE_DEV __host__ int q_stride(int K) { return K + 8; }

struct QLayout {          // dynamic shared memory of one CTA (byte offsets)
    int x, sx, total;
};

MOE_DEV __host__ QLayout q_layout(int fmt, int K) {
    QLayout L;
    L.x = 0;
    int off = kQTok * q_stride(K) * 2;
    L.sx = off;                                   // affine: sum_k x per (group, token), [G][8] fp32
    if (fmt == kQAffine) off += (K / 64) * kQTok * 4;
    L.total = off;
    return L;
}

template <int FMT, int MODE, int KS>
__global__ void __launch_bounds__(kQWarps * 32, 2) k_gemv_q4(ExpertArgs a) {
    constexpr int RBC = kQWarps / KS;            // 16-row MMA blocks per CTA
    extern __shared__ __align__(16) unsigned char q_smem[];
    __shared__ int s_base[257];
    __shared__ float s_tm[kQTok];                // per-token output multiplier (NVFP4)
    __shared__ float s_red[KS > 1 ? kQWarps : 1][32][4];
    pdl_wait();
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int g = lane >> 2, tq = lane & 3;
    constexpr bool down = MODE == kQDown;
    const int K = down ? a.I : a.H;              // reduction length
    const int N = down ? a.H : (MODE == kQUpSwiglu ? 2 * a.I : a.I);   // weight rows per expert
    const int G = K / 64;
    const int RB = MODE == kQUpSwiglu ? a.I / 8 : N / 16;              // MMA row blocks per expert
    const int NRQ = (RB + RBC - 1) / RBC;                              // row blocks of a CTA
    const int XS = q_stride(K);
    const QLayout L = q_layout(FMT, K);
    uint16_t* s_x = reinterpret_cast<uint16_t*>(q_smem + L.x);
    float* s_sx = reinterpret_cast<float*>(q_smem + L.sx);
    const uint8_t* codes = reinterpret_cast<const uint8_t*>(down ? a.w2 : a.w1);
    const uint16_t* wsc = down ? a.w2_scale : a.w1_scale;   // affine scale (bf16) / NVFP4 e4m3 bytes
    const uint16_t* wbi = down ? a.w2_bias : a.w1_bias;     // affine bias
    const float* wglob = down ? a.w2_global : a.w1_global;  // NVFP4 global scale per expert
    const uint8_t* wsc8 = reinterpret_cast<const uint8_t*>(wsc);

    // units per expert = token chunks x row blocks; prefix over experts
    if (warp == 0) {
        int run = 0;
        for (int e0 = 0; e0 < a.E; e0 += 32) {
            const int e = e0 + lane;
            const int nu = (e < a.E && e != a.skip) ? (a.counts[e] + kQTok - 1) / kQTok * NRQ : 0;
            int v = nu;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int y = __shfl_up_sync(0xffffffffu, v, o);
                if (lane >= o) v += y;
            }
            if (e < a.E) s_base[e] = run + v - nu;
            run += __shfl_sync(0xffffffffu, v, 31);
        }
        if (lane == 0) s_base[a.E] = run;
    }
    __syncthreads();
    const int total = s_base[a.E];
    const uint64_t pol = policy_evict_first();
    const size_t row_bytes = (size_t)K / 2;      // code bytes per weight row (both formats)
    const int KW = K / KS;                       // k of this warp's slice
    const int nsteps = KW / kQStepK;
    const int rbl = warp / KS, ks = warp % KS;
    const int kbeg = ks * KW;
    // affine: lane tq of a quad fetches one of (scale row g, bias row g, scale row g+8, bias row g+8)
    const uint16_t* sbsrc = tq & 1 ? wbi : wsc;

    for (int u = blockIdx.x; u < total; u += gridDim.x) {
        int lo = 0, hi = a.E;                    // expert: last e with s_base[e] <= u
        while (lo < hi) {
            const int mid = (lo + hi + 1) >> 1;
            if (s_base[mid] <= u) lo = mid;
            else hi = mid - 1;
        }
        const int e = lo;
        const int cnt = a.counts[e], off = a.offsets[e];
        const int nch = (cnt + kQTok - 1) / kQTok;
        const int local = u - s_base[e];
        const int rq = local / nch, ch = local % nch;
        const int nt = min(kQTok, cnt - ch * kQTok);
        const int slot0 = off + ch * kQTok;
        const int rb = rq * RBC + rbl;           // this warp's row block
        const bool active = rb < RB;
        // weight row (within the expert) of MMA row r of row block b
        auto wrow = [&](int b, int r) -> int {
            if (MODE == kQUpSwiglu) return r < 8 ? b * 8 + r : a.I + b * 8 + (r - 8);
            return b * 16 + r;
        };
        const size_t ebase = (size_t)e * N;
        const size_t r0 = ebase + wrow(rb, g), r1 = ebase + wrow(rb, g + 8);
        const uint8_t* p0 = codes + r0 * row_bytes + (kbeg + 16 * tq) / 2;
        const uint8_t* p1 = codes + r1 * row_bytes + (kbeg + 16 * tq) / 2;
        const uint8_t* ps0 = wsc8 + r0 * (K / 16) + kbeg / 16 + tq;   // NVFP4 block scales
        const uint8_t* ps1 = wsc8 + r1 * (K / 16) + kbeg / 16 + tq;

        // the code ring goes out first; the token rows are staged meanwhile
        uint2 q0[kQRing], q1[kQRing];
        uint32_t sc[kQRing];                     // NVFP4: the two rows' scale bytes (row g | row g+8 << 8)
        if (active) {
#pragma unroll
            for (int d = 0; d < kQRing; ++d) {
                if (d < nsteps) {
                    q0[d] = ld_codes(p0 + 32 * d, pol);
                    q1[d] = ld_codes(p1 + 32 * d, pol);
                    if (FMT == kQNvfp4) sc[d] = ld_u8(ps0 + 4 * d) | (ld_u8(ps1 + 4 * d) << 8);
                    else sc[d] = __ldg(sbsrc + (tq < 2 ? r0 : r1) * G + kbeg / 64 + d);
                }
            }
        }

        // ---- stage the chunk's token rows (one warp per row)
        for (int n = warp; n < nt; n += kQWarps) {
            const uint16_t* src = down ? a.h + (size_t)(slot0 + n) * a.I
                                       : a.x + (size_t)(a.perm[slot0 + n] / a.k) * a.H;
            const uint4* s4 = reinterpret_cast<const uint4*>(src);
            uint4* d4 = reinterpret_cast<uint4*>(s_x + n * XS);
            const int nc = K / 8;                // 8-k chunks of the row
            if (FMT == kQNvfp4) {
                float amax = 0.0f;
                for (int c = lane; c < nc; c += 32) {
                    const uint4 v = ld_nc(s4 + c);
                    const uint32_t w4[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
                    for (int i = 0; i < 4; ++i)
                        amax = fmaxf(amax, fmaxf(fabsf(bf16lo(w4[i])), fabsf(bf16hi(w4[i]))));
                }
#pragma unroll
                for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
                // 2^-ex puts the largest magnitude in [2^14, 2^15); NaN / inf rows keep 1
                int ex = 0;
                if (amax > 0.0f && amax <= 3.4e38f) {
                    int e2;
                    frexpf(amax, &e2);            // amax = m * 2^e2, m in [0.5, 1)
                    ex = max(-100, min(100, e2 - 15));
                }
                const float mul = __int_as_float((127 - ex) << 23);
                if (lane == 0) s_tm[n] = __int_as_float((127 + ex) << 23) * wglob[e];
                for (int c = lane; c < nc; c += 32) {
                    const uint4 v = ld_nc(s4 + c);
                    const uint32_t w4[4] = {v.x, v.y, v.z, v.w};
                    uint32_t o4[4];
#pragma unroll
                    for (int i = 0; i < 4; ++i) {
                        const __half2 h = __floats2half2_rn(bf16lo(w4[i]) * mul, bf16hi(w4[i]) * mul);
                        o4[i] = *reinterpret_cast<const uint32_t*>(&h);
                    }
                    d4[c] = make_uint4(o4[0], o4[1], o4[2], o4[3]);
                }
            } else {
                // affine: reorder each 8-k chunk to (x0 x4 x1 x5 x2 x6 x3 x7) and sum per group of 64
                for (int c0 = 0; c0 < nc; c0 += 32) {
                    const int c = c0 + lane;
                    float part = 0.0f;
                    if (c < nc) {
                        const uint4 v = ld_nc(s4 + c);
                        d4[c] = make_uint4(prmt(v.x, v.z, 0x5410), prmt(v.x, v.z, 0x7632),
                                           prmt(v.y, v.w, 0x5410), prmt(v.y, v.w, 0x7632));
                        part = ((bf16lo(v.x) + bf16hi(v.x)) + (bf16lo(v.y) + bf16hi(v.y))) +
                               ((bf16lo(v.z) + bf16hi(v.z)) + (bf16lo(v.w) + bf16hi(v.w)));
                    }
                    part += __shfl_xor_sync(0xffffffffu, part, 1);
                    part += __shfl_xor_sync(0xffffffffu, part, 2);
                    part += __shfl_xor_sync(0xffffffffu, part, 4);
                    if ((lane & 7) == 0 && c < nc) s_sx[(c >> 3) * kQTok + n] = part;
                }
            }
        }
        __syncthreads();

        float acc[4] = {0.f, 0.f, 0.f, 0.f};
        if (active) {
            const uint16_t* xr = s_x + g * XS + kbeg + 16 * tq;
            for (int sb = 0; sb < nsteps; sb += kQRing) {
#pragma unroll
                for (int d = 0; d < kQRing; ++d) {
                    const int st = sb + d;
                    if (st < nsteps) {
                        const uint4 xa = *reinterpret_cast<const uint4*>(xr + kQStepK * st);
                        const uint4 xb = *reinterpret_cast<const uint4*>(xr + kQStepK * st + 8);
                        if (FMT == kQNvfp4) {
                            const uint32_t s2 = e4m3x2_to_f16x2(sc[d]);           // (scale row g, scale row g+8)
                            const uint32_t sg = prmt(s2, s2, 0x1010), sh = prmt(s2, s2, 0x3232);
#pragma unroll
                            for (int j = 0; j < 2; ++j) {
                                const uint4 xv = j ? xb : xa;
                                uint32_t pa[4], pb[4];
                                e2m1x8_to_f16(j ? q0[d].y : q0[d].x, pa);
                                e2m1x8_to_f16(j ? q1[d].y : q1[d].x, pb);
#pragma unroll
                                for (int i = 0; i < 4; ++i) {
                                    pa[i] = hmul2_u32(pa[i], sg);
                                    pb[i] = hmul2_u32(pb[i], sh);
                                }
                                mma_f16_16816(acc, pa[0], pb[0], pa[1], pb[1], xv.x, xv.y);
                                mma_f16_16816(acc, pa[2], pb[2], pa[3], pb[3], xv.z, xv.w);
                            }
                        } else {
                            float cg[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
                            for (int j = 0; j < 2; ++j) {
                                const uint4 xv = j ? xb : xa;
                                const uint32_t v = j ? q0[d].y : q0[d].x;   // MMA row g
                                const uint32_t w = j ? q1[d].y : q1[d].x;   // MMA row g + 8
                                mma_bf16_16816(cg, nib_pair(v, 0), nib_pair(w, 0), nib_pair(v, 1), nib_pair(w, 1),
                                               xv.x, xv.y);
                                mma_bf16_16816(cg, nib_pair(v, 2), nib_pair(w, 2), nib_pair(v, 3), nib_pair(w, 3),
                                               xv.z, xv.w);
                            }
                            const int qb = lane & ~3;
                            const float s0 = bf16f((uint16_t)__shfl_sync(0xffffffffu, sc[d], qb + 0));
                            const float b0 = bf16f((uint16_t)__shfl_sync(0xffffffffu, sc[d], qb + 1));
                            const float s1 = bf16f((uint16_t)__shfl_sync(0xffffffffu, sc[d], qb + 2));
                            const float b1 = bf16f((uint16_t)__shfl_sync(0xffffffffu, sc[d], qb + 3));
                            const float c0 = fmaf(-128.f, s0, b0), c1 = fmaf(-128.f, s1, b1);   // exact
                            const float2 sx = *reinterpret_cast<const float2*>(s_sx + (kbeg / 64 + st) * kQTok + 2 * tq);
                            acc[0] = fmaf(s0, cg[0], fmaf(c0, sx.x, acc[0]));
                            acc[1] = fmaf(s0, cg[1], fmaf(c0, sx.y, acc[1]));
                            acc[2] = fmaf(s1, cg[2], fmaf(c1, sx.x, acc[2]));
                            acc[3] = fmaf(s1, cg[3], fmaf(c1, sx.y, acc[3]));
                        }
                        if (st + kQRing < nsteps) {                        // refill this ring slot
                            q0[d] = ld_codes(p0 + 32 * (st + kQRing), pol);
                            q1[d] = ld_codes(p1 + 32 * (st + kQRing), pol);
                            if (FMT == kQNvfp4)
                                sc[d] = ld_u8(ps0 + 4 * (st + kQRing)) | (ld_u8(ps1 + 4 * (st + kQRing)) << 8);
                            else
                                sc[d] = __ldg(sbsrc + (tq < 2 ? r0 : r1) * G + kbeg / 64 + st + kQRing);
                        }
                    }
                }
            }
        }
        // the K slices of a row block meet in a fixed order (slice 0 first)
        if (KS > 1) {
#pragma unroll
            for (int i = 0; i < 4; ++i) s_red[warp][lane][i] = acc[i];
            __syncthreads();
            if (ks == 0) {
#pragma unroll
                for (int q = 1; q < KS; ++q) {
#pragma unroll
                    for (int i = 0; i < 4; ++i) acc[i] += s_red[warp + q][lane][i];
                }
            }
        }
        if (active && ks == 0) {
            // acc[0], acc[1]: MMA row g, tokens 2tq, 2tq + 1; acc[2], acc[3]: row g + 8
#pragma unroll
            for (int jn = 0; jn < 2; ++jn) {
                const int n = 2 * tq + jn;
                if (n >= nt) continue;
                const int slot = slot0 + n;
                float va = acc[jn], vb = acc[2 + jn];
                if (FMT == kQNvfp4) {
                    va *= s_tm[n];
                    vb *= s_tm[n];
                }
                if (MODE == kQUpSwiglu) {
                    clamp_swiglu(va, vb, a.swiglu_limit);
                    a.h[(size_t)slot * a.I + rb * 8 + g] = f2bf16(act_swiglu(va, vb));
                } else if (MODE == kQUpRelu2) {
                    a.h[(size_t)slot * a.I + rb * 16 + g] = f2bf16(act_relu2(va));
                    a.h[(size_t)slot * a.I + rb * 16 + g + 8] = f2bf16(act_relu2(vb));
                } else {
                    const int pair = a.perm[slot];
                    const float wt = a.topk_w[pair];
                    if (a.ordered) {
                        float* orow = a.y_acc + (size_t)slot * a.H + rb * 16 + g;
                        orow[0] = wt * va;
                        orow[8] = wt * vb;
                    } else {
                        float* yrow = a.y_acc + (size_t)(pair / a.k) * a.H + rb * 16 + g;
                        atomicAdd(yrow, wt * va);
                        atomicAdd(yrow + 8, wt * vb);
                    }
                }
            }
        }
        __syncthreads();                         // s_x, s_sx, s_tm and s_red are rewritten by the next unit
    }
    pdl_trigger();
}

// K slices per row block: the fewest that still give about two CTA units per
// SM, with each slice a whole number of 64-k steps.
int q_choose_ks(const ExpertArgs& a, int K, int RB) {
    const long long P = (long long)a.T * a.k;
    const long long chunks = std::min<long long>(a.E, P) + P / kQTok;
    const long long want = 2LL * device_info().sm_count;
    int best = 1;
    for (int ks = 1; ks <= kQWarps; ks <<= 1) {
        if (K % (kQStepK * ks)) break;
        best = ks;
        const long long units = chunks * ((RB + (kQWarps / ks) - 1) / (kQWarps / ks));
        if (units >= want) break;
    }
    return best;
}

template <int FMT, int MODE, int KS>
cudaError_t run_q4(const ExpertArgs& a, int K, bool pdl, cudaStream_t s) {
    const QLayout L = q_layout(FMT, K);
    auto kern = k_gemv_q4<FMT, MODE, KS>;
    cudaError_t e = ensure_smem(kern, (size_t)L.total);
    if (e != cudaSuccess) return e;
    const int grid = device_info().sm_count * 2;
    return launch_k(kern, dim3(grid), dim3(kQWarps * 32), (size_t)L.total, s, pdl, a);
}

template <int FMT, int MODE>
cudaError_t run_q4_ks(const ExpertArgs& a, int K, int RB, bool pdl, cudaStream_t s) {
    switch (q_choose_ks(a, K, RB)) {
        case 1: return run_q4<FMT, MODE, 1>(a, K, pdl, s);
        case 2: return run_q4<FMT, MODE, 2>(a, K, pdl, s);
        case 4: return run_q4<FMT, MODE, 4>(a, K, pdl, s);
        default: return run_q4<FMT, MODE, 8>(a, K, pdl, s);
    }
}

template <int FMT>
cudaError_t q4_up(const ExpertArgs& a, bool pdl, cudaStream_t s) {
    if (a.H > kQMaxK) return cudaErrorNotSupported;
    if (a.act == 0) return run_q4_ks<FMT, kQUpSwiglu>(a, a.H, a.I / 8, pdl, s);
    return run_q4_ks<FMT, kQUpRelu2>(a, a.H, a.I / 16, pdl, s);
}

template <int FMT>
cudaError_t q4_down(const ExpertArgs& a, bool pdl, cudaStream_t s) {
    if (a.I > kQMaxK) return cudaErrorNotSupported;
    return run_q4_ks<FMT, kQDown>(a, a.I, a.H / 16, pdl, s);
}

}  // namespace

cudaError_t launch_gemv_q4_up(const ExpertArgs& a, bool pdl, cudaStream_t s) {
    if (gemv_q4t_fits(a, false)) return launch_gemv_q4t_up(a, pdl, s);
    if (a.fmt == kQAffine) return q4_up<kQAffine>(a, pdl, s);
    if (a.fmt == kQNvfp4) return q4_up<kQNvfp4>(a, pdl, s);
    return cudaErrorNotSupported;
}

cudaError_t launch_gemv_q4_down(const ExpertArgs& a, bool pdl, cudaStream_t s) {
    if (gemv_q4t_fits(a, true)) return launch_gemv_q4t_down(a, pdl, s);
    if (a.fmt == kQAffine) return q4_down<kQAffine>(a, pdl, s);
    if (a.fmt == kQNvfp4) return q4_down<kQNvfp4>(a, pdl, s);
    return cudaErrorNotSupported;
}

}  // namespace moe
