// Decode-sized grouped GEMV over affine 4-bit experts, dequantised in
// registers.
//
// Weight format (MLX-style affine, as TensorFold pull #1492 "What" names
// it): codes (E, N, K/8) uint32 with 8 nibbles per word, low nibble = lowest
// k; scale and bias (E, N, K/64) bf16; w[n][k] = scale[n][k/64] * q + bias.
//
// At one to a few tokens per expert the step is a stream of codes from HBM
// (half a byte per weight).  One warp owns 16 weight rows over the whole of K
// and keeps an 8-deep ring of code words in flight.  Each lane turns its
// nibbles into the bf16 value 128 + q with a mask-and-or (exact), and the
// legacy m16n8k16 tensor-core MMA forms, per group of 64 k,
//     Sq[r][n] = sum_k (128 + q[r][k]) * x[n][k]     and   Sx[n] = sum_k x[n][k]
// (Sx from an all-ones A operand on the same x fragments).  The group's scale
// and bias are then applied in fp32:
//     sum_k w[r][k] x[n][k] = s * Sq + (b - 128 s) * Sx.
// The MMA is only a dot-product engine here (N = 8 token columns); tensor
// throughput does not bound the kernel (as measured it is issue-bound, about
// four instructions per weight).
//
// Within one MMA the k order is free as long as A and B agree: a lane's word
// of 8 nibbles covers k0..k0+7, and the A slots (2t, 2t+1) / (2t+8, 2t+9) of
// the first MMA take k0+0/k0+4 and k0+1/k0+5, those of the second k0+2/k0+6 and
// k0+3/k0+7; the x fragments are permuted the same way with byte permutes.
//
// Rows of a unit: SwiGLU puts 8 gate rows (i0..i0+7) in MMA rows 0..7 and the
// matching up rows (I+i0..) in rows 8..15, so each lane holds gate and up of
// the same (column, token) and the activation needs no exchange; relu^2 and
// the down projection take 16 consecutive rows.
//
//   up   (SwiGLU): h[slot, i] = bf16_rn(silu(g) * u)
//   up   (relu^2): h[slot, i] = bf16_rn(relu(u)^2)
//   down:          y_acc[t, n] += w[pair] * (W2[e][n] . h[slot])   (fp32 atomics;
//                  a plain store per plan slot under the ordered combine)
//
// A CTA of 4 warps takes a unit (active expert, chunk of <= 8 of its tokens,
// 4 consecutive 16-row blocks -- one per warp): the chunk's token rows are
// copied into shared memory once by cp.async while the warps' code rings are
// already in flight, and the warps meet at one barrier per unit.
#include "common.cuh"
#include "internal.h"
#include "launch.h"

namespace moe {
namespace {

constexpr int kA4Warps = 4;               // warps per CTA (independent)
constexpr int kA4Tok = 8;                 // tokens per unit (the MMA's N)
constexpr int kA4Ring = 8;                // groups of codes in flight per warp
constexpr uint32_t kOnes = 0x3F803F80u;   // bf16x2 (1, 1)

enum { kA4UpSwiglu = 0, kA4UpRelu2 = 1, kA4Down = 2 };

MOE_DEV void mma_bf16_16816(float* c, uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3, uint32_t b0,
                            uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};\n"
        : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// Nibbles j and j+4 of v as the bf16 pair (128 + q_j, 128 + q_{j+4}): exact.
MOE_DEV uint32_t nib_pair(uint32_t v, int j) { return ((v >> (4 * j)) & 0x000F000Fu) | 0x43004300u; }

MOE_DEV uint32_t prmt(uint32_t a, uint32_t b, uint32_t sel) {
    uint32_t r;
    asm("prmt.b32 %0, %1, %2, %3;" : "=r"(r) : "r"(a), "r"(b), "r"(sel));
    return r;
}

MOE_DEV uint2 ld_codes(const uint32_t* p, uint64_t pol) {
    uint2 r;
    asm volatile("ld.global.nc.L1::no_allocate.L2::cache_hint.v2.u32 {%0,%1}, [%2], %3;"
                 : "=r"(r.x), "=r"(r.y)
                 : "l"(p), "l"(pol));
    return r;
}

MOE_DEV uint32_t ld_u16(const uint16_t* p) {
    unsigned short v;
    asm volatile("ld.global.nc.u16 %0, [%1];" : "=h"(v) : "l"(p));
    return v;
}

MOE_DEV void cp_async16(void* smem, const void* gmem) {
    const uint32_t sa = static_cast<uint32_t>(__cvta_generic_to_shared(smem));
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(sa), "l"(gmem) : "memory");
}

// Shared-memory row stride of the token tile, in bf16: K + 8 keeps the eight
// token rows of one LDS.128 phase on different banks.
MOE_DEV int xs_stride(int K) { return K + 8; }

template <int MODE>
__global__ void __launch_bounds__(kA4Warps * 32, 4) k_gemv_a4(ExpertArgs a) {
    extern __shared__ __align__(16) uint16_t s_x[];   // (8, K + 8) bf16: this unit's token rows
    __shared__ int s_base[257];
    pdl_wait();
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int g = lane >> 2, tq = lane & 3;
    const bool down = MODE == kA4Down;
    const int K = down ? a.I : a.H;              // reduction length
    const int N = down ? a.H : (MODE == kA4UpSwiglu ? 2 * a.I : a.I);   // weight rows per expert
    const int G = K / 64;                        // groups per row
    const int RB = MODE == kA4UpSwiglu ? a.I / 8 : N / 16;             // 16-row blocks per expert
    const int RQ = (RB + kA4Warps - 1) / kA4Warps;                      // blocks of kA4Warps row blocks
    const int XS = xs_stride(K);
    const uint32_t* codes = reinterpret_cast<const uint32_t*>(down ? a.w2 : a.w1);
    const uint16_t* wsc = down ? a.w2_scale : a.w1_scale;
    const uint16_t* wbi = down ? a.w2_bias : a.w1_bias;

    // CTA units per expert = token chunks x row-block quads; prefix over experts
    if (warp == 0) {
        int run = 0;
        for (int e0 = 0; e0 < a.E; e0 += 32) {
            const int e = e0 + lane;
            const int nu = (e < a.E && e != a.skip) ? (a.counts[e] + kA4Tok - 1) / kA4Tok * RQ : 0;
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
    const size_t wpr = (size_t)K / 8;            // code words per row

    for (int u = blockIdx.x; u < total; u += gridDim.x) {
        int lo = 0, hi = a.E;                    // expert: last e with s_base[e] <= u
        while (lo < hi) {
            const int mid = (lo + hi + 1) >> 1;
            if (s_base[mid] <= u) lo = mid;
            else hi = mid - 1;
        }
        const int e = lo;
        const int cnt = a.counts[e], off = a.offsets[e];
        const int nch = (cnt + kA4Tok - 1) / kA4Tok;
        const int local = u - s_base[e];
        const int rq = local / nch, ch = local % nch;
        const int nt = min(kA4Tok, cnt - ch * kA4Tok);
        const int slot0 = off + ch * kA4Tok;
        const int rb = rq * kA4Warps + warp;     // this warp's row block
        const bool active = rb < RB;
        // weight row (within the expert) of MMA row r
        auto wrow = [&](int r) -> int {
            if (MODE == kA4UpSwiglu) return r < 8 ? rb * 8 + r : a.I + rb * 8 + (r - 8);
            return rb * 16 + r;
        };
        const size_t ebase = (size_t)e * N;
        const uint32_t* p0 = codes + (ebase + wrow(g)) * wpr + 2 * tq;       // MMA row g
        const uint32_t* p1 = codes + (ebase + wrow(g + 8)) * wpr + 2 * tq;   // MMA row g + 8
        // lanes 0..15 fetch the scales of rows 0..15, lanes 16..31 the biases
        const uint16_t* psb = (lane < 16 ? wsc : wbi) + (ebase + wrow(lane & 15)) * G;

        // the code ring goes out first; the token rows follow through cp.async
        uint2 q0[kA4Ring], q1[kA4Ring];
        uint32_t sb[kA4Ring];
        if (active) {
#pragma unroll
            for (int d = 0; d < kA4Ring; ++d) {
                if (d < G) {
                    q0[d] = ld_codes(p0 + 8 * d, pol);
                    q1[d] = ld_codes(p1 + 8 * d, pol);
                    sb[d] = ld_u16(psb + d);
                }
            }
        }
        const int cpr = K / 8;                   // 16-byte pieces per token row
        for (int i = threadIdx.x; i < nt * cpr; i += blockDim.x) {
            const int n = i / cpr, pc = i - n * cpr;
            const uint16_t* src = down ? a.h + (size_t)(slot0 + n) * a.I
                                       : a.x + (size_t)(a.perm[slot0 + n] / a.k) * a.H;
            cp_async16(s_x + n * XS + 8 * pc, src + 8 * pc);
        }
        asm volatile("cp.async.commit_group;\ncp.async.wait_all;" ::: "memory");
        __syncthreads();

        if (active) {
            const uint16_t* xr = s_x + g * XS + 16 * tq;
            const bool has_tok = g < nt;
            float acc[4] = {0.f, 0.f, 0.f, 0.f};
            for (int cb = 0; cb < G; cb += kA4Ring) {
#pragma unroll
                for (int d = 0; d < kA4Ring; ++d) {
                    const int c = cb + d;
                    if (c < G) {
                        uint4 xv[2];
                        if (has_tok) {
                            xv[0] = *reinterpret_cast<const uint4*>(xr + 64 * c);
                            xv[1] = *reinterpret_cast<const uint4*>(xr + 64 * c + 8);
                        } else {
                            xv[0] = make_uint4(0, 0, 0, 0);
                            xv[1] = make_uint4(0, 0, 0, 0);
                        }
                        float cg[4] = {0.f, 0.f, 0.f, 0.f}, cx[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
                        for (int w2 = 0; w2 < 2; ++w2) {
                            const uint4 xw = xv[w2];
                            const uint32_t b00 = prmt(xw.x, xw.z, 0x5410), b01 = prmt(xw.x, xw.z, 0x7632);
                            const uint32_t b10 = prmt(xw.y, xw.w, 0x5410), b11 = prmt(xw.y, xw.w, 0x7632);
                            const uint32_t v0 = w2 ? q0[d].y : q0[d].x;   // MMA row g
                            const uint32_t v1 = w2 ? q1[d].y : q1[d].x;   // MMA row g + 8
                            mma_bf16_16816(cx, kOnes, kOnes, kOnes, kOnes, b00, b01);
                            mma_bf16_16816(cx, kOnes, kOnes, kOnes, kOnes, b10, b11);
                            mma_bf16_16816(cg, nib_pair(v0, 0), nib_pair(v1, 0), nib_pair(v0, 1), nib_pair(v1, 1),
                                           b00, b01);
                            mma_bf16_16816(cg, nib_pair(v0, 2), nib_pair(v1, 2), nib_pair(v0, 3), nib_pair(v1, 3),
                                           b10, b11);
                        }
                        const float s0 = bf16f((uint16_t)__shfl_sync(0xffffffffu, sb[d], g));
                        const float s1 = bf16f((uint16_t)__shfl_sync(0xffffffffu, sb[d], g + 8));
                        const float c0 = bf16f((uint16_t)__shfl_sync(0xffffffffu, sb[d], 16 + g));
                        const float c1 = bf16f((uint16_t)__shfl_sync(0xffffffffu, sb[d], 24 + g));
                        const float bb0 = fmaf(-128.f, s0, c0), bb1 = fmaf(-128.f, s1, c1);   // exact
                        acc[0] = fmaf(s0, cg[0], fmaf(bb0, cx[0], acc[0]));
                        acc[1] = fmaf(s0, cg[1], fmaf(bb0, cx[1], acc[1]));
                        acc[2] = fmaf(s1, cg[2], fmaf(bb1, cx[2], acc[2]));
                        acc[3] = fmaf(s1, cg[3], fmaf(bb1, cx[3], acc[3]));
                        if (c + kA4Ring < G) {                       // refill this ring slot
                            q0[d] = ld_codes(p0 + 8 * (c + kA4Ring), pol);
                            q1[d] = ld_codes(p1 + 8 * (c + kA4Ring), pol);
                            sb[d] = ld_u16(psb + c + kA4Ring);
                        }
                    }
                }
            }
            // acc[0], acc[1]: MMA row g, tokens 2tq, 2tq+1; acc[2], acc[3]: row g + 8
#pragma unroll
            for (int jn = 0; jn < 2; ++jn) {
                const int n = 2 * tq + jn;
                if (n >= nt) continue;
                const int slot = slot0 + n;
                if (MODE == kA4UpSwiglu) {
                    float gv = acc[jn], uv = acc[2 + jn];
                    clamp_swiglu(gv, uv, a.swiglu_limit);
                    a.h[(size_t)slot * a.I + rb * 8 + g] = f2bf16(act_swiglu(gv, uv));
                } else if (MODE == kA4UpRelu2) {
                    a.h[(size_t)slot * a.I + rb * 16 + g] = f2bf16(act_relu2(acc[jn]));
                    a.h[(size_t)slot * a.I + rb * 16 + g + 8] = f2bf16(act_relu2(acc[2 + jn]));
                } else {
                    const int pair = a.perm[slot];
                    const float wt = a.topk_w[pair];
                    if (a.ordered) {
                        float* orow = a.y_acc + (size_t)slot * a.H + rb * 16 + g;
                        orow[0] = wt * acc[jn];
                        orow[8] = wt * acc[2 + jn];
                    } else {
                        float* yrow = a.y_acc + (size_t)(pair / a.k) * a.H + rb * 16 + g;
                        atomicAdd(yrow, wt * acc[jn]);
                        atomicAdd(yrow + 8, wt * acc[2 + jn]);
                    }
                }
            }
        }
        __syncthreads();                         // s_x is rewritten by the next unit
    }
    pdl_trigger();
}

// CTA units: (distinct experts + P / 8) token chunks at most, times row-block quads.
int a4_grid(const ExpertArgs& a, int row_blocks) {
    const long long P = (long long)a.T * a.k;
    const long long chunks = std::min<long long>(a.E, P) + P / kA4Tok;
    const long long ctas = chunks * ((row_blocks + kA4Warps - 1) / kA4Warps);
    const long long cap = (long long)device_info().sm_count * 8;
    return (int)std::max<long long>(1, std::min(ctas, cap));
}

size_t a4_smem(int K) { return (size_t)kA4Tok * (K + 8) * sizeof(uint16_t); }

template <int MODE>
cudaError_t run_a4(const ExpertArgs& a, int K, int row_blocks, bool pdl, cudaStream_t s) {
    const size_t smem = a4_smem(K);
    cudaError_t e = ensure_smem(k_gemv_a4<MODE>, smem);
    if (e != cudaSuccess) return e;
    return launch_k(k_gemv_a4<MODE>, dim3(a4_grid(a, row_blocks)), dim3(kA4Warps * 32), smem, s, pdl, a);
}

}  // namespace

// The token tile (8 rows of K bf16) must fit in shared memory next to three
// other CTAs: K <= 8192.
cudaError_t launch_gemv_affine_up(const ExpertArgs& a, bool pdl, cudaStream_t s) {
    if (a.H > 8192) return cudaErrorNotSupported;
    if (a.act == 0) return run_a4<kA4UpSwiglu>(a, a.H, a.I / 8, pdl, s);
    return run_a4<kA4UpRelu2>(a, a.H, a.I / 16, pdl, s);
}

cudaError_t launch_gemv_affine_down(const ExpertArgs& a, bool pdl, cudaStream_t s) {
    if (a.I > 8192) return cudaErrorNotSupported;
    return run_a4<kA4Down>(a, a.I, a.H / 16, pdl, s);
}

}  // namespace moe
