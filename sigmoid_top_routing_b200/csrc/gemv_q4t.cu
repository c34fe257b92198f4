// Decode-sized grouped GEMV over 4-bit experts with the weight codes streamed
// by TMA: MLX-style affine 4-bit (group 64) and NVFP4 (ModelOpt layout).
//
// Formats and arithmetic are those of the register-dequant GEMV (gemv_q4.cu):
//   affine (TensorFold pull #1492, "What"): w = scale * q + bias per group of
//     64 k; a nibble pair becomes the exact bf16 pair (128 + q) and per group
//     and row  sum_k w x = s * sum_k (128 + q) x + (b - 128 s) * sum_k x.
//   NVFP4 (TensorFold issue #548, the checkpoint layout): w = e2m1 * e4m3 * g;
//     e2m1 * e4m3 is formed exactly in f16 and the token rows are staged in f16
//     after an exact per-token power-of-two scale.
// What changes is how the codes reach the tensor cores.  At a few tokens per
// expert the step is a stream of codes from HBM; here that stream is a ring of
// shared-memory stages filled by cp.async.bulk.tensor (TMA) from one producer
// warp, so the load path neither spends registers on loads in flight nor L1
// wavefronts on 8-byte pieces of 128-byte lines.
//
// Work.  A unit is (active expert, chunk of <= 8 of its tokens, 128 weight
// rows): for SwiGLU 64 features (their gate and up rows), else 128 rows.  A
// stage is the unit's 128 rows x 512 k: four 64-row x 128-byte code boxes
// (128-byte swizzle) and the rows' scales (NVFP4: 32 e4m3 bytes a row;
// affine: 8 bf16 scales and 8 biases a row).  Each CTA (one or two per SM) takes a
// contiguous range of units in (expert, chunk, row block) order, so its
// consecutive units share their token rows, which are staged in shared memory
// only when the (expert, chunk) changes.  Eight consumer warps each own one
// 16-row m16n8k16 MMA tile of the stage; a lane reads 8 bytes (16 k) of each
// of its two rows per 64-k step.  MMA row g of a warp is stage row
// sigma(g) = 2g (g < 4) or 2(g - 4) + 1 within its group of 8, so the 16 lanes
// of one 8-byte shared-memory load phase fall on 16 distinct banks under the
// swizzle (rows 0, 2, 4, 6 of a phase XOR their 16-byte chunks with distinct
// even values).
//
// Every wait on a stage barrier is bounded; on expiry the kernel records
// device error 2, raises the CTA's abort flag, drains the copies it issued and
// returns.
#include <cuda_fp16.h>

#include <algorithm>

#include "common.cuh"
#include "internal.h"
#include "launch.h"
#include "quant.cuh"
#include "sm100.cuh"
#include "tmap.h"

namespace moe {
namespace {

using namespace sm100;

constexpr int kTW = 8;                                   // consumer warps
constexpr int kTThreads = (kTW + 1) * 32;                // + the TMA producer warp
constexpr int kTTok = 8;                                 // tokens per unit (the MMA's N)
constexpr int kTStageK = 512;                            // k per stage
constexpr int kTBoxRows = 64;                            // rows per code box
constexpr int kTCodeBox = kTBoxRows * 128;               // bytes of one code box (256 k x 64 rows)
constexpr int kTCodeStage = 4 * kTCodeBox;               // [k half][row half] boxes
constexpr int kTScaleStage = 4096;                       // NVFP4 2 x 64 x 32 B; affine 2 x (2 x 64 x 16 B)
constexpr uint32_t kTStageBytes = kTCodeStage + kTScaleStage;

enum { kTUpSwiglu = 0, kTUpRelu2 = 1, kTDown = 2 };
enum { kTAffine = 1, kTNvfp4 = 2 };                      // the library's weight format codes

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

MOE_DEV uint2 lds64(uint32_t addr) {
    uint2 v;
    asm volatile("ld.shared.v2.u32 {%0,%1}, [%2];" : "=r"(v.x), "=r"(v.y) : "r"(addr));
    return v;
}
MOE_DEV uint4 lds128(uint32_t addr) {
    uint4 v;
    asm volatile("ld.shared.v4.u32 {%0,%1,%2,%3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(addr));
    return v;
}

// k of the staged token rows: K rounded up to whole stages (zeros past K).
MOE_DEV __host__ int t_kpad(int K) { return (K + kTStageK - 1) / kTStageK * kTStageK; }
// Shared-memory row stride of the token tile, in 16-bit elements: the pad
// puts the two rows of one 16-byte load phase on distinct bank groups.
MOE_DEV __host__ int t_xstride(int K) { return t_kpad(K) + 8; }

struct TLayout {          // dynamic shared memory of one CTA (byte offsets from a 1024-aligned base)
    int codes, scales, x, sx, bars, total;
};

MOE_DEV __host__ TLayout t_layout(int fmt, int K, int stages) {
    TLayout L;
    L.codes = 0;
    L.scales = L.codes + stages * kTCodeStage;
    L.x = L.scales + stages * kTScaleStage;
    int off = L.x + kTTok * t_xstride(K) * 2;
    L.sx = off;                                          // affine: sum_k x per (group, token), [G][8] fp32
    if (fmt == kTAffine) off += (t_kpad(K) / 64) * kTTok * 4;
    L.bars = (off + 7) & ~7;
    L.total = L.bars + (2 * stages) * 8 + 1024;          // + alignment slack of the base
    return L;
}

// STG stages per CTA: 4 with one CTA per SM, 2 with two (the same bytes in flight per SM)
template <int FMT, int MODE, int STG>
__global__ void __launch_bounds__(kTThreads, 4 / STG)
    k_gemv_q4t(const __grid_constant__ CUtensorMap tmC, const __grid_constant__ CUtensorMap tmS,
               const __grid_constant__ CUtensorMap tmB, ExpertArgs a, uint32_t wait_limit) {
    extern __shared__ unsigned char t_smem_raw[];
    unsigned char* sm =
        reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(t_smem_raw) + 1023) & ~uintptr_t(1023));
    __shared__ int s_base[257];
    __shared__ float s_tm[kTTok];                        // per-token output multiplier (NVFP4)
    __shared__ int s_abort;
    constexpr bool down = MODE == kTDown;
    const int K = down ? a.I : a.H;
    const int N = down ? a.H : (MODE == kTUpSwiglu ? 2 * a.I : a.I);    // weight rows per expert
    const int NRQ = MODE == kTUpSwiglu ? a.I / 64 : N / 128;             // units of rows per expert
    const int nst = t_kpad(K) / kTStageK;                               // stages per unit
    const TLayout L = t_layout(FMT, K, STG);
    const int XS = t_xstride(K);
    uint16_t* s_x = reinterpret_cast<uint16_t*>(sm + L.x);
    float* s_sx = reinterpret_cast<float*>(sm + L.sx);
    uint64_t* full = reinterpret_cast<uint64_t*>(sm + L.bars);
    uint64_t* empty = full + STG;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    if (threadIdx.x == 0) {
        for (int s = 0; s < STG; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], kTW);
        }
        s_abort = 0;
        fence_mbar_init();
    }
    if (warp == kTW && lane == 0) {
        tma_prefetch_desc(&tmC);
        tma_prefetch_desc(&tmS);
        if (FMT == kTAffine) tma_prefetch_desc(&tmB);
    }
    pdl_wait();
    // units per expert = token chunks x row blocks; prefix over experts
    if (warp == 0) {
        int run = 0;
        for (int e0 = 0; e0 < a.E; e0 += 32) {
            const int e = e0 + lane;
            const int nu = (e < a.E && e != a.skip) ? (a.counts[e] + kTTok - 1) / kTTok * NRQ : 0;
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
    const int ubeg = (int)((long long)total * blockIdx.x / gridDim.x);
    const int uend = (int)((long long)total * (blockIdx.x + 1) / gridDim.x);
    const volatile int* abort_flag = &s_abort;

    // unit u -> expert, token chunk, row block (row block innermost)
    auto unit_of = [&](int u, int& e, int& ch, int& rq) {
        int lo = 0, hi = a.E;
        while (lo < hi) {
            const int mid = (lo + hi + 1) >> 1;
            if (s_base[mid] <= u) lo = mid;
            else hi = mid - 1;
        }
        e = lo;
        const int local = u - s_base[e];
        ch = local / NRQ;
        rq = local - ch * NRQ;
    };
    // first weight row (global, in the E_w * N row space) of row half rh of a unit
    auto half_row = [&](int e, int rq, int rh) -> int {
        if (MODE == kTUpSwiglu) return e * N + (rh ? a.I : 0) + 64 * rq;
        return e * N + 128 * rq + 64 * rh;
    };

    if (warp == kTW) {
        // ---------------------------------------------------------------- TMA producer
        if (lane == 0) {
            int s = 0;
            uint32_t ph = 0;
            uint32_t used = 0, par = 0;                  // slots issued, and the parity of their last issue
            bool ok = true;
            for (int u = ubeg; u < uend && ok; ++u) {
                int e, ch, rq;
                unit_of(u, e, ch, rq);
                const int r0 = half_row(e, rq, 0), r1 = half_row(e, rq, 1);
                for (int st = 0; st < nst; ++st) {
                    if (!mbar_wait(&empty[s], ph ^ 1, abort_flag, wait_limit)) { ok = false; break; }
                    mbar_arrive_expect_tx(&full[s], kTStageBytes);
                    unsigned char* cs = sm + L.codes + s * kTCodeStage;
                    unsigned char* ss = sm + L.scales + s * kTScaleStage;
                    const int kb = st * kTStageK / 2;    // code byte offset of the stage
#pragma unroll
                    for (int kh = 0; kh < 2; ++kh) {
                        tma_load_2d(cs + (2 * kh + 0) * kTCodeBox, &tmC, kb + 128 * kh, r0, &full[s]);
                        tma_load_2d(cs + (2 * kh + 1) * kTCodeBox, &tmC, kb + 128 * kh, r1, &full[s]);
                    }
                    if (FMT == kTNvfp4) {
                        tma_load_2d(ss, &tmS, st * (kTStageK / 16), r0, &full[s]);
                        tma_load_2d(ss + 2048, &tmS, st * (kTStageK / 16), r1, &full[s]);
                    } else {
                        tma_load_2d(ss, &tmS, st * (kTStageK / 64), r0, &full[s]);
                        tma_load_2d(ss + 1024, &tmS, st * (kTStageK / 64), r1, &full[s]);
                        tma_load_2d(ss + 2048, &tmB, st * (kTStageK / 64), r0, &full[s]);
                        tma_load_2d(ss + 3072, &tmB, st * (kTStageK / 64), r1, &full[s]);
                    }
                    used |= 1u << s;
                    par = (par & ~(1u << s)) | (ph << s);
                    if (++s == STG) { s = 0; ph ^= 1; }
                }
            }
            if (!ok) {
                report_error(a.err, kErrWaitExpired);
                s_abort = 1;
            }
            // no copy of ours may still be in flight when the CTA exits
            for (int q = 0; q < STG; ++q)
                if (used & (1u << q)) mbar_wait(&full[q], (par >> q) & 1u, nullptr, wait_limit);
        }
    } else {
        // ---------------------------------------------------------------- consumers
        const int g = lane >> 2, tq = lane & 3;
        const int sg = g < 4 ? 2 * g : 2 * (g - 4) + 1;  // stage row (within 8) of MMA row g
        // MMA rows g and g + 8 of this warp: row half and row within the half
        int rh0, rr0, rh1, rr1;
        if (MODE == kTUpSwiglu) {
            rh0 = 0; rr0 = 8 * warp + sg;                // gate row of feature 8 warp + sg
            rh1 = 1; rr1 = 8 * warp + sg;                // its up row
        } else {
            rh0 = rh1 = warp >> 2;
            rr0 = 16 * (warp & 3) + sg;
            rr1 = rr0 + 8;
        }
        const uint32_t codes_u32 = smem_u32(sm + L.codes);
        const uint32_t scales_u32 = smem_u32(sm + L.scales);
        const uint32_t xr_u32 = smem_u32(s_x + g * XS + 16 * tq);
        const uint32_t c_row0 = (rh0 * kTBoxRows + rr0) * 128 + 8 * (tq & 1);
        const uint32_t c_row1 = (rh1 * kTBoxRows + rr1) * 128 + 8 * (tq & 1);
        const int cq = tq >> 1;
        // scale rows of MMA rows g and g + 8 within a stage's scale area
        const uint32_t s_row0 = FMT == kTNvfp4 ? (rh0 * kTBoxRows + rr0) * 32 : (rh0 * kTBoxRows + rr0) * 16;
        const uint32_t s_row1 = FMT == kTNvfp4 ? (rh1 * kTBoxRows + rr1) * 32 : (rh1 * kTBoxRows + rr1) * 16;
        const float* wglob = down ? a.w2_global : a.w1_global;
        int s = 0;
        uint32_t ph = 0;
        bool dead = false;
        int staged_e = -1, staged_ch = -1;
        for (int u = ubeg; u < uend; ++u) {
            int e, ch, rq;
            unit_of(u, e, ch, rq);
            const int cnt = a.counts[e], off = a.offsets[e];
            const int nt = min(kTTok, cnt - ch * kTTok);
            const int slot0 = off + ch * kTTok;
            if (e != staged_e || ch != staged_ch) {
                // ---- stage the chunk's token rows (one warp per row), zeros past K
                named_bar(1, kTW * 32);          // every consumer is done with the previous rows
                for (int n = warp; n < nt; n += kTW) {
                    const uint16_t* src = down ? a.h + (size_t)(slot0 + n) * a.I
                                               : a.x + (size_t)(a.perm[slot0 + n] / a.k) * a.H;
                    const uint4* s4 = reinterpret_cast<const uint4*>(src);
                    uint4* d4 = reinterpret_cast<uint4*>(s_x + n * XS);
                    const int nc = K / 8, ncp = t_kpad(K) / 8;   // 8-k chunks of the row, and with the pad
                    if (FMT == kTNvfp4) {
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
                            frexpf(amax, &e2);
                            ex = max(-100, min(100, e2 - 15));
                        }
                        const float mul = __int_as_float((127 - ex) << 23);
                        if (lane == 0) s_tm[n] = __int_as_float((127 + ex) << 23) * wglob[e];
                        for (int c = lane; c < ncp; c += 32) {
                            uint4 o = make_uint4(0u, 0u, 0u, 0u);
                            if (c < nc) {
                                const uint4 v = ld_nc(s4 + c);
                                const uint32_t w4[4] = {v.x, v.y, v.z, v.w};
                                uint32_t o4[4];
#pragma unroll
                                for (int i = 0; i < 4; ++i) {
                                    const __half2 h = __floats2half2_rn(bf16lo(w4[i]) * mul, bf16hi(w4[i]) * mul);
                                    o4[i] = *reinterpret_cast<const uint32_t*>(&h);
                                }
                                o = make_uint4(o4[0], o4[1], o4[2], o4[3]);
                            }
                            d4[c] = o;
                        }
                    } else {
                        // reorder each 8-k chunk to (x0 x4 x1 x5 x2 x6 x3 x7) and sum per group of 64
                        for (int c0 = 0; c0 < ncp; c0 += 32) {
                            const int c = c0 + lane;
                            float part = 0.0f;
                            if (c < ncp) {
                                uint4 v = make_uint4(0u, 0u, 0u, 0u);
                                if (c < nc) v = ld_nc(s4 + c);
                                d4[c] = make_uint4(prmt(v.x, v.z, 0x5410), prmt(v.x, v.z, 0x7632),
                                                   prmt(v.y, v.w, 0x5410), prmt(v.y, v.w, 0x7632));
                                part = ((bf16lo(v.x) + bf16hi(v.x)) + (bf16lo(v.y) + bf16hi(v.y))) +
                                       ((bf16lo(v.z) + bf16hi(v.z)) + (bf16lo(v.w) + bf16hi(v.w)));
                            }
                            part += __shfl_xor_sync(0xffffffffu, part, 1);
                            part += __shfl_xor_sync(0xffffffffu, part, 2);
                            part += __shfl_xor_sync(0xffffffffu, part, 4);
                            if ((lane & 7) == 0 && c < ncp) s_sx[(c >> 3) * kTTok + n] = part;
                        }
                    }
                }
                named_bar(1, kTW * 32);
                staged_e = e;
                staged_ch = ch;
            }

            float acc[4] = {0.f, 0.f, 0.f, 0.f};
            for (int st = 0; st < nst; ++st) {
                if (!dead && !mbar_wait(&full[s], ph, abort_flag, wait_limit)) {
                    if (lane == 0) {
                        report_error(a.err, kErrWaitExpired);
                        s_abort = 1;
                    }
                    dead = true;
                }
                dead = __any_sync(0xffffffffu, dead);
                if (!dead) {
                    const uint32_t cs = codes_u32 + s * kTCodeStage;
                    const uint32_t ss = scales_u32 + s * kTScaleStage;
#pragma unroll
                    for (int kh = 0; kh < 2; ++kh) {
                        // this half-stage's scales for rows g and g + 8
                        uint4 nsc0, nsc1;                // NVFP4: 16 block-scale bytes per row
                        uint2 asc0, asc1, abi0, abi1;    // affine: 4 scales and 4 biases per row
                        if (FMT == kTNvfp4) {
                            nsc0 = lds128(ss + s_row0 + 16 * kh);
                            nsc1 = lds128(ss + s_row1 + 16 * kh);
                        } else {
                            asc0 = lds64(ss + s_row0 + 8 * kh);
                            asc1 = lds64(ss + s_row1 + 8 * kh);
                            abi0 = lds64(ss + 2048 + s_row0 + 8 * kh);
                            abi1 = lds64(ss + 2048 + s_row1 + 8 * kh);
                        }
                        const uint32_t cb = cs + kh * 2 * kTCodeBox;
#pragma unroll
                        for (int d = 0; d < 4; ++d) {
                            const uint32_t chunk = uint32_t((2 * d + cq) ^ sg) * 16;
                            const uint2 q0 = lds64(cb + c_row0 + chunk);
                            const uint2 q1 = lds64(cb + c_row1 + chunk);
                            const int kst = st * kTStageK + kh * 256 + 64 * d;   // k of this step
                            const uint4 xa = lds128(xr_u32 + 2 * kst);
                            const uint4 xb = lds128(xr_u32 + 2 * kst + 16);
                            if (FMT == kTNvfp4) {
                                const uint32_t w0 = d == 0 ? nsc0.x : d == 1 ? nsc0.y : d == 2 ? nsc0.z : nsc0.w;
                                const uint32_t w1 = d == 0 ? nsc1.x : d == 1 ? nsc1.y : d == 2 ? nsc1.z : nsc1.w;
                                // byte tq of each word: the block (4 step + tq) of rows g and g + 8
                                const uint32_t pairb = prmt(w0, w1, uint32_t(tq | ((4 + tq) << 4)));
                                const uint32_t s2 = e4m3x2_to_f16x2(pairb & 0xFFFFu);   // (row g, row g+8)
                                const uint32_t sgv = prmt(s2, s2, 0x1010), shv = prmt(s2, s2, 0x3232);
#pragma unroll
                                for (int j = 0; j < 2; ++j) {
                                    const uint4 xv = j ? xb : xa;
                                    uint32_t pa[4], pb[4];
                                    e2m1x8_to_f16(j ? q0.y : q0.x, pa);
                                    e2m1x8_to_f16(j ? q1.y : q1.x, pb);
#pragma unroll
                                    for (int i = 0; i < 4; ++i) {
                                        pa[i] = hmul2_u32(pa[i], sgv);
                                        pb[i] = hmul2_u32(pb[i], shv);
                                    }
                                    mma_f16_16816(acc, pa[0], pb[0], pa[1], pb[1], xv.x, xv.y);
                                    mma_f16_16816(acc, pa[2], pb[2], pa[3], pb[3], xv.z, xv.w);
                                }
                            } else {
                                float cg[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
                                for (int j = 0; j < 2; ++j) {
                                    const uint4 xv = j ? xb : xa;
                                    const uint32_t v = j ? q0.y : q0.x;   // MMA row g
                                    const uint32_t w = j ? q1.y : q1.x;   // MMA row g + 8
                                    mma_bf16_16816(cg, nib_pair(v, 0), nib_pair(w, 0), nib_pair(v, 1),
                                                   nib_pair(w, 1), xv.x, xv.y);
                                    mma_bf16_16816(cg, nib_pair(v, 2), nib_pair(w, 2), nib_pair(v, 3),
                                                   nib_pair(w, 3), xv.z, xv.w);
                                }
                                // group (4 kh + d) of the stage: scale and bias of rows g, g + 8
                                const uint32_t sw0 = d < 2 ? asc0.x : asc0.y, sw1 = d < 2 ? asc1.x : asc1.y;
                                const uint32_t bw0 = d < 2 ? abi0.x : abi0.y, bw1 = d < 2 ? abi1.x : abi1.y;
                                const float s0 = (d & 1) ? bf16hi(sw0) : bf16lo(sw0);
                                const float s1 = (d & 1) ? bf16hi(sw1) : bf16lo(sw1);
                                const float b0 = (d & 1) ? bf16hi(bw0) : bf16lo(bw0);
                                const float b1 = (d & 1) ? bf16hi(bw1) : bf16lo(bw1);
                                const float c0 = fmaf(-128.f, s0, b0), c1 = fmaf(-128.f, s1, b1);   // exact
                                const float2 sx = *reinterpret_cast<const float2*>(s_sx + (kst / 64) * kTTok + 2 * tq);
                                acc[0] = fmaf(s0, cg[0], fmaf(c0, sx.x, acc[0]));
                                acc[1] = fmaf(s0, cg[1], fmaf(c0, sx.y, acc[1]));
                                acc[2] = fmaf(s1, cg[2], fmaf(c1, sx.x, acc[2]));
                                acc[3] = fmaf(s1, cg[3], fmaf(c1, sx.y, acc[3]));
                            }
                        }
                    }
                }
                __syncwarp();
                if (lane == 0) mbar_arrive(&empty[s]);   // this warp is done with the stage
                if (++s == STG) { s = 0; ph ^= 1; }
            }
            if (dead) continue;
            // acc[0], acc[1]: MMA row g, tokens 2tq, 2tq + 1; acc[2], acc[3]: row g + 8
#pragma unroll
            for (int jn = 0; jn < 2; ++jn) {
                const int n = 2 * tq + jn;
                if (n >= nt) continue;
                const int slot = slot0 + n;
                float va = acc[jn], vb = acc[2 + jn];
                if (FMT == kTNvfp4) {
                    va *= s_tm[n];
                    vb *= s_tm[n];
                }
                if (MODE == kTUpSwiglu) {
                    clamp_swiglu(va, vb, a.swiglu_limit);
                    a.h[(size_t)slot * a.I + 64 * rq + rr0] = f2bf16(act_swiglu(va, vb));
                } else {
                    const int o0 = 128 * rq + 64 * rh0 + rr0, o1 = 128 * rq + 64 * rh1 + rr1;
                    if (MODE == kTUpRelu2) {
                        a.h[(size_t)slot * a.I + o0] = f2bf16(act_relu2(va));
                        a.h[(size_t)slot * a.I + o1] = f2bf16(act_relu2(vb));
                    } else {
                        const int pair = a.perm[slot];
                        const float wt = a.topk_w[pair];
                        if (a.ordered) {
                            float* orow = a.y_acc + (size_t)slot * a.H;
                            orow[o0] = wt * va;
                            orow[o1] = wt * vb;
                        } else {
                            float* yrow = a.y_acc + (size_t)(pair / a.k) * a.H;
                            atomicAdd(yrow + o0, wt * va);
                            atomicAdd(yrow + o1, wt * vb);
                        }
                    }
                }
            }
        }
    }
    __syncthreads();
    pdl_trigger();
}

template <int FMT, int MODE, int STG>
cudaError_t run_q4t(const ExpertArgs& a, int K, int N, bool pdl, cudaStream_t s) {
    const void* codes = MODE == kTDown ? a.w2 : a.w1;
    const void* scale = MODE == kTDown ? (const void*)a.w2_scale : (const void*)a.w1_scale;
    const void* bias = MODE == kTDown ? (const void*)a.w2_bias : (const void*)a.w1_bias;
    const uint64_t rows = (uint64_t)a.E_w * N;
    CUtensorMap tC, tS, tB;
    cudaError_t e = make_tmap_2d(&tC, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, codes, (uint64_t)K / 2, rows, 128,
                                 kTBoxRows, true);
    if (e != cudaSuccess) return e;
    if (FMT == kTNvfp4) {
        e = make_tmap_2d(&tS, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, scale, (uint64_t)K / 16, rows, kTStageK / 16,
                         kTBoxRows, false);
        tB = tS;
    } else {
        e = make_tmap_2d(&tS, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, scale, (uint64_t)K / 64, rows, kTStageK / 64,
                         kTBoxRows, false);
        if (e == cudaSuccess)
            e = make_tmap_2d(&tB, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, bias, (uint64_t)K / 64, rows,
                             kTStageK / 64, kTBoxRows, false);
    }
    if (e != cudaSuccess) return e;
    const TLayout L = t_layout(FMT, K, STG);
    auto kern = k_gemv_q4t<FMT, MODE, STG>;
    if ((e = ensure_smem(kern, (size_t)L.total)) != cudaSuccess) return e;
    return launch_k(kern, dim3((4 / STG) * device_info().sm_count), dim3(kTThreads), (size_t)L.total, s, pdl, tC,
                    tS, tB, a, sm100::kWaitLimit);
}

// Units of this projection (an estimate: about one chunk per active expert
// plus one per 8 of the batch's pairs).
long long q4t_units(const ExpertArgs& a, bool down) {
    const int rows_unit = (!down && a.act == 0) ? 64 : 128;   // SwiGLU: 64 features (gate + up rows)
    const int feats = down ? a.H : a.I;
    const long long P = (long long)a.T * a.k;
    const long long chunks = std::min<long long>(a.E, P) + P / kTTok;
    return chunks * (feats / rows_unit);
}

// Two CTAs per SM (2 stages each) when there are >= 4 units per CTA and both fit, else one (4 stages).
template <int FMT, int MODE>
cudaError_t run_q4t_pick(const ExpertArgs& a, int K, int N, bool pdl, cudaStream_t s) {
    // (two CTAs only when both fit in one SM's shared memory with their static
    // arrays and the 1 KB the hardware reserves per CTA)
    const DeviceInfo& di = device_info();
    const bool two_fit = 2 * (t_layout(FMT, K, 2).total + 2048 + 1024) <= di.smem_per_sm;
    if (two_fit && q4t_units(a, MODE == kTDown) >= 8LL * di.sm_count) return run_q4t<FMT, MODE, 2>(a, K, N, pdl, s);
    return run_q4t<FMT, MODE, 4>(a, K, N, pdl, s);
}

}  // namespace

// Whether the TMA-fed GEMV takes this projection: whole 128-row units, scale
// rows that TMA can address, and the token tile within shared memory.
bool gemv_q4t_fits(const ExpertArgs& a, bool down) {
    if (a.fmt != kTAffine && a.fmt != kTNvfp4) return false;
    const int K = down ? a.I : a.H;
    const int rows_unit = (!down && a.act == 0) ? 64 : 128;
    const int feats = down ? a.H : a.I;
    if (feats % rows_unit) return false;
    if (a.fmt == kTNvfp4 ? (K % 256) : (K % 512)) return false;   // row strides of the scale tensors
    // any unit count: with few units (one token) each busy SM still streams its
    // units' codes with one pipeline ramp, where the register GEMV pays one per unit
    return t_layout(a.fmt, K, 4).total + 2048 <= device_info().max_smem_optin;
}

cudaError_t launch_gemv_q4t_up(const ExpertArgs& a, bool pdl, cudaStream_t s) {
    if (a.fmt == kTAffine) {
        if (a.act == 0) return run_q4t_pick<kTAffine, kTUpSwiglu>(a, a.H, 2 * a.I, pdl, s);
        return run_q4t_pick<kTAffine, kTUpRelu2>(a, a.H, a.I, pdl, s);
    }
    if (a.fmt == kTNvfp4) {
        if (a.act == 0) return run_q4t_pick<kTNvfp4, kTUpSwiglu>(a, a.H, 2 * a.I, pdl, s);
        return run_q4t_pick<kTNvfp4, kTUpRelu2>(a, a.H, a.I, pdl, s);
    }
    return cudaErrorNotSupported;
}

cudaError_t launch_gemv_q4t_down(const ExpertArgs& a, bool pdl, cudaStream_t s) {
    if (a.fmt == kTAffine) return run_q4t_pick<kTAffine, kTDown>(a, a.I, a.H, pdl, s);
    if (a.fmt == kTNvfp4) return run_q4t_pick<kTNvfp4, kTDown>(a, a.I, a.H, pdl, s);
    return cudaErrorNotSupported;
}

}  // namespace moe
