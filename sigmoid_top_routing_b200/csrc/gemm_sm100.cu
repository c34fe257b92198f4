// Grouped expert GEMMs on the 5th-generation tensor cores (tcgen05 + TMEM).
//
// Swap-AB form: the expert's weight rows are the MMA's M = 128 operand (A,
// streamed by TMA) and the expert's tokens are its N operand (B, N = 16..BN
// in steps of 16), so an expert with 3 tokens costs an N = 16 MMA while its
// weights stream at full rate, and an expert with 500 tokens runs 128 x 256
// tiles.  D[feature][token] accumulates in fp32 in TMEM (double-buffered so
// the epilogue overlaps the next tile's main loop).
//
//   up (SwiGLU):  gate-first W1[e] (TileGym PR #187 "Weight layout and
//                 routing").  Token tiles of 32: a tile = 64 gate rows + the
//                 64 matching up rows, TMEM lanes j and 64 + j hold gate and up
//                 of feature j and the halves meet through shared memory;
//                 tiles of 64 or more: 128 gate + 128 up rows in two TMEM
//                 accumulators.  The epilogue clamps the inputs when
//                 swiglu_limit > 0 and writes h[pos, f] = bf16_rn(silu(g) * u).
//   up (relu^2):  a tile = 128 rows of W1[e]; h = bf16_rn(relu(u)^2), NaN
//                 kept (vllm.cpp PR #684; bloomery PR #235 "What").
//   down:         a tile = 128 rows of W2[e]; y_acc[t, f] += w[p] * D (fp32
//                 reductions), the weighted combine of the pages' MoeCombine;
//                 under the ordered combine, one store of w[p] * D per plan
//                 slot instead.
//
// Prior art: the staged prompt kernels of TensorFold issue #548 ("Prompt rows
// of the grouped experts: two forms": items of 64 pairs x 128 columns staged
// through shared memory) -- kept: staged tiles and a pair's bits depending
// only on its row and expert; changed for sm_100a: TMA, tcgen05, TMEM.
//
// Warp roles (192 threads, one CTA per SM, persistent over tiles):
//   warp 0      producer: TMA for weights and for token rows (up: xs, the
//               rows gathered in plan order by k_gather_rows; down: h)
//   warp 1      TMEM owner and MMA issuer (one thread)
//   warps 2..5  epilogue (TMEM lanes 32 * (warp % 4) ...)
// Every mbarrier wait is bounded; on expiry the kernel records error code 2,
// drains what it issued, frees TMEM and returns.
#include <cuda.h>

#include <mutex>

#include "common.cuh"
#include "internal.h"
#include "launch.h"
#include "plan_dev.cuh"
#include "quant.cuh"
#include "sm100.cuh"
#include "tmap.h"

namespace moe {
namespace {

using namespace sm100;

constexpr int kBK = 64;                  // k per stage: 64 bf16 = one 128-byte swizzle row
constexpr int kARows = 128 * kBK * 2;    // 16 KB: 128 weight rows of one k-block
constexpr int kThreads = 192;            // bf16 weights: producer, MMA, 4 epilogue warps
constexpr int kDq = 256;                 // 4-bit weights: dequantisation threads (8 warps)
constexpr int kThreadsA4 = 192 + kDq;    // 4-bit weights: producer, MMA, 4 epilogue warps + dequant warps
constexpr int kSBDepth = 4;              // stages of scales/biases in flight per dequant thread

enum Mode { kUpSwiglu = 0, kUpRelu2 = 1, kDown = 2 };

struct GemmParams {
    const int32_t* counts;
    const int32_t* offsets;
    const int32_t* perm;
    const float* topk_w;
    const uint16_t* x;       // (T, H) token rows (up)
    uint16_t* h;             // (P, I) activations in plan order (written by up, read by down)
    float* y_acc;            // (T, H) (down), or (P, H) per-slot outputs when ordered
    int ordered;             // down: store w * o per plan slot instead of adding into y_acc
    int E, k, H, I;
    int K;                   // reduction length: H (up) or I (down)
    int rows_per_expert;     // rows of the A tensor per expert: 2I, I or H
    int feats;               // output features per expert: I (up) or H (down)
    const uint16_t* wscale;  // affine 4-bit: (E, rows_per_expert, K/64) bf16 scales; NVFP4: (.., K/16) e4m3 bytes
    const uint16_t* wbias;   // affine 4-bit biases
    const float* wglobal;    // NVFP4: (E) fp32 global scale, multiplied into the fp32 sum
    float swiglu_limit;      // up SwiGLU: clamp of the gate (above) and up (both sides); 0 off
    int skip;                // plan expert given no tiles (its pairs are computed nowhere), or -1
    int E_w;                 // experts the weight tensor holds
    uint32_t wait_limit;     // polls of every bounded pipeline wait (sm100::kWaitLimit)
    int dense_n;             // bf16 up at T <= 16: the token operand is x itself (rows 0..T-1, the
                             // MMA's N = dense_n = T rounded up to 16) and column t is token t;
                             // 0: token rows gathered in plan order (xs), column c is slot row0 + c
    int* err;
};

template <int BN, int STAGES, int ASTAGE, int CSTAGE, bool USE_U,
          int SBRING = (CSTAGE ? kSBDepth * 2 * kDq * 4 : 0), int BROWS = BN>
struct Smem {
    static constexpr int kBStage = BROWS * 128;                              // token rows of one stage
    static constexpr size_t kA = 0;
    static constexpr size_t kB = kA + size_t(STAGES) * ASTAGE;
    static constexpr size_t kC = kB + size_t(STAGES) * kBStage;             // packed 4-bit codes (affine)
    static constexpr size_t kBar = kC + size_t(STAGES) * CSTAGE;            // 8-byte barriers
    static constexpr int kNumBar = 3 * STAGES + 4 + 1;   // full, empty, cfull, tfull[2], tempty[2], drain
    static constexpr size_t kMisc = kBar + kNumBar * 8;                       // tmem base, abort flag
    static constexpr size_t kTileBase = kMisc + 16;                           // 257 ints
    static constexpr size_t kTok = kTileBase + 257 * 4;                       // BN ints (token of column)
    static constexpr size_t kTokW = kTok + BN * 4;                            // BN floats
    static constexpr size_t kU = kTokW + BN * 4;                              // 64 x 17 floats (split SwiGLU)
    static constexpr size_t kCnt = kU + (USE_U ? 64 * 17 * 4 : 0);           // 256 counts + 257 offsets
    static constexpr size_t kSB = kCnt + 513 * 4 + 12;                        // scale/bias ring (affine)
    static constexpr size_t kEnd = kSB + SBRING;
    static constexpr size_t kBytes = kEnd + 1024;                             // + alignment slack
};

// How a tile's A rows are laid out; the kernel and its host launcher both
// derive the shared-memory layout from here.
//   dual   SwiGLU, bf16, token tiles >= 64: 128 gate + 128 up rows, two accumulators
//   inter  SwiGLU, 4-bit, token tiles >= 64: 64 features; in each 32-row TMEM
//          quarter rows 0-15 are gate rows and 16-31 the matching up rows, so gate
//          and up of a feature meet by one warp shuffle; one accumulator, so token
//          tiles reach 256 and each dequantised A stage serves twice the tokens
//   halves SwiGLU, token tiles of 32: 64 gate rows then 64 up rows, one accumulator,
//          the halves meet through shared memory
//   pair   (PAIR = 1) two CTAs on neighbouring SMs run one M = 256 MMA
//          (tcgen05 cta_group::2): each holds its own 128 weight rows and half of
//          the tile's token rows, and gets its 128 rows of the accumulator
template <int MODE, int BN, int WFMT, int PAIR = 0>
struct Cfg {
    static constexpr int kBRows = PAIR ? BN / 2 : BN;       // token rows a CTA stages per k-block
    static constexpr bool kInter = MODE == kUpSwiglu && WFMT != 0 && BN >= 64;
    static constexpr bool kDual = MODE == kUpSwiglu && BN >= 64 && !kInter;
    static constexpr bool kHalves = MODE == kUpSwiglu && BN < 64;
    static constexpr int kAStage = kDual ? 2 * kARows : kARows;
    static constexpr int kCStage = WFMT ? kAStage / 4 : 0;   // packed 4-bit codes of one A stage
    static constexpr int kFpt = MODE == kUpSwiglu && !kDual ? 64 : 128;   // output features per tile
    static constexpr uint32_t kABox = MODE == kUpSwiglu && !kDual ? 64 : 128;   // A rows per TMA box
};

struct Tile {
    int e, wt, tt, ntok, n, row0;
    int brow;                // first token row the TMA reads (row0, or 0 when the operand is x)
    int kb0, kb1;            // k-blocks of this tile (a part of K when the reduction is split)
};

// Tile t -> (expert, weight tile, token tile).  Tiles of one expert run
// weight-tile-major with the token tiles innermost, so the CTAs working at
// one time share weight tiles in L2.
// With SPLIT, ks consecutive tile numbers share one output tile and each
// takes a contiguous part of the nkb k-blocks.
template <int BN, bool SPLIT>
MOE_DEV Tile decode_tile(int tn, const int* base, int E, const int* counts, const int* offsets, int ks, int nkb,
                         int dense_n) {
    const int t = SPLIT ? tn / ks : tn;
    int lo = 0, hi = E;
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (base[mid] <= t) lo = mid;
        else hi = mid - 1;
    }
    Tile r;
    r.e = lo;
    const int c = counts[lo];
    const int ntt = (c + BN - 1) / BN;
    const int local = t - base[lo];
    r.wt = local / ntt;
    r.tt = local % ntt;
    r.ntok = min(BN, c - r.tt * BN);
    r.n = (r.ntok + 15) & ~15;
    r.row0 = offsets[lo] + r.tt * BN;
    r.brow = r.row0;
    if (dense_n) {
        r.n = dense_n;
        r.brow = 0;
    }
    if (SPLIT) {
        const int part = tn - t * ks;
        r.kb0 = part * nkb / ks;
        r.kb1 = (part + 1) * nkb / ks;
    } else {
        r.kb0 = 0;
        r.kb1 = nkb;
    }
    return r;
}

// silu(g) * u in fp32 with the fast exponential and division (the result is
// rounded to bf16); NaN propagates, g -> -inf gives -0 * u.
MOE_DEV float silu_mul(float g, float u) { return __fdividef(g, 1.0f + __expf(-g)) * u; }


// Dequantise 16-byte chunks [c0, c0 + NC) of one 128-byte A row (8 affine
// 4-bit codes per chunk, one group per row per k-block) into the 128-byte-
// swizzled bf16 layout.  The low and high nibbles of a code word are split
// into byte lanes, PRMT pairs codes (2p, 2p + 1) and OR 0x4300 makes
// bf16(128 + q) exactly; minus 128 gives q exactly and one bf16x2 fma gives
// bf16_rn(scale * q + bias) with a single rounding.
template <int NC>
MOE_DEV void dequant_chunks(const uint32_t* codes, int c0, uint16_t scale, uint16_t bias, unsigned char* arow,
                            int r) {
    const uint32_t s2u = uint32_t(scale) | (uint32_t(scale) << 16);
    const uint32_t b2u = uint32_t(bias) | (uint32_t(bias) << 16);
    const __nv_bfloat162 s2 = *reinterpret_cast<const __nv_bfloat162*>(&s2u);
    const __nv_bfloat162 b2 = *reinterpret_cast<const __nv_bfloat162*>(&b2u);
    const uint32_t k128u = 0x43004300u;
    const __nv_bfloat162 k128 = *reinterpret_cast<const __nv_bfloat162*>(&k128u);
#pragma unroll
    for (int i = 0; i < NC; ++i) {
        const int c = c0 + i;
        const uint32_t w = codes[i];
        const uint32_t lo = w & 0x0F0F0F0Fu;           // codes 0, 2, 4, 6 in bytes 0..3
        const uint32_t hi = (w >> 4) & 0x0F0F0F0Fu;    // codes 1, 3, 5, 7
        uint32_t o[4];
#pragma unroll
        for (int p = 0; p < 4; ++p) {
            const uint32_t sel = uint32_t(p) | (uint32_t(p) << 4) | (uint32_t(4 + p) << 8) | (uint32_t(4 + p) << 12);
            uint32_t x;
            asm("prmt.b32 %0, %1, %2, %3;" : "=r"(x) : "r"(lo), "r"(hi), "r"(sel));
            const uint32_t q2u = (x & 0x00FF00FFu) | 0x43004300u;
            const __nv_bfloat162 q2 = __hsub2(*reinterpret_cast<const __nv_bfloat162*>(&q2u), k128);
            const __nv_bfloat162 v = __hfma2(q2, s2, b2);
            o[p] = *reinterpret_cast<const uint32_t*>(&v);
        }
        *reinterpret_cast<uint4*>(arow + (((c ^ (r & 7)) & 7) << 4)) = make_uint4(o[0], o[1], o[2], o[3]);
    }
}

// NVFP4: chunks [c0, c0 + NC) of one 128-byte A row from 8 e2m1 codes each
// (one 32-bit word, the low nibble first) and the row's four e4m3 block scales
// of this k-block (byte b serves chunks 2b and 2b + 1).  The code pairs and the
// scale convert exactly to f16, their f16 product is exact (at most six
// significant bits, in range), and widening to fp32 then rounding the pair to
// bf16 is exact again: A holds e2m1 * e4m3 exactly; the global scale is applied
// to the fp32 sum in the epilogue.
template <int NC>
MOE_DEV void dequant_nvfp4_chunks(const uint32_t* codes, int c0, uint32_t scales4, unsigned char* arow, int r) {
#pragma unroll
    for (int i = 0; i < NC; ++i) {
        const int c = c0 + i;
        const uint32_t sb = (scales4 >> (8 * (c >> 1))) & 0xFFu;
        const uint32_t s2 = e4m3x2_to_f16x2(sb | (sb << 8));
        uint32_t p[4];
        e2m1x8_to_f16(codes[i], p);
        uint32_t o[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) o[j] = f16x2_to_bf16x2(hmul2_u32(p[j], s2));
        *reinterpret_cast<uint4*>(arow + (((c ^ (r & 7)) & 7) << 4)) = make_uint4(o[0], o[1], o[2], o[3]);
    }
}

MOE_DEV void cp_async4(uint32_t dst, const void* src) {
    asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(dst), "l"(src) : "memory");
}
MOE_DEV void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
MOE_DEV void cp_async_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }

template <int MODE, int BN, int STAGES, int WFMT, int PAIR>
__global__ void __launch_bounds__(WFMT ? kThreadsA4 : kThreads, 1)
    k_gemm(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB, GemmParams g) {
    // SwiGLU with wide token tiles keeps two accumulators (128 gate rows and
    // 128 up rows against one token tile) so a thread holds gate and up of its
    // feature; decode-width SwiGLU tiles split 64 gate + 64 up rows over the
    // lanes of one accumulator (more, smaller tiles for a short decode step).
    using C = Cfg<MODE, BN, WFMT, PAIR>;
    static_assert(!(PAIR && WFMT), "SM pairs run bf16 weights");
    constexpr bool kDual = C::kDual;
    constexpr bool kInter = C::kInter;
    constexpr int kAStage = C::kAStage;
    constexpr int kBoxRows = BN < 64 ? 16 : 64;       // token rows per TMA box
    // affine 4-bit: the A stage is written by the dequantisation warps from
    // packed codes (a quarter of the bf16 bytes) staged by TMA
    constexpr int kCStage = C::kCStage;
    using L = Smem<BN, STAGES, kAStage, kCStage, C::kHalves, (kCStage ? kSBDepth * 2 * kDq * 4 : 0), C::kBRows>;
    extern __shared__ unsigned char smem_raw[];
    unsigned char* sm = reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    unsigned char* sA = sm + L::kA;
    unsigned char* sB = sm + L::kB;
    uint64_t* bars = reinterpret_cast<uint64_t*>(sm + L::kBar);
    uint64_t* full = bars;
    uint64_t* empty = bars + STAGES;
    uint64_t* tfull = bars + 2 * STAGES;
    uint64_t* tempty = bars + 2 * STAGES + 2;
    uint64_t* drain = bars + 2 * STAGES + 4;
    uint64_t* cfull = bars + 2 * STAGES + 5;              // codes landed (affine)
    unsigned char* sC = sm + L::kC;
    uint32_t* s_tmem = reinterpret_cast<uint32_t*>(sm + L::kMisc);
    volatile int* s_abort = reinterpret_cast<volatile int*>(sm + L::kMisc + 4);
    int* s_base = reinterpret_cast<int*>(sm + L::kTileBase);
    int* s_tok = reinterpret_cast<int*>(sm + L::kTok);
    float* s_tokw = reinterpret_cast<float*>(sm + L::kTokW);
    float* s_u = reinterpret_cast<float*>(sm + L::kU);
    int* s_cnt = reinterpret_cast<int*>(sm + L::kCnt);      // plan counts and offsets, copied once
    int* s_off = s_cnt + 256;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t rank = PAIR ? cluster_ctarank() : 0u;   // 0: the CTA that issues the pair's MMAs
    constexpr uint32_t kTmemCols = (kDual ? 4 : 2) * BN < 32 ? 32 : (kDual ? 4 : 2) * BN;
    // token rows come by TMA: from xs (up, gathered in plan order) or h (down)
    constexpr uint32_t kFullCount = 1 + (WFMT ? kDq : 0);   // expect_tx arrive + the dequant threads
    // pairs: the even CTA's full barrier counts both CTAs' bytes (its producer
    // arrives once with the total); its tempty barrier takes all 8 epilogue warps

    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(&full[s], kFullCount);
            mbar_init(&empty[s], 1);
            if (WFMT) mbar_init(&cfull[s], 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&tfull[b], 1);
            mbar_init(&tempty[b], PAIR ? 8 : 4);
        }
        mbar_init(drain, 1);
        *s_abort = 0;
        fence_mbar_init();
    }
    if (PAIR) cluster_sync();     // both CTAs' barriers exist before either signals the other
    if (warp == 0 && lane == 0) {
        tma_prefetch_desc(&tmA);
        tma_prefetch_desc(&tmB);
    }
    if (warp == 1) {
        if (PAIR) {
            tmem_alloc_pair(s_tmem, kTmemCols);
            tmem_relinquish_pair();
        } else {
            tmem_alloc(s_tmem, kTmemCols);
            tmem_relinquish();
        }
        tc_fence_before();
    }
    // The up kernels follow the plan directly: they wait for it here.  The
    // down kernel follows the up kernel and reads the plan (finished two
    // launches earlier, read through L2) before waiting, so its weight tiles
    // stream while the up kernel's last CTAs finish; only its producer waits,
    // right before the first load of h.
    if (MODE != kDown) pdl_wait();
    for (int i = threadIdx.x; i < g.E; i += blockDim.x) {
        s_cnt[i] = i == g.skip ? 0 : __ldcg(g.counts + i);   // a skipped expert gets no tiles
        s_off[i] = __ldcg(g.offsets + i);
    }
    __syncthreads();
    // tile table: tiles of expert e = weight tiles x ceil(count / BN)
    const int fpt = C::kFpt;                                     // output features per tile (per CTA)
    constexpr bool kDenseOk = MODE != kDown && BN == 32 && WFMT == 0 && !PAIR;
    const int dense_n = kDenseOk ? g.dense_n : 0;                // token operand = x (see GemmParams)
    const int n_wt = (g.feats + fpt * (1 + PAIR) - 1) / (fpt * (1 + PAIR));   // weight tiles per expert
    if (warp == 2) {
        const int per = (g.E + 31) / 32;
        int local = 0;
        for (int j = 0; j < per; ++j) {
            const int e = lane * per + j;
            if (e < g.E) local += n_wt * ((s_cnt[e] + BN - 1) / BN);
        }
        int incl = local;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int v = __shfl_up_sync(0xffffffffu, incl, o);
            if (lane >= o) incl += v;
        }
        int run = incl - local;
        for (int j = 0; j < per; ++j) {
            const int e = lane * per + j;
            if (e < g.E) {
                s_base[e] = run;
                run += n_wt * ((s_cnt[e] + BN - 1) / BN);
            }
        }
        if (lane == 31) s_base[g.E] = incl;
    }
    __syncthreads();
    tc_fence_after();
    // Every CTA of this persistent grid is resident by now, so the next kernel
    // may launch: its CTAs take SMs as ours retire and run their prologue (the
    // down kernel also its first weight loads) before waiting on this grid.
    pdl_trigger();
    const uint32_t tmem_base = *s_tmem;
    const int nkb = g.K / kBK;
    // the persistent tile loop: CTAs, or CTA pairs (both CTAs of a pair run the same tiles)
    const int tbeg = PAIR ? (int)(blockIdx.x >> 1) : (int)blockIdx.x;
    const int tstep = PAIR ? (int)(gridDim.x >> 1) : (int)gridDim.x;
    // The down projection's scatter-add is linear, so its reduction can be
    // split: with less than ~4 waves of output tiles, K is cut into ks parts
    // (>= 4 k-blocks each) whose partial sums all add into y_acc.
    constexpr bool kSplit = MODE == kDown;
    int ks = 1;
    if (kSplit && !g.ordered) {   // ordered: each slot row is stored once, whole
        const int t1 = max(s_base[g.E], 1);
        ks = min(min(4, max(1, nkb / 4)), max(1, (4 * tstep + t1 - 1) / t1));
    }
    const int total = s_base[g.E] * ks;

    if (warp == 0) {
        // ------------------------------------------------------------ producer
        int s = 0;
        uint32_t ph = 0;
        uint32_t issued_mask = 0;            // stages with a fill whose arrival is not yet known
        uint32_t issued_par = 0;             // parity of that fill
        bool ok = true;
        // weights read by one token tile are streamed once (evict first); with
        // several token tiles per weight tile the neighbours re-read it from L2
        const uint64_t pol_w = policy_evict_first();
        const bool hint_w = BN <= 32;
        // down kernel: the first tile's first stages get their weight rows before
        // the wait on the up kernel; their token rows (h) follow after it
        int pre = 0;
        if (MODE == kDown && !PAIR && blockIdx.x < total) {
            const Tile tl = decode_tile<BN, kSplit>(blockIdx.x, s_base, g.E, s_cnt, s_off, ks, nkb, dense_n);
            pre = min(STAGES, tl.kb1 - tl.kb0);
            if (lane == 0) {
                const int nbox = (tl.n + kBoxRows - 1) / kBoxRows;
                const int a_row = tl.e * g.rows_per_expert + tl.wt * fpt;
                for (int q = 0; q < pre; ++q) {      // fresh barriers: no empty wait needed
                    const int kb = tl.kb0 + q;
                    mbar_arrive_expect_tx(&full[q], (WFMT ? 0 : kAStage) + nbox * kBoxRows * 128);
                    if (WFMT) {
                        mbar_arrive_expect_tx(&cfull[q], kCStage);
                        tma_load_2d(sC + size_t(q) * kCStage, &tmA, kb * 8, a_row, &cfull[q]);
                    } else {
                        tma_load_2d(sA + size_t(q) * kAStage, &tmA, kb * kBK, a_row, &full[q]);
                    }
                }
            }
        }
        if (MODE == kDown) pdl_wait();
        for (int t = tbeg; t < total && ok; t += tstep) {
            const Tile tl = decode_tile<BN, kSplit>(t, s_base, g.E, s_cnt, s_off, ks, nkb, dense_n);
            // pairs: this CTA's 128 weight rows of the 256-row tile, and its half of the token rows
            const int a_row = tl.e * g.rows_per_expert + tl.wt * fpt * (1 + PAIR) + (int)rank * fpt;
            const int brows = PAIR ? tl.n / 2 : tl.n;
            const int brow0 = tl.brow + (int)rank * (PAIR ? tl.n / 2 : 0);
            for (int kb = tl.kb0; kb < tl.kb1; ++kb) {
                if (pre > 0) {
                    // weight rows already requested before the wait: add the token rows
                    if (lane == 0) {
                        const int nbox = (tl.n + kBoxRows - 1) / kBoxRows;
                        unsigned char* b = sB + size_t(s) * L::kBStage;
                        for (int j = 0; j < nbox; ++j)
                            tma_load_2d(b + j * kBoxRows * 128, &tmB, kb * kBK, tl.brow + kBoxRows * j, &full[s]);
                    }
                    --pre;
                    issued_mask |= 1u << s;
                    issued_par = (issued_par & ~(1u << s)) | (ph << s);
                    if (++s == STAGES) { s = 0; ph ^= 1; }
                    continue;
                }
                // all 32 lanes wait on the same phase; the decision is made warp-uniform
                const bool got = mbar_wait(&empty[s], ph ^ 1, s_abort, g.wait_limit);
                if (!__all_sync(0xffffffffu, got)) { ok = false; break; }
                if (lane == 0 && PAIR) {
                    // both CTAs' loads complete on the even CTA's full barrier; it arrives once
                    // with the bytes of both
                    const int nbox = (brows + kBoxRows - 1) / kBoxRows;
                    const uint32_t fb = mapa_shared(smem_u32(&full[s]), 0);
                    if (rank == 0) mbar_arrive_expect_tx(&full[s], 2u * (kAStage + nbox * kBoxRows * 128));
                    unsigned char* a = sA + size_t(s) * kAStage;
                    tma_load_2d_pair(a, &tmA, kb * kBK, a_row, fb);
                    if (MODE == kUpSwiglu) tma_load_2d_pair(a + kAStage / 2, &tmA, kb * kBK, a_row + g.I, fb);
                    unsigned char* b = sB + size_t(s) * L::kBStage;
                    for (int j = 0; j < nbox; ++j)
                        tma_load_2d_pair(b + j * kBoxRows * 128, &tmB, kb * kBK, brow0 + kBoxRows * j, fb);
                } else if (lane == 0) {
                    const int nbox = (tl.n + kBoxRows - 1) / kBoxRows;
                    const uint32_t bytes = (WFMT ? 0 : kAStage) + nbox * kBoxRows * 128;
                    mbar_arrive_expect_tx(&full[s], bytes);
                    if (WFMT) mbar_arrive_expect_tx(&cfull[s], kCStage);
                    // bf16: weight rows straight into the A stage; affine: codes into the staging area
                    unsigned char* a = WFMT ? sC + size_t(s) * kCStage : sA + size_t(s) * kAStage;
                    constexpr int kHalf = WFMT ? kCStage / 2 : kAStage / 2;
                    const int ax = WFMT ? kb * 8 : kb * kBK;      // codes: 8 words per row per k-block
                    // A: [gate | up] halves for SwiGLU (64 or 128 rows each), else 128 rows
                    uint64_t* abar = WFMT ? &cfull[s] : &full[s];
                    if (hint_w) {
                        tma_load_2d_hint(a, &tmA, ax, a_row, abar, pol_w);
                        if (MODE == kUpSwiglu) tma_load_2d_hint(a + kHalf, &tmA, ax, a_row + g.I, abar, pol_w);
                    } else {
                        tma_load_2d(a, &tmA, ax, a_row, abar);
                        if (MODE == kUpSwiglu) tma_load_2d(a + kHalf, &tmA, ax, a_row + g.I, abar);
                    }
                    unsigned char* b = sB + size_t(s) * L::kBStage;
                    for (int j = 0; j < nbox; ++j)
                        tma_load_2d(b + j * kBoxRows * 128, &tmB, kb * kBK, tl.brow + kBoxRows * j, &full[s]);
                }
                issued_mask |= 1u << s;
                issued_par = (issued_par & ~(1u << s)) | (ph << s);
                if (++s == STAGES) { s = 0; ph ^= 1; }
            }
        }
        if (!ok) {
            if (lane == 0) report_error(g.err, kErrWaitExpired);
            *s_abort = 1;
        }
        // wait (bounded) for every fill this warp issued to land before the CTA can exit
        // (pairs: the even CTA's full barriers count the odd CTA's bytes too, and the
        // two CTAs meet at a cluster barrier before either exits)
        if (!PAIR || rank == 0)
            for (int q = 0; q < STAGES; ++q)
                if (issued_mask >> q & 1u) mbar_wait(&full[q], issued_par >> q & 1u, nullptr, g.wait_limit);
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        // (pairs: only the even CTA issues; its MMAs cover both CTAs' rows)
        if (lane == 0 && rank == 0) {
            int s = 0;
            uint32_t ph = 0;
            int it = 0;
            bool ok = true;
            for (int t = tbeg; t < total && ok; t += tstep, ++it) {
                const Tile tl = decode_tile<BN, kSplit>(t, s_base, g.E, s_cnt, s_off, ks, nkb, dense_n);
                const int buf = it & 1;
                const uint32_t aph = (it >> 1) & 1;
                if (!mbar_wait(&tempty[buf], aph ^ 1, s_abort, g.wait_limit)) { ok = false; break; }
                tc_fence_after();
                const uint32_t d = tmem_base + buf * (kDual ? 2 * BN : BN);
                const uint32_t idesc = idesc_bf16(PAIR ? 256 : 128, tl.n);
                for (int kb = tl.kb0; kb < tl.kb1; ++kb) {
                    if (!mbar_wait(&full[s], ph, s_abort, g.wait_limit)) { ok = false; break; }
                    tc_fence_after();
                    const uint64_t ad = sdesc_sw128(smem_u32(sA + size_t(s) * kAStage));
                    const uint64_t bd = sdesc_sw128(smem_u32(sB + size_t(s) * L::kBStage));
#pragma unroll
                    for (int kk = 0; kk < kBK / 16; ++kk) {
                        const bool acc = kb != tl.kb0 || kk != 0;
                        if (PAIR) {
                            umma_bf16_pair(d, ad + uint64_t(kk * 2), bd + uint64_t(kk * 2), idesc, acc);
                            if (kDual)
                                umma_bf16_pair(d + BN, ad + uint64_t((kARows >> 4) + kk * 2), bd + uint64_t(kk * 2),
                                               idesc, acc);
                        } else {
                            umma_bf16(d, ad + uint64_t(kk * 2), bd + uint64_t(kk * 2), idesc, acc);
                            if (kDual)   // up rows: the second 16 KB of the A stage, accumulator at + BN columns
                                umma_bf16(d + BN, ad + uint64_t((kARows >> 4) + kk * 2), bd + uint64_t(kk * 2), idesc,
                                          acc);
                        }
                    }
                    if (PAIR) umma_commit_pair_both(&empty[s]);   // both CTAs' stage s is free again
                    else umma_commit(&empty[s]);
                    if (++s == STAGES) { s = 0; ph ^= 1; }
                }
                if (!ok) break;
                if (PAIR) umma_commit_pair_both(&tfull[buf]);      // both CTAs' accumulators are ready
                else umma_commit(&tfull[buf]);
            }
            if (!ok) {
                report_error(g.err, kErrWaitExpired);
                *s_abort = 1;
            }
            // all MMAs issued by this thread complete before TMEM is freed
            if (PAIR) umma_commit_pair_local(drain);
            else umma_commit(drain);
            mbar_wait(drain, 0, nullptr, g.wait_limit);
        }
        __syncwarp();
    } else if (WFMT && warp >= 6) {   // warps 6 .. 6 + kDq / 32 - 1
        // ------------------------------------------------------------ dequantisation (4-bit)
        // kDq threads.  kTpr threads share an A row, each kCPT of its 8 chunks.
        // Each thread fetches its row's scale (and bias) kSBDepth stages ahead
        // with 4-byte cp.async into a ring in shared memory (affine: the word
        // holding the bf16, the half is picked later; NVFP4: the row's four
        // e4m3 block scales of the k-block).
        const int dt = threadIdx.x - 192;
        constexpr int kRows = kDual ? 256 : 128;
        constexpr int kTpr = kDq / kRows;                  // threads per A row
        constexpr int kCPT = 8 / kTpr;                     // 16-byte chunks per thread
        const int r = dt / kTpr;
        const int cbeg = (dt % kTpr) * kCPT;
        const int halfr = kDual ? 128 : 64;                // SwiGLU: rows of the gate half
        const size_t nrows = (size_t)g.E_w * g.rows_per_expert;
        const int G = g.K / 64;
        uint32_t* s_sb = reinterpret_cast<uint32_t*>(sm + L::kSB);
        // inter layout: A row r = 32 q + j holds gate (j < 16) or up (j >= 16) of
        // feature 16 q + (j & 15) of the tile; the staged codes are 64 gate rows
        // then 64 up rows, as TMA brings them
        const int cr = kInter ? ((r & 16) ? 64 : 0) + 16 * (r >> 5) + (r & 15) : r;   // staged code row
        auto grow = [&](const Tile& tl) -> size_t {      // global weight row of A row r
            const size_t base = (size_t)tl.e * g.rows_per_expert;
            if (MODE == kUpSwiglu)
                return cr < halfr ? base + (size_t)tl.wt * halfr + cr : base + g.I + (size_t)tl.wt * halfr + (cr - halfr);
            return base + (size_t)tl.wt * 128 + r;
        };
        // look-ahead iterator over this CTA's (tile, k-block) stages
        int at = tbeg, akb = 0;
        Tile atl{};
        if (at < total) {
            atl = decode_tile<BN, kSplit>(at, s_base, g.E, s_cnt, s_off, ks, nkb, dense_n);
            akb = atl.kb0;
        }
        auto issue = [&](int slot) {
            if (at < total) {
                const size_t gr = grow(atl);
                if (WFMT == 2) {      // the row's four e4m3 block scales of this k-block: one word
                    const size_t wi = gr < nrows ? gr * (size_t)(g.K / 16) + 4 * (size_t)akb : 0;
                    cp_async4(smem_u32(s_sb + (slot * 2 + 0) * kDq + dt),
                              reinterpret_cast<const uint8_t*>(g.wscale) + wi);
                } else {
                    const size_t gi = gr < nrows ? gr * G + akb : 0;
                    cp_async4(smem_u32(s_sb + (slot * 2 + 0) * kDq + dt), g.wscale + (gi & ~size_t(1)));
                    cp_async4(smem_u32(s_sb + (slot * 2 + 1) * kDq + dt), g.wbias + (gi & ~size_t(1)));
                }
                if (++akb == atl.kb1) {
                    at += tstep;
                    if (at < total) {
                        atl = decode_tile<BN, kSplit>(at, s_base, g.E, s_cnt, s_off, ks, nkb, dense_n);
                        akb = atl.kb0;
                    }
                }
            }
            cp_async_commit();
        };
#pragma unroll
        for (int j = 0; j < kSBDepth; ++j) issue(j);
        int s = 0, slot = 0;
        uint32_t ph = 0;
        bool ok = true;
        for (int t = tbeg; t < total && ok; t += tstep) {
            const Tile tl = decode_tile<BN, kSplit>(t, s_base, g.E, s_cnt, s_off, ks, nkb, dense_n);
            const size_t gr = grow(tl);
            for (int kb = tl.kb0; kb < tl.kb1; ++kb) {
                cp_async_wait<kSBDepth - 1>();               // this stage's scale/bias landed
                const uint32_t sw = s_sb[(slot * 2 + 0) * kDq + dt];
                const uint32_t bw = s_sb[(slot * 2 + 1) * kDq + dt];
                const bool odd = ((gr * G + kb) & 1) != 0;
                const bool inb = gr < nrows;
                const uint16_t sc = inb ? uint16_t(odd ? sw >> 16 : sw & 0xFFFFu) : uint16_t(0);
                const uint16_t bi = inb ? uint16_t(odd ? bw >> 16 : bw & 0xFFFFu) : uint16_t(0);
                issue(slot);                                  // refill the slot kSBDepth stages ahead
                if (++slot == kSBDepth) slot = 0;
                if (!mbar_wait(&cfull[s], ph, s_abort, g.wait_limit)) { ok = false; break; }
                const uint32_t* crow = reinterpret_cast<const uint32_t*>(sC + size_t(s) * kCStage) + cr * 8 + cbeg;
                uint32_t cw[kCPT];
                if (kCPT >= 4) {
#pragma unroll
                    for (int q = 0; q < kCPT / 4; ++q) {
                        const uint4 c4 = reinterpret_cast<const uint4*>(crow)[q];
                        cw[4 * q + 0] = c4.x;
                        cw[4 * q + 1] = c4.y;
                        cw[4 * q + 2] = c4.z;
                        cw[4 * q + 3] = c4.w;
                    }
                } else {
#pragma unroll
                    for (int q = 0; q < kCPT / 2; ++q) {
                        const uint2 c2 = reinterpret_cast<const uint2*>(crow)[q];
                        cw[2 * q + 0] = c2.x;
                        cw[2 * q + 1] = c2.y;
                    }
                }
                if (WFMT == 2)
                    dequant_nvfp4_chunks<kCPT>(cw, cbeg, inb ? sw : 0u, sA + size_t(s) * kAStage + r * 128, r);
                else
                    dequant_chunks<kCPT>(cw, cbeg, sc, bi, sA + size_t(s) * kAStage + r * 128, r);
                fence_proxy_async_smem();                 // generic-proxy writes -> tensor core reads
                mbar_arrive(&full[s]);
                if (++s == STAGES) { s = 0; ph ^= 1; }
            }
        }
        cp_async_wait<0>();                               // no copy of this thread left in flight
        if (!ok) {
            report_error(g.err, kErrWaitExpired);
            *s_abort = 1;
        }
    } else {
        // ------------------------------------------------------------ epilogue
        // The four warps run the same tile sequence and the same named
        // barriers; after an abort they keep looping without touching TMEM or
        // global memory, so no warp is left waiting at a barrier.
        const int sub = warp & 3;                 // TMEM lane quarter this warp may access
        const int lrow = 32 * sub + lane;         // row of the 128-row tile
        const int et = threadIdx.x - 64;          // 0..127
        int it = 0;
        bool dead = false;
        for (int t = tbeg; t < total; t += tstep, ++it) {
            const Tile tl = decode_tile<BN, kSplit>(t, s_base, g.E, s_cnt, s_off, ks, nkb, dense_n);
            const int buf = it & 1;
            const uint32_t aph = (it >> 1) & 1;
            const int fbase = tl.wt * fpt * (1 + PAIR) + (int)rank * fpt;   // first output feature of this CTA
            if (MODE == kDown) {
                for (int c = et; c < tl.ntok; c += 128) {
                    const int p = g.perm[tl.row0 + c];
                    s_tok[c] = p / g.k;
                    s_tokw[c] = g.topk_w[p];
                }
                named_bar(1, 128);
            } else if (dense_n) {
                // column t is token t: its h row is the plan slot of (t, this expert), if routed here
                for (int c = et; c < tl.n; c += 128) s_tok[c] = -1;
                named_bar(1, 128);
                for (int c = et; c < tl.ntok; c += 128) s_tok[g.perm[tl.row0 + c] / g.k] = tl.row0 + c;
                named_bar(1, 128);
            }
            // h row of accumulator column c (up), or -1
            auto hrow = [&](int c) -> int {
                if (dense_n) return s_tok[c];
                return c < tl.ntok ? tl.row0 + c : -1;
            };
            if (!dead) {
                const bool ok = mbar_wait(&tfull[buf], aph, s_abort, g.wait_limit);
                if (__any_sync(0xffffffffu, !ok)) {     // warp-uniform: tcgen05.ld is warp-collective
                    if (lane == 0) report_error(g.err, kErrWaitExpired);
                    *s_abort = 1;
                    dead = true;
                }
            }
            tc_fence_after();
            const uint32_t tbase = tmem_base + (uint32_t(32 * sub) << 16) + buf * (kDual ? 2 * BN : BN);
            const float gsc = WFMT == 2 ? __ldg(g.wglobal + tl.e) : 1.0f;
            for (int c0 = 0; c0 < tl.n; c0 += 16) {
                float v[16];
                if (dead) {
#pragma unroll
                    for (int i = 0; i < 16; ++i) v[i] = 0.0f;
                } else {
                    tmem_ld16(tbase + c0, v);
                    if (WFMT == 2) {      // NVFP4: the expert's global scale on the fp32 sum
#pragma unroll
                        for (int i = 0; i < 16; ++i) v[i] *= gsc;
                    }
                }
                if (MODE == kDown) {
                    const int f = fbase + lrow;
                    if (!dead && f < g.feats) {
                        if (!g.ordered) {
#pragma unroll
                            for (int i = 0; i < 16; ++i) {
                                const int c = c0 + i;
                                if (c < tl.ntok) red_add_f32(g.y_acc + (size_t)s_tok[c] * g.H + f, s_tokw[c] * v[i]);
                            }
                        } else {   // one store per slot row (plan order)
#pragma unroll
                            for (int i = 0; i < 16; ++i) {
                                const int c = c0 + i;
                                if (c < tl.ntok) __stcg(g.y_acc + (size_t)(tl.row0 + c) * g.H + f, s_tokw[c] * v[i]);
                            }
                        }
                    }
                } else if (MODE == kUpRelu2) {
                    const int f = fbase + lrow;
                    if (!dead && f < g.feats) {
#pragma unroll
                        for (int i = 0; i < 16; ++i) {
                            const int r = hrow(c0 + i);
                            if (r >= 0) g.h[(size_t)r * g.I + f] = f2bf16(act_relu2(v[i]));
                        }
                    }
                } else if (kInter) {
                    // lanes 0-15: gate of feature f, lanes 16-31: up of f (f = 16 sub + lane % 16
                    // within the tile).  One exchange of eight values: the low lanes then
                    // hold gate and up of columns c0 .. c0+7, the high lanes of c0+8 .. c0+15.
                    const bool lo = lane < 16;
                    const int f = fbase + 16 * sub + (lane & 15);
                    float gv[8], uv[8];
#pragma unroll
                    for (int i = 0; i < 8; ++i) {
                        const float other = __shfl_xor_sync(0xffffffffu, lo ? v[8 + i] : v[i], 16);
                        gv[i] = lo ? v[i] : other;
                        uv[i] = lo ? other : v[8 + i];
                    }
                    if (!dead && f < g.feats) {
#pragma unroll
                        for (int i = 0; i < 8; ++i) {
                            const int c = c0 + (lo ? i : 8 + i);
                            if (c >= tl.ntok) continue;
                            float a_ = gv[i], b_ = uv[i];
                            clamp_swiglu(a_, b_, g.swiglu_limit);
                            g.h[(size_t)(tl.row0 + c) * g.I + f] = f2bf16(silu_mul(a_, b_));
                        }
                    }
                } else if (kDual) {
                    float u[16];
                    if (dead) {
#pragma unroll
                        for (int i = 0; i < 16; ++i) u[i] = 0.0f;
                    } else {
                        tmem_ld16(tbase + BN + c0, u);
                        if (WFMT == 2) {
#pragma unroll
                            for (int i = 0; i < 16; ++i) u[i] *= gsc;
                        }
                    }
                    const int f = fbase + lrow;
                    if (!dead && f < g.feats) {
#pragma unroll
                        for (int i = 0; i < 16; ++i) {
                            const int c = c0 + i;
                            if (c >= tl.ntok) continue;
                            float gv = v[i], uv = u[i];
                            clamp_swiglu(gv, uv, g.swiglu_limit);
                            g.h[(size_t)(tl.row0 + c) * g.I + f] = f2bf16(silu_mul(gv, uv));
                        }
                    }
                } else {
                    // up rows (lanes 64..127) hand their values to the gate rows through shared memory
                    if (sub >= 2) {
#pragma unroll
                        for (int i = 0; i < 16; ++i) s_u[(lrow - 64) * 17 + i] = v[i];
                    }
                    named_bar(1, 128);
                    if (!dead && sub < 2) {
                        const int f = fbase + lrow;
#pragma unroll
                        for (int i = 0; i < 16; ++i) {
                            const int r = hrow(c0 + i);
                            if (r < 0) continue;
                            float gv = v[i], uv = s_u[lrow * 17 + i];
                            clamp_swiglu(gv, uv, g.swiglu_limit);
                            g.h[(size_t)r * g.I + f] = f2bf16(silu_mul(gv, uv));
                        }
                    }
                    named_bar(1, 128);
                }
            }
            tc_fence_before();
            if (lane == 0) {
                if (PAIR && rank != 0) mbar_arrive_cluster(mapa_shared(smem_u32(&tempty[buf]), 0));
                else mbar_arrive(&tempty[buf]);
            }
            if (MODE == kDown || dense_n) named_bar(1, 128);   // s_tok reuse
        }
    }
    __syncthreads();
    if (PAIR) cluster_sync();     // the pair's MMAs and both epilogues are done with TMEM
    if (warp == 1) {
        tc_fence_after();
        if (PAIR) tmem_dealloc_pair(tmem_base, kTmemCols);
        else tmem_dealloc(tmem_base, kTmemCols);
    }
}

// ---------------------------------------------------------------------------- host side

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &p, 12000, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
    });
    return fn;
}

// bf16 matrix (outer rows x inner cols, row-major), 128-byte swizzled boxes.
cudaError_t make_tmap(CUtensorMap* m, const void* base, uint64_t inner, uint64_t outer, uint32_t box_inner,
                      uint32_t box_outer) {
    EncodeTiledFn enc = encode_fn();
    if (!enc) return cudaErrorNotSupported;
    const cuuint64_t dims[2] = {inner, outer};
    const cuuint64_t strides[1] = {inner * 2};
    const cuuint32_t box[2] = {box_inner, box_outer};
    const cuuint32_t estr[2] = {1, 1};
    CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
                     CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                     CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

// uint32 matrix (outer rows x inner words), no swizzle: packed 4-bit codes.
cudaError_t make_tmap_u32(CUtensorMap* m, const void* base, uint64_t inner, uint64_t outer, uint32_t box_inner,
                          uint32_t box_outer) {
    EncodeTiledFn enc = encode_fn();
    if (!enc) return cudaErrorNotSupported;
    const cuuint64_t dims[2] = {inner, outer};
    const cuuint64_t strides[1] = {inner * 4};
    const cuuint32_t box[2] = {box_inner, box_outer};
    const cuuint32_t estr[2] = {1, 1};
    CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_UINT32, 2, const_cast<void*>(base), dims, strides, box, estr,
                     CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                     CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

template <int MODE, int BN, int STAGES, int WFMT, int PAIR = 0>
cudaError_t run(const ExpertArgs& a, const GemmParams& g, const void* wbase, bool pdl, cudaStream_t s) {
    CUtensorMap tA, tB;
    using C = Cfg<MODE, BN, WFMT, PAIR>;
    const uint32_t a_box = C::kABox;
    const uint32_t b_box = BN < 64 ? 16 : 64;
    cudaError_t e;
    if (WFMT)   // 8 code words (64 codes) of one k-block per row
        e = make_tmap_u32(&tA, wbase, (uint64_t)g.K / 8, (uint64_t)g.E_w * g.rows_per_expert, 8, a_box);
    else
        e = make_tmap(&tA, wbase, (uint64_t)g.K, (uint64_t)g.E_w * g.rows_per_expert, kBK, a_box);
    if (e != cudaSuccess) return e;
    if (MODE == kDown) {
        e = make_tmap(&tB, a.h, (uint64_t)a.I, (uint64_t)a.T * a.k, kBK, b_box);
    } else if (g.dense_n) {
        e = make_tmap(&tB, a.x, (uint64_t)a.H, (uint64_t)a.T, kBK, b_box);          // x itself, rows 0..T-1
    } else {
        e = make_tmap(&tB, a.xs, (uint64_t)a.H, (uint64_t)a.T * a.k, kBK, b_box);   // rows gathered in plan order
    }
    if (e != cudaSuccess) return e;
    auto kern = k_gemm<MODE, BN, STAGES, WFMT, PAIR>;
    using L = Smem<BN, STAGES, C::kAStage, C::kCStage, C::kHalves, (C::kCStage ? kSBDepth * 2 * kDq * 4 : 0),
                   C::kBRows>;   // the kernel's own layout
    static_assert(L::kBytes <= 227 * 1024, "shared memory of one CTA");
    const size_t smem = L::kBytes;
    if ((e = ensure_smem(kern, smem)) != cudaSuccess) return e;
    if (PAIR)   // one CTA per SM, in pairs on neighbouring SMs
        return launch_k_pair(kern, dim3(device_info().sm_count & ~1), dim3(kThreads), smem, s, pdl, tA, tB, g);
    return launch_k(kern, dim3(device_info().sm_count), dim3(WFMT ? kThreadsA4 : kThreads), smem, s, pdl, tA,
                    tB, g);
}

// Token-tile width from the mean pairs per expert.
int pick_bn(const ExpertArgs& a) {
    const double mean = (double)a.T * a.k / a.E;
    if (mean <= 24.0) return 32;
    if (mean <= 96.0) return 128;
    return 256;
}

GemmParams params(const ExpertArgs& a, bool up) {
    GemmParams g{};
    g.counts = a.counts;
    g.offsets = a.offsets;
    g.perm = a.perm;
    g.topk_w = a.topk_w;
    g.x = a.x;
    g.h = a.h;
    g.y_acc = a.y_acc;
    g.ordered = a.ordered;
    g.E = a.E;
    g.k = a.k;
    g.H = a.H;
    g.I = a.I;
    g.skip = a.skip;
    g.E_w = a.E_w;
    g.wait_limit = kWaitLimit;
    g.err = a.err;
    if (up) {
        g.K = a.H;
        g.rows_per_expert = a.act == 0 ? 2 * a.I : a.I;
        g.feats = a.I;
        g.wscale = a.w1_scale;
        g.wbias = a.w1_bias;
        g.wglobal = a.w1_global;
        g.swiglu_limit = a.swiglu_limit;
    } else {
        g.K = a.I;
        g.rows_per_expert = a.H;
        g.feats = a.H;
        g.wscale = a.w2_scale;
        g.wbias = a.w2_bias;
        g.wglobal = a.w2_global;
    }
    return g;
}

// xs[pos] = x[perm[pos] / k]: token rows in plan order, one warp per row.
// The rows are stored L2 evict-last: the up GEMM reads them next, once per
// weight tile of their expert.
__global__ void __launch_bounds__(256) k_gather_rows(const uint16_t* __restrict__ x, const int32_t* __restrict__ perm,
                                                     uint16_t* __restrict__ xs, int P, int k, int H) {
    pdl_wait();
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int n16 = H / 8;
    const uint64_t keep = policy_evict_last();
    for (int pos = blockIdx.x * 8 + warp; pos < P; pos += gridDim.x * 8) {
        const uint4* src = reinterpret_cast<const uint4*>(x + (size_t)(perm[pos] / k) * H);
        uint4* dst = reinterpret_cast<uint4*>(xs + (size_t)pos * H);
        for (int c = lane; c < n16; c += 32) st_hint(dst + c, ld_nc(src + c), keep);
    }
    pdl_trigger();
}

}  // namespace


// bf16 experts at T <= 16 tokens: every up tile multiplies all T token rows
// of x (N = T rounded up to 16) and keeps the columns of the tokens routed to
// its expert, so no rows are gathered into plan order first.
bool gemm_up_reads_x(const ExpertArgs& a) { return a.fmt == 0 && a.T > 0 && a.T <= 16 && a.x != nullptr; }

cudaError_t launch_gather_x(const ExpertArgs& a, bool pdl, cudaStream_t s) {
    const int P = a.T * a.k;
    if (P == 0) return cudaSuccess;
    const int blocks = min((P + 7) / 8, device_info().sm_count * 16);
    return launch_k(k_gather_rows, dim3(blocks), dim3(256), 0, s, pdl, a.x, a.perm, a.xs, P, a.k, a.H);
}

namespace {

// 4-bit experts (WFMT 1 affine, 2 NVFP4): codes dequantised on chip.
template <int WFMT>
cudaError_t gemm_up_q4(const ExpertArgs& a, const GemmParams& g, int bn, bool pdl, cudaStream_t s) {
    if (a.act == 0) {
        if (bn == 32) return run<kUpSwiglu, 32, 8, WFMT>(a, g, a.w1, pdl, s);
        if (bn == 128) return run<kUpSwiglu, 128, 5, WFMT>(a, g, a.w1, pdl, s);   // inter layout
        return run<kUpSwiglu, 256, 3, WFMT>(a, g, a.w1, pdl, s);                   // inter layout, 256 tokens
    }
    if (bn == 32) return run<kUpRelu2, 32, 8, WFMT>(a, g, a.w1, pdl, s);
    if (bn == 128) return run<kUpRelu2, 128, 5, WFMT>(a, g, a.w1, pdl, s);
    return run<kUpRelu2, 256, 4, WFMT>(a, g, a.w1, pdl, s);
}

template <int WFMT>
cudaError_t gemm_down_q4(const ExpertArgs& a, const GemmParams& g, int bn, bool pdl, cudaStream_t s) {
    if (bn == 32) return run<kDown, 32, 8, WFMT>(a, g, a.w2, pdl, s);
    if (bn == 128) return run<kDown, 128, 5, WFMT>(a, g, a.w2, pdl, s);
    return run<kDown, 256, 4, WFMT>(a, g, a.w2, pdl, s);
}

}  // namespace

cudaError_t launch_gemm_up(const ExpertArgs& a, bool pdl, cudaStream_t s) {
    GemmParams g = params(a, true);
    const int bn = pick_bn(a);
    if (gemm_up_reads_x(a)) g.dense_n = (a.T + 15) & ~15;
    if (a.fmt == 0) {
        // token tiles of 128 and more: M = 256 tiles on SM pairs
        if (a.act == 0) {
            // bf16 SwiGLU keeps one CTA per tile with two accumulators: measured
            // faster in the benchmark loop than either layout on SM pairs
            if (bn == 32) return run<kUpSwiglu, 32, 8, 0>(a, g, a.w1, pdl, s);
            return run<kUpSwiglu, 128, 4, 0>(a, g, a.w1, pdl, s);   // two accumulators: 4 x 128 TMEM columns
        }
        if (bn == 32) return run<kUpRelu2, 32, 8, 0>(a, g, a.w1, pdl, s);
        if (bn == 128) return run<kUpRelu2, 128, 8, 0, 1>(a, g, a.w1, pdl, s);
        return run<kUpRelu2, 256, 6, 0, 1>(a, g, a.w1, pdl, s);
    }
    if (a.fmt == 1) return gemm_up_q4<1>(a, g, bn, pdl, s);
    if (a.fmt == 2) return gemm_up_q4<2>(a, g, bn, pdl, s);
    return cudaErrorNotSupported;
}

cudaError_t launch_gemm_down(const ExpertArgs& a, bool pdl, cudaStream_t s) {
    const GemmParams g = params(a, false);
    const int bn = pick_bn(a);
    if (a.fmt == 0) {
        if (bn == 32) return run<kDown, 32, 8, 0>(a, g, a.w2, pdl, s);
        if (bn == 128) return run<kDown, 128, 8, 0, 1>(a, g, a.w2, pdl, s);
        return run<kDown, 256, 6, 0, 1>(a, g, a.w2, pdl, s);
    }
    if (a.fmt == 1) return gemm_down_q4<1>(a, g, bn, pdl, s);
    if (a.fmt == 2) return gemm_down_q4<2>(a, g, bn, pdl, s);
    return cudaErrorNotSupported;
}

cudaError_t make_tmap_2d(CUtensorMap* m, CUtensorMapDataType dtype, uint32_t elem_bytes, const void* base,
                         uint64_t inner, uint64_t rows, uint32_t box_inner, uint32_t box_rows, bool swizzle128) {
    EncodeTiledFn enc = encode_fn();
    if (!enc) return cudaErrorNotSupported;
    const cuuint64_t dims[2] = {inner, rows};
    const cuuint64_t strides[1] = {inner * elem_bytes};
    const cuuint32_t box[2] = {box_inner, box_rows};
    const cuuint32_t estr[2] = {1, 1};
    CUresult r = enc(m, dtype, 2, const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                     swizzle128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_NONE,
                     CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

}  // namespace moe
