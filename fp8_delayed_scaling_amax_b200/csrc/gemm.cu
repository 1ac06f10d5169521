// FP8 x FP8 -> bf16 GEMM with dequantization and fused bias, on the sm_100a tensor cores.
//
// Computes  out[b][i][j] = RN_bf16( acc[b][i][j] * RN32(sa * sb) + bias[j] ),
//           acc = sum_k A[b][i][k] * B[b][k][j]   (fp32, tcgen05.mma kind::f8f6f4)
// for the four operand layouts and batched / broadcast operands.  Definition: AstrAI compare
// view 3e57cc8...main -- astrai/extension/ops/fp8.py (mm_fp8), csrc/kernels/fp8/common.h
// (RowMajor / ColMajor operand tags, FP8Params batch strides), csrc/kernels/fp8/gemm/
// epilogue.cuh (bias added to the fp32 accumulator before the single bf16 rounding) and the
// extension commit log (bias_scale: fp8 bias dequantized after the operand scaling).
//
// B200 design (the pages' sm_89 mma.sync / cp.async / ldmatrix design is not used):
//  * persistent grid, one CTA (or CTA pair) per SM, static schedule: tiles in grouped-raster
//    order, dealt to the CTAs boustrophedon-wise (odd rounds in reverse), the problem with the
//    longer K first when a launch carries two;
//  * warp 0 = TMA producer: 3-D tensor maps (K-major or MN-major), 128-byte swizzle, into a
//    ring of shared-memory stages guarded by full / empty mbarriers;
//  * warp 1 = MMA issuer: one thread issues tcgen05.mma (M = 128, N = BN, K = 32) into a
//    TMEM accumulator; tcgen05.commit releases each stage and, per tile, hands the
//    accumulator to the epilogue.  Two accumulators (2 x BN TMEM columns) let the epilogue
//    of tile i overlap the MMAs of tile i + 1;
//  * warps 2.. = epilogue (8 warps where shared memory allows, two per TMEM lane quarter, else
//    4): tcgen05.ld 64 columns at a time, fma with the combined scale and the bias, round to
//    bf16, stage each warp's 32 x 64 box in 128-byte-swizzled shared memory and write it with
//    a TMA bulk-tensor store (double-buffered per warp);
//  * CTA pairs: 256 x 256 tiles with one tcgen05.mma.cta_group::2 (M = 256) spanning both SMs,
//    each SM holding 128 rows of A and half of B; pair loads complete on the leader's barriers;
//  * one launch may carry two GEMMs over one tile space (the backward's dX and dW), and its
//    epilogue warps can first reduce the bias-gradient column sums (a side job, no launch).
//  * separate instances for split-K (an output tile's K range cut across CTAs: contributors
//    leave fp32 partials, the owner adds them after a bounded acquire wait; opt-in) and for
//    the fp8-output epilogue (the bf16 values also quantized at a given step, with their
//    amax), so the plain instance carries neither;
//  * every wait is bounded (globaltimer); on expiry the CTA records a status code, drains its
//    in-flight copies and MMAs, frees TMEM and returns.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>
#include <cuda_bf16.h>

#include <algorithm>
#include <atomic>
#include <cstdlib>
#include <mutex>
#include <string>
#include <vector>

#include "internal.h"

namespace fp8dsa {
namespace {

constexpr int kBM = 128;      // tile rows (TMEM lanes)
constexpr int kBK = 128;      // K bytes per stage (one 128-byte swizzle row)
constexpr int kUmmaK = 32;    // K per tcgen05.mma for 8-bit operands

constexpr int kOutBox = 64;                       // output columns per TMA store (128 bytes of bf16)
constexpr int kOutStageBytes = 32 * kOutBox * 2;  // one warp's 32 rows x 64 columns
#ifndef FP8DSA_GEMM_OUT_BUFS
#define FP8DSA_GEMM_OUT_BUFS 1
#endif
constexpr int kOutBufs = FP8DSA_GEMM_OUT_BUFS;    // staged boxes per epilogue warp (TMA stores in flight)
constexpr int kMaxStages = 8;
#ifndef FP8DSA_GEMM_GROUP_M
#define FP8DSA_GEMM_GROUP_M 16  // tile rows per group of the grouped raster
#endif
#ifndef FP8DSA_GEMM_EPI_WARPS
#define FP8DSA_GEMM_EPI_WARPS 8  // at most this many epilogue warps (8 or 4)
#endif
constexpr int kSmemLimit = 232448;                // dynamic shared memory per CTA on sm_100
constexpr int kMaxProblems = 2;

// kPair: a 2-CTA cluster computes a 256 x BN tile with one M = 256 MMA across both SMs; each CTA
// holds 128 rows of A and BN/2 rows of B, so each SM's shared memory feeds half the B operand.
// Epilogue warps: 8 (two per TMEM lane quarter, each owning half the columns) for tiles at
// least 128 wide when the stages leave room for their staging buffers, else 4.  BN = 64
// (single CTA, K-major B) serves short, wide problems: more tiles, so more SMs stream B.
template <int BN, bool kPair>
struct Cfg {
    static constexpr int kTileM = kPair ? 2 * kBM : kBM;
    static constexpr int kBRows = kPair ? BN / 2 : BN;  // rows of B (along N) this CTA loads
    static constexpr int kAStage = kBM * kBK;
    static constexpr int kBStage = kBRows * kBK;
    // N of one MMA instruction (at most 256); a 512-wide pair tile issues two per K step, into
    // TMEM columns 0..255 and 256..511, and has a single accumulator (the tile fills TMEM)
    static constexpr int kMmaN = BN > 256 ? 256 : BN;
    static constexpr int kNMma = BN / kMmaN;
    static constexpr int kAccBufs = 2 * BN <= 512 ? 2 : 1;
    static constexpr int kTmemCols = kAccBufs * BN;
    static constexpr int kEpiWarps =
        (FP8DSA_GEMM_EPI_WARPS >= 8 && BN >= 128 && ((kAStage + kBStage) <= 32768 || BN == 512)) ? 8 : 4;
    static constexpr int kThreads = 64 + 32 * kEpiWarps;
    static constexpr int kEpiThreads = 32 * kEpiWarps;
    static constexpr int kEpiCols = BN / (kEpiWarps / 4);  // columns of the tile each epilogue warp owns
    static constexpr int kOutBytes = kEpiWarps * kOutBufs * kOutStageBytes;
    static constexpr int kBarBytes = 256;
    static constexpr int kFixed = 1024 + kOutBytes + kBarBytes;
    static constexpr int kStagesFit = (kSmemLimit - kFixed) / (kAStage + kBStage);
    static constexpr int kStages = kStagesFit < kMaxStages ? kStagesFit : kMaxStages;
    static_assert(kEpiCols % kOutBox == 0, "each epilogue warp owns whole 64-column boxes");
    static_assert(!kPair || BN >= 128, "pair tiles are at least 128 wide");
    static_assert(kPair || BN <= 256, "single-CTA tiles are at most 256 wide");
    static_assert(kTmemCols <= 512, "accumulators exceed TMEM");
    static constexpr int kSmem = kFixed + kStages * (kAStage + kBStage);
    static constexpr uint32_t kTxBytes = (kPair ? 2u : 1u) * (kAStage + kBStage);
    static_assert(kStages >= 3, "too few pipeline stages");
};

// One GEMM of a launch (a launch may carry two, e.g. dX and dW, over one tile space).
struct GemmProblem {
    int m, n, k_blocks;
    int tiles_m, tiles_n, tile_begin, tiles;  // tiles: all tiles of the problem (batch included)
    int k_splits;                             // K ranges per tile (1 = no split)
    int contrib_begin, owner_begin;           // first contributor unit / first owner (see decode_unit)
    int a_batched, b_batched;
    int a_mn, b_mn;
    uint32_t idesc;
    uint32_t idesc_half;  // the same MMA with N = 128 (a half tile of the last round)
    uint16_t* out;
    int64_t ldo, stride_o;
    int vec_out;
    int tma_out;  // stage the tile in shared memory and write it with TMA bulk-tensor stores
    const void* bias;
    int bias_kind;  // 0 none, 1 bf16, 2 fp8 e4m3 * bias_scale, 3 fp8 e5m2 * bias_scale
    const float* bias_scale;
    const float* scale_a;
    const float* scale_b;
    // fp8 output (see GemmDesc): null = none
    uint8_t* out8;
    int out8_fmt;
    int out8_vec;  // out8, ldo and stride_o allow 16-byte stores
    const float* out8_step;
    float* out8_amax;
    float* out8_step_used;
};

// Optional side job of the epilogue warps, done before their first tile: the bias gradient
// out[c] = RN_bf16(sum_t partial[t][c]), summed in order t = 0, 1, ...
struct ColsumJob {
    const float* partial;
    int tiles, cols;
    uint16_t* out;
};

// A history ring whose quantize launch left its fold to this launch.
constexpr int kMaxFolds = 3;
struct RingFold {
    float* state;
    int hist_len, hist_idx;
    float fp8_max, pow2_margin;
};

struct GemmArgs {
    GemmProblem p[kMaxProblems];
    RingFold folds[kMaxFolds];
    int nfolds;
    int nprob;
    int num_tiles;
    int num_units, contrib_units;  // work units (tile, K range); the first contrib_units are split-K contributors
    int half_begin;                // (no split-K) tiles from here on are run as two 256 x 128 halves
    int splitk;                    // some problem has k_splits > 1
    float* partial;                // split-K fp32 partial tiles: [contrib unit][CTA of the pair][BN/4][128][4]
    uint32_t* counters;            // split-K arrivals per (tile, CTA of the pair); zero at launch
    ColsumJob colsum;
    WaitCtl wait;
};

// UMMA shared-memory matrix descriptor: 128-byte swizzle, sm_100 descriptor version.
__device__ __forceinline__ uint64_t smem_desc(uint32_t saddr, uint32_t lbo, uint32_t sbo) {
    uint64_t d = 0;
    d |= static_cast<uint64_t>((saddr >> 4) & 0x3FFFu);
    d |= static_cast<uint64_t>((lbo >> 4) & 0x3FFFu) << 16;
    d |= static_cast<uint64_t>((sbo >> 4) & 0x3FFFu) << 32;
    d |= static_cast<uint64_t>(1) << 46;  // descriptor version (sm_100)
    d |= static_cast<uint64_t>(2) << 61;  // SWIZZLE_128B
    return d;
}

// Tile -> (problem, batch, tile row, tile column); grouped raster of FP8DSA_GEMM_GROUP_M tile rows per problem.
__device__ __forceinline__ void decode_tile(int tile, const GemmArgs& g, int& pi, int& b, int& tm, int& tn) {
    constexpr int kGroupM = FP8DSA_GEMM_GROUP_M;
    pi = (g.nprob > 1 && tile >= g.p[1].tile_begin) ? 1 : 0;
    const GemmProblem& P = g.p[pi];
    const int t = tile - P.tile_begin;
    const int per = P.tiles_m * P.tiles_n;
    b = t / per;
    const int r = t - b * per;
    const int group = kGroupM * P.tiles_n;
    const int gi = r / group;
    const int first_m = gi * kGroupM;
    const int gm = min(P.tiles_m - first_m, kGroupM);
    const int within = r - gi * group;
    tm = first_m + within % gm;
    tn = within / gm;
}

// Work unit -> (problem, tile, split, k-block range).  Without split-K a unit is a whole tile.
// With it, tile t of problem p is cut into p.k_splits contiguous K ranges: the range s >= 1
// is a contributor unit, which leaves its fp32 partial sum in the workspace; the range 0 is
// the tile's owner, which adds the contributors' partials (in order s = 1, 2, ...) to its own
// accumulator and writes the output.  Units [0, contrib_units) are all contributors (problem
// by problem, split-major, tiles in order), the owners follow, problem by problem.  Every
// CTA walks its units in increasing order and every contributor precedes its owner, so an
// owner only ever waits for units that never wait themselves.
struct Unit {
    int pi, tile, split, kb0, kb1;
    int half;  // -1: the whole tile; 0 / 1: its left / right 128 columns
};

template <bool kSplit>
__device__ __forceinline__ Unit decode_unit(int u, const GemmArgs& g) {
    Unit r;
    r.half = -1;
    if constexpr (!kSplit) {  // one unit per tile, or per half of the tiles from half_begin on
        if (u >= g.half_begin) {
            r.tile = g.half_begin + ((u - g.half_begin) >> 1);
            r.half = (u - g.half_begin) & 1;
        } else {
            r.tile = u;
        }
        r.pi = (g.nprob > 1 && r.tile >= g.p[1].tile_begin) ? 1 : 0;
        r.split = 0;
        r.kb0 = 0;
        r.kb1 = g.p[r.pi].k_blocks;
        return r;
    }
    if (u < g.contrib_units) {
        r.pi = (g.nprob > 1 && u >= g.p[1].contrib_begin) ? 1 : 0;
        const GemmProblem& P = g.p[r.pi];
        const int local = u - P.contrib_begin;
        r.split = 1 + local / P.tiles;
        r.tile = P.tile_begin + local % P.tiles;
    } else {
        const int o = u - g.contrib_units;
        r.pi = (g.nprob > 1 && o >= g.p[1].owner_begin) ? 1 : 0;
        const GemmProblem& P = g.p[r.pi];
        r.split = 0;
        r.tile = P.tile_begin + (o - P.owner_begin);
    }
    const GemmProblem& P = g.p[r.pi];
    r.kb0 = (r.split * P.k_blocks) / P.k_splits;
    r.kb1 = ((r.split + 1) * P.k_blocks) / P.k_splits;
    return r;
}

// The unit a CTA (or pair) `unit` of `units` takes in round r: rounds alternate direction
// (boustrophedon), so a CTA that drew a long unit in one round draws a short one in the next
// when the units are ordered longest first.  Each CTA's units still increase with r.
__device__ __forceinline__ int snake_unit(int r, int unit, int units) {
    return r * units + ((r & 1) ? units - 1 - unit : unit);
}

// Contributor unit index of split s (>= 1) of tile `tile` of problem P.
__device__ __forceinline__ int contrib_slot(const GemmProblem& P, int tile, int s) {
    return P.contrib_begin + (s - 1) * P.tiles + (tile - P.tile_begin);
}

// Named barrier over `nthreads` threads that also returns whether any of them passed true.
__device__ __forceinline__ bool named_barrier_or(int id, int nthreads, bool pred) {
    uint32_t r;
    asm volatile(
        "{\n\t.reg .pred p, q;\n\t"
        "setp.ne.u32 p, %1, 0;\n\t"
        "bar.red.or.pred q, %2, %3, p;\n\t"
        "selp.u32 %0, 1, 0, q;\n\t}"
        : "=r"(r)
        : "r"(pred ? 1u : 0u), "r"(id), "r"(nthreads)
        : "memory");
    return r != 0;
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
    const __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<const uint32_t*>(&v);
}

__device__ __forceinline__ float bias_value(const GemmProblem& P, int col, float bsc) {
    if (col >= P.n || P.bias_kind == 0) return 0.0f;
    if (P.bias_kind == 1) return bf16_bits_to_float(__ldg(static_cast<const uint16_t*>(P.bias) + col));
    const uint8_t v = __ldg(static_cast<const uint8_t*>(P.bias) + col);
    return __fmul_rn(P.bias_kind == 2 ? fp8_to_float<0>(v) : fp8_to_float<1>(v), bsc);
}

template <int BN, bool kPair, bool kSplit, bool kOut8>
__global__ void __launch_bounds__(Cfg<BN, kPair>::kThreads, 1)
    fp8_gemm_kernel(const __grid_constant__ CUtensorMap tma_a0, const __grid_constant__ CUtensorMap tma_b0,
                    const __grid_constant__ CUtensorMap tma_o0, const __grid_constant__ CUtensorMap tma_a1,
                    const __grid_constant__ CUtensorMap tma_b1, const __grid_constant__ CUtensorMap tma_o1,
                    const __grid_constant__ CUtensorMap tma_bh0, const __grid_constant__ CUtensorMap tma_bh1,
                    const __grid_constant__ GemmArgs g) {
    using C = Cfg<BN, kPair>;
    constexpr int S = C::kStages;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t* sA = smem;
    uint8_t* sB = smem + S * C::kAStage;
    uint8_t* sOut = sB + S * C::kBStage;
    uint64_t* full = reinterpret_cast<uint64_t*>(sOut + C::kOutBytes);
    uint64_t* empty = full + S;
    uint64_t* acc_full = empty + S;
    uint64_t* acc_empty = acc_full + 2;
    uint64_t* drain = acc_empty + 2;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

    pdl_trigger();
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const uint32_t rank = kPair ? cluster_ctarank() : 0u;
    const bool leader = rank == 0;
    const int unit = kPair ? static_cast<int>(blockIdx.x >> 1) : static_cast<int>(blockIdx.x);
    const int units = kPair ? static_cast<int>(gridDim.x >> 1) : static_cast<int>(gridDim.x);

    if (threadIdx.x == 0) {
        for (int s = 0; s < S; ++s) {
            mbar_init(full + s, 1);
            mbar_init(empty + s, 1);
        }
        for (int a = 0; a < C::kAccBufs; ++a) {
            mbar_init(acc_full + a, 1);
            // the leader's accumulator is released by both CTAs' epilogue threads
            mbar_init(acc_empty + a, C::kEpiThreads * (kPair ? 2 : 1));
        }
        mbar_init(drain, 1);
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 0 && lane == 0) {
        prefetch_tensormap(&tma_a0);
        prefetch_tensormap(&tma_b0);
        if (g.p[0].tma_out) prefetch_tensormap(&tma_o0);
        if (g.nprob > 1) {
            prefetch_tensormap(&tma_a1);
            prefetch_tensormap(&tma_b1);
            if (g.p[1].tma_out) prefetch_tensormap(&tma_o1);
        }
    }
    if (warp == 1) {
        if constexpr (kPair) {
            tmem_alloc_pair(tmem_slot, C::kTmemCols);
            tmem_relinquish_pair();
        } else {
            tmem_alloc(tmem_slot, C::kTmemCols);
            tmem_relinquish();
        }
    }
    tc_fence_before_sync();
    __syncthreads();
    if constexpr (kPair) cluster_sync();  // the peer's loads target the leader's initialised barriers
    tc_fence_after_sync();
    const uint32_t tmem_base = *tmem_slot;
    pdl_wait();  // the operands and steps come from the previous kernels

    if (warp == 0) {
        // ------------------------------------------------------------------ TMA producer
        if (lane == 0) {
            int stage = 0;
            uint32_t phase = 0;
            uint32_t issued = 0, issued_parity = 0;  // per-stage: ever issued, parity of the last issue
            bool ok = true;
            for (int r = 0, u = unit; u < g.num_units && ok; u = snake_unit(++r, unit, units)) {
                const Unit w = decode_unit<kSplit>(u, g);
                int pi, b, tm, tn;
                decode_tile(w.tile, g, pi, b, tm, tn);
                const GemmProblem& P = g.p[pi];
                const CUtensorMap* ta = pi ? &tma_a1 : &tma_a0;
                // a half tile (pairs, K-major B only): each CTA loads 64 rows of B through the
                // 64-row map, and the stage carries that many fewer bytes
                const bool half = kPair && w.half >= 0;
                const CUtensorMap* tb = half ? (pi ? &tma_bh1 : &tma_bh0) : (pi ? &tma_b1 : &tma_b0);
                const int ba = P.a_batched ? b : 0;
                const int bb = P.b_batched ? b : 0;
                const int arow = tm * C::kTileM + static_cast<int>(rank) * kBM;
                const int brow = half ? tn * BN + w.half * 128 + static_cast<int>(rank) * 64
                                      : tn * BN + static_cast<int>(rank) * C::kBRows;
                const uint32_t tx = half ? C::kTxBytes - (kPair ? 2u : 1u) * (C::kBStage / 2) : C::kTxBytes;
                for (int kb = w.kb0; kb < w.kb1; ++kb) {
                    if (!mbar_wait_bounded(empty + stage, phase ^ 1u, g.wait, abort_flag, kStatusWaitProducer)) {
                        ok = false;
                        break;
                    }
                    if (leader) mbar_arrive_expect_tx(full + stage, tx);
                    uint8_t* a_dst = sA + stage * C::kAStage;
                    uint8_t* b_dst = sB + stage * C::kBStage;
                    if constexpr (kPair) {
                        const uint32_t fb = mapa_shared(smem_addr(full + stage), 0);
                        if (!P.a_mn)
                            tma_load_3d_pair(a_dst, ta, fb, kb * kBK, arow, ba);
                        else
                            tma_load_3d_pair(a_dst, ta, fb, arow, kb * kBK, ba);
                        if (!P.b_mn) {
                            if constexpr (C::kNMma == 1) {
                                tma_load_3d_pair(b_dst, tb, fb, kb * kBK, brow, bb);
                            } else {
                                // this CTA's half of each MMA's 256 columns: rows j * 256 + rank * 128
#pragma unroll
                                for (int j = 0; j < C::kNMma; ++j)
                                    tma_load_3d_pair(b_dst + j * (C::kMmaN / 2) * kBK, tb, fb, kb * kBK,
                                                     tn * BN + j * C::kMmaN + static_cast<int>(rank) * (C::kMmaN / 2), bb);
                            }
                        } else {
#pragma unroll
                            for (int h = 0; h < C::kBRows / 128; ++h)
                                tma_load_3d_pair(b_dst + h * 128 * kBK, tb, fb, brow + h * 128, kb * kBK, bb);
                        }
                    } else {
                        if (!P.a_mn)
                            tma_load_3d(a_dst, ta, full + stage, kb * kBK, arow, ba);
                        else
                            tma_load_3d(a_dst, ta, full + stage, arow, kb * kBK, ba);
                        if (!P.b_mn) {
                            tma_load_3d(b_dst, tb, full + stage, kb * kBK, brow, bb);
                        } else {
#pragma unroll
                            for (int h = 0; h < C::kBRows / 128; ++h)
                                tma_load_3d(b_dst + h * 128 * kBK, tb, full + stage, brow + h * 128, kb * kBK, bb);
                        }
                    }
                    issued |= 1u << stage;
                    issued_parity = (issued_parity & ~(1u << stage)) | (phase << stage);
                    if (++stage == S) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
            }
            if (!ok && leader) {
                // Let every copy already in flight land before the CTAs can exit (the leader's
                // full barriers also count the peer's bytes).
                for (int s = 0; s < S; ++s)
                    if (issued & (1u << s))
                        mbar_wait_bounded(full + s, (issued_parity >> s) & 1u, g.wait, nullptr, kStatusWaitDrain);
            }
        }
        __syncwarp();
    } else if (warp == 1) {
        // ------------------------------------------------------------------ MMA issuer (leader)
        if (leader) {
            int stage = 0, acc = 0;
            uint32_t phase = 0, acc_phase = 0;
            bool ok = true;
            constexpr uint32_t kLboB = 128 * kBK;  // distance between 128-wide MN blocks of B
            for (int r = 0, u = unit; u < g.num_units && ok; u = snake_unit(++r, unit, units)) {
                const Unit w = decode_unit<kSplit>(u, g);
                const GemmProblem& P = g.p[w.pi];
                const uint32_t idesc = w.half >= 0 ? P.idesc_half : P.idesc;
                const bool got = kPair ? mbar_wait_bounded_cluster(acc_empty + acc, acc_phase ^ 1u, g.wait, abort_flag,
                                                                   kStatusWaitMma)
                                       : mbar_wait_bounded(acc_empty + acc, acc_phase ^ 1u, g.wait, abort_flag,
                                                           kStatusWaitMma);
                if (!got) {
                    ok = false;
                    break;
                }
                tc_fence_after_sync();
                const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(acc * BN);
                for (int kb = w.kb0; kb < w.kb1; ++kb) {
                    if (!mbar_wait_bounded(full + stage, phase, g.wait, abort_flag, kStatusWaitMma)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after_sync();
                    if (lane == 0) {
                        const uint32_t a_base = smem_addr(sA + stage * C::kAStage);
                        const uint32_t b_base = smem_addr(sB + stage * C::kBStage);
#pragma unroll
                        for (int kk = 0; kk < kBK / kUmmaK; ++kk) {
                            // K-major: step 32 bytes along the swizzled row; MN-major: step 32 rows.
                            const uint64_t ad = P.a_mn ? smem_desc(a_base + kk * kUmmaK * 128, C::kAStage, 1024)
                                                       : smem_desc(a_base + kk * kUmmaK, 16, 1024);
                            const uint64_t bd = P.b_mn ? smem_desc(b_base + kk * kUmmaK * 128, kLboB, 1024)
                                                       : smem_desc(b_base + kk * kUmmaK, 16, 1024);
                            const uint32_t accumulate = (kb != w.kb0 || kk != 0) ? 1u : 0u;
#pragma unroll
                            for (int j = 0; j < C::kNMma; ++j) {
                                // the j-th 256 columns: B rows j * (kMmaN / 2) of this CTA's stage
                                const uint64_t bdj = bd + ((static_cast<uint64_t>(j * (C::kMmaN / 2) * kBK) >> 4) & 0x3FFFu);
                                const uint32_t dj = d_tmem + static_cast<uint32_t>(j * C::kMmaN);
                                if constexpr (kPair)
                                    umma_f8f6f4_pair(dj, ad, bdj, idesc, accumulate);
                                else
                                    umma_f8f6f4(dj, ad, bdj, idesc, accumulate);
                            }
                        }
                        if constexpr (kPair)
                            umma_commit_pair_multicast(empty + stage, 0x3);
                        else
                            umma_commit(empty + stage);
                    }
                    __syncwarp();
                    if (++stage == S) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
                if (!ok) break;
                if (lane == 0) {
                    if constexpr (kPair)
                        umma_commit_pair_multicast(acc_full + acc, 0x3);
                    else
                        umma_commit(acc_full + acc);
                }
                __syncwarp();
                if (++acc == C::kAccBufs) {
                    acc = 0;
                    acc_phase ^= 1u;
                }
            }
            // Every MMA this thread issued must complete before TMEM is released.
            if (lane == 0) {
                if constexpr (kPair)
                    umma_commit_pair(drain);
                else
                    umma_commit(drain);
                mbar_wait_bounded(drain, 0, g.wait, nullptr, kStatusWaitDrain);
            }
        }
        __syncwarp();
    } else {
        // ------------------------------------------------------------------ epilogue
        // Warp w may read TMEM lanes 32*(w%4) .. +31, i.e. rows 32*(w%4) + lane of this CTA's
        // 128-row half of the tile; with 8 epilogue warps, warps w and w+4 split the columns.
        // Per 64 output columns: two 32-column TMEM loads, acc * scale + bias in fp32, one
        // bf16 rounding, then either a swizzled shared-memory stage + TMA bulk store of the
        // warp's 32 x 64 box (double-buffered), or direct 128-bit stores.
        const int ew = warp - 2;
        const int q = warp & 3;
        const int cbase = (ew >> 2) * C::kEpiCols;
        uint8_t* my_stage = sOut + ew * kOutBufs * kOutStageBytes;

        // side job: the deferred ring folds of the quantize launch before (one thread)
        if (g.nfolds > 0 && blockIdx.x == 0 && ew == 0 && lane == 0) {
            for (int f = 0; f < g.nfolds; ++f)
                ring_fold_deferred(g.folds[f].state, g.folds[f].hist_len, g.folds[f].hist_idx, g.folds[f].fp8_max,
                                   g.folds[f].pow2_margin);
        }
        // side job: the bias gradient from the per-tile column sums (before the first tile)
        if (g.colsum.tiles > 0) {
            const int et = ew * 32 + lane;
            const int per_cta = C::kEpiThreads;
            for (int c = static_cast<int>(blockIdx.x) * per_cta + et; c < g.colsum.cols;
                 c += static_cast<int>(gridDim.x) * per_cta) {
                const float* col = g.colsum.partial + c;
                float sum = 0.0f;
                int t = 0;
                for (; t + 4 <= g.colsum.tiles; t += 4) {
                    const float v0 = __ldcg(col + static_cast<int64_t>(t) * g.colsum.cols);
                    const float v1 = __ldcg(col + static_cast<int64_t>(t + 1) * g.colsum.cols);
                    const float v2 = __ldcg(col + static_cast<int64_t>(t + 2) * g.colsum.cols);
                    const float v3 = __ldcg(col + static_cast<int64_t>(t + 3) * g.colsum.cols);
                    sum += v0;
                    sum += v1;
                    sum += v2;
                    sum += v3;
                }
                for (; t < g.colsum.tiles; ++t) sum += __ldcg(col + static_cast<int64_t>(t) * g.colsum.cols);
                g.colsum.out[c] = __bfloat16_as_ushort(__float2bfloat16_rn(sum));
            }
        }

        float sc[kMaxProblems], bsc[kMaxProblems];
#pragma unroll
        for (int i = 0; i < kMaxProblems; ++i) {
            sc[i] = 0.0f;
            bsc[i] = 0.0f;
            if (i < g.nprob) {
                sc[i] = __fmul_rn(__ldg(g.p[i].scale_a), __ldg(g.p[i].scale_b));
                bsc[i] = g.p[i].bias_kind >= 2 ? __ldg(g.p[i].bias_scale) : 0.0f;
            }
        }
        // fp8 output: the multiplier RN32(1 / step) per problem, and the step snapshot
        float mult8[kMaxProblems];
#pragma unroll
        for (int i = 0; i < kMaxProblems; ++i) {
            mult8[i] = 0.0f;
            if (kOut8 && i < g.nprob && g.p[i].out8 != nullptr) {
                const float step8 = __ldg(g.p[i].out8_step);
                mult8[i] = __frcp_rn(step8);
                if (g.p[i].out8_step_used != nullptr && blockIdx.x == 0 && ew == 0 && lane == 0)
                    *g.p[i].out8_step_used = step8;
            }
        }
        const uint32_t acc_empty_leader0 = kPair ? mapa_shared(smem_addr(acc_empty), 0) : 0u;
        uint32_t am8 = 0u;  // running |max| of this thread's fp8-output values (bf16x2)
        int acc = 0, buf = 0;
        uint32_t acc_phase = 0;
        constexpr int kCtas = kPair ? 2 : 1;
        const int row_in = q * 32 + lane;  // this thread's row within the CTA's 128 rows
        for (int r = 0, u = unit; u < g.num_units; u = snake_unit(++r, unit, units)) {
            const Unit w = decode_unit<kSplit>(u, g);
            int pi, b, tm, tn;
            decode_tile(w.tile, g, pi, b, tm, tn);
            const GemmProblem& P = g.p[pi];
            const bool contrib = kSplit && w.split > 0;               // leave an fp32 partial sum
            const bool owner = kSplit && !contrib && P.k_splits > 1;  // add the partials, then write
            const CUtensorMap* to = pi ? &tma_o1 : &tma_o0;
            const float scale = pi ? sc[1] : sc[0];
            // a half tile's 128 accumulator columns: every epilogue warp takes 64 of them
            const int ncols = w.half >= 0 ? kOutBox : C::kEpiCols;
            const int cbase_u = w.half >= 0 ? (ew >> 2) * kOutBox : cbase;
            const int col0 = tn * BN + (w.half >= 0 ? w.half * 128 : 0) + cbase_u;
            const int row0 = tm * C::kTileM + static_cast<int>(rank) * kBM + q * 32;
            const int64_t row = static_cast<int64_t>(row0) + lane;
            // this warp's bias columns col0 + 32 j + lane in bias_r[j], loaded before the wait
            float bias_r[C::kEpiCols / 32];
#pragma unroll
            for (int j = 0; j < C::kEpiCols / 32; ++j) bias_r[j] = bias_value(P, col0 + 32 * j + lane, pi ? bsc[1] : bsc[0]);
            const bool got = mbar_wait_bounded(acc_full + acc, acc_phase, g.wait, abort_flag, kStatusWaitEpilogue);
            if constexpr (kSplit) {
                // split-K adds named barriers below: the epilogue warps leave together
                if (named_barrier_or(1, C::kEpiThreads, !got)) break;
            } else if (!got) {
                break;
            }
            tc_fence_after_sync();
            if (owner) {
                // one thread waits (acquire) until the tile's contributors have all arrived
                bool arrived = true;
                if (ew == 0 && lane == 0)
                    arrived = counter_wait_bounded(g.counters + 2 * w.tile + rank, static_cast<uint32_t>(P.k_splits - 1),
                                                   g.wait, abort_flag, kStatusWaitSplit);
                if (named_barrier_or(1, C::kEpiThreads, !arrived)) break;
            }
#pragma unroll
            for (int c = 0; c < C::kEpiCols; c += kOutBox) {
                if (c >= ncols) break;
                uint32_t r0[32], r1[32];
                const uint32_t taddr = tmem_base + (static_cast<uint32_t>(q * 32) << 16) +
                                       static_cast<uint32_t>(acc * BN + cbase_u + c);
                tmem_load_32cols(taddr, r0);
                tmem_load_32cols(taddr + 32, r1);
                const float b_lo = bias_r[c / 32];
                const float b_hi = bias_r[c / 32 + 1];
                tmem_wait_ld();
                const int cc = cbase_u + c;  // column within the tile
                // Partial tiles are stored as [column group of 4][row][4]: for each group the 32
                // lanes (rows) of a warp cover 512 contiguous bytes, one coalesced access.
                if (contrib) {
                    float4* dst = reinterpret_cast<float4*>(g.partial) +
                                  ((static_cast<int64_t>(u) * kCtas + rank) * (BN / 4) + cc / 4) * kBM + row_in;
#pragma unroll
                    for (int v = 0; v < 8; ++v) {
                        __stcg(dst + v * kBM, make_float4(__uint_as_float(r0[4 * v]), __uint_as_float(r0[4 * v + 1]),
                                                          __uint_as_float(r0[4 * v + 2]), __uint_as_float(r0[4 * v + 3])));
                        __stcg(dst + (8 + v) * kBM,
                               make_float4(__uint_as_float(r1[4 * v]), __uint_as_float(r1[4 * v + 1]),
                                           __uint_as_float(r1[4 * v + 2]), __uint_as_float(r1[4 * v + 3])));
                    }
                    continue;
                }
                if (owner) {
                    for (int sp = 1; sp < P.k_splits; ++sp) {
                        const float4* src =
                            reinterpret_cast<const float4*>(g.partial) +
                            ((static_cast<int64_t>(contrib_slot(P, w.tile, sp)) * kCtas + rank) * (BN / 4) + cc / 4) * kBM +
                            row_in;
#pragma unroll
                        for (int v = 0; v < 8; ++v) {
                            const float4 p0 = __ldcg(src + v * kBM);
                            const float4 p1 = __ldcg(src + (8 + v) * kBM);
                            r0[4 * v] = __float_as_uint(__uint_as_float(r0[4 * v]) + p0.x);
                            r0[4 * v + 1] = __float_as_uint(__uint_as_float(r0[4 * v + 1]) + p0.y);
                            r0[4 * v + 2] = __float_as_uint(__uint_as_float(r0[4 * v + 2]) + p0.z);
                            r0[4 * v + 3] = __float_as_uint(__uint_as_float(r0[4 * v + 3]) + p0.w);
                            r1[4 * v] = __float_as_uint(__uint_as_float(r1[4 * v]) + p1.x);
                            r1[4 * v + 1] = __float_as_uint(__uint_as_float(r1[4 * v + 1]) + p1.y);
                            r1[4 * v + 2] = __float_as_uint(__uint_as_float(r1[4 * v + 2]) + p1.z);
                            r1[4 * v + 3] = __float_as_uint(__uint_as_float(r1[4 * v + 3]) + p1.w);
                        }
                    }
                }
                uint32_t packed[32];
                if (P.bias_kind != 0) {
#pragma unroll
                    for (int e = 0; e < 16; ++e) {
                        const float v0 = fmaf(__uint_as_float(r0[2 * e]), scale, __shfl_sync(0xFFFFFFFFu, b_lo, 2 * e));
                        const float v1 = fmaf(__uint_as_float(r0[2 * e + 1]), scale, __shfl_sync(0xFFFFFFFFu, b_lo, 2 * e + 1));
                        packed[e] = pack_bf16x2(v0, v1);
                    }
#pragma unroll
                    for (int e = 0; e < 16; ++e) {
                        const float v0 = fmaf(__uint_as_float(r1[2 * e]), scale, __shfl_sync(0xFFFFFFFFu, b_hi, 2 * e));
                        const float v1 = fmaf(__uint_as_float(r1[2 * e + 1]), scale, __shfl_sync(0xFFFFFFFFu, b_hi, 2 * e + 1));
                        packed[16 + e] = pack_bf16x2(v0, v1);
                    }
                } else {
                    // no bias: the same fma with a zero addend, two lanes per packed instruction
#pragma unroll
                    for (int e = 0; e < 16; ++e) {
                        float v0 = __uint_as_float(r0[2 * e]), v1 = __uint_as_float(r0[2 * e + 1]);
                        fma2_rn(v0, v1, scale, 0.0f);
                        packed[e] = pack_bf16x2(v0, v1);
                    }
#pragma unroll
                    for (int e = 0; e < 16; ++e) {
                        float v0 = __uint_as_float(r1[2 * e]), v1 = __uint_as_float(r1[2 * e + 1]);
                        fma2_rn(v0, v1, scale, 0.0f);
                        packed[16 + e] = pack_bf16x2(v0, v1);
                    }
                }
                const int colg = col0 + c;
                if (P.tma_out) {
                    uint8_t* sb = my_stage + buf * kOutStageBytes;
                    if (lane == 0) bulk_wait_group_read<kOutBufs - 1>();  // the store that last used this buffer has read it
                    __syncwarp();
                    // 128-byte swizzle: 16-byte chunk j of row r sits at chunk j ^ (r % 8)
#pragma unroll
                    for (int j = 0; j < 8; ++j)
                        *reinterpret_cast<uint4*>(sb + lane * 128 + ((j ^ (lane & 7)) << 4)) =
                            make_uint4(packed[4 * j], packed[4 * j + 1], packed[4 * j + 2], packed[4 * j + 3]);
                    fence_proxy_async_smem();
                    __syncwarp();
                    if (lane == 0 && row0 < P.m && colg < P.n) {
                        tma_store_3d(to, sb, colg, row0, b);
                        bulk_commit_group();
                    }
                    buf = buf + 1 == kOutBufs ? 0 : buf + 1;
                } else if (P.out != nullptr && row < P.m && colg < P.n) {
                    uint16_t* orow = P.out + static_cast<int64_t>(b) * P.stride_o + row * P.ldo;
                    if (P.vec_out && colg + kOutBox <= P.n) {
                        uint4* dst = reinterpret_cast<uint4*>(orow + colg);
#pragma unroll
                        for (int v = 0; v < 8; ++v)
                            dst[v] = make_uint4(packed[4 * v], packed[4 * v + 1], packed[4 * v + 2], packed[4 * v + 3]);
                    } else {
#pragma unroll
                        for (int e = 0; e < kOutBox; ++e)
                            if (colg + e < P.n) orow[colg + e] = static_cast<uint16_t>(packed[e >> 1] >> (16 * (e & 1)));
                    }
                }
                if (kOut8 && P.out8 != nullptr && row < P.m && colg < P.n) {
                    // the same bf16 values, quantized: q(RN32(v * mult8)); amax over the valid ones
                    const float m8 = pi ? mult8[1] : mult8[0];
                    uint32_t q8[16];
#pragma unroll
                    for (int qd = 0; qd < 8; ++qd) {
                        uint32_t wv[4];
#pragma unroll
                        for (int e = 0; e < 4; ++e) {
                            wv[e] = packed[4 * qd + e];
                            // columns past n hold no output: keep them out of the amax
                            const int col = colg + 8 * qd + 2 * e;
                            if (col >= P.n) wv[e] = 0u;
                            else if (col + 1 >= P.n) wv[e] &= 0xFFFFu;
                        }
                        am8 = max_abs_bf16x2(max_abs_bf16x2(am8, wv[0]), max_abs_bf16x2(wv[1], max_abs_bf16x2(wv[2], wv[3])));
                        float f[8];
#pragma unroll
                        for (int e = 0; e < 4; ++e) {
                            f[2 * e] = __uint_as_float(packed[4 * qd + e] << 16);
                            f[2 * e + 1] = __uint_as_float(packed[4 * qd + e] & 0xFFFF0000u);
                        }
#pragma unroll
                        for (int e = 0; e < 8; e += 2) mul2_rn(f[e], f[e + 1], m8);
                        if (P.out8_fmt == 0) {
                            q8[2 * qd] = cvt_fp8x4<0>(f[0], f[1], f[2], f[3]);
                            q8[2 * qd + 1] = cvt_fp8x4<0>(f[4], f[5], f[6], f[7]);
                        } else {
                            q8[2 * qd] = cvt_fp8x4<1>(f[0], f[1], f[2], f[3]);
                            q8[2 * qd + 1] = cvt_fp8x4<1>(f[4], f[5], f[6], f[7]);
                        }
                    }
                    uint8_t* orow8 = P.out8 + static_cast<int64_t>(b) * P.stride_o + row * P.ldo;
                    if (P.out8_vec && colg + kOutBox <= P.n) {
                        uint4* dst = reinterpret_cast<uint4*>(orow8 + colg);
#pragma unroll
                        for (int v = 0; v < 4; ++v) dst[v] = make_uint4(q8[4 * v], q8[4 * v + 1], q8[4 * v + 2], q8[4 * v + 3]);
                    } else {
                        for (int e = 0; e < kOutBox && colg + e < P.n; ++e)
                            orow8[colg + e] = static_cast<uint8_t>(q8[e >> 2] >> (8 * (e & 3)));
                    }
                }
            }
            if (kOut8 && P.out8 != nullptr && P.out8_amax != nullptr) {
                // this warp's share of the tile's amax: one atomic per warp and tile
                float v = fmaxf(fabsf(__uint_as_float(am8 << 16)), fabsf(__uint_as_float(am8 & 0xFFFF0000u)));
                v = warp_max(v);
                if (lane == 0) atomicMax(reinterpret_cast<unsigned*>(P.out8_amax), __float_as_uint(v));
                am8 = 0u;
            }
            tc_fence_before_sync();
            if constexpr (kPair) {
                if (leader)
                    mbar_arrive(acc_empty + acc);
                else
                    mbar_arrive_cluster(acc_empty_leader0 + static_cast<uint32_t>(acc * sizeof(uint64_t)));
            } else {
                mbar_arrive(acc_empty + acc);
            }
            if (contrib) {
                // every epilogue thread has issued its partial stores; publish them (release)
                named_barrier(1, C::kEpiThreads);
                if (ew == 0 && lane == 0) {
                    __threadfence();
                    counter_add_release(g.counters + 2 * w.tile + rank, 1u);
                }
            }
            if (++acc == C::kAccBufs) {
                acc = 0;
                acc_phase ^= 1u;
            }
        }
        if (lane == 0) bulk_wait_group_all();
        __syncwarp();
    }

    tc_fence_before_sync();
    __syncthreads();
    if constexpr (kPair) cluster_sync();  // neither CTA releases TMEM or exits while the peer still uses it
    tc_fence_after_sync();
    if (warp == 1) {
        if constexpr (kPair)
            tmem_dealloc_pair(tmem_base, C::kTmemCols);
        else
            tmem_dealloc(tmem_base, C::kTmemCols);
    }
}

// The deferred ring folds, when no GEMM kernel runs to do them.
__global__ void ring_fold_kernel(const __grid_constant__ GemmArgs g) {
    pdl_trigger();
    pdl_wait();
    if (threadIdx.x == 0)
        for (int f = 0; f < g.nfolds; ++f)
            ring_fold_deferred(g.folds[f].state, g.folds[f].hist_len, g.folds[f].hist_idx, g.folds[f].fp8_max,
                               g.folds[f].pow2_margin);
}

// k == 0: the product is empty; out = bias (or 0), rounded to bf16.
__global__ void bias_fill_kernel(uint16_t* out, int64_t m, int64_t n, int64_t ldo, int64_t stride_o, int64_t batch,
                                 const void* bias, int bias_kind, const float* bias_scale) {
    pdl_trigger();
    pdl_wait();
    const int64_t total = batch * m * n;
    const float bsc = bias_kind >= 2 ? __ldg(bias_scale) : 0.0f;
    for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < total;
         i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
        const int64_t j = i % n;
        const int64_t r = (i / n) % m;
        const int64_t b = i / (n * m);
        float v = 0.0f;
        if (bias_kind == 1)
            v = bf16_bits_to_float(static_cast<const uint16_t*>(bias)[j]);
        else if (bias_kind == 2)
            v = __fmul_rn(fp8_to_float<0>(static_cast<const uint8_t*>(bias)[j]), bsc);
        else if (bias_kind == 3)
            v = __fmul_rn(fp8_to_float<1>(static_cast<const uint8_t*>(bias)[j]), bsc);
        out[b * stride_o + r * ldo + j] = __bfloat16_as_ushort(__float2bfloat16_rn(v));
    }
}

// 3-D tensor map: dims {inner, outer, batch} elements, row stride `ld` bytes, batch stride
// `bstride` bytes, box {box_inner, box_outer, 1}, 128-byte swizzle, zero fill out of bounds.
int make_map(CUtensorMap* map, CUtensorMapDataType dtype, const void* base, int64_t inner, int64_t outer,
             int64_t batch, int64_t ld, int64_t bstride, int box_inner, int box_outer) {
    return encode_tensor_map(map, dtype, base, inner, outer, batch, ld, bstride, box_inner, box_outer,
                             CU_TENSOR_MAP_SWIZZLE_128B);
}

// Split-K planning: k_splits in 1..kMaxSplits per problem.  The automatic choice simulates
// the static schedule as a two-stage pipeline per CTA (or pair): the MMAs of unit i overlap
// the epilogue of unit i - 1, and an owner's epilogue also waits for its contributors'
// partials.  Costs are B200 measurements of this kernel: kMmaUsPerKb per 256 x 256 x 128
// k-block, and the epilogue of a plain tile, of a contributor (fp32 partial out) and of an
// owner (partials in).  A range keeps at least 2 k-blocks, the contributors must fit the
// partial workspace, and ties go to fewer splits.
constexpr int kMaxSplits = 4;
constexpr double kSetupUs = 1.5, kMmaUsPerKb = 0.42, kEpiUs = 2.5, kEpiContribUs = 4.6, kEpiOwnerUs = 3.8,
                 kEpiOwnerExtraUs = 0.8;

int range_len(const GemmProblem& P, int splits, int s) {
    return ((s + 1) * P.k_blocks) / splits - (s * P.k_blocks) / splits;
}

// 0 = automatic split choice, 1 = never split (default), 2..kMaxSplits = that many ranges per
// tile wherever the workspace and K allow (set by fp8_set_gemm_split_k).
std::atomic<int> g_split_mode{1};

// Makespan of a launch without split-K, in k-block times: the units dealt boustrophedon-wise to
// `units` pairs, a whole tile costing its k-blocks and a half tile 0.87 of them (a 256 x 128 MMA
// costs that much of a 256 x 256 one on B200), plus the last unit's epilogue (about 5.4 k-blocks
// for a whole tile, half that for a half).  Units from `half_begin` on are halves.
double plain_makespan(const GemmArgs& g, int units, int num_units, int half_begin) {
    double worst = 0.0;
    for (int c = 0; c < units; ++c) {
        double t = 0.0, last_epi = 0.0;
        for (int r = 0;; ++r) {
            const int u = r * units + ((r & 1) ? units - 1 - c : c);
            if (u >= num_units) break;
            const bool half = u >= half_begin;
            const int tile = half ? half_begin + ((u - half_begin) >> 1) : u;
            const int pi = (g.nprob > 1 && tile >= g.p[1].tile_begin) ? 1 : 0;
            t += (half ? 0.87 : 1.0) * g.p[pi].k_blocks;
            last_epi = half ? 2.7 : 5.4;
        }
        worst = std::max(worst, t + last_epi);
    }
    return worst;
}

// Tuning override: FP8DSA_GEMM_HALF_TILES=0 keeps every tile of the last round whole (read
// once; unset = half tiles where they shorten the launch).
bool half_tiles_enabled() {
    static const bool v = [] {
        const char* e = std::getenv("FP8DSA_GEMM_HALF_TILES");
        return e == nullptr || std::string(e) != "0";
    }();
    return v;
}

// Modelled makespan (us) of the unit schedule with `sp` ranges per problem on `units` CTAs.
double simulate_plan(const GemmArgs& g, const int* sp, int units, std::vector<double>& mma_end,
                     std::vector<double>& epi_end, std::vector<double>& contrib_end) {
    mma_end.assign(static_cast<size_t>(units), kSetupUs);
    epi_end.assign(static_cast<size_t>(units), kSetupUs);
    int64_t u = 0;
    int64_t ncontrib = 0;
    for (int i = 0; i < g.nprob; ++i) ncontrib += static_cast<int64_t>(sp[i] - 1) * g.p[i].tiles;
    contrib_end.assign(static_cast<size_t>(std::max<int64_t>(ncontrib, 1)), 0.0);
    auto run = [&](double mma, double epi, double ready) {
        const size_t c = static_cast<size_t>(u % units);
        mma_end[c] += mma;
        const double start = std::max(std::max(mma_end[c], epi_end[c]), ready);
        epi_end[c] = start + epi;
        ++u;
        return epi_end[c];
    };
    int64_t cb = 0;
    for (int i = 0; i < g.nprob; ++i)
        for (int sj = 1; sj < sp[i]; ++sj)
            for (int t = 0; t < g.p[i].tiles; ++t)
                contrib_end[static_cast<size_t>(cb++)] = run(range_len(g.p[i], sp[i], sj) * kMmaUsPerKb, kEpiContribUs, 0.0);
    cb = 0;
    for (int i = 0; i < g.nprob; ++i) {
        const int64_t base = cb;
        for (int t = 0; t < g.p[i].tiles; ++t) {
            double ready = 0.0;
            for (int sj = 1; sj < sp[i]; ++sj)
                ready = std::max(ready, contrib_end[static_cast<size_t>(base + static_cast<int64_t>(sj - 1) * g.p[i].tiles + t)]);
            const double epi = sp[i] > 1 ? kEpiOwnerUs + kEpiOwnerExtraUs * (sp[i] - 2) : kEpiUs;
            run(range_len(g.p[i], sp[i], 0) * kMmaUsPerKb, epi, ready);
        }
        cb += static_cast<int64_t>(sp[i] - 1) * g.p[i].tiles;
    }
    return *std::max_element(epi_end.begin(), epi_end.end());
}

void plan_units(GemmArgs& g, int units, int64_t max_contrib, int64_t counter_words) {
    int best[kMaxProblems] = {1, 1};
    const int mode = g_split_mode.load();
    const bool room = max_contrib > 0 && counter_words >= 2 * static_cast<int64_t>(g.num_tiles) && units > 0;
    if (room && mode >= 2) {
        int64_t contrib = 0;
        for (int i = 0; i < g.nprob; ++i) {
            const int64_t extra = static_cast<int64_t>(mode - 1) * g.p[i].tiles;
            if (g.p[i].k_blocks >= 2 * mode && contrib + extra <= max_contrib) {
                best[i] = mode;
                contrib += extra;
            }
        }
    } else if (room && mode == 0) {
        double best_cost = 1e300;
        int best_sum = 1 << 30;
        std::vector<double> mma_end, epi_end, contrib_end;
        const int lim1 = g.nprob > 1 ? kMaxSplits : 1;
        for (int s0 = 1; s0 <= kMaxSplits; ++s0) {
            for (int s1 = 1; s1 <= lim1; ++s1) {
                const int sp[kMaxProblems] = {s0, s1};
                int64_t contrib = 0;
                bool ok = true;
                for (int i = 0; i < g.nprob; ++i) {
                    if (sp[i] > 1 && g.p[i].k_blocks < 2 * sp[i]) ok = false;
                    contrib += static_cast<int64_t>(sp[i] - 1) * g.p[i].tiles;
                }
                if (!ok || contrib > max_contrib) continue;
                const double cost = simulate_plan(g, sp, units, mma_end, epi_end, contrib_end);
                const int sum = s0 + s1;
                if (cost < best_cost - 1e-9 || (cost < best_cost + 1e-9 && sum < best_sum)) {
                    best_cost = cost;
                    best_sum = sum;
                    best[0] = s0;
                    best[1] = s1;
                }
            }
        }
    }
    int64_t cb = 0;
    for (int i = 0; i < g.nprob; ++i) {
        g.p[i].k_splits = best[i];
        g.p[i].contrib_begin = static_cast<int>(cb);
        cb += static_cast<int64_t>(best[i] - 1) * g.p[i].tiles;
    }
    int64_t ob = 0;
    for (int i = 0; i < g.nprob; ++i) {
        g.p[i].owner_begin = static_cast<int>(ob);
        ob += g.p[i].tiles;
    }
    g.contrib_units = static_cast<int>(cb);
    g.num_units = static_cast<int>(cb + ob);
    g.splitk = cb > 0 ? 1 : 0;
}

// One-time set-up of a kernel instance: its shared-memory limit and (pairs) how many
// 2-CTA clusters fit on the device at once.
template <int BN, bool kPair, bool kSplit, bool kOut8>
cudaError_t kernel_setup(int* max_units_out) {
    using C = Cfg<BN, kPair>;
    static std::once_flag once[kMaxDevices];
    static cudaError_t attr_errs[kMaxDevices];
    static int max_units_dev[kMaxDevices];
    const int dev = current_device();
    cudaError_t& attr_err = attr_errs[dev];
    int& max_units = max_units_dev[dev];
    std::call_once(once[dev], [&attr_err, &max_units] {
        attr_err = cudaFuncSetAttribute(fp8_gemm_kernel<BN, kPair, kSplit, kOut8>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                        C::kSmem);
        if (attr_err != cudaSuccess) return;
        if (kPair) {
            // how many 2-CTA clusters of this kernel fit on the device at once
            cudaLaunchConfig_t cfg = {};
            cudaLaunchAttribute at[1];
            at[0].id = cudaLaunchAttributeClusterDimension;
            at[0].val.clusterDim.x = 2;
            at[0].val.clusterDim.y = 1;
            at[0].val.clusterDim.z = 1;
            cfg.gridDim = dim3(static_cast<unsigned>(2 * (sm_count() / 2)), 1, 1);
            cfg.blockDim = dim3(C::kThreads, 1, 1);
            cfg.dynamicSmemBytes = C::kSmem;
            cfg.attrs = at;
            cfg.numAttrs = 1;
            int n = 0;
            if (cudaOccupancyMaxActiveClusters(&n, fp8_gemm_kernel<BN, kPair, kSplit, kOut8>, &cfg) == cudaSuccess && n > 0)
                max_units = n;
            cudaGetLastError();
        }
    });
    *max_units_out = max_units;
    return attr_err;
}

template <int BN, bool kPair>
int launch_cfg(const CUtensorMap (&maps)[8], GemmArgs& g, const int64_t* batch, const SplitWorkspace* split,
               cudaStream_t stream) {
    using C = Cfg<BN, kPair>;
    int max_units = 0;
    const cudaError_t attr_err = kernel_setup<BN, kPair, false, false>(&max_units);
    if (attr_err != cudaSuccess)
        return fail(FP8DSA_ERR_CUDA, std::string("cudaFuncSetAttribute: ") + cudaGetErrorString(attr_err));
    int64_t tiles = 0;
    for (int i = 0; i < g.nprob; ++i) {
        GemmProblem& P = g.p[i];
        P.tiles_m = (P.m + C::kTileM - 1) / C::kTileM;
        P.tiles_n = (P.n + BN - 1) / BN;
        P.idesc_half = P.idesc | (static_cast<uint32_t>(128 >> 3) << 17) | (static_cast<uint32_t>(C::kTileM >> 4) << 24);
        P.idesc |= (static_cast<uint32_t>(C::kMmaN >> 3) << 17) | (static_cast<uint32_t>(C::kTileM >> 4) << 24);
        P.tile_begin = static_cast<int>(tiles);
        const int64_t pt = static_cast<int64_t>(P.tiles_m) * P.tiles_n * batch[i];
        tiles += pt;
        if (tiles > (int64_t(1) << 28)) return fail(FP8DSA_ERR_UNSUPPORTED, "too many output tiles");
        P.tiles = static_cast<int>(pt);
    }
    g.num_tiles = static_cast<int>(tiles);
    const int units = kPair ? (max_units > 0 ? max_units : sm_count() / 2) : sm_count();
    constexpr int64_t kUnitPartialBytes = int64_t(kPair ? 2 : 1) * kBM * BN * 4;
    if (split != nullptr && split->partial != nullptr && split->counters != nullptr) {
        g.partial = split->partial;
        g.counters = split->counters;
        plan_units(g, units, static_cast<int64_t>(split->partial_bytes) / kUnitPartialBytes, split->counter_words);
    } else {
        plan_units(g, units, 0, 0);
    }
    bool out8 = false;
    for (int i = 0; i < g.nprob; ++i) out8 = out8 || g.p[i].out8 != nullptr;
    if (out8 && g.splitk) {  // the fp8-output instance has no split-K: one range per tile
        g.partial = nullptr;
        g.counters = nullptr;
        plan_units(g, units, 0, 0);
    }
    auto kernel = fp8_gemm_kernel<BN, kPair, false, false>;
    if (out8) {
        int o8_units = 0;
        const cudaError_t oe = kernel_setup<BN, kPair, false, true>(&o8_units);
        if (oe != cudaSuccess) return fail(FP8DSA_ERR_CUDA, std::string("cudaFuncSetAttribute: ") + cudaGetErrorString(oe));
        if (kPair && o8_units > 0 && o8_units < units)
            return fail(FP8DSA_ERR_CUDA, "fp8-output GEMM instance fits fewer clusters than the plan");
        kernel = fp8_gemm_kernel<BN, kPair, false, true>;
    } else if (g.splitk) {
        int split_units = 0;
        const cudaError_t se = kernel_setup<BN, kPair, true, false>(&split_units);
        if (se != cudaSuccess) return fail(FP8DSA_ERR_CUDA, std::string("cudaFuncSetAttribute: ") + cudaGetErrorString(se));
        // both instances must have every cluster of the plan resident at once
        if (kPair && split_units > 0 && split_units < units) {
            g.partial = nullptr;
            g.counters = nullptr;
            plan_units(g, units, 0, 0);
        } else {
            kernel = fp8_gemm_kernel<BN, kPair, true, false>;
        }
    }
    // A last round that would keep at most half of the pairs busy runs as twice as many 256 x 128
    // half tiles (pairs, K-major B, no split-K): the last epilogue, the launch's tail, is
    // half as long, and the round's MMAs are spread over more pairs.
    g.half_begin = g.num_tiles;
    if (kPair && BN == 256 && !g.splitk) {
        bool k_major_b = true;
        for (int i = 0; i < g.nprob; ++i) k_major_b = k_major_b && !g.p[i].b_mn;
        const int64_t T = g.num_tiles, U = units;
        const int64_t R = (T + U - 1) / U, L = T - (R - 1) * U;
        // only where the dealt schedule gets shorter (halves that land on pairs already holding
        // the longest units would lengthen it), and only for launches of at most 8 rounds, so
        // the model stays cheap and the tail it trims is still a visible share of the launch
        if (k_major_b && half_tiles_enabled() && R >= 2 && R <= 8 && 2 * L <= U &&
            plain_makespan(g, units, static_cast<int>(T + L), static_cast<int>(T - L)) <
                0.98 * plain_makespan(g, units, static_cast<int>(T), static_cast<int>(T))) {
            g.half_begin = static_cast<int>(T - L);
            g.num_units = static_cast<int>(T + L);
        }
    }
    const int grid_units = static_cast<int>(std::max<int64_t>(1, std::min<int64_t>(g.num_units, units)));
    cudaError_t e = launch_ex(kernel, dim3(static_cast<unsigned>(grid_units * (kPair ? 2 : 1))), dim3(C::kThreads),
                              C::kSmem, stream, kPair ? 2 : 1, maps[0], maps[1], maps[2], maps[3], maps[4], maps[5],
                              maps[6], maps[7], g);
    if (e != cudaSuccess) return fail(FP8DSA_ERR_CUDA, std::string("fp8 gemm launch: ") + cudaGetErrorString(e));
    return FP8DSA_OK;
}

// Tile shape for a launch: 256 x 256 tiles on CTA pairs (each SM loads half of the B tile)
// whenever every problem has M > 128 and N > 128 and there are enough of them; 128 x 256 on
// single CTAs when some M is at most 128; 128 x 128 when some N is at most 128, or when the
// pair tiles would keep at most half of the CTA pairs busy.  Measured on B200, a 128-wide MMA
// tile costs almost as much time per k-block as a 256-wide one (4096^3: 1.57 vs 2.40 PFLOP/s),
// so narrower tiles pay only where the wide ones leave SMs idle.
struct TileChoice {
    int bn;
    bool pair;
};

// Tuning override: FP8DSA_GEMM_TILE = "256p", "128p", "256", "128" or "64" forces that tile shape
// wherever the problem admits it (read once; unset = the default choice below).
int tile_override() {
    static const int v = [] {
        const char* e = std::getenv("FP8DSA_GEMM_TILE");
        if (e == nullptr) return 0;
        const std::string t(e);
        if (t == "256p") return 1;
        if (t == "128p") return 2;
        if (t == "256") return 3;
        if (t == "128") return 4;
        if (t == "64") return 5;
        if (t == "512p") return 6;
        return 0;
    }();
    return v;
}

// Single-CTA tile width for launches the pair tiles do not suit (some M at most 128, or some
// N at most 128): the BN in {64, 128, 256} with the fewest rounds of tiles times the bytes a
// CTA loads per k-block (A's 128 rows plus BN rows of B), the wider one on ties -- so a short,
// wide problem (M = 64, N = 8192) spreads B over most SMs in 64-column tiles instead of
// leaving them idle.  64-wide tiles need a K-major B; 256-wide ones an N above 128.
int single_cta_width(const GemmDesc* d, int n, bool b_mn) {
    int best = 128;
    int64_t best_cost = -1;
    for (int bn : {256, 128, 64}) {
        if (bn == 64 && b_mn) continue;
        bool fits = true;
        int64_t tiles = 0;
        for (int i = 0; i < n; ++i) {
            if (bn == 256 && d[i].n <= 128) fits = false;
            tiles += ((d[i].m + kBM - 1) / kBM) * ((d[i].n + bn - 1) / bn) * d[i].batch;
        }
        if (!fits) continue;
        const int64_t rounds = (tiles + sm_count() - 1) / sm_count();
        const int64_t cost = rounds * static_cast<int64_t>(kBM * kBK + bn * kBK);
        if (best_cost < 0 || cost < best_cost) {
            best_cost = cost;
            best = bn;
        }
    }
    return best;
}

// Modelled time (us) of a launch on CTA pairs with `width`-wide tiles (256 or 512): the tiles,
// longest K first, each go to the least-loaded pair.  A tile costs its k-blocks times the time
// a k-block takes at that width -- the mainloop is bound by how fast each SM's TMA engine fills
// shared memory, 32 KB per k-block and SM at 256 wide, 48 KB at 512 -- plus, at 512 wide (one
// accumulator, so the epilogue cannot overlap the next tile's MMAs), its epilogue; at 256 wide
// only each pair's last epilogue shows.  Constants measured on B200.
double pair_width_cost(const GemmDesc* d, int n, int width, int pairs) {
    const double kb_us = width == 512 ? 0.60 : 0.40;
    const double epi_us = width == 512 ? 2.6 : 1.3;
    std::vector<std::pair<int64_t, int64_t>> probs;  // (k-blocks, tiles)
    for (int i = 0; i < n; ++i)
        probs.push_back({(d[i].k + kBK - 1) / kBK, ((d[i].m + 255) / 256) * ((d[i].n + width - 1) / width) * d[i].batch});
    std::sort(probs.begin(), probs.end(), [](const auto& x, const auto& y) { return x.first > y.first; });
    std::vector<double> load(static_cast<size_t>(pairs), 0.0);
    for (const auto& pr : probs) {
        const double cost = static_cast<double>(pr.first) * kb_us + (width == 512 ? epi_us : 0.0);
        // whole rounds go to every pair at once; the remainder to the least-loaded pairs
        const int64_t rounds = pr.second / pairs;
        if (rounds > 0)
            for (double& l : load) l += static_cast<double>(rounds) * cost;
        for (int64_t t = rounds * pairs; t < pr.second; ++t) {
            auto it = std::min_element(load.begin(), load.end());
            *it += cost;
        }
    }
    return *std::max_element(load.begin(), load.end()) + (width == 512 ? 0.0 : epi_us);
}

TileChoice choose_tiles(const GemmDesc* d, int n) {
    bool narrow = false, short_m = false, b_mn = false;
    for (int i = 0; i < n; ++i) {
        narrow = narrow || d[i].n <= 128;
        short_m = short_m || d[i].m <= kBM;
        b_mn = b_mn || d[i].b_mn;
    }
    if (narrow || short_m) return {single_cta_width(d, n, b_mn), false};
    switch (tile_override()) {
        case 1: return {256, true};
        case 2: if (!b_mn) return {128, true}; break;
        case 3: return {256, false};
        case 4: return {128, false};
        case 5: if (!b_mn) return {64, false}; break;
        case 6: if (!b_mn) return {512, true}; break;
        default: break;
    }
    // Few output tiles: when the 256 x 256 pair tiles would keep at most half of the CTA pairs
    // busy, 128 x 128 tiles on single CTAs put more SMs to work (measured on B200: 5-15% faster
    // on such launches, 6-34% slower on the larger ones).
    int64_t pair_tiles = 0;
    for (int i = 0; i < n; ++i) pair_tiles += ((d[i].m + 255) / 256) * ((d[i].n + 255) / 256) * d[i].batch;
    if (4 * pair_tiles <= sm_count()) return {128, false};
    // 512-wide pair tiles where the model says the launch gets shorter (K-major B only)
    if (!b_mn) {
        const int pairs = std::max(1, sm_count() / 2);
        if (pair_width_cost(d, n, 512, pairs) < 0.88 * pair_width_cost(d, n, 256, pairs)) return {512, true};
    }
    return {256, true};
}

}  // namespace

size_t splitk_partial_bytes(const int64_t* m, const int64_t* n, int nprob) {
    // (kMaxSplits - 1) contributors per tile; a tile's partial covers its padded output area
    size_t total = 0;
    for (int i = 0; i < nprob; ++i) {
        if (m[i] <= 0 || n[i] <= 0) continue;
        total += static_cast<size_t>(kMaxSplits - 1) * static_cast<size_t>(align_up(m[i], 256)) *
                 static_cast<size_t>(align_up(n[i], 256)) * 4u;
    }
    return total;
}

int64_t splitk_counter_words(const int64_t* m, const int64_t* n, int nprob) {
    // two counters per tile of the finest tiling (128 x 128)
    int64_t total = 0;
    for (int i = 0; i < nprob; ++i)
        if (m[i] > 0 && n[i] > 0) total += 2 * ((m[i] + kBM - 1) / kBM) * ((n[i] + 127) / 128);
    return total;
}

// Launch the one-thread fold kernel for `g.nfolds` rings.
int launch_fold_only(const GemmArgs& g, cudaStream_t stream) {
    launch_begin(kKindOther, stream);
    launch_ex(ring_fold_kernel, dim3(1), dim3(32), 0, stream, 1, g);
    launch_end(kKindOther, stream, 0.0);
    return check_launch("ring fold kernel");
}

int gemm_launch_group(const GemmDesc* descs, int ndesc, const float* colsum_partial, int64_t colsum_tiles,
                      int64_t colsum_cols, void* colsum_out, const SplitWorkspace* split, const fp8_ring_t* folds,
                      int nfolds, cudaStream_t stream) {
    if (nfolds < 0 || nfolds > kMaxFolds) return fail(FP8DSA_ERR_INVALID_ARG, "at most 3 deferred ring folds");
    GemmArgs fold_args{};
    fold_args.nfolds = nfolds;
    for (int i = 0; i < nfolds; ++i)
        fold_args.folds[i] = RingFold{folds[i].state, folds[i].hist_len, folds[i].hist_idx, folds[i].fp8_max,
                                      folds[i].pow2_margin};
    // problems with an empty product write their bias (or zeros) without the tensor cores
    GemmDesc work[kMaxProblems];
    int nwork = 0;
    double flops = 0.0;
    for (int i = 0; i < ndesc; ++i) {
        const GemmDesc& d = descs[i];
        if (d.m == 0 || d.n == 0 || d.batch == 0) continue;
        if (d.k == 0) {
            const int64_t total = d.batch * d.m * d.n;
            const int blocks = static_cast<int>(std::min<int64_t>((total + 255) / 256, sm_count() * 8));
            launch_begin(kKindOther, stream);
            launch_ex(bias_fill_kernel, dim3(blocks), dim3(256), 0, stream, 1, static_cast<uint16_t*>(d.out), d.m, d.n,
                      d.ldo, d.stride_o, d.batch, d.bias, d.bias_kind, d.bias_scale);
            launch_end(kKindOther, stream, static_cast<double>(total) * 2);
            int rc = check_launch("bias fill kernel");
            if (rc) return rc;
            continue;
        }
        work[nwork++] = d;
        flops += 2.0 * static_cast<double>(d.m) * d.n * d.k * d.batch;
    }
    // the problem with the longer K (the longer tiles) first: with the alternating rounds of
    // the tile schedule this spreads long and short tiles evenly over the CTAs
    if (nwork == 2 && work[1].k > work[0].k) std::swap(work[0], work[1]);
    const bool colsum = colsum_tiles > 0 && colsum_cols > 0;
    if (nwork == 0) {
        if (colsum) {
            const int rc = launch_colsum_finalize(colsum_partial, colsum_tiles, colsum_cols, colsum_out, stream);
            if (rc) return rc;
        } else if (colsum_cols > 0 && colsum_out != nullptr) {  // no rows: the bias gradient is zero
            cudaError_t e = cudaMemsetAsync(colsum_out, 0, sizeof(uint16_t) * colsum_cols, stream);
            if (e != cudaSuccess) return fail(FP8DSA_ERR_CUDA, std::string("memset grad_b: ") + cudaGetErrorString(e));
        }
        return nfolds > 0 ? launch_fold_only(fold_args, stream) : FP8DSA_OK;
    }
    if (colsum_cols > 0x7FFFFFFF || colsum_tiles > 0x7FFFFFFF) return fail(FP8DSA_ERR_UNSUPPORTED, "bias gradient too wide");
    const TileChoice tc = choose_tiles(work, nwork);
    // rows of B per TMA box: a CTA's share of one MMA's columns (two boxes per stage at 512 wide)
    const int b_rows = tc.pair ? std::min(tc.bn / 2, 128) : tc.bn;

    CUtensorMap maps[8];  // per problem A, B, out; then per problem B in 64-row boxes (half tiles)
    GemmArgs g = fold_args;
    int64_t batch[kMaxProblems] = {1, 1};
    const CUtensorMapDataType u8 = CU_TENSOR_MAP_DATA_TYPE_UINT8;
    for (int i = 0; i < nwork; ++i) {
        const GemmDesc& d = work[i];
        const bool a_bat = d.stride_a != 0 && d.batch > 1;
        const bool b_bat = d.stride_b != 0 && d.batch > 1;
        CUtensorMap& ma = maps[3 * i];
        CUtensorMap& mb = maps[3 * i + 1];
        CUtensorMap& mo = maps[3 * i + 2];
        int rc;
        if (!d.a_mn)
            rc = make_map(&ma, u8, d.a, d.k, d.m, a_bat ? d.batch : 1, d.lda, a_bat ? d.stride_a : d.lda * d.m, 128, kBM);
        else
            rc = make_map(&ma, u8, d.a, d.m, d.k, a_bat ? d.batch : 1, d.lda, a_bat ? d.stride_a : d.lda * d.k, 128, kBK);
        if (rc) return rc;
        if (!d.b_mn)
            rc = make_map(&mb, u8, d.b, d.k, d.n, b_bat ? d.batch : 1, d.ldb, b_bat ? d.stride_b : d.ldb * d.n, 128,
                          b_rows);
        else
            rc = make_map(&mb, u8, d.b, d.n, d.k, b_bat ? d.batch : 1, d.ldb, b_bat ? d.stride_b : d.ldb * d.k, 128, kBK);
        if (rc) return rc;
        if (!d.b_mn && tc.pair && tc.bn == 256) {
            rc = make_map(&maps[6 + i], u8, d.b, d.k, d.n, b_bat ? d.batch : 1, d.ldb,
                          b_bat ? d.stride_b : d.ldb * d.n, 128, 64);
            if (rc) return rc;
        } else {
            maps[6 + i] = mb;  // unused: no half tiles
        }
        // TMA stores need 16-byte aligned rows and batches of the output
        const bool tma_out = d.out != nullptr && aligned16(d.out) && d.ldo % 8 == 0 &&
                             (d.batch == 1 || d.stride_o % 8 == 0);
        if (tma_out) {
            rc = make_map(&mo, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, d.out, d.n, d.m, d.batch, d.ldo * 2,
                          d.batch > 1 ? d.stride_o * 2 : d.ldo * 2 * d.m, kOutBox, 32);
            if (rc) return rc;
        } else {
            mo = ma;  // unused placeholder
        }
        GemmProblem& P = g.p[i];
        P.m = static_cast<int>(d.m);
        P.n = static_cast<int>(d.n);
        P.k_blocks = static_cast<int>((d.k + kBK - 1) / kBK);
        P.a_batched = a_bat;
        P.b_batched = b_bat;
        P.a_mn = d.a_mn;
        P.b_mn = d.b_mn;
        P.idesc = (1u << 4) | (static_cast<uint32_t>(d.fmt_a) << 7) | (static_cast<uint32_t>(d.fmt_b) << 10) |
                  (static_cast<uint32_t>(d.a_mn) << 15) | (static_cast<uint32_t>(d.b_mn) << 16);
        P.out = static_cast<uint16_t*>(d.out);
        P.ldo = d.ldo;
        P.stride_o = d.stride_o;
        P.vec_out = aligned16(d.out) && d.ldo % 8 == 0 && d.stride_o % 8 == 0;
        P.tma_out = tma_out;
        P.bias = d.bias;
        P.bias_kind = d.bias_kind;
        P.bias_scale = d.bias_scale;
        P.scale_a = d.scale_a;
        P.scale_b = d.scale_b;
        P.out8 = d.out8;
        P.out8_fmt = d.out8_fmt;
        P.out8_vec = d.out8 != nullptr && aligned16(d.out8) && d.ldo % 16 == 0 && (d.batch == 1 || d.stride_o % 16 == 0);
        P.out8_step = d.out8_step;
        P.out8_amax = d.out8_amax;
        P.out8_step_used = d.out8_step_used;
        batch[i] = d.batch;
    }
    for (int i = nwork; i < kMaxProblems; ++i) maps[3 * i] = maps[3 * i + 1] = maps[3 * i + 2] = maps[6 + i] = maps[0];
    g.nprob = nwork;
    if (colsum) {
        g.colsum.partial = colsum_partial;
        g.colsum.tiles = static_cast<int>(colsum_tiles);
        g.colsum.cols = static_cast<int>(colsum_cols);
        g.colsum.out = static_cast<uint16_t*>(colsum_out);
    }
    int rc = wait_ctl(&g.wait);
    if (rc) return rc;

    launch_begin(kKindGemm, stream);
    if (tc.pair && tc.bn == 512)
        rc = launch_cfg<512, true>(maps, g, batch, split, stream);
    else if (tc.pair)
        rc = tc.bn == 256 ? launch_cfg<256, true>(maps, g, batch, split, stream)
                          : launch_cfg<128, true>(maps, g, batch, split, stream);
    else if (tc.bn == 256)
        rc = launch_cfg<256, false>(maps, g, batch, split, stream);
    else if (tc.bn == 128)
        rc = launch_cfg<128, false>(maps, g, batch, split, stream);
    else
        rc = launch_cfg<64, false>(maps, g, batch, split, stream);
    if (rc) return rc;
    launch_end(tc.pair ? kKindGemmPair : kKindGemmSingle, stream, flops);
    return check_launch("fp8 gemm kernel");
}

int gemm_set_split_mode(int mode) {
    if (mode < 0 || mode > kMaxSplits) return fail(FP8DSA_ERR_INVALID_ARG, "split_k must be 0 (automatic) .. 4");
    g_split_mode.store(mode);
    return FP8DSA_OK;
}

int gemm_launch(const uint8_t* a, const uint8_t* b, int fmt_a, int fmt_b, int a_mn, int b_mn, int64_t m,
                int64_t n, int64_t k, int64_t lda, int64_t ldb, int64_t ldo, int64_t batch, int64_t stride_a,
                int64_t stride_b, int64_t stride_o, const float* scale_a, const float* scale_b, const void* bias,
                int bias_kind, const float* bias_scale, void* out, cudaStream_t stream) {
    GemmDesc d{a, b, fmt_a, fmt_b, a_mn, b_mn, m, n, k, lda, ldb, ldo, batch, stride_a, stride_b, stride_o,
               scale_a, scale_b, bias, bias_kind, bias_scale, out};
    return gemm_launch_group(&d, 1, nullptr, 0, 0, nullptr, nullptr, nullptr, 0, stream);
}

}  // namespace fp8dsa

using namespace fp8dsa;

namespace {

// fp8_gemm / fp8_gemm_fp8out: argument checks, then one GEMM launch.  out8 == null: bf16 only.
int gemm_entry(const uint8_t* a, const uint8_t* b, fp8_fmt_t fmt_a, fp8_fmt_t fmt_b, fp8_layout_t layout, int64_t m,
               int64_t n, int64_t k, int64_t lda, int64_t ldb, int64_t ldo, int64_t batch, int64_t stride_a,
               int64_t stride_b, int64_t stride_o, const float* scale_a, const float* scale_b, const void* bias,
               const float* bias_scale, void* out, fp8_fmt_t out8_fmt, const float* out8_step, uint8_t* out8,
               float* out8_amax, float* out8_step_used, cudaStream_t stream) {
    if (!valid_fmt(fmt_a) || !valid_fmt(fmt_b)) return fail(FP8DSA_ERR_INVALID_ARG, "fmt must be FP8_E4M3 or FP8_E5M2");
    if (layout < FP8_LAYOUT_NT || layout > FP8_LAYOUT_TT) return fail(FP8DSA_ERR_INVALID_ARG, "bad layout");
    if (m < 0 || n < 0 || k < 0 || batch < 0) return fail(FP8DSA_ERR_INVALID_ARG, "negative size");
    if (m > 0x7FFFFFFF || n > 0x7FFFFFFF || k > 0x7FFFFFFF) return fail(FP8DSA_ERR_UNSUPPORTED, "sizes must be < 2^31");
    if (batch > 0x7FFFFFFF) return fail(FP8DSA_ERR_UNSUPPORTED, "batch must be < 2^31");
    const bool empty_out = m == 0 || n == 0 || batch == 0;  // an output without elements may be NULL
    if ((out == nullptr && out8 == nullptr && !empty_out) || scale_a == nullptr || scale_b == nullptr)
        return fail(FP8DSA_ERR_INVALID_ARG, "an output, scale_a and scale_b are required");
    if (bias == nullptr && bias_scale != nullptr) return fail(FP8DSA_ERR_INVALID_ARG, "bias_scale without bias");
    if (ldo < n) return fail(FP8DSA_ERR_INVALID_ARG, "ldo must be >= n");
    if (batch > 1 && stride_o < ldo * m && stride_o != 0 && m > 1)
        return fail(FP8DSA_ERR_INVALID_ARG, "stride_o overlaps batches");
    if (batch > 1 && stride_o == 0 && m > 0 && n > 0) return fail(FP8DSA_ERR_INVALID_ARG, "stride_o must be non-zero when batch > 1");
    if (out8 != nullptr) {
        if (!valid_fmt(out8_fmt)) return fail(FP8DSA_ERR_INVALID_ARG, "out8_fmt must be FP8_E4M3 or FP8_E5M2");
        if (out8_step == nullptr) return fail(FP8DSA_ERR_INVALID_ARG, "out8 needs out8_step");
        if (k == 0 && m > 0 && n > 0 && batch > 0)
            return fail(FP8DSA_ERR_UNSUPPORTED, "the fp8 output needs k > 0");
    }
    const int a_mn = (layout == FP8_LAYOUT_TN || layout == FP8_LAYOUT_TT) ? 1 : 0;
    const int b_mn = (layout == FP8_LAYOUT_NN || layout == FP8_LAYOUT_TN) ? 1 : 0;
    if (m > 0 && n > 0 && batch > 0 && k > 0) {
        if (a == nullptr || b == nullptr) return fail(FP8DSA_ERR_INVALID_ARG, "a and b are required");
        if (lda < (a_mn ? m : k)) return fail(FP8DSA_ERR_INVALID_ARG, "lda too small for the layout");
        if (ldb < (b_mn ? n : k)) return fail(FP8DSA_ERR_INVALID_ARG, "ldb too small for the layout");
        if (lda % 16 != 0 || ldb % 16 != 0)
            return fail(FP8DSA_ERR_UNSUPPORTED, "lda and ldb must be multiples of 16 (TMA row strides)");
        if (!aligned16(a) || !aligned16(b)) return fail(FP8DSA_ERR_UNSUPPORTED, "a and b must be 16-byte aligned");
        if (stride_a % 16 != 0 || stride_b % 16 != 0)
            return fail(FP8DSA_ERR_UNSUPPORTED, "batch strides must be multiples of 16");
        if (stride_a < 0 || stride_b < 0) return fail(FP8DSA_ERR_INVALID_ARG, "negative batch stride");
    }
    int rc = check_device();
    if (rc) return rc;
    int bias_kind = 0;
    if (bias != nullptr) bias_kind = bias_scale == nullptr ? 1 : (fmt_a == FP8_E4M3 ? 2 : 3);
    GemmDesc d{a, b, fmt_a, fmt_b, a_mn, b_mn, m, n, k, lda, ldb, ldo, batch, stride_a, stride_b, stride_o,
               scale_a, scale_b, bias, bias_kind, bias_scale, out};
    d.out8 = out8;
    d.out8_fmt = out8_fmt;
    d.out8_step = out8_step;
    d.out8_amax = out8_amax;
    d.out8_step_used = out8_step_used;
    return gemm_launch_group(&d, 1, nullptr, 0, 0, nullptr, nullptr, nullptr, 0, stream);
}

}  // namespace

extern "C" int fp8_gemm(const uint8_t* a, const uint8_t* b, fp8_fmt_t fmt_a, fp8_fmt_t fmt_b, fp8_layout_t layout,
                        int64_t m, int64_t n, int64_t k, int64_t lda, int64_t ldb, int64_t ldo, int64_t batch,
                        int64_t stride_a, int64_t stride_b, int64_t stride_o, const float* scale_a,
                        const float* scale_b, const void* bias, const float* bias_scale, void* out,
                        cudaStream_t stream) {
    clear_error();
    if (out == nullptr && m > 0 && n > 0 && batch > 0)
        return fail(FP8DSA_ERR_INVALID_ARG, "out, scale_a and scale_b are required");
    return gemm_entry(a, b, fmt_a, fmt_b, layout, m, n, k, lda, ldb, ldo, batch, stride_a, stride_b, stride_o, scale_a,
                      scale_b, bias, bias_scale, out, FP8_E4M3, nullptr, nullptr, nullptr, nullptr, stream);
}

extern "C" int fp8_gemm_fp8out(const uint8_t* a, const uint8_t* b, fp8_fmt_t fmt_a, fp8_fmt_t fmt_b,
                               fp8_layout_t layout, int64_t m, int64_t n, int64_t k, int64_t lda, int64_t ldb,
                               int64_t ldo, int64_t batch, int64_t stride_a, int64_t stride_b, int64_t stride_o,
                               const float* scale_a, const float* scale_b, const void* bias,
                               const float* bias_scale, void* out, fp8_fmt_t out8_fmt, const float* out8_step,
                               uint8_t* out8, float* out8_amax, float* out8_step_used, cudaStream_t stream) {
    clear_error();
    if (out8 == nullptr && m > 0 && n > 0 && batch > 0) return fail(FP8DSA_ERR_INVALID_ARG, "out8 is required");
    return gemm_entry(a, b, fmt_a, fmt_b, layout, m, n, k, lda, ldb, ldo, batch, stride_a, stride_b, stride_o, scale_a,
                      scale_b, bias, bias_scale, out, out8_fmt, out8_step, out8, out8_amax, out8_step_used, stream);
}
