// FP8 quantize kernels with fused raw-domain amax and the last-block history-ring fold.
//
// Sources (AstrAI compare view 3e57cc8...main): csrc/kernels/fp8/quantize.cuh
// (fp8_quantize_kernel, fp8_quantize_tiled_kernel, publish_amax), astrai/extension/fp8.py
// (_ScaleRing, FP8Recipe.scale_from_history, _dynamic_scale) and the extension commit log
// (amax is the max of the unscaled input; the ring is finalised in the quantize kernel's last
// block with zero extra launches).
//
// B200 design:
//  * Row-major quantize is a flat grid-stride kernel: 16 elements per thread-iteration
//    (two 128-bit loads, one 128-bit store of packed fp8x4 words), two iterations in flight;
//    one wave of 4 resident 256-thread blocks per SM, shared out to the tensors of the launch
//    in proportion to their sizes.
//  * Transposed / dual quantize is tiled 128 x 128.  Large batches run persistent (two CTAs
//    per SM walk all tiles of the batch): each input tile arrives by one TMA bulk-tensor copy
//    into a two-stage shared-memory ring, so the next tile loads while this one is converted.
//    Small batches run one tile per CTA (three per SM), loaded straight into registers.  The
//    fp8 bytes are staged in a 16 KB shared tile whose 16-byte chunks are XOR-swizzled by row
//    group, then a register 4x4 byte transpose (PRMT) and 128-byte coalesced stores of each
//    output row.  The dual mode also writes the row-major bytes straight from registers (the
//    transposed bytes may take a second format: the same products rounded twice), and can
//    emit per-tile fp32 column sums (the bias gradient) from the values it already holds.
//  * Each block reduces amax with warp shuffles, one atomicMax per block and tensor; with a
//    ring, an acq_rel ticket elects the last block, which folds the amax into the window and
//    publishes the next step.  The fold itself never waits; the tiled kernel's only wait (for
//    its input copies) is bounded and reports a status code instead of hanging.
#include <cuda_runtime.h>
#include <cuda_fp16.h>
#include <cuda_bf16.h>

#include <algorithm>
#include <atomic>
#include <cstdlib>
#include <mutex>
#include <string>

#include "internal.h"

namespace fp8dsa {
namespace {

constexpr int kThreads = 256;
constexpr int kTile = 128;
constexpr int64_t kMaxTiles = int64_t(1) << 30;  // tile indices stay far from int overflow

// ----------------------------------------------------------------------------------------
// Input element access
// ----------------------------------------------------------------------------------------
struct Bf16In {
    using E = uint16_t;
    using Raw = uint4;
    static __device__ __forceinline__ float cvt(E v) { return __uint_as_float(uint32_t(v) << 16); }
    // 8 consecutive elements (16 bytes, 16-byte aligned) as raw bits, then unpacked.
    static __device__ __forceinline__ Raw load_raw(const E* p) { return __ldg(reinterpret_cast<const uint4*>(p)); }
    static __device__ __forceinline__ void unpack(const Raw& v, float (&f)[8]) {
        const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            f[2 * i] = __uint_as_float(w[i] << 16);
            f[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
        }
    }
    static __device__ __forceinline__ void load8(const E* p, float (&f)[8]) { unpack(load_raw(p), f); }
    static __device__ __forceinline__ Raw lds_raw(const E* p) { return *reinterpret_cast<const uint4*>(p); }
    // running max of |x| over raw words, two lanes per instruction
    using Acc = uint32_t;
    static __device__ __forceinline__ Acc acc_zero() { return 0u; }
    static __device__ __forceinline__ void acc_max(Acc& acc, const Raw& v) {
        acc = max_abs_bf16x2(max_abs_bf16x2(acc, v.x), max_abs_bf16x2(v.y, max_abs_bf16x2(v.z, v.w)));
    }
    static __device__ __forceinline__ float acc_value(Acc acc) {
        return fmaxf(fabsf(__uint_as_float(acc << 16)), fabsf(__uint_as_float(acc & 0xFFFF0000u)));
    }
};

struct F16In {
    using E = uint16_t;
    using Raw = uint4;
    static __device__ __forceinline__ float cvt(E v) { return __half2float(__ushort_as_half(v)); }
    static __device__ __forceinline__ Raw load_raw(const E* p) { return __ldg(reinterpret_cast<const uint4*>(p)); }
    static __device__ __forceinline__ void unpack(const Raw& v, float (&f)[8]) {
        const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            f[2 * i] = __half2float(__ushort_as_half(static_cast<uint16_t>(w[i] & 0xFFFFu)));
            f[2 * i + 1] = __half2float(__ushort_as_half(static_cast<uint16_t>(w[i] >> 16)));
        }
    }
    static __device__ __forceinline__ void load8(const E* p, float (&f)[8]) { unpack(load_raw(p), f); }
    static __device__ __forceinline__ Raw lds_raw(const E* p) { return *reinterpret_cast<const uint4*>(p); }
    using Acc = uint32_t;
    static __device__ __forceinline__ Acc acc_zero() { return 0u; }
    static __device__ __forceinline__ void acc_max(Acc& acc, const Raw& v) {
        acc = max_abs_f16x2(max_abs_f16x2(acc, v.x), max_abs_f16x2(v.y, max_abs_f16x2(v.z, v.w)));
    }
    static __device__ __forceinline__ float acc_value(Acc acc) {
        return fmaxf(fabsf(__half2float(__ushort_as_half(static_cast<uint16_t>(acc & 0xFFFFu)))),
                     fabsf(__half2float(__ushort_as_half(static_cast<uint16_t>(acc >> 16)))));
    }
};

struct F32Raw {
    float4 a, b;
};

struct F32In {
    using E = float;
    using Raw = F32Raw;
    static __device__ __forceinline__ float cvt(E v) { return v; }
    static __device__ __forceinline__ Raw load_raw(const E* p) {
        return {__ldg(reinterpret_cast<const float4*>(p)), __ldg(reinterpret_cast<const float4*>(p) + 1)};
    }
    static __device__ __forceinline__ void unpack(const Raw& v, float (&f)[8]) {
        f[0] = v.a.x; f[1] = v.a.y; f[2] = v.a.z; f[3] = v.a.w;
        f[4] = v.b.x; f[5] = v.b.y; f[6] = v.b.z; f[7] = v.b.w;
    }
    static __device__ __forceinline__ void load8(const E* p, float (&f)[8]) { unpack(load_raw(p), f); }
    static __device__ __forceinline__ Raw lds_raw(const E* p) {
        return {reinterpret_cast<const float4*>(p)[0], reinterpret_cast<const float4*>(p)[1]};
    }
    using Acc = float;
    static __device__ __forceinline__ Acc acc_zero() { return 0.0f; }
    static __device__ __forceinline__ void acc_max(Acc& acc, const Raw& v) {
        acc = fmaxf(acc, fmaxf(fmaxf(fmaxf(fabsf(v.a.x), fabsf(v.a.y)), fmaxf(fabsf(v.a.z), fabsf(v.a.w))),
                               fmaxf(fmaxf(fabsf(v.b.x), fabsf(v.b.y)), fmaxf(fabsf(v.b.z), fabsf(v.b.w)))));
    }
    static __device__ __forceinline__ float acc_value(Acc acc) { return acc; }
};

// Arguments of the quantize kernels (one POD by value).
struct QArgs {
    const void* x;
    int64_t numel, rows, cols;
    const float* scale;        // step s; every element is multiplied by RN32(1/s)
    uint8_t* out;              // [rows][cols] or null
    uint8_t* out_t;            // [cols][rows] or null
    uint8_t* out2;             // row-major kernel: [rows][cols] in the second format, or null
    float* amax_accum;         // block maxima land here (ring amax slot or amax_out), or null
    float* amax_out;           // ring mode: receives the final amax
    float* ring_state;         // null = no fold
    int hist_len, hist_idx;
    float fp8_max, pow2_margin;
    float* scale_used_out;     // receives the step used, or null
    int defer_fold;            // ring: leave the amax in its slot; the next kernel folds it
    float* colsum;             // [row tiles][cols] per-tile column sums (tiled kernel), or null
    int vec_in, vec_out, vec_out_t;
    int tma;                   // tiled kernel: input tiles arrive by TMA through map[job]
    unsigned nblocks;          // blocks working on this tensor (the ticket count of its fold)
    int tile_begin, tiles_x;   // tiled kernel: first tile of this tensor, column tiles
    int tiles_y;               // tiled kernel: row tiles
    int tile_group;            // tiled kernel: tile rows per group of the traversal order
};

// Up to three tensors quantized by one launch; each keeps its own amax, ticket and fold.
constexpr int kMaxJobs = 3;
struct QBatch {
    CUtensorMap map[kMaxJobs];  // tiled kernel: [rows][cols] input, box 128 x 128, no swizzle
    QArgs job[kMaxJobs];
    int njobs;
    int tiles_total;            // tiled kernel: tiles of all jobs, concatenated
    int row_out_any;            // tiled kernel: some job also writes row-major bytes
    uint32_t* zero;             // side job of the launch's first block: zero[0 .. zero_words)
    int64_t zero_words;
};

// The side job: the first block of the launch clears the words (after pdl_wait, so the
// kernel that last used them has finished).
__device__ __forceinline__ void zero_side_job(const QBatch& b) {
    if (b.zero_words > 0 && blockIdx.x == 0 && blockIdx.y == 0)
        for (int64_t i = threadIdx.x; i < b.zero_words; i += blockDim.x) b.zero[i] = 0u;
}

// Chunks of 16 elements each thread of the row-major kernel has in flight (16-bit inputs).
#ifndef FP8DSA_FLAT_DEPTH
#define FP8DSA_FLAT_DEPTH 3
#endif
constexpr int kFlatDepth = FP8DSA_FLAT_DEPTH;
// 1: the row-major kernel's rounds are software-pipelined (round r + 1 loads while round r
// converts); 0: each round loads, then converts.
#ifndef FP8DSA_FLAT_PIPE
#define FP8DSA_FLAT_PIPE 0
#endif
// Resident 256-thread blocks per SM the row-major kernel is built for (its launch bounds).
#ifndef FP8DSA_FLAT_BLOCKS
#define FP8DSA_FLAT_BLOCKS 3
#endif
constexpr int kFlatBlocks = FP8DSA_FLAT_BLOCKS;

// Eight floats -> eight fp8 bytes (two words): each byte is the RN, saturating encoding of
// RN32(f * mult), the products taken two per packed instruction; amax is kept by the caller.
template <int kFmt>
__device__ __forceinline__ uint2 quant8(float (&f)[8], float mult) {
#pragma unroll
    for (int e = 0; e < 8; e += 2) mul2_rn(f[e], f[e + 1], mult);
    return make_uint2(cvt_fp8x4<kFmt>(f[0], f[1], f[2], f[3]), cvt_fp8x4<kFmt>(f[4], f[5], f[6], f[7]));
}

// The transposed bytes in format kFmtT of the products that quant8<kFmt> left in f (one
// product per element, one conversion per format); `q` are quant8's own bytes.
template <int kFmt, int kFmtT>
__device__ __forceinline__ uint2 second_format(const float (&f)[8], uint2 q) {
    if constexpr (kFmtT == kFmt)
        return q;
    else
        return make_uint2(cvt_fp8x4<kFmtT>(f[0], f[1], f[2], f[3]), cvt_fp8x4<kFmtT>(f[4], f[5], f[6], f[7]));
}

template <int kFmt>
__device__ __forceinline__ uint8_t convert1(float v, float mult) {
    return static_cast<uint8_t>(cvt_fp8x2<kFmt>(__fmul_rn(v, mult), 0.0f) & 0xFFu);
}

// Device-scope acquire-release fetch-add: orders this thread's earlier writes (its block's
// amax) before the increment, and later reads after it.
__device__ __forceinline__ unsigned ticket_acq_rel(unsigned* p) {
    unsigned old;
    asm volatile("atom.acq_rel.gpu.global.add.u32 %0, [%1], 1;" : "=r"(old) : "l"(p) : "memory");
    return old;
}

constexpr int kHistPrefetch = 64;

// The fold needs the ring's history window, which does not change during the kernel (only
// the last block writes it, at the very end).  ring_peek, called after the PDL wait, starts the
// load of slot threadIdx.x into a register; ring_stash puts it in shared memory just before the
// final barrier, so the load's latency hides behind the kernel's work instead of stalling the
// first warp, and the fold pays no dependent L2 round trip per slot.  A deferred fold (done by
// the kernel that follows) needs no window.
__device__ __forceinline__ bool ring_window_wanted(const QArgs& a) {
    return a.ring_state != nullptr && !a.defer_fold && a.hist_len <= kHistPrefetch &&
           static_cast<int>(threadIdx.x) < a.hist_len;
}
__device__ __forceinline__ float ring_peek(const QArgs& a) {
    return ring_window_wanted(a) ? __ldcg(a.ring_state + threadIdx.x) : 0.0f;
}
__device__ __forceinline__ void ring_stash(const QArgs& a, float v, float* hist) {
    if (ring_window_wanted(a)) hist[threadIdx.x] = v;
}

// One thread per block and tensor, with the block's amax `m`: one atomicMax, then (with a
// ring) the ticket; the block that draws the last ticket folds: scale_used = step,
// hist[idx] = amax, scale = max(RN32(peak / fp8_max) / 2^m, 1e-12), amax and done slots
// re-zeroed.  `hist` is the prefetched window.
__device__ __forceinline__ void job_finish(const QArgs& a, float m, float step, bool first_block,
                                           const float* hist) {
    if (a.amax_accum != nullptr) atomicMax(reinterpret_cast<unsigned*>(a.amax_accum), __float_as_uint(m));
    if (a.ring_state != nullptr && a.defer_fold) {
        // the fold runs in the kernel that follows (no ticket: the launch ends with no tail)
        if (first_block && a.scale_used_out != nullptr) *a.scale_used_out = step;
        return;
    }
    if (a.ring_state != nullptr) {
        float* st = a.ring_state;
        const int n = a.hist_len;
        unsigned* done = reinterpret_cast<unsigned*>(st + n + 3);
        const unsigned ticket = ticket_acq_rel(done);
        if (ticket != a.nblocks - 1u) return;
        const float am = __uint_as_float(atomicOr(reinterpret_cast<unsigned*>(st + n + 2), 0u));
        st[n + 1] = step;
        st[a.hist_idx] = am;
        float peak = am;
        if (n <= kHistPrefetch) {
            for (int i = 0; i < n; ++i)
                if (i != a.hist_idx) peak = fmaxf(peak, hist[i]);
        } else {
            for (int i = 0; i < n; ++i) peak = fmaxf(peak, __ldcg(st + i));
        }
        st[n] = fmaxf(__fdiv_rn(__fdiv_rn(peak, a.fp8_max), a.pow2_margin), 1e-12f);
        st[n + 2] = 0.0f;
        atomicExch(done, 0u);
        if (a.amax_out != nullptr) *a.amax_out = am;
        if (a.scale_used_out != nullptr) *a.scale_used_out = step;
    } else if (a.scale_used_out != nullptr && first_block) {
        *a.scale_used_out = step;
    }
}

// Block-wide amax reduce followed by job_finish on thread 0.  Every thread must call this.
__device__ __forceinline__ void block_finish(const QArgs& a, float amax, float step, bool first_block,
                                             const float* hist) {
    __shared__ float red[32];
    const int tid = threadIdx.x;
    amax = warp_max(amax);
    if ((tid & 31) == 0) red[tid >> 5] = amax;
    __syncthreads();
    if (tid != 0) return;
    const int nwarps = (blockDim.x + 31) >> 5;
    float m = red[0];
    for (int w = 1; w < nwarps; ++w) m = fmaxf(m, red[w]);
    job_finish(a, m, step, first_block, hist);
}

// ----------------------------------------------------------------------------------------
// Row-major quantize: flat, grid-stride, 16 elements per thread per iteration.
// ----------------------------------------------------------------------------------------
// A tensor with out2 also gets its bytes in format kFmt2 (the same products, rounded once
// more; kFmt2 == kFmt copies the same bytes), row-major like out.
template <class In, int kFmt, int kFmt2>
__global__ void __launch_bounds__(kThreads, kFlatBlocks) quant_flat_kernel(const __grid_constant__ QBatch batch) {
    pdl_trigger();
    pdl_wait();
    zero_side_job(batch);
    // each tensor owns a contiguous range of blocks, sized to its share of the elements
    int jb = 0;
    while (jb + 1 < batch.njobs && static_cast<int>(blockIdx.x) >= batch.job[jb + 1].tile_begin) ++jb;
    const QArgs& a = batch.job[jb];
    const int64_t lb = static_cast<int64_t>(blockIdx.x) - a.tile_begin;  // block within the tensor
    __shared__ float s_hist[kHistPrefetch];
    const float hist_v = ring_peek(a);
    const float step = __ldg(a.scale);
    const float mult = __frcp_rn(step);
    const auto* x = static_cast<const typename In::E*>(a.x);
    uint8_t* const out2 = a.out2;
    float amax = 0.0f;
    typename In::Acc acc = In::acc_zero();  // running max of |x| over the vector chunks
    const int64_t gstride = static_cast<int64_t>(a.nblocks) * blockDim.x;
    const int64_t tid = lb * blockDim.x + threadIdx.x;
    const int64_t n16 = a.vec_in ? a.numel / 16 : 0;
    // kDepth chunks of 16 elements per thread in flight: every load of a round is issued before
    // the round's first conversion
    constexpr int kDepth = sizeof(typename In::E) == 4 ? 2 : kFlatDepth;
    auto load_round = [&](int64_t g, typename In::Raw (&r)[kDepth][2]) {
#pragma unroll
        for (int d = 0; d < kDepth; ++d) {
            const int64_t gd = g + d * gstride;
            if (gd < n16) {
                r[d][0] = In::load_raw(x + gd * 16);
                r[d][1] = In::load_raw(x + gd * 16 + 8);
            }
        }
    };
    auto convert_round = [&](int64_t g, const typename In::Raw (&r)[kDepth][2]) {
#pragma unroll
        for (int d = 0; d < kDepth; ++d) {
            const int64_t gd = g + d * gstride;
            if (gd >= n16) break;
            float f0[8], f1[8];
            In::acc_max(acc, r[d][0]);
            In::acc_max(acc, r[d][1]);
            In::unpack(r[d][0], f0);
            In::unpack(r[d][1], f1);
            const uint2 lo = quant8<kFmt>(f0, mult);
            const uint2 hi = quant8<kFmt>(f1, mult);
            *reinterpret_cast<uint4*>(a.out + gd * 16) = make_uint4(lo.x, lo.y, hi.x, hi.y);
            if (out2 != nullptr) {
                const uint2 lo2 = second_format<kFmt, kFmt2>(f0, lo);
                const uint2 hi2 = second_format<kFmt, kFmt2>(f1, hi);
                *reinterpret_cast<uint4*>(out2 + gd * 16) = make_uint4(lo2.x, lo2.y, hi2.x, hi2.y);
            }
        }
    };
#if FP8DSA_FLAT_PIPE
    // software-pipelined: the next round's loads are in flight while this round converts
    {
        typename In::Raw r[kDepth][2];
        int64_t g = tid;
        if (g < n16) load_round(g, r);
        for (; g < n16; g += kDepth * gstride) {
            typename In::Raw nx[kDepth][2];
            const int64_t gn = g + kDepth * gstride;
            if (gn < n16) load_round(gn, nx);
            convert_round(g, r);
            if (gn < n16) {
#pragma unroll
                for (int d = 0; d < kDepth; ++d) {
                    r[d][0] = nx[d][0];
                    r[d][1] = nx[d][1];
                }
            }
        }
    }
#else
    for (int64_t g = tid; g < n16; g += kDepth * gstride) {
        typename In::Raw r[kDepth][2];
        load_round(g, r);
        convert_round(g, r);
    }
#endif
    amax = In::acc_value(acc);
    for (int64_t i = n16 * 16 + tid; i < a.numel; i += gstride) {
        const float v = In::cvt(x[i]);
        amax = fmaxf(amax, fabsf(v));
        a.out[i] = convert1<kFmt>(v, mult);
        if (out2 != nullptr) out2[i] = convert1<kFmt2>(v, mult);
    }
    ring_stash(a, hist_v, s_hist);
    block_finish(a, amax, step, lb == 0, s_hist);
}

// ----------------------------------------------------------------------------------------
// Row-major bytes plus per-tile column sums (a gradient quantized for the bias gradient), for
// batches that write no transposed bytes.  Each block covers 128 rows x 128 columns of one
// tensor: thread t owns the 8 columns 8 * (t % 16) .. + 7 and the rows t / 16 + 16 i
// (i = 0..7), issues its eight 16-byte loads at once (a warp reads two 256-byte row pieces per
// load), and keeps the 8 column sums of its rows in registers.  The two row threads of a
// column group in a warp combine through one shuffle, then the 8 warps in order through shared
// memory, into colsum[tile row][column] (the layout the dual quantize writes; the summation
// order is this kernel's own).  Eight rows per thread keep the reduction a small share of the
// work (measured on B200: 128 x 64 blocks of four rows per thread spent most of their
// instructions on it).
// ----------------------------------------------------------------------------------------
#ifndef FP8DSA_RC_ROWS
#define FP8DSA_RC_ROWS 8
#endif
constexpr int kRcRows = FP8DSA_RC_ROWS;             // rows per thread (8 or 16)
constexpr int kRcGroups = 2 * kRcRows;              // 8-column groups per block
constexpr int kRcCols = 8 * kRcGroups;              // 128 (or 256) columns per block
constexpr int kRcStride = kTile / kRcRows;          // row distance between a thread's rows
static_assert(kRcRows == 8 || kRcRows == 16, "8 or 16 rows per thread");

template <class In, int kFmt>
__global__ void __launch_bounds__(kThreads, (sizeof(typename In::E) == 4 || kRcRows > 8) ? 2 : 3)
    quant_rows_colsum_kernel(const __grid_constant__ QBatch batch) {
    pdl_trigger();
    pdl_wait();
    zero_side_job(batch);
    int jb = 0;
    while (jb + 1 < batch.njobs && static_cast<int>(blockIdx.x) >= batch.job[jb + 1].tile_begin) ++jb;
    const QArgs& a = batch.job[jb];
    const int local = static_cast<int>(blockIdx.x) - a.tile_begin;
    const int ty = local / a.tiles_x, tx = local - (local / a.tiles_x) * a.tiles_x;
    __shared__ float s_hist[kHistPrefetch];
    __shared__ float s_cs[kThreads / 32][kRcCols];
    const float hist_v = ring_peek(a);
    const float step = __ldg(a.scale);
    const float mult = __frcp_rn(step);
    const auto* x = static_cast<const typename In::E*>(a.x);
    const int64_t rows = a.rows, cols = a.cols;
    const int t = threadIdx.x, w = t >> 5, lane = t & 31;
    const int cg = t % kRcGroups, rt = t / kRcGroups;
    const int64_t r0 = static_cast<int64_t>(ty) * kTile;
    const int64_t gc = static_cast<int64_t>(tx) * kRcCols + 8 * cg;
    const bool colsum = a.colsum != nullptr;
    float cs[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) cs[e] = 0.0f;
    float amax = 0.0f;
    typename In::Acc acc = In::acc_zero();
    if (a.vec_in && a.vec_out && r0 + kTile <= rows && gc + 8 <= cols) {
        typename In::Raw raw[kRcRows];
#pragma unroll
        for (int i = 0; i < kRcRows; ++i) raw[i] = In::load_raw(x + (r0 + rt + kRcStride * i) * cols + gc);
#pragma unroll
        for (int i = 0; i < kRcRows; ++i) {
            float f[8];
            In::acc_max(acc, raw[i]);
            In::unpack(raw[i], f);
            if (colsum) {
#pragma unroll
                for (int e = 0; e < 8; e += 2) add2_rn(cs[e], cs[e + 1], f[e], f[e + 1]);
            }
            *reinterpret_cast<uint2*>(a.out + (r0 + rt + kRcStride * i) * cols + gc) = quant8<kFmt>(f, mult);
        }
    } else {
#pragma unroll 1
        for (int i = 0; i < kRcRows; ++i) {
            const int64_t gr = r0 + rt + kRcStride * i;
            float f[8];
            if (gr < rows && a.vec_in && gc + 8 <= cols) {
                In::load8(x + gr * cols + gc, f);
            } else {
#pragma unroll
                for (int e = 0; e < 8; ++e) f[e] = (gr < rows && gc + e < cols) ? In::cvt(x[gr * cols + gc + e]) : 0.0f;
            }
#pragma unroll
            for (int e = 0; e < 8; ++e) amax = fmaxf(amax, fabsf(f[e]));
            if (colsum) {
#pragma unroll
                for (int e = 0; e < 8; e += 2) add2_rn(cs[e], cs[e + 1], f[e], f[e + 1]);
            }
            const uint2 q = quant8<kFmt>(f, mult);
            if (gr < rows && gc < cols) {
                uint8_t* dst = a.out + gr * cols + gc;
                if (a.vec_out && gc + 8 <= cols) {
                    *reinterpret_cast<uint2*>(dst) = q;
                } else {
                    const uint32_t qq[2] = {q.x, q.y};
                    for (int e = 0; e < 8 && gc + e < cols; ++e) dst[e] = static_cast<uint8_t>(qq[e >> 2] >> (8 * (e & 3)));
                }
            }
        }
    }
    amax = fmaxf(amax, In::acc_value(acc));
    if (colsum) {
        // with 8 rows per thread, lanes l and l ^ 16 share the column group (rows t / 16 and
        // t / 16 + 1); then the 8 warps in order
        if constexpr (kRcGroups < 32) {
#pragma unroll
            for (int e = 0; e < 8; ++e) cs[e] += __shfl_xor_sync(0xFFFFFFFFu, cs[e], 16);
        }
        if (lane < kRcGroups) {
#pragma unroll
            for (int e = 0; e < 8; ++e) s_cs[w][8 * lane + e] = cs[e];
        }
        __syncthreads();
        const int64_t c = static_cast<int64_t>(tx) * kRcCols + t;
        if (t < kRcCols && c < cols) {
            float sum = 0.0f;
#pragma unroll
            for (int v = 0; v < kThreads / 32; ++v) sum += s_cs[v][t];
            a.colsum[static_cast<int64_t>(ty) * cols + c] = sum;
        }
    }
    ring_stash(a, hist_v, s_hist);
    block_finish(a, amax, step, local == 0, s_hist);
}

// ----------------------------------------------------------------------------------------
// Transposed / dual quantize over the 128 x 128 tiles of every tensor of the batch.
//  * Persistent (large batches): two CTAs per SM walk all tiles; each input tile arrives by
//    one TMA copy into a two-stage shared-memory ring, so the next tile loads while this one
//    is converted (tensors whose rows are not 16-byte aligned are read directly instead).
//  * One tile per CTA (small batches): three CTAs per SM, the input read straight into
//    registers, so every resident CTA has its whole tile in flight at once.
// Either way the fp8 bytes go through a swizzled shared byte tile for the transpose.
// ----------------------------------------------------------------------------------------
// Shared-memory layout of the tiled kernel.  Persistent: two input stages fed by TMA, the
// fp8 byte tile, the column sums, one mbarrier per stage.  One tile per CTA: the byte tile
// and the column sums only (its input is loaded into registers).
template <class In, bool kPersist>
struct TiledCfg {
    static constexpr bool kF32 = sizeof(typename In::E) == 4;
    static constexpr int kStages = kPersist ? 2 : 0;
    static constexpr int kRawBytes = kTile * kTile * static_cast<int>(sizeof(typename In::E));
    // persistent: byte tile and column sums double-buffered, so a tile's transposed stores
    // need no barrier before the next tile's conversion
    static constexpr int kBufs = kPersist ? 2 : 1;
    static constexpr int kOffTile = kStages * kRawBytes;               // 128 x 128 fp8 byte tile(s)
    static constexpr int kOffCsum = kOffTile + kBufs * kTile * kTile;  // 8 x 128 fp32 column sums
    static constexpr int kOffBar = kOffCsum + kBufs * 8 * kTile * 4;   // one mbarrier per stage
    static constexpr int kSmem = kOffBar + kStages * 8 + 1024; // + slack to align the base
    static constexpr int kMinBlocks = kPersist ? (kF32 ? 1 : 2) : (kF32 ? 2 : 3);
};

// Tile `local` of a tensor -> (tile row, tile column): groups of a.tile_group tile rows,
// walked column by column within a group.  Row order (group 1) keeps the tiles in flight on
// the same input rows; groups of 4 put four neighbouring 128-byte pieces of each transposed
// output row in flight together, which the dual quantize of very tall tensors prefers.
__device__ __forceinline__ void tile_coords(const QArgs& a, int local, int& ty, int& tx) {
    const int G = a.tile_group;
    if (G <= 1) {
        ty = local / a.tiles_x;
        tx = local % a.tiles_x;
        return;
    }
    const int per_group = G * a.tiles_x;
    const int grp = local / per_group;
    const int first = grp * G;
    const int gh = min(a.tiles_y - first, G);
    const int within = local - grp * per_group;
    ty = first + within % gh;
    tx = within / gh;
}

__device__ __forceinline__ int tile_job(const QBatch& b, int tl) {
    int jb = 0;
    while (jb + 1 < b.njobs && tl >= b.job[jb + 1].tile_begin) ++jb;
    return jb;
}

// kTOnly (persistent only): every job of the batch writes transposed bytes and no row-major
// ones, so full tiles take the stepped fast path; batches with row-major bytes keep the
// general loop (measured on B200: the fast path in their instance slows the dual quantize).
template <class In, int kFmt, int kFmtT, bool kPersist, bool kTOnly = false>
__global__ void __launch_bounds__(kThreads, TiledCfg<In, kPersist>::kMinBlocks)
    quant_tiled_kernel(const __grid_constant__ QBatch batch, const WaitCtl ctl) {
    using C = TiledCfg<In, kPersist>;
    using E = typename In::E;
    extern __shared__ uint8_t dsmem[];
    const uint32_t base = smem_addr(dsmem);
    uint8_t* smem = dsmem + (((base + 1023u) & ~1023u) - base);
    uint64_t* bar = reinterpret_cast<uint64_t*>(smem + C::kOffBar);
    __shared__ float s_hist[kMaxJobs][kHistPrefetch];
    __shared__ float s_red[kMaxJobs][kThreads / 32];
    __shared__ int s_abort;

    const int t = threadIdx.x;
    const int njobs = batch.njobs;
    if constexpr (kPersist) {
        if (t == 0) {
            for (int s = 0; s < C::kStages; ++s) mbar_init(&bar[s], 1);
            fence_mbar_init();
            s_abort = 0;
            for (int jb = 0; jb < njobs; ++jb)
                if (batch.job[jb].tma) prefetch_tensormap(&batch.map[jb]);
        }
        __syncthreads();
    }
    pdl_trigger();
    pdl_wait();
    zero_side_job(batch);
    // the window of each tensor this CTA may fold (one tile per CTA: only its own tensor)
    float hist_v[kMaxJobs] = {0.0f, 0.0f, 0.0f};
    const int own_job = kPersist ? 0 : tile_job(batch, static_cast<int>(blockIdx.x));
    if constexpr (kPersist) {
#pragma unroll
        for (int jb = 0; jb < kMaxJobs; ++jb)
            if (jb < njobs) hist_v[jb] = ring_peek(batch.job[jb]);
    } else {
        hist_v[0] = ring_peek(batch.job[own_job]);
    }

    const int total = batch.tiles_total;
    const int gstride = static_cast<int>(gridDim.x);
    uint32_t pending = 0;  // thread 0: stages with a load in flight
    // Thread 0: start the load of tile `tl` into stage `s` (TMA-fed tensors only).
    auto issue = [&](int tl, int s) {
        const int jb = tile_job(batch, tl);
        const QArgs& a = batch.job[jb];
        if (!kPersist || !a.tma) return;
        const int local = tl - a.tile_begin;
        mbar_arrive_expect_tx(&bar[s], C::kRawBytes);
        int ty, tx;
        tile_coords(a, local, ty, tx);
        tma_load_3d(smem + s * C::kRawBytes, &batch.map[jb], &bar[s], tx * kTile, ty * kTile, 0);
        pending |= 1u << s;
    };
    if (t == 0) {
        for (int s = 0; s < C::kStages; ++s) {
            const int tl = static_cast<int>(blockIdx.x) + s * gstride;
            if (tl < total) issue(tl, s);
        }
    }

    const int j = t & 15;   // 8-column group of the tile
    const int rr = t >> 4;  // row within each 16-row slab
    const int w = t >> 5, lane = t & 31;
    const int cgl = lane & 3, rg = lane >> 2;
    float am0 = 0.0f, am1 = 0.0f, am2 = 0.0f;  // this thread's amax per tensor
    uint32_t parity = 0;                       // bit s: parity of stage s's next completion
    bool aborted = false;
    int it = 0;
    for (int tl = static_cast<int>(blockIdx.x); tl < total; tl += gstride, ++it) {
        const int s = kPersist ? it % (C::kStages > 0 ? C::kStages : 1) : 0;
        const int jb = tile_job(batch, tl);
        const QArgs& a = batch.job[jb];
        const bool row_out = !kTOnly && a.out != nullptr;
        const bool col_out = a.out_t != nullptr;  // transposed output (else row-major + column sums only)
        const bool colsum = a.colsum != nullptr;
        const float mult = __frcp_rn(__ldg(a.scale));
        const auto* x = static_cast<const E*>(a.x);
        const int64_t rows = a.rows, cols = a.cols;
        const int local = tl - a.tile_begin;
        int tile_y, tile_x;
        tile_coords(a, local, tile_y, tile_x);
        const int64_t r0 = static_cast<int64_t>(tile_y) * kTile;
        const int64_t c0 = static_cast<int64_t>(tile_x) * kTile;
        const int64_t gc = c0 + 8 * j;
        const bool from_smem = kPersist && a.tma != 0;
        const bool interior = !from_smem && a.vec_in && r0 + kTile <= rows && c0 + kTile <= cols;
        bool ok = true;
        if (from_smem) {
            ok = mbar_wait_bounded(&bar[s], (parity >> s) & 1u, ctl, &s_abort, kStatusWaitQuantize);
            if (ok) {
                parity ^= 1u << s;
                if (t == 0) pending &= ~(1u << s);
            }
        }
        const E* stage = reinterpret_cast<const E*>(smem + s * C::kRawBytes);
        // The tile's fp8 bytes, 128 rows x 128 bytes, in the first 16 KB of stage s: the
        // 16-byte chunk c of row r lives at chunk c ^ ((r >> 4) & 7).
        const int bsel = C::kBufs > 1 ? (it & 1) : 0;
        uint32_t* tile = reinterpret_cast<uint32_t*>(smem + C::kOffTile + bsel * kTile * kTile);
        float(*csum)[kTile] = reinterpret_cast<float(*)[kTile]>(smem + C::kOffCsum + bsel * 8 * kTile * 4);

        float tamax = 0.0f;                          // amax of the rows read element-wise
        typename In::Acc acc = In::acc_zero();       // amax of the rows read as raw chunks
        float cs[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) cs[e] = 0.0f;
        typename In::Raw raw[8];
        if (from_smem) {
            // out-of-range rows / columns of an edge tile were zero-filled by the copy
#pragma unroll
            for (int i = 0; i < 8; ++i) raw[i] = In::lds_raw(stage + (rr + 16 * i) * kTile + 8 * j);
        } else if (interior) {
#pragma unroll
            for (int i = 0; i < 8; ++i) raw[i] = In::load_raw(x + (r0 + rr + 16 * i) * cols + gc);
        }
        // a full tile with vector-aligned outputs: no per-row checks, addresses stepped (in the
        // one-tile-per-CTA kernel, which is issue-bound on small batches; the persistent one keeps
        // its register budget)
        const bool full = (!kPersist || kTOnly) && (from_smem || interior) && r0 + kTile <= rows &&
                          c0 + kTile <= cols && (!row_out || a.vec_out);
        if (full) {
            uint8_t* orow = row_out ? a.out + (r0 + rr) * cols + gc : nullptr;
            const int64_t ostep = 16 * cols;
            uint32_t* trow = tile + rr * 32 + (j & 1) * 2;
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                float f[8];
                In::acc_max(acc, raw[i]);
                In::unpack(raw[i], f);
                if (colsum) {
#pragma unroll
                    for (int e = 0; e < 8; e += 2) add2_rn(cs[e], cs[e + 1], f[e], f[e + 1]);
                }
                const uint2 q = quant8<kFmt>(f, mult);  // leaves the products in f
                if (row_out) *reinterpret_cast<uint2*>(orow + i * ostep) = q;
                if (col_out)
                    *reinterpret_cast<uint2*>(trow + i * 512 + (((j >> 1) ^ i) << 2)) = second_format<kFmt, kFmtT>(f, q);
            }
        } else {
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const int r = rr + 16 * i;
            const int64_t gr = r0 + r;
            float f[8];
            if (from_smem || interior) {
                In::acc_max(acc, raw[i]);
                In::unpack(raw[i], f);
            } else {
                if (gr < rows && a.vec_in && gc + 8 <= cols) {
                    In::load8(x + gr * cols + gc, f);
                } else {
#pragma unroll
                    for (int e = 0; e < 8; ++e)
                        f[e] = (gr < rows && gc + e < cols) ? In::cvt(x[gr * cols + gc + e]) : 0.0f;
                }
#pragma unroll
                for (int e = 0; e < 8; ++e) tamax = fmaxf(tamax, fabsf(f[e]));
            }
            if (colsum) {
#pragma unroll
                for (int e = 0; e < 8; e += 2) add2_rn(cs[e], cs[e + 1], f[e], f[e + 1]);
            }
            const uint2 q = quant8<kFmt>(f, mult);  // leaves the products in f
            if (row_out && gr < rows) {
                uint8_t* dst = a.out + gr * cols + gc;
                if (a.vec_out && gc + 8 <= cols) {
                    *reinterpret_cast<uint2*>(dst) = q;
                } else {
                    const uint32_t qq[2] = {q.x, q.y};
                    for (int e = 0; e < 8 && gc + e < cols; ++e)
                        dst[e] = static_cast<uint8_t>(qq[e >> 2] >> (8 * (e & 3)));
                }
            }
            if (col_out) {
                const int chunk = (j >> 1) ^ i;  // (r >> 4) & 7 == i
                *reinterpret_cast<uint2*>(&tile[r * 32 + chunk * 4 + (j & 1) * 2]) = second_format<kFmt, kFmtT>(f, q);
            }
        }
        }
        tamax = fmaxf(tamax, In::acc_value(acc));
        if (jb == 0)
            am0 = fmaxf(am0, tamax);
        else if (jb == 1)
            am1 = fmaxf(am1, tamax);
        else
            am2 = fmaxf(am2, tamax);
        if (colsum) {
            // lanes l and l ^ 16 share the column group; then the 8 warps go through shared memory
#pragma unroll
            for (int e = 0; e < 8; ++e) cs[e] += __shfl_xor_sync(0xFFFFFFFFu, cs[e], 16);
            if ((t & 16) == 0) {
#pragma unroll
                for (int e = 0; e < 8; ++e) csum[w][8 * j + e] = cs[e];
            }
        }
        // The byte tile is complete; every thread agrees on `ok`.
        if (!__syncthreads_and(ok)) {
            aborted = true;
            break;
        }
        if (t == 0) {  // stage s has been read: refill it
            const int nt = tl + C::kStages * gstride;
            if (nt < total) issue(nt, s);
        }

        if (colsum && t < kTile && c0 + t < cols) {
            float sum = 0.0f;
#pragma unroll
            for (int v = 0; v < 8; ++v) sum += csum[v][t];
            a.colsum[static_cast<int64_t>(tile_y) * cols + c0 + t] = sum;
        }

        // Phase 2 (transposed output only): warp w owns tile columns 16w .. 16w+15; lane ->
        // (column group of 4, 16 rows).
        if (col_out) {
        uint32_t W[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) W[i] = tile[(16 * rg + i) * 32 + ((w ^ rg) << 2) + cgl];
        uint32_t O[4][4];
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            const uint32_t x0 = __byte_perm(W[4 * k], W[4 * k + 1], 0x5140);
            const uint32_t x1 = __byte_perm(W[4 * k], W[4 * k + 1], 0x7362);
            const uint32_t y0 = __byte_perm(W[4 * k + 2], W[4 * k + 3], 0x5140);
            const uint32_t y1 = __byte_perm(W[4 * k + 2], W[4 * k + 3], 0x7362);
            O[0][k] = __byte_perm(x0, y0, 0x5410);
            O[1][k] = __byte_perm(x0, y0, 0x7632);
            O[2][k] = __byte_perm(x1, y1, 0x5410);
            O[3][k] = __byte_perm(x1, y1, 0x7632);
        }
        const int64_t gr0 = r0 + 16 * rg;
#pragma unroll
        for (int jj = 0; jj < 4; ++jj) {
            const int64_t c = c0 + 4 * (4 * w + cgl) + jj;
            if (c >= cols || gr0 >= rows) continue;
            uint8_t* dst = a.out_t + c * rows + gr0;
            if (a.vec_out_t && gr0 + 16 <= rows) {
                *reinterpret_cast<uint4*>(dst) = make_uint4(O[jj][0], O[jj][1], O[jj][2], O[jj][3]);
            } else {
                for (int b = 0; b < 16 && gr0 + b < rows; ++b)
                    dst[b] = static_cast<uint8_t>(O[jj][b >> 2] >> (8 * (b & 3)));
            }
        }
        }
        // One buffer: the byte tile and the column sums are free for the next tile only after
        // every thread's transposed stores.  Two: the next tile fills the other buffer, and the
        // barrier after its conversion orders these reads before the buffer's next reuse; kept
        // anyway when row-major bytes are written (measured on B200: the dual quantize loses
        // 3-6% when its warps drift a tile apart, the transposed one gains 2%).
        if (C::kBufs == 1 || batch.row_out_any) __syncthreads();
    }

    if (aborted) {
        // A tile never arrived: let this CTA's copies in flight land, leave the fold undone
        // (the status word reports the failure) and return.
        if (t == 0) {
            for (int s = 0; s < C::kStages; ++s)
                if ((pending >> s) & 1u) mbar_wait_bounded(&bar[s], (parity >> s) & 1u, ctl, nullptr, kStatusWaitDrain);
        }
        return;
    }

    // Per-tensor block maxima; then one thread per tensor draws that tensor's ticket.
    if constexpr (kPersist) {
        am0 = warp_max(am0);
        am1 = warp_max(am1);
        am2 = warp_max(am2);
        if (lane == 0) {
            s_red[0][w] = am0;
            s_red[1][w] = am1;
            s_red[2][w] = am2;
        }
    } else {
        // one tile, one tensor: the other two maxima are zero
        am0 = warp_max(fmaxf(am0, fmaxf(am1, am2)));
        if (lane == 0) s_red[0][w] = am0;
    }
    if constexpr (kPersist) {
#pragma unroll
        for (int jb = 0; jb < kMaxJobs; ++jb)
            if (jb < njobs) ring_stash(batch.job[jb], hist_v[jb], s_hist[jb]);
    } else {
        ring_stash(batch.job[own_job], hist_v[0], s_hist[own_job]);
    }
    __syncthreads();
    // Persistent: every CTA finishes every tensor.  One tile per CTA: only its own tensor.
    if (t < njobs && (kPersist || t == own_job)) {
        const int row = kPersist ? t : 0;
        float m = s_red[row][0];
#pragma unroll
        for (int v = 1; v < kThreads / 32; ++v) m = fmaxf(m, s_red[row][v]);
        const QArgs& a = batch.job[t];
        const bool first = kPersist ? blockIdx.x == 0 : static_cast<int>(blockIdx.x) == a.tile_begin;
        job_finish(a, m, __ldg(a.scale), first, s_hist[t]);
    }
}

// ----------------------------------------------------------------------------------------
// Amax of up to three tensors in one launch (blockIdx.y = tensor); the last block of each
// tensor publishes its step / amax / ring seed and re-zeroes its scratch.
// ----------------------------------------------------------------------------------------
struct AmaxArgs {
    const void* x[3];
    int in_type[3];
    int64_t numel[3];
    float fp8_max[3], pow2_margin[3];
    float* scale_out[3];
    float* amax_out[3];
    float* ring_state[3];
    int hist_len[3], hist_idx[3];
    uint32_t* scratch[3];  // [amax bits, done]
    int vec[3];
};

template <class In>
__device__ __forceinline__ float amax_range(const void* xv, int64_t numel, int vec) {
    const auto* x = static_cast<const typename In::E*>(xv);
    float amax = 0.0f;
    const int64_t gstride = static_cast<int64_t>(gridDim.x) * blockDim.x;
    const int64_t tid = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
    const int64_t n16 = vec ? numel / 16 : 0;
    for (int64_t g = tid; g < n16; g += gstride) {
        float f0[8], f1[8];
        In::load8(x + g * 16, f0);
        In::load8(x + g * 16 + 8, f1);
#pragma unroll
        for (int e = 0; e < 8; ++e) amax = fmaxf(amax, fmaxf(fabsf(f0[e]), fabsf(f1[e])));
    }
    for (int64_t i = n16 * 16 + tid; i < numel; i += gstride) amax = fmaxf(amax, fabsf(In::cvt(x[i])));
    return amax;
}

__global__ void __launch_bounds__(kThreads) amax_jobs_kernel(AmaxArgs a) {
    pdl_trigger();
    pdl_wait();
    const int job = blockIdx.y;
    float amax;
    if (a.in_type[job] == FP8_IN_BF16)
        amax = amax_range<Bf16In>(a.x[job], a.numel[job], a.vec[job]);
    else if (a.in_type[job] == FP8_IN_F16)
        amax = amax_range<F16In>(a.x[job], a.numel[job], a.vec[job]);
    else
        amax = amax_range<F32In>(a.x[job], a.numel[job], a.vec[job]);

    __shared__ float red[32];
    amax = warp_max(amax);
    if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = amax;
    __syncthreads();
    if (threadIdx.x != 0) return;
    float m = red[0];
    for (int w = 1; w < (int)(blockDim.x >> 5); ++w) m = fmaxf(m, red[w]);
    uint32_t* scr = a.scratch[job];
    atomicMax(scr, __float_as_uint(m));
    const unsigned ticket = ticket_acq_rel(scr + 1);
    if (ticket != gridDim.x - 1u) return;
    const float am = __uint_as_float(atomicOr(scr, 0u));
    float peak = am;
    if (a.ring_state[job] != nullptr) {
        float* st = a.ring_state[job];
        const int n = a.hist_len[job];
        st[a.hist_idx[job]] = am;
        for (int i = 0; i < n; ++i) peak = fmaxf(peak, __ldcg(st + i));
        st[n] = fmaxf(__fdiv_rn(__fdiv_rn(peak, a.fp8_max[job]), a.pow2_margin[job]), 1e-12f);
    }
    if (a.scale_out[job] != nullptr)
        *a.scale_out[job] = fmaxf(__fdiv_rn(__fdiv_rn(am, a.fp8_max[job]), a.pow2_margin[job]), 1e-12f);
    if (a.amax_out[job] != nullptr) *a.amax_out[job] = am;
    atomicExch(scr, 0u);
    atomicExch(scr + 1, 0u);
}

// Ring lists for the data-parallel fold (up to kRingChunk rings per launch, by value).
constexpr int kRingChunk = 128;  // 3 KB of kernel parameters
struct RingList {
    fp8_ring_t ring[kRingChunk];
    int n;
};

// out[i] = ring i's amax slot (the maxima its quantize launches left there).
__global__ void ring_collect_kernel(const __grid_constant__ RingList L, float* out) {
    pdl_trigger();
    pdl_wait();
    const int i = static_cast<int>(blockIdx.x * blockDim.x + threadIdx.x);
    if (i < L.n) out[i] = __ldcg(L.ring[i].state + L.ring[i].hist_len + 2);
}

// Fold ring i (one thread each): with `amax` given, that value replaces the slot's (the
// maximum over all ranks), then the same fold the linear entries do after their quantize.
__global__ void ring_fold_list_kernel(const __grid_constant__ RingList L, const float* amax) {
    pdl_trigger();
    pdl_wait();
    const int i = static_cast<int>(blockIdx.x * blockDim.x + threadIdx.x);
    if (i >= L.n) return;
    const fp8_ring_t& r = L.ring[i];
    if (amax != nullptr) r.state[r.hist_len + 2] = __ldcg(amax + i);
    ring_fold_deferred(r.state, r.hist_len, r.hist_idx, r.fp8_max, r.pow2_margin);
}

__global__ void __launch_bounds__(kThreads) colsum_finalize_kernel(const float* partial, int64_t tiles,
                                                                    int64_t cols, uint16_t* out) {
    pdl_trigger();
    pdl_wait();
    const int64_t c = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
    if (c >= cols) return;
    // in-order sum (deterministic); the loads are independent and issued four at a time
    float s = 0.0f;
    int64_t t = 0;
    for (; t + 4 <= tiles; t += 4) {
        const float v0 = __ldcg(partial + t * cols + c);
        const float v1 = __ldcg(partial + (t + 1) * cols + c);
        const float v2 = __ldcg(partial + (t + 2) * cols + c);
        const float v3 = __ldcg(partial + (t + 3) * cols + c);
        s += v0;
        s += v1;
        s += v2;
        s += v3;
    }
    for (; t < tiles; ++t) s += __ldcg(partial + t * cols + c);
    out[c] = __bfloat16_as_ushort(__float2bfloat16_rn(s));
}

// Per-tile column sums of a pre-quantized operand (the bias gradient of a g that arrives as
// fp8): partial[t][c] = RN32(sum over the rows r of tile t of dec(g8[r][c])) * step, rows in
// order.  Each thread sums four adjacent columns of one 128-row tile (a warp reads 128
// contiguous bytes per row); block (0, 0) also zeroes `zero[0 .. zero_words)`.
template <int kFmt>
__global__ void __launch_bounds__(kThreads) colsum_fp8_kernel(const uint8_t* g8, int64_t rows, int64_t cols,
                                                              const float* step, float* partial, uint32_t* zero,
                                                              int64_t zero_words) {
    pdl_trigger();
    pdl_wait();
    if (zero_words > 0 && blockIdx.x == 0 && blockIdx.y == 0)
        for (int64_t i = threadIdx.x; i < zero_words; i += blockDim.x) zero[i] = 0u;
    const int64_t c = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) * 4;
    if (c >= cols) return;
    const int64_t r0 = static_cast<int64_t>(blockIdx.y) * kTile;
    const int64_t r1 = r0 + kTile < rows ? r0 + kTile : rows;
    float s0 = 0.0f, s1 = 0.0f, s2 = 0.0f, s3 = 0.0f;
    for (int64_t r = r0; r < r1; ++r) {
        const uint32_t v = __ldg(reinterpret_cast<const uint32_t*>(g8 + r * cols + c));
        s0 += fp8_to_float<kFmt>(static_cast<uint8_t>(v));
        s1 += fp8_to_float<kFmt>(static_cast<uint8_t>(v >> 8));
        s2 += fp8_to_float<kFmt>(static_cast<uint8_t>(v >> 16));
        s3 += fp8_to_float<kFmt>(static_cast<uint8_t>(v >> 24));
    }
    const float st = __ldg(step);
    float4 out;
    out.x = __fmul_rn(s0, st);
    out.y = __fmul_rn(s1, st);
    out.z = __fmul_rn(s2, st);
    out.w = __fmul_rn(s3, st);
    *reinterpret_cast<float4*>(partial + static_cast<int64_t>(blockIdx.y) * cols + c) = out;
}

// Waves of resident blocks a row-major launch is sized to (measured on B200: one wave, each
// block looping over its share, beats several waves of shorter blocks).
constexpr int kFlatWaves = 1;

// Resident 256-thread blocks per SM of the row-major kernel (its launch bounds ask for as many).
int flat_blocks_per_sm() { return kFlatBlocks; }

template <int kFmt, int kFmt2, class In>
void launch_flat(const QBatch& b, dim3 grid, cudaStream_t stream) {
    launch_ex(quant_flat_kernel<In, kFmt, kFmt2>, grid, dim3(kThreads), 0, stream, 1, b);
}

// Batches of more tiles than this run persistent; smaller ones one tile per CTA.
std::atomic<int64_t> g_persist_min_tiles{1024};
int64_t persist_min_tiles() { return g_persist_min_tiles.load(); }

// Tiled launch.  Persistent: grid = min(tiles, resident CTAs) and every CTA draws one ticket
// per tensor, so each tensor's fold counts gridDim.x blocks.  One tile per CTA: grid = tiles,
// inputs not read by TMA, and each tensor's fold counts that tensor's tiles.
template <int kFmt, int kFmtT, class In, bool kPersist, bool kTOnly = false>
int launch_tiled(QBatch& b, const WaitCtl& ctl, cudaStream_t stream) {
    using C = TiledCfg<In, kPersist>;
    auto kernel = quant_tiled_kernel<In, kFmt, kFmtT, kPersist, kTOnly>;
    static std::once_flag once[kMaxDevices];
    static cudaError_t errs[kMaxDevices];
    static int per_sm_dev[kMaxDevices];
    const int dev = current_device();
    cudaError_t& err = errs[dev];
    int& per_sm = per_sm_dev[dev];
    std::call_once(once[dev], [kernel, &err, &per_sm] {
        err = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmem);
        if (err == cudaSuccess) err = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kernel, kThreads, C::kSmem);
    });
    if (err != cudaSuccess) return fail(FP8DSA_ERR_CUDA, std::string("tiled quantize set-up: ") + cudaGetErrorString(err));
    int grid;
    if (kPersist) {
        const int64_t resident = static_cast<int64_t>(sm_count()) * std::max(1, per_sm);
        grid = static_cast<int>(std::max<int64_t>(1, std::min<int64_t>(b.tiles_total, resident)));
        for (int i = 0; i < b.njobs; ++i) b.job[i].nblocks = static_cast<unsigned>(grid);
    } else {
        grid = b.tiles_total;
        for (int i = 0; i < b.njobs; ++i) {
            const int end = i + 1 < b.njobs ? b.job[i + 1].tile_begin : b.tiles_total;
            b.job[i].nblocks = static_cast<unsigned>(end - b.job[i].tile_begin);
            b.job[i].tma = 0;
        }
    }
    launch_ex(kernel, dim3(grid), dim3(kThreads), C::kSmem, stream, 1, b, ctl);
    return FP8DSA_OK;
}

// kFmtT: format of the transposed bytes (the tiled kernel only; the flat kernel writes one
// orientation, so its launches always have kFmtT == kFmt).
template <int kFmt, int kFmtT, class In>
int launch_quant(QBatch& b, bool tiled, dim3 grid, const WaitCtl& ctl, cudaStream_t stream) {
    if (tiled) {
        bool t_only = kFmtT == kFmt;
        for (int i = 0; i < b.njobs; ++i) t_only = t_only && b.job[i].out == nullptr && b.job[i].colsum == nullptr;
        // transposed-only batches switch to the persistent kernel 8x earlier (measured on B200:
        // its fast-path instance beats one tile per CTA from 256 tiles up; batches with
        // row-major bytes only above the threshold itself)
        const int64_t thr = persist_min_tiles();
        if (t_only && b.tiles_total > thr / 8) {
            if constexpr (kFmtT == kFmt) return launch_tiled<kFmt, kFmtT, In, true, true>(b, ctl, stream);
        }
        if (b.tiles_total > thr) return launch_tiled<kFmt, kFmtT, In, true>(b, ctl, stream);
        return launch_tiled<kFmt, kFmtT, In, false>(b, ctl, stream);
    }
    // the row-major kernel writes a second format only as a second row-major copy (out2)
    launch_flat<kFmt, kFmtT, In>(b, grid, stream);
    return FP8DSA_OK;
}

template <int kFmt, int kFmtT>
int launch_quant_in(fp8_in_t in_type, QBatch& b, bool tiled, dim3 grid, const WaitCtl& ctl, cudaStream_t stream) {
    if (in_type == FP8_IN_BF16) return launch_quant<kFmt, kFmtT, Bf16In>(b, tiled, grid, ctl, stream);
    if (in_type == FP8_IN_F16) return launch_quant<kFmt, kFmtT, F16In>(b, tiled, grid, ctl, stream);
    return launch_quant<kFmt, kFmtT, F32In>(b, tiled, grid, ctl, stream);
}

template <int kFmt>
int launch_rows_colsum(fp8_in_t in_type, const QBatch& b, cudaStream_t stream) {
    const dim3 grid(static_cast<unsigned>(b.tiles_total));
    if (in_type == FP8_IN_BF16)
        launch_ex(quant_rows_colsum_kernel<Bf16In, kFmt>, grid, dim3(kThreads), 0, stream, 1, b);
    else if (in_type == FP8_IN_F16)
        launch_ex(quant_rows_colsum_kernel<F16In, kFmt>, grid, dim3(kThreads), 0, stream, 1, b);
    else
        launch_ex(quant_rows_colsum_kernel<F32In, kFmt>, grid, dim3(kThreads), 0, stream, 1, b);
    return FP8DSA_OK;
}

// Tuning override: FP8DSA_ROWS_COLSUM=0 sends row-major + column-sum batches to the tiled
// kernel instead of the row-major column-sum kernel (read once).
bool row_colsum_enabled() {
    static const bool v = [] {
        const char* e = std::getenv("FP8DSA_ROWS_COLSUM");
        return e == nullptr || std::string(e) != "0";
    }();
    return v;
}

CUtensorMapDataType map_type(fp8_in_t t) {
    return t == FP8_IN_F32 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32
                           : (t == FP8_IN_F16 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16);
}

int check_ring(const fp8_ring_t* ring) {
    if (ring == nullptr) return FP8DSA_OK;
    if (ring->state == nullptr) return fail(FP8DSA_ERR_INVALID_ARG, "ring->state is NULL");
    if (!aligned16(ring->state)) return fail(FP8DSA_ERR_UNSUPPORTED, "ring->state must be 16-byte aligned");
    if (ring->hist_len < 1) return fail(FP8DSA_ERR_INVALID_ARG, "ring->hist_len must be >= 1");
    if (ring->hist_idx < 0 || ring->hist_idx >= ring->hist_len)
        return fail(FP8DSA_ERR_INVALID_ARG, "ring->hist_idx must be in [0, hist_len)");
    if (!(ring->fp8_max > 0.0f)) return fail(FP8DSA_ERR_INVALID_ARG, "ring->fp8_max must be > 0");
    if (!(ring->pow2_margin > 0.0f)) return fail(FP8DSA_ERR_INVALID_ARG, "ring->pow2_margin must be > 0");
    return FP8DSA_OK;
}

}  // namespace

int launch_quantize_batch(const QuantJob* jobs, int njobs, cudaStream_t stream, uint32_t* zero, int64_t zero_words) {
    if (njobs < 1 || njobs > kMaxJobs) return fail(FP8DSA_ERR_INVALID_ARG, "quantize batch of 1..3 tensors");
    const fp8_fmt_t fmt = jobs[0].fmt;
    const fp8_fmt_t fmt_t = jobs[0].fmt_t < 0 ? fmt : static_cast<fp8_fmt_t>(jobs[0].fmt_t);
    const fp8_in_t in_type = jobs[0].in_type;
    // the tiled kernel serves transposed / dual outputs and anything that needs column sums
    auto wants_tiles = [](const QuantJob& j) { return j.out_t != nullptr || j.colsum_partial != nullptr; };
    const bool tiled = wants_tiles(jobs[0]);
    for (int i = 1; i < njobs; ++i)
        if (jobs[i].fmt != fmt || (jobs[i].fmt_t < 0 ? fmt : static_cast<fp8_fmt_t>(jobs[i].fmt_t)) != fmt_t ||
            jobs[i].in_type != in_type || wants_tiles(jobs[i]) != tiled)
            return fail(FP8DSA_ERR_INVALID_ARG, "a quantize batch shares formats, input type and orientation");
    bool any_out2 = false;
    for (int i = 0; i < njobs; ++i) any_out2 = any_out2 || jobs[i].out2 != nullptr;
    if (any_out2 && tiled) return fail(FP8DSA_ERR_INVALID_ARG, "a second row-major copy is a row-major launch");
    if (fmt_t != fmt && !tiled && !any_out2)
        return fail(FP8DSA_ERR_INVALID_ARG, "a second format needs the transposed output or a second row-major copy");
    // row-major bytes + column sums and no transposed bytes: the 128 x 128 block kernel
    bool rows_colsum = tiled && fmt_t == fmt && row_colsum_enabled();
    for (int i = 0; i < njobs; ++i)
        rows_colsum = rows_colsum && jobs[i].out_t == nullptr && jobs[i].out != nullptr && jobs[i].colsum_partial != nullptr;
    QBatch b{};
    b.njobs = njobs;
    b.zero = zero;
    b.zero_words = zero != nullptr ? zero_words : 0;
    const int eb = in_type_bytes(in_type);
    double bytes = 0.0;
    int64_t tiles_total = 0;
    for (int i = 0; i < njobs; ++i) {
        const QuantJob& job = jobs[i];
        QArgs& a = b.job[i];
        a.x = job.x;
        a.rows = job.rows;
        a.cols = job.cols;
        a.numel = job.rows * job.cols;
        a.scale = job.scale;
        a.out = job.out;
        a.out_t = job.out_t;
        a.out2 = job.out2;
        a.scale_used_out = job.scale_used_out;
        a.colsum = job.colsum_partial;
        a.defer_fold = job.ring != nullptr && job.defer_fold ? 1 : 0;
        if (job.ring != nullptr) {
            const int n = job.ring->hist_len;
            a.ring_state = job.ring->state;
            a.hist_len = n;
            a.hist_idx = job.ring->hist_idx;
            a.fp8_max = job.ring->fp8_max;
            a.pow2_margin = job.ring->pow2_margin;
            a.amax_accum = job.ring->state + n + 2;
            a.amax_out = job.amax_out;
        } else {
            a.amax_accum = job.amax_out;
            if (job.amax_out != nullptr) {
                cudaError_t e = cudaMemsetAsync(job.amax_out, 0, sizeof(float), stream);
                if (e != cudaSuccess) return fail(FP8DSA_ERR_CUDA, std::string("memset amax: ") + cudaGetErrorString(e));
            }
        }
        const bool rows_vec = (job.cols * eb) % 16 == 0;
        a.vec_in = aligned16(job.x) && (tiled ? rows_vec : true);
        a.vec_out = (job.out == nullptr) ||
                    (tiled ? ((reinterpret_cast<uintptr_t>(job.out) & 7) == 0 && job.cols % 8 == 0) : aligned16(job.out));
        if (job.out2 != nullptr && !aligned16(job.out2)) a.vec_out = 0;
        a.vec_out_t = job.out_t != nullptr && aligned16(job.out_t) && job.rows % 16 == 0;
        if (!tiled && !(a.vec_in && a.vec_out)) a.vec_in = 0;  // flat kernel: both or neither
        if (tiled && !rows_colsum && a.vec_in && job.rows > 0 && job.cols > 0 && job.rows < (int64_t(1) << 31) &&
            job.cols < (int64_t(1) << 31)) {
            // TMA needs a 16-byte aligned base and row stride (both implied by vec_in here)
            const int64_t ld = job.cols * eb;
            if (encode_tensor_map(&b.map[i], map_type(in_type), job.x, job.cols, job.rows, 1, ld, ld * job.rows,
                                  kTile, kTile, CU_TENSOR_MAP_SWIZZLE_NONE) == FP8DSA_OK)
                a.tma = 1;
            else
                clear_error();  // fall back to direct loads for this tensor
        }
        bytes += static_cast<double>(a.numel) * (eb + (job.out ? 1 : 0) + (job.out_t ? 1 : 0) + (job.out2 ? 1 : 0));
        if (tiled && rows_colsum) {
            // 128 x 128 blocks of the row-major + column-sum kernel (an empty tensor: one block)
            const int64_t tx = std::max<int64_t>(1, (job.cols + kRcCols - 1) / kRcCols);
            const int64_t ty = std::max<int64_t>(1, (job.rows + kTile - 1) / kTile);
            a.tiles_x = static_cast<int>(tx);
            a.tiles_y = static_cast<int>(ty);
            a.tile_group = 1;
            a.tile_begin = static_cast<int>(tiles_total);
            a.nblocks = static_cast<unsigned>(tx * ty);
            tiles_total += tx * ty;
            if (tiles_total > kMaxTiles) return fail(FP8DSA_ERR_UNSUPPORTED, "too many 128 x 128 blocks");
        } else if (tiled) {
            // an empty tensor still gets one (empty) tile
            const int64_t tx = std::max<int64_t>(1, (job.cols + kTile - 1) / kTile);
            const int64_t ty = std::max<int64_t>(1, (job.rows + kTile - 1) / kTile);
            a.tiles_x = static_cast<int>(tx);
            a.tiles_y = static_cast<int>(ty);
            // measured (persistent kernel, B200): groups of 4 tile rows pay off once transposed
            // rows are at least 16 KB apart; row order everywhere else
            a.tile_group = (job.out_t != nullptr && job.rows >= 16384) ? 4 : 1;
            a.tile_begin = static_cast<int>(tiles_total);
            tiles_total += tx * ty;
            if (tiles_total > kMaxTiles) return fail(FP8DSA_ERR_UNSUPPORTED, "too many 128 x 128 tiles");
        }
    }
    dim3 grid;
    WaitCtl ctl{};
    if (tiled) {
        b.tiles_total = static_cast<int>(tiles_total);
        for (int i = 0; i < njobs; ++i) b.row_out_any |= jobs[i].out != nullptr ? 1 : 0;
        const int rc = wait_ctl(&ctl);
        if (rc) return rc;
    } else {
        // one wave: the resident blocks are shared out in proportion to the tensors' sizes
        // (every tensor gets at least one block; none more than one thread per 16 elements)
        const int64_t budget = static_cast<int64_t>(sm_count()) * flat_blocks_per_sm() * kFlatWaves;
        int64_t groups[kMaxJobs], total_groups = 0;
        for (int i = 0; i < njobs; ++i) {
            groups[i] = std::max<int64_t>(1, (b.job[i].numel + 15) / 16);
            total_groups += groups[i];
        }
        int64_t begin = 0;
        for (int i = 0; i < njobs; ++i) {
            const int64_t want = (groups[i] + kThreads - 1) / kThreads;
            const int64_t share = std::max<int64_t>(1, budget * groups[i] / total_groups);
            const int64_t nb = std::max<int64_t>(1, std::min(want, share));
            b.job[i].nblocks = static_cast<unsigned>(nb);
            b.job[i].tile_begin = static_cast<int>(begin);
            begin += nb;
        }
        grid = dim3(static_cast<unsigned>(begin));
    }
    launch_begin(kKindQuantize, stream);
    int rc;
    if (rows_colsum) {
        b.tiles_total = static_cast<int>(tiles_total);
        if (fmt == FP8_E4M3)
            rc = launch_rows_colsum<0>(in_type, b, stream);
        else
            rc = launch_rows_colsum<1>(in_type, b, stream);
        launch_end(kKindQuantize, stream, bytes);
        if (rc) return rc;
        return check_launch("fp8 quantize kernel");
    }
    if (fmt == FP8_E4M3)
        rc = fmt_t == FP8_E4M3 ? launch_quant_in<0, 0>(in_type, b, tiled, grid, ctl, stream)
                               : launch_quant_in<0, 1>(in_type, b, tiled, grid, ctl, stream);
    else
        rc = fmt_t == FP8_E4M3 ? launch_quant_in<1, 0>(in_type, b, tiled, grid, ctl, stream)
                               : launch_quant_in<1, 1>(in_type, b, tiled, grid, ctl, stream);
    launch_end(kKindQuantize, stream, bytes);
    if (rc) return rc;
    return check_launch("fp8 quantize kernel");
}

int launch_quantize(const QuantJob& job, cudaStream_t stream) { return launch_quantize_batch(&job, 1, stream); }

int launch_amax_jobs(const AmaxJob* jobs, int njobs, uint32_t* scratch, cudaStream_t stream) {
    AmaxArgs a{};
    int64_t max_numel = 0;
    double bytes = 0.0;
    for (int i = 0; i < njobs; ++i) {
        const AmaxJob& j = jobs[i];
        a.x[i] = j.x;
        a.in_type[i] = j.in_type;
        a.numel[i] = j.numel;
        a.fp8_max[i] = j.ring.state ? j.ring.fp8_max : j.fp8_max;
        a.pow2_margin[i] = j.ring.state ? j.ring.pow2_margin : j.pow2_margin;
        a.scale_out[i] = j.scale_out;
        a.amax_out[i] = j.amax_out;
        a.ring_state[i] = j.ring.state;
        a.hist_len[i] = j.ring.hist_len;
        a.hist_idx[i] = j.ring.hist_idx;
        a.scratch[i] = j.ring.state ? reinterpret_cast<uint32_t*>(j.ring.state + j.ring.hist_len + 2)
                                    : scratch + 4 * i;
        a.vec[i] = aligned16(j.x);
        max_numel = std::max(max_numel, j.numel);
        bytes += static_cast<double>(j.numel) * in_type_bytes(j.in_type);
    }
    const int64_t want = std::max<int64_t>(1, (max_numel / 16 + kThreads - 1) / kThreads);
    const int per_job = std::max(1, static_cast<int>(std::min<int64_t>(want, static_cast<int64_t>(sm_count()) * 8 / njobs)));
    launch_begin(kKindOther, stream);
    launch_ex(amax_jobs_kernel, dim3(per_job, njobs), dim3(kThreads), 0, stream, 1, a);
    launch_end(kKindOther, stream, bytes);
    return check_launch("fp8 amax kernel");
}

int launch_colsum_finalize(const float* partial, int64_t tiles, int64_t cols, void* out_bf16,
                           cudaStream_t stream) {
    const unsigned blocks = static_cast<unsigned>((cols + kThreads - 1) / kThreads);
    launch_begin(kKindOther, stream);
    launch_ex(colsum_finalize_kernel, dim3(blocks), dim3(kThreads), 0, stream, 1, partial, tiles, cols,
              static_cast<uint16_t*>(out_bf16));
    launch_end(kKindOther, stream, static_cast<double>(tiles) * cols * 4 + cols * 2);
    return check_launch("colsum finalize kernel");
}

int launch_colsum_fp8(const uint8_t* g8, fp8_fmt_t fmt, int64_t rows, int64_t cols, const float* step,
                      float* partial, uint32_t* zero, int64_t zero_words, cudaStream_t stream) {
    if (rows <= 0 || cols <= 0) return FP8DSA_OK;
    if (cols % 4 != 0 || (reinterpret_cast<uintptr_t>(g8) & 3) != 0 || (reinterpret_cast<uintptr_t>(partial) & 15) != 0)
        return fail(FP8DSA_ERR_UNSUPPORTED, "fp8 column sums need cols % 4 == 0, a 4-byte aligned g8 and 16-byte aligned partials");
    const int64_t tiles = (rows + kTile - 1) / kTile;
    if (tiles > 65535) return fail(FP8DSA_ERR_UNSUPPORTED, "too many row tiles for the fp8 column sums");
    const dim3 grid(static_cast<unsigned>((cols / 4 + kThreads - 1) / kThreads), static_cast<unsigned>(tiles));
    launch_begin(kKindOther, stream);
    if (fmt == FP8_E4M3)
        launch_ex(colsum_fp8_kernel<0>, grid, dim3(kThreads), 0, stream, 1, g8, rows, cols, step, partial, zero,
                  zero != nullptr ? zero_words : int64_t(0));
    else
        launch_ex(colsum_fp8_kernel<1>, grid, dim3(kThreads), 0, stream, 1, g8, rows, cols, step, partial, zero,
                  zero != nullptr ? zero_words : int64_t(0));
    launch_end(kKindOther, stream, static_cast<double>(rows) * cols + static_cast<double>(tiles) * cols * 4);
    return check_launch("fp8 column-sum kernel");
}

}  // namespace fp8dsa

using namespace fp8dsa;

extern "C" {

int fp8_scale_ring_init(float* state, int hist_len, cudaStream_t stream) {
    clear_error();
    if (state == nullptr) return fail(FP8DSA_ERR_INVALID_ARG, "state is NULL");
    if (hist_len < 1) return fail(FP8DSA_ERR_INVALID_ARG, "hist_len must be >= 1");
    if (!aligned16(state)) return fail(FP8DSA_ERR_UNSUPPORTED, "state must be 16-byte aligned");
    int rc = check_device();
    if (rc) return rc;
    cudaError_t e = cudaMemsetAsync(state, 0, sizeof(float) * (static_cast<size_t>(hist_len) + 4), stream);
    if (e != cudaSuccess) return fail(FP8DSA_ERR_CUDA, std::string("memset ring: ") + cudaGetErrorString(e));
    return FP8DSA_OK;
}

int fp8_scale_ring_seed(const fp8_ring_t* ring, const void* x, fp8_in_t in_type, int64_t numel,
                        cudaStream_t stream) {
    clear_error();
    if (ring == nullptr) return fail(FP8DSA_ERR_INVALID_ARG, "ring is NULL");
    int rc = check_ring(ring);
    if (rc) return rc;
    if (!valid_in_type(in_type)) return fail(FP8DSA_ERR_INVALID_ARG, "bad in_type");
    if (numel < 0) return fail(FP8DSA_ERR_INVALID_ARG, "numel must be >= 0");
    if (numel > 0 && x == nullptr) return fail(FP8DSA_ERR_INVALID_ARG, "x is NULL");
    rc = check_device();
    if (rc) return rc;
    AmaxJob j;
    j.x = x;
    j.in_type = in_type;
    j.numel = numel;
    j.ring = *ring;
    return launch_amax_jobs(&j, 1, nullptr, stream);
}

int fp8_amax_scale(const void* x, fp8_in_t in_type, int64_t numel, float fp8_max, float pow2_margin,
                   float* scale_out, float* amax_out, uint32_t* scratch, cudaStream_t stream) {
    clear_error();
    if (!valid_in_type(in_type)) return fail(FP8DSA_ERR_INVALID_ARG, "bad in_type");
    if (numel < 0) return fail(FP8DSA_ERR_INVALID_ARG, "numel must be >= 0");
    if (numel > 0 && x == nullptr) return fail(FP8DSA_ERR_INVALID_ARG, "x is NULL");
    if (scale_out == nullptr && amax_out == nullptr) return fail(FP8DSA_ERR_INVALID_ARG, "no output");
    if (scratch == nullptr) return fail(FP8DSA_ERR_INVALID_ARG, "scratch is NULL");
    if (!aligned16(scratch)) return fail(FP8DSA_ERR_UNSUPPORTED, "scratch must be 16-byte aligned");
    if (!(fp8_max > 0.0f) || !(pow2_margin > 0.0f)) return fail(FP8DSA_ERR_INVALID_ARG, "fp8_max and pow2_margin must be > 0");
    int rc = check_device();
    if (rc) return rc;
    AmaxJob j;
    j.x = x;
    j.in_type = in_type;
    j.numel = numel;
    j.fp8_max = fp8_max;
    j.pow2_margin = pow2_margin;
    j.scale_out = scale_out;
    j.amax_out = amax_out;
    return launch_amax_jobs(&j, 1, scratch, stream);
}

static int quantize_common(const void* x, fp8_in_t in_type, int64_t rows, int64_t cols, const float* scale,
                           fp8_fmt_t fmt, uint8_t* out, uint8_t* out_t, float* amax_out,
                           const fp8_ring_t* ring, cudaStream_t stream) {
    if (!valid_in_type(in_type)) return fail(FP8DSA_ERR_INVALID_ARG, "bad in_type");
    if (!valid_fmt(fmt)) return fail(FP8DSA_ERR_INVALID_ARG, "fmt must be FP8_E4M3 or FP8_E5M2");
    if (rows < 0 || cols < 0) return fail(FP8DSA_ERR_INVALID_ARG, "rows and cols must be >= 0");
    if (rows > 0 && cols > 0 && (x == nullptr)) return fail(FP8DSA_ERR_INVALID_ARG, "x is NULL");
    if (scale == nullptr) return fail(FP8DSA_ERR_INVALID_ARG, "scale is NULL");
    const bool empty = rows == 0 || cols == 0;
    if (!empty && out == nullptr && out_t == nullptr) return fail(FP8DSA_ERR_INVALID_ARG, "output is NULL");
    if (out_t != nullptr && (cols + kTile - 1) / kTile > kMaxTiles)
        return fail(FP8DSA_ERR_UNSUPPORTED, "too many columns");
    if (out_t != nullptr && ((rows + kTile - 1) / kTile) * ((cols + kTile - 1) / kTile) > kMaxTiles)
        return fail(FP8DSA_ERR_UNSUPPORTED, "too many 128 x 128 tiles");
    int rc = check_ring(ring);
    if (rc) return rc;
    rc = check_device();
    if (rc) return rc;
    QuantJob j;
    j.x = x;
    j.in_type = in_type;
    j.rows = rows;
    j.cols = cols;
    j.scale = scale;
    j.fmt = fmt;
    j.out = out;
    j.out_t = out_t;
    j.amax_out = amax_out;
    j.ring = ring;
    return launch_quantize(j, stream);
}

int fp8_quantize(const void* x, fp8_in_t in_type, int64_t rows, int64_t cols, const float* scale,
                 fp8_fmt_t fmt, int transposed, uint8_t* out, float* amax_out, const fp8_ring_t* ring,
                 cudaStream_t stream) {
    clear_error();
    if (out == nullptr && rows > 0 && cols > 0) return fail(FP8DSA_ERR_INVALID_ARG, "out is NULL");
    return quantize_common(x, in_type, rows, cols, scale, fmt, transposed ? nullptr : out,
                           transposed ? out : nullptr, amax_out, ring, stream);
}

int fp8_set_tiled_persist_threshold(int64_t min_tiles) {
    clear_error();
    if (min_tiles < 0) return fail(FP8DSA_ERR_INVALID_ARG, "min_tiles must be >= 0");
    g_persist_min_tiles.store(min_tiles);
    return FP8DSA_OK;
}

static int ring_list_call(const fp8_ring_t* rings, int n, float* collect_out, const float* fold_amax, bool fold,
                          cudaStream_t stream) {
    if (n < 0) return fail(FP8DSA_ERR_INVALID_ARG, "n must be >= 0");
    if (n > 0 && rings == nullptr) return fail(FP8DSA_ERR_INVALID_ARG, "rings is NULL");
    for (int i = 0; i < n; ++i) {
        int rc = check_ring(&rings[i]);
        if (rc) return fail(rc, "ring " + std::to_string(i) + ": " + fp8_last_error());
    }
    if (n == 0) return FP8DSA_OK;
    int rc = check_device();
    if (rc) return rc;
    for (int base = 0; base < n; base += kRingChunk) {
        RingList L{};
        L.n = std::min(kRingChunk, n - base);
        for (int i = 0; i < L.n; ++i) L.ring[i] = rings[base + i];
        launch_begin(kKindOther, stream);
        if (fold)
            launch_ex(ring_fold_list_kernel, dim3(1), dim3(kRingChunk), 0, stream, 1, L,
                      fold_amax != nullptr ? fold_amax + base : nullptr);
        else
            launch_ex(ring_collect_kernel, dim3(1), dim3(kRingChunk), 0, stream, 1, L, collect_out + base);
        launch_end(kKindOther, stream, 0.0);
        rc = check_launch(fold ? "ring fold kernel" : "ring collect kernel");
        if (rc) return rc;
    }
    return FP8DSA_OK;
}

int fp8_scale_ring_collect_amax(const fp8_ring_t* rings, int n, float* amax_out, cudaStream_t stream) {
    clear_error();
    if (n > 0 && amax_out == nullptr) return fail(FP8DSA_ERR_INVALID_ARG, "amax_out is NULL");
    return ring_list_call(rings, n, amax_out, nullptr, false, stream);
}

int fp8_scale_ring_fold(const fp8_ring_t* rings, int n, const float* amax, cudaStream_t stream) {
    clear_error();
    return ring_list_call(rings, n, nullptr, amax, true, stream);
}

int fp8_quantize_dual(const void* x, fp8_in_t in_type, int64_t rows, int64_t cols, const float* scale,
                      fp8_fmt_t fmt, uint8_t* out, uint8_t* out_t, float* amax_out, const fp8_ring_t* ring,
                      cudaStream_t stream) {
    clear_error();
    if ((out == nullptr || out_t == nullptr) && rows > 0 && cols > 0)
        return fail(FP8DSA_ERR_INVALID_ARG, "out and out_t are required");
    return quantize_common(x, in_type, rows, cols, scale, fmt, out, out_t, amax_out, ring, stream);
}

}  // extern "C"
