// Host-side internals shared by the library's translation units: error reporting, the
// per-device status word, launch bookkeeping (timeout, optional per-kernel timing) and
// small argument-check helpers.  Nothing here is part of the C ABI.
#pragma once

#include <cuda_runtime.h>
#include <cstddef>
#include <cstdint>
#include <string>

#include "fp8dsa.h"
#include "device.cuh"

namespace fp8dsa {

// Record a message for fp8_last_error() and return `code`.
int fail(int code, const std::string& msg);
// Clear the thread-local error message.
void clear_error();

// Check the current device is compute capability 10.x (cached per device).
int check_device();
// Number of SMs of the current device (cached per device).
int sm_count();
// The current CUDA device, clamped to the library's per-device tables (0 .. kMaxDevices - 1):
// one-time kernel set-up (shared-memory attributes, occupancy) is cached per device.
constexpr int kMaxDevices = 64;
int current_device();

// WaitCtl for the current device (status word address + timeout).
int wait_ctl(WaitCtl* ctl);

// Kernel classes for the optional per-kernel timing.  GEMM launches are recorded under the
// instance they ran (256-wide tiles on CTA pairs, or single-CTA tiles); reading kKindGemm
// returns both.
enum KernelKind : int { kKindQuantize = 0, kKindGemm = 1, kKindOther = 2, kKindGemmPair = 3, kKindGemmSingle = 4 };
constexpr int kNumKinds = 5;

// Bracket a launch with timing events when profiling is on.  `work` is the algorithmic
// bytes (quantize, other) or flops (GEMM) the launch performs.
void launch_begin(int kind, cudaStream_t stream);
void launch_end(int kind, cudaStream_t stream, double work);

// Encode a 3-D tiled tensor map (TMA descriptor): dims {inner, outer, batch} elements, row
// stride `ld` bytes, batch stride `bstride` bytes, box {box_inner, box_outer, 1}, the given
// shared-memory swizzle, zero fill out of bounds.  The driver entry point is looked up once.
int encode_tensor_map(CUtensorMap* map, CUtensorMapDataType dtype, const void* base, int64_t inner,
                      int64_t outer, int64_t batch, int64_t ld, int64_t bstride, int box_inner, int box_outer,
                      CUtensorMapSwizzle swizzle);

// After a launch: map a launch failure to FP8DSA_ERR_CUDA.
int check_launch(const char* what);

// Whether the linear entries fold their rings within the call (default) or leave the measured
// amax in each ring's amax slot for fp8_scale_ring_fold (data-parallel training).
bool ring_fold_in_call();

// Whether library kernels are launched with programmatic dependent launch (default on).
bool pdl_enabled();

// Launch `kernel` with optional 1-D cluster size and, when enabled, programmatic stream
// serialization (the kernel overlaps its launch and prologue with the previous kernel's tail;
// every library kernel waits in pdl_wait before touching data an earlier kernel wrote).
template <typename... KArgs, typename... Args>
cudaError_t launch_ex(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t stream,
                      int cluster_x, Args... args) {
    cudaLaunchConfig_t cfg = {};
    cudaLaunchAttribute at[2];
    int na = 0;
    if (cluster_x > 1) {
        at[na].id = cudaLaunchAttributeClusterDimension;
        at[na].val.clusterDim.x = static_cast<unsigned>(cluster_x);
        at[na].val.clusterDim.y = 1;
        at[na].val.clusterDim.z = 1;
        ++na;
    }
    if (pdl_enabled()) {
        at[na].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        at[na].val.programmaticStreamSerializationAllowed = 1;
        ++na;
    }
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cfg.attrs = at;
    cfg.numAttrs = na;
    return cudaLaunchKernelEx(&cfg, kernel, static_cast<KArgs>(args)...);
}

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

inline size_t align_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

inline int in_type_bytes(fp8_in_t t) { return t == FP8_IN_F32 ? 4 : 2; }

inline bool valid_in_type(int t) { return t == FP8_IN_BF16 || t == FP8_IN_F16 || t == FP8_IN_F32; }
inline bool valid_fmt(int f) { return f == FP8_E4M3 || f == FP8_E5M2; }
inline float fmt_max(fp8_fmt_t f) { return f == FP8_E5M2 ? 57344.0f : 448.0f; }

// ---------------------------------------------------------------------------------------
// Internal launchers (each enqueues exactly the kernels named; arguments already checked).
// ---------------------------------------------------------------------------------------

// Amax of up to three tensors in one launch; for tensor t, its last block writes
// scale_out[t] = max(RN32(amax / fp8_max) / pow2_margin, 1e-12) (if non-null),
// amax_out[t] (if non-null), or folds into ring seed slots (if ring[t].state non-null,
// hist[idx] = amax, scale = formula over the window).  scratch: 16 bytes per tensor,
// zero on entry and left zero.
struct AmaxJob {
    const void* x = nullptr;
    fp8_in_t in_type = FP8_IN_BF16;
    int64_t numel = 0;
    float fp8_max = 448.0f;
    float pow2_margin = 1.0f;
    float* scale_out = nullptr;
    float* amax_out = nullptr;
    fp8_ring_t ring{};  // ring.state == nullptr: no seeding
};
int launch_amax_jobs(const AmaxJob* jobs, int njobs, uint32_t* scratch, cudaStream_t stream);

// Quantize launch description (row-major, transposed or dual).
struct QuantJob {
    const void* x = nullptr;
    fp8_in_t in_type = FP8_IN_BF16;
    int64_t rows = 0, cols = 0;
    const float* scale = nullptr;
    fp8_fmt_t fmt = FP8_E4M3;
    int fmt_t = -1;             // format of out_t (-1: fmt); the same product, a second rounding
    uint8_t* out = nullptr;     // [rows][cols] or nullptr
    uint8_t* out_t = nullptr;   // [cols][rows] or nullptr
    uint8_t* out2 = nullptr;    // [rows][cols] in fmt_t (row-major launches only) or nullptr
    float* amax_out = nullptr;  // final amax (may be nullptr)
    const fp8_ring_t* ring = nullptr;
    float* scale_used_out = nullptr;  // the step used, written once (may be nullptr)
    float* colsum_partial = nullptr;  // [ceil(rows/128)][cols] fp32 column sums (tiled only)
    bool defer_fold = false;          // ring: only leave the amax; a later kernel folds the ring
};
int launch_quantize(const QuantJob& job, cudaStream_t stream);
// Up to three tensors in one launch (same formats, input type and orientation); each tensor
// keeps its own amax, ticket and ring fold.
// `zero` / `zero_words` (optional): words the launch also sets to zero (split-K counters of
// the GEMM that follows).
int launch_quantize_batch(const QuantJob* jobs, int njobs, cudaStream_t stream, uint32_t* zero = nullptr,
                          int64_t zero_words = 0);

// grad_b[c] = RN_bf16(sum_t partial[t][c]) in a fixed order.
int launch_colsum_finalize(const float* partial, int64_t tiles, int64_t cols, void* out_bf16,
                           cudaStream_t stream);

// Per-tile column sums of fp8 bytes [rows][cols] (format fmt) times *step, in the layout the
// dual quantize writes ([ceil(rows/128)][cols] fp32), for a bias gradient of a pre-quantized
// g; `zero` / `zero_words` (optional) are also set to zero.  cols % 4 == 0.
int launch_colsum_fp8(const uint8_t* g8, fp8_fmt_t fmt, int64_t rows, int64_t cols, const float* step,
                      float* partial, uint32_t* zero, int64_t zero_words, cudaStream_t stream);

// One GEMM of a launch, arguments already validated.
struct GemmDesc {
    const uint8_t* a;
    const uint8_t* b;
    int fmt_a, fmt_b, a_mn, b_mn;
    int64_t m, n, k, lda, ldb, ldo, batch, stride_a, stride_b, stride_o;
    const float* scale_a;
    const float* scale_b;
    const void* bias;
    int bias_kind;
    const float* bias_scale;
    void* out;  // bf16 output, or null when only out8 is wanted
    // optional fp8 output of the same values: out8 = q(RN32(RN_bf16(v) * RN32(1 / *out8_step))),
    // same element strides as out; |RN_bf16(v)| atomically maxed into *out8_amax (if not null);
    // *out8_step written to *out8_step_used (if not null)
    uint8_t* out8 = nullptr;
    int out8_fmt = 0;
    const float* out8_step = nullptr;
    float* out8_amax = nullptr;
    float* out8_step_used = nullptr;
};

// Split-K scratch a GEMM launch may use (see gemm_launch_group): fp32 partial tiles and one
// arrival counter per (tile, CTA of a pair), which must be zero when the GEMM starts (the
// quantize launch that precedes it in the linear compositions zeroes them).
struct SplitWorkspace {
    float* partial = nullptr;
    size_t partial_bytes = 0;
    uint32_t* counters = nullptr;
    int64_t counter_words = 0;
};
// Scratch that lets a GEMM group split any of its problems' K into up to 4 ranges: partial
// bytes and counter words for problems of the given output shapes.
size_t splitk_partial_bytes(const int64_t* m, const int64_t* n, int nprob);
int64_t splitk_counter_words(const int64_t* m, const int64_t* n, int nprob);

// One or two GEMMs in one persistent launch over the union of their tiles; if colsum_tiles > 0
// the epilogue warps first write colsum_out[c] = RN_bf16(sum_t colsum_partial[t][c]).  With
// `split` (may be null) the launch may cut tiles' K ranges across CTAs where that shortens
// the schedule; the result differs from the unsplit one only in fp32 summation order.
// `folds` (up to 3, may be empty): rings whose quantize launch deferred its fold; the GEMM
// launch folds them (one thread, after its dependency wait), or a one-thread kernel does
// when no GEMM kernel runs.
int gemm_launch_group(const GemmDesc* descs, int ndesc, const float* colsum_partial, int64_t colsum_tiles,
                      int64_t colsum_cols, void* colsum_out, const SplitWorkspace* split, const fp8_ring_t* folds,
                      int nfolds, cudaStream_t stream);

// Split-K mode of later GEMM launches (0 automatic, 1 never, 2..4 forced); rejects others.
int gemm_set_split_mode(int mode);

// Workspace bytes of linear_forward_fp8 without the optional split-K region.
size_t linear_forward_base_workspace(int64_t m, int64_t k, int64_t n);

// linear_forward_fp8 with choices: x8_keep / w8_keep (may be null) receive the quantized
// operands instead of the workspace; x8t_keep / w8t_keep (both or neither; delayed scaling,
// bf16 w) also receive x^T and w^T in format fmt_t from the same products, or, with
// copies_row_major, x and w in format fmt_t row-major; allow_split = false needs only the
// base workspace and runs the GEMM without split-K.
int linear_forward_impl(const void* x, const void* w, int w_is_fp8, const float* w_step, const void* bias,
                        const float* bias_scale, int64_t m, int64_t k, int64_t n, fp8_fmt_t fmt,
                        const fp8_ring_t* x_ring, const fp8_ring_t* w_ring, float pow2_margin, float* sx_used,
                        float* sw_used, uint8_t* x8_keep, uint8_t* w8_keep, uint8_t* x8t_keep, uint8_t* w8t_keep,
                        fp8_fmt_t fmt_t, void* workspace, size_t workspace_bytes, bool allow_split, void* y,
                        cudaStream_t stream, bool copies_row_major = false);

// The GEMM entry with arguments already validated (used by the linear compositions).
int gemm_launch(const uint8_t* a, const uint8_t* b, int fmt_a, int fmt_b, int a_mn_major,
                int b_mn_major, int64_t m, int64_t n, int64_t k, int64_t lda, int64_t ldb,
                int64_t ldo, int64_t batch, int64_t stride_a, int64_t stride_b, int64_t stride_o,
                const float* scale_a, const float* scale_b, const void* bias, int bias_kind,
                const float* bias_scale, void* out, cudaStream_t stream);

}  // namespace fp8dsa
