// FP8 linear layer forward / backward, composed from the quantize and GEMM kernels.
//
// Definition: AstrAI compare view 3e57cc8...main, astrai/extension/fp8.py --
// fp8_linear_forward (delayed: snapshot the ring steps, quantize x and w folding their rings,
// NT GEMM with sx*sw and the fused bias; dynamic: measure the current amax first) and
// _LinearFp8.backward (g quantized once in both orientations folding the g ring; x and w
// re-quantized transposed with the forward's steps and no ring; grad_x = g8 . w8T^T and
// grad_w = g8T . x8T^T, both NT; grad_b = column sum of g).
//
// linear_forward_fp8_save_t / linear_backward_fp8_saved_t split the same work differently:
// the forward's quantize launch also writes x^T and w^T in the backward's format from the
// products it already forms (the backward's delayed-scaling rule quantizes them with the
// forward's steps), so the backward quantizes only g and x and w are read once per step.
//
// Launches per call (delayed scaling):
//   forward : one quantize launch for x and w + GEMM                                    = 2
//   backward: one quantize launch for g (both orientations, per-tile column sums), x^T
//             and w^T + one GEMM launch for dX and dW whose epilogue warps also reduce
//             the column sums into grad_b                                             = 2
// The quantize launch reads each ring's step, writes the snapshot (the step used) from its
// first block and leaves the measured amax in the ring's amax slot; the GEMM launch that
// follows folds the rings (one epilogue thread, after its dependency wait), so the quantize
// launch ends without a last-block tail.  The GEMM dequantizes with exactly the step the
// bytes were quantized with.
#include <cuda_runtime.h>

#include <string>

#include "internal.h"

namespace fp8dsa {
namespace {

constexpr size_t kAlign = 256;
constexpr size_t kScratchBytes = 128;  // 3 x 16 B amax scratch + 4 internal fp32 steps

// Each layout ends with the optional split-K region (the GEMM's arrival counters, then its
// fp32 partial tiles); `base` is the size without it.
struct FwdLayout {
    size_t x8, w8, scratch, base, counters, partial, total;
    int64_t counter_words;
};

FwdLayout fwd_layout(int64_t m, int64_t k, int64_t n) {
    FwdLayout L;
    size_t off = 0;
    L.x8 = off;
    off = align_up(off + static_cast<size_t>(m) * k, kAlign);
    L.w8 = off;
    off = align_up(off + static_cast<size_t>(n) * k, kAlign);
    L.scratch = off;
    off = align_up(off + kScratchBytes, kAlign);
    L.base = off;
    const int64_t om[1] = {m}, on[1] = {n};  // y [m][n]
    L.counter_words = splitk_counter_words(om, on, 1);
    L.counters = off;
    off = align_up(off + sizeof(uint32_t) * static_cast<size_t>(L.counter_words), kAlign);
    L.partial = off;
    off = align_up(off + splitk_partial_bytes(om, on, 1), kAlign);
    L.total = off;
    return L;
}

struct BwdLayout {
    size_t g8, g8t, x8t, w8t, colsum, scratch, base, counters, partial, total;
    int64_t counter_words;
};

BwdLayout bwd_layout(int64_t m, int64_t k, int64_t n) {
    BwdLayout L;
    size_t off = 0;
    const size_t mn = static_cast<size_t>(m) * n;
    L.g8 = off;
    off = align_up(off + mn, kAlign);
    L.g8t = off;
    off = align_up(off + mn, kAlign);
    L.x8t = off;
    off = align_up(off + static_cast<size_t>(k) * m, kAlign);
    L.w8t = off;
    off = align_up(off + static_cast<size_t>(k) * n, kAlign);
    L.colsum = off;
    off = align_up(off + sizeof(float) * static_cast<size_t>((m + 127) / 128) * n, kAlign);
    L.scratch = off;
    off = align_up(off + kScratchBytes, kAlign);
    L.base = off;
    const int64_t om[2] = {m, n}, on[2] = {k, k};  // grad_x [m][k], grad_w [n][k]
    L.counter_words = splitk_counter_words(om, on, 2);
    L.counters = off;
    off = align_up(off + sizeof(uint32_t) * static_cast<size_t>(L.counter_words), kAlign);
    L.partial = off;
    off = align_up(off + splitk_partial_bytes(om, on, 2), kAlign);
    L.total = off;
    return L;
}

struct MixLayout {
    size_t g8, colsum, scratch, base, counters, partial, total;
    int64_t counter_words;
};

MixLayout mix_layout(int64_t m, int64_t k, int64_t n) {
    MixLayout L;
    size_t off = 0;
    L.g8 = off;
    off = align_up(off + static_cast<size_t>(m) * n, kAlign);
    L.colsum = off;
    off = align_up(off + sizeof(float) * static_cast<size_t>((m + 127) / 128) * n, kAlign);
    L.scratch = off;
    off = align_up(off + kScratchBytes, kAlign);
    L.base = off;
    const int64_t om[2] = {m, n}, on[2] = {k, k};  // grad_x [m][k], grad_w [n][k]
    L.counter_words = splitk_counter_words(om, on, 2);
    L.counters = off;
    off = align_up(off + sizeof(uint32_t) * static_cast<size_t>(L.counter_words), kAlign);
    L.partial = off;
    off = align_up(off + splitk_partial_bytes(om, on, 2), kAlign);
    L.total = off;
    return L;
}

// Backward from transposed copies the forward saved: only g's bytes, its column sums and the
// scratch, then the split-K region.
struct SavedLayout {
    size_t g8, g8t, colsum, scratch, base, counters, partial, total;
    int64_t counter_words;
};

SavedLayout saved_layout(int64_t m, int64_t k, int64_t n) {
    SavedLayout L;
    size_t off = 0;
    const size_t mn = static_cast<size_t>(m) * n;
    L.g8 = off;
    off = align_up(off + mn, kAlign);
    L.g8t = off;
    off = align_up(off + mn, kAlign);
    L.colsum = off;
    off = align_up(off + sizeof(float) * static_cast<size_t>((m + 127) / 128) * n, kAlign);
    L.scratch = off;
    off = align_up(off + kScratchBytes, kAlign);
    L.base = off;
    const int64_t om[2] = {m, n}, on[2] = {k, k};  // grad_x [m][k], grad_w [n][k]
    L.counter_words = splitk_counter_words(om, on, 2);
    L.counters = off;
    off = align_up(off + sizeof(uint32_t) * static_cast<size_t>(L.counter_words), kAlign);
    L.partial = off;
    off = align_up(off + splitk_partial_bytes(om, on, 2), kAlign);
    L.total = off;
    return L;
}

// A tensor's pointer is required only when the tensor has elements (an empty batch may come
// with null pointers, as empty framework tensors do).
inline bool missing(const void* p, int64_t elems) { return p == nullptr && elems > 0; }

int check_ring_arg(const fp8_ring_t* r, const char* name) {
    if (r == nullptr) return FP8DSA_OK;
    if (r->state == nullptr || r->hist_len < 1 || r->hist_idx < 0 || r->hist_idx >= r->hist_len ||
        !(r->fp8_max > 0.0f) || !(r->pow2_margin > 0.0f))
        return fail(FP8DSA_ERR_INVALID_ARG, std::string(name) + ": invalid ring (state, hist_len, hist_idx, fp8_max, pow2_margin)");
    if (!aligned16(r->state)) return fail(FP8DSA_ERR_UNSUPPORTED, std::string(name) + ": ring state must be 16-byte aligned");
    return FP8DSA_OK;
}

}  // namespace
}  // namespace fp8dsa

using namespace fp8dsa;

extern "C" {

size_t linear_forward_fp8_workspace_size(int64_t m, int64_t k, int64_t n) {
    if (m < 0 || k < 0 || n < 0) return 0;
    return fwd_layout(m, k, n).total;
}

int linear_forward_fp8(const void* x, const void* w, int w_is_fp8, const float* w_step, const void* bias,
                       const float* bias_scale, int64_t m, int64_t k, int64_t n, fp8_fmt_t fmt,
                       const fp8_ring_t* x_ring, const fp8_ring_t* w_ring, float pow2_margin, float* sx_used,
                       float* sw_used, void* workspace, size_t workspace_bytes, void* y, cudaStream_t stream) {
    return linear_forward_impl(x, w, w_is_fp8, w_step, bias, bias_scale, m, k, n, fmt, x_ring, w_ring, pow2_margin,
                               sx_used, sw_used, nullptr, nullptr, nullptr, nullptr, fmt, workspace, workspace_bytes,
                               true, y, stream);
}

int linear_forward_fp8_keep(const void* x, const void* w, int w_is_fp8, const float* w_step, const void* bias,
                            const float* bias_scale, int64_t m, int64_t k, int64_t n, fp8_fmt_t fmt,
                            const fp8_ring_t* x_ring, const fp8_ring_t* w_ring, float pow2_margin, float* sx_used,
                            float* sw_used, uint8_t* x8_out, uint8_t* w8_out, void* workspace,
                            size_t workspace_bytes, void* y, cudaStream_t stream) {
    clear_error();
    if ((x8_out == nullptr && m > 0 && k > 0) || (!w_is_fp8 && w8_out == nullptr && n > 0 && k > 0))
        return fail(FP8DSA_ERR_INVALID_ARG, "x8_out (and w8_out unless w_is_fp8) are required");
    return linear_forward_impl(x, w, w_is_fp8, w_step, bias, bias_scale, m, k, n, fmt, x_ring, w_ring, pow2_margin,
                               sx_used, sw_used, x8_out, w8_out, nullptr, nullptr, fmt, workspace, workspace_bytes,
                               true, y, stream);
}

int linear_forward_fp8_save_t(const void* x, const void* w, const void* bias, const float* bias_scale, int64_t m,
                              int64_t k, int64_t n, fp8_fmt_t fmt, fp8_fmt_t fmt_t, const fp8_ring_t* x_ring,
                              const fp8_ring_t* w_ring, float* sx_used, float* sw_used, uint8_t* x8t_out,
                              uint8_t* w8t_out, void* workspace, size_t workspace_bytes, void* y, cudaStream_t stream) {
    clear_error();
    if (missing(x8t_out, m * k) || missing(w8t_out, n * k))
        return fail(FP8DSA_ERR_INVALID_ARG, "x8t_out and w8t_out are required");
    return linear_forward_impl(x, w, 0, nullptr, bias, bias_scale, m, k, n, fmt, x_ring, w_ring, 1.0f, sx_used,
                               sw_used, nullptr, nullptr, x8t_out, w8t_out, fmt_t, workspace, workspace_bytes, true, y,
                               stream);
}

int linear_forward_fp8_save_rm(const void* x, const void* w, const void* bias, const float* bias_scale, int64_t m,
                               int64_t k, int64_t n, fp8_fmt_t fmt, fp8_fmt_t fmt_b, const fp8_ring_t* x_ring,
                               const fp8_ring_t* w_ring, float* sx_used, float* sw_used, uint8_t* x8b_out,
                               uint8_t* w8b_out, void* workspace, size_t workspace_bytes, void* y,
                               cudaStream_t stream) {
    clear_error();
    if (missing(x8b_out, m * k) || missing(w8b_out, n * k))
        return fail(FP8DSA_ERR_INVALID_ARG, "x8b_out and w8b_out are required");
    return linear_forward_impl(x, w, 0, nullptr, bias, bias_scale, m, k, n, fmt, x_ring, w_ring, 1.0f, sx_used,
                               sw_used, nullptr, nullptr, x8b_out, w8b_out, fmt_b, workspace, workspace_bytes, true, y,
                               stream, true);
}

size_t linear_backward_fp8_workspace_size(int64_t m, int64_t k, int64_t n) {
    if (m < 0 || k < 0 || n < 0) return 0;
    return bwd_layout(m, k, n).total;
}

}  // extern "C"

namespace fp8dsa {

size_t linear_forward_base_workspace(int64_t m, int64_t k, int64_t n) {
    if (m < 0 || k < 0 || n < 0) return 0;
    return fwd_layout(m, k, n).base;
}

int linear_forward_impl(const void* x, const void* w, int w_is_fp8, const float* w_step, const void* bias,
                        const float* bias_scale, int64_t m, int64_t k, int64_t n, fp8_fmt_t fmt,
                        const fp8_ring_t* x_ring, const fp8_ring_t* w_ring, float pow2_margin, float* sx_used,
                        float* sw_used, uint8_t* x8_keep, uint8_t* w8_keep, uint8_t* x8t_keep, uint8_t* w8t_keep,
                        fp8_fmt_t fmt_t, void* workspace, size_t workspace_bytes, bool allow_split, void* y,
                        cudaStream_t stream, bool copies_row_major) {
    clear_error();
    if (!valid_fmt(fmt)) return fail(FP8DSA_ERR_INVALID_ARG, "fmt must be FP8_E4M3 or FP8_E5M2");
    if (m < 0 || k < 0 || n < 0) return fail(FP8DSA_ERR_INVALID_ARG, "negative size");
    if (missing(x, m * k) || missing(w, n * k) || missing(y, m * n) || workspace == nullptr)
        return fail(FP8DSA_ERR_INVALID_ARG, "x, w, y and workspace are required");
    if (k % 16 != 0 || n % 16 != 0) return fail(FP8DSA_ERR_UNSUPPORTED, "k and n must be multiples of 16");
    if (w_is_fp8 && w_step == nullptr) return fail(FP8DSA_ERR_INVALID_ARG, "w_is_fp8 needs w_step");
    if (bias == nullptr && bias_scale != nullptr) return fail(FP8DSA_ERR_INVALID_ARG, "bias_scale without bias");
    const bool dynamic = x_ring == nullptr;
    if (dynamic && w_ring != nullptr) return fail(FP8DSA_ERR_INVALID_ARG, "w_ring given without x_ring");
    if (!dynamic && !w_is_fp8 && w_ring == nullptr) return fail(FP8DSA_ERR_INVALID_ARG, "delayed scaling needs w_ring");
    if (dynamic && !(pow2_margin > 0.0f)) return fail(FP8DSA_ERR_INVALID_ARG, "pow2_margin must be > 0");
    int rc = check_ring_arg(x_ring, "x_ring");
    if (rc) return rc;
    rc = check_ring_arg(w_is_fp8 ? nullptr : w_ring, "w_ring");
    if (rc) return rc;
    if ((reinterpret_cast<uintptr_t>(workspace) & (kAlign - 1)) != 0)
        return fail(FP8DSA_ERR_UNSUPPORTED, "workspace must be 256-byte aligned");
    const FwdLayout L = fwd_layout(m, k, n);
    const size_t need = allow_split ? L.total : L.base;
    if (workspace_bytes < need)
        return fail(FP8DSA_ERR_WORKSPACE, "workspace too small: need " + std::to_string(need) + " bytes");
    if (w_is_fp8 && !aligned16(w)) return fail(FP8DSA_ERR_UNSUPPORTED, "fp8 w must be 16-byte aligned");
    if ((x8_keep != nullptr && !aligned16(x8_keep)) || (!w_is_fp8 && w8_keep != nullptr && !aligned16(w8_keep)))
        return fail(FP8DSA_ERR_UNSUPPORTED, "x8_out / w8_out must be 16-byte aligned");
    // the backward's copies are asked for by either output (one of them is null when its tensor
    // is empty)
    const bool save_t = x8t_keep != nullptr || w8t_keep != nullptr;
    if (save_t) {
        if (!valid_fmt(fmt_t)) return fail(FP8DSA_ERR_INVALID_ARG, "fmt_t must be FP8_E4M3 or FP8_E5M2");
        if (dynamic || w_is_fp8 || missing(x8t_keep, m * k) || missing(w8t_keep, n * k))
            return fail(FP8DSA_ERR_INVALID_ARG, "transposed copies need x_ring, w_ring, a bf16 w and both outputs");
        if (!aligned16(x8t_keep) || !aligned16(w8t_keep))
            return fail(FP8DSA_ERR_UNSUPPORTED, "x8t_out / w8t_out must be 16-byte aligned");
        if (!copies_row_major && m % 16 != 0) return fail(FP8DSA_ERR_UNSUPPORTED, "m must be a multiple of 16 for x8t_out");
    }
    rc = check_device();
    if (rc) return rc;

    uint8_t* ws = static_cast<uint8_t*>(workspace);
    uint8_t* x8 = x8_keep != nullptr ? x8_keep : ws + L.x8;
    uint8_t* w8 = w_is_fp8 ? static_cast<uint8_t*>(const_cast<void*>(w)) : (w8_keep != nullptr ? w8_keep : ws + L.w8);
    uint32_t* scratch = reinterpret_cast<uint32_t*>(ws + L.scratch);
    float* internal = reinterpret_cast<float*>(ws + L.scratch + 64);
    float* sx = sx_used ? sx_used : internal;
    float* sw = sw_used ? sw_used : internal + 1;

    if (w_is_fp8) {
        cudaError_t e = cudaMemcpyAsync(sw, w_step, sizeof(float), cudaMemcpyDeviceToDevice, stream);
        if (e != cudaSuccess) return fail(FP8DSA_ERR_CUDA, std::string("copy w_step: ") + cudaGetErrorString(e));
    }
    if (dynamic) {
        cudaError_t e = cudaMemsetAsync(scratch, 0, 64, stream);
        if (e != cudaSuccess) return fail(FP8DSA_ERR_CUDA, std::string("memset scratch: ") + cudaGetErrorString(e));
        AmaxJob jobs[2];
        int nj = 0;
        jobs[nj].x = x;
        jobs[nj].numel = m * k;
        jobs[nj].fp8_max = fmt_max(fmt);
        jobs[nj].pow2_margin = pow2_margin;
        jobs[nj].scale_out = sx;
        ++nj;
        if (!w_is_fp8) {
            jobs[nj].x = w;
            jobs[nj].numel = n * k;
            jobs[nj].fp8_max = fmt_max(fmt);
            jobs[nj].pow2_margin = pow2_margin;
            jobs[nj].scale_out = sw;
            ++nj;
        }
        rc = launch_amax_jobs(jobs, nj, scratch, stream);
        if (rc) return rc;
    }
    QuantJob qx;
    qx.x = x;
    qx.rows = m;
    qx.cols = k;
    qx.fmt = fmt;
    qx.out = x8;
    if (save_t) {  // the backward's copy of x from the same products, in its own format
        // an empty x writes no bytes; a placeholder keeps its job in the launch's orientation
        (copies_row_major ? qx.out2 : qx.out_t) = x8t_keep != nullptr ? x8t_keep : ws;
        qx.fmt_t = fmt_t;
    }
    if (dynamic) {
        qx.scale = sx;
    } else {
        qx.scale = x_ring->state + x_ring->hist_len;
        qx.ring = x_ring;
        qx.scale_used_out = sx;
        qx.defer_fold = true;  // folded by the GEMM launch below
    }
    QuantJob fwd_jobs[2];
    int nfj = 0;
    fwd_jobs[nfj++] = qx;
    if (!w_is_fp8) {
        QuantJob qw;
        qw.x = w;
        qw.rows = n;
        qw.cols = k;
        qw.fmt = fmt;
        qw.out = w8;
        if (save_t) {
            (copies_row_major ? qw.out2 : qw.out_t) = w8t_keep != nullptr ? w8t_keep : ws;
            qw.fmt_t = fmt_t;
        }
        if (dynamic) {
            qw.scale = sw;
        } else {
            qw.scale = w_ring->state + w_ring->hist_len;
            qw.ring = w_ring;
            qw.scale_used_out = sw;
            qw.defer_fold = true;
        }
        fwd_jobs[nfj++] = qw;
    }
    SplitWorkspace split;
    if (allow_split) {
        split.counters = reinterpret_cast<uint32_t*>(ws + L.counters);
        split.counter_words = L.counter_words;
        split.partial = reinterpret_cast<float*>(ws + L.partial);
        split.partial_bytes = L.total - L.partial;
    }
    // x and w in one launch, each with its own amax, ticket and ring fold; it also zeroes the
    // GEMM's split-K counters
    rc = launch_quantize_batch(fwd_jobs, nfj, stream, split.counters, split.counter_words);
    if (rc) return rc;
    int bias_kind = 0;
    if (bias != nullptr) bias_kind = bias_scale == nullptr ? 1 : (fmt == FP8_E4M3 ? 2 : 3);
    const GemmDesc d{x8, w8, fmt, fmt, 0, 0, m, n, k, k, k, n, 1, 0, 0, 0, sx, sw, bias, bias_kind, bias_scale, y};
    fp8_ring_t folds[2];
    int nfolds = 0;
    if (!dynamic && ring_fold_in_call()) {
        folds[nfolds++] = *x_ring;
        if (!w_is_fp8) folds[nfolds++] = *w_ring;
    }
    return gemm_launch_group(&d, 1, nullptr, 0, 0, nullptr, allow_split ? &split : nullptr, folds, nfolds, stream);
}

}  // namespace fp8dsa

extern "C" {

int linear_backward_fp8(const void* g, const void* x, const void* w, int64_t m, int64_t k, int64_t n, fp8_fmt_t fmt,
                        int need_grad_x, int need_grad_w, int need_grad_b, const float* sx_fwd, const float* sw_fwd,
                        const fp8_ring_t* g_ring, float pow2_margin, float* sg_used, void* workspace,
                        size_t workspace_bytes, void* grad_x, void* grad_w, void* grad_b, cudaStream_t stream) {
    clear_error();
    if (!valid_fmt(fmt)) return fail(FP8DSA_ERR_INVALID_ARG, "fmt must be FP8_E4M3 or FP8_E5M2");
    if (m < 0 || k < 0 || n < 0) return fail(FP8DSA_ERR_INVALID_ARG, "negative size");
    if (missing(g, m * n) || workspace == nullptr) return fail(FP8DSA_ERR_INVALID_ARG, "g and workspace are required");
    if (need_grad_x && (missing(w, n * k) || missing(grad_x, m * k)))
        return fail(FP8DSA_ERR_INVALID_ARG, "grad_x needs w and grad_x");
    if (need_grad_w && (missing(x, m * k) || missing(grad_w, n * k)))
        return fail(FP8DSA_ERR_INVALID_ARG, "grad_w needs x and grad_w");
    if (need_grad_b && missing(grad_b, n)) return fail(FP8DSA_ERR_INVALID_ARG, "grad_b is NULL");
    if (k % 16 != 0 || n % 16 != 0) return fail(FP8DSA_ERR_UNSUPPORTED, "k and n must be multiples of 16");
    if (need_grad_w && m % 16 != 0) return fail(FP8DSA_ERR_UNSUPPORTED, "m must be a multiple of 16 for grad_w");
    const bool dynamic = g_ring == nullptr;
    if (!dynamic && ((need_grad_w && sx_fwd == nullptr) || (need_grad_x && sw_fwd == nullptr)))
        return fail(FP8DSA_ERR_INVALID_ARG, "delayed scaling needs the forward's sx_fwd / sw_fwd");
    if (dynamic && !(pow2_margin > 0.0f)) return fail(FP8DSA_ERR_INVALID_ARG, "pow2_margin must be > 0");
    int rc = check_ring_arg(g_ring, "g_ring");
    if (rc) return rc;
    if ((reinterpret_cast<uintptr_t>(workspace) & (kAlign - 1)) != 0)
        return fail(FP8DSA_ERR_UNSUPPORTED, "workspace must be 256-byte aligned");
    const BwdLayout L = bwd_layout(m, k, n);
    if (workspace_bytes < L.total)
        return fail(FP8DSA_ERR_WORKSPACE, "workspace too small: need " + std::to_string(L.total) + " bytes");
    rc = check_device();
    if (rc) return rc;

    uint8_t* ws = static_cast<uint8_t*>(workspace);
    uint8_t* g8 = ws + L.g8;
    uint8_t* g8t = ws + L.g8t;
    uint8_t* x8t = ws + L.x8t;
    uint8_t* w8t = ws + L.w8t;
    float* colsum = reinterpret_cast<float*>(ws + L.colsum);
    uint32_t* scratch = reinterpret_cast<uint32_t*>(ws + L.scratch);
    float* internal = reinterpret_cast<float*>(ws + L.scratch + 64);
    float* sg = sg_used ? sg_used : internal;
    const float* sx = sx_fwd;
    const float* sw = sw_fwd;

    if (dynamic) {
        cudaError_t e = cudaMemsetAsync(scratch, 0, 64, stream);
        if (e != cudaSuccess) return fail(FP8DSA_ERR_CUDA, std::string("memset scratch: ") + cudaGetErrorString(e));
        float* sx_dyn = internal + 1;
        float* sw_dyn = internal + 2;
        AmaxJob jobs[3];
        int nj = 0;
        jobs[nj].x = g;
        jobs[nj].numel = m * n;
        jobs[nj].fp8_max = fmt_max(fmt);
        jobs[nj].pow2_margin = pow2_margin;
        jobs[nj].scale_out = sg;
        ++nj;
        if (need_grad_w) {
            jobs[nj].x = x;
            jobs[nj].numel = m * k;
            jobs[nj].fp8_max = fmt_max(fmt);
            jobs[nj].pow2_margin = pow2_margin;
            jobs[nj].scale_out = sx_dyn;
            ++nj;
        }
        if (need_grad_x) {
            jobs[nj].x = w;
            jobs[nj].numel = n * k;
            jobs[nj].fp8_max = fmt_max(fmt);
            jobs[nj].pow2_margin = pow2_margin;
            jobs[nj].scale_out = sw_dyn;
            ++nj;
        }
        rc = launch_amax_jobs(jobs, nj, scratch, stream);
        if (rc) return rc;
        sx = sx_dyn;
        sw = sw_dyn;
    }

    // g: both orientations, ring fold, per-tile column sums for grad_b.
    QuantJob qg;
    qg.x = g;
    qg.rows = m;
    qg.cols = n;
    qg.fmt = fmt;
    qg.out = g8;
    qg.out_t = g8t;
    qg.colsum_partial = need_grad_b && m > 0 ? colsum : nullptr;  // no rows: grad_b is zero, no partials
    if (dynamic) {
        qg.scale = sg;
    } else {
        qg.scale = g_ring->state + g_ring->hist_len;
        qg.ring = g_ring;
        qg.scale_used_out = sg;
        qg.defer_fold = true;  // folded by the GEMM launch below
    }
    // g (both orientations), x^T and w^T in one launch
    QuantJob bwd_jobs[3];
    int nbj = 0;
    bwd_jobs[nbj++] = qg;
    if (need_grad_w) {
        QuantJob qx;
        qx.x = x;
        qx.rows = m;
        qx.cols = k;
        qx.fmt = fmt;
        qx.out_t = x8t;
        qx.scale = sx;
        bwd_jobs[nbj++] = qx;
    }
    if (need_grad_x) {
        QuantJob qw;
        qw.x = w;
        qw.rows = n;
        qw.cols = k;
        qw.fmt = fmt;
        qw.out_t = w8t;
        qw.scale = sw;
        bwd_jobs[nbj++] = qw;
    }
    SplitWorkspace split;
    split.counters = reinterpret_cast<uint32_t*>(ws + L.counters);
    split.counter_words = L.counter_words;
    split.partial = reinterpret_cast<float*>(ws + L.partial);
    split.partial_bytes = L.total - L.partial;
    rc = launch_quantize_batch(bwd_jobs, nbj, stream, split.counters, split.counter_words);
    if (rc) return rc;
    // dX and dW in one launch over both tile spaces; its epilogue warps also finish grad_b
    GemmDesc gd[2];
    int ng = 0;
    if (need_grad_x)  // grad_x [m][k] = g8 [m][n] . (w8t [k][n])^T
        gd[ng++] = GemmDesc{g8, w8t, fmt, fmt, 0, 0, m, k, n, n, n, k, 1, 0, 0, 0, sg, sw, nullptr, 0, nullptr, grad_x};
    if (need_grad_w)  // grad_w [n][k] = g8t [n][m] . (x8t [k][m])^T
        gd[ng++] = GemmDesc{g8t, x8t, fmt, fmt, 0, 0, n, k, m, m, m, k, 1, 0, 0, 0, sg, sx, nullptr, 0, nullptr, grad_w};
    const int64_t tiles = m > 0 ? (m + 127) / 128 : 0;
    rc = gemm_launch_group(gd, ng, need_grad_b ? colsum : nullptr, need_grad_b ? tiles : 0, need_grad_b ? n : 0,
                           need_grad_b ? grad_b : nullptr, &split, g_ring, (dynamic || !ring_fold_in_call()) ? 0 : 1, stream);
    if (rc) return rc;
    return FP8DSA_OK;
}

int linear_backward_fp8_prequant(const void* g, int g_is_fp8, const float* g_step, const void* x, int x_is_fp8,
                                 const void* w, int w_is_fp8, int64_t m, int64_t k, int64_t n, fp8_fmt_t fmt,
                                 int need_grad_x, int need_grad_w, int need_grad_b, const float* sx_fwd,
                                 const float* sw_fwd, const fp8_ring_t* g_ring, float pow2_margin, float* sg_used,
                                 void* workspace, size_t workspace_bytes, void* grad_x, void* grad_w, void* grad_b,
                                 cudaStream_t stream) {
    clear_error();
    if (!valid_fmt(fmt)) return fail(FP8DSA_ERR_INVALID_ARG, "fmt must be FP8_E4M3 or FP8_E5M2");
    if (m < 0 || k < 0 || n < 0) return fail(FP8DSA_ERR_INVALID_ARG, "negative size");
    if (missing(g, m * n) || workspace == nullptr) return fail(FP8DSA_ERR_INVALID_ARG, "g and workspace are required");
    if (need_grad_x && (missing(w, n * k) || missing(grad_x, m * k)))
        return fail(FP8DSA_ERR_INVALID_ARG, "grad_x needs w and grad_x");
    if (need_grad_w && (missing(x, m * k) || missing(grad_w, n * k)))
        return fail(FP8DSA_ERR_INVALID_ARG, "grad_w needs x and grad_w");
    if (need_grad_b && missing(grad_b, n)) return fail(FP8DSA_ERR_INVALID_ARG, "grad_b is NULL");
    if (k % 16 != 0 || n % 16 != 0) return fail(FP8DSA_ERR_UNSUPPORTED, "k and n must be multiples of 16");
    if (need_grad_w && m % 16 != 0) return fail(FP8DSA_ERR_UNSUPPORTED, "m must be a multiple of 16 for grad_w");
    if (g_is_fp8 && g_step == nullptr) return fail(FP8DSA_ERR_INVALID_ARG, "a pre-quantized g needs g_step");
    const bool dynamic = g_ring == nullptr;
    // the steps of x and w: the forward's (delayed, or any pre-quantized operand), else measured
    const bool want_sx = need_grad_w && (!dynamic || x_is_fp8);
    const bool want_sw = need_grad_x && (!dynamic || w_is_fp8);
    if ((want_sx && sx_fwd == nullptr) || (want_sw && sw_fwd == nullptr))
        return fail(FP8DSA_ERR_INVALID_ARG, "sx_fwd / sw_fwd are required (delayed scaling or a pre-quantized x / w)");
    if ((g_is_fp8 && !aligned16(g)) || (need_grad_w && x_is_fp8 && !aligned16(x)) || (need_grad_x && w_is_fp8 && !aligned16(w)))
        return fail(FP8DSA_ERR_UNSUPPORTED, "pre-quantized operands must be 16-byte aligned");
    if (dynamic && !(pow2_margin > 0.0f)) return fail(FP8DSA_ERR_INVALID_ARG, "pow2_margin must be > 0");
    int rc = check_ring_arg(g_is_fp8 ? nullptr : g_ring, "g_ring");
    if (rc) return rc;
    if ((reinterpret_cast<uintptr_t>(workspace) & (kAlign - 1)) != 0)
        return fail(FP8DSA_ERR_UNSUPPORTED, "workspace must be 256-byte aligned");
    const BwdLayout L = bwd_layout(m, k, n);
    if (workspace_bytes < L.total)
        return fail(FP8DSA_ERR_WORKSPACE, "workspace too small: need " + std::to_string(L.total) + " bytes");
    rc = check_device();
    if (rc) return rc;

    uint8_t* ws = static_cast<uint8_t*>(workspace);
    float* colsum = reinterpret_cast<float*>(ws + L.colsum);
    uint32_t* scratch = reinterpret_cast<uint32_t*>(ws + L.scratch);
    float* internal = reinterpret_cast<float*>(ws + L.scratch + 64);
    // a pre-quantized g is read at its own step; a bf16 g's step is measured or taken from the ring
    const float* sg = g_is_fp8 ? g_step : (sg_used ? sg_used : internal);
    const float* sx = sx_fwd;
    const float* sw = sw_fwd;
    if (g_is_fp8 && sg_used != nullptr) {
        cudaError_t e = cudaMemcpyAsync(sg_used, g_step, sizeof(float), cudaMemcpyDeviceToDevice, stream);
        if (e != cudaSuccess) return fail(FP8DSA_ERR_CUDA, std::string("copy g_step: ") + cudaGetErrorString(e));
    }
    if (dynamic) {  // measure the bf16 operands only
        AmaxJob jobs[3];
        int nj = 0;
        auto add = [&](const void* t, int64_t numel, float* out) {
            jobs[nj].x = t;
            jobs[nj].numel = numel;
            jobs[nj].fp8_max = fmt_max(fmt);
            jobs[nj].pow2_margin = pow2_margin;
            jobs[nj].scale_out = out;
            ++nj;
        };
        if (!g_is_fp8) add(g, m * n, const_cast<float*>(sg));
        if (need_grad_w && !x_is_fp8) {
            add(x, m * k, internal + 1);
            sx = internal + 1;
        }
        if (need_grad_x && !w_is_fp8) {
            add(w, n * k, internal + 2);
            sw = internal + 2;
        }
        if (nj > 0) {
            cudaError_t e = cudaMemsetAsync(scratch, 0, 64, stream);
            if (e != cudaSuccess) return fail(FP8DSA_ERR_CUDA, std::string("memset scratch: ") + cudaGetErrorString(e));
            rc = launch_amax_jobs(jobs, nj, scratch, stream);
            if (rc) return rc;
        }
    }
    // the operands the GEMMs read: a bf16 operand's bytes in the workspace (K-major), a
    // pre-quantized one in place (MN-major where the GEMM needs it transposed)
    const uint8_t* g8 = g_is_fp8 ? static_cast<const uint8_t*>(g) : ws + L.g8;
    uint8_t* g8t = ws + L.g8t;
    uint8_t* x8t = ws + L.x8t;
    uint8_t* w8t = ws + L.w8t;
    QuantJob jobs[3];
    int nq = 0;
    if (!g_is_fp8) {  // g: both orientations, ring fold, per-tile column sums
        QuantJob& q = jobs[nq++];
        q.x = g;
        q.rows = m;
        q.cols = n;
        q.fmt = fmt;
        q.out = ws + L.g8;
        q.out_t = g8t;
        q.colsum_partial = need_grad_b && m > 0 ? colsum : nullptr;
        if (dynamic) {
            q.scale = sg;
        } else {
            q.scale = g_ring->state + g_ring->hist_len;
            q.ring = g_ring;
            q.scale_used_out = const_cast<float*>(sg);
            q.defer_fold = true;  // folded by the GEMM launch below
        }
    }
    if (need_grad_w && !x_is_fp8) {
        QuantJob& q = jobs[nq++];
        q.x = x;
        q.rows = m;
        q.cols = k;
        q.fmt = fmt;
        q.out_t = x8t;
        q.scale = sx;
    }
    if (need_grad_x && !w_is_fp8) {
        QuantJob& q = jobs[nq++];
        q.x = w;
        q.rows = n;
        q.cols = k;
        q.fmt = fmt;
        q.out_t = w8t;
        q.scale = sw;
    }
    SplitWorkspace split;
    split.counters = reinterpret_cast<uint32_t*>(ws + L.counters);
    split.counter_words = L.counter_words;
    split.partial = reinterpret_cast<float*>(ws + L.partial);
    split.partial_bytes = L.total - L.partial;
    bool zeroed = false;  // the split-K counters are zeroed by the first launch below
    if (nq > 0) {
        rc = launch_quantize_batch(jobs, nq, stream, split.counters, split.counter_words);
        if (rc) return rc;
        zeroed = true;
    }
    if (g_is_fp8 && need_grad_b && m > 0) {  // the bias gradient of the dequantized g
        rc = launch_colsum_fp8(g8, fmt, m, n, g_step, colsum, zeroed ? nullptr : split.counters,
                               zeroed ? 0 : split.counter_words, stream);
        if (rc) return rc;
        zeroed = true;
    }
    GemmDesc gd[2];
    int ng = 0;
    if (need_grad_x)  // grad_x [m][k] = g8 [m][n] . (w8t [k][n])^T, or . w8 [n][k] read as B = [K][N]
        gd[ng++] = w_is_fp8 ? GemmDesc{g8, static_cast<const uint8_t*>(w), fmt, fmt, 0, 1, m, k, n, n, k, k, 1, 0, 0, 0,
                                       sg, sw, nullptr, 0, nullptr, grad_x}
                            : GemmDesc{g8, w8t, fmt, fmt, 0, 0, m, k, n, n, n, k, 1, 0, 0, 0, sg, sw, nullptr, 0,
                                       nullptr, grad_x};
    if (need_grad_w) {  // grad_w [n][k] = g^T [n][m] . x [m][k]
        const uint8_t* a = g_is_fp8 ? g8 : g8t;                  // A = g8 [m][n] as [K][M], or g8t [n][m]
        const uint8_t* b = x_is_fp8 ? static_cast<const uint8_t*>(x) : x8t;  // B = x8 [m][k] as [K][N], or x8t [k][m]
        gd[ng++] = GemmDesc{a, b, fmt, fmt, g_is_fp8 ? 1 : 0, x_is_fp8 ? 1 : 0, n, k, m, g_is_fp8 ? n : m,
                            x_is_fp8 ? k : m, k, 1, 0, 0, 0, sg, sx, nullptr, 0, nullptr, grad_w};
    }
    const int64_t tiles = m > 0 ? (m + 127) / 128 : 0;
    const bool fold = !g_is_fp8 && !dynamic && ring_fold_in_call();
    return gemm_launch_group(gd, ng, need_grad_b ? colsum : nullptr, need_grad_b ? tiles : 0, need_grad_b ? n : 0,
                             need_grad_b ? grad_b : nullptr, zeroed ? &split : nullptr, g_ring, fold ? 1 : 0, stream);
}

size_t linear_backward_fp8_saved_t_workspace_size(int64_t m, int64_t k, int64_t n) {
    if (m < 0 || k < 0 || n < 0) return 0;
    return saved_layout(m, k, n).total;
}

int linear_backward_fp8_saved_t(const void* g, const uint8_t* x8t, const uint8_t* w8t, int64_t m, int64_t k, int64_t n,
                                fp8_fmt_t fmt, fp8_fmt_t fmt_t, int need_grad_x, int need_grad_w, int need_grad_b,
                                const float* sx, const float* sw, const fp8_ring_t* g_ring, float pow2_margin,
                                float* sg_used, void* workspace, size_t workspace_bytes, void* grad_x, void* grad_w,
                                void* grad_b, cudaStream_t stream) {
    clear_error();
    if (!valid_fmt(fmt) || !valid_fmt(fmt_t)) return fail(FP8DSA_ERR_INVALID_ARG, "formats must be FP8_E4M3 or FP8_E5M2");
    if (m < 0 || k < 0 || n < 0) return fail(FP8DSA_ERR_INVALID_ARG, "negative size");
    if (missing(g, m * n) || workspace == nullptr) return fail(FP8DSA_ERR_INVALID_ARG, "g and workspace are required");
    if (need_grad_x && (missing(w8t, n * k) || sw == nullptr || missing(grad_x, m * k)))
        return fail(FP8DSA_ERR_INVALID_ARG, "grad_x needs w8t, sw and grad_x");
    if (need_grad_w && (missing(x8t, m * k) || sx == nullptr || missing(grad_w, n * k)))
        return fail(FP8DSA_ERR_INVALID_ARG, "grad_w needs x8t, sx and grad_w");
    if (need_grad_b && missing(grad_b, n)) return fail(FP8DSA_ERR_INVALID_ARG, "grad_b is NULL");
    if (k % 16 != 0 || n % 16 != 0) return fail(FP8DSA_ERR_UNSUPPORTED, "k and n must be multiples of 16");
    if (need_grad_w && m % 16 != 0) return fail(FP8DSA_ERR_UNSUPPORTED, "m must be a multiple of 16 for grad_w");
    if ((need_grad_w && !aligned16(x8t)) || (need_grad_x && !aligned16(w8t)))
        return fail(FP8DSA_ERR_UNSUPPORTED, "x8t and w8t must be 16-byte aligned");
    const bool dynamic = g_ring == nullptr;
    if (dynamic && !(pow2_margin > 0.0f)) return fail(FP8DSA_ERR_INVALID_ARG, "pow2_margin must be > 0");
    int rc = check_ring_arg(g_ring, "g_ring");
    if (rc) return rc;
    if ((reinterpret_cast<uintptr_t>(workspace) & (kAlign - 1)) != 0)
        return fail(FP8DSA_ERR_UNSUPPORTED, "workspace must be 256-byte aligned");
    const SavedLayout L = saved_layout(m, k, n);
    if (workspace_bytes < L.total)
        return fail(FP8DSA_ERR_WORKSPACE, "workspace too small: need " + std::to_string(L.total) + " bytes");
    rc = check_device();
    if (rc) return rc;

    uint8_t* ws = static_cast<uint8_t*>(workspace);
    uint8_t* g8 = ws + L.g8;
    uint8_t* g8t = ws + L.g8t;
    float* colsum = reinterpret_cast<float*>(ws + L.colsum);
    uint32_t* scratch = reinterpret_cast<uint32_t*>(ws + L.scratch);
    float* internal = reinterpret_cast<float*>(ws + L.scratch + 64);
    float* sg = sg_used ? sg_used : internal;

    if (dynamic) {
        cudaError_t e = cudaMemsetAsync(scratch, 0, 64, stream);
        if (e != cudaSuccess) return fail(FP8DSA_ERR_CUDA, std::string("memset scratch: ") + cudaGetErrorString(e));
        AmaxJob job;
        job.x = g;
        job.numel = m * n;
        job.fp8_max = fmt_max(fmt);
        job.pow2_margin = pow2_margin;
        job.scale_out = sg;
        rc = launch_amax_jobs(&job, 1, scratch, stream);
        if (rc) return rc;
    }
    // g only: both orientations, its ring fold and (for grad_b) the per-tile column sums
    QuantJob qg;
    qg.x = g;
    qg.rows = m;
    qg.cols = n;
    qg.fmt = fmt;
    qg.out = g8;
    qg.out_t = g8t;
    qg.colsum_partial = need_grad_b && m > 0 ? colsum : nullptr;  // no rows: grad_b is zero, no partials
    if (dynamic) {
        qg.scale = sg;
    } else {
        qg.scale = g_ring->state + g_ring->hist_len;
        qg.ring = g_ring;
        qg.scale_used_out = sg;
        qg.defer_fold = true;  // folded by the GEMM launch below
    }
    SplitWorkspace split;
    split.counters = reinterpret_cast<uint32_t*>(ws + L.counters);
    split.counter_words = L.counter_words;
    split.partial = reinterpret_cast<float*>(ws + L.partial);
    split.partial_bytes = L.total - L.partial;
    rc = launch_quantize_batch(&qg, 1, stream, split.counters, split.counter_words);
    if (rc) return rc;
    // the same two NT GEMMs as linear_backward_fp8, on the saved transposes
    GemmDesc gd[2];
    int ng = 0;
    if (need_grad_x)  // grad_x [m][k] = g8 [m][n] . (w8t [k][n])^T
        gd[ng++] = GemmDesc{g8, w8t, fmt, fmt_t, 0, 0, m, k, n, n, n, k, 1, 0, 0, 0, sg, sw, nullptr, 0, nullptr, grad_x};
    if (need_grad_w)  // grad_w [n][k] = g8t [n][m] . (x8t [k][m])^T
        gd[ng++] = GemmDesc{g8t, x8t, fmt, fmt_t, 0, 0, n, k, m, m, m, k, 1, 0, 0, 0, sg, sx, nullptr, 0, nullptr, grad_w};
    const int64_t tiles = m > 0 ? (m + 127) / 128 : 0;
    return gemm_launch_group(gd, ng, need_grad_b ? colsum : nullptr, need_grad_b ? tiles : 0, need_grad_b ? n : 0,
                             need_grad_b ? grad_b : nullptr, &split, g_ring, (dynamic || !ring_fold_in_call()) ? 0 : 1, stream);
}

size_t linear_backward_fp8_mixed_workspace_size(int64_t m, int64_t k, int64_t n) {
    if (m < 0 || k < 0 || n < 0) return 0;
    return mix_layout(m, k, n).total;
}

int linear_backward_fp8_mixed(const void* g, const uint8_t* x8, const uint8_t* w8, int64_t m, int64_t k, int64_t n,
                              fp8_fmt_t fmt_g, fp8_fmt_t fmt_x, fp8_fmt_t fmt_w, int need_grad_x, int need_grad_w,
                              int need_grad_b, const float* sx, const float* sw, const fp8_ring_t* g_ring,
                              float pow2_margin, float* sg_used, void* workspace, size_t workspace_bytes,
                              void* grad_x, void* grad_w, void* grad_b, cudaStream_t stream) {
    clear_error();
    if (!valid_fmt(fmt_g) || !valid_fmt(fmt_x) || !valid_fmt(fmt_w))
        return fail(FP8DSA_ERR_INVALID_ARG, "formats must be FP8_E4M3 or FP8_E5M2");
    if (m < 0 || k < 0 || n < 0) return fail(FP8DSA_ERR_INVALID_ARG, "negative size");
    if (missing(g, m * n) || workspace == nullptr) return fail(FP8DSA_ERR_INVALID_ARG, "g and workspace are required");
    if (need_grad_x && (missing(w8, n * k) || sw == nullptr || missing(grad_x, m * k)))
        return fail(FP8DSA_ERR_INVALID_ARG, "grad_x needs w8, sw and grad_x");
    if (need_grad_w && (missing(x8, m * k) || sx == nullptr || missing(grad_w, n * k)))
        return fail(FP8DSA_ERR_INVALID_ARG, "grad_w needs x8, sx and grad_w");
    if (need_grad_b && missing(grad_b, n)) return fail(FP8DSA_ERR_INVALID_ARG, "grad_b is NULL");
    if (k % 16 != 0 || n % 16 != 0) return fail(FP8DSA_ERR_UNSUPPORTED, "k and n must be multiples of 16");
    if ((need_grad_w && !aligned16(x8)) || (need_grad_x && !aligned16(w8)))
        return fail(FP8DSA_ERR_UNSUPPORTED, "x8 and w8 must be 16-byte aligned");
    const bool dynamic = g_ring == nullptr;
    if (dynamic && !(pow2_margin > 0.0f)) return fail(FP8DSA_ERR_INVALID_ARG, "pow2_margin must be > 0");
    int rc = check_ring_arg(g_ring, "g_ring");
    if (rc) return rc;
    if ((reinterpret_cast<uintptr_t>(workspace) & (kAlign - 1)) != 0)
        return fail(FP8DSA_ERR_UNSUPPORTED, "workspace must be 256-byte aligned");
    const MixLayout L = mix_layout(m, k, n);
    if (workspace_bytes < L.total)
        return fail(FP8DSA_ERR_WORKSPACE, "workspace too small: need " + std::to_string(L.total) + " bytes");
    rc = check_device();
    if (rc) return rc;

    uint8_t* ws = static_cast<uint8_t*>(workspace);
    uint8_t* g8 = ws + L.g8;
    float* colsum = reinterpret_cast<float*>(ws + L.colsum);
    uint32_t* scratch = reinterpret_cast<uint32_t*>(ws + L.scratch);
    float* internal = reinterpret_cast<float*>(ws + L.scratch + 64);
    float* sg = sg_used ? sg_used : internal;

    if (dynamic) {
        cudaError_t e = cudaMemsetAsync(scratch, 0, 64, stream);
        if (e != cudaSuccess) return fail(FP8DSA_ERR_CUDA, std::string("memset scratch: ") + cudaGetErrorString(e));
        AmaxJob job;
        job.x = g;
        job.numel = m * n;
        job.fp8_max = fmt_max(fmt_g);
        job.pow2_margin = pow2_margin;
        job.scale_out = sg;
        rc = launch_amax_jobs(&job, 1, scratch, stream);
        if (rc) return rc;
    }
    // g only: row-major bytes, its ring fold and (for grad_b) the per-tile column sums
    QuantJob qg;
    qg.x = g;
    qg.rows = m;
    qg.cols = n;
    qg.fmt = fmt_g;
    qg.out = g8;
    qg.colsum_partial = need_grad_b && m > 0 ? colsum : nullptr;  // no rows: grad_b is zero, no partials
    if (dynamic) {
        qg.scale = sg;
    } else {
        qg.scale = g_ring->state + g_ring->hist_len;
        qg.ring = g_ring;
        qg.scale_used_out = sg;
        qg.defer_fold = true;  // folded by the GEMM launch below
    }
    SplitWorkspace split;
    split.counters = reinterpret_cast<uint32_t*>(ws + L.counters);
    split.counter_words = L.counter_words;
    split.partial = reinterpret_cast<float*>(ws + L.partial);
    split.partial_bytes = L.total - L.partial;
    rc = launch_quantize_batch(&qg, 1, stream, split.counters, split.counter_words);
    if (rc) return rc;
    // the forward's bytes are read in place: w8 [n][k] is B = [K][N] of grad_x (MN-major);
    // g8 [m][n] is A = [K][M] and x8 [m][k] is B = [K][N] of grad_w (both MN-major)
    GemmDesc gd[2];
    int ng = 0;
    if (need_grad_x)  // grad_x [m][k] = g8 [m][n] . w8 [n][k]
        gd[ng++] = GemmDesc{g8, w8, fmt_g, fmt_w, 0, 1, m, k, n, n, k, k, 1, 0, 0, 0, sg, sw, nullptr, 0, nullptr, grad_x};
    if (need_grad_w)  // grad_w [n][k] = g8^T [n][m] . x8 [m][k]
        gd[ng++] = GemmDesc{g8, x8, fmt_g, fmt_x, 1, 1, n, k, m, n, k, k, 1, 0, 0, 0, sg, sx, nullptr, 0, nullptr, grad_w};
    const int64_t tiles = m > 0 ? (m + 127) / 128 : 0;
    return gemm_launch_group(gd, ng, need_grad_b ? colsum : nullptr, need_grad_b ? tiles : 0, need_grad_b ? n : 0,
                             need_grad_b ? grad_b : nullptr, &split, g_ring, (dynamic || !ring_fold_in_call()) ? 0 : 1, stream);
}

}  // extern "C"
