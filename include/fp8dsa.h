/*
 * fp8dsa -- FP8 linear layer with per-tensor delayed scaling, for NVIDIA B200 (sm_100a).
 *
 * C ABI.  Every entry point takes plain pointers and sizes; no C++ or PyTorch types cross
 * it.  Citations name the AstrAI pages the operation is defined on:
 *   [ext-log]   AstrAI commit log of astrai/extension
 *   [compare]   AstrAI compare view 3e57cc8...main (files named after it)
 *   [by-author] AstrAI commits by author (benchmarks, dispatch notes)
 *
 * Conventions shared by all calls
 * -------------------------------
 * - Device pointers ("dev") must be CUDA device memory of the current device; host pointers
 *   ("host") are ordinary host memory.  The library never allocates, frees or retains any
 *   caller buffer: the caller owns everything, including rings and workspaces.
 * - All work is enqueued on `stream` (0 = legacy default stream) and returns without
 *   synchronising.  No scale, amax or status value ever crosses to the host implicitly.
 * - A "step" (quantization step, `scale`) is the dequantization multiplier: the quantize
 *   kernels multiply by RN32(1/step), and the GEMM multiplies the accumulator by
 *   RN32(step_a * step_b) [compare: astrai/extension/fp8.py, fp8_linear_forward].
 * - Return value: FP8DSA_OK (0) or a negative FP8DSA_ERR_* code.  On error nothing has been
 *   enqueued (argument checks run before any CUDA call) unless the code is
 *   FP8DSA_ERR_CUDA, and fp8_last_error() returns a thread-local message.
 * - fp8 bytes: E4M3FN (max 448) or E5M2 (max 57344) [compare: csrc/kernels/fp8/common.h,
 *   FP8Format].  bf16 / f16 / f32 inputs are IEEE bit patterns.
 * - Empty tensors: a tensor argument without elements (a batch of m = 0 rows, k = 0, ...) may be
 *   NULL, as empty framework tensors are.  The linear entries then compute what the
 *   definition gives: an empty tensor's amax is 0 and is recorded by its ring; y and grad_x of
 *   no rows have no elements; grad_w and grad_b, sums over no rows, are zero; with k = 0, y is
 *   the bias (or zero).  Rings, step buffers and the workspace follow their usual rules.
 */
#ifndef FP8DSA_H
#define FP8DSA_H

#include <stddef.h>
#include <stdint.h>
#include <cuda_runtime_api.h>

#ifdef __cplusplus
extern "C" {
#endif

#define FP8DSA_OK 0
#define FP8DSA_ERR_INVALID_ARG (-1)     /* null pointer, bad enum, bad size or index     */
#define FP8DSA_ERR_UNSUPPORTED (-2)     /* alignment / stride the kernels cannot take    */
#define FP8DSA_ERR_CUDA (-3)            /* a CUDA runtime call or launch failed          */
#define FP8DSA_ERR_DEVICE (-4)          /* current device is not compute capability 10.x */
#define FP8DSA_ERR_WORKSPACE (-5)       /* workspace smaller than the *_workspace_size() */

typedef enum { FP8_E4M3 = 0, FP8_E5M2 = 1 } fp8_fmt_t;
typedef enum { FP8_IN_BF16 = 0, FP8_IN_F16 = 1, FP8_IN_F32 = 2 } fp8_in_t;

/* GEMM operand layouts.  First letter: A; second letter: B.
 *   A 'N' = stored [M][K] (K contiguous)      A 'T' = stored [K][M] (M contiguous)
 *   B 'T' = stored [N][K] (K contiguous; the nn.Linear weight)
 *   B 'N' = stored [K][N] (N contiguous)
 * The training GEMMs (forward, dX, dW) are all NT [compare: astrai/extension/fp8.py,
 * _LinearFp8.backward]; NN and TN are the other layouts mm_fp8 accepts
 * [compare: csrc/kernels/fp8/common.h, RowMajor / ColMajor tags]. */
typedef enum { FP8_LAYOUT_NT = 0, FP8_LAYOUT_NN = 1, FP8_LAYOUT_TN = 2, FP8_LAYOUT_TT = 3 } fp8_layout_t;

/* One operand's delayed-scaling history ring [compare: astrai/extension/fp8.py, _ScaleRing].
 * `state` (dev, fp32, hist_len + 4 floats, 16-byte aligned) is laid out
 *     [ hist[0..hist_len) | scale | scale_used | amax | done ]
 * hist: amax history window; scale: the step the next use will quantize with;
 * scale_used: the step the last folding kernel quantized with (its snapshot);
 * amax, done: kernel scratch, zero between calls (self-cleaning).
 * hist_idx in [0, hist_len) is the slot this use records into; the caller advances it
 * host-side, (idx + 1) % hist_len, after each use.  fp8_max is 448 or 57344 for the
 * format the ring's operand is quantized to, pow2_margin = 2^margin (> 0). */
typedef struct {
    float* state;
    int hist_len;
    int hist_idx;
    float fp8_max;
    float pow2_margin;
} fp8_ring_t;

/* Zero the ring's hist_len + 4 floats.  state: dev.  [compare: _ScaleRing.__init__] */
int fp8_scale_ring_init(float* state, int hist_len, cudaStream_t stream);

/* First-use seeding [compare: _ScaleRing.seed]: hist[hist_idx] = max|x| over numel
 * elements of x (dev, in_type), then scale = max(RN32(peak / fp8_max) / pow2_margin, 1e-12)
 * with peak the max over the window.  The pages elide seed's body; this is the reading
 * that makes step 0 of delayed scaling equal dynamic scaling on the same tensor. */
int fp8_scale_ring_seed(const fp8_ring_t* ring, const void* x, fp8_in_t in_type, int64_t numel,
                        cudaStream_t stream);

/* Data-parallel scaling (the pages measure one GPU; this is the standard extension where every
 * rank's rings must agree): with fp8_set_ring_fold_mode(1) the linear entries leave each ring's
 * measured amax in its amax slot instead of folding it.  At the end of a step the caller
 *   1. gathers the slots: fp8_scale_ring_collect_amax(rings, n, amax) -- amax: dev fp32 [n];
 *   2. reduces amax over the ranks with MAX (e.g. an NCCL all-reduce);
 *   3. folds every ring with the reduced values: fp8_scale_ring_fold(rings, n, amax) --
 *      hist[hist_idx] = amax[i], scale_used = the current scale, scale = the formula over the
 *      window, amax slot zeroed (amax == NULL folds each ring's own slot).
 * rings: host array of n descriptors (hist_idx = the slot the step's quantize used); n >= 0.
 * Both run one launch per 128 rings. */
int fp8_scale_ring_collect_amax(const fp8_ring_t* rings, int n, float* amax_out, cudaStream_t stream);
int fp8_scale_ring_fold(const fp8_ring_t* rings, int n, const float* amax, cudaStream_t stream);

/* 0 (default): linear_forward_fp8 / _keep / _noalloc, linear_backward_fp8 and _mixed fold the
 * rings they quantize with, inside the call.  1: they leave the measured amax in each ring's
 * amax slot for fp8_scale_ring_fold (data-parallel training, see above).  Other values:
 * FP8DSA_ERR_INVALID_ARG.  Applies to later calls.  Not on the pages. */
int fp8_set_ring_fold_mode(int mode);

/* Dynamic (current-amax) step [compare: astrai/extension/fp8.py, _dynamic_scale]:
 * *scale_out = max(RN32(max|x| / fp8_max) / pow2_margin, 1e-12) and, if amax_out is not
 * NULL, *amax_out = max|x|.  scratch: dev, 16 bytes, 16-byte aligned, all zero before the
 * first call; the kernel leaves it zero again (self-cleaning), so one scratch may be
 * reused by calls ordered on one stream but not by calls that overlap. */
int fp8_amax_scale(const void* x, fp8_in_t in_type, int64_t numel, float fp8_max,
                   float pow2_margin, float* scale_out, float* amax_out, uint32_t* scratch,
                   cudaStream_t stream);

/* Quantize with fused raw-domain amax [compare: csrc/kernels/fp8/quantize.cuh,
 * fp8_quantize_kernel / fp8_quantize_tiled_kernel; ext-log: amax of the unscaled input].
 *   x: dev, rows x cols row-major, in_type; 16-byte aligned rows take the vector path.
 *   scale: dev, one fp32 step s; each element becomes q_fmt(RN32(x * RN32(1/s))),
 *          round-to-nearest-even, saturated to +-FP8_MAX.
 *   transposed = 0: out is [rows][cols]; = 1: out is the [cols][rows] transpose.
 *   amax_out: dev or NULL; receives max|x| (NaN ignored).
 *   ring: NULL, or a ring whose fold runs in the kernel's last block: scale_used = *scale,
 *         hist[hist_idx] = amax, scale = formula over the window, amax/done re-zeroed
 *         [compare: quantize.cuh, publish_amax; ext-log: zero extra launches].
 *         `scale` may point at ring->state[hist_len] (the ring's own step): every block
 *         reads it before the last block publishes.
 * rows * cols may be 0 (nothing is written, the ring still folds amax 0). */
int fp8_quantize(const void* x, fp8_in_t in_type, int64_t rows, int64_t cols, const float* scale,
                 fp8_fmt_t fmt, int transposed, uint8_t* out, float* amax_out,
                 const fp8_ring_t* ring, cudaStream_t stream);

/* Both orientations from one read of x [compare: astrai/extension/ops/fp8.py, quantize_dual]:
 * out = [rows][cols], out_t = [cols][rows]; amax and ring as fp8_quantize. */
int fp8_quantize_dual(const void* x, fp8_in_t in_type, int64_t rows, int64_t cols,
                      const float* scale, fp8_fmt_t fmt, uint8_t* out, uint8_t* out_t,
                      float* amax_out, const fp8_ring_t* ring, cudaStream_t stream);

/* FP8 x FP8 GEMM with dequantization and fused bias [compare: astrai/extension/ops/fp8.py,
 * mm_fp8; csrc/kernels/fp8/gemm/epilogue.cuh]:
 *     out[b][i][j] = RN_bf16( sum_k A[b][i][k] * B[b][k][j] * RN32(*scale_a * *scale_b) + bias[j] )
 * accumulated in fp32 on the tensor cores (tcgen05.mma kind::f8f6f4, TMEM accumulators).
 *   a, b: dev fp8 bytes in the stored layout named by `layout`, formats fmt_a / fmt_b (the
 *         pages require equal formats; the tensor core takes them independently).
 *   lda, ldb: row strides in elements of the stored matrices; multiples of 16; a, b 16-byte
 *         aligned (TMA).  ldo: row stride of out in elements (>= n).
 *   batch >= 1; stride_a / stride_b / stride_o: element strides between batches; 0 makes a
 *         size-1 operand broadcast over the batch [compare: mm_fp8's batch rule].  Non-zero
 *         operand strides are multiples of 16.
 *   scale_a, scale_b: dev fp32 steps.
 *   bias: NULL, or dev bf16[n] when bias_scale == NULL, or dev fp8[n] in fmt_a when
 *         bias_scale (dev fp32) is given: dequantized as byte * *bias_scale after the operand
 *         scaling [ext-log: FP8Params.bias_scale].
 *   out: dev bf16.  m, n, k >= 0; k == 0 writes the bias (or zeros). */
int fp8_gemm(const uint8_t* a, const uint8_t* b, fp8_fmt_t fmt_a, fp8_fmt_t fmt_b,
             fp8_layout_t layout, int64_t m, int64_t n, int64_t k, int64_t lda, int64_t ldb,
             int64_t ldo, int64_t batch, int64_t stride_a, int64_t stride_b, int64_t stride_o,
             const float* scale_a, const float* scale_b, const void* bias,
             const float* bias_scale, void* out, cudaStream_t stream);

/* fp8_gemm whose epilogue also quantizes its output for the next consumer (the quantize fused
 * into the producer; the pages' FP8-output GEMM, which their final state dropped, is the
 * closest counterpart) [compare: csrc/kernels/fp8/gemm/epilogue.cuh, out_dtype / out_scale in
 * an earlier state]:
 *   every output element v = acc * RN32(sa*sb) + bias is rounded to bf16 as in fp8_gemm, then
 *       out8 = q_{out8_fmt}(RN32(RN_bf16(v) * RN32(1 / *out8_step)))   (RN, saturating)
 *   i.e. exactly the bytes fp8_quantize gives for the bf16 output; |RN_bf16(v)| over the valid
 *   elements is atomically maxed into *out8_amax (dev fp32; not zeroed here -- pass a zeroed
 *   value, or a ring's amax slot and fold later with fp8_scale_ring_fold); *out8_step is
 *   copied to *out8_step_used (may be NULL) for the consumer's dequantization.
 *   out: bf16 output as in fp8_gemm, or NULL to write only out8.  out8: dev bytes with the
 *   same element strides as out (ldo, stride_o).  out8_step: dev fp32 (e.g. a ring's step).
 *   k must be > 0.  Not on the pages in their final state. */
int fp8_gemm_fp8out(const uint8_t* a, const uint8_t* b, fp8_fmt_t fmt_a, fp8_fmt_t fmt_b,
                    fp8_layout_t layout, int64_t m, int64_t n, int64_t k, int64_t lda, int64_t ldb,
                    int64_t ldo, int64_t batch, int64_t stride_a, int64_t stride_b, int64_t stride_o,
                    const float* scale_a, const float* scale_b, const void* bias,
                    const float* bias_scale, void* out, fp8_fmt_t out8_fmt, const float* out8_step,
                    uint8_t* out8, float* out8_amax, float* out8_step_used, cudaStream_t stream);

/* Workspace bytes linear_forward_fp8 needs for (m, k, n): x8, w8 and scale scratch, then the
 * GEMM's split-K region (arrival counters and fp32 partial tiles for up to 4 K ranges per
 * output tile; used only where splitting shortens the schedule). */
size_t linear_forward_fp8_workspace_size(int64_t m, int64_t k, int64_t n);

/* FP8 linear forward y = x w^T + bias [compare: astrai/extension/fp8.py, fp8_linear_forward]:
 *   x: dev bf16 [m][k]; w: dev bf16 [n][k], or fp8 bytes in `fmt` when w_is_fp8 (then
 *      w_step, dev fp32, is the step those bytes were quantized with, and w_ring is unused).
 *   bias: NULL, dev bf16[n], or dev fp8[n] in `fmt` with bias_scale (dev fp32).
 *   Delayed scaling: x_ring and w_ring given.  Each quantize reads its ring's step and
 *      measures the fresh amax; the fold (hist[idx] = amax, next step published, snapshot of
 *      the step used) runs in the GEMM launch that follows, so the GEMM dequantizes with the
 *      steps used (the snapshot) [ext-log: snapshot sx/sw before the finalize].  The ring
 *      states after the call are the same as with the quantize entry's in-kernel fold.
 *   Dynamic scaling: x_ring == NULL (and w_ring == NULL): the steps are measured from x and
 *      w first (max(amax / fp8_max / pow2_margin, 1e-12)), with fp8_max of `fmt` and
 *      pow2_margin given here.
 *   sx_used, sw_used: dev fp32 outputs, the steps the GEMM used (the backward's sx / sw).
 *   workspace: dev, >= linear_forward_fp8_workspace_size(m, k, n) bytes, 256-byte aligned;
 *      no initial contents are needed (the quantize launch clears the split-K counters).
 *   y: dev bf16 [m][n].  k and n must be multiples of 16.
 *   Where the GEMM cuts an output tile's K range across CTAs (split-K), the owner CTA adds
 *   the other ranges' fp32 partial sums in a fixed order: results are deterministic and
 *   differ from the unsplit GEMM only in fp32 summation order. */
int linear_forward_fp8(const void* x, const void* w, int w_is_fp8, const float* w_step,
                       const void* bias, const float* bias_scale, int64_t m, int64_t k, int64_t n,
                       fp8_fmt_t fmt, const fp8_ring_t* x_ring, const fp8_ring_t* w_ring,
                       float pow2_margin, float* sx_used, float* sw_used, void* workspace,
                       size_t workspace_bytes, void* y, cudaStream_t stream);

/* Size of the scratch array linear_forward_fp8_noalloc uses instead of a caller workspace. */
#define FP8DSA_NOALLOC_WORKSPACE_BYTES (16u << 20)

/* linear_forward_fp8 for callers that cannot allocate device memory -- for example a plug-in
 * whose host application owns the device-memory budget and hands it no allocator, or a
 * service that must keep a fixed device footprint after start-up.  The pages have no
 * counterpart to this entry point.
 * Same arguments and results as linear_forward_fp8, without the workspace: the scratch lives
 * in one built-in device array of FP8DSA_NOALLOC_WORKSPACE_BYTES (16 MiB), held by every GPU
 * that loads the library until the process exits.  The array holds the x8 / w8 operand
 * buffers and the scale scratch (about m*k + n*k bytes), and the GEMM here never splits K;
 * shapes whose buffers exceed the array return FP8DSA_ERR_WORKSPACE with a message.
 * The first call on each device looks up the array's address and caches it for the process
 * (make that call before any stream capture; the address belongs to the device context it
 * saw, so do not call again after cudaDeviceReset); no call allocates.  All calls share the
 * array: calls ordered on one stream are safe, calls that overlap on the GPU race. */
int linear_forward_fp8_noalloc(const void* x, const void* w, int w_is_fp8, const float* w_step,
                               const void* bias, const float* bias_scale, int64_t m, int64_t k,
                               int64_t n, fp8_fmt_t fmt, const fp8_ring_t* x_ring,
                               const fp8_ring_t* w_ring, float pow2_margin, float* sx_used,
                               float* sw_used, void* y, cudaStream_t stream);

/* Workspace bytes linear_backward_fp8 needs for (m, k, n): g8, g8T, x8T, w8T, the per-tile
 * column sums and scale scratch, then the dX / dW GEMM's split-K region. */
size_t linear_backward_fp8_workspace_size(int64_t m, int64_t k, int64_t n);

/* FP8 linear backward [compare: astrai/extension/fp8.py, _LinearFp8.backward]:
 *   g: dev bf16 [m][n] (dL/dy); x: dev bf16 [m][k]; w: dev bf16 [n][k].  fmt is the
 *   backward format (E5M2 under the HYBRID policy) for g and the re-quantized x and w.
 *   g is quantized once in both orientations (folding into g_ring); x and w are re-quantized
 *   transposed with the forward's steps and fold no ring; then
 *       grad_x [m][k] = g8 . w8T^T * RN32(sg * sw)   (NT)
 *       grad_w [n][k] = g8T . x8T^T * RN32(sg * sx)  (NT)
 *       grad_b [n]    = RN_bf16(sum over rows of g)
 *   Delayed scaling: g_ring given, sx_fwd / sw_fwd (dev fp32) are the forward's steps.
 *   Dynamic scaling: g_ring == NULL; sg, sx, sw are re-measured at fmt's FP8_MAX and
 *   pow2_margin, and sx_fwd / sw_fwd are ignored.
 *   need_grad_x / need_grad_w / need_grad_b select the outputs (the others may be NULL).
 *   sg_used: dev fp32 output (the step g was quantized with), may be NULL.
 *   workspace: dev, >= linear_backward_fp8_workspace_size(m, k, n) bytes, 256-byte aligned;
 *      no initial contents are needed.  The dX / dW GEMM may split K as in the forward.
 *   k and n must be multiples of 16; m a multiple of 16 when grad_w is needed. */
int linear_backward_fp8(const void* g, const void* x, const void* w, int64_t m, int64_t k,
                        int64_t n, fp8_fmt_t fmt, int need_grad_x, int need_grad_w,
                        int need_grad_b, const float* sx_fwd, const float* sw_fwd,
                        const fp8_ring_t* g_ring, float pow2_margin, float* sg_used,
                        void* workspace, size_t workspace_bytes, void* grad_x, void* grad_w,
                        void* grad_b, cudaStream_t stream);

/* linear_forward_fp8 that also keeps its quantized operands for linear_backward_fp8_mixed:
 *   x8_out: dev [m][k] bytes in `fmt` (16-byte aligned) receives x8;
 *   w8_out: dev [n][k] bytes in `fmt` (16-byte aligned) receives w8 (ignored when w_is_fp8:
 *      the caller's w already holds those bytes).
 * Everything else, including the workspace, is as for linear_forward_fp8; the bytes are the
 * ones the forward GEMM reads.  Not a separate step on the pages: their backward binding
 * accepts operands the forward already quantized [compare: the linear backward binding in
 * an earlier state, pre-quantized g / x / w skip their quantize kernels]. */
int linear_forward_fp8_keep(const void* x, const void* w, int w_is_fp8, const float* w_step,
                            const void* bias, const float* bias_scale, int64_t m, int64_t k,
                            int64_t n, fp8_fmt_t fmt, const fp8_ring_t* x_ring,
                            const fp8_ring_t* w_ring, float pow2_margin, float* sx_used,
                            float* sw_used, uint8_t* x8_out, uint8_t* w8_out, void* workspace,
                            size_t workspace_bytes, void* y, cudaStream_t stream);

/* FP8 linear backward whose operands may each arrive pre-quantized [AstrAI astrai/extension
 * commit log: g / x / w may each be bf16 or pre-quantized fp8 matching fmt, and a
 * pre-quantized operand skips its quantize kernel; a pre-quantized g dequantizes before the
 * bias-sum; compare view, the linear backward binding in an earlier state: a pre-quantized g
 * does not finalize its ring and reports amax_g = 0]:
 *   g: dev [m][n], bf16, or fp8 bytes in fmt (g_is_fp8) at step *g_step;
 *   x: dev [m][k], bf16, or fp8 bytes in fmt (x_is_fp8) at step *sx_fwd;
 *   w: dev [n][k], bf16, or fp8 bytes in fmt (w_is_fp8) at step *sw_fwd.
 *   A bf16 operand is quantized as in linear_backward_fp8 (g in both orientations at the
 *   ring's step, folding g_ring, or at its dynamic step; x / w transposed at sx_fwd / sw_fwd,
 *   or at their dynamic steps when g_ring == NULL).  A pre-quantized operand is read by the
 *   GEMM in place (as an MN-major operand where the product needs its transpose); a
 *   pre-quantized g leaves g_ring untouched (neither read nor folded) and *sg_used = *g_step.
 *       grad_x [m][k] = g8 . w8 * RN32(sg * sw)
 *       grad_w [n][k] = g8^T . x8 * RN32(sg * sx)
 *       grad_b [n]    = RN_bf16(sum over rows of g), a pre-quantized g summed as dec(g8) * sg
 *   sx_fwd / sw_fwd: required for grad_w / grad_x under delayed scaling and whenever x / w
 *   is pre-quantized.  Pre-quantized operands must be 16-byte aligned.  workspace: dev,
 *   >= linear_backward_fp8_workspace_size(m, k, n) bytes, 256-byte aligned.  k and n must be
 *   multiples of 16 (m too for grad_w).  Launches: at most one amax launch (dynamic), one
 *   quantize launch for the bf16 operands, one column-sum launch for a pre-quantized g's
 *   grad_b, and one GEMM launch for grad_x and grad_w. */
int linear_backward_fp8_prequant(const void* g, int g_is_fp8, const float* g_step, const void* x,
                                 int x_is_fp8, const void* w, int w_is_fp8, int64_t m, int64_t k,
                                 int64_t n, fp8_fmt_t fmt, int need_grad_x, int need_grad_w,
                                 int need_grad_b, const float* sx_fwd, const float* sw_fwd,
                                 const fp8_ring_t* g_ring, float pow2_margin, float* sg_used,
                                 void* workspace, size_t workspace_bytes, void* grad_x,
                                 void* grad_w, void* grad_b, cudaStream_t stream);

/* Workspace bytes linear_backward_fp8_mixed needs for (m, k, n): g8, the per-tile column sums,
 * scale scratch and the GEMM's split-K region. */
size_t linear_backward_fp8_mixed_workspace_size(int64_t m, int64_t k, int64_t n);

/* Mixed-format backward that reuses the forward's quantized operands as they are (a reading of
 * the pages' reuse of pre-quantized operands, with each operand keeping its own format: the
 * tensor core takes the A and B formats separately) [compare: the linear backward binding in
 * an earlier state]:
 *   g: dev bf16 [m][n], quantized once row-major in fmt_g (folding g_ring, or at the dynamic
 *      step when g_ring == NULL: max(amax / fp8_max(fmt_g) / pow2_margin, 1e-12));
 *   x8: dev [m][k] bytes in fmt_x with step *sx; w8: dev [n][k] bytes in fmt_w with step *sw
 *      (e.g. from linear_forward_fp8_keep; sx / sw are its sx_used / sw_used); 16-byte aligned.
 *       grad_x [m][k] = g8 . w8 * RN32(sg * sw)      (w8 read in place as B = [K][N])
 *       grad_w [n][k] = g8^T . x8 * RN32(sg * sx)    (g8 and x8 read in place)
 *       grad_b [n]    = RN_bf16(sum over rows of g)
 *   One quantize launch (g) and one GEMM launch (grad_x and grad_w); x and w are not
 *   re-quantized.  The numbers differ from linear_backward_fp8 under HYBRID (there x and w are
 *   re-quantized to E5M2); with fmt_g == fmt_x == fmt_w and x8 / w8 quantized at sx / sw they
 *   are the same.
 *   need_grad_x / need_grad_w / need_grad_b select the outputs (the others may be NULL).
 *   workspace: dev, >= linear_backward_fp8_mixed_workspace_size(m, k, n) bytes, 256-byte
 *      aligned, no initial contents needed.  k and n must be multiples of 16. */
int linear_backward_fp8_mixed(const void* g, const uint8_t* x8, const uint8_t* w8, int64_t m,
                              int64_t k, int64_t n, fp8_fmt_t fmt_g, fp8_fmt_t fmt_x,
                              fp8_fmt_t fmt_w, int need_grad_x, int need_grad_w, int need_grad_b,
                              const float* sx, const float* sw, const fp8_ring_t* g_ring,
                              float pow2_margin, float* sg_used, void* workspace,
                              size_t workspace_bytes, void* grad_x, void* grad_w, void* grad_b,
                              cudaStream_t stream);

/* Delayed-scaling forward that also saves the backward's transposed operands (the pages'
 * backward quantizes x^T and w^T with the forward's steps [AstrAI compare view,
 * astrai/extension/fp8.py, _LinearFp8.backward]; this entry forms them in the forward's
 * quantize launch, from the same products, so x and w are read once per step):
 *   everything as linear_forward_fp8 with w bf16 (no w_is_fp8) and both rings given, plus
 *   x8t_out: dev [k][m] bytes = q_{fmt_t}(RN32(x[r][c] * RN32(1 / sx_used)))  at [c][r];
 *   w8t_out: dev [k][n] bytes = q_{fmt_t}(RN32(w[r][c] * RN32(1 / sw_used)))  at [c][r];
 *   both required, 16-byte aligned; m a multiple of 16.  The bytes equal those
 *   linear_backward_fp8 quantizes for the same steps, so linear_backward_fp8_saved_t gives
 *   exactly its results.  Workspace as linear_forward_fp8 (linear_forward_fp8_workspace_size).
 *   One quantize launch (x and w, both orientations) and one GEMM launch.
 *   FP8DSA_ERR_INVALID_ARG without both rings or outputs, or with a bad fmt_t. */
int linear_forward_fp8_save_t(const void* x, const void* w, const void* bias,
                              const float* bias_scale, int64_t m, int64_t k, int64_t n,
                              fp8_fmt_t fmt, fp8_fmt_t fmt_t, const fp8_ring_t* x_ring,
                              const fp8_ring_t* w_ring, float* sx_used, float* sw_used,
                              uint8_t* x8t_out, uint8_t* w8t_out, void* workspace,
                              size_t workspace_bytes, void* y, cudaStream_t stream);

/* Delayed-scaling forward that also saves the backward's copies of x and w row-major (the
 * pages' backward quantizes x and w with the forward's steps in the backward's format
 * [AstrAI compare view, astrai/extension/fp8.py, _LinearFp8.backward]; this entry forms those
 * bytes in the forward's row-major quantize launch, from the same products, and keeps them
 * in the orientation they are read in, so no transpose is written):
 *   everything as linear_forward_fp8 with w bf16 (no w_is_fp8) and both rings given, plus
 *   x8b_out: dev [m][k] bytes of x in fmt_b at step *sx_used; w8b_out: dev [n][k] bytes of w
 *   in fmt_b at step *sw_used; both 16-byte aligned.
 *   linear_backward_fp8_mixed(g, x8b_out, w8b_out, ..., fmt_g = fmt_x = fmt_w = fmt_b,
 *   sx_used, sw_used, ...) then reads them in place (MN-major operands) and computes the
 *   pages' backward (g, x and w all in fmt_b at the forward's steps) with one quantize launch
 *   for g.  One quantize launch (x and w, two formats each) and one GEMM launch. */
int linear_forward_fp8_save_rm(const void* x, const void* w, const void* bias,
                               const float* bias_scale, int64_t m, int64_t k, int64_t n,
                               fp8_fmt_t fmt, fp8_fmt_t fmt_b, const fp8_ring_t* x_ring,
                               const fp8_ring_t* w_ring, float* sx_used, float* sw_used,
                               uint8_t* x8b_out, uint8_t* w8b_out, void* workspace,
                               size_t workspace_bytes, void* y, cudaStream_t stream);

/* Workspace bytes linear_backward_fp8_saved_t needs for (m, k, n): g8, g8t, the per-tile
 * column sums, scale scratch and the GEMM's split-K region. */
size_t linear_backward_fp8_saved_t_workspace_size(int64_t m, int64_t k, int64_t n);

/* linear_backward_fp8 on the transposes the forward saved (linear_forward_fp8_save_t):
 *   g: dev bf16 [m][n], quantized once in both orientations in fmt (folding g_ring, or at the
 *      dynamic step when g_ring == NULL), with the per-tile column sums for grad_b;
 *   x8t: dev [k][m] bytes in fmt_t with step *sx; w8t: dev [k][n] bytes in fmt_t with step *sw
 *      (the forward's x8t_out / w8t_out and sx_used / sw_used); 16-byte aligned.
 *       grad_x [m][k] = g8 . w8t^T * RN32(sg * sw)    (NT)
 *       grad_w [n][k] = g8t . x8t^T * RN32(sg * sx)   (NT)
 *       grad_b [n]    = RN_bf16(sum over rows of g)
 *   One quantize launch (g only) and one GEMM launch (grad_x and grad_w).  With fmt_t == fmt
 *   the results are bit-identical to linear_backward_fp8 with the same steps.
 *   need_grad_x / need_grad_w / need_grad_b select the outputs (the others may be NULL).
 *   workspace: dev, >= linear_backward_fp8_saved_t_workspace_size(m, k, n) bytes, 256-byte
 *      aligned, no initial contents needed.  k and n multiples of 16; m too for grad_w. */
int linear_backward_fp8_saved_t(const void* g, const uint8_t* x8t, const uint8_t* w8t,
                                int64_t m, int64_t k, int64_t n, fp8_fmt_t fmt, fp8_fmt_t fmt_t,
                                int need_grad_x, int need_grad_w, int need_grad_b,
                                const float* sx, const float* sw, const fp8_ring_t* g_ring,
                                float pow2_margin, float* sg_used, void* workspace,
                                size_t workspace_bytes, void* grad_x, void* grad_w, void* grad_b,
                                cudaStream_t stream);

/* Device status word of the current device: 0, or a nonzero code a kernel set when a bounded
 * wait ran out (a pipeline stall instead of a hang).  Synchronises `stream`, reads the word
 * into *status (host) and clears it.  Not on the pages: added so no kernel can hang a GPU. */
int fp8_get_device_status(cudaStream_t stream, int* status);

/* Upper bound, in nanoseconds, of every bounded wait in the library's kernels
 * (default 2e9 = 2 s).  Applies to launches after the call. */
int fp8_set_wait_timeout_ns(uint64_t ns);

/* Launch the library's kernels with programmatic dependent launch (default 1 = on): each
 * kernel's launch and set-up overlap the tail of the previous kernel on the stream, and it
 * waits for that kernel's results before reading them.  0 launches them plainly.  Applies to
 * launches after the call (and to stream captures made after it).  Not on the pages. */
int fp8_set_pdl(int enabled);

/* Split-K in the linear compositions' GEMMs: an output tile's K range may be cut across CTAs
 * (up to 4 ranges; contributors leave fp32 partials in the workspace, the owner adds them in a
 * fixed order).  1 (default) never splits -- measured on B200, the extra epilogue work of the
 * partials outweighs the shorter MMA schedule on this library's workloads; 0 splits where a
 * model of the schedule says the launch finishes sooner; 2..4 force that many ranges per tile
 * wherever the workspace holds the partials and every range keeps at least 256 bytes of K.
 * Other values: FP8DSA_ERR_INVALID_ARG.  Applies to later launches (and stream captures made
 * after the call).  Not on the pages. */
int fp8_set_gemm_split_k(int splits);

/* Transposed / dual quantize launches covering more than `min_tiles` 128 x 128 tiles (over all
 * tensors of the launch) run on the persistent TMA-fed kernel; smaller ones run one tile per
 * CTA.  Launches that write only transposed bytes switch above min_tiles / 8.  Both kernels
 * give identical bytes, amax and ring updates; the choice only moves time.  Default 1024;
 * min_tiles < 0 is rejected (FP8DSA_ERR_INVALID_ARG).  Applies to later launches.  Not on the
 * pages. */
int fp8_set_tiled_persist_threshold(int64_t min_tiles);

/* Test hook for the failure path: launches one block that waits on a barrier nothing ever
 * arrives at; the wait gives up after the timeout and sets the device status word.
 * Not on the pages. */
int fp8_debug_stalled_wait(cudaStream_t stream);

/* Per-kernel timing: when enabled, every kernel the library launches is bracketed by CUDA
 * events on its own stream (inside a stream capture, by external event-record nodes, so each
 * replay of the graph re-times them).  fp8_profiler_read synchronises, returns the total
 * device milliseconds, launch count and algorithmic bytes (quantize, other) or flops (GEMM)
 * of kernel class `kind` recorded since the last read, then resets that class: 0 quantize,
 * 1 GEMM (both instances), 2 other, 3 the GEMM instance with 256-wide tiles on CTA pairs,
 * 4 the GEMM instance with single-CTA tiles.  Not on the pages (they time with CUDA events from Python; [by-author]). */
int fp8_profiler_enable(int on);
int fp8_profiler_read(int kind, double* total_ms, int64_t* launches, double* bytes_or_flops);

/* Thread-local message describing the last error (empty string if none). */
const char* fp8_last_error(void);

/* Library version string. */
const char* fp8dsa_version(void);

#ifdef __cplusplus
}
#endif

#endif /* FP8DSA_H */
