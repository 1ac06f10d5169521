"""The C ABI without a GPU: the library loads, exports every function ``include/fp8dsa.h``
declares, and rejects bad arguments with the documented codes before touching CUDA."""

import ctypes

import pytest

import fp8_delayed_scaling_amax_b200 as F

INVALID, UNSUPPORTED, WORKSPACE = -1, -2, -5


def test_library_exports_every_header_symbol():
    lib = F.lib()
    names = F.header_functions()
    assert len(names) >= 17
    for name in names:
        assert hasattr(lib, name), name
        assert hasattr(F, name), f"binding lacks {name}"
    assert "fp8dsa" in F.fp8dsa_version()


def test_workspace_sizes_cover_the_buffers():
    m, k, n = 2048, 1024, 3072
    fwd = F.linear_forward_fp8_workspace_size(m, k, n)
    bwd = F.linear_backward_fp8_workspace_size(m, k, n)
    assert fwd >= m * k + n * k
    assert bwd >= 2 * m * n + k * m + k * n + 4 * ((m + 127) // 128) * n
    assert fwd % 256 == 0 and bwd % 256 == 0
    assert F.linear_forward_fp8_workspace_size(-1, 1, 1) == 0


def _rc(fn, *args):
    return getattr(F.lib(), fn)(*args)


def test_quantize_argument_checks():
    lib = F.lib()
    ring = F.fp8_ring_t(None, 16, 0, 448.0, 1.0)
    # bad format
    assert lib.fp8_quantize(16, 0, 4, 4, 16, 7, 0, 16, None, None, None) == INVALID
    assert "fmt" in F.last_error()
    # bad input type
    assert lib.fp8_quantize(16, 9, 4, 4, 16, 0, 0, 16, None, None, None) == INVALID
    # null scale
    assert lib.fp8_quantize(16, 0, 4, 4, None, 0, 0, 16, None, None, None) == INVALID
    # null out
    assert lib.fp8_quantize(16, 0, 4, 4, 16, 0, 0, None, None, None, None) == INVALID
    # negative size
    assert lib.fp8_quantize(16, 0, -1, 4, 16, 0, 0, 16, None, None, None) == INVALID
    # ring with null state
    assert lib.fp8_quantize(16, 0, 4, 4, 16, 0, 0, 16, None, ctypes.byref(ring), None) == INVALID
    # ring index out of range
    ring2 = F.fp8_ring_t(256, 16, 16, 448.0, 1.0)
    assert lib.fp8_quantize(16, 0, 4, 4, 16, 0, 0, 16, None, ctypes.byref(ring2), None) == INVALID
    assert "hist_idx" in F.last_error()
    # misaligned ring state
    ring3 = F.fp8_ring_t(260, 16, 0, 448.0, 1.0)
    assert lib.fp8_quantize(16, 0, 4, 4, 16, 0, 0, 16, None, ctypes.byref(ring3), None) == UNSUPPORTED
    # dual needs both outputs
    assert lib.fp8_quantize_dual(16, 0, 4, 4, 16, 0, 16, None, None, None, None) == INVALID


def test_gemm_argument_checks():
    lib = F.lib()
    g = lib.fp8_gemm
    ok = dict(a=256, b=512, fa=0, fb=0, lay=0, m=32, n=32, k=32, lda=32, ldb=32, ldo=32, batch=1,
              sa=0, sb=0, so=0, pa=64, pb=64, bias=None, bs=None, out=1024)

    def call(**kw):
        d = dict(ok, **kw)
        return g(d["a"], d["b"], d["fa"], d["fb"], d["lay"], d["m"], d["n"], d["k"], d["lda"], d["ldb"], d["ldo"],
                 d["batch"], d["sa"], d["sb"], d["so"], d["pa"], d["pb"], d["bias"], d["bs"], d["out"], None)

    assert call(fa=3) == INVALID
    assert call(lay=9) == INVALID
    assert call(m=-1) == INVALID
    assert call(out=None) == INVALID
    assert call(pa=None) == INVALID
    assert call(ldo=16) == INVALID                     # ldo < n
    assert call(lda=16) == INVALID                     # lda < k for an N-layout A
    assert call(lda=40) == UNSUPPORTED                 # not a multiple of 16
    assert call(a=257) == UNSUPPORTED                  # misaligned operand
    assert call(batch=2, sa=8, so=1024) == UNSUPPORTED  # batch stride not a multiple of 16
    assert call(batch=2, so=0) == INVALID              # batches would overwrite each other
    assert call(bias=None, bs=64) == INVALID           # bias_scale without bias
    assert "bias_scale" in F.last_error()


def test_linear_argument_checks():
    lib = F.lib()
    f = lib.linear_forward_fp8
    ws = F.linear_forward_fp8_workspace_size(64, 64, 64)
    # k not a multiple of 16
    assert f(256, 256, 0, None, None, None, 64, 60, 64, 0, None, None, 1.0, None, None, 1024, ws, 2048, None) == UNSUPPORTED
    # workspace too small
    assert f(256, 256, 0, None, None, None, 64, 64, 64, 0, None, None, 1.0, None, None, 1024, 16, 2048, None) == WORKSPACE
    # misaligned workspace
    assert f(256, 256, 0, None, None, None, 64, 64, 64, 0, None, None, 1.0, None, None, 1040, ws, 2048, None) == UNSUPPORTED
    # fp8 weight without its step
    assert f(256, 256, 1, None, None, None, 64, 64, 64, 0, None, None, 1.0, None, None, 1024, ws, 2048, None) == INVALID
    b = lib.linear_backward_fp8
    wsb = F.linear_backward_fp8_workspace_size(64, 64, 64)
    # grad_w requested without x
    assert b(256, None, 256, 64, 64, 64, 1, 0, 1, 0, None, None, None, 1.0, None, 1024, wsb, None, 4096, None, None) == INVALID
    # delayed scaling without the forward's steps
    ring = F.fp8_ring_t(256, 16, 0, 57344.0, 1.0)
    assert b(256, 256, 256, 64, 64, 64, 1, 1, 1, 1, None, None, ctypes.byref(ring), 1.0, None, 1024, wsb,
             4096, 4096, 4096, None) == INVALID


def test_keep_forward_and_mixed_backward_argument_checks():
    lib = F.lib()
    ws = F.linear_forward_fp8_workspace_size(64, 64, 64)
    kf = lib.linear_forward_fp8_keep
    # x8_out is required
    assert kf(256, 256, 0, None, None, None, 64, 64, 64, 0, None, None, 1.0, None, None, None, 4096, 1024, ws,
              4096, None) == INVALID
    # w8_out is required unless w is already fp8
    assert kf(256, 256, 0, None, None, None, 64, 64, 64, 0, None, None, 1.0, None, None, 4096, None, 1024, ws,
              4096, None) == INVALID
    # kept buffers must be 16-byte aligned (TMA reads them)
    assert kf(256, 256, 0, None, None, None, 64, 64, 64, 0, None, None, 1.0, None, None, 4104, 8192, 1024, ws,
              4096, None) == UNSUPPORTED
    mb = lib.linear_backward_fp8_mixed
    wsm = F.linear_backward_fp8_mixed_workspace_size(64, 64, 64)
    assert wsm >= 64 * 64 + 4 * 64 and wsm % 256 == 0
    assert F.linear_backward_fp8_mixed_workspace_size(-1, 1, 1) == 0
    args = dict(g=256, x8=4096, w8=8192, m=64, k=64, n=64, fg=1, fx=0, fw=0, gx=1, gw=1, gb=1, sx=512, sw=768,
                ring=None, margin=1.0, sg=None, ws=1024, wsb=wsm, dx=16384, dw=32768, db=65536)

    def call(**kw):
        a = dict(args, **kw)
        return mb(a["g"], a["x8"], a["w8"], a["m"], a["k"], a["n"], a["fg"], a["fx"], a["fw"], a["gx"], a["gw"],
                  a["gb"], a["sx"], a["sw"], a["ring"], a["margin"], a["sg"], a["ws"], a["wsb"], a["dx"], a["dw"],
                  a["db"], None)
    assert call(fg=5) == INVALID
    assert call(fx=-1) == INVALID
    assert call(w8=None) == INVALID          # grad_x without w8
    assert call(sx=None) == INVALID          # grad_w without x8's step
    assert call(db=None) == INVALID
    assert call(k=40) == UNSUPPORTED
    assert call(x8=4100) == UNSUPPORTED      # x8 not 16-byte aligned
    assert call(ws=1040) == UNSUPPORTED      # workspace not 256-byte aligned
    assert call(wsb=wsm - 256) == WORKSPACE
    assert call(margin=0.0) == INVALID       # dynamic scaling needs a positive margin


def test_save_rm_forward_argument_checks():
    f = F.lib().linear_forward_fp8_save_rm
    ws = F.linear_forward_fp8_workspace_size(64, 64, 64)
    ring = F.fp8_ring_t(256, 16, 0, 448.0, 1.0)
    r = ctypes.byref(ring)
    # both copies are required
    assert f(256, 256, None, None, 64, 64, 64, 0, 1, r, r, None, None, None, 4096, 1024, ws, 2048, None) == INVALID
    # delayed scaling only (both rings)
    assert f(256, 256, None, None, 64, 64, 64, 0, 1, None, None, None, None, 4096, 8192, 1024, ws, 2048, None) == INVALID
    # the copies must be 16-byte aligned
    assert f(256, 256, None, None, 64, 64, 64, 0, 1, r, r, None, None, 4100, 8192, 1024, ws, 2048, None) == UNSUPPORTED
    # bad second format
    assert f(256, 256, None, None, 64, 64, 64, 0, 5, r, r, None, None, 4096, 8192, 1024, ws, 2048, None) == INVALID


def test_prequant_backward_argument_checks():
    pb = F.lib().linear_backward_fp8_prequant
    wsb = F.linear_backward_fp8_workspace_size(64, 64, 64)
    ring = F.fp8_ring_t(256, 16, 0, 57344.0, 1.0)
    args = dict(g=256, gf=1, gs=512, x=4096, xf=0, w=8192, wf=0, m=64, k=64, n=64, fmt=1, gx=1, gw=1, gb=1,
                sx=768, sw=1024, ring=ctypes.byref(ring), margin=1.0, sg=None, ws=1024, wsb=wsb, dx=16384, dw=32768,
                db=65536)

    def call(**kw):
        a = dict(args, **kw)
        return pb(a["g"], a["gf"], a["gs"], a["x"], a["xf"], a["w"], a["wf"], a["m"], a["k"], a["n"], a["fmt"],
                  a["gx"], a["gw"], a["gb"], a["sx"], a["sw"], a["ring"], a["margin"], a["sg"], a["ws"], a["wsb"],
                  a["dx"], a["dw"], a["db"], None)
    assert call(fmt=7) == INVALID
    assert call(gs=None) == INVALID            # a pre-quantized g needs its step
    assert call(sx=None) == INVALID            # delayed scaling needs the forward's steps
    assert call(ring=None, xf=1, sx=None) == INVALID  # a pre-quantized x needs its step even when dynamic
    assert call(g=260) == UNSUPPORTED          # pre-quantized g not 16-byte aligned
    assert call(xf=1, x=4100) == UNSUPPORTED   # pre-quantized x not 16-byte aligned
    assert call(n=40) == UNSUPPORTED
    assert call(m=40) == UNSUPPORTED           # grad_w needs m % 16 == 0
    assert call(ws=1040) == UNSUPPORTED
    assert call(wsb=wsb - 256) == WORKSPACE
    assert call(db=None) == INVALID
    assert call(ring=None, gf=0, margin=0.0) == INVALID


def test_saved_transpose_forward_and_backward_argument_checks():
    lib = F.lib()
    ws = F.linear_forward_fp8_workspace_size(64, 64, 64)
    rx = F.fp8_ring_t(256, 16, 0, 448.0, 1.0)
    rw = F.fp8_ring_t(512, 16, 0, 448.0, 1.0)
    fa = dict(x=256, w=256, b=None, bs=None, m=64, k=64, n=64, f=0, ft=1, rx=ctypes.byref(rx), rw=ctypes.byref(rw),
              sx=None, sw=None, xt=4096, wt=8192, ws=1024, wsb=ws, y=2048)

    def fwd(**kw):
        a = dict(fa, **kw)
        return lib.linear_forward_fp8_save_t(a["x"], a["w"], a["b"], a["bs"], a["m"], a["k"], a["n"], a["f"], a["ft"],
                                             a["rx"], a["rw"], a["sx"], a["sw"], a["xt"], a["wt"], a["ws"], a["wsb"],
                                             a["y"], None)
    assert fwd(xt=None) == INVALID            # both transposed outputs are required
    assert fwd(wt=None) == INVALID
    assert fwd(ft=7) == INVALID               # bad second format
    assert fwd(rx=None, rw=None) == INVALID   # dynamic scaling: the backward's steps differ
    assert fwd(rw=None) == INVALID
    assert fwd(xt=4100) == UNSUPPORTED        # not 16-byte aligned
    assert fwd(m=72, wsb=F.linear_forward_fp8_workspace_size(72, 64, 64)) == UNSUPPORTED  # x8t rows: 16-B multiples
    assert fwd(wsb=ws - 256) == WORKSPACE
    sb = lib.linear_backward_fp8_saved_t
    wss = F.linear_backward_fp8_saved_t_workspace_size(64, 64, 64)
    assert wss >= 2 * 64 * 64 + 4 * 64 and wss % 256 == 0
    assert F.linear_backward_fp8_saved_t_workspace_size(-1, 1, 1) == 0
    assert wss < F.linear_backward_fp8_workspace_size(64, 64, 64)  # no x^T / w^T inside
    ba = dict(g=256, xt=4096, wt=8192, m=64, k=64, n=64, f=1, ft=1, gx=1, gw=1, gb=1, sx=512, sw=768, ring=None,
              margin=1.0, sg=None, ws=1024, wsb=wss, dx=16384, dw=32768, db=65536)

    def bwd(**kw):
        a = dict(ba, **kw)
        return sb(a["g"], a["xt"], a["wt"], a["m"], a["k"], a["n"], a["f"], a["ft"], a["gx"], a["gw"], a["gb"],
                  a["sx"], a["sw"], a["ring"], a["margin"], a["sg"], a["ws"], a["wsb"], a["dx"], a["dw"], a["db"],
                  None)
    assert bwd(f=3) == INVALID
    assert bwd(ft=-1) == INVALID
    assert bwd(wt=None) == INVALID           # grad_x without w8t
    assert bwd(sx=None) == INVALID           # grad_w without x8t's step
    assert bwd(db=None) == INVALID
    assert bwd(n=40) == UNSUPPORTED
    assert bwd(m=40) == UNSUPPORTED          # grad_w reads x8t rows of m bytes
    assert bwd(xt=4100) == UNSUPPORTED
    assert bwd(ws=1040) == UNSUPPORTED
    assert bwd(wsb=wss - 256) == WORKSPACE
    assert bwd(margin=0.0) == INVALID


def test_fp8_output_gemm_argument_checks():
    lib = F.lib()
    g8 = lib.fp8_gemm_fp8out
    # out8 required; out8_step required; bad out8 format; k = 0 with an fp8 output
    assert g8(16, 16, 0, 0, 0, 64, 64, 64, 64, 64, 64, 1, 0, 0, 0, 256, 256, None, None, 1024, 0, 512, None, None,
              None, None) == INVALID
    assert g8(16, 16, 0, 0, 0, 64, 64, 64, 64, 64, 64, 1, 0, 0, 0, 256, 256, None, None, 1024, 0, None, 2048, None,
              None, None) == INVALID
    assert g8(16, 16, 0, 0, 0, 64, 64, 64, 64, 64, 64, 1, 0, 0, 0, 256, 256, None, None, 1024, 7, 512, 2048, None,
              None, None) == INVALID
    assert g8(16, 16, 0, 0, 0, 64, 64, 0, 64, 64, 64, 1, 0, 0, 0, 256, 256, None, None, None, 0, 512, 2048, None,
              None, None) == UNSUPPORTED
    # fp8_gemm itself still requires its bf16 output
    assert lib.fp8_gemm(16, 16, 0, 0, 0, 64, 64, 64, 64, 64, 64, 1, 0, 0, 0, 256, 256, None, None, None,
                        None) == INVALID


def test_misc_argument_checks():
    lib = F.lib()
    assert lib.fp8_set_wait_timeout_ns(0) == INVALID
    assert lib.fp8_profiler_read(7, None, None, None) == INVALID
    assert lib.fp8_scale_ring_init(None, 16, None) == INVALID
    assert lib.fp8_scale_ring_init(256, 0, None) == INVALID
    assert lib.fp8_amax_scale(256, 0, 16, 448.0, 1.0, None, None, 256, None) == INVALID
    assert lib.fp8_get_device_status(None, None) == INVALID
    assert lib.fp8_set_tiled_persist_threshold(-1) == INVALID
    assert lib.fp8_set_tiled_persist_threshold(1024) == 0
    assert lib.fp8_set_gemm_split_k(-1) == INVALID
    assert lib.fp8_set_gemm_split_k(5) == INVALID
    assert lib.fp8_set_gemm_split_k(0) == 0
    assert lib.fp8_set_ring_fold_mode(2) == INVALID
    assert lib.fp8_set_ring_fold_mode(0) == 0
    bad = (F.fp8_ring_t * 2)(F.fp8_ring_t(256, 16, 0, 448.0, 1.0), F.fp8_ring_t(256, 0, 0, 448.0, 1.0))
    assert lib.fp8_scale_ring_fold(bad, 2, None, None) == INVALID          # second ring: hist_len 0
    assert lib.fp8_scale_ring_collect_amax(bad, 1, None, None) == INVALID  # no output
    assert lib.fp8_scale_ring_fold(None, 3, None, None) == INVALID
    assert lib.fp8_scale_ring_fold(None, 0, None, None) == 0               # nothing to fold
    assert lib.fp8_set_gemm_split_k(1) == 0
    ring = F.Ring(None, 4)
    for _ in range(5):
        ring.advance()
    assert ring.hist_idx == 1


def test_empty_tensors_may_be_null():
    """A tensor without elements may come as NULL (an empty framework tensor has no storage).
    Each call below stops at a later argument check that fails before any CUDA call (a
    misaligned workspace, or ldo < n), which proves the NULL passed the pointer checks; a NULL
    tensor that has elements is still INVALID_ARG with the pointer message.  No call reaches the
    device, so this is safe with or without a GPU."""
    lib = F.lib()
    f = lib.linear_forward_fp8
    ws = F.linear_forward_fp8_workspace_size(64, 64, 64)
    # m = 0: x and y empty; the misaligned workspace is what fails
    assert f(None, 256, 0, None, None, None, 0, 64, 64, 0, None, None, 1.0, None, None, 1040, ws, None, None) == UNSUPPORTED
    # m > 0: x is required
    assert f(None, 256, 0, None, None, None, 64, 64, 64, 0, None, None, 1.0, None, None, 1040, ws, 2048, None) == INVALID
    b = lib.linear_backward_fp8
    wsb = F.linear_backward_fp8_workspace_size(64, 64, 64)
    # m = 0: g, x and grad_x empty; w, grad_w and grad_b still have elements
    assert b(None, None, 256, 0, 64, 64, 1, 1, 1, 1, None, None, None, 1.0, None, 1040, wsb, None, 4096, 4096,
             None) == UNSUPPORTED
    # n = 0: g, w, grad_w and grad_b empty
    assert b(None, 256, None, 64, 64, 0, 1, 1, 1, 1, None, None, None, 1.0, None, 1040, wsb, 4096, None, None,
             None) == UNSUPPORTED
    # m > 0 and n > 0: g is required
    assert b(None, 256, 256, 64, 64, 64, 1, 1, 1, 1, None, None, None, 1.0, None, 1040, wsb, 4096, 4096, 4096,
             None) == INVALID
    # a GEMM output without elements: the NULL out passes, ldo < n fails
    one = 512
    assert lib.fp8_gemm(None, None, 0, 0, 0, 0, 16, 16, 16, 16, 8, 1, 0, 0, 0, one, one, None, None, None,
                        None) == INVALID
    assert "ldo" in F.last_error()
    assert lib.fp8_gemm(None, None, 0, 0, 0, 16, 16, 16, 16, 16, 16, 1, 0, 0, 0, one, one, None, None, None,
                        None) == INVALID
    assert "out" in F.last_error()
