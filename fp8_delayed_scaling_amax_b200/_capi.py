"""ctypes binding of ``libfp8dsa.so`` -- one Python function per C entry point, same names.

Marshalling only: each wrapper turns tensors into device pointers (``data_ptr()``), picks
the current CUDA stream, calls the C function and raises :class:`FP8Error` on a non-zero
status.  All arithmetic runs in the library's CUDA kernels; there is no fallback path, and
importing a wrapper fails loudly when the library has not been built.
"""

from __future__ import annotations

import ctypes
import os
import re
from ctypes import POINTER, Structure, c_char_p, c_double, c_float, c_int, c_int64, c_size_t, c_uint64, c_void_p

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libfp8dsa.so")
HEADER_PATH = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "include", "fp8dsa.h")

# enums of include/fp8dsa.h
FP8_E4M3, FP8_E5M2 = 0, 1
FP8_IN_BF16, FP8_IN_F16, FP8_IN_F32 = 0, 1, 2
FP8_LAYOUT_NT, FP8_LAYOUT_NN, FP8_LAYOUT_TN, FP8_LAYOUT_TT = 0, 1, 2, 3
FP8_MAX = {FP8_E4M3: 448.0, FP8_E5M2: 57344.0}

ERRORS = {0: "OK", -1: "INVALID_ARG", -2: "UNSUPPORTED", -3: "CUDA", -4: "DEVICE", -5: "WORKSPACE"}


class FP8Error(RuntimeError):
    def __init__(self, code: int, func: str, msg: str):
        super().__init__(f"{func} failed ({ERRORS.get(code, code)}): {msg}")
        self.code = code


class fp8_ring_t(Structure):
    _fields_ = [("state", c_void_p), ("hist_len", c_int), ("hist_idx", c_int),
                ("fp8_max", c_float), ("pow2_margin", c_float)]


_P = c_void_p
_SIGNATURES = {
    "fp8_scale_ring_init": (c_int, [_P, c_int, _P]),
    "fp8_scale_ring_seed": (c_int, [POINTER(fp8_ring_t), _P, c_int, c_int64, _P]),
    "fp8_amax_scale": (c_int, [_P, c_int, c_int64, c_float, c_float, _P, _P, _P, _P]),
    "fp8_quantize": (c_int, [_P, c_int, c_int64, c_int64, _P, c_int, c_int, _P, _P, POINTER(fp8_ring_t), _P]),
    "fp8_quantize_dual": (c_int, [_P, c_int, c_int64, c_int64, _P, c_int, _P, _P, _P, POINTER(fp8_ring_t), _P]),
    "fp8_gemm": (c_int, [_P, _P, c_int, c_int, c_int, c_int64, c_int64, c_int64, c_int64, c_int64, c_int64,
                         c_int64, c_int64, c_int64, c_int64, _P, _P, _P, _P, _P, _P]),
    "fp8_gemm_fp8out": (c_int, [_P, _P, c_int, c_int, c_int, c_int64, c_int64, c_int64, c_int64, c_int64, c_int64,
                                c_int64, c_int64, c_int64, c_int64, _P, _P, _P, _P, _P, c_int, _P, _P, _P, _P, _P]),
    "linear_forward_fp8_workspace_size": (c_size_t, [c_int64, c_int64, c_int64]),
    "linear_forward_fp8": (c_int, [_P, _P, c_int, _P, _P, _P, c_int64, c_int64, c_int64, c_int,
                                   POINTER(fp8_ring_t), POINTER(fp8_ring_t), c_float, _P, _P, _P, c_size_t, _P, _P]),
    "linear_forward_fp8_noalloc": (c_int, [_P, _P, c_int, _P, _P, _P, c_int64, c_int64, c_int64, c_int,
                                           POINTER(fp8_ring_t), POINTER(fp8_ring_t), c_float, _P, _P, _P, _P]),
    "linear_backward_fp8_workspace_size": (c_size_t, [c_int64, c_int64, c_int64]),
    "linear_backward_fp8": (c_int, [_P, _P, _P, c_int64, c_int64, c_int64, c_int, c_int, c_int, c_int, _P, _P,
                                    POINTER(fp8_ring_t), c_float, _P, _P, c_size_t, _P, _P, _P, _P]),
    "linear_backward_fp8_prequant": (c_int, [_P, c_int, _P, _P, c_int, _P, c_int, c_int64, c_int64, c_int64, c_int,
                                             c_int, c_int, c_int, _P, _P, POINTER(fp8_ring_t), c_float, _P, _P,
                                             c_size_t, _P, _P, _P, _P]),
    "linear_forward_fp8_keep": (c_int, [_P, _P, c_int, _P, _P, _P, c_int64, c_int64, c_int64, c_int,
                                        POINTER(fp8_ring_t), POINTER(fp8_ring_t), c_float, _P, _P, _P, _P, _P,
                                        c_size_t, _P, _P]),
    "linear_backward_fp8_mixed_workspace_size": (c_size_t, [c_int64, c_int64, c_int64]),
    "linear_backward_fp8_mixed": (c_int, [_P, _P, _P, c_int64, c_int64, c_int64, c_int, c_int, c_int, c_int, c_int,
                                          c_int, _P, _P, POINTER(fp8_ring_t), c_float, _P, _P, c_size_t, _P, _P, _P,
                                          _P]),
    "linear_forward_fp8_save_t": (c_int, [_P, _P, _P, _P, c_int64, c_int64, c_int64, c_int, c_int,
                                          POINTER(fp8_ring_t), POINTER(fp8_ring_t), _P, _P, _P, _P, _P, c_size_t,
                                          _P, _P]),
    "linear_forward_fp8_save_rm": (c_int, [_P, _P, _P, _P, c_int64, c_int64, c_int64, c_int, c_int,
                                           POINTER(fp8_ring_t), POINTER(fp8_ring_t), _P, _P, _P, _P, _P, c_size_t,
                                           _P, _P]),
    "linear_backward_fp8_saved_t_workspace_size": (c_size_t, [c_int64, c_int64, c_int64]),
    "linear_backward_fp8_saved_t": (c_int, [_P, _P, _P, c_int64, c_int64, c_int64, c_int, c_int, c_int, c_int, c_int,
                                            _P, _P, POINTER(fp8_ring_t), c_float, _P, _P, c_size_t, _P, _P, _P,
                                            _P]),
    "fp8_get_device_status": (c_int, [_P, POINTER(c_int)]),
    "fp8_set_wait_timeout_ns": (c_int, [c_uint64]),
    "fp8_debug_stalled_wait": (c_int, [_P]),
    "fp8_set_pdl": (c_int, [c_int]),
    "fp8_set_tiled_persist_threshold": (c_int, [c_int64]),
    "fp8_set_gemm_split_k": (c_int, [c_int]),
    "fp8_set_ring_fold_mode": (c_int, [c_int]),
    "fp8_scale_ring_collect_amax": (c_int, [POINTER(fp8_ring_t), c_int, _P, _P]),
    "fp8_scale_ring_fold": (c_int, [POINTER(fp8_ring_t), c_int, _P, _P]),
    "fp8_profiler_enable": (c_int, [c_int]),
    "fp8_profiler_read": (c_int, [c_int, POINTER(c_double), POINTER(c_int64), POINTER(c_double)]),
    "fp8_last_error": (c_char_p, []),
    "fp8dsa_version": (c_char_p, []),
}

_lib = None


def lib() -> ctypes.CDLL:
    """Load the library (once).  Raises if it has not been built -- there is no fallback."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"{LIB_PATH} is missing: build it with "
                              "`python -m fp8_delayed_scaling_amax_b200.build`")
        handle = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in _SIGNATURES.items():
            fn = getattr(handle, name)
            fn.restype = res
            fn.argtypes = args
        _lib = handle
    return _lib


def header_functions():
    """Names of the functions ``include/fp8dsa.h`` declares (parsed from the header text)."""
    with open(HEADER_PATH) as f:
        text = f.read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"^\s*(?:const\s+)?(?:int|size_t|char\s*\*|const char\s*\*)\s*\**\s*(\w+)\s*\(",
                                 text, flags=re.M)))


def _ptr(t):
    if t is None:
        return None
    if isinstance(t, int):
        return t
    if hasattr(t, "data_ptr"):
        return t.data_ptr()
    raise TypeError(f"expected a tensor, an int pointer or None, got {type(t)}")


def _stream(stream):
    if stream is not None:
        return stream if isinstance(stream, int) else stream.cuda_stream
    import torch
    return torch.cuda.current_stream().cuda_stream


def _ring(r):
    if r is None:
        return None
    if isinstance(r, fp8_ring_t):
        return ctypes.byref(r)
    return ctypes.byref(r.as_c())


def _check(name, rc):
    if rc != 0:
        raise FP8Error(rc, name, last_error())
    return rc


def last_error() -> str:
    return lib().fp8_last_error().decode()


def fp8dsa_version() -> str:
    return lib().fp8dsa_version().decode()


fp8_last_error = last_error


class Ring:
    """Host handle of one operand's history ring: the device ``state`` buffer
    (``hist_len + 4`` fp32) plus the host-side slot index, advanced after each use."""

    def __init__(self, state, hist_len: int, fmt: int = FP8_E4M3, margin: int = 0):
        self.state = state
        self.hist_len = int(hist_len)
        self.hist_idx = 0
        self.fp8_max = FP8_MAX[fmt]
        self.pow2_margin = float(2.0 ** margin)

    def as_c(self) -> fp8_ring_t:
        return fp8_ring_t(_ptr(self.state), self.hist_len, self.hist_idx, self.fp8_max, self.pow2_margin)

    def advance(self) -> None:
        self.hist_idx = (self.hist_idx + 1) % self.hist_len


def fp8_scale_ring_init(state, hist_len, stream=None):
    return _check("fp8_scale_ring_init", lib().fp8_scale_ring_init(_ptr(state), int(hist_len), _stream(stream)))


def fp8_scale_ring_seed(ring, x, in_type, numel, stream=None):
    return _check("fp8_scale_ring_seed",
                  lib().fp8_scale_ring_seed(_ring(ring), _ptr(x), int(in_type), int(numel), _stream(stream)))


def fp8_amax_scale(x, in_type, numel, fp8_max, pow2_margin, scale_out, amax_out, scratch, stream=None):
    return _check("fp8_amax_scale", lib().fp8_amax_scale(_ptr(x), int(in_type), int(numel), float(fp8_max),
                                                         float(pow2_margin), _ptr(scale_out), _ptr(amax_out),
                                                         _ptr(scratch), _stream(stream)))


def fp8_quantize(x, in_type, rows, cols, scale, fmt, transposed, out, amax_out=None, ring=None, stream=None):
    return _check("fp8_quantize", lib().fp8_quantize(_ptr(x), int(in_type), int(rows), int(cols), _ptr(scale),
                                                     int(fmt), int(bool(transposed)), _ptr(out), _ptr(amax_out),
                                                     _ring(ring), _stream(stream)))


def fp8_quantize_dual(x, in_type, rows, cols, scale, fmt, out, out_t, amax_out=None, ring=None, stream=None):
    return _check("fp8_quantize_dual", lib().fp8_quantize_dual(_ptr(x), int(in_type), int(rows), int(cols),
                                                               _ptr(scale), int(fmt), _ptr(out), _ptr(out_t),
                                                               _ptr(amax_out), _ring(ring), _stream(stream)))


def fp8_gemm(a, b, fmt_a, fmt_b, layout, m, n, k, lda, ldb, ldo, batch, stride_a, stride_b, stride_o,
             scale_a, scale_b, bias, bias_scale, out, stream=None):
    return _check("fp8_gemm", lib().fp8_gemm(_ptr(a), _ptr(b), int(fmt_a), int(fmt_b), int(layout), int(m), int(n),
                                             int(k), int(lda), int(ldb), int(ldo), int(batch), int(stride_a),
                                             int(stride_b), int(stride_o), _ptr(scale_a), _ptr(scale_b), _ptr(bias),
                                             _ptr(bias_scale), _ptr(out), _stream(stream)))


def fp8_gemm_fp8out(a, b, fmt_a, fmt_b, layout, m, n, k, lda, ldb, ldo, batch, stride_a, stride_b, stride_o,
                    scale_a, scale_b, bias, bias_scale, out, out8_fmt, out8_step, out8, out8_amax=None,
                    out8_step_used=None, stream=None):
    return _check("fp8_gemm_fp8out", lib().fp8_gemm_fp8out(
        _ptr(a), _ptr(b), int(fmt_a), int(fmt_b), int(layout), int(m), int(n), int(k), int(lda), int(ldb), int(ldo),
        int(batch), int(stride_a), int(stride_b), int(stride_o), _ptr(scale_a), _ptr(scale_b), _ptr(bias),
        _ptr(bias_scale), _ptr(out), int(out8_fmt), _ptr(out8_step), _ptr(out8), _ptr(out8_amax),
        _ptr(out8_step_used), _stream(stream)))


def linear_forward_fp8_workspace_size(m, k, n) -> int:
    return int(lib().linear_forward_fp8_workspace_size(int(m), int(k), int(n)))


def linear_backward_fp8_workspace_size(m, k, n) -> int:
    return int(lib().linear_backward_fp8_workspace_size(int(m), int(k), int(n)))


def linear_forward_fp8(x, w, w_is_fp8, w_step, bias, bias_scale, m, k, n, fmt, x_ring, w_ring, pow2_margin,
                       sx_used, sw_used, workspace, workspace_bytes, y, stream=None):
    return _check("linear_forward_fp8", lib().linear_forward_fp8(
        _ptr(x), _ptr(w), int(bool(w_is_fp8)), _ptr(w_step), _ptr(bias), _ptr(bias_scale), int(m), int(k), int(n),
        int(fmt), _ring(x_ring), _ring(w_ring), float(pow2_margin), _ptr(sx_used), _ptr(sw_used), _ptr(workspace),
        int(workspace_bytes), _ptr(y), _stream(stream)))


def linear_forward_fp8_noalloc(x, w, w_is_fp8, w_step, bias, bias_scale, m, k, n, fmt, x_ring, w_ring, pow2_margin,
                               sx_used, sw_used, y, stream=None):
    """linear_forward_fp8 with the library's built-in scratch array instead of a workspace,
    for callers that cannot allocate device memory."""
    return _check("linear_forward_fp8_noalloc", lib().linear_forward_fp8_noalloc(
        _ptr(x), _ptr(w), int(bool(w_is_fp8)), _ptr(w_step), _ptr(bias), _ptr(bias_scale), int(m), int(k), int(n),
        int(fmt), _ring(x_ring), _ring(w_ring), float(pow2_margin), _ptr(sx_used), _ptr(sw_used), _ptr(y),
        _stream(stream)))


NOALLOC_WORKSPACE_BYTES = 16 << 20


def linear_backward_fp8(g, x, w, m, k, n, fmt, need_grad_x, need_grad_w, need_grad_b, sx_fwd, sw_fwd, g_ring,
                        pow2_margin, sg_used, workspace, workspace_bytes, grad_x, grad_w, grad_b, stream=None):
    return _check("linear_backward_fp8", lib().linear_backward_fp8(
        _ptr(g), _ptr(x), _ptr(w), int(m), int(k), int(n), int(fmt), int(bool(need_grad_x)), int(bool(need_grad_w)),
        int(bool(need_grad_b)), _ptr(sx_fwd), _ptr(sw_fwd), _ring(g_ring), float(pow2_margin), _ptr(sg_used),
        _ptr(workspace), int(workspace_bytes), _ptr(grad_x), _ptr(grad_w), _ptr(grad_b), _stream(stream)))


def linear_backward_fp8_prequant(g, g_is_fp8, g_step, x, x_is_fp8, w, w_is_fp8, m, k, n, fmt, need_grad_x,
                                 need_grad_w, need_grad_b, sx_fwd, sw_fwd, g_ring, pow2_margin, sg_used, workspace,
                                 workspace_bytes, grad_x, grad_w, grad_b, stream=None):
    """linear_backward_fp8 where g / x / w may each be fp8 bytes in fmt (flags *_is_fp8)."""
    return _check("linear_backward_fp8_prequant", lib().linear_backward_fp8_prequant(
        _ptr(g), int(bool(g_is_fp8)), _ptr(g_step), _ptr(x), int(bool(x_is_fp8)), _ptr(w), int(bool(w_is_fp8)),
        int(m), int(k), int(n), int(fmt), int(bool(need_grad_x)), int(bool(need_grad_w)), int(bool(need_grad_b)),
        _ptr(sx_fwd), _ptr(sw_fwd), _ring(g_ring), float(pow2_margin), _ptr(sg_used), _ptr(workspace),
        int(workspace_bytes), _ptr(grad_x), _ptr(grad_w), _ptr(grad_b), _stream(stream)))


def linear_forward_fp8_keep(x, w, w_is_fp8, w_step, bias, bias_scale, m, k, n, fmt, x_ring, w_ring, pow2_margin,
                            sx_used, sw_used, x8_out, w8_out, workspace, workspace_bytes, y, stream=None):
    """linear_forward_fp8 that also leaves the quantized operands in x8_out / w8_out (for
    linear_backward_fp8_mixed)."""
    return _check("linear_forward_fp8_keep", lib().linear_forward_fp8_keep(
        _ptr(x), _ptr(w), int(bool(w_is_fp8)), _ptr(w_step), _ptr(bias), _ptr(bias_scale), int(m), int(k), int(n),
        int(fmt), _ring(x_ring), _ring(w_ring), float(pow2_margin), _ptr(sx_used), _ptr(sw_used), _ptr(x8_out),
        _ptr(w8_out), _ptr(workspace), int(workspace_bytes), _ptr(y), _stream(stream)))


def linear_backward_fp8_mixed_workspace_size(m, k, n) -> int:
    return int(lib().linear_backward_fp8_mixed_workspace_size(int(m), int(k), int(n)))


def linear_backward_fp8_mixed(g, x8, w8, m, k, n, fmt_g, fmt_x, fmt_w, need_grad_x, need_grad_w, need_grad_b, sx,
                              sw, g_ring, pow2_margin, sg_used, workspace, workspace_bytes, grad_x, grad_w, grad_b,
                              stream=None):
    return _check("linear_backward_fp8_mixed", lib().linear_backward_fp8_mixed(
        _ptr(g), _ptr(x8), _ptr(w8), int(m), int(k), int(n), int(fmt_g), int(fmt_x), int(fmt_w),
        int(bool(need_grad_x)), int(bool(need_grad_w)), int(bool(need_grad_b)), _ptr(sx), _ptr(sw), _ring(g_ring),
        float(pow2_margin), _ptr(sg_used), _ptr(workspace), int(workspace_bytes), _ptr(grad_x), _ptr(grad_w),
        _ptr(grad_b), _stream(stream)))


def linear_forward_fp8_save_t(x, w, bias, bias_scale, m, k, n, fmt, fmt_t, x_ring, w_ring, sx_used, sw_used, x8t_out,
                              w8t_out, workspace, workspace_bytes, y, stream=None):
    """Delayed-scaling forward that also writes x^T / w^T in fmt_t (for
    linear_backward_fp8_saved_t)."""
    return _check("linear_forward_fp8_save_t", lib().linear_forward_fp8_save_t(
        _ptr(x), _ptr(w), _ptr(bias), _ptr(bias_scale), int(m), int(k), int(n), int(fmt), int(fmt_t), _ring(x_ring),
        _ring(w_ring), _ptr(sx_used), _ptr(sw_used), _ptr(x8t_out), _ptr(w8t_out), _ptr(workspace),
        int(workspace_bytes), _ptr(y), _stream(stream)))


def linear_forward_fp8_save_rm(x, w, bias, bias_scale, m, k, n, fmt, fmt_b, x_ring, w_ring, sx_used, sw_used,
                               x8b_out, w8b_out, workspace, workspace_bytes, y, stream=None):
    """Delayed-scaling forward that also writes x and w row-major in fmt_b (for
    linear_backward_fp8_mixed with every format fmt_b)."""
    return _check("linear_forward_fp8_save_rm", lib().linear_forward_fp8_save_rm(
        _ptr(x), _ptr(w), _ptr(bias), _ptr(bias_scale), int(m), int(k), int(n), int(fmt), int(fmt_b), _ring(x_ring),
        _ring(w_ring), _ptr(sx_used), _ptr(sw_used), _ptr(x8b_out), _ptr(w8b_out), _ptr(workspace),
        int(workspace_bytes), _ptr(y), _stream(stream)))


def linear_backward_fp8_saved_t_workspace_size(m, k, n) -> int:
    return int(lib().linear_backward_fp8_saved_t_workspace_size(int(m), int(k), int(n)))


def linear_backward_fp8_saved_t(g, x8t, w8t, m, k, n, fmt, fmt_t, need_grad_x, need_grad_w, need_grad_b, sx, sw,
                                g_ring, pow2_margin, sg_used, workspace, workspace_bytes, grad_x, grad_w, grad_b,
                                stream=None):
    return _check("linear_backward_fp8_saved_t", lib().linear_backward_fp8_saved_t(
        _ptr(g), _ptr(x8t), _ptr(w8t), int(m), int(k), int(n), int(fmt), int(fmt_t), int(bool(need_grad_x)),
        int(bool(need_grad_w)), int(bool(need_grad_b)), _ptr(sx), _ptr(sw), _ring(g_ring), float(pow2_margin),
        _ptr(sg_used), _ptr(workspace), int(workspace_bytes), _ptr(grad_x), _ptr(grad_w), _ptr(grad_b),
        _stream(stream)))


def fp8_get_device_status(stream=None) -> int:
    v = c_int(0)
    _check("fp8_get_device_status", lib().fp8_get_device_status(_stream(stream), ctypes.byref(v)))
    return v.value


def fp8_set_wait_timeout_ns(ns: int):
    return _check("fp8_set_wait_timeout_ns", lib().fp8_set_wait_timeout_ns(int(ns)))


def fp8_set_pdl(enabled: bool = True):
    return _check("fp8_set_pdl", lib().fp8_set_pdl(int(bool(enabled))))


def _ring_array(rings):
    arr = (fp8_ring_t * max(1, len(rings)))()
    for i, r in enumerate(rings):
        arr[i] = r.as_c() if isinstance(r, Ring) else r
    return arr


def fp8_scale_ring_collect_amax(rings, amax_out, stream=None):
    """amax_out[i] = ring i's amax slot (dev fp32 tensor of len(rings))."""
    return _check("fp8_scale_ring_collect_amax", lib().fp8_scale_ring_collect_amax(
        _ring_array(rings), len(rings), _ptr(amax_out), _stream(stream)))


def fp8_scale_ring_fold(rings, amax=None, stream=None):
    """Fold every ring with amax[i] (or its own amax slot when amax is None)."""
    return _check("fp8_scale_ring_fold", lib().fp8_scale_ring_fold(
        _ring_array(rings), len(rings), _ptr(amax), _stream(stream)))


def fp8_set_ring_fold_mode(mode: int = 0):
    return _check("fp8_set_ring_fold_mode", lib().fp8_set_ring_fold_mode(int(mode)))


def fp8_set_gemm_split_k(splits: int = 1):
    return _check("fp8_set_gemm_split_k", lib().fp8_set_gemm_split_k(int(splits)))


def fp8_set_tiled_persist_threshold(min_tiles: int = 1024):
    return _check("fp8_set_tiled_persist_threshold", lib().fp8_set_tiled_persist_threshold(int(min_tiles)))


def fp8_debug_stalled_wait(stream=None):
    return _check("fp8_debug_stalled_wait", lib().fp8_debug_stalled_wait(_stream(stream)))


def fp8_profiler_enable(on: bool = True):
    return _check("fp8_profiler_enable", lib().fp8_profiler_enable(int(bool(on))))


def fp8_profiler_read(kind: int):
    """(total device ms, launches, algorithmic bytes or flops) of one kernel class since the last read."""
    ms, n, work = c_double(0), c_int64(0), c_double(0)
    _check("fp8_profiler_read", lib().fp8_profiler_read(int(kind), ctypes.byref(ms), ctypes.byref(n),
                                                        ctypes.byref(work)))
    return ms.value, n.value, work.value
