"""Oracle FP8 linear layer: forward, dX and dW, delayed or dynamic scaling.

Test infrastructure only (see ``oracle/__init__.py``).

What the pages fix (AstrAI compare view, ``astrai/extension/fp8.py``):

* ``fp8_linear_forward``: delayed scaling snapshots ``sx, sw`` from the rings
  before the quantize kernels fold the fresh amax and publish the next step;
  the GEMM dequantizes with ``sx * sw`` and fuses the bias.  Dynamic scaling
  measures the current amax of x and w first, with no ring.
* ``_LinearFp8.backward``: g is quantized once in both orientations
  (``quantize_dual``, folding into the g ring); x and w are re-quantized
  *transposed* with the forward's steps (no ring, amax discarded);
  ``grad_x = g8 @ w8T^T * (sg*sw)`` and ``grad_w = g8T @ x8T^T * (sg*sx)`` both in
  the NT layout; ``grad_b = g.sum(0)``.  Dynamic backward re-measures g, w and x.
* ``FP8Format.HYBRID``: E4M3 forward, E5M2 backward; the backward GEMM takes both
  operands in one format, so x and w are re-quantized to E5M2 as well.

* Reuse of the forward's operands (the C++ binding of the linear backward in an
  earlier state of the compare view): x or w already quantized by the forward is
  passed as fp8 and its quantize kernel is skipped; its forward step still
  dequantizes the GEMM.  There the reused bytes had to share the backward's
  format.

* Pre-quantized operands (the ``astrai/extension`` commit log and the binding's
  docstrings in the compare view): ``linear_forward_fp8`` takes a weight that is
  already fp8 in the forward's format, skips its quantize and reports
  ``amax_w = 0``; the bias may be fp8 too, with ``bias_scale`` (dequantized after
  the operand scaling).  ``linear_backward_fp8`` takes g, x and w each as bf16 or
  as fp8 in the backward's format: a pre-quantized operand skips its quantize and
  is read by the GEMM as it is; a pre-quantized g does not fold the g ring,
  reports ``amax_g = 0`` and is dequantized before the bias-gradient sum.

Readings: ``grad_b`` is the fp64 column sum rounded once to bf16; the gradient
outputs are returned unrounded (fp64) for the bound check.  ``backward_mixed``
reads the operand reuse with independent formats (the tensor core takes A and B
formats separately): the forward's E4M3 x8 / w8 with an E5M2 g8.  A pre-quantized
operand arrives with the step its bytes were quantized at: ``w_step`` for the
forward's weight, ``g_step`` for g, and the forward's ``sx`` / ``sw`` for x / w in
the backward (the pages pass those steps next to the operands).
"""

from __future__ import annotations

import numpy as np

from .fp8_codec import bf16_bits_to_f64, decode, round_to_bf16
from .gemm import gemm_ref
from .quantize import quantize, quantize_dual, quantize_transposed
from .scaling import Ring, dynamic_scale


def forward(x_bits, w_bits, bias_bits=None, fmt="e4m3", ring_x: Ring = None,
            ring_w: Ring = None, margin: int = 0, *, w8=None, w_step=None, bias_scale=None):
    """Returns a dict with ``y`` (fp64, unrounded), ``s_abs``, ``sc``, ``x8``, ``w8``,
    ``sx``, ``sw``, ``amax_x``, ``amax_w``.  Rings (if given) are folded in place;
    the caller advances them afterwards, as the pages' host code does.

    Pre-quantized weight: pass ``w8`` (fp8 codes ``[n, k]`` in ``fmt``) and its step
    ``w_step`` instead of ``w_bits``; no weight quantize runs, ``ring_w`` is neither
    read nor folded, and ``amax_w`` is 0.  fp8 bias: ``bias_bits`` holds fp8 codes
    in ``fmt`` and ``bias_scale`` their step."""
    xv = bf16_bits_to_f64(x_bits).astype(np.float32)
    prequant_w = w8 is not None
    dynamic = ring_x is None
    if dynamic:
        sx = dynamic_scale(xv, fmt, margin)
    else:
        sx = np.float32(ring_x.scale)
    if prequant_w:
        assert w_step is not None, "a pre-quantized weight needs its step"
        sw = np.float32(w_step)
        w8 = np.asarray(w8, dtype=np.uint8)
        aw = np.float32(0.0)
    else:
        wv = bf16_bits_to_f64(w_bits).astype(np.float32)
        sw = dynamic_scale(wv, fmt, margin) if dynamic else np.float32(ring_w.scale)
    x8, ax = quantize(xv, sx, fmt)
    if not prequant_w:
        w8, aw = quantize(wv, sw, fmt)
    if not dynamic:
        ring_x.fold(ax, sx)
        if not prequant_w:
            ring_w.fold(aw, sw)
    y, s_abs, sc = gemm_ref(x8, w8, "NT", fmt, fmt, sx, sw, bias_bits, bias_scale)
    return dict(y=y, s_abs=s_abs, sc=sc, x8=x8, w8=w8, sx=sx, sw=sw,
                amax_x=ax, amax_w=aw)


def backward(g_bits, x_bits, w_bits, fmt="e5m2", sx_fwd=None, sw_fwd=None,
             ring_g: Ring = None, margin: int = 0):
    """Returns a dict with ``dx``, ``dw`` (fp64, unrounded) and their ``s_abs``/``sc``,
    ``grad_b`` (bf16 values), the quantized operands and the steps used."""
    gv = bf16_bits_to_f64(g_bits).astype(np.float32)
    xv = bf16_bits_to_f64(x_bits).astype(np.float32)
    wv = bf16_bits_to_f64(w_bits).astype(np.float32)
    dynamic = ring_g is None
    if dynamic:
        sg = dynamic_scale(gv, fmt, margin)
        sw = dynamic_scale(wv, fmt, margin)
        sx = dynamic_scale(xv, fmt, margin)
    else:
        sg = np.float32(ring_g.scale)
        sx, sw = np.float32(sx_fwd), np.float32(sw_fwd)
    g8, g8t, ag = quantize_dual(gv, sg, fmt)
    if not dynamic:
        ring_g.fold(ag, sg)
    x8t, _ = quantize_transposed(xv, sx, fmt)
    w8t, _ = quantize_transposed(wv, sw, fmt)
    dx, dx_abs, dx_sc = gemm_ref(g8, w8t, "NT", fmt, fmt, sg, sw)
    dw, dw_abs, dw_sc = gemm_ref(g8t, x8t, "NT", fmt, fmt, sg, sx)
    grad_b = round_to_bf16(np.sum(gv.astype(np.float64), axis=0))
    return dict(dx=dx, dx_abs=dx_abs, dx_sc=dx_sc, dw=dw, dw_abs=dw_abs, dw_sc=dw_sc,
                grad_b=grad_b, g8=g8, g8t=g8t, x8t=x8t, w8t=w8t, sg=sg, sx=sx, sw=sw,
                amax_g=ag)


def backward_mixed(g_bits, x8, w8, fmt_g="e5m2", fmt_x="e4m3", fmt_w="e4m3", sx=None,
                   sw=None, ring_g: Ring = None, margin: int = 0):
    """Backward that reuses the forward's quantized operands as they are.

    ``x8`` [m,k] and ``w8`` [n,k] are the forward's fp8 codes (formats ``fmt_x`` /
    ``fmt_w``, steps ``sx`` / ``sw``).  Only g is quantized, row-major, in ``fmt_g``
    (with ``ring_g``: the ring's step, folded; without: the dynamic step).  Then

    * ``grad_x [m,k] = g8 @ w8 * RN32(sg*sw)``   (layout NN: B = w8 stored [n,k] = [K,N])
    * ``grad_w [n,k] = g8^T @ x8 * RN32(sg*sx)`` (layout TN: A = g8 stored [m,n] = [K,M],
      B = x8 stored [m,k] = [K,N])
    * ``grad_b`` as in :func:`backward`.

    Returns the same keys as :func:`backward` except the re-quantized x8T / w8T."""
    gv = bf16_bits_to_f64(g_bits).astype(np.float32)
    if ring_g is None:
        sg = dynamic_scale(gv, fmt_g, margin)
    else:
        sg = np.float32(ring_g.scale)
    g8, ag = quantize(gv, sg, fmt_g)
    if ring_g is not None:
        ring_g.fold(ag, sg)
    sx, sw = np.float32(sx), np.float32(sw)
    dx, dx_abs, dx_sc = gemm_ref(g8, w8, "NN", fmt_g, fmt_w, sg, sw)
    dw, dw_abs, dw_sc = gemm_ref(g8, x8, "TN", fmt_g, fmt_x, sg, sx)
    grad_b = round_to_bf16(np.sum(gv.astype(np.float64), axis=0))
    return dict(dx=dx, dx_abs=dx_abs, dx_sc=dx_sc, dw=dw, dw_abs=dw_abs, dw_sc=dw_sc,
                grad_b=grad_b, g8=g8, sg=sg, sx=sx, sw=sw, amax_g=ag)


def backward_prequant(g, x, w, fmt="e5m2", g_is_fp8=False, x_is_fp8=False, w_is_fp8=False,
                      g_step=None, sx=None, sw=None, ring_g: Ring = None, margin: int = 0):
    """Backward whose g, x and w may each arrive pre-quantized (fp8 codes in ``fmt``).

    ``g`` [m,n], ``x`` [m,k], ``w`` [n,k] are bf16 bits, or fp8 codes where the
    matching ``*_is_fp8`` flag is set.  Steps:

    * g: bf16 -> quantized at the ring's step (folding ``ring_g``) or, without a ring,
      at the dynamic step; fp8 -> used as it is at ``g_step``, ``ring_g`` untouched,
      ``amax_g`` = 0;
    * x / w: bf16 -> quantized at the forward's ``sx`` / ``sw`` (delayed) or at their
      dynamic steps (no ring); fp8 -> used as they are at ``sx`` / ``sw``;
    * ``grad_x [m,k] = g8 @ w8 * RN32(sg*sw)`` and ``grad_w [n,k] = g8^T @ x8 *
      RN32(sg*sx)`` (the orientation of the stored bytes does not change the values);
    * ``grad_b = RN_bf16(sum over rows of g)``, where a pre-quantized g is first
      dequantized: ``g = dec(g8) * g_step`` in fp64.

    Returns the keys of :func:`backward` (without the transposed copies), with
    ``x8`` / ``w8`` the row-major bytes the GEMMs read."""
    dynamic = ring_g is None
    if g_is_fp8:
        assert g_step is not None, "a pre-quantized g needs its step"
        g8 = np.asarray(g, dtype=np.uint8)
        sg = np.float32(g_step)
        ag = np.float32(0.0)
        g_values = decode(g8, fmt) * np.float64(sg)
    else:
        gv = bf16_bits_to_f64(g).astype(np.float32)
        sg = dynamic_scale(gv, fmt, margin) if dynamic else np.float32(ring_g.scale)
        g8, ag = quantize(gv, sg, fmt)
        if not dynamic:
            ring_g.fold(ag, sg)
        g_values = gv.astype(np.float64)
    operands = {}
    for name, t, is_fp8, step in (("x", x, x_is_fp8, sx), ("w", w, w_is_fp8, sw)):
        if is_fp8:
            assert step is not None, f"a pre-quantized {name} needs its step"
            operands[name] = (np.asarray(t, dtype=np.uint8), np.float32(step))
        else:
            tv = bf16_bits_to_f64(t).astype(np.float32)
            s = dynamic_scale(tv, fmt, margin) if dynamic else np.float32(step)
            operands[name] = (quantize(tv, s, fmt)[0], s)
    x8, sx = operands["x"]
    w8, sw = operands["w"]
    dx, dx_abs, dx_sc = gemm_ref(g8, w8, "NN", fmt, fmt, sg, sw)
    dw, dw_abs, dw_sc = gemm_ref(g8, x8, "TN", fmt, fmt, sg, sx)
    grad_b = round_to_bf16(np.sum(g_values, axis=0))
    return dict(dx=dx, dx_abs=dx_abs, dx_sc=dx_sc, dw=dw, dw_abs=dw_abs, dw_sc=dw_sc,
                grad_b=grad_b, g8=g8, x8=x8, w8=w8, sg=sg, sx=sx, sw=sw, amax_g=ag)
