"""Oracle FP8 x FP8 GEMM with dequantization and fused bias.

Test infrastructure only (see ``oracle/__init__.py``).

What the pages fix (AstrAI compare view):

* ``astrai/extension/ops/fp8.py``, ``mm_fp8``: ``a @ b * scale (+ bias)`` over fp8
  operands, fp32 accumulation, bf16 result; 2-D or 3-D with matmul-style batch
  broadcast; ``scale`` is the product of the two operands' steps, formed in fp32
  (``sx * sw`` in ``fp8_linear_forward``).
* ``csrc/kernels/fp8/gemm/epilogue.cuh``: the bias is added to the fp32
  accumulator before the single bf16 rounding.
* ``csrc/kernels/fp8/common.h``: layout tags -- A RowMajor ``[M][K]``, A ColMajor
  ``[K][M]``, B RowMajor ``[K][N]``, B ColMajor ``[N][K]`` (the nn.Linear weight).
  Here the first letter of the layout names A (``N`` = ``[M][K]``, ``T`` =
  ``[K][M]``) and the second names B (``T`` = ``[N][K]``, ``N`` = ``[K][N]``), so the
  training layout x8 @ w8^T is ``NT``.
* The extension commit log: a non-null ``bias_scale`` means the bias is stored as
  fp8 and dequantized in the epilogue after the operand scaling.

The oracle decodes the bytes exactly, forms ``sum_k a*b`` with an fp64 matrix
product, multiplies by ``RN32(sa*sb)`` and adds the bias, all in fp64, and
returns that *unrounded* value plus ``S_abs = sum_k |a*b|``.  For E4M3 operands and
K <= 8192 every partial sum is an integer multiple of 2^-18 below 2^31, so the fp64
product is exact in any summation order; for E5M2 its rounding error is far below
the bound the comparison uses:

    |gpu - ref| <= 2^-8 |ref| + 2^-20 * S_abs * RN32(sa*sb)
"""

from __future__ import annotations

import numpy as np

from .fp8_codec import decode, round_to_bf16, bf16_bits_to_f64

LAYOUTS = ("NT", "NN", "TN", "TT")

REL_TOL = 2.0 ** -8
ACC_TOL = 2.0 ** -20


def canonical_operands(a_stored, b_stored, layout: str, fmt_a, fmt_b):
    """Decode stored fp8 bytes and return canonical fp64 ``A [.., M, K]``, ``B [.., K, N]``."""
    layout = layout.upper()
    assert layout in LAYOUTS
    a = decode(a_stored, fmt_a)
    b = decode(b_stored, fmt_b)
    if layout[0] == "T":
        a = np.swapaxes(a, -1, -2)
    if layout[1] == "T":
        b = np.swapaxes(b, -1, -2)
    return a, b


def combined_scale(sa, sb) -> np.float32:
    """``RN32(sa * sb)`` -- the single dequantization multiplier."""
    return np.float32(sa) * np.float32(sb)


def bias_values(bias, bias_scale=None, bias_fmt="e4m3") -> np.ndarray:
    """The bias as exact fp64 values: bf16 bits, or fp8 codes times ``bias_scale``."""
    if bias is None:
        return None
    if bias_scale is None:
        return bf16_bits_to_f64(bias)
    return decode(bias, bias_fmt) * np.float64(np.float32(bias_scale))


def gemm_ref(a_stored, b_stored, layout="NT", fmt_a="e4m3", fmt_b="e4m3",
             sa=1.0, sb=1.0, bias=None, bias_scale=None):
    """Return ``(ref64, s_abs, sc)`` for ``out = (A @ B) * RN32(sa*sb) + bias``.

    ``a_stored`` / ``b_stored`` are uint8 arrays in their stored layout, 2-D or
    3-D; a batch dimension of 1 broadcasts.  ``bias`` is uint16 bf16 bits (or
    uint8 fp8 codes when ``bias_scale`` is given, in ``fmt_a``).
    """
    a, b = canonical_operands(a_stored, b_stored, layout, fmt_a, fmt_b)
    acc = np.matmul(a, b)
    s_abs = np.matmul(np.abs(a), np.abs(b))
    sc = combined_scale(sa, sb)
    ref = acc * np.float64(sc)
    bv = bias_values(bias, bias_scale, fmt_a)
    if bv is not None:
        ref = ref + bv
    return ref, s_abs, sc


def gemm_tolerance(ref64, s_abs, sc):
    """Per-element bound ``2^-8 |ref| + 2^-20 * S_abs * sc``."""
    return REL_TOL * np.abs(ref64) + ACC_TOL * s_abs * np.float64(sc)


def gemm_bf16(a_stored, b_stored, **kw) -> np.ndarray:
    """The oracle's bf16 output: ``RN_bf16`` of the unrounded fp64 result."""
    ref, _, _ = gemm_ref(a_stored, b_stored, **kw)
    return round_to_bf16(ref)


def gemm_entry(a_stored, b_stored, layout, fmt_a, fmt_b, sa, sb, bias, bias_scale,
               batch_index, i, j):
    """One output element ``(ref64, s_abs)`` computed on its own (for sampled
    checks at sizes where the full product is too slow)."""
    a, b = canonical_operands(a_stored, b_stored, layout, fmt_a, fmt_b)
    if a.ndim == 3:
        a = a[batch_index if a.shape[0] > 1 else 0]
    if b.ndim == 3:
        b = b[batch_index if b.shape[0] > 1 else 0]
    row = a[i, :]
    col = b[:, j]
    prod = row * col
    sc = combined_scale(sa, sb)
    ref = float(np.sum(prod)) * float(sc)
    bv = bias_values(bias, bias_scale, fmt_a)
    if bv is not None:
        ref += float(bv[j])
    return ref, float(np.sum(np.abs(prod))), sc


def gemm_fp8_out(a_stored, b_stored, layout="NT", fmt_a="e4m3", fmt_b="e4m3", sa=1.0, sb=1.0,
                 bias=None, bias_scale=None, out8_fmt="e4m3", out8_step=1.0):
    """The GEMM whose epilogue also quantizes its output (the FP8-output GEMM of an earlier
    state of the pages' epilogue, read as "quantize the bf16 output"): ``y = RN_bf16(ref)``
    as in :func:`gemm_bf16`, then ``out8 = q(RN32(y * RN32(1/out8_step)))`` and
    ``amax = max |y|`` -- the same bytes and amax the quantize gives for ``y``.

    Returns ``(ref64, s_abs, sc, y_bits, out8_codes, amax)``."""
    from .fp8_codec import f64_to_bf16_bits, bf16_bits_to_f64
    from .quantize import amax as amax_of, quantize_values
    ref, s_abs, sc = gemm_ref(a_stored, b_stored, layout, fmt_a, fmt_b, sa, sb, bias, bias_scale)
    y_bits = f64_to_bf16_bits(ref)
    y = bf16_bits_to_f64(y_bits).astype(np.float32)
    return ref, s_abs, sc, y_bits, quantize_values(y, out8_step, out8_fmt), amax_of(y)
