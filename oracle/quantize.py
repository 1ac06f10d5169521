"""Oracle quantize: fp8 bytes and raw-domain amax.

Test infrastructure only (see ``oracle/__init__.py``).

What the pages fix (AstrAI compare view):

* ``astrai/extension/fp8.py`` (``fp8_linear_forward``, ``_LinearFp8.backward``):
  a *scale* is the quantization step; the kernel is handed its reciprocal
  (``quantize(x, sx.reciprocal(), ...)``) and multiplies by it.
* ``csrc/kernels/fp8/quantize.cuh`` (``fp8_quantize_kernel``): each element is
  converted to float, multiplied by the multiplier in fp32, and converted to fp8
  with round-to-nearest-even and saturation; amax is ``fmaxf(fabsf(v))`` over the
  *unscaled* values (the extension commit log records the bug where the quantized
  max was used instead).
* ``fp8_quantize_tiled_kernel``: the transposed output is the ``[cols][rows]``
  row-major transpose of the same bytes; the dual mode writes both.

Readings: the multiplier is the correctly rounded fp32 reciprocal ``RN32(1/s)``;
amax starts at 0 and ignores NaN (``fmaxf`` semantics).
"""

from __future__ import annotations

import numpy as np

from .fp8_codec import encode


def reciprocal_f32(s) -> np.float32:
    """RN32(1/s): IEEE single-precision division."""
    return np.float32(1.0) / np.float32(s)


def amax(x: np.ndarray) -> np.float32:
    """max |x| over the raw values, NaN ignored, 0 for an empty tensor."""
    x = np.asarray(x, dtype=np.float32)
    if x.size == 0:
        return np.float32(0.0)
    return np.float32(np.fmax.reduce(np.abs(x).ravel(), initial=np.float32(0.0)))


def quantize_values(x: np.ndarray, scale, fmt) -> np.ndarray:
    """uint8 codes of ``q_fmt(RN32(x * RN32(1/scale)))``, same shape as ``x``.

    ``x`` holds the input values as fp32 (bf16 / fp16 inputs convert exactly).
    """
    x = np.asarray(x, dtype=np.float32)
    mult = reciprocal_f32(scale)
    y = x * mult  # one fp32 product, rounded to nearest even by IEEE rules
    assert y.dtype == np.float32
    return encode(y, fmt)


def quantize(x: np.ndarray, scale, fmt):
    """Row-major quantize of a 2-D (or flat) tensor: ``(x8, amax)``."""
    return quantize_values(x, scale, fmt), amax(x)


def quantize_transposed(x: np.ndarray, scale, fmt):
    """``(x8T, amax)`` with ``x8T[c][r] = q(x[r][c])``."""
    x = np.asarray(x, dtype=np.float32)
    assert x.ndim == 2
    return np.ascontiguousarray(quantize_values(x, scale, fmt).T), amax(x)


def quantize_dual(x: np.ndarray, scale, fmt):
    """``(x8, x8T, amax)`` -- both orientations from one input."""
    x8, a = quantize(x, scale, fmt)
    return x8, np.ascontiguousarray(x8.T), a
