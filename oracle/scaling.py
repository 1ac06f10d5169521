"""Oracle scale recipe and history ring.

Test infrastructure only (see ``oracle/__init__.py``).

What the pages fix (AstrAI compare view):

* ``astrai/extension/fp8.py``, ``FP8Recipe.scale_from_history``: the step is
  ``(peak / FP8_MAX[fmt]) / 2^margin`` clamped below at ``1e-12``, where ``peak`` is
  the max over the amax history window (delayed, ``dynamic=False``) or the current
  amax (``dynamic=True``).  Defaults: ``history_len=16``, ``margin=0``.
* ``_ScaleRing``: one fp32 buffer per operand, ``[hist n | scale | legacy | amax |
  done]`` (n + 4 floats), zero-initialised; ``idx`` advances host-side after each
  use, ``(idx + 1) % n``; ``seed()`` initialises from the first tensor.
* ``csrc/kernels/fp8/quantize.cuh``, ``publish_amax``: the last block to finish
  writes ``hist[idx] = amax``, takes ``peak`` as the max over all n slots, publishes
  ``scale = fmaxf(peak / fp8_max / pow2_margin, 1e-12f)`` and re-zeroes the amax and
  done slots.

Readings (the pages leave these open):

* The slot the pages call ``legacy`` holds the step the fold's own kernel
  quantized with (``scale_used``), written before the new step is published, so
  the GEMM and the backward can read the snapshot.
* ``seed()``'s body is not on the pages: it writes ``hist[idx] = amax(x)`` and
  publishes the scale with the same fp32 formula as the kernel fold.
* Every division is IEEE fp32 (``RN32``); ``pow2_margin = 2^margin`` exactly.
"""

from __future__ import annotations

import numpy as np

from .fp8_codec import FP8_MAX
from .quantize import amax as amax_of

SCALE_FLOOR = np.float32(1e-12)


def scale_from_peak(peak, fp8_max, pow2_margin=1.0) -> np.float32:
    """``fmaxf(RN32(RN32(peak / fp8_max) / pow2_margin), 1e-12f)``."""
    t = np.float32(peak) / np.float32(fp8_max)
    t = t / np.float32(pow2_margin)
    return np.float32(np.fmax(t, SCALE_FLOOR))


def dynamic_scale(x, fmt, margin: int = 0) -> np.float32:
    """Current-amax scaling (``dynamic=True``): the step from this tensor alone."""
    return scale_from_peak(amax_of(x), FP8_MAX[fmt], 2.0 ** margin)


class Ring:
    """One operand's delayed-scaling state, ``[hist n | scale | scale_used | amax | done]``."""

    def __init__(self, hist_len: int = 16, fmt="e4m3", margin: int = 0):
        assert hist_len >= 1
        self.n = hist_len
        self.fp8_max = np.float32(FP8_MAX[fmt] if isinstance(fmt, str) else FP8_MAX[["e4m3", "e5m2"][fmt]])
        self.pow2_margin = np.float32(2.0 ** margin)
        self.state = np.zeros(hist_len + 4, dtype=np.float32)
        self.idx = 0

    # views into the packed state
    @property
    def hist(self) -> np.ndarray:
        return self.state[: self.n]

    @property
    def scale(self) -> np.float32:
        return self.state[self.n]

    @property
    def scale_used(self) -> np.float32:
        return self.state[self.n + 1]

    def seed(self, x) -> None:
        """First use: ``hist[idx] = amax(x)``, then publish the formula over the window."""
        self.state[self.idx] = amax_of(x)
        self.state[self.n] = scale_from_peak(np.max(self.hist), self.fp8_max, self.pow2_margin)

    def fold(self, measured_amax, step_used) -> None:
        """The quantize kernel's last-block fold: record, reduce, publish, clean."""
        self.state[self.n + 1] = np.float32(step_used)
        self.state[self.idx] = np.float32(measured_amax)
        peak = np.float32(np.fmax.reduce(self.hist))
        self.state[self.n] = scale_from_peak(peak, self.fp8_max, self.pow2_margin)
        self.state[self.n + 2] = 0.0
        self.state[self.n + 3] = 0.0

    def advance(self) -> None:
        """Host-side rotation to the next history slot."""
        self.idx = (self.idx + 1) % self.n
