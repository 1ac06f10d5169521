"""Software FP8 (E4M3FN, E5M2) and bf16 codecs, written from the format definitions.

Test infrastructure only (see ``oracle/__init__.py``).

Formats.  The AstrAI pages fix the two formats and their maxima: E4M3 for the
forward operands (max 448) and E5M2 for gradients (max 57344)
(compare view, ``astrai/extension/fp8.py``: ``FP8_MAX``; ``csrc/kernels/fp8/common.h``:
``enum class FP8Format`` and ``kFp8Max``).  The bit layouts are the OCP FP8 ones
that those maxima imply:

* E4M3FN: 1 sign, 4 exponent (bias 7), 3 mantissa bits; no infinities; only
  ``S.1111.111`` is NaN, so the largest finite code ``0.1111.110`` = 448.
* E5M2: 1 sign, 5 exponent (bias 15), 2 mantissa bits; IEEE-like: exponent
  all-ones with mantissa 0 is +-inf, other mantissas NaN; max ``0.11110.11`` = 57344.

Encoding.  The quantize kernels convert with round-to-nearest-even and
saturation to the finite range (compare view, ``quantize.cuh``: the fp8x2
conversion with ``__NV_SATFINITE``).  Readings taken where the pages are silent:

* ``|v| >= FP8_MAX`` (including +-inf) encodes as +-FP8_MAX.
* NaN encodes as the positive canonical NaN byte 0x7F -- parity unpinned: the
  pages fix no NaN byte and no workload here contains NaN, so the GPU tests only
  check that the device writes some NaN code for a NaN input.
* The sign of zero is kept (a negative value that rounds to zero gives 0x80).
"""

from __future__ import annotations

import numpy as np

# (exponent bits, mantissa bits, bias, finite max) per format.
FORMATS = {
    "e4m3": (4, 3, 7, 448.0),
    "e5m2": (5, 2, 15, 57344.0),
}

FP8_MAX = {name: spec[3] for name, spec in FORMATS.items()}


def _fmt_name(fmt) -> str:
    if fmt in (0, "e4m3"):
        return "e4m3"
    if fmt in (1, "e5m2"):
        return "e5m2"
    raise ValueError(f"unknown fp8 format {fmt!r}")


def decode_code(code: int, fmt) -> float:
    """Value of one fp8 byte, from the sign / exponent / mantissa fields."""
    fmt = _fmt_name(fmt)
    ebits, mbits, bias, _ = FORMATS[fmt]
    sign = -1.0 if (code >> 7) & 1 else 1.0
    e = (code >> mbits) & ((1 << ebits) - 1)
    m = code & ((1 << mbits) - 1)
    e_all_ones = (1 << ebits) - 1
    if fmt == "e4m3" and e == e_all_ones and m == (1 << mbits) - 1:
        return float("nan")
    if fmt == "e5m2" and e == e_all_ones:
        return sign * float("inf") if m == 0 else float("nan")
    if e == 0:  # subnormal: 0.m * 2^(1-bias)
        return sign * (m / (1 << mbits)) * 2.0 ** (1 - bias)
    return sign * (1.0 + m / (1 << mbits)) * 2.0 ** (e - bias)


def decode_table(fmt) -> np.ndarray:
    """float64[256]: value of every byte code."""
    return np.array([decode_code(c, fmt) for c in range(256)], dtype=np.float64)


_TABLES = {name: decode_table(name) for name in FORMATS}


def max_code(fmt) -> int:
    """The largest finite positive code (0x7E for E4M3, 0x7B for E5M2)."""
    tab = _TABLES[_fmt_name(fmt)]
    fin = [c for c in range(128) if np.isfinite(tab[c])]
    return max(fin)


def decode(codes: np.ndarray, fmt) -> np.ndarray:
    """Decode an array of uint8 codes to float64."""
    return _TABLES[_fmt_name(fmt)][np.asarray(codes, dtype=np.uint8)]


def encode(v: np.ndarray, fmt) -> np.ndarray:
    """Round-to-nearest-even encode with saturation; input is converted to fp64
    exactly (it is fp32 in every use), output uint8 of the same shape."""
    fmt = _fmt_name(fmt)
    v = np.asarray(v, dtype=np.float64)
    tab = _TABLES[fmt]
    top = max_code(fmt)
    pos = tab[: top + 1]  # codes 0..top: non-negative finite values, ascending
    assert np.all(np.diff(pos) > 0)

    a = np.abs(v)
    nan = np.isnan(v)
    a_safe = np.where(nan, 0.0, a)
    sat = a_safe >= pos[-1]
    # first code whose value is >= a
    hi = np.searchsorted(pos, np.minimum(a_safe, pos[-1]), side="left")
    lo = np.maximum(hi - 1, 0)
    exact = pos[hi] == a_safe
    mid = (pos[lo] + pos[hi]) / 2.0  # exact in fp64: both are short dyadics
    pick_lo = a_safe < mid
    pick_hi = a_safe > mid
    tie = ~(pick_lo | pick_hi)
    even = np.where(lo % 2 == 0, lo, hi)
    code = np.where(pick_lo, lo, np.where(pick_hi, hi, even))
    code = np.where(exact, hi, code)
    code = np.where(sat, top, code)
    del tie
    code = code.astype(np.int64)
    neg = np.signbit(v) & ~nan
    code = np.where(neg, code | 0x80, code)
    code = np.where(nan, 0x7F, code)
    return code.astype(np.uint8)


# ---------------------------------------------------------------------------
# bf16: the top 16 bits of an IEEE binary32 (8 exponent, 7 mantissa bits).
# ---------------------------------------------------------------------------

def bf16_bits_to_f64(bits: np.ndarray) -> np.ndarray:
    """Decode bf16 bit patterns (uint16) to float64 (exact)."""
    b = np.asarray(bits, dtype=np.uint16).astype(np.uint32) << 16
    return b.view(np.float32).astype(np.float64)


def f64_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round float64 values to bf16 (round-to-nearest-even, one rounding from
    the exact value), returning uint16 bit patterns.  Overflow gives +-inf."""
    x = np.asarray(x, dtype=np.float64)
    out = np.zeros(x.shape, dtype=np.float64)
    finite = np.isfinite(x) & (x != 0)
    xf = np.where(finite, x, 1.0)
    _, e = np.frexp(np.abs(xf))  # |x| = f * 2^e, f in [0.5, 1)
    # bf16 keeps 8 significant bits; the quantum is 2^(e-8), floored at the
    # subnormal quantum 2^-133.
    q_exp = np.maximum(e - 8, -133)
    r = np.rint(np.ldexp(xf, -q_exp))  # rint rounds half to even
    y = np.ldexp(r, q_exp)
    bf16_max = float(np.ldexp(np.float64(0xFF), 127 - 7))  # (2 - 2^-7) * 2^127
    y = np.where(np.abs(y) > bf16_max, np.sign(y) * np.inf, y)
    out = np.where(finite, y, x)
    f32 = out.astype(np.float32)  # exact: every bf16 value is an fp32 value
    return (f32.view(np.uint32) >> 16).astype(np.uint16)


def round_to_bf16(x: np.ndarray) -> np.ndarray:
    """float64 -> nearest bf16 value, returned as float64."""
    return bf16_bits_to_f64(f64_to_bf16_bits(x))
